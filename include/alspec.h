/*
 * alspec.h -- C ABI of the speculative flash-decode library (libalspec.so).
 *
 * The operation (Attention-Level Speculation, ICML 2025; atlas.scime.ai
 * summary, one-line summary and "Approach"; ICML 2025 poster page,
 * abstract): for each decode query, the library computes
 *   - O_spec : softmax attention over the "attention sink", i.e. the first
 *              n_sink tokens plus the last `window` tokens of the cache
 *              (a set union, each token once), published early;
 *   - O_exact: softmax attention over every cached token (flash decoding,
 *              the method the summary lists under "Builds on");
 *   - rel_l2 : ||O_exact - O_spec||_2 / ||O_exact||_2 per decode token, over
 *              all n_q_heads * head_dim outputs of that token's attention op;
 *   - commit : 1 when rel_l2 <= lambda (the approximation is kept), else 0
 *              (it is discarded and the exact output is used).
 * The softmax scale is 1/sqrt(head_dim).  Query head h reads KV head
 * h / (n_q_heads / n_kv_heads) (grouped-query attention).
 *
 * Conventions for every entry point:
 *   - Pointers named "device" are CUDA device pointers; "host" pointers are
 *     ordinary host memory.  The caller owns every buffer.  The library never
 *     allocates device memory in alspec_decode; it owns only a
 *     lowest-priority stream and two events per device, created on first
 *     use and released by alspec_shutdown().
 *   - Streams and events are passed as `void*` holding a cudaStream_t /
 *     cudaEvent_t (NULL stream = the legacy default stream).
 *   - Calls are asynchronous on the given stream unless stated otherwise;
 *     no entry point except alspec_get_device_error synchronizes.
 *   - Arguments that can be checked on the host are checked before anything
 *     is launched; a failed check returns a status and launches nothing.
 *     Nothing aborts, traps or exits.
 *   - Calls may come from several host threads: each call enqueues its work
 *     on the library's shared streams under a per-device lock.  While one
 *     thread captures calls into a graph, no other thread may issue calls on
 *     the same device (the shared streams join that capture).
 */
#ifndef ALSPEC_H
#define ALSPEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ALSPEC_OK = 0,
    ALSPEC_ERR_INVALID_ARG = 1,  /* bad pointer, shape, alignment or value   */
    ALSPEC_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, group size */
    ALSPEC_ERR_WORKSPACE = 3,    /* workspace missing or too small            */
    ALSPEC_ERR_CUDA = 4,         /* a CUDA runtime call failed                */
    ALSPEC_ERR_TIMEOUT = 5,      /* reported by alspec_get_device_error only  */
    ALSPEC_ERR_DEVICE_DATA = 6   /* reported by alspec_get_device_error only  */
} alspec_status;

typedef enum {
    ALSPEC_F32 = 0,   /* IEEE binary32                       */
    ALSPEC_BF16 = 1   /* bfloat16 (upper half of a binary32) */
} alspec_dtype;

/* Compute engine of the attention kernels (alspec_desc.engine). */
typedef enum {
    ALSPEC_ENGINE_AUTO = 0,          /* tensor cores for bf16, CUDA cores for fp32 */
    ALSPEC_ENGINE_CUDA_CORES = 1,    /* packed fp32 FMAs; any dtype               */
    ALSPEC_ENGINE_TENSOR_CORES = 2   /* bf16 m16n8k16 MMAs; bf16 only             */
} alspec_engine;

/*
 * Launch schedule of one decode call (alspec_desc.schedule).
 *   STREAMS: three kernels in order on the caller's stream: the sink-set
 *            kernel (at high launch priority; O_spec early), the exact-path
 *            kernel and a merge kernel that also writes rel_l2 and the flags.
 *            Each launch is released as soon as every CTA of the one before
 *            it has started, so the exact-path kernel (persistent, one CTA
 *            per SM) runs beside the sink-set kernel on the SMs it leaves and
 *            takes over each SM it frees.  When the caller asks for
 *            spec_event (or the speculative projection), the library's
 *            lowest-priority stream waits for the sink-set kernel (an event
 *            recorded right behind it), records spec_event there (and runs
 *            the projection), and the caller's stream joins it at the end.
 *            Inside a CUDA graph that event record is only a dependency, so
 *            the kernels keep their overlap; outside one, the exact-path
 *            kernel may then start only once the sink-set kernel completed.
 *   FUSED:   one persistent launch on the caller's stream.  The sink-set
 *            work items come first in the same work queue as the exact
 *            path's; the CTA that completes a (sequence, KV head) writes its
 *            O_spec and O_exact, and the CTA that completes a sequence
 *            writes rel_l2 and the flag (ticket counters in the workspace).
 *            O_spec is complete only when the launch ends (spec_event marks
 *            that point); alspec_decode_oproj is not available with it.
 *   SINK_FIRST: as STREAMS, but the exact-path kernel starts only once the
 *            sink-set kernel has completed, which then has every SM: O_spec
 *            sooner when the sink set is large (many sequences or a long
 *            window), at some cost in throughput.
 */
typedef enum {
    ALSPEC_SCHEDULE_AUTO = 0,     /* STREAMS; the sink-set kernel may take every SM (rather
                                     than 3/4 of them) when a CTA would otherwise get more
                                     than 24 tiles of 32 rows, so O_spec stays early */
    ALSPEC_SCHEDULE_STREAMS = 1,
    ALSPEC_SCHEDULE_FUSED = 2,
    ALSPEC_SCHEDULE_SINK_FIRST = 3
} alspec_schedule;

/* Gating of the recomputation in alspec_decode_oproj. */
typedef enum {
    ALSPEC_GATE_KERNEL = 0,             /* a kernel that reads the flags           */
    ALSPEC_GATE_GRAPH_CONDITIONAL = 1   /* a CUDA-graph IF node (inside a capture) */
} alspec_gate;

/* Number of events alspec_decode's prof_events array holds. */
#define ALSPEC_PROF_EVENTS 5

/* Bits of the device error word (alspec_get_device_error). */
#define ALSPEC_DEVERR_SEQ_LEN 0x1u   /* a seq_lens entry outside [1, max_seq_len]; it was clamped */
#define ALSPEC_DEVERR_TIMEOUT 0x2u   /* a bounded wait inside a kernel gave up; outputs invalid   */
/* Only in the bounds-checked debug build of this library (libalspec_debug.so,
 * the same sources compiled with ALSPEC_DEBUG_BOUNDS): a kernel found an
 * index outside its buffer (shared-memory slot, chunk list, partial slot,
 * copy source or output) and skipped that access; outputs invalid. */
#define ALSPEC_DEVERR_BOUNDS 0x4u

/*
 * Problem description.  Shapes (row-major, last index fastest):
 *   q                    [batch, n_q_heads, head_dim]
 *   k_cache, v_cache     [batch, n_kv_heads, max_seq_len, head_dim]
 * q, k_cache and v_cache share `dtype`.  Supported: head_dim in {64, 128};
 * n_q_heads / n_kv_heads in {1, 2, 4, 8}.
 * batch * n_kv_heads * max_seq_len must stay below 2^31.
 * split_tokens: tokens per work item of the exact-attention split of the
 * longest sequence (rounded up to the engine's tile, 16 or 32 tokens;
 * shorter sequences get proportionally shorter items); 0 lets the library
 * choose (guided self-scheduling: items shrink towards the end of the
 * queue; at most 256 items per sequence and KV head).
 */
typedef struct {
    int batch;
    int n_q_heads;
    int n_kv_heads;
    int head_dim;
    int max_seq_len;
    int dtype;          /* alspec_dtype */
    int split_tokens;   /* 0 = automatic */
    int timeout_ms;     /* bound on any in-kernel wait; 0 = 2000 ms */
    int engine;         /* alspec_engine; 0 = automatic */
    int schedule;       /* alspec_schedule; 0 = automatic */
} alspec_desc;

/*
 * Bytes of device workspace alspec_decode needs for this description and
 * sink set.  Host only, no CUDA call.  Returns 0 if the description is
 * invalid or unsupported.
 */
size_t alspec_workspace_size(const alspec_desc* desc, int n_sink, int window);

/*
 * Zero a workspace before its first use (cudaMemsetAsync on `stream`).
 * The kernels leave every counter in the workspace at zero when they finish,
 * so a workspace needs this once, not per call.
 */
alspec_status alspec_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * One speculative decode-attention step (one layer, `batch` decode tokens).
 *
 *   desc        host; shapes as above
 *   q           device [batch, n_q_heads, head_dim], 16-byte aligned
 *   k_cache     device [batch, n_kv_heads, max_seq_len, head_dim], 16-byte aligned
 *   v_cache     device, same shape and alignment as k_cache
 *   seq_lens    device int32 [batch]; 1 <= L_b <= max_seq_len.  Sequence b
 *               attends to cache rows [0, L_b).  Out-of-range entries are
 *               clamped and flagged in the device error word.
 *   n_sink      S >= 0 sink tokens; window W >= 0 recent tokens; S + W >= 1
 *   lambda      relative-L2 threshold, finite and >= 0
 *   out_spec    device fp32 [batch, n_q_heads, head_dim]: O_spec
 *   out_exact   device fp32 [batch, n_q_heads, head_dim]: O_exact
 *   rel_l2      device fp32 [batch]
 *   commit      device uint8 [batch]: 1 commit, 0 discard
 *   workspace   device, >= alspec_workspace_size() bytes, zeroed once by
 *               alspec_workspace_init; one call at a time per workspace
 *   stream      the caller's stream; everything is ordered on it
 *   spec_event  optional cudaEvent_t (NULL for none).  It is recorded as
 *               soon as out_spec is complete, before the exact path ends,
 *               so a consumer may start work on O_spec early by waiting on
 *               it.  out_exact, rel_l2 and commit are complete when
 *               `stream` reaches the point of this call.
 *   prof_events optional array of ALSPEC_PROF_EVENTS timing-enabled
 *               cudaEvent_t (NULL for none), recorded with
 *               cudaEventRecordExternal so that they become event nodes when
 *               the call is captured in a graph:
 *                 [0] on `stream` when the call starts,
 *                 [1] on `stream` after the sink-set kernel (O_spec complete),
 *                 [2] on `stream` before the exact-path (middle) kernel,
 *                 [3] on `stream` after it,
 *                 [4] on `stream` when the call's work is complete.
 *               Events between the kernels take away their overlap: with
 *               them, the middle kernel starts once the sink-set kernel has
 *               completed, so [3]-[2] is the middle kernel's duration alone
 *               and [4]-[0] is longer than the step without events.
 *
 * Everything runs on `stream` (and, for spec_event, on the library's
 * lowest-priority stream, joined before the call's work is complete).
 * FUSED schedule: one launch on `stream`; spec_event and prof_events [1]-[3]
 * are recorded around it.  Safe to capture in a CUDA graph (no host
 * synchronization, no allocation).  With L_b <= S + W the two outputs are
 * bit-identical and rel_l2 is exactly 0.
 */
alspec_status alspec_decode(const alspec_desc* desc,
                            const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* seq_lens, int n_sink, int window,
                            float lambda, float* out_spec, float* out_exact,
                            float* rel_l2, uint8_t* commit,
                            void* workspace, size_t workspace_bytes,
                            void* stream, void* spec_event, void* const* prof_events);

/*
 * alspec_decode with publication time stamps measured by the kernels
 * themselves (no events), for timing inside CUDA graphs, where an event
 * record node does not mark when the work before it ended.
 *   trace_ns  device, 2 x uint64, 8-byte aligned, zeroed by the caller
 *             before the call.  The kernels raise (atomic max):
 *               [0] to the global timer (ns) after the last write of O_spec,
 *               [1] to the global timer after the last write of O_exact,
 *                   rel_l2 and commit.
 *             The library never reads or clears it; NULL is an
 *             ALSPEC_ERR_INVALID_ARG.
 * Other arguments as for alspec_decode (no spec event, no profiling events).
 * The stamps come from the same clock for all calls on a device, so
 * trace[0] of one call minus trace[1] of the call before it is the latency
 * of O_spec from the end of the previous step.
 */
alspec_status alspec_decode_traced(const alspec_desc* desc,
                                   const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* seq_lens, int n_sink, int window,
                                   float lambda, float* out_spec, float* out_exact,
                                   float* rel_l2, uint8_t* commit,
                                   void* workspace, size_t workspace_bytes,
                                   void* stream, unsigned long long* trace_ns);

/*
 * Output projection of attention outputs -- the linear map that follows
 * self-attention in a decoder layer (the post-attention op the pages run
 * speculatively, "Approach"):
 *     y[b, j] = sum_i x[b, i] * w[j, i]
 * on CUDA cores (decode batches are small: the op streams w once, with bulk
 * copies, two CTAs per SM).  The launch is programmatic: without `skip`, w
 * starts streaming before the kernel ahead of it on `stream` has completed
 * (x is read, and y written, only after it has), so w must not be written
 * by that kernel; with `skip`, nothing is read before it has completed.
 *   x     device fp32 [batch][k], 16-byte aligned
 *   w     device bf16 [n][k] (row j = output feature j), 16-byte aligned
 *   y     device fp32 [batch][n]
 *   skip  device uint8 [batch] or NULL: rows b with skip[b] != 0 are not
 *         written (pass the commit flags to redo only discarded tokens)
 *   err   device uint32 or NULL: ALSPEC_DEVERR_TIMEOUT is ORed in when one of
 *         the kernel's bounded waits (2 s) expires (y is then incomplete)
 *   batch 1..8; k a positive multiple of 8; n >= 1.
 * Asynchronous on `stream`; ALSPEC_ERR_INVALID_ARG for a bad argument.
 */
alspec_status alspec_oproj(const float* x, const void* w, float* y, const uint8_t* skip,
                           int batch, int k, int n, uint32_t* err, void* stream);

/*
 * alspec_decode followed by the output projection of the attention output,
 * run speculatively (the single-GPU form of the pages' speculative
 * post-attention ops with commit or discard, "Approach"):
 *   y[b] = o_proj(commit[b] ? O_spec[b] : O_exact[b]),  o_proj as in
 *   alspec_oproj with w_o bf16 [hidden][n_q_heads * head_dim].
 * The projection of O_spec runs right after the sink-set kernel, beside the
 * exact path, on the library's lowest-priority stream (a form without shared
 * memory, which shares SMs with the middle kernel).  After the merge, the
 * projection of O_exact (the bulk-copy form of alspec_oproj) overwrites the
 * rows of discarded tokens.  With every token committed, y is final when the
 * flags are, instead of one projection later.  Wait timeouts go to the
 * workspace's device error word.
 *   y        device fp32 [batch][hidden]; batch <= 8
 *   gate     how the recomputation is gated (alspec_gate):
 *            ALSPEC_GATE_KERNEL: it is always launched and reads the flags
 *            (it exits at once when every token committed);
 *            ALSPEC_GATE_GRAPH_CONDITIONAL: inside a stream capture it is an
 *            IF conditional node of the graph, enabled by a one-warp kernel
 *            after the merge when a token was discarded (outside a capture
 *            as GATE_KERNEL).
 *            Evaluating the conditional node was measured at ~7 us per layer
 *            on B200, more than the kernel launch it saves.
 *   trace_ns NULL, or device 3 x uint64 zeroed by the caller: [0] and [1] as
 *            in alspec_decode_traced, [2] raised to the global timer after
 *            each projection's last write (y is final at max([1], [2])).
 * out_spec and out_exact must be 16-byte aligned.  Other arguments as for
 * alspec_decode.
 */
alspec_status alspec_decode_oproj(const alspec_desc* desc,
                                  const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* seq_lens, int n_sink, int window,
                                  float lambda, const void* w_o, int hidden,
                                  float* out_spec, float* out_exact, float* rel_l2,
                                  uint8_t* commit, float* y, int gate,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream, unsigned long long* trace_ns);

/*
 * Test hook for failure detection: launches one CTA whose two bounded waits
 * (written like the attention kernels' producer and consumer waits) target
 * mbarriers that nothing ever arrives on.  The waits give up after
 * timeout_ms (1..10000), ALSPEC_DEVERR_TIMEOUT is ORed into the workspace's
 * device error word (read it with alspec_get_device_error), and the kernel
 * returns: no trap, no fault.  Asynchronous on `stream`.
 */
alspec_status alspec_test_wait_timeout(void* workspace, size_t workspace_bytes, int timeout_ms,
                                       void* stream);

/*
 * Work plan the library would use (host only, no CUDA call except the SM
 * count query).  info[] receives, in order:
 *   0 tokens per sink-set work item      1 sink-set items per (b, kv head)
 *   2 tokens in the first exact-path item of the longest sequence
 *   3 exact-path items per (b, kv head)
 *   4 persistent CTAs of the exact path  5 threads per CTA
 *   6 dynamic shared memory per CTA      7 pipeline stages
 *   8 engine (alspec_engine, resolved)
 *   9 schedule (alspec_schedule, resolved)
 *  10 CTAs per sequence (one thread-block cluster) of the merge kernel, or
 *     0 when the merge runs as one CTA per 32 output columns (a CTA's share
 *     of the middle partials does not fit in shared memory; and the FUSED
 *     schedule, which merges inside its one kernel)
 *  11 CTAs of the sink-set kernel (batch * n_kv_heads * entry 1; none with
 *     the FUSED schedule's one kernel, which queues those items)
 * (entries 4-7 describe the exact-path kernel, or with the FUSED schedule
 * the one kernel, whose queue holds both kinds of items).  n_info is the
 * capacity of info (12 fills all).
 */
alspec_status alspec_query_plan(const alspec_desc* desc, int n_sink, int window,
                                int* info, int n_info);

/*
 * Chunk table of the exact-path (middle) split (host only).  The middle of
 * sequence b -- rows [min(S, L_b), max(min(S, L_b), L_b - W)) -- is tiled in
 * T-row tiles (T = 32 for the tensor-core engine, 16 for the CUDA-core
 * engine; *tile receives T); with m_b tiles in it, chunk c covers tiles
 * [(m_b * fq[c]) >> 24, (m_b * fq[c + 1]) >> 24).  fq receives n2 + 1
 * entries (fq[0] = 0, fq[n2] = 1 << 24); capacity is the length of fq.
 * *n2 receives the chunk count.
 */
alspec_status alspec_query_chunks(const alspec_desc* desc, int n_sink, int window,
                                  uint32_t* fq, int capacity, int* n2, int* tile);

/*
 * Read (and clear) the device error word of a workspace: a bitwise OR of
 * ALSPEC_DEVERR_* raised by kernels since the last read.  Synchronizes
 * `stream`.  *err receives the word; returns ALSPEC_OK, or
 * ALSPEC_ERR_DEVICE_DATA / ALSPEC_ERR_TIMEOUT when the word is non-zero.
 */
alspec_status alspec_get_device_error(void* workspace, size_t workspace_bytes,
                                      void* stream, uint32_t* err);

/*
 * Static-graph helpers (the single-GPU analogue of the pages' static-graph
 * runtime with priority gating): capture a sequence of alspec_decode calls
 * on `stream` into a CUDA graph whose sink-set kernels keep their high
 * launch priority.  begin/end bracket the capture; launch replays it on a
 * stream; destroy frees it.  *graph receives an opaque handle.
 */
alspec_status alspec_graph_begin(void* stream);
alspec_status alspec_graph_end(void* stream, void** graph);
alspec_status alspec_graph_launch(void* graph, void* stream);
alspec_status alspec_graph_destroy(void* graph);

/* Release the library's streams and events on every device it touched. */
alspec_status alspec_shutdown(void);

/* Human-readable name of a status (static string, never NULL). */
const char* alspec_status_string(alspec_status status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int alspec_version(void);

/*
 * The cudaError_t of the most recent CUDA runtime call that failed inside
 * this library on the calling thread (0 if none did); it explains an
 * ALSPEC_ERR_CUDA status.
 */
int alspec_last_cuda_error(void);

/*
 * Allocation-free variant of alspec_decode (the paper has no counterpart;
 * this is a deployment convenience).  Some callers cannot allocate device
 * memory at all -- for example code running inside a host framework that
 * owns every allocation, or a callback that must not call cudaMalloc -- and
 * so cannot provide the workspace alspec_decode needs.  This entry point
 * takes the same inputs and outputs but no workspace: its scratch space is
 * a fixed array of ALSPEC_NOALLOC_SCRATCH_BYTES (8 MiB) in the library's
 * own device memory, which every GPU that loads the library holds until the
 * process exits.  It never calls cudaMalloc or cudaFree.
 *
 *   - A problem whose workspace (alspec_workspace_size) is larger than
 *     ALSPEC_NOALLOC_SCRATCH_BYTES is rejected with ALSPEC_ERR_WORKSPACE
 *     before anything is launched.  Every other argument is checked as by
 *     alspec_decode, also before anything is queued: a rejected call leaves
 *     the array untouched.
 *   - The first call on a device looks up the device address of the array
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     outside any stream capture.  The address is kept until
 *     alspec_shutdown, which must precede a cudaDeviceReset.
 *   - Each call clears the array's counters on `stream`, then runs exactly
 *     what alspec_decode runs.  All calls on a device share the one array:
 *     calls that overlap on the GPU (different streams without ordering
 *     between them) race and corrupt each other's results.  Calls ordered
 *     on one stream are fine.
 *   - There is no spec_event and no profiling events.  The device error
 *     word of the array (a clamped seq_lens entry, an in-kernel wait that
 *     gave up) is read with alspec_noalloc_device_error.
 */
#define ALSPEC_NOALLOC_SCRATCH_BYTES (8u << 20)
alspec_status alspec_decode_noalloc(const alspec_desc* desc,
                                    const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* seq_lens, int n_sink, int window,
                                    float lambda, float* out_spec, float* out_exact,
                                    float* rel_l2, uint8_t* commit, void* stream);

/*
 * Read (and clear) the device error word of alspec_decode_noalloc's scratch
 * array on the current device, as alspec_get_device_error does for a
 * workspace: synchronizes `stream`; *err (host) receives the bitwise OR of
 * ALSPEC_DEVERR_* raised since the last read.  Returns ALSPEC_OK, or
 * ALSPEC_ERR_DEVICE_DATA / ALSPEC_ERR_TIMEOUT when the word is non-zero,
 * ALSPEC_ERR_INVALID_ARG for a NULL err.  Allocates nothing.
 */
alspec_status alspec_noalloc_device_error(void* stream, uint32_t* err);

#ifdef __cplusplus
}
#endif

#endif /* ALSPEC_H */
