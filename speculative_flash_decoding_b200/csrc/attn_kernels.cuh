// Speculative flash-decode kernels for sm_100a.
//
// Operation (Attention-Level Speculation, ICML 2025; atlas.scime.ai summary,
// "Approach"): each decode query gets softmax attention over the attention
// sink (first S tokens plus the last W tokens) -- O_spec -- and over the whole
// cache -- O_exact, the latter by flash decoding ("Builds on" on the same
// page); the relative L2 distance of the two decides commit or discard.
//
// Work is split the flash-decoding way: every sequence's token list is cut
// into items; each item yields a partial (m, l, o) -- running max of the
// log2-domain scores, sum of exponentials, and the unnormalised weighted sum
// of value rows -- and partials are merged with the log-sum-exp rule.  The
// sink-set tokens and the middle tokens are separate item lists, so both
// outputs come from one read of every cache row:
//   * the sink-set kernel (SPEC) reads only the S + W tokens; the CTAs of one
//     (sequence, KV head) form a thread-block cluster, each streams a slice
//     of the sink set, and they merge their partials through distributed
//     shared memory and write O_spec;
//   * the middle kernel (MID) is persistent: CTAs pull items from an atomic
//     queue and stream the cache through shared memory;
//   * the merge kernel, after both, combines the sink-set partial with the
//     middle partials into O_exact (one CTA per 32 output columns of a query
//     head, its warps over interleaved chunks), and the CTA finishing a
//     sequence's last slot computes rel_l2 and the commit flag;
//   * the one-launch variant (FUSED) is the middle kernel with the sink-set
//     items at the head of its queue and the merges done in the kernel, by
//     the CTA whose tile ticket completes a (sequence, KV head).
//
// Inside a CTA one producer lane fills a ring of shared-memory stages with
// K and V tiles through the TMA engine (mbarrier completion); consumer warps
// compute.  Tile t of a CTA goes to consumer warp t mod (warps) ("token
// slot") and every item is padded to a multiple of the slot count; each
// stage carries a fill ticket naming the tile it holds.  At the end of an
// item the warps' states are merged through shared memory and one partial
// per query head is written.
//
// Two compute engines share that pipeline:
//   * tensor cores (bf16 caches): 32-token tiles loaded as 2-D TMA boxes
//     with 128-byte swizzle.  S^T = Q K^T and O += P V run as m16n8k16 MMAs
//     (fp32 accumulation): the query heads of a KV group are the 16 rows of
//     the A operand (rows 8..15 zero), K and V fragments come from ldmatrix,
//     and the score fragment is reused as the A operand of P V.  P is split
//     into a bf16 high part (rows 0..7) and the bf16 rounding residual
//     (rows 8..15), so P V keeps ~16 bits of P instead of 8;
//   * CUDA cores (fp32 caches, and bf16 on request): 16-token tiles loaded by
//     1-D bulk copies; 8 lanes per token row with packed fp32x2 FMAs and a
//     reduce-scatter of the partial dot products.
//
// Every wait is bounded (global nanosecond timer); on expiry the kernel sets
// an error bit, stops issuing copies, drains the ones in flight and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace alspec {

constexpr int kSmemLimit = 227 * 1024;
// Sink-set CTAs per (sequence, KV head) at most: one portable cluster.
constexpr int kMaxSpecCtas = 8;

// Sink-set tokens per CTA, in tensor-core tiles of 32 (the planner's target),
// and the consumer warps of the tensor-core sink-set kernel.
#ifndef ALSPEC_SPEC_TILES
#define ALSPEC_SPEC_TILES 5
#endif
#ifndef ALSPEC_SPEC_WARPS
#define ALSPEC_SPEC_WARPS 5
#endif

// Stages of the tensor-core middle kernel's ring: 12 stages of 16 KB keep
// up to 192 KB in flight per SM, so the producer keeps streaming through the
// few microseconds an item's end takes.  A 13th stage fits beside the
// item-end deposit (the stages' fill tickets keep any count sound, see
// Cfg::STAGES) but measured no faster on the 128K step.
#ifndef ALSPEC_MID_STAGES
#define ALSPEC_MID_STAGES 12
#endif
#ifndef ALSPEC_MID_SPW
#define ALSPEC_MID_SPW 3
#endif

constexpr unsigned kErrSeqLen = 1u;   // ALSPEC_DEVERR_SEQ_LEN
constexpr unsigned kErrTimeout = 2u;  // ALSPEC_DEVERR_TIMEOUT
constexpr unsigned kErrBounds = 4u;   // ALSPEC_DEVERR_BOUNDS (debug build)

// Counter words at the head of the workspace, then the per-sequence
// tickets [B] (merge kernel: one per CTA of the sequence; one-launch
// schedule: one per KV head), and for the one-launch schedule the per-head
// tile tickets [B * Hkv].  Whoever takes the last ticket of a group resets
// it, so the words are zero between calls.
constexpr int kCtrQueue = 0;
constexpr int kCtrDone = 1;
constexpr int kCtrError = 2;
constexpr int kCtrFixed = 4;

__host__ __device__ __forceinline__ int ctr_seq(int B, int Hkv, int b) {
    (void)Hkv;
    return kCtrFixed + b;
}
__host__ __device__ __forceinline__ int ctr_head(int B, int Hkv, int bh) {
    (void)Hkv;
    return kCtrFixed + B + bh;
}
__host__ __device__ __forceinline__ int ctr_words(int B, int Hkv) {
    return kCtrFixed + B + B * Hkv;
}

// Stage metadata word w: bit 0 marks a consumer warp's last tile of the
// item; in the one-launch schedule bits 1.. hold the item's tile count (its
// tickets count tiles).
constexpr int kLastTileFlag = 1;

// Middle work items: every (sequence, KV head) middle is cut at fixed
// fractions of its length into at most kMaxChunks chunks (guided
// self-scheduling: large chunks first, shrinking towards the end, so the
// queue drains on small items and the CTAs finish together).
constexpr int kMaxChunks = 256;
constexpr int kFracBits = 24;
// One-launch schedule: sink-set items per (sequence, KV head) at most.
constexpr int kMaxSpecItemsFused = 64;

struct Params {
    CUtensorMap tmap_k;  // 2-D views [rows = B*Hkv*Lmax, d] (tensor-core engine)
    CUtensorMap tmap_v;
    const void* q;
    const void* k;
    const void* v;
    const int* seq_lens;
    int B, Hq, Hkv, Lmax, S, W;
    float qscale;   // log2(e) / sqrt(d): scores come out in the log2 domain
    float lambda;
    int c1, n1;     // sink-set items: tokens per item, items per (b, kv head) (the
                    // sink-set kernel: CTAs of one cluster)
    int n2;         // middle chunks per (b, kv head)
    int mid_ctas;   // CTAs of the middle (or one-launch) kernel's launches together
    unsigned fq[kMaxChunks + 1];  // chunk c covers middle tiles
                                  // [mt * fq[c] >> 24, mt * fq[c+1] >> 24)
    unsigned* ctr;
    float* spec_ml;   // [B][Hq][2]       merged sink-set partial
    float* spec_pml;  // [B][Hq][n1][2]   sink-set item partials (one-launch schedule)
    float* spec_po;   // [B][Hq][n1][D]
    float* spec_o;    // [B][Hq][D]
    float* mid_ml;    // [B][Hq][n2][2]   middle item partials
    float* mid_o;     // [B][Hq][n2][D]
    float* dn;        // [B][Hq][2]       per-head squared distance / norm
    float* out_spec;
    float* out_exact;
    float* rel_l2;
    uint8_t* commit;
    unsigned long long timeout_ns;
    unsigned long long* trace;  // optional: [0] O_spec, [1] O_exact published (ns)
};

// Optional publication time stamps: after this thread's writes (and those
// ordered before them), raise trace[which] to the global timer.  The last
// writer of a result leaves its time there.
__device__ __forceinline__ void trace_publish(const Params& p, int which) {
    if (p.trace) {
        __threadfence();
        atomicMax(p.trace + which, (unsigned long long)global_ns());
    }
}

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// Bounds checks of the debug build (compiled with ALSPEC_DEBUG_BOUNDS): an
// index outside its buffer ORs kErrBounds into the workspace's error word
// and the caller skips the access (never a trap).  In the normal build
// every check is the constant true and its condition is not evaluated.
#ifdef ALSPEC_DEBUG_BOUNDS
__device__ __noinline__ bool bounds_fail(unsigned* ctr) {
    atomicOr(ctr + kCtrError, kErrBounds);
    return false;
}
#define ALSPEC_IN_BOUNDS(p, cond) ((cond) ? true : ::alspec::bounds_fail((p).ctr))
#else
#define ALSPEC_IN_BOUNDS(p, cond) true
#endif

// Token geometry of one sequence: sink tokens [0, ns), window [ws, L),
// middle [ns, ws).
struct SeqGeom {
    int L, ns, ws, mid_len;
};

__host__ __device__ __forceinline__ SeqGeom geom_of(int L, int S, int W) {
    SeqGeom g;
    g.L = L;
    g.ns = L < S ? L : S;
    const int w0 = L - W;
    g.ws = w0 > g.ns ? w0 : g.ns;
    g.mid_len = g.ws - g.ns;
    return g;
}

// Geometry of a sequence of stored length L; out-of-range lengths are
// clamped (and flagged).
__device__ __forceinline__ SeqGeom seq_geom_of_len(const Params& p, int L, bool flag) {
    if (L < 1 || L > p.Lmax) {
        if (flag) atomicOr(p.ctr + kCtrError, kErrSeqLen);
        L = L < 1 ? 1 : p.Lmax;
    }
    return geom_of(L, p.S, p.W);
}

// Reads seq_lens[b].
__device__ __forceinline__ SeqGeom seq_geom(const Params& p, int b, bool flag) {
    return seq_geom_of_len(p, __ldg(p.seq_lens + b), flag);
}

// Tiles of the sink-set list: the sink run and the window run are tiled
// separately, so every tile is one contiguous run of cache rows.
__host__ __device__ __forceinline__ int spec_tiles(const SeqGeom& g, int TT) {
    return cdiv(g.ns, TT) + cdiv(g.L - g.ws, TT);
}

// Middle tiles [t_lo, t_hi) of chunk c, for a middle of mid_tiles tiles.
__device__ __forceinline__ void mid_chunk(const Params& p, int mid_tiles, int c, int& t_lo,
                                          int& t_hi) {
    t_lo = (int)(((unsigned long long)mid_tiles * p.fq[c]) >> kFracBits);
    t_hi = (int)(((unsigned long long)mid_tiles * p.fq[c + 1]) >> kFracBits);
}

// One work item: a range of tiles of one (sequence, KV head).
struct Item {
    int b, kvh, chunk, ntiles;
    int t0, ns, ws, L;  // sink-set items
    int lo, hi;         // middle items
    bool spec;          // a sink-set item
};

// Which (sequence, KV head) and chunk a queue index names.  Sink-set items
// of one head are consecutive (one cluster); middle items are chunk-major
// across heads.  The one-launch schedule (FUSED) numbers the sink-set items
// first, then the middle items.
template <bool SPEC, bool FUSED>
__device__ __forceinline__ void item_index(const Params& p, int item, bool& spec, int& bh,
                                           int& chunk) {
    const int heads = p.B * p.Hkv;
    const int n_spec = FUSED ? heads * p.n1 : 0;
    spec = SPEC || (FUSED && item < n_spec);
    if (FUSED && !spec) item -= n_spec;
    bh = spec ? item / p.n1 : item % heads;
    chunk = spec ? item % p.n1 : item / heads;
}

// `lane_len`: with a full warp calling, lane i may hold seq_lens[i] already
// (loaded beforehand, for i < min(B, 32)); -1 to read the length here.
template <bool SPEC, int TT, bool FUSED = false>
__device__ __forceinline__ Item decode_item(const Params& p, int item, bool flag,
                                            int lane_len = -1) {
    Item it;
    int bh;
    item_index<SPEC, FUSED>(p, item, it.spec, bh, it.chunk);
    it.b = bh / p.Hkv;
    it.kvh = bh % p.Hkv;
    int L;
    if (lane_len >= 0 && it.b < 32) {
        L = __shfl_sync(0xffffffffu, lane_len, it.b);  // the warp agrees on it.b
    } else {
        L = __ldg(p.seq_lens + it.b);
    }
    const SeqGeom g = seq_geom_of_len(p, L, flag);
    it.ns = g.ns;
    it.ws = g.ws;
    it.L = g.L;
    if (SPEC || (FUSED && it.spec)) {
        const int per = p.c1 / TT;
        it.t0 = it.chunk * per;
        const int t1 = min(it.t0 + per, spec_tiles(g, TT));
        it.ntiles = max(0, t1 - it.t0);
        it.lo = it.hi = 0;
    } else {
        int tlo, thi;
        mid_chunk(p, cdiv(g.mid_len, TT), it.chunk, tlo, thi);
        it.lo = g.ns + tlo * TT;
        it.hi = min(g.ns + thi * TT, g.ws);
        it.ntiles = thi > tlo ? thi - tlo : 0;
        it.t0 = 0;
    }
    return it;
}

// First cache row (within the head) and valid row count of tile t.
template <bool SPEC, int TT, bool FUSED = false>
__device__ __forceinline__ void tile_rows(const Item& it, int t, int& start, int& nvalid) {
    if (SPEC || (FUSED && it.spec)) {
        const int tg = it.t0 + t;
        const int tsink = cdiv(it.ns, TT);
        if (tg < tsink) {
            start = tg * TT;
            nvalid = min(TT, it.ns - start);
        } else {
            start = it.ws + (tg - tsink) * TT;
            nvalid = min(TT, it.L - start);
        }
    } else {
        start = it.lo + t * TT;
        nvalid = min(TT, it.hi - start);
    }
}

// ------------------------------------------------------------ element types

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kPairs = 2;  // float2 pairs per 16-byte chunk
    __device__ __forceinline__ static void unpack(const uint4& r, float2 (&o)[2]) {
        o[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
        o[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
    }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPairs = 4;
    // bf16 is the upper half of a binary32: widen by moving each half up.
    __device__ __forceinline__ static float2 widen(uint32_t w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    __device__ __forceinline__ static void unpack(const uint4& r, float2 (&o)[4]) {
        o[0] = widen(r.x);
        o[1] = widen(r.y);
        o[2] = widen(r.z);
        o[3] = widen(r.w);
    }
};

// ------------------------------------------------------------ configuration

// Pipeline shape shared by both engines.
//   TT    tokens per stage            GW   heads a consumer warp holds
//   NHW   warps sharing a stage       NTW  token slots (stages per round)
//   SPW   stages per token slot
template <typename T, int D, int G, bool SPEC, bool MMA, bool FUSED = false>
struct Cfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int TT = MMA ? 32 : 16;
    static constexpr int GW = MMA ? G : (G < 4 ? G : 4);
    static constexpr int NHW = G / GW;
    // CUDA-core engine: warps are spread over the SM's four sub-partitions
    // with 16K registers each; 8 warps per CTA allow 255 registers a thread,
    // 9 only 168.  Holding 4 heads x 16 elements of q and o per lane needs
    // the former, so those configurations run 7 consumer warps.
    static constexpr int kLanePairs = (kRowBytes / 128) * Elem<T>::kPairs;
    static constexpr bool kHeavy = !MMA && GW * kLanePairs >= 32;
    // Tensor-core engine: 4 consumer warps stream the middle; the sink-set
    // kernel (latency-bound, a few tiles per CTA) uses one warp per tile.
    static constexpr int NTW = MMA ? (SPEC ? ALSPEC_SPEC_WARPS : 4) : (kHeavy ? 7 : 8) / NHW;
    static constexpr int NCW = NTW * NHW;
    static constexpr int kThreads = (NCW + 1) * 32;
    static constexpr int kTileBytes = TT * kRowBytes;  // K or V part of a stage
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kSlotFloats = GW * (D + 2);
    static constexpr int kDepositBytes = NCW * kSlotFloats * 4;
    static constexpr int kSpwMax = SPEC ? 3 : (MMA ? ALSPEC_MID_SPW : 4);
    // Sink-set kernel: every CTA of a cluster gathers one partial (m, l, o
    // for the G heads) per CTA of the cluster, in slots padded to 16 bytes.
    static constexpr int kGatherFloats = G * (D + 2);
    static constexpr int kGatherStride = (kGatherFloats + 3) / 4 * 4;
    static constexpr int kGatherBytes = SPEC ? kMaxSpecCtas * kGatherStride * 4 : 0;
    // One-launch schedule: scratch for the merges done inside the kernel --
    // the list of a sequence's non-empty middle chunks, one merge weight per
    // (query head of the group, chunk), (weight of the sink-set partial,
    // normaliser) per query head, the list's length, and a copy of the chunk
    // boundary table (read with a different index per lane, which parameter
    // space serialises).
    static constexpr int kScratchFloats = kMaxChunks * (G + 1) + 2 * G + 4 + kMaxChunks + 4;
    static constexpr int kScratchBytes = FUSED ? kScratchFloats * 4 : 0;

    // Tile t goes to stage t mod STAGES and to consumer warp t mod NTW.  A
    // phase-parity wait alone is only sound if no waiter can be a ring lap
    // ahead of the stage's previous fill; when STAGES is not a multiple of
    // NTW, consecutive fills of a stage belong to different warps and a fast
    // warp could pass the parity test on the previous fill's phase.  So
    // every stage carries a fill ticket: the producer stores the tile's
    // global index (release) before filling it, and a consumer first waits
    // for its own index (acquire), which proves the previous fill's phase
    // completed, then tests the parity.  The tensor-core middle kernel takes
    // as many stages as fit (ALSPEC_MID_STAGES at most); the other kernels
    // keep whole rounds of NTW stages.
    static constexpr bool kFreeRing = MMA && !SPEC && !FUSED;
    static constexpr int kStagesBudget =
        (kSmemLimit - 1024 - kDepositBytes - 4096 - 768 - kGatherBytes - kScratchBytes) /
        kStageBytes;
    static constexpr int kStagesCap = kFreeRing ? ALSPEC_MID_STAGES : NTW * kSpwMax;
    static constexpr int kStagesFit = kStagesBudget < kStagesCap ? kStagesBudget : kStagesCap;
    static constexpr int kRounds = kStagesFit / NTW < 1 ? 1 : kStagesFit / NTW;
    static constexpr int STAGES =
        kFreeRing ? (kStagesFit < NTW ? NTW : kStagesFit) : NTW * kRounds;
    // Dynamic shared memory layout (offsets from a 1024-byte aligned base;
    // every region starts on a 128-byte boundary: the stage metadata are
    // int4, the barriers 8-byte words).
    static constexpr int align128(int x) { return (x + 127) / 128 * 128; }
    static constexpr int kOffDeposit = STAGES * kStageBytes;
    static constexpr int kOffMeta = align128(kOffDeposit + kDepositBytes);
    static constexpr int kOffFill = align128(kOffMeta + STAGES * 16);
    static constexpr int kOffBar = align128(kOffFill + STAGES * 4);
    static constexpr int kNumBars = 2 * STAGES + 4;
    static constexpr int kOffMisc = align128(kOffBar + kNumBars * 8);
    static constexpr int kOffGather = align128(kOffMisc + 16);
    static constexpr int kOffScratch = align128(kOffGather + kGatherBytes);
    static constexpr int kSmemBytes = (FUSED ? kOffScratch + kScratchBytes : kOffGather + kGatherBytes) +
                                      1024;  // + alignment slack
    static_assert(kOffDeposit % 1024 == 0 && kStageBytes % 1024 == 0 && kTileBytes % 1024 == 0,
                  "TMA destinations with 128-byte swizzle need 1024-byte alignment");
    static_assert(kOffMeta % 16 == 0 && kOffBar % 8 == 0 && kOffMisc % 16 == 0 &&
                      kOffGather % 16 == 0 && (kSlotFloats * 4) % 8 == 0,
                  "shared-memory region alignment");
    static_assert(kRowBytes % 128 == 0, "row must be a multiple of 128 bytes");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    static_assert(!MMA || (sizeof(T) == 2 && G <= 8), "tensor-core engine: bf16, g <= 8");
    static_assert(kSmemBytes <= kSmemLimit, "shared memory budget");
    static_assert(NTW >= 1 && NCW <= 8, "warp split");
    static_assert(STAGES >= NTW, "every consumer warp needs a stage");
    static_assert(kFreeRing || STAGES % NTW == 0, "whole rounds of stages");
    static_assert(!(SPEC && FUSED), "the one-launch kernel is a middle-kernel variant");
};

// ---------------------------------------------------------------- waiting

struct Shared {
    int abort;
    int merge;  // one-launch schedule: KV head whose merges this CTA owns, or -1
    int pad[2];
};

// Producer-side bounded wait (one thread).
__device__ __forceinline__ bool wait_one(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         const Params& p) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31) == 0) {
            if (*abort) return false;
            if (global_ns() - t0 > p.timeout_ns) {
                *abort = 1;
                atomicOr(p.ctr + kCtrError, kErrTimeout);
                return false;
            }
        }
    }
}

// Consumer-side bounded wait: every lane of the warp probes (each acquires),
// and the warp leaves together.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const Params& p, int lane) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool ok = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, ok)) return true;
        if ((it & 31) == 31) {
            int stop = 0;
            if (lane == 0) {
                const uint64_t now = global_ns();
                if (t0 == 0) {
                    t0 = now;
                } else if (now - t0 > p.timeout_ns) {
                    *abort = 1;
                    atomicOr(p.ctr + kCtrError, kErrTimeout);
                }
                stop = *abort;
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
        }
    }
}

// Consumer-side bounded wait for the fill with global tile index `gt` of a
// stage: first the stage's fill ticket must name that tile (which proves
// the stage's previous fill completed its phase), then the phase with
// `parity` must complete.  Every lane probes; the warp leaves together.
__device__ __forceinline__ bool wait_fill(uint64_t* bar, const uint32_t* ticket, uint32_t gt,
                                          uint32_t parity, volatile int* abort, const Params& p,
                                          int lane) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool ok = ld_acquire_shared(ticket) == gt && mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, ok)) return true;
        if ((it & 31) == 31) {
            int stop = 0;
            if (lane == 0) {
                const uint64_t now = global_ns();
                if (t0 == 0) {
                    t0 = now;
                } else if (now - t0 > p.timeout_ns) {
                    *abort = 1;
                    atomicOr(p.ctr + kCtrError, kErrTimeout);
                }
                stop = *abort;
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
        }
    }
}

// Test hook for the timeout path: both waits target mbarriers that nothing
// ever arrives on.  The producer-style wait gives up at p.timeout_ns, sets
// the abort flag and ORs the timeout bit into the error word; the
// consumer-style wait sees the abort and returns.  Nothing traps or faults.
__global__ void __launch_bounds__(64) stalled_wait_kernel(const __grid_constant__ Params p) {
    __shared__ uint64_t bar[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    volatile int* abort = &abort_flag;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        if (lane == 0) (void)wait_one(&bar[0], 0, abort, p);
    } else {
        (void)wait_warp(&bar[1], 0, abort, p, lane);
    }
}

// Weight of a partial with max m against the merged max M: exactly 1 when
// m == M, so merging one partial with empty ones reproduces it bit for bit.
__device__ __forceinline__ float merge_weight(float m, float M) {
    return m == M ? 1.f : exp2f(m - M);
}

// ====================================================== CUDA-core engine

template <class C, typename T>
struct CoreEngine {
    static constexpr int kPairs = Elem<T>::kPairs;
    static constexpr int kChunks = C::kRowBytes / 128;
    static constexpr int kLanePairs = kChunks * kPairs;
    static constexpr int kElemPerChunk = 16 / (int)sizeof(T);
    static constexpr int kElemPer128 = 128 / (int)sizeof(T);
    static constexpr int kD = C::kRowBytes / (int)sizeof(T);

    float2 q[C::GW][kLanePairs];  // prescaled query slice
    float2 o[C::GW][kLanePairs];  // unnormalised output slice
    float m[C::GW];               // warp-uniform running max (log2 domain)
    float l[C::GW];               // this lane's share of the exponential sum

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
#pragma unroll
            for (int j = 0; j < kLanePairs; ++j) o[h][j] = make_float2(0.f, 0.f);
        }
    }

    __device__ __forceinline__ void load_query(const Params& p, int b, int head0, int lane) {
        const int li = lane & 7;
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            const char* row = reinterpret_cast<const char*>(p.q) +
                              ((size_t)b * p.Hq + head0 + h) * C::kRowBytes + li * 16;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4*>(row + c * 128));
                float2 f[kPairs];
                Elem<T>::unpack(raw, f);
#pragma unroll
                for (int j = 0; j < kPairs; ++j)
                    q[h][c * kPairs + j] = make_float2(f[j].x * p.qscale, f[j].y * p.qscale);
            }
        }
    }

    // One 16-token tile: lanes 8u..8u+7 ("group" u) own rows 4u..4u+3.
    // One step: the CUDA-core engine reads the stage to the end of the tile.
    __device__ __forceinline__ void tile_load(char* ks, char* vs, int nvalid, int lane,
                                              float qscale) {
        tile(ks, vs, nvalid, lane, qscale);
    }
    __device__ __forceinline__ void tile_finish(int, int, float) {}

    __device__ __forceinline__ void tile(char* ks, char* vs, int nvalid, int lane, float) {
        const int grp = lane >> 3;
        const int li = lane & 7;
        const unsigned full = 0xffffffffu;

        float acc[4][C::GW];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const char* krow = ks + (grp * 4 + t) * C::kRowBytes + li * 16;
            float2 a[C::GW];
#pragma unroll
            for (int h = 0; h < C::GW; ++h) a[h] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4*>(krow + c * 128);
                float2 kf[kPairs];
                Elem<T>::unpack(raw, kf);
#pragma unroll
                for (int j = 0; j < kPairs; ++j)
#pragma unroll
                    for (int h = 0; h < C::GW; ++h)
                        a[h] = __ffma2_rn(q[h][c * kPairs + j], kf[j], a[h]);
            }
#pragma unroll
            for (int h = 0; h < C::GW; ++h) acc[t][h] = a[h].x + a[h].y;
        }

        // Reduce-scatter over the 8 lanes of the group: lanes 2u and 2u+1
        // end up with the full score of row u of the group.
        const bool b2 = (li & 4) != 0;
        const bool b1 = (li & 2) != 0;
        const int own = li >> 1;
        const bool valid = grp * 4 + own < nvalid;
        float s[C::GW];
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            const float k0 = b2 ? acc[2][h] : acc[0][h];
            const float s0 = b2 ? acc[0][h] : acc[2][h];
            const float k1 = b2 ? acc[3][h] : acc[1][h];
            const float s1 = b2 ? acc[1][h] : acc[3][h];
            const float w0 = k0 + __shfl_xor_sync(full, s0, 4);
            const float w1 = k1 + __shfl_xor_sync(full, s1, 4);
            const float kk = b1 ? w1 : w0;
            const float ss = b1 ? w0 : w1;
            float x = kk + __shfl_xor_sync(full, ss, 2);
            x += __shfl_xor_sync(full, x, 1);
            s[h] = valid ? x : -INFINITY;
        }

        float pr[C::GW];
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            float mx = s[h];
            mx = fmaxf(mx, __shfl_xor_sync(full, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(full, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(full, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(full, mx, 16));
            if (mx > m[h]) {
                const float sc = exp2f(m[h] - mx);
                const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                for (int j = 0; j < kLanePairs; ++j) o[h][j] = __fmul2_rn(o[h][j], sc2);
                l[h] *= sc;
                m[h] = mx;
            }
            pr[h] = valid ? exp2f(s[h] - m[h]) : 0.f;
            l[h] += (li & 1) ? 0.f : pr[h];
        }

#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float pt[C::GW];
#pragma unroll
            for (int h = 0; h < C::GW; ++h) pt[h] = __shfl_sync(full, pr[h], (lane & 24) | (t << 1));
            if (grp * 4 + t < nvalid) {
                const char* vrow = vs + (grp * 4 + t) * C::kRowBytes + li * 16;
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(vrow + c * 128);
                    float2 vf[kPairs];
                    Elem<T>::unpack(raw, vf);
#pragma unroll
                    for (int h = 0; h < C::GW; ++h) {
                        const float2 pp = make_float2(pt[h], pt[h]);
#pragma unroll
                        for (int j = 0; j < kPairs; ++j)
                            o[h][c * kPairs + j] = __ffma2_rn(pp, vf[j], o[h][c * kPairs + j]);
                    }
                }
            }
        }
    }

    // Reduce over the warp and store (m, l, o) of the GW heads into `slot`.
    __device__ __forceinline__ void deposit(float* slot, int lane) {
        const unsigned fm = 0xffffffffu;
        const int li = lane & 7;
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            float lsum = l[h];
#pragma unroll
            for (int x = 1; x < 32; x <<= 1) lsum += __shfl_xor_sync(fm, lsum, x);
#pragma unroll
            for (int j = 0; j < kLanePairs; ++j) {
                float2 v = o[h][j];
                v.x += __shfl_xor_sync(fm, v.x, 8);
                v.y += __shfl_xor_sync(fm, v.y, 8);
                v.x += __shfl_xor_sync(fm, v.x, 16);
                v.y += __shfl_xor_sync(fm, v.y, 16);
                o[h][j] = v;
            }
            float* hs = slot + h * (kD + 2);
            if (lane == 0) {
                hs[0] = m[h];
                hs[1] = lsum;
            }
            if (lane < 8) {
#pragma unroll
                for (int c = 0; c < kChunks; ++c)
#pragma unroll
                    for (int j = 0; j < kPairs; ++j) {
                        const int e = c * kElemPer128 + li * kElemPerChunk + 2 * j;
                        *reinterpret_cast<float2*>(hs + 2 + e) = o[h][c * kPairs + j];
                    }
            }
        }
    }
};

// ==================================================== tensor-core engine

// Byte offset of 16-byte chunk `c` (0..7) of row `r` inside a 2-D TMA box
// written with 128-byte swizzle (rows of 128 bytes).
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <class C, int D, int G>
struct MmaEngine {
    static constexpr int TT = C::TT;            // 32 tokens: 4 score n-tiles, 2 PV k-steps
    static constexpr int KS = D / 16;            // QK k-steps
    static constexpr int NT = D / 8;             // PV n-tiles
    static constexpr int kHalf = TT * 128;       // bytes of one 64-column box
    static constexpr int kHalves = D / 64;

    uint32_t qa[KS][2];  // A fragment words (row g, k 2r..2r+1) and (row g, k 2r+8..)
    float o[NT][4];      // P V accumulators: rows g (high part of P) and g+8 (residual)
    float m;             // running max of row g (log2 domain)
    float l;             // this lane's share of the exponential sum of row g
    float s[TT / 8][4];  // the current tile's scores (between tile_load and tile_finish)
    uint32_t vf[TT / 16][NT / 2][4];  // the current tile's V fragments

    __device__ __forceinline__ void reset() {
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    }

    __device__ __forceinline__ void load_query(const Params& p, int b, int head0, int lane) {
        const int g = lane >> 2;
        const int r = lane & 3;
        if (g < G) {
            const uint32_t* row = reinterpret_cast<const uint32_t*>(
                reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + head0 + g) * D);
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                qa[kk][0] = __ldg(row + kk * 8 + r);
                qa[kk][1] = __ldg(row + kk * 8 + 4 + r);
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) qa[kk][0] = qa[kk][1] = 0u;
        }
    }

    // Row `r`, 16-byte chunk `c` (0..D/8-1) of a K or V tile in a stage.
    __device__ __forceinline__ static uint32_t addr(uint32_t base, int r, int c) {
        return base + (uint32_t)((c >> 3) * kHalf) + swz(r, c & 7);
    }

    // Everything that reads the stage: clear padded rows, S^T = Q K^T, and
    // V's fragments into registers.  The stage can be released after this.
    __device__ __forceinline__ void tile_load(char* ks, char* vs, int nvalid, int lane, float) {
        // Rows past the end of the item may hold anything (even NaN): zero
        // their values so that 0 * V stays 0 in the P V products.
        if (nvalid < TT) {
            const int n = (TT - nvalid) * kHalves * 8;  // 16-byte chunks to clear
            for (int i = lane; i < n; i += 32) {
                const int row = nvalid + i / (kHalves * 8);
                const int rem = i % (kHalves * 8);
                *reinterpret_cast<uint4*>(vs + (rem >> 3) * kHalf + row * 128 + (rem & 7) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }
        const uint32_t kb = smem_addr(ks);
        const uint32_t vb = smem_addr(vs);

        // S^T = Q K^T: 4 n-tiles of 8 tokens.  Even and odd k-steps go to
        // separate accumulators (half-length MMA dependency chains).
#pragma unroll
        for (int j = 0; j < TT / 8; ++j) {
            float s2[4] = {0.f, 0.f, 0.f, 0.f};
            s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < KS / 2; ++kp) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(addr(kb, 8 * j + (lane & 7), 4 * kp + (lane >> 3)), b0, b1, b2, b3);
                mma_bf16_16816(s[j], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b0, b1);
                mma_bf16_16816(s2, qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b2, b3);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) s[j][i] += s2[i];
        }
        // V as the B operand of P V (transposed 8x8 loads), 2 k-steps of 16.
#pragma unroll
        for (int t2 = 0; t2 < TT / 16; ++t2)
#pragma unroll
            for (int jp = 0; jp < NT / 2; ++jp) {
                const int row = 16 * t2 + ((lane >> 3) & 1) * 8 + (lane & 7);
                ldsm_x4_t(addr(vb, row, 2 * jp + (lane >> 4)), vf[t2][jp][0], vf[t2][jp][1],
                          vf[t2][jp][2], vf[t2][jp][3]);
            }
    }

    // The rest of the tile, from registers: online softmax and O += P V.
    __device__ __forceinline__ void tile_finish(int nvalid, int lane, float qscale) {
        const int g = lane >> 2;
        const int r = lane & 3;
        const unsigned full = 0xffffffffu;
        // Online softmax on row g (lanes 4g..4g+3 hold its 32 scores).
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < TT / 8; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool ok = g < G && 8 * j + 2 * r + e < nvalid;
                s[j][e] = ok ? s[j][e] * qscale : -INFINITY;
                mx = fmaxf(mx, s[j][e]);
            }
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, 2));
        const bool grow = mx > m;
        if (__any_sync(full, grow)) {
            const float sc = grow ? exp2f(m - mx) : 1.f;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                o[j][0] *= sc;
                o[j][1] *= sc;
                o[j][2] *= sc;
                o[j][3] *= sc;
            }
            l *= sc;
            m = grow ? mx : m;
        }
        uint32_t pa[TT / 16][4];
#pragma unroll
        for (int t2 = 0; t2 < TT / 16; ++t2) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 2 * t2 + h;
                const float p0 = s[j][0] == -INFINITY ? 0.f : exp2f(s[j][0] - m);
                const float p1 = s[j][1] == -INFINITY ? 0.f : exp2f(s[j][1] - m);
                l += p0 + p1;
                const uint32_t hi = pack_bf16(p0, p1);
                const float r0 = p0 - __uint_as_float(hi << 16);
                const float r1 = p1 - __uint_as_float(hi & 0xffff0000u);
                pa[t2][2 * h] = hi;                     // rows g: high part
                pa[t2][2 * h + 1] = pack_bf16(r0, r1);  // rows g+8: residual
            }
        }

        // O += P V over the 2 k-steps of 16 tokens.
#pragma unroll
        for (int t2 = 0; t2 < TT / 16; ++t2) {
#pragma unroll
            for (int jp = 0; jp < NT / 2; ++jp) {
                mma_bf16_16816(o[2 * jp], pa[t2][0], pa[t2][1], pa[t2][2], pa[t2][3],
                               vf[t2][jp][0], vf[t2][jp][1]);
                mma_bf16_16816(o[2 * jp + 1], pa[t2][0], pa[t2][1], pa[t2][2], pa[t2][3],
                               vf[t2][jp][2], vf[t2][jp][3]);
            }
        }
    }

    __device__ __forceinline__ void deposit(float* slot, int lane) {
        const int g = lane >> 2;
        const int r = lane & 3;
        float lsum = l;
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        if (g < G) {
            float* hs = slot + g * (D + 2);
            if (r == 0) {
                hs[0] = m;
                hs[1] = lsum;
            }
#pragma unroll
            for (int j = 0; j < NT; ++j)
                *reinterpret_cast<float2*>(hs + 2 + 8 * j + 2 * r) =
                    make_float2(o[j][0] + o[j][2], o[j][1] + o[j][3]);
        }
    }
};

template <class C, typename T, int D, int G, bool MMA>
struct EngineOf {
    using type = CoreEngine<C, T>;
};
template <class C, typename T, int D, int G>
struct EngineOf<C, T, D, G, true> {
    using type = MmaEngine<C, D, G>;
};

// Sink-set kernel, several CTAs per head (one cluster): every CTA merges its
// warps' states into one partial (m, l, o for the G heads) and sends it with
// asynchronous 16-byte stores into slot `rank` of the gather area of every
// CTA of the cluster; the bytes complete on each CTA's gather barrier, which
// expects all n1 slots.  Each CTA then waits (bounded), merges the slots in
// rank order for its slice [rank * per, (rank + 1) * per) of the G * D
// outputs and publishes that slice of O_spec.  A last cluster barrier, which
// each CTA reaches only after all bytes sent to it have landed, keeps every
// CTA resident until its stores are done.  Every thread of every CTA gets
// here (all waits before are bounded) and has waited once on the cluster
// barrier since the set-up, so every gather barrier is initialised.
template <int D, int G, class C>
__device__ __forceinline__ void cluster_gather(const Params& p, const float* deposit,
                                               float* gather, uint64_t* gather_bar) {
    constexpr int kF = C::kGatherFloats;
    constexpr int kStride = C::kGatherStride;
    constexpr int NTW = C::NTW;
    const int n = p.n1;
    const uint32_t rank = cluster_ctarank();
    const uint32_t dst = smem_addr(gather + rank * kStride);
    const uint32_t bar = smem_addr(gather_bar);
    for (int v = threadIdx.x; v < kStride / 4; v += C::kThreads) {
        float x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int idx = 4 * v + k;
            float val = 0.f;
            if (idx < kF) {
                const int hh = idx / (D + 2);
                const int e = idx % (D + 2);
                const float* base =
                    deposit + (hh / C::GW) * NTW * C::kSlotFloats + (hh % C::GW) * (D + 2);
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NTW; ++w) M = fmaxf(M, base[w * C::kSlotFloats]);
                if (e == 0) {
                    val = M;
                } else {
#pragma unroll
                    for (int w = 0; w < NTW; ++w) {
                        const float* ws = base + w * C::kSlotFloats;
                        val = fmaf(merge_weight(ws[0], M), ws[e < 2 ? 1 : e], val);
                    }
                }
            }
            x[k] = val;  // (m, l, o[0..D)) of head hh
        }
        if (ALSPEC_IN_BOUNDS(p, rank < (uint32_t)n && n <= kMaxSpecCtas))
            for (int j = 0; j < n; ++j)
                st_async_v4(dsmem_addr(dst, (uint32_t)j) + 16u * (uint32_t)v, x,
                            dsmem_addr(bar, (uint32_t)j));
    }

    // Wait (bounded) for the n1 slots sent to this CTA.
    bool ok = true;
    {
        const uint64_t t0 = global_ns();
        for (uint32_t it = 0; !mbar_try_wait_cluster(gather_bar, 0); ++it) {
            if ((it & 31) == 31 && global_ns() - t0 > p.timeout_ns) {
                ok = false;
                break;
            }
        }
    }
    if (!ok) atomicOr(p.ctr + kCtrError, kErrTimeout);
    const int bh0 = (int)blockIdx.x / n;
    const int b = bh0 / p.Hkv;
    const int kvh = bh0 % p.Hkv;
    const int per = (G * D + n - 1) / n;
    const int hi = min(G * D, ((int)rank + 1) * per);
    for (int idx = (int)rank * per + (int)threadIdx.x; idx < hi; idx += C::kThreads) {
        const int hh = idx / D;
        const int e = idx % D;
        const float* g = gather + hh * (D + 2);
        float m[kMaxSpecCtas];
        float M = -INFINITY;
#pragma unroll
        for (int j = 0; j < kMaxSpecCtas; ++j) {
            m[j] = j < n ? g[j * kStride] : -INFINITY;
            M = fmaxf(M, m[j]);
        }
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxSpecCtas; ++j) {
            if (j < n) {
                const float f = merge_weight(m[j], M);
                L = fmaf(f, g[j * kStride + 1], L);
                O = fmaf(f, g[j * kStride + 2 + e], O);
            }
        }
        const size_t bh = (size_t)b * p.Hq + kvh * G + hh;
        if (!ALSPEC_IN_BOUNDS(p, b < p.B && kvh * G + hh < p.Hq)) continue;
        if (e == 0) {
            p.spec_ml[bh * 2] = M;
            p.spec_ml[bh * 2 + 1] = L;
        }
        p.spec_o[bh * D + e] = O;
        p.out_spec[bh * D + e] = __fdiv_rn(O, L);
    }
    __syncthreads();
    if (threadIdx.x == 0) trace_publish(p, 0);
    __syncwarp();
    cluster_arrive_relaxed();
    cluster_wait();
}

// ------------------------------------------- relative L2 and the flag

constexpr int kMergeCols = 32;  // output columns per (squared distance, squared norm) slot

// Number of (squared distance, squared norm) slots per query head.
__host__ __device__ constexpr int merge_splits(int d) { return d / kMergeCols; }

// One warp, once every slot of sequence b is written and lane 0 has
// acquired them (the sequence's last ticket):
// rel_l2 = sqrt(sum of squared distances / sum of squared norms) over the
// sequence's H_q * d outputs (fp64, fixed order), and the commit flag
// rel_l2 <= lambda.  No distance and no norm gives 0 (commit); a distance
// with a zero norm gives infinity (discard); NaN compares false (discard).
template <int D>
__device__ __forceinline__ void write_flag(const Params& p, int b, int lane) {
    constexpr int NS = merge_splits(D);
    __syncwarp();  // orders lane 0's acquire of the ticket before every lane's loads
    if (!ALSPEC_IN_BOUNDS(p, b >= 0 && b < p.B)) return;
    double D2 = 0.0, N2 = 0.0;
    const float2* dn = reinterpret_cast<const float2*>(p.dn) + (size_t)b * p.Hq * NS;
    for (int i = lane; i < p.Hq * NS; i += 32) {
        const float2 x = __ldcg(dn + i);
        D2 += (double)x.x;
        N2 += (double)x.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        D2 += __shfl_xor_sync(0xffffffffu, D2, o);
        N2 += __shfl_xor_sync(0xffffffffu, N2, o);
    }
    if (lane == 0) {
        double r;
        if (N2 == 0.0) {
            r = D2 == 0.0 ? 0.0 : (double)INFINITY;
        } else {
            r = sqrt(D2 / N2);
        }
        p.rel_l2[b] = (float)r;
        p.commit[b] = r <= (double)p.lambda ? 1 : 0;
    }
}

// Fill stage s with tile t of item `item` (meta word, barrier arrival with
// the expected bytes, the K and V copies).  Any lane may fill any stage.
template <typename T, int D, int G, bool SPEC, bool MMA, bool FUSED>
__device__ __forceinline__ void fill_stage(const Params& p, unsigned char* smem, int4* meta,
                                           uint32_t* fill, uint64_t* full_bar, int s, uint32_t gt,
                                           int item, const Item& it, int t, int ntiles) {
    using C = Cfg<T, D, G, SPEC, MMA, FUSED>;
    constexpr int TT = C::TT;
    const int head_row = (it.b * p.Hkv + it.kvh) * p.Lmax;
    int start = 0, nvalid = 0;
    if (t < it.ntiles) tile_rows<SPEC, TT, FUSED>(it, t, start, nvalid);
    if (!ALSPEC_IN_BOUNDS(p, nvalid <= 0 || (start >= 0 && nvalid <= TT &&
                                             start + nvalid <= p.Lmax && it.b < p.B &&
                                             it.kvh < p.Hkv)))
        nvalid = 0;  // (the stage then arrives empty)
    st_release_shared(fill + s, gt);  // this fill is the one for tile gt
    meta[s] = make_int4(item, t, nvalid,
                        (FUSED ? it.ntiles << 1 : 0) | (t >= ntiles - C::NTW ? kLastTileFlag : 0));
    if (nvalid == 0) {
        mbar_arrive(full_bar + s);
        return;
    }
    char* ks = reinterpret_cast<char*>(smem) + s * C::kStageBytes;
    char* vs = ks + C::kTileBytes;
    // The cache rows are read once: evict them from L2 first.
    const uint64_t pol = l2_evict_first_policy();
    if (MMA) {
        // Whole boxes; rows past the tensor end arrive as zeros.
        mbar_arrive_expect_tx(full_bar + s, (uint32_t)C::kStageBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            tma_load_2d(ks + h * TT * 128, &p.tmap_k, 64 * h, head_row + start, full_bar + s, pol);
            tma_load_2d(vs + h * TT * 128, &p.tmap_v, 64 * h, head_row + start, full_bar + s, pol);
        }
    } else {
        const uint32_t bytes = (uint32_t)nvalid * C::kRowBytes;
        mbar_arrive_expect_tx(full_bar + s, 2u * bytes);
        const size_t off = ((size_t)head_row + start) * C::kRowBytes;
        bulk_load(ks, reinterpret_cast<const char*>(p.k) + off, bytes, full_bar + s, pol);
        bulk_load(vs, reinterpret_cast<const char*>(p.v) + off, bytes, full_bar + s, pol);
    }
}

// The ring's first fills on the tensor-core engine, by the producer warp:
// lane l issues copy l % OPS (K or V, 64 columns) of stage l / OPS, so one
// copy instruction of the warp issues stage 0's copies first, then stage
// 1's, ... (one lane per stage, each issuing all of its stage's copies,
// put the first stage's last copy behind every other stage's first ones:
// measured, the burst of 48 copies took ~1.5 us to issue).  Same stage
// state as fill_stage for tiles 0 .. fresh-1 of `it`.
template <typename T, int D, int G, bool SPEC, bool MMA, bool FUSED>
__device__ __forceinline__ void fill_fresh(const Params& p, unsigned char* smem, int4* meta,
                                           uint32_t* fill, uint64_t* full_bar, int item,
                                           const Item& it, int fresh, int ntiles, int lane) {
    using C = Cfg<T, D, G, SPEC, MMA, FUSED>;
    constexpr int TT = C::TT;
    constexpr int OPS = 2 * (D / 64);  // copies per stage
    constexpr int PER = 32 / OPS;      // stages per round of the warp
    static_assert(32 % OPS == 0, "copies per stage");
    const int head_row = (it.b * p.Hkv + it.kvh) * p.Lmax;
    const uint64_t pol = l2_evict_first_policy();
    for (int s0 = 0; s0 < fresh; s0 += PER) {
        const int s = s0 + lane / OPS;
        const int op = lane % OPS;
        const bool mine = s < fresh;
        int start = 0, nvalid = 0;
        if (mine && s < it.ntiles) tile_rows<SPEC, TT, FUSED>(it, s, start, nvalid);
        if (mine && !ALSPEC_IN_BOUNDS(p, nvalid <= 0 || (start >= 0 && nvalid <= TT &&
                                                         start + nvalid <= p.Lmax &&
                                                         it.b < p.B && it.kvh < p.Hkv)))
            nvalid = 0;  // (the stage then arrives empty)
        if (mine && op == 0) {
            st_release_shared(fill + s, (uint32_t)s);
            meta[s] = make_int4(item, s, nvalid,
                                (FUSED ? it.ntiles << 1 : 0) |
                                    (s >= ntiles - C::NTW ? kLastTileFlag : 0));
            if (nvalid == 0)
                mbar_arrive(full_bar + s);
            else
                mbar_arrive_expect_tx(full_bar + s, (uint32_t)C::kStageBytes);
        }
        __syncwarp();  // each stage's expected bytes are set before its copies
        if (mine && nvalid > 0) {
            const int h = op >> 1;
            char* dst = reinterpret_cast<char*>(smem) + s * C::kStageBytes +
                        ((op & 1) ? C::kTileBytes : 0) + h * TT * 128;
            tma_load_2d(dst, (op & 1) ? static_cast<const void*>(&p.tmap_v) : &p.tmap_k, 64 * h,
                        head_row + start, full_bar + s, pol);
        }
    }
}

// The producer warp: fill the stage ring with the tiles of the items this CTA
// pulls, then send end markers.  The first item (`item0`, taken before the
// CTA's init barrier) fills the untouched stages from every lane (one copy
// per lane on the tensor-core engine, fill_fresh; one tile per lane on the
// CUDA-core engine), so the first copies leave within a few hundred cycles;
// lane 0 alone continues with the rest, waiting for each stage to be
// released.
template <typename T, int D, int G, bool SPEC, bool MMA, bool FUSED>
__device__ __forceinline__ void produce(const Params& p, unsigned char* smem, int4* meta,
                                        uint32_t* fill, uint64_t* full_bar, uint64_t* empty_bar,
                                        volatile int* abort, int lane, int item0,
                                        const Item& it0) {
    using C = Cfg<T, D, G, SPEC, MMA, FUSED>;
    const int n_items = p.B * p.Hkv * (SPEC ? p.n1 : (FUSED ? p.n1 + p.n2 : p.n2));
    auto rounded = [](const Item& it) { return (it.ntiles + C::NTW - 1) / C::NTW * C::NTW; };
    const bool have0 = item0 < n_items && it0.ntiles > 0;
    const int fresh = have0 ? min(rounded(it0), C::STAGES) : 0;
    if constexpr (MMA) {
        fill_fresh<T, D, G, SPEC, MMA, FUSED>(p, smem, meta, fill, full_bar, item0, it0, fresh,
                                              rounded(it0), lane);
    } else {
        for (int t = lane; t < fresh; t += 32)
            fill_stage<T, D, G, SPEC, MMA, FUSED>(p, smem, meta, fill, full_bar, t, (uint32_t)t,
                                                  item0, it0, t, rounded(it0));
    }
    if (lane != 0) return;

    uint32_t gt = (uint32_t)fresh;
    bool ok = true;
    // Sequential part: wait for stage gt % STAGES, fill it.
    auto run = [&](int item, const Item& it, int t_begin) {
        const int ntiles = rounded(it);
        for (int t = t_begin; t < ntiles; ++t, ++gt) {
            const int s = gt % C::STAGES;
            if (!wait_one(empty_bar + s, ((gt / C::STAGES) & 1) ^ 1, abort, p)) {
                ok = false;
                return;
            }
            fill_stage<T, D, G, SPEC, MMA, FUSED>(p, smem, meta, fill, full_bar, s, gt, item, it, t,
                                                  ntiles);
        }
    };
    if (have0) run(item0, it0, fresh);
    if (!SPEC && item0 < n_items) {
        while (ok) {
            const int item = (int)atomicAdd(p.ctr + kCtrQueue, 1u);
            if (item >= n_items || *abort) break;
            const Item it = decode_item<SPEC, C::TT, FUSED>(p, item, true);
            if (it.ntiles > 0) run(item, it, 0);
        }
    }
    if (ok) {
        // One end marker per token slot, so every consumer warp sees one.
        for (int i = 0; i < C::NTW; ++i, ++gt) {
            const int s = gt % C::STAGES;
            if (!wait_one(empty_bar + s, ((gt / C::STAGES) & 1) ^ 1, abort, p)) {
                ok = false;
                break;
            }
            st_release_shared(fill + s, gt);
            meta[s] = make_int4(-1, 0, 0, 0);
            mbar_arrive(full_bar + s);
        }
    }
    if (!ok) {
        // Drain: wait (bounded) for the copies of the most recent fill of
        // every stage, so that none lands after this CTA exits.
        const uint32_t lo = gt > (uint32_t)C::STAGES ? gt - C::STAGES : 0;
        for (uint32_t g2 = lo; g2 < gt; ++g2) {
            const int s = g2 % C::STAGES;
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(full_bar + s, (g2 / C::STAGES) & 1)) {
                if (global_ns() - t0 > p.timeout_ns) break;
            }
        }
    }
    if (!SPEC) {
        // The CTA that stops last (of every launch sharing the queue)
        // resets the queue for the next call.
        const unsigned t = atomicAdd(p.ctr + kCtrDone, 1u);
        if (t == (unsigned)p.mid_ctas - 1) {
            atomicExch(p.ctr + kCtrQueue, 0u);
            atomicExch(p.ctr + kCtrDone, 0u);
        }
    }
}

// ------------------------------------------------ one-launch schedule merges
//
// In the one-launch schedule each (sequence, KV head) has a tile ticket in
// the workspace: every item, sink-set or middle, adds its tile count when
// its partial is written.  The CTA that completes a head merges, for the
// group's G query heads, the sink-set item partials into O_spec (and the
// merged sink-set partial) and that with the middle partials into O_exact,
// writes their (squared distance, squared norm) slots, then takes a
// per-sequence ticket; the CTA that takes a sequence's last one writes
// rel_l2 and the flag.  Every merge runs in a fixed order, so results do
// not depend on which CTA does it.  (O_spec is thus written at the end of
// the head's work, not early: in one launch, nothing outside the kernel
// could use it before the launch ends.)
//
// The merges run on the consumer warps of one CTA (`sync` is their barrier;
// every consumer thread calls with the same arguments).  Tickets are taken
// with acquire-release atomics after a barrier over the writing threads, so
// the partials of every contributor are visible to the merging CTA (loads go
// to L2).

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
// Butterfly sum: every lane ends with the same value (each step adds the
// same two operands on both partner lanes).
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// O_spec of one (sequence, KV head) from its sink-set item partials: per
// query head M = max m_j, f_j = 2^(m_j - M), l = sum f_j l_j, o = sum f_j o_j
// (items in order), O_spec = o / l; (M, l, o) is also stored as the merged
// sink-set partial for the exact merge.
template <class C, int D, int G, class Sync>
__device__ __forceinline__ bool fused_spec_merge(const Params& p, int b, int kvh, float* scratch,
                                                 int warp, int lane, Sync& sync) {
    constexpr int NCT = C::NCW * 32;
    constexpr int NQ = D / 4;               // float4 columns per head
    constexpr int kJ = kMaxSpecItemsFused;  // items per head at most
    const int ctid = warp * 32 + lane;
    const int per = p.c1 / C::TT;
    const int n = cdiv(spec_tiles(seq_geom(p, b, false), C::TT), per);  // items with rows
    float* w = scratch + kMaxChunks;  // [G][kMaxChunks]
    float* fl = w + G * kMaxChunks;   // [G][2]: M, l
    const size_t bq0 = (size_t)b * p.Hq + kvh * G;
    for (int hh = warp; hh < G; hh += C::NCW) {
        const float2* ml = reinterpret_cast<const float2*>(p.spec_pml) + (bq0 + hh) * p.n1;
        float2 x[kJ / 32];
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kJ / 32; ++k) {
            const int j = lane + 32 * k;
            x[k] = j < n ? __ldcg(ml + j) : make_float2(-INFINITY, 0.f);
            M = fmaxf(M, x[k].x);
        }
        M = warp_max(M);
        float lsum = 0.f;
#pragma unroll
        for (int k = 0; k < kJ / 32; ++k) {
            const int j = lane + 32 * k;
            if (j < n) {
                const float f = merge_weight(x[k].x, M);
                w[hh * kMaxChunks + j] = f;
                lsum = fmaf(f, x[k].y, lsum);
            }
        }
        lsum = warp_sum(lsum);
        if (lane == 0) {
            fl[2 * hh] = M;
            fl[2 * hh + 1] = lsum;
        }
    }
    if (!sync()) return false;
    // Lane j of the CTA owns 4 consecutive columns of one head; all of its
    // item loads are issued before the sums (items in order).
    constexpr int kB = 16;
    for (int j = ctid; j < G * NQ; j += NCT) {
        const int hh = j / NQ;
        const int e4 = j % NQ;
        const size_t bq = bq0 + hh;
        const float4* o = reinterpret_cast<const float4*>(p.spec_po + bq * p.n1 * D) + e4;
        const float* wh = w + hh * kMaxChunks;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j0 = 0; j0 < n; j0 += kB) {
            float4 v[kB];
#pragma unroll
            for (int u = 0; u < kB; ++u)
                v[u] = j0 + u < n ? __ldcg(o + (size_t)(j0 + u) * NQ) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                if (j0 + u < n) {
                    const float f = wh[j0 + u];
                    O.x = fmaf(f, v[u].x, O.x);
                    O.y = fmaf(f, v[u].y, O.y);
                    O.z = fmaf(f, v[u].z, O.z);
                    O.w = fmaf(f, v[u].w, O.w);
                }
            }
        }
        const float L = fl[2 * hh + 1];
        if (e4 == 0) {
            p.spec_ml[bq * 2] = fl[2 * hh];
            p.spec_ml[bq * 2 + 1] = L;
        }
        reinterpret_cast<float4*>(p.spec_o + bq * D)[e4] = O;
        // (out_spec need not be 16-byte aligned.)
        float* os = p.out_spec + bq * D + 4 * e4;
        os[0] = __fdiv_rn(O.x, L);
        os[1] = __fdiv_rn(O.y, L);
        os[2] = __fdiv_rn(O.z, L);
        os[3] = __fdiv_rn(O.w, L);
    }
    return sync();
}

// O_exact of one (sequence, KV head): the merged sink-set partial and the
// sequence's non-empty middle chunks (in chunk order) by the log-sum-exp
// rule, O_exact = o / l per query head; then each head's (squared distance,
// squared norm) against O_spec per 32 columns, and the sequence ticket.
// With no middle chunk the sink-set partial's weight is exactly 1, so
// O_exact is O_spec bit for bit.
//
// `ring` (optional): the CTA's idle stage ring (after its last item) of
// `ring_bytes`, and `mbar` a fresh mbarrier.  When the group's middle
// partials fit, they are pulled in with bulk copies -- loads through the
// registers of one SM reach only a few tens of GB/s, so a head's ~180 KB
// of partials took several microseconds that way -- and read from there.
template <class C, int D, int G, class Sync>
__device__ __forceinline__ bool fused_head_merge(const Params& p, int bh, float* scratch,
                                                 int warp, int lane, Sync& sync,
                                                 unsigned char* ring = nullptr,
                                                 size_t ring_bytes = 0, uint64_t* mbar = nullptr,
                                                 volatile int* abort = nullptr) {
    constexpr int NCT = C::NCW * 32;
    constexpr int NQ = D / 4;  // float4 columns per head
    constexpr int NS = merge_splits(D);
    constexpr int kU = 16;     // chunk loads each thread keeps in flight
    constexpr int kS = 4;      // independent partial sums per column
    static_assert(NQ % 8 == 0, "a 32-column slot is 8 lanes of float4 columns");
    const int b = bh / p.Hkv;
    const int kvh = bh % p.Hkv;
    int* list = reinterpret_cast<int*>(scratch);  // [kMaxChunks]
    float* w = scratch + kMaxChunks;               // [G][kMaxChunks]
    float* fl = w + G * kMaxChunks;                // [G][2]: weight of the sink-set partial, l
    int* nlist = reinterpret_cast<int*>(fl + 2 * G);
    const unsigned* fq = reinterpret_cast<const unsigned*>(nlist + 4);  // chunk table copy
    const size_t bq0 = (size_t)b * p.Hq + kvh * G;
    // The group's partials [G][n2][D] are contiguous in the workspace.
    const size_t blk_bytes = (size_t)G * p.n2 * D * sizeof(float);
    const bool bulk = ring != nullptr && p.n2 > 0 && blk_bytes <= ring_bytes;
    if (bulk && warp == 0) {
        constexpr uint32_t kPiece = 16384;
        const char* src = reinterpret_cast<const char*>(p.mid_o + bq0 * p.n2 * D);
        // The partials were acquired through the generic proxy (ticket).
        fence_proxy_async_global();
        if (lane == 0) mbar_arrive_expect_tx(mbar, (uint32_t)blk_bytes);
        __syncwarp();
        const uint64_t pol = l2_evict_first_policy();
        for (size_t off = (size_t)lane * kPiece; off < blk_bytes; off += 32 * (size_t)kPiece) {
            const uint32_t nb = (uint32_t)(blk_bytes - off < kPiece ? blk_bytes - off : kPiece);
            if (ALSPEC_IN_BOUNDS(p, off + nb <= ring_bytes && bq0 + G <= (size_t)p.B * p.Hq))
                bulk_load(ring + off, src + off, nb, mbar, pol);
        }
    }
    // O_spec and the merged sink-set partial, while the copies land.
    if (!fused_spec_merge<C, D, G>(p, b, kvh, scratch, warp, lane, sync)) return false;
    if (warp == 0 && lane == 0) trace_publish(p, 0);

    // Non-empty chunks of this sequence's middle, in order (warp 0).
    if (warp == 0) {
        const int mid_tiles = cdiv(seq_geom(p, b, false).mid_len, C::TT);
        int count = 0;
        for (int c0 = 0; c0 < p.n2; c0 += 32) {
            const int c = c0 + lane;
            bool ne = false;
            if (c < p.n2) {
                const int lo = (int)(((unsigned long long)mid_tiles * fq[c]) >> kFracBits);
                const int hi = (int)(((unsigned long long)mid_tiles * fq[c + 1]) >> kFracBits);
                ne = hi > lo;
            }
            const unsigned bal = __ballot_sync(0xffffffffu, ne);
            const int at = count + __popc(bal & ((1u << lane) - 1u));
            if (ne && ALSPEC_IN_BOUNDS(p, at < kMaxChunks)) list[at] = c;
            count += __popc(bal);
        }
        if (lane == 0) *nlist = count;
    }
    if (!sync()) return false;
    const int n = *nlist;

    // Per query head (one warp each): max, weights, normaliser.
    for (int hh = warp; hh < G; hh += C::NCW) {
        const float2 sml = __ldcg(reinterpret_cast<const float2*>(p.spec_ml) + bq0 + hh);
        const float2* ml = reinterpret_cast<const float2*>(p.mid_ml) + (bq0 + hh) * p.n2;
        float2 x[kMaxChunks / 32];
        float M = sml.x;
#pragma unroll
        for (int k = 0; k < kMaxChunks / 32; ++k) {
            const int i = lane + 32 * k;
            x[k] = i < n ? __ldcg(ml + list[i]) : make_float2(-INFINITY, 0.f);
            M = fmaxf(M, x[k].x);
        }
        M = warp_max(M);
        float lsum = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxChunks / 32; ++k) {
            const int i = lane + 32 * k;
            if (i < n) {
                const float f = merge_weight(x[k].x, M);
                w[hh * kMaxChunks + i] = f;
                lsum = fmaf(f, x[k].y, lsum);
            }
        }
        lsum = warp_sum(lsum);
        if (lane == 0) {
            const float f0 = merge_weight(sml.x, M);
            fl[2 * hh] = f0;
            fl[2 * hh + 1] = fmaf(f0, sml.y, lsum);
        }
    }
    if (!sync()) return false;
    if (bulk && !wait_warp(mbar, 0, abort, p, lane)) return false;

    // Columns: lane j of the CTA owns 4 consecutive columns of one head; the
    // 8 lanes of a 32-column slot reduce its distance and norm.
    for (int j0 = warp * 32; j0 < G * NQ; j0 += NCT) {
        const int j = j0 + lane;
        const bool act = j < G * NQ;
        const int hh = act ? j / NQ : 0;
        const int e4 = act ? j % NQ : 0;
        const size_t bq = bq0 + hh;
        float dd = 0.f, nn = 0.f;
        if (act) {
            const float4 so = __ldcg(reinterpret_cast<const float4*>(p.spec_o + bq * D) + e4);
            const float sl = __ldcg(p.spec_ml + bq * 2 + 1);
            const float f0 = fl[2 * hh];
            const float L = fl[2 * hh + 1];
            const float* wh = w + hh * kMaxChunks;
            float4 a = make_float4(f0 * so.x, f0 * so.y, f0 * so.z, f0 * so.w);
            // kS interleaved sums (list position i goes to sum i mod kS),
            // added in a fixed tree at the end: the same order on both
            // paths, so the bits do not depend on which one the merging
            // CTA takes.
            float4 acc[kS];
            acc[0] = a;
#pragma unroll
            for (int k = 1; k < kS; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            auto add = [&](float4& t, float f, const float4& v) {
                t.x = fmaf(f, v.x, t.x);
                t.y = fmaf(f, v.y, t.y);
                t.z = fmaf(f, v.z, t.z);
                t.w = fmaf(f, v.w, t.w);
            };
            if (bulk) {
                const float4* mo = reinterpret_cast<const float4*>(ring) + (size_t)hh * p.n2 * NQ + e4;
                int i = 0;
                for (; i + kS <= n; i += kS) {
                    float4 v[kS];
#pragma unroll
                    for (int k = 0; k < kS; ++k) v[k] = mo[(size_t)list[i + k] * NQ];
#pragma unroll
                    for (int k = 0; k < kS; ++k) add(acc[k], wh[i + k], v[k]);
                }
#pragma unroll
                for (int k = 0; k < kS - 1; ++k)
                    if (i + k < n) add(acc[k], wh[i + k], mo[(size_t)list[i + k] * NQ]);
            }
            if (!bulk) {
                static_assert(kU % kS == 0, "batches start at sum 0");
                const float4* mo = reinterpret_cast<const float4*>(p.mid_o + bq * p.n2 * D) + e4;
                for (int i0 = 0; i0 < n; i0 += kU) {
                    float4 v[kU];
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const int i = i0 + u;
                        v[u] = i < n ? __ldcg(mo + (size_t)list[i] * NQ)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const int i = i0 + u;
                        if (i < n) add(acc[u % kS], wh[i], v[u]);
                    }
                }
            }
            static_assert(kS == 4, "the final tree below");
            a.x = (acc[0].x + acc[1].x) + (acc[2].x + acc[3].x);
            a.y = (acc[0].y + acc[1].y) + (acc[2].y + acc[3].y);
            a.z = (acc[0].z + acc[1].z) + (acc[2].z + acc[3].z);
            a.w = (acc[0].w + acc[1].w) + (acc[2].w + acc[3].w);
            const float4 oe = make_float4(__fdiv_rn(a.x, L), __fdiv_rn(a.y, L), __fdiv_rn(a.z, L),
                                          __fdiv_rn(a.w, L));
            const float4 os = make_float4(__fdiv_rn(so.x, sl), __fdiv_rn(so.y, sl),
                                          __fdiv_rn(so.z, sl), __fdiv_rn(so.w, sl));
            // (out_exact need not be 16-byte aligned.)
            float* ox = p.out_exact + bq * D + 4 * e4;
            ox[0] = oe.x;
            ox[1] = oe.y;
            ox[2] = oe.z;
            ox[3] = oe.w;
            const float d0 = oe.x - os.x, d1 = oe.y - os.y, d2 = oe.z - os.z, d3 = oe.w - os.w;
            dd = d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
            nn = oe.x * oe.x + oe.y * oe.y + oe.z * oe.z + oe.w * oe.w;
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            dd += __shfl_xor_sync(0xffffffffu, dd, o);
            nn += __shfl_xor_sync(0xffffffffu, nn, o);
        }
        if (act && (lane & 7) == 0 && ALSPEC_IN_BOUNDS(p, bq < (size_t)p.B * p.Hq))
            *reinterpret_cast<float2*>(p.dn + (bq * NS + e4 / 8) * 2) = make_float2(dd, nn);
    }
    // Every slot of this head is written once this passes.
    if (!sync()) return false;
    if (warp == 0) {
        unsigned last = 0;
        if (lane == 0) {
            unsigned* word = p.ctr + ctr_seq(p.B, p.Hkv, b);
            const unsigned t = atom_add_acq_rel_gpu(word, 1u);
            last = t == (unsigned)(p.Hkv - 1);
            if (last) atomicExch(word, 0u);
        }
        if (__shfl_sync(0xffffffffu, last, 0)) write_flag<D>(p, b, lane);
        if (lane == 0) trace_publish(p, 1);
    }
    return true;
}

// Consumer warps: compute tiles; at each item's end merge the warps' states
// and write the item's partial (or, for the sink set, O_spec / this CTA's
// share of it).
template <typename T, int D, int G, bool SPEC, bool MMA, bool FUSED>
__device__ __forceinline__ void consume(const Params& p, unsigned char* smem, float* deposit,
                                        int4* meta, const uint32_t* fill, uint64_t* full_bar,
                                        uint64_t* empty_bar, uint64_t* dep_bar, uint64_t* free_bar,
                                        uint64_t* merge_bar, volatile int* abort, Shared* sh,
                                        float* scratch) {
    using C = Cfg<T, D, G, SPEC, MMA, FUSED>;
    using Engine = typename EngineOf<C, T, D, G, MMA>::type;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // -------------------------------------------------------- consumers
    const int hw = warp / C::NTW;   // which GW heads of the group
    const int tw = warp % C::NTW;   // which token slot of the round
    Engine st;
    st.reset();
    // Phase counters of the consumer-only barriers (all consumer warps run
    // the same sequence of syncs, so the counters agree across warps).
    uint32_t ph_dep = 0, ph_free = 0;
    auto sync_on = [&](uint64_t* bar, uint32_t& ph) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
        return wait_warp(bar, (ph++) & 1, abort, p, lane);
    };
    auto sync = [&]() { return sync_on(dep_bar, ph_dep); };
    const int ctid = warp * 32 + lane;
    uint32_t gt = tw;
    int b = 0, kvh = 0, chunk = 0;
    bool spec_item = SPEC;
    if (FUSED) {
        // The chunk boundary table, for the merges' per-lane lookups.
        unsigned* fq = reinterpret_cast<unsigned*>(scratch) + kMaxChunks * (G + 1) + 2 * G + 4;
        for (int i = ctid; i <= kMaxChunks; i += C::NCW * 32) fq[i] = p.fq[i];
    }
    // One-launch schedule: thread 0's head ticket still in flight (taken at
    // an item's end, looked at by the next one), and its resolution into
    // sh->merge (the head whose merges this CTA owns, or -1).
    int pend_bh = -1;
    unsigned pend_old = 0, pend_target = 0;
    auto take_head_ticket = [&](int bh, int bb, unsigned add) {
        const SeqGeom g = seq_geom(p, bb, false);
        const unsigned total = (unsigned)(cdiv(g.mid_len, C::TT) + spec_tiles(g, C::TT));
        pend_old = atom_add_acq_rel_gpu(p.ctr + ctr_head(p.B, p.Hkv, bh), add);
        pend_target = total - add;
        pend_bh = bh;
    };
    auto resolve_head_ticket = [&]() {
        int m = -1;
        if (pend_bh >= 0 && pend_old == pend_target) {
            atomicExch(p.ctr + ctr_head(p.B, p.Hkv, pend_bh), 0u);
            m = pend_bh;
        }
        pend_bh = -1;
        sh->merge = m;
    };
    if (SPEC && p.n1 > 1) {
        // Empty state (m = -inf, l = 0, o = 0) in this warp's deposit slot:
        // a CTA whose slice of a short sink set has no tiles contributes
        // nothing to the cluster merge.
        float* slot = deposit + (hw * C::NTW + tw) * C::kSlotFloats;
        for (int h = 0; h < C::GW; ++h)
            for (int e = lane; e < D + 2; e += 32) slot[h * (D + 2) + e] = e == 0 ? -INFINITY : 0.f;
        __syncwarp();
        // Every CTA of the cluster has set up its barriers once this passes
        // (long before the first tile lands).
        cluster_wait_any();
    }
    if (SPEC) {
        // The item is known up front: fetch q while the first tiles load.
        const int bh = (int)blockIdx.x / p.n1;
        chunk = (int)blockIdx.x % p.n1;
        b = bh / p.Hkv;
        kvh = bh % p.Hkv;
        st.load_query(p, b, kvh * G + hw * C::GW, lane);
    }
    for (;; gt += C::NTW) {
        const int s = gt % C::STAGES;
        if (!wait_fill(full_bar + s, fill + s, gt, (gt / C::STAGES) & 1, abort, p, lane)) break;
        const int4 mt = meta[s];
        if (mt.x < 0) break;
        if (!SPEC && mt.y < C::NTW) {
            int bh;
            item_index<SPEC, FUSED>(p, mt.x, spec_item, bh, chunk);
            b = bh / p.Hkv;
            kvh = bh % p.Hkv;
            st.load_query(p, b, kvh * G + hw * C::GW, lane);
        }
        if (mt.z > 0) {
            char* ks = reinterpret_cast<char*>(smem) + s * C::kStageBytes;
            st.tile_load(ks, ks + C::kTileBytes, mt.z, lane, p.qscale);
        }
        // The stage is released as soon as nothing more reads it (the
        // tensor-core engine holds the tile's V fragments in registers).
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar + s);
        if (mt.z > 0) st.tile_finish(mt.z, lane, p.qscale);
        if (!(mt.w & kLastTileFlag)) continue;

        // ---- end of this item: combine the warps' states into one partial.
        if (ALSPEC_IN_BOUNDS(p, (hw * C::NTW + tw + 1) * C::kSlotFloats * (int)sizeof(float) <=
                                    C::kDepositBytes))
            st.deposit(deposit + (hw * C::NTW + tw) * C::kSlotFloats, lane);
        if (SPEC && p.n1 > 1) {
            // Sink set split over a cluster: the warps' states stay in the
            // deposit slots and the cluster merge reads them directly.
            __syncwarp();
            continue;
        }
        if (FUSED && ctid == 0) resolve_head_ticket();
        if (!sync_on(dep_bar, ph_dep)) break;
        // Read before the next barrier: thread 0 rewrites it only after that.
        const int merge_bh = FUSED ? sh->merge : -1;
        {
            // The one-launch schedule keeps sink-set item partials apart.
            const bool sp = FUSED && spec_item;
            float* part_ml = sp ? p.spec_pml : p.mid_ml;
            float* part_o = sp ? p.spec_po : p.mid_o;
            const int per = SPEC || sp ? p.n1 : p.n2;
            // Partials are read back by the merge after the whole stream of
            // cache rows has gone through L2: keep them ahead of those.
            const uint64_t keep = l2_evict_last_policy();
            for (int idx = ctid; idx < G * D; idx += C::NCW * 32) {
                const int hh = idx / D;
                const int e = idx % D;
                const float* base = deposit + (hh / C::GW) * C::NTW * C::kSlotFloats +
                                    (hh % C::GW) * (D + 2);
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < C::NTW; ++w) M = fmaxf(M, base[w * C::kSlotFloats]);
                float L = 0.f, O = 0.f;
#pragma unroll
                for (int w = 0; w < C::NTW; ++w) {
                    const float* ws = base + w * C::kSlotFloats;
                    const float f = merge_weight(ws[0], M);
                    L = fmaf(f, ws[1], L);
                    O = fmaf(f, ws[2 + e], O);
                }
                const size_t bh = (size_t)b * p.Hq + kvh * G + hh;
                if (!ALSPEC_IN_BOUNDS(p, b < p.B && kvh < p.Hkv && chunk >= 0 && chunk < per))
                    continue;
                if (SPEC) {
                    // A single sink-set CTA per head holds the whole sink
                    // set: publish O_spec directly.
                    if (e == 0) {
                        st_global_hint(p.spec_ml + bh * 2, M, keep);
                        st_global_hint(p.spec_ml + bh * 2 + 1, L, keep);
                    }
                    st_global_hint(p.spec_o + bh * D + e, O, keep);
                    p.out_spec[bh * D + e] = __fdiv_rn(O, L);
                    continue;
                }
                const size_t row = bh * per + chunk;
                if (e == 0) {
                    st_global_hint(part_ml + row * 2, M, keep);
                    st_global_hint(part_ml + row * 2 + 1, L, keep);
                }
                st_global_hint(part_o + row * D + e, O, keep);
            }
        }
        // Every consumer thread's partial is written (and the deposit slots
        // are free again) once this sync passes.
        if (!sync_on(free_bar, ph_free)) break;
        if (FUSED) {
            // A head completed by this CTA's previous item: merge it now (the
            // ring is busy; rare, heads complete at the end of the queue).
            if (merge_bh >= 0 && !fused_head_merge<C, D, G>(p, merge_bh, scratch, warp, lane, sync))
                break;
            if (ctid == 0) take_head_ticket(b * p.Hkv + kvh, b, (unsigned)mt.w >> 1);
        }
        st.reset();
    }
    if (FUSED) {
        // The head ticket of this CTA's last item may be the last one.
        if (ctid == 0) resolve_head_ticket();
        if (sync()) {
            // The producer has stopped and every stage was consumed: the
            // ring is free for the merge's bulk copies.
            const int merge_bh = sh->merge;
            if (merge_bh >= 0)
                (void)fused_head_merge<C, D, G>(p, merge_bh, scratch, warp, lane, sync, smem,
                                                (size_t)C::STAGES * C::kStageBytes, merge_bar,
                                                abort);
        }
    }
}
// ------------------------------------------------------------ the kernel

template <typename T, int D, int G, bool SPEC, bool MMA, bool FUSED = false>
__global__ void __launch_bounds__(Cfg<T, D, G, SPEC, MMA, FUSED>::kThreads, 1)
    attn_kernel(const __grid_constant__ Params p) {
    using C = Cfg<T, D, G, SPEC, MMA, FUSED>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* deposit = reinterpret_cast<float*>(smem + C::kOffDeposit);
    int4* meta = reinterpret_cast<int4*>(smem + C::kOffMeta);
    uint32_t* fill = reinterpret_cast<uint32_t*>(smem + C::kOffFill);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* empty_bar = full_bar + C::STAGES;
    uint64_t* dep_bar = empty_bar + C::STAGES;  // consumer warps: phase sync
    uint64_t* free_bar = dep_bar + 1;           // consumer warps: writes done
    uint64_t* gather_bar = free_bar + 1;        // sink-set cluster leader: partials in
    uint64_t* merge_bar = gather_bar + 1;       // one-launch schedule: final merge's copies
    Shared* sh = reinterpret_cast<Shared*>(smem + C::kOffMisc);
    volatile int* abort = &sh->abort;
    float* gather = reinterpret_cast<float*>(smem + C::kOffGather);
    float* scratch = reinterpret_cast<float*>(smem + C::kOffScratch);
    // Sink-set kernel with several CTAs per head: those CTAs are one cluster.
    const bool clustered = SPEC && p.n1 > 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar + s, 1);
            mbar_init(empty_bar + s, C::NHW);
            fill[s] = 0xffffffffu;  // no tile yet
        }
        mbar_init(dep_bar, C::NCW);
        mbar_init(free_bar, C::NCW);
        mbar_init(gather_bar, 1);
        mbar_init(merge_bar, 1);
        // Every CTA of a cluster receives every CTA's slot as transaction bytes.
        if (clustered) mbar_arrive_expect_tx(gather_bar, (uint32_t)(p.n1 * C::kGatherStride * 4));
        sh->abort = 0;
        sh->merge = -1;
        fence_barrier_init();
    }
    // The producer warp fetches the tensor maps and takes its first item now,
    // so that those loads, the queue ticket and the sequence-length load
    // overlap the barrier set-up.
    const int n_items = p.B * p.Hkv * (SPEC ? p.n1 : (FUSED ? p.n1 + p.n2 : p.n2));
    int item0 = n_items;
    Item it0{};
    if (warp == C::NCW) {
        if (MMA && lane == 0) {
            prefetch_tmap(&p.tmap_k);
            prefetch_tmap(&p.tmap_v);
        }
        // The sequence lengths travel while the queue ticket does (the
        // item's sequence is known only once the ticket is back).
        const int lane_len = lane < p.B ? __ldg(p.seq_lens + lane) : 0;
        if (SPEC) {
            item0 = (int)blockIdx.x;
        } else {
            unsigned v = 0;
            if (lane == 0) v = atomicAdd(p.ctr + kCtrQueue, 1u);
            item0 = (int)__shfl_sync(0xffffffffu, v, 0);
        }
        if (item0 < n_items)
            it0 = decode_item<SPEC, C::TT, FUSED>(p, item0, lane == 0, max(lane_len, 0));
    }
    // The kernel that follows this one on its stream may be launched now
    // (when it was launched for that): after the middle kernel the merge
    // kernel, which only prepares until this grid has completed; after the
    // sink-set kernel the middle kernel's second launch, whose CTAs then
    // take each SM a sink-set CTA leaves (every sink-set CTA is resident by
    // the time all of them have passed this point).
    if (!FUSED) pdl_launch_dependents();
    __syncthreads();
    if (clustered) cluster_arrive_relaxed();  // this CTA's barriers are set up

    if (warp == C::NCW) {
        // ---------------------------------------------------- producer
        produce<T, D, G, SPEC, MMA, FUSED>(p, smem, meta, fill, full_bar, empty_bar, abort, lane,
                                           item0, it0);
        if (!clustered) return;
        cluster_wait_any();  // the cluster's barriers are set up
        __syncwarp();  // the warp waits for its producer lane, then joins the cluster merge
    } else {
        consume<T, D, G, SPEC, MMA, FUSED>(p, smem, deposit, meta, fill, full_bar, empty_bar,
                                           dep_bar, free_bar, merge_bar, abort, sh, scratch);
    }
    if (SPEC && !clustered && warp < C::NCW && p.trace) {
        // One CTA per head: its consumer warps wrote O_spec.
        __syncwarp();
        if (lane == 0) trace_publish(p, 0);
    }
    if (clustered) {
        // Every thread of the CTA is here (no early exits in this mode).
        __syncthreads();
        cluster_gather<D, G, C>(p, deposit, gather, gather_bar);
    }
    // The middle kernel, launched behind the sink-set kernel before it has
    // completed, does not complete before it: what follows on the stream
    // (the merge) may read the sink set's results.  (No-op otherwise.)
    if (!SPEC && !FUSED && threadIdx.x == 0) pdl_wait_prerequisite();
}

// ------------------------------------------------------- merge + verify

constexpr int kMergeParts = 8;   // warps per CTA, each over every 8th chunk
constexpr int kMergeBatch = 32;  // chunk loads each thread keeps in flight
constexpr int kMergeThreads = kMergeCols * kMergeParts;


// One CTA per (32 output columns of a query head, sequence): lane e of warp
// `part` owns column split * 32 + e over the chunks list[part],
// list[part + 8], ...  O_exact merges the sink-set partial with the
// sequence's non-empty middle partials; O_spec is rebuilt from the same
// sink-set partial with the same division, so the two are bit-identical when
// the middle is empty.  Each CTA's squared distance and squared norm over
// its columns are reduced in a fixed order; the CTA finishing last among a
// sequence's sums them (fixed order, fp64) and writes rel_l2 and the flag.
// Splitting a head over D / 32 CTAs spreads the partials' loads over more
// SMs: one SM pulling a head's 89 x 128 partial columns took ~2 us.
template <int D, int TT>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ Params p) {
    constexpr int NT = kMergeThreads;
    constexpr int NW = kMergeParts;
    constexpr int NS = merge_splits(D);
    const int h = (int)blockIdx.x / NS;
    const int split = (int)blockIdx.x % NS;
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int part = tid >> 5;
    const int warp = part;
    const int e = split * kMergeCols + lane;
    const size_t bh = (size_t)b * p.Hq + h;
    __shared__ int list[kMaxChunks];      // non-empty chunks, in order
    __shared__ float wts[kMaxChunks];     // their merge weights
    __shared__ float red[2][NW];
    __shared__ float accs[kMergeParts][kMergeCols];
    __shared__ int nlist;
    __shared__ int last;
    // A kernel launched programmatically after this one (the output
    // projection) may start now; it waits for this grid before it reads
    // the outputs.
    pdl_launch_dependents();

    const int mid_tiles = cdiv(seq_geom(p, b, false).mid_len, TT);
    const float2* mml = reinterpret_cast<const float2*>(p.mid_ml) + bh * p.n2;

    // Non-empty chunks, in chunk order: warp 0 tests 32 chunks at a time
    // (chunk c covers tiles [mt * fq[c] >> 24, mt * fq[c + 1] >> 24)) and
    // compacts them with a ballot (merge CTAs placed as the last middle
    // CTAs exit do this on the layer's critical path).
    if (warp == 0) {
        int count = 0;
        for (int c0 = 0; c0 < p.n2; c0 += 32) {
            const int c = c0 + lane;
            bool nonempty = false;
            if (c < p.n2) {
                const int lo = (int)(((unsigned long long)mid_tiles * p.fq[c]) >> kFracBits);
                const int hi = (int)(((unsigned long long)mid_tiles * p.fq[c + 1]) >> kFracBits);
                nonempty = hi > lo;
            }
            const unsigned m = __ballot_sync(0xffffffffu, nonempty);
            const int at = count + __popc(m & ((1u << lane) - 1u));
            if (nonempty && ALSPEC_IN_BOUNDS(p, at < kMaxChunks)) list[at] = c;
            count += __popc(m);
        }
        if (lane == 0) nlist = count;
    }
    __syncthreads();
    const int n = nlist;
#ifdef ALSPEC_DEBUG_BOUNDS
    // Every chunk of the list names a chunk of this head (a CTA-wide answer).
    if (__syncthreads_or(!(h < p.Hq && b < p.B && n >= 0 && n <= p.n2 &&
                           (tid >= n || (list[tid] >= 0 && list[tid] < p.n2))))) {
        if (tid == 0) bounds_fail(p.ctr);
        return;
    }
#endif
    // Everything above only read inputs; the partials are written by the
    // kernels this one follows, which may still be running.
    pdl_wait_prerequisite();
    // One round of independent loads: the sink-set partial, this thread's
    // chunk (m, l) (one chunk per thread: n <= kMaxChunks <= NT) and this
    // lane's column of its warp's first kMergeBatch chunks.
    static_assert(kMaxChunks <= NT, "one chunk (m, l) per thread");
    static_assert(D % kMergeCols == 0, "head size");
    const float2 sml = __ldcg(reinterpret_cast<const float2*>(p.spec_ml) + bh);
    const float os = __ldcg(p.spec_o + bh * D + e);
    const float2 cm = tid < n ? __ldcg(&mml[list[tid]]) : make_float2(-INFINITY, 0.f);
    const float* mo = p.mid_o + bh * p.n2 * D + e;
    float v[kMergeBatch];
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
        const int i = part + u * kMergeParts;
        v[u] = i < n ? __ldcg(mo + list[i] * D) : 0.f;
    }
    float M = fmaxf(sml.x, cm.x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) red[0][warp] = M;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[0][w]);
    // Weights, and the normaliser: sum of weight * l in a fixed order.
    float lsum = 0.f;
    if (tid < n) {
        const float w = merge_weight(cm.x, M);
        wts[tid] = w;
        lsum = w * cm.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    if (lane == 0) red[1][warp] = lsum;
    __syncthreads();

    // Weighted value rows, in chunk order per thread.
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
        const int i = part + u * kMergeParts;
        if (i < n) acc = fmaf(wts[i], v[u], acc);
    }
    for (int i0 = part + kMergeParts * kMergeBatch; i0 < n; i0 += kMergeParts * kMergeBatch) {
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
            const int i = i0 + u * kMergeParts;
            v[u] = i < n ? __ldcg(mo + list[i] * D) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
            const int i = i0 + u * kMergeParts;
            if (i < n) acc = fmaf(wts[i], v[u], acc);
        }
    }
    accs[part][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        const float f0 = merge_weight(sml.x, M);
        float a = f0 * os;
        float l = f0 * sml.y;
#pragma unroll
        for (int q = 0; q < kMergeParts; ++q) a += accs[q][lane];
#pragma unroll
        for (int w = 0; w < NW; ++w) l += red[1][w];
        const float o_spec = __fdiv_rn(os, sml.y);
        const float o_exact = __fdiv_rn(a, l);
        p.out_exact[bh * D + e] = o_exact;
        const float diff = o_exact - o_spec;
        float dd = diff * diff;
        float nn = o_exact * o_exact;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            dd += __shfl_xor_sync(0xffffffffu, dd, o);
            nn += __shfl_xor_sync(0xffffffffu, nn, o);
        }
        if (lane == 0) {
            *reinterpret_cast<float2*>(p.dn + (bh * NS + split) * 2) = make_float2(dd, nn);
            // Release: this CTA's (dd, nn) before the ticket; acquire: the
            // sequence's last CTA sees every CTA's.
            unsigned* word = p.ctr + ctr_seq(p.B, p.Hkv, b);
            const unsigned t = atom_add_acq_rel_gpu(word, 1u);
            last = t == (unsigned)(p.Hq * NS - 1);
            if (last) atomicExch(word, 0u);
        }
        if (__shfl_sync(0xffffffffu, lane == 0 ? last : 0, 0)) write_flag<D>(p, b, lane);
        if (lane == 0) trace_publish(p, 1);
    }
}

// ----------------------------------------- merge + verify, one cluster per sequence
//
// The same merge with one thread-block cluster of C CTAs per sequence
// (C <= 8, dividing H_q): CTA r owns query heads [r * H_q / C, (r + 1) * H_q / C),
// whose middle partials [heads][n2][d] are contiguous in the workspace and
// arrive with bulk copies into shared memory while the chunk weights are
// computed; its (squared distance, squared norm) sums go to CTA 0 of the
// cluster through distributed shared memory, which writes rel_l2 and the
// flag.  Against the 32-column merge kernel this saves the per-sequence
// ticket and the reload of the slots (two dependent global round trips).
// Used when a CTA's partials fit in shared memory.
constexpr int kCmThreads = 256;
constexpr int kCmWarps = kCmThreads / 32;
constexpr int kCmMaxHeads = 8;     // query heads per CTA at most
constexpr int kCmStatic = 16384;   // static shared memory, rounded up (for the host's budget)

template <int D, int TT>
__global__ void __launch_bounds__(kCmThreads, 1) merge_cluster_kernel(const __grid_constant__ Params p) {
    extern __shared__ unsigned char cm_raw[];
    float* blk = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(cm_raw) + 127) & ~uintptr_t(127));
    __shared__ int list[kMaxChunks];
    __shared__ float wts[kCmMaxHeads][kMaxChunks];
    __shared__ float fl[kCmMaxHeads][2];    // weight of the sink-set partial, l
    __shared__ double red[2][kCmWarps];
    __shared__ double dn_cta[2];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int nlist;
    const int C = (int)gridDim.x;
    const int rank = (int)blockIdx.x;  // the cluster spans the x dimension
    const int b = blockIdx.y;
    const int hpc = p.Hq / C;
    const int h0 = rank * hpc;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const size_t bq0 = (size_t)b * p.Hq + h0;
    static_assert(kMaxChunks <= kCmThreads, "one chunk per thread in the list scan");
    static_assert(sizeof(int) * kMaxChunks + sizeof(float) * kCmMaxHeads * (kMaxChunks + 2) +
                          sizeof(double) * (2 * kCmWarps + 2) + 8 + 4 <= kCmStatic,
                  "static shared memory");
    pdl_launch_dependents();  // as in merge_kernel

    // Inputs only: the non-empty chunks of this sequence, in order.
    if (tid == 0) {
        const int mid_tiles = cdiv(seq_geom(p, b, false).mid_len, TT);
        int count = 0, prev = 0;
#pragma unroll 8
        for (int c = 0; c < p.n2; ++c) {
            const int t = (int)(((unsigned long long)mid_tiles * p.fq[c + 1]) >> kFracBits);
            if (t > prev) list[count++] = c;
            prev = t;
        }
        nlist = count;
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    int n = nlist;
#ifdef ALSPEC_DEBUG_BOUNDS
    // Every chunk of the list names a chunk of the sequence; else no middle
    // partial is read (a CTA-wide answer; the cluster's barriers still run).
    if (__syncthreads_or(!(n >= 0 && n <= p.n2 &&
                           (tid >= n || (list[tid] >= 0 && list[tid] < p.n2))))) {
        if (tid == 0) bounds_fail(p.ctr);
        n = 0;
    }
#endif
    // The partials are written by the kernels this one follows.
    pdl_wait_prerequisite();
    const size_t bytes = (size_t)hpc * p.n2 * D * sizeof(float);
    if (warp == 0 && bytes > 0 &&
        ALSPEC_IN_BOUNDS(p, bytes + 128 <= dynamic_smem_size() &&
                                bq0 + hpc <= (size_t)p.B * p.Hq)) {
        constexpr uint32_t kPiece = 16384;
        const char* src = reinterpret_cast<const char*>(p.mid_o + bq0 * p.n2 * D);
        fence_proxy_async_global();
        if (lane == 0) mbar_arrive_expect_tx(&bar, (uint32_t)bytes);
        __syncwarp();
        const uint64_t pol = l2_evict_first_policy();
        for (size_t off = (size_t)lane * kPiece; off < bytes; off += 32 * (size_t)kPiece) {
            const uint32_t nb = (uint32_t)(bytes - off < kPiece ? bytes - off : kPiece);
            bulk_load(reinterpret_cast<unsigned char*>(blk) + off, src + off, nb, &bar, pol);
        }
    }
    // Per query head (one warp each): max, weights, normaliser, while the
    // copies land.
    for (int hh = warp; hh < hpc; hh += kCmWarps) {
        const float2 sml = __ldcg(reinterpret_cast<const float2*>(p.spec_ml) + bq0 + hh);
        const float2* ml = reinterpret_cast<const float2*>(p.mid_ml) + (bq0 + hh) * p.n2;
        float2 x[kMaxChunks / 32];
        float M = sml.x;
#pragma unroll
        for (int k = 0; k < kMaxChunks / 32; ++k) {
            const int i = lane + 32 * k;
            x[k] = i < n ? __ldcg(ml + list[i]) : make_float2(-INFINITY, 0.f);
            M = fmaxf(M, x[k].x);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float lsum = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxChunks / 32; ++k) {
            const int i = lane + 32 * k;
            if (i < n) {
                const float f = merge_weight(x[k].x, M);
                wts[hh][i] = f;
                lsum = fmaf(f, x[k].y, lsum);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
        if (lane == 0) {
            const float f0 = merge_weight(sml.x, M);
            fl[hh][0] = f0;
            fl[hh][1] = fmaf(f0, sml.y, lsum);
        }
    }
    __syncthreads();
    // The copies (bounded wait; on expiry the error bit is raised and the
    // CTA waits once more, bounded, so no copy lands after it exits).
    if (bytes > 0) {
        bool ok = true;
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(&bar, 0)) {
            if (global_ns() - t0 > p.timeout_ns) {
                ok = false;
                break;
            }
        }
        if (!ok) {
            if (tid == 0) atomicOr(p.ctr + kCtrError, kErrTimeout);
            const uint64_t t1 = global_ns();
            while (!mbar_try_wait(&bar, 0) && global_ns() - t1 < p.timeout_ns) {
            }
        }
    }
    // Columns: four interleaved sums per output (list position i goes to
    // sum i mod 4), then a fixed tree.
    double dd = 0.0, nn = 0.0;
    for (int idx = tid; idx < hpc * D; idx += kCmThreads) {
        const int hh = idx / D;
        const int e = idx % D;
        const size_t bq = bq0 + hh;
        const float os = __ldcg(p.spec_o + bq * D + e);
        const float sl = __ldcg(p.spec_ml + bq * 2 + 1);
        const float* col = blk + (size_t)hh * p.n2 * D + e;
        const float* wh = wts[hh];
        float acc[4] = {fl[hh][0] * os, 0.f, 0.f, 0.f};
        int i = 0;
        for (; i + 4 <= n; i += 4) {
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = fmaf(wh[i + k], col[(size_t)list[i + k] * D], acc[k]);
        }
#pragma unroll
        for (int k = 0; k < 3; ++k)
            if (i + k < n) acc[k] = fmaf(wh[i + k], col[(size_t)list[i + k] * D], acc[k]);
        const float a = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        const float o_exact = __fdiv_rn(a, fl[hh][1]);
        const float o_spec = __fdiv_rn(os, sl);
        if (ALSPEC_IN_BOUNDS(p, bq < (size_t)p.B * p.Hq)) p.out_exact[bq * D + e] = o_exact;
        const float diff = o_exact - o_spec;
        dd += (double)(diff * diff);
        nn += (double)(o_exact * o_exact);
    }
    // This CTA's sums (fixed order), then CTA 0 of the cluster adds the
    // CTAs' sums in rank order.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        dd += __shfl_xor_sync(0xffffffffu, dd, o);
        nn += __shfl_xor_sync(0xffffffffu, nn, o);
    }
    if (lane == 0) {
        red[0][warp] = dd;
        red[1][warp] = nn;
    }
    __syncthreads();
    if (tid == 0) {
        double s0 = 0.0, s1 = 0.0;
        for (int w = 0; w < kCmWarps; ++w) {
            s0 += red[0][w];
            s1 += red[1][w];
        }
        dn_cta[0] = s0;
        dn_cta[1] = s1;
    }
    cluster_sync();  // every CTA's sums and O_exact are written
    if (rank == 0 && tid == 0) {
        double D2 = 0.0, N2 = 0.0;
        const uint32_t local = smem_addr(dn_cta);
        for (int r = 0; r < C; ++r) {
            const uint32_t a = dsmem_addr(local, (uint32_t)r);
            double v0, v1;
            asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v0) : "r"(a) : "memory");
            asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v1) : "r"(a + 8u) : "memory");
            D2 += v0;
            N2 += v1;
        }
        double r;
        if (N2 == 0.0) {
            r = D2 == 0.0 ? 0.0 : (double)INFINITY;
        } else {
            r = sqrt(D2 / N2);
        }
        p.rel_l2[b] = (float)r;
        p.commit[b] = r <= (double)p.lambda ? 1 : 0;
    }
    cluster_sync();  // CTA 0 has read every CTA's sums
    if (rank == 0 && tid == 0) trace_publish(p, 1);
}

}  // namespace alspec
