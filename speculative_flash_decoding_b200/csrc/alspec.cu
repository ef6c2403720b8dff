// Host side of libalspec.so: argument checks, work planning, workspace
// layout, the launch schedules (the sink-set, middle and merge kernels
// chained on the caller's stream with programmatic launches, the middle
// kernel beside the sink set or after it, or one fused launch), kernel
// launches and the C ABI declared in include/alspec.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "alspec.h"
#include "attn_kernels.cuh"
#include "oproj_kernels.cuh"

namespace alspec {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSpecItems = kMaxSpecCtas;  // sink-set CTAs per (sequence, KV head)

// Share of the SMs the sink-set CTAs may take together (NUM / DEN).  More
// sink-set CTAs per head bring O_spec sooner but hold SMs the middle kernel
// would stream with: 3/4 keeps the 70B shape (32 heads, 4100-row sink set)
// at 3 CTAs per head (O_spec at 0.074 of the layer instead of 0.10, layer
// +0.7%); the whole GPU would give the 64-head ragged batch 2 CTAs per head
// (0.095 instead of 0.15) for 5% of its throughput.
#ifndef ALSPEC_SPEC_SM_SHARE_NUM
#define ALSPEC_SPEC_SM_SHARE_NUM 3
#endif
#ifndef ALSPEC_SPEC_SM_SHARE_DEN
#define ALSPEC_SPEC_SM_SHARE_DEN 4
#endif
// Sink-set tiles per CTA beyond which the automatic schedule lets the
// sink-set CTAs take every SM (see make_plan).
#ifndef ALSPEC_SPEC_TILES_WIDE
#define ALSPEC_SPEC_TILES_WIDE 24
#endif
// Smallest middle chunk of the guided self-scheduled split, in tiles, and
// the divisor of its chunk size (chunk c takes H * r_c / (DIV * P) of each
// head's middle): DIV_SINGLE for a batch of one sequence, DIV otherwise.
// Chunk boundaries are fractions of each sequence's own middle and the plan
// sees only max_seq_len, so in a batch the longest sequence's first chunks
// exceed a CTA's fair share of the real work by L_max / L_mean; DIV 1.5
// leaves room for that.  One sequence cannot be ragged, and there a first
// chunk of a whole fair share (DIV 1) means fewer items and partials:
// measured on the 32 x 128K step 2760 us against 2823 us with 1.5, while
// 1.0 cost 16% on the ragged batch of 8 (16K-64K).
#ifndef ALSPEC_GSS_MIN_TILES
#define ALSPEC_GSS_MIN_TILES 16
#endif
#ifndef ALSPEC_GSS_DIV
#define ALSPEC_GSS_DIV 1.5
#endif
#ifndef ALSPEC_GSS_DIV_SINGLE
#define ALSPEC_GSS_DIV_SINGLE 1.0
#endif
#ifndef ALSPEC_MID_SM_RESERVE
#define ALSPEC_MID_SM_RESERVE 0
#endif
// One-launch schedule: tiles per sink-set item at least (one round of the
// tensor-core kernel's consumer warps), items per head at most.
constexpr int kFusedSpecMinTiles = 4;
constexpr int kFusedSpecMaxItems = kMaxSpecItemsFused;
constexpr size_t kAlign = 256;
// SMs the middle kernel leaves free when the caller works on O_spec beside
// the exact path (spec_event, the speculative projection): a kernel of
// another stream (a transfer of O_spec, the projection) found no room on an
// SM beside a middle-kernel CTA, and with every SM holding one it ran only
// once the exact path ended (measured).
#ifndef ALSPEC_SIDE_SMS
#define ALSPEC_SIDE_SMS 2
#endif

// CTAs of the projection's bulk-copy kernel per SM (its grid).
#ifndef ALSPEC_OB_GRID_PER_SM
#define ALSPEC_OB_GRID_PER_SM 2
#endif

thread_local cudaError_t t_last_error = cudaSuccess;

// Remember the most recent failing CUDA call of this thread.
bool ok(cudaError_t e) {
    if (e != cudaSuccess) t_last_error = e;
    return e == cudaSuccess;
}

// Record an event so that, under stream capture, it becomes an event node
// whose timestamp is taken at replay; outside capture it is a plain record.
cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return e;
    return cs == cudaStreamCaptureStatusActive
               ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
               : cudaEventRecord(ev, s);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }
int round_up(int a, int b) { return ceil_div(a, b) * b; }

// Per-device library state: the lowest-priority stream, the fork/join events,
// the SM count, and which kernels already got their shared-memory attribute.
struct DeviceState {
    bool ready = false;
    cudaStream_t lo = nullptr;    // lowest priority: work on O_spec beside the exact path
    cudaEvent_t fork = nullptr;   // behind the sink-set kernel, for the lowest-priority stream
    cudaEvent_t join = nullptr;   // that stream's work of the call done
    int sm_count = 0;
    int prio_hi = 0;              // launch priority of the sink-set kernel
    std::set<const void*> attr_done;
};


std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
// One per device: a call's event records, waits and launches on the shared
// streams are enqueued as one unit, so calls from several host threads do
// not interleave their fork / join events.
std::mutex g_call_mutex[kMaxDevices];

alspec_status get_device_state(DeviceState** out) {
    int dev = 0;
    if (!ok(cudaGetDevice(&dev)) || dev < 0 || dev >= kMaxDevices) return ALSPEC_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        int lo = 0, hi = 0;
        if (!ok(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) ||
            !ok(cudaDeviceGetStreamPriorityRange(&lo, &hi)) ||
            !ok(cudaStreamCreateWithPriority(&d.lo, cudaStreamNonBlocking, lo)) ||
            !ok(cudaEventCreateWithFlags(&d.fork, cudaEventDisableTiming)) ||
            !ok(cudaEventCreateWithFlags(&d.join, cudaEventDisableTiming))) {
            return ALSPEC_ERR_CUDA;
        }
        d.prio_hi = hi;
        d.ready = true;
    }
    *out = &d;
    return ALSPEC_OK;
}

int sm_count_for_plan() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        return n;
    return 148;  // B200
}

// ------------------------------------------------------------- planning

struct Plan {
    int engine;   // ALSPEC_ENGINE_CUDA_CORES or ALSPEC_ENGINE_TENSOR_CORES
    int schedule; // ALSPEC_SCHEDULE_STREAMS or ALSPEC_SCHEDULE_FUSED
    int tt;       // tokens per pipeline tile of that engine
    int c1, n1;   // sink-set tokens per item and items per (sequence, KV head): CTAs of
                  // one cluster (STREAMS), queue items (FUSED)
    int c2, n2;   // first middle chunk (tokens, longest sequence) and chunks per head
    unsigned fq[kMaxChunks + 1];
    int grid1, grid2;
    bool sink_first;  // SINK_FIRST: the sink-set kernel alone first, then the middle kernel
    int merge_c;      // CTAs per sequence (one cluster) of the cluster merge; 0: the
                      // 32-column merge kernel
    int merge_smem;   // its dynamic shared memory
    int threads, smem, stages;
    size_t off_ctr, off_spec_ml, off_spec_o, off_spec_pml, off_spec_po, off_mid_ml, off_mid_o,
        off_dn, total;
};

bool supported_g(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

int resolve_schedule(const alspec_desc* d) {
    return d->schedule == ALSPEC_SCHEDULE_AUTO ? ALSPEC_SCHEDULE_STREAMS : d->schedule;
}

int resolve_engine(const alspec_desc* d) {
    if (d->engine == ALSPEC_ENGINE_AUTO)
        return d->dtype == ALSPEC_BF16 ? ALSPEC_ENGINE_TENSOR_CORES : ALSPEC_ENGINE_CUDA_CORES;
    return d->engine;
}

alspec_status check_desc(const alspec_desc* d, int S, int W) {
    if (!d) return ALSPEC_ERR_INVALID_ARG;
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->max_seq_len < 1 ||
        d->head_dim < 1 || d->n_q_heads % d->n_kv_heads != 0 || S < 0 || W < 0 ||
        (long long)S + W < 1 || d->split_tokens < 0 || d->timeout_ms < 0)
        return ALSPEC_ERR_INVALID_ARG;
    if (d->dtype != ALSPEC_F32 && d->dtype != ALSPEC_BF16) return ALSPEC_ERR_INVALID_ARG;
    if (d->engine < ALSPEC_ENGINE_AUTO || d->engine > ALSPEC_ENGINE_TENSOR_CORES)
        return ALSPEC_ERR_INVALID_ARG;
    if (d->schedule < ALSPEC_SCHEDULE_AUTO || d->schedule > ALSPEC_SCHEDULE_SINK_FIRST)
        return ALSPEC_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return ALSPEC_ERR_UNSUPPORTED;
    if (!supported_g(d->n_q_heads / d->n_kv_heads)) return ALSPEC_ERR_UNSUPPORTED;
    if (resolve_engine(d) == ALSPEC_ENGINE_TENSOR_CORES && d->dtype != ALSPEC_BF16)
        return ALSPEC_ERR_UNSUPPORTED;
    // Row indices (TMA coordinates, item arithmetic) are 32-bit.
    const long long rows = (long long)d->batch * d->n_kv_heads * d->max_seq_len;
    if (rows >= (1ll << 31) || (long long)d->batch * d->n_kv_heads > (1 << 20))
        return ALSPEC_ERR_UNSUPPORTED;
    return ALSPEC_OK;
}

void kernel_shape(int dtype, int D, int G, int engine, bool fused, int* threads, int* smem,
                  int* stages);

// Item sizes.  The sink-set list (at most S + W tokens per head, tiled as a
// sink run and a window run) is cut into n1 items of about
// ALSPEC_SPEC_TILES tiles, one CTA each, the n1 CTAs of a head forming one
// thread-block cluster (n1 <= 8, the portable cluster size), with all heads
// together within ALSPEC_SPEC_SM_SHARE of the SMs; n1 = 1 needs no
// cross-CTA merge.  The persistent middle kernel takes every SM: its CTAs
// that find an SM busy with the (short) sink-set kernel start when it is
// done, and its atomic queue balances the work.
// Middle chunks follow guided self-scheduling: with H heads sharing each
// chunk index and P CTAs, chunk c takes H * r_c / (DIV P) of what is left
// of a head's middle (r_c), never less than 16 tiles; chunk boundaries are
// fractions of each sequence's own middle, so ragged batches get the same
// number of (proportionally smaller) items.  A caller-given split_tokens
// instead cuts the longest middle into equal chunks of that size.
// The one-launch schedule cuts each sink set into items of at least
// kFusedSpecMinTiles tiles, as many per head as one CTA each in the first
// wave allows; they precede the middle chunks in the same queue.
void make_plan(const alspec_desc& d, int S, int W, int sms, Plan* pl) {
    pl->engine = resolve_engine(&d);
    pl->schedule = resolve_schedule(&d);
    const bool fused = pl->schedule == ALSPEC_SCHEDULE_FUSED;
    const int TT = pl->engine == ALSPEC_ENGINE_TENSOR_CORES ? 32 : 16;
    pl->tt = TT;
    const int heads = d.batch * d.n_kv_heads;
    const int L = d.max_seq_len;
    const int tiles_max = ceil_div(std::min(S, L), TT) + ceil_div(std::min(W, L), TT);
    // CTAs per head for the sink set (one thread-block cluster): about
    // ALSPEC_SPEC_TILES tiles each, at most 8 (the portable cluster size),
    // and all heads together within ALSPEC_SPEC_SM_SHARE of the SMs.
    // SINK_FIRST: the sink-set kernel runs alone, so it may take every SM.
    pl->sink_first = pl->schedule == ALSPEC_SCHEDULE_SINK_FIRST;
    auto sink_ctas = [&](int share) {
        const int room = std::max(1, share / std::max(1, heads));
        return std::max(1, std::min({kMaxSpecItems, room, ceil_div(tiles_max, ALSPEC_SPEC_TILES)}));
    };
    const int share_sms = pl->sink_first
                              ? sms
                              : sms * ALSPEC_SPEC_SM_SHARE_NUM / ALSPEC_SPEC_SM_SHARE_DEN;
    pl->n1 = sink_ctas(share_sms);
    // The automatic schedule aims at O_spec within a tenth of the layer:
    // when that share leaves each sink-set CTA more than
    // ALSPEC_SPEC_TILES_WIDE tiles (many sequences or a long window), the
    // sink-set CTAs may take every SM.  Measured: the ragged batch of 8
    // (64 heads, 65 tiles each) O_spec 27.9 -> 17.2 us, 0.150 -> 0.087 of
    // the layer, for 1.6% of its step; the 70B batch of 4 (32 heads, 129
    // tiles) 0.071 -> 0.061 for 0.3%.  An explicit STREAMS keeps the share.
    if (d.schedule == ALSPEC_SCHEDULE_AUTO &&
        ceil_div(tiles_max, pl->n1) > ALSPEC_SPEC_TILES_WIDE)
        pl->n1 = sink_ctas(sms);
    if (fused)
        pl->n1 = std::max(1, std::min({kFusedSpecMaxItems, ceil_div(tiles_max, kFusedSpecMinTiles),
                                       std::max(1, sms / std::max(1, heads))}));
    const int tiles_per_item = ceil_div(tiles_max, pl->n1);
    pl->c1 = tiles_per_item * TT;
    pl->n1 = ceil_div(tiles_max, tiles_per_item);  // no CTA without tiles at L_max
    pl->grid1 = heads * pl->n1;

    const int ns = std::min(S, L);
    const int mid_max = std::max(0, std::max(ns, L - W) - ns);
    const int mid_tiles = ceil_div(mid_max, TT);
    // The persistent middle kernel takes every SM (less ALSPEC_MID_SM_RESERVE):
    // CTAs that find an SM busy with the (short) sink-set kernel start when
    // it is done, and the atomic queue balances the work.
    const int P = std::max(1, sms - ALSPEC_MID_SM_RESERVE);
    std::vector<double> sizes;  // chunk sizes as fractions of a head's middle
    if (mid_tiles > 0) {
        if (d.split_tokens > 0) {
            const int ct = std::max(1, ceil_div(round_up(d.split_tokens, TT), TT));
            const int n = std::min(kMaxChunks, ceil_div(mid_tiles, ct));
            for (int c = 0; c < n; ++c) sizes.push_back((double)ct / mid_tiles);
        } else {
            const double smin = std::min(1.0, (double)ALSPEC_GSS_MIN_TILES / mid_tiles);
            const double div = d.batch == 1 ? ALSPEC_GSS_DIV_SINGLE : ALSPEC_GSS_DIV;
            double r = 1.0;
            while (r > 1e-9 && (int)sizes.size() < kMaxChunks) {
                double s = std::max((double)heads * r / (div * P), smin);
                s = std::min(s, r);
                sizes.push_back(s);
                r -= s;
            }
        }
    }
    pl->n2 = (int)sizes.size();
    const double scale = (double)(1u << kFracBits);
    double acc = 0.0;
    pl->fq[0] = 0;
    for (int c = 0; c < pl->n2; ++c) {
        acc += sizes[c];
        // Rounded up, so that the longest sequence gets its boundaries at
        // exactly the intended tiles.
        pl->fq[c + 1] = c + 1 == pl->n2 ? (1u << kFracBits)
                                         : (unsigned)std::min(scale, std::ceil(acc * scale - 1e-6));
        pl->fq[c + 1] = std::max(pl->fq[c + 1], pl->fq[c]);
    }
    for (int c = pl->n2 + 1; c <= kMaxChunks; ++c) pl->fq[c] = 1u << kFracBits;
    pl->c2 = pl->n2 > 0
                 ? (int)(((unsigned long long)mid_tiles * pl->fq[1]) >> kFracBits) * TT
                 : 0;
    // Merge: the 32-column merge kernel (B * H_q * d / 32 CTAs) while it
    // fits in one wave of CTAs; beyond that one cluster of C CTAs per
    // sequence, when a CTA's middle partials ([H_q / C][n2][d] fp32) fit in
    // shared memory, C the largest of 8, 4, 2, 1 dividing H_q with at most
    // kCmMaxHeads heads per CTA.  Measured (same box): the batch of 8
    // ragged sequences 805.7 -> 758.8 us per 4 layers, the 70B batch of 4
    // 1299 -> 1255 us; one 128K sequence 2758 -> 2812 us per 32 layers,
    // where the 128 small CTAs spread the loads over more SMs.
    pl->merge_c = 0;
    pl->merge_smem = 0;
    const bool one_wave =
        (long long)d.batch * d.n_q_heads * merge_splits(d.head_dim) <= (long long)sms;
    for (int c : {8, 4, 2, 1}) {
        if (fused || one_wave) break;
        if (d.n_q_heads % c != 0 || d.n_q_heads / c > kCmMaxHeads) continue;
        const long long bytes =
            (long long)(d.n_q_heads / c) * std::max(pl->n2, 0) * d.head_dim * 4 + 128;
        if (bytes <= kSmemLimit - kCmStatic) {
            pl->merge_c = c;
            pl->merge_smem = (int)bytes;
        }
        break;
    }
    const long long items2 = (long long)heads * (pl->n2 + (fused ? pl->n1 : 0));
    pl->grid2 = (int)std::min<long long>(P, items2);

    const int G = d.n_q_heads / d.n_kv_heads;
    kernel_shape(d.dtype, d.head_dim, G, pl->engine, fused, &pl->threads, &pl->smem, &pl->stages);

    const size_t B = d.batch, Hq = d.n_q_heads, D = d.head_dim;
    const size_t n2 = std::max(pl->n2, 1);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, kAlign);
        return o;
    };
    pl->off_ctr = take((size_t)ctr_words(d.batch, d.n_kv_heads) * sizeof(unsigned));
    pl->off_spec_ml = take(B * Hq * 2 * sizeof(float));
    pl->off_spec_o = take(B * Hq * D * sizeof(float));
    const size_t n1p = fused ? (size_t)pl->n1 : 0;
    pl->off_spec_pml = take(B * Hq * n1p * 2 * sizeof(float));
    pl->off_spec_po = take(B * Hq * n1p * D * sizeof(float));
    pl->off_mid_ml = take(B * Hq * n2 * 2 * sizeof(float));
    pl->off_mid_o = take(B * Hq * n2 * D * sizeof(float));
    pl->off_dn = take(B * Hq * merge_splits(D) * 2 * sizeof(float));
    pl->total = off;
}

// ------------------------------------------------------------- dispatch

using KernelFn = void (*)(Params);

struct KernelSet {
    KernelFn spec;
    KernelFn mid;
    KernelFn fused;  // the one-launch schedule's kernel
    int smem_spec, smem_mid, smem_fused;
    int threads_spec, threads_mid, threads_fused;
    int stages_mid, stages_fused;
};

template <typename T, int D, int G, bool MMA>
KernelSet kernels_for() {
    using CS = Cfg<T, D, G, true, MMA>;
    using CM = Cfg<T, D, G, false, MMA>;
    using CF = Cfg<T, D, G, false, MMA, true>;
    return KernelSet{attn_kernel<T, D, G, true, MMA>,
                     attn_kernel<T, D, G, false, MMA>,
                     attn_kernel<T, D, G, false, MMA, true>,
                     CS::kSmemBytes,
                     CM::kSmemBytes,
                     CF::kSmemBytes,
                     CS::kThreads,
                     CM::kThreads,
                     CF::kThreads,
                     CM::STAGES,
                     CF::STAGES};
}

template <typename T, int D, bool MMA>
bool pick_g(int G, KernelSet* ks) {
    switch (G) {
    case 1: *ks = kernels_for<T, D, 1, MMA>(); return true;
    case 2: *ks = kernels_for<T, D, 2, MMA>(); return true;
    case 4: *ks = kernels_for<T, D, 4, MMA>(); return true;
    case 8: *ks = kernels_for<T, D, 8, MMA>(); return true;
    default: return false;
    }
}

bool pick(int dtype, int D, int G, int engine, KernelSet* ks) {
    const bool mma = engine == ALSPEC_ENGINE_TENSOR_CORES;
    if (dtype == ALSPEC_BF16) {
        if (mma) {
            if (D == 128) return pick_g<__nv_bfloat16, 128, true>(G, ks);
            if (D == 64) return pick_g<__nv_bfloat16, 64, true>(G, ks);
        } else {
            if (D == 128) return pick_g<__nv_bfloat16, 128, false>(G, ks);
            if (D == 64) return pick_g<__nv_bfloat16, 64, false>(G, ks);
        }
    } else if (dtype == ALSPEC_F32 && !mma) {
        if (D == 128) return pick_g<float, 128, false>(G, ks);
        if (D == 64) return pick_g<float, 64, false>(G, ks);
    }
    return false;
}

void kernel_shape(int dtype, int D, int G, int engine, bool fused, int* threads, int* smem,
                  int* stages) {
    KernelSet ks{};
    const bool found = pick(dtype, D, G, engine, &ks);
    *threads = found ? (fused ? ks.threads_fused : ks.threads_mid) : 0;
    *smem = found ? (fused ? ks.smem_fused : ks.smem_mid) : 0;
    *stages = found ? (fused ? ks.stages_fused : ks.stages_mid) : 0;
}

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

alspec_status encode_kv_map(CUtensorMap* map, const void* base, const alspec_desc& d) {
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q{};
            void* fn = nullptr;
            if (!ok(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q)) ||
                q != cudaDriverEntryPointSuccess || !fn)
                return ALSPEC_ERR_CUDA;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    // A 2-D view of the cache: rows = (b, kv head, token), d columns; boxes of
    // 64 columns (128 bytes) x 32 rows with 128-byte swizzle.
    const cuuint64_t rows = (cuuint64_t)d.batch * d.n_kv_heads * d.max_seq_len;
    const cuuint64_t dims[2] = {(cuuint64_t)d.head_dim, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d.head_dim * 2};
    const cuuint32_t box[2] = {64, 32};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ALSPEC_OK : ALSPEC_ERR_INVALID_ARG;
}

alspec_status ensure_smem_attr(DeviceState* ds, const void* key, int bytes) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (ds->attr_done.count(key)) return ALSPEC_OK;
    if (!ok(cudaFuncSetAttribute(key, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)))
        return ALSPEC_ERR_CUDA;
    ds->attr_done.insert(key);
    return ALSPEC_OK;
}

enum LaunchFlags { kLaunchHighPriority = 1, kLaunchProgrammatic = 2 };

alspec_status launch(KernelFn fn, dim3 grid, dim3 block, int smem, cudaStream_t stream,
                     const Params& p, int flags, int prio, int cluster = 1) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[3];
    int n = 0;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (flags & kLaunchHighPriority) {
        attr[n].id = cudaLaunchAttributePriority;
        attr[n].val.priority = prio;
        ++n;
    }
    if (flags & kLaunchProgrammatic) {
        // May start before the preceding kernel in the stream completes; the
        // kernel waits for it (griddepcontrol.wait) before using its output.
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = n ? attr : nullptr;
    cfg.numAttrs = n;
    return ok(cudaLaunchKernelEx(&cfg, fn, p)) ? ALSPEC_OK : ALSPEC_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Forget the no-alloc scratch addresses looked up so far (alspec_shutdown).
void noalloc_forget();

}  // namespace
}  // namespace alspec

using namespace alspec;

extern "C" {

size_t alspec_workspace_size(const alspec_desc* desc, int n_sink, int window) {
    if (check_desc(desc, n_sink, window) != ALSPEC_OK) return 0;
    Plan pl{};
    make_plan(*desc, n_sink, window, sm_count_for_plan(), &pl);
    return pl.total;
}

alspec_status alspec_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes == 0) return ALSPEC_ERR_INVALID_ARG;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? ALSPEC_OK
               : ALSPEC_ERR_CUDA;
}

alspec_status alspec_query_plan(const alspec_desc* desc, int n_sink, int window, int* info,
                                int n_info) {
    const alspec_status st = check_desc(desc, n_sink, window);
    if (st != ALSPEC_OK) return st;
    if (!info || n_info < 0) return ALSPEC_ERR_INVALID_ARG;
    Plan pl{};
    make_plan(*desc, n_sink, window, sm_count_for_plan(), &pl);
    const int vals[12] = {pl.c1,   pl.n1,     pl.c2,     pl.n2,       pl.grid2,   pl.threads,
                          pl.smem, pl.stages, pl.engine, pl.schedule, pl.merge_c, pl.grid1};
    for (int i = 0; i < n_info && i < 12; ++i) info[i] = vals[i];
    return ALSPEC_OK;
}

alspec_status alspec_query_chunks(const alspec_desc* desc, int n_sink, int window, uint32_t* fq,
                                  int capacity, int* n2, int* tile) {
    const alspec_status st = check_desc(desc, n_sink, window);
    if (st != ALSPEC_OK) return st;
    if (!fq || !n2 || !tile) return ALSPEC_ERR_INVALID_ARG;
    Plan pl{};
    make_plan(*desc, n_sink, window, sm_count_for_plan(), &pl);
    if (capacity < pl.n2 + 1) return ALSPEC_ERR_INVALID_ARG;
    for (int c = 0; c <= pl.n2; ++c) fq[c] = pl.fq[c];
    *n2 = pl.n2;
    *tile = pl.tt;
    return ALSPEC_OK;
}

}  // extern "C"

namespace alspec {
namespace {

// The output projection that follows attention, run speculatively on O_spec
// and redone on O_exact for discarded tokens (alspec_decode_oproj).
struct OprojReq {
    const void* w;  // bf16 [hidden][Hq * d]
    int hidden;
    float* y;       // fp32 [B][hidden]
    int gate;       // alspec_gate
};

bool oproj_args_ok(const float* x, const void* w, const float* y, int batch, int k, int n) {
    return x && w && y && batch >= 1 && batch <= kOprojMaxB && k >= 8 && k % 8 == 0 && n >= 1 &&
           aligned16(x) && aligned16(w) && (reinterpret_cast<uintptr_t>(y) & 3u) == 0;
}

OprojParams oproj_params(const float* x, const void* w, float* y, const uint8_t* skip, int batch,
                         int k, int n, unsigned long long* trace, unsigned* err = nullptr,
                         unsigned long long timeout_ns = 2000000000ull) {
    OprojParams o{};
    o.err = err;
    o.timeout_ns = timeout_ns;
    o.x = x;
    o.w = static_cast<const uint4*>(w);
    o.y = y;
    o.skip = skip;
    o.B = batch;
    o.K = k;
    o.N = n;
    o.trace = trace;
    return o;
}

dim3 oproj_grid(int n) { return dim3((unsigned)ceil_div(n, kOprojWarps)); }

// Foreground projection: the bulk-copy kernel, ALSPEC_OB_GRID_PER_SM CTAs
// per SM (at most one per output row).
alspec_status launch_oproj_bulk(DeviceState* ds, const OprojParams& o, cudaStream_t s) {
    const OprojFn fn = oproj_bulk_kernel_for(o.B);
    alspec_status st = ensure_smem_attr(ds, reinterpret_cast<const void*>(fn), kObSmem);
    if (st != ALSPEC_OK) return st;
    // Programmatic: the weights start streaming while the kernel ahead on
    // the stream finishes (its SMs free up one by one).
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)std::min(ALSPEC_OB_GRID_PER_SM * ds->sm_count, o.N));
    cfg.blockDim = dim3(kObThreads);
    cfg.dynamicSmemBytes = kObSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return ok(cudaLaunchKernelEx(&cfg, fn, o)) ? ALSPEC_OK : ALSPEC_ERR_CUDA;
}

alspec_status decode_impl(const alspec_desc* desc, const void* q, const void* k_cache,
                          const void* v_cache, const int32_t* seq_lens, int n_sink, int window,
                          float lambda, float* out_spec, float* out_exact, float* rel_l2,
                          uint8_t* commit, void* workspace, size_t workspace_bytes, void* stream,
                          void* spec_event, void* const* prof_events,
                          unsigned long long* trace_ns, const OprojReq* op = nullptr,
                          bool clear_counters = false) {
    alspec_status st = check_desc(desc, n_sink, window);
    if (st != ALSPEC_OK) return st;
    if (reinterpret_cast<uintptr_t>(trace_ns) & 7u) return ALSPEC_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seq_lens || !out_spec || !out_exact || !rel_l2 || !commit)
        return ALSPEC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return ALSPEC_ERR_INVALID_ARG;
    if (!(lambda >= 0.f) || std::isinf(lambda)) return ALSPEC_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return ALSPEC_ERR_WORKSPACE;

    Plan pl{};
    make_plan(*desc, n_sink, window, sm_count_for_plan(), &pl);
    if (workspace_bytes < pl.total) return ALSPEC_ERR_WORKSPACE;
    const bool fused = pl.schedule == ALSPEC_SCHEDULE_FUSED;
    // The speculative projection needs O_spec before the launch ends.
    if (fused && op) return ALSPEC_ERR_UNSUPPORTED;
    DeviceState* ds = nullptr;
    if ((st = get_device_state(&ds)) != ALSPEC_OK) return st;
    std::lock_guard<std::mutex> call_lock(g_call_mutex[ds - g_dev]);
    const int G = desc->n_q_heads / desc->n_kv_heads;
    KernelSet ks{};
    if (!pick(desc->dtype, desc->head_dim, G, pl.engine, &ks)) return ALSPEC_ERR_UNSUPPORTED;
    if (fused) {
        if ((st = ensure_smem_attr(ds, reinterpret_cast<const void*>(ks.fused), ks.smem_fused)) !=
            ALSPEC_OK)
            return st;
    } else {
        if ((st = ensure_smem_attr(ds, reinterpret_cast<const void*>(ks.spec), ks.smem_spec)) !=
            ALSPEC_OK)
            return st;
        if ((st = ensure_smem_attr(ds, reinterpret_cast<const void*>(ks.mid), ks.smem_mid)) !=
            ALSPEC_OK)
            return st;
    }

    char* ws = static_cast<char*>(workspace);
    Params p{};
    if (pl.engine == ALSPEC_ENGINE_TENSOR_CORES) {
        if ((st = encode_kv_map(&p.tmap_k, k_cache, *desc)) != ALSPEC_OK) return st;
        if ((st = encode_kv_map(&p.tmap_v, v_cache, *desc)) != ALSPEC_OK) return st;
    }
    p.q = q;
    p.k = k_cache;
    p.v = v_cache;
    p.seq_lens = seq_lens;
    p.B = desc->batch;
    p.Hq = desc->n_q_heads;
    p.Hkv = desc->n_kv_heads;
    p.Lmax = desc->max_seq_len;
    p.S = n_sink;
    p.W = window;
    p.qscale = (float)(1.4426950408889634 / std::sqrt((double)desc->head_dim));
    p.lambda = lambda;
    p.c1 = pl.c1;
    p.n1 = pl.n1;
    p.n2 = pl.n2;
    p.mid_ctas = pl.grid2;
    std::memcpy(p.fq, pl.fq, sizeof p.fq);
    p.ctr = reinterpret_cast<unsigned*>(ws + pl.off_ctr);
    p.spec_ml = reinterpret_cast<float*>(ws + pl.off_spec_ml);
    p.spec_o = reinterpret_cast<float*>(ws + pl.off_spec_o);
    p.spec_pml = reinterpret_cast<float*>(ws + pl.off_spec_pml);
    p.spec_po = reinterpret_cast<float*>(ws + pl.off_spec_po);
    p.mid_ml = reinterpret_cast<float*>(ws + pl.off_mid_ml);
    p.mid_o = reinterpret_cast<float*>(ws + pl.off_mid_o);
    p.dn = reinterpret_cast<float*>(ws + pl.off_dn);
    p.out_spec = out_spec;
    p.out_exact = out_exact;
    p.trace = trace_ns;
    p.rel_l2 = rel_l2;
    p.commit = commit;
    p.timeout_ns = (unsigned long long)(desc->timeout_ms > 0 ? desc->timeout_ms : 2000) * 1000000ull;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // A workspace that is not the caller's own (alspec_decode_noalloc's
    // shared scratch) gets its counters cleared first, once every check has
    // passed, so that a rejected call leaves nothing queued.
    if (clear_counters &&
        !ok(cudaMemsetAsync(p.ctr, 0, (size_t)ctr_words(desc->batch, desc->n_kv_heads) *
                                          sizeof(unsigned), s)))
        return ALSPEC_ERR_CUDA;
    auto prof = [&](int i, cudaStream_t on) {
        return !prof_events || !prof_events[i] ||
               ok(record_event(static_cast<cudaEvent_t>(prof_events[i]), on));
    };
    if (!prof(0, s)) return ALSPEC_ERR_CUDA;
    if (fused) {
        // One persistent launch; O_spec is complete (as everything else)
        // when it ends.
        if (!prof(2, s)) return ALSPEC_ERR_CUDA;
        if ((st = launch(ks.fused, dim3(pl.grid2), dim3(ks.threads_fused), ks.smem_fused, s, p, 0,
                         0)) != ALSPEC_OK)
            return st;
        if (!prof(3, s) || !prof(1, s)) return ALSPEC_ERR_CUDA;
        if (spec_event && !ok(record_event(static_cast<cudaEvent_t>(spec_event), s)))
            return ALSPEC_ERR_CUDA;
        return prof(4, s) ? ALSPEC_OK : ALSPEC_ERR_CUDA;
    }
    // The three kernels run in order on the caller's stream.  The sink-set
    // kernel goes first, at high launch priority; each of its CTAs lets the
    // middle kernel launch as soon as it starts, so the middle kernel is
    // released once every sink-set CTA (and thread-block cluster) is
    // resident: its persistent CTAs take the SMs left over at once and each
    // SM a sink-set CTA frees -- the sink set always finds its SMs, and
    // nothing waits for it to complete.  (SINK_FIRST: the middle kernel
    // starts after it completes.)  The merge kernel follows the middle one
    // the same way.
    //
    // Work on O_spec elsewhere (spec_event, the speculative projection) runs
    // on the library's lowest-priority stream, after an event recorded
    // right behind the sink-set kernel: under stream capture that record is
    // not a node, only the sink-set kernel's dependency handed to the other
    // stream, so the programmatic edge to the middle kernel stays.  The
    // caller's stream joins that stream at the end of the call.
    const bool side = spec_event != nullptr || op != nullptr;
    const int kdim = desc->n_q_heads * desc->head_dim;
    const dim3 grid1(pl.grid1);
    if ((st = launch(ks.spec, grid1, dim3(ks.threads_spec), ks.smem_spec, s, p,
                     kLaunchHighPriority, ds->prio_hi, pl.n1)) != ALSPEC_OK)
        return st;
    if (side) {
        cudaStream_t lo = ds->lo;
        if (!ok(cudaEventRecord(ds->fork, s)) || !ok(cudaStreamWaitEvent(lo, ds->fork, 0)))
            return ALSPEC_ERR_CUDA;
        if (spec_event && !ok(record_event(static_cast<cudaEvent_t>(spec_event), lo)))
            return ALSPEC_ERR_CUDA;
        if (op) {
            // Speculative output projection of O_spec, beside the exact
            // path: a kernel without shared memory, so it fits beside the
            // middle kernel's CTAs, whose work comes first.
            const OprojParams o = oproj_params(out_spec, op->w, op->y, nullptr, desc->batch, kdim,
                                               op->hidden, trace_ns ? trace_ns + 2 : nullptr,
                                               p.ctr + kCtrError, p.timeout_ns);
            oproj_kernel_for(o.B)<<<oproj_grid(op->hidden), kOprojWarps * 32, 0, lo>>>(o);
            if (!ok(cudaGetLastError())) return ALSPEC_ERR_CUDA;
        }
        if (!ok(cudaEventRecord(ds->join, lo))) return ALSPEC_ERR_CUDA;
    }
    // Profiling events between the kernels take away their overlap: the
    // middle kernel then starts once the sink set has completed.
    if (!prof(1, s) || !prof(2, s)) return ALSPEC_ERR_CUDA;
    if (pl.n2 > 0) {
        const int flags = pl.sink_first || prof_events ? 0 : kLaunchProgrammatic;
        Params pm = p;
        if (side && pl.grid2 > ALSPEC_SIDE_SMS) pm.mid_ctas = pl.grid2 - ALSPEC_SIDE_SMS;
        if ((st = launch(ks.mid, dim3(pm.mid_ctas), dim3(ks.threads_mid), ks.smem_mid, s, pm,
                         flags, 0)) != ALSPEC_OK)
            return st;
    }
    if (!prof(3, s)) return ALSPEC_ERR_CUDA;
    KernelFn mk = nullptr;
    if (pl.merge_c > 0) {
        if (desc->head_dim == 128)
            mk = pl.tt == 32 ? merge_cluster_kernel<128, 32> : merge_cluster_kernel<128, 16>;
        else
            mk = pl.tt == 32 ? merge_cluster_kernel<64, 32> : merge_cluster_kernel<64, 16>;
        if ((st = ensure_smem_attr(ds, reinterpret_cast<const void*>(mk),
                                   kSmemLimit - kCmStatic)) != ALSPEC_OK)
            return st;
    } else if (desc->head_dim == 128) {
        mk = pl.tt == 32 ? merge_kernel<128, 32> : merge_kernel<128, 16>;
    } else {
        mk = pl.tt == 32 ? merge_kernel<64, 32> : merge_kernel<64, 16>;
    }
    // With ALSPEC_GATE_GRAPH_CONDITIONAL, inside a stream capture the
    // recomputation of discarded tokens' output projection is a conditional
    // node, enabled by a one-warp kernel that reads the flags.
    bool capturing = false;
    cudaGraphConditionalHandle cond = 0;
    if (op && op->gate == ALSPEC_GATE_GRAPH_CONDITIONAL) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaGraph_t cg = nullptr;
        if (!ok(cudaStreamGetCaptureInfo(s, &cs, nullptr, &cg, nullptr, nullptr)))
            return ALSPEC_ERR_CUDA;
        capturing = cs == cudaStreamCaptureStatusActive;
        if (capturing &&
            !ok(cudaGraphConditionalHandleCreate(&cond, cg, 0, cudaGraphCondAssignDefault)))
            return ALSPEC_ERR_CUDA;
    }
    // Programmatic launch right behind the middle kernel (or the sink-set
    // kernel, with no middle), unless a profiling event sits between them.
    const bool pdl = !prof_events;
    if (pl.merge_c > 0) {
        if ((st = launch(mk, dim3(pl.merge_c, desc->batch), dim3(kCmThreads), pl.merge_smem, s, p,
                         pdl ? kLaunchProgrammatic : 0, 0, pl.merge_c)) != ALSPEC_OK)
            return st;
    } else if ((st = launch(mk, dim3(desc->n_q_heads * merge_splits(desc->head_dim), desc->batch),
                            dim3(kMergeThreads), 0, s, p, pdl ? kLaunchProgrammatic : 0, 0)) !=
               ALSPEC_OK) {
        return st;
    }
    // The side stream's work on O_spec belongs to this call.
    if (side && !ok(cudaStreamWaitEvent(s, ds->join, 0))) return ALSPEC_ERR_CUDA;
    if (op) {
        // Redo the projection on O_exact for the discarded tokens, after the
        // speculative one (both write y).
        OprojParams r = oproj_params(out_exact, op->w, op->y, commit, desc->batch, kdim,
                                     op->hidden, trace_ns ? trace_ns + 2 : nullptr,
                                     p.ctr + kCtrError, p.timeout_ns);
        const OprojFn rfn = oproj_bulk_kernel_for(r.B);
        if ((st = ensure_smem_attr(ds, reinterpret_cast<const void*>(rfn), kObSmem)) != ALSPEC_OK)
            return st;
        if (capturing) {
            set_discard_condition<<<1, 32, 0, s>>>(commit, desc->batch, cond);
            if (!ok(cudaGetLastError())) return ALSPEC_ERR_CUDA;
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            cudaGraph_t g = nullptr;
            const cudaGraphNode_t* deps = nullptr;
            size_t ndeps = 0;
            if (!ok(cudaStreamGetCaptureInfo(s, &cs, nullptr, &g, &deps, &ndeps)))
                return ALSPEC_ERR_CUDA;
            cudaGraphNodeParams cp{};
            cp.type = cudaGraphNodeTypeConditional;
            cp.conditional.handle = cond;
            cp.conditional.type = cudaGraphCondTypeIf;
            cp.conditional.size = 1;
            cudaGraphNode_t cn = nullptr;
            if (!ok(cudaGraphAddNode(&cn, g, deps, ndeps, &cp))) return ALSPEC_ERR_CUDA;
            cudaGraphNodeParams kp{};
            kp.type = cudaGraphNodeTypeKernel;
            kp.kernel.func = reinterpret_cast<void*>(rfn);
            kp.kernel.gridDim =
                dim3((unsigned)std::min(ALSPEC_OB_GRID_PER_SM * ds->sm_count, op->hidden));
            kp.kernel.blockDim = dim3(kObThreads);
            kp.kernel.sharedMemBytes = kObSmem;
            void* args[] = {&r};
            kp.kernel.kernelParams = args;
            cudaGraphNode_t kn = nullptr;
            if (!ok(cudaGraphAddNode(&kn, cp.conditional.phGraph_out[0], nullptr, 0, &kp)) ||
                !ok(cudaStreamUpdateCaptureDependencies(s, &cn, 1,
                                                        cudaStreamSetCaptureDependencies)))
                return ALSPEC_ERR_CUDA;
        } else {
            if ((st = launch_oproj_bulk(ds, r, s)) != ALSPEC_OK) return st;
        }
    }
    if (!prof(4, s)) return ALSPEC_ERR_CUDA;
    return ALSPEC_OK;
}

}  // namespace
}  // namespace alspec

extern "C" {

alspec_status alspec_decode(const alspec_desc* desc, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens, int n_sink, int window,
                            float lambda, float* out_spec, float* out_exact, float* rel_l2,
                            uint8_t* commit, void* workspace, size_t workspace_bytes,
                            void* stream, void* spec_event, void* const* prof_events) {
    return decode_impl(desc, q, k_cache, v_cache, seq_lens, n_sink, window, lambda, out_spec,
                       out_exact, rel_l2, commit, workspace, workspace_bytes, stream, spec_event,
                       prof_events, nullptr);
}

alspec_status alspec_decode_traced(const alspec_desc* desc, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* seq_lens, int n_sink,
                                   int window, float lambda, float* out_spec, float* out_exact,
                                   float* rel_l2, uint8_t* commit, void* workspace,
                                   size_t workspace_bytes, void* stream,
                                   unsigned long long* trace_ns) {
    if (!trace_ns) return ALSPEC_ERR_INVALID_ARG;
    return decode_impl(desc, q, k_cache, v_cache, seq_lens, n_sink, window, lambda, out_spec,
                       out_exact, rel_l2, commit, workspace, workspace_bytes, stream, nullptr,
                       nullptr, trace_ns);
}

alspec_status alspec_oproj(const float* x, const void* w, float* y, const uint8_t* skip, int batch,
                           int k, int n, uint32_t* err, void* stream) {
    if (!oproj_args_ok(x, w, y, batch, k, n) || (reinterpret_cast<uintptr_t>(err) & 3u))
        return ALSPEC_ERR_INVALID_ARG;
    DeviceState* ds = nullptr;
    alspec_status st = get_device_state(&ds);
    if (st != ALSPEC_OK) return st;
    const OprojParams o = oproj_params(x, w, y, skip, batch, k, n, nullptr, err);
    return launch_oproj_bulk(ds, o, static_cast<cudaStream_t>(stream));
}

alspec_status alspec_decode_oproj(const alspec_desc* desc, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* seq_lens, int n_sink,
                                  int window, float lambda, const void* w_o, int hidden,
                                  float* out_spec, float* out_exact, float* rel_l2,
                                  uint8_t* commit, float* y, int gate, void* workspace,
                                  size_t workspace_bytes, void* stream,
                                  unsigned long long* trace_ns) {
    if (!desc) return ALSPEC_ERR_INVALID_ARG;
    const int kdim = desc->n_q_heads * desc->head_dim;
    if (!oproj_args_ok(out_spec, w_o, y, desc->batch, kdim, hidden) || !out_exact ||
        !aligned16(out_exact))
        return ALSPEC_ERR_INVALID_ARG;
    if (gate != ALSPEC_GATE_KERNEL && gate != ALSPEC_GATE_GRAPH_CONDITIONAL)
        return ALSPEC_ERR_INVALID_ARG;
    const OprojReq op{w_o, hidden, y, gate};
    return decode_impl(desc, q, k_cache, v_cache, seq_lens, n_sink, window, lambda, out_spec,
                       out_exact, rel_l2, commit, workspace, workspace_bytes, stream, nullptr,
                       nullptr, trace_ns, &op);
}

alspec_status alspec_test_wait_timeout(void* workspace, size_t workspace_bytes, int timeout_ms,
                                       void* stream) {
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < (size_t)kCtrFixed * sizeof(unsigned) || timeout_ms < 1 ||
        timeout_ms > 10000)
        return ALSPEC_ERR_INVALID_ARG;
    Params p{};
    p.ctr = static_cast<unsigned*>(workspace);
    p.timeout_ns = (unsigned long long)timeout_ms * 1000000ull;
    stalled_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return ok(cudaGetLastError()) ? ALSPEC_OK : ALSPEC_ERR_CUDA;
}

alspec_status alspec_get_device_error(void* workspace, size_t workspace_bytes, void* stream,
                                      uint32_t* err) {
    if (!workspace || !err || workspace_bytes < (kCtrFixed * sizeof(unsigned)))
        return ALSPEC_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned* word = static_cast<unsigned*>(workspace) + kCtrError;
    uint32_t host = 0;
    if (cudaMemcpyAsync(&host, word, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(word, 0, sizeof(unsigned), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return ALSPEC_ERR_CUDA;
    *err = host;
    if (host & kErrTimeout) return ALSPEC_ERR_TIMEOUT;
    if (host) return ALSPEC_ERR_DEVICE_DATA;
    return ALSPEC_OK;
}

alspec_status alspec_graph_begin(void* stream) {
    return ok(cudaStreamBeginCapture(static_cast<cudaStream_t>(stream),
                                     cudaStreamCaptureModeThreadLocal))
               ? ALSPEC_OK
               : ALSPEC_ERR_CUDA;
}

alspec_status alspec_graph_end(void* stream, void** graph) {
    if (!graph) return ALSPEC_ERR_INVALID_ARG;
    cudaGraph_t g = nullptr;
    if (!ok(cudaStreamEndCapture(static_cast<cudaStream_t>(stream), &g)) || !g)
        return ALSPEC_ERR_CUDA;
    cudaGraphExec_t exec = nullptr;
    const bool inst =
        ok(cudaGraphInstantiateWithFlags(&exec, g, cudaGraphInstantiateFlagUseNodePriority));
    cudaGraphDestroy(g);
    if (!inst) return ALSPEC_ERR_CUDA;
    *graph = exec;
    return ALSPEC_OK;
}

alspec_status alspec_graph_launch(void* graph, void* stream) {
    if (!graph) return ALSPEC_ERR_INVALID_ARG;
    return ok(cudaGraphLaunch(static_cast<cudaGraphExec_t>(graph),
                              static_cast<cudaStream_t>(stream)))
               ? ALSPEC_OK
               : ALSPEC_ERR_CUDA;
}

alspec_status alspec_graph_destroy(void* graph) {
    if (!graph) return ALSPEC_ERR_INVALID_ARG;
    return ok(cudaGraphExecDestroy(static_cast<cudaGraphExec_t>(graph))) ? ALSPEC_OK
                                                                         : ALSPEC_ERR_CUDA;
}

alspec_status alspec_shutdown(void) {
    noalloc_forget();
    std::lock_guard<std::mutex> lock(g_mutex);
    int cur = 0;
    const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
    alspec_status st = ALSPEC_OK;
    for (int d = 0; d < kMaxDevices; ++d) {
        DeviceState& s = g_dev[d];
        if (!s.ready) continue;
        if (cudaSetDevice(d) != cudaSuccess) {
            st = ALSPEC_ERR_CUDA;
            continue;
        }
        if (s.lo && cudaStreamSynchronize(s.lo) != cudaSuccess) st = ALSPEC_ERR_CUDA;
        cudaEventDestroy(s.fork);
        cudaEventDestroy(s.join);
        if (s.lo) cudaStreamDestroy(s.lo);
        s = DeviceState{};
    }
    if (have_cur) cudaSetDevice(cur);
    return st;
}

const char* alspec_status_string(alspec_status status) {
    switch (status) {
    case ALSPEC_OK: return "ok";
    case ALSPEC_ERR_INVALID_ARG: return "invalid argument";
    case ALSPEC_ERR_UNSUPPORTED: return "unsupported configuration";
    case ALSPEC_ERR_WORKSPACE: return "workspace missing or too small";
    case ALSPEC_ERR_CUDA: return "CUDA runtime error";
    case ALSPEC_ERR_TIMEOUT: return "in-kernel wait timed out";
    case ALSPEC_ERR_DEVICE_DATA: return "invalid device data (clamped)";
    default: return "unknown status";
    }
}

int alspec_version(void) { return 301; }

int alspec_last_cuda_error(void) { return (int)t_last_error; }

}  // extern "C"

// ------------------------------------------------------------ no-alloc path

namespace alspec {
namespace {

// Scratch space of alspec_decode_noalloc: a fixed array in this library's
// device memory (zero at load), used in place of a caller's workspace.  In
// host code the name is only a host-side stand-in; kernels get the device
// address looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ALSPEC_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and kept until alspec_shutdown.
alspec_status noalloc_scratch(void** out) {
    int dev = 0;
    if (!ok(cudaGetDevice(&dev)) || dev < 0 || dev >= kMaxDevices) return ALSPEC_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        if (!ok(cudaGetSymbolAddress(&ptr, g_noalloc_scratch)) || !ptr) return ALSPEC_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return ALSPEC_OK;
}

void noalloc_forget() {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    for (void*& p : g_noalloc_ptr) p = nullptr;
}

}  // namespace
}  // namespace alspec

extern "C" alspec_status alspec_decode_noalloc(const alspec_desc* desc, const void* q,
                                               const void* k_cache, const void* v_cache,
                                               const int32_t* seq_lens, int n_sink, int window,
                                               float lambda, float* out_spec, float* out_exact,
                                               float* rel_l2, uint8_t* commit, void* stream) {
    const size_t need = alspec_workspace_size(desc, n_sink, window);
    if (need == 0) {
        const alspec_status st = check_desc(desc, n_sink, window);
        return st != ALSPEC_OK ? st : ALSPEC_ERR_INVALID_ARG;
    }
    if (need > ALSPEC_NOALLOC_SCRATCH_BYTES) return ALSPEC_ERR_WORKSPACE;
    void* scratch = nullptr;
    const alspec_status st = noalloc_scratch(&scratch);
    if (st != ALSPEC_OK) return st;
    // The counters at the head of the scratch are cleared on `stream` once
    // the call's arguments have passed every check; the rest of the scratch
    // is written before it is read within a call.
    return decode_impl(desc, q, k_cache, v_cache, seq_lens, n_sink, window, lambda, out_spec,
                       out_exact, rel_l2, commit, scratch, ALSPEC_NOALLOC_SCRATCH_BYTES, stream,
                       nullptr, nullptr, nullptr, nullptr, /*clear_counters=*/true);
}

extern "C" alspec_status alspec_noalloc_device_error(void* stream, uint32_t* err) {
    if (!err) return ALSPEC_ERR_INVALID_ARG;
    void* scratch = nullptr;
    const alspec_status st = noalloc_scratch(&scratch);
    if (st != ALSPEC_OK) return st;
    return alspec_get_device_error(scratch, ALSPEC_NOALLOC_SCRATCH_BYTES, stream, err);
}
