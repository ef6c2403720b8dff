// Host side of libalspec.so: argument checks, work planning, workspace
// layout, the fork/join onto a high-priority stream, kernel launches and the
// C ABI declared in include/alspec.h.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "alspec.h"
#include "attn_kernels.cuh"

namespace alspec {
namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }
int round_up(int a, int b) { return ceil_div(a, b) * b; }

// Per-device library state: the high-priority stream, the fork/join events,
// the SM count, and which kernels already got their shared-memory attribute.
struct DeviceState {
    bool ready = false;
    cudaStream_t hi = nullptr;
    cudaEvent_t fork = nullptr;
    cudaEvent_t join = nullptr;
    int sm_count = 0;
    int prio_hi = 0;
    std::set<const void*> attr_done;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];

alspec_status get_device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ALSPEC_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        int lo = 0, hi = 0;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess ||
            cudaStreamCreateWithPriority(&d.hi, cudaStreamNonBlocking, hi) != cudaSuccess ||
            cudaEventCreateWithFlags(&d.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&d.join, cudaEventDisableTiming) != cudaSuccess) {
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
    int c1, n1, c2, n2;
    int grid2;
    int threads, smem, stages;
    size_t off_ctr, off_spart_ml, off_spart_o, off_spec_ml, off_spec_o, off_mid_ml, off_mid_o,
        off_dn, total;
};

bool supported_g(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

alspec_status check_desc(const alspec_desc* d, int S, int W) {
    if (!d) return ALSPEC_ERR_INVALID_ARG;
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->max_seq_len < 1 ||
        d->head_dim < 1 || d->n_q_heads % d->n_kv_heads != 0 || S < 0 || W < 0 ||
        (long long)S + W < 1 || d->split_tokens < 0 || d->timeout_ms < 0)
        return ALSPEC_ERR_INVALID_ARG;
    if (d->dtype != ALSPEC_F32 && d->dtype != ALSPEC_BF16) return ALSPEC_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return ALSPEC_ERR_UNSUPPORTED;
    if (!supported_g(d->n_q_heads / d->n_kv_heads)) return ALSPEC_ERR_UNSUPPORTED;
    // Item indices and row offsets must fit their integer types.
    const long long heads = (long long)d->batch * d->n_kv_heads;
    if (heads * d->max_seq_len > (1ll << 40) || heads > (1 << 20)) return ALSPEC_ERR_UNSUPPORTED;
    return ALSPEC_OK;
}

void kernel_shape(int dtype, int D, int G, int* threads, int* smem, int* stages);

// Item sizes: the sink-set list (at most S + W tokens per head) is cut so
// that all heads together give about one CTA per SM; the middle is cut so
// that the persistent grid (one CTA per SM) gets a couple of items per CTA
// for a single sequence and more for batches, whose lengths may differ.
void make_plan(const alspec_desc& d, int S, int W, int sms, Plan* pl) {
    const int heads = d.batch * d.n_kv_heads;
    const int L = d.max_seq_len;
    const int nspec_max = std::min<long long>((long long)S + W, L);
    const int per_head1 = std::max(1, sms / std::max(1, heads));
    pl->c1 = round_up(std::max(1, ceil_div(nspec_max, per_head1)), kTile);
    pl->n1 = ceil_div(nspec_max, pl->c1);

    const int ns = std::min(S, L);
    const int mid_max = std::max(0, std::max(ns, L - W) - ns);
    if (mid_max == 0) {
        pl->c2 = kTile;
        pl->n2 = 0;
    } else if (d.split_tokens > 0) {
        pl->c2 = round_up(d.split_tokens, kTile);
        pl->n2 = ceil_div(mid_max, pl->c2);
    } else {
        const int target = (d.batch == 1 ? 2 : 8) * sms;
        const int per_head2 = std::max(1, ceil_div(target, heads));
        pl->c2 = round_up(std::max(1, ceil_div(mid_max, per_head2)), kTile);
        pl->n2 = ceil_div(mid_max, pl->c2);
    }
    const long long items2 = (long long)heads * pl->n2;
    pl->grid2 = (int)std::min<long long>(sms, items2);
    const int G = d.n_q_heads / d.n_kv_heads;
    kernel_shape(d.dtype, d.head_dim, G, &pl->threads, &pl->smem, &pl->stages);

    const size_t B = d.batch, Hq = d.n_q_heads, D = d.head_dim;
    const size_t n1 = pl->n1, n2 = std::max(pl->n2, 1);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, kAlign);
        return o;
    };
    pl->off_ctr = take((kCtrFixed + B * d.n_kv_heads + B) * sizeof(unsigned));
    pl->off_spart_ml = take(B * Hq * n1 * 2 * sizeof(float));
    pl->off_spart_o = take(B * Hq * n1 * D * sizeof(float));
    pl->off_spec_ml = take(B * Hq * 2 * sizeof(float));
    pl->off_spec_o = take(B * Hq * D * sizeof(float));
    pl->off_mid_ml = take(B * Hq * n2 * 2 * sizeof(float));
    pl->off_mid_o = take(B * Hq * n2 * D * sizeof(float));
    pl->off_dn = take(B * Hq * 2 * sizeof(float));
    pl->total = off;
}

// ------------------------------------------------------------- dispatch

using KernelFn = void (*)(Params);

struct KernelSet {
    KernelFn spec;
    KernelFn mid;
    int smem;
    int stages;
    int threads;
};

template <typename T, int D, int G>
KernelSet kernels_for() {
    using C = Cfg<T, D, G>;
    return KernelSet{attn_kernel<T, D, G, true>, attn_kernel<T, D, G, false>, C::kSmemBytes,
                     C::STAGES, C::kThreads};
}

template <typename T, int D>
bool pick_g(int G, KernelSet* ks) {
    switch (G) {
    case 1: *ks = kernels_for<T, D, 1>(); return true;
    case 2: *ks = kernels_for<T, D, 2>(); return true;
    case 4: *ks = kernels_for<T, D, 4>(); return true;
    case 8: *ks = kernels_for<T, D, 8>(); return true;
    default: return false;
    }
}

bool pick(int dtype, int D, int G, KernelSet* ks) {
    if (dtype == ALSPEC_BF16) {
        if (D == 128) return pick_g<__nv_bfloat16, 128>(G, ks);
        if (D == 64) return pick_g<__nv_bfloat16, 64>(G, ks);
    } else if (dtype == ALSPEC_F32) {
        if (D == 128) return pick_g<float, 128>(G, ks);
        if (D == 64) return pick_g<float, 64>(G, ks);
    }
    return false;
}

void kernel_shape(int dtype, int D, int G, int* threads, int* smem, int* stages) {
    KernelSet ks{};
    const bool ok = pick(dtype, D, G, &ks);
    *threads = ok ? ks.threads : 0;
    *smem = ok ? ks.smem : 0;
    *stages = ok ? ks.stages : 0;
}

alspec_status ensure_smem_attr(DeviceState* ds, KernelFn fn, int bytes) {
    std::lock_guard<std::mutex> lock(g_mutex);
    const void* key = reinterpret_cast<const void*>(fn);
    if (ds->attr_done.count(key)) return ALSPEC_OK;
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return ALSPEC_ERR_CUDA;
    ds->attr_done.insert(key);
    return ALSPEC_OK;
}

alspec_status launch(KernelFn fn, dim3 grid, dim3 block, int smem, cudaStream_t stream,
                     const Params& p, bool high_priority, int prio) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (high_priority) {
        attr[0].id = cudaLaunchAttributePriority;
        attr[0].val.priority = prio;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, fn, p) == cudaSuccess ? ALSPEC_OK : ALSPEC_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
    const int vals[8] = {pl.c1, pl.n1, pl.c2, pl.n2, pl.grid2, pl.threads, pl.smem, pl.stages};
    for (int i = 0; i < n_info && i < 8; ++i) info[i] = vals[i];
    return ALSPEC_OK;
}

alspec_status alspec_decode(const alspec_desc* desc, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens, int n_sink, int window,
                            float lambda, float* out_spec, float* out_exact, float* rel_l2,
                            uint8_t* commit, void* workspace, size_t workspace_bytes,
                            void* stream, void* spec_event, void* const* prof_events) {
    alspec_status st = check_desc(desc, n_sink, window);
    if (st != ALSPEC_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !out_spec || !out_exact || !rel_l2 || !commit)
        return ALSPEC_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return ALSPEC_ERR_INVALID_ARG;
    if (!(lambda >= 0.f) || std::isinf(lambda)) return ALSPEC_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return ALSPEC_ERR_WORKSPACE;

    Plan pl{};
    make_plan(*desc, n_sink, window, sm_count_for_plan(), &pl);
    if (workspace_bytes < pl.total) return ALSPEC_ERR_WORKSPACE;
    DeviceState* ds = nullptr;
    if ((st = get_device_state(&ds)) != ALSPEC_OK) return st;
    const int G = desc->n_q_heads / desc->n_kv_heads;
    KernelSet ks{};
    if (!pick(desc->dtype, desc->head_dim, G, &ks)) return ALSPEC_ERR_UNSUPPORTED;
    if ((st = ensure_smem_attr(ds, ks.spec, ks.smem)) != ALSPEC_OK) return st;
    if ((st = ensure_smem_attr(ds, ks.mid, ks.smem)) != ALSPEC_OK) return st;

    char* ws = static_cast<char*>(workspace);
    Params p{};
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
    p.c2 = pl.c2;
    p.n2 = pl.n2;
    p.ctr = reinterpret_cast<unsigned*>(ws + pl.off_ctr);
    p.spart_ml = reinterpret_cast<float*>(ws + pl.off_spart_ml);
    p.spart_o = reinterpret_cast<float*>(ws + pl.off_spart_o);
    p.spec_ml = reinterpret_cast<float*>(ws + pl.off_spec_ml);
    p.spec_o = reinterpret_cast<float*>(ws + pl.off_spec_o);
    p.mid_ml = reinterpret_cast<float*>(ws + pl.off_mid_ml);
    p.mid_o = reinterpret_cast<float*>(ws + pl.off_mid_o);
    p.dn = reinterpret_cast<float*>(ws + pl.off_dn);
    p.out_spec = out_spec;
    p.out_exact = out_exact;
    p.rel_l2 = rel_l2;
    p.commit = commit;
    p.timeout_ns = (unsigned long long)(desc->timeout_ms > 0 ? desc->timeout_ms : 2000) * 1000000ull;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto prof = [&](int i, cudaStream_t on) {
        return !prof_events || !prof_events[i] ||
               cudaEventRecordWithFlags(static_cast<cudaEvent_t>(prof_events[i]), on,
                                        cudaEventRecordExternal) == cudaSuccess;
    };
    if (!prof(0, s)) return ALSPEC_ERR_CUDA;
    // Fork: the sink-set kernel runs on the high-priority stream.
    if (cudaEventRecord(ds->fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(ds->hi, ds->fork, 0) != cudaSuccess)
        return ALSPEC_ERR_CUDA;
    const dim3 block(pl.threads);
    const dim3 grid1(desc->batch * desc->n_kv_heads * pl.n1);
    if ((st = launch(ks.spec, grid1, block, ks.smem, ds->hi, p, true, ds->prio_hi)) != ALSPEC_OK)
        return st;
    if (spec_event && cudaEventRecordWithFlags(static_cast<cudaEvent_t>(spec_event), ds->hi,
                                               cudaEventRecordExternal) != cudaSuccess)
        return ALSPEC_ERR_CUDA;
    if (!prof(1, ds->hi)) return ALSPEC_ERR_CUDA;
    if (cudaEventRecord(ds->join, ds->hi) != cudaSuccess) return ALSPEC_ERR_CUDA;
    // The middle of every sequence on the caller's stream.
    if (!prof(2, s)) return ALSPEC_ERR_CUDA;
    if (pl.n2 > 0) {
        if ((st = launch(ks.mid, dim3(pl.grid2), block, ks.smem, s, p, false, 0)) != ALSPEC_OK)
            return st;
    }
    if (!prof(3, s)) return ALSPEC_ERR_CUDA;
    // Join, then merge + relative L2 + flag.
    if (cudaStreamWaitEvent(s, ds->join, 0) != cudaSuccess) return ALSPEC_ERR_CUDA;
    KernelFn mk = desc->head_dim == 128 ? merge_kernel<128> : merge_kernel<64>;
    if ((st = launch(mk, dim3(desc->n_q_heads, desc->batch), dim3(desc->head_dim), 0, s, p, false,
                     0)) != ALSPEC_OK)
        return st;
    if (!prof(4, s)) return ALSPEC_ERR_CUDA;
    return ALSPEC_OK;
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
    return cudaStreamBeginCapture(static_cast<cudaStream_t>(stream),
                                  cudaStreamCaptureModeThreadLocal) == cudaSuccess
               ? ALSPEC_OK
               : ALSPEC_ERR_CUDA;
}

alspec_status alspec_graph_end(void* stream, void** graph) {
    if (!graph) return ALSPEC_ERR_INVALID_ARG;
    cudaGraph_t g = nullptr;
    if (cudaStreamEndCapture(static_cast<cudaStream_t>(stream), &g) != cudaSuccess || !g)
        return ALSPEC_ERR_CUDA;
    cudaGraphExec_t exec = nullptr;
    const cudaError_t e = cudaGraphInstantiateWithFlags(&exec, g, cudaGraphInstantiateFlagUseNodePriority);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return ALSPEC_ERR_CUDA;
    *graph = exec;
    return ALSPEC_OK;
}

alspec_status alspec_graph_launch(void* graph, void* stream) {
    if (!graph) return ALSPEC_ERR_INVALID_ARG;
    return cudaGraphLaunch(static_cast<cudaGraphExec_t>(graph), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? ALSPEC_OK
               : ALSPEC_ERR_CUDA;
}

alspec_status alspec_graph_destroy(void* graph) {
    if (!graph) return ALSPEC_ERR_INVALID_ARG;
    return cudaGraphExecDestroy(static_cast<cudaGraphExec_t>(graph)) == cudaSuccess
               ? ALSPEC_OK
               : ALSPEC_ERR_CUDA;
}

alspec_status alspec_shutdown(void) {
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
        if (cudaStreamSynchronize(s.hi) != cudaSuccess) st = ALSPEC_ERR_CUDA;
        cudaEventDestroy(s.fork);
        cudaEventDestroy(s.join);
        cudaStreamDestroy(s.hi);
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

int alspec_version(void) { return 100; }

}  // extern "C"
