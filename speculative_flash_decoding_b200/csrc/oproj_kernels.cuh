// Output projection of the attention output -- the linear map that follows
// self-attention in a decoder layer, run speculatively on O_spec while the
// exact attention is computed, and redone on O_exact for the tokens whose
// speculation is discarded (attention-level speculation, "Approach":
// post-attention ops run speculatively and are committed or discarded by the
// relative-L2 check).
//
//   y[b, n] = sum_k x[b, k] * w[n, k]
//
// x fp32 [B, K] (the attention output of token b, heads concatenated), w
// bf16 [N, K] (row n = output feature n), y fp32 [B, N].  The batch is small
// (decode), so the op streams w once from HBM and is bandwidth bound: CUDA
// cores, one warp per output row, 16-byte loads of 8 weights with a whole
// 4096-wide row in flight per warp, x read through L1, fp32 accumulation and
// a fixed-order warp reduction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace alspec {

constexpr int kOprojWarps = 4;    // warps per CTA, one output row each at a time
constexpr int kOprojMaxB = 8;     // largest batch
constexpr int kOprojChunks = 16;  // 16-byte weight chunks in flight per lane (8 KB per warp)

struct OprojParams {
    const float* x;            // [B][K]
    const uint4* w;            // [N][K / 8] (8 bf16 per uint4)
    float* y;                  // [B][N]
    const uint8_t* skip;       // [B] or null: rows with skip[b] != 0 are left alone
    int B, K, N;
    unsigned long long* trace; // optional: raised to the global timer after the writes
    unsigned* err;             // optional: error bits (timeout) are ORed in here
    unsigned long long timeout_ns;
};

constexpr unsigned kOprojErrTimeout = 0x2;  // same bit as the decoder's wait timeout

__device__ __forceinline__ void bf16x8_to_float(const uint4& r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// One warp per output row n: the lanes issue the row's 16-byte chunks
// kOprojChunks at a time (a whole 4096-wide row at once), then accumulate
// each chunk against the 8 matching x values of every live batch row, as
// packed pairs (even and odd k) added at the end.  NB (1, 2, 4 or 8) is the
// batch bucket: rows B..NB-1 are masked.
template <int NB>
__global__ void __launch_bounds__(kOprojWarps * 32) oproj_kernel(const __grid_constant__ OprojParams p) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Rows of the batch this call writes (the same in every thread).
    unsigned live = 0;
    for (int b = 0; b < p.B; ++b)
        if (!p.skip || p.skip[b] == 0) live |= 1u << b;
    if (live == 0) return;

    const int KC = p.K >> 3;  // 16-byte chunks per row
    const int n = blockIdx.x * kOprojWarps + warp;
    if (n < p.N) {
        const uint4* wrow = p.w + (size_t)n * KC;
        float2 acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = make_float2(0.f, 0.f);
        for (int c0 = lane; c0 < KC; c0 += 32 * kOprojChunks) {
            uint4 wv[kOprojChunks];
#pragma unroll
            for (int u = 0; u < kOprojChunks; ++u) {
                const int c = c0 + 32 * u;
                wv[u] = c < KC ? __ldcs(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kOprojChunks; ++u) {
                const int c = c0 + 32 * u;
                if (c >= KC) break;
                const uint32_t r[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
                float2 wp[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    wp[i] = make_float2(__uint_as_float(r[i] << 16),
                                        __uint_as_float(r[i] & 0xffff0000u));
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    if (!((live >> b) & 1u)) continue;
                    const float4* xp =
                        reinterpret_cast<const float4*>(p.x + (size_t)b * p.K) + 2 * c;
                    const float4 x0 = __ldg(xp);
                    const float4 x1 = __ldg(xp + 1);
                    acc[b] = __ffma2_rn(wp[0], make_float2(x0.x, x0.y), acc[b]);
                    acc[b] = __ffma2_rn(wp[1], make_float2(x0.z, x0.w), acc[b]);
                    acc[b] = __ffma2_rn(wp[2], make_float2(x1.x, x1.y), acc[b]);
                    acc[b] = __ffma2_rn(wp[3], make_float2(x1.z, x1.w), acc[b]);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            if (!((live >> b) & 1u)) continue;
            float v = acc[b].x + acc[b].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) p.y[(size_t)b * p.N + n] = v;
        }
    }
    if (p.trace && lane == 0) {
        __threadfence();
        atomicMax(p.trace, (unsigned long long)global_ns());
    }
}

// ----------------------------------------------------------------------
// Foreground form: two CTAs per SM (a grid of twice the SM count), each
// streaming its rows with 1-D bulk copies (TMA, evict-first) into a ring of
// 12 8 KB shared-memory stages -- so the bytes in flight are not bounded by
// the L1's outstanding-miss tracking, which held plain loads near 2 TB/s;
// the two rings (192 KB per SM) hold nearly an SM's whole share of a
// 4096 x 4096 matrix at once.  A CTA of 97 KB also fits beside the merge
// kernel's CTAs, so a projection launched programmatically behind the merge
// streams its weights while the merge runs (measured: 24 stages and one CTA
// per SM streamed as fast alone, but the projection after the merge took
// 2.5 us longer per layer).  CTA c owns rows [c * R, (c + 1) * R); a row is
// P = 2K / 8192 stages; consumer warp w owns the CTA's rows w, w + 8, ...;
// one producer lane fills the stages in order; for B <= 2 each lane loads
// four chunks (and their x) before it computes on any of them.  Every wait
// is bounded: on expiry the kernel ORs the timeout bit into p.err, stops,
// lets its copies land (bounded) and returns.
#ifndef ALSPEC_OB_STAGES
#define ALSPEC_OB_STAGES 12
#endif
#ifndef ALSPEC_OB_CONSUMERS
#define ALSPEC_OB_CONSUMERS 8
#endif
#ifndef ALSPEC_OB_MIN_BLOCKS
#define ALSPEC_OB_MIN_BLOCKS (ALSPEC_OB_STAGES <= 13 ? 2 : 1)
#endif
constexpr int kObStages = ALSPEC_OB_STAGES;
constexpr int kObMinBlocks = ALSPEC_OB_MIN_BLOCKS;  // CTAs an SM can hold
constexpr int kObPiece = 8192;   // bytes per stage
constexpr int kObConsumers = ALSPEC_OB_CONSUMERS;
constexpr int kObThreads = (kObConsumers + 1) * 32;
constexpr int kObSmem = kObStages * kObPiece + 2 * kObStages * 8 + kObStages * 4 + 16 + 1024;

__device__ __forceinline__ bool ob_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                        const OprojParams& p) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31) == 0) {
            if (*abort) return false;
            if (global_ns() - t0 > p.timeout_ns) {
                *abort = 1;
                if (p.err) atomicOr(p.err, kOprojErrTimeout);
                return false;
            }
        }
    }
}

template <int NB>
__global__ void __launch_bounds__(kObThreads, kObMinBlocks) oproj_bulk_kernel(const __grid_constant__ OprojParams p) {
    extern __shared__ unsigned char ob_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(ob_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kObStages * kObPiece);
    uint64_t* empty = full + kObStages;
    // Fill tickets: the global piece index each stage was last filled with.
    // When a row spans several pieces, consecutive fills of a stage belong
    // to different consumer warps, so a waiter checks the ticket (which
    // proves the stage's previous fill completed) before the parity.
    uint32_t* ticket = reinterpret_cast<uint32_t*>(empty + kObStages);
    volatile int* abort = reinterpret_cast<volatile int*>(ticket + kObStages);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // The kernel after this one on the stream may launch now (launched for
    // that, it waits for this grid before it uses what this one writes).
    pdl_launch_dependents();
    // x, the gate and y belong to the kernels ahead of this one, which may
    // still run (programmatic launch): the gate is read once they are done,
    // and nothing streams before it says there is work.  Without a gate
    // the weights (not written by those kernels: static in decode) stream
    // at once, and the consumers wait before they read x.
    unsigned live = (1u << p.B) - 1u;
    if (p.skip) {
        pdl_wait_prerequisite();
        live = 0;
        for (int b = 0; b < p.B; ++b)
            if (p.skip[b] == 0) live |= 1u << b;
        if (live == 0) return;
    }

    const int row_bytes = p.K * 2;
    const int P = (row_bytes + kObPiece - 1) / kObPiece;  // stages per row
    // Consecutive fills of a stage (pieces g and g + kObStages) belong to
    // one consumer warp exactly when P divides kObStages / kObConsumers
    // rounds evenly (P = 1 or 3); otherwise the waits check the tickets.
    const bool tickets = ((kObStages / P) % kObConsumers != 0) || (kObStages % P != 0);
    const int R = (p.N + gridDim.x - 1) / gridDim.x;
    const int r0 = blockIdx.x * R;
    const int nrows = max(0, min(p.N, r0 + R) - r0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kObStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
            ticket[s] = 0xffffffffu;
        }
        *abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (nrows == 0) return;

    if (warp == kObConsumers) {
        // Producer (one lane): stage g holds piece g % P of local row g / P.
        // (Issuing the first round of stages from several lanes measured
        // slower here: 14.4 against 12.4 us for a 4096 x 4096 matrix.)
        if (lane != 0) return;
        const int G = nrows * P;
        const uint64_t pol = l2_evict_first_policy();
        int g = 0;
        bool ok = true;
        for (; g < G; ++g) {
            const int slot = g % kObStages;
            if (g >= kObStages && !ob_wait(empty + slot, ((g / kObStages) - 1) & 1, abort, p)) {
                ok = false;
                break;
            }
            const int row = r0 + g / P;
            const int off = (g % P) * kObPiece;
            const uint32_t bytes = (uint32_t)min(kObPiece, row_bytes - off);
            if (tickets) st_release_shared(ticket + slot, (uint32_t)g);
            mbar_arrive_expect_tx(full + slot, bytes);
            bulk_load(smem + slot * kObPiece,
                      reinterpret_cast<const char*>(p.w) + (size_t)row * row_bytes + off, bytes,
                      full + slot, pol);
        }
        if (!ok) {
            // Let the copies of the last fill of every stage land (bounded).
            for (int g2 = max(0, g - kObStages); g2 < g; ++g2) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(full + g2 % kObStages, (g2 / kObStages) & 1))
                    if (global_ns() - t0 > p.timeout_ns) break;
            }
        }
        return;
    }

    // Consumers.
    if (!p.skip) pdl_wait_prerequisite();
    for (int rl = warp; rl < nrows; rl += kObConsumers) {
        float2 acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = make_float2(0.f, 0.f);
        bool ok = true;
        for (int pc = 0; pc < P && ok; ++pc) {
            const int g = rl * P + pc;
            const int slot = g % kObStages;
            // Lane 0 waits for the stage's ticket to name piece g, then for
            // the fill's phase; every lane then probes again (each
            // acquires) and the warp leaves together.
            bool got = false;
            if (lane == 0) {
                const uint64_t t0 = global_ns();
                got = true;
                for (uint32_t it = 0; tickets && ld_acquire_shared(ticket + slot) != (uint32_t)g;
                     ++it) {
                    if ((it & 31) == 31 && (*abort || global_ns() - t0 > p.timeout_ns)) {
                        if (!*abort && p.err) atomicOr(p.err, kOprojErrTimeout);
                        *abort = 1;
                        got = false;
                        break;
                    }
                }
                if (got) got = ob_wait(full + slot, (g / kObStages) & 1, abort, p);
            }
            got = __shfl_sync(0xffffffffu, got, 0);
            if (got) got = __all_sync(0xffffffffu, mbar_try_wait(full + slot, (g / kObStages) & 1));
            if (!got) {
                ok = false;
                break;
            }
            const int off = pc * kObPiece;
            const int nch = min(kObPiece, row_bytes - off) >> 4;  // 16-byte chunks
            const uint4* ws = reinterpret_cast<const uint4*>(smem + slot * kObPiece);
            const int c_base = off >> 4;
            // Chunks per lane loaded (with their x) before use; a batch of 8
            // reads x as it goes.  Both keep the kernel within the registers
            // of two CTAs per SM.
            constexpr int U = NB == 1 ? 4 : NB == 2 ? 2 : 1;
            constexpr bool kPre = NB <= 4;
            for (int c0 = lane; c0 < nch; c0 += 32 * U) {
                uint4 wq[U];
                float4 xv[U][kPre ? NB : 1][2];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + 32 * u;
                    if (c < nch) {
                        wq[u] = ws[c];
#pragma unroll
                        for (int b = 0; b < (kPre ? NB : 0); ++b) {
                            if (!((live >> b) & 1u)) continue;
                            const float4* xp = reinterpret_cast<const float4*>(
                                                   p.x + (size_t)b * p.K) + 2 * (c_base + c);
                            xv[u][b][0] = __ldg(xp);
                            xv[u][b][1] = __ldg(xp + 1);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (c0 + 32 * u >= nch) break;
                    const uint32_t r[4] = {wq[u].x, wq[u].y, wq[u].z, wq[u].w};
                    float2 wp[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        wp[i] = make_float2(__uint_as_float(r[i] << 16),
                                            __uint_as_float(r[i] & 0xffff0000u));
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        if (!((live >> b) & 1u)) continue;
                        float4 x0, x1;
                        if constexpr (kPre) {
                            x0 = xv[u][b][0];
                            x1 = xv[u][b][1];
                        } else {
                            const float4* xp = reinterpret_cast<const float4*>(
                                                   p.x + (size_t)b * p.K) + 2 * (c_base + c0);
                            x0 = __ldg(xp);
                            x1 = __ldg(xp + 1);
                        }
                        acc[b] = __ffma2_rn(wp[0], make_float2(x0.x, x0.y), acc[b]);
                        acc[b] = __ffma2_rn(wp[1], make_float2(x0.z, x0.w), acc[b]);
                        acc[b] = __ffma2_rn(wp[2], make_float2(x1.x, x1.y), acc[b]);
                        acc[b] = __ffma2_rn(wp[3], make_float2(x1.z, x1.w), acc[b]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);
        }
        if (!ok) break;
        const int n = r0 + rl;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            if (!((live >> b) & 1u)) continue;
            float v = acc[b].x + acc[b].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) p.y[(size_t)b * p.N + n] = v;
        }
    }
    if (p.trace && lane == 0) {
        __threadfence();
        atomicMax(p.trace, (unsigned long long)global_ns());
    }
}

// Graph gating: enable the conditional node that redoes the projection when
// any token of the batch was discarded (kept out of the merge kernel, which
// the profiler could not capture while it could set a conditional handle).
__global__ void __launch_bounds__(32) set_discard_condition(const uint8_t* commit, int B,
                                                            cudaGraphConditionalHandle h) {
    const bool discard = (int)threadIdx.x < B && commit[threadIdx.x] == 0;
    if (__any_sync(0xffffffffu, discard) && threadIdx.x == 0) cudaGraphSetConditional(h, 1u);
}

using OprojFn = void (*)(OprojParams);

// The kernels for a batch of B rows (1 <= B <= kOprojMaxB): the background
// form (no shared memory, so it shares SMs with a running middle kernel) and
// the foreground form (bulk copies, two CTAs per SM).
inline OprojFn oproj_kernel_for(int B) {
    return B <= 1 ? oproj_kernel<1> : B <= 2 ? oproj_kernel<2> : B <= 4 ? oproj_kernel<4>
                                                                       : oproj_kernel<8>;
}

inline OprojFn oproj_bulk_kernel_for(int B) {
    return B <= 1 ? oproj_bulk_kernel<1> : B <= 2 ? oproj_bulk_kernel<2>
                                       : B <= 4 ? oproj_bulk_kernel<4> : oproj_bulk_kernel<8>;
}

}  // namespace alspec
