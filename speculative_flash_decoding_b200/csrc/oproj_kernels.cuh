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
// cores, one warp per output row at a time, 16-byte loads of 8 weights with
// four of them in flight per lane, x read through L1, fp32 accumulation and
// a fixed-order warp reduction.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace alspec {

constexpr int kOprojWarps = 8;   // warps per CTA
constexpr int kOprojRows = 2;    // output rows per warp (interleaved loads)
constexpr int kOprojMaxB = 8;    // largest batch
constexpr int kOprojUnroll = 4;  // 16-byte weight chunks in flight per lane and row

struct OprojParams {
    const float* x;            // [B][K]
    const uint4* w;            // [N][K / 8] (8 bf16 per uint4)
    float* y;                  // [B][N]
    const uint8_t* skip;       // [B] or null: rows with skip[b] != 0 are left alone
    int B, K, N;
    unsigned long long* trace; // optional: raised to the global timer after the writes
};

__device__ __forceinline__ void bf16x8_to_float(const uint4& r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__global__ void __launch_bounds__(kOprojWarps * 32) oproj_kernel(const __grid_constant__ OprojParams p) {
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Rows of the batch this call writes (the same in every thread).
    unsigned live = 0;
    for (int b = 0; b < p.B; ++b)
        if (!p.skip || p.skip[b] == 0) live |= 1u << b;
    if (live == 0) return;

    const int KC = p.K >> 3;  // 16-byte chunks per row
    const int n0 = (blockIdx.x * kOprojWarps + warp) * kOprojRows;
    float acc[kOprojRows][kOprojMaxB];
#pragma unroll
    for (int r = 0; r < kOprojRows; ++r)
#pragma unroll
        for (int b = 0; b < kOprojMaxB; ++b) acc[r][b] = 0.f;

    for (int c0 = lane; c0 < KC; c0 += 32 * kOprojUnroll) {
        uint4 wv[kOprojRows][kOprojUnroll];
#pragma unroll
        for (int r = 0; r < kOprojRows; ++r) {
            const int n = n0 + r;
#pragma unroll
            for (int u = 0; u < kOprojUnroll; ++u) {
                const int c = c0 + 32 * u;
                wv[r][u] = (n < p.N && c < KC) ? __ldcs(p.w + (size_t)n * KC + c)
                                               : make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < kOprojUnroll; ++u) {
            const int c = c0 + 32 * u;
            if (c >= KC) break;
            float wf[kOprojRows][8];
#pragma unroll
            for (int r = 0; r < kOprojRows; ++r) bf16x8_to_float(wv[r][u], wf[r]);
#pragma unroll
            for (int b = 0; b < kOprojMaxB; ++b) {
                if (!((live >> b) & 1u)) continue;
                const float4* xp = reinterpret_cast<const float4*>(p.x + (size_t)b * p.K) + 2 * c;
                const float4 x0 = __ldg(xp);
                const float4 x1 = __ldg(xp + 1);
                const float xf[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                for (int r = 0; r < kOprojRows; ++r)
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[r][b] = fmaf(wf[r][i], xf[i], acc[r][b]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kOprojRows; ++r) {
        const int n = n0 + r;
#pragma unroll
        for (int b = 0; b < kOprojMaxB; ++b) {
            if (!((live >> b) & 1u)) continue;
            float v = acc[r][b];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && n < p.N) p.y[(size_t)b * p.N + n] = v;
        }
    }
    if (p.trace && lane == 0) {
        __threadfence();
        atomicMax(p.trace, (unsigned long long)global_ns());
    }
}

}  // namespace alspec
