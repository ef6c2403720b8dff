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
//   * the sink-set kernel (SPEC) reads only the S + W tokens, merges its
//     items in the CTA that finishes last and writes O_spec;
//   * the middle kernel (MID) is persistent: CTAs pull items from an atomic
//     queue and stream the cache through shared memory;
//   * the merge kernel combines the sink-set partial with the middle
//     partials into O_exact, then computes rel_l2 and the flag.
//
// Inside a CTA: one producer lane issues bulk asynchronous copies (the TMA
// engine's 1-D form) of 16-token K and V tiles into a ring of shared-memory
// stages guarded by mbarriers; eight consumer warps compute.  Every token
// row is handled by 8 lanes (each owning head_dim/8 elements, read as 16-byte
// chunks at stride 128 bytes, which is free of bank conflicts), so a warp
// covers the 16 tokens of a tile: 4 rows per 8-lane group.  Dot products use
// packed fp32x2 FMAs on bf16 values widened in registers; the 8 partial dots
// of a row are combined by a reduce-scatter so that each lane pair ends up
// owning one token's scores.  Online softmax keeps a warp-uniform running
// max per head.  At the end of an item the warps' states are merged through
// shared memory and one partial per query head is written.
//
// Every wait is bounded (global nanosecond timer); on expiry the kernel sets
// an error bit, stops issuing copies, drains the ones in flight and returns.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace alspec {

constexpr int kTile = 16;             // tokens per pipeline stage
constexpr int kSmemLimit = 227 * 1024;

constexpr unsigned kErrSeqLen = 1u;   // ALSPEC_DEVERR_SEQ_LEN
constexpr unsigned kErrTimeout = 2u;  // ALSPEC_DEVERR_TIMEOUT

// Counter words at the head of the workspace; the sink-set tickets
// [B * Hkv] and merge tickets [B] follow.
constexpr int kCtrQueue = 0;
constexpr int kCtrDone = 1;
constexpr int kCtrError = 2;
constexpr int kCtrFixed = 4;

constexpr int kLastTileFlag = 1;

struct Params {
    const void* q;
    const void* k;
    const void* v;
    const int* seq_lens;
    int B, Hq, Hkv, Lmax, S, W;
    float qscale;   // log2(e) / sqrt(d): scores come out in the log2 domain
    float lambda;
    int c1, n1;     // sink-set items: tokens per item, items per (b, kv head)
    int c2, n2;     // middle items
    unsigned* ctr;
    float* spart_ml;  // [B][Hq][n1][2]   sink-set item partials
    float* spart_o;   // [B][Hq][n1][D]
    float* spec_ml;   // [B][Hq][2]       merged sink-set partial
    float* spec_o;    // [B][Hq][D]
    float* mid_ml;    // [B][Hq][n2][2]   middle item partials
    float* mid_o;     // [B][Hq][n2][D]
    float* dn;        // [B][Hq][2]       per-head squared distance / norm
    float* out_spec;
    float* out_exact;
    float* rel_l2;
    uint8_t* commit;
    unsigned long long timeout_ns;
};

// Token geometry of one sequence: sink tokens [0, ns), window [ws, L),
// middle [ns, ws).  Out-of-range lengths are clamped (and flagged).
struct SeqGeom {
    int L, ns, ws, nspec, mid_len;
};

__device__ __forceinline__ SeqGeom seq_geom(const Params& p, int b, bool flag) {
    int L = __ldg(p.seq_lens + b);
    if (L < 1 || L > p.Lmax) {
        if (flag) atomicOr(p.ctr + kCtrError, kErrSeqLen);
        L = L < 1 ? 1 : p.Lmax;
    }
    SeqGeom g;
    g.L = L;
    g.ns = min(p.S, L);
    g.ws = max(g.ns, L - p.W);
    g.nspec = g.ns + (L - g.ws);
    g.mid_len = g.ws - g.ns;
    return g;
}

// One work item: n tokens, the first na of them at [a0, a0 + na) and the
// rest at [a1, a1 + n - na).
struct Item {
    int b, kvh, chunk, n, a0, na, a1;
};

template <bool SPEC>
__device__ __forceinline__ Item decode_item(const Params& p, int item, bool flag) {
    Item it;
    const int bh = item % (p.B * p.Hkv);
    it.chunk = item / (p.B * p.Hkv);
    it.b = bh / p.Hkv;
    it.kvh = bh % p.Hkv;
    SeqGeom g = seq_geom(p, it.b, flag);
    if (SPEC) {
        const int lo = it.chunk * p.c1;
        const int hi = min(lo + p.c1, g.nspec);
        it.n = max(0, hi - lo);
        it.a0 = lo;
        it.na = max(0, min(hi, g.ns) - lo);
        it.a1 = g.ws + max(lo, g.ns) - g.ns;
    } else {
        const int lo = g.ns + it.chunk * p.c2;
        const int hi = min(lo + p.c2, g.ws);
        it.n = max(0, hi - lo);
        it.a0 = lo;
        it.na = it.n;
        it.a1 = 0;
    }
    return it;
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

template <typename T, int D, int G>
struct Cfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kChunks = kRowBytes / 128;        // 16-B chunks per lane per row
    static constexpr int kPairs = Elem<T>::kPairs;         // float2 per chunk
    static constexpr int kLanePairs = kChunks * kPairs;    // float2 per lane per row
    static constexpr int kElemPerChunk = 16 / (int)sizeof(T);
    static constexpr int kElemPer128 = 128 / (int)sizeof(T);
    static constexpr int GW = G < 4 ? G : 4;               // heads per consumer warp
    static constexpr int NHW = G / GW;                     // warps sharing a tile
    // Warps are spread over the SM's four sub-partitions, each with 16K
    // registers: 8 warps per CTA allow 255 registers a thread, 9 only 168.
    // Configurations holding 4 heads x 16 elements of q and o per lane need
    // the former, so they run 7 consumer warps plus the producer.
    static constexpr bool kHeavy = GW * kLanePairs >= 32;
    static constexpr int NTW = (kHeavy ? 7 : 8) / NHW;     // tiles in flight per round
    static constexpr int NCW = NTW * NHW;                  // consumer warps
    static constexpr int kThreads = (NCW + 1) * 32;
    static constexpr int kTileBytes = kTile * kRowBytes;   // K or V part of a stage
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kSlotFloats = GW * (D + 2);
    static constexpr int kDepositBytes = NCW * kSlotFloats * 4;
    static constexpr int kSpwBudget =
        (kSmemLimit - kDepositBytes - 4096) / (NTW * kStageBytes);
    static constexpr int SPW = kSpwBudget < 1 ? 1 : (kSpwBudget > 4 ? 4 : kSpwBudget);
    static constexpr int STAGES = NTW * SPW;
    // Dynamic shared memory layout.
    static constexpr int kOffDeposit = STAGES * kStageBytes;
    static constexpr int kOffMeta = kOffDeposit + kDepositBytes;
    static constexpr int kOffBar = kOffMeta + STAGES * 16;
    static constexpr int kNumBars = 2 * STAGES + 3;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16;
    static_assert(kRowBytes % 128 == 0, "row must be a multiple of 128 bytes");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    static_assert(kSmemBytes <= kSmemLimit, "shared memory budget");
    static_assert(NTW >= 1 && NCW <= 8, "warp split");
};

// ---------------------------------------------------------------- waiting

struct Shared {
    int abort;
    int last;
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

// ------------------------------------------------------------ consumer state

template <class C>
struct WarpState {
    float2 q[C::GW][C::kLanePairs];  // prescaled query slice
    float2 o[C::GW][C::kLanePairs];  // unnormalised output slice
    float m[C::GW];                  // warp-uniform running max (log2 domain)
    float l[C::GW];                  // this lane's share of the exponential sum
};

template <class C>
__device__ __forceinline__ void reset_state(WarpState<C>& st) {
#pragma unroll
    for (int h = 0; h < C::GW; ++h) {
        st.m[h] = -INFINITY;
        st.l[h] = 0.f;
#pragma unroll
        for (int j = 0; j < C::kLanePairs; ++j) st.o[h][j] = make_float2(0.f, 0.f);
    }
}

template <typename T, class C>
__device__ __forceinline__ void load_query(WarpState<C>& st, const Params& p, int b, int head0,
                                           int li) {
#pragma unroll
    for (int h = 0; h < C::GW; ++h) {
        const char* row = reinterpret_cast<const char*>(p.q) +
                          ((size_t)b * p.Hq + head0 + h) * C::kRowBytes + li * 16;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
            const uint4 raw = __ldg(reinterpret_cast<const uint4*>(row + c * 128));
            float2 f[C::kPairs];
            Elem<T>::unpack(raw, f);
#pragma unroll
            for (int j = 0; j < C::kPairs; ++j)
                st.q[h][c * C::kPairs + j] = make_float2(f[j].x * p.qscale, f[j].y * p.qscale);
        }
    }
}

// One 16-token tile: scores, online-softmax update, value accumulation.
template <typename T, class C>
__device__ __forceinline__ void consume_tile(WarpState<C>& st, const char* ks, const char* vs,
                                             int nvalid, int lane) {
    const int grp = lane >> 3;
    const int li = lane & 7;
    const unsigned full = 0xffffffffu;

    // Partial dot products of this lane's slice for the group's 4 rows.
    float acc[4][C::GW];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const char* krow = ks + (grp * 4 + t) * C::kRowBytes + li * 16;
        float2 a[C::GW];
#pragma unroll
        for (int h = 0; h < C::GW; ++h) a[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
            const uint4 raw = *reinterpret_cast<const uint4*>(krow + c * 128);
            float2 kf[C::kPairs];
            Elem<T>::unpack(raw, kf);
#pragma unroll
            for (int j = 0; j < C::kPairs; ++j)
#pragma unroll
                for (int h = 0; h < C::GW; ++h)
                    a[h] = __ffma2_rn(st.q[h][c * C::kPairs + j], kf[j], a[h]);
        }
#pragma unroll
        for (int h = 0; h < C::GW; ++h) acc[t][h] = a[h].x + a[h].y;
    }

    // Reduce-scatter over the 8 lanes of the group: lanes 2u and 2u+1 end up
    // with the full score of row u.
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

    // Online softmax with a warp-uniform running max.
    float pr[C::GW];
#pragma unroll
    for (int h = 0; h < C::GW; ++h) {
        float mx = s[h];
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(full, mx, 16));
        if (mx > st.m[h]) {
            const float sc = exp2f(st.m[h] - mx);
            const float2 sc2 = make_float2(sc, sc);
#pragma unroll
            for (int j = 0; j < C::kLanePairs; ++j) st.o[h][j] = __fmul2_rn(st.o[h][j], sc2);
            st.l[h] *= sc;
            st.m[h] = mx;
        }
        pr[h] = valid ? exp2f(s[h] - st.m[h]) : 0.f;
        st.l[h] += (li & 1) ? 0.f : pr[h];
    }

    // Weighted value rows.
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float pt[C::GW];
#pragma unroll
        for (int h = 0; h < C::GW; ++h) pt[h] = __shfl_sync(full, pr[h], (lane & 24) | (t << 1));
        if (grp * 4 + t < nvalid) {
            const char* vrow = vs + (grp * 4 + t) * C::kRowBytes + li * 16;
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4*>(vrow + c * 128);
                float2 vf[C::kPairs];
                Elem<T>::unpack(raw, vf);
#pragma unroll
                for (int h = 0; h < C::GW; ++h) {
                    const float2 pp = make_float2(pt[h], pt[h]);
#pragma unroll
                    for (int j = 0; j < C::kPairs; ++j)
                        st.o[h][c * C::kPairs + j] =
                            __ffma2_rn(pp, vf[j], st.o[h][c * C::kPairs + j]);
                }
            }
        }
    }
}

// Weight of a partial with max m against the merged max M: exactly 1 when
// m == M, so merging one partial with empty ones reproduces it bit for bit.
__device__ __forceinline__ float merge_weight(float m, float M) {
    return m == M ? 1.f : exp2f(m - M);
}

// ------------------------------------------------------------ the kernel

template <typename T, int D, int G, bool SPEC>
__global__ void __launch_bounds__(Cfg<T, D, G>::kThreads, 1)
    attn_kernel(const __grid_constant__ Params p) {
    using C = Cfg<T, D, G>;
    extern __shared__ __align__(128) unsigned char smem[];
    float* deposit = reinterpret_cast<float*>(smem + C::kOffDeposit);
    int4* meta = reinterpret_cast<int4*>(smem + C::kOffMeta);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* empty_bar = full_bar + C::STAGES;
    uint64_t* dep_bar = empty_bar + C::STAGES;  // warps deposited their state
    uint64_t* free_bar = dep_bar + 1;           // warps finished the merge
    uint64_t* tk_bar = dep_bar + 2;             // ticket result published
    Shared* sh = reinterpret_cast<Shared*>(smem + C::kOffMisc);
    volatile int* abort = &sh->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_items = p.B * p.Hkv * (SPEC ? p.n1 : p.n2);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar + s, 1);
            mbar_init(empty_bar + s, C::NHW);
        }
        mbar_init(dep_bar, C::NCW);
        mbar_init(free_bar, C::NCW);
        mbar_init(tk_bar, 1);
        sh->abort = 0;
        sh->last = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == C::NCW) {
        // ---------------------------------------------------- producer
        if (lane != 0) return;
        uint32_t gt = 0;
        bool ok = true;
        for (int iter = 0; ok; ++iter) {
            int item;
            if (SPEC) {
                item = iter == 0 ? (int)blockIdx.x : n_items;
            } else {
                item = (int)atomicAdd(p.ctr + kCtrQueue, 1u);
            }
            if (item >= n_items || *abort) break;
            const Item it = decode_item<SPEC>(p, item, true);
            if (it.n == 0) continue;
            const size_t head_row = ((size_t)it.b * p.Hkv + it.kvh) * (size_t)p.Lmax;
            const char* kbase = reinterpret_cast<const char*>(p.k) + head_row * C::kRowBytes;
            const char* vbase = reinterpret_cast<const char*>(p.v) + head_row * C::kRowBytes;
            int ntiles = (it.n + kTile - 1) / kTile;
            ntiles = (ntiles + C::NTW - 1) / C::NTW * C::NTW;
            for (int t = 0; t < ntiles; ++t, ++gt) {
                const int s = gt % C::STAGES;
                if (!wait_one(empty_bar + s, ((gt / C::STAGES) & 1) ^ 1, abort, p)) {
                    ok = false;
                    break;
                }
                const int first = t * kTile;
                const int nvalid = max(0, min(kTile, it.n - first));
                meta[s] = make_int4(item, t, nvalid, t >= ntiles - C::NTW ? kLastTileFlag : 0);
                if (nvalid == 0) {
                    mbar_arrive(full_bar + s);
                    continue;
                }
                mbar_arrive_expect_tx(full_bar + s, 2u * nvalid * C::kRowBytes);
                char* ks = reinterpret_cast<char*>(smem) + s * C::kStageBytes;
                char* vs = ks + C::kTileBytes;
                // Up to two contiguous runs of rows (sink run, then window run).
                const int ra = max(0, min(nvalid, it.na - first));
                if (ra > 0) {
                    const size_t tok = (size_t)(it.a0 + first);
                    bulk_load(ks, kbase + tok * C::kRowBytes, ra * C::kRowBytes, full_bar + s);
                    bulk_load(vs, vbase + tok * C::kRowBytes, ra * C::kRowBytes, full_bar + s);
                }
                if (nvalid > ra) {
                    const size_t tok = (size_t)(it.a1 + (first + ra - it.na));
                    const int rb = nvalid - ra;
                    bulk_load(ks + ra * C::kRowBytes, kbase + tok * C::kRowBytes,
                              rb * C::kRowBytes, full_bar + s);
                    bulk_load(vs + ra * C::kRowBytes, vbase + tok * C::kRowBytes,
                              rb * C::kRowBytes, full_bar + s);
                }
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
            // The CTA that stops last resets the queue for the next call.
            const unsigned t = atomicAdd(p.ctr + kCtrDone, 1u);
            if (t == gridDim.x - 1) {
                atomicExch(p.ctr + kCtrQueue, 0u);
                atomicExch(p.ctr + kCtrDone, 0u);
            }
        }
        return;
    }

    // -------------------------------------------------------- consumers
    const int hw = warp / C::NTW;   // which GW heads of the group
    const int tw = warp % C::NTW;   // which token slot of the round
    const int li = lane & 7;
    WarpState<C> st;
    reset_state(st);
    uint32_t gt = tw;
    int items_done = 0;
    bool ok = true;
    int b = 0, kvh = 0, chunk = 0;
    for (;; gt += C::NTW) {
        const int s = gt % C::STAGES;
        if (!wait_warp(full_bar + s, (gt / C::STAGES) & 1, abort, p, lane)) {
            ok = false;
            break;
        }
        const int4 mt = meta[s];
        if (mt.x < 0) break;
        if (mt.y < C::NTW) {
            const int bh = mt.x % (p.B * p.Hkv);
            chunk = mt.x / (p.B * p.Hkv);
            b = bh / p.Hkv;
            kvh = bh % p.Hkv;
            load_query<T, C>(st, p, b, kvh * G + hw * C::GW, li);
        }
        if (mt.z > 0) {
            const char* ks = reinterpret_cast<const char*>(smem) + s * C::kStageBytes;
            consume_tile<T, C>(st, ks, ks + C::kTileBytes, mt.z, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar + s);
        if (!(mt.w & kLastTileFlag)) continue;

        // ---- end of this item: combine the warps' states into one partial.
        const unsigned fm = 0xffffffffu;
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            float l = st.l[h];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) l += __shfl_xor_sync(fm, l, o);
            st.l[h] = l;
#pragma unroll
            for (int j = 0; j < C::kLanePairs; ++j) {
                float2 v = st.o[h][j];
                v.x += __shfl_xor_sync(fm, v.x, 8);
                v.y += __shfl_xor_sync(fm, v.y, 8);
                v.x += __shfl_xor_sync(fm, v.x, 16);
                v.y += __shfl_xor_sync(fm, v.y, 16);
                st.o[h][j] = v;
            }
        }
        if (items_done > 0 &&
            !wait_warp(free_bar, (items_done - 1) & 1, abort, p, lane)) {
            ok = false;
            break;
        }
        float* slot = deposit + (hw * C::NTW + tw) * C::kSlotFloats;
#pragma unroll
        for (int h = 0; h < C::GW; ++h) {
            float* hs = slot + h * (D + 2);
            if (lane == 0) {
                hs[0] = st.m[h];
                hs[1] = st.l[h];
            }
            if (lane < 8) {
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
                    for (int j = 0; j < C::kPairs; ++j) {
                        const int e = c * C::kElemPer128 + li * C::kElemPerChunk + 2 * j;
                        *reinterpret_cast<float2*>(hs + 2 + e) = st.o[h][c * C::kPairs + j];
                    }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(dep_bar);
        if (!wait_warp(dep_bar, items_done & 1, abort, p, lane)) {
            ok = false;
            break;
        }
        {
            const int ctid = warp * 32 + lane;
            float* part_ml = SPEC ? p.spart_ml : p.mid_ml;
            float* part_o = SPEC ? p.spart_o : p.mid_o;
            const int per = SPEC ? p.n1 : p.n2;
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
                const size_t row = ((size_t)b * p.Hq + kvh * G + hh) * per + chunk;
                if (e == 0) {
                    part_ml[row * 2] = M;
                    part_ml[row * 2 + 1] = L;
                }
                part_o[row * D + e] = O;
            }
        }
        if (SPEC) __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(free_bar);
        reset_state(st);
        ++items_done;
        if (!SPEC) continue;

        // ---- sink-set kernel: the CTA finishing last for (b, kv head)
        // merges every item of that head into O_spec.
        if (!wait_warp(free_bar, (items_done - 1) & 1, abort, p, lane)) {
            ok = false;
            break;
        }
        if (warp == 0 && lane == 0) {
            const SeqGeom g = seq_geom(p, b, false);
            const int nch = (g.nspec + p.c1 - 1) / p.c1;
            unsigned* ticket = p.ctr + kCtrFixed + b * p.Hkv + kvh;
            const unsigned t = atomicAdd(ticket, 1u);
            sh->last = (t == (unsigned)(nch - 1)) ? nch : 0;
            if (sh->last) atomicExch(ticket, 0u);
            __threadfence();
            mbar_arrive(tk_bar);
        }
        if (!wait_warp(tk_bar, 0, abort, p, lane)) {
            ok = false;
            break;
        }
        const int nch = sh->last;
        if (nch > 0) {
            const int ctid = warp * 32 + lane;
            for (int idx = ctid; idx < G * D; idx += C::NCW * 32) {
                const int hh = idx / D;
                const int e = idx % D;
                const size_t bh = (size_t)b * p.Hq + kvh * G + hh;
                float M = -INFINITY;
                for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(p.spart_ml + (bh * p.n1 + c) * 2));
                float L = 0.f, O = 0.f;
                for (int c = 0; c < nch; ++c) {
                    const size_t r = bh * p.n1 + c;
                    const float f = merge_weight(__ldcg(p.spart_ml + r * 2), M);
                    L = fmaf(f, __ldcg(p.spart_ml + r * 2 + 1), L);
                    O = fmaf(f, __ldcg(p.spart_o + r * D + e), O);
                }
                if (e == 0) {
                    p.spec_ml[bh * 2] = M;
                    p.spec_ml[bh * 2 + 1] = L;
                }
                p.spec_o[bh * D + e] = O;
                p.out_spec[bh * D + e] = __fdiv_rn(O, L);
            }
        }
        // A sink-set CTA owns exactly one item; its end marker follows.
    }
    (void)ok;
}

// ------------------------------------------------------- merge + verify

// One CTA per (query head, sequence); thread e owns output element e.
// O_exact merges the sink-set partial with the sequence's middle partials;
// O_spec is rebuilt from the same sink-set partial with the same division,
// so the two are bit-identical when the middle is empty.  The per-head
// squared distance and squared norm are reduced in a fixed order; the CTA
// finishing last for the sequence sums them over heads (in head order) and
// writes rel_l2 and the commit flag.
template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const __grid_constant__ Params p) {
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int e = threadIdx.x;
    const SeqGeom g = seq_geom(p, b, false);
    const int nmid = (g.mid_len + p.c2 - 1) / p.c2;
    const size_t bh = (size_t)b * p.Hq + h;

    const float ms = p.spec_ml[bh * 2];
    const float ls = p.spec_ml[bh * 2 + 1];
    const float os = p.spec_o[bh * D + e];
    const float o_spec = __fdiv_rn(os, ls);

    float M = ms;
    for (int c = 0; c < nmid; ++c) M = fmaxf(M, p.mid_ml[(bh * p.n2 + c) * 2]);
    const float f0 = merge_weight(ms, M);
    float acc = f0 * os;
    float lsum = f0 * ls;
    for (int c = 0; c < nmid; ++c) {
        const size_t r = bh * p.n2 + c;
        const float f = merge_weight(p.mid_ml[r * 2], M);
        lsum = fmaf(f, p.mid_ml[r * 2 + 1], lsum);
        acc = fmaf(f, p.mid_o[r * D + e], acc);
    }
    const float o_exact = __fdiv_rn(acc, lsum);
    p.out_exact[bh * D + e] = o_exact;

    const float diff = o_exact - o_spec;
    float dd = diff * diff;
    float nn = o_exact * o_exact;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        dd += __shfl_xor_sync(0xffffffffu, dd, o);
        nn += __shfl_xor_sync(0xffffffffu, nn, o);
    }
    __shared__ float red[2][D / 32];
    if ((e & 31) == 0) {
        red[0][e >> 5] = dd;
        red[1][e >> 5] = nn;
    }
    __syncthreads();
    if (e == 0) {
        float sd = 0.f, sn = 0.f;
        for (int w = 0; w < D / 32; ++w) {
            sd += red[0][w];
            sn += red[1][w];
        }
        p.dn[bh * 2] = sd;
        p.dn[bh * 2 + 1] = sn;
        __threadfence();
        unsigned* ticket = p.ctr + kCtrFixed + p.B * p.Hkv + b;
        const unsigned t = atomicAdd(ticket, 1u);
        if (t == (unsigned)(p.Hq - 1)) {
            atomicExch(ticket, 0u);
            __threadfence();
            double D2 = 0.0, N2 = 0.0;
            for (int hh = 0; hh < p.Hq; ++hh) {
                D2 += (double)__ldcg(p.dn + ((size_t)b * p.Hq + hh) * 2);
                N2 += (double)__ldcg(p.dn + ((size_t)b * p.Hq + hh) * 2 + 1);
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
    }
}

}  // namespace alspec
