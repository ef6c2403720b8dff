// libalspec_read_probe.so: a read-bandwidth probe, kept out of the decode
// library.  It measures how fast this GPU streams a large buffer from HBM
// into shared memory with the same machinery the attention kernels use
// (1-D bulk copies into an mbarrier-guarded ring, one CTA per SM).  The
// benchmark reports the middle kernel's rate against it, beside the
// measured copy peak and the nominal HBM bandwidth.
#include <cuda_runtime.h>

#include <cstdint>

#include "alspec_read_probe.h"
#include "ptx.cuh"

namespace alspec {

constexpr int kRpStages = 12;
constexpr int kRpStage = 16384;  // bytes per stage
constexpr int kRpSmem = kRpStages * kRpStage + 2 * kRpStages * 8 + 1024;

struct ReadProbeParams {
    const unsigned char* buf;  // 16-byte aligned
    unsigned long long bytes;  // multiple of 16
    unsigned* err;             // optional: timeout bit
    unsigned long long timeout_ns;
};

// CTA c streams bytes [c * span, (c + 1) * span) in 16 KB pieces: lane 0 of
// warp 0 issues the copies, warp 1 releases each stage once it has landed.
// Every wait is bounded; on expiry the timeout bit is ORed into err and the
// CTA lets its copies land (bounded) before it returns.
__global__ void __launch_bounds__(64, 1) read_probe_kernel(const __grid_constant__ ReadProbeParams p) {
    extern __shared__ unsigned char rp_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(rp_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRpStages * kRpStage);
    uint64_t* empty = full + kRpStages;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const unsigned long long span =
        ((p.bytes / gridDim.x) + kRpStage - 1) / kRpStage * kRpStage;
    const unsigned long long lo = span * blockIdx.x;
    const unsigned long long hi = lo + span < p.bytes ? lo + span : p.bytes;
    const long long pieces = hi > lo ? (long long)((hi - lo + kRpStage - 1) / kRpStage) : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRpStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (lane != 0) return;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(bar, parity)) {
            if (global_ns() - t0 > p.timeout_ns) {
                if (p.err) atomicOr(p.err, 0x2u);
                return false;
            }
        }
        return true;
    };
    if (warp == 0) {
        const uint64_t pol = l2_evict_first_policy();
        long long g = 0;
        for (; g < pieces; ++g) {
            const int s = (int)(g % kRpStages);
            if (g >= kRpStages && !wait(empty + s, (uint32_t)((g / kRpStages) - 1) & 1u)) break;
            const unsigned long long off = lo + (unsigned long long)g * kRpStage;
            const uint32_t n = (uint32_t)(hi - off < (unsigned long long)kRpStage ? hi - off
                                                                                  : kRpStage);
            mbar_arrive_expect_tx(full + s, n);
            bulk_load(smem + s * kRpStage, p.buf + off, n, full + s, pol);
        }
        // Let the copies of the last fill of every stage land (bounded).
        for (long long g2 = g > kRpStages ? g - kRpStages : 0; g2 < g; ++g2)
            wait(full + g2 % kRpStages, (uint32_t)(g2 / kRpStages) & 1u);
    } else {
        for (long long g = 0; g < pieces; ++g) {
            const int s = (int)(g % kRpStages);
            if (!wait(full + s, (uint32_t)(g / kRpStages) & 1u)) break;
            mbar_arrive(empty + s);
        }
    }
}

}  // namespace alspec

extern "C" int alspec_read_probe(const void* buf, size_t bytes, uint32_t* err, void* stream) {
    using namespace alspec;
    const uintptr_t a = reinterpret_cast<uintptr_t>(buf);
    if (!buf || (a & 15u) || bytes == 0 || bytes % 16 != 0 ||
        (reinterpret_cast<uintptr_t>(err) & 3u))
        return 1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaFuncSetAttribute(reinterpret_cast<const void*>(read_probe_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kRpSmem) != cudaSuccess)
        return 4;
    ReadProbeParams rp{};
    rp.buf = static_cast<const unsigned char*>(buf);
    rp.bytes = bytes;
    rp.err = err;
    rp.timeout_ns = 2000000000ull;
    read_probe_kernel<<<sms, 64, kRpSmem, static_cast<cudaStream_t>(stream)>>>(rp);
    return cudaGetLastError() == cudaSuccess ? 0 : 4;
}
