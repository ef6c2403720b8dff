/*
 * alspec_read_probe.h -- C ABI of libalspec_read_probe.so, a measurement aid
 * kept apart from the decode library (libalspec.so, include/alspec.h).
 *
 * It answers one question for the benchmark: how fast does this GPU stream
 * a large buffer from HBM into shared memory with the machinery the
 * attention kernels use -- 1-D bulk copies of the TMA engine into an
 * mbarrier-guarded ring of 16 KB stages, one CTA per SM, nothing computed?
 * The rate of that pure read is the ceiling the exact-attention kernel's
 * rate is compared with, beside the measured copy peak.  Nothing here is
 * part of the method (no passage of the pages describes it).
 */
#ifndef ALSPEC_READ_PROBE_H
#define ALSPEC_READ_PROBE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Stream `bytes` of `buf` once, in 16 KB pieces spread evenly over one CTA
 * per SM of the current device (the piece order inside a CTA's span is
 * sequential).
 *   buf     device pointer, 16-byte aligned
 *   bytes   a positive multiple of 16
 *   err     device uint32, or NULL: bit 0x2 is ORed in when a bounded wait
 *           (2 s) inside the kernel expires; the kernel then lets its copies
 *           in flight land (bounded) and returns
 *   stream  cudaStream_t as void* (NULL: legacy default stream)
 * Returns 0 on success, 1 for a bad argument (nothing launched), 4 when a
 * CUDA call failed.  Asynchronous on `stream`.
 */
int alspec_read_probe(const void* buf, size_t bytes, uint32_t* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ALSPEC_READ_PROBE_H */
