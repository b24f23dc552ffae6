/*
 * pi0x debug entry points: single kernels of libpi0x exposed for unit tests and
 * micro-benchmarks.  Same conventions as pi0x.h (int status, no aborts).  These
 * are not needed to run the sampler.
 */
#ifndef PI0X_DEBUG_H
#define PI0X_DEBUG_H

#ifdef __cplusplus
extern "C" {
#endif

/* D = A * Bw^T on the tcgen05 tensor cores (the GEMM every expert projection
 * uses in PI0X_BF16 mode): A (M, K) bf16 row-major, Bw (N, K) bf16 row-major
 * (nn.Linear weight layout), D (M, N) fp32 row-major; all device pointers,
 * 16-byte aligned.  K % 64 == 0, N % bn == 0, bn in {64, 128, 256}, M >= 1.
 * Enqueued on `stream`; returns PI0X_EINVAL for bad sizes, PI0X_ECUDA if a
 * tensor map cannot be built, PI0X_ETIMEOUT (after synchronizing the stream) if
 * a bounded device wait gave up. */
int pi0x_debug_gemm_bf16(const void *A, const void *Bw, int M, int N, int K, float *D, int bn, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PI0X_DEBUG_H */
