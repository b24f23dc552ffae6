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
 * 16-byte aligned.  K % 64 == 0, N % bn == 0, bn in {32, 64, 128, 256}, M >= 1.
 * splits > 1 splits K over that many CTAs per tile (bn 64 only, at most 148
 * tiles x splits), the partial tiles being summed in split order by the last
 * CTA to finish.  Synchronous; returns PI0X_EINVAL for bad sizes, PI0X_ECUDA if
 * a tensor map cannot be built, PI0X_ETIMEOUT if a bounded device wait gave up. */
int pi0x_debug_gemm_bf16(const void *A, const void *Bw, int M, int N, int K, float *D, int bn, int splits,
                         void *stream);

/* One layer of the suffix attention (the `_attend` step of the pi0 page) for B
 * samples with horizon H and prefix length P, all device pointers, bf16 unless
 * noted, activation rows laid out as in the sampler (state rows 0..B-1, then
 * action rows B + b*H + j-1):
 *   q (R, 2048) with R = B + B*H (post-RoPE, 8 heads x 256), ks/vs (R, 256)
 *   suffix keys/values, prefix_k/prefix_v (B, P, 256), mask (B, P) uint8.
 * step0 != 0 includes the state queries (first Euler step).  impl 0 = SIMT
 * kernel, 1 = tcgen05 kernel (split-KV as the sampler chooses), 2 = tcgen05
 * without split-KV.  Writes out (R, 2048); rows not queried are left as they
 * are.  Synchronous (allocates its scratch with cudaMalloc). */
int pi0x_debug_attention(const void *q, const void *ks, const void *vs, const void *prefix_k,
                         const void *prefix_v, const void *mask, int B, int H, int P, int step0, int impl,
                         void *out, void *stream);

/* The same attention as pi0x_debug_attention with impl 1 (tcgen05, split-KV as the
 * sampler chooses), for callers that cannot allocate device memory while they run
 * — e.g. a robot control loop that must never stall in cudaMalloc, or an
 * application whose device memory is owned by its own pool.  It calls no
 * cudaMalloc/cudaFree and no allocating library routine: all its scratch (a call
 * table, an error word, the valid-prefix index list and the split-KV partials)
 * lives in one static device array of 32 MiB inside libpi0x, which every GPU that
 * loads the library holds until the process exits.  The pages have no counterpart
 * to this entry point; it is a deployment variant of the `_attend` step.
 *
 * Arguments as for pi0x_debug_attention.  Returns PI0X_EINVAL when the problem's
 * scratch (4 B per prefix position per sample plus the split-KV partials,
 * 4 B x 258 per query row per split, at most 32.1 MB) does not fit in the 32 MiB;
 * the pi0 workloads up to B = 8 fit.  The first call on each device looks up the device
 * address of the array (cudaGetSymbolAddress, with that device current); make that
 * first call before any stream capture.  Every call clears the error word it uses;
 * the array keeps the contents of the last call.  All calls share the one array,
 * so calls that overlap on the GPU (other streams, other host threads) race.
 * Synchronous: returns after `stream` has finished the work, with PI0X_ETIMEOUT if
 * a bounded device wait gave up. */
int pi0x_attention_noalloc(const void *q, const void *ks, const void *vs, const void *prefix_k,
                           const void *prefix_v, const void *mask, int B, int H, int P, int step0, void *out,
                           void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PI0X_DEBUG_H */
