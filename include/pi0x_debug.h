/*
 * pi0x debug entry points: single kernels of libpi0x exposed for unit tests and
 * micro-benchmarks.  Same conventions as pi0x.h (int status, no aborts).  These
 * are not needed to run the sampler.
 */
#ifndef PI0X_DEBUG_H
#define PI0X_DEBUG_H

#include "pi0x.h"

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
 * — e.g. a robot control loop that must never stall in cudaMalloc (it can block
 * for milliseconds and synchronises the device), or an application whose device
 * memory is owned by its own pool.  It calls no cudaMalloc/cudaFree and no
 * allocating library routine: all its scratch (a call table, an error word, the
 * valid-prefix index list and the split-KV partials) lives in one static device
 * array of 32 MiB inside libpi0x, which every GPU that loads the library holds
 * until the process exits.  The paper has no counterpart to this entry point.
 *
 * Arguments as for pi0x_debug_attention.  Returns PI0X_EINVAL when the problem's
 * scratch does not fit in the 32 MiB: 4 B per prefix position per sample for the
 * index list, plus the split-KV partials (4 B x 258 per query row per split; split-KV
 * is used only for fewer than 96 row tiles and keeps tiles x splits <= 219, i.e.
 * at most 28.9 MB); the pi0 workloads up to B = 8 fit.  The first call on each
 * device looks up the device address of the array (cudaGetSymbolAddress, with that
 * device current).  Every call clears the error word it uses; the array keeps the
 * contents of the last call.  All calls share the one array, so calls that overlap
 * on the GPU (other streams, other host threads) race.  Synchronous: it waits for
 * `stream` and copies the error word to the host, so it cannot be captured into a
 * CUDA graph.  Returns PI0X_ETIMEOUT if a bounded device wait gave up, PI0X_ECUDA
 * for a CUDA error (text in pi0x_last_error). */
int pi0x_attention_noalloc(const void *q, const void *ks, const void *vs, const void *prefix_k,
                           const void *prefix_v, const void *mask, int B, int H, int P, int step0, void *out,
                           void *stream);

/* 1 if pi0x_sample(h, B, ...) runs the persistent small-batch loop kernel (bf16
 * mode, B * (horizon + 1) <= 128, action_dim <= 32 and a multiple of 4, a device
 * that can co-schedule one CTA per SM), else 0 (also for a NULL handle). */
int pi0x_uses_loop(const pi0x_handle *h, int B);

/* enable = 0: later pi0x_sample calls on `h` run every batch on the multi-kernel
 * path (one kernel per projection, attention and small step), so that tests can
 * compare it with the persistent loop at the same small batch; enable = 1 (the
 * default) restores the choice pi0x_uses_loop describes.  Waits for the handle's
 * last call and drops its cached graphs.  PI0X_EINVAL for a NULL handle or another
 * value. */
int pi0x_debug_set_loop(pi0x_handle *h, int enable);

/* Failure-path test hook of the persistent loop.  The next pi0x_sample call on `h`
 * that runs the loop kernel makes stage `stage` of the call (0 = the first stage of
 * Euler step 0, in program order) wait on a done-counter that nothing raises, with
 * every wait of that call bounded by `wait_ns` nanoseconds instead of the default
 * 200 ms.  The wait gives up, the kernel's other waits see
 * the error word and return, and pi0x_sync_status then reports PI0X_ETIMEOUT; the
 * call's x0 is invalid.  Later calls run normally (every call starts from zeroed
 * counters).  Returns PI0X_EINVAL for a NULL handle, a negative stage or a zero
 * limit. */
int pi0x_debug_loop_stall(pi0x_handle *h, int stage, unsigned long long wait_ns);

#ifdef __cplusplus
}
#endif

#endif /* PI0X_DEBUG_H */
