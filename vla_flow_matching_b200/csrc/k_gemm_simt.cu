// fp32 SIMT GEMM for the PI0X_FP32 mode: D[m][n] = sum_k A[m][k] * Bw[n][k]
// (nn.Linear with weights in (out, in) layout), no TF32, with the epilogues of
// kernels.cuh.  64x64 tiles, K step 16, 4x4 outputs per thread.
#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

template <typename OutT>
__global__ void __launch_bounds__(256) k_gemm_simt(const float *A, int lda, const float *Bw, int ldb, int M, int N,
                                                    int K, int epi, GemmOut o) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int r = e >> 4, kk = e & 15;
      const int gm = m0 + r, gn = n0 + r;
      As[kk][r] = gm < M ? A[(size_t)gm * lda + k0 + kk] : 0.f;
      Bs[kk][r] = gn < N ? Bw[(size_t)gn * ldb + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
    const size_t orow = (size_t)(o.out_row0 + m) * o.ldo;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      const float v = acc[i][j];
      switch (epi) {
        case EPI_STORE_F32: static_cast<float *>(o.out)[orow + n] = v; break;
        case EPI_BIAS_F32: static_cast<float *>(o.out)[orow + n] = v + o.vec[n]; break;
        case EPI_VEC_SILU: static_cast<OutT *>(o.out)[orow + n] = from_f32<OutT>(silu_f(v + o.vec[n])); break;
        case EPI_RESID_F32: static_cast<float *>(o.out)[orow + n] += v; break;
        default: break;
      }
    }
  }
}

template <typename OutT>
void launch_gemm_simt(const float *A, int lda, const float *Bw, int ldb, int M, int N, int K, int epi,
                      const GemmOut &o, cudaStream_t s) {
  if (M <= 0) return;
  dim3 grid((M + 63) / 64, (N + 63) / 64);
  launch_pdl(k_gemm_simt<OutT>, grid, 256, 0, s, A, lda, Bw, ldb, M, N, K, epi, o);
}

template void launch_gemm_simt<float>(const float *, int, const float *, int, int, int, int, int, const GemmOut &,
                                      cudaStream_t);

}  // namespace pi0x
