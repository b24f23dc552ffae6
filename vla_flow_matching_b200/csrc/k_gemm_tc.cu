// bf16 GEMM on the sm_100a tensor cores (tcgen05.mma kind::f16, fp32 accumulate in
// TMEM), D[m][n] = sum_k A[m][k] * Bw[n][k], A = activations (rows x K), Bw =
// weights in nn.Linear (out, in) layout.  Both operands are K-major; TMA loads
// 128-byte-swizzled 64-wide K slices into a STAGES-deep shared-memory ring.
//
// Roles in the 128-thread CTA: thread 0 issues the TMA loads, thread 32 issues the
// MMAs (one elected thread, as tcgen05 wants), then all four warps read the
// 128 x BN accumulator from TMEM (warp w owns TMEM lanes 32w..32w+31, i.e. rows)
// and run the epilogue.  Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

template <int BN, int STAGES>
struct TcCfg {
  static constexpr int kABytes = 128 * 128;   // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;    // BN rows x 64 bf16
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
  static constexpr int kSmem = STAGES * kStage + 1024 /* alignment slack */ + 256 /* barriers */;
};

template <int BN, int STAGES, typename OutT>
__global__ void __launch_bounds__(128, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int a_row0, int M,
              int K, int epi, GemmOut o, unsigned *err) {
  using C = TcCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStage);
  uint64_t *empty = full + STAGES;
  uint64_t *done = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN;
  const int nk = K / 64;
  // After any earlier wait gave up, later GEMMs of the call do nothing (the call's
  // results are already invalid and the host reports PI0X_ETIMEOUT).
  if (*(volatile unsigned *)err != 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0) {
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t round = kb / STAGES;
      if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, err, kErrTimeoutProducer)) break;
      uint8_t *a_dst = smem + s * C::kStage;
      mbar_arrive_expect_tx(&full[s], C::kStage);
      tma_load_2d(a_dst, &tmA, kb * 64, a_row0 + m0, &full[s]);
      tma_load_2d(a_dst + C::kABytes, &tmB, kb * 64, n0, &full[s]);
    }
  } else if (threadIdx.x == 32) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t round = kb / STAGES;
      if (!mbar_wait(&full[s], round & 1u, err, kErrTimeoutMma)) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * C::kStage);
      const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc_mma_bf16(tmem, smem_desc_k_sw128(a_base, kk * 32), smem_desc_k_sw128(b_base, kk * 32), idesc,
                    (kb | kk) != 0);
      tc_commit(&empty[s]);
    }
    tc_commit(done);
  }
  __syncwarp();
  const bool ok = mbar_wait(done, 0, err, kErrTimeoutEpilogue);
  __syncwarp();
  tc_fence_after();
  if (__all_sync(0xffffffffu, ok)) {
    const int r = m0 + warp * 32 + lane;
    const size_t orow = (size_t)(o.out_row0 + r) * o.ldo;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      if (r < M) {
        const int n = n0 + c;
        if (epi == EPI_STORE_F32 || epi == EPI_BIAS_F32 || epi == EPI_RESID_F32) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(o.out) + orow + n);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 w = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            if (epi == EPI_BIAS_F32) {
              const float4 bb = reinterpret_cast<const float4 *>(o.vec + n)[i];
              w.x += bb.x; w.y += bb.y; w.z += bb.z; w.w += bb.w;
            } else if (epi == EPI_RESID_F32) {
              const float4 old = dst[i];
              w.x += old.x; w.y += old.y; w.z += old.z; w.w += old.w;
            }
            dst[i] = w;
          }
        } else if (epi == EPI_VEC_SILU) {
          OutT *dst = static_cast<OutT *>(o.out) + orow + n;
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[i] = from_f32<OutT>(silu_f(v[i] + o.vec[n + i]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int STAGES, typename OutT>
static void launch_bn(const TcGemm &g, int a_row0, int M, int epi, const GemmOut &o, unsigned *err,
                      cudaStream_t s) {
  using C = TcCfg<BN, STAGES>;
  auto kern = k_gemm_tc<BN, STAGES, OutT>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  dim3 grid((M + 127) / 128, g.N / BN);
  kern<<<grid, 128, C::kSmem, s>>>(g.tmA, g.tmB, a_row0, M, g.K, epi, o, err);
}

template <typename OutT>
void launch_gemm_tc(const TcGemm &g, int a_row0, int M, int epi, const GemmOut &o, unsigned *err,
                    cudaStream_t s) {
  if (M <= 0) return;
  switch (g.BN) {
    case 64: launch_bn<64, 6, OutT>(g, a_row0, M, epi, o, err, s); break;
    case 128: launch_bn<128, 5, OutT>(g, a_row0, M, epi, o, err, s); break;
    case 256: launch_bn<256, 4, OutT>(g, a_row0, M, epi, o, err, s); break;
    default: break;
  }
}

template void launch_gemm_tc<bf16>(const TcGemm &, int, int, int, const GemmOut &, unsigned *, cudaStream_t);
template void launch_gemm_tc<float>(const TcGemm &, int, int, int, const GemmOut &, unsigned *, cudaStream_t);

}  // namespace pi0x
