// bf16 GEMM on the sm_100a tensor cores (tcgen05.mma kind::f16, fp32 accumulate in
// TMEM), D[m][n] = sum_k A[m][k] * Bw[n][k], A = activations (rows x K), Bw =
// weights in nn.Linear (out, in) layout.  Both operands are K-major; TMA loads
// 128-byte-swizzled 64-wide K slices into a STAGES-deep shared-memory ring.
//
// Roles in the 128-thread CTA: thread 0 issues the TMA loads, thread 32 issues the
// MMAs (one elected thread, as tcgen05 wants), then all four warps read the
// 128 x BN accumulator from TMEM (warp w owns TMEM lanes 32w..32w+31, i.e. rows)
// and run the epilogue.  Every wait is bounded (common.cuh).
//
// Split-K (small row counts): blockIdx.z takes a contiguous range of K blocks and
// stores its fp32 partial tile; the last CTA of a tile to arrive (counter in global
// memory) sums the partials in split order — so results do not depend on timing —
// and runs the epilogue.
//
// Fused epilogues (column orders are fixed by a row permutation of the weights at
// pi0x_create, see pi0x_api.cu):
//  * EPI_QKV_ROPE: columns come in groups of 16 = 8 rotation pairs (i, i+128) of
//    one head; the epilogue applies rotate-half RoPE at position n_b + j and writes
//    q (bf16, 8 heads), k and v (bf16, the layer's suffix K/V rows).
//  * EPI_GEGLU: groups of 16 = 8 gate then the matching 8 up features; writes
//    gelu_tanh(gate) * up in bf16.
#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

#ifndef PI0X_BN64_STAGES
#define PI0X_BN64_STAGES 6
#endif
constexpr int kBn64Stages = PI0X_BN64_STAGES;

// AR = rows of the activation tile loaded per stage: 128, or 64 when the GEMM has
// at most 64 rows.  The MMA is always M = 128; with AR = 64 the accumulator rows
// 64..127 see whatever follows the A tile in shared memory and are never stored.
template <int BN, int STAGES, int AR = 128>
struct TcCfg {
  static constexpr int kABytes = AR * 128;    // AR rows x 64 bf16
  static constexpr int kBBytes = BN * 128;    // BN rows x 64 bf16
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
  static constexpr int kSmem = STAGES * kStage + 1024 /* alignment slack */ + 256 /* barriers */;
};

__device__ __forceinline__ void row_to_bj_tc(int r, int B, int H, int &b, int &j) {
  if (r < B) {
    b = r;
    j = 0;
  } else {
    b = (r - B) / H;
    j = 1 + (r - B) % H;
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float *v) {
  uint32_t p[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    p[e] = *reinterpret_cast<const uint32_t *>(&h2);
  }
  return make_uint4(p[0], p[1], p[2], p[3]);
}

// 1/sqrt(mean(h^2) + eps) of an output row from the producer's partial sums.
__device__ __forceinline__ float row_rstd(const EpiArgs &e, int orow) {
  float ss = 0.f;
#pragma unroll
  for (int t = 0; t < kNormSlots; ++t) ss += e.ss_in[(size_t)t * e.ss_ld + orow];
  return 1.0f / sqrtf(ss / (float)kWidth + kRmsEps);
}

// Fused-norm scale of GEMM row r for the consumer epilogues (1 otherwise).
template <int EPI>
__device__ __forceinline__ float consumer_rstd(const EpiArgs &e, int r) {
  if constexpr (EPI == EPI_QKV_ROPE || EPI == EPI_GEGLU) {
    if (e.ss_in) return row_rstd(e, e.out_row0 + r);
  }
  return 1.f;
}

// Global operands of the epilogue of one 32-column chunk, loaded ahead of the chunk:
// the residual row slice, the bias, or the RoPE (cos, sin) pairs.  (The norm gain is
// the same for every row and is read from L1 when used.)
constexpr int kEpiAhead = 2;  // chunks loaded ahead of the one in process
struct EpiIn {
  float4 a[8];
};

// RoPE position of output row `orow` (EPI_QKV_ROPE), once per tile.
template <int EPI>
__device__ __forceinline__ int epi_pos(const EpiArgs &e, int orow) {
  if constexpr (EPI == EPI_QKV_ROPE) {
    int b, j;
    row_to_bj_tc(orow, e.B, e.H, b, j);
    return e.nvalid[b] + j;
  }
  return 0;
}

template <int EPI>
__device__ __forceinline__ void epi_fetch(const EpiArgs &e, int r, int n, int pos, EpiIn &in) {
  const int orow = e.out_row0 + r;
  if constexpr (EPI == EPI_RESID_F32) {
    const float4 *src = reinterpret_cast<const float4 *>(e.out_f32 + (size_t)orow * e.ldo + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) in.a[i] = src[i];
  } else if constexpr (EPI == EPI_BIAS_F32 || EPI == EPI_VEC_SILU) {
    const float4 *src = reinterpret_cast<const float4 *>(e.vec + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) in.a[i] = src[i];
  } else if constexpr (EPI == EPI_QKV_ROPE) {
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const int gc = (n >> 4) + gi;
      const int hd = gc >> 4, ib = (gc & 15) * 8;
      if (hd < kHeads + 1) {
        // (cos, sin) of fp32(pos) * inv_freq[i], tabulated per call (k_rope_table)
        const float4 *tab = reinterpret_cast<const float4 *>(e.rope_tab + ((size_t)pos * (kHeadDim / 2) + ib) * 2);
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) in.a[4 * gi + w2] = tab[w2];
      }
    }
  }
  (void)pos;
  (void)orow;
}

// Epilogue of 32 consecutive output columns [n, n+32) of GEMM row r (`rs` from
// consumer_rstd, `in` from epi_fetch).  Returns the row's sum of squares over these
// columns for the fused-norm producers, else 0.
template <int EPI>
__device__ __forceinline__ float epilogue32(const EpiArgs &e, int r, int n, float (&v)[32], float rs, const EpiIn &in) {
  const int orow = e.out_row0 + r;
  float ssq = 0.f;
  if constexpr (EPI == EPI_STORE_F32 || EPI == EPI_BIAS_F32 || EPI == EPI_RESID_F32) {
    float4 *dst = reinterpret_cast<float4 *>(e.out_f32 + (size_t)orow * e.ldo + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 w = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      if constexpr (EPI == EPI_BIAS_F32 || EPI == EPI_RESID_F32) {
        const float4 bb = in.a[i];  // bias, or the residual h
        w.x += bb.x; w.y += bb.y; w.z += bb.z; w.w += bb.w;
      }
      dst[i] = w;
      v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
    }
    if constexpr (EPI != EPI_STORE_F32) {
      if (e.gain) {  // fused RMSNorm producer: bf16(h * (1 + g)) and sum of h^2
        float t[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 gg = reinterpret_cast<const float4 *>(e.gain + n)[i];
          ssq = fmaf(v[4 * i], v[4 * i], ssq);
          ssq = fmaf(v[4 * i + 1], v[4 * i + 1], ssq);
          ssq = fmaf(v[4 * i + 2], v[4 * i + 2], ssq);
          ssq = fmaf(v[4 * i + 3], v[4 * i + 3], ssq);
          t[4 * i] = v[4 * i] * (1.0f + gg.x);
          t[4 * i + 1] = v[4 * i + 1] * (1.0f + gg.y);
          t[4 * i + 2] = v[4 * i + 2] * (1.0f + gg.z);
          t[4 * i + 3] = v[4 * i + 3] * (1.0f + gg.w);
        }
        uint4 *xd = reinterpret_cast<uint4 *>(e.xn_out + (size_t)orow * kWidth + n);
#pragma unroll
        for (int i = 0; i < 4; ++i) xd[i] = pack8_bf16(t + 8 * i);
      }
    }
  } else if constexpr (EPI == EPI_VEC_SILU) {
    float t[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 bb = in.a[i];
      t[4 * i] = silu_f(v[4 * i] + bb.x);
      t[4 * i + 1] = silu_f(v[4 * i + 1] + bb.y);
      t[4 * i + 2] = silu_f(v[4 * i + 2] + bb.z);
      t[4 * i + 3] = silu_f(v[4 * i + 3] + bb.w);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(e.out_bf16 + (size_t)orow * e.ldo + n);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = pack8_bf16(t + 8 * i);
  } else if constexpr (EPI == EPI_QKV_ROPE) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= rs;
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const int gc = (n >> 4) + gi;
      const int hd = gc >> 4, ib = (gc & 15) * 8;
      float lo[8], hi[8];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        lo[w] = v[16 * gi + w];
        hi[w] = v[16 * gi + 8 + w];
      }
      if (hd < kHeads + 1) {
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) {
          const float4 t = in.a[4 * gi + w2];  // (cos, sin) of pairs ib+2*w2, ib+2*w2+1
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int w = 2 * w2 + h2;
            const float cs = h2 ? t.z : t.x, sn = h2 ? t.w : t.y;
            const float a = lo[w], bb = hi[w];
            lo[w] = a * cs - bb * sn;
            hi[w] = bb * cs + a * sn;
          }
        }
      }
      bf16 *dst;
      if (hd < kHeads)
        dst = e.q + (size_t)orow * kQDim + hd * kHeadDim + ib;
      else if (hd == kHeads)
        dst = e.ks + (size_t)orow * kHeadDim + ib;
      else
        dst = e.vs + (size_t)orow * kHeadDim + ib;
      *reinterpret_cast<uint4 *>(dst) = pack8_bf16(lo);
      *reinterpret_cast<uint4 *>(dst + kHeadDim / 2) = pack8_bf16(hi);
    }
  } else if constexpr (EPI == EPI_GEGLU) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= rs;
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const int f0 = ((n >> 4) + gi) * 8;
      float a[8];
#pragma unroll
      for (int w = 0; w < 8; ++w) a[w] = gelu_tanh_f(v[16 * gi + w]) * v[16 * gi + 8 + w];
      *reinterpret_cast<uint4 *>(e.out_bf16 + (size_t)orow * kMlp + f0) = pack8_bf16(a);
    }
  }
  return ssq;
}

// After the last column chunk of a tile: store the row's partial sum of squares
// into the tile's slot (and clear the unused slots once per row).
template <int EPI>
__device__ __forceinline__ void norm_partial_store(const EpiArgs &e, int r, int n0, int BN, int N, float ssq) {
  if constexpr (EPI == EPI_BIAS_F32 || EPI == EPI_RESID_F32) {
    if (e.gain && e.ss_out) {
      const int orow = e.out_row0 + r;
      e.ss_out[(size_t)(n0 / BN) * e.ss_ld + orow] = ssq;
      if (n0 == 0)
        for (int t = N / BN; t < kNormSlots; ++t) e.ss_out[(size_t)t * e.ss_ld + orow] = 0.f;
    }
  }
}

template <int BN, int STAGES, int EPI, int AR>
__global__ void __launch_bounds__(128, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int a_row0, int M,
              int nk, int kb_per_split, EpiArgs e, unsigned *err) {
  using C = TcCfg<BN, STAGES, AR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStage);
  uint64_t *empty = full + STAGES;
  uint64_t *done = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  int *last_flag = reinterpret_cast<int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN;
  const int splits = gridDim.z;
  const int kb0 = blockIdx.z * kb_per_split;
  const int kb1 = min(nk, kb0 + kb_per_split);
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
  pdl_trigger();

  if (threadIdx.x == 0) {
    // Weight tiles do not depend on the previous kernel: start streaming the first
    // ring's worth before waiting for it, then add the activation tiles.
    const int pre = min(STAGES, kb1 - kb0);
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], C::kStage);
      tma_load_2d(smem + i * C::kStage + C::kABytes, &tmB, (kb0 + i) * 64, n0, &full[i]);
    }
    pdl_wait();
    for (int i = 0; i < pre; ++i) tma_load_2d(smem + i * C::kStage, &tmA, (kb0 + i) * 64, a_row0 + m0, &full[i]);
    for (int kb = kb0 + pre; kb < kb1; ++kb) {
      const int i = kb - kb0, s = i % STAGES;
      const uint32_t round = i / STAGES;
      if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, err, kErrTimeoutProducer)) break;
      uint8_t *a_dst = smem + s * C::kStage;
      mbar_arrive_expect_tx(&full[s], C::kStage);
      tma_load_2d(a_dst, &tmA, kb * 64, a_row0 + m0, &full[s]);
      tma_load_2d(a_dst + C::kABytes, &tmB, kb * 64, n0, &full[s]);
    }
  } else {
    pdl_wait();
  }
  if (threadIdx.x == 32) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
    for (int kb = kb0; kb < kb1; ++kb) {
      const int i = kb - kb0, s = i % STAGES;
      const uint32_t round = i / STAGES;
      if (!mbar_wait(&full[s], round & 1u, err, kErrTimeoutMma)) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * C::kStage);
      const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc_mma_bf16(tmem, smem_desc_k_sw128(a_base, kk * 32), smem_desc_k_sw128(b_base, kk * 32), idesc,
                    (i | kk) != 0);
      tc_commit(&empty[s]);
    }
    tc_commit(done);
  }
  __syncwarp();
  const bool ok = mbar_wait(done, 0, err, kErrTimeoutEpilogue);
  __syncwarp();
  tc_fence_after();
  const bool all_ok = __syncthreads_and(ok);
  const int rr = warp * 32 + lane;  // row within the tile
  const int r = m0 + rr;
  const uint32_t t_lane = (uint32_t)(warp * 32) << 16;
  if (all_ok) {
    if (splits == 1) {
      float ssq = 0.f;
      const float rs = r < M ? consumer_rstd<EPI>(e, r) : 1.f;
      const int pos = r < M ? epi_pos<EPI>(e, e.out_row0 + r) : 0;
      EpiIn in[kEpiAhead + 1];
#pragma unroll
      for (int c = 0; c < kEpiAhead * 32 && c < BN; c += 32)
        if (r < M) epi_fetch<EPI>(e, r, n0 + c, pos, in[c >> 5]);
#pragma unroll
      for (int c = 0; c < BN; c += 32) {
        const int ci = c >> 5;
        if (c + kEpiAhead * 32 < BN && r < M)
          epi_fetch<EPI>(e, r, n0 + c + kEpiAhead * 32, pos, in[(ci + kEpiAhead) % (kEpiAhead + 1)]);
        float v[32];
        tmem_ld_32x32b_x32(tmem + t_lane + (uint32_t)c, v);
        if (r < M) ssq += epilogue32<EPI>(e, r, n0 + c, v, rs, in[ci % (kEpiAhead + 1)]);
      }
      if (r < M) norm_partial_store<EPI>(e, r, n0, BN, gridDim.y * BN, ssq);
    } else {
      const int tile = blockIdx.x * gridDim.y + blockIdx.y;
      float *mine = e.part + ((size_t)tile * splits + blockIdx.z) * (128 * BN) + (size_t)rr * BN;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + t_lane + (uint32_t)c, v);
        if (r < M) {
          float4 *d4 = reinterpret_cast<float4 *>(mine + c);
#pragma unroll
          for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        const int prev = atomicAdd(e.counters + tile, 1);
        *last_flag = (prev == splits - 1);
      }
      __syncthreads();
      if (*last_flag) {
        __threadfence();
        const float *base = e.part + (size_t)tile * splits * (128 * BN) + (size_t)rr * BN;
        if (r < M) {
          float ssq = 0.f;
          const float rs = consumer_rstd<EPI>(e, r);
#pragma unroll 1
          for (int c = 0; c < BN; c += 32) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
            for (int s = 0; s < splits; ++s) {
              const float4 *p4 = reinterpret_cast<const float4 *>(base + (size_t)s * (128 * BN) + c);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 t = __ldcg(p4 + i);
                v[4 * i] += t.x; v[4 * i + 1] += t.y; v[4 * i + 2] += t.z; v[4 * i + 3] += t.w;
              }
            }
            EpiIn in;
            epi_fetch<EPI>(e, r, n0 + c, epi_pos<EPI>(e, e.out_row0 + r), in);
            ssq += epilogue32<EPI>(e, r, n0 + c, v, rs, in);
          }
          norm_partial_store<EPI>(e, r, n0, BN, gridDim.y * BN, ssq);
        }
        if (threadIdx.x == 0) e.counters[tile] = 0;  // ready for the next GEMM that uses it
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

// Persistent variant (no split-K): one CTA per SM walks the output tiles
// (row tile fastest, so concurrently running CTAs share weight tiles in L2).
// Warp 0 = TMA producer, warp 1 = MMA issuer, warps 2..5 = epilogue.  Two TMEM
// accumulators let the epilogue of one tile overlap the main loop of the next.
template <int BN, int STAGES, int EPI, int AR>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc_persist(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int a_row0,
                      int M, int N, int nk, EpiArgs e, unsigned *err) {
  using C = TcCfg<BN, STAGES, AR>;
  constexpr int kAcc = 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStage);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;
  uint64_t *acc_empty = acc_full + kAcc;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + kAcc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (M + 127) / 128, ntiles = mt * (N / BN);
  if (*(volatile unsigned *)err != 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kAcc * C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // weight tiles of this CTA's first tile before the previous kernel finishes
      const int pre = blockIdx.x < ntiles ? min(STAGES, nk) : 0;
      {
        const int n0 = (blockIdx.x / mt) * BN;
        for (int i = 0; i < pre; ++i) {
          mbar_arrive_expect_tx(&full[i], C::kStage);
          tma_load_2d(smem + i * C::kStage + C::kABytes, &tmB, i * 64, n0, &full[i]);
        }
      }
      pdl_wait();
      {
        const int m0 = (blockIdx.x % mt) * 128;
        for (int i = 0; i < pre; ++i) tma_load_2d(smem + i * C::kStage, &tmA, i * 64, a_row0 + m0, &full[i]);
      }
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int m0 = (t % mt) * 128, n0 = (t / mt) * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          if (it < pre) continue;  // issued above
          const int s = it % STAGES;
          const uint32_t round = it / STAGES;
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, err, kErrTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t *a_dst = smem + s * C::kStage;
          mbar_arrive_expect_tx(&full[s], C::kStage);
          tma_load_2d(a_dst, &tmA, kb * 64, a_row0 + m0, &full[s]);
          tma_load_2d(a_dst + C::kABytes, &tmB, kb * 64, n0, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
      int it = 0, ti = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++ti) {
        const int a = ti % kAcc;
        const uint32_t around = ti / kAcc;
        if (!mbar_wait(&acc_empty[a], (around & 1u) ^ 1u, err, kErrTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * C::kTmemCols);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t round = it / STAGES;
          if (!mbar_wait(&full[s], round & 1u, err, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * C::kStage);
          const uint32_t b_base = a_base + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16(d, smem_desc_k_sw128(a_base, kk * 32), smem_desc_k_sw128(b_base, kk * 32), idesc,
                        (kb | kk) != 0);
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[a]);
      }
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter = warp % 4
    pdl_wait();
    const int q = warp & 3;
    const uint32_t t_lane = (uint32_t)(q * 32) << 16;
    int ti = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++ti) {
      const int a = ti % kAcc;
      const uint32_t around = ti / kAcc;
      const int m0 = (t % mt) * 128, n0 = (t / mt) * BN;
      const int r = m0 + q * 32 + lane;
      // operands of the first chunk and the row's norm scale load while the MMAs run
      const float rs = r < M ? consumer_rstd<EPI>(e, r) : 1.f;
      const int pos = r < M ? epi_pos<EPI>(e, e.out_row0 + r) : 0;
      EpiIn in[kEpiAhead + 1];
#pragma unroll
      for (int c = 0; c < kEpiAhead * 32 && c < BN; c += 32)
        if (r < M) epi_fetch<EPI>(e, r, n0 + c, pos, in[c >> 5]);
      const bool ok = mbar_wait(&acc_full[a], around & 1u, err, kErrTimeoutEpilogue);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float ssq = 0.f;
#pragma unroll
      for (int c = 0; c < BN; c += 32) {
        const int ci = c >> 5;
        if (c + kEpiAhead * 32 < BN && r < M)
          epi_fetch<EPI>(e, r, n0 + c + kEpiAhead * 32, pos, in[(ci + kEpiAhead) % (kEpiAhead + 1)]);
        float v[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t)(a * C::kTmemCols) + t_lane + (uint32_t)c, v);
        if (r < M) ssq += epilogue32<EPI>(e, r, n0 + c, v, rs, in[ci % (kEpiAhead + 1)]);
      }
      if (r < M) norm_partial_store<EPI>(e, r, n0, BN, N, ssq);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAcc * C::kTmemCols);
  }
}

template <int BN, int STAGES, int EPI, int AR>
static void launch_cfg(const CUtensorMap &tmA, const CUtensorMap &tmB, int a_row0, int M, int N, int K, int splits,
                       const EpiArgs &e, unsigned *err, cudaStream_t s) {
  using C = TcCfg<BN, STAGES, AR>;
  const int nk = K / 64;
  if (splits == 1 && 2 * C::kTmemCols <= 512) {
    auto kern = k_gemm_tc_persist<BN, STAGES, EPI, AR>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = ((M + 127) / 128) * (N / BN);
    launch_pdl(kern, tiles < sms ? tiles : sms, 192, C::kSmem, s, tmA, tmB, a_row0, M, N, nk, e, err);
    return;
  }
  auto kern = k_gemm_tc<BN, STAGES, EPI, AR>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  const int kps = (nk + splits - 1) / splits;
  splits = (nk + kps - 1) / kps;
  dim3 grid((M + 127) / 128, N / BN, splits);
  launch_pdl(kern, grid, 128, C::kSmem, s, tmA, tmB, a_row0, M, nk, kps, e, err);
}

template <int EPI>
static void launch_epi(const CUtensorMap &tmA, const CUtensorMap &tmB, const TcPlan &p, int a_row0, int M, int N,
                       int K, const EpiArgs &e, unsigned *err, cudaStream_t s) {
  const int splits = p.splits;
  switch (p.bn) {
    case 32: launch_cfg<32, 8, EPI, 128>(tmA, tmB, a_row0, M, N, K, splits, e, err, s); break;
    case 64:
      // 64-wide tiles (small batches): 12 stages of 16 KB with 64-row activation
      // tiles, else kBn64Stages of 24 KB
      if (p.a_rows == 64)
        launch_cfg<64, 12, EPI, 64>(tmA, tmB, a_row0, M, N, K, splits, e, err, s);
      else
        launch_cfg<64, kBn64Stages, EPI, 128>(tmA, tmB, a_row0, M, N, K, splits, e, err, s);
      break;
    case 128: launch_cfg<128, 5, EPI, 128>(tmA, tmB, a_row0, M, N, K, splits, e, err, s); break;
    case 256: launch_cfg<256, 4, EPI, 128>(tmA, tmB, a_row0, M, N, K, splits, e, err, s); break;
    default: break;
  }
}

TcPlan plan_gemm_tc(int M, int N, int K) {
  TcPlan p;
  const int mt = (M + 127) / 128;
  const int nk = K / 64;
  if (mt >= 8) {
    p.bn = N >= 2048 ? 256 : 128;
    p.splits = 1;
    return p;
  }
  p.bn = 64;
  p.a_rows = M <= 64 ? 64 : 128;
  const int ctas = mt * (N / 64);
  int sp = ctas >= 148 ? 1 : 148 / ctas;
  if (sp > nk / 2) sp = nk / 2 > 0 ? nk / 2 : 1;
  const int kps = (nk + sp - 1) / sp;
  p.splits = (nk + kps - 1) / kps;
  return p;
}

size_t gemm_tc_partial_floats(int M, int N, const TcPlan &p) {
  if (p.splits <= 1) return 0;
  return (size_t)((M + 127) / 128) * (N / p.bn) * p.splits * 128 * p.bn;
}

void launch_gemm_tc(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const TcPlan &p, int a_row0, int M,
                    int N, int K, const EpiArgs &e, unsigned *err, cudaStream_t s) {
  if (M <= 0) return;
  switch (epi) {
    case EPI_STORE_F32: launch_epi<EPI_STORE_F32>(tmA, tmB, p, a_row0, M, N, K, e, err, s); break;
    case EPI_BIAS_F32: launch_epi<EPI_BIAS_F32>(tmA, tmB, p, a_row0, M, N, K, e, err, s); break;
    case EPI_VEC_SILU: launch_epi<EPI_VEC_SILU>(tmA, tmB, p, a_row0, M, N, K, e, err, s); break;
    case EPI_RESID_F32: launch_epi<EPI_RESID_F32>(tmA, tmB, p, a_row0, M, N, K, e, err, s); break;
    case EPI_QKV_ROPE: launch_epi<EPI_QKV_ROPE>(tmA, tmB, p, a_row0, M, N, K, e, err, s); break;
    case EPI_GEGLU: launch_epi<EPI_GEGLU>(tmA, tmB, p, a_row0, M, N, K, e, err, s); break;
    default: break;
  }
}

}  // namespace pi0x
