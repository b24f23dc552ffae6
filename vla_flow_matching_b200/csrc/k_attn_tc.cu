// Masked MQA attention on the tcgen05 tensor cores (bf16 mode).
//
// Computes, per sample and per query head, softmax(q . K^T / sqrt(256) + mask) . V
// over [valid prefix keys ; state key ; action keys] (`_attend` with the block mask
// of `denoise_step` on the vllm-omni pi0 page).  The 8 query heads share the one
// KV head, so a CTA takes 128 query rows (token-major: row = token*8 + head) of
// one sample against the sample's key list, in blocks of 64 keys.
//
// Keys are gathered by index with cp.async (16 B per thread) into 128-byte-
// swizzled shared memory, so masked prefix positions are never read; the page adds
// -2.38e38 to their logits, whose exp is exactly 0 in fp32.
//
// One pass over the key blocks with an online softmax.  S = Q K^T goes to one of
// two TMEM buffers, so the MMA of block w+1 runs while the threads (one per query
// row) turn block w into P = 2^(s - m) in bf16 and accumulate O += P V in TMEM.
// The running max m used for P is raised (and O, l rescaled in place) only when a
// block's max exceeds it by more than 2^8, so P stays <= 256 and rescaling is
// rare; O / l at the end normalises.  With split-KV (small batches) every split
// writes O/l and (m, l) and k_attn_combine merges the splits.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

namespace {
constexpr int kRowsPerCta = 128;
constexpr int kKeyBlock = 64;
constexpr int kKBufs = 4;                     // K ring depth (K tiles prefetched 3 blocks ahead)
constexpr uint32_t kKVBytes = 64 * 512;       // 4 sub-tiles of [64 keys x 64 dims]
constexpr uint32_t kPBytes = 128 * 128;       // [128 rows x 64 keys]
constexpr uint32_t kSmemK0 = 0;
constexpr uint32_t kSmemV0 = kSmemK0 + kKBufs * kKVBytes;
constexpr uint32_t kSmemP = kSmemV0 + 2 * kKVBytes;
constexpr uint32_t kSmemBar = kSmemP + kPBytes;
constexpr uint32_t kSmemTotal = kSmemBar + 64 + 1024;  // + alignment slack
// TMEM: S buffers at columns 0 and 64, Q (the A operand of S = Q K^T: bf16 pairs,
// K-major, row = lane) at 128..255, O at 256..511
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQ = 128;
constexpr uint32_t kTmemO = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;  // log2 units
}  // namespace

// Source row (256 bf16) of key `kk` of sample b: valid prefix positions first, then
// the state key, then the action keys.
__device__ __forceinline__ const bf16 *key_row(int kk, int nv, int b, const Geo &g, const bf16 *pref,
                                                const int *vi, const bf16 *suf) {
  if (kk < nv) return pref + ((size_t)b * g.P + vi[kk]) * kHeadDim;
  const int row = (kk == nv) ? b : g.B + b * g.H + (kk - nv - 1);
  return suf + (size_t)row * kHeadDim;
}

__global__ void __launch_bounds__(128, 1)
    k_attn_tc(const bf16 *q, const bf16 *ks, const bf16 *vs, const CallPtrs *cp, int layer, const int *nvalid,
              const int *vidx, Geo g, int step0, int blocks_per_split, bf16 *out, float *part_o, float *part_ml,
              unsigned *err) {
  pdl_wait();
  pdl_trigger();
  if (*(volatile unsigned *)err != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(smem + kSmemBar);  // [2]
  uint64_t *bar_o = bar_s + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_s + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, split = blockIdx.y, nsplit = gridDim.y;
  const int Tq = step0 ? g.H + 1 : g.H;
  const int nrows = kHeads * Tq;
  const int row0 = blockIdx.x * kRowsPerCta;
  const int nv = nvalid[b];
  const int nk = nv + 1 + g.H;
  const int nblk_all = (nk + kKeyBlock - 1) / kKeyBlock;
  const int blk0 = split * blocks_per_split;
  const int blk1 = min(nblk_all, blk0 + blocks_per_split);
  const int nb = blk1 > blk0 ? blk1 - blk0 : 0;

  // this thread's query row
  const int qi = row0 + tid;
  const bool row_ok = qi < nrows;
  const int jq = qi / kHeads, head = qi % kHeads;
  int tok = 0;
  if (row_ok) tok = step0 ? (jq == 0 ? b : g.B + b * g.H + jq - 1) : g.B + b * g.H + jq;
  const bool state_q = step0 && jq == 0;
  const int key_lim = state_q ? nv + 1 : nk;  // keys [0, key_lim) visible to this row

  const bf16 *pref_k = cp->prefix_k[layer], *pref_v = cp->prefix_v[layer];
  const int *vi = vidx + (size_t)b * g.P;

  if (tid == 0) {
    mbar_init(&bar_s[0], 1);
    mbar_init(&bar_s[1], 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }

  // Warp w copies keys [16w, 16w+16) of block j, lane = 16-byte chunk of the 512-byte
  // row.  Lanes 0..15 first look up one key's source row each (independent loads),
  // then every copy takes its row pointer from a shuffle.  `which`: 1 = K, 2 = V.
  auto load_block = [&](int j, int which) {
    if (j >= nb) return;
    const int blk = blk0 + j;
    const uint32_t kb = sbase + kSmemK0 + (j % kKBufs) * kKVBytes, vb = sbase + kSmemV0 + (j & 1) * kKVBytes;
    const int kk_l = blk * kKeyBlock + warp * 16 + (lane & 15);
    const bool ok_l = kk_l < nk;
    const bf16 *krow = ks, *vrow = vs;
    if (ok_l) {
      if (which & 1) krow = key_row(kk_l, nv, b, g, pref_k, vi, ks);
      if (which & 2) vrow = key_row(kk_l, nv, b, g, pref_v, vi, vs);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = warp * 16 + i;
      const bool ok = __shfl_sync(0xffffffffu, ok_l, i);
      const uint32_t off = (lane >> 3) * (64 * 128) + sw128_off(r, lane & 7);
      if (which & 1) {
        const bf16 *ksrc = reinterpret_cast<const bf16 *>(
            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(krow), i));
        cp_async16(kb + off, ksrc + lane * 8, ok);
      }
      if (which & 2) {
        const bf16 *vsrc = reinterpret_cast<const bf16 *>(
            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(vrow), i));
        cp_async16(vb + off, vsrc + lane * 8, ok);
      }
    }
  };

  // cp.async groups, committed in this order (empty groups keep the pattern):
  //   prologue: [K0, V0] [K1] [K2] [K3] [V1];
  //   iteration w: [K(w+4)] after S(w), [V(w+1)] after PV(w-1) (empty at w = 0)
  load_block(0, 3);
  cp_async_commit();
  load_block(1, 1);
  cp_async_commit();
  load_block(2, 1);
  cp_async_commit();
  load_block(3, 1);
  cp_async_commit();
  load_block(1, 2);
  cp_async_commit();

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_lane = (uint32_t)(warp * 32) << 16;

  // ---- Q: this thread's query row (256 bf16) into TMEM lane `tid`, columns 128..255,
  // two bf16 per 32-bit column (the K-major A-operand layout of tcgen05.mma) ----
  {
    const uint4 *src = reinterpret_cast<const uint4 *>(q + (size_t)tok * kQDim + head * kHeadDim);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint4 u = row_ok ? src[c * 8 + e] : make_uint4(0, 0, 0, 0);
        v[4 * e] = __uint_as_float(u.x);
        v[4 * e + 1] = __uint_as_float(u.y);
        v[4 * e + 2] = __uint_as_float(u.z);
        v[4 * e + 3] = __uint_as_float(u.w);
      }
      tmem_st_32x32b_x32(tmem + t_lane + kTmemQ + 32 * c, v);
    }
  }

  constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKeyBlock);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim) | (1u << 16);  // B (V) MN-major
  const float scale_l2 = 0.0625f * kLog2e;

  auto issue_s = [&](int j) {  // S[j&1] = Q K(j)^T, A (Q) from TMEM, 16 head dims per MMA
    const uint32_t kb = sbase + kSmemK0 + (j % kKBufs) * kKVBytes;
    const uint32_t d = tmem + (uint32_t)((j & 1) * kKeyBlock);
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc_mma_bf16_ts(d, tmem + kTmemQ + (uint32_t)(32 * s + 8 * kk), smem_desc_k_sw128(kb + s * (64 * 128), kk * 32),
                       idesc_s, (s | kk) != 0);
    tc_commit(&bar_s[j & 1]);
  };

  float m_used = -INFINITY, l = 0.f;
  uint32_t ph_s0 = 0, ph_s1 = 0, ph_o = 0;
  bool ok_all = true;
  if (nb > 0) {
    cp_async_wait<4>();
    fence_proxy_async_smem();
    tc_fence_before();
    ok_all = __syncthreads_and(ok_all);
    tc_fence_after();
    if (tid == 0 && ok_all) issue_s(0);
  }
  for (int w = 0; w < nb && ok_all; ++w) {
    const int buf = w & 1;
    // (1) K(w+1) has landed: start S(w+1) on the tensor cores before the softmax of w.
    // Groups committed after K(w+1): 3 at w = 0, 4 at w = 1, then 5.
    if (w + 1 < nb) {
      if (w == 0)
        cp_async_wait<3>();
      else if (w == 1)
        cp_async_wait<4>();
      else
        cp_async_wait<5>();
      fence_proxy_async_smem();
      tc_fence_before();
      ok_all = __syncthreads_and(ok_all);
      tc_fence_after();
      if (!ok_all) break;
      if (tid == 0) issue_s(w + 1);
    }
    // (2) softmax of block w
    {
      uint32_t &ph = buf ? ph_s1 : ph_s0;
      if (!mbar_wait(&bar_s[buf], ph, err, kErrTimeoutEpilogue)) ok_all = false;
      ph ^= 1u;
    }
    __syncwarp();
    tc_fence_after();
    // K(w)'s buffer is free again (S(w) done): prefetch K(w+4)
    load_block(w + kKBufs, 1);
    cp_async_commit();
    float sv[64];
    {
      float t0[32], t1[32];
      tmem_ld_32x32b_x32(tmem + t_lane + buf * kKeyBlock, t0);
      tmem_ld_32x32b_x32(tmem + t_lane + buf * kKeyBlock + 32, t1);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sv[i] = t0[i];
        sv[32 + i] = t1[i];
      }
    }
    const int kbase = (blk0 + w) * kKeyBlock;
    float bm = -INFINITY;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      sv[i] = (kbase + i < key_lim) ? sv[i] * scale_l2 : -INFINITY;
      bm = fmaxf(bm, sv[i]);
    }
    // P(w-1) and O are in use by PV(w-1) until it completes
    if (w >= 1) {
      if (!mbar_wait(bar_o, ph_o, err, kErrTimeoutMma)) ok_all = false;
      ph_o ^= 1u;
      __syncwarp();
      tc_fence_after();
    }
    // V(w-1)'s buffer is free: prefetch V(w+1) (V(1) came with the prologue)
    if (w >= 1) load_block(w + 1, 2);
    cp_async_commit();
    if (bm > m_used + kRescaleSlack) {
      const float alpha = ex2_approx(m_used - bm);  // 0 while m_used = -inf
      l *= alpha;
      if (w >= 1) {
        for (int c = 0; c < kHeadDim; c += 32) {
          float o[32];
          tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st_32x32b_x32(tmem + t_lane + kTmemO + c, o);
        }
      }
      m_used = bm;
    }
    {
      // no visible key seen yet <=> m_used = -inf <=> every sv is -inf: use 0 so that 2^(-inf) = 0
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      uint8_t *prow = smem + kSmemP;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i0 = cc * 8 + 2 * e;
          const float p0 = ex2_approx(sv[i0] - mu), p1 = ex2_approx(sv[i0 + 1] - mu);
          l += p0 + p1;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          pk[e] = *reinterpret_cast<const uint32_t *>(&h2);
        }
        *reinterpret_cast<uint4 *>(prow + sw128_off(tid, cc)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    // V(w) must have landed: groups committed after it are 6 at w = 0 (it came with
    // K0), 4 at w = 1 (it came last in the prologue), then the 2 of this iteration
    if (w == 0)
      cp_async_wait<6>();
    else if (w == 1)
      cp_async_wait<4>();
    else
      cp_async_wait<2>();
    fence_proxy_async_smem();
    tc_fence_before();
    ok_all = __syncthreads_and(ok_all);
    tc_fence_after();
    if (!ok_all) break;
    if (tid == 0) {
      const uint32_t vb = sbase + kSmemV0 + buf * kKVBytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc_mma_bf16(tmem + kTmemO, smem_desc_k_sw128(sbase + kSmemP, kk * 32),
                    smem_desc_mn_sw128(vb + kk * 2048, 64 * 128, 1024), idesc_o, (w | kk) != 0);
      tc_commit(bar_o);
    }
    __syncwarp();
  }
  // last PV MMA
  if (nb > 0 && ok_all) {
    if (!mbar_wait(bar_o, ph_o, err, kErrTimeoutMma)) ok_all = false;
    __syncwarp();
  }
  cp_async_wait<0>();
  tc_fence_after();
  const bool write = __syncthreads_and(ok_all);
  const float inv_l = l > 0.f ? 1.0f / l : 0.f;
  if (write) {
    if (nsplit == 1) {
      bf16 *dst = out + (size_t)tok * kQDim + head * kHeadDim;
      for (int c = 0; c < kHeadDim; c += 32) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c, v);  // warp-collective: all lanes
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * e] * inv_l, v[2 * e + 1] * inv_l);
            pk[e] = *reinterpret_cast<const uint32_t *>(&h2);
          }
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    } else {
      // split partials: O normalised by this split's l, plus (m, l) in log2 units
      const size_t prow = ((size_t)b * nsplit + split) * (size_t)(gridDim.x * kRowsPerCta) + qi;
      for (int c = 0; c < kHeadDim; c += 32) {
        float v[32];
        if (nb > 0) {
          tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c, v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
        if (row_ok) {
          float4 *d4 = reinterpret_cast<float4 *>(part_o + prow * kHeadDim + c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(v[4 * e] * inv_l, v[4 * e + 1] * inv_l, v[4 * e + 2] * inv_l, v[4 * e + 3] * inv_l);
        }
      }
      if (row_ok) {
        part_ml[2 * prow] = m_used;
        part_ml[2 * prow + 1] = l;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge split-KV partials: O = sum_s w_s O_s with w_s = l_s 2^(m_s - M) / sum_t l_t 2^(m_t - M).
__global__ void __launch_bounds__(256) k_attn_combine(const float *part_o, const float *part_ml, Geo g, int step0,
                                                       int nsplit, int rows_pad, bf16 *out) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int Tq = step0 ? g.H + 1 : g.H;
  const int qi = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (qi >= kHeads * Tq) return;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) {
    const size_t pr = ((size_t)b * nsplit + s) * rows_pad + qi;
    if (part_ml[2 * pr + 1] > 0.f) M = fmaxf(M, part_ml[2 * pr]);
  }
  float den = 0.f, acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const size_t pr = ((size_t)b * nsplit + s) * rows_pad + qi;
    const float ms = part_ml[2 * pr], ls = part_ml[2 * pr + 1];
    if (!(ls > 0.f)) continue;
    const float wgt = ls * ex2_approx(ms - M);
    den += wgt;
    const float *src = part_o + pr * kHeadDim;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, src[lane + 32 * e], acc[e]);
  }
  const int j = qi / kHeads, hd = qi % kHeads;
  const int tok = step0 ? (j == 0 ? b : g.B + b * g.H + j - 1) : g.B + b * g.H + j;
  bf16 *dst = out + (size_t)tok * kQDim + hd * kHeadDim;
  const float inv = 1.0f / den;
#pragma unroll
  for (int e = 0; e < 8; ++e) dst[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
}

int attn_tc_splits(const Geo &g, int step0, int max_keys) {
  const int Tq = step0 ? g.H + 1 : g.H;
  const int mtiles = (kHeads * Tq + kRowsPerCta - 1) / kRowsPerCta;
  const int nblk = (max_keys + kKeyBlock - 1) / kKeyBlock;
  const int ctas = mtiles * g.B;
  if (ctas >= 96) return 1;
  int splits = (148 + ctas - 1) / ctas;
  const int max_split = (nblk + 1) / 2;  // at least two key blocks per split
  if (splits > max_split) splits = max_split;
  return splits < 1 ? 1 : splits;
}

size_t attn_tc_partial_floats(const Geo &g, int step0, int splits) {
  if (splits <= 1) return 0;
  const int Tq = step0 ? g.H + 1 : g.H;
  const int mtiles = (kHeads * Tq + kRowsPerCta - 1) / kRowsPerCta;
  return (size_t)g.B * splits * mtiles * kRowsPerCta * (kHeadDim + 2);
}

void launch_attention_tc(const bf16 *q, const bf16 *ks, const bf16 *vs, const CallPtrs *cp, int layer,
                         const int *nvalid, const int *vidx, const Geo &g, int step0, int splits, bf16 *out,
                         float *part, unsigned *err, cudaStream_t s) {
  cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
  const int Tq = step0 ? g.H + 1 : g.H;
  const int mtiles = (kHeads * Tq + kRowsPerCta - 1) / kRowsPerCta;
  const int max_keys = g.P + 1 + g.H;
  const int nblk = (max_keys + kKeyBlock - 1) / kKeyBlock;
  const int bps = (nblk + splits - 1) / splits;
  float *part_o = part;
  float *part_ml = splits > 1 ? part + (size_t)g.B * splits * mtiles * kRowsPerCta * kHeadDim : nullptr;
  dim3 grid(mtiles, splits, g.B);
  launch_pdl(k_attn_tc, grid, 128, kSmemTotal, s, q, ks, vs, cp, layer, nvalid, vidx, g, step0, bps, out, part_o,
             part_ml, err);
  if (splits > 1) {
    dim3 cg((kHeads * Tq + 7) / 8, g.B);
    launch_pdl(k_attn_combine, cg, 256, 0, s, part_o, part_ml, g, step0, splits, mtiles * kRowsPerCta, out);
  }
}

}  // namespace pi0x
