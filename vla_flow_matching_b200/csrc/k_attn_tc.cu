// Masked MQA attention on the tcgen05 tensor cores (bf16 mode).
//
// Computes, per sample and per query head, softmax(q . K^T / sqrt(256) + mask) . V
// over the valid prefix keys, the state key and the action keys (`_attend` with the
// block mask of `denoise_step` on the vllm-omni pi0 page, or with the Wall-X page's
// causal action mask: action i sees actions 0..i).  The 8 query heads share
// the one KV head, so a CTA takes 128 query rows (token-major: row = token*8 + head)
// of one sample against the sample's keys, in blocks of 64 key slots.
//
// Key slots of sample b: ceil(nv/64) blocks holding the nv valid prefix positions in
// order (the compacted list of the mask), then ceil((H+1)/64) blocks holding the H
// action keys and then the state key; the remaining slots are empty.  Softmax is
// invariant to the order of the keys.  Masked prefix positions are never read (the
// page adds -2.38e38 to their logits, whose exp is exactly 0 in fp32).
//
// Warp roles (256 threads):
//  * warps 0-3: one query row per thread.  Q goes to TMEM (the A operand of
//    S = Q K^T); per key block the thread reads its S row from TMEM, forms
//    P = 2^(s - m) with an online softmax, writes P (bf16) to shared memory, and
//    rescales O in TMEM when the running max grows by more than 2^8 (rare).
//  * warp 4 / warp 5: K / V loader into 3-deep rings of 128-byte-swizzled tiles.  A
//    block whose 64 slots are consecutive rows of one tensor is one 64-row TMA box
//    per 64 dims; otherwise each such run of 8 slots is an 8-row box, and other runs
//    are copied row by row with cp.async.
//  * warp 6 / warp 7: tcgen05.mma issuers of S = Q K^T / of O += P V (the whole warp
//    runs the loop, one elected lane issues).  An MMA costs its issuing warp a fixed
//    time, so the two streams (16 and 4 MMAs per block) are issued side by side; S
//    runs up to two blocks ahead of the softmax (two S buffers).
// All hand-offs are mbarriers (TMA transaction bytes, cp.async completion, tcgen05
// commits, thread arrivals) and every wait is bounded.  O / l at the end
// normalises.  With split-KV (small batches) every split writes O/l and (m, l) and
// k_attn_combine merges the splits.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

namespace {
constexpr int kRowsPerCta = 128;
constexpr int kKeyBlock = 64;
constexpr int kKBufs = 3;
constexpr int kVBufs = 3;
constexpr int kPBufs = 2;
static_assert(kVBufs >= kPBufs, "P.V completions are tracked per V buffer");
constexpr uint32_t kKVBytes = 64 * 512;       // 4 sub-tiles of [64 keys x 64 dims]
constexpr uint32_t kSubTile = 64 * 128;       // one sub-tile
constexpr uint32_t kAtomBytes = 8 * 128;      // 8 keys x 64 dims: one TMA box
constexpr uint32_t kPBytes = 128 * 128;       // [128 rows x 64 keys]
constexpr uint32_t kSmemK0 = 0;
constexpr uint32_t kSmemV0 = kSmemK0 + kKBufs * kKVBytes;
constexpr uint32_t kSmemP0 = kSmemV0 + kVBufs * kKVBytes;
constexpr uint32_t kSmemBar = kSmemP0 + kPBufs * kPBytes;
constexpr int kNumBars = 2 * kKBufs /* k_full, k_empty */ + 2 * kVBufs /* v_full, pv_done */ +
                         2 * 2 /* s_full, s_empty */ + kPBufs /* p_full */ + 2 /* q_full, mma_done */;
constexpr uint32_t kSmemTotal = kSmemBar + kNumBars * 8 + 16 + 1024;  // + TMEM slot + alignment slack
static_assert(kSmemTotal <= 232448, "shared memory per CTA");
// TMEM: S buffers at columns 0 and 64, Q (A operand of S = Q K^T: bf16 pairs,
// K-major, row = lane) at 128..255, O at 256..511
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQ = 128;
constexpr uint32_t kTmemO = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;  // log2 units
constexpr int kThreads = 256;
constexpr unsigned kFull = 0xffffffffu;
}  // namespace

// Source of key slot kk of sample b: 2*row for row `row` of the prefix tensor (B*P
// rows), 2*row+1 for row `row` of this layer's suffix K/V, -1 for an empty slot.
// `contig`: the valid prefix positions are exactly [0, nv), so slot kk is position kk
// and the valid-index list need not be read.
__device__ __forceinline__ int slot_code(int kk, int nbp, int nv, bool contig, int b, const Geo &g, const int *vi) {
  const int pre = nbp * kKeyBlock;
  if (kk < pre) return kk < nv ? 2 * (b * g.P + (contig ? kk : vi[kk])) : -1;
  const int s = kk - pre;
  if (s < g.H) return 2 * (g.B + b * g.H + s) + 1;  // action key s
  if (s == g.H) return 2 * b + 1;                     // state key
  return -1;
}

// One warp fills the [64 keys x 256] tile at `tile` (4 sub-tiles of 64 dims) with the
// K or V rows of key block `blk`.  A block whose 64 slots are consecutive rows of one
// tensor is one 64-row TMA box per sub-tile.  Otherwise each 8-slot atom whose slots
// are consecutive rows of one tensor, or are all empty, is one 8-row box per sub-tile
// (an empty atom is read at row -8, entirely out of bounds, which fills zeros and
// reads nothing), and every other atom is copied row by row with cp.async (16 B per
// lane, zeros for empty slots).  `full` completes on the TMA bytes plus one cp.async
// arrival per lane.  Maps: p* = prefix, s* = suffix; *64 = 64-row boxes.
__device__ __forceinline__ void load_kv_tile(int blk, uint32_t tile, uint64_t *full, const CUtensorMap *pmap,
                                             const CUtensorMap *smap, const CUtensorMap *pmap64,
                                             const CUtensorMap *smap64, int sfx_row0, const bf16 *pref,
                                             const bf16 *suf, int nbp, int nv, bool contig, int b, const Geo &g,
                                             const int *vi, int lane) {
  const int kb = blk * kKeyBlock;
  int code[2];
  code[0] = slot_code(kb + lane, nbp, nv, contig, b, g, vi);
  code[1] = slot_code(kb + 32 + lane, nbp, nv, contig, b, g, vi);
  const int c0 = __shfl_sync(kFull, code[0], 0);
  if (__all_sync(kFull, c0 >= 0 && code[0] == c0 + 2 * lane && code[1] == c0 + 2 * (32 + lane))) {
    if (lane == 0) {
      mbar_expect_tx(full, kKVBytes);
      const CUtensorMap *m = (c0 & 1) ? smap64 : pmap64;
      const int y = (c0 & 1) ? sfx_row0 + (c0 >> 1) : (c0 >> 1);
#pragma unroll
      for (int sub = 0; sub < 4; ++sub) tma_load_2d(tile + sub * kSubTile, m, sub * 64, y, full);
    }
    __syncwarp();
    cp_async_mbar_arrive(full);
    return;
  }
  unsigned tma_atoms = 0, copy_atoms = 0;  // bit a: slots [8a, 8a + 8)
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int lead = __shfl_sync(kFull, code[hh], lane & ~7);
    const bool run = lead >= 0 && code[hh] == lead + 2 * (lane & 7);
    const unsigned br = __ballot_sync(kFull, run), be = __ballot_sync(kFull, code[hh] < 0);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const bool whole = ((br >> (8 * a)) & 0xffu) == 0xffu || ((be >> (8 * a)) & 0xffu) == 0xffu;
      (whole ? tma_atoms : copy_atoms) |= 1u << (4 * hh + a);
    }
  }
  if (lane == 0 && tma_atoms) mbar_expect_tx(full, (uint32_t)__popc(tma_atoms) * 4u * kAtomBytes);
  __syncwarp();
  if ((lane & 7) == 0) {  // lane 8i issues atoms i and 4 + i
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int a = 4 * hh + (lane >> 3);
      if (!((tma_atoms >> a) & 1u)) continue;
      const int c = code[hh];
      const CUtensorMap *m = (c >= 0 && !(c & 1)) ? pmap : smap;
      const int y = c < 0 ? -8 : (c & 1) ? sfx_row0 + (c >> 1) : (c >> 1);
#pragma unroll
      for (int sub = 0; sub < 4; ++sub) tma_load_2d(tile + sub * kSubTile + a * kAtomBytes, m, sub * 64, y, full);
    }
  }
  while (copy_atoms) {  // warp-uniform
    const int a = __ffs(copy_atoms) - 1;
    copy_atoms &= copy_atoms - 1;
    const int hh = a >> 2, l0 = (a & 3) * 8;
#pragma unroll 4
    for (int r = 0; r < 8; ++r) {
      const int c = __shfl_sync(kFull, hh ? code[1] : code[0], l0 + r);
      const bf16 *row = c < 0 ? suf : ((c & 1) ? suf : pref) + (size_t)(c >> 1) * kHeadDim;
      cp_async16(tile + (lane >> 3) * kSubTile + sw128_off(8 * a + r, lane & 7), row + lane * 8, c >= 0);
    }
  }
  cp_async_mbar_arrive(full);
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(const bf16 *q, const bf16 *ks, const bf16 *vs, const CallPtrs *cp, int layer, int sfx_row0,
              const int *nvalid, const int *vidx, Geo g, int step0, int causal, int blocks_per_split, bf16 *out,
              float *part_o, float *part_ml, unsigned *err) {
  pdl_wait();
  pdl_trigger();
  if (*(volatile unsigned *)err != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kSmemBar);
  uint64_t *k_full = bars, *k_empty = bars + kKBufs;
  uint64_t *v_full = bars + 2 * kKBufs, *pv_done = v_full + kVBufs;
  uint64_t *s_full = pv_done + kVBufs, *s_empty = s_full + 2;
  uint64_t *p_full = s_empty + 2, *q_full = p_full + kPBufs, *mma_done = q_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, split = blockIdx.y, nsplit = gridDim.y;
  const int Tq = step0 ? g.H + 1 : g.H;
  const int nrows = kHeads * Tq;
  const int row0 = blockIdx.x * kRowsPerCta;
  const int nv = nvalid[b];
  const int nbp = (nv + kKeyBlock - 1) / kKeyBlock;  // prefix blocks, then the suffix blocks
  const int nblk_all = nbp + (g.H + kKeyBlock) / kKeyBlock;
  const int blk0 = split * blocks_per_split;
  const int blk1 = min(nblk_all, blk0 + blocks_per_split);
  const int nb = blk1 > blk0 ? blk1 - blk0 : 0;

  if (tid == 0) {
    for (int i = 0; i < kKBufs; ++i) {
      mbar_init(&k_full[i], 32);  // one cp.async-completion arrival per loader lane (+ TMA bytes)
      mbar_init(&k_empty[i], 1);  // tcgen05.commit after S
    }
    for (int i = 0; i < kVBufs; ++i) {
      mbar_init(&v_full[i], 32);
      mbar_init(&pv_done[i], 1);  // tcgen05.commit after P.V
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);     // tcgen05.commit after S
      mbar_init(&s_empty[i], 128);  // every softmax thread has read its S row
    }
    for (int i = 0; i < kPBufs; ++i) mbar_init(&p_full[i], 128);
    mbar_init(q_full, 128);
    mbar_init(mma_done, 2);  // one commit per MMA-issuing warp
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 4 || warp == 5) {
    // ------------------------------------------------------------ K / V loaders
    const bool is_v = warp == 5;
    const CUtensorMap *pmap = &cp->kv_map[is_v][layer], *smap = &cp->sfx_map[is_v];
    const CUtensorMap *pmap64 = &cp->kv_map64[is_v][layer], *smap64 = &cp->sfx_map64[is_v];
    const bf16 *pref = is_v ? cp->prefix_v[layer] : cp->prefix_k[layer];
    const bf16 *suf = is_v ? vs : ks;
    const int *vi = vidx + (size_t)b * g.P;
    // the list is strictly increasing, so its last entry is nv - 1 iff it is 0 .. nv-1
    const bool contig = nv == 0 || vi[nv - 1] == nv - 1;
    const int nbuf = is_v ? kVBufs : kKBufs;
    uint64_t *full = is_v ? v_full : k_full;
    // a buffer is free again once S (K) or P.V (V) of the block it held has completed
    uint64_t *empty = is_v ? pv_done : k_empty;
    const uint32_t ring = sbase + (is_v ? kSmemV0 : kSmemK0);
    // (the prefix map is unused, and zero, when there is no prefix key).  Every lane that
    // may issue a tensor copy acquires the maps itself: the fence orders the executing
    // thread's tensor-map accesses only.
    if (nv > 0) {
      tma_map_acquire(pmap);
      tma_map_acquire(pmap64);
    }
    tma_map_acquire(smap);
    tma_map_acquire(smap64);
    if (lane == 0) {
      if (nv > 0) {
        tma_prefetch_desc(pmap);
        tma_prefetch_desc(pmap64);
      }
      tma_prefetch_desc(smap);
      tma_prefetch_desc(smap64);
    }
    __syncwarp();
    for (int j = 0; j < nb; ++j) {
      const int buf = j % nbuf;
      if (j >= nbuf) ok = __all_sync(kFull, mbar_wait(&empty[buf], ((j / nbuf) - 1) & 1, err, kErrTimeoutProducer));
      if (!ok) break;
      load_kv_tile(blk0 + j, ring + buf * kKVBytes, &full[buf], pmap, smap, pmap64, smap64, sfx_row0, pref, suf, nbp,
                   nv, contig, b, g, vi, lane);
    }
    cp_async_commit();  // nothing may still land in shared memory once the CTA exits
    cp_async_wait<0>();
  } else if (warp == 6 || warp == 7) {
    // ------------------------------------------------------------ MMA issuers
    // The whole warp runs the loop (waits and descriptors stay warp-uniform); one
    // elected lane issues each MMA and commit.
    if (nb > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKeyBlock);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim) | (1u << 16);  // B (V) MN-major
      // descriptor bases; the start-address field (bits 0..13, address >> 4) takes byte
      // offsets >> 4 directly: every operand lies below 256 KB
      const uint64_t kdesc0 = smem_desc_k_sw128(sbase + kSmemK0, 0);
      const uint64_t pdesc0 = smem_desc_k_sw128(sbase + kSmemP0, 0);
      const uint64_t vdesc0 = smem_desc_mn_sw128(sbase + kSmemV0, 64 * 128, 1024);
      auto issue_s = [&](int j) -> bool {  // S[j&1] = Q K(j)^T, Q from TMEM
        const int kbuf = j % kKBufs, sb = j & 1;
        if (!__all_sync(kFull, mbar_wait(&k_full[kbuf], (j / kKBufs) & 1, err, kErrTimeoutMma))) return false;
        if (j >= 2 && !__all_sync(kFull, mbar_wait(&s_empty[sb], ((j >> 1) - 1) & 1, err, kErrTimeoutMma)))
          return false;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint64_t kd = kdesc0 + (uint64_t)((kbuf * kKVBytes) >> 4);
        const uint32_t d = tmem + (uint32_t)(sb * kKeyBlock);
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16_ts_w(d, tmem + kTmemQ + (uint32_t)(32 * s + 8 * kk),
                             kd + (uint64_t)((s * kSubTile + kk * 32) >> 4), idesc_s, (s | kk) != 0);
        tc_commit_w(&s_full[sb]);
        tc_commit_w(&k_empty[kbuf]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {  // O += P(j) V(j)
        const int vbuf = j % kVBufs, pb = j % kPBufs;
        if (!__all_sync(kFull, mbar_wait(&p_full[pb], (j / kPBufs) & 1, err, kErrTimeoutMma))) return false;
        if (!__all_sync(kFull, mbar_wait(&v_full[vbuf], (j / kVBufs) & 1, err, kErrTimeoutMma))) return false;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint64_t pd = pdesc0 + (uint64_t)((pb * kPBytes) >> 4);
        const uint64_t vd = vdesc0 + (uint64_t)((vbuf * kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16_w(tmem + kTmemO, pd + (uint64_t)((kk * 32) >> 4), vd + (uint64_t)((kk * 2048) >> 4), idesc_o,
                        (j | kk) != 0);
        tc_commit_w(&pv_done[vbuf]);  // V buffer and P buffer free, O updated
        return true;
      };
      if (warp == 6) {
        ok = __all_sync(kFull, mbar_wait(q_full, 0, err, kErrTimeoutMma));
        tc_fence_after();
        for (int j = 0; j < nb && ok; ++j) ok = issue_s(j);
      } else {
        for (int j = 0; j < nb && ok; ++j) ok = issue_pv(j);
      }
      // every MMA issued by either warp (also after a failed wait) has finished before
      // TMEM is freed
      tc_commit_w(mma_done);
      mbar_wait(mma_done, 0, err, kErrTimeoutMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0..3
    const int qi = row0 + tid;
    const bool row_ok = qi < nrows;
    const int jq = qi / kHeads, head = qi % kHeads;
    int tok = 0;
    if (row_ok) tok = step0 ? (jq == 0 ? b : g.B + b * g.H + jq - 1) : g.B + b * g.H + jq;
    const bool state_q = step0 && jq == 0;
    const int ja = step0 ? jq - 1 : jq;  // action index of an action query
    // Visible suffix slots (actions at base + 0..H-1, the state at base + H): the
    // state query sees the state slot only; an action query sees all of them, or
    // under the causal action mask actions 0..ja plus the state slot.
    const int sfx_base = nbp * kKeyBlock;
    const int sfx_lo = sfx_base + (state_q ? g.H : 0);
    const int sfx_hi = state_q ? sfx_base + g.H + 1 : (causal ? sfx_base + ja + 1 : sfx_base + g.H + 1);
    const int sfx_state = sfx_base + g.H;
    const uint32_t t_lane = (uint32_t)(warp * 32) << 16;
    const float scale_l2 = 0.0625f * kLog2e;

    // Q row -> TMEM lane tid, columns 128..255 (two bf16 per 32-bit column)
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
      tc_fence_before();
      mbar_arrive(q_full);
    }

    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < nb && ok; ++j) {
      const int sb = j & 1, pb = j % kPBufs;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1, err, kErrTimeoutEpilogue));
      if (!ok) break;
      tc_fence_after();
      float sv[64];  // raw logits q.k of this row and block
      tmem_ld_32x32b_x64(tmem + t_lane + sb * kKeyBlock, sv);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      const int kbase = (blk0 + j) * kKeyBlock;
      const bool pre_blk = blk0 + j < nbp;
      const int vis_lo = pre_blk ? 0 : sfx_lo, vis_hi = pre_blk ? nv : sfx_hi;
      const int vis_st = pre_blk ? -1 : sfx_state;  // also visible (the range may end before it)
      if (kbase < vis_lo || kbase + kKeyBlock > vis_hi) {  // some slot of the block is hidden from this row
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if ((unsigned)(kbase + i - vis_lo) >= (unsigned)(vis_hi - vis_lo) && kbase + i != vis_st) sv[i] = -INFINITY;
      }
      float bm;
      {  // block max in log2 units (the scale is positive); eight independent chains
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = sv[k];
#pragma unroll
        for (int i = 8; i < 64; ++i) mx[i & 7] = fmaxf(mx[i & 7], sv[i]);
        bm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        bm *= scale_l2;
      }
      // Raise m_used (and rescale l, O) when this block's max exceeds it by more than
      // 2^8.  O lives in TMEM and tcgen05.ld/st are warp-collective, so the whole warp
      // takes the branch when any lane needs it; the other lanes scale by 1 (exact).
      const bool mine = bm > m_used + kRescaleSlack;
      if (__any_sync(0xffffffffu, mine)) {
        const float alpha = mine ? ex2_approx(m_used - bm) : 1.0f;  // 0 while m_used = -inf
        l *= alpha;
        if (j >= 1) {  // O holds P.V of blocks < j: wait for the last of them
          const int pj = j - 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[pj % kVBufs], (pj / kVBufs) & 1, err, kErrTimeoutEpilogue));
          if (!ok) break;
          tc_fence_after();
          for (int c = 0; c < kHeadDim; c += 32) {
            float o[32];
            tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st_32x32b_x32(tmem + t_lane + kTmemO + c, o);
          }
          tc_fence_before();
        }
        if (mine) m_used = bm;
      }
      // P buffer pb was last read by P.V(j - 2)
      if (j >= kPBufs) {
        const int pj = j - kPBufs;
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[pj % kVBufs], (pj / kVBufs) & 1, err, kErrTimeoutEpilogue));
        if (!ok) break;
      }
      {
        // no visible key seen yet <=> m_used = -inf <=> every sv is -inf: use 0 so that 2^(-inf) = 0
        const float mu = m_used == -INFINITY ? 0.f : m_used;
        uint8_t *prow = smem + kSmemP0 + pb * kPBytes;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};  // partial row sums (independent chains)
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = cc * 8 + 2 * e;
            const float p0 = ex2_approx(fmaf(sv[i0], scale_l2, -mu)), p1 = ex2_approx(fmaf(sv[i0 + 1], scale_l2, -mu));
            ls[e] += p0 + p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<const uint32_t *>(&h2);
          }
          *reinterpret_cast<uint4 *>(prow + sw128_off(tid, cc)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&p_full[pb]);
    }
    // final P.V
    if (nb > 0 && ok) {
      const int pj = nb - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[pj % kVBufs], (pj / kVBufs) & 1, err, kErrTimeoutEpilogue));
    }
    tc_fence_after();
    const bool write = __all_sync(0xffffffffu, ok);
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
              d4[e] = make_float4(v[4 * e] * inv_l, v[4 * e + 1] * inv_l, v[4 * e + 2] * inv_l,
                                  v[4 * e + 3] * inv_l);
          }
        }
        if (row_ok) {
          part_ml[2 * prow] = m_used;
          part_ml[2 * prow + 1] = l;
        }
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

int attn_tc_blocks(int P, int H) { return (P + kKeyBlock - 1) / kKeyBlock + (H + kKeyBlock) / kKeyBlock; }

int attn_tc_splits(const Geo &g, int step0) {
  const int Tq = step0 ? g.H + 1 : g.H;
  const int mtiles = (kHeads * Tq + kRowsPerCta - 1) / kRowsPerCta;
  const int nblk = attn_tc_blocks(g.P, g.H);
  const int ctas = mtiles * g.B;
  if (ctas >= 96) return 1;
  int splits = (148 + ctas - 1) / ctas;
  const int max_split = (nblk + 3) / 4;  // at least four key blocks per split
  if (splits > max_split) splits = max_split;
  return splits < 1 ? 1 : splits;
}

size_t attn_tc_partial_floats(const Geo &g, int step0, int splits) {
  if (splits <= 1) return 0;
  const int Tq = step0 ? g.H + 1 : g.H;
  const int mtiles = (kHeads * Tq + kRowsPerCta - 1) / kRowsPerCta;
  return (size_t)g.B * splits * mtiles * kRowsPerCta * (kHeadDim + 2);
}

bool attn_tc_maps(CallPtrs &cp, int layers, int B, int P, const void *ks, const void *vs, uint64_t sfx_rows) {
  for (int l = 0; l < layers && P > 0; ++l)
    for (int kv = 0; kv < 2; ++kv) {
      const void *base = kv ? cp.prefix_v[l] : cp.prefix_k[l];
      if (!make_map(&cp.kv_map[kv][l], base, (uint64_t)B * P, kHeadDim, kHeadDim, 8) ||
          !make_map(&cp.kv_map64[kv][l], base, (uint64_t)B * P, kHeadDim, kHeadDim, 64))
        return false;
    }
  for (int kv = 0; kv < 2; ++kv) {
    const void *base = kv ? vs : ks;
    if (!make_map(&cp.sfx_map[kv], base, sfx_rows, kHeadDim, kHeadDim, 8) ||
        !make_map(&cp.sfx_map64[kv], base, sfx_rows, kHeadDim, kHeadDim, 64))
      return false;
  }
  return true;
}

bool loop_attn_maps(CallPtrs &cp, int layers, int B, int P, const void *ks, const void *vs, uint64_t sfx_rows) {
  for (int l = 0; l < layers && P > 0; ++l)
    for (int kv = 0; kv < 2; ++kv) {
      const void *base = kv ? cp.prefix_v[l] : cp.prefix_k[l];
      if (!make_map(&cp.kv_map32[kv][l], base, (uint64_t)B * P, kHeadDim, kHeadDim, 32)) return false;
    }
  for (int kv = 0; kv < 2; ++kv)
    if (!make_map(&cp.sfx_map32[kv], kv ? vs : ks, sfx_rows, kHeadDim, kHeadDim, 32)) return false;
  return true;
}

void launch_attention_tc(const bf16 *q, const bf16 *ks, const bf16 *vs, const CallPtrs *cp, int layer,
                         int sfx_row0, const int *nvalid, const int *vidx, const Geo &g, int step0, int causal,
                         int splits, bf16 *out, float *part, unsigned *err, cudaStream_t s) {
  cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
  const int Tq = step0 ? g.H + 1 : g.H;
  const int mtiles = (kHeads * Tq + kRowsPerCta - 1) / kRowsPerCta;
  const int nblk = attn_tc_blocks(g.P, g.H);
  const int bps = (nblk + splits - 1) / splits;
  float *part_o = part;
  float *part_ml = splits > 1 ? part + (size_t)g.B * splits * mtiles * kRowsPerCta * kHeadDim : nullptr;
  dim3 grid(mtiles, splits, g.B);
  launch_pdl(k_attn_tc, grid, kThreads, kSmemTotal, s, q, ks, vs, cp, layer, sfx_row0, nvalid, vidx, g, step0,
             causal, bps, out, part_o, part_ml, err);
  if (splits > 1) {
    dim3 cg((kHeads * Tq + 7) / 8, g.B);
    launch_pdl(k_attn_combine, cg, 256, 0, s, part_o, part_ml, g, step0, splits, mtiles * kRowsPerCta, out);
  }
}

}  // namespace pi0x
