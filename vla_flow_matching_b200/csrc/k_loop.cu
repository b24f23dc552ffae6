// The whole Euler loop of a small batch as one persistent kernel (bf16 mode).
//
// At small batch every Linear of the action expert reads far more weight bytes than
// activation bytes, and a layer is a chain of five dependent contractions (QKV,
// attention, O-proj, gate/up, down) whose weights do not depend on the activations.
// One cooperative launch with one CTA per SM runs every stage of every Euler step of
// the call (`sample_actions` / `denoise_step` / `_compute_layer_suffix_only` on the
// vllm-omni pi0 page) in program order:
//
//   per step: ACTION_IN, TIN (action-time MLP in + SiLU), TOUT (MLP out -> residual
//   stream, layer-0 norm inputs), then per layer QKV (+ RoPE), ATTN (split-KV masked
//   MQA), COMBINE (merge of the splits), O (+ residual), GU (gate/up + GeGLU), DOWN
//   (+ residual, next norm inputs), and last EULER (final norm, out-projection,
//   x += dt v).
//
// Stage s of a CTA starts when the done-counter of stage s-1 (global memory, one per
// stage of the call, zeroed before the launch) reaches the number of work items that
// stage releases; every counter only grows, so the order of arrivals never matters.
// A stage's results are released with a gpu-scope fence before the counter
// increment and acquired with ld.acquire by the consumers (plus a proxy fence before
// TMA reads them).
//
// Roles (256 threads):
//   warp 0   weight TMA producer: streams this CTA's weight tiles of every stage, in
//            program order, into a 15-slot ring.  Weights are inputs, so it runs ahead
//            of the activations across stage boundaries, bounded only by the ring.
//   warp 1   tcgen05.mma issuer (GEMM units, and S = Q K^T / O += P V of attention).
//   warp 2   activation TMA loader of GEMM units; K loader of attention units.
//   warp 3   V loader of attention units.
//   warps 4-7 epilogues (TMEM lane quarter = warp % 4), the softmax of attention
//            units, and the small stages (ACTION_IN, COMBINE, EULER).
//
// GEMM units: the N columns of a Linear are cut into contiguous chunks of whole
// 16-column groups (<= 64 columns) and the K range into `splits` parts; the
// accumulator (M = 128 rows x chunk) lives in TMEM columns 448..511.  With split-K
// every unit stores its fp32 partial tile and the last unit of a chunk to arrive
// (counter) adds the partials in split order -- the result does not depend on timing
// -- and runs the epilogue.  Epilogues are those of the multi-kernel path: SiLU +
// time vector, bias, residual add with the fused RMSNorm producer (bf16 h*(1+g) and
// per-16-column sums of squares), RoPE at position n_b + j with q/k/v stores, GeGLU.
//
// Shared memory: a weight ring (15 x 8 KB) and region X (96 KB) that holds either the
// activation ring of a GEMM unit (4 x 16 KB) or the K/V rings (2 x 16 KB each) and P
// buffers (2 x 16 KB) of an attention unit.  Region X passes from one unit to the next
// through a counter of units whose MMAs have completed.
//
// Every wait is bounded (LoopArgs::wait_ns) and gives up early once the error word is
// set; on the way out each role waits for the copies it issued, the MMA warp for its
// MMAs, and TMEM is freed.
#include <math.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

namespace {

constexpr int kThreads = 256;
constexpr int kWSlots = 15;
constexpr uint32_t kWSlotBytes = 8192;
constexpr int kASlots = 4;
constexpr uint32_t kASlotBytes = 16384;
constexpr int kKB = kLoopKeyBlock;            // 32 keys per attention block
constexpr uint32_t kKVTile = kKB * 512;       // 32 keys x 256 dims bf16 = 16 KB
constexpr uint32_t kKVSub = kKB * 128;        // one 64-dim sub-tile = 4 KB
constexpr uint32_t kAtomBytes = 8 * 128;      // 8 keys x 64 dims: one 8-row box
constexpr uint32_t kPTile = 128 * 128;        // 128 rows x 128 B (32 keys used)

constexpr uint32_t kOffW = 0;
constexpr uint32_t kOffX = kOffW + kWSlots * kWSlotBytes;
constexpr uint32_t kOffA = kOffX;
constexpr uint32_t kOffK = kOffX;
constexpr uint32_t kOffV = kOffK + 2 * kKVTile;
constexpr uint32_t kOffP = kOffV + 2 * kKVTile;
constexpr uint32_t kXBytes = 6 * kKVTile;  // 96 KB
static_assert(kASlots * kASlotBytes <= kXBytes, "activation ring fits region X");
static_assert(kOffP + 2 * kPTile == kOffX + kXBytes, "attention buffers fill region X");
constexpr uint32_t kOffBar = kOffX + kXBytes;

struct Bars {
  uint64_t w_full[kWSlots], w_empty[kWSlots];
  uint64_t a_full[kASlots], a_empty[kASlots];
  uint64_t acc_full, acc_empty;
  uint64_t k_full[2], k_empty[2], v_full[2], pv_done[2];
  uint64_t s_full[2], s_empty[2], p_full[2];
  uint64_t q_full, mma_fin;
  uint32_t tmem_slot;
  uint32_t x_done;    // units that used region X and whose MMAs have completed (monotonic)
  int last;           // split-K: this CTA reduces the chunk
  float red[8];       // EULER row reduction
  uint32_t w_fills[kWSlots];  // drain bookkeeping
  uint32_t a_fills[kASlots];
  uint32_t k_fills[2], v_fills[2];
};
constexpr uint32_t kSmemTotal = kOffBar + ((sizeof(Bars) + 127) / 128) * 128 + 1024 + 4 * 1024 /* EULER row */;
static_assert(kSmemTotal <= 232448, "shared memory per CTA");

// TMEM columns: S buffers 0 and 32, Q 64..191 (bf16 pairs), O 192..447, GEMM 448..511
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemQ = 64;
constexpr uint32_t kTmemO = 192;
constexpr uint32_t kTmemAcc = 448;
constexpr uint32_t kTmemCols = 512;

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;

__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool err_set(const LoopArgs &a) { return *(volatile unsigned *)a.err != 0; }

// mbarrier wait: bounded by a.wait_ns, gives up early once the error word is set.
__device__ __forceinline__ bool lwait(uint64_t *bar, uint32_t parity, const LoopArgs &a, unsigned bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (err_set(a)) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicOr(a.err, bit);
      return false;
    }
  }
}
// Wait until *p >= target (acquire), with the same limits.
__device__ __forceinline__ bool lpoll(const int *p, int target, const LoopArgs &a) {
  if (ld_acquire(p) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 16; ++i)
      if (ld_acquire(p) >= target) return true;
    if (err_set(a)) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicOr(a.err, kErrTimeoutFlag);
      return false;
    }
  }
}

// Drain wait at exit: bounded by time only (it must wait for copies in flight even
// after the error word was set).
__device__ __forceinline__ void dwait(uint64_t *bar, uint32_t parity, const LoopArgs &a) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > a.wait_ns) return;
}
// Region X hand-off: the epilogue counts units whose MMAs completed; a loader waits
// until every earlier unit that used region X is counted (a monotonic counter, so a
// loader that looks late never misreads a phase).
__device__ __forceinline__ void x_release(Bars &bs) {
  __threadfence_block();
  atomicAdd(&bs.x_done, 1u);
}
__device__ __forceinline__ bool x_acquire(Bars &bs, uint32_t need, const LoopArgs &a, unsigned bit) {
  const volatile uint32_t *c = &bs.x_done;
  if (*c >= need) {
    __threadfence_block();
    return true;
  }
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (*c >= need) {
        __threadfence_block();
        return true;
      }
    if (err_set(a)) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicOr(a.err, bit);
      return false;
    }
  }
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  tc_wait_ld();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint4 pack8(const float *v) {
  uint32_t p[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    p[e] = *reinterpret_cast<const uint32_t *>(&h2);
  }
  return make_uint4(p[0], p[1], p[2], p[3]);
}

// ---- program geometry ------------------------------------------------------------
struct StageInfo {
  int kind, layer, step, gs;  // gs: index of the stage in the call
};
__device__ __forceinline__ int stage_count(const LoopArgs &a) { return loop_stages_per_step(a.L, a.attn_splits); }
__device__ __forceinline__ StageInfo stage_at(const LoopArgs &a, int gs) {
  StageInfo si;
  const int spp = stage_count(a);
  si.gs = gs;
  si.step = gs / spp;
  loop_stage(gs % spp, a.L, a.attn_splits, si.kind, si.layer);
  return si;
}
__device__ __forceinline__ int q_tiles(const LoopArgs &a, int step0) {
  const int Tq = step0 ? a.H + 1 : a.H;
  return (kHeads * Tq + 127) / 128;
}
__device__ __forceinline__ int attn_units(const LoopArgs &a, int step0) { return a.B * q_tiles(a, step0) * a.attn_splits; }
__device__ __forceinline__ int combine_items(const LoopArgs &a, int step0) {
  return a.B * kHeads * (step0 ? a.H + 1 : a.H);
}
__device__ __forceinline__ int combine_ctas(const LoopArgs &a, int step0) {
  const int c = (combine_items(a, step0) + 3) / 4;
  return c < a.grid ? c : a.grid;
}
__device__ __forceinline__ int action_ctas(const LoopArgs &a) { return a.grid < 128 ? a.grid : 128; }
__device__ __forceinline__ int euler_units(const LoopArgs &a) { return a.B * a.H * ((a.A + 15) / 16); }
__device__ __forceinline__ int euler_ctas(const LoopArgs &a) {
  const int u = euler_units(a);
  return u < a.grid ? u : a.grid;
}
// Arrivals that complete stage `si`.
__device__ __forceinline__ int stage_expect(const LoopArgs &a, const StageInfo &si) {
  const int step0 = si.step == 0;
  switch (si.kind) {
    case LK_ACTION_IN: return action_ctas(a);
    case LK_ATTN: return attn_units(a, step0);
    case LK_COMBINE: return combine_ctas(a, step0);
    case LK_EULER: return euler_ctas(a);
    default: return loop_gemm_plan(si.kind, a.grid).nchunks;
  }
}
// Wait (one thread) until the stage before `gs` has completed.
__device__ __forceinline__ bool wait_prev(const LoopArgs &a, int gs) {
  if (gs == 0) return true;
  const StageInfo p = stage_at(a, gs - 1);
  return lpoll(a.done + (gs - 1), stage_expect(a, p), a);
}
// Release of a stage's work item (one thread, after the item's stores are ordered
// before it by epi_bar()).
__device__ __forceinline__ void release(const LoopArgs &a, int gs) {
  __threadfence();
  atomicAdd(a.done + gs, 1);
}

struct GUnit {
  int n0, w, kb0, kb1, chunk, split;
};
__device__ __forceinline__ GUnit gemm_unit(const LoopGemm &p, int u) {
  GUnit g;
  g.chunk = u / p.splits;
  g.split = u % p.splits;
  const int G = p.N / 16;
  const int g0 = (int)((long)g.chunk * G / p.nchunks), g1 = (int)((long)(g.chunk + 1) * G / p.nchunks);
  g.n0 = g0 * 16;
  g.w = (g1 - g0) * 16;
  const int nk = p.K / 64, kps = (nk + p.splits - 1) / p.splits;
  g.kb0 = g.split * kps;
  g.kb1 = min(nk, g.kb0 + kps);
  return g;
}
__device__ __forceinline__ const CUtensorMap *weight_map(const LoopArgs &a, int kind, int layer) {
  switch (kind) {
    case LK_TIN: return a.m_tin;
    case LK_TOUT: return a.m_tout;
    case LK_QKV: return a.m_qkv[layer];
    case LK_O: return a.m_o[layer];
    case LK_GU: return a.m_gu[layer];
    default: return a.m_down[layer];
  }
}
__device__ __forceinline__ const CUtensorMap *act_map(const LoopArgs &a, int kind) {
  switch (kind) {
    case LK_TIN: return a.m_aemb;
    case LK_TOUT: return a.m_uemb;
    case LK_QKV: case LK_GU: return a.m_xn;
    case LK_O: return a.m_att;
    default: return a.m_act;
  }
}
// Activation rows of a GEMM stage: A rows [a_row0, a_row0 + M), output rows out_row0 + r.
__device__ __forceinline__ void gemm_rows(const LoopArgs &a, int kind, int step0, int &a_row0, int &M, int &out_row0) {
  const int BH = a.B * a.H;
  if (kind == LK_TIN || kind == LK_TOUT) {
    a_row0 = 0;
    M = BH;
    out_row0 = kind == LK_TOUT ? a.B : 0;
    return;
  }
  a_row0 = step0 ? 0 : a.B;
  M = a.R - a_row0;
  out_row0 = a_row0;
}

// ---- attention key slots (32-key blocks) -------------------------------------------
// Source of key slot kk of sample b: 2*row of the prefix tensor (B*P rows), 2*row+1 of
// this layer's suffix K/V, -1 for an empty slot.  Valid prefix keys come first, then
// the H action keys and the state key.
__device__ __forceinline__ int slot_code(int kk, int nbp, int nv, bool contig, int b, const LoopArgs &a,
                                         const int *vi) {
  const int pre = nbp * kKB;
  if (kk < pre) return kk < nv ? 2 * (b * a.P + (contig ? kk : vi[kk])) : -1;
  const int s = kk - pre;
  if (s < a.H) return 2 * (a.B + b * a.H + s) + 1;
  if (s == a.H) return 2 * b + 1;
  return -1;
}

// One warp fills the [32 keys x 256] tile at `tile` (4 sub-tiles of 64 dims).  32
// consecutive rows of one tensor: one 32-row box per sub-tile.  Else each 8-slot atom
// of consecutive rows (or all empty: a box at row -8, entirely out of bounds, fills
// zeros) is one 8-row box per sub-tile, and other atoms are copied row by row with
// cp.async (zeros for empty slots).  `full` completes on the TMA bytes plus one
// cp.async arrival per lane.
__device__ __forceinline__ void load_kv_tile(int blk, uint32_t tile, uint64_t *full, const CUtensorMap *pmap,
                                             const CUtensorMap *smap, const CUtensorMap *pmap32,
                                             const CUtensorMap *smap32, int sfx_row0, const bf16 *pref,
                                             const bf16 *suf, int nbp, int nv, bool contig, int b,
                                             const LoopArgs &a, const int *vi, int lane) {
  const int kb = blk * kKB;
  const int code = slot_code(kb + lane, nbp, nv, contig, b, a, vi);
  const int c0 = __shfl_sync(kFull, code, 0);
  if (__all_sync(kFull, c0 >= 0 && code == c0 + 2 * lane)) {
    if (lane == 0) {
      mbar_expect_tx(full, kKVTile);
      const CUtensorMap *m = (c0 & 1) ? smap32 : pmap32;
      const int y = (c0 & 1) ? sfx_row0 + (c0 >> 1) : (c0 >> 1);
#pragma unroll
      for (int sub = 0; sub < 4; ++sub) tma_load_2d(tile + sub * kKVSub, m, sub * 64, y, full);
    }
    __syncwarp();
    cp_async_mbar_arrive(full);
    return;
  }
  const int lead = __shfl_sync(kFull, code, lane & ~7);
  const bool run = lead >= 0 && code == lead + 2 * (lane & 7);
  const unsigned br = __ballot_sync(kFull, run), be = __ballot_sync(kFull, code < 0);
  unsigned tma_atoms = 0, copy_atoms = 0;
#pragma unroll
  for (int at = 0; at < 4; ++at) {
    const bool whole = ((br >> (8 * at)) & 0xffu) == 0xffu || ((be >> (8 * at)) & 0xffu) == 0xffu;
    (whole ? tma_atoms : copy_atoms) |= 1u << at;
  }
  if (lane == 0 && tma_atoms) mbar_expect_tx(full, (uint32_t)__popc(tma_atoms) * 4u * kAtomBytes);
  __syncwarp();
  if ((lane & 7) == 0 && ((tma_atoms >> (lane >> 3)) & 1u)) {
    const int at = lane >> 3;
    const CUtensorMap *m = (code >= 0 && !(code & 1)) ? pmap : smap;
    const int y = code < 0 ? -8 : (code & 1) ? sfx_row0 + (code >> 1) : (code >> 1);
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) tma_load_2d(tile + sub * kKVSub + at * kAtomBytes, m, sub * 64, y, full);
  }
  while (copy_atoms) {  // warp-uniform
    const int at = __ffs(copy_atoms) - 1;
    copy_atoms &= copy_atoms - 1;
#pragma unroll 4
    for (int r = 0; r < 8; ++r) {
      const int c = __shfl_sync(kFull, code, 8 * at + r);
      const bf16 *row = c < 0 ? suf : ((c & 1) ? suf : pref) + (size_t)(c >> 1) * kHeadDim;
      cp_async16(tile + (lane >> 3) * kKVSub + sw128_off(8 * at + r, lane & 7), row + lane * 8, c >= 0);
    }
  }
  cp_async_mbar_arrive(full);
}

// Attention unit geometry.
struct AUnit {
  int b, ti, split, nv, nbp, blk0, nb;
};
__device__ __forceinline__ AUnit attn_unit(const LoopArgs &a, int u, int step0) {
  AUnit t;
  const int qps = q_tiles(a, step0);
  const int qt = u / a.attn_splits;
  t.split = u % a.attn_splits;
  t.b = qt / qps;
  t.ti = qt % qps;
  t.nv = a.nvalid[t.b];
  t.nbp = (t.nv + kKB - 1) / kKB;
  const int nblk = t.nbp + (a.H + kKB) / kKB;
  t.blk0 = t.split * a.attn_bps;
  const int blk1 = min(nblk, t.blk0 + a.attn_bps);
  t.nb = blk1 > t.blk0 ? blk1 - t.blk0 : 0;
  return t;
}

// ---- role: weight producer (warp 0, one lane) ---------------------------------------
__device__ void role_weights(const LoopArgs &a, uint8_t *smem, Bars &bs) {
  const int total = a.N * stage_count(a);
  uint32_t wi = 0;
  bool ok = true;
  // the weight maps live in device memory: acquire them once
  tma_map_acquire(a.m_tin);
  tma_map_acquire(a.m_tout);
  for (int l = 0; l < a.L; ++l) {
    tma_map_acquire(a.m_qkv[l]);
    tma_map_acquire(a.m_o[l]);
    tma_map_acquire(a.m_gu[l]);
    tma_map_acquire(a.m_down[l]);
  }
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    if (!loop_is_gemm(si.kind)) continue;
    const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
    const CUtensorMap *map = weight_map(a, si.kind, si.layer);
    const int U = p.nchunks * p.splits;
    for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
      const GUnit g = gemm_unit(p, u);
      for (int kb = g.kb0; kb < g.kb1; ++kb, ++wi) {
        const int slot = wi % kWSlots;
        const uint32_t n = wi / kWSlots;
        if (n > 0 && !lwait(&bs.w_empty[slot], (n - 1) & 1u, a, kErrTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bs.w_full[slot], (uint32_t)g.w * 128u);
        for (int r = 0; r < g.w; r += 16)
          tma_load_2d(smem + kOffW + slot * kWSlotBytes + r * 128, map, kb * 64, g.n0 + r, &bs.w_full[slot]);
        bs.w_fills[slot] = n + 1;
      }
    }
  }
}

// ---- role: MMA issuer (warp 1, whole warp; one elected lane issues) ------------------
__device__ void role_mma(const LoopArgs &a, uint8_t *smem, Bars &bs, uint32_t tmem) {
  const int total = a.N * stage_count(a);
  const uint32_t sbase = smem_u32(smem);
  uint32_t wi = 0, ai = 0, acc_n = 0, kj = 0, vj = 0, sj = 0, pj = 0, qn = 0;
  bool ok = true;
  const uint64_t kdesc0 = smem_desc_k_sw128(sbase + kOffK, 0);
  const uint64_t pdesc0 = smem_desc_k_sw128(sbase + kOffP, 0);
  const uint64_t vdesc0 = smem_desc_mn_sw128(sbase + kOffV, kKVSub, 1024);
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKB);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim) | (1u << 16);  // B (V) MN-major
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    if (loop_is_gemm(si.kind)) {
      const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
      const int U = p.nchunks * p.splits;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const GUnit g = gemm_unit(p, u);
        if (acc_n > 0 && !__all_sync(kFull, lwait(&bs.acc_empty, (acc_n - 1) & 1u, a, kErrTimeoutMma))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, g.w);
        for (int kb = g.kb0; kb < g.kb1; ++kb, ++wi, ++ai) {
          const int ws = wi % kWSlots, as = ai % kASlots;
          if (!__all_sync(kFull, lwait(&bs.w_full[ws], (wi / kWSlots) & 1u, a, kErrTimeoutMma)) ||
              !__all_sync(kFull, lwait(&bs.a_full[as], (ai / kASlots) & 1u, a, kErrTimeoutMma))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ab = sbase + kOffA + as * kASlotBytes, wb = sbase + kOffW + ws * kWSlotBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16_w(tmem + kTmemAcc, smem_desc_k_sw128(ab, kk * 32), smem_desc_k_sw128(wb, kk * 32), idesc,
                          (kb > g.kb0 || kk > 0) ? 1u : 0u);
          tc_commit_w(&bs.w_empty[ws]);
          tc_commit_w(&bs.a_empty[as]);
        }
        if (!ok) break;
        tc_commit_w(&bs.acc_full);
        ++acc_n;
      }
    } else if (si.kind == LK_ATTN) {
      const int step0 = si.step == 0;
      const int U = attn_units(a, step0);
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const AUnit t = attn_unit(a, u, step0);
        if (t.nb == 0) continue;
        if (!__all_sync(kFull, lwait(&bs.q_full, qn & 1u, a, kErrTimeoutMma))) {
          ok = false;
          break;
        }
        ++qn;
        tc_fence_after();
        auto issue_s = [&]() -> bool {  // S[sj & 1] = Q K(kj)^T
          const int kbuf = kj % 2, sb = sj & 1;
          if (!__all_sync(kFull, lwait(&bs.k_full[kbuf], (kj / 2) & 1u, a, kErrTimeoutMma))) return false;
          if (sj >= 2 && !__all_sync(kFull, lwait(&bs.s_empty[sb], ((sj >> 1) - 1) & 1u, a, kErrTimeoutMma)))
            return false;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t kd = kdesc0 + (uint64_t)((kbuf * kKVTile) >> 4);
#pragma unroll
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16_ts_w(tmem + kTmemS + (uint32_t)(sb * kKB), tmem + kTmemQ + (uint32_t)(32 * s + 8 * kk),
                               kd + (uint64_t)((s * kKVSub + kk * 32) >> 4), idesc_s, (s | kk) != 0);
          tc_commit_w(&bs.s_full[sb]);
          tc_commit_w(&bs.k_empty[kbuf]);
          ++kj;
          ++sj;
          return true;
        };
        auto issue_pv = [&](int j) -> bool {  // O += P(pj) V(vj)
          const int vbuf = vj % 2, pb = pj % 2;
          if (!__all_sync(kFull, lwait(&bs.p_full[pb], (pj / 2) & 1u, a, kErrTimeoutMma))) return false;
          if (!__all_sync(kFull, lwait(&bs.v_full[vbuf], (vj / 2) & 1u, a, kErrTimeoutMma))) return false;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t pd = pdesc0 + (uint64_t)((pb * kPTile) >> 4);
          const uint64_t vd = vdesc0 + (uint64_t)((vbuf * kKVTile) >> 4);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)
            tc_mma_bf16_w(tmem + kTmemO, pd + (uint64_t)((kk * 32) >> 4), vd + (uint64_t)((kk * 2048) >> 4), idesc_o,
                          (j | kk) != 0);
          tc_commit_w(&bs.pv_done[vbuf]);
          ++vj;
          ++pj;
          return true;
        };
        ok = issue_s();
        for (int j = 0; j < t.nb && ok; ++j) {
          if (j + 1 < t.nb) ok = issue_s();
          if (ok) ok = issue_pv(j);
        }
      }
    }
  }
  // every MMA issued has completed before the CTA may free TMEM or exit
  tc_commit_w(&bs.mma_fin);
  dwait(&bs.mma_fin, 0, a);
  __syncwarp();
}

// ---- role: activation loader of GEMM units, K loader of attention units (warp 2) ------
// and V loader of attention units (warp 3, is_v).
__device__ void role_loader(const LoopArgs &a, uint8_t *smem, Bars &bs, bool is_v, int lane) {
  const int total = a.N * stage_count(a);
  const uint32_t sbase = smem_u32(smem);
  uint32_t ai = 0, kj = 0, x_units = 0;
  bool ok = true;
  if (lane == 0 && !is_v) {
    tma_map_acquire(a.m_xn);
    tma_map_acquire(a.m_att);
    tma_map_acquire(a.m_act);
    tma_map_acquire(a.m_aemb);
    tma_map_acquire(a.m_uemb);
  }
  // region X: wait until every earlier unit that used it has finished its MMAs
  auto take_x = [&]() -> bool {
    bool good = true;
    if (lane == 0) good = x_acquire(bs, x_units, a, kErrTimeoutProducer);
    ++x_units;
    good = __shfl_sync(kFull, (int)good, 0) != 0;
    __syncwarp();
    return good;
  };
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    const int step0 = si.step == 0;
    if (loop_is_gemm(si.kind)) {
      const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
      const int U = p.nchunks * p.splits;
      if (blockIdx.x >= U) continue;
      int a_row0, M, out_row0;
      gemm_rows(a, si.kind, step0, a_row0, M, out_row0);
      (void)M;
      (void)out_row0;
      const CUtensorMap *amap = act_map(a, si.kind);
      bool waited = false;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        ok = take_x();
        if (!ok) break;
        if (is_v) continue;
        if (lane == 0) {
          if (!waited) {
            ok = wait_prev(a, gs) && !(si.gs == a.debug_stall_stage && !lpoll(a.done + gs, 1 << 30, a));
            fence_proxy_async_global();
            waited = true;
          }
          const GUnit g = gemm_unit(p, u);
          for (int kb = g.kb0; kb < g.kb1 && ok; ++kb, ++ai) {
            const int slot = ai % kASlots;
            const uint32_t n = ai / kASlots;
            if (n > 0 && !lwait(&bs.a_empty[slot], (n - 1) & 1u, a, kErrTimeoutProducer)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bs.a_full[slot], (uint32_t)a.box_rows * 128u);
            tma_load_2d(smem + kOffA + slot * kASlotBytes, amap, kb * 64, a_row0, &bs.a_full[slot]);
            bs.a_fills[slot] = n + 1;
          }
        }
        ok = __all_sync(kFull, __shfl_sync(kFull, (int)ok, 0) != 0);
      }
    } else if (si.kind == LK_ATTN) {
      const int U = attn_units(a, step0);
      const int layer = si.layer;
      const CUtensorMap *pmap = &a.cp->kv_map[is_v][layer], *smap = &a.cp->sfx_map[is_v];
      const CUtensorMap *pmap32 = &a.cp->kv_map32[is_v][layer], *smap32 = &a.cp->sfx_map32[is_v];
      const bf16 *pref = is_v ? a.cp->prefix_v[layer] : a.cp->prefix_k[layer];
      const bf16 *suf = (is_v ? a.vs : a.ks) + (size_t)layer * a.R * kHeadDim;
      const int sfx_row0 = layer * a.R;
      uint64_t *full = is_v ? bs.v_full : bs.k_full;
      uint64_t *empty = is_v ? bs.pv_done : bs.k_empty;
      uint32_t *fills = is_v ? bs.v_fills : bs.k_fills;
      const uint32_t ring = sbase + (is_v ? kOffV : kOffK);
      bool maps_ready = false, sfx_ready = false;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        ok = take_x();
        if (!ok) break;
        const AUnit t = attn_unit(a, u, step0);
        if (t.nb == 0) continue;
        if (!maps_ready) {
          if (lane == 0) {
            if (a.P > 0) {
              tma_map_acquire(pmap);
              tma_map_acquire(pmap32);
            }
            tma_map_acquire(smap);
            tma_map_acquire(smap32);
          }
          maps_ready = true;
        }
        const int *vi = a.vidx + (size_t)t.b * a.P;
        const bool contig = t.nv == 0 || vi[t.nv - 1] == t.nv - 1;
        for (int j = 0; j < t.nb && ok; ++j, ++kj) {
          const int blk = t.blk0 + j;
          if (!sfx_ready && blk >= t.nbp) {  // suffix keys come from this step's QKV stage
            if (lane == 0) {
              ok = wait_prev(a, gs);
              fence_proxy_async_global();
            }
            ok = __all_sync(kFull, __shfl_sync(kFull, (int)ok, 0) != 0);
            if (!ok) break;
            sfx_ready = true;
          }
          const int buf = kj % 2;
          const uint32_t n = kj / 2;
          if (n > 0) ok = __all_sync(kFull, lwait(&empty[buf], (n - 1) & 1u, a, kErrTimeoutProducer));
          if (!ok) break;
          load_kv_tile(blk, ring + buf * kKVTile, &full[buf], pmap, smap, pmap32, smap32, sfx_row0, pref, suf, t.nbp,
                       t.nv, contig, t.b, a, vi, lane);
          if (lane == 0) fills[buf] = n + 1;
        }
      }
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
}

// ---- GEMM epilogues (one output row per thread, 16 columns) ------------------------------
__device__ __forceinline__ float row_rstd64(const float *ss, int ld, int orow) {
  float t = 0.f;
#pragma unroll 8
  for (int g = 0; g < kLoopNormSlots; ++g) t += ss[(size_t)g * ld + orow];
  return 1.0f / sqrtf(t / (float)kWidth + kRmsEps);
}

struct EpiCtx {
  int kind, layer, step, orow, b, j;
  float rs;
  int pos;
};

// Residual / bias producers with the fused RMSNorm outputs.
__device__ __forceinline__ void epi_store16(const LoopArgs &a, const EpiCtx &c, int n, float (&v)[16]) {
  const int orow = c.orow;
  if (c.kind == LK_TIN) {
    const float *vec = a.tvec + (size_t)c.step * kWidth + n;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = silu_f(v[i] + vec[i]);
    uint4 *dst = reinterpret_cast<uint4 *>(a.uemb + (size_t)orow * kWidth + n);
    dst[0] = pack8(t);
    dst[1] = pack8(t + 8);
  } else if (c.kind == LK_TOUT || c.kind == LK_O || c.kind == LK_DOWN) {
    float *hp = a.h + (size_t)orow * kWidth + n;
    float4 *h4 = reinterpret_cast<float4 *>(hp);
    if (c.kind == LK_TOUT) {
      const float4 *b4 = reinterpret_cast<const float4 *>(a.tout_b + n);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 bb = b4[i];
        v[4 * i] += bb.x; v[4 * i + 1] += bb.y; v[4 * i + 2] += bb.z; v[4 * i + 3] += bb.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 hh = h4[i];
        v[4 * i] += hh.x; v[4 * i + 1] += hh.y; v[4 * i + 2] += hh.z; v[4 * i + 3] += hh.w;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) h4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    const float *gain = c.kind == LK_TOUT ? a.in_norm[0]
                        : c.kind == LK_O  ? a.post_norm[c.layer]
                        : (c.layer + 1 < a.L ? a.in_norm[c.layer + 1] : nullptr);
    if (gain) {  // fused RMSNorm producer: bf16(h * (1 + g)) and the group's sum of h^2
      float *ss = c.kind == LK_O ? a.ss_m : a.ss_a;
      float t[16], ssq = 0.f;
      const float4 *g4 = reinterpret_cast<const float4 *>(gain + n);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 gg = g4[i];
        ssq = fmaf(v[4 * i], v[4 * i], ssq);
        ssq = fmaf(v[4 * i + 1], v[4 * i + 1], ssq);
        ssq = fmaf(v[4 * i + 2], v[4 * i + 2], ssq);
        ssq = fmaf(v[4 * i + 3], v[4 * i + 3], ssq);
        t[4 * i] = v[4 * i] * (1.0f + gg.x);
        t[4 * i + 1] = v[4 * i + 1] * (1.0f + gg.y);
        t[4 * i + 2] = v[4 * i + 2] * (1.0f + gg.z);
        t[4 * i + 3] = v[4 * i + 3] * (1.0f + gg.w);
      }
      uint4 *xd = reinterpret_cast<uint4 *>(a.xn + (size_t)orow * kWidth + n);
      xd[0] = pack8(t);
      xd[1] = pack8(t + 8);
      ss[(size_t)(n >> 4) * a.ss_ld + orow] = ssq;
    }
  } else if (c.kind == LK_QKV) {
    // group gc = 8 rotation pairs (ib .. ib+7, +128) of head hd (8 = k, 9 = v)
    const int gc = n >> 4, hd = gc >> 4, ib = (gc & 15) * 8;
    float lo[8], hi[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      lo[w] = v[w] * c.rs;
      hi[w] = v[8 + w] * c.rs;
    }
    if (hd < kHeads + 1) {
      const float4 *tab = reinterpret_cast<const float4 *>(a.rope_tab + ((size_t)c.pos * (kHeadDim / 2) + ib) * 2);
#pragma unroll
      for (int w2 = 0; w2 < 4; ++w2) {
        const float4 t = tab[w2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int w = 2 * w2 + h2;
          const float cs = h2 ? t.z : t.x, sn = h2 ? t.w : t.y;
          const float x0 = lo[w], x1 = hi[w];
          lo[w] = x0 * cs - x1 * sn;
          hi[w] = x1 * cs + x0 * sn;
        }
      }
    }
    bf16 *dst;
    if (hd < kHeads)
      dst = a.q + (size_t)orow * kQDim + hd * kHeadDim + ib;
    else
      dst = (hd == kHeads ? a.ks : a.vs) + ((size_t)c.layer * a.R + orow) * kHeadDim + ib;
    *reinterpret_cast<uint4 *>(dst) = pack8(lo);
    *reinterpret_cast<uint4 *>(dst + kHeadDim / 2) = pack8(hi);
  } else {  // LK_GU: 8 gate then the matching 8 up features
    float t[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) t[w] = gelu_tanh_f(v[w] * c.rs) * (v[8 + w] * c.rs);
    *reinterpret_cast<uint4 *>(a.act + (size_t)orow * kMlp + (n >> 4) * 8) = pack8(t);
  }
}

// ---- role: epilogues, softmax and small stages (warps 4-7) -----------------------------
__device__ void role_epi(const LoopArgs &a, uint8_t *smem, Bars &bs, uint32_t tmem, int et) {
  const int total = a.N * stage_count(a);
  const int warp = et >> 5, lane = et & 31;
  const uint32_t t_lane = (uint32_t)(warp * 32) << 16;
  uint32_t acc_n = 0, sj = 0, pj = 0, pvj = 0;
  bool ok = true;
  float *yrow = reinterpret_cast<float *>(smem + kOffBar + ((sizeof(Bars) + 127) / 128) * 128);
  auto poll_prev = [&](int gs) -> bool {
    bool good = true;
    if (lane == 0) good = wait_prev(a, gs) && !(gs == a.debug_stall_stage && !lpoll(a.done + gs, 1 << 30, a));
    good = __shfl_sync(kFull, (int)good, 0) != 0;
    __syncwarp();
    return good;
  };
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    const int step0 = si.step == 0;
    if (loop_is_gemm(si.kind)) {
      const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
      const int U = p.nchunks * p.splits;
      if (blockIdx.x >= U) continue;
      ok = poll_prev(gs);
      if (!ok) break;
      int a_row0, M, out_row0;
      gemm_rows(a, si.kind, step0, a_row0, M, out_row0);
      const int r = et;
      const bool valid = r < M;
      EpiCtx c;
      c.kind = si.kind;
      c.layer = si.layer;
      c.step = si.step;
      c.orow = out_row0 + r;
      c.rs = 1.f;
      c.pos = 0;
      if (valid && (si.kind == LK_QKV || si.kind == LK_GU))
        c.rs = row_rstd64(si.kind == LK_QKV ? a.ss_a : a.ss_m, a.ss_ld, c.orow);
      if (valid && si.kind == LK_QKV) {
        int b, j;
        if (c.orow < a.B) {
          b = c.orow;
          j = 0;
        } else {
          b = (c.orow - a.B) / a.H;
          j = 1 + (c.orow - a.B) % a.H;
        }
        c.pos = a.nvalid[b] + j;
      }
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const GUnit g = gemm_unit(p, u);
        ok = __all_sync(kFull, lwait(&bs.acc_full, acc_n & 1u, a, kErrTimeoutEpilogue));
        if (!ok) break;
        ++acc_n;
        tc_fence_after();
        if (et == 0) x_release(bs);  // the unit's MMAs have completed
        if (p.splits == 1) {
          for (int gi = 0; gi < g.w; gi += 16) {
            float v[16];
            tmem_ld_x16(tmem + t_lane + kTmemAcc + (uint32_t)gi, v);
            if (valid) epi_store16(a, c, g.n0 + gi, v);
          }
          tc_fence_before();
          fence_proxy_async_global();
          epi_bar();
          if (et == 0) {
            mbar_arrive(&bs.acc_empty);
            release(a, gs);
          }
        } else {
          float *mine = a.gpart + ((size_t)(g.chunk * p.splits + g.split) * 128 + r) * 64;
          for (int gi = 0; gi < g.w; gi += 16) {
            float v[16];
            tmem_ld_x16(tmem + t_lane + kTmemAcc + (uint32_t)gi, v);
            if (valid) {
              float4 *d4 = reinterpret_cast<float4 *>(mine + gi);
#pragma unroll
              for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
          }
          tc_fence_before();
          __threadfence();
          epi_bar();
          if (et == 0) {
            mbar_arrive(&bs.acc_empty);
            const int prev = atomicAdd(a.counters + g.chunk, 1);
            bs.last = prev == p.splits - 1;
          }
          epi_bar();
          if (bs.last) {
            __threadfence();
            if (valid) {
              const float *base = a.gpart + ((size_t)g.chunk * p.splits * 128 + r) * 64;
              for (int gi = 0; gi < g.w; gi += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.f;
                for (int s = 0; s < p.splits; ++s) {
                  const float4 *p4 = reinterpret_cast<const float4 *>(base + (size_t)s * 128 * 64 + gi);
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    const float4 t = __ldcg(p4 + i);
                    v[4 * i] += t.x; v[4 * i + 1] += t.y; v[4 * i + 2] += t.z; v[4 * i + 3] += t.w;
                  }
                }
                epi_store16(a, c, g.n0 + gi, v);
              }
            }
            fence_proxy_async_global();
            epi_bar();
            if (et == 0) {
              a.counters[g.chunk] = 0;  // ready for the next split-K stage
              release(a, gs);
            }
          }
        }
      }
    } else if (si.kind == LK_ATTN) {
      const int U = attn_units(a, step0);
      if (blockIdx.x >= U) continue;
      ok = poll_prev(gs);  // q of this step's QKV stage
      if (!ok) break;
      const int Tq = step0 ? a.H + 1 : a.H;
      const int nrows = kHeads * Tq;
      const float scale_l2 = 0.0625f * kLog2e;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const AUnit t = attn_unit(a, u, step0);
        const int qi = t.ti * 128 + et;
        const bool row_ok = qi < nrows;
        const int jq = qi / kHeads, head = qi % kHeads;
        int tok = 0;
        if (row_ok) tok = step0 ? (jq == 0 ? t.b : a.B + t.b * a.H + jq - 1) : a.B + t.b * a.H + jq;
        const bool state_q = step0 && jq == 0;
        const int ja = step0 ? jq - 1 : jq;
        const int sfx_base = t.nbp * kKB;
        const int sfx_lo = sfx_base + (state_q ? a.H : 0);
        const int sfx_hi = state_q ? sfx_base + a.H + 1 : (a.causal ? sfx_base + ja + 1 : sfx_base + a.H + 1);
        const int sfx_state = sfx_base + a.H;
        float m_used = -INFINITY, l = 0.f;
        if (t.nb > 0) {
          // Q row -> TMEM lane et, columns kTmemQ.. (two bf16 per 32-bit column)
          const uint4 *src = reinterpret_cast<const uint4 *>(a.q + (size_t)tok * kQDim + head * kHeadDim);
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint4 uu = row_ok ? src[cc * 8 + e] : make_uint4(0, 0, 0, 0);
              v[4 * e] = __uint_as_float(uu.x);
              v[4 * e + 1] = __uint_as_float(uu.y);
              v[4 * e + 2] = __uint_as_float(uu.z);
              v[4 * e + 3] = __uint_as_float(uu.w);
            }
            tmem_st_32x32b_x32(tmem + t_lane + kTmemQ + 32 * cc, v);
          }
          tc_fence_before();
          mbar_arrive(&bs.q_full);
          const uint32_t pv0 = pvj;  // global index of this unit's first P.V
          for (int j = 0; j < t.nb && ok; ++j, ++sj, ++pj) {
            const int sb = sj & 1, pb = pj & 1;
            ok = __all_sync(kFull, lwait(&bs.s_full[sb], (sj >> 1) & 1u, a, kErrTimeoutEpilogue));
            if (!ok) break;
            tc_fence_after();
            float sv[32];
            tmem_ld_32x32b_x32(tmem + t_lane + kTmemS + sb * kKB, sv);
            tc_fence_before();
            mbar_arrive(&bs.s_empty[sb]);
            const int kbase = (t.blk0 + j) * kKB;
            const bool pre_blk = t.blk0 + j < t.nbp;
            const int vis_lo = pre_blk ? 0 : sfx_lo, vis_hi = pre_blk ? t.nv : sfx_hi;
            const int vis_st = pre_blk ? -1 : sfx_state;
            if (kbase < vis_lo || kbase + kKB > vis_hi) {
#pragma unroll
              for (int i = 0; i < kKB; ++i)
                if ((unsigned)(kbase + i - vis_lo) >= (unsigned)(vis_hi - vis_lo) && kbase + i != vis_st)
                  sv[i] = -INFINITY;
            }
            float bm;
            {
              float mx[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) mx[k] = sv[k];
#pragma unroll
              for (int i = 8; i < kKB; ++i) mx[i & 7] = fmaxf(mx[i & 7], sv[i]);
              bm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
              bm *= scale_l2;
            }
            const bool mine = bm > m_used + kRescaleSlack;
            if (__any_sync(kFull, mine)) {
              const float alpha = mine ? ex2_approx(m_used - bm) : 1.0f;
              l *= alpha;
              if (j >= 1) {  // O holds P.V of this unit's blocks < j: wait for the last of them
                const uint32_t g = pj - 1;
                ok = __all_sync(kFull, lwait(&bs.pv_done[g % 2], (g / 2) & 1u, a, kErrTimeoutEpilogue));
                if (!ok) break;
                tc_fence_after();
                for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
                  float o[32];
                  tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c0, o);
#pragma unroll
                  for (int i = 0; i < 32; ++i) o[i] *= alpha;
                  tmem_st_32x32b_x32(tmem + t_lane + kTmemO + c0, o);
                }
                tc_fence_before();
              }
              if (mine) m_used = bm;
            }
            if (pj >= 2) {  // P buffer pb was last read by P.V number pj - 2 (this unit's or the last one's)
              const uint32_t g = pj - 2;
              ok = __all_sync(kFull, lwait(&bs.pv_done[g % 2], (g / 2) & 1u, a, kErrTimeoutEpilogue));
              if (!ok) break;
            }
            {
              const float mu = m_used == -INFINITY ? 0.f : m_used;
              uint8_t *prow = smem + kOffP + pb * kPTile;
              float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int cc = 0; cc < kKB / 8; ++cc) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i0 = cc * 8 + 2 * e;
                  const float p0 = ex2_approx(fmaf(sv[i0], scale_l2, -mu)), p1 = ex2_approx(fmaf(sv[i0 + 1], scale_l2, -mu));
                  ls[e] += p0 + p1;
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                  pk[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                *reinterpret_cast<uint4 *>(prow + sw128_off(et, cc)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
              l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bs.p_full[pb]);
          }
          if (ok) {
            const uint32_t g = pv0 + t.nb - 1;
            ok = __all_sync(kFull, lwait(&bs.pv_done[g % 2], (g / 2) & 1u, a, kErrTimeoutEpilogue));
          }
          pvj = pv0 + t.nb;
          tc_fence_after();
        }
        if (et == 0) x_release(bs);  // every MMA of the unit has completed
        if (!ok) break;
        const float inv_l = l > 0.f ? 1.0f / l : 0.f;
        if (a.attn_splits == 1) {
          bf16 *dst = a.att + (size_t)tok * kQDim + head * kHeadDim;
          for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
            float v[32];
            if (t.nb > 0) {
              tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c0, v);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = 0.f;
            }
            if (row_ok) {
              float w32[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) w32[e] = v[e] * inv_l;
              uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
              for (int e = 0; e < 4; ++e) d4[e] = pack8(w32 + 8 * e);
            }
          }
        } else {
          const size_t prow = (size_t)u * 128 + et;  // u = (b * qps + ti) * splits + split
          for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
            float v[32];
            if (t.nb > 0) {
              tmem_ld_32x32b_x32(tmem + t_lane + kTmemO + c0, v);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = 0.f;
            }
            if (row_ok) {
              float4 *d4 = reinterpret_cast<float4 *>(a.part_o + prow * kHeadDim + c0);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                d4[e] = make_float4(v[4 * e] * inv_l, v[4 * e + 1] * inv_l, v[4 * e + 2] * inv_l, v[4 * e + 3] * inv_l);
            }
          }
          if (row_ok) {
            a.part_ml[2 * prow] = m_used;
            a.part_ml[2 * prow + 1] = l;
          }
        }
        tc_fence_before();
        fence_proxy_async_global();
        epi_bar();
        if (et == 0) release(a, gs);
      }
    } else if (si.kind == LK_COMBINE) {
      const int nc = combine_ctas(a, step0);
      if (blockIdx.x >= nc) continue;
      ok = poll_prev(gs);
      if (!ok) break;
      const int Tq = step0 ? a.H + 1 : a.H;
      const int nrows = kHeads * Tq, qps = q_tiles(a, step0), items = a.B * nrows;
      const int S = a.attn_splits;
      for (int base = blockIdx.x * 4; base < items; base += nc * 4) {
        const int it = base + warp;
        if (it >= items) continue;
        const int b = it / nrows, qi = it % nrows, ti = qi / 128, qr = qi % 128;
        const size_t prow0 = ((size_t)(b * qps + ti) * S) * 128 + qr;
        float M = -INFINITY;
        for (int s = 0; s < S; ++s) {
          const size_t pr = prow0 + (size_t)s * 128;
          if (__ldcg(a.part_ml + 2 * pr + 1) > 0.f) M = fmaxf(M, __ldcg(a.part_ml + 2 * pr));
        }
        float den = 0.f, acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int s = 0; s < S; ++s) {
          const size_t pr = prow0 + (size_t)s * 128;
          const float ms = __ldcg(a.part_ml + 2 * pr), ls = __ldcg(a.part_ml + 2 * pr + 1);
          if (!(ls > 0.f)) continue;
          const float wgt = ls * ex2_approx(ms - M);
          den += wgt;
          const float4 *src = reinterpret_cast<const float4 *>(a.part_o + pr * kHeadDim + lane * 8);
          const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
          acc[0] = fmaf(wgt, x0.x, acc[0]); acc[1] = fmaf(wgt, x0.y, acc[1]);
          acc[2] = fmaf(wgt, x0.z, acc[2]); acc[3] = fmaf(wgt, x0.w, acc[3]);
          acc[4] = fmaf(wgt, x1.x, acc[4]); acc[5] = fmaf(wgt, x1.y, acc[5]);
          acc[6] = fmaf(wgt, x1.z, acc[6]); acc[7] = fmaf(wgt, x1.w, acc[7]);
        }
        const int j = qi / kHeads, hd = qi % kHeads;
        const int tok = step0 ? (j == 0 ? b : a.B + b * a.H + j - 1) : a.B + b * a.H + j;
        const float inv = den > 0.f ? 1.0f / den : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= inv;
        *reinterpret_cast<uint4 *>(a.att + (size_t)tok * kQDim + hd * kHeadDim + lane * 8) = pack8(acc);
      }
      fence_proxy_async_global();
      epi_bar();
      if (et == 0) release(a, gs);
    } else if (si.kind == LK_ACTION_IN) {
      const int nc = action_ctas(a);
      if (blockIdx.x >= nc) continue;
      ok = poll_prev(gs);
      if (!ok) break;
      const int BH = a.B * a.H;
      for (int cidx = blockIdx.x; cidx < kWidth / 8; cidx += nc) {
        const int n0 = cidx * 8;
        for (int r = et; r < BH; r += 128) {
          float acc[8];
#pragma unroll
          for (int o = 0; o < 8; ++o) acc[o] = 0.f;
          const float *x = a.xw + (size_t)r * a.A;
          for (int i = 0; i < a.A; ++i) {
            const float xi = x[i];
#pragma unroll
            for (int o = 0; o < 8; ++o) acc[o] = fmaf(__bfloat162float(a.ain_w[(size_t)(n0 + o) * a.A + i]), xi, acc[o]);
          }
#pragma unroll
          for (int o = 0; o < 8; ++o) acc[o] += a.ain_b[n0 + o];
          *reinterpret_cast<uint4 *>(a.aemb + (size_t)r * kWidth + n0) = pack8(acc);
        }
      }
      fence_proxy_async_global();
      epi_bar();
      if (et == 0) release(a, gs);
    } else if (si.kind == LK_EULER) {
      const int nc = euler_ctas(a);
      if (blockIdx.x >= nc) continue;
      ok = poll_prev(gs);
      if (!ok) break;
      const int nch = (a.A + 15) / 16, units = euler_units(a);
      const int k = si.step;
      float dt;
      if (a.linspace) {
        dt = (float)((double)(k + 1) / (double)a.N) - (float)((double)k / (double)a.N);
      } else {
        dt = (float)(-1.0 / (double)a.N);
      }
      const int last = k == a.N - 1;
      for (int u = blockIdx.x; u < units; u += nc) {
        const int i = u / nch, ch = u % nch;
        const float4 *src = reinterpret_cast<const float4 *>(a.h + (size_t)(a.B + i) * kWidth) + et * 2;
        const float4 x0 = src[0], x1 = src[1];
        float ss = x0.x * x0.x + x0.y * x0.y + x0.z * x0.z + x0.w * x0.w + x1.x * x1.x + x1.y * x1.y +
                   x1.z * x1.z + x1.w * x1.w;
        ss = warp_sum(ss);
        if (lane == 0) bs.red[warp] = ss;
        epi_bar();
        const float tot = (bs.red[0] + bs.red[1]) + (bs.red[2] + bs.red[3]);
        const float inv = 1.0f / sqrtf(tot / (float)kWidth + kRmsEps);
        const float4 *g4 = reinterpret_cast<const float4 *>(a.fnorm) + et * 2;
        const float4 g0 = g4[0], g1 = g4[1];
        float4 *y4 = reinterpret_cast<float4 *>(yrow) + et * 2;
        y4[0] = make_float4((x0.x * inv) * (1.0f + g0.x), (x0.y * inv) * (1.0f + g0.y), (x0.z * inv) * (1.0f + g0.z),
                            (x0.w * inv) * (1.0f + g0.w));
        y4[1] = make_float4((x1.x * inv) * (1.0f + g1.x), (x1.y * inv) * (1.0f + g1.y), (x1.z * inv) * (1.0f + g1.z),
                            (x1.w * inv) * (1.0f + g1.w));
        epi_bar();
        for (int o = warp; o < 16; o += 4) {
          const int aa = ch * 16 + o;
          if (aa >= a.A) break;
          const float4 *wr = reinterpret_cast<const float4 *>(a.aout_w + (size_t)aa * kWidth);
          const float4 *yr = reinterpret_cast<const float4 *>(yrow);
          float acc = 0.f;
          for (int c4 = lane; c4 < kWidth / 4; c4 += 32) {
            const float4 wv = wr[c4], yv = yr[c4];
            acc = fmaf(wv.x, yv.x, acc);
            acc = fmaf(wv.y, yv.y, acc);
            acc = fmaf(wv.z, yv.z, acc);
            acc = fmaf(wv.w, yv.w, acc);
          }
          acc = warp_sum(acc);
          if (lane == 0) {
            const size_t xi = (size_t)i * a.A + aa;
            float v = acc + a.aout_b[aa];
            if (a.x_pred) v -= a.cp->x1[xi];
            const float xn = __fadd_rn(a.xw[xi], __fmul_rn(dt, v));
            a.xw[xi] = xn;
            if (last) a.cp->x0[xi] = xn;
          }
        }
        epi_bar();  // yrow and red are reused by the next unit
      }
      epi_bar();
      if (et == 0) release(a, gs);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) k_loop(const __grid_constant__ LoopArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars &bs = *reinterpret_cast<Bars *>(smem + kOffBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kWSlots; ++i) {
      mbar_init(&bs.w_full[i], 1);
      mbar_init(&bs.w_empty[i], 1);
      bs.w_fills[i] = 0;
    }
    for (int i = 0; i < kASlots; ++i) {
      mbar_init(&bs.a_full[i], 1);
      mbar_init(&bs.a_empty[i], 1);
      bs.a_fills[i] = 0;
    }
    mbar_init(&bs.acc_full, 1);
    mbar_init(&bs.acc_empty, 1);
    bs.x_done = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bs.k_full[i], 32);  // one cp.async-completion arrival per loader lane (+ TMA bytes)
      mbar_init(&bs.k_empty[i], 1);
      mbar_init(&bs.v_full[i], 32);
      mbar_init(&bs.pv_done[i], 1);
      mbar_init(&bs.s_full[i], 1);
      mbar_init(&bs.s_empty[i], 128);
      mbar_init(&bs.p_full[i], 128);
      bs.k_fills[i] = bs.v_fills[i] = 0;
    }
    mbar_init(&bs.q_full, 128);
    mbar_init(&bs.mma_fin, 1);
    bs.last = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bs.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bs.tmem_slot;
  if (!err_set(a)) {
    if (warp == 0) {
      if (lane == 0) role_weights(a, smem, bs);
      __syncwarp();
    } else if (warp == 1) {
      role_mma(a, smem, bs, tmem);
    } else if (warp == 2 || warp == 3) {
      role_loader(a, smem, bs, warp == 3, lane);
    } else {
      role_epi(a, smem, bs, tmem, tid - 128);
    }
  }
  // Drain: every TMA fill issued into shared memory lands before the CTA exits (they
  // are consumed in normal operation; after an error some may still be in flight).
  if (lane == 0) {
    if (warp == 0)
      for (int i = 0; i < kWSlots; ++i)
        if (bs.w_fills[i]) dwait(&bs.w_full[i], (bs.w_fills[i] - 1) & 1u, a);
    if (warp == 2) {
      for (int i = 0; i < kASlots; ++i)
        if (bs.a_fills[i]) dwait(&bs.a_full[i], (bs.a_fills[i] - 1) & 1u, a);
      for (int i = 0; i < 2; ++i)
        if (bs.k_fills[i]) dwait(&bs.k_full[i], (bs.k_fills[i] - 1) & 1u, a);
    }
    if (warp == 3)
      for (int i = 0; i < 2; ++i)
        if (bs.v_fills[i]) dwait(&bs.v_full[i], (bs.v_fills[i] - 1) & 1u, a);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

void loop_attn_plan(int B, int H, int P, int grid, int &splits, int &bps) {
  const int qps = (kHeads * (H + 1) + 127) / 128;
  const int nblk = (P + kKB - 1) / kKB + (H + kKB) / kKB;
  const int qt = B * qps;
  int s = grid / (qt > 0 ? qt : 1);
  const int max_s = (nblk + 1) / 2;  // at least two key blocks per split
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  bps = (nblk + s - 1) / s;
  splits = (nblk + bps - 1) / bps;
}

size_t loop_smem_bytes() { return kSmemTotal; }

int loop_max_grid(int dev) {
  int sms = 0, coop = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) {
    cudaGetLastError();
    return 0;
  }
  if (cudaFuncSetAttribute(k_loop, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTotal) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_loop, kThreads, kSmemTotal) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return 0;
  }
  return sms;
}

cudaError_t launch_loop(const LoopArgs &a, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_loop, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTotal);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_loop, a);
}

}  // namespace pi0x
