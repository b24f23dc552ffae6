// The whole Euler loop of a small batch as one persistent kernel (bf16 mode).
//
// At small batch every Linear of the action expert reads far more weight bytes than
// activation bytes, and a layer is a chain of five dependent contractions (QKV,
// attention, O-proj, gate/up, down) whose weights do not depend on the activations.
// One cooperative launch with one CTA per SM runs every stage of every Euler step of
// the call (`sample_actions` / `denoise_step` / `embed_suffix` /
// `_compute_layer_suffix_only` on the vllm-omni pi0 page) in program order:
//
//   per step TIN (action-time MLP input), TOUT (MLP output -> residual stream,
//   layer-0 norm inputs), per layer QKV (+ RoPE), ATTN (masked MQA, one CTA per
//   128-row query tile), O (+ residual), GU (gate/up + GeGLU), DOWN (+ residual,
//   next norm inputs), and last XOUT (final norm, out-projection, x += dt v).
//
// The action-time MLP input `mlp_in([action_in(x); temb])` is evaluated as
// silu(w_xa x + tvec[k]) with w_xa = W_in[:, :W] W_action_in and the bias
// W_in[:, :W] b_action_in folded into tvec (products formed once, in float64, at
// pi0x_create): the same linear map with the action embedding not materialised,
// which turns a K = 1024 contraction into a K = action_dim one per row.
//
// Stage s of a CTA starts when the done-counter of stage s-1 (global memory, one
// per stage of the call, zeroed before the launch) reaches the number of work
// items that stage releases; counters only grow, so arrival order never matters.
// One poller (lane 0 of the V-loader warp) waits on the counters and opens a
// shared-memory gate for the other roles.  Work items release with a gpu-scope red.release after a CTA
// barrier over the threads that stored their results.
//
// Roles (256 threads):
//   warp 0    weight producer (lanes 0 and 1, alternate K-blocks): streams this CTA's
//             weight K-blocks of every stage, in program order, into a 6-slot ring of
//             16 KB.  Weights are inputs, so it runs ahead of the activations across
//             stage boundaries, bounded only by the ring.
//   warp 1    tcgen05.mma issuer of attention units (S = Q K^T, O += P V).
//   warp 2    activation loader of GEMM units; K loader of attention units.
//   warp 3    poller of the stage done-counters (lane 0), V loader of attention units.
//   warps 4-7 the MMAs of GEMM units (warp w: every fourth K-block, into its own
//             accumulator chain), their epilogues (TMEM lane quarter = warp % 4), the
//             softmax of attention units and the row-wise stages (TIN, COMBINE, XOUT).
//
// GEMM units: the weight is the MMA's M side.  128 weight rows (output features) form
// an m-tile and the call's rows, rounded up to 16 tokens, are N, so one tcgen05.mma
// does 128 x N x 16 of useful work (on B200 each MMA costs its issuing warp about
// 200 cycles whatever N is, so a small batch wants few, wide MMAs).  The K range of
// every m-tile is split over ksplit CTAs (ksplit = grid / m-tiles, at most one per
// K-block), so every Linear streams its weight through nearly every SM.  Each unit
// stores its fp32 partial tile (token-major), raises its m-tile's counter, waits for
// the other splits and adds a slice of the tokens over all splits in split order (the
// result does not depend on timing), then runs the epilogue for that slice: bias or
// residual with the fused RMSNorm producer (bf16 h*(1+g), per-m-tile sums of h^2),
// RoPE at position n_b + j with q/k/v stores, or GeGLU.
//
// Copies: on B200 every async copy costs its issuing thread about 0.2 us whatever its
// size, so the loop copies large contiguous runs: weights are stored once, at
// pi0x_create, as m-tiles of swizzled 128 x 64 K-blocks (one 16 KB bulk copy per
// K-block); the activation operands (norm outputs, attention output, GeGLU product,
// MLP input) are written by their producers as tiled K-blocks (tiled_off), one bulk
// copy per K-block, issued by four lanes at once.  The attention's prefix K/V (a call
// input) is prefetched into L2, a slice per CTA, when the QKV stage of its layer begins.
//
// Shared memory: region X (128 KB) holds either the activation ring of a GEMM unit
// or the K/V rings (3 x 16 KB each) and P buffers (2 x 16 KB) of an attention unit,
// handed from unit to unit through a counter of units whose MMAs have completed; then
// the weight ring (6 x 16 KB); XOUT keeps its normalised row in region X.
//
// Every wait is bounded (LoopArgs::wait_ns) and gives up early once the error word
// is set; on the way out each role waits for the copies it issued, the MMA warp for
// its MMAs, and TMEM is freed.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

#ifdef PI0X_LOOP_TIMELINE
// Profiling build: globaltimer stamps per (stage, CTA, slot) into a device buffer.
__device__ unsigned long long *g_loop_tl = nullptr;
#define LOOP_STAMP(gs, slot)                                                                           \
  do {                                                                                                 \
    if (g_loop_tl) g_loop_tl[((size_t)(gs) * gridDim.x + blockIdx.x) * 16 + (slot)] = globaltimer_ns(); \
  } while (0)
#else
#define LOOP_STAMP(gs, slot) \
  do {                       \
  } while (0)
#endif

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kXBytes = 128 * 1024;
constexpr int kWSlots = 6;
constexpr uint32_t kWSlotBytes = 16384;           // one K-block of a 128-row weight m-tile
constexpr int kKB = kLoopKeyBlock;            // 32 keys per attention block
constexpr int kKVBufs = 3;
constexpr uint32_t kKVTile = kKB * 512;       // 32 keys x 256 dims bf16 = 16 KB
constexpr uint32_t kKVSub = kKB * 128;        // one 64-dim sub-tile = 4 KB
constexpr uint32_t kAtomBytes = 8 * 128;      // 8 keys x 64 dims: one 8-row box
constexpr uint32_t kPTile = 128 * 128;        // 128 rows x 128 B (32 keys used)

constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffA = kOffX;
constexpr uint32_t kOffK = kOffX;
constexpr uint32_t kOffV = kOffK + kKVBufs * kKVTile;
constexpr uint32_t kOffP = kOffV + kKVBufs * kKVTile;
static_assert(kOffP + 2 * kPTile == kOffX + kXBytes, "attention buffers fill region X");
constexpr uint32_t kOffW = kOffX + kXBytes;
constexpr uint32_t kOffBar = kOffW + kWSlots * kWSlotBytes;
constexpr int kMaxASlots = 24;

struct Bars {
  uint64_t w_full[kWSlots], w_empty[kWSlots];
  uint64_t a_full[kMaxASlots], a_empty[kMaxASlots];
  uint64_t acc_full;
  uint64_t k_full[kKVBufs], k_empty[kKVBufs], v_full[kKVBufs], pv_done[kKVBufs];
  uint64_t s_full[2], s_empty[2], p_full[2];
  uint64_t q_full, mma_fin;
  uint64_t epi_fin;   // the epilogue warps' GEMM MMAs have completed (exit)
  uint64_t red_full;  // GEMM reduce: the m-tile's partial slices have landed in region X
  uint32_t tmem_slot;
  uint32_t x_done;    // units that used region X and whose MMAs have completed (monotonic)
  uint32_t tmem_done; // units whose accumulator reads (GEMM) / O readout (attention) are done
  uint32_t ready;     // stages whose predecessor has completed (monotonic, set by the poller)
  int last;           // epilogue broadcast: the m-tile's partials are all stored
  float red[8];
  uint32_t w_fills[kWSlots];  // drain bookkeeping
  uint32_t a_fills[kMaxASlots];
  uint32_t k_fills[kKVBufs], v_fills[kKVBufs];
  uint32_t red_fills;
  uint32_t epi_err;  // an epilogue warp's wait gave up (read by all four after a barrier)
};
constexpr uint32_t kBarBytes = ((sizeof(Bars) + 127) / 128) * 128;
// GEMM reduce scratch: the slice's per-token rstd and RoPE positions (128 + 128 words).
// (XOUT's normalised row uses region X, which no copy fills during that stage.)
constexpr uint32_t kOffScratch = kOffBar + kBarBytes;
constexpr uint32_t kSmemTotal = kOffScratch + 1024 + 1024 /* alignment slack */;
static_assert(kSmemTotal <= 232448, "shared memory per CTA");

// TMEM columns: S 0..127 (two buffers x two dim-halves of 32 columns), Q 128..255
// (bf16 pairs), O 256..511.  A GEMM unit's accumulator (128 weight rows x box_rows
// tokens) uses 256..383: units run one at a time per CTA and each starts after the
// previous one's TMEM reads.
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemQ = 128;
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kTmemAcc = 256;
constexpr uint32_t kTmemCols = 512;

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;

__device__ __forceinline__ int ld_relaxed(const int *p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int *p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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
// Drain wait at exit: bounded by time only (it must wait for copies in flight even
// after the error word was set).
__device__ __forceinline__ void dwait(uint64_t *bar, uint32_t parity, const LoopArgs &a) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > a.wait_ns) return;
}
// Wait until *c >= need for a shared-memory counter written by another role
// (monotonic, so a late reader never misreads it); bounded like lwait.
__device__ __forceinline__ bool smem_wait(const uint32_t *cnt, uint32_t need, const LoopArgs &a, unsigned bit) {
  const volatile uint32_t *c = cnt;
  if (*c >= need) {
    __threadfence_block();
    return true;
  }
  // back off between polls: a tight loop of shared-memory loads competes for the SM's
  // shared-memory / shuffle pipe with the warps doing the work being waited for
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 16; ++i) {
      if (*c >= need) {
        __threadfence_block();
        return true;
      }
      __nanosleep(64);
    }
    if (err_set(a)) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicOr(a.err, bit);
      return false;
    }
  }
}
__device__ __forceinline__ void smem_publish(uint32_t *cnt, uint32_t v) {
  __threadfence_block();
  *(volatile uint32_t *)cnt = v;
}
// Stage gate: the poller opened stage gs (its predecessor completed, acquired at gpu scope).
__device__ __forceinline__ bool gate(Bars &bs, int gs, const LoopArgs &a) {
  return smem_wait(&bs.ready, (uint32_t)gs + 1u, a, kErrTimeoutFlag);
}
// Region X hand-off.
__device__ __forceinline__ void x_release(Bars &bs) {
  __threadfence_block();
  atomicAdd(&bs.x_done, 1u);
}

// TMEM load of 32 lanes x 16 fp32 columns without its wait: issue several, then one
// tc_wait_ld_regs64 over the registers they write (named there, so that no use of
// them moves above the wait).
__device__ __forceinline__ void tmem_ld_x16_nw(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld_regs64(uint32_t (&r)[64]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
               :
               : "memory");
}

// Store of 8 bf16 at offset `off` of every replica of a tiled activation buffer.
__device__ __forceinline__ void store_reps(bf16 *buf, size_t off, size_t rep_stride, uint4 v) {
#pragma unroll
  for (int r = 0; r < kLoopReps; ++r) *reinterpret_cast<uint4 *>(buf + r * rep_stride + off) = v;
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
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
  int kind, layer, step;
};
__device__ __forceinline__ int total_stages(const LoopArgs &a) { return loop_total_stages(a.N, a.L, a.attn_splits); }
__device__ __forceinline__ StageInfo stage_at(const LoopArgs &a, int gs) {
  StageInfo si;
  loop_stage(gs, a.L, a.attn_splits, si.kind, si.layer, si.step);
  return si;
}
__device__ __forceinline__ int q_tiles(const LoopArgs &a, int step0) {
  const int Tq = step0 ? a.H + 1 : a.H;
  return (kHeads * Tq + 127) / 128;
}
__device__ __forceinline__ int attn_units(const LoopArgs &a, int step0) { return a.B * q_tiles(a, step0) * a.attn_splits; }
// COMBINE warp items: (query tile, 32-row group, 8-dim group).
__device__ __forceinline__ int combine_items(const LoopArgs &a, int step0) {
  return a.B * q_tiles(a, step0) * 4 * (kHeadDim / 8);
}
__device__ __forceinline__ int combine_ctas(const LoopArgs &a, int step0) {
  const int c = (combine_items(a, step0) + 3) / 4;
  return c < a.grid ? c : a.grid;
}
// TIN: 128 units of 8 output columns (all rows); XOUT: units of (action row, 16 outputs).
__device__ __forceinline__ int tin_ctas(const LoopArgs &a) { return a.grid < kWidth / 8 ? a.grid : kWidth / 8; }
__device__ __forceinline__ int xout_units(const LoopArgs &a) { return a.B * a.H * ((a.A + 15) / 16); }
__device__ __forceinline__ int xout_ctas(const LoopArgs &a) {
  const int u = xout_units(a);
  return u < a.grid ? u : a.grid;
}
// Arrivals that complete stage `si`.
__device__ __forceinline__ int stage_expect(const LoopArgs &a, const StageInfo &si) {
  const int step0 = si.step == 0;
  switch (si.kind) {
    case LK_TIN: return tin_ctas(a);
    case LK_XOUT: return xout_ctas(a);
    case LK_ATTN: return attn_units(a, step0);
    case LK_COMBINE: return combine_ctas(a, step0);
    default: {
      const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
      return p.mtiles * p.ksplit;
    }
  }
}
// Release of a stage's work item (one thread, after epi_bar() ordered the item's
// stores before it).
__device__ __forceinline__ void release(const LoopArgs &a, int gs) { red_release_add(a.done + gs, 1); }

// GEMM unit u: m-tile m (weight rows 128 m ..), K split s, K-blocks [kb0, kb1).
struct GUnit {
  int m, s, kb0, kb1;
};
__device__ __forceinline__ GUnit gemm_unit(const LoopGemm &p, int u) {
  GUnit g;
  g.m = u / p.ksplit;
  g.s = u % p.ksplit;
  const int nk = p.K / 64;
  g.kb0 = (int)((long)g.s * nk / p.ksplit);
  g.kb1 = (int)((long)(g.s + 1) * nk / p.ksplit);
  return g;
}
// Tokens [t0, t1) of the stored range [r_lo, r_hi) that split s of an m-tile adds up
// (an even count per split, so the paired epilogues take two tokens at a time).
__device__ __forceinline__ void red_slice(int r_lo, int r_hi, int ksplit, int s, int &t0, int &t1) {
  const int per = (((r_hi - r_lo) + ksplit - 1) / ksplit + 1) & ~1;
  t0 = min(r_hi, r_lo + s * per);
  t1 = min(r_hi, t0 + per);
}
// Bounded wait until a global counter reaches `need` (then acquired at gpu scope).
// Every poll is an acquire load: the load that sees the count is the acquire, with no
// further L2 round trip after it.
__device__ bool gwait(const int *cnt, int need, const LoopArgs &a, unsigned bit) {
  if (ld_acquire(cnt) >= need) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (ld_acquire(cnt) >= need) return true;
    if (err_set(a)) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicOr(a.err, bit);
      return false;
    }
  }
}
__device__ __forceinline__ const bf16 *weight_tiles(const LoopArgs &a, int kind, int layer) {
  switch (kind) {
    case LK_TOUT: return a.w_tout;
    case LK_QKV: return a.w_qkv[layer];
    case LK_O: return a.w_o[layer];
    case LK_GU: return a.w_gu[layer];
    default: return a.w_down[layer];
  }
}
// Activation operand of a GEMM stage (tiled K-blocks of box_rows rows).
__device__ __forceinline__ const bf16 *act_tiles(const LoopArgs &a, int kind) {
  const size_t rep = (size_t)(blockIdx.x % kLoopReps) * a.rep_rows;
  switch (kind) {
    case LK_TOUT: return a.uemb + rep * kWidth;
    case LK_QKV: case LK_GU: return a.xn + rep * kWidth;
    case LK_O: return a.att + rep * kQDim;
    default: return a.act + rep * kMlp;
  }
}
// Rows of a GEMM stage: the MMA runs over every row of the activation tile; tile rows
// [r_lo, r_hi) are stored, tile row r as output row r + out_off.
__device__ __forceinline__ void gemm_rows(const LoopArgs &a, int kind, int step0, int &r_lo, int &r_hi, int &out_off) {
  if (kind == LK_TOUT) {
    r_lo = 0;
    r_hi = a.B * a.H;
    out_off = a.B;
    return;
  }
  r_lo = step0 ? 0 : a.B;
  r_hi = a.R;
  out_off = 0;
}
__device__ __forceinline__ uint32_t a_slot_bytes(const LoopArgs &a) { return (uint32_t)a.box_rows * 128u; }
__device__ __forceinline__ int a_slots(const LoopArgs &a) {
  const int n = (int)(kXBytes / a_slot_bytes(a));
  return n < kMaxASlots ? n : kMaxASlots;
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
    if (lane == 0) mbar_expect_tx(full, kKVTile);
    __syncwarp();
    if (lane < 4) {  // one 32-row box per 64-dim sub-tile, four issuing lanes
      const CUtensorMap *m = (c0 & 1) ? smap32 : pmap32;
      const int y = (c0 & 1) ? sfx_row0 + (c0 >> 1) : (c0 >> 1);
      tma_load_2d(tile + lane * kKVSub, m, lane * 64, y, full);
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

// ---- poller (warp 3, lane 0): open stage gs once stage gs - 1 has completed ----------
__device__ bool poll_stage(const LoopArgs &a, Bars &bs, int gs) {
  if (gs > 0) {
    // acquire the predecessor's results at gpu scope (the load that sees the count)
    if (!gwait(a.done + (gs - 1), stage_expect(a, stage_at(a, gs - 1)), a, kErrTimeoutFlag)) return false;
  }
  if (gs == a.debug_stall_stage) {  // test hook: a counter that nothing raises
    const unsigned long long t0 = globaltimer_ns();
    while (ld_relaxed(a.done + gs) < (1 << 30)) {
      if (err_set(a)) return false;
      if (globaltimer_ns() - t0 > a.wait_ns) {
        atomicOr(a.err, kErrTimeoutFlag);
        return false;
      }
    }
  }
  smem_publish(&bs.ready, (uint32_t)gs + 1u);
  return true;
}

// ---- role: weight producer (warp 0, lanes 0 and 1) ----------------------------------
// One 16 KB bulk copy per K-block of the unit's m-tile (the K-blocks of a unit are one
// contiguous run of the tiled weight); the two lanes take alternate K-blocks so two
// copies are in issue at once.
__device__ void role_weights(const LoopArgs &a, uint8_t *smem, Bars &bs, int me) {
  const int total = total_stages(a);
  uint32_t wi = 0;
  bool ok = true;
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    if (!loop_is_gemm(si.kind)) continue;
    const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
    const bf16 *wt = weight_tiles(a, si.kind, si.layer);
    const int U = p.mtiles * p.ksplit;
    // the same unit's weights one layer later (the next step's first layer after the
    // last): they go to L2 now, so their copies a layer from now are L2 hits
    const bf16 *wnext = nullptr;
    if (si.kind != LK_TOUT) {
      if (si.layer + 1 < a.L)
        wnext = weight_tiles(a, si.kind, si.layer + 1);
      else if (si.step + 1 < a.N)
        wnext = weight_tiles(a, si.kind, 0);
    }
    for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
      const GUnit g = gemm_unit(p, u);
      const bf16 *src = wt + (size_t)g.m * 128 * p.K;
      if (wnext && me == 0)
        prefetch_l2(wnext + (size_t)g.m * 128 * p.K + (size_t)g.kb0 * 128 * 64, (uint32_t)(g.kb1 - g.kb0) * kWSlotBytes);
      // rounds of two K-blocks, one per lane, the two lanes in step (as the activation
      // loader's four): a lane that waited alone in a diverged warp could hold back the
      // other lane's fill that its own wait depends on
      const int nk = g.kb1 - g.kb0;
      for (int i0 = 0; i0 < nk && ok; i0 += 2) {
        const int i = i0 + me;
        bool good = true;
        if (i < nk) {
          const uint32_t f = wi + (uint32_t)i;
          const int slot = f % kWSlots;
          const uint32_t n = f / kWSlots;
          if (n > 0) good = lwait(&bs.w_empty[slot], (n - 1) & 1u, a, kErrTimeoutProducer);
          if (good) {
            mbar_arrive_expect_tx(&bs.w_full[slot], kWSlotBytes);
            bulk_load(smem_u32(smem + kOffW + slot * kWSlotBytes), src + (size_t)(g.kb0 + i) * 128 * 64, kWSlotBytes,
                      &bs.w_full[slot]);
            bs.w_fills[slot] = n + 1;
          }
        }
        ok = __all_sync(0x3u, good);
      }
      wi += (uint32_t)nk;
      LOOP_STAMP(gs, 5);
    }
  }
}

// ---- role: MMA issuer (warp 1, whole warp; one elected lane issues) ------------------
__device__ void role_mma(const LoopArgs &a, uint8_t *smem, Bars &bs, uint32_t tmem) {
  const int total = total_stages(a);
  const uint32_t sbase = smem_u32(smem);
  const int nas = a_slots(a);
  const uint32_t asb = a_slot_bytes(a);
  uint32_t kj = 0, vj = 0, sj = 0, pj = 0, qn = 0;
  bool ok = true;
  const uint64_t kdesc0 = smem_desc_k_sw128(sbase + kOffK, 0);
  const uint64_t pdesc0 = smem_desc_k_sw128(sbase + kOffP, 0);
  const uint64_t vdesc0 = smem_desc_mn_sw128(sbase + kOffV, kKVSub, 1024);
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKB);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim) | (1u << 16);  // B (V) MN-major
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    if (si.kind == LK_ATTN) {
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
          const int kbuf = kj % kKVBufs, sb = sj & 1;
          if (!__all_sync(kFull, lwait(&bs.k_full[kbuf], (kj / kKVBufs) & 1u, a, kErrTimeoutMma))) return false;
          if (sj >= 2 && !__all_sync(kFull, lwait(&bs.s_empty[sb], ((sj >> 1) - 1) & 1u, a, kErrTimeoutMma)))
            return false;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t kd = kdesc0 + (uint64_t)((kbuf * kKVTile) >> 4);
          // two independent chains: head dims 0..127 into S columns sb*64 + 0..31,
          // dims 128..255 into sb*64 + 32..63 (the softmax adds them)
#pragma unroll
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16_ts_w(tmem + kTmemS + (uint32_t)(sb * 2 * kKB + (s >> 1) * kKB),
                               tmem + kTmemQ + (uint32_t)(32 * s + 8 * kk),
                               kd + (uint64_t)((s * kKVSub + kk * 32) >> 4), idesc_s, ((s & 1) | kk) != 0);
          tc_commit_w(&bs.s_full[sb]);
          tc_commit_w(&bs.k_empty[kbuf]);
          ++kj;
          ++sj;
          return true;
        };
        auto issue_pv = [&](int j) -> bool {  // O += P(pj) V(vj)
          const int vbuf = vj % kKVBufs, pb = pj % 2;
          if (!__all_sync(kFull, lwait(&bs.p_full[pb], (pj / 2) & 1u, a, kErrTimeoutMma))) return false;
          if (!__all_sync(kFull, lwait(&bs.v_full[vbuf], (vj / kKVBufs) & 1u, a, kErrTimeoutMma))) return false;
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
  const int total = total_stages(a);
  const uint32_t sbase = smem_u32(smem);
  const int nas = a_slots(a);
  const uint32_t asb = a_slot_bytes(a);
  uint32_t ai = 0, kj = 0, x_units = 0;
  bool ok = true;
  // region X: wait until every earlier unit that used it has finished its MMAs
  auto take_x = [&]() -> bool {
    bool good = true;
    if (lane == 0) good = smem_wait(&bs.x_done, x_units, a, kErrTimeoutProducer);
    ++x_units;
    good = __shfl_sync(kFull, (int)good, 0) != 0;
    __syncwarp();
    return good;
  };
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    const int step0 = si.step == 0;
    if (is_v) {  // the stage's gate first (this warp's own V loads of stage gs come after)
      if (lane == 0) ok = poll_stage(a, bs, gs);
      ok = __shfl_sync(kFull, (int)ok, 0) != 0;
      if (!ok) break;
    }
    if (loop_is_gemm(si.kind)) {
      const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
      const int U = p.mtiles * p.ksplit;
      if (blockIdx.x >= U) continue;
      const bf16 *abase = act_tiles(a, si.kind);
      const size_t kb_elems = (size_t)a.box_rows * 64;  // one K-block tile
      if (si.kind == LK_QKV && !is_v && lane < 2 && a.P > 0) {
        // this CTA's slice of the layer's prefix K (lane 0) / V (lane 1) into L2
        const size_t bytes = (size_t)a.B * a.P * kHeadDim * 2;
        const size_t slice = ((bytes + gridDim.x - 1) / gridDim.x + 15) & ~size_t(15);
        const size_t off = (size_t)blockIdx.x * slice;
        if (off < bytes) {
          const uint8_t *base = reinterpret_cast<const uint8_t *>(lane ? a.cp->prefix_v[si.layer] : a.cp->prefix_k[si.layer]);
          prefetch_l2(base + off, (uint32_t)(bytes - off < slice ? bytes - off : slice));
        }
      }
      bool opened = false;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        ok = take_x();
        if (!ok) break;
        if (is_v) continue;
        if (!opened) {
          ok = gate(bs, gs, a);
          fence_proxy_async_global();  // the tiles were written through the generic proxy
          if (lane == 0) LOOP_STAMP(gs, 4);
          opened = true;
        }
        ok = __all_sync(kFull, ok);
        if (!ok) break;
        const GUnit g = gemm_unit(p, u);
        const int nk = g.kb1 - g.kb0;
        // lanes 0..3 copy one K-block tile each per round
        for (int i0 = 0; i0 < nk && ok; i0 += 4) {
          const int i = i0 + lane;
          bool good = true;
          if (lane < 4 && i < nk) {
            const uint32_t f = ai + (uint32_t)i;
            const int slot = f % nas;
            const uint32_t n = f / nas;
            if (n > 0) good = lwait(&bs.a_empty[slot], (n - 1) & 1u, a, kErrTimeoutProducer);
            if (good) {
              mbar_arrive_expect_tx(&bs.a_full[slot], asb);
              bulk_load(smem_u32(smem + kOffA + slot * asb), abase + (size_t)(g.kb0 + i) * kb_elems, asb,
                        &bs.a_full[slot]);
              bs.a_fills[slot] = n + 1;
            }
          }
          ok = __all_sync(kFull, good);
        }
        if (lane == 0) LOOP_STAMP(gs, 3);
        ai += (uint32_t)nk;
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
          // the maps are rewritten in global memory before every call: each lane that
          // may issue a tensor copy with them (load_kv_tile) acquires them itself, since
          // the fence orders the executing thread's tensor-map accesses only
          if (a.P > 0) {
            tma_map_acquire(pmap);
            tma_map_acquire(pmap32);
          }
          tma_map_acquire(smap);
          tma_map_acquire(smap32);
          __syncwarp();
          maps_ready = true;
        }
        const int *vi = a.vidx + (size_t)t.b * a.P;
        const bool contig = t.nv == 0 || vi[t.nv - 1] == t.nv - 1;
        for (int j = 0; j < t.nb && ok; ++j, ++kj) {
          const int blk = t.blk0 + j;
          if (!sfx_ready && blk >= t.nbp) {  // suffix keys come from this step's QKV stage
            if (lane == 0) {
              ok = gate(bs, gs, a);
              fence_proxy_async_global();
            }
            ok = __all_sync(kFull, __shfl_sync(kFull, (int)ok, 0) != 0);
            if (!ok) break;
            sfx_ready = true;
          }
          const int buf = kj % kKVBufs;
          const uint32_t n = kj / kKVBufs;
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

// ---- GEMM epilogues ---------------------------------------------------------------
// rstd of output row `orow` from the fused-norm producer's per-m-tile sums of h^2.
__device__ __forceinline__ float row_rstd(const float *ss, int ld, int orow) {
  float t = 0.f;
#pragma unroll
  for (int g = 0; g < kLoopNormSlots; ++g) t += ss[(size_t)g * ld + orow];
  return 1.0f / sqrtf(t / (float)kWidth + kRmsEps);
}
__device__ __forceinline__ const float *producer_gain(const LoopArgs &a, int kind, int layer) {
  if (kind == LK_TOUT) return a.in_norm[0];
  if (kind == LK_O) return a.post_norm[layer];
  if (kind == LK_DOWN) return layer + 1 < a.L ? a.in_norm[layer + 1] : nullptr;
  return nullptr;
}
__device__ __forceinline__ uint2 pack4(float a0, float a1, float a2, float a3) {
  const __nv_bfloat162 p0 = __floats2bfloat162_rn(a0, a1), p1 = __floats2bfloat162_rn(a2, a3);
  return make_uint2(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1));
}
__device__ __forceinline__ void store_reps4(bf16 *buf, size_t off, size_t rep_stride, uint2 v) {
#pragma unroll
  for (int r = 0; r < kLoopReps; ++r) *reinterpret_cast<uint2 *>(buf + r * rep_stride + off) = v;
}
// RoPE position of output row `orow`: the state token sits at n_b, action j at n_b + 1 + j.
__device__ __forceinline__ int rope_pos(const LoopArgs &a, int orow) {
  if (orow < a.B) return a.nvalid[orow];
  const int b = (orow - a.B) / a.H, j = (orow - a.B) % a.H;
  return a.nvalid[b] + 1 + j;
}
__device__ __forceinline__ void add4(float4 &d, const float4 &x) {
  d.x += x.x;
  d.y += x.y;
  d.z += x.z;
  d.w += x.w;
}

// Reduce + epilogue of tokens [t0, t1) of m-tile g.m (warps 4-7).  `stage` receives
// the m-tile's partial tiles for the slice, split-major (split s, slice token j, 128
// rows as 32 quads of 4 rows), from one bulk copy per split completing on `staged`; every
// output adds its splits in a fixed order, so the result does not depend on timing.
// One warp per SM sub-partition runs this, so the items of a thread are unrolled with
// independent registers (no shuffles or divergent branches) to overlap their latencies,
// and their global operands load while the copies are in flight.  A wait that runs out
// (bounded by the call's limit) leaves the error word set by the caller's next wait.
//
// Residual kinds (TOUT: bias; O, DOWN: residual), item (token, quad q = lane), a warp
// per token: update h and, with a following norm, store bf16 h*(1+g) and the token's
// sum of h^2 over the m-tile (norm slot m).  Paired kinds, item (token, pair quad):
// rows 16i+e and 16i+8+e of the m-tile hold rotation pair (d, d+128) of one head for
// QKV (the stored weight interleaves them) and gate / up of one hidden feature for GU,
// so pair quad pq (i = pq >> 1, e = 4 (pq & 1) ..) reads quads 4i + (pq & 1) and that
// + 2, scales both by the token's rstd, then rotates and stores q / k / v (QKV) or
// stores GeGLU(g, u) (GU).  rstd_s / pos_s hold the slice's per-token rstd and RoPE
// position (paired kinds).
constexpr int kRedItems = 4;
__device__ void reduce_unit(const LoopArgs &a, const StageInfo &si, const LoopGemm &p, const GUnit &g, int t0,
                            int t1, int out_off, int et, const float4 *stage, const float *rstd_s, const int *pos_s,
                            uint64_t *staged, uint32_t staged_parity, int gs) {
  (void)gs;  // timeline stamps only
  // the call's pointers and sizes in registers: read through `a` after every store
  // (which may alias it, as far as the compiler can tell) they would be reloaded
  const int kind = si.kind, layer = si.layer;
  const int lane = et & 31, ks = p.ksplit, T = t1 - t0;
  const int rb = a.box_rows, ss_ld = a.ss_ld, R = a.R, B = a.B, H = a.H;
  const int step0 = si.step == 0, qps = q_tiles(a, step0);
  const size_t rep_w = (size_t)a.rep_rows * kWidth, rep_m = (size_t)a.rep_rows * kMlp;
  float *const hbuf = a.h;
  bf16 *const xn = a.xn, *const act = a.act, *const qb = a.q, *const kbuf = a.ks, *const vbuf = a.vs;
  const float *const tout_b = a.tout_b, *const rope = a.rope_tab;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  if (kind == LK_QKV || kind == LK_GU) {
    const int items = T * 16, hd = g.m >> 1;
    const bool rot = kind == LK_QKV && hd < kHeads + 1;
    float4 c01[kRedItems], c23[kRedItems];
    auto load_ops = [&](int it0) {
#pragma unroll
      for (int i = 0; i < kRedItems; ++i) {
        const int it = it0 + 128 * i;
        c01[i] = c23[i] = zero;
        if (rot && it < items) {
          const int pq = it & 15, d0 = ((g.m & 1) * 8 + (pq >> 1)) * 8 + (pq & 1) * 4;
          const float4 *tab = reinterpret_cast<const float4 *>(rope + ((size_t)pos_s[it >> 4] * (kHeadDim / 2) + d0) * 2);
          c01[i] = tab[0];
          c23[i] = tab[1];
        }
      }
    };
    load_ops(et);
    lwait(staged, staged_parity, a, kErrTimeoutEpilogue);  // the slices have landed
    for (int it0 = et; it0 < items; it0 += 128 * kRedItems) {
      if (it0 != et) load_ops(it0);
      float4 lo4[kRedItems], hi4[kRedItems];
#pragma unroll
      for (int i = 0; i < kRedItems; ++i) {
        const int it = it0 + 128 * i;
        lo4[i] = hi4[i] = zero;
        if (it >= items) continue;
        const int j = it >> 4, pq = it & 15, ql = (pq >> 1) * 4 + (pq & 1);
        const float4 *st = stage + (size_t)j * 32;
        for (int sp = 0; sp < ks; ++sp) {
          add4(lo4[i], st[(size_t)sp * T * 32 + ql]);
          add4(hi4[i], st[(size_t)sp * T * 32 + ql + 2]);
        }
      }
#pragma unroll
      for (int i = 0; i < kRedItems; ++i) {
        const int it = it0 + 128 * i;
        if (it >= items) continue;
        const int j = it >> 4, pq = it & 15, orow = t0 + j + out_off;
        const int gq = pq >> 1, e0 = (pq & 1) * 4;
        const float rs = rstd_s[j];
        float lo[4] = {lo4[i].x * rs, lo4[i].y * rs, lo4[i].z * rs, lo4[i].w * rs};
        float hi[4] = {hi4[i].x * rs, hi4[i].y * rs, hi4[i].z * rs, hi4[i].w * rs};
        if (kind == LK_GU) {
          float t[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) t[q] = gelu_tanh_fast(lo[q]) * hi[q];
          store_reps4(act, tiled_off(orow, g.m * 64 + gq * 8 + e0, rb), rep_m, pack4(t[0], t[1], t[2], t[3]));
          continue;
        }
        if (rot) {
          const float cs[4] = {c01[i].x, c01[i].z, c23[i].x, c23[i].z}, sn[4] = {c01[i].y, c01[i].w, c23[i].y, c23[i].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float x0 = lo[q], x1 = hi[q];
            lo[q] = x0 * cs[q] - x1 * sn[q];
            hi[q] = x1 * cs[q] + x0 * sn[q];
          }
        }
        const int d0 = ((g.m & 1) * 8 + gq) * 8 + e0;
        if (hd < kHeads) {
          // query row qi = jq * 8 + head of sample b (jq: the state token at step 0, then
          // the actions): tile b * qps + qi / 128, stored as [8-dim chunk][row][8 dims]
          int b, jq;
          if (orow < B) {
            b = orow;
            jq = 0;
          } else {
            b = (orow - B) / H;
            jq = (orow - B) % H + (step0 ? 1 : 0);
          }
          const int qi = jq * kHeads + hd;
          bf16 *tile = qb + (size_t)(b * qps + (qi >> 7)) * 128 * kHeadDim + (size_t)(qi & 127) * 8 + (d0 & 7);
          *reinterpret_cast<uint2 *>(tile + (size_t)(d0 >> 3) * 128 * 8) = pack4(lo[0], lo[1], lo[2], lo[3]);
          *reinterpret_cast<uint2 *>(tile + (size_t)((d0 + kHeadDim / 2) >> 3) * 128 * 8) = pack4(hi[0], hi[1], hi[2], hi[3]);
        } else {
          bf16 *dst = (hd == kHeads ? kbuf : vbuf) + ((size_t)layer * R + orow) * kHeadDim + d0;
          *reinterpret_cast<uint2 *>(dst) = pack4(lo[0], lo[1], lo[2], lo[3]);
          *reinterpret_cast<uint2 *>(dst + kHeadDim / 2) = pack4(hi[0], hi[1], hi[2], hi[3]);
        }
      }
    }
    return;
  }
  const int items = T * 32;
  const float *gain = producer_gain(a, kind, layer);
  float *ss = kind == LK_O ? a.ss_m : a.ss_a;
  const int n = g.m * 128 + 4 * lane;  // the item's 4 features
  float4 ex[kRedItems], gx[kRedItems];
  auto load_ops = [&](int it0) {
#pragma unroll
    for (int i = 0; i < kRedItems; ++i) {
      const int it = it0 + 128 * i;
      ex[i] = gx[i] = zero;
      if (it >= items) continue;
      const int orow = t0 + (it >> 5) + out_off;
      ex[i] = kind == LK_TOUT ? *reinterpret_cast<const float4 *>(tout_b + n)
                              : *reinterpret_cast<const float4 *>(hbuf + (size_t)orow * kWidth + n);
      if (gain) gx[i] = *reinterpret_cast<const float4 *>(gain + n);
    }
  };
  load_ops(et);
  lwait(staged, staged_parity, a, kErrTimeoutEpilogue);  // the slices have landed
  for (int it0 = et; it0 < items; it0 += 128 * kRedItems) {
    if (it0 != et) load_ops(it0);
    float4 v4[kRedItems];
#pragma unroll
    for (int i = 0; i < kRedItems; ++i) {
      const int it = it0 + 128 * i;
      v4[i] = zero;
      if (it >= items) continue;
      // splits 0, 2, 4 .. and 1, 3, 5 .. in two chains, then their sum (a fixed order)
      const float4 *st = stage + (size_t)(it >> 5) * 32 + lane;
      float4 odd = zero;
      int sp = 0;
      for (; sp + 1 < ks; sp += 2) {
        add4(v4[i], st[(size_t)sp * T * 32]);
        add4(odd, st[(size_t)(sp + 1) * T * 32]);
      }
      if (sp < ks) add4(v4[i], st[(size_t)sp * T * 32]);
      add4(v4[i], odd);
    }
#pragma unroll
    for (int i = 0; i < kRedItems; ++i) {
      const int it = it0 + 128 * i;
      if (it >= items) continue;  // warp-uniform: items is a multiple of 32
      const int orow = t0 + (it >> 5) + out_off;
      float4 v = v4[i];
      add4(v, ex[i]);
      *reinterpret_cast<float4 *>(hbuf + (size_t)orow * kWidth + n) = v;
      if (gain) {
        const float4 gg = gx[i];
        store_reps4(xn, tiled_off(orow, n, rb), rep_w,
                    pack4(v.x * (1.0f + gg.x), v.y * (1.0f + gg.y), v.z * (1.0f + gg.z), v.w * (1.0f + gg.w)));
        const float sq = warp_sum(fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, v.w * v.w))));
        if (lane == 0) ss[(size_t)g.m * ss_ld + orow] = sq;
      }
    }
  }
}

// TIN unit c (warps 4-7): columns [8c, 8c + 8) of the step's action-time MLP input
// for every action row, u = silu(w_xa x + tvec[k]); thread et takes row et (x_1 at
// step 0, else the integrated x).
__device__ __forceinline__ void tin_unit(const LoopArgs &a, int cidx, int k, int et) {
  const int A = a.A, BH = a.B * a.H, n0 = cidx * 8;
  const float *xsrc = k == 0 ? a.cp->x1 : a.xw;
  const float *tv = a.tvec + (size_t)k * kWidth + n0;
  for (int r = et; r < BH; r += 128) {
    float u[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) u[o] = tv[o];
    const float4 *xr = reinterpret_cast<const float4 *>(xsrc + (size_t)r * A);
#pragma unroll 4
    for (int j4 = 0; j4 < A / 4; ++j4) {
      const float4 xv = xr[j4];
#pragma unroll
      for (int o = 0; o < 8; ++o) {
        const float4 wv = reinterpret_cast<const float4 *>(a.w_xa + (size_t)(n0 + o) * A)[j4];
        u[o] = fmaf(wv.x, xv.x, u[o]);
        u[o] = fmaf(wv.y, xv.y, u[o]);
        u[o] = fmaf(wv.z, xv.z, u[o]);
        u[o] = fmaf(wv.w, xv.w, u[o]);
      }
    }
#pragma unroll
    for (int o = 0; o < 8; ++o) u[o] = silu_f(u[o]);
    store_reps(a.uemb, tiled_off(r, n0, a.box_rows), (size_t)a.rep_rows * kWidth, pack8(u));
  }
}

// XOUT unit (warps 4-7): action row i, outputs [16 ch, 16 ch + 16): final RMSNorm of
// the row, v = action_out_proj (fp32), velocity (x-prediction: v - x_1), x <- x +
// dt v (x_0 on the last step).  Warp w takes outputs 16 ch + w + 4 o.
__device__ __forceinline__ void xout_unit(const LoopArgs &a, Bars &bs, float *yrow, int i, int ch, int k, int et) {
  const int warp = et >> 5, lane = et & 31;
  const int A = a.A;
  float xo[4], x1o[4], bo[4];
#pragma unroll
  for (int o = 0; o < 4; ++o) {
    const int aa = ch * 16 + warp + 4 * o;
    xo[o] = x1o[o] = bo[o] = 0.f;
    if (aa < A) {
      xo[o] = a.xw[(size_t)i * A + aa];
      bo[o] = a.aout_b[aa];
      if (a.x_pred) x1o[o] = a.cp->x1[(size_t)i * A + aa];
    }
  }
  const float4 *src = reinterpret_cast<const float4 *>(a.h + (size_t)(a.B + i) * kWidth) + et * 2;
  const float4 *g4 = reinterpret_cast<const float4 *>(a.fnorm) + et * 2;
  const float4 x0 = src[0], x1 = src[1], g0 = g4[0], g1 = g4[1];
  float ss = x0.x * x0.x + x0.y * x0.y + x0.z * x0.z + x0.w * x0.w + x1.x * x1.x + x1.y * x1.y + x1.z * x1.z +
             x1.w * x1.w;
  ss = warp_sum(ss);
  if (lane == 0) bs.red[warp] = ss;
  epi_bar();
  const float tot = (bs.red[0] + bs.red[1]) + (bs.red[2] + bs.red[3]);
  const float inv = 1.0f / sqrtf(tot / (float)kWidth + kRmsEps);
  float4 *y4 = reinterpret_cast<float4 *>(yrow) + et * 2;
  y4[0] = make_float4((x0.x * inv) * (1.0f + g0.x), (x0.y * inv) * (1.0f + g0.y), (x0.z * inv) * (1.0f + g0.z),
                      (x0.w * inv) * (1.0f + g0.w));
  y4[1] = make_float4((x1.x * inv) * (1.0f + g1.x), (x1.y * inv) * (1.0f + g1.y), (x1.z * inv) * (1.0f + g1.z),
                      (x1.w * inv) * (1.0f + g1.w));
  epi_bar();
  float dt;
  if (a.linspace)
    dt = (float)((double)(k + 1) / (double)a.N) - (float)((double)k / (double)a.N);
  else
    dt = (float)(-1.0 / (double)a.N);
  const float4 *yr = reinterpret_cast<const float4 *>(yrow);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int c4 = lane; c4 < kWidth / 4; c4 += 32) {
    const float4 yv = yr[c4];
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const int aa = ch * 16 + warp + 4 * o;
      if (aa < A) {
        const float4 wv = reinterpret_cast<const float4 *>(a.aout_w + (size_t)aa * kWidth)[c4];
        acc[o] = fmaf(wv.x, yv.x, acc[o]);
        acc[o] = fmaf(wv.y, yv.y, acc[o]);
        acc[o] = fmaf(wv.z, yv.z, acc[o]);
        acc[o] = fmaf(wv.w, yv.w, acc[o]);
      }
    }
  }
#pragma unroll
  for (int o = 0; o < 4; ++o) acc[o] = warp_sum(acc[o]);
  if (lane == 0) {
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const int aa = ch * 16 + warp + 4 * o;
      if (aa < A) {
        float v = acc[o] + bo[o];
        if (a.x_pred) v -= x1o[o];  // output is the clean action: velocity = x_hat - noise
        const float xn = __fadd_rn(xo[o], __fmul_rn(dt, v));
        a.xw[(size_t)i * A + aa] = xn;
        if (k == a.N - 1) a.cp->x0[(size_t)i * A + aa] = xn;
      }
    }
  }
  epi_bar();  // yrow and red are reused by the next unit
}

// ---- role: epilogues, softmax and row stages (warps 4-7) -------------------------------
__device__ void role_epi(const LoopArgs &a, uint8_t *smem, Bars &bs, uint32_t tmem, int et) {
  const int total = total_stages(a);
  const int warp = et >> 5, lane = et & 31;
  const uint32_t t_lane = (uint32_t)(warp * 32) << 16;
  uint32_t acc_n = 0, sj = 0, pj = 0, pvj = 0, tmem_units = 0, red_n = 0, wi = 0, ai = 0;
  const uint32_t sbase = smem_u32(smem);
  const int nas = a_slots(a);
  const uint32_t asb = a_slot_bytes(a);
  bool ok = true;
  float *yrow = reinterpret_cast<float *>(smem + kOffX);         // XOUT's normalised row
  float *scratch = reinterpret_cast<float *>(smem + kOffScratch);  // GEMM reduce
  auto open = [&](int gs) -> bool {
    const bool good = gate(bs, gs, a);
    LOOP_STAMP(gs, 0);
    return good;
  };
  for (int gs = 0; gs < total && ok; ++gs) {
    const StageInfo si = stage_at(a, gs);
    const int step0 = si.step == 0;
    if (loop_is_gemm(si.kind)) {
      const LoopGemm p = loop_gemm_plan(si.kind, a.grid);
      const int U = p.mtiles * p.ksplit;
      if (blockIdx.x >= U) continue;
      ok = open(gs);
      if (!ok) break;
      int r_lo, r_hi, out_off;
      gemm_rows(a, si.kind, step0, r_lo, r_hi, out_off);
      const int NT = a.box_rows;
      // U <= grid (at most 64 m-tiles, at least 128 CTAs): every unit of an m-tile
      // runs on its own CTA, so waiting for the m-tile's partials cannot wait on itself
      // D[128 weight rows, NT tokens] += W[128, 16] X[NT, 16]^T: A is the weight K-block,
      // B the activation K-block, both K-major with the 128-byte swizzle
      const uint32_t idesc = idesc_bf16_f32(128, NT);
      const int nch = NT * 4 <= 256 ? 4 : 256 / NT;  // accumulator chains in TMEM 256..511
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const GUnit g = gemm_unit(p, u);
        const int nk = g.kb1 - g.kb0;
        // MMA issue from the four warps (a tcgen05.mma costs its issuing warp a fixed
        // time): warp w takes K-blocks w, w + nch, .. of the unit into chain w, then every
        // warp commits acc_full (four arrivals) and the readout adds the chains in order.
        // The previous unit's TMEM reads finished before the barrier that ended it.
        tc_fence_after();
        bool good = true;
        for (int i = warp; i < nk && warp < nch && good; i += nch) {
          const uint32_t wk = wi + (uint32_t)i, ak = ai + (uint32_t)i;
          const int ws = wk % kWSlots, as = ak % nas;
          good = __all_sync(kFull, lwait(&bs.w_full[ws], (wk / kWSlots) & 1u, a, kErrTimeoutEpilogue)) &&
                 __all_sync(kFull, lwait(&bs.a_full[as], (ak / nas) & 1u, a, kErrTimeoutEpilogue));
          if (!good) break;
          tc_fence_after();
          const uint32_t wb = sbase + kOffW + ws * kWSlotBytes, ab = sbase + kOffA + as * asb;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16_w(tmem + kTmemAcc + (uint32_t)(warp * NT), smem_desc_k_sw128(wb, kk * 32),
                          smem_desc_k_sw128(ab, kk * 32), idesc, (i >= nch || kk > 0) ? 1u : 0u);
          tc_commit_w(&bs.a_empty[as]);
          tc_commit_w(&bs.w_empty[ws]);
        }
        wi += (uint32_t)nk;
        ai += (uint32_t)nk;
        tc_commit_w(&bs.acc_full);
        if (!good && lane == 0) atomicOr(&bs.epi_err, 1u);
        good = __all_sync(kFull, lwait(&bs.acc_full, acc_n & 1u, a, kErrTimeoutEpilogue));
        if (!good && lane == 0) atomicOr(&bs.epi_err, 1u);
        epi_bar();
        if (*(volatile uint32_t *)&bs.epi_err) {  // the same decision in all four warps
          ok = false;
          break;
        }
        ++acc_n;
        tc_fence_after();
        LOOP_STAMP(gs, 1);
        const int used = nk < nch ? nk : nch;
        // partial tile, token-major: row et of the m-tile for the stored tokens (the sum
        // of the unit's chains, in chain order)
        float *mine = a.gpart + (size_t)u * 128 * NT;
        for (int c0 = r_lo & ~15; c0 < r_hi; c0 += 16) {
          // the group's columns of every chain, loaded together under one wait
          uint32_t r[64];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < used) {
              tmem_ld_x16_nw(tmem + t_lane + kTmemAcc + (uint32_t)(c * NT + c0), r + 16 * c);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) r[16 * c + i] = 0u;
            }
          }
          tc_wait_ld_regs64(r);
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
#pragma unroll
          for (int c = 1; c < 4; ++c)
            if (c < used) {
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] += __uint_as_float(r[16 * c + i]);
            }
#pragma unroll
          for (int i = 0; i < 16; ++i) __stcg(mine + (size_t)(c0 + i) * 128 + et, v[i]);
        }
        tc_fence_before();
        epi_bar();
        LOOP_STAMP(gs, 8);
        ++tmem_units;
        int *cnt = a.mt_cnt + (size_t)gs * kLoopMaxMtiles + g.m;
        if (et == 0) {
          smem_publish(&bs.tmem_done, tmem_units);
          red_release_add(cnt, 1);
        }
        int t0, t1;
        red_slice(r_lo, r_hi, p.ksplit, g.s, t0, t1);
        if (t0 < t1) {
          // per-token rstd / RoPE position of the slice while the other splits finish
          float *rstd_s = scratch;
          int *pos_s = reinterpret_cast<int *>(scratch + kLoopMaxRows);
          if (si.kind == LK_QKV || si.kind == LK_GU) {
            const float *ssn = si.kind == LK_QKV ? a.ss_a : a.ss_m;
            for (int j = et; j < t1 - t0; j += 128) {
              const int orow = t0 + j + out_off;
              rstd_s[j] = row_rstd(ssn, a.ss_ld, orow);
              pos_s[j] = si.kind == LK_QKV ? rope_pos(a, orow) : 0;
            }
          }
          // once every split's partial is stored, every thread copies 16-byte chunks of
          // the slice of each split into region X (free: this unit's MMAs have
          // completed, and region X is handed on only after the reduce)
          if (et == 0) bs.last = gwait(cnt, p.ksplit, a, kErrTimeoutEpilogue) ? 1 : 0;
          epi_bar();
          ok = bs.last != 0;
          if (!ok) break;
          {
            // one bulk copy per split's slice (contiguous in the token-major partial tile),
            // split sp issued by lane sp / 4 of warp sp % 4: each copy costs its issuing
            // thread a fixed time, so the issues run in four warps at once
            const uint32_t slice_bytes = (uint32_t)(t1 - t0) * 512u;
            if (et == 0) {
              mbar_arrive_expect_tx(&bs.red_full, slice_bytes * (uint32_t)p.ksplit);
              bs.red_fills = red_n + 1;
            }
            const int sp = lane * 4 + warp;
            if (sp < p.ksplit) {
              fence_proxy_async_global();  // the partials were stored through the generic proxy
              bulk_load(smem_u32(smem + kOffX + (uint32_t)sp * slice_bytes),
                        a.gpart + ((size_t)(g.m * p.ksplit + sp) * NT + t0) * 128, slice_bytes, &bs.red_full);
            }
          }
          LOOP_STAMP(gs, 7);
          reduce_unit(a, si, p, g, t0, t1, out_off, et, reinterpret_cast<const float4 *>(smem + kOffX), rstd_s, pos_s,
                      &bs.red_full, red_n & 1u, gs);
          ++red_n;
          LOOP_STAMP(gs, 10);
          fence_proxy_async_global();  // outputs are read by bulk copies in the next stage
        }
        epi_bar();
        LOOP_STAMP(gs, 11);
        if (et == 0) {
          x_release(bs);  // region X: the unit's MMAs and its reduce are done
          LOOP_STAMP(gs, 2);
          release(a, gs);
        }
      }
    } else if (si.kind == LK_ATTN) {
      const int U = attn_units(a, step0);
      if (blockIdx.x >= U) continue;
      ok = open(gs);  // q of this step's QKV stage
      if (!ok) break;
      const int Tq = step0 ? a.H + 1 : a.H;
      const int nrows = kHeads * Tq;
      const float scale_l2 = 0.0625f * kLog2e;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        // the unit's query tile from u alone: its Q loads go out before the key range,
        // which waits on the sample's valid prefix length
        const int qps = q_tiles(a, step0), qt = u / a.attn_splits, qb = qt / qps;
        const int qi = (qt % qps) * 128 + et;
        const bool row_ok = qi < nrows;
        const int jq = qi / kHeads, head = qi % kHeads;
        int tok = 0;
        if (row_ok) tok = step0 ? (jq == 0 ? qb : a.B + qb * a.H + jq - 1) : a.B + qb * a.H + jq;
        // q of query tile qt is stored as [8-dim chunk][128 rows] (reduce_unit): chunk e of
        // this thread's row, for consecutive rows of a warp, is 512 contiguous bytes
        uint4 qq[32];
        {
          const uint4 *src = reinterpret_cast<const uint4 *>(a.q) + (size_t)qt * (kHeadDim / 8) * 128 + et;
#pragma unroll
          for (int e = 0; e < 32; ++e) qq[e] = row_ok ? __ldcg(src + (size_t)e * 128) : make_uint4(0, 0, 0, 0);
        }
        const AUnit t = attn_unit(a, u, step0);
        const bool state_q = step0 && jq == 0;
        const int ja = step0 ? jq - 1 : jq;
        const int sfx_base = t.nbp * kKB;
        const int sfx_lo = sfx_base + (state_q ? a.H : 0);
        const int sfx_hi = state_q ? sfx_base + a.H + 1 : (a.causal ? sfx_base + ja + 1 : sfx_base + a.H + 1);
        const int sfx_state = sfx_base + a.H;
        float m_used = -INFINITY, l = 0.f;
        if (t.nb > 0) {
          // Q row -> TMEM lane et, columns kTmemQ.. (two bf16 per 32-bit column)
          {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              float v[32];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                v[4 * e] = __uint_as_float(qq[cc * 8 + e].x);
                v[4 * e + 1] = __uint_as_float(qq[cc * 8 + e].y);
                v[4 * e + 2] = __uint_as_float(qq[cc * 8 + e].z);
                v[4 * e + 3] = __uint_as_float(qq[cc * 8 + e].w);
              }
              tmem_st_32x32b_x32(tmem + t_lane + kTmemQ + 32 * cc, v);
            }
          }
          tc_fence_before();
          mbar_arrive(&bs.q_full);
          LOOP_STAMP(gs, 1);
          const uint32_t pv0 = pvj;  // global index of this unit's first P.V
          for (int j = 0; j < t.nb && ok; ++j, ++sj, ++pj) {
            const int sb = sj & 1, pb = pj & 1;
            ok = __all_sync(kFull, lwait(&bs.s_full[sb], (sj >> 1) & 1u, a, kErrTimeoutEpilogue));
            if (!ok) break;
            tc_fence_after();
            if (j == 0) LOOP_STAMP(gs, 3);
            float sv[32];
            {
              float s2[32];
              tmem_ld_32x32b_x32(tmem + t_lane + kTmemS + sb * 2 * kKB, sv);
              tmem_ld_32x32b_x32(tmem + t_lane + kTmemS + sb * 2 * kKB + kKB, s2);
#pragma unroll
              for (int i = 0; i < 32; ++i) sv[i] += s2[i];
            }
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
                ok = __all_sync(kFull, lwait(&bs.pv_done[g % kKVBufs], (g / kKVBufs) & 1u, a, kErrTimeoutEpilogue));
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
              ok = __all_sync(kFull, lwait(&bs.pv_done[g % kKVBufs], (g / kKVBufs) & 1u, a, kErrTimeoutEpilogue));
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
            ok = __all_sync(kFull, lwait(&bs.pv_done[g % kKVBufs], (g / kKVBufs) & 1u, a, kErrTimeoutEpilogue));
          }
          pvj = pv0 + t.nb;
          tc_fence_after();
        }
        if (et == 0) x_release(bs);  // every MMA of the unit has completed
        if (!ok) break;
        LOOP_STAMP(gs, 7);
        const float inv_l = l > 0.f ? 1.0f / l : 0.f;
        if (a.attn_splits == 1) {
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
#pragma unroll
              for (int e = 0; e < 4; ++e)
                store_reps(a.att, tiled_off(tok, head * kHeadDim + c0 + 8 * e, a.box_rows),
                           (size_t)a.rep_rows * kQDim, pack8(w32 + 8 * e));
            }
          }
        } else {
          // partial O of unit u = (b * qps + ti) * splits + split, normalised by its own l
          // and rounded to bf16 (as the attention output it becomes is), as [u][8-dim
          // chunk][row]: the 32 rows of a warp store 512 contiguous bytes per chunk, and
          // the unit's release waits for half the bytes an fp32 partial would take
          uint4 *pbase = reinterpret_cast<uint4 *>(a.part_o) + (size_t)u * (kHeadDim / 8) * 128 + et;
          for (int c0 = 0; c0 < kHeadDim; c0 += 64) {
            float v[64];
            if (t.nb > 0) {
              tmem_ld_32x32b_x64(tmem + t_lane + kTmemO + c0, v);
            } else {
#pragma unroll
              for (int e = 0; e < 64; ++e) v[e] = 0.f;
            }
            if (row_ok) {
#pragma unroll
              for (int e = 0; e < 64; ++e) v[e] *= inv_l;
#pragma unroll
              for (int e = 0; e < 8; ++e) __stcg(pbase + (size_t)(c0 / 8 + e) * 128, pack8(v + 8 * e));
            }
          }
          if (row_ok) {
            const size_t prow = (size_t)u * 128 + et;
            a.part_ml[2 * prow] = m_used;
            a.part_ml[2 * prow + 1] = l;
          }
        }
        tc_fence_before();
        fence_proxy_async_global();
        epi_bar();
        ++tmem_units;
        if (et == 0) {
          smem_publish(&bs.tmem_done, tmem_units);  // O has been read out
          LOOP_STAMP(gs, 2);
          release(a, gs);
        }
      }
    } else if (si.kind == LK_COMBINE) {
      const int nc = combine_ctas(a, step0);
      if (blockIdx.x >= nc) continue;
      ok = open(gs);
      if (!ok) break;
      const int Tq = step0 ? a.H + 1 : a.H;
      const int nrows = kHeads * Tq, qps = q_tiles(a, step0), S = a.attn_splits;
      // warp item (query tile qt, 32-row group, 8 dims): lane = row, so every load of a
      // split's (m, l) and 4-dim chunk is 32 consecutive rows.  All (m, l) load at once,
      // then all chunks (at most kLoopMaxSplits splits).
      for (int it = blockIdx.x * 4 + warp; it < combine_items(a, step0); it += nc * 4) {
        const int qt = it / 128, rg = (it / 32) & 3, dg = it & 31;
        const int b = qt / qps, qi = (qt % qps) * 128 + rg * 32 + lane;
        if (qi >= nrows) continue;
        const size_t prow0 = (size_t)qt * S * 128 + rg * 32 + lane;  // split s at + s * 128
        float ms[kLoopMaxSplits], ls[kLoopMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kLoopMaxSplits; ++sp) {
          ms[sp] = ls[sp] = 0.f;
          if (sp < S) {
            const float2 ml = __ldcg(reinterpret_cast<const float2 *>(a.part_ml) + prow0 + (size_t)sp * 128);
            ms[sp] = ml.x;
            ls[sp] = ml.y;
          }
        }
        // unit (qt, sp) holds 8-dim chunk k of its row r (bf16) at part_o uint4
        // (unit * 32 + k) * 128 + r
        const uint4 *src = reinterpret_cast<const uint4 *>(a.part_o) + ((size_t)qt * S * (kHeadDim / 8) + dg) * 128 +
                           rg * 32 + lane;
        uint4 x[kLoopMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kLoopMaxSplits; ++sp)  // (every unit stores its rows)
          x[sp] = sp < S ? __ldcg(src + (size_t)sp * (kHeadDim / 8) * 128) : make_uint4(0, 0, 0, 0);
        float M = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < kLoopMaxSplits; ++sp)
          if (sp < S && ls[sp] > 0.f) M = fmaxf(M, ms[sp]);
        float den = 0.f;
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int sp = 0; sp < kLoopMaxSplits; ++sp) {
          if (!(sp < S && ls[sp] > 0.f)) continue;
          const float wgt = ls[sp] * ex2_approx(ms[sp] - M);
          den += wgt;
          const uint32_t w4[4] = {x[sp].x, x[sp].y, x[sp].z, x[sp].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[e]));
            o[2 * e] = fmaf(wgt, f.x, o[2 * e]);
            o[2 * e + 1] = fmaf(wgt, f.y, o[2 * e + 1]);
          }
        }
        const int j = qi / kHeads, hd = qi % kHeads;
        const int tok = step0 ? (j == 0 ? b : a.B + b * a.H + j - 1) : a.B + b * a.H + j;
        const float inv = den > 0.f ? 1.0f / den : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] *= inv;
        store_reps(a.att, tiled_off(tok, hd * kHeadDim + dg * 8, a.box_rows), (size_t)a.rep_rows * kQDim, pack8(o));
      }
      fence_proxy_async_global();
      epi_bar();
      if (et == 0) {
        LOOP_STAMP(gs, 2);
        release(a, gs);
      }
    } else if (si.kind == LK_TIN) {
      const int nc = tin_ctas(a);
      if (blockIdx.x >= nc) continue;
      ok = open(gs);
      if (!ok) break;
      for (int cidx = blockIdx.x; cidx < kWidth / 8; cidx += nc) tin_unit(a, cidx, si.step, et);
      fence_proxy_async_global();  // u is read by TMA in the next stage
      epi_bar();
      if (et == 0) {
        LOOP_STAMP(gs, 2);
        release(a, gs);
      }
    } else {  // LK_XOUT
      const int nc = xout_ctas(a);
      if (blockIdx.x >= nc) continue;
      ok = open(gs);
      if (!ok) break;
      const int nch = (a.A + 15) / 16;
      for (int u = blockIdx.x; u < xout_units(a); u += nc) xout_unit(a, bs, yrow, u / nch, u % nch, si.step, et);
      fence_proxy_async_smem();  // region X is next filled by bulk / tensor copies
      epi_bar();
      if (et == 0) {
        LOOP_STAMP(gs, 2);
        release(a, gs);
      }
    }
  }
  // every GEMM MMA this warp issued has completed before the CTA may free TMEM or exit
  tc_commit_w(&bs.epi_fin);
  dwait(&bs.epi_fin, 0, a);
  __syncwarp();
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
    for (int i = 0; i < kMaxASlots; ++i) {
      mbar_init(&bs.a_full[i], 1);
      mbar_init(&bs.a_empty[i], 1);
      bs.a_fills[i] = 0;
    }
    mbar_init(&bs.acc_full, 4);  // one tcgen05.commit per epilogue warp
    bs.tmem_done = 0;
    for (int i = 0; i < kKVBufs; ++i) {
      mbar_init(&bs.k_full[i], 32);  // one cp.async-completion arrival per loader lane (+ TMA bytes)
      mbar_init(&bs.k_empty[i], 1);
      mbar_init(&bs.v_full[i], 32);
      mbar_init(&bs.pv_done[i], 1);
      bs.k_fills[i] = bs.v_fills[i] = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bs.s_full[i], 1);
      mbar_init(&bs.s_empty[i], 128);
      mbar_init(&bs.p_full[i], 128);
    }
    mbar_init(&bs.q_full, 128);
    mbar_init(&bs.mma_fin, 1);
    mbar_init(&bs.red_full, 1);
    mbar_init(&bs.epi_fin, 4);
    bs.red_fills = 0;
    bs.epi_err = 0;
    bs.x_done = 0;
    bs.ready = 0;
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
      if (lane < 2) role_weights(a, smem, bs, lane);
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
      for (int i = 0; i < kMaxASlots; ++i)
        if (bs.a_fills[i]) dwait(&bs.a_full[i], (bs.a_fills[i] - 1) & 1u, a);
      for (int i = 0; i < kKVBufs; ++i)
        if (bs.k_fills[i]) dwait(&bs.k_full[i], (bs.k_fills[i] - 1) & 1u, a);
    }
    if (warp == 3)
      for (int i = 0; i < kKVBufs; ++i)
        if (bs.v_fills[i]) dwait(&bs.v_full[i], (bs.v_fills[i] - 1) & 1u, a);
    if (warp == 4 && bs.red_fills) dwait(&bs.red_full, (bs.red_fills - 1) & 1u, a);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// Split-KV plan: each 128-row query tile's key blocks are cut into `splits` ranges of
// `bps` blocks, one unit each, as many as the grid holds but at least
// kAttnMinBlocks blocks per unit (below that, writing and merging the fp32 partials
// costs more than the keys it saves).  One split means no COMBINE stage.
constexpr int kAttnMinBlocks = 4;
void loop_attn_plan(int B, int H, int P, int grid, int &splits, int &bps) {
  const int qps = (kHeads * (H + 1) + 127) / 128;
  const int nblk = (P + kKB - 1) / kKB + (H + kKB) / kKB;
  const int qt = B * qps;
  int s = grid / (qt > 0 ? qt : 1);
  const int max_s = (nblk + kAttnMinBlocks - 1) / kAttnMinBlocks;
  if (s > max_s) s = max_s;
  if (s > kLoopMaxSplits) s = kLoopMaxSplits;
  if (s < 1) s = 1;
  bps = (nblk + s - 1) / s;
  splits = (nblk + bps - 1) / bps;
}

size_t loop_smem_bytes() { return kSmemTotal; }

int loop_max_grid(int dev, const char **why) {
  int sms = 0, coop = 0, per_sm = 0;
  *why = nullptr;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) {
    cudaGetLastError();
    *why = "the device does not support cooperative launches";
    return 0;
  }
  if (cudaFuncSetAttribute(k_loop, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTotal) != cudaSuccess) {
    cudaGetLastError();
    *why = "the loop kernel's shared memory cannot be configured";
    return 0;
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_loop, kThreads, kSmemTotal) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    *why = "one loop CTA does not fit an SM (registers or shared memory)";
    return 0;
  }
  return sms;
}

// The GEMM reduce stages a unit's slice of every split in region X: the largest
// slice (an even token count) times the splits must fit, and every m-tile's units must
// fit the grid (each unit waits for the others of its m-tile).
static bool loop_plan_fits(const LoopArgs &a) {
  const int kinds[5] = {LK_TOUT, LK_QKV, LK_O, LK_GU, LK_DOWN};
  for (int k : kinds) {
    const LoopGemm p = loop_gemm_plan(k, a.grid);
    if (p.mtiles > kLoopMaxMtiles || p.mtiles * p.ksplit > a.grid) return false;
    const int rows = a.R;  // the widest stored range
    const int per = ((rows + p.ksplit - 1) / p.ksplit + 1) & ~1;
    if ((size_t)per * p.ksplit * 512 > kXBytes) return false;
  }
  return a.box_rows % 16 == 0 && a.box_rows >= 16 && a.box_rows <= kLoopMaxRows;
}

cudaError_t launch_loop(const LoopArgs &a, cudaStream_t s) {
  if (!loop_plan_fits(a)) return cudaErrorInvalidValue;
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

#ifdef PI0X_LOOP_TIMELINE
// Profiling build only: device buffer of (stages x CTAs x 8) globaltimer stamps.
extern "C" int pi0x_loop_timeline_set(void *p) { return (int)cudaMemcpyToSymbol(g_loop_tl, &p, sizeof(p)); }
#endif

}  // namespace pi0x
