// Internal launch interface of the pi0x kernels (host side).  Not part of the ABI.
//
// Row layout of every per-token activation buffer for a batch of B samples with
// horizon H (R = B + B*H rows): rows [0, B) hold the state token of sample b,
// rows B + b*H + (j-1) hold action token j = 1..H of sample b.  The state rows
// come first so that steps after the first one, which reuse the state token's
// hidden states and K/V (they depend on neither x_t nor t), run on the
// contiguous row range [B, R).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pi0x {

typedef __nv_bfloat16 bf16;

// Pointers a call hands in; kept in device memory so that a captured CUDA graph
// stays valid when the caller's buffers change between calls.
constexpr int kMaxDepth = 32;
struct CallPtrs {
  // bf16 mode: TMA maps of the attention keys and values, [0] = K, [1] = V.
  // kv_map[.][l]: layer l's prefix tensor as B*P rows of 256 (encoded per call);
  // sfx_map[.]: the suffix K/V of all layers as one tensor of rows x 256.
  // 128-byte swizzle; boxes of 64 columns x 8 rows, or x 64 rows for the *64 maps.
  CUtensorMap kv_map[2][kMaxDepth];
  CUtensorMap kv_map64[2][kMaxDepth];
  CUtensorMap sfx_map[2];
  CUtensorMap sfx_map64[2];
  // 32-row boxes of the same tensors (the persistent small-batch loop's 32-key blocks)
  CUtensorMap kv_map32[2][kMaxDepth];
  CUtensorMap sfx_map32[2];

  const bf16 *prefix_k[kMaxDepth];
  const bf16 *prefix_v[kMaxDepth];
  const uint8_t *mask;
  const float *state;
  const float *x1;
  float *x0;
};

// GEMM epilogues: D[m][n] = sum_k A[m][k] * Bw[n][k]
enum Epi : int {
  EPI_STORE_F32 = 0,   // out_f32[m][n] = D
  EPI_BIAS_F32 = 1,    // out_f32[m][n] = D + vec[n]
  EPI_VEC_SILU = 2,    // out_T[m][n] = silu(D + vec[n])
  EPI_RESID_F32 = 3,   // out_f32[m][n] += D
  EPI_QKV_ROPE = 4,    // tcgen05 only: RoPE'd q, k and v from the permuted QKV columns
  EPI_GEGLU = 5,       // tcgen05 only: gelu_tanh(gate) * up from the interleaved columns
};

// Arguments of the tcgen05 GEMM epilogues (rows of the output are out_row0 + m).
struct EpiArgs {
  float *out_f32 = nullptr;
  bf16 *out_bf16 = nullptr;
  int ldo = 0, out_row0 = 0;
  const float *vec = nullptr;
  // EPI_QKV_ROPE: destinations, per-sample valid-prefix counts, RoPE frequencies
  bf16 *q = nullptr, *ks = nullptr, *vs = nullptr;
  const int *nvalid = nullptr;
  const float *inv_freq = nullptr;
  int B = 0, H = 0;
  // split-K partial tiles and per-tile arrival counters (zero between GEMMs)
  float *part = nullptr;
  int *counters = nullptr;
  // Fused RMSNorm (bf16 mode).  Producers (EPI_BIAS_F32 / EPI_RESID_F32 with
  // gain != null) also write xn_out = bf16(h * (1 + gain)) and, per output column
  // tile t, ss_out[t * ss_ld + row] = sum of h^2 over the tile's columns (slots
  // t >= N/BN are zeroed).  Consumers (EPI_QKV_ROPE / EPI_GEGLU with ss_in) scale
  // the accumulator by 1/sqrt(sum_{t<kNormSlots} ss_in[t*ss_ld+row] / 1024 + eps).
  const float *gain = nullptr;
  bf16 *xn_out = nullptr;
  float *ss_out = nullptr;
  const float *ss_in = nullptr;
  int ss_ld = 0;
  // EPI_QKV_ROPE: (cos, sin) pairs of fp32(pos) * inv_freq[i], [pos][128] (k_rope_table)
  const float *rope_tab = nullptr;
};
constexpr int kNormSlots = 16;

// Tile width and K split of one tcgen05 GEMM launch.
struct TcPlan {
  int bn = 128;
  int splits = 1;
  int a_rows = 128;  // rows of the activation TMA box (64 when the GEMM has <= 64 rows)
};

// Activation operand: tensor maps with 128-row and 64-row boxes.
struct ActMap {
  CUtensorMap m128, m64;
  const CUtensorMap &get(int rows) const { return rows == 64 ? m64 : m128; }
};

struct GemmOut {
  void *out;      // fp32 or activation type, row-major
  int ldo;        // elements
  int out_row0;   // output row of GEMM row 0
  const float *vec;
};

// Batch geometry of one call.
struct Geo {
  int B, H, A, S, P, R;   // R = B + B*H
};

// Launch `kern` with programmatic stream serialization (it may overlap the previous
// kernel on the stream until it calls pdl_wait()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
#ifdef PI0X_NO_PDL
  cfg.numAttrs = 0;  // build option: plain stream-ordered launches
#else
  cfg.numAttrs = 1;
#endif
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- misc kernels (k_misc.cu) ----
void launch_prep_mask(const CallPtrs *cp, int B, int P, int *nvalid, int *vidx, cudaStream_t s);
template <typename TW>
void launch_time_vec(const TW *w_time, const float *bias, int num_steps, int linspace, float *tvec, cudaStream_t s);
template <typename TW>
void launch_state_embed(const CallPtrs *cp, const TW *w, const float *b, int B, int S, float *h, cudaStream_t s,
                        const float *gain = nullptr, bf16 *xn = nullptr, float *ss = nullptr, int ss_ld = 0,
                        int nslots = kNormSlots, int tiled_rb = 0, int rep_rows = 0);
// Weight copy in the persistent loop's m-tile layout (see k_tile_weight in k_misc.cu).
cudaError_t launch_tile_weight(const bf16 *src, int N, int K, bf16 *dst, cudaStream_t s);
template <typename TW, typename T>
void launch_action_in(const float *x, const TW *w, const float *b, int rows, int A, T *out, cudaStream_t s);
template <typename T>
void launch_rmsnorm(const float *h, int row0, int rows, const float *gain, T *out, cudaStream_t s);
template <typename T>
void launch_rope_qkv(const float *raw, int row0, int rows, const Geo &g, const int *nvalid, const float *inv_freq,
                     T *q, T *ks, T *vs, cudaStream_t s);
template <typename T>
void launch_geglu(const float *raw, int row0, int rows, T *act, cudaStream_t s);
// x_pred: the out-projection is the clean action; velocity = it - cp->x1.
void launch_final_euler(const float *h, const Geo &g, const float *gain, const float *w_out, const float *b_out,
                        float dt, float *x, const CallPtrs *cp, int last, int x_pred, cudaStream_t s);
void launch_copy_x1(const CallPtrs *cp, int n, float *x, cudaStream_t s);
void launch_delay_ns(unsigned long long ns, cudaStream_t s);
void launch_rope_table(const float *inv_freq, int npos, float *tab, cudaStream_t s);

// ---- attention (k_attn.cu) ----
template <typename T>
void launch_attention(const T *q, const T *ks, const T *vs, const CallPtrs *cp, int layer, const int *nvalid,
                      const int *vidx, const Geo &g, int step0, int causal, T *out, cudaStream_t s);

// tcgen05 attention (k_attn_tc.cu); `part` holds attn_tc_partial_floats() floats
// when splits > 1.
// Key slots per sample: ceil(P/64) blocks of valid prefix keys, then ceil((H+1)/64)
// blocks holding the H action keys and the state key.
int attn_tc_blocks(int P, int H);
int attn_tc_splits(const Geo &g, int step0);
size_t attn_tc_partial_floats(const Geo &g, int step0, int splits);
// Encodes cp.kv_map for layers [0, layers) (prefix tensors cp.prefix_k/v[l], B*P rows)
// and cp.sfx_map over `sfx_rows` rows at ks / vs.  False if an encode fails (e.g. a
// pointer that is not 16-byte aligned).
bool attn_tc_maps(CallPtrs &cp, int layers, int B, int P, const void *ks, const void *vs, uint64_t sfx_rows);
// The 32-row-box maps (kv_map32, sfx_map32) of the same tensors.
bool loop_attn_maps(CallPtrs &cp, int layers, int B, int P, const void *ks, const void *vs, uint64_t sfx_rows);
// ks / vs: this layer's suffix rows, which start at row `sfx_row0` of cp->sfx_map.
// causal: the causal action mask (action query i sees actions 0..i and the state).
void launch_attention_tc(const bf16 *q, const bf16 *ks, const bf16 *vs, const CallPtrs *cp, int layer,
                         int sfx_row0, const int *nvalid, const int *vidx, const Geo &g, int step0, int causal,
                         int splits, bf16 *out, float *part, unsigned *err, cudaStream_t s);
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch, uint32_t box_rows);

// Text for pi0x_last_error() (this thread).
void set_last_error(const char *msg);

// ---- GEMMs ----
template <typename OutT>
void launch_gemm_simt(const float *A, int lda, const float *Bw, int ldb, int M, int N, int K, int epi,
                      const GemmOut &o, cudaStream_t s);

// Weight operand of a tcgen05 GEMM: tensor maps with 64-row and wide boxes.
struct TcWeight {
  CUtensorMap tm64, tm_wide;
  int N = 0, K = 0, bn_wide = 128;
  const CUtensorMap &map(int bn) const { return bn == 64 ? tm64 : tm_wide; }
};
// Tile plan for M rows: wide tiles for large M, 64-wide tiles with split-K below.
TcPlan plan_gemm_tc(int M, int N, int K);
size_t gemm_tc_partial_floats(int M, int N, const TcPlan &p);
void launch_gemm_tc(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const TcPlan &p, int a_row0, int M,
                    int N, int K, const EpiArgs &e, unsigned *err, cudaStream_t s);

// ---- persistent small-batch loop (k_loop.cu) -----------------------------------
// One cooperative launch runs every Euler step of a call when every step's rows fit
// one 128-row MMA tile (B * (H + 1) <= 128): one CTA per SM, the call's stages in
// program order, each stage waiting on the done-counter of the one before it.
//
// Program of one Euler step: TIN (action-time MLP input of the step), TOUT (MLP
// output -> residual stream, layer-0 norm inputs), per layer QKV, ATTN, [COMBINE
// when attention is split over key ranges], O, GU, DOWN, and last XOUT (final norm,
// out-projection, x += dt v).
enum LoopKind : int {
  LK_TIN = 0, LK_TOUT = 1, LK_QKV = 2, LK_ATTN = 3, LK_COMBINE = 4, LK_O = 5, LK_GU = 6, LK_DOWN = 7, LK_XOUT = 8
};
constexpr int kLoopMaxRows = 128;
constexpr int kLoopNormSlots = 8;    // fused-norm partial sums: one slot per 128-feature m-tile
constexpr int kLoopKeyBlock = 32;    // attention key block of the loop kernel
constexpr int kLoopMinGrid = 128;    // enough CTAs to split every GEMM's K over most SMs
constexpr int kLoopReps = 1;         // replicas of each tiled activation operand
constexpr int kLoopMaxMtiles = 64;   // m-tiles of the widest GEMM (gate/up: 8192 / 128)
constexpr int kLoopMaxSplits = 8;    // key-range splits of a query tile (the COMBINE registers)

__host__ __device__ inline int loop_layer_stages(int attn_splits) { return attn_splits > 1 ? 6 : 5; }
__host__ __device__ inline int loop_stages_per_step(int L, int attn_splits) {
  return 2 + L * loop_layer_stages(attn_splits) + 1;
}
__host__ __device__ inline int loop_total_stages(int N, int L, int attn_splits) {
  return N * loop_stages_per_step(L, attn_splits);
}
// Kind, layer and Euler step of stage gs of the call.
__host__ __device__ inline void loop_stage(int gs, int L, int attn_splits, int &kind, int &layer, int &step) {
  const int spp = loop_stages_per_step(L, attn_splits);
  step = gs / spp;
  const int i = gs % spp;
  layer = 0;
  if (i < 2) {
    kind = i == 0 ? LK_TIN : LK_TOUT;
    return;
  }
  if (i == spp - 1) {
    kind = LK_XOUT;
    layer = L - 1;
    return;
  }
  const int ls = loop_layer_stages(attn_splits);
  layer = (i - 2) / ls;
  int sub = (i - 2) % ls;
  if (ls == 5 && sub >= 2) ++sub;  // no COMBINE stage
  switch (sub) {
    case 0: kind = LK_QKV; break;
    case 1: kind = LK_ATTN; break;
    case 2: kind = LK_COMBINE; break;
    case 3: kind = LK_O; break;
    case 4: kind = LK_GU; break;
    default: kind = LK_DOWN; break;
  }
}

// GEMM stage plan.  The weight is the MMA's M operand: 128 of its rows (output
// features) form an m-tile, and the call's rows (tokens, a multiple of 16 <= 128) are
// the N operand.  Each m-tile's K range is split over `ksplit` CTAs (as many as the
// grid allows, at most one per 64-wide K-block), unit u = m * ksplit + s.  The units
// of an m-tile then add their fp32 partial tiles in split order, each unit a slice of
// the tokens.
struct LoopGemm {
  int N, K, mtiles, ksplit;
};
__host__ __device__ inline LoopGemm loop_gemm_plan(int kind, int grid) {
  LoopGemm p{1024, 1024, 1, 1};
  switch (kind) {
    case LK_QKV: p.N = kQkvDim; break;
    case LK_O: p.K = kQDim; break;
    case LK_GU: p.N = 2 * kMlp; break;
    case LK_DOWN: p.K = kMlp; break;
    default: break;
  }
  p.mtiles = p.N / 128;
  const int nk = p.K / 64;
  int s = grid / p.mtiles;
  if (s > nk) s = nk;
  p.ksplit = s < 1 ? 1 : s;
  return p;
}
__host__ __device__ inline bool loop_is_gemm(int kind) {
  return kind == LK_TOUT || kind == LK_QKV || kind == LK_O || kind == LK_GU || kind == LK_DOWN;
}

struct LoopArgs {
  int B, H, A, S, P, R, L, N;
  int linspace, x_pred, causal;
  int grid;
  int attn_splits, attn_bps;   // split-KV: splits per query tile, 32-key blocks per split
  int box_rows;                // rows of an activation K-block tile: the call's rows rounded up to 16,
                               // the N of every GEMM MMA
  int rep_rows;                // replica r of a tiled activation with K columns starts at r * rep_rows * K
  int ss_ld;
  int debug_stall_stage;       // >= 0: that stage waits on a counter nothing raises (tests)
  unsigned long long wait_ns;  // time limit of every wait
  float *h, *ss_a, *ss_m, *gpart, *tvec, *xw, *part_o, *part_ml;
  bf16 *xn, *q, *ks, *vs, *att, *act, *uemb;
  int *counters, *done;
  int *mt_cnt;                 // per (stage, m-tile): units whose partial tile is stored
  const int *nvalid, *vidx;
  const float *rope_tab;
  const CallPtrs *cp;
  unsigned *err;
  // action-time MLP input with action_in folded in: u = silu(w_xa x + tvec[k]), w_xa =
  // W_in[:, :W] W_action_in (fp32, W x A); tvec[k] carries W_in[:, :W] b_action_in
  const float *w_xa;
  const float *tout_b, *aout_w, *aout_b, *fnorm;
  const float *in_norm[kMaxDepth], *post_norm[kMaxDepth];
  // weights as 128-row m-tiles of 64-wide swizzled K-blocks (k_tile_weight)
  const bf16 *w_tout;
  const bf16 *w_qkv[kMaxDepth], *w_o[kMaxDepth], *w_gu[kMaxDepth], *w_down[kMaxDepth];
};

// Split-KV plan of the loop attention (splits per query tile, key blocks per split).
void loop_attn_plan(int B, int H, int P, int grid, int &splits, int &bps);
size_t loop_smem_bytes();
// CTAs of the loop kernel on `dev` (one per SM), or 0 with the reason in *why.
int loop_max_grid(int dev, const char **why);
// Enqueue the loop kernel (cooperative launch) on `s`.
cudaError_t launch_loop(const LoopArgs &a, cudaStream_t s);

}  // namespace pi0x
