// Masked MQA attention of the suffix queries over [valid prefix K/V ; suffix K/V]
// (`_attend` and `_compute_layer_suffix_only` on the vllm-omni pi0 page).
//
// One KV head is shared by the 8 query heads.  Visibility (`denoise_step` +
// `make_att_2d_masks` with suffix AR flags [1, 1, 0, ...]): every suffix query sees
// the valid prefix keys; the state query sees the state key only among the suffix
// keys; action queries see the state and all action keys.  Masked keys are
// skipped: the page adds -2.38e38 to their logits, whose exp is exactly 0 in fp32.
// Softmax in fp32 with scale 1/sqrt(256), online over key chunks.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {

constexpr int kAttnQ = 16;      // queries per block (4 warps x 4)
constexpr int kAttnKeys = 32;   // keys per chunk
constexpr int kAttnSmem = (kAttnKeys * (kHeadDim + 1) + kAttnKeys * kHeadDim + kAttnQ * kHeadDim) * 4;

template <typename T>
__global__ void __launch_bounds__(128) k_attn_simt(const T *q, const T *ks, const T *vs, const CallPtrs *cp,
                                                    int layer, const int *nvalid, const int *vidx, Geo g,
                                                    int step0, int causal, T *out) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float sm[];
  float *Ks = sm;                                  // [32][257]
  float *Vs = Ks + kAttnKeys * (kHeadDim + 1);     // [32][256]
  float *Qs = Vs + kAttnKeys * kHeadDim;           // [16][256]
  const int b = blockIdx.x, head = blockIdx.y;
  const int Tq = step0 ? g.H + 1 : g.H;
  const int qbase = blockIdx.z * kAttnQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto q_row = [&](int jq) -> int {
    if (step0) return jq == 0 ? b : g.B + b * g.H + (jq - 1);
    return g.B + b * g.H + jq;
  };
  for (int e = threadIdx.x; e < kAttnQ * kHeadDim; e += blockDim.x) {
    const int qi = e / kHeadDim, d = e % kHeadDim, jq = qbase + qi;
    float v = 0.f;
    if (jq < Tq) v = to_f32(q[(size_t)q_row(jq) * kQDim + head * kHeadDim + d]);
    Qs[e] = v;
  }
  const int nv = nvalid[b];
  const bf16 *Kp = cp->prefix_k[layer] + (size_t)b * g.P * kHeadDim;
  const bf16 *Vp = cp->prefix_v[layer] + (size_t)b * g.P * kHeadDim;
  const int *vi = vidx + (size_t)b * g.P;
  const int nkeys = nv + 1 + g.H;

  float m[4], l[4], o[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) o[i][d] = 0.f;
  }
  for (int k0 = 0; k0 < nkeys; k0 += kAttnKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kAttnKeys * kHeadDim; e += blockDim.x) {
      const int i = e / kHeadDim, d = e % kHeadDim, kk = k0 + i;
      float kv = 0.f, vv = 0.f;
      if (kk < nv) {
        const size_t p = (size_t)vi[kk] * kHeadDim + d;
        kv = bf16_to_f32(Kp[p]);
        vv = bf16_to_f32(Vp[p]);
      } else if (kk < nkeys) {
        const int row = (kk == nv) ? b : g.B + b * g.H + (kk - nv - 1);
        kv = to_f32(ks[(size_t)row * kHeadDim + d]);
        vv = to_f32(vs[(size_t)row * kHeadDim + d]);
      }
      Ks[i * (kHeadDim + 1) + d] = kv;
      Vs[i * kHeadDim + d] = vv;
    }
    __syncthreads();
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      const int qi = warp * 4 + qq, jq = qbase + qi;
      if (jq >= Tq) break;
      const bool state_q = step0 && jq == 0;
      const int ja = step0 ? jq - 1 : jq;  // action index of an action query
      // keys [prefix | state | actions]: the state query sees up to the state key, a
      // causal action query up to its own action, other action queries all keys
      const int last_key = state_q ? nv : (causal ? nv + 1 + ja : nkeys - 1);
      const int kk = k0 + lane;
      const bool vis = kk < nkeys && kk <= last_key;
      float s = -INFINITY;
      if (vis) {
        const float *qv = Qs + qi * kHeadDim;
        const float *kv = Ks + lane * (kHeadDim + 1);
        float acc = 0.f;
        for (int d = 0; d < kHeadDim; ++d) acc = fmaf(qv[d], kv[d], acc);
        s = acc * 0.0625f;
      }
      const float cmax = warp_max(s);
      if (cmax == -INFINITY) continue;
      const float mnew = fmaxf(m[qq], cmax);
      const float p = vis ? expf(s - mnew) : 0.f;
      const float corr = expf(m[qq] - mnew);
      l[qq] = l[qq] * corr + warp_sum(p);
#pragma unroll
      for (int d = 0; d < 8; ++d) o[qq][d] *= corr;
      for (int j = 0; j < kAttnKeys; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
        if (pj != 0.f) {
#pragma unroll
          for (int d = 0; d < 8; ++d) o[qq][d] = fmaf(pj, Vs[j * kHeadDim + lane + 32 * d], o[qq][d]);
        }
      }
      m[qq] = mnew;
    }
  }
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const int jq = qbase + warp * 4 + qq;
    if (jq >= Tq) break;
    const size_t base = (size_t)q_row(jq) * kQDim + head * kHeadDim;
    const float inv = 1.0f / l[qq];
#pragma unroll
    for (int d = 0; d < 8; ++d) out[base + lane + 32 * d] = from_f32<T>(o[qq][d] * inv);
  }
}

template <typename T>
void launch_attention(const T *q, const T *ks, const T *vs, const CallPtrs *cp, int layer, const int *nvalid,
                      const int *vidx, const Geo &g, int step0, int causal, T *out, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(k_attn_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
    attr_set = true;
  }
  const int Tq = step0 ? g.H + 1 : g.H;
  dim3 grid(g.B, kHeads, (Tq + kAttnQ - 1) / kAttnQ);
  launch_pdl(k_attn_simt<T>, grid, 128, kAttnSmem, s, q, ks, vs, cp, layer, nvalid, vidx, g, step0, causal, out);
}

template void launch_attention<float>(const float *, const float *, const float *, const CallPtrs *, int,
                                      const int *, const int *, const Geo &, int, int, float *, cudaStream_t);
template void launch_attention<bf16>(const bf16 *, const bf16 *, const bf16 *, const CallPtrs *, int,
                                     const int *, const int *, const Geo &, int, int, bf16 *, cudaStream_t);

}  // namespace pi0x
