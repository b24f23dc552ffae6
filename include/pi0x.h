/*
 * pi0x — the pi0 flow-matching denoising loop (action expert) on one B200.
 *
 * C ABI of the shared library libpi0x.so.  Every call returns an int status
 * (PI0X_OK = 0) and never aborts the process; no C++ exception crosses it.
 *
 * The operation is the one defined on the vllm-omni page
 * "vllm_omni/diffusion/models/pi0/modeling_pi0.py": given the per-layer prefix
 * K/V cache of the vision-language prefix, the robot state and the noise chunk
 * x_1, run `num_steps` Euler steps t = 1, 1+dt, ..., -dt (dt = -1/num_steps) of
 *   v_t = action_out_proj(final_norm(expert(embed_suffix(state, x_t, t), prefix_kv)))[last H]
 *   x_t <- x_t + dt * v_t
 * and return x_0 (functions `sample_actions`, `denoise_step`, `embed_suffix`,
 * `_compute_layer_suffix_only` on that page).  The expert is a Gemma decoder
 * ("gemma_300m": width 1024, 8 query heads, 1 KV head, head_dim 256, GeGLU MLP
 * 4096; `get_gemma_config`), RMSNorm x*rsqrt(mean(x^2)+1e-6)*(1+w), rotate-half
 * RoPE with base 10000, attention scale 1/sqrt(head_dim).
 */
#ifndef PI0X_H
#define PI0X_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------- */
enum {
  PI0X_OK = 0,
  PI0X_EINVAL = 1,        /* null pointer, non-positive size, num_steps <= 0, bad config */
  PI0X_EUNSUPPORTED = 2,  /* dims other than the compiled expert dims, no sm_100 device */
  PI0X_ENOMEM = 3,        /* device or host allocation failed */
  PI0X_ECUDA = 4,         /* a CUDA runtime call failed (see pi0x_last_error) */
  PI0X_ETIMEOUT = 5,      /* a bounded device-side wait expired; results are invalid */
  PI0X_EDEVICE = 6        /* a kernel reported an invalid launch configuration */
};

/* ---- precision modes ------------------------------------------------------- */
enum {
  PI0X_BF16 = 0,  /* bf16 weights and GEMM operands, fp32 accumulate, fp32 residual
                     stream, fp32 softmax with probabilities rounded to bf16 */
  PI0X_FP32 = 1   /* every operation in fp32 (no TF32) */
};

/* ---- element type of weight arrays handed to pi0x_create -------------------- */
enum {
  PI0X_DTYPE_BF16 = 0,  /* uint16 bf16 bit patterns */
  PI0X_DTYPE_F32 = 1
};

/* Dimensions.  The library is compiled for width 1024, mlp_dim 4096, 8 query
 * heads, 1 KV head and head_dim 256 (PI0X_EUNSUPPORTED otherwise); depth is
 * 1..32, horizon 1..64, action_dim and state_dim 1..64 (action_dim a
 * multiple of 4, state_dim a multiple of 4). */
typedef struct {
  int width, depth, mlp_dim, num_heads, num_kv_heads, head_dim;
  int horizon, action_dim, state_dim;
  int precision;      /* PI0X_BF16 or PI0X_FP32 */
} pi0x_config;

/* One expert layer, nn.Linear (out, in) row-major layout, no biases (Gemma). */
typedef struct {
  const void *in_norm_w;    /* (width)                      input_layernorm gain */
  const void *q_w;          /* (num_heads*head_dim, width)  */
  const void *k_w;          /* (head_dim, width)            */
  const void *v_w;          /* (head_dim, width)            */
  const void *o_w;          /* (width, num_heads*head_dim)  */
  const void *post_norm_w;  /* (width)                      post_attention_layernorm gain */
  const void *gate_w;       /* (mlp_dim, width)             */
  const void *up_w;         /* (mlp_dim, width)             */
  const void *down_w;       /* (width, mlp_dim)             */
} pi0x_layer_weights;

/* All weights (the pi0 projections of `Pi0ForActionPrediction.__init__` plus
 * the expert).  Pointers may be host or device memory (unified addressing
 * decides); every array is read during pi0x_create only and may be freed
 * afterwards.  `dtype` gives the element type of every array. */
typedef struct {
  const void *state_proj_w, *state_proj_b;    /* (width, state_dim), (width)   */
  const void *action_in_w, *action_in_b;      /* (width, action_dim), (width)  */
  const void *time_in_w, *time_in_b;          /* (width, 2*width), (width): action_time_mlp_in */
  const void *time_out_w, *time_out_b;        /* (width, width), (width): action_time_mlp_out  */
  const void *action_out_w, *action_out_b;    /* (action_dim, width), (action_dim) */
  const void *final_norm_w;                   /* (width) */
  const pi0x_layer_weights *layers;           /* host array of `depth` entries */
  int dtype;                                  /* PI0X_DTYPE_BF16 or PI0X_DTYPE_F32 */
} pi0x_weights;

typedef struct pi0x_handle pi0x_handle;

/* Create a sampler on the current CUDA device: validates `cfg`, copies and
 * repacks the weights into device memory owned by the handle.  On success
 * *out receives the handle (destroy with pi0x_destroy).  Synchronous. */
int pi0x_create(const pi0x_config *cfg, const pi0x_weights *weights, pi0x_handle **out);

/* Run the whole num_steps Euler loop (`sample_actions` minus the prefix pass).
 *
 *  prefix_k, prefix_v : HOST arrays of `depth` pointers; entry l points to the
 *                       layer-l prefix key/value cache, shape (B, 1, P, head_dim),
 *                       bf16, contiguous, already rotated (post-RoPE), as the
 *                       prefix pass of the page caches them.
 *  prefix_valid_mask  : (B, P) uint8, nonzero = valid prefix token (may be NULL
 *                       when P == 0).  Any pattern is allowed (holes,
 *                       all-zero rows).  Suffix
 *                       positions continue at the per-sample count of valid
 *                       prefix tokens.
 *  B, P               : batch (1..4096) and prefix length (0..8192).
 *  state              : (B, state_dim) float32.
 *  x1                 : (B, horizon, action_dim) float32, the t = 1 noise.
 *  num_steps          : Euler steps (1..1024).
 *  x0                 : (B, horizon, action_dim) float32 output; may alias x1.
 *  stream             : a cudaStream_t (NULL = legacy default stream).
 *
 * Every array may live in device memory or host memory (pinned or pageable);
 * host arrays are staged through handle-owned device buffers and x0 is copied
 * back, all on `stream`.  The call enqueues its work on `stream` and returns:
 * device inputs must stay valid and x0 must not be read until the stream
 * reaches the end of the call.  The library keeps no caller pointer after it
 * returns.  Calls on one handle must not overlap on the device (they share the
 * handle's workspace); use one handle per concurrent stream.
 * Errors: PI0X_EINVAL for null pointers or sizes out of range (num_steps <= 0
 * is rejected because dt = -1/num_steps), PI0X_ENOMEM, PI0X_ECUDA. */
int pi0x_sample(pi0x_handle *h, const void *const *prefix_k, const void *const *prefix_v,
                const uint8_t *prefix_valid_mask, int B, int P, const float *state,
                const float *x1, int num_steps, float *x0, void *stream);

/* Wait for all work of the handle's last call and read the device error word.
 * Returns PI0X_OK, PI0X_ETIMEOUT (a bounded device wait gave up; the outputs
 * of that call are invalid), PI0X_EDEVICE or PI0X_ECUDA.  Clears the word. */
int pi0x_sync_status(pi0x_handle *h);

/* ---- solver / convention variants --------------------------------------------
 * The default is pi0's own loop (`sample_actions` / `denoise_step` on the
 * vllm-omni pi0 page): t from 1 (noise) to 0 with dt = -1/N, the out-projection
 * is the velocity, action tokens see each other.  pi0x_set_variant selects the
 * conventions of the Wall-X flow-matching sampler instead, each independently:
 *  - time_grid PI0X_TIME_LINSPACE: t from 0 (noise) to 1 on torch.linspace(0, 1,
 *    N+1) integrated with a fixed-grid Euler step (its odeint call), taken as
 *    t_k = fp32(k/N) correctly rounded, step size fp32(t_{k+1} - t_k);
 *  - x_prediction = 1: the out-projection is the clean action x_hat and the
 *    velocity is x_hat - x_1 (its use_x_pred branch: prediction minus noise);
 *  - causal_actions = 1: action token i sees the prefix, the state and actions
 *    0..i only (its causal_action_attention_mask, a lower-triangular suffix block).
 * The setting applies to later pi0x_sample calls on the handle; changing it
 * waits for the handle's last call and drops the cached graphs.
 * Errors: PI0X_EINVAL for a null handle or a value out of range. */
enum {
  PI0X_TIME_PI0 = 0,      /* t: 1 -> 0, dt = -1/N */
  PI0X_TIME_LINSPACE = 1  /* t: 0 -> 1 on fp32(k/N) */
};
int pi0x_set_variant(pi0x_handle *h, int time_grid, int x_prediction, int causal_actions);

/* Number of kernels one pi0x_sample(B, P, num_steps) call launches (its own
 * kernels only, not memory copies), or -1 for invalid arguments.  In bf16 mode a
 * batch whose rows fit one 128-row tile (B * (horizon + 1) <= 128) runs every
 * Euler step in one persistent kernel after five small set-up kernels; larger
 * batches run one kernel per projection, attention and small step. */
long pi0x_launch_count(const pi0x_handle *h, int B, int P, int num_steps);

/* ---- per-kernel-class device timing ------------------------------------------
 * With profiling on, the next pi0x_sample calls record a CUDA event pair around
 * every kernel launch (inside the captured graph, so kernels still run back to
 * back); pi0x_profile_read then reports, for the most recent such call, how many
 * kernels of a class ran and their summed device time in milliseconds.  It
 * synchronizes the handle's last stream.  Profiled calls use a separate graph, so
 * turning profiling on does not change the unprofiled path. */
enum {
  PI0X_K_PREP = 0,   /* mask compaction, time-MLP half, x_1 copy (once per call) */
  PI0X_K_EMBED = 1,  /* state and action input projections */
  PI0X_K_GEMM = 2,   /* every Linear of the expert and of the action-time MLP */
  PI0X_K_NORM = 3,   /* RMSNorm */
  PI0X_K_ROPE = 4,   /* RoPE of q/k, v copy */
  PI0X_K_ATTN = 5,   /* masked MQA attention */
  PI0X_K_GEGLU = 6,  /* gated GELU(tanh) */
  PI0X_K_FINAL = 7,  /* final norm + action out-proj + Euler update */
  PI0X_K_LOOP = 8,   /* the persistent small-batch loop kernel (every step of a call) */
  PI0X_K_COUNT = 9
};
int pi0x_profile_enable(pi0x_handle *h, int on);
int pi0x_profile_read(pi0x_handle *h, int kclass, long *launches, double *total_ms);

/* Human-readable name of a status code; never NULL. */
const char *pi0x_status_string(int status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char *pi0x_last_error(void);

/* Free everything the handle owns.  Waits for the handle's work first.
 * Accepts NULL. */
void pi0x_destroy(pi0x_handle *h);

/* Library version as major*10000 + minor*100 + patch. */
int pi0x_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PI0X_H */
