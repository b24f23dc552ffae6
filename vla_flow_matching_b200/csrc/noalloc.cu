// pi0x_attention_noalloc: the tcgen05 suffix attention with every byte of scratch
// memory in one fixed device array, so that the call allocates nothing.
//
// Who needs this: callers that must not allocate device memory once they are
// running — a robot control loop with a hard real-time budget (cudaMalloc can
// block for milliseconds and synchronises the device), a process whose memory is
// owned by a pool or caching allocator that other allocations would fragment, or
// code that has set up all of its memory at start-up and treats any later
// allocation as a failure.  The caller still provides inputs and outputs.
//
// The scratch array is static device memory of kScratchBytes: every GPU that
// loads this library keeps it reserved until the process exits.  All calls share
// it and it keeps the contents of the last call, so two calls that overlap on the
// GPU (on different streams, or from different host threads) race and corrupt each
// other's results.  The error word inside it is cleared at the start of each call;
// the other scratch regions are fully rewritten before they are read.
#include <mutex>
#include <string.h>
#include <string>

#include "../../include/pi0x.h"
#include "../../include/pi0x_debug.h"
#include "common.cuh"
#include "kernels.cuh"

namespace pi0x {
namespace {

// 32 MiB.  Split-KV runs only while row tiles x batch < 96 and then uses
// ceil(148 / tiles) splits (attn_tc_splits), so tiles x splits <= 73 x 3 = 219 and the
// partials take at most 219 x 128 rows x 258 floats = 28.9 MB; the valid-index list
// (4 B per prefix position per sample) and the call table share the rest.
constexpr size_t kScratchBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {nullptr};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Device address of the scratch array on the current device.  In host code the
// array's name only stands in for the symbol; the address has to be asked for,
// once per device, with that device current.
int scratch_address(void **out, std::string &why) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    why = std::string("cudaGetDevice: ") + cudaGetErrorString(e);
    return PI0X_ECUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    why = "device ordinal out of range";
    return PI0X_EUNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      why = std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e);
      cudaGetLastError();
      return PI0X_ECUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PI0X_OK;
}

}  // namespace
}  // namespace pi0x

using namespace pi0x;

extern "C" int pi0x_attention_noalloc(const void *q, const void *ks, const void *vs, const void *prefix_k,
                                      const void *prefix_v, const void *mask, int B, int H, int P, int step0,
                                      void *out, void *stream) {
  if (!q || !ks || !vs || !out || (P > 0 && (!prefix_k || !prefix_v || !mask)) || B < 1 || H < 1 || H > 64 ||
      P < 0)
    return PI0X_EINVAL;
  Geo g{B, H, 32, 32, P, B + B * H};
  const int splits = attn_tc_splits(g, step0);
  // scratch layout: [call table][error word][n_valid][valid-index list][split partials]
  const size_t off_cp = 0;
  const size_t off_err = align256(off_cp + sizeof(CallPtrs));
  const size_t off_nv = align256(off_err + sizeof(unsigned));
  const size_t off_vidx = align256(off_nv + sizeof(int) * (size_t)B);
  const size_t off_part = align256(off_vidx + sizeof(int) * (size_t)B * (P > 0 ? P : 1));
  const size_t need = off_part + sizeof(float) * attn_tc_partial_floats(g, step0, splits);
  if (need > kScratchBytes) {
    set_last_error("pi0x_attention_noalloc: the problem needs more scratch than the 32 MiB static array");
    return PI0X_EINVAL;
  }

  void *base = nullptr;
  std::string why;
  int st = scratch_address(&base, why);
  if (st != PI0X_OK) {
    set_last_error(why.c_str());
    return st;
  }
  uint8_t *sb = static_cast<uint8_t *>(base);
  CallPtrs *d_cp = reinterpret_cast<CallPtrs *>(sb + off_cp);
  unsigned *d_err = reinterpret_cast<unsigned *>(sb + off_err);
  int *nvalid = reinterpret_cast<int *>(sb + off_nv);
  int *vidx = reinterpret_cast<int *>(sb + off_vidx);
  float *part = reinterpret_cast<float *>(sb + off_part);

  CallPtrs cp;
  memset(&cp, 0, sizeof(cp));
  cp.prefix_k[0] = (const bf16 *)prefix_k;
  cp.prefix_v[0] = (const bf16 *)prefix_v;
  cp.mask = (const uint8_t *)mask;
  if (!attn_tc_maps(cp, 1, B, P, ks, vs, (uint64_t)g.R)) {
    set_last_error("pi0x_attention_noalloc: cuTensorMapEncodeTiled failed (pointers must be 16-byte aligned)");
    return PI0X_EINVAL;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(d_cp, &cp, sizeof(cp), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_err, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) {
    launch_prep_mask(d_cp, B, P, nvalid, vidx, s);
    launch_attention_tc((const bf16 *)q, (const bf16 *)ks, (const bf16 *)vs, d_cp, 0, 0, nvalid, vidx, g, step0, 0,
                        splits,
                        (bf16 *)out, part, d_err, s);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  unsigned w = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&w, d_err, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    set_last_error((std::string("pi0x_attention_noalloc: ") + cudaGetErrorString(e)).c_str());
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? PI0X_ENOMEM : PI0X_ECUDA;
  }
  if (w) {
    set_last_error(("pi0x_attention_noalloc: device error word 0x" + std::to_string(w)).c_str());
    return PI0X_ETIMEOUT;
  }
  return PI0X_OK;
}
