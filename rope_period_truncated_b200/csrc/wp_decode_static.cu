// Decode entry point that allocates nothing: the split-KV partial results live
// in a fixed-size array in this library's device image instead of a
// caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc — for instance a serving
// engine whose device memory is fully planned up front and handed out by its
// own pool (an extra allocation would break its accounting or fail), or a
// latency-critical decode loop that must not hit cudaMalloc/cudaFree, which
// can synchronise the device.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "waveprune.h"

namespace {

// Fixed scratch shared by every call on a device. Every GPU that loads the
// library holds it until the process exits.
constexpr size_t kScratchBytes = static_cast<size_t>(WP_DECODE_STATIC_SCRATCH_BYTES);
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current, and cached. Device ordinals from
// kMaxDevices on are not served.
int scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return WP_ERR_CUDA;
  if (dev >= kMaxDevices) return WP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return WP_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return WP_OK;
}

}  // namespace

extern "C" int wp_decode_static(const void *q, const void *kcache, const void *vcache, const int32_t *lens,
                                int Lmax, int B, int H_q, int H_kv, int d_h, const int32_t *group_cut,
                                float softmax_scale, void *o, float *lse, void *stream) {
  // The pointer checks of wp_decode come first, so a bad pointer is reported
  // as such whatever the batch size.
  const auto misaligned = [](const void *p, uintptr_t m) { return (reinterpret_cast<uintptr_t>(p) & m) != 0; };
  if (q == nullptr || kcache == nullptr || vcache == nullptr || lens == nullptr || o == nullptr) return WP_ERR_ARG;
  if (misaligned(q, 15) || misaligned(kcache, 15) || misaligned(vcache, 15) || misaligned(o, 15) ||
      misaligned(lens, 3) || (lse != nullptr && misaligned(lse, 3)))
    return WP_ERR_ARG;
  const size_t need = wp_decode_workspace_bytes(B, H_q, d_h, Lmax);
  if (need == 0) return WP_ERR_ARG;
  if (need > kScratchBytes) return WP_ERR_UNSUPPORTED;  // batch too large for the fixed scratch
  void *scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != WP_OK) return st;
  // Every partial the combine reads is written earlier in the same call, so
  // nothing in the scratch has to start at zero.
  return wp_decode(q, kcache, vcache, lens, Lmax, B, H_q, H_kv, d_h, group_cut, softmax_scale, o, lse, scratch,
                   kScratchBytes, stream);
}
