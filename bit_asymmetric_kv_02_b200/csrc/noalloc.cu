// kivi_decode_attention_noalloc: decode attention whose scratch space is a fixed array inside the
// library, for callers that cannot allocate device memory when they decode.
//
// The array is a file-scope __device__ variable.  Every GPU that loads this library reserves its
// KIVI_NOALLOC_SCRATCH_BYTES when the library's module is loaded there and keeps them until the
// process exits.  In host code the array's name only stands in for the variable; its device
// address is looked up once per device with cudaGetSymbolAddress (with that device current) and
// cached.  All calls share the array and it keeps the last call's contents, so calls whose work
// overlaps on the GPU (different streams, or host threads using one device) race on it.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "kivi.h"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[KIVI_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct ScratchAddresses {
  std::mutex mu;
  void* addr[kMaxDevices] = {};
};

ScratchAddresses& scratch_addresses() {
  static ScratchAddresses s;
  return s;
}

// Device address of g_decode_scratch on the current device; looked up on the first call per device.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KIVI_ERR_CUDA;
  ScratchAddresses& s = scratch_addresses();
  std::lock_guard<std::mutex> lock(s.mu);
  if (s.addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return KIVI_ERR_CUDA;
    s.addr[dev] = p;
  }
  *out = s.addr[dev];
  return KIVI_OK;
}

}  // namespace

extern "C" int kivi_decode_attention_noalloc(const kivi_config* cfg, const kivi_cache* cache, const uint16_t* q_dev,
                                             int32_t num_q_heads, float scale, uint16_t* out_dev,
                                             int32_t* dev_status, void* stream) {
  // Every argument check of kivi_decode_attention runs first: without a workspace it returns
  // KIVI_ERR_WORKSPACE when everything else is valid, and enqueues nothing either way.
  int st = kivi_decode_attention(cfg, cache, q_dev, num_q_heads, scale, out_dev, nullptr, 0, dev_status, stream);
  if (st != KIVI_ERR_WORKSPACE) return st;
  const size_t need = kivi_decode_workspace_bytes(cfg, num_q_heads);
  // decode_impl accepted every argument, so a zero size means the two size rules disagree
  if (need == 0) return KIVI_ERR_INTERNAL;
  if (need > static_cast<size_t>(KIVI_NOALLOC_SCRATCH_BYTES)) return KIVI_ERR_WORKSPACE;
  void* base = nullptr;
  if ((st = scratch_address(&base)) != KIVI_OK) return st;
  // The per-head tickets at the end of the scratch must be zero when the kernel starts.  The kernel
  // leaves them at zero, but a call that ended in a device error may not have: clear them.
  const size_t heads = static_cast<size_t>(cfg->batch) * static_cast<size_t>(cfg->num_kv_heads);
  const size_t ticket_bytes = (heads * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  if (cudaMemsetAsync(static_cast<unsigned char*>(base) + (need - ticket_bytes), 0, ticket_bytes,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KIVI_ERR_CUDA;
  return kivi_decode_attention(cfg, cache, q_dev, num_q_heads, scale, out_dev, base, need, dev_status, stream);
}
