// Allocation-free form of the non-absorbed chunk attention.
//
// vmla_chunk_attention_nonabsorbed needs a workspace for the materialised
// per-head keys and values, which its caller must allocate.  Some callers have
// no way to do that: a host program that only receives tensors from another
// runtime and owns no allocator of its own, a framework whose caching allocator
// already holds the device memory budget so that a raw cudaMalloc would fail or
// fragment it, or a latency-sensitive loop that cannot afford the device-wide
// synchronisation cudaMalloc/cudaFree imply.  For them this file provides the
// same computation with its scratch in a fixed, file-scope device array.
//
// The array is a static __device__ object of kNoAllocScratchBytes (8 MiB): every
// GPU that loads this library carries it until the process exits, whether or not
// the entry point is ever called.  Host code must not pass the array's name to a
// kernel -- on the host that name is only a stand-in for the symbol -- so the
// device address is looked up with cudaGetSymbolAddress, once per device (with
// that device current), and cached.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "videomla.h"

namespace {

constexpr int64_t kNoAllocScratchBytes = VMLA_NOALLOC_SCRATCH_BYTES;

// Scratch shared by every call on a device: it keeps whatever the last call left.
// Nothing in it needs to start at zero -- each call writes every row of the
// materialised keys/values it later reads -- but two calls that overlap on the
// GPU (other streams, or other threads' streams) would race on it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device; nullptr (and *err set) on failure.
void* scratch_address(cudaError_t* err) {
  static std::mutex mu;
  static void* cached[64] = {nullptr};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    cached[dev] = p;
  }
  return cached[dev];
}

}  // namespace

namespace vmla {
vmla_status record_error(vmla_status s, const char* msg);  // sets vmla_last_error() (api.cu)
}

extern "C" {

vmla_status vmla_chunk_attention_nonabsorbed_noalloc(const uint16_t* q, const uint16_t* q_rope,
                                                     const uint16_t* w_uk, const uint16_t* w_uv,
                                                     const uint16_t* cache, int32_t batch, int32_t n_q,
                                                     int32_t heads, int64_t cap, int64_t n_kv, int64_t t0,
                                                     int32_t grid_h, int32_t grid_w, float scale, uint16_t* out,
                                                     void* stream) {
  const int64_t need = vmla_materialized_kv_bytes(batch, heads, n_kv);
  if (need <= 0 && batch >= 1 && heads >= 1 && n_kv >= 1)  // sizes whose buffer overflows int64
    return vmla::record_error(VMLA_ERR_UNSUPPORTED,
                              "chunk_attention_nonabsorbed_noalloc: workspace size overflows int64");
  if (need <= 0) {
    // Bad sizes: the full validation (and its message) comes from the workspace form.
    return vmla_chunk_attention_nonabsorbed(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                            grid_w, scale, nullptr, 0, out, stream);
  }
  char msg[256];
  if (need > kNoAllocScratchBytes) {
    snprintf(msg, sizeof msg,
             "chunk_attention_nonabsorbed_noalloc: needs %lld bytes of scratch for batch*n_kv*heads = %lld, "
             "more than the built-in %lld (use vmla_chunk_attention_nonabsorbed with a workspace)",
             (long long)need, (long long)batch * n_kv * heads, (long long)kNoAllocScratchBytes);
    return vmla::record_error(VMLA_ERR_UNSUPPORTED, msg);
  }
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (!scratch) {
    snprintf(msg, sizeof msg, "chunk_attention_nonabsorbed_noalloc: cudaGetSymbolAddress of the scratch failed: %s",
             cudaGetErrorString(err));
    return vmla::record_error(VMLA_ERR_CUDA, msg);
  }
  return vmla_chunk_attention_nonabsorbed(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                          grid_w, scale, scratch, kNoAllocScratchBytes, out, stream);
}

}  // extern "C"
