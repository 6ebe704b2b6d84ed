// noalloc.cu — gptq_quantize_layer for callers that cannot allocate device memory.
//
// gptq_quantize_layer needs scratch (the fp32 working copy of W, the per-column errors and, for
// a permuted column order, the codes in sweep order), normally passed in by the caller as
// (ws, ws_bytes). Some callers cannot provide it: a plugin running inside another runtime that
// owns all device memory, or a service that must not allocate once it is serving. For them this
// file holds one fixed scratch array in the library itself and an entry point that uses it.
//
// The array lives in device global memory of every GPU that loads the library, for as long as
// the process runs. Its host-side name is only a host stand-in, not a device address, so the
// device address is looked up once per device with cudaGetSymbolAddress (the first call of the
// entry point on a device does this, with that device current) and cached.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = GPTQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return GPTQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GPTQ_OK;
}

}  // namespace

extern "C" int gptq_quantize_layer_noalloc(const void* W, int w_dtype, int64_t ldw,
                                           int64_t d_out, int64_t d_in, const float* U,
                                           const int32_t* perm, const uint8_t* dead,
                                           const gptq_params* p, uint8_t* codes, float* scales,
                                           float* zeros, int32_t* g_idx, int32_t* dev_status,
                                           gptq_stream_t stream) {
  const size_t need = gptq_workspace_size(d_out, d_in, p);
  if (need == 0) return GPTQ_ERR_INVALID_ARG;
  if (need > kScratchBytes) return GPTQ_ERR_WORKSPACE;  // layer too large for the fixed array
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != GPTQ_OK) return rc;
  return gptq_quantize_layer(W, w_dtype, ldw, d_out, d_in, U, perm, dead, p, codes, scales, zeros,
                             g_idx, ws, kScratchBytes, dev_status, stream);
}
