// hils_decode_noalloc: the decode step for callers that cannot allocate device
// memory, so cannot hand hils_decode a workspace.
//
// Some callers are not allowed to call cudaMalloc at all: plugins run by a host
// engine that owns every device allocation and passes kernels only their
// inputs and outputs, and services that must not allocate once they are
// serving (cudaMalloc can synchronise the device and can fail under memory
// pressure).  For them the decode scratch lives in a fixed array compiled into
// this library, kScratchBytes long; every GPU that loads the library keeps
// that much device memory until the process exits.
#include <mutex>
#include <string>

#include "hils_common.cuh"

namespace {

constexpr size_t kScratchBytes = (size_t)4 << 20;   // 4 MiB
constexpr int kMaxDevices = 64;

}  // namespace

// The scratch array.  Host code must not use its name as an address: on the
// host it is only a stand-in, and the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

int noalloc_fail(int status, const std::string& msg) {
  hils::record_error(msg.c_str());
  return status;
}

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(HILS_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(HILS_ERR_UNSUPPORTED, "device ordinal too large");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess)
      return noalloc_fail(HILS_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HILS_OK;
}

}  // namespace

extern "C" size_t hils_decode_noalloc_capacity(void) { return kScratchBytes; }

extern "C" int hils_decode_noalloc(const hils_config* cfg, const void* q, const void* k_new,
                                   const void* v_new, const float* A, const float* B,
                                   hils_kv_cache* cache, void* out, int32_t* idx_out, float* w_out,
                                   void* stream) {
  if (!cache) return noalloc_fail(HILS_ERR_INVALID_ARG, "cache is NULL");
  // validates the configuration and gives the scratch this call needs
  const size_t need = hils_workspace_size(cfg, HILS_OP_DECODE, 1, cache->max_chunks);
  if (need == 0) return HILS_ERR_INVALID_ARG;  // hils_last_error() already says why
  if (need > kScratchBytes)
    return noalloc_fail(HILS_ERR_WORKSPACE,
                        "decode needs " + std::to_string(need) + " bytes of scratch; the built-in "
                        "array holds " + std::to_string(kScratchBytes) +
                        " (use hils_decode with a workspace)");
  void* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st != HILS_OK) return st;
  // The array keeps whatever the previous call left; the step's completion
  // counters must start at zero, so the call clears them (after its checks)
  return hils::decode_call(cfg, q, k_new, v_new, A, B, cache, out, idx_out, w_out, scratch,
                           kScratchBytes, true, stream);
}
