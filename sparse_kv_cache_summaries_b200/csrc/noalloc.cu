// compkv_decode_step_static: the decode step with its scratch in a fixed device array instead of a
// caller workspace, for callers that can hand the library inputs and outputs but cannot allocate
// device memory themselves.
#include <cstdint>

#include "compkv.h"

// The scratch every call of compkv_decode_step_static uses. Static device memory: each GPU that
// loads the library holds it until the process exits, zero-filled at load.
static __device__ __align__(256) unsigned char g_compkv_static_scratch[COMPKV_STATIC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device. The host-side symbol is only a
// stand-in for it, so the address is looked up with that device current, on every call: a
// cached address would go stale if the context were torn down (cudaDeviceReset) and the module
// loaded again, and the lookup is a host-side table read once the module is loaded.
int scratch_for_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_compkv_static_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return COMPKV_ERR_CUDA;
  }
  *out = p;
  return COMPKV_OK;
}

}  // namespace

extern "C" int compkv_decode_step_static(const compkv_shape* shape, compkv_dtype dtype,
                                         compkv_mode mode, const void* q, const void* K,
                                         const void* V, const void* mean_k, const float* var_g,
                                         const void* mean_v, const int32_t* count,
                                         int32_t budget_tokens, float softmax_scale,
                                         int32_t* sel_idx, float* scores, float* out,
                                         void* stream) {
  const int32_t kb = compkv_num_selected(shape, budget_tokens);  // validates shape and budget
  if (kb < 0) return kb;
  if (compkv_workspace_bytes(shape, budget_tokens) > static_cast<size_t>(COMPKV_STATIC_SCRATCH_BYTES))
    return COMPKV_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  const int st = scratch_for_current_device(&ws);
  if (st != COMPKV_OK) return st;
  return compkv_decode_step(shape, dtype, mode, q, K, V, mean_k, var_g, mean_v, count,
                            budget_tokens, softmax_scale, sel_idx, scores, out, ws,
                            static_cast<size_t>(COMPKV_STATIC_SCRATCH_BYTES), stream);
}

extern "C" int compkv_static_read_device_status(void* stream, int32_t* status) {
  if (status == nullptr) return COMPKV_ERR_INVALID_ARG;
  void* ws = nullptr;
  const int st = scratch_for_current_device(&ws);
  if (st != COMPKV_OK) return st;
  return compkv_read_device_status(ws, stream, status);
}
