// adx_index_prefill_noalloc: the flat prefill indexer for callers that cannot allocate device
// memory.
//
// Some callers have no way to allocate: an engine that plans every device buffer ahead of
// time in its own arena and forbids allocations on the serving path, a plugin host that
// hands out no allocator, or C code with no memory manager of its own. This entry point needs
// no workspace from them. Its scratch (score matrix, folded queries, status word) lives in a
// fixed array compiled into this library, so every GPU that loads the library holds
// ADX_STATIC_SCRATCH_BYTES of device memory until the process exits. The caller still
// provides the operands and the output buffers.
//
// Rules for callers:
//  - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
//    with that device current; make that first call before any stream capture.
//  - Problems whose scratch would exceed ADX_STATIC_SCRATCH_BYTES are rejected with
//    ADX_EWORKSPACE before anything is launched.
//  - All calls on a device share the one array. Calls whose work overlaps on the GPU (other
//    streams, other host threads) race on it; serialise them, for example on one stream.
//  - The array keeps the previous call's contents. Only the status word has to start at
//    zero, and each call clears it on its stream first; everything else it reads is written
//    earlier in the same call.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/adx.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[ADX_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device, looked up once per device. In host
// code the name g_scratch is only a host-side stand-in; kernels must be given this address.
adx_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ADX_ECUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return ADX_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ADX_OK;
}

}  // namespace

extern "C" adx_status adx_index_prefill_noalloc(const adx_operands* ops, int32_t K,
                                                int32_t* topk_idx, float* topk_score,
                                                int32_t* device_status, void* stream) {
  if (!ops || K <= 0 || !topk_idx) return ADX_EINVAL;
  const size_t need = adx_workspace_size(ADX_OP_PREFILL, ops, K, 0, 0, 0);
  if (need == 0) return ADX_EINVAL;
  if (need > ADX_STATIC_SCRATCH_BYTES) return ADX_EWORKSPACE;
  void* ws = nullptr;
  adx_status r = scratch_address(&ws);
  if (r != ADX_OK) return r;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, ADX_STATUS_BYTES, s) != cudaSuccess) return ADX_ECUDA;
  r = adx_index_prefill(ops, K, topk_idx, topk_score, nullptr, 0, ws, ADX_STATIC_SCRATCH_BYTES,
                        stream);
  if (r != ADX_OK) return r;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return ADX_ECUDA;
  return ADX_OK;
}
