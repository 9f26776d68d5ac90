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
//    with that device current; make that first call before any stream capture. The address
//    is cached per device together with the context it was looked up in: after a device reset
//    (a new primary context, in which the array may sit elsewhere) the next call looks it up
//    again, so that call too belongs before any capture.
//  - Problems whose scratch would exceed ADX_STATIC_SCRATCH_BYTES are rejected with
//    ADX_EWORKSPACE before anything is launched; invalid or unsupported operands return the
//    same codes as adx_index_prefill (ADX_EINVAL, ADX_EUNSUPPORTED), also before any launch.
//  - All calls on a device share the one array. Calls whose work overlaps on the GPU (other
//    streams, other host threads) race on it; serialise them, for example on one stream.
//  - The array keeps the previous call's contents. Only the status word has to start at
//    zero, and each call clears it on its stream first; everything else it reads is written
//    earlier in the same call.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/adx.h"
#include "adx_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[ADX_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
void* g_scratch_ctx[kMaxDevices] = {nullptr};  // context the address was looked up in

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current context, through the driver entry point the runtime exposes
// (the library does not link the driver library directly).
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_scratch on the current device. In host code the name g_scratch is only
// a host-side stand-in; kernels must be given this address. Looked up once per device and
// context (with the device current), again after a device reset replaced the context.
adx_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ADX_ECUDA;
  void* ctx = current_context();  // null until the runtime made the device's context current
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr || ctx == nullptr || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return ADX_ECUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context();  // the lookup made the context current
  }
  *out = g_scratch_ptr[dev];
  return ADX_OK;
}

}  // namespace

extern "C" adx_status adx_index_prefill_noalloc(const adx_operands* ops, int32_t K,
                                                int32_t* topk_idx, float* topk_score,
                                                int32_t* device_status, void* stream) {
  if (!ops || !topk_idx) return ADX_EINVAL;
  const adx_status chk = adx::check_prefill_args(ops, K);
  if (chk != ADX_OK) return chk;
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
