// moe_layer_forward_static: the whole layer without any caller-provided
// workspace and without allocating anything.
//
// Some callers cannot hand this library device memory for scratch: code that
// runs where cudaMalloc is off limits (a host application that owns every
// device allocation through its own pool, a real-time loop that must not
// call cudaMalloc/cudaFree because they can synchronise the device and stall
// other streams, or plug-in code that only ever sees the tensors it is
// given).  This entry point serves them: its scratch is a fixed array in the
// library's own device memory, reserved when the library is loaded.
//
// The array is a file-scope __device__ object of kStaticScratchBytes bytes.
// Every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address, so the first call on
// each device (with that device current) looks its address up with
// cudaGetSymbolAddress and caches it; make that first call before starting
// any stream capture.  The entry point never calls cudaMalloc, cudaFree or any
// allocating routine.
//
// All calls share the one array and it keeps whatever the previous call left
// there.  Each call zeroes the arrival counter of the router with an
// asynchronous memset on its stream; the kernels clear the rest of the scratch
// they rely on (the row-block GEMV's split-block counters) at the start of
// every call, so calls of different shapes may follow one another.  Two calls
// whose work overlaps on the GPU (different streams, no ordering between
// them) race on the array and corrupt each other's results.  A device-side
// wait that runs out latches MOE_ERR_TIMEOUT in the array's error word, which
// no call clears: moe_get_error_static() reads and clears it.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch for the current device (looked up once
// per device).  Returns nullptr if the lookup fails.
void* static_scratch_address() {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_layer_forward_static(const uint16_t* x, const float* w_router,
                                                 const float* bias,
                                                 const moe_mxfp4_experts_t* experts,
                                                 const moe_mxfp4_experts_t* shared,
                                                 moe_shape_t shape, int32_t precision,
                                                 uint16_t* y, int32_t* topk_idx_out,
                                                 float* topk_w_out, void* stream) {
  // Host-side checks first: nothing touches the device for a bad request.
  const size_t need = moe_workspace_bytes(shape, MOE_PATH_GEMV, precision, shared != nullptr);
  if (need == 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (need > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = static_scratch_address();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the router's arrival counter (the error word in front of it stays latched
  // until moe_get_error_static reads it)
  const WsLayout L = ws_layout(shape, shared != nullptr, 0);
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + L.counters, 0, 64, s) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return moe_layer_forward(x, w_router, bias, experts, shared, shape, MOE_PATH_GEMV, precision, y,
                           topk_idx_out, topk_w_out, scratch, kStaticScratchBytes, stream);
}

extern "C" moe_status_t moe_get_error_static(void* stream) {
  void* scratch = static_scratch_address();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  return moe_get_error(scratch, stream);
}
