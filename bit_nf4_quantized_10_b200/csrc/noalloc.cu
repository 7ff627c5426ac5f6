// nf4_double_quant_noalloc: double quantization without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they quantize:
// a plugin or custom operator that is handed a stream and tensors by a host
// framework that owns the device memory pool (and exposes no allocator to it),
// or a code path that must not call cudaMalloc because cudaMalloc may
// synchronize the device.  This entry point serves them.  Its scratch for the
// float64 tree sums of the mean lives in a fixed array in device memory
// (g_dq_scratch below), statically sized, which every GPU that loads this
// library holds until the process exits.
//
// The array is shared by every call in a CUDA context and keeps the last
// call's contents.  The tree-sum kernels write every scratch entry they later
// read, so nothing needs clearing between calls; but two calls whose kernels
// overlap on the GPU (different streams, no ordering between them) race on it
// and give wrong results.
//
// The library's module is loaded once per CUDA context, so the array's device
// address belongs to a context, not to a device: a plugin running under its
// own driver-API context, or a primary context rebuilt after cudaDeviceReset,
// has its own copy at its own address.  The address is therefore looked up
// once per context and cached under the context's unique ID (cuCtxGetId),
// which is never reused within a process even when a context handle is.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace ql {
size_t dq_workspace_bytes(int64_t nb);
ql_status launch_double_quant(const float* absmax, int64_t nb, uint8_t* absmax_q, float* scale2, float* offset,
                              void* ws, cudaStream_t st);
}  // namespace ql

namespace {

// Tree sums of up to QL_NOALLOC_MAX_BLOCKS constants need ceil(nb/2048) +
// ceil(nb/2048^2) + ... doubles: 32768 + 16 + 1 at the maximum.
constexpr size_t kScratchDoubles = 32768 + 256;
static __device__ __align__(256) double g_dq_scratch[kScratchDoubles];

struct DriverFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

// Driver entry points through the runtime, so the library needs no link
// against libcuda.
const DriverFns& driver_fns() {
  static const DriverFns fns = [] {
    DriverFns f;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    return f;
  }();
  return fns;
}

std::mutex g_mu;
std::vector<std::pair<unsigned long long, void*>> g_ptr;   // (context ID, address of g_dq_scratch)

// Device address of g_dq_scratch in the current context (host code cannot use
// the symbol itself as a device pointer).  The first call in a context makes
// the context current-bound (cudaGetDevice/cudaSetDevice when the thread has
// none yet), looks the address up and caches it.
void* scratch_ptr() {
  const DriverFns& d = driver_fns();
  if (!d.get_current || !d.get_id) return nullptr;
  CUcontext ctx = nullptr;
  if (d.get_current(&ctx) != CUDA_SUCCESS) return nullptr;
  if (!ctx) {
    // no context bound to this thread yet: bind the current device's primary one
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return nullptr;
    if (d.get_current(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  }
  unsigned long long id = 0;
  if (d.get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  for (const auto& e : g_ptr)
    if (e.first == id) return e.second;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_dq_scratch) != cudaSuccess) return nullptr;
  g_ptr.emplace_back(id, p);
  return p;
}

}  // namespace

extern "C" ql_status nf4_double_quant_noalloc(const float* absmax, int64_t nb, uint8_t* absmax_q, float* scale2,
                                              float* offset, void* stream) {
  nvtxRangePushA("qlora_nf4/nf4_double_quant_noalloc");
  const ql_status st = [&]() -> ql_status {
    if (nb <= 0) return QL_ERR_INVALID_ARG;
    if (nb > QL_NOALLOC_MAX_BLOCKS) return QL_ERR_UNSUPPORTED;
    auto aligned16 = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!aligned16(absmax) || !aligned16(absmax_q) || !aligned16(scale2) || !aligned16(offset))
      return QL_ERR_INVALID_ARG;
    if (ql::dq_workspace_bytes(nb) > sizeof(g_dq_scratch)) return QL_ERR_UNSUPPORTED;
    void* ws = scratch_ptr();
    if (!ws) return QL_ERR_CUDA;
    return ql::launch_double_quant(absmax, nb, absmax_q, scale2, offset, ws, reinterpret_cast<cudaStream_t>(stream));
  }();
  nvtxRangePop();
  return st;
}
