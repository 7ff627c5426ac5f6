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
// The array is shared by every call on a device and keeps the last call's
// contents.  The tree-sum kernels write every scratch entry they later read,
// so nothing needs clearing between calls; but two calls whose kernels overlap
// on the GPU (different streams, no ordering between them) race on it and
// give wrong results.
#include <mutex>

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

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Device address of g_dq_scratch on the current device (host code cannot use
// the symbol itself as a device pointer).  Looked up once per device.
void* scratch_ptr(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dq_scratch) != cudaSuccess) return nullptr;
    g_ptr[dev] = p;
  }
  return g_ptr[dev];
}

}  // namespace

extern "C" ql_status nf4_double_quant_noalloc(const float* absmax, int64_t nb, uint8_t* absmax_q, float* scale2,
                                              float* offset, void* stream) {
  if (nb <= 0) return QL_ERR_INVALID_ARG;
  if (nb > QL_NOALLOC_MAX_BLOCKS) return QL_ERR_UNSUPPORTED;
  auto aligned16 = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!aligned16(absmax) || !aligned16(absmax_q) || !aligned16(scale2) || !aligned16(offset))
    return QL_ERR_INVALID_ARG;
  if (ql::dq_workspace_bytes(nb) > sizeof(g_dq_scratch)) return QL_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return QL_ERR_CUDA;
  void* ws = scratch_ptr(dev);
  if (!ws) return QL_ERR_CUDA;
  return ql::launch_double_quant(absmax, nb, absmax_q, scale2, offset, ws, reinterpret_cast<cudaStream_t>(stream));
}
