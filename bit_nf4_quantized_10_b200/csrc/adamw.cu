// Fused AdamW step for the adapter parameters, with fp32 states that may live
// in CUDA managed (unified) memory: the paged optimizer.
//
// "QLoRA: Quantize Base Weights to 4-Bit", §2.3, and "QLoRA — Fine-Tuning a
// 65B Model on One GPU", "Paged optimizers: surviving the spikes": the
// optimizer states are registered in unified memory; when the GPU runs short
// they are paged out to host RAM and paged back for the next update.  Paging
// moves the states and leaves the arithmetic alone, so the update is AdamW
// with decoupled weight decay (the pages give no formula); "How it's used in
// practice" names the 32-bit variant (fp32 states).
//
// The kernel only reads and writes p, g, m, v through ordinary pointers:
// device memory, or managed memory wherever the driver currently holds its
// pages (a page on the host migrates on first touch).  qlora_paged_prefetch
// moves a managed range explicitly, to the device before an update or to the
// host after it.
//
// Every operation is one IEEE fp32 operation in a fixed order (no
// contraction), with constants prepared on the host:
//   keep = fl32(1 - lr wd), c1 = fl32(1 - b1^t), c2 = fl32(1 - b2^t),
//   p = fl32(p keep)
//   m = fl32(fl32(b1 m) + fl32((1 - b1) g))
//   v = fl32(fl32(b2 v) + fl32(fl32((1 - b2) g) g))
//   d = fl32(fl32(sqrt(fl32(v / c2))) + eps)
//   p = fl32(p - fl32(lr fl32(fl32(m / c1) / d)))
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "trace.cuh"

namespace ql {

struct AdamConsts {
  float keep, b1, omb1, b2, omb2, c1, c2, lr, eps;
};

__device__ __forceinline__ void adam_one(float& p, float g, float& m, float& v, const AdamConsts& k) {
  float pp = __fmul_rn(p, k.keep);
  m = __fadd_rn(__fmul_rn(k.b1, m), __fmul_rn(k.omb1, g));
  v = __fadd_rn(__fmul_rn(k.b2, v), __fmul_rn(__fmul_rn(k.omb2, g), g));
  const float d = __fadd_rn(__fsqrt_rn(__fdiv_rn(v, k.c2)), k.eps);
  p = __fsub_rn(pp, __fmul_rn(k.lr, __fdiv_rn(__fdiv_rn(m, k.c1), d)));
}

// Four elements per thread with 16-byte accesses, grid-stride; the last n % 4
// elements one by one.
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    __nv_bfloat16* __restrict__ p_bf16, int64_t n, AdamConsts k) {
  pdl_wait();
  pdl_trigger();
  const int64_t n4 = n / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 P = reinterpret_cast<float4*>(p)[i];
    const float4 G = reinterpret_cast<const float4*>(g)[i];
    float4 Mv = reinterpret_cast<float4*>(m)[i];
    float4 V = reinterpret_cast<float4*>(v)[i];
    adam_one(P.x, G.x, Mv.x, V.x, k);
    adam_one(P.y, G.y, Mv.y, V.y, k);
    adam_one(P.z, G.z, Mv.z, V.z, k);
    adam_one(P.w, G.w, Mv.w, V.w, k);
    reinterpret_cast<float4*>(p)[i] = P;
    reinterpret_cast<float4*>(m)[i] = Mv;
    reinterpret_cast<float4*>(v)[i] = V;
    if (p_bf16) {
      uint2 b;
      b.x = pack_bf16x2(P.x, P.y);
      b.y = pack_bf16x2(P.z, P.w);
      reinterpret_cast<uint2*>(p_bf16)[i] = b;
    }
  }
  for (int64_t j = n4 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride) {
    float P = p[j], Mv = m[j], V = v[j];
    adam_one(P, g[j], Mv, V, k);
    p[j] = P;
    m[j] = Mv;
    v[j] = V;
    if (p_bf16) p_bf16[j] = __float2bfloat16_rn(P);
  }
}

ql_status launch_adamw(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int64_t t, float lr,
                       float b1, float b2, float eps, float wd, cudaStream_t st) {
  AdamConsts k;
  // host constants: float64 arithmetic on the fp32 inputs, one rounding each
  k.keep = (float)(1.0 - (double)lr * (double)wd);
  k.b1 = b1;
  k.b2 = b2;
  k.omb1 = (float)(1.0 - (double)b1);
  k.omb2 = (float)(1.0 - (double)b2);
  k.c1 = (float)(1.0 - std::pow((double)b1, (double)t));
  k.c2 = (float)(1.0 - std::pow((double)b2, (double)t));
  k.lr = lr;
  k.eps = eps;
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  const int64_t need = (std::max<int64_t>(n / 4, 1) + 255) / 256;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)sms * 8));
  TraceScope ts(TK_ADAMW, st);
  QL_CUDA_TRY(launch(adamw_kernel, dim3(grid), dim3(256), 0, st, 1, 1, p, g, m, v,
                     reinterpret_cast<__nv_bfloat16*>(p_bf16), n, k));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

// Moves a managed range to the current device (where == 0) or to host memory
// (where == 1) on the stream.  Memory that is not managed is rejected.
ql_status paged_prefetch(const void* ptr, size_t bytes, int where, cudaStream_t st) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeManaged) return QL_ERR_INVALID_ARG;
  int dev = 0;
  QL_CUDA_TRY(cudaGetDevice(&dev));
  QL_CUDA_TRY(cudaMemPrefetchAsync(ptr, bytes, where == 0 ? dev : cudaCpuDeviceId, st));
  return QL_OK;
}

}  // namespace ql
