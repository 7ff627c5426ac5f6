// Elementwise glue of the SiLU-gated MLP built from three QLoRA linears.  The
// pages adapt every linear layer of the block ("QLoRA — Fine-Tuning a 65B Model
// on One GPU", "Seeing it in code": gate_proj, up_proj, down_proj); the block
// itself is the usual gated MLP  h = silu(g) * u,  silu(x) = x * sigmoid(x).
// Both kernels stream bf16 vectors with 16-byte accesses (HBM-bound) and
// compute in fp32.
#include "common.cuh"
#include "trace.cuh"

namespace ql {

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

__global__ void __launch_bounds__(256) silu_gate_fwd_kernel(const uint4* __restrict__ g, const uint4* __restrict__ u,
                                                            uint4* __restrict__ h, int64_t n8) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 gv = g[i], uv = u[i];
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float g0 = bf16_lo(gw[q]), g1 = bf16_hi(gw[q]);
      o[q] = pack_bf16x2(g0 * sigmoidf_(g0) * bf16_lo(uw[q]), g1 * sigmoidf_(g1) * bf16_hi(uw[q]));
    }
    h[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__global__ void __launch_bounds__(256) silu_gate_bwd_kernel(const uint4* __restrict__ dh, const uint4* __restrict__ g,
                                                            const uint4* __restrict__ u, uint4* __restrict__ dg,
                                                            uint4* __restrict__ du, int64_t n8) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 dv = dh[i], gv = g[i], uv = u[i];
    const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float r_g[2], r_u[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float d = h2 ? bf16_hi(dw[q]) : bf16_lo(dw[q]);
        const float x = h2 ? bf16_hi(gw[q]) : bf16_lo(gw[q]);
        const float y = h2 ? bf16_hi(uw[q]) : bf16_lo(uw[q]);
        const float sg = sigmoidf_(x);
        r_g[h2] = d * y * sg * (1.0f + x * (1.0f - sg));
        r_u[h2] = d * x * sg;
      }
      og[q] = pack_bf16x2(r_g[0], r_g[1]);
      ou[q] = pack_bf16x2(r_u[0], r_u[1]);
    }
    dg[i] = make_uint4(og[0], og[1], og[2], og[3]);
    du[i] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  }
}

static unsigned elem_grid(int64_t n8) {
  const int c = device_sm_count();
  const int sms = c > 0 ? c : 148;
  int64_t need = (n8 + 255) / 256;
  int64_t cap = (int64_t)sms * 8;
  return (unsigned)(need < 1 ? 1 : (need < cap ? need : cap));
}

ql_status launch_silu_gate_fwd(const void* g, const void* u, void* h, int64_t n, cudaStream_t st) {
  if (n % 8) return QL_ERR_UNSUPPORTED;
  const int64_t n8 = n / 8;
  TraceScope ts(TK_SILU, st);
  QL_CUDA_TRY(launch(silu_gate_fwd_kernel, dim3(elem_grid(n8)), dim3(256), 0, st, 1, 1, (const uint4*)g, (const uint4*)u, (uint4*)h, n8));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_silu_gate_bwd(const void* dh, const void* g, const void* u, void* dg, void* du, int64_t n,
                               cudaStream_t st) {
  if (n % 8) return QL_ERR_UNSUPPORTED;
  const int64_t n8 = n / 8;
  TraceScope ts(TK_SILU, st);
  QL_CUDA_TRY(launch(silu_gate_bwd_kernel, dim3(elem_grid(n8)), dim3(256), 0, st, 1, 1, (const uint4*)dh, (const uint4*)g, (const uint4*)u,
                                                      (uint4*)dg, (uint4*)du, n8));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

}  // namespace ql
