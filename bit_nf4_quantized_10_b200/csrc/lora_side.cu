// Rank-r side products of the QLoRA linear (the adapter branch and its
// gradients), "QLoRA — Fine-Tuning a 65B Model on One GPU", "Prerequisite:
// LoRA's low-rank update" and "Where the gradients actually go":
//   U  = bf16(X  A^T)   [M, r]   forward, saved for the backward
//   V  = bf16(dY B)     [M, r]   backward
//   dB = s dY^T U       [N, r]   backward (reduction over tokens)
//   dA = s V^T X        [r, K]   backward (reduction over tokens)
// These read one activation matrix once and touch r <= 64 columns, so they are
// bound by HBM traffic on X or dY, not by arithmetic.
//
// rowproj: one warp per token row; lanes stride the row 8 elements at a time
// and keep r fp32 partial sums, reduced across the warp at the end.
// colacc: each thread owns 64/R consecutive columns of the activation and keeps
// their R fp32 sums over a slice of tokens (slices split over CTAs); the
// per-slice partials are then added in a fixed slice order, so the result does
// not depend on scheduling.
#include <algorithm>

#include "common.cuh"
#include "trace.cuh"

namespace ql {

// P(j, k) accessor: A is [r, K] (k contiguous); B is [N, r] used as P(j, n) = B[n, j].
template <int R, bool P_IS_ROWMAJOR_R_BY_K>
__global__ void __launch_bounds__(256) rowproj_kernel(const __nv_bfloat16* __restrict__ act, int64_t M, int Kd,
                                                      const __nv_bfloat16* __restrict__ P, int r,
                                                      __nv_bfloat16* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t m = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M; m += warps) {
    float acc[R];
#pragma unroll
    for (int j = 0; j < R; ++j) acc[j] = 0.0f;
    const __nv_bfloat16* row = act + m * (int64_t)Kd;
    for (int k = lane * 8; k < Kd; k += 256) {
      const uint4 xv = *reinterpret_cast<const uint4*>(row + k);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
      float x[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) { x[2 * i] = bf16_lo(xw[i]); x[2 * i + 1] = bf16_hi(xw[i]); }
      if (P_IS_ROWMAJOR_R_BY_K) {
#pragma unroll
        for (int j = 0; j < R; ++j) {
          if (j < r) {
            const uint4 pv = __ldg(reinterpret_cast<const uint4*>(P + (int64_t)j * Kd + k));
            const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[j] = fmaf(x[2 * i], bf16_lo(pw[i]), acc[j]);
              acc[j] = fmaf(x[2 * i + 1], bf16_hi(pw[i]), acc[j]);
            }
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const __nv_bfloat16* prow = P + (int64_t)(k + i) * r;
#pragma unroll
          for (int jj = 0; jj < R; jj += 8) {
            if (jj < r) {
              const uint4 pv = __ldg(reinterpret_cast<const uint4*>(prow + jj));
              const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                acc[jj + 2 * q] = fmaf(x[i], bf16_lo(pw[q]), acc[jj + 2 * q]);
                acc[jj + 2 * q + 1] = fmaf(x[i], bf16_hi(pw[q]), acc[jj + 2 * q + 1]);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < R; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < R; j += 2)
        if (j < r) *reinterpret_cast<uint32_t*>(out + m * r + j) = pack_bf16x2(acc[j], acc[j + 1]);
    }
  }
}

// partial[slice][col][j] = sum over tokens of the slice of act[m, col] * G[m, j].
// Each thread owns CPT = 64 / R consecutive columns (64 fp32 sums per thread).
template <int R>
__global__ void __launch_bounds__(256) colacc_kernel(const __nv_bfloat16* __restrict__ act, int64_t M, int ncols,
                                                     const __nv_bfloat16* __restrict__ G, int r,
                                                     int64_t tokens_per_slice, float* __restrict__ partial) {
  constexpr int CPT = 64 / R;
  __shared__ float gs[32][R];
  const int slice = blockIdx.y;
  const int64_t t0 = (int64_t)slice * tokens_per_slice;
  const int64_t t1 = min(M, t0 + tokens_per_slice);
  const int col = (blockIdx.x * blockDim.x + threadIdx.x) * CPT;
  float acc[CPT][R];
#pragma unroll
  for (int c = 0; c < CPT; ++c)
#pragma unroll
    for (int j = 0; j < R; ++j) acc[c][j] = 0.0f;
  for (int64_t tb = t0; tb < t1; tb += 32) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 32 * R; idx += blockDim.x) {
      const int tt = idx / R, j = idx % R;
      const int64_t m = tb + tt;
      gs[tt][j] = (m < t1 && j < r) ? __bfloat162float(G[m * r + j]) : 0.0f;
    }
    __syncthreads();
    const int nt = (int)min((int64_t)32, t1 - tb);
    for (int tt = 0; tt < nt; ++tt) {
      float a[CPT];
      const __nv_bfloat16* src = act + (tb + tt) * (int64_t)ncols + col;
      if (col < ncols) {
        if (CPT == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          a[0] = bf16_lo(v.x); a[1 % CPT] = bf16_hi(v.x); a[2 % CPT] = bf16_lo(v.y); a[3 % CPT] = bf16_hi(v.y);
        } else if (CPT == 2) {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
          a[0] = bf16_lo(v); a[1 % CPT] = bf16_hi(v);
        } else {
          a[0] = __bfloat162float(*src);
        }
      } else {
#pragma unroll
        for (int c = 0; c < CPT; ++c) a[c] = 0.0f;
      }
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const float g = gs[tt][j];
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c][j] = fmaf(a[c], g, acc[c][j]);
      }
    }
  }
  if (col < ncols) {
    float* dst = partial + ((int64_t)slice * ncols + col) * R;
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
      for (int j = 0; j < R; ++j) dst[c * R + j] = acc[c][j];
  }
}

// out = s * sum_slices partial, in slice order.  out_t: [ncols, r] when
// !transpose, [r, ncols] when transpose.
template <int R>
__global__ void __launch_bounds__(256) colacc_reduce_kernel(const float* __restrict__ partial, int slices,
                                                            int ncols, int r, float s, int transpose,
                                                            int out_bf16, void* __restrict__ out) {
  const int64_t total = (int64_t)ncols * r;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t col = idx / r;
    const int j = (int)(idx % r);
    float acc = 0.0f;
    for (int sl = 0; sl < slices; ++sl) acc += partial[((int64_t)sl * ncols + col) * R + j];
    const float v = __fmul_rn(s, acc);
    const int64_t o = transpose ? (int64_t)j * ncols + col : col * r + j;
    if (out_bf16) reinterpret_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(out)[o] = v;
  }
}

static int sm_count_side() {
  static int count = 0;
  if (!count) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
    if (count <= 0) count = 148;
  }
  return count;
}

template <bool ROWMAJOR>
static ql_status rowproj_dispatch(const void* act, int64_t M, int Kd, const void* P, int r, void* out,
                                  cudaStream_t st) {
  int64_t warps_needed = M;
  int64_t ctas = (warps_needed + 7) / 8;
  int64_t cap = (int64_t)sm_count_side() * 8;
  unsigned grid = (unsigned)(ctas < cap ? (ctas < 1 ? 1 : ctas) : cap);
  auto a = (const __nv_bfloat16*)act;
  auto pp = (const __nv_bfloat16*)P;
  auto o = (__nv_bfloat16*)out;
  TraceScope ts(TK_PROJ, st);
  if (r <= 16) rowproj_kernel<16, ROWMAJOR><<<grid, 256, 0, st>>>(a, M, Kd, pp, r, o);
  else if (r <= 32) rowproj_kernel<32, ROWMAJOR><<<grid, 256, 0, st>>>(a, M, Kd, pp, r, o);
  else rowproj_kernel<64, ROWMAJOR><<<grid, 256, 0, st>>>(a, M, Kd, pp, r, o);
  QL_LAUNCH_CHECK();
  return QL_OK;
}

// U = bf16(X A^T): X [M, K], A [r, K]
ql_status launch_proj_xa(const void* X, int64_t M, int K, const void* A, int r, void* U, cudaStream_t st) {
  return rowproj_dispatch<true>(X, M, K, A, r, U, st);
}

// V = bf16(dY B): dY [M, N], B [N, r]
ql_status launch_proj_dyb(const void* dY, int64_t M, int N, const void* B, int r, void* V, cudaStream_t st) {
  return rowproj_dispatch<false>(dY, M, N, B, r, V, st);
}

int colacc_slices(int64_t M) {
  int64_t s = (M + 255) / 256;
  if (s > 32) s = 32;
  if (s < 1) s = 1;
  return (int)s;
}

size_t colacc_partial_bytes(int64_t M, int64_t ncols, int r) {
  const int R = r <= 16 ? 16 : (r <= 32 ? 32 : 64);
  return (size_t)colacc_slices(M) * (size_t)ncols * R * sizeof(float);
}

// out = s * act^T G : act [M, ncols], G [M, r].  transpose=0: out [ncols, r]
// (dB); transpose=1: out [r, ncols] (dA).
ql_status launch_colacc(const void* act, int64_t M, int ncols, const void* G, int r, float s, int transpose,
                        void* out, ql_dtype out_dt, float* partial, cudaStream_t st) {
  const int slices = colacc_slices(M);
  const int64_t per = (M + slices - 1) / slices;
  const int R = r <= 16 ? 16 : (r <= 32 ? 32 : 64);
  const int cpt = 64 / R;
  dim3 grid((unsigned)((ncols / cpt + 255) / 256), (unsigned)slices);
  auto a = (const __nv_bfloat16*)act;
  auto g = (const __nv_bfloat16*)G;
  const int ob = out_dt == QL_BF16;
  const int64_t total = (int64_t)ncols * r;
  unsigned rgrid = (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count_side() * 8);
  if (r <= 16) {
    { TraceScope ts(TK_COLACC, st); colacc_kernel<16><<<grid, 256, 0, st>>>(a, M, ncols, g, r, per, partial); }
    { TraceScope ts(TK_COLACC_REDUCE, st);
      colacc_reduce_kernel<16><<<rgrid, 256, 0, st>>>(partial, slices, ncols, r, s, transpose, ob, out); }
  } else if (r <= 32) {
    { TraceScope ts(TK_COLACC, st); colacc_kernel<32><<<grid, 256, 0, st>>>(a, M, ncols, g, r, per, partial); }
    { TraceScope ts(TK_COLACC_REDUCE, st);
      colacc_reduce_kernel<32><<<rgrid, 256, 0, st>>>(partial, slices, ncols, r, s, transpose, ob, out); }
  } else {
    { TraceScope ts(TK_COLACC, st); colacc_kernel<64><<<grid, 256, 0, st>>>(a, M, ncols, g, r, per, partial); }
    { TraceScope ts(TK_COLACC_REDUCE, st);
      colacc_reduce_kernel<64><<<rgrid, 256, 0, st>>>(partial, slices, ncols, r, s, transpose, ob, out); }
  }
  QL_LAUNCH_CHECK();
  return QL_OK;
}

}  // namespace ql
