// 4-bit float block formats: NVFP4 (E2M1 elements, E4M3 scale per 16, fp32
// tensor scale) and MXFP4 (E2M1 elements, E8M0 power-of-two scale per 32).
//
// "Lesson 4 of the Finetuning Sessions", "From FP32 to the 4-Bit Horizon":
// MXFP4 shares one 8-bit power-of-two (E8M0) scale over a block of 32; NVFP4
// shares one E4M3 scale over a block of 16, whose mantissa bits allow
// fractional scales.  "From Turing to Blackwell": the 5th-generation tensor
// cores execute these formats natively.
//
// Every scale step is one fp32 operation in a fixed order, so the kernels take
// the same integer decisions as a plain restatement of the definition:
//   NVFP4: s_t = fl32(amax_tensor / 2688) (or 1), denom = fl32(6 s_t),
//          S = E4M3(fl32(amax_b / denom)), scale = fl32(S s_t),
//          code = E2M1(fl32(x / scale)) (0 where scale == 0),
//          x_hat = fl32(E2M1(code) scale).
//   MXFP4: k = floor(log2 amax_b) - 2 clamped to [-127, 127] (-127 for an
//          all-zero block), code = E2M1(x 2^-k), x_hat = E2M1(code) 2^k.
// E2M1 rounding is nearest-even with saturation at +-6; -0 keeps its sign.
// Elements 2j and 2j+1 share byte j (low nibble first), as in NF4.
#include <algorithm>

#include "common.cuh"
#include "trace.cuh"

namespace ql {

// Two fp32 values -> one byte of two E2M1 codes (lo in the low nibble).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t out;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u16.u8 %0, t;\n}" : "=h"(out) : "f"(hi), "f"(lo));
  return out & 0xFFu;
}

// E2M1 code -> fp32 value (exact).
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  const float v = mag[c & 7u];
  return (c & 8u) ? -v : v;
}

template <typename T>
__device__ __forceinline__ void load8(const T* x, int64_t e0, int64_t n, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<float>(const float* x, int64_t e0, int64_t n, float (&v)[8]) {
  if (e0 + 8 <= n) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(x + e0));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(x + e0 + 4));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (e0 + i < n) ? x[e0 + i] : 0.0f;
  }
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* x, int64_t e0, int64_t n, float (&v)[8]) {
  if (e0 + 8 <= n) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x + e0));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[2 * i] = bf16_lo(w[i]); v[2 * i + 1] = bf16_hi(w[i]); }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (e0 + i < n) ? __bfloat162float(x[e0 + i]) : 0.0f;
  }
}

__device__ __forceinline__ uint32_t absmax_bits8(const float (&v)[8]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
  return m;
}

// Stores the packed codes of elements [e0, e0 + 8) (4 bytes), clipped to n.
__device__ __forceinline__ void store_codes8(uint8_t* codes, int64_t e0, int64_t n, uint32_t word) {
  if (e0 + 8 <= n) {
    *reinterpret_cast<uint32_t*>(codes + (e0 >> 1)) = word;
  } else if (e0 < n) {
    const int valid = (int)(n - e0);
    for (int b = 0; 2 * b < valid; ++b) {
      uint32_t byte = (word >> (8 * b)) & 0xFFu;
      if (2 * b + 1 >= valid) byte &= 0x0Fu;     // a missing high nibble is +0
      codes[(e0 >> 1) + b] = (uint8_t)byte;
    }
  }
}

// Pass 1 of NVFP4: the tensor's largest |x| as an integer max over the fp32
// bit patterns (monotone for non-negative floats; NaN patterns sort above Inf).
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const T* __restrict__ x, int64_t n, unsigned* amax_bits) {
  pdl_wait();
  pdl_trigger();
  uint32_t m = 0;
  const int64_t n8 = (n + 7) / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    float v[8];
    load8<T>(x, i * 8, n, v);
    m = max(m, absmax_bits8(v));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(amax_bits, m);
}

// Pass 2 of NVFP4: two threads per 16-block (8 elements each).  Whole warps
// iterate together so the shuffle joining a block's halves sees all lanes.
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_quant_kernel(const T* __restrict__ x, int64_t n,
                                                          const unsigned* __restrict__ amax_bits, int use_ts,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                          float* __restrict__ ts_out) {
  pdl_wait();
  pdl_trigger();
  const uint32_t abits = *amax_bits;
  if (abits >= 0x7F800000u) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(ST_NONFINITE);
    return;
  }
  const float amax_t = __uint_as_float(abits);
  const float s_t = (use_ts && amax_t > 0.0f) ? __fdiv_rn(amax_t, 2688.0f) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *ts_out = s_t;
  const float denom = __fmul_rn(6.0f, s_t);
  const int64_t n8 = (n + 7) / 8;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t wb = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32; wb < n8; wb += warps * 32) {
    const int64_t i = wb + lane;
    const int64_t e0 = i * 8;
    float v[8];
    if (e0 < n) {
      load8<T>(x, e0, n, v);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.0f;
    }
    uint32_t m = absmax_bits8(v);
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    const uint8_t sc = f32_to_e4m3(__fdiv_rn(__uint_as_float(m), denom));
    const float scale = __fmul_rn(e4m3_to_f32(sc), s_t);
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float y0 = 0.0f, y1 = 0.0f;
      if (scale > 0.0f) {
        y0 = __fdiv_rn(v[2 * k], scale);
        y1 = __fdiv_rn(v[2 * k + 1], scale);
      }
      word |= e2m1x2(y0, y1) << (8 * k);
    }
    store_codes8(codes, e0, n, word);
    if ((i & 1) == 0 && e0 < n) scales[e0 >> 4] = sc;
  }
}

// MXFP4: four threads per 32-block (8 elements each); one pass.
template <typename T>
__global__ void __launch_bounds__(256) mxfp4_quant_kernel(const T* __restrict__ x, int64_t n,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int64_t n8 = (n + 7) / 8;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t wb = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32; wb < n8; wb += warps * 32) {
    const int64_t i = wb + lane;
    const int64_t e0 = i * 8;
    float v[8];
    if (e0 < n) {
      load8<T>(x, e0, n, v);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.0f;
    }
    uint32_t m = absmax_bits8(v);
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
    if (m >= 0x7F800000u) {
      if ((i & 3) == 0 && e0 < n) raise_status(ST_NONFINITE);
      m = 0;
    }
    // floor(log2 amax): the biased exponent for a normal amax, the position of
    // the leading one for a subnormal one
    int fl;
    if (m == 0) fl = -1000;
    else if (m >= 0x00800000u) fl = (int)(m >> 23) - 127;
    else fl = (31 - __clz((int)m)) - 149;
    const int k = m == 0 ? -127 : max(-127, min(127, fl - 2));
    // 2^-k as an fp32 (|k| <= 127, so it is a normal number); y = x 2^-k is
    // exact unless it falls below 2^-126, where it codes as (signed) zero anyway
    const float inv = __uint_as_float((uint32_t)(127 - k) << 23);
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) word |= e2m1x2(__fmul_rn(v[2 * q], inv), __fmul_rn(v[2 * q + 1], inv)) << (8 * q);
    store_codes8(codes, e0, n, word);
    if ((i & 3) == 0 && e0 < n) scales[e0 >> 5] = (uint8_t)(k + 127);
  }
}

// Dequantization to fp32: NVFP4 (fmt 0) x_hat = fl32(E2M1 fl32(S s_t));
// MXFP4 (fmt 1) x_hat = E2M1 2^k.  One thread per byte (two elements).
__global__ void __launch_bounds__(256) fp4_dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ scales,
                                                          const float* __restrict__ ts, int64_t n, int fmt,
                                                          float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const float s_t = fmt == 0 ? *ts : 1.0f;
  const int64_t nbytes = (n + 1) / 2;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < nbytes; j += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t byte = codes[j];
    const int64_t e = 2 * j;
    float scale;
    if (fmt == 0) {
      scale = __fmul_rn(e4m3_to_f32(scales[e >> 4]), s_t);
    } else {
      const int k = (int)scales[e >> 5] - 127;
      scale = k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << 22);   // 2^-127
    }
    out[e] = __fmul_rn(e2m1_value(byte & 15u), scale);
    if (e + 1 < n) out[e + 1] = __fmul_rn(e2m1_value(byte >> 4), scale);
  }
}

static int sm_count_fp4() {
  const int c = device_sm_count();
  return c > 0 ? c : 148;
}

static unsigned fp4_grid(int64_t items) {
  const int64_t need = (items + 255) / 256;
  const int64_t cap = (int64_t)sm_count_fp4() * 8;
  return (unsigned)std::max<int64_t>(1, std::min(need, cap));
}

ql_status launch_nvfp4_quantize(const void* x, ql_dtype dt, int64_t n, int use_ts, uint8_t* codes, uint8_t* scales,
                                float* ts, void* ws, cudaStream_t st) {
  unsigned* amax = reinterpret_cast<unsigned*>(ws);
  const unsigned grid = fp4_grid((n + 7) / 8);
  TraceScope t(TK_FP4, st);
  QL_CUDA_TRY(cudaMemsetAsync(amax, 0, sizeof(unsigned), st));
  if (dt == QL_F32) {
    QL_CUDA_TRY(launch(nvfp4_amax_kernel<float>, dim3(grid), dim3(256), 0, st, 1, 1, (const float*)x, n, amax));
    QL_CUDA_TRY(launch(nvfp4_quant_kernel<float>, dim3(grid), dim3(256), 0, st, 1, 1, (const float*)x, n,
                       (const unsigned*)amax, use_ts, codes, scales, ts));
  } else {
    const __nv_bfloat16* xb = (const __nv_bfloat16*)x;
    QL_CUDA_TRY(launch(nvfp4_amax_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 1, 1, xb, n, amax));
    QL_CUDA_TRY(launch(nvfp4_quant_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 1, 1, xb, n,
                       (const unsigned*)amax, use_ts, codes, scales, ts));
  }
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_mxfp4_quantize(const void* x, ql_dtype dt, int64_t n, uint8_t* codes, uint8_t* scales,
                                cudaStream_t st) {
  const unsigned grid = fp4_grid((n + 7) / 8);
  TraceScope t(TK_FP4, st);
  if (dt == QL_F32)
    QL_CUDA_TRY(launch(mxfp4_quant_kernel<float>, dim3(grid), dim3(256), 0, st, 1, 1, (const float*)x, n, codes,
                       scales));
  else
    QL_CUDA_TRY(launch(mxfp4_quant_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 1, 1,
                       (const __nv_bfloat16*)x, n, codes, scales));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_fp4_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts, int64_t n, int fmt,
                             float* out, cudaStream_t st) {
  TraceScope t(TK_FP4, st);
  QL_CUDA_TRY(launch(fp4_dequant_kernel, dim3(fp4_grid((n + 1) / 2)), dim3(256), 0, st, 1, 1, codes, scales, ts, n,
                     fmt, out));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

QL_DEFINE_STATUS_ACCESSOR(status_word_fp4)

}  // namespace ql
