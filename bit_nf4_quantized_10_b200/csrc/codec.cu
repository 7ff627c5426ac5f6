// NF4 codec kernels: blockwise quantize + pack, double quantization of the
// block constants, and standalone dequantization.
//
// "QLoRA — Fine-Tuning a 65B Model on One GPU", "Quantization in one
// paragraph": c = max|x| per block of 64, store the index of the nearest
// level, x_hat = c * q_index.  "QLoRA: Quantize Base Weights to 4-Bit", §2.2:
// the fp32 constants are grouped by 256 and stored as 8-bit floats with one
// fp32 second-level constant; "Double quantization: the constants are not
// free" (same page 3): the mean is subtracted first.
//
// All kernels are HBM-bound streaming passes.  Loads and stores are 16 bytes
// wide, grids are sized to a multiple of the SM count and loop grid-stride,
// and every index is 64-bit so tensors above 2^32 elements work.
#include <algorithm>

#include "common.cuh"
#include "trace.cuh"

namespace ql {

QL_DEFINE_STATUS_ACCESSOR(status_word_codec)

// ---------------------------------------------------------------- quantize
// Code of x: #{j : x > t_j} over the 15 sorted thresholds t_j = fl32(m_j c)
// (ties go to the lower level).  The search goes through y = x/c, but only to
// pick a candidate: the 33 bins round(16 y + 16) are 1/16 wide, narrower than
// the closest two midpoints (0.093 apart), so each bin (widened by 1e-5 on both
// sides, far more than the rounding of y) holds at most one threshold j.  The
// bin table gives j and the count of thresholds below the bin; one exact
// comparison x > fl32(m_j c) then settles the code.  Bins with no threshold
// carry m = 4, which no |x| <= c exceeds.
struct QuantBins {
  float m[64];
  uint32_t base[64];
};

QuantBins build_bins(const NF4Table& t) {
  QuantBins b{};
  for (int k = 0; k < 64; ++k) {
    b.m[k] = 4.0f;
    b.base[k] = 0;
    if (k > 32) continue;   // reachable only from a NaN y
    const double lo = (k - 16.5) / 16.0 - 1e-5, hi = (k - 15.5) / 16.0 + 1e-5;
    uint32_t below = 0;
    for (int j = 0; j < 15; ++j) {
      if ((double)t.m[j] < lo) ++below;
      else if ((double)t.m[j] <= hi) b.m[k] = t.m[j];
    }
    b.base[k] = below;
  }
  return b;
}

// The eight codes of v (elements 0..7 in nibbles 0..7) given the block's
// absmax c.  `bins` is the QuantBins table in shared memory as (m bits, count
// below) pairs.
__device__ __forceinline__ uint32_t encode8(const float (&v)[8], float c, const uint2* bins, const NF4Table& tab) {
  uint32_t word = 0;
  if (c >= 1e-30f) {
    // 16/c: c >= 1e-30 keeps it finite; its rounding moves y by < 1e-6
    const float s16 = __fmul_rn(16.0f, __frcp_rn(c));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // 1.5 * 2^23 + 16: the sum's low bits are round(16 y + 16), in 0..32
      const float t = __fmaf_rn(v[i], s16, 12582928.0f);
      const uint2 e = bins[__float_as_uint(t) & 63u];
      const float th = __fmul_rn(__uint_as_float(e.x), c);
      word |= (e.y + (v[i] > th ? 1u : 0u)) << (4 * i);
    }
  } else {
    // tiny (or NaN) absmax: count the thresholds directly
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t k = 0;
#pragma unroll
      for (int j = 0; j < 15; ++j) k += (v[i] > __fmul_rn(tab.m[j], c)) ? 1u : 0u;
      word |= k << (4 * i);
    }
  }
  if (c == 0.0f) word = 0x88888888u;
  return word;
}

// Eight consecutive elements as loaded (raw words), and as fp32 values.
template <typename T>
struct Raw8;
template <>
struct Raw8<float> {
  uint32_t w[8];
};
template <>
struct Raw8<__nv_bfloat16> {
  uint32_t w[4];
};

template <typename T>
__device__ __forceinline__ void load8(const T* x, int64_t e0, int64_t n, Raw8<T>& r);

template <>
__device__ __forceinline__ void load8<float>(const float* x, int64_t e0, int64_t n, Raw8<float>& r) {
  if (e0 + 8 <= n) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x + e0));
    const uint4 b = __ldcs(reinterpret_cast<const uint4*>(x + e0) + 1);
    r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
    r.w[4] = b.x; r.w[5] = b.y; r.w[6] = b.z; r.w[7] = b.w;
  } else {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(x);
#pragma unroll
    for (int i = 0; i < 8; ++i) r.w[i] = (e0 + i < n) ? u[e0 + i] : 0u;
  }
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* x, int64_t e0, int64_t n,
                                                     Raw8<__nv_bfloat16>& r) {
  if (e0 + 8 <= n) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x + e0));
    r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
  } else {
    const uint16_t* u = reinterpret_cast<const uint16_t*>(x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (e0 + 2 * i < n) ? u[e0 + 2 * i] : 0u;
      const uint32_t hi = (e0 + 2 * i + 1 < n) ? u[e0 + 2 * i + 1] : 0u;
      r.w[i] = lo | (hi << 16);
    }
  }
}

__device__ __forceinline__ void unpack8(const Raw8<float>& r, float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r.w[i]);
}
__device__ __forceinline__ void unpack8(const Raw8<__nv_bfloat16>& r, float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = bf16_lo(r.w[i]);
    v[2 * i + 1] = bf16_hi(r.w[i]);
  }
}

// The largest |x| bit pattern of eight elements, as fp32 bits: for bf16 input
// the maximum is taken on the packed halves (the sign bits cleared, two 16-bit
// maxima per instruction) before unpacking.
__device__ __forceinline__ uint32_t raw_absmax_bits(const Raw8<float>& r) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = max(m, r.w[i] & 0x7FFFFFFFu);
  return m;
}
__device__ __forceinline__ uint32_t raw_absmax_bits(const Raw8<__nv_bfloat16>& r) {
  uint32_t m = __vmaxu2(r.w[0] & 0x7FFF7FFFu, r.w[1] & 0x7FFF7FFFu);
  m = __vmaxu2(m, __vmaxu2(r.w[2] & 0x7FFF7FFFu, r.w[3] & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16) << 16;
}

// 8 threads per 64-block, 8 consecutive elements per thread.  The loop runs
// over blocks, so the 8 threads of a block always iterate together and can
// reduce the absmax with shuffles.  The absmax is the integer maximum of the
// |x| bit patterns (the same order as the values), which also flags NaN and
// Inf: their patterns are the largest.
template <typename T>
__global__ void __launch_bounds__(256) quantize_kernel(const T* __restrict__ x, int64_t n,
                                                       uint8_t* __restrict__ codes,
                                                       float* __restrict__ absmax, NF4Table tab, QuantBins bins_in) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint2 bins[64];   // (m bits, count below)
  if (threadIdx.x < 64) bins[threadIdx.x] = make_uint2(__float_as_uint(bins_in.m[threadIdx.x]), bins_in.base[threadIdx.x]);
  __syncthreads();
  const int64_t nb = (n + 63) / 64;
  const int lane8 = threadIdx.x & 7;
  const int wib = threadIdx.x >> 5;              // warp in CTA
  const int bq = (threadIdx.x >> 3) & 3;         // block within the warp's four
  // the whole warp (4 blocks) iterates together so the shuffles see all lanes
  const int64_t warps_per_grid = (int64_t)gridDim.x * (blockDim.x >> 5);
  // the next iteration's eight elements are loaded (as raw words) while this
  // one is coded
  int64_t wb = ((int64_t)blockIdx.x * (blockDim.x >> 5) + wib) * 4;
  Raw8<T> nxt;
  if (wb < nb) load8<T>(x, (wb + bq) * 64 + lane8 * 8, n, nxt);
  for (; wb < nb; wb += warps_per_grid * 4) {
    const int64_t b = wb + bq;
    const int64_t e0 = b * 64 + lane8 * 8;   // >= n for a block past the end
    float v[8];
    const uint32_t abits0 = raw_absmax_bits(nxt);
    unpack8(nxt, v);
    if (wb + warps_per_grid * 4 < nb) load8<T>(x, (wb + warps_per_grid * 4 + bq) * 64 + lane8 * 8, n, nxt);
    uint32_t abits = abits0;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) abits = max(abits, __shfl_xor_sync(0xffffffffu, abits, o));
    if (abits >= 0x7F800000u && lane8 == 0 && b < nb) raise_status(ST_NONFINITE);
    const float c = __uint_as_float(abits);
    const uint32_t word = encode8(v, c, bins, tab);
    if (e0 + 8 <= n) {
      __stcs(reinterpret_cast<uint32_t*>(codes + (e0 >> 1)), word);
    } else if (e0 < n) {
      const int valid = (int)(n - e0);          // 1..7
      for (int i = 0; i < valid; i += 2) {
        uint32_t lo = (word >> (4 * i)) & 0xFu;
        uint32_t hi = (i + 1 < valid) ? ((word >> (4 * (i + 1))) & 0xFu) : 8u;
        codes[(e0 + i) >> 1] = (uint8_t)(lo | (hi << 4));
      }
    }
    if (lane8 == 0 && b < nb) absmax[b] = c;
  }
}

// --------------------------------------------------------- double quant: mean
// Fixed adjacent-pair tree in float64.  One CTA sums 2048 consecutive inputs
// (zero beyond `count`): 8 per thread as a 3-level tree, then the xor-shuffle
// butterfly (offsets 1..16 combine adjacent subtrees), then the 8 warp sums as
// a 3-level tree.  Every CTA's result is one node of the global tree, so
// repeating the pass on the partials reproduces the whole tree.
template <typename T>
__global__ void __launch_bounds__(256) tree_sum_pass(const T* __restrict__ in, int64_t count,
                                                     double* __restrict__ out, int64_t total_nb,
                                                     float* __restrict__ mean_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ double warp_sums[8];
  const int64_t base = (int64_t)blockIdx.x * 2048 + threadIdx.x * 8;
  double v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = (base + i < count) ? (double)in[base + i] : 0.0;
  double s = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) s = s + __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    const double* w = warp_sums;
    double tot = ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
    out[blockIdx.x] = tot;
    if (mean_out) *mean_out = __double2float_rn(__ddiv_rn(tot, (double)total_nb));
  }
}

// ------------------------------------------------------- double quant: codes
// One warp per group of 256 constants, 8 per lane.
__global__ void __launch_bounds__(256) dq_encode_kernel(const float* __restrict__ absmax, int64_t nb,
                                                        const float* __restrict__ mean,
                                                        uint8_t* __restrict__ absmax_q,
                                                        float* __restrict__ scale2) {
  pdl_wait();
  pdl_trigger();
  const int64_t ng = (nb + 255) / 256;
  const int lane = threadIdx.x & 31;
  const float mu = *mean;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < ng; g += warps) {
    const int64_t b0 = g * 256 + lane * 8;
    float d[8];
    float dmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      d[i] = (b0 + i < nb) ? __fsub_rn(absmax[b0 + i], mu) : 0.0f;
      dmax = fmaxf(dmax, fabsf(d[i]));
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
    const float s2 = __fdiv_rn(dmax, 448.0f);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t e = (s2 != 0.0f) ? f32_to_e4m3(__fdiv_rn(d[i], s2)) : 0u;
      if (i < 4) lo |= e << (8 * i); else hi |= e << (8 * (i - 4));
    }
    if (b0 + 8 <= nb) {
      *reinterpret_cast<uint2*>(absmax_q + b0) = make_uint2(lo, hi);
    } else {
      for (int i = 0; i < 8; ++i)
        if (b0 + i < nb) absmax_q[b0 + i] = (uint8_t)(((i < 4 ? lo : hi) >> (8 * (i & 3))) & 0xFF);
    }
    if (lane == 0) scale2[g] = s2;
  }
}

// --------------------------------------------------------------- dequantize
// bf16 output: one thread per 64-block.  The block's 16 results
// bf16(fl32(q_j * c)) are built once into a register byte-plane table and
// looked up with prmt.
__global__ void __launch_bounds__(256) dequant_bf16_kernel(const uint8_t* __restrict__ codes, WeightConsts wc,
                                                           int64_t n, __nv_bfloat16* __restrict__ out,
                                                           NF4Table tab) {
  pdl_wait();
  pdl_trigger();
  const int64_t nb = (n + 63) / 64;
  const float mu = wc.absmax ? 0.0f : *wc.offset;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb; b += stride) {
    const float c = block_const(wc, b, mu);
    const Lut16 L = make_lut(tab, c);
    const int64_t e0 = b * 64;
    if (e0 + 64 <= n) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + (e0 >> 1));
      uint4 c0 = __ldcs(src), c1 = __ldcs(src + 1);
      uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint4* dst = reinterpret_cast<uint4*>(out + e0);
#pragma unroll
      for (int i = 0; i < 8; ++i) __stcs(dst + i, lut_lookup8(L, w[i]));
    } else {
      for (int64_t e = e0; e < n; ++e) {
        uint32_t byte = codes[e >> 1];
        uint32_t code = (e & 1) ? (byte >> 4) : (byte & 0xF);
        out[e] = __float2bfloat16_rn(__fmul_rn(tab.q[code], c));
      }
    }
  }
}

// fp32 output: 8 elements per thread, the 16 levels read from shared memory.
__global__ void __launch_bounds__(256) dequant_f32_kernel(const uint8_t* __restrict__ codes, WeightConsts wc,
                                                          int64_t n, float* __restrict__ out, NF4Table tab) {
  pdl_wait();
  pdl_trigger();
  __shared__ float q[16];
  if (threadIdx.x < 16) q[threadIdx.x] = tab.q[threadIdx.x];
  __syncthreads();
  const float mu = wc.absmax ? 0.0f : *wc.offset;
  const int64_t nchunks = (n + 7) / 8;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < nchunks; k += stride) {
    const int64_t e0 = k * 8;
    const float c = block_const(wc, e0 >> 6, mu);
    if (e0 + 8 <= n) {
      uint32_t w = __ldcs(reinterpret_cast<const uint32_t*>(codes + (e0 >> 1)));
      float r[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = __fmul_rn(q[(w >> (4 * i)) & 0xF], c);
      float4* dst = reinterpret_cast<float4*>(out + e0);
      __stcs(dst, make_float4(r[0], r[1], r[2], r[3]));
      __stcs(dst + 1, make_float4(r[4], r[5], r[6], r[7]));
    } else {
      for (int64_t e = e0; e < n; ++e) {
        uint32_t byte = codes[e >> 1];
        uint32_t code = (e & 1) ? (byte >> 4) : (byte & 0xF);
        out[e] = __fmul_rn(q[code], c);
      }
    }
  }
}

// ------------------------------------------------------------ adapter merge
// W' = bf16(fl32(w_hat + fl32(s d))), d = sum over j = 0 .. r-1 in order of
// B[n, j] A[j, k] in fp32 ("QLoRA: Quantize Base Weights to 4-Bit", FAQ on
// inference latency: W = W_dequant + (alpha / r) B A in 16 bits; "QLoRA —
// Fine-Tuning a 65B Model on One GPU", "Pitfalls": merge in 16 bits, then
// quantize the merged weight if a quantized model is wanted).  A product of two
// bf16 values is exact in fp32, so each fma is the rounded fp32 sum.
// Optionally the merged values are quantized again (same code selection as
// quantize_kernel), without a round trip of the bf16 weight through HBM.
// The rank-r product d = B A is a small matrix product, so each thread owns a
// register tile of 8 rows x 8 consecutive columns of a 64-row x 256-column CTA
// tile and accumulates its 64 sums with packed fp32 FMAs (two independent
// IEEE fmas per instruction, j in order), reading A (as fp32) and B (as
// broadcast pairs) from shared memory staged once per tile: every A and B
// value is reused by 8 rows or 8 columns.  The 8 threads holding a row's
// 64-block are 8 consecutive lanes, so the re-quantization's absmax is the same
// 8-lane shuffle as in quantize_kernel.  K % 64 == 0, so a block lies in one
// row and a tile edge never splits one.
constexpr int MG_ROWS = 64;     // rows per CTA tile: 8 warps x 8 rows
constexpr int MG_COLS = 256;    // columns per CTA tile: 32 lanes x 8 columns

__device__ __forceinline__ void fma2_rn(float2& d, float2 a, float2 b) {
  asm("{\n .reg .b64 x, y, z;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n mov.b64 z, {%0, %1};\n"
      " fma.rn.f32x2 z, x, y, z;\n mov.b64 {%0, %1}, z;\n}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
}

__global__ void __launch_bounds__(256, 2) merge_kernel(const uint8_t* __restrict__ codes, WeightConsts wc, int64_t N,
                                                    int64_t K, const __nv_bfloat16* __restrict__ A,
                                                    const __nv_bfloat16* __restrict__ B, int r, float s,
                                                    __nv_bfloat16* __restrict__ out, uint8_t* __restrict__ codes_out,
                                                    float* __restrict__ absmax_out, NF4Table tab, QuantBins bins_in) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint2 bins[64];
  __shared__ float q[16];
  extern __shared__ __align__(16) float mg_smem[];
  float* a_s = mg_smem;                                               // [r][256] fp32
  float2* b_s = reinterpret_cast<float2*>(mg_smem + (size_t)r * MG_COLS);   // [r][64] (b, b)
  if (threadIdx.x < 64) bins[threadIdx.x] = make_uint2(__float_as_uint(bins_in.m[threadIdx.x]), bins_in.base[threadIdx.x]);
  if (threadIdx.x < 16) q[threadIdx.x] = tab.q[threadIdx.x];
  const float mu = wc.absmax ? 0.0f : *wc.offset;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int lane8 = tx & 7;
  const int64_t kb = K / 64;
  const int64_t tiles_c = (K + MG_COLS - 1) / MG_COLS;
  const int64_t tiles = (N + MG_ROWS - 1) / MG_ROWS * tiles_c;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int64_t r0 = tile / tiles_c * MG_ROWS, c0 = tile % tiles_c * MG_COLS;
    const int64_t col = c0 + 8 * tx;                 // this thread's 8 columns
    const bool col_live = col < K;
    __syncthreads();                                 // the previous tile is done with a_s, b_s
    // stage A[0..r)[c0 .. c0+256) as fp32 and B[r0 .. r0+64)[0..r) as pairs
    for (int i = threadIdx.x; i < r * (MG_COLS / 8); i += blockDim.x) {
      const int j = i / (MG_COLS / 8), ch = i % (MG_COLS / 8);
      const int64_t k = c0 + 8 * ch;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (k < K) v = *reinterpret_cast<const uint4*>(A + (size_t)j * K + k);
      float4* dst = reinterpret_cast<float4*>(a_s + (size_t)j * MG_COLS + 8 * ch);
      dst[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
      dst[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
    }
    for (int i = threadIdx.x; i < r * MG_ROWS; i += blockDim.x) {
      const int row = i / r, j = i % r;
      const float b = (r0 + row < N) ? __bfloat162float(B[(size_t)(r0 + row) * r + j]) : 0.0f;
      b_s[(size_t)j * MG_ROWS + row] = make_float2(b, b);
    }
    // codes and block constants of the thread's 8 rows (in flight during the sums)
    uint32_t w[8];
    float c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t row = r0 + 8 * ty + i;
      w[i] = 0u;
      c[i] = 0.0f;
      if (row < N && col_live) {
        const int64_t e0 = row * K + col;
        w[i] = __ldcs(reinterpret_cast<const uint32_t*>(codes + (e0 >> 1)));
        c[i] = block_const(wc, row * kb + col / 64, mu);
      }
    }
    __syncthreads();
    // d[i][c] = sum over j in order of B[row i, j] A[j, col c]
    float2 d[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int h = 0; h < 4; ++h) d[i][h] = make_float2(0.0f, 0.0f);
    for (int j = 0; j < r; ++j) {
      const float4 a0 = *reinterpret_cast<const float4*>(a_s + (size_t)j * MG_COLS + 8 * tx);
      const float4 a1 = *reinterpret_cast<const float4*>(a_s + (size_t)j * MG_COLS + 8 * tx + 4);
      const float2 ap[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w), make_float2(a1.x, a1.y),
                            make_float2(a1.z, a1.w)};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const float4 bb = *reinterpret_cast<const float4*>(b_s + (size_t)j * MG_ROWS + 8 * ty + i);
        const float2 b0 = make_float2(bb.x, bb.y), b1 = make_float2(bb.z, bb.w);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          fma2_rn(d[i][h], b0, ap[h]);
          fma2_rn(d[i + 1][h], b1, ap[h]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t row = r0 + 8 * ty + i;
      const bool live = row < N && col_live;
      const int64_t e0 = row * K + col;
      float v[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float dd[2] = {d[i][h].x, d[i][h].y};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int e = 2 * h + u;
          const float wh = __bfloat162float(__float2bfloat16_rn(__fmul_rn(q[(w[i] >> (4 * e)) & 0xFu], c[i])));
          v[e] = live ? __bfloat162float(__float2bfloat16_rn(__fadd_rn(wh, __fmul_rn(s, dd[u])))) : 0.0f;
        }
      }
      if (out && live) {
        uint4 pk;
        pk.x = pack_bf16x2(v[0], v[1]);
        pk.y = pack_bf16x2(v[2], v[3]);
        pk.z = pack_bf16x2(v[4], v[5]);
        pk.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4*>(out + e0) = pk;
      }
      if (codes_out) {   // uniform over the grid: every lane takes part in the shuffles
        uint32_t abits = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) abits = max(abits, __float_as_uint(v[e]) & 0x7FFFFFFFu);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) abits = max(abits, __shfl_xor_sync(0xffffffffu, abits, o));
        if (abits >= 0x7F800000u && lane8 == 0 && live) raise_status(ST_NONFINITE);
        const float c2 = __uint_as_float(abits);
        const uint32_t word = encode8(v, c2, bins, tab);
        if (live) {
          *reinterpret_cast<uint32_t*>(codes_out + (e0 >> 1)) = word;
          if (lane8 == 0) absmax_out[e0 >> 6] = c2;
        }
      }
    }
  }
}

// ------------------------------------------------------------------- launch
static int sm_count() {
  const int c = device_sm_count();
  return c > 0 ? c : 148;
}

// Resident 256-thread CTAs per SM of a streaming kernel (4 if the calculator
// gives no answer).
template <typename K>
static int ctas_per_sm(K kernel) {
  const int b = per_device(reinterpret_cast<const void*>(kernel), 1, [kernel] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 256, 0) != cudaSuccess || n < 1) {
      cudaGetLastError();
      return -1;
    }
    return n;
  });
  return b > 0 ? b : 4;
}

static unsigned grid_for(int64_t work_items, int per_cta, int ctas_per_sm) {
  int64_t need = (work_items + per_cta - 1) / per_cta;
  int64_t cap = (int64_t)sm_count() * ctas_per_sm;
  if (need < 1) need = 1;
  return (unsigned)(need < cap ? need : cap);
}

ql_status launch_quantize(const void* x, ql_dtype dt, int64_t n, uint8_t* codes, float* absmax,
                          cudaStream_t st) {
  const int64_t nb = (n + 63) / 64;
  // one resident wave of CTAs (grid-stride loop), 32 blocks (8 warps x 4) per CTA iteration
  const int bps = dt == QL_F32 ? ctas_per_sm(quantize_kernel<float>) : ctas_per_sm(quantize_kernel<__nv_bfloat16>);
  const unsigned grid = grid_for(nb, 32, bps);
  static const QuantBins bins = build_bins(nf4_table());
  TraceScope ts(TK_QUANTIZE, st);
  if (dt == QL_F32)
    QL_CUDA_TRY(launch(quantize_kernel<float>, dim3(grid), dim3(256), 0, st, 1, 1, (const float*)x, n, codes, absmax, nf4_table(), bins));
  else
    QL_CUDA_TRY(launch(quantize_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 1, 1, (const __nv_bfloat16*)x, n, codes, absmax,
                                                         nf4_table(), bins));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

size_t dq_workspace_bytes(int64_t nb) {
  // one double per node of each tree pass above the leaves
  size_t total = 0;
  int64_t cnt = nb;
  do {
    cnt = (cnt + 2047) / 2048;
    total += (size_t)cnt * sizeof(double);
  } while (cnt > 1);
  return (total + 255) & ~(size_t)255;
}

ql_status launch_double_quant(const float* absmax, int64_t nb, uint8_t* absmax_q, float* scale2,
                              float* offset, void* ws, cudaStream_t st) {
  double* buf = reinterpret_cast<double*>(ws);
  int64_t cnt = (nb + 2047) / 2048;
  {
  TraceScope ts(TK_DQ_MEAN, st);
  QL_CUDA_TRY(launch(tree_sum_pass<float>, dim3((unsigned)cnt), dim3(256), 0, st, 1, 1, absmax, nb, buf, nb, cnt == 1 ? offset : nullptr));
  QL_LAUNCH_CHECK();
  double* prev = buf;
  while (cnt > 1) {
    int64_t next = (cnt + 2047) / 2048;
    double* dst = prev + cnt;
    QL_CUDA_TRY(launch(tree_sum_pass<double>, dim3((unsigned)next), dim3(256), 0, st, 1, 1, prev, cnt, dst, nb, next == 1 ? offset : nullptr));
    QL_LAUNCH_CHECK();
    prev = dst;
    cnt = next;
  }
  }
  const int64_t ng = (nb + 255) / 256;
  TraceScope ts(TK_DQ_ENCODE, st);
  QL_CUDA_TRY(launch(dq_encode_kernel, dim3(grid_for(ng, 8, 8)), dim3(256), 0, st, 1, 1, absmax, nb, offset, absmax_q, scale2));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

// Quantization sharded by rows: the level-1 nodes of the mean's tree (one
// float64 sum per 2048 constants) of this slab ...
ql_status launch_dq_level1(const float* absmax, int64_t nb, double* nodes, cudaStream_t st) {
  const int64_t cnt = (nb + 2047) / 2048;
  TraceScope ts(TK_DQ_MEAN, st);
  QL_CUDA_TRY(launch(tree_sum_pass<float>, dim3((unsigned)cnt), dim3(256), 0, st, 1, 1, absmax, nb, nodes, nb,
                     (float*)nullptr));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

// ... and, from every slab's nodes in order, the mean (the remaining levels of
// the same tree) and this slab's E4M3 codes and group scales.
ql_status launch_dq_finish(const double* nodes, int64_t n_nodes, int64_t nb_total, const float* absmax, int64_t nb,
                           uint8_t* absmax_q, float* scale2, float* offset, void* ws, cudaStream_t st) {
  double* dst = reinterpret_cast<double*>(ws);
  const double* prev = nodes;
  int64_t cnt = n_nodes;
  {
    TraceScope ts(TK_DQ_MEAN, st);
    do {
      const int64_t next = (cnt + 2047) / 2048;
      QL_CUDA_TRY(launch(tree_sum_pass<double>, dim3((unsigned)next), dim3(256), 0, st, 1, 1, prev, cnt, dst, nb_total,
                         next == 1 ? offset : nullptr));
      QL_LAUNCH_CHECK();
      prev = dst;
      dst += next;
      cnt = next;
    } while (cnt > 1);
  }
  const int64_t ng = (nb + 255) / 256;
  TraceScope ts(TK_DQ_ENCODE, st);
  QL_CUDA_TRY(launch(dq_encode_kernel, dim3(grid_for(ng, 8, 8)), dim3(256), 0, st, 1, 1, absmax, nb, offset, absmax_q,
                     scale2));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_dequant(const ql_nf4_weight* w, void* out, ql_dtype dt, cudaStream_t st) {
  const int64_t n = w->rows * w->cols;
  WeightConsts wc{w->absmax, w->absmax_q, w->scale2, w->offset};
  TraceScope ts(TK_DEQUANT, st);
  if (dt == QL_BF16) {
    const int64_t nb = (n + 63) / 64;
    QL_CUDA_TRY(launch(dequant_bf16_kernel, dim3(grid_for(nb, 256, 4)), dim3(256), 0, st, 1, 1, w->codes, wc, n, (__nv_bfloat16*)out,
                                                             nf4_table()));
  } else {
    QL_CUDA_TRY(launch(dequant_f32_kernel, dim3(grid_for((n + 7) / 8, 256, 8)), dim3(256), 0, st, 1, 1, w->codes, wc, n, (float*)out,
                                                                     nf4_table()));
  }
  QL_LAUNCH_CHECK();
  return QL_OK;
}


ql_status launch_merge(const ql_nf4_weight* w, const void* A, const void* B, int r, float s, void* out,
                       uint8_t* codes_out, float* absmax_out, cudaStream_t st) {
  WeightConsts wc{w->absmax, w->absmax_q, w->scale2, w->offset};
  const size_t smem = (size_t)r * (MG_COLS * sizeof(float) + MG_ROWS * sizeof(float2));
  // the shared-memory size depends on r: set the limit for the largest rank once per device
  const bool attr = per_device(reinterpret_cast<const void*>(merge_kernel), 0, [] {
                      const int most = QL_MAX_RANK * (MG_COLS * (int)sizeof(float) + MG_ROWS * (int)sizeof(float2));
                      if (cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, most) !=
                          cudaSuccess) {
                        cudaGetLastError();
                        return -1;
                      }
                      return 1;
                    }) > 0;
  if (!attr) return QL_ERR_CUDA;
  const int64_t tiles = (w->rows + MG_ROWS - 1) / MG_ROWS * ((w->cols + MG_COLS - 1) / MG_COLS);
  const int64_t cap = (int64_t)sm_count() * 2;
  static const QuantBins bins = build_bins(nf4_table());
  TraceScope ts(TK_MERGE, st);
  QL_CUDA_TRY(launch(merge_kernel, dim3((unsigned)std::max<int64_t>(1, std::min(tiles, cap))), dim3(256), smem, st, 1,
                     1, w->codes, wc, w->rows, w->cols, (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, r, s,
                     (__nv_bfloat16*)out, codes_out, absmax_out, nf4_table(), bins));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

}  // namespace ql
