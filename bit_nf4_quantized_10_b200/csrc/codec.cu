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
// (ties go to the lower level).  A first guess goes through y = x/c: one fma
// with the addend 1.5 * 2^21 + 16 (ulp 1/4) rounds 16 y + 16 to a quarter, so
// the sum's bit pattern masked with 0x1FC is 4k, k = floor(round(64 y + 64) / 4)
// the bin y lies in, [(4k - 0.5)/64 - 1, (4k + 3.5)/64 - 1).  Bins are 1/16
// wide, narrower than the closest two midpoints (0.093 apart), so each bin
// (widened by 1e-5 on both sides, far more than the error of the approximate
// 16/c) holds at most one threshold.  Per bin the tables give j, the count of
// thresholds below the bin, and m_j (4 past the last): the code is then
// j + [x > fl32(m_j c)], one exact comparison.  Bins 33..127 are reached only
// from a NaN or from a y one rounding below -1; they hold j = 0, m = 4.  m and
// j sit in tables of 4-byte words, so 32 lanes reading 33 live entries meet no
// bank conflict, and 4k is their byte offset as it is.
struct QuantTab {
  float m[128];
  uint32_t j[128];
};

QuantTab build_quant_tab(const NF4Table& t) {
  QuantTab b{};
  for (int k = 0; k < 128; ++k) {
    b.m[k] = 4.0f;
    b.j[k] = 0;
  }
  for (int k = 0; k <= 32; ++k) {
    const double lo = (4.0 * k - 0.5) / 64.0 - 1.0 - 1e-5;
    uint32_t below = 0;
    for (int j = 0; j < 15; ++j)
      if ((double)t.m[j] < lo) ++below;
    b.j[k] = below;
    b.m[k] = below < 15 ? t.m[below] : 4.0f;
  }
  return b;
}

constexpr float kBinMagic = 3145744.0f;   // 1.5 * 2^21 + 16

template <typename W>
__device__ __forceinline__ W lds_at(const W* table, uint32_t byte_off) {
  return *reinterpret_cast<const W*>(reinterpret_cast<const char*>(table) + byte_off);
}

// Shared-memory copy of the QuantTab, j once per nibble slot i of a code word
// pre-shifted to j << 4i.
struct QuantTabSmem {
  float m[128];
  uint32_t j[8][128];
};

// The eight codes of v (elements 0..7 in nibbles 0..7) given the block's
// absmax c.  Scalar fma / mul / compare: the comparison x > fl32(m c) is a
// compare, never the sign of fl32(m c) - x, which the compiler may contract
// with the product into one fma (one rounding of m c - x) and so misjudge a
// tie x = fl32(m c).
__device__ __forceinline__ uint32_t encode8(const float (&v)[8], float c, const QuantTabSmem& T,
                                            const NF4Table& tab) {
  uint32_t word = 0;
  if (c >= 1e-30f) {
    // 16/c as the reciprocal of c/16 (exact scaling; 1/(c/16) is normal for
    // every finite c >= 1e-30)
    float s16;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(s16) : "f"(c * 0.0625f));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float t = __fmaf_rn(v[i], s16, kBinMagic);
      const uint32_t o = __float_as_uint(t) & 0x1FCu;
      const float th = __fmul_rn(lds_at(T.m, o), c);
      word += lds_at(T.j[i], o) + (v[i] > th ? (1u << (4 * i)) : 0u);
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

// The QuantTab staged into shared memory by threads 0..127.
__device__ __forceinline__ void stage_quant_tab(const QuantTab& in, QuantTabSmem& T) {
  if (threadIdx.x < 128) {
    T.m[threadIdx.x] = in.m[threadIdx.x];
    const uint32_t j = in.j[threadIdx.x];
#pragma unroll
    for (int i = 0; i < 8; ++i) T.j[i][threadIdx.x] = j << (4 * i);
  }
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

// max(a, b), NaN if either is NaN.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Block absmax of the eight lanes 8b..8b+7 holding one 64-block: max |x| over
// the lane's values, then xor shuffles.  NaN propagates and Inf is the
// largest, so a non-finite block gives a non-finite constant.
__device__ __forceinline__ float block_absmax(const float (&v)[8]) {
  float m = fabsf(v[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmax_nan(m, fabsf(v[i]));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// A warp takes 4 QU consecutive 64-blocks per iteration, as QU chunks of 256
// elements: lane l holds elements 8l..8l+7 of each chunk (one 16-byte load per
// chunk for bf16, two for fp32; a warp's load is 512 or 1024 contiguous bytes),
// so lanes 8b..8b+7 hold block b of the chunk and reduce its absmax with
// shuffles.  The next iteration's chunks are loaded while this one is coded.
// Addresses are one 64-bit base per iteration plus 32-bit lane offsets; only an
// iteration that reaches past n checks element bounds.
constexpr int QU = 2;   // chunks per warp iteration
template <typename T>
__global__ void __launch_bounds__(256) quantize_kernel(const T* __restrict__ x, int64_t n,
                                                       uint8_t* __restrict__ codes,
                                                       float* __restrict__ absmax, NF4Table tab, QuantTab tab_in) {
  pdl_wait();
  pdl_trigger();
  __shared__ QuantTabSmem qt;
  stage_quant_tab(tab_in, qt);
  __syncthreads();
  constexpr int GE = 256 * QU;                   // elements per warp iteration
  const int64_t ng = (n + GE - 1) / GE;
  const int lane = threadIdx.x & 31, lane8 = lane & 7;
  const int64_t warps_per_grid = (int64_t)gridDim.x * (blockDim.x >> 5);
  int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  Raw8<T> nxt[QU];
  if (g < ng) {
#pragma unroll
    for (int u = 0; u < QU; ++u) load8<T>(x, g * GE + 256 * u + 8 * lane, n, nxt[u]);
  }
  bool nonfinite = false;
  for (; g < ng; g += warps_per_grid) {
    Raw8<T> cur[QU];
#pragma unroll
    for (int u = 0; u < QU; ++u) cur[u] = nxt[u];
    const int64_t gn = g + warps_per_grid;
    if (gn < ng) {
#pragma unroll
      for (int u = 0; u < QU; ++u) load8<T>(x, gn * GE + 256 * u + 8 * lane, n, nxt[u]);
    }
    const int64_t base = g * GE;
    const bool full = base + GE <= n;            // no element of the iteration past the end
    uint8_t* cbase = codes + (base >> 1);
    float* abase = absmax + (base >> 6);
#pragma unroll
    for (int u = 0; u < QU; ++u) {
      float v[8];
      unpack8(cur[u], v);
      const float c = block_absmax(v);
      nonfinite |= !(c <= 3.402823466e38f);
      const uint32_t word = encode8(v, c, qt, tab);
      const int off = 256 * u + 8 * lane;        // element offset in the iteration
      if (full) {
        __stcs(reinterpret_cast<uint32_t*>(cbase + (off >> 1)), word);
        if (lane8 == 0) abase[off >> 6] = c;
      } else {
        const int64_t e0 = base + off;           // >= n for a block past the end
        if (e0 + 8 <= n) {
          __stcs(reinterpret_cast<uint32_t*>(cbase + (off >> 1)), word);
        } else if (e0 < n) {
          const int valid = (int)(n - e0);       // 1..7
          for (int i = 0; i < valid; i += 2) {
            uint32_t lo = (word >> (4 * i)) & 0xFu;
            uint32_t hi = (i + 1 < valid) ? ((word >> (4 * (i + 1))) & 0xFu) : 8u;
            cbase[(off + i) >> 1] = (uint8_t)(lo | (hi << 4));
          }
        }
        if (lane8 == 0 && e0 < n) abase[off >> 6] = c;
      }
    }
  }
  // padding past n is zero, so only real elements can be non-finite
  if (nonfinite) raise_status(ST_NONFINITE);
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
// tile and accumulates its 64 sums with scalar fp32 fmas (j in order), reading
// A and B as fp32 from shared memory (a warp's B values are one broadcast):
// every A and B value is reused by 8 rows or 8 columns.  The FMA pipe takes
// scalar and packed fmas at the same element rate, and the scalar form needs no
// register-pair assembly around each instruction.  A CTA keeps one 256-column tile for its whole life and walks
// row tiles, so A's slice is staged once; B's 64 x r slice of the next row tile
// is loaded into registers while the current one computes.  The 8 threads
// holding a row's 64-block are 8 consecutive lanes, so the re-quantization's
// absmax is the same 8-lane shuffle as in quantize_kernel.  K % 64 == 0, so a
// block lies in one row and a tile edge never splits one.
constexpr int MG_ROWS = 64;     // rows per CTA tile: 8 warps x 8 rows
constexpr int MG_COLS = 256;    // columns per CTA tile: 32 lanes x 8 columns

// Element i of B's 64 x r slice of row tile rt (row i / r, column i % r), 0
// past the slice, the row tiles or N.
__device__ __forceinline__ float merge_b(const __nv_bfloat16* B, int64_t N, int r, int tiles_r, int rt, int i) {
  const int64_t row = (int64_t)rt * MG_ROWS + i / r;
  return (i < MG_ROWS * r && rt < tiles_r && row < N) ? __bfloat162float(B[(size_t)row * r + i % r]) : 0.0f;
}

// RMAX >= r: B's 64 x r slice of a row tile is spread over the 256 threads,
// MG_ROWS * RMAX / 256 values each.
template <int RMAX>
__global__ void __launch_bounds__(256, 2) merge_kernel(const uint8_t* __restrict__ codes, WeightConsts wc, int64_t N,
                                                    int64_t K, const __nv_bfloat16* __restrict__ A,
                                                    const __nv_bfloat16* __restrict__ B, int r, float s,
                                                    __nv_bfloat16* __restrict__ out, uint8_t* __restrict__ codes_out,
                                                    float* __restrict__ absmax_out, NF4Table tab, QuantTab tab_in) {
  pdl_wait();
  pdl_trigger();
  __shared__ QuantTabSmem qt;
  __shared__ float q[16];
  extern __shared__ __align__(16) float mg_smem[];
  float* a_s = mg_smem;                                               // [r][256] fp32
  float* b_s = mg_smem + (size_t)r * MG_COLS;                          // [r][64] fp32
  uint32_t* w_s = reinterpret_cast<uint32_t*>(b_s + (size_t)r * MG_ROWS);    // [64][32] code words of the tile
  stage_quant_tab(tab_in, qt);
#pragma unroll
  for (int k = 0; k < 16; ++k)                       // constant indices: the table stays in parameter space
    if (threadIdx.x == k) q[k] = tab.q[k];
  const float mu = wc.absmax ? 0.0f : *wc.offset;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int lane8 = tx & 7;
  const int64_t kb = K / 64;
  const int tiles_c = (int)((K + MG_COLS - 1) / MG_COLS);
  const int tiles_r = (int)((N + MG_ROWS - 1) / MG_ROWS);
  // this CTA's column tile, and its share of the row tiles
  const int ct = blockIdx.x % tiles_c;
  const int rt0 = blockIdx.x / tiles_c, rt_step = gridDim.x / tiles_c;
  const int64_t c0 = (int64_t)ct * MG_COLS;
  const int64_t col = c0 + 8 * tx;                   // this thread's 8 columns
  const bool col_live = col < K;
  // stage A[0..r)[c0 .. c0+256) as fp32, once
  for (int i = threadIdx.x; i < r * (MG_COLS / 8); i += blockDim.x) {
    const int j = i / (MG_COLS / 8), ch = i % (MG_COLS / 8);
    const int64_t k = c0 + 8 * ch;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < K) v = *reinterpret_cast<const uint4*>(A + (size_t)j * K + k);
    float4* dst = reinterpret_cast<float4*>(a_s + (size_t)j * MG_COLS + 8 * ch);
    dst[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    dst[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
  constexpr int MG_BPT = MG_ROWS * RMAX / 256;
  // B[r0 .. r0+64)[0..r) of a row tile, MG_BPT values per thread (element
  // i = threadIdx.x + 256 u of the slice, row i / r, column i % r)
  float bnext[MG_BPT];
#pragma unroll
  for (int u = 0; u < MG_BPT; ++u) bnext[u] = merge_b(B, N, r, tiles_r, rt0, threadIdx.x + 256 * u);
  for (int rt = rt0; rt < tiles_r; rt += rt_step) {
    const int64_t r0 = (int64_t)rt * MG_ROWS;
    __syncthreads();                                 // the previous tile is done with b_s (and A is staged)
#pragma unroll
    for (int u = 0; u < MG_BPT; ++u) {
      const int i = threadIdx.x + 256 * u;
      if (i < MG_ROWS * r) b_s[(size_t)(i % r) * MG_ROWS + i / r] = bnext[u];
    }
    // the tile's codes into shared memory (in flight during the sums): 64 rows
    // of 128 bytes, two 16-byte copies per thread, zero past N or K
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int id = threadIdx.x + 256 * u, row = id >> 3, ch = id & 7;
      const bool live = r0 + row < N && c0 + 32 * ch < K;
      const uint8_t* src = live ? codes + (((r0 + row) * K + c0) >> 1) + 16 * ch : codes;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(w_s) + 16 * id), "l"(src),
                   "r"(live ? 16u : 0u)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    // raw block constants of the thread's 8 rows (in flight during the sums;
    // decoded after them): the fp32 constant's bits, or the E4M3 byte and s_2
    uint32_t craw[8];
    float cs2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t row = r0 + 8 * ty + i;
      craw[i] = 0u;
      cs2[i] = 0.0f;
      if (row < N && col_live) {
        const int64_t b = row * kb + col / 64;
        if (wc.absmax) {
          craw[i] = __float_as_uint(__ldg(wc.absmax + b));
        } else {
          craw[i] = __ldg(wc.absmax_q + b);
          cs2[i] = __ldg(wc.scale2 + (b >> 8));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < MG_BPT; ++u)                 // the next row tile's B, in flight
      bnext[u] = merge_b(B, N, r, tiles_r, rt + rt_step, threadIdx.x + 256 * u);
    __syncthreads();
    // d[i][c] = sum over j in order of B[row i, j] A[j, col c]
    float d[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) d[i][cc] = 0.0f;
    for (int j = 0; j < r; ++j) {
      const float4 a0 = *reinterpret_cast<const float4*>(a_s + (size_t)j * MG_COLS + 8 * tx);
      const float4 a1 = *reinterpret_cast<const float4*>(a_s + (size_t)j * MG_COLS + 8 * tx + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(b_s + (size_t)j * MG_ROWS + 8 * ty);
      const float4 b1 = *reinterpret_cast<const float4*>(b_s + (size_t)j * MG_ROWS + 8 * ty + 4);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) d[i][cc] = __fmaf_rn(bv[i], av[cc], d[i][cc]);
    }
    float c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      c[i] = wc.absmax ? __uint_as_float(craw[i]) : __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)craw[i]), cs2[i]), mu);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();                                 // every thread's code copies have landed
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t row = r0 + 8 * ty + i;
      const bool live = row < N && col_live;
      const uint32_t wi = w_s[(8 * ty + i) * 32 + tx];
      const int64_t e0 = row * K + col;
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float wh = __bfloat162float(__float2bfloat16_rn(__fmul_rn(q[(wi >> (4 * e)) & 0xFu], c[i])));
        v[e] = live ? __bfloat162float(__float2bfloat16_rn(__fadd_rn(wh, __fmul_rn(s, d[i][e])))) : 0.0f;
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
        const uint32_t word = encode8(v, c2, qt, tab);
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
  // one resident wave of CTAs (grid-stride loop), 8 warps x 4 QU blocks per CTA iteration
  const int bps = dt == QL_F32 ? ctas_per_sm(quantize_kernel<float>) : ctas_per_sm(quantize_kernel<__nv_bfloat16>);
  const unsigned grid = grid_for(nb, 8 * 4 * QU, bps);
  static const QuantTab qtab = build_quant_tab(nf4_table());
  TraceScope ts(TK_QUANTIZE, st);
  if (dt == QL_F32)
    QL_CUDA_TRY(launch(quantize_kernel<float>, dim3(grid), dim3(256), 0, st, 1, 1, (const float*)x, n, codes, absmax, nf4_table(), qtab));
  else
    QL_CUDA_TRY(launch(quantize_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 1, 1, (const __nv_bfloat16*)x, n, codes, absmax,
                                                         nf4_table(), qtab));
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


template <int RMAX>
static ql_status launch_merge_r(const ql_nf4_weight* w, const void* A, const void* B, int r, float s, void* out,
                                uint8_t* codes_out, float* absmax_out, cudaStream_t st) {
  WeightConsts wc{w->absmax, w->absmax_q, w->scale2, w->offset};
  const size_t smem = (size_t)r * (MG_COLS + MG_ROWS) * sizeof(float) + MG_ROWS * MG_COLS / 2;
  // the shared-memory size depends on r: set the limit for the largest rank once per device
  const bool attr = per_device(reinterpret_cast<const void*>(merge_kernel<RMAX>), 0, [] {
                      const int most = RMAX * (MG_COLS + MG_ROWS) * (int)sizeof(float) + MG_ROWS * MG_COLS / 2;
                      if (cudaFuncSetAttribute(merge_kernel<RMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               most) != cudaSuccess) {
                        cudaGetLastError();
                        return -1;
                      }
                      return 1;
                    }) > 0;
  if (!attr) return QL_ERR_CUDA;
  // each CTA keeps one column tile: the grid is the column tiles times the
  // number of CTAs that share each one's row tiles (about two CTAs per SM)
  const int64_t tiles_c = (w->cols + MG_COLS - 1) / MG_COLS;
  const int64_t tiles_r = (w->rows + MG_ROWS - 1) / MG_ROWS;
  const int64_t rsplit = std::max<int64_t>(1, std::min<int64_t>(tiles_r, (int64_t)sm_count() * 2 / tiles_c));
  static const QuantTab qtab = build_quant_tab(nf4_table());
  TraceScope ts(TK_MERGE, st);
  QL_CUDA_TRY(launch(merge_kernel<RMAX>, dim3((unsigned)(tiles_c * rsplit)), dim3(256), smem, st, 1, 1, w->codes, wc,
                     w->rows, w->cols, (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, r, s, (__nv_bfloat16*)out,
                     codes_out, absmax_out, nf4_table(), qtab));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_merge(const ql_nf4_weight* w, const void* A, const void* B, int r, float s, void* out,
                       uint8_t* codes_out, float* absmax_out, cudaStream_t st) {
  static_assert(QL_MAX_RANK <= 64, "merge stages at most 64 adapter columns");
  if (r <= 16) return launch_merge_r<16>(w, A, B, r, s, out, codes_out, absmax_out, st);
  if (r <= 32) return launch_merge_r<32>(w, A, B, r, s, out, codes_out, absmax_out, st);
  return launch_merge_r<64>(w, A, B, r, s, out, codes_out, absmax_out, st);
}

}  // namespace ql
