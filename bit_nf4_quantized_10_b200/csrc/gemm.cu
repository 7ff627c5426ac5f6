// Fused NF4-dequant GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "QLoRA: Quantize Base Weights to 4-Bit", §3: the 4-bit weights stay
// compressed in HBM, are expanded to BF16 on chip, multiplied on the BF16
// tensor cores, and the LoRA branch (B @ (A @ x)) * (alpha / r) is added to
// the same output.  "QLoRA — Fine-Tuning a 65B Model on One GPU", "Where the
// gradients actually go": the input gradient runs through dequant(W)^T; W is
// only read.
//
// One kernel serves both directions (row-vector convention, tokens are rows):
//   forward  Y  = X  * W_hat^T + U * (s B)^T     reduction over K (W columns)
//   backward dX = dY * W_hat   + V * (s A)       reduction over N (W rows)
// CTA tile: 128 tokens x 256 outputs, 64 reduction elements per pipeline stage.
// Warp roles (320 threads):
//   warp 0      TMA: activation tile (128 x 64 bf16, 128B swizzle) and the
//               packed NF4 codes of the weight tile into shared memory
//   warp 1      TMEM allocation; one thread issues tcgen05.mma
//   warps 2-9   dequant producers: each thread expands one 64-block of codes
//               through a per-block register lookup table into the swizzled
//               BF16 operand tile, then (after the main loop) writes the LoRA
//               operands, and finally drains the TMEM accumulator.
// The B operand tile holds W rows as 128-byte rows in both directions: K-major
// for the forward (rows = output features), MN-major for the backward (rows =
// the reduction index), so the producers write the same layout either way.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "trace.cuh"
#include "sm100.cuh"

namespace ql {
using namespace sm100;

namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 32 KB
constexpr int C_BYTES = BN * BK / 2;   // 8 KB of packed codes
constexpr int PRODUCER_WARPS = 8;
constexpr int THREADS = (2 + PRODUCER_WARPS) * 32;
constexpr int TMEM_COLS = 256;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES + C_BYTES) + 256;

struct Params {
  int M;             // tokens
  int n_out;         // output columns (N forward, K backward)
  int n_steps;       // main-loop stages (K/64 forward, ceil(N/64) backward)
  int N, K;          // weight shape
  WeightConsts wc;
  const __nv_bfloat16* lora_a;  // forward U [M, r]; backward V [M, r]
  const __nv_bfloat16* lora_b;  // forward B [N, r]; backward A [r, K]
  int r, rp;                    // rank, rank padded to 16
  float s;
  void* out;
  int out_bf16;
  int accumulate;
  NF4Table tab;
  uint32_t wait_limit;
};

struct Smem {
  uint8_t* a0;   // STAGES activation tiles, A_BYTES apart
  uint8_t* b0;   // STAGES weight tiles, B_BYTES apart
  uint8_t* c0;   // STAGES packed-code tiles, C_BYTES apart
  __device__ __forceinline__ uint8_t* a(int s) const { return a0 + s * A_BYTES; }
  __device__ __forceinline__ uint8_t* b(int s) const { return b0 + s * B_BYTES; }
  __device__ __forceinline__ uint8_t* c(int s) const { return c0 + s * C_BYTES; }
  uint64_t* full_a;
  uint64_t* full_c;
  uint64_t* full_b;
  uint64_t* empty;
  uint64_t* acc_full;
  uint32_t* tmem_addr;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.a0 = p; p += STAGES * A_BYTES;
  s.b0 = p; p += STAGES * B_BYTES;
  s.c0 = p; p += STAGES * C_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p);
  s.full_a = bars;
  s.full_c = bars + STAGES;
  s.full_b = bars + 2 * STAGES;
  s.empty = bars + 3 * STAGES;
  s.acc_full = bars + 4 * STAGES;
  s.tmem_addr = reinterpret_cast<uint32_t*>(bars + 4 * STAGES + 1);
  s.abort = reinterpret_cast<int*>(s.tmem_addr + 1);
  return s;
}

__device__ __forceinline__ uint4 zero4() { return make_uint4(0, 0, 0, 0); }

// Scale 8 bf16 values by s in fp32 and round back to bf16.
__device__ __forceinline__ uint4 scale8(uint4 v, float s) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = pack_bf16x2(__fmul_rn(s, bf16_lo(w[i])), __fmul_rn(s, bf16_hi(w[i])));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool BWD>
__global__ void __launch_bounds__(THREADS, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_codes,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  const int j0 = blockIdx.x * BN;   // output-column tile start (W row in fwd, W col in bwd)
  const int steps = p.n_steps + (p.r > 0 ? 1 : 0);
  volatile int* abort_flag = sm.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&sm.full_a[i], 1);
      mbar_init(&sm.full_c[i], 1);
      mbar_init(&sm.full_b[i], PRODUCER_WARPS);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_init(sm.acc_full, 1);
    *sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_act);
    prefetch_tmap(&tmap_codes);
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem_addr, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_addr;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < p.n_steps; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (use > 0 && !mbar_wait(&sm.empty[s], (use - 1) & 1, abort_flag, p.wait_limit)) break;
        mbar_arrive_expect_tx(&sm.full_a[s], A_BYTES);
        tma_load_2d(sm.a(s), &tmap_act, &sm.full_a[s], i * BK, m0);
        mbar_arrive_expect_tx(&sm.full_c[s], C_BYTES);
        if (!BWD)
          tma_load_2d(sm.c(s), &tmap_codes, &sm.full_c[s], i * (BK / 2), j0);
        else
          tma_load_2d(sm.c(s), &tmap_codes, &sm.full_c[s], j0 / 2, i * BK);
        issued = i + 1;
      }
      // before leaving, make sure no copy is still landing in shared memory
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        mbar_wait(&sm.full_a[s], use & 1, abort_flag, p.wait_limit);
        mbar_wait(&sm.full_c[s], use & 1, abort_flag, p.wait_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(BM, BN, false, BWD);
      bool ok = true;
      for (int i = 0; i < steps && ok; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        const bool lora = (i == p.n_steps);
        if (!lora) ok = mbar_wait(&sm.full_a[s], use & 1, abort_flag, p.wait_limit);
        if (ok) ok = mbar_wait(&sm.full_b[s], use & 1, abort_flag, p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sm.a(s));
        const uint32_t b_addr = smem_u32(sm.b(s));
        const int kk_n = lora ? p.rp / 16 : BK / 16;
        for (int kk = 0; kk < kk_n; ++kk) {
          const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = BWD ? sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                  : sdesc_sw128(b_addr + kk * 32, 16, 1024);
          mma_bf16(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.empty[s]);
      }
      mma_commit(sm.acc_full);
    }
  } else {
    // ------------------------------------------------------ dequant producers
    const int pt = threadIdx.x - 64;   // 0..255
    const int kblocks = p.K / 64;      // 64-blocks per weight row
    const float mu = p.wc.absmax ? 0.0f : *p.wc.offset;
    // which weight row / 64-block column this thread expands in every stage
    int row_in_tile, col_chunk;
    if (!BWD) { row_in_tile = pt; col_chunk = 0; }
    else { row_in_tile = pt & 63; col_chunk = pt >> 6; }
    bool ok = true;
    for (int i = 0; i < p.n_steps && ok; ++i) {
      const int s = i % STAGES, use = i / STAGES;
      int wrow, kb;   // weight row, 64-block column
      if (!BWD) { wrow = j0 + row_in_tile; kb = i; }
      else { wrow = i * BK + row_in_tile; kb = j0 / 64 + col_chunk; }
      const bool valid = wrow < p.N && kb < kblocks;
      float c = 0.0f;
      if (valid) c = block_const(p.wc, (int64_t)wrow * kblocks + kb, mu);
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.full_c[s], use & 1, abort_flag, p.wait_limit));
      if (!ok) break;
      uint8_t* bt = sm.b(s);
      if (valid) {
        const uint8_t* csrc = BWD ? sm.c(s) + row_in_tile * 128 + col_chunk * 32 : sm.c(s) + row_in_tile * 32;
        const uint4 c0 = *reinterpret_cast<const uint4*>(csrc);
        const uint4 c1 = *reinterpret_cast<const uint4*>(csrc + 16);
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const Lut16 L = make_lut(p.tab, c);
        uint8_t* base = bt + (BWD ? col_chunk * 8192 : 0);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(base + sw128_offset(row_in_tile, j)) = lut_lookup8(L, w[j]);
      } else {
        uint8_t* base = bt + (BWD ? col_chunk * 8192 : 0);
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(base + sw128_offset(row_in_tile, j)) = zero4();
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.full_b[s]);
    }
    // LoRA operands into the stage after the last main step
    if (ok && p.r > 0) {
      const int i = p.n_steps;
      const int s = i % STAGES, use = i / STAGES;
      if (use > 0) ok = __all_sync(0xffffffffu, mbar_wait(&sm.empty[s], (use - 1) & 1, abort_flag, p.wait_limit));
      if (ok) {
        // A operand: U or V tile [128 tokens x rp], K-major
        {
          const int row = pt >> 1, half = pt & 1;
          const int m = m0 + row;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = half * 4 + q;
            const int e = chunk * 8;
            uint4 v = zero4();
            if (m < p.M && e < p.r) v = *reinterpret_cast<const uint4*>(p.lora_a + (size_t)m * p.r + e);
            *reinterpret_cast<uint4*>(sm.a(s) + sw128_offset(row, chunk)) = v;
          }
        }
        if (!BWD) {
          // B operand: (s B)[n, 0..rp) for the 256 output features, K-major
          const int n = j0 + pt;
#pragma unroll
          for (int chunk = 0; chunk < 8; ++chunk) {
            const int e = chunk * 8;
            uint4 v = zero4();
            if (n < p.N && e < p.r) v = scale8(*reinterpret_cast<const uint4*>(p.lora_b + (size_t)n * p.r + e), p.s);
            *reinterpret_cast<uint4*>(sm.b(s) + sw128_offset(pt, chunk)) = v;
          }
        } else {
          // B operand: (s A)[0..rp, k] for the 256 output columns, MN-major
          for (int idx = pt; idx < p.rp * 32; idx += 256) {
            const int jr = idx >> 5, rem = idx & 31;
            const int cc = rem >> 3, piece = rem & 7;
            const int k = j0 + cc * 64 + piece * 8;
            uint4 v = zero4();
            if (jr < p.r && k < p.K) v = scale8(*reinterpret_cast<const uint4*>(p.lora_b + (size_t)jr * p.K + k), p.s);
            *reinterpret_cast<uint4*>(sm.b(s) + cc * 8192 + sw128_offset(jr, piece)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.full_b[s]);
      }
    }
    // ------------------------------------------------------------ epilogue
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(sm.acc_full, 0, abort_flag, p.wait_limit) && !*abort_flag);
    if (acc_ok) {
      tc_fence_after();
      const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31
      const int col_half = (warp - 2) >> 2;      // columns 0-127 or 128-255
      const int row = m0 + quad * 32 + lane;
      for (int cc = 0; cc < 8; ++cc) {
        const int col = col_half * 128 + cc * 16;
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)col, r);
        tmem_ld_wait();
        const int gcol = j0 + col;
        if (row < p.M && gcol < p.n_out) {
          const size_t off = (size_t)row * p.n_out + gcol;
          if (p.out_bf16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + off;
            uint32_t pk[8];
            if (p.accumulate) {
              const uint4 o0 = *reinterpret_cast<const uint4*>(o), o1 = *reinterpret_cast<const uint4*>(o + 8);
              const uint32_t old[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
              for (int q = 0; q < 8; ++q)
                pk[q] = pack_bf16x2(__fadd_rn(bf16_lo(old[q]), __uint_as_float(r[2 * q])),
                                    __fadd_rn(bf16_hi(old[q]), __uint_as_float(r[2 * q + 1])));
            } else {
#pragma unroll
              for (int q = 0; q < 8; ++q) pk[q] = pack_bf16x2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
            }
            reinterpret_cast<uint4*>(o)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            reinterpret_cast<uint4*>(o)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          } else {
            float* o = reinterpret_cast<float*>(p.out) + off;
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(r[q]);
            if (p.accumulate) {
#pragma unroll
              for (int q = 0; q < 16; ++q) v[q] = __fadd_rn(v[q], o[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
              reinterpret_cast<float4*>(o)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp == 1 && lane == 0 && *abort_flag) {
    // let MMAs already issued finish before the accumulator is released
    mbar_wait(sm.acc_full, 0, abort_flag, p.wait_limit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace gemm

// ------------------------------------------------------------------ host side
QL_DEFINE_STATUS_ACCESSOR(status_word_gemm)

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D tensor map over a row-major [rows, cols] array.
static bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                     uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool BWD>
static ql_status launch_gemm_impl(const ql_nf4_weight* w, const void* act, int64_t M, const void* lora_a,
                                  const void* lora_b, int r, float s, void* out, ql_dtype out_dt, int accumulate,
                                  cudaStream_t st) {
  using namespace gemm;
  static bool attr_set = false;
  if (!attr_set) {
    QL_CUDA_TRY(cudaFuncSetAttribute(qlora_gemm_kernel<BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SMEM_BYTES));
    attr_set = true;
  }
  const int N = (int)w->rows, K = (int)w->cols;
  CUtensorMap map_act, map_codes;
  const int red = BWD ? N : K;   // reduction length = activation row length
  if (!make_map(&map_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, act, (uint64_t)red, (uint64_t)M, BK, BM,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  if (!BWD) {
    if (!make_map(&map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)K / 2, (uint64_t)N, BK / 2, BN,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return QL_ERR_CUDA;
  } else {
    if (!make_map(&map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)K / 2, (uint64_t)N, BN / 2, BK,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return QL_ERR_CUDA;
  }
  Params p;
  p.M = (int)M;
  p.n_out = BWD ? K : N;
  p.n_steps = BWD ? (N + BK - 1) / BK : K / BK;
  p.N = N;
  p.K = K;
  p.wc = WeightConsts{w->absmax, w->absmax_q, w->scale2, w->offset};
  p.lora_a = (const __nv_bfloat16*)lora_a;
  p.lora_b = (const __nv_bfloat16*)lora_b;
  p.r = r;
  p.rp = (r + 15) / 16 * 16;
  p.s = s;
  p.out = out;
  p.out_bf16 = out_dt == QL_BF16;
  p.accumulate = accumulate;
  p.tab = nf4_table();
  p.wait_limit = 1u << 22;
  dim3 grid((unsigned)((p.n_out + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
  TraceScope ts(BWD ? TK_GEMM_BWD : TK_GEMM_FWD, st);
  qlora_gemm_kernel<BWD><<<grid, THREADS, SMEM_BYTES, st>>>(map_act, map_codes, p);
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_gemm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* U, const void* B, int r,
                          float s, void* Y, ql_dtype y_dt, cudaStream_t st) {
  return launch_gemm_impl<false>(w, X, M, U, B, r, s, Y, y_dt, 0, st);
}

ql_status launch_gemm_bwd(const ql_nf4_weight* w, const void* dY, int64_t M, const void* V, const void* A, int r,
                          float s, void* dX, ql_dtype dx_dt, int accumulate, cudaStream_t st) {
  return launch_gemm_impl<true>(w, dY, M, V, A, r, s, dX, dx_dt, accumulate, st);
}

}  // namespace ql
