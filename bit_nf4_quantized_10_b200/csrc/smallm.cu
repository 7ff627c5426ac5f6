// Small-token forward: Y = X * W_hat^T + s * U * B^T for M <= 16 tokens.
//
// With a handful of tokens each dequantized weight element meets at most 16
// activations, so the layer is bound by reading the packed 4-bit weight from
// HBM ("QLoRA — Fine-Tuning a 65B Model on One GPU", "Pitfalls":
// memory-bandwidth-bound generation has less to read with 4-bit weights), and
// the dequantization must keep pace with HBM.  The design differs from the
// large-M kernel accordingly:
//   * operands are swapped: the dequantized weight tile is the MMA's A operand
//     (M = 128 weight rows) and lives in TMEM, written with tcgen05.st straight
//     from the producer registers, so it costs no shared-memory bandwidth;
//     the tokens are the N = 16 operand (zero-padded by TMA);
//   * the expansion reads the 16 fp32 levels from a shared-memory table (one
//     conflict-free LDS per element), multiplies by the block constant in fp32
//     and packs pairs to bf16 — the same bf16(fl32(q * c)) as everywhere else,
//     with fewer integer operations than the register lookup table;
//   * each TMA stage brings 128 contiguous bytes (256 codes) of every weight
//     row, four 64-deep MMA sub-steps, so HBM is read in whole 128-byte lines;
//   * the reduction over K is split across CTAs (partials stay in L2) and a
//     second kernel adds the partials in fixed order together with the rank-r
//     term s * U * B^T in fp32.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                 uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

namespace smallm {

constexpr int TM = 128;           // weight rows per CTA (MMA M)
constexpr int TN = 16;            // token slots (MMA N)
constexpr int BK = 64;            // reduction elements per MMA sub-step (one 64-block per row)
constexpr int SUB = 4;            // sub-steps per TMA stage: 256 codes = 128 contiguous bytes per row
constexpr int STAGES = 2;         // TMA ring
constexpr int A_STAGES = 3;       // TMEM ring of dequantized 128 x 64 A tiles
constexpr int C_BYTES = TM * BK * SUB / 2;   // 16 KB packed codes
constexpr int X_SUB_BYTES = TN * BK * 2;     // 2 KB activation sub-tile
constexpr int STAGE_BYTES = C_BYTES + SUB * X_SUB_BYTES;
constexpr int PRODUCER_WARPS = 8;
constexpr int THREADS = (2 + PRODUCER_WARPS) * 32;
constexpr int TMEM_COLS = 128;    // D: 16 columns; A stages: 32 columns each from column 32 (3 CTAs per SM)
constexpr int A_COL0 = 32;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;

struct Params {
  int M, N, K;
  int stages_total, stages_per_split;   // in TMA stages of SUB * BK reduction elements
  int sub_total;                        // K / 64 (the last stage may be partial)
  WeightConsts wc;
  float* partial;          // [splits][N][16]
  NF4Table tab;
  uint32_t wait_limit;
};

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(THREADS, 3)
    smallm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float qtab[16];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_c = reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  uint64_t* full_x = full_c + STAGES;
  uint64_t* empty_t = full_x + STAGES;   // MMA done with a TMA stage
  uint64_t* full_a = empty_t + STAGES;   // producers stored a TMEM A sub-stage
  uint64_t* empty_a = full_a + A_STAGES; // MMA done with a TMEM A sub-stage
  uint64_t* acc_full = empty_a + A_STAGES;
  uint32_t* tmem_addr = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<int*>(tmem_addr + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * TM;
  const int st0 = blockIdx.y * p.stages_per_split;
  const int nst = min(p.stages_per_split, p.stages_total - st0);
  const int nsub = min(nst * SUB, p.sub_total - st0 * SUB);

  if (threadIdx.x < 16) qtab[threadIdx.x] = p.tab.q[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_c[i], 1);
      mbar_init(&full_x[i], 1);
      mbar_init(&empty_t[i], 1);
    }
    for (int i = 0; i < A_STAGES; ++i) {
      mbar_init(&full_a[i], PRODUCER_WARPS);
      mbar_init(&empty_a[i], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_addr, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_addr;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      prefetch_tmap(&tmap_codes);
      int issued = 0;
      for (int i = 0; i < nst; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (use > 0 && !mbar_wait(&empty_t[s], (use - 1) & 1, abort_flag, p.wait_limit)) break;
        const int kst = st0 + i;
        uint8_t* st = base + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full_c[s], C_BYTES);
        tma_load_2d(st, &tmap_codes, &full_c[s], kst * (SUB * BK / 2), n0);
        mbar_arrive_expect_tx(&full_x[s], SUB * X_SUB_BYTES);
#pragma unroll
        for (int u = 0; u < SUB; ++u)
          tma_load_2d(st + C_BYTES + u * X_SUB_BYTES, &tmap_x, &full_x[s], (kst * SUB + u) * BK, 0);
        issued = i + 1;
      }
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
        mbar_wait(&full_c[i % STAGES], (i / STAGES) & 1, abort_flag, 1u << 22);
        mbar_wait(&full_x[i % STAGES], (i / STAGES) & 1, abort_flag, 1u << 22);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(TM, TN, false, false);
      bool ok = true;
      for (int j = 0; j < nsub && ok; ++j) {
        const int i = j / SUB, u = j % SUB;
        const int s = i % STAGES, use = i / STAGES;
        const int sa = j % A_STAGES, usea = j / A_STAGES;
        ok = (u != 0 || mbar_wait(&full_x[s], use & 1, abort_flag, p.wait_limit)) &&
             mbar_wait(&full_a[sa], usea & 1, abort_flag, p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t x_addr = smem_u32(base + s * STAGE_BYTES + C_BYTES + u * X_SUB_BYTES);
        const uint32_t a_col = A_COL0 + sa * 32;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_ts(tmem, tmem + a_col + kk * 8, sdesc_sw128(x_addr + kk * 32, 16, 1024), idesc, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty_a[sa]);
        if (u == SUB - 1 || j == nsub - 1) mma_commit(&empty_t[s]);
      }
      mma_commit(acc_full);
    }
  } else {
    // producers: warp w covers TMEM lanes 32*(w&3)..+31 (weight rows) and the
    // half (w-2)>>2 of the 64 codes of each row's block in a sub-step
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const int wrow = n0 + row;
    const bool valid = wrow < p.N;
    const int kblocks = p.K / 64;
    const float mu = p.wc.absmax ? 0.0f : *p.wc.offset;
    const char* qb = reinterpret_cast<const char*>(qtab);
    // block constant, loaded one sub-step ahead
    auto load_c = [&](int j) -> float2 {
      float2 r = make_float2(0.0f, 0.0f);
      if (!valid || j >= nsub) return r;
      const int64_t b = (int64_t)wrow * kblocks + (int64_t)st0 * SUB + j;
      if (p.wc.absmax) r.x = __ldg(p.wc.absmax + b);
      else { r.x = __ldg(p.wc.scale2 + (b >> 8)); r.y = __uint_as_float((uint32_t)__ldg(p.wc.absmax_q + b)); }
      return r;
    };
    float2 nxt = load_c(0);
    bool ok = true;
    for (int j = 0; j < nsub && ok; ++j) {
      const int i = j / SUB, u = j % SUB;
      const int s = i % STAGES, use = i / STAGES;
      const int sa = j % A_STAGES, usea = j / A_STAGES;
      const float2 cur = nxt;
      nxt = load_c(j + 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&full_c[s], use & 1, abort_flag, p.wait_limit) &&
                                       (usea == 0 || mbar_wait(&empty_a[sa], (usea - 1) & 1, abort_flag, p.wait_limit)));
      if (!ok) break;
      tc_fence_after();
      uint32_t out[16];
      if (valid) {
        const float c = p.wc.absmax ? cur.x
                                    : __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)__float_as_uint(cur.y)), cur.x), mu);
        // 128-byte code rows with the 128B swizzle: 16-byte chunk ^= row mod 8
        const uint32_t coff = row * 128 + (((2 * u + half) ^ (row & 7)) << 4);
        const uint4 cw = *reinterpret_cast<const uint4*>(base + s * STAGE_BYTES + coff);
        const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t e4 = (w[q4] << 2) & 0x3C3C3C3Cu;   // 4 * low nibble of each byte
          const uint32_t o4 = (w[q4] >> 2) & 0x3C3C3C3Cu;   // 4 * high nibble of each byte
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t ae = __byte_perm(e4, 0u, 0x4440u | b);
            const uint32_t ao = __byte_perm(o4, 0u, 0x4440u | b);
            const float fe = *reinterpret_cast<const float*>(qb + ae);
            const float fo = *reinterpret_cast<const float*>(qb + ao);
            out[4 * q4 + b] = pack_bf16x2(__fmul_rn(fe, c), __fmul_rn(fo, c));
          }
        }
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) out[t] = 0u;
      }
      tmem_st16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(A_COL0 + sa * 32 + half * 16), out);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[sa]);
    }
    // drain: warps 2-5 read the 128 x 16 accumulator and write the partial
    if (half == 0) {
      const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.wait_limit) && !*abort_flag);
      if (acc_ok) {
        tc_fence_after();
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16), v);
        tmem_ld_wait();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.partial + ((size_t)blockIdx.y * p.N + wrow) * TN);
#pragma unroll
          for (int t = 0; t < 4; ++t)
            dst[t] = make_float4(__uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]), __uint_as_float(v[4 * t + 2]),
                                 __uint_as_float(v[4 * t + 3]));
        }
      }
    }
  }
  if (warp == 1 && lane == 0 && *abort_flag) mbar_wait(acc_full, 0, abort_flag, 1u << 22);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// One thread per output (m, n), m fastest: Y[m][n] = sum over splits (fixed
// order) of partial[split][n][m] + s * sum_j U[m][j] * B[n][j], in fp32.
__global__ void __launch_bounds__(256) smallm_reduce_kernel(const float* __restrict__ partial, int splits, int M, int N,
                                                            const __nv_bfloat16* __restrict__ U,
                                                            const __nv_bfloat16* __restrict__ B, int r, float s,
                                                            int out_bf16, void* __restrict__ Y) {
  pdl_wait();
  pdl_trigger();
  __shared__ float us[TN * 64];
  for (int i = threadIdx.x; i < M * r; i += blockDim.x) us[i] = __bfloat162float(U[i]);
  __syncthreads();
  const int64_t total = (int64_t)N * M;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(idx / M), m = (int)(idx % M);
    float acc = 0.0f;
    for (int sp = 0; sp < splits; ++sp) acc = __fadd_rn(acc, partial[((int64_t)sp * N + n) * TN + m]);
    if (r > 0) {
      float l = 0.0f;
      const __nv_bfloat16* brow = B + (int64_t)n * r;
      for (int j = 0; j < r; ++j) l = fmaf(us[m * r + j], __bfloat162float(brow[j]), l);
      acc = __fadd_rn(acc, __fmul_rn(s, l));
    }
    const int64_t o = (int64_t)m * N + n;
    if (out_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(acc);
    else reinterpret_cast<float*>(Y)[o] = acc;
  }
}

}  // namespace smallm

static int sm_count_sm() {
  static int count = 0;
  if (!count) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
    if (count <= 0) count = 148;
  }
  return count;
}

static void smallm_plan(int64_t N, int64_t K, int& splits, int& per) {
  const int tiles = (int)((N + smallm::TM - 1) / smallm::TM);
  const int stages = (int)((K + smallm::BK * smallm::SUB - 1) / (smallm::BK * smallm::SUB));
  // three resident CTAs per SM, about two work units each
  int want = std::max(1, (6 * sm_count_sm() + tiles - 1) / tiles);
  want = std::min(want, stages);
  per = (stages + want - 1) / want;
  splits = (stages + per - 1) / per;
}

size_t smallm_partial_bytes(int64_t N, int64_t K) {
  int splits, per;
  smallm_plan(N, K, splits, per);
  return (size_t)splits * N * smallm::TN * sizeof(float);
}

// Y = X W_hat^T + s U B^T for M <= 16; U [M, r] given (bf16), partial from the workspace.
ql_status launch_smallm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* U, const void* B, int r,
                            float s, void* Y, ql_dtype y_dt, float* partial, cudaStream_t st) {
  using namespace smallm;
  static bool attr_set = false;
  if (!attr_set) {
    QL_CUDA_TRY(cudaFuncSetAttribute(smallm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES));
    attr_set = true;
  }
  const int N = (int)w->rows, K = (int)w->cols;
  CUtensorMap map_x, map_codes;
  if (!make_map_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, TN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  if (!make_map_2d(&map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)K / 2, (uint64_t)N,
                   (uint64_t)K / 2, SUB * BK / 2, TM, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  int splits, per;
  smallm_plan(N, K, splits, per);
  Params p;
  p.M = (int)M;
  p.N = N;
  p.K = K;
  p.stages_total = (K + BK * SUB - 1) / (BK * SUB);
  p.sub_total = K / BK;
  p.stages_per_split = per;
  p.wc = WeightConsts{w->absmax, w->absmax_q, w->scale2, w->offset};
  p.partial = partial;
  p.tab = nf4_table();
  p.wait_limit = 1u << 22;
  dim3 grid((unsigned)((N + TM - 1) / TM), (unsigned)splits);
  {
    TraceScope ts(TK_SMALLM, st);
    QL_CUDA_TRY(launch(smallm_kernel, dim3(grid), dim3(THREADS), SMEM_BYTES, st, 1, 1, map_x, map_codes, p));
  }
  QL_LAUNCH_CHECK();
  const unsigned rg =
      (unsigned)std::max<int64_t>(1, std::min<int64_t>((M * (int64_t)N + 255) / 256, (int64_t)sm_count_sm() * 8));
  {
    TraceScope ts(TK_COLACC_REDUCE, st);
    QL_CUDA_TRY(launch(smallm_reduce_kernel, dim3(rg), dim3(256), 0, st, 1, 1, partial, splits, (int)M, N, (const __nv_bfloat16*)U,
                                             (const __nv_bfloat16*)B, r, s, y_dt == QL_BF16, Y));
  }
  QL_LAUNCH_CHECK();
  return QL_OK;
}

}  // namespace ql
