// FP4 x FP4 GEMM on the block-scaled tensor cores ("Lesson 4 of the Finetuning
// Sessions", "From Turing to Blackwell": the 5th-generation tensor cores
// execute the 4-bit block formats natively; "From FP32 to the 4-Bit Horizon":
// NVFP4 is E2M1 elements with one E4M3 scale per 16 and an fp32 tensor scale,
// MXFP4 E2M1 elements with one power-of-two (E8M0) scale per 32):
//   Y[m, n] = s_a s_b sum_k (E_a[m, k] S_a[m, k/VS]) (E_b[n, k] S_b[n, k/VS])
// with E the E2M1 values, S the block scales (VS = 16 or 32) and s the NVFP4
// tensor scales (1 for MXFP4), for operands quantized by nvfp4_quantize /
// mxfp4_quantize as row-major [rows, K] tensors (so a block runs along K).
//
// One CTA per 128 x 128 output tile, cta_group::1, the token (M) tiles
// fastest so that the CTAs resident at once share a few weight (N) tiles in L2:
//   * warp 0, one thread: TMA of the A and B code tiles (128 rows x 256
//     elements = 128 bytes per row, 128-byte swizzle) and a 1-D bulk copy of
//     each operand's scale atoms for the stage, into a 3-stage ring (two CTAs
//     fit on an SM, so one's drain overlaps the other's main loop);
//   * warp 1, one thread: tcgen05.cp of the stage's A and B scale atoms into
//     TMEM (32 lanes x 128 bits, broadcast to the four lane quarters), then
//     per 64-element K block tcgen05.mma kind::mxf4nvf4 with 16- or 32-element
//     scale blocks, accumulating in TMEM; a thread's tcgen05.cp and
//     tcgen05.mma execute in issue order, so the same TMEM scale columns serve
//     every stage;
//   * warps 2-5: the 128 x 128 fp32 accumulator out of TMEM, times s_a s_b,
//     staged in shared memory and written to Y a row per store instruction.
// Scale atoms: the tensor cores take 4 scales of each row of a 128-row block as
// 512 bytes, row m = m0 + 32 m1 (m0 < 32, m1 < 4) and scale kb < 4 at byte
// 16 m0 + 4 m1 + kb; one atom covers 4 VS elements of K (one MMA for NVFP4,
// two for MXFP4, each MMA then taking 2 of the 4 bytes, selected by the byte
// offset in the scale address and the descriptor's scale-factor ids).
// nvfp4_scale_atoms / mxfp4_scale_atoms write the quantizers' row-major scales
// in that order, [row tile][atom][512].
// Every wait is bounded: a lost arrival ends the kernel with QL_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

QL_DEFINE_STATUS_ACCESSOR(status_word_fp4g)

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                 uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

namespace fp4g {

constexpr int BM = 128, BN = 128;
constexpr int KS = 256;                                   // K elements per stage: 128 code bytes per row
constexpr int KBLK = 64;                                  // K elements per MMA
constexpr int STAGES = 3;                                 // <= 109 KB: two CTAs per SM
constexpr int A_BYTES = BM * KS / 2;                      // 16 KB
constexpr int B_BYTES = BN * KS / 2;                      // 16 KB
constexpr int THREADS = 6 * 32;
constexpr int TMEM_COLS = 256;                            // accumulator 0..127, scales from 128
constexpr int SFA_COL = 128, SFB_COL = 144;

// Per scale block VS (16: NVFP4, E4M3 scales; 32: MXFP4, E8M0 scales): a
// 512-byte atom holds 4 scales of each of 128 rows, so it covers 4 VS
// elements of K, one MMA (VS = 16) or two (VS = 32).
template <int VS>
__host__ __device__ constexpr int atom_k() { return 4 * VS; }
template <int VS>
__host__ __device__ constexpr int sf_bytes() { return (KS / atom_k<VS>()) * 512; }      // per operand and stage
template <int VS>
__host__ __device__ constexpr int stage_bytes() { return A_BYTES + B_BYTES + 2 * sf_bytes<VS>(); }
template <int VS>
__host__ __device__ constexpr size_t smem_bytes() { return 1024 + (size_t)STAGES * stage_bytes<VS>() + 256; }

// Instruction descriptor, kind::mxf4nvf4: E2M1 A and B (format 1), K-major,
// N >> 3 at bit 17, M >> 4 at bit 24, K = 64; scale format at bit 23 (0 E4M3,
// 1 E8M0).  The scale-factor ids (bits 29-30 for A, 4-5 for B) are the byte
// offset of the MMA's scales within the TMEM column, the top two bits of the
// scale addresses.
template <int VS>
__host__ __device__ constexpr uint32_t idesc_base() {
  return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((VS == 32 ? 1u : 0u) << 23) |
         ((uint32_t)(BM >> 4) << 24);
}

struct Params {
  int M, N, K;
  int ksteps;                 // K / KS
  const uint8_t* sfa;         // scale atoms of A, [ceil(M/128)][K/(4 VS)][512]
  const uint8_t* sfb;         // scale atoms of B, [ceil(N/128)][K/(4 VS)][512]
  int64_t sf_tile_bytes;      // (K / (4 VS)) * 512
  const float* sa;            // tensor scales (device), or NULL (scale 1)
  const float* sb;
  float* Y;                   // [M, N] fp32
  uint32_t wait_limit;
};

// Global -> shared bulk copy completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor without swizzle, K-major core matrices of
// 8 rows x 16 bytes: SBO = byte distance between 8-row groups.
__device__ __forceinline__ uint64_t sdesc_plain(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}

// One 512-byte scale atom (32 rows x 16 bytes in shared memory) into 4 TMEM
// columns of all 128 lanes (each lane quarter receives the same 32 rows).
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= (A * SFA)[smem] * (B * SFB)[smem]^T, kind::mxf4nvf4 with
// 16-element (NVFP4) or 32-element (MXFP4) scale blocks.
template <int VS>
__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  if constexpr (VS == 16) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %6, 0;\n"
        " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %6, 0;\n"
        " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
  }
}

template <int VS>
__global__ void __launch_bounds__(THREADS, 2)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const Params p) {
  constexpr int STAGE_BYTES = stage_bytes<VS>();
  constexpr int SF_BYTES = sf_bytes<VS>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_addr = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<int*>(tmem_addr + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;   // token tiles fastest: resident CTAs share B tiles in L2

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
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
      prefetch_tmap(&tmap_a);
      prefetch_tmap(&tmap_b);
      const uint8_t* sfa = p.sfa + (int64_t)blockIdx.x * p.sf_tile_bytes;
      const uint8_t* sfb = p.sfb + (int64_t)blockIdx.y * p.sf_tile_bytes;
      int issued = 0;
      for (int i = 0; i < p.ksteps; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, abort_flag, p.wait_limit)) break;
        uint8_t* st = base + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tma_load_2d(st, &tmap_a, &full[s], i * (KS / 2), m0);
        tma_load_2d(st + A_BYTES, &tmap_b, &full[s], i * (KS / 2), n0);
        bulk_load(st + A_BYTES + B_BYTES, sfa + (int64_t)i * SF_BYTES, SF_BYTES, &full[s]);
        bulk_load(st + A_BYTES + B_BYTES + SF_BYTES, sfb + (int64_t)i * SF_BYTES, SF_BYTES, &full[s]);
        issued = i + 1;
      }
      // no copy may still be landing when the CTA exits
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, abort_flag, p.wait_limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int i = 0; i < p.ksteps; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (!mbar_wait(&full[s], use & 1, abort_flag, p.wait_limit)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(base + s * STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
        const uint32_t sfa_addr = b_addr + B_BYTES, sfb_addr = sfa_addr + SF_BYTES;
#pragma unroll
        for (int at = 0; at < KS / atom_k<VS>(); ++at) {
          tmem_cp_atom(tmem + SFA_COL + 4 * at, sdesc_plain(sfa_addr + 512 * at, 16, 128));
          tmem_cp_atom(tmem + SFB_COL + 4 * at, sdesc_plain(sfb_addr + 512 * at, 16, 128));
        }
#pragma unroll
        for (int kk = 0; kk < KS / KBLK; ++kk) {
          // the atom holding this 64-element block's scales, and the byte of
          // its 4-byte group where they start (0, or 2 for the second half of
          // a 32-element-block atom)
          constexpr int PER_ATOM = atom_k<VS>() / KBLK;
          const uint32_t at = (uint32_t)(kk / PER_ATOM), byte = (uint32_t)((kk % PER_ATOM) * (4 / PER_ATOM));
          const uint32_t idesc = idesc_base<VS>() | (byte << 29) | (byte << 4);
          const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
          mma_fp4<VS>(tmem, ad, bd, idesc, (tmem + SFA_COL + 4 * at) | (byte << 30), (tmem + SFB_COL + 4 * at) | (byte << 30),
                      (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);
    }
  } else {
    // drain (warps 2-5): warp w reads TMEM lanes 32 (w % 4) .. +31 (one output
    // row per thread, 16 columns per load), scales them and stages its
    // 32 x 128 block in the idle stage buffers (row pitch 132 floats keeps the
    // 16-byte writes conflict-free), then writes it a row at a time: 32 lanes x
    // 16 bytes, one contiguous 512-byte row per store instruction.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.wait_limit) && !*abort_flag);
    const int quad = warp & 3;
    const float scale = p.sa ? __fmul_rn(*p.sa, *p.sb) : 1.0f;
    constexpr int PITCH = BN + 4;
    float* stage_out = reinterpret_cast<float*>(base) + quad * 32 * PITCH;
    if (ok) {
      tc_fence_after();
      for (int c16 = 0; c16 < BN / 16; ++c16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(c16 * 16), v);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(stage_out + lane * PITCH + c16 * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_float4(__fmul_rn(__uint_as_float(v[4 * q]), scale), __fmul_rn(__uint_as_float(v[4 * q + 1]), scale),
                               __fmul_rn(__uint_as_float(v[4 * q + 2]), scale),
                               __fmul_rn(__uint_as_float(v[4 * q + 3]), scale));
      }
      __syncwarp();
      const int col = n0 + 4 * lane;
      for (int rr = 0; rr < 32; ++rr) {
        const int row = m0 + quad * 32 + rr;
        if (row >= p.M) break;
        const float4 val = *reinterpret_cast<const float4*>(stage_out + rr * PITCH + 4 * lane);
        float* y = p.Y + (size_t)row * p.N + col;
        if ((p.N & 3) == 0 && col + 4 <= p.N) {
          *reinterpret_cast<float4*>(y) = val;
        } else {
          const float e[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (col + q < p.N) y[q] = e[q];
        }
      }
    }
  }
  if (warp == 1 && lane == 0 && *abort_flag) mbar_wait(acc_full, 0, abort_flag, p.wait_limit);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Row-major block scales [rows][K/VS] -> scale atoms [ceil(rows/128)][K/(4 VS)][512]
// (zero for the rows past `rows` that pad the last tile).
__global__ void __launch_bounds__(256) fp4_atoms_kernel(const uint8_t* __restrict__ sf, int64_t rows, int64_t K, int vs,
                                                        uint8_t* __restrict__ out, int64_t total) {
  pdl_wait();
  pdl_trigger();
  const int64_t kblocks = K / (4 * vs), per_row = K / vs;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t atom = idx >> 9;
    const int within = (int)(idx & 511);
    const int64_t t = atom / kblocks, q = atom % kblocks;
    const int mm0 = within >> 4, m1 = (within >> 2) & 3, kb = within & 3;
    const int64_t r = t * 128 + m1 * 32 + mm0;
    out[idx] = r < rows ? sf[r * per_row + q * 4 + kb] : (uint8_t)0;
  }
}

}  // namespace fp4g

size_t fp4_atoms_bytes(int64_t rows, int64_t K, int vs) {
  return (size_t)((rows + 127) / 128) * (size_t)(K / (4 * vs)) * 512;
}

ql_status launch_fp4_atoms(const uint8_t* scales, int64_t rows, int64_t K, int vs, uint8_t* atoms, cudaStream_t st) {
  const int64_t total = (int64_t)fp4_atoms_bytes(rows, K, vs);
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, (int64_t)sms * 8));
  TraceScope ts(TK_FP4, st);
  QL_CUDA_TRY(launch(fp4g::fp4_atoms_kernel, dim3(grid), dim3(256), 0, st, 1, 1, scales, rows, K, vs, atoms, total));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

template <int VS>
static ql_status launch_fp4_gemm_vs(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_ts,
                                    const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_ts, int64_t M,
                                    int64_t N, int64_t K, float* Y, cudaStream_t st) {
  using namespace fp4g;
  constexpr size_t SMEM = smem_bytes<VS>();
  if (per_device(reinterpret_cast<const void*>(fp4_gemm_kernel<VS>), 0, [] {
        if (cudaFuncSetAttribute(fp4_gemm_kernel<VS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM) !=
                cudaSuccess ||
            cudaFuncSetAttribute(fp4_gemm_kernel<VS>, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
                cudaSuccess) {
          cudaGetLastError();
          return -1;
        }
        return 1;
      }) < 0)
    return QL_ERR_CUDA;
  CUtensorMap map_a, map_b;
  if (!make_map_2d(&map_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a_codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2,
                   KS / 2, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&map_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b_codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                   KS / 2, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  Params p;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.ksteps = (int)(K / KS);
  p.sfa = a_atoms;
  p.sfb = b_atoms;
  p.sf_tile_bytes = (K / atom_k<VS>()) * 512;
  p.sa = a_ts;
  p.sb = b_ts;
  p.Y = Y;
  p.wait_limit = 1u << 22;
  const dim3 grid((unsigned)((M + BM - 1) / BM), (unsigned)((N + BN - 1) / BN));
  TraceScope ts(TK_FP4GEMM, st);
  QL_CUDA_TRY(launch(fp4_gemm_kernel<VS>, grid, dim3(THREADS), SMEM, st, 1, 1, map_a, map_b, p));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

ql_status launch_fp4_gemm(int vs, const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_ts,
                          const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_ts, int64_t M, int64_t N,
                          int64_t K, float* Y, cudaStream_t st) {
  return vs == 16 ? launch_fp4_gemm_vs<16>(a_codes, a_atoms, a_ts, b_codes, b_atoms, b_ts, M, N, K, Y, st)
                  : launch_fp4_gemm_vs<32>(a_codes, a_atoms, nullptr, b_codes, b_atoms, nullptr, M, N, K, Y, st);
}

}  // namespace ql
