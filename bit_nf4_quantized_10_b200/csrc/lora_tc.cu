// Rank-r adapter gradients on the tensor cores ("QLoRA — Fine-Tuning a 65B
// Model on One GPU", "Where the gradients actually go": only A and B receive
// gradients; "Prerequisite: LoRA's low-rank update": B is d x r, A is r x k):
//   dB = s dY^T U   [N, r]     dA = s V^T X   [r, K]
// and the rank-r side products U = bf16(X A^T), V = bf16(dY B).
//
// All three are skinny products C[rows x r] = Z_op[rows x red] * G[red x r]
// with r <= 64: tcgen05.mma with M = 128 output rows and N = r (padded to 16),
// the long reduction split over up to 8 CTAs (split-K) that form one
// thread-block cluster per row tile; the fp32 partials are summed across the
// cluster's shared memory in split order (deterministic), and the result is
// written row-major and/or transposed.
//   dB: Z_op = dY^T (MN-major view of dY [M, N]), G^T = U^T [r, M]
//   dA: Z_op = X^T  (MN-major view of X  [M, K]), G^T = V^T [r, M]
//   U:  Z_op = X    (K-major),                     G^T = A   [r, K]
//   V:  Z_op = dY   (K-major),                     G^T = B^T [r, N]
// They stream one activation matrix once, so they are bound by its HBM read.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

QL_DEFINE_STATUS_ACCESSOR(status_word_lora)

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                 uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

namespace skinny {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = 64 * BK * 2;   // 8 KB (r <= 64)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 6 * 32;        // TMA, MMA, 4 drain warps
constexpr int TMEM_COLS = 64;
// Ring depth.  The K-major form (U, V) has only M/128 row tiles (16 at 2048
// tokens), so a cluster of split CTAs per tile leaves one CTA per SM, whose
// ring alone must cover HBM latency: 8 stages (128 KB of activations in
// flight).  The MN-major form (dA, dB) has a row tile per 128 columns and two
// CTAs per SM, with 4 stages each.
template <bool A_MN>
__host__ __device__ constexpr int stages() { return A_MN ? 4 : 8; }
template <bool A_MN>
__host__ __device__ constexpr size_t smem_bytes() { return 1024 + (size_t)stages<A_MN>() * STAGE_BYTES + 256; }

constexpr int MAX_SPLITS = 8;           // portable cluster size

struct Params {
  int rows;             // output rows (M of the MMA)
  int r, rp;            // rank, padded to 16
  int steps_total;      // ceil(red / 64)
  int steps_per_split;
  float scale;
  void* out_row;        // [rows, r] of row_bf16 ? bf16 : fp32, or NULL
  int row_bf16;
  void* out_t;          // [r, ld_t] of t_bf16 ? bf16 : fp32, or NULL
  int ld_t;
  int t_bf16;
  uint32_t wait_limit;
};

// Final value of output row `row`, columns j .. j+3, written to both layouts.
__device__ __forceinline__ void store_out4(const Params& p, int row, int j, float4 v) {
  v.x = __fmul_rn(p.scale, v.x);
  v.y = __fmul_rn(p.scale, v.y);
  v.z = __fmul_rn(p.scale, v.z);
  v.w = __fmul_rn(p.scale, v.w);
  if (p.out_row) {
    if (p.row_bf16) {
      uint2 pk;
      pk.x = pack_bf16x2(v.x, v.y);
      pk.y = pack_bf16x2(v.z, v.w);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out_row) + (size_t)row * p.r + j) = pk;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out_row) + (size_t)row * p.r + j) = v;
    }
  }
  if (p.out_t) {
    const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (p.t_bf16) reinterpret_cast<__nv_bfloat16*>(p.out_t)[(size_t)(j + q) * p.ld_t + row] = __float2bfloat16_rn(f[q]);
      else reinterpret_cast<float*>(p.out_t)[(size_t)(j + q) * p.ld_t + row] = f[q];
    }
  }
}

template <bool A_MN>
__global__ void __launch_bounds__(THREADS, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const Params p) {
  constexpr int STAGES = stages<A_MN>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_addr = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<int*>(tmem_addr + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * BM;
  const int step0 = blockIdx.y * p.steps_per_split;
  const int nsteps = min(p.steps_per_split, p.steps_total - step0);

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
      const uint32_t tx = A_BYTES + p.rp * 128;
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, abort_flag, p.wait_limit)) break;
        const int k0 = (step0 + i) * BK;
        uint8_t* a = base + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], tx);
        if (!A_MN) {
          tma_load_2d(a, &tmap_a, &full[s], k0, row0);
        } else {
          tma_load_2d(a, &tmap_a, &full[s], row0, k0);
          tma_load_2d(a + 8192, &tmap_a, &full[s], row0 + 64, k0);
        }
        tma_load_2d(a + A_BYTES, &tmap_b, &full[s], k0, 0);
        issued = i + 1;
      }
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, abort_flag, p.wait_limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, p.rp, A_MN, false);
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (!mbar_wait(&full[s], use & 1, abort_flag, p.wait_limit)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(base + s * STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = A_MN ? sdesc_sw128(a_addr + kk * 2048, 8192, 1024) : sdesc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
          mma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);
    }
  } else {
    // drain (warps 2-5): this CTA's fp32 partial of its 128 rows into shared
    // memory (the stage buffers are idle once the last MMA has completed);
    // row stride rp + 4 floats keeps the 16-byte accesses conflict-free
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.wait_limit) && !*abort_flag);
    const int quad = warp & 3;
    const int lrow = quad * 32 + lane;
    float* red = reinterpret_cast<float*>(base);
    if (ok) tc_fence_after();
    for (int c16 = 0; c16 < p.rp / 16; ++c16) {
      uint32_t v[16];
      if (ok) {
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(c16 * 16), v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = 0u;
      }
      float4* dst = reinterpret_cast<float4*>(red + lrow * (p.rp + 4) + c16 * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                             __uint_as_float(v[4 * q + 3]));
    }
  }
  if (warp == 1 && lane == 0 && *abort_flag) mbar_wait(acc_full, 0, abort_flag, p.wait_limit);

  // The CTAs of one row tile (one per split of the reduction) form a cluster.
  // After every partial is in shared memory, CTA k of the cluster sums 1/splits
  // of the tile's (row, 4 columns) items over all CTAs of the cluster in split
  // order (so the result does not depend on scheduling) and writes them.
  cluster_sync();
  {
    const int splits = (int)gridDim.y;
    const int rank = (int)cluster_rank();
    const int c4s = p.rp / 4;
    const int items = BM * c4s;
    const int i0 = (int)((int64_t)items * rank / splits), i1 = (int)((int64_t)items * (rank + 1) / splits);
    const uint32_t red_base = smem_u32(base);
    for (int it = i0 + (int)threadIdx.x; it < i1; it += THREADS) {
      const int c4 = it / BM, lrow = it % BM;     // rows fastest: coalesced transposed stores
      const int row = row0 + lrow, j = c4 * 4;
      if (row >= p.rows || j >= p.r) continue;
      const uint32_t off = red_base + (uint32_t)((lrow * (p.rp + 4) + j) * 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < splits; ++sp) {
        const float4 x = ld_cluster_f4(cluster_map(off, (uint32_t)sp));
        acc.x = __fadd_rn(acc.x, x.x);
        acc.y = __fadd_rn(acc.y, x.y);
        acc.z = __fadd_rn(acc.z, x.z);
        acc.w = __fadd_rn(acc.w, x.w);
      }
      store_out4(p, row, j, acc);
    }
  }
  cluster_sync();   // no CTA leaves while another still reads its shared memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// dst [cols, ld_dst] = src [rows, cols]^T (bf16, cols = r <= 64, a multiple of
// 8): one thread per source row reads it with 16-byte loads; for each output
// row the warp's 32 consecutive source rows give 64 contiguous bytes.
// Row-per-thread transpose of a bf16 [rows, cols] matrix into [cols, ld_dst]
// (consecutive threads write consecutive columns of dst).  One launch can do
// two independent transposes: CTAs below `split` take the first matrix, the
// rest the second (the backward transposes B and U together).
struct TransposeJob {
  const uint16_t* src;
  int rows, cols;
  uint16_t* dst;
  int ld_dst;
};

__global__ void __launch_bounds__(256) transpose_kernel(TransposeJob j0, TransposeJob j1, int split) {
  pdl_wait();
  pdl_trigger();
  const bool first = (int)blockIdx.x < split;
  const TransposeJob& jb = first ? j0 : j1;
  const uint16_t* src = jb.src;
  const int rows = jb.rows, cols = jb.cols, ld_dst = jb.ld_dst;
  uint16_t* dst = jb.dst;
  const int row = (int)(first ? blockIdx.x : blockIdx.x - split) * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)row * cols);
  for (int c8 = 0; c8 < cols / 8; ++c8) {
    const uint4 v = s[c8];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dst[(size_t)(c8 * 8 + 2 * e) * ld_dst + row] = (uint16_t)(w[e] & 0xFFFFu);
      dst[(size_t)(c8 * 8 + 2 * e + 1) * ld_dst + row] = (uint16_t)(w[e] >> 16);
    }
  }
}

}  // namespace skinny

static int sm_count_tc() {
  const int c = device_sm_count();
  return c > 0 ? c : 148;
}

// One wave of clusters where the row tiles allow: the most splits (at most
// MAX_SPLITS, one cluster of CTAs per row tile) such that every tile's cluster
// is resident at once, per the occupancy calculator (a cluster's CTAs share a
// GPC); each split a whole number of 64-deep steps.
static void split_plan_compute(bool a_mn, int rows, int64_t red, int& splits, int& per) {
  const int tiles = (rows + skinny::BM - 1) / skinny::BM;
  const int steps = (int)((red + skinny::BK - 1) / skinny::BK);
  int want = std::max(1, std::min(std::min(2 * sm_count_tc() / tiles, steps), skinny::MAX_SPLITS));
  for (; want > 1; --want) {
    const int pw = (steps + want - 1) / want;
    const int sp = (steps + pw - 1) / pw;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tiles, (unsigned)sp);
    cfg.blockDim = dim3(skinny::THREADS);
    cfg.dynamicSmemBytes = a_mn ? skinny::smem_bytes<true>() : skinny::smem_bytes<false>();
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = (unsigned)sp;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = a_mn ? cudaOccupancyMaxActiveClusters(&n, skinny::skinny_kernel<true>, &cfg)
                               : cudaOccupancyMaxActiveClusters(&n, skinny::skinny_kernel<false>, &cfg);
    if (e != cudaSuccess) {
      cudaGetLastError();
      break;   // no answer: keep the arithmetic choice
    }
    if (n >= tiles) break;
  }
  per = (steps + want - 1) / want;
  splits = (steps + per - 1) / per;
}

// The plan depends only on the shape and the device; launches repeat the same
// few shapes.
static void split_plan(bool a_mn, int rows, int64_t red, int& splits, int& per) {
  struct Entry {
    bool a_mn;
    int rows;
    int64_t red;
    int dev;
    int splits, per;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(mu);
  for (const Entry& e : cache)
    if (e.a_mn == a_mn && e.rows == rows && e.red == red && e.dev == dev) {
      splits = e.splits;
      per = e.per;
      return;
    }
  split_plan_compute(a_mn, rows, red, splits, per);
  if (cache.size() < 256) cache.push_back(Entry{a_mn, rows, red, dev, splits, per});
}

// C = scale * Z_op G, see the file comment.  a_mn: Z_op is the transpose of a
// row-major [red, rows] array z (ld = rows); else Z_op = z, [rows, red].
// gt: G^T, row-major [r, red] with row pitch ld_gt.  C is written row-major
// to out_row [rows, r] and/or transposed to out_t [r, ld_t].
static ql_status skinny_launch(bool a_mn, const void* z, int rows, int64_t red, const void* gt, int r, int64_t ld_gt,
                               float scale, void* out_row, ql_dtype row_dt, void* out_t, int64_t ld_t, ql_dtype t_dt,
                               int kind, cudaStream_t st) {
  using namespace skinny;
  // two CTAs per SM need the largest shared-memory carveout (per-device attributes)
  auto k = a_mn ? skinny_kernel<true> : skinny_kernel<false>;
  const size_t smem = a_mn ? smem_bytes<true>() : smem_bytes<false>();
  if (per_device(reinterpret_cast<const void*>(k), 0, [k, smem] {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
            cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) {
          cudaGetLastError();
          return -1;
        }
        return 1;
      }) < 0)
    return QL_ERR_CUDA;
  const int rp = (r + 15) / 16 * 16;
  CUtensorMap ma, mb;
  if (a_mn) {
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, z, (uint64_t)rows, (uint64_t)red, (uint64_t)rows, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return QL_ERR_CUDA;
  } else {
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, z, (uint64_t)red, (uint64_t)rows, (uint64_t)red, BK, BM,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return QL_ERR_CUDA;
  }
  if (!make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, gt, (uint64_t)red, (uint64_t)r, (uint64_t)ld_gt, BK,
                   (uint32_t)rp, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  int splits, per;
  split_plan(a_mn, rows, red, splits, per);
  const int tiles = (rows + BM - 1) / BM;
  Params p;
  p.rows = rows;
  p.r = r;
  p.rp = rp;
  p.steps_total = (int)((red + BK - 1) / BK);
  p.steps_per_split = per;
  p.scale = scale;
  p.out_row = out_row;
  p.row_bf16 = row_dt == QL_BF16;
  p.out_t = out_t;
  p.ld_t = (int)ld_t;
  p.t_bf16 = t_dt == QL_BF16;
  p.wait_limit = 1u << 22;
  const dim3 grid((unsigned)tiles, (unsigned)splits);
  {
    TraceScope ts(kind, st);
    if (a_mn) QL_CUDA_TRY(launch(skinny_kernel<true>, grid, dim3(THREADS), smem, st, 1, (unsigned)splits, ma, mb, p));
    else QL_CUDA_TRY(launch(skinny_kernel<false>, grid, dim3(THREADS), smem, st, 1, (unsigned)splits, ma, mb, p));
  }
  return QL_OK;
}

// side = bf16(Z G): Z [M, red] (X or dY), G^T [r, ld_gt] (A or B^T);
// out [M, r] and/or out_t [r, ld_t], both bf16
ql_status launch_proj(const void* Z, int64_t M, int64_t red, const void* Gt, int64_t ld_gt, int r, void* out,
                      void* out_t, int64_t ld_t, cudaStream_t st) {
  return skinny_launch(false, Z, (int)M, red, Gt, r, ld_gt, 1.0f, out, QL_BF16, out_t, ld_t, QL_BF16, TK_PROJ, st);
}

// dB = s dY^T U: dY [M, N], U^T [r, ld_ut]; dB [N, r]
ql_status launch_grad_b(const void* dY, int64_t M, int N, const void* Ut, int64_t ld_ut, int r, float s, void* dB,
                        ql_dtype dt, cudaStream_t st) {
  return skinny_launch(true, dY, N, M, Ut, r, ld_ut, s, dB, dt, nullptr, 0, dt, TK_COLACC, st);
}

// dA = s V^T X: X [M, K], V^T [r, ld_vt]; dA [r, K]
ql_status launch_grad_a(const void* X, int64_t M, int K, const void* Vt, int64_t ld_vt, int r, float s, void* dA,
                        ql_dtype dt, cudaStream_t st) {
  return skinny_launch(true, X, K, M, Vt, r, ld_vt, s, nullptr, dt, dA, K, dt, TK_COLACC, st);
}

// dst [cols, ld_dst] = src [rows, cols]^T, bf16; two transposes in one launch
// (the second may be empty: src1 == NULL).
ql_status launch_transpose2(const void* src0, int64_t rows0, int cols0, void* dst0, int64_t ld0, const void* src1,
                            int64_t rows1, int cols1, void* dst1, int64_t ld1, cudaStream_t st) {
  if (cols0 % 8 != 0 || rows0 <= 0) return QL_ERR_UNSUPPORTED;
  if (src1 && (cols1 % 8 != 0 || rows1 <= 0)) return QL_ERR_UNSUPPORTED;
  const int g0 = (int)((rows0 + 255) / 256), g1 = src1 ? (int)((rows1 + 255) / 256) : 0;
  const skinny::TransposeJob j0{(const uint16_t*)src0, (int)rows0, cols0, (uint16_t*)dst0, (int)ld0};
  const skinny::TransposeJob j1{(const uint16_t*)src1, (int)rows1, cols1, (uint16_t*)dst1, (int)ld1};
  TraceScope ts(TK_TRANSPOSE, st);
  QL_CUDA_TRY(launch(skinny::transpose_kernel, dim3((unsigned)(g0 + g1)), dim3(256), 0, st, 1, 1, j0, j1, g0));
  return QL_OK;
}

ql_status launch_transpose(const void* src, int64_t rows, int cols, void* dst, int64_t ld_dst, cudaStream_t st) {
  return launch_transpose2(src, rows, cols, dst, ld_dst, nullptr, 0, 0, nullptr, 0, st);
}

}  // namespace ql
