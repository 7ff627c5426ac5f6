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
//   forward  Y  = X  * W_hat^T + U * (s B)^T      reduction over K (W columns)
//   backward dX = dY * W_hat   + V * (s A)        reduction over N (W rows)
// U = bf16(X A^T) and V = bf16(dY B) come in precomputed (rank-r side kernels).
//
// Two CTAs on two SMs form a pair (a cluster of 2) that shares one tile of 256
// output columns: each CTA expands only its half of the weight tile (128
// output columns), and one thread of the even CTA issues cta_group::2 MMAs
// (M = 256, N = 256) that read both halves.  Each CTA holds 256 tokens as two
// M = 128 halves, so a pair instruction pairs the even CTA's half h with the
// odd CTA's half h, into TMEM columns 0-255 (h = 0) and 256-511 (h = 1) of
// each CTA.  Per expanded weight element this is 512 multiply-adds on each SM,
// and each SM's tensor core reads only its own 128 rows of B from its shared
// memory: half the expansion work and half the operand reads of a single-CTA
// 256 x 256 tile, which is what bounded the single-CTA form.
// The r LoRA K-steps (U or V against the scaled adapter) run into the same
// accumulators after the main loop, before the drain.
//
// Shared memory per CTA: rings of 4 activation tiles (256 x 64 bf16), 8
// packed-code tiles of the CTA's 128 x 64 weight half (loaded 4 stages ahead,
// so expanding a stage never waits on a TMA) and 4 expanded weight halves.
// Synchronisation: TMA loads complete on local barriers (full_a, full_c); each
// producer warp, in both CTAs, arrives on the even CTA's full_b[s] (8 warps)
// once its part of the weight tile is written (in the odd CTA, also once the
// CTA's activation tile of the stage has landed); the MMA commits multicast
// to empty[s] and acc_full in both CTAs.
// Warp roles (576 threads per CTA):
//   warp 0      TMA producer
//   warp 1      TMEM allocation (both CTAs); one thread of the even CTA
//               issues the MMAs
//   warps 2-17  dequant producers, four groups of 4 warps on stages
//               g, g+4, ...; each thread expands one 64-block (levels from a
//               shared fp32 table, times the block constant, packed to bf16)
//               into the swizzled BF16 tile;
//               then the LoRA operands; then all 16 warps drain TMEM
//               (a bf16 output is staged in the idle activation ring and
//               leaves by bulk tensor stores, 128-byte lines).
// The weight tile holds W rows as 128-byte rows in both directions: K-major
// for the forward (rows = output features), MN-major for the backward (rows =
// the reduction index), so the producers write the same layout either way.
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

namespace gemm {

constexpr int BM = 256;                 // tokens per CTA (two M = 128 halves)
constexpr int BMH = 128;
constexpr int BN = 256;                 // output columns per pair
constexpr int BNH = 128;                // output columns expanded by one CTA
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;    // 32 KB activation tile
constexpr int AH_BYTES = BMH * BK * 2;  // 16 KB: the second half
constexpr int B_BYTES = BNH * BK * 2;   // 16 KB expanded weight half
constexpr int C_BYTES = BNH * BK / 2;   // 4 KB of packed codes
constexpr int STAGES = 4;               // activation and expanded-weight rings
constexpr int C_STAGES = 8;             // packed-code ring, filled 4 stages ahead
constexpr int C_AHEAD = C_STAGES - STAGES;
constexpr int GROUPS = 4;               // producer groups, one stage each in turn
constexpr int GROUP_WARPS = 4;
constexpr int PRODUCER_WARPS = GROUPS * GROUP_WARPS;
constexpr int THREADS = (2 + PRODUCER_WARPS) * 32;
constexpr int TMEM_COLS = 512;
constexpr size_t SMEM_BYTES =
    1024 + (size_t)STAGES * A_BYTES + (size_t)C_STAGES * C_BYTES + (size_t)STAGES * B_BYTES + 256;

struct Params {
  int M;             // tokens
  int n_out;         // output columns (N forward, K backward)
  int n_steps;       // main-loop stages (K/64 forward, ceil(N/64) backward)
  int N, K;          // weight shape
  WeightConsts wc;
  int r, rp;         // rank, rank padded to 16 (0 when no adapter)
  float s;
  const __nv_bfloat16* lora_a;   // forward U [M, r]; backward V [M, r]
  const __nv_bfloat16* lora_b;   // forward B [N, r]; backward A [r, K]; scaled by s here
  void* out;
  int out_bf16;
  int accumulate;
  int tma_store;     // bf16 output written through shared memory by bulk tensor stores
  int token_fast;    // tile order: token tiles of a column tile consecutive
  NF4Table tab;
  uint32_t wait_limit;
};

struct Smem {
  uint8_t* base;
  __device__ __forceinline__ uint8_t* a(int s) const { return base + s * A_BYTES; }
  __device__ __forceinline__ uint8_t* b(int s) const { return base + STAGES * A_BYTES + s * B_BYTES; }
  __device__ __forceinline__ uint8_t* c(int s) const { return base + STAGES * (A_BYTES + B_BYTES) + s * C_BYTES; }
  uint64_t* full_a;    // [STAGES] activation tile landed (local TMA)
  uint64_t* full_c;    // [C_STAGES] packed codes landed (local TMA)
  uint64_t* full_b;    // [STAGES] even CTA: both CTAs' weight halves written and activations landed
  uint64_t* empty;     // [STAGES] pair MMA done with the stage (commit to both CTAs)
  uint64_t* acc_full;
  uint32_t* tmem_addr;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.base = p;
  p += STAGES * (A_BYTES + B_BYTES) + C_STAGES * C_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p);
  s.full_a = bars;
  s.full_c = bars + STAGES;
  s.full_b = s.full_c + C_STAGES;
  s.empty = s.full_b + STAGES;
  s.acc_full = s.empty + STAGES;
  s.tmem_addr = reinterpret_cast<uint32_t*>(s.acc_full + 1);
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

// Raw constant of one 64-block, loaded a stage ahead of use: the fp32 absmax,
// or the E4M3 code and group scale of the double-quantized form.
struct RawConst {
  float v;      // absmax, or the group scale s2
  uint32_t e;   // E4M3 code (double quant)
};

__device__ __forceinline__ RawConst load_const(const WeightConsts& wc, int64_t b, bool valid) {
  RawConst r{0.0f, 0u};
  if (!valid) return r;
  if (wc.absmax) {
    r.v = __ldg(wc.absmax + b);
  } else {
    r.e = __ldg(wc.absmax_q + b);
    r.v = __ldg(wc.scale2 + (b >> 8));
  }
  return r;
}

__device__ __forceinline__ float decode_const(const WeightConsts& wc, RawConst r, float mu) {
  if (wc.absmax) return r.v;
  return __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)r.e), r.v), mu);
}

__device__ __forceinline__ uint64_t b_desc(uint32_t b_addr, int kk, bool bwd) {
  return bwd ? sdesc_sw128(b_addr + kk * 2048, 8192, 1024) : sdesc_sw128(b_addr + kk * 32, 16, 1024);
}

template <bool BWD>
__global__ void __launch_bounds__(THREADS, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_codes,
                      const __grid_constant__ CUtensorMap tmap_out, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // the 16 fp32 levels, 256-byte aligned: an LDS address is the table base with
  // the level's byte offset (4 * code) in its low byte
  __shared__ __align__(256) float qlev[64];
  if (threadIdx.x < 16) qlev[threadIdx.x] = p.tab.q[threadIdx.x];
  Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();          // 0 = even CTA (issues the MMAs)
  // The pair's tile.  Pairs are dispatched roughly in order of their linear
  // index; with token_fast the token tiles of one column tile are consecutive,
  // so that column tile's codes come from DRAM once and from L2 for the other
  // token tiles (for outputs much wider than the token count, whose codes do
  // not stay in L2 across a whole pass over the columns).
  int col_tile = blockIdx.x >> 1, tok_tile = blockIdx.y;
  if (p.token_fast) {
    const int pidx = blockIdx.y * (gridDim.x >> 1) + (blockIdx.x >> 1);
    tok_tile = pidx % gridDim.y;
    col_tile = pidx / gridDim.y;
  }
  const int j0 = col_tile * BN;                  // the pair's output-column tile
  const int jb = j0 + (int)rank * BNH;           // this CTA's weight half
  const int m0 = tok_tile * (2 * BM) + (int)rank * BM;   // this CTA's 256 tokens
  const bool lora = p.r > 0;
  volatile int* abort_flag = sm.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&sm.full_a[i], 1);
      mbar_init(&sm.full_b[i], 2 * GROUP_WARPS);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < C_STAGES; ++i) mbar_init(&sm.full_c[i], 1);
    mbar_init(sm.acc_full, 1);
    *sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_act);
    prefetch_tmap(&tmap_codes);
    if (p.tma_store) prefetch_tmap(&tmap_out);
  }
  if (warp == 1) {
    tmem_alloc2(sm.tmem_addr, TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_addr;
  pdl_wait();       // earlier kernels on the stream are complete from here on
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA warp
    // Codes run C_AHEAD stages ahead of the activations.  The code slot of
    // stage j was last used by stage j - 8, whose producers read it before
    // the pair MMA of stage j - 8 could start; codes for stage j are issued
    // after waiting for that MMA (the activation slot wait for stage j - 4).
    if (lane == 0) {
      auto load_codes = [&](int j) {
        const int c = j % C_STAGES;
        mbar_arrive_expect_tx(&sm.full_c[c], C_BYTES);
        if (!BWD)
          tma_load_2d(sm.c(c), &tmap_codes, &sm.full_c[c], j * (BK / 2), jb);
        else
          tma_load_2d(sm.c(c), &tmap_codes, &sm.full_c[c], jb / 2, j * BK);
      };
      int issued_c = 0, issued_a = 0;
      for (; issued_c < C_AHEAD && issued_c < p.n_steps; ++issued_c) load_codes(issued_c);
      for (int i = 0; i < p.n_steps; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        if (use > 0 && !mbar_wait(&sm.empty[s], (use - 1) & 1, abort_flag, p.wait_limit)) break;
        mbar_arrive_expect_tx(&sm.full_a[s], A_BYTES);
        tma_load_2d(sm.a(s), &tmap_act, &sm.full_a[s], i * BK, m0);
        issued_a = i + 1;
        if (i + C_AHEAD < p.n_steps) {
          load_codes(i + C_AHEAD);
          issued_c = i + C_AHEAD + 1;
        }
      }
      // before leaving, make sure no copy is still landing in shared memory
      for (int i = (issued_a > STAGES ? issued_a - STAGES : 0); i < issued_a; ++i)
        mbar_wait(&sm.full_a[i % STAGES], (i / STAGES) & 1, abort_flag, p.wait_limit);
      for (int j = (issued_c > C_STAGES ? issued_c - C_STAGES : 0); j < issued_c; ++j)
        mbar_wait(&sm.full_c[j % C_STAGES], (j / C_STAGES) & 1, abort_flag, p.wait_limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t IDESC = idesc_bf16(2 * BMH, BN, false, BWD);
      bool ok = true;
      for (int i = 0; i < p.n_steps && ok; ++i) {
        const int s = i % STAGES, use = i / STAGES;
        ok = mbar_wait(&sm.full_a[s], use & 1, abort_flag, p.wait_limit) &&
             mbar_wait_cluster(&sm.full_b[s], use & 1, abort_flag, p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sm.a(s));
        const uint32_t b_addr = smem_u32(sm.b(s));
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = b_desc(b_addr, kk, BWD);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_bf16_pair(tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024), bd, IDESC, acc);
          mma_bf16_pair(tmem + 256, sdesc_sw128(a_addr + AH_BYTES + kk * 32, 16, 1024), bd, IDESC, acc);
        }
        mma_commit_pair(&sm.empty[s]);
      }
      if (ok && lora) {
        // LoRA K-steps: A = U or V tile, B = scaled adapter, into both accumulators
        const int i = p.n_steps;
        const int s = i % STAGES, use = i / STAGES;
        ok = mbar_wait_cluster(&sm.full_b[s], use & 1, abort_flag, p.wait_limit);
        if (ok) {
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm.a(s));
          const uint32_t b_addr = smem_u32(sm.b(s));
          for (int kk = 0; kk < p.rp / 16; ++kk) {
            const uint64_t bd = b_desc(b_addr, kk, BWD);
            mma_bf16_pair(tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024), bd, IDESC, 1u);
            mma_bf16_pair(tmem + 256, sdesc_sw128(a_addr + AH_BYTES + kk * 32, 16, 1024), bd, IDESC, 1u);
          }
        }
      }
      mma_commit_pair(sm.acc_full);
    }
  } else {
    // ------------------------------------------------------ dequant producers
    // Group g (4 warps, 128 threads) expands stages g, g+4, ...: thread t owns
    // one 64-block of the CTA's 128 x 64 weight half.
    // fwd: thread t owns weight row jb + t (the stage is 64-block i of the row);
    // bwd: thread t owns weight row i*64 + t % 64 and the 64-column chunk t / 64
    // of the CTA's 128 columns.  Consecutive lanes take consecutive rows, so the
    // swizzled shared-memory stores below are free of bank conflicts.
    const int wp = warp - 2;                 // 0..15
    const int grp = wp / GROUP_WARPS;        // producer group
    const int gt = ((wp % GROUP_WARPS) << 5) | lane;   // thread within the group, 0..127
    const int kblocks = p.K / 64;            // 64-blocks per weight row
    const float mu = p.wc.absmax ? 0.0f : *p.wc.offset;
    const uint32_t qbase = opaque_after_barrier(smem_u32(qlev));   // low byte 0
    int row_in_tile, col_chunk;
    if (!BWD) { row_in_tile = gt; col_chunk = 0; }
    else { row_in_tile = gt & 63; col_chunk = gt >> 6; }
    // byte offsets of this thread's two 16-byte code chunks in the code tile
    uint32_t coff0, coff1;
    if (!BWD) {   // 32-byte rows, 32B swizzle: chunk ^= bit 2 of the row
      const uint32_t x = (row_in_tile >> 2) & 1;
      coff0 = row_in_tile * 32 + ((0 ^ x) << 4);
      coff1 = row_in_tile * 32 + ((1 ^ x) << 4);
    } else {      // 64-byte rows (the CTA's 128 columns), no swizzle
      coff0 = row_in_tile * 64 + col_chunk * 32;
      coff1 = coff0 + 16;
    }
    // byte offsets of the 8 16-byte chunks this thread writes in a weight tile
    uint32_t boff[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) boff[j] = (BWD ? col_chunk * 8192 : 0) + sw128_offset(row_in_tile, j);
    auto step_row = [&](int i, int& wrow, int& kb) {
      if (!BWD) { wrow = jb + row_in_tile; kb = i; }
      else { wrow = i * BK + row_in_tile; kb = jb / 64 + col_chunk; }
    };
    int wrow, kb;
    step_row(grp, wrow, kb);
    bool valid = grp < p.n_steps && wrow < p.N && kb < kblocks;
    RawConst next = load_const(p.wc, (int64_t)wrow * kblocks + kb, valid);
    bool ok = true;
    for (int i = grp; i < p.n_steps && ok; i += GROUPS) {
      const int s = i % STAGES, use = i / STAGES;
      const RawConst cur = next;
      const bool cur_valid = valid;
      if (i + GROUPS < p.n_steps) {   // constants of this group's next stage
        step_row(i + GROUPS, wrow, kb);
        valid = wrow < p.N && kb < kblocks;
        next = load_const(p.wc, (int64_t)wrow * kblocks + kb, valid);
      }
      // the stage's codes landed, and the pair MMA is done with the slot's previous use
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.full_c[i % C_STAGES], (i / C_STAGES) & 1, abort_flag, p.wait_limit) &&
                                       (use == 0 || mbar_wait(&sm.empty[s], (use - 1) & 1, abort_flag, p.wait_limit)));
      if (!ok) break;
      uint8_t* base = sm.b(s);
      const uint8_t* cs = sm.c(i % C_STAGES);
      if (cur_valid) {
        const uint4 c0 = *reinterpret_cast<const uint4*>(cs + coff0);
        const uint4 c1 = *reinterpret_cast<const uint4*>(cs + coff1);
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        // w_hat = bf16(fl32(q[code] * c)): the level from the shared table (one
        // byte permute forms the address), a packed pair of RN fp32 products,
        // one conversion per pair
        const float c = decode_const(p.wc, cur, mu);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t e4 = (w[j] << 2) & 0x3C3C3C3Cu;   // 4 * low nibble of each byte
          const uint32_t o4 = (w[j] >> 2) & 0x3C3C3C3Cu;   // 4 * high nibble of each byte
          uint32_t o[4];
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            const float fe = lds_f32_const(__byte_perm(e4, qbase, 0x7650u | bb));
            const float fo = lds_f32_const(__byte_perm(o4, qbase, 0x7650u | bb));
            float pe, po;
            mul2_rn(fe, fo, c, pe, po);
            o[bb] = pack_bf16x2(pe, po);
          }
          *reinterpret_cast<uint4*>(base + boff[j]) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(base + boff[j]) = zero4();
      }
      fence_proxy_async_smem();
      // the odd CTA's arrival also vouches for its activation tile of the stage
      if (rank != 0) ok = __all_sync(0xffffffffu, mbar_wait(&sm.full_a[s], use & 1, abort_flag, p.wait_limit));
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive_cluster(&sm.full_b[s], 0);
    }
    const int pt = gt;
    // LoRA operands into the slot after the last main step, written by the
    // group whose turn that step is
    if (ok && lora && grp == (p.n_steps % GROUPS)) {
      const int i = p.n_steps;
      const int s = i % STAGES, use = i / STAGES;
      ok = __all_sync(0xffffffffu, use == 0 || mbar_wait(&sm.empty[s], (use - 1) & 1, abort_flag, p.wait_limit));
      if (ok) {
        // A operand: U or V rows m0 .. m0+255, K-major (256 rows x rp), two rows per thread
        for (int row = pt; row < BM; row += 128) {
          const int m = m0 + row;
          for (int chunk = 0; chunk < 8; ++chunk) {
            const int e = chunk * 8;
            if (e >= p.rp) break;
            uint4 v = zero4();
            if (m < p.M && e < p.r) v = *reinterpret_cast<const uint4*>(p.lora_a + (size_t)m * p.r + e);
            *reinterpret_cast<uint4*>(sm.a(s) + (row >> 7) * AH_BYTES + sw128_offset(row & 127, chunk)) = v;
          }
        }
        if (!BWD) {
          // B operand: (s B)[n, 0..rp) for the CTA's 128 output features, K-major
          const int n = jb + pt;
          for (int chunk = 0; chunk < 8; ++chunk) {
            const int e = chunk * 8;
            if (e >= p.rp) break;
            uint4 v = zero4();
            if (n < p.N && e < p.r) v = scale8(*reinterpret_cast<const uint4*>(p.lora_b + (size_t)n * p.r + e), p.s);
            *reinterpret_cast<uint4*>(sm.b(s) + sw128_offset(pt, chunk)) = v;
          }
        } else {
          // B operand: (s A)[0..rp, k] for the CTA's 128 output columns, MN-major
          for (int idx = pt; idx < p.rp * 16; idx += 128) {
            const int jr = idx >> 4, rem = idx & 15;
            const int cc = rem >> 3, piece = rem & 7;
            const int k = jb + cc * 64 + piece * 8;
            uint4 v = zero4();
            if (jr < p.r && k < p.K) v = scale8(*reinterpret_cast<const uint4*>(p.lora_b + (size_t)jr * p.K + k), p.s);
            *reinterpret_cast<uint4*>(sm.b(s) + cc * 8192 + sw128_offset(jr, piece)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(&sm.full_b[s], 0);
      }
    }
    // ------------------------------------------------------------ epilogue
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(sm.acc_full, 0, abort_flag, p.wait_limit) && !*abort_flag);
    if (p.tma_store) {
      // bf16 output through shared memory.  Once the accumulators are complete
      // no MMA reads the rings any more, so the activation ring holds the
      // CTA's 256 x 256 bf16 tile: group g (TMEM half g >> 1, columns
      // (g & 1) * 128 ..) writes its 128 rows x 128 columns as two boxes of 64
      // columns in the 128-byte swizzled layout of the output tensor map, and
      // one thread of the group stores them with two bulk tensor copies (the
      // copy skips rows and columns outside the output).
      const int quad = warp & 3;
      const int g = wp >> 2;
      const int accn = g >> 1;
      const int lrow = quad * 32 + lane;
      uint8_t* box0 = sm.base + g * 2 * (BMH * 128);
      if (acc_ok) {
        tc_fence_after();
        for (int cc = 0; cc < 8; ++cc) {
          const int col = (g & 1) * 128 + cc * 16;
          uint32_t r[16];
          tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(accn * 256 + col), r);
          tmem_ld_wait();
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) pk[q] = pack_bf16x2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
          uint8_t* box = box0 + (cc >> 2) * (BMH * 128);
          const int ch = (cc & 3) * 2;
          *reinterpret_cast<uint4*>(box + sw128_offset(lrow, ch)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(box + sw128_offset(lrow, ch + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        fence_proxy_async_smem();
      }
      // every warp of the group reaches this barrier, whatever its waits returned
      __syncwarp();
      asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory");
      if ((wp & 3) == 0 && lane == 0 && acc_ok && !*abort_flag) {
        const int y = m0 + accn * BMH;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int x = j0 + (g & 1) * 128 + b * 64;
          if (x < p.n_out && y < p.M) tma_store_2d(&tmap_out, box0 + b * (BMH * 128), x, y);
        }
        bulk_commit();
        bulk_wait_all();
      }
    } else if (acc_ok) {
      tc_fence_after();
      const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31
      const int g = wp >> 2;                     // 0..3: half g>>1, columns (g&1)*128 ..
      const int accn = g >> 1;
      const int row = m0 + accn * BMH + quad * 32 + lane;
      for (int cc = 0; cc < 8; ++cc) {
        const int col = (g & 1) * 128 + cc * 16;
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(accn * 256 + col), r);
        tmem_ld_wait();
        const int gcol = j0 + col;
        if (row < p.M && gcol < p.n_out) {
          // n_out is a multiple of 8: the last chunk of a row may hold 8 columns
          const bool full16 = gcol + 16 <= p.n_out;
          const size_t off = (size_t)row * p.n_out + gcol;
          if (p.out_bf16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + off;
            uint32_t pk[8];
            if (p.accumulate) {
              const uint4 o0 = *reinterpret_cast<const uint4*>(o);
              const uint4 o1 = full16 ? *reinterpret_cast<const uint4*>(o + 8) : zero4();
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
            if (full16) reinterpret_cast<uint4*>(o)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          } else {
            float* o = reinterpret_cast<float*>(p.out) + off;
            const int nq = full16 ? 4 : 2;
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(r[q]);
            if (p.accumulate) {
#pragma unroll
              for (int q = 0; q < 16; ++q)
                if (q < 4 * nq) v[q] = __fadd_rn(v[q], o[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q < nq)
                reinterpret_cast<float4*>(o)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp == 1 && lane == 0 && rank == 0 && *abort_flag) {
    // let MMAs already issued finish before the accumulators are released
    mbar_wait(sm.acc_full, 0, abort_flag, p.wait_limit);
  }
  tc_fence_before();
  cluster_sync();   // neither CTA leaves while the pair's MMAs or arrivals may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, TMEM_COLS);
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

// 2-D tensor map over a row-major [rows, cols] array with row pitch `ld`
// elements (ld >= cols; ld * elem_bytes must be a multiple of 16).
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                 uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * (uint64_t)elem_bytes};
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
  // the shared-memory limit is a per-device attribute of the kernel
  if (per_device(reinterpret_cast<const void*>(qlora_gemm_kernel<BWD>), 0, [] {
        if (cudaFuncSetAttribute(qlora_gemm_kernel<BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES) != cudaSuccess) {
          cudaGetLastError();
          return -1;
        }
        return 1;
      }) < 0)
    return QL_ERR_CUDA;
  const int N = (int)w->rows, K = (int)w->cols;
  CUtensorMap map_act, map_codes, map_out;
  const int red = BWD ? N : K;   // reduction length = activation row length
  if (!make_map_2d(&map_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, act, (uint64_t)red, (uint64_t)M, (uint64_t)red, BK,
                   BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  if (!BWD) {
    if (!make_map_2d(&map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)K / 2, (uint64_t)N,
                     (uint64_t)K / 2, BK / 2, BNH, CU_TENSOR_MAP_SWIZZLE_32B))
      return QL_ERR_CUDA;
  } else {
    if (!make_map_2d(&map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)K / 2, (uint64_t)N,
                     (uint64_t)K / 2, BNH / 2, BK, CU_TENSOR_MAP_SWIZZLE_NONE))
      return QL_ERR_CUDA;
  }
  Params p;
  p.M = (int)M;
  p.n_out = BWD ? K : N;
  p.n_steps = BWD ? (N + BK - 1) / BK : K / BK;
  p.N = N;
  p.K = K;
  p.wc = WeightConsts{w->absmax, w->absmax_q, w->scale2, w->offset};
  p.r = r;
  p.rp = r > 0 ? (r + 15) / 16 * 16 : 0;
  p.s = s;
  p.lora_a = (const __nv_bfloat16*)lora_a;
  p.lora_b = (const __nv_bfloat16*)lora_b;
  p.out = out;
  p.out_bf16 = out_dt == QL_BF16;
  p.accumulate = accumulate;
  // bf16 output that is written, not accumulated: bulk tensor stores of
  // 64-column boxes, 128 rows high
  p.tma_store = out_dt == QL_BF16 && !accumulate && (reinterpret_cast<uintptr_t>(out) & 15) == 0 &&
                make_map_2d(&map_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, (uint64_t)p.n_out, (uint64_t)M,
                            (uint64_t)p.n_out, 64, BMH, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!p.tma_store) memset(&map_out, 0, sizeof(map_out));
  p.tab = nf4_table();
  p.wait_limit = 1u << 22;
  // token tiles first when the weight side is the larger operand and the
  // activations (all token tiles) fit in half of L2
  p.token_fast = (int64_t)M * red * 2 <= (int64_t)64 << 20 && (int64_t)p.n_out > 4 * M;
  const dim3 grid(2u * (unsigned)((p.n_out + BN - 1) / BN), (unsigned)((M + 2 * BM - 1) / (2 * BM)));
  TraceScope ts(BWD ? TK_GEMM_BWD : TK_GEMM_FWD, st);
  QL_CUDA_TRY(launch(qlora_gemm_kernel<BWD>, grid, dim3(THREADS), SMEM_BYTES, st, 2, 1, map_act, map_codes, map_out, p));
  return QL_OK;
}

// Y = X W_hat^T + U (s B)^T, U = bf16(X A^T) given [M, r]
ql_status launch_gemm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* U, const void* B, int r,
                          float s, void* Y, ql_dtype y_dt, cudaStream_t st) {
  return launch_gemm_impl<false>(w, X, M, U, B, r, s, Y, y_dt, 0, st);
}

// dX (+)= dY W_hat + V (s A), V = bf16(dY B) given [M, r]
ql_status launch_gemm_bwd(const ql_nf4_weight* w, const void* dY, int64_t M, const void* V, const void* A, int r,
                          float s, void* dX, ql_dtype dx_dt, int accumulate, cudaStream_t st) {
  return launch_gemm_impl<true>(w, dY, M, V, A, r, s, dX, dx_dt, accumulate, st);
}

}  // namespace ql
