// Small-token forward: Y = X * W_hat^T + s * U * B^T, U = bf16(X * A^T), for
// M <= 16 tokens.
//
// With a handful of tokens each dequantized weight element meets at most 16
// activations, so the layer is bound by reading the packed 4-bit weight from
// HBM ("QLoRA — Fine-Tuning a 65B Model on One GPU", "Pitfalls":
// memory-bandwidth-bound generation has less to read with 4-bit weights) and
// by the work of expanding it, which must keep pace with HBM.  On this part
// the expansion's floor is the shared-memory read of one fp32 NF4 level per
// element (128 bytes per clock per SM), so everything else is kept off the
// shared-memory and issue budget:
//   * No staging of the expanded weight: each thread expands its codes straight
//     into the A-operand registers of warp-level tensor-core MMAs
//     (mma.sync m16n8k16, bf16 in, fp32 accumulate), weight rows as M = 16 and
//     tokens as N = 8 (one or two token tiles).
//   * The reduction dimension is permuted so that each thread reads 8
//     contiguous code bytes (16 codes) of a 64-block per row: for k-step u of
//     block j, thread quad-index t's MMA slots {2t, 2t+1} and {2t+8, 2t+9} hold
//     the elements at k = 64 j + 16 t + 4 u + {0, 1} and {2, 3}.  The
//     activation fragments use the same permutation, so every k is summed once.
//   * K is split over the 16 warps of a CTA (KV codes per row each) and over
//     parts of K handled by different CTAs; each warp keeps the activation
//     fragments of its K range in registers for the whole kernel and walks the
//     CTA's row blocks.  A row block's codes and block constants reach the
//     warp through its own ring of STAGES shared-memory buffers filled by
//     cp.async, STAGES - 1 row blocks ahead (about 48-96 KB per SM in flight,
//     what HBM latency times bandwidth asks for).  The 16 warps' partial sums
//     meet in shared memory in warp order; each part's sums go to the
//     workspace.
//   * The CTA that owns the last row block of each part also computes that
//     part's share of U = X A^T with the same fragments (A rows as M).
//   * A second kernel sums the parts in order, rounds U to bf16, adds
//     s * (U B^T) in fp32 and writes Y (and U).
// Every sum has a fixed order, so results do not depend on scheduling.  There
// are no inter-CTA waits: the kernels only use __syncthreads.
#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

QL_DEFINE_STATUS_ACCESSOR(status_word_smallm)

namespace smallm {

constexpr int WARPS = 16;
constexpr int THREADS = WARPS * 32;
constexpr int MAX_M = 16;
constexpr int MAX_R = 64;

struct Params {
  int M, N, K, r;
  int kb;            // K / 64 (blocks per weight row)
  int cw_two;        // a warp's E4M3 constants of a row can span two words or two groups (K / 64 % 4 != 0)
  int parts;         // CTAs' K parts
  int part_k;        // reduction elements per part (WARPS * KV)
  int row_blocks;    // ceil(N / (16 T))
  WeightConsts wc;
  NF4Table tab;
  const uint8_t* codes;
  const __nv_bfloat16* X;    // [M, K]
  const __nv_bfloat16* A;    // [r, K]
  float* part_y;             // [parts][N][M] fp32
  float* part_u;             // [parts][M][r] fp32
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// {c, c} in one 64-bit register, the multiplier of a packed product.
__device__ __forceinline__ uint64_t pack_cc(float c) {
  uint64_t cc;
  asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
  return cc;
}

// Two codes (the low and high nibble of byte b of `w`) -> bf16x2 of
// bf16(fl32(q * c)), the low code in the low half.  e4 / o4 hold 4 * low / high
// nibble of each byte; the level table's low address byte is replaced by it.
// cc = {c, c}: one packed instruction takes both fp32 products.
__device__ __forceinline__ uint32_t expand_pair(uint32_t e4, uint32_t o4, uint32_t qbase, uint32_t sel, uint64_t cc) {
  const float lo = lds_f32_const(__byte_perm(e4, qbase, sel));
  const float hi = lds_f32_const(__byte_perm(o4, qbase, sel));
  float pl, ph;
  asm("{\n .reg .b64 x, z;\n mov.b64 x, {%2, %3};\n mul.rn.f32x2 z, x, %4;\n mov.b64 {%0, %1}, z;\n}"
      : "=f"(pl), "=f"(ph)
      : "f"(lo), "f"(hi), "l"(cc));
  return pack_bf16x2(pl, ph);
}

// Ring stages per warp, and the bytes of one stage: 16 T rows of KV / 2 code
// bytes, then the block constants of those rows: four words per row for E4M3
// constants (two code words, two group scales), KV / 64 words per row for
// plain fp32 constants (layouts at issue_codes).
constexpr int STAGES = 4;
template <int KV, int T>
__host__ __device__ constexpr int code_bytes() { return 16 * T * (KV / 2); }
template <int KV, int T>
__host__ __device__ constexpr int stage_bytes() {
  return code_bytes<KV, T>() + 4 * 16 * T * (KV / 64 > 4 ? KV / 64 : 4);
}

// In a stage, row `row`'s 32-byte segment of block j sits at segment
// j ^ seg_swizzle(row): the 8 rows g a warp's 64-bit fragment read touches
// then cover every bank twice (two wavefronts, the least for 256 bytes).
template <int KV>
__device__ __forceinline__ int seg_swizzle(int row) { return KV == 128 ? ((row >> 1) & 1) : (row & 3); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The warp's codes of row block rb (16 T rows x KV codes from block kb0) into
// the stage at shared address `stage`, 16 bytes per copy.  Rows past N and
// blocks past K are zero-filled (source size 0), and expand to zero.
template <int KV, int T>
__device__ __forceinline__ void issue_codes(const Params& p, uint32_t stage, int rb, int kb0, int nbw, int lane) {
  constexpr int CPR = KV / 32;                 // 16-byte chunks per row
#pragma unroll
  for (int i = 0; i < 16 * T * CPR / 32; ++i) {
    const int c = lane + 32 * i;
    const int row = c / CPR, cc = c % CPR, j = cc >> 1;
    const int grow = rb * 16 * T + row;
    const bool live = grow < p.N && j < nbw;
    const uint8_t* src = live ? p.codes + (size_t)grow * (p.K / 2) + (size_t)kb0 * 32 + cc * 16 : p.codes;
    cp_async16(stage + row * (KV / 2) + ((((j ^ seg_swizzle<KV>(row)) << 1) | (cc & 1)) << 4), src, live ? 16u : 0u);
  }
  // Block constants.  Plain fp32 constants: one (row, block) pair per lane and
  // round, as [block][row] words.  E4M3 constants: the warp's NB = KV / 64
  // bytes of a row are consecutive, so per row the aligned word holding the
  // first of them (and the next word if they run past it), and the group scale
  // s_2 of the first block (and of the last block if it lies in the next group
  // of 256): [w0 | s0 | w1 | s1] x 16 T rows.  The second pair is only needed
  // when K / 64 is not a multiple of 4 (p.cw_two).  An aligned word around a
  // live byte never straddles a page, so the bytes beside it are safe to read.
  constexpr int ROWS = 16 * T;
  const uint32_t cw = stage + code_bytes<KV, T>();
  if (p.wc.absmax) {
    constexpr int PAIRS = ROWS * (KV / 64);
#pragma unroll
    for (int i = 0; i < (PAIRS + 31) / 32; ++i) {
      const int idx = lane + 32 * i;
      if (idx < PAIRS) {
        const int row = idx % ROWS, j = idx / ROWS;
        const int grow = rb * ROWS + row;
        const bool live = grow < p.N && j < nbw;
        const int64_t b = live ? (int64_t)grow * p.kb + kb0 + j : 0;
        cp_async4(cw + 4 * idx, p.wc.absmax + b, live ? 4u : 0u);
      }
    }
  } else {
    const int rounds = p.cw_two ? 4 : 2;           // word kinds: w0, s0 (, w1, s1)
#pragma unroll
    for (int i = 0; i < (4 * ROWS + 31) / 32; ++i) {
      const int idx = lane + 32 * i, kind = idx / ROWS, row = idx % ROWS;
      if (kind < rounds) {
        const int grow = rb * ROWS + row;
        const bool live = grow < p.N && nbw > 0;
        const int64_t b0 = live ? (int64_t)grow * p.kb + kb0 : 0, bl = b0 + (nbw > 0 ? nbw - 1 : 0);
        const void* src = p.wc.absmax_q;
        bool need = live;
        if (kind == 0) {
          src = p.wc.absmax_q + (b0 & ~(int64_t)3);
        } else if (kind == 1) {
          src = p.wc.scale2 + (b0 >> 8);
        } else if (kind == 2) {
          need = live && (b0 >> 2) != (bl >> 2);
          src = need ? p.wc.absmax_q + (bl & ~(int64_t)3) : p.wc.absmax_q;
        } else {
          need = live && (b0 >> 8) != (bl >> 8);
          src = need ? p.wc.scale2 + (bl >> 8) : p.wc.scale2;
        }
        cp_async4(cw + 4 * idx, src, need ? 4u : 0u);
      }
    }
  }
}

// c_hat = fl32(fl32(E4M3(q) s_2) + mu) (double quant) or the plain fp32 value.
__device__ __forceinline__ float decode_const(const WeightConsts& wc, uint32_t q, float s2, float mu) {
  if (wc.absmax) return __uint_as_float(q);
  return __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)q), s2), mu);
}

template <int NT, int KV, int T>
__device__ __forceinline__ void compute_frag(const Params& p, const uint8_t* stage, int rb, int kb0, float mu,
                                             const uint32_t (&xb)[KV / 16][NT][2], uint32_t qbase, int nbw,
                                             int g, int tq, float (&acc)[T][NT][4]) {
  // this thread's 16 codes of each (row, block): rows 16 t + g (+ 8)
  uint2 w[T][2][KV / 64];
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = 16 * t + g + 8 * h;
#pragma unroll
      for (int j = 0; j < KV / 64; ++j)
        w[t][h][j] = *reinterpret_cast<const uint2*>(stage + row * (KV / 2) + ((j ^ seg_swizzle<KV>(row)) << 5) + tq * 8);
    }
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][n][i] = 0.0f;
  // this thread's decoded constants (its quad index's block, rows g and g+8):
  // each is decoded once per quad and handed to the other three by shuffles
  constexpr int NB = KV / 64, ROWS = 16 * T;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(stage + code_bytes<KV, T>());
  float cmine[T][2];
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = 16 * t + g + 8 * h;
      const int jq = tq < NB ? tq : 0;
      if (p.wc.absmax) {
        cmine[t][h] = __uint_as_float(cw[jq * ROWS + row]);
      } else {
        // byte jq of the row's window starting at block b0 (words w0, w1), and
        // the scale of its group (s0, or s1 past a group boundary)
        const int64_t b0 = (int64_t)(rb * ROWS + row) * p.kb + kb0, b = b0 + jq;
        const uint32_t word = (b >> 2) == (b0 >> 2) ? cw[row] : cw[2 * ROWS + row];
        const uint32_t q = (word >> (8 * (int)(b & 3))) & 0xFFu;
        const float s2 = __uint_as_float((b >> 8) == (b0 >> 8) ? cw[ROWS + row] : cw[3 * ROWS + row]);
        cmine[t][h] = decode_const(p.wc, q, s2, mu);
      }
    }
#pragma unroll
  for (int j = 0; j < KV / 64; ++j) {
    if (j < nbw) {
#pragma unroll
      for (int t = 0; t < T; ++t) {
        // block j's constants come from quad lane j (all lanes take part)
        const uint64_t cg = pack_cc(__shfl_sync(0xffffffffu, cmine[t][0], 4 * g + j));
        const uint64_t c8 = pack_cc(__shfl_sync(0xffffffffu, cmine[t][1], 4 * g + j));
#pragma unroll
        for (int half = 0; half < 2; ++half) {        // word .x: k-steps 0, 1; word .y: k-steps 2, 3
          const uint32_t wg = half ? w[t][0][j].y : w[t][0][j].x;
          const uint32_t w8 = half ? w[t][1][j].y : w[t][1][j].x;
          const uint32_t eg = (wg << 2) & 0x3C3C3C3Cu, og = (wg >> 2) & 0x3C3C3C3Cu;
          const uint32_t e8 = (w8 << 2) & 0x3C3C3C3Cu, o8 = (w8 >> 2) & 0x3C3C3C3Cu;
#pragma unroll
          for (int s = 0; s < 2; ++s) {               // k-step u = 2 half + s: bytes 2s (slots 2t..) and 2s+1 (slots 2t+8..)
            const uint32_t a0 = expand_pair(eg, og, qbase, 0x7650u | (2 * s), cg);
            const uint32_t a1 = expand_pair(e8, o8, qbase, 0x7650u | (2 * s), c8);
            const uint32_t a2 = expand_pair(eg, og, qbase, 0x7650u | (2 * s + 1), cg);
            const uint32_t a3 = expand_pair(e8, o8, qbase, 0x7650u | (2 * s + 1), c8);
            const int ks = 4 * j + 2 * half + s;
#pragma unroll
            for (int n = 0; n < NT; ++n) mma_bf16(acc[t][n], a0, a1, a2, a3, xb[ks][n][0], xb[ks][n][1]);
          }
        }
      }
    }
  }
}

// Partials of a row block (16 T rows x M tokens): warp w's C fragments into
// red, then the CTA sums the 16 warps in order and writes part_y.
template <int NT, int T>
__device__ __forceinline__ void stash(float* red, const float (&acc)[T][NT][4], int warp, int g, int tq) {
  // red layout: [warp][16 T rows][8 NT tokens]
  constexpr int TOK = 8 * NT;
  float* base = red + warp * (16 * T * TOK);
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = 8 * n + 2 * tq;
      *reinterpret_cast<float2*>(base + (16 * t + g) * TOK + tok) = make_float2(acc[t][n][0], acc[t][n][1]);
      *reinterpret_cast<float2*>(base + (16 * t + g + 8) * TOK + tok) = make_float2(acc[t][n][2], acc[t][n][3]);
    }
}

// Dynamic shared memory of the main kernel: two reduction buffers, then the
// warps' code rings.
template <int NT, int T>
__host__ __device__ constexpr size_t red_floats() { return (size_t)WARPS * 16 * T * 8 * NT; }
template <int NT, int KV, int T>
__host__ __device__ constexpr size_t smallm_smem_bytes() {
  return sizeof(float) * 2 * red_floats<NT, T>() + (size_t)WARPS * STAGES * stage_bytes<KV, T>();
}

template <int NT, int KV, int T>
__global__ void __launch_bounds__(THREADS, 1) smallm_kernel(Params p) {
  constexpr int ROWS = 16 * T;
  constexpr int TOK = 8 * NT;
  __shared__ __align__(256) float qlev[64];
  extern __shared__ __align__(16) float red_dyn[];   // two reduction buffers of red_floats<NT, T>(), the rings
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  if (threadIdx.x < 16) qlev[threadIdx.x] = p.tab.q[threadIdx.x];
  pdl_wait();
  pdl_trigger();
  const int part = blockIdx.x;
  // this warp's K range: blocks [kb0, kb0 + nbw) of every row
  const int k0 = part * p.part_k + warp * KV;
  const int kb0 = k0 / 64;
  const int nbw = max(0, min(KV, p.K - k0)) / 64;
  const float mu = p.wc.absmax ? 0.0f : __ldg(p.wc.offset);
  // activation fragments of the K range, in the permuted order (0 past M or K)
  uint32_t xb[KV / 16][NT][2];
#pragma unroll
  for (int j = 0; j < KV / 64; ++j)
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tok = 8 * n + g;
        uint2 v = make_uint2(0u, 0u);
        if (tok < p.M && j < nbw)
          v = __ldg(reinterpret_cast<const uint2*>(p.X + (size_t)tok * p.K + k0 + 64 * j + 16 * tq + 4 * u));
        xb[4 * j + u][n][0] = v.x;
        xb[4 * j + u][n][1] = v.y;
      }
  __syncthreads();
  const uint32_t qbase = opaque_after_barrier(smem_u32(qlev));   // table reads stay below the barrier
  const int rb_first = blockIdx.y, rb_step = gridDim.y;
  constexpr int SB = stage_bytes<KV, T>();
  uint8_t* ring = reinterpret_cast<uint8_t*>(red_dyn + 2 * red_floats<NT, T>()) + (size_t)warp * STAGES * SB;
  const uint32_t ring_s = smem_u32(ring);
#pragma unroll
  for (int st = 0; st < STAGES - 1; ++st) {
    const int rb = rb_first + st * rb_step;
    if (rb < p.row_blocks) issue_codes<KV, T>(p, ring_s + st * SB, rb, kb0, nbw, lane);
    cp_async_commit();
  }
  int it = 0;
  for (int rb = rb_first; rb < p.row_blocks; rb += rb_step, ++it) {
    // refill the stage the previous row block used, STAGES - 1 row blocks ahead
    const int ahead = rb + (STAGES - 1) * rb_step;
    if (ahead < p.row_blocks) issue_codes<KV, T>(p, ring_s + ((it + STAGES - 1) % STAGES) * SB, ahead, kb0, nbw, lane);
    cp_async_commit();
    cp_async_wait<STAGES - 1>();                 // this row block's copies (this lane's) have landed
    __syncwarp();                                // ... and every lane's
    const uint8_t* stage = ring + (it % STAGES) * SB;
    float acc[T][NT][4];
    compute_frag<NT, KV, T>(p, stage, rb, kb0, mu, xb, qbase, nbw, g, tq, acc);
    __syncwarp();                                // the stage is free for the next refill
    float* rbuf = red_dyn + (it & 1) * red_floats<NT, T>();
    stash<NT, T>(rbuf, acc, warp, g, tq);
    __syncthreads();
    // thread -> (row, token) of the row block; the 16 warps summed in order
    const int row_l = threadIdx.x / TOK, tok = threadIdx.x % TOK;
    const int row = rb * ROWS + row_l;
    if (row_l < ROWS && tok < p.M && row < p.N) {
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) sum = __fadd_rn(sum, rbuf[w * (ROWS * TOK) + row_l * TOK + tok]);
      p.part_y[((size_t)part * p.N + row) * p.M + tok] = sum;
    }
  }
  cp_async_wait<0>();
  // this part's share of U = X A^T: the CTA with the last row block of the part
  if (blockIdx.y == (p.row_blocks - 1) % gridDim.y && p.r > 0) {
    __syncthreads();
    float* ubuf = red_dyn;                      // [warp][16 adapter rows][TOK tokens] fits in one buffer
    for (int rt = 0; rt < (p.r + 15) / 16; ++rt) {
      float acc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;
      const int ja = 16 * rt + g, jb = ja + 8;
#pragma unroll
      for (int j = 0; j < KV / 64; ++j) {
        if (j < nbw) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const size_t off = (size_t)k0 + 64 * j + 16 * tq + 4 * u;
            uint2 va = make_uint2(0u, 0u), vb = make_uint2(0u, 0u);
            if (ja < p.r) va = __ldg(reinterpret_cast<const uint2*>(p.A + (size_t)ja * p.K + off));
            if (jb < p.r) vb = __ldg(reinterpret_cast<const uint2*>(p.A + (size_t)jb * p.K + off));
#pragma unroll
            for (int n = 0; n < NT; ++n) mma_bf16(acc[n], va.x, vb.x, va.y, vb.y, xb[4 * j + u][n][0], xb[4 * j + u][n][1]);
          }
        }
      }
      float* base = ubuf + warp * (16 * TOK);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tok = 8 * n + 2 * tq;
        *reinterpret_cast<float2*>(base + g * TOK + tok) = make_float2(acc[n][0], acc[n][1]);
        *reinterpret_cast<float2*>(base + (g + 8) * TOK + tok) = make_float2(acc[n][2], acc[n][3]);
      }
      __syncthreads();
      const int jl = threadIdx.x / TOK, tok = threadIdx.x % TOK;
      const int jr = 16 * rt + jl;
      if (jl < 16 && jr < p.r && tok < p.M) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) sum = __fadd_rn(sum, ubuf[w * (16 * TOK) + jl * TOK + tok]);
        p.part_u[((size_t)part * p.M + tok) * p.r + jr] = sum;
      }
      __syncthreads();
    }
  }
}

// Y[m, n] = (sum over parts, in order) + fl32(s * sum_j U[m, j] B[n, j]),
// U = bf16(sum over parts of the U shares, in order); U_out gets U.
__global__ void __launch_bounds__(256) smallm_finish_kernel(const float* __restrict__ part_y,
                                                            const float* __restrict__ part_u, int parts, int M, int N,
                                                            int r, float s, const __nv_bfloat16* __restrict__ B,
                                                            void* Y, int y_bf16, __nv_bfloat16* U_out) {
  __shared__ float u_s[MAX_M * MAX_R];
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
    float sum = 0.0f;
    for (int q = 0; q < parts; ++q) sum = __fadd_rn(sum, part_u[(size_t)q * M * r + i]);
    const __nv_bfloat16 ub = __float2bfloat16_rn(sum);
    u_s[i] = __bfloat162float(ub);
    if (blockIdx.x == 0 && U_out) U_out[i] = ub;
  }
  __syncthreads();
  const int64_t total = (int64_t)N * M;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(i / M), m = (int)(i % M);
    float y = 0.0f;
    for (int q = 0; q < parts; ++q) y = __fadd_rn(y, part_y[(size_t)q * total + i]);
    if (r > 0) {
      float l = 0.0f;
      const __nv_bfloat16* brow = B + (size_t)n * r;
      for (int j = 0; j < r; ++j) l = __fadd_rn(l, __fmul_rn(u_s[m * r + j], __bfloat162float(brow[j])));
      y = __fadd_rn(y, __fmul_rn(s, l));
    }
    const int64_t o = (int64_t)m * N + n;
    if (y_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(y);
    else reinterpret_cast<float*>(Y)[o] = y;
  }
}

}  // namespace smallm

// Tile shape per token count: one token tile of 8 (KV = 256 reduction
// elements per warp) or two (KV = 128), one 16-row tile per row block: the
// activation fragments take 32 registers either way.
struct SmallmShape {
  int nt, kv, t;
};
static SmallmShape smallm_shape(int64_t M) { return M <= 8 ? SmallmShape{1, 256, 1} : SmallmShape{2, 128, 1}; }

static int smallm_parts(int64_t M, int64_t K) {
  const SmallmShape sh = smallm_shape(M);
  const int64_t part_k = (int64_t)smallm::WARPS * sh.kv;
  return (int)((K + part_k - 1) / part_k);
}

// Workspace of the small-token forward: part sums of Y [parts][N][M] and of U
// [parts][M][r] (fp32), then U [M, r] bf16 when the caller does not take it.
size_t smallm_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  const size_t parts = (size_t)smallm_parts(M, K);
  auto a256 = [](size_t b) { return (b + 255) & ~(size_t)255; };
  return a256(parts * N * M * 4) + a256(parts * M * std::max(r, 1) * 4) + a256((size_t)M * std::max(r, 1) * 2);
}

bool smallm_supported(int64_t N, int64_t K) { return N >= 1 && K >= 64 && K % 64 == 0; }

ql_status launch_smallm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* A, const void* B, int r,
                            float s, void* Y, ql_dtype y_dt, void* U_out, void* ws, cudaStream_t st) {
  using namespace smallm;
  if (M < 1 || M > MAX_M || r > MAX_R) return QL_ERR_UNSUPPORTED;
  const int N = (int)w->rows, K = (int)w->cols;
  const SmallmShape sh = smallm_shape(M);
  const int parts = smallm_parts(M, K);
  auto a256 = [](size_t b) { return (b + 255) & ~(size_t)255; };
  uint8_t* wp = reinterpret_cast<uint8_t*>(ws);
  float* part_y = reinterpret_cast<float*>(wp);
  float* part_u = reinterpret_cast<float*>(wp + a256((size_t)parts * N * M * 4));
  __nv_bfloat16* U = U_out ? reinterpret_cast<__nv_bfloat16*>(U_out)
                           : reinterpret_cast<__nv_bfloat16*>(wp + a256((size_t)parts * N * M * 4) +
                                                              a256((size_t)parts * M * std::max(r, 1) * 4));
  Params p;
  p.M = (int)M;
  p.N = N;
  p.K = K;
  p.r = r;
  p.kb = K / 64;
  p.cw_two = (p.kb % 4) != 0;
  p.parts = parts;
  p.part_k = WARPS * sh.kv;
  p.row_blocks = (N + 16 * sh.t - 1) / (16 * sh.t);
  p.wc = WeightConsts{w->absmax, w->absmax_q, w->scale2, w->offset};
  p.tab = nf4_table();
  p.codes = w->codes;
  p.X = reinterpret_cast<const __nv_bfloat16*>(X);
  p.A = reinterpret_cast<const __nv_bfloat16*>(A);
  p.part_y = part_y;
  p.part_u = part_u;
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  const int gy = std::max(1, std::min(p.row_blocks, std::max(1, sms / parts)));
  const dim3 grid((unsigned)parts, (unsigned)gy);
  const size_t smem = sh.nt == 1 ? smallm_smem_bytes<1, 256, 1>() : smallm_smem_bytes<2, 128, 1>();
  auto set_smem = [smem](const void* k) {
    return per_device(k, 0, [k, smem] {
             if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
               cudaGetLastError();
               return -1;
             }
             return 1;
           }) > 0;
  };
  TraceScope ts(TK_SMALLM, st);
  if (sh.nt == 1) {
    if (!set_smem(reinterpret_cast<const void*>(smallm_kernel<1, 256, 1>))) return QL_ERR_CUDA;
    QL_CUDA_TRY(launch(smallm_kernel<1, 256, 1>, grid, dim3(THREADS), smem, st, 1, 1, p));
  } else {
    if (!set_smem(reinterpret_cast<const void*>(smallm_kernel<2, 128, 1>))) return QL_ERR_CUDA;
    QL_CUDA_TRY(launch(smallm_kernel<2, 128, 1>, grid, dim3(THREADS), smem, st, 1, 1, p));
  }
  const int64_t total = (int64_t)N * M;
  const unsigned fgrid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, (int64_t)sms * 4));
  QL_CUDA_TRY(launch(smallm_finish_kernel, dim3(fgrid), dim3(256), 0, st, 1, 1, (const float*)part_y,
                     (const float*)part_u, parts, (int)M, N, r, s, reinterpret_cast<const __nv_bfloat16*>(B), Y,
                     y_dt == QL_BF16 ? 1 : 0, U));
  QL_LAUNCH_CHECK();
  return QL_OK;
}

}  // namespace ql
