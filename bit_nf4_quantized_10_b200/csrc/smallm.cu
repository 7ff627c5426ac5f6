// Small-token forward: Y = X * W_hat^T + s * U * B^T for M <= 16 tokens.
//
// With a handful of tokens each dequantized weight element meets at most 16
// activations, so the layer is bound by reading the packed 4-bit weight from
// HBM ("QLoRA — Fine-Tuning a 65B Model on One GPU", "Pitfalls":
// memory-bandwidth-bound generation has less to read with 4-bit weights) and
// by the integer work of expanding it, which must keep pace with HBM.
//   * Operands are swapped: the expanded weight tile is the MMA's A operand
//     (M = 128 weight rows) and lives in TMEM, written with tcgen05.st from the
//     producer registers; the tokens are the N = 16 operand (zero-padded).
//   * Expansion: the 16 fp32 levels sit in a shared-memory table (one
//     conflict-free LDS per element), times the block constant in fp32, pairs
//     packed to bf16: bf16(fl32(q * c)), as everywhere else.
//   * Persistent clusters: the CTAs of a cluster (up to 8) split K, so each
//     CTA owns one fixed K slice and keeps the tokens' slice of X in shared
//     memory for the whole kernel; the clusters walk over 128-row weight
//     tiles.  Each TMA stage brings 128 contiguous bytes (256 codes) of every
//     row of the tile.
//   * The split-K partials meet in shared memory: each CTA drains its 128 x 16
//     fp32 partial (TMEM, double-buffered) into shared memory, and CTA q of the
//     cluster adds the slices of its share of the tile's outputs in slice
//     order through distributed shared memory, adds s * U * B^T in fp32 and
//     writes Y.  Hand-offs between the CTAs go through mbarriers with remote
//     arrivals (release/acquire at cluster scope), so the expansion of the
//     next tile overlaps the reduction of the last.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

QL_DEFINE_STATUS_ACCESSOR(status_word_smallm)

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t cols,
                 uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

namespace smallm {

constexpr int TM = 128;           // weight rows per tile (MMA M)
constexpr int TN = 16;            // token slots (MMA N)
constexpr int BK = 64;            // reduction elements per MMA sub-step (one 64-block per row)
constexpr int SUB = 4;            // sub-steps per code stage: 256 codes = 128 contiguous bytes per row
constexpr int C_STAGE_BYTES = TM * BK * SUB / 2;   // 16 KB packed codes
constexpr int MAX_C_STAGES = 8;
constexpr int X_SUB_BYTES = TN * BK * 2;           // 2 KB activation sub-tile
constexpr int MAX_PER = 80;       // sub-steps per K slice (bounded by shared memory)
constexpr int MAX_CS = 8;         // CTAs per cluster (portable cluster size)
constexpr int A_STAGES = 3;       // TMEM ring of expanded A stages (128 rows x 256 codes each)
constexpr int GROUP_WARPS = 8;    // producer warps per group; two groups take alternate sub-steps
constexpr int PRODUCER_WARPS = 2 * GROUP_WARPS;
constexpr int DRAIN_WARP0 = 2 + PRODUCER_WARPS;
constexpr int DRAIN_WARPS = 4;
constexpr int THREADS = (DRAIN_WARP0 + DRAIN_WARPS) * 32;
constexpr int TMEM_COLS = 512;    // D[b] at columns 16 b; A stage s at 128 + 128 s (32 per sub-step)
constexpr int A_COL0 = 128;
constexpr int A_STAGE_COLS = 128;
constexpr int RED_LD = 18;        // floats per row of a reduction buffer (conflict-free float2 reads)
constexpr int RED_BYTES = TM * RED_LD * 4;
constexpr int MAX_R = 64;

struct Params {
  int M, N, K, r;
  int kb_total;       // K / 64
  int per;            // sub-steps per K slice (the last slice may be shorter)
  int tiles;          // ceil(N / 128)
  int c_stages;       // code ring depth (a power of two)
  int c_log;          // log2(c_stages)
  float s;
  WeightConsts wc;
  NF4Table tab;
  const __nv_bfloat16* U;   // [M, r]
  const __nv_bfloat16* B;   // [N, r]
  void* Y;
  int y_bf16;
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

// Arrive on the barrier at this offset in CTA `rank`, release at cluster
// scope: publishes this thread's (and, through a preceding warp barrier, its
// warp's) shared-memory accesses to the other CTA.
__device__ __forceinline__ void arrive_remote_release(uint64_t* bar, uint32_t rank) {
  asm volatile(
      "{\n .reg .b32 ra;\n"
      " mapa.shared::cluster.u32 ra, %0, %1;\n"
      " mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}

__device__ __forceinline__ float2 ld_cluster_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(THREADS, 1)
    smallm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float us[TN * MAX_R];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int cs = (int)gridDim.x;                 // CTAs per cluster = K slices
  const int q = (int)blockIdx.x;                 // this CTA's slice (its cluster rank)
  const int kb0 = q * p.per;
  const int per_q = min(p.per, p.kb_total - kb0);
  const int nst = (per_q + SUB - 1) / SUB;       // code stages per tile
  const int nt = (p.tiles - (int)blockIdx.y + (int)gridDim.y - 1) / (int)gridDim.y;   // tiles of this cluster
  const int C = p.c_stages;
  uint8_t* xs = base;                                            // per_q x 2 KB
  uint8_t* cring = xs + p.per * X_SUB_BYTES;                     // C x 16 KB
  float* red = reinterpret_cast<float*>(cring + C * C_STAGE_BYTES);   // 2 x 128 x RED_LD
  // the 16 fp32 levels, 256-byte aligned: an LDS address is the table base
  // with the level's byte offset (4 * code) in its low byte
  float* qtab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + 2 * RED_BYTES);
  uint64_t* full_x = reinterpret_cast<uint64_t*>(qtab + 64);
  uint64_t* full_c = full_x + 1;
  uint64_t* empty_c = full_c + MAX_C_STAGES;
  uint64_t* a_full = empty_c + MAX_C_STAGES;
  uint64_t* a_empty = a_full + A_STAGES;
  uint64_t* acc_full = a_empty + A_STAGES;
  uint64_t* tmem_free = acc_full + 2;
  uint64_t* ready = tmem_free + 2;
  uint64_t* freed = ready + 2;
  uint32_t* tmem_addr = reinterpret_cast<uint32_t*>(freed + 2);
  volatile int* abort_flag = reinterpret_cast<int*>(tmem_addr + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto tile_of = [&](int ti) { return (int)blockIdx.y + ti * (int)gridDim.y; };

  if (threadIdx.x < 16) qtab[threadIdx.x] = p.tab.q[threadIdx.x];
  if (threadIdx.x == 0) {
    mbar_init(full_x, 1);
    for (int i = 0; i < MAX_C_STAGES; ++i) {
      mbar_init(&full_c[i], 1);
      mbar_init(&empty_c[i], 1);
    }
    for (int i = 0; i < A_STAGES; ++i) {
      mbar_init(&a_full[i], GROUP_WARPS);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&tmem_free[i], DRAIN_WARPS);
      mbar_init(&ready[i], cs * DRAIN_WARPS);
      mbar_init(&freed[i], cs * DRAIN_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_addr, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();   // every CTA's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_addr;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      prefetch_tmap(&tmap_codes);
      mbar_arrive_expect_tx(full_x, per_q * X_SUB_BYTES);
      for (int j = 0; j < per_q; ++j) tma_load_2d(xs + j * X_SUB_BYTES, &tmap_x, full_x, (kb0 + j) * BK, 0);
      int issued = 0;
      bool ok = true;
      for (int ti = 0; ti < nt && ok; ++ti) {
        for (int st = 0; st < nst; ++st) {
          const int g = ti * nst + st, cslot = g % C;
          if (g >= C && !mbar_wait(&empty_c[cslot], ((g / C) - 1) & 1, abort_flag, p.wait_limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_c[cslot], C_STAGE_BYTES);
          tma_load_2d(cring + cslot * C_STAGE_BYTES, &tmap_codes, &full_c[cslot], (kb0 + st * SUB) * (BK / 2),
                      tile_of(ti) * TM);
          issued = g + 1;
        }
      }
      // before leaving, make sure no copy is still landing in shared memory
      mbar_wait(full_x, 0, abort_flag, p.wait_limit);
      for (int g = (issued > C ? issued - C : 0); g < issued; ++g)
        mbar_wait(&full_c[g % C], (g / C) & 1, abort_flag, p.wait_limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(TM, TN, false, false);
      bool ok = mbar_wait(full_x, 0, abort_flag, p.wait_limit);
      for (int ti = 0; ti < nt && ok; ++ti) {
        const int b = ti & 1;
        if (ti >= 2) ok = mbar_wait(&tmem_free[b], ((ti >> 1) - 1) & 1, abort_flag, p.wait_limit);
        // one A stage = one code stage: up to four 64-deep sub-steps, 16 MMAs
        for (int st = 0; st < nst && ok; ++st) {
          const int G = ti * nst + st, aslot = G % A_STAGES;
          ok = mbar_wait(&a_full[aslot], (G / A_STAGES) & 1, abort_flag, p.wait_limit);
          if (!ok) break;
          tc_fence_after();
          const int nsub = min(SUB, per_q - st * SUB);
          for (int u = 0; u < nsub; ++u) {
            const int j = st * SUB + u;
            const uint32_t x_addr = smem_u32(xs + j * X_SUB_BYTES);
            const uint32_t a_col = A_COL0 + aslot * A_STAGE_COLS + u * 32;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_ts(tmem + 16 * b, tmem + a_col + kk * 8, sdesc_sw128(x_addr + kk * 32, 16, 1024), idesc,
                     (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&a_empty[aslot]);
          mma_commit(&empty_c[G % C]);
        }
        if (ok) mma_commit(&acc_full[b]);
      }
    }
  } else if (warp < DRAIN_WARP0) {
    // ------------------------------------------------------ dequant producers
    // group grp expands the A stages G = grp, grp+2, ... of this CTA's
    // sequence (tile by tile; one A stage = the up to four 64-deep sub-steps
    // of one code stage); warp: TMEM lanes 32*(warp&3) (weight rows) and half
    // of the 64 codes of each sub-step
    const int grp = (warp - 2) / GROUP_WARPS;
    const int half = ((warp - 2) >> 2) & 1;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const float mu = p.wc.absmax ? 0.0f : *p.wc.offset;
    const uint32_t qbase = smem_u32(qtab);   // low byte 0
    // block constants of the sub-steps of stage st of tile ti (raw: absmax, or
    // scale2 and the E4M3 code)
    auto load_c = [&](int ti, int st, float2 (&r)[SUB]) {
#pragma unroll
      for (int u = 0; u < SUB; ++u) r[u] = make_float2(0.0f, 0.0f);
      if (ti >= nt) return;
      const int n = tile_of(ti) * TM + row;
      if (n >= p.N) return;
#pragma unroll
      for (int u = 0; u < SUB; ++u) {
        const int j = st * SUB + u;
        if (j >= per_q) break;
        const int64_t b = (int64_t)n * p.kb_total + kb0 + j;
        if (p.wc.absmax) r[u].x = __ldg(p.wc.absmax + b);
        else { r[u].x = __ldg(p.wc.scale2 + (b >> 8)); r[u].y = __uint_as_float((uint32_t)__ldg(p.wc.absmax_q + b)); }
      }
    };
    // (tile, stage) two stages further on: this group's next stage
    auto advance2 = [&](int& ti, int& st) {
      st += 2;
      while (st >= nst) { st -= nst; ++ti; }
    };
    int ti = 0, st = grp;
    while (st >= nst) { st -= nst; ++ti; }
    int nti = ti, nst2 = st;
    advance2(nti, nst2);
    float2 cur[SUB], nxt[SUB];
    load_c(ti, st, cur);
    bool ok = true;
    for (int G = grp; ti < nt && ok; G += 2) {
      const int cslot = G & (C - 1);
      const int aslot = G % A_STAGES;
      const bool valid = tile_of(ti) * TM + row < p.N;
      const int nsub = min(SUB, per_q - st * SUB);
      load_c(nti, nst2, nxt);
      ok = __all_sync(0xffffffffu, mbar_wait(&full_c[cslot], (G >> p.c_log) & 1, abort_flag, p.wait_limit) &&
                                       (G < A_STAGES ||
                                        mbar_wait(&a_empty[aslot], ((G / A_STAGES) - 1) & 1, abort_flag, p.wait_limit)));
      if (!ok) break;
      tc_fence_after();
      const uint8_t* cst = cring + cslot * C_STAGE_BYTES;
#pragma unroll
      for (int u = 0; u < SUB; ++u) {
        if (u >= nsub) break;
        uint32_t out[16];
        if (valid) {
          const float c = p.wc.absmax ? cur[u].x
                                      : __fadd_rn(__fmul_rn(e4m3_to_f32((uint8_t)__float_as_uint(cur[u].y)), cur[u].x), mu);
          // 128-byte code rows with the 128B swizzle: 16-byte chunk ^= row mod 8
          const uint32_t coff = row * 128 + (((2 * u + half) ^ (row & 7)) << 4);
          const uint4 cw = *reinterpret_cast<const uint4*>(cst + coff);
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            // element i of the word is nibble i; its level sits at qbase + 4 * nibble
            const uint32_t e4 = (w[q4] << 2) & 0x3C3C3C3Cu;   // 4 * low nibble of each byte
            const uint32_t o4 = (w[q4] >> 2) & 0x3C3C3C3Cu;   // 4 * high nibble of each byte
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
              // byte bb of e4 / o4 under the table base's upper three bytes
              const float fe = lds_f32(__byte_perm(e4, qbase, 0x7650u | bb));
              const float fo = lds_f32(__byte_perm(o4, qbase, 0x7650u | bb));
              float pe, po;
              mul2_rn(fe, fo, c, pe, po);
              out[4 * q4 + bb] = pack_bf16x2(pe, po);
            }
          }
        } else {
#pragma unroll
          for (int t = 0; t < 16; ++t) out[t] = 0u;
        }
        tmem_st16(tmem + ((uint32_t)(quad * 32) << 16) +
                      (uint32_t)(A_COL0 + aslot * A_STAGE_COLS + u * 32 + half * 16),
                  out);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[aslot]);
#pragma unroll
      for (int u = 0; u < SUB; ++u) cur[u] = nxt[u];
      ti = nti;
      st = nst2;
      advance2(nti, nst2);
    }
  } else {
    // ---------------------------------------- drain, cluster reduction, output
    const int t = threadIdx.x - DRAIN_WARP0 * 32;   // 0..127
    const int quad = warp & 3;
    const int drow = quad * 32 + lane;              // the TMEM lane this thread drains
    for (int i = t; i < p.M * p.r; i += DRAIN_WARPS * 32) us[i] = __bfloat162float(p.U[i]);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // this CTA's share of the tile's (row, token pair) outputs, token pair fastest
    const int items = TM * (TN / 2);
    const int i0 = items * q / cs, i1 = items * (q + 1) / cs;
    // adapter row of an item, 16-byte loads issued together
    uint4 bv[MAX_R / 8];
    auto load_brow = [&](int n) {
#pragma unroll
      for (int c8 = 0; c8 < MAX_R / 8; ++c8)
        if (c8 * 8 < p.r && n < p.N) bv[c8] = *reinterpret_cast<const uint4*>(p.B + (size_t)n * p.r + c8 * 8);
    };
    bool ok = true;
    for (int ti = 0; ti < nt && ok; ++ti) {
      const int b = ti & 1;
      const int n0 = tile_of(ti) * TM;
      float* rb = red + b * (TM * RED_LD);
      // the first item's adapter row is fetched while the tile is still being computed
      if (p.r > 0 && i0 + t < i1) load_brow(n0 + ((i0 + t) >> 3));
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], (ti >> 1) & 1, abort_flag, p.wait_limit));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(16 * b), v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_free[b]);
      // the other CTAs are done reading this buffer's previous tile
      if (ti >= 2) ok = __all_sync(0xffffffffu, mbar_wait_cluster(&freed[b], ((ti >> 1) - 1) & 1, abort_flag, p.wait_limit));
      if (!ok) break;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        *reinterpret_cast<float2*>(rb + drow * RED_LD + 2 * k) =
            make_float2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
      __syncwarp();
      if (lane == 0)
        for (int pr = 0; pr < cs; ++pr) arrive_remote_release(&ready[b], (uint32_t)pr);
      ok = __all_sync(0xffffffffu, mbar_wait_cluster(&ready[b], (ti >> 1) & 1, abort_flag, p.wait_limit));
      if (!ok) break;
      const uint32_t rb_addr = smem_u32(rb);
      for (int it = i0 + t; it < i1; it += DRAIN_WARPS * 32) {
        const int r_in = it >> 3, tp = it & 7;
        const int n = n0 + r_in, m0 = 2 * tp;
        if (p.r > 0 && it != i0 + t) load_brow(n);
        if (n >= p.N || m0 >= p.M) continue;
        const uint32_t off = rb_addr + (uint32_t)((r_in * RED_LD + m0) * 4);
        // every slice's partial in flight at once, added in slice order
        float2 x[MAX_CS];
#pragma unroll
        for (int pr = 0; pr < MAX_CS; ++pr)
          if (pr < cs) x[pr] = ld_cluster_f2(cluster_map(off, (uint32_t)pr));
        float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int pr = 0; pr < MAX_CS; ++pr)
          if (pr < cs) {
            acc.x = __fadd_rn(acc.x, x[pr].x);
            acc.y = __fadd_rn(acc.y, x[pr].y);
          }
        float o[2] = {acc.x, acc.y};
        if (p.r > 0) {
#pragma unroll
          for (int mm = 0; mm < 2; ++mm) {
            if (m0 + mm >= p.M) break;
            const float* um = us + (m0 + mm) * p.r;
            float l = 0.0f;
#pragma unroll
            for (int c8 = 0; c8 < MAX_R / 8; ++c8) {
              if (c8 * 8 >= p.r) break;
              const uint32_t bw[4] = {bv[c8].x, bv[c8].y, bv[c8].z, bv[c8].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                l = fmaf(um[c8 * 8 + 2 * e], bf16_lo(bw[e]), l);
                l = fmaf(um[c8 * 8 + 2 * e + 1], bf16_hi(bw[e]), l);
              }
            }
            o[mm] = __fadd_rn(o[mm], __fmul_rn(p.s, l));
          }
        }
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          if (m0 + mm >= p.M) break;
          const size_t yo = (size_t)(m0 + mm) * p.N + n;
          if (p.y_bf16) reinterpret_cast<__nv_bfloat16*>(p.Y)[yo] = __float2bfloat16_rn(o[mm]);
          else reinterpret_cast<float*>(p.Y)[yo] = o[mm];
        }
      }
      __syncwarp();
      if (lane == 0)
        for (int pr = 0; pr < cs; ++pr) arrive_remote_release(&freed[b], (uint32_t)pr);
    }
  }
  tc_fence_before();
  cluster_sync();   // no CTA leaves while another may still read its shared memory or arrive on its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace smallm

static int sm_count_sm() {
  const int c = device_sm_count();
  return c > 0 ? c : 148;
}

struct SmallmPlan {
  int cs, per, c_stages, c_log, clusters;
  size_t smem;
};

static size_t smallm_static_smem() { return sizeof(float) * (smallm::TN * smallm::MAX_R); }

// Shared memory for a K slice of `per` sub-steps; false if it cannot fit.
static bool smallm_layout(int per, SmallmPlan& pl) {
  using namespace smallm;
  if (per > MAX_PER) return false;
  // alignment slack, the X slice, two reduction buffers, the level table,
  // 33 mbarriers + TMEM address + abort flag
  const size_t fixed = 1024 + (size_t)per * X_SUB_BYTES + 2 * RED_BYTES + 256 + 512;
  const size_t limit = 227 * 1024 - smallm_static_smem();
  if (fixed + 2 * C_STAGE_BYTES > limit) return false;
  int c = 2, lg = 1;
  while (c * 2 <= MAX_C_STAGES && fixed + (size_t)(c * 2) * C_STAGE_BYTES <= limit) {
    c *= 2;
    ++lg;
  }
  pl.per = per;
  pl.c_stages = c;
  pl.c_log = lg;
  pl.smem = fixed + (size_t)c * C_STAGE_BYTES;
  return true;
}

static bool smallm_attr() {
  return per_device(reinterpret_cast<const void*>(smallm::smallm_kernel), 0, [] {
           if (cudaFuncSetAttribute(smallm::smallm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)(227 * 1024 - smallm_static_smem())) != cudaSuccess ||
               cudaFuncSetAttribute(smallm::smallm_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
                   cudaSuccess) {
             cudaGetLastError();
             return -1;
           }
           return 1;
         }) > 0;
}

// Cluster size (CTAs sharing K) and cluster count: the tiles are handed out in
// rounds of `clusters`, each round costing about `per` sub-steps, scaled up
// when the code ring is shallower than 8 stages; pick the cheapest among the
// cluster sizes that fit (the cluster count comes from the occupancy
// calculator: a cluster's CTAs must share a GPC, which caps it below SMs / cs).
static bool smallm_plan(int64_t N, int64_t K, SmallmPlan& best, bool query) {
  using namespace smallm;
  const int kb = (int)(K / BK);
  if (kb < 1) return false;
  const int tiles = (int)((N + TM - 1) / TM);
  bool found = false;
  long best_cost = 0;
  for (int cs0 = std::min(MAX_CS, kb); cs0 >= 1; --cs0) {
    SmallmPlan pl;
    const int per = (kb + cs0 - 1) / cs0;
    if (!smallm_layout(per, pl)) continue;
    pl.cs = (kb + per - 1) / per;
    int maxc = sm_count_sm() / pl.cs;
    if (query) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)pl.cs, (unsigned)std::max(1, maxc));
      cfg.blockDim = dim3(THREADS);
      cfg.dynamicSmemBytes = pl.smem;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = (unsigned)pl.cs;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, smallm_kernel, &cfg) == cudaSuccess && n > 0) maxc = std::min(maxc, n);
      else cudaGetLastError();
    }
    pl.clusters = std::max(1, std::min(tiles, maxc));
    const long rounds = (tiles + pl.clusters - 1) / pl.clusters;
    // a CTA streams its codes at a rate that grows with the bytes it has in
    // flight, up to about 8 stages (128 KB): shallower rings cost in proportion
    const long cost = rounds * per * (MAX_C_STAGES / pl.c_stages);
    if (!found || cost < best_cost) {
      best = pl;
      best_cost = cost;
      found = true;
    }
  }
  return found;
}

// Whether the small-token kernel handles this shape (its K slice of X must fit
// in shared memory: K <= 40960 with eight slices).
bool smallm_supported(int64_t N, int64_t K) {
  SmallmPlan pl;
  return smallm_plan(N, K, pl, false);
}

// Y = X W_hat^T + s U B^T for M <= 16; U [M, r] given (bf16).
ql_status launch_smallm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* U, const void* B, int r,
                            float s, void* Y, ql_dtype y_dt, cudaStream_t st) {
  using namespace smallm;
  if (M < 1 || M > TN || r > MAX_R) return QL_ERR_UNSUPPORTED;
  const int N = (int)w->rows, K = (int)w->cols;
  if (!smallm_attr()) return QL_ERR_CUDA;
  // the plan for a weight shape is fixed: computed once per shape and device
  // (the layers of a model alternate a few shapes)
  struct Entry {
    int64_t N, K;
    int dev;
    SmallmPlan pl;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  const int dev = current_device();
  SmallmPlan pl;
  bool have = false;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const Entry& e : cache)
      if (e.N == N && e.K == K && e.dev == dev) {
        pl = e.pl;
        have = true;
        break;
      }
  }
  if (!have) {
    if (!smallm_plan(N, K, pl, true)) return QL_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(mu);
    if (cache.size() < 256) cache.push_back(Entry{N, K, dev, pl});
  }
  CUtensorMap map_x, map_codes;
  if (!make_map_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, TN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  if (!make_map_2d(&map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->codes, (uint64_t)K / 2, (uint64_t)N,
                   (uint64_t)K / 2, SUB * BK / 2, TM, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  Params p;
  p.M = (int)M;
  p.N = N;
  p.K = K;
  p.r = r;
  p.kb_total = K / BK;
  p.per = pl.per;
  p.tiles = (N + TM - 1) / TM;
  p.c_stages = pl.c_stages;
  p.c_log = pl.c_log;
  p.s = s;
  p.wc = WeightConsts{w->absmax, w->absmax_q, w->scale2, w->offset};
  p.tab = nf4_table();
  p.U = (const __nv_bfloat16*)U;
  p.B = (const __nv_bfloat16*)B;
  p.Y = Y;
  p.y_bf16 = y_dt == QL_BF16;
  p.wait_limit = 1u << 22;
  TraceScope ts(TK_SMALLM, st);
  QL_CUDA_TRY(launch(smallm_kernel, dim3((unsigned)pl.cs, (unsigned)pl.clusters), dim3(THREADS), pl.smem, st,
                     (unsigned)pl.cs, 1, map_x, map_codes, p));
  return QL_OK;
}

}  // namespace ql
