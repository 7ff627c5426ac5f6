// Shared definitions for the sm_100a kernels of the QLoRA NF4 library.
#pragma once

#include <cstdint>
#include <functional>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "qlora_nf4.h"

namespace ql {

// Status bits the kernels may raise (read back by qlora_get_status).
enum : unsigned { ST_NONFINITE = 1u, ST_TIMEOUT = 2u };

// Status word: one per translation unit and device (internal linkage, so the
// library builds without relocatable device code).  Kernels OR bits into it;
// the host reads and clears every unit's word through the accessor that
// QL_DEFINE_STATUS_ACCESSOR defines in that unit.
static __device__ unsigned int g_status = 0;

__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_status, bits); }

#define QL_DEFINE_STATUS_ACCESSOR(fn)                                                   \
  unsigned fn(cudaStream_t st) {                                                        \
    unsigned v = 0;                                                                     \
    if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st) \
        != cudaSuccess) return ~0u;                                                     \
    const unsigned zero = 0;                                                            \
    if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) \
        != cudaSuccess) return ~0u;                                                     \
    if (cudaStreamSynchronize(st) != cudaSuccess) return ~0u;                           \
    return v;                                                                           \
  }

// The NF4 table as used by the kernels: levels q_j and decision thresholds
// m_j = fl32(fl32(q_j + q_{j+1}) / 2).  Passed by value as a kernel argument,
// so it lives in the constant bank and needs no per-device set-up.
struct NF4Table {
  float q[16];
  float m[15];
};

// Built once on the host from the page formula (codebook.cu).
const NF4Table& nf4_table();

// Constants of a weight, decoded per 64-block on the device.
struct WeightConsts {
  const float* absmax;      // non-NULL: plain fp32 constants
  const uint8_t* absmax_q;  // double-quant codes
  const float* scale2;
  const float* offset;
};

// E4M3 -> fp32, exact (every E4M3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_f32(uint8_t e) {
  uint32_t h2;
  uint16_t in = e;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// fp32 -> E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return (uint8_t)(out & 0xFF);
}

// Reconstructed block constant.  Double-quant form: two separate roundings,
// fl32(fl32(E4M3(e) * s2) + mu), written with _rn intrinsics so nothing fuses.
__device__ __forceinline__ float block_const(const WeightConsts& wc, int64_t b, float mu) {
  if (wc.absmax) return __ldg(wc.absmax + b);
  float e = e4m3_to_f32(__ldg(wc.absmax_q + b));
  float s2 = __ldg(wc.scale2 + (b >> 8));
  return __fadd_rn(__fmul_rn(e, s2), mu);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Per-block lookup table of the 16 dequantized bf16 values, split into byte
// planes so that prmt can do the lookup in registers:
//   lo[i] = low bytes  of entries 4i..4i+3
//   hi[i] = high bytes of entries 4i..4i+3
struct Lut16 {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ Lut16 make_lut(const NF4Table& T, float c) {
  Lut16 L;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t p0 = pack_bf16x2(__fmul_rn(T.q[4 * i + 0], c), __fmul_rn(T.q[4 * i + 1], c));
    uint32_t p1 = pack_bf16x2(__fmul_rn(T.q[4 * i + 2], c), __fmul_rn(T.q[4 * i + 3], c));
    L.lo[i] = __byte_perm(p0, p1, 0x6420);
    L.hi[i] = __byte_perm(p0, p1, 0x7531);
  }
  return L;
}

// Four codes (nibbles 0..3 of `c`) -> four bf16 values as two bf16x2 words.
__device__ __forceinline__ void lut_lookup4(const Lut16& L, uint32_t c, uint32_t& o0, uint32_t& o1) {
  uint32_t s = c & 0x7777u;                           // index within a half table
  uint32_t sel = ((c >> 1) & 0x4444u) | 0x3210u;      // bit 3 of each code picks the half
  uint32_t la = __byte_perm(L.lo[0], L.lo[1], s);
  uint32_t lb = __byte_perm(L.lo[2], L.lo[3], s);
  uint32_t ha = __byte_perm(L.hi[0], L.hi[1], s);
  uint32_t hb = __byte_perm(L.hi[2], L.hi[3], s);
  uint32_t lo = __byte_perm(la, lb, sel);
  uint32_t hi = __byte_perm(ha, hb, sel);
  o0 = __byte_perm(lo, hi, 0x5140);
  o1 = __byte_perm(lo, hi, 0x7362);
}

// Eight codes (one packed word, element order = nibble order) -> 4 words.
__device__ __forceinline__ uint4 lut_lookup8(const Lut16& L, uint32_t w) {
  uint4 r;
  lut_lookup4(L, w & 0xFFFFu, r.x, r.y);
  lut_lookup4(L, w >> 16, r.z, r.w);
  return r;
}

// ------------------------------------------------------- dependent launches
// Every kernel of the library is launched through launch() with programmatic
// stream serialization, so it can be scheduled (and run its prologue: barrier
// set-up, TMEM allocation, descriptor prefetch) while the previous kernel on
// the stream is still finishing.  Each kernel calls pdl_wait() before its
// first global-memory access (that returns once every earlier kernel on the
// stream has completed and its writes are visible) and pdl_trigger() once it
// holds its on-chip resources, which lets the next kernel be scheduled.
// QL_PDL=0 in the environment launches without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

bool pdl_enabled();

// Host-side values of a (kernel, device) pair, such as a function attribute
// that has been set or an occupancy answer, computed once per device: a process
// may drive several devices, and host threads may launch concurrently.
// `compute` runs outside the lock; its result is kept when it is >= 0 (a
// negative result is an error and is computed again on the next call).
int per_device_impl(const void* key, int tag, const std::function<int()>& compute);
template <typename F>
int per_device(const void* key, int tag, F&& compute) {
  return per_device_impl(key, tag, std::function<int()>(std::forward<F>(compute)));
}
int current_device();
int device_sm_count();

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, unsigned cluster_x,
                   unsigned cluster_y, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  unsigned n = 0;
  if (cluster_x * cluster_y > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster_x;
    at[n].val.clusterDim.y = cluster_y;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace ql

#define QL_CUDA_TRY(expr)                               \
  do {                                                  \
    cudaError_t _e = (expr);                            \
    if (_e != cudaSuccess) return QL_ERR_CUDA;          \
  } while (0)

#define QL_LAUNCH_CHECK()                               \
  do {                                                  \
    cudaError_t _e = cudaGetLastError();                \
    if (_e != cudaSuccess) return QL_ERR_CUDA;          \
  } while (0)
