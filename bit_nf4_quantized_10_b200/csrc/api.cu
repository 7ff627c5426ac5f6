// C ABI of the library: argument checks, workspace carving and the launch
// sequences of each call.  Argument errors return before anything is launched.
#include <algorithm>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace ql {
// codec.cu
ql_status launch_quantize(const void* x, ql_dtype dt, int64_t n, uint8_t* codes, float* absmax, cudaStream_t st);
size_t dq_workspace_bytes(int64_t nb);
ql_status launch_double_quant(const float* absmax, int64_t nb, uint8_t* absmax_q, float* scale2, float* offset,
                              void* ws, cudaStream_t st);
ql_status launch_dequant(const ql_nf4_weight* w, void* out, ql_dtype dt, cudaStream_t st);
unsigned status_word_codec(cudaStream_t st);
ql_status launch_dq_level1(const float* absmax, int64_t nb, double* nodes, cudaStream_t st);
ql_status launch_dq_finish(const double* nodes, int64_t n_nodes, int64_t nb_total, const float* absmax, int64_t nb,
                           uint8_t* absmax_q, float* scale2, float* offset, void* ws, cudaStream_t st);
ql_status launch_merge(const ql_nf4_weight* w, const void* A, const void* B, int r, float s, void* out,
                       uint8_t* codes_out, float* absmax_out, cudaStream_t st);
// gemm.cu
ql_status launch_gemm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* U, const void* B, int r,
                          float s, void* Y, ql_dtype y_dt, cudaStream_t st);
ql_status launch_gemm_bwd(const ql_nf4_weight* w, const void* dY, int64_t M, const void* V, const void* A, int r,
                          float s, void* dX, ql_dtype dx_dt, int accumulate, cudaStream_t st);
unsigned status_word_gemm(cudaStream_t st);
unsigned status_word_lora(cudaStream_t st);
unsigned status_word_smallm(cudaStream_t st);
unsigned status_word_diag(cudaStream_t st);
ql_status launch_wait_timeout(uint32_t polls, cudaStream_t st);
// lora_tc.cu
ql_status launch_proj(const void* Z, int64_t M, int64_t red, const void* Gt, int64_t ld_gt, int r, void* out,
                      void* out_t, int64_t ld_t, cudaStream_t st);
ql_status launch_grad_b(const void* dY, int64_t M, int N, const void* Ut, int64_t ld_ut, int r, float s, void* dB,
                        ql_dtype dt, cudaStream_t st);
ql_status launch_grad_a(const void* X, int64_t M, int K, const void* Vt, int64_t ld_vt, int r, float s, void* dA,
                        ql_dtype dt, cudaStream_t st);
ql_status launch_transpose(const void* src, int64_t rows, int cols, void* dst, int64_t ld_dst, cudaStream_t st);
ql_status launch_transpose2(const void* src0, int64_t rows0, int cols0, void* dst0, int64_t ld0, const void* src1,
                            int64_t rows1, int cols1, void* dst1, int64_t ld1, cudaStream_t st);
// smallm.cu
bool smallm_supported(int64_t N, int64_t K);
size_t smallm_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);
ql_status launch_smallm_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* A, const void* B, int r,
                            float s, void* Y, ql_dtype y_dt, void* U_out, void* ws, cudaStream_t st);
// fp4.cu
ql_status launch_nvfp4_quantize(const void* x, ql_dtype dt, int64_t n, int use_ts, uint8_t* codes, uint8_t* scales,
                                float* ts, void* ws, cudaStream_t st);
ql_status launch_mxfp4_quantize(const void* x, ql_dtype dt, int64_t n, uint8_t* codes, uint8_t* scales,
                                cudaStream_t st);
ql_status launch_fp4_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts, int64_t n, int fmt,
                             float* out, cudaStream_t st);
unsigned status_word_fp4(cudaStream_t st);
unsigned status_word_fp4g(cudaStream_t st);
size_t fp4_atoms_bytes(int64_t rows, int64_t K, int vs);
ql_status launch_fp4_atoms(const uint8_t* scales, int64_t rows, int64_t K, int vs, uint8_t* atoms, cudaStream_t st);
ql_status launch_fp4_gemm(int vs, const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_ts,
                          const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_ts, int64_t M, int64_t N,
                          int64_t K, float* Y, cudaStream_t st);
// adamw.cu
ql_status launch_adamw(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int64_t t, float lr,
                       float b1, float b2, float eps, float wd, cudaStream_t st);
ql_status paged_prefetch(const void* ptr, size_t bytes, int where, cudaStream_t st);
// mlp.cu
ql_status launch_silu_gate_fwd(const void* g, const void* u, void* h, int64_t n, cudaStream_t st);
ql_status launch_silu_gate_bwd(const void* dh, const void* g, const void* u, void* dg, void* du, int64_t n,
                               cudaStream_t st);
}  // namespace ql

namespace {

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dtype_ok(ql_dtype d) { return d == QL_F32 || d == QL_BF16; }
inline size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Weight descriptor checks shared by dequant and the GEMM calls.
ql_status check_weight(const ql_nf4_weight* w) {
  if (!w || w->rows <= 0 || w->cols <= 0) return QL_ERR_INVALID_ARG;
  if (!aligned16(w->codes)) return QL_ERR_INVALID_ARG;
  if (w->absmax) {
    if (!aligned16(w->absmax)) return QL_ERR_INVALID_ARG;
  } else {
    if (!aligned16(w->absmax_q) || !aligned16(w->scale2) || !aligned16(w->offset)) return QL_ERR_INVALID_ARG;
  }
  return QL_OK;
}

ql_status check_gemm_shape(const ql_nf4_weight* w, int64_t M, int r) {
  ql_status st = check_weight(w);
  if (st != QL_OK) return st;
  if (M < 0) return QL_ERR_INVALID_ARG;
  if (w->cols % 64 != 0 || w->rows % 8 != 0) return QL_ERR_INVALID_ARG;
  if (M >= (1ll << 31) || w->rows >= (1ll << 31) || w->cols >= (1ll << 31)) return QL_ERR_UNSUPPORTED;
  if (r < 0 || r % 8 != 0) return QL_ERR_INVALID_ARG;
  if (r > QL_MAX_RANK) return QL_ERR_UNSUPPORTED;
  return QL_OK;
}

// Tokens up to this count take the small-token (HBM-bound) forward kernels.
constexpr int64_t kSmallM = 16;

bool use_smallm(int64_t M, int64_t N, int64_t K) { return M >= 1 && M <= kSmallM && ql::smallm_supported(N, K); }

// Forward workspace: U [M, r] (when U_out is not given); for the small-token
// path also the fp32 part sums of Y and U (smallm.cu).
size_t ws_fwd(int64_t M, int64_t N, int64_t K, int r) {
  if (use_smallm(M, N, K)) return ql::smallm_workspace_bytes(M, N, K, r);
  return align256((size_t)M * r * 2);
}

// Backward workspace, carved in this order (each piece 256-byte aligned):
//   B^T [r, N], U^T [r, Mp], V [M, r], V^T [r, Mp].   Mp = M rounded up to 8.
struct BwdWs {
  size_t bt, ut, v, vt, total;
};

BwdWs ws_bwd_layout(int64_t M, int64_t N, int64_t K, int r) {
  BwdWs w{};
  if (r == 0) return w;
  const int64_t Mp = (M + 7) / 8 * 8;
  size_t off = 0;
  w.bt = off; off += align256((size_t)r * N * 2);
  w.ut = off; off += align256((size_t)r * Mp * 2);
  w.v = off;  off += align256((size_t)M * r * 2);
  w.vt = off; off += align256((size_t)r * Mp * 2);
  w.total = off;
  return w;
}

size_t ws_bwd(int64_t M, int64_t N, int64_t K, int r) { return ws_bwd_layout(M, N, K, r).total; }

}  // namespace

// An NVTX range around each public call ("qlora_nf4/<call>"), so a timeline
// profiler shows which library call launched which kernels.  Without a tool
// attached the push and pop do nothing.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

extern "C" {

ql_status nf4_quantize(const void* x, ql_dtype x_dt, int64_t n, uint8_t* codes, float* absmax, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nf4_quantize");
  if (n <= 0 || !dtype_ok(x_dt)) return QL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(absmax)) return QL_ERR_INVALID_ARG;
  return ql::launch_quantize(x, x_dt, n, codes, absmax, as_stream(stream));
}

ql_status nf4_double_quant(const float* absmax, int64_t nb, uint8_t* absmax_q, float* scale2, float* offset,
                           void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nf4_double_quant");
  if (nb <= 0) return QL_ERR_INVALID_ARG;
  if (!aligned16(absmax) || !aligned16(absmax_q) || !aligned16(scale2) || !aligned16(offset) || !aligned16(ws))
    return QL_ERR_INVALID_ARG;
  if (ws_bytes < ql::dq_workspace_bytes(nb)) return QL_ERR_WORKSPACE;
  return ql::launch_double_quant(absmax, nb, absmax_q, scale2, offset, ws, as_stream(stream));
}

ql_status nf4_double_quant_level1(const float* absmax, int64_t nb, double* nodes, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nf4_double_quant_level1");
  if (nb <= 0 || !aligned16(absmax) || !aligned16(nodes)) return QL_ERR_INVALID_ARG;
  return ql::launch_dq_level1(absmax, nb, nodes, as_stream(stream));
}

ql_status nf4_double_quant_finish(const double* nodes, int64_t n_nodes, int64_t nb_total, const float* absmax,
                                  int64_t nb, uint8_t* absmax_q, float* scale2, float* offset, void* ws,
                                  size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nf4_double_quant_finish");
  if (n_nodes <= 0 || nb <= 0 || nb_total < nb || n_nodes != (nb_total + 2047) / 2048) return QL_ERR_INVALID_ARG;
  if (!aligned16(nodes) || !aligned16(absmax) || !aligned16(absmax_q) || !aligned16(scale2) || !aligned16(offset) ||
      !aligned16(ws))
    return QL_ERR_INVALID_ARG;
  if (ws_bytes < ql::dq_workspace_bytes(nb_total)) return QL_ERR_WORKSPACE;
  return ql::launch_dq_finish(nodes, n_nodes, nb_total, absmax, nb, absmax_q, scale2, offset, ws, as_stream(stream));
}

ql_status nf4_dequant(const ql_nf4_weight* w, void* out, ql_dtype out_dt, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nf4_dequant");
  ql_status st = check_weight(w);
  if (st != QL_OK) return st;
  if (!dtype_ok(out_dt) || !aligned16(out)) return QL_ERR_INVALID_ARG;
  return ql::launch_dequant(w, out, out_dt, as_stream(stream));
}

ql_status qlora_merge(const ql_nf4_weight* w, const void* A, const void* B, int r, float s, void* W_out,
                      uint8_t* codes_out, float* absmax_out, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_merge");
  ql_status st = check_weight(w);
  if (st != QL_OK) return st;
  if (w->cols % 64 != 0) return QL_ERR_INVALID_ARG;
  if (r < 0) return QL_ERR_INVALID_ARG;
  if (r > QL_MAX_RANK) return QL_ERR_UNSUPPORTED;
  if (r > 0 && (!aligned16(A) || !aligned16(B))) return QL_ERR_INVALID_ARG;
  if ((codes_out == nullptr) != (absmax_out == nullptr)) return QL_ERR_INVALID_ARG;
  if (!W_out && !codes_out) return QL_ERR_INVALID_ARG;
  if ((W_out && !aligned16(W_out)) || (codes_out && (!aligned16(codes_out) || !aligned16(absmax_out))))
    return QL_ERR_INVALID_ARG;
  return ql::launch_merge(w, r > 0 ? A : nullptr, r > 0 ? B : nullptr, r, s, W_out, codes_out, absmax_out,
                          as_stream(stream));
}

ql_status qlora_linear_fwd(const ql_nf4_weight* w, const void* X, int64_t M, const void* A, const void* B, int r,
                           float s, void* Y, ql_dtype y_dt, void* U_out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_linear_fwd");
  ql_status st = check_gemm_shape(w, M, r);
  if (st != QL_OK) return st;
  if (!dtype_ok(y_dt) || !aligned16(X) || !aligned16(Y)) return QL_ERR_INVALID_ARG;
  if (r > 0 && (!aligned16(A) || !aligned16(B))) return QL_ERR_INVALID_ARG;
  if (U_out && !aligned16(U_out)) return QL_ERR_INVALID_ARG;
  if (M == 0) return QL_OK;
  cudaStream_t cs = as_stream(stream);
  const int64_t N = w->rows, K = w->cols;
  const bool small = use_smallm(M, N, K);
  if (r == 0 && !small) return ql::launch_gemm_fwd(w, X, M, nullptr, nullptr, 0, s, Y, y_dt, cs);
  if (ws_bytes < ws_fwd(M, N, K, r)) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_INVALID_ARG;
  // small token counts: U = bf16(X A^T) comes out of the same pass over K
  if (small) return ql::launch_smallm_fwd(w, X, M, A, B, r, s, Y, y_dt, U_out, ws, cs);
  void* U = U_out ? U_out : ws;
  st = ql::launch_proj(X, M, K, A, K, r, U, nullptr, 0, cs);      // U = bf16(X A^T)
  if (st != QL_OK) return st;
  return ql::launch_gemm_fwd(w, X, M, U, B, r, s, Y, y_dt, cs);
}

ql_status qlora_linear_bwd(const ql_nf4_weight* w, const void* X, const void* dY, int64_t M, const void* A,
                           const void* B, int r, float s, const void* U, void* dX, ql_dtype dx_dt, int accumulate_dx,
                           void* dA, void* dB, ql_dtype grad_dt, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_linear_bwd");
  ql_status st = check_gemm_shape(w, M, r);
  if (st != QL_OK) return st;
  if (!dtype_ok(dx_dt) || !dtype_ok(grad_dt) || !aligned16(dY) || !aligned16(dX)) return QL_ERR_INVALID_ARG;
  if (r > 0 && (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB)))
    return QL_ERR_INVALID_ARG;
  if (U && !aligned16(U)) return QL_ERR_INVALID_ARG;
  const int64_t N = w->rows, K = w->cols;
  if (r > 0 && ws_bytes < ws_bwd(M, N, K, r)) return QL_ERR_WORKSPACE;
  if (r > 0 && !aligned16(ws)) return QL_ERR_INVALID_ARG;
  cudaStream_t cs = as_stream(stream);
  if (M == 0) {
    // no tokens: the adapter gradients are zero, dX is empty
    if (r > 0) {
      const size_t e = grad_dt == QL_F32 ? 4 : 2;
      QL_CUDA_TRY(cudaMemsetAsync(dA, 0, (size_t)r * K * e, cs));
      QL_CUDA_TRY(cudaMemsetAsync(dB, 0, (size_t)N * r * e, cs));
    }
    return QL_OK;
  }
  if (r == 0) return ql::launch_gemm_bwd(w, dY, M, nullptr, nullptr, 0, s, dX, dx_dt, accumulate_dx, cs);
  const BwdWs L = ws_bwd_layout(M, N, K, r);
  uint8_t* wp = reinterpret_cast<uint8_t*>(ws);
  const int64_t Mp = (M + 7) / 8 * 8;
  void* Bt = wp + L.bt;
  void* Ut = wp + L.ut;
  void* V = wp + L.v;
  void* Vt = wp + L.vt;
  if (!U) {
    st = ql::launch_transpose(B, N, r, Bt, N, cs);                            // B^T [r, N]
    if (st != QL_OK) return st;
    st = ql::launch_proj(X, M, K, A, K, r, nullptr, Ut, Mp, cs);     // U^T = bf16(X A^T)^T
  } else {
    st = ql::launch_transpose2(B, N, r, Bt, N, U, M, r, Ut, Mp, cs);          // B^T [r, N] and U^T [r, Mp]
  }
  if (st != QL_OK) return st;
  st = ql::launch_proj(dY, M, N, Bt, N, r, V, Vt, Mp, cs);          // V = bf16(dY B), and V^T
  if (st != QL_OK) return st;
  st = ql::launch_gemm_bwd(w, dY, M, V, A, r, s, dX, dx_dt, accumulate_dx, cs);  // dX
  if (st != QL_OK) return st;
  st = ql::launch_grad_b(dY, M, (int)N, Ut, Mp, r, s, dB, grad_dt, cs);  // dB = s dY^T U
  if (st != QL_OK) return st;
  return ql::launch_grad_a(X, M, (int)K, Vt, Mp, r, s, dA, grad_dt, cs);   // dA = s V^T X
}

ql_status nvfp4_quantize(const void* x, ql_dtype x_dt, int64_t n, int use_tensor_scale, uint8_t* codes,
                         uint8_t* scales, float* tensor_scale, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nvfp4_quantize");
  if (n <= 0 || !dtype_ok(x_dt)) return QL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(tensor_scale) || !aligned16(ws))
    return QL_ERR_INVALID_ARG;
  if (ws_bytes < qlora_workspace_size(QL_OP_NVFP4, n, 0, 0, 0)) return QL_ERR_WORKSPACE;
  return ql::launch_nvfp4_quantize(x, x_dt, n, use_tensor_scale ? 1 : 0, codes, scales, tensor_scale, ws,
                                   as_stream(stream));
}

ql_status mxfp4_quantize(const void* x, ql_dtype x_dt, int64_t n, uint8_t* codes, uint8_t* scales, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/mxfp4_quantize");
  if (n <= 0 || !dtype_ok(x_dt)) return QL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return QL_ERR_INVALID_ARG;
  return ql::launch_mxfp4_quantize(x, x_dt, n, codes, scales, as_stream(stream));
}

ql_status nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t n,
                        float* out, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nvfp4_dequant");
  if (n <= 0 || !aligned16(codes) || !aligned16(scales) || !aligned16(tensor_scale) || !aligned16(out))
    return QL_ERR_INVALID_ARG;
  return ql::launch_fp4_dequant(codes, scales, tensor_scale, n, 0, out, as_stream(stream));
}

ql_status mxfp4_dequant(const uint8_t* codes, const uint8_t* scales, int64_t n, float* out, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/mxfp4_dequant");
  if (n <= 0 || !aligned16(codes) || !aligned16(scales) || !aligned16(out)) return QL_ERR_INVALID_ARG;
  return ql::launch_fp4_dequant(codes, scales, nullptr, n, 1, out, as_stream(stream));
}

size_t nvfp4_scale_atoms_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 64) return 0;
  return ql::fp4_atoms_bytes(rows, K, 16);
}

size_t mxfp4_scale_atoms_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 128) return 0;
  return ql::fp4_atoms_bytes(rows, K, 32);
}

static ql_status fp4_scale_atoms(const uint8_t* scales, int64_t rows, int64_t K, int vs, uint8_t* atoms, void* stream) {
  if (rows < 1 || K < 1 || !aligned16(scales) || !aligned16(atoms)) return QL_ERR_INVALID_ARG;
  if (K % 256 != 0 || rows >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31)) return QL_ERR_UNSUPPORTED;
  return ql::launch_fp4_atoms(scales, rows, K, vs, atoms, as_stream(stream));
}

ql_status nvfp4_scale_atoms(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* atoms, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nvfp4_scale_atoms");
  return fp4_scale_atoms(scales, rows, K, 16, atoms, stream);
}

ql_status mxfp4_scale_atoms(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* atoms, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/mxfp4_scale_atoms");
  return fp4_scale_atoms(scales, rows, K, 32, atoms, stream);
}

static ql_status fp4_gemm_checked(int vs, const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_ts,
                                  const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_ts, int64_t M,
                                  int64_t N, int64_t K, float* Y, void* stream) {
  if (M < 1 || N < 1 || K < 1) return QL_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_atoms) || !aligned16(b_codes) || !aligned16(b_atoms) || !aligned16(Y))
    return QL_ERR_INVALID_ARG;
  if (vs == 16 && (!a_ts || !b_ts)) return QL_ERR_INVALID_ARG;
  if (K % 256 != 0 || M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 23) || K >= ((int64_t)1 << 31))
    return QL_ERR_UNSUPPORTED;
  return ql::launch_fp4_gemm(vs, a_codes, a_atoms, a_ts, b_codes, b_atoms, b_ts, M, N, K, Y, as_stream(stream));
}

ql_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_tensor_scale,
                     const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_tensor_scale, int64_t M,
                     int64_t N, int64_t K, float* Y, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/nvfp4_gemm");
  return fp4_gemm_checked(16, a_codes, a_atoms, a_tensor_scale, b_codes, b_atoms, b_tensor_scale, M, N, K, Y, stream);
}

ql_status mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_atoms, const uint8_t* b_codes, const uint8_t* b_atoms,
                     int64_t M, int64_t N, int64_t K, float* Y, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/mxfp4_gemm");
  return fp4_gemm_checked(32, a_codes, a_atoms, nullptr, b_codes, b_atoms, nullptr, M, N, K, Y, stream);
}

ql_status qlora_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int64_t t, float lr,
                           float beta1, float beta2, float eps, float weight_decay, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_adamw_step");
  if (n <= 0 || t < 1) return QL_ERR_INVALID_ARG;
  if (!aligned16(p) || !aligned16(g) || !aligned16(m) || !aligned16(v) || (p_bf16 && !aligned16(p_bf16)))
    return QL_ERR_INVALID_ARG;
  if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps >= 0.0f)) return QL_ERR_INVALID_ARG;
  return ql::launch_adamw(p, g, m, v, p_bf16, n, t, lr, beta1, beta2, eps, weight_decay, as_stream(stream));
}

ql_status qlora_paged_prefetch(const void* ptr, size_t bytes, int where, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_paged_prefetch");
  if (!ptr || bytes == 0 || (where != QL_PAGE_DEVICE && where != QL_PAGE_HOST)) return QL_ERR_INVALID_ARG;
  return ql::paged_prefetch(ptr, bytes, where, as_stream(stream));
}

ql_status qlora_selftest_wait_timeout(int64_t polls, void* stream) {
  if (polls < 1 || polls > (1 << 20)) return QL_ERR_INVALID_ARG;
  return ql::launch_wait_timeout((uint32_t)polls, as_stream(stream));
}

ql_status qlora_silu_gate_fwd(const void* g, const void* u, void* h, int64_t n, void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_silu_gate_fwd");
  if (n <= 0 || !aligned16(g) || !aligned16(u) || !aligned16(h)) return QL_ERR_INVALID_ARG;
  return ql::launch_silu_gate_fwd(g, u, h, n, as_stream(stream));
}

ql_status qlora_silu_gate_bwd(const void* dh, const void* g, const void* u, void* dg, void* du, int64_t n,
                              void* stream) {
  NvtxRange nvtx_range("qlora_nf4/qlora_silu_gate_bwd");
  if (n <= 0 || !aligned16(dh) || !aligned16(g) || !aligned16(u) || !aligned16(dg) || !aligned16(du))
    return QL_ERR_INVALID_ARG;
  return ql::launch_silu_gate_bwd(dh, g, u, dg, du, n, as_stream(stream));
}

size_t qlora_workspace_size(int op, int64_t M, int64_t N, int64_t K, int r) {
  switch (op) {
    case QL_OP_DOUBLE_QUANT: return M > 0 ? ql::dq_workspace_bytes(M) : 0;
    case QL_OP_FWD: return ws_fwd(M, N, K, r);
    case QL_OP_BWD: return ws_bwd(M, N, K, r);
    case QL_OP_NVFP4: return M > 0 ? 256 : 0;
    default: return 0;
  }
}

int64_t nf4_storage_bytes(int64_t n, int dq) {
  if (n <= 0) return 0;
  const int64_t nb = (n + 63) / 64;
  const int64_t ng = (nb + 255) / 256;
  return (n + 1) / 2 + (dq ? nb + 4 * ng + 4 : 4 * nb);
}

void nf4_codebook(float out[16]) {
  if (out) std::memcpy(out, ql::nf4_table().q, sizeof(float) * 16);
}

ql_status qlora_get_status(void* stream) {
  cudaStream_t cs = as_stream(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return QL_ERR_CUDA;
  // one status word per translation unit that raises status bits
  unsigned v = 0;
  for (unsigned (*word)(cudaStream_t) : {ql::status_word_codec, ql::status_word_gemm, ql::status_word_lora,
                                         ql::status_word_smallm, ql::status_word_diag, ql::status_word_fp4,
                                         ql::status_word_fp4g}) {
    const unsigned w = word(cs);
    if (w == ~0u) return QL_ERR_CUDA;
    v |= w;
  }
  if (v & ql::ST_NONFINITE) return QL_ERR_NONFINITE;
  if (v & ql::ST_TIMEOUT) return QL_ERR_TIMEOUT;
  return QL_OK;
}

const char* qlora_status_string(ql_status s) {
  switch (s) {
    case QL_OK: return "ok";
    case QL_ERR_INVALID_ARG: return "invalid argument";
    case QL_ERR_UNSUPPORTED: return "unsupported";
    case QL_ERR_WORKSPACE: return "workspace too small";
    case QL_ERR_CUDA: return "CUDA error";
    case QL_ERR_NONFINITE: return "non-finite input";
    case QL_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
