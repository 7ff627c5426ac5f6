/*
 * qlora_nf4.h — C ABI of the B200 (sm_100a) QLoRA NF4 library.
 *
 * The library implements the data-parallel hot path of QLoRA:
 *   - blockwise NF4 quantization of a frozen weight (blocks of 64, a 16-level
 *     normal-quantile table with an exact zero, two codes per byte);
 *   - double quantization of the fp32 block constants to 8-bit floats in
 *     groups of 256;
 *   - the frozen-4-bit + LoRA linear  Y = X * dequant(W)^T + s * (X A^T) B^T,
 *     s = alpha / r, forward and backward (dX, dA, dB; W is never written);
 *   - the adapter merge W' = dequant(W) + s B A after training, as a bf16
 *     weight and/or quantized again.
 *
 * Sources (the web pages this library restates):
 *   [P2] "QLoRA: Quantize Base Weights to 4-Bit": §2.1 (NF4 quantile formula),
 *        §2.2 (B_1 = 64 fp32 constants, double quantization to 8-bit floats with
 *        B_2 = 256), §3 (dequantize to BF16 on chip, BF16 matmul, LoRA branch
 *        (B @ (A @ x)) * (alpha / r), gradients only into the adapters).
 *   [P3] "QLoRA — Fine-Tuning a 65B Model on One GPU": "Prerequisite: LoRA's
 *        low-rank update" (B is d x r, A is r x k), "Quantization in one
 *        paragraph" (absmax c = max|x|, nearest level of x/c, x_hat = c * q),
 *        "NF4: sixteen levels shaped like the weights" (8 negative / 8
 *        non-negative levels, exact 0, endpoints +-1), "Double quantization:
 *        the constants are not free" (256 constants per group, 8-bit floats, one
 *        fp32 second-level constant, mean subtracted first), "Where the
 *        gradients actually go" (chain rule through dequant(W)^T; only A and B
 *        get gradients).
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must point to memory of the current
 *     CUDA device and be 16-byte aligned.  The library never allocates or frees
 *     caller memory; the caller owns every buffer, including the workspace.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     is asynchronous on that stream.
 *   - Argument errors return QL_ERR_INVALID_ARG / QL_ERR_UNSUPPORTED /
 *     QL_ERR_WORKSPACE synchronously, before anything is launched.  A failed
 *     launch returns QL_ERR_CUDA.  Conditions the device detects (a non-finite
 *     input, a bounded wait that ran out) set bits in a per-device status word,
 *     which qlora_get_status() reads and clears.
 *   - Layouts are row-major.  A weight W in R^{N x K} (N = d_out, K = d_in) is
 *     quantized as the flat array of its N*K elements.  Element i is in 64-block
 *     i / 64, and that block is in double-quant group (i / 64) / 256.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or shape */
  QL_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype, r > 64, ...) */
  QL_ERR_WORKSPACE = 3,     /* workspace smaller than qlora_workspace_size() */
  QL_ERR_CUDA = 4,          /* a CUDA runtime / launch error */
  QL_ERR_NONFINITE = 5,     /* device: NaN or Inf met in a quantized block */
  QL_ERR_TIMEOUT = 6        /* device: a bounded wait inside a kernel ran out */
} ql_status;

typedef enum { QL_F32 = 0, QL_BF16 = 1 } ql_dtype;

/* Block sizes fixed by the method ([P2] §2.2). */
#define QL_BLOCK 64
#define QL_DQ_GROUP 256
#define QL_MAX_RANK 64

/*
 * An NF4 weight as stored on the device (all device pointers, caller-owned,
 * only read by the library):
 *   codes    uint8 [ceil(n/2)], n = rows*cols.  Byte k holds element 2k in its
 *            low nibble and element 2k+1 in its high nibble.
 *   absmax   fp32 [nb], nb = ceil(n/64): the block constants c_1.  NULL when
 *            the double-quantized form below is used.
 *   absmax_q uint8 [nb] E4M3 codes of (c_1 - mu) / s_2 (double quant).
 *   scale2   fp32 [ng], ng = ceil(nb/256): second-level constants s_2.
 *   offset   fp32 [1]: the mean mu subtracted before double quantization.
 * Reconstructed constant ([P3] "Double quantization"):
 *   c_hat = fl32(fl32(E4M3(absmax_q[b]) * scale2[b/256]) + offset[0]).
 */
typedef struct {
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* scale2;
  const float* offset;
  int64_t rows;   /* N */
  int64_t cols;   /* K */
} ql_nf4_weight;

/*
 * nf4_quantize — blockwise absmax NF4 quantization ([P3] "Quantization in one
 * paragraph"; levels per [P2] §2.1 and [P3] "NF4").
 *   x       device, n elements of type x_dt (QL_F32 or QL_BF16)
 *   codes   device out, uint8 [ceil(n/2)] packed as in ql_nf4_weight
 *   absmax  device out, fp32 [ceil(n/64)]: c_b = max|x| over the block (a
 *           partial last block uses its valid elements)
 * Code of element x in block b: with the fp32 decision thresholds
 * t_j = fl32(m_j * c_b), m_j = fl32(fl32(q_j + q_{j+1}) / 2), the code is
 * #{j : x > t_j} (ties go to the lower level).  A block with c_b == 0 codes
 * every element as the zero level (8).  An odd n pads the last high nibble
 * with 8.  NaN/Inf in a block sets QL_ERR_NONFINITE in the status word
 * (that block's outputs are then unspecified).  n may exceed 2^32.
 * Errors: QL_ERR_INVALID_ARG (n <= 0, a NULL or misaligned pointer, an
 * unknown dtype), QL_ERR_CUDA.
 */
ql_status nf4_quantize(const void* x, ql_dtype x_dt, int64_t n,
                       uint8_t* codes, float* absmax, void* stream);

/*
 * nf4_double_quant — quantize the fp32 block constants ([P2] §2.2, [P3]
 * "Double quantization: the constants are not free").
 *   absmax    device, fp32 [nb] (c_1 from nf4_quantize)
 *   absmax_q  device out, uint8 [nb] E4M3 codes
 *   scale2    device out, fp32 [ceil(nb/256)]
 *   offset    device out, fp32 [1]: mu
 *   ws        device workspace, >= qlora_workspace_size(QL_OP_DOUBLE_QUANT, nb, 0, 0, 0)
 * mu = fl32(S / nb) with S the float64 sum over a fixed adjacent-pair tree
 * (zero padded to a power of two).  Per group of 256: d = fl32(c - mu),
 * s_2 = fl32(max|d| / 448), code = E4M3_rne_satfinite(fl32(d / s_2)); a group
 * with s_2 == 0 stores code 0x00.
 * Errors: QL_ERR_INVALID_ARG (nb <= 0, a NULL or misaligned pointer),
 * QL_ERR_WORKSPACE (ws_bytes too small), QL_ERR_CUDA.
 */
ql_status nf4_double_quant(const float* absmax, int64_t nb, uint8_t* absmax_q,
                           float* scale2, float* offset, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Double quantization of a weight quantized in row slabs on several ranks
 * (data parallelism, each rank holding one slab).  The result is the double
 * quantization of [P2] §2.2 and [P3] "Double quantization: the constants are
 * not free" for the whole tensor; the split is this library's data-parallel
 * layout (the pages quantize on one GPU).  The mean is a sum over a
 * fixed adjacent-pair tree whose level-1 nodes are float64 sums of 2048
 * consecutive constants, so a slab whose constants start on a multiple of 2048
 * owns whole nodes:
 *   nf4_double_quant_level1  this slab's nodes: nodes[ceil(nb/2048)] (float64)
 *   nf4_double_quant_finish  given every slab's nodes in slab order
 *                            (n_nodes = ceil(nb_total/2048)), the mean of the
 *                            whole tensor and this slab's codes and scales
 * The concatenated results equal nf4_double_quant of the whole tensor bit for
 * bit.  The caller moves the nodes between ranks (an all-gather).  ws as for
 * nf4_double_quant with nb_total.  Errors: QL_ERR_INVALID_ARG (counts, a NULL
 * or misaligned pointer, n_nodes inconsistent with nb_total),
 * QL_ERR_WORKSPACE, QL_ERR_CUDA.
 */
ql_status nf4_double_quant_level1(const float* absmax, int64_t nb, double* nodes, void* stream);
ql_status nf4_double_quant_finish(const double* nodes, int64_t n_nodes, int64_t nb_total, const float* absmax,
                                  int64_t nb, uint8_t* absmax_q, float* scale2, float* offset, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * nf4_double_quant_noalloc — nf4_double_quant for callers that cannot
 * allocate device memory (no workspace argument).  The pages have no
 * counterpart; this is a library convenience.  Callers such as a plugin or
 * custom operator handed only tensors and a stream by a framework that owns
 * the device memory pool, or code that must not call cudaMalloc (it can
 * synchronize the device), use this instead of providing `ws`.
 *   Same arguments, outputs and results as nf4_double_quant, bit for bit.
 *   nb must be <= QL_NOALLOC_MAX_BLOCKS (64 Mi constants, i.e. weights of up
 *   to 4 Gi elements); larger nb returns QL_ERR_UNSUPPORTED.
 *   The scratch is a fixed 256.5 KiB array of device memory inside the
 *   library, held by every GPU that loads it until the process exits (one
 *   copy per CUDA context, since the library's module is loaded per context).
 *   The first call in a context looks its address up (cudaGetSymbolAddress)
 *   and caches it under the context's unique ID, so make that first call
 *   before any stream capture.  All calls in a context share the array: calls
 *   whose kernels may overlap on the GPU (different streams with no ordering)
 *   race and must not be issued.  The library never calls cudaMalloc, cudaFree
 *   or an allocating routine here.
 */
#define QL_NOALLOC_MAX_BLOCKS (1ll << 26)
ql_status nf4_double_quant_noalloc(const float* absmax, int64_t nb, uint8_t* absmax_q,
                                   float* scale2, float* offset, void* stream);

/*
 * qlora_merge — fold a trained adapter into the base weight:
 *   W' = W_hat + s B A  as a bf16 [N, K] weight, and/or that weight quantized
 *   again to NF4.  [P2] FAQ "Does QLoRA introduce inference latency overhead
 *   once the model is fine-tuned and deployed?": dequantize the base to 16 bits
 *   and merge, W = W_dequant + (alpha / r) B A.  [P3] "Pitfalls": merge in 16
 *   bits, then quantize the merged result if a quantized model is wanted
 *   ("How it's used in practice": peft's merge_and_unload()).
 * Arithmetic, per element (n, k), in this order:
 *   d  = sum_{j = 0 .. r-1} B[n, j] A[j, k]   fp32, each partial sum rounded
 *        (a bf16 x bf16 product is exact in fp32),
 *   W' = bf16(fl32(w_hat + fl32(s d))),   w_hat = bf16(fl32(q_code c_hat)).
 * Re-quantization codes W' exactly as nf4_quantize would code that bf16 tensor.
 *   w          NF4 weight (either constant form); K = w->cols % 64 == 0.
 *   A          device bf16 [r, K]; B device bf16 [N, r] (unused when r == 0).
 *   r          0 <= r <= QL_MAX_RANK (no multiple-of-8 rule here).
 *   s          alpha / r.
 *   W_out      device bf16 [N, K], or NULL.
 *   codes_out  device uint8 [N*K/2] and absmax_out device fp32 [N*K/64] (the
 *              fp32 constants; nf4_double_quant compresses them), both or
 *              neither.  At least one output must be given.  Outputs must not
 *              overlap the inputs.
 * A non-finite merged value sets QL_ERR_NONFINITE in the status word (when
 * re-quantizing).  Errors: QL_ERR_INVALID_ARG (bad pointer, alignment, K % 64,
 * output combination), QL_ERR_UNSUPPORTED (r > QL_MAX_RANK), QL_ERR_CUDA.
 */
ql_status qlora_merge(const ql_nf4_weight* w, const void* A, const void* B, int r, float s,
                      void* W_out, uint8_t* codes_out, float* absmax_out, void* stream);

/*
 * nf4_dequant — x_hat = bf16(fl32(q_code * c)) ([P3] "Quantization in one
 * paragraph"; [P2] §3 dequantize to BF16), c = absmax[b] or the double-quant
 * reconstruction when w->absmax is NULL.  out: device, rows*cols elements of
 * out_dt (QL_F32 skips the bf16 rounding).
 * Errors: QL_ERR_INVALID_ARG (NULL w, rows or cols <= 0, a misaligned weight
 * buffer or output, an unknown dtype), QL_ERR_CUDA.
 */
ql_status nf4_dequant(const ql_nf4_weight* w, void* out, ql_dtype out_dt, void* stream);

/*
 * qlora_linear_fwd — Y = X * W_hat^T + s * U * B^T, U = bf16(X * A^T)
 * ([P3] "Where the gradients actually go", [P2] §3).
 *   w      NF4 weight, rows = N, cols = K; K % 64 == 0
 *   X      device bf16 [M, K]
 *   A      device bf16 [r, K];  B device bf16 [N, r];  1 <= r <= 64, r % 8 == 0
 *   s      alpha / r
 *   Y      device out [M, N] of y_dt
 *   U_out  device out bf16 [M, r] (the tensor the backward reuses) or NULL
 *   ws     workspace >= qlora_workspace_size(QL_OP_FWD, M, N, K, r) (0 when
 *          r == 0 and M > 16; ws may then be NULL).  For 1 <= M <= 16 the
 *          small-token kernels keep fp32 part sums of Y and U there.
 * The main product accumulates in fp32 on the tensor cores from the exact
 * bf16 W_hat.  U is accumulated in fp32 (split over K, summed in a fixed
 * order) and rounded to bf16; the adapter term U (s B)^T enters the main fp32
 * accumulator with s B rounded to bf16 (exact when s is a power of two).
 * M == 0 launches nothing.  Errors: QL_ERR_INVALID_ARG (bad weight
 * descriptor, M < 0, K % 64 or N % 8 != 0, r < 0 or r % 8 != 0, a NULL or
 * misaligned pointer, an unknown dtype), QL_ERR_UNSUPPORTED (r > QL_MAX_RANK,
 * M, N or K >= 2^31), QL_ERR_WORKSPACE (ws_bytes too small), QL_ERR_CUDA; a
 * bounded device wait that ran out sets QL_ERR_TIMEOUT in the status word.
 */
ql_status qlora_linear_fwd(const ql_nf4_weight* w, const void* X, int64_t M,
                           const void* A, const void* B, int r, float s,
                           void* Y, ql_dtype y_dt, void* U_out,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * qlora_linear_bwd — gradients of <dY, Y> for the forward above
 * ([P3] "Where the gradients actually go": chain rule through W_hat^T, no
 * gradient for W; [P2] §3 step 5):
 *   V  = bf16(dY * B)                 [M, r]
 *   dX = dY * W_hat + s * V * A       [M, K]   (+= when accumulate_dx != 0)
 *   dA = s * V^T * X                  [r, K]
 *   dB = s * dY^T * U                 [N, r]
 *   X, dY, A, B: device bf16;  U: device bf16 [M, r] from the forward, or NULL
 *   to recompute it.  dX of dx_dt; dA, dB of grad_dt (overwritten).
 *   ws >= qlora_workspace_size(QL_OP_BWD, M, N, K, r).
 * M == 0 only zeroes dA and dB.  Errors: those of qlora_linear_fwd
 * (QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED, QL_ERR_WORKSPACE, QL_ERR_CUDA;
 * QL_ERR_TIMEOUT in the status word); U may be NULL (it is then recomputed)
 * but must be 16-byte aligned when given.
 */
ql_status qlora_linear_bwd(const ql_nf4_weight* w, const void* X, const void* dY, int64_t M,
                           const void* A, const void* B, int r, float s, const void* U,
                           void* dX, ql_dtype dx_dt, int accumulate_dx,
                           void* dA, void* dB, ql_dtype grad_dt,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * SiLU-gated MLP glue between three QLoRA linears (the pages adapt every
 * linear, [P3] "Seeing it in code": gate_proj, up_proj, down_proj).
 *   qlora_silu_gate_fwd: h = bf16(silu(g) * u), silu(x) = x * sigmoid(x)
 *   qlora_silu_gate_bwd: dg = bf16(dh * u * sig(g) * (1 + g (1 - sig(g)))),
 *                        du = bf16(dh * silu(g))
 * All device bf16 [n], n % 8 == 0.  Errors: QL_ERR_INVALID_ARG (n <= 0, a
 * NULL or misaligned pointer), QL_ERR_UNSUPPORTED (n % 8 != 0), QL_ERR_CUDA.
 */
ql_status qlora_silu_gate_fwd(const void* g, const void* u, void* h, int64_t n, void* stream);
ql_status qlora_silu_gate_bwd(const void* dh, const void* g, const void* u,
                              void* dg, void* du, int64_t n, void* stream);

/*
 * 4-bit float block formats ([P1] "Lesson 4 of the Finetuning Sessions",
 * "From FP32 to the 4-Bit Horizon": MXFP4 shares one 8-bit power-of-two (E8M0)
 * scale over 32 elements; NVFP4 shares one E4M3 scale over 16; "From Turing to
 * Blackwell": the 5th-generation tensor cores execute them natively).
 * Elements are E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), rounded to
 * nearest even and saturated at +-6; elements 2j, 2j+1 share byte j (low
 * nibble first); an odd n pads the last high nibble with +0.
 *
 * nvfp4_quantize: x device (x_dt) [n]; codes out uint8 [ceil(n/2)]; scales
 *   out uint8 [ceil(n/16)] E4M3 codes S_b; tensor_scale out fp32 [1]: s_t =
 *   fl32(amax / 2688) when use_tensor_scale (1 otherwise; 2688 = 6 * 448).
 *   Steps (fp32, one rounding each): denom = fl32(6 s_t), S_b =
 *   E4M3_rne_satfinite(fl32(amax_b / denom)), scale = fl32(S_b s_t), code =
 *   E2M1(fl32(x / scale)), 0 where scale == 0.  ws >=
 *   qlora_workspace_size(QL_OP_NVFP4, n, 0, 0, 0) (the tensor maximum).
 * mxfp4_quantize: scales out uint8 [ceil(n/32)] E8M0 codes k_b + 127, k_b =
 *   floor(log2 amax_b) - 2 clamped to [-127, 127] (-127 for an all-zero
 *   block); code = E2M1(x 2^-k_b).
 * nvfp4_dequant / mxfp4_dequant: out fp32 [n], x_hat = fl32(E2M1(code)
 *   fl32(S_b s_t)) / E2M1(code) 2^k_b (exact).
 * NaN/Inf in the input sets QL_ERR_NONFINITE in the status word (outputs are
 * then unspecified).  Errors: QL_ERR_INVALID_ARG (n <= 0, a NULL or misaligned
 * pointer, an unknown dtype), QL_ERR_WORKSPACE, QL_ERR_CUDA.
 */
ql_status nvfp4_quantize(const void* x, ql_dtype x_dt, int64_t n, int use_tensor_scale, uint8_t* codes,
                         uint8_t* scales, float* tensor_scale, void* ws, size_t ws_bytes, void* stream);
ql_status mxfp4_quantize(const void* x, ql_dtype x_dt, int64_t n, uint8_t* codes, uint8_t* scales, void* stream);
ql_status nvfp4_dequant(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t n,
                        float* out, void* stream);
ql_status mxfp4_dequant(const uint8_t* codes, const uint8_t* scales, int64_t n, float* out, void* stream);

/*
 * NVFP4 x NVFP4 GEMM on the block-scaled tensor cores ([P1] "Lesson 4 of the
 * Finetuning Sessions", "From Turing to Blackwell": the 5th-generation tensor
 * cores execute the 4-bit block formats natively; "From FP32 to the 4-Bit
 * Horizon": E2M1 elements, one E4M3 scale per 16, one fp32 tensor scale):
 *   Y[m, n] = s_a s_b sum_k (E2M1(a[m, k]) S_a[m, k/16]) (E2M1(b[n, k]) S_b[n, k/16])
 * for A [M, K] and B [N, K] row-major, each quantized by nvfp4_quantize as one
 * tensor of rows x K elements (so each block of 16 runs along K).  This is
 * W4A4: both operands are 4-bit, not the QLoRA linear's bf16 activations.
 *
 * nvfp4_scale_atoms: scales device uint8 [rows * K/16] (row-major, as
 *   nvfp4_quantize writes them) -> atoms device out uint8
 *   [nvfp4_scale_atoms_bytes(rows, K)]: per 128-row tile and 64-element K
 *   block, 512 bytes with row m = m0 + 32 m1 (m0 < 32, m1 < 4) and scale kb < 4
 *   at byte 16 m0 + 4 m1 + kb (the tensor cores' scale layout); rows past
 *   `rows` in the last tile are 0.
 * nvfp4_gemm: a_codes / b_codes device uint8 [M * K/2] / [N * K/2]; a_atoms /
 *   b_atoms from nvfp4_scale_atoms with rows = M / N; a_tensor_scale /
 *   b_tensor_scale device fp32 [1]; Y device out fp32 [M, N] row-major.  The
 *   products are exact and accumulate in fp32 on the tensor cores (order
 *   unspecified); then Y = fl32(acc fl32(s_a s_b)).
 * Constraints: K a multiple of 256; M, K < 2^31; N < 2^23.  Errors:
 * QL_ERR_INVALID_ARG (M, N or K < 1, a NULL or misaligned pointer),
 * QL_ERR_UNSUPPORTED (K % 256 != 0, sizes past the constraints), QL_ERR_CUDA.
 * A bounded wait that runs out sets QL_ERR_TIMEOUT in the status word.
 */
size_t nvfp4_scale_atoms_bytes(int64_t rows, int64_t K);
ql_status nvfp4_scale_atoms(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* atoms, void* stream);
ql_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_atoms, const float* a_tensor_scale,
                     const uint8_t* b_codes, const uint8_t* b_atoms, const float* b_tensor_scale, int64_t M,
                     int64_t N, int64_t K, float* Y, void* stream);

/*
 * MXFP4 x MXFP4 GEMM on the same tensor-core path ("From FP32 to the 4-Bit
 * Horizon": MXFP4 is E2M1 elements with one power-of-two E8M0 scale per 32 and
 * no tensor scale):
 *   Y[m, n] = sum_k (E2M1(a[m, k]) 2^{k_a[m, k/32]}) (E2M1(b[n, k]) 2^{k_b[n, k/32]})
 * for A [M, K] and B [N, K] row-major, each quantized by mxfp4_quantize as one
 * tensor of rows x K elements.
 *
 * mxfp4_scale_atoms: scales device uint8 [rows * K/32] (the E8M0 bytes
 *   mxfp4_quantize writes, row-major) -> atoms device out uint8
 *   [mxfp4_scale_atoms_bytes(rows, K)]: per 128-row tile and 128-element K
 *   block, 512 bytes in the layout nvfp4_scale_atoms uses (scale kb < 4 of the
 *   block now covering elements 32 kb .. 32 kb + 31); rows past `rows` are 0.
 *   mxfp4_scale_atoms_bytes returns 0 for rows < 1 or K < 128.
 * mxfp4_gemm: a_codes / b_codes device uint8 [M * K/2] / [N * K/2]; a_atoms /
 *   b_atoms from mxfp4_scale_atoms with rows = M / N; Y device out fp32 [M, N]
 *   row-major.  Products are exact and accumulate in fp32 on the tensor cores
 *   (order unspecified); no scaling after the accumulation.
 * Constraints and errors as for nvfp4_gemm.
 */
size_t mxfp4_scale_atoms_bytes(int64_t rows, int64_t K);
ql_status mxfp4_scale_atoms(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* atoms, void* stream);
ql_status mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_atoms, const uint8_t* b_codes, const uint8_t* b_atoms,
                     int64_t M, int64_t N, int64_t K, float* Y, void* stream);

/*
 * qlora_adamw_step — one AdamW update of adapter parameters with fp32 states
 * (the paged optimizer: [P2] §2.3 and [P3] "Paged optimizers: surviving the
 * spikes" keep the states in unified memory, paged to host RAM under memory
 * pressure and back for the next update; [P3] "How it's used in practice"
 * names the 32-bit variant).  The pages give no update formula; paging leaves
 * the arithmetic alone, so this is AdamW with decoupled weight decay.  Per
 * element, each operation one fp32 IEEE operation in this order, with keep =
 * fl32(1 - lr wd), c1 = fl32(1 - beta1^t), c2 = fl32(1 - beta2^t) computed on
 * the host in float64 from the fp32 arguments:
 *   p = fl32(p keep);  m = fl32(fl32(beta1 m) + fl32((1 - beta1) g));
 *   v = fl32(fl32(beta2 v) + fl32(fl32((1 - beta2) g) g));
 *   d = fl32(fl32(sqrt(fl32(v / c2))) + eps);
 *   p = fl32(p - fl32(lr fl32(fl32(m / c1) / d))).
 *   p, m, v  fp32 [n], updated in place; g fp32 [n].  Device memory or CUDA
 *            managed memory (wherever its pages currently are).
 *   p_bf16   bf16 [n] copy of the updated p (the adapter the linear reads), or
 *            NULL.   t: step number, >= 1.
 * Errors: QL_ERR_INVALID_ARG (n <= 0, t < 1, a beta outside [0, 1), eps < 0,
 * a NULL or misaligned pointer), QL_ERR_CUDA.
 *
 * qlora_paged_prefetch — move a managed range (cudaMallocManaged memory owned
 * by the caller) to the current device (QL_PAGE_DEVICE), before an update, or
 * to host memory (QL_PAGE_HOST), to free device memory after one; stream
 * ordered.  Errors: QL_ERR_INVALID_ARG (NULL, bytes == 0, an unknown `where`,
 * memory that is not managed), QL_ERR_CUDA.
 */
#define QL_PAGE_DEVICE 0
#define QL_PAGE_HOST 1
ql_status qlora_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int64_t t,
                           float lr, float beta1, float beta2, float eps, float weight_decay, void* stream);
ql_status qlora_paged_prefetch(const void* ptr, size_t bytes, int where, void* stream);

/* Workspace query.  op: one of the QL_OP_* values; unused sizes are ignored. */
#define QL_OP_DOUBLE_QUANT 0   /* M = nb */
#define QL_OP_FWD 1
#define QL_OP_BWD 2
#define QL_OP_NVFP4 3          /* M = n */
size_t qlora_workspace_size(int op, int64_t M, int64_t N, int64_t K, int r);

/* Bytes needed for n parameters: ceil(n/2) codes + (dq ? nb + 4*ng + 4 : 4*nb)
 * ([P2] §2.2 and §4: 0.5 + 0.016 bytes per parameter with double quant). */
int64_t nf4_storage_bytes(int64_t n, int dq);

/* The 16 NF4 levels as fp32, increasing; index 8 is the exact zero
 * ([P2] §2.1 formula, read per [P3] "NF4": see nf4_quantize).  Host memory. */
void nf4_codebook(float out[16]);

/* Synchronizes `stream`, then reads and clears the current device's status
 * word.  Returns QL_OK, QL_ERR_NONFINITE or QL_ERR_TIMEOUT (the first set). */
ql_status qlora_get_status(void* stream);

/*
 * Per-kernel device timing, for profiling.  qlora_trace_enable(1) starts
 * recording a CUDA event pair around every kernel the library launches (on the
 * caller's stream); qlora_trace_enable(0) stops; qlora_trace_enable_kinds(mask)
 * records only the kinds k with bit k of mask set.  Each of these calls
 * discards earlier records.  An event pair around a kernel also keeps that
 * launch from starting while the previous kernel on the stream finishes (the
 * library otherwise overlaps consecutive launches: programmatic dependent
 * launch), so trace only the kinds you need.  qlora_trace_read waits for the
 * recorded events, writes for each kernel kind k < max_kinds the total device
 * milliseconds and launch count, clears the records and returns the number of
 * kinds written.  Kind names come from qlora_trace_kind_name.  Host-side only;
 * the caller owns the arrays.  No counterpart on the pages (instrumentation).
 */
void qlora_trace_enable(int on);
void qlora_trace_enable_kinds(unsigned mask);
int qlora_trace_read(double* total_ms, int* launches, int max_kinds);
const char* qlora_trace_kind_name(int kind);

/*
 * Failure-detection self-test (no counterpart on the pages).  Every pipelined
 * kernel of the library waits on mbarriers with a bounded number of polls
 * (each poll suspends at most about 1 us); a wait that runs out records
 * QL_ERR_TIMEOUT in the device status word and the kernel returns instead of
 * hanging.  This entry point launches one CTA whose wait nothing ever
 * satisfies, limited to `polls` polls, on `stream`; the next qlora_get_status
 * returns QL_ERR_TIMEOUT and the CUDA context stays usable.
 * polls: 1 .. 2^20 (QL_ERR_INVALID_ARG otherwise).  Allocates nothing.
 */
ql_status qlora_selftest_wait_timeout(int64_t polls, void* stream);

/* Human-readable name of a status code (static string). */
const char* qlora_status_string(ql_status s);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
