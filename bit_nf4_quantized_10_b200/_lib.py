"""ctypes binding of libqlora_nf4.so (argument marshalling only).

Every function here has the name of the C entry point it calls (see
include/qlora_nf4.h), takes torch tensors for device buffers, passes their
data pointers and the current CUDA stream, and raises QLoraError on a non-OK
status.  All computation happens in the library's kernels; there is no
fallback: if the library cannot be loaded, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QL_OK, QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED, QL_ERR_WORKSPACE, QL_ERR_CUDA, QL_ERR_NONFINITE, QL_ERR_TIMEOUT = range(7)
QL_F32, QL_BF16 = 0, 1
QL_OP_DOUBLE_QUANT, QL_OP_FWD, QL_OP_BWD, QL_OP_NVFP4 = 0, 1, 2, 3
QL_PAGE_DEVICE, QL_PAGE_HOST = 0, 1

EXPORTS = ("nf4_quantize", "nf4_double_quant", "nf4_double_quant_noalloc", "nf4_dequant", "qlora_linear_fwd", "qlora_linear_bwd",
           "qlora_silu_gate_fwd", "qlora_silu_gate_bwd", "qlora_workspace_size", "nf4_storage_bytes",
           "nf4_codebook", "qlora_get_status", "qlora_status_string", "qlora_selftest_wait_timeout",
           "qlora_merge", "nf4_double_quant_level1", "nf4_double_quant_finish", "nvfp4_quantize", "mxfp4_quantize",
           "nvfp4_dequant", "mxfp4_dequant", "qlora_adamw_step", "qlora_paged_prefetch", "nvfp4_scale_atoms_bytes",
           "nvfp4_scale_atoms", "nvfp4_gemm", "mxfp4_scale_atoms_bytes", "mxfp4_scale_atoms", "mxfp4_gemm")


class QLoraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class ql_nf4_weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p), ("absmax_q", ctypes.c_void_p),
                ("scale2", ctypes.c_void_p), ("offset", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python bit_nf4_quantized_10_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    W = ctypes.POINTER(ql_nf4_weight)
    sig = {
        "nf4_quantize": (i32, [vp, i32, i64, vp, vp, vp]),
        "nf4_double_quant": (i32, [vp, i64, vp, vp, vp, vp, sz, vp]),
        "nf4_double_quant_noalloc": (i32, [vp, i64, vp, vp, vp, vp]),
        "nf4_dequant": (i32, [W, vp, i32, vp]),
        "qlora_linear_fwd": (i32, [W, vp, i64, vp, vp, i32, f32, vp, i32, vp, vp, sz, vp]),
        "qlora_linear_bwd": (i32, [W, vp, vp, i64, vp, vp, i32, f32, vp, vp, i32, i32, vp, vp, i32, vp, sz, vp]),
        "qlora_silu_gate_fwd": (i32, [vp, vp, vp, i64, vp]),
        "qlora_silu_gate_bwd": (i32, [vp, vp, vp, vp, vp, i64, vp]),
        "qlora_workspace_size": (sz, [i32, i64, i64, i64, i32]),
        "nf4_storage_bytes": (i64, [i64, i32]),
        "nf4_codebook": (None, [ctypes.POINTER(ctypes.c_float)]),
        "qlora_get_status": (i32, [vp]),
        "qlora_status_string": (ctypes.c_char_p, [i32]),
        "qlora_selftest_wait_timeout": (i32, [i64, vp]),
        "qlora_merge": (i32, [W, vp, vp, i32, f32, vp, vp, vp, vp]),
        "nf4_double_quant_level1": (i32, [vp, i64, vp, vp]),
        "nf4_double_quant_finish": (i32, [vp, i64, i64, vp, i64, vp, vp, vp, vp, sz, vp]),
        "nvfp4_quantize": (i32, [vp, i32, i64, i32, vp, vp, vp, vp, sz, vp]),
        "mxfp4_quantize": (i32, [vp, i32, i64, vp, vp, vp]),
        "nvfp4_dequant": (i32, [vp, vp, vp, i64, vp, vp]),
        "mxfp4_dequant": (i32, [vp, vp, i64, vp, vp]),
        "qlora_adamw_step": (i32, [vp, vp, vp, vp, vp, i64, i64, f32, f32, f32, f32, f32, vp]),
        "qlora_paged_prefetch": (i32, [vp, sz, i32, vp]),
        "nvfp4_scale_atoms_bytes": (sz, [i64, i64]),
        "nvfp4_scale_atoms": (i32, [vp, i64, i64, vp, vp]),
        "nvfp4_gemm": (i32, [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]),
        "mxfp4_scale_atoms_bytes": (sz, [i64, i64]),
        "mxfp4_scale_atoms": (i32, [vp, i64, i64, vp, vp]),
        "mxfp4_gemm": (i32, [vp, vp, vp, vp, i64, i64, i64, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.qlora_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != QL_OK:
        raise QLoraError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return QL_F32
    if t == torch.bfloat16:
        return QL_BF16
    raise TypeError(f"unsupported dtype {t}")


# ----------------------------------------------------------------- host helpers
def nf4_codebook() -> list[float]:
    buf = (ctypes.c_float * 16)()
    LIB.nf4_codebook(buf)
    return list(buf)


def nf4_storage_bytes(n: int, dq: bool) -> int:
    return int(LIB.nf4_storage_bytes(int(n), 1 if dq else 0))


def qlora_workspace_size(op: int, M: int, N: int = 0, K: int = 0, r: int = 0) -> int:
    return int(LIB.qlora_workspace_size(int(op), int(M), int(N), int(K), int(r)))


def qlora_get_status(stream=None) -> int:
    return int(LIB.qlora_get_status(_stream(stream)))


def qlora_selftest_wait_timeout(polls: int, stream=None) -> None:
    """Launch the bounded-wait self-test (a wait nothing satisfies, limited to
    `polls` polls); the next qlora_get_status reports QL_ERR_TIMEOUT."""
    _check(LIB.qlora_selftest_wait_timeout(int(polls), _stream(stream)), "qlora_selftest_wait_timeout")


# ------------------------------------------------------------------ device calls
def nf4_quantize(x: torch.Tensor, codes: torch.Tensor, absmax: torch.Tensor, stream=None) -> None:
    _check(LIB.nf4_quantize(_ptr(x), _dt(x.dtype), x.numel(), _ptr(codes), _ptr(absmax), _stream(stream)),
           "nf4_quantize")


def nf4_double_quant(absmax: torch.Tensor, absmax_q: torch.Tensor, scale2: torch.Tensor, offset: torch.Tensor,
                     ws: torch.Tensor, stream=None) -> None:
    _check(LIB.nf4_double_quant(_ptr(absmax), absmax.numel(), _ptr(absmax_q), _ptr(scale2), _ptr(offset),
                                _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "nf4_double_quant")


def nf4_double_quant_noalloc(absmax: torch.Tensor, absmax_q: torch.Tensor, scale2: torch.Tensor,
                             offset: torch.Tensor, stream=None) -> None:
    """nf4_double_quant without a workspace, for callers that cannot allocate
    device memory; the library uses a fixed internal scratch array instead."""
    _check(LIB.nf4_double_quant_noalloc(_ptr(absmax), absmax.numel(), _ptr(absmax_q), _ptr(scale2), _ptr(offset),
                                        _stream(stream)), "nf4_double_quant_noalloc")


def nf4_double_quant_level1(absmax: torch.Tensor, nodes: torch.Tensor, stream=None) -> None:
    _check(LIB.nf4_double_quant_level1(_ptr(absmax), absmax.numel(), _ptr(nodes), _stream(stream)),
           "nf4_double_quant_level1")


def nf4_double_quant_finish(nodes: torch.Tensor, nb_total: int, absmax: torch.Tensor, absmax_q: torch.Tensor,
                            scale2: torch.Tensor, offset: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(LIB.nf4_double_quant_finish(_ptr(nodes), nodes.numel(), int(nb_total), _ptr(absmax), absmax.numel(),
                                       _ptr(absmax_q), _ptr(scale2), _ptr(offset), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "nf4_double_quant_finish")


def nvfp4_quantize(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, tensor_scale: torch.Tensor,
                   ws: torch.Tensor, use_tensor_scale: bool = True, stream=None) -> None:
    _check(LIB.nvfp4_quantize(_ptr(x), _dt(x.dtype), x.numel(), 1 if use_tensor_scale else 0, _ptr(codes),
                              _ptr(scales), _ptr(tensor_scale), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)), "nvfp4_quantize")


def nvfp4_scale_atoms_bytes(rows: int, K: int) -> int:
    return int(LIB.nvfp4_scale_atoms_bytes(int(rows), int(K)))


def nvfp4_scale_atoms(scales: torch.Tensor, rows: int, K: int, atoms: torch.Tensor, stream=None) -> None:
    _check(LIB.nvfp4_scale_atoms(_ptr(scales), int(rows), int(K), _ptr(atoms), _stream(stream)), "nvfp4_scale_atoms")


def nvfp4_gemm(a_codes: torch.Tensor, a_atoms: torch.Tensor, a_tensor_scale: torch.Tensor, b_codes: torch.Tensor,
               b_atoms: torch.Tensor, b_tensor_scale: torch.Tensor, M: int, N: int, K: int, Y: torch.Tensor,
               stream=None) -> None:
    _check(LIB.nvfp4_gemm(_ptr(a_codes), _ptr(a_atoms), _ptr(a_tensor_scale), _ptr(b_codes), _ptr(b_atoms),
                          _ptr(b_tensor_scale), int(M), int(N), int(K), _ptr(Y), _stream(stream)), "nvfp4_gemm")


def mxfp4_scale_atoms_bytes(rows: int, K: int) -> int:
    return int(LIB.mxfp4_scale_atoms_bytes(int(rows), int(K)))


def mxfp4_scale_atoms(scales: torch.Tensor, rows: int, K: int, atoms: torch.Tensor, stream=None) -> None:
    _check(LIB.mxfp4_scale_atoms(_ptr(scales), int(rows), int(K), _ptr(atoms), _stream(stream)), "mxfp4_scale_atoms")


def mxfp4_gemm(a_codes: torch.Tensor, a_atoms: torch.Tensor, b_codes: torch.Tensor, b_atoms: torch.Tensor, M: int,
               N: int, K: int, Y: torch.Tensor, stream=None) -> None:
    _check(LIB.mxfp4_gemm(_ptr(a_codes), _ptr(a_atoms), _ptr(b_codes), _ptr(b_atoms), int(M), int(N), int(K),
                          _ptr(Y), _stream(stream)), "mxfp4_gemm")


def mxfp4_quantize(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    _check(LIB.mxfp4_quantize(_ptr(x), _dt(x.dtype), x.numel(), _ptr(codes), _ptr(scales), _stream(stream)),
           "mxfp4_quantize")


def nvfp4_dequant(codes: torch.Tensor, scales: torch.Tensor, tensor_scale: torch.Tensor, n: int, out: torch.Tensor,
                  stream=None) -> None:
    _check(LIB.nvfp4_dequant(_ptr(codes), _ptr(scales), _ptr(tensor_scale), int(n), _ptr(out), _stream(stream)),
           "nvfp4_dequant")


def mxfp4_dequant(codes: torch.Tensor, scales: torch.Tensor, n: int, out: torch.Tensor, stream=None) -> None:
    _check(LIB.mxfp4_dequant(_ptr(codes), _ptr(scales), int(n), _ptr(out), _stream(stream)), "mxfp4_dequant")


def qlora_adamw_step(p, g, m, v, n: int, t: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                     eps: float = 1e-8, weight_decay: float = 0.0, p_bf16=None, stream=None) -> None:
    """p, g, m, v: fp32 tensors or raw device / managed-memory addresses (ints)."""
    _check(LIB.qlora_adamw_step(_ptr(p), _ptr(g), _ptr(m), _ptr(v), _ptr(p_bf16), int(n), int(t), float(lr),
                                float(beta1), float(beta2), float(eps), float(weight_decay), _stream(stream)),
           "qlora_adamw_step")


def qlora_paged_prefetch(ptr, nbytes: int, where: int, stream=None) -> None:
    _check(LIB.qlora_paged_prefetch(_ptr(ptr), int(nbytes), int(where), _stream(stream)), "qlora_paged_prefetch")


def nf4_dequant(w: "NF4Weight", out: torch.Tensor, stream=None) -> None:
    d = w.desc()
    _check(LIB.nf4_dequant(ctypes.byref(d), _ptr(out), _dt(out.dtype), _stream(stream)), "nf4_dequant")


def qlora_linear_fwd(w: "NF4Weight", X, A, B, r: int, s: float, Y, U_out=None, ws=None, stream=None) -> None:
    d = w.desc()
    M = X.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(LIB.qlora_linear_fwd(ctypes.byref(d), _ptr(X), M, _ptr(A), _ptr(B), int(r), float(s), _ptr(Y),
                                _dt(Y.dtype), _ptr(U_out), _ptr(ws), ws_bytes, _stream(stream)), "qlora_linear_fwd")


def qlora_linear_bwd(w: "NF4Weight", X, dY, A, B, r: int, s: float, U, dX, dA, dB, accumulate_dx: bool = False,
                     ws=None, stream=None) -> None:
    d = w.desc()
    M = dY.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(LIB.qlora_linear_bwd(ctypes.byref(d), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B), int(r), float(s), _ptr(U),
                                _ptr(dX), _dt(dX.dtype), 1 if accumulate_dx else 0, _ptr(dA), _ptr(dB),
                                _dt(dA.dtype), _ptr(ws), ws_bytes, _stream(stream)), "qlora_linear_bwd")


def qlora_merge(w: "NF4Weight", A, B, r: int, s: float, W_out=None, codes_out=None, absmax_out=None,
                stream=None) -> None:
    """W' = W_hat + s B A as bf16 (W_out) and/or quantized again (codes_out, absmax_out)."""
    d = w.desc()
    _check(LIB.qlora_merge(ctypes.byref(d), _ptr(A), _ptr(B), int(r), float(s), _ptr(W_out), _ptr(codes_out),
                           _ptr(absmax_out), _stream(stream)), "qlora_merge")


def qlora_silu_gate_fwd(g, u, h, stream=None) -> None:
    _check(LIB.qlora_silu_gate_fwd(_ptr(g), _ptr(u), _ptr(h), g.numel(), _stream(stream)), "qlora_silu_gate_fwd")


def qlora_silu_gate_bwd(dh, g, u, dg, du, stream=None) -> None:
    _check(LIB.qlora_silu_gate_bwd(_ptr(dh), _ptr(g), _ptr(u), _ptr(dg), _ptr(du), g.numel(), _stream(stream)),
           "qlora_silu_gate_bwd")


# ------------------------------------------------------------- weight container
class NF4Weight:
    """Device buffers of one quantized weight [rows, cols] (see ql_nf4_weight)."""

    def __init__(self, rows: int, cols: int, codes, absmax=None, absmax_q=None, scale2=None, offset=None):
        self.rows, self.cols = int(rows), int(cols)
        self.codes, self.absmax = codes, absmax
        self.absmax_q, self.scale2, self.offset = absmax_q, scale2, offset
        self._desc = None

    @property
    def double_quant(self) -> bool:
        return self.absmax is None

    def desc(self) -> ql_nf4_weight:
        if self._desc is None:
            self._desc = ql_nf4_weight(_ptr(self.codes), _ptr(self.absmax), _ptr(self.absmax_q),
                                       _ptr(self.scale2), _ptr(self.offset), self.rows, self.cols)
        return self._desc

    @staticmethod
    def allocate(rows: int, cols: int, device, dq: bool = True) -> "NF4Weight":
        n = rows * cols
        nb = -(-n // 64)
        ng = -(-nb // 256)
        codes = torch.empty(-(-n // 2), dtype=torch.uint8, device=device)
        if not dq:
            return NF4Weight(rows, cols, codes, absmax=torch.empty(nb, dtype=torch.float32, device=device))
        return NF4Weight(rows, cols, codes, absmax_q=torch.empty(nb, dtype=torch.uint8, device=device),
                         scale2=torch.empty(ng, dtype=torch.float32, device=device),
                         offset=torch.empty(1, dtype=torch.float32, device=device))


def quantize_weight(W: torch.Tensor, dq: bool = True, stream=None, keep_absmax: bool = False):
    """Quantize a device weight [rows, cols] (fp32 or bf16) with nf4_quantize and,
    when dq, nf4_double_quant.  Buffers are allocated with torch.  Returns the
    NF4Weight (and the fp32 constants when keep_absmax)."""
    rows, cols = W.shape
    n = W.numel()
    nb = -(-n // 64)
    dev = W.device
    codes = torch.empty(-(-n // 2), dtype=torch.uint8, device=dev)
    absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    nf4_quantize(W, codes, absmax, stream)
    if not dq:
        return NF4Weight(rows, cols, codes, absmax=absmax)
    ng = -(-nb // 256)
    absmax_q = torch.empty(nb, dtype=torch.uint8, device=dev)
    scale2 = torch.empty(ng, dtype=torch.float32, device=dev)
    offset = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, qlora_workspace_size(QL_OP_DOUBLE_QUANT, nb)), dtype=torch.uint8, device=dev)
    nf4_double_quant(absmax, absmax_q, scale2, offset, ws, stream)
    w = NF4Weight(rows, cols, codes, absmax_q=absmax_q, scale2=scale2, offset=offset)
    return (w, absmax) if keep_absmax else w
