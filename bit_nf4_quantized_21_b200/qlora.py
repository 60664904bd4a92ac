"""Python binding of libqlora (ctypes): argument marshalling only.

Every function here has the name of the C entry point it calls
(include/qlora.h) and does nothing but turn torch tensors into device
pointers, pick up the current CUDA stream, call the library and raise on a
non-OK status.  There is no fallback path: if libqlora.so is missing, or a
tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# the library to load: libqlora.so, or another build of it (the debug build
# with index-range checks, libqlora_debug.so) named by QLORA_LIB
LIB_PATH = os.environ.get("QLORA_LIB") or os.path.join(_PKG, "libqlora.so")

QLORA_OK = 0
QLORA_F32 = 0
QLORA_BF16 = 1
DEV_NONFINITE = 1
DEV_TIMEOUT = 2

EXPORTED = (
    "qlora_nf4_sizes", "qlora_nf4_codebook", "qlora_quantize_nf4", "qlora_dequantize",
    "qlora_workspace_bytes", "qlora_linear_fwd", "qlora_linear_bwd", "qlora_status_string",
    "qlora_version", "qlora_linear_fwd_noalloc", "qlora_lora_linear_fwd", "qlora_lora_linear_bwd",
    "qlora_adam_step", "qlora_merge_nf4", "qlora_workspace_bytes_dropout", "qlora_lora_dropout_mask",
    "qlora_linear_fwd_dropout", "qlora_linear_bwd_dropout", "qlora_paged_alloc", "qlora_paged_free",
    "qlora_paged_prefetch", "qlora_debug_set_wait_limit", "qlora_debug_inject_stall",
    "qlora_debug_set_pair_mtiles", "qlora_debug_checks_enabled", "qlora_debug_range_check",
    "qlora_debug_range_selftest",
)


class QloraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class GemmEventsC(ctypes.Structure):
    _fields_ = [("gemm_start", ctypes.c_void_p), ("gemm_end", ctypes.c_void_p)]


def _events(ev):
    """(start, end) torch.cuda.Event pair -> qlora_gemm_events, or None."""
    if ev is None:
        return None
    for e in ev:
        if not e.cuda_event:      # torch creates the CUDA event on first record
            e.record()
    return ctypes.byref(GemmEventsC(ev[0].cuda_event, ev[1].cuda_event))


class NF4WeightC(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
        ("blocksize", ctypes.c_int32), ("group", ctypes.c_int32),
        ("double_quant", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("absmax_q8", ctypes.c_void_p),
        ("group_scale", ctypes.c_void_p), ("absmax_f32", ctypes.c_void_p),
    ]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libqlora.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libqlora.so not found at {LIB_PATH}; build it with "
                    "`python -m bit_nf4_quantized_21_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
            L.qlora_nf4_sizes.argtypes = [I64, I64, I32, P, P, P]
            L.qlora_nf4_sizes.restype = I32
            L.qlora_nf4_codebook.argtypes = [P]
            L.qlora_nf4_codebook.restype = None
            L.qlora_quantize_nf4.argtypes = [P, I32, ctypes.POINTER(NF4WeightC), P, P]
            L.qlora_quantize_nf4.restype = I32
            L.qlora_dequantize.argtypes = [ctypes.POINTER(NF4WeightC), P, P]
            L.qlora_dequantize.restype = I32
            L.qlora_workspace_bytes.argtypes = [I64, I64, I64, I32]
            L.qlora_workspace_bytes.restype = ctypes.c_size_t
            L.qlora_linear_fwd.argtypes = [P, I64, ctypes.POINTER(NF4WeightC), P, P, I32, F, P, P, P,
                                           ctypes.c_size_t, P, P, P]
            L.qlora_linear_fwd.restype = I32
            L.qlora_linear_bwd.argtypes = [P, P, I64, ctypes.POINTER(NF4WeightC), P, P, I32, F, P, P,
                                           P, P, I32, P, ctypes.c_size_t, P, P, P]
            L.qlora_linear_bwd.restype = I32
            L.qlora_linear_fwd_noalloc.argtypes = [P, I64, ctypes.POINTER(NF4WeightC), P, P, I32, F, P,
                                                   P, P, P]
            L.qlora_linear_fwd_noalloc.restype = I32
            L.qlora_lora_linear_fwd.argtypes = [P, I64, P, I64, I64, P, P, I32, F, P, P, P, ctypes.c_size_t,
                                                P, P, P]
            L.qlora_lora_linear_fwd.restype = I32
            L.qlora_lora_linear_bwd.argtypes = [P, P, I64, P, I64, I64, P, P, I32, F, P, P, P, P, I32, P,
                                                ctypes.c_size_t, P, P, P]
            L.qlora_lora_linear_bwd.restype = I32
            L.qlora_adam_step.argtypes = [P, P, P, P, P, I32, I64, I64, F, F, F, F, F, F, P, P]
            L.qlora_adam_step.restype = I32
            L.qlora_merge_nf4.argtypes = [ctypes.POINTER(NF4WeightC), P, P, I32, F, P, ctypes.POINTER(NF4WeightC),
                                          P, P]
            L.qlora_merge_nf4.restype = I32
            D, U64 = ctypes.c_double, ctypes.c_uint64
            L.qlora_workspace_bytes_dropout.argtypes = [I64, I64, I64, I32]
            L.qlora_workspace_bytes_dropout.restype = ctypes.c_size_t
            L.qlora_lora_dropout_mask.argtypes = [I64, I64, D, U64, P, P]
            L.qlora_lora_dropout_mask.restype = I32
            L.qlora_linear_fwd_dropout.argtypes = [P, I64, ctypes.POINTER(NF4WeightC), P, P, I32, F, D, U64, P, P,
                                                   P, ctypes.c_size_t, P, P, P]
            L.qlora_linear_fwd_dropout.restype = I32
            L.qlora_linear_bwd_dropout.argtypes = [P, P, I64, ctypes.POINTER(NF4WeightC), P, P, I32, F, D, U64, P,
                                                   P, P, P, I32, P, ctypes.c_size_t, P, P, P]
            L.qlora_linear_bwd_dropout.restype = I32
            L.qlora_paged_alloc.argtypes = [ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p)]
            L.qlora_paged_alloc.restype = I32
            L.qlora_paged_free.argtypes = [P]
            L.qlora_paged_free.restype = I32
            L.qlora_paged_prefetch.argtypes = [P, ctypes.c_size_t, I32, P]
            L.qlora_paged_prefetch.restype = I32
            L.qlora_debug_set_wait_limit.argtypes = [U64]
            L.qlora_debug_set_wait_limit.restype = I32
            L.qlora_debug_inject_stall.argtypes = [I32]
            L.qlora_debug_inject_stall.restype = I32
            L.qlora_debug_set_pair_mtiles.argtypes = [I32]
            L.qlora_debug_set_pair_mtiles.restype = I32
            L.qlora_debug_checks_enabled.argtypes = []
            L.qlora_debug_checks_enabled.restype = I32
            L.qlora_debug_range_check.argtypes = [ctypes.POINTER(ctypes.c_uint)]
            L.qlora_debug_range_check.restype = I32
            L.qlora_debug_range_selftest.argtypes = [P]
            L.qlora_debug_range_selftest.restype = I32
            L.qlora_status_string.argtypes = [I32]
            L.qlora_status_string.restype = ctypes.c_char_p
            L.qlora_version.argtypes = []
            L.qlora_version.restype = ctypes.c_char_p
            _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().qlora_status_string(int(s)).decode()


def _check(rc: int, where: str) -> None:
    if rc != QLORA_OK:
        raise QloraError(rc, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libqlora takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous (row-major)")
    return t.data_ptr()


def _stream(stream=None) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ------------------------------------------------------------------ weights

@dataclass
class NF4Weight:
    """Device arrays of one NF4 weight [rows, cols] (see qlora_nf4_weight)."""
    rows: int
    cols: int
    double_quant: bool
    codes: torch.Tensor                 # uint8 [rows, cols/2]
    absmax_q8: torch.Tensor | None      # uint8 [blocks]
    group_scale: torch.Tensor | None    # fp32 [groups]
    absmax_f32: torch.Tensor | None     # fp32 [blocks]

    def c(self) -> NF4WeightC:
        return NF4WeightC(self.rows, self.cols, 64, 256, int(self.double_quant), 0,
                          _ptr(self.codes), _ptr(self.absmax_q8), _ptr(self.group_scale),
                          _ptr(self.absmax_f32))

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.absmax_q8, self.group_scale, self.absmax_f32) if t is not None)


def qlora_nf4_sizes(rows: int, cols: int, double_quant: bool = True) -> tuple[int, int, int]:
    c, a, g = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qlora_nf4_sizes(rows, cols, int(double_quant), ctypes.byref(c), ctypes.byref(a),
                                 ctypes.byref(g)), "qlora_nf4_sizes")
    return c.value, a.value, g.value


def qlora_nf4_codebook() -> list[float]:
    out = (ctypes.c_float * 16)()
    lib().qlora_nf4_codebook(out)
    return list(out)


def qlora_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes(M, N, K, r))


def empty_nf4(rows: int, cols: int, device, double_quant: bool = True,
              keep_absmax_f32: bool = False) -> NF4Weight:
    """Allocate (torch) the arrays of an NF4 weight."""
    c, a, g = qlora_nf4_sizes(rows, cols, double_quant)
    blocks = rows * cols // 64
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    if double_quant:
        q8 = torch.empty(a, dtype=torch.uint8, device=device)
        s2 = torch.empty(g // 4, dtype=torch.float32, device=device)
        af = torch.empty(blocks, dtype=torch.float32, device=device) if keep_absmax_f32 else None
    else:
        q8 = s2 = None
        af = torch.empty(blocks, dtype=torch.float32, device=device)
    return NF4Weight(rows, cols, double_quant, codes, q8, s2, af)


def qlora_quantize_nf4(W: torch.Tensor, out: NF4Weight | None = None, double_quant: bool = True,
                       d_status: torch.Tensor | None = None, stream=None) -> NF4Weight:
    if W.dim() != 2:
        raise ValueError("W must be 2-D [rows, cols]")
    if W.dtype == torch.float32:
        dt = QLORA_F32
    elif W.dtype == torch.bfloat16:
        dt = QLORA_BF16
    else:
        raise ValueError("W must be fp32 or bf16")
    if out is None:
        out = empty_nf4(W.shape[0], W.shape[1], W.device, double_quant)
    cw = out.c()
    _check(lib().qlora_quantize_nf4(_ptr(W), dt, ctypes.byref(cw), _ptr(d_status), _stream(stream)),
           "qlora_quantize_nf4")
    return out


def qlora_merge_nf4(Wq: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                    out: NF4Weight | None = None, W_merged: torch.Tensor | None = None,
                    double_quant: bool = True, d_status: torch.Tensor | None = None, stream=None,
                    keep_merged: bool = True):
    """NF4(W^ + (alpha/r) B A) into `out` (new, or Wq itself for in place);
    returns (out, W_merged) with W_merged the fp32 merged weight.  With
    keep_merged=False the merge is one fused pass (no fp32 buffer; not in
    place) and W_merged is None."""
    r = A.shape[0]
    dev = Wq.codes.device
    if out is None:
        out = empty_nf4(Wq.rows, Wq.cols, dev, double_quant)
    if not keep_merged:
        W_merged = None
    elif W_merged is None:
        W_merged = torch.empty((Wq.rows, Wq.cols), dtype=torch.float32, device=dev)
    cw, co = Wq.c(), out.c()
    _check(lib().qlora_merge_nf4(ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha), _ptr(W_merged),
                                 ctypes.byref(co), _ptr(d_status), _stream(stream)), "qlora_merge_nf4")
    return out, W_merged


def qlora_dequantize(Wq: NF4Weight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((Wq.rows, Wq.cols), dtype=torch.bfloat16, device=Wq.codes.device)
    cw = Wq.c()
    _check(lib().qlora_dequantize(ctypes.byref(cw), _ptr(out), _stream(stream)), "qlora_dequantize")
    return out


def qlora_linear_fwd(X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     Y: torch.Tensor | None = None, T_save: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, d_status: torch.Tensor | None = None,
                     gemm_events=None, stream=None) -> torch.Tensor:
    M = X.shape[0]
    r = A.shape[0]
    if Y is None:
        Y = torch.empty((M, Wq.rows), dtype=torch.bfloat16, device=X.device)
    need = qlora_workspace_bytes(M, Wq.rows, Wq.cols, r)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    cw = Wq.c()
    _check(lib().qlora_linear_fwd(_ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha),
                                  _ptr(Y), _ptr(T_save), _ptr(workspace), workspace.numel(),
                                  _ptr(d_status), _events(gemm_events), _stream(stream)),
           "qlora_linear_fwd")
    return Y


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor,
                     B: torch.Tensor, alpha: float, T_saved: torch.Tensor | None = None,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                     dB: torch.Tensor | None = None, grad_dtype=torch.float32, want_dX: bool = True,
                     workspace: torch.Tensor | None = None, d_status: torch.Tensor | None = None,
                     gemm_events=None, stream=None):
    M = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if want_dX and dX is None:
        dX = torch.empty((M, Wq.cols), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, Wq.cols), dtype=grad_dtype, device=dev)
    if dB is None:
        dB = torch.empty((Wq.rows, r), dtype=grad_dtype, device=dev)
    gdt = QLORA_F32 if dA.dtype == torch.float32 else QLORA_BF16
    need = qlora_workspace_bytes(M, Wq.rows, Wq.cols, r)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    cw = Wq.c()
    _check(lib().qlora_linear_bwd(_ptr(dY), _ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r,
                                  float(alpha), _ptr(T_saved), _ptr(dX) if want_dX else None,
                                  _ptr(dA), _ptr(dB), gdt, _ptr(workspace), workspace.numel(),
                                  _ptr(d_status), _events(gemm_events), _stream(stream)),
           "qlora_linear_bwd")
    return dX, dA, dB


def qlora_lora_linear_fwd(X: torch.Tensor, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                          Y: torch.Tensor | None = None, T_save: torch.Tensor | None = None,
                          workspace: torch.Tensor | None = None, d_status: torch.Tensor | None = None,
                          gemm_events=None, stream=None) -> torch.Tensor:
    """qlora_linear_fwd over a dense bf16 weight W [N, K] (plain LoRA)."""
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise ValueError("W must be a 2-D bf16 tensor")
    M, r = X.shape[0], A.shape[0]
    N, K = W.shape
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = torch.empty(max(qlora_workspace_bytes(M, N, K, r), 16), dtype=torch.uint8, device=X.device)
    _check(lib().qlora_lora_linear_fwd(_ptr(X), M, _ptr(W), N, K, _ptr(A), _ptr(B), r, float(alpha), _ptr(Y),
                                       _ptr(T_save), _ptr(workspace), workspace.numel(), _ptr(d_status),
                                       _events(gemm_events), _stream(stream)), "qlora_lora_linear_fwd")
    return Y


def qlora_lora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, W: torch.Tensor, A: torch.Tensor,
                          B: torch.Tensor, alpha: float, T_saved: torch.Tensor | None = None,
                          dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                          dB: torch.Tensor | None = None, grad_dtype=torch.float32, want_dX: bool = True,
                          workspace: torch.Tensor | None = None, d_status: torch.Tensor | None = None,
                          gemm_events=None, stream=None):
    """qlora_linear_bwd over a dense bf16 weight W [N, K] (plain LoRA)."""
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise ValueError("W must be a 2-D bf16 tensor")
    M, r = X.shape[0], A.shape[0]
    N, K = W.shape
    dev = X.device
    if want_dX and dX is None:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, K), dtype=grad_dtype, device=dev)
    if dB is None:
        dB = torch.empty((N, r), dtype=grad_dtype, device=dev)
    gdt = QLORA_F32 if dA.dtype == torch.float32 else QLORA_BF16
    if workspace is None:
        workspace = torch.empty(max(qlora_workspace_bytes(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    _check(lib().qlora_lora_linear_bwd(_ptr(dY), _ptr(X), M, _ptr(W), N, K, _ptr(A), _ptr(B), r, float(alpha),
                                       _ptr(T_saved), _ptr(dX) if want_dX else None, _ptr(dA), _ptr(dB), gdt,
                                       _ptr(workspace), workspace.numel(), _ptr(d_status), _events(gemm_events),
                                       _stream(stream)), "qlora_lora_linear_bwd")
    return dX, dA, dB


def qlora_adam_step(master: torch.Tensor, m: torch.Tensor, v: torch.Tensor, grad: torch.Tensor, step: int,
                    lr: float, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                    param: torch.Tensor | None = None, grad_scale: float = 1.0,
                    d_status: torch.Tensor | None = None, stream=None) -> None:
    """One Adam step in place over flat fp32 master/m/v (and an optional bf16
    copy `param`), with fp32 or bf16 gradients of the same length."""
    n = master.numel()
    for t in (m, v, grad) + ((param,) if param is not None else ()):
        if t.numel() != n:
            raise ValueError("master, m, v, grad (and param) must have the same number of elements")
    if master.dtype != torch.float32 or m.dtype != torch.float32 or v.dtype != torch.float32:
        raise ValueError("master, m and v are fp32")
    if param is not None and param.dtype != torch.bfloat16:
        raise ValueError("param is bf16")
    gdt = QLORA_F32 if grad.dtype == torch.float32 else QLORA_BF16
    _check(lib().qlora_adam_step(_ptr(master), _ptr(m), _ptr(v), _ptr(param), _ptr(grad), gdt, n, int(step),
                                 float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay),
                                 float(grad_scale), _ptr(d_status), _stream(stream)), "qlora_adam_step")


def qlora_linear_fwd_noalloc(X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                             alpha: float, Y: torch.Tensor | None = None,
                             T_save: torch.Tensor | None = None,
                             d_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The forward with the library's fixed device scratch instead of a
    workspace, for callers that cannot allocate device memory (see
    qlora.h).  Allocates Y only when the caller passes none."""
    M = X.shape[0]
    r = A.shape[0]
    if Y is None:
        Y = torch.empty((M, Wq.rows), dtype=torch.bfloat16, device=X.device)
    cw = Wq.c()
    _check(lib().qlora_linear_fwd_noalloc(_ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r,
                                          float(alpha), _ptr(Y), _ptr(T_save), _ptr(d_status),
                                          _stream(stream)), "qlora_linear_fwd_noalloc")
    return Y


# ------------------------------------------------------------- LoRA dropout

def qlora_workspace_bytes_dropout(M: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes_dropout(M, N, K, r))


def qlora_lora_dropout_mask(M: int, K: int, p: float, seed: int, device="cuda", stream=None) -> torch.Tensor:
    """The keep mask of a dropout call, uint8 [M, K] (1 = kept)."""
    keep = torch.empty((M, K), dtype=torch.uint8, device=device)
    _check(lib().qlora_lora_dropout_mask(M, K, float(p), int(seed), _ptr(keep), _stream(stream)),
           "qlora_lora_dropout_mask")
    return keep


def qlora_linear_fwd_dropout(X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                             p: float, seed: int, Y: torch.Tensor | None = None,
                             T_save: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                             d_status: torch.Tensor | None = None, gemm_events=None, stream=None) -> torch.Tensor:
    """qlora_linear_fwd with LoRA dropout (rate p, mask from seed) on the adapter input."""
    M, r = X.shape[0], A.shape[0]
    if Y is None:
        Y = torch.empty((M, Wq.rows), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = torch.empty(max(qlora_workspace_bytes_dropout(M, Wq.rows, Wq.cols, r), 16), dtype=torch.uint8,
                                device=X.device)
    cw = Wq.c()
    _check(lib().qlora_linear_fwd_dropout(_ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha),
                                          float(p), int(seed), _ptr(Y), _ptr(T_save), _ptr(workspace),
                                          workspace.numel(), _ptr(d_status), _events(gemm_events),
                                          _stream(stream)), "qlora_linear_fwd_dropout")
    return Y


def qlora_linear_bwd_dropout(dY: torch.Tensor, X: torch.Tensor, Wq: NF4Weight, A: torch.Tensor,
                             B: torch.Tensor, alpha: float, p: float, seed: int,
                             T_saved: torch.Tensor | None = None, dX: torch.Tensor | None = None,
                             dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                             grad_dtype=torch.float32, want_dX: bool = True,
                             workspace: torch.Tensor | None = None, d_status: torch.Tensor | None = None,
                             gemm_events=None, stream=None):
    """qlora_linear_bwd with the same LoRA dropout as the forward (same p and seed)."""
    M, r = X.shape[0], A.shape[0]
    dev = X.device
    if want_dX and dX is None:
        dX = torch.empty((M, Wq.cols), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, Wq.cols), dtype=grad_dtype, device=dev)
    if dB is None:
        dB = torch.empty((Wq.rows, r), dtype=grad_dtype, device=dev)
    gdt = QLORA_F32 if dA.dtype == torch.float32 else QLORA_BF16
    if workspace is None:
        workspace = torch.empty(max(qlora_workspace_bytes_dropout(M, Wq.rows, Wq.cols, r), 16), dtype=torch.uint8,
                                device=dev)
    cw = Wq.c()
    _check(lib().qlora_linear_bwd_dropout(_ptr(dY), _ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r,
                                          float(alpha), float(p), int(seed), _ptr(T_saved),
                                          _ptr(dX) if want_dX else None, _ptr(dA), _ptr(dB), gdt,
                                          _ptr(workspace), workspace.numel(), _ptr(d_status),
                                          _events(gemm_events), _stream(stream)), "qlora_linear_bwd_dropout")
    return dX, dA, dB


# ------------------------------------------------------ paged optimiser state

def qlora_paged_alloc(nbytes: int) -> int:
    """Managed (pageable) device memory for optimiser state; returns the pointer."""
    p = ctypes.c_void_p()
    _check(lib().qlora_paged_alloc(int(nbytes), ctypes.byref(p)), "qlora_paged_alloc")
    return int(p.value)


def qlora_paged_free(ptr: int) -> None:
    _check(lib().qlora_paged_free(ptr or None), "qlora_paged_free")


def qlora_paged_prefetch(ptr: int, nbytes: int, to_device: bool = True, stream=None) -> None:
    """Migrate [ptr, ptr + nbytes) to the current GPU, or page it out to the host."""
    _check(lib().qlora_paged_prefetch(ptr, int(nbytes), 1 if to_device else 0, _stream(stream)),
           "qlora_paged_prefetch")
