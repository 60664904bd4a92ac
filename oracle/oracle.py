"""Python face of the CPU oracle -- TEST INFRASTRUCTURE ONLY.

The storage format (quantise, double-quantise, pack, dequantise) runs in the
plain C of ``qlora_oracle.c`` through ctypes.  The linear layer is written
here with numpy in binary64: each product is one ``numpy.matmul`` of the
bf16 operands upcast exactly to binary64, with no blocking, fusion or
reordering beyond the definitions.

Forward ("QLoRA", learning-llms.pages.dev/topics/qlora, the forward equation
h = W^x + (alpha/r) B(Ax) with W^ = dequant(W_4bit)), written for row-major
activations X [M, K], W [N, K], A [r, K], B [N, r] and s = alpha / r:

    T  = X A^T                       [M, r]
    Y  = X W^T + s T B^T             [M, N]

Backward ("QLoRA", infra.bea.ai, section "The Backward Pass Through
Quantization": the gradient passes through the dequantised frozen base;
only the adapters get gradients; the NF4 base is never updated):

    G  = dY B                        [M, r]
    dX = dY W^ + s G A               [M, K]
    dA = s G^T X                     [r, K]
    dB = s dY^T T                    [N, r]

T and G stay unrounded (binary64).  There is no bias: the pages show none.

Adapter optimiser ("QLoRA", infra.bea.ai, "How QLoRA Works", precision
table: Adam state in fp32, 12 bytes per adapter parameter -- a master copy
and two moments).  The pages print no update rule; ``adam_step`` is Adam as
published (Kingma & Ba, moment averages with bias correction) with optional
decoupled weight decay (Loshchilov & Hutter), in binary64.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

__all__ = [
    "BLOCK", "GROUP", "load", "build_oracle", "nf4_levels", "f32_to_bf16",
    "bf16_to_f32", "absmax_int_quantize", "nf4_nearest", "nf4_sizes",
    "nf4_quantize", "nf4_dequantize", "linear_fwd", "linear_bwd",
    "adam_step", "merge_nf4", "e4m3_values", "e4m3_encode", "nf4_quantize_fp8", "nf4_dequantize_fp8",
    "philox4x64_10", "philox4x64_10_blocks", "dropout_threshold",
    "lora_dropout_keep", "linear_fwd_dropout", "linear_bwd_dropout", "rel_fro", "OracleError",
]

BLOCK = 64
GROUP = 256

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlora_oracle.c")
_INC = os.path.join(_HERE, "nf4_levels.inc")
_LIB = os.path.join(_HERE, "libqlora_oracle.so")
_lock = threading.Lock()
_lib = None


class OracleError(RuntimeError):
    pass


def build_oracle(force: bool = False) -> str:
    """Compile the plain-C oracle with gcc (no fast-math, no contraction)."""
    stale = (not os.path.exists(_LIB)
             or os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_INC)))
    if force or stale:
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def load():
    global _lib
    with _lock:
        if _lib is None:
            build_oracle()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_nf4_levels.argtypes = [P]
            lib.oracle_f32_to_bf16.argtypes = [P, I64, P]
            lib.oracle_bf16_to_f32.argtypes = [P, I64, P]
            lib.oracle_absmax_int_quantize.argtypes = [P, I64, ctypes.c_int, P, P]
            lib.oracle_absmax_int_quantize.restype = ctypes.c_float
            lib.oracle_nf4_nearest.argtypes = [ctypes.c_float]
            lib.oracle_nf4_nearest.restype = ctypes.c_int
            lib.oracle_nf4_sizes.argtypes = [I64, I64, ctypes.c_int, P, P, P]
            lib.oracle_nf4_quantize.argtypes = [P, I64, I64, ctypes.c_int, P, P, P, P]
            lib.oracle_nf4_dequantize.argtypes = [P, P, P, P, I64, I64, ctypes.c_int, P]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ------------------------------------------------------------------ scalars

def nf4_levels() -> np.ndarray:
    out = np.zeros(16, np.float32)
    load().oracle_nf4_levels(_ptr(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """binary32 -> bf16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    load().oracle_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    load().oracle_bf16_to_f32(_ptr(h), h.size, _ptr(out))
    return out


def absmax_int_quantize(w: np.ndarray, bits: int = 4):
    """Symmetric absmax grid of the learning-llms page: returns (q, scale, w_hat)."""
    w = np.ascontiguousarray(w, np.float32).ravel()
    q = np.empty(w.size, np.int32)
    w_hat = np.empty(w.size, np.float32)
    scale = load().oracle_absmax_int_quantize(_ptr(w), w.size, bits, _ptr(q), _ptr(w_hat))
    return q, np.float32(scale), w_hat


def nf4_nearest(x: float) -> int:
    return int(load().oracle_nf4_nearest(float(x)))


def nf4_sizes(rows: int, cols: int, double_quant: bool = True):
    c, a, g = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    rc = load().oracle_nf4_sizes(rows, cols, int(double_quant), ctypes.byref(c),
                                 ctypes.byref(a), ctypes.byref(g))
    if rc != 0:
        raise OracleError(f"invalid shape {rows}x{cols}")
    return c.value, a.value, g.value


# ------------------------------------------------------------------ format

def nf4_quantize(w: np.ndarray, double_quant: bool = True) -> dict:
    """Encode a [rows, cols] matrix (binary32 values; pass bf16 inputs as their
    exact binary32 upcast).  Returns codes [rows, cols/2] uint8, absmax [blocks]
    fp32, and with double quantisation q8 [blocks] uint8 and s2 [groups] fp32."""
    w = np.ascontiguousarray(w, np.float32)
    rows, cols = w.shape
    blocks = rows * cols // BLOCK
    groups = (blocks + GROUP - 1) // GROUP
    codes = np.zeros((rows, cols // 2), np.uint8)
    absmax = np.zeros(blocks, np.float32)
    q8 = np.zeros(blocks, np.uint8) if double_quant else None
    s2 = np.zeros(groups, np.float32) if double_quant else None
    rc = load().oracle_nf4_quantize(_ptr(w), rows, cols, int(double_quant), _ptr(codes),
                                    _ptr(absmax), _ptr(q8), _ptr(s2))
    if rc == 1:
        raise OracleError("invalid shape")
    if rc == 2:
        raise OracleError("non-finite input")
    out = {"codes": codes, "absmax": absmax, "rows": rows, "cols": cols,
           "double_quant": bool(double_quant)}
    if double_quant:
        out["q8"] = q8
        out["s2"] = s2
    return out


def nf4_dequantize(q: dict) -> np.ndarray:
    """Decode to bf16 bit patterns [rows, cols] (uint16)."""
    rows, cols = q["rows"], q["cols"]
    out = np.empty((rows, cols), np.uint16)
    dq = q["double_quant"]
    rc = load().oracle_nf4_dequantize(
        _ptr(np.ascontiguousarray(q["codes"])), _ptr(q.get("q8")) if dq else None,
        _ptr(q.get("s2")) if dq else None, None if dq else _ptr(q["absmax"]),
        rows, cols, int(dq), _ptr(out))
    if rc != 0:
        raise OracleError("invalid shape")
    return out


# ------------------------------------------------------------- linear layer

def _f64(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) or floats -> binary64 (exact)."""
    if a.dtype == np.uint16:
        return bf16_to_f32(a).astype(np.float64)
    return np.asarray(a, np.float64)


def linear_fwd(X, W_hat, A, B, alpha: float, r: int):
    """Returns (Y, T) in binary64.  All operands as bf16 bit patterns or floats."""
    X, W, A, B = _f64(X), _f64(W_hat), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    T = X @ A.T
    Y = X @ W.T + s * (T @ B.T)
    return Y, T


def linear_bwd(dY, X, W_hat, A, B, alpha: float, r: int, T=None):
    """Returns dict(dX, dA, dB, G) in binary64.  T is recomputed as X A^T when
    not given.  W_hat = None skips dX (returned as None): dA and dB need only
    the rank-r products, so they can be checked over many more tokens than
    the M x N x K product allows."""
    dY, X, A, B = _f64(dY), _f64(X), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    if T is None:
        T = X @ A.T
    else:
        T = np.asarray(T, np.float64)
    G = dY @ B
    dX = None if W_hat is None else dY @ _f64(W_hat) + s * (G @ A)
    dA = s * (G.T @ X)
    dB = s * (dY.T @ T)
    return {"dX": dX, "dA": dA, "dB": dB, "G": G, "T": T}


def merge_nf4(q: dict, A, B, alpha: float, r: int, W_hat=None) -> np.ndarray:
    """The merged weight W^ + s B A as fp32 [N, K], before re-quantisation
    ("QLoRA", learning-llms page, the fine-print bullet on merging: adding
    the bf16 update into 4-bit weights forces a re-quantisation).  The pages
    fix no precision for it; the merged values decide integer codes, so this
    takes the library's precision and order: fp32, every operation rounded
    once, acc = sum over j of B[:, j] * A[j, :] in j order, then W^ + s acc
    with s = fp32(alpha) / fp32(r).  numpy float32 arithmetic rounds each
    operation (no fused multiply-add).  W_hat: the dequantised weight as
    bf16 bits, for a source in another scale format (default: decoded from
    q with nf4_dequantize)."""
    W = bf16_to_f32(nf4_dequantize(q) if W_hat is None else np.asarray(W_hat, np.uint16)).astype(np.float32)
    a = bf16_to_f32(np.asarray(A, np.uint16)).astype(np.float32)
    b = bf16_to_f32(np.asarray(B, np.uint16)).astype(np.float32)
    s = np.float32(alpha) / np.float32(r)
    acc = np.zeros(W.shape, np.float32)
    for j in range(r):
        acc = acc + b[:, j:j + 1] * a[j:j + 1, :]
    return W + s * acc


# ------------------------------------------------ FP8 second-level scales
# "QLoRA" (infra.bea.ai), §1 "Double Quantization": the fp32 block scales are
# themselves quantised "to FP8" (0.125 bits per weight).  Reading: FP8 E4M3
# (bias 7, 3 mantissa bits, largest finite 448, code 0x7F is NaN), one fp32
# scale per group of 256 blocks s2 = fp32(m / 448) with m the group's
# largest absmax, q = E4M3 round-to-nearest-even, saturating at 448, of
# fp32(absmax / s2); m < FLT_MIN gives s2 = 0 and q = 0.  The NF4 codes come
# from the fp32 absmax as in the 8-bit format; dequantisation uses
# absmax' = fp32(E4M3(q) * s2).  (The QLoRA paper also subtracts the group
# mean first; the pages do not, so neither does this reading.)

def e4m3_values() -> np.ndarray:
    """The 127 non-negative finite E4M3 values, by code 0..126."""
    v = []
    for code in range(127):
        e, m = code >> 3, code & 7
        v.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(v, np.float64)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes of non-negative values: nearest value, ties to the even
    code, values above 448 saturate to 448 (code 126).  Brute force over the
    codebook (the codes are sorted by value)."""
    vals = e4m3_values()
    x = np.asarray(x, np.float64).reshape(-1)
    if np.any(~np.isfinite(x)) or np.any(x < 0):
        raise ValueError("e4m3_encode takes finite non-negative values")
    d = np.abs(x[:, None] - vals[None, :])
    best = d.min(axis=1, keepdims=True)
    ties = d == best
    codes = np.arange(127)
    # among the nearest, the even code (two values can tie; their codes are adjacent)
    pick = np.where(ties & (codes[None, :] % 2 == 0), codes[None, :], 1000).min(axis=1)
    pick = np.where(pick == 1000, np.argmax(ties, axis=1), pick)
    return np.minimum(pick, 126).astype(np.uint8)


def nf4_quantize_fp8(w: np.ndarray) -> dict:
    """NF4 codes with FP8 (E4M3) second-level scales: codes and fp32 absmax
    from the C quantiser, then the group scales and E4M3 codes as above."""
    base = nf4_quantize(w, double_quant=False)
    a = base["absmax"].astype(np.float32)
    n = a.size
    groups = (n + GROUP - 1) // GROUP
    s2 = np.zeros(groups, np.float32)
    q = np.zeros(n, np.uint8)
    for g in range(groups):
        blk = a[g * GROUP:(g + 1) * GROUP]
        m = np.float32(blk.max())
        if not m >= np.float32(np.finfo(np.float32).tiny):
            continue
        s2[g] = np.float32(m) / np.float32(448.0)
        q[g * GROUP:(g + 1) * GROUP] = e4m3_encode(blk / s2[g])
    return {"codes": base["codes"], "absmax": base["absmax"], "q8": q, "s2": s2,
            "rows": base["rows"], "cols": base["cols"], "fp8": True}


def nf4_dequantize_fp8(q: dict) -> np.ndarray:
    """bf16 bits of the dequantised weight under FP8 scales: absmax' =
    fp32(E4M3(q) * s2) per block, then bf16(level * absmax') as for the
    fp32-absmax format."""
    vals = e4m3_values().astype(np.float32)
    s2 = np.repeat(q["s2"], GROUP)[:q["q8"].size]
    absmax = (vals[q["q8"]] * s2).astype(np.float32)
    return nf4_dequantize({"codes": q["codes"], "absmax": absmax, "rows": q["rows"], "cols": q["cols"],
                           "double_quant": False})


# ---------------------------------------------------------------- LoRA dropout
# The infra.bea.ai "QLoRA" page, §3 "Implementation", configures the
# adapters with lora_dropout = 0.05 (a PEFT LoraConfig) without defining it.
# Reading: inverted dropout on the adapter's input X -- each element kept
# with probability 1 - p, kept elements scaled by 1/(1 - p) -- with one mask
# per call drawn from a counter-based generator, so that a kernel can
# regenerate it anywhere.  Because X * keep is still exactly bf16, the
# 1/(1 - p) is applied to the fp32 products (T, dA, and dX's adapter term).
#
# Generator: Philox-4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
# numbers: as easy as 1, 2, 3", SC 2011): 10 rounds of two 64x64 -> 128-bit
# products on a 4-word counter with a 2-word key bumped by two Weyl
# constants after every round.

_PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)   # round multipliers
_PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)   # key increments (Weyl)
_U64 = (1 << 64) - 1


def philox4x64_10(counter, key):
    """One Philox-4x64-10 block: 4 words out of a 4-word counter and a 2-word
    key (Python integers, the definition written out)."""
    c0, c1, c2, c3 = (int(x) & _U64 for x in counter)
    k0, k1 = (int(x) & _U64 for x in key)
    for _ in range(10):
        p0, p1 = _PHILOX_M[0] * c0, _PHILOX_M[1] * c2
        c0, c1, c2, c3 = ((p1 >> 64) ^ c1 ^ k0) & _U64, p1 & _U64, ((p0 >> 64) ^ c3 ^ k1) & _U64, p0 & _U64
        k0, k1 = (k0 + _PHILOX_W[0]) & _U64, (k1 + _PHILOX_W[1]) & _U64
    return c0, c1, c2, c3


def _mulhilo64(a: np.ndarray, b: int):
    """(high, low) 64-bit halves of a * b for uint64 arrays a, from 32-bit parts."""
    m32 = np.uint64(0xFFFFFFFF)
    a = a.astype(np.uint64)
    al, ah = a & m32, a >> np.uint64(32)
    bl, bh = np.uint64(b & 0xFFFFFFFF), np.uint64(b >> 32)
    p0, p1, p2, p3 = al * bl, al * bh, ah * bl, ah * bh
    mid = (p0 >> np.uint64(32)) + (p1 & m32) + (p2 & m32)
    hi = p3 + (p1 >> np.uint64(32)) + (p2 >> np.uint64(32)) + (mid >> np.uint64(32))
    lo = (mid << np.uint64(32)) | (p0 & m32)
    return hi, lo


def philox4x64_10_blocks(c0: np.ndarray, key):
    """Philox-4x64-10 of counters (c0[i], 0, 0, 0) under one key, vectorised
    over i; returns a [len(c0), 4] uint64 array.  Same rounds as the scalar
    definition above."""
    with np.errstate(over="ignore"):
        x0 = np.asarray(c0, np.uint64)
        x1 = np.zeros_like(x0); x2 = np.zeros_like(x0); x3 = np.zeros_like(x0)
        k0, k1 = int(key[0]) & _U64, int(key[1]) & _U64
        for _ in range(10):
            h0, l0 = _mulhilo64(x0, _PHILOX_M[0])
            h1, l1 = _mulhilo64(x2, _PHILOX_M[1])
            x0, x1, x2, x3 = h1 ^ x1 ^ np.uint64(k0), l1, h0 ^ x3 ^ np.uint64(k1), l0
            k0, k1 = (k0 + _PHILOX_W[0]) & _U64, (k1 + _PHILOX_W[1]) & _U64
    return np.stack([x0, x1, x2, x3], axis=1)


def dropout_threshold(p: float) -> int:
    """Integer cut: an element is dropped when the top 32 bits of its word are
    below ceil(p * 2^32) (exact: scaling by 2^32 is exact in binary64)."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout p must be in [0, 1)")
    return int(math.ceil(float(p) * 4294967296.0))


def lora_dropout_keep(seed: int, M: int, K: int, p: float) -> np.ndarray:
    """Keep mask [M, K] of one call: element e = m K + k takes word e % 4 of
    Philox-4x64-10 at counter (e // 4, 0, 0, 0), key (seed, 0), and is kept
    when that word's top 32 bits are >= dropout_threshold(p)."""
    n = M * K
    words = philox4x64_10_blocks(np.arange((n + 3) // 4, dtype=np.uint64), (seed, 0)).reshape(-1)[:n]
    return ((words >> np.uint64(32)) >= np.uint64(dropout_threshold(p))).reshape(M, K)


def linear_fwd_dropout(X, W_hat, A, B, alpha: float, r: int, keep: np.ndarray, p: float):
    """Forward with dropout on the adapter input, binary64: T = (X * keep) A^T
    / (1 - p); Y = X W^T + s T B^T (the frozen path sees X undropped)."""
    X, W, A, B = _f64(X), _f64(W_hat), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    T = ((X * keep) @ A.T) / (1.0 - float(p))
    Y = X @ W.T + s * (T @ B.T)
    return Y, T


def linear_bwd_dropout(dY, X, W_hat, A, B, alpha: float, r: int, keep: np.ndarray, p: float, T=None):
    """Backward of linear_fwd_dropout for the same mask, binary64: G = dY B;
    dX = dY W^ + s (G A) * keep / (1 - p); dA = s G^T (X * keep) / (1 - p);
    dB = s dY^T T."""
    dY, X, A, B = _f64(dY), _f64(X), _f64(A), _f64(B)
    s = float(alpha) / float(r)
    q = 1.0 - float(p)
    Xk = X * keep
    T = (Xk @ A.T) / q if T is None else np.asarray(T, np.float64)
    G = dY @ B
    dX = None if W_hat is None else dY @ _f64(W_hat) + s * ((G @ A) * keep) / q
    return {"dX": dX, "dA": s * (G.T @ Xk) / q, "dB": s * (dY.T @ T), "G": G}


def adam_step(theta, m, v, g, t: int, lr: float, beta1: float, beta2: float, eps: float,
              weight_decay: float = 0.0, grad_scale: float = 1.0):
    """One Adam step at step number t >= 1, in binary64; returns the new
    (theta, m, v).  Steps in the published order: the decoupled decay of the
    parameter, the two moment averages, their bias corrections, the update."""
    theta, m, v = (np.asarray(a, np.float64) for a in (theta, m, v))
    g = np.asarray(g, np.float64) * float(grad_scale)
    theta = theta * (1.0 - float(lr) * float(weight_decay))
    m = float(beta1) * m + (1.0 - float(beta1)) * g
    v = float(beta2) * v + (1.0 - float(beta2)) * g * g
    m_hat = m / (1.0 - float(beta1) ** t)
    v_hat = v / (1.0 - float(beta2) ** t)
    theta = theta - float(lr) * m_hat / (np.sqrt(v_hat) + float(eps))
    return theta, m, v


def rel_fro(got, ref) -> float:
    """Relative Frobenius error ||got - ref|| / ||ref|| in binary64."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)
