"""GPU parity of the fused QLoRA linear layer (forward, dX, dA, dB) against the
binary64 CPU oracle on the same dequantised weights.

Bar: relative Frobenius error <= 2e-3 for Y, dX, dA, dB (bf16 outputs carry
~1.66e-3 of rounding alone); fp32 T and fp32 dA/dB are held to tighter bars.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import inputs
from gpu_util import bits, f64, host_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def _problem(M, N, K, r, seed, w_std=0.02, dtype=torch.bfloat16, ab_std=0.01):
    W = inputs.weight((N, K), w_std, seed, dtype=dtype)
    X = inputs.normal((M, K), 1.0, seed * 16 + 1)
    dY = inputs.normal((M, N), 1.0, seed * 16 + 2)
    A = inputs.normal((r, K), ab_std, seed * 16 + 3)
    B = inputs.normal((N, r), ab_std, seed * 16 + 4)
    return W, X, dY, A, B


def _run(W, X, dY, A, B, alpha, grad_dtype=torch.float32, save_T=True, want_dX=True):
    M, r = X.shape[0], A.shape[0]
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    Xd, dYd, Ad, Bd = (t.to(DEV) for t in (X, dY, A, B))
    N, K = W.shape
    nan = lambda shape, dt: torch.full(shape, float("nan"), dtype=dt, device=DEV)
    # every output starts as NaN: an element a kernel fails to write shows up
    T = nan((M, r), torch.float32) if save_T else None
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Y = q.qlora_linear_fwd(Xd, Wq, Ad, Bd, alpha, Y=nan((M, N), torch.bfloat16), T_save=T, d_status=st)
    dX, dA, dB = q.qlora_linear_bwd(dYd, Xd, Wq, Ad, Bd, alpha, T_saved=T, grad_dtype=grad_dtype,
                                    dX=nan((M, K), torch.bfloat16) if want_dX else None,
                                    dA=nan((r, K), grad_dtype), dB=nan((N, r), grad_dtype),
                                    want_dX=want_dX, d_status=st)
    Wh = q.qlora_dequantize(Wq)
    torch.cuda.synchronize()
    assert st.item() == 0
    return dict(Y=Y, T=T, dX=dX, dA=dA, dB=dB, Wh=Wh)


def _oracle(W, X, dY, A, B, alpha):
    r = A.shape[0]
    ref = O.nf4_quantize(host_f32(W))
    Wh = O.nf4_dequantize(ref)
    Y, T = O.linear_fwd(bits(X), Wh, bits(A), bits(B), alpha, r)
    g = O.linear_bwd(bits(dY), bits(X), Wh, bits(A), bits(B), alpha, r)
    return dict(Y=Y, T=T, dX=g["dX"], dA=g["dA"], dB=g["dB"], Wh=Wh)


def _compare(got, want, grad_tol=TOL, check_dX=True):
    assert np.array_equal(bits(got["Wh"]), want["Wh"]), "in-library dequant differs from the oracle"
    errs = {}
    for k in ("Y", "dX", "dA", "dB") + (("T",) if got["T"] is not None else ()):
        if k == "dX" and not check_dX:
            continue
        g = f64(got[k])
        assert np.isfinite(g).all(), f"{k}: {int((~np.isfinite(g)).sum())} elements not written"
        errs[k] = O.rel_fro(g, want[k])
    for k, e in errs.items():
        bar = {"T": 1e-4, "dA": grad_tol, "dB": grad_tol}.get(k, TOL)
        assert e <= bar, f"{k}: relative Frobenius error {e:.3e} > {bar:.1e} (all: {errs})"
    return errs


def test_single_layer_config():
    p = inputs.projection_inputs(inputs.SINGLE, 0, 0)
    args = (p["W"], p["X"], p["dY"], p["A"], p["B"])
    _compare(_run(*args, p["alpha"]), _oracle(*args, p["alpha"]), grad_tol=1e-4)


@pytest.mark.parametrize("M,N,K,r", [
    (200, 264, 576, 8),      # ragged in every dimension (M, N tiles; K not a multiple of 256)
    (1, 256, 512, 16),       # a single token
    (16, 512, 1024, 16),     # decode-sized M
    (129, 392, 704, 5),      # r not a multiple of 8 (padded adapter B)
    (64, 136, 448, 64),
    (130, 256, 320, 130),    # rank above 128: the gradient pass takes two column chunks
    (96, 8, 128, 256),       # narrow weight, maximum rank
])
def test_ragged_and_edge_shapes(M, N, K, r):
    args = _problem(M, N, K, r, seed=M + N + K + r)
    alpha = 2.0 * r
    _compare(_run(*args, alpha), _oracle(*args, alpha), grad_tol=1e-4)


@pytest.mark.parametrize("mtiles", [1, 2])
@pytest.mark.parametrize("M,N,K,r", [
    (600, 264, 576, 8),      # two 512-row tiles, the second ragged; N, K ragged
    (1100, 512, 1024, 16),   # three 512-row tiles, the last with 76 rows
    (300, 320, 64, 5),       # one 64-deep weight stage; r not a multiple of 8
    (520, 136, 448, 64),     # 8 rows in the second 512-row tile
])
def test_pair_one_and_two_m_tiles(mtiles, M, N, K, r):
    # the 2-SM GEMM (M > 128) with one 256-row or two 256-row M tiles per
    # pair, forced for forward and dX alike
    L = q.lib()
    assert L.qlora_debug_set_pair_mtiles(mtiles) == 0
    try:
        args = _problem(M, N, K, r, seed=3 * M + N + K + r + mtiles)
        alpha = 2.0 * r
        _compare(_run(*args, alpha), _oracle(*args, alpha), grad_tol=1e-4)
    finally:
        assert L.qlora_debug_set_pair_mtiles(0) == 0


def test_pair_m_tiles_hook_rejects_bad_values():
    L = q.lib()
    assert L.qlora_debug_set_pair_mtiles(3) != 0
    assert L.qlora_debug_set_pair_mtiles(-1) != 0
    assert L.qlora_debug_set_pair_mtiles(0) == 0


@pytest.mark.parametrize("proj", [0, 4, 6])   # q 4096x4096, gate 11008x4096, down 4096x11008
def test_llama7b_projection_full(proj):
    wl = inputs.LLAMA7B
    p = inputs.projection_inputs(wl, 0, proj)
    args = (p["W"], p["X"], p["dY"], p["A"], p["B"])
    errs = _compare(_run(*args, p["alpha"]), _oracle(*args, p["alpha"]), grad_tol=1e-4)
    print(p["name"], errs)


def test_bf16_gradients_and_recomputed_T():
    args = _problem(256, 512, 1024, 16, seed=21)
    got = _run(*args, 32.0, grad_dtype=torch.bfloat16, save_T=False)
    _compare(got, _oracle(*args, 32.0), grad_tol=TOL)
    assert got["dA"].dtype == torch.bfloat16


def test_no_dX_requested():
    args = _problem(128, 256, 512, 8, seed=22)
    got = _run(*args, 16.0, want_dX=False)
    _compare(got, _oracle(*args, 16.0), grad_tol=1e-4, check_dX=False)


def test_special_cases():
    W, X, dY, A, B = _problem(128, 256, 512, 16, seed=23)
    # B = 0: the frozen-base GEMM alone
    Bz = torch.zeros_like(B)
    _compare(_run(W, X, dY, A, Bz, 32.0), _oracle(W, X, dY, A, Bz, 32.0), grad_tol=1e-4)
    # alpha = 0: no adapter contribution, zero adapter gradients
    got = _run(W, X, dY, A, B, 0.0)
    want = _oracle(W, X, dY, A, B, 0.0)
    assert O.rel_fro(f64(got["Y"]), want["Y"]) <= TOL
    assert float(got["dA"].abs().max()) == 0.0 and float(got["dB"].abs().max()) == 0.0
    # an all-zero weight (every code 7): only the adapter path remains
    Wz = torch.zeros_like(W)
    _compare(_run(Wz, X, dY, A, B, 32.0), _oracle(Wz, X, dY, A, B, 32.0), grad_tol=1e-4)


def test_llama65b_shape_row_slice():
    # 65B gate shape (22016 x 8192, r = 64): the full weight on the GPU, the
    # oracle on a 512-row slice of the tokens.
    wl = inputs.LLAMA65B
    name, N, K = wl.shapes[4]
    Wd = inputs.weight((N, K), wl.w_std, 5004, device=DEV)
    M = 512
    X = inputs.normal((M, K), 1.0, 11)
    dY = inputs.normal((M, N), 1.0, 12)
    A = inputs.normal((wl.r, K), 0.01, 13)
    B = inputs.normal((N, wl.r), 0.01, 14)
    got = _run(Wd, X, dY, A, B, wl.alpha)
    want = _oracle(Wd.cpu(), X, dY, A, B, wl.alpha)
    _compare(got, want, grad_tol=1e-4)
