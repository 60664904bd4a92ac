"""GPU parity of the decode-shaped forward (M <= 16 tokens: the
weight-streaming kernel) against the binary64 CPU oracle on the same
dequantised weights.

The kernel splits the weight into 128-row x 64-column units and gives every
CTA an equal run of them, so a 128-row tile can be finished by one CTA or
summed from the partials of several; the shapes below cover both (and
tiles cut into many pieces, and a ragged last tile), ranks 1..256, the
format without double quantisation, and the two full 70B MLP matrices
(28672 x 8192 and 8192 x 28672 with 0.1% x10 outliers) at M = 1, 4, 16.

Bar: relative Frobenius error <= 2e-3 on Y (bf16 rounding of Y alone costs
~1.66e-3); T (fp32) <= 1e-4.
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


def _problem(M, N, K, r, seed, outliers=0.0):
    W = inputs.weight((N, K), 0.02, seed, outlier_frac=outliers)
    X = inputs.normal((M, K), 1.0, seed * 16 + 1)
    A = inputs.normal((r, K), 0.01, seed * 16 + 3)
    B = inputs.normal((N, r), 0.01, seed * 16 + 4)
    return W, X, A, B


def _oracle_Y(Wh, X, A, B, alpha):
    Y, T = O.linear_fwd(bits(X), Wh, bits(A), bits(B), alpha, A.shape[0])
    return Y, T


def _fwd(Wq, X, A, B, alpha):
    M, r = X.shape[0], A.shape[0]
    T = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Y = q.qlora_linear_fwd(X.to(DEV), Wq, A.to(DEV), B.to(DEV), alpha, T_save=T, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return Y, T


@pytest.mark.parametrize("M,N,K,r", [
    (1, 392, 704, 16),       # 4 tiles (last ragged), 11 units per tile: every tile summed from partials
    (4, 128, 64, 8),         # a single unit
    (16, 4096, 4096, 16),    # 32 tiles of 64 units over 148 CTAs: each tile in ~5 pieces
    (3, 1000, 2048, 5),      # odd rank, ragged tile, odd M
    (16, 256, 512, 256),     # maximum rank
    (7, 20480, 1024, 16),    # 160 tiles: most CTAs finish whole tiles
    (16, 8, 128, 1),         # fewer rows than one tile, rank 1
])
def test_decode_shapes(M, N, K, r):
    W, X, A, B = _problem(M, N, K, r, seed=M * 7 + N + K + r)
    alpha = 2.0 * r
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    Y, T = _fwd(Wq, X, A, B, alpha)
    Wh = O.nf4_dequantize(O.nf4_quantize(host_f32(W)))
    assert np.array_equal(bits(q.qlora_dequantize(Wq)), Wh)
    Yo, To = _oracle_Y(Wh, X, A, B, alpha)
    e = O.rel_fro(f64(Y), Yo)
    assert e <= TOL, f"Y: relative Frobenius error {e:.3e}"
    assert O.rel_fro(f64(T), To) <= 1e-4


def test_decode_without_double_quant():
    W, X, A, B = _problem(16, 640, 1536, 16, seed=31)
    Wq = q.qlora_quantize_nf4(W.to(DEV), double_quant=False)
    Y, _ = _fwd(Wq, X, A, B, 32.0)
    Wh = O.nf4_dequantize(O.nf4_quantize(host_f32(W), double_quant=False))
    Yo, _ = _oracle_Y(Wh, X, A, B, 32.0)
    assert O.rel_fro(f64(Y), Yo) <= TOL


def test_decode_is_deterministic_and_matches_wider_path():
    # same inputs twice: bit-identical (partials are summed in a fixed order);
    # and the same rows through the M = 17 path (the fused GEMM) agree to
    # within both paths' rounding.
    W, X, A, B = _problem(17, 4096, 4096, 16, seed=32)
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    Y1, _ = _fwd(Wq, X[:16], A, B, 32.0)
    Y2, _ = _fwd(Wq, X[:16], A, B, 32.0)
    assert torch.equal(Y1, Y2)
    Yg, _ = _fwd(Wq, X, A, B, 32.0)
    assert O.rel_fro(f64(Y1), f64(Yg[:16])) <= 3e-3


def test_decode_zero_weight_and_zero_adapter():
    W, X, A, B = _problem(4, 512, 1024, 16, seed=33)
    Wq = q.qlora_quantize_nf4(torch.zeros_like(W).to(DEV))
    Y, T = _fwd(Wq, X, A, B, 32.0)       # every code 7: the adapter term alone
    Yo, _ = _oracle_Y(np.zeros(W.shape, np.uint16), X, A, B, 32.0)
    assert O.rel_fro(f64(Y), Yo) <= TOL
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    Y, _ = _fwd(Wq, X, A, torch.zeros_like(B), 32.0)   # B = 0: the frozen base alone
    Yo, _ = _oracle_Y(O.nf4_dequantize(O.nf4_quantize(host_f32(W))), X, A, torch.zeros_like(B), 32.0)
    assert O.rel_fro(f64(Y), Yo) <= TOL


@pytest.mark.parametrize("proj", [0, 1])   # 28672 x 8192 and 8192 x 28672
def test_decode_70b_mlp_full(proj):
    wl = inputs.DECODE
    name, N, K = wl.shapes[proj]
    p = inputs.projection_inputs(wl, 0, proj, M=16, with_grad=False)
    W, X, A, B = p["W"], p["X"], p["A"], p["B"]
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    Wh = O.nf4_dequantize(O.nf4_quantize(host_f32(W)))
    del W
    Yo, To = _oracle_Y(Wh, X, A, B, wl.alpha)   # rows of a shorter X are the first rows of this
    for M in inputs.DECODE_M:
        Y, T = _fwd(Wq, X[:M], A, B, wl.alpha)
        e = O.rel_fro(f64(Y), Yo[:M])
        print(name, M, f"{e:.3e}")
        assert e <= TOL, f"{name} M={M}: relative Frobenius error {e:.3e}"
        assert O.rel_fro(f64(T), To[:M]) <= 1e-4
