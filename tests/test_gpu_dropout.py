"""GPU parity of LoRA dropout against the oracle.

"QLoRA" (infra.bea.ai), §3 "Implementation", sets lora_dropout = 0.05.  The
library's reading (inverted dropout on the adapter's input, one Philox
mask per call) is the oracle's: the keep mask must match bit for bit, and
T, Y, dX, dA, dB within the layer's tolerances of the binary64 oracle over
the same mask and the same dequantised weights.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import inputs
from gpu_util import bits, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


@pytest.mark.parametrize("M,K,p,seed", [(64, 512, 0.05, 7), (3, 1024, 0.5, 2 ** 40 + 3), (200, 576, 0.0, 1),
                                        (16, 64, 0.999, 5)])
def test_keep_mask_bit_exact(M, K, p, seed):
    got = q.qlora_lora_dropout_mask(M, K, p, seed).cpu().numpy().astype(bool)
    want = O.lora_dropout_keep(seed, M, K, p)
    assert np.array_equal(got, want)


def _nan(shape, dt):
    return torch.full(shape, float("nan"), dtype=dt, device=DEV)


@pytest.mark.parametrize("M,N,K,r,p", [
    (256, 512, 1024, 16, 0.05),   # the pages' rate, the fused 2-SM GEMM path
    (200, 264, 576, 8, 0.3),      # ragged tiles in every dimension, a higher rate
    (300, 64, 576, 8, 0.05),      # N = 64: the dX GEMM (adapter not folded) has a single stage
    (96, 136, 448, 5, 0.05),      # 16 < M <= 128: the 1-CTA GEMM; r not a multiple of 8
    (16, 1024, 2048, 16, 0.05),   # decode shape: T inside the weight-streaming kernel
    (1, 8192, 8192, 8, 0.2),      # a single token (8192 outputs in Y and in dX)
])
def test_dropout_layer_matches_oracle(M, N, K, r, p):
    seed = 1000 + M + N
    alpha = 2.0 * r
    W = inputs.weight((N, K), 0.02, seed, device=DEV)
    Wq = q.qlora_quantize_nf4(W)
    X = inputs.normal((M, K), 1.0, seed + 1, DEV)
    dY = inputs.normal((M, N), 1.0, seed + 2, DEV)
    A = inputs.normal((r, K), 0.01, seed + 3, DEV)
    B = inputs.normal((N, r), 0.01, seed + 4, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    T = _nan((M, r), torch.float32)
    Y = q.qlora_linear_fwd_dropout(X, Wq, A, B, alpha, p, seed, Y=_nan((M, N), torch.bfloat16), T_save=T,
                                   d_status=st)
    dX, dA, dB = q.qlora_linear_bwd_dropout(dY, X, Wq, A, B, alpha, p, seed, T_saved=T,
                                            dX=_nan((M, K), torch.bfloat16), dA=_nan((r, K), torch.float32),
                                            dB=_nan((N, r), torch.float32), d_status=st)
    # the backward again with T recomputed from the regenerated mask
    dX2, dA2, dB2 = q.qlora_linear_bwd_dropout(dY, X, Wq, A, B, alpha, p, seed, d_status=st)
    Wh = q.qlora_dequantize(Wq)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = O.nf4_quantize(W.float().cpu().numpy())
    Wh_ref = O.nf4_dequantize(ref)
    assert np.array_equal(bits(Wh), Wh_ref)
    keep = O.lora_dropout_keep(seed, M, K, p)
    Yo, To = O.linear_fwd_dropout(bits(X), Wh_ref, bits(A), bits(B), alpha, r, keep, p)
    g = O.linear_bwd_dropout(bits(dY), bits(X), Wh_ref, bits(A), bits(B), alpha, r, keep, p)
    for name, got, want, bar in (("T", T, To, 1e-4), ("Y", Y, Yo, TOL), ("dX", dX, g["dX"], TOL),
                                 ("dA", dA, g["dA"], 1e-4), ("dB", dB, g["dB"], 1e-4),
                                 ("dX (T recomputed)", dX2, g["dX"], TOL), ("dA (T recomputed)", dA2, g["dA"], 1e-4),
                                 ("dB (T recomputed)", dB2, g["dB"], 1e-4)):
        v = f64(got)
        assert np.isfinite(v).all(), f"{name}: unwritten elements"
        e = O.rel_fro(v, want)
        assert e <= bar, f"{name}: relative Frobenius error {e:.3e} > {bar:.0e}"


def test_zero_rate_is_the_plain_layer():
    # p = 0 keeps every element: the dropout entries compute the plain layer
    # (the same kernels except the extra mask pass and, for dX, the fp32
    # GEMM output plus one rounding pass: equal up to that rounding)
    M, N, K, r = 256, 512, 1024, 16
    W = inputs.weight((N, K), 0.02, 31, device=DEV)
    Wq = q.qlora_quantize_nf4(W)
    X = inputs.normal((M, K), 1.0, 32, DEV)
    dY = inputs.normal((M, N), 1.0, 33, DEV)
    A = inputs.normal((r, K), 0.01, 34, DEV)
    B = inputs.normal((N, r), 0.01, 35, DEV)
    T0 = torch.empty((M, r), dtype=torch.float32, device=DEV)
    T1 = torch.empty((M, r), dtype=torch.float32, device=DEV)
    Y0 = q.qlora_linear_fwd(X, Wq, A, B, 32.0, T_save=T0)
    Y1 = q.qlora_linear_fwd_dropout(X, Wq, A, B, 32.0, 0.0, 9, T_save=T1)
    g0 = q.qlora_linear_bwd(dY, X, Wq, A, B, 32.0, T_saved=T0)
    g1 = q.qlora_linear_bwd_dropout(dY, X, Wq, A, B, 32.0, 0.0, 9, T_saved=T1)
    torch.cuda.synchronize()
    assert torch.equal(T0, T1) and torch.equal(Y0, Y1)
    assert torch.equal(g0[1], g1[1]) and torch.equal(g0[2], g1[2])
    assert O.rel_fro(f64(g1[0]), f64(g0[0])) <= 0.25 * TOL


def test_invalid_rate_rejected():
    W = inputs.weight((64, 64), 0.02, 3, device=DEV)
    Wq = q.qlora_quantize_nf4(W)
    X = torch.zeros((32, 64), dtype=torch.bfloat16, device=DEV)
    A = torch.zeros((8, 64), dtype=torch.bfloat16, device=DEV)
    B = torch.zeros((64, 8), dtype=torch.bfloat16, device=DEV)
    for p in (-0.1, 1.0, float("nan")):
        with pytest.raises(q.QloraError):
            q.qlora_linear_fwd_dropout(X, Wq, A, B, 16.0, p, 1)
