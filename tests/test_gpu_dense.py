"""GPU parity of the dense-bf16 LoRA entries (plain LoRA on a 16-bit base,
the baseline the QLoRA pages compare against) against the binary64 CPU
oracle on the same bf16 weight, and against the NF4 path itself: over the
dequantised copy of an NF4 weight the dense GEMM sees the very bf16 tiles
that the NF4 GEMM builds in shared memory, in the same order, so forward
and dX must agree bit for bit (M > 128, where both take the 2-SM GEMM).

Bar: relative Frobenius error <= 2e-3 for Y, dX (bf16 outputs carry ~1.66e-3
of rounding alone); 1e-4 for fp32 T, dA, dB.
"""
from __future__ import annotations

import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import inputs
from gpu_util import bits, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def _problem(M, N, K, r, seed):
    W = inputs.weight((N, K), 0.02, seed, dtype=torch.bfloat16)
    X = inputs.normal((M, K), 1.0, seed * 16 + 1)
    dY = inputs.normal((M, N), 1.0, seed * 16 + 2)
    A = inputs.normal((r, K), 0.01, seed * 16 + 3)
    B = inputs.normal((N, r), 0.01, seed * 16 + 4)
    return W, X, dY, A, B


def _dense(W, X, dY, A, B, alpha, grad_dtype=torch.float32):
    M, r = X.shape[0], A.shape[0]
    Wd, Xd, dYd, Ad, Bd = (t.to(DEV) for t in (W, X, dY, A, B))
    T = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Y = q.qlora_lora_linear_fwd(Xd, Wd, Ad, Bd, alpha, T_save=T, d_status=st)
    dX, dA, dB = q.qlora_lora_linear_bwd(dYd, Xd, Wd, Ad, Bd, alpha, T_saved=T, grad_dtype=grad_dtype, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return dict(Y=Y, T=T, dX=dX, dA=dA, dB=dB)


@pytest.mark.parametrize("M,N,K,r", [
    (200, 264, 576, 8),      # ragged in every dimension
    (1, 256, 512, 16),       # a single token (the 2-SM GEMM with one real row)
    (16, 512, 1024, 16),     # decode-sized M
    (129, 392, 704, 5),      # r not a multiple of 8 (padded adapter B)
    (300, 1024, 2048, 64),   # several tiles, r = 64
    (2048, 4096, 4096, 16),  # LLaMA-7B q projection, full token count
])
def test_dense_matches_oracle(M, N, K, r):
    W, X, dY, A, B = _problem(M, N, K, r, seed=M + N + K + r)
    alpha = 2.0 * r
    got = _dense(W, X, dY, A, B, alpha)
    Wb = bits(W)
    Yo, To = O.linear_fwd(bits(X), Wb, bits(A), bits(B), alpha, r)
    g = O.linear_bwd(bits(dY), bits(X), Wb, bits(A), bits(B), alpha, r)
    errs = {"Y": O.rel_fro(f64(got["Y"]), Yo), "dX": O.rel_fro(f64(got["dX"]), g["dX"]),
            "T": O.rel_fro(f64(got["T"]), To), "dA": O.rel_fro(f64(got["dA"]), g["dA"]),
            "dB": O.rel_fro(f64(got["dB"]), g["dB"])}
    for k, e in errs.items():
        bar = TOL if k in ("Y", "dX") else 1e-4
        assert e <= bar, f"{k}: relative Frobenius error {e:.3e} > {bar:.1e} (all: {errs})"


@pytest.mark.parametrize("M,N,K,r", [(256, 512, 1024, 16), (300, 264, 576, 5), (2048, 11008, 4096, 16)])
def test_dense_over_dequantised_weight_equals_nf4_path(M, N, K, r):
    W, X, dY, A, B = _problem(M, N, K, r, seed=7 * M + N + K + r)
    alpha = 2.0 * r
    Xd, dYd, Ad, Bd = (t.to(DEV) for t in (X, dY, A, B))
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    Wh = q.qlora_dequantize(Wq)
    T = torch.empty((M, r), dtype=torch.float32, device=DEV)
    Yq = q.qlora_linear_fwd(Xd, Wq, Ad, Bd, alpha, T_save=T)
    dXq, _, _ = q.qlora_linear_bwd(dYd, Xd, Wq, Ad, Bd, alpha, T_saved=T)
    Yd = q.qlora_lora_linear_fwd(Xd, Wh, Ad, Bd, alpha)
    dXd, _, _ = q.qlora_lora_linear_bwd(dYd, Xd, Wh, Ad, Bd, alpha, T_saved=T)
    torch.cuda.synchronize()
    assert torch.equal(Yq, Yd), "forward: dense GEMM over the dequantised weight differs from the NF4 GEMM"
    assert torch.equal(dXq, dXd), "dX: dense GEMM over the dequantised weight differs from the NF4 GEMM"


def test_dense_bf16_gradients_and_determinism():
    W, X, dY, A, B = _problem(384, 768, 1536, 16, seed=41)
    a = _dense(W, X, dY, A, B, 32.0, grad_dtype=torch.bfloat16)
    b = _dense(W, X, dY, A, B, 32.0, grad_dtype=torch.bfloat16)
    for k in ("Y", "T", "dX", "dA", "dB"):
        assert torch.equal(a[k], b[k]), f"{k} differs between two identical calls"
    g = O.linear_bwd(bits(dY), bits(X), bits(W), bits(A), bits(B), 32.0, 16)
    assert O.rel_fro(f64(a["dA"]), g["dA"]) <= TOL
    assert O.rel_fro(f64(a["dB"]), g["dB"]) <= TOL
