"""GPU parity of the FP8 (E4M3) second-level scale format against the oracle.

"QLoRA" (infra.bea.ai), §1 subsection "Double Quantization", quantises the
fp32 block scales to FP8.  Read as E4M3 codes with one fp32 scale per 256
blocks (max absmax / 448); the format is double_quant = 2 of the weight.
Codes, E4M3 codes and group scales must match the oracle bit for bit, the
dequantised weights too, and every GEMM path (2-SM pair, 1-CTA, decode)
must match the oracle's layer over those weights within tolerance.
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
FP8 = 2


def _check_codec(W: torch.Tensor):
    Wq = q.empty_nf4(W.shape[0], W.shape[1], DEV, FP8, keep_absmax_f32=True)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlora_quantize_nf4(W.to(DEV).contiguous(), out=Wq, d_status=st)
    Wh = q.qlora_dequantize(Wq)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = O.nf4_quantize_fp8(host_f32(W))
    assert np.array_equal(Wq.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(Wq.absmax_f32.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    assert np.array_equal(Wq.absmax_q8.cpu().numpy(), ref["q8"])
    assert np.array_equal(Wq.group_scale.cpu().numpy().view(np.uint32), ref["s2"].view(np.uint32))
    assert np.array_equal(bits(Wh), O.nf4_dequantize_fp8(ref))
    return Wq, ref


@pytest.mark.parametrize("rows,cols", [(256, 512), (7, 11008), (33, 320), (1, 64)])
def test_fp8_scales_codec_bit_exact(rows, cols):
    W = inputs.weight((rows, cols), 0.02, rows + cols, dtype=torch.float32, outlier_frac=1e-2, outlier_scale=10.0)
    _check_codec(W)


def test_fp8_scales_wide_absmax_range_and_zero_groups():
    # blocks whose absmax spans many binades inside one group exercise the
    # E4M3 subnormals and saturation; an all-zero group gives s2 = 0, q = 0
    W = inputs.weight((64, 1024), 1.0, 9, dtype=torch.float32)
    # inside every 256-block group the block scales fall from 2^0 to 2^-20,
    # beyond E4M3's normal range (2^-6 .. 448) relative to the group maximum
    b = torch.arange(64 * 16, dtype=torch.float64) % 256
    scale = (2.0 ** (-20.0 * b / 255.0)).reshape(64, 16).repeat_interleave(64, dim=1)
    W = (W.double() * scale).float()
    W[:16] = 0.0
    _check_codec(W)


@pytest.mark.parametrize("M,N,K,r", [(256, 512, 1024, 16), (96, 136, 448, 5), (16, 1024, 2048, 16),
                                     (1, 8192, 8192, 8)])
def test_fp8_scales_layer_matches_oracle(M, N, K, r):
    seed = 500 + M
    alpha = 2.0 * r
    W = inputs.weight((N, K), 0.02, seed, outlier_frac=1e-3, outlier_scale=10.0)
    Wq, ref = _check_codec(W)
    X = inputs.normal((M, K), 1.0, seed + 1, DEV)
    dY = inputs.normal((M, N), 1.0, seed + 2, DEV)
    A = inputs.normal((r, K), 0.01, seed + 3, DEV)
    B = inputs.normal((N, r), 0.01, seed + 4, DEV)
    T = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
    Y = q.qlora_linear_fwd(X, Wq, A, B, alpha, T_save=T)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, Wq, A, B, alpha, T_saved=T)
    torch.cuda.synchronize()
    Wh = O.nf4_dequantize_fp8(ref)
    Yo, To = O.linear_fwd(bits(X), Wh, bits(A), bits(B), alpha, r)
    g = O.linear_bwd(bits(dY), bits(X), Wh, bits(A), bits(B), alpha, r)
    for name, got, want, bar in (("Y", Y, Yo, TOL), ("T", T, To, 1e-4), ("dX", dX, g["dX"], TOL),
                                 ("dA", dA, g["dA"], 1e-4), ("dB", dB, g["dB"], 1e-4)):
        e = O.rel_fro(f64(got), want)
        assert e <= bar, f"{name}: relative Frobenius error {e:.3e} > {bar:.0e}"
