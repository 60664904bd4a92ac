"""GPU parity of the adapter merge (qlora_merge_nf4: NF4(W^ + s B A)) against
the CPU oracle.  The merged values decide integer codes, so both sides form
them in the same precision and order (fp32, one rounding per operation):
the fp32 merged weight, the codes, the q8 scales and the group scales are
compared bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import inputs
from gpu_util import bits, host_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _merge_check(N, K, r, seed, dq=True, in_place=False):
    W = inputs.weight((N, K), 0.02, seed, dtype=torch.bfloat16)
    A = inputs.normal((r, K), 0.01, seed * 16 + 3)
    B = inputs.normal((N, r), 0.01, seed * 16 + 4)
    alpha = 2.0 * r
    Wq = q.qlora_quantize_nf4(W.to(DEV))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    if in_place:
        out, Wm = q.qlora_merge_nf4(Wq, A.to(DEV), B.to(DEV), alpha, out=Wq, d_status=st)
    else:
        out, Wm = q.qlora_merge_nf4(Wq, A.to(DEV), B.to(DEV), alpha, double_quant=dq, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    merged = O.merge_nf4(O.nf4_quantize(host_f32(W)), bits(A), bits(B), alpha, r)
    assert np.array_equal(Wm.cpu().numpy().view(np.uint32), merged.view(np.uint32)), "merged fp32 weight"
    ref = O.nf4_quantize(merged, double_quant=dq)
    assert np.array_equal(out.codes.cpu().numpy(), ref["codes"]), "codes"
    if dq:
        assert np.array_equal(out.absmax_q8.cpu().numpy(), ref["q8"]), "q8"
        assert np.array_equal(out.group_scale.cpu().numpy().view(np.uint32), ref["s2"].view(np.uint32)), "s2"
    else:
        assert np.array_equal(out.absmax_f32.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    return out


@pytest.mark.parametrize("N,K,r", [
    (256, 576, 8),       # groups that straddle rows, K not a multiple of 256
    (264, 704, 5),       # odd rank
    (8, 64, 1),          # one block per row, rank 1
    (64, 1024, 256),     # maximum rank
])
def test_merge_matches_oracle(N, K, r):
    _merge_check(N, K, r, seed=N + K + r)


def test_merge_without_double_quant_and_in_place():
    _merge_check(128, 512, 16, seed=3, dq=False)
    _merge_check(128, 512, 16, seed=4, in_place=True)


def test_merge_llama7b_gate_full():
    _merge_check(11008, 4096, 16, seed=inputs.matrix_seed(2, 0, 4))


def _fused_check(N, K, r, seed, src_dq=1, out_dq=1):
    # the one-pass form (no fp32 buffer) against the oracle, for every pair
    # of source and output second-level formats
    W = inputs.weight((N, K), 0.02, seed, dtype=torch.bfloat16)
    A = inputs.normal((r, K), 0.01, seed * 16 + 3)
    B = inputs.normal((N, r), 0.01, seed * 16 + 4)
    alpha = 2.0 * r
    Wq = q.qlora_quantize_nf4(W.to(DEV), out=q.empty_nf4(N, K, DEV, src_dq))
    out = q.empty_nf4(N, K, DEV, out_dq)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, Wm = q.qlora_merge_nf4(Wq, A.to(DEV), B.to(DEV), alpha, out=out, keep_merged=False, d_status=st)
    torch.cuda.synchronize()
    assert Wm is None and st.item() == 0
    src = {0: O.nf4_quantize(host_f32(W), double_quant=False), 1: O.nf4_quantize(host_f32(W)),
           2: O.nf4_quantize_fp8(host_f32(W))}[src_dq]
    Wh = O.nf4_dequantize_fp8(src) if src_dq == 2 else O.nf4_dequantize(src)
    merged = O.merge_nf4(src, bits(A), bits(B), alpha, r, W_hat=Wh)
    ref = {0: lambda m: O.nf4_quantize(m, double_quant=False), 1: O.nf4_quantize,
           2: O.nf4_quantize_fp8}[out_dq](merged)
    assert np.array_equal(out.codes.cpu().numpy(), ref["codes"]), "codes"
    if out_dq:
        assert np.array_equal(out.absmax_q8.cpu().numpy(), ref["q8"]), "q8"
        assert np.array_equal(out.group_scale.cpu().numpy().view(np.uint32), ref["s2"].view(np.uint32)), "s2"
    else:
        assert np.array_equal(out.absmax_f32.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))


@pytest.mark.parametrize("N,K,r,src_dq,out_dq", [
    (256, 576, 8, 1, 1),     # groups straddling rows
    (264, 704, 5, 1, 0),     # odd rank, output without a second level
    (8, 64, 1, 0, 1),        # one block per row, rank 1, fp32 source scales
    (64, 1024, 256, 2, 2),   # maximum rank, FP8 scales in and out
    (128, 512, 16, 2, 1),
])
def test_fused_merge_matches_oracle(N, K, r, src_dq, out_dq):
    _fused_check(N, K, r, seed=7 * N + K + r, src_dq=src_dq, out_dq=out_dq)


def test_fused_merge_equals_two_pass_on_llama7b_gate():
    N, K, r = 11008, 4096, 16
    seed = inputs.matrix_seed(2, 0, 4)
    W = inputs.weight((N, K), 0.02, seed, device=DEV)
    A = inputs.normal((r, K), 0.01, seed * 16 + 3, DEV)
    B = inputs.normal((N, r), 0.01, seed * 16 + 4, DEV)
    Wq = q.qlora_quantize_nf4(W)
    two, _ = q.qlora_merge_nf4(Wq, A, B, 32.0)
    one, _ = q.qlora_merge_nf4(Wq, A, B, 32.0, keep_merged=False)
    torch.cuda.synchronize()
    for name in ("codes", "absmax_q8", "group_scale"):
        assert torch.equal(getattr(one, name), getattr(two, name)), name


def test_fused_merge_refuses_in_place():
    Wq = q.qlora_quantize_nf4(inputs.weight((64, 256), 0.02, 5, device=DEV))
    A = inputs.normal((4, 256), 0.01, 6, DEV)
    B = inputs.normal((64, 4), 0.01, 7, DEV)
    with pytest.raises(q.QloraError):
        q.qlora_merge_nf4(Wq, A, B, 8.0, out=Wq, keep_merged=False)
