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
