"""The no-allocation forward (qlora_linear_fwd_noalloc), called through the
C ABI, against the workspace forward (qlora_linear_fwd).

It serves callers that cannot allocate device memory themselves (plugin
hosts that pass only inputs and outputs, processes whose memory sits in
another allocator's pool, loops that must not synchronise on an
allocation); its scratch is the library's fixed 16 MiB device array, which
keeps the previous call's contents -- hence two calls in a row with
different inputs.  This file sorts last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import inputs
from bit_nf4_quantized_21_b200.qlora import NF4WeightC
from gpu_util import bits, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def _call_noalloc(X, Wq, A, B, alpha, Y, T):
    cw = Wq.c()
    rc = q.lib().qlora_linear_fwd_noalloc(
        X.data_ptr(), X.shape[0], ctypes.byref(cw), A.data_ptr(), B.data_ptr(), A.shape[0],
        float(alpha), Y.data_ptr(), T.data_ptr() if T is not None else None, None,
        torch.cuda.current_stream().cuda_stream)
    return rc


@pytest.mark.parametrize("M,N,K,r", [
    (200, 264, 576, 8), (2048, 4096, 4096, 16), (96, 136, 448, 5),
    (16, 512, 1024, 16), (1, 8192, 512, 8),     # decode shapes: the weight-streaming kernel on the fixed scratch
])
def test_noalloc_forward_matches_workspace_forward_twice(M, N, K, r):
    # (every case has >= 8192 outputs: the bf16 rounding of Y alone gives a
    # relative error near 1.7e-3 on average, and on a few hundred outputs it
    # can exceed the 2e-3 bar by chance)
    # The entry point runs the same kernels with the same plans as the
    # workspace forward, only on other scratch memory, so Y and T must be
    # bit-identical to it; both are also held to the oracle's tolerance.
    # The outputs are NaN-poisoned first, so an unwritten element fails.
    alpha = 2.0 * r
    for call, seed in enumerate((101, 202)):          # two calls in a row, different inputs
        W = inputs.weight((N, K), 0.02, seed + M, device=DEV)
        Wq = q.qlora_quantize_nf4(W)
        X = inputs.normal((M, K), 1.0, seed + 1, DEV)
        A = inputs.normal((r, K), 0.01, seed + 3, DEV)
        B = inputs.normal((N, r), 0.01, seed + 4, DEV)
        Y_ref = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        T_ref = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
        q.qlora_linear_fwd(X, Wq, A, B, alpha, Y=Y_ref, T_save=T_ref)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
        assert _call_noalloc(X, Wq, A, B, alpha, Y, T) == 0
        Y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(X, Wq, A, B, alpha, Y2, None) == 0   # T kept in the scratch
        torch.cuda.synchronize()
        for got in (Y, Y2):
            assert torch.equal(got.view(torch.int16), Y_ref.view(torch.int16)), f"call {call}: Y differs"
        assert torch.equal(T.view(torch.int32), T_ref.view(torch.int32)), f"call {call}: T differs"
        # the oracle, on the same dequantised weights
        ref = O.nf4_quantize(W.float().cpu().numpy())
        Wh = O.nf4_dequantize(ref)
        Yo, To = O.linear_fwd(bits(X), Wh, bits(A), bits(B), alpha, r)
        assert O.rel_fro(f64(Y), Yo) <= TOL
        assert O.rel_fro(f64(T), To) <= 1e-4


def test_noalloc_rejects_problems_beyond_the_scratch():
    W = inputs.weight((256, 64), 0.02, 7, device=DEV)
    Wq = q.qlora_quantize_nf4(W)
    cw = Wq.c()
    # rank 64 at M = 65536: fp32 T (16 MiB) plus the two bf16 planes of s*T
    # (16 MiB) alone are twice the fixed scratch
    M = 65536
    X = torch.empty((M, 64), dtype=torch.bfloat16, device=DEV)
    A = torch.empty((64, 64), dtype=torch.bfloat16, device=DEV)
    B = torch.empty((256, 64), dtype=torch.bfloat16, device=DEV)
    Y = torch.empty((M, 256), dtype=torch.bfloat16, device=DEV)
    rc = q.lib().qlora_linear_fwd_noalloc(X.data_ptr(), M, ctypes.byref(cw), A.data_ptr(), B.data_ptr(), 64,
                                          16.0, Y.data_ptr(), None, None,
                                          torch.cuda.current_stream().cuda_stream)
    assert rc == 7 and "scratch" in q.status_string(rc)
