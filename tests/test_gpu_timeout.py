"""A bounded device wait that runs out, made to happen without faulting the GPU.

Every pipeline wait in the library's kernels gives up after a bound, sets
QLORA_DEV_TIMEOUT_BIT in the call's status word, and lets the kernel free
its tensor memory and return.  Here the bound is shortened to 1 ms and one
stage of an adapter-product launch withholds its loads (a flag that
nothing sets), so that the wait on it runs out: the call must return, the
status must carry the timeout bit, and the next ordinary call on the same
stream must be correct -- nothing left waiting, no tensor memory leaked.
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


def _layer(M=256, N=512, K=1024, r=16, seed=61):
    W = inputs.weight((N, K), 0.02, seed, device=DEV)
    Wq = q.qlora_quantize_nf4(W)
    X = inputs.normal((M, K), 1.0, seed + 1, DEV)
    A = inputs.normal((r, K), 0.01, seed + 3, DEV)
    B = inputs.normal((N, r), 0.01, seed + 4, DEV)
    return W, Wq, X, A, B


def test_wait_that_runs_out_sets_status_and_the_next_call_is_correct():
    W, Wq, X, A, B = _layer()
    L = q.lib()
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert L.qlora_debug_set_wait_limit(1_000_000) == 0      # 1 ms
    assert L.qlora_debug_inject_stall(1) == 0
    try:
        q.qlora_linear_fwd(X, Wq, A, B, 32.0, d_status=st)   # T = X A^T's launch stalls
        torch.cuda.synchronize()
    finally:
        assert L.qlora_debug_inject_stall(0) == 0
        assert L.qlora_debug_set_wait_limit(0) == 0
    assert st.item() & q.qlora.DEV_TIMEOUT, f"status {st.item()}"
    # the same stream again, ordinary call: correct against the oracle
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    T = torch.full((X.shape[0], A.shape[0]), float("nan"), dtype=torch.float32, device=DEV)
    Y = q.qlora_linear_fwd(X, Wq, A, B, 32.0, T_save=T, d_status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    ref = O.nf4_quantize(W.float().cpu().numpy())
    Yo, To = O.linear_fwd(bits(X), O.nf4_dequantize(ref), bits(A), bits(B), 32.0, A.shape[0])
    assert O.rel_fro(f64(Y), Yo) <= 2e-3
    assert O.rel_fro(f64(T), To) <= 1e-4


def test_backward_stall_is_reported_too():
    W, Wq, X, A, B = _layer(seed=62)
    dY = inputs.normal((X.shape[0], W.shape[0]), 1.0, 99, DEV)
    T = torch.empty((X.shape[0], A.shape[0]), dtype=torch.float32, device=DEV)
    q.qlora_linear_fwd(X, Wq, A, B, 32.0, T_save=T)
    L = q.lib()
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert L.qlora_debug_set_wait_limit(1_000_000) == 0
    assert L.qlora_debug_inject_stall(1) == 0
    try:
        q.qlora_linear_bwd(dY, X, Wq, A, B, 32.0, T_saved=T, d_status=st)   # G and dA/dB launches stall
        torch.cuda.synchronize()
    finally:
        assert L.qlora_debug_inject_stall(0) == 0
        assert L.qlora_debug_set_wait_limit(0) == 0
    assert st.item() & q.qlora.DEV_TIMEOUT
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, Wq, A, B, 32.0, T_saved=T, d_status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    ref = O.nf4_quantize(W.float().cpu().numpy())
    g = O.linear_bwd(bits(dY), bits(X), O.nf4_dequantize(ref), bits(A), bits(B), 32.0, A.shape[0])
    for name, got, want, bar in (("dX", dX, g["dX"], 2e-3), ("dA", dA, g["dA"], 1e-4), ("dB", dB, g["dB"], 1e-4)):
        assert O.rel_fro(f64(got), want) <= bar, name
