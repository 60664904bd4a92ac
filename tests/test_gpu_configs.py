"""GPU checks of the two whole-model workloads:

  * the 32-layer LLaMA-7B-shaped stack (6.5B weights, ~N(0, 0.02), r = 16,
    4096 tokens = batch 8 x seq 512), and
  * the 80-layer LLaMA-65B-shaped model (64.7B weights, ~N(0, 0.015), r = 64,
    8192 tokens), whose NF4 form (~33.4 GB) stays resident on one GPU.

Every weight of both models is generated on the device and quantised; two
double-quantisation groups (256 blocks = 16384 consecutive weights) per
matrix are compared bit-exactly (codes, q8, s2) with the oracle quantising
the same weights.  The linear layer runs at the models' full token counts on
their largest projection: Y and dX are compared on a 512-token slice (their
rows are independent), dA and dB in full (rank-r products, cheap in the
oracle).
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
GROUP_W = 256 * 64


def _check_sampled_groups(W, Wq, rng, n=2):
    N, K = W.shape
    nblocks = N * K // 64
    ngroups = (nblocks + 255) // 256
    codes = Wq.codes.view(-1)
    for g in rng.choice(ngroups, size=min(n, ngroups), replace=False):
        b0, b1 = int(g) * 256, min(nblocks, int(g) * 256 + 256)
        w = host_f32(W.view(-1)[b0 * 64:b1 * 64]).reshape(b1 - b0, 64)
        ref = O.nf4_quantize(w)
        assert np.array_equal(codes[b0 * 32:b1 * 32].cpu().numpy(), ref["codes"].reshape(-1)), f"codes, group {g}"
        assert np.array_equal(Wq.absmax_q8[b0:b1].cpu().numpy(), ref["q8"]), f"q8, group {g}"
        assert Wq.group_scale[g:g + 1].cpu().numpy().view(np.uint32)[0] == ref["s2"].view(np.uint32)[0], \
            f"s2, group {g}"


@pytest.mark.parametrize("wl", [inputs.STACK7B, inputs.LLAMA65B], ids=["stack7b-32l", "llama65b-80l"])
def test_whole_model_quantisation_sampled_groups(wl):
    rng = np.random.default_rng(wl.base_seed)
    resident = []
    for L in range(wl.layers):
        for i, (name, N, K) in enumerate(wl.shapes):
            W = inputs.weight((N, K), wl.w_std, inputs.matrix_seed(wl.base_seed, L, i), device=DEV)
            Wq = q.qlora_quantize_nf4(W)
            _check_sampled_groups(W, Wq, rng)
            del W
            resident.append(Wq)
    gb = sum(w.nbytes() for w in resident) / 1e9
    print(wl.name, f"{len(resident)} matrices, {gb:.2f} GB NF4 resident")
    # 4.127 bits per weight: 3.34 GB (7B stack), 33.4 GB (65B)
    params = wl.layers * sum(N * K for _, N, K in wl.shapes)
    assert abs(gb * 1e9 - params * (0.5 + 1 / 64 + 4 / 16384)) < 1e6


@pytest.mark.parametrize("wl,proj", [(inputs.STACK7B, 6), (inputs.LLAMA65B, 4)], ids=["stack7b-down-m4096",
                                                                                      "llama65b-gate-m8192"])
def test_full_token_count_linear(wl, proj):
    name, N, K = wl.shapes[proj]
    M, r, alpha = wl.M, wl.r, wl.alpha
    seed = inputs.matrix_seed(wl.base_seed, wl.layers - 1, proj)
    W = inputs.weight((N, K), wl.w_std, seed, device=DEV)
    Wq = q.qlora_quantize_nf4(W)
    X = inputs.normal((M, K), 1.0, seed * 16 + 1)
    dY = inputs.normal((M, N), 1.0, seed * 16 + 2)
    A = inputs.normal((r, K), 0.01, seed * 16 + 3)
    B = inputs.normal((N, r), 0.01, seed * 16 + 4)
    T = torch.empty((M, r), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Xd, dYd, Ad, Bd = (t.to(DEV) for t in (X, dY, A, B))
    Y = q.qlora_linear_fwd(Xd, Wq, Ad, Bd, alpha, T_save=T, d_status=st)
    dX, dA, dB = q.qlora_linear_bwd(dYd, Xd, Wq, Ad, Bd, alpha, T_saved=T, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Wh = O.nf4_dequantize(O.nf4_quantize(host_f32(W)))
    del W
    assert np.array_equal(bits(q.qlora_dequantize(Wq)), Wh)
    S = 512
    Yo, To = O.linear_fwd(bits(X[:S]), Wh, bits(A), bits(B), alpha, r)
    gs = O.linear_bwd(bits(dY[:S]), bits(X[:S]), Wh, bits(A), bits(B), alpha, r)
    gf = O.linear_bwd(bits(dY), bits(X), None, bits(A), bits(B), alpha, r)
    errs = {"Y": O.rel_fro(f64(Y[:S]), Yo), "dX": O.rel_fro(f64(dX[:S]), gs["dX"]),
            "T": O.rel_fro(f64(T), gf["T"]), "dA": O.rel_fro(f64(dA), gf["dA"]), "dB": O.rel_fro(f64(dB), gf["dB"])}
    print(wl.name, name, M, errs)
    bars = {"Y": TOL, "dX": TOL, "T": 1e-4, "dA": 1e-4, "dB": 1e-4}
    for k, e in errs.items():
        assert e <= bars[k], f"{k}: relative Frobenius error {e:.3e} > {bars[k]:.0e} ({errs})"
