"""The library's calls captured into CUDA graphs give the eager results bit
for bit.

Every kernel of the library is deterministic (fixed-order reductions), so
a forward + backward replayed from a graph -- with independent projections
on side streams forked from and joined back into the capturing stream, and
the fused GEMMs launched as programmatic dependents of the adapter kernels
ahead of them -- must reproduce the outputs of the same calls made one by
one.  Three projections share one input, as q/k/v do in a decoder layer.
"""
from __future__ import annotations

import pytest
import torch

import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(M, N, K, r, n, seed):
    X = inputs.normal((M, K), 1.0, seed, DEV)
    proj = []
    for i in range(n):
        s = seed + 10 * (i + 1)
        proj.append(dict(
            Wq=q.qlora_quantize_nf4(inputs.weight((N, K), 0.02, s, device=DEV)),
            A=inputs.normal((r, K), 0.01, s + 1, DEV), B=inputs.normal((N, r), 0.01, s + 2, DEV),
            dY=inputs.normal((M, N), 1.0, s + 3, DEV),
            Y=torch.empty((M, N), dtype=torch.bfloat16, device=DEV),
            T=torch.empty((M, r), dtype=torch.float32, device=DEV),
            dX=torch.empty((M, K), dtype=torch.bfloat16, device=DEV),
            dA=torch.empty((r, K), dtype=torch.float32, device=DEV),
            dB=torch.empty((N, r), dtype=torch.float32, device=DEV),
            ws=torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=DEV)))
    return X, proj


def _call(X, p, alpha):
    q.qlora_linear_fwd(X, p["Wq"], p["A"], p["B"], alpha, Y=p["Y"], T_save=p["T"], workspace=p["ws"])
    q.qlora_linear_bwd(p["dY"], X, p["Wq"], p["A"], p["B"], alpha, T_saved=p["T"], dX=p["dX"], dA=p["dA"],
                       dB=p["dB"], workspace=p["ws"])


def _outputs(proj):
    return [torch.cat([p[k].reshape(-1).view(torch.uint8) for k in ("Y", "T", "dX", "dA", "dB")]).clone()
            for p in proj]


def _poison(proj):
    for p in proj:
        for k in ("Y", "T", "dX", "dA", "dB"):
            p[k].fill_(float("nan"))


@pytest.mark.parametrize("M,N,K,r,mtiles", [
    (600, 512, 1024, 16, 0),    # 2-SM GEMM (two M tiles chosen), split-K adapter products
    (1100, 264, 576, 8, 1),     # one M tile per pair, ragged N and K
    (96, 256, 512, 16, 0),      # the 1-CTA GEMM (no dependent launch)
])
def test_graph_replay_with_side_streams_equals_eager(M, N, K, r, mtiles):
    L = q.lib()
    assert L.qlora_debug_set_pair_mtiles(mtiles) == 0
    try:
        alpha = 2.0 * r
        X, proj = _layer(M, N, K, r, 3, seed=M + N + K)
        for p in proj:
            _call(X, p, alpha)
        torch.cuda.synchronize()
        want = _outputs(proj)

        side = [torch.cuda.Stream() for _ in proj]

        def step():
            main = torch.cuda.current_stream()
            fork = torch.cuda.Event()
            fork.record(main)
            joins = []
            for s, p in zip(side, proj):
                s.wait_event(fork)
                with torch.cuda.stream(s):
                    _call(X, p, alpha)
                    e = torch.cuda.Event()
                    e.record(s)
                joins.append(e)
            for e in joins:
                main.wait_event(e)

        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(2):
            _poison(proj)
            g.replay()
            torch.cuda.synchronize()
            got = _outputs(proj)
            for i, (a, b) in enumerate(zip(got, want)):
                assert torch.equal(a, b), f"projection {i}: graph replay differs from the eager calls"
    finally:
        assert L.qlora_debug_set_pair_mtiles(0) == 0
