"""One pass over every kernel path of the library, for the debug-build test.

Run as a script (python tests/debug_build_workload.py) with QLORA_LIB naming
the library to load; prints one JSON line: the SHA-256 of every output,
whether the library has range checks compiled in, the site recorded by the
self-test kernel, and the range-failure word after the workload (0 when no
check failed).  Inputs are seeded; every kernel of the library is
deterministic, so two builds must print the same hashes.
"""
from __future__ import annotations

import ctypes
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

import torch  # noqa: E402

import bit_nf4_quantized_21_b200 as q  # noqa: E402
from bit_nf4_quantized_21_b200 import inputs  # noqa: E402

DEV = "cuda"


def digest(t: torch.Tensor) -> str:
    return hashlib.sha256(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()).hexdigest()[:16]


def main() -> None:
    L = q.lib()
    out = {"checks": int(L.qlora_debug_checks_enabled())}
    site = ctypes.c_uint(0)
    assert L.qlora_debug_range_check(ctypes.byref(site)) == 0          # clear
    assert L.qlora_debug_range_selftest(None) == 0
    torch.cuda.synchronize()
    assert L.qlora_debug_range_check(ctypes.byref(site)) == 0
    out["selftest_site"] = int(site.value)

    N, K = 512, 1024
    W = inputs.weight((N, K), 0.02, 71, device=DEV)
    for dq in (0, 1, 2):   # no second level, 8-bit linear, FP8 E4M3
        Wq = q.qlora_quantize_nf4(W, out=q.empty_nf4(N, K, DEV, dq))
        out[f"codes_dq{dq}"] = digest(Wq.codes)
        out[f"deq_dq{dq}"] = digest(q.qlora_dequantize(Wq))
    Wq32 = q.qlora_quantize_nf4(W.float())
    out["codes_f32"] = digest(Wq32.codes)
    Wq = q.qlora_quantize_nf4(W)
    for M, r, mt in ((600, 16, 2), (300, 16, 1), (300, 5, 0), (96, 16, 0), (16, 16, 0), (1, 8, 0)):
        assert L.qlora_debug_set_pair_mtiles(mt) == 0
        X = inputs.normal((M, K), 1.0, 72 + M, DEV)
        dY = inputs.normal((M, N), 1.0, 73 + M, DEV)
        A = inputs.normal((r, K), 0.01, 74 + M, DEV)
        B = inputs.normal((N, r), 0.01, 75 + M, DEV)
        T = torch.empty((M, r), dtype=torch.float32, device=DEV)
        Y = q.qlora_linear_fwd(X, Wq, A, B, 2.0 * r, T_save=T)
        dX, dA, dB = q.qlora_linear_bwd(dY, X, Wq, A, B, 2.0 * r, T_saved=T)
        for name, t in (("Y", Y), ("T", T), ("dX", dX), ("dA", dA), ("dB", dB)):
            out[f"{name}_M{M}_r{r}_mt{mt}"] = digest(t)
        if M >= 96:
            Yd = q.qlora_linear_fwd_dropout(X, Wq, A, B, 2.0 * r, 0.1, 99)
            gd = q.qlora_linear_bwd_dropout(dY, X, Wq, A, B, 2.0 * r, 0.1, 99)
            out[f"drop_M{M}_r{r}_mt{mt}"] = [digest(Yd)] + [digest(t) for t in gd]
            Wd = q.qlora_dequantize(Wq)
            Yl = q.qlora_lora_linear_fwd(X, Wd, A, B, 2.0 * r)
            gl = q.qlora_lora_linear_bwd(dY, X, Wd, A, B, 2.0 * r)
            out[f"lora_M{M}_r{r}_mt{mt}"] = [digest(Yl)] + [digest(t) for t in gl]
    assert L.qlora_debug_set_pair_mtiles(0) == 0
    n = 40000
    master = inputs.normal((n,), 1.0, 81, DEV, torch.float32)
    m1, m2 = torch.zeros_like(master), torch.zeros_like(master)
    grad = inputs.normal((n,), 1.0, 82, DEV, torch.float32)
    q.qlora_adam_step(master, m1, m2, grad, 1, 1e-3)
    out["adam"] = [digest(master), digest(m1), digest(m2)]
    A = inputs.normal((16, K), 0.01, 83, DEV)
    B = inputs.normal((N, 16), 0.01, 84, DEV)
    merged, Wm = q.qlora_merge_nf4(Wq, A, B, 32.0)
    out["merge"] = [digest(merged.codes), digest(Wm)]
    torch.cuda.synchronize()
    assert L.qlora_debug_range_check(ctypes.byref(site)) == 0
    out["range_site"] = int(site.value)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
