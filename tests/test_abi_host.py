"""Host-side checks of libqlora that need no GPU: the library loads, exports
every entry point include/qlora.h declares, answers the size/codebook/
workspace queries, and rejects bad arguments before touching the device."""
from __future__ import annotations

import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle as O
import bit_nf4_quantized_21_b200 as q
from bit_nf4_quantized_21_b200 import qlora as binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _header_functions()
    assert len(names) >= 9
    L = q.lib()
    for n in names:
        assert hasattr(L, n), f"libqlora.so does not export {n}"
    assert set(names) == set(binding.EXPORTED)


def test_codebook_matches_oracle():
    assert np.array_equal(np.array(q.qlora_nf4_codebook(), np.float32), O.nf4_levels())


@pytest.mark.parametrize("rows,cols", [(1, 64), (256, 512), (4096, 4096), (11008, 4096),
                                       (4096, 11008), (28672, 8192), (3, 192)])
def test_sizes_match_oracle_and_closed_form(rows, cols):
    for dq in (True, False):
        assert q.qlora_nf4_sizes(rows, cols, dq) == O.nf4_sizes(rows, cols, dq)
    c, a, g = q.qlora_nf4_sizes(rows, cols, True)
    assert c + a + g == rows * cols // 2 + rows * cols // 64 + 4 * math.ceil(rows * cols / 16384)


@pytest.mark.parametrize("rows,cols", [(0, 64), (4, 0), (4, 65), (4, 100), (-1, 64)])
def test_sizes_reject_bad_shapes(rows, cols):
    with pytest.raises(q.QloraError):
        q.qlora_nf4_sizes(rows, cols, True)


def test_workspace_query():
    assert q.qlora_workspace_bytes(2048, 4096, 4096, 16) > 0
    assert q.qlora_workspace_bytes(0, 4096, 4096, 16) == 0
    assert q.qlora_workspace_bytes(16, 4096, 100, 16) == 0
    assert q.qlora_workspace_bytes(16, 4096, 4096, 0) == 0
    assert q.qlora_workspace_bytes(16, 4096, 4096, 257) == 0


def test_status_strings():
    for s in range(8):
        assert q.status_string(s)
    assert q.status_string(0) == "ok"


def _w(rows=256, cols=512, **kw):
    w = binding.NF4WeightC(rows, cols, 64, 256, 1, 0, 16 * 1024, 16 * 2048, 16 * 4096, None)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


# Fake, 16-byte-aligned, never-dereferenced device addresses: every call below
# must fail validation on the host, before anything is enqueued.
FAKE = 1 << 40


@pytest.mark.parametrize("field,value,expect", [
    ("blocksize", 32, 2), ("group", 128, 2), ("cols", 100, 1), ("rows", 0, 1),
    ("reserved", 1, 1), ("double_quant", 3, 1), ("double_quant", -1, 1), ("codes", None, 1), ("codes", FAKE + 8, 1),
])
def test_quantize_rejects_bad_weight_descriptor(field, value, expect):
    w = _w(**{field: value})
    rc = q.lib().qlora_quantize_nf4(FAKE, 1, ctypes.byref(w), None, None)
    assert rc == expect


def test_quantize_rejects_bad_input_pointer_and_dtype():
    w = _w()
    assert q.lib().qlora_quantize_nf4(None, 1, ctypes.byref(w), None, None) == 1
    assert q.lib().qlora_quantize_nf4(FAKE + 4, 1, ctypes.byref(w), None, None) == 1
    assert q.lib().qlora_quantize_nf4(FAKE, 7, ctypes.byref(w), None, None) == 1
    assert q.lib().qlora_dequantize(ctypes.byref(w), None, None) == 1


def _fwd(M=16, r=8, alpha=16.0, ws=None, ws_bytes=None, **ptrs):
    w = ptrs.pop("w", _w())
    need = q.qlora_workspace_bytes(M, w.rows, max(w.cols, 64), r) if r >= 1 else 0
    p = dict(X=FAKE, A=FAKE, B=FAKE, Y=FAKE, T=None)
    p.update(ptrs)
    return q.lib().qlora_linear_fwd(p["X"], M, ctypes.byref(w), p["A"], p["B"], r, alpha, p["Y"],
                                    p["T"], FAKE if ws is None else ws,
                                    need if ws_bytes is None else ws_bytes, None, None, None)


def test_linear_fwd_validation():
    assert _fwd(X=None) == 1
    assert _fwd(Y=FAKE + 2) == 1
    assert _fwd(M=0) == 1
    assert _fwd(r=0) == 1
    assert _fwd(r=257) == 1
    assert _fwd(alpha=float("nan")) == 1
    assert _fwd(ws=0) == 6
    assert _fwd(ws_bytes=16) == 6
    assert _fwd(w=_w(rows=252)) == 2            # N % 8 != 0 is not built
    assert _fwd(w=_w(blocksize=128)) == 2


def test_linear_bwd_validation():
    w = _w()
    need = q.qlora_workspace_bytes(16, 256, 512, 8)
    L = q.lib()
    args = [FAKE, FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 16.0, None, FAKE, FAKE, FAKE, 0, FAKE,
            need, None, None, None]
    bad = list(args); bad[0] = None
    assert L.qlora_linear_bwd(*bad) == 1
    bad = list(args); bad[10] = None                 # dA
    assert L.qlora_linear_bwd(*bad) == 1
    bad = list(args); bad[12] = 5                    # grad dtype
    assert L.qlora_linear_bwd(*bad) == 1
    bad = list(args); bad[14] = need - 1             # workspace too small
    assert L.qlora_linear_bwd(*bad) == 6
    bad = list(args); bad[8] = FAKE + 4              # misaligned T_saved
    assert L.qlora_linear_bwd(*bad) == 1


def test_dropout_validation():
    # an invalid rate or a workspace sized for the plain layer is rejected
    # before anything is enqueued (no GPU needed for these answers)
    w = _w()
    L = q.lib()
    need = q.qlora_workspace_bytes_dropout(16, 256, 512, 8)
    assert need > q.qlora_workspace_bytes(16, 256, 512, 8) + 16 * 512 * 6
    assert q.qlora_workspace_bytes_dropout(0, 256, 512, 8) == 0
    args = [FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 16.0, 0.05, 7, FAKE, None, FAKE, need, None, None, None]
    for p in (-0.01, 1.0, float("nan"), float("inf")):
        bad = list(args); bad[7] = p
        assert L.qlora_linear_fwd_dropout(*bad) == 1
    bad = list(args); bad[12] = q.qlora_workspace_bytes(16, 256, 512, 8)
    assert L.qlora_linear_fwd_dropout(*bad) == 6
    bargs = [FAKE, FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 16.0, 0.05, 7, None, FAKE, FAKE, FAKE, 0, FAKE,
             need, None, None, None]
    bad = list(bargs); bad[8] = 1.5
    assert L.qlora_linear_bwd_dropout(*bad) == 1
    bad = list(bargs); bad[12] = None                # dA
    assert L.qlora_linear_bwd_dropout(*bad) == 1
    assert L.qlora_lora_dropout_mask(16, 512, 1.0, 7, FAKE, None) == 1
    assert L.qlora_lora_dropout_mask(16, 100, 0.1, 7, FAKE, None) == 1      # K % 64 != 0
    assert L.qlora_lora_dropout_mask(16, 512, 0.1, 7, None, None) == 1


def test_fp8_scale_format_sizes():
    # E4M3 second-level scales take the same storage as the 8-bit format
    assert q.qlora_nf4_sizes(256, 512, 2) == q.qlora_nf4_sizes(256, 512, 1)


def test_lora_dense_validation():
    # the dense-bf16 entries apply the NF4 entries' shape rules to (N, K)
    L = q.lib()
    M, N, K, r = 16, 256, 512, 8
    need = q.qlora_workspace_bytes(M, N, K, r)
    fwd = [FAKE, M, FAKE, N, K, FAKE, FAKE, r, 16.0, FAKE, None, FAKE, need, None, None, None]

    def f(i, v):
        a = list(fwd); a[i] = v
        return L.qlora_lora_linear_fwd(*a)
    assert f(2, None) == 1                  # W
    assert f(2, FAKE + 8) == 1              # misaligned W
    assert f(0, None) == 1                  # X
    assert f(4, 500) == 1                   # K % 64 != 0
    assert f(3, 252) == 2                   # N % 8 != 0 is not built
    assert f(1, 0) == 1                     # M
    assert f(7, 0) == 1 and f(7, 257) == 1  # r
    assert f(8, float("inf")) == 1          # alpha
    assert f(12, need - 1) == 6             # workspace too small
    assert f(11, None) == 6                 # no workspace
    bwd = [FAKE, FAKE, M, FAKE, N, K, FAKE, FAKE, r, 16.0, None, FAKE, FAKE, FAKE, 0, FAKE, need, None, None,
           None]

    def b(i, v):
        a = list(bwd); a[i] = v
        return L.qlora_lora_linear_bwd(*a)
    assert b(3, None) == 1                  # W
    assert b(0, None) == 1                  # dY
    assert b(12, None) == 1                 # dA
    assert b(14, 7) == 1                    # grad dtype
    assert b(5, 96) == 1                    # K % 64 != 0
    assert b(16, need - 1) == 6
    assert b(10, FAKE + 4) == 1             # misaligned T_saved


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        q.qlora_quantize_nf4(torch.zeros(4, 64), out=q.NF4Weight(4, 64, True, torch.zeros(4, 32, dtype=torch.uint8),
                                                                  torch.zeros(4, dtype=torch.uint8),
                                                                  torch.zeros(1), None))
