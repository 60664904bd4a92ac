"""The debug build (libqlora_debug.so, -DQLORA_DEBUG_CHECKS) against the
release build.

The debug build checks its kernels' shared-memory, tensor-memory, workspace
and TMA-coordinate computations; a failed check records its site in a
device word and skips the access (it never traps).  The same seeded
workload (tests/debug_build_workload.py: the quantiser in every
second-level format, the dequantiser, the forward and backward on the 2-SM
GEMM with one and two M tiles, the 1-CTA GEMM, the decode kernel, dropout,
the dense-bf16 baseline, Adam and the merge) runs through each build in a
process of its own: no check may fail, the self-test kernel's record must
reach the host, and every output must be bit-identical between the builds.
"""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.join(os.path.dirname(HERE), "bit_nf4_quantized_21_b200")


def _run(lib: str) -> dict:
    env = dict(os.environ, QLORA_LIB=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_build_workload.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_debug_build_checks_pass_and_match_release():
    debug_lib = os.path.join(PKG, "libqlora_debug.so")
    assert os.path.exists(debug_lib), "libqlora_debug.so not built (bit_nf4_quantized_21_b200.build)"
    dbg = _run(debug_lib)
    rel = _run(os.path.join(PKG, "libqlora.so"))
    assert dbg.pop("checks") == 1 and rel.pop("checks") == 0
    assert dbg.pop("selftest_site") == 0xFFFF and rel.pop("selftest_site") == 0xFFFF
    assert dbg.pop("range_site") == 0, "a range check failed in the debug build"
    rel.pop("range_site")
    diff = [k for k in rel if rel[k] != dbg.get(k)]
    assert not diff, f"outputs differ between the debug and release builds: {diff}"
