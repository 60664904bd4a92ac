"""The adapter optimiser step over paged (unified-memory) state.

"QLoRA" (learning-llms page), the paragraph on paged optimizers, and
"QLoRA" (scalata.ai), "How it works": the optimiser state lives in unified
memory, which the driver pages out to host RAM under a memory spike and
back on the next access.  Here the fp32 master copy and both moments are
allocated with qlora_paged_alloc (CUDA managed memory); qlora_adam_step
runs on them unchanged, with the state prefetched to the GPU, paged out to
the host and faulted back in, and paged out and prefetched back.  Every
step is checked against the binary64 oracle with the bars of the device-
memory test.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _host_view(ptr: int, n: int) -> np.ndarray:
    """numpy view of n fp32 in managed memory (the host may read and write it
    between GPU work, after a synchronisation)."""
    return np.ctypeslib.as_array((ctypes.c_float * n).from_address(ptr))


def test_paged_state_adam_matches_oracle():
    n = (1 << 20) + 36                      # a multiple of 4 with a ragged tail of the 4-wide loop
    lr, b1, b2, eps, wd = 1e-3, 0.9, 0.999, 1e-8, 0.01
    ptrs = [q.qlora_paged_alloc(4 * n) for _ in range(3)]
    try:
        master, m, v = (_host_view(p, n) for p in ptrs)
        g = torch.Generator().manual_seed(11)
        master[:] = (torch.randn(n, generator=g) * 0.02).numpy()
        m[:] = 0.0
        v[:] = 0.0
        ref = [master.astype(np.float64), np.zeros(n), np.zeros(n)]
        stream = torch.cuda.current_stream()
        f = lambda x: float(np.float32(x))
        # where the state is before each step: on the GPU, paged out and
        # faulted back in by the kernel, paged out and prefetched back
        for step, where in enumerate(("device", "host-fault", "host-prefetch", "device"), start=1):
            if where == "device" or where == "host-prefetch":
                if where == "host-prefetch":
                    for p in ptrs:
                        q.qlora_paged_prefetch(p, 4 * n, to_device=False, stream=stream)
                for p in ptrs:
                    q.qlora_paged_prefetch(p, 4 * n, to_device=True, stream=stream)
            else:
                for p in ptrs:
                    q.qlora_paged_prefetch(p, 4 * n, to_device=False, stream=stream)
            grad = (torch.randn(n, generator=g) * 1e-2).float()
            st = torch.zeros(1, dtype=torch.int32, device=DEV)
            gd = grad.to(DEV)
            rc = q.lib().qlora_adam_step(ptrs[0], ptrs[1], ptrs[2], None, gd.data_ptr(), q.qlora.QLORA_F32, n,
                                         step, lr, b1, b2, eps, wd, 1.0, st.data_ptr(), stream.cuda_stream)
            assert rc == 0
            torch.cuda.synchronize()
            assert st.item() == 0
            old_theta, old_m = ref[0].copy(), ref[1].copy()
            ref = list(O.adam_step(ref[0], ref[1], ref[2], grad.double().numpy(), step, f(lr), f(b1), f(b2), f(eps),
                                   weight_decay=f(wd)))
            g64 = grad.double().numpy()
            m_scale = b1 * np.abs(old_m) + (1 - b1) * np.abs(g64)
            assert np.all(np.abs(m.astype(np.float64) - ref[1]) <= 1e-6 * m_scale + 1e-37), (where, "m")
            assert np.all(np.abs(v.astype(np.float64) - ref[2]) <= 1e-6 * np.abs(ref[2]) + 1e-37), (where, "v")
            assert np.all(np.abs(master.astype(np.float64) - ref[0]) <= 1e-6 * np.abs(old_theta) + 1e-5 * lr), \
                (where, "master")
            # the next step starts from the state as the GPU left it (fp32)
            ref = [master.astype(np.float64), m.astype(np.float64), v.astype(np.float64)]
    finally:
        torch.cuda.synchronize()
        for p in ptrs:
            q.qlora_paged_free(p)


def test_paged_alloc_rejects_zero_and_frees_null():
    with pytest.raises(q.QloraError):
        q.qlora_paged_alloc(0)
    q.qlora_paged_free(0)          # freeing nothing is a no-op
