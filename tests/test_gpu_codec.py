"""GPU parity of the NF4 quantiser and dequantiser against the CPU oracle:
bit-exact codes, q8 scales, group scales, fp32 absmax and bf16 weights."""
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


def _roundtrip(W: torch.Tensor, dq: bool = True):
    """Quantise + dequantise W on the GPU, return the arrays on the host."""
    Wq = q.empty_nf4(W.shape[0], W.shape[1], DEV, dq, keep_absmax_f32=True)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlora_quantize_nf4(W.to(DEV).contiguous(), out=Wq, d_status=st)
    Wh = q.qlora_dequantize(Wq)
    torch.cuda.synchronize()
    return Wq, Wh, int(st.item())


def _check_exact(W: torch.Tensor, dq: bool = True):
    Wq, Wh, st = _roundtrip(W, dq)
    assert st == 0
    ref = O.nf4_quantize(host_f32(W), double_quant=dq)
    assert np.array_equal(Wq.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(Wq.absmax_f32.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    if dq:
        assert np.array_equal(Wq.absmax_q8.cpu().numpy(), ref["q8"])
        assert np.array_equal(Wq.group_scale.cpu().numpy().view(np.uint32), ref["s2"].view(np.uint32))
    assert np.array_equal(bits(Wh), O.nf4_dequantize(ref))
    return Wq, Wh


def test_single_layer_fp32_weight():
    p = inputs.projection_inputs(inputs.SINGLE, 0, 0)
    _check_exact(p["W"], dq=True)
    _check_exact(p["W"], dq=False)


@pytest.mark.parametrize("proj", [0, 4, 6])   # q 4096x4096, gate 11008x4096, down 4096x11008
def test_llama7b_projection_bf16(proj):
    p = inputs.projection_inputs(inputs.LLAMA7B, 0, proj, with_grad=False)
    _check_exact(p["W"])


@pytest.mark.parametrize("rows,cols", [(1, 64), (3, 192), (7, 11008), (5, 16448), (33, 320)])
def test_ragged_shapes(rows, cols):
    # partial last groups, groups that straddle rows, a single block
    W = inputs.weight((rows, cols), 0.02, rows * 31 + cols, dtype=torch.bfloat16)
    _check_exact(W, dq=True)
    _check_exact(W, dq=False)


def test_outliers_zero_and_subnormal_blocks():
    W = inputs.weight((64, 1024), 0.02, 77, dtype=torch.float32, outlier_frac=1e-2,
                      outlier_scale=10.0)
    W[3, :64] = 0.0                       # zero block
    W[5, 128:192] = 1e-40                 # subnormal block -> code 7
    W[6, :] = 0.0                         # whole group of zeros in one row
    W[7, 64:128] = -0.0
    W[8, 0:64] = torch.from_numpy(O.nf4_levels())[None].repeat(4, 1).reshape(-1) * 3.0   # exact levels
    # absmax 1 so that x = w exactly; the binary32 neighbours just below and
    # just above every level midpoint (and the midpoint itself when exact)
    lv = O.nf4_levels().astype(np.float64)
    mids = (lv[:-1] + lv[1:]) / 2
    dn = np.array([np.nextafter(np.float32(m), np.float32(-2)) if float(np.float32(m)) >= m
                   else np.float32(m) for m in mids], np.float32)
    up = np.nextafter(dn, np.float32(2))
    row = np.zeros(64, np.float32)
    row[0] = 1.0
    row[1:16], row[16:31] = dn, up
    row[31:46] = -dn[::-1]
    W[9, 0:64] = torch.from_numpy(row)
    _check_exact(W, dq=True)
    W2 = torch.zeros(2, 16384, dtype=torch.float32)   # all-zero groups: s2 = 0, q8 = 0
    _check_exact(W2, dq=True)


def test_decode_shape_sampled_groups():
    # 70B MLP shape with outliers: every output bit-exact would need 235M oracle
    # encodes, so check the whole GPU result on sampled 256-block groups.
    W = inputs.weight((28672, 8192), 0.02, 3000, device=DEV, dtype=torch.bfloat16,
                      outlier_frac=1e-3, outlier_scale=10.0)
    Wq, Wh, st = _roundtrip(W)
    assert st == 0
    flat = W.view(-1)
    ngroups = W.numel() // 16384
    rng = np.random.default_rng(0)
    for g in list(rng.choice(ngroups, 12, replace=False)) + [0, ngroups - 1]:
        src = flat[g * 16384:(g + 1) * 16384].float().cpu().numpy()[None]
        ref = O.nf4_quantize(src)
        got_codes = Wq.codes.view(-1)[g * 8192:(g + 1) * 8192].cpu().numpy()
        assert np.array_equal(got_codes, ref["codes"].ravel())
        assert np.array_equal(Wq.absmax_q8[g * 256:(g + 1) * 256].cpu().numpy(), ref["q8"])
        assert Wq.group_scale[g].item() == ref["s2"][0]
        got_w = bits(Wh.view(-1)[g * 16384:(g + 1) * 16384])
        assert np.array_equal(got_w, O.nf4_dequantize(ref).ravel())


def test_nonfinite_sets_status_bit():
    for bad in (float("inf"), float("-inf"), float("nan")):
        W = torch.zeros(4, 256, dtype=torch.float32)
        W[2, 100] = bad
        _, _, st = _roundtrip(W)
        assert st & q.qlora.DEV_NONFINITE


def test_repeated_calls_are_deterministic():
    W = inputs.weight((512, 4096), 0.02, 5, device=DEV)
    a, ah, _ = _roundtrip(W)
    b, bh, _ = _roundtrip(W)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.absmax_q8, b.absmax_q8)
    assert torch.equal(ah.view(torch.int16), bh.view(torch.int16))


def _sweep_blocks(absmax: float, centres, half_width: int) -> np.ndarray:
    """fp32 blocks [n, 64]: element 0 is +/-absmax (alternating), elements
    1..63 walk every binary32 w within `half_width` ulps of fp32(x0 * absmax)
    for each centre x0, so that the normalised value x = w * fp32(1/absmax)
    steps across x0 one binary32 at a time (exactly so for absmax a power of
    two).  Values with |w| > absmax are dropped."""
    a = np.float32(absmax)
    vals = []
    for x0 in centres:
        w0 = np.float32(np.float64(x0) * np.float64(a))
        k = np.arange(-half_width, half_width + 1, dtype=np.int64)
        if w0 == 0:   # the edge at x = 0: the smallest magnitudes of both signs
            mag = np.arange(1, half_width + 1, dtype=np.int32).view(np.float32)
            vals.append(np.concatenate([mag, -mag]))
            continue
        base = np.int64(np.abs(w0).view(np.int32))
        mag = (base + k).astype(np.int32).view(np.float32)
        w = np.where(w0 < 0, -mag, mag).astype(np.float32)
        vals.append(w[np.abs(w) <= a])
    v = np.concatenate(vals)
    nb = -(-v.size // 63)
    v = np.concatenate([v, np.zeros(nb * 63 - v.size, np.float32)]).reshape(nb, 63)
    head = np.where(np.arange(nb) % 2 == 0, a, -a).astype(np.float32)[:, None]
    return np.concatenate([head, v], axis=1)


def test_encoder_cells_and_thresholds_swept_binary32():
    # The kernel counts #{i : x > t_i} through a table of 33 cells of width
    # 1/16 (one compare per cell; edges at the odd multiples of 1/32).  Sweep
    # every binary32 within 1500 ulps of each of the 15 thresholds and of
    # every multiple of 1/32 in [-1, 1] (the edges and the cell centres), at
    # absmax values that are powers of two (x = w / absmax exactly) and not,
    # and require the codes, scales and dequantised weights bit for bit.
    lv = O.nf4_levels().astype(np.float64)
    thr = (lv[:-1] + lv[1:]) / 2
    centres = np.concatenate([thr, np.arange(-32, 33) / 32.0])
    for absmax in (1.0, 2.0 ** -6, 2.0 ** 5, 0.02, 3.7, 0.0513):
        W = torch.from_numpy(_sweep_blocks(absmax, centres, 1500))
        _check_exact(W, dq=True)
        _check_exact(W, dq=False)
