"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: numbers
printed on the pages (tests/golden/, each file citing its source), closed
forms, invariants, an independent library routine, or brute force.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from bit_nf4_quantized_21_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    kv, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            try:
                rows.append([float(p) for p in parts])
            except ValueError:
                kv[parts[0]] = parts[1:]
    return kv, rows


# ------------------------------------------------- symmetric int4 (page 1)

def test_worked_int4_block_matches_page():
    kv, rows = _read_golden("int4_worked_block.txt")
    w = np.array([r[0] for r in rows], np.float32)
    q, scale, w_hat = O.absmax_int_quantize(w, bits=4)
    assert round(float(scale), 4) == float(kv["scale"][0])
    for i, r in enumerate(rows):
        assert round(float(w[i] / scale), 2) == pytest.approx(r[1], abs=1e-9)
        assert q[i] == int(r[2])
        assert round(float(w_hat[i]), 3) == pytest.approx(r[3], abs=1e-9)
        assert round(float(w[i] - w_hat[i]), 3) == pytest.approx(r[4], abs=1e-9)
    err = np.abs(w - w_hat)
    assert round(float(err.mean()), 3) == float(kv["mean_abs_error"][0])
    assert round(float(scale / 2), 3) == float(kv["half_step"][0])
    assert err.max() <= scale / 2


def test_outlier_block_matches_page():
    kv, _ = _read_golden("int4_outlier_block.txt")
    w = np.array([float(v) for v in kv["w"]], np.float32)
    _, scale0, _ = O.absmax_int_quantize(np.array(
        [0.42, -0.31, 0.07, -0.18, 0.55, -0.44, 0.12, -0.09], np.float32), bits=4)
    q, scale, w_hat = O.absmax_int_quantize(w, bits=4)
    assert round(float(scale), 3) == float(kv["scale"][0])
    assert round(float(np.abs(w - w_hat).mean()), 3) == float(kv["mean_abs_error"][0])
    assert round(float(scale / scale0), 1) == float(kv["coarser_ratio"][0])


@pytest.mark.parametrize("bits", [4, 8])
def test_int_grid_error_at_most_half_step(bits):
    # "QLoRA" (learning-llms page), the paragraph after the absmax equation:
    # rounding to the grid moves each weight by no more than half a step
    for seed in range(10):
        w = inputs.normal((64,), 1.0, seed, dtype=torch.float32).numpy()
        q, scale, w_hat = O.absmax_int_quantize(w, bits=bits)
        assert np.all(np.abs(w - w_hat) <= scale / 2 * (1 + 1e-6))
        assert q.max() <= 2 ** (bits - 1) - 1 and q.min() >= -(2 ** (bits - 1))


def test_int4_widget_statistics_and_spread():
    kv, _ = _read_golden("int4_widget.txt")
    n = int(float(kv["n_weights"][0]))
    means, worsts, ratios = [], [], []
    for seed in range(20):
        w = inputs.normal((n,), 1.0, seed, dtype=torch.float32).numpy()
        _, s4, h4 = O.absmax_int_quantize(w, bits=4)
        _, s8, h8 = O.absmax_int_quantize(w, bits=8)
        e4, e8 = np.abs(w - h4), np.abs(w - h8)
        assert e4.max() <= s4 / 2 * (1 + 1e-6)
        means.append(e4.mean())
        worsts.append(e4.max())
        ratios.append(e4.mean() / e8.mean())
    # statistical consistency with the widget's sample (its values are not printed)
    assert abs(np.mean(means) - float(kv["mean_abs_error"][0])) < 0.012
    assert abs(np.mean(worsts) - float(kv["worst_error"][0])) < 0.03
    # the page puts the int4 error spread at about 18x the int8 one: the step ratio is 127/7 exactly; measured mean-error ratio near it
    assert round(127 / 7) == int(float(kv["int4_vs_int8_spread"][0]))
    assert abs(np.mean(ratios) - 127 / 7) < 1.5


# ------------------------------------------------------------ NF4 codebook

def test_nf4_codebook_construction_independent_routine():
    from scipy.special import ndtri  # a second, independent inverse normal CDF
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    pos = ndtri(np.linspace(delta, 0.5, 9)[:8])
    neg = -ndtri(np.linspace(delta, 0.5, 8)[:7])
    ref = np.sort(np.concatenate([pos, neg, [0.0]]))
    ref = (ref / np.abs(ref).max()).astype(np.float32)
    lv = O.nf4_levels()
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(lv - ref) <= ulp)


def test_nf4_codebook_invariants():
    lv = O.nf4_levels().astype(np.float64)
    assert len(set(lv.tolist())) == 16                     # all 16 codes used
    assert np.all(np.diff(lv) > 0)                         # sorted
    assert lv[0] == -1.0 and lv[15] == 1.0 and lv[7] == 0.0
    assert (lv > 0).sum() == 8 and (lv < 0).sum() == 7
    gaps = np.diff(lv)
    # dense near zero, sparse in the tails: gaps grow away from zero on each side
    assert np.all(np.diff(gaps[7:]) > 0)                   # positive side
    assert np.all(np.diff(gaps[:7]) < 0)                   # negative side


def test_nf4_nearest_is_optimal_with_lower_tie():
    lv = O.nf4_levels().astype(np.float64)
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.uniform(-1.05, 1.05, 4000), lv, -lv]).astype(np.float32)
    for x in xs:
        c = O.nf4_nearest(float(x))
        d = np.abs(float(x) - lv)
        assert d[c] == d.min()
        assert c == int(np.argmin(d))                      # first minimum = lower code
    # exact midpoints that binary32 can hold: the tie goes to the lower code
    for i in range(15):
        m = (lv[i] + lv[i + 1]) / 2
        if float(np.float32(m)) == m:
            assert O.nf4_nearest(float(m)) == i
        up = float(np.nextafter(np.float32(m), np.float32(2)))
        dn = float(np.nextafter(np.float32(m), np.float32(-2)))
        if up > m:
            assert O.nf4_nearest(up) == i + 1
        if dn < m:
            assert O.nf4_nearest(dn) == i


def test_nf4_lower_error_than_uniform_grids():
    kv, _ = _read_golden("int4_widget.txt")
    lv = O.nf4_levels().astype(np.float64)
    red = []
    for seed in range(20):   # one absmax for 2,048 N(0,1) weights, as in the widget
        w = inputs.normal((2048,), 1.0, 100 + seed, dtype=torch.float32).numpy()
        am = np.abs(w).max()
        codes = np.array([O.nf4_nearest(float(np.float32(v / am))) for v in w])
        e_nf4 = np.abs(w - lv[codes] * am).mean()
        _, _, h4 = O.absmax_int_quantize(w, bits=4)
        red.append(1 - e_nf4 / np.abs(w - h4).mean())
    r = float(np.mean(red))
    assert abs(r - float(kv["nf4_error_reduction"][0])) < 0.06, r
    # 64-weight blocks of N(0, 0.02): NF4 beats int4 and a linspace(-1, 1, 16) grid
    W = inputs.normal((64, 1024), 0.02, 7, dtype=torch.float32).numpy()
    q = O.nf4_quantize(W, double_quant=False)
    w_nf4 = O.bf16_to_f32(O.nf4_dequantize(q)).astype(np.float64)
    blocks = W.reshape(-1, 64).astype(np.float64)
    am = np.abs(blocks).max(axis=1, keepdims=True)
    lin = np.linspace(-1, 1, 16)
    nearest_lin = lin[np.abs(blocks[..., None] / am[..., None] - lin).argmin(-1)] * am
    int4 = np.clip(np.rint(blocks / (am / 7)), -8, 7) * (am / 7)
    e_nf4 = np.abs(W.astype(np.float64) - w_nf4).mean()
    assert e_nf4 < np.abs(blocks - int4).mean()
    assert e_nf4 < np.abs(blocks - nearest_lin).mean()


# ------------------------------------------------------- NF4 storage format

def test_pack_order_hand_example():
    kv, _ = _read_golden("nf4_pack_example.txt")
    want = bytes(int(b, 16) for b in kv["bytes"])
    lv = O.nf4_levels()
    w = np.tile(lv, 4).reshape(1, 64).astype(np.float32)
    q = O.nf4_quantize(w, double_quant=True)
    assert q["codes"].tobytes() == want
    assert q["absmax"][0] == 1.0 and q["q8"][0] == 255
    assert q["s2"][0] == np.float32(1.0) / np.float32(255.0)


def test_zero_block_and_tiny_block():
    w = np.zeros((2, 128), np.float32)
    w[1, 64:] = np.float32(1e-40)            # a subnormal absmax counts as a zero block
    w[1, :64] = inputs.normal((64,), 0.02, 1, dtype=torch.float32).numpy()
    q = O.nf4_quantize(w, double_quant=True)
    assert np.all(q["codes"][0] == 0x77)
    assert np.all(q["codes"][1, 32:] == 0x77)
    deq = O.bf16_to_f32(O.nf4_dequantize(q))
    assert np.all(deq[0] == 0) and np.all(deq[1, 64:] == 0)
    allzero = O.nf4_quantize(np.zeros((1, 256), np.float32))
    assert np.all(allzero["q8"] == 0) and allzero["s2"][0] == 0


def test_nonfinite_rejected():
    for bad in (np.inf, -np.inf, np.nan):
        w = np.zeros((1, 64), np.float32)
        w[0, 5] = bad
        with pytest.raises(O.OracleError):
            O.nf4_quantize(w)


def test_double_quant_bounds_and_group_layout():
    # K = 11008 gives 172 blocks per row, so 256-block groups straddle rows
    W = inputs.weight((6, 11008), 0.02, 11, dtype=torch.float32, outlier_frac=1e-3).numpy()
    q = O.nf4_quantize(W, double_quant=True)
    blocks = W.reshape(-1, 64)
    am = np.abs(blocks).max(axis=1)
    assert np.array_equal(q["absmax"], am)
    groups = (len(am) + 255) // 256
    assert len(q["s2"]) == groups
    for g in range(groups):
        seg = slice(g * 256, min((g + 1) * 256, len(am)))
        m = am[seg].max()
        assert q["s2"][g] == np.float32(m) / np.float32(255)
        assert q["q8"][seg].max() == 255
        rec = q["q8"][seg].astype(np.float64) * float(q["s2"][g])
        assert np.all(np.abs(rec - am[seg]) <= float(q["s2"][g]) * (0.5 + 1e-5))


def test_dequant_special_values_and_error_bound():
    W = inputs.weight((32, 512), 0.02, 12, dtype=torch.float32).numpy()
    lv = O.nf4_levels().astype(np.float64)
    for dq in (False, True):
        q = O.nf4_quantize(W, double_quant=dq)
        deq = O.bf16_to_f32(O.nf4_dequantize(q)).astype(np.float64).reshape(-1, 64)
        codes = np.stack([q["codes"] & 0xF, q["codes"] >> 4], -1).reshape(-1, 64)
        assert np.all(deq[codes == 7] == 0)
        if dq:
            scale = (q["q8"].astype(np.float32) * q["s2"][np.arange(len(q["q8"])) // 256]
                     ).astype(np.float64)
        else:
            scale = q["absmax"].astype(np.float64)
        blocks = W.reshape(-1, 64).astype(np.float64)
        # the element that sets the absmax decodes to +-scale (levels +-1), in bf16
        idx = np.abs(blocks).argmax(axis=1)
        top = deq[np.arange(len(idx)), idx]
        want = np.sign(blocks[np.arange(len(idx)), idx]) * O.bf16_to_f32(
            O.f32_to_bf16(scale.astype(np.float32))).astype(np.float64)
        assert np.array_equal(top, want)
        if not dq:
            # nearest-level error bound: half the local gap times absmax, plus bf16 rounding
            gap = np.diff(lv).max()
            bound = gap / 2 * scale[:, None] * (1 + 1e-6) + np.abs(deq) * 2.0 ** -8
            assert np.all(np.abs(blocks - deq) <= bound)


def test_bf16_rounding_against_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8,
                                  3.3895314e38, 1e-40, 0.0, -0.0], np.float32)])
    mine = O.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_storage_sizes_closed_form():
    kv, _ = _read_golden("storage_overhead.txt")
    g = lambda k: float(kv[k][0])
    for N, K in [(256, 512), (4096, 4096), (11008, 4096), (4096, 11008), (28672, 8192)]:
        c, a, s = O.nf4_sizes(N, K, True)
        assert c == N * K // 2 and a == N * K // 64
        assert s == 4 * math.ceil(N * K / 64 / 256)
        c0, a0, s0 = O.nf4_sizes(N, K, False)
        assert a0 == 4 * N * K // 64 and s0 == 0
    N = K = 4096
    c, a, s = O.nf4_sizes(N, K, True)
    bits = 8 * (c + a + s) / (N * K)
    c0, a0, _ = O.nf4_sizes(N, K, False)
    bits0 = 8 * (c0 + a0) / (N * K)
    assert round(bits - 4, 3) == g("overhead_dq_bits")
    assert bits0 - 4 == g("overhead_fp32_bits") and bits0 == g("total_fp32_bits")
    assert round(bits0 / 8, 2) == g("total_fp32_bytes")
    assert round(bits, 2) == g("total_dq_bits")
    assert round(bits / 8, 2) == g("total_dq_bytes")
    assert round(bits0 - bits, 2) == g("saved_bits")
    assert round(65e9 * (bits0 - bits) / 8 / 1e9) == g("saved_65b_gb")
    assert 8 * a / (N * K) == g("overhead_dq_bits_without_group_scale")


# --------------------------------------------------- linear layer identities

def _small_problem(seed=0, M=12, N=40, K=128, r=8):
    wl = inputs.SINGLE
    W = inputs.weight((N, K), 0.02, seed, dtype=torch.float32).numpy()
    q = O.nf4_quantize(W)
    Wh = O.nf4_dequantize(q)
    X = inputs.normal((M, K), 1.0, seed + 1).view(torch.int16).numpy().view(np.uint16)
    dY = inputs.normal((M, N), 1.0, seed + 2).view(torch.int16).numpy().view(np.uint16)
    A = inputs.normal((r, K), 0.01, seed + 3).view(torch.int16).numpy().view(np.uint16)
    B = inputs.normal((N, r), 0.01, seed + 4).view(torch.int16).numpy().view(np.uint16)
    return X, Wh, A, B, dY, wl.alpha, r


def test_linear_backward_matches_autograd():
    X, Wh, A, B, dY, alpha, r = _small_problem()
    f = lambda a: torch.from_numpy(O.bf16_to_f32(a).astype(np.float64))
    Xt, Wt, At, Bt, dYt = (f(v) for v in (X, Wh, A, B, dY))
    Xt.requires_grad_(True); At.requires_grad_(True); Bt.requires_grad_(True)
    s = alpha / r
    Y = torch.nn.functional.linear(Xt, Wt) + s * torch.nn.functional.linear(
        torch.nn.functional.linear(Xt, At), Bt)
    (Y * dYt).sum().backward()
    Yo, _ = O.linear_fwd(X, Wh, A, B, alpha, r)
    g = O.linear_bwd(dY, X, Wh, A, B, alpha, r)
    assert np.allclose(Yo, Y.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(g["dX"], Xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(g["dA"], At.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dB"], Bt.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_linear_finite_differences():
    X, Wh, A, B, dY, alpha, r = _small_problem(seed=5, M=6, N=16, K=64, r=4)
    x, w, a, b, dy = (O.bf16_to_f32(v).astype(np.float64) for v in (X, Wh, A, B, dY))
    g = O.linear_bwd(dy, x, w, a, b, alpha, r)
    loss = lambda x_, a_, b_: float((O.linear_fwd(x_, w, a_, b_, alpha, r)[0] * dy).sum())
    h = 1e-6
    rng = np.random.default_rng(1)
    for _ in range(6):
        i, k = rng.integers(0, a.shape[0]), rng.integers(0, a.shape[1])
        ap, am = a.copy(), a.copy(); ap[i, k] += h; am[i, k] -= h
        assert (loss(x, ap, b) - loss(x, am, b)) / (2 * h) == pytest.approx(g["dA"][i, k], rel=1e-6, abs=1e-9)
        n, j = rng.integers(0, b.shape[0]), rng.integers(0, b.shape[1])
        bp, bm = b.copy(), b.copy(); bp[n, j] += h; bm[n, j] -= h
        assert (loss(x, a, bp) - loss(x, a, bm)) / (2 * h) == pytest.approx(g["dB"][n, j], rel=1e-6, abs=1e-9)
        m, k2 = rng.integers(0, x.shape[0]), rng.integers(0, x.shape[1])
        xp, xm = x.copy(), x.copy(); xp[m, k2] += h; xm[m, k2] -= h
        assert (loss(xp, a, b) - loss(xm, a, b)) / (2 * h) == pytest.approx(g["dX"][m, k2], rel=1e-6, abs=1e-9)


def test_linear_special_cases():
    X, Wh, A, B, dY, alpha, r = _small_problem(seed=9)
    x = O.bf16_to_f32(X).astype(np.float64)
    w = O.bf16_to_f32(Wh).astype(np.float64)
    # B = 0: plain frozen-base GEMM (torch's linear as the second routine)
    Y0, _ = O.linear_fwd(X, Wh, A, np.zeros_like(B), alpha, r)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(w)).numpy()
    assert np.allclose(Y0, ref, rtol=1e-13, atol=1e-13)
    # alpha = 0: no adapter contribution
    Ya, _ = O.linear_fwd(X, Wh, A, B, 0.0, r)
    assert np.allclose(Ya, ref, rtol=1e-13, atol=1e-13)
    # all codes 7: the dequantised base is exactly zero and only the adapter remains
    q = O.nf4_quantize(np.zeros((Wh.shape[0], Wh.shape[1]), np.float32))
    Wz = O.nf4_dequantize(q)
    assert np.all(Wz == 0)
    Yz, T = O.linear_fwd(X, Wz, A, B, alpha, r)
    b = O.bf16_to_f32(B).astype(np.float64)
    assert np.allclose(Yz, alpha / r * (T @ b.T), rtol=1e-13, atol=1e-15)


def test_linear_backward_is_linear_in_dY():
    X, Wh, A, B, dY, alpha, r = _small_problem(seed=13)
    dy1 = O.bf16_to_f32(dY).astype(np.float64)
    dy2 = np.roll(dy1, 3, axis=1)
    g1 = O.linear_bwd(dy1, X, Wh, A, B, alpha, r)
    g2 = O.linear_bwd(dy2, X, Wh, A, B, alpha, r)
    g3 = O.linear_bwd(2.0 * dy1 - 0.5 * dy2, X, Wh, A, B, alpha, r)
    for k in ("dX", "dA", "dB"):
        assert np.allclose(g3[k], 2.0 * g1[k] - 0.5 * g2[k], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- Adam step
# The pages fix only Adam's precision (fp32 state, 12 bytes per adapter
# parameter); the update is Adam as published.  Pins: its closed forms and
# an independent implementation (torch.optim.AdamW in binary64).

def test_adam_first_step_is_signed_step_of_lr():
    # from zero moments the bias-corrected moments are g and g^2 exactly, so
    # the first step moves every parameter by lr * g / (|g| + eps)
    rng = np.random.default_rng(1)
    theta, g = rng.normal(size=257), rng.normal(size=257) * 1e-3
    z = np.zeros(257)
    lr, eps = 1e-3, 1e-8
    t1, m, v = O.adam_step(theta, z, z, g, 1, lr, 0.9, 0.999, eps)
    assert np.allclose(t1, theta - lr * g / (np.abs(g) + eps), rtol=0, atol=1e-15)
    assert np.allclose(m, 0.1 * g, rtol=1e-15) and np.allclose(v, 0.001 * g * g, rtol=1e-12)


def test_adam_constant_gradient_moves_linearly():
    # with a constant gradient the bias corrections undo the averages exactly:
    # every step is the same lr * g / (|g| + eps)
    rng = np.random.default_rng(2)
    theta0, g = rng.normal(size=64), rng.normal(size=64)
    theta, m, v = theta0, np.zeros(64), np.zeros(64)
    lr, eps = 2e-3, 1e-6
    for t in range(1, 11):
        theta, m, v = O.adam_step(theta, m, v, g, t, lr, 0.8, 0.95, eps)
    assert np.allclose(theta, theta0 - 10 * lr * g / (np.abs(g) + eps), rtol=0, atol=1e-12)


def test_adam_decoupled_decay_alone_is_geometric():
    theta0 = np.linspace(-2.0, 2.0, 33)
    theta, m, v = theta0, np.zeros(33), np.zeros(33)
    lr, wd = 1e-2, 0.1
    for t in range(1, 6):
        theta, m, v = O.adam_step(theta, m, v, np.zeros(33), t, lr, 0.9, 0.999, 1e-8, weight_decay=wd)
    assert np.allclose(theta, theta0 * (1 - lr * wd) ** 5, rtol=1e-14, atol=0)


def test_adam_is_gradient_scale_invariant_without_eps():
    rng = np.random.default_rng(3)
    theta, g1, g2 = rng.normal(size=50), rng.normal(size=50), rng.normal(size=50)
    z = np.zeros(50)
    a = O.adam_step(*O.adam_step(theta, z, z, g1, 1, 1e-3, 0.9, 0.99, 0.0)[:3], g2, 2, 1e-3, 0.9, 0.99, 0.0)
    b = O.adam_step(*O.adam_step(theta, z, z, g1, 1, 1e-3, 0.9, 0.99, 0.0, grad_scale=64.0)[:3], g2, 2, 1e-3,
                    0.9, 0.99, 0.0, grad_scale=64.0)
    assert np.allclose(a[0], b[0], rtol=0, atol=1e-14)


def test_adam_matches_torch_adamw_in_binary64():
    rng = np.random.default_rng(4)
    n, lr, betas, eps, wd = 300, 3e-3, (0.85, 0.97), 1e-7, 0.05
    theta0 = rng.normal(size=n)
    grads = [rng.normal(size=n) for _ in range(6)]
    p = torch.nn.Parameter(torch.tensor(theta0, dtype=torch.float64))
    opt = torch.optim.AdamW([p], lr=lr, betas=betas, eps=eps, weight_decay=wd)
    theta, m, v = theta0, np.zeros(n), np.zeros(n)
    for t, g in enumerate(grads, start=1):
        p.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        theta, m, v = O.adam_step(theta, m, v, g, t, lr, betas[0], betas[1], eps, weight_decay=wd)
    st = opt.state[p]
    assert np.allclose(theta, p.detach().numpy(), rtol=0, atol=1e-13)
    assert np.allclose(m, st["exp_avg"].numpy(), rtol=0, atol=1e-15)
    assert np.allclose(v, st["exp_avg_sq"].numpy(), rtol=0, atol=1e-15)


# ------------------------------------------------------------- adapter merge

def _int_adapters(N, K, r, seed):
    """Small-integer adapters: every product and partial sum is exact in fp32."""
    rng = np.random.default_rng(seed)
    A = rng.integers(-4, 5, size=(r, K)).astype(np.float32)
    B = rng.integers(-4, 5, size=(N, r)).astype(np.float32)
    return O.f32_to_bf16(A), O.f32_to_bf16(B), A.astype(np.float64), B.astype(np.float64)


def test_merge_with_zero_adapter_is_the_dequantised_weight():
    rng = np.random.default_rng(21)
    W = (rng.normal(size=(16, 256)) * 0.02).astype(np.float32)
    q = O.nf4_quantize(W)
    r = 8
    A = O.f32_to_bf16(rng.normal(size=(r, 256)).astype(np.float32))
    Bz = np.zeros((16, r), np.uint16)
    merged = O.merge_nf4(q, A, Bz, 16.0, r)
    assert np.array_equal(merged, O.bf16_to_f32(O.nf4_dequantize(q)))


def test_merge_of_a_zero_weight_is_the_exact_adapter_product():
    # a zero weight dequantises to exact zeros (all codes 7), so with integer
    # adapters the merged weight is s (B A) exactly; B A is not symmetric, so
    # a transposed operand or a wrong index fails
    N, K, r = 24, 192, 8
    q = O.nf4_quantize(np.zeros((N, K), np.float32))
    A, B, a, b = _int_adapters(N, K, r, seed=22)
    merged = O.merge_nf4(q, A, B, 2.0 * r, r)
    assert np.array_equal(merged.astype(np.float64), 2.0 * (b @ a))
    merged = O.merge_nf4(q, A, B, 0.5 * r, r)       # s = 0.5
    assert np.array_equal(merged.astype(np.float64), 0.5 * (b @ a))


# --------------------------------------------------------------- LoRA dropout

def test_philox_matches_numpy_philox():
    # numpy's Philox (an independent implementation of Philox-4x64-10)
    # increments its 256-bit counter before each block, so its counter
    # c - 1 produces our block at counter c
    rng = np.random.default_rng(31)
    for _ in range(20):
        c = [int(rng.integers(1, 1 << 62)), int(rng.integers(0, 1 << 62)), int(rng.integers(0, 1 << 62)),
             int(rng.integers(0, 1 << 62))]
        k = [int(rng.integers(0, 1 << 62)), int(rng.integers(0, 1 << 62))]
        bg = np.random.Philox(key=np.array(k, dtype=np.uint64),
                              counter=np.array([c[0] - 1, c[1], c[2], c[3]], dtype=np.uint64))
        assert tuple(int(x) for x in bg.random_raw(4)) == O.philox4x64_10(c, k)


def test_philox_blocks_match_scalar_definition():
    rng = np.random.default_rng(32)
    c0 = rng.integers(0, 1 << 63, size=64, dtype=np.uint64)
    key = (int(rng.integers(0, 1 << 63)), int(rng.integers(0, 1 << 63)))
    got = O.philox4x64_10_blocks(c0, key)
    for i in range(64):
        assert tuple(int(x) for x in got[i]) == O.philox4x64_10((int(c0[i]), 0, 0, 0), key)


def test_dropout_cut_and_keep_rate():
    assert O.dropout_threshold(0.0) == 0
    assert O.dropout_threshold(0.5) == 1 << 31
    assert O.dropout_threshold(0.05) == 214748365          # ceil(0.05 * 2^32) = ceil(214748364.8)
    for p in (0.05, 0.5):
        keep = O.lora_dropout_keep(11, 512, 2048, p)
        n = keep.size
        sigma = math.sqrt(n * p * (1 - p))
        assert abs(keep.sum() - n * (1 - p)) <= 5 * sigma
    assert O.lora_dropout_keep(11, 64, 128, 0.0).all()


def test_dropout_mask_is_per_element_and_seeded():
    a = O.lora_dropout_keep(5, 40, 192, 0.3)
    b = O.lora_dropout_keep(5, 45, 192, 0.3)               # a taller matrix: same first rows
    assert np.array_equal(a, b[:40])
    flat = O.lora_dropout_keep(5, 1, 40 * 192, 0.3)        # element e = m K + k, whatever the shape
    assert np.array_equal(a.reshape(-1), flat.reshape(-1))
    assert not np.array_equal(a, O.lora_dropout_keep(6, 40, 192, 0.3))


def test_dropout_layer_without_dropout_is_the_plain_layer():
    X, Wh, A, B, dY, alpha, r = _small_problem(seed=41)
    keep = np.ones((X.shape[0], X.shape[1]), bool)
    Y0, T0 = O.linear_fwd(X, Wh, A, B, alpha, r)
    Y1, T1 = O.linear_fwd_dropout(X, Wh, A, B, alpha, r, keep, 0.0)
    assert np.allclose(Y1, Y0, rtol=1e-14, atol=1e-14) and np.allclose(T1, T0, rtol=1e-14, atol=1e-14)
    g0 = O.linear_bwd(dY, X, Wh, A, B, alpha, r)
    g1 = O.linear_bwd_dropout(dY, X, Wh, A, B, alpha, r, keep, 0.0)
    for k in ("dX", "dA", "dB"):
        assert np.allclose(g1[k], g0[k], rtol=1e-13, atol=1e-13)


def test_dropout_layer_gradients_by_central_differences():
    # with the mask fixed the layer is linear in X, A and B, so for the loss
    # L = <dY, Y> a central difference along any direction is exact up to
    # rounding; it checks every term of dX, dA, dB (mask, 1/(1-p), s)
    X, Wh, A, B, dY, alpha, r = _small_problem(seed=42)
    x, a, b, dy = (O.bf16_to_f32(t).astype(np.float64) for t in (X, A, B, dY))
    p = 0.3
    keep = O.lora_dropout_keep(9, x.shape[0], x.shape[1], p)
    g = O.linear_bwd_dropout(dy, x, Wh, a, b, alpha, r, keep, p)
    loss = lambda xx, aa, bb: float(np.sum(dy * O.linear_fwd_dropout(xx, Wh, aa, bb, alpha, r, keep, p)[0]))
    rng = np.random.default_rng(43)
    h = 1e-3
    for name, base, grad in (("dX", x, g["dX"]), ("dA", a, g["dA"]), ("dB", b, g["dB"])):
        D = rng.normal(size=base.shape)
        args = {"dX": lambda e: (x + e * D, a, b), "dA": lambda e: (x, a + e * D, b),
                "dB": lambda e: (x, a, b + e * D)}[name]
        fd = (loss(*args(h)) - loss(*args(-h))) / (2 * h)
        assert abs(fd - float(np.sum(grad * D))) <= 1e-8 * max(1.0, abs(fd)), name


# ------------------------------------------------ FP8 second-level scales

def test_e4m3_encoder_matches_torch_float8():
    # torch's float8_e4m3fn conversion (independent) rounds to nearest even;
    # it agrees with the saturating encoder everywhere up to 464
    vals = O.e4m3_values()
    mids = (vals[1:] + vals[:-1]) / 2
    rng = np.random.default_rng(51)
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rng.uniform(0, 460, 2000), rng.uniform(0, 1e-2, 500)]).astype(np.float32)
    x = x[x <= 460]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), ref)


def test_e4m3_codebook_and_saturation():
    v = O.e4m3_values()
    assert v[0] == 0 and v[1] == 2.0 ** -9 and v[126] == 448.0 and v[56] == 1.0
    assert np.all(np.diff(v) > 0)
    assert O.e4m3_encode(np.array([448.0, 470.0, 1e6], np.float32)).tolist() == [126, 126, 126]


def test_fp8_scales_sizes_and_error_bound():
    rng = np.random.default_rng(52)
    w = (rng.normal(size=(64, 1024)) * 0.02).astype(np.float32)
    q = O.nf4_quantize_fp8(w)
    blocks = w.size // 64
    assert q["q8"].size == blocks and q["s2"].size == -(-blocks // 256)
    bits = (8 * blocks + 32 * q["s2"].size) / w.size            # second-level cost per weight
    assert abs(bits - (0.125 + 32 / 16384)) < 1e-12              # BEA's 0.125 plus the group scales
    ref = O.nf4_quantize(w, double_quant=False)
    assert np.array_equal(q["codes"], ref["codes"])             # codes from the fp32 absmax
    rec = (O.e4m3_values()[q["q8"]] * np.repeat(q["s2"], 256)[:blocks]).astype(np.float32)
    a = ref["absmax"].astype(np.float64)
    # E4M3 keeps 3 mantissa bits: <= 2^-4 relative in the normal range (the
    # group scale puts the largest absmax at 448, so blocks within 2^14 of it
    # stay normal)
    normal = a >= a.max() * 2.0 ** -14
    assert np.all(np.abs(rec[normal] - a[normal]) <= 2.0 ** -4 * a[normal] * (1 + 1e-6))


def test_fp8_dequantise_uses_the_reconstructed_absmax():
    w = np.zeros((4, 512), np.float32)
    w[1, 70] = 0.5; w[2, 300] = -0.25
    q = O.nf4_quantize_fp8(w)
    Wh = O.bf16_to_f32(O.nf4_dequantize_fp8(q))
    # a block whose absmax is the group maximum reconstructs it exactly
    # (448 * m / 448 rounds back to m) and its extreme weight is +-absmax
    assert Wh[1, 70] == 0.5 and Wh[2, 300] == -0.25
    assert np.all(Wh[0] == 0) and np.all(Wh[3] == 0)
    z = O.nf4_quantize_fp8(np.zeros((2, 256), np.float32))
    assert np.all(z["s2"] == 0) and np.all(z["q8"] == 0)
