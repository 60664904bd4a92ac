"""Print the NF4 constants that nf4_constants.cuh holds as literals.

Levels: 16 normal quantiles normalised to [-1, 1] with an exact zero (the
QLoRA paper's construction, which the scalata.ai "QLoRA" page cites):
delta = 1 - (1/32 + 1/30)/2; Phi^-1 at the first 8 of 9 points evenly
spaced from delta to 0.5, minus Phi^-1 at the first 7 of 8 such points,
and 0; sorted and divided by the largest magnitude; binary64, rounded once
to binary32.  This generator uses scipy's ndtri for Phi^-1.

Thresholds: t_i = RD32((level_i + level_{i+1}) / 2), the midpoint (exact in
binary64) rounded toward -inf to binary32.  For a binary32 x,
x > t_i holds exactly when x lies strictly above the real midpoint, so
code(x) = #{i : x > t_i} is the nearest level with ties going to the lower
code.

Run:  python bit_nf4_quantized_21_b200/csrc/gen_nf4_constants.py
"""
import numpy as np
from scipy.special import ndtri


def levels() -> np.ndarray:
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    v = np.concatenate([ndtri(np.linspace(delta, 0.5, 9)[:8]),
                        -ndtri(np.linspace(delta, 0.5, 8)[:7]), [0.0]])
    v = np.sort(v)
    return (v / np.abs(v).max()).astype(np.float32)


def thresholds(lv: np.ndarray) -> np.ndarray:
    out = []
    for i in range(15):
        m = (float(lv[i]) + float(lv[i + 1])) / 2.0
        t = np.float32(m)
        if float(t) > m:
            t = np.nextafter(t, np.float32(-np.inf))
        out.append(t)
    return np.array(out, np.float32)


def main():
    lv = levels()
    th = thresholds(lv)
    print("// levels")
    for c, v in enumerate(lv):
        print(f"    {float(v).hex()}f,  // {c:2d}: {v:+.9f}")
    print("// thresholds")
    for i, v in enumerate(th):
        print(f"    {float(v).hex()}f,  // {i:2d}: {v:+.9f}")


if __name__ == "__main__":
    main()
