"""Derive the coefficients of the FMA-pipe exp2 used by the softmax.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2];
2^f is approximated by a polynomial c0 + c1 f + ... + cn f^n whose maximum
RELATIVE error on [-1/2, 1/2] is minimised (Remez exchange with weight
2^-f).  Two degrees are used: 3 in ``attn_fwd_kernel.cuh`` (bf16 weights,
error far below bf16 rounding) and 5 in ``attn_fwd_fp8_kernel.cuh`` (E4M3
weights: an error as small as the special-function unit's keeps rounding
flips at E4M3 boundaries as rare as with ex2.approx).  Run this file to
print the fp32 coefficients and the resulting error bounds:

    python tiled_attention_forward_sm_b200/csrc/gen_exp2_poly.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int = DEGREE, iters: int = 30):
    """Minimax polynomial for 2^f on [LO, HI] in relative error."""
    n = degree + 2  # reference points
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # Solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = ((-1) ** i) * (2.0 ** x[i])
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        idx = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            seg = np.abs(err[a:b])
            ext.append(a + int(np.argmax(seg)))
        if len(ext) != n:
            break
        x = grid[ext]
    return coef


X_MIN = -125.0  # inputs are clamped here so 2^j stays a normal exponent


def _fma32(a, b, c):  # a * b + c
    """fp32 fused multiply-add: the fp32 product is exact in fp64, so one
    rounding of the fp64 sum to fp32 models the hardware FMA."""
    return (a.astype(np.float64) * np.float64(b) + np.float64(c)).astype(np.float32)


def fp32_exp2_emulation(x: np.ndarray, c) -> np.ndarray:
    """Numpy model of the kernel's instruction sequence in fp32:
    x = max(x, -125); t = x + 1.5*2^23 (round to nearest); f = x - (t - 1.5*2^23);
    p = ((c3 f + c2) f + c1) f + c0 (FMAs); result bits = bits(p) + (bits(t) << 23)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(X_MIN))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c = [np.float32(v) for v in c]
    p = _fma32(f, c[-1], c[-2])
    for ck in reversed(c[:-2]):
        p = _fma32(f, p, ck)
    bits = p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23)
                                                   & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def main():
    for degree in (3, 5):
        c = remez_relative(degree)
        c32 = [float(np.float32(v)) for v in c]
        g = np.linspace(LO, HI, 1000001)
        rel = np.abs(np.polyval(np.array(c32)[::-1], g) / 2.0 ** g - 1.0)
        xs = np.linspace(X_MIN, 8.0, 2000001).astype(np.float32)
        emu = fp32_exp2_emulation(xs, c32).astype(np.float64)
        rel_emu = np.abs(emu / np.exp2(xs.astype(np.float64)) - 1.0)
        print(f"degree {degree}:")
        for i, v in enumerate(c32):
            print(f"  c{i} = {v!r}  ({np.float32(v).view(np.uint32):#010x})")
        print(f"  max relative error, polynomial on [-1/2,1/2]: {rel.max():.3e}")
        print(f"  max relative error, fp32 sequence on [{X_MIN:g}, 8]: {rel_emu.max():.3e}")


if __name__ == "__main__":
    main()
