#!/usr/bin/env python3
"""Fits the polynomial that rf_exp2_poly (rf_device.cuh) uses for 2^r on [-1/2, 1/2].

Method: minimise the maximum RELATIVE error |p(r) / 2^r - 1| over r in
[-1/2, 1/2] with p(0) = 1 enforced (so that exact powers of two stay exact),
by a discrete Remez exchange started from a weighted least-squares fit on a
dense grid.  Together with the range reduction x = j + r (j = round(x), via
adding 1.5 * 2^23) and the exponent reassembly 2^x = p(r) * 2^j (an integer
add on the bit pattern) this gives 2^x on the FMA/ALU pipes.

Run:  python gen_exp2_poly.py [degree]   (prints the coefficients and the
error bound; the constants in rf_device.cuh were produced by degree 3).
"""
import sys

import numpy as np


def fit(deg: int, grid: int = 20001, iters: int = 30):
    r = np.linspace(-0.5, 0.5, grid)
    f = np.exp2(r)
    # p(r) = 1 + sum_{k=1..deg} c_k r^k; relative error e = (p - f) / f
    A = np.stack([r ** k / f for k in range(1, deg + 1)], axis=1)
    b = (f - 1.0) / f
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    best_c, best_e = c, float(np.max(np.abs(A @ c - b)))
    # Remez exchange on the (linear in c) relative error; the reference starts
    # at the alternating extrema of the least-squares error.
    err = A @ c - b
    for _ in range(iters):
        sign = np.sign(err)
        idx, start = [], 0
        for i in range(1, grid + 1):
            if i == grid or sign[i] != sign[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = i
        idx = np.array(idx)
        if len(idx) < deg + 1:
            break
        s0 = max(range(len(idx) - deg), key=lambda t: np.min(np.abs(err[idx[t:t + deg + 1]])))
        ref = idx[s0:s0 + deg + 1]
        M = np.concatenate([A[ref], ((-1.0) ** np.arange(deg + 1))[:, None]], axis=1)
        c = np.linalg.solve(M, b[ref])[:-1]
        err = A @ c - b
        e = float(np.max(np.abs(err)))
        if e < best_e:
            best_c, best_e = c, e
    c = best_c
    err = A @ c - b
    return np.concatenate([[1.0], c]), float(np.max(np.abs(err)))


def eval_f32(coef, x):
    """fp32 evaluation exactly as the kernel does it (Horner with fused multiply-add)."""
    x = np.asarray(x, dtype=np.float32)
    x = np.maximum(x, np.float32(-127.0))
    shifter = np.float32(12582912.0)             # 1.5 * 2^23: adding it rounds to an integer
    t = (x + shifter).astype(np.float32)
    j = t.view(np.int32) - np.float32(shifter).view(np.int32)
    r = (x - (t - shifter)).astype(np.float32)
    p = np.float32(coef[-1])
    for ck in coef[-2::-1]:
        p = (p.astype(np.float64) * r + np.float32(ck)).astype(np.float32)   # fma, one rounding
    bits = p.view(np.int32) + (j << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef, e = fit(deg)
    print(f"degree {deg}: max relative error of the real-coefficient fit {e:.3e}")
    c32 = [float(np.float32(c)) for c in coef]
    print("coefficients (float32, c0..c%d):" % deg)
    for k, c in enumerate(c32):
        print(f"  c{k} = {c!r}f  ({np.float32(c).view(np.uint32):#010x})")
    xs = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    got = eval_f32(c32, xs).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.max(np.abs(got / ref - 1.0))
    print(f"fp32 evaluation over [-126, 8]: max relative error {rel:.3e}")
