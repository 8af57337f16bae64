"""Derive the polynomial used for part of the softmax exponentials in attention_sm100.cu.

2^x is split as 2^i * 2^f with i = round(x) and f = x - i in [-1/2, 1/2] (Cody and Waite's
argument reduction, W. J. Cody and W. Waite, "Software Manual for the Elementary Functions",
1980).  2^f is approximated by the degree-3 polynomial that minimises the maximum RELATIVE
error on [-1/2, 1/2], found with the Remez exchange algorithm (E. Ya. Remez, 1934): alternate
between solving for the coefficients that equioscillate on the current reference points and
moving the reference points to the extrema of the error, until the extrema are equal.

Run ``python pose_retrieved_kv_b200/csrc/gen_exp2_poly.py`` to print the coefficients (float32,
c0..c3) and the achieved maximum relative error; the values are pasted into the kernel.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # initial reference: Chebyshev extrema mapped to [LO, HI]
    k = np.arange(n)
    x = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve sum_j c_j x_i^j - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillation)
        A = np.zeros((n, n))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * f(x)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        # new reference: extrema of the relative error between sign changes
        t = np.linspace(LO, HI, 200001)
        err = (np.polyval(c[::-1], t) - f(t)) / f(t)
        idx = [0]
        for i in range(1, len(t) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(t) - 1)
        cand = t[idx]
        # keep n alternating extrema of largest magnitude
        e = err[idx]
        groups, cur = [], [0]
        for i in range(1, len(cand)):
            if np.sign(e[i]) == np.sign(e[cur[-1]]):
                cur.append(i)
            else:
                groups.append(cur)
                cur = [i]
        groups.append(cur)
        pts = [max(g, key=lambda i: abs(e[i])) for g in groups]
        while len(pts) > n:
            # drop the smaller end
            if abs(e[pts[0]]) < abs(e[pts[-1]]):
                pts = pts[1:]
            else:
                pts = pts[:-1]
        if len(pts) == n:
            x = cand[pts]
    return c


def max_rel_error(c):
    t = np.linspace(LO, HI, 2000001)
    c32 = np.asarray(c, dtype=np.float32).astype(np.float64)
    return np.max(np.abs((np.polyval(c32[::-1], t) - np.exp2(t)) / np.exp2(t)))


if __name__ == "__main__":
    c = remez()
    c32 = np.asarray(c, dtype=np.float32)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c32):.3e}")
