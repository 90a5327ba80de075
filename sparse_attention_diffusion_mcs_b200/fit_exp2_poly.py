"""Derive the coefficients of the FMA-pipe exponential used by the group
scores kernel: p(f) ~ 2^f on f in [-1/2, 1/2], degree 5, chosen to minimise
the maximum relative error (Remez exchange on the relative-error
equioscillation condition, started from Chebyshev nodes).  Prints the
coefficients c0..c5 and the achieved maximum relative error in exact
arithmetic (fp64) and with the fp32 Horner evaluation the kernel performs.

    python -m sparse_attention_diffusion_mcs_b200.fit_exp2_poly
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    dense = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative error equioscillates)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], dense) - 2.0 ** dense) / 2.0 ** dense
        # new reference: the extremum of the error in each sign run
        s = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(s))[0] + 1, [len(dense)]))
        ext = [a + np.argmax(np.abs(err[a:b])) for a, b in zip(idx[:-1], idx[1:])]
        if len(ext) >= n:
            best = sorted(ext, key=lambda i: -abs(err[i]))[:n] if len(ext) > n else ext
            x = np.sort(dense[np.array(best)])
    return c, np.max(np.abs(err))


def horner_f32(c, f):
    f = np.float32(f)
    p = np.float32(c[-1])
    for ci in c[-2::-1]:
        p = np.float32(np.float32(p * f) + np.float32(ci))   # the kernel uses fmaf; this bounds it
    return p


if __name__ == "__main__":
    c, e = remez()
    c32 = np.float32(c)
    fs = np.linspace(LO, HI, 100001, dtype=np.float32)
    got = np.array([horner_f32(c32, f) for f in fs[::50]], dtype=np.float64)
    ref = 2.0 ** fs[::50].astype(np.float64)
    print("coefficients c0..c5 (fp32):", ", ".join(f"{float(v):.9e}" for v in c32))
    print(f"max relative error: exact {e:.3e}, fp32 Horner {np.max(np.abs(got - ref) / ref):.3e}")
