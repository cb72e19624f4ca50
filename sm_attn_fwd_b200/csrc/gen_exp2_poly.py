"""Derive the polynomial used for exp2 on the FMA pipe (attn_prefill.cu).

exp2(x) = 2^n * 2^r with n = round(x) and r = x - n in [-1/2, 1/2].  2^r is
approximated by q(r) = 1 + r*(c1 + r*(c2 + r*c3)): the constant term is fixed
at 1 so that integer arguments (in particular x = 0 at the row maximum) are
exact.  c1..c3 minimise the maximum RELATIVE error |q(r)/2^r - 1| on
[-1/2, 1/2].  With q(r) = 1 + r*g(r), this is a weighted minimax problem for
g(r) ~ (2^r - 1)/r with weight |r| / 2^r, solved by the Remez exchange
(written here from the textbook algorithm: solve for an equioscillating error
on a reference set, move the reference to the error's extrema, repeat).  The
coefficients are then rounded to float32 and the float32 error re-measured.

Run:  python sm_attn_fwd_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

LO, HI = -0.5, 0.5


def g(x):
    return np.where(np.abs(x) < 1e-12, np.log(2.0), np.expm1(x * np.log(2.0)) / np.where(x == 0, 1, x))


def weight(x):
    return np.abs(x) / np.exp2(x)


def rel_err(coef, x):
    q = 1.0 + x * np.polyval(coef[::-1], x)
    return q / np.exp2(x) - 1.0


def remez(deg=2, iters=40):
    n = deg + 2
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (k[::-1] + 0.5) / n)
    coef = None
    xs = np.linspace(LO, HI, 400001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) / weight(x)
        sol = np.linalg.solve(A, g(ref))
        coef = sol[:deg + 1]
        err = rel_err(coef, xs)
        # extrema of the relative error between its zeros (r = 0 is always a zero)
        sign = np.sign(err)
        sign[sign == 0] = 1
        cuts = np.nonzero(np.diff(sign))[0] + 1
        bounds = np.concatenate([[0], cuts, [len(xs)]])
        ext = [xs[lo + np.argmax(np.abs(err[lo:hi]))] for lo, hi in zip(bounds[:-1], bounds[1:])
               if hi > lo]
        ext = sorted(ext, key=lambda e: -abs(rel_err(coef, np.array([e]))[0]))[:n]
        ext = np.sort(np.array(ext))
        if len(ext) < n or np.allclose(ext, ref):
            break
        ref = ext
    return coef, np.abs(rel_err(coef, xs)).max()


def f32_q(c32, r):
    """q(r) in float32 with fused multiply-adds, as the kernel evaluates it."""
    r = r.astype(np.float32)
    q = np.float32(c32[2])
    for c in (c32[1], c32[0], np.float32(1.0)):
        q = (np.float64(q) * np.float64(r) + np.float64(c)).astype(np.float32)
    return q


def main():
    coef, err = remez()
    c32 = np.array(coef, dtype=np.float32)  # c1, c2, c3
    r = np.linspace(LO, HI, 2000001)
    rel32 = np.abs(f32_q(c32, r).astype(np.float64) / np.exp2(r) - 1).max()
    print("q(r) = 1 + r*(c1 + r*(c2 + r*c3)) on [-1/2, 1/2]")
    print("minimax relative error (exact coefficients): %.3e" % err)
    print("max relative error, float32 coefficients and FMA: %.3e" % rel32)
    for i, c in enumerate(c32, start=1):
        print(f"  c{i} = {float(c):.9e}f  (0x{np.float32(c).view(np.uint32):08x})")


if __name__ == "__main__":
    main()
