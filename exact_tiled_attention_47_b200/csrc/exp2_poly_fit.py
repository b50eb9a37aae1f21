"""Derivation of the cubic used for 2^f, |f| <= 1/2, by the prefill softmax (exp2_poly_pair).

Remez exchange on the relative error of a degree-n polynomial against 2^f over [-1/2, 1/2]; prints
the coefficients and the maximum relative error before and after rounding them to float32 and
evaluating in float32 Horner form.  Degree 3 gives 7.5e-5, far below the 2^-9 rounding that P gets
when it is converted to bf16 for the P*V product.  Run: python exp2_poly_fit.py
"""
import numpy as np
def remez(deg, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    x = 0.5*(lo+hi) + 0.5*(hi-lo)*np.cos(np.pi*np.arange(n)[::-1]/(n-1))
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i,:deg+1] = x[i]**np.arange(deg+1) / f(x[i])
            A[i,deg+1] = (-1)**i
        sol = np.linalg.solve(A, np.ones(n))
        c, E = sol[:deg+1], sol[deg+1]
        t = np.linspace(lo, hi, 200001)
        err = np.polyval(c[::-1], t)/f(t) - 1
        # new extremal points: locate sign-alternating extrema
        idx = [0]
        for k in range(1, len(t)-1):
            if (err[k]-err[k-1])*(err[k+1]-err[k]) <= 0: idx.append(k)
        idx.append(len(t)-1)
        idx = np.array(idx)
        # pick n points with alternating signs and largest |err|
        pts = []
        for k in idx:
            if pts and np.sign(err[k]) == np.sign(err[pts[-1]]):
                if abs(err[k]) > abs(err[pts[-1]]): pts[-1] = k
            else: pts.append(k)
        while len(pts) > n:
            if abs(err[pts[0]]) < abs(err[pts[-1]]): pts.pop(0)
            else: pts.pop()
        if len(pts) == n: x = t[pts]
    return c, np.max(np.abs(err))
for d in (3,4,5):
    c, e = remez(d)
    c32 = c.astype(np.float32)
    t = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.zeros_like(t)
    for ci in c32[::-1]: p = (p*t + ci).astype(np.float32)
    e32 = np.max(np.abs(p.astype(np.float64)/np.exp2(t.astype(np.float64)) - 1))
    print(d, "max rel err (exact)", e, "float32 coeffs+horner", e32, [float(v) for v in c32], [hex(np.float32(v).view(np.uint32)) for v in c32])
