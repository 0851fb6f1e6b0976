"""Fits the polynomials the S6 kernels (s6_scan_impl.cuh) use:

* 2^f for |f| <= 1/2 (ex2_poly2): degree 5, 2.1e-7 relative error in fp32,
  the class of the MUFU ex2.approx instruction;
* log1p(e) / e for e in [0, 1] (softplus_f): degree 7, 3.4e-7 relative.

Remez exchange on the relative error, then the coefficients are rounded to
float32 and the error of float32 Horner evaluation is re-measured.

    python fit_polys.py
"""
import numpy as np
def remez(deg, a=-0.5, b=0.5, iters=30, f=lambda t: np.exp2(t)):
    n = deg + 2
    k = np.arange(n)
    x = 0.5*(a+b) + 0.5*(b-a)*np.cos(np.pi*k/(n-1))[::-1]
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)   (relative error)
        M = np.zeros((n, n)); 
        for i in range(n):
            M[i,:deg+1] = x[i]**np.arange(deg+1)
            M[i,deg+1] = (-1)**i * f(x[i])
        sol = np.linalg.solve(M, f(x))
        c, E = sol[:deg+1], sol[deg+1]
        t = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], t) - f(t))/f(t)
        # new extrema
        idx = [0]
        s = np.sign(err)
        ext = []
        # split into sign runs, take max |err| in each
        runs = np.split(np.arange(len(t)), np.where(np.diff(s) != 0)[0]+1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n: break
        # keep n largest alternating
        while len(ext) > n:
            # drop the smaller end
            if abs(err[ext[0]]) < abs(err[ext[-1]]): ext = ext[1:]
            else: ext = ext[:-1]
        x = t[ext]
    return c, np.max(np.abs(err))
for deg in (4,5,6):
    c, e = remez(deg)
    c32 = c.astype(np.float32)
    # emulate fp32 Horner with fma (use float64 fma then round: close enough)
    t = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.float32(c32[-1])
    for ci in c32[-2::-1]:
        p = (p.astype(np.float64)*t.astype(np.float64) + np.float64(ci)).astype(np.float32)
    e32 = np.max(np.abs(p.astype(np.float64)/np.exp2(t.astype(np.float64)) - 1))
    print(deg, 'minimax rel err %.3e, fp32 coeffs+Horner %.3e' % (e, e32))
    print('   coeffs (c0..cdeg):', ', '.join('%.9ef' % v for v in c32))

# log1p(e) / e on [0, 1]
g = lambda e: np.where(e == 0, 1.0, np.log1p(e) / np.where(e == 0, 1, e))
for deg in (7,):
    c, e = remez(deg, 0.0, 1.0, 40, g)
    c32 = c.astype(np.float32)
    t = np.linspace(0, 1, 200001).astype(np.float32)
    p = np.float32(c32[-1])
    for ci in c32[-2::-1]:
        p = (p.astype(np.float64)*t.astype(np.float64) + np.float64(ci)).astype(np.float32)
    val = (p.astype(np.float64)*t).astype(np.float32)
    ref = np.log1p(t.astype(np.float64)); m = ref > 0
    print('log1p', deg, 'minimax rel err %.3e, fp32 %.3e' % (e, np.max(np.abs(val[m]/ref[m]-1))))
    print('   coeffs (c0..cdeg):', ', '.join('%.9ef' % v for v in c32))
