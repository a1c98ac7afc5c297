"""Low-rank adapter fixtures built the way the pages describe -- TEST INFRASTRUCTURE.

Quant Experts (MCISLAB DeepRead summary), Method, Shared Expert: the layer
quantization error E = W_f - W_q gets a shared low-rank approximation,
following the low-rank reconstruction line of work. The remaining error goes
to the routed experts, one per cluster. The wispaper / longzhangge pages add
that the shared expert is fitted by whitening SVD. The objective is
min || (E - A_s B_s - A_r B_r) x ||.

Construction (fp64 numpy, plain):
  * the effective quantized weight seen by the raw input is
    W_q = dequant(codes, sw) / s (column-wise), so E = W - W_q, and the output
    error of token x is x E^T;
  * whitening: C = X^T X + lam*I = L L^T (Cholesky). Then ||X M||_F = ||L^T M||_F,
    so the rank-r minimiser of ||X (E^T - A B)||_F is A = L^{-T} U_r S_r,
    B = V_r^T from the SVD L^T E^T = U S V^T (Eckart-Young);
  * the shared expert is fitted on all calibration tokens. Routed expert c is
    fitted on the residual E^T - A_s B_s over the tokens routed to c.
"""
from __future__ import annotations

import numpy as np


def effective_quantized_weight(codes, scales, s, group: int) -> np.ndarray:
    """W_q [N,K] fp64 such that the quantized path equals (x/s) . dequant^T = x . W_q^T."""
    codes = np.asarray(codes, dtype=np.float64)
    scales = np.asarray(scales, dtype=np.float64)
    deq = codes * np.repeat(scales, group, axis=1)
    return deq / np.asarray(s, dtype=np.float64)[None, :]


def whitened_lowrank(M: np.ndarray, X: np.ndarray, r: int, ridge: float = 1e-9):
    """Rank-r (A [K,r], B [r,N]) minimising ||X (M - A B)||_F for M [K,N]."""
    X = np.asarray(X, dtype=np.float64)
    K = M.shape[0]
    C = X.T @ X
    lam = ridge * max(np.trace(C) / K, 1e-30)
    L = np.linalg.cholesky(C + lam * np.eye(K))
    Z = L.T @ M
    U, S, Vt = np.linalg.svd(Z, full_matrices=False)
    r = min(r, S.shape[0])
    A = np.linalg.solve(L.T, U[:, :r] * S[:r][None, :])
    B = Vt[:r, :]
    return A, B


def qe_adapters(W, codes, scales, s, group: int, X_calib, experts, rs: int, Nr: int, rr: int):
    """Shared + routed adapters of the pages' construction.

    experts [T_calib] gives each calibration token's cluster (the tokens a
    routed expert is fitted on). Returns fp64 A_s [K,rs], B_s [rs,N],
    A_r [Nr,K,rr], B_r [Nr,rr,N].
    """
    W = np.asarray(W, dtype=np.float64)
    X = np.asarray(X_calib, dtype=np.float64)
    E = W - effective_quantized_weight(codes, scales, s, group)
    Et = E.T
    A_s, B_s = whitened_lowrank(Et, X, rs)
    R = Et - A_s @ B_s
    K, N = Et.shape
    A_r = np.zeros((Nr, K, rr))
    B_r = np.zeros((Nr, rr, N))
    experts = np.asarray(experts)
    for c in range(Nr):
        Xc = X[experts == c]
        if Xc.shape[0] == 0:
            continue
        a, b = whitened_lowrank(R, Xc, rr)
        A_r[c, :, :a.shape[1]] = a
        B_r[c, :b.shape[0], :] = b
    return A_s, B_s, A_r, B_r


def reconstruction_errors(W, codes, scales, s, group, X, experts, A_s, B_s, A_r, B_r):
    """(sum_t ||E x_t||^2, sum_t ||(E - SE) x_t||^2, sum_t ||(E - SE - RE_e(t)) x_t||^2)."""
    W = np.asarray(W, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    Et = (W - effective_quantized_weight(codes, scales, s, group)).T
    e0 = X @ Et
    e1 = e0 - (X @ A_s) @ B_s
    e2 = e1.copy()
    for c in range(A_r.shape[0]):
        m = np.asarray(experts) == c
        if m.any():
            e2[m] -= (X[m] @ A_r[c]) @ B_r[c]
    return float((e0 ** 2).sum()), float((e1 ** 2).sum()), float((e2 ** 2).sum())
