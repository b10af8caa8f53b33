"""Oracle for the hierarchical butterfly factorization (TEST INFRASTRUCTURE
ONLY: imported by tests, the smoke check and the benchmark's CPU legs, never
by the product path).

What it follows: the taxoreview.com page's third abstract (hierarchical
butterfly factorization): a matrix is factored into sparse factors with butterfly supports
by recursively splitting it into two factors, each split a two-factor
fixed-support factorization, with exact recovery when the matrix is such a
product.  The page gives no formulas; the steps below are the plain reading
for KS supports, written from the structure of the product:

Two chainable KS factors, K1 of pattern (a1, b1, c1, d1) applied first and
K2 of pattern (a2, b2, c2, d2), with a2 = a1*b1 and d1 = c2*d2, multiply to
the KS pattern (a1, b1*b2, c1*c2, d2), and every entry of the product is one
product of two values:

    P[i1][l2][k1*b2 + k2][j1*c2 + j2] = V2[i1*b1 + k1][l2][k2][j2] * V1[i1][j2*d2 + l2][k1][j1].

So for each (i1, k1, j2, l2) the b2 x c1 block B[k2][j1] of P is the outer
product of a column of V2 and a row of V1: fitting the two factors to a
given P is, block by block, the best rank-one approximation of B, i.e. its
top singular triplet (Eckart-Young), split as sqrt(s) u and sqrt(s) v.

The butterfly of size 2^L has factors F_k = (2^(k-1), 2, 2, 2^(L-k)),
k = 1..L, F_1 applied first; the product of F_p..F_q is KS with pattern
(2^(p-1), 2^(q-p+1), 2^(q-p+1), 2^(L-q)), and splitting the range [p, q] at
r gives two chainable factors.  The hierarchy splits every range in the
middle, r = floor((p + q - 1) / 2), down to single factors.

numpy's SVD is the one library step.  Singular vectors have a sign each; the
oracle makes the largest-magnitude entry of v positive (first one on ties).
"""
from __future__ import annotations

import numpy as np


def butterfly_range_pattern(p: int, q: int, L: int):
    """KS pattern of the product of butterfly factors F_p .. F_q (1-based)."""
    return (2 ** (p - 1), 2 ** (q - p + 1), 2 ** (q - p + 1), 2 ** (L - q))


def rank_one(B: np.ndarray):
    """Best rank-one approximation of B: (s, u, v) with B ~ s u v^T, |u| = |v| = 1,
    the largest-|v| entry of v positive."""
    U, S, Vt = np.linalg.svd(B, full_matrices=False)
    u, s, v = U[:, 0], S[0], Vt[0]
    if v[np.argmax(np.abs(v))] < 0:
        u, v = -u, -v
    return s, u, v


def two_factor(P: np.ndarray, p1, p2):
    """Fit K2 K1 to the KS values P of the product pattern, K1 of pattern p1
    applied first, K2 of pattern p2 (chainable: a2 = a1*b1, d1 = c2*d2).
    Returns (V1, V2) in the values layouts [a][d][b][c]."""
    a1, b1, c1, d1 = p1
    a2, b2, c2, d2 = p2
    if a2 != a1 * b1 or d1 != c2 * d2:
        raise ValueError("patterns are not chainable")
    P = np.asarray(P, dtype=np.float64).reshape(a1, d2, b1 * b2, c1 * c2)
    V1 = np.zeros((a1, d1, b1, c1))
    V2 = np.zeros((a2, d2, b2, c2))
    for i1 in range(a1):
        for k1 in range(b1):
            for j2 in range(c2):
                for l2 in range(d2):
                    B = P[i1, l2, k1 * b2:(k1 + 1) * b2, j2::c2]  # B[k2][j1]
                    s, u, v = rank_one(B)
                    V2[i1 * b1 + k1, l2, :, j2] = np.sqrt(s) * u
                    V1[i1, j2 * d2 + l2, k1, :] = np.sqrt(s) * v
    return V1.reshape(-1), V2.reshape(-1)


def hierarchical_butterfly(A: np.ndarray):
    """Factor a dense 2^L x 2^L matrix A (the K of Y = X K^T) into the L
    butterfly factors; returns their values, F_1 (applied first) first."""
    A = np.asarray(A, dtype=np.float64)
    N = A.shape[0]
    L = int(round(np.log2(N)))
    if A.shape != (N, N) or 2 ** L != N or L < 1:
        raise ValueError("A must be square with a power-of-two size")
    out = [None] * L

    def split(P, p, q):
        if p == q:
            out[p - 1] = P.reshape(-1)
            return
        r = (p + q - 1) // 2
        V1, V2 = two_factor(P, butterfly_range_pattern(p, r, L), butterfly_range_pattern(r + 1, q, L))
        split(V1, p, r)
        split(V2, r + 1, q)

    split(A.reshape(-1), 1, L)  # the whole matrix is KS with pattern (1, N, N, 1)
    return out
