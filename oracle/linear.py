"""Weight reconstruction and the BitStack linear, explicit and factored (oracle).

Test infrastructure: see the package docstring.  float64 throughout, computed from
the exact stored values (fp16 factors, fp32 inverse scale, fp16/bf16 inputs widened
without rounding).
"""
from __future__ import annotations

import numpy as np


def _signs(neg: np.ndarray) -> np.ndarray:
    return np.where(np.asarray(neg, dtype=bool), -1.0, 1.0)


def reconstruct_scaled(negs, Us, Vs, n: int, m: int, d: int) -> np.ndarray:
    """W_s,n = sum_{i < n} S_i * (U_i V_i^T), float64 m x d (scaled domain).

    Follows: Rebuttal, weight restoration snippet (an out x in accumulator starts at
    zero and, for every loaded block, adds the unpacked sign matrix times the product
    of the block's singular vectors).  With n = 0 the result is the zero matrix.
    """
    W = np.zeros((m, d), dtype=np.float64)
    for i in range(n):
        P = np.asarray(Us[i], dtype=np.float64) @ np.asarray(Vs[i], dtype=np.float64).T
        W += _signs(negs[i]) * P
    return W


def reconstruct(negs, Us, Vs, inv_s, n: int, m: int | None = None) -> np.ndarray:
    """W_hat_n = W_s,n diag(1/s), float64 m x d.

    Follows: the weight restoration snippet (Rebuttal) for the sum over blocks, and
    Review Fig. 5 caption for the activation-aware scaling, which is undone per input
    channel (column) at inference.
    """
    inv_s = np.asarray(inv_s, dtype=np.float64)
    d = inv_s.shape[0]
    mm = m if m is not None else np.asarray(negs[0]).shape[0]
    return reconstruct_scaled(negs, Us, Vs, n, mm, d) * inv_s[None, :]


def linear_explicit(x: np.ndarray, negs, Us, Vs, inv_s, n: int, m: int | None = None) -> np.ndarray:
    """y = x W_hat_n^T (float64 b x m): reconstruct, then a dense product.

    This is the unfused evaluation order of the Rebuttal's restoration snippet (an
    accumulator the size of the weight, then an ordinary matmul).
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    W = reconstruct(negs, Us, Vs, inv_s, n, m)
    return x @ W.T


def linear_factored(x: np.ndarray, negs, Us, Vs, inv_s, n: int, m: int | None = None) -> np.ndarray:
    """y = sum_i rowdot_k(U_i, S_i ((x * 1/s) (.) V_i)) (float64 b x m).

    The same value as linear_explicit, by associativity:
    y[b, r] = sum_i sum_j U_i[r, j] sum_c S_i[r, c] x'[b, c] V_i[c, j] with
    x' = x * (1/s).  A separate code path, so that the two forms check each other.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    bsz = x.shape[0]
    mm = m if m is not None else negs[0].shape[0]
    y = np.zeros((bsz, mm), dtype=np.float64)
    if n == 0:
        return y
    xs = x * np.asarray(inv_s, dtype=np.float64)[None, :]            # b x d
    for i in range(n):
        V = np.asarray(Vs[i], dtype=np.float64)                       # d x k
        U = np.asarray(Us[i], dtype=np.float64)                       # m x k
        k = V.shape[1]
        Z = (xs.T[:, None, :] * V[:, :, None]).reshape(V.shape[0], k * bsz)   # d x (k b)
        T = _signs(negs[i]) @ Z                                       # m x (k b)
        y += np.einsum("rj,rjb->br", U, T.reshape(mm, k, bsz))
    return y


def linear_bruteforce(x, negs, Us, Vs, inv_s, n: int, m: int) -> np.ndarray:
    """Pure-Python quadruple loop over (b, r, c, i, j); tiny shapes only."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    bsz, d = x.shape
    y = np.zeros((bsz, m), dtype=np.float64)
    for b in range(bsz):
        for r in range(m):
            acc = 0.0
            for c in range(d):
                xc = float(x[b, c]) * float(inv_s[c])
                for i in range(n):
                    sgn = -1.0 if negs[i][r, c] else 1.0
                    w = 0.0
                    for j in range(Us[i].shape[1]):
                        w += float(Us[i][r, j]) * float(Vs[i][c, j])
                    acc += xc * sgn * w
            y[b, r] = acc
    return y


def linear_rows(x: np.ndarray, negs, Us, Vs, inv_s, n: int, rows: np.ndarray) -> np.ndarray:
    """y[:, rows] computed row by row (float64), for spot checks at full size.

    For each requested output row r: W_hat[r, :] = sum_i S_i[r, :] (U_i[r, :] V_i^T)
    times 1/s, then x W_hat[r, :]^T.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    inv_s = np.asarray(inv_s, dtype=np.float64)
    out = np.zeros((x.shape[0], len(rows)), dtype=np.float64)
    for idx, r in enumerate(rows):
        w = np.zeros(inv_s.shape[0], dtype=np.float64)
        for i in range(n):
            p = np.asarray(Vs[i], dtype=np.float64) @ np.asarray(Us[i][r], dtype=np.float64)
            w += _signs(negs[i][r]) * p
        out[:, idx] = x @ (w * inv_s)
    return out


# ------------------------------------------------------------ "w/o AVD" blocks ------
def reconstruct_plain(Us, Vs, inv_s, n: int, m: int) -> np.ndarray:
    """W_hat_n = (sum_{i < n} U_i V_i^T) diag(1/s) for vanilla-SVD blocks (float64).

    Follows: Review, Fig. 5 caption ("w/o AVD" blocks are plain low-rank factors, the
    scaling undone per input channel as for BitStack blocks).
    """
    inv_s = np.asarray(inv_s, dtype=np.float64)
    W = np.zeros((m, inv_s.shape[0]), dtype=np.float64)
    for i in range(n):
        W += np.asarray(Us[i], dtype=np.float64) @ np.asarray(Vs[i], dtype=np.float64).T
    return W * inv_s[None, :]


def linear_plain_explicit(x: np.ndarray, Us, Vs, inv_s, n: int, m: int) -> np.ndarray:
    """y = x W_hat_n^T (float64 b x m) with W_hat_n from reconstruct_plain."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    return x @ reconstruct_plain(Us, Vs, inv_s, n, m).T


def linear_plain_factored(x: np.ndarray, Us, Vs, inv_s, n: int, m: int) -> np.ndarray:
    """y = sum_i ((x * 1/s) V_i) U_i^T (float64 b x m): the same value by
    associativity, never forming the weight."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    y = np.zeros((x.shape[0], m), dtype=np.float64)
    xs = x * np.asarray(inv_s, dtype=np.float64)[None, :]
    for i in range(n):
        t = xs @ np.asarray(Vs[i], dtype=np.float64)
        y += t @ np.asarray(Us[i], dtype=np.float64).T
    return y


def linear_plain_bruteforce(x, Us, Vs, inv_s, n: int, m: int) -> np.ndarray:
    """Pure-Python loops over (b, r, c, i, j); tiny shapes only."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    bsz, d = x.shape
    y = np.zeros((bsz, m), dtype=np.float64)
    for b in range(bsz):
        for r in range(m):
            acc = 0.0
            for c in range(d):
                xc = float(x[b, c]) * float(inv_s[c])
                for i in range(n):
                    for j in range(Us[i].shape[1]):
                        acc += xc * float(Us[i][r, j]) * float(Vs[i][c, j])
            y[b, r] = acc
    return y
