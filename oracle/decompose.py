"""Activation-aware scaling and iterative absolute-value decomposition (oracle).

Test infrastructure: see the package docstring.  float64 throughout; the stored
factors are rounded to fp16 exactly as the block record stores them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Matrices whose smaller side is at most this use LAPACK's full SVD; larger ones use
# the randomized subspace iteration below.  LAPACK's full SVD of a 4096 x 4096
# residual takes minutes per block in float64, while the iteration reaches the same
# rank-16 subspace in seconds; the limit trades that time, not accuracy (the
# iteration records whether it converged).
EXACT_SVD_LIMIT = 1024


class SvdNotConverged(RuntimeError):
    """The randomized subspace iteration hit its iteration cap before the leading
    singular values settled to the requested relative tolerance."""


def activation_scale(X: np.ndarray) -> np.ndarray:
    """Per-input-channel activation statistic s (float64, length d).

    Follows: Review, Fig. 5 caption (activation-aware scaling, "Eq. 4", is applied
    before the decomposition and ablated as "w/o scaling"); Rebuttal A3 (no Hessian
    and no whitening: the scaling uses activation magnitudes only).  The equation
    itself is not printed on the pages.

    Reading taken: s_c = sqrt(mean_r X[r, c]^2), the RMS of input channel c over the
    calibration rows, floored at 1e-8 * max(s) so that 1/s stays finite.  Because
    the decomposition is equivariant to a global factor on s (invariant I6 in the
    tests), the RMS and the L2 norm readings give the same reconstructed weight.

    The pages do not fix the statistic, so what is pinned is this reading: the
    tests check it against hand-computed values on a calibration matrix whose
    per-column RMS is known in closed form (alternating +-a, a single spike, two
    alternating levels, an all-zero column that takes the floor), which a mean of
    |X|, a maximum of |X| or a missing floor would each fail.  The CUDA path
    consumes whatever 1/s the oracle stores, so GPU parity does not depend on it.
    """
    X = np.asarray(X, dtype=np.float64)
    s = np.sqrt(np.mean(X * X, axis=0))
    floor = 1e-8 * float(s.max()) if s.size else 0.0
    return np.maximum(s, floor if floor > 0 else np.finfo(np.float64).tiny)


def _orient(U: np.ndarray, Vt: np.ndarray):
    """Flip each singular pair so that the column sum of U is >= 0.

    The product U diag(sigma) V^T does not depend on this choice; it only makes the
    stored factors reproducible.
    """
    flip = np.where(U.sum(axis=0) < 0, -1.0, 1.0)
    return U * flip[None, :], Vt * flip[:, None]


def truncated_svd(A: np.ndarray, k: int, gen: np.random.Generator | None = None,
                  oversample: int = 16, max_iter: int = 60, tol: float = 1e-10,
                  info: dict | None = None, strict: bool = False):
    """Rank-k truncated SVD of A: (U m x k, sigma k, Vt k x d), float64.

    Small matrices (min side <= EXACT_SVD_LIMIT) use LAPACK's full SVD.  Larger ones
    use randomized subspace iteration (Halko, Martinsson & Tropp, "Finding structure
    with randomness", SIAM Review 2011, Algorithms 4.4 and 5.1): an l = k + oversample
    column Gaussian sketch, power iterations with QR re-orthonormalisation after every
    product, stopped when the k leading singular values change by less than ``tol``
    (relative) between iterations.

    Convergence is never assumed silently: when ``info`` is a dict it receives
    ``method`` ("lapack" or "randomized"), ``iterations``, ``converged`` and
    ``max_rel_change`` (of the last iteration); with ``strict`` an iteration that
    reaches ``max_iter`` without settling raises SvdNotConverged.
    """
    A = np.asarray(A, dtype=np.float64)
    m, d = A.shape
    k = int(min(k, m, d))
    if min(m, d) <= EXACT_SVD_LIMIT:
        U, sig, Vt = np.linalg.svd(A, full_matrices=False)
        U, Vt = _orient(U[:, :k], Vt[:k, :])
        if info is not None:
            info.update(method="lapack", iterations=0, converged=True, max_rel_change=0.0)
        return U, sig[:k].copy(), Vt
    if gen is None:
        gen = np.random.default_rng(0)
    ell = min(k + oversample, m, d)
    Omega = gen.standard_normal((d, ell))
    Q, _ = np.linalg.qr(A @ Omega)
    prev = None
    sig = None
    converged = False
    change = float("inf")
    it = 0
    for it in range(1, max_iter + 1):
        Qt, _ = np.linalg.qr(A.T @ Q)
        Q, _ = np.linalg.qr(A @ Qt)
        B = Q.T @ A
        Ub, sig_all, Vt_all = np.linalg.svd(B, full_matrices=False)
        sig = sig_all[:k]
        if prev is not None:
            change = float(np.max(np.abs(sig - prev) / np.maximum(sig, 1e-300)))
            if change < tol:
                converged = True
                break
        prev = sig
    if info is not None:
        info.update(method="randomized", iterations=it, converged=converged, max_rel_change=change)
    if strict and not converged:
        raise SvdNotConverged(f"randomized SVD: relative change {change:.3e} >= {tol:.1e} after {it} iterations")
    U = Q @ Ub[:, :k]
    U, Vt = _orient(U, Vt_all[:k, :])
    return U, sig.copy(), Vt


@dataclass
class Decomposition:
    """Result of the oracle decomposition of one weight matrix.

    neg[i]: bool m x d, True where the sign of block i is -1.
    U[i]:   fp16 m x k, V[i]: fp16 d x k, with sqrt(sigma) folded into both.
    inv_s:  float32 length d, 1/s as stored for inference.
    s:      float64 length d, the scale the decomposition used.
    res_norms[i]: Frobenius norm of the scaled residual R_i (R_0 = W * s).
    sigmas[i]: the k singular values of |R_{i-1}| used by block i (float64).
    svd_info[i]: how block i's truncated SVD was computed and whether it converged.
    """
    neg: list = field(default_factory=list)
    U: list = field(default_factory=list)
    V: list = field(default_factory=list)
    inv_s: np.ndarray | None = None
    s: np.ndarray | None = None
    res_norms: list = field(default_factory=list)
    sigmas: list = field(default_factory=list)
    svd_info: list = field(default_factory=list)

    @property
    def n_blocks(self) -> int:
        return len(self.U)


def avd_step(R: np.ndarray, k: int, gen: np.random.Generator | None = None,
             round_fp16: bool = True, info: dict | None = None):
    """One absolute-value decomposition step on a residual R (float64, m x d).

    Follows: Review, Fig. 3 caption (a residual block is a sign matrix plus singular
    vectors obtained by absolute value decomposition); Rebuttal A3 (SVD is applied to
    the absolute value of the previous approximation error; the sign matrix is kept
    separately); Abstract (about 1 bit per parameter per iteration).

    Readings taken:
    * sign: S = +1 where R >= 0 (both signed zeros included), else -1.  The pages
      are silent on zeros; S must be +-1 to fit one bit.
    * sqrt(sigma) is folded into both factors, U_i = Ut diag(sqrt(sigma)),
      V_i = Vt^T diag(sqrt(sigma)), so a block stores no separate sigma (the block
      size formula in the Review, Fig. 5 caption, counts only 2 k (m + n) fp16
      values besides the bits).
    * the next residual is formed with the factors as stored (fp16-rounded when
      ``round_fp16``), so it is the true residual of what the block holds.

    Returns (neg, U, V, R_next, sigma).
    """
    neg = ~(R >= 0)
    A = np.abs(R)
    Ut, sig, Vt = truncated_svd(A, k, gen, info=info)
    root = np.sqrt(sig)
    U = Ut * root[None, :]
    V = Vt.T * root[None, :]
    if round_fp16:
        U16 = U.astype(np.float16)
        V16 = V.astype(np.float16)
        Ue, Ve = U16.astype(np.float64), V16.astype(np.float64)
    else:
        U16, V16 = U, V
        Ue, Ve = U, V
    S = np.where(neg, -1.0, 1.0)
    R_next = R - S * (Ue @ Ve.T)
    return neg, U16, V16, R_next, sig


def decompose(W: np.ndarray, s: np.ndarray, n_blocks: int, k: int,
              gen: np.random.Generator | None = None, round_fp16: bool = True) -> Decomposition:
    """Iterative residual decomposition of W into ``n_blocks`` residual blocks.

    Follows: README "Decomposition" (``--niter``: number of decomposition
    iterations; ``--k``: singular vectors kept); Rebuttal A3 (the iteration count is
    forward-compatible because each iteration decomposes the residual of the
    previous ones; SVD runs on the absolute value of the approximation error);
    Review Fig. 5 caption (scaling before decomposition, undone at inference).

    R_0 = W diag(s) (column c, an input channel, scaled by s_c).  For i = 1..n:
    block i = avd_step(R_{i-1}); R_i = R_{i-1} - S_i * (U_i V_i^T).
    The stored inverse scale is fp32(1 / s).
    """
    W = np.asarray(W, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    out = Decomposition()
    out.s = s.copy()
    out.inv_s = (1.0 / s).astype(np.float32)
    R = W * s[None, :]
    out.res_norms.append(float(np.linalg.norm(R)))
    for _ in range(n_blocks):
        info: dict = {}
        neg, U, V, R, sig = avd_step(R, k, gen, round_fp16, info=info)
        out.svd_info.append(info)
        out.neg.append(neg)
        out.U.append(U)
        out.V.append(V)
        out.sigmas.append(sig)
        out.res_norms.append(float(np.linalg.norm(R)))
    return out


# ------------------------------------------------------------ "w/o AVD" blocks ------
def plain_rank(m: int, d: int, k: int) -> int:
    """Rank k' of a vanilla-SVD block that takes the bytes of a BitStack block.

    Follows: Review, Fig. 5 caption (the "w/o AVD" ablation sets k' = k + m n / (16
    (m + n)) for an m x n weight so that a block keeps the size of the main
    experiments' blocks).  Reading taken where the fraction is not whole: k' is
    rounded down to a multiple of 8, so that the block never grows past the block it
    stands in for and every factor row is a whole number of 16-byte units (the
    library's layout).  For 4096 x 4096 and k = 16 the fraction is whole: k' = 144,
    and 2 k' (m + d) = m d / 8 + 2 k (m + d) exactly.
    """
    kp = k + (m * d) // (16 * (m + d))
    return kp - kp % 8


def plain_step(R: np.ndarray, kp: int, gen: np.random.Generator | None = None,
               round_fp16: bool = True, info: dict | None = None):
    """One vanilla-SVD residual block: the rank-k' truncated SVD of the residual R
    itself (signed, no sign matrix), sqrt(sigma) folded into both fp16 factors as in
    avd_step.

    Follows: Review, Fig. 5 caption ("w/o AVD": vanilla SVD, Eq. 5, replaces the
    absolute value decomposition; the iteration over residuals is unchanged).
    Returns (U, V, R_next, sigma) with R_next = R - U V^T from the stored factors.
    """
    Ut, sig, Vt = truncated_svd(R, kp, gen, info=info)
    root = np.sqrt(sig)
    U = Ut * root[None, :]
    V = Vt.T * root[None, :]
    if round_fp16:
        U16, V16 = U.astype(np.float16), V.astype(np.float16)
        Ue, Ve = U16.astype(np.float64), V16.astype(np.float64)
    else:
        U16, V16 = U, V
        Ue, Ve = U, V
    return U16, V16, R - Ue @ Ve.T, sig


def decompose_plain(W: np.ndarray, s: np.ndarray, n_blocks: int, kp: int,
                    gen: np.random.Generator | None = None, round_fp16: bool = True) -> Decomposition:
    """The "w/o AVD" decomposition: as ``decompose`` (activation-aware scaling, then one
    block per iteration on the previous residual), with plain_step in place of
    avd_step.  The result has no sign matrices (``neg`` stays empty)."""
    W = np.asarray(W, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    out = Decomposition()
    out.s = s.copy()
    out.inv_s = (1.0 / s).astype(np.float32)
    R = W * s[None, :]
    out.res_norms.append(float(np.linalg.norm(R)))
    for _ in range(n_blocks):
        info: dict = {}
        U, V, R, sig = plain_step(R, kp, gen, round_fp16, info=info)
        out.svd_info.append(info)
        out.U.append(U)
        out.V.append(V)
        out.sigmas.append(sig)
        out.res_norms.append(float(np.linalg.norm(R)))
    return out
