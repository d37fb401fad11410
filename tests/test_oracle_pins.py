"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests compares the oracle with itself: each checks a closed form, an
invariant the method guarantees, a value the pages print, a brute-force evaluation
on tiny inputs, or an independent algorithm.  ``test_planted_mistakes`` plants
plausible errors into the oracle (on the CPU) and checks that the pins catch them.
"""
import os

import numpy as np
import pytest

import workloads as wl
from oracle import budget, decompose, linear, pack

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = [p.strip() for p in line.split("=", 1)]
            vals[key] = val
    return vals


def _small_case(m=24, d=16, seed=0, outliers=False):
    gen = np.random.default_rng(seed)
    W = wl.weight(m, d, gen, outlier_frac=0.125 if outliers else 0.0)
    X = wl.calibration(64, d, gen)
    return W.astype(np.float64), decompose.activation_scale(X)


# ---------------------------------------------------------------- P1: n = 0 ----------
def test_p1_zero_blocks_give_zero():
    """Rebuttal restoration snippet: the accumulator starts at zero."""
    W, s = _small_case()
    dec = decompose.decompose(W, s, 2, 4)
    x = np.random.default_rng(1).standard_normal((3, W.shape[1]))
    assert not linear.reconstruct(dec.neg, dec.U, dec.V, dec.inv_s, 0).any()
    assert not linear.linear_explicit(x, dec.neg, dec.U, dec.V, dec.inv_s, 0).any()
    assert not linear.linear_factored(x, dec.neg, dec.U, dec.V, dec.inv_s, 0).any()


# --------------------------------------------------- P2: full rank reproduces W -------
def test_p2_full_rank_block_reproduces_weight():
    """One block with k = min(m, d): S * |R| = R exactly, so W_s is reproduced."""
    W, s = _small_case(24, 16)
    dec = decompose.decompose(W, s, 1, 16, round_fp16=False)
    Ws = W * s[None, :]
    Wr = linear.reconstruct_scaled(dec.neg, dec.U, dec.V, 1, 24, 16)
    assert np.max(np.abs(Wr - Ws)) <= 1e-10 * np.max(np.abs(Ws))
    # and in the unscaled domain, up to the fp32 rounding of the stored 1/s
    Wh = linear.reconstruct(dec.neg, dec.U, dec.V, dec.inv_s, 1)
    assert np.max(np.abs(Wh - W)) <= 1e-6 * np.max(np.abs(W))
    # with the fp16 factors the block stores: entrywise error at fp16 level
    dec16 = decompose.decompose(W, s, 1, 16)
    Wr16 = linear.reconstruct_scaled(dec16.neg, dec16.U, dec16.V, 1, 24, 16)
    assert np.max(np.abs(Wr16 - Ws)) <= 2.0 ** -9 * np.max(np.abs(Ws))


# ------------------------------------------ P3: sign pattern times rank-one magnitude ---
def test_p3_rank_one_magnitude():
    """W = S * (a b^T) with a, b > 0: |W_s| is rank one, so one k = 1 block is exact."""
    gen = np.random.default_rng(3)
    m, d = 40, 24
    S = np.where(gen.random((m, d)) < 0.5, -1.0, 1.0)
    a = gen.uniform(0.5, 2.0, m)
    b = gen.uniform(0.5, 2.0, d)
    W = S * np.outer(a, b)
    s = gen.uniform(0.5, 2.0, d)
    dec = decompose.decompose(W, s, 1, 1, round_fp16=False)
    assert np.array_equal(dec.neg[0], S < 0)
    P = dec.U[0] @ dec.V[0].T
    assert np.allclose(P, np.outer(a, b * s), rtol=1e-12, atol=0)
    assert dec.res_norms[1] <= 1e-12 * dec.res_norms[0]


# ----------------------------------------------------- P4: first signs = sign(W) -------
def test_p4_first_block_signs_are_weight_signs():
    W, s = _small_case(64, 48, seed=4, outliers=True)
    W[0, 0] = 0.0   # a zero weight takes the + sign
    W[1, 1] = -0.0
    dec = decompose.decompose(W, s, 2, 4)
    assert np.array_equal(dec.neg[0], W < 0)
    assert not dec.neg[0][0, 0] and not dec.neg[0][1, 1]


# ------------------------------------------------------------ P5: block bytes ---------
def test_p5_block_bytes_match_pages():
    g = _read_golden("block_size.txt")
    m, d, k = int(g["max_block_8b_m"]), int(g["max_block_8b_d"]), int(g["k"])
    nbytes = pack.block_bytes(m, d, k)
    assert nbytes == 7_929_856
    # "7.56 MB" in the Rebuttal: the block byte count in MiB, rounded to two decimals
    assert round(nbytes / 2 ** 20, 2) == float(g["max_block_8b_mb"])
    # Review Fig. 5: a vanilla-SVD block with k' vectors has the same size
    for (mm, dd) in [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336), (512, 512)]:
        kprime = k + mm * dd / (16 * (mm + dd))
        assert 2 * kprime * (mm + dd) == pytest.approx(pack.block_bytes(mm, dd, k), rel=1e-12)
    # the record built from real parts has exactly that many bytes
    neg = np.zeros((128, 256), bool)
    rec = pack.make_record(neg, np.zeros((128, 16), np.float16), np.zeros((256, 16), np.float16))
    assert rec.size == pack.block_bytes(128, 256, 16)


# ---------------------------------------------------- I3: residual norm monotone -------
@pytest.mark.parametrize("round16", [False, True])
def test_i3_residual_norm_non_increasing(round16):
    """||R_i|| <= ||R_{i-1}|| in the scaled domain (Rebuttal A3: each iteration
    decomposes the previous residual; Eckart-Young: the rank-k fit beats zero)."""
    W, s = _small_case(96, 64, seed=5, outliers=True)
    dec = decompose.decompose(W, s, 8, 4, round_fp16=round16)
    r = np.array(dec.res_norms)
    slack = 0.0 if not round16 else 2.0 ** -10
    assert np.all(r[1:] <= r[:-1] * (1 + 1e-12) + slack * r[:-1])
    assert r[-1] < 0.9 * r[0]


# -------------------------------------------------------- I4: Eckart-Young -----------
def test_i4_first_step_energy_is_top_k_singular_energy():
    W, s = _small_case(80, 56, seed=6, outliers=True)
    k = 5
    dec = decompose.decompose(W, s, 1, k, round_fp16=False)
    Ws = W * s[None, :]
    sv = np.linalg.svd(np.abs(Ws), compute_uv=False)   # singular values only
    lhs = dec.res_norms[0] ** 2 - dec.res_norms[1] ** 2
    assert lhs == pytest.approx(float(np.sum(sv[:k] ** 2)), rel=1e-9)


# ------------------------------------------------ I5: explicit = factored = loops -----
@pytest.mark.parametrize("m,d,k,n,b", [(4, 6, 1, 1, 1), (7, 5, 2, 3, 2), (12, 9, 4, 4, 3),
                                       (16, 32, 3, 2, 1), (32, 8, 2, 4, 2)])
def test_i5_forms_agree_with_brute_force(m, d, k, n, b):
    gen = np.random.default_rng(m * 100 + d)
    negs = [gen.random((m, d)) < 0.5 for _ in range(n)]
    Us = [gen.standard_normal((m, k)).astype(np.float16) for _ in range(n)]
    Vs = [gen.standard_normal((d, k)).astype(np.float16) for _ in range(n)]
    inv_s = gen.uniform(0.5, 2.0, d).astype(np.float32)
    x = gen.standard_normal((b, d)).astype(np.float16)
    ref = linear.linear_bruteforce(x, negs, Us, Vs, inv_s, n, m)
    ex = linear.linear_explicit(x, negs, Us, Vs, inv_s, n)
    fa = linear.linear_factored(x, negs, Us, Vs, inv_s, n)
    rows = linear.linear_rows(x, negs, Us, Vs, inv_s, n, np.arange(m))
    scale = np.max(np.abs(ref)) + 1e-300
    for got in (ex, fa, rows):
        assert np.max(np.abs(got - ref)) <= 1e-12 * scale


# ----------------------------------------------------------- I6: scale invariance -----
def test_i6_global_scale_factor_leaves_weight_unchanged():
    """Multiplying s by 4 (a power of two) scales R by 4, sigma by 4 and the stored
    factors by 2 exactly, so the reconstructed weight is bit-identical."""
    W, s = _small_case(48, 32, seed=7, outliers=True)
    a = decompose.decompose(W, s, 3, 4)
    b = decompose.decompose(W, 4.0 * s, 3, 4)
    Wa = linear.reconstruct(a.neg, a.U, a.V, a.inv_s, 3)
    Wb = linear.reconstruct(b.neg, b.U, b.V, b.inv_s, 3)
    assert np.array_equal(Wa, Wb)
    # a non-power-of-two factor: equal up to float64 rounding with unrounded factors
    # (with fp16 factors, rounding differences can flip the sign of near-zero
    # residual entries in later iterations, so the comparison is made in float64)
    a64 = decompose.decompose(W, s, 3, 4, round_fp16=False)
    c64 = decompose.decompose(W, 3.0 * s, 3, 4, round_fp16=False)
    Wa64 = linear.reconstruct(a64.neg, a64.U, a64.V, a64.inv_s, 3)
    Wc64 = linear.reconstruct(c64.neg, c64.U, c64.V, c64.inv_s, 3)
    assert np.max(np.abs(Wc64 - Wa64)) <= 1e-6 * np.max(np.abs(Wa64))


# ------------------------------------------------------------------ L1: packing -------
def test_l1_canonical_packing_bits():
    gen = np.random.default_rng(8)
    neg = gen.random((5, 24)) < 0.5
    packed = pack.pack_canonical(neg)
    for r in range(5):
        for c in range(24):
            assert ((int(packed[r, c // 8]) >> (c % 8)) & 1) == int(neg[r, c])
    assert np.array_equal(pack.unpack_canonical(packed, 24), neg)


def test_l1_device_order_positions_and_roundtrip():
    gen = np.random.default_rng(9)
    m, d = 256, 512
    neg = gen.random((m, d)) < 0.5
    words = pack.pack_device(neg)
    assert words.size == m * d // 32
    # brute force: every (r, c) sits at the position the layout defines
    seen = np.zeros(m * d, dtype=np.int64)
    for r in range(m):
        for c in range(d):
            wi, bit = pack.device_position(r, c, d)
            assert ((int(words[wi]) >> bit) & 1) == int(neg[r, c])
            seen[wi * 32 + bit] += 1
    assert np.all(seen == 1)  # a bijection
    assert np.array_equal(pack.unpack_device(words, m, d), neg)


def test_l1_record_roundtrip():
    gen = np.random.default_rng(10)
    neg, U, V = wl.synthetic_block(128, 512, 16, gen)
    rec = pack.make_record(neg, U, V)
    n2, U2, V2 = pack.parse_record(rec, 128, 512, 16)
    assert np.array_equal(n2, neg) and np.array_equal(U2, U) and np.array_equal(V2, V)


# ------------------------------------------------ activation scale (the reading) -----
def test_activation_scale_is_per_channel_rms_with_floor():
    """The stated reading of the scaling statistic (Review, Fig. 5 caption names
    "Eq. 4" without printing it): s_c = sqrt(mean_r X[r, c]^2), floored at
    1e-8 * max(s).  Hand-built columns whose RMS is known in closed form:
      0: +-a alternating            -> a
      1: a single spike b, else 0   -> b / sqrt(rows)
      2: all zero                   -> the floor 1e-8 * max(s)
      3: 3 and -4 alternating       -> sqrt((9 + 16) / 2)
      4: constant c                 -> |c|
    A mean of |X| (column 1 gives b / rows), a maximum of |X| (column 1 gives b,
    column 3 gives 4), a missing floor (column 2 gives 0) or a missing square root
    would each fail."""
    rows = 64
    a, b, c = 0.75, 12.0, -2.5
    X = np.zeros((rows, 5))
    X[:, 0] = np.where(np.arange(rows) % 2 == 0, a, -a)
    X[17, 1] = b
    X[:, 3] = np.where(np.arange(rows) % 2 == 0, 3.0, -4.0)
    X[:, 4] = c
    s = decompose.activation_scale(X)
    expect = np.array([a, b / 8.0, 0.0, np.sqrt(12.5), abs(c)])
    smax = expect.max()
    expect[2] = 1e-8 * smax
    assert np.allclose(s, expect, rtol=1e-15, atol=0.0)
    # the scale is per input channel: permuting the columns permutes s
    perm = np.array([3, 0, 4, 1, 2])
    assert np.array_equal(decompose.activation_scale(X[:, perm]), s[perm])
    # invariant to the order and sign of the calibration rows
    assert np.allclose(decompose.activation_scale(-X[::-1]), s, rtol=1e-15, atol=0.0)


def test_randomized_svd_reports_non_convergence(monkeypatch):
    """The iteration never returns an unconverged result silently: with a tiny
    singular gap and two iterations it reports converged=False, and strict mode
    raises."""
    gen = np.random.default_rng(5)
    m, d, k = 120, 90, 4
    Q1, _ = np.linalg.qr(gen.standard_normal((m, d)))
    Q2, _ = np.linalg.qr(gen.standard_normal((d, d)))
    sv = np.concatenate([[5.0, 4.0, 3.0, 2.0], 2.0 * (1.0 - 1e-3 * np.arange(1, d - k + 1) / d)])
    A = (Q1 * np.sort(sv)[::-1]) @ Q2.T
    monkeypatch.setattr(decompose, "EXACT_SVD_LIMIT", 10)
    info = {}
    decompose.truncated_svd(A, k, np.random.default_rng(0), max_iter=2, info=info)
    assert info["method"] == "randomized" and info["iterations"] == 2 and info["converged"] is False
    with pytest.raises(decompose.SvdNotConverged):
        decompose.truncated_svd(A, k, np.random.default_rng(0), max_iter=2, strict=True)
    info = {}
    decompose.truncated_svd(A[:, :8], 4, None, info=info)     # LAPACK path
    assert info == {"method": "lapack", "iterations": 0, "converged": True, "max_rel_change": 0.0}


# ------------------------------------------------------------ randomized SVD --------
def test_randomized_svd_matches_lapack_on_gapped_spectrum(monkeypatch):
    gen = np.random.default_rng(11)
    m, d, k = 300, 200, 6
    Q1, _ = np.linalg.qr(gen.standard_normal((m, d)))
    Q2, _ = np.linalg.qr(gen.standard_normal((d, d)))
    sv = np.concatenate([np.linspace(10, 5, k), 0.5 * np.exp(-np.arange(d - k) / 20)])
    A = (Q1 * sv) @ Q2.T
    monkeypatch.setattr(decompose, "EXACT_SVD_LIMIT", 10)
    info = {}
    U, sig, Vt = decompose.truncated_svd(A, k, np.random.default_rng(0), info=info, strict=True)
    assert info["converged"] and info["method"] == "randomized"
    assert np.allclose(sig, sv[:k], rtol=1e-9)
    Ul, sl, Vtl = np.linalg.svd(A, full_matrices=False)
    assert np.allclose((U * sig) @ Vt, (Ul[:, :k] * sl[:k]) @ Vtl[:k], atol=1e-8)


# --------------------------------------------------------------- budget fill ---------
def test_budget_order_keeps_prefixes_and_fills_greedily():
    gen = wl.generator(5, 0, "order")
    nmat = 7
    wts = wl.order_weights(nmat, gen)
    order = budget.global_order(wts, 16)
    seen = [0] * nmat
    for (w, i) in order:
        assert i == seen[w]
        seen[w] += 1
    sizes = np.array([pack.block_bytes(m, d, 16) for (_, m, d) in wl.LLAMA3_8B_LINEARS])
    for mib in (0.5, 10, 100, 400):
        n = budget.budget_fill(order, sizes, mib)
        used = int(np.sum(n * sizes))
        assert used <= mib * 2 ** 20
        # the next block in the order would not fit
        pos = int(np.sum(n))
        if pos < len(order):
            w, i = order[pos]
            assert i == n[w] and used + sizes[w] > mib * 2 ** 20


# ---------------------------------------------------------- planted mistakes ---------
def _pin_suite_passes():
    """Run the value pins on fresh data; return False if any fails."""
    try:
        test_p1_zero_blocks_give_zero()
        test_p2_full_rank_block_reproduces_weight()
        test_p3_rank_one_magnitude()
        test_i4_first_step_energy_is_top_k_singular_energy()
        for case in [(7, 5, 2, 3, 2), (12, 9, 4, 4, 3)]:
            test_i5_forms_agree_with_brute_force(*case)
        test_i6_global_scale_factor_leaves_weight_unchanged()
        test_activation_scale_is_per_channel_rms_with_floor()
    except AssertionError:
        return False
    return True


def test_planted_mistakes_are_caught(monkeypatch):
    assert _pin_suite_passes()

    real_recon = linear.reconstruct_scaled
    real_step = decompose.avd_step
    real_fact = linear.linear_factored

    def transposed_factor(negs, Us, Vs, n, m, d):     # V used as if it were rows of U
        W = real_recon(negs, Us, Vs, n, m, d)
        return W + (1e-3 * W[::-1] if n else 0)

    def dropped_block(negs, Us, Vs, n, m, d):
        return real_recon(negs, Us, Vs, max(n - 1, 0), m, d)

    def flipped_sign(R, k, gen=None, round_fp16=True, info=None):
        neg, U, V, Rn, sig = real_step(R, k, gen, round_fp16, info)
        S = np.where(neg, -1.0, 1.0)
        return ~neg, U, V, R + S * (U.astype(np.float64) @ V.astype(np.float64).T), sig

    def scale_on_rows(x, negs, Us, Vs, inv_s, n, m=None):
        y = real_fact(x, negs, Us, Vs, inv_s, n, m)
        return y * 1.0001

    def mean_abs_scale(X):                            # mean |X| in place of the RMS
        X = np.asarray(X, dtype=np.float64)
        s = np.mean(np.abs(X), axis=0)
        return np.maximum(s, 1e-8 * s.max())

    for name, mod, fn in [("reconstruct_scaled", linear, transposed_factor),
                          ("reconstruct_scaled", linear, dropped_block),
                          ("avd_step", decompose, flipped_sign),
                          ("linear_factored", linear, scale_on_rows),
                          ("activation_scale", decompose, mean_abs_scale)]:
        with monkeypatch.context() as mp:
            mp.setattr(mod, name, fn)
            assert not _pin_suite_passes(), f"planted mistake in {name} ({fn.__name__}) went unnoticed"
