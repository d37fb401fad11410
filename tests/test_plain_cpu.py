"""CPU: the "w/o AVD" blocks (vanilla rank-k' SVD in place of the absolute value
decomposition) -- oracle pins and the C ABI's host-side sizes.

The oracle's vanilla-SVD decomposition and linear are pinned to things other than
themselves: the Eckart-Young tail energy of the scaled weight (n blocks of rank k'
without fp16 rounding are its best rank-n k' approximation), exact reproduction by a
full-rank block, the block-size identity the pages state, and a pure-Python loop
evaluation of the linear.  Planted mistakes in the oracle must fail these pins.
"""
import numpy as np
import pytest

import residual_block_decomp_b200 as R
import workloads as wl
from oracle import decompose, linear, pack


def _small(m, d, seed):
    gen = np.random.default_rng(seed)
    W = wl.weight(m, d, gen, outlier_frac=0.1).astype(np.float64)
    s = decompose.activation_scale(wl.calibration(64, d, gen))
    return W, s


def test_plain_rank_keeps_the_block_size():
    # whole fraction: 16 + 4096 * 4096 / (16 * 8192) = 144, and the sizes agree exactly
    assert decompose.plain_rank(4096, 4096, 16) == 144
    assert pack.plain_block_bytes(4096, 4096, 144) == pack.block_bytes(4096, 4096, 16) == 2_359_296
    # 14336 x 4096: 16 + 199.1 -> 215, rounded down to a multiple of 8
    assert decompose.plain_rank(14336, 4096, 16) == 208
    for (_, m, d) in wl.LLAMA3_8B_LINEARS:
        kp = decompose.plain_rank(m, d, 16)
        gap = pack.block_bytes(m, d, 16) - pack.plain_block_bytes(m, d, kp)
        assert kp % 8 == 0 and 0 <= gap < 2 * 8 * (m + d), (m, d, kp)


def test_plain_blocks_reach_the_eckart_young_tail():
    """Without fp16 rounding, n vanilla blocks of rank k' leave exactly the energy of
    the singular values of W diag(s) past index n k'."""
    W, s = _small(40, 28, 21)
    kp, n = 3, 4
    dec = decompose.decompose_plain(W, s, n, kp, round_fp16=False)
    sv = np.linalg.svd(W * s[None, :], compute_uv=False)
    for i in range(n + 1):
        assert dec.res_norms[i] ** 2 == pytest.approx(float(np.sum(sv[i * kp:] ** 2)), rel=1e-9, abs=1e-24)
    assert dec.n_blocks == n and dec.neg == []


def test_full_rank_plain_block_reproduces_the_weight():
    W, s = _small(12, 20, 22)
    dec = decompose.decompose_plain(W, s, 1, 12, round_fp16=False)
    inv_s = dec.inv_s.astype(np.float64)
    Wh = linear.reconstruct_plain(dec.U, dec.V, inv_s, 1, 12)
    # W_hat = (W diag(s)) diag(fp32(1/s)): W up to the fp32 rounding of 1/s
    assert np.max(np.abs(Wh - W * s[None, :] * inv_s[None, :])) < 1e-12 * np.max(np.abs(W))
    # rounded factors: the stored fp16 values, so the residual is that of the rounding only
    dec16 = decompose.decompose_plain(W, s, 1, 12, round_fp16=True)
    assert dec16.res_norms[1] < 1e-3 * dec16.res_norms[0]


@pytest.mark.parametrize("m,d,kp,n,b", [(5, 7, 2, 3, 2), (9, 6, 3, 2, 1)])
def test_plain_linear_forms_agree_with_loops(m, d, kp, n, b):
    gen = np.random.default_rng(23 + m)
    Us = [gen.standard_normal((m, kp)).astype(np.float16) for _ in range(n)]
    Vs = [gen.standard_normal((d, kp)).astype(np.float16) for _ in range(n)]
    inv_s = gen.uniform(0.5, 2.0, d).astype(np.float32)
    x = gen.standard_normal((b, d))
    loops = linear.linear_plain_bruteforce(x, Us, Vs, inv_s, n, m)
    np.testing.assert_allclose(linear.linear_plain_explicit(x, Us, Vs, inv_s, n, m), loops, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(linear.linear_plain_factored(x, Us, Vs, inv_s, n, m), loops, rtol=1e-12, atol=1e-12)
    assert np.all(linear.linear_plain_factored(x, Us, Vs, inv_s, 0, m) == 0.0)


def test_plain_record_layout():
    gen = np.random.default_rng(24)
    U = gen.standard_normal((6, 8)).astype(np.float16)
    V = gen.standard_normal((10, 8)).astype(np.float16)
    rec = pack.make_plain_record(U, V)
    assert rec.size == pack.plain_block_bytes(6, 10, 8)
    assert np.array_equal(rec[:96].view(np.float16).reshape(6, 8), U)
    assert np.array_equal(rec[96:].view(np.float16).reshape(10, 8), V)


def _plain_pins_pass():
    try:
        test_plain_blocks_reach_the_eckart_young_tail()
        test_full_rank_plain_block_reproduces_the_weight()
        test_plain_linear_forms_agree_with_loops(5, 7, 2, 3, 2)
    except AssertionError:
        return False
    return True


def test_planted_plain_mistakes_are_caught(monkeypatch):
    assert _plain_pins_pass()
    real_step, real_fact, real_expl = decompose.plain_step, linear.linear_plain_factored, linear.linear_plain_explicit

    def abs_residual(R, kp, gen=None, round_fp16=True, info=None):      # SVD of |R| as in AVD
        U, V, _, sig = real_step(np.abs(R), kp, gen, round_fp16, info)
        Ue, Ve = U.astype(np.float64), V.astype(np.float64)
        return U, V, R - Ue @ Ve.T, sig

    def residual_not_updated(R, kp, gen=None, round_fp16=True, info=None):
        U, V, _, sig = real_step(R, kp, gen, round_fp16, info)
        return U, V, R - 0.5 * (U.astype(np.float64) @ V.astype(np.float64).T), sig

    def scale_not_undone(x, Us, Vs, inv_s, n, m):
        return real_fact(x, Us, Vs, np.ones_like(np.asarray(inv_s)), n, m)

    def dropped_block(x, Us, Vs, inv_s, n, m):
        return real_expl(x, Us, Vs, inv_s, max(n - 1, 0), m)

    for mod, name, fn in [(decompose, "plain_step", abs_residual), (decompose, "plain_step", residual_not_updated),
                          (linear, "linear_plain_factored", scale_not_undone),
                          (linear, "linear_plain_explicit", dropped_block)]:
        with monkeypatch.context() as mp:
            mp.setattr(mod, name, fn)
            assert not _plain_pins_pass(), f"planted mistake {fn.__name__} in {name} went unnoticed"


# ------------------------------------------------------------------- host ABI ------
def test_abi_plain_sizes_equal_the_oracle():
    for (_, m, d) in wl.LLAMA3_8B_LINEARS:
        kp = decompose.plain_rank(m, d, 16)
        assert R.bs_plain_rank(m, d, 16) == kp
        assert R.bs_plain_block_bytes(m, d, kp) == pack.plain_block_bytes(m, d, kp)
    assert R.bs_plain_rank(4096, 4096, 16) == 144
    assert R.bs_plain_block_bytes(4096, 4096, 12) == 0          # rank must be a multiple of 8
    assert R.bs_plain_block_bytes(0, 4096, 8) == 0
    assert R.bs_plain_rank(-1, 4096, 16) == 0
