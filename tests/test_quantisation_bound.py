"""CPU: the decode path's activation quantisation stays inside the parity bar.

The decode kernel does not multiply the signs by Z = (x / s) (.) V_i in floating point:
for each chunk group of C x 256 input columns (C = 4 at one row of x, 2 at 2-4 rows)
and each column (b, j) it rounds Z to multiples of sigma = max |Z| / 32512 over the
group, and the int8 tensor cores then sum the integers exactly.  This test restates that
rounding in NumPy (a model of the reading, not the kernel's code) and checks, against
the exact float64 oracle linear, that

  * the error of y is at most the analytic bound sum_i sum_j |U_i[r, j]| sum_groups
    (cols x sigma / 2), and
  * it is far below the 2e-3 * max|y| bar the GPU parity tests apply,

for a batch of one and of four rows and a ragged last group.  A mistake in the model
(a lost 1/2, the wrong group size) shows up as a bound violation."""
import numpy as np
import pytest

from oracle import linear
from tests import cases

BAR = 2e-3


def _quantised_factored(x, st, n, C):
    """y with Z rounded per (chunk group, column) as the decode kernel does, plus the
    analytic error bound per output element."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    bsz = x.shape[0]
    xs = (x.astype(np.float32) * st.inv_s.astype(np.float32)[None, :]).astype(np.float32)
    y = np.zeros((bsz, st.m))
    bound = np.zeros((bsz, st.m))
    group = C * 256
    for i in range(n):
        S = 1.0 - 2.0 * st.negs[i].astype(np.float64)                  # +-1, m x d
        V = np.asarray(st.Vs[i], dtype=np.float32)                     # d x 16
        U = np.asarray(st.Us[i], dtype=np.float64)                     # m x 16
        for c0 in range(0, st.d, group):
            c1 = min(st.d, c0 + group)
            # Z[c, b, j] in fp32, as the kernel forms it
            Z = (xs[:, c0:c1].T[:, :, None] * V[c0:c1, None, :]).astype(np.float32)
            amax = np.abs(Z).max(axis=0)                               # b x 16
            sigma = np.where(amax > 0, amax.astype(np.float64) / 32512.0, 1.0)
            q = np.clip(np.rint(Z / sigma[None]), -32512, 32512)
            T = np.einsum("rc,cbj->brj", S[:, c0:c1], q * sigma[None])  # b x m x 16
            y += np.einsum("rj,brj->br", U, T)
            bound += np.einsum("rj,bj->br", np.abs(U), (c1 - c0) * sigma / 2.0)
    return y, bound


@pytest.mark.parametrize("m,d,n,b,C", [(256, 2048, 3, 1, 4), (256, 1280, 2, 4, 2), (128, 768, 2, 1, 4)])
def test_decode_quantisation_within_bound_and_bar(m, d, n, b, C):
    st = cases.synthetic_stack(98, m, d, n, matrix=m + d)
    x, _ = cases.inputs(98, b, d, matrix=b)
    y_ref = linear.linear_factored(x, st.negs, st.Us, st.Vs, st.inv_s, n, m)
    y_q, bound = _quantised_factored(x, st, n, C)
    err = np.abs(y_q - y_ref)
    # the model's own rounding of x (.) 1/s and of Z to fp32 adds a little on top of
    # the quantisation term; 1e-5 of the output scale covers it
    scale = np.abs(y_ref).max()
    assert np.all(err <= bound + 1e-5 * scale)
    assert err.max() <= 0.05 * BAR * scale      # 20x inside the bar


def test_bound_fails_for_a_coarser_step():
    """Planted mistake: a step 256 times coarser (one int8 plane instead of two) breaks
    the stated bound, so the bound is not vacuous."""
    st = cases.synthetic_stack(98, 128, 1024, 2, matrix=5)
    x, _ = cases.inputs(98, 1, 1024, matrix=5)
    y_ref = linear.linear_factored(x, st.negs, st.Us, st.Vs, st.inv_s, 2, 128)
    y_q, bound = _quantised_factored(x, st, 2, 4)
    xs = (x.astype(np.float32) * st.inv_s.astype(np.float32)[None, :]).astype(np.float32)
    # one plane: q in [-127, 127]
    y1 = np.zeros_like(y_ref)
    for i in range(2):
        S = 1.0 - 2.0 * st.negs[i].astype(np.float64)
        Z = (xs[0][:, None] * np.asarray(st.Vs[i], np.float32)).astype(np.float32)
        sig = np.abs(Z).max(axis=0).astype(np.float64) / 127.0
        q = np.rint(Z / sig)
        y1[0] += np.einsum("rj,rj->r", np.asarray(st.Us[i], np.float64), S @ (q * sig))
    assert np.abs(y1 - y_ref).max() > bound.max()
