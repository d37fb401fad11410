"""GPU: the decomposition on the GPU (bs_decompose) against the oracle.

The GPU's SVD is randomized (its own sketch), so its factors are not the oracle's bit
for bit.  What is fixed and checked:
  * the first block's signs are the signs of W diag(s): bit-exact;
  * the residual norms the GPU reports are the norms of the residuals of the records it
    wrote (recomputed here in float64 from those records);
  * every residual is within 2 % of the oracle's (exact LAPACK SVD at these sizes), and
    the first is no better than the Eckart-Young optimum allows;
  * each factor pair is oriented as the oracle orients it (column sum of U >= 0);
  * the records work: a stack of them through bs_linear meets the parity bar against the
    oracle linear of the same records.
"""
import numpy as np
import pytest
import torch

import residual_block_decomp_b200 as R
import workloads as wl
from oracle import decompose, linear, pack
from tests import cases
from tests.gpu_util import assert_close, load_stack

pytestmark = pytest.mark.gpu


def _gpu_decompose(W, s, n, seed=5, power_iters=6):
    m, d = W.shape
    Wt = torch.from_numpy(W.astype(np.float32)).cuda()
    st = torch.from_numpy(s.astype(np.float32)).cuda()
    bb = R.bs_block_bytes(m, d, 16)
    recs = torch.zeros(n * bb, dtype=torch.uint8, device="cuda")
    norms = torch.zeros(n + 1, dtype=torch.float64, device="cuda")
    ws = torch.empty(R.bs_decompose_workspace_bytes(m, d), dtype=torch.uint8, device="cuda")
    R.bs_decompose(Wt, st, n, recs, norms, ws, seed=seed, power_iters=power_iters)
    torch.cuda.synchronize()
    host = recs.cpu().numpy()
    parts = [pack.parse_record(host[i * bb:(i + 1) * bb], m, d, 16) for i in range(n)]
    return parts, np.sqrt(norms.cpu().numpy()), [host[i * bb:(i + 1) * bb] for i in range(n)]


@pytest.mark.parametrize("m,d,n,config", [(512, 768, 4, 81), (1024, 1024, 3, 82)])
def test_gpu_decomposition_matches_oracle(m, d, n, config):
    W = wl.weight(m, d, wl.generator(config, 0, "W"), outlier_frac=0.01,
                  outlier_gen=wl.generator(config, 0, "outlier")).astype(np.float64)
    s = decompose.activation_scale(wl.calibration(64, d, wl.generator(config, 0, "calib")))
    s32 = s.astype(np.float32).astype(np.float64)          # the GPU is given fp32 s
    dec = decompose.decompose(W, s32, n, 16, round_fp16=True)
    parts, gnorms, records = _gpu_decompose(W, s32, n)
    negs = [p[0] for p in parts]
    Us = [p[1] for p in parts]
    Vs = [p[2] for p in parts]
    # first block: the signs of the scaled weight
    assert np.array_equal(negs[0], ~(W * s32[None, :] >= 0))
    # the reported norms are those of the records' own residuals
    Ws = W * s32[None, :]
    for i in range(n + 1):
        res = np.linalg.norm(Ws - linear.reconstruct_scaled(negs, Us, Vs, i, m, d))
        assert gnorms[i] == pytest.approx(res, rel=2e-4), (i, gnorms[i], res)
    # quality against the oracle's exact-SVD decomposition, and Eckart-Young for block 1
    assert gnorms[0] == pytest.approx(dec.res_norms[0], rel=1e-6)
    for i in range(1, n + 1):
        assert gnorms[i] <= dec.res_norms[i] * 1.02, (i, gnorms[i], dec.res_norms[i])
    sv = np.linalg.svd(np.abs(Ws), compute_uv=False)
    assert gnorms[1] ** 2 >= (np.sum(sv ** 2) - np.sum(sv[:16] ** 2)) * (1 - 1e-3)
    # orientation: column sums of U non-negative (up to the fp16 rounding of tiny sums)
    for U in Us:
        cs = U.astype(np.float64).sum(axis=0)
        assert np.all(cs >= -1e-3 * np.abs(U.astype(np.float64)).sum(axis=0))
    # the records serve the linear
    st = cases.Stack(m, d, negs, Us, Vs, (1.0 / s32).astype(np.float32), records)
    layer = load_stack(st)
    x64, xt = cases.inputs(config, 2, d)
    y = layer.forward(xt.cuda(), n)
    torch.cuda.synchronize()
    assert layer.device_error() == R.BS_OK
    assert_close(y, st.y_ref(x64, n), what=f"linear over GPU-decomposed {m}x{d} n={n}")


def test_gpu_decomposition_argument_errors():
    W = torch.zeros((128, 256), dtype=torch.float32, device="cuda")
    s = torch.ones(256, dtype=torch.float32, device="cuda")
    bb = R.bs_block_bytes(128, 256, 16)
    recs = torch.zeros(2 * bb, dtype=torch.uint8, device="cuda")
    norms = torch.zeros(3, dtype=torch.float64, device="cuda")
    ws = torch.empty(R.bs_decompose_workspace_bytes(128, 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_decompose(W, s, 3, recs, norms, ws)            # records hold only two blocks
    assert e.value.status == R.BS_ERR_CAPACITY
    with pytest.raises(R.BsError) as e:
        R.bs_decompose(W[:, :200].contiguous(), s[:200].contiguous(), 1, recs, norms, ws)
    assert e.value.status == R.BS_ERR_UNSUPPORTED_SHAPE
    # an all-zero weight: every block is zero and the residual stays zero
    R.bs_decompose(W, s, 2, recs, norms, ws)
    torch.cuda.synchronize()
    assert np.all(norms.cpu().numpy() == 0.0)
