"""GPU: "w/o AVD" stacks (vanilla rank-k' SVD blocks) through the C ABI against the oracle.

Bar: max|y - y_ref| <= 2e-3 * max|y_ref| (fp16/bf16 inputs and outputs, fp32 sums,
fp64 oracle), the same as for BitStack stacks; the weight rebuilt by bs_reconstruct
in fp32 within 1e-5 * max|W|."""
import numpy as np
import pytest
import torch

import residual_block_decomp_b200 as R
import workloads as wl
from oracle import decompose, linear, pack
from residual_block_decomp_b200 import BitStackLinear
from tests import cases
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu


class PlainCase:
    """Oracle blocks of a "w/o AVD" stack and their records."""

    def __init__(self, m, d, kp, Us, Vs, inv_s):
        self.m, self.d, self.kp, self.Us, self.Vs, self.inv_s = m, d, kp, Us, Vs, inv_s
        self.records = [pack.make_plain_record(u, v) for u, v in zip(Us, Vs)]

    @property
    def n(self):
        return len(self.Us)

    def y_ref(self, x, n):
        return linear.linear_plain_factored(x, self.Us, self.Vs, self.inv_s, n, self.m)

    def layer(self, n_loaded=None):
        L = BitStackLinear(self.m, self.d, max(self.n, 1), self.inv_s, k=self.kp, plain=True)
        for rec in self.records:
            L.add_record(rec)
        L.set_loaded(self.n if n_loaded is None else n_loaded)
        torch.cuda.synchronize()
        return L


def decomposed_case(m, d, n, seed):
    gen = wl.generator(seed, 0, "W")
    W = wl.weight(m, d, gen, outlier_frac=0.01, outlier_gen=wl.generator(seed, 0, "outlier"))
    s = decompose.activation_scale(wl.calibration(64, d, wl.generator(seed, 0, "calib")))
    kp = decompose.plain_rank(m, d, 16)
    dec = decompose.decompose_plain(W, s, n, kp, wl.generator(seed, 0, "svd"))
    return PlainCase(m, d, kp, dec.U, dec.V, dec.inv_s)


def synthetic_case(m, d, kp, n, seed):
    gen = wl.generator(seed, 0, "blocks")
    Us = [wl.random_factors(m, kp, gen, 0.12 / np.sqrt(i + 1.0)) for i in range(n)]
    Vs = [wl.random_factors(d, kp, gen, 0.12 / np.sqrt(i + 1.0)) for i in range(n)]
    return PlainCase(m, d, kp, Us, Vs, wl.synthetic_inv_scale(d, gen))


def _forward(layer, xt, n):
    y = layer.forward(xt.cuda(), n)
    torch.cuda.synchronize()
    assert layer.device_error() == R.BS_OK
    return y


@pytest.mark.parametrize("b,dtype", [(1, "f16"), (3, "bf16"), (17, "f16")])
def test_decomposed_plain_stack_matches_oracle(b, dtype):
    pc = decomposed_case(256, 512, 3, 61)
    assert pc.kp == 24
    layer = pc.layer()
    x, xt = cases.inputs(61, b, pc.d, dtype=dtype)
    for n in range(0, pc.n + 1):
        y = _forward(layer, xt, n)
        if n == 0:
            assert not y.float().abs().sum().item()
        else:
            assert_close(y, pc.y_ref(x, n), what=f"plain 256x512 k'=24 n={n} b={b} {dtype}")


@pytest.mark.parametrize("m,d,kp,n,b", [(200, 328, 8, 2, 2), (33, 1000, 256, 3, 5), (4096, 4096, 144, 8, 1),
                                        (4096, 4096, 144, 8, 16), (1024, 4096, 64, 4, 40)])
def test_synthetic_plain_shapes_match_oracle(m, d, kp, n, b):
    pc = synthetic_case(m, d, kp, n, 62)
    layer = pc.layer()
    x, xt = cases.inputs(62, b, d)
    y = _forward(layer, xt, n)
    assert_close(y, pc.y_ref(x, n), what=f"plain {m}x{d} k'={kp} n={n} b={b}")
    # fixed association: the same call twice gives the same bits
    assert torch.equal(y, _forward(layer, xt, n))


def test_plain_append_drop_and_reconstruct():
    pc = synthetic_case(160, 288, 16, 4, 63)
    layer = pc.layer(n_loaded=2)
    assert layer.n_blocks == 2
    x, xt = cases.inputs(63, 2, pc.d)
    assert_close(_forward(layer, xt, 2), pc.y_ref(x, 2), what="two of four blocks loaded")
    with pytest.raises(R.BsError) as e:
        layer.forward(xt.cuda(), 3)
    assert e.value.status == R.BS_ERR_RANGE
    layer.set_loaded(4)
    layer.drop()
    assert layer.n_blocks == 3
    assert_close(_forward(layer, xt, 3), pc.y_ref(x, 3), what="after a drop")
    W = layer.reconstruct(3).cpu().numpy().astype(np.float64)
    Wr = linear.reconstruct_plain(pc.Us, pc.Vs, pc.inv_s, 3, pc.m)
    assert np.max(np.abs(W - Wr)) <= 1e-5 * np.max(np.abs(Wr))
    assert not layer.reconstruct(0).abs().sum().item()


def test_plain_stack_rejects_sign_calls():
    pc = synthetic_case(128, 256, 16, 1, 64)
    layer = pc.layer()
    with pytest.raises(R.BsError) as e:
        layer.unpack_signs(0)
    assert e.value.status == R.BS_ERR_INVALID_ARG
    x = torch.zeros((1, pc.d), dtype=torch.float16, device="cuda")
    y = torch.empty((1, pc.m), dtype=torch.float16, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_linear_no_alloc(layer.handle, x, 1, y)
    assert e.value.status == R.BS_ERR_INVALID_ARG
    # a workspace one byte short is refused before any launch
    need = R.bs_plain_workspace_bytes(pc.m, pc.d, pc.kp, 1, 1)
    ws = torch.zeros(need - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_linear(layer.handle, x, 1, y, ws)
    assert e.value.status == R.BS_ERR_CAPACITY
