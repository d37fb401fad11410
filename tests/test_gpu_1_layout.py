"""GPU: block stack layout, append/drop bookkeeping, sign unpacking, reconstruction.

Bit-exact checks: the device stack bytes equal the oracle's records after append/drop
sequences, and the GPU unpack of every block equals the oracle's signs."""
import numpy as np
import pytest
import torch

import residual_block_decomp_b200 as R
import workloads as wl
from tests import cases
from tests.gpu_util import load_stack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def c1():
    return cases.config1()


def test_append_drop_bytes_bit_exact(c1):
    layer = load_stack(c1, n_append=0, capacity=4)
    assert layer.n_blocks == 0
    for i in range(4):
        layer.append()
        assert layer.n_blocks == i + 1
    torch.cuda.synchronize()
    for i in range(4):
        assert np.array_equal(layer.device_record(i).cpu().numpy(), c1.records[i])
    # offload two, load them again: slots are overwritten by the same bytes
    layer.drop()
    layer.drop()
    assert layer.n_blocks == 2
    layer.device_record(2).zero_()
    layer.device_record(3).zero_()
    layer.append()
    layer.append()
    torch.cuda.synchronize()
    for i in range(4):
        assert np.array_equal(layer.device_record(i).cpu().numpy(), c1.records[i])
    # a fifth block does not fit a capacity-4 stack
    with pytest.raises(R.BsError) as e:
        R.bs_append_block(layer.handle, layer.host_records[0])
    assert e.value.status == R.BS_ERR_CAPACITY
    assert layer.n_blocks == 4


def test_unpack_signs_bit_exact(c1):
    layer = load_stack(c1)
    for i in range(c1.n):
        s = layer.unpack_signs(i).cpu().numpy()
        assert np.array_equal(s < 0, c1.negs[i])
        assert set(np.unique(s).tolist()) <= {-1, 1}


def test_unpack_signs_multi_tile():
    st = cases.synthetic_stack(90, 384, 768, 2)
    layer = load_stack(st)
    for i in range(2):
        assert np.array_equal(layer.unpack_signs(i).cpu().numpy() < 0, st.negs[i])


@pytest.mark.parametrize("dtype,tol", [(torch.float32, 1e-5), (torch.float16, 2.0 ** -10),
                                       (torch.bfloat16, 2.0 ** -8)])
def test_reconstruct_parity(c1, dtype, tol):
    layer = load_stack(c1)
    for n in range(0, c1.n + 1):
        W = layer.reconstruct(n, dtype).float().cpu().numpy().astype(np.float64)
        ref = c1.w_ref(n)
        if n == 0:
            assert not W.any()
            continue
        assert np.max(np.abs(W - ref)) <= tol * np.max(np.abs(ref)), n


def test_reconstruct_multi_tile_synthetic():
    st = cases.synthetic_stack(91, 256, 1024, 3)
    layer = load_stack(st)
    W = layer.reconstruct(3).cpu().numpy().astype(np.float64)
    ref = st.w_ref(3)
    assert np.max(np.abs(W - ref)) <= 1e-5 * np.max(np.abs(ref))
