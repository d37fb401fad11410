"""GPU: error paths of the C ABI, and the bounded-wait timeout path.

The timeout is injected on the host: the decode call is told to leave out the first
sign-tile copy of every CTA, with a 2 ms bound on each wait.  The kernel records
BS_ERR_TIMEOUT in the stack's device error word, drains its copies and MMAs, frees
tensor memory and returns; the context stays usable, which the next call shows.
Nothing here faults, traps or hangs the GPU."""
import pytest
import torch

import residual_block_decomp_b200 as R
from tests import cases
from tests.gpu_util import assert_close, load_stack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def small():
    st = cases.synthetic_stack(95, 256, 512, 3)
    return st, load_stack(st)


def test_range_and_capacity_errors(small):
    st, layer = small
    _, xt = cases.inputs(95, 1, st.d)
    x = xt.cuda()
    y = torch.empty((1, st.m), dtype=x.dtype, device="cuda")
    ws = layer.workspace(3, 1)
    with pytest.raises(R.BsError) as e:
        R.bs_linear(layer.handle, x, 4, y, ws)
    assert e.value.status == R.BS_ERR_RANGE
    with pytest.raises(R.BsError) as e:
        R.bs_linear(layer.handle, x, 3, y, ws[:256])
    assert e.value.status == R.BS_ERR_CAPACITY
    with pytest.raises(R.BsError) as e:
        R.bs_linear(layer.handle, x, 3, y, None)
    assert e.value.status == R.BS_ERR_CAPACITY
    with pytest.raises(R.BsError) as e:
        R.bs_reconstruct(layer.handle, 4, torch.empty((st.m, st.d), device="cuda"))
    assert e.value.status == R.BS_ERR_RANGE
    with pytest.raises(R.BsError) as e:
        R.bs_unpack_signs(layer.handle, 3, torch.empty((st.m, st.d), dtype=torch.int8, device="cuda"))
    assert e.value.status == R.BS_ERR_RANGE


def test_alignment_errors(small):
    st, layer = small
    buf = torch.zeros(2 * st.d + 8, dtype=torch.float16, device="cuda")
    y = torch.empty((1, st.m), dtype=torch.float16, device="cuda")
    x_off = buf[1:1 + st.d].view(1, st.d)          # 2-byte offset
    with pytest.raises(R.BsError) as e:
        R.bs_linear(layer.handle, x_off, 3, y, layer.workspace(3, 1))
    assert e.value.status == R.BS_ERR_ALIGNMENT
    need = R.bs_workspace_bytes(st.m, st.d, 16, 3, 1)
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_linear(layer.handle, buf[:st.d].view(1, st.d), 3, y, ws[64:])   # 64-byte offset
    assert e.value.status == R.BS_ERR_ALIGNMENT


def test_drop_at_zero_is_rejected():
    st = cases.synthetic_stack(96, 128, 256, 1)
    layer = load_stack(st)
    layer.drop()
    with pytest.raises(R.BsError) as e:
        layer.drop()
    assert e.value.status == R.BS_ERR_RANGE
    assert layer.n_blocks == 0


def test_bounded_wait_times_out_and_context_survives(small):
    st, layer = small
    x, xt = cases.inputs(95, 1, st.d)
    R.bs_debug_set_wait(layer.handle, 2_000_000, unreachable_flag=True)
    layer.forward(xt.cuda(), 3)
    torch.cuda.synchronize()
    assert layer.device_error() == R.BS_ERR_TIMEOUT
    assert layer.device_error() == R.BS_OK          # the word was cleared by the read
    R.bs_debug_set_wait(layer.handle, 500_000_000, unreachable_flag=False)
    y = layer.forward(xt.cuda(), 3)
    torch.cuda.synchronize()
    assert layer.device_error() == R.BS_OK
    assert_close(y, st.y_ref(x, 3), what="after a timed-out call")
