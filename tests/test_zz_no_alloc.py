"""GPU: bs_linear_no_alloc, the decode entry point that allocates nothing.

Some callers cannot hand the library a workspace (plugin hosts that pass only inputs
and outputs, serving loops that forbid device allocation after start-up).  For them
bs_linear_no_alloc keeps its scratch in a fixed array inside the library.  This test
calls it through the C ABI twice in a row and checks each output against the
workspace entry point bs_linear on the same inputs, within the tolerance the other
parity tests use.  It sits in a file of its own that pytest collects last."""
import numpy as np
import pytest
import torch

import residual_block_decomp_b200 as R
from residual_block_decomp_b200 import BitStackLinear
from tests import cases
from tests.gpu_util import assert_close, load_stack

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,d,n,b,dtype", [(512, 1024, 4, 1, "f16"), (4096, 4096, 8, 1, "f16"),
                                           (640, 1280, 3, 3, "bf16")])
def test_no_alloc_matches_workspace_entry_point(m, d, n, b, dtype):
    st = cases.synthetic_stack(97, m, d, n, matrix=m + b)
    layer = load_stack(st)
    _, xt = cases.inputs(97, b, d, matrix=b, dtype=dtype)
    x = xt.cuda()
    y_ws = layer.forward(x, n)                    # the existing entry point, with a workspace
    torch.cuda.synchronize()
    ref = y_ws.double().cpu().numpy()
    for call in range(2):                         # two calls in a row share the scratch array
        y = torch.full_like(y_ws, float("nan"))
        R.bs_linear_no_alloc(layer.handle, x, n, y)
        torch.cuda.synchronize()
        assert layer.device_error() == R.BS_OK
        assert_close(y, ref, what=f"no-alloc call {call} {m}x{d} n={n} b={b} {dtype}")


def test_no_alloc_rejects_oversize_and_prefill_batches():
    st = cases.synthetic_stack(97, 128, 16384, 5, matrix=2)
    layer = load_stack(st)
    # batch 5 is the prefill path, which needs no scratch: not offered here
    x5 = torch.zeros((5, st.d), dtype=torch.float16, device="cuda")
    y5 = torch.empty((5, st.m), dtype=torch.float16, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_linear_no_alloc(layer.handle, x5, 5, y5)
    assert e.value.status == R.BS_ERR_INVALID_ARG
    # 128 x 16384, n = 5 at batch 1 fits, and agrees with the workspace entry point
    _, xt = cases.inputs(97, 1, st.d, matrix=7)
    x1 = xt.cuda()
    y_ws = layer.forward(x1, 5)
    y1 = torch.empty_like(y_ws)
    R.bs_linear_no_alloc(layer.handle, x1, 5, y1)
    torch.cuda.synchronize()
    assert_close(y1, y_ws.double().cpu().numpy(), what="128x16384 n=5 b=1")
    # 9 blocks of 2048 x 16384 at batch 4 need more scratch than the 8 MiB array
    # (zero records: only the size check runs)
    m, d, n = 2048, 16384, 9
    assert R.bs_workspace_bytes(m, d, 16, n, 4) > 8 << 20
    big = BitStackLinear(m, d, n, np.ones(d, dtype=np.float32))
    for _ in range(n):
        big.add_record(np.zeros(big.block_bytes, dtype=np.uint8))
    big.set_loaded(n)
    torch.cuda.synchronize()
    x4 = torch.zeros((4, d), dtype=torch.float16, device="cuda")
    y4 = torch.empty((4, m), dtype=torch.float16, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_linear_no_alloc(big.handle, x4, n, y4)
    assert e.value.status == R.BS_ERR_CAPACITY
