"""GPU: bs_linear_no_alloc, the decode entry point that allocates nothing.

Some callers cannot hand the library a workspace (plugin hosts that pass only inputs
and outputs, serving loops that forbid device allocation after start-up).  For them
bs_linear_no_alloc keeps its scratch in a fixed array inside the library.  These
tests call it through the C ABI twice in a row and check each output against the
CPU oracle, within the tolerance the other parity tests use, and against the
workspace entry point bs_linear (the same kernels: identical bits).  The array is
shared by every stack on a device, so a timed-out call on one stack must not leave
the next no-alloc call on another stack wrong.  The file is collected last."""
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
def test_no_alloc_matches_oracle_and_workspace_entry_point(m, d, n, b, dtype):
    st = cases.synthetic_stack(97, m, d, n, matrix=m + b)
    layer = load_stack(st)
    x64, xt = cases.inputs(97, b, d, matrix=b, dtype=dtype)
    x = xt.cuda()
    ref = st.y_ref(x64, n)                        # the oracle, float64
    y_ws = layer.forward(x, n)                    # the workspace entry point
    torch.cuda.synchronize()
    for call in range(2):                         # two calls in a row share the scratch array
        y = torch.full_like(y_ws, float("nan"))
        R.bs_linear_no_alloc(layer.handle, x, n, y)
        torch.cuda.synchronize()
        assert layer.device_error() == R.BS_OK
        assert_close(y, ref, what=f"no-alloc call {call} {m}x{d} n={n} b={b} {dtype}")
        assert torch.equal(y, y_ws), "no-alloc and workspace entry points differ"


def test_no_alloc_recovers_after_a_timeout_on_another_stack():
    """A call that runs out of its bounded waits can leave row-tile counters behind in
    the shared array (the timed-out CTA never counts its partials, the others do).
    Once the error has been read on stack A, the next no-alloc call on the device --
    here on stack B -- must clear the array first and give the right answer."""
    a = cases.synthetic_stack(98, 1024, 4096, 4, matrix=1)
    b = cases.synthetic_stack(98, 1024, 4096, 4, matrix=2)
    la, lb = load_stack(a), load_stack(b)
    xa64, xat = cases.inputs(98, 1, a.d, matrix=1)
    xb64, xbt = cases.inputs(98, 1, b.d, matrix=2)
    xa, xb = xat.cuda(), xbt.cuda()
    ya = torch.empty((1, a.m), dtype=torch.float16, device="cuda")
    R.bs_debug_set_wait(la.handle, 2_000_000, unreachable_flag=True)   # CTA 0 loses its first copy
    R.bs_linear_no_alloc(la.handle, xa, 4, ya)
    torch.cuda.synchronize()
    assert la.device_error() == R.BS_ERR_TIMEOUT
    R.bs_debug_set_wait(la.handle, 500_000_000, unreachable_flag=False)
    for _ in range(2):
        yb = torch.full((1, b.m), float("nan"), dtype=torch.float16, device="cuda")
        R.bs_linear_no_alloc(lb.handle, xb, 4, yb)
        torch.cuda.synchronize()
        assert lb.device_error() == R.BS_OK
        assert_close(yb, b.y_ref(xb64, 4), what="stack B after a timeout on stack A")
        ya = torch.full((1, a.m), float("nan"), dtype=torch.float16, device="cuda")
        R.bs_linear_no_alloc(la.handle, xa, 4, ya)
        torch.cuda.synchronize()
        assert la.device_error() == R.BS_OK
        assert_close(ya, a.y_ref(xa64, 4), what="stack A after its own timeout")


def test_no_alloc_rejects_oversize_and_prefill_batches():
    st = cases.synthetic_stack(97, 128, 16384, 5, matrix=2)
    layer = load_stack(st)
    # batch 5 is the prefill path, which needs no scratch: not offered here
    x5 = torch.zeros((5, st.d), dtype=torch.float16, device="cuda")
    y5 = torch.empty((5, st.m), dtype=torch.float16, device="cuda")
    with pytest.raises(R.BsError) as e:
        R.bs_linear_no_alloc(layer.handle, x5, 5, y5)
    assert e.value.status == R.BS_ERR_INVALID_ARG
    # 128 x 16384, n = 5 at batch 1 fits, and agrees with the oracle
    x64, xt = cases.inputs(97, 1, st.d, matrix=7)
    x1 = xt.cuda()
    y1 = torch.empty((1, st.m), dtype=torch.float16, device="cuda")
    R.bs_linear_no_alloc(layer.handle, x1, 5, y1)
    torch.cuda.synchronize()
    assert_close(y1, st.y_ref(x64, 5), what="128x16384 n=5 b=1")
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
