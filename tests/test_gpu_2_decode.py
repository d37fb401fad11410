"""GPU: the decode kernel (batch <= 4) against the oracle.

Bar: max|y - y_ref| <= 2e-3 * max|y_ref| (fp16/bf16 operands, fp64 oracle)."""
import numpy as np
import pytest
import torch

from tests import cases
from tests.gpu_util import TOL, assert_close, load_stack

pytestmark = pytest.mark.gpu


def _run(layer, xt, n):
    y = layer.forward(xt.cuda(), n)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    return y


def test_config1_all_n():
    st = cases.config1()
    layer = load_stack(st)
    x, xt = cases.inputs(1, 1, st.d)
    for n in range(0, st.n + 1):
        y = _run(layer, xt, n)
        if n == 0:
            assert not y.float().abs().sum().item()
        else:
            assert_close(y, st.y_ref(x, n), what=f"config 1, n={n}")


@pytest.mark.parametrize("m,d,n,b,dtype", [
    (128, 256, 1, 1, "f16"),      # a single unit
    (256, 512, 3, 2, "f16"),
    (384, 768, 2, 3, "bf16"),     # rows split unevenly across CTAs
    (640, 1280, 4, 4, "f16"),
    (1024, 4096, 5, 1, "bf16"),
    (512, 2560, 7, 2, "f16"),
])
def test_decode_shapes(m, d, n, b, dtype):
    st = cases.synthetic_stack(92, m, d, n, matrix=m + d + n)
    layer = load_stack(st)
    x, xt = cases.inputs(92, b, d, matrix=m, dtype=dtype)
    y = _run(layer, xt, n)
    assert_close(y, st.y_ref(x, n), what=f"{m}x{d} n={n} b={b} {dtype}")


@pytest.fixture(scope="module")
def c2():
    return cases.config2()


@pytest.mark.parametrize("b", [1, 4])
def test_config2_sweep(c2, b):
    layer = load_stack(c2)
    x, xt = cases.inputs(2, b, c2.d)
    worst = 0.0
    for n in range(1, c2.n + 1):
        y = _run(layer, xt, n)
        worst = max(worst, assert_close(y, c2.y_ref(x, n), what=f"config 2 b={b} n={n}"))
    print(f"config 2 b={b}: worst max|err|/max|y| = {worst:.2e} (bar {TOL})")


def test_decode_is_deterministic_across_calls(c2):
    layer = load_stack(c2)
    _, xt = cases.inputs(2, 1, c2.d)
    y1 = _run(layer, xt, 8).clone()
    y2 = _run(layer, xt, 8).clone()
    assert torch.equal(y1, y2)


def test_decode_shared_workspace_between_stacks():
    a = cases.synthetic_stack(93, 256, 512, 2, matrix=1)
    b = cases.synthetic_stack(93, 512, 512, 3, matrix=2)
    la, lb = load_stack(a), load_stack(b)
    ws = torch.zeros(max(la.workspace(2, 1).numel(), lb.workspace(3, 1).numel()), dtype=torch.uint8, device="cuda")
    x, xt = cases.inputs(93, 1, 512)
    ya = la.forward(xt.cuda(), 2, workspace=ws)
    yb = lb.forward(xt.cuda(), 3, workspace=ws)
    torch.cuda.synchronize()
    assert_close(ya, a.y_ref(x, 2), what="stack a")
    assert_close(yb, b.y_ref(x, 3), what="stack b")


def test_decode_workspace_reused_across_n_and_batch():
    """One workspace, sized for the largest call, serves calls with other n_loaded and
    batch in any order: the row-tile counters sit at a fixed place and every call
    leaves them at zero, while the partial outputs move with the sizes."""
    st = cases.synthetic_stack(97, 512, 1024, 4, matrix=7)
    layer = load_stack(st)
    need = max(layer.workspace(n, b).numel() for n in (1, 4) for b in (1, 4))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for n, b in [(4, 1), (1, 1), (3, 4), (1, 2), (4, 4), (2, 1), (4, 1)]:
        x, xt = cases.inputs(97, b, st.d, matrix=10 * n + b)
        y = layer.forward(xt.cuda(), n, workspace=ws)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        assert_close(y, st.y_ref(x, n), what=f"reused workspace n={n} b={b}")
