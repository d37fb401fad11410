"""GPU: the prefill kernel (batch > 4: W_hat tiles rebuilt on chip + tcgen05 GEMM)."""
import numpy as np
import pytest
import torch

from tests import cases
from tests.gpu_util import assert_close, load_stack

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,d,n,M,dtype", [
    (128, 256, 1, 5, "bf16"),       # smallest prefill batch, one token tile
    (256, 512, 3, 40, "bf16"),      # ragged token tile
    (256, 512, 3, 40, "f16"),
    (384, 1024, 9, 100, "bf16"),    # two P rounds (n > 8)
    (512, 768, 12, 300, "f16"),     # two token tiles, the second ragged
    (1024, 2048, 8, 16, "f16"),     # a decode batch of 16 through the prefill path
    (640, 2560, 5, 600, "bf16"),    # five token tiles: clusters of 4 sharing the rebuild, the last padded
    (256, 1024, 16, 2100, "f16"),   # 256-token tiles in clusters of 4, 16 blocks
])
def test_prefill_shapes(m, d, n, M, dtype):
    st = cases.synthetic_stack(94, m, d, n, matrix=m + n)
    layer = load_stack(st)
    x, xt = cases.inputs(94, M, d, matrix=M, dtype=dtype)
    y = layer.forward(xt.cuda(), n)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert_close(y, st.y_ref(x, n), what=f"prefill {m}x{d} n={n} M={M} {dtype}")


def test_prefill_all_n_small():
    st = cases.config1()
    layer = load_stack(st)
    x, xt = cases.inputs(1, 64, st.d, dtype="bf16")
    for n in range(1, st.n + 1):
        y = layer.forward(xt.cuda(), n)
        torch.cuda.synchronize()
        assert_close(y, st.y_ref(x, n), what=f"config 1 prefill n={n}")
