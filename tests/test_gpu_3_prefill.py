"""GPU: the prefill kernel (batch > 4: W_hat tiles rebuilt on chip + tcgen05 GEMM).

Grids that would leave SMs idle split K (the partials summed by the last CTA of each
tile), so most shapes below run split: 40 tokens of 256 x 512 in 2 splits, 16 tokens of
1024 x 2048 in 8, 600 tokens of 640 x 2560 in splits of 32, 32 and 16 K-tiles with
clusters of 4; each is called twice on one workspace (the counters must come back to
zero) and once without a workspace (one pass over K)."""
import numpy as np
import pytest
import torch

import residual_block_decomp_b200 as R
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
    ref = st.y_ref(x, n)
    y = layer.forward(xt.cuda(), n)
    y2 = layer.forward(xt.cuda(), n)          # same workspace: counters back at zero
    y3 = torch.empty_like(y)
    R.bs_linear(layer.handle, xt.cuda(), n, y3, None)   # no workspace: one pass over K
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert_close(y, ref, what=f"prefill {m}x{d} n={n} M={M} {dtype}")
    assert torch.equal(y, y2), "a second call on the same workspace differs"
    assert_close(y3, ref, what=f"prefill {m}x{d} n={n} M={M} {dtype} without a workspace")
    if layer._ws is not None:
        cnt = layer._ws[:256].cpu()
        assert int(cnt.sum()) == 0, "split-K counters not left at zero"


def test_prefill_all_n_small():
    st = cases.config1()
    layer = load_stack(st)
    x, xt = cases.inputs(1, 64, st.d, dtype="bf16")
    for n in range(1, st.n + 1):
        y = layer.forward(xt.cuda(), n)
        torch.cuda.synchronize()
        assert_close(y, st.y_ref(x, n), what=f"config 1 prefill n={n}")
