"""Helpers of the GPU tests: load an oracle stack into the library, compare outputs."""
from __future__ import annotations

import numpy as np
import torch

from residual_block_decomp_b200 import BitStackLinear

TOL = 2e-3  # max|y - y_ref| <= TOL * max|y_ref|


def load_stack(st, n_append=None, capacity=None) -> BitStackLinear:
    cap = capacity or max(st.n, 1)
    layer = BitStackLinear(st.m, st.d, cap, st.inv_s)
    for rec in st.records:
        layer.add_record(rec)
    layer.set_loaded(st.n if n_append is None else n_append)
    torch.cuda.synchronize()
    return layer


def rel_err(y_gpu, y_ref) -> tuple[float, float]:
    y = y_gpu.float().cpu().numpy().astype(np.float64) if torch.is_tensor(y_gpu) else np.asarray(y_gpu, np.float64)
    err = float(np.max(np.abs(y - y_ref))) if y.size else 0.0
    scale = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    return err, scale


# Half a unit in the last place of a bf16 output, relative to the stored value.  A
# bf16 result's own final rounding (up to 2^-8 relative, 3.9e-3) can exceed the
# 2e-3 * max|y_ref| bar by itself, so for bf16 outputs the bar applies to the value
# before that rounding.  An fp16 result's rounding (at most 2^-11 relative) fits well
# inside the bar, so fp16 outputs get no allowance: they must meet the raw bar.
HALF_ULP = {torch.float16: 0.0, torch.bfloat16: 2.0 ** -8, torch.float32: 0.0}


def assert_close(y_gpu, y_ref, tol=TOL, what=""):
    """max|y - y_ref| <= tol * max|y_ref|; a bf16 output's elements are allowed the
    half-ulp rounding of bf16 on top, fp16 and fp32 outputs nothing."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    scale = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    excess = np.abs(y - y_ref) - HALF_ULP[y_gpu.dtype] * np.abs(y)
    worst = float(np.max(excess)) if y.size else 0.0
    err = float(np.max(np.abs(y - y_ref))) if y.size else 0.0
    assert worst <= tol * scale, (f"{what}: max(|y - y_ref| - half-ulp) = {worst:.3e} > {tol} * max|y_ref| = "
                                  f"{tol * scale:.3e} (raw max|y - y_ref| = {err:.3e})")
    return max(worst, 0.0) / scale if scale else 0.0
