"""GPU: configs 3-5 at full size against the oracle.

Config 3: Llama-3-8B MLP shapes, 12-block stacks, per-matrix n drawn from U{2..12},
decode batches 1, 4 and 16.  Config 4: prefill of 4096x4096 (the decomposed config-2
stack) and 14336x4096, 8 blocks, M in {512, 2048, 4096} bf16 tokens, checked on
sampled rows and tokens.  Config 5: the 224 linears of a 32-layer stack, per-matrix n
from the greedy fill of a 3000 MiB budget over the stand-in global order; one linear
of each kind is checked, then the budget moves to 2000 and 4500 MiB (blocks are
dropped and appended between tokens) and the same linears are checked again."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests import cases
from tests.gpu_util import assert_close, load_stack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mlp():
    n_draw = cases.config3_n_loaded(3)
    return {
        "gate": (cases.synthetic_stack(3, 14336, 4096, 12, matrix=0), int(n_draw[0])),
        "up": (cases.synthetic_stack(3, 14336, 4096, 12, matrix=1), int(n_draw[1])),
        "down": (cases.synthetic_stack(3, 4096, 14336, 12, matrix=2), int(n_draw[2])),
    }


@pytest.mark.parametrize("kind", ["gate", "up", "down"])
def test_config3_mlp(mlp, kind):
    st, n = mlp[kind]
    layer = load_stack(st)
    W = st.w_ref(n)
    for b in (1, 4, 16):
        x, xt = cases.inputs(3, b, st.d, matrix=b)
        y = layer.forward(xt.cuda(), n)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        assert_close(y, x @ W.T, what=f"config 3 {kind} n={n} b={b}")


def _sampled_check(y_gpu, x, W, what, n_rows=64, n_tok=48, seed=0):
    gen = np.random.default_rng(seed)
    M, m = y_gpu.shape
    rows = np.unique(np.concatenate([[0, m - 1], gen.choice(m, n_rows, replace=False)]))
    toks = np.unique(np.concatenate([[0, M - 1], gen.choice(M, min(n_tok, M), replace=False)]))
    y = y_gpu
    assert_close(y[:, torch.as_tensor(rows, device=y.device)], x @ W[rows].T, what=f"{what} sampled rows")
    assert_close(y[torch.as_tensor(toks, device=y.device)], x[toks] @ W.T, what=f"{what} sampled tokens")


@pytest.mark.parametrize("shape", ["4096x4096", "14336x4096"])
def test_config4_prefill(shape):
    st = cases.config2() if shape == "4096x4096" else cases.synthetic_stack(4, 14336, 4096, 8, matrix=1)
    layer = load_stack(st)
    W = st.w_ref(8)
    for M in (512, 2048, 4096):
        x, xt = cases.inputs(4, M, st.d, matrix=M, dtype="bf16")
        y = layer.forward(xt.cuda(), 8)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        _sampled_check(y, x, W, f"config 4 {shape} M={M}", seed=M)


def test_config5_budget_plan_and_swaps():
    plans = {mib: cases.config5_plan(mib) for mib in (3000, 2000, 4500)}
    mats, sizes, order, n3000 = plans[3000]
    for mib, (_, _, _, n) in plans.items():
        assert int(np.sum(n * sizes)) <= mib * 2 ** 20
    # one linear of each kind, from a seeded layer
    gen = wl.generator(5, 0, "x")
    picks = []
    for kind_idx in range(len(wl.LLAMA3_8B_LINEARS)):
        layer_idx = int(gen.integers(0, wl.LLAMA3_8B_LAYERS))
        picks.append(layer_idx * len(wl.LLAMA3_8B_LINEARS) + kind_idx)
    n_max = {g: max(int(plans[mib][3][g]) for mib in plans) for g in picks}
    layers = {}
    stacks = {}
    for g in picks:
        _, kind, m, d = mats[g]
        st = cases.synthetic_stack(5, m, d, max(n_max[g], 1), matrix=g)
        stacks[g] = st
        layers[g] = load_stack(st, n_append=0, capacity=16)
    for mib in (3000, 2000, 4500):
        n_plan = plans[mib][3]
        for g in picks:
            layers[g].set_loaded(int(n_plan[g]))   # drop or append between tokens
        torch.cuda.synchronize()
        for g in picks:
            st, layer = stacks[g], layers[g]
            n = int(n_plan[g])
            assert layer.n_blocks == n
            x, xt = cases.inputs(5, 1, st.d, matrix=g)
            y = layer.forward(xt.cuda(), n)
            torch.cuda.synchronize()
            if n == 0:
                assert not y.float().abs().sum().item()
            else:
                assert_close(y, st.y_ref(x, n), what=f"config 5 budget {mib} MiB {mats[g][1]} n={n}")
