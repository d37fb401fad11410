"""GPU: one decode launch over many linears (bs_linear_group).

A grouped launch must give, for every linear, the same bits as one bs_linear call per
linear (the same units, sets and fixed-order sums), and within the parity bar of the
oracle where the oracle is run.  The model cases follow the whole-model workload:
Llama-3-8B-shaped linears with per-linear loaded counts from a greedy fill of a memory
budget over a global block order, then budget changes between tokens (blocks dropped
and appended) with the same workspace."""
import numpy as np
import pytest
import torch

import residual_block_decomp_b200 as R
import workloads as wl
from oracle import budget, pack
from residual_block_decomp_b200 import BitStackLinear
from residual_block_decomp_b200.layer import record_from_parts
from tests import cases
from tests.gpu_util import assert_close, load_stack
from tests.test_decode_geometry import group_ws_bytes

pytestmark = pytest.mark.gpu


def random_stack(m, d, cap, gen, n_records=None):
    """A stack of random records (random sign words, decomposition-scale factors)."""
    layer = BitStackLinear(m, d, cap, wl.synthetic_inv_scale(d, gen))
    for i in range(cap if n_records is None else n_records):
        words = gen.integers(0, 2 ** 32, size=m * d // 32, dtype=np.uint64).astype(np.uint32)
        U = wl.random_factors(m, 16, gen, 0.12 / np.sqrt(i + 1.0))
        V = wl.random_factors(d, 16, gen, 0.12 / np.sqrt(i + 1.0))
        layer.add_record(record_from_parts(words, U, V))
    return layer


def run_group(layers, xs, counts, ws=None):
    b = xs[0].shape[0]
    ys = [torch.full((b, L.m), float("nan"), dtype=xs[0].dtype, device="cuda") for L in layers]
    need = R.bs_group_workspace_bytes([L.handle for L in layers], counts, b)
    if ws is None:
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    R.bs_linear_group([L.handle for L in layers], xs, counts, ys, ws)
    torch.cuda.synchronize()
    assert layers[0].device_error() == R.BS_OK
    return ys, ws


def singles(layers, xs, counts):
    out = []
    for L, x, n in zip(layers, xs, counts):
        out.append(L.forward(x, n))
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("b,dtype", [(1, "f16"), (3, "bf16")])
def test_small_group_matches_oracle_and_singles(b, dtype):
    shapes = [(128, 256, 1), (256, 512, 3), (384, 768, 2), (128, 256, 0), (1024, 4096, 5), (512, 2560, 4)]
    stacks = [cases.synthetic_stack(71, m, d, max(n, 1), matrix=j) for j, (m, d, n) in enumerate(shapes)]
    layers = [load_stack(st) for st in stacks]
    counts = [n for (_, _, n) in shapes]
    xin = [cases.inputs(71, b, d, matrix=j, dtype=dtype) for j, (_, d, _) in enumerate(shapes)]
    xs = [xt.cuda() for (_, xt) in xin]
    assert R.bs_group_workspace_bytes([L.handle for L in layers], counts, b) == group_ws_bytes(shapes, b)
    ys, ws = run_group(layers, xs, counts)
    ref = singles(layers, xs, counts)
    for j, (st, (x64, _), n) in enumerate(zip(stacks, xin, counts)):
        if n == 0:
            assert not ys[j].float().abs().sum().item()
            continue
        assert torch.equal(ys[j], ref[j]), f"linear {j}: grouped and single launches differ"
        assert_close(ys[j], st.y_ref(x64, n), what=f"grouped linear {j} {st.m}x{st.d} n={n} b={b}")
    # the same workspace again (the counters were left at zero)
    ys2, _ = run_group(layers, xs, counts, ws)
    assert all(torch.equal(a, c) for a, c in zip(ys, ys2))


def _model(layers_n, cap, gen):
    shapes = [(m, d) for _ in range(layers_n) for (_, m, d) in wl.LLAMA3_8B_LINEARS]
    return shapes, [random_stack(m, d, cap, gen) for (m, d) in shapes]


def test_model_group_across_budget_changes():
    """Two decoder layers (14 linears, 16-block stacks): per-linear counts from the greedy
    fill of a budget over the seeded global order, for three budgets in turn, blocks
    dropped and appended between tokens; grouped == single launches bit for bit."""
    gen = wl.generator(5, 0, "blocks")
    shapes, layers = _model(2, 16, gen)
    sizes = np.array([pack.block_bytes(m, d, 16) for (m, d) in shapes])
    order = budget.global_order(wl.order_weights(len(shapes), wl.generator(5, 0, "order")), 16)
    per_layer_mib = sizes.sum() / 2 ** 20 / 2          # one block of every linear of one layer
    ws = None
    xs = [torch.randn((1, d), device="cuda").half() for (_, d) in shapes]
    for scale in (3.0, 2.0, 4.5):
        counts = budget.budget_fill(order, sizes, scale * per_layer_mib).tolist()
        for L, n in zip(layers, counts):
            L.set_loaded(n)
        torch.cuda.synchronize()
        need = R.bs_group_workspace_bytes([L.handle for L in layers], counts, 1)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(max(need, 1), dtype=torch.uint8, device="cuda")
        ys, _ = run_group(layers, xs, counts, ws)
        ref = singles(layers, xs, counts)
        for j in range(len(layers)):
            assert torch.equal(ys[j], ref[j]), f"budget x{scale}: linear {j} ({shapes[j]}, n={counts[j]})"


def test_group_argument_errors():
    gen = wl.generator(5, 1, "blocks")
    layers = [random_stack(128, 256, 2, gen), random_stack(256, 512, 2, gen)]
    hs = [L.handle for L in layers]
    for L in layers:
        L.set_loaded(2)
    xs = [torch.zeros((1, 256), dtype=torch.float16, device="cuda"), torch.zeros((1, 512), dtype=torch.float16,
                                                                                 device="cuda")]
    ys = [torch.empty((1, 128), dtype=torch.float16, device="cuda"), torch.empty((1, 256), dtype=torch.float16,
                                                                                 device="cuda")]
    need = R.bs_group_workspace_bytes(hs, [2, 2], 1)
    with pytest.raises(R.BsError) as e:
        R.bs_linear_group(hs, xs, [2, 3], ys, torch.zeros(need, dtype=torch.uint8, device="cuda"))
    assert e.value.status == R.BS_ERR_RANGE
    with pytest.raises(R.BsError) as e:
        R.bs_linear_group(hs, xs, [2, 2], ys, torch.zeros(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == R.BS_ERR_CAPACITY
    x5 = [torch.zeros((5, 256), dtype=torch.float16, device="cuda"), torch.zeros((5, 512), dtype=torch.float16,
                                                                                 device="cuda")]
    with pytest.raises(R.BsError) as e:
        R.bs_linear_group(hs, x5, [2, 2], ys, torch.zeros(need, dtype=torch.uint8, device="cuda"))
    assert e.value.status == R.BS_ERR_INVALID_ARG
    assert R.bs_group_workspace_bytes(hs, [2, -1], 1) == 0
