"""Seeded test cases for configs 1-5, built with the oracle (test infrastructure).

Every case holds the oracle's blocks (signs, fp16 factors), the fp32 inverse scale,
the oracle-packed device records, and seeded inputs.  Nothing here comes from the
CUDA path.  Decompositions of large weights are cached under .oracle_cache/.
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field

import numpy as np

import workloads as wl
from oracle import budget, decompose, linear, pack

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CACHE = os.path.join(ROOT, ".oracle_cache")
K = 16


@dataclass
class Stack:
    m: int
    d: int
    negs: list = field(default_factory=list)
    Us: list = field(default_factory=list)
    Vs: list = field(default_factory=list)
    inv_s: np.ndarray | None = None
    records: list = field(default_factory=list)

    @property
    def n(self):
        return len(self.negs)

    def y_ref(self, x, n):
        return linear.linear_explicit(x, self.negs, self.Us, self.Vs, self.inv_s, n, self.m)

    def y_ref_rows(self, x, n, rows):
        return linear.linear_rows(x, self.negs, self.Us, self.Vs, self.inv_s, n, rows)

    def w_ref(self, n):
        return linear.reconstruct(self.negs, self.Us, self.Vs, self.inv_s, n, self.m)


def _records(st: Stack) -> Stack:
    st.records = [pack.make_record(a, u, v) for a, u, v in zip(st.negs, st.Us, st.Vs)]
    return st


def decomposed_stack(config: int, m: int, d: int, n_blocks: int, outlier_frac: float = 0.0,
                     matrix: int = 0, cache: bool = True) -> Stack:
    """W ~ N(0, 0.02^2) (with outlier input channels), calibration 64 x d N(0,1),
    decomposed by the oracle into n_blocks residual blocks with k = 16."""
    path = os.path.join(CACHE, f"dec_c{config}_m{matrix}_{m}x{d}_n{n_blocks}_o{outlier_frac}.npz")
    if cache and os.path.exists(path):
        z = np.load(path)
        st = Stack(m, d, [z[f"neg{i}"] for i in range(n_blocks)], [z[f"U{i}"] for i in range(n_blocks)],
                   [z[f"V{i}"] for i in range(n_blocks)], z["inv_s"])
        return _records(st)
    W = wl.weight(m, d, wl.generator(config, matrix, "W"), outlier_frac=outlier_frac,
                  outlier_gen=wl.generator(config, matrix, "outlier"))
    X = wl.calibration(64, d, wl.generator(config, matrix, "calib"))
    s = decompose.activation_scale(X)
    dec = decompose.decompose(W, s, n_blocks, K, wl.generator(config, matrix, "svd"))
    st = Stack(m, d, dec.neg, dec.U, dec.V, dec.inv_s)
    if cache:
        os.makedirs(CACHE, exist_ok=True)
        arrs = {"inv_s": dec.inv_s}
        for i in range(n_blocks):
            arrs[f"neg{i}"], arrs[f"U{i}"], arrs[f"V{i}"] = dec.neg[i], dec.U[i], dec.V[i]
        np.savez(path, **arrs)
    return _records(st)


def synthetic_stack(config: int, m: int, d: int, n_blocks: int, matrix: int = 0) -> Stack:
    """Random signs and factors shaped like decomposed blocks (timing-shaped data)."""
    gen = wl.generator(config, matrix, "blocks")
    st = Stack(m, d)
    for i in range(n_blocks):
        neg, U, V = wl.synthetic_block(m, d, K, gen, level=i)
        st.negs.append(neg)
        st.Us.append(U)
        st.Vs.append(V)
    st.inv_s = wl.synthetic_inv_scale(d, gen)
    return _records(st)


def inputs(config: int, b: int, d: int, matrix: int = 0, dtype: str = "f16"):
    """(x as the exact values in float64, x as a torch CPU tensor of the dtype)."""
    import torch
    x32 = wl.activations(b, d, wl.generator(config, matrix, "x"))
    if dtype == "f16":
        xt = torch.from_numpy(x32.astype(np.float16))
    else:
        xt = torch.from_numpy(wl.to_bf16_bits(x32).view(np.int16)).view(torch.bfloat16)
    return xt.float().double().numpy(), xt


def config1() -> Stack:
    return decomposed_stack(1, 512, 512, 4)


def config2() -> Stack:
    return decomposed_stack(2, 4096, 4096, 8, outlier_frac=0.01)


def config3_n_loaded(count: int = 3) -> np.ndarray:
    return wl.n_loaded_draws(count, wl.generator(3, 0, "n"))


def config5_plan(budget_mib: float):
    """(matrices, per-matrix block bytes, global order, per-matrix n) for a budget."""
    mats = wl.llama3_8b_matrices()
    sizes = np.array([pack.block_bytes(m, d, K) for (_, _, m, d) in mats], dtype=np.int64)
    wts = wl.order_weights(len(mats), wl.generator(5, 0, "order"))
    order = budget.global_order(wts, 16)
    return mats, sizes, order, budget.budget_fill(order, sizes, budget_mib)
