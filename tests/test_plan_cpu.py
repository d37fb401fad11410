"""CPU: the load-order planner (bs_plan_order / bs_plan_budget) and its oracle.

First the oracle's orders are pinned to things other than themselves: brute force
over every prefix-closed loading of tiny stacks (Greedy is the best energy drop for
its bytes when scores fall within each weight), a library sort (the same case), the
level-major closed form (Average), hand-worked draws (Random), and residual
energies recomputed from reconstructed weights (the scores).  Planted mistakes in
the oracle must fail these pins.  Then the C ABI must give the oracle's orders and
budget fills exactly, on random instances and on the 224 linears of an 8B model.
"""
import itertools

import numpy as np
import pytest

import residual_block_decomp_b200 as R
import workloads as wl
from oracle import budget, decompose, linear, pack


def _is_prefix_order(order, counts):
    seen = [0] * len(counts)
    for (w, i) in order:
        if i != seen[w]:
            return False
        seen[w] += 1
    return seen == [int(c) for c in counts]


def _falling_scores(gen, counts, levels):
    """Per-weight scores that fall with the block index (as energy drops of a
    decomposition do), padded to ``levels`` columns with NaN."""
    out = np.full((len(counts), levels), np.nan)
    for w, c in enumerate(counts):
        out[w, :c] = np.sort(gen.random(c))[::-1] * gen.uniform(0.5, 2.0)
    return out


def _rows(scores, counts):
    return [list(scores[w, :c]) for w, c in enumerate(counts)]


# ------------------------------------------------------------------ oracle pins ----
def test_greedy_is_optimal_for_its_bytes_by_brute_force():
    """Every prefix of the Greedy order holds the largest energy drop of all loadings
    (block counts per weight) that take no more bytes, when scores fall within each
    weight: the fractional-knapsack exchange argument, checked exhaustively."""
    gen = np.random.default_rng(11)
    for trial in range(20):
        counts = [int(c) for c in gen.integers(0, 4, size=3)]
        sizes = [int(s) for s in gen.integers(1, 5, size=3)]
        sc = _falling_scores(gen, counts, max(max(counts), 1))
        order = budget.order_greedy(_rows(sc, counts))
        assert _is_prefix_order(order, counts)
        gain = lambda n: sum(sc[w, i] * sizes[w] for w in range(3) for i in range(n[w]))
        n = [0, 0, 0]
        for (w, _) in order:
            n[w] += 1
            used = sum(n[j] * sizes[j] for j in range(3))
            best = max(gain(c) for c in itertools.product(*[range(k + 1) for k in counts])
                       if sum(c[j] * sizes[j] for j in range(3)) <= used)
            assert gain(n) >= best - 1e-12, (trial, counts, sizes, n)


def test_greedy_equals_a_stable_sort_when_scores_fall():
    """With scores falling within each weight, Greedy is the descending sort of all
    blocks by score (ties: lower weight first, then lower block)."""
    gen = np.random.default_rng(12)
    counts = [5, 0, 3, 7, 1]
    sc = _falling_scores(gen, counts, 7)
    sc[2, 1] = sc[0, 2]                      # a tie across weights
    entries = [(w, i) for w in range(5) for i in range(counts[w])]
    want = sorted(entries, key=lambda e: (-sc[e[0], e[1]], e[0], e[1]))
    assert budget.order_greedy(_rows(sc, counts)) == want


def test_greedy_waits_for_a_blocked_better_block():
    """A weight whose first block scores low but second high is taken only when its
    next block wins: Greedy looks at the next block of each weight, not at all."""
    got = budget.order_greedy([[1.0, 9.0], [3.0, 2.0]])
    assert got == [(1, 0), (1, 1), (0, 0), (0, 1)]


def test_average_is_level_major():
    counts = [4] * 6
    order = budget.order_average(counts)
    assert [order.index((w, i)) for w in range(6) for i in range(4)] == [i * 6 + w for w in range(6) for i in range(4)]
    # unequal counts: in every prefix, the weights that still have blocks differ by at
    # most one in their loaded counts
    counts = [3, 0, 5, 1, 4]
    order = budget.order_average(counts)
    assert _is_prefix_order(order, counts)
    n = [0] * 5
    for (w, _) in order:
        n[w] += 1
        live = [n[j] for j in range(5) if counts[j] > n[j] or j == w]
        assert max(live) - min(live) <= 1


def test_random_order_special_draws():
    counts = [2, 3, 1]
    # u = 0 always picks the lowest weight with blocks left: weight-major order
    assert budget.order_random(counts, [0.0] * 6) == [(0, 0), (0, 1), (1, 0), (1, 1), (1, 2), (2, 0)]
    # u just below 1 picks the highest such weight
    top = float(np.nextafter(1.0, 0.0))
    assert budget.order_random(counts, [top] * 6) == [(2, 0), (1, 0), (1, 1), (1, 2), (0, 0), (0, 1)]
    # worked by hand: live {0,1,2}: 0.5*3 -> #1 = weight 1; live {0,1,2}: 0.9*3 -> #2 =
    # weight 2 (now empty); live {0,1}: 0.2*2 -> weight 0; 0.7*2 -> weight 1;
    # 0.6*2 -> weight 1 (now empty); live {0}: weight 0
    assert budget.order_random(counts, [0.5, 0.9, 0.2, 0.7, 0.6, 0.3]) == \
        [(1, 0), (2, 0), (0, 0), (1, 1), (1, 2), (0, 1)]


def test_random_first_pick_is_uniform():
    counts = [2] * 8
    gen = np.random.default_rng(13)
    firsts = np.bincount([budget.order_random(counts, gen.random(16))[0][0] for _ in range(4000)], minlength=8)
    assert firsts.min() > 400 and firsts.max() < 600      # 500 expected, sd ~ 21


def test_scores_are_energy_drops_per_byte_of_a_real_decomposition():
    """block_scores times the block bytes sums to ||W s||^2 - ||W s - W_hat_n s||^2,
    the residual energies recomputed from the reconstructed scaled weight."""
    gen = np.random.default_rng(14)
    m, d, k, n = 48, 32, 4, 3
    W = wl.weight(m, d, gen).astype(np.float64)
    s = decompose.activation_scale(wl.calibration(64, d, gen))
    dec = decompose.decompose(W, s, n, k, round_fp16=False)
    nbytes = pack.block_bytes(m, d, k)
    sc = budget.block_scores(dec.res_norms, nbytes)
    Ws = W * s[None, :]
    for j in range(n + 1):
        Rj = Ws - linear.reconstruct_scaled(dec.neg, dec.U, dec.V, j, m, d)
        drop = float(np.sum(Ws ** 2) - np.sum(Rj ** 2))
        assert float(np.sum(sc[:j])) * nbytes == pytest.approx(drop, rel=1e-9, abs=1e-9 * float(np.sum(Ws ** 2)))
    assert np.all(sc > 0) and np.all(np.diff(sc) <= 0)     # each block removes less


def _planner_pins_pass():
    try:
        test_greedy_is_optimal_for_its_bytes_by_brute_force()
        test_greedy_equals_a_stable_sort_when_scores_fall()
        test_greedy_waits_for_a_blocked_better_block()
        test_average_is_level_major()
        test_random_order_special_draws()
        test_scores_are_energy_drops_per_byte_of_a_real_decomposition()
    except AssertionError:
        return False
    return True


def test_planted_planner_mistakes_are_caught(monkeypatch):
    assert _planner_pins_pass()
    real_greedy, real_random, real_scores = budget.order_greedy, budget.order_random, budget.block_scores

    def lowest_first(scores):                    # comparison turned around
        return real_greedy([[-v for v in row] for row in scores])

    def ties_to_higher_weight(scores):           # tie-break turned around
        out = real_greedy(scores[::-1])
        return [(len(scores) - 1 - w, i) for (w, i) in out]

    def weight_major(counts):                    # Average without the levels
        return [(w, i) for w, c in enumerate(counts) for i in range(int(c))]

    def draw_over_all_weights(counts, draws):    # picks among all weights, not the live ones
        counts = [int(c) for c in counts]
        nxt, out = [0] * len(counts), []
        for t in range(sum(counts)):
            w = min(int(draws[t] * len(counts)), len(counts) - 1)
            while nxt[w] >= counts[w]:
                w = (w + 1) % len(counts)
            out.append((w, nxt[w]))
            nxt[w] += 1
        return out

    def norms_not_squared(res_norms, block_bytes):
        r = np.asarray(res_norms, dtype=np.float64)
        return (r[:-1] - r[1:]) / float(block_bytes)

    for name, fn in [("order_greedy", lowest_first), ("order_greedy", ties_to_higher_weight),
                     ("order_average", weight_major), ("order_random", draw_over_all_weights),
                     ("block_scores", norms_not_squared)]:
        with monkeypatch.context() as mp:
            mp.setattr(budget, name, fn)
            assert not _planner_pins_pass(), f"planted mistake {fn.__name__} in {name} went unnoticed"
    assert (real_greedy, real_random, real_scores) == (budget.order_greedy, budget.order_random, budget.block_scores)


# ------------------------------------------------------------ C ABI == oracle ------
def _abi_order(counts, kind, scores=None, draws=None):
    w, b = R.bs_plan_order(counts, kind, scores=scores, draws=draws)
    return list(zip(w.tolist(), b.tolist()))


@pytest.mark.parametrize("seed", range(6))
def test_abi_orders_equal_the_oracle(seed):
    gen = np.random.default_rng(100 + seed)
    nw = int(gen.integers(1, 40))
    counts = [int(c) for c in gen.integers(0, 17, size=nw)]
    levels = max(max(counts), 1)
    # arbitrary (not only falling) scores, with repeated values to exercise ties
    sc = np.round(gen.random((nw, levels)) * 8) / 8
    assert _abi_order(counts, R.BS_ORDER_GREEDY, scores=sc) == budget.order_greedy(_rows(sc, counts))
    assert _abi_order(counts, R.BS_ORDER_AVERAGE) == budget.order_average(counts)
    draws = gen.random(sum(counts))
    draws[: len(draws) // 7] = 0.0
    assert _abi_order(counts, R.BS_ORDER_RANDOM, draws=draws) == budget.order_random(counts, draws)


def test_abi_plans_an_8b_model_like_the_oracle():
    """224 linears of an 8B model, 16 blocks each, scores from seeded falling
    residual norms, and budgets across the range the evaluation sweeps."""
    gen = wl.generator(5, 0, "plan")
    sizes = np.array([pack.block_bytes(m, d, 16) for (_, _, m, d) in wl.llama3_8b_matrices()], dtype=np.uint64)
    counts = [16] * len(sizes)
    norms = np.cumprod(np.concatenate([np.ones((len(sizes), 1)), gen.uniform(0.8, 0.99, (len(sizes), 16))], 1), 1)
    sc = np.stack([budget.block_scores(r, int(b)) for r, b in zip(norms, sizes)])
    want = budget.order_greedy(_rows(sc, counts))
    got = _abi_order(counts, R.BS_ORDER_GREEDY, scores=sc)
    assert got == want
    for mib in (0, 500, 2000, 3000, 4500, 10_000):
        n_abi = R.bs_plan_budget([w for (w, _) in got], sizes, int(mib * budget.MIB))
        assert n_abi.tolist() == budget.budget_fill(want, sizes, mib).tolist()
        assert int(np.sum(n_abi * sizes)) <= mib * budget.MIB


def test_abi_edge_cases_and_errors():
    assert _abi_order([0, 0], R.BS_ORDER_AVERAGE) == []
    assert _abi_order([0, 0], R.BS_ORDER_GREEDY, scores=np.zeros((2, 0))) == []
    assert _abi_order([3], R.BS_ORDER_RANDOM, draws=[0.99, 0.0, 0.5]) == [(0, 0), (0, 1), (0, 2)]
    for bad in [dict(counts=[1, -1], kind=R.BS_ORDER_AVERAGE),
                dict(counts=[2, 3], kind=R.BS_ORDER_GREEDY, scores=np.ones((2, 2))),   # stride < 3
                dict(counts=[2, 3], kind=R.BS_ORDER_GREEDY),                           # no scores
                dict(counts=[1, 1], kind=R.BS_ORDER_RANDOM, draws=[0.5, 1.0]),         # draw = 1
                dict(counts=[1, 1], kind=R.BS_ORDER_RANDOM),
                dict(counts=[1], kind=7)]:
        with pytest.raises(R.BsError) as e:
            R.bs_plan_order(bad["counts"], bad["kind"], scores=bad.get("scores"), draws=bad.get("draws"))
        assert e.value.status == R.BS_ERR_INVALID_ARG
    # a budget smaller than every block loads nothing; an exact fit loads everything
    assert R.bs_plan_budget([0, 1, 0], [10, 20], 9).tolist() == [0, 0]
    assert R.bs_plan_budget([0, 1, 0], [10, 20], 40).tolist() == [2, 1]
    assert R.bs_plan_budget([0, 1, 0], [10, 20], 39).tolist() == [1, 1]
    assert R.bs_plan_budget([], [10, 20], 100).tolist() == [0, 0]
    with pytest.raises(R.BsError):
        R.bs_plan_budget([0, 2], [10, 20], 100)
