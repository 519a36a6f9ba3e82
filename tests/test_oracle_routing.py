"""Pins for the oracle's router, top-k selection and dispatch.

Routing as the layer specification states it: fp32 logits (+ optional
per-expert bias), softmax over all experts, the top-k picks with the lower
expert id winning a tie, renormalised to sum 1.  The pages fix 512 experts with
10 routed per token ("Strata Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU
at Up to 94 Tokens/s", section "What it is").  Dispatch: per-expert histogram,
exclusive prefix sum, stable token-ascending scatter.
"""
import numpy as np
import pytest

import gen
import oracle
from tests import npref
from tests.conftest import golden


def _order_cases():
    out = []
    for line in open(golden("router_order.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        name, entries, expect = [s.strip() for s in line.split("|")]
        w = np.zeros(64, dtype=np.float32)
        for ent in entries.split():
            i, v = ent.split(":")
            w[int(i)] = float(v)
        out.append((name, w, float(expect)))
    return out


@pytest.mark.parametrize("name,w,expect", _order_cases())
def test_canonical_order_worked_sums(name, w, expect):
    x = np.full((1, 64), 0x3F80, dtype=np.uint16)  # bf16 1.0
    got = oracle.router_logits(x, w[None, :], None)
    assert float(got[0, 0]) == expect, name


def test_logits_within_fp32_error_bound_of_exact_dot():
    rng = np.random.default_rng(3)
    shape = gen.LayerShape(hidden=512, n_experts=24, top_k=3, inter=64, router_bias=True)
    x = gen.hidden(16, 512, seed=3)
    W = gen.router_weight(shape, seed=3)
    b = gen.router_bias(shape, seed=3)
    got = oracle.router_logits(x, W, b).astype(np.float64)
    xf = npref.bf16_bits_to_f64(x)
    exact = xf @ W.astype(np.float64).T + b.astype(np.float64)
    mag = np.abs(xf) @ np.abs(W.astype(np.float64)).T + np.abs(b)
    u = 2.0 ** -24
    bound = (512 / 32 + 5 + 1 + 1) * u * mag
    assert np.all(np.abs(got - exact) <= bound)
    # a dropped or misplaced term would be far outside the bound
    assert np.max(np.abs(got - exact) / mag) < 1e-6
    del rng


def test_bias_is_added():
    x = gen.hidden(2, 64, seed=1)
    W = np.zeros((5, 64), dtype=np.float32)
    b = np.array([0.5, -1.0, 2.0, 0.0, 3.25], dtype=np.float32)
    assert np.array_equal(oracle.router_logits(x, W, b), np.tile(b, (2, 1)))


def test_all_ties_pick_lowest_ids_with_equal_weights():
    logits = np.zeros((3, 16), dtype=np.float32)
    idx, w = oracle.route(logits, 4)
    assert np.array_equal(idx, np.tile(np.arange(4), (3, 1)))
    assert np.array_equal(w, np.full((3, 4), 0.25))


def test_zero_router_distinct_bias_picks_topk_of_bias():
    b = np.array([0.1, 3.0, -2.0, 3.0, 0.7, 2.5], dtype=np.float32)
    logits = np.tile(b, (1, 1))
    idx, _ = oracle.route(logits, 3)
    assert list(idx[0]) == [1, 3, 5]  # tie 3.0 at ids 1 and 3 -> lower id first


def test_worked_weights():
    # logits [0, ln 3, -10, -20]: picks 1 then 0, weights 3/4 and 1/4
    logits = np.array([[0.0, np.log(3.0), -10.0, -20.0]], dtype=np.float32)
    idx, w = oracle.route(logits, 2)
    assert list(idx[0]) == [1, 0]
    l1 = float(np.float32(np.log(3.0)))
    assert w[0, 0] == pytest.approx(np.exp(l1) / (np.exp(l1) + 1.0), rel=1e-15)
    assert w[0, 0] == pytest.approx(0.75, rel=1e-7)
    assert w[0, 0] + w[0, 1] == pytest.approx(1.0, rel=1e-15)


@pytest.mark.parametrize("E,k", [(16, 2), (64, 10), (512, 10)])
def test_route_matches_library_sort_and_softmax(E, k):
    rng = np.random.default_rng(E + k)
    logits = rng.standard_normal((40, E)).astype(np.float32)
    logits[0, 5] = logits[0, 9] = logits[0].max() + 1  # an exact tie at the top
    idx, w = oracle.route(logits, k)
    ridx, rw = npref.topk_softmax(logits, k)
    assert np.array_equal(idx, ridx)
    assert np.allclose(w, rw, rtol=1e-13, atol=0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=1e-13)
    assert list(idx[0, :2]) == [5, 9]


def test_dispatch_matches_stable_sort_and_invariants():
    rng = np.random.default_rng(9)
    T, E, k = 300, 37, 5
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    cnt, off, lst, slot = oracle.dispatch(idx, E)
    assert np.array_equal(cnt, np.bincount(idx.ravel(), minlength=E))
    assert off[0] == 0 and off[E] == T * k
    assert np.array_equal(np.diff(off), cnt)
    order = np.argsort(idx.ravel(), kind="stable")
    assert np.array_equal(lst, order // k)
    for e in range(E):
        seg = lst[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)
    # slot round trip: list[slot[t, j]] == t and slot lies in expert idx[t, j]'s range
    tt = np.repeat(np.arange(T), k).reshape(T, k)
    assert np.array_equal(lst[slot], tt)
    ee = idx
    assert np.all((slot >= off[ee]) & (slot < off[ee + 1]))
    assert np.array_equal(np.sort(slot.ravel()), np.arange(T * k))


def test_dispatch_empty_and_single():
    cnt, off, lst, slot = oracle.dispatch(np.zeros((0, 3), dtype=np.int32), 8)
    assert cnt.sum() == 0 and np.all(off == 0) and lst.size == 0
    cnt, off, lst, slot = oracle.dispatch(np.array([[7, 2]], dtype=np.int32), 8)
    assert list(off) == [0, 0, 0, 1, 1, 1, 1, 1, 2]
    assert list(lst) == [0, 0] and list(slot[0]) == [1, 0]
