"""Pins of the CPU oracle to facts fixed by the pages and by mathematics
(worked examples, closed forms, invariants, library special cases, brute
force), so that a plausible slip in the oracle fails at least one of them.
CPU only."""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


# ----------------------------------------------------------------- router GEMM
def test_router_logits_one_hot_rows_pick_rows_of_wr():
    d, E = 7, 5  # d != E: a transposed operand cannot pass
    w_r = _rand(1, d, E)
    x = np.eye(d)
    lg = orc.router_logits(x, w_r)
    assert lg.shape == (d, E) and lg.dtype == np.float32
    np.testing.assert_array_equal(lg, w_r.astype(np.float32))


def test_router_logits_linear_and_bias():
    x, w_r = _rand(2, 9, 6), _rand(3, 6, 4)
    b = np.array([0.5, -1.0, 2.0, 0.0])
    a = orc.router_logits(x, w_r).astype(np.float64)
    ab = orc.router_logits(x, w_r, b).astype(np.float64)
    np.testing.assert_allclose(ab - a, np.broadcast_to(b, a.shape), atol=1e-6)
    two = orc.router_logits(2 * x, w_r).astype(np.float64)
    np.testing.assert_allclose(two, 2 * a, rtol=1e-6, atol=1e-6)
    # column sums for an all-ones token
    ones = orc.router_logits(np.ones((1, 6)), w_r)[0]
    np.testing.assert_allclose(ones, w_r.sum(axis=0), rtol=1e-6)


# ----------------------------------------------------------------- top-k
def _brute_topk(row, K):
    # python's own stable sort on the (value desc, id asc) key
    return sorted(range(len(row)), key=lambda e: (-float(row[e]), e))[:K]


@pytest.mark.parametrize("seed", range(5))
def test_topk_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 20))
    K = int(rng.integers(1, E + 1))
    lg = rng.integers(-3, 4, size=(40, E)).astype(np.float32)  # many ties
    ids = orc.topk_ids(lg, K)
    for t in range(lg.shape[0]):
        assert list(ids[t]) == _brute_topk(lg[t], K)


def test_topk_all_equal_gives_lowest_ids():
    ids = orc.topk_ids(np.zeros((3, 8), np.float32), 3)
    np.testing.assert_array_equal(ids, np.tile([0, 1, 2], (3, 1)))


def test_topk_signed_zero_is_a_tie():
    lg = np.array([[-0.0, 0.0, -1.0, 0.0]], np.float32)
    np.testing.assert_array_equal(orc.topk_ids(lg, 3), [[0, 1, 3]])


def test_topk_k_equals_e_is_a_descending_sort():
    lg = _rand(4, 6, 9).astype(np.float32)
    ids = orc.topk_ids(lg, 9)
    for t in range(6):
        assert sorted(ids[t]) == list(range(9))
        vals = lg[t, ids[t]]
        assert np.all(np.diff(vals) <= 0)


# ----------------------------------------------------------------- weights
def test_weights_sum_to_one_renormalised():
    lg = (3 * _rand(5, 100, 16)).astype(np.float32)
    ids, w = orc.route(lg, 4)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 1e-6)
    assert np.all(w > 0)
    assert np.all(np.diff(w, axis=1) <= 0)  # descending with the logits


def test_weights_k_equals_e_is_full_softmax():
    lg = _rand(6, 20, 7).astype(np.float32)
    ids, w = orc.route(lg, 7)
    sm = scipy.special.softmax(lg.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(sm, ids.astype(np.int64), 1), rtol=1e-6)


def test_weights_not_renormalised_is_softmax_at_selected():
    lg = _rand(7, 20, 10).astype(np.float32)
    ids, w = orc.route(lg, 3, renormalize=False)
    sm = scipy.special.softmax(lg.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(sm, ids.astype(np.int64), 1), rtol=1e-6)
    assert np.all(w.sum(1) < 1.0)


def test_weights_k1_is_one_and_two_experts_is_logistic():
    lg = _rand(8, 30, 5).astype(np.float32)
    _, w1 = orc.route(lg, 1)
    np.testing.assert_array_equal(w1, np.ones((30, 1), np.float32))
    l2 = _rand(9, 30, 2).astype(np.float32)
    ids, w = orc.route(l2, 2)
    hi = np.take_along_axis(l2, ids[:, :1].astype(np.int64), 1)[:, 0].astype(np.float64)
    lo = np.take_along_axis(l2, ids[:, 1:].astype(np.int64), 1)[:, 0].astype(np.float64)
    np.testing.assert_allclose(w[:, 0], 1.0 / (1.0 + np.exp(lo - hi)), rtol=1e-6)


# ----------------------------------------------------------------- capacity
def test_capacity_values():
    assert orc.capacity(1.25, 8192, 4, 32) == 1280  # the skewed workload
    assert orc.capacity(0.0, 100, 2, 8) is None
    assert orc.capacity(-1.0, 100, 2, 8) is None
    assert orc.capacity(1.0, 10, 3, 4) == math.ceil(7.5)


# ----------------------------------------------------------------- permutation
def _read_golden():
    routing, expert_tokens, sec = {}, {}, None
    with open(os.path.join(GOLDEN, "omnimoe_expert_centric_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                sec = line
                continue
            k, v = line.split(":")
            vals = [int(s) for s in v.split()]
            (routing if sec == "[routing]" else expert_tokens)[int(k)] = vals
    return routing, expert_tokens


def test_permutation_worked_example():
    routing, printed = _read_golden()
    T = len(routing)
    K = len(routing[0])
    uniq = sorted({e for v in routing.values() for e in v})
    dense = {e: i for i, e in enumerate(uniq)}  # order-preserving remap to 0..E-1
    ids = np.array([[dense[e] for e in routing[t]] for t in range(T)], np.int32)
    counts, offsets, a2p, p2a = orc.permute(ids, len(uniq), None)
    got = {}
    for orig, e in dense.items():
        lo, hi = offsets[e], offsets[e + 1]
        got[orig] = [int(a) // K for a in p2a[lo:hi]]
    for orig, toks in printed.items():
        assert got[orig] == toks
    for orig in set(uniq) - set(printed):
        assert len(got[orig]) == 1
    assert counts.sum() == T * K


def _check_perm_invariants(ids, E, C):
    T, K = ids.shape
    counts, offsets, a2p, p2a = orc.permute(ids, E, C)
    flat = ids.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    kept = counts if C is None else np.minimum(counts, C)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(kept)]))
    nk = offsets[-1]
    # bijection between kept assignments and slots [0, nk)
    assert np.all(p2a[nk:] == -1)
    assert sorted(p2a[:nk]) == sorted(np.nonzero(a2p >= 0)[0])
    np.testing.assert_array_equal(a2p[p2a[:nk]], np.arange(nk))
    # expert ids non-decreasing along p; tokens strictly increasing in an expert
    ex = flat[p2a[:nk]]
    assert np.all(np.diff(ex) >= 0)
    for e in range(E):
        tok = p2a[offsets[e]:offsets[e + 1]] // K
        assert np.all(np.diff(tok) > 0)
        assert np.all(ex[offsets[e]:offsets[e + 1]] == e)
        if C is not None:
            dropped = [a // K for a in np.nonzero((flat == e) & (a2p < 0))[0]]
            if len(tok) and dropped:
                assert min(dropped) > tok.max()
    return counts, offsets, a2p, p2a


@pytest.mark.parametrize("seed", range(6))
def test_permutation_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    E = int(rng.integers(1, 12))
    K = int(rng.integers(1, E + 1))
    T = int(rng.integers(1, 60))
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    _check_perm_invariants(ids, E, None)
    for C in (0, 1, 3, T):
        _check_perm_invariants(ids, E, C)


def test_permutation_is_the_stable_sort():
    rng = np.random.default_rng(11)
    E, K, T = 9, 3, 200
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    _, _, a2p, p2a = orc.permute(ids, E, None)
    np.testing.assert_array_equal(p2a, np.argsort(ids.reshape(-1), kind="stable"))


def test_capacity_large_enough_changes_nothing():
    rng = np.random.default_rng(12)
    E, K, T = 6, 2, 80
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    a = orc.permute(ids, E, None)
    b = orc.permute(ids, E, int(np.bincount(ids.reshape(-1)).max()))
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_capacity_drops_in_token_order_direct_rule():
    rng = np.random.default_rng(13)
    E, K, T, C = 5, 2, 50, 7
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    _, _, a2p, _ = orc.permute(ids, E, C)
    seen = np.zeros(E, int)
    for t in range(T):  # direct rule: an assignment survives iff fewer than C earlier tokens hold e
        for k in range(K):
            e = ids[t, k]
            assert (a2p[t * K + k] >= 0) == (seen[e] < C)
        for k in range(K):
            seen[ids[t, k]] += 1


def test_gather_rows_moves_token_rows():
    rng = np.random.default_rng(14)
    E, K, T = 4, 2, 10
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    x = np.arange(T * 3, dtype=np.float32).reshape(T, 3)
    _, offsets, a2p, p2a = orc.permute(ids, E, None)
    xp = orc.gather_rows(x, p2a, offsets, K)
    for t in range(T):
        for k in range(K):
            np.testing.assert_array_equal(xp[a2p[t * K + k]], x[t])


# ----------------------------------------------------------------- experts and layer
def test_swiglu_is_torch_silu_times_up():
    g, u = _rand(15, 50), _rand(16, 50)
    ref = torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)
    np.testing.assert_allclose(orc.swiglu(g, u), ref.numpy(), rtol=1e-13, atol=1e-15)


def test_single_expert_is_dense_swiglu_mlp():
    T, d, n = 12, 8, 5  # d != n so a transposed weight cannot pass
    x, wg, wu, wd = _rand(17, T, d), _rand(18, 1, d, n), _rand(19, 1, d, n), _rand(20, 1, n, d)
    w_r = _rand(21, d, 1)
    res = orc.forward(x, w_r, wg, wu, wd, K=1)
    xt = torch.from_numpy(x)
    ref = (torch.nn.functional.silu(xt @ torch.from_numpy(wg[0])) * (xt @ torch.from_numpy(wu[0]))
           ) @ torch.from_numpy(wd[0])
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_layer_equals_dense_sum_over_all_experts(seed):
    rng = np.random.default_rng(200 + seed)
    E = int(rng.integers(2, 7))
    K = int(rng.integers(1, E + 1))
    T, d, n = int(rng.integers(1, 24)), 6, 4
    x, w_r = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    wg, wu = rng.standard_normal((E, d, n)), rng.standard_normal((E, d, n))
    wd = rng.standard_normal((E, n, d))
    res = orc.forward(x, w_r, wg, wu, wd, K=K)
    dense = orc.dense_reference(x, wg, wu, wd, res["topk_ids"], res["topk_w"], E)
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-12)
    rows = orc.forward_rows(np.arange(T), x, wg, wu, wd, res["topk_ids"], res["topk_w"],
                            res["assign_to_perm"], K)
    np.testing.assert_allclose(rows, dense, rtol=1e-12, atol=1e-12)


def test_layer_with_capacity_equals_dense_with_dropped_gates_zeroed():
    rng = np.random.default_rng(300)
    E, K, T, d, n = 4, 2, 30, 5, 3
    x, w_r = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    w_r[:, 0] += 2.0  # skew toward expert 0 so it overflows
    wg, wu = rng.standard_normal((E, d, n)), rng.standard_normal((E, d, n))
    wd = rng.standard_normal((E, n, d))
    cf = 0.5
    res = orc.forward(x, w_r, wg, wu, wd, K=K, capacity_factor=cf)
    C = orc.capacity(cf, T, K, E)
    w = res["topk_w"].astype(np.float64).copy()
    seen = np.zeros(E, int)
    for t in range(T):
        for k in range(K):
            if seen[res["topk_ids"][t, k]] >= C:
                w[t, k] = 0.0
        for k in range(K):
            seen[res["topk_ids"][t, k]] += 1
    assert (w == 0).any()
    dense = orc.dense_reference(x, wg, wu, wd, res["topk_ids"], w, E)
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-12)


def test_grouped_ffn_rows_are_rows_of_grouped_ffn():
    """The chosen-slot form returns exactly the rows the whole grouped FFN computes (same
    slots, any order, slots of several experts mixed), on a small routed problem."""
    g = np.random.default_rng(3)
    T, d, n, E, K = 40, 16, 24, 5, 2
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)  # noqa: E731
    x = bf(g.standard_normal((T, d)))  # bf16 tensors, as the workloads hold them
    wg, wu, wd = (bf(g.standard_normal((E, d, n))), bf(g.standard_normal((E, d, n))),
                  bf(g.standard_normal((E, n, d))))
    ids, _ = orc.route(g.standard_normal((T, E)).astype(np.float32), K)
    _, offsets, _, p2a = orc.permute(ids, E, orc.capacity(1.2, T, K, E))
    a_all, y_all = orc.grouped_ffn(x, p2a, offsets, K, wg, wu, wd)
    slots = g.permutation(int(offsets[-1]))[:30]
    a_rows, y_rows = orc.grouped_ffn_rows(slots, x, p2a, offsets, K, wg, wu, wd)
    np.testing.assert_allclose(a_rows, a_all[slots], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(y_rows, y_all[slots], rtol=1e-13, atol=1e-12)


def test_identity_experts_give_back_x():
    """Dispatch/combine-only workload: identity experts, sum of weights 1 => out = x."""
    cfg = mi.DISPATCH_COMBINE.with_T(64)
    inp = mi.make_inputs(cfg)
    x = orc.as_f64(inp.x)
    ids, w = orc.route(inp.logits.numpy(), cfg.K)
    _, offsets, a2p, p2a = orc.permute(ids, cfg.E, None)
    xp = orc.gather_rows(x, p2a, offsets, cfg.K)
    out = orc.combine(xp, a2p, w, cfg.T, cfg.K)
    np.testing.assert_allclose(out, x, rtol=1e-6, atol=1e-6)


def test_tiny_workload_forward_is_self_consistent():
    cfg = mi.TINY_FP32
    inp = mi.make_inputs(cfg)
    res = orc.forward(inp.x.numpy(), inp.w_r.numpy(), inp.w_gate.numpy(), inp.w_up.numpy(),
                      inp.w_down.numpy(), cfg.K)
    assert res["counts"].sum() == cfg.T * cfg.K
    dense = orc.dense_reference(inp.x.numpy(), inp.w_gate.numpy(), inp.w_up.numpy(),
                                inp.w_down.numpy(), res["topk_ids"], res["topk_w"], cfg.E)
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-12)


def test_zipf_alpha_reaches_five_times_mean_load():
    cfg = mi.SKEWED_CAPACITY_BF16
    inp = mi.make_inputs(cfg, with_experts=False)
    lg = orc.router_logits(inp.x, inp.w_r, inp.bias.numpy())
    counts, _, _, _ = orc.permute(orc.topk_ids(lg, cfg.K), cfg.E, None)
    ratio = counts.max() / (cfg.T * cfg.K / cfg.E)
    assert abs(ratio - 5.0) <= 0.1
    assert int(np.argmax(counts)) == 0


# ----------------------------------------------------------------- planted mistakes
def test_planted_mistakes_are_caught(monkeypatch):
    """Mutate the oracle on the CPU and check that a pin above notices."""
    rng = np.random.default_rng(400)
    E, K, T, d, n = 4, 2, 9, 5, 3
    x, w_r = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    wg, wu = rng.standard_normal((E, d, n)), rng.standard_normal((E, d, n))
    wd = rng.standard_normal((E, n, d))

    def dense_ok():
        res = orc.forward(x, w_r, wg, wu, wd, K=K)
        dense = orc.dense_reference(x, wg, wu, wd, res["topk_ids"], res["topk_w"], E)
        return np.allclose(res["out"], dense, rtol=1e-12, atol=1e-12)

    assert dense_ok()
    real_combine = orc.combine

    def combine_drops_last_slot(y, a2p, w, T_, K_):
        a2p = np.asarray(a2p).reshape(T_, K_).copy()
        a2p[:, -1] = -1
        return real_combine(y, a2p.reshape(-1), w, T_, K_)

    monkeypatch.setattr(orc, "combine", combine_drops_last_slot)
    assert not dense_ok()
    monkeypatch.undo()

    real_permute = orc.permute

    def permute_off_by_one(ids, E_, C_, keep=None):
        c, o, a2p, p2a = real_permute(ids, E_, C_, keep)
        nk = o[-1]
        p2a = p2a.copy()
        p2a[:nk] = np.roll(p2a[:nk], 1)
        return c, o, a2p, p2a

    monkeypatch.setattr(orc, "permute", permute_off_by_one)
    assert not dense_ok()
    monkeypatch.undo()

    g, u = rng.standard_normal(20), rng.standard_normal(20)
    wrong = g / (1.0 + np.exp(g)) * u  # sign slip inside silu
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    assert not np.allclose(wrong, ref)
    assert np.allclose(orc.swiglu(g, u), ref)


# ------------------------------------------------------------------ token rounding
# SonicMoE explainer (gitcode.csdn.net), section 6.5 names tile-aware token rounding
# without a rule; the rule pinned here is the library's reading: an expert with c >= R
# routed assignments keeps R * floor(c / R) of them, the ones with the largest logit for
# that expert (equal logits: the earlier token stays), experts with c < R keep all.
def _hand_logits():
    # K = 1: t0 t1 t3 t5 t6 pick e0 (scores 3 2 2 5 2), t2 t4 pick e1 (4, 1), t7 picks e2
    lg = np.zeros((8, 3), np.float32)
    for t, (e, v) in enumerate([(0, 3), (0, 2), (1, 4), (0, 2), (1, 1), (0, 5), (0, 2), (2, 7)]):
        lg[t, e] = v
    return lg


@pytest.mark.parametrize("R,dropped_tokens", [
    (1, []),        # nothing to round
    (2, [6]),       # e0: 5 -> 4; the weakest logit 2 is held by t1, t3, t6: the latest goes
    (3, [3, 6]),    # e0: 5 -> 3: t6 then t3; e1 (2 < 3) and e2 keep theirs
    (4, [6]),       # e0: 5 -> 4
    (8, []),        # every expert below R
])
def test_token_rounding_hand_worked(R, dropped_tokens):
    lg = _hand_logits()
    ids, _ = orc.route(lg, 1)
    np.testing.assert_array_equal(ids[:, 0], [0, 0, 1, 0, 1, 0, 0, 2])
    keep = orc.tile_round_keep(ids, lg, 3, R)
    assert sorted(np.nonzero(~keep[:, 0])[0].tolist()) == dropped_tokens


def test_token_rounding_hand_worked_two_slots():
    # K = 2; t3 ties e0 and e2 at 2 (both picked, e0 first). e0 gets t0(3) t1(1) t3(2):
    # 3 -> 2 drops t1's slot 1; e1 gets t0(2) t2(4): kept; e2 gets t1(5) t2(1) t3(2):
    # 3 -> 2 drops t2's slot 1.
    lg = np.array([[3, 2, 0], [1, 0, 5], [0, 4, 1], [2, 0, 2]], np.float32)
    ids, _ = orc.route(lg, 2)
    np.testing.assert_array_equal(ids, [[0, 1], [2, 0], [1, 2], [0, 2]])
    keep = orc.tile_round_keep(ids, lg, 3, 2)
    np.testing.assert_array_equal(keep, [[True, True], [True, False], [True, False],
                                         [True, True]])


def _rounding_brute_force(ids, lg, E, R):
    """Every subset of the right size whose kept members all outrank its dropped members by
    (logit, then earlier token); exactly one exists per expert."""
    import itertools
    T, K = ids.shape
    keep = np.ones((T, K), bool)
    for e in range(E):
        members = [(t, k) for t in range(T) for k in range(K) if ids[t, k] == e]
        c = len(members)
        if c < R:
            continue
        r = (c // R) * R
        found = []
        for kept in itertools.combinations(range(c), r):
            dropped = [i for i in range(c) if i not in kept]

            def outranks(i, j):
                (ti, ki), (tj, kj) = members[i], members[j]
                si, sj = lg[ti, e], lg[tj, e]
                return si > sj or (si == sj and ti < tj)
            if all(outranks(i, j) for i in kept for j in dropped):
                found.append(dropped)
        assert len(found) == 1
        for i in found[0]:
            keep[members[i]] = False
    return keep


@pytest.mark.parametrize("seed", range(6))
def test_token_rounding_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    T, E, K, R = 9, 3, 2, 2 + seed % 3
    lg = rng.integers(-2, 3, size=(T, E)).astype(np.float32)  # many ties
    ids, _ = orc.route(lg, K)
    np.testing.assert_array_equal(orc.tile_round_keep(ids, lg, E, R),
                                  _rounding_brute_force(ids, lg, E, R))


@pytest.mark.parametrize("seed", range(4))
def test_token_rounding_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    T, E, K, R = 500, 8, 2, 16
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids, _ = orc.route(lg, K)
    keep = orc.tile_round_keep(ids, lg, E, R)
    counts, offsets, a2p, p2a = orc.permute(ids, E, None, keep)
    assert counts.sum() == T * K
    kept = np.diff(offsets)
    for e in range(E):
        c = int(counts[e])
        assert kept[e] == (c if c < R else (c // R) * R)
        mask = ids == e
        ks, ds = lg[:, e][(mask & keep).any(1)], lg[:, e][(mask & ~keep).any(1)]
        if ds.size:
            assert ks.min() >= ds.max()
    assert np.all(a2p.reshape(T, K)[~keep] == -1)
    assert np.all(a2p.reshape(T, K)[keep] >= 0)


def test_token_rounding_by_one_changes_nothing_and_excludes_capacity():
    rng = np.random.default_rng(3)
    E, K, T, d, n = 4, 2, 30, 6, 4
    x, w_r = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    wg, wu = rng.standard_normal((E, d, n)), rng.standard_normal((E, d, n))
    wd = rng.standard_normal((E, n, d))
    a = orc.forward(x, w_r, wg, wu, wd, K=K)
    b = orc.forward(x, w_r, wg, wu, wd, K=K, tile_round=1)
    np.testing.assert_array_equal(a["assign_to_perm"], b["assign_to_perm"])
    np.testing.assert_array_equal(a["out"], b["out"])
    with pytest.raises(ValueError):
        orc.forward(x, w_r, wg, wu, wd, K=K, capacity_factor=1.0, tile_round=4)


def test_token_rounding_planted_mistake_is_caught(monkeypatch):
    lg = _hand_logits()
    E, K, R = 3, 1, 3
    ids, _ = orc.route(lg, K)
    real = np.lexsort

    def keeps_the_weakest(keys):  # a reversed sort inside the rounding
        return real(keys)[::-1]

    monkeypatch.setattr(orc.np, "lexsort", keeps_the_weakest)
    wrong = orc.tile_round_keep(ids, lg, E, R)
    monkeypatch.undo()
    assert not np.array_equal(wrong, _rounding_brute_force(ids, lg, E, R))


# ------------------------------------------------------------------ token rounding up / nearest
def _up_case():
    # T = 6, E = 2, K = 1: routed e0 = {0, 1, 4, 5} (t5 ties 2 = 2: the lower id), e1 = {2, 3}
    return np.array([[5, 1], [4, 2], [0, 3], [3, 3.5], [1, 0], [2, 2]], dtype=np.float32)


def test_rounding_up_hand_worked():
    """R = 4: e0 holds 4 (unchanged); e1 holds 2 and gains 2 of t0 (1), t1 (2), t4 (0),
    t5 (2): t1 and t5 (equal logits, both taken). Renormalised weights over the enlarged
    selections: t1 {e0, e1} = softmax(4, 2), t5 {e0, e1} = softmax(2, 2) = (1/2, 1/2)."""
    lg = _up_case()
    ids, _ = orc.route(lg, 1)
    np.testing.assert_array_equal(ids[:, 0], [0, 0, 1, 1, 0, 0])
    keep, at, ae = orc.tile_round_select(ids, lg, 2, 4, "up")
    assert keep.all()
    np.testing.assert_array_equal(at, [1, 5])
    np.testing.assert_array_equal(ae, [1, 1])
    w, aw = orc.round_weights(lg, ids, at, ae)
    s1 = 1.0 / (1.0 + math.exp(-2.0))
    np.testing.assert_allclose([w[1, 0], aw[0]], [s1, 1.0 - s1], rtol=1e-6)
    np.testing.assert_allclose([w[5, 0], aw[1]], [0.5, 0.5], rtol=1e-7)
    np.testing.assert_allclose(w[[0, 2, 3, 4], 0], 1.0)
    # nearest: e1 has r = 2 = R - r: rounds down, and with c < R it keeps all (no change)
    keep, at, ae = orc.tile_round_select(ids, lg, 2, 4, "nearest")
    assert keep.all() and at.size == 0


def test_rounding_nearest_hand_worked():
    """R = 4, e1 routed 3 times (r = 3 > R - r = 1): nearest rounds up by one, the best
    non-routed token for e1; e0 routed 5 times (r = 1): nearest drops its weakest."""
    lg = np.array([[9, 1], [8, 2], [0, 7], [1, 6], [2, 5], [7, 4], [6, 3], [5, 0]],
                  dtype=np.float32)
    ids, _ = orc.route(lg, 1)
    np.testing.assert_array_equal(ids[:, 0], [0, 0, 1, 1, 1, 0, 0, 0])
    keep, at, ae = orc.tile_round_select(ids, lg, 2, 4, "nearest")
    # e0 = {0, 1, 5, 6, 7} with logits 9, 8, 7, 6, 5: drop t7 (the weakest)
    np.testing.assert_array_equal(keep[:, 0], [True] * 7 + [False])
    # e1 gains the best of t0 (1), t1 (2), t5 (4), t6 (3), t7 (0): t5
    np.testing.assert_array_equal(at, [5])
    np.testing.assert_array_equal(ae, [1])


def _is_top_m(cand, chosen, score):
    """Brute force over pairs: every chosen token ranks above every unchosen candidate
    (larger logit, or equal logit and earlier token)."""
    ch = set(int(c) for c in chosen)
    for c in ch:
        for u in cand:
            u = int(u)
            if u in ch:
                continue
            if not (score[c] > score[u] or (score[c] == score[u] and c < u)):
                return False
    return True


@pytest.mark.parametrize("seed", range(6))
def test_rounding_up_adds_the_best_non_routed_tokens(seed):
    g = np.random.default_rng(100 + seed)
    T, E, K, R = 30, 5, 2, 7
    lg = g.integers(-3, 4, size=(T, E)).astype(np.float32)  # ties on purpose
    ids, _ = orc.route(lg, K)
    keep, at, ae = orc.tile_round_select(ids, lg, E, R, "up")
    assert keep.all()
    for e in range(E):
        routed = np.unique(np.nonzero(ids == e)[0])
        c = routed.size
        chosen = at[ae == e]
        cand = np.setdiff1d(np.arange(T), routed)
        want = 0 if c % R == 0 else min(R - c % R, cand.size)
        assert chosen.size == want
        assert np.all(np.diff(chosen) > 0) and not np.isin(chosen, routed).any()
        assert _is_top_m(cand, chosen, lg[:, e])
        final = c + chosen.size
        assert final % R == 0 or final == T


@pytest.mark.parametrize("seed", range(4))
def test_rounding_nearest_invariants(seed):
    g = np.random.default_rng(200 + seed)
    T, E, K, R = 60, 6, 2, 8
    lg = g.standard_normal((T, E)).astype(np.float32)
    ids, _ = orc.route(lg, K)
    keep, at, ae = orc.tile_round_select(ids, lg, E, R, "nearest")
    down_keep = orc.tile_round_keep(ids, lg, E, R)
    for e in range(E):
        c = int((ids == e).sum())
        r = c % R
        final = int((keep & (ids == e)).sum()) + int((ae == e).sum())
        if r == 0:
            assert final == c
        elif r <= R - r:  # down: the down rule's result for this expert
            assert final == (c if c < R else c - r)
            np.testing.assert_array_equal(keep[ids == e], down_keep[ids == e])
        else:
            assert final == min(c + R - r, T)
    # mode "down" is tile_round_keep with nothing added
    k2, at2, _ = orc.tile_round_select(ids, lg, E, R, "down")
    np.testing.assert_array_equal(k2, down_keep)
    assert at2.size == 0


@pytest.mark.parametrize("renorm", [True, False])
def test_rounded_up_layer_equals_dense_sum_with_enlarged_gates(renorm):
    """The layer with added assignments equals the dense sum over all E experts gated by
    each token's weights over its enlarged selection (0 elsewhere), and the renormalised
    weights of a token sum to one."""
    g = np.random.default_rng(7)
    T, d, n, E, K, R = 24, 16, 32, 4, 2, 5
    x = g.standard_normal((T, d))
    w_r = 0.5 * g.standard_normal((d, E))
    wg, wu, wd = (0.3 * g.standard_normal((E, d, n)), 0.3 * g.standard_normal((E, d, n)),
                  0.3 * g.standard_normal((E, n, d)))
    f = orc.forward(x, w_r, wg, wu, wd, K, renormalize=renorm, tile_round=R, round_mode="up")
    at, ae, aw = f["add_tok"], f["add_exp"], f["add_w"]
    assert at.size > 0
    gate = np.zeros((T, E))
    for t in range(T):
        for k in range(K):
            gate[t, f["topk_ids"][t, k]] = f["topk_w"][t, k]
    for j in range(at.size):
        gate[at[j], ae[j]] = aw[j]
    if renorm:
        np.testing.assert_allclose(gate.sum(axis=1), 1.0, rtol=1e-6)
    dense = np.zeros((T, d))
    for e in range(E):
        dense += gate[:, e:e + 1] * orc.expert_ffn(x, wg[e], wu[e], wd[e])
    np.testing.assert_allclose(f["out"], dense, rtol=1e-9, atol=1e-9)
    counts = np.diff(f["offsets"])
    assert np.all((counts % R == 0) | (counts == T))


def test_rounding_up_planted_mistakes_are_caught(monkeypatch):
    """A tie rule reversed inside the selection, and added weights over the routed
    denominator only, both fail the pins above."""
    lg = _up_case()
    ids, _ = orc.route(lg, 1)
    real = np.lexsort

    def later_token_first(keys):  # the selection's tie-break inverted
        return real((-np.asarray(keys[0]),) + tuple(keys[1:]))

    # R = 3: e1 (routed 2) gains one token, t1 and t5 tie at 2: the earlier one, t1
    _, at, ae = orc.tile_round_select(ids, lg, 2, 3, "up")
    np.testing.assert_array_equal(at[ae == 1], [1])
    monkeypatch.setattr(orc.np, "lexsort", later_token_first)
    _, at, ae = orc.tile_round_select(ids, lg, 2, 3, "up")
    monkeypatch.undo()
    assert not np.array_equal(at[ae == 1], [1])
    # weights of the added slot over the routed selection only: the token's weights no
    # longer sum to one
    w, aw = orc.round_weights(lg, ids, [1, 5], [1, 1])
    wrong = math.exp(2.0 - 4.0)  # exp(l_add - l_top) / (routed sum = 1)
    assert abs(w[1, 0] + wrong - 1.0) > 1e-3 and abs(w[1, 0] + aw[0] - 1.0) < 1e-6


# ------------------------------------------------------------------ backward (expert half)
def _autograd_backward(x, lg, wg, wu, wd, K, cf, d_out):
    """The same layer written with torch ops in fp64 and differentiated by autograd: the
    gradients of <d_out, out> with respect to the pre-activations (g, u) of every kept
    slot and to the routing weights."""
    T, E = lg.shape
    ids, w = orc.route(lg, K)
    counts, offsets, a2p, p2a = orc.permute(ids, E, orc.capacity(cf, T, K, E))
    nk = int(offsets[-1])
    xt = torch.from_numpy(np.asarray(x, np.float64))
    G = torch.zeros(nk, wg.shape[2], dtype=torch.float64)
    U = torch.zeros(nk, wg.shape[2], dtype=torch.float64)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        tok = torch.from_numpy(np.asarray(p2a[lo:hi], np.int64) // K)
        G[lo:hi] = xt[tok] @ torch.from_numpy(wg[e])
        U[lo:hi] = xt[tok] @ torch.from_numpy(wu[e])
    G.requires_grad_(True)
    U.requires_grad_(True)
    W = torch.from_numpy(np.asarray(w, np.float64)).requires_grad_(True)
    A = torch.nn.functional.silu(G) * U
    # the same pre-activations as functions of x (routing held fixed), for the input gradient
    Xl = xt.clone().requires_grad_(True)
    G2 = torch.zeros_like(G)
    U2 = torch.zeros_like(U)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        tok = torch.from_numpy(np.asarray(p2a[lo:hi], np.int64) // K)
        G2[lo:hi] = Xl[tok] @ torch.from_numpy(wg[e])
        U2[lo:hi] = Xl[tok] @ torch.from_numpy(wu[e])
    Y = torch.zeros(nk, wd.shape[2], dtype=torch.float64)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        Y[lo:hi] = A[lo:hi] @ torch.from_numpy(wd[e])
    out = torch.zeros(T, wd.shape[2], dtype=torch.float64)
    for t in range(T):
        for k in range(K):
            p = int(a2p[t * K + k])
            if p >= 0:
                out[t] = out[t] + W[t, k] * Y[p]
    (out * torch.from_numpy(d_out)).sum().backward()
    # dx: d<d_out, out>/dx through G2, U2 with the upstream gradients G.grad, U.grad
    (G2 * G.grad).sum().add_((U2 * U.grad).sum()).backward()
    _autograd_backward.dx = Xl.grad.numpy()
    return (G.detach().numpy(), U.detach().numpy(), G.grad.numpy(), U.grad.numpy(),
            W.grad.numpy(), (offsets, a2p, p2a, w))


@pytest.mark.parametrize("cf", [0.0, 0.7])
def test_backward_matches_autograd(cf):
    rng = np.random.default_rng(31)
    T, d, n, E, K = 11, 6, 5, 4, 2
    x = rng.standard_normal((T, d))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    wg, wu = rng.standard_normal((E, d, n)), rng.standard_normal((E, d, n))
    wd = rng.standard_normal((E, n, d))
    d_out = rng.standard_normal((T, d))
    g, u, gg, gu, gw, (offsets, a2p, p2a, w) = _autograd_backward(x, lg, wg, wu, wd, K, cf, d_out)
    g2, u2 = orc.gate_up_preact(x, p2a, offsets, K, wg, wu)
    np.testing.assert_allclose(g2, g, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(u2, u, rtol=1e-13, atol=1e-13)
    dG, dU, d_w = orc.backward_act(d_out, w, a2p, p2a, offsets, K, wd, g2, u2)
    np.testing.assert_allclose(dG, gg, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dU, gu, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(d_w, gw, rtol=1e-11, atol=1e-12)
    dx = orc.backward_dx(dG, dU, a2p, p2a, offsets, K, T, wg, wu)
    np.testing.assert_allclose(dx, _autograd_backward.dx, rtol=1e-11, atol=1e-12)
    if cf > 0:
        assert np.all(d_w.reshape(-1)[a2p < 0] == 0)  # dropped slots carry no gradient
        assert (a2p < 0).any()


def test_backward_planted_mistake_is_caught(monkeypatch):
    rng = np.random.default_rng(32)
    T, d, n, E, K = 9, 4, 3, 3, 2
    x = rng.standard_normal((T, d))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    wg, wu = rng.standard_normal((E, d, n)), rng.standard_normal((E, d, n))
    wd = rng.standard_normal((E, n, d))
    d_out = rng.standard_normal((T, d))
    g, u, gg, gu, gw, (offsets, a2p, p2a, w) = _autograd_backward(x, lg, wg, wu, wd, K, 0.0, d_out)
    real_exp = orc.np.exp

    def exp_sign_slip(v):  # s = 1 / (1 + e^{+g}) instead of e^{-g}
        return real_exp(-v)

    monkeypatch.setattr(orc.np, "exp", exp_sign_slip)
    dG, _, _ = orc.backward_act(d_out, w, a2p, p2a, offsets, K, wd, g, u)
    monkeypatch.undo()
    assert not np.allclose(dG, gg, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("renorm", [True, False])
def test_router_backward_matches_autograd(renorm):
    rng = np.random.default_rng(41)
    T, d, E, K = 10, 6, 5, 2
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((d, E))
    bias = rng.standard_normal(E)
    d_w = rng.standard_normal((T, K))
    lg32 = orc.router_logits(x, w_r, bias)
    ids, _ = orc.route(lg32, K, renorm)
    # autograd: the weights as a function of x, W_r and the bias with the selection fixed
    X = torch.from_numpy(x).requires_grad_(True)
    W = torch.from_numpy(w_r).requires_grad_(True)
    B = torch.from_numpy(bias).requires_grad_(True)
    L = X @ W + B
    L.retain_grad()
    idx = torch.from_numpy(ids.astype(np.int64))
    if renorm:
        wts = torch.softmax(torch.gather(L, 1, idx), dim=1)
    else:
        wts = torch.gather(torch.softmax(L, dim=1), 1, idx)
    (wts * torch.from_numpy(d_w)).sum().backward()
    # the oracle differentiates at the fp32 logits the selection saw; autograd at the fp64
    # ones: the same function of nearly the same point
    d_logits, d_w_r, d_bias, d_x = orc.backward_router(d_w, ids, lg32, x, w_r, renorm)
    np.testing.assert_allclose(d_logits, L.grad.numpy(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(d_w_r, W.grad.numpy(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(d_bias, B.grad.numpy(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(d_x, X.grad.numpy(), rtol=1e-5, atol=1e-6)
    if renorm:  # only the selected logits receive a gradient, and each row sums to zero
        mask = np.zeros((T, E), bool)
        np.put_along_axis(mask, ids, True, axis=1)
        assert np.all(d_logits[~mask] == 0)
    np.testing.assert_allclose(d_logits.sum(axis=1), 0.0, atol=1e-12)
