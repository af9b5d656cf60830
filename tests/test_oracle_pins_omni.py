"""Pins of the atomic-expert oracle (Cartesian-product router, expert-centric
schedule, rank-1 experts) to facts fixed by the page and by mathematics: a
hand-worked grid, closed forms, the reduction to the dense router, brute force,
the page's worked schedule example, and a closed-form layer with unit-vector
experts. Planted slips at the end show that each pin bites. CPU only."""
import math
import os

import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as dense_orc
from oracle import omni_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _logits(seed, T, nr, nc, integer=False):
    r = _rng(seed)
    if integer:
        return r.integers(-3, 4, size=(T, nr + nc)).astype(np.float32)
    return r.standard_normal((T, nr + nc)).astype(np.float32)


# ----------------------------------------------------------------- router GEMM
def test_cartesian_logits_one_hot_rows_pick_rows_of_both_tables():
    d, nr, nc = 7, 3, 5  # all different: a transposed or swapped operand cannot pass
    r = _rng(1)
    w_row, w_col = r.standard_normal((d, nr)), r.standard_normal((d, nc))
    lg = orc.cartesian_logits(np.eye(d), w_row, w_col)
    assert lg.shape == (d, nr + nc) and lg.dtype == np.float32
    np.testing.assert_array_equal(lg[:, :nr], w_row.astype(np.float32))
    np.testing.assert_array_equal(lg[:, nr:], w_col.astype(np.float32))


# ----------------------------------------------------------------- selection
HAND = np.array([[0.0, 1.0, 0.0, 2.0, 1.0]], np.float32)  # p_r = [0, 1], p_c = [0, 2, 1]
# pair sums on the 2 x 3 grid, id = i_r * 3 + i_c:
#   id 0: 0   id 1: 2   id 2: 1
#   id 3: 1   id 4: 3   id 5: 2
HAND_ORDER = [4, 1, 5, 2, 3, 0]  # descending sum, ties to the lower id


@pytest.mark.parametrize("K", [1, 2, 3, 4, 6])
def test_hand_worked_grid_selection(K):
    ids = orc.cartesian_topk(HAND, 2, K)
    assert list(ids[0]) == HAND_ORDER[:K]


def test_hand_worked_grid_weights():
    ids = orc.cartesian_topk(HAND, 2, 3)
    e = math.e
    w = orc.cartesian_weights(HAND, 2, ids, renormalize=True)[0]
    np.testing.assert_allclose(w, [e / (e + 2), 1 / (e + 2), 1 / (e + 2)], atol=1e-7)
    # plain: softmax over each axis, multiplied
    sr = [1 / (1 + e), e / (1 + e)]
    zc = 1 + e * e + e
    sc = [1 / zc, e * e / zc, e / zc]
    want = [sr[1] * sc[1], sr[0] * sc[1], sr[1] * sc[2]]
    wp = orc.cartesian_weights(HAND, 2, ids, renormalize=False)[0]
    np.testing.assert_allclose(wp, want, atol=1e-7)


def _python_sorted_topk(lg_t, nr, K):
    a, b = lg_t[:nr], lg_t[nr:]
    nc = b.size
    keys = {}
    for i in range(nr):
        for j in range(nc):
            keys[i * nc + j] = float(np.float32(a[i]) + np.float32(b[j]))  # fp32 add
    return sorted(keys, key=lambda e: (-keys[e], e))[:K]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("integer", [True, False])
def test_selection_matches_python_sort(seed, integer):
    r = _rng(50 + seed)
    nr, nc = int(r.integers(1, 7)), int(r.integers(1, 7))
    K = int(r.integers(1, nr * nc + 1))
    lg = _logits(seed, 12, nr, nc, integer)
    ids = orc.cartesian_topk(lg, nr, K)
    for t in range(lg.shape[0]):
        assert list(ids[t]) == _python_sorted_topk(lg[t], nr, K)


@pytest.mark.parametrize("seed", range(8))
def test_pruned_axis_search_equals_full_grid_on_exact_sums(seed):
    """The page's implementation note (top-k0 per axis, then the k0 x k0 pairs) selects
    the same experts as the full grid when the pair sums are exact (small integers):
    a pair outside the per-axis top-K rows is beaten by K pairs of the same column."""
    r = _rng(70 + seed)
    nr, nc = int(r.integers(1, 12)), int(r.integers(1, 12))
    K = int(r.integers(1, nr * nc + 1))
    lg = _logits(seed, 20, nr, nc, integer=True)
    np.testing.assert_array_equal(orc.cartesian_topk(lg, nr, K),
                                  orc.cartesian_topk_pruned(lg, nr, K))


def test_pruned_axis_search_equals_full_grid_on_random_logits():
    lg = _logits(5, 30, 16, 24)
    for K in (1, 7, 40, 200):
        np.testing.assert_array_equal(orc.cartesian_topk(lg, 16, K),
                                      orc.cartesian_topk_pruned(lg, 16, K))


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("axis", ["row", "col"])
def test_single_line_grid_is_the_dense_router(renorm, axis):
    """N_r = 1 (or N_c = 1): the grid is one line and the router is the dense top-K
    router over that line's logits (its log-softmax over one entry is 0)."""
    lg1 = _logits(9, 25, 1, 10)[:, 1:]  # 10 logits per token
    z = np.zeros((25, 1), np.float32)
    if axis == "row":  # p_r = [0], p_c = the line
        lg, nr = np.concatenate([z, lg1], axis=1), 1
    else:              # p_r = the line, p_c = [0]
        lg, nr = np.concatenate([lg1, z], axis=1), 10
    for K in (1, 3, 10):
        ids = orc.cartesian_topk(lg, nr, K)
        want_ids, want_w = dense_orc.route(lg1, K, renormalize=renorm)
        np.testing.assert_array_equal(ids, want_ids)
        np.testing.assert_allclose(orc.cartesian_weights(lg, nr, ids, renorm), want_w, atol=1e-7)


def test_plain_weights_are_a_distribution_over_the_grid():
    lg = _logits(11, 10, 4, 6)
    ids = orc.cartesian_topk(lg, 4, 24)
    w = orc.cartesian_weights(lg, 4, ids, renormalize=False).astype(np.float64)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-6)
    # K = N: renormalising changes nothing
    wr = orc.cartesian_weights(lg, 4, ids, renormalize=True)
    np.testing.assert_allclose(wr, w, atol=1e-7)


def test_renormalised_weights_sum_to_one_and_follow_the_order():
    lg = _logits(12, 40, 8, 8)
    for K in (1, 5, 17):
        ids = orc.cartesian_topk(lg, 8, K)
        w = orc.cartesian_weights(lg, 8, ids, renormalize=True).astype(np.float64)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-6)
        assert np.all(np.diff(w, axis=1) <= 1e-7)  # best slot first
        if K == 1:
            np.testing.assert_array_equal(w, 1.0)


# ----------------------------------------------------------------- schedule
def _read_golden():
    routing, printed, sec = {}, {}, None
    with open(os.path.join(GOLDEN, "omnimoe_expert_centric_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                sec = line
                continue
            k, v = line.split(":")
            vals = [int(z) for z in v.split()]
            (routing if sec == "[routing]" else printed)[int(k)] = vals
    return routing, printed


def test_schedule_worked_example():
    routing, printed = _read_golden()
    T, K = len(routing), len(routing[0])
    ids = np.array([routing[t] for t in range(T)], np.int32)
    N = int(ids.max()) + 1  # the page's ids as they are
    counts, offsets, a2p, p2a = orc.task_schedule(ids, N)
    for e, toks in printed.items():
        got = [int(a) // K for a in p2a[offsets[e]:offsets[e + 1]]]
        assert got == toks
    assert counts.sum() == T * K and offsets[-1] == T * K
    np.testing.assert_array_equal(a2p[p2a], np.arange(T * K))


@pytest.mark.parametrize("seed", range(4))
def test_schedule_equals_the_counting_sort(seed):
    r = _rng(90 + seed)
    N, K, T = int(r.integers(2, 30)), 0, int(r.integers(1, 40))
    K = int(r.integers(1, min(N, 6) + 1))
    ids = np.stack([r.permutation(N)[:K] for _ in range(T)]).astype(np.int32)
    got = orc.task_schedule(ids, N)
    want = dense_orc.permute(ids, N, None)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g, w)


# ----------------------------------------------------------------- experts
def _small_layer(seed, T=12, d=6, nr=3, nc=4, K=5):
    r = _rng(seed)
    x = r.standard_normal((T, d))
    w_row, w_col = r.standard_normal((d, nr)), r.standard_normal((d, nc))
    w_in, w_out = r.standard_normal((nr * nc, d)), r.standard_normal((nr * nc, d))
    return x, w_row, w_col, w_in, w_out, K


@pytest.mark.parametrize("seed", range(3))
def test_three_traversals_agree(seed):
    """Token-centric sum, the page's expert-centric scatter-add, and the dense masked
    product Y = (G * sigma(X W^T)) V compute the same layer."""
    x, w_row, w_col, w_in, w_out, K = _small_layer(seed)
    lg, ids, w, y = orc.forward(x, w_row, w_col, w_in, w_out, K)
    N = w_in.shape[0]
    np.testing.assert_allclose(orc.expert_centric_outputs(x, w_in, w_out, ids, w, N), y,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.dense_outputs(x, w_in, w_out, ids, w, N), y,
                               rtol=1e-12, atol=1e-12)


def test_unit_vector_experts_closed_form():
    """N = d experts with w_in = w_out = the unit vectors: expert i reads and writes
    coordinate i, so y_t[i] = w_{t,i} * silu(x_t[i]) for the selected i, else 0."""
    d, nr, nc, K, T = 6, 2, 3, 4, 9
    r = _rng(21)
    x = r.standard_normal((T, d))
    lg = r.standard_normal((T, nr + nc)).astype(np.float32)
    ids, w = orc.cartesian_route(lg, nr, K)
    y = orc.token_outputs(x, np.eye(d), np.eye(d), ids, w)
    silu = torch.nn.functional.silu(torch.from_numpy(x)).numpy()
    want = np.zeros((T, d))
    for t in range(T):
        for k in range(K):
            want[t, ids[t, k]] = w[t, k] * silu[t, ids[t, k]]
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_workload_sizes():
    c = mi.OMNI_102K
    assert c.N == 102_400 and c.n_rows == c.n_cols == 320
    assert 2 * c.N * c.d == 209_715_200  # the ~200M-parameter layer
    assert c.T == 4096 and c.K == 512


# ----------------------------------------------------------------- planted slips
def test_planted_slips_are_caught(monkeypatch):
    # 1. expert id built column-major (i_c * N_r + i_r): the hand-worked grid notices
    def transposed(a_, b_):
        a = np.asarray(a_, np.float32)
        b = np.asarray(b_, np.float32)
        return (a[None, :] + b[:, None]).reshape(-1)

    monkeypatch.setattr(orc, "pair_sums", transposed)
    assert list(orc.cartesian_topk(HAND, 2, 6)[0]) != HAND_ORDER
    monkeypatch.undo()

    # 2. sign slip inside silu: the unit-vector closed form notices
    monkeypatch.setattr(orc, "silu", lambda s: np.asarray(s, np.float64) /
                        (1.0 + np.exp(np.asarray(s, np.float64))))
    with pytest.raises(AssertionError):
        test_unit_vector_experts_closed_form()
    monkeypatch.undo()

    # 3. plain weights that forget the column axis' normaliser: the sum-to-one pin notices
    real = orc.cartesian_weights

    def no_col_norm(lg_, nr_, ids_, renormalize=True):
        if renormalize:
            return real(lg_, nr_, ids_, True)
        lg = np.asarray(lg_, np.float32).astype(np.float64)
        nc = lg.shape[1] - nr_
        ids = np.asarray(ids_, np.int64)
        pr, pc = lg[:, :nr_], lg[:, nr_:]
        a = np.take_along_axis(pr, ids // nc, axis=1)
        b = np.take_along_axis(pc, ids % nc, axis=1)
        zr = np.exp(pr - pr.max(1, keepdims=True)).sum(1, keepdims=True)
        return (np.exp(a - pr.max(1, keepdims=True)) / zr *
                np.exp(b - pc.max(1, keepdims=True))).astype(np.float32)

    monkeypatch.setattr(orc, "cartesian_weights", no_col_norm)
    with pytest.raises(AssertionError):
        test_plain_weights_are_a_distribution_over_the_grid()
    monkeypatch.undo()

    # 4. a schedule whose expert-major list is rotated by one slot: the worked example notices
    real_s = orc.task_schedule

    def rotated(ids_, N_):
        c, o, a2p, p2a = real_s(ids_, N_)
        return c, o, a2p, np.roll(p2a, 1)

    monkeypatch.setattr(orc, "task_schedule", rotated)
    with pytest.raises(AssertionError):
        test_schedule_worked_example()
    monkeypatch.undo()
