"""CPU oracle of the single-GPU MoE-layer forward (router -> top-k -> counts and
scan -> stable permutation -> grouped SwiGLU FFN -> weighted combine).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs do. It shares no code with the CUDA library and
imports nothing from it.

Plain numpy, float64 arithmetic unless a step is an integer decision that the
kernels take in fp32 (the top-k selection compares fp32 logits, as the kernels
do). Slow and obviously correct is the goal: no blocking, no fusion, no
reordering beyond what each definition states. Library primitives used as
steps: ``numpy.matmul``/``dot`` (fp64), ``numpy.lexsort``, ``numpy.exp``.

Sources (page title, section):
  [P1] "Operators & compilers: MoE routing and sparse kernels"
       (charles2530.github.io), sections 2-4: top-k routing, token permutation
       by counting + prefix sum, capacity factor with drops.
  [P2] "Two upstream innovations of MoE: Routing-Free and OmniMoE"
       (chatdocs.ruinique.com), section 1.1 (Router -> Softmax -> TopK) and
       section 2.3 (expert-centric scheduling: flatten the (token, expert)
       tasks, sort by (expert, token), run grouped, scatter-add back).
  [P4] "How AI chips support MoE", chapter 4, sections 4.2-4.3 (gating is a
       linear map, then softmax, then top-K selection).
  [P5] SonicMoE explainer (gitcode.csdn.net), section 1 (y = sum_i gate_i(x) *
       expert_i(x) over the top-k experts), section 3 (the GPU pipeline:
       route, regroup to expert-major, grouped GEMM, SwiGLU, second grouped
       GEMM, scatter/combine), section 6.4 (the backward without caching Y:
       dA' = dO W_down^T, dS = <dA', A>), section 11 (expert-major metadata:
       per-expert counts, expert-major slot -> token, token-major slot ->
       expert-major slot).

Readings where the pages are silent (each also listed in the design notes):
  * top-k order: descending logit, ties to the lower expert id, +0 == -0;
    selection is on the fp32 logits (softmax is monotone);
  * weights: softmax restricted to the K selected, i.e. renormalised;
  * capacity C = ceil(cf * T * K / E); an expert keeps its first C
    assignments in token order and drops the rest;
  * order inside an expert: ascending token id (the section 2.3 example of
    [P2] shows it); dropped slots contribute 0 and are not re-renormalised;
  * SwiGLU(g, u) = g / (1 + exp(-g)) * u with g from W_gate, u from W_up;
  * tile-aware token rounding ([P5] 6.5 names it without a rule): an expert
    with c >= R routed assignments keeps R * floor(c / R) of them, those with
    the largest router logit for that expert, among equal logits the earlier
    token; experts with c < R keep all; nothing is added (rounding down only).
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

F64 = np.float64


def as_f64(a) -> np.ndarray:
    """Widen an array (numpy, or a CPU torch tensor of any float dtype) to fp64."""
    if hasattr(a, "detach"):  # torch tensor: bf16 has no numpy dtype
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=F64)


# --------------------------------------------------------------------------- router
def router_logits(x, w_r, bias=None) -> np.ndarray:
    """[P4] 4.2 / [P2] 1.1: router scores are a linear map, logits = x . W_r.

    x[T, d], W_r[d, E]; fp64 products and sums, optional per-expert bias added
    to every token's logits, then rounded to fp32 (the precision in which the
    top-k decision is taken on both sides)."""
    z = as_f64(x) @ as_f64(w_r)
    if bias is not None:
        z = z + as_f64(bias)[None, :]
    return z.astype(np.float32)


def topk_ids(logits_f32, K: int) -> np.ndarray:
    """[P1] 2, [P4] 4.3: per token, the K experts with the largest logits.

    Order key (logit descending, expert id ascending); slot 0 holds the best.
    ``np.lexsort`` sorts by its last key first, so the keys are (id, -logit).
    Comparisons are on fp32 values, where +0 and -0 are equal."""
    lg = np.asarray(logits_f32, dtype=np.float32)
    T, E = lg.shape
    if not (1 <= K <= E):
        raise ValueError("need 1 <= K <= E")
    ids = np.broadcast_to(np.arange(E), (T, E))
    neg = -lg.astype(F64)  # exact; -(+0) == -(-0) compare equal
    order = np.lexsort((ids, neg), axis=1)
    return order[:, :K].astype(np.int32)


def topk_weights(logits_f32, ids, renormalize: bool = True) -> np.ndarray:
    """[P2] 1.1 Router -> Softmax -> TopK, with the top-K probabilities renormalised.

    w_k = exp(l_k - m) / sum_{j in S} exp(l_j - m), m the token's largest
    logit, S = the K selected experts (renormalised) or all E experts (plain
    softmax, ``renormalize=False``). fp64, rounded to fp32."""
    lg = np.asarray(logits_f32, dtype=np.float32).astype(F64)
    T, E = lg.shape
    m = lg.max(axis=1, keepdims=True)
    p = np.exp(lg - m)
    sel = np.take_along_axis(p, np.asarray(ids, dtype=np.int64), axis=1)
    den = sel.sum(axis=1, keepdims=True) if renormalize else p.sum(axis=1, keepdims=True)
    return (sel / den).astype(np.float32)


def route(logits_f32, K: int, renormalize: bool = True):
    ids = topk_ids(logits_f32, K)
    return ids, topk_weights(logits_f32, ids, renormalize)


# --------------------------------------------------------------------------- dispatch
def capacity(capacity_factor: float, T: int, K: int, E: int) -> Optional[int]:
    """[P1] 4: an upper bound on the tokens one expert receives.

    C = ceil(cf * T * K / E), computed in double from the fp32 factor; cf <= 0
    means no limit (None)."""
    cf = float(np.float32(capacity_factor))
    if cf <= 0.0:
        return None
    return int(math.ceil(cf * T * K / E))


def tile_round_keep(topk_ids_, logits_f32, E: int, R: int) -> np.ndarray:
    """[P5] 6.5: routing that takes the GEMM's M tile into account, so that each
    expert's row count fits whole tiles. Reading (the pages give no rule):
    expert e with c_e >= R routed assignments keeps R * floor(c_e / R) of them,
    the ones whose router logit for e is largest; among equal logits the
    earlier token is kept and the later one dropped; an expert with c_e < R
    keeps all of its assignments. Nothing is added.
    Returns keep[T, K] (bool): False marks a dropped assignment."""
    ids = np.asarray(topk_ids_, dtype=np.int64)
    lg = np.asarray(logits_f32, dtype=np.float32)
    T, K = ids.shape
    keep = np.ones((T, K), dtype=bool)
    if R <= 1:
        return keep
    for e in range(E):
        tok, slot = np.nonzero(ids == e)  # ascending token
        c = tok.size
        if c < R or c % R == 0:
            continue
        n_drop = c % R
        score = lg[tok, e].astype(F64)
        # ascending by (score, -token): the first n_drop are the weakest
        order = np.lexsort((-tok, score))
        drop = order[:n_drop]
        keep[tok[drop], slot[drop]] = False
    return keep


def tile_round_select(topk_ids_, logits_f32, E: int, R: int, mode: str = "down"):
    """[P5] 6.5 with rounding in either direction (the library's reading: the page says
    only that expert token counts are brought closer to kernel-friendly tile shapes).
    For expert e with c routed assignments and r = c mod R != 0:
      down    - c >= R: drop its r weakest assignments (tile_round_keep); c < R: keep all;
      up      - add the m = min(R - r, T - c) tokens that did not route to e with the
                largest router logit for e (equal logits: the earlier token), each gaining
                one more slot;
      nearest - down when r <= R - r, else up.
    Returns (keep [T, K] bool, add_tok [n], add_exp [n]); the added assignments are
    listed by expert, then by ascending token."""
    if mode not in ("down", "up", "nearest"):
        raise ValueError(mode)
    ids = np.asarray(topk_ids_, dtype=np.int64)
    lg = np.asarray(logits_f32, dtype=np.float32)
    T, K = ids.shape
    keep = np.ones((T, K), dtype=bool)
    add_tok, add_exp = [], []
    if R <= 1:
        return keep, np.zeros(0, np.int64), np.zeros(0, np.int64)
    for e in range(E):
        tok, slot = np.nonzero(ids == e)  # ascending token
        c = tok.size
        r = c % R
        if r == 0:
            continue
        up = mode == "up" or (mode == "nearest" and r > R - r)
        if not up:
            if c >= R:
                order = np.lexsort((-tok, lg[tok, e].astype(F64)))  # weakest first
                drop = order[:r]
                keep[tok[drop], slot[drop]] = False
            continue
        routed = np.zeros(T, dtype=bool)
        routed[tok] = True
        cand = np.nonzero(~routed)[0]
        m = min(R - r, cand.size)
        if m == 0:
            continue
        # strongest first: larger logit, then the earlier token
        order = np.lexsort((cand, -lg[cand, e].astype(F64)))
        chosen = np.sort(cand[order[:m]])
        add_tok.extend(chosen.tolist())
        add_exp.extend([e] * m)
    return keep, np.asarray(add_tok, np.int64), np.asarray(add_exp, np.int64)


def round_weights(logits_f32, topk_ids_, add_tok, add_exp, renormalize: bool = True):
    """Weights after rounding up: each token's selection is its K routed experts plus the
    experts it was added to. Renormalised: w = exp(l - l_max) / (sum over the enlarged
    selection of exp(l_j - l_max)) (they still sum to 1); plain: softmax(l) over all E at
    every selected expert (the routed weights are unchanged). Dropped assignments keep
    their place in the sum (reading 6: no re-renormalisation). fp64, rounded to fp32.
    Returns (topk_w [T, K], add_w [n])."""
    lg = np.asarray(logits_f32, dtype=np.float32).astype(F64)
    ids = np.asarray(topk_ids_, dtype=np.int64)
    T, K = ids.shape
    add_tok = np.asarray(add_tok, np.int64)
    add_exp = np.asarray(add_exp, np.int64)
    w = np.zeros((T, K), dtype=F64)
    add_w = np.zeros(add_tok.size, dtype=F64)
    for t in range(T):
        extra = np.nonzero(add_tok == t)[0]
        sel = np.concatenate([ids[t], add_exp[extra]])
        if renormalize:
            top = lg[t, ids[t, 0]]
            z = np.exp(lg[t, sel] - top)
            p = z / z.sum()
        else:
            m = lg[t].max()
            p = np.exp(lg[t, sel] - m) / np.exp(lg[t] - m).sum()
        w[t] = p[:K]
        add_w[extra] = p[K:]
    return w.astype(np.float32), add_w.astype(np.float32)


def permute_ext(ids_ext, E: int):
    """The stable permutation over an extended assignment list (routed assignments a =
    t*K + k first, then the added ones): expert-major, ascending flat index inside an
    expert; -1 marks an assignment that does not exist (dropped). Returns (offsets,
    assign_to_perm, perm_to_assign) over len(ids_ext) assignments."""
    ids = np.asarray(ids_ext, dtype=np.int64).reshape(-1)
    A = ids.size
    offsets = np.zeros(E + 1, dtype=np.int64)
    members = [np.nonzero(ids == e)[0] for e in range(E)]
    for e in range(E):
        offsets[e + 1] = offsets[e] + members[e].size
    p2a = np.full(A, -1, dtype=np.int64)
    a2p = np.full(A, -1, dtype=np.int64)
    for e in range(E):
        for r, a in enumerate(members[e]):
            p2a[offsets[e] + r] = a
            a2p[a] = offsets[e] + r
    return offsets.astype(np.int32), a2p.astype(np.int32), p2a.astype(np.int32)


def permute(topk_ids_, E: int, C: Optional[int] = None, keep=None):
    """[P1] 3 (counting + prefix sum), [P2] 2.3 (sort tasks by (expert, token)),
    [P5] 11 (expert-major metadata).

    Flat assignment a = t*K + k. For each expert e, its assignments in
    ascending a (= ascending token t, since one token picks an expert once);
    the first C are kept, the rest dropped.
    ``keep`` (optional, [T, K] or [T*K] bool) removes assignments first (token
    rounding); they count in ``counts`` and are dropped like capacity overflow.
      counts[e]          raw number of assignments to e (sums to T*K)
      offsets[E+1]       exclusive scan of kept counts min(counts, C)
      perm_to_assign[p]  expert-major slot -> a   (first offsets[E] valid, rest -1)
      assign_to_perm[a]  a -> expert-major slot, or -1 when dropped
    """
    ids = np.asarray(topk_ids_, dtype=np.int64).reshape(-1)
    A = ids.size
    if A and (ids.min() < 0 or ids.max() >= E):
        raise ValueError("expert id out of range")
    keep_mask = None if keep is None else np.asarray(keep, dtype=bool).reshape(-1)
    counts = np.zeros(E, dtype=np.int64)
    kept = np.zeros(E, dtype=np.int64)
    members = []
    for e in range(E):
        a_e = np.nonzero(ids == e)[0]  # ascending flat index
        counts[e] = a_e.size
        if keep_mask is not None:  # assignments removed by token rounding
            a_e = a_e[keep_mask[a_e]]
        kept_e = a_e if C is None else a_e[:C]
        kept[e] = kept_e.size
        members.append(kept_e)
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + kept[e]
    perm_to_assign = np.full(A, -1, dtype=np.int64)
    assign_to_perm = np.full(A, -1, dtype=np.int64)
    for e in range(E):
        for r, a in enumerate(members[e]):
            p = offsets[e] + r
            perm_to_assign[p] = a
            assign_to_perm[a] = p
    return (counts.astype(np.int32), offsets.astype(np.int32),
            assign_to_perm.astype(np.int32), perm_to_assign.astype(np.int32))


def expert_of_slot(offsets, p: int) -> int:
    """The expert that owns expert-major slot p (offsets[e] <= p < offsets[e+1])."""
    off = np.asarray(offsets)
    for e in range(off.size - 1):
        if off[e] <= p < off[e + 1]:
            return e
    raise IndexError(p)


def gather_rows(x, perm_to_assign, offsets, K: int) -> np.ndarray:
    """[P5] 6.2 "pre-gather": X_perm[p] = x[token(p)] for the kept slots
    (a pure data move, compared bit-exactly)."""
    xa = np.asarray(x)
    n_kept = int(np.asarray(offsets)[-1])
    tok = np.asarray(perm_to_assign[:n_kept], dtype=np.int64) // K
    return xa[tok]


# --------------------------------------------------------------------------- experts
def swiglu(g, u) -> np.ndarray:
    """[P5] 3 item 4 (activation between the GEMMs, SwiGLU):
    silu(g) * u with silu(g) = g / (1 + exp(-g))."""
    g = as_f64(g)
    return g / (1.0 + np.exp(-g)) * as_f64(u)


def expert_ffn(x_rows, w_gate_e, w_up_e, w_down_e) -> np.ndarray:
    """[P5] 3 items 3-5 for one expert: (SwiGLU(x W_gate, x W_up)) W_down, fp64."""
    xr = as_f64(x_rows)
    g = xr @ as_f64(w_gate_e)
    u = xr @ as_f64(w_up_e)
    return swiglu(g, u) @ as_f64(w_down_e)


def grouped_ffn(x, perm_to_assign, offsets, K: int, w_gate, w_up, w_down):
    """[P5] 3 items 3-5 and 6.2: for each expert e, the rows p in
    [offsets[e], offsets[e+1]) hold token perm_to_assign[p] // K; both GEMMs
    run on them. Returns (a_act, y_perm) in fp64 (no intermediate rounding)."""
    off = np.asarray(offsets, dtype=np.int64)
    E = off.size - 1
    n_kept = int(off[-1])
    xa = as_f64(x)
    n = w_gate.shape[2]
    d = w_down.shape[2]
    a_act = np.zeros((n_kept, n), dtype=F64)
    y_perm = np.zeros((n_kept, d), dtype=F64)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        tok = np.asarray(perm_to_assign[lo:hi], dtype=np.int64) // K
        xr = xa[tok]
        g = xr @ as_f64(w_gate[e])
        u = xr @ as_f64(w_up[e])
        a_act[lo:hi] = swiglu(g, u)
        y_perm[lo:hi] = a_act[lo:hi] @ as_f64(w_down[e])
    return a_act, y_perm


def grouped_ffn_rows(slots, x, perm_to_assign, offsets, K: int, w_gate, w_up, w_down):
    """grouped_ffn for chosen expert-major slots only (the sampled full-size check): row p of
    a_act and y_perm, with p's expert found from offsets and its token perm_to_assign[p] // K.
    The slots of one expert run together, so each expert's weights are widened once.
    Returns (a_rows, y_rows) in the order of `slots`, fp64."""
    slots = np.asarray(slots, dtype=np.int64)
    off = np.asarray(offsets, dtype=np.int64)
    n = w_gate.shape[2]
    d = w_down.shape[2]
    a_rows = np.zeros((slots.size, n), dtype=F64)
    y_rows = np.zeros((slots.size, d), dtype=F64)
    by_expert = {}
    for i, p in enumerate(slots):
        by_expert.setdefault(expert_of_slot(off, int(p)), []).append(i)
    for e, idx in by_expert.items():
        tok = np.asarray(perm_to_assign, dtype=np.int64)[slots[idx]] // K
        xr = as_f64(x[tok])
        a = swiglu(xr @ as_f64(w_gate[e]), xr @ as_f64(w_up[e]))
        a_rows[idx] = a
        y_rows[idx] = a @ as_f64(w_down[e])
    return a_rows, y_rows


def gate_up_preact(x, perm_to_assign, offsets, K: int, w_gate, w_up):
    """[P5] 3 item 3: the pre-activations of the kept slots, g[p] = x[tok(p)] W_gate[e] and
    u[p] = x[tok(p)] W_up[e] (fp64), which the backward below reads."""
    off = np.asarray(offsets, dtype=np.int64)
    E = off.size - 1
    n_kept = int(off[-1])
    xa = as_f64(x)
    n = w_gate.shape[2]
    g = np.zeros((n_kept, n), dtype=F64)
    u = np.zeros((n_kept, n), dtype=F64)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        tok = np.asarray(perm_to_assign[lo:hi], dtype=np.int64) // K
        g[lo:hi] = xa[tok] @ as_f64(w_gate[e])
        u[lo:hi] = xa[tok] @ as_f64(w_up[e])
    return g, u


def backward_act(d_out, topk_w_, assign_to_perm, perm_to_assign, offsets, K: int, w_down, g, u):
    """[P5] 6.4, the backward of the expert half of the layer without caching Y: for the
    kept slot p of expert e holding token t's slot k (a = t*K + k = perm_to_assign[p]),
      dA'[p] = dO[t] W_down[e]^T               (the rows of dO gathered by token)
      dS[p]  = <dA'[p], A[p]>, A = silu(g) * u   (= dL/dw[t, k]: out = sum_k w y, y = A W_down)
      dA[p]  = w[t, k] dA'[p]
      dG[p]  = dA[p] * u * silu'(g),  silu'(g) = s (1 + g (1 - s)),  s = 1 / (1 + e^-g)
      dU[p]  = dA[p] * silu(g)
    Returns dG, dU ([kept, n], fp64) and d_w ([T, K], fp64; 0 at dropped slots)."""
    off = np.asarray(offsets, dtype=np.int64)
    E = off.size - 1
    dO = as_f64(d_out)
    T = dO.shape[0]
    w = as_f64(topk_w_).reshape(-1)
    a2p = np.asarray(assign_to_perm, dtype=np.int64)
    n_kept = int(off[-1])
    n = g.shape[1]
    dG = np.zeros((n_kept, n), dtype=F64)
    dU = np.zeros((n_kept, n), dtype=F64)
    dS = np.zeros(n_kept, dtype=F64)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        a = np.asarray(perm_to_assign[lo:hi], dtype=np.int64)
        dA1 = dO[a // K] @ as_f64(w_down[e]).T
        ge, ue = g[lo:hi], u[lo:hi]
        sg = 1.0 / (1.0 + np.exp(-ge))
        silu = ge * sg
        dS[lo:hi] = np.sum(dA1 * (silu * ue), axis=1)
        dA = w[a][:, None] * dA1
        dG[lo:hi] = dA * ue * sg * (1.0 + ge * (1.0 - sg))
        dU[lo:hi] = dA * silu
    d_w = np.zeros(T * K, dtype=F64)
    kept = a2p >= 0
    d_w[kept] = dS[a2p[kept]]
    return dG, dU, d_w.reshape(T, K)


def backward_dx(dG, dU, assign_to_perm, perm_to_assign, offsets, K: int, T: int, w_gate, w_up):
    """[P5] 6.4 continued: the input gradient through the experts (routing held fixed),
      dX_perm[p] = dG[p] W_gate[e]^T + dU[p] W_up[e]^T
      dx[t]      = sum over t's kept slots k of dX_perm[assign_to_perm[t*K + k]], in k order.
    Returns dx [T, d] (fp64)."""
    off = np.asarray(offsets, dtype=np.int64)
    E = off.size - 1
    d = w_gate.shape[1]
    n_kept = int(off[-1])
    dXp = np.zeros((n_kept, d), dtype=F64)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        dXp[lo:hi] = (as_f64(dG[lo:hi]) @ as_f64(w_gate[e]).T
                      + as_f64(dU[lo:hi]) @ as_f64(w_up[e]).T)
    a2p = np.asarray(assign_to_perm, dtype=np.int64).reshape(T, K)
    dx = np.zeros((T, d), dtype=F64)
    for k in range(K):
        kept = a2p[:, k] >= 0
        dx[kept] += dXp[a2p[kept, k]]
    return dx


def backward_router(d_w, topk_ids_, logits_f32, x, w_r, renormalize: bool = True):
    """The router's backward with the top-K selection held fixed ([P2] 1.1 Router ->
    Softmax -> TopK read backwards; [P4] 4.2: the gate is the linear map x W_r + bias).
      renormalised: w_k = exp(l_{i_k}) / sum_{j in S} exp(l_{i_j})  =>
        dL/dl_{i_j} = w_j (d_w_j - sum_k w_k d_w_k), 0 off the selected set S;
      plain: w_k = p_{i_k}, p = softmax over all E  =>
        dL/dl_e = p_e (g_e - sum_k w_k d_w_k), g_e = d_w of e if selected else 0.
    Then d_W_r = x^T dL/dl, d_bias = sum_t dL/dl_t, and the router's term of the input
    gradient d_x = dL/dl W_r^T. Returns (d_logits [T, E], d_w_r [d, E], d_bias [E],
    d_x [T, d]), fp64."""
    ids = np.asarray(topk_ids_, dtype=np.int64)
    T, K = ids.shape
    lg = as_f64(logits_f32)
    E = lg.shape[1]
    gw = as_f64(d_w).reshape(T, K)
    if renormalize:
        sel = np.take_along_axis(lg, ids, axis=1)
        m = sel[:, :1]
        ex = np.exp(sel - m)
        w = ex / ex.sum(axis=1, keepdims=True)
    else:
        m = lg.max(axis=1, keepdims=True)
        p = np.exp(lg - m)
        p /= p.sum(axis=1, keepdims=True)
        w = np.take_along_axis(p, ids, axis=1)
    s = np.sum(w * gw, axis=1, keepdims=True)
    d_logits = np.zeros((T, E), dtype=F64)
    if renormalize:
        np.put_along_axis(d_logits, ids, w * (gw - s), axis=1)
    else:
        g = np.zeros((T, E), dtype=F64)
        np.put_along_axis(g, ids, gw, axis=1)
        d_logits = p * (g - s)
    xa = as_f64(x)
    d_w_r = xa.T @ d_logits
    d_bias = d_logits.sum(axis=0)
    d_x = d_logits @ as_f64(w_r).T
    return d_logits, d_w_r, d_bias, d_x


def combine(y_perm, assign_to_perm, topk_w, T: int, K: int) -> np.ndarray:
    """[P5] 1 and 3 item 6: out[t] = sum_k w[t,k] * y[assign_to_perm[t*K+k]],
    summed in k order; a dropped slot (-1) adds nothing and the other weights
    are not rescaled. fp64."""
    y = as_f64(y_perm)
    a2p = np.asarray(assign_to_perm, dtype=np.int64).reshape(T, K)
    w = as_f64(topk_w).reshape(T, K)
    out = np.zeros((T, y.shape[1]), dtype=F64)
    for k in range(K):
        p = a2p[:, k]
        keep = p >= 0
        out[keep] += w[keep, k, None] * y[p[keep]]
    return out


def slot_tokens(perm_to_assign, n_kept: int, K: int, T: int, add_tok) -> np.ndarray:
    """Token of each kept expert-major slot over the extended assignment list: a < T*K is
    token a // K, an added assignment a = T*K + j is add_tok[j]."""
    p2a = np.asarray(perm_to_assign, dtype=np.int64)[:n_kept]
    add_tok = np.asarray(add_tok, np.int64)
    A0 = T * K
    return np.where(p2a < A0, p2a // K, add_tok[np.maximum(p2a - A0, 0)] if add_tok.size else 0)


def combine_ext(y_perm, assign_to_perm, topk_w, T: int, K: int, add_tok, add_w) -> np.ndarray:
    """combine over the extended assignments: out[t] = sum_k w[t,k] y[slot(t*K+k)] (k order,
    dropped slots add nothing), then the token's added assignments in expert order
    (= their order in the added list), w y[slot(T*K+j)]. fp64."""
    y = as_f64(y_perm)
    a2p = np.asarray(assign_to_perm, dtype=np.int64)
    out = combine(y, a2p[:T * K], topk_w, T, K)
    add_tok = np.asarray(add_tok, np.int64)
    aw = as_f64(add_w)
    for j in range(add_tok.size):
        p = a2p[T * K + j]
        if p >= 0:
            out[add_tok[j]] += aw[j] * y[p]
    return out


# --------------------------------------------------------------------------- layer
def forward(x, w_r, w_gate, w_up, w_down, K: int, capacity_factor: float = 0.0,
            bias=None, logits=None, renormalize: bool = True, tile_round: int = 0,
            round_mode: str = "down"):
    """The whole layer forward ([P5] section 3 pipeline), every intermediate kept.

    ``logits`` (fp32 [T, E]) replaces x . W_r + bias when given: this is how
    ids/counts/permutation parity is checked on identical logits. ``tile_round``
    = R > 0 applies token rounding to R-row tiles (see tile_round_keep); round_mode "up"
    or "nearest" may add assignments (see tile_round_select), laid out after the routed
    ones (a = T*K + j) and reported in add_tok / add_exp / add_w."""
    T = x.shape[0]
    lg = router_logits(x, w_r, bias) if logits is None else np.asarray(logits, np.float32)
    E = lg.shape[1]
    ids, w = route(lg, K, renormalize)
    C = capacity(capacity_factor, T, K, E)
    if tile_round > 0 and round_mode != "down":
        if C is not None:
            raise ValueError("token rounding and a capacity limit are exclusive")
        keep, add_tok, add_exp = tile_round_select(ids, lg, E, tile_round, round_mode)
        counts = np.bincount(ids.reshape(-1), minlength=E).astype(np.int32)
        ids_ext = np.concatenate([np.where(keep, ids, -1).reshape(-1), add_exp])
        offsets, a2p, p2a = permute_ext(ids_ext, E)
        w, add_w = round_weights(lg, ids, add_tok, add_exp, renormalize)
        n_kept = int(offsets[-1])
        tok = slot_tokens(p2a, n_kept, K, T, add_tok)
        a_act, y_perm = grouped_ffn(x, tok, offsets, 1, w_gate, w_up, w_down)
        out = combine_ext(y_perm, a2p, w, T, K, add_tok, add_w)
        return dict(logits=lg, topk_ids=ids, topk_w=w, counts=counts, offsets=offsets,
                    assign_to_perm=a2p, perm_to_assign=p2a, a_act=a_act, y_perm=y_perm,
                    out=out, capacity=C, add_tok=add_tok, add_exp=add_exp, add_w=add_w,
                    slot_tokens=tok)
    keep = None
    if tile_round > 0:
        if C is not None:
            raise ValueError("token rounding and a capacity limit are exclusive")
        keep = tile_round_keep(ids, lg, E, tile_round)
    counts, offsets, a2p, p2a = permute(ids, E, C, keep)
    a_act, y_perm = grouped_ffn(x, p2a, offsets, K, w_gate, w_up, w_down)
    out = combine(y_perm, a2p, w, T, K)
    return dict(logits=lg, topk_ids=ids, topk_w=w, counts=counts, offsets=offsets,
                assign_to_perm=a2p, perm_to_assign=p2a, a_act=a_act, y_perm=y_perm,
                out=out, capacity=C)


def forward_rows(tokens, x, w_gate, w_up, w_down, topk_ids_, topk_w_, assign_to_perm, K: int):
    """Layer output for a few chosen tokens only (the sampled full-size check):
    out[t] = sum over kept slots k of w[t,k] * FFN_{id[t,k]}(x[t]), summed in k order.
    Each expert's FFN runs once on all chosen tokens routed to it, so its weights are
    widened to fp64 once."""
    tokens = np.asarray(tokens, dtype=np.int64)
    ids = np.asarray(topk_ids_).reshape(-1, K)
    w = as_f64(topk_w_).reshape(-1, K)
    a2p = np.asarray(assign_to_perm).reshape(-1, K)
    d = w_down.shape[2]
    per_slot = np.zeros((tokens.size, K, d), dtype=F64)
    pairs = {}
    for i, t in enumerate(tokens):
        for k in range(K):
            if a2p[t, k] >= 0:
                pairs.setdefault(int(ids[t, k]), []).append((i, k))
    for e, lst in pairs.items():
        rows = np.array([tokens[i] for i, _ in lst], dtype=np.int64)
        y = expert_ffn(as_f64(x[rows]), w_gate[e], w_up[e], w_down[e])
        for j, (i, k) in enumerate(lst):
            per_slot[i, k] = w[tokens[i], k] * y[j]
    out = np.zeros((tokens.size, d), dtype=F64)
    for k in range(K):
        out += per_slot[:, k]
    return out


def dense_reference(x, w_gate, w_up, w_down, topk_ids_, topk_w_, E: int) -> np.ndarray:
    """[P5] 1 read literally: y_t = sum over ALL E experts of gate_{t,e} * expert_e(x_t),
    with gate_{t,e} the routed weight when e is among the token's top-K and 0
    otherwise. No permutation or capacity (used with no capacity limit)."""
    xa = as_f64(x)
    T = xa.shape[0]
    K = np.asarray(topk_ids_).shape[1]
    gate = np.zeros((T, E), dtype=F64)
    for t in range(T):
        for k in range(K):
            gate[t, int(topk_ids_[t, k])] = float(topk_w_[t, k])
    out = np.zeros((T, w_down.shape[2]), dtype=F64)
    for e in range(E):
        out += gate[:, e:e + 1] * expert_ffn(xa, w_gate[e], w_up[e], w_down[e])
    return out
