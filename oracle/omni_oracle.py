"""CPU oracle of fine-grained ("atomic", rank-1) experts behind a Cartesian-product
router, run expert-centric.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs do. It shares no code with the CUDA library and
imports nothing from it.

Plain numpy, float64 arithmetic, except the top-K decision, which both sides
take on fp32 sums (below). Library primitives used as steps: ``numpy.matmul``
(fp64), ``numpy.lexsort`` / stable ``numpy.argsort``, ``numpy.exp``.

Source: "Two upstream innovations of MoE: Routing-Free and OmniMoE"
(chatdocs.ruinique.com):
  section 2.1  an atomic expert is two d-vectors, E_i(x) = sigma(x . w_in_i) w_out_i,
               stacked into two (N, d) tables W (in) and V (out);
  section 2.2  Cartesian-product router: expert id i <-> (i_r, i_c) on an
               N_r x N_c grid; p_r = x W_r (d x N_r), p_c = x W_c (d x N_c);
               score S_ij = LogSoftmax(p_r)_i + LogSoftmax(p_c)_j; the
               implementation note: top-k0 along each axis first, k0 = min(sqrt N, K),
               then the top-K among the k0 x k0 candidate pairs;
  section 2.3  expert-centric scheduling: the M = L K (token, expert) tasks are
               flattened, sorted by (expert group, token), run grouped per
               expert, and the outputs are added back per token; the worked
               example lists each expert's tokens in ascending order;
  section 3.2  only a 1-D scalar per task is materialised; token rows are read
               by id inside the kernel;
  section 4    sizes: N = 102,400 = 320 x 320 per layer, K from 512 to 4096,
               4096 tokens through a ~200M-parameter layer.
The layer output is the gate-weighted sum over the selected experts, as for the
dense layer ([P5] SonicMoE explainer, section 1).

Readings where the page is silent (each also listed in the design notes):
  * expert id i = i_r * N_c + i_c (row-major over the grid);
  * sigma: the page instantiates it as "SwiGLU", but an atomic expert has one
    input vector, so there is one pre-activation s = x . w_in and no separate
    gate/up pair; sigma is read as SiLU, the gating nonlinearity of SwiGLU:
    sigma(s) = s / (1 + exp(-s));
  * selection: the K largest S_ij. The two log-sum-exp terms are the same for
    every pair of one token, so the ranking is that of p_r[i] + p_c[j]; the
    decision is taken on the fp32 sum fl32(p_r[i] + p_c[j]) (round to nearest
    even), ties to the lower expert id, slot 0 the best (as the dense router
    selects on fp32 logits rather than on rounded probabilities);
  * weights: renormalised (default): softmax of S over the K selected, i.e.
    exp(s_k - s_0) / sum_j exp(s_j - s_0) with s = p_r[i] + p_c[j] in fp64;
    plain (renormalize=False): exp(S_ij) = softmax(p_r)_i * softmax(p_c)_j,
    the factorised probability over all N experts (it sums to 1 over the grid);
  * expert group = one expert: the page does not say how experts are grouped,
    and the grouping changes the execution order only, not the result.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def as_f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=F64)


# --------------------------------------------------------------------------- router
def cartesian_logits(x, w_row, w_col):
    """Section 2.2: p_r = x W_r, p_c = x W_c; fp64 products, rounded to fp32.
    Returns one [T, N_r + N_c] fp32 array, row-axis logits first."""
    xf = as_f64(x)
    return np.concatenate([xf @ as_f64(w_row), xf @ as_f64(w_col)], axis=1).astype(np.float32)


def pair_sums(p_r_t, p_c_t) -> np.ndarray:
    """fl32(p_r[i] + p_c[j]) for one token on the N_r x N_c grid (numpy float32
    addition rounds to nearest even); flattened index = expert id i*N_c + j."""
    a = np.asarray(p_r_t, dtype=np.float32)
    b = np.asarray(p_c_t, dtype=np.float32)
    return (a[:, None] + b[None, :]).reshape(-1)


def cartesian_topk(logits_f32, n_rows: int, K: int) -> np.ndarray:
    """Section 2.2: the K best experts of each token over the whole grid (brute
    force over all N pairs). Order key (fp32 pair sum descending, expert id
    ascending): ``np.lexsort`` sorts by its last key first."""
    lg = np.asarray(logits_f32, dtype=np.float32)
    T = lg.shape[0]
    n_cols = lg.shape[1] - n_rows
    N = n_rows * n_cols
    if not (1 <= K <= N):
        raise ValueError("need 1 <= K <= N")
    ids = np.arange(N)
    out = np.empty((T, K), dtype=np.int32)
    for t in range(T):
        s = pair_sums(lg[t, :n_rows], lg[t, n_rows:]).astype(F64)
        order = np.lexsort((ids, -s))
        out[t] = order[:K]
    return out


def cartesian_topk_pruned(logits_f32, n_rows: int, K: int) -> np.ndarray:
    """Section 2.2, the implementation note: top-k0 along each axis first (k0 =
    min(axis length, K); with N_r = N_c = sqrt N this is the page's min(sqrt N, K)),
    then the K best pairs among the k0_r x k0_c candidates. Same order keys as
    ``cartesian_topk``; a second algorithm for the same selection."""
    lg = np.asarray(logits_f32, dtype=np.float32)
    T = lg.shape[0]
    n_cols = lg.shape[1] - n_rows
    k_r, k_c = min(n_rows, K), min(n_cols, K)
    out = np.empty((T, K), dtype=np.int32)
    for t in range(T):
        a = lg[t, :n_rows]
        b = lg[t, n_rows:]
        rows = np.lexsort((np.arange(n_rows), -a.astype(F64)))[:k_r]
        cols = np.lexsort((np.arange(n_cols), -b.astype(F64)))[:k_c]
        cand = (rows[:, None] * n_cols + cols[None, :]).reshape(-1)
        s = (a[rows][:, None] + b[cols][None, :]).reshape(-1).astype(F64)
        order = np.lexsort((cand, -s))
        out[t] = cand[order[:K]]
    return out


def cartesian_weights(logits_f32, n_rows: int, ids, renormalize: bool = True) -> np.ndarray:
    """Gate weights of the selected experts (readings in the module docstring), fp64,
    rounded to fp32."""
    lg = np.asarray(logits_f32, dtype=np.float32).astype(F64)
    ids = np.asarray(ids, dtype=np.int64)
    n_cols = lg.shape[1] - n_rows
    pr, pc = lg[:, :n_rows], lg[:, n_rows:]
    ir, ic = ids // n_cols, ids % n_cols
    a = np.take_along_axis(pr, ir, axis=1)
    b = np.take_along_axis(pc, ic, axis=1)
    if renormalize:
        s = a + b
        e = np.exp(s - s.max(axis=1, keepdims=True))
        return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)
    mr = pr.max(axis=1, keepdims=True)
    mc = pc.max(axis=1, keepdims=True)
    zr = np.exp(pr - mr).sum(axis=1, keepdims=True)
    zc = np.exp(pc - mc).sum(axis=1, keepdims=True)
    return (np.exp(a - mr) / zr * np.exp(b - mc) / zc).astype(np.float32)


def cartesian_route(logits_f32, n_rows: int, K: int, renormalize: bool = True):
    ids = cartesian_topk(logits_f32, n_rows, K)
    return ids, cartesian_weights(logits_f32, n_rows, ids, renormalize)


# --------------------------------------------------------------------------- schedule
def task_schedule(topk_ids_, N: int):
    """Section 2.3: flatten the tasks a = t*K + k and sort them by (expert, token),
    i.e. a stable sort of the flat assignments by expert id (one token picks an
    expert once, so ascending a is ascending token inside an expert).
      counts[N]          tasks per expert
      offsets[N+1]       exclusive scan of counts
      perm_to_assign[p]  expert-major task slot -> a
      assign_to_perm[a]  a -> expert-major task slot
    """
    ids = np.asarray(topk_ids_, dtype=np.int64).reshape(-1)
    if ids.size and (ids.min() < 0 or ids.max() >= N):
        raise ValueError("expert id out of range")
    p2a = np.argsort(ids, kind="stable")
    counts = np.bincount(ids, minlength=N)
    offsets = np.zeros(N + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    a2p = np.empty_like(p2a)
    a2p[p2a] = np.arange(p2a.size)
    return (counts.astype(np.int32), offsets.astype(np.int32), a2p.astype(np.int32),
            p2a.astype(np.int32))


# --------------------------------------------------------------------------- experts
def silu(s):
    s = as_f64(s)
    return s / (1.0 + np.exp(-s))


def task_scalars(x, w_in, topk_ids_, topk_w_, tokens=None) -> np.ndarray:
    """Per task (t, k): h = w_{t,k} * sigma(x_t . w_in[i_{t,k}]) (section 2.1; the
    1-D per-task scalar of section 3.2). Rows ``tokens`` only (default all);
    returns [len(tokens), K] fp64."""
    ids = np.asarray(topk_ids_, dtype=np.int64)
    w = as_f64(topk_w_)
    T, K = ids.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    xf = as_f64(x[tokens] if not hasattr(x, "detach") else x[tokens.tolist()])
    W = w_in
    h = np.empty((tokens.size, K), dtype=F64)
    for j, t in enumerate(tokens):
        rows = as_f64(W[ids[t].tolist()] if hasattr(W, "detach") else W[ids[t]])  # [K, d]
        h[j] = w[t] * silu(rows @ xf[j])
    return h


def token_outputs(x, w_in, w_out, topk_ids_, topk_w_, tokens=None) -> np.ndarray:
    """y_t = sum_k w_{t,k} sigma(x_t . w_in[i_k]) w_out[i_k] for the rows ``tokens``
    (token-centric traversal of the same sum), fp64 [len(tokens), d]."""
    ids = np.asarray(topk_ids_, dtype=np.int64)
    T, K = ids.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    h = task_scalars(x, w_in, ids, topk_w_, tokens)
    out = np.empty((tokens.size, np.asarray(x.shape)[1]), dtype=F64)
    for j, t in enumerate(tokens):
        V = as_f64(w_out[ids[t].tolist()] if hasattr(w_out, "detach") else w_out[ids[t]])
        out[j] = h[j] @ V
    return out


def expert_centric_outputs(x, w_in, w_out, topk_ids_, topk_w_, N: int) -> np.ndarray:
    """Section 2.3 as written: for each expert in the (expert, token) task order,
    load its two vectors once, compute its tokens' scalars and add each token's
    share into the output rows (scatter-add). fp64 [T, d]."""
    ids = np.asarray(topk_ids_, dtype=np.int64)
    T, K = ids.shape
    w = as_f64(topk_w_).reshape(-1)
    xf = as_f64(x)
    Wf, Vf = as_f64(w_in), as_f64(w_out)
    _, offsets, _, p2a = task_schedule(ids, N)
    y = np.zeros((T, xf.shape[1]), dtype=F64)
    for e in range(N):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        a = p2a[lo:hi].astype(np.int64)
        tok = a // K
        h = w[a] * silu(xf[tok] @ Wf[e])
        y[tok] += h[:, None] * Vf[e][None, :]
    return y


def dense_outputs(x, w_in, w_out, topk_ids_, topk_w_, N: int) -> np.ndarray:
    """Every expert evaluated for every token, then masked: Y = (G * sigma(X W^T)) V
    with G[t, i] the gate weight when i is selected by t, else 0 (the plain
    definition of the sparse layer; small shapes only). fp64 [T, d]."""
    ids = np.asarray(topk_ids_, dtype=np.int64)
    T, K = ids.shape
    G = np.zeros((T, N), dtype=F64)
    np.put_along_axis(G, ids, as_f64(topk_w_), axis=1)
    S = as_f64(x) @ as_f64(w_in).T
    return (G * silu(S)) @ as_f64(w_out)


def forward(x, w_row, w_col, w_in, w_out, K: int, renormalize: bool = True):
    """The whole layer on small shapes: (logits, ids, weights, y)."""
    n_rows = np.asarray(w_row.shape)[1]
    lg = cartesian_logits(x, w_row, w_col)
    ids, w = cartesian_route(lg, int(n_rows), K, renormalize)
    y = token_outputs(x, w_in, w_out, ids, w)
    return lg, ids, w, y
