"""GPU parity of the atomic-expert path (Cartesian-product router, expert-centric
schedule, rank-1 experts), called through the C ABI, against the CPU oracle on the
same seeded inputs.

Bars: expert ids, counts, offsets and both task maps bit-exact given identical
logits (the oracle selects on the logits the GPU produced); weights within 1e-6;
the router GEMM within 1e-3 of the largest |logit| (bf16 inputs, fp32 sums); the
per-task scalars within 1e-4 relative to their largest magnitude (fp32 dot products
of bf16 rows); the layer output max|err| / max|ref| <= 2e-2 and ||err|| / ||ref|| <=
2e-2 (bf16 output)."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import omni_oracle as orc

pytestmark = pytest.mark.gpu

W_ABS = 1e-6
BF16_REL = 2e-2


def cfg_of(T, d, nr, nc, K, renorm=True, logits_given=False, seed=0):
    return mi.OmniConfig(f"omni_T{T}_d{d}_{nr}x{nc}_K{K}", T=T, d=d, n_rows=nr, n_cols=nc, K=K,
                         renormalize=renorm, logits_given=logits_given, seed=seed)


def shape_of(tdr, c, output_mode=0):
    return tdr.make_omni_shape(c.T, c.d, c.n_rows, c.n_cols, c.K, c.renormalize, output_mode)


def rel_errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    return (np.abs(diff).max() / max(np.abs(ref).max(), 1e-30),
            np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30))


def assert_bf16_close(got, ref, what):
    mx, l2 = rel_errors(got, ref)
    assert mx <= BF16_REL and l2 <= BF16_REL, f"{what}: max-rel {mx:.3e} l2-rel {l2:.3e}"


def check_route(lg, nr, K, renorm, ids_gpu, w_gpu, tokens=None):
    lg = np.asarray(lg, np.float32)
    ids_gpu = np.asarray(ids_gpu)
    w_gpu = np.asarray(w_gpu, np.float64)
    if tokens is not None:
        lg, ids_gpu, w_gpu = lg[tokens], ids_gpu[tokens], w_gpu[tokens]
    ids_ref = orc.cartesian_topk(lg, nr, K)
    np.testing.assert_array_equal(ids_gpu, ids_ref)
    w_ref = orc.cartesian_weights(lg, nr, ids_ref, renorm)
    assert np.abs(w_gpu - w_ref).max() <= W_ABS
    return ids_ref, w_ref


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("T,nr,nc,K", [
    (64, 8, 8, 1), (64, 8, 8, 64), (100, 16, 24, 40), (33, 32, 32, 200), (40, 320, 320, 512),
    (20, 13, 7, 50), (17, 1000, 3, 100), (12, 64, 64, 4096), (9, 1024, 1024, 300),
    (5, 1024, 1024, 4096),  # staircase above the shared-memory key store: keys recomputed
])
@pytest.mark.parametrize("renorm", [True, False])
def test_route_on_given_logits(cuda_lib, T, nr, nc, K, renorm):
    tdr = cuda_lib
    c = cfg_of(T, 256, nr, nc, K, renorm, logits_given=True, seed=nr + K)
    inp = mi.make_omni_inputs(c, with_experts=False)
    lg = inp.logits.cuda()
    ids, w, _ = tdr.omni_route(shape_of(tdr, c), logits_in=lg)
    torch.cuda.synchronize()
    assert tdr.device_status() == 0
    check_route(inp.logits.numpy(), nr, K, renorm, ids.cpu().numpy(), w.cpu().numpy())


@pytest.mark.parametrize("kind", ["small_integers", "all_equal", "one_row_tied", "signed_zero"])
def test_route_ties_go_to_the_lower_id(cuda_lib, kind):
    tdr = cuda_lib
    T, nr, nc, K = 24, 16, 12, 30
    r = np.random.default_rng(5)
    if kind == "small_integers":
        lg = r.integers(-2, 3, size=(T, nr + nc)).astype(np.float32)
    elif kind == "all_equal":
        lg = np.full((T, nr + nc), 0.5, np.float32)
    elif kind == "one_row_tied":  # columns all equal: the row order alone decides
        lg = np.concatenate([r.standard_normal((T, nr)), np.zeros((T, nc))], 1).astype(np.float32)
    else:
        lg = np.where(r.random((T, nr + nc)) < 0.5, 0.0, -0.0).astype(np.float32)
    c = cfg_of(T, 256, nr, nc, K)
    ids, w, _ = tdr.omni_route(shape_of(tdr, c), logits_in=torch.from_numpy(lg).cuda())
    torch.cuda.synchronize()
    check_route(lg, nr, K, True, ids.cpu().numpy(), w.cpu().numpy())


@pytest.mark.parametrize("T,d,nr,nc", [(300, 256, 32, 32), (130, 1024, 320, 320),
                                       (128, 512, 8, 256), (77, 2048, 200, 136)])
def test_router_gemm(cuda_lib, T, d, nr, nc):
    tdr = cuda_lib
    c = cfg_of(T, d, nr, nc, min(64, nr * nc))
    inp = mi.make_omni_inputs(c, with_experts=False)
    ids, w, lg = tdr.omni_route(shape_of(tdr, c), inp.x.cuda(), inp.w_row.cuda(),
                                inp.w_col.cuda())
    torch.cuda.synchronize()
    assert tdr.device_status() == 0
    ref = orc.cartesian_logits(inp.x, inp.w_row, inp.w_col).astype(np.float64)
    got = lg.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() <= 1e-3 * np.abs(ref).max()
    check_route(got.astype(np.float32), nr, c.K, True, ids.cpu().numpy(), w.cpu().numpy())


# ------------------------------------------------------------------ schedule
def check_schedule(tdr, ids_np, c):
    N = c.n_rows * c.n_cols
    sch = tdr.omni_schedule(shape_of(tdr, c), torch.from_numpy(ids_np).cuda())
    torch.cuda.synchronize()
    assert tdr.device_status() == 0
    counts, offsets, a2p, p2a = orc.task_schedule(ids_np, N)
    np.testing.assert_array_equal(sch["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(sch["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(sch["perm_to_assign"].cpu().numpy(), p2a)
    np.testing.assert_array_equal(sch["assign_to_perm"].cpu().numpy(), a2p)


@pytest.mark.parametrize("T,nr,nc,K", [(1, 8, 8, 3), (257, 16, 16, 50), (1000, 32, 32, 64),
                                       (3000, 64, 40, 100)])
def test_schedule_random_routing(cuda_lib, T, nr, nc, K):
    r = np.random.default_rng(T)
    N = nr * nc
    ids = np.stack([r.permutation(N)[:K] for _ in range(T)]).astype(np.int32)
    check_schedule(cuda_lib, ids, cfg_of(T, 256, nr, nc, K))


@pytest.mark.parametrize("T,K", [(40, 8), (1500, 4), (20000, 2)])
def test_schedule_every_token_on_the_same_experts(cuda_lib, T, K):
    """Degenerate routing: K experts hold T tasks each (warp, shared-memory and
    compaction sorts: 40, 1500 and 20000 slots per expert)."""
    ids = np.tile(np.arange(K, dtype=np.int32)[::-1], (T, 1)).copy()
    check_schedule(cuda_lib, ids, cfg_of(T, 256, 8, 8, K))


def test_schedule_skewed_sizes(cuda_lib):
    """Expert sizes from 0 to ~3000 in one call: every sorting tier at once."""
    r = np.random.default_rng(3)
    T, nr, nc, K = 4000, 16, 16, 8
    N = nr * nc
    p = 1.0 / np.arange(1, N + 1) ** 1.3
    ids = np.stack([r.choice(N, size=K, replace=False, p=p / p.sum()) for _ in range(T)])
    check_schedule(cuda_lib, ids.astype(np.int32), cfg_of(T, 256, nr, nc, K))


# ------------------------------------------------------------------ experts and layer
@pytest.mark.parametrize("T,d,nr,nc,K", [(64, 256, 8, 8, 16), (200, 512, 16, 16, 40),
                                         (50, 768, 8, 8, 64), (37, 1024, 32, 32, 100),
                                         (24, 2048, 8, 16, 33), (16, 4096, 8, 8, 10)])
def test_experts_given_routing(cuda_lib, T, d, nr, nc, K):
    tdr = cuda_lib
    c = cfg_of(T, d, nr, nc, K, seed=d + K)
    inp = mi.make_omni_inputs(c)
    lg = orc.cartesian_logits(inp.x, inp.w_row, inp.w_col)
    ids, w = orc.cartesian_route(lg, nr, K)
    _, offsets, _, p2a = orc.task_schedule(ids, nr * nc)
    out, h = tdr.omni_experts(shape_of(tdr, c), inp.x.cuda(), inp.w_in.cuda(), inp.w_out.cuda(),
                              torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                              torch.from_numpy(offsets).cuda(), torch.from_numpy(p2a).cuda())
    torch.cuda.synchronize()
    assert tdr.device_status() == 0
    h_ref = orc.task_scalars(inp.x, inp.w_in, ids, w)
    h_got = h.cpu().numpy().reshape(T, K).astype(np.float64)
    assert np.abs(h_got - h_ref).max() <= 1e-4 * np.abs(h_ref).max()
    y_ref = orc.token_outputs(inp.x, inp.w_in, inp.w_out, ids, w)
    assert_bf16_close(out.float().cpu().numpy(), y_ref, "out")


@pytest.fixture(params=[0, 1], ids=["gather_out", "scatter_add_out"])
def output_mode(request):
    """Run a forward test with the token-centric gather and with the expert-centric
    scatter-add on the output side (the shape's output_mode)."""
    return request.param


@pytest.mark.parametrize("renorm", [True, False])
def test_forward_small(cuda_lib, renorm, output_mode):
    tdr = cuda_lib
    c = cfg_of(256, 256, 32, 32, 64, renorm)
    inp = mi.make_omni_inputs(c)
    s = shape_of(tdr, c, output_mode)
    out, ws = tdr.omni_forward(s, inp.x.cuda(), inp.w_row.cuda(), inp.w_col.cuda(),
                               inp.w_in.cuda(), inp.w_out.cuda())
    torch.cuda.synchronize()
    assert tdr.device_status() == 0
    v = tdr.omni_workspace_views(s, ws)
    lg = v["logits"].cpu().numpy()
    ref = orc.cartesian_logits(inp.x, inp.w_row, inp.w_col).astype(np.float64)
    assert np.abs(lg - ref).max() <= 1e-3 * np.abs(ref).max()
    ids, w = check_route(lg, c.n_rows, c.K, renorm, v["topk_ids"].cpu().numpy(),
                         v["topk_w"].cpu().numpy())
    counts, offsets, a2p, p2a = orc.task_schedule(ids, c.N)
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    # the forward groups the tasks by expert; the order inside an expert is free
    got = v["perm_to_assign"].cpu().numpy()
    for e in range(c.N):
        lo, hi = offsets[e], offsets[e + 1]
        np.testing.assert_array_equal(np.sort(got[lo:hi]), p2a[lo:hi])
    y_ref = orc.token_outputs(inp.x, inp.w_in, inp.w_out, ids, w)
    assert_bf16_close(out.float().cpu().numpy(), y_ref, "out")
    # the page's expert-centric scatter-add computes the same layer
    y_ec = orc.expert_centric_outputs(inp.x, inp.w_in, inp.w_out, ids, w, c.N)
    assert_bf16_close(out.float().cpu().numpy(), y_ec, "out (expert-centric oracle)")


def test_forward_102k_experts_sampled_tokens(cuda_lib, output_mode):
    """The 4096-token layer with 320 x 320 = 102,400 experts, K = 512, d = 1024: every
    routing output is checked on 12 sampled tokens (brute force over all N pairs), the
    schedule by its invariants and counts, the output on the same tokens."""
    tdr = cuda_lib
    c = mi.OMNI_102K
    inp = mi.make_omni_inputs(c)
    s = shape_of(tdr, c, output_mode)
    out, ws = tdr.omni_forward(s, inp.x.cuda(), inp.w_row.cuda(), inp.w_col.cuda(),
                               inp.w_in.cuda(), inp.w_out.cuda())
    torch.cuda.synchronize()
    assert tdr.device_status() == 0
    v = {k: t.cpu().numpy() for k, t in tdr.omni_workspace_views(s, ws).items()}
    toks = np.random.default_rng(0).choice(c.T, 12, replace=False)
    toks[0], toks[-1] = 0, c.T - 1
    ref_lg = orc.cartesian_logits(inp.x[toks.tolist()], inp.w_row, inp.w_col).astype(np.float64)
    assert np.abs(v["logits"][toks] - ref_lg).max() <= 1e-3 * np.abs(ref_lg).max()
    ids_s, w_s = check_route(v["logits"], c.n_rows, c.K, True, v["topk_ids"], v["topk_w"], toks)
    ids = v["topk_ids"]
    np.testing.assert_array_equal(v["counts"], np.bincount(ids.reshape(-1), minlength=c.N))
    np.testing.assert_array_equal(v["offsets"][1:], np.cumsum(v["counts"]))
    p2a = v["perm_to_assign"]  # grouped by expert, any order inside an expert
    np.testing.assert_array_equal(np.sort(p2a), np.arange(c.A))
    ex = ids.reshape(-1)[p2a]
    assert np.all(np.diff(ex) >= 0)
    y_ref = orc.token_outputs(inp.x, inp.w_in, inp.w_out, ids, v["topk_w"], toks)
    assert_bf16_close(out.float().cpu().numpy()[toks], y_ref, "out")
