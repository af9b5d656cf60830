"""GPU parity: every stage of the CUDA path, called through the C ABI, against the
CPU oracle on the same seeded inputs.

Bars (stated by the workloads): top-k ids, counts, offsets and both permutation maps
bit-exact given identical router logits (the oracle routes on the logits the GPU
produced); top-k weights within 1e-6; layer output max abs error <= 1e-4 for fp32
shapes; for bf16 shapes max|err| / max|ref| <= 2e-2 and ||err|| / ||ref|| <= 2e-2.
Pure data moves (the materialised gather) are bit-exact."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu

BF16_REL = 2e-2
F32_ABS = 1e-4
W_ABS = 1e-6


# ------------------------------------------------------------------ helpers
def cuda(t):
    return None if t is None else t.cuda()


def shape_of(cfg, tdr, T=None, ffn_variant=0):
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    return tdr.make_shape(cfg.T if T is None else T, cfg.d, cfg.E, cfg.K, cfg.n,
                          cfg.capacity_factor, True, dt, ffn_variant=ffn_variant)


def assert_status_ok(tdr):
    assert tdr.device_status() == 0


def rel_errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    scale = max(np.abs(ref).max(), 1e-30)
    l2 = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    return np.abs(diff).max() / scale, l2


def assert_bf16_close(got, ref, what):
    mx, l2 = rel_errors(got, ref)
    assert mx <= BF16_REL and l2 <= BF16_REL, f"{what}: max-rel {mx:.3e} l2-rel {l2:.3e}"


def check_routing(tdr, logits_gpu, ids_gpu, w_gpu, K, renorm=True):
    lg = logits_gpu.cpu().numpy()
    ids_ref, w_ref = orc.route(lg, K, renorm)
    np.testing.assert_array_equal(ids_gpu.cpu().numpy(), ids_ref)
    assert np.abs(w_gpu.cpu().numpy().astype(np.float64) - w_ref).max() <= W_ABS
    return ids_ref, w_ref


def check_permutation(perm, ids, E, C):
    counts, offsets, a2p, p2a = orc.permute(ids, E, C)
    np.testing.assert_array_equal(perm["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(perm["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(perm["assign_to_perm"].cpu().numpy(), a2p)
    nk = int(offsets[-1])
    np.testing.assert_array_equal(perm["perm_to_assign"].cpu().numpy()[:nk], p2a[:nk])
    return counts, offsets, a2p, p2a


_INPUTS = {}


@pytest.fixture(params=[1, 2, 3], ids=["single_cta", "cta_pair", "cta_pair_tma_a"])
def ffn_variant(request):
    """Run a test with the single-CTA grouped GEMM, the CTA-pair one gathering its rows, and
    the CTA-pair one reading rows copied expert-major beforehand (the shape's ffn_variant)."""
    return request.param


@pytest.fixture(params=[1, 2], ids=["topk_rounds", "topk_bitonic"])
def route_topk(request):
    """Run a warp-per-token routing test with K rounds of a warp arg-max and with the bitonic
    merges (the shape's route_topk; the bitonic form applies for E <= 64 and K <= 8)."""
    return request.param


def inputs_for(cfg):
    if cfg.name not in _INPUTS:
        _INPUTS.clear()  # keep one large workload in host memory at a time
        _INPUTS[cfg.name] = mi.make_inputs(cfg)
    return _INPUTS[cfg.name]


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_times_out_and_reports(cuda_lib):
    tdr = cuda_lib
    assert tdr.device_status() == 0
    assert tdr.selftest_timeout(2_000_000) == 5  # 2 ms limit, nothing completes the barrier
    assert tdr.device_status() == 0  # cleared by the read
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0  # the context is still usable


# ------------------------------------------------------------------ route
@pytest.mark.parametrize("T,d,E,K,dtype,bias,renorm", [
    (256, 128, 8, 2, "f32", False, True),      # the tiny workload's router
    (300, 4096, 8, 2, "bf16", False, True),
    (257, 2048, 128, 8, "bf16", False, True),
    (500, 2880, 32, 4, "bf16", True, True),
    (100, 128, 256, 32, "bf16", False, True),
    (33, 64, 6, 3, "f32", False, False),
    (1, 64, 1, 1, "bf16", False, True),
    (129, 192, 64, 6, "bf16", True, False),
    # bf16 with few experts: ragged tiles, E below 8, K up to E, long d
    (301, 2880, 8, 3, "bf16", True, False),
    (5, 2048, 4, 4, "bf16", True, True),
    (1027, 256, 7, 2, "bf16", False, False),
    (9001, 4096, 8, 8, "bf16", True, True),
    (70, 4160, 8, 2, "bf16", False, True),
    # per tile: 16, 21, 32 and 128 rows when one tile per SM runs over the whole of d
    (2300, 1024, 16, 4, "bf16", True, True),
    (3000, 512, 256, 8, "bf16", False, True),
    (4736, 2048, 32, 4, "bf16", False, True),
    (18900, 256, 64, 6, "bf16", True, False),
    (18945, 128, 8, 2, "bf16", False, True),   # 129 rows per SM: split form again
])
def test_route_matches_oracle(cuda_lib, T, d, E, K, dtype, bias, renorm):
    tdr = cuda_lib
    cfg = mi.MoEConfig("route", T=T, d=d, E=E, K=K, n=64, dtype=dtype, seed=T + E)
    inp = mi.make_inputs(cfg, with_experts=False)
    b = mi.zipf_bias(E, 1.2, 1.75) if bias else None
    s = tdr.make_shape(T, d, E, K, 64, 0.0, renorm,
                       torch.bfloat16 if dtype == "bf16" else torch.float32)
    lo = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ids, w, _ = tdr.route(s, cuda(inp.x), cuda(inp.w_r), bias=cuda(b), logits_out=lo)
    ref_lg = orc.router_logits(inp.x, inp.w_r, None if b is None else b.numpy())
    if dtype == "f32":  # fp32 inputs, fp32 accumulation: relative 1e-5 of the logit scale
        assert np.abs(lo.cpu().numpy() - ref_lg).max() <= 1e-5 * np.abs(ref_lg).max()
    else:  # bf16 inputs (exact products), fp32 accumulation on the tensor cores
        np.testing.assert_allclose(lo.cpu().numpy(), ref_lg, rtol=1e-4, atol=2e-4)
    check_routing(tdr, lo, ids, w, K, renorm)
    assert_status_ok(tdr)


@pytest.mark.parametrize("E,K", [(64, 6), (40, 8), (32, 2), (128, 4)])
def test_route_ties_go_to_lower_id(cuda_lib, route_topk, E, K):
    tdr = cuda_lib
    g = np.random.default_rng(5)
    T = 777
    lg = g.integers(-2, 3, size=(T, E)).astype(np.float32)  # heavy ties
    lg[0] = 0.0
    lg[1, ::2] = -0.0  # signed zeros tie with +0
    s = tdr.make_shape(T, 64, E, K, 64, 0.0, True, torch.bfloat16, route_topk=route_topk)
    ids, w, lo = tdr.route(s, logits_in=torch.from_numpy(lg).cuda(),
                           logits_out=torch.empty(T, E, device="cuda"))
    np.testing.assert_array_equal(lo.cpu().numpy(), lg)
    ids_ref, _ = check_routing(tdr, lo, ids, w, K)
    np.testing.assert_array_equal(ids_ref[0], np.arange(K))
    assert_status_ok(tdr)


@pytest.mark.parametrize("d", [1024, 4096])
def test_route_identical_router_columns_tie_exactly(cuda_lib, d):
    """Experts with identical router columns get bit-identical logits from x, so their
    order is decided by the id alone."""
    tdr = cuda_lib
    T, E, K = 203, 8, 4
    cfg = mi.MoEConfig("ties", T=T, d=d, E=E, K=K, n=64, dtype="bf16", seed=11)
    inp = mi.make_inputs(cfg, with_experts=False)
    w_r = inp.w_r.clone()
    for e in (1, 3, 6):
        w_r[:, e] = w_r[:, 5]
    s = tdr.make_shape(T, d, E, K, 64, 0.0, True, torch.bfloat16)
    lo = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ids, w, _ = tdr.route(s, cuda(inp.x), cuda(w_r), logits_out=lo)
    lg = lo.cpu().numpy()
    for e in (1, 3, 6):
        np.testing.assert_array_equal(lg[:, e], lg[:, 5])
    ids_ref, _ = check_routing(tdr, lo, ids, w, K)
    got = ids.cpu().numpy()
    for t in range(T):  # a tied group appears in ascending id order
        tied = [e for e in got[t] if e in (1, 3, 5, 6)]
        assert tied == sorted(tied)
    assert_status_ok(tdr)


@pytest.mark.parametrize("T", mi.DISPATCH_COMBINE_T)
def test_route_given_logits_sweep(cuda_lib, route_topk, T):
    tdr = cuda_lib
    cfg = mi.DISPATCH_COMBINE.with_T(T)
    inp = mi.make_inputs(cfg)
    s = tdr.make_shape(T, cfg.d, cfg.E, cfg.K, cfg.n, cfg.capacity_factor, True,
                       torch.bfloat16, route_topk=route_topk)
    ids, w, _ = tdr.route(s, logits_in=cuda(inp.logits))
    check_routing(tdr, inp.logits, ids, w, cfg.K)
    assert_status_ok(tdr)


# ------------------------------------------------------------------ permute
def _random_ids(rng, T, E, K, skew=0.0):
    if T == 0:
        return np.zeros((0, K), np.int32)
    scores = rng.standard_normal((T, E)) + skew * (np.arange(E)[None, :] == 0)
    return np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int32)


@pytest.mark.parametrize("T,E,K,cf,skew", [
    (1, 1, 1, 0.0, 0.0),
    (37, 8, 2, 0.0, 0.0),
    (4095, 8, 2, 0.0, 0.0),
    (5000, 64, 6, 0.0, 0.0),
    (16384, 128, 8, 0.0, 0.0),
    (8192, 32, 4, 1.25, 3.0),
    (3001, 256, 32, 0.5, 0.0),
    (700, 16, 4, 0.3, 5.0),
    (65536, 64, 6, 0.0, 0.0),
    # around the one-launch cluster path's bounds (2048 < T*K <= 32768 assignments)
    (1025, 8, 2, 0.0, 0.0),
    (4097, 8, 2, 1.0, 2.0),
    (4097, 8, 8, 0.0, 0.0),
])
def test_permute_matches_oracle(cuda_lib, T, E, K, cf, skew):
    tdr = cuda_lib
    rng = np.random.default_rng(T * 31 + E)
    ids = _random_ids(rng, T, E, K, skew)
    s = tdr.make_shape(T, 64, E, K, 64, cf, True, torch.bfloat16)
    perm = tdr.permute(s, torch.from_numpy(ids).cuda())
    check_permutation(perm, ids, E, orc.capacity(cf, T, K, E))
    assert_status_ok(tdr)


def test_permute_materialised_gather_is_exact(cuda_lib):
    tdr = cuda_lib
    rng = np.random.default_rng(9)
    T, E, K, d = 1234, 16, 3, 256
    ids = _random_ids(rng, T, E, K, 1.0)
    x = torch.randn(T, d).to(torch.bfloat16)
    s = tdr.make_shape(T, d, E, K, 64, 0.9, True, torch.bfloat16)
    perm = tdr.permute(s, torch.from_numpy(ids).cuda(), x=x.cuda(), materialize=True)
    _, offsets, _, p2a = check_permutation(perm, ids, E, orc.capacity(0.9, T, K, E))
    nk = int(offsets[-1])
    ref = orc.gather_rows(x.float().numpy(), p2a, offsets, K)
    np.testing.assert_array_equal(perm["x_perm"][:nk].float().cpu().numpy(), ref)
    assert_status_ok(tdr)


def test_permute_flags_out_of_range_ids(cuda_lib):
    tdr = cuda_lib
    T, E, K = 100, 8, 2
    ids = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    ids[7, 1] = E  # out of range: skipped and reported, never used as an index
    s = tdr.make_shape(T, 64, E, K, 64, 0.0, True, torch.bfloat16)
    perm = tdr.permute(s, torch.from_numpy(ids).cuda())
    assert tdr.device_status() == 6
    a2p = perm["assign_to_perm"].cpu().numpy()
    assert a2p[7 * K + 1] == -1
    assert int(perm["counts"].cpu().sum()) == T * K - 1


# ------------------------------------------------------------------ dispatch (route + permute)
@pytest.mark.parametrize("T,E,K,cf,renorm,ties", [
    (64, 64, 6, 0.0, True, False),      # the dispatch workload's decode-regime sizes
    (256, 64, 6, 0.0, True, False),
    (1024, 64, 6, 0.0, True, False),
    (1, 1, 1, 0.0, True, False),
    (33, 8, 2, 1.0, False, False),
    (128, 200, 16, 1.25, True, False),  # capacity drops
    (100, 256, 11, 0.3, False, True),
    (64, 256, 32, 0.0, True, True),     # E = 256, K = 32, integer logits (ties)
    (128, 256, 32, 0.0, True, True),
    (800, 37, 5, 0.5, False, True),
    (1365, 64, 6, 1.25, True, False),   # the cluster permutation
    (7000, 64, 6, 0.0, True, False),    # the chunked permutation, four tokens a router warp
])
def test_dispatch_matches_oracle_and_the_two_calls(cuda_lib, route_topk, T, E, K, cf, renorm,
                                                   ties):
    tdr = cuda_lib
    rng = np.random.default_rng(T * 7 + E)
    if ties:
        lg = rng.integers(-3, 4, size=(T, E)).astype(np.float32)
        lg[0, ::2] = -0.0
    else:
        lg = rng.standard_normal((T, E)).astype(np.float32)
    s = tdr.make_shape(T, 64, E, K, 64, cf, renorm, torch.bfloat16, route_topk=route_topk)
    lgd = torch.from_numpy(lg).cuda()
    lo = torch.empty(T, E, device="cuda")
    out = tdr.dispatch(s, logits_in=lgd, logits_out=lo)
    np.testing.assert_array_equal(lo.cpu().numpy(), lg)
    ids_ref, w_ref = orc.route(lg, K, renorm)
    np.testing.assert_array_equal(out["topk_ids"].cpu().numpy(), ids_ref)
    assert np.abs(out["topk_w"].cpu().numpy().astype(np.float64) - w_ref).max() <= W_ABS
    _, offsets, _, _ = check_permutation(out, ids_ref, E, orc.capacity(cf, T, K, E))
    ids2, w2, _ = tdr.route(s, logits_in=lgd)
    p2 = tdr.permute(s, ids2)
    assert torch.equal(out["topk_ids"], ids2) and torch.equal(out["topk_w"], w2)
    nk = int(offsets[-1])
    for k in ("counts", "offsets", "assign_to_perm"):
        assert torch.equal(out[k], p2[k])
    assert torch.equal(out["perm_to_assign"][:nk], p2["perm_to_assign"][:nk])
    assert_status_ok(tdr)


@pytest.mark.parametrize("T,E,K,cf,mat", [
    (100, 8, 2, 0.0, False), (1000, 8, 2, 0.0, True), (4096, 8, 2, 0.0, True),
    (4097, 8, 2, 0.9, True), (3000, 64, 6, 0.0, False), (2000, 256, 8, 1.1, True),
    (8192, 16, 4, 0.0, False), (40000, 8, 2, 0.0, False)])
def test_dispatch_from_x_matches_oracle(cuda_lib, T, E, K, cf, mat):
    """moe_dispatch from x and W_r (tensor-core router, then the permutation): equal to the
    oracle on the router's own logits, with and without capacity drops, with the rows
    gathered exactly."""
    tdr = cuda_lib
    d = 256
    cfg = mi.MoEConfig("dispatch_x", T=T, d=d, E=E, K=K, n=0, dtype="bf16", seed=T + E)
    inp = mi.make_inputs(cfg, with_experts=False)
    s = tdr.make_shape(T, d, E, K, 0, cf, True, torch.bfloat16)
    x = inp.x.cuda()
    out = tdr.dispatch(s, x=x, w_r=inp.w_r.cuda(), logits_out=torch.empty(T, E, device="cuda"),
                       materialize=mat)
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    lg = out["logits_out"].cpu().numpy() if "logits_out" in out else None
    assert lg is not None
    ids_ref, w_ref = orc.route(lg, K, True)
    np.testing.assert_array_equal(out["topk_ids"].cpu().numpy(), ids_ref)
    assert np.abs(out["topk_w"].cpu().numpy() - w_ref).max() <= W_ABS
    C = orc.capacity(cf, T, K, E)
    _, offsets, _, p2a = check_permutation(out, ids_ref, E, C)
    if mat:
        nk = int(offsets[-1])
        xp = out["x_perm"][:nk].cpu()
        np.testing.assert_array_equal(xp.view(torch.int16).numpy(),
                                      inp.x[torch.from_numpy(p2a[:nk] // K)].view(torch.int16).numpy())


@pytest.mark.parametrize("T,E,K,d,cf", [
    (300, 16, 3, 256, 0.9),     # rows copied by the one-launch kernel (small gather)
    (64, 64, 6, 4096, 0.0),     # the dispatch workload at T = 64: 3 MB, still in one launch
    (7, 64, 6, 4096, 0.5),      # fewer tokens than CTAs; capacity drops
    (256, 64, 6, 4096, 0.0),    # 12.6 MB: the separate gather kernel
    (500, 8, 2, 320, 1.0),      # ragged row (40 vectors)
])
def test_dispatch_materialised_gather_is_exact(cuda_lib, route_topk, T, E, K, d, cf):
    tdr = cuda_lib
    rng = np.random.default_rng(17 + T)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    x = torch.randn(T, d).to(torch.bfloat16)
    s = tdr.make_shape(T, d, E, K, 64, cf, True, torch.bfloat16, route_topk=route_topk)
    out = tdr.dispatch(s, x=x.cuda(), logits_in=torch.from_numpy(lg).cuda(), materialize=True)
    ids_ref, _ = orc.route(lg, K, True)
    _, offsets, _, p2a = check_permutation(out, ids_ref, E, orc.capacity(cf, T, K, E))
    nk = int(offsets[-1])
    ref = orc.gather_rows(x.float().numpy(), p2a, offsets, K)
    np.testing.assert_array_equal(out["x_perm"][:nk].float().cpu().numpy(), ref)
    assert_status_ok(tdr)


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_combine_matches_oracle(cuda_lib, dtype):
    tdr = cuda_lib
    rng = np.random.default_rng(21)
    T, E, K, d = 999, 16, 4, 192
    ids = _random_ids(rng, T, E, K, 2.0)
    C = orc.capacity(0.8, T, K, E)
    _, offsets, a2p, _ = orc.permute(ids, E, C)
    w = rng.random((T, K)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    y = torch.randn(T * K, d).to(tdt)
    s = tdr.make_shape(T, d, E, K, 64, 0.8, True, tdt)
    out = tdr.combine(s, y.cuda(), torch.from_numpy(a2p).cuda(), torch.from_numpy(w).cuda())
    ref = orc.combine(y.float().numpy(), a2p, w, T, K)
    got = out.float().cpu().numpy()
    if dtype == "f32":
        np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-5)
    else:  # fp32 sum rounded once to bf16: within half a bf16 ulp plus fp32 rounding
        np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-6)
    assert_status_ok(tdr)


# ------------------------------------------------------------------ grouped FFN
def _ffn_case(tdr, T, d, n, E, K, cf, dtype, seed, ffn_variant=0):
    cfg = mi.MoEConfig("ffn", T=T, d=d, E=E, K=K, n=n, dtype=dtype, capacity_factor=cf,
                       seed=seed)
    inp = mi.make_inputs(cfg)
    s = shape_of(cfg, tdr, ffn_variant=ffn_variant)
    lo = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ids, w, _ = tdr.route(s, cuda(inp.x), cuda(inp.w_r), logits_out=lo)
    perm = tdr.permute(s, ids)
    a_act, y_perm = tdr.grouped_ffn(s, cuda(inp.x), perm["offsets"], perm["perm_to_assign"],
                                    cuda(inp.w_gate), cuda(inp.w_up), cuda(inp.w_down))
    out = tdr.combine(s, y_perm, perm["assign_to_perm"], w)
    ids_ref, w_ref = check_routing(tdr, lo, ids, w, K)
    _, offsets, a2p, p2a = check_permutation(perm, ids_ref, E, orc.capacity(cf, T, K, E))
    a_ref, y_ref = orc.grouped_ffn(inp.x, p2a, offsets, K, inp.w_gate, inp.w_up, inp.w_down)
    out_ref = orc.combine(y_ref, a2p, w_ref, T, K)
    nk = int(offsets[-1])
    return (a_act[:nk].float().cpu().numpy(), a_ref, y_perm[:nk].float().cpu().numpy(), y_ref,
            out.float().cpu().numpy(), out_ref)


def test_grouped_ffn_fp32_tiny_workload(cuda_lib):
    tdr = cuda_lib
    c = mi.TINY_FP32
    a, a_ref, y, y_ref, out, out_ref = _ffn_case(tdr, c.T, c.d, c.n, c.E, c.K, 0.0, "f32", 0)
    assert np.abs(a - a_ref).max() <= 1e-5
    assert np.abs(y - y_ref).max() <= F32_ABS
    assert np.abs(out - out_ref).max() <= F32_ABS
    assert_status_ok(tdr)


@pytest.mark.parametrize("T,d,n,E,K,cf", [
    (300, 256, 384, 4, 2, 0.0),     # gate/up tail tile of 128 columns (n = 3 x 128)
    (1000, 512, 192, 16, 4, 1.1),   # n = 192: last gate/up tile half valid; capacity drops
    (64, 128, 128, 8, 8, 0.0),      # K = E; down tile wider than d
    (2500, 320, 256, 3, 1, 0.0),    # d = 320: down tile 256 + ragged 64
    (129, 64, 64, 1, 1, 0.0),       # one expert; one k-block; 2 M-tiles, the last has 1 row
])
def test_grouped_ffn_bf16_tensor_cores(cuda_lib, ffn_variant, T, d, n, E, K, cf):
    tdr = cuda_lib
    a, a_ref, y, y_ref, out, out_ref = _ffn_case(tdr, T, d, n, E, K, cf, "bf16", T + d,
                                                 ffn_variant)
    assert_bf16_close(a, a_ref, "a_act")
    assert_bf16_close(y, y_ref, "y_perm")
    assert_bf16_close(out, out_ref, "out")
    assert_status_ok(tdr)


# ------------------------------------------------------------------ whole layer
def test_forward_tiny_fp32(cuda_lib):
    tdr = cuda_lib
    cfg = mi.TINY_FP32
    inp = mi.make_inputs(cfg)
    s = shape_of(cfg, tdr)
    out, ws = tdr.forward(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                          cuda(inp.w_down))
    v = tdr.workspace_views(s, ws)
    ref = orc.forward(inp.x.numpy(), inp.w_r.numpy(), inp.w_gate.numpy(), inp.w_up.numpy(),
                      inp.w_down.numpy(), cfg.K, logits=v["logits"].cpu().numpy())
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["topk_ids"])
    assert np.abs(out.cpu().numpy() - ref["out"]).max() <= F32_ABS
    dense = orc.dense_reference(inp.x.numpy(), inp.w_gate.numpy(), inp.w_up.numpy(),
                                inp.w_down.numpy(), ref["topk_ids"], ref["topk_w"], cfg.E)
    assert np.abs(out.cpu().numpy() - dense).max() <= F32_ABS
    assert_status_ok(tdr)


def _boundary_slots(offsets, rng):
    """Expert-major slots where the grouped GEMMs' masked-row paths run: for every expert
    its first and last slot, and the first and a random slot of its last 128-row tile
    (single-CTA tiles) and of its last 256-row tile (CTA-pair tiles)."""
    off = np.asarray(offsets, dtype=np.int64)
    slots = set()
    for e in range(off.size - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        slots.update((lo, hi - 1))
        for tile in (128, 256):
            start = lo + ((hi - lo - 1) // tile) * tile
            slots.update((start, int(rng.integers(start, hi))))
    return np.array(sorted(slots), dtype=np.int64)


def _capacity_edge_tokens(ids, K, E, C):
    """For every expert routed more than C assignments: the token of its last kept
    assignment and of its first dropped one (assignments kept in token order)."""
    flat = np.asarray(ids).reshape(-1)
    toks = set()
    for e in range(E):
        a = np.flatnonzero(flat == e)
        if C is not None and a.size > C:
            toks.update((int(a[C - 1]) // K, int(a[C]) // K))
    return toks


def assert_rows_close(got, ref, what):
    """Per-row bound: max|err| <= 2e-2 max|ref| in every row (a zero row must be zero),
    beside the global bounds."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    for r in range(ref.shape[0]):
        scale = np.abs(ref[r]).max()
        err = np.abs(got[r] - ref[r]).max()
        if scale == 0:
            assert err == 0, f"{what}: row {r} should be zero"
        else:
            assert err <= BF16_REL * scale, f"{what}: row {r} max-rel {err / scale:.3e}"
    assert_bf16_close(got, ref, what)


@pytest.mark.parametrize("name", ["mixtral_bf16", "fine_grained_bf16", "skewed_capacity_bf16"])
def test_forward_full_size_workloads(cuda_lib, ffn_variant, name):
    """The whole layer at the full workload sizes: routing and permutation bit-exact on every
    token; a_act and y_perm element by element on the slots of every expert's last partial
    128- and 256-row tile (where masked rows are handled) plus its first and last slot; the
    output of 16 random tokens, of the tokens of those slots and, with a capacity limit, of
    the last kept and first dropped token of every overfull expert, each row within the bf16
    bar."""
    tdr = cuda_lib
    cfg = mi.CONFIGS[name]
    inp = inputs_for(cfg)
    s = shape_of(cfg, tdr, ffn_variant=ffn_variant)
    out, ws = tdr.forward(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                          cuda(inp.w_down), bias=cuda(inp.bias))
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    v = tdr.workspace_views(s, ws)
    lg = v["logits"].cpu().numpy()
    rng = np.random.default_rng(7)
    sample = np.sort(rng.choice(cfg.T, size=64, replace=False))
    ref_lg = orc.router_logits(inp.x[sample], inp.w_r,
                               None if inp.bias is None else inp.bias.numpy())
    np.testing.assert_allclose(lg[sample], ref_lg, rtol=1e-4, atol=2e-4)
    ids_ref, w_ref = check_routing(tdr, v["logits"], v["topk_ids"], v["topk_w"], cfg.K)
    C = orc.capacity(cfg.capacity_factor, cfg.T, cfg.K, cfg.E)
    _, offsets, a2p, p2a = check_permutation(v, ids_ref, cfg.E, C)
    if C is not None:
        assert (a2p < 0).any()  # the skewed workload really drops
    # a_act and y_perm on the tile-boundary slots
    slots = _boundary_slots(offsets, rng)
    a_ref, y_ref = orc.grouped_ffn_rows(slots, inp.x, p2a, offsets, cfg.K, inp.w_gate,
                                        inp.w_up, inp.w_down)
    sl = torch.from_numpy(slots).cuda()
    assert_rows_close(v["a_act"][sl].float().cpu().numpy(), a_ref, f"{name} a_act")
    assert_rows_close(v["y_perm"][sl].float().cpu().numpy(), y_ref, f"{name} y_perm")
    # outputs: random tokens, the tokens of the boundary slots, the capacity edges
    toks = set(sample[:16].tolist())
    toks.update(int(t) for t in rng.choice(np.asarray(p2a)[slots] // cfg.K,
                                           size=min(32, slots.size), replace=False))
    edge = _capacity_edge_tokens(ids_ref, cfg.K, cfg.E, C)
    toks.update(edge)
    tokens = np.array(sorted(toks), dtype=np.int64)
    ref_rows = orc.forward_rows(tokens, inp.x, inp.w_gate, inp.w_up, inp.w_down, ids_ref, w_ref,
                                a2p, cfg.K)
    assert_rows_close(out[torch.from_numpy(tokens).cuda()].float().cpu().numpy(), ref_rows,
                      f"{name} out")
    if C is not None:
        assert len(edge) > 0


# ------------------------------------------------------------------ token rounding
def _rounded_reference(lg, ids_ref, E, R):
    keep = orc.tile_round_keep(ids_ref, lg, E, R)
    return keep, orc.permute(ids_ref, E, None, keep)


@pytest.mark.parametrize("T,E,K,R,ties", [
    (1000, 8, 2, 64, False),
    (4096, 8, 2, 128, False),      # the Mixtral-like routing shape
    (3001, 32, 4, 128, True),      # integer logits: equal scores split by token order
    (300, 4, 1, 128, False),       # experts below R keep everything
    (16384, 128, 8, 128, False),   # three-kernel permutation
    (500, 16, 3, 1, False),        # R = 1 changes nothing
])
def test_dispatch_token_rounding_matches_oracle(cuda_lib, T, E, K, R, ties):
    tdr = cuda_lib
    rng = np.random.default_rng(T + E + R)
    if ties:
        lg = rng.integers(-3, 4, size=(T, E)).astype(np.float32)
    else:
        lg = rng.standard_normal((T, E)).astype(np.float32)
    s = tdr.make_shape(T, 64, E, K, 64, 0.0, True, torch.bfloat16, tile_round=R)
    out = tdr.dispatch(s, logits_in=torch.from_numpy(lg).cuda())
    ids_ref, w_ref = orc.route(lg, K, True)
    np.testing.assert_array_equal(out["topk_ids"].cpu().numpy(), ids_ref)
    keep, (counts, offsets, a2p, p2a) = _rounded_reference(lg, ids_ref, E, R)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(out["assign_to_perm"].cpu().numpy(), a2p)
    nk = int(offsets[-1])
    np.testing.assert_array_equal(out["perm_to_assign"].cpu().numpy()[:nk], p2a[:nk])
    kept = np.diff(offsets)
    assert all(k % R == 0 or c < R for k, c in zip(kept, counts))
    if R > 1 and T >= 1000:
        assert (~keep).any()  # the case really rounds
    assert_status_ok(tdr)


def test_forward_token_rounding_full_size(cuda_lib):
    tdr = cuda_lib
    cfg = mi.CONFIGS["mixtral_bf16"]
    inp = inputs_for(cfg)
    s = tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, 0.0, True, torch.bfloat16,
                       tile_round=128)
    out, ws = tdr.forward(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                          cuda(inp.w_down))
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    v = tdr.workspace_views(s, ws)
    lg = v["logits"].cpu().numpy()
    ids_ref, w_ref = check_routing(tdr, v["logits"], v["topk_ids"], v["topk_w"], cfg.K)
    keep, (counts, offsets, a2p, p2a) = _rounded_reference(lg, ids_ref, cfg.E, 128)
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(v["assign_to_perm"].cpu().numpy(), a2p)
    assert np.all(np.diff(offsets) % 128 == 0) and (~keep).any()
    rng = np.random.default_rng(11)
    dropped_tok = np.nonzero((~keep).any(1))[0]
    tokens = np.unique(np.concatenate([rng.choice(cfg.T, size=12, replace=False),
                                       dropped_tok[:4]]))
    ref_rows = orc.forward_rows(tokens, inp.x, inp.w_gate, inp.w_up, inp.w_down, ids_ref, w_ref,
                                a2p, cfg.K)
    assert_bf16_close(out[torch.from_numpy(tokens).cuda()].float().cpu().numpy(), ref_rows,
                      "rounded forward out")


def test_token_rounding_rejected_where_it_cannot_apply(cuda_lib):
    tdr = cuda_lib
    s = tdr.make_shape(64, 64, 8, 2, 64, 0.0, True, torch.bfloat16, tile_round=16)
    ids = torch.zeros(64, 2, dtype=torch.int32, device="cuda")
    with pytest.raises(tdr.MoEError):
        tdr.permute(s, ids)  # no logits: unsupported
    bad = tdr.make_shape(64, 64, 8, 2, 64, 1.0, True, torch.bfloat16, tile_round=16)
    with pytest.raises(tdr.MoEError):
        tdr.dispatch(bad, logits_in=torch.zeros(64, 8, device="cuda"))


# ------------------------------------------------------------------ token rounding up / nearest
def _check_rounded_up(tdr, s, v, ref, R, T, E, K, f32):
    """Every intermediate of a forward that rounds up or to the nearest tile against the
    oracle's: the discrete ones exactly, the weights within W_ABS, the rows within the
    dtype's bar. Returns the number of added assignments."""
    ids_ref = ref["topk_ids"]
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ids_ref)
    np.testing.assert_array_equal(v["counts"].cpu().numpy(), ref["counts"])
    NA = E * (R - 1)
    n_add = ref["add_tok"].size
    assert n_add <= NA
    keep = (ref["assign_to_perm"][:T * K] >= 0).reshape(T, K)
    ids_ext = np.full(T * K + NA, -1, np.int64)
    ids_ext[:T * K] = np.where(keep, ids_ref, -1).reshape(-1)
    ids_ext[T * K:T * K + n_add] = ref["add_exp"]
    np.testing.assert_array_equal(v["round_ids"].cpu().numpy(), ids_ext)
    add_tok = v["add_tok"].cpu().numpy()
    np.testing.assert_array_equal(add_tok[:n_add], ref["add_tok"])
    assert np.all(add_tok[n_add:] == -1)
    offsets = ref["offsets"]
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    a2p_ref = np.full(T * K + NA, -1, np.int64)
    a2p_ref[:ref["assign_to_perm"].size] = ref["assign_to_perm"]
    np.testing.assert_array_equal(v["assign_to_perm"].cpu().numpy(), a2p_ref)
    nk = int(offsets[-1])
    np.testing.assert_array_equal(v["perm_to_assign"].cpu().numpy()[:nk],
                                  ref["perm_to_assign"][:nk])
    np.testing.assert_array_equal(v["slot_token"].cpu().numpy()[:nk], ref["slot_tokens"])
    assert np.abs(v["topk_w"].cpu().numpy().astype(np.float64) - ref["topk_w"]).max() <= W_ABS
    if n_add:
        got_aw = v["add_w"].cpu().numpy()[:n_add].astype(np.float64)
        assert np.abs(got_aw - ref["add_w"]).max() <= W_ABS
    # the token-major lists: each token's added entries, ascending
    ptr = v["add_ptr"].cpu().numpy()
    idx = v["add_idx"].cpu().numpy()
    assert ptr[0] == 0 and ptr[-1] == n_add
    for t in np.unique(ref["add_tok"])[:64]:
        np.testing.assert_array_equal(idx[ptr[t]:ptr[t + 1]],
                                      np.nonzero(ref["add_tok"] == t)[0])
    return n_add


@pytest.mark.parametrize("T,d,n,E,K,R,mode,dtype,renorm,ties", [
    (1000, 128, 128, 8, 2, 64, "up", "bf16", True, False),
    (1000, 128, 128, 8, 2, 64, "nearest", "bf16", True, False),
    (3001, 64, 64, 32, 4, 128, "up", "bf16", True, True),     # integer logits: ties
    (300, 64, 64, 4, 1, 128, "up", "bf16", False, False),     # c < R: every expert gains
    (200, 64, 128, 8, 2, 256, "up", "bf16", True, False),     # R > T: every token everywhere
    (500, 64, 64, 16, 3, 16, "nearest", "f32", True, False),  # the fp32 grouped FFN
    (16384, 64, 64, 128, 8, 128, "nearest", "bf16", True, False),  # chunked permutation
    (129, 64, 64, 3, 1, 1, "up", "bf16", True, False),        # R = 1 changes nothing
    (1, 64, 64, 8, 2, 16, "up", "bf16", True, False),         # one token: nothing to add
    (700, 64, 64, 8, 8, 64, "nearest", "bf16", True, False),  # K = E: every token everywhere
    (900, 64, 128, 16, 4, 32, "nearest", "bf16", False, True),  # plain softmax, ties
])
def test_forward_token_rounding_up_matches_oracle(cuda_lib, T, d, n, E, K, R, mode, dtype,
                                                  renorm, ties):
    tdr = cuda_lib
    cfg = mi.MoEConfig("round_up", T=T, d=d, E=E, K=K, n=n, dtype=dtype, seed=T + R)
    inp = mi.make_inputs(cfg)
    rng = np.random.default_rng(T + E + R)
    if ties:
        lg = rng.integers(-3, 4, size=(T, E)).astype(np.float32)
    else:
        lg = rng.standard_normal((T, E)).astype(np.float32)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    m = {"up": 1, "nearest": 2}[mode]
    s = tdr.make_shape(T, d, E, K, n, 0.0, renorm, dt, tile_round=R, tile_round_mode=m)
    out, ws = tdr.forward(s, cuda(inp.x), None, cuda(inp.w_gate), cuda(inp.w_up),
                          cuda(inp.w_down), logits_in=torch.from_numpy(lg).cuda())
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    v = tdr.workspace_views(s, ws)
    ref = orc.forward(inp.x, None, inp.w_gate, inp.w_up, inp.w_down, K, logits=lg,
                      renormalize=renorm, tile_round=R, round_mode=mode)
    if R == 1:  # nothing to round: the plain forward, its workspace without added entries
        plain = orc.forward(inp.x, None, inp.w_gate, inp.w_up, inp.w_down, K, logits=lg,
                            renormalize=renorm)
        assert ref["add_tok"].size == 0 and "add_tok" not in v
        np.testing.assert_array_equal(v["offsets"].cpu().numpy(), plain["offsets"])
        np.testing.assert_array_equal(v["assign_to_perm"].cpu().numpy(),
                                      plain["assign_to_perm"])
        assert_bf16_close(out.float().cpu().numpy(), ref["out"], "out")
        return
    n_add = _check_rounded_up(tdr, s, v, ref, R, T, E, K, dtype == "f32")
    nk = int(ref["offsets"][-1])
    got = [v["a_act"][:nk].float().cpu().numpy(), v["y_perm"][:nk].float().cpu().numpy(),
           out.float().cpu().numpy()]
    for g, r, what in zip(got, (ref["a_act"], ref["y_perm"], ref["out"]),
                          ("a_act", "y_perm", "out")):
        if dtype == "f32":
            assert np.abs(g - r).max() <= F32_ABS, what
        else:
            assert_bf16_close(g, r, what)
    kept = np.diff(ref["offsets"])
    if R > 1 and mode == "up" and T >= R:
        assert n_add > 0
        assert all(k % R == 0 or k == T for k in kept)
    if R > T and mode == "up":  # every expert with a routed token holds every token
        assert np.all((kept == T) | (kept == 0))


def _added_rows(tokens, x, w_gate, w_up, w_down, add_tok, add_exp, add_w):
    """The added assignments' share of out[t] for the chosen tokens, in expert order."""
    tokens = np.asarray(tokens, np.int64)
    extra = np.zeros((tokens.size, w_down.shape[2]), np.float64)
    for i, t in enumerate(tokens):
        for j in np.nonzero(add_tok == t)[0]:
            e = int(add_exp[j])
            extra[i] += float(add_w[j]) * orc.expert_ffn(orc.as_f64(x[t:t + 1]), w_gate[e],
                                                         w_up[e], w_down[e])[0]
    return extra


@pytest.mark.parametrize("mode", [1, 2], ids=["up", "nearest"])
def test_forward_token_rounding_up_full_size(cuda_lib, mode):
    """The Mixtral-like workload rounded up or to the nearest 128-row tile, routed from x:
    the discrete intermediates in full, the layer output on sampled tokens (a token that
    gained an expert among them)."""
    tdr = cuda_lib
    cfg = mi.CONFIGS["mixtral_bf16"]
    inp = inputs_for(cfg)
    R = 128
    s = tdr.make_shape(cfg.T, cfg.d, cfg.E, cfg.K, cfg.n, 0.0, True, torch.bfloat16,
                       tile_round=R, tile_round_mode=mode)
    out, ws = tdr.forward(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                          cuda(inp.w_down))
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    v = tdr.workspace_views(s, ws)
    lg = v["logits"].cpu().numpy()
    ids_ref, _ = orc.route(lg, cfg.K, True)
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ids_ref)
    keep, add_tok, add_exp = orc.tile_round_select(ids_ref, lg, cfg.E, R,
                                                   {1: "up", 2: "nearest"}[mode])
    ids_ext = np.concatenate([np.where(keep, ids_ref, -1).reshape(-1), add_exp])
    offsets, a2p, p2a = orc.permute_ext(ids_ext, cfg.E)
    w_ref, add_w = orc.round_weights(lg, ids_ref, add_tok, add_exp, True)
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(v["assign_to_perm"].cpu().numpy()[:a2p.size], a2p)
    np.testing.assert_array_equal(v["add_tok"].cpu().numpy()[:add_tok.size], add_tok)
    nk = int(offsets[-1])
    np.testing.assert_array_equal(v["slot_token"].cpu().numpy()[:nk],
                                  orc.slot_tokens(p2a, nk, cfg.K, cfg.T, add_tok))
    assert np.abs(v["topk_w"].cpu().numpy().astype(np.float64) - w_ref).max() <= W_ABS
    assert np.abs(v["add_w"].cpu().numpy()[:add_w.size] - add_w).max() <= W_ABS
    assert add_tok.size > 0 and np.all(np.diff(offsets) % R == 0)
    rng = np.random.default_rng(13)
    tokens = np.unique(np.concatenate([rng.choice(cfg.T, size=10, replace=False),
                                       add_tok[:3], np.nonzero((~keep).any(1))[0][:2]]))
    ref_rows = orc.forward_rows(tokens, inp.x, inp.w_gate, inp.w_up, inp.w_down, ids_ref, w_ref,
                                a2p[:cfg.T * cfg.K], cfg.K)
    ref_rows += _added_rows(tokens, inp.x, inp.w_gate, inp.w_up, inp.w_down, add_tok, add_exp,
                            add_w)
    assert_bf16_close(out[torch.from_numpy(tokens).cuda()].float().cpu().numpy(), ref_rows,
                      "rounded-up forward out")


def test_token_rounding_up_rejected_where_it_cannot_apply(cuda_lib):
    """Up and nearest run in moe_forward only: moe_dispatch and moe_forward_h refuse them."""
    tdr = cuda_lib
    T, d, E, K, n = 64, 64, 8, 2, 64
    s = tdr.make_shape(T, d, E, K, n, 0.0, True, torch.bfloat16, tile_round=16,
                       tile_round_mode=1)
    lg = torch.randn(T, E, device="cuda")
    with pytest.raises(tdr.MoEError):
        tdr.dispatch(s, logits_in=lg)
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    wg = torch.randn(E, d, n, device="cuda").to(torch.bfloat16)
    wd = torch.randn(E, n, d, device="cuda").to(torch.bfloat16)
    with pytest.raises(tdr.MoEError):
        tdr.forward_h(s, x, None, wg, wg, wd, logits_in=lg)


# ------------------------------------------------------------------ backward (expert half)
def _bwd_case(tdr, cfg, seed, ffn_variant=0, input_grad=True):
    inp = mi.make_inputs(cfg)
    s = shape_of(cfg, tdr, ffn_variant=ffn_variant)
    out_h, ws, h = tdr.forward_h(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                                 cuda(inp.w_down), bias=cuda(inp.bias))
    v = tdr.workspace_views(s, ws)
    rng = np.random.default_rng(seed)
    d_out = torch.from_numpy(rng.standard_normal((cfg.T, cfg.d)).astype(np.float32)).to(
        torch.bfloat16)
    d_h, d_w, d_x = tdr.backward(s, d_out.cuda(), v["topk_w"], v["offsets"], v["perm_to_assign"],
                                 v["assign_to_perm"], cuda(inp.w_down), h,
                                 w_gate=cuda(inp.w_gate), w_up=cuda(inp.w_up),
                                 input_grad=input_grad)
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    return inp, s, out_h, v, h, d_out, d_h, d_w, d_x


@pytest.mark.parametrize("bwd_rows", [3, 1], ids=["rows_copied", "rows_gathered"])
@pytest.mark.parametrize("T,d,n,E,K,cf", [
    (300, 128, 128, 8, 2, 0.0),
    (513, 256, 384, 4, 2, 0.8),    # a half n-tile, capacity drops
    (1000, 512, 768, 16, 4, 0.0),
])
def test_backward_act_matches_oracle(cuda_lib, bwd_rows, T, d, n, E, K, cf):
    """dA' with the dO rows copied expert-major first (ffn_variant 3) and gathered inside the
    GEMM (ffn_variant 1); the full-size case below takes the automatic choice (copied)."""
    tdr = cuda_lib
    cfg = mi.MoEConfig("bwd", T=T, d=d, E=E, K=K, n=n, dtype="bf16", capacity_factor=cf,
                       seed=T + n)
    inp, s, out_h, v, h, d_out, d_h, d_w, d_x = _bwd_case(tdr, cfg, 5, ffn_variant=bwd_rows)
    # the forward is the plain one, and h holds the pre-activations
    out_plain, _ = tdr.forward(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                               cuda(inp.w_down))
    assert torch.equal(out_plain, out_h)
    offsets = v["offsets"].cpu().numpy()
    p2a = v["perm_to_assign"].cpu().numpy()
    a2p = v["assign_to_perm"].cpu().numpy()
    nk = int(offsets[-1])
    g, u = orc.gate_up_preact(inp.x, p2a, offsets, K, inp.w_gate, inp.w_up)
    hh = h[:nk].float().cpu().numpy()
    assert_bf16_close(hh[:, :n], g, "h (g)")
    assert_bf16_close(hh[:, n:], u, "h (u)")
    dG, dU, dw_ref = orc.backward_act(d_out.float().numpy(), v["topk_w"].cpu().numpy(), a2p, p2a,
                                      offsets, K, inp.w_down, g, u)
    dh = d_h[:nk].float().cpu().numpy()
    assert_bf16_close(dh[:, :n], dG, "dG")
    assert_bf16_close(dh[:, n:], dU, "dU")
    assert_bf16_close(d_w.cpu().numpy(), dw_ref, "d_w")
    dx_ref = orc.backward_dx(dG, dU, a2p, p2a, offsets, K, T, inp.w_gate, inp.w_up)
    assert_bf16_close(d_x.float().cpu().numpy(), dx_ref, "d_x")
    if cf > 0:
        assert np.all(d_w.cpu().numpy().reshape(-1)[a2p < 0] == 0)


def test_backward_without_input_grad_matches_with(cuda_lib):
    """moe_backward without d_x (the row buffer still holds the copied dO rows) gives the
    same d_h and d_w as with it."""
    tdr = cuda_lib
    cfg = mi.MoEConfig("bwd", T=700, d=256, E=8, K=2, n=256, dtype="bf16", seed=3)
    _, _, _, _, _, _, d_h1, d_w1, _ = _bwd_case(tdr, cfg, 6, ffn_variant=3, input_grad=True)
    _, _, _, _, _, _, d_h0, d_w0, d_x0 = _bwd_case(tdr, cfg, 6, ffn_variant=3,
                                                   input_grad=False)
    assert d_x0 is None
    assert torch.equal(d_h0, d_h1) and torch.equal(d_w0, d_w1)


def test_backward_act_full_size_sampled_slots(cuda_lib):
    tdr = cuda_lib
    cfg = mi.CONFIGS["mixtral_bf16"]
    inp, s, _, v, h, d_out, d_h, d_w, d_x = _bwd_case(tdr, cfg, 9)
    offsets = v["offsets"].cpu().numpy()
    p2a = v["perm_to_assign"].cpu().numpy()
    w = v["topk_w"].cpu().numpy().reshape(-1)
    rng = np.random.default_rng(4)
    slots = np.sort(rng.choice(int(offsets[-1]), size=12, replace=False))
    K, n = cfg.K, cfg.n
    dO = d_out.float().numpy().astype(np.float64)
    dh = d_h.float().cpu().numpy()
    got_g, got_u, ref_g, ref_u, got_w, ref_w = [], [], [], [], [], []
    for p in slots:
        e = orc.expert_of_slot(offsets, int(p))
        a = int(p2a[p])
        t = a // K
        xt = orc.as_f64(inp.x[t])
        g = xt @ orc.as_f64(inp.w_gate[e])
        u = xt @ orc.as_f64(inp.w_up[e])
        dA1 = dO[t] @ orc.as_f64(inp.w_down[e]).T
        sg = 1.0 / (1.0 + np.exp(-g))
        silu = g * sg
        ref_w.append(float(np.dot(dA1, silu * u)))
        dA = w[a] * dA1
        ref_g.append(dA * u * sg * (1.0 + g * (1.0 - sg)))
        ref_u.append(dA * silu)
        got_g.append(dh[p, :n])
        got_u.append(dh[p, n:])
        got_w.append(float(d_w.reshape(-1)[a]))
    assert_bf16_close(np.array(got_g), np.array(ref_g), "full-size dG")
    assert_bf16_close(np.array(got_u), np.array(ref_u), "full-size dU")
    assert_bf16_close(np.array(got_w), np.array(ref_w), "full-size d_w")
    # the input gradient of a few tokens: every kept slot of the token, in slot order
    a2p = v["assign_to_perm"].cpu().numpy().reshape(cfg.T, K)
    ids = v["topk_ids"].cpu().numpy()
    toks = rng.choice(cfg.T, size=3, replace=False)
    ref_dx = np.zeros((toks.size, cfg.d))
    for i, t in enumerate(toks):
        xt = orc.as_f64(inp.x[t])
        for k in range(K):
            if a2p[t, k] < 0:
                continue
            e = int(ids[t, k])
            g = xt @ orc.as_f64(inp.w_gate[e])
            u = xt @ orc.as_f64(inp.w_up[e])
            sg = 1.0 / (1.0 + np.exp(-g))
            dA = w[t * K + k] * (dO[t] @ orc.as_f64(inp.w_down[e]).T)
            dG = dA * u * sg * (1.0 + g * (1.0 - sg))
            dU = dA * g * sg
            ref_dx[i] += dG @ orc.as_f64(inp.w_gate[e]).T + dU @ orc.as_f64(inp.w_up[e]).T
    assert_bf16_close(d_x[torch.from_numpy(toks).cuda()].float().cpu().numpy(), ref_dx,
                      "full-size d_x")


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("E,K", [(16, 3), (40, 4), (128, 8)])  # > 16: the tensor-core forms
def test_backward_router_matches_oracle(cuda_lib, renorm, E, K):
    tdr = cuda_lib
    T, d, n = 700, 256, 128
    cfg = mi.MoEConfig("rbwd", T=T, d=d, E=E, K=K, n=n, dtype="bf16", seed=77)
    inp = mi.make_inputs(cfg)
    bias = mi.zipf_bias(E, 1.2, 1.75)
    s = tdr.make_shape(T, d, E, K, n, 0.0, renorm, torch.bfloat16)
    _, ws, h = tdr.forward_h(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                             cuda(inp.w_down), bias=cuda(bias))
    v = tdr.workspace_views(s, ws)
    rng = np.random.default_rng(8)
    d_out = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(torch.bfloat16)
    d_h, d_w, d_x = tdr.backward(s, d_out.cuda(), v["topk_w"], v["offsets"], v["perm_to_assign"],
                                 v["assign_to_perm"], cuda(inp.w_down), h, w_gate=cuda(inp.w_gate),
                                 w_up=cuda(inp.w_up), input_grad=True)
    dx_experts = d_x.float().cpu().numpy()
    d_logits, d_w_r, d_bias = tdr.backward_router(s, cuda(inp.x), cuda(inp.w_r), v["topk_ids"],
                                                  v["topk_w"], d_w, logits=v["logits"], d_x=d_x,
                                                  with_bias=True)
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    ref = orc.backward_router(d_w.cpu().numpy(), v["topk_ids"].cpu().numpy(),
                              v["logits"].cpu().numpy(), inp.x, inp.w_r, renorm)
    np.testing.assert_allclose(d_logits.cpu().numpy(), ref[0], rtol=1e-4, atol=1e-6)
    np.testing.assert_allclose(d_w_r.cpu().numpy(), ref[1], rtol=1e-3, atol=1e-4)
    np.testing.assert_allclose(d_bias.cpu().numpy(), ref[2], rtol=1e-3, atol=1e-4)
    assert_bf16_close(d_x.float().cpu().numpy() - dx_experts, ref[3], "router term of d_x")
    if renorm:
        ids = v["topk_ids"].cpu().numpy()
        mask = np.zeros((T, E), bool)
        np.put_along_axis(mask, ids, True, axis=1)
        assert np.all(d_logits.cpu().numpy()[~mask] == 0)


@pytest.mark.parametrize("T,d,E,K,renorm,with_bias,misalign_w_r", [
    (5, 192, 24, 2, True, True, False),        # one block of tokens: most ranks sum nothing
    (1000, 320, 200, 8, False, True, False),   # 4 expert chunks; the last column tile half out
    (2049, 128, 64, 4, True, False, False),    # one expert chunk, no bias
    (300, 256, 136, 6, False, True, False),    # 3 expert chunks, E not a multiple of 32
    (4100, 2048, 128, 8, True, True, False),   # 16 column tiles x 8 token ranges
    (700, 256, 36, 3, True, True, False),      # E % 8 != 0: the CUDA-core forms
    (700, 256, 64, 4, True, True, True),       # W_r not 16-byte aligned: CUDA-core d_x term
])
def test_backward_router_forms(cuda_lib, T, d, E, K, renorm, with_bias, misalign_w_r):
    """moe_backward_router against the oracle over the shapes that select its kernel forms:
    d_W_r, d_bias and the d_x term (added to a non-zero d_x) for uneven token blocks, partial
    column tiles, 1-4 expert chunks, and the CUDA-core fallbacks."""
    tdr = cuda_lib
    rng = np.random.default_rng(T + d + E)
    x = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(torch.bfloat16)
    w_r = torch.from_numpy((0.05 * rng.standard_normal((d, E))).astype(np.float32)).to(
        torch.bfloat16)
    logits = torch.from_numpy(rng.standard_normal((T, E)).astype(np.float32))
    d_w = torch.from_numpy(rng.standard_normal((T, K)).astype(np.float32))
    s = tdr.make_shape(T, d, E, K, 64, 0.0, renorm, torch.bfloat16)
    ids, w, _ = tdr.route(s, logits_in=logits.cuda())
    ref = orc.backward_router(d_w.numpy(), ids.cpu().numpy(), logits.numpy(), x, w_r, renorm)
    # a d_x to add to, at a tenth of the router term's spread (its bf16 rounding stays small
    # against the term)
    d_x0 = torch.from_numpy((0.1 * ref[3].std() * rng.standard_normal((T, d))).astype(
        np.float32)).to(torch.bfloat16)
    w_r_dev = w_r.cuda()
    if misalign_w_r:  # the same values 2 bytes past a 16-byte boundary
        buf = torch.empty(d * E + 8, dtype=torch.bfloat16, device="cuda")
        w_r_dev = buf[1:1 + d * E].view(d, E)
        w_r_dev.copy_(w_r.cuda())
        assert w_r_dev.data_ptr() % 16 != 0
    d_x = d_x0.cuda()
    d_logits, d_w_r, d_bias = tdr.backward_router(s, x.cuda(), w_r_dev, ids, w, d_w.cuda(),
                                                  logits=logits.cuda(), d_x=d_x,
                                                  with_bias=with_bias)
    torch.cuda.synchronize()
    assert_status_ok(tdr)
    np.testing.assert_allclose(d_logits.cpu().numpy(), ref[0], rtol=1e-4, atol=1e-6)
    np.testing.assert_allclose(d_w_r.cpu().numpy(), ref[1], rtol=1e-3, atol=1e-4)
    if with_bias:
        np.testing.assert_allclose(d_bias.cpu().numpy(), ref[2], rtol=1e-3, atol=1e-4)
    else:
        assert d_bias is None
    assert_bf16_close(d_x.float().cpu().numpy() - d_x0.float().numpy(), ref[3],
                      "router term of d_x")


@pytest.mark.parametrize("T", mi.DISPATCH_COMBINE_T)
def test_dispatch_combine_identity_experts(cuda_lib, T):
    """route (given logits) -> permute with x_perm -> combine(y_perm = x_perm) returns x."""
    tdr = cuda_lib
    cfg = mi.DISPATCH_COMBINE.with_T(T)
    inp = mi.make_inputs(cfg)
    s = shape_of(cfg, tdr)
    x = cuda(inp.x)
    ids, w, _ = tdr.route(s, logits_in=cuda(inp.logits))
    perm = tdr.permute(s, ids, x=x, materialize=True)
    out = tdr.combine(s, perm["x_perm"], perm["assign_to_perm"], w)
    ids_ref, w_ref = check_routing(tdr, inp.logits, ids, w, cfg.K)
    check_permutation(perm, ids_ref, cfg.E, None)
    got = out.float().cpu().numpy()
    xr = inp.x.float().numpy()
    ulp = np.abs(xr) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(got - xr) <= ulp)
    assert_status_ok(tdr)


def test_forward_edge_cases(cuda_lib, ffn_variant):
    tdr = cuda_lib
    # one token; one expert with K = 1; all tokens forced onto one expert; tiny capacity
    for (T, d, n, E, K, cf, force) in [(1, 64, 64, 4, 2, 0.0, False),
                                       (77, 64, 128, 1, 1, 0.0, False),
                                       (300, 128, 64, 8, 2, 0.0, True),
                                       (300, 128, 64, 8, 2, 0.1, True)]:
        cfg = mi.MoEConfig("edge", T=T, d=d, E=E, K=K, n=n, dtype="bf16", capacity_factor=cf,
                           seed=T + E)
        inp = mi.make_inputs(cfg)
        s = shape_of(cfg, tdr, ffn_variant=ffn_variant)
        logits = None
        if force:
            lg = np.zeros((T, E), np.float32)
            lg[:, 3] = 5.0
            lg[:, 5] = 4.0
            logits = torch.from_numpy(lg)
        out, ws = tdr.forward(s, cuda(inp.x), cuda(inp.w_r), cuda(inp.w_gate), cuda(inp.w_up),
                              cuda(inp.w_down), logits_in=cuda(logits))
        v = tdr.workspace_views(s, ws)
        ref = orc.forward(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, K,
                          capacity_factor=cf, logits=v["logits"].cpu().numpy())
        np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["topk_ids"])
        np.testing.assert_array_equal(v["assign_to_perm"].cpu().numpy(), ref["assign_to_perm"])
        got = out.float().cpu().numpy()
        if np.abs(ref["out"]).max() == 0:
            assert np.abs(got).max() == 0
        else:
            assert_bf16_close(got, ref["out"], f"edge T={T} E={E} cf={cf}")
        assert_status_ok(tdr)
    s0 = tdr.make_shape(0, 64, 4, 2, 64, 0.0, True, torch.bfloat16, ffn_variant=ffn_variant)
    z = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64, 4, dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros(4, 64, 64, dtype=torch.bfloat16, device="cuda")
    out0, _ = tdr.forward(s0, z, w, wg, wg, wg)
    assert out0.shape == (0, 64)
    assert_status_ok(tdr)
