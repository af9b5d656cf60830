"""The C-ABI library loads on a host without a GPU, exports every symbol that
include/moe.h declares, and rejects bad arguments on the host (no CUDA call is
made for these: argument checks return before anything is enqueued)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import token_dispatch_router_b200 as tdr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\**\s+\**(moe_[a-z_0-9]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from token_dispatch_router_b200 import build
    build.build()
    return tdr.load_library()


def test_header_declares_the_pipeline_entry_points():
    names = _declared_functions()
    for required in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", tdr.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    for n in _declared_functions():
        assert getattr(lib, n) is not None


def test_library_has_no_torch_dependency():
    r = subprocess.run(["ldd", tdr.LIB_PATH], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    needed = [line.split()[0] for line in r.stdout.splitlines() if line.strip()]
    assert not [n for n in needed if "torch" in n or "c10" in n], r.stdout


def test_status_strings_and_kernel_names(lib):
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(5) == b"device wait timed out"
    names = [lib.moe_kernel_name(i).decode() for i in range(lib.moe_kernel_count())]
    assert "gateup_tc" in names and "combine" in names and "route" in names


def test_workspace_sizes_are_host_arithmetic(lib):
    s = tdr.make_shape(4096, 4096, 8, 2, 14336)
    size = tdr.forward_workspace_size(s)
    L = tdr.forward_workspace_layout(s)
    assert size == L.total
    A = 4096 * 2
    assert L.y_perm - L.a_act >= A * 14336 * 2
    assert L.total - L.y_perm >= A * 4096 * 2
    for off in (L.logits, L.topk_ids, L.topk_w, L.counts, L.offsets, L.assign_to_perm,
                L.perm_to_assign, L.permute_scratch, L.a_act, L.y_perm):
        assert off % 256 == 0
    assert tdr.permute_workspace_size(s) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(T=16, d=128, E=8, K=9, n=128), 1),            # K > E
    (dict(T=16, d=128, E=300, K=2, n=128), 2),          # E > 256
    (dict(T=16, d=128, E=64, K=33, n=128), 2),          # K > 32
    (dict(T=16, d=100, E=8, K=2, n=128), 1),            # d not a multiple of 64
    (dict(T=16, d=128, E=8, K=2, n=100), 1),            # n not a multiple of 64 (bf16)
    (dict(T=-1, d=128, E=8, K=2, n=128), 1),            # negative T
])
def test_bad_shapes_rejected_on_host(lib, kw, code):
    s = tdr.make_shape(**kw)
    assert lib.moe_forward_workspace_size(ctypes.byref(s)) == 0
    r = lib.moe_forward(ctypes.byref(s), None, None, None, None, None, None, None, None, None, 0,
                        None)
    assert r == code


def test_null_pointers_and_short_workspace_rejected(lib):
    s = tdr.make_shape(16, 128, 8, 2, 128)
    assert lib.moe_route(ctypes.byref(s), None, None, None, None, None, None, None, None) == 1
    assert lib.moe_combine(ctypes.byref(s), None, None, None, None, None) == 1
    dummy = ctypes.c_void_p(256)  # never dereferenced: the workspace check fails first
    r = lib.moe_permute(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, None, None, None, 0,
                        None)
    assert r == 4
    r = lib.moe_forward(ctypes.byref(s), dummy, dummy, None, None, dummy, dummy, dummy, dummy,
                        None, 0, None)
    assert r == 4
    assert lib.moe_selftest_timeout(0, None) == 1


def test_dispatch_argument_checks_on_host(lib):
    s = tdr.make_shape(16, 128, 8, 2, 128)
    dummy = ctypes.c_void_p(256)  # never dereferenced: every check below fails first
    # a missing output
    r = lib.moe_dispatch(ctypes.byref(s), None, None, None, dummy, None, None, dummy, dummy,
                         dummy, dummy, dummy, None, None, 0, None)
    assert r == 1
    # given logits, but no workspace for the permute scratch
    r = lib.moe_dispatch(ctypes.byref(s), None, None, None, dummy, None, dummy, dummy, dummy,
                         dummy, dummy, dummy, None, None, 0, None)
    assert r == 4
    # a gather without x
    r = lib.moe_dispatch(ctypes.byref(s), None, None, None, dummy, None, dummy, dummy, dummy,
                         dummy, dummy, dummy, dummy, None, 0, None)
    assert r == 1
    bad = tdr.make_shape(16, 128, 8, 9, 128)  # K > E
    r = lib.moe_dispatch(ctypes.byref(bad), None, None, None, dummy, None, dummy, dummy, dummy,
                         dummy, dummy, dummy, None, None, 0, None)
    assert r == 1


def test_token_rounding_shape_checks(lib):
    ok = tdr.make_shape(4096, 128, 8, 2, 128, 0.0, True, tile_round=128)
    plain = tdr.make_shape(4096, 128, 8, 2, 128)
    assert lib.moe_forward_workspace_size(ctypes.byref(ok)) > \
        lib.moe_forward_workspace_size(ctypes.byref(plain))
    assert lib.moe_permute_workspace_size(ctypes.byref(ok)) >= \
        lib.moe_permute_workspace_size(ctypes.byref(plain)) + 4096 * 2 * 4
    neg = tdr.make_shape(16, 128, 8, 2, 128, 0.0, True, tile_round=-1)
    both = tdr.make_shape(16, 128, 8, 2, 128, 1.0, True, tile_round=16)
    for s in (neg, both):
        assert lib.moe_forward_workspace_size(ctypes.byref(s)) == 0
        assert lib.moe_forward(ctypes.byref(s), None, None, None, None, None, None, None, None,
                               None, 0, None) == 1
    dummy = ctypes.c_void_p(256)
    r = lib.moe_permute(ctypes.byref(ok), dummy, dummy, dummy, dummy, dummy, None, None, dummy,
                        1 << 30, None)
    assert r == 2  # rounding needs the logits: not available to moe_permute


# ------------------------------------------------------------------ atomic experts
@pytest.mark.parametrize("kw,code", [
    (dict(T=16, d=200, n_rows=8, n_cols=8, K=4), 1),      # d not a multiple of 256
    (dict(T=16, d=256, n_rows=8, n_cols=8, K=65), 1),     # K > N
    (dict(T=16, d=256, n_rows=0, n_cols=8, K=1), 1),      # empty axis
    (dict(T=-1, d=256, n_rows=8, n_cols=8, K=4), 1),      # negative T
    (dict(T=16, d=2304, n_rows=8, n_cols=8, K=4), 2),     # d / 256 = 9: no kernel variant
    (dict(T=16, d=256, n_rows=2048, n_cols=8, K=4), 2),   # axis above 1024
    (dict(T=16, d=256, n_rows=1024, n_cols=1024, K=5000), 2),  # K above 4096
])
def test_omni_bad_shapes_rejected_on_host(lib, kw, code):
    s = tdr.make_omni_shape(**kw)
    assert lib.moe_omni_workspace_size(ctypes.byref(s)) == 0
    r = lib.moe_omni_forward(ctypes.byref(s), None, None, None, None, None, None, None, None, 0,
                             None)
    assert r == code


def test_omni_workspace_layout_is_host_arithmetic(lib):
    T, d, nr, nc, K = 4096, 1024, 320, 320, 512
    s = tdr.make_omni_shape(T, d, nr, nc, K)
    L = tdr.omni_workspace_layout(s)
    N, M = nr * nc, T * K
    assert L.logits == 0 and L.topk_ids >= T * (nr + nc) * 4
    assert L.h - L.perm_to_assign >= M * 4 and L.scratch - L.h >= M * 4
    assert L.y32 >= L.scratch + (2 * N + M) * 4 and L.total >= L.y32 + T * d * 4
    for f in ("topk_ids", "topk_w", "counts", "offsets", "assign_to_perm", "perm_to_assign",
              "h", "scratch", "y32", "total"):
        assert getattr(L, f) % 256 == 0
    assert lib.moe_omni_workspace_size(ctypes.byref(s)) == L.total


def test_omni_argument_checks_on_host(lib):
    s = tdr.make_omni_shape(16, 256, 12, 8, 4)  # n_rows not a multiple of 8: no router GEMM
    dummy = ctypes.c_void_p(256)  # never dereferenced: every check below fails first
    # missing outputs
    assert lib.moe_omni_route(ctypes.byref(s), dummy, dummy, dummy, None, dummy, None, None,
                              None) == 1
    # the router GEMM needs both axes in multiples of 8
    assert lib.moe_omni_route(ctypes.byref(s), dummy, dummy, dummy, None, dummy, dummy, dummy,
                              None) == 2
    # no logits at all
    assert lib.moe_omni_route(ctypes.byref(s), None, None, None, None, None, dummy, dummy,
                              None) == 1
    # schedule and forward without a workspace
    assert lib.moe_omni_schedule(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, None, 0,
                                 None) == 4
    assert lib.moe_omni_forward(ctypes.byref(s), dummy, dummy, dummy, None, dummy, dummy, dummy,
                                None, 0, None) == 4
    # experts without the scalar buffer
    assert lib.moe_omni_experts(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, dummy, dummy,
                                None, dummy, None) == 1
    # output modes: 0 and 1 only (a field of the shape, checked per call)
    bad = tdr.make_omni_shape(16, 256, 8, 8, 4, output_mode=2)
    assert lib.moe_omni_workspace_size(ctypes.byref(bad)) == 0
    assert lib.moe_omni_forward(ctypes.byref(bad), dummy, dummy, dummy, None, dummy, dummy, dummy,
                                dummy, 1 << 30, None) == 1
    # T = 0 is a no-op
    z = tdr.make_omni_shape(0, 256, 8, 8, 4)
    assert lib.moe_omni_route(ctypes.byref(z), None, None, None, None, None, None, None,
                              None) == 0


@pytest.mark.parametrize("variant,code", [(0, 0), (3, 0), (4, 1), (-1, 1)])
def test_ffn_variant_is_a_checked_shape_field(lib, variant, code):
    """The grouped-GEMM tile variant travels with each call's shape (no process-wide state):
    valid values size a workspace, others are rejected on the host."""
    s = tdr.make_shape(64, 128, 8, 2, 128, 0.0, True, torch.bfloat16, ffn_variant=variant)
    size = lib.moe_forward_workspace_size(ctypes.byref(s))
    assert (size > 0) == (code == 0)
    if code:
        assert lib.moe_grouped_ffn(ctypes.byref(s), *([ctypes.c_void_p(256)] * 8), None) == code


def test_no_process_wide_switches_exported(lib):
    """Variant and output-mode selection are per-call shape fields, not library state."""
    for name in ("moe_set_ffn_variant", "moe_get_ffn_variant", "moe_set_route_layout",
                 "moe_get_route_layout", "moe_omni_set_output_mode", "moe_omni_get_output_mode"):
        assert not hasattr(lib, name), name


@pytest.mark.parametrize("form,ok", [(0, True), (1, True), (2, True), (3, False)])
def test_route_topk_is_a_checked_shape_field(lib, form, ok):
    """The top-K form of the warp-per-token routers is a per-call shape field."""
    s = tdr.make_shape(64, 128, 8, 2, 128, 0.0, True, torch.bfloat16, route_topk=form)
    assert (lib.moe_forward_workspace_size(ctypes.byref(s)) > 0) == ok


@pytest.mark.parametrize("mode,ok", [(0, True), (1, True), (2, True), (3, False), (-1, False)])
def test_tile_round_mode_is_a_checked_shape_field(lib, mode, ok):
    """The rounding direction is a per-call shape field: 0 down, 1 up, 2 nearest."""
    s = tdr.make_shape(64, 128, 8, 2, 128, 0.0, True, torch.bfloat16, tile_round=16,
                       tile_round_mode=mode)
    assert (lib.moe_forward_workspace_size(ctypes.byref(s)) > 0) == ok


def test_rounding_up_layout_spans_the_added_assignments(lib):
    """Rounding up or to the nearest tile lays out T*K + E*(R-1) entries in both maps, the
    activations and the expert outputs, plus the added-assignment lists; rounding down and
    no rounding lay out T*K."""
    T, d, E, K, n, R = 1000, 128, 8, 2, 128, 16
    lays = {}
    for mode in (0, 1, 2):
        s = tdr.make_shape(T, d, E, K, n, 0.0, True, torch.bfloat16, tile_round=R,
                           tile_round_mode=mode)
        lays[mode] = tdr.forward_workspace_layout(s)
    assert lays[0].n_assign == T * K
    for mode in (1, 2):
        L = lays[mode]
        assert L.n_assign == T * K + E * (R - 1)
        assert L.y_perm - L.a_act >= L.n_assign * n * 2
        assert L.add_w - L.add_tok >= E * (R - 1) * 4
        assert L.add_idx - L.add_ptr >= (T + 1) * 4
        assert L.total - L.slot_token >= L.n_assign * 4
        offs = [L.logits, L.topk_ids, L.topk_w, L.counts, L.offsets, L.assign_to_perm,
                L.perm_to_assign, L.permute_scratch, L.a_act, L.y_perm, L.round_ids,
                L.round_counts, L.add_tok, L.add_w, L.add_ptr, L.add_idx, L.add_cursor,
                L.slot_token, L.total]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    plain = tdr.forward_workspace_layout(tdr.make_shape(T, d, E, K, n, 0.0, True,
                                                        torch.bfloat16))
    assert plain.n_assign == T * K and plain.slot_token == plain.total


def test_rounding_up_limits(lib):
    """Up and nearest: one bit a token in shared memory (T <= 131072); moe_dispatch only
    rounds down."""
    big = tdr.make_shape(131073, 128, 8, 2, 128, 0.0, True, torch.bfloat16, tile_round=16,
                         tile_round_mode=1)
    assert lib.moe_forward_workspace_size(ctypes.byref(big)) == 0
    edge = tdr.make_shape(131072, 128, 8, 2, 128, 0.0, True, torch.bfloat16, tile_round=16,
                          tile_round_mode=1)
    assert lib.moe_forward_workspace_size(ctypes.byref(edge)) > 0
    down = tdr.make_shape(131073, 128, 8, 2, 128, 0.0, True, torch.bfloat16, tile_round=16)
    assert lib.moe_forward_workspace_size(ctypes.byref(down)) > 0
