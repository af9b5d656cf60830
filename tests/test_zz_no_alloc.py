"""moe_permute_static: the permute entry point for callers that may not allocate device memory
while they run (a serving engine whose memory plan is fixed at start-up, an embedded runtime
with a fixed arena): its scratch is a fixed device array inside the library, not a caller
workspace. Called through the C ABI and checked against moe_permute, the workspace entry
point, on calls in a row that all take the chunked path whose histogram, scan and scatter
kernels keep per-chunk counts and rank bases in that array (more than 32768 assignments, and
more than 8192 chunk-experts, so the scan is not fused into the scatter). The second call is
smaller than the first, so entries the first call left behind would show up as a mismatch if
any kernel read one it had not written. This file sorts last so that a run stopping at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

LIMIT = 1 << 20  # MOE_PERMUTE_STATIC_SCRATCH_BYTES


def _ids(rng, T, E, K):
    scores = rng.standard_normal((T, E)) + 2.0 * (np.arange(E)[None, :] == 1)
    return torch.from_numpy(np.argsort(-scores, axis=1, kind="stable")[:, :K].astype(np.int32))


def _call_static(tdr, shape, ids, x, x_perm, outs):
    lib = tdr.load_library()
    return lib.moe_permute_static(
        ctypes.byref(shape), ctypes.c_void_p(ids.data_ptr()),
        ctypes.c_void_p(outs["counts"].data_ptr()), ctypes.c_void_p(outs["offsets"].data_ptr()),
        ctypes.c_void_p(outs["assign_to_perm"].data_ptr()),
        ctypes.c_void_p(outs["perm_to_assign"].data_ptr()), ctypes.c_void_p(x.data_ptr()),
        ctypes.c_void_p(x_perm.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("calls", [[(40000, 256, 8, 0.0, 128), (10000, 128, 8, 1.1, 64),
                                    (12000, 128, 6, 0.0, 64)]])
def test_static_scratch_permute_matches_workspace_permute(cuda_lib, calls):
    tdr = cuda_lib
    rng = np.random.default_rng(77)
    for T, E, K, cf, d in calls:  # calls in a row, each smaller than the one before
        A = T * K
        chunks = -(-A // 1024)
        assert A > 32768 and chunks * E > 8192  # the unfused chunked path
        assert 2 * chunks * E * 4 <= LIMIT
        ids = _ids(rng, T, E, K).cuda()
        x = torch.randn(T, d).to(torch.bfloat16).cuda()
        s = tdr.make_shape(T, d, E, K, 64, cf, True, torch.bfloat16)
        ref = tdr.permute(s, ids, x=x, materialize=True)
        outs = {k: torch.full_like(v, -7) for k, v in ref.items()}
        assert _call_static(tdr, s, ids, x, outs["x_perm"], outs) == 0
        torch.cuda.synchronize()
        assert tdr.device_status() == 0
        nk = int(ref["offsets"][E].item())
        for key in ("counts", "offsets", "assign_to_perm"):
            assert torch.equal(outs[key], ref[key]), key
        assert torch.equal(outs["perm_to_assign"][:nk], ref["perm_to_assign"][:nk])
        assert torch.equal(outs["x_perm"][:nk], ref["x_perm"][:nk])


def test_static_scratch_rejects_sizes_beyond_its_limit(cuda_lib):
    tdr = cuda_lib
    lib = tdr.load_library()
    # 2 * ceil(T*K / 1024) * E * 4 bytes > 1 MiB
    s = tdr.make_shape(2_000_000, 64, 256, 8, 64, 0.0, True, torch.bfloat16)
    dummy = ctypes.c_void_p(256)  # never used: the size check fails first
    r = lib.moe_permute_static(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, None, None,
                               None)
    assert r == 2  # MOE_ERR_UNSUPPORTED
