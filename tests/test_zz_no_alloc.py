"""dflash_lmhead_topk_static: the LM-head top-16 entry point that takes no
workspace, for callers that cannot allocate device memory at call time
(allocator hooks, engines with a fully reserved memory pool).

Called through the C ABI (ctypes), two calls in a row on different shapes
plus a repeat of the first, each checked against dflash_lmhead_topk on the
same inputs with the tolerances the other LM-head tests use (indices equal,
log-probs and lse within 2e-2).  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

import block_draft_synth as syn

pytestmark = pytest.mark.gpu


def _lib():
    from helpers_build import build_library
    lib = ctypes.CDLL(build_library())
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.dflash_lmhead_topk.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]
    lib.dflash_lmhead_topk_static.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.dflash_lmhead_topk_workspace.restype = sz
    lib.dflash_lmhead_topk_workspace.argtypes = [i32, i32, i32]
    return lib


def _inputs(M, V, d, seed):
    rng = syn.rng_for(seed, "H")
    H = syn.f32_to_bf16_bits(rng.standard_normal((M, d), dtype=np.float32))
    W = syn.f32_to_bf16_bits(rng.standard_normal((V, d), dtype=np.float32) / np.float32(np.sqrt(d)))
    t = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda()
    return t(H), t(W)


def _outs(M):
    return (torch.empty((M, 16), dtype=torch.float32, device="cuda"),
            torch.empty((M, 16), dtype=torch.int32, device="cuda"),
            torch.empty(M, dtype=torch.float32, device="cuda"),
            torch.zeros(1, dtype=torch.int32, device="cuda"))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _with_workspace(lib, H, W, stream):
    M, d = H.shape
    V = W.shape[0]
    lp, ix, lse, st = _outs(M)
    ws = torch.empty(lib.dflash_lmhead_topk_workspace(M, V, d), dtype=torch.uint8, device="cuda")
    rc = lib.dflash_lmhead_topk(_p(H), _p(W), M, V, d, 16, _p(lp), _p(ix), _p(lse), _p(ws), ws.numel(),
                                _p(st), stream)
    assert rc == 0
    return lp, ix, lse, st


def _static(lib, H, W, stream):
    M, d = H.shape
    V = W.shape[0]
    lp, ix, lse, st = _outs(M)
    rc = lib.dflash_lmhead_topk_static(_p(H), _p(W), M, V, d, 16, _p(lp), _p(ix), _p(lse), _p(st), stream)
    assert rc == 0
    return lp, ix, lse, st


def _same(a, b):
    lp_a, ix_a, lse_a, st_a = [t.cpu().numpy() for t in a]
    lp_b, ix_b, lse_b, st_b = [t.cpu().numpy() for t in b]
    assert st_a[0] == 0 and st_b[0] == 0
    np.testing.assert_array_equal(ix_a, ix_b)
    assert np.abs(lp_a - lp_b).max() <= 2e-2
    assert np.abs(lse_a - lse_b).max() <= 2e-2


def test_static_matches_workspace_version_two_calls_in_a_row():
    lib = _lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    A = _inputs(7, 151936, 2560, 1)      # weight-streaming orientation, the bs1 drafter shape
    B = _inputs(200, 3000, 128, 2)       # large-M orientation, small enough for the array
    ref_a = _with_workspace(lib, *A, stream)
    ref_b = _with_workspace(lib, *B, stream)
    got_a = _static(lib, *A, stream)
    got_b = _static(lib, *B, stream)      # second call in a row, reusing the same array
    got_a2 = _static(lib, *A, stream)     # and back: nothing stale leaks between calls
    torch.cuda.synchronize()
    _same(ref_a, got_a)
    _same(ref_b, got_b)
    _same(ref_a, got_a2)


def test_static_rejects_sizes_beyond_the_array():
    lib = _lib()
    # a shape whose partial records need far more than DFLASH_STATIC_SCRATCH_BYTES
    M, V, d = next((m, v, dd) for m, v, dd in [(10240, 151936, 4096), (20480, 151936, 4096), (40960, 262144, 1024)]
                   if lib.dflash_lmhead_topk_workspace(m, v, dd) > (8 << 20))
    fake = ctypes.c_void_p(0x1000)        # never dereferenced: rejected on the host
    rc = lib.dflash_lmhead_topk_static(fake, fake, M, V, d, 16, fake, fake, None, None, None)
    assert rc == 2
