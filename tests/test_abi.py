"""The C-ABI library: it loads, exports every declared symbol, and rejects bad
arguments on the host before touching the GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dflash.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from helpers_build import build_library
    return ctypes.CDLL(build_library())


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n


def test_build_id_matches_sources(lib):
    """The library loaded here was compiled from the sources in this tree."""
    from helpers_build import build_module
    lib.dflash_build_id.restype = ctypes.c_char_p
    assert lib.dflash_build_id().decode() == build_module().source_hash()


def test_stale_library_is_rebuilt(tmp_path, monkeypatch):
    """A recorded hash that differs from the sources' hash means the library
    is out of date, whatever the files' modification times say."""
    mod = __import__("helpers_build").build_module()
    stamp = tmp_path / "stamp"
    stamp.write_text("0123456789abcdef\n")
    monkeypatch.setattr(mod, "HASH_FILE", str(stamp))
    assert not mod.up_to_date()
    stamp.write_text(mod.source_hash() + "\n")
    assert mod.up_to_date() == os.path.exists(mod.LIB)


def test_status_strings(lib):
    lib.dflash_status_string.restype = ctypes.c_char_p
    seen = set()
    for code in range(7):
        s = lib.dflash_status_string(code).decode()
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 7
    assert lib.dflash_status_string(99).decode() == "unknown status"


def test_host_side_rejections(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)  # never dereferenced: every call below fails validation first
    # K != 16
    r = lib.dflash_lmhead_topk(fake, fake, 4, 4096, 256, 15, fake, fake, None, fake, ctypes.c_size_t(1 << 20),
                               None, None)
    assert r == 1
    # null H
    r = lib.dflash_lmhead_topk(None, fake, 4, 4096, 256, 16, fake, fake, None, fake, ctypes.c_size_t(1 << 20),
                               None, None)
    assert r == 1
    # conv: d not a multiple of 8, null x
    assert lib.dflash_conv2tap(fake, None, fake, fake, fake, 1, 5, 12, None) == 1
    assert lib.dflash_conv2tap(None, None, fake, fake, fake, 1, 5, 16, None) == 1
    # select: r not a multiple of 8, L > 16, K != 16
    assert lib.dflash_path_select(fake, fake, fake, fake, 1, 4, 16, 12, 100, fake, None, None, None, None, None) == 1
    assert lib.dflash_path_select(fake, fake, fake, fake, 1, 17, 16, 32, 100, fake, None, None, None, None, None) == 1
    assert lib.dflash_path_select(fake, fake, fake, fake, 1, 4, 8, 32, 100, fake, None, None, None, None, None) == 1
    # verify: L out of range
    assert lib.dflash_verify(fake, fake, 1, 0, fake, fake, None) == 1
    assert lib.dflash_verify(fake, fake, 1, 33, fake, fake, None) == 1
    # walk: no anchor; sampling at temperature 0; target without outputs
    f32 = ctypes.c_float
    lib.dflash_path_walk.argtypes = [vp, vp, vp, vp, vp, vp, f32] + [ctypes.c_int] * 5 + [vp] * 9
    assert lib.dflash_path_walk(fake, fake, fake, fake, None, None, 1.0, 1, 4, 16, 32, 100,
                                fake, None, None, None, None, None, None, None, None) == 1
    assert lib.dflash_path_walk(fake, fake, fake, fake, fake, fake, 0.0, 1, 4, 16, 32, 100,
                                fake, None, None, None, None, None, None, None, None) == 1
    assert lib.dflash_path_walk(fake, fake, fake, fake, fake, None, 1.0, 1, 4, 16, 32, 100,
                                fake, None, None, None, fake, None, None, None, None) == 1
    # rejection verify: temperature <= 0, L > 31, V too large, workspace too small
    i32 = ctypes.c_int
    lib.dflash_verify_rejection.argtypes = ([vp, f32] + [vp] * 6 + [ctypes.c_int] * 3 + [vp, vp, vp,
                                            ctypes.c_size_t, vp, vp])
    big = ctypes.c_size_t(1 << 30)
    args = lambda T, B, L, V, ws: (fake, T, fake, fake, fake, fake, fake, fake, B, L, V, fake, fake, fake, ws,
                                   None, None)
    assert lib.dflash_verify_rejection(*args(0.0, 1, 4, 1000, big)) == 1
    assert lib.dflash_verify_rejection(*args(1.0, 1, 32, 1000, big)) == 1
    assert lib.dflash_verify_rejection(*args(1.0, 1, 4, 524289, big)) == 1
    assert lib.dflash_verify_rejection(*args(1.0, 1, 4, 1000, ctypes.c_size_t(8))) == 4
    lib.dflash_verify_rejection_workspace.restype = ctypes.c_size_t
    assert lib.dflash_verify_rejection_workspace(2, 3, 8193) == 2 * 4 * 2 * 16
    # vocabulary-parallel pieces: negative offset, K != 16, bad record counts
    lib.dflash_lmhead_topk_partial.argtypes = [vp, vp, i32, i32, i32, i32, vp, ctypes.c_size_t, vp, vp]
    assert lib.dflash_lmhead_topk_partial(fake, fake, 4, 4096, 256, -16, fake, big, None, None) == 1
    lib.dflash_lmhead_topk_merge.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    assert lib.dflash_lmhead_topk_merge(fake, 4, 148, 2, 15, fake, fake, None, None) == 1
    assert lib.dflash_lmhead_topk_merge(fake, 4, 0, 2, 16, fake, fake, None, None) == 1
    assert lib.dflash_lmhead_topk_merge(fake, 4, 148, 0, 16, fake, fake, None, None) == 1
    # context-gated scorer: e not a multiple of 8 or out of range, d not a multiple of 8, K != 16, unknown
    # walk, sampling without uniforms
    i32 = ctypes.c_int
    lib.dflash_ctx_table.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    assert lib.dflash_ctx_table(fake, fake, 100, 256, 20, fake, None) == 1
    assert lib.dflash_ctx_table(fake, fake, 100, 250, 32, fake, None) == 1
    assert lib.dflash_ctx_table(fake, fake, 100, 256, 1032, fake, None) == 1
    assert lib.dflash_ctx_table(None, fake, 100, 256, 32, fake, None) == 1
    lib.dflash_ctx_gate.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    assert lib.dflash_ctx_gate(fake, fake, 4, 256, 12, fake, None) == 1
    assert lib.dflash_ctx_gate(fake, fake, 0, 256, 32, fake, None) == 1
    lib.dflash_ctx_walk.argtypes = [vp] * 5 + [i32] * 6 + [vp, f32] + [vp] * 10
    walk = lambda K, walkid, u, T: lib.dflash_ctx_walk(fake, fake, fake, fake, fake, 1, 4, K, 32, 100, walkid, u, T,
                                                       fake, None, None, None, None, None, None, None, None, None)
    assert walk(8, 0, None, 1.0) == 1
    assert walk(16, 3, None, 1.0) == 1
    assert walk(16, 2, None, 1.0) == 1
    assert walk(16, 2, fake, 0.0) == 1


def test_workspace_rejects_bad_sizes(lib):
    lib.dflash_lmhead_topk_workspace.restype = ctypes.c_size_t
    assert lib.dflash_lmhead_topk_workspace(0, 4096, 256) == 0
    assert lib.dflash_lmhead_topk_workspace(4, 8, 256) == 0
    assert lib.dflash_lmhead_topk_workspace(4, 4096, 100) == 0


def test_binding_exposes_every_entry_point():
    """The Python package has a function named after every entry point the
    header declares (the binding is argument marshalling over the same names)."""
    import block_draft_selection_b200 as bds
    missing = [n for n in _declared() if not hasattr(bds, n)]
    assert not missing, missing
