"""ctypes binding of libdflash.so: argument marshalling only.

Each function here has the name of the C entry point it calls, checks that
the torch tensors it is given are CUDA tensors of the layout the C ABI
documents (include/dflash.h), allocates outputs the caller did not pass, and
forwards raw device pointers and the current CUDA stream.  Every step of the
computation runs in the library's kernels; there is no CPU path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdflash.so")

DFLASH_OK = 0
DFLASH_ERR_INVALID_ARG = 1
DFLASH_ERR_UNSUPPORTED = 2
DFLASH_ERR_CUDA = 3
DFLASH_ERR_WORKSPACE = 4
DFLASH_ERR_TIMEOUT = 5
DFLASH_ERR_BAD_INDEX = 6
K_TOP = 16


class DFlashError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {dflash_status_string(code)} (status {code})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python block_draft_selection_b200/build.py` "
            "(this package has no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "dflash_status_string": (ctypes.c_char_p, [i32]),
        "dflash_build_id": (ctypes.c_char_p, []),
        "dflash_conv2tap": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, vp]),
        "dflash_lmhead_topk_workspace": (sz, [i32, i32, i32]),
        "dflash_lmhead_topk": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]),
        "dflash_lmhead_logits_debug": (i32, [vp, vp, i32, i32, i32, vp, vp, sz, vp, vp]),
        "dflash_path_select": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
        "dflash_verify": (i32, [vp, vp, i32, i32, vp, vp, vp]),
        "dflash_select_verify": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]),
        "dflash_lmhead_topk_static": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
        "dflash_gemm_bf16": (i32, [vp, vp, vp, i32, i32, i32, vp]),
        "dflash_conv2tap_dynamic_workspace": (sz, [i32, i32, i32]),
        "dflash_conv2tap_dynamic": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, sz, vp]),
        "dflash_path_walk": (i32, [vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, i32, i32, i32, i32,
                                   vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "dflash_verify_rejection_workspace": (sz, [i32, i32, i32]),
        "dflash_lmhead_topk_records": (i32, [i32, i32, i32]),
        "dflash_lmhead_topk_partial": (i32, [vp, vp, i32, i32, i32, i32, vp, sz, vp, vp]),
        "dflash_lmhead_topk_merge": (i32, [vp, i32, i32, i32, i32, vp, vp, vp, vp]),
        "dflash_ctx_table": (i32, [vp, vp, i32, i32, i32, vp, vp]),
        "dflash_ctx_gate": (i32, [vp, vp, i32, i32, i32, vp, vp]),
        "dflash_ctx_walk": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, ctypes.c_float,
                                  vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "dflash_verify_rejection": (i32, [vp, ctypes.c_float, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                          vp, vp, vp, sz, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _check_build_id(lib)
    return lib


def _check_build_id(lib):
    """Refuse a library compiled from other sources than the ones beside it
    (when the sources are present): stale native code must not pass for the
    current code."""
    build_py = os.path.join(os.path.dirname(LIB_PATH), "build.py")
    if not os.path.isdir(os.path.join(os.path.dirname(LIB_PATH), "csrc")) or not os.path.exists(build_py):
        return
    import importlib.util
    spec = importlib.util.spec_from_file_location("_dflash_build_check", build_py)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    have, want = lib.dflash_build_id().decode(), mod.source_hash()
    if have != want:
        raise ImportError(f"{LIB_PATH} was built from other sources (build id {have}, sources {want}): "
                          "rebuild it with `python block_draft_selection_b200/build.py`")


lib = _load()


def dflash_status_string(code: int) -> str:
    return lib.dflash_status_string(int(code)).decode()


def dflash_build_id() -> str:
    return lib.dflash_build_id().decode()


def _check(fn: str, code: int):
    if code != DFLASH_OK:
        raise DFlashError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _out(t, name, dtype, shape, device):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _need(t, name, dtype, shape)


def dflash_conv2tap(x, a0, a1, prev=None, y=None, stream=None):
    """y[b,t,c] = a0[c] x[b,t,c] + a1[c] x[b,t-1,c], x[b,-1,:] = prev[b,:] (zeros if None).
    x [B,P,d] bf16; a0, a1 [d] bf16; prev [B,d] bf16 or None."""
    _need(x, "x", torch.bfloat16)
    B, P, d = x.shape
    _need(a0, "a0", torch.bfloat16, (d,))
    _need(a1, "a1", torch.bfloat16, (d,))
    if prev is not None:
        _need(prev, "prev", torch.bfloat16, (B, d))
    y = _out(y, "y", torch.bfloat16, (B, P, d), x.device)
    _check("dflash_conv2tap", lib.dflash_conv2tap(_ptr(x), _ptr(prev), _ptr(a0), _ptr(a1), _ptr(y),
                                                  B, P, d, _stream(stream)))
    return y


def dflash_gemm_bf16(A, B, C=None, stream=None):
    """C [M,N] fp32 = A [M,K] bf16 . B [N,K]^T, on the tensor-core path."""
    _need(A, "A", torch.bfloat16)
    _need(B, "B", torch.bfloat16)
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B disagree on K")
    C = _out(C, "C", torch.float32, (M, N), A.device)
    _check("dflash_gemm_bf16", lib.dflash_gemm_bf16(_ptr(A), _ptr(B), _ptr(C), M, N, K, _stream(stream)))
    return C


def dflash_conv2tap_dynamic_workspace(B: int, P: int, d: int) -> int:
    return int(lib.dflash_conv2tap_dynamic_workspace(B, P, d))


def dflash_conv2tap_dynamic(x, a0, a1, wc, prev=None, y=None, ws=None, stream=None):
    """Two-tap conv with per-16-channel tap corrections delta = x . Wc^T.
    x [B,P,d], a0/a1 [d], wc [2*d/16, d], prev [B,d] or None: bf16."""
    _need(x, "x", torch.bfloat16)
    B, P, d = x.shape
    _need(a0, "a0", torch.bfloat16, (d,))
    _need(a1, "a1", torch.bfloat16, (d,))
    _need(wc, "wc", torch.bfloat16, (2 * (d // 16), d))
    if prev is not None:
        _need(prev, "prev", torch.bfloat16, (B, d))
    y = _out(y, "y", torch.bfloat16, (B, P, d), x.device)
    if ws is None:
        n = dflash_conv2tap_dynamic_workspace(B, P, d)
        if n == 0:
            raise DFlashError("dflash_conv2tap_dynamic_workspace", DFLASH_ERR_INVALID_ARG)
        ws = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check("dflash_conv2tap_dynamic", lib.dflash_conv2tap_dynamic(
        _ptr(x), _ptr(prev), _ptr(a0), _ptr(a1), _ptr(wc), _ptr(y), B, P, d, _ptr(ws), ws.numel(),
        _stream(stream)))
    return y


def dflash_lmhead_topk_workspace(M: int, V: int, d: int) -> int:
    return int(lib.dflash_lmhead_topk_workspace(M, V, d))


def workspace(M: int, V: int, d: int, device="cuda") -> torch.Tensor:
    n = dflash_lmhead_topk_workspace(M, V, d)
    if n == 0:
        raise DFlashError("dflash_lmhead_topk_workspace", DFLASH_ERR_INVALID_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device)


def dflash_lmhead_topk(H, W, K=K_TOP, topk_logp=None, topk_idx=None, lse=None, ws=None,
                       dev_status=None, stream=None, want_lse=True):
    """H [M,d] bf16, W [V,d] bf16 -> (topk_logp [M,16] f32, topk_idx [M,16] i32, lse [M] f32)."""
    _need(H, "H", torch.bfloat16)
    _need(W, "W", torch.bfloat16)
    M, d = H.shape
    V = W.shape[0]
    if W.shape[1] != d:
        raise ValueError("H and W disagree on d")
    topk_logp = _out(topk_logp, "topk_logp", torch.float32, (M, K), H.device)
    topk_idx = _out(topk_idx, "topk_idx", torch.int32, (M, K), H.device)
    if lse is None and want_lse:
        lse = torch.empty(M, dtype=torch.float32, device=H.device)
    elif lse is not None:
        _need(lse, "lse", torch.float32, (M,))
    if ws is None:
        ws = workspace(M, V, d, H.device)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, (1,))
    _check("dflash_lmhead_topk", lib.dflash_lmhead_topk(
        _ptr(H), _ptr(W), M, V, d, K, _ptr(topk_logp), _ptr(topk_idx), _ptr(lse), _ptr(ws),
        ws.numel(), _ptr(dev_status), _stream(stream)))
    return topk_logp, topk_idx, lse


def dflash_lmhead_logits_debug(H, W, z=None, ws=None, dev_status=None, stream=None):
    """Raw logits z [M,V] f32 through the same GEMM path (diagnostic)."""
    _need(H, "H", torch.bfloat16)
    _need(W, "W", torch.bfloat16)
    M, d = H.shape
    V = W.shape[0]
    z = _out(z, "z", torch.float32, (M, V), H.device)
    if ws is None:
        ws = workspace(M, V, d, H.device)
    _check("dflash_lmhead_logits_debug", lib.dflash_lmhead_logits_debug(
        _ptr(H), _ptr(W), M, V, d, _ptr(z), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))
    return z


def dflash_path_select(topk_logp, topk_idx, E, Msel, B, L, path_tok=None, path_slot=None,
                       path_score=None, pair_scores=False, dev_status=None, stream=None):
    """Returns (path_tok [B,L] i32, path_slot [B,L] i32, path_score [B] f32, pair scores
    [B,L-1,16,16] f32 or None)."""
    _need(topk_logp, "topk_logp", torch.float32, (B * L, K_TOP))
    _need(topk_idx, "topk_idx", torch.int32, (B * L, K_TOP))
    _need(E, "E", torch.bfloat16)
    V, r = E.shape
    _need(Msel, "Msel", torch.bfloat16, (r, r))
    dev = topk_logp.device
    path_tok = _out(path_tok, "path_tok", torch.int32, (B, L), dev)
    path_slot = _out(path_slot, "path_slot", torch.int32, (B, L), dev)
    path_score = _out(path_score, "path_score", torch.float32, (B,), dev)
    pair = torch.empty((B, max(L - 1, 0), K_TOP, K_TOP), dtype=torch.float32, device=dev) if pair_scores else None
    _check("dflash_path_select", lib.dflash_path_select(
        _ptr(topk_logp), _ptr(topk_idx), _ptr(E), _ptr(Msel), B, L, K_TOP, r, V, _ptr(path_tok),
        _ptr(path_slot), _ptr(path_score), _ptr(pair) if pair is not None and pair.numel() else None,
        _ptr(dev_status), _stream(stream)))
    return path_tok, path_slot, path_score, pair


def dflash_select_verify(topk_logp, topk_idx, E, Msel, target, B, L, path_tok=None, path_slot=None,
                         path_score=None, accept_len=None, next_token=None, dev_status=None, stream=None):
    """Path selection and greedy verification of the chosen path in one kernel.
    Returns (path_tok, path_slot, path_score, accept_len, next_token)."""
    _need(topk_logp, "topk_logp", torch.float32, (B * L, K_TOP))
    _need(topk_idx, "topk_idx", torch.int32, (B * L, K_TOP))
    _need(E, "E", torch.bfloat16)
    V, r = E.shape
    _need(Msel, "Msel", torch.bfloat16, (r, r))
    _need(target, "target", torch.int32, (B, L + 1))
    dev = topk_logp.device
    path_tok = _out(path_tok, "path_tok", torch.int32, (B, L), dev)
    path_slot = _out(path_slot, "path_slot", torch.int32, (B, L), dev)
    path_score = _out(path_score, "path_score", torch.float32, (B,), dev)
    accept_len = _out(accept_len, "accept_len", torch.int32, (B,), dev)
    next_token = _out(next_token, "next_token", torch.int32, (B,), dev)
    _check("dflash_select_verify", lib.dflash_select_verify(
        _ptr(topk_logp), _ptr(topk_idx), _ptr(E), _ptr(Msel), _ptr(target), B, L, K_TOP, r, V,
        _ptr(path_tok), _ptr(path_slot), _ptr(path_score), _ptr(accept_len), _ptr(next_token),
        _ptr(dev_status), _stream(stream)))
    return path_tok, path_slot, path_score, accept_len, next_token


def dflash_lmhead_topk_static(H, W, K=K_TOP, topk_logp=None, topk_idx=None, lse=None, dev_status=None,
                              stream=None):
    """dflash_lmhead_topk without a workspace (library-owned scratch; see the header)."""
    _need(H, "H", torch.bfloat16)
    _need(W, "W", torch.bfloat16)
    M, d = H.shape
    V = W.shape[0]
    topk_logp = _out(topk_logp, "topk_logp", torch.float32, (M, K), H.device)
    topk_idx = _out(topk_idx, "topk_idx", torch.int32, (M, K), H.device)
    lse = _out(lse, "lse", torch.float32, (M,), H.device)
    _check("dflash_lmhead_topk_static", lib.dflash_lmhead_topk_static(
        _ptr(H), _ptr(W), M, V, d, K, _ptr(topk_logp), _ptr(topk_idx), _ptr(lse), _ptr(dev_status),
        _stream(stream)))
    return topk_logp, topk_idx, lse


def dflash_verify(draft, target, accept_len=None, next_token=None, stream=None):
    """draft [B,L] i32, target [B,L+1] i32 -> (accept_len [B] i32, next_token [B] i32)."""
    _need(draft, "draft", torch.int32)
    B, L = draft.shape
    _need(target, "target", torch.int32, (B, L + 1))
    accept_len = _out(accept_len, "accept_len", torch.int32, (B,), draft.device)
    next_token = _out(next_token, "next_token", torch.int32, (B,), draft.device)
    _check("dflash_verify", lib.dflash_verify(_ptr(draft), _ptr(target), B, L, _ptr(accept_len),
                                              _ptr(next_token), _stream(stream)))
    return accept_len, next_token


def dflash_path_walk(topk_logp, topk_idx, E, Msel, anchor, B, L, uniforms=None, temperature=1.0,
                     path_tok=None, path_slot=None, path_score=None, path_q=None, want_q=True,
                     target=None, accept_len=None, next_token=None, dev_status=None, stream=None):
    """Walk from the last verified token: greedy when `uniforms` is None, else sampled
    at `temperature`.  Returns (path_tok, path_slot, path_score, path_q or None,
    accept_len or None, next_token or None); the last two only when `target` is given."""
    _need(topk_logp, "topk_logp", torch.float32, (B * L, K_TOP))
    _need(topk_idx, "topk_idx", torch.int32, (B * L, K_TOP))
    _need(E, "E", torch.bfloat16)
    V, r = E.shape
    _need(Msel, "Msel", torch.bfloat16, (r, r))
    _need(anchor, "anchor", torch.int32, (B,))
    dev = topk_logp.device
    if uniforms is not None:
        _need(uniforms, "uniforms", torch.float32, (B, L))
    path_tok = _out(path_tok, "path_tok", torch.int32, (B, L), dev)
    path_slot = _out(path_slot, "path_slot", torch.int32, (B, L), dev)
    path_score = _out(path_score, "path_score", torch.float32, (B,), dev)
    if uniforms is not None and (want_q or path_q is not None):
        path_q = _out(path_q, "path_q", torch.float32, (B, L, K_TOP), dev)
    else:
        path_q = None
    if target is not None:
        _need(target, "target", torch.int32, (B, L + 1))
        accept_len = _out(accept_len, "accept_len", torch.int32, (B,), dev)
        next_token = _out(next_token, "next_token", torch.int32, (B,), dev)
    else:
        accept_len = next_token = None
    _check("dflash_path_walk", lib.dflash_path_walk(
        _ptr(topk_logp), _ptr(topk_idx), _ptr(E), _ptr(Msel), _ptr(anchor), _ptr(uniforms),
        float(temperature), B, L, K_TOP, r, V, _ptr(path_tok), _ptr(path_slot), _ptr(path_score),
        _ptr(path_q), _ptr(target), _ptr(accept_len), _ptr(next_token), _ptr(dev_status), _stream(stream)))
    return path_tok, path_slot, path_score, path_q, accept_len, next_token


def dflash_verify_rejection_workspace(B: int, L: int, V: int) -> int:
    return int(lib.dflash_verify_rejection_workspace(B, L, V))


def dflash_verify_rejection(target_logits, temperature, draft, draft_slot, cand_idx, draft_q, u_accept,
                            u_resample, accept_len=None, next_token=None, ws=None, dev_status=None,
                            stream=None):
    """Rejection-sampling verification.  target_logits [B*(L+1), V] f32; draft, draft_slot
    [B, L] i32; cand_idx [B*L, 16] i32; draft_q [B, L, 16] f32; u_accept [B, L] f32;
    u_resample [B] f32.  Returns (accept_len [B] i32, next_token [B] i32)."""
    _need(draft, "draft", torch.int32)
    B, L = draft.shape
    _need(target_logits, "target_logits", torch.float32)
    V = target_logits.shape[1]
    _need(target_logits, "target_logits", torch.float32, (B * (L + 1), V))
    _need(draft_slot, "draft_slot", torch.int32, (B, L))
    _need(cand_idx, "cand_idx", torch.int32, (B * L, K_TOP))
    _need(draft_q, "draft_q", torch.float32, (B, L, K_TOP))
    _need(u_accept, "u_accept", torch.float32, (B, L))
    _need(u_resample, "u_resample", torch.float32, (B,))
    dev = draft.device
    accept_len = _out(accept_len, "accept_len", torch.int32, (B,), dev)
    next_token = _out(next_token, "next_token", torch.int32, (B,), dev)
    if ws is None:
        ws = torch.empty(max(16, dflash_verify_rejection_workspace(B, L, V)), dtype=torch.uint8, device=dev)
    _check("dflash_verify_rejection", lib.dflash_verify_rejection(
        _ptr(target_logits), float(temperature), _ptr(draft), _ptr(draft_slot), _ptr(cand_idx),
        _ptr(draft_q), _ptr(u_accept), _ptr(u_resample), B, L, V, _ptr(accept_len), _ptr(next_token),
        _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))
    return accept_len, next_token


def dflash_ctx_table(Emb, Pab, tab=None, stream=None):
    """A and B of the context-gated scorer for every token: tab [V, 2e] fp32
    = Emb . Pab^T (row v: A(v), then B(v)).  Computed once per weight set."""
    _need(Emb, "Emb", torch.bfloat16)
    V, d = Emb.shape
    _need(Pab, "Pab", torch.bfloat16)
    e = Pab.shape[0] // 2
    _need(Pab, "Pab", torch.bfloat16, (2 * e, d))
    tab = _out(tab, "tab", torch.float32, (V, 2 * e), Emb.device)
    _check("dflash_ctx_table", lib.dflash_ctx_table(_ptr(Emb), _ptr(Pab), V, d, e, _ptr(tab), _stream(stream)))
    return tab


def dflash_ctx_gate(H, Pg, gate=None, stream=None):
    """The context gate before its sigmoid: gate [M, e] fp32 = H . Pg^T."""
    _need(H, "H", torch.bfloat16)
    M, d = H.shape
    _need(Pg, "Pg", torch.bfloat16)
    e = Pg.shape[0]
    _need(Pg, "Pg", torch.bfloat16, (e, d))
    gate = _out(gate, "gate", torch.float32, (M, e), H.device)
    _check("dflash_ctx_gate", lib.dflash_ctx_gate(_ptr(H), _ptr(Pg), M, d, e, _ptr(gate), _stream(stream)))
    return gate


_WALKS = {"maxsum": 0, "greedy": 1, "sample": 2}


def dflash_ctx_walk(topk_logp, topk_idx, anchor, tab, gate, B, L, V, walk="maxsum", uniforms=None,
                    temperature=1.0, want_tables=False, target=None, path_tok=None, path_slot=None,
                    path_score=None, path_q=None, accept_len=None, next_token=None, dev_status=None, stream=None):
    """Scores of the context-gated scorer and a walk from the anchor.  Returns
    (path_tok, path_slot, path_score, path_q or None, tables or None,
    accept_len or None, next_token or None)."""
    _need(topk_logp, "topk_logp", torch.float32, (B * L, K_TOP))
    _need(topk_idx, "topk_idx", torch.int32, (B * L, K_TOP))
    _need(anchor, "anchor", torch.int32, (B,))
    _need(gate, "gate", torch.float32)
    e = gate.shape[1]
    _need(gate, "gate", torch.float32, (B * L, e))
    _need(tab, "tab", torch.float32, (V, 2 * e))
    dev = tab.device
    if walk == "sample":
        _need(uniforms, "uniforms", torch.float32, (B, L))
    path_tok = _out(path_tok, "path_tok", torch.int32, (B, L), dev)
    path_slot = _out(path_slot, "path_slot", torch.int32, (B, L), dev)
    path_score = _out(path_score, "path_score", torch.float32, (B,), dev)
    path_q = _out(path_q, "path_q", torch.float32, (B, L, K_TOP), dev) if walk == "sample" else None
    tables = torch.empty((B, L, K_TOP, K_TOP), dtype=torch.float32, device=dev) if want_tables else None
    if target is not None:
        _need(target, "target", torch.int32, (B, L + 1))
        accept_len = _out(accept_len, "accept_len", torch.int32, (B,), dev)
        next_token = _out(next_token, "next_token", torch.int32, (B,), dev)
    else:
        accept_len = next_token = None
    _check("dflash_ctx_walk", lib.dflash_ctx_walk(
        _ptr(topk_logp), _ptr(topk_idx), _ptr(anchor), _ptr(tab), _ptr(gate), B, L, K_TOP, e, V, _WALKS[walk],
        _ptr(uniforms) if walk == "sample" else None, float(temperature), _ptr(path_tok), _ptr(path_slot),
        _ptr(path_score), _ptr(path_q), _ptr(tables), _ptr(target), _ptr(accept_len), _ptr(next_token),
        _ptr(dev_status), _stream(stream)))
    return path_tok, path_slot, path_score, path_q, tables, accept_len, next_token


RECORD_WORDS = 36   # one partial record: max, sum, 2 unused, 16 values, 16 indices


def dflash_lmhead_topk_records(M: int, V: int, d: int) -> int:
    return int(lib.dflash_lmhead_topk_records(M, V, d))


def dflash_lmhead_topk_partial(H, W, v_offset=0, records=None, dev_status=None, stream=None):
    """Partial records [M, P, 36] (float32 words) of H . W^T over this shard of
    the head, vocabulary indices shifted by v_offset."""
    _need(H, "H", torch.bfloat16)
    _need(W, "W", torch.bfloat16)
    M, d = H.shape
    V = W.shape[0]
    P = dflash_lmhead_topk_records(M, V, d)
    if P <= 0:
        raise DFlashError("dflash_lmhead_topk_records", DFLASH_ERR_INVALID_ARG)
    records = _out(records, "records", torch.float32, (M, P, RECORD_WORDS), H.device)
    _check("dflash_lmhead_topk_partial", lib.dflash_lmhead_topk_partial(
        _ptr(H), _ptr(W), M, V, d, int(v_offset), _ptr(records), records.numel() * 4, _ptr(dev_status),
        _stream(stream)))
    return records


def dflash_lmhead_topk_merge(records, topk_logp=None, topk_idx=None, lse=None, stream=None):
    """records [nrank, M, P, 36] float32 -> (topk_logp [M,16], topk_idx [M,16], lse [M])."""
    _need(records, "records", torch.float32)
    if records.dim() == 3:
        records = records.unsqueeze(0)
    nrank, M, P, w = records.shape
    if w != RECORD_WORDS:
        raise ValueError("records must have 36 words per record")
    topk_logp = _out(topk_logp, "topk_logp", torch.float32, (M, K_TOP), records.device)
    topk_idx = _out(topk_idx, "topk_idx", torch.int32, (M, K_TOP), records.device)
    lse = _out(lse, "lse", torch.float32, (M,), records.device)
    _check("dflash_lmhead_topk_merge", lib.dflash_lmhead_topk_merge(
        _ptr(records), M, P, nrank, K_TOP, _ptr(topk_logp), _ptr(topk_idx), _ptr(lse), _stream(stream)))
    return topk_logp, topk_idx, lse
