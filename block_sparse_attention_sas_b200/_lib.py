"""Python binding of the SAS C-ABI library (libsas_b200.so), through ctypes.

Argument marshalling only: every function takes CUDA tensors, allocates the
outputs (and cached workspaces) with torch, passes raw device pointers, the
sizes and torch's current stream to the C entry point of the same name, and
raises SasError on a non-OK status. All computation happens in the library's
CUDA kernels; there is no other implementation behind these calls, and
importing this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsas_b200.so")

SAS_F32, SAS_BF16 = 0, 1
PHI = {"softmax": 0, "sigmoid": 1, "raw": 2}
GATING = {"inner": 0, "outer": 1}
STATUS = {0: "SAS_OK", 1: "SAS_ERR_INVALID_ARG", 2: "SAS_ERR_UNSUPPORTED", 3: "SAS_ERR_CUDA",
          4: "SAS_ERR_TIMEOUT", 5: "SAS_ERR_WORKSPACE", 6: "SAS_ERR_DEVICE"}


class SasError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")


_i, _f, _p, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/sas.h
SIGNATURES = {
    "sas_status_string": (ctypes.c_char_p, [_i]),
    "sas_version": (_i, []),
    "sas_launch_count": (ctypes.c_uint64, []),
    "sas_gate_topk": (_i, [_p, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "sas_gate_topk_phi": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "sas_attn_fwd_gated": (_i, [_i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _i, _p,
                                _p, _p]),
    "sas_attn_bwd_gated": (_i, [_i, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                _f, _i, _i, _p, _p, _p, _p, _p, _sz, _p]),
    "sas_attn_fwd_res": (_i, [_i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p,
                              _p]),
    "sas_attn_bwd_res": (_i, [_i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                              _f, _p, _p, _p, _p, _p, _sz, _p]),
    "sas_attn_fwd": (_i, [_i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p]),
    "sas_attn_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "sas_attn_bwd": (_i, [_i, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f,
                          _p, _p, _p, _p, _p, _sz, _p]),
    "sas_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "sas_decode": (_i, [_i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p,
                        _sz, _p]),
    "sas_decode_select_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "sas_decode_select": (_i, [_i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p,
                               _p, _p, _sz, _p]),
    "sas_decode_select_pooled_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "sas_decode_select_pooled": (_i, [_i, _p, _p, _p, _p, _f, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                      _f, _p, _p, _p, _p, _sz, _p]),
    "sas_decode_noalloc": (_i, [_i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                _p, _p]),
    "sas_decode_noalloc_max_scratch": (_sz, []),
    "sas_decode_paged_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "sas_decode_paged": (_i, [_i, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                              _i, _i, _i, _f, _p, _p, _sz, _p]),
    "sas_selector_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "sas_selector_scores": (_i, [_i, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _sz, _p]),
    "sas_block_summaries": (_i, [_i, _p, _i, _i, _i, _i, _i, _i, _p, _p]),
    "sas_selector_scores_decode": (_i, [_i, _p, _p, _i, _i, _i, _i, _i, _f, _p, _p]),
    "sas_dense_fwd": (_i, [_i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p]),
    "sas_dense_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "sas_dense_bwd": (_i, [_i, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p,
                           _p, _sz, _p]),
    "sas_dense_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "sas_dense_decode": (_i, [_i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _sz, _p]),
    "sas_get_device_error": (_i, [_p, ctypes.POINTER(ctypes.c_uint32)]),
    "sas_set_wait_limit": (None, [ctypes.c_uint64]),
    "sas_selftest_wait_timeout": (_i, [_p]),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"SAS CUDA library not built: {path} is missing "
                          "(run `python -m block_sparse_attention_sas_b200.build`)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = load_library()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SasError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev=None):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SAS_F32
    if t.dtype == torch.bfloat16:
        return SAS_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


_WS: dict = {}


def _workspace(kind: str, nbytes: int, device, zero: bool) -> torch.Tensor:
    """Cached device workspace (grows on demand; contents never matter)."""
    key = (kind, device.index if device.index is not None else torch.cuda.current_device())
    buf = _WS.get(key)
    if buf is None or buf.numel() < nbytes:
        n = max(nbytes, 256)
        buf = torch.zeros(n, dtype=torch.uint8, device=device) if zero else \
            torch.empty(n, dtype=torch.uint8, device=device)
        _WS[key] = buf
    return buf


# ---------------------------------------------------------------------------

def gate_topk(scores: torch.Tensor, K: int, causal: bool = True, gates=None, idx=None,
              phi: str = "softmax"):
    """Gates [B,Hkv,R,C] fp32 and Top-K indices [B,Hkv,R,K] int32 of `scores`
    (phi: the gate activation, "softmax" for the method, "sigmoid" / "raw"
    for the ablation variants)."""
    _need(scores, "scores", torch.float32)
    B, H, R, C = scores.shape
    if gates is None:
        gates = torch.empty_like(scores)
    if idx is None:
        idx = torch.empty((B, H, R, K), dtype=torch.int32, device=scores.device)
    if phi == "softmax":
        _check("sas_gate_topk", LIB.sas_gate_topk(_ptr(scores), B, H, R, C, int(causal), K,
                                                  _ptr(gates), _ptr(idx), _stream(scores.device)))
    else:
        _check("sas_gate_topk_phi",
               LIB.sas_gate_topk_phi(_ptr(scores), B, H, R, C, int(causal), K, PHI[phi],
                                     _ptr(gates), _ptr(idx), _stream(scores.device)))
    return gates, idx


def attn_fwd(q, k, v, idx, gates, b: int, scale: float = 0.0, o=None, lse=None,
             gating: str = "inner"):
    """Gated sparse forward (gating "inner" is the method's Eq. 9; "outer"
    the ablation variant). Returns (o, lse)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype)
    _need(idx, "idx", torch.int32)
    if gates is not None:
        _need(gates, "gates", torch.float32)
    B, Hq, T, d = q.shape
    Hkv, K = k.shape[1], idx.shape[-1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    if gating == "inner":
        _check("sas_attn_fwd", LIB.sas_attn_fwd(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                                _ptr(gates), B, Hq, Hkv, T, d, b, K, scale,
                                                _ptr(o), _ptr(lse), _stream(q.device)))
    else:
        _check("sas_attn_fwd_gated",
               LIB.sas_attn_fwd_gated(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                      _ptr(gates), B, Hq, Hkv, T, d, b, K, scale, GATING[gating],
                                      _ptr(o), _ptr(lse), _stream(q.device)))
    return o, lse


def attn_bwd(q, k, v, o, lse, dO, idx, gates, b: int, scale: float = 0.0,
             want_dscores: bool = True, phi: str = "softmax", gating: str = "inner"):
    """Backward (phi and gating as passed to gate_topk and attn_fwd).
    Returns (dq, dk, dv, dscores or None)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO)):
        _need(t, n, q.dtype)
    _need(lse, "lse", torch.float32)
    _need(idx, "idx", torch.int32)
    B, Hq, T, d = q.shape
    Hkv, K = k.shape[1], idx.shape[-1]
    N = (T + b - 1) // b
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = None
    if gates is not None and want_dscores:
        ds = torch.empty((B, Hkv, N, N), dtype=torch.float32, device=q.device)
    nbytes = LIB.sas_attn_bwd_workspace_size(_dtype(q), B, Hq, Hkv, T, d, b, K)
    ws = _workspace("bwd", nbytes, q.device, zero=False)
    if phi == "softmax" and gating == "inner":
        _check("sas_attn_bwd", LIB.sas_attn_bwd(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                                _ptr(lse), _ptr(dO), _ptr(idx), _ptr(gates), B,
                                                Hq, Hkv, T, d, b, K, scale, _ptr(dq), _ptr(dk),
                                                _ptr(dv), _ptr(ds), _ptr(ws), ws.numel(),
                                                _stream(q.device)))
    else:
        _check("sas_attn_bwd_gated",
               LIB.sas_attn_bwd_gated(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      _ptr(dO), _ptr(idx), _ptr(gates), B, Hq, Hkv, T, d, b, K,
                                      scale, PHI[phi], GATING[gating], _ptr(dq), _ptr(dk),
                                      _ptr(dv), _ptr(ds), _ptr(ws), ws.numel(),
                                      _stream(q.device)))
    return dq, dk, dv, ds


def attn_fwd_res(q, k, v, idx, gates, b: int, scale: float = 0.0):
    """Forward that also returns o's residual (o + o_res = the fp32 output).
    Returns (o, o_res, lse); tensor-core shapes only."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype)
    _need(idx, "idx", torch.int32)
    if gates is not None:
        _need(gates, "gates", torch.float32)
    B, Hq, T, d = q.shape
    Hkv, K = k.shape[1], idx.shape[-1]
    o, o_res = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    _check("sas_attn_fwd_res",
           LIB.sas_attn_fwd_res(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(gates), B,
                                Hq, Hkv, T, d, b, K, scale, _ptr(o), _ptr(o_res), _ptr(lse),
                                _stream(q.device)))
    return o, o_res, lse


def attn_bwd_res(q, k, v, o, o_res, lse, dO, idx, gates, b: int, scale: float = 0.0,
                 want_dscores: bool = True):
    """Backward with D from o and its residual. Returns (dq, dk, dv, dscores or None)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("o_res", o_res), ("dO", dO)):
        _need(t, n, q.dtype)
    _need(lse, "lse", torch.float32)
    _need(idx, "idx", torch.int32)
    B, Hq, T, d = q.shape
    Hkv, K = k.shape[1], idx.shape[-1]
    N = (T + b - 1) // b
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = None
    if gates is not None and want_dscores:
        ds = torch.empty((B, Hkv, N, N), dtype=torch.float32, device=q.device)
    nbytes = LIB.sas_attn_bwd_workspace_size(_dtype(q), B, Hq, Hkv, T, d, b, K)
    ws = _workspace("bwd", nbytes, q.device, zero=False)
    _check("sas_attn_bwd_res",
           LIB.sas_attn_bwd_res(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o_res),
                                _ptr(lse), _ptr(dO), _ptr(idx), _ptr(gates), B, Hq, Hkv, T, d, b,
                                K, scale, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds), _ptr(ws),
                                ws.numel(), _stream(q.device)))
    return dq, dk, dv, ds


def decode(q, kcache, vcache, idx, gates, use_gates: bool, b: int, L: int | None = None,
           scale: float = 0.0, o=None):
    """One-token sparse decode. q [B,Hq,d]; caches [B,Hkv,Lcap,d]; idx [B,Hkv,K]."""
    for n, t in (("q", q), ("kcache", kcache), ("vcache", vcache)):
        _need(t, n, q.dtype)
    _need(idx, "idx", torch.int32)
    B, Hq, d = q.shape
    Hkv, Lcap = kcache.shape[1], kcache.shape[2]
    L = Lcap if L is None else L
    K = idx.shape[-1]
    if o is None:
        o = torch.empty_like(q)
    nbytes = LIB.sas_decode_workspace_size(B, Hq, Hkv, L, d, b, K)
    ws = _workspace("decode", nbytes, q.device, zero=False)
    _check("sas_decode", LIB.sas_decode(_dtype(q), _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(idx),
                                        _ptr(gates), int(use_gates), B, Hq, Hkv, L, Lcap, d, b, K,
                                        scale, _ptr(o), _ptr(ws), ws.numel(), _stream(q.device)))
    return o


def decode_select(q, kcache, vcache, scores, K: int, use_gates: bool, b: int,
                  L: int | None = None, scale: float = 0.0, o=None, gates=None, idx=None):
    """One decode step from the selector scores [B,Hkv,C] (C = (L-1)//b):
    gates and Top-K, then the decode; one launch where the shape allows.
    gates [B,Hkv,C] / idx [B,Hkv,K], when given, receive the selection."""
    for n, t in (("q", q), ("kcache", kcache), ("vcache", vcache)):
        _need(t, n, q.dtype)
    _need(scores, "scores", torch.float32)
    B, Hq, d = q.shape
    Hkv, Lcap = kcache.shape[1], kcache.shape[2]
    L = Lcap if L is None else L
    if o is None:
        o = torch.empty_like(q)
    if gates is not None:
        _need(gates, "gates", torch.float32)
    if idx is not None:
        _need(idx, "idx", torch.int32)
    nbytes = LIB.sas_decode_select_workspace_size(B, Hq, Hkv, L, d, b, K)
    ws = _workspace("decode_select", nbytes, q.device, zero=False)
    _check("sas_decode_select",
           LIB.sas_decode_select(_dtype(q), _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(scores),
                                 int(use_gates), B, Hq, Hkv, L, Lcap, d, b, K, scale, _ptr(o),
                                 _ptr(gates), _ptr(idx), _ptr(ws), ws.numel(),
                                 _stream(q.device)))
    return o


def decode_select_pooled(q, kcache, vcache, kbar, K: int, use_gates: bool, b: int,
                         L: int | None = None, scale: float = 0.0, sel_scale: float = 0.0,
                         o=None, gates=None, idx=None):
    """decode_select with the pooled selector's scores formed from the key
    summaries kbar [B,Hkv,C,d] (fp32) and the query: one launch where the
    shape allows."""
    for n, t in (("q", q), ("kcache", kcache), ("vcache", vcache)):
        _need(t, n, q.dtype)
    B, Hq, d = q.shape
    Hkv, Lcap = kcache.shape[1], kcache.shape[2]
    L = Lcap if L is None else L
    if kbar is not None:  # None: the library reports the missing summaries
        _need(kbar, "kbar", torch.float32)
        if tuple(kbar.shape) != (B, Hkv, (L - 1) // b, d):
            raise ValueError(f"kbar must be [B, Hkv, (L-1)//b, d], got {tuple(kbar.shape)}")
    if o is None:
        o = torch.empty_like(q)
    if gates is not None:
        _need(gates, "gates", torch.float32)
    if idx is not None:
        _need(idx, "idx", torch.int32)
    nbytes = LIB.sas_decode_select_pooled_workspace_size(B, Hq, Hkv, L, d, b, K)
    ws = _workspace("decode_select", nbytes, q.device, zero=False)
    _check("sas_decode_select_pooled",
           LIB.sas_decode_select_pooled(_dtype(q), _ptr(q), _ptr(kcache), _ptr(vcache),
                                        _ptr(kbar), sel_scale, int(use_gates), B, Hq, Hkv, L,
                                        Lcap, d, b, K, scale, _ptr(o), _ptr(gates), _ptr(idx),
                                        _ptr(ws), ws.numel(), _stream(q.device)))
    return o


def decode_noalloc(q, kcache, vcache, idx, gates, use_gates: bool, b: int,
                   L: int | None = None, scale: float = 0.0, o=None):
    """sas_decode without a workspace: the library's fixed device scratch is
    used instead (see include/sas.h for who needs this and its limits)."""
    for n, t in (("q", q), ("kcache", kcache), ("vcache", vcache)):
        _need(t, n, q.dtype)
    _need(idx, "idx", torch.int32)
    B, Hq, d = q.shape
    Hkv, Lcap = kcache.shape[1], kcache.shape[2]
    L = Lcap if L is None else L
    if o is None:
        o = torch.empty_like(q)
    _check("sas_decode_noalloc",
           LIB.sas_decode_noalloc(_dtype(q), _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(idx),
                                  _ptr(gates), int(use_gates), B, Hq, Hkv, L, Lcap, d, b,
                                  idx.shape[-1], scale, _ptr(o), _stream(q.device)))
    return o


def decode_paged(q, kpages, vpages, page_indptr, page_indices, seq_lens, idx, gates,
                 use_gates: bool, b: int, max_len: int, scale: float = 0.0, o=None):
    """Sparse decode over a paged cache: q [B,Hq,d]; pages [num_pages,Hkv,P,d];
    page_indptr [B+1], page_indices, seq_lens [B], idx [B,Hkv,K] int32;
    gates [B,Hkv,(max_len-1)//b] fp32 or None."""
    for n, t in (("q", q), ("kpages", kpages), ("vpages", vpages)):
        _need(t, n, q.dtype)
    for n, t in (("page_indptr", page_indptr), ("page_indices", page_indices),
                 ("seq_lens", seq_lens), ("idx", idx)):
        _need(t, n, torch.int32)
    B, Hq, d = q.shape
    num_pages, Hkv, P = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    K = idx.shape[-1]
    if o is None:
        o = torch.empty_like(q)
    nbytes = LIB.sas_decode_paged_workspace_size(B, Hq, Hkv, max_len, d, b, K)
    ws = _workspace("decode", nbytes, q.device, zero=False)
    _check("sas_decode_paged",
           LIB.sas_decode_paged(_dtype(q), _ptr(q), _ptr(kpages), _ptr(vpages), _ptr(page_indptr),
                                _ptr(page_indices), _ptr(seq_lens), _ptr(idx), _ptr(gates),
                                int(use_gates), B, Hq, Hkv, num_pages, P, max_len, d, b, K, scale,
                                _ptr(o), _ptr(ws), ws.numel(), _stream(q.device)))
    return o


def selector_scores(q, k, b: int, scale: float = 0.0):
    """Pooled-summary selector scores [B,Hkv,N,N] fp32 of q [B,Hq,T,d], k [B,Hkv,T,d]."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    N = (T + b - 1) // b
    s = torch.empty((B, Hkv, N, N), dtype=torch.float32, device=q.device)
    nbytes = LIB.sas_selector_workspace_size(B, Hkv, T, d, b)
    ws = _workspace("selector", nbytes, q.device, zero=False)
    _check("sas_selector_scores",
           LIB.sas_selector_scores(_dtype(q), _ptr(q), _ptr(k), B, Hq, Hkv, T, d, b, scale,
                                   _ptr(s), _ptr(ws), ws.numel(), _stream(q.device)))
    return s


def block_summaries(kcache, b: int, L: int | None = None):
    """Mean key of each full history block of a cache [B,Hkv,Lcap,d] -> [B,Hkv,C,d] fp32."""
    _need(kcache, "kcache")
    B, Hkv, Lcap, d = kcache.shape
    L = Lcap if L is None else L
    C = (L - 1) // b
    kbar = torch.empty((B, Hkv, C, d), dtype=torch.float32, device=kcache.device)
    _check("sas_block_summaries",
           LIB.sas_block_summaries(_dtype(kcache), _ptr(kcache), B, Hkv, L, Lcap, d, b,
                                   _ptr(kbar), _stream(kcache.device)))
    return kbar


def selector_scores_decode(q, kbar, scale: float = 0.0):
    """Decode selector scores [B,Hkv,C] of q [B,Hq,d] against kbar [B,Hkv,C,d]."""
    _need(q, "q")
    _need(kbar, "kbar", torch.float32)
    B, Hq, d = q.shape
    Hkv, C = kbar.shape[1], kbar.shape[2]
    s = torch.empty((B, Hkv, C), dtype=torch.float32, device=q.device)
    _check("sas_selector_scores_decode",
           LIB.sas_selector_scores_decode(_dtype(q), _ptr(q), _ptr(kbar), B, Hq, Hkv, C, d,
                                          scale, _ptr(s), _stream(q.device)))
    return s


def dense_fwd(q, k, v, b: int = 64, scale: float = 0.0):
    B, Hq, T, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    _check("sas_dense_fwd", LIB.sas_dense_fwd(_dtype(q), _ptr(q), _ptr(k), _ptr(v), B, Hq,
                                              k.shape[1], T, d, b, scale, _ptr(o), _ptr(lse),
                                              _stream(q.device)))
    return o, lse


def dense_bwd(q, k, v, o, lse, dO, b: int = 64, scale: float = 0.0):
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = LIB.sas_dense_bwd_workspace_size(B, Hq, Hkv, T, d, b)
    ws = _workspace("bwd", nbytes, q.device, zero=False)
    _check("sas_dense_bwd", LIB.sas_dense_bwd(_dtype(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                              _ptr(lse), _ptr(dO), B, Hq, Hkv, T, d, b, scale,
                                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                              _stream(q.device)))
    return dq, dk, dv


def dense_decode(q, kcache, vcache, L: int | None = None, scale: float = 0.0):
    B, Hq, d = q.shape
    Hkv, Lcap = kcache.shape[1], kcache.shape[2]
    L = Lcap if L is None else L
    o = torch.empty_like(q)
    nbytes = LIB.sas_dense_decode_workspace_size(B, Hq, Hkv, L, d)
    ws = _workspace("dense_decode", nbytes, q.device, zero=False)
    _check("sas_dense_decode", LIB.sas_dense_decode(_dtype(q), _ptr(q), _ptr(kcache), _ptr(vcache),
                                                    B, Hq, Hkv, L, Lcap, d, scale, _ptr(o),
                                                    _ptr(ws), ws.numel(), _stream(q.device)))
    return o


def device_error(stream=None) -> tuple[int, int]:
    """(status, raw bits) of the current device's error word; clears it."""
    raw = ctypes.c_uint32(0)
    st = LIB.sas_get_device_error(stream if stream is not None else _stream(), ctypes.byref(raw))
    return st, raw.value


def launch_count() -> int:
    """Kernels launched through the library so far in this process."""
    return int(LIB.sas_launch_count())


def set_wait_limit(iterations: int) -> None:
    LIB.sas_set_wait_limit(iterations)


def selftest_wait_timeout() -> None:
    _check("sas_selftest_wait_timeout", LIB.sas_selftest_wait_timeout(_stream()))
