"""sas_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers (a serving process whose framework owns every device
allocation, or a latency-critical loop that cannot pay for cudaMalloc's
implicit synchronisation) cannot hand the library a workspace. For them the
library keeps decode's scratch in a fixed 2 MiB device array. These tests call
that entry point through the C ABI with raw device pointers and check it
against the float64 oracle and against the workspace-taking sas_decode, on
two calls in a row with different inputs, so leftovers of the first call
must not leak into the second. One case runs the tensor-core decode (bf16,
d = 128, b = 64), the other the general decode kernel (fp32, d = 64).

This file is collected last on purpose: a run that stops at the first
failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, host


def test_scratch_limit_covers_the_decode_presets():
    from block_sparse_attention_sas_b200 import _lib as S
    cap = S.LIB.sas_decode_noalloc_max_scratch()
    assert cap == 2 << 20
    for cfg in (W.QWEN3_4B_DECODE, W.QWEN3_14B_DECODE):
        need = S.LIB.sas_decode_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.L, cfg.d, cfg.b, cfg.K)
        assert 0 < need <= cap


def _noalloc(S, dtype_code, q, kc, vc, idx, gates, use_gates, cfg):
    got = torch.full_like(q, float("nan"))
    st = S.LIB.sas_decode_noalloc(
        dtype_code, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
        ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(gates.data_ptr()), use_gates, cfg.B, cfg.Hq, cfg.Hkv, cfg.L, cfg.L,
        cfg.d, cfg.b, cfg.K, 0.0, ctypes.c_void_p(got.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, got


@pytest.mark.gpu
@pytest.mark.parametrize("kw", [
    dict(B=2, Hq=8, Hkv=2, L=5000, d=128, b=64, K=16, dtype="bf16"),   # tensor-core decode
    dict(B=2, Hq=4, Hkv=2, L=3000, d=64, b=32, K=12, dtype="f32"),     # general decode
])
def test_decode_noalloc_matches_oracle_twice(cuda_lib, kw):
    S = cuda_lib
    cfg = W.small_decode_config(**kw)
    code = 1 if cfg.dtype == "bf16" else 0
    for call, (seed, use_gates) in enumerate(((11, 0), (12, 1))):
        x = W.make_decode_inputs(cfg, seed=seed)
        q, kc, vc = (dev(a, cfg.dtype) for a in (x.q, x.kcache, x.vcache))
        s = x.scores[:, :, None, :].copy()
        gates, idx = S.gate_topk(dev(s, "f32"), cfg.K, causal=False)
        idx = idx[:, :, 0].contiguous()
        gates = gates[:, :, 0].contiguous()
        st, got = _noalloc(S, code, q, kc, vc, idx, gates, use_gates, cfg)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert S.device_error()[0] == 0
        _, olg, oi = O.gate_topk(s, cfg.K, causal=False)
        want = O.decode(x.q, x.kcache, x.vcache, oi[:, :, 0], olg[:, :, 0], cfg.b,
                        use_gates=bool(use_gates))
        check(f"decode_noalloc call {call} vs oracle", host(got), want, cfg.dtype)
        ref = S.decode(q, kc, vc, idx, gates, bool(use_gates), cfg.b, L=cfg.L)
        torch.cuda.synchronize()
        check(f"decode_noalloc call {call} vs sas_decode", host(got), host(ref), cfg.dtype)
