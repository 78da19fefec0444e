"""GPU parity of the gate-variant kernels against the float64 oracle.

The ablation axes of the method (evolve.pub review, Summary; picx.dev
summary, Methodology Eq. 4 and Gradient Analysis Eq. 5): the gate activation
phi (softmax, sigmoid, raw logits) and inner versus outer gating. Each case
runs gate + Top-K, the forward and the backward through the C-ABI library
and compares every element with the oracle's variant functions, on the
tensor-core kernels (bf16, d = 128, b = 64, G = 2 and 4) and the general
kernels (fp32).
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, floor_of, host

pytestmark = pytest.mark.gpu

CASES = [
    dict(B=1, Hq=8, Hkv=2, T=1000, d=128, b=64, K=3, dtype="bf16", hot_key_frac=0.1,
         hot_key_scale=3.0),
    dict(B=1, Hq=4, Hkv=2, T=448, d=128, b=64, K=4, dtype="bf16"),
    dict(B=1, Hq=4, Hkv=2, T=200, d=64, b=16, K=3, dtype="f32"),
]


@pytest.mark.parametrize("phi", ["sigmoid", "raw"])
@pytest.mark.parametrize("causal,C,K", [(True, 40, 5), (True, 700, 16), (False, 3000, 32),
                                        (False, 9000, 64)])
def test_gate_topk_phi(cuda_lib, phi, causal, C, K):
    rng = np.random.default_rng(C + K)
    rows = C if causal else 3
    s = (rng.standard_normal((1, 2, rows, C)) * 2).astype(np.float32)
    g, ix = cuda_lib.gate_topk(dev(s, "f32"), K, causal=causal, phi=phi)
    og, _, oi = O.gate_topk_phi(s, K, phi, causal=causal)
    np.testing.assert_array_equal(ix.cpu().numpy(), oi)
    check(f"gates ({phi})", host(g), og, "f32")


def _inputs(kw):
    cfg = W.small_train_config(**kw)
    x = W.make_train_inputs(cfg)
    q, k, v, dO = (dev(a, cfg.dtype) for a in (x.q, x.k, x.v, x.dO))
    return cfg, x, q, k, v, dO


@pytest.mark.parametrize("kw", CASES)
@pytest.mark.parametrize("phi", ["sigmoid", "raw"])
def test_inner_gating_with_phi(cuda_lib, kw, phi):
    cfg, x, q, k, v, dO = _inputs(kw)
    gates, idx = cuda_lib.gate_topk(dev(x.scores, "f32"), cfg.K, phi=phi)
    o, lse = cuda_lib.attn_fwd(q, k, v, idx, gates, cfg.b)
    dq, dk, dv, ds = cuda_lib.attn_bwd(q, k, v, o, lse, dO, idx, gates, cfg.b, phi=phi)
    torch.cuda.synchronize()
    assert cuda_lib.device_error()[0] == 0
    _, lg, ix = O.gate_topk_phi(x.scores, cfg.K, phi)
    np.testing.assert_array_equal(idx.cpu().numpy(), ix)
    oo, ol = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b)
    odq, odk, odv, ods = O.attn_bwd_phi(x.q, x.k, x.v, x.dO, ix, x.scores, cfg.b, phi)
    dt = cfg.dtype
    fl = [None] * 4
    if dt == "bf16":  # the rounding floor of bf16 MMA operands
        oe, _ = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b, operands="bf16")
        e = O.attn_bwd_phi(x.q, x.k, x.v, x.dO, ix, x.scores, cfg.b, phi, operands="bf16")
        fl = [floor_of(oo, oe), floor_of(odq, e[0]), floor_of(odk, e[1]), floor_of(odv, e[2])]
    check("o", host(o), oo, dt, floor=fl[0])
    check("lse", host(lse), ol, dt, stored="f32")
    check("dq", host(dq), odq, dt, floor=fl[1])
    check("dk", host(dk), odk, dt, floor=fl[2])
    check("dv", host(dv), odv, dt, floor=fl[3])
    check(f"dscores ({phi})", host(ds), ods, dt, stored="f32")


@pytest.mark.parametrize("kw", CASES)
@pytest.mark.parametrize("phi", ["softmax", "sigmoid"])
def test_outer_gating(cuda_lib, kw, phi):
    cfg, x, q, k, v, dO = _inputs(kw)
    gates, idx = cuda_lib.gate_topk(dev(x.scores, "f32"), cfg.K, phi=phi)
    o, lse = cuda_lib.attn_fwd(q, k, v, idx, gates, cfg.b, gating="outer")
    dq, dk, dv, ds = cuda_lib.attn_bwd(q, k, v, o, lse, dO, idx, gates, cfg.b, phi=phi,
                                       gating="outer")
    torch.cuda.synchronize()
    assert cuda_lib.device_error()[0] == 0
    og, _, ix = O.gate_topk_phi(x.scores, cfg.K, phi)
    np.testing.assert_array_equal(idx.cpu().numpy(), ix)
    oo, ol = O.attn_fwd_outer(x.q, x.k, x.v, ix, og, cfg.b)
    odq, odk, odv, ods = O.attn_bwd_outer(x.q, x.k, x.v, x.dO, ix, x.scores, cfg.b, phi)
    dt = cfg.dtype
    fl = [None] * 4
    if dt == "bf16":
        oe, _ = O.attn_fwd_outer(x.q, x.k, x.v, ix, og, cfg.b, operands="bf16")
        e = O.attn_bwd_outer(x.q, x.k, x.v, x.dO, ix, x.scores, cfg.b, phi, operands="bf16")
        fl = [floor_of(oo, oe), floor_of(odq, e[0]), floor_of(odk, e[1]), floor_of(odv, e[2])]
    check("o (outer)", host(o), oo, dt, floor=fl[0])
    check("lse (outer)", host(lse), ol, dt, stored="f32")
    check("dq (outer)", host(dq), odq, dt, floor=fl[1])
    check("dk (outer)", host(dk), odk, dt, floor=fl[2])
    check("dv (outer)", host(dv), odv, dt, floor=fl[3])
    check(f"dscores (outer, {phi})", host(ds), ods, dt, stored="f32")


def test_outer_gating_without_gates_is_plain_sparse_attention(cuda_lib):
    cfg, x, q, k, v, dO = _inputs(CASES[1])
    _, idx = cuda_lib.gate_topk(dev(x.scores, "f32"), cfg.K)
    o1, l1 = cuda_lib.attn_fwd(q, k, v, idx, None, cfg.b, gating="outer")
    o2, l2 = cuda_lib.attn_fwd(q, k, v, idx, None, cfg.b)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
