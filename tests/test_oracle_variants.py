"""Pins of the oracle's gate variants (the pages' ablation axes): the gate
activations phi = sigmoid and raw logits, and outer gating.

Pinned against things other than the oracle's own formulas:
* sigmoid gates against scipy's logistic function (a library routine);
* raw-logit gates: the log gate is the score, bit for bit;
* with every gate at 1, outer gating is ungated block-sparse attention,
  checked against torch's scaled_dot_product_attention with a block mask;
* central finite differences of sum(o * dO) in float64 for every phi, inner
  and outer, with the selection held fixed (q, k, v and the scores);
* torch autograd through a masked-dense outer-gated formulation;
* Eq. 5 (outer form) term by term: dg_m = sum_i p_i dO^T v_i.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O


def _cfg(**kw):
    base = dict(B=1, Hq=2, Hkv=1, T=32, d=8, b=8, K=2)
    base.update(kw)
    return W.small_train_config(**base)


# ----------------------------------------------------------------- phi

def test_sigmoid_gates_are_the_logistic_function():
    x = W.make_train_inputs(_cfg(T=64))
    g, lg, idx = O.gate_topk_phi(x.scores, 2, "sigmoid")
    _, _, idx0 = O.gate_topk(x.scores, 2)
    np.testing.assert_array_equal(idx, idx0)  # Top-K is over the scores whatever phi
    N = x.scores.shape[-1]
    assert (g[0, 0, 0] == 0).all()  # row 0 has no history
    for j in range(1, N):
        ref = scipy.special.expit(x.scores[0, 0, j, :j].astype(np.float64))
        assert np.abs(g[0, 0, j, :j] - ref).max() < 1e-15
        assert (g[0, 0, j, j:] == 0).all()
        assert (lg[0, 0, j, :j] < 0).all()


def test_raw_log_gates_are_the_scores():
    x = W.make_train_inputs(_cfg(T=64))
    _, lg, _ = O.gate_topk_phi(x.scores, 2, "raw")
    N = x.scores.shape[-1]
    for j in range(N):
        np.testing.assert_array_equal(lg[0, 0, j, :j], x.scores[0, 0, j, :j].astype(np.float64))


def _fd_check(loss, arrays, grads, s, ds, N, h=1e-6, n_each=10, tol=1e-6):
    rng = np.random.default_rng(1)
    for name, arr, grad in zip(("q", "k", "v"), arrays, grads):
        for _ in range(n_each):
            pos = tuple(int(rng.integers(0, n)) for n in arr.shape)
            p, m = arr.copy(), arr.copy()
            p[pos] += h
            m[pos] -= h
            fd = (loss(**{name: p}) - loss(**{name: m})) / (2 * h)
            assert abs(fd - grad[pos]) <= tol * max(1.0, abs(grad[pos])), (name, pos, fd, grad[pos])
    for j in range(1, N):
        for kk in range(j):
            p, m = s.copy(), s.copy()
            p[0, 0, j, kk] += h
            m[0, 0, j, kk] -= h
            fd = (loss(s=p) - loss(s=m)) / (2 * h)
            assert abs(fd - ds[0, 0, j, kk]) <= tol * max(1.0, abs(ds[0, 0, j, kk])), (j, kk, fd)


@pytest.mark.parametrize("phi", O.PHIS)
def test_inner_gating_finite_differences(phi):
    cfg = _cfg()
    x = W.make_train_inputs(cfg)
    q, k, v, dO = (a.astype(np.float64) for a in (x.q, x.k, x.v, x.dO))
    s = x.scores.astype(np.float64)
    _, _, idx = O.gate_topk(x.scores, cfg.K)
    dq, dk, dv, ds = O.attn_bwd_phi(q, k, v, dO, idx, s, cfg.b, phi)

    def loss(**over):
        a = dict(q=q, k=k, v=v, s=s)
        a.update(over)
        _, logg, _ = O.gate_topk_phi(a["s"], cfg.K, phi)
        o, _ = O.attn_fwd(a["q"], a["k"], a["v"], idx, logg, cfg.b)
        return (o * dO).sum()

    _fd_check(loss, (q, k, v), (dq, dk, dv), s, ds, cfg.N)


@pytest.mark.parametrize("phi", O.PHIS)
def test_outer_gating_finite_differences(phi):
    cfg = _cfg()
    x = W.make_train_inputs(cfg)
    q, k, v, dO = (a.astype(np.float64) for a in (x.q, x.k, x.v, x.dO))
    s = x.scores.astype(np.float64)
    _, _, idx = O.gate_topk(x.scores, cfg.K)
    dq, dk, dv, ds = O.attn_bwd_outer(q, k, v, dO, idx, s, cfg.b, phi)

    def loss(**over):
        a = dict(q=q, k=k, v=v, s=s)
        a.update(over)
        gates, _, _ = O.gate_topk_phi(a["s"], cfg.K, phi)
        o, _ = O.attn_fwd_outer(a["q"], a["k"], a["v"], idx, gates, cfg.b)
        return (o * dO).sum()

    _fd_check(loss, (q, k, v), (dq, dk, dv), s, ds, cfg.N)


# ----------------------------------------------------------------- outer

def _block_mask(idx, T, b, N):
    """[B,Hkv,T,T] additive mask: 0 on the selected blocks and the causal
    part of the diagonal block, -inf elsewhere."""
    B, H = idx.shape[:2]
    M = np.full((B, H, T, T), -np.inf)
    for bi in range(B):
        for h in range(H):
            for j in range(N):
                r0, r1 = j * b, min(T, (j + 1) * b)
                for m in idx[bi, h, j]:
                    if m >= 0:
                        M[bi, h, r0:r1, m * b:(m + 1) * b] = 0.0
                for i in range(r0, r1):
                    M[bi, h, i, r0:i + 1] = 0.0
    return M


def test_outer_with_unit_gates_is_ungated_sparse_attention():
    cfg = _cfg(B=1, Hq=4, Hkv=2, T=72, d=8, b=8, K=3)
    x = W.make_train_inputs(cfg)
    _, _, idx = O.gate_topk(x.scores, cfg.K)
    ones = np.ones(x.scores.shape)
    o, _ = O.attn_fwd_outer(x.q, x.k, x.v, idx, ones, cfg.b)
    m = torch.from_numpy(_block_mask(idx, cfg.T, cfg.b, cfg.N)).repeat_interleave(cfg.G, 1)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(x.q), t(x.k).repeat_interleave(cfg.G, 1), t(x.v).repeat_interleave(cfg.G, 1), attn_mask=m)
    assert np.abs(o - ref.numpy()).max() < 1e-12


def test_outer_backward_matches_autograd():
    """Autograd through a masked-dense outer-gated attention (softmax of the
    masked logits, weights scaled per column by the selected block's gate, or
    1 on the diagonal block, then times V), with the scores as the leaf."""
    cfg = _cfg(B=1, Hq=2, Hkv=1, T=48, d=8, b=8, K=2)
    x = W.make_train_inputs(cfg)
    _, _, idx = O.gate_topk(x.scores, cfg.K)
    dq, dk, dv, ds = O.attn_bwd_outer(x.q, x.k, x.v, x.dO, idx, x.scores, cfg.b, "softmax")
    T, b, N, G = cfg.T, cfg.b, cfg.N, cfg.G
    t = lambda a: torch.tensor(np.asarray(a, np.float64), requires_grad=True)
    q, k, v, s = t(x.q), t(x.k), t(x.v), t(x.scores)
    mask = torch.from_numpy(_block_mask(idx, T, b, N))
    # column gates from log_softmax over each row's history, selected blocks only
    W_ = torch.ones(1, 1, T, T, dtype=torch.float64)
    rows = []
    for j in range(N):
        g = torch.exp(torch.log_softmax(s[0, 0, j, :j], 0)) if j > 0 else None
        row = torch.ones(T, dtype=torch.float64)
        for m in idx[0, 0, j]:
            if m >= 0:
                row = row.index_put((torch.arange(m * b, (m + 1) * b),), g[m].expand(b))
        rows.append(row.expand(min(T, (j + 1) * b) - j * b, T))
    W_ = torch.cat(rows, 0)[None, None]
    logits = (q @ k.repeat_interleave(G, 1).transpose(-1, -2)) / math.sqrt(cfg.d) + mask
    P = torch.softmax(logits, -1)
    o = (P * W_) @ v.repeat_interleave(G, 1)
    (o * torch.from_numpy(x.dO.astype(np.float64))).sum().backward()
    assert np.abs(q.grad.numpy() - dq).max() < 1e-10
    assert np.abs(k.grad.numpy() - dk).max() < 1e-10
    assert np.abs(v.grad.numpy() - dv).max() < 1e-10
    assert np.abs(s.grad.numpy() - ds).max() < 1e-10


def test_eq5_outer_gate_gradient():
    cfg = _cfg(B=1, Hq=2, Hkv=1, T=40, d=8, b=8, K=2)
    x = W.make_train_inputs(cfg)
    gates, _, idx = O.gate_topk(x.scores, cfg.K)
    for j in range(1, cfg.N):
        r = O.attn_bwd_outer_block(x.q, x.k, x.v, x.dO, idx, gates, 0, 0, j, cfg.b)
        lit = O.gate_grad_eq5_outer(x.q, x.k, x.v, x.dO, idx, gates, 0, 0, j, cfg.b)
        for m, dg in lit.items():
            assert abs(r["da"][m] - gates[0, 0, j, m] * dg) <= 1e-12 * max(1.0, abs(r["da"][m]))
