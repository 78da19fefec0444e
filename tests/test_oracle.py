"""Pins for the float64 oracle, against things other than the oracle itself.

Each check below is chosen so that a plausible slip in the oracle (a dropped
bias, a wrong scale, a transposed operand, a wrong sign in the gate Jacobian,
an off-by-one in the causal mask or the history length) fails at least one:

* hand-derived worked examples (tests/golden/hand_cases.json);
* invariants of Eq. 6 (gates sum to one, shift invariance);
* brute-force Top-K (numpy lexsort) including tie-heavy rows;
* library special cases in float64: with every history block selected and
  gates off the method is dense causal attention (torch SDPA); with gates on
  it is SDPA with a block-constant additive mask; in general it is SDPA with
  a -inf mask on the unselected blocks;
* central finite differences of sum(o * dO) with the selection held fixed;
* torch.autograd through the masked-dense route, with the scores as leaf;
* Eq. 5 (inner form) term by term against the backward's da.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))


def _inputs(**kw):
    cfg = W.small_train_config(**kw)
    x = W.make_train_inputs(cfg)
    gates, logg, idx = O.gate_topk(x.scores, cfg.K, causal=True)
    return cfg, x, gates, logg, idx


# ----------------------------------------------------------------- golden cases

def test_golden_gate_softmax():
    for key in ("gate_softmax_uniform", "gate_softmax_ln3"):
        c = GOLD[key]
        s = np.asarray(c["scores"], dtype=np.float32)
        g = np.exp(O.log_gates_row(s, len(s)))
        np.testing.assert_allclose(g, c["gates"], rtol=0, atol=c.get("tol", 1e-15))


def test_golden_topk_ties():
    c = GOLD["topk_ties"]
    s = np.asarray(c["scores"], dtype=np.float32)
    for case in c["cases"]:
        assert O.topk_row(s, case["n"], case["K"]) == case["idx"], case


def test_golden_zero_query_gated():
    c = GOLD["zero_query_gated"]
    T, b, d, K = c["T"], c["b"], c["d"], c["K"]
    q = np.zeros((1, 1, T, d), np.float32)
    k = np.ones((1, 1, T, d), np.float32)
    v = np.asarray(c["v"], np.float32).reshape(1, 1, T, d)
    s = np.asarray(c["scores"], np.float32).reshape(1, 1, 3, 3)
    gates, logg, idx = O.gate_topk(s, K, causal=True)
    o, lse = O.attn_fwd(q, k, v, idx, logg, b)
    np.testing.assert_allclose(o[0, 0, :, 0], c["o"], rtol=0, atol=c["tol"])
    np.testing.assert_allclose(lse[0, 0], c["lse"], rtol=0, atol=c["tol"])
    o2, _ = O.attn_fwd(q, k, v, idx, logg, b, use_gates=False)
    np.testing.assert_allclose(o2[0, 0, :, 0], c["o_gates_off"], rtol=0, atol=c["tol"])


def test_golden_zero_query_decode():
    c = GOLD["zero_query_decode"]
    L, b, d, K = c["L"], c["b"], c["d"], c["K"]
    q = np.zeros((1, 1, d), np.float32)
    kc = np.ones((1, 1, L, d), np.float32)
    vc = np.asarray(c["v"], np.float32).reshape(1, 1, L, d)
    s = np.asarray(c["scores"], np.float32).reshape(1, 1, 1, 2)
    gates, logg, idx = O.gate_topk(s, K, causal=False)
    on = O.decode(q, kc, vc, idx[:, :, 0], logg[:, :, 0], b, use_gates=True)
    off = O.decode(q, kc, vc, idx[:, :, 0], logg[:, :, 0], b, use_gates=False)
    assert abs(on[0, 0, 0] - c["o_gates_on"]) < c["tol"]
    assert abs(off[0, 0, 0] - c["o_gates_off"]) < c["tol"]


def test_golden_scale():
    c = GOLD["scale_two_keys"]
    T, b, d = c["T"], c["b"], c["d"]
    q = np.zeros((1, 1, T, d), np.float32)
    q[0, 0, 1] = c["q_row1"]
    k = np.asarray(c["k"], np.float32).reshape(1, 1, T, d)
    v = np.asarray(c["v"], np.float32).reshape(1, 1, T, d)
    idx = np.full((1, 1, 1, 1), -1, np.int32)
    o, _ = O.attn_fwd(q, k, v, idx, None, b, use_gates=False)
    np.testing.assert_allclose(o[0, 0, 1], c["o_row1"], rtol=0, atol=c["tol"])


# ------------------------------------------------------------ gate invariants

def test_gates_sum_to_one_and_positive():
    cfg, x, gates, logg, idx = _inputs(T=160, b=16, K=3)
    N = cfg.N
    for j in range(1, N):
        row = gates[0, 0, j]
        assert abs(row[:j].sum() - 1.0) < 1e-12
        assert (row[:j] > 0).all() and (row[j:] == 0).all()
        assert np.all(np.isneginf(logg[0, 0, j, j:]))
    assert (gates[0, 0, 0] == 0).all() and (idx[0, 0, 0] == -1).all()


def test_shift_invariance():
    """s + c per row leaves gates, idx, o and dscores unchanged (Eq. 6)."""
    cfg = W.small_train_config(T=96, b=16, K=2, Hq=2, Hkv=1, d=8)
    x = W.make_train_inputs(cfg)
    s1 = (np.round(x.scores * 8) / 8).astype(np.float32)     # exact under +3
    s2 = (s1 + np.float32(3.0)).astype(np.float32)
    g1, l1, i1 = O.gate_topk(s1, cfg.K)
    g2, l2, i2 = O.gate_topk(s2, cfg.K)
    assert (i1 == i2).all()
    np.testing.assert_allclose(g1, g2, rtol=0, atol=1e-14)
    o1, _ = O.attn_fwd(x.q, x.k, x.v, i1, l1, cfg.b)
    o2, _ = O.attn_fwd(x.q, x.k, x.v, i2, l2, cfg.b)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    r1 = O.attn_bwd(x.q, x.k, x.v, x.dO, i1, g1, l1, cfg.b)
    r2 = O.attn_bwd(x.q, x.k, x.v, x.dO, i2, g2, l2, cfg.b)
    for a, c in zip(r1, r2):
        np.testing.assert_allclose(a, c, rtol=0, atol=1e-11)


# ------------------------------------------------------------------ Top-K

@pytest.mark.parametrize("levels", [None, 3, 1])
def test_topk_brute_force(levels):
    rng = np.random.default_rng(1)
    for trial in range(200):
        n = int(rng.integers(0, 40))
        K = int(rng.integers(1, 12))
        s = rng.standard_normal(n).astype(np.float32)
        if levels:
            s = rng.integers(0, levels, n).astype(np.float32)
        got = O.topk_row(s, n, K)
        order = np.lexsort((np.arange(n), -s.astype(np.float64)))
        want = list(order[:min(K, n)]) + [-1] * (K - min(K, n))
        assert got == want


def test_topk_all_equal_rows():
    s = np.full((1, 1, 10, 10), 0.5, np.float32)
    _, _, idx = O.gate_topk(s, 4)
    for j in range(10):
        n = min(4, j)
        assert list(idx[0, 0, j, :n]) == list(range(n))
        assert (idx[0, 0, j, n:] == -1).all()


# ---------------------------------------------- library special cases (SDPA)

def _t(a):
    return torch.from_numpy(np.asarray(a, np.float64))


def _block_bias(idx, logg, T, b, use_gates, N):
    """Full [B,Hkv,T,T] additive mask: lg (or 0) on selected blocks, 0 on the
    causal part of the diagonal block, -inf elsewhere."""
    B, H = idx.shape[:2]
    M = np.full((B, H, T, T), -np.inf)
    for bi in range(B):
        for h in range(H):
            for j in range(N):
                r0, r1 = j * b, min(T, (j + 1) * b)
                for m in idx[bi, h, j]:
                    if m < 0:
                        continue
                    M[bi, h, r0:r1, m * b:(m + 1) * b] = logg[bi, h, j, m] if use_gates else 0.0
                for i in range(r0, r1):
                    M[bi, h, i, r0:i + 1] = 0.0
    return M


def _sdpa(q, k, v, mask, G, scale=None):
    qt, kt, vt = _t(q), _t(k), _t(v)
    kt = kt.repeat_interleave(G, dim=1)
    vt = vt.repeat_interleave(G, dim=1)
    m = torch.from_numpy(mask).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)


def test_fwd_reduces_to_dense_causal():
    """Gates off and every history block selected: dense causal attention."""
    cfg = W.small_train_config(B=2, Hq=4, Hkv=2, T=80, d=16, b=16, K=8)
    x = W.make_train_inputs(cfg)
    _, logg, idx = O.gate_topk(x.scores, cfg.K)
    o, lse = O.attn_fwd(x.q, x.k, x.v, idx, logg, cfg.b, use_gates=False)
    ref = torch.nn.functional.scaled_dot_product_attention(
        _t(x.q), _t(x.k).repeat_interleave(2, 1), _t(x.v).repeat_interleave(2, 1), is_causal=True)
    assert np.abs(o - ref.numpy()).max() < 1e-12
    od, _ = O.dense_fwd(x.q, x.k, x.v, cfg.b)
    assert np.abs(od - ref.numpy()).max() < 1e-12
    # lse against its definition on the dense causal logits
    qk = np.einsum("bhid,bhjd->bhij", x.q.astype(np.float64),
                   np.repeat(x.k, 2, 1).astype(np.float64)) / math.sqrt(cfg.d)
    qk = np.where(np.tril(np.ones((80, 80), bool)), qk, -np.inf)
    mx = qk.max(-1, keepdims=True)
    assert np.abs(lse - (mx + np.log(np.exp(qk - mx).sum(-1, keepdims=True)))[..., 0]).max() < 1e-12


def test_fwd_gates_on_all_selected_is_block_masked_sdpa():
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=96, d=16, b=16, K=8)
    x = W.make_train_inputs(cfg)
    _, logg, idx = O.gate_topk(x.scores, cfg.K)
    o, _ = O.attn_fwd(x.q, x.k, x.v, idx, logg, cfg.b)
    mask = _block_bias(idx, logg, cfg.T, cfg.b, True, cfg.N)
    ref = _sdpa(x.q, x.k, x.v, mask, cfg.G)
    assert np.abs(o - ref.numpy()).max() < 1e-12


@pytest.mark.parametrize("T,b,K", [(128, 16, 3), (100, 16, 2), (72, 8, 4)])
def test_fwd_general_matches_masked_dense(T, b, K):
    cfg = W.small_train_config(B=1, Hq=3, Hkv=1, T=T, d=8, b=b, K=K)
    x = W.make_train_inputs(cfg)
    _, logg, idx = O.gate_topk(x.scores, K)
    for gates_on in (True, False):
        o, _ = O.attn_fwd(x.q, x.k, x.v, idx, logg, b, use_gates=gates_on)
        mask = _block_bias(idx, logg, T, b, gates_on, cfg.N)
        ref = _sdpa(x.q, x.k, x.v, mask, cfg.G)
        assert np.abs(o - ref.numpy()).max() < 1e-12


# ------------------------------------------------------------------ backward

def _loss_from_scores(x, s64, idx, b, dO):
    """sum(o * dO) with log-gates computed from float64 scores (idx fixed)."""
    B, H, N, _ = s64.shape
    logg = np.full(s64.shape, -np.inf)
    for bi in range(B):
        for h in range(H):
            for j in range(N):
                logg[bi, h, j, :j] = O.log_gates_row(s64[bi, h, j], j)
    o, _ = O.attn_fwd(x.q, x.k, x.v, idx, logg, b)
    return (o * dO).sum()


def test_bwd_finite_differences():
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=32, d=8, b=8, K=2)
    x = W.make_train_inputs(cfg)
    q, k, v, dO = (a.astype(np.float64) for a in (x.q, x.k, x.v, x.dO))
    s = x.scores.astype(np.float64)
    gates, logg, idx = O.gate_topk(x.scores, cfg.K)
    dq, dk, dv, ds = O.attn_bwd(q, k, v, dO, idx, gates, logg, cfg.b)
    h = 1e-6

    def loss(**over):
        a = dict(q=q, k=k, v=v, s=s)
        a.update(over)
        x2 = W.TrainInputs(a["q"], a["k"], a["v"], dO, a["s"])
        return _loss_from_scores(x2, a["s"], idx, cfg.b, dO)

    rng = np.random.default_rng(0)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            pos = tuple(int(rng.integers(0, n)) for n in arr.shape)
            p, m = arr.copy(), arr.copy()
            p[pos] += h
            m[pos] -= h
            fd = (loss(**{name: p}) - loss(**{name: m})) / (2 * h)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(grad[pos])), (name, pos, fd, grad[pos])
    for j in range(1, cfg.N):
        for kk in range(j):
            p, m = s.copy(), s.copy()
            p[0, 0, j, kk] += h
            m[0, 0, j, kk] -= h
            fd = (loss(s=p) - loss(s=m)) / (2 * h)
            assert abs(fd - ds[0, 0, j, kk]) <= 1e-6 * max(1.0, abs(ds[0, 0, j, kk])), (j, kk)
    assert (ds[0, 0][np.triu_indices(cfg.N)] == 0).all()


def test_bwd_matches_autograd_masked_dense():
    cfg = W.small_train_config(B=1, Hq=4, Hkv=2, T=64, d=8, b=8, K=3)
    x = W.make_train_inputs(cfg)
    gates, logg, idx = O.gate_topk(x.scores, cfg.K)
    dq, dk, dv, ds = O.attn_bwd(x.q, x.k, x.v, x.dO, idx, gates, logg, cfg.b)
    qt = _t(x.q).requires_grad_()
    kt = _t(x.k).requires_grad_()
    vt = _t(x.v).requires_grad_()
    st = _t(x.scores).requires_grad_()
    T, b, N, G = cfg.T, cfg.b, cfg.N, cfg.G
    rows = []
    for j in range(N):
        if j == 0:
            rows.append(torch.full((2, N), float("-inf"), dtype=torch.float64))
            continue
        lg = torch.log_softmax(st[0, :, j, :j], dim=-1)
        rows.append(torch.cat([lg, torch.full((2, N - j), float("-inf"), dtype=torch.float64)], 1))
    LG = torch.stack(rows, 1)  # [Hkv, N, N]
    sel = np.zeros((2, N, N), bool)
    for h in range(2):
        for j in range(N):
            for m in idx[0, h, j]:
                if m >= 0:
                    sel[h, j, m] = True
    selt = torch.from_numpy(sel)
    blockbias = torch.where(selt, LG, torch.full_like(LG, float("-inf")))
    full = blockbias.repeat_interleave(b, 1).repeat_interleave(b, 2)[:, :T, :T]
    diag = torch.from_numpy(np.kron(np.eye(N), np.ones((b, b)))[:T, :T].astype(bool))
    causal = torch.from_numpy(np.tril(np.ones((T, T), bool)))
    full = torch.where(diag & causal, torch.zeros_like(full), full)
    full = torch.where(diag & ~causal, torch.full_like(full, float("-inf")), full)
    m = full.repeat_interleave(G, 0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(G, 1), vt.repeat_interleave(G, 1), attn_mask=m)
    (o * _t(x.dO)).sum().backward()
    assert np.abs(qt.grad.numpy() - dq).max() < 1e-10
    assert np.abs(kt.grad.numpy() - dk).max() < 1e-10
    assert np.abs(vt.grad.numpy() - dv).max() < 1e-10
    assert np.abs(st.grad.numpy() - ds).max() < 1e-10


def test_dscores_rows_sum_to_zero():
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=128, d=8, b=16, K=3)
    x = W.make_train_inputs(cfg)
    gates, logg, idx = O.gate_topk(x.scores, cfg.K)
    _, _, _, ds = O.attn_bwd(x.q, x.k, x.v, x.dO, idx, gates, logg, cfg.b)
    scale = np.abs(ds).max()
    for j in range(1, cfg.N):
        assert abs(ds[0, 0, j].sum()) < 1e-12 * max(1.0, scale)


def test_eq5_inner_gate_gradient():
    """g_m * dg_m (Eq. 5, inner form, written literally) equals da_m."""
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=96, d=8, b=16, K=3)
    x = W.make_train_inputs(cfg)
    gates, logg, idx = O.gate_topk(x.scores, cfg.K)
    for j in range(1, cfg.N):
        r = O.attn_bwd_block(x.q, x.k, x.v, x.dO, idx, logg, 0, 0, j, cfg.b)
        dg = O.gate_grad_eq5(x.q, x.k, x.v, x.dO, idx, gates, logg, 0, 0, j, cfg.b)
        assert set(dg) == set(r["da"])
        for m in dg:
            assert abs(gates[0, 0, j, m] * dg[m] - r["da"][m]) < 1e-11


def test_gates_off_bwd_is_dense_causal_grad():
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=48, d=8, b=16, K=4)
    x = W.make_train_inputs(cfg)
    gates, logg, idx = O.gate_topk(x.scores, cfg.K)
    dq, dk, dv, ds = O.attn_bwd(x.q, x.k, x.v, x.dO, idx, gates, logg, cfg.b, use_gates=False)
    assert (ds == 0).all()
    qt, kt, vt = (_t(a).requires_grad_() for a in (x.q, x.k, x.v))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(2, 1), vt.repeat_interleave(2, 1), is_causal=True)
    (o * _t(x.dO)).sum().backward()
    assert np.abs(qt.grad.numpy() - dq).max() < 1e-11
    assert np.abs(kt.grad.numpy() - dk).max() < 1e-11
    assert np.abs(vt.grad.numpy() - dv).max() < 1e-11


# -------------------------------------------------------------------- decode

@pytest.mark.parametrize("L", [97, 96, 17, 16])
def test_decode_is_last_row_of_forward(L):
    """Decode over a cache equals row L-1 of the training-layout forward with
    the same selection for the block holding L-1."""
    b, K, d = 16, 2, 8
    dc = W.small_decode_config(B=2, Hq=4, Hkv=2, L=L, d=d, b=b, K=K)
    x = W.make_decode_inputs(dc)
    C = dc.C
    gates, logg, idx = O.gate_topk(x.scores[:, :, None, :], K, causal=False)
    for use_gates in (False, True):
        o_dec = O.decode(x.q, x.kcache, x.vcache, idx[:, :, 0], logg[:, :, 0], b,
                         use_gates=use_gates)
        N = (L + b - 1) // b
        q = np.zeros((2, 4, L, d), np.float32)
        q[:, :, L - 1] = x.q
        tidx = np.full((2, 2, N, K), -1, np.int32)
        tidx[:, :, C] = idx[:, :, 0]
        tlogg = np.full((2, 2, N, N), -np.inf)
        tlogg[:, :, C, :C] = logg[:, :, 0, :C]
        o_fwd, _ = O.attn_fwd(q, x.kcache, x.vcache, tidx, tlogg, b, use_gates=use_gates)
        assert np.abs(o_fwd[:, :, L - 1] - o_dec).max() < 1e-12


def test_dense_decode_matches_sdpa_and_full_selection():
    dc = W.small_decode_config(B=2, Hq=4, Hkv=2, L=70, d=8, b=16, K=8)
    x = W.make_decode_inputs(dc)
    od = O.dense_decode(x.q, x.kcache, x.vcache)
    ref = torch.nn.functional.scaled_dot_product_attention(
        _t(x.q)[:, :, None], _t(x.kcache).repeat_interleave(2, 1),
        _t(x.vcache).repeat_interleave(2, 1))[:, :, 0]
    assert np.abs(od - ref.numpy()).max() < 1e-12
    gates, logg, idx = O.gate_topk(x.scores[:, :, None, :], dc.K, causal=False)
    osp = O.decode(x.q, x.kcache, x.vcache, idx[:, :, 0], logg[:, :, 0], dc.b, use_gates=False)
    assert np.abs(osp - od).max() < 1e-12


def test_attended_pairs_brute_force():
    for T, b, K in ((256, 16, 4), (100, 16, 2), (64, 64, 3)):
        N = (T + b - 1) // b
        cnt = 0
        for i in range(T):
            j = i // b
            cnt += min(K, j) * b + (i - j * b + 1)
        assert O.attended_pairs(1, 1, T, b, K) == cnt
    # the two bf16 training layers
    assert O.attended_pairs(1, 32, 16384, 64, 16) * 4 * 128 == pytest.approx(0.2745e12, rel=1e-3)


def test_round_bf16_matches_torch_conversion():
    """The bf16 rounding the oracle uses to measure operand-rounding floors is
    torch's float32 -> bfloat16 conversion (nearest, ties to even)."""
    import torch
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -3.0e38, 1e-40]])
    # exact ties between two bf16 neighbours: both directions of ties-to-even
    x = np.concatenate([x, 1.0 + (2 * np.arange(64) + 1) * 2.0 ** -9])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().double().numpy()
    np.testing.assert_array_equal(O.round_bf16(x), want)
