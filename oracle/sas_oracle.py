"""Float64 CPU oracle for SAS gated block-sparse causal attention.

TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg may import this module. The product path (the
C-ABI library and its Python binding) never calls it, and it shares no code
with that path: nothing here imports the package, and the package imports
nothing from here.

What it computes, in the pages' notation (sources named by page title and
section; none of the pages prints code for this path):

* [Methodology, Eq. 4] and [Gradient Analysis, Eq. 6] of the picx.dev summary
  of "SAS: Simple Attention Sparsification via End-to-End Optimization of
  Context Ranking", and [Core equations] of the reproduction README "SAS:
  End-to-end learning of sparse attention rankings from language-model loss":
  history gates g = softmax(s) over the history blocks of a query block,
  log g_m = s_m - LSE(s); the always-retained current block has g0 = 1.
* [Theoretical Foundation, Eq. 3] (picx.dev) and [Core equations] (README):
  I = Top-K(s, K) over the history blocks, S = union of the selected blocks.
* [Methodology, Eq. 9] (picx.dev) with the 1/sqrt(d) scale from [Core
  equations] (README): o = softmax(q K_S^T / sqrt(d) + log g_S) V_S over the
  selected blocks plus the causally masked current block.
* [Gradient Analysis, Eq. 5, inner form] (picx.dev): the gradient reaching a
  gate; composed here with the Jacobian of Eq. 6 to give d loss / d scores.

Readings where the pages leave a step open (each is listed in the design
notes with its reason):
  - the 1/sqrt(d) scale multiplies q.k only, never log g;
  - the LSE of Eq. 6 runs over all history blocks m < j of query block j
    (not only the selected ones), so selected gates are not renormalised;
  - Top-K is taken over the fp32 scores, descending, ties to the lower block
    index, and returned in that rank order, padded with -1;
  - K counts history blocks only; block j has n_j = min(K, j) selections;
  - one selection and one gate vector per (batch, KV head, query block),
    shared by the G = Hq/Hkv query heads of that KV head;
  - no gradient flows through the hard selection (idx is piecewise constant);
  - decode: the query sits at position L-1 and its key is already in the
    cache; the block holding L-1 is the current block (fully visible), and
    the C = floor((L-1)/b) blocks before it are the history.

All arithmetic is float64; inputs (fp32 or bf16 values) convert to float64
exactly. The optional ``operands="bf16"`` of the attention functions rounds
the weights P and dL/dX to bf16 where they enter a product, as the operands
of a bf16 tensor-core kernel are: the tests use it only to measure the
rounding floor of such arithmetic, never as the reference result. Parity of every function here is pinned by tests against closed
forms, brute force, library special cases and finite differences.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Gate softmax (Eq. 4 with phi = softmax; Eq. 6) and Top-K (Eq. 3)
# ---------------------------------------------------------------------------

def log_gates_row(s_row, n: int) -> np.ndarray:
    """Eq. 6: log g_m = s_m - LSE(s_0 .. s_{n-1}) for the n history blocks."""
    s = _f64(s_row[:n])
    if n == 0:
        return s
    mx = s.max()
    lse = mx + math.log(np.exp(s - mx).sum())
    return s - lse


def topk_row(s_row_f32, n: int, K: int) -> list[int]:
    """Eq. 3: the min(K, n) history blocks with the largest fp32 score.

    A full stable sort by (-score, index): ties go to the lower block index,
    and the result is in rank order. Scores compare as fp32 values (so -0.0
    and +0.0 are equal). Returns exactly K entries, padded with -1.
    """
    vals = [float(np.float32(x)) for x in s_row_f32[:n]]
    order = sorted(range(n), key=lambda m: (-vals[m], m))
    sel = order[:min(K, n)]
    return sel + [-1] * (K - len(sel))


def gate_topk(scores, K: int, causal: bool = True):
    """Gates and Top-K indices for every row of ``scores``.

    scores: [B, Hkv, R, C] fp32. causal=True: R = C = N and row j has j valid
    entries (the history of query block j). causal=False: every row has C
    valid entries (decode). Returns (gates float64 [B,Hkv,R,C], zero past the
    valid length; log_gates float64, -inf past it; idx int32 [B,Hkv,R,K]).
    """
    s = np.asarray(scores)
    B, H, R, C = s.shape
    gates = np.zeros((B, H, R, C), dtype=np.float64)
    logg = np.full((B, H, R, C), -np.inf, dtype=np.float64)
    idx = np.full((B, H, R, K), -1, dtype=np.int32)
    for bi in range(B):
        for h in range(H):
            for r in range(R):
                n = min(r, C) if causal else C
                lg = log_gates_row(s[bi, h, r], n)
                logg[bi, h, r, :n] = lg
                gates[bi, h, r, :n] = np.exp(lg)
                idx[bi, h, r] = topk_row(s[bi, h, r], n, K)
    return gates, logg, idx


# ---------------------------------------------------------------------------
# Key set of one query block (Eq. 3 selection + the always-retained block)
# ---------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """x rounded to bfloat16 and returned as float64: first to float32
    (nearest), then to the 8-bit-mantissa bfloat16 grid (nearest, ties to even
    on the 16 dropped bits). This is the data path of a bf16 MMA operand
    formed in fp32 registers. Used only to measure the rounding floor of
    bf16-operand arithmetic (``operands="bf16"`` below), never for results."""
    f = np.asarray(x, np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    keep = (u >> 16) & 1
    r = (((u + 0x7FFF + keep) >> 16) << 16).astype(np.uint32)
    out = r.view(np.float32).astype(np.float64)
    return np.where(np.isfinite(f), out, f.astype(np.float64))


def _ops(a, operands):
    """An MMA operand as the arithmetic under test sees it."""
    return round_bf16(a) if operands == "bf16" else a


def _key_set(j: int, b: int, T: int, sel_row, logg_row, use_gates: bool):
    """Columns and additive biases for query block j.

    The selected history blocks contribute all their b keys with bias
    log g_m (Eq. 9) or 0 (Eq. 2, gates off); the current block j contributes
    its keys with bias 0 (g0 = 1, Eq. 4). Returns (cols, bias, n_hist_cols).
    """
    cols, bias = [], []
    for m in sel_row:
        m = int(m)
        if m < 0:
            continue
        cols.extend(range(m * b, (m + 1) * b))
        bias.extend([float(logg_row[m]) if use_gates else 0.0] * b)
    nh = len(cols)
    cur = list(range(j * b, min(T, (j + 1) * b)))
    cols.extend(cur)
    bias.extend([0.0] * len(cur))
    return np.asarray(cols, dtype=np.int64), np.asarray(bias, dtype=np.float64), nh


def _block_logits(Qb, Kc, bias, nh, scale, row0, col0_cur):
    """Gated logits for the rows of one query block against its key set.

    Row r (global position row0 + r) may see current-block key c (global
    position col0_cur + c) only when col0_cur + c <= row0 + r (causal mask).
    """
    X = scale * (Qb @ Kc.T) + bias[None, :]
    ncur = Kc.shape[0] - nh
    if ncur:
        rows = row0 + np.arange(Qb.shape[0])[:, None]
        keys = col0_cur + np.arange(ncur)[None, :]
        X[:, nh:] = np.where(keys <= rows, X[:, nh:], -np.inf)
    return X


def _lse_rows(X):
    mx = X.max(axis=1, keepdims=True)
    return (mx + np.log(np.exp(X - mx).sum(axis=1, keepdims=True)))[:, 0]


def _default_scale(d, scale):
    return 1.0 / math.sqrt(d) if not scale else float(scale)


# ---------------------------------------------------------------------------
# Forward (Eq. 9)
# ---------------------------------------------------------------------------

def attn_fwd_block(q, k, v, idx, logg, bi, kvh, j, b, scale=0.0, use_gates=True,
                   operands=None):
    """Eq. 9 for the G query heads of KV head ``kvh`` and the rows of block j.

    Returns (o [G, rows, d], lse [G, rows]) in float64. With operands="bf16"
    the weights P enter P V rounded to bf16 (the error floor of bf16-operand
    arithmetic; the method's result is operands=None).
    """
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    Hq, T, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[1]
    scale = _default_scale(d, scale)
    cols, bias, nh = _key_set(j, b, T, idx[bi, kvh, j],
                              logg[bi, kvh, j] if logg is not None else None, use_gates)
    Kc = _f64(k[bi, kvh, cols])
    Vc = _f64(v[bi, kvh, cols])
    r0, r1 = j * b, min(T, (j + 1) * b)
    O = np.empty((G, r1 - r0, d))
    L = np.empty((G, r1 - r0))
    for g in range(G):
        h = kvh * G + g
        X = _block_logits(_f64(q[bi, h, r0:r1]), Kc, bias, nh, scale, r0, j * b)
        lse = _lse_rows(X)
        P = np.exp(X - lse[:, None])
        O[g] = _ops(P, operands) @ Vc
        L[g] = lse
    return O, L


def attn_fwd(q, k, v, idx, logg, b, scale=0.0, use_gates=True, operands=None):
    """Eq. 9 over every query block. Returns (o [B,Hq,T,d], lse [B,Hq,T])."""
    B, Hq, T, d = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    N = (T + b - 1) // b
    o = np.empty((B, Hq, T, d))
    lse = np.empty((B, Hq, T))
    for bi in range(B):
        for kvh in range(Hkv):
            for j in range(N):
                O, L = attn_fwd_block(q, k, v, idx, logg, bi, kvh, j, b, scale, use_gates,
                                      operands)
                r0, r1 = j * b, min(T, (j + 1) * b)
                o[bi, kvh * G:(kvh + 1) * G, r0:r1] = O
                lse[bi, kvh * G:(kvh + 1) * G, r0:r1] = L
    return o, lse


# ---------------------------------------------------------------------------
# Backward: chain rule through Eq. 9, then Eq. 5 (inner) and the Eq. 6 Jacobian
# ---------------------------------------------------------------------------

def attn_bwd_block(q, k, v, dO, idx, logg, bi, kvh, j, b, scale=0.0, use_gates=True,
                   operands=None):
    """Gradients contributed by query block j of KV head ``kvh``.

    For the loss L = sum(o * dO): returns a dict with
      dq   [G, rows, d]        gradient for the block's query rows (complete),
      cols, dk_c, dv_c         key columns touched and their partial dk/dv,
      da   {m: value}          dL/d log g_m for every selected history block m,
    where dL/dX = P * (dP - rowsum(P * dP)) is the softmax Jacobian applied to
    dP = dO V^T, and da_m sums dL/dX over block m's columns, all rows and all
    G heads (log g_m enters every logit of block m, shared by the group).
    operands="bf16" rounds P and dL/dX to bf16 where they enter the products
    (dv, dq, dk), the floor of bf16-operand arithmetic; da stays exact.
    """
    q, k, v, dO = np.asarray(q), np.asarray(k), np.asarray(v), np.asarray(dO)
    Hq, T, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[1]
    scale = _default_scale(d, scale)
    cols, bias, nh = _key_set(j, b, T, idx[bi, kvh, j],
                              logg[bi, kvh, j] if logg is not None else None, use_gates)
    Kc = _f64(k[bi, kvh, cols])
    Vc = _f64(v[bi, kvh, cols])
    r0, r1 = j * b, min(T, (j + 1) * b)
    dq = np.zeros((G, r1 - r0, d))
    dk_c = np.zeros_like(Kc)
    dv_c = np.zeros_like(Vc)
    dX_hist = np.zeros(nh)
    for g in range(G):
        h = kvh * G + g
        Qb = _f64(q[bi, h, r0:r1])
        dOb = _f64(dO[bi, h, r0:r1])
        X = _block_logits(Qb, Kc, bias, nh, scale, r0, j * b)
        P = np.exp(X - _lse_rows(X)[:, None])
        dP = dOb @ Vc.T
        dX = P * (dP - (P * dP).sum(axis=1, keepdims=True))
        dXo = _ops(dX, operands)
        dq[g] = scale * (dXo @ Kc)
        dk_c += scale * (dXo.T @ Qb)
        dv_c += _ops(P, operands).T @ dOb
        dX_hist += dX[:, :nh].sum(axis=0)
    da = {}
    pos = 0
    for m in idx[bi, kvh, j]:
        m = int(m)
        if m < 0:
            continue
        da[m] = dX_hist[pos:pos + b].sum()
        pos += b
    return {"dq": dq, "cols": cols, "dk_c": dk_c, "dv_c": dv_c, "da": da}


def dscores_row(da: dict, gates_row, n: int) -> np.ndarray:
    """Eq. 6 Jacobian: dL/ds_k = [k in I] da_k - g_k * sum_{m in I} da_m, k < n.

    d log g_m / d s_k = delta_mk - g_k, so only the selected blocks' da enter;
    no gradient flows through the (piecewise constant) selection itself.
    """
    out = np.zeros(n)
    tot = sum(da.values())
    g = _f64(gates_row[:n])
    out[:] = -g * tot
    for m, a in da.items():
        out[m] += a
    return out


def attn_bwd(q, k, v, dO, idx, gates, logg, b, scale=0.0, use_gates=True, operands=None):
    """Full backward. Returns (dq, dk, dv, dscores) in float64.

    dscores has the shape of the training score tensor [B, Hkv, N, N]: row j
    holds dL/ds_{j,k} for k < j and zero elsewhere; all zero when gates are off.
    """
    B, Hq, T, d = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    N = (T + b - 1) // b
    dq = np.zeros((B, Hq, T, d))
    dk = np.zeros((B, Hkv, T, d))
    dv = np.zeros((B, Hkv, T, d))
    ds = np.zeros((B, Hkv, N, N))
    for bi in range(B):
        for kvh in range(Hkv):
            for j in range(N):
                r = attn_bwd_block(q, k, v, dO, idx, logg, bi, kvh, j, b, scale, use_gates,
                                   operands)
                r0, r1 = j * b, min(T, (j + 1) * b)
                dq[bi, kvh * G:(kvh + 1) * G, r0:r1] = r["dq"]
                np.add.at(dk[bi, kvh], r["cols"], r["dk_c"])
                np.add.at(dv[bi, kvh], r["cols"], r["dv_c"])
                if use_gates:
                    ds[bi, kvh, j, :j] = dscores_row(r["da"], gates[bi, kvh, j], j)
    return dq, dk, dv, ds


# ---------------------------------------------------------------------------
# Gate variants: the ablation axes of the pages (the functions above are the
# method itself; these are its ablated forms, for the variant kernels)
# ---------------------------------------------------------------------------
# [Methodology, Eq. 4] (picx.dev) leaves the gate activation phi open, and
# the summary's ablations (Table 1 as summarised there) compare phi =
# softmax with sigmoid and raw-logit gates. [Gradient Analysis, Eq. 5]
# contrasts inner gating (log g added to the logits, Eq. 9) with outer
# gating. Readings, for lack of a formula on the pages:
#   - sigmoid: g_m = 1 / (1 + exp(-s_m)), elementwise, no normalisation over
#     the history, so log g_m = -log(1 + exp(-s_m));
#   - raw logits: log g_m = s_m, the score enters the logits as it is;
#   - outer gating: o = sum_i g_{m(i)} p_i v_i with p the ungated softmax
#     over the selected keys plus the current block (g0 = 1): the form whose
#     derivative in g_m is the outer form of Eq. 5.
# Top-K is over the scores in every variant (every phi is increasing).

PHIS = ("softmax", "sigmoid", "raw")


def log_gates_row_phi(s_row, n: int, phi: str) -> np.ndarray:
    """log g over the n history blocks for the gate activation ``phi``."""
    s = _f64(s_row[:n])
    if phi == "softmax":
        return log_gates_row(s_row, n)
    if phi == "sigmoid":
        return -np.logaddexp(0.0, -s)
    if phi == "raw":
        return s.copy()
    raise ValueError(phi)


def gate_topk_phi(scores, K: int, phi: str, causal: bool = True):
    """gate_topk with the activation ``phi``: (gates, log_gates, idx)."""
    gates, logg, idx = gate_topk(scores, K, causal)
    if phi == "softmax":
        return gates, logg, idx
    s = np.asarray(scores)
    B, H, R, C = s.shape
    for bi in range(B):
        for h in range(H):
            for r in range(R):
                n = min(r, C) if causal else C
                lg = log_gates_row_phi(s[bi, h, r], n, phi)
                logg[bi, h, r, :n] = lg
                gates[bi, h, r, :n] = np.exp(lg)
    return gates, logg, idx


def dscores_row_phi(da: dict, s_row, n: int, phi: str) -> np.ndarray:
    """dL/ds_k for k < n from da_m = dL/d log g_m of the selected blocks.

    softmax: d log g_m / d s_k = delta_mk - g_k (Eq. 6, as dscores_row);
    sigmoid: d log g_m / d s_k = delta_mk (1 - sigmoid(s_k));
    raw:     d log g_m / d s_k = delta_mk.
    """
    if phi == "softmax":
        return dscores_row(da, np.exp(log_gates_row(s_row, n)), n)
    out = np.zeros(n)
    s = _f64(s_row[:n])
    for m, a in da.items():
        out[m] = a * (np.exp(-np.logaddexp(0.0, s[m])) if phi == "sigmoid" else 1.0)
    return out


def attn_bwd_phi(q, k, v, dO, idx, scores, b, phi: str, scale=0.0, operands=None):
    """Inner gating (Eq. 9) with gates from ``phi``: (dq, dk, dv, dscores)."""
    _, logg, _ = gate_topk_phi(scores, idx.shape[-1], phi)
    B, Hq, T, d = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    N = (T + b - 1) // b
    dq = np.zeros((B, Hq, T, d))
    dk = np.zeros((B, Hkv, T, d))
    dv = np.zeros((B, Hkv, T, d))
    ds = np.zeros((B, Hkv, N, N))
    for bi in range(B):
        for kvh in range(Hkv):
            for j in range(N):
                r = attn_bwd_block(q, k, v, dO, idx, logg, bi, kvh, j, b, scale,
                                   operands=operands)
                r0, r1 = j * b, min(T, (j + 1) * b)
                dq[bi, kvh * G:(kvh + 1) * G, r0:r1] = r["dq"]
                np.add.at(dk[bi, kvh], r["cols"], r["dk_c"])
                np.add.at(dv[bi, kvh], r["cols"], r["dv_c"])
                ds[bi, kvh, j, :j] = dscores_row_phi(r["da"], scores[bi, kvh, j], j, phi)
    return dq, dk, dv, ds


def _col_gates(j, b, T, sel_row, gates_row):
    """Per-column gate of query block j's key set (g_m on block m, 1 on block j)."""
    w = []
    for m in sel_row:
        m = int(m)
        if m >= 0:
            w.extend([float(gates_row[m])] * b)
    w.extend([1.0] * (min(T, (j + 1) * b) - j * b))
    return np.asarray(w)


def attn_fwd_outer_block(q, k, v, idx, gates, bi, kvh, j, b, scale=0.0, operands=None):
    """Outer gating for the G heads of KV head ``kvh`` and block j's rows:
    o = (P * w) V with P the ungated softmax and w the per-column gates.
    Returns (o [G, rows, d], lse [G, rows]) where lse is the ungated one."""
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    Hq, T, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[1]
    scale = _default_scale(d, scale)
    cols, bias, nh = _key_set(j, b, T, idx[bi, kvh, j], None, False)
    w = _col_gates(j, b, T, idx[bi, kvh, j], gates[bi, kvh, j])
    Kc, Vc = _f64(k[bi, kvh, cols]), _f64(v[bi, kvh, cols])
    r0, r1 = j * b, min(T, (j + 1) * b)
    O = np.empty((G, r1 - r0, d))
    L = np.empty((G, r1 - r0))
    for g in range(G):
        X = _block_logits(_f64(q[bi, kvh * G + g, r0:r1]), Kc, bias, nh, scale, r0, j * b)
        lse = _lse_rows(X)
        O[g] = _ops(np.exp(X - lse[:, None]) * w[None, :], operands) @ Vc
        L[g] = lse
    return O, L


def attn_fwd_outer(q, k, v, idx, gates, b, scale=0.0, operands=None):
    """Outer gating over every query block: (o [B,Hq,T,d], lse [B,Hq,T])."""
    B, Hq, T, d = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    N = (T + b - 1) // b
    o = np.empty((B, Hq, T, d))
    lse = np.empty((B, Hq, T))
    for bi in range(B):
        for kvh in range(Hkv):
            for j in range(N):
                O, L = attn_fwd_outer_block(q, k, v, idx, gates, bi, kvh, j, b, scale, operands)
                r0, r1 = j * b, min(T, (j + 1) * b)
                o[bi, kvh * G:(kvh + 1) * G, r0:r1] = O
                lse[bi, kvh * G:(kvh + 1) * G, r0:r1] = L
    return o, lse


def attn_bwd_outer_block(q, k, v, dO, idx, gates, bi, kvh, j, b, scale=0.0, operands=None):
    """Gradients of L = sum(o * dO) under outer gating from query block j.

    With W = P * w: dv += W^T dO; dL/dP = w * dP (dP = dO V^T), so the
    softmax Jacobian gives dX = P * (w dP - rowsum(P w dP)); dq = scale dX K,
    dk += scale dX^T Q; dg_m = sum over block m's columns, all rows and all G
    heads of P * dP (Eq. 5, outer form), returned as da_m = g_m dg_m
    (= dL/d log g_m, the input of the phi Jacobians above).
    """
    q, k, v, dO = np.asarray(q), np.asarray(k), np.asarray(v), np.asarray(dO)
    Hq, T, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[1]
    scale = _default_scale(d, scale)
    cols, bias, nh = _key_set(j, b, T, idx[bi, kvh, j], None, False)
    w = _col_gates(j, b, T, idx[bi, kvh, j], gates[bi, kvh, j])
    Kc, Vc = _f64(k[bi, kvh, cols]), _f64(v[bi, kvh, cols])
    r0, r1 = j * b, min(T, (j + 1) * b)
    dq = np.zeros((G, r1 - r0, d))
    dk_c, dv_c = np.zeros_like(Kc), np.zeros_like(Vc)
    pdp_hist = np.zeros(nh)
    for g in range(G):
        Qb = _f64(q[bi, kvh * G + g, r0:r1])
        dOb = _f64(dO[bi, kvh * G + g, r0:r1])
        X = _block_logits(Qb, Kc, bias, nh, scale, r0, j * b)
        P = np.exp(X - _lse_rows(X)[:, None])
        dP = dOb @ Vc.T
        wdP = dP * w[None, :]
        dX = P * (wdP - (P * wdP).sum(axis=1, keepdims=True))
        dXo = _ops(dX, operands)
        dq[g] = scale * (dXo @ Kc)
        dk_c += scale * (dXo.T @ Qb)
        dv_c += _ops(P * w[None, :], operands).T @ dOb
        pdp_hist += (P * dP)[:, :nh].sum(axis=0)
    da, pos = {}, 0
    for m in idx[bi, kvh, j]:
        m = int(m)
        if m < 0:
            continue
        da[m] = float(gates[bi, kvh, j, m]) * pdp_hist[pos:pos + b].sum()
        pos += b
    return {"dq": dq, "cols": cols, "dk_c": dk_c, "dv_c": dv_c, "da": da}


def gate_grad_eq5_outer(q, k, v, dO, idx, gates, bi, kvh, j, b, scale=0.0):
    """Eq. 5, outer form, literally: dg_m = sum_i p_i dO^T v_i over the keys i
    of selected block m, for every row and every head of the group, with p
    the ungated softmax over the block's key set. Returns {m: dg_m}."""
    q, k, v, dO = np.asarray(q), np.asarray(k), np.asarray(v), np.asarray(dO)
    Hq, T, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[1]
    scale = _default_scale(d, scale)
    cols, bias, nh = _key_set(j, b, T, idx[bi, kvh, j], None, False)
    Kc, Vc = _f64(k[bi, kvh, cols]), _f64(v[bi, kvh, cols])
    r0, r1 = j * b, min(T, (j + 1) * b)
    out, pos = {}, 0
    for m in idx[bi, kvh, j]:
        m = int(m)
        if m < 0:
            continue
        tot = 0.0
        for g in range(G):
            Qb = _f64(q[bi, kvh * G + g, r0:r1])
            dOb = _f64(dO[bi, kvh * G + g, r0:r1])
            X = _block_logits(Qb, Kc, bias, nh, scale, r0, j * b)
            P = np.exp(X - _lse_rows(X)[:, None])
            for row in range(r1 - r0):
                for c in range(pos, pos + b):
                    tot += P[row, c] * float(dOb[row] @ Vc[c])
        out[m] = tot
        pos += b
    return out


def attn_bwd_outer(q, k, v, dO, idx, scores, b, phi: str = "softmax", scale=0.0,
                   operands=None):
    """Outer gating with gates from ``phi``: (dq, dk, dv, dscores)."""
    gates, _, _ = gate_topk_phi(scores, idx.shape[-1], phi)
    B, Hq, T, d = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    N = (T + b - 1) // b
    dq = np.zeros((B, Hq, T, d))
    dk = np.zeros((B, Hkv, T, d))
    dv = np.zeros((B, Hkv, T, d))
    ds = np.zeros((B, Hkv, N, N))
    for bi in range(B):
        for kvh in range(Hkv):
            for j in range(N):
                r = attn_bwd_outer_block(q, k, v, dO, idx, gates, bi, kvh, j, b, scale,
                                         operands)
                r0, r1 = j * b, min(T, (j + 1) * b)
                dq[bi, kvh * G:(kvh + 1) * G, r0:r1] = r["dq"]
                np.add.at(dk[bi, kvh], r["cols"], r["dk_c"])
                np.add.at(dv[bi, kvh], r["cols"], r["dv_c"])
                ds[bi, kvh, j, :j] = dscores_row_phi(r["da"], scores[bi, kvh, j], j, phi)
    return dq, dk, dv, ds


def gate_grad_eq5(q, k, v, dO, idx, gates, logg, bi, kvh, j, b, scale=0.0):
    """Eq. 5, inner form, literally: dg_m = sum_i (p~_i / g_m) dO^T (v_i - o).

    The sum runs over the keys i of selected block m, for every row and every
    head of the group, with p~ the gated attention probability and o that
    row's output. Returns {m: dg_m}. Used as an independent pin: g_m * dg_m
    must equal da_m of ``attn_bwd_block``.
    """
    q, k, v, dO = np.asarray(q), np.asarray(k), np.asarray(v), np.asarray(dO)
    Hq, T, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[1]
    scale = _default_scale(d, scale)
    cols, bias, nh = _key_set(j, b, T, idx[bi, kvh, j], logg[bi, kvh, j], True)
    Kc = _f64(k[bi, kvh, cols])
    Vc = _f64(v[bi, kvh, cols])
    r0, r1 = j * b, min(T, (j + 1) * b)
    out = {}
    sel = [int(m) for m in idx[bi, kvh, j] if m >= 0]
    for g in range(G):
        h = kvh * G + g
        X = _block_logits(_f64(q[bi, h, r0:r1]), Kc, bias, nh, scale, r0, j * b)
        P = np.exp(X - _lse_rows(X)[:, None])
        O = P @ Vc
        dOb = _f64(dO[bi, h, r0:r1])
        for pos, m in enumerate(sel):
            blk = slice(pos * b, (pos + 1) * b)
            term = (P[:, blk] / gates[bi, kvh, j, m]) * (dOb @ Vc[blk].T - (dOb * O).sum(1)[:, None])
            out[m] = out.get(m, 0.0) + term.sum()
    return out


# ---------------------------------------------------------------------------
# Decode (Eq. 2 with gates dropped, or Eq. 9) for one query token
# ---------------------------------------------------------------------------

def decode(q, kcache, vcache, idx, logg, b, scale=0.0, use_gates=False):
    """One query token per (batch, q head) at position L-1 of the cache.

    q [B,Hq,d]; kcache/vcache [B,Hkv,L,d]; idx [B,Hkv,K] over the
    C = floor((L-1)/b) history blocks; logg [B,Hkv,C] (used when use_gates).
    Keys: the selected history blocks (bias log g_m, or 0 with gates off)
    plus every position of the current block up to L-1 (bias 0).
    Returns o [B,Hq,d] float64.
    """
    q, kc, vc = np.asarray(q), np.asarray(kcache), np.asarray(vcache)
    B, Hq, d = q.shape
    Hkv, L = kc.shape[1], kc.shape[2]
    G = Hq // Hkv
    scale = _default_scale(d, scale)
    cb = (L - 1) // b
    o = np.empty((B, Hq, d))
    for bi in range(B):
        for kvh in range(Hkv):
            cols, bias = [], []
            for m in idx[bi, kvh]:
                m = int(m)
                if m < 0:
                    continue
                cols.extend(range(m * b, (m + 1) * b))
                bias.extend([float(logg[bi, kvh, m]) if use_gates else 0.0] * b)
            cols.extend(range(cb * b, L))
            bias.extend([0.0] * (L - cb * b))
            Kc = _f64(kc[bi, kvh, cols])
            Vc = _f64(vc[bi, kvh, cols])
            bias = np.asarray(bias)
            for g in range(G):
                h = kvh * G + g
                x = scale * (Kc @ _f64(q[bi, h])) + bias
                mx = x.max()
                p = np.exp(x - mx)
                o[bi, h] = (p @ Vc) / p.sum()
    return o


def decode_paged(q, kpages, vpages, page_indptr, page_indices, seq_lens, idx, logg, b,
                 scale=0.0, use_gates=False):
    """Decode over a paged KV cache, one sequence per batch entry.

    The pages mention that deployment decodes on a paged cache (SGLang /
    FlashInfer) without fixing a layout. Reading: kpages / vpages are
    [num_pages, Hkv, P, d] (P tokens per page); sequence bi owns the pages
    page_indices[page_indptr[bi]:page_indptr[bi+1]] in logical order, token t
    sits at offset t % P of its (t // P)-th page, and it has seq_lens[bi]
    tokens (the last page may be partly used). Its query is at position
    seq_lens[bi] - 1; idx[bi] selects among its floor((seq_lens[bi]-1)/b)
    history blocks, and logg[bi] holds their log gates. The result is that of
    ``decode`` on the sequence's gathered contiguous cache.
    Returns o [B,Hq,d] float64.
    """
    q = np.asarray(q)
    kp, vp = np.asarray(kpages), np.asarray(vpages)
    B = q.shape[0]
    P = kp.shape[2]
    o = np.empty(q.shape, dtype=np.float64)
    for bi in range(B):
        L = int(seq_lens[bi])
        pages = np.asarray(page_indices[page_indptr[bi]:page_indptr[bi + 1]], np.int64)
        t = np.arange(L)
        kc = kp[pages[t // P], :, t % P].transpose(1, 0, 2)  # [Hkv, L, d]
        vc = vp[pages[t // P], :, t % P].transpose(1, 0, 2)
        C = (L - 1) // b
        lg = np.asarray(logg)[bi:bi + 1, :, :C] if logg is not None else None
        o[bi] = decode(q[bi:bi + 1], kc[None], vc[None], np.asarray(idx)[bi:bi + 1], lg, b,
                       scale, use_gates)[0]
    return o


# ---------------------------------------------------------------------------
# Dense comparison (Eq. 1 with a causal mask): every block, gates off
# ---------------------------------------------------------------------------

def all_blocks_idx(B, Hkv, N):
    """Selection of every history block (rank order = ascending index)."""
    idx = np.full((B, Hkv, N, max(N - 1, 1)), -1, dtype=np.int32)
    for j in range(N):
        idx[:, :, j, :j] = np.arange(j, dtype=np.int32)
    return idx


def dense_fwd(q, k, v, b, scale=0.0):
    B, Hq, T, d = np.shape(q)
    N = (T + b - 1) // b
    return attn_fwd(q, k, v, all_blocks_idx(B, np.shape(k)[1], N), None, b, scale,
                    use_gates=False)


def dense_decode(q, kcache, vcache, scale=0.0):
    """Every cache position 0..L-1 attends, gates off."""
    q, kc, vc = np.asarray(q), np.asarray(kcache), np.asarray(vcache)
    B, Hq, d = q.shape
    G = Hq // kc.shape[1]
    scale = _default_scale(d, scale)
    o = np.empty((B, Hq, d))
    for bi in range(B):
        for kvh in range(kc.shape[1]):
            Kc = _f64(kc[bi, kvh])
            Vc = _f64(vc[bi, kvh])
            for g in range(G):
                h = kvh * G + g
                x = scale * (Kc @ _f64(q[bi, h]))
                p = np.exp(x - x.max())
                o[bi, h] = (p @ Vc) / p.sum()
    return o


# ---------------------------------------------------------------------------
# Block-selector scores from pooled block summaries
# ---------------------------------------------------------------------------
# The evolve.pub review (Frequently asked questions) says the selector (the
# AttnGate architecture it shares with SeerAttention-R) works from
# "pooling-based block summaries" and scores history blocks per query block
# and KV-head group; no page gives its layers or weights. Reading (weight-free,
# the plainest one the pages support): a block's key summary is the mean of
# its keys, a query block's summary the mean of its query rows over the G
# heads of the group, and the score is their scaled dot product,
#   s[j, m] = scale * qbar_j . kbar_m   for history blocks m < j (0 otherwise),
# with scale = 1/sqrt(d) as in the attention logits. At decode the query
# summary is the mean of the G heads' single query token.

def block_summaries(x, b):
    """Mean over each block's rows (the last block may be partial):
    x [..., T, d] -> [..., N, d] float64."""
    x = _f64(x)
    T = x.shape[-2]
    N = (T + b - 1) // b
    out = np.empty(x.shape[:-2] + (N, x.shape[-1]))
    for m in range(N):
        out[..., m, :] = x[..., m * b:min(T, (m + 1) * b), :].mean(axis=-2)
    return out


def selector_scores(q, k, b, scale=0.0):
    """Training scores [B, Hkv, N, N] (row j meaningful for m < j, 0 elsewhere)."""
    q, k = _f64(q), _f64(k)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    scale = _default_scale(d, scale)
    qbar = block_summaries(q.reshape(B, Hkv, G, T, d), b).mean(axis=2)  # [B, Hkv, N, d]
    kbar = block_summaries(k, b)                                          # [B, Hkv, N, d]
    N = kbar.shape[2]
    s = np.zeros((B, Hkv, N, N))
    for j in range(N):
        s[:, :, j, :j] = scale * np.einsum("bhd,bhmd->bhm", qbar[:, :, j], kbar[:, :, :j])
    return s


def selector_scores_decode(q, kcache, L, b, scale=0.0):
    """Decode scores [B, Hkv, C] over the C = floor((L-1)/b) history blocks of
    a cache holding L tokens; q [B, Hq, d] is the token at L-1."""
    q, kc = _f64(q), _f64(kcache)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    scale = _default_scale(d, scale)
    C = (L - 1) // b
    qbar = q.reshape(B, Hkv, G, d).mean(axis=2)
    kbar = block_summaries(kc[:, :, :C * b], b) if C else np.zeros((B, Hkv, 0, d))
    return scale * np.einsum("bhd,bhmd->bhm", qbar, kbar)


# ---------------------------------------------------------------------------
# Algorithmic work counts (for throughput figures, not for any result)
# ---------------------------------------------------------------------------

def attended_pairs(B, Hq, T, b, K):
    """Sum over query rows of the number of keys each row attends."""
    N = (T + b - 1) // b
    total = 0
    for j in range(N):
        rows = min(T, (j + 1) * b) - j * b
        total += rows * b * min(K, j) + rows * (rows + 1) // 2
    return total * B * Hq
