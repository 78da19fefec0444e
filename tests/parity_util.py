"""Shared helpers of the GPU parity tests: tolerances and oracle sampling.

Tolerances (stated by the workload definitions, read as follows):
  * fp32 tensors of an fp32 workload: max|x - y| / max|y| <= 1e-4 (normwise).
  * tensors of a bf16 workload: every element |x - y| <= 2e-2, and
    ||x - y||_2 / ||y||_2 <= 1e-2. A tensor the library stores in bf16 (o,
    dq, dk, dv) may in addition be off by half an ulp of its stored value,
    2^-8 |y|, which alone exceeds 2e-2 once |y| >= 8. fp32-stored outputs of
    a bf16 workload (lse, dscores) get the plain 2e-2 bound.
  * indices: bit-exact.
"""
from __future__ import annotations

import os

import numpy as np
import torch

from oracle import sas_oracle as O

BF16_ATOL = 2e-2
BF16_RTOL_ULP = 2.0 ** -8
BF16_REL_L2 = 1e-2
F32_NORMWISE = 1e-4


def dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16" and t.dtype == torch.float32:
        t = t.to(torch.bfloat16)
    return t.to(device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def _log(name, dtype, stored, err, l2, scale):
    """Appends the measured margin of a check to $SAS_PARITY_LOG (if set)."""
    path = os.environ.get("SAS_PARITY_LOG")
    if path:
        test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
        with open(path, "a") as f:
            f.write(f"{test}\t{name}\t{dtype}/{stored}\terr={err:.4e}\tl2={l2:.4e}\t"
                    f"max|y|={scale:.3e}\n")


def check(name: str, got, want, dtype: str, stored: str | None = None, floor=None):
    """Compare at the workload's tolerance. `stored` is the dtype the library
    writes the tensor in (defaults to the workload dtype); the half-ulp
    allowance applies only to bf16-stored tensors. `floor` (bf16 workloads):
    per element |emulated - exact|, where `emulated` is the oracle with its
    MMA operands (P, dS) rounded to bf16; twice it is allowed on top of the
    2e-2 bound, since no bf16-operand arithmetic can avoid that rounding."""
    stored = dtype if stored is None else stored
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = np.abs(got - want)
    scale = np.abs(want).max() if want.size else 0.0
    if dtype == "f32":
        rel = err.max() / max(scale, 1e-30) if want.size else 0.0
        _log(name, dtype, stored, rel, rel, scale)
        assert rel <= F32_NORMWISE, f"{name}: normwise rel err {rel:.3e} > {F32_NORMWISE}"
        return rel
    ulp = BF16_RTOL_ULP if stored == "bf16" else 0.0
    allow = ulp * np.abs(want)
    if floor is not None:
        allow = allow + 2.0 * np.asarray(floor, np.float64)
    excess = (err - allow).max() if want.size else 0.0
    l2 = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    _log(name, dtype, stored, excess, l2, scale)
    assert excess <= BF16_ATOL, f"{name}: max abs err {excess:.3e} > {BF16_ATOL} (stored {stored})"
    assert l2 <= BF16_REL_L2, f"{name}: rel L2 err {l2:.3e} > {BF16_REL_L2}"
    return l2


def floor_of(exact, emulated):
    """Per-element rounding floor of bf16-operand arithmetic."""
    return np.abs(np.asarray(emulated, np.float64) - np.asarray(exact, np.float64))


def oracle_gates_slice(scores, bi, kvh, K, causal=True):
    """Oracle gates / log-gates / idx for one (batch, kv head)."""
    g, lg, ix = O.gate_topk(scores[bi:bi + 1, kvh:kvh + 1], K, causal=causal)
    return g[0, 0], lg[0, 0], ix[0, 0]


def oracle_fwd_rows(x, b, K, bi, kvh, j, use_gates=True, cache=None, operands=None):
    """Oracle o [G, rows, d] and lse [G, rows] for query block j of (bi, kvh)."""
    g, lg, ix = cache if cache is not None else oracle_gates_slice(x.scores, bi, kvh, K)
    idx = np.zeros((bi + 1, kvh + 1) + ix.shape, np.int32)
    idx[bi, kvh] = ix
    logg = np.zeros((bi + 1, kvh + 1) + lg.shape)
    logg[bi, kvh] = lg
    return O.attn_fwd_block(x.q, x.k, x.v, idx, logg, bi, kvh, j, b, use_gates=use_gates,
                            operands=operands)


def oracle_bwd_sample(x, b, K, bi, kvh, js, ms, use_gates=True, cache=None, operands=None):
    """Oracle gradients for sampled query blocks js (dq rows, dscores rows) and
    sampled key blocks ms (dk, dv rows; summed over every query block whose
    key set contains block m)."""
    g, lg, ix = cache if cache is not None else oracle_gates_slice(x.scores, bi, kvh, K)
    idx = np.zeros((bi + 1, kvh + 1) + ix.shape, np.int32)
    idx[bi, kvh] = ix
    logg = np.zeros((bi + 1, kvh + 1) + lg.shape)
    logg[bi, kvh] = lg
    T = x.q.shape[2]
    N = ix.shape[0]
    out = {"dq": {}, "ds": {}, "dk": {}, "dv": {}}
    for j in js:
        r = O.attn_bwd_block(x.q, x.k, x.v, x.dO, idx, logg, bi, kvh, j, b, use_gates=use_gates,
                             operands=operands)
        out["dq"][j] = r["dq"]
        if use_gates:
            out["ds"][j] = np.concatenate([O.dscores_row(r["da"], g[j], j), np.zeros(N - j)])
    for m in ms:
        rows = min(T, (m + 1) * b) - m * b
        dk = np.zeros((rows, x.q.shape[3]))
        dv = np.zeros_like(dk)
        for j in range(m, N):
            if j != m and m not in set(int(t) for t in ix[j]):
                continue
            r = O.attn_bwd_block(x.q, x.k, x.v, x.dO, idx, logg, bi, kvh, j, b,
                                 use_gates=use_gates, operands=operands)
            sel = (r["cols"] >= m * b) & (r["cols"] < m * b + rows)
            dk += r["dk_c"][sel]
            dv += r["dv_c"][sel]
        out["dk"][m] = dk
        out["dv"][m] = dv
    return out
