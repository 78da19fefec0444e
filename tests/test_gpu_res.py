"""GPU parity of the training pair with the forward's output residual
(sas_attn_fwd_res / sas_attn_bwd_res) against the float64 oracle, at the
same tolerances as sas_attn_fwd / sas_attn_bwd: the backward takes its row
sums D from o and the residual instead of recomputing every attended tile.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, floor_of, host, oracle_bwd_sample, oracle_fwd_rows, \
    oracle_gates_slice

pytestmark = pytest.mark.gpu


def _run(lib, x, cfg, use_gates=True):
    q, k, v, dO = (dev(a, cfg.dtype) for a in (x.q, x.k, x.v, x.dO))
    gates, idx = lib.gate_topk(dev(x.scores, "f32"), cfg.K, causal=True)
    gg = gates if use_gates else None
    o, o_res, lse = lib.attn_fwd_res(q, k, v, idx, gg, cfg.b)
    dq, dk, dv, ds = lib.attn_bwd_res(q, k, v, o, o_res, lse, dO, idx, gg, cfg.b)
    o_plain, lse_plain = lib.attn_fwd(q, k, v, idx, gg, cfg.b)
    torch.cuda.synchronize()
    st, raw = lib.device_error()
    assert st == 0, f"device error bits {raw:#x}"
    return dict(o=o, o_res=o_res, lse=lse, dq=dq, dk=dk, dv=dv, ds=ds, idx=idx, gates=gates,
                o_plain=o_plain, lse_plain=lse_plain)


@pytest.mark.parametrize("kw", [
    # G = 4 (two tiles a CTA) and G = 2 (one), ragged T, hot key blocks
    dict(B=1, Hq=8, Hkv=2, T=1000, d=128, b=64, K=3, dtype="bf16", hot_key_frac=0.1,
         hot_key_scale=3.0),
    dict(B=2, Hq=4, Hkv=1, T=512, d=128, b=64, K=16, dtype="bf16"),
    dict(B=1, Hq=8, Hkv=4, T=1000, d=128, b=64, K=3, dtype="bf16", hot_key_frac=0.1,
         hot_key_scale=3.0),
    dict(B=2, Hq=4, Hkv=2, T=700, d=128, b=64, K=5, dtype="bf16"),
])
@pytest.mark.parametrize("use_gates", [True, False])
def test_res_pair_matches_oracle(cuda_lib, kw, use_gates):
    cfg = W.small_train_config(**kw)
    x = W.make_train_inputs(cfg)
    r = _run(cuda_lib, x, cfg, use_gates)
    g, lg, ix = O.gate_topk(x.scores, cfg.K)
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), ix)
    o, lse = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b, use_gates=use_gates)
    dq, dk, dv, ds = O.attn_bwd(x.q, x.k, x.v, x.dO, ix, g, lg, cfg.b, use_gates=use_gates)
    oe, _ = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b, use_gates=use_gates, operands="bf16")
    e = O.attn_bwd(x.q, x.k, x.v, x.dO, ix, g, lg, cfg.b, use_gates=use_gates, operands="bf16")
    check("o", host(r["o"]), o, "bf16", floor=floor_of(o, oe))
    check("lse", host(r["lse"]), lse, "bf16", stored="f32")
    # o + o_res is the output to fp32 rounding (P entered PV as two bf16 terms)
    full = host(r["o"]) + host(r["o_res"])
    rel = np.abs(full - o).max() / np.abs(o).max()
    assert rel < 2e-4, f"o + o_res: normwise rel err {rel:.3e}"
    # the residual is at most about half an ulp of o
    assert (np.abs(host(r["o_res"])) <= 2.0 ** -7 * np.abs(host(r["o"])) + 1e-30).all()
    check("dq", host(r["dq"]), dq, "bf16", floor=floor_of(dq, e[0]))
    check("dk", host(r["dk"]), dk, "bf16", floor=floor_of(dk, e[1]))
    check("dv", host(r["dv"]), dv, "bf16", floor=floor_of(dv, e[2]))
    if use_gates:
        check("dscores", host(r["ds"]), ds, "bf16", stored="f32")
    # the plain forward's lse is the same computation
    np.testing.assert_allclose(host(r["lse"]), host(r["lse_plain"]), rtol=0, atol=1e-5)


def test_res_rejects_shapes_without_tensor_cores(cuda_lib):
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=128, d=64, b=32, K=2, dtype="f32")
    x = W.make_train_inputs(cfg)
    q, k, v = (dev(a, "f32") for a in (x.q, x.k, x.v))
    gates, idx = cuda_lib.gate_topk(dev(x.scores, "f32"), cfg.K, causal=True)
    with pytest.raises(cuda_lib.SasError):
        cuda_lib.attn_fwd_res(q, k, v, idx, gates, cfg.b)


@pytest.mark.slow
def test_res_pair_full_size_sampled(cuda_lib):
    cfg = W.PRESETS["qwen3-4b-train"]
    x = W.make_train_inputs(cfg)
    r = _run(cuda_lib, x, cfg)
    N, G, b = cfg.N, cfg.G, cfg.b
    js = [0, 1, cfg.K, cfg.K + 1, N // 2, N - 1]
    ms = [0, 1, N // 3, N - 1]
    for bi, kvh in ((0, 0), (cfg.B - 1, cfg.Hkv - 1)):
        cache = oracle_gates_slice(x.scores, bi, kvh, cfg.K)
        for j in js:
            o, lse = oracle_fwd_rows(x, b, cfg.K, bi, kvh, j, cache=cache)
            oe, _ = oracle_fwd_rows(x, b, cfg.K, bi, kvh, j, cache=cache, operands="bf16")
            sl = slice(j * b, (j + 1) * b)
            check(f"o[{j}]", host(r["o"][bi, kvh * G:(kvh + 1) * G, sl]), o, cfg.dtype,
                  floor=floor_of(o, oe))
        ob = oracle_bwd_sample(x, b, cfg.K, bi, kvh, js, ms, cache=cache)
        eb = oracle_bwd_sample(x, b, cfg.K, bi, kvh, js, ms, cache=cache, operands="bf16")
        for j in js:
            sl = slice(j * b, (j + 1) * b)
            check(f"dq[{j}]", host(r["dq"][bi, kvh * G:(kvh + 1) * G, sl]), ob["dq"][j], cfg.dtype,
                  floor=floor_of(ob["dq"][j], eb["dq"][j]))
            check(f"ds[{j}]", host(r["ds"][bi, kvh, j]), ob["ds"][j], cfg.dtype, stored="f32")
        for m in ms:
            sl = slice(m * b, (m + 1) * b)
            check(f"dk[{m}]", host(r["dk"][bi, kvh, sl]), ob["dk"][m], cfg.dtype,
                  floor=floor_of(ob["dk"][m], eb["dk"][m]))
            check(f"dv[{m}]", host(r["dv"][bi, kvh, sl]), ob["dv"][m], cfg.dtype,
                  floor=floor_of(ob["dv"][m], eb["dv"][m]))
