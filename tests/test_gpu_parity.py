"""GPU parity: every call of the C-ABI library against the float64 oracle on
the same seeded inputs.

Small cases compare every element and span several tiles and a ragged tail;
the full-size training layers compare sampled query blocks and key blocks
(the oracle computes those one by one); decode compares every output.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, floor_of, host, oracle_bwd_sample, oracle_fwd_rows, \
    oracle_gates_slice

pytestmark = pytest.mark.gpu


# --------------------------------------------------------------------- gates

@pytest.mark.parametrize("C,K,spread", [(1023, 32, 20.0), (8191, 64, 30.0), (5000, 256, 3.0)])
def test_gate_topk_wide_rows(cuda_lib, C, K, spread):
    """Rows whose k-th largest score lies far below the maximum (a wide
    spread, or a large k): the selection's second histogram level."""
    rng = np.random.default_rng(C + K)
    s = (rng.standard_normal((2, 1, 2, C)) * spread).astype(np.float32)
    _gate_case(cuda_lib, s, K, False)


@pytest.mark.parametrize("C,K", [(1023, 32), (8191, 64), (3000, 100)])
def test_gate_topk_narrow_rows(cuda_lib, C, K):
    """Rows whose scores span far less than one unit (std 0.01, as the
    weight-free selector gives on random data): the selection's buckets
    narrow to the row's span instead of sending every entry to the exact
    path."""
    rng = np.random.default_rng(C + 3 * K)
    s = (rng.standard_normal((2, 1, 2, C)) * 0.01).astype(np.float32)
    _gate_case(cuda_lib, s, K, False)


@pytest.mark.parametrize("C,K", [(1023, 32), (8191, 64), (3000, 64)])
def test_gate_topk_skewed_rows(cuda_lib, C, K):
    """Rows whose largest scores all sit in the entries one lane of a warp
    reads (indices = 0 mod 32): the lanes' own two largest then say little
    about the row, so far more than 256 entries pass the first threshold and
    the warp falls back to sorting its whole chunk."""
    rng = np.random.default_rng(C)
    s = (rng.standard_normal((1, 2, 3, C)) * 0.1).astype(np.float32)
    s[..., ::32] += 5.0 + rng.standard_normal(s[..., ::32].shape).astype(np.float32)
    _gate_case(cuda_lib, s, K, False)


def _gate_case(lib, scores, K, causal):
    g, ix = lib.gate_topk(dev(scores, "f32"), K, causal=causal)
    og, _, oi = O.gate_topk(scores, K, causal=causal)
    np.testing.assert_array_equal(ix.cpu().numpy(), oi)
    check("gates", host(g), og, "f32")


@pytest.mark.parametrize("name", ["tiny", "qwen3-4b-train", "qwen3-8b-train"])
def test_gate_topk_training_configs(cuda_lib, name):
    cfg = W.PRESETS[name]
    _gate_case(cuda_lib, W.make_train_scores(cfg), cfg.K, True)


@pytest.mark.parametrize("name", ["qwen3-4b-decode", "qwen3-14b-decode"])
def test_gate_topk_decode_configs(cuda_lib, name):
    cfg = W.PRESETS[name]
    _gate_case(cuda_lib, W.make_decode_scores(cfg)[:, :, None, :], cfg.K, False)


@pytest.mark.parametrize("C,K,causal,levels", [
    (16, 4, True, 0), (64, 64, True, 0), (200, 5, True, 2), (33, 1, True, 1),
    (1500, 16, True, 0), (5000, 64, False, 0), (70000, 256, False, 0), (3000, 100, False, 3),
    (1, 3, False, 0), (40, 256, False, 0),
    # long-row paths: first chunked size, one block with K = 256 (full-sort
    # fallback), chunked rows with heavy ties, chunked causal rows, many chunks
    (2049, 8, False, 0), (2048, 256, False, 0), (9000, 256, False, 2), (2100, 16, True, 0),
    (20000, 64, False, 0),
    # decode-sized rows (warp-threshold path): 1, 2, 4 and 8 warps per row, ties
    (1023, 32, False, 0), (8191, 64, False, 0), (4096, 64, False, 1), (1800, 64, True, 0),
    (600, 1, False, 3), (7000, 33, False, 2),
    # rows of one warp on either side of the argmax path's K bound (K <= 64:
    # rounds of warp argmax; K = 65: the radix select), with ties, and a
    # full 512-entry row (16 keys a lane)
    (300, 64, True, 2), (300, 65, True, 2), (257, 64, True, 3), (512, 64, False, 0),
    (512, 17, False, 2),
])
def test_gate_topk_edges(cuda_lib, C, K, causal, levels):
    rng = np.random.default_rng(C * 7 + K)
    rows = C if causal else 3
    s = rng.standard_normal((2, 1, rows, C)).astype(np.float32) * 2
    if levels:
        s = rng.integers(0, levels, s.shape).astype(np.float32)
        s[s == 0] = -0.0 if levels > 1 else 0.0  # -0.0 must tie with +0.0
        if levels > 1:
            s[..., ::7] = 0.0
    _gate_case(cuda_lib, s, K, causal)


# ------------------------------------------------------------- fwd + bwd

def _run_train(lib, x, cfg, use_gates=True):
    dt = cfg.dtype
    q, k, v, dO = (dev(a, dt) for a in (x.q, x.k, x.v, x.dO))
    gates, idx = lib.gate_topk(dev(x.scores, "f32"), cfg.K, causal=True)
    gg = gates if use_gates else None
    o, lse = lib.attn_fwd(q, k, v, idx, gg, cfg.b)
    dq, dk, dv, ds = lib.attn_bwd(q, k, v, o, lse, dO, idx, gg, cfg.b)
    torch.cuda.synchronize()
    st, raw = lib.device_error()
    assert st == 0, f"device error bits {raw:#x}"
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, ds=ds, idx=idx, gates=gates)


def _full_compare(lib, cfg, use_gates=True):
    x = W.make_train_inputs(cfg)
    r = _run_train(lib, x, cfg, use_gates)
    g, lg, ix = O.gate_topk(x.scores, cfg.K)
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), ix)
    o, lse = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b, use_gates=use_gates)
    dq, dk, dv, ds = O.attn_bwd(x.q, x.k, x.v, x.dO, ix, g, lg, cfg.b, use_gates=use_gates)
    dt = cfg.dtype
    fl = {n: None for n in ("o", "dq", "dk", "dv")}
    if dt == "bf16":  # the rounding floor of bf16 MMA operands
        oe, _ = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b, use_gates=use_gates, operands="bf16")
        e = O.attn_bwd(x.q, x.k, x.v, x.dO, ix, g, lg, cfg.b, use_gates=use_gates,
                       operands="bf16")
        fl = {"o": floor_of(o, oe), "dq": floor_of(dq, e[0]), "dk": floor_of(dk, e[1]),
              "dv": floor_of(dv, e[2])}
    check("o", host(r["o"]), o, dt, floor=fl["o"])
    check("lse", host(r["lse"]), lse, dt, stored="f32")
    check("dq", host(r["dq"]), dq, dt, floor=fl["dq"])
    check("dk", host(r["dk"]), dk, dt, floor=fl["dk"])
    check("dv", host(r["dv"]), dv, dt, floor=fl["dv"])
    if use_gates:
        check("dscores", host(r["ds"]), ds, dt, stored="f32")
    else:
        assert r["ds"] is None


def test_tiny_f32_config_full(cuda_lib):
    _full_compare(cuda_lib, W.TINY_F32)


@pytest.mark.parametrize("kw", [
    dict(B=1, Hq=4, Hkv=2, T=200, d=64, b=16, K=3, dtype="f32"),
    dict(B=2, Hq=2, Hkv=1, T=130, d=128, b=32, K=2, dtype="f32"),
    dict(B=1, Hq=8, Hkv=2, T=1000, d=128, b=64, K=3, dtype="bf16", hot_key_frac=0.1,
         hot_key_scale=3.0),
    dict(B=2, Hq=4, Hkv=1, T=512, d=128, b=64, K=16, dtype="bf16"),
    dict(B=1, Hq=5, Hkv=1, T=320, d=64, b=64, K=2, dtype="bf16"),
    dict(B=1, Hq=3, Hkv=3, T=64, d=128, b=64, K=4, dtype="bf16"),   # single block, j = 0 only
    dict(B=1, Hq=2, Hkv=1, T=77, d=64, b=16, K=1, dtype="f32"),
    # G = 2 on the tensor-core kernels (one 128-row tile per query block):
    # ragged T, 10% hot key blocks
    dict(B=1, Hq=8, Hkv=4, T=1000, d=128, b=64, K=3, dtype="bf16", hot_key_frac=0.1,
         hot_key_scale=3.0),
    dict(B=2, Hq=4, Hkv=2, T=700, d=128, b=64, K=5, dtype="bf16"),
])
@pytest.mark.parametrize("use_gates", [True, False])
def test_train_small_full(cuda_lib, kw, use_gates):
    _full_compare(cuda_lib, W.small_train_config(**kw), use_gates)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["qwen3-4b-train", "qwen3-8b-train"])
def test_train_full_size_sampled(cuda_lib, name):
    cfg = W.PRESETS[name]
    x = W.make_train_inputs(cfg)
    r = _run_train(cuda_lib, x, cfg)
    N, G, b = cfg.N, cfg.G, cfg.b
    js = [0, 1, 2, cfg.K - 1, cfg.K, cfg.K + 1, N // 2, N - 2, N - 1]
    ms = [0, 1, N // 3, N - 2, N - 1]
    for bi, kvh in ((0, 0), (cfg.B - 1, cfg.Hkv - 1)):
        cache = oracle_gates_slice(x.scores, bi, kvh, cfg.K)
        np.testing.assert_array_equal(r["idx"][bi, kvh].cpu().numpy(), cache[2])
        check("gates", host(r["gates"][bi, kvh]), cache[0], "f32")
        for j in js:
            o, lse = oracle_fwd_rows(x, b, cfg.K, bi, kvh, j, cache=cache)
            oe, _ = oracle_fwd_rows(x, b, cfg.K, bi, kvh, j, cache=cache, operands="bf16")
            sl = slice(j * b, (j + 1) * b)
            check(f"o[{j}]", host(r["o"][bi, kvh * G:(kvh + 1) * G, sl]), o, cfg.dtype,
                  floor=floor_of(o, oe))
            check(f"lse[{j}]", host(r["lse"][bi, kvh * G:(kvh + 1) * G, sl]), lse, cfg.dtype,
                  stored="f32")
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


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_train_reverse_index_past_1024_blocks(cuda_lib, dtype):
    """N = 1025 query blocks: the backward builds its reverse index with the
    warp-ranked list kernel (the bitmap one covers N <= 1024)."""
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=16400, d=64, b=16, K=2, dtype=dtype)
    assert cfg.N > 1024
    _full_compare(cuda_lib, cfg, True)


@pytest.mark.parametrize("kw", [
    dict(B=1, Hq=4, Hkv=2, T=300, d=128, b=64, K=8, dtype="bf16"),     # tensor cores, G = 2
    dict(B=2, Hq=8, Hkv=2, T=1000, d=128, b=64, K=8, dtype="bf16"),    # tensor cores, G = 4
    dict(B=1, Hq=2, Hkv=2, T=200, d=64, b=16, K=8, dtype="bf16"),      # general kernels
])
def test_dense_matches_all_blocks_selected(cuda_lib, kw):
    cfg = W.small_train_config(**kw)
    x = W.make_train_inputs(cfg)
    q, k, v, dO = (dev(a, "bf16") for a in (x.q, x.k, x.v, x.dO))
    o, lse = cuda_lib.dense_fwd(q, k, v, b=cfg.b)
    dq, dk, dv = cuda_lib.dense_bwd(q, k, v, o, lse, dO, b=cfg.b)
    torch.cuda.synchronize()
    assert cuda_lib.device_error()[0] == 0
    oo, ol = O.dense_fwd(x.q, x.k, x.v, cfg.b)
    idx = O.all_blocks_idx(cfg.B, cfg.Hkv, cfg.N)
    odq, odk, odv, _ = O.attn_bwd(x.q, x.k, x.v, x.dO, idx, None, None, cfg.b, use_gates=False)
    oe, _ = O.attn_fwd(x.q, x.k, x.v, idx, None, cfg.b, use_gates=False, operands="bf16")
    e = O.attn_bwd(x.q, x.k, x.v, x.dO, idx, None, None, cfg.b, use_gates=False, operands="bf16")
    check("dense o", host(o), oo, "bf16", floor=floor_of(oo, oe))
    check("dense lse", host(lse), ol, "bf16", stored="f32")
    check("dense dq", host(dq), odq, "bf16", floor=floor_of(odq, e[0]))
    check("dense dk", host(dk), odk, "bf16", floor=floor_of(odk, e[1]))
    check("dense dv", host(dv), odv, "bf16", floor=floor_of(odv, e[2]))


@pytest.mark.slow
def test_dense_long_sequence_sampled(cuda_lib):
    """N = 300 blocks (more than a sparse block list holds): dense forward and
    backward on the tensor cores, checked on sampled query and key blocks
    against the oracle's all-blocks selection."""
    cfg = W.small_train_config(B=1, Hq=4, Hkv=1, T=19200, d=128, b=64, K=8, dtype="bf16")
    x = W.make_train_inputs(cfg)
    q, k, v, dO = (dev(a, "bf16") for a in (x.q, x.k, x.v, x.dO))
    o, lse = cuda_lib.dense_fwd(q, k, v, b=64)
    dq, dk, dv = cuda_lib.dense_bwd(q, k, v, o, lse, dO, b=64)
    torch.cuda.synchronize()
    assert cuda_lib.device_error()[0] == 0
    N = cfg.N
    idx = O.all_blocks_idx(1, 1, N)
    logg = np.zeros((1, 1, N, N))
    for j in (0, 1, 150, N - 1):
        oo, ol = O.attn_fwd_block(x.q, x.k, x.v, idx, logg, 0, 0, j, 64, use_gates=False)
        oe, _ = O.attn_fwd_block(x.q, x.k, x.v, idx, logg, 0, 0, j, 64, use_gates=False,
                                 operands="bf16")
        sl = slice(j * 64, (j + 1) * 64)
        check(f"dense o[{j}]", host(o[0, :, sl]), oo, "bf16", floor=floor_of(oo, oe))
        check(f"dense lse[{j}]", host(lse[0, :, sl]), ol, "bf16", stored="f32")
        r = O.attn_bwd_block(x.q, x.k, x.v, x.dO, idx, logg, 0, 0, j, 64, use_gates=False)
        re_ = O.attn_bwd_block(x.q, x.k, x.v, x.dO, idx, logg, 0, 0, j, 64, use_gates=False,
                               operands="bf16")
        check(f"dense dq[{j}]", host(dq[0, :, sl]), r["dq"], "bf16",
              floor=floor_of(r["dq"], re_["dq"]))
    for m in (N - 1, N - 3):
        acc = {op: [np.zeros((64, 128)), np.zeros((64, 128))] for op in (None, "bf16")}
        for j in range(m, N):
            for op in (None, "bf16"):
                r = O.attn_bwd_block(x.q, x.k, x.v, x.dO, idx, logg, 0, 0, j, 64,
                                     use_gates=False, operands=op)
                sel = (r["cols"] >= m * 64) & (r["cols"] < (m + 1) * 64)
                acc[op][0] += r["dk_c"][sel]
                acc[op][1] += r["dv_c"][sel]
        sl = slice(m * 64, (m + 1) * 64)
        (dkm, dvm), (dke, dve) = acc[None], acc["bf16"]
        check(f"dense dk[{m}]", host(dk[0, 0, sl]), dkm, "bf16", floor=floor_of(dkm, dke))
        check(f"dense dv[{m}]", host(dv[0, 0, sl]), dvm, "bf16", floor=floor_of(dvm, dve))


# ------------------------------------------------------------------ decode

def _decode_case(lib, dc, use_gates, dense_too=False):
    x = W.make_decode_inputs(dc)
    s = x.scores[:, :, None, :]
    gates, idx = lib.gate_topk(dev(s, "f32"), dc.K, causal=False)
    og, olg, oi = O.gate_topk(s, dc.K, causal=False)
    np.testing.assert_array_equal(idx.cpu().numpy(), oi)
    q, kc, vc = (dev(a, dc.dtype) for a in (x.q, x.kcache, x.vcache))
    o = lib.decode(q, kc, vc, idx[:, :, 0].contiguous(), gates[:, :, 0].contiguous(), use_gates,
                   dc.b, L=dc.L)
    torch.cuda.synchronize()
    assert lib.device_error()[0] == 0
    want = O.decode(x.q, x.kcache, x.vcache, oi[:, :, 0], olg[:, :, 0], dc.b, use_gates=use_gates)
    check("decode o", host(o), want, dc.dtype)
    if dense_too:
        od = lib.dense_decode(q, kc, vc, L=dc.L)
        torch.cuda.synchronize()
        check("dense decode o", host(od), O.dense_decode(x.q, x.kcache, x.vcache), dc.dtype)


@pytest.mark.parametrize("kw", [
    dict(B=2, Hq=4, Hkv=2, L=1000, d=128, b=64, K=4, dtype="f32"),
    dict(B=3, Hq=5, Hkv=1, L=777, d=64, b=16, K=9, dtype="bf16"),
    dict(B=1, Hq=8, Hkv=1, L=64, d=128, b=64, K=2, dtype="bf16"),     # no history
    dict(B=1, Hq=2, Hkv=2, L=65, d=128, b=64, K=2, dtype="bf16"),     # 1 token current block
    dict(B=2, Hq=12, Hkv=4, L=4099, d=128, b=32, K=200, dtype="bf16"),
    dict(B=2, Hq=16, Hkv=2, L=5000, d=128, b=64, K=16, dtype="bf16"),  # G = 8 with history
    dict(B=1, Hq=1, Hkv=1, L=50000, d=64, b=64, K=7, dtype="f32"),
])
@pytest.mark.parametrize("use_gates", [False, True])
def test_decode_small(cuda_lib, kw, use_gates):
    _decode_case(cuda_lib, W.small_decode_config(**kw), use_gates, dense_too=True)


@pytest.mark.slow
@pytest.mark.parametrize("name,use_gates", [("qwen3-4b-decode", 0), ("qwen3-4b-decode", 1),
                                            ("qwen3-14b-decode", 0)])
def test_decode_full_size(cuda_lib, name, use_gates):
    _decode_case(cuda_lib, W.PRESETS[name], bool(use_gates), dense_too=(use_gates == 0))


# ------------------------------------------------------------ device errors

def test_bad_index_is_reported_not_faulted(cuda_lib):
    cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=128, d=64, b=32, K=2, dtype="f32")
    x = W.make_train_inputs(cfg)
    q, k, v = (dev(a, "f32") for a in (x.q, x.k, x.v))
    idx = torch.full((1, 1, cfg.N, 2), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, 1, 0] = 3   # block 3 is not in the history of block 1
    cuda_lib.device_error()
    cuda_lib.attn_fwd(q, k, v, idx, None, cfg.b)
    st, raw = cuda_lib.device_error()
    assert st == 6 and raw & 2


@pytest.mark.parametrize("path", ["simt", "tc"])
def test_negative_index_other_than_minus_one_is_reported(cuda_lib, path):
    """-1 marks an empty slot; any other negative entry is a bad index."""
    if path == "simt":
        cfg = W.small_train_config(B=1, Hq=2, Hkv=1, T=128, d=64, b=32, K=2, dtype="f32")
    else:
        cfg = W.small_train_config(B=1, Hq=4, Hkv=1, T=256, d=128, b=64, K=2, dtype="bf16")
    x = W.make_train_inputs(cfg)
    q, k, v = (dev(a, cfg.dtype) for a in (x.q, x.k, x.v))
    idx = torch.full((1, 1, cfg.N, 2), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, 2, 1] = -5
    cuda_lib.device_error()
    cuda_lib.attn_fwd(q, k, v, idx, None, cfg.b)
    st, raw = cuda_lib.device_error()
    assert st == 6 and raw & 2
    dc = W.small_decode_config(B=1, Hq=4, Hkv=1, L=1000, d=128, b=64, K=4,
                               dtype=cfg.dtype if path == "tc" else "f32")
    xd = W.make_decode_inputs(dc)
    qd, kc, vc = (dev(a, dc.dtype) for a in (xd.q, xd.kcache, xd.vcache))
    ix = torch.tensor([[[0, -7, 3, -1]]], dtype=torch.int32, device="cuda")
    cuda_lib.decode(qd, kc, vc, ix, None, False, dc.b, L=dc.L)
    st, raw = cuda_lib.device_error()
    assert st == 6 and raw & 2


def test_wait_timeout_is_reported(cuda_lib):
    cuda_lib.device_error()
    cuda_lib.set_wait_limit(2000)
    try:
        cuda_lib.selftest_wait_timeout()
        st, raw = cuda_lib.device_error()
    finally:
        cuda_lib.set_wait_limit(0)
    assert st == 4 and raw & 1
    # the context stays usable
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


@pytest.mark.parametrize("kw", [
    dict(B=2, Hq=8, Hkv=2, L=1000, d=128, b=64, K=6, dtype="bf16"),
    dict(B=1, Hq=5, Hkv=1, L=4033, d=128, b=64, K=9, dtype="bf16"),
    dict(B=2, Hq=4, Hkv=2, L=1000, d=128, b=64, K=4, dtype="f32"),
])
def test_decode_cache_capacity_tail_is_ignored(cuda_lib, kw):
    """Caches of capacity Lcap > L: rows L.. hold NaN and must not reach o."""
    dc = W.small_decode_config(**kw)
    x = W.make_decode_inputs(dc)
    s = x.scores[:, :, None, :]
    gates, idx = cuda_lib.gate_topk(dev(s, "f32"), dc.K, causal=False)
    og, olg, oi = O.gate_topk(s, dc.K, causal=False)
    q = dev(x.q, dc.dtype)
    Lcap = dc.L + 200
    caches = []
    for a in (x.kcache, x.vcache):
        full = torch.full((dc.B, dc.Hkv, Lcap, dc.d), float("nan"), device="cuda",
                          dtype=torch.bfloat16 if dc.dtype == "bf16" else torch.float32)
        full[:, :, :dc.L] = dev(a, dc.dtype)
        caches.append(full)
    for use_gates in (False, True):
        o = cuda_lib.decode(q, caches[0], caches[1], idx[:, :, 0].contiguous(),
                            gates[:, :, 0].contiguous(), use_gates, dc.b, L=dc.L)
        torch.cuda.synchronize()
        assert cuda_lib.device_error()[0] == 0
        want = O.decode(x.q, x.kcache, x.vcache, oi[:, :, 0], olg[:, :, 0], dc.b,
                        use_gates=use_gates)
        check("decode o (Lcap > L)", host(o), want, dc.dtype)
    od = cuda_lib.dense_decode(q, caches[0], caches[1], L=dc.L)
    torch.cuda.synchronize()
    check("dense decode o (Lcap > L)", host(od), O.dense_decode(x.q, x.kcache, x.vcache),
          dc.dtype)


def test_decode_idx_with_holes(cuda_lib):
    """-1 entries anywhere in an idx row are skipped (decode and oracle alike)."""
    dc = W.small_decode_config(B=2, Hq=8, Hkv=2, L=3000, d=128, b=64, K=12, dtype="bf16")
    x = W.make_decode_inputs(dc)
    s = x.scores[:, :, None, :]
    og, olg, oi = O.gate_topk(s, dc.K, causal=False)
    oi = oi.copy()
    oi[0, 0, 0, 3] = -1
    oi[1, 1, 0, 0] = -1
    oi[1, 0, 0, 5:9] = -1
    q, kc, vc = (dev(a, "bf16") for a in (x.q, x.kcache, x.vcache))
    idx = torch.from_numpy(oi[:, :, 0].copy()).cuda()
    gates = dev(og[:, :, 0].astype(np.float32), "f32")
    for use_gates in (False, True):
        o = cuda_lib.decode(q, kc, vc, idx, gates, use_gates, dc.b, L=dc.L)
        torch.cuda.synchronize()
        assert cuda_lib.device_error()[0] == 0
        lg = np.log(og[:, :, 0].astype(np.float32).astype(np.float64))
        want = O.decode(x.q, x.kcache, x.vcache, oi[:, :, 0], lg, dc.b, use_gates=use_gates)
        check("decode o (holes)", host(o), want, "bf16")
