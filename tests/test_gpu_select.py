"""GPU parity of sas_decode_select (the gates and Top-K of the selector
scores, then the decode, in one call) against the float64 oracle: the same
Top-K indices and gates as the oracle's gate_topk, and its decode of the
selected blocks. Tensor-core shapes run the selection inside the decode's
own launch (a cluster of the unit's splits); the others take two launches.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, host

pytestmark = pytest.mark.gpu


def _select_case(lib, dc, use_gates, scores=None):
    x = W.make_decode_inputs(dc)
    s = x.scores if scores is None else scores
    q, kc, vc = (dev(a, dc.dtype) for a in (x.q, x.kcache, x.vcache))
    g = torch.full((dc.B, dc.Hkv, dc.C), float("nan"), device="cuda")
    ix = torch.full((dc.B, dc.Hkv, dc.K), -7, dtype=torch.int32, device="cuda")
    sd = dev(s, "f32")
    lib.device_error()
    o = lib.decode_select(q, kc, vc, sd, dc.K, use_gates, dc.b, L=dc.L, gates=g, idx=ix)
    o2 = lib.decode_select(q, kc, vc, sd, dc.K, use_gates, dc.b, L=dc.L)
    torch.cuda.synchronize()
    assert lib.device_error()[0] == 0
    og, olg, oi = O.gate_topk(s[:, :, None, :], dc.K, causal=False)
    np.testing.assert_array_equal(ix.cpu().numpy(), oi[:, :, 0])
    check("gates", host(g), og[:, :, 0], "f32")
    want = O.decode(x.q, x.kcache, x.vcache, oi[:, :, 0], olg[:, :, 0], dc.b, use_gates=use_gates)
    check("decode_select o", host(o), want, dc.dtype)
    # the optional outputs change nothing in o
    assert torch.equal(o, o2)


@pytest.mark.parametrize("kw", [
    dict(B=2, Hq=8, Hkv=2, L=5000, d=128, b=64, K=16, dtype="bf16"),    # G = 4, 9 splits
    dict(B=1, Hq=10, Hkv=2, L=20000, d=128, b=64, K=64, dtype="bf16"),  # G = 5, 13 splits
    dict(B=3, Hq=24, Hkv=3, L=40000, d=128, b=64, K=32, dtype="bf16"),  # G = 8
    dict(B=2, Hq=4, Hkv=2, L=300, d=128, b=64, K=8, dtype="bf16"),      # K > C
    dict(B=1, Hq=8, Hkv=1, L=64, d=128, b=64, K=2, dtype="bf16"),       # no history
    dict(B=1, Hq=2, Hkv=1, L=3000, d=128, b=64, K=256, dtype="bf16"),   # K = 256
    dict(B=1, Hq=4, Hkv=1, L=70401, d=128, b=64, K=1, dtype="bf16"),    # row wider than its splits
    dict(B=2, Hq=4, Hkv=2, L=1000, d=128, b=64, K=4, dtype="f32"),      # two launches
    dict(B=3, Hq=5, Hkv=1, L=777, d=64, b=16, K=9, dtype="bf16"),       # two launches
])
@pytest.mark.parametrize("use_gates", [False, True])
def test_decode_select_small(cuda_lib, kw, use_gates):
    _select_case(cuda_lib, W.small_decode_config(**kw), use_gates)


@pytest.mark.parametrize("C,levels", [(1000, 1), (3000, 1), (3000, 2), (2500, 0), (2500, -1)])
def test_decode_select_ties_and_spread(cuda_lib, C, levels):
    """Mass ties (every score equal: the long placement, and past 1024
    candidates the per-chunk exact path), two levels, a wide spread (the
    k-th score more than 63/8 below the max: the second histogram), and a
    narrow one (std 0.01: buckets narrowed to the row's span)."""
    dc = W.small_decode_config(B=1, Hq=4, Hkv=1, L=C * 64 + 1, d=128, b=64, K=32, dtype="bf16")
    rng = np.random.default_rng(C + levels)
    if levels > 0:
        s = rng.integers(0, levels, (1, 1, C)).astype(np.float32)
    elif levels == 0:
        s = (rng.standard_normal((1, 1, C)) * 40.0).astype(np.float32)
    else:
        s = (rng.standard_normal((1, 1, C)) * 0.01).astype(np.float32)
    _select_case(cuda_lib, dc, True, scores=s)


@pytest.mark.slow
@pytest.mark.parametrize("name,use_gates", [("qwen3-4b-decode", 1), ("qwen3-14b-decode", 0)])
def test_decode_select_full_size(cuda_lib, name, use_gates):
    _select_case(cuda_lib, W.PRESETS[name], bool(use_gates))


def _pooled_case(lib, dc, use_gates):
    """sas_decode_select_pooled: the scores are the weight-free pooled
    selector's, formed from the key summaries inside the call. The oracle's
    float64 scores decide the selection; a row whose K-th and (K+1)-th oracle
    scores lie within 1e-6 of each other could fall either way in fp32, so
    such a row's indices are compared as a valid Top-K instead."""
    x = W.make_decode_inputs(dc)
    q, kc, vc = (dev(a, dc.dtype) for a in (x.q, x.kcache, x.vcache))
    kbar = lib.block_summaries(kc, dc.b, L=dc.L)
    g = torch.full((dc.B, dc.Hkv, dc.C), float("nan"), device="cuda")
    ix = torch.full((dc.B, dc.Hkv, dc.K), -7, dtype=torch.int32, device="cuda")
    lib.device_error()
    o = lib.decode_select_pooled(q, kc, vc, kbar, dc.K, use_gates, dc.b, L=dc.L, gates=g, idx=ix)
    # the same step through the standalone selector kernel and sas_decode_select
    s_gpu = lib.selector_scores_decode(q, kbar)
    g2 = torch.empty_like(g)
    ix2 = torch.empty_like(ix)
    o2 = lib.decode_select(q, kc, vc, s_gpu, dc.K, use_gates, dc.b, L=dc.L, gates=g2, idx=ix2)
    torch.cuda.synchronize()
    assert lib.device_error()[0] == 0
    assert torch.equal(ix, ix2) and torch.equal(o, o2)
    assert torch.equal(g, g2) or dc.C == 0
    s = O.selector_scores_decode(x.q, x.kcache, dc.L, dc.b)
    og, olg, oi = O.gate_topk(s[:, :, None, :], dc.K, causal=False)
    got = ix.cpu().numpy()
    kk = min(dc.K, dc.C)
    ambiguous = False
    for bi in range(dc.B):
        for h in range(dc.Hkv):
            row = np.sort(s[bi, h])[::-1]
            if kk < dc.C and row[kk - 1] - row[kk] < 1e-6:
                ambiguous = True
                sel = got[bi, h, :kk]
                assert len(set(sel.tolist())) == kk and sel.min() >= 0 and sel.max() < dc.C
                assert s[bi, h, sel].min() >= row[kk - 1] - 1e-6
            else:
                np.testing.assert_array_equal(got[bi, h], oi[bi, h, 0])
    check("pooled gates", host(g), og[:, :, 0], "f32")
    if not ambiguous:
        want = O.decode(x.q, x.kcache, x.vcache, oi[:, :, 0], olg[:, :, 0], dc.b,
                        use_gates=use_gates)
        check("decode_select_pooled o", host(o), want, dc.dtype)


@pytest.mark.parametrize("kw", [
    dict(B=2, Hq=8, Hkv=2, L=5000, d=128, b=64, K=16, dtype="bf16"),    # G = 4, one launch
    dict(B=1, Hq=16, Hkv=2, L=40000, d=128, b=64, K=32, dtype="bf16"),  # G = 8, 2 x 512 + tail
    dict(B=2, Hq=4, Hkv=2, L=300, d=128, b=64, K=8, dtype="bf16"),      # K > C
    dict(B=1, Hq=8, Hkv=1, L=64, d=128, b=64, K=2, dtype="bf16"),       # no history
    dict(B=1, Hq=4, Hkv=1, L=70401, d=128, b=64, K=4, dtype="bf16"),    # row wider than its splits
    dict(B=2, Hq=4, Hkv=2, L=1000, d=128, b=64, K=4, dtype="f32"),      # three launches
    dict(B=3, Hq=5, Hkv=1, L=777, d=64, b=16, K=9, dtype="bf16"),       # three launches
])
@pytest.mark.parametrize("use_gates", [False, True])
def test_decode_select_pooled(cuda_lib, kw, use_gates):
    _pooled_case(cuda_lib, W.small_decode_config(**kw), use_gates)


def test_decode_select_pooled_unaligned_kbar(cuda_lib):
    """Key summaries that are not 16-byte aligned take the three-launch
    path (the selector kernel, then the selection and the decode); the
    results equal the fused call's."""
    dc = W.small_decode_config(B=2, Hq=8, Hkv=2, L=5000, d=128, b=64, K=16, dtype="bf16")
    x = W.make_decode_inputs(dc)
    q, kc, vc = (dev(a, dc.dtype) for a in (x.q, x.kcache, x.vcache))
    kbar = cuda_lib.block_summaries(kc, dc.b, L=dc.L)
    store = torch.empty(kbar.numel() + 1, dtype=torch.float32, device="cuda")
    shifted = store[1:].view(kbar.shape)  # 4 bytes past a 16-byte boundary
    shifted.copy_(kbar)
    assert shifted.data_ptr() % 16 == 4
    ix1 = torch.empty((dc.B, dc.Hkv, dc.K), dtype=torch.int32, device="cuda")
    ix2 = torch.empty_like(ix1)
    o1 = cuda_lib.decode_select_pooled(q, kc, vc, kbar, dc.K, True, dc.b, L=dc.L, idx=ix1)
    o2 = cuda_lib.decode_select_pooled(q, kc, vc, shifted, dc.K, True, dc.b, L=dc.L, idx=ix2)
    torch.cuda.synchronize()
    assert torch.equal(ix1, ix2) and torch.equal(o1, o2)


def test_decode_select_pooled_rejects(cuda_lib):
    """A missing kbar with history, a non-finite selector scale and a kbar of
    the wrong shape are argument errors raised before any launch."""
    dc = W.small_decode_config(B=1, Hq=4, Hkv=1, L=1000, d=128, b=64, K=4, dtype="bf16")
    x = W.make_decode_inputs(dc)
    q, kc, vc = (dev(a, dc.dtype) for a in (x.q, x.kcache, x.vcache))
    kbar = cuda_lib.block_summaries(kc, dc.b, L=dc.L)
    with pytest.raises(RuntimeError):
        cuda_lib.decode_select_pooled(q, kc, vc, kbar, dc.K, True, dc.b, sel_scale=float("nan"))
    with pytest.raises(RuntimeError):
        cuda_lib.decode_select_pooled(q, kc, vc, None, dc.K, True, dc.b)
    with pytest.raises(ValueError):
        cuda_lib.decode_select_pooled(q, kc, vc, kbar[:, :, :-1].contiguous(), dc.K, True, dc.b)


@pytest.mark.slow
@pytest.mark.parametrize("name,use_gates", [("qwen3-14b-decode", 1), ("qwen3-4b-decode", 0)])
def test_decode_select_pooled_full_size(cuda_lib, name, use_gates):
    """The bench's shapes: 512-entry chunks, nine staged pieces a split."""
    _pooled_case(cuda_lib, W.PRESETS[name], bool(use_gates))
