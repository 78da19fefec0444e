"""GPU parity of the block-selector scores (pooled block summaries, scaled
dot product; evolve.pub review, Frequently asked questions) against the
float64 oracle, training layout and decode, fp32 and bf16 inputs; and the
scores feeding gate + Top-K end to end."""
import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kw", [
    dict(B=1, Hq=8, Hkv=2, T=1000, d=128, b=64, K=3, dtype="bf16"),
    dict(B=2, Hq=4, Hkv=1, T=333, d=64, b=16, K=3, dtype="f32"),
    dict(B=1, Hq=32, Hkv=8, T=4096, d=128, b=64, K=16, dtype="bf16"),
])
def test_selector_scores_training(cuda_lib, kw):
    cfg = W.small_train_config(**kw)
    x = W.make_train_inputs(cfg)
    q, k = dev(x.q, cfg.dtype), dev(x.k, cfg.dtype)
    s = cuda_lib.selector_scores(q, k, cfg.b)
    torch.cuda.synchronize()
    want = O.selector_scores(x.q, x.k, cfg.b)
    check("selector scores", host(s), want, "f32")
    # the scores drive the selection like any others
    _, idx = cuda_lib.gate_topk(s, cfg.K)
    _, _, oi = O.gate_topk(host(s).astype(np.float32), cfg.K)
    np.testing.assert_array_equal(idx.cpu().numpy(), oi)


@pytest.mark.parametrize("kw", [
    dict(B=2, Hq=8, Hkv=2, L=5000, d=128, b=64, K=16, dtype="bf16"),
    dict(B=1, Hq=5, Hkv=1, L=777, d=64, b=16, K=8, dtype="f32"),
])
def test_selector_scores_decode(cuda_lib, kw):
    dc = W.small_decode_config(**kw)
    x = W.make_decode_inputs(dc)
    q, kc = dev(x.q, dc.dtype), dev(x.kcache, dc.dtype)
    kbar = cuda_lib.block_summaries(kc, dc.b, L=dc.L)
    s = cuda_lib.selector_scores_decode(q, kbar)
    torch.cuda.synchronize()
    check("block summaries", host(kbar), O.block_summaries(x.kcache[:, :, :dc.C * dc.b], dc.b),
          "f32")
    check("decode selector scores", host(s), O.selector_scores_decode(x.q, x.kcache, dc.L, dc.b),
          "f32")
