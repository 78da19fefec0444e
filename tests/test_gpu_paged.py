"""GPU parity of the paged KV-cache decode against the float64 oracle.

The pages' deployment decodes from a paged cache (picx.dev summary,
Efficiency Benefits: SGLang with FlashInfer kernels, GQA per-group
selection). These cases use ragged sequence lengths, a partly used last page
per sequence, pages at random physical slots, and NaN in every row the decode
must not read (unused pages and the tail of each last page). Each sequence's
gate + Top-K runs on its own score row through the library, and the decode
through sas_decode_paged; the oracle's decode_paged is the reference.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_sas_b200 import workloads as W
from oracle import sas_oracle as O
from tests.parity_util import check, dev, host

pytestmark = pytest.mark.gpu


def _select(lib, x, K, b):
    """Per-sequence gates / Top-K on the GPU and in the oracle."""
    B, Hkv, Cmax = x.scores.shape
    idx = torch.full((B, Hkv, K), -1, dtype=torch.int32, device="cuda")
    gates = torch.zeros((B, Hkv, Cmax), dtype=torch.float32, device="cuda")
    oidx = np.full((B, Hkv, K), -1, np.int32)
    ologg = np.full((B, Hkv, Cmax), -np.inf)
    for bi, L in enumerate(x.seq_lens):
        C = (int(L) - 1) // b
        if C == 0:
            continue
        s = np.ascontiguousarray(x.scores[bi:bi + 1, :, None, :C])
        g, ix = lib.gate_topk(dev(s, "f32"), K, causal=False)
        idx[bi] = ix[0, :, 0]
        gates[bi, :, :C] = g[0, :, 0]
        _, lg, oi = O.gate_topk(s, K, causal=False)
        oidx[bi] = oi[0, :, 0]
        ologg[bi, :, :C] = lg[0, :, 0]
    np.testing.assert_array_equal(idx.cpu().numpy(), oidx)
    return idx, gates, oidx, ologg


def _paged_tensors(x, dtype="bf16"):
    return (dev(x.q, dtype), dev(x.kpages, dtype), dev(x.vpages, dtype),
            torch.from_numpy(x.page_indptr).cuda(), torch.from_numpy(x.page_indices).cuda(),
            torch.from_numpy(x.seq_lens).cuda())


@pytest.mark.parametrize("P", [16, 32, 64, 128])
@pytest.mark.parametrize("G,Hkv,K", [(4, 2, 8), (5, 1, 16), (8, 2, 4)])
def test_decode_paged_ragged(cuda_lib, P, G, Hkv, K):
    b = 64
    lens = [700, 64, 1000, 1, 129, 2049][: 4 if G == 8 else 6]
    x = W.make_paged_decode_inputs(len(lens), G * Hkv, Hkv, lens, 128, b, P, seed=P + G)
    idx, gates, oidx, ologg = _select(cuda_lib, x, K, b)
    q, kp, vp, ip, ix, ln = _paged_tensors(x)
    for use_gates in (False, True):
        o = cuda_lib.decode_paged(q, kp, vp, ip, ix, ln, idx, gates, use_gates, b,
                                  max_len=int(max(lens)))
        torch.cuda.synchronize()
        assert cuda_lib.device_error()[0] == 0
        want = O.decode_paged(x.q, x.kpages, x.vpages, x.page_indptr, x.page_indices,
                              x.seq_lens, oidx, ologg, b, use_gates=use_gates)
        check(f"paged decode P={P} gates={use_gates}", host(o), want, "bf16")


def test_decode_paged_equals_contiguous_decode(cuda_lib):
    """Uniform lengths: the paged call gives exactly the contiguous decode of
    the gathered caches (same selection, same arithmetic)."""
    b, L, K, P = 64, 3000, 16, 32
    x = W.make_paged_decode_inputs(4, 8, 2, [L] * 4, 128, b, P, seed=3)
    idx, gates, _, _ = _select(cuda_lib, x, K, b)
    q, kp, vp, ip, ix, ln = _paged_tensors(x)
    t = np.arange(L)
    kc = np.stack([x.kpages[x.page_indices[x.page_indptr[bi]:x.page_indptr[bi + 1]][t // P], :,
                            t % P].transpose(1, 0, 2) for bi in range(4)])
    vc = np.stack([x.vpages[x.page_indices[x.page_indptr[bi]:x.page_indptr[bi + 1]][t // P], :,
                            t % P].transpose(1, 0, 2) for bi in range(4)])
    kc, vc = dev(np.ascontiguousarray(kc), "bf16"), dev(np.ascontiguousarray(vc), "bf16")
    for use_gates in (False, True):
        a = cuda_lib.decode_paged(q, kp, vp, ip, ix, ln, idx, gates, use_gates, b, max_len=L)
        c = cuda_lib.decode(q, kc, vc, idx, gates, use_gates, b, L=L)
        torch.cuda.synchronize()
        assert torch.equal(a, c)


def test_decode_paged_bad_page_is_reported(cuda_lib):
    b, K, P = 64, 4, 64
    x = W.make_paged_decode_inputs(2, 4, 1, [500, 300], 128, b, P, seed=9)
    idx, gates, _, _ = _select(cuda_lib, x, K, b)
    q, kp, vp, ip, ix, ln = _paged_tensors(x)
    ix_bad = ix.clone()
    # the last page of sequence 0 holds its current block, which is always read
    ix_bad[int(x.page_indptr[1]) - 1] = kp.shape[0] + 7  # a page past the pool
    cuda_lib.device_error()
    cuda_lib.decode_paged(q, kp, vp, ip, ix_bad, ln, idx, gates, False, b, max_len=500)
    st, raw = cuda_lib.device_error()
    assert st == 6 and raw & 2
