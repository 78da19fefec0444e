"""Pins of the oracle's paged-cache decode (a "next" row: decode over a
paged KV cache as the pages' deployment uses): it must equal the contiguous
decode it reduces to, be blind to where the pages sit, handle ragged
sequence lengths and partly used last pages, and, with every block selected
and gates off, be plain attention of the last token (torch SDPA)."""
import numpy as np
import torch

from oracle import sas_oracle as O


def _case(seed, B, Hq, Hkv, lens, d, b, K, P, spare=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, d))
    npages = [(L + P - 1) // P for L in lens]
    total = sum(npages) + spare
    kpages = rng.standard_normal((total, Hkv, P, d))
    vpages = rng.standard_normal((total, Hkv, P, d))
    perm = rng.permutation(total)
    indptr = np.concatenate([[0], np.cumsum(npages)])
    indices = perm[:indptr[-1]]
    Cmax = max((L - 1) // b for L in lens)
    scores = rng.standard_normal((B, Hkv, max(Cmax, 1))) * 2
    idx = np.full((B, Hkv, K), -1, np.int32)
    logg = np.full((B, Hkv, max(Cmax, 1)), -np.inf)
    for bi, L in enumerate(lens):
        C = (L - 1) // b
        for h in range(Hkv):
            s = scores[bi, h, :C].astype(np.float32)
            idx[bi, h] = O.topk_row(s, C, K)
            logg[bi, h, :C] = O.log_gates_row(s, C)
    return q, kpages, vpages, indptr, indices, np.asarray(lens), idx, logg


def _gather(kpages, indptr, indices, bi, L):
    P = kpages.shape[2]
    pages = indices[indptr[bi]:indptr[bi + 1]]
    t = np.arange(L)
    return kpages[pages[t // P], :, t % P].transpose(1, 0, 2)


def test_uniform_lengths_equal_contiguous_decode():
    for P in (16, 64):
        q, kp, vp, ip, ix, lens, idx, logg = _case(1, B=3, Hq=4, Hkv=2, lens=[300] * 3, d=8,
                                                   b=64, K=2, P=P)
        kc = np.stack([_gather(kp, ip, ix, bi, 300) for bi in range(3)])
        vc = np.stack([_gather(vp, ip, ix, bi, 300) for bi in range(3)])
        for gates in (False, True):
            got = O.decode_paged(q, kp, vp, ip, ix, lens, idx, logg, 64, use_gates=gates)
            want = O.decode(q, kc, vc, idx, logg, 64, use_gates=gates)
            np.testing.assert_array_equal(got, want)


def test_page_placement_does_not_matter():
    q, kp, vp, ip, ix, lens, idx, logg = _case(2, B=2, Hq=2, Hkv=1, lens=[257, 130], d=8,
                                               b=32, K=3, P=16)
    a = O.decode_paged(q, kp, vp, ip, ix, lens, idx, logg, 32, use_gates=True)
    # move every page to a new physical slot and rewrite the page table
    rng = np.random.default_rng(7)
    perm = rng.permutation(kp.shape[0])
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    b_ = O.decode_paged(q, kp2, vp2, ip, perm[ix], lens, idx, logg, 32, use_gates=True)
    np.testing.assert_array_equal(a, b_)


def test_ragged_lengths_match_single_sequence_decode():
    lens = [65, 200, 64, 1000]
    q, kp, vp, ip, ix, lens_, idx, logg = _case(3, B=4, Hq=6, Hkv=2, lens=lens, d=8, b=64,
                                                K=4, P=32)
    got = O.decode_paged(q, kp, vp, ip, ix, lens_, idx, logg, 64, use_gates=True)
    for bi, L in enumerate(lens):
        kc = _gather(kp, ip, ix, bi, L)[None]
        vc = _gather(vp, ip, ix, bi, L)[None]
        C = (L - 1) // 64
        want = O.decode(q[bi:bi + 1], kc, vc, idx[bi:bi + 1], logg[bi:bi + 1, :, :C], 64,
                        use_gates=True)
        np.testing.assert_array_equal(got[bi], want[0])


def test_full_selection_is_attention_of_the_last_token():
    lens = [193, 77]
    b = 16
    q, kp, vp, ip, ix, lens_, _, logg = _case(4, B=2, Hq=4, Hkv=2, lens=lens, d=8, b=b, K=1,
                                             P=8)
    Cmax = max((L - 1) // b for L in lens)
    idx = np.full((2, 2, Cmax), -1, np.int32)
    for bi, L in enumerate(lens):
        C = (L - 1) // b
        idx[bi, :, :C] = np.arange(C)
    got = O.decode_paged(q, kp, vp, ip, ix, lens_, idx, None, b, use_gates=False)
    for bi, L in enumerate(lens):
        kc = torch.from_numpy(_gather(kp, ip, ix, bi, L)).repeat_interleave(2, 0)
        vc = torch.from_numpy(_gather(vp, ip, ix, bi, L)).repeat_interleave(2, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[bi])[:, None, :], kc, vc)[:, 0]
        assert np.abs(got[bi] - ref.numpy()).max() < 1e-12
