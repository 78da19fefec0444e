"""Pins of the oracle's block-selector scores (pooled block summaries and a
scaled dot product; the weight-free reading of the evolve.pub review's
"pooling-based block summaries").

The score is bilinear, so it must equal the mean over every (query row, head,
key) pair of the two blocks of the attention logit scale * q_i . k_t, taken
here by brute force from the full logit matrix: a different route than
pooling first. Further pins: constant keys pool to themselves, a partial last
block averages only its valid rows, and the decode scores are the training
scores' row of the block holding the last token when that token is the only
query row (G = 1, b = 1 reduces to plain logits)."""
import numpy as np

from oracle import sas_oracle as O


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_scores_equal_mean_of_pair_logits():
    B, Hq, Hkv, T, d, b = 2, 4, 2, 45, 8, 8
    q, k = _rand(1, B, Hq, T, d), _rand(2, B, Hkv, T, d)
    s = O.selector_scores(q, k, b)
    G, N, scale = Hq // Hkv, (T + b - 1) // b, 1 / np.sqrt(d)
    for bi in range(B):
        for h in range(Hkv):
            logits = np.stack([q[bi, h * G + g] @ k[bi, h].T for g in range(G)]) * scale
            for j in range(N):
                rows = slice(j * b, min(T, (j + 1) * b))
                for m in range(N):
                    cols = slice(m * b, min(T, (m + 1) * b))
                    want = logits[:, rows, cols].mean() if m < j else 0.0
                    assert abs(s[bi, h, j, m] - want) < 1e-12


def test_constant_and_partial_blocks():
    k = np.zeros((1, 1, 10, 3))
    k[0, 0, :4] = [1.0, 2.0, 3.0]     # block 0 constant
    k[0, 0, 8:] = [[2.0, 0, 0], [4.0, 0, 0]]  # partial last block of 2 rows (b = 4)
    kbar = O.block_summaries(k, 4)
    np.testing.assert_array_equal(kbar[0, 0, 0], [1.0, 2.0, 3.0])
    np.testing.assert_array_equal(kbar[0, 0, 2], [3.0, 0.0, 0.0])


def test_decode_scores_are_plain_logits_for_single_rows():
    q, k = _rand(3, 2, 3, 16), _rand(4, 2, 3, 9, 16)
    s = O.selector_scores_decode(q, k, L=9, b=1)
    want = np.einsum("bhd,bhmd->bhm", q, k[:, :, :8]) / 4.0
    np.testing.assert_allclose(s, want, rtol=0, atol=1e-12)


def test_decode_scores_match_training_rows():
    B, Hq, Hkv, T, d, b = 1, 2, 1, 96, 8, 16
    q, k = _rand(5, B, Hq, T, d), _rand(6, B, Hkv, T, d)
    s = O.selector_scores(q, k, b)
    # a decode query whose group summary equals block j's query summary
    j = 5
    qbar = q[:, :, j * b:(j + 1) * b].mean(axis=2)          # [B, Hq, d]
    sd = O.selector_scores_decode(qbar, k, L=j * b + 1, b=b)  # history = blocks 0..j-1
    np.testing.assert_allclose(sd[0, 0], s[0, 0, j, :j], rtol=0, atol=1e-12)
