"""Seeded synthetic inputs for gated block-sparse attention (SAS).

This module only draws random numbers and arranges them into arrays. It holds
none of the method's arithmetic (no softmax, no selection, no attention), so
both the CUDA path and the float64 oracle can take their inputs from it.

Every array is produced on the host with numpy's PCG64, split into fixed
chunks that each own a child ``SeedSequence``; the result is therefore the
same on every machine and for every thread count. bf16 inputs are fp32 draws
rounded to nearest-even and returned as float32 arrays whose values are
exactly representable in bf16, so ``torch.from_numpy(x).to(torch.bfloat16)``
is lossless and the oracle sees the exact values the GPU sees.

The presets are shaped like the layers the SAS pages report on (Qwen3-4B,
-8B and -14B attention with grouped-query heads; decode over 64K and 512K
token caches). Draw order: q, k, v, dO, scores (training); q, kcache, vcache,
scores (decode); then the structural tweaks (hot key blocks, recency bias).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_CHUNK = 1 << 22  # elements per independently seeded chunk


def _round_bf16_inplace(x: np.ndarray) -> None:
    """Round float32 values to the nearest bf16 value (ties to even), in place."""
    u = x.view(np.uint32)
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    u &= np.uint32(0xFFFF0000)


def normal(seed_seq: np.random.SeedSequence, shape, std: float = 1.0,
           bf16: bool = False, threads: int | None = None) -> np.ndarray:
    """N(0, std^2) float32 array of ``shape``; optionally rounded to bf16 values."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.float32)
    nch = (n + _CHUNK - 1) // _CHUNK
    kids = seed_seq.spawn(max(nch, 1))

    def fill(i):
        s = i * _CHUNK
        e = min(n, s + _CHUNK)
        g = np.random.Generator(np.random.PCG64(kids[i]))
        g.standard_normal(e - s, dtype=np.float32, out=out[s:e])
        if std != 1.0:
            out[s:e] *= np.float32(std)
        if bf16:
            _round_bf16_inplace(out[s:e])

    if nch <= 1:
        for i in range(nch):
            fill(i)
    else:
        with ThreadPoolExecutor(threads or min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nch)))
    return out.reshape(shape)


@dataclass(frozen=True)
class TrainConfig:
    """A training-layer workload: one gated sparse forward + backward."""
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    d: int
    b: int
    K: int
    dtype: str              # "f32" or "bf16"
    score_std: float = 2.0
    hot_key_frac: float = 0.0   # fraction of key blocks per (batch, kv head) ...
    hot_key_scale: float = 1.0  # ... whose K rows are multiplied by this
    recency: float = 0.0        # scores[j, m] += recency * m / (j - 1) for j >= 2
    seed: int = 0

    @property
    def N(self) -> int:
        return (self.T + self.b - 1) // self.b

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


@dataclass(frozen=True)
class DecodeConfig:
    """A decode workload: one query token per sequence over a KV cache."""
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    b: int
    K: int
    dtype: str = "bf16"
    score_std: float = 2.0
    gate_modes: tuple = (0,)   # use_gates values the workload is run with
    seed: int = 0

    @property
    def C(self) -> int:
        """History blocks before the block holding position L-1."""
        return (self.L - 1) // self.b

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


# The five workloads. Sizes follow the SAS pages' Qwen3 settings; the tiny one
# is the fp32 case the oracle finishes in well under a second.
TINY_F32 = TrainConfig("tiny-f32 B1 Hq2/Hkv1 T256 d64 b16 K4", 1, 2, 1, 256, 64, 16, 4,
                       "f32", score_std=2.0)
QWEN3_4B_TRAIN = TrainConfig("qwen3-4b-train B1 Hq32/Hkv8 T16384 d128 b64 K16", 1, 32, 8,
                             16384, 128, 64, 16, "bf16", score_std=2.0,
                             hot_key_frac=0.05, hot_key_scale=3.0)
QWEN3_8B_TRAIN = TrainConfig("qwen3-8b-train B2 Hq32/Hkv8 T32768 d128 b64 K32", 2, 32, 8,
                             32768, 128, 64, 32, "bf16", score_std=1.5, recency=2.0)
QWEN3_4B_DECODE = DecodeConfig("qwen3-4b-decode B8 Hq32/Hkv8 L65536 d128 b64 K32", 8, 32, 8,
                               65536, 128, 64, 32, score_std=2.0, gate_modes=(0, 1))
QWEN3_14B_DECODE = DecodeConfig("qwen3-14b-decode B1 Hq40/Hkv8 L524288 d128 b64 K64", 1, 40,
                                8, 524288, 128, 64, 64, score_std=2.0, gate_modes=(0,))

PRESETS = {
    "tiny": TINY_F32,
    "qwen3-4b-train": QWEN3_4B_TRAIN,
    "qwen3-8b-train": QWEN3_8B_TRAIN,
    "qwen3-4b-decode": QWEN3_4B_DECODE,
    "qwen3-14b-decode": QWEN3_14B_DECODE,
}


@dataclass
class TrainInputs:
    q: np.ndarray       # [B, Hq, T, d] float32 (bf16-exact when dtype is bf16)
    k: np.ndarray       # [B, Hkv, T, d]
    v: np.ndarray       # [B, Hkv, T, d]
    dO: np.ndarray      # [B, Hq, T, d]
    scores: np.ndarray  # [B, Hkv, N, N] float32; row j is meaningful for m < j
    meta: dict = field(default_factory=dict)


@dataclass
class DecodeInputs:
    q: np.ndarray       # [B, Hq, d]
    kcache: np.ndarray  # [B, Hkv, L, d]
    vcache: np.ndarray  # [B, Hkv, L, d]
    scores: np.ndarray  # [B, Hkv, C] float32
    meta: dict = field(default_factory=dict)


def make_train_inputs(cfg: TrainConfig, seed: int | None = None) -> TrainInputs:
    seed = cfg.seed if seed is None else seed
    root = np.random.SeedSequence(seed)
    s_q, s_k, s_v, s_do, s_s, s_hot = root.spawn(6)
    bf = cfg.dtype == "bf16"
    B, Hq, Hkv, T, d, b, N = cfg.B, cfg.Hq, cfg.Hkv, cfg.T, cfg.d, cfg.b, cfg.N
    q = normal(s_q, (B, Hq, T, d), bf16=bf)
    k = normal(s_k, (B, Hkv, T, d), bf16=False)
    v = normal(s_v, (B, Hkv, T, d), bf16=bf)
    dO = normal(s_do, (B, Hq, T, d), bf16=bf)
    scores = _train_scores(cfg, s_s)
    hot = []
    if cfg.hot_key_frac > 0:
        g = np.random.Generator(np.random.PCG64(s_hot))
        nhot = int(round(cfg.hot_key_frac * N))
        for bi in range(B):
            for h in range(Hkv):
                blocks = np.sort(g.choice(N, size=nhot, replace=False))
                hot.append((bi, h, blocks))
                for m in blocks:
                    k[bi, h, m * b:min(T, (m + 1) * b)] *= np.float32(cfg.hot_key_scale)
    if bf:
        _round_bf16_inplace(k)
    return TrainInputs(q, k, v, dO, scores, meta={"hot_blocks": hot, "seed": seed})


def _train_scores(cfg: TrainConfig, s_s: np.random.SeedSequence) -> np.ndarray:
    N = cfg.N
    scores = normal(s_s, (cfg.B, cfg.Hkv, N, N), std=cfg.score_std)
    if cfg.recency:
        j = np.arange(N, dtype=np.float64)[:, None]
        m = np.arange(N, dtype=np.float64)[None, :]
        ramp = np.where(j >= 2, cfg.recency * m / np.maximum(j - 1, 1), 0.0)
        ramp = np.where(m < j, ramp, 0.0).astype(np.float32)
        scores += ramp[None, None]
    return scores


def make_train_scores(cfg: TrainConfig, seed: int | None = None) -> np.ndarray:
    """Only the selector scores of make_train_inputs (the same values)."""
    seed = cfg.seed if seed is None else seed
    return _train_scores(cfg, np.random.SeedSequence(seed).spawn(6)[4])


def make_decode_scores(cfg: DecodeConfig, seed: int | None = None) -> np.ndarray:
    """Only the selector scores of make_decode_inputs (the same values)."""
    seed = cfg.seed if seed is None else seed
    return normal(np.random.SeedSequence(seed).spawn(4)[3], (cfg.B, cfg.Hkv, cfg.C),
                  std=cfg.score_std)


def make_decode_inputs(cfg: DecodeConfig, seed: int | None = None) -> DecodeInputs:
    seed = cfg.seed if seed is None else seed
    root = np.random.SeedSequence(seed)
    s_q, s_k, s_v, s_s = root.spawn(4)
    bf = cfg.dtype == "bf16"
    q = normal(s_q, (cfg.B, cfg.Hq, cfg.d), bf16=bf)
    kc = normal(s_k, (cfg.B, cfg.Hkv, cfg.L, cfg.d), bf16=bf)
    vc = normal(s_v, (cfg.B, cfg.Hkv, cfg.L, cfg.d), bf16=bf)
    scores = normal(s_s, (cfg.B, cfg.Hkv, cfg.C), std=cfg.score_std)
    return DecodeInputs(q, kc, vc, scores, meta={"seed": seed})


def small_train_config(B=1, Hq=2, Hkv=1, T=64, d=16, b=16, K=2, dtype="f32",
                       score_std=2.0, seed=0, **kw) -> TrainConfig:
    """An ad-hoc training workload for tests (any sizes, including a ragged T)."""
    return TrainConfig(f"adhoc B{B} Hq{Hq}/Hkv{Hkv} T{T} d{d} b{b} K{K} {dtype}", B, Hq, Hkv,
                       T, d, b, K, dtype, score_std=score_std, seed=seed, **kw)


def small_decode_config(B=1, Hq=2, Hkv=1, L=100, d=16, b=16, K=2, dtype="f32",
                        score_std=2.0, seed=0) -> DecodeConfig:
    return DecodeConfig(f"adhoc-decode B{B} Hq{Hq}/Hkv{Hkv} L{L} d{d} b{b} K{K} {dtype}", B,
                        Hq, Hkv, L, d, b, K, dtype, score_std=score_std, seed=seed)


@dataclass
class PagedDecodeInputs:
    q: np.ndarray             # [B, Hq, d]
    kpages: np.ndarray        # [num_pages, Hkv, P, d]
    vpages: np.ndarray        # [num_pages, Hkv, P, d]
    page_indptr: np.ndarray   # [B + 1] int32
    page_indices: np.ndarray  # [page_indptr[-1]] int32, a random placement
    seq_lens: np.ndarray      # [B] int32
    scores: np.ndarray        # [B, Hkv, Cmax] float32; row bi meaningful for its own C
    meta: dict = field(default_factory=dict)


def make_paged_decode_inputs(B: int, Hq: int, Hkv: int, lens, d: int, b: int, P: int,
                             dtype: str = "bf16", score_std: float = 2.0, spare_pages: int = 5,
                             seed: int = 0) -> PagedDecodeInputs:
    """A paged KV cache for decode tests: ragged sequence lengths, pages
    placed at random physical slots (plus unused spare pages, filled with NaN
    so that a read of one shows), the last page of a sequence partly used."""
    root = np.random.SeedSequence(seed)
    s_q, s_k, s_v, s_s, s_p = root.spawn(5)
    bf = dtype == "bf16"
    lens = np.asarray(lens, np.int32)
    npages = [(int(L) + P - 1) // P for L in lens]
    total = sum(npages) + spare_pages
    q = normal(s_q, (B, Hq, d), bf16=bf)
    kp = normal(s_k, (total, Hkv, P, d), bf16=bf)
    vp = normal(s_v, (total, Hkv, P, d), bf16=bf)
    perm = np.random.default_rng(s_p).permutation(total).astype(np.int32)
    indptr = np.concatenate([[0], np.cumsum(npages)]).astype(np.int32)
    indices = perm[:indptr[-1]].copy()
    used = np.zeros(total, bool)
    used[indices] = True
    kp[~used] = np.nan
    vp[~used] = np.nan
    # rows past each sequence's end in its last page: NaN as well
    for bi, L in enumerate(lens):
        last = indices[indptr[bi + 1] - 1]
        tail = int(L) - (npages[bi] - 1) * P
        kp[last, :, tail:] = np.nan
        vp[last, :, tail:] = np.nan
    Cmax = max(1, (int(lens.max()) - 1) // b)
    scores = normal(s_s, (B, Hkv, Cmax), std=score_std)
    return PagedDecodeInputs(q, kp, vp, indptr, indices, lens, scores,
                             meta={"seed": seed, "P": P})
