"""The multi-process plumbing on CPU ranks (gloo, world size 2).

Gated sparse attention has no exchange step: every (batch, KV head) unit is
independent in the gate softmax, selection, forward and backward. These
tests run two gloo ranks that each take a disjoint share of the units of a
small workload (through the oracle, on the CPU), and check that the shares
reassemble into the single-process result, that shard ranges partition the
units, that rank seeds differ, and that the timing reduction returns the
slowest rank's value.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from block_sparse_attention_sas_b200 import dist as D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    from block_sparse_attention_sas_b200 import workloads as W
    from oracle import sas_oracle as O
    assert D.init("gloo", timeout_s=60)
    # timing reduction: slowest rank wins
    t = D.max_over_ranks(1.0 + rank)
    tot = D.sum_over_ranks(1.0)
    # sharded oracle forward+backward over (batch, kv head) units
    cfg = W.small_train_config(B=2, Hq=4, Hkv=2, T=96, d=8, b=16, K=2)
    x = W.make_train_inputs(cfg)
    units = [(bi, h) for bi in range(cfg.B) for h in range(cfg.Hkv)]
    lo, hi = D.shard_range(len(units), world, rank)
    res = {}
    for bi, h in units[lo:hi]:
        sl_b, sl_h = slice(bi, bi + 1), slice(h, h + 1)
        qh = slice(h * cfg.G, (h + 1) * cfg.G)
        g, lg, ix = O.gate_topk(x.scores[sl_b, sl_h], cfg.K)
        o, lse = O.attn_fwd(x.q[sl_b, qh], x.k[sl_b, sl_h], x.v[sl_b, sl_h], ix, lg, cfg.b)
        dq, dk, dv, ds = O.attn_bwd(x.q[sl_b, qh], x.k[sl_b, sl_h], x.v[sl_b, sl_h],
                                    x.dO[sl_b, qh], ix, g, lg, cfg.b)
        res[(bi, h)] = (o, dq, dk, dv, ds)
    D.barrier()
    np.save(os.path.join(out_dir, f"rank{rank}.npy"),
            np.array([t, tot, lo, hi, D.rank_seed(0, rank)], dtype=np.float64))
    np.save(os.path.join(out_dir, f"units{rank}.npy"), np.array(res, dtype=object),
            allow_pickle=True)
    D.shutdown()


def test_shard_range_partitions():
    for n in range(0, 20):
        for world in range(1, 9):
            got = [D.shard_range(n, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [h - l for l, h in got]
            assert max(sizes) - min(sizes) <= 1


def test_rank_seeds_distinct():
    seeds = {D.rank_seed(0, r) for r in range(64)}
    assert len(seeds) == 64 and D.rank_seed(5, 0) == 5


def test_gloo_two_ranks_sharded_units(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    meta = [np.load(tmp_path / f"rank{r}.npy") for r in range(world)]
    assert all(m[0] == 2.0 for m in meta)          # max over ranks
    assert all(m[1] == 2.0 for m in meta)          # sum over ranks
    assert meta[0][4] != meta[1][4]                # distinct rank seeds
    merged = {}
    for r in range(world):
        merged.update(np.load(tmp_path / f"units{r}.npy", allow_pickle=True).item())
    from block_sparse_attention_sas_b200 import workloads as W
    from oracle import sas_oracle as O
    cfg = W.small_train_config(B=2, Hq=4, Hkv=2, T=96, d=8, b=16, K=2)
    x = W.make_train_inputs(cfg)
    g, lg, ix = O.gate_topk(x.scores, cfg.K)
    o, _ = O.attn_fwd(x.q, x.k, x.v, ix, lg, cfg.b)
    dq, dk, dv, ds = O.attn_bwd(x.q, x.k, x.v, x.dO, ix, g, lg, cfg.b)
    assert len(merged) == cfg.B * cfg.Hkv
    for (bi, h), (uo, udq, udk, udv, uds) in merged.items():
        qh = slice(h * cfg.G, (h + 1) * cfg.G)
        np.testing.assert_array_equal(uo[0], o[bi, qh])
        np.testing.assert_array_equal(udq[0], dq[bi, qh])
        np.testing.assert_array_equal(udk[0, 0], dk[bi, h])
        np.testing.assert_array_equal(udv[0, 0], dv[bi, h])
        np.testing.assert_array_equal(uds[0, 0], ds[bi, h])


def test_bench_gpus_flag_launches_ranks_itself():
    """`bench.py --gpus 2` without a torchrun environment re-launches itself
    with two ranks; the dry run does the rank plumbing on gloo/CPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--dry-run", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["dry_run"] is True
