"""Data-parallel exchange of the statistics step on 2 gloo ranks (CPU).

Each rank accumulates the oracle's integer channel moments over its own shard of the tokens; the
all-reduce bench.py performs between ranks (SUM of s1, s2, n; MAX of amax and flags) must give the
full batch's moments exactly, so every rank reselects the same protected channels (FourSight §5.2:
reselection from the statistics gathered over the step).
"""
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from oracle import stats

K, M, P = 256, 96, 16


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _state_tensors(st):
    return types.SimpleNamespace(
        n=torch.tensor([st["n"]], dtype=torch.int64), s1=torch.from_numpy(st["s1"].copy()),
        s2=torch.from_numpy(st["s2"].copy()), amax=torch.from_numpy(st["amax"].view(np.int32).copy()),
        flags=torch.tensor([st["flags"]], dtype=torch.int32))


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    x, _ = synth.outlier_activations(123, M, K, as_bf16=False)
    shard = x[rank::world]                                   # this rank's tokens
    st = stats.accumulate(stats.new_state(K), shard)
    t = _state_tensors(st)
    bench.stats_allreduce_fn(dist)(t)
    merged = {"n": int(t.n.item()), "s1": t.s1.numpy(), "s2": t.s2.numpy(),
              "amax": t.amax.numpy().view(np.float32), "flags": int(t.flags.item())}
    sel = stats.select_topk(merged, P)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), s1=merged["s1"], s2=merged["s2"], amax=merged["amax"],
             n=merged["n"], sel=sel)
    dist.barrier()
    dist.destroy_process_group()


def test_statistics_allreduce_matches_full_batch(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    x, _ = synth.outlier_activations(123, M, K, as_bf16=False)
    full = stats.accumulate(stats.new_state(K), x)
    ref_sel = stats.select_topk(full, P)
    for r in range(world):
        d = np.load(tmp_path / f"rank{r}.npz")
        assert int(d["n"]) == full["n"]
        assert np.array_equal(d["s1"], full["s1"]) and np.array_equal(d["s2"], full["s2"])
        assert np.array_equal(d["amax"], full["amax"])
        assert np.array_equal(d["sel"], ref_sel)
