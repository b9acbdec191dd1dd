"""Data-parallel exchanges of the SpliceGEMM path on 2 gloo ranks (CPU): nvfp4_w4a4_gemm_fs_b200.dp.

Statistics: each rank accumulates the oracle's integer channel moments over its own shard of the
tokens; dp.allreduce_stats (SUM of s1, s2, n; MAX of amax and flags) must give the full batch's
moments exactly, so every rank reselects the same protected channels (FourSight §5.2: reselection
from the statistics gathered over the step).

Packed weights: rank 0's pre-split (codes, tiled scales, W'_S, gW, alpha) is broadcast with
dp.broadcast_packed; every rank must then hold the oracle's pre-split for the agreed channels byte for
byte, with no requantisation (FourSight §5.2: packed weights synchronised without re-quantization), and
its own shard's SpliceGEMM rows with those weights equal the full batch's.
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
    from nvfp4_w4a4_gemm_fs_b200 import dp
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    x, _ = synth.outlier_activations(123, M, K, as_bf16=False)
    shard = x[rank::world]                                   # this rank's tokens
    st = stats.accumulate(stats.new_state(K), shard)
    t = _state_tensors(st)
    dp.allreduce_stats(t)
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


N_W = 128


def _packed_from_oracle(ref, K, p):
    """Torch CPU tensors of a pre-split in the library's packed layout (q, tiled sf, side bf16)."""
    from nvfp4_w4a4_gemm_fs_b200 import foursight as Fs
    from oracle import nvfp4
    q = torch.from_numpy(nvfp4.pack_codes(ref["codes"]))
    sf = torch.from_numpy(nvfp4.sf_to_tiled(ref["sf"], K))
    side = torch.from_numpy(nvfp4.bf16_bits(ref["ws"]).view(np.int16)).view(torch.bfloat16)
    return Fs.Packed(q, sf, side, ref["codes"].shape[0], K, p)


def _broadcast_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from datetime import timedelta

    from nvfp4_w4a4_gemm_fs_b200 import dp
    from nvfp4_w4a4_gemm_fs_b200 import foursight as Fs
    from oracle import splice
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    x, _ = synth.outlier_activations(321, M, K, as_bf16=False)
    w = synth.gaussian_weights(322, N_W, K, as_bf16=False)
    t = _state_tensors(stats.accumulate(stats.new_state(K), x[rank::world]))
    dp.allreduce_stats(t)
    merged = {"n": int(t.n.item()), "s1": t.s1.numpy(), "s2": t.s2.numpy(),
              "amax": t.amax.numpy().view(np.float32), "flags": int(t.flags.item())}
    sel = stats.select_topk(merged, P)
    gA = stats.next_gain(merged, sel)
    pp = splice.padded_p(P)
    if rank == 0:                                            # the only rank that runs the pre-split
        ref = splice.prepare_weights(w, sel, gA)
        packed = _packed_from_oracle(ref, K, P)
        gW = torch.tensor([float(ref["gW"])], dtype=torch.float32)
        alpha = torch.tensor([float(ref["alpha"])], dtype=torch.float32)
    else:                                                    # receivers: empty buffers of the same shapes
        packed = Fs.Packed(torch.zeros(N_W, K // 2, dtype=torch.uint8),
                           torch.zeros(((N_W + 127) // 128) * 128 * ((K // 16 + 3) // 4) * 4, dtype=torch.uint8),
                           torch.zeros(N_W, pp, dtype=torch.bfloat16), N_W, K, P)
        gW = torch.zeros(1, dtype=torch.float32)
        alpha = torch.zeros(1, dtype=torch.float32)
    dp.broadcast_packed(packed, gW, alpha, src=0)
    # this rank's shard through the oracle's activation path and the received weights
    from oracle import nvfp4
    wr = {"codes": nvfp4.unpack_codes(packed.q.numpy()), "sf": nvfp4.sf_from_tiled(packed.sf.numpy(), N_W, K),
          "ws": nvfp4.bf16_value(packed.side.contiguous().view(torch.int16).numpy().view(np.uint16)),
          "alpha": np.float32(alpha.item())}
    xr = splice.quantize_splice(x[rank::world], sel, gA)
    Y, _ = splice.splice_gemm(xr, wr, wr["alpha"])
    np.savez(os.path.join(out_dir, f"bc{rank}.npz"), q=packed.q.numpy(), sf=packed.sf.numpy(),
             side=packed.side.contiguous().view(torch.int16).numpy(), gW=gW.numpy(), alpha=alpha.numpy(),
             sel=sel, Y=Y)
    dist.barrier()
    dist.destroy_process_group()


def test_packed_weight_broadcast_without_requantisation(tmp_path):
    from oracle import nvfp4, splice
    world = 2
    mp.spawn(_broadcast_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    x, _ = synth.outlier_activations(321, M, K, as_bf16=False)
    w = synth.gaussian_weights(322, N_W, K, as_bf16=False)
    full = stats.accumulate(stats.new_state(K), x)
    sel = stats.select_topk(full, P)
    gA = stats.next_gain(full, sel)
    ref = splice.prepare_weights(w, sel, gA)
    Yfull, _ = splice.splice_gemm(splice.quantize_splice(x, sel, gA), ref, ref["alpha"])
    for r in range(world):
        d = np.load(tmp_path / f"bc{r}.npz")
        assert np.array_equal(d["sel"], sel)
        assert np.array_equal(d["q"], nvfp4.pack_codes(ref["codes"]))
        assert np.array_equal(d["sf"], nvfp4.sf_to_tiled(ref["sf"], K))
        assert np.array_equal(d["side"].view(np.uint16), nvfp4.bf16_bits(ref["ws"]))
        assert d["gW"][0] == ref["gW"] and d["alpha"][0] == ref["alpha"]
        assert np.array_equal(d["Y"], Yfull[r::world])           # rank r's rows of the full batch


def _mismatch_worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from datetime import timedelta

    from nvfp4_w4a4_gemm_fs_b200 import dp
    from nvfp4_w4a4_gemm_fs_b200 import foursight as Fs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    pp = 64 if rank == 0 else 16                                   # rank 1 holds side columns of another p
    packed = Fs.Packed(torch.zeros(N_W, K // 2, dtype=torch.uint8), torch.zeros(1024, dtype=torch.uint8),
                       torch.zeros(N_W, pp, dtype=torch.bfloat16), N_W, K, pp)
    try:
        dp.broadcast_packed(packed, torch.zeros(1), torch.zeros(1), src=0)
        outcome = "sent"
    except ValueError:
        outcome = "refused"
    with open(os.path.join(out_dir, f"mm{rank}.txt"), "w") as f:
        f.write(outcome)
    dist.barrier()
    dist.destroy_process_group()


def test_packed_weight_broadcast_refuses_mismatched_buffers_on_every_rank(tmp_path):
    """A receiver whose buffers differ in size from the sender's makes every rank raise before any
    weight bytes move (no rank is left in a broadcast of another size)."""
    world = 2
    mp.spawn(_mismatch_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        assert open(os.path.join(tmp_path, f"mm{r}.txt")).read() == "refused"
