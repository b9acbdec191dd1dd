"""Benchmark of the SpliceGEMM hot path on B200.

Default workload (one GPU): the Qwen3-8B-shaped prefill pass of FourSight's data-parallel hot
path, M = 8192 tokens (8 x 1024) in bf16, P = 64 protected channels per projection.  One step is
one pass of the per-step path over one layer:

  fs_channel_stats   on the 4 input groups (qkv / o / gate-up / down inputs)
  fs_select_topk     top-64 reselection (batched per K)
  fs_prepare_weights pre-split of the 7 projections with the new protected set
  fs_quantize_splice the 4 activation groups
  fs_splice_gemm_segmented  one launch per input group: q|k|v, o, gate|up, down
                     (--unfused: fs_splice_gemm per projection)

`value` is the whole-step throughput in TFLOP/s, counting 2*M*N*K per projection (the same
numerator for every P).  Inputs (activations and bf16 weights, about 0.85 GB) are larger than the
126 MB L2 and are resident in HBM when timing starts.  Extra keys report the decode path (M in
{1,4,16}, 36 distinct layers per CUDA-graph replay) in GB/s and the overhead against P = 0, and
the mixture-of-experts projections (64 experts: a 32768-row prefill batch in TFLOP/s, decode
batches of 16 and 64 tokens in GB/s).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extras]
                  [--case step|gemm|decode|prep|moe] [--shape ...] [--unfused]

Under torchrun each rank runs its own batch (weak scaling); the only exchange is an all-reduce of
the integer channel statistics before reselection, so every rank selects the same channels.
`--impl reference` times the CPU oracle, as it stands, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SpliceGEMM prefill TFLOPS & decode GB/s at P=64, % of roofline, overhead vs P=0"
PROJ = (("q", 4096, 4096, 0), ("k", 1024, 4096, 0), ("v", 1024, 4096, 0), ("o", 4096, 4096, 1),
        ("gate", 12288, 4096, 2), ("up", 12288, 4096, 2), ("down", 4096, 12288, 3))
GROUP_K = (4096, 4096, 4096, 12288)          # input groups: qkv, o, gate/up, down
GROUP_NAMES = ("qkv", "o", "gate_up", "down")
GROUP_PROJ = tuple(tuple(j for j, pr in enumerate(PROJ) if pr[3] == gi) for gi in range(4))
M_PREFILL = 8192
P_DEFAULT = 64
DECODE_LAYERS = 36


# DRAM traffic of the tensor-core SpliceGEMM over one step (M = 8192, P = 64): ncu
# dram__bytes_read.sum + dram__bytes_write.sum of one launch per shape of the current kernel, summed
# over the step's launches (qkv, o, gate_up, down).  None where no capture of the current kernel
# exists (the one-launch-per-projection form, --unfused).
GEMM_DRAM_BYTES_PER_STEP = {"fused": 1361701376, "unfused": None}


# Issue rate of this kernel's block-scaled MMA alone (kind::mxf4nvf4, 256 x 256 x 64 on CTA pairs and
# 128 x 256 on one CTA, no operand loads or stores), measured once on this machine's B200s: the
# tensor cores' own ceiling for the instruction the SpliceGEMM issues, beside the 4 x BF16 estimate.
FP4_MMA_ONLY_TFLOPS = 8900.0


def gemm_alg_bytes(p, fused=True):
    """Operand and output bytes the GEMMs of a step must move: A and B codes, scales and side
    columns, and the fp32 output.  Fused, each input group's packed activations are read once;
    unfused, once per projection."""
    pp = (p + 15) // 16 * 16
    M = M_PREFILL
    a_bytes = lambda K: M * K // 2 + M * K // 16 + 2 * M * pp
    tot = sum(a_bytes(K) for K in GROUP_K) if fused else sum(a_bytes(K) for _, _, K, _ in PROJ)
    for _, N, K, _ in PROJ:
        tot += N * K // 2 + N * K // 16 + 2 * N * pp + 4 * M * N
    return tot


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# workload
# ------------------------------------------------------------------------------------------
def make_activations(M, K, seed, device):
    """X ~ N(0,1) bf16 with 1% of channels (seeded) scaled by 30."""
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    idx = torch.randperm(K, generator=g, device=device)[: math.ceil(0.01 * K)]
    x[:, idx] *= 30.0
    return x.to(torch.bfloat16)


def make_weights(N, K, seed, device):
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * 0.02).to(torch.bfloat16)


class PrefillLayer:
    """Buffers and launches of one per-step pass over a Qwen3-8B layer."""

    def __init__(self, F, M, p, seed, device, out_bf16=False, fused=True, compact=False, fused_prep=False):
        import torch
        self.F, self.M, self.p, self.fused = F, M, p, fused
        # fused_prep: the paper's order within a step -- reselect from the moments gathered during
        # the previous step, pre-split the weights, then one pass over X that quantises with the
        # new set and gathers the moments for the next step (fs_quantize_splice_stats); otherwise
        # statistics, reselection, pre-split and quantise run as four separate passes
        self.fused_prep = fused_prep and not compact
        self.PHASES = (("select", "prepare_weights", "quantize_stats", "gemm") if self.fused_prep
                       else ("stats", "select", "prepare_weights", "quantize", "gemm"))
        # compacted-K operands (FS_COMPACT_K): the NVFP4 operands hold the K - p unprotected
        # channels, padded to a multiple of 256; the GEMMs run with K = that width
        self.qopts = F.FS_COMPACT_K if compact else 0
        self.KQ = [F.compact_cols(K, p) if compact else K for K in GROUP_K]
        self.X = [make_activations(M, K, seed * 100 + i, device) for i, K in enumerate(GROUP_K)]
        self.W = [make_weights(N, K, seed * 100 + 10 + j, device) for j, (_, N, K, _) in enumerate(PROJ)]
        self.st4 = F.StatsState(3, 4096, device=device)
        self.st12 = F.StatsState(1, 12288, device=device)
        self.P4 = torch.empty(3, max(p, 1), dtype=torch.int32, device=device)[:, :p]
        self.m4 = torch.empty(3, 128, dtype=torch.int32, device=device)
        self.g4 = torch.empty(3, dtype=torch.float32, device=device)
        self.P12 = torch.empty(1, max(p, 1), dtype=torch.int32, device=device)[:, :p]
        self.m12 = torch.empty(1, 384, dtype=torch.int32, device=device)
        self.g12 = torch.empty(1, dtype=torch.float32, device=device)
        self.xq = [F.alloc_packed(M, Kq, p, device) for Kq in self.KQ]
        self.gW = torch.empty(len(PROJ), dtype=torch.float32, device=device)
        self.alpha = torch.empty(len(PROJ), dtype=torch.float32, device=device)   # PROJ order: a group's are adjacent
        popts = F.FS_OUT_BF16 if out_bf16 else 0
        dt = torch.bfloat16 if out_bf16 else torch.float32
        if fused:
            # projections of one input group stacked by rows: one segmented GEMM per group
            self.wq, self.wq_group, self.seg = [None] * len(PROJ), [], []
            for gi, js in enumerate(GROUP_PROJ):
                rows = [PROJ[j][1] for j in js]
                allp, views = F.stacked_packed(rows, self.KQ[gi], p, device)
                self.wq_group.append(allp)
                for j, v in zip(js, views):
                    self.wq[j] = v
                self.seg.append([0] + [sum(rows[:i + 1]) for i in range(len(rows))])
            self.plans = [F.Plan(self.seg[gi][-1], self.KQ[gi], max(p, 1), popts) for gi in range(4)]
            self.Y = [torch.empty(M, self.seg[gi][-1], dtype=dt, device=device) for gi in range(4)]
        else:
            self.wq = [F.alloc_packed(N, self.KQ[gi], p, device) for (_, N, K, gi) in PROJ]
            self.plans = [F.Plan(N, self.KQ[gi], max(p, 1), popts) for (_, N, K, gi) in PROJ]
            self.Y = [torch.empty(M, N, dtype=dt, device=device) for (_, N, K, _) in PROJ]
        self.flops = sum(2.0 * M * N * K for (_, N, K, _) in PROJ)
        # per-group views for the multi-stream step (one selection problem per group)
        self.gstate = []
        for gi in range(4):
            st, gidx = (self.st4, gi) if gi < 3 else (self.st12, 0)
            v = F.StatsState.__new__(F.StatsState)
            v.nprob, v.K = 1, st.K
            v.n, v.s1, v.s2 = st.n[gidx:gidx + 1], st.s1[gidx:gidx + 1], st.s2[gidx:gidx + 1]
            v.amax, v.flags = st.amax[gidx:gidx + 1], st.flags[gidx:gidx + 1]
            self.gstate.append(v)
        self.gP = [self.P4[i:i + 1] for i in range(3)] + [self.P12]
        self.gm = [self.m4[i:i + 1] for i in range(3)] + [self.m12]
        self.gg = [self.g4[i:i + 1] for i in range(3)] + [self.g12]

    def launches_per_step(self, serial=False):
        """Kernel launches of one step: statistics per group, selection (one launch per statistics
        state when serial, one per group on streams), weight pre-split = amax + gain + quantise per
        projection, activation quantise per group, the GEMMs."""
        stats = 0 if self.fused_prep else 4
        return stats + (2 if serial else 4) + 3 * len(PROJ) + 4 + len(self.gemm_fns())

    def mask_gain(self, gi):
        if gi < 3:
            return self.m4[gi], self.g4[gi:gi + 1]
        return self.m12[0], self.g12[0:1]

    def step(self, allreduce=None):
        for fn in self.phase_fns(allreduce):
            fn()

    def group_chain(self, gi, allreduce=None):
        """Everything of input group gi, in dependency order: statistics, reselection, weight
        pre-split of its projections, activation quantise, its GEMMs."""
        F = self.F
        st, gidx = (self.st4, gi) if gi < 3 else (self.st12, 0)
        if not self.fused_prep:
            F.fs_channel_stats(self.X[gi], st, group=gidx)
        if allreduce is not None:
            allreduce(self.gstate[gi])
        g = self.gstate[gi]
        F.fs_select_topk(g, self.p, reset=True, P=self.gP[gi], mask=self.gm[gi], gA=self.gg[gi])
        mask, gA = self.gm[gi][0], self.gg[gi][0:1]
        for j, (_, N, K, pg) in enumerate(PROJ):
            if pg == gi:
                F.fs_prepare_weights(self.W[j], mask, self.p, gA, out=self.wq[j], gW=self.gW[j:j + 1],
                                     alpha=self.alpha[j:j + 1], opts=self.qopts)
        if self.fused_prep:
            F.fs_quantize_splice_stats(self.X[gi], mask, self.p, gA, st, group=gidx, out=self.xq[gi])
        else:
            F.fs_quantize_splice(self.X[gi], mask, self.p, gA, out=self.xq[gi], opts=self.qopts)
        for fn in self.gemm_fns(gi):
            fn()

    def step_streams(self, streams, allreduce=None):
        """The same work as step(), with the four independent input-group chains on four streams."""
        import torch
        main = torch.cuda.current_stream()
        for s_ in streams:
            s_.wait_stream(main)
        for gi, s_ in enumerate(streams):
            with torch.cuda.stream(s_):
                self.group_chain(gi, allreduce)
        for s_ in streams:
            main.wait_stream(s_)

    def phase_fns(self, allreduce=None):
        """The step split into its phases (same order and launches as step())."""
        F = self.F

        def stats():
            for gi in range(4):
                st, gidx = (self.st4, gi) if gi < 3 else (self.st12, 0)
                F.fs_channel_stats(self.X[gi], st, group=gidx)
            if allreduce is not None:
                allreduce(self.st4)
                allreduce(self.st12)

        def select():
            F.fs_select_topk(self.st4, self.p, reset=True, P=self.P4, mask=self.m4, gA=self.g4)
            F.fs_select_topk(self.st12, self.p, reset=True, P=self.P12, mask=self.m12, gA=self.g12)

        def prepare():
            for j, (_, N, K, gi) in enumerate(PROJ):
                mask, g = self.mask_gain(gi)
                F.fs_prepare_weights(self.W[j], mask, self.p, g, out=self.wq[j], gW=self.gW[j:j + 1],
                                     alpha=self.alpha[j:j + 1], opts=self.qopts)

        def quantize():
            for gi in range(4):
                mask, g = self.mask_gain(gi)
                F.fs_quantize_splice(self.X[gi], mask, self.p, g, out=self.xq[gi], opts=self.qopts)

        def quantize_stats():
            for gi in range(4):
                mask, g = self.mask_gain(gi)
                st, gidx = (self.st4, gi) if gi < 3 else (self.st12, 0)
                F.fs_quantize_splice_stats(self.X[gi], mask, self.p, g, st, group=gidx, out=self.xq[gi])

        def gemm():
            for fn in self.gemm_fns():
                fn()
        if self.fused_prep:
            # the moments the reselection reads come from the previous step's pass
            def select_after_exchange():
                if allreduce is not None:
                    allreduce(self.st4)
                    allreduce(self.st12)
                select()
            return [select_after_exchange, prepare, quantize_stats, gemm]
        return [stats, select, prepare, quantize, gemm]

    def gemm_fns(self, group=None):
        """The GEMM launches (of one input group, or all): one segmented launch per group when
        fused, else one per projection."""
        F = self.F
        groups = range(4) if group is None else (group,)
        if self.fused:
            def make_g(gi):
                js = GROUP_PROJ[gi]
                return lambda: F.fs_splice_gemm_segmented(self.plans[gi], self.xq[gi], self.wq_group[gi],
                                                          self.alpha[js[0]:js[-1] + 1], self.seg[gi], Y=self.Y[gi])
            return [make_g(gi) for gi in groups]

        def make(j, gi):
            return lambda: F.fs_splice_gemm(self.plans[j], self.xq[gi], self.wq[j], self.alpha[j:j + 1], Y=self.Y[j])
        return [make(j, gi) for j, (_, N, K, gi) in enumerate(PROJ) if gi in groups]

    def gemm_names(self):
        return list(GROUP_NAMES) if self.fused else [name for name, _, _, _ in PROJ]

    def check(self):
        for pl in self.plans:
            pl.check()


def capture(fn):
    """Capture fn's launches (on a side stream) into a CUDA graph."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        fn()                                   # warm: sets kernel attributes before capture
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def stats_allreduce_fn(dist):
    """The DP exchange: sum the integer moments and counts, max the per-channel maxima
    (nvfp4_w4a4_gemm_fs_b200.dp.allreduce_stats)."""
    from nvfp4_w4a4_gemm_fs_b200 import dp
    return dp.allreduce_stats


def timed(fn, steps, dist=None):
    import torch
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if dist is not None:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms


# ------------------------------------------------------------------------------------------
# decode sweep (M <= 16), CUDA-graph replay over 36 distinct layers
# ------------------------------------------------------------------------------------------
def moe_case(F, p, device, reps=10):
    """Mixture-of-experts projections (grouped path): 64 experts, top-8 routing of 4096 tokens with
    Zipf(1.2) expert popularity (32768 routed rows, expert-contiguous), the up projection (gate and
    up fused, 4096 <- 4096) and the down projection (4096 <- 2048), P = 64 per expert with its own
    statistics, protected set, gains and packed weights.  Times the grouped quantise + grouped
    GEMM and the grouped GEMM alone (graph replays), TFLOP/s = sum over experts of 2*rows*N*K / t."""
    import numpy as np
    import torch

    import synth
    counts = synth.moe_routing_counts(0)
    E, total = len(counts), int(counts.sum())
    offs = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int64, device=device)
    out = {"experts": E, "routed_rows": total, "rows_min_median_max": [int(counts.min()), int(np.median(counts)),
                                                                         int(counts.max())]}
    for name, N, K in (("up", 4096, 4096), ("down", 4096, 2048)):
        X = make_activations(total, K, 31 if name == "up" else 32, device)
        st = F.StatsState(E, K, device=device)
        for e in range(E):
            F.fs_channel_stats(X[int(counts[:e].sum()):int(counts[:e + 1].sum())], st, group=e)
        _, masks, gA = F.fs_select_topk(st, p)
        pp = F.side_cols(p)
        wq = F.Packed(torch.empty(E * N, K // 2, dtype=torch.uint8, device=device),
                      torch.empty(F.sf_bytes(E * N, K), dtype=torch.uint8, device=device),
                      torch.zeros(E * N, max(pp, 8), dtype=torch.bfloat16, device=device)[:, :pp], E * N, K, p)
        alpha = torch.empty(E, dtype=torch.float32, device=device)
        gW = torch.empty(E, dtype=torch.float32, device=device)
        sfb = F.sf_bytes(N, K)
        for e in range(E):
            W = make_weights(N, K, 7000 + e, device)
            F.fs_prepare_weights(W, masks[e], p, gA[e:e + 1], gW=gW[e:e + 1], alpha=alpha[e:e + 1],
                                 out=F.Packed(wq.q[e * N:(e + 1) * N], wq.sf[e * sfb:(e + 1) * sfb],
                                              wq.side[e * N:(e + 1) * N], N, K, p))
            del W
        xq = F.alloc_packed(F.grouped_rows(total, E), K, p, device)
        plan = F.Plan(N, K, max(p, 1))
        Y = torch.empty(total, N, dtype=torch.float32, device=device)

        def gemm():
            F.fs_splice_gemm_grouped(plan, offs, total, xq, wq, alpha, Y=Y)

        def quant_gemm():
            F.fs_quantize_splice_grouped(X, offs, masks, p, gA, out=xq, max_rows=total)
            gemm()
        quant_gemm()
        torch.cuda.synchronize()
        plan.check()
        flops = 2.0 * total * N * K
        res = {"N": N, "K": K}
        for tag, fn in (("gemm", gemm), ("quant+gemm", quant_gemm)):
            g = capture(fn)
            for _ in range(3):
                g.replay()
            ms = timed(g.replay, reps) / reps
            res[tag] = {"us": ms * 1000.0, "TFLOPs": flops / (ms * 1e-3) / 1e12}
            del g
        plan.check()
        # Decode steps of the same layer (the protected sets and packed weights above): 16 and 64
        # tokens routed top-8 (128 / 512 rows; with 16 tokens no expert can exceed 16 rows).  Every
        # expert on the tensor-core kernel (the default) against FS_PATH_DECODE, which sends
        # experts of at most 16 rows to the weight-streaming decode kernel.  GB/s counts the
        # packed weights of the experts with rows, the packed activations and the fp32 outputs.
        pw = N * K // 2 + N * (K // 16) + N * pp * 2
        for tokens in (16, 64):
            dc = synth.moe_routing_counts(1, tokens=tokens)
            dtot = int(dc.sum())
            doffs = torch.tensor(np.concatenate([[0], np.cumsum(dc)]), dtype=torch.int64, device=device)
            Xd = make_activations(dtot, K, 33, device)
            xqd = F.fs_quantize_splice_grouped(Xd, doffs, masks, p, gA, max_rows=dtot)
            Yd = torch.empty(dtot, N, dtype=torch.float32, device=device)
            dbytes = int((dc > 0).sum()) * pw + F.grouped_rows(dtot, E) * (K // 2 + K // 16 + pp * 2) + dtot * N * 4
            dres = {"rows": dtot, "experts_with_rows": int((dc > 0).sum()), "max_rows_per_expert": int(dc.max())}
            for tag, popts in (("tensor_only", 0), ("small_experts_on_decode", F.FS_PATH_DECODE)):
                dplan = F.Plan(N, K, max(p, 1), popts)
                g = capture(lambda: F.fs_splice_gemm_grouped(dplan, doffs, dtot, xqd, wq, alpha, Y=Yd))
                for _ in range(3):
                    g.replay()
                ms = timed(g.replay, reps) / reps
                dplan.check()
                dres[tag] = {"us": ms * 1000.0, "GBps": dbytes / (ms * 1e-3) / 1e9}
                del g
            res[f"decode_{tokens}_tokens"] = dres
            del Xd, xqd, Yd
        out[name] = res
        del X, xq, wq, Y, st
        torch.cuda.empty_cache()
    return out


def rollout_case(F, device, reps=20):
    """The rollout-batch configuration: statistics over 16384 x 4096 bf16 activations (1% channels
    x30), top-64 reselection, and the dual-gate filter over 1024 x 4096 float32 train-engine
    log-probs with groups of G = 16 sequences (tau = 1e-4, K1 = ceil(0.01 * 4096) = 41, K2 = 5,
    35% of sequences with injected tail tokens and runs).  GB/s = bytes read / time."""
    import numpy as np
    import torch

    import synth
    res = {}
    X = make_activations(16384, 4096, 41, device)
    st = F.StatsState(1, 4096, device=device)
    P = torch.empty(1, 64, dtype=torch.int32, device=device)
    mask = torch.empty(1, 128, dtype=torch.int32, device=device)
    gA = torch.empty(1, dtype=torch.float32, device=device)
    g = capture(lambda: F.fs_channel_stats(X, st))
    for _ in range(3):
        g.replay()
    ms = timed(g.replay, reps) / reps
    res["stats"] = {"us": ms * 1000.0, "GBps": X.numel() * 2 / (ms * 1e-3) / 1e9}
    g = capture(lambda: F.fs_select_topk(st, 64, reset=False, P=P, mask=mask, gA=gA))
    for _ in range(3):
        g.replay()
    ms = timed(g.replay, reps) / reps
    res["select"] = {"us": ms * 1000.0, "K": 4096, "p": 64}
    del g, X
    lp, lengths, rewards, _ = synth.rollout_logprobs(5)
    S, T = lp.shape
    logp = torch.from_numpy(lp).to(device)
    lens = torch.from_numpy(lengths).to(device)
    rew = torch.from_numpy(rewards).to(device)
    log_tau = float(np.float32(np.log(1e-4)))
    K1 = int(np.ceil(0.01 * T))
    adv = torch.empty(S, dtype=torch.float32, device=device)
    outs = F.fs_seq_filter(logp, log_tau, K1, 5, lengths=lens, G=16, rewards=rew, adv=adv)
    g = capture(lambda: F.fs_seq_filter(logp, log_tau, K1, 5, lengths=lens, G=16, rewards=rew, adv=adv))
    for _ in range(3):
        g.replay()
    ms = timed(g.replay, reps) / reps
    nbytes = S * T * 4 + S * (4 + 4 + 4 + 1 + 4 + 4)
    res["filter"] = {"us": ms * 1000.0, "GBps": nbytes / (ms * 1e-3) / 1e9, "S": S, "T": T, "K1": K1, "K2": 5,
                     "G": 16, "kept": int(outs[0].sum().item())}
    return res


def training_case(F, device, reps=10):
    """The training-side kernels: the straight-through backward of the q projection at M = 8192
    (dX = dY W, dW = dY^T X in BF16 on the tensor-core kernel, three operand transposes), and the
    Eq. 4 objective with gradient and the K3 metric over 1024 x 4096 fp32 log-probs."""
    import numpy as np
    import torch
    out = {}
    M, N, K = M_PREFILL, 4096, 4096
    g = torch.Generator(device=device).manual_seed(77)
    dY = (torch.randn(M, N, generator=g, device=device) * 1e-3).to(torch.bfloat16)
    X = make_activations(M, K, 78, device)
    W = make_weights(N, K, 79, device)
    plan = F.Plan(256, 256, 1)
    work = torch.empty(F.load().fs_ste_backward_work_bytes(M, N, K), dtype=torch.uint8, device=device)
    dX = torch.empty(M, K, device=device)
    dW = torch.empty(N, K, device=device)
    run = lambda: F.fs_ste_backward(plan, dY, X, W, work=work, dX=dX, dW=dW)
    gr = capture(run)
    for _ in range(3):
        gr.replay()
    ms = timed(gr.replay, reps) / reps
    flops = 2 * 2.0 * M * N * K
    out["ste_backward_q"] = {"us": ms * 1000.0, "TFLOPs": flops / (ms * 1e-3) / 1e12, "M": M, "N": N, "K": K}
    gg = capture(lambda: F.fs_gemm_bf16(plan, dY, W, Y=dX))        # one GEMM alone (W untransposed: timing only)
    for _ in range(3):
        gg.replay()
    ms = timed(gg.replay, reps) / reps
    out["gemm_bf16_8192x4096x4096"] = {"us": ms * 1000.0, "TFLOPs": 2.0 * M * N * K / (ms * 1e-3) / 1e12}
    plan.check()
    del gr, gg, work, dX, dW, dY, X, W
    S, T = 1024, 4096
    rng = np.random.default_rng(5)
    lo = torch.from_numpy((-rng.exponential(0.5, (S, T))).astype(np.float32)).to(device)
    lp = lo + torch.randn(S, T, generator=g, device=device) * 0.1
    adv = torch.randn(S, generator=g, device=device)
    lengths = torch.full((S,), T, dtype=torch.int32, device=device)
    gobj = capture(lambda: F.fs_grpo_objective(lp, lo, adv, 0.2, lengths=lengths))
    for _ in range(3):
        gobj.replay()
    ms = timed(gobj.replay, reps) / reps
    out["grpo_objective"] = {"us": ms * 1000.0, "GBps": 12.0 * S * T / (ms * 1e-3) / 1e9, "S": S, "T": T}
    gk3 = capture(lambda: F.fs_k3_kl(lp, lo, lengths=lengths))
    for _ in range(3):
        gk3.replay()
    ms = timed(gk3.replay, reps) / reps
    out["k3_kl"] = {"us": ms * 1000.0, "GBps": 8.0 * S * T / (ms * 1e-3) / 1e9, "S": S, "T": T}
    return out


def decode_sweep(F, p, device, Ms=(1, 4, 16), layers=DECODE_LAYERS, reps=20, fused=True):
    """Decode GEMMs over `layers` distinct layers' weights (larger than L2 together), M tokens per
    layer: one segmented launch per input group (fused) or one launch per projection."""
    import torch
    res = {}
    st = F.StatsState(1, 4096, device=device)
    calib = make_activations(4096, 4096, 999, device)
    F.fs_channel_stats(calib, st)
    _, m4, g4 = F.fs_select_topk(st, p)
    st12 = F.StatsState(1, 12288, device=device)
    F.fs_channel_stats(make_activations(4096, 12288, 998, device), st12)
    _, m12, g12 = F.fs_select_topk(st12, p)
    units = [list(js) for js in GROUP_PROJ] if fused else [[j] for j in range(len(PROJ))]
    packed = []          # per layer: list of (stacked weights, alpha, segment starts) per launch
    for layer in range(layers):
        row = []
        for js in units:
            rows, K = [PROJ[j][1] for j in js], PROJ[js[0]][2]
            mask, g = (m4[0], g4[0:1]) if K == 4096 else (m12[0], g12[0:1])
            wall, views = F.stacked_packed(rows, K, p, device)
            alpha = torch.empty(len(js), dtype=torch.float32, device=device)
            for i, (j, v) in enumerate(zip(js, views)):
                W = make_weights(PROJ[j][1], K, 5000 + layer * 10 + j, device)
                F.fs_prepare_weights(W, mask, p, g, out=v, alpha=alpha[i:i + 1])
                del W
            row.append((wall, alpha, [0] + [sum(rows[:i + 1]) for i in range(len(rows))]))
        packed.append(row)
    torch.cuda.synchronize()
    wbytes = sum(N * K // 2 + N * (K // 16) + N * F.side_cols(p) * 2 for (_, N, K, _) in PROJ)
    for M in Ms:
        Xs = [make_activations(M, K, 77 + gi, device) for gi, K in enumerate(GROUP_K)]
        xq = [F.alloc_packed(M, K, p, device) for K in GROUP_K]
        plans = [F.Plan(sum(PROJ[j][1] for j in js), PROJ[js[0]][2], max(p, 1)) for js in units]
        Ys = [torch.empty(M, pl_n, dtype=torch.float32, device=device)
              for pl_n in (sum(PROJ[j][1] for j in js) for js in units)]

        def run_layers(mode: str):
            # packed: GEMMs on activations prepared beforehand; quant: fs_quantize_splice per input
            # group, then the GEMMs; fused: fs_decode_splice_gemm, the preparation inside the GEMM
            for layer in range(layers):
                if mode == "quant":
                    for gi, K in enumerate(GROUP_K):
                        mask, g = (m4[0], g4[0:1]) if K == 4096 else (m12[0], g12[0:1])
                        F.fs_quantize_splice(Xs[gi], mask, p, g, out=xq[gi])
                for u, js in enumerate(units):
                    wall, alpha, seg = packed[layer][u]
                    gi = PROJ[js[0]][3]
                    if mode == "fused":
                        K = GROUP_K[gi]
                        mask, g = (m4[0], g4[0:1]) if K == 4096 else (m12[0], g12[0:1])
                        F.fs_decode_splice_gemm(plans[u], Xs[gi], mask, p, g, wall, alpha,
                                                seg_start=seg if len(js) > 1 else None, Y=Ys[u])
                    elif len(js) == 1:
                        F.fs_splice_gemm(plans[u], xq[gi], wall, alpha, Y=Ys[u])
                    else:
                        F.fs_splice_gemm_segmented(plans[u], xq[gi], wall, alpha, seg, Y=Ys[u])

        out = {}
        for tag, mode in (("gemm", "packed"), ("quant+gemm", "quant"), ("fused_prep", "fused")):
            run_layers("quant")
            torch.cuda.synchronize()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                run_layers(mode)             # warm (also sets kernel attributes before capture)
                with torch.cuda.graph(graph, stream=s):
                    run_layers(mode)
            torch.cuda.synchronize()
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            # algorithmic bytes: the weights once; packed activations once per projection (packed,
            # quant) plus the quantiser's bf16 read and packed write per input group (quant), or the
            # bf16 activations once per launch (fused); fp32 outputs
            ybytes = sum(M * N * 4 for (_, N, _, _) in PROJ)
            if mode == "fused":
                abytes = sum(M * PROJ[js[0]][2] * 2 for js in units) + ybytes
            else:
                abytes = sum(M * (K // 2 + K // 16 + F.side_cols(p) * 2) for (_, _, K, _) in PROJ) + ybytes
            xbytes = sum(M * K * 2 + M * (K // 2 + K // 16 + F.side_cols(p) * 2) for K in GROUP_K) if mode == "quant" else 0
            total = layers * (wbytes + abytes + xbytes)
            out[tag] = {"us_per_layer": 1000.0 * ms / layers, "GBps": total / (ms * 1e-3) / 1e9,
                        "bytes_per_layer": wbytes + abytes + xbytes,
                        "launches_per_layer": len(units) + (len(GROUP_K) if mode == "quant" else 0)}
            del graph
        for pl in plans:
            pl.check()
        res[f"M{M}"] = out
    return res, wbytes


def side_slice_bound(p):
    """Tensor time of the BF16 slice relative to the NVFP4 product when both run at their peak
    rates: 2*M*N*Pp flops at a quarter of the NVFP4 rate against 2*M*N*K (4*Pp/K per projection,
    weighted by N*K over the layer).  A kernel whose NVFP4 part runs below peak pays less than this
    in relative terms, since its BF16 slice is the smaller share of a longer loop."""
    pp = (p + 15) // 16 * 16
    return sum(4.0 * N * pp for _, N, K, _ in PROJ) / sum(float(N) * K for _, N, K, _ in PROJ)


def p_variant(F, p, device, streams, args, rank, compact=False):
    """The timed step and its GEMMs at another protected-channel count p (compact: the
    compacted-K operands): step time (one graph replay, captured as the main step) and the sum of
    the GEMM launches' times."""
    import torch
    lay = PrefillLayer(F, M_PREFILL, p, seed=2 + rank, device=device, fused=not args.unfused, compact=compact,
                       fused_prep=args.prep == "fused")
    for _ in range(3):
        lay.step()
    gs = capture(lay.step if args.serial else (lambda: lay.step_streams(streams)))
    for _ in range(3):
        gs.replay()
    ms = timed(gs.replay, args.steps) / args.steps
    gg = [capture(fn) for fn in lay.gemm_fns()]
    for g_ in gg:
        g_.replay()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.steps):
        for g_ in gg:
            g_.replay()
    ev[1].record()
    torch.cuda.synchronize()
    gms = ev[0].elapsed_time(ev[1]) / args.steps
    # per-phase device times (each phase one graph, replayed back to back)
    pg = [capture(fn) for fn in lay.phase_fns()]
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(pg) + 1)]
    evs[0].record()
    for k, g_ in enumerate(pg):
        g_.replay()
        evs[k + 1].record()
    torch.cuda.synchronize()
    phase_us = {name: 1000.0 * evs[k].elapsed_time(evs[k + 1]) for k, name in enumerate(lay.PHASES)}
    lay.check()
    out = {"step_ms": ms, "gemm_ms": gms, "gemm_tflops": lay.flops / (gms * 1e-3) / 1e12,
           "step_tflops": lay.flops / (ms * 1e-3) / 1e12, "phase_us": phase_us}
    del gs, gg, pg, lay
    return out


# ------------------------------------------------------------------------------------------
# reference arm / CPU baseline: the oracle as it stands on a bounded sample
# ------------------------------------------------------------------------------------------
def oracle_sample_step(rows=M_PREFILL, seed=0):
    """One bounded sample of the step through the CPU oracle: the q projection (4096 <- 4096) of
    `rows` tokens (all 8192 by default, 1/11.5 of the step's FLOPs): statistics, top-64 selection,
    weight pre-split, activation quantisation and the float64 SpliceGEMM.  Returns (seconds,
    flops counted as 2*rows*N*K)."""
    import numpy as np

    import synth
    from oracle import splice, stats
    x, _ = synth.outlier_activations(seed, rows, 4096)
    w = synth.gaussian_weights(seed + 1, 4096, 4096)
    X, W = splice.as_f32(x, True), splice.as_f32(w, True)
    t0 = time.perf_counter()
    st = stats.accumulate(stats.new_state(4096), X)
    P = stats.select_topk(st, P_DEFAULT)
    gA = stats.next_gain(st, P)
    wq = splice.prepare_weights(W, P, gA)
    xq = splice.quantize_splice(X, P, gA)
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    dt = time.perf_counter() - t0
    assert np.isfinite(Y).all()
    return dt, 2.0 * rows * 4096 * 4096


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(rows=M_PREFILL):
    dt, flops = oracle_sample_step(rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"q projection 4096x4096 of {rows} of the 8192 tokens, P=64: stats, select, "
                      f"weight pre-split, quantise, float64 SpliceGEMM ({dt:.1f} s)",
            "seconds": dt}


def step_config(world, p, prep):
    """The `config` of both arms' JSON lines: the workload the metric is quoted on."""
    return {"workload": "Qwen3-8B-shaped prefill layer: M=8192 bf16 tokens (8x1024), 7 projections, P=64; "
                        "per step stats + top-64 reselect + weight pre-split + quantise + SpliceGEMM",
            "global_batch": world * M_PREFILL, "seq_len": 1024, "parallelism": f"dp{world}",
            "p": p, "prep": prep,
            "l2": "inputs larger than L2 (0.85 GB of bf16 activations and weights per step)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(max(0, args.warmup)):
        oracle_sample_step(32)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample_step(M_PREFILL)
        times.append(dt)
        flops = fl
    tot = sum(times)
    value = flops * len(times) / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": step_config(args.gpus, args.p, args.prep),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": "q projection 4096x4096 of all 8192 tokens per step, P=64: stats, select, "
                                       "weight pre-split, quantise, float64 SpliceGEMM"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def prep_case(F, args, device):
    """The preparation kernels alone on the q-projection input (8192 x 4096) and weights, for profiling."""
    import torch
    X = make_activations(M_PREFILL, 4096, 3, device)
    W = make_weights(4096, 4096, 4, device)
    st = F.StatsState(1, 4096, device=device)
    xq = F.alloc_packed(M_PREFILL, 4096, args.p, device)
    wq = F.alloc_packed(4096, 4096, args.p, device)
    P = torch.empty(1, args.p, dtype=torch.int32, device=device)
    mask = torch.empty(1, 128, dtype=torch.int32, device=device)
    g = torch.empty(1, dtype=torch.float32, device=device)
    gW = torch.empty(1, dtype=torch.float32, device=device)
    alpha = torch.empty(1, dtype=torch.float32, device=device)

    def run():
        F.fs_channel_stats(X, st)
        F.fs_select_topk(st, args.p, reset=True, P=P, mask=mask, gA=g)
        F.fs_prepare_weights(W, mask[0], args.p, g, out=wq, gW=gW, alpha=alpha)
        F.fs_quantize_splice(X, mask[0], args.p, g, out=xq)

    def run_fused():
        F.fs_select_topk(st, args.p, reset=True, P=P, mask=mask, gA=g)
        F.fs_prepare_weights(W, mask[0], args.p, g, out=wq, gW=gW, alpha=alpha)
        F.fs_quantize_splice_stats(X, mask[0], args.p, g, st, out=xq)
    res = {"case": "prep"}
    for name, fn in (("separate", run), ("fused", run_fused)):
        for _ in range(args.warmup):
            fn()
        res[name + "_us_per_pass"] = timed(fn, args.steps) / args.steps * 1000.0
    # the statistics + quantise part alone, each form as one graph replay
    parts = {"stats+quantize": lambda: (F.fs_channel_stats(X, st), F.fs_quantize_splice(X, mask[0], args.p, g, out=xq)),
             "quantize_stats_fused": lambda: F.fs_quantize_splice_stats(X, mask[0], args.p, g, st, out=xq)}
    for name, fn in parts.items():
        gr = capture(fn)
        for _ in range(3):
            gr.replay()
        us = timed(gr.replay, args.steps) / args.steps * 1000.0
        res[name + "_us"] = us
        res[name + "_GBps"] = (X.numel() * 2 + X.shape[0] * (X.shape[1] // 2 + X.shape[1] // 16)) / (us * 1e-6) / 1e9
    print(json.dumps(res))


def kernel_case(F, args, device):
    """fs_splice_gemm alone on one projection shape (--shape; M=8192 for `gemm`, M=--decode-m for
    `decode`), or fs_splice_gemm_segmented on one fused input group (--shape qkv / gate_up), for
    profiling one kernel."""
    import torch
    if args.case == "prep":
        return prep_case(F, args, device)
    if args.case == "moe":
        print(json.dumps({"case": "moe", **moe_case(F, args.p, device, reps=args.steps)}))
        return
    if args.case == "rollout":
        print(json.dumps({"case": "rollout", **rollout_case(F, device, reps=args.steps)}))
        return
    if args.case == "training":
        print(json.dumps({"case": "training", **training_case(F, device, reps=args.steps)}))
        return
    if args.case == "decode_sweep":
        dec, wbytes = decode_sweep(F, args.p, device, fused=not args.unfused, reps=args.steps)
        print(json.dumps({"case": "decode_sweep", "weight_bytes_per_layer": wbytes, **dec}))
        return
    if args.shape in GROUP_NAMES:
        gi = GROUP_NAMES.index(args.shape)
        rows = [PROJ[j][1] for j in GROUP_PROJ[gi]]
        K = GROUP_K[gi]
    else:
        N, K = {name: (n, k) for name, n, k, _ in PROJ}[args.shape]
        rows = [N]
    N = sum(rows)
    M = M_PREFILL if args.case == "gemm" else args.decode_m
    X = make_activations(M, K, 3, device)
    st = F.StatsState(1, K, device=device)
    F.fs_channel_stats(make_activations(max(M, 2048), K, 3, device), st)
    _, mask, g = F.fs_select_topk(st, args.p)
    wall, views = F.stacked_packed(rows, K, args.p, device)
    alpha = torch.empty(len(rows), dtype=torch.float32, device=device)
    for i, (n, v) in enumerate(zip(rows, views)):
        F.fs_prepare_weights(make_weights(n, K, 4 + i, device), mask[0], args.p, g, out=v, alpha=alpha[i:i + 1])
    seg = [0] + [sum(rows[:i + 1]) for i in range(len(rows))]
    xq = F.fs_quantize_splice(X, mask[0], args.p, g)
    plan = F.Plan(N, K, max(args.p, 1))
    Y = torch.empty(M, N, dtype=torch.float32, device=device)
    if args.case == "decode" and args.decode_prep == "fused":
        run = lambda: F.fs_decode_splice_gemm(plan, X, mask[0], args.p, g, wall, alpha,
                                              seg_start=seg if len(rows) > 1 else None, Y=Y)
    elif len(rows) == 1:
        run = lambda: F.fs_splice_gemm(plan, xq, wall, alpha, Y=Y)
    else:
        run = lambda: F.fs_splice_gemm_segmented(plan, xq, wall, alpha, seg, Y=Y)
    for _ in range(args.warmup):
        run()
    ms = timed(run, args.steps) / args.steps
    plan.check()
    print(json.dumps({"case": args.case, "shape": args.shape, "M": M, "N": N, "K": K, "p": args.p,
                      "decode_prep": args.decode_prep if args.case == "decode" else None,
                      "us": ms * 1000.0, "tflops": 2.0 * M * N * K / (ms * 1e-3) / 1e12}))


# ------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--p", type=int, default=P_DEFAULT)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--serial", action="store_true", help="one stream for the whole step (no group concurrency)")
    ap.add_argument("--case", default="step", choices=["step", "gemm", "decode", "prep", "moe", "decode_sweep", "rollout", "training"],
                    help="step: the full benchmark; gemm / decode: only fs_splice_gemm on one projection "
                         "shape (M=8192, or M=--decode-m) for profiling one kernel; prep: the preparation "
                         "kernels on the q projection; moe: the grouped 64-expert projections alone")
    ap.add_argument("--shape", default="q", choices=[name for name, _, _, _ in PROJ] + list(GROUP_NAMES[::2]),
                    help="projection shape of --case gemm / decode")
    ap.add_argument("--decode-m", type=int, default=16, help="tokens of --case decode (1..16)")
    ap.add_argument("--decode-prep", default="packed", choices=["packed", "fused"],
                    help="--case decode: GEMM on prepared activations, or fs_decode_splice_gemm (preparation "
                         "inside the launch)")
    ap.add_argument("--prep", default="separate", choices=["fused", "separate"],
                    help="fused: reselect from the previous step's moments, then one pass over X for the "
                         "quantise and the next moments (fs_quantize_splice_stats); separate: statistics, "
                         "reselection and quantise as their own passes")
    ap.add_argument("--unfused", action="store_true",
                    help="one GEMM launch per projection instead of one segmented launch per input group")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    use_dist = world > 1
    if use_dist:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device(device))

    import nvfp4_w4a4_gemm_fs_b200 as F
    F.load()
    peaks = _peaks()
    p = args.p

    if args.case != "step":
        return kernel_case(F, args, device)

    layer = PrefillLayer(F, M_PREFILL, p, seed=2 + rank, device=device, fused=not args.unfused,
                         fused_prep=args.prep == "fused")
    allreduce = stats_allreduce_fn(dist) if use_dist else None
    for _ in range(args.warmup):
        layer.step(allreduce)
    torch.cuda.synchronize()
    layer.check()

    # The step is captured once into a CUDA graph and replayed: host launch latency of the 35-38
    # small library calls would otherwise show up as GPU idle time.  Each phase (and each GEMM)
    # is also captured on its own, replayed back to back with events in between, to attribute
    # time per kernel on the device.
    streams = [torch.cuda.Stream() for _ in range(4)]
    if use_dist:
        args.serial = True          # collectives on concurrent streams could be ordered differently per rank
    if args.serial:
        step_graph = capture(lambda: layer.step(allreduce))
    else:
        step_graph = capture(lambda: layer.step_streams(streams, allreduce))
    for _ in range(args.warmup):
        step_graph.replay()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        ms = timed(step_graph.replay, args.steps, dist if use_dist else None)
    layer.check()
    ms_step = ms / args.steps
    value = world * layer.flops / (ms_step * 1e-3) / 1e12

    phase_graphs = [capture(fn) for fn in layer.phase_fns(allreduce)]
    gemm_graphs = [capture(fn) for fn in layer.gemm_fns()]
    phase_us = {name: 0.0 for name in layer.PHASES}
    gemm_names = layer.gemm_names()
    gemm_ms = [[0.0] * len(gemm_names) for _ in range(args.steps)]
    for it_ in range(args.steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(phase_graphs) + len(gemm_graphs) + 1)]
        evs[0].record()
        k = 1
        for g_ in phase_graphs[:-1]:
            g_.replay(); evs[k].record(); k += 1
        for g_ in gemm_graphs:
            g_.replay(); evs[k].record(); k += 1
        torch.cuda.synchronize()
        for i, name in enumerate(layer.PHASES[:-1]):
            phase_us[name] += evs[i].elapsed_time(evs[i + 1]) * 1000.0 / args.steps
        base = len(phase_graphs) - 1
        for j in range(len(gemm_names)):
            gemm_ms[it_][j] = evs[base + j].elapsed_time(evs[base + j + 1])
    layer.check()
    gemm_total_ms = sum(sum(r) for r in gemm_ms) / args.steps
    phase_us["gemm"] = gemm_total_ms * 1000.0
    gemm_tflops = layer.flops / (gemm_total_ms * 1e-3) / 1e12
    per_proj = {name: statistics.mean(r[j] for r in gemm_ms) * 1000.0 for j, name in enumerate(gemm_names)}
    fp4_peak = peaks["bf16_tflops"] * 4.0         # dense NVFP4 = 4x dense BF16 (nominal 9 vs 2.25 PFLOP/s)
    del phase_graphs, gemm_graphs

    # End to end: every step copies its activations in from pinned host memory, runs the step
    # through the library calls and copies all outputs back.  Two buffer sets alternate so that
    # the host->device copy of step i+1, the step i itself and the device->host copy of step i-1
    # run at once on three streams (the copies use the two DMA directions).
    layer2 = PrefillLayer(F, M_PREFILL, p, seed=2 + rank, device=device, fused=not args.unfused,
                          fused_prep=args.prep == "fused")
    sets = [layer, layer2]
    host_x = [x.cpu().pin_memory() for x in layer.X]
    host_y = [[torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in L.Y] for L in sets]
    h2d = sum(x.numel() * x.element_size() for x in host_x)
    d2h = sum(y.numel() * y.element_size() for y in host_y[0])
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in sets]
    ev_run = [torch.cuda.Event() for _ in sets]
    ev_out = [torch.cuda.Event() for _ in sets]
    e2e_i = [0]

    def e2e_step():
        i = e2e_i[0]
        e2e_i[0] += 1
        b = i % 2
        L = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_run[b])          # step i-2 has read this set's activations
            for dx, hx in zip(L.X, host_x):
                dx.copy_(hx, non_blocking=True)
            ev_in[b].record()
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[b])
            if i >= 2:
                s_run.wait_event(ev_out[b])         # step i-2's outputs have left this set
            L.step(allreduce)
            ev_run[b].record()
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            for hy, dy in zip(host_y[b], L.Y):
                hy.copy_(dy, non_blocking=True)
            ev_out[b].record()

    def e2e_run(n):
        main = torch.cuda.current_stream()
        for s_ in (s_in, s_run, s_out):             # after the start event on the main stream ...
            s_.wait_stream(main)
        for _ in range(n):
            e2e_step()
        for s_ in (s_in, s_run, s_out):             # ... and before its end event
            main.wait_stream(s_)

    e2e_steps = max(3, min(args.steps, 6))
    e2e_run(2)
    ms_e2e = timed(lambda: e2e_run(e2e_steps), 1, dist if use_dist else None) / e2e_steps
    e2e_value = world * layer.flops / (ms_e2e * 1e-3) / 1e12
    layer2.check()
    del layer2, sets

    fkey = "fused" if layer.fused else "unfused"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 e2m1/ue4m3 + bf16 side, fp32 accumulate and output",
        "data": "synthetic (seeded N(0,1) activations with 1% channels x30, N(0,0.02) weights)",
        "config": step_config(world, p, args.prep),
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp4_peak, "traffic": GEMM_DRAM_BYTES_PER_STEP[fkey],
                     "traffic_unit": f"DRAM bytes per step (the {len(gemm_names)} GEMM launches; ncu "
                                     "dram__bytes_read.sum + dram__bytes_write.sum per shape; the "
                                     "kernel's later changes move no bytes on this path: a skip of "
                                     "small experts in the grouped tile map, which dense problems "
                                     "never take, and the producer's drain of its copies in flight "
                                     "at loop end, which only waits on barriers)",
                     "algorithmic_bytes": gemm_alg_bytes(p, layer.fused),
                     "kernel": f"splice_gemm_tc_kernel ({len(gemm_names)} launches: {', '.join(gemm_names)}; "
                               "sum 2MNK / sum of CUDA-event times)",
                     "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} x 4 (nominal fp4/bf16 ratio), "
                                    f"of {peaks['source']}",
                     "peak_fp4_mma_only_tflops": FP4_MMA_ONLY_TFLOPS,
                     "frac_vs_mma_only": gemm_tflops / FP4_MMA_ONLY_TFLOPS},
        "gemm_us": per_proj,
        "phase_us": phase_us,
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e,
                "schedule": "two buffer sets; copy-in of step i+1, step i and copy-out of step i-1 on three streams"},
        "gpu_launches": layer.launches_per_step(args.serial) * args.steps,
        "graph": "each timed step is one CUDA-graph replay of the step's launches" +
                 ("" if args.serial else "; the 4 independent input-group chains run on 4 streams"),
    }

    if not args.no_extras and rank == 0:
        # the protected-channel budget: the same step and its GEMMs at P = 0 (the overhead
        # reference) and at P = 256 (FourSight §6.4's larger budget), each captured like the timed step
        del host_x, host_y
        torch.cuda.empty_cache()
        sweep = {}
        for pv in sorted({0, 256} - {p}):
            sweep[pv] = p_variant(F, pv, device, streams, args, rank)
            torch.cuda.empty_cache()
        sweep[p] = {"step_ms": ms_step, "gemm_ms": gemm_total_ms, "gemm_tflops": gemm_tflops,
                    "step_tflops": value / world, "phase_us": phase_us}
        s0 = sweep[0]
        line["overhead_vs_p0"] = {"step_ms_p0": s0["step_ms"], "step_ms_p": ms_step,
                                  "step_overhead": ms_step / s0["step_ms"] - 1.0,
                                  "gemm_ms_p0": s0["gemm_ms"], "gemm_ms_p": gemm_total_ms,
                                  "gemm_overhead": gemm_total_ms / s0["gemm_ms"] - 1.0,
                                  "gemm_tflops_p0": s0["gemm_tflops"]}
        line["p_sweep"] = {str(pv): {**r, "step_overhead_vs_p0": r["step_ms"] / s0["step_ms"] - 1.0,
                                     "gemm_overhead_vs_p0": r["gemm_ms"] / s0["gemm_ms"] - 1.0,
                                     "side_slice_tensor_time": side_slice_bound(pv)}
                           for pv, r in sorted(sweep.items())}
        # compacted-K operands at P = 256 (whole k-tiles of NVFP4 work removed)
        rc = p_variant(F, 256, device, streams, args, rank, compact=True)
        line["p_sweep"]["256_compact_k"] = {**rc, "step_overhead_vs_p0": rc["step_ms"] / s0["step_ms"] - 1.0,
                                            "gemm_overhead_vs_p0": rc["gemm_ms"] / s0["gemm_ms"] - 1.0}
        torch.cuda.empty_cache()
        dec, wbytes = decode_sweep(F, p, device, fused=not args.unfused)
        dec0, wbytes0 = decode_sweep(F, 0, device, Ms=(16,), fused=not args.unfused)
        hbm = peaks["hbm_gbs"]
        line["decode"] = {k: {**v["gemm"], "frac_hbm": v["gemm"]["GBps"] / hbm,
                              "with_quantise": {**v["quant+gemm"], "frac_hbm": v["quant+gemm"]["GBps"] / hbm},
                              "fused_prep": {**v["fused_prep"], "frac_hbm": v["fused_prep"]["GBps"] / hbm}}
                          for k, v in dec.items()}
        line["decode"]["layers"] = DECODE_LAYERS
        line["decode"]["weight_bytes_per_layer"] = wbytes
        line["decode"]["overhead_vs_p0_M16"] = dec["M16"]["gemm"]["us_per_layer"] / dec0["M16"]["gemm"]["us_per_layer"] - 1.0
        line["decode"]["hbm_peak_gbs"] = hbm
        torch.cuda.empty_cache()
        moe = moe_case(F, p, device)
        moe["fp4_peak_tflops"] = fp4_peak
        for nm in ("up", "down"):
            moe[nm]["gemm"]["frac_fp4_peak"] = moe[nm]["gemm"]["TFLOPs"] / fp4_peak
        line["moe"] = moe
        torch.cuda.empty_cache()
        ro = rollout_case(F, device)
        for nm in ("stats", "filter"):
            ro[nm]["frac_hbm"] = ro[nm]["GBps"] / hbm
        line["rollout"] = ro
        torch.cuda.empty_cache()
        tr = training_case(F, device)
        for nm in ("ste_backward_q", "gemm_bf16_8192x4096x4096"):
            tr[nm]["frac_bf16_peak"] = tr[nm]["TFLOPs"] / peaks["bf16_tflops"]
        for nm in ("grpo_objective", "k3_kl"):
            tr[nm]["frac_hbm"] = tr[nm]["GBps"] / hbm
        line["training"] = tr
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line))
    if use_dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
