"""Host-side logic of bench.py, checked without a GPU: the grouping of the Qwen3-8B projections
into segmented launches, the byte and launch counts the JSON line reports, and the order of the
library calls one step makes (recorded through a stand-in for the binding)."""
import types

import torch

import bench
import nvfp4_w4a4_gemm_fs_b200.foursight as FS


def test_groups_cover_every_projection_once():
    seen = sorted(j for js in bench.GROUP_PROJ for j in js)
    assert seen == list(range(len(bench.PROJ)))
    for gi, js in enumerate(bench.GROUP_PROJ):
        assert all(bench.PROJ[j][2] == bench.GROUP_K[gi] for j in js)      # one input per group
        assert list(js) == list(range(js[0], js[-1] + 1))                  # adjacent: one alpha slice
        starts = [0]
        for j in js:
            starts.append(starts[-1] + bench.PROJ[j][1])
        assert all(b % 256 == 0 for b in starts[1:-1])                     # no tile straddles two


def test_algorithmic_bytes_read_each_group_input_once_when_fused():
    M, pp = bench.M_PREFILL, 64
    a_bytes = lambda K: M * K // 2 + M * K // 16 + 2 * M * pp
    saved = sum(a_bytes(bench.PROJ[j][2]) for js in bench.GROUP_PROJ for j in js[1:])
    assert bench.gemm_alg_bytes(64, False) - bench.gemm_alg_bytes(64, True) == saved


class _Plan:
    def __init__(self, N, K, p, opts=0):
        self.N, self.K, self.p, self.opts = N, K, p, opts

    def check(self):
        pass


def _fake_lib(calls):
    F = types.SimpleNamespace(Plan=_Plan, StatsState=FS.StatsState, alloc_packed=FS.alloc_packed,
                              stacked_packed=FS.stacked_packed, side_cols=FS.side_cols, FS_OUT_BF16=8)

    def rec(name):
        def f(*a, **k):
            calls.append((name, a, k))
            if name == "fs_select_topk":
                return None, torch.zeros(1, 128, dtype=torch.int32), torch.ones(1)
            return None
        return f
    for n in ("fs_channel_stats", "fs_select_topk", "fs_prepare_weights", "fs_quantize_splice", "fs_splice_gemm",
              "fs_splice_gemm_segmented"):
        setattr(F, n, rec(n))
    return F


def test_fused_step_issues_one_segmented_gemm_per_group(monkeypatch):
    monkeypatch.setattr(bench, "M_PREFILL", 256)
    calls = []
    layer = bench.PrefillLayer(_fake_lib(calls), 256, 64, 2, "cpu", fused=True)
    layer.step()
    names = [c[0] for c in calls]
    assert names.count("fs_splice_gemm_segmented") == 4 and "fs_splice_gemm" not in names
    assert names.count("fs_prepare_weights") == 7 and names.count("fs_quantize_splice") == 4
    for name, a, k in calls:
        if name == "fs_splice_gemm_segmented":
            plan, xq, wq, alpha, seg = a[:5]
            assert seg[0] == 0 and seg[-1] == plan.N == wq.rows and alpha.numel() == len(seg) - 1
            assert k["Y"].shape == (xq.rows, plan.N) and xq.K == plan.K
        if name == "fs_prepare_weights":
            W, out = a[0], k["out"]
            assert out.rows == W.shape[0] and out.K == W.shape[1]
    # the pre-split writes into row slices of the stacked operands
    for gi, js in enumerate(bench.GROUP_PROJ):
        r0 = 0
        for j in js:
            v = layer.wq[j]
            assert v.q.data_ptr() == layer.wq_group[gi].q.data_ptr() + r0 * v.q.stride(0)
            r0 += bench.PROJ[j][1]
    # launch counts the JSON line reports: stats, selection, 3 per pre-split, quantise, GEMMs
    assert layer.launches_per_step(serial=True) == 4 + 2 + 21 + 4 + 4
    assert layer.launches_per_step(serial=False) == 4 + 4 + 21 + 4 + 4


def test_unfused_step_issues_one_gemm_per_projection(monkeypatch):
    monkeypatch.setattr(bench, "M_PREFILL", 256)
    calls = []
    layer = bench.PrefillLayer(_fake_lib(calls), 256, 0, 2, "cpu", fused=False)
    layer.step()
    names = [c[0] for c in calls]
    assert names.count("fs_splice_gemm") == 7 and "fs_splice_gemm_segmented" not in names
    assert layer.gemm_names() == [name for name, _, _, _ in bench.PROJ]


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with the
    keys the benchmark contract names, with no GPU."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"] and "model" not in d["config"]


def test_moe_routing_workloads():
    """The routed-row counts bench.py times: top-8 of 4096 tokens over 64 experts sums to 32768
    rows, and the decode batches (16 / 64 tokens) to 128 / 512 rows; a token picks 8 distinct
    experts, so with 16 tokens no expert holds more than 16 rows (every expert fits the decode
    kernel's 16 token columns)."""
    import synth
    c = synth.moe_routing_counts(0)
    assert c.sum() == 32768 and len(c) == 64
    for tokens in (16, 64):
        d = synth.moe_routing_counts(1, tokens=tokens)
        assert d.sum() == 8 * tokens and d.max() <= tokens and d.min() >= 0
    assert synth.moe_routing_counts(1, tokens=16).max() <= 16
