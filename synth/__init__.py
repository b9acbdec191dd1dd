"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke run.

This module only draws random numbers and stores them; it holds none of the
method's arithmetic (no quantisation, statistics, selection or filtering).
Every generator takes an explicit seed and uses numpy's PCG64, so the CPU
oracle and the CUDA path always see the same bytes.

BF16 tensors are returned as ``uint16`` bit patterns (numpy has no bfloat16);
``bf16_to_f32`` widens them for callers that want float values.  The rounding
from the drawn float32 values to bf16 storage is round-to-nearest-even, the
usual way a bf16 activation or weight tensor comes to exist.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rng", "f32_to_bf16_bits", "bf16_to_f32", "outlier_activations",
    "gaussian_weights", "single_projection", "QWEN3_8B_PROJECTIONS",
    "moe_routing_counts", "rollout_logprobs", "filter_cases_8x64",
]

# Qwen3-8B linear layers as (name, N out features, K in features).
QWEN3_8B_PROJECTIONS = (
    ("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
    ("gate", 12288, 4096), ("up", 12288, 4096), ("down", 4096, 12288),
)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 storage (nearest, ties to even); NaN stays NaN."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(a, dtype=np.float32))
    if nan.any():
        r = np.where(nan, np.uint16(0x7FC0), r)
    return r


def bf16_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_activations(seed: int, M: int, K: int, frac: float = 0.01, scale: float = 30.0,
                        n_outliers: int | None = None, as_bf16: bool = True):
    """X ~ N(0,1) [M,K] with a seeded set of outlier channels multiplied by ``scale``.

    ``n_outliers`` defaults to ceil(frac*K).  Returns (X, outlier_channel_indices);
    X is bf16 bits (uint16) when ``as_bf16`` else float32.
    """
    g = rng(seed)
    n_out = int(np.ceil(frac * K)) if n_outliers is None else int(n_outliers)
    ch = np.sort(g.choice(K, size=n_out, replace=False)) if n_out else np.zeros(0, np.int64)
    x = g.standard_normal((M, K), dtype=np.float32)
    if n_out:
        x[:, ch] *= np.float32(scale)
    return (f32_to_bf16_bits(x) if as_bf16 else x), ch


def gaussian_weights(seed: int, N: int, K: int, std: float = 0.02, as_bf16: bool = True):
    g = rng(seed)
    w = g.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(w) if as_bf16 else w


def single_projection(seed: int = 0):
    """The small single-projection case: X 8x512 fp32 with 8 channels x50, W 256x512 fp32."""
    x, ch = outlier_activations(seed, 8, 512, n_outliers=8, scale=50.0, as_bf16=False)
    w = gaussian_weights(seed + 1000, 256, 512, as_bf16=False)
    return x, w, ch


def moe_routing_counts(seed: int, tokens: int = 4096, experts: int = 64, topk: int = 8,
                       zipf_s: float = 1.2):
    """Per-expert routed-row counts for top-k routing without replacement.

    Expert popularity follows Zipf(s) rank weights, assigned to experts through a
    seeded permutation; each token draws ``topk`` distinct experts with probability
    proportional to those weights (Gumbel-top-k).  Returns int64 counts [experts].
    """
    g = rng(seed)
    w = np.arange(1, experts + 1, dtype=np.float64) ** (-zipf_s)
    perm = g.permutation(experts)
    logw = np.log(w[perm])
    counts = np.zeros(experts, np.int64)
    chunk = 1024
    for t0 in range(0, tokens, chunk):
        n = min(chunk, tokens - t0)
        gum = g.gumbel(size=(n, experts)) + logw
        top = np.argpartition(-gum, topk - 1, axis=1)[:, :topk]
        np.add.at(counts, top.ravel(), 1)
    return counts


def rollout_logprobs(seed: int, S: int = 1024, T: int = 4096, frac_injected: float = 0.35,
                     max_run: int = 512, log_tau: float = float(np.float32(np.log(1e-4)))):
    """Train-engine log-probs [S,T] float32 with tail tokens injected into a seeded subset.

    Normal tokens: logp = -Exp(mean 0.3).  Injected sequences get a mix of isolated tail
    tokens and runs of length U[1,max_run] at random positions, tail logp ~ U(ln 1e-10, ln 1e-4),
    plus a few values exactly at ``log_tau`` and one float32 ulp either side of it.
    Also returns lengths [S] int32 (every 8th sequence shorter) and rewards [S] float32
    (Bernoulli(0.5)).
    """
    g = rng(seed)
    lp = (-g.exponential(0.3, size=(S, T))).astype(np.float32)
    inj = np.sort(g.choice(S, size=int(round(frac_injected * S)), replace=False))
    lo, hi = np.log(1e-10), np.log(1e-4)
    lt = np.float32(log_tau)
    for s in inj:
        n_iso = int(g.integers(0, 12))
        pos = g.integers(0, T, size=n_iso)
        lp[s, pos] = g.uniform(lo, hi, size=n_iso).astype(np.float32)
        for _ in range(int(g.integers(0, 3))):
            L = int(g.integers(1, max_run + 1))
            p0 = int(g.integers(0, T))
            p1 = min(T, p0 + L)
            lp[s, p0:p1] = g.uniform(lo, hi, size=p1 - p0).astype(np.float32)
        edge = g.integers(0, T, size=3)
        lp[s, edge[0]] = lt
        lp[s, edge[1]] = np.nextafter(lt, np.float32(0))
        lp[s, edge[2]] = np.nextafter(lt, np.float32(-np.inf))
    lengths = np.full(S, T, np.int32)
    lengths[::8] = g.integers(T // 4, T + 1, size=lengths[::8].shape[0]).astype(np.int32)
    rewards = (g.random(S) < 0.5).astype(np.float32)
    return lp, lengths, rewards, inj


def filter_cases_8x64(log_tau: float):
    """Hand-built 8x64 log-prob batch for the dual-gate filter (threshold count 9, run 5).

    Row 0 clean; row 1 one isolated tail token; row 2 eight isolated (kept); row 3 nine
    isolated (dropped by the count gate); row 4 a run of 4 (kept); row 5 a run of 5
    (dropped by the run gate); row 6 a run of 5 ending at the last token; row 7 values
    exactly at the threshold, one ulp above and below, and a NaN.
    """
    lt = np.float32(log_tau)
    lp = np.full((8, 64), np.float32(-0.05), np.float32)
    tail = np.float32(-15.0)
    lp[1, 20] = tail
    lp[2, 3:64:8] = tail                      # 8 isolated
    lp[3, 1:64:7][:9] = tail                  # 9 isolated
    lp[4, 10:14] = tail                       # run 4
    lp[5, 30:35] = tail                       # run 5
    lp[6, 59:64] = tail                       # run 5 at the end
    lp[7, 5] = lt                             # exactly tau: tail (<=)
    lp[7, 9] = np.nextafter(lt, np.float32(0))          # just above: not tail
    lp[7, 13] = np.nextafter(lt, np.float32(-np.inf))   # just below: tail
    lp[7, 17] = np.float32(np.nan)                       # NaN: tail
    return lp
