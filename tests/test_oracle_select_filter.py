"""Pins for the oracle's channel statistics, top-s selection and the dual-gate filter.

FourSight §5.2 (running moments, reselection), §9.3 Prop. 2 and Cor. 1 (second moment vs
variance), Fig. 13 (variance selection beats random selection), §4.1 Eq. 3-4 and §2.1 (filter,
GRPO advantage), §6.1 (tau, K1, K2 defaults).
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import nvfp4, seqfilter, splice, stats


# ----------------------------------------------------------------------------- statistics
def test_integer_moments_equal_exact_big_int_sums():
    x, _ = synth.outlier_activations(21, 37, 48, as_bf16=False)
    st = stats.accumulate(stats.new_state(48), x, row_stride=3)
    rows = x[::3]
    for j in range(48):
        s1 = sum(round(Fraction(float(v)) * 65536) for v in rows[:, j])      # Python round: ties to even
        s2 = sum(round(Fraction(float(v)) ** 2 * 16384) for v in rows[:, j])
        assert st["s1"][j] == s1 and st["s2"][j] == s2
    assert st["n"] == rows.shape[0]
    assert np.array_equal(st["amax"], np.abs(rows).max(axis=0))
    assert st["flags"] == 0


def test_moments_are_order_independent_and_split_invariant():
    x, _ = synth.outlier_activations(22, 64, 32, as_bf16=False)
    a = stats.accumulate(stats.new_state(32), x)
    b = stats.accumulate(stats.new_state(32), x[np.random.default_rng(0).permutation(64)])
    c = stats.accumulate(stats.accumulate(stats.new_state(32), x[:20]), x[20:])
    for other in (b, c):
        assert np.array_equal(a["s1"], other["s1"]) and np.array_equal(a["s2"], other["s2"])
        assert a["n"] == other["n"] and np.array_equal(a["amax"], other["amax"])


def test_variance_key_matches_population_variance():
    x, _ = synth.outlier_activations(23, 512, 64, as_bf16=False)
    st = stats.accumulate(stats.new_state(64), x)
    v = np.var(x.astype(np.float64), axis=0)
    assert np.allclose(stats.keys(st), v, rtol=1e-6, atol=2.0 ** -13)
    assert np.allclose(stats.keys(st, second_moment=True), (x.astype(np.float64) ** 2).mean(0), rtol=1e-6, atol=2.0 ** -13)


def test_range_flag():
    x = np.zeros((2, 16), np.float32); x[1, 3] = 70000.0; x[0, 3] = 2.0
    st = stats.accumulate(stats.new_state(16), x)
    assert st["flags"] == 1 and st["s1"][3] == 2 * 65536 and st["amax"][3] == 2.0
    x[1, 3] = np.inf
    assert stats.accumulate(stats.new_state(16), x)["flags"] == 1
    x[1, 3] = 32767.0
    assert stats.accumulate(stats.new_state(16), x)["flags"] == 0
    x[1, 3] = 32768.0
    assert stats.accumulate(stats.new_state(16), x)["flags"] == 1


def test_topk_order_and_ties():
    st = stats.new_state(8)
    st["n"] = 1
    st["s2"] = np.array([5, 9, 9, 1, 9, 0, 7, 9], np.int64) * 16384
    P = stats.select_topk(st, 3, second_moment=True)
    assert P.tolist() == [1, 2, 4]               # ties broken by the lower index
    assert stats.select_topk(st, 0).tolist() == []
    assert stats.select_topk(st, 8).tolist() == list(range(8))
    m = stats.protect_mask([0, 31, 32, 40], 64)
    assert m.tolist() == [0x80000001, 0x101]


def test_prop2_brute_force_over_all_subsets():
    """Top-s second moments minimise sum_{j not in S} m_j over every subset (Prop. 2)."""
    rs = np.random.default_rng(24)
    for trial in range(20):
        K = int(rs.integers(4, 13))
        p = int(rs.integers(1, 4))
        x = (rs.standard_normal((16, K)) * rs.uniform(0.1, 5, K)).astype(np.float32)
        st = stats.accumulate(stats.new_state(K), x)
        m = stats.keys(st, second_moment=True)
        best = min(itertools.combinations(range(K), p), key=lambda S: (sum(m[j] for j in range(K) if j not in S), S))
        assert stats.select_topk(st, p, second_moment=True).tolist() == list(best)


def test_cor1_zero_mean_variance_equals_second_moment_ranking():
    x, _ = synth.outlier_activations(25, 100, 128, as_bf16=False)
    x = np.concatenate([x, -x])                    # exactly zero mean per channel
    st = stats.accumulate(stats.new_state(128), x)
    assert np.all(st["s1"] == 0)
    assert stats.select_topk(st, 16).tolist() == stats.select_topk(st, 16, second_moment=True).tolist()


def test_variance_selection_beats_random_selection():
    """Fig. 13's qualitative claim: top-variance protection beats 30 random protected sets."""
    for seed in (31, 32, 33):
        x, _ = synth.outlier_activations(seed, 64, 512, as_bf16=True)
        w = synth.gaussian_weights(seed + 50, 64, 512)
        X, W = nvfp4.bf16_value(x), nvfp4.bf16_value(w)
        st = stats.accumulate(stats.new_state(512), X)
        y = X.astype(np.float64) @ W.astype(np.float64).T

        def err(P):
            gA = stats.next_gain(st, P)
            xq = splice.quantize_splice(X, P, gA)
            wq = splice.prepare_weights(W, P, gA)
            return ((splice.splice_gemm(xq, wq, wq["alpha"])[0] - y) ** 2).mean()

        e_var = err(stats.select_topk(st, 64))
        rs = np.random.default_rng(seed)
        e_rand = [err(np.sort(rs.choice(512, 64, replace=False))) for _ in range(30)]
        assert e_var < min(e_rand)


def test_next_gain_excludes_protected_channels():
    x = np.ones((4, 32), np.float32); x[:, 5] = 3000.0
    st = stats.accumulate(stats.new_state(32), x)
    assert stats.next_gain(st, [5]) == nvfp4.gain_pow2(1.0)
    assert stats.next_gain(st, [5], residual=True) == nvfp4.gain_pow2(3000.0)


# ----------------------------------------------------------------------------- filter
def _defaults(golden_dir):
    out = {}
    with open(os.path.join(golden_dir, "filter_defaults.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split()
            out[k] = float(v)
    return out


def test_hand_built_8x64_cases(golden_dir):
    d = _defaults(golden_dir)
    lt = seqfilter.log_tau(d["tau"])
    assert lt == np.float32(math.log(1e-4))
    lp = synth.filter_cases_8x64(lt)
    r = seqfilter.seq_filter(lp, None, lt, K1=9, K2=int(d["K2"]))
    # row: 0 clean, 1 one isolated, 2 eight isolated, 3 nine isolated, 4 run 4, 5 run 5,
    # 6 run 5 at the end, 7 tau itself + one ulp below + NaN are tail, one ulp above is not
    assert r["tail_count"].tolist() == [0, 1, 8, 9, 4, 5, 5, 3]
    assert r["max_run"].tolist() == [0, 1, 1, 1, 4, 5, 5, 1]
    assert r["keep"].tolist() == [1, 1, 1, 0, 1, 0, 0, 1]


def _plain_loop(bits, K1, K2):
    count = run = best = 0
    for b in bits:
        count += b
        run = run + 1 if b else 0
        best = max(best, run)
    return count, best, int(count < K1 and best < K2)


def test_filter_brute_force_all_patterns():
    lt = np.float32(-9.0)
    for L in range(1, 15):
        pats = np.array(list(itertools.product([0, 1], repeat=L)), dtype=bool)
        lp = np.where(pats, np.float32(-20), np.float32(-1)).astype(np.float32)
        r = seqfilter.seq_filter(lp, None, lt, K1=4, K2=3)
        for i, row in enumerate(pats):
            c, b, k = _plain_loop(list(row), 4, 3)
            assert (r["tail_count"][i], r["max_run"][i], r["keep"][i]) == (c, b, k)


def test_lengths_truncate_and_runs_do_not_cross_sequences():
    lp = np.full((2, 10), np.float32(-1))
    lp[0, 7:] = -20
    lp[1, :3] = -20
    r = seqfilter.seq_filter(lp, np.array([8, 10]), np.float32(-9), K1=100, K2=3)
    assert r["tail_count"].tolist() == [1, 3] and r["max_run"].tolist() == [1, 3]
    assert r["keep"].tolist() == [1, 0]


def test_group_advantage_and_original_denominator():
    rewards = np.array([1, 0, 1, 0, 1, 1, 1, 1], np.float32)
    A = seqfilter.group_advantages(rewards, 4)
    assert A.tolist() == [1, -1, 1, -1, 0, 0, 0, 0]            # sigma = 0 -> 0
    lp = np.full((8, 16), np.float32(-1)); lp[1, 2:9] = -20     # sequence 1 dropped by the run gate
    r = seqfilter.seq_filter(lp, None, np.float32(-9), K1=50, K2=5, G=4, rewards=rewards)
    assert r["keep"].tolist() == [1, 0, 1, 1, 1, 1, 1, 1]
    assert r["adv"].tolist() == [1, 0, 1, -1, 0, 0, 0, 0]
    # the GRPO loss weight stays 1/G: the surviving advantages are not rescaled by G / sum(keep)
    assert r["adv"][:4].sum() / 4 == (A[:4] * r["keep"][:4]).sum() / 4
    given = np.arange(8, dtype=np.float32)
    r2 = seqfilter.seq_filter(lp, None, np.float32(-9), K1=50, K2=5, adv=given)
    assert r2["adv"].tolist() == [0, 0, 2, 3, 4, 5, 6, 7]


def test_gates_at_the_rollout_defaults():
    """§4.1: G1 drops a trajectory with AT LEAST K1 tail tokens, G2 one with AT LEAST K2
    consecutive ones (Eq. 3 keeps count < K1 and run < K2).  At the rollout defaults (K1 = 41 for a
    4096-token response limit, K2 = 5) a sequence with 40 isolated tail tokens and runs of 4 is kept;
    one more isolated tail token, or one run of 5, drops it."""
    lt = np.float32(-9.0)
    T = 4096

    def seq(isolated, run):
        lp = np.full(T, np.float32(-0.5))
        lp[np.arange(isolated) * 50] = -20                 # isolated tails, 49 normal tokens apart
        if run:
            lp[3000:3000 + run] = -20
        return lp

    batch = np.stack([seq(40, 0), seq(41, 0), seq(36, 4), seq(36, 5), seq(0, 4), seq(0, 5)])
    r = seqfilter.seq_filter(batch, None, lt, K1=41, K2=5)
    assert r["tail_count"].tolist() == [40, 41, 40, 41, 4, 5]
    assert r["max_run"].tolist() == [1, 1, 4, 5, 4, 5]
    assert r["keep"].tolist() == [1, 0, 1, 0, 1, 0]
