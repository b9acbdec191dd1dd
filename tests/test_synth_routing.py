"""The MoE routing synthesis (``synth.moe_routing_counts``) against the exact law of its reading:
each token draws ``topk`` distinct experts, one after another, each with probability proportional
to its Zipf(s) rank weight among the experts not yet drawn (sampling without replacement,
Plackett-Luce).  Perturbing log-weights with Gumbel noise and keeping the top k draws from exactly
that law, so for small expert counts the per-expert inclusion probabilities are enumerated over
every ordered draw and the generated counts must match them within binomial noise.
"""
import itertools

import numpy as np
import pytest

import synth


def inclusion_probabilities(w, k):
    """P(expert e is among the k drawn), summed over every ordered sequence of k distinct experts."""
    w = np.asarray(w, np.float64)
    total = w.sum()
    p = np.zeros(len(w))
    for seq in itertools.permutations(range(len(w)), k):
        prob, left = 1.0, total
        for e in seq:
            prob *= w[e] / left
            left -= w[e]
        for e in seq:
            p[e] += prob
    return p


@pytest.mark.parametrize("experts,topk,s", [(5, 2, 1.2), (6, 3, 1.2), (8, 2, 2.0), (4, 1, 1.2)])
def test_counts_follow_sampling_without_replacement(experts, topk, s):
    tokens = 200000
    seed = 3
    counts = synth.moe_routing_counts(seed, tokens=tokens, experts=experts, topk=topk, zipf_s=s)
    assert counts.sum() == tokens * topk
    perm = synth.rng(seed).permutation(experts)          # the generator's first draw assigns the ranks
    w = (np.arange(1, experts + 1, dtype=np.float64) ** (-s))[perm]
    p = inclusion_probabilities(w, topk)
    assert abs(p.sum() - topk) < 1e-12                   # k distinct experts per token
    sd = np.sqrt(tokens * p * (1 - p))
    z = (counts - tokens * p) / np.maximum(sd, 1e-9)
    assert np.all(np.abs(z) < 5), z
    # with replacement the law would differ measurably: the generator is not that
    with_repl = topk * w / w.sum()
    if topk > 1:
        assert np.max(np.abs(counts - tokens * with_repl) / np.maximum(sd, 1e-9)) > 5


def test_ranks_are_a_permutation_and_the_popular_expert_is_the_rank_one():
    seed, experts = 0, 64
    counts = synth.moe_routing_counts(seed, experts=experts)
    perm = synth.rng(seed).permutation(experts)
    assert sorted(perm.tolist()) == list(range(experts))
    assert int(np.argmax(counts)) == int(np.argmin(perm))   # rank weight 1 (the largest) sits there
