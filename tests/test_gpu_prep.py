"""GPU parity of the preparation kernels against the oracle (bit-exact).

fs_channel_stats / fs_select_topk (FourSight §5.2), fs_quantize_splice / fs_prepare_weights
(§5.1 "Data preparation", Eq. 9), fs_seq_filter (§4.1 Eq. 3-4).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import nvfp4, seqfilter, splice, stats
from tests._util import bf16_tensor, check_packed, f32_tensor, mask_tensor

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _x(seed, M, K, dtype, frac=0.01, scale=30.0):
    x, ch = synth.outlier_activations(seed, M, K, frac=frac, scale=scale, as_bf16=(dtype == "bf16"))
    X = splice.as_f32(x, dtype == "bf16")
    T = bf16_tensor(x) if dtype == "bf16" else f32_tensor(x)
    return X, T


def _state_np(st: "F.StatsState", i=0):
    return {"n": int(st.n[i].item()), "s1": st.s1[i].cpu().numpy(), "s2": st.s2[i].cpu().numpy(),
            "amax": st.amax[i].cpu().numpy().view(np.float32), "flags": int(st.flags[i].item())}


# ----------------------------------------------------------------------------- statistics
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,stride", [(1, 64, 1), (333, 512, 1), (1000, 4096, 3), (4096, 12288, 1)])
def test_channel_stats_bit_exact(dtype, M, K, stride):
    X, T = _x(1 + M, M, K, dtype)
    st = F.StatsState(1, K)
    F.fs_channel_stats(T, st, row_stride=stride)
    F.fs_channel_stats(T[: M // 2 + 1], st, row_stride=stride)       # a second call accumulates
    ref = stats.accumulate(stats.accumulate(stats.new_state(K), X, stride), X[: M // 2 + 1], stride)
    got = _state_np(st)
    assert got["n"] == ref["n"] and got["flags"] == ref["flags"] == 0
    assert np.array_equal(got["s1"], ref["s1"]) and np.array_equal(got["s2"], ref["s2"])
    assert np.array_equal(got["amax"], ref["amax"])


def test_channel_stats_range_flag():
    x = np.zeros((4, 64), np.float32); x[2, 7] = 40000.0; x[1, 9] = np.nan; x[0, 7] = 3.0; x[3, 11] = 32767.0
    st = F.StatsState(1, 64)
    F.fs_channel_stats(f32_tensor(x), st)
    ref = stats.accumulate(stats.new_state(64), x)
    got = _state_np(st)
    assert got["flags"] == 1 == ref["flags"]
    assert np.array_equal(got["s1"], ref["s1"]) and np.array_equal(got["amax"], ref["amax"])
    with pytest.raises(F.FoursightError):
        F.fs_stats_check(st)


# ----------------------------------------------------------------------------- selection
@pytest.mark.parametrize("K,p,opts", [(512, 64, 0), (4096, 64, 0), (12288, 256, 0), (4096, 64, 2), (4096, 64, 1),
                                      (4096, 64, 4), (64, 64, 0), (512, 0, 0), (100 * 16, 3, 0)])
def test_select_topk_bit_exact(K, p, opts):
    nprob = 3
    st = F.StatsState(nprob, K)
    refs = []
    for i in range(nprob):
        X, T = _x(100 + i, 257, K, "bf16")
        F.fs_channel_stats(T, st, group=i)
        refs.append(stats.accumulate(stats.new_state(K), X))
    P, mask, gA = F.fs_select_topk(st, p, opts=opts, reset=True)
    for i in range(nprob):
        Pr = stats.select_topk(refs[i], p, second_moment=bool(opts & 2))
        assert np.array_equal(P[i].cpu().numpy(), Pr)
        assert np.array_equal(mask[i].cpu().numpy().view(np.uint32), stats.protect_mask(Pr, K))
        g = stats.next_gain(refs[i], Pr, residual=bool(opts & 1), exact=bool(opts & 4))
        assert gA[i].item() == float(g)
    assert int(st.n.abs().sum()) == 0 and int(st.s2.abs().sum()) == 0 and int(st.amax.abs().sum()) == 0


def test_select_topk_ties_and_empty_state():
    K = 256
    st = F.StatsState(1, K)
    x = np.zeros((2, K), np.float32)
    x[0, [5, 9, 100, 200]] = 2.0; x[1, [5, 9, 100, 200]] = -2.0        # four equal variances
    x[:, 50] = 1.0                                                       # zero variance, non-zero mean
    F.fs_channel_stats(f32_tensor(x), st)
    P, _, _ = F.fs_select_topk(st, 3)
    ref = stats.select_topk(stats.accumulate(stats.new_state(K), x), 3)
    assert P[0].cpu().tolist() == ref.tolist() == [5, 9, 100]
    st2 = F.StatsState(1, K)                                             # n == 0: all keys 0 -> lowest indices
    P2, _, g2 = F.fs_select_topk(st2, 4)
    assert P2[0].cpu().tolist() == [0, 1, 2, 3] and g2.item() == 1.0


@pytest.mark.parametrize("K,p", [(16384, 256), (16384, 1), (8256, 64), (1000, 17), (96, 96), (96, 5)])
def test_select_topk_ranges_of_the_cluster(K, p):
    """The selection splits K over the CTAs of a cluster (512 channels per CTA per round, up to 4
    rounds): K = 16384 fills every round, 8256 leaves the last CTAs partly or wholly empty, 1000
    ends inside a mask word, 96 sits inside the first CTA."""
    nprob = 2
    st = F.StatsState(nprob, K)
    refs = []
    for i in range(nprob):
        X, T = _x(300 + i + K, 129, K, "bf16")
        F.fs_channel_stats(T, st, group=i)
        refs.append(stats.accumulate(stats.new_state(K), X))
    P, mask, gA = F.fs_select_topk(st, p, reset=True)
    for i in range(nprob):
        Pr = stats.select_topk(refs[i], p)
        assert np.array_equal(P[i].cpu().numpy(), Pr)
        assert np.array_equal(mask[i].cpu().numpy().view(np.uint32), stats.protect_mask(Pr, K))
        assert gA[i].item() == float(stats.next_gain(refs[i], Pr))
    assert int(st.n.abs().sum()) == 0 and int(st.s1.abs().sum()) == 0 and int(st.flags.abs().sum()) == 0


@pytest.mark.parametrize("p", [2, 5, 8])
def test_select_topk_ties_across_ctas(p):
    """Equal variances at channels that fall to different CTAs (K = 8192: 1024 channels per CTA):
    two larger keys come first, then the tied channels in index order until p are taken."""
    K = 8192
    tied = [100, 1500, 3000, 5000, 7000, 8100]
    x = np.zeros((2, K), np.float32)
    x[0, tied] = 2.0; x[1, tied] = -2.0
    x[0, [4000, 6500]] = 3.0; x[1, [4000, 6500]] = -3.0
    x[:, 2000] = 1.5                                                     # zero variance, largest mean
    st = F.StatsState(1, K)
    F.fs_channel_stats(f32_tensor(x), st)
    P, mask, gA = F.fs_select_topk(st, p)
    ref_state = stats.accumulate(stats.new_state(K), x)
    ref = stats.select_topk(ref_state, p)
    assert P[0].cpu().tolist() == ref.tolist() == sorted([4000, 6500] + tied[:p - 2])
    assert np.array_equal(mask[0].cpu().numpy().view(np.uint32), stats.protect_mask(ref, K))
    assert gA.item() == float(stats.next_gain(ref_state, ref))


# ----------------------------------------------------------------------------- quantisation
def _prep_inputs(seed, M, K, p, dtype):
    X, T = _x(seed, M, K, dtype)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    return X, T, P, st


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,p", [(1, 64, 0), (8, 512, 64), (130, 512, 5), (300, 4096, 64), (16, 12288, 256),
                                   (257, 2048, 64), (4, 4096, 0)])
@pytest.mark.parametrize("residual", [False, True])
def test_quantize_splice_bit_exact(dtype, M, K, p, residual):
    X, T, P, st = _prep_inputs(7 + M + K, M, K, p, dtype)
    gA = stats.next_gain(st, P, residual=residual)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], dtype=torch.float32, device="cuda")
    opts = F.FS_RESIDUAL if residual else 0
    for _ in range(2):                                                   # repeatable
        out = F.fs_quantize_splice(T, mask, p, g, opts=opts)
        torch.cuda.synchronize()
        ref = splice.quantize_splice(X, P, gA, splice.RESIDUAL if residual else splice.SPLIT)
        check_packed(out, ref, M, K, p)


@pytest.mark.parametrize("M,K,p,stride,residual", [(1, 64, 0, 1, False), (8, 512, 64, 1, False), (130, 576, 5, 1, True),
                                                   (300, 4096, 64, 3, False), (16, 12288, 256, 1, False),
                                                   (1000, 2048, 64, 2, True), (8192, 4096, 64, 1, False),
                                                   (2049, 12288, 64, 1, False), (257, 4096, 0, 1, False)])
def test_quantize_splice_stats_bit_exact(M, K, p, stride, residual):
    """The fused pass (NEXT-1): moments of the raw rows into a state that already holds a previous
    batch, and the packed operand under the current protected set, both bit-exact against the
    oracle's statistics and activation preparation; a second call is repeatable."""
    X, T, P, st = _prep_inputs(17 + M + K, M, K, p, "bf16")
    Xprev, Tprev = _x(5 + K, 33, K, "bf16")
    gA = stats.next_gain(st, P, residual=residual)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], dtype=torch.float32, device="cuda")
    opts = F.FS_RESIDUAL if residual else 0
    ref = splice.quantize_splice(X, P, gA, splice.RESIDUAL if residual else splice.SPLIT)
    for rep in range(2):
        state = F.StatsState(1, K)
        F.fs_channel_stats(Tprev, state)                                  # earlier batch of the window
        out = F.fs_quantize_splice_stats(T, mask, p, g, state, row_stride=stride, opts=opts)
        torch.cuda.synchronize()
        check_packed(out, ref, M, K, p)
        want = stats.accumulate(stats.accumulate(stats.new_state(K), Xprev), X, stride)
        got = _state_np(state)
        assert got["n"] == want["n"] and got["flags"] == want["flags"] == 0, rep
        assert np.array_equal(got["s1"], want["s1"]) and np.array_equal(got["s2"], want["s2"]), rep
        assert np.array_equal(got["amax"], want["amax"]), rep


def test_quantize_splice_stats_range_flag_and_outliers():
    """Elements at and past the statistics range (|x| >= 2^15) raise the flag and add nothing to the
    moments, values just below it are counted; the quantised operand is unaffected by the flag."""
    K, M = 512, 64
    X, T, P, st = _prep_inputs(3, M, K, 16, "bf16")
    x = nvfp4.bf16_bits(X)
    x[5, 7] = 0x4700                                                     # 2^15: out of range
    x[9, 100] = 0xC700                                                   # -2^15
    x[10, 101] = 0x46FF                                                  # just below 2^15: counted
    X = nvfp4.bf16_value(x)
    gA = stats.next_gain(stats.accumulate(stats.new_state(K), X), P)
    state = F.StatsState(1, K)
    out = F.fs_quantize_splice_stats(bf16_tensor(x), mask_tensor(stats.protect_mask(P, K)), 16,
                                     torch.tensor([float(gA)], device="cuda"), state)
    want = stats.accumulate(stats.new_state(K), X)
    got = _state_np(state)
    assert got["flags"] == want["flags"] == 1
    assert np.array_equal(got["s1"], want["s1"]) and np.array_equal(got["s2"], want["s2"])
    assert np.array_equal(got["amax"], want["amax"])
    check_packed(out, splice.quantize_splice(X, P, gA), M, K, 16)


def test_quantize_every_scale_code_and_rounding_boundary():
    """Blocks built so that every normal UE4M3 scale is hit and elements sit on E2M1 midpoints +-1 ulp."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 6.5, 0.1, 0.0], np.float32)
    probes = [mids]
    up, down = mids.copy(), mids.copy()
    for _ in range(4):                                  # +-1..4 ulps around every midpoint
        up, down = np.nextafter(up, np.float32(np.inf)), np.nextafter(down, np.float32(0))
        probes += [up, down]
    probes = np.concatenate(probes)
    probes = np.concatenate([probes, -probes, np.float32([-0.0])])
    rows = []
    for code in range(1, 126):
        s = np.float32(nvfp4.ue4m3_decode(code))
        vals = (probes * s).astype(np.float32)
        for c0 in range(0, len(vals), 15):
            blk = np.zeros(16, np.float32)
            blk[0] = np.float32(6.0) * s
            chunk = vals[c0:c0 + 15]
            blk[1:1 + len(chunk)] = chunk
            rows.append(blk)
    X = np.stack(rows).reshape(-1, 64) if len(rows) % 4 == 0 else np.concatenate([np.stack(rows), np.zeros((4 - len(rows) % 4, 16), np.float32)]).reshape(-1, 64)
    g = np.float32(1.0)
    out = F.fs_quantize_splice(f32_tensor(X), None, 0, torch.tensor([1.0], device="cuda"))
    ref = splice.quantize_splice(X, [], g)
    check_packed(out, ref, X.shape[0], 64, 0)


def test_quantize_exact_gain_and_zero_and_subnormal_scales():
    rs = np.random.default_rng(5)
    X = (rs.standard_normal((64, 256)) * np.float32(1e-3)).astype(np.float32)
    X[3, :16] = 0.0; X[4, :16] = -0.0; X[5, 16:32] = 1e-30; X[6, 32:48] = -1e-30
    X[7, 48:64] = 300.0                                              # saturating block scale
    for gain in (float(nvfp4.gain_exact(np.abs(X).max())), 1.0, 2.0 ** 20):
        out = F.fs_quantize_splice(f32_tensor(X), None, 0, torch.tensor([gain], device="cuda"))
        ref = splice.quantize_splice(X, [], np.float32(gain))
        check_packed(out, ref, 64, 256, 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N,K,p,opts", [(256, 512, 64, 0), (1024, 4096, 64, 0), (200, 2048, 64, 1), (384, 4096, 0, 0),
                                        (128, 12288, 256, 0), (256, 512, 64, 4)])
def test_prepare_weights_bit_exact(dtype, N, K, p, opts):
    X, _, P, st = _prep_inputs(3, 64, K, p, "bf16")
    w = synth.gaussian_weights(9 + N, N, K, as_bf16=(dtype == "bf16"))
    W = splice.as_f32(w, dtype == "bf16")
    Wt = bf16_tensor(w) if dtype == "bf16" else f32_tensor(w)
    residual, exact = bool(opts & 1), bool(opts & 4)
    gA = stats.next_gain(st, P, residual=residual, exact=exact)
    out, gW, alpha = F.fs_prepare_weights(Wt, mask_tensor(stats.protect_mask(P, K)), p,
                                          torch.tensor([float(gA)], device="cuda"), opts=opts)
    ref = splice.prepare_weights(W, P, gA, splice.RESIDUAL if residual else splice.SPLIT, exact_gain=exact)
    assert gW.item() == float(ref["gW"]) and alpha.item() == float(ref["alpha"])
    check_packed(out, ref, N, K, p)


def test_exact_gain_saturates_for_subnormal_weights():
    """FS_GAIN_EXACT on weights whose largest magnitude is subnormal: fl32(2688/amax) overflows and
    the gain saturates to the largest finite float32; codes, scales and side columns stay bit-exact."""
    N, K, p = 256, 512, 16
    _, _, P, st = _prep_inputs(5, 64, K, p, "bf16")
    w = (synth.gaussian_weights(13, N, K, as_bf16=False) * np.float32(2.0 ** -130)).astype(np.float32)
    assert 0 < np.abs(w).max() < np.finfo(np.float32).tiny
    gA = np.float32(2.0 ** -100)
    out, gW, alpha = F.fs_prepare_weights(f32_tensor(w), mask_tensor(stats.protect_mask(P, K)), p,
                                          torch.tensor([float(gA)], device="cuda"), opts=F.FS_GAIN_EXACT)
    ref = splice.prepare_weights(w, P, gA, exact_gain=True)
    assert float(ref["gW"]) == float(np.finfo(np.float32).max)
    assert gW.item() == float(ref["gW"]) and alpha.item() == float(ref["alpha"])
    check_packed(out, ref, N, K, p)


@pytest.mark.parametrize("opts", [0, 1])
def test_prepare_weights_gain_sees_every_element(opts):
    """One planted large weight decides the gain, wherever it sits: first and last element, the
    ragged last 64 columns (K = 576 is not a multiple of 256), a middle row; a larger one in a
    protected column is ignored by the split form and counted by the residual form."""
    N, K, p = 300, 576, 16
    _, _, P, st = _prep_inputs(5, 64, K, p, "bf16")
    gA = stats.next_gain(st, P, residual=bool(opts & 1))
    mask = mask_tensor(stats.protect_mask(P, K))
    unprot = [c for c in range(K) if c not in set(int(v) for v in P)]
    spots = [(0, unprot[0], 0x40A0), (N - 1, unprot[-1], 0xC0F0), (N // 2, unprot[len(unprot) // 2], 0x4110),
             (N - 1, unprot[200], 0x40E0)]
    for r, c, bits in spots:
        w = synth.gaussian_weights(11, N, K, as_bf16=True).copy()
        w[r, c] = bits
        w[N // 3, int(P[0])] = 0x42C8                      # 100.0 in a protected column
        ref = splice.prepare_weights(splice.as_f32(w, True), P, gA, splice.RESIDUAL if opts & 1 else splice.SPLIT)
        _, gW, alpha = F.fs_prepare_weights(bf16_tensor(w), mask, p, torch.tensor([float(gA)], device="cuda"), opts=opts)
        assert gW.item() == float(ref["gW"]) and alpha.item() == float(ref["alpha"]), (r, c)


# ----------------------------------------------------------------------------- filter
def test_seq_filter_hand_built_cases():
    lt = seqfilter.log_tau(1e-4)
    lp = synth.filter_cases_8x64(lt)
    keep, cnt, run, _ = F.fs_seq_filter(f32_tensor(lp), float(lt), 9, 5)
    ref = seqfilter.seq_filter(lp, None, lt, 9, 5)
    assert keep.cpu().tolist() == ref["keep"].tolist() == [1, 1, 1, 0, 1, 0, 0, 1]
    assert cnt.cpu().tolist() == ref["tail_count"].tolist()
    assert run.cpu().tolist() == ref["max_run"].tolist()


@pytest.mark.parametrize("S,T", [(1024, 4096), (64, 1000), (16, 8192), (3, 5)])
def test_seq_filter_rollout_batch(S, T):
    lt = seqfilter.log_tau(1e-4)
    lp, lengths, rewards, _ = synth.rollout_logprobs(11, S=S, T=T, max_run=min(512, T))
    K1 = math.ceil(0.01 * T)
    G = 1 if S % 16 else 16
    lpt, lent, rwt = f32_tensor(lp), torch.from_numpy(lengths).cuda(), f32_tensor(rewards)
    keep, cnt, run, adv = F.fs_seq_filter(lpt, float(lt), K1, 5, lengths=lent, G=G, rewards=rwt)
    ref = seqfilter.seq_filter(lp, lengths, lt, K1, 5, G=G, rewards=rewards)
    assert np.array_equal(keep.cpu().numpy(), ref["keep"])
    assert np.array_equal(cnt.cpu().numpy(), ref["tail_count"])
    assert np.array_equal(run.cpu().numpy(), ref["max_run"])
    assert np.array_equal(adv.cpu().numpy().view(np.uint32), ref["adv"].view(np.uint32))
    # in-place masking of given advantages
    a0 = np.arange(S, dtype=np.float32) - S / 2
    at = f32_tensor(a0)
    F.fs_seq_filter(lpt, float(lt), K1, 5, lengths=lent, adv=at)
    assert np.array_equal(at.cpu().numpy(), np.where(ref["keep"] == 1, a0, np.float32(0)))
