"""Checkpoint and resume of the channel statistics (FourSight §5.2: running channel moments kept
across steps in a GPU buffer).  The moments are exact integer sums, so a state saved after some
batches, restored and fed the remaining batches equals the state of one pass; the binding's
``StatsState.state_dict`` / ``load_state_dict`` move the five caller-owned buffers as they are.

On the CPU: the oracle's state through a byte round trip in the library's buffer layout, and the
binding's checkpoint round trip and refusals.  (On the GPU, a second ``fs_channel_stats`` call on
the same state is the resumed pass; its bit-exact test covers the kernel side.)
"""
import io

import numpy as np
import pytest
import torch

import nvfp4_w4a4_gemm_fs_b200 as F
from oracle import stats as ostats


def to_buffers(st):
    """The oracle's state in the library's layout: n, s1, s2 int64; amax as float32 bits; flags."""
    return {"n": np.array([st["n"]], np.int64), "s1": st["s1"].copy(), "s2": st["s2"].copy(),
            "amax": st["amax"].view(np.int32).copy(), "flags": np.array([st["flags"]], np.int32)}


def from_buffers(b):
    return {"n": int(b["n"][0]), "s1": b["s1"].copy(), "s2": b["s2"].copy(),
            "amax": b["amax"].view(np.float32).copy(), "flags": int(b["flags"][0])}


@pytest.mark.parametrize("stride", [1, 4])
def test_a_saved_and_restored_state_resumes_bit_exactly(stride):
    rng = np.random.default_rng(stride)
    K = 512
    X = (rng.standard_normal((1024, K)) * np.where(rng.random(K) < 0.02, 40.0, 1.0)).astype(np.float32)
    batches = [X[:256], X[256:640], X[640:]]                         # cut at multiples of the stride
    whole = ostats.accumulate(ostats.new_state(K), X, stride)
    st = ostats.new_state(K)
    for b in batches:
        st = ostats.accumulate(st, b, stride)
        buf = io.BytesIO()
        np.savez(buf, **to_buffers(st))                             # checkpoint ...
        buf.seek(0)
        st = from_buffers(dict(np.load(buf)))                       # ... and resume
    for k in ("s1", "s2"):
        assert np.array_equal(st[k], whole[k])
    assert st["n"] == whole["n"] and st["flags"] == whole["flags"]
    assert np.array_equal(st["amax"].view(np.int32), whole["amax"].view(np.int32))
    for second in (False, True):
        assert np.array_equal(ostats.select_topk(st, 64, second), ostats.select_topk(whole, 64, second))


def test_subsampling_restarts_at_each_call():
    """With a stride, a batch cut off the stride's grid takes other rows than one pass would:
    each call takes its own rows 0, stride, ... (the reading of §5.2's uniform subsampling)."""
    rng = np.random.default_rng(9)
    X = rng.standard_normal((30, 64)).astype(np.float32)
    whole = ostats.accumulate(ostats.new_state(64), X, 4)
    cut = ostats.accumulate(ostats.accumulate(ostats.new_state(64), X[:10], 4), X[10:], 4)
    assert whole["n"] == 8 and cut["n"] == 3 + 5
    assert not np.array_equal(whole["s1"], cut["s1"])


def test_binding_checkpoint_round_trip_and_refusals():
    st = F.StatsState(2, 256, device="cpu")
    g = torch.Generator().manual_seed(1)
    st.n.copy_(torch.tensor([7, 9]))
    st.s1.copy_(torch.randint(-2**40, 2**40, (2, 256), generator=g))
    st.s2.copy_(torch.randint(0, 2**50, (2, 256), generator=g))
    st.amax.copy_(torch.randint(0, 0x47000000, (2, 256), generator=g, dtype=torch.int32))
    st.flags.copy_(torch.tensor([0, 1], dtype=torch.int32))
    ck = st.state_dict()
    st.s1.zero_()                                                   # the checkpoint is a copy
    fresh = F.StatsState(2, 256, device="cpu")
    fresh.load_state_dict(ck)
    for name in ("n", "s2", "amax", "flags"):
        assert torch.equal(getattr(fresh, name), getattr(st, name))
    assert torch.equal(fresh.s1, ck["s1"]) and not torch.equal(fresh.s1, st.s1)
    with pytest.raises(F.ArgumentError):
        F.StatsState(2, 512, device="cpu").load_state_dict(ck)      # another K
    with pytest.raises(F.ArgumentError):
        F.StatsState(1, 256, device="cpu").load_state_dict(ck)      # another group count
    bad = dict(ck, amax=ck["amax"].to(torch.int64))
    with pytest.raises(F.ArgumentError):
        fresh.load_state_dict(bad)                                  # another dtype
