"""CPU oracle for the SpliceGEMM hot path — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct numpy restatement of what FourSight (arXiv
2611.04887, "FourSight: Stable FP4 RL Post-Training via Sequence Filtering and
Sparse Channel Compensation") computes on its data-parallel hot path:

* ``nvfp4``   — E2M1 / UE4M3 codecs, the masked 16-element block quantiser,
                encode gains, packing and the MMA-ready scale-factor layout
                (§2.1 "Quantized RL Post-training"; §9.3.1 Eq. 9).
* ``splice``  — weight pre-split, activation mask/quantise/extract and the
                SpliceGEMM output (§4.2 Eq. 5, §5.1 "Data preparation").
* ``stats``   — running channel moments and top-s reselection
                (§5.2 "System Implementation"; §9.3 Prop. 2, Cor. 1).
* ``seqfilter`` — dual-gate TIM-aware sequence filter and advantage masking
                (§4.1 Eq. 3-4; §2.1 GRPO advantage).
* ``bounds``  — the error-bound constants of §9.3 (Lemma 2, Lemma 3, Thm. 1).
* ``train``   — the training side: STE backward in BF16, the Eq. 4 GRPO objective
                with filtered advantages and its gradient, the K3 TIM metric
                (§5.2, §4.1 Eq. 4, §6.1).
``splice`` also holds the compacted-K variant (``COMPACT``): protected columns
removed from the NVFP4 operand, blocks re-formed over the rest.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA library and never
imports it.  Every function is pinned by ``-m "not gpu"`` tests to facts the
paper fixes (value sets, worked examples, closed forms, bounds, brute force);
the one reading that no page fact can pin is marked "parity unpinned" where it
lives: the absolute accumulation error of the tensor cores (covered only by the
stated tolerance).  The MoE routing synthesis is an input drawn by ``synth``,
not a result, and is pinned there to the law of its reading.
"""
from . import nvfp4, splice, stats, seqfilter, bounds, train  # noqa: F401
