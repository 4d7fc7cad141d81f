"""Reference oracle for the MiMo-V2-Flash hybrid attention operator.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, float64 CPU
restatement of what the operator computes, written from the MiMo-V2-Flash
model documentation (Transformers model doc, "Key features: hybrid attention"
bullet and the ``MiMoV2FlashConfig`` parameter list).  Only the test suite,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The CUDA library never calls it and
shares no code, constant table or helper with it.

Modules
-------
``attention``  vectorised fp64 prefill and decode (NumPy matmuls per query block).
``brute``      scalar triple loops for tiny shapes, used to pin ``attention``.
``merge``      merging decode results over disjoint parts of a cache (context
               parallelism) with the sink.
``rope``       rotary embedding and the decode-step cache append.
``fp8``        e4m3 decoding from the format's definition and decode over FP8
               KV caches with per-KV-head scales (``attention.decode`` on the
               dequantised caches).
``backward``   gradients of the prefill (q, k, v and the sink logits) from
               explicit probability matrices, pinned to finite differences;
               ``prefill_backward_sampled`` gives them at chosen positions of
               one long sequence.

Every function here is pinned by a ``-m "not gpu"`` test against something
other than itself (brute force, closed forms, a library special case, or the
constants the documentation prints).  One choice is *not* pinned by the
pages: the exact sink formula.  The documentation names a "learnable attention
sink bias" but prints no formula; the reading used here (one logit per query
head added as ``exp(sink)`` to the softmax normaliser, no value vector, not
multiplied by the softmax scale) is a stated reading, so parity of the sink
term is "parity unpinned" with respect to the original model and pinned only
with respect to that reading.
"""

from .attention import (  # noqa: F401
    DEFAULT_SCALE_DQK,
    decode,
    prefill,
    ring_slot_position,
    visible,
)
