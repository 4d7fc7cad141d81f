"""mimo_attn_decode_noalloc: decode for callers that cannot allocate.

Some callers cannot call cudaMalloc -- they run inside a process whose device
memory belongs to another allocator (a serving runtime or a framework memory
pool), or in latency-critical loops that cannot take the synchronisation an
allocation may cause.  The no-alloc entry point keeps the split-KV partials in
a fixed-size array compiled into the library instead of a caller workspace.
These tests call it through the C ABI and compare it with mimo_attn_decode,
which uses a caller-provided workspace, on two calls in a row (the shared
array keeps the previous call's contents, which must not leak into the next).

This file is named to be collected last.
"""

import ctypes

import pytest
import torch

import workloads as W
from tests import parity_util as P

import global_attention_swa_b200 as mimo

SCRATCH_BYTES = 16 << 20


def _call(dims, q, k, v, sl, B, C, window, sinks, out, lse):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return mimo.lib.mimo_attn_decode_noalloc(ctypes.byref(dims), p(q), p(k), p(v), p(sl), B, C,
                                             window, p(sinks), p(out), p(lse), stream)


def test_oversize_is_rejected_before_device_work():
    """Sizes whose split-KV scratch exceeds the built-in 16 MiB are refused."""
    dims = mimo.make_dims(64, 4)
    need = mimo.mimo_attn_decode_workspace_size(64, 4, 64, 262144, 0)
    assert need > SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)
    st = mimo.lib.mimo_attn_decode_noalloc(ctypes.byref(dims), fake, fake, fake, fake, 64, 262144,
                                           0, None, fake, None, None)
    assert st == mimo.MIMO_ERR_WORKSPACE
    assert "scratch" in mimo.lib.mimo_attn_last_error().decode()


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_on_consecutive_calls():
    """Calls in a row through the shared array: first a plan with many splits
    (it fills much of the array), then smaller plans, a ring cache (no scratch at
    all) and a windowed linear cache.  Both entry points run the same kernels
    on the same split plan, so each result must equal mimo_attn_decode's bit for
    bit; a partial left over from an earlier call would break that."""
    import oracle

    cases = [  # seed, lengths, capacity, window, out dtype
        (31, [60000, 33000], 65536, 0, torch.bfloat16),
        (32, [2048, 1, 700, 1500], 2048, 0, torch.float32),
        (33, [300, 129, 5], 129, 129, torch.float32),
        (34, [900, 1300, 129, 5], 8192, 129, torch.bfloat16),
    ]
    needs = [mimo.mimo_attn_decode_workspace_size(64, 4, len(L), C, w) for _, L, C, w, _ in cases]
    assert needs[0] > needs[1] > 0 and needs[2] == 0 and needs[0] <= SCRATCH_BYTES
    for (seed, lengths, C, window, odt), need in zip(cases, needs):
        x = W.decode_inputs(lengths, C, window, seed=seed, device="cuda")
        ref_out, ref_lse = mimo.mimo_attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, window,
                                                 x.sinks, out_dtype=odt)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        dims = mimo.make_dims(64, 4, out_dtype=odt)
        st = _call(dims, x.q, x.k_cache, x.v_cache, x.seqlens, len(lengths), C, window, x.sinks,
                   out, lse)
        assert st == mimo.MIMO_OK, mimo.lib.mimo_attn_last_error().decode()
        mimo.mimo_attn_device_status()
        assert torch.equal(out, ref_out), f"seed {seed}: out differs from the workspace decode"
        assert torch.equal(lse, ref_lse), f"seed {seed}: lse differs from the workspace decode"
        if seed == 32:  # and against the oracle (fp32 output, several splits)
            ro, rl = oracle.decode(x.q.cpu(), x.k_cache.cpu(), x.v_cache.cpu(), x.seqlens.cpu(),
                                   window, x.sinks.cpu())
            P.check(out, ro, lse, rl, what="noalloc vs oracle")
