"""Device-side failure reporting, tested without a failing GPU.

Nothing here faults or waits without a bound.  One real time-out runs: the
library's self-test kernel waits about a second on a barrier that nothing
arrives at, as a bounded wait would in a stuck pipeline, and records
MIMO_ERR_TIMEOUT.  Elsewhere a timed-out wait is stood in for by pre-loading
the device status word (mimo_attn_set_device_status), after which every kernel
with bounded waits returns at entry; bad sequence metadata is caught by the
kernels' own bounds checks before any access.  Each test checks the reported
status, that nothing was written where nothing may be, and that the next call
after the status is read runs normally.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle.fp8 import decode_fp8
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def nan_like(shape, dtype=torch.float32):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


def expect_status(code):
    with pytest.raises(mimo.MimoAttnError) as ei:
        mimo.mimo_attn_device_status()
    assert ei.value.status == code, ei.value
    mimo.mimo_attn_device_status()  # read and cleared: OK now


def test_a_wait_that_runs_out_records_timeout_and_the_next_calls_run():
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    mimo.mimo_attn_wait_selftest()
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert waited >= 0.9, waited  # it gave up at the bound, not before
    expect_status(mimo.MIMO_ERR_TIMEOUT)
    # the context still works: a decode after the time-out matches the oracle
    x = W.decode_inputs([1, 300, 4000], 4096, 0, seed=9)
    out, lse = mimo.mimo_attn_decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(),
                                     0, x.sinks.cuda(), out_dtype=torch.float32)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    P.check(out, ro, lse, rl, what="decode after a time-out")


def test_kernels_return_at_entry_after_a_recorded_timeout():
    d = lambda t: None if t is None else t.to("cuda")  # noqa: E731
    # sliding-window prefill (G = 16: the packed kernel) and global prefill (the general one)
    x = W.prefill_inputs([300, 129], hq=16, hkv=1, seed=5)
    q, k, v, s, cu = d(x.q), d(x.k), d(x.v), d(x.sinks), d(x.cu_seqlens)
    # global decode with several splits (split kernel + combine), a ring decode, FP8 decode
    dg = W.decode_inputs([5000, 70], 8192, 0, seed=6)
    dr = W.decode_inputs([300, 5], 129, 129, seed=7)
    d8 = W.decode_inputs_fp8([5000, 70], 8192, 0, seed=8)
    assert mimo.mimo_attn_decode_workspace_size(64, 4, 2, 8192, 0) > 0

    def launch_all(outs):
        mimo.mimo_attn_prefill(q, k, v, s, 129, cu, 300, out=outs[0], lse=outs[1])
        mimo.mimo_attn_prefill(q, k, v, s, 0, cu, 300, out=outs[2], lse=outs[3])
        mimo.mimo_attn_decode(d(dg.q), d(dg.k_cache), d(dg.v_cache), d(dg.seqlens), 0, d(dg.sinks),
                              out=outs[4], lse=outs[5])
        mimo.mimo_attn_decode(d(dr.q), d(dr.k_cache), d(dr.v_cache), d(dr.seqlens), 129,
                              d(dr.sinks), out=outs[6], lse=outs[7])
        mimo.mimo_attn_decode_fp8(d(d8.q), d(d8.k_codes), d(d8.v_codes), d(d8.k_scale),
                                  d(d8.v_scale_kv), d(d8.seqlens), 0, d(d8.sinks), out=outs[8],
                                  lse=outs[9])

    shapes = [(429, 16, 128), (16, 429)] * 2 + [(2, 64, 128), (2, 64)] * 3
    outs = [nan_like(sh) for sh in shapes]
    mimo.mimo_attn_set_device_status(mimo.MIMO_ERR_TIMEOUT)
    launch_all(outs)
    expect_status(mimo.MIMO_ERR_TIMEOUT)
    for i, t in enumerate(outs):
        assert torch.isnan(t).all(), f"output {i} was written after the recorded timeout"

    # the status was cleared: the same calls now compute the results
    launch_all(outs)
    mimo.mimo_attn_device_status()
    for window, (o, l) in ((129, outs[0:2]), (0, outs[2:4])):
        ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
        P.check(o, ro, l, rl, what=f"prefill W={window} after recovery")
    ro, rl = oracle.decode(dg.q, dg.k_cache, dg.v_cache, dg.seqlens, 0, dg.sinks)
    P.check(outs[4], ro, outs[5], rl, what="decode after recovery")
    ro, rl = oracle.decode(dr.q, dr.k_cache, dr.v_cache, dr.seqlens, 129, dr.sinks)
    P.check(outs[6], ro, outs[7], rl, what="ring decode after recovery")
    ro, rl = decode_fp8(d8.q, d8.k_codes, d8.v_codes, d8.k_scale, d8.v_scale_kv, d8.seqlens, 0,
                        d8.sinks)
    P.check(outs[8], ro, outs[9], rl, what="fp8 decode after recovery")


# cu_seqlens arrays that break the contract, for tokens [0, 300): the first
# sequence [0, 100) is always valid; the second is not.
BAD_CU = {
    "past total_tokens": ([0, 100, 400], 300),
    "decreasing": ([0, 100, 60], 100),
    "longer than max_seqlen": ([0, 100, 300], 150),
}


@pytest.mark.parametrize("case", sorted(BAD_CU))
@pytest.mark.parametrize("hq,hkv,window", [(16, 1, 129), (4, 1, 0), (4, 1, 129)])
def test_bad_cu_seqlens_is_reported_and_touches_nothing(case, hq, hkv, window):
    """Both prefill kernels check every sequence against total_tokens and
    max_seqlen on the device: a bad one is skipped (no row read or written) and
    reported as MIMO_ERR_INVALID_ARG; the valid sequence is still computed."""
    cu_list, max_seqlen = BAD_CU[case]
    x = W.prefill_inputs([100, 200], hq=hq, hkv=hkv, seed=9)
    cu = torch.tensor(cu_list, dtype=torch.int32, device="cuda")
    out, lse = nan_like((300, hq, 128)), nan_like((hq, 300))
    mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.sinks.cuda(), window, cu,
                           max_seqlen, out=out, lse=lse)
    expect_status(mimo.MIMO_ERR_INVALID_ARG)
    assert torch.isnan(out[100:]).all() and torch.isnan(lse[:, 100:]).all()
    ro, rl = oracle.prefill(x.q[:100], x.k[:100], x.v[:100], x.sinks, window,
                            W.cu_seqlens_of([100]))
    P.check(out[:100], ro, lse[:, :100], rl, what=f"valid sequence beside a bad one ({case})")


@pytest.mark.parametrize("case", sorted(BAD_CU))
def test_bad_cu_seqlens_in_the_backward_is_reported(case):
    """The backward kernels check sequences the same way: the valid sequence's
    gradients equal those of a clean call; the status reports the bad one."""
    cu_list, max_seqlen = BAD_CU[case]
    x = W.prefill_inputs([100, 200], hq=16, hkv=2, seed=10)
    q, k, v, s = (t.cuda() for t in (x.q, x.k, x.v, x.sinks))
    good = W.cu_seqlens_of([100, 200]).cuda()
    out, lse = mimo.mimo_attn_prefill(q, k, v, s, 0, good, 200)
    g = torch.Generator().manual_seed(11)
    dout = torch.randn(out.shape, generator=g).to(out.dtype).cuda()
    ref = mimo.mimo_attn_prefill_backward(q, k, v, out, lse, dout, s, 0, good, 200)
    mimo.mimo_attn_device_status()
    bad = torch.tensor(cu_list, dtype=torch.int32, device="cuda")
    got = mimo.mimo_attn_prefill_backward(q, k, v, out, lse, dout, s, 0, bad, max_seqlen)
    expect_status(mimo.MIMO_ERR_INVALID_ARG)
    for name, a, b in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        assert torch.equal(a[:100], b[:100]), name


def test_decode_lengths_outside_the_cache_are_reported():
    """A negative length, or one past a linear cache's capacity, is recorded as
    MIMO_ERR_INVALID_ARG (the length is clamped into the cache, nothing outside
    it is read); the other sequences are unaffected."""
    x = W.decode_inputs([700, 64, 3], 1024, 0, hq=16, hkv=1, seed=12, poison=False)
    sl = torch.tensor([700, 2000, -4], dtype=torch.int32, device="cuda")
    out, lse = mimo.mimo_attn_decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), sl, 0,
                                     x.sinks.cuda(), out_dtype=torch.float32)
    expect_status(mimo.MIMO_ERR_INVALID_ARG)
    ro, rl = oracle.decode(x.q[:1], x.k_cache[:1], x.v_cache[:1], x.seqlens[:1], 0, x.sinks)
    P.check(out[:1], ro, lse[:1], rl, what="valid sequence beside bad lengths")
    assert np.isfinite(out.cpu().numpy()).all()
