"""Prefill backward (mimo_attn_prefill_backward) vs the fp64 oracle backward.

The forward runs on the GPU (its out and lse feed the backward, as in
training); the oracle recomputes everything in fp64.  Tolerance per gradient
tensor: relative Frobenius error <= 1e-2 and every element within
1e-2 * max|ref| + 1e-4 -- the kernels round P and dS to bf16 as MMA operands
(2^-8 relative each), like P in the forward, and accumulate in fp32; the
1e-4 floor covers gradients that are exactly zero in exact arithmetic (a row
with one visible key and no sink: D and dP cancel up to fp32 summation order),
next to gradient magnitudes of 0.1-10 here.
"""

import numpy as np
import pytest
import torch

import workloads as W
from oracle.backward import prefill_backward, prefill_backward_sampled
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def grad_check(got, ref, what):
    g = P.to64(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    scale = np.abs(ref).max()
    err = np.abs(g - ref)
    assert err.max() <= 1e-2 * scale + 1e-4, f"{what}: max err {err.max():.3e} vs scale {scale:.3e}"
    if scale > 1e-3:
        fro = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        assert fro <= 1e-2, f"{what}: rel-Frobenius {fro:.3e}"
    else:
        fro = 0.0
    return fro


def _run(lengths, hq, hkv, window, sinks, out_dtype, seed, v_scale=1.0):
    x = W.prefill_inputs(lengths, hq=hq, hkv=hkv, seed=seed, sinks=sinks, device="cuda")
    maxlen = max(lengths)
    out, lse = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, maxlen,
                                      out_dtype=out_dtype, v_scale=v_scale)
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    dout = torch.randn(out.shape, generator=g, device="cuda").to(out_dtype)
    dq, dk, dv, ds = mimo.mimo_attn_prefill_backward(x.q, x.k, x.v, out, lse, dout, x.sinks, window,
                                                     x.cu_seqlens, maxlen, v_scale=v_scale)
    mimo.mimo_attn_device_status()
    rq, rk, rv, rs = prefill_backward(x.q, x.k, x.v, dout, x.sinks, window, x.cu_seqlens,
                                      v_scale=v_scale)
    return (dq, dk, dv, ds), (rq, rk, rv, rs)


# fp32 out / dout take the two warp-level dV and dK passes, bf16 the tcgen05 pass
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("window", [129, 0, 1])
@pytest.mark.parametrize("sinks", [True, False])
def test_tiny_heads(window, sinks, io):
    got, ref = _run([512], 16, 1, window, sinks, io, seed=window + 3)
    for name, a, b in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        grad_check(a, b, f"{name} W={window}")
    if sinks:
        grad_check(got[3], ref[3], "dsinks")
    else:
        assert got[3] is None


def test_small_groups_bf16():
    """Two query heads per KV head and ragged lengths around the 128-key tile."""
    got, ref = _run([127, 128, 129, 300], 4, 2, 0, True, torch.bfloat16, seed=21)
    for name, a, b in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        grad_check(a, b, name)


@pytest.mark.parametrize("window", [129, 0])
def test_model_heads_varlen_bf16(window):
    got, ref = _run([300, 0, 129, 64, 1], 64, 4, window, True, torch.bfloat16, seed=11, v_scale=0.707)
    for name, a, b in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        grad_check(a, b, f"{name} W={window}")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_many_short_sequences(io):
    """Three hundred sequences of 0 to 9 tokens: every key tile and query tile
    is a sequence's first and last."""
    lengths = [int(L) for L in np.random.default_rng(81).integers(0, 10, 300)]
    got, ref = _run(lengths, 16, 1, 129, True, io, seed=82)
    for name, a, b in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        grad_check(a, b, f"{name} short sequences")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_deterministic(io):
    a, _ = _run([200, 70], 16, 2, 129, True, io, seed=5)
    b, _ = _run([200, 70], 16, 2, 129, True, io, seed=5)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def sampled_check(got, ref, what):
    """Per-element bound of grad_check over a sample (scale = the sample's max |ref|)."""
    g = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    scale = np.abs(ref).max()
    err = np.abs(g - ref).max()
    assert err <= 1e-2 * scale + 1e-4, f"{what}: max err {err:.3e} vs scale {scale:.3e}"
    fro = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert fro <= 1e-2, f"{what}: rel-Frobenius {fro:.3e}"


@pytest.mark.parametrize("T,window,q_rows,k_rows", [
    # the benchmark's backward: one global layer at T=8192 (keys near the end: the
    # oracle needs every query row that sees a key)
    (8192, 0, [0, 1, 63, 64, 127, 128, 4095, 4096, 8190, 8191], [7690, 8000, 8127, 8128, 8191]),
    # a sliding-window layer at T=32768, keys anywhere
    (32768, 129, [0, 128, 129, 16383, 32767], [0, 1, 63, 64, 20000, 32640, 32767]),
])
def test_full_size_sampled(T, window, q_rows, k_rows):
    """Model head shape, bf16 forward output, full length, in the launch configuration the
    benchmark times; the oracle gives dq, dk, dv and dsinks at sampled positions."""
    x = W.prefill_inputs([T], seed=T + window, device="cuda")
    out, lse = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, T)
    g = torch.Generator(device="cuda").manual_seed(T + window + 1)
    dout = torch.randn(out.shape, generator=g, device="cuda").to(out.dtype)
    dq, dk, dv, ds = mimo.mimo_attn_prefill_backward(x.q, x.k, x.v, out, lse, dout, x.sinks, window,
                                                     x.cu_seqlens, T)
    mimo.mimo_attn_device_status()
    q_heads, kv_heads, sink_heads = [0, 17, 63], [0, 3], [5, 60]
    rq, rk, rv, rs = prefill_backward_sampled(x.q.cpu(), x.k.cpu(), x.v.cpu(), dout.cpu(), x.sinks.cpu(),
                                              window, q_rows, q_heads, k_rows, kv_heads,
                                              sink_heads=sink_heads)
    sampled_check(dq[q_rows][:, q_heads].cpu(), rq, f"dq T={T}")
    sampled_check(dk[k_rows][:, kv_heads].cpu(), rk, f"dk T={T}")
    sampled_check(dv[k_rows][:, kv_heads].cpu(), rv, f"dv T={T}")
    sampled_check(ds[sink_heads].cpu(), rs, f"dsinks T={T}")
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
