"""The entry points run inside a captured CUDA graph (decode, prefill, backward).

A serving loop captures a decode step once and replays it every token with
new inputs copied into the captured buffers; a training or prefill loop can
do the same for fixed shapes.  None of the calls synchronises the host or
allocates device memory when its buffers are given, so each is captured as
its kernel launches.  Each test captures the calls, replays the graph with
two different sets of inputs, and compares every replay with the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first calls outside the capture (one-time host setup)
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_step_replays():
    lengths = [1, 700, 5000, 129]
    ga = W.decode_inputs(lengths, 8192, 0, seed=41, device="cuda")        # several splits + combine
    sw = W.decode_inputs(lengths, 129, 129, seed=42, device="cuda")       # 129-slot ring
    ws = torch.empty(max(1, mimo.mimo_attn_decode_workspace_size(64, 4, 4, 8192, 0)),
                     dtype=torch.uint8, device="cuda")
    o_ga = torch.empty((4, 64, 128), dtype=torch.float32, device="cuda")
    l_ga = torch.empty((4, 64), dtype=torch.float32, device="cuda")
    o_sw, l_sw = torch.empty_like(o_ga), torch.empty_like(l_ga)

    def step():
        mimo.mimo_attn_decode(ga.q, ga.k_cache, ga.v_cache, ga.seqlens, 0, ga.sinks,
                              out=o_ga, lse=l_ga, workspace=ws)
        mimo.mimo_attn_decode(sw.q, sw.k_cache, sw.v_cache, sw.seqlens, 129, sw.sinks,
                              out=o_sw, lse=l_sw)

    g = _capture(step)
    gen = torch.Generator(device="cuda").manual_seed(43)
    for trial in range(2):
        ga.q.copy_(torch.randn(ga.q.shape, generator=gen, device="cuda").to(ga.q.dtype))
        sw.q.copy_(torch.randn(sw.q.shape, generator=gen, device="cuda").to(sw.q.dtype))
        o_ga.fill_(float("nan"))
        o_sw.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        mimo.mimo_attn_device_status()
        ro, rl = oracle.decode(ga.q, ga.k_cache, ga.v_cache, ga.seqlens, 0, ga.sinks)
        P.check(o_ga, ro, l_ga, rl, what=f"graph replay {trial}: global decode")
        ro, rl = oracle.decode(sw.q, sw.k_cache, sw.v_cache, sw.seqlens, 129, sw.sinks)
        P.check(o_sw, ro, l_sw, rl, what=f"graph replay {trial}: ring decode")
    del g


def test_prefill_replays():
    lengths = [300, 1, 129, 0, 513]
    x = W.prefill_inputs(lengths, seed=44, device="cuda")
    nt = sum(lengths)
    outs = {w: (torch.empty((nt, 64, 128), dtype=torch.float32, device="cuda"),
                torch.empty((64, nt), dtype=torch.float32, device="cuda")) for w in (129, 0)}

    def step():
        for w, (o, l) in outs.items():
            mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, w, x.cu_seqlens, max(lengths), out=o, lse=l)

    g = _capture(step)
    gen = torch.Generator(device="cuda").manual_seed(45)
    for trial in range(2):
        for t in (x.q, x.k, x.v):
            t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(t.dtype))
        for o, _ in outs.values():
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        mimo.mimo_attn_device_status()
        for w, (o, l) in outs.items():
            ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, w, x.cu_seqlens)
            P.check(o, ro, l, rl, what=f"graph replay {trial}: prefill W={w}")
    del g


def test_backward_replays():
    lengths = [200, 0, 129]
    x = W.prefill_inputs(lengths, hq=16, hkv=1, seed=46, device="cuda")
    nt = sum(lengths)
    out = torch.empty((nt, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((16, nt), dtype=torch.float32, device="cuda")
    dout = torch.empty_like(out)
    res = {}

    def step():
        mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, 0, x.cu_seqlens, 200, out=out, lse=lse)
        res["g"] = mimo.mimo_attn_prefill_backward(x.q, x.k, x.v, out, lse, dout, x.sinks, 0,
                                                   x.cu_seqlens, 200)

    from oracle.backward import prefill_backward

    gen = torch.Generator(device="cuda").manual_seed(47)
    dout.copy_(torch.randn(dout.shape, generator=gen, device="cuda").to(dout.dtype))
    g = _capture(step)
    for trial in range(2):
        for t in (x.q, x.k, x.v, dout):
            t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(t.dtype))
        g.replay()
        torch.cuda.synchronize()
        mimo.mimo_attn_device_status()
        ref = prefill_backward(x.q, x.k, x.v, dout, x.sinks, 0, x.cu_seqlens)
        for name, a, b in zip(("dq", "dk", "dv", "dsinks"), res["g"], ref):
            err = np.abs(P.to64(a) - b).max()
            assert err <= 1e-2 * np.abs(b).max() + 1e-4, f"graph replay {trial}: {name} {err:.3e}"
    del g


def test_calls_on_two_streams_at_once():
    """A prefill on one stream and a decode on another, launched back to back
    so that they can run concurrently: each result matches the oracle."""
    x = W.prefill_inputs([700, 129], seed=48, device="cuda")
    d = W.decode_inputs([1, 3000, 129], 4096, 0, seed=49, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s1):
        po, pl = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens, 700,
                                        out_dtype=torch.float32, stream=s1)
    with torch.cuda.stream(s2):
        do, dl = mimo.mimo_attn_decode(d.q, d.k_cache, d.v_cache, d.seqlens, 0, d.sinks,
                                       out_dtype=torch.float32, stream=s2)
    torch.cuda.synchronize()
    mimo.mimo_attn_device_status()
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens)
    P.check(po, ro, pl, rl, what="prefill on its own stream")
    ro, rl = oracle.decode(d.q, d.k_cache, d.v_cache, d.seqlens, 0, d.sinks)
    P.check(do, ro, dl, rl, what="decode on its own stream")
