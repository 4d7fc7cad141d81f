"""Seeded random configurations against the fp64 oracle: prefill, decode,
FP8 decode and the prefill backward.

Each case draws packed lengths (or cache lengths and capacity), a window, a
head grouping, sinks on or off and an output type, so that combinations no
hand-written case names (a window just past a run of tile edges, an odd group
size on the packed path, empty sequences between long ones) are compared
element by element under the same bounds as the other parity tests.
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

GROUPS = [(1, 1), (2, 1), (6, 2), (8, 1), (16, 1), (16, 2), (32, 1), (64, 4), (64, 2)]


def _case(seed):
    rng = np.random.default_rng(seed)
    hq, hkv = GROUPS[rng.integers(len(GROUPS))]
    n = int(rng.integers(1, 6))
    lengths = [int(x) for x in rng.integers(0, 600, n)]
    if rng.random() < 0.3:  # a length on a 128-row tile edge
        lengths[int(rng.integers(n))] = int(128 * rng.integers(1, 5) + rng.integers(-1, 2))
    if rng.random() < 0.3:
        lengths[int(rng.integers(n))] = 0
    window = int(rng.choice([0, 0, 1, 2, 97, 127, 128, 129, 130, 145, 153, 154,
                             int(rng.integers(3, 400)), int(rng.integers(3, 400))]))
    sinks = bool(rng.random() < 0.8)
    odt = torch.float32 if rng.random() < 0.5 else torch.bfloat16
    return hq, hkv, lengths, window, sinks, odt


@pytest.mark.parametrize("seed", range(24))
def test_prefill_random_configuration(seed):
    hq, hkv, lengths, window, sinks, odt = _case(1000 + seed)
    if max(lengths) == 0:
        lengths[0] = 1
    x = W.prefill_inputs(lengths, hq=hq, hkv=hkv, seed=seed, sinks=sinks)
    out, lse = mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(),
                                      None if x.sinks is None else x.sinks.cuda(), window,
                                      x.cu_seqlens.cuda(), max(lengths), out_dtype=odt)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    P.check(out, ro, lse, rl, what=f"seed {seed}: Hq={hq} Hkv={hkv} W={window} L={lengths}")


@pytest.mark.parametrize("seed", range(16))
def test_decode_random_configuration(seed):
    rng = np.random.default_rng(2000 + seed)
    hq, hkv = [(8, 1), (16, 1), (16, 2), (64, 4), (6, 2), (2, 2)][int(rng.integers(6))]
    ring = bool(rng.random() < 0.4)
    window = 129 if ring else int(rng.choice([0, 0, 1, int(rng.integers(2, 3000))]))
    cap = 129 if ring else int(rng.integers(1, 9000))
    B = int(rng.integers(1, 7))
    lengths = [int(x) for x in rng.integers(0, 3 * cap if ring else cap + 1, B)]
    sinks = bool(rng.random() < 0.8)
    odt = torch.float32 if rng.random() < 0.5 else torch.bfloat16
    x = W.decode_inputs(lengths, cap, window, hq=hq, hkv=hkv, seed=seed, sinks=sinks)
    out, lse = mimo.mimo_attn_decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(),
                                     window, None if x.sinks is None else x.sinks.cuda(), out_dtype=odt)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, window, x.sinks)
    P.check(out, ro, lse, rl, what=f"seed {seed}: Hq={hq} Hkv={hkv} C={cap} W={window} L={lengths}")


@pytest.mark.parametrize("seed", range(10))
def test_backward_random_configuration(seed):
    from oracle.backward import prefill_backward

    rng = np.random.default_rng(3000 + seed)
    hq, hkv = [(2, 1), (4, 2), (8, 1), (16, 1), (6, 2)][int(rng.integers(5))]
    n = int(rng.integers(1, 4))
    lengths = [int(x) for x in rng.integers(0, 300, n)]
    lengths[0] = max(lengths[0], 1)
    window = int(rng.choice([0, 1, 64, 129, int(rng.integers(2, 300))]))
    sinks = bool(rng.random() < 0.8)
    io = torch.float32 if rng.random() < 0.4 else torch.bfloat16
    x = W.prefill_inputs(lengths, hq=hq, hkv=hkv, seed=seed, sinks=sinks, device="cuda")
    out, lse = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, max(lengths),
                                      out_dtype=io)
    dout = torch.randn(out.shape, generator=torch.Generator(device="cuda").manual_seed(seed),
                       device="cuda").to(io)
    got = mimo.mimo_attn_prefill_backward(x.q, x.k, x.v, out, lse, dout, x.sinks, window,
                                          x.cu_seqlens, max(lengths))
    mimo.mimo_attn_device_status()
    ref = prefill_backward(x.q, x.k, x.v, dout, x.sinks, window, x.cu_seqlens)
    for name, a, b in zip(("dq", "dk", "dv", "dsinks"), got, ref):
        if b is None:
            assert a is None
            continue
        g = P.to64(a)
        scale = np.abs(b).max()
        err = np.abs(g - b).max()
        assert err <= 1e-2 * scale + 1e-4, (
            f"seed {seed} {name}: Hq={hq} Hkv={hkv} W={window} L={lengths} {io}: {err:.3e} vs {scale:.3e}")


@pytest.mark.parametrize("seed", range(8))
def test_decode_fp8_random_configuration(seed):
    from oracle.fp8 import decode_fp8

    rng = np.random.default_rng(4000 + seed)
    hq, hkv = [(8, 1), (16, 1), (16, 2), (64, 4), (6, 2)][int(rng.integers(5))]
    ring = bool(rng.random() < 0.4)
    window = 129 if ring else int(rng.choice([0, 0, 1, int(rng.integers(2, 3000))]))
    cap = 129 if ring else int(rng.integers(1, 9000))
    B = int(rng.integers(1, 6))
    lengths = [int(x) for x in rng.integers(0, 3 * cap if ring else cap + 1, B)]
    x = W.decode_inputs_fp8(lengths, cap, window, hq=hq, hkv=hkv, seed=seed,
                            sinks=bool(rng.random() < 0.8))
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    out, lse = mimo.mimo_attn_decode_fp8(d(x.q), d(x.k_codes), d(x.v_codes), d(x.k_scale),
                                         d(x.v_scale_kv), d(x.seqlens), x.window, d(x.sinks),
                                         out_dtype=torch.float32)
    mimo.mimo_attn_device_status()
    ro, rl = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, x.window,
                        x.sinks)
    P.check(out, ro, lse, rl, what=f"fp8 seed {seed}: Hq={hq} Hkv={hkv} C={cap} W={window} L={lengths}")
