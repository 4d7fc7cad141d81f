"""Context-parallel decode on one GPU: the keys of each sequence split into parts
("virtual ranks"), each part decoded by mimo_attn_decode without the sink, the
parts merged by mimo_attn_decode_merge -- against the fp64 oracle decode over all
keys, and the merge kernel alone against the oracle merge.  (The exchange between
ranks is an all_gather, covered on CPU with gloo.)"""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle.merge import merge as oracle_merge
from tests import parity_util as P

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import global_attention_swa_b200 as mimo


def _split(x, parts_of):
    """parts_of(b, L) -> list of position lists; returns per-part (k, v, lens) on the GPU."""
    B = x.q.shape[0]
    lengths = x.seqlens.tolist()
    nparts = len(parts_of(0, lengths[0]))
    out = []
    for r in range(nparts):
        pos = [parts_of(b, L)[r] for b, L in enumerate(lengths)]
        cap = max(1, max(len(p) for p in pos))
        k = torch.zeros((B, cap) + tuple(x.k_cache.shape[2:]), dtype=torch.bfloat16)
        v = torch.zeros((B, cap) + tuple(x.v_cache.shape[2:]), dtype=torch.bfloat16)
        for b, p in enumerate(pos):
            if p:
                k[b, :len(p)] = x.k_cache[b, p]
                v[b, :len(p)] = x.v_cache[b, p]
        lens = torch.tensor([len(p) for p in pos], dtype=torch.int32)
        out.append((k.cuda(), v.cuda(), lens.cuda()))
    return out


SPLITS = {
    "halves": lambda b, L: [list(range(0, L // 2)), list(range(L // 2, L))],
    "three_with_empty": lambda b, L: [list(range(0, min(L, 100))), [], list(range(min(L, 100), L))],
    "interleaved": lambda b, L: [list(range(0, L, 2)), list(range(1, L, 2))],
}


@pytest.mark.parametrize("split", sorted(SPLITS))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_virtual_ranks_merge_to_the_full_decode(split, out_dtype):
    lengths = [1, 2, 100, 101, 3000, 8191]
    x = W.decode_inputs(lengths, 8192, 0, seed=51, poison=False)
    q = x.q.cuda()
    parts = _split(x, SPLITS[split])
    outs, lses = [], []
    for k, v, lens in parts:
        o, l = mimo.mimo_attn_decode(q, k, v, lens, 0, None, out_dtype=torch.float32)
        outs.append(o)
        lses.append(l)
    out, lse = mimo.mimo_attn_decode_merge(torch.stack(outs), torch.stack(lses), x.sinks.cuda(),
                                           out_dtype=out_dtype, v_scale=0.707)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks, v_scale=0.707)
    P.check(out, ro, lse, rl, what=f"context-parallel {split}")
    full, full_lse = mimo.mimo_attn_decode(q, x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(),
                                           0, x.sinks.cuda(), out_dtype=out_dtype, v_scale=0.707)
    torch.cuda.synchronize()
    assert (lse - full_lse).abs().max().item() < 1e-4


def test_merge_kernel_matches_oracle_merge():
    g = torch.Generator().manual_seed(5)
    R, B, H = 5, 7, 64
    po = torch.randn((R, B, H, 128), generator=g)
    pl = torch.randn((R, B, H), generator=g) * 3
    pl[1, 2] = -float("inf")          # empty part for one sequence
    po[1, 2] = float("nan")           # whose output must be ignored
    pl[:, 4] = -float("inf")          # a sequence with no keys anywhere
    sinks = torch.randn(H, generator=g)
    out, lse = mimo.mimo_attn_decode_merge(po.cuda(), pl.cuda(), sinks.cuda(), out_dtype=torch.float32,
                                           v_scale=1.3)
    mimo.mimo_attn_device_status()
    ro, rl = oracle_merge(po, pl, sinks, v_scale=1.3)
    P.check(out, ro, lse, rl, what="merge kernel")
    out2, lse2 = mimo.mimo_attn_decode_merge(po.cuda(), pl.cuda(), None, out_dtype=torch.float32)
    ro2, rl2 = oracle_merge(po, pl, None)
    P.check(out2, ro2, lse2, rl2, what="merge kernel, no sink")
    assert torch.all(out2[4] == 0) and torch.all(torch.isneginf(lse2[4]))
