"""Context-parallel decode of a global layer: each sequence's keys are split
across the ranks of a process group (one GPU each), each rank decodes its
part without the sink, the ranks exchange their (out, lse) and every rank
merges them with the sink.

The exchange is the one collective of the operator: an all-gather of
B x Hq x (Dv + 1) fp32 values per rank (NCCL over NVLink on B200 nodes).
Softmax over a union of disjoint key sets is the log-sum-exp merge of the
parts (see ``mimo_attn_decode_merge`` in include/mimo_attn.h), so any split
of the positions works and the ranks' order does not matter.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def _local_part_cuda(q, k_cache, v_cache, part_lens, softmax_scale):
    from . import mimo_attn_decode

    return mimo_attn_decode(q, k_cache, v_cache, part_lens, 0, None, out_dtype=torch.float32,
                            softmax_scale=softmax_scale)


def _merge_cuda(part_out, part_lse, sinks, out_dtype, v_scale):
    from . import mimo_attn_decode_merge

    return mimo_attn_decode_merge(part_out, part_lse, sinks, out_dtype=out_dtype, v_scale=v_scale)


def context_parallel_decode(q, k_cache, v_cache, part_lens, sinks, group=None,
                            out_dtype=torch.bfloat16, v_scale=1.0, softmax_scale=None,
                            local_part=None, merge=None):
    """One decode step of a global layer whose caches are split across ``group``.

    Args:
      q: [B, Hq, Dqk] the new token's queries, the same on every rank.
      k_cache, v_cache: [B, C, Hkv, D] this rank's part of each sequence's keys
        and values (slots 0 .. part_lens[b] - 1 hold them, in any order).
      part_lens: [B] int32, keys of each sequence held by this rank (0 allowed).
      sinks: [Hq] fp32 or None; applied once, in the merge.

    Returns (out [B, Hq, Dv], lse [B, Hq]) on every rank.

    ``local_part`` and ``merge`` default to this library's CUDA entry points
    (mimo_attn_decode without the sink, then mimo_attn_decode_merge).
    """
    local_part = local_part or _local_part_cuda
    merge = merge or _merge_cuda
    part_out, part_lse = local_part(q, k_cache, v_cache, part_lens, softmax_scale)
    B, hq, dv = part_out.shape
    # one exchange: each rank's (out, lse) packed as [B, Hq, Dv + 1], in fp32 at least
    # (lse rounded to a 16-bit type would shift the merge weights)
    dt = torch.promote_types(torch.promote_types(part_out.dtype, part_lse.dtype), torch.float32)
    packed = torch.cat([part_out.reshape(B, hq, dv).to(dt), part_lse.reshape(B, hq, 1).to(dt)],
                       dim=2).contiguous()
    world = dist.get_world_size(group)
    gathered = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(gathered, packed, group=group)
    g = torch.stack(gathered)
    return merge(g[..., :dv].contiguous(), g[..., dv].contiguous(), sinks, out_dtype, v_scale)
