"""Context-parallel decode plumbing on CPU: two gloo ranks each hold part of every
sequence's keys, exchange their partial results with all_gather and merge.

The CUDA steps (local decode, merge) are replaced here by CPU stand-ins from
the oracle, so this checks what the module itself does -- which rank holds
what, the collective's shapes and order, the merge input layout -- against
the decode over all keys.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_part(q, k, v, lens, scale):
    import oracle

    o, l = oracle.decode(q, k, v, lens, 0, None, ring=False, scale=scale)
    return torch.from_numpy(o), torch.from_numpy(l)


def _cpu_merge(po, pl, sinks, out_dtype, v_scale):
    from oracle.merge import merge

    o, l = merge(po, pl, sinks, v_scale)
    return torch.from_numpy(o), torch.from_numpy(l)


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from global_attention_swa_b200.context_parallel import context_parallel_decode
    from workloads import decode_inputs

    lengths = [1, 9, 30, 64]
    x = decode_inputs(lengths, 64, 0, hq=4, hkv=2, dqk=8, dv=4, seed=21, poison=False)
    # rank r holds positions [r*L/2, (r+1)*L/2) of each sequence, rank 1 in reverse slot order
    kc = torch.zeros_like(x.k_cache)
    vc = torch.zeros_like(x.v_cache)
    lens = []
    for b, L in enumerate(lengths):
        lo, hi = (0, L // 2) if rank == 0 else (L // 2, L)
        idx = list(range(lo, hi))
        if rank == 1:
            idx = idx[::-1]
        lens.append(len(idx))
        for s, p in enumerate(idx):
            kc[b, s] = x.k_cache[b, p]
            vc[b, s] = x.v_cache[b, p]
    out, lse = context_parallel_decode(x.q, kc, vc, torch.tensor(lens, dtype=torch.int32), x.sinks,
                                       v_scale=0.9, softmax_scale=0.3, local_part=_cpu_part,
                                       merge=_cpu_merge)
    results[rank] = (out.numpy(), lse.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_merge_to_the_full_decode():
    import oracle
    from workloads import decode_inputs

    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    x = decode_inputs([1, 9, 30, 64], 64, 0, hq=4, hkv=2, dqk=8, dv=4, seed=21, poison=False)
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks, scale=0.3, v_scale=0.9)
    for r in range(world):
        out, lse = results[r]
        np.testing.assert_allclose(out, ro, atol=1e-12)
        np.testing.assert_allclose(lse, rl, atol=1e-12)
