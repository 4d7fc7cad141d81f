"""Every entry point once through the bounds-checked build of the library.

Run as its own process with MIMO_ATTN_CHECKED=1 (tests/test_checked_build_gpu.py
does so): the binding then loads libmimo_attn_checked.so, in which every kernel
checks the row index of each global read or write against its buffer.  Each
call here must match the fp64 oracle, leave the device status word clear and
record no bounds site.  The last step runs the build's self-test, whose check
fails without touching memory, and expects MIMO_ERR_BOUNDS and its site.
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import global_attention_swa_b200 as mimo  # noqa: E402
import oracle  # noqa: E402
import workloads as W  # noqa: E402
from oracle.fp8 import decode_fp8  # noqa: E402
from oracle.rope import rope_append  # noqa: E402
from tests import parity_util as P  # noqa: E402


def clean(what):
    st = mimo.lib.mimo_attn_device_status(None)
    site = mimo.mimo_attn_checked_site()
    assert st == mimo.MIMO_OK and site == 0, f"{what}: status {st}, bounds site {site}"


def main():
    assert mimo.CHECKED and mimo.mimo_attn_is_checked_build(), "not the checked build"
    torch.cuda.set_device(0)

    # prefill: packed sliding window (G=16), the per-head kernel (global and a
    # window too wide to pack), a pack with empty and one-token sequences
    for hq, hkv, lengths, window in (
        (16, 1, [300, 1, 129], 129), (16, 1, [300, 1, 129], 0), (8, 2, [0, 260, 5, 0], 300),
        (64, 4, [700], 129), (64, 4, [700], 0),
    ):
        x = W.prefill_inputs(lengths, hq=hq, hkv=hkv, seed=len(lengths) + window)
        for odt in (torch.float32, torch.bfloat16):
            out, lse = mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.sinks.cuda(), window,
                                              x.cu_seqlens.cuda(), max(lengths), out_dtype=odt)
            clean(f"prefill W={window}")
            ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
            P.check(out, ro, lse, rl, what=f"checked prefill W={window} {odt}")

    # decode: split linear cache (several splits and the combine), windowed
    # linear cache, 129-slot ring
    for lengths, cap, window in (([1, 700, 5000, 0], 8192, 0), ([900, 129, 5], 2048, 129),
                                 ([300, 129, 5, 1], 129, 129)):
        x = W.decode_inputs(lengths, cap, window, seed=cap + window)
        out, lse = mimo.mimo_attn_decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(),
                                         window, x.sinks.cuda(), out_dtype=torch.float32)
        clean(f"decode C={cap} W={window}")
        ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, window, x.sinks)
        P.check(out, ro, lse, rl, what=f"checked decode C={cap} W={window}")

    # the decode entry point without a caller workspace (partials in the library's own array)
    x = W.decode_inputs([1, 700, 5000, 0], 8192, 0, seed=21)
    out = torch.empty((4, 64, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((4, 64), dtype=torch.float32, device="cuda")
    mimo.mimo_attn_decode_noalloc(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), 0,
                                  x.sinks.cuda(), out, lse)
    clean("decode without workspace")
    ro, rl = oracle.decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0, x.sinks)
    P.check(out, ro, lse, rl, what="checked decode without workspace")

    # FP8 (e4m3) cache decode
    x = W.decode_inputs_fp8([1, 65, 1000, 129], 1024, 0, hq=8, hkv=2, seed=7)
    out, lse = mimo.mimo_attn_decode_fp8(x.q.cuda(), x.k_codes.cuda(), x.v_codes.cuda(), x.k_scale.cuda(),
                                         x.v_scale_kv.cuda(), x.seqlens.cuda(), x.window, x.sinks.cuda(),
                                         out_dtype=torch.float32)
    clean("fp8 decode")
    ro, rl = decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale_kv, x.seqlens, x.window, x.sinks)
    P.check(out, ro, lse, rl, what="checked fp8 decode")

    # rotary embedding + append into a ring and a linear cache
    for lengths, cap, window in (([1, 128, 130], 129, 129), ([1, 100, 4096], 4096, 0)):
        x = W.decode_inputs(lengths, cap, window, seed=11, poison=False)
        g = torch.Generator().manual_seed(12)
        q = torch.randn((len(lengths), 64, 192), generator=g).to(torch.bfloat16)
        kn = torch.randn((len(lengths), 4, 192), generator=g).to(torch.bfloat16)
        vn = torch.randn((len(lengths), 4, 128), generator=g).to(torch.bfloat16)
        rq, _, _ = rope_append(q, kn, vn, x.k_cache, x.v_cache, x.seqlens, window, 10000.0, 192)
        qd, kc, vc = q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
        mimo.mimo_attn_rope_append(qd, kn.cuda(), vn.cuda(), kc, vc, x.seqlens.cuda(), window, 10000.0, 192)
        clean(f"rope append C={cap}")
        assert np.all(np.abs(P.to64(qd) - rq) <= 2.0 ** -8 * np.abs(rq) + 1e-5), "rope q"

    # context-parallel merge of three parts
    g = torch.Generator().manual_seed(13)
    po = torch.randn((3, 5, 64, 128), generator=g)
    pl = torch.randn((3, 5, 64), generator=g)
    sinks = torch.randn(64, generator=g)
    out, lse = mimo.mimo_attn_decode_merge(po.cuda(), pl.cuda(), sinks.cuda(), out_dtype=torch.float32)
    clean("merge")

    # prefill backward: tcgen05 passes (bf16 out / dout) and the warp-level ones (fp32)
    x = W.prefill_inputs([300, 0, 129], hq=16, hkv=1, seed=14)
    for window in (0, 129):
        for odt in (torch.bfloat16, torch.float32):
            out, lse = mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.sinks.cuda(), window,
                                              x.cu_seqlens.cuda(), 300, out_dtype=odt)
            dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(15)).to(odt).cuda()
            grads = mimo.mimo_attn_prefill_backward(x.q.cuda(), x.k.cuda(), x.v.cuda(), out, lse, dout,
                                                    x.sinks.cuda(), window, x.cu_seqlens.cuda(), 300)
            clean(f"backward W={window} {odt}")
            assert all(torch.isfinite(t).all() for t in grads if t is not None)

    # the bench's full-size workloads (and its backward case): no row index of
    # any kernel may leave its buffer at these sizes either (results are checked
    # by the parity tests)
    for window in (129, 0):
        x = W.prefill_inputs([32768], seed=40 + window, device="cuda")
        out, lse = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, 32768)
        clean(f"full-size prefill W={window}")
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        del x, out, lse
    x = W.prefill_inputs([8192], seed=43, device="cuda")
    out, lse = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, 0, x.cu_seqlens, 8192)
    dout = torch.randn(out.shape, device="cuda").to(out.dtype)
    grads = mimo.mimo_attn_prefill_backward(x.q, x.k, x.v, out, lse, dout, x.sinks, 0, x.cu_seqlens, 8192)
    clean("full-size backward T=8192")
    assert all(torch.isfinite(t).all() for t in grads)
    del x, out, lse, dout, grads
    lengths = W.decode_b64_lengths(0)
    for cap, window in ((W.DECODE_GA_CAPACITY, 0), (129, 129)):
        x = W.decode_inputs(lengths, cap, window, seed=42, device="cuda")
        out, lse = mimo.mimo_attn_decode(x.q, x.k_cache, x.v_cache, x.seqlens, window, x.sinks)
        clean(f"full-size decode C={cap}")
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        del x, out, lse
    torch.cuda.empty_cache()

    # the self-test: a failing check that touches no memory
    mimo.mimo_attn_checked_selftest()
    st = mimo.lib.mimo_attn_device_status(None)
    site = mimo.mimo_attn_checked_site()
    src = open(os.path.join(ROOT, "global_attention_swa_b200", "csrc", "mimo_attn.cu")).read().splitlines()
    line = next(i + 1 for i, l in enumerate(src) if "MIMO_ROW_OK(row, 4)" in l)
    assert st == mimo.MIMO_ERR_BOUNDS and site == 10 * 10000 + line, (st, site, line)
    clean("after the self-test")
    print("checked ok")


if __name__ == "__main__":
    main()
