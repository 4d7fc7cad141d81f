"""Prefill kernel (tcgen05) vs the fp64 oracle, through the C ABI.

Small cases are compared element by element on every row; the full-size
workloads (T = 32768 sliding-window and global layers, the 16-sequence
varlen 5:1 stack) on sampled rows the oracle computes one by one, plus
properties that hold at any size.
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


def run_gpu(x, window, out_dtype=torch.float32, v_scale=1.0):
    dev = "cuda"
    q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
    s = None if x.sinks is None else x.sinks.to(dev)
    cu = x.cu_seqlens.to(dev)
    maxlen = max(x.lengths) if x.lengths else 0
    out, lse = mimo.mimo_attn_prefill(q, k, v, s, window, cu, maxlen, out_dtype=out_dtype,
                                      v_scale=v_scale)
    mimo.mimo_attn_device_status()
    return out, lse


def test_tiny_swa_config():
    """T=512, Hq=16, Hkv=1, window 129, fp32 out, seed 0: every element."""
    x = W.prefill_inputs([512], hq=16, hkv=1, seed=0)
    out, lse = run_gpu(x, 129, torch.float32)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens)
    P.check(out, ro, lse, rl, what="tiny SWA")


@pytest.mark.parametrize("window", [1, 2, 128, 129, 130, 0])
@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 130, 255, 256, 257, 1000])
def test_lengths_and_windows(T, window):
    sinks = (T + window) % 2 == 0
    x = W.prefill_inputs([T], hq=4, hkv=2, seed=T * 7 + window, sinks=sinks)
    out_dtype = torch.bfloat16 if T % 2 else torch.float32
    out, lse = run_gpu(x, window, out_dtype)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    P.check(out, ro, lse, rl, what=f"T={T} W={window}")


@pytest.mark.parametrize("window", [0, 129, 3])
def test_varlen_pack_with_empty_and_single_token_sequences(window):
    lengths = [0, 1, 300, 0, 129, 1000, 5, 128]
    x = W.prefill_inputs(lengths, hq=8, hkv=2, seed=41 + window)
    out, lse = run_gpu(x, window, torch.bfloat16)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    P.check(out, ro, lse, rl, what=f"varlen W={window}")


# global layers (window 0) and windows the packed sliding-window kernel cannot
# hold (N > 160) run on the per-head kernel: every length class around the
# 128-row tile edge, at several head groupings


@pytest.mark.parametrize("hq,hkv,window", [(8, 2, 0), (8, 2, 1), (8, 2, 2), (8, 2, 129),
                                           (32, 2, 0), (32, 4, 300), (4, 1, 128)])
def test_per_head_kernel_lengths(hq, hkv, window):
    for T in (1, 2, 127, 128, 129, 255, 256, 257, 1000):
        sinks = (T + window) % 2 == 1
        x = W.prefill_inputs([T], hq=hq, hkv=hkv, seed=T * 13 + window + hq, sinks=sinks)
        out_dtype = torch.bfloat16 if T % 3 == 0 else torch.float32
        out, lse = run_gpu(x, window, out_dtype)
        ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
        P.check(out, ro, lse, rl, what=f"per-head Hq={hq} Hkv={hkv} T={T} W={window}")


def test_per_head_kernel_varlen_every_length_class():
    """Sequences of every length class packed into one call."""
    lengths = [1, 1000, 0, 129, 2000, 127, 3, 700, 128, 1500]
    x = W.prefill_inputs(lengths, hq=16, hkv=2, seed=61)
    for window in (0, 500):
        out, lse = run_gpu(x, window, torch.float32)
        ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
        P.check(out, ro, lse, rl, what=f"per-head varlen W={window}")


@pytest.mark.parametrize("window", [0, 129])
def test_many_short_sequences(window):
    """A thousand sequences of 0 to 9 tokens in one pack (16 query heads on one
    key/value head: the packed kernel for the window, the per-head kernel for
    global): almost every work item starts a new sequence."""
    rng = np.random.default_rng(71)
    lengths = [int(L) for L in rng.integers(0, 10, 1000)]
    x = W.prefill_inputs(lengths, hq=16, hkv=1, seed=72 + window)
    out, lse = run_gpu(x, window, torch.float32)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    P.check(out, ro, lse, rl, what=f"1000 short sequences W={window}")


def test_varlen_pack_equals_separate_calls():
    lengths = [200, 1, 513]
    x = W.prefill_inputs(lengths, hq=8, hkv=2, seed=5)
    out, lse = run_gpu(x, 129, torch.bfloat16)
    b0 = 0
    for L in lengths:
        y = W.PrefillInputs(x.q[b0:b0 + L], x.k[b0:b0 + L], x.v[b0:b0 + L], x.sinks,
                            W.cu_seqlens_of([L]), [L])
        o1, l1 = run_gpu(y, 129, torch.bfloat16)
        assert torch.equal(o1, out[b0:b0 + L])
        assert torch.equal(l1, lse[:, b0:b0 + L])
        b0 += L


@pytest.mark.parametrize("hq,hkv", [(6, 2), (16, 1), (64, 4), (2, 2)])
def test_head_groupings(hq, hkv):
    """Odd group size (unpaired last head), MQA, the model's 64/4, and MHA."""
    x = W.prefill_inputs([300], hq=hq, hkv=hkv, seed=hq + hkv)
    for window in (0, 129):
        out, lse = run_gpu(x, window, torch.float32)
        ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
        P.check(out, ro, lse, rl, what=f"Hq={hq} Hkv={hkv} W={window}")


def test_no_sink_and_v_scale():
    x = W.prefill_inputs([400], hq=4, hkv=1, seed=77, sinks=False)
    out, lse = run_gpu(x, 0, torch.float32, v_scale=0.707)
    ro, rl = oracle.prefill(x.q, x.k, x.v, None, 0, x.cu_seqlens, v_scale=0.707)
    P.check(out, ro, lse, rl, what="no sink, v_scale")


def test_large_sink_dominates():
    """Sinks far above every score: the output shrinks toward 0, lse toward sigma."""
    x = W.prefill_inputs([260], hq=4, hkv=1, seed=3)
    x.sinks = torch.full_like(x.sinks, 30.0)
    out, lse = run_gpu(x, 129, torch.float32)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens)
    P.check(out, ro, lse, rl, what="large sink")


def test_rescale_path_with_growing_scores():
    """Keys whose scores grow along the sequence force repeated running-max moves."""
    x = W.prefill_inputs([1024], hq=4, hkv=1, seed=8, sinks=False)
    ramp = torch.linspace(0.0, 6.0, 1024).to(torch.float32)[:, None, None]
    x.k = (x.k.float() * 0.25 + ramp * x.q[:, :1].float().sign()).to(torch.bfloat16)
    out, lse = run_gpu(x, 0, torch.float32)
    ro, rl = oracle.prefill(x.q, x.k, x.v, None, 0, x.cu_seqlens)
    # Attention here is nearly one-hot (|out| ~ |v|); the scaled scores grow
    # by ~96 (base 2) along the keys, so later tiles overflow the first tile's
    # reference and move it (O rescaled); the flat bound holds for fp32 output.
    P.check(out, ro, lse, rl, what="rescale")


@pytest.mark.parametrize("window", [0, 300])
def test_reference_moves_above_the_sink(window):
    """Scores far above the sink logit (base-2 spread ~23 per key): P against
    the sink's reference overflows and the kernel moves it, on the first tile
    of a row and on later ones."""
    x = W.prefill_inputs([1000, 300], hq=8, hkv=2, seed=9)
    x.q = (x.q.float() * 4).to(torch.bfloat16)
    x.k = (x.k.float() * 4).to(torch.bfloat16)
    out, lse = run_gpu(x, window, torch.float32)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    P.check(out, ro, lse, rl, what=f"reference moves W={window}")


# ----------------------------------------------------------------------------
# full-size workloads (sampled rows)


def sample_rows(lengths, window, per_seq_random=8, seed=0):
    rng = np.random.default_rng(seed)
    rows = []
    b0 = 0
    for L in lengths:
        if L == 0:
            continue
        r = set(range(min(L, 256)))                       # first two query tiles
        r |= {x for x in (127, 128, 129, 255, 256, 257, L - 129, L - 128, L - 1) if 0 <= x < L}
        r |= set(range(max(0, L - 128), L, 8))             # the last tile, every 8th row
        if window > 0:
            r |= {x for x in (window - 1, window, window + 1, 2 * window) if 0 <= x < L}
        r |= set(int(x) for x in rng.integers(0, L, per_seq_random))
        rows.extend(b0 + x for x in sorted(r))
        b0 += L
    return np.array(rows, dtype=np.int64)


def full_size_check(lengths, window, hq=64, hkv=4, seed=0, per_seq_random=64, sinks=None,
                    what=""):
    """One full-size layer with both output types: fp32 output under the flat
    stated bound, bf16 output (the bench's) under it plus its own rounding."""
    x = W.prefill_inputs(lengths, hq=hq, hkv=hkv, seed=seed, device="cuda")
    if sinks is not None:
        x.sinks = sinks.to("cuda")
    rows = sample_rows(lengths, window, per_seq_random, seed)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens, rows=rows)
    idx = torch.as_tensor(rows, device="cuda")
    errs = {}
    for odt in (torch.float32, torch.bfloat16):
        out, lse = mimo.mimo_attn_prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens,
                                          max(lengths), out_dtype=odt)
        mimo.mimo_attn_device_status()
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        errs[str(odt)] = P.check(out[idx], ro, lse[:, idx], rl,
                                 what=f"full size {what} W={window} {odt}")
        del out, lse
    print(f"max-abs {what} W={window} rows={len(rows)}: {errs}")


def test_full_size_swa_32k():
    full_size_check([32768], 129, what="T=32768")


def test_full_size_global_32k():
    full_size_check([32768], 0, per_seq_random=32, what="T=32768")


def test_longest_position_swa():
    """One sequence as long as the model's positions go (MiMoV2FlashConfig
    max_position_embeddings = 131072) on the packed sliding-window kernel."""
    full_size_check([131072], 129, per_seq_random=16, what="T=131072")


def test_longest_position_global():
    """The same length on a global layer: rows up to 131072 keys long."""
    full_size_check([131072], 0, per_seq_random=4, what="T=131072")


def test_full_size_varlen_stack():
    lengths = W.varlen_stack_lengths(0)
    sinks = W.stack_sinks(len(W.STACK_WINDOWS), seed=0)
    for layer, window in enumerate(W.STACK_WINDOWS):
        full_size_check(lengths, window, seed=100 + layer, per_seq_random=4, sinks=sinks[layer],
                        what=f"stack layer {layer}")


@pytest.mark.parametrize("odt", [torch.bfloat16, torch.float32])
def test_output_only_16_byte_aligned(odt):
    """An output pointer aligned to 16 but not 32 bytes takes the 16-byte store path."""
    x = W.prefill_inputs([300], hq=4, hkv=1, seed=17)
    n = 300 * 4 * 128
    flat = torch.empty(n + 16, dtype=odt, device="cuda")
    shift = 16 // flat.element_size()
    out = flat[shift:shift + n].view(300, 4, 128)
    assert out.data_ptr() % 32 == 16
    mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.sinks.cuda(), 129,
                           x.cu_seqlens.cuda(), 300, out=out)
    mimo.mimo_attn_device_status()
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens)
    P.check(out, ro, what="16-byte aligned out")


# ----------------------------------------------------------------------------
# sliding window with the key/value group packed into the MMA rows
# (G = Hq/Hkv in {8, 16, 32}; N = roundup16(W + 256/G - 1) <= 160, else the
# per-head kernel takes the call: the largest packed windows are 129 at G=8,
# 145 at G=16 and 153 at G=32, and the next window up crosses to the other kernel)


@pytest.mark.parametrize("hq,hkv", [(16, 1), (16, 2), (64, 2)])
@pytest.mark.parametrize("window", [1, 2, 8, 128, 129, 130, 145, 146, 153, 154, 186])
def test_packed_window_lengths(hq, hkv, window):
    for T in (1, 2, 7, 8, 9, 127, 129, 300, 1000):
        sinks = (T + window) % 3 != 0
        x = W.prefill_inputs([T], hq=hq, hkv=hkv, seed=T * 31 + window + hq, sinks=sinks)
        out, lse = run_gpu(x, window, torch.float32 if T % 2 else torch.bfloat16)
        ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
        P.check(out, ro, lse, rl, what=f"packed Hq={hq} Hkv={hkv} T={T} W={window}")


@pytest.mark.parametrize("window", [129, 5])
def test_packed_window_varlen(window):
    lengths = [0, 1, 300, 0, 129, 1000, 5, 128, 7]
    x = W.prefill_inputs(lengths, hq=16, hkv=1, seed=88 + window)
    out, lse = run_gpu(x, window, torch.bfloat16)
    ro, rl = oracle.prefill(x.q, x.k, x.v, x.sinks, window, x.cu_seqlens)
    P.check(out, ro, lse, rl, what=f"packed varlen W={window}")


def test_packed_window_16_byte_aligned_output():
    x = W.prefill_inputs([300], hq=16, hkv=1, seed=19)
    n = 300 * 16 * 128
    flat = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    out = flat[8:8 + n].view(300, 16, 128)
    assert out.data_ptr() % 32 == 16
    mimo.mimo_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.sinks.cuda(), 129,
                           x.cu_seqlens.cuda(), 300, out=out)
    mimo.mimo_attn_device_status()
    ro, _ = oracle.prefill(x.q, x.k, x.v, x.sinks, 129, x.cu_seqlens)
    P.check(out, ro, what="packed, 16-byte aligned out")
