"""The C-ABI library loads, exports what include/*.h declares, and validates
arguments on the host.  CPU only: no call here reaches a kernel launch."""

import ctypes
import glob
import os
import re

import pytest

import global_attention_swa_b200 as mimo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced (validation fails first)


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(mimo_attn_\w+)\s*\(", src))
    return names


def test_header_declares_the_entry_points():
    assert set(mimo.EXPORTED) <= declared_symbols()


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(mimo.LIB_PATH)
    for name in sorted(declared_symbols()):
        assert hasattr(lib, name), name


CHECKED_LIB = os.path.join(os.path.dirname(mimo.LIB_PATH), "libmimo_attn_checked.so")


@pytest.mark.skipif(not os.path.exists(CHECKED_LIB), reason="checked build not built")
def test_checked_build_exports_the_same_symbols_and_says_so():
    lib = ctypes.CDLL(CHECKED_LIB)
    for name in sorted(declared_symbols()):
        assert hasattr(lib, name), name
    assert lib.mimo_attn_is_checked_build() == 1
    assert ctypes.CDLL(os.path.join(os.path.dirname(mimo.LIB_PATH), "libmimo_attn.so")
                       ).mimo_attn_is_checked_build() == 0


def test_checked_runner_compiles():
    """tests/checked_calls.py runs only on a GPU, in its own process: at least
    keep it syntactically valid here."""
    path = os.path.join(ROOT, "tests", "checked_calls.py")
    compile(open(path).read(), path, "exec")


def test_wait_selftest_without_a_device_reports_a_cuda_error():
    # no GPU here: the launch fails and the status says so (nothing waits)
    import torch

    if torch.cuda.is_available():
        pytest.skip("a device is present: the GPU test runs the real time-out")
    assert mimo.lib.mimo_attn_wait_selftest(None) == mimo.MIMO_ERR_CUDA


def test_selftest_is_refused_outside_the_checked_build():
    if mimo.CHECKED:
        pytest.skip("the checked build is loaded")
    assert mimo.lib.mimo_attn_checked_selftest(None) == mimo.MIMO_ERR_UNSUPPORTED


def _dims(hq=64, hkv=4, dqk=192, dv=128):
    return mimo.make_dims(hq, hkv, dqk, dv)


def _prefill(dims, q=FAKE, k=FAKE, v=FAKE, window=129, cu=FAKE, nseq=1, total=128, maxlen=128,
             out=FAKE):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    d = ctypes.byref(dims) if dims is not None else None
    return mimo.lib.mimo_attn_prefill(d, p(q), p(k), p(v), None, window, p(cu), nseq, total,
                                      maxlen, p(out), None, None)


def test_prefill_rejects_bad_arguments():
    assert _prefill(None) == mimo.MIMO_ERR_INVALID_ARG
    assert _prefill(_dims(), window=-1) == mimo.MIMO_ERR_INVALID_ARG
    assert _prefill(_dims(hq=6, hkv=4)) == mimo.MIMO_ERR_INVALID_ARG
    assert _prefill(_dims(dqk=128)) == mimo.MIMO_ERR_UNSUPPORTED
    assert _prefill(_dims(dv=192)) == mimo.MIMO_ERR_UNSUPPORTED
    assert _prefill(_dims(), q=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _prefill(_dims(), cu=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _prefill(_dims(), k=FAKE + 2) == mimo.MIMO_ERR_INVALID_ARG   # misaligned
    assert _prefill(_dims(), maxlen=129, total=128) == mimo.MIMO_ERR_INVALID_ARG


def test_prefill_empty_is_a_no_op():
    assert _prefill(_dims(), total=0, maxlen=0) == mimo.MIMO_OK
    assert _prefill(_dims(), nseq=0, total=0, maxlen=0) == mimo.MIMO_OK


def _decode(dims, batch=2, cap=1024, window=0, ws=None, ws_bytes=0, q=FAKE, out=FAKE):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    return mimo.lib.mimo_attn_decode(ctypes.byref(dims), p(q), p(FAKE), p(FAKE), p(FAKE), batch,
                                     cap, window, None, p(out), None, p(ws), ws_bytes, None)


def test_decode_rejects_bad_arguments():
    assert _decode(_dims(), window=-3) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode(_dims(), q=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode(_dims(), out=FAKE + 4) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode(_dims(hq=64, hkv=2)) == mimo.MIMO_ERR_UNSUPPORTED   # 32 heads per group
    assert _decode(_dims(), cap=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode(_dims(), batch=0) == mimo.MIMO_OK


def test_decode_workspace_contract():
    need = mimo.mimo_attn_decode_workspace_size(64, 4, 64, 262144, 0)
    assert need > 0 and need % 16 == 0
    assert _decode(_dims(), batch=64, cap=262144, ws=None) == mimo.MIMO_ERR_WORKSPACE
    assert _decode(_dims(), batch=64, cap=262144, ws=FAKE, ws_bytes=need - 16) == mimo.MIMO_ERR_WORKSPACE
    assert "workspace" in mimo.lib.mimo_attn_last_error().decode()


def test_ring_decode_needs_no_workspace():
    # a 129-slot ring with window 129 is covered by one split per (sequence, KV head)
    assert mimo.mimo_attn_decode_workspace_size(64, 4, 64, 129, 129) == 0


def _decode_fp8(dims, batch=2, cap=1024, window=0, ks=FAKE, vs=FAKE, ws=None, ws_bytes=0, q=FAKE):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    return mimo.lib.mimo_attn_decode_fp8(ctypes.byref(dims), p(q), p(FAKE), p(FAKE), p(ks), p(vs),
                                         p(FAKE), batch, cap, window, None, p(FAKE), None, p(ws),
                                         ws_bytes, None)


def test_decode_fp8_rejects_bad_arguments():
    assert _decode_fp8(_dims(), ks=0) == mimo.MIMO_ERR_INVALID_ARG
    assert "k_scale" in mimo.lib.mimo_attn_last_error().decode()
    assert _decode_fp8(_dims(), vs=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode_fp8(_dims(), ks=FAKE + 2) == mimo.MIMO_ERR_INVALID_ARG   # misaligned scales
    assert _decode_fp8(_dims(), window=-1) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode_fp8(_dims(), q=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _decode_fp8(_dims(dqk=128)) == mimo.MIMO_ERR_UNSUPPORTED
    assert _decode_fp8(_dims(), batch=0) == mimo.MIMO_OK


def test_decode_fp8_workspace_matches_bf16_plan():
    for args in ((64, 4, 64, 262144, 0), (64, 4, 64, 129, 129), (16, 1, 3, 5000, 0)):
        dims = mimo.make_dims(args[0], args[1])
        assert (mimo.lib.mimo_attn_decode_fp8_workspace_size(ctypes.byref(dims), *args[2:])
                == mimo.mimo_attn_decode_workspace_size(*args))
    need = mimo.mimo_attn_decode_workspace_size(64, 4, 64, 262144, 0)
    assert _decode_fp8(_dims(), batch=64, cap=262144, ws=None) == mimo.MIMO_ERR_WORKSPACE
    assert _decode_fp8(_dims(), batch=64, cap=262144, ws=FAKE, ws_bytes=need - 16) == mimo.MIMO_ERR_WORKSPACE


def _rope(dims, batch=2, cap=64, window=0, theta=10000.0, rd=192, q=FAKE):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    return mimo.lib.mimo_attn_rope_append(ctypes.byref(dims), p(q), p(FAKE), p(FAKE), p(FAKE),
                                          p(FAKE), p(FAKE), batch, cap, window, theta, rd, None)


def test_rope_append_rejects_bad_arguments():
    assert _rope(_dims(), theta=0.0) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), theta=float("nan")) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), theta=float("inf")) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), rd=7) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), rd=194) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), rd=-2) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), window=-1) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), cap=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), q=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(), q=FAKE + 2) == mimo.MIMO_ERR_INVALID_ARG
    assert _rope(_dims(dqk=128)) == mimo.MIMO_ERR_UNSUPPORTED
    assert _rope(_dims(), batch=0) == mimo.MIMO_OK


def test_decode_merge_rejects_bad_arguments():
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    call = lambda nparts=2, batch=2, po=FAKE, out=FAKE: mimo.lib.mimo_attn_decode_merge(  # noqa: E731
        ctypes.byref(_dims()), p(po), p(FAKE), nparts, batch, None, p(out), None, None)
    assert call(nparts=0) == mimo.MIMO_ERR_INVALID_ARG
    assert call(batch=-1) == mimo.MIMO_ERR_INVALID_ARG
    assert call(po=0) == mimo.MIMO_ERR_INVALID_ARG
    assert call(out=FAKE + 8) == mimo.MIMO_ERR_INVALID_ARG
    assert call(batch=0) == mimo.MIMO_OK


def _bwd(dims, sinks=None, dsinks=None, ws=FAKE, ws_bytes=1 << 30, total=128, maxlen=128, dq=FAKE):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    return mimo.lib.mimo_attn_prefill_backward(
        ctypes.byref(dims), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(FAKE), p(sinks), 0,
        p(FAKE), 1, total, maxlen, p(dq), p(FAKE), p(FAKE), p(dsinks), p(ws), ws_bytes, None)


def test_prefill_backward_rejects_bad_arguments():
    need = mimo.lib.mimo_attn_prefill_backward_workspace_size(ctypes.byref(_dims()), 128)
    assert need == 2 * 64 * 128 * 4
    assert _bwd(_dims(), sinks=FAKE, dsinks=None) == mimo.MIMO_ERR_INVALID_ARG
    assert "dsinks" in mimo.lib.mimo_attn_last_error().decode()
    assert _bwd(_dims(), ws=None) == mimo.MIMO_ERR_WORKSPACE
    assert _bwd(_dims(), ws_bytes=need - 4) == mimo.MIMO_ERR_WORKSPACE
    assert _bwd(_dims(), dq=0) == mimo.MIMO_ERR_INVALID_ARG
    assert _bwd(_dims(), dq=FAKE + 4) == mimo.MIMO_ERR_INVALID_ARG
    assert _bwd(_dims(), maxlen=129) == mimo.MIMO_ERR_INVALID_ARG
    assert _bwd(_dims(dv=192)) == mimo.MIMO_ERR_UNSUPPORTED
    assert _bwd(_dims(), total=0, maxlen=0) == mimo.MIMO_OK


def test_last_error_is_empty_after_success():
    assert _prefill(_dims(), total=0, maxlen=0) == mimo.MIMO_OK
    assert mimo.lib.mimo_attn_last_error().decode() == ""


def test_binding_refuses_tensors_it_cannot_pass_as_plain_pointers():
    """The binding passes raw device addresses: host tensors, strided views and
    wrong dtypes are refused before the library is called."""
    import types

    import torch

    assert mimo._ptr(None) is None
    with pytest.raises(ValueError, match="CUDA"):
        mimo._ptr(torch.zeros(4), "x")
    fake = lambda contig, dt: types.SimpleNamespace(  # noqa: E731
        is_cuda=True, is_contiguous=lambda: contig, dtype=dt, data_ptr=lambda: 4096)
    with pytest.raises(ValueError, match="contiguous"):
        mimo._ptr(fake(False, torch.bfloat16), "q", torch.bfloat16)
    with pytest.raises(TypeError, match="q must be"):
        mimo._ptr(fake(True, torch.float16), "q", torch.bfloat16)
    with pytest.raises(TypeError):
        mimo._ptr(fake(True, torch.float16), "out", (torch.bfloat16, torch.float32))
    assert mimo._ptr(fake(True, torch.float32), "out", (torch.bfloat16, torch.float32)).value == 4096
    # a wrapper given host tensors fails in the binding, not in the library
    q = torch.zeros((8, 4, 192), dtype=torch.bfloat16)
    k = torch.zeros((8, 1, 192), dtype=torch.bfloat16)
    v = torch.zeros((8, 1, 128), dtype=torch.bfloat16)
    cu = torch.tensor([0, 8], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        mimo.mimo_attn_prefill(q, k, v, None, 0, cu, 8)


def test_every_wrapper_accepts_its_documented_dtypes(monkeypatch):
    """Dry run of each wrapper on host tensors of the documented dtypes against a
    stand-in library that records its calls (the device check alone is bypassed):
    argument checks and marshalling raise nothing for valid inputs."""
    import types

    import torch

    calls = []

    class FakeLib:
        def __getattr__(self, name):
            def fn(*args):
                calls.append(name)
                return 0
            return fn

    real_ptr = mimo._ptr

    def host_ptr(t, name="tensor", dtype=None):
        if t is None:
            return None
        proxy = types.SimpleNamespace(is_cuda=True, is_contiguous=t.is_contiguous, dtype=t.dtype,
                                      data_ptr=t.data_ptr)
        return real_ptr(proxy, name, dtype)

    monkeypatch.setattr(mimo, "lib", FakeLib())
    monkeypatch.setattr(mimo, "_ptr", host_ptr)
    monkeypatch.setattr(mimo, "_stream", lambda stream, dev: None)
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    B, C, Hq, Hkv, Nt = 2, 16, 4, 1, 24
    q = torch.zeros((Nt, Hq, 192), dtype=bf)
    k = torch.zeros((Nt, Hkv, 192), dtype=bf)
    v = torch.zeros((Nt, Hkv, 128), dtype=bf)
    sinks = torch.zeros(Hq, dtype=f32)
    cu = torch.tensor([0, 10, 24], dtype=i32)
    for odt in (bf, f32):
        out, lse = mimo.mimo_attn_prefill(q, k, v, sinks, 129, cu, 14, out_dtype=odt)
        assert out.dtype == odt and lse.dtype == f32
        dout = torch.zeros_like(out)
        dq, dk, dv, ds = mimo.mimo_attn_prefill_backward(q, k, v, out, lse, dout, sinks, 0, cu, 14)
        assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
        with pytest.raises(TypeError):
            mimo.mimo_attn_prefill_backward(q, k, v, out, lse, dout.to(f32 if odt == bf else bf),
                                            sinks, 0, cu, 14)
    qd = torch.zeros((B, Hq, 192), dtype=bf)
    kc = torch.zeros((B, C, Hkv, 192), dtype=bf)
    vc = torch.zeros((B, C, Hkv, 128), dtype=bf)
    sl = torch.tensor([3, 16], dtype=i32)
    mimo.mimo_attn_decode(qd, kc, vc, sl, 0, sinks)
    mimo.mimo_attn_decode(qd, kc, vc, sl, 0, None, out_dtype=f32)
    codes_k = torch.zeros((B, C, Hkv, 192), dtype=torch.uint8)
    codes_v = torch.zeros((B, C, Hkv, 128), dtype=torch.uint8)
    scale = torch.ones(Hkv, dtype=f32)
    mimo.mimo_attn_decode_fp8(qd, codes_k, codes_v, scale, scale, sl, 0, sinks)
    mimo.mimo_attn_rope_append(qd, torch.zeros((B, Hkv, 192), dtype=bf), torch.zeros((B, Hkv, 128), dtype=bf),
                               kc, vc, sl, 16, 10000.0)
    mimo.mimo_attn_decode_merge(torch.zeros((3, B, Hq, 128)), torch.zeros((3, B, Hq)), sinks)
    mimo.mimo_attn_decode_noalloc(qd, kc, vc, sl, 0, sinks, torch.zeros((B, Hq, 128), dtype=bf))
    seen = list(calls)
    with pytest.raises(TypeError, match="seqlens"):
        mimo.mimo_attn_decode(qd, kc, vc, sl.long(), 0, sinks)
    # sizes that disagree with the ones derived from q would be read past their end
    with pytest.raises(ValueError, match="k has shape"):
        mimo.mimo_attn_prefill(q, k[:-1], v, sinks, 0, cu, 14)
    with pytest.raises(ValueError, match="v_cache"):
        mimo.mimo_attn_decode(qd, kc, vc[:1], sl, 0, sinks)
    with pytest.raises(ValueError, match="seqlens"):
        mimo.mimo_attn_decode(qd, kc, vc, sl[:1], 0, sinks)
    with pytest.raises(ValueError, match="sinks"):
        mimo.mimo_attn_decode(qd, kc, vc, sl, 0, torch.zeros(Hq + 1))
    with pytest.raises(ValueError, match="part_lse"):
        mimo.mimo_attn_decode_merge(torch.zeros((3, B, Hq, 128)), torch.zeros((2, B, Hq)), sinks)
    with pytest.raises(ValueError, match="contiguous"):
        mimo.mimo_attn_decode(qd, kc[:, ::2], vc[:, ::2], sl, 0, sinks)
    # every tensor must be on the call's device (q's): the library launches on one
    # device and would dereference another GPU's addresses
    calls.clear()
    meta = lambda t: t.to("meta")  # noqa: E731  (a device other than q's)
    with pytest.raises(ValueError, match="v is on meta"):
        mimo.mimo_attn_prefill(q, k, meta(v), sinks, 0, cu, 14)
    with pytest.raises(ValueError, match="cu_seqlens is on meta"):
        mimo.mimo_attn_prefill(q, k, v, sinks, 0, meta(cu), 14)
    with pytest.raises(ValueError, match="out is on meta"):
        mimo.mimo_attn_prefill(q, k, v, sinks, 0, cu, 14, out=torch.empty((Nt, Hq, 128), device="meta"))
    with pytest.raises(ValueError, match="k_cache is on meta"):
        mimo.mimo_attn_decode(qd, meta(kc), vc, sl, 0, sinks)
    with pytest.raises(ValueError, match="workspace is on meta"):
        mimo.mimo_attn_decode(qd, kc, vc, sl, 0, sinks, workspace=torch.empty(16, device="meta"))
    with pytest.raises(ValueError, match="k_scale is on meta"):
        mimo.mimo_attn_decode_fp8(qd, codes_k, codes_v, meta(scale), scale, sl, 0, sinks)
    with pytest.raises(ValueError, match="v_cache is on meta"):
        mimo.mimo_attn_rope_append(qd, torch.zeros((B, Hkv, 192), dtype=bf),
                                   torch.zeros((B, Hkv, 128), dtype=bf), kc, meta(vc), sl, 16, 1e4)
    with pytest.raises(ValueError, match="sinks is on meta"):
        mimo.mimo_attn_decode_merge(torch.zeros((3, B, Hq, 128)), torch.zeros((3, B, Hq)), meta(sinks))
    with pytest.raises(ValueError, match="dout is on meta"):
        mimo.mimo_attn_prefill_backward(q, k, v, out, lse, meta(torch.zeros_like(out)), sinks, 0, cu, 14)
    with pytest.raises(ValueError, match="seqlens is on meta"):
        mimo.mimo_attn_decode_noalloc(qd, kc, vc, meta(sl), 0, sinks, torch.zeros((B, Hq, 128), dtype=bf))
    # refused before any entry point that touches the device (size queries are host-only)
    assert [c for c in calls if not c.endswith("_workspace_size")] == []
    assert {"mimo_attn_prefill", "mimo_attn_prefill_backward", "mimo_attn_decode", "mimo_attn_decode_fp8",
            "mimo_attn_rope_append", "mimo_attn_decode_merge", "mimo_attn_decode_noalloc"} <= set(seen)


def test_a_failed_launch_reaches_the_caller_as_an_exception(monkeypatch):
    """A launch failure inside the library (simulated: a stand-in library whose
    entry points return MIMO_ERR_CUDA, as the real one does when
    cudaGetLastError reports one) reaches the caller of every wrapper as
    MimoAttnError carrying the status and the library's message."""
    import types

    import torch

    class FailingLib:
        def mimo_attn_last_error(self):
            return b"prefill launch: unspecified launch failure"

        def mimo_attn_decode_workspace_size(self, *a):
            return 1024

        def mimo_attn_decode_fp8_workspace_size(self, *a):
            return 1024

        def mimo_attn_prefill_backward_workspace_size(self, *a):
            return 1024

        def __getattr__(self, name):
            return lambda *a: mimo.MIMO_ERR_CUDA

    real_ptr = mimo._ptr

    def host_ptr(t, name="tensor", dtype=None):
        if t is None:
            return None
        proxy = types.SimpleNamespace(is_cuda=True, is_contiguous=t.is_contiguous, dtype=t.dtype,
                                      data_ptr=t.data_ptr)
        return real_ptr(proxy, name, dtype)

    monkeypatch.setattr(mimo, "lib", FailingLib())
    monkeypatch.setattr(mimo, "_ptr", host_ptr)
    monkeypatch.setattr(mimo, "_stream", lambda stream, dev: None)
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    q = torch.zeros((24, 4, 192), dtype=bf)
    k = torch.zeros((24, 1, 192), dtype=bf)
    v = torch.zeros((24, 1, 128), dtype=bf)
    cu = torch.tensor([0, 24], dtype=i32)
    qd = torch.zeros((2, 4, 192), dtype=bf)
    kc = torch.zeros((2, 16, 1, 192), dtype=bf)
    vc = torch.zeros((2, 16, 1, 128), dtype=bf)
    sl = torch.tensor([3, 16], dtype=i32)
    calls = [
        lambda: mimo.mimo_attn_prefill(q, k, v, None, 129, cu, 24),
        lambda: mimo.mimo_attn_decode(qd, kc, vc, sl, 0, None),
        lambda: mimo.mimo_attn_decode_merge(torch.zeros((2, 2, 4, 128)), torch.zeros((2, 2, 4)), None),
        lambda: mimo.mimo_attn_device_status(device="cpu"),
    ]
    for call in calls:
        with pytest.raises(mimo.MimoAttnError) as e:
            call()
        assert e.value.status == mimo.MIMO_ERR_CUDA
        assert "launch failure" in str(e.value)


def test_binding_refuses_a_stream_of_another_device():
    """A caller's stream must belong to the device the tensors live on."""
    import types

    import torch

    other = types.SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=0)
    with pytest.raises(ValueError, match="stream belongs to cuda:1"):
        mimo._stream(other, torch.device("cuda", 0))
    same = types.SimpleNamespace(device=torch.device("cuda", 0), cuda_stream=1234)
    assert mimo._stream(same, torch.device("cuda", 0)).value == 1234


def test_set_device_status_rejects_codes_outside_the_enum():
    assert mimo.lib.mimo_attn_set_device_status(6, None) == mimo.MIMO_ERR_INVALID_ARG
    assert mimo.lib.mimo_attn_set_device_status(-1, None) == mimo.MIMO_ERR_INVALID_ARG
    assert "status code" in mimo.lib.mimo_attn_last_error().decode()
