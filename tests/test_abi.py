"""The C-ABI library builds, loads without a GPU, exports every declared entry point,
and rejects bad arguments on the host before touching CUDA."""
import ctypes
import pathlib
import re

import pytest

ROOT = pathlib.Path(__file__).resolve().parent.parent


@pytest.fixture(scope="module")
def lib():
    from hybrid_linear_attention_step_b200 import build

    path = build.build()
    return ctypes.CDLL(str(path))


def declared_functions():
    names = []
    for h in sorted((ROOT / "include").glob("*.h")):
        text = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names += re.findall(r"^\s*(?:gdn_status|const\s+char\s*\*|void|int32_t|size_t)\s*(gdn_\w+)\s*\(", text,
                            flags=re.M)
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdn_decode_step", "gdn_commit", "gdn_get_error", "gdn_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_status_string.argtypes = [ctypes.c_int32]
    assert [lib.gdn_status_string(i).decode() for i in range(7)] == [
        "GDN_OK", "GDN_ERR_INVALID_ARG", "GDN_ERR_CUDA", "GDN_ERR_INDEX", "GDN_ERR_TIMEOUT", "GDN_ERR_ALIAS",
        "GDN_ERR_CAPACITY"]
    assert lib.gdn_status_string(99).decode() == "GDN_UNKNOWN_STATUS"


def _decode(lib, **kw):
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    f = lib.gdn_decode_step
    f.restype = i32
    f.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    a = dict(pool=8, num_slots=4, src=8, dst=8, q=8, k=8, v=8, alpha=8, beta=8, out=8,
             B=1, T=1, Hk=1, Hv=1, dk=16, dv=16, dtype=1, err=None, stream=None)
    a.update(kw)
    return f(*a.values())


def test_host_validation_before_any_cuda_call(lib):
    # Each of these must be rejected on the host (no device is present here).
    assert _decode(lib, B=-1) == 1
    assert _decode(lib, T=0) == 1
    assert _decode(lib, Hk=3, Hv=4) == 1
    assert _decode(lib, dk=5000) == 1
    assert _decode(lib, dtype=7) == 1
    assert _decode(lib, num_slots=0) == 1
    assert _decode(lib, pool=None) == 1
    assert _decode(lib, out=None) == 1
    assert _decode(lib, B=0, pool=None, src=None, dst=None) == 0  # empty batch: no-op
    f = lib.gdn_commit
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int32] * 3 + [ctypes.c_void_p] * 2
    assert f(8, 8, 8, -1, 1, 4, None, None) == 1
    assert f(8, 8, 8, 1, 0, 4, None, None) == 1
    assert f(None, 8, 8, 1, 1, 4, None, None) == 1
    assert f(None, None, None, 0, 1, 4, None, None) == 0
    h = lib.gdn_check_step
    h.restype = ctypes.c_int32
    h.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int32] * 3 + [ctypes.c_void_p] * 3
    assert h(8, 8, -1, 1, 4, 8, 8, None) == 1
    assert h(8, 8, 1, 1, 4, None, 8, None) == 1   # scratch required
    assert h(8, 8, 1, 1, 4, 8, None, None) == 1   # err_word required
    assert h(None, None, 0, 1, 4, None, None, None) == 0
    g = lib.gdn_get_error
    g.restype = ctypes.c_int32
    g.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert g(None, None, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    pytest.importorskip("torch")
    from hybrid_linear_attention_step_b200 import gdn

    monkeypatch.setattr(gdn, "LIB_PATH", tmp_path / "missing.so")
    monkeypatch.setattr(gdn, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        gdn.load_library()


def test_product_path_never_imports_the_oracle():
    pkg = ROOT / "hybrid_linear_attention_step_b200"
    for p in list(pkg.rglob("*.py")) + list(pkg.rglob("*.cu")) + list((ROOT / "include").glob("*.h")):
        text = p.read_text()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), p
        assert "gdn_oracle" not in text, p


def test_wait_selftest_validates_on_the_host(lib):
    f = lib.gdn_wait_selftest
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    assert f(1000, None, None) == 1          # no error word
    assert f(0, 8, None) == 1                # empty limit
    assert f(2_000_000_001, 8, None) == 1    # above the pipelines' own limit


def _prefill_chunked(lib, **kw):
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    f = lib.gdn_prefill_chunked
    f.restype = i32
    f.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, ctypes.c_size_t,
                  vp, vp]
    a = dict(pool=16, num_slots=4, src=16, dst=16, q=16, k=16, v=16, alpha=16, beta=16, out=16,
             B=1, L=100, Hk=1, Hv=2, dk=128, dv=128, dtype=1, ws=16, ws_bytes=1 << 30, err=16, stream=None)
    a.update(kw)
    return f(*a.values())


def test_prefill_workspace_size(lib):
    w = lib.gdn_prefill_workspace_bytes
    w.restype = ctypes.c_size_t
    w.argtypes = [ctypes.c_int32] * 5
    one = w(1, 1, 1, 128, 128)
    assert one > 0 and one % 16 == 0
    assert w(1, 64, 1, 128, 128) == one          # one chunk holds 64 tokens
    assert w(1, 65, 1, 128, 128) == 2 * one      # a ragged tail takes a chunk of its own
    assert w(3, 130, 5, 128, 128) == 3 * 5 * 3 * one
    assert w(1, 64, 1, 64, 64) == 0              # shapes the chunked path does not support
    assert w(1, 0, 1, 128, 128) == 0


def test_prefill_chunked_validates_on_the_host(lib):
    lib.gdn_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_prefill_workspace_bytes.argtypes = [ctypes.c_int32] * 5
    need = lib.gdn_prefill_workspace_bytes(1, 100, 2, 128, 128)
    assert _prefill_chunked(lib, dk=64, dv=64) == 1                  # unsupported head size
    assert _prefill_chunked(lib, Hk=3, Hv=4) == 1                    # Hv not a multiple of Hk
    assert _prefill_chunked(lib, L=0) == 1
    assert _prefill_chunked(lib, dtype=5) == 1
    assert _prefill_chunked(lib, ws=None) == 1                       # no workspace
    assert _prefill_chunked(lib, ws_bytes=need - 16) == 1            # short workspace
    assert _prefill_chunked(lib, ws=24, ws_bytes=need) == 1          # workspace not 16-byte aligned
    assert _prefill_chunked(lib, out=20, ws_bytes=need) == 1         # out not 16-byte aligned
    assert _prefill_chunked(lib, err=None, ws_bytes=need) == 1       # the error word is required
    assert _prefill_chunked(lib, B=0, pool=None, ws=None) == 0       # empty batch: no-op


def test_prefill_validates_on_the_host(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    f = lib.gdn_prefill
    f.restype = i32
    f.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    a = dict(pool=16, num_slots=4, src=16, dst=16, q=16, k=16, v=16, alpha=16, beta=16, out=16,
             B=1, L=10, Hk=1, Hv=2, dk=128, dv=128, dtype=1, err=None, stream=None)
    call = lambda **kw: f(*{**a, **kw}.values())
    assert call(L=0) == 1
    assert call(Hk=2, Hv=3) == 1
    assert call(dtype=9) == 1
    assert call(src=None) == 1
    assert call(B=0, pool=None) == 0  # empty batch: no-op


def test_stream_variant_requires_the_error_word(lib):
    """The bulk-copy decode kernel reports a timed-out copy only through the error word, so
    the call is refused without one (checked on the host, before any CUDA call)."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    f = lib.gdn_decode_step_variant
    f.restype = i32
    f.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    args = [16, 8, 16, 16, 16, 16, 16, 16, 16, 16, 4, 1, 1, 1, 128, 128, 1]
    assert f(*args, None, 1, None) == 1      # GDN_VARIANT_STREAM, no error word
    assert f(*args, None, 9, None) == 1      # no such variant


def test_prepared_decode_step_checks_its_buffers_once():
    """The prepared decode call validates shapes and devices when it is made (no GPU needed:
    the checks come before any call into the library)."""
    import torch

    from hybrid_linear_attention_step_b200 import gdn

    B, T, Hk, Hv, d = 2, 1, 1, 2, 128
    pool = torch.zeros((4, Hv, d, d))
    q = torch.zeros((B, T, Hk, d), dtype=torch.bfloat16)
    v = torch.zeros((B, T, Hv, d), dtype=torch.bfloat16)
    gates = torch.zeros((B, T, Hv))
    idx = torch.zeros(B, dtype=torch.int32)
    out = torch.zeros((B, T, Hv, d))
    with pytest.raises(ValueError):
        gdn.PreparedDecodeStep(pool, idx, idx, q, q, v, gates, gates, torch.zeros((B, T, Hv, d + 1)))
    with pytest.raises(TypeError):
        gdn.PreparedDecodeStep(pool, idx, idx, q, q, v, gates, gates, out)  # host tensors


def test_fused_flags_are_checked_on_the_host(lib):
    """gdn_decode_step_fused accepts GDN_FUSE_GATES, GDN_FUSE_QK_NORM and the
    GDN_SHARED_SOURCES hint, and refuses any other bit before doing anything."""
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    f = lib.gdn_decode_step_fused
    f.restype = i32
    f.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    args = [16, 8, 16, 16, 16, 16, 16, 16, 16, 16, 0, 1, 1, 1, 128, 128, 1]  # B = 0: a no-op when valid
    for flags in (0, 1, 2, 3, 4, 5, 7):
        assert f(*args, flags, None, None) == 0, flags
    for flags in (8, 16, 12, -1):
        assert f(*args, flags, None, None) == 1, flags


def test_calls_take_tensors_of_one_device_the_current_one(monkeypatch):
    """The binding refuses, before any launch, a call whose tensors sit on more than one
    device, or whose launch stream (torch's current one, a given torch stream, or for a
    raw handle the current device) belongs to another device: the library would launch
    there with another GPU's pointers."""
    import types

    import torch

    from hybrid_linear_attention_step_b200 import gdn

    on = lambda i: types.SimpleNamespace(get_device=lambda: i)
    assert gdn._one_device(on(0), on(0), None) == 0
    assert gdn._one_device(on(1), on(1)) == 1
    with pytest.raises(ValueError, match="one CUDA device"):
        gdn._one_device(on(0), on(1))
    stream = lambda i: types.SimpleNamespace(cuda_stream=1000 + i, device_index=i)
    assert gdn._stream_handle(stream(1), 1) == 1001
    with pytest.raises(ValueError, match="launch stream is on cuda:0"):
        gdn._stream_handle(stream(0), 1)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda: stream(0))
    assert gdn._stream_handle(None, 0) == 1000
    with pytest.raises(ValueError, match="launch stream is on cuda:0"):
        gdn._stream_handle(None, 1)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    assert gdn._stream_handle(12345, 0) == 12345  # a raw handle: checked against the current device
    with pytest.raises(ValueError, match="current CUDA device is cuda:0"):
        gdn._stream_handle(12345, 1)
