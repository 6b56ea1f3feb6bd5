"""Thin ctypes binding of ``libgdn_b200.so`` (C ABI declared in include/gdn_step.h).

The functions here carry the C entry points' names and only marshal arguments:
torch CUDA tensors become device pointers, sizes are read off their shapes, and
the stream defaults to torch's current stream.  All compute runs in the CUDA
library; there is no fallback.  Loading fails loudly if the library is missing.
"""
from __future__ import annotations

import ctypes
import pathlib
from typing import Optional

import torch

LIB_PATH = pathlib.Path(__file__).resolve().parent / "libgdn_b200.so"

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_CUDA = 2
GDN_ERR_INDEX = 3
GDN_ERR_TIMEOUT = 4
GDN_ERR_ALIAS = 5

GDN_SLOT_NONE = -1

GDN_FUSE_GATES = 1
GDN_FUSE_QK_NORM = 2
GDN_SHARED_SOURCES = 4  # scheduling hint: many requests share source slots (same results)

GDN_F32 = 0
GDN_BF16 = 1

GDN_VARIANT_AUTO = 0
GDN_VARIANT_STREAM = 1
GDN_VARIANT_TILE = 2
GDN_VARIANT_COLUMN = 3
VARIANTS = {"auto": GDN_VARIANT_AUTO, "stream": GDN_VARIANT_STREAM, "tile": GDN_VARIANT_TILE,
            "column": GDN_VARIANT_COLUMN}

_DTYPES = {torch.float32: GDN_F32, torch.bfloat16: GDN_BF16}

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load_library() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"CUDA extension {LIB_PATH.name} is missing: run "
                           "`python -m hybrid_linear_attention_step_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(str(LIB_PATH))
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.gdn_decode_step.restype = i32
    lib.gdn_decode_step.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                    i32, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.gdn_decode_step_variant.restype = i32
    lib.gdn_decode_step_variant.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                            i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    lib.gdn_decode_step_fused.restype = i32
    lib.gdn_decode_step_fused.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                          i32, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.gdn_prefill.restype = i32
    lib.gdn_prefill.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.gdn_prefill_chunked.restype = i32
    lib.gdn_prefill_chunked.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                        vp, ctypes.c_size_t, vp, vp]
    lib.gdn_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_prefill_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.gdn_commit.restype = i32
    lib.gdn_commit.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp]
    lib.gdn_check_step.restype = i32
    lib.gdn_check_step.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
    lib.gdn_wait_selftest.restype = i32
    lib.gdn_wait_selftest.argtypes = [ctypes.c_uint64, vp, vp]
    lib.gdn_get_error.restype = i32
    lib.gdn_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), vp]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_status_string.argtypes = [i32]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().gdn_status_string(int(status)).decode()


def _stream_handle(stream, dev: Optional[int] = None) -> int:
    """The launch stream's handle: torch's current stream when ``stream`` is None.  With
    ``dev`` (the index of the call's tensors' device) the stream must belong to that
    device: the library launches on the calling thread's current device and takes the
    pointers as they are, so another device's buffers would be read from the wrong GPU.
    torch's current stream belongs to the current device; a raw handle is checked
    against the current device."""
    if stream is None:
        stream = torch.cuda.current_stream()
    if hasattr(stream, "cuda_stream"):
        if dev is not None and stream.device_index != dev:
            raise ValueError(f"the tensors are on cuda:{dev} but the launch stream is on cuda:{stream.device_index}"
                             f" (the current device, unless a stream was given); call inside torch.cuda.device({dev})")
        return int(stream.cuda_stream)
    if dev is not None and torch.cuda.current_device() != dev:
        raise ValueError(f"the tensors are on cuda:{dev} but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}; call inside torch.cuda.device({dev})")
    return int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _one_device(*tensors) -> int:
    """The CUDA device index of a call's tensors, which must all be on one device (the
    launch stream's: see _stream_handle)."""
    devs = {t.get_device() for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError("the tensors of one call must be on one CUDA device, got devices "
                         + ", ".join(str(d) for d in sorted(devs)))
    return devs.pop()


def _ptr_or_null(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    return None if t is None else _dev(t, name, torch.int32)


def _decode_args(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, dst_per_request=None, extra=(), stream=None):
    """Pointers and sizes for the decode and prefill entry points.  The library sees plain
    pointers, so every tensor's shape is checked against pool and q here: a mismatch
    would otherwise read or write past a buffer.  dst_idx holds dst_per_request entries
    per request (T by default; 1 for a prefill).  ``extra`` tensors of the call (error
    word, workspace) join the one-device check; returns the pointers and sizes, and the
    launch stream's handle."""
    if pool.dim() != 4 or q.dim() != 4 or v.dim() != 4:
        raise ValueError("pool, q, k, v must be 4-D")
    num_slots, Hv, dk, dv = pool.shape
    B, T, Hk = q.shape[0], q.shape[1], q.shape[2]
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype: bfloat16 or float32")
    want = {"q": (B, T, Hk, dk), "k": (B, T, Hk, dk), "v": (B, T, Hv, dv), "alpha": (B, T, Hv),
            "beta": (B, T, Hv), "out": (B, T, Hv, dv)}
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta), ("out", out)):
        if tuple(t.shape) != want[name]:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want[name]} from pool {tuple(pool.shape)}"
                             f" and q {tuple(q.shape)}")
    per = T if dst_per_request is None else dst_per_request
    if src_idx.numel() != B or dst_idx.numel() != B * per:
        raise ValueError(f"src_idx must hold B = {B} entries and dst_idx B * {per}")
    args = (_dev(pool, "pool", torch.float32), int(num_slots),
            _dev(src_idx, "src_idx", torch.int32), _dev(dst_idx, "dst_idx", torch.int32),
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
            _dev(alpha, "alpha", torch.float32), _dev(beta, "beta", torch.float32),
            _dev(out, "out", torch.float32),
            int(B), int(T), int(Hk), int(Hv), int(dk), int(dv), _DTYPES[q.dtype])
    return args, _stream_handle(stream, _one_device(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, *extra))


def gdn_decode_step(pool: torch.Tensor, src_idx: torch.Tensor, dst_idx: torch.Tensor,
                    q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor,
                    err_word: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """Enqueue one GDN decode step (see gdn_decode_step in include/gdn_step.h).

    pool [num_slots, Hv, dk, dv] fp32; src_idx [B] int32; dst_idx [B, T] (or [B]) int32;
    q, k [B, T, Hk, dk] and v [B, T, Hv, dv] bf16 or fp32; alpha, beta [B, T, Hv] fp32;
    out [B, T, Hv, dv] fp32.  Returns the status; raises GdnError on failure when ``check``.
    """
    args, sh = _decode_args(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, extra=(err_word,), stream=stream)
    status = load_library().gdn_decode_step(*args, _ptr_or_null(err_word, "err_word"), sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_decode_step")
    return status


class PreparedDecodeStep:
    """gdn_decode_step on buffers checked once: for a serving loop that reuses the same
    tensors every step (as a CUDA graph does), each call then only passes the pointers.

    The tensors must stay alive and keep their storage while the object is used; their
    contents may change between calls (new inputs, indices, gates).  ``variant`` is None
    for the automatic kernel choice or a GDN_VARIANT_* value or name (then the call is
    gdn_decode_step_variant); nonzero ``flags`` (GDN_FUSE_*, GDN_SHARED_SOURCES) make it
    gdn_decode_step_fused, with the automatic choice.  A ``stream`` given here is used by
    every call that names none (looking up torch's current stream costs about as much host
    time as the launch); without one, each call enqueues on the current stream, which is
    what stream capture into a CUDA graph needs.
    """

    def __init__(self, pool: torch.Tensor, src_idx: torch.Tensor, dst_idx: torch.Tensor,
                 q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor,
                 err_word: Optional[torch.Tensor] = None, variant=None, stream=None, flags: int = 0):
        lib = load_library()
        args, sh = _decode_args(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, extra=(err_word,), stream=stream)
        err = _ptr_or_null(err_word, "err_word")
        self._device = pool.get_device()
        if flags and variant is not None:
            raise ValueError("flags go with the automatic kernel choice: pass variant=None")
        if flags:
            self._fn, self._name = lib.gdn_decode_step_fused, "gdn_decode_step_fused"
            args = args + (int(flags), err)
        elif variant is None:
            self._fn, self._name = lib.gdn_decode_step, "gdn_decode_step"
            args = args + (err,)
        else:
            if isinstance(variant, str):
                variant = VARIANTS[variant]
            self._fn, self._name = lib.gdn_decode_step_variant, "gdn_decode_step_variant"
            args = args + (err, int(variant))
        self._args = args
        self._stream = None if stream is None else sh
        self._keep = (pool, src_idx, dst_idx, q, k, v, alpha, beta, out, err_word, stream)

    def __call__(self, stream=None, check: bool = True) -> int:
        if stream is None and self._stream is not None:
            handle = self._stream  # a stream of the buffers' device, checked once
        else:
            handle = _stream_handle(stream, self._device)
        status = self._fn(*self._args, handle)
        if check and status != GDN_OK:
            raise GdnError(status, self._name)
        return status


def gdn_decode_step_variant(pool: torch.Tensor, src_idx: torch.Tensor, dst_idx: torch.Tensor,
                            q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor, variant,
                            err_word: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """gdn_decode_step with an explicit kernel: ``variant`` is a GDN_VARIANT_* value or a name
    ("auto", "stream", "tile", "column")."""
    if isinstance(variant, str):
        variant = VARIANTS[variant]
    args, sh = _decode_args(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, extra=(err_word,), stream=stream)
    status = load_library().gdn_decode_step_variant(*args, _ptr_or_null(err_word, "err_word"), int(variant), sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_decode_step_variant")
    return status


def gdn_decode_step_fused(pool: torch.Tensor, src_idx: torch.Tensor, dst_idx: torch.Tensor,
                          q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          alpha_or_x: torch.Tensor, beta_or_y: torch.Tensor, out: torch.Tensor, flags: int,
                          err_word: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """gdn_decode_step with the input prologue folded in (see gdn_decode_step_fused in
    include/gdn_step.h): GDN_FUSE_GATES makes alpha_or_x / beta_or_y the raw x, y;
    GDN_FUSE_QK_NORM L2-normalises q and k inside the kernel; GDN_SHARED_SOURCES tells the
    kernels that many requests share source slots (an ordering hint, same results)."""
    args, sh = _decode_args(pool, src_idx, dst_idx, q, k, v, alpha_or_x, beta_or_y, out, extra=(err_word,),
                            stream=stream)
    status = load_library().gdn_decode_step_fused(*args, int(flags), _ptr_or_null(err_word, "err_word"), sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_decode_step_fused")
    return status


def gdn_prefill(pool: torch.Tensor, src_idx: torch.Tensor, dst_idx: torch.Tensor,
                q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor,
                err_word: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """Enqueue a prefill (see gdn_prefill in include/gdn_step.h): q, k [B, L, Hk, dk],
    v [B, L, Hv, dv], alpha/beta [B, L, Hv], out [B, L, Hv, dv]; only the state after the
    last token is stored, to pool[dst_idx[b]] (dst_idx [B])."""
    args, sh = _decode_args(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, dst_per_request=1,
                            extra=(err_word,), stream=stream)
    status = load_library().gdn_prefill(*args, _ptr_or_null(err_word, "err_word"), sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_prefill")
    return status


def gdn_prefill_workspace_bytes(B: int, L: int, Hv: int, dk: int, dv: int) -> int:
    return int(load_library().gdn_prefill_workspace_bytes(int(B), int(L), int(Hv), int(dk), int(dv)))


def gdn_prefill_chunked(pool: torch.Tensor, src_idx: torch.Tensor, dst_idx: torch.Tensor,
                        q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                        err_word: torch.Tensor, stream=None, check: bool = True) -> int:
    """gdn_prefill computed chunk by chunk (see gdn_prefill_chunked in include/gdn_step.h);
    ``workspace`` is a CUDA tensor of at least gdn_prefill_workspace_bytes(...) bytes.
    ``err_word`` (int32 CUDA tensor) is required: a copy or tensor-core wait that runs out is
    reported only there."""
    wp, ep = _dev(workspace, "workspace"), _dev(err_word, "err_word", torch.int32)
    args, sh = _decode_args(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, dst_per_request=1,
                            extra=(err_word, workspace), stream=stream)
    nbytes = workspace.numel() * workspace.element_size()
    status = load_library().gdn_prefill_chunked(*args, wp, nbytes, ep, sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_prefill_chunked")
    return status


def gdn_commit(accept_len: torch.Tensor, committed: torch.Tensor, cur: torch.Tensor, num_slots: int,
               err_word: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> int:
    """Enqueue the accept-length commit (see gdn_commit in include/gdn_step.h).

    accept_len [B] int32; committed [B] int32 (updated in place); cur [B, T] int32.
    """
    if cur.dim() != 2:
        raise ValueError("cur must be [B, T]")
    B, T = cur.shape
    if accept_len.numel() != B or committed.numel() != B:
        raise ValueError("accept_len and committed must hold B entries")
    ptrs = (_dev(accept_len, "accept_len", torch.int32), _dev(committed, "committed", torch.int32),
            _dev(cur, "cur", torch.int32))
    err = _ptr_or_null(err_word, "err_word")
    sh = _stream_handle(stream, _one_device(accept_len, committed, cur, err_word))
    status = load_library().gdn_commit(*ptrs, int(B), int(T), int(num_slots), err, sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_commit")
    return status


def gdn_check_step(src_idx: torch.Tensor, dst_idx: torch.Tensor, num_slots: int, scratch: torch.Tensor,
                   err_word: torch.Tensor, stream=None, check: bool = True) -> int:
    """Enqueue the device-side precondition check of a decode call's slot indices
    (see gdn_check_step in include/gdn_step.h).  scratch: int32 [>= num_slots]."""
    B = src_idx.shape[0]
    T = dst_idx.shape[1] if dst_idx.dim() == 2 else 1
    if dst_idx.numel() != B * T:
        raise ValueError("dst_idx must hold B*T entries")
    if scratch.numel() < num_slots:
        raise ValueError("scratch must hold num_slots int32 entries")
    ptrs = (_dev(src_idx, "src_idx", torch.int32), _dev(dst_idx, "dst_idx", torch.int32))
    sp, ep = _dev(scratch, "scratch", torch.int32), _dev(err_word, "err_word", torch.int32)
    sh = _stream_handle(stream, _one_device(src_idx, dst_idx, scratch, err_word))
    status = load_library().gdn_check_step(*ptrs, int(B), int(T), int(num_slots), sp, ep, sh)
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_check_step")
    return status


def gdn_wait_selftest(limit_ns: int, err_word: torch.Tensor, stream=None, check: bool = True) -> int:
    """Enqueue the bounded-wait self-test (see gdn_wait_selftest in include/gdn_step.h):
    a wait on an mbarrier nothing arrives on, which records GDN_ERR_TIMEOUT after limit_ns."""
    ep = _dev(err_word, "err_word", torch.int32)
    status = load_library().gdn_wait_selftest(int(limit_ns), ep, _stream_handle(stream, _one_device(err_word)))
    if check and status != GDN_OK:
        raise GdnError(status, "gdn_wait_selftest")
    return status


def gdn_get_error(err_word: torch.Tensor, stream=None) -> int:
    """Synchronise the stream, return the device error word's status code and clear it."""
    code = ctypes.c_int32(-1)
    ep = _dev(err_word, "err_word", torch.int32)
    status = load_library().gdn_get_error(ep, ctypes.byref(code), _stream_handle(stream, _one_device(err_word)))
    if status != GDN_OK:
        raise GdnError(status, "gdn_get_error")
    return int(code.value)
