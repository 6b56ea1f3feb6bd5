"""CPU oracle for the decode-time Gated DeltaNet state update -- TEST INFRASTRUCTURE.

This package is the independent checker, not the product.  Only the test
suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline and
reference legs may import it.  It shares no code with the CUDA library: the
arithmetic lives in ``gdn_oracle.cpp`` (plain loops in double, built with g++),
and this module only marshals numpy arrays into it.

Every function here that computes follows the gated delta rule of Gated
DeltaNet (Yang, Kautz & Hatamizadeh, ICLR 2025) as named by the TokenSpeed
580 tok/s article (24-ai.news, English edition) and its slot semantics
("Mamba State Update optimization" and "Hybrid prefix caching for GDN/Mamba"
items of "What are the key optimizations behind the record?"; zubnet.ai
LightSeek TokenSpeed article, second paragraph).  The C++ source states the
readings taken where the pages are silent.

Pinning: every part of the oracle is pinned by tests that do not re-use its
formula (tests/test_oracle_pins.py): closed forms (identity, reset, delta-rule
retrieval, pure write, decay), a hand-derived 2x2 worked example, an
independent rank-one restatement on tiny shapes, copy-on-write byte identity,
sequential == speculative, slot relabelling, the grouped key-head map and
brute-force commit.
"""
from __future__ import annotations

import ctypes
import os
import pathlib
import subprocess

import numpy as np

_HERE = pathlib.Path(__file__).resolve().parent
SOURCE = _HERE / "gdn_oracle.cpp"
LIB_PATH = _HERE / "libgdn_oracle.so"

F32 = 0
BF16 = 1

_lib = None


def build(force: bool = False) -> pathlib.Path:
    """Compile the oracle with g++ (plain -O2, no FMA contraction)."""
    if not force and LIB_PATH.exists() and LIB_PATH.stat().st_mtime >= SOURCE.stat().st_mtime:
        return LIB_PATH
    tmp = LIB_PATH.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
           "-o", str(tmp), str(SOURCE)]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # GDN_ORACLE_LIB lets the mutation test load a deliberately broken build.
        override = os.environ.get("GDN_ORACLE_LIB")
        if override:
            path = override
        else:
            path = str(build())
        lib = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        lib.oracle_gdn_decode_step.restype = i64
        lib.oracle_gdn_decode_step.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp, vp,
                                               i64, i64, i64, i64, i64, i64, i32, i32]
        lib.oracle_gdn_decode_step_fused.restype = i64
        lib.oracle_gdn_decode_step_fused.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp, vp,
                                                     i64, i64, i64, i64, i64, i64, i32, i32, i32]
        lib.oracle_gdn_prefill.restype = i64
        lib.oracle_gdn_prefill.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp, vp,
                                           i64, i64, i64, i64, i64, i64, i32, i32]
        lib.oracle_gdn_check_step.restype = i32
        lib.oracle_gdn_check_step.argtypes = [vp, vp, i64, i64, i64]
        lib.oracle_gdn_commit.restype = i64
        lib.oracle_gdn_commit.argtypes = [vp, vp, vp, i64, i64, i64]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _need(a: np.ndarray, dtype, name: str) -> None:
    if not isinstance(a, np.ndarray) or a.dtype != dtype or not a.flags.c_contiguous:
        raise TypeError(f"{name} must be a C-contiguous numpy array of {np.dtype(dtype)}")


FUSE_GATES = 1
FUSE_QK_NORM = 2


def decode_step(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, *, nthreads: int = 1, flags: int = 0) -> int:
    """One decode call on host arrays; ``pool`` and ``out`` are updated in place.

    pool  [num_slots, Hv, dk, dv] float32
    src_idx [B] int32, dst_idx [B, T] (or [B] for T = 1) int32
    q, k  [B, T, Hk, dk] and v [B, T, Hv, dv]: float32, or uint16 bfloat16 bit patterns
    alpha, beta [B, T, Hv] float32 (raw x, y when flags & FUSE_GATES); out [B, T, Hv, dv] float32
    flags: FUSE_GATES (alpha = exp(-softplus(x)), beta = sigmoid(y)) | FUSE_QK_NORM
    Returns the number of requests skipped for an out-of-range index.
    """
    _need(pool, np.float32, "pool")
    num_slots, Hv, dk, dv = pool.shape
    _need(src_idx, np.int32, "src_idx")
    B = src_idx.shape[0]
    _need(dst_idx, np.int32, "dst_idx")
    T = dst_idx.shape[1] if dst_idx.ndim == 2 else 1
    if dst_idx.size != B * T:
        raise ValueError("dst_idx must hold B*T entries")
    if q.dtype == np.uint16:
        dtype = BF16
    elif q.dtype == np.float32:
        dtype = F32
    else:
        raise TypeError("q/k/v must be float32 or uint16 (bfloat16 bits)")
    for name, a in (("q", q), ("k", k), ("v", v)):
        _need(a, q.dtype, name)
    Hk = q.shape[-2]
    if q.shape != (B, T, Hk, dk) or k.shape != q.shape:
        raise ValueError(f"q/k must be [B, T, Hk, dk] = [{B}, {T}, Hk, {dk}], got {q.shape}, {k.shape}")
    if v.shape != (B, T, Hv, dv):
        raise ValueError("v must be [B, T, Hv, dv]")
    for name, a in (("alpha", alpha), ("beta", beta)):
        _need(a, np.float32, name)
        if a.shape != (B, T, Hv):
            raise ValueError(f"{name} must be [B, T, Hv]")
    _need(out, np.float32, "out")
    if out.shape != (B, T, Hv, dv):
        raise ValueError("out must be [B, T, Hv, dv]")
    if flags:
        r = _load().oracle_gdn_decode_step_fused(
            _ptr(pool), num_slots, _ptr(src_idx), _ptr(dst_idx), _ptr(q), _ptr(k), _ptr(v),
            _ptr(alpha), _ptr(beta), _ptr(out), B, T, Hk, Hv, dk, dv, dtype, int(flags), int(nthreads))
    else:
        r = _load().oracle_gdn_decode_step(
            _ptr(pool), num_slots, _ptr(src_idx), _ptr(dst_idx), _ptr(q), _ptr(k), _ptr(v),
            _ptr(alpha), _ptr(beta), _ptr(out), B, T, Hk, Hv, dk, dv, dtype, int(nthreads))
    if r < 0:
        raise ValueError("oracle rejected the sizes")
    return int(r)


def commit(accept_len, committed, cur, num_slots: int) -> int:
    """Accept-length commit on host arrays; ``committed`` [B] is updated in place.

    cur [B, T] int32 holds the per-draft-token slots; accept_len [B] int32.
    Returns the number of requests skipped for an out-of-range length or slot.
    """
    _need(accept_len, np.int32, "accept_len")
    _need(committed, np.int32, "committed")
    _need(cur, np.int32, "cur")
    B = accept_len.shape[0]
    T = cur.shape[1]
    if committed.shape != (B,) or cur.shape != (B, T):
        raise ValueError("committed must be [B] and cur [B, T]")
    r = _load().oracle_gdn_commit(_ptr(accept_len), _ptr(committed), _ptr(cur), B, T, int(num_slots))
    if r < 0:
        raise ValueError("oracle rejected the sizes")
    return int(r)


def check_step(src_idx, dst_idx, num_slots: int) -> int:
    """Precondition check of one call's slot indices: 0 ok, 3 index out of range,
    5 aliasing slots (see oracle_gdn_check_step)."""
    _need(src_idx, np.int32, "src_idx")
    _need(dst_idx, np.int32, "dst_idx")
    B = src_idx.shape[0]
    T = dst_idx.shape[1] if dst_idx.ndim == 2 else 1
    if dst_idx.size != B * T:
        raise ValueError("dst_idx must hold B*T entries")
    r = _load().oracle_gdn_check_step(_ptr(src_idx), _ptr(dst_idx), B, T, int(num_slots))
    if r < 0:
        raise ValueError("oracle rejected the sizes")
    return int(r)


def prefill(pool, src_idx, dst_idx, q, k, v, alpha, beta, out, *, nthreads: int = 1) -> int:
    """Prefill on host arrays: L tokens per request (q [B, L, Hk, dk] ...), only the final
    state stored, to dst_idx[b] (dst_idx [B]); ``out`` [B, L, Hv, dv] gets every token."""
    _need(pool, np.float32, "pool")
    num_slots, Hv, dk, dv = pool.shape
    _need(src_idx, np.int32, "src_idx")
    _need(dst_idx, np.int32, "dst_idx")
    B, L, Hk = q.shape[0], q.shape[1], q.shape[2]
    if src_idx.shape != (B,) or dst_idx.size != B:
        raise ValueError("src_idx and dst_idx must hold B entries")
    dtype = BF16 if q.dtype == np.uint16 else F32
    for name, a in (("q", q), ("k", k), ("v", v)):
        _need(a, q.dtype, name)
    for name, a in (("alpha", alpha), ("beta", beta), ("out", out)):
        _need(a, np.float32, name)
    if k.shape != (B, L, Hk, dk) or v.shape != (B, L, Hv, dv) or alpha.shape != (B, L, Hv) or \
            beta.shape != (B, L, Hv) or out.shape != (B, L, Hv, dv):
        raise ValueError("shapes must follow q [B, L, Hk, dk]")
    r = _load().oracle_gdn_prefill(_ptr(pool), num_slots, _ptr(src_idx), _ptr(dst_idx), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(alpha), _ptr(beta), _ptr(out), B, L, Hk, Hv, dk, dv, dtype, int(nthreads))
    if r < 0:
        raise ValueError("oracle rejected the sizes")
    return int(r)
