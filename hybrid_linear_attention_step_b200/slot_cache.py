"""ctypes binding of the host slot allocator / prefix cache (include/gdn_slot_cache.h).

``SlotCache`` wraps one ``gdn_slot_cache`` handle; its methods carry the C entry points'
names without the ``gdn_slot_cache_`` prefix and only marshal numpy arrays.  All logic
is in the native library; there is no Python fallback.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import numpy as np

from . import gdn

_configured = False


def _lib():
    global _configured
    lib = gdn.load_library()
    if not _configured:
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        P = ctypes.POINTER
        lib.gdn_slot_cache_create.restype = i32
        lib.gdn_slot_cache_create.argtypes = [i32, P(vp)]
        lib.gdn_slot_cache_destroy.restype = None
        lib.gdn_slot_cache_destroy.argtypes = [vp]
        lib.gdn_slot_cache_open.restype = i32
        lib.gdn_slot_cache_open.argtypes = [vp, vp, i64, P(i32), P(i32), P(i64), P(i32)]
        lib.gdn_slot_cache_plan.restype = i32
        lib.gdn_slot_cache_plan.argtypes = [vp, vp, i32, i32, vp, vp]
        lib.gdn_slot_cache_commit.restype = i32
        lib.gdn_slot_cache_commit.argtypes = [vp, vp, i32, i32, vp, vp]
        lib.gdn_slot_cache_checkpoint.restype = i32
        lib.gdn_slot_cache_checkpoint.argtypes = [vp, i32, vp, i64, P(i32)]
        lib.gdn_slot_cache_close.restype = i32
        lib.gdn_slot_cache_close.argtypes = [vp, i32]
        lib.gdn_slot_cache_evict.restype = i32
        lib.gdn_slot_cache_evict.argtypes = [vp, i32, P(i32)]
        lib.gdn_slot_cache_stats.restype = i32
        lib.gdn_slot_cache_stats.argtypes = [vp, P(i32), P(i32), P(i32)]
        lib.gdn_slot_cache_refcount.restype = i32
        lib.gdn_slot_cache_refcount.argtypes = [vp, i32]
        _configured = True
    return lib


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class SlotCacheError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {gdn.status_string(status)} ({status})")


def _check(status: int, where: str) -> None:
    if status != gdn.GDN_OK:
        raise SlotCacheError(status, where)


class SlotCache:
    """Slots, checkpoints and requests of one GDN layer's slot pool (see gdn_slot_cache.h)."""

    def __init__(self, num_slots: int):
        self._h = ctypes.c_void_p()
        _check(_lib().gdn_slot_cache_create(int(num_slots), ctypes.byref(self._h)), "gdn_slot_cache_create")
        self.num_slots = int(num_slots)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            try:
                _lib().gdn_slot_cache_destroy(h)
            except TypeError:  # interpreter shutdown: the module's globals are already gone
                return
            self._h = None

    def open(self, tokens) -> Tuple[int, int, int, bool]:
        """Returns (request id, slot, matched prefix length, needs_init)."""
        t = _i32(tokens)
        req, slot, needs = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        matched = ctypes.c_int64()
        _check(_lib().gdn_slot_cache_open(self._h, _ptr(t) if t.size else None, t.size, ctypes.byref(req),
                                          ctypes.byref(slot), ctypes.byref(matched), ctypes.byref(needs)),
               "gdn_slot_cache_open")
        return req.value, slot.value, matched.value, bool(needs.value)

    def plan(self, reqs, T: int = 1) -> Tuple[np.ndarray, np.ndarray]:
        """Returns (src_idx [B], dst_idx [B, T]) for one decode call."""
        r = _i32(reqs)
        src = np.empty(r.size, np.int32)
        dst = np.empty((r.size, T), np.int32)
        _check(_lib().gdn_slot_cache_plan(self._h, _ptr(r), r.size, int(T), _ptr(src), _ptr(dst)),
               "gdn_slot_cache_plan")
        return src, dst

    def commit(self, reqs, T: int = 1, accept_len=None) -> np.ndarray:
        """Applies the planned call's outcome; returns each request's new state slot."""
        r = _i32(reqs)
        acc = None if accept_len is None else _i32(accept_len)
        out = np.empty(r.size, np.int32)
        _check(_lib().gdn_slot_cache_commit(self._h, _ptr(r), r.size, int(T), _ptr(acc), _ptr(out)),
               "gdn_slot_cache_commit")
        return out

    def checkpoint(self, req: int, tokens) -> int:
        t = _i32(tokens)
        slot = ctypes.c_int32()
        _check(_lib().gdn_slot_cache_checkpoint(self._h, int(req), _ptr(t), t.size, ctypes.byref(slot)),
               "gdn_slot_cache_checkpoint")
        return slot.value

    def close(self, req: int) -> None:
        _check(_lib().gdn_slot_cache_close(self._h, int(req)), "gdn_slot_cache_close")

    def evict(self, want_free: int) -> int:
        n = ctypes.c_int32()
        _check(_lib().gdn_slot_cache_evict(self._h, int(want_free), ctypes.byref(n)), "gdn_slot_cache_evict")
        return n.value

    def stats(self) -> Tuple[int, int, int]:
        """(free slots, checkpoints, open requests)"""
        a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(_lib().gdn_slot_cache_stats(self._h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
               "gdn_slot_cache_stats")
        return a.value, b.value, c.value

    def refcount(self, slot: int) -> int:
        return int(_lib().gdn_slot_cache_refcount(self._h, int(slot)))
