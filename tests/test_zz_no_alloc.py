"""gdn_check_step_noalloc: the slot-precondition check for callers that cannot allocate.

Some callers cannot hand the check a scratch buffer.  For example, a serving process
may have given all of its device memory to its own allocator, or a latency-critical
loop may forbid cudaMalloc/cudaFree because they can synchronise the device.  The
no-allocation entry point uses an owner map kept in the library's own device memory
instead.

These tests call it through the C ABI (ctypes on libgdn_b200.so).  Each call's verdict
must equal both the oracle's brute-force verdict and the verdict of gdn_check_step,
which is given a scratch buffer.  The verdict is an integer, so it must match exactly.  Calls come in consecutive pairs, so a second
call would see anything the first one left behind in the shared array.  The file sorts
last so that a run stopping at the first failure has already run every other test.  It
also passes when run on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch

    from hybrid_linear_attention_step_b200 import gdn

    lib = gdn.load_library()
    f = lib.gdn_check_step_noalloc
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_void_p, ctypes.c_void_p]
    return torch, gdn, f


def _noalloc(env, src, dst, num_slots, err):
    torch, gdn, f = env
    s = torch.from_numpy(src).cuda()
    d = torch.from_numpy(dst).cuda()
    status = f(s.data_ptr(), d.data_ptr(), src.shape[0], dst.shape[1], num_slots, err.data_ptr(),
               torch.cuda.current_stream().cuda_stream)
    assert status == gdn.GDN_OK
    return gdn.gdn_get_error(err)


def _with_scratch(env, src, dst, num_slots, err):
    torch, gdn, _ = env
    scratch = torch.empty(num_slots, dtype=torch.int32, device="cuda")
    gdn.gdn_check_step(torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda(), num_slots, scratch, err)
    return gdn.gdn_get_error(err)


def _mutate(src, dst, num_slots, kind):
    src, dst = src.copy(), dst.copy()
    if kind == "alias":
        dst[-1, -1] = src[0]            # a destination is another request's source
    elif kind == "dup":
        dst[0, 0] = dst[-1, -1]         # two writes to one slot
    elif kind == "range":
        dst[dst.shape[0] // 2, 0] = num_slots
    elif kind == "pad":
        src[0] = -1
        dst[0, :] = num_slots + 7       # ignored for a padding row
    return src, dst


def test_two_calls_in_a_row_match_the_scratch_entry_point(env):
    torch, gdn, _ = env
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(90)
    kinds = ["ok", "alias", "dup", "range", "pad"]
    verdicts = set()
    for trial in range(40):
        T = int(rng.integers(1, 4))
        B = int(rng.integers(2, 17))
        num_slots = int(rng.integers(B + 2 * B * T, 4096))
        perm = rng.permutation(num_slots).astype(np.int32)
        src1 = perm[:B].copy()
        dst1 = perm[B:B + B * T].reshape(B, T).copy()
        # Call 2 reads exactly the slots call 1 claimed (rolled by one request, so
        # each was claimed by a different request) and writes fresh ones.  It is
        # valid only if call 2 starts from a cleared owner map: any entry that call 1
        # left in the shared array would turn its verdict into GDN_ERR_ALIAS.
        src2 = np.roll(dst1[:, 0], 1).copy()
        dst2 = perm[B + B * T:B + 2 * B * T].reshape(B, T).copy()
        calls = [_mutate(src1, dst1, num_slots, kinds[trial % len(kinds)]), (src2, dst2)]
        for n, (src, dst) in enumerate(calls):
            want = oracle.check_step(src, dst, num_slots)
            assert _with_scratch(env, src, dst, num_slots, err) == want
            got = _noalloc(env, src, dst, num_slots, err)
            assert got == want, (trial, n, src.tolist(), dst.tolist(), got, want)
            if n == 1:
                assert got == gdn.GDN_OK
            verdicts.add(got)
    assert verdicts >= {gdn.GDN_OK, gdn.GDN_ERR_ALIAS, gdn.GDN_ERR_INDEX}


def test_largest_pool_and_beyond(env):
    torch, gdn, f = env
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    limit = 1 << 18  # GDN_CHECK_NOALLOC_MAX_SLOTS
    rng = np.random.default_rng(91)
    perm = rng.permutation(limit).astype(np.int32)
    src, dst = perm[:64].copy(), perm[64:192].reshape(64, 2).copy()
    src[1], dst[1, 0] = limit - 1, 0  # touch both ends of the array
    src[src == 0] = perm[200]
    dst[dst == limit - 1] = perm[201]
    for kind in ("ok", "alias"):
        s_, d_ = _mutate(src, dst, limit, kind)
        got = _noalloc(env, s_, d_, limit, err)
        assert got == _with_scratch(env, s_, d_, limit, err) == oracle.check_step(s_, d_, limit)
        assert got == (gdn.GDN_OK if kind == "ok" else gdn.GDN_ERR_ALIAS)
    src, dst = perm[:4].copy(), perm[4:8].reshape(4, 1).copy()
    s, d = torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda()
    status = f(s.data_ptr(), d.data_ptr(), 4, 1, limit + 1, err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert status == gdn.GDN_ERR_INVALID_ARG
    assert gdn.gdn_get_error(err) == gdn.GDN_OK  # nothing was enqueued
