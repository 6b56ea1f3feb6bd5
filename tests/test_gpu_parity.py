"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded bytes.

Bit-exact: which slots are written, untouched slots' bytes, committed index
tables, error reporting.  Within tolerance: fp32 states (1e-4) and outputs
(2e-3 with bf16 inputs, 1e-4 with fp32 inputs), as max relative error with the
reference RMS as floor.
"""
import zlib

import numpy as np
import pytest

from hybrid_linear_attention_step_b200 import workloads as wl
from tests.gpu_helpers import (TOL_OUT_BF16, TOL_OUT_F32, TOL_STATE, check_pool, rel_err, run_gpu, run_oracle,
                               step_to_device, to_torch)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    from hybrid_linear_attention_step_b200 import gdn

    gdn.load_library()
    return torch


def _tol_out(s):
    return TOL_OUT_BF16 if s.dtype == wl.BF16 else TOL_OUT_F32


def test_tiny_chain_matches_oracle_and_golden(torch_cuda):
    from tests.golden import make_golden

    w = wl.tiny(0)
    dev = to_torch(w.pool)
    ref_pool = w.pool.copy()
    outs = []
    for s in w.steps:
        before, ref_before = dev.cpu().numpy(), ref_pool
        out = run_gpu(dev, s)
        ref_pool, ref_out, _ = run_oracle(ref_pool, s)
        assert rel_err(out, ref_out) <= TOL_OUT_F32
        check_pool(dev.cpu().numpy(), ref_pool, before, s.dst_idx, ref_before)
        outs.append(out.reshape(-1))
    g_outs, g_pool = make_golden.load()
    assert rel_err(np.stack(outs), g_outs) <= TOL_OUT_F32
    assert rel_err(dev.cpu().numpy(), g_pool) <= TOL_STATE


@pytest.mark.parametrize("variant", [None, "stream", "tile", "column"])
@pytest.mark.parametrize("name", ["decode_b16", "prefix_cow"])
def test_decode_workloads(torch_cuda, name, variant):
    w = wl.WORKLOADS[name]()
    s = w.steps[0]
    dev = to_torch(w.pool)
    out = run_gpu(dev, s, variant=variant)
    ref_pool, ref_out, skipped = run_oracle(w.pool, s)
    assert skipped == 0
    got = dev.cpu().numpy()
    check_pool(got, ref_pool, w.pool, s.dst_idx)
    assert rel_err(out, ref_out) <= _tol_out(s)
    # copy-on-write: every source slot is byte-identical after the call unless it is also written
    src_only = np.setdiff1d(s.src_idx, s.dst_idx.ravel())
    assert np.array_equal(got[src_only].view(np.uint32), w.pool[src_only].view(np.uint32))


@pytest.mark.parametrize("variant", [None, "column"])
def test_speculative_and_commit(torch_cuda, variant):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    w = wl.speculative()
    s = w.steps[0]
    dev = to_torch(w.pool)
    out = run_gpu(dev, s, variant=variant)
    ref_pool, ref_out, _ = run_oracle(w.pool, s)
    got = dev.cpu().numpy()
    check_pool(got, ref_pool, w.pool, s.dst_idx)
    assert rel_err(out, ref_out) <= TOL_OUT_BF16

    # commit: bit-exact index table, no pool byte changes
    import oracle

    committed = torch.from_numpy(s.src_idx.copy()).cuda()
    cur = torch.from_numpy(s.dst_idx.copy()).cuda()
    accept = torch.from_numpy(s.accept_len.copy()).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool_before = dev.clone()
    gdn.gdn_commit(accept, committed, cur, w.num_slots, err_word=err)
    want = s.src_idx.copy()
    assert oracle.commit(s.accept_len, want, s.dst_idx, w.num_slots) == 0
    assert np.array_equal(committed.cpu().numpy(), want)
    assert torch.equal(dev.view(torch.int32), pool_before.view(torch.int32))
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    gdn.gdn_commit(accept, committed, cur, w.num_slots)  # idempotent
    assert np.array_equal(committed.cpu().numpy(), want)


@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
def test_sequential_equals_speculative_bitwise(torch_cuda, dtype):
    """T chained single-token calls and one T-token call give identical bits on the GPU."""
    rng = np.random.default_rng(40)
    num_slots, B, T, Hk, Hv, dk, dv = 40, 4, 4, 2, 4, 128, 128
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, Hk, Hv, dk, dv, dtype)
    src = np.arange(B, dtype=np.int32)
    cur = (B + np.arange(B * T, dtype=np.int32)).reshape(B, T)
    spec = to_torch(pool)
    out_spec = run_gpu(spec, wl.Step(q, k, v, a, b, src, cur))
    seq = to_torch(pool)
    prev = src
    for t in range(T):
        sl = lambda x: np.ascontiguousarray(x[:, t:t + 1])
        o = run_gpu(seq, wl.Step(sl(q), sl(k), sl(v), sl(a), sl(b), prev.copy(), sl(cur)))
        assert np.array_equal(o[:, 0], out_spec[:, t])
        prev = cur[:, t].copy()
    assert np.array_equal(seq.cpu().numpy().view(np.uint32), spec.cpu().numpy().view(np.uint32))


SHAPES = [
    # (B, T, Hk, Hv, dk, dv, dtype, in_place)
    (3, 1, 1, 1, 16, 16, wl.F32, False),
    (5, 2, 2, 4, 3, 5, wl.BF16, False),
    (4, 1, 2, 2, 64, 64, wl.BF16, True),
    (3, 3, 1, 3, 64, 64, wl.F32, False),
    (2, 2, 1, 2, 100, 72, wl.BF16, False),
    (6, 1, 4, 8, 128, 128, wl.F32, True),
    (3, 2, 2, 2, 256, 128, wl.BF16, False),
    (2, 1, 1, 1, 128, 300, wl.BF16, True),
    (1, 5, 1, 1, 1, 1, wl.F32, False),
    (7, 1, 1, 2, 33, 257, wl.F32, False),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}T{}Hk{}Hv{}dk{}dv{}{}{}".format(*s[:7], "ip" if s[7] else ""))
def test_shapes_and_ragged_tails(torch_cuda, shape):
    B, T, Hk, Hv, dk, dv, dtype, in_place = shape
    rng = np.random.default_rng(zlib.crc32(repr(shape).encode()))
    num_slots = B * (T + 1) + 3
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, Hk, Hv, dk, dv, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = src.reshape(B, 1).copy() if in_place else perm[B:B + B * T].reshape(B, T).copy()
    s = wl.Step(q, k, v, a, b, src, dst)
    dev = to_torch(pool)
    out = run_gpu(dev, s)
    ref_pool, ref_out, _ = run_oracle(pool, s)
    check_pool(dev.cpu().numpy(), ref_pool, pool, dst)
    assert rel_err(out, ref_out) <= _tol_out(s)


def test_empty_batch_is_a_no_op(torch_cuda):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    pool = torch.ones((2, 1, 128, 128), device="cuda")
    e = torch.zeros((0, 1, 1, 128), dtype=torch.bfloat16, device="cuda")
    ab = torch.zeros((0, 1, 1), device="cuda")
    idx = torch.zeros((0,), dtype=torch.int32, device="cuda")
    out = torch.zeros((0, 1, 1, 128), device="cuda")
    assert gdn.gdn_decode_step(pool, idx, idx.view(0, 1), e, e, e, ab, ab, out) == gdn.GDN_OK
    assert gdn.gdn_commit(idx, idx, idx.view(0, 1), 2) == gdn.GDN_OK
    torch.cuda.synchronize()
    assert bool((pool == 1).all())


@pytest.mark.parametrize("dk,dv,T", [(128, 128, 2), (20, 24, 2), (128, 128, 1)])
def test_out_of_range_indices_skip_and_report(torch_cuda, dk, dv, T):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(50)
    num_slots, B = 12, 4
    pool = wl.init_pool(rng, num_slots, 2, dk, dv)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, 1, 2, dk, dv, wl.BF16)
    src = np.array([0, num_slots, 2, -3], np.int32)
    dst = np.array([[4, 5], [6, 7], [8, 99], [10, 11]], np.int32)[:, :T].copy()
    if T == 1:
        dst[2, 0] = 99
    s = wl.Step(q, k, v, a, b, src, dst)
    dev = to_torch(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_gpu(dev, s, err=err)
    ref_pool, ref_out, skipped = run_oracle(pool, s)
    assert skipped == 3
    assert gdn.gdn_get_error(err) == gdn.GDN_ERR_INDEX
    assert gdn.gdn_get_error(err) == gdn.GDN_OK  # read-and-clear
    got = dev.cpu().numpy()
    check_pool(got, ref_pool, pool, dst[:1])
    assert np.all(out[1:] == -7.0)
    assert rel_err(out[:1], ref_out[:1]) <= TOL_OUT_BF16

    T = 2
    accept = torch.tensor([1, -1, T + 1, 2], dtype=torch.int32, device="cuda")
    cur = torch.tensor([[4, 5], [6, 7], [8, 9], [10, num_slots + 4]], dtype=torch.int32, device="cuda")
    committed = torch.tensor([0, 1, 2, 3], dtype=torch.int32, device="cuda")
    gdn.gdn_commit(accept, committed, cur, num_slots, err_word=err)
    assert committed.cpu().tolist() == [4, 1, 2, 3]
    assert gdn.gdn_get_error(err) == gdn.GDN_ERR_INDEX


@pytest.mark.parametrize("variant", [None, "stream", "column"])
@pytest.mark.parametrize("T", [1, 3])
def test_padding_requests_are_silent(torch_cuda, variant, T):
    """src = GDN_SLOT_NONE (-1) rows are skipped without an error, whatever their dst holds."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    if variant == "stream" and T != 1:
        pytest.skip("the streaming kernel serves single-token calls")
    rng = np.random.default_rng(70 + T)
    B, num_slots, Hk, Hv = 8, 40, 2, 4
    pool = wl.init_pool(rng, num_slots, Hv, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, Hk, Hv, 128, 128, wl.BF16)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = perm[B:B + B * T].reshape(B, T).copy()
    src[[1, 4, 7]] = -1
    dst[1, 0], dst[4, -1] = 10 ** 6, -9   # ignored for padding rows
    s = wl.Step(q, k, v, a, b, src, dst)
    dev = to_torch(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_gpu(dev, s, err=err, variant=variant)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    ref_pool, ref_out, skipped = run_oracle(pool, s)
    assert skipped == 0
    live = np.array([0, 2, 3, 5, 6])
    check_pool(dev.cpu().numpy(), ref_pool, pool, dst[live])
    assert np.all(out[[1, 4, 7]] == -7.0)
    assert rel_err(out[live], ref_out[live]) <= TOL_OUT_BF16


def test_unaligned_pool_uses_column_path(torch_cuda):
    """A pool that starts off a 16-byte boundary still gives oracle results."""
    torch = torch_cuda
    w = wl.decode_b16()
    s = w.steps[0]
    n = w.pool.size
    buf = torch.empty(n + 1, dtype=torch.float32, device="cuda")
    dev = buf[1:].view(w.pool.shape)
    dev.copy_(torch.from_numpy(w.pool))
    out = run_gpu(dev, s)
    ref_pool, ref_out, _ = run_oracle(w.pool, s)
    check_pool(dev.cpu().numpy(), ref_pool, w.pool, s.dst_idx)
    assert rel_err(out, ref_out) <= TOL_OUT_BF16


def test_side_stream(torch_cuda):
    torch = torch_cuda
    w = wl.decode_b16()
    s = w.steps[0]
    dev = to_torch(w.pool)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        out = run_gpu(dev, s, stream=st)
    ref_pool, ref_out, _ = run_oracle(w.pool, s)
    check_pool(dev.cpu().numpy(), ref_pool, w.pool, s.dst_idx)
    assert rel_err(out, ref_out) <= TOL_OUT_BF16


def test_invalid_arguments_raise(torch_cuda):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    w = wl.decode_b16()
    s = w.steps[0]
    x = step_to_device(s)
    pool = torch.zeros((4, 32, 128, 128), device="cuda")
    out = torch.zeros((16, 1, 32, 128), device="cuda")
    with pytest.raises(gdn.GdnError) as ei:  # Hv = 32 not a multiple of Hk = 3
        gdn.gdn_decode_step(pool, x["src"], x["dst"], x["q"][:, :, :3].contiguous(), x["k"][:, :, :3].contiguous(),
                            x["v"], x["alpha"], x["beta"], out)
    assert ei.value.status == gdn.GDN_ERR_INVALID_ARG
    with pytest.raises(TypeError):
        gdn.gdn_decode_step(pool, x["src"], x["dst"], x["q"], x["k"], x["v"].float(), x["alpha"], x["beta"], out)


def test_mismatched_shapes_are_rejected_by_the_binding(torch_cuda):
    """The library takes plain pointers and cannot see buffer sizes; the binding checks every
    tensor's shape against pool and q before anything is enqueued."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    s = wl.decode_b16().steps[0]
    x = step_to_device(s)
    pool = torch.zeros((64, 32, 128, 128), device="cuda")
    out = torch.zeros((16, 1, 32, 128), device="cuda")
    good = dict(pool=pool, src_idx=x["src"], dst_idx=x["dst"], q=x["q"], k=x["k"], v=x["v"], alpha=x["alpha"],
                beta=x["beta"], out=out)
    bad = {"k": x["k"][:8], "v": x["v"][:, :, :16], "alpha": x["alpha"][:, :, :8], "out": out[:, :, :, :64],
           "dst_idx": x["dst"][:8], "src_idx": x["src"][:4]}
    for name, t in bad.items():
        with pytest.raises(ValueError):
            gdn.gdn_decode_step(**{**good, name: t.contiguous()})
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):  # a prefill takes one destination per request
        gdn.gdn_prefill_chunked(**{**good, "dst_idx": torch.zeros(32, dtype=torch.int32, device="cuda")},
                                workspace=ws, err_word=torch.zeros(1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert not bool(pool.any())  # nothing ran


def test_variant_conditions_are_checked(torch_cuda):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    w = wl.speculative()
    s = w.steps[0]
    x = step_to_device(s)
    pool = to_torch(w.pool)
    out = torch.zeros((s.B, s.T, s.Hv, s.dv), device="cuda")
    args = (pool, x["src"], x["dst"], x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
    for bad in ("stream", 9):  # the streaming kernel serves single-token calls only; 9 is no variant
        with pytest.raises(gdn.GdnError) as ei:
            gdn.gdn_decode_step_variant(*args, bad)
        assert ei.value.status == gdn.GDN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert np.array_equal(pool.cpu().numpy(), w.pool)  # nothing ran


@pytest.mark.parametrize("B", [1, 3, 37, 300])
def test_stream_kernel_partial_waves(torch_cuda, B):
    """Unit counts below, at and above one unit per SM, and not a multiple of the grid."""
    rng = np.random.default_rng(60 + B)
    Hk, Hv = 2, 4
    num_slots = 2 * B + 5
    pool = wl.init_pool(rng, num_slots, Hv, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, 1, Hk, Hv, 128, 128, wl.BF16)
    perm = rng.permutation(num_slots).astype(np.int32)
    s = wl.Step(q, k, v, a, b, perm[:B].copy(), perm[B:2 * B].reshape(B, 1).copy())
    dev = to_torch(pool)
    out = run_gpu(dev, s, variant="stream")
    ref_pool, ref_out, _ = run_oracle(pool, s)
    check_pool(dev.cpu().numpy(), ref_pool, pool, s.dst_idx)
    assert rel_err(out, ref_out) <= TOL_OUT_BF16


def test_check_step_matches_oracle(torch_cuda):
    """The device precondition check returns exactly the oracle's verdict (integer work: bit-exact)."""
    torch = torch_cuda
    import oracle
    from hybrid_linear_attention_step_b200 import gdn

    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    scratch = torch.empty(64, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(80)
    seen = set()
    for trial in range(300):
        T = int(rng.integers(1, 4))
        num_slots = int(rng.integers(4, 48))
        B = int(rng.integers(1, 9))
        src = rng.integers(-2, num_slots + 1, size=B).astype(np.int32)
        dst = rng.integers(-1, num_slots + 1, size=(B, T)).astype(np.int32)
        if trial % 2 == 0:
            perm = rng.permutation(num_slots + B * T + B)[: B + B * T] % num_slots
            src, dst = perm[:B].astype(np.int32), perm[B:].reshape(B, T).astype(np.int32)
            if trial % 4 == 0:
                src[rng.integers(0, B)] = -1
        want = oracle.check_step(src, dst, num_slots)
        gdn.gdn_check_step(torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda(), num_slots, scratch, err)
        got = gdn.gdn_get_error(err)
        assert got == want, (src.tolist(), dst.tolist(), num_slots, got, want)
        seen.add(want)
    assert seen == {0, 3, 5}


@pytest.mark.parametrize("name", ["decode_b16", "prefix_cow", "speculative"])
def test_check_step_accepts_the_workloads(torch_cuda, name):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    w = wl.WORKLOADS[name]()
    s = w.steps[0]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    scratch = torch.empty(w.num_slots, dtype=torch.int32, device="cuda")
    gdn.gdn_check_step(torch.from_numpy(s.src_idx).cuda(), torch.from_numpy(s.dst_idx).cuda(), w.num_slots,
                       scratch, err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    bad = s.dst_idx.copy()
    bad[-1, -1] = s.src_idx[0]  # the last request writes the first request's source
    gdn.gdn_check_step(torch.from_numpy(s.src_idx).cuda(), torch.from_numpy(bad).cuda(), w.num_slots, scratch, err)
    assert gdn.gdn_get_error(err) == gdn.GDN_ERR_ALIAS


def test_cuda_graph_replay_of_padded_batches(torch_cuda):
    """Static-shape decode calls captured once in a CUDA graph and replayed: the batch is padded
    to a fixed size with GDN_SLOT_NONE rows, the slot tables are rewritten between replays, and
    every replay matches the oracle (single-token and speculative calls in one graph)."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(100)
    Bmax, Hk, Hv, dk, dv, num_slots, T = 12, 2, 4, 128, 128, 96, 2
    pool_np = wl.init_pool(rng, num_slots, Hv, dk, dv)
    pool = to_torch(pool_np)
    q1, k1, v1, a1, b1 = (to_torch(x) for x in wl.random_step_inputs(rng, Bmax, 1, Hk, Hv, dk, dv, wl.BF16))
    q2, k2, v2, a2, b2 = (to_torch(x) for x in wl.random_step_inputs(rng, Bmax, T, Hk, Hv, dk, dv, wl.BF16))
    src1 = torch.full((Bmax,), -1, dtype=torch.int32, device="cuda")
    dst1 = torch.full((Bmax, 1), -1, dtype=torch.int32, device="cuda")
    src2 = torch.full((Bmax,), -1, dtype=torch.int32, device="cuda")
    cur2 = torch.full((Bmax, T), -1, dtype=torch.int32, device="cuda")
    out1 = torch.zeros((Bmax, 1, Hv, dv), device="cuda")
    out2 = torch.zeros((Bmax, T, Hv, dv), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def calls():
        gdn.gdn_decode_step(pool, src1, dst1, q1, k1, v1, a1, b1, out1, err_word=err)
        gdn.gdn_decode_step(pool, src2, cur2, q2, k2, v2, a2, b2, out2, err_word=err)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        calls()  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        calls()

    def to_host(t):  # bf16 tensors come back as their uint16 bit patterns
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).cpu().numpy().view(np.uint16)
        return t.cpu().numpy()

    host = {n: to_host(t) for n, t in dict(q1=q1, k1=k1, v1=v1, a1=a1, b1=b1, q2=q2, k2=k2, v2=v2, a2=a2,
                                            b2=b2).items()}
    bits = lambda t: t
    for replay in range(3):
        n1, n2 = int(rng.integers(1, Bmax)), int(rng.integers(1, Bmax))
        perm = rng.permutation(num_slots).astype(np.int32)
        s1 = np.full(Bmax, -1, np.int32)
        d1 = np.full((Bmax, 1), -1, np.int32)
        s2 = np.full(Bmax, -1, np.int32)
        c2 = np.full((Bmax, T), -1, np.int32)
        rows1 = np.sort(rng.choice(Bmax, n1, replace=False))
        rows2 = np.sort(rng.choice(Bmax, n2, replace=False))
        s1[rows1] = perm[:n1]
        d1[rows1, 0] = perm[:n1]                                   # in place
        s2[rows2] = perm[n1:n1 + n2]
        c2[rows2] = perm[n1 + n2:n1 + n2 + n2 * T].reshape(n2, T)  # fresh draft slots
        for t_, a_ in ((src1, s1), (dst1, d1), (src2, s2), (cur2, c2)):
            t_.copy_(torch.from_numpy(a_))
        before = pool.cpu().numpy()
        out1.fill_(-7.0)
        out2.fill_(-7.0)
        graph.replay()
        torch.cuda.synchronize()
        assert gdn.gdn_get_error(err) == gdn.GDN_OK
        ref = before
        ref, ref_o1, sk1 = run_oracle(ref, wl.Step(bits(host["q1"]), bits(host["k1"]), bits(host["v1"]), host["a1"],
                                                   host["b1"], s1, d1))
        ref, ref_o2, sk2 = run_oracle(ref, wl.Step(bits(host["q2"]), bits(host["k2"]), bits(host["v2"]), host["a2"],
                                                   host["b2"], s2, c2))
        assert sk1 == sk2 == 0
        written = np.concatenate([d1[rows1].ravel(), c2[rows2].ravel()])
        check_pool(pool.cpu().numpy(), ref, before, written)
        o1, o2 = out1.cpu().numpy(), out2.cpu().numpy()
        assert rel_err(o1[rows1], ref_o1[rows1]) <= TOL_OUT_BF16
        assert rel_err(o2[rows2], ref_o2[rows2]) <= TOL_OUT_BF16
        pad1 = np.setdiff1d(np.arange(Bmax), rows1)
        pad2 = np.setdiff1d(np.arange(Bmax), rows2)
        assert np.all(o1[pad1] == -7.0) and np.all(o2[pad2] == -7.0)


FUSED_SHAPES = [
    # (B, T, Hk, Hv, dk, dv, dtype)
    (16, 1, 16, 32, 128, 128, wl.BF16),   # single-token register tiles
    (6, 3, 2, 4, 128, 128, wl.BF16),      # multi-token register tiles
    (5, 1, 2, 2, 64, 64, wl.F32),
    (3, 2, 1, 2, 33, 72, wl.BF16),        # column kernel
]


@pytest.mark.parametrize("flags", [1, 2, 3], ids=["gates", "qknorm", "both"])
@pytest.mark.parametrize("shape", FUSED_SHAPES, ids=lambda s: "B{}T{}Hk{}Hv{}dk{}dv{}{}".format(*s))
def test_fused_prologue_matches_oracle(torch_cuda, shape, flags):
    """gdn_decode_step_fused: raw gate pre-activations and/or unnormalised q, k enter the kernel."""
    torch = torch_cuda
    import oracle
    from hybrid_linear_attention_step_b200 import gdn

    B, T, Hk, Hv, dk, dv, dtype = shape
    rng = np.random.default_rng(zlib.crc32(repr((shape, flags)).encode()))
    num_slots = B * (T + 1) + 2
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv)
    qr, kr, v, x, y = wl.random_raw_step_inputs(rng, B, T, Hk, Hv, dk, dv, dtype)
    qn, kn, _, alpha, beta = wl.random_step_inputs(rng, B, T, Hk, Hv, dk, dv, dtype)
    q, k = (qr, kr) if flags & gdn.GDN_FUSE_QK_NORM else (qn, kn)
    g1, g2 = (x, y) if flags & gdn.GDN_FUSE_GATES else (alpha, beta)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = perm[B:B + B * T].reshape(B, T).copy()
    s = wl.Step(q, k, v, g1, g2, src, dst)
    dev = to_torch(pool)
    xd = step_to_device(s)
    out = torch.full((B, T, Hv, dv), -7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.gdn_decode_step_fused(dev, xd["src"], xd["dst"], xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out,
                              flags, err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    ref_pool, ref_out = pool.copy(), np.zeros((B, T, Hv, dv), np.float32)
    oracle.decode_step(ref_pool, src, dst, q, k, v, g1, g2, ref_out, flags=flags, nthreads=8)
    check_pool(dev.cpu().numpy(), ref_pool, pool, dst)
    assert rel_err(out.cpu().numpy(), ref_out) <= _tol_out(s)


def test_fused_without_flags_equals_plain_bitwise(torch_cuda):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    w = wl.decode_b16()
    s = w.steps[0]
    xd = step_to_device(s)
    outs, pools = [], []
    for fused in (False, True):
        dev = to_torch(w.pool)
        out = torch.zeros((s.B, 1, s.Hv, s.dv), device="cuda")
        args = (dev, xd["src"], xd["dst"], xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out)
        gdn.gdn_decode_step_fused(*args, 0) if fused else gdn.gdn_decode_step(*args)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
        pools.append(dev.cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(pools[0].view(np.uint32), pools[1].view(np.uint32))
    with pytest.raises(gdn.GdnError):
        gdn.gdn_decode_step_fused(*args, 8)  # no such flag


PREFILL_SHAPES = [
    # (B, L, Hk, Hv, dk, dv, dtype, in_place)
    (4, 1, 2, 4, 128, 128, wl.BF16, False),
    (3, 7, 2, 4, 128, 128, wl.BF16, True),
    (2, 96, 1, 2, 128, 128, wl.BF16, False),
    (3, 33, 2, 2, 64, 64, wl.F32, True),
    (2, 9, 1, 2, 40, 24, wl.BF16, False),   # column kernel
]


@pytest.mark.parametrize("shape", PREFILL_SHAPES, ids=lambda s: "B{}L{}Hk{}Hv{}dk{}dv{}{}{}".format(*s[:7], "ip" if s[7] else ""))
def test_prefill_matches_oracle(torch_cuda, shape):
    torch = torch_cuda
    import oracle
    from hybrid_linear_attention_step_b200 import gdn

    B, L, Hk, Hv, dk, dv, dtype, in_place = shape
    rng = np.random.default_rng(zlib.crc32(repr(shape).encode()))
    num_slots = 2 * B + 3
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, dk, dv, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = src.copy() if in_place else perm[B:2 * B].copy()
    s = wl.Step(q, k, v, a, b, src, dst.reshape(B, 1))
    xd = step_to_device(s)
    dev = to_torch(pool)
    out = torch.full((B, L, Hv, dv), -7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.gdn_prefill(dev, xd["src"], to_torch(dst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out,
                    err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    ref_pool, ref_out = pool.copy(), np.zeros((B, L, Hv, dv), np.float32)
    assert oracle.prefill(ref_pool, src, dst, q, k, v, a, b, ref_out, nthreads=8) == 0
    check_pool(dev.cpu().numpy(), ref_pool, pool, dst)
    assert rel_err(out.cpu().numpy(), ref_out) <= _tol_out(s)


def test_prefill_equals_decode_last_state_bitwise(torch_cuda):
    """On the GPU the prefill's final state is the bits a T = L decode call stores for its last token."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(44)
    B, L, Hk, Hv = 3, 12, 2, 4
    pool = wl.init_pool(rng, 3 * B + B * L, Hv, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, 128, 128, wl.BF16)
    src = np.arange(B, dtype=np.int32)
    pdst = np.arange(B, 2 * B, dtype=np.int32)
    cur = (3 * B + np.arange(B * L, dtype=np.int32)).reshape(B, L)
    xd = step_to_device(wl.Step(q, k, v, a, b, src, cur))
    dev = to_torch(pool)
    o1 = torch.zeros((B, L, Hv, 128), device="cuda")
    o2 = torch.zeros_like(o1)
    gdn.gdn_prefill(dev, xd["src"], to_torch(pdst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o1)
    gdn.gdn_decode_step(dev, xd["src"], xd["dst"], xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o2)
    torch.cuda.synchronize()
    got = dev.cpu().numpy()
    assert np.array_equal(got[pdst].view(np.uint32), got[cur[:, -1]].view(np.uint32))
    assert torch.equal(o1, o2)


def test_prefill_padding_rows_are_silent(torch_cuda):
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(45)
    B, L = 4, 5
    pool = wl.init_pool(rng, 10, 4, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, 2, 4, 128, 128, wl.BF16)
    src = np.array([0, -1, 2, -1], np.int32)
    dst = np.array([4, 99, 5, -3], np.int32)  # padding rows' destinations are ignored
    xd = step_to_device(wl.Step(q, k, v, a, b, src, dst.reshape(B, 1)))
    dev = to_torch(pool)
    out = torch.full((B, L, 4, 128), -7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.gdn_prefill(dev, xd["src"], to_torch(dst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out,
                    err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    o = out.cpu().numpy()
    assert np.all(o[[1, 3]] == -7.0) and not np.any(o[[0, 2]] == -7.0)
    untouched = [0, 1, 2, 3, 6, 7, 8, 9]
    assert np.array_equal(dev.cpu().numpy()[untouched].view(np.uint32), pool[untouched].view(np.uint32))


CHUNKED_SHAPES = [
    # (B, L, Hk, Hv, dtype, in_place)
    (2, 1, 1, 2, wl.BF16, False),
    (3, 64, 2, 4, wl.BF16, True),
    (2, 65, 1, 2, wl.BF16, False),
    (2, 200, 2, 2, wl.F32, False),
    (1, 1000, 1, 2, wl.BF16, True),
    (4, 130, 2, 2, wl.BF16, False),   # one value head per key head, ragged last chunk
    (2, 96, 1, 4, wl.BF16, True),     # four value heads per key head, in place
    (10, 130, 16, 32, wl.BF16, False),  # 320 scan CTAs: more (request, head) chains than SMs
]


@pytest.mark.parametrize("shape", CHUNKED_SHAPES, ids=lambda s: "B{}L{}Hk{}Hv{}{}{}".format(*s[:5], "ip" if s[5] else ""))
def test_prefill_chunked_matches_oracle(torch_cuda, shape):
    """The chunked prefill (per-chunk triangular solve + dense contractions) against the
    token-by-token oracle, for chunk-aligned, ragged and multi-chunk lengths."""
    torch = torch_cuda
    import oracle
    from hybrid_linear_attention_step_b200 import gdn

    B, L, Hk, Hv, dtype, in_place = shape
    rng = np.random.default_rng(zlib.crc32(repr(shape).encode()))
    num_slots = 2 * B + 3
    pool = wl.init_pool(rng, num_slots, Hv, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, 128, 128, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = src.copy() if in_place else perm[B:2 * B].copy()
    xd = step_to_device(wl.Step(q, k, v, a, b, src, dst.reshape(B, 1)))
    dev = to_torch(pool)
    out = torch.full((B, L, Hv, 128), -7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, 128, 128), dtype=torch.uint8, device="cuda")
    gdn.gdn_prefill_chunked(dev, xd["src"], to_torch(dst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out,
                            ws, err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    ref_pool, ref_out = pool.copy(), np.zeros((B, L, Hv, 128), np.float32)
    assert oracle.prefill(ref_pool, src, dst, q, k, v, a, b, ref_out, nthreads=8) == 0
    check_pool(dev.cpu().numpy(), ref_pool, pool, dst)
    assert rel_err(out.cpu().numpy(), ref_out) <= TOL_OUT_BF16


@pytest.mark.parametrize("L", [200, 700, 4096])
def test_prefill_chunked_slow_decay(torch_cuda, L):
    """Gates close to one (alpha ~ 0.97, the slow forgetting of trained models): the chunk-start
    state then reaches every token of a chunk, so the products with the carried state (W M,
    and the state update) carry the result and their precision is what is tested.  L = 4096
    carries the state through 64 chunks, where a part product left out would accumulate."""
    torch = torch_cuda
    import oracle
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(47 + L)
    B, Hk, Hv = 2, 1, 2
    pool = wl.init_pool(rng, 2 * B, Hv, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, 128, 128, wl.BF16)
    a = np.exp(np.log(a) * np.float32(0.03)).astype(np.float32)
    src = np.arange(B, dtype=np.int32)
    dst = np.arange(B, 2 * B, dtype=np.int32)
    xd = step_to_device(wl.Step(q, k, v, a, b, src, dst.reshape(B, 1)))
    dev = to_torch(pool)
    out = torch.full((B, L, Hv, 128), -7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, 128, 128), dtype=torch.uint8, device="cuda")
    gdn.gdn_prefill_chunked(dev, xd["src"], to_torch(dst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out,
                            ws, err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    ref_pool, ref_out = pool.copy(), np.zeros((B, L, Hv, 128), np.float32)
    assert oracle.prefill(ref_pool, src, dst, q, k, v, a, b, ref_out, nthreads=8) == 0
    check_pool(dev.cpu().numpy(), ref_pool, pool, dst)
    assert rel_err(out.cpu().numpy(), ref_out) <= TOL_OUT_BF16


def test_prefill_chunked_edge_cases(torch_cuda):
    """Padding rows, an out-of-range slot, a full reset (alpha = 0) and a short workspace."""
    torch = torch_cuda
    import oracle
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(46)
    B, L, Hv = 4, 130, 2
    pool = wl.init_pool(rng, 12, Hv, 128, 128)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, 1, Hv, 128, 128, wl.BF16)
    a[2, 70, :] = 0.0  # request 2 forgets its history at token 70
    src = np.array([0, -1, 2, 3], np.int32)
    dst = np.array([4, 99, 6, 12], np.int32)  # request 3: destination out of range
    xd = step_to_device(wl.Step(q, k, v, a, b, src, dst.reshape(B, 1)))
    dev = to_torch(pool)
    out = torch.full((B, L, Hv, 128), -7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbytes = gdn.gdn_prefill_workspace_bytes(B, L, Hv, 128, 128)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GdnError):
        gdn.gdn_prefill_chunked(dev, xd["src"], to_torch(dst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"],
                                out, ws[: nbytes - 16], err_word=err)
    gdn.gdn_prefill_chunked(dev, xd["src"], to_torch(dst), xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], out,
                            ws, err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_ERR_INDEX
    ref_pool, ref_out = pool.copy(), np.full((B, L, Hv, 128), -7.0, np.float32)
    assert oracle.prefill(ref_pool, src, dst, q, k, v, a, b, ref_out, nthreads=8) == 1
    check_pool(dev.cpu().numpy(), ref_pool, pool, np.array([4, 6]))
    o = out.cpu().numpy()
    assert np.all(o[[1, 3]] == -7.0)
    assert rel_err(o[[0, 2]], ref_out[[0, 2]]) <= TOL_OUT_BF16


def test_bounded_wait_runs_out_and_reports_timeout(torch_cuda):
    """The pipelines' bounded mbarrier wait, run on a barrier that nothing arrives on:
    it gives up after its limit, records GDN_ERR_TIMEOUT, and the context stays usable."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    gdn.gdn_wait_selftest(20_000_000, err)  # 20 ms
    e1.record()
    torch.cuda.synchronize()
    assert gdn.gdn_get_error(err) == gdn.GDN_ERR_TIMEOUT
    assert e0.elapsed_time(e1) >= 19.0
    w = wl.decode_b16()
    dev = to_torch(w.pool)
    out = run_gpu(dev, w.steps[0], err=err)
    ref_pool, ref_out, _ = run_oracle(w.pool, w.steps[0])
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    check_pool(dev.cpu().numpy(), ref_pool, w.pool, w.steps[0].dst_idx)
    assert rel_err(out, ref_out) <= TOL_OUT_BF16


@pytest.mark.parametrize("T", [1, 3])
def test_prepared_decode_step_equals_the_checked_call(torch_cuda, T):
    """The prepared form (buffers checked once, stream bound or not) enqueues the same call:
    bit for bit the checked call's results, and the oracle's; its buffers' contents change
    between calls (new inputs and slot tables) while their storage stays."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(300 + T)
    B, Hk, Hv, d = 6, 2, 4, 128
    num_slots = B * (T + 1) + 2
    pool_np = wl.init_pool(rng, num_slots, Hv, d, d)
    dev_a, dev_b = to_torch(pool_np), to_torch(pool_np)
    q, k, v, a, b = (to_torch(x) for x in wl.random_step_inputs(rng, B, T, Hk, Hv, d, d, wl.BF16))
    src = torch.zeros(B, dtype=torch.int32, device="cuda")
    dst = torch.zeros((B, T), dtype=torch.int32, device="cuda")
    out_a = torch.zeros((B, T, Hv, d), device="cuda")
    out_b = torch.zeros((B, T, Hv, d), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bound = gdn.PreparedDecodeStep(dev_b, src, dst, q, k, v, a, b, out_b, err_word=err,
                                   stream=torch.cuda.current_stream())
    unbound = gdn.PreparedDecodeStep(dev_b, src, dst, q, k, v, a, b, out_b, err_word=err)
    ref = pool_np.copy()
    for it, call in enumerate((bound, unbound, bound)):
        perm = rng.permutation(num_slots).astype(np.int32)
        src_np = perm[:B].copy()
        dst_np = (src_np.reshape(B, 1).copy() if T == 1 else perm[B:B + B * T].reshape(B, T).copy())
        src.copy_(torch.from_numpy(src_np))
        dst.copy_(torch.from_numpy(dst_np))
        hq, hk_, hv, ha, hb = wl.random_step_inputs(rng, B, T, Hk, Hv, d, d, wl.BF16)
        for t_dev, x in ((q, hq), (k, hk_), (v, hv), (a, ha), (b, hb)):
            t_dev.copy_(to_torch(x))
        gdn.gdn_decode_step(dev_a, src, dst, q, k, v, a, b, out_a, err_word=err)
        call()
        torch.cuda.synchronize()
        assert gdn.gdn_get_error(err) == gdn.GDN_OK
        got_a, got_b = dev_a.cpu().numpy(), dev_b.cpu().numpy()
        assert np.array_equal(got_a.view(np.uint32), got_b.view(np.uint32)), it
        assert np.array_equal(out_a.cpu().numpy().view(np.uint32), out_b.cpu().numpy().view(np.uint32)), it
        s = wl.Step(hq, hk_, hv, ha, hb, src_np, dst_np)
        before = ref.copy()
        ref, ref_out, skipped = run_oracle(ref, s)
        assert skipped == 0
        check_pool(got_b, ref, before, dst_np)
        assert rel_err(out_b.cpu().numpy(), ref_out) <= TOL_OUT_BF16
        ref = got_b.copy()  # carry the device state on, so that each call is checked alone


@pytest.mark.parametrize("T,d,fuse", [(1, 128, 0), (3, 128, 0), (6, 128, 0), (1, 64, 0), (2, 128, 1), (1, 128, 3)],
                         ids=["T1", "T3", "T6", "d64", "T2gates", "T1fused"])
def test_shared_sources_hint_changes_no_bit(torch_cuda, T, d, fuse):
    """GDN_SHARED_SOURCES only reorders the register-tile kernels' CTAs (head-major): with
    a batch whose requests share source slots, every state and output equals the call
    without the hint bit for bit, and the oracle's within tolerance."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(400 + 10 * T + d + fuse)
    B, Hk, Hv = 12, 2, 4
    num_slots = 4 + B * T + 2
    pool_np = wl.init_pool(rng, num_slots, Hv, d, d)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, Hk, Hv, d, d, wl.BF16)
    src = rng.integers(0, 4, size=B).astype(np.int32)          # 12 requests over 4 shared checkpoints
    dst = (4 + np.arange(B * T, dtype=np.int32)).reshape(B, T)  # fresh slots, copy-on-write
    s = wl.Step(q, k, v, a, b, src, dst)
    x = step_to_device(s)
    results = []
    for flags in (fuse, fuse | gdn.GDN_SHARED_SOURCES):
        dev = to_torch(pool_np)
        out = torch.full((B, T, Hv, d), -7.0, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        args = (dev, x["src"], x["dst"], x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
        if flags:
            gdn.gdn_decode_step_fused(*args, flags, err_word=err)
        else:
            gdn.gdn_decode_step(*args, err_word=err)
        torch.cuda.synchronize()
        assert gdn.gdn_get_error(err) == gdn.GDN_OK
        results.append((dev.cpu().numpy(), out.cpu().numpy()))
    (p0, o0), (p1, o1) = results
    assert np.array_equal(p0.view(np.uint32), p1.view(np.uint32))
    assert np.array_equal(o0.view(np.uint32), o1.view(np.uint32))
    if fuse == 0:
        ref_pool, ref_out, skipped = run_oracle(pool_np, s)
        assert skipped == 0
        check_pool(p1, ref_pool, pool_np, dst)
        assert rel_err(o1, ref_out) <= TOL_OUT_BF16


def test_prefill_chunked_replays_from_a_cuda_graph(torch_cuda):
    """The chunked prefill captured once in a CUDA graph (its tensor maps are kernel
    arguments, its second kernel a programmatic dependent launch) and replayed with new
    inputs written into the captured buffers: every replay equals an eager call bit for bit."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(71)
    B, L, Hk, Hv = 2, 200, 2, 4
    pool0 = wl.init_pool(rng, 2 * B, Hv, 128, 128)
    src = to_torch(np.arange(B, dtype=np.int32))
    dst = to_torch(np.arange(B, 2 * B, dtype=np.int32))

    def inputs():
        q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, 128, 128, wl.BF16)
        return [to_torch(x) for x in (q, k, v, a, b)]

    bufs = inputs()
    pool = to_torch(pool0)
    out = torch.zeros((B, L, Hv, 128), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, 128, 128), dtype=torch.uint8, device="cuda")
    call = lambda: gdn.gdn_prefill_chunked(pool, src, dst, *bufs, out, ws, err_word=err)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(3):
        for t_dev, x in zip(bufs, inputs()):
            t_dev.copy_(x)
        pool.copy_(to_torch(pool0))
        graph.replay()
        torch.cuda.synchronize()
        got_pool, got_out = pool.cpu().numpy(), out.cpu().numpy()
        pool.copy_(to_torch(pool0))
        out.zero_()
        call()
        torch.cuda.synchronize()
        assert gdn.gdn_get_error(err) == gdn.GDN_OK
        assert np.array_equal(got_pool.view(np.uint32), pool.cpu().numpy().view(np.uint32))
        assert np.array_equal(got_out.view(np.uint32), out.cpu().numpy().view(np.uint32))
        assert np.isfinite(got_out).all()
