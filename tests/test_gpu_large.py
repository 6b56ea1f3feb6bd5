"""The large decode at full size, in the launch configuration the benchmark times.

B=256 requests x 8 layers, 2048-slot pools (32 GiB on the device).  The oracle
cannot redo all 65,536 units of a step in test time, so whole requests (all 32
heads) are sampled from every layer: their source tiles are read back before
the step, the oracle updates them in a private pool, and the CUDA results are
compared element by element.  Slots no request owns are checked byte for byte
on a sample too.
"""
import numpy as np
import pytest

import oracle
from tests.gpu_helpers import TOL_OUT_BF16, TOL_STATE, rel_err

pytestmark = pytest.mark.gpu

SAMPLES_PER_LAYER = 4


def test_large_decode_sampled_parity():
    import torch

    import bench

    wk = bench.LargeDecode(layers=8, num_slots=2048, B=256)
    rng = np.random.default_rng(7)
    # The first and last request of every layer are always among the samples: they sit at
    # the two ends of the launch grid (blockIdx.x 0 and the last CTAs).
    picks = [np.sort(np.concatenate([[0, wk.B - 1], 1 + rng.choice(wk.B - 2, SAMPLES_PER_LAYER - 2, replace=False)]))
             for _ in range(wk.layers)]
    before, untouched = [], []
    for l in range(wk.layers):
        slots = wk.host_steps[l].src_idx[picks[l]]
        before.append(wk.pools[l][torch.from_numpy(slots).long().cuda()].cpu().numpy())
        free = np.setdiff1d(np.arange(wk.num_slots), wk.host_steps[l].dst_idx.ravel())
        u = rng.choice(free, 4, replace=False)
        untouched.append((u, wk.pools[l][torch.from_numpy(u).long().cuda()].cpu().numpy()))
    wk.step()
    torch.cuda.synchronize()
    assert wk.gdn.gdn_get_error(wk.err) == 0
    for l in range(wk.layers):
        s = wk.host_steps[l]
        bsel = picks[l]
        n = len(bsel)
        pool = before[l].copy()                       # private pool: slot i holds request bsel[i]'s state
        idx = np.arange(n, dtype=np.int32)
        out = np.zeros((n, 1, wk.Hv, wk.dv), np.float32)
        sl = lambda a: np.ascontiguousarray(a[bsel])
        oracle.decode_step(pool, idx, idx.reshape(n, 1).copy(), sl(s.q), sl(s.k), sl(s.v), sl(s.alpha),
                           sl(s.beta), out, nthreads=n)
        got_state = wk.pools[l][torch.from_numpy(s.dst_idx[bsel, 0]).long().cuda()].cpu().numpy()
        got_out = wk.outs[l][torch.from_numpy(bsel).long().cuda()].cpu().numpy()
        assert rel_err(got_state, pool) <= TOL_STATE
        assert rel_err(got_out, out) <= TOL_OUT_BF16
        u, ub = untouched[l]
        now = wk.pools[l][torch.from_numpy(u).long().cuda()].cpu().numpy()
        assert np.array_equal(now.view(np.uint32), ub.view(np.uint32))


@pytest.mark.parametrize("chunked", [False, True], ids=["token_steps", "chunked"])
def test_prefill_bench_size_sampled_parity(chunked):
    """The prefill benchmark's launch (B=4 requests x L=2048 tokens, Hk=16, Hv=32, bf16):
    sampled (request, head) pairs are re-run by the oracle as a B=n, Hk=Hv=1 problem, and
    their checkpoint states and all 2048 outputs compared element by element."""
    import torch

    from hybrid_linear_attention_step_b200 import gdn, workloads as wl

    B, L, Hk, Hv, D = 4, 2048, 16, 32, 128
    rng = np.random.default_rng(6)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, D, D, wl.BF16)
    bits = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    pool = torch.empty((2 * B, Hv, D, D), dtype=torch.float32, device="cuda")
    wl.fill_pool_device(pool, 6, 0)
    before = pool[:B].cpu().numpy()
    src = torch.arange(B, dtype=torch.int32, device="cuda")
    dst = torch.arange(B, 2 * B, dtype=torch.int32, device="cuda")
    out = torch.full((B, L, Hv, D), -7.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (pool, src, dst, bits(q), bits(k), bits(v), torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), out)
    if chunked:
        ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, D, D), dtype=torch.uint8, device="cuda")
        gdn.gdn_prefill_chunked(*args, ws, err_word=err)
    else:
        gdn.gdn_prefill(*args, err_word=err)
    torch.cuda.synchronize()
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    picks = [(0, 0), (1, 17), (2, 31), (3, 6)]
    n = len(picks)
    hk = lambda h: h // (Hv // Hk)
    sq = np.stack([q[bb, :, hk(h)] for bb, h in picks])[:, :, None, :].copy()
    sk = np.stack([k[bb, :, hk(h)] for bb, h in picks])[:, :, None, :].copy()
    sv = np.stack([v[bb, :, h] for bb, h in picks])[:, :, None, :].copy()
    sa = np.stack([a[bb, :, h] for bb, h in picks])[:, :, None].copy()
    sb = np.stack([b[bb, :, h] for bb, h in picks])[:, :, None].copy()
    ref_pool = np.zeros((2 * n, 1, D, D), np.float32)
    ref_pool[:n, 0] = [before[bb, h] for bb, h in picks]
    ref_out = np.zeros((n, L, 1, D), np.float32)
    idx = np.arange(n, dtype=np.int32)
    assert oracle.prefill(ref_pool, idx, idx + n, sq, sk, sv, sa, sb, ref_out, nthreads=n) == 0
    got_pool = pool[B:].cpu().numpy()
    got_out = out.cpu().numpy()
    for i, (bb, h) in enumerate(picks):
        assert rel_err(got_pool[bb, h], ref_pool[n + i, 0]) <= TOL_STATE, (bb, h)
        assert rel_err(got_out[bb, :, h], ref_out[i, :, 0]) <= TOL_OUT_BF16, (bb, h)
    assert np.array_equal(pool[:B].cpu().numpy().view(np.uint32), before.view(np.uint32))  # sources untouched
