"""GPU parity at the gates' boundary values, and containment of non-finite inputs.

The gated delta rule has four boundary cases with closed forms (per token, value head):

* alpha = 1, beta = 0:  S' = S          (identity; the tile is stored unchanged, bit for bit)
* alpha = 0, beta = 0:  S' = 0, o = 0   (reset)
* alpha = 1, beta = 1, |k| = 1:  S' k = v   (delta-rule retrieval of v under key k)
* alpha = 0, beta = 1:  S' = v k^T      (pure write; each element one rounded product)

Every decode kernel (the register tiles, the bulk-copy pipeline, the column kernel) runs
all four and an interior pair in one call, one gate pair per request, and is compared
with the CPU oracle at the usual tolerances, plus the closed forms above exactly where
the arithmetic makes them exact.

Then a NaN in one request's q, k or v, or an infinite alpha, must stay inside the
(request, head) units whose inputs hold it: every other unit's state and outputs are
bitwise those of a run with clean inputs, and no slot outside the call's destinations
changes.  The poison is written on the host; nothing faults.
"""
import numpy as np
import pytest

from hybrid_linear_attention_step_b200 import workloads as wl
from tests.gpu_helpers import (TOL_OUT_BF16, TOL_OUT_F32, TOL_STATE, check_pool, rel_err, run_gpu, run_oracle,
                               step_to_device, to_torch)

pytestmark = pytest.mark.gpu

# (alpha, beta) per request; None draws an interior pair from the workload recipe.
GATES = [(1.0, 0.0), (0.0, 0.0), (1.0, 1.0), (0.0, 1.0), None]
BF16_NAN, BF16_INF = np.uint16(0x7FC0), np.uint16(0x7F80)


@pytest.fixture(scope="module")
def torch_cuda():
    import torch

    from hybrid_linear_attention_step_b200 import gdn

    gdn.load_library()
    return torch


def _as_f64(x):
    return (wl.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x).astype(np.float64)


def _boundary_step(rng, T, Hk, Hv, d, dtype):
    B = len(GATES)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, Hk, Hv, d, d, dtype)
    for r, g in enumerate(GATES):
        if g is not None:
            a[r], b[r] = g
    return q, k, v, a, b


@pytest.mark.parametrize("d", [128, 64], ids=["d128", "d64"])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F32])
@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("variant", [None, "stream", "column"])
def test_boundary_gates_match_oracle_and_closed_forms(torch_cuda, variant, T, dtype, d):
    if variant == "stream" and (T != 1 or d != 128):
        pytest.skip("the bulk-copy kernel serves single-token calls at dk = dv = 128")
    if variant is not None and d != 128:
        pytest.skip("one head size per pinned kernel is enough")
    rng = np.random.default_rng(1000 + 10 * T + (d == 64) + 2 * (dtype == wl.F32))
    Hk, Hv = 2, 4
    B = len(GATES)
    num_slots = B * (T + 1) + 3
    pool = wl.init_pool(rng, num_slots, Hv, d, d)
    q, k, v, a, b = _boundary_step(rng, T, Hk, Hv, d, dtype)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = src.reshape(B, 1).copy() if T == 1 else perm[B:B + B * T].reshape(B, T).copy()
    s = wl.Step(q, k, v, a, b, src, dst)
    dev = to_torch(pool)
    out = run_gpu(dev, s, variant=variant)
    got = dev.cpu().numpy()
    ref_pool, ref_out, skipped = run_oracle(pool, s)
    assert skipped == 0
    check_pool(got, ref_pool, pool, dst)
    assert rel_err(out, ref_out) <= (TOL_OUT_BF16 if dtype == wl.BF16 else TOL_OUT_F32)

    G = Hv // Hk
    kf, vf = _as_f64(k), _as_f64(v)
    for t in range(T):
        # identity: the stored tile is the source tile, bit for bit, at every token
        assert np.array_equal(got[dst[0, t]].view(np.uint32), pool[src[0]].view(np.uint32))
        # reset
        assert not np.any(got[dst[1, t]]) and not np.any(out[1, t])
        # pure write: M'[i][j] = k_i v_j, one rounded product per element
        for h in range(Hv):
            want = (kf[3, t, h // G][:, None] * vf[3, t, h][None, :]).astype(np.float32)
            assert np.array_equal(got[dst[3, t], h], want), (t, h)
        # retrieval: S' k = v for a key of unit norm (fp32 keys are normalised in fp32)
        if dtype == wl.F32:
            for h in range(Hv):
                Sk = got[dst[2, t], h].astype(np.float64).T @ kf[2, t, h // G]
                assert np.max(np.abs(Sk - vf[2, t, h])) <= 1e-5 * max(1.0, np.max(np.abs(vf[2, t, h]))), (t, h)


def _poison(s, T):
    """Non-finite values in three requests' inputs; returns the poisoned step and the set of
    (request, value head) units whose inputs hold them."""
    q, k, v, a = s.q.copy(), s.k.copy(), s.v.copy(), s.alpha.copy()
    nan = BF16_NAN if k.dtype == np.uint16 else np.float32(np.nan)
    G = s.Hv // s.Hk
    k[1, 0, 0, 7] = nan                 # key head 0 of request 1: value heads 0 .. G-1
    a[3, T - 1, 2] = np.inf             # last token of request 3, value head 2
    v[4, 0, 1, 3] = nan                 # request 4, value head 1
    q[5, T - 1, 1, 0] = nan             # query of request 5, key head 1 (outputs only)
    bad_state = {(1, h) for h in range(G)} | {(3, 2), (4, 1)}
    bad_out = bad_state | {(5, h) for h in range(G, 2 * G)}
    return wl.Step(q, k, v, a, s.beta, s.src_idx, s.dst_idx), bad_state, bad_out


@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("variant", [None, "stream", "column"])
def test_non_finite_inputs_stay_in_their_units(torch_cuda, variant, T):
    if variant == "stream" and T != 1:
        pytest.skip("the bulk-copy kernel serves single-token calls")
    rng = np.random.default_rng(1100 + T)
    B, Hk, Hv, d = 7, 2, 4, 128
    num_slots = B * (T + 1) + 5
    pool = wl.init_pool(rng, num_slots, Hv, d, d)
    q, k, v, a, b = wl.random_step_inputs(rng, B, T, Hk, Hv, d, d, wl.BF16)
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    dst = src.reshape(B, 1).copy() if T == 1 else perm[B:B + B * T].reshape(B, T).copy()
    clean = wl.Step(q, k, v, a, b, src, dst)
    bad, bad_state, bad_out = _poison(clean, T)
    dev_c, dev_p = to_torch(pool), to_torch(pool)
    out_c = run_gpu(dev_c, clean, variant=variant)
    out_p = run_gpu(dev_p, bad, variant=variant)
    got_c, got_p = dev_c.cpu().numpy(), dev_p.cpu().numpy()
    assert np.isnan(out_p[1]).any() and not np.isfinite(out_p[3, T - 1, 2]).all()
    for r in range(B):
        for h in range(Hv):
            if (r, h) not in bad_out:
                assert np.array_equal(out_p[r, :, h].view(np.uint32), out_c[r, :, h].view(np.uint32)), (r, h)
            if (r, h) not in bad_state:
                for t in range(T):
                    assert np.array_equal(got_p[dst[r, t], h].view(np.uint32), got_c[dst[r, t], h].view(np.uint32))
    untouched = np.setdiff1d(np.arange(num_slots), dst.ravel())
    assert np.array_equal(got_p[untouched].view(np.uint32), pool[untouched].view(np.uint32))
    # the clean run itself is the oracle's
    ref_pool, ref_out, _ = run_oracle(pool, clean)
    check_pool(got_c, ref_pool, pool, dst)
    assert rel_err(out_c, ref_out) <= TOL_OUT_BF16


@pytest.mark.parametrize("chunked", [False, True], ids=["token_steps", "chunked"])
def test_non_finite_prefill_inputs_stay_in_their_units(torch_cuda, chunked):
    """The same containment for the prefill: a NaN key in the middle of one request's
    prompt and an infinite gate in another's reach only their own (request, head) units."""
    torch = torch_cuda
    from hybrid_linear_attention_step_b200 import gdn

    rng = np.random.default_rng(1200 + chunked)
    B, L, Hk, Hv, d = 4, 150, 2, 4, 128
    pool = wl.init_pool(rng, 2 * B, Hv, d, d)
    q, k, v, a, b = wl.random_step_inputs(rng, B, L, Hk, Hv, d, d, wl.BF16)
    kp, ap = k.copy(), a.copy()
    kp[1, 70, 1, 5] = BF16_NAN        # request 1, key head 1 -> value heads 2, 3 from token 70
    ap[2, 100, 0] = np.inf            # request 2, value head 0 from token 100
    bad = {(1, 2), (1, 3), (2, 0)}
    src = np.arange(B, dtype=np.int32)
    dst = np.arange(B, 2 * B, dtype=np.int32)
    outs, pools = [], []
    for kk, aa in ((k, a), (kp, ap)):
        x = step_to_device(wl.Step(q, kk, v, aa, b, src, dst.reshape(B, 1)))
        dev = to_torch(pool)
        out = torch.full((B, L, Hv, d), -7.0, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        args = (dev, x["src"], to_torch(dst), x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
        if chunked:
            ws = torch.empty(gdn.gdn_prefill_workspace_bytes(B, L, Hv, d, d), dtype=torch.uint8, device="cuda")
            gdn.gdn_prefill_chunked(*args, ws, err_word=err)
        else:
            gdn.gdn_prefill(*args, err_word=err)
        assert gdn.gdn_get_error(err) == gdn.GDN_OK
        outs.append(out.cpu().numpy())
        pools.append(dev.cpu().numpy())
    (out_c, out_p), (pool_c, pool_p) = outs, pools
    assert np.isnan(out_p[1, 70:, 2:]).any() and not np.isfinite(out_p[2, 100:, 0]).all()
    for r in range(B):
        for h in range(Hv):
            if (r, h) in bad:
                continue
            assert np.array_equal(out_p[r, :, h].view(np.uint32), out_c[r, :, h].view(np.uint32)), (r, h)
            assert np.array_equal(pool_p[dst[r], h].view(np.uint32), pool_c[dst[r], h].view(np.uint32)), (r, h)
    # Outputs before the poisoned token keep their bits.  The chunked form solves a chunk's
    # tokens together (a NaN key turns its chunk's products NaN), so there the guarantee
    # starts at the chunk that holds the token: 64-token chunks, token 70 in the second.
    first = 64 if chunked else 70
    assert np.array_equal(out_p[1, :first].view(np.uint32), out_c[1, :first].view(np.uint32))
    assert np.array_equal(pool_p[:B].view(np.uint32), pool[:B].view(np.uint32))  # sources are only read
