"""Pins for the CPU oracle against what the mathematics fixes (no GPU).

None of these re-uses the oracle's own formulation (the explicit product
alpha * S * (I - beta k k^T) + beta * v k^T): they check closed forms, a
hand-derived worked example, an independent rank-one restatement, structural
invariants of the slot scheme, and brute force.  A dropped term, a wrong sign,
a transposed state or a wrong key-head map each fails at least one of them.
"""
import numpy as np
import pytest

import oracle
from hybrid_linear_attention_step_b200 import workloads as wl


def _inputs(rng, B, T, Hk, Hv, dk, dv, dtype=wl.F32):
    return wl.random_step_inputs(rng, B, T, Hk, Hv, dk, dv, dtype)


def _run(pool, src, dst, q, k, v, a, b, nthreads=1):
    pool = pool.copy()
    B, T = q.shape[0], q.shape[1]
    out = np.full((B, T, v.shape[2], v.shape[3]), np.float32(-7.0), np.float32)
    skipped = oracle.decode_step(pool, np.asarray(src, np.int32), np.asarray(dst, np.int32).reshape(B, T),
                                 q, k, v, a, b, out, nthreads=nthreads)
    return pool, out, skipped


def _full(shape, val):
    return np.full(shape, np.float32(val), np.float32)


# ---------------------------------------------------------------- closed forms

def test_identity_gate_keeps_state_and_reads_out_matvec():
    """alpha = 1, beta = 0: S' = S bit for bit, and o = S q (a plain mat-vec)."""
    rng = np.random.default_rng(10)
    Hv, dk, dv = 3, 16, 8
    pool = wl.init_pool(rng, 4, Hv, dk, dv)
    q, k, v, _, _ = _inputs(rng, 1, 1, Hv, Hv, dk, dv)
    new, out, _ = _run(pool, [1], [2], q, k, v, _full((1, 1, Hv), 1.0), _full((1, 1, Hv), 0.0))
    assert np.array_equal(new[2].view(np.uint32), pool[1].view(np.uint32))
    for h in range(Hv):
        S = pool[1, h].astype(np.float64).T            # stored [dk][dv] is S transposed
        ref = S @ q[0, 0, h].astype(np.float64)
        np.testing.assert_allclose(out[0, 0, h], ref, rtol=1e-6, atol=1e-9)


def test_zero_gates_reset_state_and_output():
    """alpha = 0, beta = 0: the state resets to zero and so does o (value equality)."""
    rng = np.random.default_rng(11)
    pool = wl.init_pool(rng, 3, 2, 16, 16)
    q, k, v, _, _ = _inputs(rng, 1, 1, 2, 2, 16, 16)
    new, out, _ = _run(pool, [0], [0], q, k, v, _full((1, 1, 2), 0.0), _full((1, 1, 2), 0.0))
    assert np.all(new[0] == 0.0)
    assert np.all(out == 0.0)
    assert np.array_equal(new[1:], pool[1:])


@pytest.mark.parametrize("axis_k", [True, False])
def test_delta_rule_retrieval(axis_k):
    """alpha = 1, beta = 1, |k| = 1: the updated state maps k exactly to v (S'k = v)."""
    rng = np.random.default_rng(12)
    dk, dv = 16, 16
    pool = wl.init_pool(rng, 2, 1, dk, dv)
    q, k, v, _, _ = _inputs(rng, 1, 1, 1, 1, dk, dv)
    if axis_k:
        k = np.zeros_like(k)
        k[0, 0, 0, 5] = 1.0
    new, _, _ = _run(pool, [0], [1], q, k, v, _full((1, 1, 1), 1.0), _full((1, 1, 1), 1.0))
    S_new = new[1, 0].astype(np.float64).T
    kd = k[0, 0, 0].astype(np.float64)
    got = S_new @ kd
    want = v[0, 0, 0].astype(np.float64)
    # |k|^2 = 1 up to fp32 normalisation error; S' is stored in fp32.
    np.testing.assert_allclose(got, want, rtol=0, atol=2e-6 * np.abs(want).max())


def test_pure_write_is_outer_product():
    """alpha = 0, beta = 1: S' = v k^T exactly (one fp32 product), o = v (k . q)."""
    rng = np.random.default_rng(13)
    dk, dv = 16, 12
    pool = wl.init_pool(rng, 2, 1, dk, dv)
    q, k, v, _, _ = _inputs(rng, 1, 1, 1, 1, dk, dv)
    new, out, _ = _run(pool, [0], [1], q, k, v, _full((1, 1, 1), 0.0), _full((1, 1, 1), 1.0))
    kk, vv, qq = k[0, 0, 0], v[0, 0, 0], q[0, 0, 0]
    outer = (kk[:, None] * vv[None, :]).astype(np.float32)  # stored [dk][dv]: M[i][j] = v_j k_i
    assert np.array_equal(new[1, 0], outer)
    want = vv.astype(np.float64) * float(np.dot(kk.astype(np.float64), qq.astype(np.float64)))
    np.testing.assert_allclose(out[0, 0, 0], want, rtol=1e-6, atol=1e-7)


def test_decay_only_scales_state():
    """beta = 0 for three tokens with alpha = 1/2: S''' = S / 8 bit for bit (exact scaling)."""
    rng = np.random.default_rng(14)
    pool = wl.init_pool(rng, 5, 2, 16, 16)
    q, k, v, _, _ = _inputs(rng, 1, 3, 2, 2, 16, 16)
    new, _, _ = _run(pool, [0], [[1, 2, 3]], q, k, v, _full((1, 3, 2), 0.5), _full((1, 3, 2), 0.0))
    assert np.array_equal(new[1], pool[0] * np.float32(0.5))
    assert np.array_equal(new[2], pool[0] * np.float32(0.25))
    assert np.array_equal(new[3], pool[0] * np.float32(0.125))


def test_orthonormal_keys_store_independent_associations():
    """alpha = beta = 1 with orthonormal keys k0, k1 over two tokens: S'' k0 = v0 and S'' k1 = v1."""
    rng = np.random.default_rng(15)
    dk, dv = 16, 16
    pool = wl.init_pool(rng, 3, 1, dk, dv)
    q, k, v, _, _ = _inputs(rng, 1, 2, 1, 1, dk, dv)
    k = np.zeros_like(k)
    k[0, 0, 0, 3] = 1.0
    k[0, 1, 0, 9] = 1.0
    new, _, _ = _run(pool, [0], [[1, 2]], q, k, v, _full((1, 2, 1), 1.0), _full((1, 2, 1), 1.0))
    S2 = new[2, 0].astype(np.float64).T
    np.testing.assert_array_equal(S2[:, 3], v[0, 0, 0].astype(np.float64))
    np.testing.assert_array_equal(S2[:, 9], v[0, 1, 0].astype(np.float64))
    # Columns of S for keys never written keep the (undecayed) old state.
    S0 = pool[0, 0].astype(np.float64).T
    np.testing.assert_array_equal(S2[:, 0], S0[:, 0])


# ------------------------------------------------------ hand-derived examples

def test_worked_example_2x2():
    """Worked by hand: S = [[1, 2], [3, 4]], k = (1/2, 1/2), v = (1, -2), q = (1, 2), alpha = beta = 1.

    I - k k^T = [[3/4, -1/4], [-1/4, 3/4]];  S (I - k k^T) = [[1/4, 5/4], [5/4, 9/4]];
    v k^T = [[1/2, 1/2], [-1, -1]];  S' = [[3/4, 7/4], [1/4, 5/4]];  o = S' q = (17/4, 11/4).
    Stored layout is S transposed.
    """
    pool = np.zeros((2, 1, 2, 2), np.float32)
    pool[0, 0] = np.array([[1, 2], [3, 4]], np.float32).T
    f = lambda *x: np.array(x, np.float32).reshape(1, 1, 1, -1)
    new, out, _ = _run(pool, [0], [1], f(1, 2), f(0.5, 0.5), f(1, -2), _full((1, 1, 1), 1.0),
                       _full((1, 1, 1), 1.0))
    np.testing.assert_array_equal(new[1, 0].T, np.array([[0.75, 1.75], [0.25, 1.25]], np.float32))
    np.testing.assert_array_equal(out[0, 0, 0], np.array([4.25, 2.75], np.float32))
    np.testing.assert_array_equal(new[0], pool[0])


def test_worked_example_non_square():
    """Worked by hand with dk = 3, dv = 2: S = [[1, 0, 2], [0, 1, -1]], k = e_1, v = (4, 8),
    q = (1, 1, 1), alpha = 2, beta = 1/2.

    I - k k^T / 2 = diag(1, 1/2, 1);  2 S diag(1, 1/2, 1) = [[2, 0, 4], [0, 1, -2]];
    v k^T / 2 = [[0, 2, 0], [0, 4, 0]];  S' = [[2, 2, 4], [0, 5, -2]];  o = (8, 3).
    """
    pool = np.zeros((2, 1, 3, 2), np.float32)
    pool[0, 0] = np.array([[1, 0, 2], [0, 1, -1]], np.float32).T
    f = lambda *x: np.array(x, np.float32).reshape(1, 1, 1, -1)
    new, out, _ = _run(pool, [0], [1], f(1, 1, 1), f(0, 1, 0), f(4, 8), _full((1, 1, 1), 2.0),
                       _full((1, 1, 1), 0.5))
    np.testing.assert_array_equal(new[1, 0], np.array([[2, 0], [2, 5], [4, -2]], np.float32))
    np.testing.assert_array_equal(out[0, 0, 0], np.array([8, 3], np.float32))


# ------------------------------------------- independent rank-one restatement

def _rank_one_reference(S0, q, k, v, alpha, beta):
    """S' = alpha S + c k^T with c = beta (v - alpha S k); carried in fp32; o = S' q.

    S0 is the logical state [dv][dk] (float64). q, k, v are per-token vectors.
    """
    S = S0.copy()
    states, outs = [], []
    for t in range(len(alpha)):
        u = S @ k[t]
        c = beta[t] * (v[t] - alpha[t] * u)
        S = alpha[t] * S + np.outer(c, k[t])
        S = S.astype(np.float32).astype(np.float64)
        states.append(S.copy())
        outs.append(S @ q[t])
    return states, outs


@pytest.mark.parametrize("dk,dv,Hk,Hv,T", [(1, 1, 1, 1, 1), (2, 3, 1, 2, 2), (3, 2, 2, 2, 3),
                                           (16, 16, 1, 2, 2), (3, 16, 2, 4, 1), (16, 1, 1, 1, 3)])
def test_matches_rank_one_form(dk, dv, Hk, Hv, T):
    rng = np.random.default_rng(100 + dk * 7 + dv + T)
    B, num_slots = 2, 2 * (T + 1)
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv, std=0.5)
    q, k, v, a, b = _inputs(rng, B, T, Hk, Hv, dk, dv)
    src = np.array([0, 1], np.int32)
    dst = np.arange(2, 2 + B * T, dtype=np.int32).reshape(B, T)
    new, out, skipped = _run(pool, src, dst, q, k, v, a, b)
    assert skipped == 0
    G = Hv // Hk
    for bi in range(B):
        for h in range(Hv):
            hk = h // G
            states, outs = _rank_one_reference(
                pool[src[bi], h].astype(np.float64).T,
                q[bi, :, hk].astype(np.float64), k[bi, :, hk].astype(np.float64),
                v[bi, :, h].astype(np.float64), a[bi, :, h].astype(np.float64), b[bi, :, h].astype(np.float64))
            for t in range(T):
                np.testing.assert_allclose(new[dst[bi, t], h].astype(np.float64).T, states[t],
                                           rtol=2e-6, atol=1e-7)
                np.testing.assert_allclose(out[bi, t, h].astype(np.float64), outs[t], rtol=2e-6, atol=1e-6)


# ------------------------------------------------------- slot-scheme invariants

def test_copy_on_write_leaves_sources_byte_identical():
    """Shared source slots are read, never written; every slot outside dst keeps its bytes."""
    rng = np.random.default_rng(20)
    num_slots, B, Hk, Hv, dk, dv = 12, 6, 2, 4, 16, 16
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv)
    src = np.array([1, 1, 1, 4, 4, 7], np.int32)
    dst = np.array([0, 2, 3, 5, 6, 8], np.int32)
    q, k, v, a, b = _inputs(rng, B, 1, Hk, Hv, dk, dv, wl.BF16)
    new, _, _ = _run(pool, src, dst, q, k, v, a, b)
    untouched = np.setdiff1d(np.arange(num_slots), dst)
    assert np.array_equal(new[untouched].view(np.uint32), pool[untouched].view(np.uint32))
    for d in dst:
        assert not np.array_equal(new[d], pool[d])
    # Requests that share a source see the same pre-call state: same inputs, same result.
    q2, k2, v2, a2, b2 = (x.copy() for x in (q, k, v, a, b))
    for x in (q2, k2, v2, a2, b2):
        x[1] = x[0]
    new2, out2, _ = _run(pool, src, dst, q2, k2, v2, a2, b2)
    assert np.array_equal(new2[dst[0]], new2[dst[1]])
    assert np.array_equal(out2[0], out2[1])


def test_reads_see_pre_call_state():
    """A request whose source is another request's destination reads the pre-call bytes."""
    rng = np.random.default_rng(21)
    pool = wl.init_pool(rng, 4, 1, 16, 16)
    q, k, v, a, b = _inputs(rng, 2, 1, 1, 1, 16, 16)
    both, out_both, _ = _run(pool, [0, 1], [1, 2], q, k, v, a, b)
    alone, out_alone, _ = _run(pool, [1], [2], q[1:], k[1:], v[1:], a[1:], b[1:])
    assert np.array_equal(both[2], alone[2])
    assert np.array_equal(out_both[1], out_alone[0])


def test_in_place_update_equals_out_of_place():
    rng = np.random.default_rng(22)
    pool = wl.init_pool(rng, 4, 2, 16, 16)
    q, k, v, a, b = _inputs(rng, 1, 1, 1, 2, 16, 16)
    inplace, o1, _ = _run(pool, [2], [2], q, k, v, a, b)
    moved, o2, _ = _run(pool, [2], [3], q, k, v, a, b)
    assert np.array_equal(inplace[2], moved[3])
    assert np.array_equal(o1, o2)


def test_sequential_equals_speculative():
    """T single-token calls chained src -> d0 -> d1 -> d2 equal one T = 3 call with cur = [d0, d1, d2]."""
    rng = np.random.default_rng(23)
    num_slots, B, T, Hk, Hv, dk, dv = 10, 2, 3, 1, 2, 16, 8
    pool = wl.init_pool(rng, num_slots, Hv, dk, dv)
    q, k, v, a, b = _inputs(rng, B, T, Hk, Hv, dk, dv, wl.BF16)
    src = np.array([0, 1], np.int32)
    cur = np.array([[2, 3, 4], [5, 6, 7]], np.int32)
    spec, out_spec, _ = _run(pool, src, cur, q, k, v, a, b)
    seq = pool.copy()
    out_seq = np.zeros_like(out_spec)
    prev = src.copy()
    for t in range(T):
        seq, o, _ = _run(seq, prev, cur[:, t].copy(), *(np.ascontiguousarray(x[:, t:t + 1]) for x in (q, k, v, a, b)))
        out_seq[:, t] = o[:, 0]
        prev = cur[:, t].copy()
    assert np.array_equal(spec.view(np.uint32), seq.view(np.uint32))
    assert np.array_equal(out_spec, out_seq)


def test_slot_relabelling_permutes_results():
    """Renaming slots through a permutation renames the result exactly (indirection is pure)."""
    rng = np.random.default_rng(24)
    num_slots, B = 9, 3
    pool = wl.init_pool(rng, num_slots, 2, 16, 16)
    q, k, v, a, b = _inputs(rng, B, 2, 1, 2, 16, 16)
    src = np.array([0, 3, 3], np.int32)
    dst = np.array([[1, 2], [4, 5], [6, 7]], np.int32)
    ref, out_ref, _ = _run(pool, src, dst, q, k, v, a, b)
    sigma = rng.permutation(num_slots).astype(np.int32)
    pool_p = np.empty_like(pool)
    pool_p[sigma] = pool
    got, out_got, _ = _run(pool_p, sigma[src], sigma[dst], q, k, v, a, b)
    assert np.array_equal(got[sigma].view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(out_got, out_ref)


def test_grouped_key_heads_are_contiguous():
    """Hv = 4 value heads over Hk = 2 key heads: heads 0, 1 read key head 0 and heads 2, 3 key head 1."""
    rng = np.random.default_rng(25)
    pool = wl.init_pool(rng, 4, 4, 16, 16)
    q, k, v, a, b = _inputs(rng, 2, 1, 2, 4, 16, 16)
    grouped, out_g, _ = _run(pool, [0, 1], [2, 3], q, k, v, a, b)
    qe, ke = (np.ascontiguousarray(np.repeat(x, 2, axis=2)) for x in (q, k))
    expanded, out_e, _ = _run(pool, [0, 1], [2, 3], qe, ke, v, a, b)
    assert np.array_equal(grouped, expanded)
    assert np.array_equal(out_g, out_e)
    qi, ki = (np.ascontiguousarray(np.tile(x, (1, 1, 2, 1))) for x in (q, k))  # the h mod Hk map
    wrong, _, _ = _run(pool, [0, 1], [2, 3], qi, ki, v, a, b)
    assert not np.array_equal(grouped, wrong)


def test_out_of_range_index_skips_request():
    rng = np.random.default_rng(26)
    pool = wl.init_pool(rng, 6, 1, 16, 16)
    q, k, v, a, b = _inputs(rng, 3, 2, 1, 1, 16, 16)
    src = np.array([0, 6, 1], np.int32)           # request 1: source out of range
    dst = np.array([[2, 3], [4, 5], [-1, 4]], np.int32)  # request 2: a destination out of range
    new, out, skipped = _run(pool, src, dst, q, k, v, a, b)
    assert skipped == 2
    assert np.array_equal(new[[0, 1, 4, 5]], pool[[0, 1, 4, 5]])
    assert np.all(out[1:] == -7.0)
    good, out_good, _ = _run(pool, src[:1], dst[:1], q[:1], k[:1], v[:1], a[:1], b[:1])
    assert np.array_equal(new, good)
    assert np.array_equal(out[0], out_good[0])


def test_padding_requests_are_skipped_silently():
    """src = -1 marks padding: nothing is read or written and it is not an error,
    whatever its destination entries hold; other negative sources are errors."""
    rng = np.random.default_rng(29)
    pool = wl.init_pool(rng, 6, 1, 16, 16)
    q, k, v, a, b = _inputs(rng, 3, 2, 1, 1, 16, 16)
    src = np.array([0, -1, -2], np.int32)
    dst = np.array([[2, 3], [99, -5], [4, 5]], np.int32)
    new, out, skipped = _run(pool, src, dst, q, k, v, a, b)
    assert skipped == 1  # only the -2 source counts
    assert np.all(out[1:] == -7.0)
    alone, out_alone, _ = _run(pool, src[:1], dst[:1], q[:1], k[:1], v[:1], a[:1], b[:1])
    assert np.array_equal(new, alone) and np.array_equal(out[0], out_alone[0])


def test_bf16_inputs_widen_exactly():
    """bf16 inputs give the same result as their exactly widened fp32 values."""
    rng = np.random.default_rng(27)
    pool = wl.init_pool(rng, 4, 2, 16, 16)
    q, k, v, a, b = _inputs(rng, 2, 1, 1, 2, 16, 16, wl.BF16)
    r16, o16, _ = _run(pool, [0, 1], [2, 3], q, k, v, a, b)
    r32, o32, _ = _run(pool, [0, 1], [2, 3], *(wl.bf16_bits_to_f32(x) for x in (q, k, v)), a, b)
    assert np.array_equal(r16, r32)
    assert np.array_equal(o16, o32)


def test_bf16_rounding_known_values():
    x = np.array([1.0, -2.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 3.140625, 0.0], np.float32)
    bits = wl.f32_to_bf16_bits(x)
    assert list(bits) == [0x3F80, 0xC000, 0x3F80, 0x3F82, 0x4049, 0x0000]
    assert list(wl.bf16_bits_to_f32(bits)) == [1.0, -2.0, 1.0, 1 + 2 ** -6, 3.140625, 0.0]


def test_threads_do_not_change_results():
    rng = np.random.default_rng(28)
    pool = wl.init_pool(rng, 16, 2, 16, 16)
    q, k, v, a, b = _inputs(rng, 5, 2, 1, 2, 16, 16, wl.BF16)
    dst = np.arange(5, 15, dtype=np.int32).reshape(5, 2)
    r1, o1, _ = _run(pool, np.arange(5, dtype=np.int32), dst, q, k, v, a, b, nthreads=1)
    r4, o4, _ = _run(pool, np.arange(5, dtype=np.int32), dst, q, k, v, a, b, nthreads=4)
    assert np.array_equal(r1, r4) and np.array_equal(o1, o4)


def test_empty_batch_is_a_no_op():
    pool = np.ones((2, 1, 4, 4), np.float32)
    z = np.zeros((0, 1, 1, 4), np.float32)
    out = np.zeros((0, 1, 1, 4), np.float32)
    ab = np.zeros((0, 1, 1), np.float32)
    assert oracle.decode_step(pool, np.zeros(0, np.int32), np.zeros((0, 1), np.int32), z, z, z, ab, ab, out) == 0
    assert np.all(pool == 1.0)


# ------------------------------------------------------------------- commit

def _commit_brute(accept, committed, cur, num_slots):
    committed = committed.copy()
    bad = 0
    for b_ in range(len(accept)):
        a_ = int(accept[b_])
        if not 0 <= a_ <= cur.shape[1]:
            bad += 1
        elif a_ > 0:
            s = int(cur[b_, a_ - 1])
            if 0 <= s < num_slots:
                committed[b_] = s
            else:
                bad += 1
    return committed, bad


def test_commit_matches_brute_force_and_is_idempotent():
    rng = np.random.default_rng(30)
    B, T, num_slots = 64, 4, 1024
    cur = rng.integers(0, num_slots, size=(B, T)).astype(np.int32)
    cur[5, 1] = num_slots + 3
    accept = rng.integers(0, T + 1, size=B).astype(np.int32)
    accept[5], accept[7], accept[9] = 2, -1, T + 1
    committed0 = rng.integers(0, num_slots, size=B).astype(np.int32)
    want, bad_want = _commit_brute(accept, committed0, cur, num_slots)
    got = committed0.copy()
    assert oracle.commit(accept, got, cur, num_slots) == bad_want == 3
    assert np.array_equal(got, want)
    again = got.copy()
    oracle.commit(accept, again, cur, num_slots)
    assert np.array_equal(again, got)
    zero = np.zeros(B, np.int32)
    kept = committed0.copy()
    oracle.commit(zero, kept, cur, num_slots)
    assert np.array_equal(kept, committed0)


# ------------------------------------------------------- precondition check

def _check_brute(src, dst, num_slots):
    """The preconditions restated over explicit sets."""
    B, T = dst.shape
    live = [b for b in range(B) if src[b] != -1]
    if any(not 0 <= src[b] < num_slots or not all(0 <= d < num_slots for d in dst[b]) for b in live):
        return 3
    writes = [(int(d), b) for b in live for d in dst[b]]
    if len({d for d, _ in writes}) != len(writes):
        return 5
    for b in live:
        for d, w in writes:
            if d == src[b] and (w != b or T > 1):
                return 5
    return 0


@pytest.mark.parametrize("T", [1, 3])
def test_check_step_matches_brute_force(T):
    rng = np.random.default_rng(31 + T)
    seen = set()
    for trial in range(400):
        num_slots = int(rng.integers(4, 24))
        B = int(rng.integers(0, 6))
        src = rng.integers(-2, num_slots + 1, size=B).astype(np.int32)
        dst = rng.integers(-1, num_slots + 1, size=(B, T)).astype(np.int32)
        if trial % 3 == 0 and B:  # mostly-valid cases: distinct fresh destinations
            perm = rng.permutation(num_slots + B * T + B)[: B + B * T] % num_slots
            src = perm[:B].astype(np.int32)
            dst = perm[B:].reshape(B, T).astype(np.int32)
        want = _check_brute(src, dst, num_slots)
        assert oracle.check_step(src, dst, num_slots) == want
        seen.add(want)
    assert seen == {0, 3, 5}


def test_check_step_named_cases():
    ok = lambda s, d, n=10: oracle.check_step(np.array(s, np.int32), np.array(d, np.int32).reshape(len(s), -1), n)
    assert ok([1, 2], [[1], [2]]) == 0          # in place, T = 1
    assert ok([1, 1], [[3], [4]]) == 0          # shared source (copy-on-write)
    assert ok([1, 2], [[3], [3]]) == 5          # two writes to one slot
    assert ok([1, 2], [[2], [4]]) == 5          # writes another request's source
    assert ok([1, 2], [[1, 3], [4, 5]]) == 5    # T > 1 writes its own source
    assert ok([1, 2], [[3, 3], [4, 5]]) == 5    # duplicate within one request
    assert ok([-1, 2], [[2, 2], [4, 5]]) == 0   # padding rows are ignored
    assert ok([1, 2], [[3], [10]]) == 3         # out of range
    assert ok([1, 2], [[2], [10]]) == 3         # index error takes precedence over aliasing


# ------------------------------------------------------- fused prologue

def _run_fused(pool, src, dst, q, k, v, x, y, flags):
    pool = pool.copy()
    B, T = q.shape[0], q.shape[1]
    out = np.zeros((B, T, v.shape[2], v.shape[3]), np.float32)
    oracle.decode_step(pool, np.asarray(src, np.int32), np.asarray(dst, np.int32).reshape(B, T), q, k, v,
                       x, y, out, flags=flags)
    return pool, out


@pytest.mark.parametrize("x,alpha", [(0.0, 0.5), (np.log(3.0), 0.25), (-50.0, 1.0), (50.0, 0.0)])
@pytest.mark.parametrize("y,beta", [(0.0, 0.5), (np.log(3.0), 0.75), (50.0, 1.0), (-50.0, 0.0)])
def test_fused_gates_closed_forms(x, alpha, y, beta):
    """exp(-softplus(0)) = 1/2, exp(-softplus(ln 3)) = 1/4, sigmoid(ln 3) = 3/4, and the saturated ends."""
    rng = np.random.default_rng(40)
    pool = wl.init_pool(rng, 3, 2, 16, 16)
    q, k, v, _, _ = _inputs(rng, 1, 2, 1, 2, 16, 16)
    fused, of = _run_fused(pool, [0], [[1, 2]], q, k, v, _full((1, 2, 2), x), _full((1, 2, 2), y), oracle.FUSE_GATES)
    plain, op, _ = _run(pool, [0], [[1, 2]], q, k, v, _full((1, 2, 2), alpha), _full((1, 2, 2), beta))
    np.testing.assert_allclose(fused, plain, rtol=2e-6, atol=1e-9)
    np.testing.assert_allclose(of, op, rtol=2e-6, atol=1e-7)


def test_fused_norm_is_scale_invariant():
    """Normalising inside the step makes the result independent of the scale of q and k, and
    leaves already-unit q and k unchanged (to the 1e-6 epsilon)."""
    rng = np.random.default_rng(41)
    pool = wl.init_pool(rng, 4, 4, 16, 16)
    q, k, v, x, y = wl.random_raw_step_inputs(rng, 2, 1, 2, 4, 16, 16, wl.F32)
    src, dst = [0, 1], [[2], [3]]
    a_, oa = _run_fused(pool, src, dst, q, k, v, x, y, oracle.FUSE_GATES | oracle.FUSE_QK_NORM)
    b_, ob = _run_fused(pool, src, dst, (q * 7.0).astype(np.float32), (k * 0.3).astype(np.float32), v, x, y,
                        oracle.FUSE_GATES | oracle.FUSE_QK_NORM)
    np.testing.assert_allclose(a_, b_, rtol=2e-5, atol=1e-8)
    np.testing.assert_allclose(oa, ob, rtol=2e-5, atol=1e-6)
    # unit q and k (normalised in double, rounded to fp32), gates given directly
    qn = (q / np.linalg.norm(q.astype(np.float64), axis=-1, keepdims=True)).astype(np.float32)
    kn = (k / np.linalg.norm(k.astype(np.float64), axis=-1, keepdims=True)).astype(np.float32)
    alpha, beta = _full((2, 1, 4), 0.75), _full((2, 1, 4), 0.5)
    c_, oc = _run_fused(pool, src, dst, qn, kn, v, alpha, beta, oracle.FUSE_QK_NORM)
    d_, od, _ = _run(pool, src, dst, qn, kn, v, alpha, beta)
    np.testing.assert_allclose(c_, d_, rtol=1e-5, atol=1e-6 * float(np.abs(d_).max()))
    np.testing.assert_allclose(oc, od, rtol=1e-5, atol=1e-7)


def test_fused_norm_retrieval_of_unnormalised_key():
    """Raw k = (3, 4, 0, ...), saturated gates (alpha = 1, beta = 1): S' (k / 5) = v."""
    rng = np.random.default_rng(42)
    dk, dv = 16, 16
    pool = wl.init_pool(rng, 2, 1, dk, dv)
    q, _, v, _, _ = _inputs(rng, 1, 1, 1, 1, dk, dv)
    k = np.zeros((1, 1, 1, dk), np.float32)
    k[0, 0, 0, :2] = (3.0, 4.0)
    new, _ = _run_fused(pool, [0], [[1]], q, k, v, _full((1, 1, 1), -60.0), _full((1, 1, 1), 60.0), 3)
    got = new[1, 0].astype(np.float64).T @ (k[0, 0, 0].astype(np.float64) / 5.0)
    np.testing.assert_allclose(got, v[0, 0, 0].astype(np.float64), rtol=0, atol=2e-6 * np.abs(v).max())


# ------------------------------------------------------------------ prefill

def test_prefill_equals_chained_single_token_calls():
    """A prefill over L tokens ends in the state, bit for bit, that L chained single-token calls
    reach, emits the same outputs, and writes nothing but its destination slot."""
    rng = np.random.default_rng(43)
    B, L, Hk, Hv, dk, dv = 2, 5, 1, 2, 16, 8
    pool = wl.init_pool(rng, 6, Hv, dk, dv)
    q, k, v, a, b = _inputs(rng, B, L, Hk, Hv, dk, dv, wl.BF16)
    src = np.array([0, 1], np.int32)
    dst = np.array([2, 1], np.int32)            # request 1 continues in place
    pre = pool.copy()
    out = np.zeros((B, L, Hv, dv), np.float32)
    assert oracle.prefill(pre, src, dst, q, k, v, a, b, out) == 0
    chain = pool.copy()
    for bi in range(B):
        cur = int(src[bi])
        for t in range(L):
            nxt = [4, 5][t % 2]                 # scratch slots
            sl = lambda x: np.ascontiguousarray(x[bi:bi + 1, t:t + 1])
            chain, o, _ = _run(chain, [cur], [[nxt]], sl(q), sl(k), sl(v), sl(a), sl(b))
            assert np.array_equal(o[0, 0], out[bi, t])
            cur = nxt
        assert np.array_equal(pre[dst[bi]].view(np.uint32), chain[cur].view(np.uint32))
    untouched = [0, 3, 4, 5]
    assert np.array_equal(pre[untouched].view(np.uint32), pool[untouched].view(np.uint32))
