"""Seeded inputs: determinism, the slot structure each workload promises, and the golden fixture."""
import numpy as np

import oracle
from hybrid_linear_attention_step_b200 import workloads as wl
from tests.golden import make_golden


def test_seeded_generation_is_deterministic():
    a, b = wl.decode_b16(1), wl.decode_b16(1)
    s, t = a.steps[0], b.steps[0]
    for x, y in ((s.q, t.q), (s.v, t.v), (s.alpha, t.alpha), (s.src_idx, t.src_idx)):
        assert np.array_equal(x, y)
    assert np.array_equal(a.pool, b.pool)
    assert not np.array_equal(wl.decode_b16(2).steps[0].q, s.q)


def test_input_distributions():
    w = wl.decode_b16(1)
    s = w.steps[0]
    assert s.q.dtype == np.uint16 and s.q.shape == (16, 1, 16, 128) and s.v.shape == (16, 1, 32, 128)
    n = np.linalg.norm(wl.bf16_bits_to_f32(s.k).astype(np.float64), axis=-1)
    assert np.all(np.abs(n - 1) < 1e-2)
    assert np.all((s.alpha > 0) & (s.alpha < 1)) and np.all((s.beta > 0) & (s.beta < 1))
    assert abs(float(w.pool.std()) - wl.STATE_STD) < 1e-3
    assert np.array_equal(s.src_idx, s.dst_idx[:, 0]) and len(set(s.src_idx.tolist())) == 16


def test_tiny_chain():
    w = wl.tiny(0)
    assert [int(s.src_idx[0]) for s in w.steps] == [0, 1, 2, 3, 0, 1, 2, 3]
    assert [int(s.dst_idx[0, 0]) for s in w.steps] == [1, 2, 3, 0, 1, 2, 3, 0]
    assert w.steps[0].q.dtype == np.float32


def test_prefix_cow_structure():
    s = wl.prefix_cow(2).steps[0]
    src, dst = s.src_idx, s.dst_idx[:, 0]
    vals, counts = np.unique(src, return_counts=True)
    assert int(counts[counts >= 2].sum()) == 115 and int((counts == 1).sum()) == 13
    assert counts.max() <= 16
    assert len(set(dst.tolist())) == 128 and not set(dst.tolist()) & set(src.tolist())


def test_share_groups_never_leave_singletons():
    rng = np.random.default_rng(0)
    for _ in range(200):
        g = wl.share_groups(rng, int(rng.integers(2, 300)))
        assert min(g) >= 2 and max(g) <= 16


def test_speculative_structure():
    s = wl.speculative(3).steps[0]
    cur = s.dst_idx
    assert cur.shape == (32, 4) and len(set(cur.ravel().tolist())) == 128
    assert not set(cur.ravel().tolist()) & set(s.src_idx.tolist())
    assert s.accept_len.min() >= 0 and s.accept_len.max() <= 4


def test_large_layer_slots():
    s0, s1 = wl.large_layer_step(0), wl.large_layer_step(1)
    assert len(set(s0.src_idx.tolist())) == 256 and np.array_equal(s0.src_idx, s0.dst_idx[:, 0])
    assert not np.array_equal(s0.src_idx, s1.src_idx)
    assert s0.q.shape == (256, 1, 16, 128)


def test_oracle_reproduces_golden_fixture():
    outs, pool = make_golden.compute()
    g_outs, g_pool = make_golden.load()
    assert np.array_equal(outs, g_outs)
    assert np.array_equal(pool, g_pool)
