"""The chunkwise form of the gated delta rule that gdn_prefill_chunked evaluates, restated
in numpy float64 and checked against the oracle's token-by-token prefill (no GPU).

Within a chunk of C tokens starting from M0 (the stored state, S0 transposed), with
g_t = alpha_1 ... alpha_t, A[t][i] = beta_t (g_t / g_i) k_t.k_i (i < t), T = (I + A)^-1:
    U  = T diag(beta) V,   Tb = T diag(beta g)
    E  = U - Tb (K M0)
    O  = diag(g) Q M0 + P E,       P[t][i] = (g_t / g_i) q_t.k_i  (i <= t)
    M_C = g_C M0 + K^T diag(g_C / g) E
These tests pin that derivation, including ragged last chunks and a full reset
(alpha = 0), to the definition the oracle implements.
"""
import numpy as np
import pytest

import oracle
from hybrid_linear_attention_step_b200 import workloads as wl


def chunked_prefill_f64(M0, q, k, v, alpha, beta, C):
    """One (request, head): q, k [L, dk], v [L, dv], gates [L] -> (M_L, out [L, dv])."""
    L = q.shape[0]
    M = M0.astype(np.float64)
    out = np.zeros((L, v.shape[1]))
    for t0 in range(0, L, C):
        sl = slice(t0, min(t0 + C, L))
        K, Q, V = k[sl], q[sl], v[sl]
        a, bt = alpha[sl].astype(np.float64), beta[sl].astype(np.float64)
        n = K.shape[0]
        g = np.cumprod(a)
        ratio = np.zeros((n, n))
        for t in range(n):
            for i in range(t + 1):
                ratio[t, i] = np.prod(a[i + 1:t + 1])  # g_t / g_i without dividing by a zero g_i
        A = np.tril(bt[:, None] * ratio * (K @ K.T), -1)
        T = np.linalg.inv(np.eye(n) + A)
        U = T @ (bt[:, None] * V)
        Tb = T * (bt * g)[None, :]
        E = U - Tb @ (K @ M)
        P = np.tril(ratio * (Q @ K.T))
        out[sl] = g[:, None] * (Q @ M) + P @ E
        M = g[-1] * M + K.T @ (ratio[-1][:, None] * E)
    return M, out


@pytest.mark.parametrize("L,C,reset", [(1, 64, None), (64, 64, None), (150, 64, 70), (37, 8, 5), (40, 16, None)])
def test_chunk_algebra_matches_token_steps(L, C, reset):
    rng = np.random.default_rng(L * 31 + C)
    dk = dv = 16
    q, k, v, a, b = wl.random_step_inputs(rng, 1, L, 1, 1, dk, dv, wl.F32)
    if reset is not None:
        a[0, reset, 0] = 0.0
    pool = (rng.standard_normal((2, 1, dk, dv)) * 0.02).astype(np.float32)
    out = np.zeros((1, L, 1, dv), np.float32)
    ref_pool = pool.copy()
    assert oracle.prefill(ref_pool, np.array([0], np.int32), np.array([1], np.int32), q, k, v, a, b, out) == 0
    M, o = chunked_prefill_f64(pool[0, 0], q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0], b[0, :, 0], C)
    # The oracle rounds the state to fp32 after every token; the float64 chunk form does
    # not, so the two agree to fp32 rounding accumulated over L tokens.
    scale = np.abs(ref_pool[1, 0]).max()
    assert np.abs(M - ref_pool[1, 0]).max() <= 1e-5 * scale * max(1, L / 16)
    assert np.abs(o - out[0, :, 0]).max() <= 1e-5 * np.abs(out).max() * max(1, L / 16)


def test_chunk_algebra_detects_a_dropped_gate_ratio():
    """The same check fails when the state update drops the g_C / g factor (a plausible
    slip in the chunked form), so the comparison above has teeth."""
    rng = np.random.default_rng(3)
    L, C, dk = 40, 16, 16
    q, k, v, a, b = wl.random_step_inputs(rng, 1, L, 1, 1, dk, dk, wl.F32)
    pool = (rng.standard_normal((2, 1, dk, dk)) * 0.02).astype(np.float32)
    out = np.zeros((1, L, 1, dk), np.float32)
    ref_pool = pool.copy()
    oracle.prefill(ref_pool, np.array([0], np.int32), np.array([1], np.int32), q, k, v, a, b, out)

    def wrong(M0):
        M = M0.astype(np.float64)
        for t0 in range(0, L, C):
            K, V = k[0, t0:t0 + C, 0], v[0, t0:t0 + C, 0]
            aa, bt = a[0, t0:t0 + C, 0].astype(np.float64), b[0, t0:t0 + C, 0].astype(np.float64)
            n = K.shape[0]
            g = np.cumprod(aa)
            ratio = np.array([[np.prod(aa[i + 1:t + 1]) if i <= t else 0.0 for i in range(n)] for t in range(n)])
            T = np.linalg.inv(np.eye(n) + np.tril(bt[:, None] * ratio * (K @ K.T), -1))
            E = T @ (bt[:, None] * V) - (T * (bt * g)[None, :]) @ (K @ M)
            M = g[-1] * M + K.T @ E  # missing diag(g_C / g)
        return M

    assert np.abs(wrong(pool[0, 0]) - ref_pool[1, 0]).max() > 1e-3 * np.abs(ref_pool[1, 0]).max()
