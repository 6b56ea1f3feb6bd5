"""Shared helpers for the GPU parity tests: move seeded host inputs to the device,
run the CUDA path and the oracle on the same bytes, and compare."""
from __future__ import annotations

import numpy as np

import oracle
from hybrid_linear_attention_step_b200 import workloads as wl

# Tolerances: max relative error with the reference RMS as floor (see rel_err).
TOL_STATE = 1e-4        # fp32 state
TOL_OUT_BF16 = 2e-3     # outputs of bf16-input calls
TOL_OUT_F32 = 1e-4      # outputs of fp32-input calls


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max_i |g_i - r_i| / max(|r_i|, rho), rho = RMS of the reference tensor.

    The RMS floor keeps near-zero reference entries from blowing the ratio up.
    An all-zero reference demands exact zeros.
    """
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    if g.shape != r.shape:
        raise ValueError(f"shape mismatch {g.shape} vs {r.shape}")
    if r.size == 0:
        return 0.0
    rho = float(np.sqrt(np.mean(r * r)))
    if rho == 0.0:
        return 0.0 if np.all(g == 0) else float("inf")
    if not np.all(np.isfinite(g)):
        return float("inf")
    return float(np.max(np.abs(g - r) / np.maximum(np.abs(r), rho)))


def to_torch(a: np.ndarray, device="cuda"):
    import torch

    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def step_to_device(s: wl.Step, device="cuda"):
    return dict(q=to_torch(s.q, device), k=to_torch(s.k, device), v=to_torch(s.v, device),
                alpha=to_torch(s.alpha, device), beta=to_torch(s.beta, device),
                src=to_torch(s.src_idx, device),
                dst=to_torch(np.ascontiguousarray(s.dst_idx.reshape(s.B, -1)), device))


def run_gpu(pool_dev, s: wl.Step, out_fill=-7.0, err=None, stream=None, variant=None):
    """Runs one CUDA decode call on ``pool_dev`` (updated in place); returns out (host).

    ``variant`` None goes through gdn_decode_step; a name pins one kernel through
    gdn_decode_step_variant.  Without ``err`` the call gets an error word of its own,
    which must read GDN_OK afterwards."""
    import torch

    from hybrid_linear_attention_step_b200 import gdn

    x = step_to_device(s, pool_dev.device)
    out = torch.full((s.B, s.T, s.Hv, s.dv), out_fill, dtype=torch.float32, device=pool_dev.device)
    args = (pool_dev, x["src"], x["dst"], x["q"], x["k"], x["v"], x["alpha"], x["beta"], out)
    own_err = err is None
    if own_err:
        err = torch.zeros(1, dtype=torch.int32, device=pool_dev.device)
    if variant is None:
        gdn.gdn_decode_step(*args, err_word=err, stream=stream)
    else:
        gdn.gdn_decode_step_variant(*args, variant, err_word=err, stream=stream)
    torch.cuda.synchronize()
    if own_err:
        assert gdn.gdn_get_error(err, stream=stream) == gdn.GDN_OK
    return out.cpu().numpy()


def run_oracle(pool: np.ndarray, s: wl.Step, out_fill=-7.0, nthreads=8):
    """Runs the oracle on a copy of ``pool``; returns (pool_after, out, skipped)."""
    pool = pool.copy()
    out = np.full((s.B, s.T, s.Hv, s.dv), np.float32(out_fill), np.float32)
    skipped = oracle.decode_step(pool, s.src_idx, np.ascontiguousarray(s.dst_idx.reshape(s.B, s.T)), s.q, s.k,
                                 s.v, s.alpha, s.beta, out, nthreads=nthreads)
    return pool, out, skipped


def check_pool(got: np.ndarray, ref: np.ndarray, before: np.ndarray, written: np.ndarray,
               ref_before: np.ndarray = None):
    """Bit-exact slot behaviour plus in-tolerance state values.

    * every slot outside ``written`` keeps its bytes: ``got`` against ``before``
      (the device pool before the call) and ``ref`` against ``ref_before`` (the
      oracle's pool before the call, by default the same array);
    * the written slots agree with the oracle within TOL_STATE.
    """
    if ref_before is None:
        ref_before = before
    num_slots = before.shape[0]
    untouched = np.setdiff1d(np.arange(num_slots), np.asarray(written).ravel())
    assert np.array_equal(got[untouched].view(np.uint32), before[untouched].view(np.uint32)), \
        "CUDA path changed a slot it does not own"
    assert np.array_equal(ref[untouched].view(np.uint32), ref_before[untouched].view(np.uint32))
    w = np.unique(np.asarray(written).ravel())
    e = rel_err(got[w], ref[w])
    assert e <= TOL_STATE, f"state rel err {e:.3g} > {TOL_STATE}"
    return e
