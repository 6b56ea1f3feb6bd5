"""Seeded synthetic inputs for the decode-time Gated DeltaNet state update.

This module is shared by the CUDA path's callers (tests, benchmark) and by the
CPU oracle's callers.  It holds none of the update's arithmetic: only random
draws, the input-side recipe of each workload (L2 normalisation of q and k per
head, the gate maps alpha = exp(-softplus(x)) and beta = sigmoid(y)), rounding
to bfloat16, and the choice of slots.

The five workloads:

* ``tiny``        B=1, Hk=Hv=1, dk=dv=16, eight sequential T=1 calls chained
                  through a 4-slot pool (src != dst), fp32 q/k/v, seed 0.
* ``decode_b16``  B=16, Hk=16, Hv=32, dk=dv=128, bf16 q/k/v, 64-slot pool,
                  distinct random slots updated in place, seed 1.
* ``prefix_cow``  B=128, 512-slot pool; 115 of the 128 requests (90 %) read a
                  source slot shared with other requests (group sizes from a
                  power law n^-2 on [2, 16]); every request writes a fresh,
                  distinct destination slot; seed 2.
* ``speculative`` B=32, T=4 draft tokens, 1024-slot pool; per-token
                  destinations (current_input_indices) distinct and disjoint
                  from the sources; accept_len ~ Uniform{0..4}; seed 3.
* ``large``       B=256 x 8 independent layers, 2048-slot pool per layer
                  (2 MiB of fp32 state per request per layer), in place on a
                  random slot permutation; seed 4.  Its pools are filled on the
                  device (``fill_pool_device``), everything else here.

The prefix-sharing ratio stands in for the >90 % KV/state cache hit rate the
TokenSpeed article reports for multi-turn agentic traffic ("Hybrid prefix
caching for GDN/Mamba" item); no trace or dataset is involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"

STATE_STD = 0.02  # pool initialisation N(0, 0.02): standard deviation 0.02

LARGE = dict(B=256, layers=8, num_slots=2048, Hk=16, Hv=32, dk=128, dv=128, dtype=BF16, seed=4)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Step:
    """The per-call inputs of one decode call (host arrays)."""

    q: np.ndarray          # [B, T, Hk, dk] float32 or uint16 (bf16 bits)
    k: np.ndarray          # [B, T, Hk, dk]
    v: np.ndarray          # [B, T, Hv, dv]
    alpha: np.ndarray      # [B, T, Hv] float32
    beta: np.ndarray       # [B, T, Hv] float32
    src_idx: np.ndarray    # [B] int32
    dst_idx: np.ndarray    # [B, T] int32
    accept_len: Optional[np.ndarray] = None  # [B] int32, speculative workloads only

    @property
    def B(self) -> int:
        return int(self.q.shape[0])

    @property
    def T(self) -> int:
        return int(self.q.shape[1])

    @property
    def Hk(self) -> int:
        return int(self.q.shape[2])

    @property
    def Hv(self) -> int:
        return int(self.v.shape[2])

    @property
    def dk(self) -> int:
        return int(self.q.shape[3])

    @property
    def dv(self) -> int:
        return int(self.v.shape[3])

    @property
    def dtype(self) -> str:
        return BF16 if self.q.dtype == np.uint16 else F32


@dataclass
class Workload:
    name: str
    num_slots: int
    Hk: int
    Hv: int
    dk: int
    dv: int
    pool: Optional[np.ndarray]            # [num_slots, Hv, dk, dv] float32 (None: filled on device)
    steps: List[Step] = field(default_factory=list)


def _unit_rows(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0, 1) draws, L2-normalised along the last axis in float32."""
    x = rng.standard_normal(shape, dtype=np.float32)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))
    return (x / n).astype(np.float32)


def _gates(rng: np.random.Generator, shape):
    """alpha = exp(-softplus(x)), beta = sigmoid(y), x, y ~ N(0, 1), rounded to float32."""
    x = rng.standard_normal(shape)
    y = rng.standard_normal(shape)
    softplus = np.logaddexp(0.0, x)
    alpha = np.exp(-softplus).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-y))).astype(np.float32)
    return alpha, beta


def random_step_inputs(rng: np.random.Generator, B: int, T: int, Hk: int, Hv: int, dk: int, dv: int,
                       dtype: str = BF16):
    """q, k (unit-norm per head), v ~ N(0, 1) and the gates, in the workloads' distributions."""
    q = _unit_rows(rng, (B, T, Hk, dk))
    k = _unit_rows(rng, (B, T, Hk, dk))
    v = rng.standard_normal((B, T, Hv, dv), dtype=np.float32)
    alpha, beta = _gates(rng, (B, T, Hv))
    if dtype == BF16:
        q, k, v = f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)
    elif dtype != F32:
        raise ValueError(dtype)
    return q, k, v, alpha, beta


def random_raw_step_inputs(rng: np.random.Generator, B: int, T: int, Hk: int, Hv: int, dk: int, dv: int,
                           dtype: str = BF16):
    """Raw per-token projections for the fused prologue: q, k, v ~ N(0, 1) without
    normalisation, and the gate pre-activations x, y ~ N(0, 1) (fp32)."""
    q = rng.standard_normal((B, T, Hk, dk), dtype=np.float32)
    k = rng.standard_normal((B, T, Hk, dk), dtype=np.float32)
    v = rng.standard_normal((B, T, Hv, dv), dtype=np.float32)
    x = rng.standard_normal((B, T, Hv)).astype(np.float32)
    y = rng.standard_normal((B, T, Hv)).astype(np.float32)
    if dtype == BF16:
        q, k, v = f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)
    elif dtype != F32:
        raise ValueError(dtype)
    return q, k, v, x, y


def init_pool(rng: np.random.Generator, num_slots: int, Hv: int, dk: int, dv: int,
              std: float = STATE_STD) -> np.ndarray:
    """A host slot pool with every element ~ N(0, std), float32."""
    pool = rng.standard_normal((num_slots, Hv, dk, dv), dtype=np.float32)
    pool *= np.float32(std)
    return pool


def share_groups(rng: np.random.Generator, n_shared: int, lo: int = 2, hi: int = 16) -> List[int]:
    """Group sizes n in [lo, hi] with P(n) ~ n^-2, drawn until ``n_shared`` requests are placed.

    The last group is clipped to what is left; a remainder of one is never left
    behind (the group before it grows by one, or shrinks by one at ``hi``), so
    every group shares its slot between at least ``lo`` requests.
    """
    sizes = np.arange(lo, hi + 1)
    p = sizes.astype(np.float64) ** -2.0
    p /= p.sum()
    groups: List[int] = []
    rem = n_shared
    while rem > 0:
        n = int(min(rng.choice(sizes, p=p), rem))
        if rem - n == 1:
            n = n + 1 if n < hi else n - 1
        groups.append(n)
        rem -= n
    return groups


def tiny(seed: int = 0) -> Workload:
    """Eight sequential single-token calls on a 4-slot 16x16 pool, slot i -> i+1 (mod 4)."""
    rng = np.random.default_rng(seed)
    num_slots, Hk, Hv, dk, dv = 4, 1, 1, 16, 16
    pool = init_pool(rng, num_slots, Hv, dk, dv)
    steps = []
    for i in range(8):
        q, k, v, a, b = random_step_inputs(rng, 1, 1, Hk, Hv, dk, dv, F32)
        steps.append(Step(q, k, v, a, b, np.array([i % 4], np.int32), np.array([[(i + 1) % 4]], np.int32)))
    return Workload("tiny", num_slots, Hk, Hv, dk, dv, pool, steps)


def decode_b16(seed: int = 1) -> Workload:
    """B=16 in-place decode on distinct random slots of a 64-slot pool."""
    rng = np.random.default_rng(seed)
    num_slots, B, Hk, Hv, dk, dv = 64, 16, 16, 32, 128, 128
    pool = init_pool(rng, num_slots, Hv, dk, dv)
    slots = rng.permutation(num_slots)[:B].astype(np.int32)
    q, k, v, a, b = random_step_inputs(rng, B, 1, Hk, Hv, dk, dv, BF16)
    step = Step(q, k, v, a, b, slots.copy(), slots.reshape(B, 1).copy())
    return Workload("decode_b16", num_slots, Hk, Hv, dk, dv, pool, [step])


def prefix_cow(seed: int = 2) -> Workload:
    """B=128 copy-on-write decode: 90 % of requests share a source slot, all write fresh slots."""
    rng = np.random.default_rng(seed)
    num_slots, B, Hk, Hv, dk, dv = 512, 128, 16, 32, 128, 128
    n_shared = int(round(0.9 * B))  # 115
    groups = share_groups(rng, n_shared)
    n_src = len(groups) + (B - n_shared)
    perm = rng.permutation(num_slots).astype(np.int32)
    src_slots, dst_slots = perm[:n_src], perm[n_src:n_src + B]
    src = np.concatenate([np.full(g, src_slots[i], np.int32) for i, g in enumerate(groups)]
                         + [src_slots[len(groups):]])
    src = src[rng.permutation(B)].astype(np.int32)
    pool = init_pool(rng, num_slots, Hv, dk, dv)
    q, k, v, a, b = random_step_inputs(rng, B, 1, Hk, Hv, dk, dv, BF16)
    step = Step(q, k, v, a, b, src, dst_slots.reshape(B, 1).copy())
    return Workload("prefix_cow", num_slots, Hk, Hv, dk, dv, pool, [step])


def speculative(seed: int = 3) -> Workload:
    """B=32, T=4 draft tokens; per-token slots from current_input_indices; accept_len ~ U{0..4}."""
    rng = np.random.default_rng(seed)
    num_slots, B, T, Hk, Hv, dk, dv = 1024, 32, 4, 16, 32, 128, 128
    perm = rng.permutation(num_slots).astype(np.int32)
    src = perm[:B].copy()
    cur = perm[B:B + B * T].reshape(B, T).copy()
    pool = init_pool(rng, num_slots, Hv, dk, dv)
    q, k, v, a, b = random_step_inputs(rng, B, T, Hk, Hv, dk, dv, BF16)
    accept = rng.integers(0, T + 1, size=B).astype(np.int32)
    step = Step(q, k, v, a, b, src, cur, accept)
    return Workload("speculative", num_slots, Hk, Hv, dk, dv, pool, [step])


def large_layer_step(layer: int, seed: int = LARGE["seed"], B: int = LARGE["B"],
                     num_slots: int = LARGE["num_slots"], raw: bool = False) -> Step:
    """Inputs of one layer of the large decode: in place on a random slot permutation.

    raw=True draws the fused prologue's inputs instead (unnormalised q, k and the gate
    pre-activations x, y in the alpha/beta fields)."""
    c = LARGE
    rng = np.random.default_rng([seed, layer])
    slots = rng.permutation(num_slots)[:B].astype(np.int32)
    draw = random_raw_step_inputs if raw else random_step_inputs
    q, k, v, a, b = draw(rng, B, 1, c["Hk"], c["Hv"], c["dk"], c["dv"], c["dtype"])
    return Step(q, k, v, a, b, slots.copy(), slots.reshape(B, 1).copy())


def fill_pool_device(pool, seed: int, layer: int, std: float = STATE_STD) -> None:
    """Fill a device pool tensor with N(0, std) from a seeded torch CUDA generator."""
    import torch

    g = torch.Generator(device=pool.device)
    g.manual_seed(int(seed) * 1_000_003 + int(layer))
    flat = pool.view(-1)
    chunk = 1 << 28
    for s in range(0, flat.numel(), chunk):
        flat[s:s + chunk].normal_(0.0, std, generator=g)


WORKLOADS = {
    "tiny": tiny,
    "decode_b16": decode_b16,
    "prefix_cow": prefix_cow,
    "speculative": speculative,
}
