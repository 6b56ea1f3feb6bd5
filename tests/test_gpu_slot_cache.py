"""The host slot cache driving the CUDA kernels through a multi-turn, multi-request session.

Each token's q, k, v and gates are a deterministic function of the token prefix that ends
at it, as in a model, where they are projections of the context.  So the GDN state after a
prefix does not depend on how it was reached.  The session opens requests that extend
cached prefixes (copy-on-write forks), decodes single tokens in place, runs speculative
steps with random accept lengths, checkpoints and closes.  It checks:
  * every call against the oracle, run on the same index tables (states 1e-4, outputs 2e-3);
  * the device commit table against the allocator's, bit for bit;
  * every checkpoint's bytes, which must stay identical from the moment it is taken;
  * at the end, each live request's state against an oracle replay of its whole token
    history from the zero state: prefix reuse is transparent.
"""
import zlib

import numpy as np
import pytest

import oracle
from hybrid_linear_attention_step_b200 import workloads as wl
from tests.gpu_helpers import TOL_OUT_BF16, TOL_STATE, rel_err, to_torch

pytestmark = pytest.mark.gpu

Hk, Hv, DK, DV = 2, 4, 128, 128


def token_inputs(seq):
    """q, k, v (bf16 bits), alpha, beta of the last token of ``seq``, from the whole prefix."""
    rng = np.random.default_rng(zlib.crc32(np.asarray(seq, np.int32).tobytes()))
    return wl.random_step_inputs(rng, 1, 1, Hk, Hv, DK, DV, wl.BF16)


def batch_inputs(prefixes, drafts):
    """Inputs [B, T, ...] for requests with token histories ``prefixes`` and new tokens ``drafts``."""
    rows = []
    for pre, new in zip(prefixes, drafts):
        rows.append([token_inputs(list(pre) + list(new[:t + 1])) for t in range(len(new))])
    stack = lambda i: np.ascontiguousarray(np.concatenate([np.concatenate([r[t][i] for t in range(len(r))], 1)
                                                           for r in rows], 0))
    return [stack(i) for i in range(5)]


def test_slot_cache_session_on_gpu():
    import torch

    from hybrid_linear_attention_step_b200 import gdn
    from hybrid_linear_attention_step_b200.slot_cache import SlotCache

    num_slots = 160
    cache = SlotCache(num_slots)
    pool_h = np.zeros((num_slots, Hv, DK, DV), np.float32)
    pool_d = to_torch(pool_h)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(5)
    hist = {}          # request -> tokens whose effect its state holds
    slot_of = {}       # request -> slot holding that state
    ckpts = {}         # slot -> bytes at checkpoint time
    calls = {"T1": 0, "spec": 0, "fork": 0, "hits": 0}

    def decode(reqs, T, new_tokens):
        src, dst = cache.plan(reqs, T)
        assert oracle.check_step(src, dst, num_slots) == 0
        calls["fork"] += int(np.sum((T == 1) & (src != dst[:, 0])))
        q, k, v, a, b = batch_inputs([hist[r] for r in reqs], new_tokens)
        x = [to_torch(t) for t in (q, k, v, a, b)]
        src_d, dst_d = to_torch(src), to_torch(dst)
        out = torch.zeros((len(reqs), T, Hv, DV), device="cuda")
        gdn.gdn_decode_step(pool_d, src_d, dst_d, *x, out, err_word=err)
        ref_out = np.zeros((len(reqs), T, Hv, DV), np.float32)
        oracle.decode_step(pool_h, src, dst, q, k, v, a, b, ref_out, nthreads=4)
        assert rel_err(out.cpu().numpy(), ref_out) <= TOL_OUT_BF16
        if T == 1:
            committed = cache.commit(reqs)
            accept = np.ones(len(reqs), np.int32)
            calls["T1"] += 1
        else:
            accept = rng.integers(0, T + 1, len(reqs)).astype(np.int32)
            committed_d = src_d.clone()
            gdn.gdn_commit(to_torch(accept), committed_d, dst_d, num_slots, err_word=err)
            committed = cache.commit(reqs, T, accept)
            assert np.array_equal(committed_d.cpu().numpy(), committed)  # device commit == host allocator
            calls["spec"] += 1
        for r, new, acc, s_ in zip(reqs, new_tokens, accept, committed):
            hist[r] = hist[r] + list(new[:acc])
            slot_of[r] = int(s_)
        assert gdn.gdn_get_error(err) == gdn.GDN_OK

    def open_request(context):
        r, slot, matched, needs_init = cache.open(context)
        if needs_init:
            pool_h[slot] = 0.0
            pool_d[slot].zero_()
        else:
            calls["hits"] += 1
        hist[r] = list(context[:matched])
        slot_of[r] = slot
        for t in context[matched:]:  # feed the rest of the context one token at a time
            decode(np.array([r], np.int32), 1, [[t]])
        return r

    vocab = 7
    for rnd in range(28):
        op = rng.integers(0, 6)
        if op <= 1 or len(hist) < 2:
            # a new turn: extend a prefix of a live history (or start fresh)
            base = list(hist.values())[rng.integers(0, len(hist))] if hist and rng.random() < 0.8 else []
            ctx = base[: rng.integers(0, len(base) + 1)] + list(rng.integers(0, vocab, rng.integers(1, 4)))
            open_request(ctx)
        elif op <= 3:
            reqs = rng.choice(list(hist), size=rng.integers(1, min(len(hist), 6) + 1), replace=False).astype(np.int32)
            T = int(rng.choice([1, 3]))
            decode(reqs, T, [list(rng.integers(0, vocab, T)) for _ in reqs])
        elif op == 4:
            r = int(rng.choice(list(hist)))
            if hist[r]:
                s = cache.checkpoint(r, hist[r])
                if s not in ckpts:
                    ckpts[s] = pool_d[s].cpu().numpy().copy()
        else:
            r = int(rng.choice(list(hist)))
            cache.close(r)
            del hist[r], slot_of[r]
        for s, snap in ckpts.items():  # checkpoints are never written
            assert np.array_equal(pool_d[s].cpu().numpy().view(np.uint32), snap.view(np.uint32))

    assert calls["spec"] > 0 and calls["fork"] > 0 and calls["hits"] > 0, calls
    # every live request's state equals a from-scratch replay of its history
    for r, seq in hist.items():
        if not seq:
            continue
        slot = slot_of[r]
        replay = np.zeros((2, Hv, DK, DV), np.float32)
        for i in range(len(seq)):
            q, k, v, a, b = token_inputs(seq[: i + 1])
            o = np.zeros((1, 1, Hv, DV), np.float32)
            oracle.decode_step(replay, np.array([i % 2], np.int32), np.array([[(i + 1) % 2]], np.int32), q, k, v, a,
                               b, o)
        assert rel_err(pool_d[slot].cpu().numpy(), replay[len(seq) % 2]) <= TOL_STATE


@pytest.mark.parametrize("chunked", [False, True], ids=["token_steps", "chunked"])
def test_prefill_checkpoint_then_fork_and_decode(chunked):
    """The intended flow end to end: a prefill writes a prompt's state into the request's
    slot, the cache keeps it as a checkpoint, a second request extending the prompt shares
    it and forks on its first decode step.  States match an oracle replay of each token
    history; the checkpoint's bytes never change."""
    import torch

    from hybrid_linear_attention_step_b200 import gdn
    from hybrid_linear_attention_step_b200.slot_cache import SlotCache

    num_slots = 8
    cache = SlotCache(num_slots)
    pool_d = torch.zeros((num_slots, Hv, DK, DV), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(11)
    ctx = [int(x) for x in rng.integers(0, 50, 130)]  # two chunks and a ragged tail

    r0, slot, matched, needs_init = cache.open(ctx)
    assert matched == 0 and needs_init
    x = [to_torch(t) for t in batch_inputs([[]], [ctx])]
    idx = torch.tensor([slot], dtype=torch.int32, device="cuda")
    out = torch.zeros((1, len(ctx), Hv, DV), device="cuda")
    if chunked:
        ws = torch.empty(gdn.gdn_prefill_workspace_bytes(1, len(ctx), Hv, DK, DV), dtype=torch.uint8,
                         device="cuda")
        gdn.gdn_prefill_chunked(pool_d, idx, idx, *x, out, ws, err_word=err)
    else:
        gdn.gdn_prefill(pool_d, idx, idx, *x, out, err_word=err)
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    assert cache.checkpoint(r0, ctx) == slot
    ckpt = pool_d[slot].cpu().numpy().copy()

    def replay(seq, st=None, start=0):
        """Oracle state after the tokens seq[start:], from st (zero if None), one token at a time."""
        st = np.zeros((1, Hv, DK, DV), np.float32) if st is None else st.copy()
        for i in range(start, len(seq)):
            q, k, v, a, b = token_inputs(seq[: i + 1])
            o = np.zeros((1, 1, Hv, DV), np.float32)
            zero = np.zeros(1, np.int32)
            oracle.decode_step(st, zero, zero.reshape(1, 1), q, k, v, a, b, o, nthreads=8)
        return st

    ref_ctx = replay(ctx)
    assert rel_err(ckpt, ref_ctx[0]) <= TOL_STATE
    ext = ctx + [7]
    r1, s1, matched1, needs1 = cache.open(ext)
    assert (s1, matched1, needs1) == (slot, len(ctx), False)
    src, dst = cache.plan([r1])
    assert src[0] == slot and dst[0, 0] != slot  # copy-on-write fork
    x1 = [to_torch(t) for t in batch_inputs([ctx], [[7]])]
    out1 = torch.zeros((1, 1, Hv, DV), device="cuda")
    gdn.gdn_decode_step(pool_d, to_torch(src), to_torch(dst), *x1, out1, err_word=err)
    cache.commit([r1])
    assert gdn.gdn_get_error(err) == gdn.GDN_OK
    assert np.array_equal(pool_d[slot].cpu().numpy().view(np.uint32), ckpt.view(np.uint32))
    assert rel_err(pool_d[int(dst[0, 0])].cpu().numpy(), replay(ext, ref_ctx, len(ctx))[0]) <= TOL_STATE
