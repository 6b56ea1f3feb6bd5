/*
 * gdn_slot_cache.h -- host-side slot allocator and prefix cache for GDN state slots.
 *
 * The source pages describe this part as the logical cache layer.
 * - [DE/EN] the 24-ai.news TokenSpeed article, "What are the key optimizations behind the
 *   record?", item "Hybrid prefix caching for GDN/Mamba": a C++ layer keeps the logical
 *   cache, radix-tree matching extended with Mamba state slots reuses states with
 *   copy-on-write semantics, and the cache hit rate exceeds 90 % on multi-turn agentic
 *   traffic.
 * - [PT/HI] the zubnet.ai LightSeek TokenSpeed article, second paragraph: recurrent states
 *   are checkpointed beside the KV pages; cached checkpoints are reused without mutation;
 *   speculative decoding goes through current_input_indices instead of tensor copies.
 *
 * This library provides that layer for the slot pool of gdn_decode_step (gdn_step.h).  It
 * only decides which int32 slot each request reads and writes.  It never touches device
 * memory: the index tables it fills are the src_idx / dst_idx / current_input_indices of
 * the decode and commit calls.
 *
 *   slots        0 .. num_slots-1, each with a reference count.  A slot is free at count 0.
 *                Holders are the requests whose current state lives there and the
 *                checkpoints that point at it.
 *   checkpoints  a radix tree over int32 token ids.  A node may name a slot that holds the
 *                GDN state after exactly the tokens on its root-to-node path.  Checkpoints
 *                are read, never written.
 *   requests     an active sequence.  Its current state lives in one slot, which it either
 *                owns (count 1) or shares with a checkpoint or other requests.
 *
 * Per decode step, gdn_slot_cache_plan fills src/dst for a batch of requests.
 *   - T = 1: a request that owns its slot updates it in place (dst = src).  A request whose
 *     slot is shared gets a fresh destination slot: the copy-on-write fork.  The shared
 *     state is read and left untouched.
 *   - T > 1: every request gets T fresh draft slots (current_input_indices).
 * gdn_slot_cache_commit then applies the outcome.
 *   - T = 1: each request moves to its destination.
 *   - T > 1: with accept_len a, the request moves to draft a-1 (a >= 1) or keeps its slot
 *     (a = 0).  The rejected drafts are freed.  This is the host-side mirror of the device
 *     gdn_commit.
 *
 * Ownership and threading: a cache is a plain host object.  Calls on one cache must not
 * overlap (no internal locking); different caches are independent.  All memory is host
 * memory owned by the cache; every pointer argument is host memory owned by the caller.
 *
 * Errors: GDN_ERR_INVALID_ARG for bad sizes, unknown request ids, null pointers or a commit
 * that does not match the last plan.  GDN_ERR_CAPACITY when no free slot is left and no
 * checkpoint can be evicted (every cached state is still in use).  A failing call changes
 * nothing.
 */
#ifndef GDN_SLOT_CACHE_H
#define GDN_SLOT_CACHE_H

#include <stdint.h>

#include "gdn_step.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gdn_slot_cache gdn_slot_cache;

/* New cache over a pool of num_slots (>= 1) slots, all free.  *cache receives the handle. */
gdn_status gdn_slot_cache_create(int32_t num_slots, gdn_slot_cache** cache);

/* Frees the cache and everything it holds.  NULL is a no-op. */
void gdn_slot_cache_destroy(gdn_slot_cache* cache);

/*
 * Starts a request whose context is tokens[0..n).  The longest prefix of it that has a
 * checkpoint is matched.
 * - On a hit, the request starts from that checkpoint's slot: it shares the slot, and
 *   its first decode step writes a fresh one.  *matched_len is the checkpoint's length.
 *   *needs_init is 0.
 * - On a miss, a free slot is taken for the request.  *matched_len is 0 and *needs_init is
 *   1: the caller must fill that slot with the initial (zero) state before it is read.
 * *req receives the request id and *slot the slot that holds the request's state.
 * n >= 0; tokens may be NULL when n == 0.
 */
gdn_status gdn_slot_cache_open(gdn_slot_cache* cache, const int32_t* tokens, int64_t n, int32_t* req,
                               int32_t* slot, int64_t* matched_len, int32_t* needs_init);

/*
 * Plans one decode call of T tokens (T >= 1) for the B requests reqs[0..B).  Fills
 * src_idx[B] and dst_idx[B*T] as described above, and takes the fresh slots the plan
 * needs.  A request may appear at most once per plan.  Each request must be committed
 * (gdn_slot_cache_commit) before it is planned again.
 */
gdn_status gdn_slot_cache_plan(gdn_slot_cache* cache, const int32_t* reqs, int32_t B, int32_t T,
                               int32_t* src_idx, int32_t* dst_idx);

/*
 * Applies the outcome of the planned call for reqs[0..B) (the same requests and T as the
 * plan, any order).  accept_len[B] holds the accepted draft counts in [0, T]; it is
 * ignored (and may be NULL) when T == 1.  committed[B] (may be NULL) receives each
 * request's new state slot: the table gdn_commit produces on the device, and the src_idx
 * of the next step.
 */
gdn_status gdn_slot_cache_commit(gdn_slot_cache* cache, const int32_t* reqs, int32_t B, int32_t T,
                                 const int32_t* accept_len, int32_t* committed);

/*
 * Records the request's current state as the checkpoint of tokens[0..n) (n >= 1).  The
 * state must be the one after exactly those tokens.  The slot becomes shared, so the
 * request's next single-token step forks it.  If that prefix already has a checkpoint,
 * nothing changes.  *slot (may be NULL) receives the checkpoint's slot.
 */
gdn_status gdn_slot_cache_checkpoint(gdn_slot_cache* cache, int32_t req, const int32_t* tokens, int64_t n,
                                     int32_t* slot);

/* Ends a request: releases its slot and any planned, uncommitted draft slots. */
gdn_status gdn_slot_cache_close(gdn_slot_cache* cache, int32_t req);

/*
 * Evicts least-recently-used checkpoints that nothing else holds until at least
 * want_free slots are free, or none is left to evict.  *evicted (may be NULL) receives
 * the number of checkpoints dropped.  A plan or open that finds no free slot evicts in
 * the same way by itself.
 */
gdn_status gdn_slot_cache_evict(gdn_slot_cache* cache, int32_t want_free, int32_t* evicted);

/* Free slots, checkpoints and open requests.  Any output pointer may be NULL. */
gdn_status gdn_slot_cache_stats(const gdn_slot_cache* cache, int32_t* free_slots, int32_t* checkpoints,
                                int32_t* open_requests);

/* Reference count of one slot (0 = free), or -1 for a bad slot or cache. */
int32_t gdn_slot_cache_refcount(const gdn_slot_cache* cache, int32_t slot);

#ifdef __cplusplus
}
#endif

#endif /* GDN_SLOT_CACHE_H */
