/*
 * gdn_step.h -- C ABI of the decode-time Gated DeltaNet state update for B200 (sm_100a).
 *
 * What is computed.  A hybrid full/linear-attention model keeps, in each Gated
 * DeltaNet (GDN) linear-attention layer, a recurrent state per request and value
 * head (TokenSpeed 580 tok/s article, 24-ai.news English edition, opening section
 * "What is TokenSpeed and how does it differ from vLLM?").  One decode token
 * updates it with the gated delta rule (Yang, Kautz & Hatamizadeh, "Gated Delta
 * Networks", ICLR 2025):
 *
 *     S' = alpha * S * (I - beta * k k^T) + beta * v k^T,      o = S' q,
 *
 * with S the dv x dk fp32 state, k, q in R^dk, v in R^dv and scalar gates alpha,
 * beta per token and value head.  The library evaluates it in the equivalent
 * rank-one form u = S k, c = beta * (v - alpha * u), S' = alpha * S + c k^T,
 * o = alpha * (S q) + c * (k . q), streaming each state through the SM once.
 *
 * Where states live.  States sit in a slot pool and are addressed through int32
 * indices: each request reads slot src and writes slot dst, which may differ.
 * This is the index indirection that replaces per-step state copies ("Mamba
 * State Update optimization" item of the 24-ai.news article's "What are the key
 * optimizations behind the record?"), the copy-on-write reuse of cached prefix
 * checkpoints (same section, "Hybrid prefix caching for GDN/Mamba"; zubnet.ai
 * LightSeek TokenSpeed article, second paragraph), and the speculative path in
 * which per-draft-token states go to the slots named by current_input_indices
 * (zubnet.ai article, second paragraph).
 *
 * Layouts (all row-major, innermost last):
 *   pool    float [num_slots][Hv][dk][dv]   element [s][h][i][j] = S_h[j][i] of slot s
 *                                           (the stored tile is S transposed: dv contiguous)
 *   q, k    [B][T][Hk][dk]   bf16 or fp32 (qkv_dtype)
 *   v       [B][T][Hv][dv]   bf16 or fp32 (qkv_dtype)
 *   alpha, beta  float [B][T][Hv]
 *   out     float [B][T][Hv][dv]
 *   src_idx int32 [B];  dst_idx int32 [B][T] (current_input_indices when T > 1)
 * Value head h reads key head h / (Hv / Hk) (contiguous groups); Hv % Hk == 0.
 * No scaling or normalisation of q and k happens inside the step.
 *
 * Ownership and execution.  Every pointer is device memory owned by the caller;
 * the library allocates nothing and frees nothing.  Between calls it keeps only
 * per-device constants read on first use (the SM count, a symbol address, the
 * tensor-map encoder), which concurrent host threads fill safely, and the one
 * device array of gdn_check_step_noalloc (see there).  All work is enqueued on
 * `stream` (0 = legacy default stream) of the calling thread's current device;
 * no call synchronises except gdn_get_error.
 *
 * Errors.  Each entry returns a gdn_status.  Bad sizes, a null pointer or an
 * unknown dtype return GDN_ERR_INVALID_ARG before anything is enqueued; a failed
 * launch returns GDN_ERR_CUDA.  Index errors are found on the device: the
 * affected request is skipped (nothing of it is written) and GDN_ERR_INDEX is
 * recorded in *err_word (first error wins) when err_word is not NULL; read and
 * clear it with gdn_get_error.  Kernels never trap or assert, and every wait a
 * kernel spins on (copy and tensor-core completions) gives up after 2 s and
 * records GDN_ERR_TIMEOUT.  One wait is not the kernel's own: the chunked
 * prefill's tensor-memory allocation (tcgen05.alloc) blocks until the SM has the
 * columns free.  Its kernels ask for no more than one resident CTA of theirs
 * leaves (shared memory keeps a second one off the SM), so only a tensor-memory
 * user outside this library running on the same SM (another stream's sm_100
 * kernel that holds columns) can delay it, until that kernel releases them.
 */
#ifndef GDN_STEP_H
#define GDN_STEP_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* sizes, null pointers, dtype: rejected before launch */
    GDN_ERR_CUDA = 2,        /* a CUDA runtime call or launch failed */
    GDN_ERR_INDEX = 3,       /* device-side: a slot index or accept length was out of range */
    GDN_ERR_TIMEOUT = 4,     /* device-side: a bounded wait gave up */
    GDN_ERR_ALIAS = 5,       /* device-side (gdn_check_step): the slot indices break a precondition */
    GDN_ERR_CAPACITY = 6     /* host-side (gdn_slot_cache_*): no free slot and nothing evictable, or out of memory */
} gdn_status;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Padding sentinel for src_idx: a request whose source slot is GDN_SLOT_NONE is
 * skipped without an error (nothing read or written, its dst entries ignored),
 * so a batch can be padded to a fixed size, e.g. for a captured CUDA graph. */
#define GDN_SLOT_NONE (-1)

/* Kernel choice for gdn_decode_step_variant. */
typedef enum gdn_variant {
    GDN_VARIANT_AUTO = 0,   /* what gdn_decode_step uses: the first of TILE, STREAM, COLUMN that applies */
    GDN_VARIANT_STREAM = 1, /* persistent bulk-copy pipeline through shared memory: T == 1,
                               dk == dv == 128, every buffer 16-byte aligned, B*Hv % 4 == 0,
                               err_word not NULL (a timed-out copy is reported there only) */
    GDN_VARIANT_TILE = 2,   /* state tile held in registers: (dk, dv) in {(128, 128), (64, 64)},
                               pool and out 16-byte aligned, any T; one CTA per 64-column block
                               of a (request, head) tile, which for T > 1 carries its columns
                               across the tokens */
    GDN_VARIANT_COLUMN = 3  /* one thread per value column: any shape and alignment */
} gdn_variant;

/*
 * gdn_decode_step -- one GDN layer's decode update for B requests and T tokens each.
 *
 * Defined by the gated delta rule above and the slot scheme of the 24-ai.news
 * article ("Mamba State Update optimization", "Hybrid prefix caching for
 * GDN/Mamba") and the zubnet.ai article (second paragraph: state slots,
 * current_input_indices, copy-on-write checkpoints).
 *
 * For each request b, value head h and token t = 0..T-1 the state carried from
 * pool[src_idx[b]][h] (token 0) or from the previous token is updated with
 * token t's q, k, v, alpha, beta; the fp32 result is stored to
 * pool[dst_idx[b*T + t]][h] and carried to token t+1, and o is written to
 * out[b][t][h][:].  The src slot is only read (copy-on-write) unless it is
 * also the destination (T == 1 in-place update).
 *
 *   pool       device, [num_slots][Hv][dk][dv] fp32, read and written
 *   num_slots  number of slots in pool (>= 1)
 *   src_idx    device, int32 [B]
 *   dst_idx    device, int32 [B*T]
 *   q, k, v    device, layouts above, element type qkv_dtype
 *   alpha, beta device, fp32 [B][T][Hv]
 *   out        device, fp32 [B][T][Hv][dv], written
 *   B >= 0 (0 is a no-op), T >= 1, Hk >= 1, Hv >= 1 with Hv % Hk == 0,
 *   1 <= dk <= 4096, dv >= 1, B*Hv < 2^31
 *   qkv_dtype  GDN_F32 or GDN_BF16
 *   err_word   device int32, may be NULL (index errors then skip silently)
 *   stream     CUDA stream the work is enqueued on
 *
 * Preconditions (results are unspecified if violated; nothing is written out of
 * bounds either way): the B*T destination slots are pairwise distinct; no
 * destination equals another request's source; for T > 1 no destination equals
 * the request's own source.  Many requests may share one source slot.
 * Index check: a request whose src is GDN_SLOT_NONE is padding and is skipped
 * silently.  Any other request whose src or any of its T dst entries lies
 * outside [0, num_slots) is skipped entirely (no state, no output) and
 * GDN_ERR_INDEX is recorded.
 */
gdn_status gdn_decode_step(float* pool, int32_t num_slots, const int32_t* src_idx,
                           const int32_t* dst_idx, const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta, float* out, int32_t B, int32_t T,
                           int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int32_t qkv_dtype,
                           int32_t* err_word, cudaStream_t stream);

/*
 * gdn_decode_step_variant -- gdn_decode_step with an explicit kernel choice.
 *
 * Same operation, arguments, preconditions and errors as gdn_decode_step, plus
 * `variant` (a gdn_variant).  All variants compute the same update; they differ
 * in how work maps onto the GPU and may differ in floating-point rounding order
 * (never in which slots are written).  A variant whose conditions (listed with
 * gdn_variant) the call does not meet returns GDN_ERR_INVALID_ARG before any
 * launch.  Meant for tests and measurements that pin one kernel.
 */
gdn_status gdn_decode_step_variant(float* pool, int32_t num_slots, const int32_t* src_idx,
                                   const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, float* out, int32_t B, int32_t T,
                                   int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int32_t qkv_dtype,
                                   int32_t* err_word, int32_t variant, cudaStream_t stream);

/* Flags of gdn_decode_step_fused. */
#define GDN_FUSE_GATES 1   /* alpha/beta arguments are raw x, y: alpha = exp(-softplus(x)), beta = sigmoid(y) */
#define GDN_FUSE_QK_NORM 2 /* q and k are L2-normalised per (token, key head): x / sqrt(sum x^2 + 1e-6) */
#define GDN_SHARED_SOURCES 4 /* scheduling hint, no arithmetic: many requests share source slots */

/*
 * gdn_decode_step_fused -- gdn_decode_step with its input prologue folded in.
 *
 * The pages collapse multi-step prologues (norms, gate maps) into the kernel that
 * consumes them, keeping intermediates in registers (zubnet.ai article, second
 * paragraph: QK-RMSNorm + partial RoPE + gate split, 5 kernels to 1).  This entry
 * does the same for the GDN step: the raw per-token projections enter directly.
 *   flags & GDN_FUSE_GATES:   `alpha_or_x`, `beta_or_y` hold raw x, y [B][T][Hv]
 *                             (fp32); the step uses alpha = exp(-softplus(x)) and
 *                             beta = sigmoid(y).  A model's own scale or bias on x,
 *                             if it has one, is applied by the caller.
 *   flags & GDN_FUSE_QK_NORM: q and k are used as q / sqrt(|q|^2 + 1e-6) and
 *                             k / sqrt(|k|^2 + 1e-6), per (token, key head).
 *   flags & GDN_SHARED_SOURCES: a hint that many of the batch's requests share
 *                             source slots (prefix-checkpoint hits; a caller that
 *                             plans with gdn_slot_cache_plan sees it as repeated
 *                             src entries).  The single-token register-tile kernel
 *                             then visits every request of one value head before
 *                             the next head, so a shared tile is read from HBM once
 *                             and then from L2; other kernels ignore the hint.  The result is bit for bit the same with or
 *                             without it; without sharing it only costs bandwidth
 *                             (request-major order keeps each slot's 2 MiB together).
 * Without flags the call is gdn_decode_step.  Same layouts, preconditions, errors
 * and bytes moved as gdn_decode_step; unknown flag bits return GDN_ERR_INVALID_ARG.
 * Served by the register-tile kernels (column kernel for other shapes/alignments).
 */
gdn_status gdn_decode_step_fused(float* pool, int32_t num_slots, const int32_t* src_idx,
                                 const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                 const float* alpha_or_x, const float* beta_or_y, float* out, int32_t B,
                                 int32_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int32_t qkv_dtype,
                                 int32_t flags, int32_t* err_word, cudaStream_t stream);

/*
 * gdn_prefill -- feed L tokens per request and store only the final state: the
 * checkpoint of the prefix.
 *
 * The pages checkpoint the recurrent state of a prefix next to its KV pages so that
 * later requests reuse it (zubnet.ai article, second paragraph; 24-ai.news article,
 * "Hybrid prefix caching for GDN/Mamba").  This call produces such a checkpoint:
 * for each request b it applies the same per-token update as gdn_decode_step with
 * T = L, starting from pool[src_idx[b]], writes o for every token to
 * out[b][t][h][:], and stores only the state after token L-1, to
 * pool[dst_idx[b]][h].  The intermediate states stay on chip (or, in the column
 * kernel, in the destination slot).  dst may equal src (continue a sequence in place).
 *
 *   Same arguments and layouts as gdn_decode_step with T = L, except dst_idx: int32 [B].
 *   Preconditions: destinations distinct; no destination equals another request's
 *   source.  Padding (src GDN_SLOT_NONE), index errors and the error word behave as in
 *   gdn_decode_step.  A fresh sequence starts from a slot the caller zero-filled.
 */
gdn_status gdn_prefill(float* pool, int32_t num_slots, const int32_t* src_idx, const int32_t* dst_idx,
                       const void* q, const void* k, const void* v, const float* alpha, const float* beta,
                       float* out, int32_t B, int32_t L, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                       int32_t qkv_dtype, int32_t* err_word, cudaStream_t stream);

/*
 * gdn_prefill_chunked -- gdn_prefill computed chunk by chunk (64 tokens) with dense
 * per-chunk contractions instead of one token step at a time.
 *
 * Same operation, arguments, preconditions and errors as gdn_prefill (the result
 * equals it within fp32 rounding, not bit for bit).  Within a chunk the token
 * dependencies reduce to a unit lower-triangular system (I + A) E = R whose inverse
 * depends only on the chunk's keys and gates; a first kernel builds it for all
 * chunks in parallel, a second walks each sequence's chunks in order carrying the
 * state.  Supports dk = dv = 128.  With bf16 inputs both kernels run their products on
 * the tensor cores; with fp32 inputs they run on the CUDA cores and, on B200, take
 * longer than gdn_prefill's token steps, which is then the faster call.
 *
 *   workspace        device memory of at least gdn_prefill_workspace_bytes(B, L, Hv,
 *                    dk, dv) bytes, 16-byte aligned, caller-owned; contents on entry
 *                    do not matter and on return are unspecified.  Calls sharing one
 *                    workspace must not overlap.
 *   err_word         device int32, required here (unlike gdn_prefill): besides index
 *                    errors, a copy or tensor-core wait that runs out (2 s) records
 *                    GDN_ERR_TIMEOUT; the affected requests' checkpoints are then left
 *                    unwritten and their outputs are unspecified.
 * Unsupported shapes, a missing or short workspace, a NULL err_word, or a workspace,
 * pool, out, q, k or v that is not 16-byte aligned return GDN_ERR_INVALID_ARG.
 */
gdn_status gdn_prefill_chunked(float* pool, int32_t num_slots, const int32_t* src_idx, const int32_t* dst_idx,
                               const void* q, const void* k, const void* v, const float* alpha,
                               const float* beta, float* out, int32_t B, int32_t L, int32_t Hk, int32_t Hv,
                               int32_t dk, int32_t dv, int32_t qkv_dtype, void* workspace,
                               size_t workspace_bytes, int32_t* err_word, cudaStream_t stream);

/* Workspace bytes gdn_prefill_chunked needs for these sizes; 0 if it does not support them. */
size_t gdn_prefill_workspace_bytes(int32_t B, int32_t L, int32_t Hv, int32_t dk, int32_t dv);

/*
 * gdn_commit -- accept speculative draft tokens by rewriting an int32 index table.
 *
 * Defined by the O(1) index update that replaces an O(L*D) state copy (24-ai.news
 * article, "Mamba State Update optimization") and by speculative decoding through
 * current_input_indices (zubnet.ai article, second paragraph).  No state byte moves.
 *
 * For each request b with a = accept_len[b]:
 *   a == 0          committed[b] is kept (the pre-draft state stays current);
 *   1 <= a <= T     committed[b] = cur[b*T + a - 1] (the state after draft token a-1).
 * The call is idempotent.  The committed table is what the next decode step
 * passes as src_idx.
 *
 *   accept_len device int32 [B]
 *   committed  device int32 [B], updated in place
 *   cur        device int32 [B*T] (current_input_indices of the decode call)
 *   B >= 0 (0 is a no-op), T >= 1, num_slots >= 1
 *   err_word   device int32, may be NULL
 * Errors: accept_len outside [0, T], or a selected slot outside [0, num_slots),
 * leaves committed[b] unchanged and records GDN_ERR_INDEX.
 */
gdn_status gdn_commit(const int32_t* accept_len, int32_t* committed, const int32_t* cur, int32_t B,
                      int32_t T, int32_t num_slots, int32_t* err_word, cudaStream_t stream);

/*
 * gdn_check_step -- verify on the device that a decode call's slot indices meet
 * gdn_decode_step's preconditions, without touching the pool.
 *
 * Copy-on-write reuse of cached checkpoints (24-ai.news article, "Hybrid prefix
 * caching for GDN/Mamba"; zubnet.ai article, second paragraph) is only sound if no
 * call writes a slot that another request of the same call reads, and if no two
 * writes land in one slot.  This call checks exactly that for the indices a
 * gdn_decode_step(src_idx, dst_idx, B, T, num_slots) would receive:
 *   1. every non-padding request's src and its T dst entries lie in [0, num_slots)
 *      (otherwise GDN_ERR_INDEX is recorded);
 *   2. the destinations of all non-padding requests are pairwise distinct;
 *   3. no destination equals the source of a different request;
 *   4. for T > 1, no destination equals the request's own source
 *      (2-4 otherwise record GDN_ERR_ALIAS).
 * Requests whose src is GDN_SLOT_NONE are ignored.  In-place updates (T == 1,
 * dst == src of the same request) and shared sources are allowed.
 *
 *   src_idx    device int32 [B]; dst_idx device int32 [B*T]
 *   scratch    device int32 [num_slots], caller-owned working memory; its contents
 *              on entry do not matter and on return are unspecified
 *   err_word   device int32, required: the first error found is recorded there
 *              (GDN_ERR_INDEX or GDN_ERR_ALIAS; read it with gdn_get_error)
 * Three operations are enqueued on `stream` (a fill of scratch and two kernels);
 * nothing synchronises.  Calls sharing one scratch buffer must not overlap.
 * B >= 0 (0 is a no-op), T >= 1, num_slots >= 1; null pointers or bad sizes return
 * GDN_ERR_INVALID_ARG.
 */
gdn_status gdn_check_step(const int32_t* src_idx, const int32_t* dst_idx, int32_t B, int32_t T,
                          int32_t num_slots, int32_t* scratch, int32_t* err_word, cudaStream_t stream);

/*
 * gdn_check_step_noalloc -- gdn_check_step for callers that cannot allocate.
 *
 * No counterpart on the source pages: this is a convenience of this library.
 * gdn_check_step needs a caller-provided scratch buffer of num_slots int32.  Some
 * callers cannot get one: a serving process whose device memory has been handed
 * in full to its own allocator (a raw cudaMalloc then fails or waits on that
 * allocator), or a latency-critical loop with a no-allocation rule because
 * cudaMalloc and cudaFree may synchronise the whole device.  This entry point
 * performs the same check with no scratch argument: it uses a fixed array of
 * GDN_CHECK_NOALLOC_MAX_SLOTS int32 (1 MiB) that lives in the library's device
 * memory on every GPU that loads the library, until the process exits.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *
 *   Arguments, checks and error codes are those of gdn_check_step without
 *   `scratch`.  num_slots > GDN_CHECK_NOALLOC_MAX_SLOTS returns GDN_ERR_INVALID_ARG
 *   before anything is enqueued.
 *   Set-up: the first call on a device (with that device current) looks up the
 *   array's device address with cudaGetSymbolAddress and keeps it for later calls;
 *   make that first call before any stream capture begins.  The kept address
 *   belongs to the device's current primary context: it does not survive
 *   cudaDeviceReset (after a reset the module is loaded afresh and the array may
 *   move), so do not call this entry point again after resetting a device it was
 *   used on.
 *   Sharing: every call on a device uses the same array.  Each call resets the part
 *   it uses before checking, but calls that overlap on the GPU (different streams,
 *   or different host threads, without ordering between them) race on the array
 *   and may report wrong results.  Order such calls, or use gdn_check_step with
 *   separate scratch buffers.
 */
#define GDN_CHECK_NOALLOC_MAX_SLOTS (1 << 18)
gdn_status gdn_check_step_noalloc(const int32_t* src_idx, const int32_t* dst_idx, int32_t B, int32_t T,
                                  int32_t num_slots, int32_t* err_word, cudaStream_t stream);

/*
 * gdn_wait_selftest -- exercise the bounded wait of the copy and MMA pipelines.
 *
 * No counterpart on the source pages: a self-test of this library's failure
 * detection.  The bulk-copy pipelines (the STREAM decode variant, the chunked
 * prefill) wait on mbarriers with a limit on global time; a wait that runs out
 * records GDN_ERR_TIMEOUT and the kernel drains and returns instead of hanging.
 * This call runs that same wait in one CTA on an mbarrier that nothing arrives
 * on, so it always runs out after limit_ns nanoseconds and records
 * GDN_ERR_TIMEOUT in *err_word.  Nothing faults; the context stays usable.
 *
 *   limit_ns   1 .. 2,000,000,000 (the pipelines' own limit is the maximum)
 *   err_word   device int32, required
 * Returns GDN_ERR_INVALID_ARG for a null err_word or a limit out of range.
 */
gdn_status gdn_wait_selftest(uint64_t limit_ns, int32_t* err_word, cudaStream_t stream);

/*
 * gdn_get_error -- read and clear a device error word.
 *
 * Synchronises `stream`, copies *err_word (device) to *host_code (host) and
 * resets the device word to 0.  *host_code is a gdn_status value (GDN_OK when no
 * device-side error was recorded).  Returns GDN_ERR_INVALID_ARG for null
 * pointers and GDN_ERR_CUDA when a runtime call fails.
 */
gdn_status gdn_get_error(int32_t* err_word, int32_t* host_code, cudaStream_t stream);

/* Static, NUL-terminated name of a status code ("GDN_OK", ...); never NULL. */
const char* gdn_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_STEP_H */
