// gdn_prefill_chunked.cu -- chunked prefill of the Gated DeltaNet state
// (contract: gdn_prefill_chunked in gdn_step.h).
//
// Same result as gdn_prefill (L tokens of the gated delta rule, Yang, Kautz &
// Hatamizadeh, ICLR 2025; the state after the last token stored as the prefix
// checkpoint that the zubnet.ai LightSeek TokenSpeed article, second paragraph,
// keeps beside the KV pages), computed chunk by chunk instead of token by token.
//
// Within a chunk of C tokens, with the state S0 (stored M0 = S0^T, [dk][dv]) at
// its start, the per-token rule S_t = alpha_t S_{t-1} + e_t k_t^T with
// e_t = beta_t (v_t - alpha_t S_{t-1} k_t) unrolls to
//     S_t = g_t S0 + sum_{i<=t} (g_t / g_i) e_i k_i^T,      g_t = alpha_1 ... alpha_t,
// and the e_t solve the unit lower-triangular system (rows = tokens)
//     (I + A) E = diag(beta) V - diag(beta g) K M0,
//     A[t][i] = beta_t (g_t / g_i) (k_t . k_i) for i < t.
// With T = (I + A)^-1, U = T diag(beta) V and Tb = T diag(beta g):
//     E   = U - Tb (K M0)                              (C x dv)
//     O   = diag(g) (Q M0) + P E,  P[t][i] = (g_t/g_i)(q_t . k_i), i <= t
//     M_C = g_C M0 + K^T diag(g_C / g) E                (dk x dv)
// Kernel 1 builds, for every (request, head, chunk) in parallel, everything that
// does not depend on the state into the caller's workspace; kernel 2 walks each
// sequence's chunks in order, carrying the state.
//
// bf16 inputs (tensor cores, tcgen05 with accumulators in TMEM; k, q, v tiles brought
// by tensor copies).  Kernel 1 forms [K; Q] K^T as one MMA (exact bf16 products),
// inverts I + A in fp32 by 16 x 16 blocks, and forms U = T diag(beta) V and
// W = T diag(beta g) K = Tb K as MMAs, so that kernel 2 evaluates the same algebra
// re-associated:
//     E = U - W M0,   O = diag(g) (Q M0) + P E,   M_C = g_C M0 + K^T diag(g_C / g) E,
// all as MMAs.  Kernel 2 runs one CTA per (request, head) with the whole state: its
// 128 value rows are the MMA's M dimension and the TMEM lanes.  An operand that is not
// a bf16 input is fp32 and enters as bf16 parts (hi + mid + lo carries 24 bits); the
// part products that matter at fp32 precision are formed (the ones left out are named
// with kernel 2).  With fp32 inputs (not exact in bf16) both kernels run on the CUDA
// cores in the first form, with T explicit and kernel 2 split into 32-column blocks.
// Ratios g_t / g_i are formed as exp(log g_t - log g_i) <= 1, so nothing overflows;
// g_t itself may underflow to zero, which is its true value to fp32 precision.
//
// The workspace holds one record per (request, head, chunk); its layouts (one for
// each input type) are given with the constants below.

#include "gdn_step.h"

#include <cuda.h>  // CUtensorMap and its encoder's types (the encoder comes from the runtime)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kC = 64;          // tokens per chunk
constexpr int kD = 128;         // dk = dv supported here
constexpr int kDVC = 32;        // value columns per CTA in the sequential kernel
constexpr int kNCB = kD / kDVC; // column blocks per (request, head)
constexpr int kNT = 256;        // threads per CTA (both kernels)
constexpr int kUS = kDVC + 4;   // row stride of the 64 x 32 fp32 tiles (16-byte rows, bank spread)
constexpr int kPad = 4;         // row padding of [C][D] shared arrays in the fp32 scan kernel

// Workspace record of the fp32-input path (CUDA cores), bytes.
constexpr size_t kRecU = 0;                             // U in four column slabs [4][64][36] fp32
constexpr size_t kUSlab = (size_t)kC * kUS * 4;
constexpr size_t kRecTb = kRecU + kNCB * kUSlab;        // TbT [64][64] fp32
constexpr size_t kRecP = kRecTb + (size_t)kC * kC * 4;  // PT [64][64] fp32
constexpr size_t kRecG = kRecP + (size_t)kC * kC * 4;   // log g [64]
constexpr size_t kRecF32Bytes = kRecG + (size_t)kC * 4;

// Workspace record of the bf16-input path (tensor cores), bytes.  The tiles the scan
// gives the tensor cores straight from the inputs (Q, K) are not in it: it loads them
// itself.
//   W   [W_lo | W_mid | W_hi] for dk 0..63, then the same for dk 64..127: six tiles of
//       64 tokens x 64 features (bf16 parts of W = T diag(beta g) K), each in the
//       128-byte-swizzled K-major layout a tensor copy writes (row t at 128 t, its
//       16-byte granule q at position q ^ (t & 7))
//   P   [P_mid | P_hi]: 128 rows (t, per part) x 64 (i), bf16 parts of P, K-major
//       no-swizzle core-matrix layout
//   G   g_t [64], g_C / g_t [64], g_C, 3 zero words
//   UT  U^T fp32 as 16 x 128 float4 granules: granule q of value row j (tokens 4q..4q+3
//       of U[t][j]) at index q * dv + j, so that 32 consecutive rows are 512 contiguous
//       bytes for the writer and the reader alike
// G and UT are one contiguous range (the scan copies them together).
constexpr uint32_t kSwTile = kC * 64 * 2;              // one 64 x 64 bf16 swizzled tile
constexpr size_t kR2W = 0;
constexpr uint32_t kR2WBytes = 6 * kSwTile;
constexpr size_t kR2P = kR2W + kR2WBytes;
constexpr uint32_t kR2PBytes = 2 * kC * kC * 2;
constexpr size_t kR2G = kR2P + kR2PBytes;
constexpr uint32_t kR2GBytes = (2 * kC + 4) * 4;
constexpr size_t kR2UT = kR2G + kR2GBytes;
constexpr uint32_t kR2UTBytes = kD * kC * 4;
constexpr size_t kR2Bytes = kR2UT + kR2UTBytes;
constexpr uint32_t kImgA = 8 * kSwTile;                // [W_lo W_mid W_hi Q] x two feature halves
constexpr uint32_t kImgB = 2 * kSwTile + kR2PBytes;    // K (two feature halves) | P parts
constexpr uint32_t kImgC = kR2GBytes + kR2UTBytes;     // G | UT

constexpr size_t kRecMax = kR2Bytes > kRecF32Bytes ? kR2Bytes : kRecF32Bytes;
constexpr size_t kRecBytes = (kRecMax + 255) / 256 * 256;
static_assert(kRecTb % 16 == 0 && kRecP % 16 == 0 && kRecG % 16 == 0 && kR2P % 16 == 0 && kR2G % 16 == 0 &&
                  kR2UT % 16 == 0,
              "16-byte record fields");
static_assert(kImgC % 16 == 0 && kR2PBytes % 16 == 0 && (3 * kSwTile) % 16 == 0, "16-byte bulk copies");

struct ChunkArgs {
    float* pool;
    const int32_t* src_idx;
    const int32_t* dst_idx;
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    float* out;
    unsigned char* ws;  // workspace: per (b, h, chunk) one record of kRecBytes
    int32_t* err;
    int num_slots, B, L, Hk, Hv, G, nchunks;
};

__device__ __forceinline__ unsigned char* record_of(const ChunkArgs& a, int bh, int c) {
    return a.ws + ((size_t)bh * a.nchunks + c) * kRecBytes;
}

// 8 consecutive fp32 input elements (32 bytes, 16-byte aligned).
template <typename InT>
__device__ __forceinline__ void ld8(const void* base, size_t idx, float (&x)[8]);
template <>
__device__ __forceinline__ void ld8<float>(const void* base, size_t idx, float (&x)[8]) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
}
template <typename InT>
__device__ __forceinline__ float ld_in(const void* base, size_t idx);
template <>
__device__ __forceinline__ float ld_in<float>(const void* base, size_t idx) {
    return __ldg(static_cast<const float*>(base) + idx);
}

__device__ __forceinline__ void record(int32_t* err, int32_t code) {
    if (err != nullptr) atomicCAS(err, 0, code);
}

// Byte offset of element (row r, column k) of a K-major bf16 tensor-core operand
// with Kdim columns: 8 x 8 core matrices of 128 contiguous bytes (8 rows of 16
// bytes), K-adjacent core matrices 128 bytes apart, 8-row groups Kdim*16 apart.
__host__ __device__ constexpr uint32_t core_off(int r, int k, int Kdim) {
    return (uint32_t)((r >> 3) * (Kdim >> 3) * 128 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// tcgen05 / bulk-copy helpers (sm_100a PTX).
// ---------------------------------------------------------------------------
// 2^x by the ex2.approx.ftz instruction (PTX ISA: relative error about 2^-22, subnormal
// results flushed to zero), for the 8192 gate ratios g_t / g_i <= 1 of a chunk.  A ratio
// below 2^-126 multiplies a dot product of unit-norm vectors, so flushing it is below fp32
// precision of the sums it enters.
__device__ __forceinline__ float ex2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor: no swizzle, K-adjacent core matrices 128 B apart
// (leading byte offset), 8-row groups `sbo` bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) |
           (1ull << 46);
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor of a 128-byte-swizzled operand (layout type 2, version 1),
// in the canonical forms of the tcgen05 shared-memory descriptor:
//   K-major:  rows 128 B apart, 8-row atoms (1024 B) `sbo` apart; the 32-byte step of one
//             MMA along K is added to the start address (lbo is not used: 16)
//   MN-major: 64 consecutive M (or N) elements per 128-byte row, one row per K index,
//             8-row atoms `sbo` apart along K, 64-element blocks `lbo` apart along M (N)
// The tiles start on 1024-byte boundaries, where the swizzle pattern starts.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}
constexpr uint32_t kIdescAmn = 1u << 15;  // instruction descriptor: A is MN-major
constexpr uint32_t kIdescBmn = 1u << 16;  // B is MN-major

// The k, q and v tensors as 4-d tensor maps {feature, head, token, request} with a box
// of 64 features x 1 head x 64 tokens, 128-byte swizzle: one load is one 8 KB operand
// tile of a chunk; tokens past L read as zero.
struct TileMaps {
    CUtensorMap k, q, v;
};

// One tile load into this CTA's shared memory, completing on `bar` with its byte count.
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, int feat, int head, int tok, int req,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(feat), "r"(head), "r"(tok), "r"(req), "r"(smem_u32(bar))
        : "memory");
}

// Dynamic shared memory rounded up to the next 1024-byte boundary (kernels that hold
// swizzled tiles allocate 1 KB more than their plan).
__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// Byte offset of the 16-byte granule q (features 8q..8q+7) of row t in a 128-byte-swizzled
// 64-row tile.
__host__ __device__ constexpr uint32_t sw128_off(int t, int q) {
    return (uint32_t)(t * 128 + ((q ^ (t & 7)) << 4));
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc)
        : "memory");
}

// The same with A in TMEM: row m of A on lane m, its 16 K-elements packed two to a 32-bit
// column (the lower K index in the low half) over 8 columns from tmem_a.
__device__ __forceinline__ void umma_bf16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                             uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count = 1) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bounded wait for the completion of the mbarrier phase with this parity: false
// once limit_ns of global time have passed without it (2 s in every pipeline).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __forceinline__ bool wait_parity(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    uint32_t done = 0;
    uint64_t t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    while (true) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
        uint64_t t1;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
        if (t1 - t0 > limit_ns) return false;
    }
}

// 16 consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t addr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Loads of 16 TMEM columns whose completion is awaited once for several of them:
// issue them, then tmem_wait_ld(), then tie_regs() on each destination so that no
// use of the registers is scheduled before the wait.
__device__ __forceinline__ void tmem_ld16_issue(uint32_t addr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(addr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tie_regs(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]));
}

// Eight fp32 values as three 16-byte granules of bf16 parts, x = hi + mid + lo up to
// |x - (hi + mid + lo)| < 2^-23 |x|: hi and mid are the fp32 bit patterns truncated to
// their upper 16 bits (a byte permute, no rounding, no conversion), lo is rounded.  Each
// residual is exact in fp32.
__device__ __forceinline__ void split3x8_fast(const float (&x)[8], uint4& hi, uint4& mid, uint4& lo) {
    uint32_t h[4], m[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t u0 = __float_as_uint(x[2 * j]), u1 = __float_as_uint(x[2 * j + 1]);
        h[j] = __byte_perm(u0, u1, 0x7632);
        const float r0 = x[2 * j] - __uint_as_float(u0 & 0xffff0000u);
        const float r1 = x[2 * j + 1] - __uint_as_float(u1 & 0xffff0000u);
        const uint32_t v0 = __float_as_uint(r0), v1 = __float_as_uint(r1);
        m[j] = __byte_perm(v0, v1, 0x7632);
        l[j] = pack_bf16x2(r0 - __uint_as_float(v0 & 0xffff0000u), r1 - __uint_as_float(v1 & 0xffff0000u));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    mid = make_uint4(m[0], m[1], m[2], m[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Two parts, hi truncated and mid rounded: |x - (hi + mid)| <= 2^-16 |x|.
__device__ __forceinline__ void split2x8_fast(const float (&x)[8], uint4& hi, uint4& mid) {
    uint32_t h[4], m[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t u0 = __float_as_uint(x[2 * j]), u1 = __float_as_uint(x[2 * j + 1]);
        h[j] = __byte_perm(u0, u1, 0x7632);
        m[j] = pack_bf16x2(x[2 * j] - __uint_as_float(u0 & 0xffff0000u), x[2 * j + 1] - __uint_as_float(u1 & 0xffff0000u));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    mid = make_uint4(m[0], m[1], m[2], m[3]);
}

// ---------------------------------------------------------------------------
// Kernel 1 pieces shared by its two forms.
// ---------------------------------------------------------------------------

// Warp 0: log g_t = sum_{i<=t} log alpha_i by a warp scan over two 32-token
// halves, beta_t, and log g into the record (when Gs is not null).  With log2 the
// logarithms are base 2 (ratios then come from exp2f).
__device__ __forceinline__ void gate_scan(const ChunkArgs& a, int b, int h, int t0, int n, int lane, float* lg,
                                          float* bt, float* Gs, bool log2 = false) {
    float al2[2] = {1.f, 1.f}, be2[2] = {0.f, 0.f};
#pragma unroll
    for (int half = 0; half < 2; ++half) {  // all loads first
        const int t = half * 32 + lane;
        if (t < n) {
            const size_t gi = (((size_t)b * a.L + t0 + t) * a.Hv + h);
            al2[half] = __ldg(a.alpha + gi);
            be2[half] = __ldg(a.beta + gi);
        }
    }
    float carry = 0.f;
    for (int half = 0; half < 2; ++half) {
        const int t = half * 32 + lane;
        float la = 0.f, be = 0.f;
        if (t < n) {
            // alpha = 0 (a full reset) would make log g = -inf and the ratios
            // -inf - -inf; e^-80 ~ 2e-35 is zero at fp32 precision instead.
            la = log2 ? fmaxf(log2f(al2[half]), -80.f * 1.44269504f) : fmaxf(logf(al2[half]), -80.f);
            be = be2[half];
        }
        float x = la;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        lg[t] = carry + x;
        bt[t] = be;
        if (Gs != nullptr) Gs[t] = carry + x;
        carry += __shfl_sync(0xffffffffu, x, 31);
    }
}

// T = (I + A)^-1 for strictly lower-triangular A (all threads; A complete and zero
// on and above the diagonal on entry, T complete on return).  Blocked in 16 x 16:
// diagonal blocks by forward substitution (one warp each, lane j owns column j),
// then block rows I = 1..3: T_I,<I = -T_II (A_I,<I T_<I,<I).  Every dot product runs
// over a fixed, unrolled length: the terms beyond the triangle are exact zeros (A
// above its diagonal, T above its diagonal, which starts zeroed), so no loop bound
// depends on the lane and the loads pipeline.
__device__ __forceinline__ void invert_unit_lower(const float (*A)[kC + 1], float (*T)[kC + 1], float (*Y)[48],
                                                  int tid) {
    const int w = tid / 32, lane = tid % 32;
    for (int e = tid; e < kC * kC; e += kNT) T[e / kC][e % kC] = 0.f;
    __syncthreads();
    if (w < 4 && lane < 16) {
        const int o = w * 16, j = lane;
        for (int r = 0; r < 16; ++r) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; m += 2) {
                acc0 = fmaf(A[o + r][o + m], T[o + m][o + j], acc0);
                acc1 = fmaf(A[o + r][o + m + 1], T[o + m + 1][o + j], acc1);
            }
            T[o + r][o + j] = (r == j ? 1.f : 0.f) - (acc0 + acc1);
            __syncwarp(0x0000ffffu);
        }
    }
    __syncthreads();
#pragma unroll
    for (int I = 1; I < 4; ++I) {
        // Y[r][col] = sum_{kk < 16 I} A[16 I + r][kk] T[kk][col], col < 16 I
        for (int e = tid; e < 16 * 16 * I; e += kNT) {
            const int r = e / (16 * I), col = e % (16 * I);
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int kk = 0; kk < 16 * I; kk += 2) {
                acc0 = fmaf(A[16 * I + r][kk], T[kk][col], acc0);
                acc1 = fmaf(A[16 * I + r][kk + 1], T[kk + 1][col], acc1);
            }
            Y[r][col] = acc0 + acc1;
        }
        __syncthreads();
        // T[16 I + r][col] = -sum_m T[16 I + r][16 I + m] Y[m][col]
        for (int e = tid; e < 16 * 16 * I; e += kNT) {
            const int r = e / (16 * I), col = e % (16 * I);
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; m += 2) {
                acc0 = fmaf(T[16 * I + r][16 * I + m], Y[m][col], acc0);
                acc1 = fmaf(T[16 * I + r][16 * I + m + 1], Y[m + 1][col], acc1);
            }
            T[16 * I + r][col] = -(acc0 + acc1);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Kernel 1, CUDA-core form (fp32 inputs): per (b, h, chunk), independent of the state.
// ---------------------------------------------------------------------------
struct Smem1 {
    float K[kC][kD + 1];     // odd row stride: rows r and r+1 sit in different banks
    float X[kC][kD + 1];     // Q, later V
    float A[kC][kC + 1];
    float T[kC][kC + 1];
    float Y[16][48];         // off-diagonal block partial products
    float lg[kC];
    float bt[kC];
};

template <typename InT>
__global__ void __launch_bounds__(kNT, 1) gdn_chunk_prepare_kernel(ChunkArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem1& sm = *reinterpret_cast<Smem1*>(smem_raw);
    const int tid = threadIdx.x;
    const int c = blockIdx.x % a.nchunks;
    const int bh = blockIdx.x / a.nchunks;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int hk = h / a.G;
    const int t0 = c * kC;
    const int n = min(kC, a.L - t0);  // valid tokens; the rest are inert (k = q = v = 0, beta = 0, alpha = 1)
    unsigned char* rec = record_of(a, bh, c);
    float* TbT = reinterpret_cast<float*>(rec + kRecTb);
    float* PT = reinterpret_cast<float*>(rec + kRecP);
    float* Gs = reinterpret_cast<float*>(rec + kRecG);

    // Load K, Q (fp32) in groups of 8 and the gates.
    for (int e = tid; e < kC * (kD / 8); e += kNT) {
        const int t = e / (kD / 8), d0 = (e % (kD / 8)) * 8;
        float kv[8] = {}, qv[8] = {};
        if (t < n) {
            const size_t row = (((size_t)b * a.L + t0 + t) * a.Hk + hk) * kD + d0;
            ld8<InT>(a.k, row, kv);
            ld8<InT>(a.q, row, qv);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            sm.K[t][d0 + j] = kv[j];
            sm.X[t][d0 + j] = qv[j];
        }
    }
    if (tid < 32) gate_scan(a, b, h, t0, n, tid, sm.lg, sm.bt, Gs);
    __syncthreads();

    // KK (strictly lower, scaled into A) and QK (lower, scaled into P), 4x4 per thread:
    // rows ty*4 + r (broadcast within a half-warp), columns tx + 16 s (16 consecutive
    // rows of K, conflict-free with the odd row stride).  P goes to the workspace, transposed.
    {
        const int ty = tid / 16, tx = tid % 16;
        float kk[4][4] = {}, qk[4][4] = {};
        for (int d = 0; d < kD; ++d) {
            float kr[4], qr[4], kc[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                kr[r] = sm.K[ty * 4 + r][d];
                qr[r] = sm.X[ty * 4 + r][d];
                kc[r] = sm.K[tx + 16 * r][d];
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    kk[r][s] = fmaf(kr[r], kc[s], kk[r][s]);
                    qk[r][s] = fmaf(qr[r], kc[s], qk[r][s]);
                }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int t = ty * 4 + r, i = tx + 16 * s;
                const float ratio = i <= t ? expf(sm.lg[t] - sm.lg[i]) : 0.f;
                sm.A[t][i] = i < t ? sm.bt[t] * ratio * kk[r][s] : 0.f;
                PT[i * kC + t] = ratio * qk[r][s];
            }
    }
    __syncthreads();

    invert_unit_lower(sm.A, sm.T, sm.Y, tid);

    // V (scaled by beta) replaces Q in X; U = T diag(beta) V, and Tb = T diag(beta g).
    for (int e = tid; e < kC * (kD / 8); e += kNT) {
        const int t = e / (kD / 8), d0 = (e % (kD / 8)) * 8;
        float vv[8] = {};
        if (t < n) ld8<InT>(a.v, (((size_t)b * a.L + t0 + t) * a.Hv + h) * kD + d0, vv);
#pragma unroll
        for (int j = 0; j < 8; ++j) sm.X[t][d0 + j] = vv[j] * sm.bt[t];
    }
    __syncthreads();
    {
        // 64 x 128 outputs; thread: 4 rows x 8 columns (columns strided by 16 for bank spread)
        float* U = reinterpret_cast<float*>(rec + kRecU);
        const int ty = tid / 16, tx = tid % 16;
        float u[4][8] = {};
        for (int i = 0; i < kC; ++i) {
            float tr[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) tr[r] = sm.T[ty * 4 + r][i];
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const float xv = sm.X[i][tx + 16 * s];
#pragma unroll
                for (int r = 0; r < 4; ++r) u[r][s] = fmaf(tr[r], xv, u[r][s]);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int col = tx + 16 * s;
                U[(col / kDVC) * (kC * kUS) + (ty * 4 + r) * kUS + col % kDVC] = u[r][s];
            }
        for (int e = tid; e < kC * kC; e += kNT) {
            const int i = e / kC, t = e % kC;
            TbT[e] = i <= t ? sm.T[t][i] * (sm.bt[i] * expf(sm.lg[i])) : 0.f;
        }
    }
}

// T = (I + A)^-1 for the strictly lower 64 x 64 A, in 16 x 16 blocks (all threads;
// A complete on entry, T complete and zero above its diagonal on return, P scratch of
// 3 x 16 x 16 floats).  Diagonal blocks by forward substitution (warp I, lane j < 16
// owns column j of block I); then the blocks below the diagonal, one diagonal distance
// d at a time: P = sum_{K=J}^{I-1} A_IK T_KJ and T_IJ = -T_II P for J = I - d.  Every
// step is a set of independent dot products over all 256 threads, unrolled so that the
// shared-memory loads of a step are in flight together.
template <int D>
__device__ __forceinline__ void merge_step(const float (*A)[kC + 4], float (*T)[kC + 4], float* P, int r, int cc) {
#pragma unroll
    for (int I = D; I < 4; ++I) {  // P = A_I,[J, I) T_[J, I),J with J = I - D
        const int J = I - D;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16 * D; k += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(&A[16 * I + r][16 * J + k]);
            acc[0] = fmaf(a4.x, T[16 * J + k][16 * J + cc], acc[0]);
            acc[1] = fmaf(a4.y, T[16 * J + k + 1][16 * J + cc], acc[1]);
            acc[2] = fmaf(a4.z, T[16 * J + k + 2][16 * J + cc], acc[2]);
            acc[3] = fmaf(a4.w, T[16 * J + k + 3][16 * J + cc], acc[3]);
        }
        P[(I - D) * 256 + r * 16 + cc] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
#pragma unroll
    for (int I = D; I < 4; ++I) {  // T_IJ = -T_II P
        const int J = I - D;
        const float* p = P + (I - D) * 256;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < 16; m += 4) {
            const float4 t4 = *reinterpret_cast<const float4*>(&T[16 * I + r][16 * I + m]);
            acc[0] = fmaf(t4.x, p[m * 16 + cc], acc[0]);
            acc[1] = fmaf(t4.y, p[(m + 1) * 16 + cc], acc[1]);
            acc[2] = fmaf(t4.z, p[(m + 2) * 16 + cc], acc[2]);
            acc[3] = fmaf(t4.w, p[(m + 3) * 16 + cc], acc[3]);
        }
        T[16 * I + r][16 * J + cc] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
    }
    __syncthreads();
}

__device__ __forceinline__ void invert_blocked(const float (*A)[kC + 4], float (*T)[kC + 4], float* P, int tid) {
    const int w = tid / 32, lane = tid % 32;
    if (w < 4) {
        if (lane < 16) {
            const int o = 16 * w, j = lane;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc0 = r == j ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                for (int m = 0; m < (r & ~3); m += 4) {
                    const float4 a4 = *reinterpret_cast<const float4*>(&A[o + r][o + m]);
                    acc0 = fmaf(-a4.x, x[m], acc0);
                    acc1 = fmaf(-a4.y, x[m + 1], acc1);
                    acc0 = fmaf(-a4.z, x[m + 2], acc0);
                    acc1 = fmaf(-a4.w, x[m + 3], acc1);
                }
#pragma unroll
                for (int m = r & ~3; m < r; ++m) acc0 = fmaf(-A[o + r][o + m], x[m], acc0);
                x[r] = acc0 + acc1;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) T[o + r][o + j] = x[r];
        }
    } else {
        // zero the six blocks above the diagonal
#pragma unroll
        for (int e = tid - 128; e < 6 * 256; e += 128) {
            const int blk = e / 256, r = (e / 16) % 16, cc = e % 16;
            const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            T[16 * I + r][16 * J + cc] = 0.f;
        }
    }
    __syncthreads();
    const int r = tid / 16, cc = tid % 16;
    merge_step<1>(A, T, P, r, cc);
    merge_step<2>(A, T, P, r, cc);
    merge_step<3>(A, T, P, r, cc);
}

// ---------------------------------------------------------------------------
// Kernel 1, tensor-core form (bf16 inputs), one CTA per (request, head, chunk):
//   the chunk's k, q and v tiles arrive by tensor copies in the 128-byte-swizzled layout;
//   D0  = [K; Q] K^T on the tensor cores (M = 128, N = 64, K = dk; exact bf16 products),
//         read out as A[t][i] = beta_t (g_t / g_i) k_t.k_i (i < t) and
//         P[t][i] = (g_t / g_i) q_t.k_i (i <= t);
//   T   = (I + A)^-1 in fp32 on the CUDA cores, in 16 x 16 blocks (invert_blocked);
//   D_U = V^T (T diag(beta))^T = U^T  and  D_W = K^T (T diag(beta g))^T = W^T on the tensor
//         cores, V^T and K^T read from the same tiles as MN-major operands (exact in bf16),
//         each T factor in three bf16 parts (24 bits).
// The record receives the scan's operands that are not inputs: W in bf16 parts,
// [P_mid | P_hi], the gate factors g_t, g_C / g_t, g_C, and U^T in fp32.
// ---------------------------------------------------------------------------
struct SmemP {
    // [K lo | Q lo | K hi | Q hi] (lo, hi: features 0..63, 64..127), 128-byte swizzled:
    // A operand of D0 (K rows also its B), K^T of D_W; once D0 is complete the two Q
    // tiles hold the first two bf16 parts of D_W's B operand.
    unsigned char KQ[4 * kSwTile];
    unsigned char V[2 * kSwTile];            // [V lo | V hi]: V^T of D_U
    union {
        struct {
            float A[kC][kC + 4];             // the system's strictly lower part (float4 rows)
            float P[3 * 16 * 16];            // scratch of the blocked inverse
        } ra;
        unsigned char Bp[4][kC * kC * 2];    // B of D_U: T diag(beta) in 3 parts; D_W's third part
        float W[kC][kD + 4];                 // W staged for its split (row stride spreads banks)
    } u;
    float T[kC][kC + 4];                     // (I + A)^-1
    float lg[kC];
    float bt[kC];
    float bg[kC];                            // beta_t g_t
    uint64_t mma, ld;
    uint32_t tmem;
};
constexpr int kSmemP = (int)sizeof(SmemP) + 1024;  // + alignment slack
static_assert(kSmemP <= 112 * 1024, "two prepare CTAs per SM");

__global__ void __launch_bounds__(kNT, 2)
    gdn_chunk_prepare_tc_kernel(ChunkArgs a, const __grid_constant__ TileMaps maps) {
    extern __shared__ __align__(1024) unsigned char smem_p[];
    SmemP& sm = *reinterpret_cast<SmemP*>(align1024(smem_p));
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    // Chunks in descending order: the records written last are the first ones the scan
    // reads, so they are still in L2 when it starts.
    const int nbh = a.B * a.Hv;
    const int c = a.nchunks - 1 - (int)(blockIdx.x / nbh);
    const int bh = blockIdx.x % nbh;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int hk = h / a.G;
    const int t0 = c * kC;
    const int n = min(kC, a.L - t0);  // valid tokens; the rest are inert (k = q = v = 0, beta = 0, alpha = 1)
    unsigned char* rec = record_of(a, bh, c);
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const int half = warp / 4;  // TMEM columns 32*half .. +31 of each 64-column accumulator
    constexpr uint32_t kIdesc = umma_idesc(128, kC);
    constexpr uint32_t kSbo64 = (kC / 8) * 128;

    // The scan may be scheduled as soon as every CTA here has started: its CTAs take
    // whole SMs, so they only land on SMs this grid has left, and wait for it to finish.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) {
        mbar_init(&sm.mma);
        mbar_init(&sm.ld);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_expect_tx(&sm.ld, 6 * kSwTile);
        tma_tile(sm.KQ, &maps.k, 0, hk, t0, b, &sm.ld);
        tma_tile(sm.KQ + kSwTile, &maps.q, 0, hk, t0, b, &sm.ld);
        tma_tile(sm.KQ + 2 * kSwTile, &maps.k, 64, hk, t0, b, &sm.ld);
        tma_tile(sm.KQ + 3 * kSwTile, &maps.q, 64, hk, t0, b, &sm.ld);
        tma_tile(sm.V, &maps.v, 0, h, t0, b, &sm.ld);
        tma_tile(sm.V + kSwTile, &maps.v, 64, h, t0, b, &sm.ld);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(128)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 1) gate_scan(a, b, h, t0, n, lane, sm.lg, sm.bt, nullptr, true);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    const uint32_t kq = smem_u32(sm.KQ), vt = smem_u32(sm.V);
    bool got = true, ld_done = false;
    if (tid == 0) {
        got = ld_done = wait_parity(&sm.ld, 0);
        if (got) {
            tc_fence_after();
            // D0: K-steps of 16 features, 32 bytes apart within a tile, the second
            // feature half two tiles on.
            for (int ks = 0; ks < kD / 16; ++ks) {
                const uint32_t at = kq + (ks < 4 ? 32u * ks : 2 * kSwTile + 32u * (ks - 4));
                umma_bf16(tmem, umma_desc_sw128(at, 16, 1024), umma_desc_sw128(at, 16, 1024), kIdesc,
                          ks != 0 ? 1u : 0u);
            }
            umma_commit(&sm.mma);
        }
    }
    int waits = 0, issued = got ? 1 : 0;
    bool ok = !__syncthreads_or(got ? 0 : 1);
    if (ok) {
        ok = !__syncthreads_or(wait_parity(&sm.mma, 0) ? 0 : 1);
        if (ok) ++waits;
    }
    if (ok) {
        tc_fence_after();
        // D0 row r < 64: k_r . k_i -> A (scaled); row 64 + t: q_t . k_i -> P (record).
        const int r = (warp % 4) * 32 + lane;
        uint32_t d0r[2][16];  // both halves of this thread's D0 row, one completion wait
        tmem_ld16_issue(tmem + lane_base + (uint32_t)(32 * half), d0r[0]);
        tmem_ld16_issue(tmem + lane_base + (uint32_t)(32 * half + 16), d0r[1]);
        tmem_wait_ld();
        tie_regs(d0r[0]), tie_regs(d0r[1]);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float v[16];
            const int i0 = 32 * half + 16 * part;
#pragma unroll
            for (int m = 0; m < 16; ++m) v[m] = __uint_as_float(d0r[part][m]);
            if (r < kC) {
                const float lt = sm.lg[r], bt = sm.bt[r];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    float x[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int i = i0 + j + m;
                        x[m] = i < r ? bt * ex2a(lt - sm.lg[i]) * v[j + m] : 0.f;
                    }
                    *reinterpret_cast<float4*>(&sm.u.ra.A[r][i0 + j]) = make_float4(x[0], x[1], x[2], x[3]);
                }
            } else {
                // P row t, columns i0..i0+15: its mid and hi bf16 parts into [P_mid | P_hi].
                const int t = r - kC;
                const float lt = sm.lg[t];
#pragma unroll
                for (int g8 = 0; g8 < 16; g8 += 8) {
                    float x[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int i = i0 + g8 + j;
                        x[j] = i <= t ? ex2a(lt - sm.lg[i]) * v[g8 + j] : 0.f;
                    }
                    uint4 p0, p1;
                    split2x8_fast(x, p0, p1);
                    unsigned char* bp = rec + kR2P;
                    *reinterpret_cast<uint4*>(bp + core_off(t, i0 + g8, kC)) = p1;
                    *reinterpret_cast<uint4*>(bp + core_off(kC + t, i0 + g8, kC)) = p0;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        if (tid < kC) sm.bg[tid] = sm.bt[tid] * exp2f(sm.lg[tid]);  // beta_t g_t
        invert_blocked(sm.u.ra.A, sm.T, sm.u.ra.P, tid);  // ends with a barrier
        // B operands of D_U and D_W: rows t, columns i, T[t][i] beta_i and T[t][i] beta_i g_i,
        // each in three bf16 parts; D_W's first two parts go to the Q tiles, free since D0.
        auto bpart = [&](int which, int p) -> unsigned char* {
            return which == 0 ? sm.u.Bp[p] : (p == 0 ? sm.KQ + kSwTile : p == 1 ? sm.KQ + 3 * kSwTile : sm.u.Bp[3]);
        };
        for (int e = tid; e < 2 * kC * (kC / 8); e += kNT) {
            const int which = e / (kC * (kC / 8)), rem = e % (kC * (kC / 8));
            const int t = (rem & 7) | ((rem >> 6) << 3), g = (rem >> 3) & 7;
            const float* sc = which ? sm.bg : sm.bt;
            const float4 t0v = *reinterpret_cast<const float4*>(&sm.T[t][8 * g]);
            const float4 t1v = *reinterpret_cast<const float4*>(&sm.T[t][8 * g + 4]);
            const float xs[8] = {t0v.x * sc[8 * g], t0v.y * sc[8 * g + 1], t0v.z * sc[8 * g + 2], t0v.w * sc[8 * g + 3],
                                 t1v.x * sc[8 * g + 4], t1v.y * sc[8 * g + 5], t1v.z * sc[8 * g + 6],
                                 t1v.w * sc[8 * g + 7]};
            uint4 p0, p1, p2;
            split3x8_fast(xs, p0, p1, p2);
            const uint32_t off = core_off(t, 8 * g, kC);
            *reinterpret_cast<uint4*>(bpart(which, 0) + off) = p0;
            *reinterpret_cast<uint4*>(bpart(which, 1) + off) = p1;
            *reinterpret_cast<uint4*>(bpart(which, 2) + off) = p2;
        }
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            // A = V^T and K^T, MN-major: features 64 to a row, tokens one row each
            // (16 tokens per MMA: 2048 bytes), the second feature half lbo bytes on.
            constexpr uint32_t kIdescMN = kIdesc | kIdescAmn;
            for (int p = 0; p < 3; ++p)
                for (int ks = 0; ks < kC / 16; ++ks)
                    umma_bf16(tmem, umma_desc_sw128(vt + 2048u * ks, kSwTile, 1024),
                              umma_desc(smem_u32(bpart(0, p)) + 256 * ks, kSbo64), kIdescMN, (p | ks) != 0 ? 1u : 0u);
            for (int p = 0; p < 3; ++p)
                for (int ks = 0; ks < kC / 16; ++ks)
                    umma_bf16(tmem + kC, umma_desc_sw128(kq + 2048u * ks, 2 * kSwTile, 1024),
                              umma_desc(smem_u32(bpart(1, p)) + 256 * ks, kSbo64), kIdescMN, (p | ks) != 0 ? 1u : 0u);
            umma_commit(&sm.mma);
        }
        ++issued;
        ok = !__syncthreads_or(wait_parity(&sm.mma, 1) ? 0 : 1);
        if (ok) {
            ++waits;
            tc_fence_after();
            // D_U row j = U^T[j][t] for this warp's 32 tokens -> the record, granule q of row j
            // at index q * dv + j; D_W row d = W[.][d] -> W staged row-major.
            const int j = (warp % 4) * 32 + lane;
            float4* ut = reinterpret_cast<float4*>(rec + kR2UT) + j;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float uv[16], wv[16];
                const int tb = 32 * half + 16 * part;
                tmem_ld16(tmem + lane_base + (uint32_t)tb, uv);
                tmem_ld16(tmem + lane_base + kC + (uint32_t)tb, wv);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    ut[((tb >> 2) + q4) * kD] = make_float4(uv[4 * q4], uv[4 * q4 + 1], uv[4 * q4 + 2], uv[4 * q4 + 3]);
#pragma unroll
                for (int m = 0; m < 16; ++m) sm.u.W[tb + m][j] = wv[m];
            }
        }
    }
    if (!ok && tid == 0) {
        record(a.err, GDN_ERR_TIMEOUT);
        if (!ld_done) wait_parity(&sm.ld, 0);
        for (; waits < issued; ++waits) wait_parity(&sm.mma, (uint32_t)waits & 1u);
    }
    float* G = reinterpret_cast<float*>(rec + kR2G);
    if (tid < kC) {
        G[tid] = exp2f(sm.lg[tid]);
        G[kC + tid] = exp2f(sm.lg[kC - 1] - sm.lg[tid]);
    } else if (tid < kC + 4) {
        G[kC + tid] = tid == kC ? exp2f(sm.lg[kC - 1]) : 0.f;  // g_C, then zero padding
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128) : "memory");
    if (!ok) return;

    // W in three bf16 parts into the record's six swizzled tiles: for each feature half,
    // W_lo, W_mid, W_hi.  Consecutive threads take consecutive granules of a row.
    for (int e = tid; e < kC * (kD / 8); e += kNT) {
        const int t = e >> 4, g = e & 15;
        const float4 w0 = *reinterpret_cast<const float4*>(&sm.u.W[t][8 * g]);
        const float4 w1 = *reinterpret_cast<const float4*>(&sm.u.W[t][8 * g + 4]);
        const float xw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint4 p0, p1, p2;
        split3x8_fast(xw, p0, p1, p2);
        unsigned char* wt = rec + kR2W + (size_t)(g >> 3) * 3 * kSwTile + sw128_off(t, g & 7);
        *reinterpret_cast<uint4*>(wt) = p2;
        *reinterpret_cast<uint4*>(wt + kSwTile) = p1;
        *reinterpret_cast<uint4*>(wt + 2 * kSwTile) = p0;
    }
}

// Reads (src, dst) of request b and classifies it: 0 run, 1 padding (skipped
// silently), 2 bad index (skipped, reported).
__device__ __forceinline__ void scan_prologue(const ChunkArgs& a, int b, int& src, int& dst, int& status) {
    const int s = __ldg(a.src_idx + b), d = __ldg(a.dst_idx + b);
    int st = 0;
    if (s == GDN_SLOT_NONE)
        st = 1;
    else if (s < 0 || s >= a.num_slots || d < 0 || d >= a.num_slots)
        st = 2;
    src = s;
    dst = d;
    status = st;
    if (st == 2) record(a.err, GDN_ERR_INDEX);
}

// ---------------------------------------------------------------------------
// Kernel 2, CUDA-core form (fp32 inputs): per (b, h, column block of kDVC), the
// chunks in order.
// ---------------------------------------------------------------------------
struct Smem2 {
    float M[kD][kDVC + 1];      // state block, [dk][dv cols]
    float Q[kC][kD + kPad];     // Q, scaled by g_t
    float K[kC][kD + kPad];     // K
    float U[kC][kDVC + 1];      // U, then E
    float Tb[kC][kC + 1];
    float P[kC][kC + 1];
    float KM[kC][kDVC + 1];
    float QM[kC][kDVC + 1];
    float lg[kC];
    float gq[kC];  // g_t
    float gk[kC];  // g_C / g_t
    int src, dst, status;
};

template <typename InT>
__global__ void __launch_bounds__(kNT, 1) gdn_chunk_scan_kernel(ChunkArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem2& sm = *reinterpret_cast<Smem2*>(smem_raw);
    const int tid = threadIdx.x;
    const int cb = blockIdx.x % kNCB;
    const int bh = blockIdx.x / kNCB;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int hk = h / a.G;
    const int col0 = cb * kDVC;

    if (tid == 0) scan_prologue(a, b, sm.src, sm.dst, sm.status);
    __syncthreads();
    if (sm.status != 0) return;

    const float* M0 = a.pool + ((size_t)sm.src * a.Hv + h) * (kD * kD);
    for (int e = tid; e < kD * kDVC; e += kNT) {
        const int i = e / kDVC, j = e % kDVC;
        sm.M[i][j] = M0[(size_t)i * kD + col0 + j];
    }

    const int ty = tid / 8, tx = tid % 8;  // 64 x 32 tiles: rows ty*2 + r, columns tx + 8 s
    for (int c = 0; c < a.nchunks; ++c) {
        const int t0 = c * kC;
        const int n = min(kC, a.L - t0);
        const unsigned char* rec = record_of(a, bh, c);
        const float* Ur = reinterpret_cast<const float*>(rec + kRecU + cb * kUSlab);
        const float* TbT = reinterpret_cast<const float*>(rec + kRecTb);
        const float* PT = reinterpret_cast<const float*>(rec + kRecP);
        const float* Gs = reinterpret_cast<const float*>(rec + kRecG);
        if (tid < kC) {
            const float lgt = Gs[tid], lgC_ = Gs[kC - 1];
            sm.lg[tid] = lgt;
            sm.gq[tid] = expf(lgt);
            sm.gk[tid] = expf(lgC_ - lgt);
        }
        __syncthreads();  // M of the previous chunk and the gate scales are ready
        const float lgC = sm.lg[kC - 1];
        for (int e = tid; e < kC * kD; e += kNT) {
            const int t = e / kD, d = e % kD;
            float qv = 0.f, kv = 0.f;
            if (t < n) {
                const size_t row = (((size_t)b * a.L + t0 + t) * a.Hk + hk) * kD;
                qv = ld_in<InT>(a.q, row + d) * sm.gq[t];
                kv = ld_in<InT>(a.k, row + d);
            }
            sm.Q[t][d] = qv;
            sm.K[t][d] = kv;
        }
        for (int e = tid; e < kC * kDVC; e += kNT) {
            const int t = e / kDVC, jj = e % kDVC;
            sm.U[t][jj] = Ur[t * kUS + jj];
        }
        for (int e = tid; e < kC * kC; e += kNT) {
            const int t = e / kC, i = e % kC;
            sm.Tb[t][i] = TbT[i * kC + t];
            sm.P[t][i] = PT[i * kC + t];
        }
        __syncthreads();

        // KM = K M and QM = (g Q) M
        {
            float km[2][4] = {}, qm[2][4] = {};
            for (int d = 0; d < kD; ++d) {
                float mv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) mv[q] = sm.M[d][tx + 8 * q];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float kr = sm.K[ty * 2 + r][d], qr = sm.Q[ty * 2 + r][d];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        km[r][q] = fmaf(kr, mv[q], km[r][q]);
                        qm[r][q] = fmaf(qr, mv[q], qm[r][q]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sm.KM[ty * 2 + r][tx + 8 * q] = km[r][q];
                    sm.QM[ty * 2 + r][tx + 8 * q] = qm[r][q];
                }
        }
        __syncthreads();
        // E = U - Tb KM (over U); each thread reads and writes only its own entries.
        {
            float e[2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int q = 0; q < 4; ++q) e[r][q] = sm.U[ty * 2 + r][tx + 8 * q];
            for (int i = 0; i < kC; ++i) {
                float km[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) km[q] = sm.KM[i][tx + 8 * q];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float tb = sm.Tb[ty * 2 + r][i];
#pragma unroll
                    for (int q = 0; q < 4; ++q) e[r][q] = fmaf(-tb, km[q], e[r][q]);
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int q = 0; q < 4; ++q) sm.U[ty * 2 + r][tx + 8 * q] = e[r][q];
        }
        __syncthreads();
        // O = QM + P E for the chunk's valid rows
        {
            float o[2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int q = 0; q < 4; ++q) o[r][q] = sm.QM[ty * 2 + r][tx + 8 * q];
            for (int i = 0; i < kC; ++i) {
                float ev[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) ev[q] = sm.U[i][tx + 8 * q];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float pr = sm.P[ty * 2 + r][i];
#pragma unroll
                    for (int q = 0; q < 4; ++q) o[r][q] = fmaf(pr, ev[q], o[r][q]);
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int t = ty * 2 + r;
                if (t < n) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        a.out[(((size_t)b * a.L + t0 + t) * a.Hv + h) * kD + col0 + tx + 8 * q] = o[r][q];
                }
            }
        }
        // M = g_C M + K^T diag(g_C / g) E; each thread reads and writes only its own rows of M.
        {
            const float gC = expf(lgC);
            const int ry = tid / 8;  // rows ry*4 .. +3
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = ry * 4 + r;
                float acc[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] = gC * sm.M[i][tx + 8 * q];
                for (int t = 0; t < kC; ++t) {
                    const float kv = sm.K[t][i] * sm.gk[t];
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[q] = fmaf(kv, sm.U[t][tx + 8 * q], acc[q]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) sm.M[i][tx + 8 * q] = acc[q];
            }
        }
        __syncthreads();
    }

    float* MD = a.pool + ((size_t)sm.dst * a.Hv + h) * (kD * kD);
    for (int e = tid; e < kD * kDVC; e += kNT) {
        const int i = e / kDVC, jj = e % kDVC;
        MD[(size_t)i * kD + col0 + jj] = sm.M[i][jj];
    }
}

// ---------------------------------------------------------------------------
// Kernel 2, tensor-core form (bf16 inputs): one CTA per (request, head) walks the
// chunks in order with the whole state in registers, transposed.  Sixteen compute
// warps hold it: thread (w, lane), w < 16, owns S[j][i] = M[i][j] for value row
// j = 32 (w % 4) + lane and key columns i in [32 (w / 4), +32), and handles the
// chunk's tokens [16 (w / 4), +16).  Row j is TMEM lane j of every accumulator, so
// the thread that reads an accumulator row is one that owns that row of the state.
// Thread 0 also issues every MMA and bulk copy; the previous chunk's outputs are
// stored while the next chunk's first products run (a separate issuing warp would
// cost registers: a 17-warp CTA is allocated as 20 warps).
// Per chunk, with S split into three bf16 parts (S = S_hi + S_mid + S_lo) as the A
// operand (M = 128 value rows, K = dk) and [W_lo | W_mid | W_hi | Q] as B (N = 64 tokens
// per part; the record's W parts and the chunk's Q tiles, all 128-byte swizzled):
//   G   = S_hi [W_lo W_mid W_hi Q] + S_mid [W_mid W_hi Q] + S_lo [W_hi]   (TMEM cols 0..255)
//   E^T = U^T - (G0 + G1 + G2) = (U - W M)^T,    QM^T = G3 (q M per token), scaled by g_t
// (the part products left out are below 2^-24 of W M, and 2^-16 of Q M, an output-only
// term).  Then with E' = diag(g_C / g) E split in three parts and E in two as A operands
// (K = 64 tokens), held in TMEM: each thread writes its parts over columns of G it has
// already read (8 columns per part and 16 tokens, see the E phase), so they take neither
// shared memory nor its bandwidth:
//   D_U = E'^T K              (B = the K tiles, MN-major; cols 256..383) ->  S <- g_C S + D_U
//   D_O = E_hi [P_mid P_hi] + E_mid [P_hi]   (cols 384..511)  ->  o = g Q M + P E
// The state update is committed first; the chain waits only for it, and the next S parts
// are written while the outputs' products run.  The issuing
// thread streams three shared-memory images, record fields by cp.async.bulk and the
// chunk's Q and K tiles by tensor copies: each buffer is refilled for the next chunk as
// soon as its last reader is done.  Every wait is bounded (2 s);
// a timeout is recorded and the CTA drains and exits.
// ---------------------------------------------------------------------------
constexpr uint32_t kSPart = (uint32_t)kD * kD * 2;  // one bf16 part of S (128 x 128)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemDU = 256;
constexpr uint32_t kTmemDO = 384;
constexpr int kScanThreads = 512;                   // 16 warps, all of them compute
constexpr int kIssuer = 0;                          // the thread that also issues MMAs and copies

struct SmemS {
    unsigned char aop[3 * kSPart];  // A operands of the first products: S parts
    unsigned char imgA[kImgA];      // [W_lo W_mid W_hi Q] for features 0..63, then 64..127
    unsigned char imgB[kImgB];      // [K lo | K hi] | [P_mid | P_hi]
    unsigned char imgC[kImgC];      // g_t, g_C / g_t, g_C | U^T
    uint64_t bar_a, bar_b, bar_c, mma_g, mma_u, mma_o;
    uint64_t e01, e23;  // quarters 0-1 / 2-3 have written their E parts
    uint32_t tmem;
    int src, dst, status;
};
constexpr int kSmemS = (int)sizeof(SmemS) + 1024;  // + alignment slack
static_assert(kSmemS <= 227 * 1024, "scan shared memory plan exceeds the per-CTA limit");
static_assert(3 * kSPart % 1024 == 0 && kImgA % 1024 == 0, "swizzled images start on 1024-byte boundaries");

// 8 consecutive TMEM columns of this warp's 32 lanes (completion awaited separately).
__device__ __forceinline__ void tmem_ld8_issue(uint32_t addr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(addr));
}
__device__ __forceinline__ void tie_regs8(uint32_t (&r)[8]) {
    asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
}
// 4 or 8 consecutive TMEM columns of this warp's 32 lanes, from registers.
__device__ __forceinline__ void tmem_st4(uint32_t addr, const uint4& v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t addr, const uint4& v, const uint4& w) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(kScanThreads, 1)
    gdn_chunk_scan_tc_kernel(ChunkArgs a, const __grid_constant__ TileMaps maps) {
    extern __shared__ __align__(1024) unsigned char smem_tc[];
    SmemS& sm = *reinterpret_cast<SmemS*>(align1024(smem_tc));
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    const bool issuer = tid == kIssuer;
    const int bh = blockIdx.x;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int hk = h / a.G;
    const int quarter = (warp / 4) & 3;            // key columns 32*quarter.., tokens 16*quarter..
    const int j = (warp % 4) * 32 + lane;          // value row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const int nch = a.nchunks;

    auto issue_a = [&](int c) {
        const unsigned char* w = record_of(a, bh, c) + kR2W;
        mbar_expect_tx(&sm.bar_a, kImgA);
        bulk_g2s(sm.imgA, w, 3 * kSwTile, &sm.bar_a);
        bulk_g2s(sm.imgA + 4 * kSwTile, w + 3 * kSwTile, 3 * kSwTile, &sm.bar_a);
        tma_tile(sm.imgA + 3 * kSwTile, &maps.q, 0, hk, c * kC, b, &sm.bar_a);
        tma_tile(sm.imgA + 7 * kSwTile, &maps.q, 64, hk, c * kC, b, &sm.bar_a);
    };
    auto issue_b = [&](int c) {
        mbar_expect_tx(&sm.bar_b, kImgB);
        tma_tile(sm.imgB, &maps.k, 0, hk, c * kC, b, &sm.bar_b);
        tma_tile(sm.imgB + kSwTile, &maps.k, 64, hk, c * kC, b, &sm.bar_b);
        bulk_g2s(sm.imgB + 2 * kSwTile, record_of(a, bh, c) + kR2P, kR2PBytes, &sm.bar_b);
    };
    auto issue_c = [&](int c) {
        mbar_expect_tx(&sm.bar_c, kImgC);
        bulk_g2s(sm.imgC, record_of(a, bh, c) + kR2G, kImgC, &sm.bar_c);
    };

    if (issuer) {
        mbar_init(&sm.bar_a);
        mbar_init(&sm.bar_b);
        mbar_init(&sm.bar_c);
        mbar_init(&sm.mma_g);
        mbar_init(&sm.mma_u);
        mbar_init(&sm.mma_o);
        mbar_init(&sm.e01, kScanThreads / 2);
        mbar_init(&sm.e23, kScanThreads / 2);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Launched with programmatic dependent launch behind the prepare kernel: the set-up
    // above overlaps its tail; the records, indices and pool are read only after it.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (issuer) {
        scan_prologue(a, b, sm.src, sm.dst, sm.status);
        if (sm.status == 0) {
            issue_a(0);
            issue_b(0);
            issue_c(0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    if (sm.status != 0) {
        if (warp == 0)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                         : "memory");
        return;
    }

    float s[32];  // S[j][32 quarter + i]
    {
        const float* M0 = a.pool + ((size_t)sm.src * a.Hv + h) * (kD * kD) + (size_t)(32 * quarter) * kD + j;
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = M0[(size_t)i * kD];
    }
    // A operand of the first products: S in three bf16 parts, row j, 8 key columns per granule.
    auto split_s = [&]() {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float x8[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) x8[m] = s[8 * u + m];
            uint4 p0, p1, p2;
            split3x8_fast(x8, p0, p1, p2);
            const uint32_t off = core_off(j, 32 * quarter + 8 * u, kD);
            *reinterpret_cast<uint4*>(sm.aop + off) = p0;
            *reinterpret_cast<uint4*>(sm.aop + kSPart + off) = p1;
            *reinterpret_cast<uint4*>(sm.aop + 2 * kSPart + off) = p2;
        }
    };
    split_s();

    constexpr uint32_t kIdesc256 = umma_idesc(128, 256), kIdesc192 = umma_idesc(128, 192);
    constexpr uint32_t kIdesc128 = umma_idesc(128, 128), kIdesc64 = umma_idesc(128, 64);
    bool ok = true;
    // The issuer's bookkeeping of what it started and saw complete (for the drain).
    int done_a = 0, done_b = 0, done_c = 0, issued_a = 1, issued_b = 1, issued_c = 1;
    int waits_g = 0, waits_u = 0, waits_o = 0, issued_g = 0, issued_u = 0, issued_o = 0;
    float qm[16];   // g_t (q_t M)_j for this thread's 16 tokens of the current chunk
    int out_t0 = 0, out_n = 0;  // chunk whose outputs are pending

    // Outputs of the chunk whose D_O was last completed, o = g q M + P E: tokens
    // 16 quarter + 8 part .. +8 of this thread's value row (warp-collective TMEM reads).
    auto store_outputs = [&](int part) {
        const uint32_t col = (uint32_t)(16 * quarter + 8 * part);
        uint32_t r0[8], r1[8];
        tmem_ld8_issue(tmem + lane_base + kTmemDO + col, r0);
        tmem_ld8_issue(tmem + lane_base + kTmemDO + kC + col, r1);
        tmem_wait_ld();
        tie_regs8(r0), tie_regs8(r1);
        float* ob = a.out + (((size_t)b * a.L + out_t0) * a.Hv + h) * kD + j;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int t = (int)col + m;
            if (t < out_n)
                ob[(size_t)t * a.Hv * kD] = qm[8 * part + m] + (__uint_as_float(r1[m]) + __uint_as_float(r0[m]));
        }
    };

    // One CTA barrier per chunk, before the first products (the S parts are written).
    // Every other hand-off is an mbarrier: the E parts of token quarters 0-1, then of
    // 2-3 (the state update's products on the first start while the second are formed),
    // and the copy and MMA completions, which each thread waits on itself.  What those
    // waits saw is carried to the next barrier, which stops the walk if any ran out.
    bool carry = true;
    int c = 0;
    for (; c < nch; ++c) {
        // --- the chunk's first products: S parts x [W parts | Q]
        bool got = carry;
        async_proxy_fence();  // the S parts just written, for the tensor cores
        if (issuer) got = wait_parity(&sm.bar_a, (uint32_t)c & 1u) && got;
        tc_fence_before();
        if (__syncthreads_or(got ? 0 : 1)) {
            ok = false;
            break;
        }
        tc_fence_after();
        carry = true;
        // The chunk's first products, issued by thread 0 in three batches (one per S
        // part) with its warp's share of the previous chunk's outputs stored in between;
        // the other warps store theirs while the products run.
        // B: K-steps of 16 features 32 bytes apart within a tile, the second feature half
        // four tiles on; each batch starts one tile (64 token rows) further in.
        const uint32_t aS = smem_u32(sm.aop), bW = smem_u32(sm.imgA);
        constexpr uint32_t kSboG = (kD / 8) * 128;
        auto bdesc = [&](int part, int ks) {
            return umma_desc_sw128(bW + part * kSwTile + (ks < 4 ? 32u * ks : 4 * kSwTile + 32u * (ks - 4)), 16, 1024);
        };
        if (warp == 0) {
            if (issuer) {
                ++done_a;
                for (int ks = 0; ks < kD / 16; ++ks)
                    umma_bf16(tmem, umma_desc(aS + 256 * ks, kSboG), bdesc(0, ks), kIdesc256, ks != 0 ? 1u : 0u);
            }
            __syncwarp();
            if (c > 0) store_outputs(0);
            if (issuer) {
                for (int ks = 0; ks < kD / 16; ++ks)
                    umma_bf16(tmem + kC, umma_desc(aS + kSPart + 256 * ks, kSboG), bdesc(1, ks), kIdesc192, 1u);
            }
            __syncwarp();
            if (c > 0) store_outputs(1);
            if (issuer) {
                for (int ks = 0; ks < kD / 16; ++ks)
                    umma_bf16(tmem + 2 * kC, umma_desc(aS + 2 * kSPart + 256 * ks, kSboG), bdesc(2, ks), kIdesc64,
                              1u);
                umma_commit(&sm.mma_g);
                ++issued_g;
            }
            __syncwarp();
        } else if (c > 0) {
            store_outputs(0);
            store_outputs(1);
        }

        got = wait_parity(&sm.mma_g, (uint32_t)c & 1u);
        if (issuer && got) {
            ++waits_g;
            if (c + 1 < nch) {  // the BW buffer is free again
                issue_a(c + 1);
                ++issued_a;
            }
        }
        {
            const bool gc = wait_parity(&sm.bar_c, (uint32_t)c & 1u);
            if (issuer && gc) ++done_c;
            got = got && gc;
        }
        tc_fence_after();
        // --- E = U - W M and g Q M for this thread's 16 tokens
        const float* gq = reinterpret_cast<const float*>(sm.imgC);
        const float gC = gq[2 * kC];
        // Quarters 0-1 (tokens 0..31) first: the state update's products on their E parts
        // run while quarters 2-3 form theirs.
        if (quarter >= 2) got = wait_parity(&sm.e01, (uint32_t)c & 1u) && got;
        {
            const float* gk = gq + kC;
            const float4* ut = reinterpret_cast<const float4*>(sm.imgC + kR2GBytes) + j;
            uint4 emid0;  // E_mid of the first 8 tokens (stored with the second 8)
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint32_t col = (uint32_t)(16 * quarter + 8 * p);
                uint32_t r0[8], r1[8], r2[8], r3[8];
                tmem_ld8_issue(tmem + lane_base + col, r0);
                tmem_ld8_issue(tmem + lane_base + kC + col, r1);
                tmem_ld8_issue(tmem + lane_base + 2 * kC + col, r2);
                tmem_ld8_issue(tmem + lane_base + 3 * kC + col, r3);
                tmem_wait_ld();
                tie_regs8(r0), tie_regs8(r1), tie_regs8(r2), tie_regs8(r3);
                float e[8], ep[8];
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4) {
                    const int gi = (int)(col / 4) + q4;
                    const float4 uu = ut[gi * kD];
                    const float uv[4] = {uu.x, uu.y, uu.z, uu.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int mm = 4 * q4 + m, t = (int)col + mm;
                        const float wm =
                            (__uint_as_float(r0[mm]) + __uint_as_float(r1[mm])) + __uint_as_float(r2[mm]);
                        e[mm] = uv[m] - wm;
                        ep[mm] = e[mm] * gk[t];
                        qm[8 * p + mm] = __uint_as_float(r3[mm]) * gq[t];
                    }
                }
                // Parts 0..3 over columns 4p.. of the first 8 of this thread's 16 columns of
                // G block 0..3 (read in pass 0); part 4 after pass 1, over the last 8 of block 0.
                uint4 p0, p1, p2, p3, p4;
                split3x8_fast(ep, p0, p1, p2);
                split2x8_fast(e, p3, p4);
                const uint32_t gb = tmem + lane_base + (uint32_t)(16 * quarter);
                tmem_st4(gb + 4 * p, p0);
                tmem_st4(gb + kC + 4 * p, p1);
                tmem_st4(gb + 2 * kC + 4 * p, p2);
                tmem_st4(gb + 3 * kC + 4 * p, p3);
                if (p == 0)
                    emid0 = p4;
                else
                    tmem_st8(gb + 8, emid0, p4);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(quarter < 2 ? &sm.e01 : &sm.e23);
        out_t0 = c * kC;
        out_n = min(kC, a.L - out_t0);
        // --- state update (committed first: the chain waits for it), then the outputs' products
        if (issuer) {
            // B = K, MN-major: features 64 to a row, tokens one row each (16 tokens per
            // MMA: 2048 bytes), the second feature half one tile on.
            const uint32_t bK = smem_u32(sm.imgB), bP = bK + 2 * kSwTile;
            constexpr uint32_t kSbo = (kC / 8) * 128;
            // A: E part p of the 16 tokens of K-step ks, in TMEM (written by token quarter ks).
            auto epart = [&](int p, int ks) -> uint32_t {
                return tmem + (uint32_t)(16 * ks) + (p < 4 ? (uint32_t)(p * kC) : 8u);
            };
            auto issue_du = [&](int k0) {  // K-steps k0, k0 + 1 (the tokens of two quarters)
                for (int ks = k0; ks < k0 + 2; ++ks)
                    for (int part = 0; part < 3; ++part)
                        umma_bf16_ta(tmem + kTmemDU, epart(part, ks),
                                     umma_desc_sw128(bK + 2048u * ks, kSwTile, 1024), kIdesc128 | kIdescBmn,
                                     (part | ks) != 0 ? 1u : 0u);
            };
            const bool g01 = wait_parity(&sm.e01, (uint32_t)c & 1u);
            const bool gb = wait_parity(&sm.bar_b, (uint32_t)c & 1u);
            if (gb) ++done_b;
            tc_fence_after();
            issue_du(0);
            const bool g23 = wait_parity(&sm.e23, (uint32_t)c & 1u);
            tc_fence_after();
            issue_du(2);
            umma_commit(&sm.mma_u);
            for (int ks = 0; ks < kC / 16; ++ks)
                umma_bf16_ta(tmem + kTmemDO, epart(3, ks), umma_desc(bP + 256 * ks, kSbo), kIdesc128,
                             ks != 0 ? 1u : 0u);
            for (int ks = 0; ks < kC / 16; ++ks)
                umma_bf16_ta(tmem + kTmemDO + kC, epart(4, ks), umma_desc(bP + (kC / 8) * kSbo + 256 * ks, kSbo),
                             kIdesc64, 1u);
            umma_commit(&sm.mma_o);
            ++issued_u, ++issued_o;
            got = got && g01 && gb && g23;
            if (got && c + 1 < nch) {  // U^T and the gate factors are consumed
                issue_c(c + 1);
                ++issued_c;
            }
        }
        {
            const bool gu = wait_parity(&sm.mma_u, (uint32_t)c & 1u);
            if (issuer && gu) ++waits_u;
            carry = gu && got;
        }
        tc_fence_after();
        {
            uint32_t r0[16], r1[16];
            tmem_ld16_issue(tmem + lane_base + kTmemDU + (uint32_t)(32 * quarter), r0);
            tmem_ld16_issue(tmem + lane_base + kTmemDU + (uint32_t)(32 * quarter + 16), r1);
            tmem_wait_ld();
            tie_regs(r0), tie_regs(r1);
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                s[m] = fmaf(gC, s[m], __uint_as_float(r0[m]));
                s[16 + m] = fmaf(gC, s[16 + m], __uint_as_float(r1[m]));
            }
        }
        // The next S parts (the first products are complete: the state update's commit
        // covers them), written while the outputs' products run.
        if (c + 1 < nch) split_s();
        // The outputs' products read the E parts in TMEM, which the next first products
        // overwrite, and the outputs are read from their accumulator next chunk.
        {
            const bool go = wait_parity(&sm.mma_o, (uint32_t)c & 1u);
            if (issuer && go) {
                ++waits_o;
                if (c + 1 < nch) {  // K^T and the P tile are consumed
                    issue_b(c + 1);
                    ++issued_b;
                }
            }
            carry = carry && go;
        }
        tc_fence_before();
    }
    if (ok) ok = !__syncthreads_or(carry ? 0 : 1);  // the last chunk's waits
    tc_fence_after();

    if (ok) {
        {
            store_outputs(0);  // the last chunk's
            store_outputs(1);
            float* MD = a.pool + ((size_t)sm.dst * a.Hv + h) * (kD * kD) + (size_t)(32 * quarter) * kD + j;
#pragma unroll
            for (int i = 0; i < 32; ++i) MD[(size_t)i * kD] = s[i];
        }
    } else if (issuer) {
        // Something never arrived: record it, then give every copy and MMA still
        // outstanding one more bounded wait before shared memory and TMEM go.
        record(a.err, GDN_ERR_TIMEOUT);
        for (; done_a < issued_a; ++done_a) wait_parity(&sm.bar_a, (uint32_t)done_a & 1u);
        for (; done_b < issued_b; ++done_b) wait_parity(&sm.bar_b, (uint32_t)done_b & 1u);
        for (; done_c < issued_c; ++done_c) wait_parity(&sm.bar_c, (uint32_t)done_c & 1u);
        for (; waits_g < issued_g; ++waits_g) wait_parity(&sm.mma_g, (uint32_t)waits_g & 1u);
        for (; waits_u < issued_u; ++waits_u) wait_parity(&sm.mma_u, (uint32_t)waits_u & 1u);
        for (; waits_o < issued_o; ++waits_o) wait_parity(&sm.mma_o, (uint32_t)waits_o & 1u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// Self-test of the bounded wait: one CTA waits on an mbarrier that nothing ever
// arrives on, with the given limit, and records GDN_ERR_TIMEOUT when it gives up.
__global__ void gdn_wait_selftest_kernel(uint64_t limit_ns, int32_t* err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const bool got = wait_parity(&bar, 0u, limit_ns);
    if (__syncthreads_or(got ? 0 : 1) && threadIdx.x == 0) record(err, GDN_ERR_TIMEOUT);
}

}  // namespace

extern "C" gdn_status gdn_wait_selftest(uint64_t limit_ns, int32_t* err_word, cudaStream_t stream) {
    if (err_word == nullptr || limit_ns == 0 || limit_ns > kWaitLimitNs) return GDN_ERR_INVALID_ARG;
    gdn_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err_word);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// The driver's tensor-map encoder, looked up once through the runtime (no link to the
// driver library); null if the driver does not export it.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn tensor_map_encoder() {
    static const EncodeTiledFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// Tensor maps of k, q ([B][L][Hk][dk]) and v ([B][L][Hv][dv]), bf16: dims {feature, head,
// token, request}, box 64 x 1 x 64 x 1, 128-byte swizzle, zero fill past L.  The
// addresses are 16-byte aligned and every stride a multiple of 256 bytes (checked by
// the caller), which is what the encoder asks for.
static gdn_status encode_tile_maps(TileMaps& m, const ChunkArgs& a) {
    const EncodeTiledFn enc = tensor_map_encoder();
    if (enc == nullptr) return GDN_ERR_CUDA;
    auto one = [&](CUtensorMap* map, const void* base, int H) {
        const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)a.L, (cuuint64_t)a.B};
        const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)a.L * H * kD * 2};
        const cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
        const cuuint32_t step[4] = {1, 1, 1, 1};
        return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, step,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!one(&m.k, a.k, a.Hk) || !one(&m.q, a.q, a.Hk) || !one(&m.v, a.v, a.Hv)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

extern "C" size_t gdn_prefill_workspace_bytes(int32_t B, int32_t L, int32_t Hv, int32_t dk, int32_t dv) {
    if (B < 0 || L < 1 || Hv < 1 || dk != kD || dv != kD) return 0;
    const size_t nchunks = ((size_t)L + kC - 1) / kC;
    return (size_t)B * Hv * nchunks * kRecBytes;
}

extern "C" gdn_status gdn_prefill_chunked(float* pool, int32_t num_slots, const int32_t* src_idx,
                                          const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                          const float* alpha, const float* beta, float* out, int32_t B, int32_t L,
                                          int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int32_t qkv_dtype,
                                          void* workspace, size_t workspace_bytes, int32_t* err_word,
                                          cudaStream_t stream) {
    if (B < 0 || L < 1 || Hk < 1 || Hv < 1 || num_slots < 1 || Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
    if (dk != kD || dv != kD) return GDN_ERR_INVALID_ARG;
    if (qkv_dtype != GDN_F32 && qkv_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    // err_word is required: a bounded wait that runs out leaves the request's checkpoint
    // and outputs unwritten and reports it only there.
    if (!pool || !src_idx || !dst_idx || !q || !k || !v || !alpha || !beta || !out || !workspace || !err_word)
        return GDN_ERR_INVALID_ARG;
    const int nchunks = (L + kC - 1) / kC;
    if (workspace_bytes < gdn_prefill_workspace_bytes(B, L, Hv, dk, dv)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Hv * nchunks * kNCB >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    // 16-byte vector accesses: workspace, pool, out, q, k, v (rows of 128 elements keep the alignment).
    const uintptr_t align = reinterpret_cast<uintptr_t>(workspace) | reinterpret_cast<uintptr_t>(pool) |
                            reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(q) |
                            reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v);
    if ((align & 15u) != 0) return GDN_ERR_INVALID_ARG;

    const ChunkArgs a{pool, src_idx, dst_idx, q, k, v, alpha, beta, out, static_cast<unsigned char*>(workspace),
                      err_word, num_slots, B, L, Hk, Hv, Hv / Hk, nchunks};
    const bool bf = qkv_dtype == GDN_BF16;
    const int s1 = bf ? kSmemP : (int)sizeof(Smem1), s2 = bf ? kSmemS : (int)sizeof(Smem2);
    TileMaps maps;
    if (bf) {
        const gdn_status st = encode_tile_maps(maps, a);
        if (st != GDN_OK) return st;
    }
    cudaError_t e = bf ? cudaFuncSetAttribute(gdn_chunk_prepare_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s1)
                       : cudaFuncSetAttribute(gdn_chunk_prepare_kernel<float>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    if (bf) {  // two prepare CTAs per SM need the largest shared-memory carveout
        e = cudaFuncSetAttribute(gdn_chunk_prepare_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return GDN_ERR_CUDA;
    }
    e = bf ? cudaFuncSetAttribute(gdn_chunk_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s2)
           : cudaFuncSetAttribute(gdn_chunk_scan_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const unsigned g1 = (unsigned)(B * Hv * nchunks);
    if (bf) {
        gdn_chunk_prepare_tc_kernel<<<g1, kNT, s1, stream>>>(a, maps);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
        // The scan starts behind the prepare kernel with programmatic dependent launch.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(B * Hv));
        cfg.blockDim = dim3(kScanThreads);
        cfg.dynamicSmemBytes = (size_t)s2;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, gdn_chunk_scan_tc_kernel, a, maps) != cudaSuccess) return GDN_ERR_CUDA;
    } else {
        const unsigned g2 = (unsigned)(B * Hv * kNCB);
        gdn_chunk_prepare_kernel<float><<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_kernel<float><<<g2, kNT, s2, stream>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
