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
// does not depend on the state into the caller's workspace; kernel 2 walks the
// chunks of each (request, head, column block) in order, carrying M in shared
// memory.  With bf16 inputs both kernels run their products on the tensor cores
// (tcgen05, accumulators in TMEM).  An operand that is not a bf16 input is fp32
// and enters as three bf16 parts (hi + mid + lo carries 24 bits), with every part
// product formed, which keeps fp32 accuracy.  In that form kernel 1 also computes
// W = Tb K, so that kernel 2 evaluates the same algebra re-associated:
//     E = U - W M0,   O = diag(g) (Q M0) + P E,   M_C = g_C M0 + K^T diag(g_C / g) E,
// all as MMAs.  With fp32 inputs (not exact in bf16) both kernels run on the CUDA
// cores in the first form.  Ratios g_t / g_i are formed as exp(log g_t - log g_i)
// <= 1, so nothing overflows; g_t itself may underflow to zero, which is its true
// value to fp32 precision.
//
// Workspace record of one (request, head, chunk), bytes.  The first parts are laid
// out as the shared-memory images the scan copies in (bulk copies, 16-byte granules):
//   A1  [W_hi; W_mid] then [W_lo; Q] as bf16, two 128 x 128 (dk) tiles in the
//       no-swizzle K-major core layout of the tensor-core operand, where
//       W = Tb K is split into three bf16 parts (bf16 inputs only)
//   A2  K^T as bf16, 128 (dk) rows x 64 tokens, same layout (bf16 inputs only)
//   PA  [P_hi; P_mid] then [P_lo; P_lo], P split into three bf16 parts, two 128 x 64
//       operand tiles (bf16 inputs only)
//   U   four column slabs [4][64][36] fp32 (32 columns + 4 padding each)
//   TbT [64][64] fp32: Tb transposed, TbT[i][t] = Tb[t][i], zero for t < i (fp32 inputs)
//   PT  [64][64] fp32: P transposed, PT[i][t] = P[t][i], zero for t < i (fp32 inputs)
//   G   log g [64]

#include "gdn_step.h"

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

// Workspace record (bytes).
constexpr size_t kRecA1 = 0;
constexpr size_t kA1Tile = (size_t)2 * kC * kD * 2;  // one 128 x 128 bf16 operand tile
constexpr size_t kRecA2 = kRecA1 + 2 * kA1Tile;
constexpr size_t kA2Tile = (size_t)kD * kC * 2;       // one 128 x 64 bf16 operand tile
constexpr size_t kRecPA = kRecA2 + kA2Tile;
constexpr size_t kRecU = kRecPA + 2 * kA2Tile;
constexpr size_t kUSlab = (size_t)kC * kUS * 4;
constexpr size_t kRecTb = kRecU + kNCB * kUSlab;
constexpr size_t kRecP = kRecTb + (size_t)kC * kC * 4;
constexpr size_t kRecG = kRecP + (size_t)kC * kC * 4;
constexpr size_t kRecBytes = kRecG + (size_t)kC * 4;
// One scan CTA's small image of a chunk in shared memory: its U slab | log g.
constexpr uint32_t kImgG = (uint32_t)kUSlab;
constexpr uint32_t kImgBytes = kImgG + (uint32_t)(kC * 4);
static_assert(kRecA2 % 16 == 0 && kRecPA % 16 == 0 && kRecU % 16 == 0 && kRecTb % 16 == 0 && kRecP % 16 == 0 &&
                  kRecBytes % 16 == 0,
              "16-byte records");
static_assert(kUSlab % 16 == 0 && kImgBytes % 16 == 0, "16-byte bulk copies");

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

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t* bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(1) : "memory");
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

// Eight fp32 values as three 16-byte granules of bf16 parts: x = hi + mid + lo.
__device__ __forceinline__ void split3x8(const float (&x)[8], uint4& hi, uint4& mid, uint4& lo) {
    uint32_t h[4], m[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a0 = x[2 * j], a1 = x[2 * j + 1];
        h[j] = pack_bf16x2(a0, a1);
        a0 -= __uint_as_float(h[j] << 16);
        a1 -= __uint_as_float(h[j] & 0xffff0000u);
        m[j] = pack_bf16x2(a0, a1);
        a0 -= __uint_as_float(m[j] << 16);
        a1 -= __uint_as_float(m[j] & 0xffff0000u);
        l[j] = pack_bf16x2(a0, a1);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    mid = make_uint4(m[0], m[1], m[2], m[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// ---------------------------------------------------------------------------
// Kernel 1 pieces shared by its two forms.
// ---------------------------------------------------------------------------

// Warp 0: log g_t = sum_{i<=t} log alpha_i by a warp scan over two 32-token
// halves, beta_t, and log g into the record.
__device__ __forceinline__ void gate_scan(const ChunkArgs& a, int b, int h, int t0, int n, int lane, float* lg,
                                          float* bt, float* Gs) {
    float carry = 0.f;
    for (int half = 0; half < 2; ++half) {
        const int t = half * 32 + lane;
        const size_t gi = (((size_t)b * a.L + t0 + t) * a.Hv + h);
        float la = 0.f, be = 0.f;
        if (t < n) {
            // alpha = 0 (a full reset) would make log g = -inf and the ratios
            // -inf - -inf; e^-80 ~ 2e-35 is zero at fp32 precision instead.
            la = fmaxf(logf(__ldg(a.alpha + gi)), -80.f);
            be = __ldg(a.beta + gi);
        }
        float x = la;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        lg[t] = carry + x;
        bt[t] = be;
        Gs[t] = carry + x;
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

// ---------------------------------------------------------------------------
// Kernel 1, tensor-core form (bf16 inputs).  The products with a bf16 input
// operand run as tcgen05 MMAs with fp32 accumulation in TMEM:
//   D0 = [K; Q] K^T                    (M = 128, N = 64, K = dk: 8 MMAs, exact products)
//   D1 = V^T (T diag(beta))^T = U^T    (M = 128 = dv, N = 64, K = 64 tokens; the fp32
//                                       factor in three bf16 parts: 12 MMAs)
//   D2 = K^T (T diag(beta g))^T = W^T  (the same with Tb: W = Tb K, 12 MMAs)
// W is split into three bf16 parts and stored as the scan's A operands
// [W_hi; W_mid] and [W_lo; Q], so that the scan forms E = U - W M0 and Q M0 on the
// tensor cores with no triangular product.  The inverse T and the gate scalings
// stay on the CUDA cores.
// ---------------------------------------------------------------------------
struct SmemP {
    union {
        unsigned char A1[2 * kC * kD * 2];        // [K; Q] operand of D0 (also B = K)
        float Y[16][48];                          // scratch of the inverse (after D0)
        struct {
            unsigned char VT[kD * kC * 2];        // V^T operand of D1
            unsigned char Bp[3][kC * kC * 2];     // (T diag(beta)) parts, B of D1
        } d1;
        struct {
            unsigned char KT[kD * kC * 2];        // K^T operand of D2
            unsigned char Bt[3][kC * kC * 2];     // (T diag(beta g)) parts, B of D2
        } d2;
        float W[kC][kD + 4];                      // W staged for its split (row stride spreads banks)
    } op;
    union {
        float A[kC][kC + 1];
        __nv_bfloat16 R[kC][kD + 2];  // V rows, later K rows (odd word stride for the column gathers)
    } av;
    float T[kC][kC + 1];
    float lg[kC];
    float bt[kC];
    uint64_t mma;
    uint32_t tmem;
};
static_assert(sizeof(SmemP) <= 74 * 1024 + 1024, "three prepare CTAs per SM");

// Column gather of a bf16 row block R (rows = tokens) into a K-major operand image
// with kD rows (dk or dv) and kC columns (tokens); optionally also to global memory.
// Consecutive threads write consecutive 16-byte granules.
__device__ __forceinline__ void gather_transposed(const __nv_bfloat16 (*R)[kD + 2], unsigned char* img,
                                                  unsigned char* global_img, int tid) {
    for (int e = tid; e < kD * (kC / 8); e += kNT) {
        const int j = (e & 7) | ((e >> 6) << 3), g = (e >> 3) & 7;  // row j, tokens 8g..8g+7
        uint16_t x[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) x[m] = *reinterpret_cast<const uint16_t*>(&R[8 * g + m][j]);
        uint4 w;
        w.x = x[0] | ((uint32_t)x[1] << 16);
        w.y = x[2] | ((uint32_t)x[3] << 16);
        w.z = x[4] | ((uint32_t)x[5] << 16);
        w.w = x[6] | ((uint32_t)x[7] << 16);
        const uint32_t off = core_off(j, 8 * g, kC);
        *reinterpret_cast<uint4*>(img + off) = w;
        if (global_img != nullptr) *reinterpret_cast<uint4*>(global_img + off) = w;
    }
}

// B operand (rows t, columns i) = T[t][i] * scale[i], in three bf16 parts.
__device__ __forceinline__ void split_scaled_T(const float (*T)[kC + 1], const float* scale,
                                               unsigned char (*parts)[kC * kC * 2], int tid) {
    for (int e = tid; e < kC * (kC / 8); e += kNT) {
        const int t = e % kC, g = e / kC;
        float x[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) x[m] = T[t][8 * g + m] * scale[8 * g + m];
        uint4 p0, p1, p2;
        split3x8(x, p0, p1, p2);
        const uint32_t off = core_off(t, 8 * g, kC);
        *reinterpret_cast<uint4*>(parts[0] + off) = p0;
        *reinterpret_cast<uint4*>(parts[1] + off) = p1;
        *reinterpret_cast<uint4*>(parts[2] + off) = p2;
    }
}

__global__ void __launch_bounds__(kNT, 3) gdn_chunk_prepare_tc_kernel(ChunkArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_p[];
    SmemP& sm = *reinterpret_cast<SmemP*>(smem_p);
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    const int c = blockIdx.x % a.nchunks;
    const int bh = blockIdx.x / a.nchunks;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int hk = h / a.G;
    const int t0 = c * kC;
    const int n = min(kC, a.L - t0);  // valid tokens; the rest are inert (k = q = v = 0, beta = 0, alpha = 1)
    unsigned char* rec = record_of(a, bh, c);
    float* Gs = reinterpret_cast<float*>(rec + kRecG);
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const int half = warp / 4;  // TMEM columns 32*half .. +31 of each accumulator
    constexpr uint32_t kIdesc = umma_idesc(128, kC);
    constexpr uint32_t kTmemU = 64;  // D1; D0 and then D2 use columns 0..63

    if (tid == 0) {
        mbar_init(&sm.mma);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(128)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        gate_scan(a, b, h, t0, n, lane, sm.lg, sm.bt, Gs);
    }
    // k, q, v in 16-byte granules: [K; Q] into the D0 operand image, Q also into the
    // record's [W_lo; Q] tile (rows 64..127); V stays in registers until the inverse is
    // done.  Consecutive threads take consecutive granules of the image: token
    // t = (e & 7) + 8 (e >> 7), group g = (e >> 3) & 15, e = tid + 256 u.
    constexpr int kGr = kC * (kD / 8) / kNT;  // granules per thread
    uint4 vkeep[kGr];
#pragma unroll
    for (int u = 0; u < kGr; ++u) {
        const int e = tid + kNT * u;
        const int t = (e & 7) | ((e >> 7) << 3), g = (e >> 3) & 15;
        uint4 kq = make_uint4(0, 0, 0, 0), qq = kq, vv = kq;
        if (t < n) {
            const size_t row = (((size_t)b * a.L + t0 + t) * a.Hk + hk) * kD + 8 * g;
            const size_t vrow = (((size_t)b * a.L + t0 + t) * a.Hv + h) * kD + 8 * g;
            kq = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + row));
            qq = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + row));
            vv = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.v) + vrow));
        }
        const uint32_t oq = core_off(kC + t, 8 * g, kD);
        *reinterpret_cast<uint4*>(sm.op.A1 + core_off(t, 8 * g, kD)) = kq;
        *reinterpret_cast<uint4*>(sm.op.A1 + oq) = qq;
        *reinterpret_cast<uint4*>(rec + kRecA1 + kA1Tile + oq) = qq;
        vkeep[u] = vv;
    }
    async_proxy_fence();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    if (tid == 0) {
        const uint32_t a1 = smem_u32(sm.op.A1);
        for (int ks = 0; ks < kD / 16; ++ks)
            umma_bf16(tmem, umma_desc(a1 + 256 * ks, (kD / 8) * 128), umma_desc(a1 + 256 * ks, (kD / 8) * 128),
                      kIdesc, ks != 0 ? 1u : 0u);
        umma_commit(&sm.mma);
    }
    int waits = 0, issued = 1;
    bool ok = !__syncthreads_or(wait_parity(&sm.mma, 0) ? 0 : 1);
    if (ok) {
        ++waits;
        tc_fence_after();
        // D0 row r < 64: k_r . k_i -> A (scaled); row 64 + t: q_t . k_i -> P (record).
        const int r = (warp % 4) * 32 + lane;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float v[16];
            const int i0 = 32 * half + 16 * part;
            tmem_ld16(tmem + lane_base + (uint32_t)i0, v);
            if (r < kC) {
                const float lt = sm.lg[r], bt = sm.bt[r];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int i = i0 + j;
                    sm.av.A[r][i] = i < r ? bt * expf(lt - sm.lg[i]) * v[j] : 0.f;
                }
            } else {
                // P row t, columns i0..i0+15, in three bf16 parts: [P_hi; P_mid] and [P_lo; P_lo].
                const int t = r - kC;
                const float lt = sm.lg[t];
#pragma unroll
                for (int g8 = 0; g8 < 16; g8 += 8) {
                    float x[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int i = i0 + g8 + j;
                        x[j] = i <= t ? expf(lt - sm.lg[i]) * v[g8 + j] : 0.f;
                    }
                    uint4 p0, p1, p2;
                    split3x8(x, p0, p1, p2);
                    unsigned char* pa = rec + kRecPA;
                    *reinterpret_cast<uint4*>(pa + core_off(t, i0 + g8, kC)) = p0;
                    *reinterpret_cast<uint4*>(pa + core_off(kC + t, i0 + g8, kC)) = p1;
                    *reinterpret_cast<uint4*>(pa + kA2Tile + core_off(t, i0 + g8, kC)) = p2;
                    *reinterpret_cast<uint4*>(pa + kA2Tile + core_off(kC + t, i0 + g8, kC)) = p2;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        invert_unit_lower(sm.av.A, sm.T, sm.op.Y, tid);  // the [K; Q] image is dead: D0 is complete
        // V rows over A (dead after the inverse)
#pragma unroll
        for (int u = 0; u < kGr; ++u) {
            const int e = tid + kNT * u;
            const int t = (e & 7) | ((e >> 7) << 3), g = (e >> 3) & 15;
            uint32_t* vr = reinterpret_cast<uint32_t*>(&sm.av.R[t][8 * g]);
            vr[0] = vkeep[u].x, vr[1] = vkeep[u].y, vr[2] = vkeep[u].z, vr[3] = vkeep[u].w;
        }
        if (tid < kC) sm.lg[tid] = sm.bt[tid] * expf(sm.lg[tid]);  // beta g: log g is in the record already
        __syncthreads();

        // D1 = U^T: V^T and (T diag(beta)) in parts.
        gather_transposed(sm.av.R, sm.op.d1.VT, nullptr, tid);
        split_scaled_T(sm.T, sm.bt, sm.op.d1.Bp, tid);
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t vt = smem_u32(sm.op.d1.VT);
            for (int part = 0; part < 3; ++part)
                for (int ks = 0; ks < kC / 16; ++ks)
                    umma_bf16(tmem + kTmemU, umma_desc(vt + 256 * ks, (kC / 8) * 128),
                              umma_desc(smem_u32(sm.op.d1.Bp[part]) + 256 * ks, (kC / 8) * 128), kIdesc,
                              (part | ks) != 0 ? 1u : 0u);
            umma_commit(&sm.mma);
        }
        ++issued;
        // K rows again (just read, so from L2) into the row buffer for the K^T image.
#pragma unroll
        for (int u = 0; u < kGr; ++u) {
            const int e = tid + kNT * u;
            const int t = (e & 7) | ((e >> 7) << 3), g = (e >> 3) & 15;
            uint4 kq = make_uint4(0, 0, 0, 0);
            if (t < n)
                kq = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) +
                                                          (((size_t)b * a.L + t0 + t) * a.Hk + hk) * kD + 8 * g));
            uint32_t* kr = reinterpret_cast<uint32_t*>(&sm.av.R[t][8 * g]);
            kr[0] = kq.x, kr[1] = kq.y, kr[2] = kq.z, kr[3] = kq.w;
        }
        ok = !__syncthreads_or(wait_parity(&sm.mma, 1) ? 0 : 1);
        if (ok) {
            ++waits;
            tc_fence_after();
            // D1[j][t] = U[t][j]: lane j of this warp's quadrant, tokens 32*half .. +31.
            const int j = (warp % 4) * 32 + lane;
            float* U = reinterpret_cast<float*>(rec + kRecU) + (j / kDVC) * (kC * kUS) + j % kDVC;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[16];
                const int tb = 32 * half + 16 * part;
                tmem_ld16(tmem + lane_base + kTmemU + (uint32_t)tb, v);
#pragma unroll
                for (int m = 0; m < 16; ++m) U[(tb + m) * kUS] = v[m];
            }
            // D2 = W^T: K^T (also the scan's operand, to the record) and (T diag(beta g)) in parts.
            gather_transposed(sm.av.R, sm.op.d2.KT, rec + kRecA2, tid);
            split_scaled_T(sm.T, sm.lg, sm.op.d2.Bt, tid);
            async_proxy_fence();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (tid == 0) {
                const uint32_t kt = smem_u32(sm.op.d2.KT);
                for (int part = 0; part < 3; ++part)
                    for (int ks = 0; ks < kC / 16; ++ks)
                        umma_bf16(tmem, umma_desc(kt + 256 * ks, (kC / 8) * 128),
                                  umma_desc(smem_u32(sm.op.d2.Bt[part]) + 256 * ks, (kC / 8) * 128), kIdesc,
                                  (part | ks) != 0 ? 1u : 0u);
                umma_commit(&sm.mma);
            }
            ++issued;
            ok = !__syncthreads_or(wait_parity(&sm.mma, 0) ? 0 : 1);
            if (ok) {
                ++waits;
                tc_fence_after();
                // D2[d][t] = W[t][d] -> W staged row-major (the operands of D2 are dead).
                const int d = (warp % 4) * 32 + lane;
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float v[16];
                    const int tb = 32 * half + 16 * part;
                    tmem_ld16(tmem + lane_base + (uint32_t)tb, v);
#pragma unroll
                    for (int m = 0; m < 16; ++m) sm.op.W[tb + m][d] = v[m];
                }
                __syncthreads();
                // [W_hi; W_mid] and [W_lo; (Q, written above)] to the record.
                for (int e = tid; e < kC * (kD / 8); e += kNT) {
                    const int t = (e & 7) | ((e >> 7) << 3), g = (e >> 3) & 15;
                    const float4 w0 = *reinterpret_cast<const float4*>(&sm.op.W[t][8 * g]);
                    const float4 w1 = *reinterpret_cast<const float4*>(&sm.op.W[t][8 * g + 4]);
                    const float x[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    uint4 p0, p1, p2;
                    split3x8(x, p0, p1, p2);
                    *reinterpret_cast<uint4*>(rec + kRecA1 + core_off(t, 8 * g, kD)) = p0;
                    *reinterpret_cast<uint4*>(rec + kRecA1 + core_off(kC + t, 8 * g, kD)) = p1;
                    *reinterpret_cast<uint4*>(rec + kRecA1 + kA1Tile + core_off(t, 8 * g, kD)) = p2;
                }
            }
        }
    }
    if (!ok && tid == 0) {
        record(a.err, GDN_ERR_TIMEOUT);
        for (; waits < issued; ++waits) wait_parity(&sm.mma, (uint32_t)waits & 1u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128) : "memory");
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
// Kernel 2, tensor-core form (bf16 inputs).  Per chunk, with the fp32 state block M
// (128 x 32, held in registers: each thread owns the 16 elements it reads from D2)
// split into three bf16 parts stacked along N = 3 x 32:
//   D1a = [W_hi; W_mid] [M_hi M_mid M_lo]   (8 MMAs, K = dk)
//   D1b = [W_lo; Q]     [M_hi M_mid M_lo]   (8 MMAs)
//   E   = U - (W_hi + W_mid + W_lo) M       (rows 0..63 of D1a and D1b, rows 64..127 of D1a)
//   QM  = diag(g) Q M                       (rows 64..127 of D1b)
//   D2  = K^T [E'_hi E'_mid E'_lo],  E' = diag(g_C / g) E   (4 MMAs, K = 64 tokens)
//   DOa = [P_hi; P_mid] [E_hi E_mid E_lo],  DOb = [P_lo; P_lo] [E parts]  (4 + 4 MMAs)
//   O   = QM + (P_hi + P_mid + P_lo) E,     M <- g_C M + D2
// The sequential chain holds no CUDA-core contraction.  The column groups of each
// accumulator are added when TMEM is read, and rows that two TMEM quadrants hold
// are combined through shared memory.  Operands sit in shared memory in the
// no-swizzle K-major core layout; the accumulators take 3 x 96 of 512 TMEM columns
// (D1a, then DOa, at 0; D1b, then DOb, at 128; D2 at 256), allocated by warp 0.
// Thread 0 issues the MMAs, commits them to an mbarrier, and streams the chunk
// images with cp.async.bulk: the A operands ([W; Q] tiles; K^T with the P tiles;
// one buffer each, refilled for the next chunk as soon as their MMAs complete) and
// the small image (U slab, log g; two buffers, two chunks ahead).  Every wait is bounded (2 s); a timeout is
// recorded and the CTA drains and exits.
// ---------------------------------------------------------------------------
constexpr uint32_t kBopPart = (uint32_t)kDVC * kD * 2;   // one bf16 part of M^T (32 x 128)
constexpr uint32_t kBopPartE = (uint32_t)kDVC * kC * 2;  // one bf16 part of E'^T (32 x 64)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemD1b = 128;
constexpr uint32_t kTmemD2 = 256;

struct SmemTC {
    unsigned char a1[2 * kA1Tile];      // [W_hi; W_mid] | [W_lo; Q]
    unsigned char a2[3 * kA2Tile];      // K^T (D2), [P_hi; P_mid] (DOa), [P_lo; P_lo] (DOb)
    unsigned char img[2][kImgBytes];    // small images, double-buffered
    unsigned char bop[3 * kBopPart];    // B operand, three stacked parts: M^T, later E'^T
    unsigned char bopE[3 * kBopPartE];  // B operand of DO: E^T in three stacked parts
    float S[kC][kUS];                   // rows handed between TMEM quadrants: W_mid M, then QM + P_mid E
    float QM[kC][kUS];                  // diag(g) Q M
    uint64_t full[2];                   // small images
    uint64_t bar_a1, bar_a2, mma;
    uint32_t tmem;
    int src, dst, status;
};

// 8 x 8 transpose of 32-bit values across each group of 8 lanes: on entry lane l
// (l = lane % 8) holds row l of the block in x[0..7]; on return it holds column l
// (x[r] = row r's element l).  Three butterfly stages exchange 4 x 4, 2 x 2 and
// 1 x 1 sub-blocks with the partner lane l ^ s.
__device__ __forceinline__ void transpose8(float (&x)[8], int lane) {
#pragma unroll
    for (int s = 4; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (c & s) continue;
            const float send = upper ? x[c] : x[c + s];
            const float got = __shfl_xor_sync(0xffffffffu, send, s);
            if (upper)
                x[c] = got;
            else
                x[c + s] = got;
        }
    }
}

__global__ void __launch_bounds__(kNT, 1) gdn_chunk_scan_tc_kernel(ChunkArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_tc[];
    SmemTC& sm = *reinterpret_cast<SmemTC*>(smem_tc);
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    const int cb = blockIdx.x % kNCB;
    const int bh = blockIdx.x / kNCB;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int col0 = cb * kDVC;
    constexpr uint32_t kIdesc = umma_idesc(128, 3 * kDVC);
    const int nch = a.nchunks;

    // Thread 0's copies.  Every barrier completes once per chunk (or once per
    // use of its buffer), so the parity of the n-th completion is n & 1.
    auto issue_small = [&](int c) {
        const unsigned char* rec = record_of(a, bh, c);
        unsigned char* dst = sm.img[c & 1];
        uint64_t* bar = &sm.full[c & 1];
        mbar_expect_tx(bar, kImgBytes);
        bulk_g2s(dst, rec + kRecU + cb * kUSlab, (uint32_t)kUSlab, bar);
        bulk_g2s(dst + kImgG, rec + kRecG, (uint32_t)(kC * 4), bar);
    };
    auto issue_a1 = [&](int c) {
        mbar_expect_tx(&sm.bar_a1, (uint32_t)(2 * kA1Tile));
        bulk_g2s(sm.a1, record_of(a, bh, c) + kRecA1, (uint32_t)(2 * kA1Tile), &sm.bar_a1);
    };
    auto issue_a2 = [&](int c) {
        mbar_expect_tx(&sm.bar_a2, (uint32_t)(3 * kA2Tile));
        bulk_g2s(sm.a2, record_of(a, bh, c) + kRecA2, (uint32_t)(3 * kA2Tile), &sm.bar_a2);
    };

    if (tid == 0) {
        scan_prologue(a, b, sm.src, sm.dst, sm.status);
        mbar_init(&sm.full[0]);
        mbar_init(&sm.full[1]);
        mbar_init(&sm.bar_a1);
        mbar_init(&sm.bar_a2);
        mbar_init(&sm.mma);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (sm.status == 0) {
            issue_a1(0);
            issue_a2(0);
            issue_small(0);
            if (nch > 1) issue_small(1);
        }
    }
    __syncthreads();
    if (sm.status != 0) return;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const int half = warp / 4;             // TMEM columns half*16 .. +15 of each 32-column group
    const int row = (warp % 4) * 32 + lane;  // TMEM lane
    // The state block lives in registers: this thread owns M[row][half*16 .. +15], the
    // elements it reads from D2 in every state update.
    float m[16];
    {
        const float4* M0 = reinterpret_cast<const float4*>(a.pool + ((size_t)sm.src * a.Hv + h) * (kD * kD) +
                                                           (size_t)row * kD + col0 + half * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 v = M0[j];
            m[4 * j] = v.x, m[4 * j + 1] = v.y, m[4 * j + 2] = v.z, m[4 * j + 3] = v.w;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    const uint64_t da1 = umma_desc(smem_u32(sm.a1), (kD / 8) * 128);
    const uint64_t da1b = umma_desc(smem_u32(sm.a1 + kA1Tile), (kD / 8) * 128);
    const uint64_t da2 = umma_desc(smem_u32(sm.a2), (kC / 8) * 128);
    const uint64_t dpa = umma_desc(smem_u32(sm.a2 + kA2Tile), (kC / 8) * 128);
    const uint64_t dpb = umma_desc(smem_u32(sm.a2 + 2 * kA2Tile), (kC / 8) * 128);
    bool ok = true;
    int c = 0;
    int waits_mma = 0;   // completed waits per barrier (all threads); thread 0 also
    int done_a1 = 0, done_a2 = 0, done_small = 0;  // counts what it issued, below
    int issued_a1 = 1, issued_a2 = 1, issued_small = min(nch, 2), issued_mma = 0;

    // Sum of the three column groups (bf16 parts) of an accumulator, 16 columns at col:
    // the three loads are in flight together.
    auto read3 = [&](uint32_t col, float (&v)[16]) {
        uint32_t r0[16], r1[16], r2[16];
        tmem_ld16_issue(tmem + lane_base + col, r0);
        tmem_ld16_issue(tmem + lane_base + col + kDVC, r1);
        tmem_ld16_issue(tmem + lane_base + col + 2 * kDVC, r2);
        tmem_wait_ld();
        tie_regs(r0), tie_regs(r1), tie_regs(r2);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            v[j] = (__uint_as_float(r2[j]) + __uint_as_float(r1[j])) + __uint_as_float(r0[j]);
    };

    // B of D1: M^T (32 rows x 128) in three bf16 parts, 8 k-values per granule.  Each
    // group of 8 lanes transposes its 8 rows x 16 columns, so that lane l holds columns
    // l and 8 + l of those rows: two granules.  The caller fences and synchronises.
    auto split_m = [&]() {
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = m[8 * blk + j];
            transpose8(x, lane);
            uint4 p0, p1, p2;
            split3x8(x, p0, p1, p2);
            const uint32_t off = core_off(half * 16 + 8 * blk + (lane & 7), row & ~7, kD);
            *reinterpret_cast<uint4*>(sm.bop + off) = p0;
            *reinterpret_cast<uint4*>(sm.bop + kBopPart + off) = p1;
            *reinterpret_cast<uint4*>(sm.bop + 2 * kBopPart + off) = p2;
        }
        async_proxy_fence();
    };
    split_m();  // the first chunk's; the barrier after the first wait orders it before the MMAs

    for (; c < nch; ++c) {
        const int s = c & 1;
        bool got = wait_parity(&sm.full[s], (uint32_t)(c >> 1) & 1u);
        got = wait_parity(&sm.bar_a1, (uint32_t)c & 1u) && got;
        if (__syncthreads_or(got ? 0 : 1)) {
            ok = false;
            break;
        }
        ++done_small, ++done_a1;
        unsigned char* img = sm.img[s];
        float* U = reinterpret_cast<float*>(img);  // [64][kUS]: U, then E
        const float* lg = reinterpret_cast<const float*>(img + kImgG);
        const int t0 = c * kC;
        const int n = min(kC, a.L - t0);

        // (B of D1, the parts of M, was built after the previous state update.)
        if (tid == 0) {
            const uint64_t db = umma_desc(smem_u32(sm.bop), (kD / 8) * 128);
            for (int ks = 0; ks < kD / 16; ++ks) umma_bf16(tmem, da1 + 16 * ks, db + 16 * ks, kIdesc, ks != 0 ? 1u : 0u);
            for (int ks = 0; ks < kD / 16; ++ks)
                umma_bf16(tmem + kTmemD1b, da1b + 16 * ks, db + 16 * ks, kIdesc, ks != 0 ? 1u : 0u);
            umma_commit(&sm.mma);
        }
        ++issued_mma;
        // The decision to read TMEM is block-uniform (tcgen05.ld is warp-collective).
        if (__syncthreads_or(wait_parity(&sm.mma, (uint32_t)waits_mma & 1u) ? 0 : 1)) {
            ok = false;
            break;
        }
        ++waits_mma;
        tc_fence_after();
        if (c + 1 < nch) {  // the [W; Q] buffer is free again
            if (tid == 0) issue_a1(c + 1);
            ++issued_a1;
        }
        // Rows 64..127: W_mid M (handed over through S) and Q M (scaled by g, to the record).
        // Rows 0..63: E = U - (W_hi M + W_lo M + W_mid M), in place over U and to the record.
        {
            float va[16], vb[16];
            read3((uint32_t)(half * 16), va);
            read3(kTmemD1b + (uint32_t)(half * 16), vb);
            if (row >= kC) {
                const int t = row - kC;
                const float g = expf(lg[t]);
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    *reinterpret_cast<float4*>(&sm.S[t][half * 16 + j]) = make_float4(va[j], va[j + 1], va[j + 2], va[j + 3]);
                    *reinterpret_cast<float4*>(&sm.QM[t][half * 16 + j]) =
                        make_float4(vb[j] * g, vb[j + 1] * g, vb[j + 2] * g, vb[j + 3] * g);
                }
            }
            tc_fence_before();
            __syncthreads();
            if (row < kC) {
                float* ur = U + row * kUS + half * 16;
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 u = *reinterpret_cast<const float4*>(ur + j);
                    const float4 m = *reinterpret_cast<const float4*>(&sm.S[row][half * 16 + j]);
                    *reinterpret_cast<float4*>(ur + j) =
                        make_float4(u.x - ((vb[j] + m.x) + va[j]), u.y - ((vb[j + 1] + m.y) + va[j + 1]),
                                    u.z - ((vb[j + 2] + m.z) + va[j + 2]), u.w - ((vb[j + 3] + m.w) + va[j + 3]));
                }
            }
        }
        __syncthreads();

        // B of D2: E' = diag(g_C / g) E, and B of DO: E, both transposed (32 rows x 64
        // tokens) in three bf16 parts.
        {
            const int jj = tid % kDVC, g = tid / kDVC;  // 32 x 8 granules, one per thread
            const float lgC = lg[kC - 1];
            float x[8], y[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                x[j] = U[(8 * g + j) * kUS + jj];
                y[j] = x[j] * expf(lgC - lg[8 * g + j]);
            }
            uint4 p0, p1, p2;
            const uint32_t off = core_off(jj, 8 * g, kC);
            split3x8(y, p0, p1, p2);
            *reinterpret_cast<uint4*>(sm.bop + off) = p0;
            *reinterpret_cast<uint4*>(sm.bop + kBopPartE + off) = p1;
            *reinterpret_cast<uint4*>(sm.bop + 2 * kBopPartE + off) = p2;
            split3x8(x, p0, p1, p2);
            *reinterpret_cast<uint4*>(sm.bopE + off) = p0;
            *reinterpret_cast<uint4*>(sm.bopE + kBopPartE + off) = p1;
            *reinterpret_cast<uint4*>(sm.bopE + 2 * kBopPartE + off) = p2;
        }
        got = wait_parity(&sm.bar_a2, (uint32_t)c & 1u);
        async_proxy_fence();
        tc_fence_before();
        if (__syncthreads_or(got ? 0 : 1)) {
            ok = false;
            break;
        }
        ++done_a2;
        tc_fence_after();
        if (tid == 0) {
            const uint64_t db = umma_desc(smem_u32(sm.bop), (kC / 8) * 128);
            const uint64_t de = umma_desc(smem_u32(sm.bopE), (kC / 8) * 128);
            for (int ks = 0; ks < kC / 16; ++ks)
                umma_bf16(tmem + kTmemD2, da2 + 16 * ks, db + 16 * ks, kIdesc, ks != 0 ? 1u : 0u);
            for (int ks = 0; ks < kC / 16; ++ks)
                umma_bf16(tmem, dpa + 16 * ks, de + 16 * ks, kIdesc, ks != 0 ? 1u : 0u);
            for (int ks = 0; ks < kC / 16; ++ks)
                umma_bf16(tmem + kTmemD1b, dpb + 16 * ks, de + 16 * ks, kIdesc, ks != 0 ? 1u : 0u);
            umma_commit(&sm.mma);
        }
        ++issued_mma;

        if (__syncthreads_or(wait_parity(&sm.mma, (uint32_t)waits_mma & 1u) ? 0 : 1)) {
            ok = false;
            break;
        }
        ++waits_mma;
        tc_fence_after();
        if (c + 1 < nch) {  // the K^T and P buffer is free again
            if (tid == 0) issue_a2(c + 1);
            ++issued_a2;
        }
        // O: rows 64..127 of DOa (P_mid E) plus QM go through S to the warps holding rows
        // 0..63 of DOa (P_hi E) and DOb (P_lo E), which write the chunk's outputs.
        {
            float vo[16];
            read3((uint32_t)(half * 16), vo);
            if (row >= kC) {
                const int t = row - kC;
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 q = *reinterpret_cast<const float4*>(&sm.QM[t][half * 16 + j]);
                    *reinterpret_cast<float4*>(&sm.S[t][half * 16 + j]) =
                        make_float4(q.x + vo[j], q.y + vo[j + 1], q.z + vo[j + 2], q.w + vo[j + 3]);
                }
            }
            float vl[16];
            read3(kTmemD1b + (uint32_t)(half * 16), vl);
            tc_fence_before();
            __syncthreads();
            if (row < n) {
                float* ob = a.out + (((size_t)b * a.L + t0 + row) * a.Hv + h) * kD + col0 + half * 16;
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 sq = *reinterpret_cast<const float4*>(&sm.S[row][half * 16 + j]);
                    *reinterpret_cast<float4*>(ob + j) =
                        make_float4(sq.x + (vl[j] + vo[j]), sq.y + (vl[j + 1] + vo[j + 1]),
                                    sq.z + (vl[j + 2] + vo[j + 2]), sq.w + (vl[j + 3] + vo[j + 3]));
                }
            }
        }
        {
            float v[16];
            read3(kTmemD2 + (uint32_t)(half * 16), v);
            const float gC = expf(lg[kC - 1]);
#pragma unroll
            for (int j = 0; j < 16; ++j) m[j] = fmaf(gC, m[j], v[j]);
        }
        if (c + 1 < nch) split_m();  // the next chunk's B of D1 (the D2 MMAs, last readers of bop, are done)
        // Small buffer s (E was written into it) is refilled next by the async proxy.
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (c + 2 < nch) {
            if (tid == 0) issue_small(c + 2);
            ++issued_small;
        }
    }

    if (ok) {
        float4* MD = reinterpret_cast<float4*>(a.pool + ((size_t)sm.dst * a.Hv + h) * (kD * kD) + (size_t)row * kD +
                                               col0 + half * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) MD[j] = make_float4(m[4 * j], m[4 * j + 1], m[4 * j + 2], m[4 * j + 3]);
    } else if (tid == 0) {
        // Something never arrived: record it, then give every copy and MMA still
        // outstanding one more bounded wait before shared memory and TMEM go.
        record(a.err, GDN_ERR_TIMEOUT);
        for (; done_small < issued_small; ++done_small)
            wait_parity(&sm.full[done_small & 1], (uint32_t)(done_small >> 1) & 1u);
        for (; done_a1 < issued_a1; ++done_a1) wait_parity(&sm.bar_a1, (uint32_t)done_a1 & 1u);
        for (; done_a2 < issued_a2; ++done_a2) wait_parity(&sm.bar_a2, (uint32_t)done_a2 & 1u);
        for (; waits_mma < issued_mma; ++waits_mma) wait_parity(&sm.mma, (uint32_t)waits_mma & 1u);
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
    const int s1 = bf ? (int)sizeof(SmemP) : (int)sizeof(Smem1), s2 = bf ? (int)sizeof(SmemTC) : (int)sizeof(Smem2);
    cudaError_t e = bf ? cudaFuncSetAttribute(gdn_chunk_prepare_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s1)
                       : cudaFuncSetAttribute(gdn_chunk_prepare_kernel<float>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    if (bf) {  // three prepare CTAs per SM need the largest shared-memory carveout
        e = cudaFuncSetAttribute(gdn_chunk_prepare_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return GDN_ERR_CUDA;
    }
    e = bf ? cudaFuncSetAttribute(gdn_chunk_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s2)
           : cudaFuncSetAttribute(gdn_chunk_scan_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const unsigned g1 = (unsigned)(B * Hv * nchunks), g2 = (unsigned)(B * Hv * kNCB);
    if (bf) {
        gdn_chunk_prepare_tc_kernel<<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_tc_kernel<<<g2, kNT, s2, stream>>>(a);
    } else {
        gdn_chunk_prepare_kernel<float><<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_kernel<float><<<g2, kNT, s2, stream>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
