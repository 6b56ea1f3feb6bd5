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
// Kernel 1 builds, for every (request, head, chunk) in parallel, U, Tb, P and
// the log-gates (log g_t) into the caller's workspace; kernel 2 walks the chunks
// of each (request, head, column block) in order, carrying M in shared memory.
// The large products of kernel 2 ([K; Q] M0 and K^T E) have one operand that is
// exact in bf16 (the bf16 inputs k, q) and one fp32 operand; with bf16 inputs
// they run on the tensor cores (tcgen05, accumulators in TMEM) with the fp32
// operand split into three bf16 parts (hi + mid + lo carries 24 bits), which
// keeps fp32 accuracy.  The triangular products stay on the CUDA cores.
// Ratios g_t / g_i are formed as exp(log g_t - log g_i) <= 1, so nothing
// overflows; g_t itself may underflow to zero, which is its true value to fp32
// precision.
//
// Workspace record of one (request, head, chunk), bytes, laid out as the
// shared-memory image kernel 2 copies in (bulk copies, 16-byte granules):
//   A1  [K; Q] as bf16, 128 rows x 128 (dk) in the no-swizzle K-major core
//       layout of the tensor-core operand (bf16 inputs only)
//   A2  K^T as bf16, 128 (dk) rows x 64 tokens, same layout (bf16 inputs only)
//   U   four column slabs [4][64][36] fp32 (32 columns + 4 padding each)
//   TP  [64][65] fp32: Tb on and below the diagonal, P^T strictly above it
//   G   log g [64], then the diagonal of P [64]

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
constexpr int kTS = kC + 1;     // row stride of TP
constexpr int kPad = 4;         // row padding of [C][D] shared arrays in the fp32 scan kernel

// Workspace record (bytes).
constexpr size_t kRecA1 = 0;
constexpr size_t kRecA2 = kRecA1 + (size_t)2 * kC * kD * 2;
constexpr size_t kRecU = kRecA2 + (size_t)kD * kC * 2;
constexpr size_t kUSlab = (size_t)kC * kUS * 4;
constexpr size_t kRecTP = kRecU + kNCB * kUSlab;
constexpr size_t kRecG = kRecTP + (size_t)kC * kTS * 4;
constexpr size_t kRecBytes = kRecG + (size_t)2 * kC * 4;
// One CTA's image of a chunk in shared memory: A1 A2 | its U slab | TP G.
constexpr uint32_t kBufA2 = (uint32_t)kRecA2;
constexpr uint32_t kBufU = (uint32_t)kRecU;
constexpr uint32_t kBufTP = kBufU + (uint32_t)kUSlab;
constexpr uint32_t kBufG = kBufTP + (uint32_t)((size_t)kC * kTS * 4);
constexpr uint32_t kBufBytes = kBufG + 2 * kC * 4;
static_assert(kRecU % 16 == 0 && kRecTP % 16 == 0 && kRecG % 16 == 0 && kRecBytes % 16 == 0, "16-byte records");
static_assert(kUSlab % 16 == 0 && kBufTP % 16 == 0 && kBufBytes % 16 == 0, "16-byte bulk copies");
static_assert(kRecG - kRecTP == kBufG - kBufTP, "TP and G are copied together");

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

// 8 consecutive input elements (a 16-byte aligned group for bf16, 32 bytes for fp32) as fp32.
template <typename InT>
__device__ __forceinline__ void ld8(const void* base, size_t idx, float (&x)[8]);
template <>
__device__ __forceinline__ void ld8<float>(const void* base, size_t idx, float (&x)[8]) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
}
template <>
__device__ __forceinline__ void ld8<__nv_bfloat16>(const void* base, size_t idx, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[2 * j] = __uint_as_float(w[j] << 16);
        x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
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
// Kernel 1: per (b, h, chunk), independent of the state.
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
    float* TP = reinterpret_cast<float*>(rec + kRecTP);
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
    if (tid < 32) {
        // log g_t = sum_{i<=t} log alpha_i by a warp scan over two 32-token halves.
        float carry = 0.f;
        for (int half = 0; half < 2; ++half) {
            const int t = half * 32 + tid;
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
                if (tid >= off) x += y;
            }
            sm.lg[t] = carry + x;
            sm.bt[t] = be;
            Gs[t] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    __syncthreads();

    // KK (strictly lower, scaled into A) and QK (lower, scaled into P), 4x4 per thread:
    // rows ty*4 + r (broadcast within a half-warp), columns tx + 16 s (16 consecutive
    // rows of K, conflict-free with the odd row stride).  P goes to the workspace:
    // strictly below the diagonal transposed into TP's upper triangle, the diagonal to G.
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
                if (i < t)
                    TP[i * kTS + t] = ratio * qk[r][s];
                else if (i == t)
                    Gs[kC + t] = qk[r][s];
            }
    }
    // The tensor-core operands of kernel 2: [K; Q] and K^T as bf16 (exact: the
    // inputs are bf16) in the K-major core layout, one 16-byte granule per store;
    // consecutive threads write consecutive granules.
    if constexpr (sizeof(InT) == 2) {
        for (int e = tid; e < 2 * kC * (kD / 8); e += kNT) {
            const int r = (e & 7) | ((e >> 7) << 3), g = (e >> 3) & 15;  // row, k-group
            const float* src = r < kC ? &sm.K[r][8 * g] : &sm.X[r - kC][8 * g];
            uint4 w;
            w.x = pack_bf16x2(src[0], src[1]);
            w.y = pack_bf16x2(src[2], src[3]);
            w.z = pack_bf16x2(src[4], src[5]);
            w.w = pack_bf16x2(src[6], src[7]);
            *reinterpret_cast<uint4*>(rec + kRecA1 + core_off(r, 8 * g, kD)) = w;
        }
        for (int e = tid; e < kD * (kC / 8); e += kNT) {
            const int d = (e & 7) | ((e >> 6) << 3), g = (e >> 3) & 7;  // dk row, token group
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = sm.K[8 * g + j][d];
            uint4 w;
            w.x = pack_bf16x2(x[0], x[1]);
            w.y = pack_bf16x2(x[2], x[3]);
            w.z = pack_bf16x2(x[4], x[5]);
            w.w = pack_bf16x2(x[6], x[7]);
            *reinterpret_cast<uint4*>(rec + kRecA2 + core_off(d, 8 * g, kC)) = w;
        }
    }
    __syncthreads();

    // T = (I + A)^-1, blocked in 16 x 16: diagonal blocks by forward substitution
    // (one warp each), then block rows I = 1..3: T_IJ = -T_II sum_{J<=K<I} A_IK T_KJ.
    {
        const int w = tid / 32, lane = tid % 32;
        if (w < 4) {
            const int o = w * 16;
            for (int r = 0; r < 16; ++r) {
                if (lane < 16) {
                    const int j = lane;
                    float val = (r == j) ? 1.f : 0.f;
                    if (j < r) {
                        float acc = 0.f;
                        for (int m = j; m < r; ++m) acc = fmaf(sm.A[o + r][o + m], sm.T[o + m][o + j], acc);
                        val = -acc;
                    }
                    sm.T[o + r][o + j] = val;
                }
                __syncwarp();
            }
        }
        // zero the strictly upper blocks
        for (int e = tid; e < kC * kC; e += kNT) {
            const int r = e / kC, j = e % kC;
            if (j / 16 > r / 16) sm.T[r][j] = 0.f;
        }
        __syncthreads();
        for (int I = 1; I < 4; ++I) {
            // Y[r][J*16 + j] = sum_{K=J}^{I-1} sum_m A[16I + r][16K + m] T[16K + m][16J + j]
            for (int e = tid; e < 16 * 16 * I; e += kNT) {
                const int r = e / (16 * I), col = e % (16 * I);
                const int J = col / 16, j = col % 16;
                float acc = 0.f;
                for (int kk2 = 16 * J; kk2 < 16 * I; ++kk2) acc = fmaf(sm.A[16 * I + r][kk2], sm.T[kk2][16 * J + j], acc);
                sm.Y[r][col] = acc;
            }
            __syncthreads();
            for (int e = tid; e < 16 * 16 * I; e += kNT) {
                const int r = e / (16 * I), col = e % (16 * I);
                float acc = 0.f;
                for (int m = 0; m <= r; ++m) acc = fmaf(sm.T[16 * I + r][16 * I + m], sm.Y[m][col], acc);
                sm.T[16 * I + r][col] = -acc;
            }
            __syncthreads();
        }
    }

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
            const int t = e / kC, i = e % kC;
            if (i <= t) TP[t * kTS + i] = sm.T[t][i] * (sm.bt[i] * expf(sm.lg[i]));
        }
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
        const float* TP = reinterpret_cast<const float*>(rec + kRecTP);
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
            sm.Tb[t][i] = i <= t ? TP[t * kTS + i] : 0.f;
            sm.P[t][i] = i < t ? TP[i * kTS + t] : (i == t ? Gs[kC + t] : 0.f);
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
// Kernel 2, tensor-core form (bf16 inputs).  Per chunk:
//   D1 = [K; Q] M      (M=128: rows 0..63 are K M, rows 64..127 Q M; N = kDVC;
//                       K = dk in 8 steps; M split into 3 bf16 parts -> 24 MMAs)
//   D2 = K^T E'        (M=128 rows of dk, N = kDVC, K = 64 tokens in 4 steps,
//                       E' = diag(g_C / g) E split into 3 bf16 parts -> 12 MMAs)
// Operands sit in shared memory in the no-swizzle K-major core layout;
// accumulators live in 64 TMEM columns (D1 at column 0, D2 at column 32)
// allocated by warp 0.  Thread 0 issues the MMAs and commits them to an
// mbarrier, and streams the chunk images: the image of chunk c + 2 is copied
// (cp.async.bulk, two buffers) while chunk c + 1's waits and chunk c computes.
// The triangular products (Tb KM, P E) run on the CUDA cores, each thread on a
// row pair (p, 63 - p) so that every thread does the same 65 row-steps.  Every
// wait is bounded (2 s); a timeout is recorded and the CTA drains and exits.
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

__device__ __forceinline__ bool wait_parity(uint64_t* bar, uint32_t parity) {
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
        if (t1 - t0 > 2000000000ull) return false;  // 2 s
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

constexpr uint32_t kBopPart = (uint32_t)kDVC * kD * 2;  // one bf16 part of M^T (32 x 128)

struct SmemTC {
    unsigned char buf[2][kBufBytes];  // chunk images (A1 A2 U TP G), double-buffered
    unsigned char bop[3][kBopPart];   // B operand parts: M^T, later E'^T (32 x 64, same slots)
    float M[kD][kUS];                 // state block [dk][32 columns]
    float KM[kC][kUS];
    float QM[kC][kUS];                // g Q M
    uint64_t full[2];
    uint64_t mma;
    uint32_t tmem;
    int src, dst, status;
};

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
    constexpr uint32_t kIdesc = umma_idesc(128, kDVC);
    const int nch = a.nchunks;

    // Thread 0 copies chunk c's image into buffer c & 1.
    auto issue = [&](int c) {
        const unsigned char* rec = record_of(a, bh, c);
        unsigned char* dst = sm.buf[c & 1];
        uint64_t* bar = &sm.full[c & 1];
        mbar_expect_tx(bar, kBufBytes);
        bulk_g2s(dst, rec, (uint32_t)kRecU, bar);
        bulk_g2s(dst + kBufU, rec + kRecU + cb * kUSlab, (uint32_t)kUSlab, bar);
        bulk_g2s(dst + kBufTP, rec + kRecTP, (uint32_t)(kRecBytes - kRecTP), bar);
    };

    if (tid == 0) {
        scan_prologue(a, b, sm.src, sm.dst, sm.status);
        mbar_init(&sm.full[0]);
        mbar_init(&sm.full[1]);
        mbar_init(&sm.mma);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (sm.status == 0) {
            issue(0);
            if (nch > 1) issue(1);
        }
    }
    __syncthreads();
    if (sm.status != 0) return;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(64)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    {
        const float* M0 = a.pool + ((size_t)sm.src * a.Hv + h) * (kD * kD) + col0;
        for (int e = tid; e < kD * (kDVC / 4); e += kNT) {
            const int i = e / (kDVC / 4), j4 = e % (kDVC / 4);
            *reinterpret_cast<float4*>(&sm.M[i][4 * j4]) = *reinterpret_cast<const float4*>(M0 + (size_t)i * kD + 4 * j4);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const int half = warp / 4;          // TMEM columns half*16 .. +15
    const int tx = tid % 8, p = tid / 8; // triangular phases: columns 4tx..4tx+3, rows p and 63-p
    const int rlo = p, rhi = kC - 1 - p;
    bool ok = true;
    int c = 0;

    for (; c < nch; ++c) {
        const int s = c & 1;
        const int t0 = c * kC;
        const int n = min(kC, a.L - t0);
        if (__syncthreads_or(wait_parity(&sm.full[s], (uint32_t)(c >> 1) & 1u) ? 0 : 1)) {
            ok = false;
            break;
        }
        unsigned char* img = sm.buf[s];
        float* U = reinterpret_cast<float*>(img + kBufU);          // [64][kUS]: U, then E
        const float* TP = reinterpret_cast<const float*>(img + kBufTP);
        const float* lg = reinterpret_cast<const float*>(img + kBufG);
        const float* pd = lg + kC;

        // B of D1: M^T (32 rows x 128) in three bf16 parts, 8 k-values per granule.
        for (int e = tid; e < kDVC * (kD / 8); e += kNT) {
            const int jj = e % kDVC, g = e / kDVC;
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = sm.M[8 * g + j][jj];
            uint4 p0, p1, p2;
            split3x8(x, p0, p1, p2);
            const uint32_t off = core_off(jj, 8 * g, kD);
            *reinterpret_cast<uint4*>(sm.bop[0] + off) = p0;
            *reinterpret_cast<uint4*>(sm.bop[1] + off) = p1;
            *reinterpret_cast<uint4*>(sm.bop[2] + off) = p2;
        }
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t a1 = smem_u32(img);
            for (int part = 0; part < 3; ++part)
                for (int ks = 0; ks < kD / 16; ++ks)
                    umma_bf16(tmem, umma_desc(a1 + 256 * ks, (kD / 8) * 128),
                              umma_desc(smem_u32(sm.bop[part]) + 256 * ks, (kD / 8) * 128), kIdesc,
                              (part | ks) != 0 ? 1u : 0u);
            umma_commit(&sm.mma);
        }
        // The decision to read TMEM is block-uniform (tcgen05.ld is warp-collective).
        if (__syncthreads_or(wait_parity(&sm.mma, 0) ? 0 : 1)) {
            ok = false;
            break;
        }
        tc_fence_after();
        {
            float v[16];
            tmem_ld16(tmem + lane_base + (uint32_t)(half * 16), v);
            const int row = (warp % 4) * 32 + lane;
            float* dstrow;
            float g = 1.f;
            if (row < kC) {
                dstrow = &sm.KM[row][half * 16];
            } else {
                dstrow = &sm.QM[row - kC][half * 16];
                g = expf(lg[row - kC]);
            }
#pragma unroll
            for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4*>(dstrow + j) = make_float4(v[j] * g, v[j + 1] * g, v[j + 2] * g, v[j + 3] * g);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // E = U - Tb KM over U: Tb[t][i] = TP[t][i] for i <= t.
        {
            float4 elo = *reinterpret_cast<const float4*>(&U[rlo * kUS + 4 * tx]);
            float4 ehi = *reinterpret_cast<const float4*>(&U[rhi * kUS + 4 * tx]);
            for (int i = 0; i <= rhi; ++i) {
                const float4 km = *reinterpret_cast<const float4*>(&sm.KM[i][4 * tx]);
                const float th = TP[rhi * kTS + i];
                ehi.x = fmaf(-th, km.x, ehi.x), ehi.y = fmaf(-th, km.y, ehi.y);
                ehi.z = fmaf(-th, km.z, ehi.z), ehi.w = fmaf(-th, km.w, ehi.w);
                if (i <= rlo) {
                    const float tl = TP[rlo * kTS + i];
                    elo.x = fmaf(-tl, km.x, elo.x), elo.y = fmaf(-tl, km.y, elo.y);
                    elo.z = fmaf(-tl, km.z, elo.z), elo.w = fmaf(-tl, km.w, elo.w);
                }
            }
            *reinterpret_cast<float4*>(&U[rlo * kUS + 4 * tx]) = elo;
            *reinterpret_cast<float4*>(&U[rhi * kUS + 4 * tx]) = ehi;
        }
        __syncthreads();

        // B of D2: E' = diag(g_C / g) E, transposed (32 rows x 64 tokens), three bf16 parts.
        {
            const int jj = tid % kDVC, g = tid / kDVC;  // 32 x 8 granules, one per thread
            const float lgC = lg[kC - 1];
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = U[(8 * g + j) * kUS + jj] * expf(lgC - lg[8 * g + j]);
            uint4 p0, p1, p2;
            split3x8(x, p0, p1, p2);
            const uint32_t off = core_off(jj, 8 * g, kC);
            *reinterpret_cast<uint4*>(sm.bop[0] + off) = p0;
            *reinterpret_cast<uint4*>(sm.bop[1] + off) = p1;
            *reinterpret_cast<uint4*>(sm.bop[2] + off) = p2;
        }
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            const uint32_t a2 = smem_u32(img + kBufA2);
            for (int part = 0; part < 3; ++part)
                for (int ks = 0; ks < kC / 16; ++ks)
                    umma_bf16(tmem + 32, umma_desc(a2 + 256 * ks, (kC / 8) * 128),
                              umma_desc(smem_u32(sm.bop[part]) + 256 * ks, (kC / 8) * 128), kIdesc,
                              (part | ks) != 0 ? 1u : 0u);
            umma_commit(&sm.mma);
        }

        // O = QM + P E while the tensor core works; P[t][i] = TP[i][t] for i < t, P[t][t] = pd[t].
        {
            float4 olo = *reinterpret_cast<const float4*>(&sm.QM[rlo][4 * tx]);
            float4 ohi = *reinterpret_cast<const float4*>(&sm.QM[rhi][4 * tx]);
            for (int i = 0; i < rhi; ++i) {
                const float4 ev = *reinterpret_cast<const float4*>(&U[i * kUS + 4 * tx]);
                const float ph = TP[i * kTS + rhi];
                ohi.x = fmaf(ph, ev.x, ohi.x), ohi.y = fmaf(ph, ev.y, ohi.y);
                ohi.z = fmaf(ph, ev.z, ohi.z), ohi.w = fmaf(ph, ev.w, ohi.w);
                if (i < rlo) {
                    const float pl = TP[i * kTS + rlo];
                    olo.x = fmaf(pl, ev.x, olo.x), olo.y = fmaf(pl, ev.y, olo.y);
                    olo.z = fmaf(pl, ev.z, olo.z), olo.w = fmaf(pl, ev.w, olo.w);
                }
            }
            {
                const float4 eh = *reinterpret_cast<const float4*>(&U[rhi * kUS + 4 * tx]);
                const float4 el = *reinterpret_cast<const float4*>(&U[rlo * kUS + 4 * tx]);
                const float dh = pd[rhi], dl = pd[rlo];
                ohi.x = fmaf(dh, eh.x, ohi.x), ohi.y = fmaf(dh, eh.y, ohi.y);
                ohi.z = fmaf(dh, eh.z, ohi.z), ohi.w = fmaf(dh, eh.w, ohi.w);
                olo.x = fmaf(dl, el.x, olo.x), olo.y = fmaf(dl, el.y, olo.y);
                olo.z = fmaf(dl, el.z, olo.z), olo.w = fmaf(dl, el.w, olo.w);
            }
            float* ob = a.out + (((size_t)b * a.L + t0) * a.Hv + h) * kD + col0 + 4 * tx;
            const size_t row_stride = (size_t)a.Hv * kD;
            if (rlo < n) *reinterpret_cast<float4*>(ob + rlo * row_stride) = olo;
            if (rhi < n) *reinterpret_cast<float4*>(ob + rhi * row_stride) = ohi;
        }

        if (__syncthreads_or(wait_parity(&sm.mma, 1) ? 0 : 1)) {
            ok = false;
            break;
        }
        tc_fence_after();
        {
            float v[16];
            tmem_ld16(tmem + lane_base + 32u + (uint32_t)(half * 16), v);
            const int i = (warp % 4) * 32 + lane;  // dk row
            const float gC = expf(lg[kC - 1]);
            float* mrow = &sm.M[i][half * 16];
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                float4 m = *reinterpret_cast<float4*>(mrow + j);
                m.x = fmaf(gC, m.x, v[j]), m.y = fmaf(gC, m.y, v[j + 1]);
                m.z = fmaf(gC, m.z, v[j + 2]), m.w = fmaf(gC, m.w, v[j + 3]);
                *reinterpret_cast<float4*>(mrow + j) = m;
            }
        }
        // Buffer s (E was written into it) is refilled next by the async proxy.
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && c + 2 < nch) issue(c + 2);
    }

    if (ok) {
        float* MD = a.pool + ((size_t)sm.dst * a.Hv + h) * (kD * kD) + col0;
        for (int e = tid; e < kD * (kDVC / 4); e += kNT) {
            const int i = e / (kDVC / 4), j4 = e % (kDVC / 4);
            *reinterpret_cast<float4*>(MD + (size_t)i * kD + 4 * j4) = *reinterpret_cast<const float4*>(&sm.M[i][4 * j4]);
        }
    } else if (tid == 0) {
        // Something never arrived: record it, then give the copies and MMAs still
        // in flight one more bounded wait each before the shared memory and TMEM go.
        record(a.err, GDN_ERR_TIMEOUT);
        for (int cc = c; cc < min(c + 2, nch); ++cc) wait_parity(&sm.full[cc & 1], (uint32_t)(cc >> 1) & 1u);
        wait_parity(&sm.mma, 0);
        wait_parity(&sm.mma, 1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(64) : "memory");
}

}  // namespace

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
    if (!pool || !src_idx || !dst_idx || !q || !k || !v || !alpha || !beta || !out || !workspace)
        return GDN_ERR_INVALID_ARG;
    const int nchunks = (L + kC - 1) / kC;
    if (workspace_bytes < gdn_prefill_workspace_bytes(B, L, Hv, dk, dv)) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Hv * nchunks >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    // 16-byte vector accesses: workspace, pool, out, q, k, v (rows of 128 elements keep the alignment).
    const uintptr_t align = reinterpret_cast<uintptr_t>(workspace) | reinterpret_cast<uintptr_t>(pool) |
                            reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(q) |
                            reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v);
    if ((align & 15u) != 0) return GDN_ERR_INVALID_ARG;

    const ChunkArgs a{pool, src_idx, dst_idx, q, k, v, alpha, beta, out, static_cast<unsigned char*>(workspace),
                      err_word, num_slots, B, L, Hk, Hv, Hv / Hk, nchunks};
    const bool bf = qkv_dtype == GDN_BF16;
    const int s1 = (int)sizeof(Smem1), s2 = bf ? (int)sizeof(SmemTC) : (int)sizeof(Smem2);
    cudaError_t e = bf ? cudaFuncSetAttribute(gdn_chunk_prepare_kernel<__nv_bfloat16>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, s1)
                       : cudaFuncSetAttribute(gdn_chunk_prepare_kernel<float>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    e = bf ? cudaFuncSetAttribute(gdn_chunk_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s2)
           : cudaFuncSetAttribute(gdn_chunk_scan_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const unsigned g1 = (unsigned)(B * Hv * nchunks), g2 = (unsigned)(B * Hv * kNCB);
    if (bf) {
        gdn_chunk_prepare_kernel<__nv_bfloat16><<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_tc_kernel<<<g2, kNT, s2, stream>>>(a);
    } else {
        gdn_chunk_prepare_kernel<float><<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_kernel<float><<<g2, kNT, s2, stream>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
