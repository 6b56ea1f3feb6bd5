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

#include "gdn_step.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kC = 64;     // tokens per chunk
constexpr int kD = 128;    // dk = dv supported here
constexpr int kDVC = 32;   // value columns per CTA in the sequential kernel
constexpr int kNT = 256;   // threads per CTA (both kernels)
constexpr int kPad = 4;    // row padding of [C][D] shared arrays (bank spread)

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
    float* ws;  // workspace: per (b, h, chunk) a ChunkWs record
    int32_t* err;
    int num_slots, B, L, Hk, Hv, G, nchunks;
};

// Workspace record of one (request, head, chunk), floats.
constexpr size_t kWsU = 0;                        // U = T diag(beta) V    [C][D]
constexpr size_t kWsT = kWsU + (size_t)kC * kD;   // Tb = T diag(beta g)   [C][C]
constexpr size_t kWsP = kWsT + (size_t)kC * kC;   // P                     [C][C]
constexpr size_t kWsG = kWsP + (size_t)kC * kC;   // log g                 [C]
constexpr size_t kWsFloats = kWsG + kC;

template <typename InT>
__device__ __forceinline__ float ld_in(const void* base, size_t idx);
template <>
__device__ __forceinline__ float ld_in<float>(const void* base, size_t idx) {
    return __ldg(static_cast<const float*>(base) + idx);
}
template <>
__device__ __forceinline__ float ld_in<__nv_bfloat16>(const void* base, size_t idx) {
    return __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(base) + idx));
}

__device__ __forceinline__ void record(int32_t* err, int32_t code) {
    if (err != nullptr) atomicCAS(err, 0, code);
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

    // Load K, Q (fp32) and the gates.
    for (int e = tid; e < kC * kD; e += kNT) {
        const int t = e / kD, d = e % kD;
        float kv = 0.f, qv = 0.f;
        if (t < n) {
            const size_t row = (((size_t)b * a.L + t0 + t) * a.Hk + hk) * kD;
            kv = ld_in<InT>(a.k, row + d);
            qv = ld_in<InT>(a.q, row + d);
        }
        sm.K[t][d] = kv;
        sm.X[t][d] = qv;
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
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    __syncthreads();

    // KK (strictly lower, scaled into A) and QK (lower, scaled into P), 4x4 per thread:
    // rows ty*4 + r (broadcast within a half-warp), columns tx + 16 s (16 consecutive
    // rows of K, conflict-free with the odd row stride).
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
        float* P = a.ws + ((size_t)bh * a.nchunks + c) * kWsFloats + kWsP;
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int t = ty * 4 + r, i = tx + 16 * s;
                const float ratio = i <= t ? expf(sm.lg[t] - sm.lg[i]) : 0.f;
                sm.A[t][i] = i < t ? sm.bt[t] * ratio * kk[r][s] : 0.f;
                P[t * kC + i] = i <= t ? ratio * qk[r][s] : 0.f;
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
    for (int e = tid; e < kC * kD; e += kNT) {
        const int t = e / kD, d = e % kD;
        float vv = 0.f;
        if (t < n) vv = ld_in<InT>(a.v, (((size_t)b * a.L + t0 + t) * a.Hv + h) * kD + d);
        sm.X[t][d] = vv * sm.bt[t];
    }
    __syncthreads();
    {
        float* rec = a.ws + ((size_t)bh * a.nchunks + c) * kWsFloats;
        // 64 x 128 outputs; thread: 4 rows x 8 columns (columns strided by 16 for bank spread)
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
            for (int s = 0; s < 8; ++s) rec[kWsU + (ty * 4 + r) * kD + tx + 16 * s] = u[r][s];
        for (int e = tid; e < kC * kC; e += kNT) {
            const int t = e / kC, i = e % kC;
            rec[kWsT + e] = sm.T[t][i] * (sm.bt[i] * expf(sm.lg[i]));
        }
        if (tid < kC) rec[kWsG + tid] = sm.lg[tid];
    }
}

// ---------------------------------------------------------------------------
// Kernel 2 pieces shared by its two forms.
// ---------------------------------------------------------------------------

// Reads (src, dst) of request b into shared memory and classifies it: 0 run,
// 1 padding (skipped silently), 2 bad index (skipped, reported).
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

// E = U - Tb KM (stored over U), then O = QM + P E for the chunk's valid rows.
// 64 x kDVC tiles: thread rows ty*2 + r, columns tx + 8 q.  QM already holds g Q M.
__device__ __forceinline__ void scan_tail(const ChunkArgs& a, float (*U)[kDVC + 1], const float (*Tb)[kC + 1],
                                          const float (*P)[kC + 1], const float (*KM)[kDVC + 1],
                                          const float (*QM)[kDVC + 1], int b, int h, int t0, int n, int col0,
                                          int tid) {
    const int ty = tid / 8, tx = tid % 8;
    float e[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) e[r][q] = U[ty * 2 + r][tx + 8 * q];
    for (int i = 0; i < kC; ++i) {
        float km[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) km[q] = KM[i][tx + 8 * q];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float tb = Tb[ty * 2 + r][i];
#pragma unroll
            for (int q = 0; q < 4; ++q) e[r][q] = fmaf(-tb, km[q], e[r][q]);
        }
    }
    // Each thread has read only its own U entries; E replaces them.
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) U[ty * 2 + r][tx + 8 * q] = e[r][q];
    __syncthreads();
    float o[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) o[r][q] = QM[ty * 2 + r][tx + 8 * q];
    for (int i = 0; i < kC; ++i) {
        float ev[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) ev[q] = U[i][tx + 8 * q];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float pr = P[ty * 2 + r][i];
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

// ---------------------------------------------------------------------------
// Kernel 2, CUDA-core form: per (b, h, column block of kDVC), the chunks in order.
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
    constexpr int NCB = kD / kDVC;
    const int cb = blockIdx.x % NCB;
    const int bh = blockIdx.x / NCB;
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
        const float* rec = a.ws + ((size_t)bh * a.nchunks + c) * kWsFloats;
        if (tid < kC) {
            const float lgt = rec[kWsG + tid], lgC_ = rec[kWsG + kC - 1];
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
            sm.U[t][jj] = rec[kWsU + (size_t)t * kD + col0 + jj];
        }
        for (int e = tid; e < kC * kC; e += kNT) {
            sm.Tb[e / kC][e % kC] = rec[kWsT + e];
            sm.P[e / kC][e % kC] = rec[kWsP + e];
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
        scan_tail(a, sm.U, sm.Tb, sm.P, sm.KM, sm.QM, b, h, t0, n, col0, tid);
        // M is updated from K^T E on the CUDA cores
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
                // Each thread reads and writes only its own rows of M in this phase.
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
// Operands sit in shared memory in the no-swizzle K-major canonical layout
// (8 x 8 bf16 core matrices of 128 contiguous bytes); accumulators live in
// 64 TMEM columns (D1 at column 0, D2 at column 32) allocated by warp 0.
// Thread 0 issues the MMAs and commits them to an mbarrier; every wait is
// bounded.  The triangular products (Tb KM, P E) run on the CUDA cores.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (row r, column k) of a K-major bf16 tile with Kdim columns.
__device__ __forceinline__ uint32_t core_off(int r, int k, int Kdim) {
    return (uint32_t)((r >> 3) * (Kdim >> 3) * 128 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
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

// x = hi + mid + lo with each part in bf16 (24 significant bits in total).
__device__ __forceinline__ void split3(float x, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
    hi = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(hi);
    mid = __float2bfloat16_rn(r1);
    lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
}

struct SmemTC {
    unsigned char A1[128 * kD * 2];        // [K; Q] rows x dk, K-major core tiles
    unsigned char A2[kD * kC * 2];         // K^T: dk rows x 64 tokens
    unsigned char B1[3][kDVC * kD * 2];    // M^T parts: kDVC rows x dk
    unsigned char B2[3][kDVC * kC * 2];    // E'^T parts: kDVC rows x 64 tokens
    float M[kD][kDVC + 1];
    float U[kC][kDVC + 1];                 // U, then E
    float Tb[kC][kC + 1];
    float P[kC][kC + 1];
    float KM[kC][kDVC + 1];
    float QM[kC][kDVC + 1];
    float lg[kC];
    float gq[kC];
    float gk[kC];
    uint64_t bar;
    uint32_t tmem;
    int src, dst, status;
};

__global__ void __launch_bounds__(kNT, 1) gdn_chunk_scan_tc_kernel(ChunkArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_tc[];
    SmemTC& sm = *reinterpret_cast<SmemTC*>(smem_tc);
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    constexpr int NCB = kD / kDVC;
    const int cb = blockIdx.x % NCB;
    const int bh = blockIdx.x / NCB;
    const int h = bh % a.Hv;
    const int b = bh / a.Hv;
    const int hk = h / a.G;
    const int col0 = cb * kDVC;
    constexpr uint32_t kIdesc = umma_idesc(128, kDVC);

    if (tid == 0) {
        scan_prologue(a, b, sm.src, sm.dst, sm.status);
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&sm.bar)), "r"(1) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (sm.status != 0) return;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(64)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }

    const float* M0 = a.pool + ((size_t)sm.src * a.Hv + h) * (kD * kD);
    for (int e = tid; e < kD * kDVC; e += kNT) {
        const int i = e / kDVC, j = e % kDVC;
        sm.M[i][j] = M0[(size_t)i * kD + col0 + j];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const int half = warp / 4;  // TMEM columns half*16 .. +15
    const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(a.k);
    const __nv_bfloat16* qin = static_cast<const __nv_bfloat16*>(a.q);
    uint32_t phase = 0;
    bool ok = true;

    for (int c = 0; c < a.nchunks && ok; ++c) {
        const int t0 = c * kC;
        const int n = min(kC, a.L - t0);
        const float* rec = a.ws + ((size_t)bh * a.nchunks + c) * kWsFloats;
        if (tid < kC) {
            const float lgt = rec[kWsG + tid], lgC_ = rec[kWsG + kC - 1];
            sm.lg[tid] = lgt;
            sm.gq[tid] = expf(lgt);
            sm.gk[tid] = expf(lgC_ - lgt);
        }
        // Operands of D1 and D2's A: K and Q rows as they are (exact bf16).
        for (int e = tid; e < kC * kD; e += kNT) {
            const int t = e / kD, d = e % kD;
            __nv_bfloat16 kv = __float2bfloat16_rn(0.f), qv = kv;
            if (t < n) {
                const size_t row = (((size_t)b * a.L + t0 + t) * a.Hk + hk) * kD;
                kv = kin[row + d];
                qv = qin[row + d];
            }
            *reinterpret_cast<__nv_bfloat16*>(sm.A1 + core_off(t, d, kD)) = kv;
            *reinterpret_cast<__nv_bfloat16*>(sm.A1 + core_off(kC + t, d, kD)) = qv;
            *reinterpret_cast<__nv_bfloat16*>(sm.A2 + core_off(d, t, kC)) = kv;
        }
        for (int e = tid; e < kC * kDVC; e += kNT) {
            const int t = e / kDVC, jj = e % kDVC;
            sm.U[t][jj] = rec[kWsU + (size_t)t * kD + col0 + jj];
        }
        for (int e = tid; e < kC * kC; e += kNT) {
            sm.Tb[e / kC][e % kC] = rec[kWsT + e];
            sm.P[e / kC][e % kC] = rec[kWsP + e];
        }
        // B of D1: M^T in three bf16 parts.
        for (int e = tid; e < kD * kDVC; e += kNT) {
            const int i = e / kDVC, jj = e % kDVC;
            __nv_bfloat16 p0, p1, p2;
            split3(sm.M[i][jj], p0, p1, p2);
            const uint32_t off = core_off(jj, i, kD);
            *reinterpret_cast<__nv_bfloat16*>(sm.B1[0] + off) = p0;
            *reinterpret_cast<__nv_bfloat16*>(sm.B1[1] + off) = p1;
            *reinterpret_cast<__nv_bfloat16*>(sm.B1[2] + off) = p2;
        }
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            for (int part = 0; part < 3; ++part)
                for (int s = 0; s < kD / 16; ++s)
                    umma_bf16(tmem, umma_desc(smem_u32(sm.A1) + 256 * s, (kD / 8) * 128),
                              umma_desc(smem_u32(sm.B1[part]) + 256 * s, (kD / 8) * 128), kIdesc,
                              (part | s) != 0 ? 1u : 0u);
            umma_commit(&sm.bar);
        }
        // The decision to read TMEM is block-uniform (tcgen05.ld is warp-collective).
        if (__syncthreads_or(wait_parity(&sm.bar, phase) ? 0 : 1)) {
            ok = false;
            break;
        }
        phase ^= 1u;
        tc_fence_after();
        {
            float v[16];
            tmem_ld16(tmem + lane_base + (uint32_t)(half * 16), v);
            const int row = (warp % 4) * 32 + lane;
            if (row < kC) {
#pragma unroll
                for (int j = 0; j < 16; ++j) sm.KM[row][half * 16 + j] = v[j];
            } else {
                const float g = sm.gq[row - kC];
#pragma unroll
                for (int j = 0; j < 16; ++j) sm.QM[row - kC][half * 16 + j] = v[j] * g;
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        scan_tail(a, sm.U, sm.Tb, sm.P, sm.KM, sm.QM, b, h, t0, n, col0, tid);

        // B of D2: E' = diag(g_C / g) E, transposed, in three bf16 parts.
        for (int e = tid; e < kC * kDVC; e += kNT) {
            const int t = e / kDVC, jj = e % kDVC;
            __nv_bfloat16 p0, p1, p2;
            split3(sm.U[t][jj] * sm.gk[t], p0, p1, p2);
            const uint32_t off = core_off(jj, t, kC);
            *reinterpret_cast<__nv_bfloat16*>(sm.B2[0] + off) = p0;
            *reinterpret_cast<__nv_bfloat16*>(sm.B2[1] + off) = p1;
            *reinterpret_cast<__nv_bfloat16*>(sm.B2[2] + off) = p2;
        }
        async_proxy_fence();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            for (int part = 0; part < 3; ++part)
                for (int s = 0; s < kC / 16; ++s)
                    umma_bf16(tmem + 32, umma_desc(smem_u32(sm.A2) + 256 * s, (kC / 8) * 128),
                              umma_desc(smem_u32(sm.B2[part]) + 256 * s, (kC / 8) * 128), kIdesc,
                              (part | s) != 0 ? 1u : 0u);
            umma_commit(&sm.bar);
        }
        if (__syncthreads_or(wait_parity(&sm.bar, phase) ? 0 : 1)) {
            ok = false;
            break;
        }
        phase ^= 1u;
        tc_fence_after();
        {
            float v[16];
            tmem_ld16(tmem + lane_base + 32u + (uint32_t)(half * 16), v);
            const int i = (warp % 4) * 32 + lane;  // dk row
            const float gC = expf(sm.lg[kC - 1]);
#pragma unroll
            for (int j = 0; j < 16; ++j) sm.M[i][half * 16 + j] = fmaf(gC, sm.M[i][half * 16 + j], v[j]);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (ok) {
        float* MD = a.pool + ((size_t)sm.dst * a.Hv + h) * (kD * kD);
        for (int e = tid; e < kD * kDVC; e += kNT) {
            const int i = e / kDVC, jj = e % kDVC;
            MD[(size_t)i * kD + col0 + jj] = sm.M[i][jj];
        }
    } else {
        // A commit that never arrived: give the tensor core one more bounded wait
        // to finish with this CTA's TMEM before it is freed.
        if (tid == 0) {
            record(a.err, GDN_ERR_TIMEOUT);
            wait_parity(&sm.bar, phase);
        }
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
    return (size_t)B * Hv * nchunks * kWsFloats * sizeof(float);
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
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return GDN_ERR_INVALID_ARG;

    const ChunkArgs a{pool, src_idx, dst_idx, q, k, v, alpha, beta, out, static_cast<float*>(workspace), err_word,
                      num_slots, B, L, Hk, Hv, Hv / Hk, nchunks};
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
    const unsigned g1 = (unsigned)(B * Hv * nchunks), g2 = (unsigned)(B * Hv * (kD / kDVC));
    if (bf) {
        gdn_chunk_prepare_kernel<__nv_bfloat16><<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_tc_kernel<<<g2, kNT, s2, stream>>>(a);
    } else {
        gdn_chunk_prepare_kernel<float><<<g1, kNT, s1, stream>>>(a);
        gdn_chunk_scan_kernel<float><<<g2, kNT, s2, stream>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
