// gdn_step.cu -- sm_100a kernels and C ABI for the decode-time Gated DeltaNet
// state update with slot indirection (declarations and contract: gdn_step.h).
//
// The update per (request b, value head h, token t) is the gated delta rule of
// Gated DeltaNet (Yang, Kautz & Hatamizadeh, ICLR 2025), the mechanism the
// TokenSpeed 580 tok/s article (24-ai.news, English edition, opening section)
// names for the model's linear-attention layers.  It is evaluated in rank-one
// form on the stored tile M = S^T ([dk][dv], dv contiguous):
//
//     u_j = sum_i M[i][j] k_i          (= (S k)_j)
//     w_j = sum_i M[i][j] q_i          (= (S q)_j)
//     c_j = beta * (v_j - alpha * u_j)
//     M'[i][j] = alpha * M[i][j] + k_i * c_j
//     o_j = alpha * w_j + c_j * (k . q)            (= (S' q)_j)
//
// Every value column j is independent, so a tile splits along dv without any
// cross-block exchange.  Work per unit is ~7 flop per 8 bytes of state moved:
// the kernels are HBM-bound and use no tensor cores.  Each state tile is read
// from the slot named by src_idx and written to the slot named by dst_idx: the
// index indirection / copy-on-write scheme of the article's "Mamba State Update
// optimization" and "Hybrid prefix caching for GDN/Mamba" items, and the
// current_input_indices speculative path of the zubnet.ai LightSeek TokenSpeed
// article (second paragraph).

#include "gdn_step.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

struct StepArgs {
    float* pool;
    const int32_t* src_idx;
    const int32_t* dst_idx;
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    float* out;
    int32_t* err;
    int num_slots, B, T, Hk, Hv, dk, dv, G;
};

__device__ __forceinline__ void record_error(int32_t* err, int32_t code) {
    if (err != nullptr) atomicCAS(err, 0, code);
}

template <typename InT>
__device__ __forceinline__ float load_in(const void* base, size_t idx);

template <>
__device__ __forceinline__ float load_in<float>(const void* base, size_t idx) {
    return __ldg(static_cast<const float*>(base) + idx);
}

template <>
__device__ __forceinline__ float load_in<__nv_bfloat16>(const void* base, size_t idx) {
    return __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(base) + idx));
}

// True when src and all T destination slots of request b are inside the pool.
// Every thread of a block evaluates the same indices, so the result is uniform.
__device__ __forceinline__ bool request_in_range(const StepArgs& a, int b, int& src) {
    src = __ldg(a.src_idx + b);
    bool ok = src >= 0 && src < a.num_slots;
    for (int t = 0; t < a.T; ++t) {
        const int d = __ldg(a.dst_idx + (size_t)b * a.T + t);
        ok = ok && d >= 0 && d < a.num_slots;
    }
    return ok;
}

__device__ __forceinline__ void fma4(float4& acc, const float4& m, float x) {
    acc.x = fmaf(m.x, x, acc.x);
    acc.y = fmaf(m.y, x, acc.y);
    acc.z = fmaf(m.z, x, acc.z);
    acc.w = fmaf(m.w, x, acc.w);
}

__device__ __forceinline__ void add4(float4& acc, const float4& x) {
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
}

// ---------------------------------------------------------------------------
// Register-tile kernel for fixed (DK, DV).  One CTA owns one (b, h) state tile
// and keeps it in registers across all T tokens.  Thread layout: CG = DV/4
// column groups (one float4 each) x RG = NT/CG row groups; thread (rg, cg)
// holds rows i = m*RG + rg, m < DK/RG, so each warp-wide load instruction
// reads whole 512-byte rows and the CTA sweeps the 64 KiB tile front to back.
// Reductions over i: in-thread over its rows, then across row groups through
// shared memory.  The tile is read once from HBM and written once per token.
// ---------------------------------------------------------------------------
template <int DK, int DV, int NT, typename InT>
__global__ void __launch_bounds__(NT, 2) gdn_tile_kernel(StepArgs a) {
    constexpr int CG = DV / 4;
    static_assert(DV % 4 == 0 && NT % CG == 0, "tile shape");
    constexpr int RG = NT / CG;
    static_assert(DK % RG == 0, "tile shape");
    constexpr int RPT = DK / RG;

    __shared__ float ks[DK];
    __shared__ float qs[DK];
    __shared__ float4 red_u[RG][CG];
    __shared__ float4 red_w[RG][CG];
    __shared__ float kq_s;

    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;
    const int h = blockIdx.x % a.Hv;
    const int b = blockIdx.x / a.Hv;
    const int hk = h / a.G;

    int src;
    if (!request_in_range(a, b, src)) {
        if (tid == 0) record_error(a.err, GDN_ERR_INDEX);
        return;
    }

    const float4* S = reinterpret_cast<const float4*>(a.pool + ((size_t)src * a.Hv + h) * (DK * DV));
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldcs(S + (size_t)(m * RG + rg) * CG + cg);

    for (int t = 0; t < a.T; ++t) {
        const size_t tok = (size_t)b * a.T + t;
        if (t > 0) __syncthreads();  // the previous token is done with ks/qs/red
        const size_t kbase = (tok * a.Hk + hk) * DK;
        for (int i = tid; i < DK; i += NT) {
            ks[i] = load_in<InT>(a.k, kbase + i);
            qs[i] = load_in<InT>(a.q, kbase + i);
        }
        __syncthreads();

        float4 pu = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 pw = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int i = m * RG + rg;
            fma4(pu, s[m], ks[i]);
            fma4(pw, s[m], qs[i]);
        }
        red_u[rg][cg] = pu;
        red_w[rg][cg] = pw;
        if (tid < 32) {
            float acc = 0.f;
            for (int i = tid; i < DK; i += 32) acc = fmaf(ks[i], qs[i], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (tid == 0) kq_s = acc;
        }
        __syncthreads();

        float4 u = red_u[0][cg];
        float4 w = red_w[0][cg];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            add4(u, red_u[r][cg]);
            add4(w, red_w[r][cg]);
        }
        const size_t gh = tok * a.Hv + h;
        const float al = __ldg(a.alpha + gh);
        const float be = __ldg(a.beta + gh);
        const size_t vb = gh * DV + (size_t)cg * 4;
        float4 c;
        c.x = be * (load_in<InT>(a.v, vb + 0) - al * u.x);
        c.y = be * (load_in<InT>(a.v, vb + 1) - al * u.y);
        c.z = be * (load_in<InT>(a.v, vb + 2) - al * u.z);
        c.w = be * (load_in<InT>(a.v, vb + 3) - al * u.w);
        if (rg == 0) {
            const float kq = kq_s;
            float4 o;
            o.x = fmaf(c.x, kq, al * w.x);
            o.y = fmaf(c.y, kq, al * w.y);
            o.z = fmaf(c.z, kq, al * w.z);
            o.w = fmaf(c.w, kq, al * w.w);
            __stcs(reinterpret_cast<float4*>(a.out + gh * DV) + cg, o);
        }

        const int dst = __ldg(a.dst_idx + tok);
        float4* D = reinterpret_cast<float4*>(a.pool + ((size_t)dst * a.Hv + h) * (DK * DV));
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float ki = ks[m * RG + rg];
            s[m].x = fmaf(ki, c.x, al * s[m].x);
            s[m].y = fmaf(ki, c.y, al * s[m].y);
            s[m].z = fmaf(ki, c.z, al * s[m].z);
            s[m].w = fmaf(ki, c.w, al * s[m].w);
            __stcs(D + (size_t)(m * RG + rg) * CG + cg, s[m]);
        }
    }
}

// ---------------------------------------------------------------------------
// Column kernel for any (dk, dv): one thread per value column j, one CTA per
// (b, h, chunk of columns).  Pass 1 reduces u_j, w_j down column j; pass 2
// re-reads the column and writes the update.  Token t > 0 reads the slot token
// t-1 wrote; only thread j ever touches column j, so in-place and chained
// updates need no synchronisation beyond program order.
// ---------------------------------------------------------------------------
template <typename InT>
__global__ void gdn_column_kernel(StepArgs a) {
    extern __shared__ float smem[];
    float* ks = smem;
    float* qs = smem + a.dk;

    const int h = blockIdx.x % a.Hv;
    const int b = blockIdx.x / a.Hv;
    const int hk = h / a.G;
    const int j = blockIdx.y * blockDim.x + threadIdx.x;
    const bool active = j < a.dv;
    const size_t tile = (size_t)a.dk * a.dv;

    int src;
    if (!request_in_range(a, b, src)) {
        if (threadIdx.x == 0) record_error(a.err, GDN_ERR_INDEX);
        return;
    }

    const float* S = a.pool + ((size_t)src * a.Hv + h) * tile;
    for (int t = 0; t < a.T; ++t) {
        const size_t tok = (size_t)b * a.T + t;
        if (t > 0) __syncthreads();
        const size_t kbase = (tok * a.Hk + hk) * a.dk;
        for (int i = threadIdx.x; i < a.dk; i += blockDim.x) {
            ks[i] = load_in<InT>(a.k, kbase + i);
            qs[i] = load_in<InT>(a.q, kbase + i);
        }
        __syncthreads();

        const int dst = __ldg(a.dst_idx + tok);
        float* D = a.pool + ((size_t)dst * a.Hv + h) * tile;
        if (active) {
            float u = 0.f, w = 0.f, kq = 0.f;
            for (int i = 0; i < a.dk; ++i) {
                const float m = S[(size_t)i * a.dv + j];
                u = fmaf(m, ks[i], u);
                w = fmaf(m, qs[i], w);
                kq = fmaf(ks[i], qs[i], kq);
            }
            const size_t gh = tok * a.Hv + h;
            const float al = __ldg(a.alpha + gh);
            const float be = __ldg(a.beta + gh);
            const float c = be * (load_in<InT>(a.v, gh * a.dv + j) - al * u);
            a.out[gh * a.dv + j] = fmaf(c, kq, al * w);
            for (int i = 0; i < a.dk; ++i) {
                const float m = S[(size_t)i * a.dv + j];
                D[(size_t)i * a.dv + j] = fmaf(ks[i], c, al * m);
            }
        }
        S = D;
    }
}

__global__ void gdn_commit_kernel(const int32_t* __restrict__ accept_len, int32_t* __restrict__ committed,
                                  const int32_t* __restrict__ cur, int B, int T, int num_slots, int32_t* err) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int acc = accept_len[b];
    if (acc < 0 || acc > T) {
        record_error(err, GDN_ERR_INDEX);
        return;
    }
    if (acc == 0) return;
    const int s = cur[(size_t)b * T + (acc - 1)];
    if (s < 0 || s >= num_slots) {
        record_error(err, GDN_ERR_INDEX);
        return;
    }
    committed[b] = s;
}

constexpr int kMaxDk = 4096;

template <int DK, int DV, int NT>
gdn_status launch_tile(const StepArgs& a, int32_t dtype, cudaStream_t stream) {
    const dim3 grid((unsigned)(a.B * a.Hv));
    if (dtype == GDN_BF16)
        gdn_tile_kernel<DK, DV, NT, __nv_bfloat16><<<grid, NT, 0, stream>>>(a);
    else
        gdn_tile_kernel<DK, DV, NT, float><<<grid, NT, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_column(const StepArgs& a, int32_t dtype, cudaStream_t stream) {
    int threads = ((a.dv + 31) / 32) * 32;
    if (threads > 256) threads = 256;
    const dim3 grid((unsigned)(a.B * a.Hv), (unsigned)((a.dv + threads - 1) / threads));
    const size_t smem = 2 * sizeof(float) * (size_t)a.dk;
    if (dtype == GDN_BF16)
        gdn_column_kernel<__nv_bfloat16><<<grid, threads, smem, stream>>>(a);
    else
        gdn_column_kernel<float><<<grid, threads, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" gdn_status gdn_decode_step(float* pool, int32_t num_slots, const int32_t* src_idx,
                                      const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                      const float* alpha, const float* beta, float* out, int32_t B, int32_t T,
                                      int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int32_t qkv_dtype,
                                      int32_t* err_word, cudaStream_t stream) {
    if (B < 0 || T < 1 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || num_slots < 1) return GDN_ERR_INVALID_ARG;
    if (Hv % Hk != 0 || dk > kMaxDk) return GDN_ERR_INVALID_ARG;
    if (qkv_dtype != GDN_F32 && qkv_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Hv >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!pool || !src_idx || !dst_idx || !q || !k || !v || !alpha || !beta || !out) return GDN_ERR_INVALID_ARG;

    StepArgs a{pool, src_idx, dst_idx, q, k, v, alpha, beta, out, err_word,
               num_slots, B, T, Hk, Hv, dk, dv, Hv / Hk};
    const bool vec_ok = aligned16(pool) && aligned16(out);
    if (dk == 128 && dv == 128 && vec_ok) return launch_tile<128, 128, 256>(a, qkv_dtype, stream);
    if (dk == 64 && dv == 64 && vec_ok) return launch_tile<64, 64, 128>(a, qkv_dtype, stream);
    return launch_column(a, qkv_dtype, stream);
}

extern "C" gdn_status gdn_commit(const int32_t* accept_len, int32_t* committed, const int32_t* cur, int32_t B,
                                 int32_t T, int32_t num_slots, int32_t* err_word, cudaStream_t stream) {
    if (B < 0 || T < 1 || num_slots < 1) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!accept_len || !committed || !cur) return GDN_ERR_INVALID_ARG;
    const int threads = 256;
    gdn_commit_kernel<<<(B + threads - 1) / threads, threads, 0, stream>>>(accept_len, committed, cur, B, T,
                                                                           num_slots, err_word);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" gdn_status gdn_get_error(int32_t* err_word, int32_t* host_code, cudaStream_t stream) {
    if (!err_word || !host_code) return GDN_ERR_INVALID_ARG;
    int32_t value = 0;
    if (cudaMemcpyAsync(&value, err_word, sizeof value, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    *host_code = value;
    if (value != 0 && cudaMemsetAsync(err_word, 0, sizeof value, stream) != cudaSuccess) return GDN_ERR_CUDA;
    return GDN_OK;
}

extern "C" const char* gdn_status_string(int32_t status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_INDEX: return "GDN_ERR_INDEX";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        default: return "GDN_UNKNOWN_STATUS";
    }
}
