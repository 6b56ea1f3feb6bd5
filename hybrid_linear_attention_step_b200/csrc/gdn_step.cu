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

#include <atomic>

// Launch single-token tile kernels with programmatic dependent launch: the
// next call's CTAs are scheduled while the previous kernel drains, and wait
// (griddepcontrol.wait) before their first memory access.  Measured on B200,
// large decode: 1.311 ms per 8-layer step with it, 1.325 ms without.
#ifndef GDN_USE_PDL
#define GDN_USE_PDL 1
#endif

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
    int flags;    // GDN_FUSE_* and GDN_SHARED_SOURCES bits (gdn_decode_step_fused); 0 for plain calls
    int prefill;  // 1 (gdn_prefill): dst_idx is [B], only the state after the last token is stored
};

// The flags that change the arithmetic (and pick the fused kernels).
constexpr int kFuseFlags = GDN_FUSE_GATES | GDN_FUSE_QK_NORM;

// unit_order: the register-tile kernels number their CTAs (request, head, column block)
// request-major, so that consecutive CTAs walk one slot's contiguous 2 MiB (the faster
// order when every request has a state of its own).  With GDN_SHARED_SOURCES the
// single-token kernel goes head-major: every request of one value head within a fraction
// of a wave, so that a source tile that several requests share is read from HBM once and
// then from L2.  (The multi-token kernels keep request-major order: the extra index
// arithmetic cost them registers and time, and prefix sharing is a single-token case.)

// Fused prologue (gdn_decode_step_fused).  alpha = exp(-softplus(x)) equals
// 1 / (1 + e^x) exactly, and beta = sigmoid(y) = 1 / (1 + e^-y); both limits
// (e^x overflowing to +inf, or underflowing to 0) give the right 0 and 1.
constexpr float kQkNormEps = 1e-6f;  // q_hat = q / sqrt(sum q^2 + eps), same for k

__device__ __forceinline__ float alpha_from_raw(float x) { return 1.0f / (1.0f + expf(x)); }
__device__ __forceinline__ float beta_from_raw(float y) { return 1.0f / (1.0f + expf(-y)); }
__device__ __forceinline__ float inv_norm(float sum_sq) { return 1.0f / sqrtf(sum_sq + kQkNormEps); }

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

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Request status: kRun when src and all T destination slots of request b lie
// inside the pool; kPad when src is the padding sentinel GDN_SLOT_NONE (the
// request is skipped silently, its destinations are not looked at); kBad
// otherwise (skipped and reported).  Every thread of a block evaluates the
// same indices, so the result is uniform across the block.
enum RequestStatus { kRun = 0, kPad = 1, kBad = 2 };

// All index loads are issued before any branch on their values, so a CTA
// pays one load latency here, not one per index.
__device__ __forceinline__ int request_status(const StepArgs& a, int b, int T, int& src, int& dst0) {
    src = __ldg(a.src_idx + b);
    bool ok = true;
    for (int t = 0; t < T; ++t) {
        const int d = __ldg(a.dst_idx + (size_t)b * T + t);
        if (t == 0) dst0 = d;
        ok &= (d >= 0) & (d < a.num_slots);
    }
    if (src == GDN_SLOT_NONE) return kPad;
    ok &= (src >= 0) & (src < a.num_slots);
    return ok ? kRun : kBad;
}

// Programmatic dependent launch (sm_90+): wait until the preceding grid in the
// stream has completed and its writes are visible; let the next grid's CTAs be
// scheduled once every CTA of this grid has issued its loads.  Both are no-ops
// when the launch carries no programmatic-serialization attribute.
__device__ __forceinline__ void grid_dependency_wait() {
#if GDN_USE_PDL
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

__device__ __forceinline__ void allow_dependent_launch() {
#if GDN_USE_PDL
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

__device__ __forceinline__ void fma4(float4& acc, const float4& m, float x) {
    acc.x = fmaf(m.x, x, acc.x);
    acc.y = fmaf(m.y, x, acc.y);
    acc.z = fmaf(m.z, x, acc.z);
    acc.w = fmaf(m.w, x, acc.w);
}

__device__ __forceinline__ void add4_rn(float4& acc, const float4& x) {
    acc.x = __fadd_rn(acc.x, x.x);
    acc.y = __fadd_rn(acc.y, x.y);
    acc.z = __fadd_rn(acc.z, x.z);
    acc.w = __fadd_rn(acc.w, x.w);
}

__device__ __forceinline__ void add4(float4& acc, const float4& x) {
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
}

// ---------------------------------------------------------------------------
// Single-token form of the register-tile kernel below (same thread layout, same
// per-token arithmetic in the same order, hence identical bits), written out
// on its own: with 5 CTAs per SM the budget is 96 registers, and the general
// form's token bookkeeping tips the single-token case into spills.  The slot
// indices are loaded together and branched on once; the destination slot, v
// and the gates are staged in shared memory so that no register holds them
// while the tile is in flight.
// ---------------------------------------------------------------------------
template <int DK, int DV, int DVC, int NT, int MINB, typename InT, bool FUSE>
__global__ void __launch_bounds__(NT, MINB) gdn_tile1_kernel(StepArgs a) {
    constexpr int CG = DVC / 4;
    static_assert(DV % DVC == 0 && DVC % 4 == 0 && NT % CG == 0 && NT >= 32, "tile shape");
    constexpr int RG = NT / CG;
    static_assert(DK % RG == 0, "tile shape");
    constexpr int RPT = DK / RG;
    constexpr int NC = DV / DVC;

    __shared__ float ks[DK];
    __shared__ float qs[DK];
    __shared__ float vs[DVC];
    __shared__ float gates[2];
    __shared__ int dst_s;
    __shared__ float4 red_u[RG][CG];
    __shared__ float4 red_w[RG][CG];
    __shared__ float kq_s;
    __shared__ float rk_s, rq_s;  // 1 / |k|, 1 / |q| (fused q/k normalisation)

    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;
    const int chunk = blockIdx.x % NC;
    const int unit = blockIdx.x / NC;
    const bool by_head = (a.flags & GDN_SHARED_SOURCES) != 0;  // see unit_order
    const int h = by_head ? unit / a.B : unit % a.Hv;
    const int b = by_head ? unit % a.B : unit / a.Hv;

    // With programmatic dependent launch this grid may start while the previous
    // kernel in the stream is finishing: wait for it before touching memory.
    grid_dependency_wait();
    const int src = __ldg(a.src_idx + b);
    const int dst = __ldg(a.dst_idx + b);
    if (src == GDN_SLOT_NONE) return;
    if (src < 0 || src >= a.num_slots || dst < 0 || dst >= a.num_slots) {
        if (tid == 0) record_error(a.err, GDN_ERR_INDEX);
        return;
    }

    // float4 offset of (row i, this thread's columns) in a tile: i * DV / 4 + chunk * CG + cg.
    const int col4 = chunk * CG + cg;
    const int toff = rg * (DV / 4) + col4;
    constexpr int kRowStep = RG * (DV / 4);
    const float4* S = reinterpret_cast<const float4*>(a.pool + ((size_t)src * a.Hv + h) * (DK * DV)) + toff;
    float4 s[RPT];
    // Default L2 priority, not evict-first: a prefix checkpoint shared by several requests
    // then stays in L2 for its other readers (the stores below are the streaming ones).
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldg(S + m * kRowStep);
    allow_dependent_launch();

    const size_t gh = (size_t)b * a.Hv + h;  // token index = b for a single token
    const size_t kbase = ((size_t)b * a.Hk + h / a.G) * DK;
    for (int i = tid; i < DK; i += NT) {
        ks[i] = load_in<InT>(a.k, kbase + i);
        qs[i] = load_in<InT>(a.q, kbase + i);
    }
    for (int j = tid; j < DVC; j += NT) vs[j] = load_in<InT>(a.v, gh * DV + (size_t)chunk * DVC + j);
    if (tid == 0) {
        const float x = __ldg(a.alpha + gh), y = __ldg(a.beta + gh);
        const bool raw = FUSE && (a.flags & GDN_FUSE_GATES);
        gates[0] = raw ? alpha_from_raw(x) : x;
        gates[1] = raw ? beta_from_raw(y) : y;
        dst_s = dst;
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
#pragma unroll
        for (int i = tid; i < DK; i += 32) acc = fmaf(ks[i], qs[i], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
        if (FUSE && (a.flags & GDN_FUSE_QK_NORM)) {
            // |k|^2 and |q|^2 alongside k.q: with k_hat = k rk and q_hat = q rq the
            // update needs only S k_hat = (S k) rk, S q_hat = (S q) rq, k_hat.q_hat = (k.q) rk rq.
            float kk = 0.f, qq = 0.f;
#pragma unroll
            for (int i = tid; i < DK; i += 32) {
                kk = fmaf(ks[i], ks[i], kk);
                qq = fmaf(qs[i], qs[i], qq);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                kk = __fadd_rn(kk, __shfl_xor_sync(0xffffffffu, kk, off));
                qq = __fadd_rn(qq, __shfl_xor_sync(0xffffffffu, qq, off));
            }
            if (tid == 0) {
                const float rk = inv_norm(kk), rq = inv_norm(qq);
                rk_s = rk;
                rq_s = rq;
                acc = __fmul_rn(__fmul_rn(acc, rk), rq);
            }
        }
        if (tid == 0) kq_s = acc;
    }
    __syncthreads();

    float4 u = red_u[0][cg];
    float4 w = red_w[0][cg];
#pragma unroll
    for (int r = 1; r < RG; ++r) {
        add4_rn(u, red_u[r][cg]);
        add4_rn(w, red_w[r][cg]);
    }
    const float al = gates[0];
    const float be = gates[1];
    const float4 vv = reinterpret_cast<const float4*>(vs)[cg];
    float rk = 1.f;
    if (FUSE && (a.flags & GDN_FUSE_QK_NORM)) {
        rk = rk_s;
        const float rq = rq_s;
        u = make_float4(__fmul_rn(u.x, rk), __fmul_rn(u.y, rk), __fmul_rn(u.z, rk), __fmul_rn(u.w, rk));
        w = make_float4(__fmul_rn(w.x, rq), __fmul_rn(w.y, rq), __fmul_rn(w.z, rq), __fmul_rn(w.w, rq));
    }
    float4 c;
    c.x = __fmul_rn(be, fmaf(-al, u.x, vv.x));
    c.y = __fmul_rn(be, fmaf(-al, u.y, vv.y));
    c.z = __fmul_rn(be, fmaf(-al, u.z, vv.z));
    c.w = __fmul_rn(be, fmaf(-al, u.w, vv.w));
    if (rg == 0) {
        const float kq = kq_s;
        float4 o;
        o.x = fmaf(c.x, kq, __fmul_rn(al, w.x));
        o.y = fmaf(c.y, kq, __fmul_rn(al, w.y));
        o.z = fmaf(c.z, kq, __fmul_rn(al, w.z));
        o.w = fmaf(c.w, kq, __fmul_rn(al, w.w));
        __stcs(reinterpret_cast<float4*>(a.out + gh * DV) + col4, o);
    }
    if (FUSE && (a.flags & GDN_FUSE_QK_NORM)) {
        // k_hat_i c_j = k_i (rk c_j): scale c once instead of every k_i
        c = make_float4(__fmul_rn(c.x, rk), __fmul_rn(c.y, rk), __fmul_rn(c.z, rk), __fmul_rn(c.w, rk));
    }
    float4* D = reinterpret_cast<float4*>(a.pool + ((size_t)dst_s * a.Hv + h) * (DK * DV)) + toff;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const float ki = ks[m * RG + rg];
        s[m].x = fmaf(ki, c.x, __fmul_rn(al, s[m].x));
        s[m].y = fmaf(ki, c.y, __fmul_rn(al, s[m].y));
        s[m].z = fmaf(ki, c.z, __fmul_rn(al, s[m].z));
        s[m].w = fmaf(ki, c.w, __fmul_rn(al, s[m].w));
        __stcs(D + m * kRowStep, s[m]);
    }
}

// ---------------------------------------------------------------------------
// Register-tile kernel.  Value columns are independent, so a (b, h) tile is
// split into DV / DVC column blocks, one CTA each (a column block's rows are
// DVC * 4 contiguous bytes, read and written as float4 runs).  Thread layout
// per CTA: CG = DVC / 4 column groups x RG = NT / CG row groups; thread
// (rg, cg) holds rows i = m * RG + rg of its four columns in registers for
// the whole call.
//
// Per token: partial sums of u = S k and w = S q over the thread's rows (k.q
// alongside, in warp 0), one barrier, the cross-row-group sums from shared
// memory, then c = beta (v - alpha u), o = alpha w + c (k.q) and the update
// S' = alpha S + k c^T in registers, streamed to the token's destination slot.
//
// Everything a token needs besides the tile (k and q rows, its v columns, the
// gates) is staged in shared memory.  Token 0's inputs are requested together
// with the tile at kernel start; token t+1's are fetched while token t's tile
// is being stored.  Shared memory stays small (a few KiB), which leaves the
// unified L1 large enough to track the outstanding misses of the MINB CTAs
// resident per SM -- measured on B200, a large shared-memory footprint caps
// read+write streaming well below what register-resident tiles reach.
//
// MULTI = false is a single-token form of the same template (not launched:
// gdn_tile1_kernel above serves T = 1).  Every form runs the same per-token
// arithmetic in the same order, so T chained single-token calls and one
// T-token call give identical bits.
// ---------------------------------------------------------------------------
template <int DK, int DV, int DVC, int NT, int MINB, typename InT, bool MULTI, bool FUSE>
__global__ void __launch_bounds__(NT, MINB) gdn_tile_kernel(StepArgs a) {
    constexpr int CG = DVC / 4;
    static_assert(DV % DVC == 0 && DVC % 4 == 0 && NT % CG == 0 && NT >= 32 && NT >= DVC, "tile shape");
    constexpr int RG = NT / CG;
    static_assert(DK % RG == 0, "tile shape");
    constexpr int RPT = DK / RG;
    constexpr int NC = DV / DVC;
    constexpr int NB = MULTI ? 2 : 1;  // token-input and reduction buffers (by token parity)

    __shared__ float ks[NB][DK];
    __shared__ float qs[NB][DK];
    __shared__ float vs[NB][DVC];
    __shared__ float gates[NB][2];
    __shared__ int dst_s[NB];
    __shared__ float4 red_u[NB][RG][CG];
    __shared__ float4 red_w[NB][RG][CG];
    __shared__ float kq_s[NB];
    __shared__ float rk_s[NB], rq_s[NB];  // 1 / |k|, 1 / |q| (fused q/k normalisation)

    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;
    const int chunk = blockIdx.x % NC;
    const int unit = blockIdx.x / NC;
    const int h = unit % a.Hv;  // request-major (the ordering hint serves single-token calls)
    const int b = unit / a.Hv;
    const int T = MULTI ? a.T : 1;

    grid_dependency_wait();  // launched with programmatic dependent launch, as gdn_tile1_kernel
    int src, dst0 = 0;
    const int status = request_status(a, b, a.prefill ? 1 : T, src, dst0);
    if (status != kRun) {
        if (status == kBad && tid == 0) record_error(a.err, GDN_ERR_INDEX);
        return;
    }

    // float4 offset of (row i, this thread's columns) in a tile: i * DV / 4 + chunk * CG + cg.
    const int col4 = chunk * CG + cg;
    const int toff = rg * (DV / 4) + col4;
    constexpr int kRowStep = RG * (DV / 4);
    const float4* S = reinterpret_cast<const float4*>(a.pool + ((size_t)src * a.Hv + h) * (DK * DV)) + toff;
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldg(S + m * kRowStep);  // default L2 priority (see gdn_tile1_kernel)
    allow_dependent_launch();

    const int hk = h / a.G;
    // Token t's inputs: thread j < DK fetches k_j and q_j, thread j < DVC its v
    // column, thread 0 the gates.  They stay in their input type until staged: a
    // conversion right after the load would wait for it ahead of this token's stores.
    auto fetch = [&](int t, InT& kx, InT& qx, InT& vx, float& ax, float& bx, int& dx) {
        const size_t tok = (size_t)b * T + t;
        if (tid < DK) {
            kx = __ldg(static_cast<const InT*>(a.k) + (tok * a.Hk + hk) * DK + tid);
            qx = __ldg(static_cast<const InT*>(a.q) + (tok * a.Hk + hk) * DK + tid);
        }
        if (tid < DVC) vx = __ldg(static_cast<const InT*>(a.v) + (tok * a.Hv + h) * DV + (size_t)chunk * DVC + tid);
        if (tid == 0) {
            ax = __ldg(a.alpha + tok * a.Hv + h);  // raw x, y with GDN_FUSE_GATES: mapped when staged
            bx = __ldg(a.beta + tok * a.Hv + h);
            dx = (t == 0 || a.prefill) ? dst0 : __ldg(a.dst_idx + tok);
        }
    };
    // The destination slot goes through shared memory as well: re-reading it
    // from global memory at store time would put a cache miss in front of the
    // stores, and holding it in a register costs occupancy.
    auto stage = [&](int buf, InT kx, InT qx, InT vx, float ax, float bx, int dx) {
        if (tid < DK) {
            ks[buf][tid] = to_f32(kx);
            qs[buf][tid] = to_f32(qx);
        }
        if (tid < DVC) vs[buf][tid] = to_f32(vx);
        if (tid == 0) {
            const bool raw = FUSE && (a.flags & GDN_FUSE_GATES);
            gates[buf][0] = raw ? alpha_from_raw(ax) : ax;
            gates[buf][1] = raw ? beta_from_raw(bx) : bx;
            dst_s[buf] = dx;
        }
    };
    static_assert(NT >= DK || !MULTI, "one thread per k/q element when staging tokens");
    {
        InT kx = InT(0.f), qx = InT(0.f), vx = InT(0.f);
        float ax = 0.f, bx = 0.f;
        int dx = 0;
        if (NT >= DK) {
            fetch(0, kx, qx, vx, ax, bx, dx);
            stage(0, kx, qx, vx, ax, bx, dx);
        } else {
            const size_t kbase = ((size_t)b * a.Hk + hk) * DK;
            for (int i = tid; i < DK; i += NT) {
                ks[0][i] = load_in<InT>(a.k, kbase + i);
                qs[0][i] = load_in<InT>(a.q, kbase + i);
            }
            fetch(0, kx, qx, vx, ax, bx, dx);
            if (tid < DVC) vs[0][tid] = to_f32(vx);
            if (tid == 0) {
                const bool raw = FUSE && (a.flags & GDN_FUSE_GATES);
                gates[0][0] = raw ? alpha_from_raw(ax) : ax;
                gates[0][1] = raw ? beta_from_raw(bx) : bx;
                dst_s[0] = dx;
            }
        }
    }
    __syncthreads();

    for (int t = 0; t < T; ++t) {
        const int cb = MULTI ? (t & 1) : 0;
        float4 pu = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 pw = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int i = m * RG + rg;
            fma4(pu, s[m], ks[cb][i]);
            fma4(pw, s[m], qs[cb][i]);
        }
        red_u[cb][rg][cg] = pu;
        red_w[cb][rg][cg] = pw;
        if (tid < 32) {
            float acc = 0.f;
#pragma unroll
            for (int i = tid; i < DK; i += 32) acc = fmaf(ks[cb][i], qs[cb][i], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
            if (FUSE && (a.flags & GDN_FUSE_QK_NORM)) {
                float kk = 0.f, qq = 0.f;
#pragma unroll
                for (int i = tid; i < DK; i += 32) {
                    kk = fmaf(ks[cb][i], ks[cb][i], kk);
                    qq = fmaf(qs[cb][i], qs[cb][i], qq);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    kk = __fadd_rn(kk, __shfl_xor_sync(0xffffffffu, kk, off));
                    qq = __fadd_rn(qq, __shfl_xor_sync(0xffffffffu, qq, off));
                }
                if (tid == 0) {
                    const float rk = inv_norm(kk), rq = inv_norm(qq);
                    rk_s[cb] = rk;
                    rq_s[cb] = rq;
                    acc = __fmul_rn(__fmul_rn(acc, rk), rq);
                }
            }
            if (tid == 0) kq_s[cb] = acc;
        }
        __syncthreads();

        // Next token's inputs are requested now; their latency hides behind this token's stores.
        InT kx = InT(0.f), qx = InT(0.f), vx = InT(0.f);
        float ax = 0.f, bx = 0.f;
        int dx = 0;
        if (MULTI && t + 1 < T) fetch(t + 1, kx, qx, vx, ax, bx, dx);

        float4 u = red_u[cb][0][cg];
        float4 w = red_w[cb][0][cg];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            add4_rn(u, red_u[cb][r][cg]);
            add4_rn(w, red_w[cb][r][cg]);
        }
        const float al = gates[cb][0];
        const float be = gates[cb][1];
        const float4 vv = reinterpret_cast<const float4*>(vs[cb])[cg];
        float rk = 1.f;
        if (FUSE && (a.flags & GDN_FUSE_QK_NORM)) {
            rk = rk_s[cb];
            const float rq = rq_s[cb];
            u = make_float4(__fmul_rn(u.x, rk), __fmul_rn(u.y, rk), __fmul_rn(u.z, rk), __fmul_rn(u.w, rk));
            w = make_float4(__fmul_rn(w.x, rq), __fmul_rn(w.y, rq), __fmul_rn(w.z, rq), __fmul_rn(w.w, rq));
        }
        // Rounding is spelled out (fmaf / __fmul_rn) so that every form of this
        // kernel, and every compiler context, evaluates the same operations.
        float4 c;
        c.x = __fmul_rn(be, fmaf(-al, u.x, vv.x));
        c.y = __fmul_rn(be, fmaf(-al, u.y, vv.y));
        c.z = __fmul_rn(be, fmaf(-al, u.z, vv.z));
        c.w = __fmul_rn(be, fmaf(-al, u.w, vv.w));
        const size_t gh = ((size_t)b * T + t) * a.Hv + h;
        if (rg == 0) {
            const float kq = kq_s[cb];
            float4 o;
            o.x = fmaf(c.x, kq, __fmul_rn(al, w.x));
            o.y = fmaf(c.y, kq, __fmul_rn(al, w.y));
            o.z = fmaf(c.z, kq, __fmul_rn(al, w.z));
            o.w = fmaf(c.w, kq, __fmul_rn(al, w.w));
            __stcs(reinterpret_cast<float4*>(a.out + gh * DV) + col4, o);
        }
        if (FUSE && (a.flags & GDN_FUSE_QK_NORM))
            c = make_float4(__fmul_rn(c.x, rk), __fmul_rn(c.y, rk), __fmul_rn(c.z, rk), __fmul_rn(c.w, rk));
        const int dst = dst_s[cb];
        float4* D = reinterpret_cast<float4*>(a.pool + ((size_t)dst * a.Hv + h) * (DK * DV)) + toff;
        const bool store = !a.prefill || t == T - 1;  // prefill keeps intermediate states on chip
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float ki = ks[cb][m * RG + rg];
            s[m].x = fmaf(ki, c.x, __fmul_rn(al, s[m].x));
            s[m].y = fmaf(ki, c.y, __fmul_rn(al, s[m].y));
            s[m].z = fmaf(ki, c.z, __fmul_rn(al, s[m].z));
            s[m].w = fmaf(ki, c.w, __fmul_rn(al, s[m].w));
            if (store) __stcs(D + m * kRowStep, s[m]);
        }
        if (MULTI && t + 1 < T) {
            // The other buffer was last read during token t-1, before this token's barrier.
            stage(cb ^ 1, kx, qx, vx, ax, bx, dx);
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// Multi-token form for short drafts (2 <= T <= kStageT = 4, no fused prologue): every
// token's inputs are requested together with the state tile at kernel start and
// staged in shared memory (in their input type), so the token loop waits on no
// global load and takes one barrier per token (the reduction buffers alternate by
// token parity; a buffer is rewritten two tokens later, after every thread has
// passed the barrier in between).  Same thread layout and the same per-token
// arithmetic in the same order as gdn_tile1_kernel and gdn_tile_kernel: identical
// bits.
// ---------------------------------------------------------------------------
constexpr int kStageT = 4;

template <int DK, int DV, int DVC, int NT, int MINB, typename InT>
__global__ void __launch_bounds__(NT, MINB) gdn_tileT_kernel(StepArgs a) {
    constexpr int CG = DVC / 4;
    static_assert(DV % DVC == 0 && DVC % 4 == 0 && NT % CG == 0 && NT >= DK && NT >= DVC, "tile shape");
    constexpr int RG = NT / CG;
    static_assert(DK % RG == 0, "tile shape");
    constexpr int RPT = DK / RG;
    constexpr int NC = DV / DVC;

    __shared__ InT ks[kStageT][DK];
    __shared__ InT qs[kStageT][DK];
    __shared__ InT vs[kStageT][DVC];
    __shared__ float gates[kStageT][2];
    __shared__ int dst_s[kStageT];
    __shared__ float4 red_u[2][RG][CG];
    __shared__ float4 red_w[2][RG][CG];
    __shared__ float kq_s[2];

    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;
    const int chunk = blockIdx.x % NC;
    const int unit = blockIdx.x / NC;
    const int h = unit % a.Hv;  // request-major (the ordering hint serves single-token calls)
    const int b = unit / a.Hv;
    const int T = a.T;

    grid_dependency_wait();
    int src, dst0 = 0;
    const int status = request_status(a, b, T, src, dst0);
    if (status != kRun) {
        if (status == kBad && tid == 0) record_error(a.err, GDN_ERR_INDEX);
        return;
    }
    const int col4 = chunk * CG + cg;
    const int toff = rg * (DV / 4) + col4;
    constexpr int kRowStep = RG * (DV / 4);
    const float4* S = reinterpret_cast<const float4*>(a.pool + ((size_t)src * a.Hv + h) * (DK * DV)) + toff;
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldg(S + m * kRowStep);  // default L2 priority (see gdn_tile1_kernel)
    allow_dependent_launch();

    const int hk = h / a.G;
    const InT* kin = static_cast<const InT*>(a.k);
    const InT* qin = static_cast<const InT*>(a.q);
    const InT* vin = static_cast<const InT*>(a.v);
    // Every token's loads are in flight together before any of them is staged.
    InT kr[kStageT], qr[kStageT], vr[kStageT];
#pragma unroll
    for (int t = 0; t < kStageT; ++t) {
        if (t < T) {
            const size_t tok = (size_t)b * T + t;
            if (tid < DK) {
                kr[t] = kin[(tok * a.Hk + hk) * DK + tid];
                qr[t] = qin[(tok * a.Hk + hk) * DK + tid];
            }
            if (tid < DVC) vr[t] = vin[(tok * a.Hv + h) * DV + (size_t)chunk * DVC + tid];
        }
    }
#pragma unroll
    for (int t = 0; t < kStageT; ++t) {
        if (t < T) {
            if (tid < DK) {
                ks[t][tid] = kr[t];
                qs[t][tid] = qr[t];
            }
            if (tid < DVC) vs[t][tid] = vr[t];
        }
    }
    if (tid < T) {
        const size_t tok = (size_t)b * T + tid;
        gates[tid][0] = __ldg(a.alpha + tok * a.Hv + h);
        gates[tid][1] = __ldg(a.beta + tok * a.Hv + h);
        dst_s[tid] = tid == 0 ? dst0 : __ldg(a.dst_idx + tok);
    }
    __syncthreads();

    for (int t = 0; t < T; ++t) {
        const int cb = t & 1;
        float4 pu = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 pw = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int i = m * RG + rg;
            fma4(pu, s[m], to_f32(ks[t][i]));
            fma4(pw, s[m], to_f32(qs[t][i]));
        }
        red_u[cb][rg][cg] = pu;
        red_w[cb][rg][cg] = pw;
        if (tid < 32) {
            float acc = 0.f;
#pragma unroll
            for (int i = tid; i < DK; i += 32) acc = fmaf(to_f32(ks[t][i]), to_f32(qs[t][i]), acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
            if (tid == 0) kq_s[cb] = acc;
        }
        __syncthreads();

        float4 u = red_u[cb][0][cg];
        float4 w = red_w[cb][0][cg];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            add4_rn(u, red_u[cb][r][cg]);
            add4_rn(w, red_w[cb][r][cg]);
        }
        const float al = gates[t][0];
        const float be = gates[t][1];
        const float4 vv = make_float4(to_f32(vs[t][4 * cg]), to_f32(vs[t][4 * cg + 1]), to_f32(vs[t][4 * cg + 2]),
                                      to_f32(vs[t][4 * cg + 3]));
        float4 c;
        c.x = __fmul_rn(be, fmaf(-al, u.x, vv.x));
        c.y = __fmul_rn(be, fmaf(-al, u.y, vv.y));
        c.z = __fmul_rn(be, fmaf(-al, u.z, vv.z));
        c.w = __fmul_rn(be, fmaf(-al, u.w, vv.w));
        const size_t gh = ((size_t)b * T + t) * a.Hv + h;
        if (rg == 0) {
            const float kq = kq_s[cb];
            float4 o;
            o.x = fmaf(c.x, kq, __fmul_rn(al, w.x));
            o.y = fmaf(c.y, kq, __fmul_rn(al, w.y));
            o.z = fmaf(c.z, kq, __fmul_rn(al, w.z));
            o.w = fmaf(c.w, kq, __fmul_rn(al, w.w));
            __stcs(reinterpret_cast<float4*>(a.out + gh * DV) + col4, o);
        }
        float4* D = reinterpret_cast<float4*>(a.pool + ((size_t)dst_s[t] * a.Hv + h) * (DK * DV)) + toff;
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float ki = to_f32(ks[t][m * RG + rg]);
            s[m].x = fmaf(ki, c.x, __fmul_rn(al, s[m].x));
            s[m].y = fmaf(ki, c.y, __fmul_rn(al, s[m].y));
            s[m].z = fmaf(ki, c.z, __fmul_rn(al, s[m].z));
            s[m].w = fmaf(ki, c.w, __fmul_rn(al, s[m].w));
            __stcs(D + m * kRowStep, s[m]);
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

    int src, dst0 = 0;
    const int status = request_status(a, b, a.prefill ? 1 : a.T, src, dst0);
    if (status != kRun) {
        if (status == kBad && threadIdx.x == 0) record_error(a.err, GDN_ERR_INDEX);
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

        // Prefill works in its destination slot: token 0 reads the source and
        // every token writes the destination, which the next token reads back.
        const int dst = a.prefill ? dst0 : __ldg(a.dst_idx + tok);
        float* D = a.pool + ((size_t)dst * a.Hv + h) * tile;
        if (active) {
            float u = 0.f, w = 0.f, kq = 0.f, kk = 0.f, qq = 0.f;
            for (int i = 0; i < a.dk; ++i) {
                const float m = S[(size_t)i * a.dv + j];
                u = fmaf(m, ks[i], u);
                w = fmaf(m, qs[i], w);
                kq = fmaf(ks[i], qs[i], kq);
                kk = fmaf(ks[i], ks[i], kk);
                qq = fmaf(qs[i], qs[i], qq);
            }
            const size_t gh = tok * a.Hv + h;
            float al = __ldg(a.alpha + gh);
            float be = __ldg(a.beta + gh);
            if (a.flags & GDN_FUSE_GATES) {
                al = alpha_from_raw(al);
                be = beta_from_raw(be);
            }
            float rk = 1.f;
            if (a.flags & GDN_FUSE_QK_NORM) {  // see gdn_tile1_kernel: normalisation folded into u, w, k.q, c
                rk = inv_norm(kk);
                const float rq = inv_norm(qq);
                u *= rk;
                w *= rq;
                kq = kq * rk * rq;
            }
            float c = be * (load_in<InT>(a.v, gh * a.dv + j) - al * u);
            a.out[gh * a.dv + j] = fmaf(c, kq, al * w);
            c *= rk;
            for (int i = 0; i < a.dk; ++i) {
                const float m = S[(size_t)i * a.dv + j];
                D[(size_t)i * a.dv + j] = fmaf(ks[i], c, al * m);
            }
        }
        S = D;
    }
}

// ---------------------------------------------------------------------------
// Bulk-copy helpers (sm_90+ PTX, used on sm_100a): mbarrier transaction
// counting and one-dimensional cp.async.bulk global -> shared copies into this
// CTA's own shared memory, without tensor maps: every copy is a contiguous,
// 16-byte aligned range of this GPU's own memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every wait on a copy gives up after this long and reports GDN_ERR_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Waits for the phase with the given parity; false if the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

template <typename InT>
__device__ __forceinline__ float smem_in(const InT* p, int i);
template <>
__device__ __forceinline__ float smem_in<float>(const float* p, int i) {
    return p[i];
}
template <>
__device__ __forceinline__ float smem_in<__nv_bfloat16>(const __nv_bfloat16* p, int i) {
    return __bfloat162float(p[i]);
}

// Shared-memory plan of the streaming kernel (dk = dv = 128, one token).
// Each of the STAGES buffers holds one unit's state tile plus its q, k and v
// rows and the 16-byte chunks of alpha and beta that contain its gate values.
// The cross-row-group reduction buffers and k.q are double-buffered by unit
// parity, so one barrier per unit suffices.
template <int NT, typename InT>
struct StreamPlan {
    static constexpr int DK = 128, DV = 128, STAGES = 3;
    static constexpr int CG = DV / 4, RG = NT / CG, RPT = DK / RG;
    static constexpr uint32_t TILE_BYTES = DK * DV * 4;
    static constexpr uint32_t ROW_BYTES = 128 * sizeof(InT);
    static constexpr uint32_t Q_OFF = TILE_BYTES, K_OFF = Q_OFF + ROW_BYTES, V_OFF = K_OFF + ROW_BYTES;
    static constexpr uint32_t A_OFF = V_OFF + ROW_BYTES, B_OFF = A_OFF + 16;
    static constexpr uint32_t STAGE_TX = B_OFF + 16;  // bytes landed per unit
    static constexpr uint32_t STAGE_STRIDE = (STAGE_TX + 127) / 128 * 128;
    static constexpr uint32_t RED_OFF = STAGES * STAGE_STRIDE;
    static constexpr uint32_t RED_BYTES = 2 * RG * CG * 16;  // u and w partials of one unit
    static constexpr uint32_t BAR_OFF = RED_OFF + 2 * RED_BYTES;
    static constexpr uint32_t META_OFF = BAR_OFF + STAGES * 8;
    static constexpr uint32_t KQ_OFF = META_OFF + STAGES * 8;
    static constexpr uint32_t SMEM_BYTES = KQ_OFF + 16;
    static_assert(NT % CG == 0 && DK % RG == 0, "thread layout");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory plan exceeds the per-CTA limit");
};

// ---------------------------------------------------------------------------
// Streaming kernel for single-token decode at dk = dv = 128.  Persistent: one
// CTA per SM walks units u = blockIdx.x + n * gridDim.x (u = b * Hv + h).
// Thread 0 keeps STAGES units in flight with bulk copies (state tile, q/k/v
// rows, gate chunks) and prefetches slot indices one unit ahead.  All threads
// consume one landed unit at a time: tile, k, v and gates -> registers and
// partial reductions; one barrier, after which the stage is refilled with the
// unit STAGES ahead while the threads finish the reduction, update the tile in
// registers and stream it straight to the destination slot.  The tile is read
// from HBM once and written once; the next STAGES tiles are in flight while
// the current one is reduced and stored.
// ---------------------------------------------------------------------------
template <int NT, typename InT>
__global__ void __launch_bounds__(NT, 1) gdn_stream_kernel(StepArgs a) {
    using P = StreamPlan<NT, InT>;
    constexpr int CG = P::CG, RG = P::RG, RPT = P::RPT, STAGES = P::STAGES;
    extern __shared__ __align__(128) unsigned char sbuf[];
    float4* red_base = reinterpret_cast<float4*>(sbuf + P::RED_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sbuf + P::BAR_OFF);
    int2* meta = reinterpret_cast<int2*>(sbuf + P::META_OFF);
    float* kq_s = reinterpret_cast<float*>(sbuf + P::KQ_OFF);

    const int tid = threadIdx.x;
    const int cg = tid % CG;
    const int rg = tid / CG;
    const int units = a.B * a.Hv;
    const int grid = gridDim.x;
    const int n_local = (units - (int)blockIdx.x + grid - 1) / grid;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
        mbar_fence_init();
    }
    __syncthreads();

    // Producer state, meaningful in thread 0 only.
    int p_next = 0;
    int nx_src = 0, nx_dst = 0;
    auto fetch_indices = [&](int n) {
        const int b = ((int)blockIdx.x + n * grid) / a.Hv;
        nx_src = __ldg(a.src_idx + b);
        nx_dst = __ldg(a.dst_idx + b);
    };
    auto issue = [&]() {
        const int n = p_next;
        const int u = (int)blockIdx.x + n * grid;
        const int b = u / a.Hv, h = u % a.Hv;
        const int src = nx_src, dst = nx_dst;
        ++p_next;
        if (p_next < n_local) fetch_indices(p_next);
        const int stage = n % STAGES;
        const bool valid = src >= 0 && src < a.num_slots && dst >= 0 && dst < a.num_slots;
        // meta.y: 1 run, 0 out-of-range (reported), -1 padding (skipped silently)
        meta[stage] = make_int2(dst, valid ? 1 : (src == GDN_SLOT_NONE ? -1 : 0));
        uint64_t* bar = &bars[stage];
        if (!valid) {
            mbar_arrive(bar);
            return;
        }
        unsigned char* st = sbuf + stage * P::STAGE_STRIDE;
        const size_t gh = (size_t)b * a.Hv + h;
        const size_t row = ((size_t)b * a.Hk + h / a.G) * P::DK;
        mbar_arrive_expect_tx(bar, P::STAGE_TX);
        bulk_g2s(st, a.pool + ((size_t)src * a.Hv + h) * (P::DK * P::DV), P::TILE_BYTES, bar);
        bulk_g2s(st + P::Q_OFF, static_cast<const InT*>(a.q) + row, P::ROW_BYTES, bar);
        bulk_g2s(st + P::K_OFF, static_cast<const InT*>(a.k) + row, P::ROW_BYTES, bar);
        bulk_g2s(st + P::V_OFF, static_cast<const InT*>(a.v) + gh * P::DV, P::ROW_BYTES, bar);
        bulk_g2s(st + P::A_OFF, a.alpha + (gh & ~(size_t)3), 16, bar);
        bulk_g2s(st + P::B_OFF, a.beta + (gh & ~(size_t)3), 16, bar);
    };

    if (tid == 0) {
        if (n_local > 0) fetch_indices(0);
        while (p_next < n_local && p_next < STAGES) issue();
    }
    __syncthreads();  // meta[] of the prologue's units is visible to every thread

    for (int n = 0; n < n_local; ++n) {
        const int stage = n % STAGES;
        const uint32_t parity = (uint32_t)(n / STAGES) & 1u;
        const int2 m = meta[stage];
        const bool landed = mbar_wait_bounded(&bars[stage], parity);

        const unsigned char* st = sbuf + stage * P::STAGE_STRIDE;
        const float4* tile = reinterpret_cast<const float4*>(st);
        const InT* qsm = reinterpret_cast<const InT*>(st + P::Q_OFF);
        const InT* ksm = reinterpret_cast<const InT*>(st + P::K_OFF);
        const InT* vsm = reinterpret_cast<const InT*>(st + P::V_OFF);
        float4* red_u = red_base + (n & 1) * (2 * RG * CG);
        float4* red_w = red_u + RG * CG;
        const int u = (int)blockIdx.x + n * grid;  // = b * Hv + h = gh for a single token

        // Everything this unit needs from its stage goes to registers before
        // the barrier.  The reads happen whether or not this thread saw the
        // copy land, so warp 0's shuffles never diverge; a unit that did not
        // land is abandoned at the barrier, its values unused.
        float4 s[RPT];
        float kr[RPT];
        float4 vr = make_float4(0.f, 0.f, 0.f, 0.f);
        float al = 0.f, be = 0.f;
        if (m.y == 1) {
            float4 pu = make_float4(0.f, 0.f, 0.f, 0.f);
            float4 pw = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int i = r * RG + rg;
                s[r] = tile[i * CG + cg];
                kr[r] = smem_in<InT>(ksm, i);
                fma4(pu, s[r], kr[r]);
                fma4(pw, s[r], smem_in<InT>(qsm, i));
            }
            red_u[rg * CG + cg] = pu;
            red_w[rg * CG + cg] = pw;
            vr = make_float4(smem_in<InT>(vsm, cg * 4 + 0), smem_in<InT>(vsm, cg * 4 + 1),
                             smem_in<InT>(vsm, cg * 4 + 2), smem_in<InT>(vsm, cg * 4 + 3));
            al = reinterpret_cast<const float*>(st + P::A_OFF)[u & 3];
            be = reinterpret_cast<const float*>(st + P::B_OFF)[u & 3];
            if (tid < 32) {
                float acc = 0.f;
#pragma unroll
                for (int i = tid; i < P::DK; i += 32) acc = fmaf(smem_in<InT>(ksm, i), smem_in<InT>(qsm, i), acc);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (tid == 0) kq_s[n & 1] = acc;
            }
        }
        if (__syncthreads_or(landed ? 0 : 1)) {
            // A copy never completed: report, let thread 0 wait (bounded) for
            // the copies it has issued so none lands in freed shared memory.
            if (tid == 0) {
                record_error(a.err, GDN_ERR_TIMEOUT);
                for (int j = n; j < p_next; ++j)
                    if (!mbar_wait_bounded(&bars[j % STAGES], (uint32_t)(j / STAGES) & 1u)) break;
            }
            return;
        }
        // The stage is consumed: refill it with the unit STAGES ahead.
        if (tid == 0 && p_next < n_local) issue();

        if (m.y == 1) {
            float4 uu = red_u[cg];
            float4 ww = red_w[cg];
#pragma unroll
            for (int r = 1; r < RG; ++r) {
                add4(uu, red_u[r * CG + cg]);
                add4(ww, red_w[r * CG + cg]);
            }
            float4 c;
            c.x = be * (vr.x - al * uu.x);
            c.y = be * (vr.y - al * uu.y);
            c.z = be * (vr.z - al * uu.z);
            c.w = be * (vr.w - al * uu.w);
            if (rg == 0) {
                const float kq = kq_s[n & 1];
                float4 o;
                o.x = fmaf(c.x, kq, al * ww.x);
                o.y = fmaf(c.y, kq, al * ww.y);
                o.z = fmaf(c.z, kq, al * ww.z);
                o.w = fmaf(c.w, kq, al * ww.w);
                __stcs(reinterpret_cast<float4*>(a.out + (size_t)u * P::DV) + cg, o);
            }
            const int h = u % a.Hv;
            float4* D = reinterpret_cast<float4*>(a.pool + ((size_t)m.x * a.Hv + h) * (P::DK * P::DV));
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                s[r].x = fmaf(kr[r], c.x, al * s[r].x);
                s[r].y = fmaf(kr[r], c.y, al * s[r].y);
                s[r].z = fmaf(kr[r], c.z, al * s[r].z);
                s[r].w = fmaf(kr[r], c.w, al * s[r].w);
                __stcs(D + (size_t)(r * RG + rg) * CG + cg, s[r]);
            }
        } else if (m.y == 0 && tid == 0) {
            record_error(a.err, GDN_ERR_INDEX);
        }
        // No second barrier: the next unit writes the other reduction buffer,
        // and this one is rewritten only after every thread has passed the
        // next unit's barrier, i.e. has finished reading it here.
    }
}

__global__ void gdn_commit_kernel(const int32_t* __restrict__ accept_len, int32_t* __restrict__ committed,
                                  const int32_t* __restrict__ cur, int B, int T, int num_slots, int32_t* err) {
    // Launched with programmatic dependent launch: the decode call before it may still
    // be draining when this grid starts, so wait for it before reading its tables.
    grid_dependency_wait();
    allow_dependent_launch();
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

// ---------------------------------------------------------------------------
// Precondition check of a decode call's slot indices (gdn_check_step).
// owner[] (int32 per slot, filled with -1 beforehand) records which request
// writes each slot: claiming a slot twice means two writes alias; a request
// whose source slot is owned by another request (or, with T > 1, by itself)
// would read a slot written in the same call.
// ---------------------------------------------------------------------------
__global__ void gdn_claim_dst_kernel(const int32_t* __restrict__ src_idx, const int32_t* __restrict__ dst_idx,
                                     int B, int T, int num_slots, int32_t* __restrict__ owner, int32_t* err) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)B * T) return;
    const int b = (int)(e / T);
    const int src = src_idx[b];
    if (src == GDN_SLOT_NONE) return;
    const int d = dst_idx[e];
    if (d < 0 || d >= num_slots || src < 0 || src >= num_slots) {
        // An index error outranks an alias report, whichever thread gets there first.
        if (atomicCAS(err, 0, GDN_ERR_INDEX) == GDN_ERR_ALIAS) atomicCAS(err, GDN_ERR_ALIAS, GDN_ERR_INDEX);
        return;
    }
    if (atomicCAS(owner + d, -1, b) != -1) record_error(err, GDN_ERR_ALIAS);
}

__global__ void gdn_check_src_kernel(const int32_t* __restrict__ src_idx, int B, int T, int num_slots,
                                     const int32_t* __restrict__ owner, int32_t* err) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int src = src_idx[b];
    if (src == GDN_SLOT_NONE || src < 0 || src >= num_slots) return;  // range errors: reported by the claim pass
    const int o = owner[src];
    if (o != -1 && (o != b || T > 1)) record_error(err, GDN_ERR_ALIAS);
}

constexpr int kMaxDk = 4096;

// Column-block width of the register-tile kernel (value columns per CTA) and
// its per-thread register budget, which sets how many CTAs stay resident per
// SM.  Compile-time tunables; the defaults are the measured best on B200
// (64 columns, 128 threads, 96 registers: 5 CTAs and 160 KiB in flight per SM).
#ifndef GDN_TILE_COLS
#define GDN_TILE_COLS 64
#endif
#ifndef GDN_TILE_MAXREG
#define GDN_TILE_MAXREG 100
#endif

// Launches a kernel that calls grid_dependency_wait() before its first memory
// access with programmatic dependent launch (plain stream order without it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, unsigned threads, cudaStream_t stream, Args... args) {
#if GDN_USE_PDL
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
#else
    kernel<<<grid, threads, 0, stream>>>(args...);
    return cudaSuccess;
#endif
}

template <int DK, int DV, bool FUSE>
gdn_status launch_tile_impl(const StepArgs& a, int32_t dtype, cudaStream_t stream) {
    constexpr int DVC = DV < GDN_TILE_COLS ? DV : GDN_TILE_COLS;
    constexpr int NT = (DVC / 4) * 8;  // 8 row groups
    constexpr int MINB0 = 65536 / (NT * GDN_TILE_MAXREG);
    constexpr int MINB = MINB0 < 1 ? 1 : (MINB0 > 16 ? 16 : MINB0);
    const dim3 grid((unsigned)(a.B * a.Hv * (DV / DVC)));
    const bool bf = dtype == GDN_BF16;
    cudaError_t e;
    if (a.T == 1) {
        e = bf ? launch_pdl(gdn_tile1_kernel<DK, DV, DVC, NT, MINB, __nv_bfloat16, FUSE>, grid, NT, stream, a)
               : launch_pdl(gdn_tile1_kernel<DK, DV, DVC, NT, MINB, float, FUSE>, grid, NT, stream, a);
    } else if (!FUSE && !a.prefill && a.T <= kStageT) {
        e = bf ? launch_pdl(gdn_tileT_kernel<DK, DV, DVC, NT, MINB, __nv_bfloat16>, grid, NT, stream, a)
               : launch_pdl(gdn_tileT_kernel<DK, DV, DVC, NT, MINB, float>, grid, NT, stream, a);
    } else {
        // The fused multi-token form needs a few more registers than 5 CTAs/SM allow.
        constexpr int MINB_T = (FUSE && MINB > 1) ? MINB - 1 : MINB;
        e = bf ? launch_pdl(gdn_tile_kernel<DK, DV, DVC, NT, MINB_T, __nv_bfloat16, true, FUSE>, grid, NT, stream, a)
               : launch_pdl(gdn_tile_kernel<DK, DV, DVC, NT, MINB_T, float, true, FUSE>, grid, NT, stream, a);
    }
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

template <int DK, int DV>
gdn_status launch_tile(const StepArgs& a, int32_t dtype, cudaStream_t stream) {
    return (a.flags & kFuseFlags) ? launch_tile_impl<DK, DV, true>(a, dtype, stream)
                                  : launch_tile_impl<DK, DV, false>(a, dtype, stream);
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

constexpr int kMaxDevices = 64;

int sm_count() {
    // Per-device SM counts, filled on first use; atomics because host threads may call
    // the library concurrently (every writer stores the same value).
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < kMaxDevices) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

template <int NT, typename InT>
gdn_status launch_stream(const StepArgs& a, cudaStream_t stream) {
    using P = StreamPlan<NT, InT>;
    const int sms = sm_count();
    if (sms <= 0) return GDN_ERR_CUDA;
    // The opt-in above 48 KiB is a per-function attribute: setting it on every
    // launch keeps the library free of device-state caches and costs ~1 us.
    if (cudaFuncSetAttribute(gdn_stream_kernel<NT, InT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)P::SMEM_BYTES) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int units = a.B * a.Hv;
    const int grid = units < sms ? units : sms;
    gdn_stream_kernel<NT, InT><<<grid, NT, P::SMEM_BYTES, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Which kernel serves a call: the streaming kernel needs one token, 128 x 128
// tiles, 16-byte aligned buffers (bulk copies) and B * Hv a multiple of 4 (the
// 16-byte gate chunks stay inside alpha/beta); the register-tile kernel needs
// a compiled tile shape and 16-byte aligned pool/out; the column kernel takes
// anything.
bool stream_ok(const StepArgs& a) {
    return (a.flags & kFuseFlags) == 0 && a.T == 1 && a.dk == 128 && a.dv == 128 && ((int64_t)a.B * a.Hv) % 4 == 0 && aligned16(a.pool) &&
           aligned16(a.out) && aligned16(a.q) && aligned16(a.k) && aligned16(a.v) && aligned16(a.alpha) &&
           aligned16(a.beta);
}

bool tile_ok(const StepArgs& a) {
    return ((a.dk == 128 && a.dv == 128) || (a.dk == 64 && a.dv == 64)) && aligned16(a.pool) && aligned16(a.out);
}

gdn_status launch(const StepArgs& a, int32_t dtype, int32_t variant, cudaStream_t stream) {
    const bool bf = dtype == GDN_BF16;
    if (variant == GDN_VARIANT_AUTO) {
        // Measured on B200 (large decode, 8192 tiles per call): register tiles
        // 164.8 us per call, bulk-copy pipeline 184.4 us, so the register-tile
        // family serves every shape it supports.
        if (tile_ok(a))
            variant = GDN_VARIANT_TILE;
        else if (stream_ok(a) && a.err != nullptr)
            variant = GDN_VARIANT_STREAM;
        else
            variant = GDN_VARIANT_COLUMN;
    }
    switch (variant) {
        case GDN_VARIANT_STREAM:
            // Its bounded waits report a timeout only through the error word, and a
            // unit abandoned that way leaves its destination unwritten: without the
            // word such a call could not be told from a successful one.
            if (!stream_ok(a) || a.err == nullptr) return GDN_ERR_INVALID_ARG;
            return bf ? launch_stream<256, __nv_bfloat16>(a, stream) : launch_stream<256, float>(a, stream);
        case GDN_VARIANT_TILE:
            if (!tile_ok(a)) return GDN_ERR_INVALID_ARG;
            return a.dk == 128 ? launch_tile<128, 128>(a, dtype, stream) : launch_tile<64, 64>(a, dtype, stream);
        case GDN_VARIANT_COLUMN:
            return launch_column(a, dtype, stream);
        default:
            return GDN_ERR_INVALID_ARG;
    }
}

}  // namespace

extern "C" gdn_status gdn_decode_step_variant(float* pool, int32_t num_slots, const int32_t* src_idx,
                                              const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                              const float* alpha, const float* beta, float* out, int32_t B,
                                              int32_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                                              int32_t qkv_dtype, int32_t* err_word, int32_t variant,
                                              cudaStream_t stream) {
    if (B < 0 || T < 1 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || num_slots < 1) return GDN_ERR_INVALID_ARG;
    if (Hv % Hk != 0 || dk > kMaxDk) return GDN_ERR_INVALID_ARG;
    if (qkv_dtype != GDN_F32 && qkv_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (variant < GDN_VARIANT_AUTO || variant > GDN_VARIANT_COLUMN) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Hv * 4 >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;  // grid: up to 4 CTAs per (b, h)
    if (B == 0) return GDN_OK;
    if (!pool || !src_idx || !dst_idx || !q || !k || !v || !alpha || !beta || !out) return GDN_ERR_INVALID_ARG;

    const StepArgs a{pool, src_idx, dst_idx, q, k, v, alpha, beta, out, err_word,
                     num_slots, B, T, Hk, Hv, dk, dv, Hv / Hk, 0, 0};
    return launch(a, qkv_dtype, variant, stream);
}

extern "C" gdn_status gdn_decode_step_fused(float* pool, int32_t num_slots, const int32_t* src_idx,
                                            const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                            const float* alpha_or_x, const float* beta_or_y, float* out, int32_t B,
                                            int32_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                                            int32_t qkv_dtype, int32_t flags, int32_t* err_word,
                                            cudaStream_t stream) {
    if (B < 0 || T < 1 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || num_slots < 1) return GDN_ERR_INVALID_ARG;
    if (Hv % Hk != 0 || dk > kMaxDk) return GDN_ERR_INVALID_ARG;
    if (qkv_dtype != GDN_F32 && qkv_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if ((flags & ~(kFuseFlags | GDN_SHARED_SOURCES)) != 0) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Hv * 4 >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!pool || !src_idx || !dst_idx || !q || !k || !v || !alpha_or_x || !beta_or_y || !out)
        return GDN_ERR_INVALID_ARG;
    const StepArgs a{pool, src_idx, dst_idx, q, k, v, alpha_or_x, beta_or_y, out, err_word,
                     num_slots, B, T, Hk, Hv, dk, dv, Hv / Hk, flags, 0};
    return launch(a, qkv_dtype, GDN_VARIANT_AUTO, stream);
}

extern "C" gdn_status gdn_decode_step(float* pool, int32_t num_slots, const int32_t* src_idx,
                                      const int32_t* dst_idx, const void* q, const void* k, const void* v,
                                      const float* alpha, const float* beta, float* out, int32_t B, int32_t T,
                                      int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int32_t qkv_dtype,
                                      int32_t* err_word, cudaStream_t stream) {
    return gdn_decode_step_variant(pool, num_slots, src_idx, dst_idx, q, k, v, alpha, beta, out, B, T, Hk, Hv, dk,
                                   dv, qkv_dtype, err_word, GDN_VARIANT_AUTO, stream);
}

extern "C" gdn_status gdn_prefill(float* pool, int32_t num_slots, const int32_t* src_idx, const int32_t* dst_idx,
                                  const void* q, const void* k, const void* v, const float* alpha, const float* beta,
                                  float* out, int32_t B, int32_t L, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                                  int32_t qkv_dtype, int32_t* err_word, cudaStream_t stream) {
    if (B < 0 || L < 1 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || num_slots < 1) return GDN_ERR_INVALID_ARG;
    if (Hv % Hk != 0 || dk > kMaxDk) return GDN_ERR_INVALID_ARG;
    if (qkv_dtype != GDN_F32 && qkv_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if ((int64_t)B * Hv * 4 >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!pool || !src_idx || !dst_idx || !q || !k || !v || !alpha || !beta || !out) return GDN_ERR_INVALID_ARG;
    const StepArgs a{pool, src_idx, dst_idx, q, k, v, alpha, beta, out, err_word,
                     num_slots, B, L, Hk, Hv, dk, dv, Hv / Hk, 0, 1};
    return launch(a, qkv_dtype, GDN_VARIANT_AUTO, stream);
}

extern "C" gdn_status gdn_commit(const int32_t* accept_len, int32_t* committed, const int32_t* cur, int32_t B,
                                 int32_t T, int32_t num_slots, int32_t* err_word, cudaStream_t stream) {
    if (B < 0 || T < 1 || num_slots < 1) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!accept_len || !committed || !cur) return GDN_ERR_INVALID_ARG;
    const int threads = 256;
    if (launch_pdl(gdn_commit_kernel, dim3((unsigned)((B + threads - 1) / threads)), threads, stream, accept_len,
                   committed, cur, (int)B, (int)T, (int)num_slots, err_word) != cudaSuccess)
        return GDN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" gdn_status gdn_check_step(const int32_t* src_idx, const int32_t* dst_idx, int32_t B, int32_t T,
                                     int32_t num_slots, int32_t* scratch, int32_t* err_word, cudaStream_t stream) {
    if (B < 0 || T < 1 || num_slots < 1 || (int64_t)B * T >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!src_idx || !dst_idx || !scratch || !err_word) return GDN_ERR_INVALID_ARG;
    // 0xFF bytes make every int32 owner entry -1 ("unclaimed").
    if (cudaMemsetAsync(scratch, 0xFF, sizeof(int32_t) * (size_t)num_slots, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int threads = 256;
    const int64_t n = (int64_t)B * T;
    gdn_claim_dst_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, stream>>>(src_idx, dst_idx, B, T,
                                                                                         num_slots, scratch, err_word);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    gdn_check_src_kernel<<<(B + threads - 1) / threads, threads, 0, stream>>>(src_idx, B, T, num_slots, scratch,
                                                                              err_word);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free precondition check.  The owner map lives in this file-scope
// device array (1 MiB per GPU that loads the library).  Host code must not pass
// `g_check_owner` itself to a kernel: on the host that name is only a stand-in
// for the device symbol.  Its device address is looked up once per device with
// cudaGetSymbolAddress and cached; the claim and source kernels above then run
// on it exactly as they run on a caller's scratch buffer.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t g_check_owner[GDN_CHECK_NOALLOC_MAX_SLOTS];

namespace {

std::atomic<int32_t*> g_check_owner_addr[kMaxDevices];

// Device address of g_check_owner on the current device (nullptr on failure).
int32_t* check_owner_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
    if (dev < kMaxDevices) {
        int32_t* cached = g_check_owner_addr[dev].load(std::memory_order_acquire);
        if (cached != nullptr) return cached;
    }
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_check_owner) != cudaSuccess || addr == nullptr) return nullptr;
    int32_t* owner = static_cast<int32_t*>(addr);
    if (dev < kMaxDevices) g_check_owner_addr[dev].store(owner, std::memory_order_release);
    return owner;
}

}  // namespace

extern "C" gdn_status gdn_check_step_noalloc(const int32_t* src_idx, const int32_t* dst_idx, int32_t B, int32_t T,
                                             int32_t num_slots, int32_t* err_word, cudaStream_t stream) {
    if (B < 0 || T < 1 || num_slots < 1 || (int64_t)B * T >= (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (num_slots > GDN_CHECK_NOALLOC_MAX_SLOTS) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!src_idx || !dst_idx || !err_word) return GDN_ERR_INVALID_ARG;
    int32_t* owner = check_owner_address();
    if (owner == nullptr) return GDN_ERR_CUDA;
    // Reset the entries this call uses (0xFF bytes = -1, "unclaimed"): the array
    // still holds whatever the previous call left there.
    if (cudaMemsetAsync(owner, 0xFF, sizeof(int32_t) * (size_t)num_slots, stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int threads = 256;
    const int64_t n = (int64_t)B * T;
    gdn_claim_dst_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, stream>>>(src_idx, dst_idx, B, T,
                                                                                         num_slots, owner, err_word);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    gdn_check_src_kernel<<<(B + threads - 1) / threads, threads, 0, stream>>>(src_idx, B, T, num_slots, owner,
                                                                              err_word);
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
        case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS";
        case GDN_ERR_CAPACITY: return "GDN_ERR_CAPACITY";
        default: return "GDN_UNKNOWN_STATUS";
    }
}
