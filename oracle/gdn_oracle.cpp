// gdn_oracle.cpp -- TEST INFRASTRUCTURE, not part of the product path.
//
// A plain, slow, obviously-correct CPU statement of the decode-time Gated
// DeltaNet (GDN) recurrent-state update with slot indirection.  Only the test
// suite, the package smoke check and the benchmark's CPU-baseline / reference
// legs load this library; the CUDA library never links, includes or calls it,
// and this file includes nothing from the CUDA side.
//
// What it follows:
//   * The recurrence is the gated delta rule of Gated DeltaNet (Yang, Kautz &
//     Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta Rule",
//     ICLR 2025), the mechanism that the TokenSpeed 580 tok/s article
//     (24-ai.news, English edition, opening section "What is TokenSpeed and
//     how does it differ from vLLM?") names for the model's linear-attention
//     layers.  Per token and value head, with S the dv x dk state:
//         S' = alpha * S * (I - beta * k k^T) + beta * v k^T,   o = S' q.
//     It is written here as the literal matrix product, in double.
//   * Slot semantics follow the same article's "Mamba State Update
//     optimization" item of "What are the key optimizations behind the
//     record?" (index indirection instead of tensor scatter) and its "Hybrid
//     prefix caching for GDN/Mamba" item (copy-on-write reuse), and the
//     zubnet.ai LightSeek TokenSpeed article, second paragraph (states in
//     Mamba state slots checkpointed beside the KV pages, speculative decoding
//     through current_input_indices, cached checkpoints reused without
//     mutation).
//
// Readings where the pages are silent (each one also listed in the design
// notes): state stored as M[i][j] = S[j][i] in a [slot][Hv][dk][dv] pool with
// dv contiguous; value head h reads key head h / (Hv / Hk); no q/k scaling or
// normalisation inside the step; alpha/beta are given per token and value head;
// every read sees the pool as it was before the call; the state is rounded to
// fp32 after every token (that is the stored value) and carried forward from
// the rounded value; o is computed in double from the fp32-rounded state and
// rounded to fp32; a request whose source index is -1 is padding and is
// skipped; any other request whose source or any destination index lies
// outside [0, num_slots) is skipped as a whole (no state, no output written)
// and counted.
//
// Commit: accept_len[b] draft tokens were accepted.  0 keeps the committed
// slot; a >= 1 selects the state written after draft token a-1, i.e.
// cur[b][a-1].  accept_len outside [0, T], or a selected slot outside
// [0, num_slots), skips the request and counts it.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// bfloat16 is the upper half of an IEEE binary32: widening is exact.
double bf16_to_double(uint16_t bits) {
    uint32_t u = static_cast<uint32_t>(bits) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

double input_at(const void* base, int32_t dtype, int64_t idx) {
    if (dtype == 1) return bf16_to_double(static_cast<const uint16_t*>(base)[idx]);
    return static_cast<double>(static_cast<const float*>(base)[idx]);
}

struct Problem {
    const float* pool;
    int64_t num_slots;
    const int32_t* src_idx;
    const int32_t* dst_idx;
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    int64_t B, T, Hk, Hv, dk, dv;
    int32_t dtype;
    int32_t flags;  // 1: alpha/beta are raw x, y; 2: L2-normalise q and k
    bool last_only; // prefill: dst_idx is [B]; only the state after the last token is kept
};

// Fused prologue, from its definition: alpha = exp(-softplus(x)) with
// softplus(x) = log(1 + e^x) (written so that e^x never overflows), beta =
// sigmoid(y) = 1 / (1 + e^-y), and x_hat = x / sqrt(sum x^2 + 1e-6).
double softplus(double x) { return x > 0.0 ? x + std::log1p(std::exp(-x)) : std::log1p(std::exp(x)); }
double alpha_of(double x) { return std::exp(-softplus(x)); }
double beta_of(double y) { return 1.0 / (1.0 + std::exp(-y)); }

void l2_normalise(std::vector<double>& x) {
    double ss = 0.0;
    for (double e : x) ss += e * e;
    const double n = std::sqrt(ss + 1e-6);
    for (double& e : x) e /= n;
}

// A source index of -1 marks a padding request: skipped, not an error.
bool request_is_padding(const Problem& p, int64_t b) { return p.src_idx[b] == -1; }

bool request_is_valid(const Problem& p, int64_t b) {
    const int64_t s = p.src_idx[b];
    if (s < 0 || s >= p.num_slots) return false;
    const int64_t nd = p.last_only ? 1 : p.T;
    for (int64_t t = 0; t < nd; ++t) {
        const int64_t d = p.dst_idx[b * nd + t];
        if (d < 0 || d >= p.num_slots) return false;
    }
    return true;
}

// Computes every token's new state (stored layout [T][Hv][dk][dv], fp32) and
// output ([T][Hv][dv], fp32) for request b.  Reads the pool only.
void solve_request(const Problem& p, int64_t b, float* states, float* outs) {
    const int64_t dk = p.dk, dv = p.dv;
    const int64_t G = p.Hv / p.Hk;
    const int64_t src = p.src_idx[b];

    std::vector<double> S(dv * dk);      // logical S[j][i], j < dv, i < dk
    std::vector<double> P(dk * dk);      // I - beta k k^T
    std::vector<double> SP(dv * dk);     // S * P
    std::vector<double> kv(dk), qv(dk), vv(dv);
    std::vector<float> Sf(dv * dk);      // fp32-rounded S'

    for (int64_t h = 0; h < p.Hv; ++h) {
        // Gather the source state of head h: stored M[i][j] = S[j][i].
        const float* M = p.pool + ((src * p.Hv + h) * dk) * dv;
        for (int64_t j = 0; j < dv; ++j)
            for (int64_t i = 0; i < dk; ++i) S[j * dk + i] = static_cast<double>(M[i * dv + j]);

        const int64_t hk = h / G;
        for (int64_t t = 0; t < p.T; ++t) {
            const int64_t tok = b * p.T + t;
            for (int64_t i = 0; i < dk; ++i) {
                kv[i] = input_at(p.k, p.dtype, (tok * p.Hk + hk) * dk + i);
                qv[i] = input_at(p.q, p.dtype, (tok * p.Hk + hk) * dk + i);
            }
            for (int64_t j = 0; j < dv; ++j) vv[j] = input_at(p.v, p.dtype, (tok * p.Hv + h) * dv + j);
            double a = p.alpha[tok * p.Hv + h];
            double be = p.beta[tok * p.Hv + h];
            if (p.flags & 1) {
                a = alpha_of(a);
                be = beta_of(be);
            }
            if (p.flags & 2) {
                l2_normalise(kv);
                l2_normalise(qv);
            }

            // P = I - beta k k^T
            for (int64_t r = 0; r < dk; ++r)
                for (int64_t c = 0; c < dk; ++c) P[r * dk + c] = (r == c ? 1.0 : 0.0) - be * kv[r] * kv[c];

            // SP = S P
            for (int64_t j = 0; j < dv; ++j)
                for (int64_t i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int64_t l = 0; l < dk; ++l) acc += S[j * dk + l] * P[l * dk + i];
                    SP[j * dk + i] = acc;
                }

            // S' = alpha SP + beta v k^T, rounded to fp32 (the stored value),
            // and carried to the next token from the rounded value.
            for (int64_t j = 0; j < dv; ++j)
                for (int64_t i = 0; i < dk; ++i) {
                    const double s_new = a * SP[j * dk + i] + be * vv[j] * kv[i];
                    Sf[j * dk + i] = static_cast<float>(s_new);
                    S[j * dk + i] = static_cast<double>(Sf[j * dk + i]);
                }

            // Stored layout of token t, head h: [dk][dv] (prefill keeps the last token only).
            if (!p.last_only || t == p.T - 1) {
                float* St = states + (((p.last_only ? 0 : t) * p.Hv + h) * dk) * dv;
                for (int64_t i = 0; i < dk; ++i)
                    for (int64_t j = 0; j < dv; ++j) St[i * dv + j] = Sf[j * dk + i];
            }

            // o = S' q from the fp32-rounded S'.
            float* ot = outs + (t * p.Hv + h) * dv;
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < dk; ++i) acc += static_cast<double>(Sf[j * dk + i]) * qv[i];
                ot[j] = static_cast<float>(acc);
            }
        }
    }
}

}  // namespace

namespace {

int64_t run_calls(float* pool, int64_t num_slots, const int32_t* src_idx, const int32_t* dst_idx, const void* q,
                  const void* k, const void* v, const float* alpha, const float* beta, float* out, int64_t B,
                  int64_t T, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, int32_t dtype, int32_t flags,
                  bool last_only, int32_t nthreads) {
    if (B < 0 || T < 1 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || num_slots < 1) return -1;
    if (Hv % Hk != 0 || (dtype != 0 && dtype != 1) || (flags & ~3) != 0) return -1;
    if (B == 0) return 0;

    Problem p{pool, num_slots, src_idx, dst_idx, q, k, v, alpha, beta, B, T, Hk, Hv, dk, dv, dtype, flags,
              last_only};
    const int64_t kept = last_only ? 1 : T;  // states kept per request
    const int64_t state_elems = kept * Hv * dk * dv;
    const int64_t out_elems = T * Hv * dv;
    std::vector<float> states(static_cast<size_t>(B * state_elems));
    std::vector<float> outs(static_cast<size_t>(B * out_elems));
    std::vector<char> valid(static_cast<size_t>(B));

    auto work = [&](int64_t b0, int64_t b1) {
        for (int64_t b = b0; b < b1; ++b) {
            valid[b] = request_is_padding(p, b) ? 2 : (request_is_valid(p, b) ? 1 : 0);
            if (valid[b] == 1) solve_request(p, b, &states[b * state_elems], &outs[b * out_elems]);
        }
    };
    int64_t nt = nthreads < 1 ? 1 : nthreads;
    if (nt > B) nt = B;
    if (nt == 1) {
        work(0, B);
    } else {
        std::vector<std::thread> pool_threads;
        for (int64_t w = 0; w < nt; ++w)
            pool_threads.emplace_back(work, B * w / nt, B * (w + 1) / nt);
        for (auto& th : pool_threads) th.join();
    }

    int64_t skipped = 0;
    const int64_t tile = dk * dv;
    for (int64_t b = 0; b < B; ++b) {
        if (valid[b] != 1) {
            if (valid[b] == 0) ++skipped;
            continue;
        }
        for (int64_t t = 0; t < T; ++t) {
            if (!last_only || t == T - 1) {
                const int64_t d = last_only ? dst_idx[b] : dst_idx[b * T + t];
                const int64_t ts = last_only ? 0 : t;
                for (int64_t h = 0; h < Hv; ++h)
                    std::memcpy(pool + (d * Hv + h) * tile, &states[b * state_elems + (ts * Hv + h) * tile],
                                sizeof(float) * tile);
            }
            std::memcpy(out + (b * T + t) * Hv * dv, &outs[b * out_elems + t * Hv * dv],
                        sizeof(float) * Hv * dv);
        }
    }
    return skipped;
}

}  // namespace

extern "C" {

// One decode call, with the optional fused prologue (flags: 1 = alpha/beta hold
// raw x, y; 2 = L2-normalise q and k).  pool: [num_slots][Hv][dk][dv] fp32,
// updated in place.
// src_idx: [B]; dst_idx: [B][T]; q, k: [B][T][Hk][dk]; v: [B][T][Hv][dv]
// (dtype 0 = fp32, 1 = bf16 bit patterns); alpha, beta: [B][T][Hv] fp32;
// out: [B][T][Hv][dv] fp32.  All buffers are host memory owned by the caller.
// Every request is solved from the pre-call pool before anything is written;
// writes then go out in (b, t) order.  nthreads <= 1 runs single-threaded.
// Returns the number of requests skipped for an out-of-range index (padding
// requests are not counted), or -1 for invalid sizes.
int64_t oracle_gdn_decode_step_fused(float* pool, int64_t num_slots, const int32_t* src_idx,
                                     const int32_t* dst_idx, const void* q, const void* k,
                                     const void* v, const float* alpha, const float* beta, float* out,
                                     int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk,
                                     int64_t dv, int32_t dtype, int32_t flags, int32_t nthreads) {
    return run_calls(pool, num_slots, src_idx, dst_idx, q, k, v, alpha, beta, out, B, T, Hk, Hv, dk, dv, dtype,
                     flags, false, nthreads);
}

// Prefill: the same per-token update over T = L tokens, keeping only the state
// after the last token (written to dst_idx[b], dst_idx is [B]); every token's
// output is written.  Returns skipped requests as above.
int64_t oracle_gdn_prefill(float* pool, int64_t num_slots, const int32_t* src_idx, const int32_t* dst_idx,
                           const void* q, const void* k, const void* v, const float* alpha, const float* beta,
                           float* out, int64_t B, int64_t L, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                           int32_t dtype, int32_t nthreads) {
    return run_calls(pool, num_slots, src_idx, dst_idx, q, k, v, alpha, beta, out, B, L, Hk, Hv, dk, dv, dtype, 0,
                     true, nthreads);
}

// The plain call: alpha and beta given, q and k used as they are.
int64_t oracle_gdn_decode_step(float* pool, int64_t num_slots, const int32_t* src_idx,
                               const int32_t* dst_idx, const void* q, const void* k,
                               const void* v, const float* alpha, const float* beta, float* out,
                               int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk,
                               int64_t dv, int32_t dtype, int32_t nthreads) {
    return oracle_gdn_decode_step_fused(pool, num_slots, src_idx, dst_idx, q, k, v, alpha, beta, out,
                                        B, T, Hk, Hv, dk, dv, dtype, 0, nthreads);
}

// Precondition check of one decode call's slot indices, by brute force over
// all pairs.  Returns 0 when they hold, 3 when a non-padding request has a
// source or destination outside [0, num_slots), 5 when two destinations
// coincide, a destination equals another request's source, or (T > 1) a
// destination equals the request's own source; an index error takes
// precedence.  Requests whose source is -1 are ignored.  -1 for invalid sizes.
int32_t oracle_gdn_check_step(const int32_t* src_idx, const int32_t* dst_idx, int64_t B, int64_t T,
                              int64_t num_slots) {
    if (B < 0 || T < 1 || num_slots < 1) return -1;
    auto live = [&](int64_t b) { return src_idx[b] != -1; };
    for (int64_t b = 0; b < B; ++b) {
        if (!live(b)) continue;
        if (src_idx[b] < 0 || src_idx[b] >= num_slots) return 3;
        for (int64_t t = 0; t < T; ++t)
            if (dst_idx[b * T + t] < 0 || dst_idx[b * T + t] >= num_slots) return 3;
    }
    for (int64_t e = 0; e < B * T; ++e) {
        if (!live(e / T)) continue;
        for (int64_t f = e + 1; f < B * T; ++f)
            if (live(f / T) && dst_idx[e] == dst_idx[f]) return 5;
    }
    for (int64_t b = 0; b < B; ++b) {
        if (!live(b)) continue;
        for (int64_t e = 0; e < B * T; ++e) {
            const int64_t w = e / T;
            if (!live(w) || dst_idx[e] != src_idx[b]) continue;
            if (w != b || T > 1) return 5;
        }
    }
    return 0;
}

// Accept-length commit.  committed: [B] int32 (updated in place); cur: [B][T].
// Returns the number of skipped requests, or -1 for invalid sizes.
int64_t oracle_gdn_commit(const int32_t* accept_len, int32_t* committed, const int32_t* cur,
                          int64_t B, int64_t T, int64_t num_slots) {
    if (B < 0 || T < 1 || num_slots < 1) return -1;
    int64_t skipped = 0;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t a = accept_len[b];
        if (a < 0 || a > T) {
            ++skipped;
            continue;
        }
        if (a == 0) continue;
        const int64_t s = cur[b * T + (a - 1)];
        if (s < 0 || s >= num_slots) {
            ++skipped;
            continue;
        }
        committed[b] = static_cast<int32_t>(s);
    }
    return skipped;
}

}  // extern "C"
