// Float64 CPU oracle for exact scaled-dot-product attention.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
// this file: only the tests, the smoke check and the bench's CPU-baseline leg
// use it. It shares no code, header or constant with the CUDA library.
//
// What it computes follows "1-Flash-Attention.md" (huajishe.fun), section
// "问题分析" (standard attention: S = Q K^T, A = softmax(S / sqrt(d)), O = A V on
// (batch, heads, seq_len, head_dim) tensors), with the caller's softmax scale in
// place of 1/sqrt(d) (section "框架集成", softmax_scale). Every value is widened
// to double before any arithmetic and nothing is rounded on the way out.
//
// Readings where the pages are silent (each also listed in the design notes):
//  * causal: query row i sees key j iff j <= i (prefill has Nq == Nk);
//  * LSE_i = ln sum_{j visible} exp(scale * q_i . k_j)  (natural log, scale in);
//  * GQA/MQA: query head h reads key/value head h / (Hq / Hkv) (consecutive
//    query heads share one key/value head);
//  * split-KV partials are normalised: O_s = sum_s p v / l_s with lse_s; an
//    empty split has lse_s = -inf, O_s = 0 and weight 0 in the merge.
//
// Functions:
//  oracle_attention_rows            direct definition, selected rows
//  oracle_attention_blockwise_rows  the tiled online-softmax recurrence
//                                   ("递归计算softmax" section) - must equal
//                                   the direct definition
//  oracle_decode_partials           per-split partial (O_s, lse_s)
//  oracle_combine                   logsumexp-weighted merge of partials
//  oracle_attention_backward        dQ, dK, dV from the definition
//  oracle_quant_fp8                 block quantisation to FP8 (E4M3) codes
//  oracle_e4m3_decode               FP8 (E4M3) code -> value
//  oracle_hadamard_rotate           the rotation of incoherent processing
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

// ORACLE_PLANT selects one deliberate mistake for the mutation tests, which
// check that the pins catch it; 0 (the default build) plants nothing.
#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

namespace {

constexpr int kPlant = ORACLE_PLANT;

enum InType { IN_F64 = 0, IN_BF16 = 1, IN_F32 = 2, IN_F16 = 3 };

// IEEE 754 binary16 -> double from the format's definition: sign bit, 5
// exponent bits with bias 15, 10 fraction bits; exponent 0 holds zero and the
// subnormals (fraction * 2^-24), exponent 31 the infinities and NaN.
inline double half_to_double(uint16_t h) {
    const int sign = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
    double mag;
    if (e == 0)
        mag = std::ldexp(static_cast<double>(f), -24);
    else if (e == 31)
        mag = f ? std::numeric_limits<double>::quiet_NaN() : std::numeric_limits<double>::infinity();
    else
        mag = std::ldexp(1.0 + f / 1024.0, e - 15);
    return sign ? -mag : mag;
}

// bf16 -> double: a bf16 value is the top 16 bits of an IEEE float32.
inline double load_elem(int dtype, const void* base, int64_t idx) {
    switch (dtype) {
        case IN_F64: return static_cast<const double*>(base)[idx];
        case IN_F32: return static_cast<const float*>(base)[idx];
        case IN_F16: return half_to_double(static_cast<const uint16_t*>(base)[idx]);
        default: {
            uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(base)[idx]) << 16;
            float f;
            std::memcpy(&f, &bits, sizeof f);
            return f;
        }
    }
}

// FP8 E4M3 (the "fn" variant: 1 sign bit, 4 exponent bits with bias 7, 3
// fraction bits, no infinities, S.1111.111 is NaN, largest finite 448), from
// the format's definition: exponent field 0 holds zero and the subnormals
// (fraction * 2^-9); otherwise (1 + fraction / 8) * 2^(e - 7).
inline double e4m3_value(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, f = c & 7;
    double mag;
    if (e == 15 && f == 7)
        mag = std::numeric_limits<double>::quiet_NaN();
    else if (e == 0)
        mag = std::ldexp(static_cast<double>(f), -9);
    else
        mag = std::ldexp(1.0 + f / 8.0, e - 7);
    return sign ? -mag : mag;
}

// Nearest E4M3 value to a finite float, ties to the even code, magnitudes past
// 448 saturated to 448. The step between neighbours is 2^(E-3) in the binade
// [2^E, 2^(E+1)) for E >= -6, and 2^-9 below 2^-6 (the subnormals); dividing by
// the step is exact, so one rounding to an integer count of steps decides it.
inline uint8_t e4m3_code(float x) {
    const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
    const double a = std::fabs(static_cast<double>(x));
    if (a >= 448.0) return sign | 0x7E;  // saturate (448 = 1.75 * 2^8)
    int E = a > 0.0 ? std::ilogb(a) : -7;
    if (E < -6) E = -6;
    const double step = std::ldexp(1.0, E - 3);
    double n = a / step;
    double r = std::floor(n);
    const double frac = n - r;
    if (kPlant == 10) {
        // 10: rounds toward zero
    } else if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) {
        r += 1.0;
    }
    // r steps of 2^(E-3): r in [8, 16] for a normal binade (16 carries into
    // the next binade), r in [0, 8] for the subnormal range
    const double v = r * step;
    if (v == 0.0) return sign;
    if (v >= 448.0) return sign | 0x7E;
    int Ev = std::ilogb(v);
    if (Ev < -6) return sign | static_cast<uint8_t>(r);  // subnormal: fraction = r
    const int frac_bits = static_cast<int>(std::ldexp(v, -Ev) * 8.0) - 8;
    return sign | static_cast<uint8_t>(((Ev + 7) << 3) | frac_bits);
}

struct Problem {
    int dtype;
    const void *q, *k, *v;
    int B, Hq, Hkv, Nq, Nk, d, causal;
    double scale;
};

// Visible keys of query row i: [0, Nk) or [0, i] when causal.
inline int64_t visible_keys(const Problem& p, int64_t i) {
    if (kPlant == 3) return p.causal ? std::min<int64_t>(i + 2, p.Nk) : p.Nk;  // off by one
    if (kPlant == 8) return p.causal ? std::max<int64_t>(i, 1) : std::max(p.Nk - 1, 1);  // drops a key
    return p.causal ? std::min<int64_t>(i + 1, p.Nk) : p.Nk;
}

// Query head h reads key/value head h / G.
inline int64_t kv_head(const Problem& p, int64_t h) {
    if (kPlant == 2) return h % p.Hkv;  // wrong GQA grouping
    return h / (p.Hq / p.Hkv);
}

// s_j = scale * sum_t q[t] k_j[t] for the visible keys of one row.
void scores(const Problem& p, int64_t b, int64_t h, int64_t i, std::vector<double>& s) {
    const int64_t hk = kv_head(p, h);
    const int64_t qoff = ((b * p.Hq + h) * p.Nq + i) * p.d;
    const int64_t koff = (b * p.Hkv + hk) * static_cast<int64_t>(p.Nk) * p.d;
    const int64_t J = visible_keys(p, i);
    s.assign(J, 0.0);
    for (int64_t j = 0; j < J; ++j) {
        double acc = 0.0;
        for (int t = 0; t < p.d; ++t) {
            const int64_t kidx = (kPlant == 7) ? koff + t * p.Nk + j : koff + j * p.d + t;  // 7: K^T
            acc += load_elem(p.dtype, p.q, qoff + t) * load_elem(p.dtype, p.k, kidx);
        }
        s[j] = (kPlant == 1) ? acc : p.scale * acc;  // 1: scale dropped
    }
}

// Direct definition for one row: softmax over the visible scores, then A V.
void direct_row(const Problem& p, int64_t row, double* o, double* lse, double* prob) {
    const int64_t i = row % p.Nq;
    const int64_t bh = row / p.Nq;
    const int64_t h = bh % p.Hq, b = bh / p.Hq;
    const int64_t hk = kv_head(p, h);
    const int64_t voff = (b * p.Hkv + hk) * static_cast<int64_t>(p.Nk) * p.d;
    std::vector<double> s;
    scores(p, b, h, i, s);
    const int64_t J = static_cast<int64_t>(s.size());
    double m = -std::numeric_limits<double>::infinity();
    for (double x : s) m = std::max(m, x);
    double l = 0.0;
    for (int64_t j = 0; j < J; ++j) { s[j] = std::exp(s[j] - m); l += s[j]; }
    for (int t = 0; t < p.d; ++t) o[t] = 0.0;
    for (int64_t j = 0; j < J; ++j) {
        const double a = s[j] / l;
        if (prob) prob[j] = a;
        for (int t = 0; t < p.d; ++t) o[t] += a * load_elem(p.dtype, p.v, voff + j * p.d + t);
    }
    if (prob) for (int64_t j = J; j < p.Nk; ++j) prob[j] = 0.0;
    *lse = (kPlant == 4) ? m + std::log2(l) : m + std::log(l);  // 4: log base 2
}

// The page's block recurrence, keys visited in blocks of Bk:
//   rowmax = max_j S_ij;  P_ij = exp(S_ij - rowmax)
//   m_new = max(m_old, rowmax)
//   d_new = d_old * exp(m_old - m_new) + exp(rowmax - m_new) * sum_j P_ij
//   O_new = O_old * exp(m_old - m_new) + exp(rowmax - m_new) * (P_ij @ V_j)
// and the normalisation O / d once at the end.
void blockwise_row(const Problem& p, int64_t row, int Bk, double* o, double* lse) {
    const int64_t i = row % p.Nq;
    const int64_t bh = row / p.Nq;
    const int64_t h = bh % p.Hq, b = bh / p.Hq;
    const int64_t hk = kv_head(p, h);
    const int64_t voff = (b * p.Hkv + hk) * static_cast<int64_t>(p.Nk) * p.d;
    std::vector<double> s;
    scores(p, b, h, i, s);
    const int64_t J = static_cast<int64_t>(s.size());
    double m_old = -std::numeric_limits<double>::infinity();
    double d_old = 0.0;
    std::vector<double> acc(p.d, 0.0), pv(p.d);
    for (int64_t j0 = 0; j0 < J; j0 += Bk) {
        const int64_t j1 = std::min<int64_t>(J, j0 + Bk);
        double rowmax = -std::numeric_limits<double>::infinity();
        for (int64_t j = j0; j < j1; ++j) rowmax = std::max(rowmax, s[j]);
        double psum = 0.0;
        std::fill(pv.begin(), pv.end(), 0.0);
        for (int64_t j = j0; j < j1; ++j) {
            const double pij = std::exp(s[j] - rowmax);
            psum += pij;
            for (int t = 0; t < p.d; ++t) pv[t] += pij * load_elem(p.dtype, p.v, voff + j * p.d + t);
        }
        const double m_new = std::max(m_old, rowmax);
        double f_old = (d_old == 0.0) ? 0.0 : std::exp(m_old - m_new);
        if (kPlant == 5 && d_old != 0.0) f_old = 1.0;  // 5: old state not rescaled
        const double f_blk = std::exp(rowmax - m_new);
        const double d_new = d_old * f_old + f_blk * psum;
        for (int t = 0; t < p.d; ++t) acc[t] = acc[t] * f_old + f_blk * pv[t];
        m_old = m_new;
        d_old = d_new;
    }
    for (int t = 0; t < p.d; ++t) o[t] = acc[t] / d_old;
    *lse = m_old + std::log(d_old);
}

int resolve_threads(int nthreads) {
    if (nthreads > 0) return nthreads;
    unsigned hc = std::thread::hardware_concurrency();
    return hc ? static_cast<int>(hc) : 1;
}

template <class F>
void parallel_rows(int64_t nrows, int nthreads, F fn) {
    nthreads = static_cast<int>(std::min<int64_t>(resolve_threads(nthreads), std::max<int64_t>(nrows, 1)));
    if (nthreads <= 1) { for (int64_t r = 0; r < nrows; ++r) fn(r); return; }
    std::vector<std::thread> pool;
    for (int t = 0; t < nthreads; ++t)
        pool.emplace_back([=] { for (int64_t r = t; r < nrows; r += nthreads) fn(r); });
    for (auto& th : pool) th.join();
}

int check(const Problem& p) {
    if (p.B < 1 || p.Hq < 1 || p.Hkv < 1 || p.Nq < 1 || p.Nk < 1 || p.d < 1) return 1;
    if (p.Hq % p.Hkv != 0) return 2;
    if (p.causal && p.Nq != p.Nk) return 3;
    return 0;
}

}  // namespace

extern "C" {

int oracle_hardware_threads() { return resolve_threads(0); }

// Direct attention for `nrows` rows; rows[r] = (b*Hq + h)*Nq + i.
// o: nrows x d, lse: nrows, prob (optional): nrows x Nk. Returns 0 on success.
int oracle_attention_rows(int dtype, const void* q, const void* k, const void* v,
                          int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, double scale,
                          const int64_t* rows, int64_t nrows, double* o, double* lse, double* prob,
                          int nthreads) {
    Problem p{dtype, q, k, v, B, Hq, Hkv, Nq, Nk, d, causal, scale};
    if (int e = check(p)) return e;
    const int64_t total = static_cast<int64_t>(B) * Hq * Nq;
    for (int64_t r = 0; r < nrows; ++r) if (rows[r] < 0 || rows[r] >= total) return 4;
    parallel_rows(nrows, nthreads, [&](int64_t r) {
        direct_row(p, rows[r], o + r * d, lse + r, prob ? prob + r * static_cast<int64_t>(Nk) : nullptr);
    });
    return 0;
}

// The blockwise online-softmax recurrence with key block size block_k.
int oracle_attention_blockwise_rows(int dtype, const void* q, const void* k, const void* v,
                                    int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                                    double scale, int block_k, const int64_t* rows, int64_t nrows,
                                    double* o, double* lse, int nthreads) {
    Problem p{dtype, q, k, v, B, Hq, Hkv, Nq, Nk, d, causal, scale};
    if (int e = check(p)) return e;
    if (block_k < 1) return 5;
    const int64_t total = static_cast<int64_t>(B) * Hq * Nq;
    for (int64_t r = 0; r < nrows; ++r) if (rows[r] < 0 || rows[r] >= total) return 4;
    parallel_rows(nrows, nthreads, [&](int64_t r) { blockwise_row(p, rows[r], block_k, o + r * d, lse + r); });
    return 0;
}

// Split-KV partials for single-query decode: q [B,Hq,d], k/v [B,Hkv,L,d].
// Split s covers keys [s*chunk, min(L, (s+1)*chunk)).
// o_part [B,Hq,S,d] (normalised), lse_part [B,Hq,S]; empty split -> 0 / -inf.
int oracle_decode_partials(int dtype, const void* q, const void* k, const void* v,
                           int B, int Hq, int Hkv, int L, int d, int num_splits, int chunk,
                           double scale, double* o_part, double* lse_part, int nthreads) {
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || d < 1 || num_splits < 1 || chunk < 1) return 1;
    if (Hq % Hkv != 0) return 2;
    const int64_t G = Hq / Hkv;
    const int64_t units = static_cast<int64_t>(B) * Hq * num_splits;
    parallel_rows(units, nthreads, [&](int64_t u) {
        const int64_t s = u % num_splits, bh = u / num_splits;
        const int64_t h = bh % Hq, b = bh / Hq, hk = h / G;
        const int64_t j0 = s * chunk, j1 = std::min<int64_t>(L, j0 + chunk);
        double* o = o_part + u * d;
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        if (j0 >= j1) { lse_part[u] = -std::numeric_limits<double>::infinity(); return; }
        const int64_t qoff = bh * d;
        const int64_t kvoff = (b * Hkv + hk) * static_cast<int64_t>(L) * d;
        std::vector<double> sc(j1 - j0);
        double m = -std::numeric_limits<double>::infinity();
        for (int64_t j = j0; j < j1; ++j) {
            double acc = 0.0;
            for (int t = 0; t < d; ++t)
                acc += load_elem(dtype, q, qoff + t) * load_elem(dtype, k, kvoff + j * d + t);
            sc[j - j0] = scale * acc;
            m = std::max(m, sc[j - j0]);
        }
        double l = 0.0;
        for (auto& x : sc) { x = std::exp(x - m); l += x; }
        for (int64_t j = j0; j < j1; ++j)
            for (int t = 0; t < d; ++t)
                o[t] += (kPlant == 9 ? sc[j - j0] : sc[j - j0] / l) * load_elem(dtype, v, kvoff + j * d + t);
        lse_part[u] = m + std::log(l);
    });
    return 0;
}

// Gradients of the scalar sum(dO * O) with respect to Q, K and V, from the
// definition (backward pass; the forward's LSE is recomputed, not taken from
// the GPU): for the visible keys j of row i, with P the softmax of the row,
//   dP_ij = dO_i . v_j,   Delta_i = sum_j P_ij dP_ij,   dS_ij = P_ij (dP_ij - Delta_i),
//   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,  dV_j = sum_i P_ij dO_i,
// dK and dV summed over every query head that reads the key/value head.
// Threads take whole (batch, key/value head) groups, so no sums are shared.
int oracle_attention_backward(int dtype, const void* q, const void* k, const void* v, const void* dout, int B,
                              int Hq, int Hkv, int N, int d, int causal, double scale, double* dq, double* dk,
                              double* dv, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1 ||
        Hq % Hkv != 0)
        return 1;
    Problem p{dtype, q, k, v, B, Hq, Hkv, N, N, d, causal, scale};
    const int G = Hq / Hkv;
    const int64_t groups = static_cast<int64_t>(B) * Hkv;
    const int nt = nthreads > 0 ? nthreads : std::max(1u, std::thread::hardware_concurrency());
    auto work = [&](int tid) {
        std::vector<double> s, dp;
        for (int64_t gidx = tid; gidx < groups; gidx += nt) {
            const int64_t b = gidx / Hkv, hk = gidx % Hkv;
            const int64_t kvoff = (b * Hkv + hk) * static_cast<int64_t>(N) * d;
            for (int64_t e = 0; e < static_cast<int64_t>(N) * d; ++e) dk[kvoff + e] = dv[kvoff + e] = 0.0;
            for (int64_t h = hk * G; h < (hk + 1) * G; ++h) {
                for (int64_t i = 0; i < N; ++i) {
                    const int64_t qoff = ((b * Hq + h) * N + i) * d;
                    scores(p, b, h, i, s);
                    const int64_t J = static_cast<int64_t>(s.size());
                    double m = -std::numeric_limits<double>::infinity();
                    for (double x : s) m = std::max(m, x);
                    double l = 0.0;
                    for (int64_t j = 0; j < J; ++j) { s[j] = std::exp(s[j] - m); l += s[j]; }
                    for (int64_t j = 0; j < J; ++j) s[j] /= l;  // P_ij
                    dp.assign(J, 0.0);
                    double delta = 0.0;
                    for (int64_t j = 0; j < J; ++j) {
                        double acc = 0.0;
                        for (int t = 0; t < d; ++t)
                            acc += load_elem(dtype, dout, qoff + t) * load_elem(dtype, v, kvoff + j * d + t);
                        dp[j] = acc;
                        delta += s[j] * acc;
                    }
                    for (int t = 0; t < d; ++t) dq[qoff + t] = 0.0;
                    for (int64_t j = 0; j < J; ++j) {
                        const double ds = s[j] * (dp[j] - delta);
                        for (int t = 0; t < d; ++t) {
                            dq[qoff + t] += scale * ds * load_elem(dtype, k, kvoff + j * d + t);
                            dk[kvoff + j * d + t] += scale * ds * load_elem(dtype, q, qoff + t);
                            dv[kvoff + j * d + t] += s[j] * load_elem(dtype, dout, qoff + t);
                        }
                    }
                }
            }
        }
    };
    std::vector<std::thread> pool;
    for (int t = 0; t < nt; ++t) pool.emplace_back(work, t);
    for (auto& th : pool) th.join();
    return 0;
}

// Widens n elements of one of the input types to double (exposes load_elem to
// the tests that pin the format conversions).
int oracle_widen(int dtype, const void* x, int64_t n, double* out) {
    if (x == nullptr || out == nullptr || n < 0 || dtype < IN_F64 || dtype > IN_F16) return 1;
    for (int64_t i = 0; i < n; ++i) out[i] = load_elem(dtype, x, i);
    return 0;
}

// Logsumexp-weighted merge: M = max_s lse_s, w_s = exp(lse_s - M),
// O = sum_s w_s O_s / sum_s w_s, LSE = M + ln sum_s w_s.
int oracle_combine(const double* o_part, const double* lse_part, int B, int Hq, int num_splits,
                   int d, double* o, double* lse) {
    if (B < 1 || Hq < 1 || num_splits < 1 || d < 1) return 1;
    for (int64_t bh = 0; bh < static_cast<int64_t>(B) * Hq; ++bh) {
        const double* ls = lse_part + bh * num_splits;
        double M = -std::numeric_limits<double>::infinity();
        for (int s = 0; s < num_splits; ++s) M = std::max(M, ls[s]);
        double wsum = 0.0;
        for (int t = 0; t < d; ++t) o[bh * d + t] = 0.0;
        if (M == -std::numeric_limits<double>::infinity()) { lse[bh] = M; continue; }
        for (int s = 0; s < num_splits; ++s) {
            if (ls[s] == -std::numeric_limits<double>::infinity()) continue;
            const double w = (kPlant == 6) ? 1.0 : std::exp(ls[s] - M);  // 6: plain average
            wsum += w;
            for (int t = 0; t < d; ++t) o[bh * d + t] += w * o_part[(bh * num_splits + s) * d + t];
        }
        for (int t = 0; t < d; ++t) o[bh * d + t] /= wsum;
        lse[bh] = M + std::log(wsum);
    }
    return 0;
}

// FP8 block quantisation (FlashAttention-3 page: FP8 through block
// quantisation). Reading taken where the page gives no detail: one fp32 scale
// per block of 128 consecutive rows of a (batch, head) plane, or one per plane
// when per_plane != 0; s = amax / 448 (amax = largest |x| in the block, s = 1
// for an all-zero block), computed in fp32, and code = E4M3(x / s) with the
// division in fp32, ties to even. The value a code stands for is
// e4m3_value(code) * s.
//   x      [planes, N, d] in dtype (bf16, f32 or f16)
//   codes  [planes, N, d] uint8 (written)
//   scales [planes, ceil(N / 128)] fp32 (written)
int oracle_quant_fp8(int dtype, const void* x, int planes, int N, int d, int per_plane, uint8_t* codes,
                     float* scales) {
    if (x == nullptr || codes == nullptr || scales == nullptr || planes < 1 || N < 1 || d < 1 ||
        dtype < IN_BF16 || dtype > IN_F16)
        return 1;
    const int nblk = (N + 127) / 128;
    std::vector<float> amax(nblk);
    for (int64_t pl = 0; pl < planes; ++pl) {
        for (int bk = 0; bk < nblk; ++bk) {
            float m = 0.f;
            for (int64_t n = bk * 128; n < std::min<int64_t>(N, (bk + 1) * 128); ++n)
                for (int t = 0; t < d; ++t)
                    m = std::max(m, static_cast<float>(std::fabs(load_elem(dtype, x, (pl * N + n) * d + t))));
            amax[bk] = m;
        }
        float plane_max = 0.f;
        for (float m : amax) plane_max = std::max(plane_max, m);
        for (int bk = 0; bk < nblk; ++bk) {
            const float m = per_plane ? plane_max : amax[bk];
            const float sc = m > 0.f ? m / 448.0f : 1.0f;
            scales[pl * nblk + bk] = sc;
            for (int64_t n = bk * 128; n < std::min<int64_t>(N, (bk + 1) * 128); ++n)
                for (int t = 0; t < d; ++t) {
                    const int64_t i = (pl * N + n) * d + t;
                    codes[i] = e4m3_code(static_cast<float>(load_elem(dtype, x, i)) / sc);
                }
        }
    }
    return 0;
}

// Values of n E4M3 codes.
int oracle_e4m3_decode(const uint8_t* codes, int64_t n, double* out) {
    if (codes == nullptr || out == nullptr || n < 0) return 1;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
    return 0;
}

// E4M3 codes of n floats (exposes the rounding to the pin tests).
int oracle_e4m3_encode(const float* x, int64_t n, uint8_t* out) {
    if (x == nullptr || out == nullptr || n < 0) return 1;
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_code(x[i]);
    return 0;
}

// Incoherent processing (FlashAttention-3 page, FP8 with "incoherent
// processing"; the page gives no detail). Reading taken: each row x of Q and
// of K is replaced by y = H (sigma o x) / sqrt(d), H the d x d Sylvester
// Hadamard matrix (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]) and sigma a
// vector of random signs shared by Q and K. H H^T = d I, so the rotation is
// orthogonal and Q K^T is unchanged, while an outlier in one coordinate is
// spread over all d of them before quantisation. Computed in fp32 as the fast
// Walsh-Hadamard transform of the Sylvester recursion (butterflies of span
// 1, 2, 4, ..., d/2: (a, b) -> (a + b, a - b)), then one multiplication by the
// fp32 value nearest 1 / sqrt(d).
//   x, y   [rows, d] fp32 (y written; may equal x)
//   signs  [d] fp32, each +1 or -1
int oracle_hadamard_rotate(const float* x, const float* signs, int64_t rows, int d, float* y) {
    if (x == nullptr || signs == nullptr || y == nullptr || rows < 0 || d < 1 || (d & (d - 1)) != 0) return 1;
    for (int t = 0; t < d; ++t)
        if (signs[t] != 1.0f && signs[t] != -1.0f) return 1;
    const float r = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    std::vector<float> w(d);
    for (int64_t i = 0; i < rows; ++i) {
        for (int t = 0; t < d; ++t) w[t] = signs[t] * x[i * d + t];
        for (int h = 1; h < d; h *= 2)
            for (int b = 0; b < d; b += 2 * h)
                for (int t = b; t < b + h; ++t) {
                    const float a = w[t], c = w[t + h];
                    w[t] = a + c;
                    w[t + h] = a - c;
                }
        for (int t = 0; t < d; ++t) y[i * d + t] = (kPlant == 11) ? w[t] : w[t] * r;  // 11: 1/sqrt(d) dropped
    }
    return 0;
}

}  // extern "C"
