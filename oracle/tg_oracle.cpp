// TokenGate gated-prefill oracle: a plain, slow CPU implementation in fp64.
//
// THIS IS TEST INFRASTRUCTURE.  Only the test suite, the package smoke check
// and the benchmark's CPU-baseline leg may load it.  It shares no code, no
// header and no constant with the CUDA library: it is written directly from
// the method's description so that the GPU path can be checked against it.
//
// What it computes (citations are to the pages describing TokenGate):
//   score   RMSNorm of the post-attention residual at the gate layer, then a
//           small MLP giving one scalar per prunable token.
//           (TokenGate AI summary, "Key Contributions" 1; TokenGate explained
//           blog, "how the gate works")
//   select  keep the K highest-scoring prunable tokens plus every
//           non-prunable token.  (AI summary, "Key Contributions" 1 and
//           "Methodology in Plain English"; README copy, "How it works")
//   compact upper layers see the kept tokens only, in their original order.
//           (AI summary, "Key Contributions" 1: no KV entries for pruned tokens)
//   attend  token-gated attention: causal GQA attention over the kept tokens
//           with a per-key, per-head additive gate bias and a per-query
//           temperature.  (AI summary, "Key Contributions" 2 and 3;
//           "Methodology in Plain English")
//
// The pages describe the bias and the temperature only in prose.  The exact
// formulas used here are the library's stated definitions:
//   b[h,j]  = softplus(g_h) * logsigmoid(s_j)   (0 for non-prunable keys)
//   tau_q,h = 1 + c_h * ln(pos_q / rank_q)
//   logit   = (q.k * sm_scale + b[h,j]) / tau_q,h
// The temperature divides the whole logit (the ordinary meaning of a softmax
// temperature).  `tau_on_qk_only` switches to the other reading, in which only
// q.k is divided; it is off everywhere the library is checked.
//
// The gate's first layer absorbs the RMSNorm weight: Wg[j][i] = bf16(gamma_i *
// W1[i][j]) (round to nearest even), and the normalisation factor r_t
// multiplies after the contraction.  This is RMSNorm followed by Linear with
// the product gamma*W1 held in bf16.  `oracle_score_unfolded` keeps gamma
// separate in fp64 and reports how far the fold moves the scores.
//
// Parity pins: every function here is checked on the CPU against closed
// forms, brute force, invariants and library routines (see tests/).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

double bf16_to_double(uint16_t b) {
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

// float -> bfloat16, round to nearest with ties to even (NaN -> quiet NaN).
uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, sizeof u);
    if (std::isnan(f)) return 0x7FC0;
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return static_cast<uint16_t>(u >> 16);
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

double softplus(double x) { return std::max(x, 0.0) + std::log1p(std::exp(-std::fabs(x))); }

double logsigmoid(double x) { return std::min(x, 0.0) - std::log1p(std::exp(-std::fabs(x))); }

int64_t span_len(const int32_t* span, int b) { return static_cast<int64_t>(span[2 * b + 1]) - span[2 * b]; }

int64_t kept_prunable(int64_t p, int32_t k) { return (k < 0 || k > p) ? p : static_cast<int64_t>(k); }

}  // namespace

extern "C" {

int oracle_abi_version() { return 4; }

// Thread count of the parallel loops (one row per iteration; no reduction
// crosses threads, so results do not depend on it).
void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads() {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

// Wg [I, D] (row j = gate unit j) = bf16(gamma_i * W1[i][j]).  W1 is [D, I].
// The product of two bf16 values is exact in fp32, so the only rounding is
// the final one to bf16.
void oracle_gate_fold(const uint16_t* gamma, const uint16_t* W1, int D, int I, uint16_t* Wg) {
    for (int j = 0; j < I; ++j)
        for (int i = 0; i < D; ++i) {
            float p = static_cast<float>(bf16_to_double(gamma[i])) *
                      static_cast<float>(bf16_to_double(W1[static_cast<int64_t>(i) * I + j]));
            Wg[static_cast<int64_t>(j) * D + i] = float_to_bf16_rne(p);
        }
}

// Gate score of every prunable token (TokenGate AI summary, "Key
// Contributions" 1):
//   r_t = 1 / sqrt(mean_i x_ti^2 + eps)
//   z_j = r_t * sum_i Wg[j][i] x_ti + b1_j
//   s_t = sum_j w2_j * SiLU(z_j) + b2
// Entries of non-prunable tokens are left untouched.
void oracle_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B, int D,
                  const uint16_t* Wg, const float* b1, const float* w2, float b2, int I, double eps,
                  double* scores) {
    std::vector<double> wg(static_cast<size_t>(I) * D);
    for (size_t e = 0; e < wg.size(); ++e) wg[e] = bf16_to_double(Wg[e]);
    for (int b = 0; b < B; ++b) {
        const int64_t t0 = cu_seqlens[b] + static_cast<int64_t>(span[2 * b]);
        const int64_t t1 = cu_seqlens[b] + static_cast<int64_t>(span[2 * b + 1]);
#pragma omp parallel for schedule(static)
        for (int64_t t = t0; t < t1; ++t) {
            std::vector<double> x(D);
            double ss = 0.0;
            for (int i = 0; i < D; ++i) {
                x[i] = bf16_to_double(hidden[t * D + i]);
                ss += x[i] * x[i];
            }
            const double r = 1.0 / std::sqrt(ss / D + eps);
            double s = static_cast<double>(b2);
            for (int j = 0; j < I; ++j) {
                const double* wj = &wg[static_cast<size_t>(j) * D];
                double acc = 0.0;
                for (int i = 0; i < D; ++i) acc += wj[i] * x[i];
                const double z = r * acc + static_cast<double>(b1[j]);
                s += static_cast<double>(w2[j]) * silu(z);
            }
            scores[t] = s;
        }
    }
}

// Same gate with gamma kept apart from W1 (u = gamma * x * r in fp64, then the
// Linear).  Reported beside oracle_score to show the effect of the bf16 fold.
void oracle_score_unfolded(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B,
                           int D, const uint16_t* gamma, const uint16_t* W1, const float* b1, const float* w2,
                           float b2, int I, double eps, double* scores) {
    for (int b = 0; b < B; ++b) {
        const int64_t t0 = cu_seqlens[b] + static_cast<int64_t>(span[2 * b]);
        const int64_t t1 = cu_seqlens[b] + static_cast<int64_t>(span[2 * b + 1]);
#pragma omp parallel for schedule(static)
        for (int64_t t = t0; t < t1; ++t) {
            std::vector<double> u(D);
            double ss = 0.0;
            for (int i = 0; i < D; ++i) {
                const double x = bf16_to_double(hidden[t * D + i]);
                ss += x * x;
                u[i] = x;
            }
            const double r = 1.0 / std::sqrt(ss / D + eps);
            for (int i = 0; i < D; ++i) u[i] = u[i] * r * bf16_to_double(gamma[i]);
            double s = static_cast<double>(b2);
            for (int j = 0; j < I; ++j) {
                double z = static_cast<double>(b1[j]);
                for (int i = 0; i < D; ++i) z += bf16_to_double(W1[static_cast<int64_t>(i) * I + j]) * u[i];
                s += static_cast<double>(w2[j]) * silu(z);
            }
            scores[t] = s;
        }
    }
}

// Kept count per sequence: every non-prunable token plus min(K_b, |P_b|)
// prunable ones (K_b < 0 keeps all).  Writes cu_kept[B+1]; returns the total.
int64_t oracle_kept_count(const int32_t* cu_seqlens, const int32_t* span, const int32_t* k, int B,
                          int32_t* cu_kept) {
    int64_t tot = 0;
    cu_kept[0] = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t n = static_cast<int64_t>(cu_seqlens[b + 1]) - cu_seqlens[b];
        const int64_t p = span_len(span, b);
        tot += (n - p) + kept_prunable(p, k[b]);
        cu_kept[b + 1] = static_cast<int32_t>(tot);
    }
    return tot;
}

// Top-K over each sequence's prunable span (AI summary, "Key Contributions"
// 1).  Order: higher score first, then lower index.  -0 and +0 compare equal
// (fp32 comparison); NaN ranks below every number.  keep[t] = 1 for every
// non-prunable token.  Implemented as a full stable sort.
void oracle_select_topk(const float* scores, const int32_t* cu_seqlens, const int32_t* span, const int32_t* k,
                        int B, uint8_t* keep) {
    for (int b = 0; b < B; ++b) {
        const int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
        const int64_t p0 = s0 + span[2 * b], p1 = s0 + span[2 * b + 1];
        for (int64_t t = s0; t < s1; ++t) keep[t] = (t < p0 || t >= p1) ? 1 : 0;
        std::vector<int64_t> idx(static_cast<size_t>(p1 - p0));
        std::iota(idx.begin(), idx.end(), p0);
        std::stable_sort(idx.begin(), idx.end(), [&](int64_t a, int64_t c) {
            const float sa = scores[a], sc = scores[c];
            const bool na = std::isnan(sa), nc = std::isnan(sc);
            if (na || nc) return !na && nc;
            return sa > sc;
        });
        const int64_t kk = kept_prunable(p1 - p0, k[b]);
        for (int64_t r = 0; r < kk; ++r) keep[idx[static_cast<size_t>(r)]] = 1;
    }
}

// Stable compaction of the kept tokens (AI summary, "Key Contributions" 1).
// For kept token t of sequence b, in original order:
//   pos  = t - start_b + 1           (1-indexed original position)
//   rank = number of kept tokens of b up to and including t
//   gls  = logsigmoid(s_t) for a prunable token, 0 otherwise
//   src  = t                         (global row of the source token)
// hidden_kept receives the row bytes unchanged.  cu_kept[B+1] is written.
void oracle_compact(const uint16_t* hidden, const float* scores, const uint8_t* keep, const int32_t* cu_seqlens,
                    const int32_t* span, int B, int D, int32_t* cu_kept, uint16_t* hidden_kept, int32_t* pos,
                    int32_t* rank, double* gls, int32_t* src) {
    int64_t m = 0;
    cu_kept[0] = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
        const int64_t p0 = s0 + span[2 * b], p1 = s0 + span[2 * b + 1];
        int64_t r = 0;
        for (int64_t t = s0; t < s1; ++t) {
            if (!keep[t]) continue;
            ++r;
            if (hidden_kept)
                std::memcpy(hidden_kept + m * D, hidden + t * D, sizeof(uint16_t) * static_cast<size_t>(D));
            pos[m] = static_cast<int32_t>(t - s0 + 1);
            rank[m] = static_cast<int32_t>(r);
            gls[m] = (t >= p0 && t < p1) ? logsigmoid(static_cast<double>(scores[t])) : 0.0;
            if (src) src[m] = static_cast<int32_t>(t);
            ++m;
        }
        cu_kept[b + 1] = static_cast<int32_t>(m);
    }
}

// Token-gated causal GQA attention over the kept tokens (AI summary, "Key
// Contributions" 2 and 3).  Row-major layouts: q [M, Hq, d], k/v [M, Hkv, d]
// (bf16 bits); pos, rank [M]; gls [M] fp32; g, c [Hq].
// Query i of sequence b attends to kept keys j of b with rank_j <= rank_i.
// Query head h reads KV head h / (Hq / Hkv).
// `rows` (n_rows entries) selects which kept rows to compute; rows == nullptr
// computes all M rows.  out is [n_rows, Hq, d]; lse (natural log of the
// softmax denominator, max included) is [n_rows, Hq], may be null.
// Several gate modules (AI summary, "Future Directions": each gate selects
// from what the lower ones kept and contributes to the token-gated attention
// above it): gls is [n_gates, M] and g is [n_gates, Hq], and each gate adds
// its own term softplus(g_i,h) * gls_i,j to the logit.  n_gates = 1 is the
// single gate of the method.
void oracle_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                            int B, int Hq, int Hkv, int d, const int32_t* pos, const int32_t* rank,
                            const float* gls, const float* g, const float* c, double sm_scale,
                            const int64_t* rows, int64_t n_rows, double* out, double* lse, int tau_on_qk_only,
                            int n_gates) {
    const int64_t M = cu_kept[B];
    if (!rows) n_rows = M;
    const int group = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t ri = 0; ri < n_rows; ++ri) {
        const int64_t i = rows ? rows[ri] : ri;
        int b = 0;
        while (cu_kept[b + 1] <= i) ++b;
        const int64_t j0 = cu_kept[b];
        std::vector<double> logit(static_cast<size_t>(i - j0 + 1));
        std::vector<double> acc(d);
        for (int h = 0; h < Hq; ++h) {
            const int hk = h / group;
            const double tau = 1.0 + static_cast<double>(c[h]) *
                                         std::log(static_cast<double>(pos[i]) / static_cast<double>(rank[i]));
            double mx = -INFINITY;
            for (int64_t j = j0; j <= i; ++j) {
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += bf16_to_double(q[(i * Hq + h) * d + e]) * bf16_to_double(k[(j * Hkv + hk) * d + e]);
                double bias = 0.0;
                for (int gi = 0; gi < n_gates; ++gi)
                    bias += softplus(static_cast<double>(g[gi * Hq + h])) * static_cast<double>(gls[gi * M + j]);
                const double l = tau_on_qk_only ? (dot * sm_scale / tau + bias) : ((dot * sm_scale + bias) / tau);
                logit[static_cast<size_t>(j - j0)] = l;
                mx = std::max(mx, l);
            }
            double den = 0.0;
            std::fill(acc.begin(), acc.end(), 0.0);
            for (int64_t j = j0; j <= i; ++j) {
                const double p = std::exp(logit[static_cast<size_t>(j - j0)] - mx);
                den += p;
                for (int e = 0; e < d; ++e) acc[e] += p * bf16_to_double(v[(j * Hkv + hk) * d + e]);
            }
            for (int e = 0; e < d; ++e) out[(ri * Hq + h) * d + e] = acc[e] / den;
            if (lse) lse[ri * Hq + h] = mx + std::log(den);
        }
    }
}

// The same attention written over the full, uncompacted sequence: every
// token keeps its row, pruned keys are excluded (bias -inf) and pruned query
// rows are defined as 0.  This is the training-time form (full budget plus a
// masked sampled budget; AI summary, "Key Contributions" 4) and must equal the
// compacted form row for row.  q [T, Hq, d], k/v [T, Hkv, d]; keep [T];
// scores [T] fp32; out [T, Hq, d].
void oracle_masked_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                   const int32_t* cu_seqlens, const int32_t* span, int B, int Hq, int Hkv, int d,
                                   const uint8_t* keep, const float* scores, const float* g, const float* c,
                                   double sm_scale, const int64_t* rows, int64_t n_rows, double* out) {
    const int64_t T = cu_seqlens[B];
    if (!rows) n_rows = T;
    const int group = Hq / Hkv;
    // rank of every kept token (1-indexed within its sequence)
    std::vector<int64_t> rk(static_cast<size_t>(T), 0);
    for (int b = 0; b < B; ++b) {
        int64_t r = 0;
        for (int64_t t = cu_seqlens[b]; t < cu_seqlens[b + 1]; ++t)
            if (keep[t]) rk[static_cast<size_t>(t)] = ++r;
    }
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t ri = 0; ri < n_rows; ++ri) {
        const int64_t i = rows ? rows[ri] : ri;
        int b = 0;
        while (cu_seqlens[b + 1] <= i) ++b;
        const int64_t s0 = cu_seqlens[b];
        const int64_t p0 = s0 + span[2 * b], p1 = s0 + span[2 * b + 1];
        if (!keep[i]) {
            for (int64_t e = 0; e < static_cast<int64_t>(Hq) * d; ++e) out[ri * Hq * d + e] = 0.0;
            continue;
        }
        std::vector<double> logit(static_cast<size_t>(i - s0 + 1));
        std::vector<double> acc(d);
        for (int h = 0; h < Hq; ++h) {
            const int hk = h / group;
            const double gain = softplus(static_cast<double>(g[h]));
            const double tau = 1.0 + static_cast<double>(c[h]) *
                                         std::log(static_cast<double>(i - s0 + 1) / static_cast<double>(rk[i]));
            double mx = -INFINITY;
            for (int64_t j = s0; j <= i; ++j) {
                double l = -INFINITY;
                if (keep[j]) {
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e)
                        dot += bf16_to_double(q[(i * Hq + h) * d + e]) *
                               bf16_to_double(k[(j * Hkv + hk) * d + e]);
                    const double bias =
                        (j >= p0 && j < p1) ? gain * logsigmoid(static_cast<double>(scores[j])) : 0.0;
                    l = (dot * sm_scale + bias) / tau;
                }
                logit[static_cast<size_t>(j - s0)] = l;
                mx = std::max(mx, l);
            }
            double den = 0.0;
            std::fill(acc.begin(), acc.end(), 0.0);
            for (int64_t j = s0; j <= i; ++j) {
                const double l = logit[static_cast<size_t>(j - s0)];
                if (l == -INFINITY) continue;
                const double p = std::exp(l - mx);
                den += p;
                for (int e = 0; e < d; ++e) acc[e] += p * bf16_to_double(v[(j * Hkv + hk) * d + e]);
            }
            for (int e = 0; e < d; ++e) out[(ri * Hq + h) * d + e] = acc[e] / den;
        }
    }
}

// Backward of the token-gated attention (the gradient path that top-K alone
// lacks: AI summary, "Key Contributions" 2 -- the bias carries the task loss's
// gradient to the scoring network -- and 3 -- the gain and temperature are
// learned).  One gate.  Given dL/d out, every derivative follows the forward
// definitions by the chain rule, per (query i, head h, causal key j), for n_gates gate
// modules (gate i with logsigmoids gls_i and gains g_i; one gate is n_gates = 1):
//   l_ij   = (sm * q_i.k_j + sum_i beta_ih * gls_ij) / tau_ih,  beta_ih = softplus(g_ih)
//   P_ij   = softmax_j(l_ij),  out_i = sum_j P_ij v_j
//   dP_ij  = dout_i . v_j,  D_i = sum_j P_ij dP_ij,  dl_ij = P_ij (dP_ij - D_i)
//   dq_i  += sm dl_ij / tau * k_j,   dk_j += sm dl_ij / tau * q_i
//   dv_j  += P_ij dout_i,            dgls_ij += beta_ih dl_ij / tau
//   dbeta_ih += dl_ij gls_ij / tau,  dtau_ih = -sum_j dl_ij l_ij / tau
//   dg_ih = dbeta_ih * sigmoid(g_ih),   dc_h = sum_i dtau_ih ln(pos_i / rank_i)
// dout is [M, Hq, d] fp64; dq [M, Hq, d], dk/dv [M, Hkv, d], dgls [n_gates, M], dg
// [n_gates, Hq] and dc [Hq] are fp64 outputs; gls is [n_gates, M], g [n_gates, Hq].
// Heads run in parallel, each into its own partial sums, added in head order (results do
// not depend on the threads).
void oracle_gated_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                     int B, int Hq, int Hkv, int d, const int32_t* pos, const int32_t* rank,
                                     const float* gls, const float* g, const float* c, double sm_scale,
                                     const double* dout, double* dq, double* dk, double* dv, double* dgls, double* dg,
                                     double* dc, int n_gates) {
    const int64_t M = cu_kept[B];
    const int group = Hq / Hkv;
    const int G = n_gates;
    const size_t kv = static_cast<size_t>(M) * Hkv * d;
    std::vector<double> dk_h(static_cast<size_t>(Hq) * kv, 0.0), dv_h(static_cast<size_t>(Hq) * kv, 0.0);
    std::vector<double> dgls_h(static_cast<size_t>(Hq) * G * M, 0.0);
    std::fill(dq, dq + static_cast<size_t>(M) * Hq * d, 0.0);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < Hq; ++h) {
        const int hk = h / group;
        std::vector<double> beta(G), dbeta(G, 0.0);
        for (int gi = 0; gi < G; ++gi) beta[gi] = softplus(static_cast<double>(g[gi * Hq + h]));
        double dcs = 0.0;
        double* dkp = dk_h.data() + static_cast<size_t>(h) * kv;
        double* dvp = dv_h.data() + static_cast<size_t>(h) * kv;
        double* dglp = dgls_h.data() + static_cast<size_t>(h) * G * M;
        std::vector<double> logit, p, dp;
        for (int b = 0; b < B; ++b) {
            for (int64_t i = cu_kept[b]; i < cu_kept[b + 1]; ++i) {
                const int64_t j0 = cu_kept[b];
                const size_t n = static_cast<size_t>(i - j0 + 1);
                logit.assign(n, 0.0);
                p.assign(n, 0.0);
                dp.assign(n, 0.0);
                const double lr = std::log(static_cast<double>(pos[i]) / static_cast<double>(rank[i]));
                const double tau = 1.0 + static_cast<double>(c[h]) * lr;
                const double* go = dout + (i * Hq + h) * d;
                double mx = -INFINITY;
                for (int64_t j = j0; j <= i; ++j) {
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e)
                        dot += bf16_to_double(q[(i * Hq + h) * d + e]) * bf16_to_double(k[(j * Hkv + hk) * d + e]);
                    double bias = 0.0;
                    for (int gi = 0; gi < G; ++gi) bias += beta[gi] * static_cast<double>(gls[gi * M + j]);
                    const double l = (dot * sm_scale + bias) / tau;
                    logit[static_cast<size_t>(j - j0)] = l;
                    mx = std::max(mx, l);
                }
                double den = 0.0;
                for (size_t t = 0; t < n; ++t) {
                    p[t] = std::exp(logit[t] - mx);
                    den += p[t];
                }
                double D = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    const size_t t = static_cast<size_t>(j - j0);
                    p[t] /= den;
                    double s = 0.0;
                    for (int e = 0; e < d; ++e) s += go[e] * bf16_to_double(v[(j * Hkv + hk) * d + e]);
                    dp[t] = s;
                    D += p[t] * s;
                }
                double dtau = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    const size_t t = static_cast<size_t>(j - j0);
                    const double dl = p[t] * (dp[t] - D);
                    const double Gq = dl / tau;
                    for (int e = 0; e < d; ++e) {
                        dq[(i * Hq + h) * d + e] += sm_scale * Gq * bf16_to_double(k[(j * Hkv + hk) * d + e]);
                        dkp[(j * Hkv + hk) * d + e] += sm_scale * Gq * bf16_to_double(q[(i * Hq + h) * d + e]);
                        dvp[(j * Hkv + hk) * d + e] += p[t] * go[e];
                    }
                    for (int gi = 0; gi < G; ++gi) {
                        dglp[gi * M + j] += beta[gi] * Gq;
                        dbeta[gi] += Gq * static_cast<double>(gls[gi * M + j]);
                    }
                    if (dl != 0.0) dtau -= dl * logit[t] / tau;
                }
                dcs += dtau * lr;
            }
        }
        for (int gi = 0; gi < G; ++gi)
            dg[gi * Hq + h] = dbeta[gi] / (1.0 + std::exp(-static_cast<double>(g[gi * Hq + h])));
        dc[h] = dcs;
    }
    std::fill(dk, dk + kv, 0.0);
    std::fill(dv, dv + kv, 0.0);
    std::fill(dgls, dgls + static_cast<size_t>(G) * M, 0.0);
    for (int h = 0; h < Hq; ++h) {
        for (size_t e = 0; e < kv; ++e) {
            dk[e] += dk_h[static_cast<size_t>(h) * kv + e];
            dv[e] += dv_h[static_cast<size_t>(h) * kv + e];
        }
        for (size_t e = 0; e < static_cast<size_t>(G) * M; ++e) dgls[e] += dgls_h[static_cast<size_t>(h) * G * M + e];
    }
}

}  // extern "C"
