/*
 * TEST INFRASTRUCTURE ONLY: plain, slow fp64 CPU oracle for the gated delta-rule recurrence.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg may load this
 * library.  It shares no source, header, table or helper with the CUDA path, and the CUDA path
 * never calls it.  Inputs are the exact values the GPU sees (bf16 or fp32 upcast to double).
 *
 * What it follows (page title, section):
 *  - Update and readout: Gated DeltaNet-2 summary (gist.science, arXiv 2605.22791),
 *    «Méthodologie», §1 «Règle Delta Portée-2»:  S_t = (I - k_t e_t^T) D_t S_{t-1} + k_t z_t^T,
 *    e_t = b_t (.) k_t, z_t = w_t (.) v_t, D_t = Diag(alpha_t);  o_t = S_t^T q_t  (the
 *    dk x dv convention of the same page; restated by the zubnet.ai news item).  A scale factor
 *    multiplies the readout (the pages use 1).
 *  - Scalar-gate reductions (alpha, b, w collapse to scalars: Gated DeltaNet; alpha = 1:
 *    DeltaNet): same page, end of §1, and the Gated DeltaNet explainer (docsaid.org),
 *    «Réunir les deux».
 *  - Chunkwise form: explainer «Rendre l'entraînement parallèle» and the GDN-2 summary §3
 *    «Entraînement Parallèle Efficace par Blocs» (decay absorbed into the erase and write
 *    factors, lower-triangular solve (I+T)^-1 giving the erase-side and write-side auxiliaries).
 *  - Short causal convolution (kernel 4, no bias), SiLU, L2 norm of q,k, swish output gate:
 *    explainer «Architecture et versions hybrides» (Figure 1 caption) and the mkdocs chapter
 *    «Gated DeltaNet», «La convolution causale» and «La porte de sortie».
 *
 * Parity pins live in tests/test_oracle_pins.py (printed worked example, reductions, exact
 * recall, edit invariant, orthogonal keys, closed forms, chunk form == sequential form, finite
 * differences for the backward, split/decode carry).  Parity unpinned: none of the functions
 * below; the L2-norm epsilon (1e-6) is a reading, the pages give none.
 *
 * Build: g++ -O2 -std=c++17 -fPIC -shared -pthread (no -ffast-math), see build() in oracle/oracle.py.
 */
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

struct Dims {
    int B, T, Hk, Hv, dk, dv;
    int a_ch, b_ch, w_ch;  // 1 (one value per token and head) or the channel count
};

// Index helpers for the token-major layouts [B,T,H,D].
inline long tok(const Dims& d, int b, int t, int h, int H, int D) {
    return ((static_cast<long>(b) * d.T + t) * H + h) * static_cast<long>(D);
}

template <class F>
void parallel_for(int n, int nthreads, F&& f) {
    if (nthreads <= 1 || n <= 1) {
        for (int i = 0; i < n; ++i) f(i);
        return;
    }
    std::atomic<int> next{0};
    std::vector<std::thread> pool;
    int nt = nthreads < n ? nthreads : n;
    for (int w = 0; w < nt; ++w)
        pool.emplace_back([&]() {
            for (int i = next.fetch_add(1); i < n; i = next.fetch_add(1)) f(i);
        });
    for (auto& th : pool) th.join();
}

// Pointers to one token's vectors for one (batch, value head).
struct Token {
    const double *q, *k, *v, *a, *bg, *wg;
};

inline Token token_at(const Dims& d, const double* q, const double* k, const double* v,
                      const double* a, const double* bg, const double* wg, const int* map,
                      int b, int t, int hv) {
    int hk = map[hv];
    Token x;
    x.q = q + tok(d, b, t, hk, d.Hk, d.dk);
    x.k = k + tok(d, b, t, hk, d.Hk, d.dk);
    x.v = v + tok(d, b, t, hv, d.Hv, d.dv);
    x.a = a + tok(d, b, t, hv, d.Hv, d.a_ch);
    x.bg = bg + tok(d, b, t, hv, d.Hv, d.b_ch);
    x.wg = wg + tok(d, b, t, hv, d.Hv, d.w_ch);
    return x;
}

// One step of the recurrence on S (dk x dv, row-major), in place:
//   decay rows by alpha, read r = Sbar^T e, write S = Sbar + k (z - r)^T, readout o = scale S^T q.
void step(const Dims& d, double* S, const Token& x, double scale, double* o,
          std::vector<double>& e, std::vector<double>& u) {
    const int dk = d.dk, dv = d.dv;
    for (int i = 0; i < dk; ++i) {
        double ai = x.a[d.a_ch == 1 ? 0 : i];
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= ai;
    }
    for (int i = 0; i < dk; ++i) e[i] = x.bg[d.b_ch == 1 ? 0 : i] * x.k[i];
    for (int j = 0; j < dv; ++j) u[j] = x.wg[d.w_ch == 1 ? 0 : j] * x.v[j];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) u[j] -= e[i] * S[i * dv + j];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] += x.k[i] * u[j];
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) o[j] += x.q[i] * S[i * dv + j];
        for (int j = 0; j < dv; ++j) o[j] *= scale;
    }
}

int check(const Dims& d, const int* map) {
    if (d.B < 0 || d.T < 0 || d.Hk <= 0 || d.Hv <= 0 || d.dk <= 0 || d.dv <= 0) return 1;
    if (!(d.a_ch == 1 || d.a_ch == d.dk)) return 1;
    if (!(d.b_ch == 1 || d.b_ch == d.dk)) return 1;
    if (!(d.w_ch == 1 || d.w_ch == d.dv)) return 1;
    for (int h = 0; h < d.Hv; ++h)
        if (map[h] < 0 || map[h] >= d.Hk) return 1;
    return 0;
}

// (b, hv) pairs to evaluate: all of them, or a caller-given subset (flattened b * Hv + hv).
std::vector<int> pair_list(const Dims& d, const int* pairs, int npairs) {
    std::vector<int> out;
    if (pairs) {
        out.assign(pairs, pairs + npairs);
    } else {
        for (int p = 0; p < d.B * d.Hv; ++p) out.push_back(p);
    }
    return out;
}

}  // namespace

extern "C" {

/* Sequential forward: o [B,T,Hv,dv] and final state hT [B,Hv,dk,dv] (hT may be NULL).
 * Returns 0, or 1 on inconsistent sizes. */
int oracle_fwd(const double* q, const double* k, const double* v, const double* alpha,
               const double* bg, const double* wg, const double* h0, const int* head_map,
               int B, int T, int Hk, int Hv, int dk, int dv, int a_ch, int b_ch, int w_ch,
               double scale, const int* pairs, int npairs, double* o, double* hT, int nthreads) {
    Dims d{B, T, Hk, Hv, dk, dv, a_ch, b_ch, w_ch};
    if (check(d, head_map)) return 1;
    std::vector<int> plist = pair_list(d, pairs, npairs);
    parallel_for(static_cast<int>(plist.size()), nthreads, [&](int idx) {
        int b = plist[idx] / Hv, hv = plist[idx] % Hv;
        std::vector<double> S(static_cast<size_t>(dk) * dv, 0.0), e(dk), u(dv);
        if (h0) std::memcpy(S.data(), h0 + (static_cast<long>(b) * Hv + hv) * dk * dv,
                            sizeof(double) * dk * dv);
        for (int t = 0; t < T; ++t) {
            Token x = token_at(d, q, k, v, alpha, bg, wg, head_map, b, t, hv);
            step(d, S.data(), x, scale, o + tok(d, b, t, hv, Hv, dv), e, u);
        }
        if (hT) std::memcpy(hT + (static_cast<long>(b) * Hv + hv) * dk * dv, S.data(),
                            sizeof(double) * dk * dv);
    });
    return 0;
}

/* Hand-written reverse mode of oracle_fwd.  Inputs as oracle_fwd plus dout [B,T,Hv,dv] and
 * dhT [B,Hv,dk,dv] (NULL = 0).  Outputs, all per value head (the caller sums dq_v/dk_v over the
 * value heads that share a key head):
 *   dq_v, dk_v [B,T,Hv,dk]; dv [B,T,Hv,dv]; dalpha, db, dw with the shapes of alpha, bg, wg;
 *   dh0 [B,Hv,dk,dv].
 * States are checkpointed every `seg` steps and recomputed inside each segment. */
int oracle_bwd(const double* q, const double* k, const double* v, const double* alpha,
               const double* bg, const double* wg, const double* h0, const int* head_map,
               int B, int T, int Hk, int Hv, int dk, int dv, int a_ch, int b_ch, int w_ch,
               double scale, const double* dout, const double* dhT, const int* pairs, int npairs,
               double* dq_v, double* dk_v, double* dv_out, double* dalpha, double* db,
               double* dw, double* dh0, int nthreads) {
    Dims d{B, T, Hk, Hv, dk, dv, a_ch, b_ch, w_ch};
    if (check(d, head_map)) return 1;
    const int seg = 64;
    std::vector<int> plist = pair_list(d, pairs, npairs);
    parallel_for(static_cast<int>(plist.size()), nthreads, [&](int idx) {
        int b = plist[idx] / Hv, hv = plist[idx] % Hv;
        const size_t n = static_cast<size_t>(dk) * dv;
        std::vector<double> e(dk), u(dv), de(dk), du(dv), Sbar(n), dSbar(n), dS(n, 0.0);
        // Checkpoints S_{0}, S_{seg}, S_{2 seg}, ...
        int nseg = (T + seg - 1) / seg;
        std::vector<double> ckpt(static_cast<size_t>(nseg + 1) * n, 0.0);
        {
            std::vector<double> S(n, 0.0);
            if (h0) std::memcpy(S.data(), h0 + (static_cast<long>(b) * Hv + hv) * n, sizeof(double) * n);
            for (int t = 0; t < T; ++t) {
                if (t % seg == 0) std::memcpy(&ckpt[(t / seg) * n], S.data(), sizeof(double) * n);
                Token x = token_at(d, q, k, v, alpha, bg, wg, head_map, b, t, hv);
                step(d, S.data(), x, scale, nullptr, e, u);
            }
        }
        if (dhT) std::memcpy(dS.data(), dhT + (static_cast<long>(b) * Hv + hv) * n, sizeof(double) * n);
        std::vector<double> states(static_cast<size_t>(seg + 1) * n);
        for (int s = nseg - 1; s >= 0; --s) {
            int t0 = s * seg, t1 = (t0 + seg < T) ? t0 + seg : T;
            // states[i] = S_{t0 + i}, i.e. the state after t0 + i tokens.
            std::memcpy(states.data(), &ckpt[s * n], sizeof(double) * n);
            for (int t = t0; t < t1; ++t) {
                std::memcpy(&states[(t - t0 + 1) * n], &states[(t - t0) * n], sizeof(double) * n);
                Token x = token_at(d, q, k, v, alpha, bg, wg, head_map, b, t, hv);
                step(d, &states[(t - t0 + 1) * n], x, scale, nullptr, e, u);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const double* Sp = &states[(t - t0) * n];      // S_{t-1} in 1-based terms
                const double* Sc = &states[(t - t0 + 1) * n];  // S_t
                Token x = token_at(d, q, k, v, alpha, bg, wg, head_map, b, t, hv);
                const double* gout = dout + tok(d, b, t, hv, Hv, dv);
                double* gq = dq_v + tok(d, b, t, hv, Hv, dk);
                double* gk = dk_v + tok(d, b, t, hv, Hv, dk);
                double* gv = dv_out + tok(d, b, t, hv, Hv, dv);
                double* ga = dalpha + tok(d, b, t, hv, Hv, a_ch);
                double* gb = db + tok(d, b, t, hv, Hv, b_ch);
                double* gw = dw + tok(d, b, t, hv, Hv, w_ch);
                // Recompute the step's intermediates.
                for (int i = 0; i < dk; ++i) {
                    double ai = x.a[a_ch == 1 ? 0 : i];
                    for (int j = 0; j < dv; ++j) Sbar[i * dv + j] = ai * Sp[i * dv + j];
                    e[i] = x.bg[b_ch == 1 ? 0 : i] * x.k[i];
                }
                for (int j = 0; j < dv; ++j) u[j] = x.wg[w_ch == 1 ? 0 : j] * x.v[j];
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) u[j] -= e[i] * Sbar[i * dv + j];
                // Readout o_t = scale * S_t^T q_t.
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += Sc[i * dv + j] * gout[j];
                    gq[i] = scale * acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) dS[i * dv + j] += scale * x.q[i] * gout[j];
                // S_t = Sbar + k u^T.
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dS[i * dv + j] * u[j];
                    gk[i] = acc;
                }
                for (int j = 0; j < dv; ++j) du[j] = 0.0;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) du[j] += dS[i * dv + j] * x.k[i];
                // u = z - Sbar^T e:  dz = du,  dSbar = dS - e du^T,  de = -Sbar du.
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        dSbar[i * dv + j] = dS[i * dv + j] - e[i] * du[j];
                        acc += Sbar[i * dv + j] * du[j];
                    }
                    de[i] = -acc;
                }
                // e = b (.) k.
                if (b_ch == 1) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += de[i] * x.k[i];
                    gb[0] = acc;
                } else {
                    for (int i = 0; i < dk; ++i) gb[i] = de[i] * x.k[i];
                }
                for (int i = 0; i < dk; ++i) gk[i] += de[i] * x.bg[b_ch == 1 ? 0 : i];
                // z = w (.) v.
                if (w_ch == 1) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += du[j] * x.v[j];
                    gw[0] = acc;
                } else {
                    for (int j = 0; j < dv; ++j) gw[j] = du[j] * x.v[j];
                }
                for (int j = 0; j < dv; ++j) gv[j] = du[j] * x.wg[w_ch == 1 ? 0 : j];
                // Sbar = Diag(alpha) S_{t-1}.
                if (a_ch == 1) {
                    double acc = 0.0;
                    for (size_t m = 0; m < n; ++m) acc += dSbar[m] * Sp[m];
                    ga[0] = acc;
                } else {
                    for (int i = 0; i < dk; ++i) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += dSbar[i * dv + j] * Sp[i * dv + j];
                        ga[i] = acc;
                    }
                }
                for (int i = 0; i < dk; ++i) {
                    double ai = x.a[a_ch == 1 ? 0 : i];
                    for (int j = 0; j < dv; ++j) dS[i * dv + j] = ai * dSbar[i * dv + j];
                }
            }
        }
        std::memcpy(dh0 + (static_cast<long>(b) * Hv + hv) * n, dS.data(), sizeof(double) * n);
    });
    return 0;
}

/* The chunkwise-parallel form written out plainly (chunk length C; the last chunk may be
 * shorter).  Per chunk, with g_r = sum_{i<=r} log alpha_i (per key channel, inclusive):
 *   A_rs = sum_c e_r[c] k_s[c] exp(g_r[c]-g_s[c])  (s < r),   T = (I + A)^-1 by substitution,
 *   W = T Ehat (Ehat_r = e_r exp(g_r)),  U = T Z,  V' = U - W S0,
 *   O = scale (Qhat S0 + P V'),  P_rs = sum_c q_r[c] k_s[c] exp(g_r[c]-g_s[c]) (s <= r),
 *   S_end = Diag(exp(g_last)) S0 + sum_s (k_s exp(g_last - g_s)) V'_s^T.
 * Same arguments as oracle_fwd plus C. */
int oracle_chunk_fwd(const double* q, const double* k, const double* v, const double* alpha,
                     const double* bg, const double* wg, const double* h0, const int* head_map,
                     int B, int T, int Hk, int Hv, int dk, int dv, int a_ch, int b_ch, int w_ch,
                     double scale, int C, double* o, double* hT, int nthreads) {
    Dims d{B, T, Hk, Hv, dk, dv, a_ch, b_ch, w_ch};
    if (check(d, head_map) || C <= 0) return 1;
    parallel_for(B * Hv, nthreads, [&](int p) {
        int b = p / Hv, hv = p % Hv;
        const size_t n = static_cast<size_t>(dk) * dv;
        std::vector<double> S(n, 0.0);
        if (h0) std::memcpy(S.data(), h0 + (static_cast<long>(b) * Hv + hv) * n, sizeof(double) * n);
        std::vector<double> g(static_cast<size_t>(C) * dk), E(C * dk), Z(C * dv), A(C * C), P(C * C),
            Tm(C * C), W(C * dk), U(C * dv), Vp(C * dv);
        for (int c0 = 0; c0 < T; c0 += C) {
            int L = (c0 + C <= T) ? C : T - c0;
            std::vector<Token> x(L);
            for (int r = 0; r < L; ++r) x[r] = token_at(d, q, k, v, alpha, bg, wg, head_map, b, c0 + r, hv);
            // Cumulative log decay, gated erase/write vectors.
            for (int r = 0; r < L; ++r)
                for (int c = 0; c < dk; ++c) {
                    double la = std::log(x[r].a[a_ch == 1 ? 0 : c]);
                    g[r * dk + c] = (r ? g[(r - 1) * dk + c] : 0.0) + la;
                    E[r * dk + c] = x[r].bg[b_ch == 1 ? 0 : c] * x[r].k[c];
                }
            for (int r = 0; r < L; ++r)
                for (int j = 0; j < dv; ++j) Z[r * dv + j] = x[r].wg[w_ch == 1 ? 0 : j] * x[r].v[j];
            // Key affinities with the decay ratio between positions.
            for (int r = 0; r < L; ++r)
                for (int s = 0; s < L; ++s) {
                    double a_rs = 0.0, p_rs = 0.0;
                    if (s <= r)
                        for (int c = 0; c < dk; ++c) {
                            double ratio = std::exp(g[r * dk + c] - g[s * dk + c]);
                            a_rs += E[r * dk + c] * x[s].k[c] * ratio;
                            p_rs += x[r].q[c] * x[s].k[c] * ratio;
                        }
                    A[r * C + s] = (s < r) ? a_rs : 0.0;
                    P[r * C + s] = (s <= r) ? p_rs : 0.0;
                }
            // T = (I + A)^-1: solve (I + A) X = I column by column, forward substitution.
            for (int col = 0; col < L; ++col)
                for (int r = 0; r < L; ++r) {
                    double acc = (r == col) ? 1.0 : 0.0;
                    for (int s = 0; s < r; ++s) acc -= A[r * C + s] * Tm[s * C + col];
                    Tm[r * C + col] = acc;
                }
            // W = T Ehat, U = T Z.
            for (int r = 0; r < L; ++r) {
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int s = 0; s < L; ++s) acc += Tm[r * C + s] * E[s * dk + c] * std::exp(g[s * dk + c]);
                    W[r * dk + c] = acc;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int s = 0; s < L; ++s) acc += Tm[r * C + s] * Z[s * dv + j];
                    U[r * dv + j] = acc;
                }
            }
            // V' = U - W S0.
            for (int r = 0; r < L; ++r)
                for (int j = 0; j < dv; ++j) {
                    double acc = U[r * dv + j];
                    for (int c = 0; c < dk; ++c) acc -= W[r * dk + c] * S[c * dv + j];
                    Vp[r * dv + j] = acc;
                }
            // O = scale (Qhat S0 + P V').
            for (int r = 0; r < L; ++r) {
                double* orow = o + tok(d, b, c0 + r, hv, Hv, dv);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += x[r].q[c] * std::exp(g[r * dk + c]) * S[c * dv + j];
                    for (int s = 0; s <= r; ++s) acc += P[r * C + s] * Vp[s * dv + j];
                    orow[j] = scale * acc;
                }
            }
            // S_end = Diag(exp(g_last)) S0 + Kbar^T V'.
            for (int c = 0; c < dk; ++c) {
                double glast = g[(L - 1) * dk + c];
                for (int j = 0; j < dv; ++j) {
                    double acc = std::exp(glast) * S[c * dv + j];
                    for (int s = 0; s < L; ++s) acc += x[s].k[c] * std::exp(glast - g[s * dk + c]) * Vp[s * dv + j];
                    S[c * dv + j] = acc;
                }
            }
        }
        if (hT) std::memcpy(hT + (static_cast<long>(b) * Hv + hv) * n, S.data(), sizeof(double) * n);
    });
    return 0;
}

/* Causal depthwise convolution, kernel 4, no bias, followed by SiLU.
 * x [B,T,Cch]; w [Cch,4] with w[ch][3] weighting the current token and w[ch][0] the token three
 * steps back; hist [B,Cch,3] holds the three inputs before t = 0 (oldest first; NULL = zeros).
 * y [B,T,Cch] = silu(conv); hist_out [B,Cch,3] (may be NULL) receives the last three inputs. */
int oracle_conv_silu(const double* x, const double* w, const double* hist, int B, int T, int Cch,
                     double* y, double* hist_out) {
    if (B < 0 || T < 0 || Cch <= 0) return 1;
    for (int b = 0; b < B; ++b)
        for (int ch = 0; ch < Cch; ++ch) {
            auto in = [&](int t) -> double {
                if (t >= 0) return x[(static_cast<long>(b) * T + t) * Cch + ch];
                if (!hist || t < -3) return 0.0;
                return hist[(static_cast<long>(b) * Cch + ch) * 3 + (3 + t)];
            };
            for (int t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int i = 0; i < 4; ++i) acc += w[ch * 4 + i] * in(t - 3 + i);
                y[(static_cast<long>(b) * T + t) * Cch + ch] = acc / (1.0 + std::exp(-acc));
            }
            if (hist_out)
                for (int i = 0; i < 3; ++i) hist_out[(static_cast<long>(b) * Cch + ch) * 3 + i] = in(T - 3 + i);
        }
    return 0;
}

/* Rows of length d divided by sqrt(sum of squares + eps), in place. */
void oracle_l2norm_rows(double* x, long rows, int d, double eps) {
    for (long r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += x[r * d + c] * x[r * d + c];
        double inv = 1.0 / std::sqrt(ss + eps);
        for (int c = 0; c < d; ++c) x[r * d + c] *= inv;
    }
}

/* Swish output gate: y = o * z * sigmoid(z), elementwise over n values. */
void oracle_swish_gate(const double* o, const double* z, long n, double* y) {
    for (long m = 0; m < n; ++m) y[m] = o[m] * z[m] / (1.0 + std::exp(-z[m]));
}

}  // extern "C"
