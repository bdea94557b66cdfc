/*
 * Engram conditional-memory forward pass: plain float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference legs of bench.py may load this code.  It shares no
 * code, header, table or helper with the CUDA library and never calls it.
 *
 * Sources (cited by page and section):
 *   "formulas page"  = the Engram formula document at kwkr.cn/news/37585
 *   "explainer page" = the Engram paper walk-through at yaoyuxiang.cn/news/830577
 *   (the extracted pages print no titles; they are named by their subject)
 *
 * Every step is written out as its definition, in the pages' order, with no
 * blocking or reordering:
 *   a1 compressed ids       explainer §2.2 1), §4.1
 *   a2 time shift / pad     formulas §4.2, worked example §4.3
 *   a3 n-gram hash          formulas §1.2 steps 1-2, §1.3; explainer §4.2
 *   a4 row gather / concat  explainer §2.2 1), §4.3; formulas §5.2
 *   a5 projections          formulas §2.2 steps 1 and 3; explainer §2.2 4), §4.3
 *   a6 RMSNorm + dot / sqrt(d)  formulas §2.2 step 1
 *   a7 gate                 formulas §2.2 step 2 (magnitude floored at gate_eps,
 *                           square root, sign restored, logistic)
 *   a8 gate (x) V           formulas §2.2 step 3
 *   a9 short conv + residual formulas §3.2; explainer §2.2 3)
 *
 * Readings where the pages are silent or garbled (each also listed in the
 * design notes): multipliers are one vector per layer shared by all orders and
 * heads, m_0 multiplies the current token; hash arithmetic follows NumPy int64
 * (wrapping products, floor modulo); RMSNorm(x) = x / sqrt(mean(x^2) + eps) * w
 * with eps = rms_eps; d in sqrt(d) is the hidden size; sign(0) = 0; the conv
 * is depthwise, causal, bias-free, no activation, PyTorch Conv1d tap order:
 * y[t] = sum_i w[c,i] * u[t - (K-1-i)*dil], zero before the sequence start.
 *
 * Element storage codes for tensors given in their native type:
 *   0 = float32, 1 = bfloat16 (upper 16 bits of a float32).  Values are
 *   widened to double exactly.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* Exact widening of one stored element to double. */
static double load_elem(const void* base, int64_t i, int code) {
    if (code == ORACLE_F32) {
        return (double)((const float*)base)[i];
    } else {
        uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
}

void oracle_widen(const void* src, int64_t n, int code, double* dst) {
    for (int64_t i = 0; i < n; ++i) dst[i] = load_elem(src, i, code);
}

/* ---- a1: compressed id = lookup[raw id] (explainer §2.2 1), §4.1) ---- */
void oracle_compress_ids(const int64_t* raw, int64_t n, const int64_t* lookup,
                         int64_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = lookup[raw[i]];
}

/* ---- a2: shift_k(x)[b, t] (formulas §4.2, §4.3 example) ----
 * The sequence is left-padded with k copies of pad_id and cut back to T, so
 * position t sees x[t-k]; positions before the start read pad_id, or, when a
 * history of the previous hist_len ids is given (most recent last), that
 * history. */
int64_t oracle_shifted_token(const int64_t* x, int T, int b, int t, int k,
                             const int64_t* hist, int hist_len, int64_t pad_id) {
    int s = t - k;
    if (s >= 0) return x[(int64_t)b * T + s];
    if (hist != NULL && -s <= hist_len) return hist[(int64_t)b * hist_len + hist_len + s];
    return pad_id;
}

void oracle_shift(const int64_t* x, int B, int T, int k, const int64_t* hist,
                  int hist_len, int64_t pad_id, int64_t* out) {
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            out[(int64_t)b * T + t] = oracle_shifted_token(x, T, b, t, k, hist, hist_len, pad_id);
}

/* NumPy int64 remainder: result has the sign of the (positive) modulus. */
static int64_t floor_mod(int64_t a, int64_t p) {
    int64_t r = a % p;
    if (r < 0) r += p;
    return r;
}

/* ---- a3: hash_{n,j} = ((t0*m0) xor (t1*m1) xor ... xor (t_{n-1}*m_{n-1})) mod p_{n,j}
 * (formulas §1.2 steps 1-2, §1.3; explainer §4.2).
 * tokens[k] = shift_k(x): t_k of the n-gram ending at position t is x[t-k].
 * idx layout: [B, T, n_orders * J], head index o*J + j. */
void oracle_hash(const int64_t* x, int B, int T, const int64_t* hist, int hist_len,
                 int n_orders, const int32_t* orders, int J, const int64_t* mult,
                 const int64_t* primes, int64_t pad_id, int64_t* idx) {
    int nh = n_orders * J;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < T; ++t) {
            for (int o = 0; o < n_orders; ++o) {
                int n = orders[o];
                /* int64 products wrap like NumPy's (computed in uint64). */
                uint64_t mix = (uint64_t)oracle_shifted_token(x, T, b, t, 0, hist, hist_len, pad_id)
                             * (uint64_t)mult[0];
                for (int k = 1; k < n; ++k) {
                    uint64_t tk = (uint64_t)oracle_shifted_token(x, T, b, t, k, hist, hist_len, pad_id);
                    mix = mix ^ (tk * (uint64_t)mult[k]);
                }
                for (int j = 0; j < J; ++j) {
                    int64_t p = primes[o * J + j];
                    idx[((int64_t)b * T + t) * nh + o * J + j] = floor_mod((int64_t)mix, p);
                }
            }
        }
    }
}

/* ---- a4: e = concat over (order asc, head asc) of Table_{n,j}[idx] ----
 * (explainer §2.2 1): all retrieved rows are concatenated into e_t; §4.3).
 * The per-head tables are stacked; head h starts at row row_offsets[h].
 * Output e: [M, nh * Dh] in the storage type of the table (a byte copy). */
void oracle_gather(const void* table, int elem_bytes, int Dh, const int64_t* row_offsets,
                   const int64_t* idx, int64_t M, int nh, void* e) {
    size_t row_bytes = (size_t)Dh * (size_t)elem_bytes;
    for (int64_t m = 0; m < M; ++m)
        for (int h = 0; h < nh; ++h) {
            int64_t row = row_offsets[h] + idx[m * nh + h];
            memcpy((char*)e + ((size_t)m * nh + h) * row_bytes,
                   (const char*)table + (size_t)row * row_bytes, row_bytes);
        }
}

/* ---- a5: y = x W^T for a torch-style Linear without bias, W [N, E] ----
 * (formulas §2.2 steps 1 and 3: keys and values are bias-free linear maps of e).
 * Accumulated naively in float64. */
static void linear_row(const double* x, int E, const void* W, int wcode, int64_t row0,
                       int N, double* y) {
    for (int n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int k = 0; k < E; ++k) acc += x[k] * load_elem(W, (row0 + n) * (int64_t)E + k, wcode);
        y[n] = acc;
    }
}

/* ---- a6: RMSNorm(x; w) = x / sqrt(mean(x^2) + eps) * w (formulas §2.2 step 1:
 * one learnable norm per branch for the key, another for the query). */
static void rmsnorm(const double* x, int H, const double* w, double eps, double* out) {
    double ss = 0.0;
    for (int c = 0; c < H; ++c) ss += x[c] * x[c];
    double inv = 1.0 / sqrt(ss / (double)H + eps);
    for (int c = 0; c < H; ++c) out[c] = x[c] * inv * w[c];
}

/* ---- a7: gate = sigmoid(sign(s) * sqrt(max(|s|, gate_eps))) ----
 * (formulas §2.2 step 2: the magnitude of s is floored at 1e-6 before the
 * square root, the sign of s is put back, then the logistic function).
 * sign(0) = 0, so s = 0 gives exactly 0.5. */
double oracle_gate_value(double s, double gate_eps) {
    double a = fabs(s);
    if (a < gate_eps) a = gate_eps;
    double sg = (s > 0.0) ? 1.0 : ((s < 0.0) ? -1.0 : 0.0);
    double z = sqrt(a) * sg;
    return 1.0 / (1.0 + exp(-z));
}

/* ---- a5-a7 for one token ----
 * e: [E] row of the token (double); hidden: [hc, H] starting at row
 * hidden_row0 of a [*, H] array (storage code hcode); weights in storage code
 * wcode: w_value [H, E], w_key [hc, H, E], norm_key / norm_query [hc, H].
 * Outputs V [H], s [hc], g [hc].  work: scratch of 6*H doubles. */
void oracle_token_gate(const double* e, int E, int H, int hc,
                       const void* w_value, const void* w_key,
                       const void* norm_key, const void* norm_query, int wcode,
                       const void* hidden, int64_t hidden_row0, int hcode,
                       double rms_eps, double gate_eps,
                       double* V, double* s, double* g, double* work) {
    double* K = work;
    double* Q = work + H;
    double* wk = work + 2 * H;
    double* wq = work + 3 * H;
    double* Kn = work + 4 * H;
    double* Qn = work + 5 * H;
    linear_row(e, E, w_value, wcode, 0, H, V);                       /* V = value projection of e */
    for (int h = 0; h < hc; ++h) {
        linear_row(e, E, w_key, wcode, (int64_t)h * H, H, K);        /* K_h = key projection h of e */
        for (int c = 0; c < H; ++c)                                   /* Q_h = branch h of the hidden state */
            Q[c] = load_elem(hidden, (hidden_row0 + h) * (int64_t)H + c, hcode);
        for (int c = 0; c < H; ++c) wk[c] = load_elem(norm_key, (int64_t)h * H + c, wcode);
        for (int c = 0; c < H; ++c) wq[c] = load_elem(norm_query, (int64_t)h * H + c, wcode);
        rmsnorm(K, H, wk, rms_eps, Kn);                               /* key norm of branch h */
        rmsnorm(Q, H, wq, rms_eps, Qn);                               /* query norm of branch h */
        double dot = 0.0;
        for (int c = 0; c < H; ++c) dot += Kn[c] * Qn[c];             /* sum over channels */
        s[h] = dot / sqrt((double)H);                                 /* divided by sqrt(H) */
        g[h] = oracle_gate_value(s[h], gate_eps);
    }
}

/* Stand-alone RMSNorm for the tests. */
void oracle_rmsnorm(const double* x, int H, const double* w, double eps, double* out) {
    rmsnorm(x, H, w, eps, out);
}

/* ---- a9: short conv + residual for one output position ----
 * Y[h, c] = U(t)[h, c] + sum_{i<K} conv_w[h*H + c, i] * U(t - (K-1-i)*dil)[h, c]
 * with U(t')[h, c] = g(t')[h] * V(t')[c] (a8, formulas §2.2 step 3) and U = 0
 * for positions before the sequence start (formulas §3.2: the gated value plus its
 * short convolution; explainer §2.2 3): depthwise causal conv, kernel 4,
 * dilation = max order).
 * Vtap: [K, H] value rows of positions t-(K-1)*dil ... t (tap i = row i);
 * gtap: [K, hc]; valid: [K] 0/1 (0 = before the start). Output Y [hc, H]. */
void oracle_conv_point(const double* Vtap, const double* gtap, const int32_t* valid,
                       int K, int H, int hc, const void* conv_w, int wcode, double* Y) {
    for (int h = 0; h < hc; ++h)
        for (int c = 0; c < H; ++c) {
            double u_t = valid[K - 1] ? gtap[(K - 1) * hc + h] * Vtap[(int64_t)(K - 1) * H + c] : 0.0;
            double conv = 0.0;
            for (int i = 0; i < K; ++i) {
                double u = valid[i] ? gtap[i * hc + h] * Vtap[(int64_t)i * H + c] : 0.0;
                conv += load_elem(conv_w, ((int64_t)h * H + c) * K + i, wcode) * u;
            }
            Y[(int64_t)h * H + c] = u_t + conv;
        }
}

/* Stand-alone short conv + residual over a whole [B, T, C] tensor U (double),
 * optionally continuing from prev = the last (K-1)*dil positions before this
 * chunk ([B, (K-1)*dil, C], oldest first).  conv_w [C, K]. */
void oracle_short_conv(const double* U, int B, int T, int C, const double* conv_w,
                       int K, int dil, const double* prev, double* Y) {
    int R = (K - 1) * dil;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int i = 0; i < K; ++i) {
                    int tp = t - (K - 1 - i) * dil;
                    double u;
                    if (tp >= 0) u = U[((int64_t)b * T + tp) * C + c];
                    else if (prev != NULL && R + tp >= 0) u = prev[((int64_t)b * R + R + tp) * C + c];
                    else u = 0.0;
                    acc += conv_w[(int64_t)c * K + i] * u;
                }
                Y[((int64_t)b * T + t) * C + c] = U[((int64_t)b * T + t) * C + c] + acc;
            }
}

/* ---- whole forward over [B, T] with every input on the host ----
 * x: compressed ids [B, T]; table [total_rows, Dh], weights, hidden [B, T, hc, H]
 * and conv_w [hc*H, K] in storage code `code`.  Outputs (double):
 * Y [B, T, hc, H]; optional idx [B, T, nh], V [B, T, H], s and g [B, T, hc].
 * Runs the steps above one after another; the per-token projections are
 * independent and spread over OpenMP threads. */
void oracle_forward(const int64_t* x, int B, int T, int n_orders, const int32_t* orders,
                    int J, int Dh, const int64_t* mult, const int64_t* primes,
                    const int64_t* row_offsets, int64_t pad_id,
                    const void* table, const void* w_value, const void* w_key,
                    const void* norm_key, const void* norm_query, const void* conv_w,
                    const void* hidden, int code, int H, int hc, int K, int dil,
                    double rms_eps, double gate_eps,
                    double* Y, int64_t* idx_out, double* V_out, double* s_out, double* g_out,
                    double* work /* M*(nh + H + 2*hc) + nthreads*(E + 6*H) doubles */,
                    int nthreads) {
    int nh = n_orders * J;
    int E = nh * Dh;
    int64_t M = (int64_t)B * T;
    /* a2 + a3 */
    int64_t* idx = (int64_t*)work;                      /* M*nh int64 */
    double* V = work + M * nh;                          /* M*H */
    double* s = V + M * H;                              /* M*hc */
    double* g = s + M * hc;                             /* M*hc */
    double* thr = g + M * hc;                           /* nthreads * (E + 6H) */
    oracle_hash(x, B, T, NULL, 0, n_orders, orders, J, mult, primes, pad_id, idx);
    /* a4 - a7 per token */
    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double* e = thr + (int64_t)tid * (E + 6 * H);
        double* wk = e + E;
        for (int h = 0; h < nh; ++h) {
            int64_t row = row_offsets[h] + idx[m * nh + h];
            for (int c = 0; c < Dh; ++c) e[h * Dh + c] = load_elem(table, row * Dh + c, code);
        }
        oracle_token_gate(e, E, H, hc, w_value, w_key, norm_key, norm_query, code,
                          hidden, m * hc, code, rms_eps, gate_eps,
                          V + m * H, s + m * hc, g + m * hc, wk);
    }
    /* a8 + a9 */
    #pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        int b = (int)(m / T), t = (int)(m % T);
        for (int h = 0; h < hc; ++h)
            for (int c = 0; c < H; ++c) {
                double u_t = g[m * hc + h] * V[m * H + c];
                double conv = 0.0;
                for (int i = 0; i < K; ++i) {
                    int tp = t - (K - 1 - i) * dil;
                    double u = 0.0;
                    if (tp >= 0) {
                        int64_t mp = (int64_t)b * T + tp;
                        u = g[mp * hc + h] * V[mp * H + c];
                    }
                    conv += load_elem(conv_w, ((int64_t)h * H + c) * K + i, code) * u;
                }
                Y[(m * hc + h) * (int64_t)H + c] = u_t + conv;
            }
    }
    if (idx_out) memcpy(idx_out, idx, sizeof(int64_t) * (size_t)(M * nh));
    if (V_out) memcpy(V_out, V, sizeof(double) * (size_t)(M * H));
    if (s_out) memcpy(s_out, s, sizeof(double) * (size_t)(M * hc));
    if (g_out) memcpy(g_out, g, sizeof(double) * (size_t)(M * hc));
}

/* a5-a7 for n independent tokens (rows of e and of hidden), spread over
 * OpenMP threads; each token is exactly oracle_token_gate above. */
void oracle_tokens_gate(const double* e, int64_t n, int E, int H, int hc,
                        const void* w_value, const void* w_key,
                        const void* norm_key, const void* norm_query, int wcode,
                        const void* hidden, int hcode, double rms_eps, double gate_eps,
                        double* V, double* s, double* g, double* work, int nthreads) {
    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        oracle_token_gate(e + i * (int64_t)E, E, H, hc, w_value, w_key, norm_key, norm_query,
                          wcode, hidden, i * hc, hcode, rms_eps, gate_eps,
                          V + i * (int64_t)H, s + i * hc, g + i * hc, work + (int64_t)tid * 6 * H);
    }
}
