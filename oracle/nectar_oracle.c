/*
 * CPU oracle for the Nectar hot path -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may
 * load this library.  It shares no code with the CUDA path.
 *
 * Source of every formula: "Nectar: Neural Estimation of Cached-Token
 * Attention via Regression" (Monteiro, Klein, Ablin, Cuturi), as given in the
 * reading notes of arXiv 2605.09778v2.  Section / equation numbers below are
 * the paper's.
 *
 * Everything is computed in IEEE double from bf16 inputs (passed as raw
 * uint16 bit patterns and widened exactly) or from double inputs.  There is
 * no blocking, fusion or reordering beyond what each definition states; the
 * loops are written in the order the formulas are read.  OpenMP only runs
 * independent (head, query) items side by side.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* q . k  for a d-vector, both bf16. */
static double dot_bf16(const uint16_t *q, const uint16_t *k, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += bf16_to_double(q[c]) * bf16_to_double(k[c]);
    return s;
}

/*
 * Exact cached-token attention, §2.1 Eq. (3.1):
 *   s_j = scale * q . k_j,  alpha = log sum_j e^{s_j},
 *   A   = sum_j e^{s_j} v_j / sum_j e^{s_j}.
 * Evaluated in two passes with the maximum M = max_j s_j factored out
 * (e^{s_j} = e^M e^{s_j - M}; the factor cancels in A and adds M to alpha),
 * which is the same quantity without overflow.
 *
 * K, V : [heads][n][d] bf16     Q : [heads][rows][d] bf16
 * alpha: [heads][rows]          A : [heads][rows][d]      (double)
 */
void oracle_cache_attn(int64_t heads, int64_t n, int64_t rows, int d,
                       const uint16_t *K, const uint16_t *V, const uint16_t *Q,
                       double scale, double *alpha, double *A) {
    int64_t items = heads * rows;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        int64_t hd = it / rows;
        const uint16_t *q = Q + it * d;
        const uint16_t *Kh = K + hd * n * d;
        const uint16_t *Vh = V + hd * n * d;
        double *out = A + it * d;
        double M = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double s = scale * dot_bf16(q, Kh + j * d, d);
            if (s > M) M = s;
        }
        double l = 0.0;
        for (int c = 0; c < d; ++c) out[c] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double w = exp(scale * dot_bf16(q, Kh + j * d, d) - M);
            l += w;
            for (int c = 0; c < d; ++c) out[c] += w * bf16_to_double(Vh[j * d + c]);
        }
        for (int c = 0; c < d; ++c) out[c] /= l;
        alpha[it] = (n > 0) ? M + log(l) : -INFINITY;
    }
}

static double silu(double x) { return x / (1.0 + exp(-x)); }

/*
 * Nectar MLP with input re-injection, §2.4 Eq. (3.6):
 *   h_0     = SiLU(U_0 q + b_0)
 *   h_{k+1} = SiLU(V_{k+1} q + U_{k+1} h_k + b_{k+1})
 *   y       = W_out h_{D-1} + c        (linear readout, no activation)
 * The readout reading (one linear map from the last hidden layer, no
 * re-injection) is the plainest one the notes' statement "score outputs 1
 * dim, target outputs d dims" supports.
 *
 * params: [units][P] double, per unit in this plain order (row-major):
 *   U_0 [H][d], b_0 [H],
 *   for k = 1..depth-1:  V_k [H][d], U_k [H][H], b_k [H],
 *   W_out [dout][H], c [dout]
 * X : [units][rows][d] bf16 (the queries),   Y : [units][rows][dout] double
 */
int64_t oracle_mlp_param_count(int d, int depth, int H, int dout) {
    int64_t P = (int64_t)H * d + H;
    for (int k = 1; k < depth; ++k) P += (int64_t)H * d + (int64_t)H * H + H;
    return P + (int64_t)dout * H + dout;
}

void oracle_mlp(int64_t units, int64_t rows, int d, int depth, int H, int dout,
                const double *params, const uint16_t *X, double *Y) {
    int64_t P = oracle_mlp_param_count(d, depth, H, dout);
    int64_t items = units * rows;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        int64_t u = it / rows;
        const double *p = params + u * P;
        const uint16_t *xq = X + it * d;
        double *q = (double *)malloc(sizeof(double) * d);
        double *h = (double *)malloc(sizeof(double) * H);
        double *hn = (double *)malloc(sizeof(double) * H);
        for (int c = 0; c < d; ++c) q[c] = bf16_to_double(xq[c]);
        /* layer 0 */
        const double *U0 = p;
        const double *b0 = U0 + (int64_t)H * d;
        for (int i = 0; i < H; ++i) {
            double z = b0[i];
            for (int c = 0; c < d; ++c) z += U0[(int64_t)i * d + c] * q[c];
            h[i] = silu(z);
        }
        p = b0 + H;
        /* layers 1..depth-1, each re-injecting q */
        for (int k = 1; k < depth; ++k) {
            const double *Vk = p;
            const double *Uk = Vk + (int64_t)H * d;
            const double *bk = Uk + (int64_t)H * H;
            for (int i = 0; i < H; ++i) {
                double z = bk[i];
                for (int c = 0; c < d; ++c) z += Vk[(int64_t)i * d + c] * q[c];
                for (int j = 0; j < H; ++j) z += Uk[(int64_t)i * H + j] * h[j];
                hn[i] = silu(z);
            }
            memcpy(h, hn, sizeof(double) * H);
            p = bk + H;
        }
        /* linear readout */
        const double *W = p;
        const double *cb = W + (int64_t)dout * H;
        double *y = Y + it * dout;
        for (int o = 0; o < dout; ++o) {
            double z = cb[o];
            for (int j = 0; j < H; ++j) z += W[(int64_t)o * H + j] * h[j];
            y[o] = z;
        }
        free(q); free(h); free(hn);
    }
}

/*
 * A chain of `nl` hidden layers of the Eq. (3.6) recursion with its own
 * width per layer, then the linear readout -- the shape of a score or a
 * target net when a backbone is shared (§2.4, App. A.3: depths
 * (D_b, D_s, D_t)).  Layer 0 sees only q, layer k >= 1 sees q and layer
 * k - 1 (width W[k-1]):
 *   h_0 = SiLU(U_0 q + b_0),  h_k = SiLU(V_k q + U_k h_{k-1} + b_k).
 * params per unit, in order:
 *   U_0 [W0][d], b_0 [W0],
 *   for k = 1..nl-1:  V_k [Wk][d], U_k [Wk][W(k-1)], b_k [Wk],
 *   W_out [dout][W(nl-1)], c [dout]
 */
int64_t oracle_chain_param_count(int d, int nl, const int *W, int dout) {
    int64_t P = (int64_t)W[0] * d + W[0];
    for (int k = 1; k < nl; ++k) P += (int64_t)W[k] * d + (int64_t)W[k] * W[k - 1] + W[k];
    return P + (int64_t)dout * W[nl - 1] + dout;
}

void oracle_chain(int64_t units, int64_t rows, int d, int nl, const int *W, int dout,
                  const double *params, const uint16_t *X, double *Y) {
    int64_t P = oracle_chain_param_count(d, nl, W, dout);
    int Wmax = 0;
    for (int k = 0; k < nl; ++k) Wmax = W[k] > Wmax ? W[k] : Wmax;
    int64_t items = units * rows;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        int64_t u = it / rows;
        const double *p = params + u * P;
        const uint16_t *xq = X + it * d;
        double *q = (double *)malloc(sizeof(double) * d);
        double *h = (double *)malloc(sizeof(double) * Wmax);
        double *hn = (double *)malloc(sizeof(double) * Wmax);
        for (int c = 0; c < d; ++c) q[c] = bf16_to_double(xq[c]);
        const double *U0 = p;
        const double *b0 = U0 + (int64_t)W[0] * d;
        for (int i = 0; i < W[0]; ++i) {
            double z = b0[i];
            for (int c = 0; c < d; ++c) z += U0[(int64_t)i * d + c] * q[c];
            h[i] = silu(z);
        }
        p = b0 + W[0];
        for (int k = 1; k < nl; ++k) {
            const int Hk = W[k], Hp = W[k - 1];
            const double *Vk = p;
            const double *Uk = Vk + (int64_t)Hk * d;
            const double *bk = Uk + (int64_t)Hk * Hp;
            for (int i = 0; i < Hk; ++i) {
                double z = bk[i];
                for (int c = 0; c < d; ++c) z += Vk[(int64_t)i * d + c] * q[c];
                for (int j = 0; j < Hp; ++j) z += Uk[(int64_t)i * Hp + j] * h[j];
                hn[i] = silu(z);
            }
            memcpy(h, hn, sizeof(double) * Hk);
            p = bk + Hk;
        }
        const int Hl = W[nl - 1];
        const double *Wo = p;
        const double *cb = Wo + (int64_t)dout * Hl;
        double *y = Y + it * dout;
        for (int o = 0; o < dout; ++o) {
            double z = cb[o];
            for (int j = 0; j < Hl; ++j) z += Wo[(int64_t)o * Hl + j] * h[j];
            y[o] = z;
        }
        free(q); free(h); free(hn);
    }
}

/*
 * Visible local set of a query token (§2.2): local tokens i of its sequence
 * with i <= t (t = its local position, the token itself included) and
 * i < local_len.  Returns the count of visible tokens.
 */
static int64_t visible_count(int32_t pos, int32_t len) {
    int64_t v = (int64_t)pos + 1;
    if (v > len) v = len;
    if (v < 0) v = 0;
    return v;
}

/*
 * Merge with exact causal local attention, §2.2 Eqs. (3.4)-(3.5):
 *   out = (e^{a} A + N_local) / (e^{a} + Z_local),
 *   Z_local = sum_{i vis} e^{s_i},  N_local = sum_{i vis} e^{s_i} v_i,
 *   s_i = scale * q . k_i.
 * The document term acts as one extra logit a with value A.  Written with
 * the common maximum m = max(a, max_i s_i) divided out of numerator and
 * denominator.  With no visible local token the output is A.
 *
 * a : [heads][rows]  Adoc : [heads][rows][d]   (double)
 * Q : [heads][rows][d] bf16, row r = g*nq + i is token i of query head g
 * q_seq, q_pos : [nq]     local_len : [B]
 * Kloc, Vloc : [heads][B][T][d] bf16           out : [heads][rows][d]
 */
void oracle_merge_local(int64_t heads, int64_t rows, int64_t nq, int d,
                        const double *a, const double *Adoc, const uint16_t *Q,
                        const int32_t *q_seq, const int32_t *q_pos,
                        const uint16_t *Kloc, const uint16_t *Vloc,
                        int64_t B, int64_t T, const int32_t *local_len,
                        double scale, double *out) {
    int64_t items = heads * rows;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t it = 0; it < items; ++it) {
        int64_t hd = it / rows, r = it % rows, i = r % nq;
        int64_t b = q_seq[i];
        int64_t nv = visible_count(q_pos[i], local_len[b]);
        const uint16_t *q = Q + it * d;
        const uint16_t *Kb = Kloc + ((hd * B + b) * T) * d;
        const uint16_t *Vb = Vloc + ((hd * B + b) * T) * d;
        double m = a[it];
        for (int64_t j = 0; j < nv; ++j) {
            double s = scale * dot_bf16(q, Kb + j * d, d);
            if (s > m) m = s;
        }
        double wdoc = exp(a[it] - m);
        double den = wdoc;
        double *o = out + it * d;
        for (int c = 0; c < d; ++c) o[c] = wdoc * Adoc[it * d + c];
        for (int64_t j = 0; j < nv; ++j) {
            double w = exp(scale * dot_bf16(q, Kb + j * d, d) - m);
            den += w;
            for (int c = 0; c < d; ++c) o[c] += w * bf16_to_double(Vb[j * d + c]);
        }
        for (int c = 0; c < d; ++c) o[c] /= den;
    }
}

/*
 * Full attention over [document ; visible local tokens] as ONE softmax, the
 * left-hand side of §2.2 Eq. (3.4).  Used only to check that the merge of
 * the exact (alpha, A) reproduces it.
 */
void oracle_full_attention(int64_t heads, int64_t n, int64_t rows, int64_t nq, int d,
                           const uint16_t *K, const uint16_t *V, const uint16_t *Q,
                           const int32_t *q_seq, const int32_t *q_pos,
                           const uint16_t *Kloc, const uint16_t *Vloc,
                           int64_t B, int64_t T, const int32_t *local_len,
                           double scale, double *out) {
    int64_t items = heads * rows;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        int64_t hd = it / rows, r = it % rows, i = r % nq;
        int64_t b = q_seq[i];
        int64_t nv = visible_count(q_pos[i], local_len[b]);
        const uint16_t *q = Q + it * d;
        const uint16_t *Kh = K + hd * n * d, *Vh = V + hd * n * d;
        const uint16_t *Kb = Kloc + ((hd * B + b) * T) * d;
        const uint16_t *Vb = Vloc + ((hd * B + b) * T) * d;
        int64_t tot = n + nv;
        double m = -INFINITY;
        for (int64_t j = 0; j < tot; ++j) {
            const uint16_t *k = (j < n) ? Kh + j * d : Kb + (j - n) * d;
            double s = scale * dot_bf16(q, k, d);
            if (s > m) m = s;
        }
        double den = 0.0;
        double *o = out + it * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int64_t j = 0; j < tot; ++j) {
            const uint16_t *k = (j < n) ? Kh + j * d : Kb + (j - n) * d;
            const uint16_t *v = (j < n) ? Vh + j * d : Vb + (j - n) * d;
            double w = exp(scale * dot_bf16(q, k, d) - m);
            den += w;
            for (int c = 0; c < d; ++c) o[c] += w * bf16_to_double(v[c]);
        }
        for (int c = 0; c < d; ++c) o[c] /= den;
    }
}

/* Threads OpenMP will use (for reporting the CPU baseline's core count). */
/*
 * Fitting metrics of a module against the exact targets, per (l, h)
 * (notes §4 "score / target MSE"; App. C.4, Eq. (C.1)):
 *   score_mse  = mean_q (a(q) - alpha(q))^2
 *   target_mse = mean_q (1/d) sum_c (A_theta(q)_c - A(q)_c)^2
 *   rte        = mean_q log( ||A_theta(q) - A(q)||^2 / ||q - A(q)||^2 )
 * (the RTE of Eq. (C.1) is the sum of rte over (l, h)).  q is the bf16 query
 * row as stored; the others are double.
 *
 * alpha, a: [heads][rows]   A, At: [heads][rows][d]   Q: [heads][rows][d] bf16
 * out: [heads][3] = {score_mse, target_mse, rte}
 */
void oracle_fit_metrics(int64_t heads, int64_t rows, int d, const double *alpha, const double *A,
                        const double *a, const double *At, const uint16_t *Q, double *out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t hd = 0; hd < heads; ++hd) {
        double s_sum = 0.0, t_sum = 0.0, r_sum = 0.0;
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t it = hd * rows + r;
            const double ds = a[it] - alpha[it];
            s_sum += ds * ds;
            double num = 0.0, den = 0.0;
            for (int c = 0; c < d; ++c) {
                const double e = At[it * d + c] - A[it * d + c];
                const double b = bf16_to_double(Q[it * d + c]) - A[it * d + c];
                num += e * e;
                den += b * b;
            }
            t_sum += num / d;
            r_sum += log(num / den);
        }
        out[hd * 3 + 0] = rows > 0 ? s_sum / rows : 0.0;
        out[hd * 3 + 1] = rows > 0 ? t_sum / rows : 0.0;
        out[hd * 3 + 2] = rows > 0 ? r_sum / rows : 0.0;
    }
}

#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_threads(int t) { omp_set_num_threads(t); }
#else
int oracle_num_threads(void) { return 1; }
void oracle_set_threads(int t) { (void)t; }
#endif
