/*
 * uno_oracle.c — plain, slow, fp64 CPU statement of what the Uno draft-and-verify hot
 * path computes.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA path is checked
 * against. Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * load it. It shares no code, header, table or helper with the CUDA library, and the
 * product path never calls it.
 *
 * Sources (page, section):
 *   [LU-how]    LoopUno project page, "How it works": one LoRA switched on only for noise
 *               positions; a block is drafted in one forward, the unmodified model
 *               verifies it and the longest correct prefix is kept; the first position is
 *               always the exact AR token.
 *   [LU-train]  LoopUno project page, "Training is self-distillation": the loss is the
 *               total-variation distance between the frozen model's and the student's
 *               next-token distributions on response tokens; acceptance probability
 *               under lossless verification is exactly 1 - TV.
 *   [LU-recipe] LoopUno project page, "Setup / Recipe": gated LoRA r=128, alpha=2048, all
 *               seven projections, noise rows only.
 *   [MC-intro]  uno-qwen3-8B model card, introduction: the adapter is applied only on
 *               draft-noise rows; seed, prefill, verification and AR rows use the frozen
 *               base weights.
 *   [MC-proto]  uno-qwen3-8B model card, "Evaluation protocol" table: temperature 1.0,
 *               top-p 0.95, top-k 50, block 16.
 *
 * Readings where the pages are silent (each restated where it is used):
 *   - Linear layout: W0 [d_out, d_in], A [r, d_in], B [d_out, r]; no bias.
 *   - Warping order: temperature, then top-k, then softmax, then top-p, then renormalise.
 *   - Top-k keeps exactly k tokens, ties at the k-th value to the lower token id.
 *   - Top-p keeps the shortest prefix of the (probability desc, id asc) order whose
 *     cumulative mass is >= top_p; the crossing token is kept; at least one token.
 *   - Inverse-CDF sampling walks token ids in ascending order and returns the first id
 *     whose cumulative (unnormalised) weight exceeds u times the total: strict ">".
 *   - Accept draft d iff u * q(d) < p(d) (strict).
 *   - Residual at the first rejection j: normalise(max(0, p_j - q_j)); if it has no mass,
 *     sample from p_j.
 *   - Position 0 is always emitted (x_0 ~ p_0); the drafter's row 0 is not used.
 *   - Count n = 1 + (number of leading accepted drafts); the correction token is returned
 *     separately and is -1 when every draft was accepted.
 *   - TV loss: T = 1, no filtering; mean over the masked (response) tokens; gradient
 *     w.r.t. the student logits with sign(0) = 0; the teacher is constant.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------------------
 * Gated LoRA linear  [LU-how], [LU-recipe], [MC-intro]
 *
 *   t[m, j] = sum_k x[m, k] * a[j, k]                       (LoRA down-projection)
 *   y[m, o] = sum_k x[m, k] * w0[o, k]  +  scale * g[m] * sum_j t[m, j] * b[o, j]
 *
 * Frozen base on every row; the adapter term is switched by the per-row gate g (0 on
 * seed / verify / AR rows, 1 on draft-noise rows). gate == NULL means all zeros.
 * ------------------------------------------------------------------------------------ */
int oracle_gated_lora(const double* x, const double* w0, const double* a, const double* b,
                      const double* gate, double scale, int64_t M, int64_t d_in, int64_t d_out,
                      int64_t rank, double* y)
{
    if (M < 0 || d_in < 0 || d_out < 0 || rank < 0) return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        const double* xm = x + m * d_in;
        double* t = (double*)malloc((size_t)(rank > 0 ? rank : 1) * sizeof(double));
        for (int64_t j = 0; j < rank; ++j) {
            double s = 0.0;
            for (int64_t k = 0; k < d_in; ++k) s += xm[k] * a[j * d_in + k];
            t[j] = s;
        }
        double gm = gate ? gate[m] : 0.0;
        for (int64_t o = 0; o < d_out; ++o) {
            double base = 0.0;
            for (int64_t k = 0; k < d_in; ++k) base += xm[k] * w0[o * d_in + k];
            double lora = 0.0;
            for (int64_t j = 0; j < rank; ++j) lora += t[j] * b[o * rank + j];
            y[m * d_out + o] = base + scale * gm * lora;
        }
        free(t);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Row warping  [MC-proto]
 * ------------------------------------------------------------------------------------ */
typedef struct {
    double key;   /* value ordered descending */
    int64_t id;   /* ties: ascending id */
} ranked_t;

static int cmp_desc_then_id(const void* pa, const void* pb)
{
    const ranked_t* a = (const ranked_t*)pa;
    const ranked_t* b = (const ranked_t*)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->id < b->id) ? -1 : (a->id > b->id);
}

/*
 * Warp one row of logits into an unnormalised weight vector.
 *   1. z = logit / T
 *   2. top_k > 0 and top_k < V: keep the top_k largest z; ties go to the lower id
 *   3. w = exp(z - max_kept z) on kept tokens, 0 elsewhere; p = w / sum(w)
 *   4. top_p < 1: order kept tokens by (p desc, id asc); keep the shortest prefix with
 *      cumulative p >= top_p (the crossing token included); drop the rest (w = 0)
 * Returns Z = sum of the surviving w in ascending-id order, so that w / Z is the warped
 * distribution. *topp_margin = distance of the top-p crossing from top_p
 * (min(cum - top_p, top_p - cum_before)), +inf when top-p is off or cuts nothing.
 * *n_keep = number of surviving tokens.
 */
double oracle_warp_row(const double* logit, int64_t V, double T, int64_t top_k, double top_p,
                       double* w, double* topp_margin, int64_t* n_keep)
{
    ranked_t* r = (ranked_t*)malloc((size_t)V * sizeof(ranked_t));
    unsigned char* keep = (unsigned char*)malloc((size_t)V);
    for (int64_t v = 0; v < V; ++v) {
        r[v].key = logit[v] / T;
        r[v].id = v;
        keep[v] = 1;
        w[v] = 0.0;
    }
    /* 2. top-k: a full sort by (z desc, id asc); keep the first k */
    if (top_k > 0 && top_k < V) {
        qsort(r, (size_t)V, sizeof(ranked_t), cmp_desc_then_id);
        for (int64_t j = top_k; j < V; ++j) keep[r[j].id] = 0;
    }
    /* 3. softmax over the kept tokens */
    double zmax = -INFINITY;
    for (int64_t v = 0; v < V; ++v)
        if (keep[v] && logit[v] / T > zmax) zmax = logit[v] / T;
    double S = 0.0;
    for (int64_t v = 0; v < V; ++v) {
        if (keep[v]) {
            w[v] = exp(logit[v] / T - zmax);
            S += w[v];
        }
    }
    /* 4. top-p on the normalised kept distribution */
    double margin = INFINITY;
    if (top_p < 1.0) {
        int64_t nk = 0;
        for (int64_t v = 0; v < V; ++v)
            if (keep[v]) { r[nk].key = w[v] / S; r[nk].id = v; ++nk; }
        qsort(r, (size_t)nk, sizeof(ranked_t), cmp_desc_then_id);
        double cum = 0.0;
        int64_t cut = nk; /* number kept */
        for (int64_t j = 0; j < nk; ++j) {
            double before = cum;
            cum += r[j].key;
            if (cum >= top_p) {
                cut = j + 1;
                margin = fmin(cum - top_p, top_p - before);
                break;
            }
        }
        for (int64_t j = cut; j < nk; ++j) {
            keep[r[j].id] = 0;
            w[r[j].id] = 0.0;
        }
    }
    double Z = 0.0;
    int64_t count = 0;
    for (int64_t v = 0; v < V; ++v) {
        if (keep[v]) { Z += w[v]; ++count; }
    }
    if (topp_margin) *topp_margin = margin;
    if (n_keep) *n_keep = count;
    free(r);
    free(keep);
    return Z;
}

/*
 * Inverse-CDF draw: the smallest id t (ascending) with sum_{s<=t} w_s > u * Z.
 * *margin = distance of u from the chosen token's CDF interval ends, in probability
 * units. If rounding leaves no crossing, the largest id with w > 0 is returned with
 * margin 0.
 */
int64_t oracle_inv_cdf(const double* w, int64_t V, double Z, double u, double* margin)
{
    double target = u * Z;
    double cum = 0.0;
    int64_t last = -1;
    for (int64_t t = 0; t < V; ++t) {
        if (w[t] <= 0.0) continue;
        double before = cum;
        cum += w[t];
        last = t;
        if (cum > target) {
            if (margin) *margin = fmin(target - before, cum - target) / Z;
            return t;
        }
    }
    if (margin) *margin = 0.0;
    return last;
}

/* ------------------------------------------------------------------------------------
 * Lossless block verify  [LU-how], [LU-train], [MC-proto]
 *
 * Inputs (row-major): P, Q logits [B, K, V] (verifier, drafter); u [B, K, 3] uniforms
 * (sample, accept, resample); drafts [B, K] (NULL: d_i drawn from Q_i with u[b,i,0]);
 * pos0 [B] (NULL, or an entry < 0: x_0 drawn from P_0 with u[b,0,0]).
 * For each sequence b:
 *   x_0 = pos0[b] if given and >= 0, else invCDF(P_0, u[b,0,0])   (always emitted)
 *   for i = 1..K-1: d_i = drafts[b,i] or invCDF(Q_i, u[b,i,0])
 *                   accept iff u[b,i,1] * Q_i(d_i) < P_i(d_i); stop at the first reject j
 *   out_tokens = [x_0, d_1, ..., d_{n-1}, -1, ...], out_count = n (= j, or K if none)
 *   out_next   = invCDF(normalise(max(0, P_j - Q_j)), u[b,j,2]) at a rejection, else -1
 * Per position (for every i, reached or not): out_p_tok[b,i] = P_i(tok_i),
 * out_q_tok[b,i] = Q_i(tok_i) with tok_0 = x_0 and tok_i = d_i (out_q_tok[b,0] = 0: the
 * drafter's row 0 is not used); out_tv[b,i] = TV(P_i, Q_i) for i >= 1, 0 at i = 0.
 * margins [B, K, 5] (nullable): per position
 *   [0] sampling margin of x_0 / d_i   (inf if the token was supplied)
 *   [1] acceptance margin |u1 - P(d)/Q(d)|  (i >= 1; inf when Q(d) = 0 or i = 0)
 *   [2] residual sampling margin       (only at the rejected position; else inf)
 *   [3] top-p margin of row P_i, [4] top-p margin of row Q_i (inf at i = 0)
 * ------------------------------------------------------------------------------------ */
int oracle_block_verify(const double* P, const double* Q, int64_t B, int64_t K, int64_t V,
                        double T, int64_t top_k, double top_p,
                        const int32_t* drafts, const int32_t* pos0, const double* u,
                        int32_t* out_tokens, int32_t* out_count, int32_t* out_next,
                        double* out_p_tok, double* out_q_tok, double* out_tv, double* margins)
{
    if (B < 0 || K < 1 || V < 1 || !(T > 0.0)) return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < B; ++b) {
        double* wp = (double*)malloc((size_t)V * sizeof(double));
        double* wq = (double*)malloc((size_t)V * sizeof(double));
        double* res = (double*)malloc((size_t)V * sizeof(double));
        int32_t* tok = (int32_t*)malloc((size_t)K * sizeof(int32_t));
        unsigned char* acc = (unsigned char*)malloc((size_t)K);
        int64_t first_reject = -1;
        double mg[5];

        for (int64_t i = 0; i < K; ++i) {
            const double* prow = P + (b * K + i) * V;
            const double* qrow = Q + (b * K + i) * V;
            const double* ui = u + (b * K + i) * 3;
            for (int c = 0; c < 5; ++c) mg[c] = INFINITY;
            double Zp = oracle_warp_row(prow, V, T, top_k, top_p, wp, &mg[3], NULL);
            if (i == 0) {
                int64_t x0;
                if (pos0 && pos0[b] >= 0) x0 = pos0[b];
                else x0 = oracle_inv_cdf(wp, V, Zp, ui[0], &mg[0]);
                tok[0] = (int32_t)x0;
                acc[0] = 1;
                if (out_p_tok) out_p_tok[b * K] = (x0 >= 0 && x0 < V) ? wp[x0] / Zp : 0.0;
                if (out_q_tok) out_q_tok[b * K] = 0.0;
                if (out_tv) out_tv[b * K] = 0.0;
            } else {
                double Zq = oracle_warp_row(qrow, V, T, top_k, top_p, wq, &mg[4], NULL);
                int64_t d;
                if (drafts) d = drafts[b * K + i];
                else d = oracle_inv_cdf(wq, V, Zq, ui[0], &mg[0]);
                tok[i] = (int32_t)d;
                double pd = (d >= 0 && d < V) ? wp[d] / Zp : 0.0;
                double qd = (d >= 0 && d < V) ? wq[d] / Zq : 0.0;
                acc[i] = (ui[1] * qd < pd) ? 1 : 0;
                if (qd > 0.0) mg[1] = fabs(ui[1] - pd / qd);
                if (out_p_tok) out_p_tok[b * K + i] = pd;
                if (out_q_tok) out_q_tok[b * K + i] = qd;
                if (out_tv) {
                    double tv = 0.0;
                    for (int64_t v = 0; v < V; ++v) tv += fabs(wp[v] / Zp - wq[v] / Zq);
                    out_tv[b * K + i] = 0.5 * tv;
                }
                if (!acc[i] && first_reject < 0) {
                    first_reject = i;
                    /* residual: max(0, P_j - Q_j); no mass -> P_j itself */
                    double R = 0.0;
                    for (int64_t v = 0; v < V; ++v) {
                        double dlt = wp[v] / Zp - wq[v] / Zq;
                        res[v] = dlt > 0.0 ? dlt : 0.0;
                        R += res[v];
                    }
                    int64_t nxt;
                    if (R > 0.0) nxt = oracle_inv_cdf(res, V, R, ui[2], &mg[2]);
                    else nxt = oracle_inv_cdf(wp, V, Zp, ui[2], &mg[2]);
                    if (out_next) out_next[b] = (int32_t)nxt;
                }
            }
            if (margins)
                for (int c = 0; c < 5; ++c) margins[(b * K + i) * 5 + c] = mg[c];
        }
        int64_t n = first_reject < 0 ? K : first_reject;
        if (out_count) out_count[b] = (int32_t)n;
        if (out_tokens)
            for (int64_t i = 0; i < K; ++i) out_tokens[b * K + i] = i < n ? tok[i] : -1;
        if (first_reject < 0 && out_next) out_next[b] = -1;
        free(wp);
        free(wq);
        free(res);
        free(tok);
        free(acc);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * TV self-distillation loss and its gradient  [LU-train]
 *
 *   p = softmax(teacher_t), q = softmax(student_t)                  (T = 1, no filter)
 *   TV_t = 1/2 * sum_v |p_v - q_v|
 *   mean = sum_{t in mask} TV_t / N_mask          (0 when the mask is empty)
 *   dL/dstudent_{t,v} = grad_scale / N_mask * q_v * (s_v - sum_w q_w s_w),
 *                       s = 1/2 * sign(q - p), sign(0) = 0; 0 on unmasked tokens
 * (d TV / d q_v = s_v and d q_v / d z_w = q_v (delta_vw - q_w); the teacher is frozen.)
 * grad and absdiff ([N, V], |p - q|) are optional.
 * ------------------------------------------------------------------------------------ */
int oracle_tv_loss(const double* teacher, const double* student, int64_t N, int64_t V,
                   const uint8_t* mask, double grad_scale, double* tv, double* mean,
                   double* grad, double* absdiff)
{
    if (N < 0 || V < 1) return 1;
    int64_t n_mask = 0;
    for (int64_t t = 0; t < N; ++t) n_mask += (mask == NULL || mask[t]) ? 1 : 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < N; ++t) {
        const double* zt = teacher + t * V;
        const double* zs = student + t * V;
        double* p = (double*)malloc((size_t)V * sizeof(double));
        double* q = (double*)malloc((size_t)V * sizeof(double));
        double mt = -INFINITY, ms = -INFINITY;
        for (int64_t v = 0; v < V; ++v) {
            if (zt[v] > mt) mt = zt[v];
            if (zs[v] > ms) ms = zs[v];
        }
        double St = 0.0, Ss = 0.0;
        for (int64_t v = 0; v < V; ++v) {
            p[v] = exp(zt[v] - mt);
            q[v] = exp(zs[v] - ms);
            St += p[v];
            Ss += q[v];
        }
        double d = 0.0, c = 0.0;
        for (int64_t v = 0; v < V; ++v) {
            p[v] /= St;
            q[v] /= Ss;
            double diff = q[v] - p[v];
            d += fabs(diff);
            double sv = diff > 0.0 ? 0.5 : (diff < 0.0 ? -0.5 : 0.0);
            c += q[v] * sv;
            if (absdiff) absdiff[t * V + v] = fabs(diff);
        }
        tv[t] = 0.5 * d;
        if (grad) {
            int on = (mask == NULL || mask[t]) && n_mask > 0;
            double f = on ? grad_scale / (double)n_mask : 0.0;
            for (int64_t v = 0; v < V; ++v) {
                double diff = q[v] - p[v];
                double sv = diff > 0.0 ? 0.5 : (diff < 0.0 ? -0.5 : 0.0);
                grad[t * V + v] = f * q[v] * (sv - c);
            }
        }
        free(p);
        free(q);
    }
    double s = 0.0;
    for (int64_t t = 0; t < N; ++t)
        if (mask == NULL || mask[t]) s += tv[t];
    *mean = n_mask > 0 ? s / (double)n_mask : 0.0;
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Block noising, noise mode random_uniform [LU-train: the student reads a block-noised
 * copy of each sequence; MC-proto: noise mode random_uniform].
 * Readings: position 0 of every block keeps its token (it is the exact AR token, [LU-how])
 * and each draft position 1..K-1 gets a token drawn uniformly from the vocabulary from a
 * supplied uniform u in [0, 1):
 *   out[b, 0] = clean[b, 0];   out[b, i] = min(V - 1, floor(u[b, i] * V))   (i >= 1)
 * (u is a float32 and V < 2^24, so u * V is exact in fp64 and the floor is exact).
 * gate[b*K + i] (optional) is the row gate of the adapter: 0 at i = 0, 1 at the noise rows.
 * ------------------------------------------------------------------------------------ */
int oracle_block_noise(const int32_t* clean, const float* u, int64_t B, int64_t K, int64_t V, int32_t* out,
                       double* gate)
{
    if (B < 0 || K < 1 || V < 1 || V >= (1 << 24)) return 1;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t i = 0; i < K; ++i) {
            const int64_t o = b * K + i;
            if (i == 0) {
                out[o] = clean[o];
            } else {
                double t = floor((double)u[o] * (double)V);
                if (t > (double)(V - 1)) t = (double)(V - 1);
                out[o] = (int32_t)t;
            }
            if (gate) gate[o] = i == 0 ? 0.0 : 1.0;
        }
    }
    return 0;
}
