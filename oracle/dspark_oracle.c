/*
 * fp64 CPU oracle for the DSpark draft MLA attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously-correct
 * definition that the CUDA path is checked against. Only the test suite, the
 * smoke entry point and the benchmark's CPU-baseline leg may load it. The
 * product library never links, loads or calls it, and the two share no code.
 *
 * Source: "GLM 5.2 DSpark speculative-training design" page.
 *   - §2 (model inputs, QKV construction): the KV axis is [S context | N draft
 *     blocks x 5]; Q holds only the 5N draft positions; RoPE positions are
 *     0..S-1 for context and A_n..A_n+4 for block n.
 *   - §3 (attention mask): a query of block n sees the context window
 *     A-W+1 <= kv < A (shared by the 5 block offsets, position A excluded) and
 *     the 5 positions of its own block, bidirectionally; other blocks are
 *     invisible; a block with block_keep_mask = 0 sees nothing.
 *   - §4 (MLA): per head the key is [k^C ; k^R] where k^R (d_r wide) is shared
 *     by all heads; scale (d_c + d_r)^(-1/2); RoPE rotates only the d_r slice,
 *     interleaved adjacent pairs.
 *   - appendix "Attention implementation": softmax(Q K^T / sqrt(d) + Lambda(M)) V
 *     with Lambda = 0 where M = 1 and -inf where M = 0; rows of a padding block
 *     are all zero.
 *
 * Readings taken where the page leaves a step open:
 *   - rotation angle of pair (2i, 2i+1) is pos * base^(-2i/d_r);
 *   - the rope slice is the last d_r entries of each query / key head vector;
 *   - the context window is clipped at 0: [max(0, A-W+1), A);
 *   - a padding block's rows give O = 0, LSE = -inf and zero gradients;
 *   - LSE is the natural-log log-sum-exp of the scaled scores of the row.
 *
 * Layouts (all contiguous, row-major):
 *   q  [B, n_h, 5N, d_c + d_r]      kc [B, n_h, S + 5N, d_c]
 *   kr [B, S + 5N, d_r]             v  [B, n_h, S + 5N, d_v]
 *   anchors int32 [B, N]            keep uint8 [B, N]
 *   o  [B, n_h, 5N, d_v]            lse [B, n_h, 5N]
 * Gradients have the layout of the tensor they belong to.
 *
 * Return value of every entry point: 0 on success, -1 for a bad size,
 * -2 for a kept anchor outside [0, S-2] (the range the anchor-sampling rule of
 * §2 allows), -3 for an allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define BLOCK 5 /* block_size = 5 (page §2, draft block) */

typedef struct {
    int B, n_h, S, N, W, d_c, d_r, d_v;
    double base;
} prob_t;

static int check_sizes(const prob_t *p) {
    if (p->B < 0 || p->n_h < 0 || p->S < 1 || p->N < 0 || p->W < 1) return -1;
    if (p->d_c < 0 || p->d_r < 0 || (p->d_r % 2) != 0 || p->d_v < 1) return -1;
    if (p->d_c + p->d_r < 1) return -1;
    return 0;
}

static int check_anchors(const prob_t *p, const int32_t *anchors, const uint8_t *keep) {
    for (int b = 0; b < p->B; b++)
        for (int n = 0; n < p->N; n++) {
            if (!keep[(size_t)b * p->N + n]) continue;
            int a = anchors[(size_t)b * p->N + n];
            if (a < 0 || a > p->S - 2) return -2;
        }
    return 0;
}

/* RoPE of page §4: pair (2i, 2i+1) is rotated by angle pos * theta_i,
 * theta_i = base^(-2i/d_r). sign = +1 rotates, sign = -1 applies the
 * transpose (the inverse rotation), used to pull gradients back. */
static void rope(const double *x, double *y, int d_r, double pos, double base, double sign) {
    for (int i = 0; i < d_r / 2; i++) {
        double theta = pow(base, -2.0 * i / (double)d_r);
        double c = cos(pos * theta), s = sign * sin(pos * theta);
        double x0 = x[2 * i], x1 = x[2 * i + 1];
        y[2 * i] = x0 * c - x1 * s;
        y[2 * i + 1] = x0 * s + x1 * c;
    }
}

/* Key set of block n (page §3): context positions [max(0, A-W+1), A) and the
 * block's own draft positions S+5n .. S+5n+4. keys[] gets KV indices, pos[]
 * their RoPE positions (context c -> c, draft S+5n+i -> A+i, page §2).
 * Returns the number of keys. */
static int key_set(const prob_t *p, int n, int a, int *keys, double *pos) {
    int lo = a - p->W + 1;
    if (lo < 0) lo = 0;
    int cnt = 0;
    for (int c = lo; c < a; c++) {
        keys[cnt] = c;
        pos[cnt] = (double)c;
        cnt++;
    }
    for (int i = 0; i < BLOCK; i++) {
        keys[cnt] = p->S + BLOCK * n + i;
        pos[cnt] = (double)(a + i);
        cnt++;
    }
    return cnt;
}

/* Scores, probabilities and LSE of one query row (b, h, block n, offset j).
 * qr (d_c+d_r) receives the rotated query; kk (cnt x (d_c+d_r)) the rotated
 * keys; prob (cnt) the softmax weights. Returns the LSE. */
static double row_forward(const prob_t *p, const double *q, const double *kc, const double *kr,
                          int b, int h, int n, int j, int a, int cnt, const int *keys,
                          const double *pos, double *qr, double *kk, double *prob) {
    const int dqk = p->d_c + p->d_r;
    const int L = p->S + BLOCK * p->N;
    const double scale = 1.0 / sqrt((double)dqk);
    const double *qrow = q + (((size_t)b * p->n_h + h) * (BLOCK * (size_t)p->N) + BLOCK * n + j) * dqk;
    memcpy(qr, qrow, sizeof(double) * p->d_c);
    rope(qrow + p->d_c, qr + p->d_c, p->d_r, (double)(a + j), p->base, +1.0);
    double m = -INFINITY;
    for (int t = 0; t < cnt; t++) {
        double *k = kk + (size_t)t * dqk;
        memcpy(k, kc + (((size_t)b * p->n_h + h) * L + keys[t]) * p->d_c, sizeof(double) * p->d_c);
        rope(kr + ((size_t)b * L + keys[t]) * p->d_r, k + p->d_c, p->d_r, pos[t], p->base, +1.0);
        double s = 0.0;
        for (int d = 0; d < dqk; d++) s += qr[d] * k[d];
        prob[t] = s * scale;
        if (prob[t] > m) m = prob[t];
    }
    double l = 0.0;
    for (int t = 0; t < cnt; t++) {
        prob[t] = exp(prob[t] - m);
        l += prob[t];
    }
    for (int t = 0; t < cnt; t++) prob[t] /= l;
    return m + log(l);
}

/* Forward: O and LSE for every row (appendix formula with the §3 mask). */
int oracle_attn_fwd(int B, int n_h, int S, int N, int W, int d_c, int d_r, int d_v, double base,
                    const double *q, const double *kc, const double *kr, const double *v,
                    const int32_t *anchors, const uint8_t *keep, double *o, double *lse) {
    prob_t p = {B, n_h, S, N, W, d_c, d_r, d_v, base};
    if (check_sizes(&p)) return -1;
    if (check_anchors(&p, anchors, keep)) return -2;
    const int dqk = d_c + d_r;
    const int L = S + BLOCK * N;
    const int kmax = W - 1 + BLOCK;
    int err = 0;
#pragma omp parallel
    {
        int *keys = (int *)malloc(sizeof(int) * kmax);
        double *pos = (double *)malloc(sizeof(double) * kmax);
        double *qr = (double *)malloc(sizeof(double) * dqk);
        double *kk = (double *)malloc(sizeof(double) * (size_t)kmax * dqk);
        double *prob = (double *)malloc(sizeof(double) * kmax);
        if (!keys || !pos || !qr || !kk || !prob) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for collapse(3) schedule(dynamic)
            for (int b = 0; b < B; b++)
                for (int h = 0; h < n_h; h++)
                    for (int n = 0; n < N; n++) {
                        size_t row0 = ((size_t)b * n_h + h) * (BLOCK * (size_t)N) + BLOCK * n;
                        if (!keep[(size_t)b * N + n]) {
                            for (int j = 0; j < BLOCK; j++) {
                                memset(o + (row0 + j) * d_v, 0, sizeof(double) * d_v);
                                lse[row0 + j] = -INFINITY;
                            }
                            continue;
                        }
                        int a = anchors[(size_t)b * N + n];
                        int cnt = key_set(&p, n, a, keys, pos);
                        for (int j = 0; j < BLOCK; j++) {
                            lse[row0 + j] = row_forward(&p, q, kc, kr, b, h, n, j, a, cnt, keys, pos, qr, kk, prob);
                            double *orow = o + (row0 + j) * d_v;
                            for (int d = 0; d < d_v; d++) orow[d] = 0.0;
                            for (int t = 0; t < cnt; t++) {
                                const double *vk = v + (((size_t)b * n_h + h) * L + keys[t]) * d_v;
                                for (int d = 0; d < d_v; d++) orow[d] += prob[t] * vk[d];
                            }
                        }
                    }
        }
        free(keys); free(pos); free(qr); free(kk); free(prob);
    }
    return err;
}

/* Backward of the forward above for the loss sum(dO * O), written out by hand:
 *   D = dO . O;  dP_t = dO . v_t;  dS_t = p_t (dP_t - D)
 *   dq_rot = scale * sum_t dS_t k_rot_t;  dk_rot_t += scale * dS_t q_rot;  dv_t += p_t dO
 * and the rope slices are pulled back through the rotation by its transpose.
 * dkr is shared by all heads (the rope key is copied to every head, page §4),
 * so its gradient is the sum over heads.
 * kr_part is scratch of B*n_h*(S+5N)*d_r doubles holding each head's pulled-back
 * rope-key gradient; the heads are summed in a fixed order afterwards. */
int oracle_attn_bwd(int B, int n_h, int S, int N, int W, int d_c, int d_r, int d_v, double base,
                    const double *q, const double *kc, const double *kr, const double *v,
                    const int32_t *anchors, const uint8_t *keep, const double *dout,
                    double *dq, double *dkc, double *dkr, double *dv) {
    prob_t p = {B, n_h, S, N, W, d_c, d_r, d_v, base};
    if (check_sizes(&p)) return -1;
    if (check_anchors(&p, anchors, keep)) return -2;
    const int dqk = d_c + d_r;
    const int L = S + BLOCK * N;
    const int kmax = W - 1 + BLOCK;
    const double scale = 1.0 / sqrt((double)dqk);
    double *kr_part = NULL;
    if (d_r > 0) {
        kr_part = (double *)calloc((size_t)B * n_h * L * d_r + 1, sizeof(double));
        if (!kr_part) return -3;
    }
    memset(dq, 0, sizeof(double) * (size_t)B * n_h * BLOCK * N * dqk);
    memset(dkc, 0, sizeof(double) * ((size_t)B * n_h * L * d_c + 0));
    memset(dv, 0, sizeof(double) * (size_t)B * n_h * L * d_v);
    int err = 0;
#pragma omp parallel
    {
        int *keys = (int *)malloc(sizeof(int) * kmax);
        double *pos = (double *)malloc(sizeof(double) * kmax);
        double *qr = (double *)malloc(sizeof(double) * dqk);
        double *kk = (double *)malloc(sizeof(double) * (size_t)kmax * dqk);
        double *prob = (double *)malloc(sizeof(double) * kmax);
        double *orow = (double *)malloc(sizeof(double) * d_v);
        double *dqr = (double *)malloc(sizeof(double) * dqk);
        double *dkr_rot = (double *)malloc(sizeof(double) * (d_r + 1));
        double *dkr_back = (double *)malloc(sizeof(double) * (d_r + 1));
        if (!keys || !pos || !qr || !kk || !prob || !orow || !dqr || !dkr_rot || !dkr_back) {
#pragma omp atomic write
            err = -3;
        } else {
            /* one (b, h) pair per task: every array written below is private to it */
#pragma omp for collapse(2) schedule(dynamic)
            for (int b = 0; b < B; b++)
                for (int h = 0; h < n_h; h++)
                    for (int n = 0; n < N; n++) {
                        if (!keep[(size_t)b * N + n]) continue; /* zero gradients */
                        int a = anchors[(size_t)b * N + n];
                        int cnt = key_set(&p, n, a, keys, pos);
                        for (int j = 0; j < BLOCK; j++) {
                            size_t row = ((size_t)b * n_h + h) * (BLOCK * (size_t)N) + BLOCK * n + j;
                            row_forward(&p, q, kc, kr, b, h, n, j, a, cnt, keys, pos, qr, kk, prob);
                            const double *dorow = dout + row * d_v;
                            for (int d = 0; d < d_v; d++) orow[d] = 0.0;
                            for (int t = 0; t < cnt; t++) {
                                const double *vk = v + (((size_t)b * n_h + h) * L + keys[t]) * d_v;
                                for (int d = 0; d < d_v; d++) orow[d] += prob[t] * vk[d];
                            }
                            double D = 0.0;
                            for (int d = 0; d < d_v; d++) D += dorow[d] * orow[d];
                            for (int d = 0; d < dqk; d++) dqr[d] = 0.0;
                            for (int t = 0; t < cnt; t++) {
                                const size_t kidx = ((size_t)b * n_h + h) * L + keys[t];
                                const double *vk = v + kidx * d_v;
                                double dP = 0.0;
                                for (int d = 0; d < d_v; d++) dP += dorow[d] * vk[d];
                                double dS = prob[t] * (dP - D);
                                const double *k = kk + (size_t)t * dqk;
                                for (int d = 0; d < dqk; d++) dqr[d] += scale * dS * k[d];
                                for (int d = 0; d < d_c; d++) dkc[kidx * d_c + d] += scale * dS * qr[d];
                                for (int d = 0; d < d_r; d++) dkr_rot[d] = scale * dS * qr[d_c + d];
                                rope(dkr_rot, dkr_back, d_r, pos[t], base, -1.0);
                                double *part = kr_part + kidx * d_r;
                                for (int d = 0; d < d_r; d++) part[d] += dkr_back[d];
                                double *dvk = dv + kidx * d_v;
                                for (int d = 0; d < d_v; d++) dvk[d] += prob[t] * dorow[d];
                            }
                            double *dqrow = dq + row * dqk;
                            for (int d = 0; d < d_c; d++) dqrow[d] = dqr[d];
                            rope(dqr + d_c, dqrow + d_c, d_r, (double)(a + j), base, -1.0);
                        }
                    }
        }
        free(keys); free(pos); free(qr); free(kk); free(prob); free(orow); free(dqr);
        free(dkr_rot); free(dkr_back);
    }
    if (err) { free(kr_part); return err; }
    memset(dkr, 0, sizeof(double) * ((size_t)B * L * d_r + 0));
    for (int b = 0; b < B; b++)
        for (int h = 0; h < n_h; h++)
            for (size_t e = 0; e < (size_t)L * d_r; e++)
                dkr[(size_t)b * L * d_r + e] += kr_part[(((size_t)b * n_h + h) * L) * d_r + e];
    free(kr_part);
    return 0;
}

/* Forward of a chosen list of rows only, for checks at sizes where the full
 * forward is too slow: row i is (b, h, r) with r = 5n + j. Outputs are packed
 * in list order: o [count, d_v], lse [count]. */
int oracle_attn_fwd_rows(int B, int n_h, int S, int N, int W, int d_c, int d_r, int d_v, double base,
                         const double *q, const double *kc, const double *kr, const double *v,
                         const int32_t *anchors, const uint8_t *keep,
                         int count, const int32_t *row_b, const int32_t *row_h, const int32_t *row_r,
                         double *o, double *lse) {
    prob_t p = {B, n_h, S, N, W, d_c, d_r, d_v, base};
    if (check_sizes(&p)) return -1;
    if (check_anchors(&p, anchors, keep)) return -2;
    const int dqk = d_c + d_r;
    const int L = S + BLOCK * N;
    const int kmax = W - 1 + BLOCK;
    int *keys = (int *)malloc(sizeof(int) * kmax);
    double *pos = (double *)malloc(sizeof(double) * kmax);
    double *qr = (double *)malloc(sizeof(double) * dqk);
    double *kk = (double *)malloc(sizeof(double) * (size_t)kmax * dqk);
    double *prob = (double *)malloc(sizeof(double) * kmax);
    int err = (!keys || !pos || !qr || !kk || !prob) ? -3 : 0;
    for (int i = 0; i < count && !err; i++) {
        int b = row_b[i], h = row_h[i], r = row_r[i];
        if (b < 0 || b >= B || h < 0 || h >= n_h || r < 0 || r >= BLOCK * N) { err = -1; break; }
        int n = r / BLOCK, j = r % BLOCK;
        double *orow = o + (size_t)i * d_v;
        for (int d = 0; d < d_v; d++) orow[d] = 0.0;
        if (!keep[(size_t)b * N + n]) { lse[i] = -INFINITY; continue; }
        int a = anchors[(size_t)b * N + n];
        int cnt = key_set(&p, n, a, keys, pos);
        lse[i] = row_forward(&p, q, kc, kr, b, h, n, j, a, cnt, keys, pos, qr, kk, prob);
        for (int t = 0; t < cnt; t++) {
            const double *vk = v + (((size_t)b * n_h + h) * L + keys[t]) * d_v;
            for (int d = 0; d < d_v; d++) orow[d] += prob[t] * vk[d];
        }
    }
    free(keys); free(pos); free(qr); free(kk); free(prob);
    return err;
}

/* Gradient of one query row (dq) or one key (dkc, dv for one head; dkr summed
 * over all heads) for a chosen list, computed by visiting every block whose key
 * set holds that key. This is a gather over the same definition the scatter in
 * oracle_attn_bwd uses, so the two can be compared.
 * kind 0: (b, h, r) -> dq row [d_c + d_r]
 * kind 1: (b, h, key) -> dkc [d_c] then dv [d_v]   (packed, d_c + d_v values)
 * kind 2: (b, -, key) -> dkr [d_r]                  (sum over heads)
 * out is packed in list order with the per-kind width above. */
int oracle_attn_bwd_items(int B, int n_h, int S, int N, int W, int d_c, int d_r, int d_v, double base,
                          const double *q, const double *kc, const double *kr, const double *v,
                          const int32_t *anchors, const uint8_t *keep, const double *dout,
                          int kind, int count, const int32_t *it_b, const int32_t *it_h,
                          const int32_t *it_x, double *out) {
    prob_t p = {B, n_h, S, N, W, d_c, d_r, d_v, base};
    if (check_sizes(&p)) return -1;
    if (check_anchors(&p, anchors, keep)) return -2;
    if (kind < 0 || kind > 2) return -1;
    const int dqk = d_c + d_r;
    const int L = S + BLOCK * N;
    const int kmax = W - 1 + BLOCK;
    const double scale = 1.0 / sqrt((double)dqk);
    const int width = kind == 0 ? dqk : (kind == 1 ? d_c + d_v : d_r);
    int err = 0;
#pragma omp parallel
    {
        int *keys = (int *)malloc(sizeof(int) * kmax);
        double *pos = (double *)malloc(sizeof(double) * kmax);
        double *qr = (double *)malloc(sizeof(double) * dqk);
        double *kk = (double *)malloc(sizeof(double) * (size_t)kmax * dqk);
        double *prob = (double *)malloc(sizeof(double) * kmax);
        double *orow = (double *)malloc(sizeof(double) * d_v);
        double *tmp = (double *)malloc(sizeof(double) * (dqk + 1));
        double *tmp2 = (double *)malloc(sizeof(double) * (dqk + 1));
        if (!keys || !pos || !qr || !kk || !prob || !orow || !tmp || !tmp2) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic)
            for (int i = 0; i < count; i++) {
                double *res = out + (size_t)i * width;
                for (int d = 0; d < width; d++) res[d] = 0.0;
                int b = it_b[i], x = it_x[i];
                int h0 = kind == 2 ? 0 : it_h[i];
                int h1 = kind == 2 ? n_h : it_h[i] + 1;
                if (b < 0 || b >= B || h0 < 0 || h1 > n_h) continue;
                if (kind == 0 && (x < 0 || x >= BLOCK * N)) continue;
                if (kind != 0 && (x < 0 || x >= L)) continue;
                for (int h = h0; h < h1; h++)
                    for (int n = 0; n < N; n++) {
                        if (!keep[(size_t)b * N + n]) continue;
                        if (kind == 0 && n != x / BLOCK) continue;
                        int a = anchors[(size_t)b * N + n];
                        int cnt = key_set(&p, n, a, keys, pos);
                        int tk = -1;
                        if (kind != 0) {
                            for (int t = 0; t < cnt; t++)
                                if (keys[t] == x) tk = t;
                            if (tk < 0) continue; /* block n does not see key x */
                        }
                        for (int j = 0; j < BLOCK; j++) {
                            if (kind == 0 && j != x % BLOCK) continue;
                            size_t row = ((size_t)b * n_h + h) * (BLOCK * (size_t)N) + BLOCK * n + j;
                            row_forward(&p, q, kc, kr, b, h, n, j, a, cnt, keys, pos, qr, kk, prob);
                            const double *dorow = dout + row * d_v;
                            for (int d = 0; d < d_v; d++) orow[d] = 0.0;
                            for (int t = 0; t < cnt; t++) {
                                const double *vk = v + (((size_t)b * n_h + h) * L + keys[t]) * d_v;
                                for (int d = 0; d < d_v; d++) orow[d] += prob[t] * vk[d];
                            }
                            double D = 0.0;
                            for (int d = 0; d < d_v; d++) D += dorow[d] * orow[d];
                            if (kind == 0) {
                                for (int d = 0; d < dqk; d++) tmp[d] = 0.0;
                                for (int t = 0; t < cnt; t++) {
                                    const double *vk = v + (((size_t)b * n_h + h) * L + keys[t]) * d_v;
                                    double dP = 0.0;
                                    for (int d = 0; d < d_v; d++) dP += dorow[d] * vk[d];
                                    double dS = prob[t] * (dP - D);
                                    for (int d = 0; d < dqk; d++) tmp[d] += scale * dS * kk[(size_t)t * dqk + d];
                                }
                                for (int d = 0; d < d_c; d++) res[d] += tmp[d];
                                rope(tmp + d_c, tmp2, d_r, (double)(a + j), base, -1.0);
                                for (int d = 0; d < d_r; d++) res[d_c + d] += tmp2[d];
                            } else {
                                const double *vk = v + (((size_t)b * n_h + h) * L + x) * d_v;
                                double dP = 0.0;
                                for (int d = 0; d < d_v; d++) dP += dorow[d] * vk[d];
                                double dS = prob[tk] * (dP - D);
                                if (kind == 1) {
                                    for (int d = 0; d < d_c; d++) res[d] += scale * dS * qr[d];
                                    for (int d = 0; d < d_v; d++) res[d_c + d] += prob[tk] * dorow[d];
                                } else {
                                    for (int d = 0; d < d_r; d++) tmp[d] = scale * dS * qr[d_c + d];
                                    rope(tmp, tmp2, d_r, pos[tk], base, -1.0);
                                    for (int d = 0; d < d_r; d++) res[d] += tmp2[d];
                                }
                            }
                        }
                    }
            }
        }
        free(keys); free(pos); free(qr); free(kk); free(prob); free(orow); free(tmp); free(tmp2);
    }
    return err;
}

/* Candidate anchors of page §2 (anchor sampling): A in [0, S-2] with
 * loss_mask[A] = loss_mask[A+1] = 1, where loss_mask[S-1] is read as 0
 * (appendix A, option 2: the last position is neither an anchor nor a label).
 * Writes the candidates in increasing order; returns their count. */
int oracle_anchor_candidates(int S, const uint8_t *loss_mask, int32_t *out) {
    int cnt = 0;
    for (int a = 0; a + 1 < S; a++) {
        int next = (a + 1 == S - 1) ? 0 : loss_mask[a + 1];
        if (loss_mask[a] && next) out[cnt++] = a;
    }
    return cnt;
}
