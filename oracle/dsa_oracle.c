/*
 * dsa_oracle.c -- plain single-threaded CPU oracle for DeepSeek Sparse
 * Attention (DSA): lightning indexer, per-query top-k, sparse MLA.
 *
 * TEST INFRASTRUCTURE ONLY. This file is built into oracle/liboracle.so and
 * is called by the tests, by __graft_entry__.smoke() and by bench.py's CPU
 * baseline. The product library never links, loads or calls it, and it shares
 * no code with the CUDA path.
 *
 * Arithmetic is in double, from the stored input codes (e4m3 bytes, bf16
 * bits) decoded from their format definitions. Loops run in the order the
 * pages state the steps, with no blocking or fusion.
 *
 * Sources (page titles, sections):
 *  - "DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理" (agent.csdn.net), section 4
 *    "DSA 的四步工作流程": step 2 scores S_h = scale(mask(Q_h K^T)) and
 *    reweights them per head, S'_h = a_h * S_h; step 3 I = topk(S', k=2048),
 *    all keys when the context has <= 2048 tokens; step 4 softmax over the
 *    selected positions only, then the weighted sum of the selected values.
 *  - "DeepSeek V3.2 ... DSA" (m.gxzdkb.com/media/457.html), section
 *    "秘密武器": the indexer uses FP8 and ReLU instead of softmax.
 *  - The per-head sum: one score per (query, key) is needed for a per-query
 *    top-k; the sum over heads I[t,s] = sum_h w[t,h] * ReLU(scale*q[t,h].k[s])
 *    is the reading taken for the head reduction the pages leave implicit.
 *  - Causal mask: a query at position p sees keys 0..p (inclusive), from the
 *    page-5 workflow's remark that masking hides future tokens
 *    (devpress.csdn.net, section 3 "第二步").
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* e4m3 (the "fn" variant: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 is NaN). Written from the format
 * definition: exponent field 0 is subnormal, value m/8 * 2^-6. */
double dsa_oracle_e4m3(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bf16: the upper 16 bits of an IEEE binary32. */
double dsa_oracle_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Lightning indexer scores for a subset of query rows.
 *
 *   q8      [T][Hi][128] e4m3 codes; q_scale [T] or NULL (=1)
 *   k8      [S][128]     e4m3 codes; k_scale [S] or NULL (=1)
 *   w       [T][Hi]      per-head weights a_h
 *   query row t sits at position q_pos0 + t and sees keys 0..q_pos0+t.
 *   rows    [nrows]      which query rows to compute
 *   out_I   [nrows][S]   I[t,s] = sum_h w[t,h] * max(0, scale * qf[t,h].kf[s]),
 *                        rounded to float once; -INFINITY for masked keys
 *   out_A   [nrows][S]   sum_h |w[t,h]| * max(0, ...): the magnitude that
 *                        bounds the rounding of I (NULL to skip)
 * with qf = e4m3(q8) * q_scale[t], kf = e4m3(k8) * k_scale[s].
 */
int dsa_oracle_indexer(const uint8_t *q8, const float *q_scale,
                       const uint8_t *k8, const float *k_scale,
                       const float *w, int64_t T, int64_t S, int Hi,
                       int64_t q_pos0, double scale, const int64_t *rows,
                       int64_t nrows, float *out_I, float *out_A) {
    double lut[256];
    for (int i = 0; i < 256; ++i) lut[i] = dsa_oracle_e4m3((uint8_t)i);
    double *qf = (double *)malloc(sizeof(double) * (size_t)Hi * 128);
    double *kf = (double *)malloc(sizeof(double) * 128);
    if (!qf || !kf) { free(qf); free(kf); return -1; }
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        if (t < 0 || t >= T) { free(qf); free(kf); return -2; }
        double qs = q_scale ? (double)q_scale[t] : 1.0;
        for (int h = 0; h < Hi; ++h)
            for (int d = 0; d < 128; ++d)
                qf[h * 128 + d] = lut[q8[(t * Hi + h) * 128 + d]] * qs;
        int64_t pos = q_pos0 + t;
        for (int64_t s = 0; s < S; ++s) {
            if (s > pos) {                       /* causal mask */
                out_I[r * S + s] = -INFINITY;
                if (out_A) out_A[r * S + s] = 0.0f;
                continue;
            }
            double ks = k_scale ? (double)k_scale[s] : 1.0;
            for (int d = 0; d < 128; ++d) kf[d] = lut[k8[s * 128 + d]] * ks;
            double acc = 0.0, mag = 0.0;
            for (int h = 0; h < Hi; ++h) {
                double dot = 0.0;
                for (int d = 0; d < 128; ++d) dot += qf[h * 128 + d] * kf[d];
                double x = scale * dot;              /* scale(mask(q.k)) */
                double relu = x > 0.0 ? x : 0.0;     /* ReLU */
                double wh = (double)w[t * Hi + h];   /* per-head weight */
                acc += wh * relu;                    /* sum over heads */
                mag += fabs(wh) * relu;
            }
            out_I[r * S + s] = (float)acc;
            if (out_A) out_A[r * S + s] = (float)mag;
        }
    }
    free(qf);
    free(kf);
    return 0;
}

/* Total order used for selection: larger score first, then smaller index. */
typedef struct { float v; int32_t s; } cand_t;

static int cand_cmp(const void *a, const void *b) {
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

/*
 * Per-query top-k over score rows (step 3 of the four-step workflow).
 *
 *   I        [nrows][ld] float scores; row r has row_len[r] candidate keys,
 *            the keys 0..row_len[r]-1
 *   idx      [nrows][k]  selected key positions in the order (score desc,
 *            index asc); when row_len[r] <= k every key 0..row_len[r]-1 is
 *            selected (the short-context fallback), and slots past the
 *            selection hold -1.
 */
int dsa_oracle_topk(const float *I, int64_t nrows, int64_t ld,
                    const int64_t *row_len, int k, int32_t *idx) {
    if (k <= 0) return -3;
    cand_t *buf = NULL;
    int64_t cap = 0;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t n = row_len[r];
        int32_t *out = idx + r * k;
        if (n < 0 || n > ld) { free(buf); return -2; }
        if (n <= k) {
            for (int64_t j = 0; j < k; ++j) out[j] = j < n ? (int32_t)j : -1;
            continue;
        }
        if (n > cap) {
            free(buf);
            cap = n;
            buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)cap);
            if (!buf) return -1;
        }
        for (int64_t s = 0; s < n; ++s) {
            buf[s].v = I[r * ld + s];
            buf[s].s = (int32_t)s;
        }
        qsort(buf, (size_t)n, sizeof(cand_t), cand_cmp);
        for (int j = 0; j < k; ++j) out[j] = buf[j].s;
    }
    free(buf);
    return 0;
}

/*
 * Projection to the indexer inputs (step 1 of the workflow: "DeepSeek-V3.2-
 * Exp 模型优势与 DSA 工作原理", section 4 "步骤一：查询与键的投影"): queries
 * Q = H W_Q and keys K = H W_K with rotary position encoding, and per-head
 * weights a_h, a linear map of H.
 *
 *   h    [T][d] bf16 bits, wt [N][d] bf16 bits with N = Hi*128 + 128 + Hi:
 *        the rows of W_Q (Hi heads x 128), then W_K (128), then W_a (Hi)
 *   rope [T][64][2] (cos, sin) per token and dimension pair
 *   For each selected row t: y[n] = sum_j h[t][j] * wt[n][j] in double; then
 *   every (2i, 2i+1) pair of a q head and of k becomes
 *   (y0 cos_i - y1 sin_i, y0 sin_i + y1 cos_i) with token t's table entry i.
 *   out [nrows][N] double.
 */
int dsa_oracle_project(const uint16_t *h, const uint16_t *wt, const float *rope, int64_t T,
                       int64_t d, int Hi, const int64_t *rows, int64_t nrows, double *out) {
    if (Hi < 1 || d < 1) return -3;
    const int64_t N = (int64_t)Hi * 128 + 128 + Hi;
    const int64_t nqk = (int64_t)Hi * 128 + 128;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t t = rows[r];
        if (t < 0 || t >= T) return -2;
        double *y = out + r * N;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < d; ++j)
                acc += dsa_oracle_bf16(h[t * d + j]) * dsa_oracle_bf16(wt[n * d + j]);
            y[n] = acc;
        }
        for (int64_t n = 0; n < nqk; n += 2) {
            const int64_t i = (n % 128) / 2;
            const double c = rope[(t * 64 + i) * 2], sn = rope[(t * 64 + i) * 2 + 1];
            const double y0 = y[n], y1 = y[n + 1];
            y[n] = y0 * c - y1 * sn;
            y[n + 1] = y0 * sn + y1 * c;
        }
    }
    return 0;
}

/*
 * The indexer's warm-up objective ("ele-yufo.com/posts/deepseek-v3-2-exp",
 * section "四、训练的两步走冷启动"): dense attention gives each token's weight
 * distribution as the target, and the indexer is fitted to it by a KL
 * divergence. Row t sits at position q_pos0 + t and sees keys 0 .. min(that,
 * S - 1).
 *
 * dsa_oracle_attn_probs: out[r][s] = (1/H) sum_h softmax_s(sm_scale q[t,h].kv[s])
 *   over the row's keys, 0 past them. q [T][H][576], kv [S][576] bf16 bits;
 *   out [nrows][S] double.
 */
int dsa_oracle_attn_probs(const uint16_t *q, const uint16_t *kv, int64_t T, int64_t S, int H,
                          int64_t q_pos0, double sm_scale, const int64_t *rows, int64_t nrows,
                          double *out) {
    if (S < 1 || H < 1) return -3;
    double *z = (double *)malloc(sizeof(double) * (size_t)S);
    if (!z) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t t = rows[r];
        if (t < 0 || t >= T) { free(z); return -2; }
        int64_t pos = q_pos0 + t;
        if (pos > S - 1) pos = S - 1;
        double *o = out + r * S;
        for (int64_t s = 0; s < S; ++s) o[s] = 0.0;
        for (int h = 0; h < H; ++h) {
            const uint16_t *qr = q + ((int64_t)t * H + h) * 576;
            double m = -INFINITY;
            for (int64_t s = 0; s <= pos; ++s) {
                double acc = 0.0;
                for (int d = 0; d < 576; ++d)
                    acc += dsa_oracle_bf16(qr[d]) * dsa_oracle_bf16(kv[s * 576 + d]);
                z[s] = sm_scale * acc;
                if (z[s] > m) m = z[s];
            }
            double sum = 0.0;
            for (int64_t s = 0; s <= pos; ++s) sum += exp(z[s] - m);
            for (int64_t s = 0; s <= pos; ++s) o[s] += exp(z[s] - m) / sum / H;
        }
    }
    free(z);
    return 0;
}

/*
 * dsa_oracle_indexer_kl: for each row (n = row_len[r] keys), r_s = softmax(I)_s,
 *   loss[r] = sum_{s: p_s > 0} p_s (log p_s - log r_s), grad[r][s] = r_s - p_s
 *   (0 for s >= n). I, p, grad [nrows][ld] double.
 */
int dsa_oracle_indexer_kl(const double *I, const double *p, int64_t nrows, int64_t ld,
                          const int64_t *row_len, double *loss, double *grad) {
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t n = row_len[r];
        if (n < 1 || n > ld) return -2;
        const double *ir = I + r * ld, *pr = p + r * ld;
        double m = -INFINITY;
        for (int64_t s = 0; s < n; ++s) if (ir[s] > m) m = ir[s];
        double z = 0.0;
        for (int64_t s = 0; s < n; ++s) z += exp(ir[s] - m);
        const double logz = m + log(z);
        double kl = 0.0;
        for (int64_t s = 0; s < ld; ++s) {
            double g = 0.0;
            if (s < n) {
                const double lr = ir[s] - logz;
                if (pr[s] > 0.0) kl += pr[s] * (log(pr[s]) - lr);
                g = exp(lr) - pr[s];
            }
            grad[r * ld + s] = g;
        }
        loss[r] = kl;
    }
    return 0;
}

/*
 * dsa_oracle_indexer_backward: gradients through I[t,s] = sum_h w[t,h] *
 * ReLU(scale * x[t,h,s]), x = qf[t,h] . kf[s], qf = e4m3(q8) * q_scale[t],
 * kf = e4m3(k8) * k_scale[s], given grad[t][s] = dloss/dI over each row's keys
 * (the ReLU's decision [x > 0] is taken on the exact raw product e4m3(q8) .
 * e4m3(k8), which has the sign of x since the scales are positive):
 *   dq[t][h][:] = sum_s grad * w[t,h] * scale * [x > 0] * kf[s][:]
 *   dk[s][:]    = sum_{t,h} grad * w[t,h] * scale * [x > 0] * qf[t][h][:]
 *   dw[t][h]    = sum_s grad * ReLU(scale * x)
 * grad [T][S] double; dq [T][Hi][128], dk [S][128], dw [T][Hi] double out.
 */
int dsa_oracle_indexer_backward(const uint8_t *q8, const float *q_scale, const uint8_t *k8,
                                const float *k_scale, const float *w, int64_t T, int64_t S,
                                int Hi, int64_t q_pos0, double scale, const double *grad,
                                double *dq, double *dk, double *dw) {
    for (int64_t i = 0; i < T * Hi * 128; ++i) dq[i] = 0.0;
    for (int64_t i = 0; i < S * 128; ++i) dk[i] = 0.0;
    for (int64_t i = 0; i < T * Hi; ++i) dw[i] = 0.0;
    double qf[128], kf[128];
    for (int64_t t = 0; t < T; ++t) {
        int64_t pos = q_pos0 + t;
        if (pos > S - 1) pos = S - 1;
        const double qs = q_scale ? q_scale[t] : 1.0;
        for (int h = 0; h < Hi; ++h) {
            for (int d = 0; d < 128; ++d)
                qf[d] = dsa_oracle_e4m3(q8[(t * Hi + h) * 128 + d]) * qs;
            for (int64_t s = 0; s <= pos; ++s) {
                const double ks = k_scale ? k_scale[s] : 1.0;
                double xr = 0.0;               /* raw e4m3 dot product: exact in double */
                for (int d = 0; d < 128; ++d) {
                    kf[d] = dsa_oracle_e4m3(k8[s * 128 + d]) * ks;
                    xr += dsa_oracle_e4m3(q8[(t * Hi + h) * 128 + d]) * dsa_oracle_e4m3(k8[s * 128 + d]);
                }
                const double x = qs * ks * xr;
                const double g = grad[t * S + s];
                if (xr > 0.0) {
                    const double c = g * w[t * Hi + h] * scale;
                    for (int d = 0; d < 128; ++d) {
                        dq[(t * Hi + h) * 128 + d] += c * kf[d];
                        dk[s * 128 + d] += c * qf[d];
                    }
                    dw[t * Hi + h] += g * scale * x;
                }
            }
        }
    }
    return 0;
}

/*
 * Sliding-window selection, the fixed-distance rule DSA generalises
 * ("m.gxzdkb.com/media/457.html", section "秘密武器": a token attends only to
 * a fixed number of the keys before it; "oilbeater.com ... deepseek-sparse-
 * attention", section "Sparse Attention"). With a window covering the whole
 * prefix it is dense causal attention's index set.
 *
 *   Row r sits at position p = min(q_pos0 + r, S - 1) and takes every key s
 *   with p - window < s <= p and s >= 0, in increasing order; the rest of
 *   the row is -1. Requires 1 <= window <= k.
 */
int dsa_oracle_window(int64_t nrows, int64_t S, int64_t q_pos0, int window, int k,
                      int32_t *idx) {
    if (window < 1 || k < window || S < 1) return -3;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t p = q_pos0 + r;
        if (p > S - 1) p = S - 1;
        int32_t *out = idx + r * k;
        int j = 0;
        for (int64_t s = p - window + 1; s <= p; ++s)
            if (s >= 0) out[j++] = (int32_t)s;
        while (j < k) out[j++] = -1;
    }
    return 0;
}

/*
 * Sparse MLA forward for a subset of query rows (step 4 of the workflow).
 *
 *   q    [T][H][576] bf16 bits; kv [S][576] bf16 bits (512 latent + 64 rope)
 *   idx  [T][k] selected key positions; entries < 0 are skipped
 *   For each selected row t and head h, over the selected positions j:
 *     z_j = sm_scale * sum_{d<576} q[t,h,d] * kv[idx_j, d]
 *     p_j = exp(z_j - max z),  Z = sum p_j
 *     out[t,h,:] = sum_j p_j * kv[idx_j, :512] / Z      (values = the latent)
 *     lse[t,h]   = max z + ln Z
 *   out [nrows][H][512], lse [nrows][H] (double). A row with no selected
 *   position gets out = 0 and lse = -inf.
 */
int dsa_oracle_sparse_mla(const uint16_t *q, const uint16_t *kv,
                          const int32_t *idx, int64_t T, int64_t S, int H,
                          int k, double sm_scale, const int64_t *rows,
                          int64_t nrows, double *out, double *lse) {
    double *qd = (double *)malloc(sizeof(double) * 576);
    double *z = (double *)malloc(sizeof(double) * (size_t)k);
    double *acc = (double *)malloc(sizeof(double) * 512);
    if (!qd || !z || !acc) { free(qd); free(z); free(acc); return -1; }
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        if (t < 0 || t >= T) { free(qd); free(z); free(acc); return -2; }
        const int32_t *sel = idx + t * k;
        for (int j = 0; j < k; ++j)
            if (sel[j] >= S) { free(qd); free(z); free(acc); return -2; }
        for (int h = 0; h < H; ++h) {
            for (int d = 0; d < 576; ++d)
                qd[d] = dsa_oracle_bf16(q[(t * H + h) * 576 + d]);
            double m = -INFINITY;
            for (int j = 0; j < k; ++j) {
                if (sel[j] < 0) continue;
                const uint16_t *row = kv + (int64_t)sel[j] * 576;
                double dot = 0.0;
                for (int d = 0; d < 576; ++d) dot += qd[d] * dsa_oracle_bf16(row[d]);
                z[j] = sm_scale * dot;
                if (z[j] > m) m = z[j];
            }
            double *o = out + (r * H + h) * 512;
            for (int d = 0; d < 512; ++d) acc[d] = 0.0;
            double Z = 0.0;
            if (m != -INFINITY) {
                for (int j = 0; j < k; ++j) {
                    if (sel[j] < 0) continue;
                    const uint16_t *row = kv + (int64_t)sel[j] * 576;
                    double p = exp(z[j] - m);
                    Z += p;
                    for (int d = 0; d < 512; ++d) acc[d] += p * dsa_oracle_bf16(row[d]);
                }
            }
            for (int d = 0; d < 512; ++d) o[d] = Z > 0.0 ? acc[d] / Z : 0.0;
            if (lse) lse[r * H + h] = Z > 0.0 ? m + log(Z) : -INFINITY;
        }
    }
    free(qd);
    free(z);
    free(acc);
    return 0;
}
