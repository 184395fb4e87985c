/*
 * oracle.c -- plain fp64 CPU reference for the batch-invariant forward path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * bench's CPU-baseline leg may load this library.  It shares no code, header
 * or table with the CUDA library; the two meet only through the seeded input
 * generators.
 *
 * The reports on "Defeating Nondeterminism in LLM Inference" name the three
 * operations whose batch-invariant versions make up the path -- RMSNorm,
 * matrix multiplication and attention (xitu-tech news, "构建确定性解决方案";
 * neican.ai insight, "技术原理与创新点解析") -- but print no formula for any of
 * them.  Each result the invariant kernels reach has a plain mathematical
 * definition (the kernels only fix the order of the floating-point
 * operations), so every function below is that definition written out in
 * double precision, in the most direct loop order, with no blocking, no
 * splitting of reductions and no reordering.
 *
 * Inputs are bfloat16 bit patterns (uint16_t), widened exactly to double.
 * Outputs are double.
 *
 * Readings of points the pages leave open (each listed in the design notes):
 *   - RMSNorm: y = x / sqrt(mean(x^2) + eps) * w, eps inside the root, plain
 *     weight (not 1 + w).
 *   - Matmul: C = A * W^T with W stored [N, K] (output-feature-major).
 *   - Attention: softmax(q.k * scale) over the keys a query may see,
 *     key j visible to the query at absolute position t iff j <= t;
 *     query head h reads kv head floor(h / (Hq / Hkv)); the paged cache is
 *     [num_pages, Hkv, 16, d] with the page of token j of sequence b being
 *     block_table[b][j / 16] and its slot j % 16.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_PAGE 16

static double bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

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

/*
 * RMSNorm of each row (xitu-tech news, "构建确定性解决方案", RMSNorm item;
 * neican.ai insight, "技术原理与创新点解析", batch-invariant RMSNorm bullet):
 *   y[r, j] = x[r, j] / sqrt( (1/H) * sum_i x[r, i]^2 + eps ) * w[j]
 */
void oracle_rmsnorm(const uint16_t *x, const uint16_t *w, int64_t M, int64_t H,
                    double eps, double *y)
{
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < M; ++r) {
        const uint16_t *xr = x + r * H;
        double ss = 0.0;
        for (int64_t i = 0; i < H; ++i) {
            double v = bf16_to_double(xr[i]);
            ss += v * v;
        }
        double denom = sqrt(ss / (double)H + eps);
        for (int64_t j = 0; j < H; ++j)
            y[r * H + j] = bf16_to_double(xr[j]) / denom * bf16_to_double(w[j]);
    }
}

/*
 * Matrix product (xitu-tech news, "构建确定性解决方案", matmul item;
 * neican.ai insight, "技术原理与创新点解析", batch-invariant matmul bullet):
 *   C[m, n] = sum_k A[m, k] * W[n, k]        A: [M, K], W: [N, K], C: [M, N]
 */
void oracle_matmul(const uint16_t *a, const uint16_t *w, int64_t M, int64_t N, int64_t K,
                   double *c)
{
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        const uint16_t *am = a + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint16_t *wn = w + n * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += bf16_to_double(am[k]) * bf16_to_double(wn[k]);
            c[m * N + n] = s;
        }
    }
}

/*
 * Write new tokens' keys and values into the paged cache before attention
 * runs (neican.ai insight, "技术原理与创新点解析", batch-invariant attention
 * bullet: the KV-cache page table is updated before the kernel launches).
 *   cache[slot / 16][g][slot % 16][:] = new[t][g][:]   for slot = slots[t] >= 0
 * Bit copy; slots < 0 are skipped.
 */
void oracle_kv_write(uint16_t *k_cache, uint16_t *v_cache, int32_t Hkv, int32_t d,
                     const uint16_t *k_new, const uint16_t *v_new, const int64_t *slots,
                     int64_t T)
{
    for (int64_t t = 0; t < T; ++t) {
        int64_t slot = slots[t];
        if (slot < 0) continue;
        int64_t page = slot / ORACLE_PAGE, off = slot % ORACLE_PAGE;
        for (int32_t g = 0; g < Hkv; ++g) {
            int64_t dst = ((page * Hkv + g) * ORACLE_PAGE + off) * d;
            int64_t src = (t * Hkv + g) * (int64_t)d;
            memcpy(k_cache + dst, k_new + src, (size_t)d * sizeof(uint16_t));
            memcpy(v_cache + dst, v_new + src, (size_t)d * sizeof(uint16_t));
        }
    }
}

/*
 * Causal softmax attention of single query rows over a paged KV cache
 * (neican.ai insight, "技术原理与创新点解析", batch-invariant attention bullet;
 * liuwei.blog, "破解之道", the attention example: parallel over queries,
 * reduce over keys and values).
 *
 * Row r is query head row_head[r] of sequence row_seq[r] at absolute position
 * row_pos[r] = t.  With g = floor(h / (Hq / Hkv)):
 *   s_j   = scale * sum_i q[r, i] * K_b[j, g, i]          j = 0 .. t
 *   p_j   = exp(s_j - max_j s_j) / sum_j exp(s_j - max_j s_j)
 *   o[r]  = sum_j p_j * V_b[j, g, :]
 *   lse[r] = max_j s_j + log(sum_j exp(s_j - max_j s_j))
 * where K_b[j] is read from page block_table[b][j / 16], slot j % 16.
 * The sequence is never split: the whole key range is reduced in one pass.
 * lse may be NULL.
 */
void oracle_attention(const uint16_t *q, int64_t R, int32_t d,
                      const int32_t *row_seq, const int32_t *row_head, const int32_t *row_pos,
                      int32_t Hq, const uint16_t *k_cache, const uint16_t *v_cache,
                      int32_t Hkv, const int32_t *block_table, int32_t max_pages,
                      double scale, double *o, double *lse)
{
    int32_t group = Hq / Hkv;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < R; ++r) {
        int32_t b = row_seq[r], h = row_head[r], t = row_pos[r];
        int32_t g = h / group;
        const uint16_t *qr = q + r * d;
        int64_t n = (int64_t)t + 1;
        double mx = -INFINITY;
        /* first pass: the logits and their maximum */
        for (int64_t j = 0; j < n; ++j) {
            int64_t page = block_table[(int64_t)b * max_pages + j / ORACLE_PAGE];
            const uint16_t *kj = k_cache + ((page * Hkv + g) * ORACLE_PAGE + j % ORACLE_PAGE) * d;
            double s = 0.0;
            for (int32_t i = 0; i < d; ++i)
                s += bf16_to_double(qr[i]) * bf16_to_double(kj[i]);
            s *= scale;
            if (s > mx) mx = s;
        }
        /* second pass: exponentials, their sum, and the weighted values */
        double *orow = o + r * d;
        for (int32_t i = 0; i < d; ++i) orow[i] = 0.0;
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            int64_t page = block_table[(int64_t)b * max_pages + j / ORACLE_PAGE];
            int64_t base = ((page * Hkv + g) * ORACLE_PAGE + j % ORACLE_PAGE) * d;
            const uint16_t *kj = k_cache + base;
            const uint16_t *vj = v_cache + base;
            double s = 0.0;
            for (int32_t i = 0; i < d; ++i)
                s += bf16_to_double(qr[i]) * bf16_to_double(kj[i]);
            double p = exp(s * scale - mx);
            l += p;
            for (int32_t i = 0; i < d; ++i)
                orow[i] += p * bf16_to_double(vj[i]);
        }
        for (int32_t i = 0; i < d; ++i) orow[i] /= l;
        if (lse) lse[r] = mx + log(l);
    }
}

/* ------------------------------------------------------------------------
 * The toy decoder's glue operations.  The reports on "Defeating
 * Nondeterminism in LLM Inference" restate an experiment in which one
 * prompt is completed greedily many times among other requests and the
 * distinct completions are counted (xitu-tech news, "显著成果与高昂成本";
 * liuwei.blog, "实验成果").  They name no layer of the model beyond the three
 * kernels, so the decoder around them is read as the plain pre-norm
 * transformer: token embedding, rotary position embedding (base theta,
 * rotate-half pairing), SwiGLU feed-forward, residual additions, greedy
 * argmax (lowest index on ties).  Each function is that definition in fp64.
 * ------------------------------------------------------------------------ */

/* out[t, :] = table[ids[t], :]  (bit copy; ids outside 0..V-1 leave the row
 * untouched). */
void oracle_embedding(const uint16_t *table, int64_t V, int64_t H, const int32_t *ids,
                      int64_t T, uint16_t *out)
{
    for (int64_t t = 0; t < T; ++t) {
        int64_t id = ids[t];
        if (id < 0 || id >= V) continue;
        memcpy(out + t * H, table + id * H, (size_t)H * sizeof(uint16_t));
    }
}

/*
 * Rotary position embedding of x [T, nh, d] at absolute positions pos[t]:
 * for i < d/2, with angle = pos * theta^(-2i/d), the pair (x_i, x_{i+d/2})
 * is rotated by that angle:
 *   out_i       = x_i cos(angle) - x_{i+d/2} sin(angle)
 *   out_{i+d/2} = x_{i+d/2} cos(angle) + x_i sin(angle)
 */
void oracle_rope(const uint16_t *x, int64_t T, int32_t nh, int32_t d, const int32_t *pos,
                 double theta, double *out)
{
    int32_t half = d / 2;
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        for (int32_t h = 0; h < nh; ++h) {
            const uint16_t *xr = x + (t * nh + h) * (int64_t)d;
            double *orow = out + (t * nh + h) * (int64_t)d;
            for (int32_t i = 0; i < half; ++i) {
                double angle = (double)pos[t] * pow(theta, -2.0 * (double)i / (double)d);
                double c = cos(angle), s = sin(angle);
                double a = bf16_to_double(xr[i]), b = bf16_to_double(xr[i + half]);
                orow[i] = a * c - b * s;
                orow[i + half] = b * c + a * s;
            }
        }
    }
}

/*
 * SwiGLU of gu [T, 2F] = [gate | up]:  out[t, j] = silu(g) * u with
 * g = gu[t, j], u = gu[t, F + j], silu(g) = g / (1 + exp(-g)).
 */
void oracle_swiglu(const uint16_t *gu, int64_t T, int64_t F, double *out)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        for (int64_t j = 0; j < F; ++j) {
            double g = bf16_to_double(gu[t * 2 * F + j]);
            double u = bf16_to_double(gu[t * 2 * F + F + j]);
            out[t * F + j] = g / (1.0 + exp(-g)) * u;
        }
    }
}

/*
 * Residual addition followed by RMSNorm of the sum:
 *   s[r, :] = x[r, :] + delta[r, :]
 *   y[r, j] = s[r, j] / sqrt( (1/H) * sum_i s[r, i]^2 + eps ) * w[j]
 * Both s and y are returned.
 */
void oracle_add_rmsnorm(const uint16_t *x, const uint16_t *delta, const uint16_t *w, int64_t M,
                        int64_t H, double eps, double *s, double *y)
{
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < M; ++r) {
        double ss = 0.0;
        for (int64_t i = 0; i < H; ++i) {
            double v = bf16_to_double(x[r * H + i]) + bf16_to_double(delta[r * H + i]);
            s[r * H + i] = v;
            ss += v * v;
        }
        double mean_sq = ss / (double)H;
        double rms = sqrt(mean_sq + eps);
        for (int64_t j = 0; j < H; ++j)
            y[r * H + j] = bf16_to_double(w[j]) * (s[r * H + j] / rms);
    }
}

/*
 * Greedy choice: out[t] = the lowest index j with logits[t, j] equal to the
 * row's maximum.  The logits are taken in the precision they are given in
 * (fp32), so the decision is the one that precision makes.
 */
void oracle_argmax(const float *logits, int64_t T, int64_t V, int32_t *out)
{
    for (int64_t t = 0; t < T; ++t) {
        const float *row = logits + t * V;
        int64_t best = 0;
        for (int64_t j = 1; j < V; ++j)
            if (row[j] > row[best]) best = j;
        out[t] = (int32_t)best;
    }
}

/* ------------------------------------------------------------------------
 * Sampling at temperature > 0 with nucleus (top-p) truncation, each request
 * drawing from its own counter-based random stream, so that a request's
 * token never depends on the other requests of the batch.  The reports tie
 * bitwise-identical sampling to on-policy reinforcement learning (xitu-tech
 * news, "强化学习的突破"; neican.ai insight, "未来发展路径预测") and set the
 * random seed aside as the cause of run-to-run differences (vpshk.cn,
 * "AI随机性的根源探析"); they describe no sampler.  Reading taken: the random
 * draw belongs to the request -- its seed and its position -- and every
 * reduction over the vocabulary has a fixed order.
 *
 * Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC 2011): a 128-bit counter, a 64-bit key,
 * ten rounds of two 32x32->64 multiplications with the key bumped by the
 * Weyl constants between rounds.
 * ------------------------------------------------------------------------ */

static void philox_round(uint32_t c[4], const uint32_t k[2])
{
    uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0], n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        philox_round(c, k);
    }
    for (int i = 0; i < 4; ++i) out[i] = c[i];
}

static int oracle_cmp_desc(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/*
 * One token per row of logits [T, V] (fp32, the precision the lm_head
 * produces them in):
 *   temperature 0: the greedy choice (lowest index of the maximum);
 *   otherwise, with z_i = logits_i / temperature and w_i = exp(z_i - max z):
 *     kept set K = { i : w_i >= tau }, tau the largest w-value such that the
 *       weights >= tau hold at least top_p of the total weight (ties at tau
 *       are all kept);  W_K = sum over K of w_i;
 *     u = the first Philox4x32-10 output word for key (seed lo, seed hi) and
 *       counter (offset lo, offset hi, 0, 0), u = (word >> 8) * 2^-24;
 *     the token is the first i of K, in index order, at which the running
 *       sum of w over K exceeds u * W_K.
 * r_out (may be NULL) receives u * W_K / W (the target as a fraction of the
 * total weight), zk_out (may be NULL) W_K / W.
 */
void oracle_sample(const float *logits, int64_t T, int64_t V, const float *temperature,
                   const float *top_p, const uint64_t *seed, const uint64_t *offset, int32_t *out,
                   double *r_out, double *zk_out)
{
    int64_t t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < T; ++t) {
        const float *row = logits + t * V;
        int64_t best = 0;
        for (int64_t j = 1; j < V; ++j)
            if (row[best] < row[j]) best = j;
        if (!(temperature[t] > 0.0f)) {
            out[t] = (int32_t)best;
            if (r_out) r_out[t] = 0.0;
            if (zk_out) zk_out[t] = 0.0;
            continue;
        }
        double *w = (double *)malloc((size_t)V * sizeof(double));
        double *sorted = (double *)malloc((size_t)V * sizeof(double));
        double mx = (double)row[best] / (double)temperature[t];
        double total = 0.0;
        for (int64_t j = 0; j < V; ++j) {
            w[j] = exp((double)row[j] / (double)temperature[t] - mx);
            total += w[j];
            sorted[j] = w[j];
        }
        qsort(sorted, (size_t)V, sizeof(double), oracle_cmp_desc);  /* descending */
        double need = (double)top_p[t] * total, acc = 0.0, tau = sorted[V - 1];
        for (int64_t j = 0; j < V; ++j) {
            acc += sorted[j];
            if (acc >= need) {
                tau = sorted[j];
                break;
            }
        }
        double zk = 0.0;
        for (int64_t j = 0; j < V; ++j)
            if (w[j] >= tau) zk += w[j];
        uint32_t ctr[4] = {(uint32_t)offset[t], (uint32_t)(offset[t] >> 32), 0u, 0u};
        uint32_t key[2] = {(uint32_t)seed[t], (uint32_t)(seed[t] >> 32)};
        uint32_t rnd[4];
        oracle_philox4x32_10(ctr, key, rnd);
        double u = (double)(rnd[0] >> 8) * (1.0 / 16777216.0);
        double target = u * zk, run = 0.0;
        int64_t tok = -1, last = -1;
        for (int64_t j = 0; j < V; ++j) {
            if (w[j] < tau) continue;
            last = j;
            run += w[j];
            if (run > target) {
                tok = j;
                break;
            }
        }
        out[t] = (int32_t)(tok >= 0 ? tok : last);
        if (r_out) r_out[t] = target / total;
        if (zk_out) zk_out[t] = zk / total;
        free(w);
        free(sorted);
    }
}

/* ------------------------------------------------------------------------
 * Mixture-of-experts feed-forward.  The model of the reports' experiment is
 * a mixture of experts (Qwen3-235B-A22B; xitu-tech news, "显著成果与高昂成本";
 * neican.ai insight, "技术原理与创新点解析"); they describe no router.  Reading
 * taken (the common top-k router): each token's router logits over E
 * experts pick its k experts by largest logit (lowest index on ties); the
 * gate weights are the softmax of the selected logits (the full softmax
 * renormalised over the k); the token's output is the gate-weighted sum of
 * its experts' outputs, taken in rank order.
 * ------------------------------------------------------------------------ */

/* experts[t, i] = the i-th largest logit's index (ties: lower index first);
 * weights[t, i] = exp(l_i - l_0) / sum_j exp(l_j - l_0) over the k chosen. */
void oracle_moe_route(const float *logits, int64_t T, int32_t E, int32_t k, int32_t *experts,
                      double *weights)
{
    for (int64_t t = 0; t < T; ++t) {
        const float *row = logits + t * E;
        int32_t *ex = experts + t * k;
        for (int32_t i = 0; i < k; ++i) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                int taken = 0;
                for (int32_t j = 0; j < i; ++j)
                    if (ex[j] == e) taken = 1;
                if (taken) continue;
                if (best < 0 || row[e] > row[best]) best = e;
            }
            ex[i] = best;
        }
        double sum = 0.0;
        for (int32_t i = 0; i < k; ++i) sum += exp((double)row[ex[i]] - (double)row[ex[0]]);
        for (int32_t i = 0; i < k; ++i)
            weights[t * k + i] = exp((double)row[ex[i]] - (double)row[ex[0]]) / sum;
    }
}

/* Group the T*k (token, rank) entries by expert: offsets[e] .. offsets[e+1]
 * hold expert e's entries in increasing entry index (entry = t*k + i);
 * order[p] is the entry at position p, pos[entry] its position. */
void oracle_moe_dispatch(const int32_t *experts, int64_t N, int32_t E, int64_t *offsets,
                         int64_t *order, int64_t *pos)
{
    int64_t p = 0;
    for (int32_t e = 0; e < E; ++e) {
        offsets[e] = p;
        for (int64_t i = 0; i < N; ++i)
            if (experts[i] == e) {
                order[p] = i;
                pos[i] = p;
                ++p;
            }
    }
    offsets[E] = p;
}

/* out[t, :] = sum over i of weights[t, i] * y[pos[t*k + i], :]. */
void oracle_moe_combine(const uint16_t *y, const int64_t *pos, const double *weights, int64_t T,
                        int32_t k, int64_t H, double *out)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        for (int64_t h = 0; h < H; ++h) out[t * H + h] = 0.0;
        for (int32_t i = 0; i < k; ++i) {
            const uint16_t *yr = y + pos[t * k + i] * H;
            for (int64_t h = 0; h < H; ++h) out[t * H + h] += weights[t * k + i] * bf16_to_double(yr[h]);
        }
    }
}

/*
 * Fused forms of the adjacent RMSNorm and matmul steps (xitu-tech news,
 * "构建确定性解决方案": the RMSNorm item followed by the matmul item; each
 * transformer block normalises a row and multiplies it by a weight).
 *
 * Norm weight folded into a matmul weight:
 *   wf[n, k] = W[n, k] * w[k]
 * (the product of two bfloat16 values, exact in double).
 */
void oracle_fold_norm_weight(const uint16_t *W, const uint16_t *w, int64_t N, int64_t K,
                             double *wf)
{
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            wf[n * K + k] = bf16_to_double(W[n * K + k]) * bf16_to_double(w[k]);
}

/*
 * RMSNorm (weight folded into wf) followed by the matrix product:
 *   y[m, k] = x[m, k] / sqrt( (1/K) * sum_i x[m, i]^2 + eps )
 *   C[m, n] = sum_k y[m, k] * wf[n, k]             x: [M, K], wf: [N, K]
 */
void oracle_rmsnorm_matmul(const uint16_t *x, const uint16_t *wf, int64_t M, int64_t N,
                           int64_t K, double eps, double *c)
{
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        const uint16_t *xm = x + m * K;
        double sum_sq = 0.0;
        for (int64_t i = 0; i < K; ++i) sum_sq += bf16_to_double(xm[i]) * bf16_to_double(xm[i]);
        const double root = sqrt(sum_sq / (double)K + eps);
        for (int64_t n = 0; n < N; ++n) {
            const uint16_t *wn = wf + n * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += (bf16_to_double(xm[k]) / root) * bf16_to_double(wn[k]);
            c[m * N + n] = s;
        }
    }
}

/*
 * Matrix product added to the residual stream (the residual connection of a
 * transformer block):
 *   C[m, n] = R[m, n] + sum_k A[m, k] * W[n, k]    R: [M, N], A: [M, K], W: [N, K]
 */
void oracle_matmul_residual(const uint16_t *r, const uint16_t *a, const uint16_t *w, int64_t M,
                            int64_t N, int64_t K, double *c)
{
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double dot = 0.0;
            for (int64_t k = 0; k < K; ++k)
                dot += bf16_to_double(a[m * K + k]) * bf16_to_double(w[n * K + k]);
            c[m * N + n] = bf16_to_double(r[m * N + n]) + dot;
        }
    }
}

/*
 * The rotary angles as a table: out[p][i] = (cos a, sin a) with
 * a = p * theta^(-2i/d), for positions p < P and i < d/2 -- the angles of
 * oracle_rope above, listed once per position.
 */
void oracle_rope_angles(int32_t P, int32_t d, double theta, double *out)
{
    int32_t p;
#pragma omp parallel for schedule(static)
    for (p = 0; p < P; ++p) {
        for (int32_t i = 0; i < d / 2; ++i) {
            const double freq = pow(theta, -(double)(2 * i) / (double)d);
            out[((int64_t)p * (d / 2) + i) * 2] = cos((double)p * freq);
            out[((int64_t)p * (d / 2) + i) * 2 + 1] = sin((double)p * freq);
        }
    }
}

/*
 * Backward of the RMSNorm above, for the trainer side of on-policy RL
 * (xitu-tech news, "强化学习的突破": the trainer must reproduce the sampler's
 * numbers, so its passes run on the same deterministic kernels).  With
 * r = 1 / sqrt((1/H) sum_i x_i^2 + eps) and y_j = x_j r w_j, the gradients of
 * a loss with upstream gradient dy are
 *   dx_j = r w_j dy_j - x_j (r^3 / H) sum_i w_i dy_i x_i        (per row)
 *   dw_j = sum over rows of dy_j x_j r
 */
void oracle_rmsnorm_backward(const uint16_t *x, const uint16_t *w, const uint16_t *dy,
                             int64_t M, int64_t H, double eps, double *dx, double *dw)
{
    double *rs = (double *)malloc((size_t)(M > 0 ? M : 1) * sizeof(double));
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < M; ++r) {
        double sq = 0.0, dot = 0.0;
        for (int64_t i = 0; i < H; ++i) {
            const double xi = bf16_to_double(x[r * H + i]);
            sq += xi * xi;
            dot += bf16_to_double(w[i]) * bf16_to_double(dy[r * H + i]) * xi;
        }
        const double inv = 1.0 / sqrt(sq / (double)H + eps);
        rs[r] = inv;
        for (int64_t j = 0; j < H; ++j)
            dx[r * H + j] = bf16_to_double(w[j]) * inv * bf16_to_double(dy[r * H + j]) -
                            bf16_to_double(x[r * H + j]) * inv * inv * inv / (double)H * dot;
    }
    for (int64_t j = 0; j < H; ++j) {
        double acc = 0.0;
        for (int64_t m = 0; m < M; ++m)
            acc += bf16_to_double(dy[m * H + j]) * bf16_to_double(x[m * H + j]) * rs[m];
        dw[j] = acc;
    }
    free(rs);
}

/*
 * Backward of oracle_attention for an upstream gradient dO of each query row
 * (the trainer side of on-policy RL; xitu-tech news, "强化学习的突破").  With
 * p_j the softmax weights of the visible keys and o = sum_j p_j v_j:
 *   dv_j += p_j dO,   dp_j = dO . v_j,   ds_j = p_j (dp_j - sum_i p_i dp_i),
 *   dq = scale sum_j ds_j k_j,           dk_j += scale ds_j q.
 * dk and dv are sums over every row that sees the key (all query heads of
 * the kv group, all positions), returned in the logical cache layout
 * [num_pages, Hkv, 16, d].  Rows are taken one after another.
 */
void oracle_attention_backward(const uint16_t *q, const uint16_t *dout, int64_t R, int32_t d,
                               const int32_t *row_seq, const int32_t *row_head,
                               const int32_t *row_pos, int32_t Hq, const uint16_t *k_cache,
                               const uint16_t *v_cache, int32_t Hkv, int32_t num_pages,
                               const int32_t *block_table, int32_t max_pages, double scale,
                               double *dq, double *dk, double *dv)
{
    const int64_t cache_elems = (int64_t)num_pages * Hkv * ORACLE_PAGE * d;
    for (int64_t e = 0; e < cache_elems; ++e) {
        dk[e] = 0.0;
        dv[e] = 0.0;
    }
    for (int64_t r = 0; r < R; ++r) {
        const int32_t kvh = row_head[r] / (Hq / Hkv);
        const int64_t visible = (int64_t)row_pos[r] + 1;
        const uint16_t *qr = q + r * d, *gr = dout + r * d;
        double *logit = (double *)malloc((size_t)visible * sizeof(double));
        double *wt = (double *)malloc((size_t)visible * sizeof(double));
        double *dp = (double *)malloc((size_t)visible * sizeof(double));
        int64_t *off = (int64_t *)malloc((size_t)visible * sizeof(int64_t));
        double top = -INFINITY;
        for (int64_t key = 0; key < visible; ++key) {
            const int64_t phys = block_table[(int64_t)row_seq[r] * max_pages + key / ORACLE_PAGE];
            off[key] = ((phys * Hkv + kvh) * ORACLE_PAGE + key % ORACLE_PAGE) * d;
            double dot = 0.0;
            for (int32_t i = 0; i < d; ++i)
                dot += bf16_to_double(qr[i]) * bf16_to_double(k_cache[off[key] + i]);
            logit[key] = scale * dot;
            if (logit[key] > top) top = logit[key];
        }
        double total = 0.0;
        for (int64_t key = 0; key < visible; ++key) {
            wt[key] = exp(logit[key] - top);
            total += wt[key];
        }
        double mean_dp = 0.0;
        for (int64_t key = 0; key < visible; ++key) {
            wt[key] /= total;
            double s = 0.0;
            for (int32_t i = 0; i < d; ++i)
                s += bf16_to_double(gr[i]) * bf16_to_double(v_cache[off[key] + i]);
            dp[key] = s;
            mean_dp += wt[key] * dp[key];
        }
        for (int32_t i = 0; i < d; ++i) dq[r * d + i] = 0.0;
        for (int64_t key = 0; key < visible; ++key) {
            const double ds = wt[key] * (dp[key] - mean_dp);
            for (int32_t i = 0; i < d; ++i) {
                dq[r * d + i] += scale * ds * bf16_to_double(k_cache[off[key] + i]);
                dk[off[key] + i] += scale * ds * bf16_to_double(qr[i]);
                dv[off[key] + i] += wt[key] * bf16_to_double(gr[i]);
            }
        }
        free(logit);
        free(wt);
        free(dp);
        free(off);
    }
}

/*
 * Backward of oracle_swiglu: with s = 1 / (1 + e^(-g)) and out = g s u,
 *   dgate = dout u s (1 + g (1 - s)),   dup = dout g s.
 * gu [T, 2F] = [gate | up], dout [T, F] -> dgu [T, 2F] = [dgate | dup].
 */
void oracle_swiglu_backward(const uint16_t *gu, const uint16_t *dout, int64_t T, int64_t F,
                            double *dgu)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        for (int64_t j = 0; j < F; ++j) {
            const double gate = bf16_to_double(gu[t * 2 * F + j]);
            const double up = bf16_to_double(gu[t * 2 * F + F + j]);
            const double sig = 1.0 / (1.0 + exp(-gate));
            const double dy = bf16_to_double(dout[t * F + j]);
            dgu[t * 2 * F + j] = dy * up * sig * (1.0 + gate * (1.0 - sig));
            dgu[t * 2 * F + F + j] = dy * gate * sig;
        }
    }
}

/*
 * Backward of oracle_rope: the rotation by the angle is orthogonal, so the
 * gradient is the upstream gradient rotated back by the same angle:
 *   dx_i       =  dy_i cos(a) + dy_{i+d/2} sin(a)
 *   dx_{i+d/2} = -dy_i sin(a) + dy_{i+d/2} cos(a),   a = pos theta^(-2i/d).
 */
void oracle_rope_backward(const uint16_t *dy, int64_t T, int32_t nh, int32_t d,
                          const int32_t *pos, double theta, double *dx)
{
    const int32_t half = d / 2;
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        for (int32_t h = 0; h < nh; ++h) {
            const uint16_t *gr = dy + (t * nh + h) * (int64_t)d;
            double *xr = dx + (t * nh + h) * (int64_t)d;
            for (int32_t i = 0; i < half; ++i) {
                const double ang = (double)pos[t] / pow(theta, (double)(2 * i) / (double)d);
                const double cs = cos(ang), sn = sin(ang);
                const double lo = bf16_to_double(gr[i]), hi = bf16_to_double(gr[i + half]);
                xr[i] = lo * cs + hi * sn;
                xr[i + half] = hi * cs - lo * sn;
            }
        }
    }
}
