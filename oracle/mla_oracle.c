/*
 * fp64 CPU oracle for DeepSeek-style Multi-head Latent Attention (MLA) decode
 * over a paged latent KV cache.
 *
 * TEST INFRASTRUCTURE ONLY. This file is built into its own shared library and
 * is loaded solely by the tests, by the smoke check and by the CPU-baseline leg
 * of the benchmark. It shares no code, header or constant with the CUDA path.
 *
 * Sources (page title, section):
 *  - "MLA operator design" page (bhfrc.com/news/60867) §1: per token and layer
 *    the cache holds the 512-d latent c_KV plus the 64-d decoupled RoPE key k_R.
 *  - same page §3: page_size 64 for the latent cache, block-table paging.
 *  - same page §4: path A (decompress: K_nope = c_KV W_UK per head) and path B
 *    (absorb: q_c W_UK first, then dot with c_KV); scale 1/sqrt(d_hc + d_R);
 *    weight layout w_uk[h][d][c].
 *  - "MHA2MLA" page (lpnh.cn/news/2494972) §2.1: k_nope = c_kv W_uk,
 *    v = c_kv W_uv, o = softmax(q_rope k_rope^T + q_nope k_nope^T) v.
 *
 * Every routine works in double precision. Inputs arrive as bf16 bit patterns
 * (uint16_t) and are widened exactly (bf16 -> fp32 is a 16-bit shift, fp32 ->
 * fp64 is exact). Loops follow the definitions term by term; the only
 * parallelism is across independent (batch, query, head) outputs.
 *
 * Conventions shared by all routines:
 *  - Query position: a sequence of length L (tokens already in the cache,
 *    including the n_q new ones) has queries i = 0..n_q-1 at positions
 *    L - n_q + i; query i sees tokens t in [0, L - n_q + i].
 *  - Paging: token t of sequence b lives in pool row
 *    block_table[b * max_pages + t / P] * P + t % P.
 *  - Return value: 0 on success, -1 on an invalid argument (bad page id,
 *    seq_len beyond the table, seq_len < n_q), in which case outputs are
 *    unspecified.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Row of the pool that holds token t of sequence b, or -1 if the table entry
 * is outside [0, num_pages). */
static int64_t pool_row(const int32_t *block_table, int max_pages, int P, int num_pages,
                        int b, int t) {
    int32_t page = block_table[(int64_t)b * max_pages + t / P];
    if (page < 0 || page >= num_pages) return -1;
    return (int64_t)page * P + (t % P);
}

static int check_lengths(const int32_t *seq_lens, int B, int n_q, int max_pages, int P) {
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < n_q) return -1;
        if ((int64_t)seq_lens[b] > (int64_t)max_pages * P) return -1;
    }
    return 0;
}

/*
 * Page gather (cache step of the "MLA operator design" page §3): copies the
 * bf16 bit patterns of tokens [0, L_b) of every sequence, in order, into
 * out[b][t][0..width). Rows t >= L_b are left untouched.
 * pool: [num_pages, P, width] with the given token stride (elements) and
 * page stride (elements).
 */
int oracle_gather(const uint16_t *pool, int64_t page_stride, int64_t token_stride, int width,
                  int num_pages, int P, const int32_t *block_table, int max_pages,
                  const int32_t *seq_lens, int B, int max_len, uint16_t *out) {
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || seq_lens[b] > max_len) return -1;
        if ((int64_t)seq_lens[b] > (int64_t)max_pages * P) return -1;
        for (int t = 0; t < seq_lens[b]; ++t) {
            int32_t page = block_table[(int64_t)b * max_pages + t / P];
            if (page < 0 || page >= num_pages) return -1;
            const uint16_t *src = pool + (int64_t)page * page_stride + (int64_t)(t % P) * token_stride;
            uint16_t *dst = out + ((int64_t)b * max_len + t) * width;
            for (int j = 0; j < width; ++j) dst[j] = src[j];
        }
    }
    return 0;
}

/*
 * The definition (path A of the "MLA operator design" page §4, the attention
 * formula of the "MHA2MLA" page §2.1), one (b, i, h) at a time:
 *   K_nope[t][d] = sum_c c_KV[t][c] * W_UK[h][d][c]
 *   V[t][e]      = sum_c c_KV[t][c] * W_UV[h][c][e]
 *   s[t]         = scale * (sum_d q_c[d] K_nope[t][d] + sum_j q_r[j] k_R[t][j])
 *   p            = softmax(s) over visible t
 *   out[e]       = sum_t p[t] V[t][e]
 * q_c [B,n_q,H,d_n], q_r [B,n_q,H,d_r], ckv pool [num_pages,P,d_c],
 * kr pool [num_pages,P,d_r], w_uk [H,d_n,d_c], w_uv [H,d_c,d_v], all bf16,
 * contiguous. out [B,n_q,H,d_v] fp64.
 * sel: optional list of flat (b*n_q + i)*H + h indices to compute (n_sel of
 * them); NULL computes every output.
 */
int oracle_decode_decompress(int B, int n_q, int H, int d_n, int d_c, int d_r, int d_v, int P,
                             double scale, const uint16_t *q_c, const uint16_t *q_r,
                             const uint16_t *ckv, const uint16_t *kr, int num_pages,
                             const int32_t *block_table, int max_pages, const int32_t *seq_lens,
                             const uint16_t *w_uk, const uint16_t *w_uv, const int64_t *sel,
                             int64_t n_sel, double *out) {
    if (check_lengths(seq_lens, B, n_q, max_pages, P)) return -1;
    int64_t total = sel ? n_sel : (int64_t)B * n_q * H;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < total; ++u) {
        int64_t flat = sel ? sel[u] : u;
        int h = (int)(flat % H);
        int i = (int)((flat / H) % n_q);
        int b = (int)(flat / ((int64_t)H * n_q));
        int L = seq_lens[b];
        int nvis = L - n_q + i + 1;
        double *s = (double *)malloc(sizeof(double) * (size_t)nvis);
        double *knope = (double *)malloc(sizeof(double) * (size_t)d_n);
        double *v = (double *)malloc(sizeof(double) * (size_t)d_v);
        double *acc = out + flat * d_v;
        const uint16_t *qc = q_c + flat * d_n;
        const uint16_t *qr = q_r + flat * d_r;
        for (int e = 0; e < d_v; ++e) acc[e] = 0.0;
        /* scores */
        double m = -INFINITY;
        for (int t = 0; t < nvis; ++t) {
            int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
            if (row < 0) { bad = 1; s[t] = 0.0; continue; }
            const uint16_t *c = ckv + row * d_c;
            const uint16_t *r = kr + row * d_r;
            for (int d = 0; d < d_n; ++d) {
                const uint16_t *w = w_uk + ((int64_t)h * d_n + d) * d_c;
                double k = 0.0;
                for (int cc = 0; cc < d_c; ++cc) k += bf16_to_f64(c[cc]) * bf16_to_f64(w[cc]);
                knope[d] = k;
            }
            double dot = 0.0;
            for (int d = 0; d < d_n; ++d) dot += bf16_to_f64(qc[d]) * knope[d];
            for (int j = 0; j < d_r; ++j) dot += bf16_to_f64(qr[j]) * bf16_to_f64(r[j]);
            s[t] = scale * dot;
            if (s[t] > m) m = s[t];
        }
        /* softmax */
        double z = 0.0;
        for (int t = 0; t < nvis; ++t) { s[t] = exp(s[t] - m); z += s[t]; }
        /* values */
        for (int t = 0; t < nvis; ++t) {
            int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
            if (row < 0) continue;
            const uint16_t *c = ckv + row * d_c;
            for (int e = 0; e < d_v; ++e) v[e] = 0.0;
            for (int cc = 0; cc < d_c; ++cc) {
                double cv = bf16_to_f64(c[cc]);
                const uint16_t *w = w_uv + ((int64_t)h * d_c + cc) * d_v;
                for (int e = 0; e < d_v; ++e) v[e] += cv * bf16_to_f64(w[e]);
            }
            double p = s[t] / z;
            for (int e = 0; e < d_v; ++e) acc[e] += p * v[e];
        }
        free(s);
        free(knope);
        free(v);
    }
    return bad ? -1 : 0;
}

/*
 * Absorb-in (path B of the "MLA operator design" page §4):
 *   q_lat[t][h][c] = sum_d q_c[t][h][d] * W_UK[h][d][c]
 * q_c [T,H,d_n] bf16, w_uk [H,d_n,d_c] bf16 -> q_lat [T,H,d_c] fp64.
 */
int oracle_absorb_q(int T, int H, int d_n, int d_c, const uint16_t *q_c, const uint16_t *w_uk,
                    double *q_lat) {
#pragma omp parallel for schedule(static)
    for (int64_t th = 0; th < (int64_t)T * H; ++th) {
        int h = (int)(th % H);
        const uint16_t *q = q_c + th * d_n;
        double *o = q_lat + th * d_c;
        for (int c = 0; c < d_c; ++c) o[c] = 0.0;
        for (int d = 0; d < d_n; ++d) {
            double qd = bf16_to_f64(q[d]);
            const uint16_t *w = w_uk + ((int64_t)h * d_n + d) * d_c;
            for (int c = 0; c < d_c; ++c) o[c] += qd * bf16_to_f64(w[c]);
        }
    }
    return 0;
}

/*
 * Rotary position embedding of the query's RoPE part ("MHA2MLA" page §3.2,
 * rope_theta 10000; the "MLA operator design" page §3 computes it in fp32,
 * this reference in fp64). Consecutive pairs (2i, 2i + 1) of x[t][h][:] turn
 * by the angle a = pos[t] * theta^(-2i / d_r):
 *   y[2i]     = x[2i] cos(a) - x[2i + 1] sin(a)
 *   y[2i + 1] = x[2i] sin(a) + x[2i + 1] cos(a)
 * x [T,H,d_r] bf16, pos [T] int32 (>= 0), y [T,H,d_r] fp64. Returns -1 on a
 * negative position or an odd d_r.
 */
int oracle_rope(int T, int H, int d_r, const uint16_t *x, const int32_t *pos, double theta,
                double *y) {
    if (d_r % 2 != 0 || theta <= 0.0) return -1;
    for (int t = 0; t < T; ++t)
        if (pos[t] < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t th = 0; th < (int64_t)T * H; ++th) {
        const int t = (int)(th / H);
        const uint16_t *xi = x + th * d_r;
        double *yo = y + th * d_r;
        for (int i = 0; i < d_r / 2; ++i) {
            const double freq = pow(theta, -2.0 * i / d_r);
            const double a = (double)pos[t] * freq;
            const double c = cos(a), sn = sin(a);
            const double x0 = bf16_to_f64(xi[2 * i]), x1 = bf16_to_f64(xi[2 * i + 1]);
            yo[2 * i] = x0 * c - x1 * sn;
            yo[2 * i + 1] = x0 * sn + x1 * c;
        }
    }
    return 0;
}

/*
 * Attention in latent space (the absorbed score and value steps):
 *   s[t]   = scale * (sum_c Q[c] c_KV[t][c] + sum_j Q[d_c + j] k_R[t][j])
 *   o[c]   = sum_t softmax(s)[t] * c_KV[t][c]
 *   lse    = log sum_t exp(s[t])        (natural log)
 * over the visible tokens of each query that also fall in the window
 * [t_lo, t_hi) (t_hi < 0 means no upper bound). A window with no visible
 * token gives o = 0 and lse = -inf.
 * Q is given either as bf16 (q_bf16, [B,n_q,H,d_c+d_r]) or as fp64 (q_f64,
 * same shape); exactly one of the two is non-NULL.
 * o_lat [B,n_q,H,d_c] fp64, lse [B,n_q,H] fp64.
 */
int oracle_attend_latent(int B, int n_q, int H, int d_c, int d_r, int P, double scale,
                         const uint16_t *q_bf16, const double *q_f64, const uint16_t *ckv,
                         const uint16_t *kr, int num_pages, const int32_t *block_table,
                         int max_pages, const int32_t *seq_lens, int t_lo, int t_hi,
                         const int64_t *sel, int64_t n_sel, double *o_lat, double *lse) {
    if (check_lengths(seq_lens, B, n_q, max_pages, P)) return -1;
    if ((q_bf16 == NULL) == (q_f64 == NULL)) return -1;
    const int D = d_c + d_r;
    int64_t total = sel ? n_sel : (int64_t)B * n_q * H;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < total; ++u) {
        int64_t flat = sel ? sel[u] : u;
        int i = (int)((flat / H) % n_q);
        int b = (int)(flat / ((int64_t)H * n_q));
        int L = seq_lens[b];
        int lo = t_lo > 0 ? t_lo : 0;
        int hi = L - n_q + i + 1;
        if (t_hi >= 0 && t_hi < hi) hi = t_hi;
        double *o = o_lat + flat * d_c;
        for (int c = 0; c < d_c; ++c) o[c] = 0.0;
        if (hi <= lo) { lse[flat] = -INFINITY; continue; }
        double *q = (double *)malloc(sizeof(double) * (size_t)D);
        double *s = (double *)malloc(sizeof(double) * (size_t)(hi - lo));
        for (int k = 0; k < D; ++k)
            q[k] = q_bf16 ? bf16_to_f64(q_bf16[flat * D + k]) : q_f64[flat * D + k];
        double m = -INFINITY;
        for (int t = lo; t < hi; ++t) {
            int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
            if (row < 0) { bad = 1; s[t - lo] = -INFINITY; continue; }
            const uint16_t *c = ckv + row * d_c;
            const uint16_t *r = kr + row * d_r;
            double dot = 0.0;
            for (int cc = 0; cc < d_c; ++cc) dot += q[cc] * bf16_to_f64(c[cc]);
            for (int j = 0; j < d_r; ++j) dot += q[d_c + j] * bf16_to_f64(r[j]);
            s[t - lo] = scale * dot;
            if (s[t - lo] > m) m = s[t - lo];
        }
        double z = 0.0;
        for (int t = lo; t < hi; ++t) { s[t - lo] = exp(s[t - lo] - m); z += s[t - lo]; }
        for (int t = lo; t < hi; ++t) {
            int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
            if (row < 0) continue;
            const uint16_t *c = ckv + row * d_c;
            double p = s[t - lo] / z;
            for (int cc = 0; cc < d_c; ++cc) o[cc] += p * bf16_to_f64(c[cc]);
        }
        lse[flat] = m + log(z);
        free(q);
        free(s);
    }
    return bad ? -1 : 0;
}

/*
 * Log-sum-exp merge of normalised partial results over disjoint token sets:
 *   L     = log sum_s exp(lse_s)
 *   o[c]  = sum_s exp(lse_s - L) * o_s[c]
 * A partial with lse = -inf has weight 0; if every partial is -inf the result
 * is o = 0, L = -inf.
 * o_part [R, S, d_c] fp64, lse_part [R, S] fp64 -> o [R, d_c], lse_out [R].
 */
int oracle_combine(int64_t R, int S, int d_c, const double *o_part, const double *lse_part,
                   double *o, double *lse_out) {
    for (int64_t r = 0; r < R; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (lse_part[r * S + s] > m) m = lse_part[r * S + s];
        double *dst = o + r * d_c;
        for (int c = 0; c < d_c; ++c) dst[c] = 0.0;
        if (m == -INFINITY) { lse_out[r] = -INFINITY; continue; }
        double z = 0.0;
        for (int s = 0; s < S; ++s) z += exp(lse_part[r * S + s] - m);
        double L = m + log(z);
        for (int s = 0; s < S; ++s) {
            double w = exp(lse_part[r * S + s] - L);
            const double *src = o_part + (r * S + s) * d_c;
            for (int c = 0; c < d_c; ++c) dst[c] += w * src[c];
        }
        lse_out[r] = L;
    }
    return 0;
}

/*
 * Absorb-out (up-projection of the latent result, the "MHA2MLA" page §2.1
 * v = c_kv W_uv applied after attention):
 *   out[t][h][e] = sum_c o_lat[t][h][c] * W_UV[h][c][e]
 * o_lat is given as bf16 (o_bf16) or fp64 (o_f64), exactly one non-NULL,
 * shape [T,H,d_c]; w_uv [H,d_c,d_v] bf16 -> out [T,H,d_v] fp64.
 */
int oracle_absorb_out(int T, int H, int d_c, int d_v, const uint16_t *o_bf16, const double *o_f64,
                      const uint16_t *w_uv, double *out) {
    if ((o_bf16 == NULL) == (o_f64 == NULL)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t th = 0; th < (int64_t)T * H; ++th) {
        int h = (int)(th % H);
        double *dst = out + th * d_v;
        for (int e = 0; e < d_v; ++e) dst[e] = 0.0;
        for (int c = 0; c < d_c; ++c) {
            double oc = o_bf16 ? bf16_to_f64(o_bf16[th * d_c + c]) : o_f64[th * d_c + c];
            const uint16_t *w = w_uv + ((int64_t)h * d_c + c) * d_v;
            for (int e = 0; e < d_v; ++e) dst[e] += oc * bf16_to_f64(w[e]);
        }
    }
    return 0;
}

/*
 * Decompression of the latent cache, path A of the "MLA operator design" page
 * §4 ("MHA2MLA" page §2.1: k_nope = c_kv W_uk, v = c_kv W_uv), per sequence b,
 * head h and cached token t < L_b:
 *   K_nope[b][h][t][d] = sum_c c_KV[t][c] * W_UK[h][d][c]
 *   V[b][h][t][e]      = sum_c c_KV[t][c] * W_UV[h][c][e]
 * k_nope [B,H,max_len,d_n] fp64, v [B,H,max_len,d_v] fp64; rows t >= L_b are
 * left untouched. Either output may be NULL.
 */
int oracle_decompress_kv(int B, int H, int d_n, int d_c, int d_v, int P, const uint16_t *ckv,
                         int num_pages, const int32_t *block_table, int max_pages,
                         const int32_t *seq_lens, const uint16_t *w_uk, const uint16_t *w_uv,
                         int max_len, double *k_nope, double *v) {
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > max_len ||
            (int64_t)seq_lens[b] > (int64_t)max_pages * P) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        for (int t = 0; t < seq_lens[b]; ++t) {
            int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
            if (row < 0) { bad = 1; continue; }
            const uint16_t *c = ckv + row * d_c;
            if (k_nope) {
                double *k = k_nope + (bh * max_len + t) * d_n;
                for (int d = 0; d < d_n; ++d) {
                    const uint16_t *w = w_uk + ((int64_t)h * d_n + d) * d_c;
                    double acc = 0.0;
                    for (int cc = 0; cc < d_c; ++cc) acc += bf16_to_f64(c[cc]) * bf16_to_f64(w[cc]);
                    k[d] = acc;
                }
            }
            if (v) {
                double *vv = v + (bh * max_len + t) * d_v;
                for (int e = 0; e < d_v; ++e) vv[e] = 0.0;
                for (int cc = 0; cc < d_c; ++cc) {
                    double cv = bf16_to_f64(c[cc]);
                    const uint16_t *w = w_uv + ((int64_t)h * d_c + cc) * d_v;
                    for (int e = 0; e < d_v; ++e) vv[e] += cv * bf16_to_f64(w[e]);
                }
            }
        }
    }
    return bad ? -1 : 0;
}

/*
 * Prefill through the decompress branch (the "MLA operator design" page §3 and
 * §6: a query count M at or above the prefill threshold takes path A, decode
 * takes path B). The M queries of sequence b are its last M tokens: query i sits
 * at position L_b - M + i and sees tokens t <= L_b - M + i (causal). For each
 * (b, h), K_nope and V are decompressed once (as in oracle_decompress_kv), then
 * per query:
 *   s[t] = scale * (sum_d q_c[d] K_nope[t][d] + sum_j q_r[j] k_R[t][j])
 *   out[e] = sum_t softmax(s)[t] V[t][e],   lse = m + log(sum_t exp(s[t] - m))
 * q_c [B,M,H,d_n], q_r [B,M,H,d_r], out [B,M,H,d_v] fp64, lse [B,M,H] fp64.
 * sel: optional flat (b*M + i)*H + h indices (n_sel of them); only those
 * outputs are written, and only the (b, h) pairs they touch are decompressed.
 */
int oracle_prefill_decompress(int B, int M, int H, int d_n, int d_c, int d_r, int d_v, int P,
                              double scale, const uint16_t *q_c, const uint16_t *q_r,
                              const uint16_t *ckv, const uint16_t *kr, int num_pages,
                              const int32_t *block_table, int max_pages, const int32_t *seq_lens,
                              const uint16_t *w_uk, const uint16_t *w_uv, const int64_t *sel,
                              int64_t n_sel, double *out, double *lse) {
    if (M < 1 || check_lengths(seq_lens, B, M, max_pages, P)) return -1;
    /* which queries of which (b, h) to compute */
    char *want = (char *)calloc((size_t)B * M * H, 1);
    if (!want) return -1;
    if (sel) {
        for (int64_t u = 0; u < n_sel; ++u) {
            if (sel[u] < 0 || sel[u] >= (int64_t)B * M * H) { free(want); return -1; }
            want[sel[u]] = 1;
        }
    } else {
        memset(want, 1, (size_t)B * M * H);
    }
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        int any = 0;
        for (int i = 0; i < M && !any; ++i) any = want[((int64_t)b * M + i) * H + h];
        if (!any) continue;
        int L = seq_lens[b];
        double *kn = (double *)malloc(sizeof(double) * (size_t)L * d_n);
        double *vv = (double *)malloc(sizeof(double) * (size_t)L * d_v);
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        /* decompress this head's keys and values once */
        for (int t = 0; t < L; ++t) {
            int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
            if (row < 0) { bad = 1; row = 0; }
            const uint16_t *c = ckv + row * d_c;
            for (int d = 0; d < d_n; ++d) {
                const uint16_t *w = w_uk + ((int64_t)h * d_n + d) * d_c;
                double acc = 0.0;
                for (int cc = 0; cc < d_c; ++cc) acc += bf16_to_f64(c[cc]) * bf16_to_f64(w[cc]);
                kn[(int64_t)t * d_n + d] = acc;
            }
            double *vt = vv + (int64_t)t * d_v;
            for (int e = 0; e < d_v; ++e) vt[e] = 0.0;
            for (int cc = 0; cc < d_c; ++cc) {
                double cv = bf16_to_f64(c[cc]);
                const uint16_t *w = w_uv + ((int64_t)h * d_c + cc) * d_v;
                for (int e = 0; e < d_v; ++e) vt[e] += cv * bf16_to_f64(w[e]);
            }
        }
        for (int i = 0; i < M; ++i) {
            int64_t flat = ((int64_t)b * M + i) * H + h;
            if (!want[flat]) continue;
            int nvis = L - M + i + 1;
            const uint16_t *qc = q_c + flat * d_n;
            const uint16_t *qr = q_r + flat * d_r;
            double m = -INFINITY;
            for (int t = 0; t < nvis; ++t) {
                int64_t row = pool_row(block_table, max_pages, P, num_pages, b, t);
                if (row < 0) row = 0;
                const uint16_t *r = kr + row * d_r;
                double dot = 0.0;
                for (int d = 0; d < d_n; ++d) dot += bf16_to_f64(qc[d]) * kn[(int64_t)t * d_n + d];
                for (int j = 0; j < d_r; ++j) dot += bf16_to_f64(qr[j]) * bf16_to_f64(r[j]);
                s[t] = scale * dot;
                if (s[t] > m) m = s[t];
            }
            double z = 0.0;
            for (int t = 0; t < nvis; ++t) { s[t] = exp(s[t] - m); z += s[t]; }
            double *o = out + flat * d_v;
            for (int e = 0; e < d_v; ++e) o[e] = 0.0;
            for (int t = 0; t < nvis; ++t) {
                double p = s[t] / z;
                for (int e = 0; e < d_v; ++e) o[e] += p * vv[(int64_t)t * d_v + e];
            }
            lse[flat] = m + log(z);
        }
        free(kn);
        free(vv);
        free(s);
    }
    free(want);
    return bad ? -1 : 0;
}

/*
 * Low-precision latent cache: fp8 E4M3 codes with one fp32 scale per cached
 * token (the "MLA operator design" page, introduction and §5, names a
 * quantised latent-cache gather but not its format; the E4M3 format used here
 * is the OCP 8-bit floating point one: sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits, subnormals at exponent field 0, S.1111.111 = NaN, no
 * infinities, largest finite 448).
 */

/* Value of an E4M3 code (NaN for S.1111.111). */
double oracle_e4m3_value(uint8_t code) {
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                 /* m/8 * 2^-6 */
    else v = ldexp(8.0 + m, e - 10);                      /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Nearest E4M3 code to the fp32 value y, ties to even mantissa, magnitudes
 * above 448 saturated to 448 (finite saturation). y must not be NaN. */
uint8_t oracle_e4m3_encode(float y) {
    const int sign = signbit(y) ? 1 : 0;
    double a = fabs((double)y);
    if (a >= 448.0) return (uint8_t)((sign << 7) | 0x7E);
    if (a == 0.0) return (uint8_t)(sign << 7);
    int e2;
    frexp(a, &e2);                                         /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                                        /* a in [2^e, 2^(e+1)) */
    if (e < -6) e = -6;                                    /* subnormal range */
    const double q = ldexp(1.0, e - 3);                    /* spacing of codes at this exponent */
    double n = rint(a / q);                                /* exact quotient, ties to even */
    double v = n * q;                                      /* <= 448: 448 is a code, 480 needs a >= 464 */
    int code;
    if (v < ldexp(1.0, -6)) {
        code = (int)(v / ldexp(1.0, -9));                  /* subnormal: m in 0..7 */
    } else {
        int ev2;
        frexp(v, &ev2);
        const int ev = ev2 - 1;
        code = ((ev + 7) << 3) | (int)(v / ldexp(1.0, ev - 3) - 8.0);
    }
    return (uint8_t)((sign << 7) | code);
}

/* bf16 bits of an fp32 value, round to nearest even (finite inputs). */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/*
 * Quantisation of rows x[r][0..d) (bf16 bits) to E4M3 with one scale per row,
 * all in IEEE fp32 (the arithmetic the kernels use, so codes agree bit for bit):
 *   amax = max |x|;  inv = 448 / amax  and  scale = amax / 448  (1 and 1 if amax = 0)
 *   code[j] = E4M3(x[j] * inv)
 */
void oracle_quantize_fp8_rows(int64_t R, int d, const uint16_t *x, uint8_t *codes, float *scales) {
    for (int64_t r = 0; r < R; ++r) {
        const uint16_t *xr = x + r * d;
        float amax = 0.0f;
        for (int j = 0; j < d; ++j) {
            const float v = fabsf((float)bf16_to_f64(xr[j]));
            if (v > amax) amax = v;
        }
        volatile float num = 448.0f;
        const float inv = amax > 0.0f ? num / amax : 1.0f;
        scales[r] = amax > 0.0f ? amax / num : 1.0f;
        for (int j = 0; j < d; ++j) {
            volatile float y = (float)bf16_to_f64(xr[j]) * inv;
            codes[r * d + j] = oracle_e4m3_encode(y);
        }
    }
}

/* Dequantisation to bf16 bits: bf16( fp32( value(code) * scale ) ). */
void oracle_dequant_fp8_rows(int64_t R, int d, const uint8_t *codes, const float *scales,
                             uint16_t *out) {
    for (int64_t r = 0; r < R; ++r)
        for (int j = 0; j < d; ++j) {
            volatile float v = (float)oracle_e4m3_value(codes[r * d + j]) * scales[r];
            out[r * d + j] = f32_to_bf16_rne(v);
        }
}
