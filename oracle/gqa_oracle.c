/*
 * gqa_oracle.c -- plain fp64 CPU oracle for the Qwen3 attention sub-block
 * (per-head q/k RMSNorm -> RoPE -> grouped-query causal softmax(QK^T/sqrt(d) + M) V).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may load, call or link
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * Every step is the plain definition written out in double precision, with no
 * blocking, fusion or reordering beyond the loops of the definition.  bf16
 * inputs arrive as their raw 16-bit patterns and are widened to double exactly;
 * fp32 norm weights are widened exactly; nothing is rounded on the way.
 *
 * Sources (pages of the reference, by title and section):
 *  [A] "Qwen3系列1-理论基础&真实结构" (zhanghao0806.com), D1-2 (stable softmax
 *      via z - max z), D1-4 (softmax(QK^T/sqrt(d_k) + M) V, row-wise softmax),
 *      D1-5 (causal mask: position i sees j <= i, -inf before the softmax),
 *      D2-1 (RMSNorm = gamma * x / sqrt(mean(x^2) + eps)), D2-2 (QK-Norm per
 *      head on Q and K after projection, then RoPE; V gets neither; one scale
 *      vector shared by all Q heads and one by all K heads; RoPE matrix R(pos)
 *      with 2x2 rotation blocks on adjacent pairs), D2-3 (GQA; KV cache holds
 *      K and V per KV head; decode attends one new token to the cache).
 *  [B] "深入剖析Qwen3模型架构" (ewbang.com), 3.1.2 (GQA with K/V
 *      repeat_interleave over query heads; RoPE on (x[::2], x[1::2]) pairs),
 *      3.4.1 (inv_freq = base^(-2i/dim), base 1e6).
 *  [C] "Qwen3" (selfknow.cn, nano-vllm walkthrough), "Attention 的 Forward 流程"
 *      (order: q/k RMSNorm, then rotary embedding, then attention).
 *  [D] "Qwen3学习日志" (2048ai.net), section 一 (GQA: H query heads in G groups
 *      of h = H/G sharing one K/V head; G = H is MHA, G = 1 is MQA).
 *  [E] the zizhi168.cn summary of the Qwen3 report (no title), 4.2 "序列长度扩展的技术方案"
 *      (linear position interpolation; an NTK-aware variant).
 *
 * Readings where the pages are silent or disagree (each also listed in the
 * design notes): adjacent-pair RoPE; weight multiplies the normalised vector
 * (not 1 + w) and eps sits inside the square root; the L2-normalize variant
 * shown once in [B] 3.1.2 is not used; the 1/sqrt(D) scale is applied after
 * RoPE; query head hq uses KV head hq / (H/Hkv); the causal mask is on the
 * token index inside the sequence while `pos` only drives RoPE; decode sees
 * every cached row (cache rows are already normed and rotated K, raw V).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of a bf16 bit pattern: the bf16 value is the top half of an
 * IEEE binary32, so shifting it up 16 bits gives the same number as a float. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* RMSNorm over one head vector, [A] D2-1: out_d = w_d * x_d / sqrt(mean(x^2) + eps). */
void oracle_rmsnorm(const double *x, const double *w, double eps, int D, double *out)
{
    double ss = 0.0;
    for (int d = 0; d < D; ++d)
        ss += x[d] * x[d];
    double inv_rms = 1.0 / sqrt(ss / (double)D + eps);
    for (int d = 0; d < D; ++d)
        out[d] = w[d] * x[d] * inv_rms;
}

/* RoPE on one head vector, [A] D2-2 (R(pos) block-diagonal with 2x2 rotations on
 * adjacent pairs) and [B] 3.1.2 / 3.4.1 (pairs x[2i], x[2i+1]; angle pos * theta_i,
 * theta_i = base^(-2i/D), i = 0 .. D/2-1):
 *   out[2i]   = x[2i] cos(phi) - x[2i+1] sin(phi)
 *   out[2i+1] = x[2i] sin(phi) + x[2i+1] cos(phi),   phi = pos * base^(-2i/D). */
void oracle_rope(const double *x, double pos, double base, int D, double *out)
{
    for (int i = 0; i < D / 2; ++i) {
        double theta_i = pow(base, -2.0 * (double)i / (double)D);
        double phi = pos * theta_i;
        double c = cos(phi), s = sin(phi);
        double a = x[2 * i], b = x[2 * i + 1];
        out[2 * i] = a * c - b * s;
        out[2 * i + 1] = a * s + b * c;
    }
}

/* ---- RoPE variants: the frequency table, the pairing and the logit multiplier ----
 *
 * Frequencies theta_i, i = 0 .. D/2-1, for a base b and an extension factor s >= 1:
 *   none    b^(-2i/D)                                   ([B] 3.4.1)
 *   linear  b^(-2i/D) / s: the position divided by s (the linear interpolation of [E] 4.2,
 *           i.e. Position Interpolation, Chen et al. 2023)
 *   ntk     (b * s^(D/(D-2)))^(-2i/D): the base raised so that the lowest frequency is
 *           divided by s and the highest is kept ("NTK-aware" scaling; [E] 4.2 prints a
 *           garbled formula, so the published form is used)
 *   yarn    "NTK-by-parts" of YaRN (Peng, Quesnelle, Fan, Shippole 2023, sec. 3.2-3.4;
 *           [B] 3.4.2 prints a garbled formula): with wavelength lambda_i = 2 pi / theta_i
 *           and r_i = L / lambda_i (L the training context length),
 *           gamma_i = clamp((r_i - beta_slow) / (beta_fast - beta_slow), 0, 1) and
 *           theta'_i = (1 - gamma_i) theta_i / s + gamma_i theta_i;
 *           the logits are multiplied by (0.1 ln s + 1)^2 (YaRN's temperature, applied
 *           as sqrt(1/t) = 0.1 ln s + 1 on both q and k).
 * Pairing: adjacent rotates (x[2i], x[2i+1]) by pos * theta_i ([A] D2-2, [B] 3.1.2);
 * half rotates (x[i], x[i + D/2]) by the same angle (the rotate-half layout). */
void oracle_rope_inv_freq(double base, int D, int scaling, double factor, int orig_max_pos,
                          double beta_fast, double beta_slow, double *inv_freq)
{
    const double two_pi = 6.283185307179586476925286766559;
    for (int i = 0; i < D / 2; ++i) {
        double th = pow(base, -2.0 * (double)i / (double)D);
        if (scaling == 1) {
            th = th / factor;
        } else if (scaling == 2) {
            double b2 = base * pow(factor, (double)D / (double)(D - 2));
            th = pow(b2, -2.0 * (double)i / (double)D);
        } else if (scaling == 3) {
            double r = (double)orig_max_pos / (two_pi / th);
            double gamma = (r - beta_slow) / (beta_fast - beta_slow);
            if (gamma < 0.0)
                gamma = 0.0;
            if (gamma > 1.0)
                gamma = 1.0;
            th = (1.0 - gamma) * th / factor + gamma * th;
        }
        inv_freq[i] = th;
    }
}

double oracle_rope_logit_mult(int scaling, double factor)
{
    if (scaling == 3) {
        double m = 0.1 * log(factor) + 1.0;
        return m * m;
    }
    return 1.0;
}

/* RoPE of one head vector with a given frequency table and pairing (0 adjacent, 1 half). */
void oracle_rope_ex(const double *x, double pos, const double *inv_freq, int pairing, int D,
                    double *out)
{
    for (int i = 0; i < D / 2; ++i) {
        double phi = pos * inv_freq[i];
        double c = cos(phi), s = sin(phi);
        int ia = pairing ? i : 2 * i;
        int ib = pairing ? i + D / 2 : 2 * i + 1;
        double a = x[ia], b = x[ib];
        out[ia] = a * c - b * s;
        out[ib] = a * s + b * c;
    }
}

/* The plain frequency table b^(-2i/D) of [B] 3.4.1 (as oracle_rope uses), caller frees. */
static double *plain_inv_freq(double base, int D)
{
    double *f = (double *)malloc(sizeof(double) * (D / 2 > 0 ? D / 2 : 1));
    oracle_rope_inv_freq(base, D, 0, 1.0, 1, 32.0, 1.0, f);
    return f;
}

/* q-hat / k-hat of one head vector: RMSNorm, then RoPE ([A] D2-2, [C] forward steps 4-5). */
static void norm_then_rope(const uint16_t *xbits, const double *w, int32_t pos,
                           const double *inv_freq, int pairing, double eps, int D, double *tmp,
                           double *out)
{
    for (int d = 0; d < D; ++d)
        out[d] = bf16_bits_to_double(xbits[d]);
    oracle_rmsnorm(out, w, eps, D, tmp);
    oracle_rope_ex(tmp, (double)pos, inv_freq, pairing, D, out);
}

/* Apply norm + RoPE to every head vector of x [N, nheads, D] with positions pos [N].
 * Exposes the oracle's q-hat / k-hat (used by the tests to build a decode cache). */
void oracle_qk_transform_ex(const uint16_t *x, const int32_t *pos, const float *w,
                            const double *inv_freq, int pairing, double eps, int64_t N, int nheads,
                            int D, double *out)
{
    double *wd = (double *)malloc(sizeof(double) * D);
    for (int d = 0; d < D; ++d)
        wd[d] = (double)w[d];
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n)
            for (int h = 0; h < nheads; ++h)
                norm_then_rope(x + (n * nheads + h) * D, wd, pos[n], inv_freq, pairing, eps, D, tmp,
                               out + (n * nheads + h) * D);
        free(tmp);
    }
    free(wd);
}

void oracle_qk_transform(const uint16_t *x, const int32_t *pos, const float *w, double base,
                         double eps, int64_t N, int nheads, int D, double *out)
{
    double *f = plain_inv_freq(base, D);
    oracle_qk_transform_ex(x, pos, w, f, 0, eps, N, nheads, D, out);
    free(f);
}

/* One output row of attention, [A] D1-4 / D1-2: given the scores s_j of the visible
 * keys (already masked to the visible set), p_j = e^{s_j - max s} / sum_l e^{s_l - max s},
 * out = sum_j p_j v_j.  v_rows[j] points at key j's value vector. */
static void softmax_weighted_sum(const double *s, int n, const double *const *v_rows, int D,
                                 double *p, double *out)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m)
            m = s[j];
    double z = 0.0;
    for (int j = 0; j < n; ++j) {
        p[j] = exp(s[j] - m);
        z += p[j];
    }
    for (int j = 0; j < n; ++j)
        p[j] /= z;
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    for (int j = 0; j < n; ++j)
        for (int d = 0; d < D; ++d)
            out[d] += p[j] * v_rows[j][d];
}

/* Grouped-query scaled dot-product attention on already-transformed fp64 tensors.
 * q [B,T,H,D], k/v [B,T,Hkv,D], out [B,T,H,D].  [D] section 一 and [B] 3.1.2: query
 * head hq reads KV head hq / (H/Hkv).  causal != 0 applies [A] D1-5 (key j visible to
 * row i iff j <= i); causal == 0 lets every row see every key.  Scores are
 * q.k / sqrt(D), [A] D1-4.  If attn_w is not NULL it receives the weights
 * [B,H,T,T] (zero where masked). */
void oracle_sdpa_gqa(const double *q, const double *k, const double *v, int B, int T, int H,
                     int Hkv, int D, int causal, double *out, double *attn_w)
{
    int h_per_kv = H / Hkv;
    double inv_sqrt_d = 1.0 / sqrt((double)D);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
        double *p = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (T > 0 ? T : 1));
#pragma omp for collapse(3) schedule(dynamic, 16)
        for (int b = 0; b < B; ++b)
            for (int hq = 0; hq < H; ++hq)
                for (int i = 0; i < T; ++i) {
                    int g = hq / h_per_kv;
                    int n = causal ? i + 1 : T;
                    const double *qi = q + (((int64_t)b * T + i) * H + hq) * D;
                    for (int j = 0; j < n; ++j) {
                        const double *kj = k + (((int64_t)b * T + j) * Hkv + g) * D;
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d)
                            dot += qi[d] * kj[d];
                        s[j] = dot * inv_sqrt_d;
                        vr[j] = v + (((int64_t)b * T + j) * Hkv + g) * D;
                    }
                    softmax_weighted_sum(s, n, vr, D, p, out + (((int64_t)b * T + i) * H + hq) * D);
                    if (attn_w) {
                        double *wrow = attn_w + (((int64_t)b * H + hq) * T + i) * T;
                        for (int j = 0; j < T; ++j)
                            wrow[j] = j < n ? p[j] : 0.0;
                    }
                }
        free(s);
        free(p);
        free(vr);
    }
}

/* Prefill: the whole sub-block on bf16 inputs ([C] forward steps 4-6).
 * q [B,T,H,D], k/v [B,T,Hkv,D] bf16 bits; pos [B,T]; wq/wk [D] fp32; out [B,T,H,D] fp64. */
void oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *pos,
                    const float *wq, const float *wk, double base, double eps, int B, int T,
                    int H, int Hkv, int D, double *out)
{
    int64_t ntok = (int64_t)B * T;
    double *qh = (double *)malloc(sizeof(double) * (size_t)(ntok * H * D + 1));
    double *kh = (double *)malloc(sizeof(double) * (size_t)(ntok * Hkv * D + 1));
    double *vd = (double *)malloc(sizeof(double) * (size_t)(ntok * Hkv * D + 1));
    oracle_qk_transform(q, pos, wq, base, eps, ntok, H, D, qh);
    oracle_qk_transform(k, pos, wk, base, eps, ntok, Hkv, D, kh);
    for (int64_t e = 0; e < ntok * Hkv * D; ++e)
        vd[e] = bf16_bits_to_double(v[e]);
    oracle_sdpa_gqa(qh, kh, vd, B, T, H, Hkv, D, 1, out, NULL);
    free(qh);
    free(kh);
    free(vd);
}

/* Prefill for a chosen set of output rows only (for workloads too large to run in
 * full on a CPU).  rows holds nrows triples (b, hq, i); out is [nrows, D].  Each row
 * is computed from scratch by the same definition as oracle_prefill: q-hat of row i,
 * k-hat of keys 0..i of KV head hq / (H/Hkv), causal softmax, weighted sum of V. */
void oracle_prefill_rows_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *pos, const float *wq, const float *wk,
                            const double *inv_freq, int pairing, double logit_mult, double eps,
                            int B, int T, int H, int Hkv, int D, int64_t nrows, const int64_t *rows,
                            double *out)
{
    (void)B;
    int h_per_kv = H / Hkv;
    double inv_sqrt_d = logit_mult / sqrt((double)D);
    double *wqd = (double *)malloc(sizeof(double) * D);
    double *wkd = (double *)malloc(sizeof(double) * D);
    for (int d = 0; d < D; ++d) {
        wqd[d] = (double)wq[d];
        wkd[d] = (double)wk[d];
    }
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
        double *qi = (double *)malloc(sizeof(double) * D);
        double *kj = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
        double *p = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
        double *vbuf = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * D);
        const double **vr = (const double **)malloc(sizeof(double *) * (T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t b = rows[3 * r], hq = rows[3 * r + 1], i = rows[3 * r + 2];
            int64_t g = hq / h_per_kv;
            norm_then_rope(q + ((b * T + i) * H + hq) * D, wqd, pos[b * T + i], inv_freq, pairing, eps, D,
                           tmp, qi);
            for (int64_t j = 0; j <= i; ++j) {
                norm_then_rope(k + ((b * T + j) * Hkv + g) * D, wkd, pos[b * T + j], inv_freq, pairing, eps,
                               D, tmp, kj);
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += qi[d] * kj[d];
                s[j] = dot * inv_sqrt_d;
                const uint16_t *vj = v + ((b * T + j) * Hkv + g) * D;
                for (int d = 0; d < D; ++d)
                    vbuf[j * D + d] = bf16_bits_to_double(vj[d]);
                vr[j] = vbuf + j * D;
            }
            softmax_weighted_sum(s, (int)(i + 1), vr, D, p, out + r * D);
        }
        free(tmp);
        free(qi);
        free(kj);
        free(s);
        free(p);
        free(vbuf);
        free(vr);
    }
    free(wqd);
    free(wkd);
}

void oracle_prefill_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const int32_t *pos, const float *wq, const float *wk, double base,
                         double eps, int B, int T, int H, int Hkv, int D, int64_t nrows,
                         const int64_t *rows, double *out)
{
    double *f = plain_inv_freq(base, D);
    oracle_prefill_rows_ex(q, k, v, pos, wq, wk, f, 0, 1.0, eps, B, T, H, Hkv, D, nrows, rows, out);
    free(f);
}

/* Decode: one new query token per sequence against its KV cache ([A] D2-3: prefill
 * writes K/V to the cache, decode feeds one token and reads the cache).
 * q [B,H,D] bf16 bits (raw: normed and rotated here at position qpos[b], or at
 * position seqlens[b] when qpos is NULL); k_cache/v_cache [rows,Hkv,D] bf16 bits,
 * sequence b owning rows offsets[b] .. offsets[b]+seqlens[b]-1, which are used as
 * already-normed, already-rotated K and raw V; all of them are visible (the cache
 * holds only earlier positions).  out [B,H,D] fp64. */
void oracle_decode_ex(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                      const int64_t *offsets, const int32_t *seqlens, const int32_t *qpos,
                      const float *wq, const double *inv_freq, int pairing, double logit_mult,
                      double eps, int B, int H, int Hkv, int D, double *out)
{
    int h_per_kv = H / Hkv;
    double inv_sqrt_d = logit_mult / sqrt((double)D);
    int32_t maxlen = 1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] > maxlen)
            maxlen = seqlens[b];
    double *wqd = (double *)malloc(sizeof(double) * D);
    for (int d = 0; d < D; ++d)
        wqd[d] = (double)wq[d];
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
        double *qi = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * maxlen);
        double *p = (double *)malloc(sizeof(double) * maxlen);
        double *vbuf = (double *)malloc(sizeof(double) * (size_t)maxlen * D);
        const double **vr = (const double **)malloc(sizeof(double *) * maxlen);
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int b = 0; b < B; ++b)
            for (int hq = 0; hq < H; ++hq) {
                int g = hq / h_per_kv;
                int32_t len = seqlens[b];
                int32_t position = qpos ? qpos[b] : len;
                norm_then_rope(q + ((int64_t)b * H + hq) * D, wqd, position, inv_freq, pairing, eps, D, tmp,
                               qi);
                for (int32_t j = 0; j < len; ++j) {
                    int64_t row = offsets[b] + j;
                    const uint16_t *kj = k_cache + (row * Hkv + g) * D;
                    const uint16_t *vj = v_cache + (row * Hkv + g) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += qi[d] * bf16_bits_to_double(kj[d]);
                    s[j] = dot * inv_sqrt_d;
                    for (int d = 0; d < D; ++d)
                        vbuf[(int64_t)j * D + d] = bf16_bits_to_double(vj[d]);
                    vr[j] = vbuf + (int64_t)j * D;
                }
                softmax_weighted_sum(s, len, vr, D, p, out + ((int64_t)b * H + hq) * D);
            }
        free(tmp);
        free(qi);
        free(s);
        free(p);
        free(vbuf);
        free(vr);
    }
    free(wqd);
}

void oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                   const int64_t *offsets, const int32_t *seqlens, const int32_t *qpos,
                   const float *wq, double base, double eps, int B, int H, int Hkv, int D,
                   double *out)
{
    double *f = plain_inv_freq(base, D);
    oracle_decode_ex(q, k_cache, v_cache, offsets, seqlens, qpos, wq, f, 0, 1.0, eps, B, H, Hkv, D, out);
    free(f);
}

/* Number of threads the OpenMP runtime will use (reported beside the CPU timing). */
/* One decode step with the new token appended to the cache first.  [A] D2-3: the new
 * token's K and V go into the KV cache, and the token then attends to the whole cache;
 * [C] "Attention 的 Forward 流程": q and k are normed, then rotated, before attention.
 * Sequence b holds len_b = seqlens[b] >= 0 cached rows from row offsets[b] on (already
 * normed and rotated K, raw V).  Its new token brings raw q [H, D], k_new [Hkv, D] and
 * v_new [Hkv, D] (bf16 bits) and sits at position qpos[b] (default len_b).  The appended
 * key of KV head g is k-hat = RoPE(RMSNorm(k_new[g]; w_k), position), the appended value
 * is v_new[g] unchanged, and query head hq attends to the len_b cached rows of KV head
 * hq / (H/Hkv) followed by that appended row: len_b + 1 keys, none masked.  khat_out
 * [B, Hkv, D] receives the appended keys (fp64, before any storage rounding). */
void oracle_decode_append_ex(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                             const uint16_t *k_cache, const uint16_t *v_cache,
                             const int64_t *offsets, const int32_t *seqlens, const int32_t *qpos,
                             const float *wq, const float *wk, const double *inv_freq, int pairing,
                             double logit_mult, double eps, int B, int H, int Hkv, int D,
                             double *out, double *khat_out)
{
    int h_per_kv = H / Hkv;
    double inv_sqrt_d = logit_mult / sqrt((double)D);
    int32_t maxkeys = 1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] + 1 > maxkeys)
            maxkeys = seqlens[b] + 1;
    double *wqd = (double *)malloc(sizeof(double) * D);
    double *wkd = (double *)malloc(sizeof(double) * D);
    for (int d = 0; d < D; ++d) {
        wqd[d] = (double)wq[d];
        wkd[d] = (double)wk[d];
    }
    /* the appended keys first: one per (sequence, KV head) */
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
        for (int b = 0; b < B; ++b) {
            int32_t position = qpos ? qpos[b] : seqlens[b];
            for (int g = 0; g < Hkv; ++g)
                norm_then_rope(k_new + ((int64_t)b * Hkv + g) * D, wkd, position, inv_freq, pairing, eps, D,
                               tmp, khat_out + ((int64_t)b * Hkv + g) * D);
        }
        free(tmp);
    }
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
        double *qi = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * maxkeys);
        double *p = (double *)malloc(sizeof(double) * maxkeys);
        double *vbuf = (double *)malloc(sizeof(double) * (size_t)maxkeys * D);
        const double **vr = (const double **)malloc(sizeof(double *) * maxkeys);
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int b = 0; b < B; ++b)
            for (int hq = 0; hq < H; ++hq) {
                int g = hq / h_per_kv;
                int32_t len = seqlens[b];
                int32_t position = qpos ? qpos[b] : len;
                norm_then_rope(q + ((int64_t)b * H + hq) * D, wqd, position, inv_freq, pairing, eps, D, tmp,
                               qi);
                for (int32_t j = 0; j <= len; ++j) {
                    double dot = 0.0;
                    if (j < len) {
                        int64_t row = offsets[b] + j;
                        const uint16_t *kj = k_cache + (row * Hkv + g) * D;
                        const uint16_t *vj = v_cache + (row * Hkv + g) * D;
                        for (int d = 0; d < D; ++d) {
                            dot += qi[d] * bf16_bits_to_double(kj[d]);
                            vbuf[(int64_t)j * D + d] = bf16_bits_to_double(vj[d]);
                        }
                    } else {
                        const double *kj = khat_out + ((int64_t)b * Hkv + g) * D;
                        const uint16_t *vj = v_new + ((int64_t)b * Hkv + g) * D;
                        for (int d = 0; d < D; ++d) {
                            dot += qi[d] * kj[d];
                            vbuf[(int64_t)j * D + d] = bf16_bits_to_double(vj[d]);
                        }
                    }
                    s[j] = dot * inv_sqrt_d;
                    vr[j] = vbuf + (int64_t)j * D;
                }
                softmax_weighted_sum(s, len + 1, vr, D, p, out + ((int64_t)b * H + hq) * D);
            }
        free(tmp);
        free(qi);
        free(s);
        free(p);
        free(vbuf);
        free(vr);
    }
    free(wqd);
    free(wkd);
}

void oracle_decode_append(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                          const uint16_t *k_cache, const uint16_t *v_cache,
                          const int64_t *offsets, const int32_t *seqlens, const int32_t *qpos,
                          const float *wq, const float *wk, double base, double eps, int B,
                          int H, int Hkv, int D, double *out, double *khat_out)
{
    double *f = plain_inv_freq(base, D);
    oracle_decode_append_ex(q, k_new, v_new, k_cache, v_cache, offsets, seqlens, qpos, wq, wk, f, 0, 1.0,
                            eps, B, H, Hkv, D, out, khat_out);
    free(f);
}

/* One output row of the chunk: chunk row i of query head hq of sequence b against the
 * sequence's P_b cached rows (k-hat and v, from row offsets[b] on) and the chunk's k-hat
 * rows 0 .. i (khat [B, C, Hkv, D], already computed).  Scratch: tmp, qi [D]; s, p
 * [P_b + C]; vbuf [(P_b + C) * D]; vr [P_b + C]. */
static void chunk_one_row(const uint16_t *q, const uint16_t *v, const uint16_t *k_cache,
                          const uint16_t *v_cache, const int64_t *offsets, const int32_t *prefix_len,
                          const int32_t *pos, const double *wqd, const double *inv_freq, int pairing,
                          double inv_sqrt_d, double eps, int C, int H, int Hkv, int D, const double *khat,
                          int b, int hq, int i, double *tmp, double *qi, double *s, double *p, double *vbuf,
                          const double **vr, double *out_row)
{
    int g = hq / (H / Hkv);
    int32_t P = prefix_len[b];
    int64_t n = (int64_t)b * C + i;
    norm_then_rope(q + (n * H + hq) * D, wqd, pos[n], inv_freq, pairing, eps, D, tmp, qi);
    int nkeys = P + i + 1;
    for (int j = 0; j < nkeys; ++j) {
        double dot = 0.0;
        if (j < P) {
            int64_t row = offsets[b] + j;
            const uint16_t *kj = k_cache + (row * Hkv + g) * D;
            const uint16_t *vj = v_cache + (row * Hkv + g) * D;
            for (int d = 0; d < D; ++d) {
                dot += qi[d] * bf16_bits_to_double(kj[d]);
                vbuf[(int64_t)j * D + d] = bf16_bits_to_double(vj[d]);
            }
        } else {
            int64_t m = (int64_t)b * C + (j - P);
            const double *kj = khat + (m * Hkv + g) * D;
            const uint16_t *vj = v + (m * Hkv + g) * D;
            for (int d = 0; d < D; ++d) {
                dot += qi[d] * kj[d];
                vbuf[(int64_t)j * D + d] = bf16_bits_to_double(vj[d]);
            }
        }
        s[j] = dot * inv_sqrt_d;
        vr[j] = vbuf + (int64_t)j * D;
    }
    softmax_weighted_sum(s, nkeys, vr, D, p, out_row);
}

/* Chunked prefill against a cache prefix ([A] D2-3: a sequence's earlier tokens already
 * sit in the KV cache; [A] D1-5: the causal mask on the token index).  Sequence b has
 * P_b = prefix_len[b] cached rows (k-hat and v) from row offsets[b] on, and brings a
 * chunk of C new tokens: raw q [B, C, H, D], k and v [B, C, Hkv, D] (bf16 bits), at
 * positions pos [B, C].  Chunk row i of query head hq attends to the P_b cached rows of
 * KV head hq / (H/Hkv) and to the chunk's rows 0 .. i (token indices up to P_b + i).
 * The chunk's k-hat goes to khat_out [B, C, Hkv, D] (what a caller appends to the
 * cache).  With rows == NULL, out is [B, C, H, D], every row; else out is [nrows, D], the
 * rows (b, hq, i) listed in rows [nrows, 3]. */
static void prefill_chunk_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               const uint16_t *k_cache, const uint16_t *v_cache,
                               const int64_t *offsets, const int32_t *prefix_len, const int32_t *pos,
                               const float *wq, const float *wk, const double *inv_freq, int pairing,
                               double logit_mult, double eps, int B, int C, int H, int Hkv, int D,
                               int64_t nrows, const int64_t *rows, double *out, double *khat_out)
{
    double inv_sqrt_d = logit_mult / sqrt((double)D);
    int32_t maxkeys = 1;
    for (int b = 0; b < B; ++b)
        if (prefix_len[b] + C > maxkeys)
            maxkeys = prefix_len[b] + C;
    double *wqd = (double *)malloc(sizeof(double) * D);
    double *wkd = (double *)malloc(sizeof(double) * D);
    for (int d = 0; d < D; ++d) {
        wqd[d] = (double)wq[d];
        wkd[d] = (double)wk[d];
    }
    /* k-hat of the chunk's keys */
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
        for (int64_t n = 0; n < (int64_t)B * C; ++n)
            for (int g = 0; g < Hkv; ++g)
                norm_then_rope(k + (n * Hkv + g) * D, wkd, pos[n], inv_freq, pairing, eps, D, tmp,
                               khat_out + (n * Hkv + g) * D);
        free(tmp);
    }
    int64_t count = rows ? nrows : (int64_t)B * H * C;
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * D);
        double *qi = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * maxkeys);
        double *p = (double *)malloc(sizeof(double) * maxkeys);
        double *vbuf = (double *)malloc(sizeof(double) * (size_t)maxkeys * D);
        const double **vr = (const double **)malloc(sizeof(double *) * maxkeys);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < count; ++r) {
            int b, hq, i;
            double *dst;
            if (rows) {
                b = (int)rows[3 * r];
                hq = (int)rows[3 * r + 1];
                i = (int)rows[3 * r + 2];
                dst = out + r * D;
            } else {
                b = (int)(r / ((int64_t)H * C));
                hq = (int)(r / C % H);
                i = (int)(r % C);
                dst = out + (((int64_t)b * C + i) * H + hq) * D;
            }
            chunk_one_row(q, v, k_cache, v_cache, offsets, prefix_len, pos, wqd, inv_freq, pairing,
                          inv_sqrt_d, eps, C, H, Hkv, D, khat_out, b, hq, i, tmp, qi, s, p, vbuf, vr, dst);
        }
        free(tmp);
        free(qi);
        free(s);
        free(p);
        free(vbuf);
        free(vr);
    }
    free(wqd);
    free(wkd);
}

void oracle_prefill_chunk_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const uint16_t *k_cache, const uint16_t *v_cache,
                             const int64_t *offsets, const int32_t *prefix_len, const int32_t *pos,
                             const float *wq, const float *wk, const double *inv_freq, int pairing,
                             double logit_mult, double eps, int B, int C, int H, int Hkv, int D,
                             double *out, double *khat_out)
{
    prefill_chunk_impl(q, k, v, k_cache, v_cache, offsets, prefix_len, pos, wq, wk, inv_freq, pairing,
                       logit_mult, eps, B, C, H, Hkv, D, 0, NULL, out, khat_out);
}

/* The rows (b, hq, i) of oracle_prefill_chunk_ex listed in rows [nrows, 3] (for checks of
 * launches too large to compute whole); out [nrows, D], khat_out as there. */
void oracle_prefill_chunk_rows_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  const uint16_t *k_cache, const uint16_t *v_cache,
                                  const int64_t *offsets, const int32_t *prefix_len, const int32_t *pos,
                                  const float *wq, const float *wk, const double *inv_freq, int pairing,
                                  double logit_mult, double eps, int B, int C, int H, int Hkv, int D,
                                  int64_t nrows, const int64_t *rows, double *out, double *khat_out)
{
    prefill_chunk_impl(q, k, v, k_cache, v_cache, offsets, prefix_len, pos, wq, wk, inv_freq, pairing,
                       logit_mult, eps, B, C, H, Hkv, D, nrows, rows, out, khat_out);
}

/* Variable-length packed prefill: B sequences laid end to end, sequence b owning tokens
 * cu_seqlens[b] .. cu_seqlens[b+1]-1 of q [N, H, D], k and v [N, Hkv, D] (bf16 bits), with
 * positions pos [N].  Each token attends causally within its own sequence only ([A]
 * D1-5 per sequence); out is [N, H, D]. */
void oracle_prefill_varlen_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const int64_t *cu_seqlens, const int32_t *pos, const float *wq,
                              const float *wk, const double *inv_freq, int pairing,
                              double logit_mult, double eps, int B, int H, int Hkv, int D,
                              double *out)
{
    int h_per_kv = H / Hkv;
    double inv_sqrt_d = logit_mult / sqrt((double)D);
    int64_t N = cu_seqlens[B];
    int64_t maxlen = 1;
    for (int b = 0; b < B; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > maxlen)
            maxlen = cu_seqlens[b + 1] - cu_seqlens[b];
    double *qh = (double *)malloc(sizeof(double) * (size_t)(N * H * D + 1));
    double *kh = (double *)malloc(sizeof(double) * (size_t)(N * Hkv * D + 1));
    oracle_qk_transform_ex(q, pos, wq, inv_freq, pairing, eps, N, H, D, qh);
    oracle_qk_transform_ex(k, pos, wk, inv_freq, pairing, eps, N, Hkv, D, kh);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * maxlen);
        double *p = (double *)malloc(sizeof(double) * maxlen);
        double *vbuf = (double *)malloc(sizeof(double) * (size_t)maxlen * D);
        const double **vr = (const double **)malloc(sizeof(double *) * maxlen);
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < N; ++n) {
            int b = 0;
            while (cu_seqlens[b + 1] <= n)
                ++b;
            int64_t t0 = cu_seqlens[b];
            for (int hq = 0; hq < H; ++hq) {
                int g = hq / h_per_kv;
                const double *qi = qh + (n * H + hq) * D;
                int nkeys = (int)(n - t0 + 1);
                for (int j = 0; j < nkeys; ++j) {
                    const double *kj = kh + ((t0 + j) * Hkv + g) * D;
                    const uint16_t *vj = v + ((t0 + j) * Hkv + g) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) {
                        dot += qi[d] * kj[d];
                        vbuf[(int64_t)j * D + d] = bf16_bits_to_double(vj[d]);
                    }
                    s[j] = dot * inv_sqrt_d;
                    vr[j] = vbuf + (int64_t)j * D;
                }
                softmax_weighted_sum(s, nkeys, vr, D, p, out + (n * H + hq) * D);
            }
        }
        free(s);
        free(p);
        free(vbuf);
        free(vr);
    }
    free(qh);
    free(kh);
}

/* Linear projection without bias ([A] D1-2: a linear layer is Y = XW + b, and Qwen3's
 * projections carry no b; [B] 3.1.2: Qwen3 removed the QKV bias; [C] forward steps 1
 * and 7: the fused qkv_proj before the attention and o_proj after it, nn.Linear
 * semantics y = x W^T): y[m][n] = sum_k x[m][k] w[n][k].  x [M, K] and w [N, K] are bf16
 * bits, y [M, N] fp64, summed in the order k = 0 .. K-1. */
void oracle_linear(const uint16_t *x, const uint16_t *w, int64_t M, int64_t N, int64_t K, double *y)
{
#pragma omp parallel
    {
        double *xr = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t m = 0; m < M; ++m) {
            for (int64_t k = 0; k < K; ++k)
                xr[k] = bf16_bits_to_double(x[m * K + k]);
            for (int64_t n = 0; n < N; ++n) {
                const uint16_t *wr = w + n * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += xr[k] * bf16_bits_to_double(wr[k]);
                y[m * N + n] = acc;
            }
        }
        free(xr);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
