/*
 * Oracle for per-RoPE-wavelength windowed causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library: every quantity here is derived again from
 * the definition, in plain C, single-threaded, in IEEE double precision.
 *
 * What it computes (sources are the pages of the ATFlash / WavePrune papers):
 *
 *  - "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the RoPE
 *    attention score splits exactly into one term per 2-D rotation pair, and
 *    the window drops a pair's term once the query-key distance exceeds a
 *    length proportional to that pair's wavelength.  The window is a slice of
 *    the query-key contraction axis; the softmax itself is unchanged, so a
 *    dropped term contributes zero to the score (it is not a -inf mask).
 *  - "WavePrune: One period is often enough for RoPE", Original abstract:
 *    alpha = 1 keeps each pair inside its first rotation period; the kernel
 *    description there groups head dimensions in blocks of 16 (g = 8 pairs).
 *  - "The Heterogeneous Feature of RoPE-based Attention", Length
 *    Extrapolation formula: RoPE wavelengths have the form 2*pi*base^(2p/d).
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *  - pair p = dims (p, p + D/2) (half-split RoPE layout);
 *  - lambda_p = 2*pi * base^(2p/D);  T_p = floor(alpha * lambda_p) evaluated
 *    in double as  floor(alpha * ((2*pi) * pow(base, (2p)/D)));  pair p is kept
 *    at distance d iff d <= T_p (inclusive);  alpha = +inf disables the window;
 *  - g = 8: the 8 pairs {8m..8m+7} share the threshold of the group's
 *    longest wavelength, T_{8m+7} (the group stays while any member would);
 *  - d = q_pos - k_pos, keys with k_pos > q_pos are causally excluded;
 *  - scale multiplies the whole windowed score; lse is the natural log of
 *    sum_j exp(scale * s_j); a row without any causal key has out = 0 and
 *    lse = -inf.
 *
 * Every function returns 0 on success and a negative value on bad input.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_T_INF INT64_MAX
/* 2*pi rounded to the nearest double */
#define ORACLE_TWO_PI 6.28318530717958647692528676655900577

/* bf16 bit pattern -> double.  bf16 is the top half of an IEEE binary32. */
static double bf16_to_double(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Per-pair distance thresholds T_eff[p], p = 0 .. D/2-1 (ATFlash Abstract:
 * "wavelength-proportional distance"; WavePrune: first rotation period at
 * alpha = 1).  Also reports the smallest distance between alpha*lambda_p and
 * an integer, so a caller can refuse inputs whose floor sits on a tie.
 */
int oracle_thresholds(int D, double base, double alpha, int g,
                      int64_t *T_eff, double *min_tie_margin)
{
    if (D <= 0 || (D % 2) != 0 || !(base > 1.0) || !(alpha > 0.0)) return -1;
    if (g != 1 && g != 8) return -1;
    const int P = D / 2;
    if (g == 8 && (P % 8) != 0) return -1;
    int64_t T[4096];
    if (P > 4096) return -1;
    double margin = INFINITY;
    for (int p = 0; p < P; ++p) {
        if (isinf(alpha)) { T[p] = ORACLE_T_INF; continue; }
        double lambda = ORACLE_TWO_PI * pow(base, (double)(2 * p) / (double)D);
        double reach = alpha * lambda;
        double fl = floor(reach);
        double gap = fmin(reach - fl, fl + 1.0 - reach);
        if (gap < margin) margin = gap;
        T[p] = (reach >= 4.0e18) ? ORACLE_T_INF : (int64_t)fl;
    }
    for (int p = 0; p < P; ++p) {
        if (g == 1) {
            T_eff[p] = T[p];
        } else {
            /* thresholds grow with p, so the group's largest is its last */
            int64_t mx = T[p];
            for (int q = (p / 8) * 8; q < (p / 8) * 8 + 8; ++q)
                if (T[q] > mx) mx = T[q];
            T_eff[p] = mx;
        }
    }
    if (min_tie_margin) *min_tie_margin = margin;
    return 0;
}

/*
 * Windowed causal attention for an explicit list of query rows.
 *
 * q  : bf16 [B, Nq, Hq, D]     query t sits at position q_pos0 + t
 * k,v: bf16 [B, Nk, Hkv, D]    key j sits at position k_pos0 + j
 * kv_len: optional [B]; when given, batch b only has keys j < kv_len[b]
 * rows: nrows triples (b, h, t)
 * out: [nrows, D] double, lse: [nrows] double (natural log)
 *
 * Query head h reads kv head h / (Hq / Hkv).  The score of key j is
 *   s = sum_p [d <= T_eff[p]] * (q[p] k[p] + q[p+P] k[p+P]),   d = q_pos - k_pos
 * and the row is softmax(scale * s) . v over the causal keys (ATFlash
 * Abstract: the window slices the contraction, the softmax is untouched).
 */
int oracle_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int64_t *kv_len,
                          int B, int64_t Nq, int64_t Nk, int Hq, int Hkv, int D,
                          int64_t q_pos0, int64_t k_pos0,
                          double base, double alpha, int g, double scale,
                          int64_t nrows, const int64_t *rows,
                          double *out, double *lse)
{
    if (Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0 || B <= 0 || D <= 0) return -1;
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    const int group = Hq / Hkv;
    double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    if (!s) return -2;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= Nq) { free(s); return -1; }
        const int64_t kvh = h / group;
        const int64_t qpos = q_pos0 + t;
        const int64_t nkeys = kv_len ? kv_len[b] : Nk;
        const uint16_t *qr = q + ((b * Nq + t) * Hq + h) * (int64_t)D;
        double m = -INFINITY;
        int64_t used = 0;
        for (int64_t j = 0; j < nkeys; ++j) {
            const int64_t kpos = k_pos0 + j;
            if (kpos > qpos) { s[j] = NAN; continue; }
            const int64_t d = qpos - kpos;
            const uint16_t *kr = k + ((b * Nk + j) * Hkv + kvh) * (int64_t)D;
            double acc = 0.0;
            for (int p = 0; p < P; ++p) {
                if (d > T[p]) continue; /* pruned term: contributes 0 */
                acc += bf16_to_double(qr[p]) * bf16_to_double(kr[p]);
                acc += bf16_to_double(qr[p + P]) * bf16_to_double(kr[p + P]);
            }
            s[j] = scale * acc;
            if (s[j] > m) m = s[j];
            ++used;
        }
        double *o = out + r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        if (used == 0) { lse[r] = -INFINITY; continue; }
        double l = 0.0;
        for (int64_t j = 0; j < nkeys; ++j) {
            if (isnan(s[j])) continue;
            const double w = exp(s[j] - m);
            l += w;
            const uint16_t *vr = v + ((b * Nk + j) * Hkv + kvh) * (int64_t)D;
            for (int e = 0; e < D; ++e) o[e] += w * bf16_to_double(vr[e]);
        }
        for (int e = 0; e < D; ++e) o[e] /= l;
        lse[r] = m + log(l);
    }
    free(s);
    return 0;
}

/*
 * The same rows under a block mask (token-level block sparsity stacked on the
 * window; ATFlash Abstract: the window is orthogonal to token selection and
 * composes with it).  block_mask: uint8 [B, Hq, nqb, nkb]; key j of row t is
 * attended only if block_mask[b, h, t / block_q, j / block_k] != 0, on top of
 * causality; the window then applies to the attended keys as above.  A row
 * left with no key gets out = 0, lse = -inf.
 */
int oracle_attention_rows_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                 int B, int64_t Nq, int64_t Nk, int Hq, int Hkv, int D,
                                 int64_t q_pos0, int64_t k_pos0,
                                 double base, double alpha, int g, double scale,
                                 const uint8_t *block_mask, int64_t block_q, int64_t block_k,
                                 int64_t nrows, const int64_t *rows,
                                 double *out, double *lse)
{
    if (Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0 || B <= 0 || D <= 0) return -1;
    if (!block_mask || block_q <= 0 || block_k <= 0) return -1;
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    const int group = Hq / Hkv;
    const int64_t nqb = (Nq + block_q - 1) / block_q, nkb = (Nk + block_k - 1) / block_k;
    double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    if (!s) return -2;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= Nq) { free(s); return -1; }
        const int64_t kvh = h / group;
        const int64_t qpos = q_pos0 + t;
        const uint8_t *mrow = block_mask + ((b * Hq + h) * nqb + t / block_q) * nkb;
        const uint16_t *qr = q + ((b * Nq + t) * Hq + h) * (int64_t)D;
        double m = -INFINITY;
        int64_t used = 0;
        for (int64_t j = 0; j < Nk; ++j) {
            const int64_t kpos = k_pos0 + j;
            if (kpos > qpos || mrow[j / block_k] == 0) { s[j] = NAN; continue; }
            const int64_t d = qpos - kpos;
            const uint16_t *kr = k + ((b * Nk + j) * Hkv + kvh) * (int64_t)D;
            double acc = 0.0;
            for (int p = 0; p < P; ++p) {
                if (d > T[p]) continue; /* pruned term: contributes 0 */
                acc += bf16_to_double(qr[p]) * bf16_to_double(kr[p]);
                acc += bf16_to_double(qr[p + P]) * bf16_to_double(kr[p + P]);
            }
            s[j] = scale * acc;
            if (s[j] > m) m = s[j];
            ++used;
        }
        double *o = out + r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        if (used == 0) { lse[r] = -INFINITY; continue; }
        double l = 0.0;
        for (int64_t j = 0; j < Nk; ++j) {
            if (isnan(s[j])) continue;
            const double w = exp(s[j] - m);
            l += w;
            const uint16_t *vr = v + ((b * Nk + j) * Hkv + kvh) * (int64_t)D;
            for (int e = 0; e < D; ++e) o[e] += w * bf16_to_double(vr[e]);
        }
        for (int e = 0; e < D; ++e) o[e] /= l;
        lse[r] = m + log(l);
    }
    free(s);
    return 0;
}

/*
 * Prefill rows with explicit positions: query t of sequence b at
 * q_pos[b * q_stride + t], key j at k_pos[b * k_stride + j].  The same
 * definition as oracle_attention_rows with d = q_pos - k_pos; a key after its
 * query is excluded; a row with no key left gets out = 0, lse = -inf.
 * rows: nrows triples (b, h, t).
 */
int oracle_attention_positions(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               int B, int64_t Nq, int64_t Nk, int Hq, int Hkv, int D,
                               const int64_t *q_pos, int64_t q_stride,
                               const int64_t *k_pos, int64_t k_stride,
                               double base, double alpha, int g, double scale,
                               int64_t nrows, const int64_t *rows, double *out, double *lse)
{
    if (Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0 || B <= 0 || D <= 0) return -1;
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    const int group = Hq / Hkv;
    double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    if (!s) return -2;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= Nq) { free(s); return -1; }
        const int64_t kvh = h / group;
        const int64_t qpos = q_pos[b * q_stride + t];
        const uint16_t *qr = q + ((b * Nq + t) * Hq + h) * (int64_t)D;
        double m = -INFINITY;
        int64_t used = 0;
        for (int64_t j = 0; j < Nk; ++j) {
            const int64_t kpos = k_pos[b * k_stride + j];
            if (kpos > qpos) { s[j] = NAN; continue; }
            const int64_t d = qpos - kpos;
            const uint16_t *kr = k + ((b * Nk + j) * Hkv + kvh) * (int64_t)D;
            double acc = 0.0;
            for (int p = 0; p < P; ++p) {
                if (d > T[p]) continue; /* pruned term: contributes 0 */
                acc += bf16_to_double(qr[p]) * bf16_to_double(kr[p]);
                acc += bf16_to_double(qr[p + P]) * bf16_to_double(kr[p + P]);
            }
            s[j] = scale * acc;
            if (s[j] > m) m = s[j];
            ++used;
        }
        double *o = out + r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        if (used == 0) { lse[r] = -INFINITY; continue; }
        double l = 0.0;
        for (int64_t j = 0; j < Nk; ++j) {
            if (isnan(s[j])) continue;
            const double w = exp(s[j] - m);
            l += w;
            const uint16_t *vr = v + ((b * Nk + j) * Hkv + kvh) * (int64_t)D;
            for (int e = 0; e < D; ++e) o[e] += w * bf16_to_double(vr[e]);
        }
        for (int e = 0; e < D; ++e) o[e] /= l;
        lse[r] = m + log(l);
    }
    free(s);
    return 0;
}

/*
 * Decode with explicit positions (a serving cache whose keys are not at
 * positions 0..n-1: evicted or reordered tokens): sequence b has one query at
 * position q_pos[b] and keys j < kv_len[b] at positions
 * k_pos[b * kpos_stride + j].  The same definition as oracle_attention_rows:
 * d = q_pos - k_pos, pair p kept iff d <= T_eff[p], pruned terms are 0, a key
 * with k_pos > q_pos is causally excluded, softmax over the rest.
 * q: bf16 [B, Hq, D];  k, v: bf16 [B, Lmax, Hkv, D];  rows: nrows pairs (b, h)
 * out: [nrows, D] double, lse: [nrows] double (natural log).
 */
int oracle_decode_positions(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int64_t *kv_len, const int64_t *q_pos,
                            const int64_t *k_pos, int64_t kpos_stride,
                            int B, int64_t Lmax, int Hq, int Hkv, int D,
                            double base, double alpha, int g, double scale,
                            int64_t nrows, const int64_t *rows,
                            double *out, double *lse)
{
    if (Hkv <= 0 || Hq <= 0 || (Hq % Hkv) != 0 || B <= 0 || D <= 0) return -1;
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    const int group = Hq / Hkv;
    double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
    if (!s) return -2;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t b = rows[2 * r], h = rows[2 * r + 1];
        if (b < 0 || b >= B || h < 0 || h >= Hq || kv_len[b] < 0 || kv_len[b] > Lmax) {
            free(s);
            return -1;
        }
        const int64_t kvh = h / group;
        const int64_t qpos = q_pos[b];
        const uint16_t *qr = q + (b * Hq + h) * (int64_t)D;
        double m = -INFINITY;
        int64_t used = 0;
        for (int64_t j = 0; j < kv_len[b]; ++j) {
            const int64_t kpos = k_pos[b * kpos_stride + j];
            if (kpos > qpos) { s[j] = NAN; continue; }
            const int64_t d = qpos - kpos;
            const uint16_t *kr = k + ((b * Lmax + j) * Hkv + kvh) * (int64_t)D;
            double acc = 0.0;
            for (int p = 0; p < P; ++p) {
                if (d > T[p]) continue; /* pruned term: contributes 0 */
                acc += bf16_to_double(qr[p]) * bf16_to_double(kr[p]);
                acc += bf16_to_double(qr[p + P]) * bf16_to_double(kr[p + P]);
            }
            s[j] = scale * acc;
            if (s[j] > m) m = s[j];
            ++used;
        }
        double *o = out + r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        if (used == 0) { lse[r] = -INFINITY; continue; }
        double l = 0.0;
        for (int64_t j = 0; j < kv_len[b]; ++j) {
            if (isnan(s[j])) continue;
            const double w = exp(s[j] - m);
            l += w;
            const uint16_t *vr = v + ((b * Lmax + j) * Hkv + kvh) * (int64_t)D;
            for (int e = 0; e < D; ++e) o[e] += w * bf16_to_double(vr[e]);
        }
        for (int e = 0; e < D; ++e) o[e] /= l;
        lse[r] = m + log(l);
    }
    free(s);
    return 0;
}

/*
 * Round a double to bf16 bits, to nearest with ties to even, in one step from
 * the exact value (no intermediate float).  Values below the smallest normal
 * float go through a float first (their bf16 has fewer than 8 significant
 * bits); the inputs here never produce them except exact zeros.
 */
static uint16_t double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -126)) {
        float f = (float)x;
        uint32_t u;
        memcpy(&u, &f, 4);
        const uint32_t lsb = (u >> 16) & 1u;
        u += 0x7FFFu + lsb;
        return (uint16_t)(u >> 16);
    }
    int e;
    const double m = frexp(a, &e);              /* a = m * 2^e, m in [0.5, 1) */
    double r = nearbyint(ldexp(m, 8));          /* 8 significant bits, ties to even */
    const double y = ldexp(r, e - 8);
    if (y >= ldexp(1.0, 128)) return sign | 0x7F80;   /* overflow: inf */
    const float f = (float)y;                   /* exact: y has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

/*
 * RoPE (WavePrune, Original abstract: each 2-D channel of a query or key is
 * rotated at a channel-specific frequency, so logits depend on the position
 * difference only).  Pair p = dims (p, p + D/2) turns by pos * theta_p with
 * theta_p = base^(-2p/D) (the wavelength 2*pi*base^(2p/D) of the Length
 * Extrapolation formula):
 *   y_p       = x_p cos(a) - x_{p+D/2} sin(a)
 *   y_{p+D/2} = x_p sin(a) + x_{p+D/2} cos(a),   a = pos * theta_p.
 * x: bf16 [n, H, D] (token i at position pos[i]).  out_bf16 (optional): the
 * result rounded to bf16; out_f64 (optional): the exact double result.
 */
int oracle_rope(const uint16_t *x, const int64_t *pos, int64_t n, int H, int D, double base,
                uint16_t *out_bf16, double *out_f64)
{
    if (n < 0 || H <= 0 || D <= 0 || (D % 2) != 0 || !(base > 1.0)) return -1;
    const int P = D / 2;
    for (int64_t i = 0; i < n; ++i) {
        for (int h = 0; h < H; ++h) {
            const uint16_t *xr = x + (i * H + h) * (int64_t)D;
            for (int p = 0; p < P; ++p) {
                const double theta = pow(base, -(2.0 * p) / D);
                const double a = (double)pos[i] * theta;
                const double c = cos(a), sn = sin(a);
                const double x0 = bf16_to_double(xr[p]), x1 = bf16_to_double(xr[p + P]);
                const double y0 = x0 * c - x1 * sn;
                const double y1 = x0 * sn + x1 * c;
                const int64_t o = (i * H + h) * (int64_t)D;
                if (out_f64) { out_f64[o + p] = y0; out_f64[o + p + P] = y1; }
                if (out_bf16) { out_bf16[o + p] = double_to_bf16(y0); out_bf16[o + p + P] = double_to_bf16(y1); }
            }
        }
    }
    return 0;
}

/*
 * Windowed scores (before scale) of one query row against keys [0, nkeys):
 * used by tests that check the score formula itself on hand-worked inputs.
 * Causally excluded keys get NaN.
 */
int oracle_scores(const uint16_t *qrow, const uint16_t *keys, int64_t nkeys, int D,
                  int64_t q_pos, int64_t k_pos0,
                  double base, double alpha, int g, double *scores)
{
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    for (int64_t j = 0; j < nkeys; ++j) {
        const int64_t kpos = k_pos0 + j;
        if (kpos > q_pos) { scores[j] = NAN; continue; }
        const int64_t d = q_pos - kpos;
        const uint16_t *kr = keys + j * (int64_t)D;
        double acc = 0.0;
        for (int p = 0; p < P; ++p) {
            if (d > T[p]) continue;
            acc += bf16_to_double(qrow[p]) * bf16_to_double(kr[p]);
            acc += bf16_to_double(qrow[p + P]) * bf16_to_double(kr[p + P]);
        }
        scores[j] = acc;
    }
    return 0;
}

/*
 * Pair-terms of one (batch, head): every causal (query, key) pair counts
 * D/2 terms; a term is pruned when its distance exceeds the pair's threshold.
 * Brute force: enumerate every (row, key, pair).  Only for tiny sizes.
 */
int oracle_count_bruteforce(int D, double base, double alpha, int g,
                            int64_t Nq, int64_t Nk, int64_t q_pos0, int64_t k_pos0,
                            uint64_t *pruned, uint64_t *total)
{
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    uint64_t pr = 0, tot = 0;
    for (int64_t t = 0; t < Nq; ++t) {
        const int64_t qpos = q_pos0 + t;
        for (int64_t j = 0; j < Nk; ++j) {
            const int64_t kpos = k_pos0 + j;
            if (kpos > qpos) continue;
            const int64_t d = qpos - kpos;
            for (int p = 0; p < P; ++p) {
                ++tot;
                if (d > T[p]) ++pr;
            }
        }
    }
    *pruned = pr;
    *total = tot;
    return 0;
}

/*
 * Same count, one query row at a time: row i sees distances
 * [max(0, i - last_key_pos), i - k_pos0], and pair p keeps the distances of
 * that range that are <= T_p.  O(Nq * D) instead of O(Nq * Nk * D).
 */
int oracle_count_rows(int D, double base, double alpha, int g,
                      int64_t Nq, int64_t Nk, int64_t q_pos0, int64_t k_pos0,
                      uint64_t *pruned, uint64_t *total)
{
    const int P = D / 2;
    int64_t T[4096];
    if (oracle_thresholds(D, base, alpha, g, T, NULL) != 0) return -1;
    uint64_t kept = 0, tot = 0;
    const int64_t last_kpos = k_pos0 + Nk - 1;
    for (int64_t t = 0; t < Nq; ++t) {
        const int64_t qpos = q_pos0 + t;
        if (Nk <= 0 || qpos < k_pos0) continue;
        const int64_t dlo = qpos > last_kpos ? qpos - last_kpos : 0;
        const int64_t dhi = qpos - k_pos0;
        tot += (uint64_t)(dhi - dlo + 1) * (uint64_t)P;
        for (int p = 0; p < P; ++p) {
            const int64_t top = T[p] < dhi ? T[p] : dhi;
            if (top >= dlo) kept += (uint64_t)(top - dlo + 1);
        }
    }
    *pruned = tot - kept;
    *total = tot;
    return 0;
}
