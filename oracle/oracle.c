/*
 * CPU oracle for QK4V8 mixed-precision attention (test infrastructure only).
 *
 * This file is test infrastructure. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it. The library path never calls it,
 * and it shares no code, header or table with the CUDA implementation.
 *
 * What it computes (MpFA QK4V8 article, mhpn.cn "MpFA免训练量化：QK4V8混合精度在
 * Blackwell上的推理加速实践"; MiMo FP4 article, wmrh.cn "MXFP4专家量化"):
 *  - Q and K are quantized to 4-bit, V to 8-bit (article §1.1, §2.1, §2.2).
 *  - Scales are computed per block of the data as it is quantized, without any
 *    calibration set (article §1.2, §3.2). The block is a group of 32 elements
 *    with one shared power-of-two scale (MiMo article, "MXFP4专家量化": one
 *    block scale per 32 values). This is OCP Microscaling (MX):
 *      E2M1 elements (max 6, emax 2) for Q and K, grouped along head_dim;
 *      E4M3 elements (max 448, emax 8) for V, grouped along the token axis;
 *      shared exponent X = floor(log2(amax)) - emax, stored as E8M0 (X + 127);
 *      element code = round-to-nearest-even(x / 2^X) onto the element grid,
 *      saturating at the largest finite magnitude.
 *  - Attention then uses the dequantized values (article §2.3, §3.3): scores
 *    s = scale * q.k, softmax over the allowed keys, output sum_j p_j v_j.
 *    Here everything after dequantization is done in fp64, which is the exact
 *    result up to rounding order.
 *
 * Readings taken where the articles are silent:
 *  - amax is the largest |x| of the group's valid elements (the article's
 *    "min/max" describes an asymmetric integer scheme; MX uses a symmetric
 *    amax). floor(log2 amax) comes from frexp, exactly. amax = 0 gives X = -127.
 *  - X is clamped to [-127, 127]; the E8M0 byte 0xFF is never produced.
 *  - A zero or a value that rounds to zero keeps the input's sign bit.
 *  - E2M1 codes are packed two per byte, element 2i in the low nibble.
 *  - V groups of 32 tokens: a trailing partial group takes its amax over the
 *    valid tokens only; codes past the valid length are 0, and scale bytes of
 *    groups with no valid token are 0.
 *  - Causal masking is bottom-right aligned: query i of Sq attends keys
 *    j <= i + (L - Sq), where L is that sequence's KV length.
 *  - GQA: query head h uses KV head h / (Hq / Hkv).
 *  - A row with no allowed key has output 0 and log-sum-exp -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_E2M1 0
#define ORACLE_E4M3 1

/* Number of magnitude codes (sign bit excluded) that are finite. */
static int n_finite_mags(int fmt) { return fmt == ORACLE_E2M1 ? 8 : 127; }
static int sign_bit(int fmt) { return fmt == ORACLE_E2M1 ? 0x8 : 0x80; }
static int elem_emax(int fmt) { return fmt == ORACLE_E2M1 ? 2 : 8; }

/* Value of a magnitude code, from the format definition:
 * E2M1: 2 exponent bits (bias 1), 1 mantissa bit, subnormal when the exponent is 0.
 * E4M3: 4 exponent bits (bias 7), 3 mantissa bits, subnormal when the exponent
 *       is 0; magnitude code 0x7F is NaN (OCP "FN" variant: no infinities). */
static double mag_value(int fmt, int m) {
    if (fmt == ORACLE_E2M1) {
        int e = (m >> 1) & 3, f = m & 1;
        if (e == 0) return f * 0.5;
        return (1.0 + f / 2.0) * ldexp(1.0, e - 1);
    } else {
        if (m == 0x7F) return NAN;
        int e = (m >> 3) & 15, f = m & 7;
        if (e == 0) return (f / 8.0) * ldexp(1.0, -6);
        return (1.0 + f / 8.0) * ldexp(1.0, e - 7);
    }
}

double oracle_decode(int fmt, int code) {
    int sb = sign_bit(fmt);
    double v = mag_value(fmt, code & (sb - 1));
    return (code & sb) ? -v : v;
}

/* Round y onto the element grid: nearest finite magnitude, ties to the code
 * with an even mantissa LSB (bit 0 of the code), magnitudes beyond the largest
 * finite value saturate to it. The sign bit is copied from y. */
int oracle_encode(int fmt, double y) {
    int sb = sign_bit(fmt);
    int neg = signbit(y) ? 1 : 0;
    double a = fabs(y);
    int nmag = n_finite_mags(fmt);
    int code;
    if (a >= mag_value(fmt, nmag - 1)) {
        code = nmag - 1;
    } else {
        /* largest magnitude code lo with value(lo) <= a (binary search). */
        int lo = 0, hi = nmag - 1;
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (mag_value(fmt, mid) <= a) lo = mid; else hi = mid;
        }
        double dlo = a - mag_value(fmt, lo);
        double dhi = mag_value(fmt, hi) - a;
        if (dlo < dhi) code = lo;
        else if (dhi < dlo) code = hi;
        else code = (lo & 1) ? hi : lo;
    }
    return code | (neg ? sb : 0);
}

/* Shared exponent X = floor(log2(amax)) - emax, clamped to [-127, 127]. */
int oracle_shared_exponent(int fmt, double amax) {
    if (!(amax > 0.0)) return -127;
    int e;
    frexp(amax, &e); /* amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e - 1 */
    int X = (e - 1) - elem_emax(fmt);
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    return X;
}

static inline double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/*
 * Quantize rows of bf16 values in groups of 32 along the row.
 * x       [n_rows][n_cols] bf16 bit patterns
 * valid   per-row number of valid leading elements (NULL: all n_cols)
 * codes   [n_rows][n_cols]   one element code per byte (unpacked)
 * scales  [n_rows][ceil(n_cols/32)] E8M0 bytes
 */
int oracle_quantize_rows(const uint16_t *x, int64_t n_rows, int64_t n_cols, const int32_t *valid,
                         int fmt, uint8_t *codes, uint8_t *scales) {
    if (!x || !codes || !scales || n_cols <= 0 || n_rows < 0) return -1;
    const int64_t ng = (n_cols + 31) / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint16_t *xr = x + r * n_cols;
        uint8_t *cr = codes + r * n_cols;
        uint8_t *sr = scales + r * ng;
        int64_t nv = valid ? (int64_t)valid[r] : n_cols;
        if (nv > n_cols) nv = n_cols;
        if (nv < 0) nv = 0;
        for (int64_t g = 0; g < ng; ++g) {
            int64_t c0 = g * 32, c1 = c0 + 32 < n_cols ? c0 + 32 : n_cols;
            int64_t cv = c1 < nv ? c1 : nv; /* valid end within the group */
            if (cv <= c0) {
                sr[g] = 0;
                for (int64_t c = c0; c < c1; ++c) cr[c] = 0;
                continue;
            }
            double amax = 0.0;
            for (int64_t c = c0; c < cv; ++c) {
                double a = fabs(bf16_to_double(xr[c]));
                if (a > amax) amax = a;
            }
            int X = oracle_shared_exponent(fmt, amax);
            sr[g] = (uint8_t)(X + 127);
            for (int64_t c = c0; c < cv; ++c) cr[c] = (uint8_t)oracle_encode(fmt, ldexp(bf16_to_double(xr[c]), -X));
            for (int64_t c = cv; c < c1; ++c) cr[c] = 0;
        }
    }
    return 0;
}

/* Two E2M1 codes per byte, element 2i in the low nibble; n must be even. */
int oracle_pack_e2m1(const uint8_t *codes, int64_t n, uint8_t *packed) {
    if (n % 2) return -1;
    for (int64_t i = 0; i < n / 2; ++i)
        packed[i] = (uint8_t)((codes[2 * i] & 0xF) | ((codes[2 * i + 1] & 0xF) << 4));
    return 0;
}

/* value = decode(code) * 2^(scale - 127) */
int oracle_dequantize_rows(const uint8_t *codes, const uint8_t *scales, int64_t n_rows, int64_t n_cols,
                           int fmt, double *out) {
    const int64_t ng = (n_cols + 31) / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int64_t c = 0; c < n_cols; ++c)
            out[r * n_cols + c] = ldexp(oracle_decode(fmt, codes[r * n_cols + c]), (int)scales[r * ng + c / 32] - 127);
    return 0;
}

/*
 * Keys visible to query row i (of Sq) of a sequence of L keys: lo <= j < hi.
 *   hi = L, or with causal = 1, min(L, i + (L - Sq) + 1): bottom-right
 *        alignment, so the Sq queries are the last Sq positions;
 *   lo = 0, or with window > 0, max(0, L - Sq - window): the draft-block
 *        attention of the MiMo DFlash article (section "DFlash块扩散推测解码")
 *        uses sliding-window attention over the most recent 1024 context
 *        tokens; the reading taken is that every row of the block sees the
 *        last `window` keys before the block and all keys of the block.
 */
static void visible_keys(int L, int Sq, int i, int causal, int window, int *lo, int *hi) {
    int h = L;
    if (causal) {
        int lim = i + (L - Sq) + 1;
        if (lim < h) h = lim;
    }
    if (h < 0) h = 0;
    int l = 0;
    if (window > 0) {
        l = L - Sq - window;
        if (l < 0) l = 0;
    }
    if (l > h) l = h;
    *lo = l;
    *hi = h;
}

/*
 * Attention over the dequantized tensors, in fp64.
 *
 * qc, qs  [B][Hq][Sq][d] codes, [B][Hq][Sq][d/32] scales   (E2M1)
 * kc, ks  [B][Hkv][Lk][d] codes, [B][Hkv][Lk][d/32] scales (E2M1)
 * vc, vs  [B][Hkv][d][Lk] codes, [B][Hkv][d][ceil(Lk/32)] scales, element
 *         format v_fmt: E4M3 (QK4V8), or E2M1 for the QK4V4 comparison point
 *         of the MpFA article (section 2.2: V at 4 bits costs about 0.8
 *         perplexity; section 5.3: a pitfall on long texts)
 * seqlens [B] KV length per sequence (NULL: Lk)
 * causal, window  the visible keys of each row (visible_keys above)
 * sel     [n_sel][3] rows (b, h_q, i) to compute; NULL computes every row in
 *         (b, i, h_q) order, n_sel = B*Sq*Hq
 * out     [n_sel][d]; lse [n_sel] natural-log log-sum-exp of the scaled scores
 */
int oracle_attention_window(const uint8_t *qc, const uint8_t *qs, const uint8_t *kc, const uint8_t *ks,
                            const uint8_t *vc, const uint8_t *vs, const int32_t *seqlens,
                            int B, int Hq, int Hkv, int Sq, int Lk, int d, int causal, int window, int v_fmt,
                            double scale, const int32_t *sel, int64_t n_sel, double *out, double *lse) {
    if (d % 32 || Hkv <= 0 || Hq % Hkv) return -1;
    const int G = Hq / Hkv;
    const int dg = d / 32;
    const int64_t lg = (Lk + 31) / 32;
    if (!sel) n_sel = (int64_t)B * Sq * Hq;
    /* Rows grouped by KV unit (b, h_kv) so each unit is dequantized once. */
    const int64_t n_units = (int64_t)B * Hkv;
    int64_t *cnt = (int64_t *)calloc((size_t)n_units + 1, sizeof(int64_t));
    int64_t *order = (int64_t *)malloc((size_t)(n_sel > 0 ? n_sel : 1) * sizeof(int64_t));
    if (!cnt || !order) { free(cnt); free(order); return -2; }
    for (int64_t r = 0; r < n_sel; ++r) {
        int b, h;
        if (sel) { b = sel[3 * r]; h = sel[3 * r + 1]; }
        else { b = (int)(r / ((int64_t)Sq * Hq)); h = (int)(r % Hq); }
        cnt[(int64_t)b * Hkv + h / G + 1]++;
    }
    for (int64_t u = 0; u < n_units; ++u) cnt[u + 1] += cnt[u];
    {
        int64_t *fillp = (int64_t *)malloc((size_t)n_units * sizeof(int64_t));
        if (!fillp) { free(cnt); free(order); return -2; }
        memcpy(fillp, cnt, (size_t)n_units * sizeof(int64_t));
        for (int64_t r = 0; r < n_sel; ++r) {
            int b, h;
            if (sel) { b = sel[3 * r]; h = sel[3 * r + 1]; }
            else { b = (int)(r / ((int64_t)Sq * Hq)); h = (int)(r % Hq); }
            order[fillp[(int64_t)b * Hkv + h / G]++] = r;
        }
        free(fillp);
    }
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < n_units; ++u) {
        if (cnt[u + 1] == cnt[u]) continue;
        const int b = (int)(u / Hkv);
        int L = seqlens ? seqlens[b] : Lk;
        if (L > Lk) L = Lk;
        if (L < 0) L = 0;
        double *kd = (double *)malloc((size_t)(L > 0 ? L : 1) * d * sizeof(double));
        double *vd = (double *)malloc((size_t)(L > 0 ? L : 1) * d * sizeof(double));
        double *qd = (double *)malloc((size_t)d * sizeof(double));
        double *p = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
        if (!kd || !vd || !qd || !p) {
#pragma omp atomic write
            err = -2;
            free(kd); free(vd); free(qd); free(p);
            continue;
        }
        const uint8_t *kcu = kc + (int64_t)u * Lk * d, *ksu = ks + (int64_t)u * Lk * dg;
        for (int j = 0; j < L; ++j)
            for (int c = 0; c < d; ++c)
                kd[(int64_t)j * d + c] = ldexp(oracle_decode(ORACLE_E2M1, kcu[(int64_t)j * d + c]),
                                               (int)ksu[(int64_t)j * dg + c / 32] - 127);
        const uint8_t *vcu = vc + (int64_t)u * d * Lk, *vsu = vs + (int64_t)u * d * lg;
        for (int c = 0; c < d; ++c)
            for (int j = 0; j < L; ++j)
                vd[(int64_t)j * d + c] = ldexp(oracle_decode(v_fmt, vcu[(int64_t)c * Lk + j]),
                                               (int)vsu[(int64_t)c * lg + j / 32] - 127);
        for (int64_t oi = cnt[u]; oi < cnt[u + 1]; ++oi) {
            const int64_t r = order[oi];
            int h, i;
            if (sel) { h = sel[3 * r + 1]; i = sel[3 * r + 2]; }
            else { i = (int)((r / Hq) % Sq); h = (int)(r % Hq); }
            const int64_t qrow = (((int64_t)b * Hq + h) * Sq + i);
            for (int c = 0; c < d; ++c)
                qd[c] = ldexp(oracle_decode(ORACLE_E2M1, qc[qrow * d + c]), (int)qs[qrow * dg + c / 32] - 127);
            int jmin, jmax; /* allowed keys: jmin <= j < jmax */
            visible_keys(L, Sq, i, causal, window, &jmin, &jmax);
            double *o = out + r * d;
            if (jmax <= jmin) {
                for (int c = 0; c < d; ++c) o[c] = 0.0;
                if (lse) lse[r] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int j = jmin; j < jmax; ++j) {
                double s = 0.0;
                const double *kr = kd + (int64_t)j * d;
                for (int c = 0; c < d; ++c) s += qd[c] * kr[c];
                s *= scale;
                p[j] = s;
                if (s > m) m = s;
            }
            double l = 0.0;
            for (int j = jmin; j < jmax; ++j) { p[j] = exp(p[j] - m); l += p[j]; }
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int j = jmin; j < jmax; ++j) {
                const double w = p[j] / l;
                const double *vr = vd + (int64_t)j * d;
                for (int c = 0; c < d; ++c) o[c] += w * vr[c];
            }
            if (lse) lse[r] = m + log(l);
        }
        free(kd); free(vd); free(qd); free(p);
    }
    free(cnt);
    free(order);
    return err;
}

/* oracle_attention_window with no window: every key up to the causal bound. */
int oracle_attention(const uint8_t *qc, const uint8_t *qs, const uint8_t *kc, const uint8_t *ks,
                     const uint8_t *vc, const uint8_t *vs, const int32_t *seqlens,
                     int B, int Hq, int Hkv, int Sq, int Lk, int d, int causal, double scale,
                     const int32_t *sel, int64_t n_sel, double *out, double *lse) {
    return oracle_attention_window(qc, qs, kc, ks, vc, vs, seqlens, B, Hq, Hkv, Sq, Lk, d, causal, 0, ORACLE_E4M3,
                                   scale, sel, n_sel, out, lse);
}

/*
 * Hadamard rotation of 128-channel rows before MXFP4 quantization.
 *
 * The MpFA article (section 3.1, and the outlier discussion of section 2.1)
 * expects outlier channels to be handled by a light rotation applied per group
 * before the 4-bit quantization. Q.K^T is unchanged by an orthonormal rotation
 * R applied to both Q and K, because (qR).(kR) = q R R^T k^T = q.k.
 * Reading taken: R = H / sqrt(128) with H the 128 x 128 Sylvester Hadamard
 * matrix, H[i][j] = (-1)^popcount(i & j), applied to each (token, head) row
 * of 128 channels, so that one outlier channel is spread over all four MX
 * groups of the row.
 *
 * The rotated values decide the quantized codes, so they are computed in the
 * precision the GPU kernel uses: fp32, as the fast Walsh-Hadamard transform
 * (butterfly stages of stride 1, 2, 4, ..., 64; each stage maps the pair
 * (a, b) at indices (i, i + stride) to (a + b, a - b)), then one fp32 multiply
 * by the fp32 value nearest to 2^-3.5 = 1/sqrt(128).
 * x  [n_rows][128] bf16 bit patterns;  y  [n_rows][128] fp32.
 */
#define ORACLE_RSQRT128_F32 0x1.6a09e6p-4f

int oracle_hadamard_rows(const uint16_t *x, int64_t n_rows, float *y) {
    if (!x || !y || n_rows < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        float *yr = y + r * 128;
        for (int c = 0; c < 128; ++c) {
            uint32_t u = (uint32_t)x[r * 128 + c] << 16;
            memcpy(&yr[c], &u, 4);
        }
        for (int stride = 1; stride < 128; stride *= 2)
            for (int i = 0; i < 128; ++i) {
                if (i & stride) continue;
                const float a = yr[i], b = yr[i + stride];
                yr[i] = a + b;
                yr[i + stride] = a - b;
            }
        for (int c = 0; c < 128; ++c) yr[c] = yr[c] * ORACLE_RSQRT128_F32;
    }
    return 0;
}

/*
 * oracle_quantize_rows for fp32 inputs (the rotated rows): the same OCP MX
 * rule, group amax, shared exponent and nearest-even encode, in fp64 on the
 * exact fp32 values.
 */
int oracle_quantize_rows_f32(const float *x, int64_t n_rows, int64_t n_cols, const int32_t *valid,
                             int fmt, uint8_t *codes, uint8_t *scales) {
    if (!x || !codes || !scales || n_cols <= 0 || n_rows < 0) return -1;
    const int64_t ng = (n_cols + 31) / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        const float *xr = x + r * n_cols;
        uint8_t *cr = codes + r * n_cols;
        uint8_t *sr = scales + r * ng;
        int64_t nv = valid ? (int64_t)valid[r] : n_cols;
        if (nv > n_cols) nv = n_cols;
        if (nv < 0) nv = 0;
        for (int64_t g = 0; g < ng; ++g) {
            int64_t c0 = g * 32, c1 = c0 + 32 < n_cols ? c0 + 32 : n_cols;
            int64_t cv = c1 < nv ? c1 : nv;
            if (cv <= c0) {
                sr[g] = 0;
                for (int64_t c = c0; c < c1; ++c) cr[c] = 0;
                continue;
            }
            double amax = 0.0;
            for (int64_t c = c0; c < cv; ++c) {
                double a = fabs((double)xr[c]);
                if (a > amax) amax = a;
            }
            int X = oracle_shared_exponent(fmt, amax);
            sr[g] = (uint8_t)(X + 127);
            for (int64_t c = c0; c < cv; ++c) cr[c] = (uint8_t)oracle_encode(fmt, ldexp((double)xr[c], -X));
            for (int64_t c = cv; c < c1; ++c) cr[c] = 0;
        }
    }
    return 0;
}

/*
 * Softmax attention over unquantized inputs, in fp64: the reference the
 * quantized method is compared against (the error against it is context, not
 * a pass/fail bar). Also the visible-key rule with a window, shared with
 * oracle_attention_window.
 *
 * q [B][Sq][Hq][d], k and v [B][Lk][Hkv][d], fp32 values (bf16 inputs are
 * exact in fp32). For sequence b of length L (seqlens, NULL: Lk) query row i
 * attends keys j with lo <= j < hi, where
 *   hi = L, or with causal = 1, min(L, i + (L - Sq) + 1) (bottom-right);
 *   lo = 0, or with window > 0, max(0, L - Sq - window): the last `window`
 *        keys before the query block, and every key of the block.
 * sel, out, lse as for oracle_attention.
 */
int oracle_attention_ref(const float *q, const float *k, const float *v, const int32_t *seqlens,
                         int B, int Hq, int Hkv, int Sq, int Lk, int d, int causal, int window, double scale,
                         const int32_t *sel, int64_t n_sel, double *out, double *lse) {
    if (Hkv <= 0 || Hq % Hkv || d <= 0) return -1;
    const int G = Hq / Hkv;
    if (!sel) n_sel = (int64_t)B * Sq * Hq;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_sel; ++r) {
        int b, h, i;
        if (sel) { b = sel[3 * r]; h = sel[3 * r + 1]; i = sel[3 * r + 2]; }
        else { b = (int)(r / ((int64_t)Sq * Hq)); i = (int)((r / Hq) % Sq); h = (int)(r % Hq); }
        int L = seqlens ? seqlens[b] : Lk;
        if (L > Lk) L = Lk;
        if (L < 0) L = 0;
        int lo, hi;
        visible_keys(L, Sq, i, causal, window, &lo, &hi);
        double *o = out + r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (hi <= lo) {
            if (lse) lse[r] = -INFINITY;
            continue;
        }
        double *p = (double *)malloc((size_t)(hi - lo) * sizeof(double));
        if (!p) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        const int hk = h / G;
        const float *qr = q + (((int64_t)b * Sq + i) * Hq + h) * d;
        double m = -INFINITY;
        for (int j = lo; j < hi; ++j) {
            const float *kr = k + (((int64_t)b * Lk + j) * Hkv + hk) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += (double)qr[c] * (double)kr[c];
            s *= scale;
            p[j - lo] = s;
            if (s > m) m = s;
        }
        double l = 0.0;
        for (int j = lo; j < hi; ++j) { p[j - lo] = exp(p[j - lo] - m); l += p[j - lo]; }
        for (int j = lo; j < hi; ++j) {
            const double w = p[j - lo] / l;
            const float *vr = v + (((int64_t)b * Lk + j) * Hkv + hk) * d;
            for (int c = 0; c < d; ++c) o[c] += w * (double)vr[c];
        }
        if (lse) lse[r] = m + log(l);
        free(p);
    }
    return err;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
