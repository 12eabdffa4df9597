/*
 * fqa_oracle.c -- plain, slow CPU checker for the FP8 quantized attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline / reference arm use it.  It shares no code, header,
 * table or constant with the CUDA library.
 *
 * What it computes (sources, by page title and section):
 *  - Scaled dot-product attention with Q, K and V quantized to FP8, attention
 *    kept in FP8 for numerical stability: "NVIDIA RTX AI optimiert FLUX.1 fuer
 *    Bilddaten mit niedriger Genauigkeit" (the SDPA quantization paragraph and
 *    the Table-1 paragraph) and "NVIDIA RTX AI, 저정밀 양자화로 FLUX.1 Kontext
 *    최적화" (the SDPA paragraph).  SageAttention is named there as the lineage.
 *  - The pages fix no scale granularity, smoothing, rounding or P rule.  This
 *    file follows the readings stated beside each function: per-64-token-block
 *    per-head absmax scales onto the E4M3 maximum 448, K smoothed by its
 *    per-channel mean, KV tiles of Bc keys in ascending order with an exact
 *    running maximum, P = E4M3(p * 448 * sv_J / sv_max), row sum of the
 *    unquantized p, output scaled by sv_max / 448 / l.
 *
 * Precision: the quantizer runs in IEEE binary32 in a pinned operation order
 * (compile with -ffp-contract=off, no fast-math) so that codes and scales are
 * exact; attention runs in binary64 with roundings only at the pinned
 * quantization points.  E4M3 follows the OCP 8-bit floating point
 * specification (E4M3: bias 7, no infinities, NaN = S.1111.111, largest finite
 * 448, subnormal step 2^-9); BF16 output rounding is round-to-nearest-even.
 *
 * Multithreaded with OpenMP over independent heads / query rows only; each
 * result is computed by one thread in the order written here.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define ORC_E4M3_MAX 448.0

/* ---------------------------------------------------------------- codecs */

/* OCP E4M3: value of an 8-bit code. NaN codes (S.1111.111) return NaN. */
double orc_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);              /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* OCP E4M3, round to nearest (ties to even), saturating to +-448.
 * x must not be NaN.  The sign of zero is kept (-0 -> 0x80). */
uint8_t orc_e4m3_encode(double x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= ORC_E4M3_MAX)                       /* includes +inf */
        return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: multiples of 2^-9; q = 8 is the smallest normal,
         * whose encoding (exponent field 1, mantissa 0) is also 8. */
        double q = nearbyint(a * 512.0);
        return sign | (uint8_t)q;
    }
    int e;
    frexp(a, &e);                                /* a = f * 2^e, 0.5 <= f < 1 */
    e -= 1;                                      /* a in [2^e, 2^(e+1)) */
    double q = nearbyint(ldexp(a, 3 - e));       /* in [8, 16] */
    if (q == 16.0) { q = 8.0; e += 1; }
    if (e > 8 || (e == 8 && q > 14.0))           /* rounded above 448 */
        return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)q - 8));
}

/* BF16 bit pattern -> float (exact). */
float orc_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary64 -> BF16, one round to nearest even (finite, normal-range inputs;
 * subnormal results are rounded on the same 2^-133 grid). */
uint16_t orc_bf16_round(double x)
{
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    int e;
    double f = frexp(x, &e);                     /* 0.5 <= |f| < 1 */
    if (e < -125) {                              /* below the normal range */
        double q = nearbyint(ldexp(x, 133));
        float r = (float)ldexp(q, -133);
        uint32_t u; memcpy(&u, &r, 4);
        return (uint16_t)(u >> 16);
    }
    double q = nearbyint(f * 256.0);             /* 8 significant bits */
    float r = (float)ldexp(q, e - 8);            /* exact */
    uint32_t u; memcpy(&u, &r, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------- quantizer */

#define IDX4(b, h, n, c, H, N, d) ((((size_t)(b) * (H) + (h)) * (N) + (n)) * (d) + (c))

/* K per-channel mean, pinned order [reading: the pages give no summation
 * order]: p_j[c] = ((0 + k[64j][c]) + k[64j+1][c]) + ... in binary32 over the
 * tokens of block j (64 of them; the last block of a sequence whose length is
 * not a multiple of 64 holds the remaining N - 64*(nblk-1)); T[c] =
 * ((0 + p_0[c]) + p_1[c]) + ... over blocks; mu[c] = T[c] / (float)N, one
 * binary32 division. */
void orc_k_mean(const uint16_t *k, int B, int H, int N, int d, float *mu)
{
    int nblk = (N + 63) / 64;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            for (int c = 0; c < d; c++) {
                float T = 0.0f;
                for (int j = 0; j < nblk; j++) {
                    float p = 0.0f;
                    int n1 = 64 * j + 64 < N ? 64 * j + 64 : N;
                    for (int n = 64 * j; n < n1; n++)
                        p = p + orc_bf16_to_float(k[IDX4(b, h, n, c, H, N, d)]);
                    T = T + p;
                }
                mu[((size_t)b * H + h) * d + c] = T / (float)N;
            }
}

/* One block of one head (n_tok tokens, at most 64): absmax scale onto 448
 * and E4M3 codes.  x[n*d + c] are the binary32 values to quantize.
 * Readings: s = amax/448 and inv = 448/amax as binary32 divisions; amax == 0
 * gives s = inv = 0; the code is E4M3_RNE_sat(fl32(x * inv)) -- the product
 * is rounded to binary32 first, then encoded.
 * Two regimes of tiny blocks, on which the pages are silent:
 *  - 448/amax overflows binary32 (amax below about 1.3e-36; BF16 inputs can
 *    hold such values): inv = +inf would turn the block's zeros into
 *    0 * inf = NaN.  The reading keeps the intent, amax onto 448, by dividing
 *    instead: code = E4M3_RNE_sat(fl32(x / s)).
 *  - amax / 448 underflows to s = 0 (amax below about 3e-43; only smoothed K,
 *    whose binary32 differences can be subnormal, gets there): the block is
 *    flushed, inv = 0, so every code is a signed zero, as for amax == 0. */
static void quantize_block(const float *x, int n_tok, int d, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (int i = 0; i < n_tok * d; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s = 0.0f, inv = 0.0f;
    if (amax > 0.0f) {
        s = amax / 448.0f;
        inv = 448.0f / amax;
        if (s == 0.0f)
            inv = 0.0f;
    }
    int divide = isinf(inv);
    for (int i = 0; i < n_tok * d; i++) {
        float y = divide ? x[i] / s : x[i] * inv;
        codes[i] = orc_e4m3_encode((double)y);
    }
    *scale = s;
}

/* The whole quantizer.  Inputs BF16 [B,H,N,d], any N >= 1; codes written in
 * the same natural [B,H,N,d] layout (the CUDA library's own V layout is its
 * business); sq, sk, sv: [B,H,ceil(N/64)]; sv_max: [B,H]; k_mean: [B,H,d].
 * K is smoothed as fl32(k - mu[c]) before its block scales are taken.
 * [reading] When N is not a multiple of 64 the last block of each head holds
 * the remaining tokens and its scale is the absmax of those tokens alone. */
void orc_quantize(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  int B, int H, int N, int d,
                  uint8_t *q8, uint8_t *k8, uint8_t *v8,
                  float *sq, float *sk, float *sv, float *sv_max, float *k_mean)
{
    int nblk = (N + 63) / 64;
    orc_k_mean(k, B, H, N, d, k_mean);
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++) {
            float *x = (float *)malloc(sizeof(float) * 64 * d);
            const float *mu = k_mean + ((size_t)b * H + h) * d;
            float vmax = 0.0f;
            for (int j = 0; j < nblk; j++) {
                int nt = N - 64 * j < 64 ? N - 64 * j : 64;
                size_t base = IDX4(b, h, 64 * j, 0, H, N, d);
                size_t sidx = ((size_t)b * H + h) * nblk + j;
                for (int i = 0; i < nt * d; i++)
                    x[i] = orc_bf16_to_float(q[base + i]);
                quantize_block(x, nt, d, q8 + base, &sq[sidx]);
                for (int i = 0; i < nt * d; i++)
                    x[i] = orc_bf16_to_float(k[base + i]) - mu[i % d];
                quantize_block(x, nt, d, k8 + base, &sk[sidx]);
                for (int i = 0; i < nt * d; i++)
                    x[i] = orc_bf16_to_float(v[base + i]);
                quantize_block(x, nt, d, v8 + base, &sv[sidx]);
                if (sv[sidx] > vmax) vmax = sv[sidx];
            }
            sv_max[(size_t)b * H + h] = vmax;
            free(x);
        }
}

/* ------------------------------------------------------------- attention */

/* Tiled attention core in binary64 for one head, on already dequantized
 * operands: qc [N,d], kc [N,d], vc [N,d] are the code VALUES (not yet
 * multiplied by their block scales), sq/sk/sv the per-64-token scales.
 *
 * For query row i (block I = i/64), KV tiles t of bc keys in ascending order
 * (when bc does not divide N, the last tile holds the remaining keys; there
 * are no keys beyond N to mask):
 *   x_ij   = (sum_c qc_ic kc_jc) * sq_I * sk_J * scale * log2(e)
 *   m_t    = max(m_{t-1}, max_{j in t} x_ij),  m_{-1} = -inf  (exact, no
 *            threshold / lazy rescale)
 *   p_ij   = 2^(x_ij - m_t)
 *   P_ij   = E4M3(p_ij * 448 * sv_J / sv_max)    [quantize_p != 0]
 *          = p_ij * 448 * sv_J / sv_max          [quantize_p == 0]
 *   l      = l * 2^(m_{t-1} - m_t) + sum_j p_ij   (unquantized p)
 *   acc_c  = acc_c * 2^(m_{t-1} - m_t) + sum_j P_ij vc_jc
 *   O_ic   = acc_c * (sv_max / 448) / l
 * sv_max == 0 (V entirely zero) gives O = 0.
 * rows: the query rows of this head to evaluate; out: [n_rows, d].
 * amb (optional, [n_rows, d]): bound on |O - O'| over every O' whose P codes
 * differ from these only where a binary32 evaluation of p * 448 * rv can fall
 * on the other side of an E4M3 rounding midpoint (see p_eval_bound); namb
 * (optional, [n_rows]): how many P codes of the row are such. */
/* Relative error bound of a binary32 evaluation of one P value p * 448 * rv
 * (before E4M3 rounding), used to flag P codes that a kernel working in
 * binary32 may legitimately round the other way.  Sources: the FP32
 * accumulation of the 128 code products (2^-22 of their magnitude sum), the
 * binary32 roundings of the score, its scale and the running maximum
 * (2^-22 of |x| + 2|m|, in log2 units), the hardware exp2 approximation
 * (2^-21 relative) and the final products (2^-22). */
static double p_eval_bound(double abs_prod_sum, double a, double x, double m)
{
    const double LN2 = 0.69314718055994530942;
    double dx = ldexp(a * abs_prod_sum + fabs(x) + 2.0 * fabs(m), -22);
    return LN2 * dx + ldexp(1.0, -21) + ldexp(1.0, -22);
}

/* skip (optional, [N]): keys with skip[j] != 0 take no part in the rule (no
 * maximum, p, row-sum term or P code) -- the keys an error-corrected pass
 * handles exactly; a tile with none left changes nothing.  m_out, l_out
 * (optional, [n_rows]): the final running maximum and row sum (l = 0 when
 * every key is skipped; the output row is then 0). */
static void attention_core_head(const double *qc, const double *kc, const double *vc,
                                const float *sq, const float *sk, const float *sv, float sv_max,
                                int N, int d, double scale, int bc, int quantize_p,
                                const int *rows, int n_rows, double *out,
                                double *amb, int *namb, const uint8_t *skip,
                                double *m_out, double *l_out)
{
    const double LOG2E = 1.4426950408889634073599246810019;  /* log2(e) */
    #pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < n_rows; r++) {
        int i = rows[r];
        double *o = out + (size_t)r * d;
        double *x = (double *)malloc(sizeof(double) * bc);
        double *aps = (double *)malloc(sizeof(double) * bc);
        double *acc = (double *)calloc(d, sizeof(double));
        double *aacc = (double *)calloc(d, sizeof(double));
        double m = -INFINITY, l = 0.0;
        int n_amb = 0;
        if (sv_max == 0.0f) {
            for (int c = 0; c < d; c++) o[c] = 0.0;
            if (amb) for (int c = 0; c < d; c++) amb[(size_t)r * d + c] = 0.0;
            if (namb) namb[r] = 0;
            if (m_out) m_out[r] = 0.0;           /* V is all zero: any weight gives 0 */
            if (l_out) l_out[r] = 1.0;
            free(x); free(aps); free(acc); free(aacc);
            continue;
        }
        for (int t0 = 0; t0 < N; t0 += bc) {
            int t1 = t0 + bc < N ? t0 + bc : N;
            double tmax = -INFINITY;
            for (int j = t0; j < t1; j++) {
                double s = 0.0, sa = 0.0;
                if (skip && skip[j]) {
                    x[j - t0] = -INFINITY;
                    aps[j - t0] = 0.0;
                    continue;
                }
                for (int c = 0; c < d; c++) {
                    double pr = qc[(size_t)i * d + c] * kc[(size_t)j * d + c];
                    s += pr;
                    sa += fabs(pr);
                }
                x[j - t0] = s * (double)sq[i / 64] * (double)sk[j / 64] * scale * LOG2E;
                aps[j - t0] = sa;
                if (x[j - t0] > tmax) tmax = x[j - t0];
            }
            double m_new = tmax > m ? tmax : m;
            if (m_new == -INFINITY)              /* no key yet: nothing to do */
                continue;
            double alpha = exp2(m - m_new);      /* 0 on the first tile */
            l *= alpha;
            for (int c = 0; c < d; c++) acc[c] *= alpha;
            for (int c = 0; c < d; c++) aacc[c] *= alpha;
            for (int j = t0; j < t1; j++) {
                if (skip && skip[j])
                    continue;
                double p = exp2(x[j - t0] - m_new);
                double rv = (double)sv[j / 64] / (double)sv_max;
                double P = p * 448.0 * rv;
                if (quantize_p) {
                    double Pv = P;
                    uint8_t code = orc_e4m3_encode(Pv);
                    P = orc_e4m3_decode(code);
                    if (amb || namb) {
                        /* both neighbours of a rounding midpoint are valid codes
                         * when the binary32 evaluation can cross it */
                        double a = (double)sq[i / 64] * (double)sk[j / 64] * scale * LOG2E;
                        double eta = p_eval_bound(aps[j - t0], a, x[j - t0], m_new);
                        uint8_t lo = orc_e4m3_encode(Pv * (1.0 - eta));
                        uint8_t hi = orc_e4m3_encode(Pv * (1.0 + eta));
                        if (lo != code || hi != code) {
                            double dP = fmax(fabs(orc_e4m3_decode(lo) - P),
                                             fabs(orc_e4m3_decode(hi) - P));
                            n_amb++;
                            for (int c = 0; c < d; c++)
                                aacc[c] += dP * fabs(vc[(size_t)j * d + c]);
                        }
                    }
                }
                l += p;
                for (int c = 0; c < d; c++)
                    acc[c] += P * vc[(size_t)j * d + c];
            }
            m = m_new;
        }
        for (int c = 0; c < d; c++)
            o[c] = l > 0.0 ? acc[c] * ((double)sv_max / 448.0) / l : 0.0;
        if (amb)
            for (int c = 0; c < d; c++)
                amb[(size_t)r * d + c] = l > 0.0 ? aacc[c] * ((double)sv_max / 448.0) / l : 0.0;
        if (namb) namb[r] = n_amb;
        if (m_out) m_out[r] = m;
        if (l_out) l_out[r] = l;
        free(x);
        free(aps);
        free(acc);
        free(aacc);
    }
}

/* Exported core for the pins: operands given as binary64 values. */
void orc_attention_core(const double *qc, const double *kc, const double *vc,
                        const float *sq, const float *sk, const float *sv, float sv_max,
                        int N, int d, double scale, int bc, int quantize_p,
                        const int *rows, int n_rows, double *out, double *amb, int *namb)
{
    attention_core_head(qc, kc, vc, sq, sk, sv, sv_max, N, d, scale, bc, quantize_p,
                        rows, n_rows, out, amb, namb, NULL, NULL, NULL);
}

/* FP8 attention on quantizer outputs (codes in natural [B,H,N,d] layout).
 * heads: n_heads pairs (b, h); rows: n_rows query rows evaluated in every
 * listed head; out: [n_heads, n_rows, d] binary64. */
void orc_attention_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8,
                       const float *sq, const float *sk, const float *sv, const float *sv_max,
                       int B, int H, int N, int d, float softmax_scale, int bc,
                       const int *heads, int n_heads, const int *rows, int n_rows,
                       double *out, double *amb, int *namb)
{
    int nblk = (N + 63) / 64;
    (void)B;
    double *qc = (double *)malloc(sizeof(double) * N * d);
    double *kc = (double *)malloc(sizeof(double) * N * d);
    double *vc = (double *)malloc(sizeof(double) * N * d);
    double dec[256];
    for (int i = 0; i < 256; i++) dec[i] = orc_e4m3_decode((uint8_t)i);
    for (int hh = 0; hh < n_heads; hh++) {
        int b = heads[2 * hh], h = heads[2 * hh + 1];
        size_t base = IDX4(b, h, 0, 0, H, N, d);
        for (size_t i = 0; i < (size_t)N * d; i++) {
            qc[i] = dec[q8[base + i]];
            kc[i] = dec[k8[base + i]];
            vc[i] = dec[v8[base + i]];
        }
        size_t sidx = ((size_t)b * H + h) * nblk;
        attention_core_head(qc, kc, vc, sq + sidx, sk + sidx, sv + sidx,
                            sv_max[(size_t)b * H + h], N, d, (double)softmax_scale, bc, 1,
                            rows, n_rows, out + (size_t)hh * n_rows * d,
                            amb ? amb + (size_t)hh * n_rows * d : NULL,
                            namb ? namb + (size_t)hh * n_rows : NULL, NULL, NULL, NULL);
    }
    free(qc); free(kc); free(vc);
}

/* ------------------------------------------------- NVFP4 Q and K (FP4) */
/* The FP4 scheme: "NVIDIA RTX AI optimiert FLUX.1 fuer Bilddaten mit
 * niedriger Genauigkeit", SDPA quantization paragraph (the FP8 and FP4
 * schemes differ only in the precision of the Q, K, V projections; attention
 * itself stays in FP8).  The pages name no FP4 format; the reading is NVFP4
 * for the Q and K operands of Q K^T -- E2M1 elements with one unsigned E4M3
 * scale per 16 consecutive channels -- on top of the FP8 path's per-(b, h,
 * 64-token block) FP32 scale; V, P and P.V stay FP8. */

/* E2M1 value of a 4-bit code: sign in bit 3, exponent bits [1,3) (bias 1),
 * mantissa bit 0; subnormal 0.5 for exponent 0.  Values 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6. */
double orc_e2m1_decode(uint8_t code)
{
    int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -v : v;
}

/* E2M1, round to nearest (ties to the even code), saturating to +-6; the
 * sign of zero is kept.  x must not be NaN.  Nearest-even over the table. */
uint8_t orc_e2m1_encode(double x)
{
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs(x);
    if (a >= 6.0)
        return sign | 7;
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; c++) {
        double dlt = fabs(orc_e2m1_decode((uint8_t)c) - a);
        if (dlt < bd || (dlt == bd && (c & 1) == 0 && (best & 1) == 1)) {
            bd = dlt;
            best = c;
        }
    }
    return sign | (uint8_t)best;
}

/* One block (n_tok tokens x d channels, x binary32, K already smoothed) in
 * NVFP4 [reading, pinned binary32 order]:
 *   s1  = fl32(amax / 2688)          (6 * 448: the largest group scale is 448)
 *   per token and 16-channel group g: den = fl32(s1 * 6), t = fl32(amax_g / den),
 *   s2  = E4M3(t)  (unsigned, round to nearest even, saturating at 448)
 *   dg  = fl32(s1 * dec(s2)),  code = E2M1(fl32(x / dg))   (0 when dg = 0)
 * amax == 0, or s1 underflowing to 0, flushes the block (s1 = 0, every s2
 * and code 0).  codes: [n_tok][d/2] bytes, element 2i in the low nibble;
 * sf: [n_tok][d/16] E4M3 bytes. */
static void quantize_block_nvfp4(const float *x, int n_tok, int d, uint8_t *codes, uint8_t *sf,
                                 float *s1_out)
{
    float amax = 0.0f;
    for (int i = 0; i < n_tok * d; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s1 = amax > 0.0f ? amax / 2688.0f : 0.0f;
    for (int n = 0; n < n_tok; n++)
        for (int g = 0; g < d / 16; g++) {
            const float *xg = x + (size_t)n * d + 16 * g;
            float ag = 0.0f;
            for (int c = 0; c < 16; c++) {
                float a = fabsf(xg[c]);
                if (a > ag) ag = a;
            }
            uint8_t s2 = 0;
            float dg = 0.0f;
            if (s1 > 0.0f) {
                float den = s1 * 6.0f;
                float t = ag / den;
                s2 = orc_e4m3_encode((double)t);
                dg = s1 * (float)orc_e4m3_decode(s2);
            }
            sf[(size_t)n * (d / 16) + g] = s2;
            for (int c = 0; c < 16; c += 2) {
                uint8_t lo = 0, hi = 0;
                if (dg > 0.0f) {
                    float y0 = xg[c] / dg, y1 = xg[c + 1] / dg;
                    lo = orc_e2m1_encode((double)y0);
                    hi = orc_e2m1_encode((double)y1);
                }
                codes[(size_t)n * (d / 2) + (16 * g + c) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    *s1_out = s1;
}

/* Q and smoothed K in NVFP4 (k_mean from orc_k_mean): q4, k4 [B,H,N,d/2]
 * packed codes; sfq, sfk [B,H,N,d/16]; sq1, sk1 [B,H,ceil(N/64)]. */
void orc_quantize_nvfp4_qk(const uint16_t *q, const uint16_t *k, const float *k_mean,
                           int B, int H, int N, int d, uint8_t *q4, uint8_t *k4,
                           uint8_t *sfq, uint8_t *sfk, float *sq1, float *sk1)
{
    int nblk = (N + 63) / 64;
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++) {
            float *x = (float *)malloc(sizeof(float) * 64 * d);
            const float *mu = k_mean + ((size_t)b * H + h) * d;
            for (int j = 0; j < nblk; j++) {
                int nt = N - 64 * j < 64 ? N - 64 * j : 64;
                size_t row = ((size_t)b * H + h) * N + 64 * j;
                size_t sidx = ((size_t)b * H + h) * nblk + j;
                for (int i = 0; i < nt * d; i++)
                    x[i] = orc_bf16_to_float(q[row * d + i]);
                quantize_block_nvfp4(x, nt, d, q4 + row * (d / 2), sfq + row * (d / 16), &sq1[sidx]);
                for (int i = 0; i < nt * d; i++)
                    x[i] = orc_bf16_to_float(k[row * d + i]) - mu[i % d];
                quantize_block_nvfp4(x, nt, d, k4 + row * (d / 2), sfk + row * (d / 16), &sk1[sidx]);
            }
            free(x);
        }
}

/* NVFP4 Q.K with the FP8 P.V path: the tiled rule of attention_core_head on
 * the dequantized Q and K (code value x its group scale; the block scale s1
 * plays the role of sq / sk) and the FP8 V codes and scales.  heads/rows/out
 * as orc_attention_fp8. */
void orc_attention_nvfp4(const uint8_t *q4, const uint8_t *k4, const uint8_t *sfq, const uint8_t *sfk,
                         const float *sq1, const float *sk1, const uint8_t *v8, const float *sv,
                         const float *sv_max, int B, int H, int N, int d, float softmax_scale,
                         const int *heads, int n_heads, const int *rows, int n_rows,
                         double *out, double *amb, int *namb)
{
    int nblk = (N + 63) / 64;
    (void)B;
    double *qc = (double *)malloc(sizeof(double) * N * d);
    double *kc = (double *)malloc(sizeof(double) * N * d);
    double *vc = (double *)malloc(sizeof(double) * N * d);
    for (int hh = 0; hh < n_heads; hh++) {
        int b = heads[2 * hh], h = heads[2 * hh + 1];
        size_t row0 = ((size_t)b * H + h) * N;
        for (size_t n = 0; n < (size_t)N; n++)
            for (int c = 0; c < d; c++) {
                size_t r = row0 + n;
                uint8_t qb = q4[r * (d / 2) + c / 2], kb = k4[r * (d / 2) + c / 2];
                uint8_t qn = (c & 1) ? (qb >> 4) : (qb & 15), kn = (c & 1) ? (kb >> 4) : (kb & 15);
                qc[n * d + c] = orc_e2m1_decode(qn) * orc_e4m3_decode(sfq[r * (d / 16) + c / 16]);
                kc[n * d + c] = orc_e2m1_decode(kn) * orc_e4m3_decode(sfk[r * (d / 16) + c / 16]);
                vc[n * d + c] = orc_e4m3_decode(v8[r * d + c]);
            }
        size_t sidx = ((size_t)b * H + h) * nblk;
        attention_core_head(qc, kc, vc, sq1 + sidx, sk1 + sidx, sv + sidx, sv_max[(size_t)b * H + h], N, d,
                            (double)softmax_scale, 128, 1, rows, n_rows, out + (size_t)hh * n_rows * d,
                            amb ? amb + (size_t)hh * n_rows * d : NULL,
                            namb ? namb + (size_t)hh * n_rows : NULL, NULL, NULL, NULL);
    }
    free(qc); free(kc); free(vc);
}

/* --------------------------------------------- error-corrected attention */
/* FP8 attention that corrects only the tokens with large error: "FLUX 3
 * Image Klein Base: 생성 3.46배, 8장 확장 병목", section "왜 이런 차이가 나나"
 * (VC-Attention FP8, rho = 0.005, against cuDNN FP8 and VANILLA BF16 on
 * B200).  The page gives the name, the idea and rho only; the readings:
 *  - the tokens are key/value tokens and the error is each key's own
 *    quantization error (orc_key_error);
 *  - per (b, h) the ceil(rho * N) keys with the largest error are corrected
 *    (orc_select_keys);
 *  - correction: the FP8 rule runs over the other keys, the corrected keys'
 *    part is exact (binary64 from the BF16 inputs, scores on the smoothed
 *    keys so both parts share one per-row offset), and the two partial
 *    softmaxes are merged by their maxima and row sums. */

/* Per-key quantization error [reading]: the squared distance between the
 * smoothed key and its dequantized code, in binary32 in a pinned order:
 *   r_c = fl32(x_c - fl32(dec(code_c) * s_J)),  x_c = fl32(k_c - mu_c)
 *   g_i = ((r_8i^2 + r_8i+1^2) + ...) + r_8i+7^2   (i = 0..15, squares rounded)
 *   then pairwise: a_i = g_i + g_i+8, b_i = a_i + a_i+4, c_i = b_i + b_i+2,
 *   e = c_0 + c_1.
 * err: [B,H,N]. */
void orc_key_error(const uint16_t *k, const uint8_t *k8, const float *sk, const float *k_mean,
                   int B, int H, int N, int d, float *err)
{
    int nblk = (N + 63) / 64;
    float dec[256];
    for (int i = 0; i < 256; i++) dec[i] = (float)orc_e4m3_decode((uint8_t)i);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++) {
            const float *mu = k_mean + ((size_t)b * H + h) * d;
            for (int n = 0; n < N; n++) {
                float s = sk[((size_t)b * H + h) * nblk + n / 64];
                float g[16];
                for (int i = 0; i < 16; i++) {
                    float acc = 0.0f;
                    for (int c = 8 * i; c < 8 * i + 8; c++) {
                        size_t at = IDX4(b, h, n, c, H, N, d);
                        float x = orc_bf16_to_float(k[at]) - mu[c];
                        float dq = dec[k8[at]] * s;
                        float rr = x - dq;
                        float sq = rr * rr;
                        acc = acc + sq;
                    }
                    g[i] = acc;
                }
                float a[8], bb[4], cc[2];
                for (int i = 0; i < 8; i++) a[i] = g[i] + g[i + 8];
                for (int i = 0; i < 4; i++) bb[i] = a[i] + a[i + 4];
                for (int i = 0; i < 2; i++) cc[i] = bb[i] + bb[i + 2];
                err[((size_t)b * H + h) * N + n] = cc[0] + cc[1];
            }
        }
}

/* The kc keys of each (b, h) with the largest error, ties to the lower token
 * index: sel[B,H,N] = 1 for them, 0 otherwise (kc is clamped to [0, N]). */
static const float *g_sel_err;
static int sel_cmp(const void *pa, const void *pb)
{
    int ia = *(const int *)pa, ib = *(const int *)pb;
    float ea = g_sel_err[ia], eb = g_sel_err[ib];
    if (ea > eb) return -1;
    if (ea < eb) return 1;
    return ia < ib ? -1 : (ia > ib ? 1 : 0);
}

void orc_select_keys(const float *err, int B, int H, int N, int kc, uint8_t *sel)
{
    if (kc < 0) kc = 0;
    if (kc > N) kc = N;
    int *idx = (int *)malloc(sizeof(int) * N);
    for (int bh = 0; bh < B * H; bh++) {
        const float *e = err + (size_t)bh * N;
        for (int j = 0; j < N; j++) idx[j] = j;
        g_sel_err = e;                          /* single-threaded: qsort has no context */
        qsort(idx, N, sizeof(int), sel_cmp);
        memset(sel + (size_t)bh * N, 0, N);
        for (int t = 0; t < kc; t++) sel[(size_t)bh * N + idx[t]] = 1;
    }
    free(idx);
}

/* The FP8 part alone: the tiled rule over the keys with sel = 0 (normalized
 * output, and each row's final maximum and row sum; l = 0 and a zero row
 * when every key is selected).  out: [n_heads, n_rows, d]; m_out, l_out:
 * [n_heads, n_rows]. */
void orc_attention_fp8_part(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8,
                            const float *sq, const float *sk, const float *sv, const float *sv_max,
                            const uint8_t *sel, int B, int H, int N, int d, float softmax_scale,
                            const int *heads, int n_heads, const int *rows, int n_rows,
                            double *out, double *m_out, double *l_out)
{
    int nblk = (N + 63) / 64;
    (void)B;
    double *qc = (double *)malloc(sizeof(double) * N * d);
    double *kc = (double *)malloc(sizeof(double) * N * d);
    double *vc = (double *)malloc(sizeof(double) * N * d);
    double dec[256];
    for (int i = 0; i < 256; i++) dec[i] = orc_e4m3_decode((uint8_t)i);
    for (int hh = 0; hh < n_heads; hh++) {
        int b = heads[2 * hh], h = heads[2 * hh + 1];
        size_t base = IDX4(b, h, 0, 0, H, N, d);
        for (size_t i = 0; i < (size_t)N * d; i++) {
            qc[i] = dec[q8[base + i]];
            kc[i] = dec[k8[base + i]];
            vc[i] = dec[v8[base + i]];
        }
        size_t sidx = ((size_t)b * H + h) * nblk;
        attention_core_head(qc, kc, vc, sq + sidx, sk + sidx, sv + sidx, sv_max[(size_t)b * H + h], N, d,
                            (double)softmax_scale, 128, 1, rows, n_rows, out + (size_t)hh * n_rows * d,
                            NULL, NULL, sel + ((size_t)b * H + h) * N, m_out + (size_t)hh * n_rows,
                            l_out + (size_t)hh * n_rows);
    }
    free(qc); free(kc); free(vc);
}

/* Error-corrected FP8 attention for the listed heads and rows.  q, k, v: the
 * BF16 inputs; the code/scale arrays and k_mean from orc_quantize; sel from
 * orc_select_keys.  For row i:
 *   FP8 part over keys with sel = 0 (the tiled rule): O1, m1, l1
 *   exact part over keys with sel = 1: s_j = (q_i . (k_j - mu)) * scale * log2(e),
 *     m2 = max s_j, p_j = 2^(s_j - m2), l2 = sum p_j, A2 = sum p_j v_j
 *   M = max(m1, m2), w1 = 2^(m1 - M), w2 = 2^(m2 - M) (0 for an empty part),
 *   out = (O1 * l1 * w1 + A2 * w2) / (l1 * w1 + l2 * w2).
 * quantize_p = 0 leaves the FP8 part's P unrounded (for the pins).  amb
 * (optional): the FP8 part's ambiguity bound, carried through the merge. */
void orc_attention_fp8_corrected(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                 const uint8_t *q8, const uint8_t *k8, const uint8_t *v8,
                                 const float *sq, const float *sk, const float *sv,
                                 const float *sv_max, const float *k_mean, const uint8_t *sel,
                                 int B, int H, int N, int d, float softmax_scale, int quantize_p,
                                 const int *heads, int n_heads, const int *rows, int n_rows,
                                 double *out, double *amb)
{
    const double LOG2E = 1.4426950408889634073599246810019;
    int nblk = (N + 63) / 64;
    (void)B;
    double *qc = (double *)malloc(sizeof(double) * N * d);
    double *kc = (double *)malloc(sizeof(double) * N * d);
    double *vc = (double *)malloc(sizeof(double) * N * d);
    double *m1 = (double *)malloc(sizeof(double) * n_rows);
    double *l1 = (double *)malloc(sizeof(double) * n_rows);
    double dec[256];
    for (int i = 0; i < 256; i++) dec[i] = orc_e4m3_decode((uint8_t)i);
    for (int hh = 0; hh < n_heads; hh++) {
        int b = heads[2 * hh], h = heads[2 * hh + 1];
        size_t base = IDX4(b, h, 0, 0, H, N, d);
        const uint8_t *sl = sel + ((size_t)b * H + h) * N;
        const float *mu = k_mean + ((size_t)b * H + h) * d;
        for (size_t i = 0; i < (size_t)N * d; i++) {
            qc[i] = dec[q8[base + i]];
            kc[i] = dec[k8[base + i]];
            vc[i] = dec[v8[base + i]];
        }
        size_t sidx = ((size_t)b * H + h) * nblk;
        double *o = out + (size_t)hh * n_rows * d;
        double *ab = amb ? amb + (size_t)hh * n_rows * d : NULL;
        attention_core_head(qc, kc, vc, sq + sidx, sk + sidx, sv + sidx,
                            sv_max[(size_t)b * H + h], N, d, (double)softmax_scale, 128,
                            quantize_p, rows, n_rows, o, ab, NULL, sl, m1, l1);
        #pragma omp parallel for schedule(dynamic, 4)
        for (int r = 0; r < n_rows; r++) {
            int i = rows[r];
            double qi[512];
            for (int c = 0; c < d && c < 512; c++)
                qi[c] = orc_bf16_to_float(q[base + (size_t)i * d + c]);
            double m2 = -INFINITY;
            for (int j = 0; j < N; j++) {
                if (!sl[j]) continue;
                double s = 0.0;
                for (int c = 0; c < d; c++)
                    s += qi[c] * ((double)orc_bf16_to_float(k[base + (size_t)j * d + c]) - (double)mu[c]);
                s *= (double)softmax_scale * LOG2E;
                if (s > m2) m2 = s;
            }
            double l2 = 0.0, a2[512];
            for (int c = 0; c < d; c++) a2[c] = 0.0;
            if (m2 > -INFINITY)
                for (int j = 0; j < N; j++) {
                    if (!sl[j]) continue;
                    double s = 0.0;
                    for (int c = 0; c < d; c++)
                        s += qi[c] * ((double)orc_bf16_to_float(k[base + (size_t)j * d + c]) - (double)mu[c]);
                    double p = exp2(s * (double)softmax_scale * LOG2E - m2);
                    l2 += p;
                    for (int c = 0; c < d; c++)
                        a2[c] += p * orc_bf16_to_float(v[base + (size_t)j * d + c]);
                }
            double mm = m1[r] > m2 ? m1[r] : m2;
            double w1 = (l1[r] > 0.0) ? exp2(m1[r] - mm) : 0.0;
            double w2 = (m2 > -INFINITY) ? exp2(m2 - mm) : 0.0;
            double L = l1[r] * w1 + l2 * w2;
            for (int c = 0; c < d; c++) {
                double v1 = o[(size_t)r * d + c] * l1[r] * w1;
                o[(size_t)r * d + c] = L > 0.0 ? (v1 + a2[c] * w2) / L : 0.0;
                if (ab) ab[(size_t)r * d + c] = L > 0.0 ? ab[(size_t)r * d + c] * l1[r] * w1 / L : 0.0;
            }
        }
    }
    free(qc); free(kc); free(vc); free(m1); free(l1);
}

/* Exact attention, binary64, no quantization: softmax(Q K^T * scale) V on the
 * BF16 inputs with a two-pass row maximum.  Same heads/rows/out convention. */
void orc_attention_exact(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int B, int H, int N, int d, double scale,
                         const int *heads, int n_heads, const int *rows, int n_rows,
                         double *out)
{
    (void)B;
    double *kd = (double *)malloc(sizeof(double) * N * d);
    double *vd = (double *)malloc(sizeof(double) * N * d);
    for (int hh = 0; hh < n_heads; hh++) {
        int b = heads[2 * hh], h = heads[2 * hh + 1];
        size_t base = IDX4(b, h, 0, 0, H, N, d);
        for (size_t i = 0; i < (size_t)N * d; i++) {
            kd[i] = orc_bf16_to_float(k[base + i]);
            vd[i] = orc_bf16_to_float(v[base + i]);
        }
        #pragma omp parallel for schedule(dynamic, 4)
        for (int r = 0; r < n_rows; r++) {
            int i = rows[r];
            double *o = out + ((size_t)hh * n_rows + r) * d;
            double *s = (double *)malloc(sizeof(double) * N);
            double qi[512];
            for (int c = 0; c < d && c < 512; c++)
                qi[c] = orc_bf16_to_float(q[base + (size_t)i * d + c]);
            double mx = -INFINITY;
            for (int j = 0; j < N; j++) {
                double acc = 0.0;
                for (int c = 0; c < d; c++) acc += qi[c] * kd[(size_t)j * d + c];
                s[j] = acc * scale;
                if (s[j] > mx) mx = s[j];
            }
            double l = 0.0;
            for (int c = 0; c < d; c++) o[c] = 0.0;
            for (int j = 0; j < N; j++) {
                double p = exp(s[j] - mx);
                l += p;
                for (int c = 0; c < d; c++) o[c] += p * vd[(size_t)j * d + c];
            }
            for (int c = 0; c < d; c++) o[c] /= l;
            free(s);
        }
    }
    free(kd); free(vd);
}

/* Vectorised encoder over binary32 inputs, for the exhaustive codec check
 * against the GPU's conversion instruction. */
void orc_e4m3_encode_f32_array(const float *x, size_t n, uint8_t *out)
{
    #pragma omp parallel for schedule(static)
    for (size_t i = 0; i < n; i++)
        out[i] = isnan(x[i]) ? 0x7F : orc_e4m3_encode((double)x[i]);
}

/* Vectorised BF16 rounding of binary64 values. */
void orc_bf16_round_array(const double *x, size_t n, uint16_t *out)
{
    #pragma omp parallel for schedule(static)
    for (size_t i = 0; i < n; i++)
        out[i] = orc_bf16_round(x[i]);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
