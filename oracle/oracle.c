/*
 * oracle.c -- plain, slow CPU reference for causal prefill attention with the
 * ZYFA FP8 method (Lean P, per-64-key power-of-two block scale, row sum from
 * rounded P) and its quantize + Hadamard prepass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py load this library.  It shares no code, header,
 * table or constant with the CUDA library in bf16_causal_prefill_fp8_b200/csrc,
 * and neither side includes or links the other.
 *
 * Sources (news pages about Zyphra's ZYFA kernels; cited by page and section):
 *   [NL] the-ai.news, "Zyphra presenteert ZYFA: FlashAttention FP8 voor AMD MI355X"
 *   [ES] ai-daily-news.org, "Zyphra ZYFA: FP8 FlashAttention para AMD MI355X"
 *   [ZH] kongchang.com, "Zyphra ZYFA: AMD MI355X 上的 FP8 FlashAttention 提速 1.76 倍"
 *   [JA] spke.com, "Zyphra ZYFA: AMD MI355X向けFP8 FlashAttention、最大1.76倍高速化"
 *
 * Precision.  Attention itself is computed in fp64.  Two parts are integer
 * decisions taken in floating point (the e4m3 quantization code and the Lean-P
 * code); the pages do not fix their precision, so both are taken in fp32, the
 * kernel's precision, step by step as specified below, so that the GPU codes
 * can be compared byte for byte.
 *
 * Pins (tests/test_oracle_pins.py, run without a GPU):
 *   oracle_e4m3_value / oracle_e4m3_from_f32 : exhaustive over all 256 codes
 *       against torch's float8_e4m3fn and ml_dtypes decoders, the power-of-two
 *       ladder code(2^k) = 8k + 56 (tests/golden/e4m3_pow2_ladder.txt), RNE ties.
 *   oracle_fwht128 : against scipy.linalg.hadamard(128)/sqrt(128); H H^T = I.
 *   oracle_fwht64 : against scipy.linalg.hadamard(64)/8; with the 128-point
 *       block it keeps Q K^T of Dqk 192 rows (rotation invariance).
 *   oracle_quantize : amax/448 scale and codes against a brute-force nearest
 *       search over the 127 finite non-negative e4m3 values; rotation
 *       invariance of Q K^T in fp64.
 *   oracle_attention_rows : torch scaled_dot_product_attention (fp64, causal)
 *       on small cases; row 0 == V[0]; Q = 0 gives prefix means of V; GQA with
 *       one kv head equals MHA with replicated K/V.
 *   oracle_leanp_* : code == 8j + 56 when s == m == 0; monotone in s; decoded
 *       weight / exact weight inside Mitchell's band (2^-1/8, 1.0615] for
 *       normal codes; largest code of a block in (112, 120].
 *   oracle_exactp_code : code 8j + 56 at s = m (a power of two: exact); monotone
 *       in s; decoded weight within e4m3's half-ulp bound (2^-4 relative) of
 *       the exact weight for normal codes.
 *   oracle_fp8_model_rows : with p_mode = 1 equals oracle_attention_rows on
 *       the dequantized inputs to 1e-6 (pins tile order, running max, the
 *       rescale factor and the row sum), also with the deferred reference max
 *       on scores that grow by many binades across the keys; Q = 0 gives
 *       prefix means exactly.
 * No function here is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* e4m3 ("fn" variant: 4 exponent bits, bias 7, 3 mantissa bits, no         */
/* infinities, 0x7F/0xFF = NaN, largest finite 448).  The pages rely on the */
/* fact that the bit pattern read as an integer grows by 8 per doubling     */
/* ([NL] "Drie technieken om de bottleneck te omzeilen"; [JA] "Lean P").    */
/* ------------------------------------------------------------------------ */

/* Value of an e4m3 code, from the format definition. */
double oracle_e4m3_value(unsigned code)
{
    unsigned sign = (code >> 7) & 1u;
    unsigned e = (code >> 3) & 15u;
    unsigned m = code & 7u;
    double v;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u)
        v = ldexp((double)m, -9);          /* subnormal: m * 2^-6 / 8 */
    else
        v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return sign ? -v : v;
}

/* Round an fp32 value to the nearest e4m3 code, ties to the even code,
 * saturating to +-448 (the behaviour of a round-to-nearest, satfinite
 * conversion).  Brute force: scan the 127 finite non-negative codes. */
unsigned oracle_e4m3_from_f32(float x)
{
    unsigned sign = signbit(x) ? 0x80u : 0u;
    double a = fabs((double)x);
    unsigned best = 0;
    double best_d;
    unsigned c;
    if (isnan(x)) return 0x7Fu | sign;
    if (a >= 448.0) return 0x7Eu | sign;
    best_d = a;                                    /* distance to code 0 */
    for (c = 1; c <= 0x7Eu; ++c) {
        double d = fabs(oracle_e4m3_value(c) - a);
        if (d < best_d || (d == best_d && (c & 1u) == 0u && (best & 1u) == 1u)) {
            best = c;
            best_d = d;
        }
    }
    return best | sign;
}

/* ------------------------------------------------------------------------ */
/* 128-point Sylvester Walsh-Hadamard transform, orthonormal.               */
/* [JA] "ZYFAのFP8アテンションの精度はどのくらいか?": a Hadamard rotation of */
/* Q and K roughly halves the quantization error.  The pages give no        */
/* normalisation; the orthonormal H/sqrt(128) keeps Q K^T unchanged.        */
/* Specified step order (the GPU follows it so codes match bit for bit):    */
/*   for h = 1, 2, 4, ..., 64: for each pair (i, i+h) with (i & h) == 0:    */
/*       (x[i], x[i+h]) <- (x[i] + x[i+h], x[i] - x[i+h])   in fp32         */
/*   then every element is multiplied by fl32(2^-3.5) once.                 */
/* ------------------------------------------------------------------------ */
void oracle_fwht128(float *x)
{
    int h, i;
    const float norm = (float)0.08838834764831844055;   /* 2^-3.5 rounded to fp32 */
    for (h = 1; h < 128; h <<= 1) {
        for (i = 0; i < 128; ++i) {
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
        }
    }
    for (i = 0; i < 128; ++i) x[i] = x[i] * norm;
}

/* The 64-point companion for the MLA shape (reading: Dqk 192 = 128 + 64 is */
/* rotated block-diagonally, H128/sqrt(128) on dims 0..127 and              */
/* H64/sqrt(64) on dims 128..191; orthonormal, so Q K^T is unchanged).      */
/* Stages of stride 1, 2, ..., 32 in fp32, then one multiply by 2^-3.       */
void oracle_fwht64(float *x)
{
    int h, i;
    for (h = 1; h < 64; h <<= 1) {
        for (i = 0; i < 64; ++i) {
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
        }
    }
    for (i = 0; i < 64; ++i) x[i] = x[i] * 0.125f;
}

/* The rotation the prepass applies to a row of D = 128 or 192 values. */
static void oracle_rotate_row(float *row, int D)
{
    oracle_fwht128(row);
    if (D == 192) oracle_fwht64(row + 128);
}

/* ------------------------------------------------------------------------ */
/* Per-(batch, head) FP8 quantization.  [ZH] "ZYFA 的性能与精度数据": FP8     */
/* attention maps values into the e4m3 range with per-tensor or per-head    */
/* scale factors.  [JA] accuracy section: most of the FP8 error comes from  */
/* quantizing Q, K and V.                                                   */
/*   x      : [B, S, H, D] fp32 (bf16 inputs are widened exactly by caller) */
/*   amax   : max |x'| over (s, d) of one (b, h), x' = rotated row when     */
/*            hadamard != 0 (D 128: H128; D 192: H128 on dims 0..127 and  */
/*            H64 on dims 128..191), else x' = x                            */
/*   scale  : amax / 448 in fp32 (IEEE division); 1 when amax == 0          */
/*   code   : e4m3 RNE satfinite of fl32(x' / scale) (IEEE division)        */
/* Returns 0, or -1 for bad arguments.                                      */
/* ------------------------------------------------------------------------ */
int oracle_quantize(const float *x, int B, int S, int H, int D, int hadamard,
                    uint8_t *codes, float *scale)
{
    int b, h;
    if (!x || !codes || !scale || B < 1 || S < 1 || H < 1 || D < 1) return -1;
    if (hadamard && D != 128 && D != 192) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (b = 0; b < B; ++b) {
        for (h = 0; h < H; ++h) {
            float row[1024];
            float amax = 0.0f, sc;
            int s, d;
            for (s = 0; s < S; ++s) {
                const float *src = x + (((size_t)b * S + s) * H + h) * (size_t)D;
                for (d = 0; d < D; ++d) row[d] = src[d];
                if (hadamard) oracle_rotate_row(row, D);
                for (d = 0; d < D; ++d) {
                    float a = fabsf(row[d]);
                    if (a > amax) amax = a;
                }
            }
            sc = (amax > 0.0f) ? amax / 448.0f : 1.0f;
            scale[(size_t)b * H + h] = sc;
            for (s = 0; s < S; ++s) {
                size_t off = (((size_t)b * S + s) * H + h) * (size_t)D;
                for (d = 0; d < D; ++d) row[d] = x[off + d];
                if (hadamard) oracle_rotate_row(row, D);
                for (d = 0; d < D; ++d)
                    codes[off + d] = (uint8_t)oracle_e4m3_from_f32(row[d] / sc);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Causal attention in fp64: the plain definition.                          */
/* [ES] "Qué cubren los kernels": causal forward (prefill) attention.       */
/* For query row i of head hq (kv head hq / (Hq/Hkv)):                      */
/*   s_j = sm_scale * sum_d q_i,d k_j,d      for keys j <= i                */
/*   o_i = sum_j exp(s_j - max) v_j / sum_j exp(s_j - max)                  */
/* q [B,S,Hq,Dqk], k [B,S,Hkv,Dqk], v [B,S,Hkv,Dv] (already dequantized),   */
/* rows: the query rows to compute (NULL = all S rows, nrows = S),          */
/* o [B, nrows, Hq, Dv].                                                    */
/* ------------------------------------------------------------------------ */
int oracle_attention_rows(const double *q, const double *k, const double *v,
                          int B, int Hq, int Hkv, int S, int Dqk, int Dv,
                          double sm_scale, const int *rows, int nrows, double *o)
{
    int b;
    if (!q || !k || !v || !o || B < 1 || Hq < 1 || Hkv < 1 || S < 1) return -1;
    if (Hq % Hkv != 0 || Dqk < 1 || Dv < 1) return -1;
    if (!rows) nrows = S;
    for (b = 0; b < B; ++b) {
        int task;
#pragma omp parallel for schedule(dynamic, 4)
        for (task = 0; task < Hq * nrows; ++task) {
            int hq = task / nrows, r = task % nrows;
            int i = rows ? rows[r] : r;
            int kvh = hq / (Hq / Hkv);
            double *s = (double *)malloc(sizeof(double) * (size_t)(i + 1));
            double *acc = (double *)calloc((size_t)Dv, sizeof(double));
            const double *qi = q + (((size_t)b * S + i) * Hq + hq) * (size_t)Dqk;
            double mx = -INFINITY, den = 0.0;
            int j, d;
            for (j = 0; j <= i; ++j) {
                const double *kj = k + (((size_t)b * S + j) * Hkv + kvh) * (size_t)Dqk;
                double dot = 0.0;
                for (d = 0; d < Dqk; ++d) dot += qi[d] * kj[d];
                s[j] = dot * sm_scale;
                if (s[j] > mx) mx = s[j];
            }
            for (j = 0; j <= i; ++j) {
                const double *vj = v + (((size_t)b * S + j) * Hkv + kvh) * (size_t)Dv;
                double w = exp(s[j] - mx);
                den += w;
                for (d = 0; d < Dv; ++d) acc[d] += w * vj[d];
            }
            for (d = 0; d < Dv; ++d)
                o[(((size_t)b * nrows + r) * Hq + hq) * (size_t)Dv + d] = acc[d] / den;
            free(s);
            free(acc);
        }
    }
    return 0;
}

/* Log-sum-exp of each row's causal scores in fp64, the plain definition:   */
/*   lse_i = max_j s_j + log(sum_j exp(s_j - max_j s_j)),  s_j as above.    */
/* lse [B, Hq, nrows].                                                      */
int oracle_attention_lse_rows(const double *q, const double *k, int B, int Hq, int Hkv, int S, int Dqk,
                              double sm_scale, const int *rows, int nrows, double *lse)
{
    int b;
    if (!q || !k || !lse || B < 1 || Hq < 1 || Hkv < 1 || S < 1) return -1;
    if (Hq % Hkv != 0 || Dqk < 1) return -1;
    if (!rows) nrows = S;
    for (b = 0; b < B; ++b) {
        int task;
#pragma omp parallel for schedule(dynamic, 4)
        for (task = 0; task < Hq * nrows; ++task) {
            int hq = task / nrows, r = task % nrows;
            int i = rows ? rows[r] : r;
            int kvh = hq / (Hq / Hkv);
            double *s = (double *)malloc(sizeof(double) * (size_t)(i + 1));
            const double *qi = q + (((size_t)b * S + i) * Hq + hq) * (size_t)Dqk;
            double mx = -INFINITY, den = 0.0;
            int j, d;
            for (j = 0; j <= i; ++j) {
                const double *kj = k + (((size_t)b * S + j) * Hkv + kvh) * (size_t)Dqk;
                double dot = 0.0;
                for (d = 0; d < Dqk; ++d) dot += qi[d] * kj[d];
                s[j] = dot * sm_scale;
                if (s[j] > mx) mx = s[j];
            }
            for (j = 0; j <= i; ++j) den += exp(s[j] - mx);
            lse[((size_t)b * Hq + hq) * (size_t)nrows + r] = mx + log(den);
            free(s);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Lean P, bit level ([NL] "Drie technieken om de bottleneck te omzeilen";  */
/* [JA] "Lean P: 指数関数の代わりに1回の乗算加算" and "ブロックごとの       */
/* スケーリングと丸められた行和").                                          */
/* The e4m3 code of 2^x is about 8x + 56, so each probability is written as */
/* one multiply-add plus one integer conversion; each 64-key block of P is  */
/* multiplied by a power of two 2^j before rounding, and the matrix unit    */
/* removes 2^-j again.  All steps are fp32 with fused multiply-add:         */
/*   C    = fl32(8 log2(e) / sqrt(Dqk))            (rounded once, from fp64) */
/*   A    = fl32(fl32(q_s * k_s) * C)              slope per (row's head)    */
/*   j    = 8 if bmax == -inf, else                                          */
/*          min(126, 8 + floor(fl32(fl32(m - bmax) * A) * 0.125))            */
/*   B    = fmaf(-m, A, 56 + 8j)                                             */
/*   u    = fmaf(s, A, B)                                                    */
/*   code = 0 if s is masked, else clamp(trunc(u), 0, 126)                   */
/* s: raw fp32 score (sum of products of e4m3 values); m: running row max   */
/* after this tile; bmax: max of the 64-key block holding s.  The weight    */
/* the matrix unit uses is value(code) * 2^-j (E8M0 scale code 127 - j).    */
/* ------------------------------------------------------------------------ */
float oracle_leanp_slope(float q_s, float k_s, int Dqk)
{
    const float C = (float)(8.0 * 1.4426950408889634074 / sqrt((double)Dqk));
    float qk = q_s * k_s;
    return qk * C;
}

int oracle_leanp_block_shift(float m, float bmax, float A)
{
    float d, e, f;
    if (isinf(bmax) && bmax < 0.0f) return 8;
    d = m - bmax;
    e = d * A;
    f = e * 0.125f;
    f = floorf(f);
    if (f >= 118.0f) return 126;
    return 8 + (int)f;
}

unsigned oracle_leanp_code(float s, float m, float A, int j, int masked)
{
    float B, u, t;
    if (masked) return 0u;
    B = fmaf(-m, A, (float)(56 + 8 * j));
    u = fmaf(s, A, B);
    if (!(u > 0.0f)) return 0u;                    /* also catches -inf */
    t = truncf(u);
    if (t > 126.0f) return 126u;
    return (unsigned)t;
}

/* The exact-P alternative (the pages' baseline that Lean P replaces, [NL]   */
/* "Drie technieken", [JA] "Lean P": an exponential, then a conversion to   */
/* e4m3): the same block shift j, then                                       */
/*   code = e4m3 RNE-satfinite of fl32(exp2((s - m) A / 8 + j))             */
/* (exp2 in fp64, rounded once to fp32); 0 for a masked key.  The weight is  */
/* value(code) * 2^-j, as for Lean P.                                        */
unsigned oracle_exactp_code(float s, float m, float A, int j, int masked)
{
    double x;
    if (masked || (isinf(s) && s < 0.0f)) return 0u;
    x = ((double)s - (double)m) * (double)A / 8.0 + (double)j;
    return oracle_e4m3_from_f32((float)exp2(x));
}

/* Element-wise batch form used by the bit-exactness test. */
void oracle_leanp_batch(const float *s, const float *m, const float *bmax,
                        const float *A, const uint8_t *masked, int n,
                        uint8_t *code, int32_t *jout)
{
    int i;
    for (i = 0; i < n; ++i) {
        int j = oracle_leanp_block_shift(m[i], bmax[i], A[i]);
        code[i] = (uint8_t)oracle_leanp_code(s[i], m[i], A[i], j, masked ? masked[i] : 0);
        if (jout) jout[i] = j;
    }
}

/* ------------------------------------------------------------------------ */
/* Model oracle: the FP8 pipeline in the pages' order, in fp64 except the   */
/* Lean-P decisions (fp32, above).  Per query row i, KV tiles of kv_tile    */
/* keys (128 or 256: the tile a kernel processes at a time, which is where  */
/* the deferred reference max is decided) are visited in ascending order    */
/* (tiles 0 .. i/kv_tile); each tile is kv_tile/64 blocks of 64 keys.       */
/* For tile t:                                                              */
/*   s_j   = fl32(sum_d value(qcode) * value(kcode))   keys j <= i, j < S    */
/*   bmax  = max s_j over each block (-inf if the block has no live key)    */
/*   m'    = max(m, bmax_0, bmax_1, ..)      running max after this tile    */
/*           (rescale_log2 > 0: reference max instead -- m' = tile max on    */
/*           tile 0; later m' = max(bmax_0, bmax_1, ..) only when           */
/*           fl32(fl32(that - m) * A) > 8 rescale_log2, i.e. when the tile  */
/*           max is more than rescale_log2 binades above m, else m' = m.    */
/*           The softmax is unchanged: O and l share the reference and the */
/*           per-block shift j renormalises each block to its own max.)     */
/*   w_j   = value(leanp code) * 2^-j_block                                  */
/*           p_mode 1: exp2((s_j-m')A/8) in fp64 (no rounding of P);          */
/*           p_mode 2: value(exact-P e4m3 code) * 2^-j_block                 */
/*   alpha = exp2((m - m') A / 8)            (0 on the first tile)          */
/*   O     = alpha O + sum_j w_j value(vcode_j);  l = alpha l + sum_j w_j   */
/* Every block shift j must stay >= 8 with the exact max, and >= 8 - r     */
/* with the deferred one (a block at most r binades above the reference);  */
/* a violation (a reference that does not move when it must) returns -2.   */
/* lse (may be NULL) [B, Hq, nrows]: ln 2 (m A/8 + log2 l) at the last tile. */
/* The row sum l comes from the rounded weights, like the extra matrix      */
/* instruction per block on the pages.  Output o_i = O / l * v_s.           */
/* q [B,S,Hq,Dqk], k [B,S,Hkv,Dqk], v [B,S,Hkv,Dv] codes; q_s [B*Hq],       */
/* k_s, v_s [B*Hkv]; rows NULL = all; o [B, nrows, Hq, Dv].                 */
/* ------------------------------------------------------------------------ */
int oracle_fp8_model_rows(const uint8_t *qc, const uint8_t *kc, const uint8_t *vc,
                          const float *q_s, const float *k_s, const float *v_s,
                          int B, int Hq, int Hkv, int S, int Dqk, int Dv,
                          int p_mode, float rescale_log2, int kv_tile,
                          const int *rows, int nrows, double *o, double *lse)
{
    int b, shift_err = 0;
    const int nblk = kv_tile / 64;
    if (!qc || !kc || !vc || !q_s || !k_s || !v_s || !o) return -1;
    if (kv_tile != 128 && kv_tile != 256) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Hq % Hkv != 0 || Dqk < 1 || Dv < 1) return -1;
    if (!rows) nrows = S;
    for (b = 0; b < B; ++b) {
        int task;
#pragma omp parallel for schedule(dynamic, 4)
        for (task = 0; task < Hq * nrows; ++task) {
            int hq = task / nrows, r = task % nrows;
            int i = rows ? rows[r] : r;
            int kvh = hq / (Hq / Hkv);
            float A = oracle_leanp_slope(q_s[(size_t)b * Hq + hq], k_s[(size_t)b * Hkv + kvh], Dqk);
            double *qv = (double *)malloc(sizeof(double) * (size_t)Dqk);
            double *acc = (double *)calloc((size_t)Dv, sizeof(double));
            float sj[256];
            int live[256];
            double l = 0.0;
            float m = -INFINITY;
            int t, d, n;
            for (d = 0; d < Dqk; ++d)
                qv[d] = oracle_e4m3_value(qc[(((size_t)b * S + i) * Hq + hq) * (size_t)Dqk + d]);
            for (t = 0; t <= i / kv_tile; ++t) {
                float bmax[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                float mnew, tmax;
                double alpha;
                for (n = 0; n < kv_tile; ++n) {
                    int j = kv_tile * t + n;
                    live[n] = (j <= i && j < S);
                    sj[n] = -INFINITY;
                    if (live[n]) {
                        const uint8_t *kj = kc + (((size_t)b * S + j) * Hkv + kvh) * (size_t)Dqk;
                        double dot = 0.0;
                        for (d = 0; d < Dqk; ++d) dot += qv[d] * oracle_e4m3_value(kj[d]);
                        sj[n] = (float)dot;
                        if (sj[n] > bmax[n / 64]) bmax[n / 64] = sj[n];
                    }
                }
                tmax = bmax[0];
                for (n = 1; n < nblk; ++n)
                    if (bmax[n] > tmax) tmax = bmax[n];
                if (rescale_log2 > 0.0f) {
                    float grow;
                    if (t == 0) {
                        mnew = tmax;
                    } else {
                        grow = tmax - m;
                        grow = grow * A;
                        mnew = (grow > 8.0f * rescale_log2) ? tmax : m;
                    }
                } else {
                    mnew = tmax > m ? tmax : m;
                }
                for (n = 0; n < nblk; ++n)
                    if (oracle_leanp_block_shift(mnew, bmax[n], A) <
                        (rescale_log2 > 0.0f ? 8 - (int)ceilf(rescale_log2) : 8)) {
#pragma omp atomic write
                        shift_err = 1;
                    }
                alpha = (t == 0) ? 0.0 : exp2(((double)m - (double)mnew) * (double)A / 8.0);
                l *= alpha;
                for (d = 0; d < Dv; ++d) acc[d] *= alpha;
                for (n = 0; n < kv_tile; ++n) {
                    int j = kv_tile * t + n;
                    double w;
                    const uint8_t *vj;
                    if (!live[n]) continue;
                    if (p_mode == 1) {
                        w = exp2(((double)sj[n] - (double)mnew) * (double)A / 8.0);
                    } else if (p_mode == 2) {
                        int sh = oracle_leanp_block_shift(mnew, bmax[n / 64], A);
                        unsigned c = oracle_exactp_code(sj[n], mnew, A, sh, 0);
                        w = ldexp(oracle_e4m3_value(c), -sh);
                    } else {
                        int sh = oracle_leanp_block_shift(mnew, bmax[n / 64], A);
                        unsigned c = oracle_leanp_code(sj[n], mnew, A, sh, 0);
                        w = ldexp(oracle_e4m3_value(c), -sh);
                    }
                    l += w;
                    vj = vc + (((size_t)b * S + j) * Hkv + kvh) * (size_t)Dv;
                    for (d = 0; d < Dv; ++d) acc[d] += w * oracle_e4m3_value(vj[d]);
                }
                m = mnew;
            }
            for (d = 0; d < Dv; ++d)
                o[(((size_t)b * nrows + r) * Hq + hq) * (size_t)Dv + d] =
                    acc[d] / l * (double)v_s[(size_t)b * Hkv + kvh];
            /* the weights are 2^((s - m) A / 8) relative to the reference m:  */
            /* log-sum-exp of the scaled scores = ln 2 (m A / 8 + log2 l)      */
            if (lse)
                lse[((size_t)b * Hq + hq) * (size_t)nrows + r] =
                    0.69314718055994530942 * ((double)m * (double)A / 8.0 + log2(l));
            free(qv);
            free(acc);
        }
    }
    return shift_err ? -2 : 0;
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
