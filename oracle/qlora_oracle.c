/*
 * qlora_oracle.c -- plain, slow, obviously-correct CPU reference of the QLoRA
 * NF4 frozen-linear hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg may load this library.  It shares no source,
 * header, table or constant with the CUDA library: it builds the NF4 code
 * book itself from the normal quantile function, searches codes by brute
 * force, and accumulates every matrix product in fp64 with a naive loop.
 *
 * Sources (web pages on QLoRA, cited by page title and section):
 *  [P1] "QLoRA" blog note (p19e99): sec. 2 NF4, sec. 3 double quantization.
 *  [P2] "11.3 QLoRA: single-GPU finetuning" tutorial: "NF4 data type",
 *       "double quantization" (64 parameters share one fp32 constant;
 *       constants compressed from fp32 to 8 bit).
 *  [P3] "QLoRA - fitting 65B finetuning on one 48GB GPU" paper notes:
 *       "Key design 1: NF4" quantile equation, "Key design 2: double
 *       quantization", "Key design 3: frozen 4-bit base + LoRA" equation.
 *  [P4] "QLoRA: Efficient Finetuning of Quantized LLMs" digest (aipaper.cc),
 *       sec. 4 Methodology: NF4 equation q_i, double quantization
 *       (c2^FP32 -> 8-bit c2 plus c1^FP32, 8/64 + 32/(64*256) bits), the full
 *       equation Y = X doubleDequant(c1, c2, W) + X L1 L2 and
 *       doubleDequant = dequant(dequant(c1, c2), W) = W^BF16; steps 3-4
 *       (gradients flow through W^BF16, W frozen).
 *  [P5] "LoRA / QLoRA low-rank update, quantization and memory budget"
 *       reproduction blog: "LoRA formula and tensor shapes"
 *       (W0 [d_out,d_in], A [r,d_in], B [d_out,r], y = x W0^T + (a/r) x A^T B^T),
 *       "minimal experiment and acceptance protocol" (four invariants).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  R1 code book: 7 negative codes, an exact 0 and 8 positive codes; the
 *     positive half is Q(p) at p = linspace(1/2, 1-d, 9)[1:], the negative
 *     half Q(p) at p = linspace(d, 1/2, 8)[:-1], d = (1/32 + 1/30)/2, each
 *     half divided by its own extreme so min = -1 and max = +1, then rounded
 *     to fp32.  ([P4] quantile equation is infinite at its ends taken
 *     literally; [P4] says the ranges are asymmetric so 0 is exact.)
 *  R2 blocks are 64 consecutive elements of the row-major flattened tensor;
 *     a last partial block uses the elements it has.
 *  R3 x = fl32((w*p) * fl32(1/(absmax*p))) with the exact power-of-two
 *     prescale p = 2^64 when absmax < 2^-126 (the reciprocal of a subnormal
 *     would overflow), p = 1 otherwise; a zero block uses factor 0 (all
 *     codes 7).
 *  R4 nearest code = argmin |x - nf4[j]|, exact ties to the lower index.
 *  R5 element 2i goes to the high nibble of byte i, 2i+1 to the low nibble.
 *  R6 double quantization: offset = fl32(mean of all absmax), the sum taken
 *     in fp64 as a pairwise tree over the absmax array zero-padded to a power
 *     of two; d_b = fl32(a_b - offset); c1[g] = max |d_b| over 256 blocks;
 *     y = fl32((d_b*p) * fl32(1/(c1*p))) (prescale p as in R3; factor 0 when
 *     c1 = 0); q8 = nearest entry
 *     of t8[k] = fl32((k-127)/127), k = 0..254, ties to the lower index.
 *  R7 dequant: a' = fl32(fl32(t8[q8] * c1) + offset) (or absmax without DQ);
 *     w' = bf16_rne(fl32(nf4[code] * a')).
 *  R8 forward Y = X W'^T + s (X A^T) B^T and backward (G = dY B):
 *     dX = dY W' + s G A, dA = s G^T X, dB = s dY^T U; no dW.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no -ffast-math):
 * every fp32 operation below is one IEEE round-to-nearest operation.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* scalar helpers                                                       */
/* ------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
static float bf16_to_f32(uint16_t h) { return f32_from_bits(((uint32_t)h) << 16); }

/* fp32 -> bf16, round to nearest, ties to even (inputs are finite). */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u = bits_from_f32(f);
    uint32_t lsb = (u >> 16) & 1u;
    uint32_t rounded = u + 0x7FFFu + lsb;
    return (uint16_t)(rounded >> 16);
}

/* Standard normal CDF from libm's erfc. */
static double normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Quantile function Q(p) of N(0,1) by bisection on the CDF ([P3]/[P4]:
 * Phi^{-1}, the inverse CDF).  For p > 1/2 it uses Q(p) = -Q(1 - p) (1 - p is
 * exact there), so the bisection always runs on the lower tail where erfc of
 * a positive argument keeps full relative precision.  Runs until the bracket
 * stops shrinking. */
double oracle_normal_quantile(double p)
{
    if (p > 0.5) return -oracle_normal_quantile(1.0 - p);
    double lo = -40.0, hi = 0.0;
    for (int it = 0; it < 4000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* ------------------------------------------------------------------ */
/* code books                                                           */
/* ------------------------------------------------------------------ */

/* NF4 code book, reading R1 of [P4] sec. 4 "NF4" quantile equation with the
 * asymmetric split of [P4] ("exact 0") and [P1] sec. 2 (normalized to
 * [-1, 1]).  Sorted ascending; index 7 is the exact zero. */
void oracle_nf4_table(float out[16])
{
    const double d = 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    double qmax = oracle_normal_quantile(1.0 - d);
    double qmin = oracle_normal_quantile(d); /* negative */
    /* negative half: p = d + i*(1/2 - d)/7, i = 0..6 */
    for (int i = 0; i < 7; ++i) {
        double p = d + (double)i * ((0.5 - d) / 7.0);
        out[i] = (float)(oracle_normal_quantile(p) / -qmin);
    }
    out[7] = 0.0f;
    /* positive half: p = 1/2 + i*(1/2 - d)/8, i = 1..8 */
    for (int i = 1; i <= 8; ++i) {
        double p = (i == 8) ? 1.0 - d : 0.5 + (double)i * ((0.5 - d) / 8.0);
        out[7 + i] = (float)(oracle_normal_quantile(p) / qmax);
    }
    out[0] = -1.0f;  /* Q(d)/(-Q(d)) is exactly -1 by construction */
    out[15] = 1.0f;  /* Q(1-d)/Q(1-d) */
}

/* 8-bit code book of reading R6: t8[k] = fl32((k - 127) / 127). */
void oracle_t8_table(float out[255])
{
    for (int k = 0; k < 255; ++k) out[k] = (float)(k - 127) / 127.0f;
}

/* FP4 code book (reading R11 of [P4] sec. 6 "Float4 (FP4)"): the values of a
 * 4-bit float with 1 sign, 2 exponent and 1 mantissa bit (exponent bias 1,
 * exponent field 0 = subnormal: 0 and 0.5), i.e. magnitudes
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}, divided by the largest (6) so that they span
 * [-1, 1], each rounded to fp32, all 16 codes sorted ascending: -0 and +0
 * both appear (indices 7 and 8). */
void oracle_fp4_table(float out[16])
{
    double mag[8];
    for (int code = 0; code < 8; ++code) {
        int e = code >> 1, m = code & 1;
        mag[code] = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    }
    for (int i = 0; i < 8; ++i) {
        out[7 - i] = -(float)(mag[i] / mag[7]);  /* index 7 = -0 */
        out[8 + i] = (float)(mag[i] / mag[7]);
    }
}

/* FP8 code book of the double quantization (reading R12 of [P4] sec. 4
 * "c2^FP8"): the 253 distinct finite values of the 8-bit float E4M3 (1 sign,
 * 4 exponent, 3 mantissa bits, bias 7, exponent field 0 = subnormal; the
 * all-ones exponent with all-ones mantissa is not a number, so the largest
 * value is 1.75 * 2^8 = 448), divided by 448, rounded to fp32, sorted
 * ascending; -0 and +0 count once.  Returns the count (253). */
int oracle_e4m3_table(float out[256])
{
    double pos[127];
    int np = 0;
    for (int e = 0; e < 16; ++e)
        for (int m = 0; m < 8; ++m) {
            if (e == 15 && m == 7) continue;        /* not a number */
            if (e == 0 && m == 0) continue;         /* zero, added once below */
            pos[np++] = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
        }
    /* pos is ascending by construction */
    int k = 0;
    for (int i = np - 1; i >= 0; --i) out[k++] = (float)(-pos[i] / 448.0);
    out[k++] = 0.0f;
    for (int i = 0; i < np; ++i) out[k++] = (float)(pos[i] / 448.0);
    return k;
}

/* Brute-force nearest entry of a sorted table, distances in fp64,
 * exact ties to the lower index (readings R4 and R6). */
static int nearest_index(float x, const float *tab, int n)
{
    int best = 0;
    double bd = fabs((double)x - (double)tab[0]);
    for (int j = 1; j < n; ++j) {
        double dj = fabs((double)x - (double)tab[j]);
        if (dj < bd) { bd = dj; best = j; }
    }
    return best;
}

int oracle_nf4_nearest(float x)
{
    float nf4[16];
    oracle_nf4_table(nf4);
    return nearest_index(x, nf4, 16);
}

int oracle_t8_nearest(float y)
{
    float t8[255];
    oracle_t8_table(t8);
    return nearest_index(y, t8, 255);
}

/* Nearest NF4 codes of n consecutive fp32 bit patterns starting at `start`
 * (one code per byte).  Used to pin the GPU's fast search exhaustively. */
void oracle_nf4_nearest_bits(uint32_t start, int64_t n, uint8_t *codes)
{
    float nf4[16];
    oracle_nf4_table(nf4);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        codes[i] = (uint8_t)nearest_index(f32_from_bits(start + (uint32_t)i), nf4, 16);
}

/* Nearest entry of the 8-bit code book dq_type (0 linear, 1 E4M3) of n
 * consecutive fp32 bit patterns from `start` (brute force over the table,
 * distances in fp64, ties to the lower index).  Pins the GPU's search. */
void oracle_dq_nearest_bits(uint32_t start, int64_t n, int dq_type, uint8_t *codes)
{
    float tab[256];
    int nt;
    if (dq_type == 1) nt = oracle_e4m3_table(tab);
    else { oracle_t8_table(tab); nt = 255; }
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        codes[i] = (uint8_t)nearest_index(f32_from_bits(start + (uint32_t)i), tab, nt);
}

/* ------------------------------------------------------------------ */
/* quantize                                                             */
/* ------------------------------------------------------------------ */

static double pairwise_sum_padded(const float *v, int64_t n)
{
    if (n == 0) return 0.0;
    int64_t p = 1;
    while (p < n) p <<= 1;
    double *t = (double *)calloc((size_t)p, sizeof(double));
    for (int64_t i = 0; i < n; ++i) t[i] = (double)v[i];
    for (int64_t len = p; len > 1; len >>= 1)
        for (int64_t i = 0; i < len / 2; ++i) t[i] = t[2 * i] + t[2 * i + 1];
    double s = t[0];
    free(t);
    return s;
}

/*
 * Blockwise NF4 quantization with optional double quantization.
 *   w      : n input values; bf16 bits when is_bf16, else fp32
 *   codes  : ceil(n/2) bytes (R5)
 *   absmax : ceil(n/64) fp32 block maxima (always written)
 *   q8, c1, offset : written when double_quant (R6); c1 has ceil(nb/256)
 * [P1] sec. 2: rescale a block by its absolute maximum into [-1, 1], map each
 * weight to the nearest code, store the 4-bit index.  [P2]/[P4]: 64
 * parameters share one constant, and the constants are quantized again to
 * 8 bits with one fp32 constant per 256 of them.
 */
/* The 16-value code book of a 4-bit code type (0: NF4, 1: FP4) and the 8-bit
 * code book of a double-quantization type (0: linear t8, 255 values; 1: FP8
 * E4M3, 253 values); the latter returns its size. */
static void code_table(int code_type, float out[16])
{
    if (code_type == 1) oracle_fp4_table(out); else oracle_nf4_table(out);
}

static int dq_table(int dq_type, float out[256])
{
    if (dq_type == 1) return oracle_e4m3_table(out);
    oracle_t8_table(out);
    return 255;
}

/*
 * Blockwise 4-bit quantization with optional double quantization, for any
 * block size (64, 128 or 256 consecutive elements share one constant), code
 * type and double-quantization code book; oracle_nf4_quantize is the case
 * (64, NF4, linear 8-bit).  Same steps and readings as below.
 */
void oracle_quantize_ex(const void *w, int is_bf16, int64_t n, int double_quant, int blocksize,
                        int code_type, int dq_type, uint8_t *codes, float *absmax, uint8_t *q8,
                        float *c1, float *offset);

void oracle_nf4_quantize(const void *w, int is_bf16, int64_t n, int double_quant,
                         uint8_t *codes, float *absmax, uint8_t *q8, float *c1,
                         float *offset)
{
    oracle_quantize_ex(w, is_bf16, n, double_quant, 64, 0, 0, codes, absmax, q8, c1, offset);
}

void oracle_quantize_ex(const void *w, int is_bf16, int64_t n, int double_quant, int blocksize,
                        int code_type, int dq_type, uint8_t *codes, float *absmax, uint8_t *q8,
                        float *c1, float *offset)
{
    float nf4[16];
    code_table(code_type, nf4);
    const int64_t bs = blocksize;
    const int64_t nb = (n + bs - 1) / bs;
    memset(codes, 0, (size_t)((n + 1) / 2));

    #pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        int64_t lo = b * bs, hi = lo + bs < n ? lo + bs : n;
        float vals[256];
        float a = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            float v = is_bf16 ? bf16_to_f32(((const uint16_t *)w)[i]) : ((const float *)w)[i];
            vals[i - lo] = v;
            float av = fabsf(v);
            if (av > a) a = av;
        }
        absmax[b] = a;
        float p = (a < FLT_MIN) ? 0x1p64f : 1.0f;
        float rcp = (a == 0.0f) ? 0.0f : 1.0f / (a * p);
        for (int64_t i = lo; i < hi; ++i) {
            float x = (vals[i - lo] * p) * rcp;
            int c = nearest_index(x, nf4, 16);
            /* element 2j -> high nibble of byte j; blocks hold an even count
             * of elements except a last odd one, so bytes are never shared
             * between blocks */
            if ((i & 1) == 0) codes[i >> 1] |= (uint8_t)(c << 4);
            else              codes[i >> 1] |= (uint8_t)c;
        }
    }
    if (!double_quant) return;

    float t8[256];
    const int nt8 = dq_table(dq_type, t8);
    double sum = pairwise_sum_padded(absmax, nb);
    float off = (nb > 0) ? (float)(sum / (double)nb) : 0.0f;
    *offset = off;
    const int64_t nb2 = (nb + 255) / 256;
    #pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < nb2; ++g) {
        int64_t lo = g * 256, hi = lo + 256 < nb ? lo + 256 : nb;
        float c = 0.0f;
        for (int64_t b = lo; b < hi; ++b) {
            float d = absmax[b] - off;
            if (fabsf(d) > c) c = fabsf(d);
        }
        c1[g] = c;
        float p = (c < FLT_MIN) ? 0x1p64f : 1.0f;
        float rc = (c == 0.0f) ? 0.0f : 1.0f / (c * p);
        for (int64_t b = lo; b < hi; ++b) {
            float d = absmax[b] - off;
            float y = (d * p) * rc;
            q8[b] = (uint8_t)nearest_index(y, t8, nt8);
        }
    }
}

/* Per-block constant a' of reading R7. */
static float block_scale(int64_t b, int double_quant, const float *absmax,
                         const uint8_t *q8, const float *c1, float offset,
                         const float *t8)
{
    if (!double_quant) return absmax[b];
    float t = t8[q8[b]] * c1[b / 256];
    return t + offset;
}

/* doubleDequant of [P4] sec. 4: dequant(dequant(c1, c2), W) = W^BF16, for
 * any block size, code type and double-quantization code book.
 * Writes n bf16 values (bits). */
void oracle_dequantize_ex(int64_t n, int double_quant, int blocksize, int code_type, int dq_type,
                          const uint8_t *codes, const float *absmax, const uint8_t *q8,
                          const float *c1, float offset, uint16_t *out)
{
    float nf4[16], t8[256];
    code_table(code_type, nf4);
    dq_table(dq_type, t8);
    const int64_t bs = blocksize;
    const int64_t nb = (n + bs - 1) / bs;
    #pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        float a = block_scale(b, double_quant, absmax, q8, c1, offset, t8);
        int64_t lo = b * bs, hi = lo + bs < n ? lo + bs : n;
        for (int64_t i = lo; i < hi; ++i) {
            uint8_t byte = codes[i >> 1];
            int c = (i & 1) ? (byte & 15) : (byte >> 4);
            out[i] = f32_to_bf16_rne(nf4[c] * a);
        }
    }
}

void oracle_nf4_dequantize(int64_t n, int double_quant, const uint8_t *codes,
                           const float *absmax, const uint8_t *q8, const float *c1,
                           float offset, uint16_t *out)
{
    oracle_dequantize_ex(n, double_quant, 64, 0, 0, codes, absmax, q8, c1, offset, out);
}

/* ------------------------------------------------------------------ */
/* linear forward / backward in fp64                                   */
/* ------------------------------------------------------------------ */

/*
 * Forward of [P5] "LoRA formula and tensor shapes" with W0 replaced by the
 * dequantized frozen weight ([P4] full equation):
 *   U[m,j] = sum_k X[m,k] A[j,k]
 *   Y[m,n] = sum_k X[m,k] W[n,k] + s * sum_j U[m,j] B[n,j]
 * All inputs are bf16 bits; every sum runs in fp64 in index order.
 * rows (length nrows) selects which rows of Y to compute; NULL means all M.
 * Y is [nrows, N] fp64.
 */
void oracle_linear_fwd(int64_t M, int64_t N, int64_t K, int r, double s,
                       const uint16_t *X, const uint16_t *W, const uint16_t *A,
                       const uint16_t *B, const int64_t *rows, int64_t nrows,
                       double *Y)
{
    if (!rows) nrows = M;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t ii = 0; ii < nrows; ++ii) {
        int64_t m = rows ? rows[ii] : ii;
        double *u = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)bf16_to_f32(X[m * K + k]) * (double)bf16_to_f32(A[(int64_t)j * K + k]);
            u[j] = acc;
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)bf16_to_f32(X[m * K + k]) * (double)bf16_to_f32(W[n * K + k]);
            double lora = 0.0;
            for (int j = 0; j < r; ++j)
                lora += u[j] * (double)bf16_to_f32(B[n * r + j]);
            Y[ii * N + n] = acc + s * lora;
        }
        free(u);
    }
}

/*
 * Backward of the same layer ([P4] steps 4: gradients pass through W^BF16
 * to the adapters only; [P5] invariant: the frozen weight has no gradient).
 *   G[m,j]  = sum_n dY[m,n] B[n,j]
 *   dX[m,k] = sum_n dY[m,n] W[n,k] + s * sum_j G[m,j] A[j,k]
 *   dA[j,k] = s * sum_m G[m,j] X[m,k]
 *   dB[n,j] = s * sum_m dY[m,n] U[m,j],  U[m,j] = sum_k X[m,k] A[j,k]
 * dX is computed for the selected rows only ([nrows, K]); dA [r,K] and
 * dB [N,r] always over all M rows.  Pass dX = NULL to skip it.
 */
void oracle_linear_bwd(int64_t M, int64_t N, int64_t K, int r, double s,
                       const uint16_t *dY, const uint16_t *X, const uint16_t *W,
                       const uint16_t *A, const uint16_t *B, const int64_t *rows,
                       int64_t nrows, double *dX, double *dA, double *dB)
{
    double *G = (double *)calloc((size_t)(M * r + 1), sizeof(double));
    double *U = (double *)calloc((size_t)(M * r + 1), sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int j = 0; j < r; ++j) {
            double g = 0.0, u = 0.0;
            for (int64_t n = 0; n < N; ++n)
                g += (double)bf16_to_f32(dY[m * N + n]) * (double)bf16_to_f32(B[n * r + j]);
            for (int64_t k = 0; k < K; ++k)
                u += (double)bf16_to_f32(X[m * K + k]) * (double)bf16_to_f32(A[(int64_t)j * K + k]);
            G[m * r + j] = g;
            U[m * r + j] = u;
        }
    }
    if (dX) {
        if (!rows) nrows = M;
        #pragma omp parallel for schedule(dynamic, 1)
        for (int64_t ii = 0; ii < nrows; ++ii) {
            int64_t m = rows ? rows[ii] : ii;
            double *acc = (double *)calloc((size_t)K, sizeof(double));
            /* the sum over n for each dX[m,k] still runs in index order */
            for (int64_t n = 0; n < N; ++n) {
                double g = (double)bf16_to_f32(dY[m * N + n]);
                for (int64_t k = 0; k < K; ++k)
                    acc[k] += g * (double)bf16_to_f32(W[n * K + k]);
            }
            for (int64_t k = 0; k < K; ++k) {
                double lora = 0.0;
                for (int j = 0; j < r; ++j)
                    lora += G[m * r + j] * (double)bf16_to_f32(A[(int64_t)j * K + k]);
                dX[ii * K + k] = acc[k] + s * lora;
            }
            free(acc);
        }
    }
    /* dA and dB: each output element sums over m = 0..M-1 in index order;
     * the loops run m outermost only so that rows are read contiguously. */
    #pragma omp parallel for schedule(static)
    for (int64_t k0 = 0; k0 < K; k0 += 64) {
        int64_t k1 = k0 + 64 < K ? k0 + 64 : K;
        double *acc = (double *)calloc((size_t)(r * 64 + 1), sizeof(double));
        for (int64_t m = 0; m < M; ++m)
            for (int j = 0; j < r; ++j) {
                double g = G[m * r + j];
                for (int64_t k = k0; k < k1; ++k)
                    acc[j * 64 + (k - k0)] += g * (double)bf16_to_f32(X[m * K + k]);
            }
        for (int j = 0; j < r; ++j)
            for (int64_t k = k0; k < k1; ++k)
                dA[(int64_t)j * K + k] = s * acc[j * 64 + (k - k0)];
        free(acc);
    }
    #pragma omp parallel for schedule(static)
    for (int64_t n0 = 0; n0 < N; n0 += 64) {
        int64_t n1 = n0 + 64 < N ? n0 + 64 : N;
        double *acc = (double *)calloc((size_t)(r * 64 + 1), sizeof(double));
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = n0; n < n1; ++n) {
                double g = (double)bf16_to_f32(dY[m * N + n]);
                for (int j = 0; j < r; ++j)
                    acc[(n - n0) * r + j] += g * U[m * r + j];
            }
        for (int64_t n = n0; n < n1; ++n)
            for (int j = 0; j < r; ++j)
                dB[n * r + j] = s * acc[(n - n0) * r + j];
        free(acc);
    }
    free(G);
    free(U);
}

/* ------------------------------------------------------------------ */
/* LoRA merge / unmerge                                                 */
/* ------------------------------------------------------------------ */

/* double -> bf16 with one round-to-nearest-even step: the value is scaled by
 * a power of two so that its bf16 unit in the last place becomes 1 (8
 * significant bits; below 2^-126 the subnormal spacing 2^-133), rounded with
 * nearbyint (ties to even in the default rounding mode) and scaled back;
 * both scalings are exact.  The result has at most 8 significant bits, so
 * the conversion to fp32 is exact and its top 16 bits are the bf16 code. */
static uint16_t f64_to_bf16_rne(double x)
{
    if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
    double ax = fabs(x);
    int e;
    frexp(ax, &e);          /* ax = m 2^e, m in [1/2, 1) */
    int ulp_exp = e - 8;
    if (ulp_exp < -133) ulp_exp = -133;
    double v = ldexp(nearbyint(ldexp(ax, -ulp_exp)), ulp_exp);
    uint16_t h = (uint16_t)(bits_from_f32((float)v) >> 16);
    return signbit(x) ? (uint16_t)(h | 0x8000u) : h;
}

/*
 * LoRA merge ([P2] pitfalls: dequantize the 4-bit base before merging; [P5]
 * "LoRA formula and tensor shapes": the adapter adds (alpha/r) B A to W0):
 *   out[n,k] = bf16_rne( W[n,k] + sign * s * sum_j B[n,j] A[j,k] )
 * W [N,K] (the dequantized base for a merge, the merged weight for an
 * unmerge with sign = -1), A [r,K], B [N,r]: bf16 bits.  The sum runs in
 * fp64 in index order and the value is rounded once.  `exact` (optional)
 * receives the fp64 value before the rounding.
 */
void oracle_lora_merge(int64_t N, int64_t K, int r, double s, int sign, const uint16_t *W,
                       const uint16_t *A, const uint16_t *B, uint16_t *out, double *exact)
{
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double acc = 0.0;
            for (int j = 0; j < r; ++j)
                acc += (double)bf16_to_f32(B[n * r + j]) * (double)bf16_to_f32(A[(int64_t)j * K + k]);
            double v = (double)bf16_to_f32(W[n * K + k]) + (double)sign * s * acc;
            out[n * K + k] = f64_to_bf16_rne(v);
            if (exact) exact[n * K + k] = v;
        }
    }
}

/* ------------------------------------------------------------------ */
/* optimizer step of the adapters                                       */
/* ------------------------------------------------------------------ */

/*
 * AdamW ([P4] sec. 4 steps: Adam updates L1 and L2 only) with decoupled
 * weight decay and bias correction at step t >= 1, in fp64:
 *   g = grad * grad_scale
 *   p <- p (1 - lr wd)
 *   m <- b1 m + (1 - b1) g,  v <- b2 v + (1 - b2) g^2
 *   p <- p - lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 */
void oracle_adamw_step(int64_t n, double lr, double b1, double b2, double eps, double wd,
                       double grad_scale, int64_t t, double *p, double *m, double *v,
                       const double *grad)
{
    const double bc1 = 1.0 - pow(b1, (double)t);
    const double bc2 = 1.0 - pow(b2, (double)t);
    for (int64_t i = 0; i < n; ++i) {
        double g = grad[i] * grad_scale;
        p[i] = p[i] * (1.0 - lr * wd);
        m[i] = b1 * m[i] + (1.0 - b1) * g;
        v[i] = b2 * v[i] + (1.0 - b2) * g * g;
        p[i] = p[i] - lr * (m[i] / bc1) / (sqrt(v[i] / bc2) + eps);
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

/* Number of OpenMP threads the oracle's loops use from now on (n >= 1);
 * used to time the oracle on one core beside all of them. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
