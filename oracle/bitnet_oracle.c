/*
 * bitnet_oracle.c -- plain, slow CPU oracle for the BitLinear forward (W1.58A8).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant generator with the
 * CUDA library.
 *
 * Source of truth: the "BitNet" model page of the transformers documentation
 * (five translated copies of one page).  Its section "Model details", item
 * "Quantization", states the scheme:
 *   - weights are quantised to the ternary values {-1, 0, +1} with absmean
 *     quantisation;
 *   - activations are quantised to 8-bit integers with absmax quantisation,
 *     per token;
 *   - the pair is called W1.58A8.
 * Item "Architecture" of the same section says the linear layers are BitLinear
 * layers, carry no bias, and that the FFN uses squared ReLU (ReLU^2); the
 * BitNetConfig section gives hidden_act = "relu2".  Section "Model variants"
 * says the deployable checkpoint stores the 1.58-bit weights packed.
 *
 * The page gives no formulas.  This oracle takes the plainest reading:
 *   gamma  = mean |W| over the whole weight matrix (one scale per matrix)
 *   W_q    = clamp(round(W / (gamma + eps)), -1, 1), eps = 1e-5
 *   s_m    = 127 / max_k |x_mk|      (one scale per token = per row of x)
 *   x_q    = clamp(round(x * s_m), -128, 127)
 *   acc    = x_q . W_q^T             (exact integers)
 *   y      = acc * gamma / s_m
 *   h      = relu(g)^2 * u           (gated FFN: g, u are two BitLinear outputs)
 * "round" is round-half-to-even everywhere.
 *
 * Precision.  The page fixes none.  The quantisers decide integers, so they are
 * evaluated in IEEE binary32 exactly as written (one fp32 division for s, one
 * fp32 product x*s rounded once, then round-half-to-even to an integer; one
 * fp32 add for gamma+eps, one fp32 division W/(gamma+eps)); the GPU takes the
 * same decisions in the same precision.  gamma is accumulated in binary64 in a
 * fixed order (each row left to right, then the row sums top to bottom) and
 * rounded once to binary32.  Everything that does not decide an integer
 * (dequantisation, the ReLU^2 gate) is computed in binary64.
 *
 * Special cases (the page is silent): an all-zero row has max|x| = 0; the
 * divisor is clamped to 1e-5 so s is finite and x_q = 0.  Inputs are required
 * to be finite.
 *
 * Packed layout (the page only says "packed"; this layout is this project's
 * choice): code c = W_q + 1 in {0, 1, 2}.  Row n occupies bytes
 * [n*K/4, (n+1)*K/4).  Weights are grouped by 16; group g of row n is the
 * little-endian 32-bit word at byte offset n*K/4 + 4*g, and weight
 * k = 16*g + 4*j + b (j, b in 0..3) sits in byte b at bits 2*j .. 2*j+1.
 * K must be a multiple of 16 here (the library requires a multiple of 64).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_QUANT_EPS 1e-5f /* floor of max|x| and additive eps of gamma */

/* ---- bf16 input ------------------------------------------------------- */

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
void oracle_bf16_to_f32(const uint16_t *src, int64_t count, float *dst)
{
    for (int64_t i = 0; i < count; ++i) {
        uint32_t bits = ((uint32_t)src[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        dst[i] = f;
    }
}

/* ---- absmean weight ternarisation (page: "absmean", ternary) --------- */

/* mean |W| in binary64: each row summed left to right, then the row sums
 * summed top to bottom, divided by N*K.  Returned unrounded. */
double oracle_absmean_f64(const float *w, int64_t n_rows, int64_t k_cols)
{
    double total = 0.0;
    for (int64_t n = 0; n < n_rows; ++n) {
        double row = 0.0;
        for (int64_t k = 0; k < k_cols; ++k)
            row += fabs((double)w[n * k_cols + k]);
        total += row;
    }
    return total / (double)(n_rows * k_cols);
}

/* gamma as stored: the binary64 mean rounded once to binary32. */
float oracle_gamma(const float *w, int64_t n_rows, int64_t k_cols)
{
    return (float)oracle_absmean_f64(w, n_rows, k_cols);
}

/* W_q = clamp(round_half_even(W / (gamma + eps)), -1, 1), fp32 arithmetic. */
void oracle_ternarize(const float *w, int64_t n_rows, int64_t k_cols,
                      float gamma, float eps, int8_t *w_q)
{
    const float d = gamma + eps;
    for (int64_t i = 0; i < n_rows * k_cols; ++i) {
        float q = nearbyintf(w[i] / d);
        if (q > 1.0f) q = 1.0f;
        if (q < -1.0f) q = -1.0f;
        w_q[i] = (int8_t)q;
    }
}

/* ---- 2-bit packing (page: "packed" 1.58-bit weights; layout ours) ---- */

void oracle_pack(const int8_t *w_q, int64_t n_rows, int64_t k_cols, uint8_t *packed)
{
    const int64_t row_bytes = k_cols / 4;
    memset(packed, 0, (size_t)(n_rows * row_bytes));
    for (int64_t n = 0; n < n_rows; ++n) {
        for (int64_t k = 0; k < k_cols; ++k) {
            int64_t group = k / 16;
            int64_t j = (k % 16) / 4;
            int64_t b = k % 4;
            uint8_t code = (uint8_t)(w_q[n * k_cols + k] + 1);
            packed[n * row_bytes + 4 * group + b] |= (uint8_t)(code << (2 * j));
        }
    }
}

/* Inverse of oracle_pack.  Returns the number of invalid codes (3) seen;
 * an invalid code decodes to 0. */
int64_t oracle_unpack(const uint8_t *packed, int64_t n_rows, int64_t k_cols, int8_t *w_q)
{
    const int64_t row_bytes = k_cols / 4;
    int64_t bad = 0;
    for (int64_t n = 0; n < n_rows; ++n) {
        for (int64_t k = 0; k < k_cols; ++k) {
            int64_t group = k / 16;
            int64_t j = (k % 16) / 4;
            int64_t b = k % 4;
            int code = (packed[n * row_bytes + 4 * group + b] >> (2 * j)) & 3;
            if (code == 3) {
                ++bad;
                code = 1;
            }
            w_q[n * k_cols + k] = (int8_t)(code - 1);
        }
    }
    return bad;
}

/* ---- per-token absmax activation quantisation (page: absmax, per token, 8-bit) */

/* x: [m_rows][k_cols] fp32 (bf16 inputs are converted exactly beforehand).
 * Writes x_q [m_rows][k_cols], s [m_rows] and, if non-NULL, rowsum [m_rows]
 * (sum of x_q over the row, used by the code-offset form of the product). */
void oracle_quant_act_amax(const float *x, int64_t m_rows, int64_t k_cols, const float *amax_in,
                           int8_t *x_q, float *s, int32_t *rowsum);

void oracle_quant_act(const float *x, int64_t m_rows, int64_t k_cols,
                      int8_t *x_q, float *s, int32_t *rowsum)
{
    oracle_quant_act_amax(x, m_rows, k_cols, NULL, x_q, s, rowsum);
}

/* Same quantiser with the per-token maximum supplied by the caller (amax_in
 * [m_rows], NULL: computed from x).  A BitLinear whose input was written by
 * another BitLinear's epilogue gets max|x| from that epilogue instead of
 * reducing the row again; given the true maximum the result is identical. */
void oracle_quant_act_amax(const float *x, int64_t m_rows, int64_t k_cols, const float *amax_in,
                           int8_t *x_q, float *s, int32_t *rowsum)
{
    for (int64_t m = 0; m < m_rows; ++m) {
        const float *row = x + m * k_cols;
        float amax = 0.0f;
        for (int64_t k = 0; k < k_cols; ++k) {
            float a = fabsf(row[k]);
            if (a > amax) amax = a;
        }
        if (amax_in) amax = amax_in[m];
        const float denom = amax > ORACLE_QUANT_EPS ? amax : ORACLE_QUANT_EPS;
        const float scale = 127.0f / denom;
        int64_t sum = 0;
        for (int64_t k = 0; k < k_cols; ++k) {
            float prod = row[k] * scale;
            float q = nearbyintf(prod);
            if (q > 127.0f) q = 127.0f;
            if (q < -128.0f) q = -128.0f;
            x_q[m * k_cols + k] = (int8_t)q;
            sum += (int64_t)q;
        }
        s[m] = scale;
        if (rowsum) rowsum[m] = (int32_t)sum;
    }
}

/* ---- exact integer contraction (implied by W1.58A8) -------------------- */

/* acc[m][n] = sum_k x_q[m][k] * w_q[n][k], accumulated in int64. */
void oracle_int_matmul(const int8_t *x_q, const int8_t *w_q,
                       int64_t m_rows, int64_t n_rows, int64_t k_cols, int64_t *acc)
{
    for (int64_t m = 0; m < m_rows; ++m) {
        for (int64_t n = 0; n < n_rows; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < k_cols; ++k)
                sum += (int64_t)x_q[m * k_cols + k] * (int64_t)w_q[n * k_cols + k];
            acc[m * n_rows + n] = sum;
        }
    }
}

/* Same contraction restricted to a list of (m, n) output coordinates, for
 * spot checks on problems too large to contract in full. */
void oracle_int_dot_samples(const int8_t *x_q, const int8_t *w_q, int64_t k_cols,
                            const int64_t *m_idx, const int64_t *n_idx, int64_t count,
                            int64_t *acc)
{
    for (int64_t i = 0; i < count; ++i) {
        const int8_t *xr = x_q + m_idx[i] * k_cols;
        const int8_t *wr = w_q + n_idx[i] * k_cols;
        int64_t sum = 0;
        for (int64_t k = 0; k < k_cols; ++k)
            sum += (int64_t)xr[k] * (int64_t)wr[k];
        acc[i] = sum;
    }
}

/* ---- dequantising epilogue -------------------------------------------- */

/* y[m][n] = acc[m][n] * gamma / s[m], in binary64. */
void oracle_dequant(const int64_t *acc, const float *s, float gamma,
                    int64_t m_rows, int64_t n_rows, double *y)
{
    for (int64_t m = 0; m < m_rows; ++m)
        for (int64_t n = 0; n < n_rows; ++n)
            y[m * n_rows + n] = (double)acc[m * n_rows + n] * (double)gamma / (double)s[m];
}

/* ---- ReLU^2-gated FFN epilogue (page: ReLU^2 in the FFN, hidden_act relu2) */

/* h = relu(g)^2 * u, elementwise, binary64. */
void oracle_relu2_gate(const double *g, const double *u, int64_t count, double *h)
{
    for (int64_t i = 0; i < count; ++i) {
        double r = g[i] > 0.0 ? g[i] : 0.0;
        h[i] = r * r * u[i];
    }
}

/* ---- RMS normalisation in front of the activation quantiser ------------- */

/* Page, "Model details" / "Architecture": the model uses subln normalisation
 * and no bias terms in its normalisation layers; BitNetConfig: rms_norm_eps =
 * 1e-5, the epsilon of the rms normalisation layers.  Reading (the page gives
 * no formula): y = x / sqrt(mean_k(x_k^2) + eps) * g, with a per-feature
 * weight g and no bias; BitLinear then quantises y per token as above.
 *
 * Precision (the page is silent; one ulp in 1/rms can move a quantised code,
 * so this reading fixes it):
 *   ss  = sum_k x_k^2, the exact sum (every x_k^2 of a binary32 value is an
 *         exact binary64 number), rounded ONCE to the nearest binary64, ties
 *         to even -- the correctly rounded sum, independent of any order;
 *   r   = (float)(1 / sqrt(ss / K + eps)), every step in binary64 (correctly
 *         rounded division and square root), rounded once to binary32;
 *   y_k = (x_k * r) * g_k in binary32, two roundings in this order.
 *
 * The exact sum is kept as an integer.  A finite binary32 value is
 * v = +-mant * 2^(e - 150) with mant < 2^24 an integer and e the biased
 * exponent field (e = 1 for subnormals, whose mant has no hidden bit), so
 * v^2 = mant^2 * 2^(2e - 2) * 2^-298: an integer multiple of 2^-298 below
 * 2^256.  The integers mant^2 * 2^(2e - 2) are added into a long accumulator
 * of SS_DIGITS little-endian 32-bit digits (640 bits; 2^31 terms need at most
 * 587), then the accumulator is rounded to 53 significant bits. */
#define SS_DIGITS 20

/* acc += mant2 * 2^shift, carries propagated (mant2 < 2^48, shift < 512) */
static void ss_add(uint32_t *acc, uint64_t mant2, int shift)
{
    const int d = shift / 32, b = shift % 32;
    const uint64_t lo = mant2 << b;                  /* bits 0..63 of mant2 * 2^b */
    const uint64_t hi = b ? mant2 >> (64 - b) : 0;    /* bits 64..79 */
    const uint32_t piece[3] = {(uint32_t)lo, (uint32_t)(lo >> 32), (uint32_t)hi};
    uint64_t carry = 0;
    for (int i = 0; d + i < SS_DIGITS; ++i) {
        const uint64_t t = (uint64_t)acc[d + i] + (i < 3 ? piece[i] : 0) + carry;
        acc[d + i] = (uint32_t)t;
        carry = t >> 32;
        if (i >= 2 && carry == 0) break;
    }
}

static int ss_bit(const uint32_t *acc, int i) { return (int)((acc[i / 32] >> (i % 32)) & 1u); }

/* the accumulator times 2^-298, rounded to the nearest binary64, ties to even */
static double ss_round(const uint32_t *acc)
{
    int top = -1; /* position of the highest set bit */
    for (int i = 32 * SS_DIGITS - 1; i >= 0 && top < 0; --i)
        if (ss_bit(acc, i)) top = i;
    if (top < 0) return 0.0;
    const int sh = top > 52 ? top - 52 : 0; /* bits below the 53 kept ones */
    uint64_t mant = 0;
    for (int i = top; i >= sh; --i) mant = (mant << 1) | (uint64_t)ss_bit(acc, i);
    if (sh > 0) {
        const int round = ss_bit(acc, sh - 1);
        int sticky = 0;
        for (int i = 0; i < sh - 1; ++i) sticky |= ss_bit(acc, i);
        if (round && (sticky || (mant & 1u))) mant += 1; /* mant <= 2^53: exact in binary64 */
    }
    return ldexp((double)mant, sh - 298);
}

double oracle_sumsq(const float *row, int64_t k_cols)
{
    uint32_t acc[SS_DIGITS];
    memset(acc, 0, sizeof(acc));
    for (int64_t k = 0; k < k_cols; ++k) {
        uint32_t bits;
        memcpy(&bits, &row[k], 4);
        const int field = (int)((bits >> 23) & 0xffu);
        const uint64_t mant = (bits & 0x7fffffu) | (field ? 0x800000u : 0u);
        const int e = field ? field : 1;
        ss_add(acc, mant * mant, 2 * e - 2);
    }
    return ss_round(acc);
}

/* x, y: [m_rows][k_cols]; g: [k_cols]; r_out: [m_rows] (may be NULL). */
void oracle_rmsnorm(const float *x, const float *g, int64_t m_rows, int64_t k_cols, float eps, float *y,
                    float *r_out)
{
    for (int64_t m = 0; m < m_rows; ++m) {
        const float *row = x + m * k_cols;
        const double ss = oracle_sumsq(row, k_cols);
        const float r = (float)(1.0 / sqrt(ss / (double)k_cols + (double)eps));
        for (int64_t k = 0; k < k_cols; ++k) {
            const float xr = row[k] * r;
            y[m * k_cols + k] = xr * g[k];
        }
        if (r_out) r_out[m] = r;
    }
}

/* ---- fp32 epilogue, bf16 outputs and the emitted per-token maximum ------ */

/* Page, "Model details" / "Quantization": the integer product is rescaled by
 * gamma / s.  The page fixes no output precision.  Reading, so that an output
 * stored in fp32 or bf16 is one well-defined number:
 *   r   = fl32(gamma / s)                 (one correctly rounded division)
 *   y32 = fl32(acc * r)                   (acc is an integer, |acc| < 2^24,
 *                                          so it converts to binary32 exactly)
 * and for the gated FFN (page, "Architecture": ReLU^2 in the FFN)
 *   h32 = fl32(fl32(p * p) * u32),  p = max(g32, 0),  g32, u32 as y32;
 * a bf16 output is y32 (h32) rounded to the nearest bf16, ties to even. */
void oracle_epilogue_f32(const int64_t *acc_g, const int64_t *acc_u, const float *s, float gamma_g,
                         float gamma_u, int64_t m_rows, int64_t n_rows, float *y)
{
    for (int64_t m = 0; m < m_rows; ++m) {
        const float rg = gamma_g / s[m];
        const float ru = gamma_u / s[m];
        for (int64_t n = 0; n < n_rows; ++n) {
            const int64_t i = m * n_rows + n;
            const float g = (float)acc_g[i] * rg;
            if (!acc_u) {
                y[i] = g;
                continue;
            }
            const float u = (float)acc_u[i] * ru;
            const float p = g > 0.0f ? g : 0.0f;
            const float pp = p * p;
            y[i] = pp * u;
        }
    }
}

/* binary32 -> bfloat16 (the upper half of the binary32 encoding), rounded to
 * nearest with ties to even; a NaN stays a (quiet) NaN. */
static uint16_t oracle_f32_to_bf16_one(float v)
{
    uint32_t bits;
    memcpy(&bits, &v, sizeof bits);
    if ((bits & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((bits >> 16) | 0x0040u);
    uint32_t upper = bits >> 16;
    const uint32_t lower = bits & 0xffffu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

void oracle_f32_to_bf16(const float *src, int64_t count, uint16_t *dst)
{
    for (int64_t i = 0; i < count; ++i) dst[i] = oracle_f32_to_bf16_one(src[i]);
}

/* amax[m] = max over n of |v[m][n]|, the row maxima a BitLinear epilogue
 * emits for the next quantiser (v: the values as stored, widened to fp32). */
void oracle_row_absmax(const float *v, int64_t m_rows, int64_t n_rows, float *amax)
{
    for (int64_t m = 0; m < m_rows; ++m) {
        float best = 0.0f;
        for (int64_t n = 0; n < n_rows; ++n) {
            const float a = fabsf(v[m * n_rows + n]);
            if (a > best) best = a;
        }
        amax[m] = best;
    }
}
