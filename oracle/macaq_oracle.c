/*
 * macaq_oracle.c -- plain, slow CPU oracle for the MACaQ W4A4 / MXFP4 linear layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this library. The product path (the CUDA library) shares no code, header,
 * table or helper with this file, and never calls it.
 *
 * What it computes, and where that comes from:
 *
 *   [MACaQ-fa]  Page "Huawei's research lab in Switzerland open-sources the four-bit quantization
 *               tool MACaQ for running models locally" (aipolix.com, Persian), paragraph 2: at
 *               inference each layer's activations get a per-channel scale and a small
 *               block-diagonal Hadamard transform, and the inverse is absorbed into the same
 *               layer's weights. Paragraph 3: the target format is MXFP4, W4A4.
 *   [MACaQ-en]  Page "MACaQ quantizer from huawei-csl targets GGUF, vLLM and Diffusers models"
 *               (glonce.com), paragraph 5: W4A4 dense and grouped matmul kernels.
 *   [OCP-MX]    OCP Microscaling Formats (MX) Specification v1.0: the FP32 -> MX block conversion
 *               (shared exponent floor(log2(amax)) - emax_elem with emax_elem = 2 for E2M1,
 *               E8M0 scale, round-to-nearest-even element conversion) and the E2M1 value table.
 *
 * Readings taken where the pages are silent (each one is listed in the design notes):
 *   - the Hadamard matrix is the Sylvester matrix in natural order, H[i][j] = (-1)^popcount(i&j),
 *     unnormalised; the activations get x * diag(1/s) * H and the weights get
 *     W * diag(s) * H * (1/b), so that the product equals X * W^T in exact arithmetic;
 *   - the transform is evaluated in fp32 with the butterfly order fixed below (h = 1, 2, ..., b/2),
 *     because the quantization decision (a code) is taken in the kernel's precision;
 *   - 1/s is computed once, as an IEEE fp32 division;
 *   - E8M0 exponent E = clamp(floor(log2 amax) - 2 + 127, 0, 254), E = 0 for amax = 0;
 *   - E2M1 rounding is round-to-nearest, ties to the even mantissa bit, saturating at +-6;
 *     the sign bit is kept for negative values that round to zero;
 *   - FP4 codes are packed two per byte, the lower K index in the low nibble;
 *   - the GEMM is the exact sum of dequantized products, evaluated in float64.
 *
 * Scale factors are emitted in canonical row-major order [rows, K/32]; the GPU's tiled layout is
 * the library's business, and the tests undo it before comparing.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define MX_GROUP 32

/* bf16 bit pattern -> float (exact: bf16 is the upper half of an fp32). */
static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * In-place fast Walsh-Hadamard transform of b consecutive fp32 values, in the fixed order used
 * throughout: stages h = 1, 2, 4, ..., b/2; in each stage every pair (j, j+h) with bit h of j clear
 * becomes (v[j] + v[j+h], v[j] - v[j+h]), each rounded to fp32. The result is v * H_b with H_b the
 * Sylvester Hadamard matrix (symmetric, so also H_b * v). [MACaQ-fa] paragraph 2.
 */
void oracle_fwht_f32(float *v, int b)
{
    for (int h = 1; h < b; h <<= 1) {
        for (int j = 0; j < b; ++j) {
            if ((j & h) == 0) {
                float a = v[j];
                float c = v[j + h];
                v[j] = a + c;
                v[j + h] = a - c;
            }
        }
    }
}

/*
 * The unquantized per-layer transform, one row at a time, in fp32. [MACaQ-fa] paragraph 2.
 *   activations (absorb = 0): out[r, k] = fl32(x[r, k] * mul[k]) with mul = 1/s, then H_b on each
 *                             aligned block of b channels;
 *   weights     (absorb = 1): out[r, k] = fl32(w[r, k] * mul[k]) with mul = s, then H_b, then the
 *                             exact factor 1/b (a power of two).
 * mul == NULL means a scale of 1 (no per-channel scale); b == 1 means no Hadamard (plain MXFP4).
 */
void oracle_transform_rows(const uint16_t *x_bf16, const float *mul, int64_t rows, int64_t K,
                           int b, int absorb, float *out)
{
    for (int64_t r = 0; r < rows; ++r) {
        float *o = out + r * K;
        const uint16_t *x = x_bf16 + r * K;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_float(x[k]);
            o[k] = mul ? v * mul[k] : v;
        }
        if (b > 1) {
            for (int64_t k0 = 0; k0 < K; k0 += b)
                oracle_fwht_f32(o + k0, b);
            if (absorb) {
                float inv_b = 1.0f / (float)b; /* exact: b is a power of two */
                for (int64_t k = 0; k < K; ++k)
                    o[k] = o[k] * inv_b;
            }
        }
    }
}

/*
 * Shared E8M0 exponent of one 32-element group. [OCP-MX]: shared exponent
 * floor(log2(amax)) - emax_elem, emax_elem = 2 for E2M1, stored with bias 127 and clamped to the
 * representable range [0, 254] (255 is NaN). floor(log2) is read from frexp, which normalises
 * subnormals. amax == 0 gives E = 0.
 */
int oracle_e8m0_exponent(float amax)
{
    if (amax == 0.0f)
        return 0;
    int e2;
    (void)frexpf(amax, &e2); /* amax = f * 2^e2, f in [0.5, 1): floor(log2 amax) = e2 - 1 */
    int E = (e2 - 1) - 2 + 127;
    if (E < 0)
        E = 0;
    if (E > 254)
        E = 254;
    return E;
}

/*
 * E2M1 code of an fp32 value already divided by the block scale. [OCP-MX] E2M1 table:
 * magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} have codes 0..7 (exponent bits 2..1, mantissa bit 0),
 * bit 3 is the sign. Rounding is to nearest; a tie goes to the even mantissa bit; magnitudes above 6
 * saturate to 6. Inside each binade the grid is a uniform lattice whose index parity equals the
 * mantissa bit, so rint() (round-half-even) on the lattice index is exactly that rule.
 */
uint8_t oracle_e2m1_code(float t)
{
    uint8_t sign = signbit(t) ? 8u : 0u;
    float a = fabsf(t);
    float q; /* the chosen grid magnitude */
    if (a < 2.0f)
        q = rintf(a * 2.0f) * 0.5f; /* spacing 0.5 on [0, 2] */
    else if (a < 4.0f)
        q = rintf(a); /* spacing 1 on [2, 4] */
    else if (a <= 6.0f)
        q = rintf(a * 0.5f) * 2.0f; /* spacing 2 on [4, 6] */
    else
        q = 6.0f; /* saturate */
    uint8_t mag;
    if (q == 0.0f) mag = 0;
    else if (q == 0.5f) mag = 1;
    else if (q == 1.0f) mag = 2;
    else if (q == 1.5f) mag = 3;
    else if (q == 2.0f) mag = 4;
    else if (q == 3.0f) mag = 5;
    else if (q == 4.0f) mag = 6;
    else mag = 7; /* 6.0 */
    return (uint8_t)(sign | mag);
}

/* E2M1 code -> value (float64, exact). [OCP-MX] E2M1 table. */
double oracle_e2m1_value(uint8_t code)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[code & 7u];
    return (code & 8u) ? -v : v;
}

/*
 * MXFP4 quantization of one row of K fp32 values (K a multiple of 32): for each group of 32
 * contiguous values, the E8M0 exponent from the group's amax, then each element divided by the
 * scale 2^(E-127) (an exact power of two, formed with ldexpf) and converted to E2M1; codes are
 * packed two per byte, the even index in the low nibble. [OCP-MX]; [MACaQ-fa] paragraph 3.
 */
void oracle_mxfp4_quantize_row(const float *y, int64_t K, uint8_t *codes, uint8_t *sf)
{
    for (int64_t g = 0; g < K / MX_GROUP; ++g) {
        const float *v = y + g * MX_GROUP;
        float amax = 0.0f;
        for (int i = 0; i < MX_GROUP; ++i) {
            float a = fabsf(v[i]);
            if (a > amax)
                amax = a;
        }
        int E = oracle_e8m0_exponent(amax);
        sf[g] = (uint8_t)E;
        float inv_scale = ldexpf(1.0f, 127 - E); /* 2^(127-E), exact, 127-E in [-127, 127] */
        for (int i = 0; i < MX_GROUP; i += 2) {
            uint8_t lo = oracle_e2m1_code(v[i] * inv_scale);
            uint8_t hi = oracle_e2m1_code(v[i + 1] * inv_scale);
            codes[(g * MX_GROUP + i) / 2] = (uint8_t)(lo | (hi << 4));
        }
    }
}

/*
 * Offline weight preparation. [MACaQ-fa] paragraph 2 (absorb the inverse transform into the same
 * layer's weights): W' = MXFP4(W * diag(s) * H_b * (1/b)), row by row along K, plus inv_s = 1/s
 * (IEEE fp32 division) for the activation side.
 *   W [N, K] bf16 bits, s [K] fp32 (NULL: no scale) -> Wq [N, K/2], Wsf [N, K/32] row-major,
 *   inv_s [K] (skipped when s or inv_s is NULL).
 * work: N*K floats of scratch owned by the caller.
 */
void oracle_prep_weights(const uint16_t *W, const float *s, int64_t N, int64_t K, int b,
                         uint8_t *Wq, uint8_t *Wsf, float *inv_s, float *work)
{
    oracle_transform_rows(W, s, N, K, b, 1, work);
    for (int64_t n = 0; n < N; ++n)
        oracle_mxfp4_quantize_row(work + n * K, K, Wq + n * (K / 2), Wsf + n * (K / MX_GROUP));
    if (s && inv_s)
        for (int64_t k = 0; k < K; ++k)
            inv_s[k] = 1.0f / s[k];
}

/*
 * Online activation quantization. [MACaQ-fa] paragraph 2: X * diag(1/s) * H_b, then MXFP4.
 *   X [M, K] bf16 bits, inv_s [K] fp32 (NULL: no scale) -> Xq [M, K/2], Xsf [M, K/32] row-major.
 * Grouped form ([MACaQ-en] paragraph 5, grouped matmul): when offsets != NULL, rows
 * [offsets[e], offsets[e+1]) belong to expert e and use inv_s + e*K.
 * work: K floats of scratch owned by the caller.
 */
void oracle_act_quant(const uint16_t *X, const float *inv_s, int64_t M, int64_t K, int b,
                      const int32_t *offsets, int32_t E, uint8_t *Xq, uint8_t *Xsf, float *work)
{
    int32_t e = 0;
    for (int64_t m = 0; m < M; ++m) {
        const float *mul = inv_s;
        if (offsets) {
            while (e < E && m >= offsets[e + 1])
                ++e;
            mul = inv_s ? inv_s + (int64_t)e * K : NULL;
        }
        oracle_transform_rows(X + m * K, mul, 1, K, b, 0, work);
        oracle_mxfp4_quantize_row(work, K, Xq + m * (K / 2), Xsf + m * (K / MX_GROUP));
    }
}

/* Dequantize one MXFP4 row into float64: value(code) * 2^(E-127), exact. [OCP-MX] */
void oracle_dequant_row(const uint8_t *codes, const uint8_t *sf, int64_t K, double *out)
{
    for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = codes[k / 2];
        uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
        out[k] = ldexp(oracle_e2m1_value(c), (int)sf[k / MX_GROUP] - 127);
    }
}

/*
 * W4A4 block-scaled GEMM, the plain definition: Y[m, n] = sum_k dq(A[m, k]) * dq(W[n, k]) in
 * float64, and T[m, n] = sum_k |dq(A[m, k]) * dq(W[n, k])| (the scale of the rounding error an
 * fp32 accumulation may make). [MACaQ-en] paragraph 5 (dense matmul); [OCP-MX] (dequantization).
 * Only the rows listed in rows[0..n_rows) are computed (all rows when rows == NULL, n_rows = M);
 * output row i of Y/T is A row rows[i].
 *   Aq [M, K/2], Asf [M, K/32], Wq [N, K/2], Wsf [N, K/32] -> Y, T [n_rows, N].
 * work: (n_rows + 1) * K doubles of scratch owned by the caller.
 */
void oracle_linear(const uint8_t *Aq, const uint8_t *Asf, const int64_t *rows, int64_t n_rows,
                   const uint8_t *Wq, const uint8_t *Wsf, int64_t N, int64_t K, double *Y,
                   double *T, double *work)
{
    double *a = work;                  /* n_rows * K */
    double *w = work + n_rows * K;     /* K */
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t m = rows ? rows[i] : i;
        oracle_dequant_row(Aq + m * (K / 2), Asf + m * (K / MX_GROUP), K, a + i * K);
    }
    for (int64_t n = 0; n < N; ++n) {
        oracle_dequant_row(Wq + n * (K / 2), Wsf + n * (K / MX_GROUP), K, w);
        for (int64_t i = 0; i < n_rows; ++i) {
            const double *ai = a + i * K;
            double y = 0.0, t = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = ai[k] * w[k];
                y += p;
                t += fabs(p);
            }
            Y[i * N + n] = y;
            T[i * N + n] = t;
        }
    }
}

/*
 * Grouped (MoE) W4A4 GEMM, the plain definition: row m in [offsets[e], offsets[e+1]) is multiplied
 * by expert e's weights, Wq + e*N*K/2 and Wsf + e*N*K/32. [MACaQ-en] paragraph 5 (grouped matmul).
 * Only the listed rows are computed (all when rows == NULL, n_rows = total rows); rows must be
 * sorted ascending. work: 2 * K doubles.
 */
void oracle_grouped_linear(const uint8_t *Aq, const uint8_t *Asf, const int32_t *offsets,
                           int32_t E, const int64_t *rows, int64_t n_rows, const uint8_t *Wq,
                           const uint8_t *Wsf, int64_t N, int64_t K, double *Y, double *T,
                           double *work)
{
    double *a = work;
    double *w = work + K;
    int32_t e = 0;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t m = rows ? rows[i] : i;
        while (e < E && m >= offsets[e + 1])
            ++e;
        oracle_dequant_row(Aq + m * (K / 2), Asf + m * (K / MX_GROUP), K, a);
        const uint8_t *wq = Wq + (int64_t)e * N * (K / 2);
        const uint8_t *wsf = Wsf + (int64_t)e * N * (K / MX_GROUP);
        for (int64_t n = 0; n < N; ++n) {
            oracle_dequant_row(wq + n * (K / 2), wsf + n * (K / MX_GROUP), K, w);
            double y = 0.0, t = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = a[k] * w[k];
                y += p;
                t += fabs(p);
            }
            Y[i * N + n] = y;
            T[i * N + n] = t;
        }
    }
}

/*
 * fp32 -> bf16 bit pattern, round to nearest, ties to even (finite inputs): the upper 16 bits of the
 * fp32 pattern after adding 0x7FFF plus the lowest kept bit. This is the cast the GPU path applies
 * to its fp32 results.
 */
uint16_t oracle_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/*
 * Weighted top-k combine of a mixture-of-experts layer, the plain definition with a fixed order:
 * out[t, n] = sum over j = 0 .. topk-1 of fl32(w[t, j] * Y[pos[t, j], n]), accumulated in fp32 from
 * +0 in the order j = 0, 1, ..., every product and sum rounded on its own; choices whose pos is
 * outside [0, y_rows) are skipped. [MACaQ-en] paragraph 5 (grouped matmul: the combine returns the
 * expert-sorted rows to token order).
 *   Y [y_rows, N] bf16 bits, pos/w [T, topk] -> out [T, N] fp32.
 */
void oracle_moe_combine(const uint16_t *Y, int64_t y_rows, int64_t N, const int32_t *pos, const float *w,
                        int64_t T, int32_t topk, float *out)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int32_t j = 0; j < topk; ++j) {
                int64_t p = pos[t * topk + j];
                if (p < 0 || p >= y_rows)
                    continue;
                float prod = w[t * topk + j] * bf16_to_float(Y[p * N + n]);
                acc = acc + prod;
            }
            out[t * N + n] = acc;
        }
    }
}

/*
 * exp(x) in fp32, the evaluation both sides of the fused SwiGLU use (the pages leave the MLP's
 * activation function to the model; this fixes one exact fp32 evaluation of it). Method: Cody and
 * Waite's argument reduction (W. J. Cody, W. Waite, "Software Manual for the Elementary Functions",
 * 1980): n = rint(x * log2(e)), r = (x - n*C1) - n*C2 with ln 2 = C1 + C2 split so that n*C1 is exact;
 * then the Taylor polynomial 1 + r + r^2/2! + ... + r^6/6! by Horner's rule, and the result p * 2^n.
 * Every operation is one fp32 operation rounded to nearest (no multiply-add contraction). x is
 * clamped to [-100, 88] first, so 2^n is always a representable float (normal or subnormal) and the
 * final product rounds once.
 */
static float f32_from_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

float oracle_exp_f32(float x)
{
    const float log2e = f32_from_bits(0x3FB8AA3Bu); /* 1.44269504 */
    const float c1 = f32_from_bits(0x3F317200u);    /* 0.693145751953125 (ln 2, high part) */
    const float c2 = f32_from_bits(0x35BFBE8Eu);    /* 1.42860677e-06 (ln 2 - c1) */
    static const float inv_fact[7] = {1.0f, 1.0f, 0.5f, 1.0f / 6.0f, 1.0f / 24.0f, 1.0f / 120.0f, 1.0f / 720.0f};
    if (x < -100.0f)
        x = -100.0f;
    if (x > 88.0f)
        x = 88.0f;
    float t = x * log2e;
    float nf = rintf(t);
    float a = nf * c1;
    float r = x - a;
    float b = nf * c2;
    r = r - b;
    float p = inv_fact[6];
    for (int k = 5; k >= 0; --k) {
        float pr = p * r;
        p = pr + inv_fact[k];
    }
    int n = (int)nf;                       /* in [-145, 127] */
    float scale = ldexpf(1.0f, n);         /* 2^n, exact: normal or subnormal */
    return p * scale;
}

/* silu(g) * u with silu(g) = g / (1 + exp(-g)), each operation one fp32 rounding. */
float oracle_swiglu_f32(float g, float u)
{
    float e = oracle_exp_f32(-g);
    float den = 1.0f + e;
    float s = g / den;
    return s * u;
}

/*
 * The fused gate/up epilogue's output, the plain definition: H[m, i] = swiglu(G[m, i], U[m, i]) in
 * fp32 (the gate/up GEMM outputs rounded to fp32), then the down projection's activation
 * quantization of H (its per-channel 1/s and block Hadamard, then MXFP4), exactly as
 * oracle_act_quant. [MACaQ-fa] paragraph 2 (the transform at the input of every linear, here the
 * down projection's input).
 *   G, U [M, I] fp32 -> Hq [M, I/2], Hsf [M, I/32] row-major. work: I floats.
 */
void oracle_swiglu_act_quant(const float *G, const float *U, const float *inv_s, int64_t M, int64_t I, int b,
                             uint8_t *Hq, uint8_t *Hsf, float *work)
{
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t i = 0; i < I; ++i) {
            float h = oracle_swiglu_f32(G[m * I + i], U[m * I + i]);
            work[i] = inv_s ? h * inv_s[i] : h;
        }
        if (b > 1)
            for (int64_t k0 = 0; k0 < I; k0 += b)
                oracle_fwht_f32(work + k0, b);
        oracle_mxfp4_quantize_row(work, I, Hq + m * (I / 2), Hsf + m * (I / MX_GROUP));
    }
}

/* Signed grid index t in [-7, 7] of an E2M1 code (+0 and -0 are both t = 0), and back. */
static int e2m1_index(uint8_t code)
{
    int m = code & 7;
    return (code & 8u) ? -m : m;
}

static uint8_t e2m1_from_index(int t)
{
    return t > 0 ? (uint8_t)t : (t < 0 ? (uint8_t)(8 - t) : 0u);
}

/*
 * Flip-Refinement of prepared weights. [MACaQ-fa] paragraph 3: a coordinate-descent step, guided by
 * the Hessian, that moves single FP4 codes to the neighbouring representable values (in place of
 * GPTQ-style updates). The plain reading taken here, per weight row n:
 *   w      = the row's transformed fp32 weights, exactly as weight preparation computes them
 *            (fl32(W s), the fixed-order butterflies per block of b, times 1/b);
 *   w_hat  = the dequantized codes at the row's E8M0 scales, which never change;
 *   L      = (w_hat - w)^T H (w_hat - w), H symmetric (e.g. X'^T X' of the layer's transformed
 *            calibration activations), so L is the squared output error the row's quantization adds.
 * Keep g = H (w_hat - w) in float64: g[i] = sum over k in order 0..K-1 of H[k][i] * (w_hat[k] - w[k]).
 * Then `sweeps` times, for k = 0 .. K-1 in order: the candidates are the neighbouring values on the
 * signed grid {-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, ..., 6} times the group's scale, the lower one
 * first; moving by d changes L by dL = d * (2 g[k] + d * H[k][k]); the candidate with the smaller dL
 * (the upper one only if strictly smaller) is taken if dL < 0, and then g[i] += d * H[k][i] for every i.
 * Every value is exact in float64 (grid values times powers of two); each arithmetic step is one
 * float64 operation (no multiply-add contraction). A move to zero writes code 0x0.
 *   W [N, K] bf16 bits, s [K] (NULL: 1), H [K, K] fp32, Wq [N, K/2] (in: the prepared codes; out:
 *   refined), Wsf [N, K/32] row-major (read), flips [N] (out: accepted moves per row, may be NULL).
 *   work: K floats (w), K doubles (g).
 */
void oracle_flip_refine(const uint16_t *W, const float *s, int64_t N, int64_t K, int b, const float *H, int sweeps,
                        uint8_t *Wq, const uint8_t *Wsf, int32_t *flips, float *w, double *g)
{
    for (int64_t n = 0; n < N; ++n) {
        uint8_t *q = Wq + n * (K / 2);
        const uint8_t *sf = Wsf + n * (K / MX_GROUP);
        oracle_transform_rows(W + n * K, s, 1, K, b, 1, w);
        for (int64_t i = 0; i < K; ++i)
            g[i] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            uint8_t c = (uint8_t)((q[k / 2] >> (4 * (k & 1))) & 15u);
            double e = ldexp(oracle_e2m1_value(c), (int)sf[k / MX_GROUP] - 127) - (double)w[k];
            for (int64_t i = 0; i < K; ++i) {
                double t = (double)H[k * K + i] * e;
                g[i] = g[i] + t;
            }
        }
        int32_t nflip = 0;
        for (int sw = 0; sw < sweeps; ++sw) {
            for (int64_t k = 0; k < K; ++k) {
                uint8_t c = (uint8_t)((q[k / 2] >> (4 * (k & 1))) & 15u);
                int t = e2m1_index(c);
                int E = (int)sf[k / MX_GROUP] - 127;
                double v = ldexp(oracle_e2m1_value(c), E);
                double hkk = (double)H[k * K + k];
                int best_t = t;
                double best_d = 0.0, best_dl = 0.0;
                for (int dir = -1; dir <= 1; dir += 2) {
                    int tc = t + dir;
                    if (tc < -7 || tc > 7)
                        continue;
                    double d = ldexp(oracle_e2m1_value(e2m1_from_index(tc)), E) - v;
                    double two_g = 2.0 * g[k];
                    double dh = d * hkk;
                    double dl = d * (two_g + dh);
                    if (dl < best_dl) {
                        best_dl = dl;
                        best_d = d;
                        best_t = tc;
                    }
                }
                if (best_t != t) {
                    uint8_t nc = e2m1_from_index(best_t);
                    q[k / 2] = (uint8_t)((k & 1) ? ((q[k / 2] & 0x0Fu) | (nc << 4)) : ((q[k / 2] & 0xF0u) | nc));
                    for (int64_t i = 0; i < K; ++i) {
                        double t2 = best_d * (double)H[k * K + i];
                        g[i] = g[i] + t2;
                    }
                    ++nflip;
                }
            }
        }
        if (flips)
            flips[n] = nflip;
    }
}

/*
 * The weight-only mode's activations: X * diag(1/s) * H_b in fp32 (the act_quant transform), each value
 * then rounded once to bf16 (nearest even). [MACaQ-en] paragraph 3 (vLLM serves W4A4 or weight-only
 * checkpoints); [MACaQ-fa] paragraph 2 (the transform at the input of every linear).
 *   X [M, K] bf16 bits, inv_s [K] (NULL: 1) -> Xt [M, K] bf16 bits. work: K floats.
 */
void oracle_act_transform_bf16(const uint16_t *X, const float *inv_s, int64_t M, int64_t K, int b, uint16_t *Xt,
                               float *work)
{
    for (int64_t m = 0; m < M; ++m) {
        oracle_transform_rows(X + m * K, inv_s, 1, K, b, 0, work);
        for (int64_t k = 0; k < K; ++k)
            Xt[m * K + k] = oracle_bf16_rne(work[k]);
    }
}
