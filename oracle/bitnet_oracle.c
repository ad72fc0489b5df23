/*
 * bitnet_oracle.c -- the plain, slow CPU definition of the H-BitLinear forward path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may load this file or
 * the library built from it: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library; the only thing both sides see is the seeded synthetic inputs.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (see build.py in
 * this folder).  -ffp-contract=off keeps every a*b+c as two IEEE roundings, so
 * each fp32 expression below means exactly what it says.  Single-threaded.
 *
 * Sources (page titles as given on the pages):
 *   [v2]   "bitnet_v2_engine.py" (Quillan-Ronin colab bundle): the BitNet v2
 *          restatement, Eq. 1-7 in its module docstring, fast_hadamard_transform,
 *          quantize_weight_ternary, quantize_act_int8, quantize_act_int4,
 *          HBitLinear.forward.
 *   [b158] "BitNet 论文解析" (youngju.dev transcription), section on BitNet b1.58:
 *          weight_quant_ternary and the integer-GEMM + rescale form of
 *          BitLinear_b158.forward; the {-1,0,+1} -> {0,1,2} code map of its
 *          tl2_lookup_simulation listing.
 *   [edge] "bitnet_cpp_edge.py": pack-once / forward-many (prepare_weights) and the
 *          claim that per-token integer kernels are lossless.
 *   [v2] BitNetV2FFN.forward also defines the SwiGLU input of the down projection
 *          (oracle_swiglu).
 *
 * Readings where the pages are silent or disagree (each one is listed in the
 * design notes with its reason):
 *   - eps = 1e-5 is passed in by the caller (the pages use 1e-7 and 1e-5).
 *   - Rounding is round-half-to-even (the pages call torch.round).
 *   - RMSNorm is y = (x * r) * g with r = 1 / sqrt(sum(x^2)/K + eps).
 *   - The FWHT scales every butterfly stage by c = (float)(1/sqrt 2), as the
 *     listing of fast_hadamard_transform does, in natural (Sylvester) order.
 *   - The per-token scale returned is gamma (or beta) without eps (Eq. 5/6).
 *   - alpha = mean|W| is summed in double in index order, rounded once to float.
 *   - The dequant epilogue is out = (float)acc * ((alpha * scale_x) / Q).
 *   - silu(g) = g / (1 + e^-g) in fp32 (the page calls F.silu = g * sigmoid(g)).
 *   - A bf16 output is the fp32 output rounded once to bf16, to nearest, ties to
 *     even (the pages fix the epilogue's value, not its storage type).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_ACT_INT8 0
#define ORACLE_ACT_INT4 1

/* return codes */
#define ORACLE_OK 0
#define ORACLE_NOT_POW2 3
#define ORACLE_BAD_ARG 1

static float q_int8(void) { return 127.0f; }
static float q_int4(void) { return (float)sqrt(7.0); } /* sqrt(7) rounded once to float */

static int is_pow2(int64_t n) { return n > 0 && (n & (n - 1)) == 0; }

/* Round to nearest, ties to even, in the current (default) rounding mode. */
static float rne(float v) { return nearbyintf(v); }

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ---------------------------------------------------------------------------
 * Step 1. RMSNorm, per token.  [v2] HBitLinear.forward "Normalization" (the page
 * builds nn.RMSNorm(in_features, eps) but does not define it; this is the usual
 * root-mean-square normalisation with a per-channel gain).
 *   ss  = sum_k x[k]*x[k]        (fp32, k ascending)
 *   r   = 1 / sqrt(ss/K + eps)   (IEEE sqrt and division)
 *   y_k = (x_k * r) * g_k        (g == NULL means g = 1)
 * ------------------------------------------------------------------------- */
int oracle_rmsnorm(const float *x, int64_t M, int64_t K, const float *g, float eps,
                   float *y)
{
    if (K <= 0 || M < 0) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const float *xr = x + m * K;
        float *yr = y + m * K;
        float ss = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float sq = xr[k] * xr[k];
            ss = ss + sq;
        }
        float mean = ss / (float)K;
        float r = 1.0f / sqrtf(mean + eps);
        for (int64_t k = 0; k < K; ++k) {
            float v = xr[k] * r;
            yr[k] = g ? v * g[k] : v;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 2. Fast Walsh-Hadamard transform along each row, in place.
 * [v2] Eq. 3/4: H_m = (1/sqrt 2) [[H_{m-1}, H_{m-1}], [H_{m-1}, -H_{m-1}]], H_0 = [1];
 * fast_hadamard_transform: radix-2 butterflies with half-width h = 1, 2, 4, ...,
 * each stage scaled by 1/sqrt 2, computed in fp32.  K must be a power of two
 * (the page raises ValueError otherwise; here the call returns ORACLE_NOT_POW2).
 * ------------------------------------------------------------------------- */
int oracle_fwht(float *y, int64_t M, int64_t K)
{
    if (!is_pow2(K)) return ORACLE_NOT_POW2;
    const float c = (float)(1.0 / sqrt(2.0));
    for (int64_t m = 0; m < M; ++m) {
        float *row = y + m * K;
        for (int64_t h = 1; h < K; h *= 2) {
            for (int64_t j0 = 0; j0 < K; j0 += 2 * h) {
                for (int64_t j = j0; j < j0 + h; ++j) {
                    float u = row[j];
                    float v = row[j + h];
                    row[j] = (u + v) * c;
                    row[j + h] = (u - v) * c;
                }
            }
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 3. Per-token activation quantisation.
 * int8 absmax  [v2] Eq. 5: gamma = max|y|,  q = RoundClip(127 * y / (gamma+eps), -128, 127)
 * int4 absmean [v2] Eq. 6: beta  = mean|y|, q = RoundClip(sqrt7 * y / (beta+eps),  -8,   7)
 * The listings form the per-token multiplier first, s = Q / (gamma + eps), and then
 * multiply: q = clamp(rne(y * s)).  scale_x[m] = gamma (or beta), without eps.
 * ------------------------------------------------------------------------- */
int oracle_act_quant(const float *y, int64_t M, int64_t K, int mode, float eps,
                     int8_t *q, float *scale_x)
{
    if (K <= 0 || M < 0) return ORACLE_BAD_ARG;
    if (mode != ORACLE_ACT_INT8 && mode != ORACLE_ACT_INT4) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const float *yr = y + m * K;
        int8_t *qr = q + m * K;
        float stat, s, lo, hi;
        if (mode == ORACLE_ACT_INT8) {
            float gamma = 0.0f;
            for (int64_t k = 0; k < K; ++k) {
                float a = fabsf(yr[k]);
                if (a > gamma) gamma = a;
            }
            stat = gamma;
            s = q_int8() / (gamma + eps);
            lo = -128.0f;
            hi = 127.0f;
        } else {
            float sum = 0.0f;
            for (int64_t k = 0; k < K; ++k) sum = sum + fabsf(yr[k]);
            float beta = sum / (float)K;
            stat = beta;
            s = q_int4() / (beta + eps);
            lo = -8.0f;
            hi = 7.0f;
        }
        for (int64_t k = 0; k < K; ++k) {
            float v = yr[k] * s;
            qr[k] = (int8_t)clampf(rne(v), lo, hi);
        }
        scale_x[m] = stat;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * fp64 shadow of steps 1-3: the pre-rounding value y*s of every code, with every
 * step carried in double (the FWHT as the same butterflies in double).  Tests use
 * it to tell a rounding near-tie, where two correct fp32 evaluation orders may
 * land on different codes, from a real disagreement.
 * ------------------------------------------------------------------------- */
/* Steps 1-3 in double on one token row (overwritten), pre-rounding values into v. */
static void shadow_row(double *row, int64_t K, const float *g, double eps, int fwht, int mode, double *v)
{
    const double c = 1.0 / sqrt(2.0);
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) ss += row[k] * row[k];
    double r = 1.0 / sqrt(ss / (double)K + eps);
    for (int64_t k = 0; k < K; ++k) row[k] = row[k] * r * (g ? (double)g[k] : 1.0);
    if (fwht) {
        for (int64_t h = 1; h < K; h *= 2)
            for (int64_t j0 = 0; j0 < K; j0 += 2 * h)
                for (int64_t j = j0; j < j0 + h; ++j) {
                    double a = row[j], b = row[j + h];
                    row[j] = (a + b) * c;
                    row[j + h] = (a - b) * c;
                }
    }
    double s;
    if (mode == ORACLE_ACT_INT8) {
        double gamma = 0.0;
        for (int64_t k = 0; k < K; ++k) gamma = fabs(row[k]) > gamma ? fabs(row[k]) : gamma;
        s = 127.0 / (gamma + eps);
    } else {
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k) sum += fabs(row[k]);
        s = sqrt(7.0) / (sum / (double)K + eps);
    }
    for (int64_t k = 0; k < K; ++k) v[k] = row[k] * s;
}

int oracle_shadow_prerounding(const float *x, int64_t M, int64_t K, const float *g,
                              double eps, int fwht, int mode, double *v)
{
    if (K <= 0 || M < 0) return ORACLE_BAD_ARG;
    if (fwht && !is_pow2(K)) return ORACLE_NOT_POW2;
    double *row = (double *)malloc((size_t)K * sizeof(double));
    if (!row) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) row[k] = (double)x[m * K + k];
        shadow_row(row, K, g, eps, fwht, mode, v + m * K);
    }
    free(row);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * SwiGLU input of the FFN down projection.  [v2] BitNetV2FFN.forward:
 *   gate = F.silu(gate_proj(x)); up = up_proj(x); inter = gate * up
 * with silu(g) = g * sigmoid(g) = g / (1 + e^-g), here one fp32 rounding per
 * operation:  inter = (g / (1.0f + expf(-g))) * u.
 * ------------------------------------------------------------------------- */
int oracle_swiglu(const float *gate, const float *up, int64_t count, float *out)
{
    if (count < 0) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < count; ++i) {
        float gv = gate[i];
        float den = 1.0f + expf(-gv);
        float silu = gv / den;
        out[i] = silu * up[i];
    }
    return ORACLE_OK;
}

/* fp64 shadow of the SwiGLU product followed by steps 1-3 (see oracle_shadow_prerounding). */
int oracle_shadow_swiglu(const float *gate, const float *up, int64_t M, int64_t K, const float *g,
                         double eps, int fwht, int mode, double *v)
{
    if (K <= 0 || M < 0) return ORACLE_BAD_ARG;
    if (fwht && !is_pow2(K)) return ORACLE_NOT_POW2;
    double *row = (double *)malloc((size_t)K * sizeof(double));
    if (!row) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            double gv = (double)gate[m * K + k];
            row[k] = gv / (1.0 + exp(-gv)) * (double)up[m * K + k];
        }
        shadow_row(row, K, g, eps, fwht, mode, v + m * K);
    }
    free(row);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 4a. Ternary weights, per tensor.  [v2] Eq. 1/2, quantize_weight_ternary;
 * [b158] weight_quant_ternary.
 *   alpha = mean|W|   (summed in double, index order, one rounding to float)
 *   t     = RoundClip(W / (alpha + eps), -1, 1)   (fp32 division)
 * ------------------------------------------------------------------------- */
float oracle_weight_alpha(const float *W, int64_t count)
{
    double sum = 0.0;
    for (int64_t i = 0; i < count; ++i) sum += fabs((double)W[i]);
    return (float)(sum / (double)count);
}

int oracle_ternarize(const float *W, int64_t count, float alpha, float eps, int8_t *t)
{
    float d = alpha + eps;
    for (int64_t i = 0; i < count; ++i) {
        float v = W[i] / d;
        t[i] = (int8_t)clampf(rne(v), -1.0f, 1.0f);
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 4b. 2-bit packing of the ternary codes (layout fixed by the library
 * header; restated here from that document, not shared with it).
 * Code map [b158] tl2_lookup_simulation: -1 -> 0, 0 -> 1, +1 -> 2 (3 is never
 * written).  packed is [N][K/4] bytes, row n starting at byte n*K/4.  A row is a
 * sequence of little-endian 32-bit words; word w holds k in [16w, 16w+16): the code
 * of k = 16*w + 8*h + i (h in {0,1}, i in [0,8)) sits at bits [4i + 2h, 4i + 2h + 2)
 * of the word, i.e. in byte 4*w + i/2 at bit 4*(i%2) + 2*h.  K must be a multiple
 * of 16.
 * ------------------------------------------------------------------------- */
int oracle_pack(const int8_t *t, int64_t N, int64_t K, uint8_t *packed)
{
    if (K <= 0 || K % 16 != 0 || N < 0) return ORACLE_BAD_ARG;
    const int64_t row_bytes = K / 4;
    memset(packed, 0, (size_t)(N * row_bytes));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int v = t[n * K + k];
            if (v < -1 || v > 1) return ORACLE_BAD_ARG;
            unsigned code = (unsigned)(v + 1);
            int64_t w = k / 16, h = (k % 16) / 8, i = k % 8;
            packed[n * row_bytes + 4 * w + i / 2] |= (uint8_t)(code << (4 * (i % 2) + 2 * h));
        }
    }
    return ORACLE_OK;
}

int oracle_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *t)
{
    if (K <= 0 || K % 16 != 0 || N < 0) return ORACLE_BAD_ARG;
    const int64_t row_bytes = K / 4;
    int bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t w = k / 16, h = (k % 16) / 8, i = k % 8;
            unsigned code = (packed[n * row_bytes + 4 * w + i / 2] >> (4 * (i % 2) + 2 * h)) & 3u;
            if (code == 3u) bad = 1;
            t[n * K + k] = (int8_t)((int)code - 1);
        }
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 5. Integer GEMM of activation codes with ternary weights.
 * [v2] HBitLinear.forward: F.linear(x_q, w_q), i.e. out[m][n] = sum_k x[m][k] W[n][k];
 * [b158] BitLinear_b158.forward does it on the integer codes and rescales after.
 *   acc[m][n] = sum_k q[m][k] * t[n][k]    (exact in int32: |acc| <= 128*K)
 * The packed variant reads each weight code straight out of the packed bytes.
 * ------------------------------------------------------------------------- */
int oracle_gemm_int(const int8_t *q, const int8_t *t, int64_t M, int64_t N, int64_t K,
                    int32_t *acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int32_t)q[m * K + k] * (int32_t)t[n * K + k];
            acc[m * N + n] = s;
        }
    return ORACLE_OK;
}

int oracle_gemm_packed(const int8_t *q, const uint8_t *packed, int64_t M, int64_t N,
                       int64_t K, int32_t *acc)
{
    if (K <= 0 || K % 16 != 0) return ORACLE_BAD_ARG;
    const int64_t row_bytes = K / 4;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t w = k / 16, h = (k % 16) / 8, i = k % 8;
                int code = (packed[n * row_bytes + 4 * w + i / 2] >> (4 * (i % 2) + 2 * h)) & 3;
                s += (int32_t)q[m * K + k] * (int32_t)(code - 1);
            }
            acc[m * N + n] = s;
        }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 6. Dequant epilogue.  The forward's F.linear of the two dequantised
 * operands equals acc * alpha * scale_x / Q ([b158]: output*(w_scale*x_scale)/Qb;
 * [v2] Eq. 5/6 give gamma/127 and beta/sqrt7 as the activation step sizes).
 *   f_m = (alpha * scale_x[m]) / Q ;  out[m][n] = (float)acc[m][n] * f_m
 * ------------------------------------------------------------------------- */
int oracle_dequant(const int32_t *acc, const float *scale_x, float alpha, int mode,
                   int64_t M, int64_t N, float *out)
{
    if (mode != ORACLE_ACT_INT8 && mode != ORACLE_ACT_INT4) return ORACLE_BAD_ARG;
    const float Q = mode == ORACLE_ACT_INT8 ? q_int8() : q_int4();
    for (int64_t m = 0; m < M; ++m) {
        float f = (alpha * scale_x[m]) / Q;
        for (int64_t n = 0; n < N; ++n) out[m * N + n] = (float)acc[m * N + n] * f;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * bf16 output (NEXT row f4: a storage option for the epilogue's fp32 value).  bf16 keeps the sign, the 8 exponent bits and the top
 * 7 fraction bits of an fp32 value.  A finite x lies between two adjacent bf16
 * values: lo, x with its low 16 bits cleared (toward zero), and hi, the next one
 * away from zero.  The result is the nearer of the two; at the exact midpoint,
 * the one whose last kept bit is 0.  Stepping past the largest finite bf16 gives
 * infinity, as IEEE rounding to nearest does.  A NaN stays a NaN (its top
 * fraction bit set, so that dropping the low bits cannot make it infinite).
 * out holds the bf16 bit patterns.
 * ------------------------------------------------------------------------- */
int oracle_round_bf16(const float *x, int64_t count, uint16_t *out)
{
    if (count < 0) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < count; ++i) {
        uint32_t u;
        memcpy(&u, &x[i], sizeof u);
        const uint32_t kept = u >> 16;       /* sign, exponent, 7 fraction bits */
        const uint32_t dropped = u & 0xFFFFu; /* what the truncation loses */
        if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0) {
            out[i] = (uint16_t)(kept | 0x0040u); /* NaN: quiet, never infinity */
            continue;
        }
        uint32_t r = kept;
        if (dropped > 0x8000u) r = kept + 1;                         /* nearer to hi */
        else if (dropped == 0x8000u && (kept & 1u)) r = kept + 1;    /* midpoint: to even */
        out[i] = (uint16_t)r; /* kept + 1 carries into the exponent when it must */
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Low-bit KV cache (NEXT row f3).  [v2] BitNetV2Attention._quantize_kv_head with
 * ActQuantINT8STE / ActQuantINT4STE: per row of D values of a [B, H, S, D] key or
 * value tensor (rows ordered (b, h, s)):
 *   token s = 0 (the BOS token) always int8 absmax:
 *       scale = max|x| + eps;  code = clamp(rne((127 / scale) * x), -128, 127);
 *       step = scale / 127
 *   tokens s >= 1 with bits = 4: int4 absmean:
 *       scale = mean|x| + eps; code = clamp(rne((sqrt7 / scale) * x), -8, 7);
 *       step = scale / sqrt7
 *   tokens s >= 1 with bits = 3:
 *       scale = max|x| + eps;  code = clamp(rne((3 / scale) * x), -4, 3);
 *       step = scale / 3
 *   tokens s >= 1 with bits = 8: as the BOS token.
 * The page returns the fake-quantised values step * code; deq (if not NULL) gets
 * them, codes and step are the stored form.  mean|x| is summed sequentially.
 * ------------------------------------------------------------------------- */
int oracle_kv_quant(const float *kv, int64_t BH, int64_t S, int64_t D, int bits, float eps,
                    int8_t *codes, float *step, float *deq)
{
    if (BH < 0 || S < 0 || D <= 0) return ORACLE_BAD_ARG;
    if (bits != 3 && bits != 4 && bits != 8) return ORACLE_BAD_ARG;
    for (int64_t r = 0; r < BH * S; ++r) {
        const float *x = kv + r * D;
        const int rbits = (r % S == 0) ? 8 : bits;
        float stat = 0.0f, Q, lo, hi;
        if (rbits == 4) {
            float sum = 0.0f;
            for (int64_t k = 0; k < D; ++k) sum += fabsf(x[k]);
            stat = sum / (float)D;
            Q = q_int4(); lo = -8.0f, hi = 7.0f;
        } else {
            for (int64_t k = 0; k < D; ++k) stat = fabsf(x[k]) > stat ? fabsf(x[k]) : stat;
            if (rbits == 8) { Q = q_int8(); lo = -128.0f; hi = 127.0f; }
            else { Q = 3.0f; lo = -4.0f; hi = 3.0f; }
        }
        float scale = stat + eps;
        float s = Q / scale;
        float st = scale / Q;
        step[r] = st;
        for (int64_t k = 0; k < D; ++k) {
            float c = clampf(rne(s * x[k]), lo, hi);
            codes[r * D + k] = (int8_t)c;
            if (deq) deq[r * D + k] = st * c;
        }
    }
    return ORACLE_OK;
}

/* fp64 pre-rounding value s * x of every KV code (see oracle_shadow_prerounding). */
int oracle_shadow_kv(const float *kv, int64_t BH, int64_t S, int64_t D, int bits, double eps, double *v)
{
    if (BH < 0 || S < 0 || D <= 0) return ORACLE_BAD_ARG;
    if (bits != 3 && bits != 4 && bits != 8) return ORACLE_BAD_ARG;
    for (int64_t r = 0; r < BH * S; ++r) {
        const float *x = kv + r * D;
        const int rbits = (r % S == 0) ? 8 : bits;
        double stat = 0.0, Q;
        if (rbits == 4) {
            for (int64_t k = 0; k < D; ++k) stat += fabs((double)x[k]);
            stat /= (double)D;
            Q = sqrt(7.0);
        } else {
            for (int64_t k = 0; k < D; ++k) stat = fabs((double)x[k]) > stat ? fabs((double)x[k]) : stat;
            Q = rbits == 8 ? 127.0 : 3.0;
        }
        const double s = Q / (stat + eps);
        for (int64_t k = 0; k < D; ++k) v[r * D + k] = s * (double)x[k];
    }
    return ORACLE_OK;
}


/* ---------------------------------------------------------------------------
 * TL2 weight format (1.67 bits per weight).  [edge] SignedUnsignedWeightPacker and
 * TL2KernelEdge: the K ternary weights of a row are taken three at a time, triplet
 * j = (t[3j], t[3j+1], t[3j+2]); element-wise mirror consolidation maps each of the
 * 27 triplets to a 4-bit index into the 14 "non-negative" base triplets plus a sign
 * bit (1 = the triplet is the negation of its base).  Read as a balanced-ternary
 * number, v = 9 t0 + 3 t1 + t2 lies in [-13, 13]; negating the triplet negates v, the
 * page's base triplets (first nonzero element +1, and the zero triplet) are exactly the
 * 14 with v >= 0, listed in order of v.  So
 *   index = |v|,  sign = (v < 0).
 * Storage (this library's byte layout of the page's two arrays): a row is padded with
 * zero weights to a multiple of 96 (32 triplets); each group of 32 triplets is 20
 * bytes: four little-endian 32-bit index words (word i: triplets 8i..8i+7, triplet
 * 8i + j in bits [4j, 4j+4)) and one little-endian 32-bit sign word (triplet j in bit
 * j).  Row n starts at byte n * 20 * ceil(K/96).
 * ------------------------------------------------------------------------- */
int64_t oracle_tl2_row_bytes(int64_t K) { return K <= 0 ? 0 : 20 * ((K + 95) / 96); }

int oracle_pack_tl2(const int8_t *t, int64_t N, int64_t K, uint8_t *tl2)
{
    if (K <= 0 || N < 0) return ORACLE_BAD_ARG;
    const int64_t rb = oracle_tl2_row_bytes(K), groups = rb / 20;
    memset(tl2, 0, (size_t)(N * rb));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < groups * 32; ++j) {
            int w[3];
            for (int e = 0; e < 3; ++e) {
                const int64_t k = 3 * j + e;
                w[e] = k < K ? t[n * K + k] : 0;
                if (w[e] < -1 || w[e] > 1) return ORACLE_BAD_ARG;
            }
            const int v = 9 * w[0] + 3 * w[1] + w[2];
            const unsigned idx = (unsigned)(v < 0 ? -v : v), sign = v < 0 ? 1u : 0u;
            uint8_t *grp = tl2 + n * rb + (j / 32) * 20;
            const int64_t jj = j % 32;
            const uint32_t word = (uint32_t)idx << (4 * (jj % 8));
            for (int b = 0; b < 4; ++b) grp[4 * (jj / 8) + b] |= (uint8_t)(word >> (8 * b));
            grp[16 + jj / 8] |= (uint8_t)(sign << (jj % 8));
        }
    }
    return ORACLE_OK;
}

/* The triplet of (index, sign), by the definition above; returns 0 for an index > 13. */
static int tl2_triplet(unsigned idx, unsigned sign, int *w)
{
    if (idx > 13) return 0;
    int v = (int)idx;
    /* balanced-ternary digits of v in [0, 13]: v = 9 w0 + 3 w1 + w2, digits in {-1, 0, 1} */
    for (int e = 2; e >= 0; --e) {
        int d = ((v % 3) + 3) % 3;   /* 0, 1 or 2 */
        if (d == 2) d = -1;
        w[e] = d;
        v = (v - d) / 3;
    }
    if (sign)
        for (int e = 0; e < 3; ++e) w[e] = -w[e];
    return 1;
}

int oracle_unpack_tl2(const uint8_t *tl2, int64_t N, int64_t K, int8_t *t)
{
    if (K <= 0 || N < 0) return ORACLE_BAD_ARG;
    const int64_t rb = oracle_tl2_row_bytes(K);
    int bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; k += 3) {
            const int64_t j = k / 3;
            const uint8_t *grp = tl2 + n * rb + (j / 32) * 20;
            const int64_t jj = j % 32;
            const unsigned idx = (grp[4 * (jj / 8) + (jj % 8) / 2] >> (4 * (jj % 2))) & 15u;
            const unsigned sign = (grp[16 + jj / 8] >> (jj % 8)) & 1u;
            int w[3] = {0, 0, 0};
            if (!tl2_triplet(idx, sign, w)) bad = 1;
            for (int e = 0; e < 3 && k + e < K; ++e) t[n * K + k + e] = (int8_t)w[e];
        }
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* acc[m][n] = sum_k q[m][k] * t[n][k] with each weight read out of the TL2 bytes. */
int oracle_gemm_tl2(const int8_t *q, const uint8_t *tl2, int64_t M, int64_t N, int64_t K, int32_t *acc)
{
    if (K <= 0) return ORACLE_BAD_ARG;
    const int64_t rb = oracle_tl2_row_bytes(K);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; k += 3) {
                const int64_t j = k / 3;
                const uint8_t *grp = tl2 + n * rb + (j / 32) * 20;
                const int64_t jj = j % 32;
                const unsigned idx = (grp[4 * (jj / 8) + (jj % 8) / 2] >> (4 * (jj % 2))) & 15u;
                const unsigned sign = (grp[16 + jj / 8] >> (jj % 8)) & 1u;
                int w[3] = {0, 0, 0};
                if (!tl2_triplet(idx, sign, w)) return ORACLE_BAD_ARG;
                for (int e = 0; e < 3 && k + e < K; ++e) s += (int32_t)q[m * K + k + e] * (int32_t)w[e];
            }
            acc[m * N + n] = s;
        }
    return ORACLE_OK;
}
