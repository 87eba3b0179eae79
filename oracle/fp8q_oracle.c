/*
 * fp8q_oracle.c — plain, slow, CPU reference for the FP8 quantize / scaling-aware
 * direct-transpose path.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check
 * and the benchmark's CPU-baseline leg are its only users.  It shares no code,
 * header, table or constant with the CUDA library; the two meet only on the seeded
 * inputs produced by the synthetic-input module.
 *
 * Every result is computed from its definition, element by element, in exact
 * double (or integer) arithmetic.  The SwiGLU activation is the one place where a
 * floating-point sequence is itself the definition: it is evaluated in IEEE fp32,
 * one correctly rounded operation at a time, following the written arithmetic spec
 * (Cody & Waite range reduction + Taylor polynomial for exp).
 *
 * Sources (page title, section):
 *  [FLOW]  "FP8-Flow-MoE: A Casting-Free FP8 Recipe without Double Quantization
 *          Error (MLSys 2026)" review — sections 核心方法 (core method: scaling-aware
 *          transpose, fused permute+padding, fused SwiGLU+quantization), 关键观察
 *          (observation 2: power-of-two scales turn the layout change into an
 *          exponent adjustment; align to the block's max scale), 设计取舍 (trade-off 2).
 *  [DSV3]  "01 · DeepSeek FP8 与 DeepGEMM：Hopper 软件方案" — §3 细粒度量化 (1x128
 *          activation tiles, SF shape [T, C/128], online amax), §1 (Wgrad reduces over
 *          tokens, hence the column-wise layout), §5.6 (M-grouped contiguous layout),
 *          §8 (UE8M0: scale restricted to a power of two).
 *  [LP]    "低精度（Low Precision）：从 FP8 到 FP4 的训练与推理" — §2 format table
 *          (E4M3: 1/4/3 bits, max magnitude 448, no Inf).
 *
 * Readings where the pages leave a step open are listed with each function.
 * parity pins: every function here is pinned by tests/test_oracle_*.py against
 * something other than itself (torch's float8_e4m3fn cast, brute-force nearest
 * search, closed forms, invariants, hand-worked fixtures).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Format definitions                                                  */
/* ------------------------------------------------------------------ */

/* E4M3 ("FN" variant) as in [LP] §2: 1 sign bit, 4 exponent bits (bias 7),
 * 3 mantissa bits, largest finite magnitude 448, no infinities; exponent field 0
 * holds the subnormals m * 2^-9; S.1111.111 is NaN (never produced here). */
double orc_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int E = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (E == 15 && m == 7)
        return NAN;
    if (E == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(8.0 + m, E - 10); /* (1 + m/8) * 2^(E-7) */
    return s ? -v : v;
}

/* Round a non-negative double to the nearest integer, ties to even. */
static double rne_int(double t)
{
    double fl = floor(t);
    double d = t - fl; /* exact: t carries far fewer than 53 significant bits here */
    if (d > 0.5)
        return fl + 1.0;
    if (d < 0.5)
        return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Nearest E4M3 code to the exact value y, ties to the even code, magnitudes at or
 * above 448 saturated to 448 ("q = RNE(x/S) saturating at 448"); the sign bit is
 * kept even when the magnitude rounds to zero.  Precondition: y finite. */
uint8_t orc_e4m3_encode(double y)
{
    uint8_t s = signbit(y) ? 0x80 : 0x00;
    double a = fabs(y);
    if (a >= 448.0)
        return (uint8_t)(s | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal binade: grid step 2^-9; m == 8 is the smallest normal, 0x08 */
        double m = rne_int(ldexp(a, 9));
        return (uint8_t)(s | (uint8_t)m);
    }
    int E2;
    (void)frexp(a, &E2); /* a = f * 2^E2, f in [0.5, 1) */
    int e = E2 - 1;      /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double m = rne_int(ldexp(a, 3 - e)); /* 3 mantissa bits: m in [8, 16] */
    if (m == 16.0) {
        m = 8.0;
        e += 1;
    }
    if (e > 8)
        return (uint8_t)(s | 0x7E);
    return (uint8_t)(s | (uint8_t)(((e + 7) << 3) | ((int)m - 8)));
}

/* Power-of-two scale exponent of a 1x128 tile ([DSV3] §3, §8; [FLOW] 关键观察 2):
 * e = the smallest integer with amax <= 448 * 2^e, i.e. S = 2^ceil(log2(amax/448)).
 * An all-zero tile takes e = 0 (S = 1).  Reading: e is clamped to [-127, 127] so that
 * the UE8M0 byte e + 127 stays a finite scale; finite BF16/FP32 inputs never exceed
 * the top (amax < 2^128 gives e <= 120), only tiny tiles (amax < 448 * 2^-128) hit
 * the bottom clamp.  Computed by exact comparisons, not by a floating log2. */
int orc_scale_exponent(double amax)
{
    if (amax == 0.0)
        return 0;
    int E2;
    (void)frexp(amax, &E2);
    int e = E2 - 9; /* first guess, then enforce the definition exactly */
    while (amax > ldexp(448.0, e))
        e++;
    while (amax <= ldexp(448.0, e - 1))
        e--;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* bf16 bit pattern -> exact double */
static double bf16_to_double(uint16_t b)
{
    union {
        uint32_t u;
        float f;
    } v;
    v.u = (uint32_t)b << 16;
    return (double)v.f;
}

/* fp32 -> bf16 bit pattern, round to nearest even (finite inputs). */
static uint16_t f32_to_bf16_rne(float f)
{
    union {
        uint32_t u;
        float f;
    } v;
    v.f = f;
    uint32_t lsb = (v.u >> 16) & 1u;
    return (uint16_t)((v.u + 0x7FFFu + lsb) >> 16);
}

/* ------------------------------------------------------------------ */
/* Elementwise helpers exported for the codec pins                     */
/* ------------------------------------------------------------------ */

void orc_e4m3_encode_array(const double *y, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_e4m3_encode(y[i]);
}

void orc_e4m3_decode_array(const uint8_t *c, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_e4m3_decode(c[i]);
}

void orc_scale_exponent_array(const double *amax, int64_t n, int32_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_scale_exponent(amax[i]);
}

/* Scaling-aware shift of one code, value level ([FLOW] 核心方法):
 * q' = RNE_e4m3(decode(q) * 2^-k), k >= 0. */
uint8_t orc_shift_code_value(uint8_t c, int k)
{
    return orc_e4m3_encode(ldexp(orc_e4m3_decode(c), -k));
}

/* The same shift stated on the bit fields ([FLOW] 设计取舍 2: an exponent operation
 * instead of a requantization): while the result stays normal the exponent field
 * drops by k and the mantissa is untouched; once it would go subnormal, the integer
 * significand (hidden bit included) is shifted right with round-to-nearest-even,
 * a carry into 0x08 being the smallest normal.  Kept as a second, independent
 * formulation so that the tests can hold it against the value-level rule. */
uint8_t orc_shift_code_bytes(uint8_t c, int k)
{
    uint8_t s = c & 0x80;
    int E = (c >> 3) & 15;
    int m = c & 7;
    if (k == 0)
        return c;
    if (E > k)
        return (uint8_t)(s | ((E - k) << 3) | m);
    int sig = E ? (8 | m) : m;
    int sh = E ? (k - E + 1) : k;
    if (sh >= 5)
        return s; /* sig <= 15 < 2^4: below half of the smallest step */
    int q = sig >> sh;
    int rem = sig - (q << sh);
    int half = 1 << (sh - 1);
    if (rem > half || (rem == half && (q & 1)))
        q++;
    return (uint8_t)(s | q);
}

void orc_shift_codes(const uint8_t *c, int64_t n, int k, int bytes_rule, uint8_t *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = bytes_rule ? orc_shift_code_bytes(c[i], k) : orc_shift_code_value(c[i], k);
}

/* ------------------------------------------------------------------ */
/* Row-wise 1x128 quantization ([DSV3] §3; [FLOW] 一句话总结/核心方法)  */
/* ------------------------------------------------------------------ */

/* One 1x128 tile given as exact doubles: amax, e, codes.  zero_e is the exponent an
 * all-zero tile takes: 0 by the pages' rule (S = 1), or -127 under the zero-tile option
 * of the single-pass quantizer (below). */
static void quantize_tile_z(const double *v, int zero_e, uint8_t *q, uint8_t *sf)
{
    double amax = 0.0;
    for (int i = 0; i < 128; i++) {
        double a = fabs(v[i]);
        if (a > amax)
            amax = a;
    }
    int e = amax == 0.0 ? zero_e : orc_scale_exponent(amax);
    for (int i = 0; i < 128; i++)
        q[i] = orc_e4m3_encode(ldexp(v[i], -e)); /* x * 2^-e is exact in double */
    *sf = (uint8_t)(e + 127);                        /* UE8M0 byte, bias 127 */
}

static void quantize_tile(const double *v, uint8_t *q, uint8_t *sf) { quantize_tile_z(v, 0, q, sf); }

/* X bf16 [rows, cols] (cols % 128 == 0) -> Q u8 [rows, cols], SF u8 [rows, cols/128]. */
void orc_quantize_rowwise(const uint16_t *x, int64_t rows, int64_t cols, uint8_t *q, uint8_t *sf)
{
    int64_t nt = cols / 128;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; t++) {
        double v[128];
        for (int64_t j = 0; j < nt; j++) {
            for (int i = 0; i < 128; i++)
                v[i] = bf16_to_double(x[t * cols + j * 128 + i]);
            quantize_tile(v, q + t * cols + j * 128, sf + t * nt + j);
        }
    }
}

/* Same on fp32 input (the SwiGLU output y). */
void orc_quantize_rowwise_f32(const float *y, int64_t rows, int64_t cols, uint8_t *q, uint8_t *sf)
{
    int64_t nt = cols / 128;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; t++) {
        double v[128];
        for (int64_t j = 0; j < nt; j++) {
            for (int i = 0; i < 128; i++)
                v[i] = (double)y[t * cols + j * 128 + i];
            quantize_tile(v, q + t * cols + j * 128, sf + t * nt + j);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Groups ([DSV3] §5.6 M-grouped contiguous; [FLOW] fused permute+pad) */
/* ------------------------------------------------------------------ */

/* Checks a group-offset vector: offsets[0] == 0, non-decreasing, every group a
 * multiple of 128 rows, offsets[G] <= rows.  A NULL vector means one group of all
 * rows.  Returns 0 when valid. */
static int check_groups(const int32_t *off, int32_t G, int64_t rows)
{
    if (!off)
        return (rows % 128) ? 2 : 0;
    if (G < 1 || off[0] != 0)
        return 2;
    for (int32_t g = 0; g < G; g++)
        if (off[g + 1] < off[g] || (off[g + 1] - off[g]) % 128)
            return 2;
    return off[G] > rows ? 2 : 0;
}

/* Row block b's group: the layout of group g's transposed output is [cols, M_g]
 * starting at byte cols*off_g (codes) and cols*off_g/128 (scales). */
static void group_of_row(const int32_t *off, int32_t G, int64_t rows, int64_t r, int64_t *o, int64_t *M)
{
    if (!off) {
        *o = 0;
        *M = rows;
        return;
    }
    for (int32_t g = 0; g < G; g++)
        if (r >= off[g] && r < off[g + 1]) {
            *o = off[g];
            *M = off[g + 1] - off[g];
            return;
        }
    *o = -1;
    *M = 0;
}

/* ------------------------------------------------------------------ */
/* Scaling-aware direct transpose ([FLOW] 核心方法; 关键观察 2)         */
/* ------------------------------------------------------------------ */

/* Per 128x128 block (row block b, column block j):
 *   e_max = max over the block's 128 rows of the row-tile exponent e_(t,j)
 *           (reading: the page's "S_col" in k = log2(Smax/S) is the scale of the
 *            row tile being converted; Smax is shared by all 128 output channels);
 *   k_t   = e_max - e_(t,j) >= 0;
 *   Q^T[h, t] = RNE_e4m3(decode(Q[t, h]) * 2^-k_t);  SF^T[h, b] = e_max + 127.
 * Dense layout: Q^T [cols, rows], SF^T [cols, rows/128].  Grouped layout: group g
 * (rows off_g..off_g+1) goes to [cols, M_g] at cols*off_g, scales [cols, M_g/128]
 * at cols*off_g/128.  Returns 0, or 2 on invalid groups/shape. */
int orc_direct_transpose(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols,
                         const int32_t *off, int32_t G, uint8_t *qt, uint8_t *sft)
{
    if (cols % 128 || check_groups(off, G, rows))
        return 2;
    int64_t nt = cols / 128;
    int64_t nb = (off ? off[G] : rows) / 128;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; b++) {
        int64_t o, M;
        group_of_row(off, G, rows, b * 128, &o, &M);
        for (int64_t j = 0; j < nt; j++) {
            int emax = -1000;
            for (int t = 0; t < 128; t++) {
                int e = (int)sf[(b * 128 + t) * nt + j] - 127;
                if (e > emax)
                    emax = e;
            }
            for (int t = 0; t < 128; t++) {
                int64_t row = b * 128 + t;
                int k = emax - ((int)sf[row * nt + j] - 127);
                for (int h = 0; h < 128; h++) {
                    int64_t ch = j * 128 + h;
                    qt[cols * o + ch * M + (row - o)] = orc_shift_code_value(q[row * cols + ch], k);
                }
            }
            for (int h = 0; h < 128; h++) {
                int64_t ch = j * 128 + h;
                sft[cols * o / 128 + ch * (M / 128) + (b * 128 - o) / 128] = (uint8_t)(emax + 127);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Naive dequant -> transpose -> requant ([FLOW] 问题与动机, 核心方法)   */
/* ------------------------------------------------------------------ */

/* The three-pass conversion that the direct transpose replaces:
 *   (1) dequantize each code to the BF16 backbone dtype: v = bf16(fp32(decode(q) * 2^e))
 *       (reading: the pages' dataflow is BF16-dominated; the product is exact in fp32
 *        and in bf16 for every exponent e >= -124);
 *   (2) transpose v;
 *   (3) requantize each 128-token column tile with a fresh power-of-two scale by the
 *       same rule as the row-wise quantization.
 * Same layouts and return codes as orc_direct_transpose. */
int orc_naive_transpose(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols,
                        const int32_t *off, int32_t G, uint8_t *qt, uint8_t *sft)
{
    if (cols % 128 || check_groups(off, G, rows))
        return 2;
    int64_t nt = cols / 128;
    int64_t nr = off ? off[G] : rows;
    uint16_t *v = (uint16_t *)malloc((size_t)(nr * cols) * sizeof(uint16_t));
    uint16_t *vt = (uint16_t *)malloc((size_t)(nr * cols) * sizeof(uint16_t));
    if (!v || !vt) {
        free(v);
        free(vt);
        return 5;
    }
    /* (1) dequantize */
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nr; t++)
        for (int64_t h = 0; h < cols; h++) {
            int e = (int)sf[t * nt + h / 128] - 127;
            float p = (float)ldexp(orc_e4m3_decode(q[t * cols + h]), e);
            v[t * cols + h] = f32_to_bf16_rne(p);
        }
    /* (2) transpose, per group */
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nr; t++) {
        int64_t o, M;
        group_of_row(off, G, rows, t, &o, &M);
        for (int64_t h = 0; h < cols; h++)
            vt[cols * o + h * M + (t - o)] = v[t * cols + h];
    }
    /* (3) requantize: the transposed buffer, read as consecutive 128-element tiles,
     * is exactly the set of 128-token column tiles of every group. */
    int64_t ntiles = nr * cols / 128;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < ntiles; i++) {
        double w[128];
        for (int u = 0; u < 128; u++)
            w[u] = bf16_to_double(vt[i * 128 + u]);
        quantize_tile(w, qt + i * 128, sft + i);
    }
    free(v);
    free(vt);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Tile size as a parameter: the 1x32 / 32x32 MX granularity            */
/* ------------------------------------------------------------------ */

/* [LP] format table: MXFP8 keeps E4M3 elements with one power-of-two (E8M0) scale per
 * 32 elements; [FLOW] 局限与 Future Work 2 names the extension of the scaling-aware
 * layout conversion to MX formats.  Reading: the same scale rule, on 1 x G tiles, and
 * the same direct transpose on G x G blocks (G = 128 is the path above, G = 32 the MX
 * granularity).  Layouts: SF [rows, cols/G], Q^T [cols, rows], SF^T [cols, rows/G].
 * rows (for the transpose) and cols must be multiples of G.  Returns 0 or 2. */
int orc_quantize_rowwise_g(const uint16_t *x, int64_t rows, int64_t cols, int32_t G, uint8_t *q, uint8_t *sf)
{
    if (G < 1 || G > 128 || cols % G)
        return 2;
    int64_t nt = cols / G;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; t++)
        for (int64_t j = 0; j < nt; j++) {
            double amax = 0.0;
            for (int i = 0; i < G; i++) {
                double a = fabs(bf16_to_double(x[t * cols + j * G + i]));
                if (a > amax)
                    amax = a;
            }
            int e = orc_scale_exponent(amax);
            for (int i = 0; i < G; i++)
                q[t * cols + j * G + i] = orc_e4m3_encode(ldexp(bf16_to_double(x[t * cols + j * G + i]), -e));
            sf[t * nt + j] = (uint8_t)(e + 127);
        }
    return 0;
}

int orc_direct_transpose_g(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols, int32_t G, uint8_t *qt,
                           uint8_t *sft)
{
    if (G < 1 || G > 128 || cols % G || rows % G)
        return 2;
    int64_t nt = cols / G, nb = rows / G;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; b++)
        for (int64_t j = 0; j < nt; j++) {
            int emax = -1000;
            for (int t = 0; t < G; t++) {
                int e = (int)sf[(b * G + t) * nt + j] - 127;
                if (e > emax)
                    emax = e;
            }
            for (int t = 0; t < G; t++) {
                int64_t row = b * G + t;
                int k = emax - ((int)sf[row * nt + j] - 127);
                for (int h = 0; h < G; h++) {
                    int64_t ch = j * G + h;
                    qt[ch * rows + row] = orc_shift_code_value(q[row * cols + ch], k);
                }
            }
            for (int h = 0; h < G; h++)
                sft[(j * G + h) * nb + b] = (uint8_t)(emax + 127);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Single-pass quantization into both layouts, packed UE8M0 scales      */
/* ------------------------------------------------------------------ */

/* Packed UE8M0 ([DSV3] §8: the SM100 GEMM takes power-of-two scales four to a 32-bit
 * word, each byte being the exponent byte of the fp32 scale, i.e. e + 127).
 * Input: unpacked scales sf [mn, ktiles] (one byte per 1x128 tile along K).
 * Output: words [ceil(ktiles/4), mn_pad], MN-major, word (g, m) at index g*mn_pad + m,
 * holding the scale of K tile 4g+i in byte i (bits 8i..8i+7).
 * Readings (the pages give only "four 8-bit scales in one int32"): bytes in K order
 * from the least significant end; MN-major so that a GEMM tile of consecutive rows
 * reads consecutive words; mn padded up to a multiple of 4 (16-byte rows); bytes of K
 * tiles past the last one, and words of padding rows, are 0. */
void orc_pack_ue8m0(const uint8_t *sf, int64_t mn, int64_t ktiles, uint32_t *out)
{
    int64_t groups = (ktiles + 3) / 4;
    int64_t mn_pad = (mn + 3) / 4 * 4;
    for (int64_t g = 0; g < groups; g++)
        for (int64_t m = 0; m < mn_pad; m++) {
            uint32_t w = 0;
            for (int i = 0; i < 4; i++) {
                int64_t kt = 4 * g + i;
                if (m < mn && kt < ktiles)
                    w |= (uint32_t)sf[m * ktiles + kt] << (8 * i);
            }
            out[g * mn_pad + m] = w;
        }
}

/* Row-wise quantization with the zero-tile option: zero_tile_min != 0 gives an
 * all-zero tile e = -127 (scale byte 0x00) instead of e = 0.  Reading: the pages fix
 * S = 1 for a zero tile, which lets zero rows (padding, dead tokens) raise a block's
 * Smax in the direct transpose and push the other rows' small values toward zero; the
 * option (ours, off by default) gives such tiles the smallest scale, so Smax is the max
 * over the nonzero tiles.  The codes of a zero tile are +-0 either way. */
void orc_quantize_rowwise_opt(const uint16_t *x, int64_t rows, int64_t cols, int zero_tile_min, uint8_t *q,
                              uint8_t *sf)
{
    int64_t nt = cols / 128;
    int zero_e = zero_tile_min ? -127 : 0;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; t++) {
        double v[128];
        for (int64_t j = 0; j < nt; j++) {
            for (int i = 0; i < 128; i++)
                v[i] = bf16_to_double(x[t * cols + j * 128 + i]);
            quantize_tile_z(v, zero_e, q + t * cols + j * 128, sf + t * nt + j);
        }
    }
}

/* BF16 X [rows, cols] -> the row-wise (Q, SF) and, when qt is non-NULL, the
 * column-wise (Q^T, SF^T) layouts: by definition the row-wise quantization followed by
 * the scaling-aware direct transpose of its result ([FLOW] 核心方法).  flags bit 0:
 * zero-tile option; bit 1: scales written packed (orc_pack_ue8m0) - sf as
 * [ceil(cols/512), rows] words, sft as [ceil(rows/512), cols] words - instead of bytes
 * [rows, cols/128] and [cols, rows/128].  Returns 0, 2 (shape), 5 (allocation). */
int orc_quantize_rowwise_colwise(const uint16_t *x, int64_t rows, int64_t cols, uint32_t flags, uint8_t *q,
                                 void *sf, uint8_t *qt, void *sft)
{
    if (cols % 128 || (qt && rows % 128))
        return 2;
    int packed = (flags & 2u) != 0;
    uint8_t *sf_b = packed ? (uint8_t *)malloc((size_t)(rows * cols / 128)) : (uint8_t *)sf;
    uint8_t *sft_b = (packed && qt) ? (uint8_t *)malloc((size_t)(rows * cols / 128)) : (uint8_t *)sft;
    if (!sf_b || (qt && !sft_b)) {
        if (packed) {
            free(sf_b);
            free(sft_b);
        }
        return 5;
    }
    orc_quantize_rowwise_opt(x, rows, cols, (int)(flags & 1u), q, sf_b);
    int rc = 0;
    if (qt)
        rc = orc_direct_transpose(q, sf_b, rows, cols, NULL, 1, qt, sft_b);
    if (packed) {
        orc_pack_ue8m0(sf_b, rows, cols / 128, (uint32_t *)sf);
        if (qt)
            orc_pack_ue8m0(sft_b, cols, rows / 128, (uint32_t *)sft);
        free(sf_b);
        free(sft_b);
    }
    return rc;
}

/* ------------------------------------------------------------------ */
/* SwiGLU arithmetic spec ([FLOW] 核心方法: fused SwiGLU+quantization)  */
/* ------------------------------------------------------------------ */

/* fp32 constants, each derived from its mathematical definition:
 *   L2E    = fp32(log2 e)
 *   LN2_HI = ln 2 with the fp32 mantissa cut to its top 15 bits (0x3F317200)
 *   LN2_LO = fp32(ln 2 - LN2_HI)
 *   C_k    = fp32(1/k!), k = 0..7 (Taylor series of exp)                        */
static const float ORC_L2E = 0x1.715476p+0f;
static const float ORC_LN2_HI = 0x1.62e4p-1f;
static const float ORC_LN2_LO = 0x1.7f7d1cp-20f;
static const float ORC_C[8] = {0x1p+0f,        0x1p+0f,        0x1p-1f,        0x1.555556p-3f,
                               0x1.555556p-5f, 0x1.111112p-7f, 0x1.6c16c2p-10f, 0x1.a01a02p-13f};

void orc_exp_spec_constants(float *out11)
{
    out11[0] = ORC_L2E;
    out11[1] = ORC_LN2_HI;
    out11[2] = ORC_LN2_LO;
    for (int i = 0; i < 8; i++)
        out11[3 + i] = ORC_C[i];
}

static float pow2_f32(int n) /* 2^n for n in [-126, 127] */
{
    union {
        uint32_t u;
        float f;
    } v;
    v.u = (uint32_t)(n + 127) << 23;
    return v.f;
}

/* exp(a) in fp32 (Cody & Waite, "Software Manual for the Elementary Functions",
 * 1980: additive range reduction by n*ln2 in two parts, then a polynomial):
 *   a > 89 -> +inf;  a < -104 -> +0;
 *   n = rint(a*L2E);  r = fma(-n, LN2_HI, a);  r = fma(-n, LN2_LO, r);
 *   p = Horner over C_7..C_0 with fma;   result = (p * 2^floor(n/2)) * 2^(n-floor(n/2)).
 * Every step is one IEEE fp32 operation rounded to nearest even. */
float orc_exp_spec(float a)
{
    if (a > 89.0f)
        return INFINITY;
    if (a < -104.0f)
        return 0.0f;
    float t = a * ORC_L2E;
    float n = rintf(t);
    float r = fmaf(-n, ORC_LN2_HI, a);
    r = fmaf(-n, ORC_LN2_LO, r);
    float p = ORC_C[7];
    for (int i = 6; i >= 0; i--)
        p = fmaf(p, r, ORC_C[i]);
    int ni = (int)n;
    int n1 = (ni >= 0) ? ni / 2 : -((-ni + 1) / 2); /* floor(n/2) */
    int n2 = ni - n1;
    float s = p * pow2_f32(n1);
    return s * pow2_f32(n2);
}

/* silu(g) * u in fp32: silu(g) = g / (1 + exp(-g)); each operation one IEEE fp32
 * rounding (no contraction). */
float orc_swiglu_f32(float g, float u)
{
    float den = 1.0f + orc_exp_spec(-g);
    float s = g / den;
    return s * u;
}

void orc_exp_spec_array(const float *a, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_exp_spec(a[i]);
}

void orc_swiglu_array(const float *g, const float *u, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = orc_swiglu_f32(g[i], u[i]);
}

/* Fused SwiGLU + quantize: y = silu(gate)*up in fp32, then the row-wise 1x128
 * quantization of y; when qt is non-NULL also the direct transpose of (Q, SF). */
int orc_swiglu_quant(const uint16_t *gate, const uint16_t *up, int64_t rows, int64_t cols,
                     uint8_t *q, uint8_t *sf, uint8_t *qt, uint8_t *sft)
{
    if (cols % 128 || (qt && rows % 128))
        return 2;
    float *y = (float *)malloc((size_t)(rows * cols) * sizeof(float));
    if (!y)
        return 5;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows * cols; i++) {
        union {
            uint32_t u;
            float f;
        } g, u;
        g.u = (uint32_t)gate[i] << 16;
        u.u = (uint32_t)up[i] << 16;
        y[i] = orc_swiglu_f32(g.f, u.f);
    }
    orc_quantize_rowwise_f32(y, rows, cols, q, sf);
    free(y);
    if (qt)
        return orc_direct_transpose(q, sf, rows, cols, NULL, 1, qt, sft);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Fused permute + pad + quantize ([FLOW] 核心方法: Fused Permute+Padding; */
/* [DSV3] §5.6: experts' rows concatenated along M)                      */
/* ------------------------------------------------------------------ */

/* topk_idx [T, K] in [0, E).  Expert e collects the pairs (t, s) with idx == e,
 * in row-major (t, s) order (reading: stable order; the pages do not fix one);
 * its segment is padded with zero rows to a multiple of `align`:
 *   c_e = #pairs, P_e = ceil(c_e/align)*align, off = exclusive scan of P,
 *   row(t, s) = off_e + rank of (t, s) among expert e's pairs.
 * Row payload: the row-wise quantization of X[t]; padding rows: codes 0x00,
 * scale byte 127 (the all-zero tile rule).  Rows at or beyond off[E] are not
 * written.  Returns 0, 2 (bad shape), 4 (bad argument/capacity), 7 (index out of
 * range). */
int orc_permute_pad_quant(const uint16_t *x, int64_t T, int64_t H, const int32_t *idx, int32_t K,
                          int32_t E, int32_t align, uint8_t *q, uint8_t *sf, int64_t max_rows,
                          int32_t *offsets, int32_t *row_id_map)
{
    if (H % 128 || T < 0 || K < 1 || E < 1 || align < 1)
        return 2;
    int64_t nt = H / 128;
    int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    if (!cnt)
        return 5;
    for (int64_t p = 0; p < T * K; p++) {
        if (idx[p] < 0 || idx[p] >= E) {
            free(cnt);
            return 7;
        }
        cnt[idx[p]]++;
    }
    int64_t acc = 0;
    for (int32_t e = 0; e < E; e++) {
        offsets[e] = (int32_t)acc;
        acc += (cnt[e] + align - 1) / align * align;
    }
    offsets[E] = (int32_t)acc;
    if (acc > max_rows) {
        free(cnt);
        return 4;
    }
    /* ranks in (t, s) order */
    int64_t *seen = cnt;
    memset(seen, 0, (size_t)E * sizeof(int64_t));
    for (int64_t p = 0; p < T * K; p++) {
        int32_t e = idx[p];
        row_id_map[p] = (int32_t)(offsets[e] + seen[e]);
        seen[e]++;
    }
    /* payload rows */
    uint8_t *qrow = (uint8_t *)malloc((size_t)H);
    uint8_t *sfrow = (uint8_t *)malloc((size_t)nt);
    for (int64_t t = 0; t < T; t++) {
        orc_quantize_rowwise(x + t * H, 1, H, qrow, sfrow);
        for (int32_t s = 0; s < K; s++) {
            int64_t r = row_id_map[t * K + s];
            memcpy(q + r * H, qrow, (size_t)H);
            memcpy(sf + r * nt, sfrow, (size_t)nt);
        }
    }
    /* padding rows */
    for (int32_t e = 0; e < E; e++)
        for (int64_t r = offsets[e] + seen[e]; r < offsets[e + 1]; r++) {
            memset(q + r * H, 0x00, (size_t)H);
            memset(sf + r * nt, 127, (size_t)nt);
        }
    free(qrow);
    free(sfrow);
    free(cnt);
    return 0;
}

/* FP8-input permute + pad ([FLOW] 核心方法 with the pages' FP8 dataflow: the
 * dispatch already delivers row-wise FP8 codes and their scales, so the permute moves
 * codes instead of quantizing).  Same routing, offsets, padding and return codes as
 * orc_permute_pad_quant; the payload of row (t, s) is the token's codes and scale
 * bytes, copied. */
int orc_permute_pad_fp8(const uint8_t *xq, const uint8_t *xsf, int64_t T, int64_t H, const int32_t *idx, int32_t K,
                        int32_t E, int32_t align, uint8_t *q, uint8_t *sf, int64_t max_rows, int32_t *offsets,
                        int32_t *row_id_map)
{
    if (H % 128 || T < 0 || K < 1 || E < 1 || align < 1)
        return 2;
    int64_t nt = H / 128;
    int64_t *cnt = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    if (!cnt)
        return 5;
    for (int64_t p = 0; p < T * K; p++) {
        if (idx[p] < 0 || idx[p] >= E) {
            free(cnt);
            return 7;
        }
        cnt[idx[p]]++;
    }
    int64_t acc = 0;
    for (int32_t e = 0; e < E; e++) {
        offsets[e] = (int32_t)acc;
        acc += (cnt[e] + align - 1) / align * align;
    }
    offsets[E] = (int32_t)acc;
    if (acc > max_rows) {
        free(cnt);
        return 4;
    }
    int64_t *seen = cnt;
    memset(seen, 0, (size_t)E * sizeof(int64_t));
    for (int64_t p = 0; p < T * K; p++) {
        int32_t e = idx[p];
        row_id_map[p] = (int32_t)(offsets[e] + seen[e]);
        seen[e]++;
    }
    for (int64_t t = 0; t < T; t++)
        for (int32_t s = 0; s < K; s++) {
            int64_t r = row_id_map[t * K + s];
            memcpy(q + r * H, xq + t * H, (size_t)H);
            memcpy(sf + r * nt, xsf + t * nt, (size_t)nt);
        }
    for (int32_t e = 0; e < E; e++)
        for (int64_t r = offsets[e] + seen[e]; r < offsets[e + 1]; r++) {
            memset(q + r * H, 0x00, (size_t)H);
            memset(sf + r * nt, 127, (size_t)nt);
        }
    free(cnt);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Expert-parallel FP8 dispatch ([FLOW] 核心方法: the dispatch carries   */
/* row-wise FP8 codes with their scale metadata, Table 1: FP8 all-to-all */
/* beats BF16; [DSV3] §5.6: each rank's experts read contiguous rows)    */
/* ------------------------------------------------------------------ */

/* Send side of one source rank.  Experts are numbered globally, expert e living on
 * rank e / Eloc as its local expert e % Eloc (W ranks, Eloc experts each).  A token is
 * sent once to every rank that holds at least one of its K experts (its destination
 * set), carrying its row-wise codes, its scale bytes and its K slot ids re-expressed
 * for that rank: the local expert id where the slot's expert lives there, -1 where it
 * lives elsewhere.  The send buffer is grouped by destination rank, tokens in order
 * within a group: send_offsets[d] = number of rows for ranks below d, and the row of
 * (token t, rank d) is send_offsets[d] + (number of tokens before t sent to d);
 * send_map[t*W + d] holds it, or -1 where t is not sent to d.
 * Returns 2 on bad sizes, 7 on an expert id outside [0, W*Eloc), 4 when the rows
 * exceed max_rows. */
int orc_ep_dispatch_pack(const uint8_t *xq, const uint8_t *xsf, int64_t T, int64_t H, const int32_t *idx,
                         int32_t K, int32_t W, int32_t Eloc, uint8_t *send_q, uint8_t *send_sf, int32_t *send_ids,
                         int64_t max_rows, int32_t *send_offsets, int32_t *send_map)
{
    if (H % 128 || T < 0 || K < 1 || W < 1 || Eloc < 1)
        return 2;
    int64_t nt = H / 128;
    for (int64_t p = 0; p < T * K; p++)
        if (idx[p] < 0 || idx[p] >= (int64_t)W * Eloc)
            return 7;
    int64_t *cnt = (int64_t *)calloc((size_t)W, sizeof(int64_t));
    if (!cnt)
        return 5;
    /* destination set of each token, counted per rank */
    for (int64_t t = 0; t < T; t++)
        for (int32_t d = 0; d < W; d++) {
            int hit = 0;
            for (int32_t k = 0; k < K; k++)
                hit |= idx[t * K + k] / Eloc == d;
            send_map[t * W + d] = hit ? 0 : -1;
            cnt[d] += hit;
        }
    int64_t acc = 0;
    for (int32_t d = 0; d < W; d++) {
        send_offsets[d] = (int32_t)acc;
        acc += cnt[d];
    }
    send_offsets[W] = (int32_t)acc;
    if (acc > max_rows) {
        free(cnt);
        return 4;
    }
    memset(cnt, 0, (size_t)W * sizeof(int64_t));
    for (int64_t t = 0; t < T; t++)
        for (int32_t d = 0; d < W; d++) {
            if (send_map[t * W + d] < 0)
                continue;
            int64_t r = send_offsets[d] + cnt[d]++;
            send_map[t * W + d] = (int32_t)r;
            memcpy(send_q + r * H, xq + t * H, (size_t)H);
            memcpy(send_sf + r * nt, xsf + t * nt, (size_t)nt);
            for (int32_t k = 0; k < K; k++) {
                int32_t e = idx[t * K + k];
                send_ids[r * K + k] = e / Eloc == d ? e - d * Eloc : -1;
            }
        }
    free(cnt);
    return 0;
}

/* Receive side of one destination rank: the rows received from all source ranks,
 * concatenated in source-rank order (rank 0's rows first, each source's rows in its
 * send order), with their slot ids (local expert ids, -1 for slots whose expert lives
 * on another rank).  Slot (r, s) with id e >= 0 goes to local expert e; the rows of an
 * expert follow (r, s) row-major order and each expert's segment is padded with zero
 * rows (codes 0x00, scale byte 127) to a multiple of align, exactly as the FP8-input
 * permute does; a slot with id -1 gets row_id_map -1 and no row.
 * Returns 2 on bad sizes, 7 on an id outside [-1, Eloc), 4 when rows exceed max_rows. */
int orc_ep_recv_permute(const uint8_t *rq, const uint8_t *rsf, const int32_t *rids, int64_t R, int64_t H, int32_t K,
                        int32_t Eloc, int32_t align, uint8_t *q, uint8_t *sf, int64_t max_rows, int32_t *offsets,
                        int32_t *row_id_map)
{
    if (H % 128 || R < 0 || K < 1 || Eloc < 1 || align < 1)
        return 2;
    int64_t nt = H / 128;
    int64_t *cnt = (int64_t *)calloc((size_t)Eloc, sizeof(int64_t));
    if (!cnt)
        return 5;
    for (int64_t p = 0; p < R * K; p++) {
        if (rids[p] < -1 || rids[p] >= Eloc) {
            free(cnt);
            return 7;
        }
        if (rids[p] >= 0)
            cnt[rids[p]]++;
    }
    int64_t acc = 0;
    for (int32_t e = 0; e < Eloc; e++) {
        offsets[e] = (int32_t)acc;
        acc += (cnt[e] + align - 1) / align * align;
    }
    offsets[Eloc] = (int32_t)acc;
    if (acc > max_rows) {
        free(cnt);
        return 4;
    }
    int64_t *seen = cnt;
    memset(seen, 0, (size_t)Eloc * sizeof(int64_t));
    for (int64_t p = 0; p < R * K; p++) {
        int32_t e = rids[p];
        if (e < 0) {
            row_id_map[p] = -1;
            continue;
        }
        int64_t r = offsets[e] + seen[e]++;
        row_id_map[p] = (int32_t)r;
        memcpy(q + r * H, rq + (p / K) * H, (size_t)H);
        memcpy(sf + r * nt, rsf + (p / K) * nt, (size_t)nt);
    }
    for (int32_t e = 0; e < Eloc; e++)
        for (int64_t r = offsets[e] + seen[e]; r < offsets[e + 1]; r++) {
            memset(q + r * H, 0x00, (size_t)H);
            memset(sf + r * nt, 127, (size_t)nt);
        }
    free(cnt);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Fused unpermute + unpad ([FLOW] 核心方法: Fused Permute+Padding /    */
/* Unpermute+Unpadding; the combine side of the expert path)           */
/* ------------------------------------------------------------------ */

/* Expert-ordered rows Y (the permuted, padded buffer after the expert) -> one BF16
 * row per token: out[t] = sum over slots s of w[t,s] * Y[row_id_map[t,s]].  The
 * padding rows are simply never read (unpad).  With w == NULL every weight is 1: the
 * backward of the permute, which sums the gradients of a token's K copies.
 * Y is either BF16 (y_sf == NULL) or row-wise FP8: E4M3 codes with UE8M0 scales
 * [rows, H/128], dequantized to fp32 as decode(q) * 2^e (exact unless the product
 * overflows fp32, which only codes >= 256 at e >= 120 can).
 * Reading (the pages fix no arithmetic for the combine): accumulate in fp32, one
 * fused multiply-add per slot in slot order s = 0..K-1 starting from -0 (the additive
 * identity that also keeps the sign of a zero product, so one slot gives its product
 * exactly and K = 1 inverts the permute bit for bit), then round to BF16 with
 * round-to-nearest-even.  Results must be finite (NaN unspecified).
 * Returns 0, 2 (shape), 7 (a row index outside [0, rows)). */
int orc_unpermute_unpad(const void *y, const uint8_t *y_sf, int64_t rows, int64_t H, const int32_t *row_id_map,
                        const float *w, int64_t T, int32_t K, uint16_t *out)
{
    if (H % 128 || T < 0 || K < 1 || rows < 0)
        return 2;
    for (int64_t p = 0; p < T * K; p++)
        if (row_id_map[p] < 0 || row_id_map[p] >= rows)
            return 7;
    int64_t nt = H / 128;
    const uint16_t *yb = (const uint16_t *)y;
    const uint8_t *yq = (const uint8_t *)y;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++)
        for (int64_t h = 0; h < H; h++) {
            float acc = -0.0f;
            for (int32_t s = 0; s < K; s++) {
                int64_t r = row_id_map[t * K + s];
                float v;
                if (y_sf)
                    v = (float)ldexp(orc_e4m3_decode(yq[r * H + h]), (int)y_sf[r * nt + h / 128] - 127);
                else
                    v = (float)bf16_to_double(yb[r * H + h]);
                float ws = w ? w[t * K + s] : 1.0f;
                acc = fmaf(ws, v, acc);
            }
            out[t * H + h] = f32_to_bf16_rne(acc);
        }
    return 0;
}

/* Range helpers for the exhaustive cross-checks: inputs are the fp32 values with bit
 * patterns first .. first + n - 1 (n <= 2^32 - first). */
void orc_e4m3_encode_f32_range(uint32_t first, int64_t n, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        union {
            uint32_t u;
            float f;
        } v;
        v.u = first + (uint32_t)i;
        out[i] = isfinite(v.f) ? orc_e4m3_encode((double)v.f) : 0;
    }
}

void orc_exp_spec_f32_range(uint32_t first, int64_t n, float *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        union {
            uint32_t u;
            float f;
        } v;
        v.u = first + (uint32_t)i;
        out[i] = isnan(v.f) ? 0.0f : orc_exp_spec(v.f);
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Thread count for the OpenMP loops (the baseline timing at one thread and at all). */
void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
