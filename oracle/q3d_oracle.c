/*
 * q3d_oracle.c -- plain, slow CPU oracle for the Conv3D implicit-GEMM path
 * with fused NVFP4 activation fake-quantisation.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the timed
 * CPU baseline of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library; neither side
 * includes or links the other.
 *
 * Source of truth: the Model-Optimizer "Conv3D Implicit GEMM CUDA kernel"
 * article (lpqz.cn/news/178135):
 *   sec. 3    inputs are taken as FP32, arithmetic in BF16 with FP32 accumulation,
 *             output returned in the input dtype;
 *   sec. 5.1  GEMM view: M = N*OD*OH*OW rows decomposed as (n, od, oh, ow),
 *             K = Cin*kD*kH*kW columns decomposed as (c, kd, kh, kw), input
 *             coordinate od*sd + kd*dd (same for h, w) on the padded input;
 *   sec. 6.1  E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6};
 *   sec. 6.2  global_scale = act_amax / (6*448); block scale =
 *             E4M3(min(block_max / (6*global_scale), 448)) * global_scale;
 *             a scale below 1e-5 is replaced by 1.0;
 *   sec. 6.3  blocks of 16 consecutive K elements of one A row; each value is
 *             sign * E2M1(|v| * inv_scale) * scale, stored as BF16;
 *   sec. 6.4  the standalone fake-quant views the input as [num_blocks, 16];
 *   sec. 7.1  output has the shape torch.nn.functional.conv3d gives,
 *             padding may be asymmetric (applied before the convolution).
 * Where the article stops (rounding of E2M1 ties and of the E4M3 scale) the
 * specification of this library fixes round-to-nearest-even for both.
 *
 * The NVFP4-operand functions (oracle_nvfp4_block_exact, the qfmt 3
 * convolution) define the true-FP4 variant of the same quantiser: the
 * article fixes the formats (sec. 6.1, 6.2) and the weight quantisation
 * along K (sec. 7.2), and the product of the codes is taken exactly; see the
 * comment above oracle_nvfp4_block_exact.
 *
 * The MXFP4 functions follow a second page, the CANN aclnnFlatQuantV2
 * article (its per-group route with E2M1 output: groups of 32, a
 * power-of-two E8M0 scale, the dstTypeMax rule); see the comment above
 * oracle_mx_scale_exp.
 *
 * Every floating-point step of the fake-quantiser is one IEEE-754 binary32
 * operation with round-to-nearest-even, written in the order the article
 * gives it.  Build with -ffp-contract=off and without -ffast-math so the C
 * compiler keeps each float operation separate.  The convolution sums in
 * binary64.
 *
 * Parity pins live in tests/test_oracle_*.py: worked examples derived by
 * hand (tests/golden/), closed forms, invariants, brute force on tiny shapes
 * and library special cases (torch float64 conv3d, torch float8/bfloat16
 * conversions).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* Scalar formats                                                            */
/* ------------------------------------------------------------------------ */

/* E2M1 (1 sign, 2 exponent, 1 mantissa bit): the eight magnitudes listed in
 * sec. 6.1 of the article, indexed by the 3-bit magnitude code.  A code is
 * "even" when its mantissa bit (bit 0) is clear. */
static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Nearest E2M1 value to a, ties to the even code, magnitudes at or above 6
 * saturate to 6.  Sign is carried through (so -0.1 gives -0). */
float oracle_e2m1_rne_sat(float a)
{
    double m = fabs((double)a);
    double q;
    if (isnan(a)) return a;
    if (m >= 6.0) {
        q = 6.0;
    } else {
        int i = 0;
        while (i < 7 && kE2M1Mag[i + 1] <= m) ++i;   /* grid[i] <= m < grid[i+1] */
        double lo = kE2M1Mag[i], hi = kE2M1Mag[i + 1];
        double mid = 0.5 * (lo + hi);                /* exact in binary64 */
        if (m < mid)      q = lo;
        else if (m > mid) q = hi;
        else              q = (i % 2 == 0) ? lo : hi; /* tie: even code */
    }
    return copysignf((float)q, a);
}

/* Value of the non-negative E4M3FN code c in [0, 126] (OCP FP8: bias 7,
 * exponent field 0 holds subnormals m * 2^-9, code 127 is NaN). */
static double e4m3_value(int c)
{
    int e = c >> 3, m = c & 7;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp(1.0 + m / 8.0, e - 7);
}

/* Nearest E4M3FN value to r, ties to the even code, magnitudes above the
 * largest finite value 448 saturate to 448.  Sign is carried through. */
float oracle_e4m3_rne_sat(float r)
{
    double m = fabs((double)r);
    double q;
    if (isnan(r)) return r;
    if (m >= 448.0) {
        q = 448.0;
    } else {
        int c = 0;
        while (c < 126 && e4m3_value(c + 1) <= m) ++c;
        double lo = e4m3_value(c), hi = e4m3_value(c + 1);
        double mid = 0.5 * (lo + hi);
        if (m < mid)      q = lo;
        else if (m > mid) q = hi;
        else              q = (c % 2 == 0) ? lo : hi;
    }
    return copysignf((float)q, r);
}

/* Round a binary32 value to bfloat16 (8 significant bits) with
 * round-to-nearest-even, returned as a binary32 holding that value.
 * bfloat16 is the upper half of binary32, so this rounds away the low 16
 * bits of the pattern. */
float oracle_bf16_round(float v)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {          /* inf / nan: keep */
        if (u & 0x007fffffu) u |= 0x00400000u;
        u &= 0xffff0000u;
    } else {
        uint32_t low = u & 0xffffu;
        uint32_t keep = u & 0xffff0000u;
        uint32_t lsb = (u >> 16) & 1u;
        if (low > 0x8000u || (low == 0x8000u && lsb)) keep += 0x10000u;
        u = keep;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

uint16_t oracle_bf16_bits(float v)
{
    float r = oracle_bf16_round(v);
    uint32_t u;
    memcpy(&u, &r, 4);
    return (uint16_t)(u >> 16);
}

/* binary32 -> binary16 with round-to-nearest-even, via the compiler's
 * _Float16 conversion (IEEE-754 correctly rounded). */
uint16_t oracle_f16_bits(float v)
{
    _Float16 h = (_Float16)v;
    uint16_t b;
    memcpy(&b, &h, 2);
    return b;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 fake-quantisation of one block (sec. 6.2 and 6.3 of the article)    */
/* ------------------------------------------------------------------------ */

/* Fake-quantise n fp32 values as one block: n = 16 (the fused path), a
 * short last block of the fused path (as if zero-filled to 16: zeros change
 * neither the block maximum nor the other outputs), or a block of 32 .. 256
 * (the standalone call's other block sizes, sec. 7.1 / 7.3).  act_amax is
 * the tensor-wide absolute maximum.  out[i] receives the dequantised
 * binary32 value. */
void oracle_fq_block(const float* v, int n, float act_amax, float* out)
{
    /* global scale: act_amax / (6 * 448) */
    float g = act_amax / 2688.0f;
    /* denominator of the block scale: 6 * global_scale */
    float t = 6.0f * g;

    /* block maximum of |v| (exact) */
    float bmax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > bmax) bmax = a;
    }

    /* block_max / (6*global_scale), clamped to the E4M3 range; fminf returns
     * 448 for a NaN quotient (0/0 when act_amax and the block are 0). */
    float r = bmax / t;
    r = fminf(r, 448.0f);
    /* FP8 E4M3 round trip of the per-block scale */
    float s8 = oracle_e4m3_rne_sat(r);
    float scale = s8 * g;
    /* tiny-scale fallback */
    if (scale < 1e-5f) scale = 1.0f;
    float inv = 1.0f / scale;

    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]) * inv;
        float q = oracle_e2m1_rne_sat(a);      /* magnitude on the E2M1 grid */
        float d = q * scale;                   /* dequantised magnitude */
        out[i] = copysignf(d, v[i]);
    }
}

/* Standalone fake-quantisation (sec. 6.4): the flat tensor is split into
 * consecutive blocks of 16.  Returns 0, or -1 if numel is not a multiple of
 * 16. */
int oracle_fp4_fake_quant(const float* x, int64_t numel, float amax, float* out)
{
    if (numel % 16 != 0) return -1;
    for (int64_t b = 0; b < numel; b += 16) oracle_fq_block(x + b, 16, amax, out + b);
    return 0;
}

/* Standalone fake-quantisation with the block size the article's call
 * accepts (sec. 7.1: 16, 32, 64, 128 or 256; sec. 7.3: numel a multiple of
 * it): consecutive blocks of `block` elements.  Returns 0, or -1 for another
 * block size or a numel that is not a multiple of it. */
int oracle_fp4_fake_quant_bs(const float* x, int64_t numel, float amax, int block, float* out)
{
    if (block != 16 && block != 32 && block != 64 && block != 128 && block != 256) return -1;
    if (numel % block != 0) return -1;
    for (int64_t b = 0; b < numel; b += block) oracle_fq_block(x + b, block, amax, out + b);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 operands taken exactly (the true-FP4 product)                        */
/* ------------------------------------------------------------------------ */

/* One block of n values (n <= 16; fewer as if zero-filled) quantised to an
 * NVFP4 operand: the E2M1 magnitude codes q and the E4M3 block scale s8 are
 * the ones oracle_fq_block takes (sec. 6.2, 6.3), and the operand value is
 * sign * q * s8 * g computed exactly in binary64 (q has two significant
 * bits, s8 four and g twenty-four, so the product is exact), without the
 * binary32 rounding of scale and of q * scale, nor the BF16 rounding, of the
 * fake-quantised path.  A block whose scale s8 * g falls below 1e-5 takes
 * the fallback scale 1.0 in the article; that scale is not an E4M3 value
 * times g, so in this variant such a block contributes zero. */
void oracle_nvfp4_block_exact(const float* v, int n, float amax, double* out)
{
    /* global scale and the denominator of the block scale, as in oracle_fq_block */
    float g = amax / 2688.0f;
    float t = 6.0f * g;
    float bmax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > bmax) bmax = a;
    }
    float r = bmax / t;
    r = fminf(r, 448.0f);
    float s8 = oracle_e4m3_rne_sat(r);
    float scale = s8 * g;
    if (scale < 1e-5f) {
        for (int i = 0; i < n; ++i) out[i] = 0.0;
        return;
    }
    float inv = 1.0f / scale;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]) * inv;
        float q = oracle_e2m1_rne_sat(a);
        double d = (double)q * (double)s8 * (double)g;
        out[i] = signbit(v[i]) ? -d : d;
    }
}

/* The flat tensor in consecutive blocks of 16 (sec. 6.4's view), each as
 * oracle_nvfp4_block_exact.  Returns 0, or -1 if numel is not a multiple of
 * 16. */
int oracle_nvfp4_exact(const float* x, int64_t numel, float amax, double* out)
{
    if (numel % 16 != 0) return -1;
    for (int64_t b = 0; b < numel; b += 16) oracle_nvfp4_block_exact(x + b, 16, amax, out + b);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MXFP4 (E2M1 values, power-of-two E8M0 scale, groups of 32)                */
/* ------------------------------------------------------------------------ */

/* Source: the CANN aclnnFlatQuantV2 page (its step 3, the per-group route
 * with FLOAT4_E2M1 output, and step 4, the dstTypeMax rule).  A group of 32
 * consecutive elements shares one scale 2^E stored as E8M0 (exponent only,
 * E in [-127, 127], biased code E + 127):
 *   dst_max == 0  (step 3): E = floor(log2(max|v|)) - emax, emax = 2, the
 *                 exponent of E2M1's largest magnitude 6 = 1.5 * 2^2;
 *   dst_max != 0  (step 4): S = max|v| / dst_max in binary32; E is the
 *                 unbiased exponent of S, raised by one when S is a normal
 *                 number with a biased exponent below 254 and a nonzero
 *                 mantissa (the scale rounds up, so no element exceeds
 *                 dst_max before the E2M1 rounding).
 * Each element becomes E2M1_RNE_SAT(v * 2^-E) (the product is exact) and
 * dequantises to that code times 2^E.  Readings where the page is silent:
 * floor(log2) of a zero or subnormal maximum, and the exponent of a
 * subnormal S, clamp to -127 (the E8M0 minimum); E is clamped to <= 127. */
static int mx_floor_log2(float a)
{
    /* exponent of a binary32 value; zero and subnormals give -127 */
    uint32_t u;
    memcpy(&u, &a, 4);
    int be = (int)((u >> 23) & 0xffu);
    if (be == 0) return -127;
    return be - 127;
}

int oracle_mx_scale_exp(float amax, float dst_max)
{
    int e;
    if (dst_max == 0.0f) {
        e = mx_floor_log2(amax) - 2;
    } else {
        float s = amax / dst_max;
        uint32_t u;
        memcpy(&u, &s, 4);
        int be = (int)((u >> 23) & 0xffu);
        e = mx_floor_log2(s);
        if (be != 0 && be < 254 && (u & 0x007fffffu) != 0) e += 1;
    }
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* One group of n values (n = 32 in the call below): codes[i] receives the
 * signed 4-bit E2M1 code (sign bit 3, magnitude code 0..7), out[i] the
 * dequantised binary32 value; returns E. */
int oracle_mxfp4_block(const float* v, int n, float dst_max, float* out, uint8_t* codes)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    int e = oracle_mx_scale_exp(amax, dst_max);
    double down = ldexp(1.0, -e), up = ldexp(1.0, e);
    for (int i = 0; i < n; ++i) {
        float x = (float)((double)v[i] * down);      /* exact: a power of two */
        float q = oracle_e2m1_rne_sat(x);
        int mag = 0;
        while (mag < 7 && kE2M1Mag[mag] != fabs((double)q)) ++mag;
        if (codes) codes[i] = (uint8_t)(mag | (signbit(q) ? 8 : 0));
        out[i] = (float)((double)q * up);
    }
    return e;
}

/* MXFP4 over a flat tensor (numel % 32 == 0): out receives the dequantised
 * values, scales (if not NULL) the E8M0 byte E + 127 of each group, codes (if
 * not NULL) the signed 4-bit code of each element.  Returns 0, or -1 for a
 * numel that is not a multiple of 32 or a dst_max that is neither 0 nor in
 * [6, 12]. */
int oracle_mxfp4_fake_quant(const float* x, int64_t numel, float dst_max, float* out, uint8_t* scales,
                            uint8_t* codes)
{
    if (numel % 32 != 0) return -1;
    if (!(dst_max == 0.0f || (dst_max >= 6.0f && dst_max <= 12.0f))) return -1;
    for (int64_t b = 0; b < numel; b += 32) {
        int e = oracle_mxfp4_block(x + b, 32, dst_max, out + b, codes ? codes + b : NULL);
        if (scales) scales[b / 32] = (uint8_t)(e + 127);
    }
    return 0;
}

/* The global amax the quantiser takes (sec. 7.2 passes x.abs().max(); the
 * sec. 8.3 inference path gets it from the input quantizer): the largest
 * |x[i]| over the fp32 values of x, 0 for an empty x.  A plain scan; the
 * maximum of magnitudes involves no rounding. */
float oracle_act_amax(const float* x, int64_t numel)
{
    float m = 0.0f;
    for (int64_t i = 0; i < numel; ++i) {
        const float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

/* Round an fp32 array to the storage dtype (0 = fp32, 1 = fp16, 2 = bf16);
 * bits receives the raw pattern (16-bit types) or the binary32 pattern. */
void oracle_round_to_dtype_bits(const float* v, int64_t n, int dtype, void* bits)
{
    for (int64_t i = 0; i < n; ++i) {
        if (dtype == 0)      memcpy((uint32_t*)bits + i, v + i, 4);
        else if (dtype == 1) ((uint16_t*)bits)[i] = oracle_f16_bits(v[i]);
        else                 ((uint16_t*)bits)[i] = oracle_bf16_bits(v[i]);
    }
}

/* ------------------------------------------------------------------------ */
/* Convolution (sec. 5.1): direct sum over (c, kd, kh, kw) in binary64        */
/* ------------------------------------------------------------------------ */

typedef struct {
    /* problem */
    const float* x; int64_t N, C, D, H, W;
    const float* w; int64_t Cout, KD, KH, KW;
    const float* bias;
    int64_t sd, sh, sw, pd, ph, pw, dd, dh, dw;   /* stride, front pad, dilation */
    int64_t OD, OH, OW;
    int quant; float amax;
    int qfmt; int qblock; float dst_max;   /* quantiser: 1 NVFP4 blocks of qblock, 2 MXFP4 groups of 32,
                                               3 NVFP4 operands taken exactly (blocks of 16) */
    const double* wb;        /* the B operand as binary64, [Cout][K]: bf16(w), or for qfmt 3 the
                                exact NVFP4 operand of w */
    /* work list */
    const int64_t* m_list; int64_t n_m;
    double* y;               /* [n_m][Cout] */
    int64_t lo, hi;          /* slice of the work list for one thread */
} conv_job;

/* Row m of the implicit im2col matrix A, in the article's (c, kd, kh, kw)
 * order, as fp32 values of x; zero where the tap falls in the padding. */
static void im2col_row(const conv_job* j, int64_t m, float* row)
{
    int64_t ow = m % j->OW, r = m / j->OW;
    int64_t oh = r % j->OH;  r /= j->OH;
    int64_t od = r % j->OD;
    int64_t n  = r / j->OD;
    int64_t k = 0;
    for (int64_t c = 0; c < j->C; ++c)
        for (int64_t kd = 0; kd < j->KD; ++kd)
            for (int64_t kh = 0; kh < j->KH; ++kh)
                for (int64_t kw = 0; kw < j->KW; ++kw, ++k) {
                    int64_t id = od * j->sd + kd * j->dd - j->pd;
                    int64_t ih = oh * j->sh + kh * j->dh - j->ph;
                    int64_t iw = ow * j->sw + kw * j->dw - j->pw;
                    float v = 0.0f;
                    if (id >= 0 && id < j->D && ih >= 0 && ih < j->H && iw >= 0 && iw < j->W)
                        v = j->x[(((n * j->C + c) * j->D + id) * j->H + ih) * j->W + iw];
                    row[k] = v;
                }
}

static void* conv_worker(void* arg)
{
    const conv_job* j = (const conv_job*)arg;
    int64_t K = j->C * j->KD * j->KH * j->KW;
    float* row = (float*)malloc(sizeof(float) * (size_t)K);
    float* fq = (float*)malloc(sizeof(float) * (size_t)K);
    double* a = (double*)malloc(sizeof(double) * (size_t)K);
    for (int64_t i = j->lo; i < j->hi; ++i) {
        int64_t m = j->m_list[i];
        im2col_row(j, m, row);
        if (j->quant && j->qfmt == 3) {
            /* exact NVFP4 operand: blocks of 16 consecutive K elements of this
             * row, a short last block as if zero-filled; no BF16 rounding */
            for (int64_t b = 0; b < K; b += 16) {
                int nb = (int)((K - b) < 16 ? (K - b) : 16);
                oracle_nvfp4_block_exact(row + b, nb, j->amax, a + b);
            }
        } else if (j->quant && j->qfmt == 2) {
            /* MXFP4 groups of 32 consecutive K elements of this row; a short
             * last group as if zero-filled (zeros leave its maximum alone) */
            for (int64_t b = 0; b < K; b += 32) {
                int nb = (int)((K - b) < 32 ? (K - b) : 32);
                oracle_mxfp4_block(row + b, nb, j->dst_max, fq + b, NULL);
            }
        } else if (j->quant) {
            /* NVFP4 blocks of qblock (16 in the article's kernel, sec. 6.3;
             * 32..256 its call's other block sizes, sec. 7.1) consecutive K
             * elements of this row; a short last block as if zero-filled */
            for (int64_t b = 0; b < K; b += j->qblock) {
                int nb = (int)((K - b) < j->qblock ? (K - b) : j->qblock);
                oracle_fq_block(row + b, nb, j->amax, fq + b);
            }
        } else {
            memcpy(fq, row, sizeof(float) * (size_t)K);
        }
        /* the tensor-core operand is BF16 (the exact NVFP4 operand is final) */
        if (!(j->quant && j->qfmt == 3))
            for (int64_t k = 0; k < K; ++k) a[k] = (double)oracle_bf16_round(fq[k]);
        for (int64_t co = 0; co < j->Cout; ++co) {
            const double* wr = j->wb + co * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += a[k] * wr[k];
            if (j->bias) s += (double)j->bias[co];
            j->y[i * j->Cout + co] = s;
        }
    }
    free(row); free(fq); free(a);
    return NULL;
}

/* Output extent along one dimension (standard convolution arithmetic). */
int64_t oracle_out_dim(int64_t in, int64_t k, int64_t s, int64_t plo, int64_t phi, int64_t d)
{
    if (s < 1 || d < 1 || k < 1 || plo < 0 || phi < 0) return -1;
    int64_t span = in + plo + phi - d * (k - 1) - 1;
    if (span < 0) return 0;
    return span / s + 1;
}

/*
 * y[i][co] for each output row m = m_list[i] (flattened (n, od, oh, ow)),
 * or for every row in order when m_list is NULL (then y is [M][Cout]).
 * x: [N][C][D][H][W] fp32 values of the input; w: [Cout][C][KD][KH][KW] fp32
 * values of the weights (rounded to BF16 here); bias: [Cout] or NULL.
 * stride/pad_lo/pad_hi/dil are (d, h, w).  Returns 0, or -1 on bad
 * arguments.  nthreads <= 0 uses every online core.
 */
static int conv3d_core(const float* x, int64_t N, int64_t C, int64_t D, int64_t H, int64_t W,
                       const float* w, int64_t Cout, int64_t KD, int64_t KH, int64_t KW,
                       const float* bias,
                       const int32_t* stride, const int32_t* pad_lo, const int32_t* pad_hi,
                       const int32_t* dil, int qfmt, int qblock, float act_amax, float dst_max, float w_amax,
                       const int64_t* m_list, int64_t n_m, int nthreads, double* y)
{
    if (qfmt < 0 || qfmt > 3) return -1;
    if (qfmt == 3 && qblock != 16) return -1;
    if (qfmt == 1 && qblock != 16 && qblock != 32 && qblock != 64 && qblock != 128 && qblock != 256) return -1;
    if (qfmt == 2 && (qblock != 32 || !(dst_max == 0.0f || (dst_max >= 6.0f && dst_max <= 12.0f)))) return -1;
    for (int i = 0; i < 3; ++i)
        if (stride[i] < 1 || dil[i] < 1 || pad_lo[i] < 0 || pad_hi[i] < 0) return -1;
    conv_job base;
    memset(&base, 0, sizeof(base));
    base.x = x; base.N = N; base.C = C; base.D = D; base.H = H; base.W = W;
    base.w = w; base.Cout = Cout; base.KD = KD; base.KH = KH; base.KW = KW;
    base.bias = bias;
    base.sd = stride[0]; base.sh = stride[1]; base.sw = stride[2];
    base.pd = pad_lo[0]; base.ph = pad_lo[1]; base.pw = pad_lo[2];
    base.dd = dil[0]; base.dh = dil[1]; base.dw = dil[2];
    base.OD = oracle_out_dim(D, KD, stride[0], pad_lo[0], pad_hi[0], dil[0]);
    base.OH = oracle_out_dim(H, KH, stride[1], pad_lo[1], pad_hi[1], dil[1]);
    base.OW = oracle_out_dim(W, KW, stride[2], pad_lo[2], pad_hi[2], dil[2]);
    base.quant = qfmt != 0; base.amax = act_amax;
    base.qfmt = qfmt; base.qblock = qblock; base.dst_max = dst_max;
    int64_t M = N * base.OD * base.OH * base.OW;
    int64_t K = C * KD * KH * KW;
    if (M <= 0 || K <= 0 || Cout <= 0) return -1;

    int64_t* all = NULL;
    if (!m_list) {
        all = (int64_t*)malloc(sizeof(int64_t) * (size_t)M);
        for (int64_t m = 0; m < M; ++m) all[m] = m;
        m_list = all; n_m = M;
    }
    for (int64_t i = 0; i < n_m; ++i)
        if (m_list[i] < 0 || m_list[i] >= M) { free(all); return -1; }

    double* wb = (double*)malloc(sizeof(double) * (size_t)(Cout * K));
    if (qfmt == 3) {
        /* weights as NVFP4 operands: blocks of 16 along each row's K (sec. 7.2
         * quantises the weights along the reduction axis), scale from w_amax */
        for (int64_t co = 0; co < Cout; ++co)
            for (int64_t b = 0; b < K; b += 16) {
                int nb = (int)((K - b) < 16 ? (K - b) : 16);
                oracle_nvfp4_block_exact(w + co * K + b, nb, w_amax, wb + co * K + b);
            }
    } else {
        for (int64_t i = 0; i < Cout * K; ++i) wb[i] = (double)oracle_bf16_round(w[i]);
    }
    base.wb = wb; base.m_list = m_list; base.n_m = n_m; base.y = y;

    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_m) nthreads = (int)n_m;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    conv_job* jobs = (conv_job*)malloc(sizeof(conv_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = base;
        jobs[t].lo = n_m * t / nthreads;
        jobs[t].hi = n_m * (t + 1) / nthreads;
        pthread_create(&th[t], NULL, conv_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th); free(jobs); free(wb); free(all);
    return 0;
}

/* The convolution with a fake-quantised activation operand: qfmt 0 (none),
 * 1 (NVFP4 blocks of qblock) or 2 (MXFP4 groups of 32, qblock 32). */
int oracle_conv3d_ex(const float* x, int64_t N, int64_t C, int64_t D, int64_t H, int64_t W,
                     const float* w, int64_t Cout, int64_t KD, int64_t KH, int64_t KW,
                     const float* bias,
                     const int32_t* stride, const int32_t* pad_lo, const int32_t* pad_hi,
                     const int32_t* dil, int qfmt, int qblock, float act_amax, float dst_max,
                     const int64_t* m_list, int64_t n_m, int nthreads, double* y)
{
    if (qfmt == 3) return -1;
    return conv3d_core(x, N, C, D, H, W, w, Cout, KD, KH, KW, bias, stride, pad_lo, pad_hi, dil, qfmt, qblock,
                       act_amax, dst_max, 0.0f, m_list, n_m, nthreads, y);
}

/* The true-FP4 convolution: both operands quantised to NVFP4 in blocks of 16
 * along K (activations with act_amax, weights with w_amax) and multiplied as
 * exact operands (oracle_nvfp4_block_exact), summed in binary64, plus the
 * bias. */
int oracle_conv3d_nvfp4(const float* x, int64_t N, int64_t C, int64_t D, int64_t H, int64_t W,
                        const float* w, int64_t Cout, int64_t KD, int64_t KH, int64_t KW,
                        const float* bias,
                        const int32_t* stride, const int32_t* pad_lo, const int32_t* pad_hi,
                        const int32_t* dil, float act_amax, float w_amax,
                        const int64_t* m_list, int64_t n_m, int nthreads, double* y)
{
    return conv3d_core(x, N, C, D, H, W, w, Cout, KD, KH, KW, bias, stride, pad_lo, pad_hi, dil, 3, 16,
                       act_amax, 0.0f, w_amax, m_list, n_m, nthreads, y);
}

/* The article's convolution: NVFP4 blocks of 16 when quant_act is set. */
int oracle_conv3d(const float* x, int64_t N, int64_t C, int64_t D, int64_t H, int64_t W,
                  const float* w, int64_t Cout, int64_t KD, int64_t KH, int64_t KW,
                  const float* bias,
                  const int32_t* stride, const int32_t* pad_lo, const int32_t* pad_hi,
                  const int32_t* dil, int quant_act, float act_amax,
                  const int64_t* m_list, int64_t n_m, int nthreads, double* y)
{
    return oracle_conv3d_ex(x, N, C, D, H, W, w, Cout, KD, KH, KW, bias, stride, pad_lo, pad_hi, dil,
                            quant_act ? 1 : 0, 16, act_amax, 0.0f, m_list, n_m, nthreads, y);
}
