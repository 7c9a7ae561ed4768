/*
 * hq_oracle.c -- plain, slow, single-threaded CPU reference for the three
 * Hadamard-rotation + block-quantization paths.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this file's library.  It shares no code, header,
 * table or constant generator with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (FLT_EVAL_METHOD == 0 on x86-64: every float operation below is one IEEE
 * binary32 operation rounded to nearest even; fmaf() is the fused multiply-add
 * with a single rounding).  No multiply-add is contracted unless fmaf() is
 * written out.
 *
 * Sources (page title, then the part of the page):
 *  [QMOE]  onnxruntime PR #33644, "Add opt-in activation_quantization=
 *          dynamic_fp8 to com.microsoft::QMoE", Description: consecutive K128
 *          groups, saturating nearest-even E4M3, scale max(amax,1e-10) *
 *          float32(1/448), FP32 normalization, FP32 SiLU/SwiGLU before the
 *          second quantizer, and the review note that NaN must stay NaN.
 *  [DSA]   TensorRT-LLM PR #15158 "[#13061][bugfix] Add rotate_activation to
 *          DSA fused_cat_fp8 path", Summary and code flow: cat([pe, nope]) ->
 *          rotate_activation (orthonormal Hadamard) -> fp8_quantize_1x128,
 *          scales transposed; the review thread's (Hq).(Hk) = q.k argument.
 *  [GRP]   TransformerEngine PR #2564 "[NVFP4][MOE] Bug Fix for NVFP4 Grouped
 *          Quant", Greptile summary and changed-file list: grouped row cast +
 *          column Hadamard transform + cast with scale factors, per MoE split.
 *  [FUS]   TransformerEngine PR #2555 review comments (cast.cpp, quantizer.cpp):
 *          split_section % 128 fusion rule, rht_matrix, rowwise output needs
 *          no RHT, the RHT'd columnwise output is the transposed layout.
 *
 * Where the pages leave a step open, the reading taken is stated beside it
 * and listed in the repository's design notes.  Function names start hqo_.
 *
 * Pins (tests/test_oracle_pins.py): E4M3/E2M1 encoders against exact
 * nearest-even brute force over the bit-field grids and torch's e4m3 cast;
 * the butterfly against scipy's Sylvester matrix; FP8 scales/codes against
 * the printed rule with exact rational quotients and crafted midpoint cases;
 * exp against FP64; NVFP4 against exact block-scale/code brute force,
 * dequantization bounds and the inverse-rotation round trip.
 * Scale formats for direct GEMM consumption (TensorRT-LLM PR #15158 review
 * thread: a use_ue8m0 option of the 1x128 quantizer; DeepGEMM issue #320: the
 * tcgen05 data-path layouts of scale factors): UE8M0 FP8 scales and the
 * 128 x 4 interleaved NVFP4 block-scale tiles, pinned by closed forms and an
 * independent construction of the tile permutation.
 * Parity unpinned (readings the pages leave open, each moving results only
 * inside the 2^-20 midpoint window or the 1e-5 rotation tolerance): the
 * ascending butterfly stage order, and the operation order of the NVFP4
 * block scale ((a_b / 6) * S_enc) and of enc = S_enc / sf.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------- helpers */

static float bf16_value(uint16_t bits)
{
    /* BF16 is the upper half of an IEEE binary32 word. */
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ E4M3 */
/*
 * E4M3 ("e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 * infinities, NaN = S.1111.111, largest finite 448 = 1.75 * 2^8, smallest
 * normal 2^-6, subnormals m * 2^-9 (m = 1..7).  [QMOE] asks for saturating
 * nearest-even conversion.  Reading: round the exact binary32 value to the
 * nearest E4M3 value, ties to the even code; a magnitude that rounds above 448
 * (and +-inf) saturates to +-448; the sign of zero is kept; NaN stays NaN.
 */
float hqo_e4m3_decode(uint8_t c)
{
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexpf((float)m, -9);
    else
        v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return sign ? -v : v;
}

uint8_t hqo_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v))
        return sign | 0x7F;
    float a = fabsf(v);
    if (a >= 448.0f)                     /* everything from 448 up saturates */
        return sign | 0x7E;
    if (a == 0.0f)
        return sign;
    int ex;
    frexpf(a, &ex);                      /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                      /* a in [2^E, 2^(E+1)) */
    if (E < -6)
        E = -6;                          /* subnormal range keeps 2^-9 spacing */
    float quantum = ldexpf(1.0f, E - 3); /* spacing of E4M3 values near a */
    float n = nearbyintf(a / quantum);   /* a / quantum is exact; RNE to integer */
    float r = n * quantum;               /* exact E4M3 value, r <= 448 */
    if (r == 0.0f)
        return sign;
    if (r < ldexpf(1.0f, -6))            /* subnormal code: r = m * 2^-9 */
        return sign | (uint8_t)(r / ldexpf(1.0f, -9));
    int rex;
    frexpf(r, &rex);
    int RE = rex - 1;
    int m = (int)((r / ldexpf(1.0f, RE) - 1.0f) * 8.0f);
    return sign | (uint8_t)(((RE + 7) << 3) | m);
}

/* ------------------------------------------------------------------ E2M1 */
/*
 * E2M1 (the element type of NVFP4): magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6},
 * code = sign << 3 | index into that list.  The pages name NVFP4 but no
 * detail.  Reading: the OCP FP4 E2M1 format, round to nearest with ties to the
 * even code, magnitudes from 6 up saturate to 6, the sign of zero is kept.
 * NaN has no code and is outside the contract (returns 0xFF as a marker).
 */
float hqo_e2m1_decode(uint8_t nib)
{
    static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    float v = mag[nib & 7];
    return (nib & 8) ? -v : v;
}

uint8_t hqo_e2m1_encode(float v)
{
    if (isnan(v))
        return 0xFF;
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    float a = fabsf(v);
    if (a >= 6.0f)
        return sign | 7;
    /* spacing of the grid: 0.5 below 2, 1 in [2, 4), 2 in [4, 6] */
    float quantum = a < 2.0f ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
    float r = nearbyintf(a / quantum) * quantum;
    for (uint8_t i = 0; i < 8; ++i)
        if (hqo_e2m1_decode(i) == r)
            return sign | i;
    return 0xFF; /* unreachable */
}

void hqo_encode_array(int fmt, const float *in, uint8_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = fmt == 0 ? hqo_e4m3_encode(in[i]) : hqo_e2m1_encode(in[i]);
}

/* -------------------------------------------------------------- Hadamard */
/*
 * Unnormalised Sylvester-ordered Walsh-Hadamard transform, H[i][j] =
 * (-1)^popcount(i & j), applied in place as butterflies: for h = 1, 2, 4, ...,
 * n/2 (ascending) and every i with (i & h) == 0, (a, b) -> (a + b, a - b).
 * The pages fix only "Hadamard rotation" ([DSA]) and "random Hadamard
 * transform" with a 16x16 rht_matrix ([FUS]); the Sylvester order, the
 * ascending stage order and a single scaling multiply at the end are the
 * reading taken here.
 */
void hqo_fwht(float *v, int n)
{
    for (int h = 1; h < n; h <<= 1)
        for (int i = 0; i < n; ++i)
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

/* 1/sqrt(128) = 2^-3.5 rounded to binary32 (0x3DB504F3); the pages scale the
 * 128-point rotation by 1/sqrt(128) so that it is orthonormal. */
static float c128(void)
{
    uint32_t u = 0x3DB504F3u;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------- scale formats */
/*
 * UE8M0 scale (an 8-bit exponent, no mantissa: a power of two).  The review
 * of [DSA] asks for a use_ue8m0 option of the 1x128 quantizer; the pages give
 * no rounding rule.  Reading: the FP32 scale s of the FP8 rule is rounded up
 * to the smallest power of two not below it (s itself when it is one), so no
 * value quantizes above E4M3's largest (|y| / s_ue <= |y| / s <= 448, up to
 * the rounding of s); +inf stays +inf.  The stored scale is that FP32 power
 * of two; its UE8M0 byte is the binary32 exponent field (bits 30..23).
 */
static float ue8m0_ceil(float s)
{
    if (!(s > 0.0f) || isinf(s))
        return s;
    int e;
    const float f = frexpf(s, &e); /* s = f * 2^e, f in [0.5, 1) */
    return f == 0.5f ? s : ldexpf(1.0f, e);
}

/*
 * Interleaved block-scale layout read by block-scaled tcgen05 MMAs (the
 * layout DeepGEMM issue #320's discussion of tcgen05 data paths refers to;
 * the pages print no formula).  Reading: a scale matrix of R rows (a
 * multiple of 128) and C columns (a multiple of 4) is cut into tiles of 128
 * rows x 4 columns, stored tile-row major (tile (R/128 index, C/4 index) at
 * byte 512 * (tr * C/4 + tc)); inside a tile, element (r, c) sits at byte
 * 16 * (r % 32) + 4 * (r / 32) + c, i.e. 32 lines of 16 bytes, line i holding
 * rows i, i + 32, i + 64, i + 96, four scales each.
 */
static int64_t sf_swizzled(int64_t r, int64_t c, int64_t C)
{
    return ((r / 128) * (C / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4;
}

int64_t hqo_sf_swizzled_offset(int64_t r, int64_t c, int64_t C)
{
    return sf_swizzled(r, c, C);
}

/* ---------------------------------------------------------------- FP8 1xN */
/*
 * One group of n values -> n E4M3 codes and one FP32 scale, as [QMOE] states:
 *   amax = max |y|                      (fmaxf, so a NaN element is skipped)
 *   s    = max(amax, 1e-10f) * float32(1/448)
 *   q_i  = e4m3(y_i / s)                (IEEE binary32 division)
 * The page says "FP32 div.full normalization" and notes that the choice of
 * division changes codes by one ulp at FP8 midpoints.  Reading: correctly
 * rounded IEEE division.  `pre`, when given, receives y_i / s (the value that
 * is rounded to E4M3); `amax_out`, when given, receives amax.
 */
static void quant_group_fp8(const float *y, int n, uint8_t *q, float *scale, float *amax_out, float *pre,
                            int ue8m0)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        amax = fmaxf(amax, fabsf(y[i]));
    const float inv448 = 1.0f / 448.0f; /* binary32 constant, 0x3B124925 */
    float s = fmaxf(amax, 1e-10f) * inv448;
    if (ue8m0)
        s = ue8m0_ceil(s);  /* y / s is then exact (a power of two), unless it underflows */
    for (int i = 0; i < n; ++i) {
        float t = y[i] / s;
        if (pre)
            pre[i] = t;
        q[i] = hqo_e4m3_encode(t);
    }
    *scale = s;
    if (amax_out)
        *amax_out = amax;
}

/*
 * DSA indexer prep [DSA]: for token t and group (head) g the 128-vector is
 * a[t, g, 0:a_width] followed by b[t, g, 0:b_width] (pe first, then nope),
 * optionally rotated by the orthonormal 128-point Hadamard (Sylvester
 * butterfly, then * 1/sqrt(128)), then quantized as one 1x128 FP8 group.
 * Element (t, g, j) of a is a[t * a_row_stride + g * a_width + j]; b likewise.
 * Output codes: out[(t * G + g) * 128 + j].  Scales: scale_layout 0 (row
 * major) puts group (t, g) at scales[t * G + g]; layout 1 (transposed, as the
 * indexer stores them) at scales[g * scale_ld + t].  amax_opt, when given,
 * receives each group's amax in the scales' layout.  scale_layout may add
 * 256: UE8M0 scales (ue8m0_ceil).
 * Returns 0, or -1 for arguments this reference does not accept.
 */
int hqo_cat_rotate_fp8(const uint16_t *a, int64_t a_row_stride, int a_width,
                       const uint16_t *b, int64_t b_row_stride, int b_width,
                       int64_t M, int G, int hadamard_n,
                       uint8_t *out, float *scales, int scale_layout, int64_t scale_ld,
                       float *amax_opt, float *pre)
{
    const int ue8m0 = (scale_layout & 256) != 0;
    scale_layout &= ~256;
    if (a_width < 0 || b_width < 0 || a_width + b_width != 128 || (b_width > 0 && !b))
        return -1;
    if (hadamard_n != 0 && hadamard_n != 128)
        return -1;
    const float c = c128();
    float v[128];
    for (int64_t t = 0; t < M; ++t)
        for (int g = 0; g < G; ++g) {
            for (int j = 0; j < a_width; ++j)
                v[j] = bf16_value(a[t * a_row_stride + (int64_t)g * a_width + j]);
            for (int j = 0; j < b_width; ++j)
                v[a_width + j] = bf16_value(b[t * b_row_stride + (int64_t)g * b_width + j]);
            if (hadamard_n == 128) {
                hqo_fwht(v, 128);
                for (int j = 0; j < 128; ++j)
                    v[j] = v[j] * c;
            }
            int64_t grp = t * G + g;
            float s, am;
            quant_group_fp8(v, 128, out + grp * 128, &s, &am, pre ? pre + grp * 128 : 0, ue8m0);
            const int64_t si = scale_layout == 0 ? grp : (int64_t)g * scale_ld + t;
            scales[si] = s;
            if (amax_opt)
                amax_opt[si] = am;
        }
    return 0;
}

/* ------------------------------------------------------------ SwiGLU exp */
/*
 * exp(x) in binary32, written from the mathematics so that both sides of the
 * comparison evaluate one fixed sequence of IEEE operations (the pages give
 * no exp algorithm; [QMOE] only says SiLU/SwiGLU run in FP32):
 *  - Cody & Waite argument reduction (W. J. Cody, W. Waite, "Software Manual
 *    for the Elementary Functions", 1980): k = rint(x * log2(e)),
 *    r = (x - k * LN2_HI) - k * LN2_LO, each step one fmaf;
 *  - e^r by its Taylor series to degree 7 (|r| <= ln2/2, truncation error
 *    below 6e-9 relative), Horner form with fmaf;
 *  - multiply by 2^k, split in two exact power-of-two steps at the ends of
 *    the exponent range so that only the last multiply rounds.
 * x > 88.8 -> +inf, x < -104 -> +0 (both beyond binary32 range), NaN -> NaN.
 */
static float pow2i(int k) /* 2^k for -126 <= k <= 127 */
{
    uint32_t u = (uint32_t)(k + 127) << 23;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

float hqo_exp(float x)
{
    if (isnan(x))
        return x;
    if (x > 88.8f)
        return INFINITY;
    if (x < -104.0f)
        return 0.0f;
    const float LOG2E = 1.44269502f;       /* 0x3FB8AA3B */
    const float LN2_HI = 0.693145752f;     /* 0x3F317200: 15 significant bits */
    const float LN2_LO = 1.42860677e-06f;  /* 0x35BFBE8E: ln2 - LN2_HI */
    float k = nearbyintf(x * LOG2E);
    float r = fmaf(-k, LN2_HI, x);
    r = fmaf(-k, LN2_LO, r);
    /* Taylor coefficients 1/n!, each rounded once to binary32, n = 7 .. 0 */
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ki = (int)k;
    if (ki > 127)
        return (p * pow2i(127)) * pow2i(ki - 127);
    if (ki < -126)
        return (p * pow2i(ki + 100)) * pow2i(-100);
    return p * pow2i(ki);
}

void hqo_exp_array(const float *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = hqo_exp(in[i]);
}

/* SiLU(g) * u in binary32 [QMOE]: silu = g / (1 + exp(-g)), one IEEE
 * division; no rounding to a narrower type in between. */
static float swiglu(float g, float u)
{
    float e = hqo_exp(-g);
    float silu = g / (1.0f + e);
    return silu * u;
}

/*
 * QMoE dynamic FP8 activations [QMOE]: rows of K_out values, quantized in
 * consecutive groups of 128 with the FP8 rule above.
 *   mode 0: in is BF16 [M, K_out]
 *   mode 1: in is FP32 [M, K_out]
 *   mode 2: in is FP32 [M, 2*K_out]; gate = columns 0..K_out-1, up = columns
 *           K_out..2*K_out-1 ("2x2048": the reading is two halves, not an
 *           interleave); the quantized value is SiLU(gate) * up.
 * out: [M, K_out] codes; scales (and amax_opt, when given, each group's
 * amax): [M, K_out/128] row major.  mode may add 256: UE8M0 scales.
 */
int hqo_swiglu_fp8_k128(int mode, const void *in, int64_t M, int64_t K_out,
                        uint8_t *out, float *scales, float *amax_opt, float *pre)
{
    const int ue8m0 = (mode & 256) != 0;
    mode &= ~256;
    if (K_out % 128 != 0 || mode < 0 || mode > 2)
        return -1;
    const int64_t groups = K_out / 128;
    float y[128];
    for (int64_t m = 0; m < M; ++m)
        for (int64_t g = 0; g < groups; ++g) {
            for (int j = 0; j < 128; ++j) {
                int64_t col = g * 128 + j;
                if (mode == 0)
                    y[j] = bf16_value(((const uint16_t *)in)[m * K_out + col]);
                else if (mode == 1)
                    y[j] = ((const float *)in)[m * K_out + col];
                else {
                    const float *row = (const float *)in + m * 2 * K_out;
                    y[j] = swiglu(row[col], row[K_out + col]);
                }
            }
            int64_t grp = m * groups + g;
            quant_group_fp8(y, 128, out + grp * 128, &scales[grp], amax_opt ? &amax_opt[grp] : 0,
                            pre ? pre + grp * 128 : 0, ue8m0);
        }
    return 0;
}

/* ----------------------------------------------------------------- NVFP4 */
/*
 * NVFP4 two-level scaling.  The pages name the format ("NVFP4", E2M1 codes
 * with E4M3 1x16 block scales and an FP32 global scale) but print no formula.
 * Reading, per section and per direction:
 *   A     = max |v| over the section's values
 *   S_enc = 2688 / A   (6 * 448: the section's amax maps to the largest
 *                       E2M1 value times the largest E4M3 value); 1 if A == 0
 *                       or the quotient is not finite
 *   sdec  = 1 / S_enc
 * and per block of 16 values:
 *   a_b   = max |v_i|
 *   sf    = e4m3((a_b / 6) * S_enc)
 *   enc   = sf == 0 ? 0 : S_enc / float(sf)
 *   code  = e2m1(v_i * enc)
 * so that v_i ~= e2m1_value(code) * float(sf) * sdec.
 */
/* S_enc = 2688 / A; 1 when A is not positive (0, or a negative or NaN amax
 * given by the caller: reading, treated like A = 0) or 2688 / A is not
 * finite. */
static float global_encode_scale(float A)
{
    float S = 2688.0f / A;
    if (!(A > 0.0f) || !isfinite(S))
        S = 1.0f;
    return S;
}

/* ------------------------------------------------ stochastic rounding */
/*
 * Philox4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
 * "Parallel random numbers: as easy as 1, 2, 3", SC 2011): ten rounds of
 * the 4x32 Philox bijection on the counter, the key bumped by the Weyl
 * increments before every round but the first.  A round maps
 * (c0, c1, c2, c3) to (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1,
 * lo(M0 c0)) with the paper's multipliers M0, M1.
 */
void hqo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;  /* multipliers */
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;  /* Weyl increments of the key */
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        const uint64_t p0 = (uint64_t)M0 * c[0], p1 = (uint64_t)M1 * c[2];
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c[1] ^ k0, n1 = (uint32_t)p1;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c[3] ^ k1, n3 = (uint32_t)p0;
        c[0] = n0;
        c[1] = n1;
        c[2] = n2;
        c[3] = n3;
    }
    for (int i = 0; i < 4; ++i)
        out[i] = c[i];
}

/* Byte `pos` of the random byte stream of `seed`: the little-endian bytes of
 * the 32-bit words w_i = word (i mod 4) of Philox4x32-10(counter = i / 4 as
 * a 64-bit number in the two low words, key = seed's two halves). */
static uint8_t sr_byte(uint64_t seed, uint64_t pos)
{
    const uint64_t blk = pos / 16;
    const uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    hqo_philox4x32_10(ctr, key, out);
    return (uint8_t)(out[(pos % 16) / 4] >> (8 * (pos % 4)));
}

/* E2M1 code of t by stochastic rounding with the random byte r: |t| rounds up
 * to the next E2M1 value iff r < floor(256 * f), f the fraction of |t| above
 * the value below it in units of the grid step there (0.5 below 2, 1 below
 * 4, 2 below 6); |t| >= 6 (and NaN) saturate to 6; the sign is kept, zero
 * included (reading: the pages name stochastic rounding but give no rule). */
static uint8_t e2m1_sr(float t, uint8_t r)
{
    const uint8_t sign = signbit(t) ? 8 : 0;
    const float a = fabsf(t);
    if (!(a < 6.0f))
        return sign | 7;
    const float step = a < 2.0f ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
    const float q = a / step;      /* exact: a power-of-two step */
    const float n = floorf(q);
    const float f = q - n;         /* exact */
    const unsigned F = (unsigned)(f * 256.0f);   /* floor: f * 256 < 256 */
    const unsigned kk = (unsigned)n + (r < F ? 1u : 0u);
    return sign | (uint8_t)(step == 0.5f ? kk : (step == 1.0f ? kk + 2u : kk + 4u));
}

/* e2m1_sr over arrays (for the pins). */
void hqo_e2m1_sr_array(const float *t, const uint8_t *r, uint8_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = e2m1_sr(t[i], r[i]);
}

/* Quantize one block of 16 values; codes packed two per byte, element 2k in
 * the low nibble and 2k+1 in the high nibble (reading: the pages are silent
 * on the packing).  rnd, when given, holds the 16 random bytes of stochastic
 * rounding; else round to nearest even. */
static void nvfp4_block_r(const float *v, float S_enc, uint8_t *codes8, uint8_t *sf_out, float *pre,
                          const uint8_t *rnd)
{
    float ab = 0.0f;
    for (int i = 0; i < 16; ++i)
        ab = fmaxf(ab, fabsf(v[i]));
    uint8_t sf = hqo_e4m3_encode((ab / 6.0f) * S_enc);
    float sff = hqo_e4m3_decode(sf);
    float enc = sff == 0.0f ? 0.0f : S_enc / sff;
    for (int k = 0; k < 8; ++k) {
        float t0 = v[2 * k] * enc, t1 = v[2 * k + 1] * enc;
        if (pre) {
            pre[2 * k] = t0;
            pre[2 * k + 1] = t1;
        }
        const uint8_t q0 = rnd ? e2m1_sr(t0, rnd[2 * k]) : (uint8_t)(hqo_e2m1_encode(t0) & 0xF);
        const uint8_t q1 = rnd ? e2m1_sr(t1, rnd[2 * k + 1]) : (uint8_t)(hqo_e2m1_encode(t1) & 0xF);
        codes8[k] = (uint8_t)(q0 | (q1 << 4));
    }
    *sf_out = sf;
}

static void nvfp4_block(const float *v, float S_enc, uint8_t *codes8, uint8_t *sf_out, float *pre)
{
    nvfp4_block_r(v, S_enc, codes8, sf_out, pre, 0);
}

/* The 16-point random Hadamard transform of [GRP]/[FUS]: v = 0.25 * H16 *
 * diag(sigma) * x, sigma_i = -1 where bit i of sign_mask is set (i is the
 * position inside the block). */
static void rht16(const float *x, uint16_t sign_mask, float *v)
{
    for (int i = 0; i < 16; ++i)
        v[i] = ((sign_mask >> i) & 1) ? -x[i] : x[i];
    hqo_fwht(v, 16);
    for (int i = 0; i < 16; ++i)
        v[i] = v[i] * 0.25f;
}

/*
 * Grouped RHT + NVFP4 cast [GRP], [FUS].  x: BF16 [M, K] row major, rows split
 * into S consecutive sections of split_rows[s] rows (each a multiple of 128,
 * [FUS]'s fusion rule; K a multiple of 128).
 * flags bit 0 (rowwise): plain cast of x along K (the pages' rowwise output
 *   carries no RHT):  row_codes [M, K/2], row_sf [M, K/16].
 * flags bit 2 (with bit 0): the rowwise output instead casts the 16-point RHT
 *   of every 16-element row block along K (the same sign mask, sigma by the
 *   position inside the block): the other reading of "RHT ... rowwise and
 *   columnwise"; section amax and block scales then come from the rotated
 *   values.
 * flags bit 1 (columnwise): per section, the 16-point RHT along M (16
 *   consecutive rows of one column), cast, stored transposed: section s
 *   starting at row r0 owns col_codes[K*r0/2 ...] as [K, M_s/2] and
 *   col_sf[K*r0/16 ...] as [K, M_s/16].
 * amax_*[s], sdec_*[s] receive A and 1/S_enc of the requested directions;
 * an empty section gives A = 0, sdec = 1.
 * flags bit 4 (amax given): amax_*[s] are inputs instead, the section amax a
 *   caller computed beforehand (of the rotated values where the direction is
 *   rotated); there is no amax pass, S_enc and everything after it follow
 *   from the given A, and sdec_*[s] = 1/S_enc(A) for every section, empty
 *   ones included.  The pages do not describe this mode: it is the one-pass
 *   cast that a known amax allows, checked here by its definition.
 * flags bit 5 / bit 6 (stochastic rounding, rowwise / columnwise; P2
 *   discusses the Philox generator and deterministic offsets of TE's
 *   stochastic rounding for this cast but gives no rule): the E2M1 codes of
 *   that direction round stochastically (e2m1_sr) with random byte
 *   offset + e of the stream of seed (rowwise) or seed + 1 (columnwise), e
 *   the element's index in its output (r*K + c rowwise; the index inside
 *   col_codes' element order columnwise).  Block scales stay nearest-even.
 * flags bit 7 (128, scale layout for block-scaled MMAs): row_sf and each
 *   section's col_sf block are stored in the interleaved 128 x 4 tiles of
 *   sf_swizzled (rows M and K, columns K/16 and M_s/16: all multiples of the
 *   tile, so the layout is a permutation of the plain one, section by
 *   section).
 * row_pre / col_pre, when given, receive the value rounded to E2M1 per
 * element, in the output's layout.
 */
int hqo_group_rht_quant_sr(const uint16_t *x, int64_t M, int64_t K,
                           const int64_t *split_rows, int S, uint16_t sign_mask, unsigned flags,
                           uint64_t seed, uint64_t offset,
                           uint8_t *row_codes, uint8_t *row_sf, uint8_t *col_codes, uint8_t *col_sf,
                           float *amax_row, float *amax_col, float *sdec_row, float *sdec_col,
                           float *row_pre, float *col_pre)
{
    uint8_t rnd[16];
    if (K % 128 != 0 || S < 0)
        return -1;
    int64_t total = 0;
    for (int s = 0; s < S; ++s) {
        if (split_rows[s] < 0 || split_rows[s] % 128 != 0)
            return -1;
        total += split_rows[s];
    }
    if (total != M)
        return -1;

    int64_t r0 = 0;
    float blk[16], v[16];
    for (int s = 0; s < S; ++s) {
        const int64_t Ms = split_rows[s];
        const int given = (flags & 16) != 0;
        if (flags & 1) {
            const int rotate = (flags & 4) != 0;
            /* first pass: section amax (of the rotated blocks if rotating) */
            float A = 0.0f;
            for (int64_t r = r0; r < r0 + Ms && !given; ++r)
                for (int64_t kb = 0; kb < K / 16; ++kb) {
                    for (int i = 0; i < 16; ++i)
                        blk[i] = bf16_value(x[r * K + kb * 16 + i]);
                    if (rotate)
                        rht16(blk, sign_mask, v);
                    for (int i = 0; i < 16; ++i)
                        A = fmaxf(A, fabsf(rotate ? v[i] : blk[i]));
                }
            if (given)
                A = amax_row[s];
            float S_enc = global_encode_scale(A);
            amax_row[s] = A;
            sdec_row[s] = 1.0f / S_enc;
            /* second pass: cast */
            for (int64_t r = r0; r < r0 + Ms; ++r)
                for (int64_t kb = 0; kb < K / 16; ++kb) {
                    for (int i = 0; i < 16; ++i)
                        blk[i] = bf16_value(x[r * K + kb * 16 + i]);
                    if (rotate)
                        rht16(blk, sign_mask, v);
                    if (flags & 32)  /* element r*K + c of the rowwise output: stream of seed */
                        for (int i = 0; i < 16; ++i)
                            rnd[i] = sr_byte(seed, offset + (uint64_t)(r * K + kb * 16 + i));
                    nvfp4_block_r(rotate ? v : blk, S_enc, row_codes + r * (K / 2) + kb * 8,
                                  row_sf + ((flags & 128) ? sf_swizzled(r, kb, K / 16) : r * (K / 16) + kb),
                                  row_pre ? row_pre + r * K + kb * 16 : 0, (flags & 32) ? rnd : 0);
                }
        }
        if (flags & 2) {
            /* first pass: section amax of the rotated values */
            float A = 0.0f;
            for (int64_t c = 0; c < K && !given; ++c)
                for (int64_t mb = 0; mb < Ms / 16; ++mb) {
                    for (int i = 0; i < 16; ++i)
                        blk[i] = bf16_value(x[(r0 + mb * 16 + i) * K + c]);
                    rht16(blk, sign_mask, v);
                    for (int i = 0; i < 16; ++i)
                        A = fmaxf(A, fabsf(v[i]));
                }
            if (given)
                A = amax_col[s];
            float S_enc = global_encode_scale(A);
            amax_col[s] = A;
            sdec_col[s] = 1.0f / S_enc;
            uint8_t *cc = col_codes + K * r0 / 2;
            uint8_t *cs = col_sf + K * r0 / 16;
            /* second pass: cast, transposed [K, Ms] */
            for (int64_t c = 0; c < K; ++c)
                for (int64_t mb = 0; mb < Ms / 16; ++mb) {
                    for (int i = 0; i < 16; ++i)
                        blk[i] = bf16_value(x[(r0 + mb * 16 + i) * K + c]);
                    rht16(blk, sign_mask, v);
                    if (flags & 64)  /* element of col_codes: stream of seed + 1 */
                        for (int i = 0; i < 16; ++i)
                            rnd[i] = sr_byte(seed + 1, offset + (uint64_t)(K * r0 + c * Ms + mb * 16 + i));
                    nvfp4_block_r(v, S_enc, cc + c * (Ms / 2) + mb * 8,
                                  cs + ((flags & 128) ? sf_swizzled(c, mb, Ms / 16) : c * (Ms / 16) + mb),
                                  col_pre ? col_pre + K * r0 + c * Ms + mb * 16 : 0, (flags & 64) ? rnd : 0);
                }
        }
        if (Ms == 0 && !given) {
            if (flags & 1) { amax_row[s] = 0.0f; sdec_row[s] = 1.0f; }
            if (flags & 2) { amax_col[s] = 0.0f; sdec_col[s] = 1.0f; }
        }
        r0 += Ms;
    }
    return 0;
}

/* hqo_group_rht_quant_sr with seed and offset 0. */
int hqo_group_rht_quant(const uint16_t *x, int64_t M, int64_t K,
                        const int64_t *split_rows, int S, uint16_t sign_mask, unsigned flags,
                        uint8_t *row_codes, uint8_t *row_sf, uint8_t *col_codes, uint8_t *col_sf,
                        float *amax_row, float *amax_col, float *sdec_row, float *sdec_col,
                        float *row_pre, float *col_pre)
{
    return hqo_group_rht_quant_sr(x, M, K, split_rows, S, sign_mask, flags, 0, 0, row_codes, row_sf, col_codes,
                                  col_sf, amax_row, amax_col, sdec_row, sdec_col, row_pre, col_pre);
}

/* ------------------------------------------------------------ FP4 DSA */
/*
 * The DSA indexer prep with an NVFP4 output instead of FP8 ([DSA]: the FP4
 * path, fused_cat_fp4, lacks the rotation; restoring it is the follow-up the
 * page names).  The pages give no FP4 format; reading: the vector (t, g) is
 * concatenated and rotated exactly as in hqo_cat_rotate_fp8, then quantized
 * with the two-level NVFP4 scheme of hqo_group_rht_quant, the 128-vector
 * taking the place of a section:
 *   A = max |v| over the 128 values, S_enc = global_encode_scale(A),
 *   eight blocks of 16 consecutive values: E4M3 block scale and E2M1 codes
 *   (nvfp4_block), the vector's decode scale 1/S_enc stored like the FP8
 *   scales (row major [M, G] or transposed [G, scale_ld]).
 * codes: [M, G*64] bytes (vector (t, g) at (t*G + g)*64, element 2k in the
 * low nibble); block_sf: [M, G*8] E4M3 codes (scale_layout + 128: the
 * interleaved tiles of sf_swizzled, M a multiple of 128); amax_opt: A per vector in the
 * scales' layout; pre: the value rounded to E2M1 per element, [M, G*128].
 * Returns 0, or -1 for arguments this reference does not accept.
 */
int hqo_cat_rotate_nvfp4(const uint16_t *a, int64_t a_row_stride, int a_width,
                         const uint16_t *b, int64_t b_row_stride, int b_width,
                         int64_t M, int G, int hadamard_n,
                         uint8_t *codes, uint8_t *block_sf, float *sdec, int scale_layout, int64_t scale_ld,
                         float *amax_opt, float *pre)
{
    const int swz = (scale_layout & 128) != 0;
    scale_layout &= ~128;
    if (swz && M % 128 != 0)
        return -1;
    if (a_width < 0 || b_width < 0 || a_width + b_width != 128 || (b_width > 0 && !b))
        return -1;
    if (hadamard_n != 0 && hadamard_n != 128)
        return -1;
    const float c = c128();
    float v[128];
    for (int64_t t = 0; t < M; ++t)
        for (int g = 0; g < G; ++g) {
            for (int j = 0; j < a_width; ++j)
                v[j] = bf16_value(a[t * a_row_stride + (int64_t)g * a_width + j]);
            for (int j = 0; j < b_width; ++j)
                v[a_width + j] = bf16_value(b[t * b_row_stride + (int64_t)g * b_width + j]);
            if (hadamard_n == 128) {
                hqo_fwht(v, 128);
                for (int j = 0; j < 128; ++j)
                    v[j] = v[j] * c;
            }
            float A = 0.0f;
            for (int j = 0; j < 128; ++j)
                A = fmaxf(A, fabsf(v[j]));
            const float S_enc = global_encode_scale(A);
            const int64_t vec = t * G + g;
            for (int blk = 0; blk < 8; ++blk)
                nvfp4_block(v + 16 * blk, S_enc, codes + vec * 64 + 8 * blk,
                            block_sf + (swz ? sf_swizzled(t, (int64_t)g * 8 + blk, (int64_t)G * 8) : vec * 8 + blk),
                            pre ? pre + vec * 128 + 16 * blk : 0);
            const int64_t si = scale_layout == 0 ? vec : (int64_t)g * scale_ld + t;
            sdec[si] = 1.0f / S_enc;
            if (amax_opt)
                amax_opt[si] = A;
        }
    return 0;
}
