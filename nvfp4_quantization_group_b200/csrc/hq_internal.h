// hq_internal.h -- kernel parameter blocks and declarations shared by the
// hq host layer (hq_api.cu) and the kernels (hq_fp8.cu, hq_nvfp4.cu).
#pragma once

#include <cuda.h>  // CUtensorMap (types only: the encoder is reached through the runtime)
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq.h"
#include "hq_device.cuh"

namespace hq {

// --------------------------------------------------------------- FP8 paths
struct CatRotateParams {
    const uint16_t* a;
    const uint16_t* b;
    int64_t a_row_stride, b_row_stride;
    int a_width, b_width;
    int64_t nvec;  // M * G vectors of 128
    int64_t M;     // rows (tokens)
    int64_t ntiles;  // tiles of 32 vectors (see cat_rotate_tiles)
    uint32_t g_magic;      // floor((2^32 - 1) / G): v / G by multiply-high
    uint32_t gt_magic;     // the same for the group tiles of the transposed layout
    int wide32;            // 32-element quarters never straddle a and b, 32-byte aligned: 32-byte loads
    int G;
    int rotate;    // 1: H128 / sqrt(128); 0: none
    uint8_t* out;     // FP8: codes [M, G*128]; FP4: E2M1 codes [M, G*64]
    float* scales;    // FP8: group scales; FP4: per-vector decode scales (1 / S_enc)
    uint8_t* sf;      // FP4: E4M3 block scales [M, G*8]
    float* amax;  // NULL or per-group amax, in the scales' layout
    int scale_layout;
    int64_t scale_ld;
    int ue8m0;       // FP8: scales rounded up to powers of two
    int sf_swizzle;  // FP4: block scales in the interleaved 128 x 4 tiles
};

struct K128Params {
    const void* in;
    int64_t K_out;
    int64_t ngroups;    // M * K_out / 128 (< 2^31)
    uint32_t gpr_magic;  // floor((2^32 - 1) / (K_out / 128)): row of a group by multiply-high
    uint8_t* out;
    float* scales;
    float* amax;  // NULL or per-group amax [M, K_out / 128]
    int ue8m0;    // scales rounded up to powers of two
};

constexpr int K128_THREADS = 256;   // 8 warps, two K128 groups per warp step
constexpr int K128_UNROLL = 4;      // warp steps with loads in flight

int cat_rotate_blocks_per_sm(bool fp4);  // resident CTAs of the FP8 / FP4 kernel
int64_t cat_rotate_tiles(const CatRotateParams& p);
int cat_rotate_group_tiles(int G);  // group tiles of the transposed-scale layout
void launch_cat_rotate(const CatRotateParams& p, int grid, cudaStream_t st, bool fp4);
void launch_k128(int mode, const K128Params& p, int grid, cudaStream_t st);
void launch_convert(int fmt, const float* in, uint8_t* out, int64_t n, int grid, cudaStream_t st);
void launch_convert_e2m1_sr(const float* in, const uint8_t* rnd, uint8_t* out, int64_t n, int grid,
                            cudaStream_t st);

// exp(x) in binary32 by one fixed sequence of IEEE operations: Cody & Waite
// reduction k = rint(x * log2(e)), r = (x - k*LN2_HI) - k*LN2_LO (two FMAs),
// e^r by its degree-7 Taylor polynomial (Horner, FMA), times 2^k in at most
// two exact power-of-two steps.  x > 88.8 -> +inf, x < -104 -> +0.
__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

__device__ __forceinline__ float hq_exp_core(float x, float& p) {
    const float LOG2E = __uint_as_float(0x3FB8AA3Bu);
    const float LN2_HI = __uint_as_float(0x3F317200u);
    const float LN2_LO = __uint_as_float(0x35BFBE8Eu);
    const float k = rintf(__fmul_rn(x, LOG2E));
    float r = __fmaf_rn(-k, LN2_HI, x);
    r = __fmaf_rn(-k, LN2_LO, r);
    p = __uint_as_float(0x39500D01u);                  // RN(1/5040)
    p = __fmaf_rn(p, r, __uint_as_float(0x3AB60B61u)); // RN(1/720)
    p = __fmaf_rn(p, r, __uint_as_float(0x3C088889u)); // RN(1/120)
    p = __fmaf_rn(p, r, __uint_as_float(0x3D2AAAABu)); // RN(1/24)
    p = __fmaf_rn(p, r, __uint_as_float(0x3E2AAAABu)); // RN(1/6)
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    return k;
}

__device__ __forceinline__ float hq_exp(float x) {
    // |x| < 87 (NaN fails the test): k = rint(x log2 e) lies in [-126, 126]
    // and the scaling is one exact step, the same operations as below.  Here
    // rint is the addition of 1.5 * 2^23 (round to nearest even, exact for
    // |t| < 2^22), whose bits also give k and 2^k as integers.
    if (fabsf(x) < 87.0f) {
        const float LOG2E = __uint_as_float(0x3FB8AA3Bu);
        const float LN2_HI = __uint_as_float(0x3F317200u);
        const float LN2_LO = __uint_as_float(0x35BFBE8Eu);
        const float big = __fadd_rn(__fmul_rn(x, LOG2E), 12582912.0f);  // 1.5 * 2^23 + rint(x log2 e)
        const float k = __fsub_rn(big, 12582912.0f);
        float r = __fmaf_rn(-k, LN2_HI, x);
        r = __fmaf_rn(-k, LN2_LO, r);
        float p = __uint_as_float(0x39500D01u);                  // RN(1/5040)
        p = __fmaf_rn(p, r, __uint_as_float(0x3AB60B61u)); // RN(1/720)
        p = __fmaf_rn(p, r, __uint_as_float(0x3C088889u)); // RN(1/120)
        p = __fmaf_rn(p, r, __uint_as_float(0x3D2AAAABu)); // RN(1/24)
        p = __fmaf_rn(p, r, __uint_as_float(0x3E2AAAABu)); // RN(1/6)
        p = __fmaf_rn(p, r, 0.5f);
        p = __fmaf_rn(p, r, 1.0f);
        p = __fmaf_rn(p, r, 1.0f);
        const uint32_t two_k = (__float_as_uint(big) - 0x4B400000u + 127u) << 23;  // bits of 2^k
        return __fmul_rn(p, __uint_as_float(two_k));
    }
    if (isnan(x)) return x;
    if (x > 88.8f) return __uint_as_float(0x7F800000u);
    if (x < -104.0f) return 0.0f;
    float p;
    const int ki = (int)hq_exp_core(x, p);
    if (ki > 127) return __fmul_rn(__fmul_rn(p, pow2i(127)), pow2i(ki - 127));
    if (ki < -126) return __fmul_rn(__fmul_rn(p, pow2i(ki + 100)), pow2i(-100));
    return __fmul_rn(p, pow2i(ki));
}

// -(SiLU(g) * u) in binary32: SiLU(g) = g / (1 + exp(-g)) (IEEE division);
// the product is negated through its operand (u -> -u), which rounding to
// nearest maps to the exact negation of SiLU(g) * u.
__device__ __forceinline__ float neg_swiglu(float g, float u) {
    const float e = hq_exp(-g);
    const float silu = __fdiv_rn(g, __fadd_rn(1.0f, e));
    return __fmul_rn(silu, -u);
}

// ------------------------------------------------------------ NVFP4 path
constexpr int NV_TILE = 128;                 // tile = 128 rows x 128 columns
#ifndef HQ_NV_CONSUMER_WARPS
#define HQ_NV_CONSUMER_WARPS 8
#define HQ_NV_STAGES 3
#define HQ_NV_CTAS_PER_SM 2
#endif
constexpr int NV_CONSUMER_WARPS = HQ_NV_CONSUMER_WARPS;  // compute warps of a CTA (divides 16)
constexpr int NV_THREADS = 32 * (NV_CONSUMER_WARPS + 1);  // + the producer warp
constexpr int NV_STAGES = HQ_NV_STAGES;                  // shared-memory tile buffers per CTA
constexpr int NV_CTAS_PER_SM = HQ_NV_CTAS_PER_SM;        // resident CTAs the kernel is built for
#ifndef HQ_NV_CLAIM
#define HQ_NV_CLAIM 2
#endif
constexpr int NV_CLAIM = HQ_NV_CLAIM;                    // consecutive tiles per scheduler claim
constexpr int NV_MAX_SEG = 2 * HQ_MAX_SECTIONS;
constexpr int NV_WS_HEADER = 4;              // counter, exit count, error, abort

// Workspace words (uint32): [0] claim counter (claims of NV_CLAIM tiles), [1] CTAs finished, [2] sticky
// error word (cleared by hq_get_error), [3] abort flag of the running call,
// then amax_row bits [S], amax_col bits [S], amax tiles finished per
// section [S] (the streaming amax kernel counts none).  All but [2] are zero
// between calls.
struct NvParams {
    CUtensorMap tmap;   // x as [M/16][16][K] BF16 blocks, 64 x 8 x 16 boxes, 128-byte swizzle
    const uint16_t* x;
    int64_t K;
    uint8_t *row_codes, *row_sf, *col_codes, *col_sf;
    float *amax_row, *amax_col, *sdec_row, *sdec_col;
    uint32_t* ws;
    int S;
    uint32_t sign_mask;
    uint32_t flags;
    uint64_t sr_seed;    // stochastic rounding: stream keys (rowwise seed, columnwise seed + 1)
    uint64_t sr_offset;  //   and the byte the streams start at (a multiple of 16)
    int col_tiles;      // K / 128
    int nseg;           // schedule segments
    uint32_t total_items;
    uint32_t multi_claims;  // claims of NV_CLAIM tiles; the claims after them take one tile each
    int finalize;       // last launch of the call: publish amax/sdec, reset ws
    int reset_counter;  // reset the tile counter / exit count at the end
    uint32_t done_per_tile;  // amax counts wanted per tile: 1 (amax tiles), 0 (after the streaming amax kernel)
    int sec_row0[HQ_MAX_SECTIONS + 1];
    uint32_t seg_start[NV_MAX_SEG + 1];
    uint16_t seg_info[NV_MAX_SEG];  // section | (phase << 15); phase 0 amax, 1 cast
};

int nvfp4_blocks_per_sm();
int nvfp4_tiles_in_flight_per_cta();  // buffers + the claims in flight
int nvfp4_tiles_per_claim();
void launch_nvfp4(const NvParams& p, int grid, cudaStream_t st);
// The section maxima alone (no row RHT), for the two-pass schedule: leaves
// the workspace as the amax launch of nvfp4_group_kernel does.
int nvfp4_amax_blocks_per_sm();
void launch_nvfp4_amax(const NvParams& p, uint32_t ntiles, int grid, cudaStream_t st);

}  // namespace hq
