// hq_fp8.cu -- FP8 E4M3 group quantizers for sm_100a, and the FP4 variant
// of the DSA indexer prep.
//
//  * cat_rotate4_kernel<false>: DSA indexer prep (TensorRT-LLM PR #15158,
//    code flow "torch.cat -> rotate_activation -> fp8_quantize_1x128"):
//    concat of the pe and nope parts of each (token, head) vector, 128-point
//    Sylvester Hadamard rotation scaled by 1/sqrt(128), then one E4M3 group of
//    128 with the scale rule of onnxruntime PR #33644.
//  * cat_rotate4_kernel<true>: the same concat and rotation, then NVFP4 per
//    vector (the FP4 path the same PR names as lacking the rotation): the
//    vector's amax gives its global encode scale, each 16-element block an
//    E4M3 scale and E2M1 codes, as in the grouped NVFP4 cast.
//  * k128_fp8_kernel: QMoE dynamic FP8 activations (onnxruntime PR #33644,
//    Description): consecutive K128 groups of BF16/FP32 rows, or of the FP32
//    SwiGLU product SiLU(gate) * up.
//  * convert_kernel: element-wise E4M3 / E2M1 codec.
//
// Both quantizers stream: every input byte is read once with coalesced 16- or
// 32-byte loads and every output byte written once (the lanes of one store
// instruction cover whole 32-byte sectors, or halves of them for the FP4
// DSA codes).
#include "hq_internal.h"

namespace hq {

// ---------------------------------------------------------------- helpers
// Quantize 8 values given as negated numerators (ny = -y) with the group's
// scale: codes = E4M3(y / s), returned as two 32-bit words (element 0 in the
// low byte of word 0).
__device__ __forceinline__ uint2 quant8_neg(const f2 (&ny)[4], f2 b2, f2 nr2) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack2(div2_rn_neg(ny[i], b2, nr2), q[2 * i], q[2 * i + 1]);
    uint2 r;
    r.x = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
    r.y = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
    return r;
}

// Rare path: group scale is +inf (an infinite input); plain IEEE division.
__device__ __noinline__ uint2 quant8_slow(f2 n0, f2 n1, f2 n2, f2 n3, float s) {
    const f2 ny[4] = {n0, n1, n2, n3};
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float a, b;
        unpack2(ny[i], a, b);
        q[2 * i] = __fdiv_rn(-a, s);
        q[2 * i + 1] = __fdiv_rn(-b, s);
    }
    uint2 r;
    r.x = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
    r.y = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
    return r;
}

__device__ __forceinline__ uint2 quant8(const f2 (&ny)[4], float s) {
    if (isinf(s)) return quant8_slow(ny[0], ny[1], ny[2], ny[3], s);
    Recip d = make_recip(s);
    return quant8_neg(ny, pack2(d.b, d.b), pack2(d.nr, d.nr));
}

// ------------------------------------------- cat -> H128 -> FP8 / NVFP4: tiles
// A tile is 32 consecutive vectors, or, for transposed scales, CAT_TT
// consecutive rows x CAT_TG groups: slot k = (k / CAT_TT) groups on,
// (k % CAT_TT) rows on, so each group's CAT_TT scales are contiguous;
// consecutive tiles walk the groups of a row block.
constexpr int CAT_VEC = 32;  // vectors per tile
#ifndef HQ_CAT_TT
#define HQ_CAT_TT 8
#endif
constexpr int CAT_TT = HQ_CAT_TT, CAT_TG = CAT_VEC / CAT_TT;

// x / d and x % d for 32-bit x by multiply-high with m = floor((2^32 - 1) / d)
// and at most two corrections.
__device__ __forceinline__ uint32_t udivmod(uint32_t x, uint32_t d, uint32_t m, uint32_t& r) {
    uint32_t q = __umulhi(x, m);
    r = x - q * d;
    while (r >= d) {
        ++q;
        r -= d;
    }
    return q;
}

struct CatVec {
    int t, g;  // row and group; t < 0 past the end
};

// Row and group of slot k (0..31) of tile `tile` (host: tiles, vectors < 2^31).
__device__ __forceinline__ CatVec cat_vector(const CatRotateParams& p, uint32_t tile, int k) {
    CatVec r;
    if (p.scale_layout == 0) {
        const uint32_t v = tile * CAT_VEC + k;
        uint32_t g;
        r.t = (int)udivmod(v, (uint32_t)p.G, p.g_magic, g);
        r.g = (int)g;
        if ((int64_t)v >= p.nvec) r.t = -1;
        return r;
    }
    const uint32_t g_tiles = ((uint32_t)p.G + CAT_TG - 1) / CAT_TG;
    uint32_t gb;
    const uint32_t tb = udivmod(tile, g_tiles, p.gt_magic, gb);
    r.g = (int)(gb * CAT_TG) + k / CAT_TT;
    r.t = (int)(tb * CAT_TT) + k % CAT_TT;
    if (r.t >= p.M || r.g >= p.G) r.t = -1;
    return r;
}

// Base and strides of one thread's elements in one input.
struct CatSrc {
    const uint16_t* base;  // thread j's first element of vector (0, 0)
    int64_t tstride;       // per row t
    int gwidth;            // per group g
};

// ------------------------------------------------ cat -> H128 -> FP8 / NVFP4
// Four threads share one 128-vector, 32 elements each; a CTA of 128 threads
// takes a tile of 32 vectors.  The next tile's loads are issued before the
// current tile is computed.
//  * thread j loads elements 32j..32j+31 (two 32-byte loads when the pe/nope
//    split is a multiple of 32, else four 16-byte chunks, each from pe or
//    nope) and runs butterfly stages 1, 2, 4, 8, 16 on them; stage 1 takes
//    the BF16 pair straight from the load word (mixed-precision add / FMA,
//    one rounding each, as FP32 additions of the widened values);
//  * one exchange through shared memory (within the warp) gives thread j the
//    elements 32m + 8j .. 32m + 8j + 7 for m = 0..3, on which it runs stages
//    32 and 64;
//  * the 4 threads reduce the amax with 2 shuffles and quantize their 32
//    values; for each m the codes of elements 32m + 8j .. 32m + 8j + 7 are 8
//    contiguous output bytes (FP8), stored without a second exchange.
//  * NVFP4 (FP4): the 16-element block 2m + j/2 is split over threads j and
//    j ^ 1 (8 elements each); one shuffle gives its amax, both threads form
//    its scale and encode factor, and each stores its 4 bytes of codes.
// The stages run in ascending order.
constexpr int CAT4_THREADS = 128;
// resident CTAs the register allocation is capped for (FP8: 120 registers,
// FP4: 93; measured best of 3 to 6)
constexpr int CAT4_MINB_FP8 = 4, CAT4_MINB_FP4 = 5;

struct Cat4Shared {
    // per vector: thread m's 32 floats at float4 8m .. 8m + 7, its chunk q
    // (elements 32m + 4q .. 4q + 3) at 8m + ((q + 2m) & 7); 33 float4 per
    // vector.  A quarter-warp (2 vectors x 4 threads) then hits 8 different
    // 4-bank groups in both the writes and the reads.
    float4 t[CAT_VEC][33];
};

// Where thread j's 32 elements of every vector come from when they lie in
// one input (wide32): its base and strides, chosen once.
__device__ __forceinline__ CatSrc cat4_src(const CatRotateParams& p, int j) {
    CatSrc s;
    if (32 * j < p.a_width) {
        s.base = p.a + 32 * j;
        s.tstride = p.a_row_stride;
        s.gwidth = p.a_width;
    } else {
        s.base = p.b + (32 * j - p.a_width);
        s.tstride = p.b_row_stride;
        s.gwidth = p.b_width;
    }
    return s;
}

// Elements 32j..32j+31 of vector (t, g) as 16 BF16 pairs (zeros past the end).
__device__ __forceinline__ void cat4_load(const CatRotateParams& p, const CatSrc& src, CatVec cv, int j,
                                          uint4 (&c)[4]) {
#pragma unroll
    for (int h = 0; h < 4; ++h) c[h] = make_uint4(0u, 0u, 0u, 0u);
    if (cv.t < 0) return;
    const int64_t t = cv.t;
    const int g = cv.g;
    if (p.wide32) {
        const uint16_t* s = src.base + (t * src.tstride + (int64_t)g * src.gwidth);
        ld_nc_v8(s, c[0], c[1]);
        ld_nc_v8(s + 16, c[2], c[3]);
        return;
    }
    const int a_chunks = p.a_width / 8;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const int ch = 4 * j + h;
        const uint16_t* s = ch < a_chunks
            ? p.a + t * p.a_row_stride + (int64_t)g * p.a_width + ch * 8
            : p.b + t * p.b_row_stride + (int64_t)g * p.b_width + (ch - a_chunks) * 8;
        c[h] = ld_nc_v4(s);
    }
}

template <bool FP4>
__global__ void __launch_bounds__(CAT4_THREADS, FP4 ? CAT4_MINB_FP4 : CAT4_MINB_FP8)
    cat_rotate4_kernel(CatRotateParams p) {
    __shared__ Cat4Shared sh;
    __shared__ float2 vr[FP4 ? 128 : 1];  // FP4: per E4M3 code {value, -RN(1 / value)}
    const int tid = threadIdx.x, k = tid >> 2, j = tid & 3;
    if constexpr (FP4) {
        static_assert(CAT4_THREADS >= 128, "one thread per code");
        if (tid < 128) {
            const bool zc = tid == 0 || tid == 127;
            const float v = zc ? 0.0f : e4m3_value((uint32_t)tid);
            vr[tid] = make_float2(v, zc ? -0.0f : -__frcp_rn(v));
        }
        __syncthreads();
    }
    const float neg_c128 = -__uint_as_float(0x3DB504F3u);  // -RN(1/sqrt(128)): negated numerators
    const bf16_t minus_one = (bf16_t)0xBF80u;

    const CatVec none{-1, 0};
    uint32_t tile = blockIdx.x;
    const uint32_t ntiles = (uint32_t)p.ntiles;
    uint4 nc[4];  // the next tile's load words
    const CatSrc src = cat4_src(p, j);
    CatVec nv = tile < ntiles ? cat_vector(p, tile, k) : none;
    cat4_load(p, src, nv, j, nc);
    float4* const row = sh.t[k];
    for (; tile < ntiles; tile += gridDim.x) {
        const CatVec cv = nv;
        const uint32_t w[16] = {nc[0].x, nc[0].y, nc[0].z, nc[0].w, nc[1].x, nc[1].y, nc[1].z, nc[1].w,
                                nc[2].x, nc[2].y, nc[2].z, nc[2].w, nc[3].x, nc[3].y, nc[3].z, nc[3].w};
        const uint32_t nt = tile + gridDim.x;
        nv = nt < ntiles ? cat_vector(p, nt, k) : none;
        cat4_load(p, src, nv, j, nc);

        // ---- elements 32j + 2i, 32j + 2i + 1
        f2 y[16];
        if (p.rotate) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                bf16_t lo, hi;
                split_bf16x2(w[i], lo, hi);
                const float x0 = bf16_lo(w[i]);
                y[i] = pack2(add_bf16(hi, x0), fma_bf16(hi, minus_one, x0));  // stage 1
            }
#pragma unroll
            for (int h = 1; h < 16; h <<= 1) {  // stages 2, 4, 8, 16
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if ((i & h) == 0) {
                        const f2 a = y[i], b = y[i + h];
                        y[i] = add2(a, b);
                        y[i + h] = sub2(a, b);
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) y[i] = pack2(bf16_lo(w[i]), bf16_hi(w[i]));
        }
        // ---- exchange: thread j now takes elements 32m + 8j .. 32m + 8j + 7
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float a0, a1, b0, b1;
            unpack2(y[2 * q], a0, a1);
            unpack2(y[2 * q + 1], b0, b1);
            row[8 * j + ((q + 2 * j) & 7)] = make_float4(a0, a1, b0, b1);
        }
        __syncwarp();
        f2 z[4][4];  // z[m][l]: elements 32m + 8j + 2l, 32m + 8j + 2l + 1
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 e = row[8 * m + ((2 * j + h + 2 * m) & 7)];
                z[m][2 * h] = pack2(e.x, e.y);
                z[m][2 * h + 1] = pack2(e.z, e.w);
            }
        }
        __syncwarp();  // every read is done before the next tile's writes
        if (p.rotate) {
#pragma unroll
            for (int h = 1; h < 4; h <<= 1) {  // stages 32 (m, m + 1) and 64 (m, m + 2)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    if ((m & h) == 0) {
#pragma unroll
                        for (int l = 0; l < 4; ++l) {
                            const f2 a = z[m][l], b = z[m + h][l];
                            z[m][l] = add2(a, b);
                            z[m + h][l] = sub2(a, b);
                        }
                    }
                }
            }
        }
        const f2 nc2 = pack2(p.rotate ? neg_c128 : -1.0f, p.rotate ? neg_c128 : -1.0f);
        float amax = 0.0f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                z[m][l] = mul2(z[m][l], nc2);  // -y (exact negation when not rotating)
                float a, b;
                unpack2(z[m][l], a, b);
                amax = absmax3(amax, a, b);
            }
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        if constexpr (FP4) {
            const float S = global_encode(amax);
            const bool slow = slow_scale(S);
            uint32_t codes[4], sfs[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float yv[8];  // y = -z exactly
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                    float a, b;
                    unpack2(z[m][l], a, b);
                    yv[2 * l] = -a;
                    yv[2 * l + 1] = -b;
                }
                // the block's amax: this thread's 8 values and its partner's
                // (max is exact and skips a NaN, as over the 16 at once)
                const float a8 = max3(max3(fabsf(yv[0]), fabsf(yv[1]), fabsf(yv[2])),
                                      max3(fabsf(yv[3]), fabsf(yv[4]), fabsf(yv[5])),
                                      max3(fabsf(yv[6]), fabsf(yv[7]), 0.0f));
                const float ab = fmaxf(a8, __shfl_xor_sync(0xFFFFFFFFu, a8, 1));
                const uint32_t sf = block_sf(ab, S);
                const float enc = block_enc(vr, sf, S, slow);
                const f2 e2 = pack2(enc, enc);
                float qv[8];
#pragma unroll
                for (int l = 0; l < 4; ++l) unpack2(mul2(pack2(yv[2 * l], yv[2 * l + 1]), e2), qv[2 * l], qv[2 * l + 1]);
                codes[m] = e2m1x8(qv[0], qv[1], qv[2], qv[3], qv[4], qv[5], qv[6], qv[7]);
                sfs[m] = sf;
            }
            if (cv.t >= 0) {
                const int64_t v = (int64_t)cv.t * p.G + cv.g;
                // elements 32m + 8j .. 32m + 8j + 7: bytes 16m + 4j .. 16m + 4j + 3
                uint8_t* const o = p.out + v * 64 + 4 * j;
#pragma unroll
                for (int m = 0; m < 4; ++m) *reinterpret_cast<uint32_t*>(o + 16 * m) = codes[m];
                if ((j & 1) == 0) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint64_t blk = (uint64_t)(2 * m + (j >> 1));
                        p.sf[p.sf_swizzle ? sf_swizzled((uint64_t)cv.t, (uint64_t)cv.g * 8u + blk, (uint64_t)p.G * 8u)
                                          : (uint64_t)v * 8u + blk] = (uint8_t)sfs[m];
                    }
                }
                if (j == 0) {
                    const int64_t si = p.scale_layout == 0 ? v : (int64_t)cv.g * p.scale_ld + cv.t;
                    p.scales[si] = __fdiv_rn(1.0f, S);
                    if (p.amax) p.amax[si] = amax;
                }
            }
            continue;
        }
        const float sc = p.ue8m0 ? ue8m0_up(fp8_group_scale(amax)) : fp8_group_scale(amax);
        uint2 q[4];
        if (!isinf(sc)) {
            const Recip d = make_recip(sc);
            const f2 b2 = pack2(d.b, d.b), nr2 = pack2(d.nr, d.nr);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t c[4];
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                    float a, b;
                    unpack2(div2_rn_neg(z[m][l], b2, nr2), a, b);
                    c[l] = e4m3x2(a, b);
                }
                q[m] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
            }
        } else {  // an infinite input: plain IEEE division
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t c[4];
#pragma unroll
                for (int l = 0; l < 4; ++l) {
                    float a, b;
                    unpack2(z[m][l], a, b);
                    c[l] = e4m3x2(__fdiv_rn(-a, sc), __fdiv_rn(-b, sc));
                }
                q[m] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
            }
        }
        if (cv.t >= 0) {
            const int64_t v = (int64_t)cv.t * p.G + cv.g;
            uint8_t* const o = p.out + v * 128 + 8 * j;
#pragma unroll
            for (int m = 0; m < 4; ++m) *reinterpret_cast<uint2*>(o + 32 * m) = q[m];
            if (j == 0) {
                const int64_t si = p.scale_layout == 0 ? v : (int64_t)cv.g * p.scale_ld + cv.t;
                p.scales[si] = sc;
                if (p.amax) p.amax[si] = amax;
            }
        }
    }
}

// ------------------------------------------------------------ K128 quant
// A half-warp (16 lanes x 8 values) owns one group of 128; a warp works on
// two consecutive groups (adjacent in memory) per step.  BF16 / FP32 input:
// the raw load words of the next batch of steps are fetched before the
// current batch is computed (two register buffers), so loads stay in flight
// during the arithmetic; the same for the SwiGLU input (gate and up words).
template <int MODE> struct K128Raw;
template <> struct K128Raw<HQ_ACT_NONE_BF16> { static constexpr int U = 4; uint4 w[U]; };
template <> struct K128Raw<HQ_ACT_NONE_F32> { static constexpr int U = 2; uint4 w[U][2]; };
#ifndef HQ_K128_SWIGLU_U
#define HQ_K128_SWIGLU_U 1  // steps per buffer (2 or more: register pressure halves the occupancy, 30 % slower)
#endif
template <> struct K128Raw<HQ_ACT_SWIGLU_F32> { static constexpr int U = HQ_K128_SWIGLU_U; uint4 w[U][4]; };

// Scale, codes and the stores of one group whose negated values are ny
// (AMAX: the group's amax too).
template <bool AMAX>
__device__ __forceinline__ void k128_finish(const K128Params& p, uint32_t g, bool valid, int l, const f2 (&ny)[4],
                                            bool split_store) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        unpack2(ny[j], a, b);
        m = absmax3(m, a, b);
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const float s = p.ue8m0 ? ue8m0_up(fp8_group_scale(m)) : fp8_group_scale(m);
    if (valid) {
        const uint2 c = quant8(ny, s);
        uint8_t* out = p.out + (uint64_t)g * 128;
        if (!split_store) {
            *reinterpret_cast<uint2*>(out + 8 * l) = c;
        } else {
            *reinterpret_cast<uint32_t*>(out + 4 * l) = c.x;
            *reinterpret_cast<uint32_t*>(out + 64 + 4 * l) = c.y;
        }
        if (l == 0) {
            p.scales[g] = s;
            if (AMAX) p.amax[g] = m;
        }
    }
}

template <int MODE, bool AMAX>
__global__ void __launch_bounds__(K128_THREADS) k128_fp8_kernel(K128Params p) {
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, l = lane & 15;
    const uint32_t warp = (blockIdx.x * K128_THREADS + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * K128_THREADS) >> 5;
    const uint32_t ngroups = (uint32_t)p.ngroups;  // < 2^31 (host check)
    const uint32_t npairs = (ngroups + 1) >> 1;

    {
        using Raw = K128Raw<MODE>;
        const uint32_t gpr = (uint32_t)(p.K_out / 128);  // groups per row (SwiGLU addressing)
        constexpr int U = Raw::U;
        const uint32_t stride = nwarps * U;
        auto load = [&](uint32_t base, Raw& r) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t g = (base + u) * 2 + half;
                const bool ok = base + u < npairs && g < ngroups;
                if constexpr (MODE == HQ_ACT_NONE_BF16) {
                    r.w[u] = ok ? ld_nc_v4(reinterpret_cast<const uint16_t*>(p.in) + (uint64_t)g * 128 + 8 * l)
                                : make_uint4(0u, 0u, 0u, 0u);
                } else if constexpr (MODE == HQ_ACT_SWIGLU_F32) {
                    // gate = columns [0, K_out) of the row, up = [K_out, 2 K_out)
                    uint32_t colg;
                    const uint32_t row = udivmod(ok ? g : 0u, gpr, p.gpr_magic, colg);
                    const float* gate = reinterpret_cast<const float*>(p.in) + (uint64_t)row * 2 * p.K_out + colg * 128;
                    const float* up = gate + p.K_out;
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    r.w[u][0] = ok ? ld_nc_v4(gate + 4 * l) : z;
                    r.w[u][1] = ok ? ld_nc_v4(gate + 64 + 4 * l) : z;
                    r.w[u][2] = ok ? ld_nc_v4(up + 4 * l) : z;
                    r.w[u][3] = ok ? ld_nc_v4(up + 64 + 4 * l) : z;
                } else {
                    const float* in = reinterpret_cast<const float*>(p.in) + (uint64_t)g * 128;
                    r.w[u][0] = ok ? ld_nc_v4(in + 4 * l) : make_uint4(0u, 0u, 0u, 0u);
                    r.w[u][1] = ok ? ld_nc_v4(in + 64 + 4 * l) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
        };
        auto compute = [&](uint32_t base, const Raw& r) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t g = (base + u) * 2 + half;
                const bool ok = base + u < npairs && g < ngroups;
                f2 ny[4];
                if constexpr (MODE == HQ_ACT_NONE_BF16) {
                    // negate both BF16 halves before widening: exact
                    const uint4 w = r.w[u];
                    ny[0] = bf16x2_to_f2(w.x ^ 0x80008000u);
                    ny[1] = bf16x2_to_f2(w.y ^ 0x80008000u);
                    ny[2] = bf16x2_to_f2(w.z ^ 0x80008000u);
                    ny[3] = bf16x2_to_f2(w.w ^ 0x80008000u);
                } else if constexpr (MODE == HQ_ACT_SWIGLU_F32) {
                    const uint4 g0 = r.w[u][0], g1 = r.w[u][1], u0 = r.w[u][2], u1 = r.w[u][3];
                    const uint32_t gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                    const uint32_t uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                    float act[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) act[j] = neg_swiglu(__uint_as_float(gg[j]), __uint_as_float(uu[j]));
#pragma unroll
                    for (int j = 0; j < 4; ++j) ny[j] = pack2(act[2 * j], act[2 * j + 1]);
                } else {
                    const uint4 w0 = r.w[u][0], w1 = r.w[u][1];
                    ny[0] = pack2(-__uint_as_float(w0.x), -__uint_as_float(w0.y));
                    ny[1] = pack2(-__uint_as_float(w0.z), -__uint_as_float(w0.w));
                    ny[2] = pack2(-__uint_as_float(w1.x), -__uint_as_float(w1.y));
                    ny[3] = pack2(-__uint_as_float(w1.z), -__uint_as_float(w1.w));
                }
                k128_finish<AMAX>(p, g, ok, l, ny, MODE != HQ_ACT_NONE_BF16);
            }
        };
        Raw r0, r1;
        uint32_t base = warp * U;
        load(base, r0);
        while (base < npairs) {
            load(base + stride, r1);
            compute(base, r0);
            base += stride;
            if (base >= npairs) break;
            load(base + stride, r0);
            compute(base, r1);
            base += stride;
        }
    }
}

// ------------------------------------------------------------------ codec
__global__ void convert_kernel(int fmt, const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = fmt == HQ_FMT_E4M3 ? e4m3_one(in[i]) : e2m1_one(in[i]);
}

// Four elements per thread: their random bytes packed as in the grouped
// kernel (byte k for element k), one stochastic conversion of the four.
__global__ void convert_e2m1_sr_kernel(const float* in, const uint8_t* rnd, uint8_t* out, int64_t n) {
    const int64_t quads = (n + 3) / 4;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < quads;
         q += (int64_t)gridDim.x * blockDim.x) {
        float v[4];
        uint32_t w = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t i = 4 * q + k;
            v[k] = i < n ? in[i] : 0.0f;
            w |= (i < n ? (uint32_t)rnd[i] : 0u) << (8 * k);
        }
        const uint32_t c = e2m1x4_sr(v[0], v[1], v[2], v[3], w);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (4 * q + k < n) out[4 * q + k] = (uint8_t)((c >> (4 * k)) & 0xFu);
    }
}

// ------------------------------------------------------------ launchers
int cat_rotate_group_tiles(int G) { return (G + CAT_TG - 1) / CAT_TG; }

int64_t cat_rotate_tiles(const CatRotateParams& p) {
    return p.scale_layout == 0 ? (p.nvec + CAT_VEC - 1) / CAT_VEC
                               : ((p.G + CAT_TG - 1) / CAT_TG) * ((p.M + CAT_TT - 1) / CAT_TT);
}

int cat_rotate_blocks_per_sm(bool fp4) {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fp4 ? cat_rotate4_kernel<true> : cat_rotate4_kernel<false>,
                                                  CAT4_THREADS, 0);
    return n > 0 ? n : 1;
}

void launch_cat_rotate(const CatRotateParams& p, int grid, cudaStream_t st, bool fp4) {
    if (fp4)
        cat_rotate4_kernel<true><<<grid, CAT4_THREADS, 0, st>>>(p);
    else
        cat_rotate4_kernel<false><<<grid, CAT4_THREADS, 0, st>>>(p);
}

template <bool AMAX>
static void launch_k128_mode(int mode, const K128Params& p, int grid, cudaStream_t st) {
    switch (mode) {
        case HQ_ACT_NONE_BF16: k128_fp8_kernel<HQ_ACT_NONE_BF16, AMAX><<<grid, K128_THREADS, 0, st>>>(p); break;
        case HQ_ACT_NONE_F32: k128_fp8_kernel<HQ_ACT_NONE_F32, AMAX><<<grid, K128_THREADS, 0, st>>>(p); break;
        default: k128_fp8_kernel<HQ_ACT_SWIGLU_F32, AMAX><<<grid, K128_THREADS, 0, st>>>(p); break;
    }
}

void launch_k128(int mode, const K128Params& p, int grid, cudaStream_t st) {
    // the amax store is a separate instance: the plain kernels keep their registers
    if (p.amax)
        launch_k128_mode<true>(mode, p, grid, st);
    else
        launch_k128_mode<false>(mode, p, grid, st);
}

void launch_convert(int fmt, const float* in, uint8_t* out, int64_t n, int grid, cudaStream_t st) {
    convert_kernel<<<grid, 256, 0, st>>>(fmt, in, out, n);
}

void launch_convert_e2m1_sr(const float* in, const uint8_t* rnd, uint8_t* out, int64_t n, int grid,
                            cudaStream_t st) {
    convert_e2m1_sr_kernel<<<grid, 256, 0, st>>>(in, rnd, out, n);
}

}  // namespace hq
