// hq_fp8.cu -- FP8 E4M3 group quantizers for sm_100a, and the FP4 variant
// of the DSA indexer prep.
//
//  * cat_rotate_kernel<false>: DSA indexer prep (TensorRT-LLM PR #15158, code
//    flow "torch.cat -> rotate_activation -> fp8_quantize_1x128"): concat of
//    the pe and nope parts of each (token, head) vector, 128-point Sylvester
//    Hadamard rotation scaled by 1/sqrt(128), then one E4M3 group of 128
//    with the scale rule of onnxruntime PR #33644.
//  * cat_rotate_kernel<true>: the same concat and rotation, then NVFP4 per
//    vector (the FP4 path the same PR names as lacking the rotation): the
//    vector's amax gives its global encode scale, each 16-element block an
//    E4M3 scale and E2M1 codes, as in the grouped NVFP4 cast.
//  * k128_fp8_kernel: QMoE dynamic FP8 activations (onnxruntime PR #33644,
//    Description): consecutive K128 groups of BF16/FP32 rows, or of the FP32
//    SwiGLU product SiLU(gate) * up.
//  * convert_kernel: element-wise E4M3 / E2M1 codec.
//
// Both quantizers are HBM-bound streams: every input byte is read once with
// coalesced 16-byte loads and every output byte written once.
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

// ------------------------------------------------ cat -> H128 -> FP8 1x128
// Eight threads share one 128-vector, 16 elements each; a CTA of 256 threads
// takes a tile of 32 vectors.  The butterfly runs in two halves:
//  * thread j loads elements 16j..16j+15 (two 16-byte loads, from the pe or
//    the nope part) and runs stages 1, 2, 4, 8 on them; stage 1 takes the
//    BF16 pair straight from the load word (mixed-precision add / FMA, one
//    rounding each, as FP32 additions of the widened values);
//  * the 8 threads exchange values through shared memory (within the warp,
//    no CTA barrier) so that thread j then holds elements 16s + 2j and
//    16s + 2j + 1 for s = 0..7, and runs stages 16, 32, 64 on them.
// The 8 threads then reduce the amax with 3 shuffles, quantize their 16
// values, and exchange the codes through shared memory once more so that
// each writes 16 contiguous bytes.  Tiles are 32 consecutive vectors, or, for
// transposed scales, 32 consecutive rows of one group (the 32 scales are then
// contiguous).  The next tile's loads are issued before the current tile is
// computed.
constexpr int CAT_THREADS = 256;
constexpr int CAT_VEC = 32;  // vectors per tile

struct CatShared {
    float2 t[CAT_VEC][72];       // 64 pairs of one vector + 8 of padding (bank spread)
    uint32_t codes[CAT_VEC][36];  // 128 code bytes of one vector + 16 of padding
};

#ifndef HQ_CAT_TT
#define HQ_CAT_TT 8
#endif
#ifndef HQ_CAT_MINB
#define HQ_CAT_MINB 3
#endif
// Transposed scales: a tile is CAT_TT consecutive rows x CAT_TG groups, slot
// k = (k / CAT_TT) groups on, (k % CAT_TT) rows on, so each group's CAT_TT
// scales are contiguous; consecutive tiles walk the groups of a row block.
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

// Where thread j's 16 elements of every vector come from in the wide layout
// (whole segments in a or in b): the same input for all vectors, so the
// choice and its strides are made once per thread.
struct CatSrc {
    const uint16_t* base;  // element 16j of vector (0, 0)
    int64_t tstride;       // per row t
    int gwidth;            // per group g
};
__device__ __forceinline__ CatSrc cat_src(const CatRotateParams& p, int j) {
    const int a_chunks = p.a_width / 8;
    CatSrc s;
    if (2 * j < a_chunks) {
        s.base = p.a + j * 16;
        s.tstride = p.a_row_stride;
        s.gwidth = p.a_width;
    } else {
        s.base = p.b + (2 * j - a_chunks) * 8;
        s.tstride = p.b_row_stride;
        s.gwidth = p.b_width;
    }
    return s;
}

// The two 16-byte chunks (elements 16j..16j+15) of vector (t, g).
__device__ __forceinline__ void cat_load(const CatRotateParams& p, const CatSrc& src, CatVec cv, int j, uint4& c0,
                                         uint4& c1) {
    c0 = c1 = make_uint4(0u, 0u, 0u, 0u);
    if (cv.t < 0) return;
    const int64_t t = cv.t;
    const int g = cv.g;
    const int a_chunks = p.a_width / 8;
    if (p.wide) {
        ld_nc_v8(src.base + (t * src.tstride + (int64_t)g * src.gwidth), c0, c1);
        return;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = 2 * j + h;
        const uint16_t* src = c < a_chunks
            ? p.a + t * p.a_row_stride + (int64_t)g * p.a_width + c * 8
            : p.b + t * p.b_row_stride + (int64_t)g * p.b_width + (c - a_chunks) * 8;
        (h ? c1 : c0) = ld_nc_v4(src);
    }
}

template <bool FP4>
__global__ void __launch_bounds__(CAT_THREADS, HQ_CAT_MINB) cat_rotate_kernel(CatRotateParams p) {
    __shared__ CatShared sh;
    __shared__ float2 vr[FP4 ? 128 : 1];  // FP4: per E4M3 code {value, -RN(1 / value)}
    const int tid = threadIdx.x, k = tid >> 3, j = tid & 7;
    if constexpr (FP4) {
        if (tid < 128) {
            const bool z = tid == 0 || tid == 127;
            const float v = z ? 0.0f : e4m3_value((uint32_t)tid);
            vr[tid] = make_float2(v, z ? -0.0f : -__frcp_rn(v));
        }
        __syncthreads();
    }
    const float neg_c128 = -__uint_as_float(0x3DB504F3u);  // -RN(1/sqrt(128)): negated numerators
    const bf16_t minus_one = (bf16_t)0xBF80u;

    const CatVec none{-1, 0};
    uint32_t tile = blockIdx.x;
    const uint32_t ntiles = (uint32_t)p.ntiles;
    uint4 n0, n1;  // the next tile's chunks
    const CatSrc src = cat_src(p, j);
    CatVec nv = tile < ntiles ? cat_vector(p, tile, k) : none;
    cat_load(p, src, nv, j, n0, n1);
    for (; tile < ntiles; tile += gridDim.x) {
        const CatVec cv = nv;
        const uint32_t w[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
        const uint32_t nt = tile + gridDim.x;
        nv = nt < ntiles ? cat_vector(p, nt, k) : none;
        cat_load(p, src, nv, j, n0, n1);

        // ---- elements 16j..16j+15 as 8 pairs (2i, 2i+1) of this segment
        f2 y[8];
        if (p.rotate) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                bf16_t lo, hi;
                split_bf16x2(w[i], lo, hi);
                const float x0 = bf16_lo(w[i]);
                y[i] = pack2(add_bf16(hi, x0), fma_bf16(hi, minus_one, x0));  // stage 1
            }
#pragma unroll
            for (int h = 1; h < 8; h <<= 1) {  // stages 2, 4, 8
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if ((i & h) == 0) {
                        const f2 a = y[i], b = y[i + h];
                        y[i] = add2(a, b);
                        y[i + h] = sub2(a, b);
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = pack2(bf16_lo(w[i]), bf16_hi(w[i]));
        }
        // ---- exchange: thread j now takes pair j of every segment s
        // (16-byte piece c of segment s is stored at position (c + s/2) & 3 of
        // the segment's 64 bytes: the 8 lanes of a vector then hit 8
        // different bank groups when writing)
        float4* row = reinterpret_cast<float4*>(&sh.t[k][8 * j]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float a0, a1, b0, b1;
            unpack2(y[2 * c], a0, a1);
            unpack2(y[2 * c + 1], b0, b1);
            row[(c + (j >> 1)) & 3] = make_float4(a0, a1, b0, b1);
        }
        __syncwarp();
        f2 z[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const float2 e = sh.t[k][8 * s + 2 * (((j >> 1) + (s >> 1)) & 3) + (j & 1)];
            z[s] = pack2(e.x, e.y);
        }
        if (p.rotate) {
#pragma unroll
            for (int h = 1; h < 8; h <<= 1) {  // stages 16, 32, 64
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    if ((s & h) == 0) {
                        const f2 a = z[s], b = z[s + h];
                        z[s] = add2(a, b);
                        z[s + h] = sub2(a, b);
                    }
                }
            }
        }
        const f2 nc2 = pack2(p.rotate ? neg_c128 : -1.0f, p.rotate ? neg_c128 : -1.0f);
        float amax = 0.0f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            z[s] = mul2(z[s], nc2);  // -y (exact negation when not rotating)
            float a, b;
            unpack2(z[s], a, b);
            amax = absmax3(amax, a, b);
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
        if constexpr (FP4) {
            // ---- NVFP4: back to one 16-element block per thread (pair j of
            // segment s at position (j + s) & 7 of the segment: both sides
            // free of bank conflicts), then block scale and codes
            const float S = global_encode(amax);
            __syncwarp();  // the first exchange is read
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                float a, b;
                unpack2(z[s], a, b);
                sh.t[k][8 * s + ((j + s) & 7)] = make_float2(-a, -b);  // y = -z exactly
            }
            __syncwarp();
            float y[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 e = sh.t[k][8 * j + ((i + j) & 7)];
                y[2 * i] = e.x;
                y[2 * i + 1] = e.y;
            }
            const uint32_t sf = block_sf(absmax16(y), S);
            const float enc = block_enc(vr, sf, S, slow_scale(S));
            const f2 e2 = pack2(enc, enc);
            float q[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) unpack2(mul2(pack2(y[2 * i], y[2 * i + 1]), e2), q[2 * i], q[2 * i + 1]);
            if (cv.t >= 0) {
                const int64_t v = (int64_t)cv.t * p.G + cv.g;
                *reinterpret_cast<uint2*>(p.out + v * 64 + 8 * j) =
                    make_uint2(e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]),
                               e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]));
                p.sf[p.sf_swizzle ? sf_swizzled((uint64_t)cv.t, (uint64_t)cv.g * 8u + (uint64_t)j, (uint64_t)p.G * 8u)
                                  : (uint64_t)v * 8u + (uint64_t)j] = (uint8_t)sf;
                if (j == 0) {
                    const int64_t si = p.scale_layout == 0 ? v : (int64_t)cv.g * p.scale_ld + cv.t;
                    p.scales[si] = __fdiv_rn(1.0f, S);
                    if (p.amax) p.amax[si] = amax;
                }
            }
            __syncwarp();  // the exchange buffer is reused by the next tile
            continue;
        }
        const float sc = p.ue8m0 ? ue8m0_up(fp8_group_scale(amax)) : fp8_group_scale(amax);
        // ---- codes of elements 16s + 2j, 16s + 2j + 1
        uint32_t q[8];
        if (!isinf(sc)) {
            const Recip d = make_recip(sc);
            const f2 b2 = pack2(d.b, d.b), nr2 = pack2(d.nr, d.nr);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                float a, b;
                unpack2(div2_rn_neg(z[s], b2, nr2), a, b);
                q[s] = e4m3x2(a, b);
            }
        } else {  // an infinite input: plain IEEE division
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                float a, b;
                unpack2(z[s], a, b);
                q[s] = e4m3x2(__fdiv_rn(-a, sc), __fdiv_rn(-b, sc));
            }
        }
        uint16_t* cb = reinterpret_cast<uint16_t*>(sh.codes[k]);
#pragma unroll
        for (int s = 0; s < 8; ++s) cb[8 * s + j] = (uint16_t)q[s];
        __syncwarp();
        if (cv.t >= 0) {
            const int64_t v = (int64_t)cv.t * p.G + cv.g;
            const uint4 out = *reinterpret_cast<const uint4*>(&sh.codes[k][4 * j]);
            *reinterpret_cast<uint4*>(p.out + v * 128 + 16 * j) = out;
            if (j == 0) {
                const int64_t si = p.scale_layout == 0 ? v : (int64_t)cv.g * p.scale_ld + cv.t;
                p.scales[si] = sc;
                if (p.amax) p.amax[si] = amax;
            }
        }
        __syncwarp();  // the exchange buffers are reused by the next tile
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

int cat_rotate_blocks_per_sm() {
    // both variants: the grid is sized for the one with fewer resident CTAs
    int n0 = 0, n1 = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n0, cat_rotate_kernel<false>, CAT_THREADS, 0);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n1, cat_rotate_kernel<true>, CAT_THREADS, 0);
    const int n = n0 < n1 ? n0 : n1;
    return n > 0 ? n : 1;
}

void launch_cat_rotate(const CatRotateParams& p, int grid, cudaStream_t st, bool fp4) {
    if (fp4)
        cat_rotate_kernel<true><<<grid, CAT_THREADS, 0, st>>>(p);
    else
        cat_rotate_kernel<false><<<grid, CAT_THREADS, 0, st>>>(p);
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
