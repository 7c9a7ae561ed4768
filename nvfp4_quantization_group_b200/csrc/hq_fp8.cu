// hq_fp8.cu -- FP8 E4M3 group quantizers for sm_100a.
//
//  * cat_rotate_fp8_kernel: DSA indexer prep (TensorRT-LLM PR #15158, code
//    flow "torch.cat -> rotate_activation -> fp8_quantize_1x128"): concat of
//    the pe and nope parts of each (token, head) vector, 128-point Sylvester
//    Hadamard rotation scaled by 1/sqrt(128), then one E4M3 group of 128
//    with the scale rule of onnxruntime PR #33644.
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
// One thread owns one 128-vector per tile.  A tile of 128 vectors is staged
// through shared memory twice: the BF16 inputs arrive with coalesced 16-byte
// loads (16 consecutive threads read one vector's 256 bytes) and are read
// back one vector per thread; the codes go out the same way in reverse.
// 16-byte chunk c of vector v sits at slot v * W + (c ^ (v & 7)), which keeps
// both access patterns free of shared-memory bank conflicts.
constexpr int CAT_THREADS = 128;

__global__ void __launch_bounds__(CAT_THREADS, 2) cat_rotate_fp8_kernel(CatRotateParams p) {
    __shared__ __align__(16) uint4 stage[CAT_THREADS * 16];  // 32 KB
    const int tid = threadIdx.x;
    const int a_chunks = p.a_width / 8;
    const int64_t ntiles = (p.nvec + CAT_THREADS - 1) / CAT_THREADS;
    // -1 / sqrt(128): the negated numerators feed the division directly
    const float neg_c128 = -__uint_as_float(0x3DB504F3u);

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t v0 = tile * CAT_THREADS;
        // ---- coalesced load of 128 vectors x 16 chunks
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
            const int q = it * CAT_THREADS + tid;
            const int vv = q >> 4, c = q & 15;
            const int64_t v = v0 + vv;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (v < p.nvec) {
                const int64_t t = v / p.G;
                const int g = (int)(v - t * p.G);
                const uint16_t* src = c < a_chunks
                    ? p.a + t * p.a_row_stride + (int64_t)g * p.a_width + c * 8
                    : p.b + t * p.b_row_stride + (int64_t)g * p.b_width + (c - a_chunks) * 8;
                val = ld_nc_v4(src);
            }
            stage[vv * 16 + (c ^ (vv & 7))] = val;
        }
        __syncthreads();

        // ---- own vector: BF16 -> FP32, negated (the quantizer takes -y)
        float y[128];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            uint4 w = stage[tid * 16 + (c ^ (tid & 7))];
            y[8 * c + 0] = bf16_lo(w.x); y[8 * c + 1] = bf16_hi(w.x);
            y[8 * c + 2] = bf16_lo(w.y); y[8 * c + 3] = bf16_hi(w.y);
            y[8 * c + 4] = bf16_lo(w.z); y[8 * c + 5] = bf16_hi(w.z);
            y[8 * c + 6] = bf16_lo(w.w); y[8 * c + 7] = bf16_hi(w.w);
        }
        __syncthreads();  // the staging buffer is reused for the codes

        if (p.rotate) {
            // Sylvester butterfly, stages 1, 2, ..., 64 (ascending), then
            // the orthonormal scale; stage 1 is scalar, the rest packed.
#pragma unroll
            for (int i = 0; i < 128; i += 2) {
                float a = y[i], b = y[i + 1];
                y[i] = __fadd_rn(a, b);
                y[i + 1] = __fsub_rn(a, b);
            }
            f2 v2[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) v2[i] = pack2(y[2 * i], y[2 * i + 1]);
#pragma unroll
            for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if ((i & h) == 0) {
                        f2 a = v2[i], b = v2[i + h];
                        v2[i] = add2(a, b);
                        v2[i + h] = sub2(a, b);
                    }
                }
            }
            const f2 nc2 = pack2(neg_c128, neg_c128);
#pragma unroll
            for (int i = 0; i < 64; ++i) unpack2(mul2(v2[i], nc2), y[2 * i], y[2 * i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < 128; ++i) y[i] = -y[i];
        }

        // ---- group scale and codes
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 128; i += 2) amax = absmax3(amax, y[i], y[i + 1]);
        const float s = fp8_group_scale(amax);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            f2 a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = pack2(y[16 * c + 2 * i], y[16 * c + 2 * i + 1]);
                b[i] = pack2(y[16 * c + 8 + 2 * i], y[16 * c + 8 + 2 * i + 1]);
            }
            uint2 lo = quant8(a, s), hi = quant8(b, s);
            stage[tid * 8 + (c ^ (tid & 7))] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        const int64_t v = v0 + tid;
        if (v < p.nvec) {
            if (p.scale_layout == 0) {
                p.scales[v] = s;
            } else {
                const int64_t t = v / p.G;
                const int g = (int)(v - t * p.G);
                p.scales[(int64_t)g * p.scale_ld + t] = s;
            }
        }
        __syncthreads();
        // ---- coalesced store of 128 vectors x 8 chunks of codes
        uint4* out = reinterpret_cast<uint4*>(p.out) + v0 * 8;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int q = it * CAT_THREADS + tid;
            const int vv = q >> 3, c = q & 7;
            if (v0 + vv < p.nvec) out[q] = stage[vv * 8 + (c ^ (vv & 7))];
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------ K128 quant
// A half-warp (16 lanes x 8 values) owns one group of 128; a warp works on
// two consecutive groups (adjacent in memory) per step and keeps UNROLL
// steps of loads in flight before computing.
template <int MODE>
__global__ void __launch_bounds__(K128_THREADS) k128_fp8_kernel(K128Params p) {
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, l = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * K128_THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * K128_THREADS) >> 5;
    const int64_t npairs = (p.ngroups + 1) >> 1;
    const int64_t gpr = p.K_out / 128;  // groups per row

    for (int64_t base = warp * K128_UNROLL; base < npairs; base += nwarps * K128_UNROLL) {
        f2 ny[K128_UNROLL][4];
        // ---- loads (all steps first)
#pragma unroll
        for (int u = 0; u < K128_UNROLL; ++u) {
            const int64_t g = (base + u) * 2 + half;
            if (base + u < npairs && g < p.ngroups) {
                if (MODE == HQ_ACT_NONE_BF16) {
                    const uint16_t* in = reinterpret_cast<const uint16_t*>(p.in) + g * 128 + 8 * l;
                    uint4 w = ld_nc_v4(in);
                    // negate both BF16 halves before widening: exact
                    ny[u][0] = bf16x2_to_f2(w.x ^ 0x80008000u);
                    ny[u][1] = bf16x2_to_f2(w.y ^ 0x80008000u);
                    ny[u][2] = bf16x2_to_f2(w.z ^ 0x80008000u);
                    ny[u][3] = bf16x2_to_f2(w.w ^ 0x80008000u);
                } else if (MODE == HQ_ACT_NONE_F32) {
                    const float* in = reinterpret_cast<const float*>(p.in) + g * 128;
                    uint4 w0 = ld_nc_v4(in + 4 * l), w1 = ld_nc_v4(in + 64 + 4 * l);
                    ny[u][0] = pack2(-__uint_as_float(w0.x), -__uint_as_float(w0.y));
                    ny[u][1] = pack2(-__uint_as_float(w0.z), -__uint_as_float(w0.w));
                    ny[u][2] = pack2(-__uint_as_float(w1.x), -__uint_as_float(w1.y));
                    ny[u][3] = pack2(-__uint_as_float(w1.z), -__uint_as_float(w1.w));
                } else {
                    const int64_t row = g / gpr;
                    const int64_t col = (g - row * gpr) * 128;
                    const float* gate = reinterpret_cast<const float*>(p.in) + row * 2 * p.K_out + col;
                    const float* up = gate + p.K_out;
                    uint4 g0 = ld_nc_v4(gate + 4 * l), g1 = ld_nc_v4(gate + 64 + 4 * l);
                    uint4 u0 = ld_nc_v4(up + 4 * l), u1 = ld_nc_v4(up + 64 + 4 * l);
                    const uint32_t gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                    const uint32_t uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                    float act[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        act[j] = neg_swiglu(__uint_as_float(gg[j]), __uint_as_float(uu[j]));
#pragma unroll
                    for (int j = 0; j < 4; ++j) ny[u][j] = pack2(act[2 * j], act[2 * j + 1]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) ny[u][j] = 0;
            }
        }
        // ---- per group: amax over 16 lanes, scale, codes
#pragma unroll
        for (int u = 0; u < K128_UNROLL; ++u) {
            const int64_t g = (base + u) * 2 + half;
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float a, b;
                unpack2(ny[u][j], a, b);
                m = absmax3(m, a, b);
            }
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            const float s = fp8_group_scale(m);
            if (base + u < npairs && g < p.ngroups) {
                uint2 c = quant8(ny[u], s);
                if (MODE == HQ_ACT_NONE_BF16) {
                    *reinterpret_cast<uint2*>(p.out + g * 128 + 8 * l) = c;
                } else {
                    *reinterpret_cast<uint32_t*>(p.out + g * 128 + 4 * l) = c.x;
                    *reinterpret_cast<uint32_t*>(p.out + g * 128 + 64 + 4 * l) = c.y;
                }
                if (l == 0) p.scales[g] = s;
            }
        }
    }
}

// ------------------------------------------------------------------ codec
__global__ void convert_kernel(int fmt, const float* in, uint8_t* out, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = fmt == HQ_FMT_E4M3 ? e4m3_one(in[i]) : e2m1_one(in[i]);
}

// ------------------------------------------------------------ launchers
int cat_rotate_blocks_per_sm() {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, cat_rotate_fp8_kernel, CAT_THREADS, 0);
    return n > 0 ? n : 1;
}

void launch_cat_rotate(const CatRotateParams& p, int grid, cudaStream_t st) {
    cat_rotate_fp8_kernel<<<grid, CAT_THREADS, 0, st>>>(p);
}

void launch_k128(int mode, const K128Params& p, int grid, cudaStream_t st) {
    switch (mode) {
        case HQ_ACT_NONE_BF16: k128_fp8_kernel<HQ_ACT_NONE_BF16><<<grid, K128_THREADS, 0, st>>>(p); break;
        case HQ_ACT_NONE_F32: k128_fp8_kernel<HQ_ACT_NONE_F32><<<grid, K128_THREADS, 0, st>>>(p); break;
        default: k128_fp8_kernel<HQ_ACT_SWIGLU_F32><<<grid, K128_THREADS, 0, st>>>(p); break;
    }
}

void launch_convert(int fmt, const float* in, uint8_t* out, int64_t n, int grid, cudaStream_t st) {
    convert_kernel<<<grid, 256, 0, st>>>(fmt, in, out, n);
}

}  // namespace hq
