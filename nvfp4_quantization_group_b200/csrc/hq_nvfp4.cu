// hq_nvfp4.cu -- grouped 16-point random Hadamard transform + NVFP4 cast
// over MoE split sections (TransformerEngine PR #2564 "[NVFP4][MOE] Bug Fix
// for NVFP4 Grouped Quant": row cast + column Hadamard transform + cast with
// scale factors, tile scheduler driven by a 4-byte caller workspace; PR #2555
// review: the RHT'd columnwise output is the transposed tensor).
//
// One persistent kernel.  Work items are 128x128 tiles; a CTA claims the
// next item from the workspace's tile counter.  Each non-empty section
// contributes an amax segment (its tiles, computing the section's rowwise
// amax and the amax of its column RHT) and a cast segment (the same tiles,
// quantized).  Segments are ordered A(s0) A(s1) C(s0) A(s2) C(s1) ... so the
// cast of a section runs one section after its amax: its rows are read a
// second time while still resident in L2, and a cast tile finds its
// section's amax complete (it waits, with a bounded spin, only if not).
// Every item depends only on items claimed before it, so the schedule cannot
// deadlock whatever number of CTAs is resident.
#include "hq_internal.h"

namespace hq {

namespace {

constexpr uint32_t SPIN_LIMIT = 1u << 20;  // polls of >= 64 ns + a load: bounded wait of ~0.1-1 s

struct NvShared {
    float enc_row[128];  // S_enc_row / value(sf) for every E4M3 code sf
    float enc_col[128];
    uint32_t red[2][NV_THREADS / 32];
    uint32_t item;
    int cur_section;     // section whose tables are loaded
    int abort;
    float senc_row, senc_col;
};

// Section encode scale: 2688 / A (6 * 448), 1 when A == 0 or not finite.
__device__ __forceinline__ float global_encode(float A) {
    float S = __fdiv_rn(2688.0f, A);
    if (A == 0.0f || !isfinite(S)) S = 1.0f;
    return S;
}

__device__ __forceinline__ uint32_t bf16x2_absmax4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    const uint32_t M = 0x7FFF7FFFu;  // |x| of both halves; magnitudes order as integers
    return __vmaxu2(__vmaxu2(a & M, b & M), __vmaxu2(c & M, d & M));
}

// E4M3 block scale of a 16-block: E4M3((a_b / 6) * S_enc); t >= 0.
__device__ __forceinline__ uint32_t block_sf(float ab, float senc) {
    return e4m3x2(__fmul_rn(div6_rn(ab), senc), 0.0f) & 0xFFu;
}

}  // namespace

__global__ void __launch_bounds__(NV_THREADS) nvfp4_group_kernel(const __grid_constant__ NvParams p) {
    __shared__ NvShared sh;
    uint32_t* const counter = p.ws;
    uint32_t* const exit_count = p.ws + 1;
    uint32_t* const err = p.ws + 2;        // sticky, read by hq_get_error
    uint32_t* const abort_flag = p.ws + 3; // this call only; cleared at exit
    uint32_t* const amax_row_ws = p.ws + NV_WS_HEADER;
    uint32_t* const amax_col_ws = amax_row_ws + p.S;
    uint32_t* const done_ws = amax_col_ws + p.S;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rg = lane >> 2;  // 16-row block of this thread inside the tile
    const int cc = lane & 3;   // 8-column chunk inside the warp's 32 columns
    const int64_t K = p.K;
    const bool do_row = p.flags & HQ_ROWWISE, do_col = p.flags & HQ_COLWISE;

    // sigma_i applied to both BF16 halves of a word by flipping sign bits
    uint32_t sg[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) sg[i] = ((p.sign_mask >> i) & 1u) ? 0x80008000u : 0u;

    if (tid == 0) {
        sh.cur_section = -1;
        sh.abort = 0;
    }
    const uint64_t keep = policy_evict_last(), drop = policy_evict_first();

    for (;;) {
        __syncthreads();
        if (tid == 0) sh.item = atomicAdd(counter, 1u);
        __syncthreads();
        const uint32_t item = sh.item;
        if (item >= p.total_items) break;

        // ---- decode: segment -> (phase, section), tile (row-tile fastest)
        int lo = 0, hi = p.nseg - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.seg_start[mid] <= item) lo = mid; else hi = mid - 1;
        }
        const uint32_t info = p.seg_info[lo];
        const int s = (int)(info & 0x7FFFu);
        const int phase = (int)(info >> 15);
        const uint32_t local = item - p.seg_start[lo];
        const int r0s = p.sec_row0[s];
        const int ms = p.sec_row0[s + 1] - r0s;
        const int trows = ms / NV_TILE;
        const int tile_r = (int)(local % (uint32_t)trows);
        const int tile_c = (int)(local / (uint32_t)trows);
        const int row_in_sec = tile_r * NV_TILE + 16 * rg;
        const int64_t row = (int64_t)r0s + row_in_sec;
        const int64_t col = (int64_t)tile_c * NV_TILE + 32 * warp + 8 * cc;

        if (phase == 1) {
            // ---- section scales (wait for the section's amax tiles if needed)
            if (tid == 0 && sh.cur_section != s) {
                const uint32_t target = (uint32_t)trows * (uint32_t)p.col_tiles;
                uint32_t spins = 0;
                while (ld_acquire(done_ws + s) < target) {
                    if (*(volatile uint32_t*)abort_flag != 0) {  // another CTA gave up already
                        sh.abort = 1;
                        break;
                    }
                    if (++spins > SPIN_LIMIT) {
                        atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                        atomicExch(abort_flag, 1u);
                        sh.abort = 1;
                        break;
                    }
                    __nanosleep(64);
                }
                const float Ar = __uint_as_float(*(volatile uint32_t*)(amax_row_ws + s));
                const float Ac = __uint_as_float(*(volatile uint32_t*)(amax_col_ws + s));
                sh.senc_row = global_encode(Ar);
                sh.senc_col = global_encode(Ac);
            }
            __syncthreads();
            if (sh.abort) continue;  // drain the remaining items without work
            if (sh.cur_section != s) {
                const float v = tid == 0 || tid == 127 ? 0.0f : e4m3_value((uint32_t)tid);
                sh.enc_row[tid] = tid == 0 || tid == 127 ? 0.0f : __fdiv_rn(sh.senc_row, v);
                sh.enc_col[tid] = tid == 0 || tid == 127 ? 0.0f : __fdiv_rn(sh.senc_col, v);
                __syncthreads();
                if (tid == 0) sh.cur_section = s;
            }
        }

        // ---- load this thread's 16 rows x 8 columns (BF16)
        uint32_t w[16][4];
        {
            const uint16_t* src = p.x + row * K + col;
            const uint64_t pol = phase == 0 ? keep : drop;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint4 v = ld_nc_v4_hint(src + i * K, pol);
                w[i][0] = v.x; w[i][1] = v.y; w[i][2] = v.z; w[i][3] = v.w;
            }
        }

        if (phase == 0) {
            // ================================================= amax pass
            uint32_t m2 = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) m2 = __vmaxu2(m2, bf16x2_absmax4(w[i][0], w[i][1], w[i][2], w[i][3]));
            uint32_t mrow = max(m2 & 0xFFFFu, m2 >> 16) << 16;  // binary32 bits of max |x|
            float mcol = 0.0f;
            if (do_col) {
#pragma unroll
                for (int kp = 0; kp < 4; ++kp) {
                    f2 v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = bf16x2_to_f2(w[i][kp] ^ sg[i]);
                    fwht16_x2(v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float a, b;
                        unpack2(v[i], a, b);
                        mcol = absmax3(mcol, a, b);
                    }
                }
                // max |0.25 y| == 0.25 max |y| exactly (rounding is monotone)
                mcol = __fmul_rn(mcol, 0.25f);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                mrow = max(mrow, __shfl_xor_sync(0xFFFFFFFFu, mrow, o));
                mcol = fmaxf(mcol, __shfl_xor_sync(0xFFFFFFFFu, mcol, o));
            }
            if (lane == 0) {
                sh.red[0][warp] = mrow;
                sh.red[1][warp] = __float_as_uint(mcol);
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t r = 0, c = 0;
#pragma unroll
                for (int k = 0; k < NV_THREADS / 32; ++k) {
                    r = max(r, sh.red[0][k]);
                    c = max(c, sh.red[1][k]);  // non-negative binary32 order as integers
                }
                if (do_row) atomicMax(amax_row_ws + s, r);
                if (do_col) atomicMax(amax_col_ws + s, c);
                __threadfence();
                red_release_add(done_ws + s, 1u);
            }
            continue;
        }

        // ===================================================== cast pass
        if (do_row) {
            const float senc = sh.senc_row;
            uint8_t* rc = p.row_codes + row * (K / 2) + col / 2;
            uint8_t* rs = p.row_sf + row * (K / 16) + col / 16;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                uint32_t m2 = bf16x2_absmax4(w[i][0], w[i][1], w[i][2], w[i][3]);
                uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));  // the block spans lanes cc, cc^1
                const uint32_t sf = block_sf(__uint_as_float(m << 16), senc);
                const float enc = sh.enc_row[sf];
                const f2 e2 = pack2(enc, enc);
                float q[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) unpack2(mul2(bf16x2_to_f2(w[i][k]), e2), q[2 * k], q[2 * k + 1]);
                *reinterpret_cast<uint32_t*>(rc + i * (K / 2)) = e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
                if ((cc & 1) == 0) rs[i * (K / 16)] = (uint8_t)sf;
            }
        }
        if (do_col) {
            const float senc = sh.senc_col;
            uint8_t* cbase = p.col_codes + K * r0s / 2 + row_in_sec / 2;
            uint8_t* sbase = p.col_sf + K * r0s / 16 + row_in_sec / 16;
            const f2 quarter = pack2(0.25f, 0.25f);
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                f2 v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = bf16x2_to_f2(w[i][kp] ^ sg[i]);
                fwht16_x2(v);
                float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    v[i] = mul2(v[i], quarter);
                    v[i + 1] = mul2(v[i + 1], quarter);
                    float x0, x1, y0, y1;
                    unpack2(v[i], x0, x1);
                    unpack2(v[i + 1], y0, y1);
                    a0 = absmax3(a0, x0, y0);
                    a1 = absmax3(a1, x1, y1);
                }
                const uint32_t sf0 = block_sf(a0, senc), sf1 = block_sf(a1, senc);
                const f2 e2 = pack2(sh.enc_col[sf0], sh.enc_col[sf1]);
                float q0[16], q1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) unpack2(mul2(v[i], e2), q0[i], q1[i]);
                const int64_t c0 = col + 2 * kp;
                uint2 o0, o1;
                o0.x = e2m1x8(q0[0], q0[1], q0[2], q0[3], q0[4], q0[5], q0[6], q0[7]);
                o0.y = e2m1x8(q0[8], q0[9], q0[10], q0[11], q0[12], q0[13], q0[14], q0[15]);
                o1.x = e2m1x8(q1[0], q1[1], q1[2], q1[3], q1[4], q1[5], q1[6], q1[7]);
                o1.y = e2m1x8(q1[8], q1[9], q1[10], q1[11], q1[12], q1[13], q1[14], q1[15]);
                *reinterpret_cast<uint2*>(cbase + c0 * (ms / 2)) = o0;
                *reinterpret_cast<uint2*>(cbase + (c0 + 1) * (ms / 2)) = o1;
                sbase[c0 * (ms / 16)] = (uint8_t)sf0;
                sbase[(c0 + 1) * (ms / 16)] = (uint8_t)sf1;
            }
        }
    }

    // ---- the last CTA to leave publishes the section scales and resets the
    // workspace to its rest state (all CTAs have made their last claim)
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        sh.item = atomicAdd(exit_count, 1u) == gridDim.x - 1 ? 1u : 0u;
    }
    __syncthreads();
    if (sh.item == 0) return;
    __threadfence();
    if (p.finalize) {
        for (int s = tid; s < p.S; s += NV_THREADS) {
            if (do_row) {
                const float A = __uint_as_float(*(volatile uint32_t*)(amax_row_ws + s));
                p.amax_row[s] = A;
                p.sdec_row[s] = __fdiv_rn(1.0f, global_encode(A));
                amax_row_ws[s] = 0;
            }
            if (do_col) {
                const float A = __uint_as_float(*(volatile uint32_t*)(amax_col_ws + s));
                p.amax_col[s] = A;
                p.sdec_col[s] = __fdiv_rn(1.0f, global_encode(A));
                amax_col_ws[s] = 0;
            }
            done_ws[s] = 0;
        }
    }
    if (tid == 0 && p.reset_counter) {
        *counter = 0;
        *exit_count = 0;
        *abort_flag = 0;
    }
}

int nvfp4_blocks_per_sm() {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4_group_kernel, NV_THREADS, 0);
    return n > 0 ? n : 1;
}

void launch_nvfp4(const NvParams& p, int grid, cudaStream_t st) {
    nvfp4_group_kernel<<<grid, NV_THREADS, 0, st>>>(p);
}

}  // namespace hq
