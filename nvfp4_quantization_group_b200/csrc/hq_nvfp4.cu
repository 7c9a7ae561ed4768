// hq_nvfp4.cu -- grouped 16-point random Hadamard transform + NVFP4 cast
// over MoE split sections (TransformerEngine PR #2564 "[NVFP4][MOE] Bug Fix
// for NVFP4 Grouped Quant": row cast + column Hadamard transform + cast with
// scale factors, tile scheduler driven by a 4-byte caller workspace; PR #2555
// review: the RHT'd columnwise output is the transposed tensor).
//
// One persistent kernel, one CTA per SM: a producer warp and 16 compute
// warps around a ring of shared-memory tile buffers (128 x 128 BF16 each).
//
//  * The producer claims 128x128 tiles from the workspace's tile counter (two
//    claims in flight) and writes a small header per buffer.  Before the
//    first cast tile of a section it waits (bounded) until the section's amax
//    is complete and fills the buffer's encode tables.  The tile itself comes
//    in with two TMA loads (the copy engine signals the bytes on the buffer's
//    "full" mbarrier): no load/store-unit traffic competes with the compute
//    warps' shared-memory reads.
//  * Compute warps wait on "full", work on the tile, and release the buffer
//    on its "empty" mbarrier.  No CTA-wide barrier in the main loop.
//
// Each non-empty section contributes an amax segment (its tiles: rowwise amax
// and amax of the column RHT) and a cast segment (the same tiles, quantized).
// A cast segment is scheduled a fixed number of tiles (the host's estimate of
// the tiles in flight) after its amax segment, so that its rows are read a
// second time while still in L2 and its amax is normally complete.  Every
// tile depends only on tiles claimed before it, and compute warps never wait
// on the producer's section wait, so the schedule cannot deadlock.
//
// Work split of a tile among the 16 compute warps (w) and their lanes (l):
//  * rowwise: warp w owns rows 8w..8w+7; lane l takes row 8w + l/8 (+4) and
//    16-column block l%8: two 16-byte shared loads (lanes of blocks 4..7
//    load their odd chunk first), no cross-lane traffic.
//  * columnwise: warp w owns columns 8w..8w+7 (4 BF16 pairs); lane l takes
//    pair 4w + l/8 and 16-row block l%8: 16 four-byte shared loads, the
//    16-point transform of two columns in packed FP32, and two 8-byte
//    stores; the 8 lanes of a pair write 64 contiguous bytes of the
//    transposed output.
// Shared layout of a buffer: the tensor map views x as [M/16][16][K] (16-row
// block, row in block, column) and a TMA box holds 64 columns x 8 blocks x 16
// rows, stored row-in-block major: tile row 16 rb + i of column half h sits
// at h * 16384 + (8 i + rb) * 128, its 16-byte chunk q at position q ^ rb
// (the 128-byte swizzle XORs with the 128-byte row index mod 8, which is rb).
// Both access patterns are then free of bank conflicts.
#include "hq_internal.h"

namespace hq {

namespace {

constexpr uint32_t SPIN_LIMIT = 1u << 20;  // section polls of >= 64 ns + a load: ~0.1-1 s
constexpr uint32_t MBAR_LIMIT = 1u << 22;  // barrier polls: far above the section wait
constexpr int NCW = NV_CONSUMER_WARPS;
constexpr int NST = NV_STAGES;
constexpr int TILE_BYTES = NV_TILE * NV_TILE * 2;

constexpr uint32_t H_VALID = 1u, H_CAST = 2u, H_GAVE_UP = 4u, H_FOLD = 8u;

struct StageHdr {
    int64_t row0;      // first global row of the tile
    int32_t col0;      // first column
    int32_t s;         // section
    int32_t r0s;       // first global row of the section
    int32_t ms;        // rows of the section
    int32_t row_in_sec0;  // tile's first row inside the section
    uint32_t flags;    // H_*
    float senc_r, senc_c;  // section encode scales (cast tiles)
    int32_t pad;
};

struct NvShared {
    float enc_row[NST][128];  // S_enc_row / value(sf) for every E4M3 code sf
    float enc_col[NST][128];  // S_enc_col / value(sf), times 0.25 when folded
    StageHdr hdr[NST];
    uint32_t acc_row[NST], acc_col[NST], acc_cnt[NST];  // amax tiles: CTA partial maxima
    int32_t tab_section[NST];  // section whose tables the buffer holds (producer only)
    uint32_t seg_start[NV_MAX_SEG + 1];  // copies of the schedule (parameter space is slow
    uint16_t seg_info[NV_MAX_SEG];       //   to index dynamically)
    int32_t sec_row0[HQ_MAX_SECTIONS + 1];
    uint64_t full[NST], empty[NST];
    uint32_t last;  // this CTA is the last to leave
};
// + 1 KB: the buffers start at the first 1024-byte boundary (the 128-byte
// swizzle pattern is defined on 1024-byte aligned addresses)
constexpr int NV_DYN_SMEM = NST * TILE_BYTES + (int)sizeof(NvShared) + 1024;

// Section encode scale: 2688 / A (6 * 448), 1 when A == 0 or not finite.
__device__ __forceinline__ float global_encode(float A) {
    float S = __fdiv_rn(2688.0f, A);
    if (A == 0.0f || !isfinite(S)) S = 1.0f;
    return S;
}

// E4M3 block scale of a 16-block: E4M3((a_b / 6) * S_enc); t >= 0.
__device__ __forceinline__ uint32_t block_sf(float ab, float senc) {
    return e4m3x2(__fmul_rn(div6_rn(ab), senc), 0.0f) & 0xFFu;
}

__device__ __forceinline__ uint32_t hmax_abs(uint32_t a, uint32_t b) {
    uint32_t m;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    return m;
}

// binary32 bits of the larger magnitude of the two BF16 halves of m (which
// holds magnitudes with arbitrary sign bits)
__device__ __forceinline__ uint32_t halves_max_bits(uint32_t m) {
    m &= 0x7FFF7FFFu;  // magnitudes order as integers
    return max(m & 0xFFFFu, m >> 16) << 16;
}

// Stage 1 of the column butterfly with the random signs folded in, straight
// from BF16: for rows i (even) and i + 1 of two columns (words wi, wj),
//   b = sigma_{i+1} x_{i+1} (exact), out_i = sigma_i x_i + b, out_{i+1} = sigma_i x_i - b,
// each an FMA with BF16 operands (widened exactly, one rounding): the same
// roundings as adding the signed FP32 values.  The -0.0 addend keeps the
// sign of a zero product.
__device__ __forceinline__ void rht_stage1(uint32_t wi, uint32_t wj, bf16_t si, bf16_t sj, f2& oi, f2& oj) {
    bf16_t xi0, xi1, xj0, xj1;
    split_bf16x2(wi, xi0, xi1);
    split_bf16x2(wj, xj0, xj1);
    const float b0 = fma_bf16(xj0, sj, -0.0f), b1 = fma_bf16(xj1, sj, -0.0f);
    oi = pack2(fma_bf16(xi0, si, b0), fma_bf16(xi1, si, b1));
    oj = pack2(fma_bf16(xi0, si, -b0), fma_bf16(xi1, si, -b1));
}

// Unnormalised column RHT, H16 diag(sigma), of a BF16 column pair (16 rows):
// two columns per packed f32x2 lane; stages 1, 2, 4, 8 in ascending order.
__device__ __forceinline__ void column_rht(const uint32_t (&w)[16], const bf16_t (&sg)[16], f2 (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) rht_stage1(w[i], w[i + 1], sg[i], sg[i + 1], v[i], v[i + 1]);
#pragma unroll
    for (int h = 2; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & h) == 0) {
                const f2 a = v[i], b = v[i + h];
                v[i] = add2(a, b);
                v[i + h] = sub2(a, b);
            }
        }
    }
}

// Shared byte offset of 16-byte chunk q (0..7) of column half h of tile row
// 16 rb + i.
__device__ __forceinline__ uint32_t chunk_off(int h, int rb, int i, int q) {
    return (uint32_t)(h * 16384 + (8 * i + rb) * 128 + 16 * ((q ^ rb) & 7));
}

struct TileInfo {
    int phase, s, r0s, ms, trows, row_in_sec0;
    int64_t row0;
    int col0;
};

// Tile -> (phase, section, position).  A CTA claims tiles in increasing
// order, so the segment is found by moving the cursor `seg` forward over the
// shared copy of the segment starts (tiles run row-tile fastest inside a
// segment).
__device__ __forceinline__ TileInfo decode(const NvParams& p, const NvShared& sh, uint32_t tile, int& seg) {
    while (seg + 1 < p.nseg && sh.seg_start[seg + 1] <= tile) ++seg;
    const uint32_t info = sh.seg_info[seg];
    TileInfo t;
    t.s = (int)(info & 0x7FFFu);
    t.phase = (int)(info >> 15);
    const uint32_t local = tile - sh.seg_start[seg];
    t.r0s = sh.sec_row0[t.s];
    t.ms = sh.sec_row0[t.s + 1] - t.r0s;
    t.trows = t.ms / NV_TILE;
    t.row_in_sec0 = (int)(local % (uint32_t)t.trows) * NV_TILE;
    t.row0 = (int64_t)t.r0s + t.row_in_sec0;
    t.col0 = (int)(local / (uint32_t)t.trows) * NV_TILE;
    return t;
}

}  // namespace

namespace {

// Header (and, for a cast tile, the section wait and the encode tables) of
// buffer st for `tile`; returns the header flags.
__device__ __forceinline__ uint32_t nv_prepare(const NvParams& p, NvShared& sh, StageHdr& h, int st, uint32_t tile,
                                           int lane, int& seg, int& cached_s, uint32_t& c_fl, uint32_t& gave_up,
                                           float& c_sr, float& c_sc) {
    uint32_t* const err = p.ws + 2;
    uint32_t* const abort_flag = p.ws + 3;
    const uint32_t* const amax_row_ws = p.ws + NV_WS_HEADER;
    const uint32_t* const amax_col_ws = amax_row_ws + p.S;
    const uint32_t* const done_ws = amax_col_ws + p.S;
    {
        const TileInfo t = decode(p, sh, tile, seg);
        uint32_t fl = H_VALID;
        if (t.phase == 1) {
            fl |= H_CAST;
            if (t.s != cached_s) {
                // ---- wait (bounded) until every amax tile of the section is in
                uint32_t f = 0u;
                float sr = 1.0f, sc = 1.0f;
                if (lane == 0) {
                    const uint32_t target = (uint32_t)t.trows * (uint32_t)p.col_tiles;
                    uint32_t spins = 0;
                    uint32_t g = gave_up;
                    while (!g && ld_acquire(done_ws + t.s) < target) {
                        if (*(volatile uint32_t*)abort_flag != 0u) { g = 1u; break; }
                        if (++spins > SPIN_LIMIT) {
                            atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                            atomicExch(abort_flag, 1u);
                            g = 1u;
                            break;
                        }
                        __nanosleep(64);
                    }
                    const float Ar = __uint_as_float(*(volatile const uint32_t*)(amax_row_ws + t.s));
                    const float Ac = __uint_as_float(*(volatile const uint32_t*)(amax_col_ws + t.s));
                    sr = global_encode(Ar);
                    sc = global_encode(Ac);
                    if (g) f |= H_GAVE_UP;
                    // 0.25 folds into the column encode factor when neither 0.25 y
                    // nor 0.25 enc can leave the normal range: A in [2^-100, 2^100]
                    if (Ac >= 7.8886091e-31f && Ac <= 1.2676506e30f) f |= H_FOLD;
                }
                c_sr = __shfl_sync(0xFFFFFFFFu, sr, 0);
                c_sc = __shfl_sync(0xFFFFFFFFu, sc, 0);
                c_fl = __shfl_sync(0xFFFFFFFFu, f, 0);
                gave_up = c_fl & H_GAVE_UP;
                cached_s = t.s;
            }
            fl |= c_fl;
            if (!(fl & H_GAVE_UP) && sh.tab_section[st] != t.s) {
                // ---- this buffer's encode tables for section s (each lane
                // writes and later reads only its own tab_section copy)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int code = lane + 32 * j;
                    const bool z = code == 0 || code == 127;
                    const float v = z ? 1.0f : e4m3_value((uint32_t)code);
                    sh.enc_row[st][code] = z ? 0.0f : __fdiv_rn(c_sr, v);
                    const float ec = z ? 0.0f : __fdiv_rn(c_sc, v);
                    sh.enc_col[st][code] = (fl & H_FOLD) ? __fmul_rn(ec, 0.25f) : ec;
                }
                sh.tab_section[st] = t.s;
            }
        }
        if (lane == 0) {
            h.row0 = t.row0;
            h.col0 = t.col0;
            h.s = t.s;
            h.r0s = t.r0s;
            h.ms = t.ms;
            h.row_in_sec0 = t.row_in_sec0;
            h.flags = fl;
            h.senc_r = c_sr;
            h.senc_c = c_sc;
        }
        return fl;
    }
}

// ---------------------------------------------------------------- producer
// Returns the number of buffer fills started (the last one may be the
// end-of-work header).
__device__ __forceinline__ uint32_t nv_producer(const NvParams& p, NvShared& sh, uint32_t tiles_u32, int lane) {
    uint32_t* const counter = p.ws;
    uint32_t* const err = p.ws + 2;
    uint32_t* const abort_flag = p.ws + 3;
    const uint32_t total = p.total_items;
    int seg = 0, cached_s = -1;
    uint32_t c_fl = 0, gave_up = 0;
    float c_sr = 1.0f, c_sc = 1.0f;
    // Lane 0 keeps two claims in flight: fill k takes its tile from ca (k
    // even) or cb (k odd) and refills that register with a new claim, read
    // two fills later, so a claim's round trip overlaps two tile preparations.
    uint32_t ca = 0, cb = 0;
    if (lane == 0) {
        ca = atomicAdd(counter, 1u);
        cb = atomicAdd(counter, 1u);
    }
    uint32_t k = 0;
    // One buffer fill; false when the producer is done.
    auto fill = [&](uint32_t& claim) -> bool {
        const int st = (int)(k % NST);
        StageHdr& h = sh.hdr[st];
        if (k >= NST && !mbar_wait_bounded(&sh.empty[st], ((k / NST) - 1u) & 1u, MBAR_LIMIT)) {
            if (lane == 0) {
                atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                atomicExch(abort_flag, 1u);
            }
            return false;  // the compute warps' own bounded waits end them
        }
        const uint32_t tile = __shfl_sync(0xFFFFFFFFu, claim, 0);
        ++k;
        if (tile >= total) {  // end of work: an empty header for the compute warps
            if (lane == 0) h.flags = 0u;
            mbar_arrive(&sh.full[st]);
            return false;
        }
        if (lane == 0) claim = atomicAdd(counter, 1u);
        const uint32_t fl = nv_prepare(p, sh, h, st, tile, lane, seg, cached_s, c_fl, gave_up, c_sr, c_sc);
        if (lane == 0 && !(fl & H_GAVE_UP)) {
            const uint32_t dst = tiles_u32 + (uint32_t)st * TILE_BYTES;
            const int c1 = (int)(h.row0 / 16);
            mbar_expect_tx(&sh.full[st], (uint32_t)TILE_BYTES);
            tma_load_3d(dst, &p.tmap, h.col0, c1, 0, &sh.full[st]);
            tma_load_3d(dst + TILE_BYTES / 2, &p.tmap, h.col0 + 64, c1, 0, &sh.full[st]);
        }
        mbar_arrive(&sh.full[st]);  // every lane: releases the header and table writes
        return true;
    };
    while (fill(ca) && fill(cb)) {
    }
    return k;
}

// ------------------------------------------------------------ compute warps
__device__ __forceinline__ void nv_consumer(const NvParams& p, NvShared& sh, const uint8_t* tiles, int w,
                                            int lane) {
    uint32_t* const err = p.ws + 2;
    uint32_t* const abort_flag = p.ws + 3;
    uint32_t* const amax_row_ws = p.ws + NV_WS_HEADER;
    uint32_t* const amax_col_ws = amax_row_ws + p.S;
    uint32_t* const done_ws = amax_col_ws + p.S;
    const int64_t K = p.K;
    const bool do_row = p.flags & HQ_ROWWISE, do_col = p.flags & HQ_COLWISE;

    bf16_t sg[16];  // sigma_i as BF16 +-1
#pragma unroll
    for (int i = 0; i < 16; ++i) sg[i] = ((p.sign_mask >> i) & 1u) ? (bf16_t)0xBF80u : (bf16_t)0x3F80u;

    // rowwise: rows rr and rr + 4 (row block w / 2), 16-column block b =
    // chunks 2b, 2b + 1; blocks 4..7 load the odd chunk first (swap = 1)
    const int b = lane & 7;
    const int rr = 8 * w + (lane >> 3);
    const uint32_t swap = b >= 4 ? 1u : 0u;
    const uint32_t re = chunk_off(b >> 2, rr >> 4, rr & 15, 2 * (b & 3));      // even chunk
    const uint32_t ro = chunk_off(b >> 2, rr >> 4, rr & 15, 2 * (b & 3) + 1);  // odd chunk
    const uint32_t r1 = swap ? ro : re;
    const uint32_t roff[2] = {r1, r1 + 4u * 8u * 128u};  // row rr + 4: row in block + 4
    const uint32_t roff2 = (swap ? re : ro) - r1;         // the other chunk, relative (mod 2^32)
    // columnwise: BF16 pair 4w + jw (chunk w & 7 of half w >> 3), rows 16 rb + i
    const int rb = lane & 7, jw = lane >> 3;
    const uint32_t coff = chunk_off(w >> 3, rb, 0, w & 7) + 4u * (uint32_t)jw;
    const int cpair = 8 * w + 2 * jw;  // first of the two columns, inside the tile

    for (uint32_t k = 0;; ++k) {
        const int st = (int)(k % NST);
        if (!mbar_wait_bounded(&sh.full[st], (k / NST) & 1u, MBAR_LIMIT)) {
            if (lane == 0) {
                atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                atomicExch(abort_flag, 1u);
            }
            break;
        }
        const StageHdr h = sh.hdr[st];
        if (!(h.flags & H_VALID)) break;
        const uint8_t* T = tiles + (size_t)st * TILE_BYTES;

        if (!(h.flags & H_CAST)) {
            // ===================================================== amax tile
            uint32_t mrow = 0u;
            float mcol = 0.0f;
            if (do_row) {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint4 lo = *reinterpret_cast<const uint4*>(T + roff[kk]);  // (odd chunk if swap)
                    const uint4 hi = *reinterpret_cast<const uint4*>(T + (roff[kk] + roff2));
                    const uint32_t m = hmax_abs(hmax_abs(hmax_abs(lo.x, lo.y), hmax_abs(lo.z, lo.w)),
                                                hmax_abs(hmax_abs(hi.x, hi.y), hmax_abs(hi.z, hi.w)));
                    mrow = max(mrow, halves_max_bits(m));
                }
            }
            if (do_col) {
                uint32_t x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = *reinterpret_cast<const uint32_t*>(T + coff + 1024 * i);
                f2 v[16];
                column_rht(x, sg, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float a0, a1;
                    unpack2(v[i], a0, a1);
                    mcol = absmax3(mcol, a0, a1);
                }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                mrow = max(mrow, __shfl_xor_sync(0xFFFFFFFFu, mrow, o));
                mcol = fmaxf(mcol, __shfl_xor_sync(0xFFFFFFFFu, mcol, o));
            }
            if (lane == 0) {
                // max |0.25 y| == RN(0.25 max |y|): rounding is monotone
                atomicMax(&sh.acc_row[st], mrow);
                atomicMax(&sh.acc_col[st], __float_as_uint(__fmul_rn(mcol, 0.25f)));  // >= 0: integer order
                __threadfence_block();
                if (atomicAdd(&sh.acc_cnt[st], 1u) == (uint32_t)(NCW - 1)) {
                    // the last warp on this tile publishes the tile's maxima
                    __threadfence_block();
                    const uint32_t ar = *(volatile uint32_t*)&sh.acc_row[st];
                    const uint32_t ac = *(volatile uint32_t*)&sh.acc_col[st];
                    sh.acc_row[st] = 0u;
                    sh.acc_col[st] = 0u;
                    sh.acc_cnt[st] = 0u;
                    if (do_row) atomicMax(amax_row_ws + h.s, ar);
                    if (do_col) atomicMax(amax_col_ws + h.s, ac);
                    red_release_add(done_ws + h.s, 1u);  // release: the maxima above are visible first
                }
            }
        } else if (!(h.flags & H_GAVE_UP)) {
            // ===================================================== cast tile
            if (do_row) {
                const float* enc_tab = sh.enc_row[st];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint4 lo = *reinterpret_cast<const uint4*>(T + roff[kk]);  // (odd chunk if swap)
                    const uint4 hi = *reinterpret_cast<const uint4*>(T + (roff[kk] + roff2));
                    const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    const uint32_t m = hmax_abs(hmax_abs(hmax_abs(wd[0], wd[1]), hmax_abs(wd[2], wd[3])),
                                                hmax_abs(hmax_abs(wd[4], wd[5]), hmax_abs(wd[6], wd[7])));
                    const uint32_t sf = block_sf(__uint_as_float(halves_max_bits(m)), h.senc_r);
                    const float enc = enc_tab[sf];
                    const f2 e2 = pack2(enc, enc);
                    float q[16];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        bf16_t xl, xh;
                        split_bf16x2(wd[c], xl, xh);
                        unpack2(mul2(pack2(add_bf16(xl, -0.0f), add_bf16(xh, -0.0f)), e2), q[2 * c], q[2 * c + 1]);
                    }
                    const int64_t row = h.row0 + rr + 4 * kk;
                    const int64_t col = h.col0 + 16 * b;
                    const uint32_t c0 = e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
                    const uint32_t c1 = e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
                    *reinterpret_cast<uint2*>(p.row_codes + row * (K / 2) + col / 2) =
                        swap ? make_uint2(c1, c0) : make_uint2(c0, c1);
                    p.row_sf[row * (K / 16) + col / 16] = (uint8_t)sf;
                }
            }
            if (do_col) {
                uint32_t x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = *reinterpret_cast<const uint32_t*>(T + coff + 1024 * i);
                f2 v[16];
                column_rht(x, sg, v);
                float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    float x0, x1, y0, y1;
                    unpack2(v[i], x0, x1);
                    unpack2(v[i + 1], y0, y1);
                    a0 = absmax3(a0, x0, y0);
                    a1 = absmax3(a1, x1, y1);
                }
                const uint32_t sf0 = block_sf(__fmul_rn(a0, 0.25f), h.senc_c);
                const uint32_t sf1 = block_sf(__fmul_rn(a1, 0.25f), h.senc_c);
                const f2 e2 = pack2(sh.enc_col[st][sf0], sh.enc_col[st][sf1]);
                if (!(h.flags & H_FOLD)) {
                    const f2 quarter = pack2(0.25f, 0.25f);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], quarter);
                }
                float q0[16], q1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) unpack2(mul2(v[i], e2), q0[i], q1[i]);
                const int64_t ms = h.ms;
                const int64_t c = h.col0 + cpair;
                uint8_t* cb = p.col_codes + K * (int64_t)h.r0s / 2 + (h.row_in_sec0 + 16 * rb) / 2;
                uint8_t* sb = p.col_sf + K * (int64_t)h.r0s / 16 + (h.row_in_sec0 / 16 + rb);
                *reinterpret_cast<uint2*>(cb + c * (ms / 2)) =
                    make_uint2(e2m1x8(q0[0], q0[1], q0[2], q0[3], q0[4], q0[5], q0[6], q0[7]),
                               e2m1x8(q0[8], q0[9], q0[10], q0[11], q0[12], q0[13], q0[14], q0[15]));
                *reinterpret_cast<uint2*>(cb + (c + 1) * (ms / 2)) =
                    make_uint2(e2m1x8(q1[0], q1[1], q1[2], q1[3], q1[4], q1[5], q1[6], q1[7]),
                               e2m1x8(q1[8], q1[9], q1[10], q1[11], q1[12], q1[13], q1[14], q1[15]));
                sb[c * (ms / 16)] = (uint8_t)sf0;
                sb[(c + 1) * (ms / 16)] = (uint8_t)sf1;
            }
        }
        mbar_arrive(&sh.empty[st]);  // every compute thread: this thread is done with the buffer
    }
}

}  // namespace

__global__ void __launch_bounds__(NV_THREADS, 1) nvfp4_group_kernel(const __grid_constant__ NvParams p) {
    extern __shared__ __align__(1024) uint8_t nv_smem_raw[];
    uint8_t* const nv_smem = nv_smem_raw + ((1024u - (smem_u32(nv_smem_raw) & 1023u)) & 1023u);
    NvShared& sh = *reinterpret_cast<NvShared*>(nv_smem + NST * TILE_BYTES);
    uint32_t* const counter = p.ws;
    uint32_t* const exit_count = p.ws + 1;
    uint32_t* const abort_flag = p.ws + 3;
    uint32_t* const amax_row_ws = p.ws + NV_WS_HEADER;
    uint32_t* const amax_col_ws = amax_row_ws + p.S;
    uint32_t* const done_ws = amax_col_ws + p.S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool do_row = p.flags & HQ_ROWWISE, do_col = p.flags & HQ_COLWISE;

    if (tid == 0) {
        for (int st = 0; st < NST; ++st) {
            mbar_init(&sh.full[st], 32u);                // producer lanes (+ the TMA bytes)
            mbar_init(&sh.empty[st], 32u * NCW);         // every compute thread
            sh.acc_row[st] = 0u;
            sh.acc_col[st] = 0u;
            sh.acc_cnt[st] = 0u;
            sh.tab_section[st] = -1;
        }
        fence_mbar_init();
    }
    for (int i = tid; i <= p.nseg; i += NV_THREADS) sh.seg_start[i] = p.seg_start[i];
    for (int i = tid; i < p.nseg; i += NV_THREADS) sh.seg_info[i] = p.seg_info[i];
    for (int i = tid; i <= p.S; i += NV_THREADS) sh.sec_row0[i] = p.sec_row0[i];
    __syncthreads();
    if (warp == NCW) {
        const uint32_t fills = nv_producer(p, sh, smem_u32(nv_smem), lane);
        // No copy may still be landing when the CTA leaves: wait (bounded) for
        // the last fill of every buffer (complete already, unless a compute
        // warp gave up waiting for it).
        for (uint32_t st = 0; st < (uint32_t)NST && st < fills; ++st) {
            const uint32_t last_use = (fills - 1u - st) / NST;
            mbar_wait_bounded(&sh.full[st], last_use & 1u, MBAR_LIMIT);
        }
    } else {
        nv_consumer(p, sh, nv_smem, warp, lane);
    }

    // ---- the last CTA to leave publishes the section scales and resets the
    // workspace to its rest state (all CTAs have made their last claim)
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        sh.last = atomicAdd(exit_count, 1u) == gridDim.x - 1 ? 1u : 0u;
    }
    __syncthreads();
    if (sh.last == 0) return;
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
    cudaFuncSetAttribute(nvfp4_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, NV_DYN_SMEM);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4_group_kernel, NV_THREADS, NV_DYN_SMEM);
    return n > 0 ? n : 1;
}

int nvfp4_tiles_in_flight_per_cta() { return NST + 2; }

void launch_nvfp4(const NvParams& p, int grid, cudaStream_t st) {
    nvfp4_group_kernel<<<grid, NV_THREADS, NV_DYN_SMEM, st>>>(p);
}
}  // namespace hq
