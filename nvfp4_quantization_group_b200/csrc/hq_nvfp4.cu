// hq_nvfp4.cu -- grouped 16-point random Hadamard transform + NVFP4 cast
// over MoE split sections (TransformerEngine PR #2564 "[NVFP4][MOE] Bug Fix
// for NVFP4 Grouped Quant": row cast + column Hadamard transform + cast with
// scale factors, tile scheduler driven by a 4-byte caller workspace; PR #2555
// review: the RHT'd columnwise output is the transposed tensor).
//
// One persistent kernel, two CTAs per SM (each its own TMA stream): per CTA a
// producer warp and 8 compute warps around a ring of 3 shared-memory tile
// buffers (128 x 128 BF16 each).
//
//  * The producer claims 128x128 tiles from the workspace's tile counter (two
//    claims in flight).  As soon as a buffer is free it starts the tile's two
//    TMA loads (the copy engine signals the bytes on the buffer's "full"
//    mbarrier: no load/store-unit traffic competes with the compute warps'
//    shared-memory reads), then, while the copy runs, writes the buffer's
//    header and, before the first cast tile of a section, waits (bounded)
//    until the section's amax is complete and fills the buffer's encode
//    tables.
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
// Work split of a tile into 16 parts (w), shared out among the compute warps
// (a warp takes parts w, w + 8), and their lanes (l):
//  * rowwise: part w is rows 8w..8w+7; lane l takes row 8w + l/8 (+4) and
//    16-column block l%8: two 16-byte shared loads (lanes of blocks 4..7
//    load their odd chunk first), no cross-lane traffic.
//  * columnwise: part w is columns 8w..8w+7 (4 BF16 pairs); lane l takes
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
constexpr uint32_t MBAR_LIMIT = 1u << 22;  // barrier sleeps of <= 1 us: far above the section wait
constexpr int NCW = NV_CONSUMER_WARPS;
constexpr int NST = NV_STAGES;
constexpr int CLAIM = NV_CLAIM;  // consecutive tiles per claim
constexpr int TILE_BYTES = NV_TILE * NV_TILE * 2;

// header flags; H_SLOW_R / H_SLOW_C: the numerator of the per-block encode
// factor is outside [2^-100, 2^100], where the division takes the slow exact
// path; H_FOLD / H_FOLD_R: 0.25 is folded into the columnwise / rotated
// rowwise encode factors
constexpr uint32_t H_VALID = 1u, H_CAST = 2u, H_GAVE_UP = 4u, H_FOLD = 8u, H_SLOW_R = 16u, H_SLOW_C = 32u,
                   H_FOLD_R = 64u;

struct alignas(16) StageHdr {  // 48 bytes, moved as three 16-byte words
    int64_t row0;      // first global row of the tile
    int32_t col0;      // first column
    int32_t s;         // section
    int32_t r0s;       // first global row of the section
    int32_t ms;        // rows of the section
    int32_t row_in_sec0;  // tile's first row inside the section
    uint32_t flags;    // H_*
    float senc_r;      // section encode scale, rowwise (cast tiles)
    float senc_c;      // columnwise
    float senc_cq;     // numerator of the columnwise block encode factor: senc_c, times 0.25 when H_FOLD
    int32_t tab;       // encode-table slot of the section (cast tiles)
};

struct NvShared {
    float2 vr[128];  // per E4M3 code: {value, -RN(1 / value)}; {0, -0} for codes 0 and 127
    // Encode tables S_enc / value(sf) for every code, rowwise and columnwise,
    // in NST slots taken in turn at each change of section along the
    // producer's cast fills.  A slot is rewritten at the NST-th section change
    // after its own, NST or more fills after the last fill that used it, and
    // after the producer waited for that fill's buffer to be released.
    float enc[NST][2][128];
    int32_t tab_section[NST];  // section a slot holds (producer only)
    StageHdr hdr[NST];
    uint32_t acc_row[NST], acc_col[NST], acc_cnt[NST];  // amax tiles: CTA partial maxima
    uint32_t seg_start[NV_MAX_SEG + 1];  // copies of the schedule (parameter space is slow
    uint16_t seg_info[NV_MAX_SEG];       //   to index dynamically)
    int32_t sec_row0[HQ_MAX_SECTIONS + 1];
    uint32_t sec_magic[HQ_MAX_SECTIONS];  // floor((2^32 - 1) / row tiles of the section)
    uint64_t full[NST], empty[NST];
    uint32_t last;  // this CTA is the last to leave
};
// + 1 KB: the buffers start at the first 1024-byte boundary (the 128-byte
// swizzle pattern is defined on 1024-byte aligned addresses)
constexpr int NV_DYN_SMEM = NST * TILE_BYTES + (int)sizeof(NvShared) + 1024;

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

// Butterfly stages 2, 4, 8 of the 16-point transform, in ascending order, on
// two independent vectors (the two halves of each packed lane).
__device__ __forceinline__ void rht_stages(f2 (&v)[16]) {
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

// max over the 16 outputs of the last butterfly stage (h = 8) of |v|, both
// halves, and m, without forming the outputs: for the pair (a, b) the stage
// writes RN(a + b) and RN(a - b), and the larger magnitude of the two is
// RN(|a| + |b|) (the operation whose operands have equal signs adds the
// magnitudes; the other one's magnitude is RN(||a| - |b||), no larger, as
// rounding is monotone and symmetric).  NaN sums are skipped like NaN outputs.
__device__ __forceinline__ float last_stage_absmax(const f2 (&v)[16], float m) {
    float s[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float a0, a1, b0, b1;
        unpack2(v[i], a0, a1);
        unpack2(v[i + 8], b0, b1);
        s[2 * i] = __fadd_rn(fabsf(a0), fabsf(b0));
        s[2 * i + 1] = __fadd_rn(fabsf(a1), fabsf(b1));
    }
    const float p = max3(max3(s[0], s[1], s[2]), max3(s[3], s[4], s[5]), max3(s[6], s[7], s[8]));
    const float q = max3(max3(s[9], s[10], s[11]), max3(s[12], s[13], s[14]), max3(s[15], m, 0.0f));
    return max3(p, q, 0.0f);
}

// Butterfly stages 2 and 4 (the first three stages with stage 1).
__device__ __forceinline__ void rht_stages_24(f2 (&v)[16]) {
#pragma unroll
    for (int h = 2; h < 8; h <<= 1) {
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

// Unnormalised column RHT, H16 diag(sigma), of a BF16 column pair (16 rows):
// two columns per packed f32x2 lane; stages 1, 2, 4, 8 in ascending order.
__device__ __forceinline__ void column_rht(const uint32_t (&w)[16], const bf16_t (&sg)[16], f2 (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) rht_stage1(w[i], w[i + 1], sg[i], sg[i + 1], v[i], v[i + 1]);
    rht_stages(v);
}
// max(m, |column RHT outputs|) of a BF16 column pair: stages 1, 2, 4 and the
// last stage's maximum by last_stage_absmax.
__device__ __forceinline__ float column_rht_absmax(const uint32_t (&w)[16], const bf16_t (&sg)[16], float m) {
    f2 v[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) rht_stage1(w[i], w[i + 1], sg[i], sg[i + 1], v[i], v[i + 1]);
    rht_stages_24(v);
    return last_stage_absmax(v, m);
}

// Unnormalised RHT along K of one 16-column block of two rows a and b (word c
// holds elements 2c, 2c + 1, the even one in the low half): v[i] = {a_i, b_i}
// of the output.  Stage 1 pairs the two halves of a word, with the signs
// folded in as in rht_stage1.
__device__ __forceinline__ void row_rht_stage1(const uint32_t (&wa)[8], const uint32_t (&wb)[8],
                                               const bf16_t (&sg)[16], f2 (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        bf16_t a0, a1, b0, b1;
        split_bf16x2(wa[c], a0, a1);
        split_bf16x2(wb[c], b0, b1);
        const float pa = fma_bf16(a1, sg[2 * c + 1], -0.0f), pb = fma_bf16(b1, sg[2 * c + 1], -0.0f);
        v[2 * c] = pack2(fma_bf16(a0, sg[2 * c], pa), fma_bf16(b0, sg[2 * c], pb));
        v[2 * c + 1] = pack2(fma_bf16(a0, sg[2 * c], -pa), fma_bf16(b0, sg[2 * c], -pb));
    }
}
__device__ __forceinline__ void row_rht(const uint32_t (&wa)[8], const uint32_t (&wb)[8], const bf16_t (&sg)[16],
                                        f2 (&v)[16]) {
    row_rht_stage1(wa, wb, sg, v);
    rht_stages(v);
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
    // local = q * trows + r by multiply-high and at most two corrections
    uint32_t q = __umulhi(local, sh.sec_magic[t.s]);
    uint32_t r = local - q * (uint32_t)t.trows;
    while (r >= (uint32_t)t.trows) {
        ++q;
        r -= (uint32_t)t.trows;
    }
    t.row_in_sec0 = (int)r * NV_TILE;
    t.row0 = (int64_t)t.r0s + t.row_in_sec0;
    t.col0 = (int)q * NV_TILE;
    return t;
}

// decode() of tile = (the tile `prev` describes) + 1, with the cursor where
// decode() left it for prev: inside the same segment the next row tile, or
// the first row tile of the next column tile.
__device__ __forceinline__ TileInfo decode_successor(const NvParams& p, const NvShared& sh, const TileInfo& prev,
                                                     uint32_t tile, int& seg) {
    if (seg + 1 < p.nseg && sh.seg_start[seg + 1] <= tile) return decode(p, sh, tile, seg);
    TileInfo t = prev;
    if (t.row_in_sec0 + NV_TILE < t.ms) {
        t.row_in_sec0 += NV_TILE;
        t.row0 += NV_TILE;
    } else {
        t.row_in_sec0 = 0;
        t.row0 = t.r0s;
        t.col0 += NV_TILE;
    }
    return t;
}

}  // namespace

namespace {

// ------------------------------------------------------ section completion
// Compute warps publish an amax tile with reductions that return nothing (the
// tile's maxima, then a release increment of the section's tile count), so
// no compute warp waits on a global round trip.  The producer, about to fill
// a buffer with the section's first cast tile, waits (bounded) until the
// count reaches the section's amax tiles, then reads the maxima after an
// acquire fence and derives the section record: low word senc_r, high word
// senc_c | fold << 31.
__device__ __forceinline__ uint64_t make_record(float Ar, float Ac) {
    // 0.25 folds into the column encode factor when neither 0.25 y nor
    // 0.25 enc can leave the normal range: A in [2^-100, 2^100]
    const uint32_t fold = (Ac >= 7.8886091e-31f && Ac <= 1.2676506e30f) ? 1u : 0u;
    return (uint64_t)__float_as_uint(global_encode(Ar)) |
           ((uint64_t)(__float_as_uint(global_encode(Ac)) | (fold << 31)) << 32);
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* q) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(q) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* q) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(q) : "memory");
    return v;
}
// with a relaxed load before it that saw the final count: an acquire pattern
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void red_max_u32(uint32_t* q, uint32_t v) {
    asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" :: "l"(q), "r"(v) : "memory");
}
// orders this thread's earlier writes and reductions (the maxima) before it
__device__ __forceinline__ void red_release_add_u32(uint32_t* q, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(q), "r"(v) : "memory");
}

// ---------------------------------------------------------------- producer
// Producer state that persists across buffer fills.
struct ProducerState {
    int seg = 0;                // schedule cursor
    int ready_s = -1;           // section whose record is held below
    uint32_t r_fl = 0;          // its header flags (H_FOLD, H_SLOW_*, H_GAVE_UP)
    float r_sr = 1.0f, r_srq = 1.0f, r_sc = 1.0f, r_scq = 1.0f;
    uint32_t gave_up = 0;       // sticky once a section wait gave up
    // Prefetched one fill ahead for the next tile's section (lane 0): its
    // amax tile count (an acquire load) and, after it, its maxima (final when
    // the count is complete), or the caller's amax.
    int pf_s = -1;
    uint32_t pf = 0;
    float pf_ar = 0.0f, pf_ac = 0.0f;
    int tab = 0, tab_s = -1;    // encode-table slot in use and its section
    TileInfo nt;                // the next fill's tile, decoded one fill ahead
};

// Header of buffer st for `tile` (and, for a cast tile, the section wait);
// returns the header flags.
__device__ __forceinline__ uint32_t nv_prepare(const NvParams& p, StageHdr& h, const TileInfo& t, int lane,
                                               ProducerState& ps) {
    uint32_t* const err = p.ws + 2;
    uint32_t* const abort_flag = p.ws + 3;
    uint32_t fl = H_VALID;
    if (t.phase == 1) {
        fl |= H_CAST;
        if (t.s != ps.ready_s) {
            // ---- the section's scales: from the caller's amax, or once the
            // section's amax tiles are all counted (the count is prefetched
            // one fill ahead and normally complete; else wait, bounded)
            uint32_t f = 0u;
            float sr = 1.0f, srq = 1.0f, sc = 1.0f, scq = 1.0f;
            if (lane == 0) {
                uint64_t rec = 0u;
                uint32_t g = ps.gave_up;
                if (p.flags & HQ_AMAX_GIVEN) {
                    const bool pre = ps.pf_s == t.s;  // prefetched with the tile
                    rec = make_record((p.flags & HQ_ROWWISE) ? (pre ? ps.pf_ar : p.amax_row[t.s]) : 0.0f,
                                      (p.flags & HQ_COLWISE) ? (pre ? ps.pf_ac : p.amax_col[t.s]) : 0.0f);
                } else if (!g) {
                    const uint32_t* const done = p.ws + NV_WS_HEADER + 2 * p.S + t.s;
                    const uint32_t target = (uint32_t)(t.ms / NV_TILE) * (uint32_t)p.col_tiles * p.done_per_tile;
                    uint32_t d = ps.pf_s == t.s ? ps.pf : ld_relaxed_u32(done);
                    const bool pf_final = ps.pf_s == t.s && d >= target;  // the prefetched maxima are final
                    uint32_t spins = 0;
                    while (!g && d < target) {
                        if (*(volatile uint32_t*)abort_flag != 0u) {
                            g = 1u;
                        } else if (++spins > SPIN_LIMIT) {
                            atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                            atomicExch(abort_flag, 1u);
                            g = 1u;
                        } else {
                            __nanosleep(64);
                            d = ld_relaxed_u32(done);
                        }
                    }
                    if (pf_final) {
                        rec = make_record(ps.pf_ar, ps.pf_ac);
                    } else if (!g) {
                        fence_acq_rel_gpu();  // every counted tile's maxima are visible now
                        rec = make_record(__uint_as_float(ld_relaxed_u32(p.ws + NV_WS_HEADER + t.s)),
                                          __uint_as_float(ld_relaxed_u32(p.ws + NV_WS_HEADER + p.S + t.s)));
                    }
                }
                if (g) {
                    f |= H_GAVE_UP;
                } else {
                    sr = __uint_as_float((uint32_t)rec);
                    sc = __uint_as_float((uint32_t)(rec >> 32) & 0x7FFFFFFFu);
                    scq = sc;
                    srq = sr;
                    if (rec >> 63) {
                        f |= H_FOLD;
                        scq = __fmul_rn(sc, 0.25f);  // exact: sc is in [2^-89, 2^111]
                    }
                    // rotated rows: sr in [2^-88, 2^111] implies (sr = RN(2688 /
                    // A) is monotone) A in [2^-100, 2^100], the range in which
                    // the fold is exact; sr = 1 (A zero or not finite) folds
                    // exactly as well
                    if ((p.flags & HQ_ROW_RHT) && sr >= 0x1p-88f && sr <= 0x1p111f) {
                        f |= H_FOLD_R;
                        srq = __fmul_rn(sr, 0.25f);
                    }
                    if (slow_scale(srq)) f |= H_SLOW_R;
                    if (slow_scale(scq)) f |= H_SLOW_C;
                }
            }
            ps.r_sr = __shfl_sync(0xFFFFFFFFu, sr, 0);
            ps.r_srq = __shfl_sync(0xFFFFFFFFu, srq, 0);
            ps.r_sc = __shfl_sync(0xFFFFFFFFu, sc, 0);
            ps.r_scq = __shfl_sync(0xFFFFFFFFu, scq, 0);
            ps.r_fl = __shfl_sync(0xFFFFFFFFu, f, 0);
            ps.gave_up = ps.r_fl & H_GAVE_UP;
            ps.ready_s = t.s;
        }
        fl |= ps.r_fl;
    }
    if (lane == 0) {
        StageHdr v;
        v.row0 = t.row0;
        v.col0 = t.col0;
        v.s = t.s;
        v.r0s = t.r0s;
        v.ms = t.ms;
        v.row_in_sec0 = t.row_in_sec0;
        v.flags = fl;
        v.senc_r = ps.r_sr;
        v.senc_c = ps.r_sc;
        v.senc_cq = ps.r_scq;
        v.tab = ps.tab;
        const uint4* src = reinterpret_cast<const uint4*>(&v);
        uint4* dst = reinterpret_cast<uint4*>(&h);
        dst[0] = src[0];
        dst[1] = src[1];
        dst[2] = src[2];
    }
    return fl;
}

// Returns the number of buffer fills started (the last one may be the
// end-of-work header).
__device__ __forceinline__ uint32_t nv_producer(const NvParams& p, NvShared& sh, uint32_t tiles_u32, int lane) {
    uint32_t* const counter = p.ws;
    uint32_t* const err = p.ws + 2;
    uint32_t* const abort_flag = p.ws + 3;
    const uint32_t total = p.total_items;
    ProducerState ps;
    // A claim is CLAIM consecutive tiles (the counter counts claims): one
    // atomic per CLAIM fills, and consecutive tiles nearly always share their
    // section, so the section state is looked up less often.  The last tiles
    // (about two per CTA; host's choice) go one per claim, for an even tail.  Lane 0 keeps two
    // claims in flight in ca, cb: the tiles of ca are filled while its
    // register is refilled with a new claim (read two claims later), and cb,
    // claimed one claim earlier, gives the tile after the last one (to
    // prefetch its section's amax tile count).  (More claims in flight
    // measured slower: tiles are reserved longer before they are worked on,
    // so sections complete later and the tail is longer.)
    // first tile of a claim
    auto claim_first = [&](uint32_t c) -> uint32_t {
        return c < p.multi_claims ? c * (uint32_t)CLAIM : c + p.multi_claims * (uint32_t)(CLAIM - 1);
    };
    uint32_t ca = 0, cb = 0;
    if (lane == 0) {
        ca = atomicAdd(counter, 1u);
        cb = atomicAdd(counter, 1u);
    }
    uint32_t k = 0;
    // Waits (bounded) until the buffer of fill k is free; false on timeout.
    auto wait_free = [&](int st) -> bool {
        if (k >= NST && !mbar_wait_bounded(&sh.empty[st], ((k / NST) - 1u) & 1u, MBAR_LIMIT)) {
            if (lane == 0) {
                atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                atomicExch(abort_flag, 1u);
            }
            return false;  // the compute warps' own bounded waits end them
        }
        return true;
    };
    // One buffer fill with `tile` (< total).  The following fill's tile is
    // `next`, or (last tile of a claim) the first tile of claim cb.
    auto fill = [&](uint32_t tile, uint32_t next, bool next_from_cb) -> bool {
        const int st = (int)(k % NST);
        StageHdr& h = sh.hdr[st];
        if (!wait_free(st)) return false;
        ++k;
        const TileInfo t = k == 1u ? decode(p, sh, tile, ps.seg) : ps.nt;
        if (lane == 0) {
            // the data first: the header work below overlaps the copy
            const uint32_t dst = tiles_u32 + (uint32_t)st * TILE_BYTES;
            const int c1 = (int)(t.row0 / 16);
            mbar_expect_tx(&sh.full[st], (uint32_t)TILE_BYTES);
            tma_load_3d(dst, &p.tmap, t.col0, c1, 0, &sh.full[st]);
            tma_load_3d(dst + TILE_BYTES / 2, &p.tmap, t.col0 + 64, c1, 0, &sh.full[st]);
        }
        if (t.phase == 1 && t.s != ps.tab_s) {
            ps.tab = ps.tab + 1 == NST ? 0 : ps.tab + 1;  // a new section: the next table slot
            ps.tab_s = t.s;
        }
        const uint32_t fl = nv_prepare(p, h, t, lane, ps);
        if ((fl & H_CAST) && !(fl & H_GAVE_UP) && sh.tab_section[ps.tab] != t.s) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t code = (uint32_t)lane + 32u * m;
                sh.enc[ps.tab][0][code] = block_enc(sh.vr, code, ps.r_srq, fl & H_SLOW_R);
                sh.enc[ps.tab][1][code] = block_enc(sh.vr, code, ps.r_scq, fl & H_SLOW_C);
            }
            sh.tab_section[ps.tab] = t.s;  // (each lane reads back only its own write)
        }
        mbar_arrive(&sh.full[st]);  // every lane: releases the header writes
        // ---- decode the next fill's tile; prefetch its section's amax tile count
        const uint32_t nt = next_from_cb ? claim_first(__shfl_sync(0xFFFFFFFFu, cb, 0)) : next;
        if (nt < total) {
            ps.nt = next_from_cb ? decode(p, sh, nt, ps.seg) : decode_successor(p, sh, t, nt, ps.seg);
            if (lane == 0 && ps.nt.phase == 1 && ps.nt.s != ps.ready_s && ps.nt.s != ps.pf_s) {
                if (p.flags & HQ_AMAX_GIVEN) {
                    ps.pf_ar = (p.flags & HQ_ROWWISE) ? p.amax_row[ps.nt.s] : 0.0f;
                    ps.pf_ac = (p.flags & HQ_COLWISE) ? p.amax_col[ps.nt.s] : 0.0f;
                } else {
                    // the acquire orders the maxima loads after the count
                    ps.pf = ld_acquire_u32(p.ws + NV_WS_HEADER + 2 * p.S + ps.nt.s);
                    ps.pf_ar = __uint_as_float(ld_relaxed_u32(p.ws + NV_WS_HEADER + ps.nt.s));
                    ps.pf_ac = __uint_as_float(ld_relaxed_u32(p.ws + NV_WS_HEADER + p.S + ps.nt.s));
                }
                ps.pf_s = ps.nt.s;
            }
        }
        return true;
    };
    for (;;) {
        const uint32_t claim = __shfl_sync(0xFFFFFFFFu, ca, 0);
        const uint32_t first = claim_first(claim);
        const uint32_t count = claim < p.multi_claims ? (uint32_t)CLAIM : 1u;
        if (first >= total) {
            // end of work: an empty header for the compute warps
            const int st = (int)(k % NST);
            if (wait_free(st)) {
                if (lane == 0) sh.hdr[st].flags = 0u;
                mbar_arrive(&sh.full[st]);
                ++k;
            }
            break;
        }
        if (lane == 0) ca = atomicAdd(counter, 1u);  // read two claims later
        bool ok = true;
#pragma unroll 1
        for (uint32_t j = 0; j < count && ok && first + j < total; ++j) {
            const bool last = j + 1 == count || first + j + 1 >= total;
            ok = fill(first + j, first + j + 1, last);
        }
        if (!ok) break;
        const uint32_t c = ca;  // lane 0: the claim after cb
        ca = cb;
        cb = c;
    }
    return k;
}

// ------------------------------------------------------------ compute warps
// RowRht: the rowwise blocks are rotated along K before their amax and cast.
// SR: the codes of the directions HQ_ROW_SR / HQ_COL_SR select round
// stochastically (one Philox block per 16-element block).
template <bool RowRht, bool SR, bool Swz>
__device__ __forceinline__ void nv_consumer(const NvParams& p, NvShared& sh, const uint8_t* tiles, int w,
                                            int lane) {
    uint32_t* const err = p.ws + 2;
    uint32_t* const abort_flag = p.ws + 3;
    uint32_t* const amax_row_ws = p.ws + NV_WS_HEADER;
    uint32_t* const amax_col_ws = amax_row_ws + p.S;
    uint32_t* const done_ws = amax_col_ws + p.S;
    const bool do_row = p.flags & HQ_ROWWISE, do_col = p.flags & HQ_COLWISE;
    const bool sr_row = SR && (p.flags & HQ_ROW_SR), sr_col = SR && (p.flags & HQ_COL_SR);

    const uint8_t* T_cur = tiles;  // the buffer being worked on
    bf16_t sg[16];  // sigma_i as BF16 +-1
#pragma unroll
    for (int i = 0; i < 16; ++i) sg[i] = ((p.sign_mask >> i) & 1u) ? (bf16_t)0xBF80u : (bf16_t)0x3F80u;

    const int b = lane & 7;                  // rowwise 16-column block
    const int rb = lane & 7, jw = lane >> 3;  // columnwise 16-row block, BF16 pair in the chunk
    const uint32_t swap = b >= 4 ? 1u : 0u;  // blocks 4..7 load their odd chunk first
    const uint64_t K2 = (uint64_t)p.K / 2, K16 = (uint64_t)p.K / 16;
    // The 16 parts of a tile (see the header) are shared out among the NCW
    // compute warps: warp w takes parts w, w + NCW, ...  Per part, this lane's
    // shared offsets and output offsets:
    struct Part {
        uint32_t roff0;    // rowwise: first chunk of row rr (row rr + 4: + 4096)
        uint32_t roff2;    //   the other chunk, relative (mod 2^32)
        uint32_t coff;     // columnwise: pair 4 vw + jw, row 16 rb
        int cpair;         //   first of its two columns, inside the tile
        uint64_t rs_off0;  // row rr's block-scale offset (+ 4 K16 for rr + 4; codes at 8x)
        uint32_t rs_swz;   // the same inside the tile's 1 KB of interleaved row scales (+ 64 for rr + 4)
        uint32_t cs_swz;   // column cpair's scale of row block rb inside the tile's 1 KB of
                           //   interleaved column scales (+ 16 for cpair + 1)
    };
    // This lane's two rows (rr, rr + 4) of part pt in element order: lanes with
    // `swap` loaded the odd chunk first.
    auto load_row_pair = [&](const Part& pt, uint32_t (&wa)[8], uint32_t (&wb)[8]) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const uint32_t ro = pt.roff0 + 4096u * kk;
            const uint4 lo = *reinterpret_cast<const uint4*>(T_cur + ro);
            const uint4 hi = *reinterpret_cast<const uint4*>(T_cur + (ro + pt.roff2));
            const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) (kk ? wb : wa)[c] = swap ? wd[c ^ 4] : wd[c];
        }
    };
    auto part = [&](int vw) {
        Part q;
        const int rr = 8 * vw + (lane >> 3);  // rows rr, rr + 4 in row block vw / 2
        const uint32_t re = chunk_off(b >> 2, rr >> 4, rr & 15, 2 * (b & 3));      // even chunk
        const uint32_t ro = chunk_off(b >> 2, rr >> 4, rr & 15, 2 * (b & 3) + 1);  // odd chunk
        q.roff0 = swap ? ro : re;
        q.roff2 = (swap ? re : ro) - q.roff0;
        q.coff = chunk_off(vw >> 3, rb, 0, vw & 7) + 4u * (uint32_t)jw;  // chunk vw & 7 of half vw >> 3
        q.cpair = 8 * vw + 2 * jw;
        q.rs_off0 = (uint64_t)rr * K16 + b;
        // interleaved tiles: a 128-row x 128-column tile of x owns two whole
        // 128 x 4 scale tiles per direction (1 KB); rr + 4 and cpair + 1 stay
        // in the same 32-row line group
        q.rs_swz = (uint32_t)((b >> 2) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (b & 3));
        q.cs_swz = (uint32_t)((rb >> 2) * 512 + (q.cpair & 31) * 16 + (q.cpair >> 5) * 4 + (rb & 3));
        return q;
    };
    Part parts[16 / NCW];  // the same for every tile
#pragma unroll
    for (int pi = 0; pi < 16 / NCW; ++pi) parts[pi] = part(w + pi * NCW);

    for (uint32_t k = 0;; ++k) {
        const int st = (int)(k % NST);
        if (!mbar_wait_bounded(&sh.full[st], (k / NST) & 1u, MBAR_LIMIT)) {
            if (lane == 0) {
                atomicOr(err, (uint32_t)HQ_ERR_TIMEOUT);
                atomicExch(abort_flag, 1u);
            }
            break;
        }
        StageHdr h;
        {
            const uint4* src = reinterpret_cast<const uint4*>(&sh.hdr[st]);
            uint4* dst = reinterpret_cast<uint4*>(&h);
            dst[0] = src[0];
            dst[1] = src[1];
            dst[2] = src[2];
        }
        if (!(h.flags & H_VALID)) break;
        const uint8_t* T = tiles + (size_t)st * TILE_BYTES;
        T_cur = T;

        if (!(h.flags & H_CAST)) {
            // ===================================================== amax tile
            uint32_t mrow = 0u, mrow2 = 0u;  // mrow2: BF16 pair of running magnitude maxima
            float mrf = 0.0f, mcol = 0.0f;
#pragma unroll
            for (int pi = 0; pi < 16 / NCW; ++pi) {
            const Part& pt = parts[pi];
            if (do_row && RowRht) {
                uint32_t wa[8], wb[8];
                load_row_pair(pt, wa, wb);
                f2 v[16];
                row_rht_stage1(wa, wb, sg, v);
                rht_stages_24(v);
                mrf = last_stage_absmax(v, mrf);
            } else if (do_row) {
                // rows rr and rr + 4 into the running pair (a NaN is skipped:
                // the maximum returns the other operand, and the running pair
                // starts at zero)
                uint32_t m[2];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint32_t ro = pt.roff0 + 4096u * kk;
                    const uint4 lo = *reinterpret_cast<const uint4*>(T + ro);  // (odd chunk if swap)
                    const uint4 hi = *reinterpret_cast<const uint4*>(T + (ro + pt.roff2));
                    m[kk] = hmax_abs(hmax_abs(hmax_abs(lo.x, lo.y), hmax_abs(lo.z, lo.w)),
                                     hmax_abs(hmax_abs(hi.x, hi.y), hmax_abs(hi.z, hi.w)));
                }
                mrow2 = hmax_abs(mrow2, hmax_abs(m[0], m[1]));
            }
            if (do_col) {
                uint32_t x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = *reinterpret_cast<const uint32_t*>(T + pt.coff + 1024 * i);
                mcol = column_rht_absmax(x, sg, mcol);
            }
            }  // parts
            // rotated rows: the maximum of |0.25 y| as binary32 bits (>= 0:
            // integer order)
            mrow = RowRht ? __float_as_uint(__fmul_rn(mrf, 0.25f)) : halves_max_bits(mrow2);
            // (both non-negative and not NaN: binary32 bits order as integers)
            mrow = __reduce_max_sync(0xFFFFFFFFu, mrow);
            mcol = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mcol)));
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
                    if (do_row) red_max_u32(amax_row_ws + h.s, ar);
                    if (do_col) red_max_u32(amax_col_ws + h.s, ac);
                    // release: a producer that sees the count sees the maxima
                    red_release_add_u32(done_ws + h.s, 1u);
                }
            }
        } else if (!(h.flags & H_GAVE_UP)) {
            // ===================================================== cast tile
            uint8_t* const rc_base = p.row_codes + (uint64_t)h.row0 * K2 + (uint32_t)h.col0 / 2u;
            constexpr bool swz = Swz;
            // row scales: the plain [M, K/16] rows, or the tile's 1 KB of interleaved tiles
            uint8_t* const rs_base = swz ? p.row_sf + (((uint64_t)h.row0 >> 7) * (K16 >> 2) + ((uint32_t)h.col0 >> 6)) * 512u
                                         : p.row_sf + (uint64_t)h.row0 * K16 + (uint32_t)h.col0 / 16u;
            const uint64_t rs_4 = swz ? 64u : 4u * K16;  // row rr + 4
#pragma unroll
            for (int pi = 0; pi < 16 / NCW; ++pi) {
            const Part& pt = parts[pi];
            if (do_row && RowRht) {
                uint32_t wa[8], wb[8];
                load_row_pair(pt, wa, wb);
                f2 v[16];
                row_rht(wa, wb, sg, v);
                float r0[16], r1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) unpack2(v[i], r0[i], r1[i]);
                const uint32_t sf0 = block_sf(__fmul_rn(absmax16(r0), 0.25f), h.senc_r);
                const uint32_t sf1 = block_sf(__fmul_rn(absmax16(r1), 0.25f), h.senc_r);
                const f2 e2 = pack2(sh.enc[h.tab][0][sf0], sh.enc[h.tab][0][sf1]);
                if (!(h.flags & H_FOLD_R)) {
                    const f2 quarter = pack2(0.25f, 0.25f);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], quarter);
                }
                float q0[16], q1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) unpack2(mul2(v[i], e2), q0[i], q1[i]);
                // rows rr and rr + 4: codes in element order (no chunk swap)
                uint2 ca, cbw;
                if (sr_row) {
                    // element index of the block's first element in row_codes' order
                    const uint64_t e0 = (uint64_t)h.row0 * (uint64_t)p.K + (uint32_t)h.col0 + 16u * pt.rs_off0;
                    const uint4 wa = sr_block(p.sr_seed, (p.sr_offset + e0) / 16u);
                    const uint4 wb = sr_block(p.sr_seed, (p.sr_offset + e0 + 64u * K16) / 16u);
                    ca = make_uint2(e2m1x8_sr(q0, wa.x, wa.y), e2m1x8_sr(q0 + 8, wa.z, wa.w));
                    cbw = make_uint2(e2m1x8_sr(q1, wb.x, wb.y), e2m1x8_sr(q1 + 8, wb.z, wb.w));
                } else {
                    ca = make_uint2(e2m1x8(q0[0], q0[1], q0[2], q0[3], q0[4], q0[5], q0[6], q0[7]),
                                    e2m1x8(q0[8], q0[9], q0[10], q0[11], q0[12], q0[13], q0[14], q0[15]));
                    cbw = make_uint2(e2m1x8(q1[0], q1[1], q1[2], q1[3], q1[4], q1[5], q1[6], q1[7]),
                                     e2m1x8(q1[8], q1[9], q1[10], q1[11], q1[12], q1[13], q1[14], q1[15]));
                }
                *reinterpret_cast<uint2*>(rc_base + 8u * pt.rs_off0) = ca;
                *reinterpret_cast<uint2*>(rc_base + 8u * (pt.rs_off0 + 4u * K16)) = cbw;
                const uint64_t so = swz ? pt.rs_swz : pt.rs_off0;
                rs_base[so] = (uint8_t)sf0;
                rs_base[so + rs_4] = (uint8_t)sf1;
            } else if (do_row) {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint32_t ro = pt.roff0 + 4096u * kk;
                    const uint4 lo = *reinterpret_cast<const uint4*>(T + ro);  // (odd chunk if swap)
                    const uint4 hi = *reinterpret_cast<const uint4*>(T + (ro + pt.roff2));
                    const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    const uint32_t m = hmax_abs(hmax_abs(hmax_abs(wd[0], wd[1]), hmax_abs(wd[2], wd[3])),
                                                hmax_abs(hmax_abs(wd[4], wd[5]), hmax_abs(wd[6], wd[7])));
                    const uint32_t sf = block_sf(__uint_as_float(halves_max_bits(m)), h.senc_r);
                    const float enc = sh.enc[h.tab][0][sf];
                    const f2 e2 = pack2(enc, enc);
                    float q[16];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        bf16_t xl, xh;
                        split_bf16x2(wd[c], xl, xh);
                        unpack2(mul2(pack2(add_bf16(xl, -0.0f), add_bf16(xh, -0.0f)), e2), q[2 * c], q[2 * c + 1]);
                    }
                    const uint64_t rs_off = pt.rs_off0 + (kk ? 4u * K16 : 0u);
                    uint32_t c0, c1;
                    if (sr_row) {
                        const uint64_t e0 = (uint64_t)h.row0 * (uint64_t)p.K + (uint32_t)h.col0 + 16u * rs_off;
                        const uint4 w4 = sr_block(p.sr_seed, (p.sr_offset + e0) / 16u);
                        // q[0..7] are elements 8..15 of the block on lanes that loaded the odd chunk first
                        c0 = e2m1x8_sr(q, swap ? w4.z : w4.x, swap ? w4.w : w4.y);
                        c1 = e2m1x8_sr(q + 8, swap ? w4.x : w4.z, swap ? w4.y : w4.w);
                    } else {
                        c0 = e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
                        c1 = e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
                    }
                    *reinterpret_cast<uint2*>(rc_base + 8u * rs_off) =
                        swap ? make_uint2(c1, c0) : make_uint2(c0, c1);
                    rs_base[(swz ? pt.rs_swz : pt.rs_off0) + (kk ? rs_4 : 0u)] = (uint8_t)sf;
                }
            }
            if (do_col) {
                uint32_t x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = *reinterpret_cast<const uint32_t*>(T + pt.coff + 1024 * i);
                f2 v[16];
                column_rht(x, sg, v);
                float c0[16], c1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) unpack2(v[i], c0[i], c1[i]);
                const float a0 = absmax16(c0), a1 = absmax16(c1);
                const uint32_t sf0 = block_sf(__fmul_rn(a0, 0.25f), h.senc_c);
                const uint32_t sf1 = block_sf(__fmul_rn(a1, 0.25f), h.senc_c);
                const f2 e2 = pack2(sh.enc[h.tab][1][sf0], sh.enc[h.tab][1][sf1]);
                if (!(h.flags & H_FOLD)) {
                    const f2 quarter = pack2(0.25f, 0.25f);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = mul2(v[i], quarter);
                }
                float q0[16], q1[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) unpack2(mul2(v[i], e2), q0[i], q1[i]);
                // transposed section block: column c of the section at c * ms / 2
                const uint32_t ms2 = (uint32_t)h.ms / 2u, ms16 = (uint32_t)h.ms / 16u;
                const uint64_t c = (uint32_t)(h.col0 + pt.cpair);
                uint8_t* const cb = p.col_codes + (uint64_t)h.r0s * K2 + c * ms2 +
                                    ((uint32_t)h.row_in_sec0 / 2u + 8u * (uint32_t)rb);
                // (interleaved: the section's [K, M_s/16] scales in 128 x 4 tiles; this
                // tile of x owns 1 KB of them)
                uint8_t* const sbz = p.col_sf + (uint64_t)h.r0s * K16 +
                                     (((uint64_t)(uint32_t)h.col0 >> 7) * (ms16 >> 2) + ((uint32_t)h.row_in_sec0 >> 6)) * 512u +
                                     pt.cs_swz;
                uint8_t* const sb = p.col_sf + (uint64_t)h.r0s * K16 + c * ms16 +
                                    ((uint32_t)h.row_in_sec0 / 16u + (uint32_t)rb);
                if (sr_col) {
                    // element index in col_codes' order: twice the byte offset of cb
                    const uint64_t e0 = 2u * (uint64_t)(cb - p.col_codes);
                    const uint4 wa = sr_block(p.sr_seed + 1u, (p.sr_offset + e0) / 16u);
                    const uint4 wb = sr_block(p.sr_seed + 1u, (p.sr_offset + e0 + 2u * ms2) / 16u);
                    *reinterpret_cast<uint2*>(cb) = make_uint2(e2m1x8_sr(q0, wa.x, wa.y), e2m1x8_sr(q0 + 8, wa.z, wa.w));
                    *reinterpret_cast<uint2*>(cb + ms2) =
                        make_uint2(e2m1x8_sr(q1, wb.x, wb.y), e2m1x8_sr(q1 + 8, wb.z, wb.w));
                } else {
                    *reinterpret_cast<uint2*>(cb) =
                        make_uint2(e2m1x8(q0[0], q0[1], q0[2], q0[3], q0[4], q0[5], q0[6], q0[7]),
                                   e2m1x8(q0[8], q0[9], q0[10], q0[11], q0[12], q0[13], q0[14], q0[15]));
                    *reinterpret_cast<uint2*>(cb + ms2) =
                        make_uint2(e2m1x8(q1[0], q1[1], q1[2], q1[3], q1[4], q1[5], q1[6], q1[7]),
                                   e2m1x8(q1[8], q1[9], q1[10], q1[11], q1[12], q1[13], q1[14], q1[15]));
                }
                if (swz) {
                    sbz[0] = (uint8_t)sf0;
                    sbz[16] = (uint8_t)sf1;
                } else {
                    sb[0] = (uint8_t)sf0;
                    sb[ms16] = (uint8_t)sf1;
                }
            }
            }  // parts
        }
        mbar_arrive(&sh.empty[st]);  // every compute thread: this thread is done with the buffer
    }
}

// ------------------------------------------------------------ amax kernel
// The section maxima of the two-pass schedule's first launch, streamed
// through registers (rowwise output without the row RHT).  The unit of work
// is a strip of 16 rows x 128 columns of a tile (8 per tile), taken by one
// warp: lane l reads columns 4l..4l+3 of the 16 rows (16 eight-byte loads,
// each warp load instruction one 256-byte row segment), and the next strip's
// loads are issued before the current one is computed (2 CTAs of 8 warps and
// 128 registers per SM).  Strips are numbered in tile order (the 8 strips of
// a tile, then the next tile) and every warp takes one contiguous run of
// them, on its own: lane 0 keeps the warp's running maxima of its current
// section and adds them to the section's workspace maxima (two relaxed
// GPU-scope reductions) when the section changes and at the end, so no warp
// waits for another and a section's words see a few reductions per warp.  No counts:
// the cast launch that follows starts after this kernel has finished, which
// orders every reduction before it, and it reads the maxima as final (zero
// counts wanted per tile).  The rowwise maximum is taken on the BF16
// magnitudes, the columnwise one over the RHT16 outputs of the lane's two
// column pairs (the functions of the fused kernel's amax tiles).  It reads
// about 4.9 TB/s.  Measured against it on the grouped MoE call: a CTA-wide
// maximum and a count per tile behind a barrier, the same time; a count with
// release semantics per strip, 56 us slower (each release waits for the
// prefetched loads); strips dealt to warps round robin, 27 us slower (a
// reduction per strip, on the same few words); no prefetch, up to 11 us
// slower; a TMA-fed version, one CTA per SM with 6 buffers and 16 compute
// warps, 22 us slower.
constexpr int NA_THREADS = 256;
constexpr uint32_t NA_STRIPS = NV_TILE / 16;  // strips per tile

__global__ void __launch_bounds__(NA_THREADS, 2) nvfp4_amax_kernel(const __grid_constant__ NvParams p, uint32_t ntiles) {
    __shared__ int32_t sec_row0[HQ_MAX_SECTIONS + 1];
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    for (int i = tid; i <= p.S; i += NA_THREADS) sec_row0[i] = p.sec_row0[i];
    bf16_t sg[16];  // sigma_i as BF16 +-1
#pragma unroll
    for (int i = 0; i < 16; ++i) sg[i] = ((p.sign_mask >> i) & 1u) ? (bf16_t)0xBF80u : (bf16_t)0x3F80u;
    const bool do_row = p.flags & HQ_ROWWISE, do_col = p.flags & HQ_COLWISE;
    uint32_t* const amax_row_ws = p.ws + NV_WS_HEADER;
    uint32_t* const amax_col_ws = amax_row_ws + p.S;
    const uint32_t ct = (uint32_t)p.col_tiles;
    const uint32_t nstrips = ntiles * NA_STRIPS, nwarps = gridDim.x * (NA_THREADS / 32);
    const uint32_t gw = blockIdx.x * (NA_THREADS / 32) + (uint32_t)w;
    const uint32_t u_begin = (uint32_t)((uint64_t)nstrips * gw / nwarps);
    const uint32_t u_end = (uint32_t)((uint64_t)nstrips * (gw + 1u) / nwarps);  // this warp's run
    __syncthreads();
    int s = 0;  // lane 0: section of the current strip (a warp's strips come in increasing order)
    uint32_t run_row = 0u, run_col = 0u;  // lane 0: the warp's maxima of section s so far
    auto flush = [&]() {
        if (do_row && run_row) red_max_u32(amax_row_ws + s, run_row);
        if (do_col && run_col) red_max_u32(amax_col_ws + s, run_col);
        run_row = run_col = 0u;
    };
    uint32_t na[16], nb[16];
    auto load = [&](uint32_t u) {
        const uint32_t t = u / NA_STRIPS, rt = t / ct, cti = t - rt * ct;
        const uint16_t* src = p.x + ((int64_t)rt * NV_TILE + 16 * (u % NA_STRIPS)) * p.K + (int64_t)cti * NV_TILE +
                              4 * lane;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + i * p.K));
            na[i] = v.x;
            nb[i] = v.y;
        }
    };
    if (u_begin < u_end) load(u_begin);
    for (uint32_t u = u_begin; u < u_end; ++u) {
        const int row0 = (int)((u / NA_STRIPS / ct) * NV_TILE);
        uint32_t wa[16], wb[16];  // row i: columns 4l, 4l + 1 and 4l + 2, 4l + 3
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            wa[i] = na[i];
            wb[i] = nb[i];
        }
        if (u + 1u < u_end) load(u + 1u);
        uint32_t mrow = 0u;
        float mcol = 0.0f;
        if (do_row) {
            uint32_t m2 = 0u;  // BF16 pair of running magnitude maxima (a NaN is skipped)
#pragma unroll
            for (int i = 0; i < 16; ++i) m2 = hmax_abs(m2, hmax_abs(wa[i], wb[i]));
            mrow = halves_max_bits(m2);
        }
        if (do_col) {
            mcol = column_rht_absmax(wa, sg, 0.0f);
            mcol = column_rht_absmax(wb, sg, mcol);
        }
        // non-negative binary32 bits order as integers; max |0.25 y| == RN(0.25 max |y|)
        mrow = __reduce_max_sync(0xFFFFFFFFu, mrow);
        const uint32_t mc = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(__fmul_rn(mcol, 0.25f)));
        if (lane == 0) {
            if (sec_row0[s + 1] <= row0) {
                flush();
                while (sec_row0[s + 1] <= row0) ++s;
            }
            run_row = max(run_row, mrow);
            run_col = max(run_col, mc);
        }
    }
    if (lane == 0) flush();
}

}  // namespace

template <bool RowRht, bool SR, bool Swz>
__global__ void __launch_bounds__(NV_THREADS, NV_CTAS_PER_SM) nvfp4_group_kernel(const __grid_constant__ NvParams p) {
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
    for (int i = tid; i < p.S; i += NV_THREADS) {
        const uint32_t trows = (uint32_t)(p.sec_row0[i + 1] - p.sec_row0[i]) / NV_TILE;
        sh.sec_magic[i] = trows ? 0xFFFFFFFFu / trows : 0u;
    }
    if (tid < 128) {
        const bool z = tid == 0 || tid == 127;
        const float v = z ? 0.0f : e4m3_value((uint32_t)tid);
        sh.vr[tid] = make_float2(v, z ? -0.0f : -__frcp_rn(v));
    }
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
        nv_consumer<RowRht, SR, Swz>(p, sh, nv_smem, warp, lane);
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
        const bool given = p.flags & HQ_AMAX_GIVEN;  // amax_* are inputs: only sdec is written
        for (int s = tid; s < p.S; s += NV_THREADS) {
            if (do_row) {
                const float A = given ? p.amax_row[s] : __uint_as_float(*(volatile uint32_t*)(amax_row_ws + s));
                if (!given) p.amax_row[s] = A;
                p.sdec_row[s] = __fdiv_rn(1.0f, global_encode(A));
                amax_row_ws[s] = 0;
            }
            if (do_col) {
                const float A = given ? p.amax_col[s] : __uint_as_float(*(volatile uint32_t*)(amax_col_ws + s));
                if (!given) p.amax_col[s] = A;
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

// The instances, indexed by HQ_ROW_RHT | SR << 1 | interleaved scales << 2.
static void (*const nv_kernels[8])(NvParams) = {
    nvfp4_group_kernel<false, false, false>, nvfp4_group_kernel<true, false, false>,
    nvfp4_group_kernel<false, true, false>,  nvfp4_group_kernel<true, true, false>,
    nvfp4_group_kernel<false, false, true>,  nvfp4_group_kernel<true, false, true>,
    nvfp4_group_kernel<false, true, true>,   nvfp4_group_kernel<true, true, true>};

int nvfp4_blocks_per_sm() {
    // every instance: the grid is sized for the one with fewest resident CTAs
    int n = 1 << 30;
    for (auto* k : nv_kernels) {
        int m = 0;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, NV_DYN_SMEM);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, k, NV_THREADS, NV_DYN_SMEM);
        n = m < n ? m : n;
    }
    return n > 0 ? n : 1;
}

// Tiles per CTA the fused schedule puts between a section's amax and cast
// segments: the buffers and the claims in flight, enough for the amax tiles
// to be done and small enough for the rows to stay in L2.
int nvfp4_tiles_in_flight_per_cta() { return NST + 2; }

int nvfp4_tiles_per_claim() { return CLAIM; }

int nvfp4_amax_blocks_per_sm() {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4_amax_kernel, NA_THREADS, 0);
    return n > 0 ? n : 1;
}

void launch_nvfp4_amax(const NvParams& p, uint32_t ntiles, int grid, cudaStream_t st) {
    nvfp4_amax_kernel<<<grid, NA_THREADS, 0, st>>>(p, ntiles);
}

void launch_nvfp4(const NvParams& p, int grid, cudaStream_t st) {
    const int v = ((p.flags & HQ_ROW_RHT) ? 1 : 0) | ((p.flags & (HQ_ROW_SR | HQ_COL_SR)) ? 2 : 0) |
                  ((p.flags & HQ_SF_SWIZZLED) ? 4 : 0);
    nv_kernels[v]<<<grid, NV_THREADS, NV_DYN_SMEM, st>>>(p);
}
}  // namespace hq
