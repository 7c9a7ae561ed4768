// hq_api.cu -- the extern "C" entry points of include/hq.h: argument checks,
// kernel parameter blocks, grid sizing and launches.  No allocation (a fixed
// set of CUDA events per device for the host-buffer entry, created once), no
// synchronization (hq_get_error excepted), no environment reads.
#include <cudaTypedefs.h>
#include <string.h>

#include <mutex>

#include "hq_internal.h"

using namespace hq;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sms = 0;
    int nv_blocks_per_sm = 0;
    int cat_blocks_per_sm[2] = {0, 0};  // FP8, FP4 DSA kernels
    int amax_blocks_per_sm = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

// SM count and resident CTAs per SM of the persistent kernels, per device.
const DeviceInfo* device_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_dev_once[dev], [dev] {
        DeviceInfo d;
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        d.nv_blocks_per_sm = nvfp4_blocks_per_sm();
        d.cat_blocks_per_sm[0] = cat_rotate_blocks_per_sm(false);
        d.cat_blocks_per_sm[1] = cat_rotate_blocks_per_sm(true);
        d.amax_blocks_per_sm = nvfp4_amax_blocks_per_sm();
        g_dev[dev] = d;
    });
    const DeviceInfo* d = &g_dev[dev];
    return d->sms > 0 ? d : nullptr;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

inline hq_status launch_status() {
    return cudaPeekAtLastError() == cudaSuccess ? HQ_OK : (cudaGetLastError(), HQ_ERR_CUDA);
}

// header, amax_row[S], amax_col[S], done[S] (amax tiles counted per section)
size_t nv_ws_words(int S) { return (size_t)NV_WS_HEADER + 3 * (size_t)S; }

// The driver's tensor-map encoder, reached once through the runtime (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// x (BF16 [M, K], rows of K elements) viewed as [M/16][16][K]: 16-row block,
// row in block, column.  Boxes of 64 columns x 8 blocks x 16 rows land
// row-in-block major with the 128-byte swizzle.
bool encode_x_map(CUtensorMap* map, const void* x, int64_t M, int64_t K) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)(M / 16), 16};
    const cuuint64_t strides[2] = {(cuuint64_t)(16 * K * 2), (cuuint64_t)(K * 2)};  // bytes, dims 1 and 2
    const cuuint32_t box[3] = {64, 8, 16};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Offsets (bytes, 256-aligned) of the host-buffer entry's device staging:
// x, the four code / scale buffers, the four per-section arrays, workspace.
struct StagingLayout {
    size_t x, row_codes, row_sf, col_codes, col_sf, amax_row, amax_col, sdec_row, sdec_col, ws, total;
};
StagingLayout staging_layout(int64_t M, int64_t K, int S, size_t ws_bytes) {
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const size_t e = (size_t)M * (size_t)K;
    StagingLayout L;
    size_t o = 0;
    L.x = o;         o = up(o + 2 * e);
    L.row_codes = o; o = up(o + e / 2);
    L.row_sf = o;    o = up(o + e / 16);
    L.col_codes = o; o = up(o + e / 2);
    L.col_sf = o;    o = up(o + e / 16);
    L.amax_row = o;  o = up(o + 4 * (size_t)S);
    L.amax_col = o;  o = up(o + 4 * (size_t)S);
    L.sdec_row = o;  o = up(o + 4 * (size_t)S);
    L.sdec_col = o;  o = up(o + 4 * (size_t)S);
    L.ws = o;        o = up(o + ws_bytes);
    L.total = o;
    return L;
}

// Events of the host-buffer entry, per device: created on first use; a
// mutex serializes the enqueueing of calls (a stream wait takes the event's
// latest record at the time of the wait, so a later call may re-record).
struct HostEvents {
    cudaEvent_t start = nullptr, end = nullptr, in[HQ_HOST_MAX_GROUPS] = {}, out[HQ_HOST_MAX_GROUPS] = {};
    bool ok = false;
    std::mutex mu;
};
HostEvents g_host_ev[kMaxDevices];
std::once_flag g_host_ev_once[kMaxDevices];

HostEvents* host_events() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_host_ev_once[dev], [dev] {
        HostEvents& h = g_host_ev[dev];
        bool ok = cudaEventCreateWithFlags(&h.start, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&h.end, cudaEventDisableTiming) == cudaSuccess;
        for (int g = 0; g < HQ_HOST_MAX_GROUPS && ok; ++g)
            ok = cudaEventCreateWithFlags(&h.in[g], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h.out[g], cudaEventDisableTiming) == cudaSuccess;
        h.ok = ok;
    });
    return g_host_ev[dev].ok ? &g_host_ev[dev] : nullptr;
}

}  // namespace

extern "C" {

int hq_version(void) { return (0 << 16) | 1; }

const char* hq_status_string(hq_status s) {
    switch (s) {
        case HQ_OK: return "ok";
        case HQ_ERR_NULL: return "required pointer is NULL";
        case HQ_ERR_SHAPE: return "sizes negative, inconsistent or too large";
        case HQ_ERR_ALIGN: return "misaligned pointer/stride or size not a multiple of the block";
        case HQ_ERR_WORKSPACE: return "workspace missing or too small";
        case HQ_ERR_UNSUPPORTED: return "unsupported flag, mode, layout or transform size";
        case HQ_ERR_CUDA: return "CUDA runtime error";
        case HQ_ERR_TIMEOUT: return "bounded device wait gave up";
    }
    return "unknown status";
}

size_t hq_group_rht_quant_workspace_size(int num_sections) {
    if (num_sections < 1 || num_sections > HQ_MAX_SECTIONS) return 0;
    const size_t bytes = nv_ws_words(num_sections) * sizeof(uint32_t);
    return (bytes + 255) & ~(size_t)255;
}

hq_status hq_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws) return HQ_ERR_NULL;
    if (!aligned16(ws)) return HQ_ERR_ALIGN;
    if (cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) != cudaSuccess) return HQ_ERR_CUDA;
    return HQ_OK;
}

hq_status hq_get_error(void* ws, size_t ws_bytes, uint32_t* err_out, void* stream) {
    if (!ws || !err_out) return HQ_ERR_NULL;
    if (ws_bytes < NV_WS_HEADER * sizeof(uint32_t)) return HQ_ERR_WORKSPACE;
    uint32_t* err = static_cast<uint32_t*>(ws) + 2;
    uint32_t host = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&host, err, sizeof host, cudaMemcpyDeviceToHost, st) != cudaSuccess) return HQ_ERR_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return HQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return HQ_ERR_CUDA;
    *err_out = host;
    return HQ_OK;
}

static hq_status group_rht_quant(const void* x, int64_t M, int64_t K, const int64_t* split_rows, int S,
                                 uint16_t sign_mask, unsigned flags, uint64_t sr_seed, uint64_t sr_offset,
                                 uint8_t* row_codes, uint8_t* row_sf, uint8_t* col_codes, uint8_t* col_sf,
                                 float* amax_row, float* amax_col, float* sdec_row, float* sdec_col, void* ws,
                                 size_t ws_bytes, void* stream) {
    // ---- argument checks (nothing is launched on failure)
    if (flags & ~(HQ_ROWWISE | HQ_COLWISE | HQ_ROW_RHT | HQ_AMAX_GIVEN | HQ_TWO_PASS | HQ_ROW_SR | HQ_COL_SR | HQ_SF_SWIZZLED))
        return HQ_ERR_UNSUPPORTED;
    if ((flags & HQ_ROW_SR) && !(flags & HQ_ROWWISE)) return HQ_ERR_UNSUPPORTED;
    if ((flags & HQ_COL_SR) && !(flags & HQ_COLWISE)) return HQ_ERR_UNSUPPORTED;
    if (sr_offset % 16 != 0) return HQ_ERR_ALIGN;  // a 16-element block takes one random block
    const bool do_row = flags & HQ_ROWWISE, do_col = flags & HQ_COLWISE;
    if (!do_row && !do_col) return HQ_ERR_UNSUPPORTED;
    if ((flags & HQ_ROW_RHT) && !do_row) return HQ_ERR_UNSUPPORTED;
    if (!split_rows || !ws) return HQ_ERR_NULL;
    // code and block-scale buffers are empty (and may be NULL) when M == 0
    if (do_row && (!amax_row || !sdec_row || (M > 0 && (!row_codes || !row_sf)))) return HQ_ERR_NULL;
    if (do_col && (!amax_col || !sdec_col || (M > 0 && (!col_codes || !col_sf)))) return HQ_ERR_NULL;
    if (S < 1 || S > HQ_MAX_SECTIONS || M < 0 || K <= 0) return HQ_ERR_SHAPE;
    if (M > 0 && !x) return HQ_ERR_NULL;
    if (K % NV_TILE != 0) return HQ_ERR_ALIGN;
    if (M * K >= ((int64_t)1 << 40) || M >= ((int64_t)1 << 31)) return HQ_ERR_SHAPE;
    int64_t total = 0;
    for (int s = 0; s < S; ++s) {
        if (split_rows[s] < 0) return HQ_ERR_SHAPE;
        if (split_rows[s] % NV_TILE != 0) return HQ_ERR_ALIGN;
        total += split_rows[s];
    }
    if (total != M) return HQ_ERR_SHAPE;
    if ((M > 0 && !aligned16(x)) || !aligned16(ws)) return HQ_ERR_ALIGN;
    if (do_row && (!aligned16(row_codes) || !aligned16(row_sf) || !aligned4(amax_row) || !aligned4(sdec_row)))
        return HQ_ERR_ALIGN;
    if (do_col && (!aligned16(col_codes) || !aligned16(col_sf) || !aligned4(amax_col) || !aligned4(sdec_col)))
        return HQ_ERR_ALIGN;  // (NULL is 16-byte aligned: empty buffers pass)
    if (ws_bytes < hq_group_rht_quant_workspace_size(S)) return HQ_ERR_WORKSPACE;
    const DeviceInfo* dev = device_info();
    if (!dev) return HQ_ERR_CUDA;

    // ---- schedule: per non-empty section an amax segment and a cast segment
    NvParams p;
    memset(&p, 0, sizeof p);
    p.x = static_cast<const uint16_t*>(x);
    p.K = K;
    if (M > 0 && K > 0 && !encode_x_map(&p.tmap, x, M, K)) return HQ_ERR_CUDA;
    p.row_codes = row_codes; p.row_sf = row_sf; p.col_codes = col_codes; p.col_sf = col_sf;
    p.amax_row = amax_row; p.amax_col = amax_col; p.sdec_row = sdec_row; p.sdec_col = sdec_col;
    p.ws = static_cast<uint32_t*>(ws);
    p.S = S;
    p.sign_mask = sign_mask;
    p.flags = flags & (HQ_ROWWISE | HQ_COLWISE | HQ_ROW_RHT | HQ_AMAX_GIVEN | HQ_ROW_SR | HQ_COL_SR | HQ_SF_SWIZZLED);
    p.sr_seed = sr_seed;
    p.sr_offset = sr_offset;
    p.col_tiles = (int)(K / NV_TILE);
    p.done_per_tile = 1;
    int row0 = 0;
    int live[HQ_MAX_SECTIONS];
    int nlive = 0;
    for (int s = 0; s < S; ++s) {
        p.sec_row0[s] = row0;
        row0 += (int)split_rows[s];
        if (split_rows[s] > 0) live[nlive++] = s;
    }
    p.sec_row0[S] = row0;

    auto tiles_of = [&](int s) { return (uint32_t)(split_rows[s] / NV_TILE) * (uint32_t)p.col_tiles; };
    auto add_seg = [&](NvParams& q, int s, int phase, uint32_t& next) {
        q.seg_start[q.nseg] = next;
        q.seg_info[q.nseg] = (uint16_t)(s | (phase << 15));
        ++q.nseg;
        next += tiles_of(s);
    };
    cudaStream_t st = (cudaStream_t)stream;
    const int max_grid = dev->sms * (dev->nv_blocks_per_sm > 0 ? dev->nv_blocks_per_sm : 1);
    const uint32_t per_claim = (uint32_t)nvfp4_tiles_per_claim();
    auto grid_for = [&](uint32_t items) {  // no more CTAs than claims
        const uint32_t claims = (items + per_claim - 1) / per_claim;
        return (int)(claims < (uint32_t)max_grid ? (claims > 0 ? claims : 1) : (uint32_t)max_grid);
    };
    auto launch = [&](NvParams& q, uint32_t items) -> hq_status {
        q.seg_start[q.nseg] = items;
        q.total_items = items;
        // multi-tile claims, then single tiles for about two per CTA at the end
        const uint32_t tail = 2u * (uint32_t)grid_for(items);
        q.multi_claims = items > tail ? (items - tail) / per_claim : 0u;
        launch_nvfp4(q, grid_for(items), st);
        return launch_status();
    };

    if (flags & HQ_AMAX_GIVEN) {
        // One pass: the cast segments alone; each section's record comes from
        // the caller's amax.
        uint32_t next = 0;
        for (int k = 0; k < nlive; ++k) add_seg(p, live[k], 1, next);
        p.finalize = 1;
        p.reset_counter = 1;
        return launch(p, next);
    }
    // One non-empty section (a dense tensor): its casts wait for the whole
    // amax pass in one launch too, and the streaming amax kernel reads faster
    // than amax tiles do, so two launches unless the section is smaller than
    // one wave of the grid (then the second launch costs more).
    const bool one_section = nlive == 1 && !(flags & HQ_ROW_RHT) && tiles_of(live[0]) >= (uint32_t)max_grid;
    if (!(flags & HQ_TWO_PASS) && !one_section) {
        // One launch.  The cast segment of a section follows its amax segment
        // once `lag` more tiles have been scheduled (the tiles the grid holds
        // in flight), so its amax is normally complete when its first tile is
        // claimed and its rows are still in L2 (the distance between a tile's
        // two reads is the section's tiles plus the lag; interleaving amax and
        // cast tiles more finely measured no faster and doubled that distance
        // for the first tiles, reading a third more from DRAM).  Every tile
        // depends only on tiles scheduled before it.
        uint32_t all = 0;
        for (int k = 0; k < nlive; ++k) all += 2 * tiles_of(live[k]);
        const uint32_t lag = (uint32_t)grid_for(all) * (uint32_t)nvfp4_tiles_in_flight_per_cta();
        uint32_t next = 0, a_end[HQ_MAX_SECTIONS];
        int pend = 0;  // next section whose cast segment is still to be scheduled
        for (int k = 0; k < nlive; ++k) {
            add_seg(p, live[k], 0, next);
            a_end[k] = next;
            while (pend < k && next - a_end[pend] >= lag) {
                add_seg(p, live[pend], 1, next);
                ++pend;
            }
        }
        while (pend < nlive) {
            add_seg(p, live[pend], 1, next);
            ++pend;
        }
        p.finalize = 1;
        p.reset_counter = 1;
        return launch(p, next);
    }
    // two launches: all amax tiles, then all cast tiles, the sections in
    // reverse order (the last rows the amax launch read are still in L2)
    NvParams pa = p, pc = p;
    uint32_t na = 0, nc = 0;
    for (int k = 0; k < nlive; ++k) add_seg(pa, live[k], 0, na);
    for (int k = nlive - 1; k >= 0; --k) add_seg(pc, live[k], 1, nc);
    pa.finalize = 0;
    pa.reset_counter = 1;
    pc.finalize = 1;
    pc.reset_counter = 1;
    hq_status r;
    if (!(flags & HQ_ROW_RHT)) {
        // the streaming amax kernel over all tiles (empty sections have none)
        const uint32_t ntiles = (uint32_t)(M / NV_TILE) * (uint32_t)p.col_tiles;
        const uint32_t cap = (uint32_t)dev->sms * (uint32_t)dev->amax_blocks_per_sm;
        if (ntiles > 0) launch_nvfp4_amax(pa, ntiles, (int)(ntiles < cap ? ntiles : cap), st);
        pc.done_per_tile = 0;  // the launch boundary orders the maxima: no counts to wait for
        r = launch_status();
    } else {
        r = launch(pa, na);
    }
    if (r != HQ_OK) return r;
    return launch(pc, nc);
}

hq_status hq_group_rht_quant(const void* x, int64_t M, int64_t K, const int64_t* split_rows, int S,
                             uint16_t sign_mask, unsigned flags, uint8_t* row_codes, uint8_t* row_sf,
                             uint8_t* col_codes, uint8_t* col_sf, float* amax_row, float* amax_col,
                             float* sdec_row, float* sdec_col, void* ws, size_t ws_bytes, void* stream) {
    if (flags & (HQ_ROW_SR | HQ_COL_SR)) return HQ_ERR_UNSUPPORTED;  // needs a seed: hq_group_rht_quant_sr
    return group_rht_quant(x, M, K, split_rows, S, sign_mask, flags, 0, 0, row_codes, row_sf, col_codes, col_sf,
                           amax_row, amax_col, sdec_row, sdec_col, ws, ws_bytes, stream);
}

hq_status hq_group_rht_quant_sr(const void* x, int64_t M, int64_t K, const int64_t* split_rows, int S,
                                uint16_t sign_mask, unsigned flags, uint64_t seed, uint64_t offset,
                                uint8_t* row_codes, uint8_t* row_sf, uint8_t* col_codes, uint8_t* col_sf,
                                float* amax_row, float* amax_col, float* sdec_row, float* sdec_col, void* ws,
                                size_t ws_bytes, void* stream) {
    return group_rht_quant(x, M, K, split_rows, S, sign_mask, flags, seed, offset, row_codes, row_sf, col_codes,
                           col_sf, amax_row, amax_col, sdec_row, sdec_col, ws, ws_bytes, stream);
}

size_t hq_group_rht_quant_host_device_bytes(int64_t M, int64_t K, int S) {
    if (S < 1 || S > HQ_MAX_SECTIONS || M < 0 || K <= 0 || K % NV_TILE != 0) return 0;
    if (M * K >= ((int64_t)1 << 40) || M >= ((int64_t)1 << 31)) return 0;
    return staging_layout(M, K, S, hq_group_rht_quant_workspace_size(S)).total;
}

hq_status hq_group_rht_quant_host(const void* x, int64_t M, int64_t K, const int64_t* split_rows, int S,
                                  uint16_t sign_mask, unsigned flags, uint64_t seed, uint64_t offset,
                                  uint8_t* row_codes, uint8_t* row_sf, uint8_t* col_codes, uint8_t* col_sf,
                                  float* amax_row, float* amax_col, float* sdec_row, float* sdec_col,
                                  void* dev_buf, size_t dev_buf_bytes, int groups, void* stream,
                                  void* h2d_stream, void* d2h_stream) {
    // ---- checks of what the per-group calls cannot see (they check the rest
    // again on the staging pointers)
    if (flags & ~(HQ_ROWWISE | HQ_COLWISE | HQ_ROW_RHT | HQ_AMAX_GIVEN | HQ_TWO_PASS | HQ_ROW_SR | HQ_COL_SR | HQ_SF_SWIZZLED))
        return HQ_ERR_UNSUPPORTED;
    const bool do_row = flags & HQ_ROWWISE, do_col = flags & HQ_COLWISE;
    if (!do_row && !do_col) return HQ_ERR_UNSUPPORTED;
    if ((flags & HQ_ROW_RHT) && !do_row) return HQ_ERR_UNSUPPORTED;
    if ((flags & HQ_ROW_SR) && !do_row) return HQ_ERR_UNSUPPORTED;
    if ((flags & HQ_COL_SR) && !do_col) return HQ_ERR_UNSUPPORTED;
    if ((flags & (HQ_ROW_SR | HQ_COL_SR)) && offset % 16 != 0) return HQ_ERR_ALIGN;
    if (!split_rows || !dev_buf) return HQ_ERR_NULL;
    if (S < 1 || S > HQ_MAX_SECTIONS || M < 0 || K <= 0) return HQ_ERR_SHAPE;
    if (K % NV_TILE != 0) return HQ_ERR_ALIGN;
    if (M * K >= ((int64_t)1 << 40) || M >= ((int64_t)1 << 31)) return HQ_ERR_SHAPE;
    int64_t total = 0;
    for (int s = 0; s < S; ++s) {
        if (split_rows[s] < 0) return HQ_ERR_SHAPE;
        if (split_rows[s] % NV_TILE != 0) return HQ_ERR_ALIGN;
        total += split_rows[s];
    }
    if (total != M) return HQ_ERR_SHAPE;
    if (M > 0 && !x) return HQ_ERR_NULL;
    if (do_row && (!amax_row || !sdec_row || (M > 0 && (!row_codes || !row_sf)))) return HQ_ERR_NULL;
    if (do_col && (!amax_col || !sdec_col || (M > 0 && (!col_codes || !col_sf)))) return HQ_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(dev_buf) & 255u) != 0) return HQ_ERR_ALIGN;
    const size_t ws_bytes = hq_group_rht_quant_workspace_size(S);
    const StagingLayout L = staging_layout(M, K, S, ws_bytes);
    if (dev_buf_bytes < L.total) return HQ_ERR_WORKSPACE;
    if (groups == 0) groups = 16;
    if (groups < 1 || groups > HQ_HOST_MAX_GROUPS) return HQ_ERR_UNSUPPORTED;
    if (h2d_stream == d2h_stream || h2d_stream == stream || d2h_stream == stream) return HQ_ERR_UNSUPPORTED;
    HostEvents* ev = host_events();
    if (!ev) return HQ_ERR_CUDA;

    // ---- section groups of about M / groups rows (whole sections)
    int gs[HQ_HOST_MAX_GROUPS + 1];
    int ng = 0;
    gs[0] = 0;
    const int64_t target = (M + groups - 1) / groups;
    int64_t acc = 0;
    for (int s = 0; s < S; ++s) {
        acc += split_rows[s];
        if (acc >= target && acc > 0 && ng + 1 < groups && s + 1 < S) {
            gs[++ng] = s + 1;
            acc = 0;
        }
    }
    gs[++ng] = S;

    uint8_t* const base = static_cast<uint8_t*>(dev_buf);
    const uint8_t* const hx = static_cast<const uint8_t*>(x);
    const cudaStream_t st = (cudaStream_t)stream, hs = (cudaStream_t)h2d_stream, ds = (cudaStream_t)d2h_stream;
    const size_t fS = 4 * (size_t)S;
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    std::lock_guard<std::mutex> lock(ev->mu);
    // the copies start after the work already on `stream`
    if (!ok(cudaEventRecord(ev->start, st)) || !ok(cudaStreamWaitEvent(hs, ev->start, 0)) ||
        !ok(cudaStreamWaitEvent(ds, ev->start, 0)))
        return HQ_ERR_CUDA;
    if (flags & HQ_AMAX_GIVEN) {
        if (do_row && !ok(cudaMemcpyAsync(base + L.amax_row, amax_row, fS, cudaMemcpyHostToDevice, hs)))
            return HQ_ERR_CUDA;
        if (do_col && !ok(cudaMemcpyAsync(base + L.amax_col, amax_col, fS, cudaMemcpyHostToDevice, hs)))
            return HQ_ERR_CUDA;
    }
    int64_t r0 = 0;
    for (int g = 0; g < ng; ++g) {
        const int sa = gs[g], sb = gs[g + 1];
        int64_t rows = 0;
        for (int s = sa; s < sb; ++s) rows += split_rows[s];
        const size_t e0 = (size_t)r0 * (size_t)K, e = (size_t)rows * (size_t)K;
        if (rows > 0 && !ok(cudaMemcpyAsync(base + L.x + 2 * e0, hx + 2 * e0, 2 * e, cudaMemcpyHostToDevice, hs)))
            return HQ_ERR_CUDA;
        if (!ok(cudaEventRecord(ev->in[g], hs)) || !ok(cudaStreamWaitEvent(st, ev->in[g], 0))) return HQ_ERR_CUDA;
        // the group's sections as one call; the random streams keep their
        // element indices (offset + first element of the group)
        const hq_status r = group_rht_quant(
            base + L.x + 2 * e0, rows, K, split_rows + sa, sb - sa, sign_mask, flags, seed,
            (flags & (HQ_ROW_SR | HQ_COL_SR)) ? offset + e0 : 0, do_row ? base + L.row_codes + e0 / 2 : nullptr,
            do_row ? base + L.row_sf + e0 / 16 : nullptr, do_col ? base + L.col_codes + e0 / 2 : nullptr,
            do_col ? base + L.col_sf + e0 / 16 : nullptr,
            do_row ? reinterpret_cast<float*>(base + L.amax_row) + sa : nullptr,
            do_col ? reinterpret_cast<float*>(base + L.amax_col) + sa : nullptr,
            do_row ? reinterpret_cast<float*>(base + L.sdec_row) + sa : nullptr,
            do_col ? reinterpret_cast<float*>(base + L.sdec_col) + sa : nullptr, base + L.ws, ws_bytes, stream);
        if (r != HQ_OK) return r;
        if (!ok(cudaEventRecord(ev->out[g], st)) || !ok(cudaStreamWaitEvent(ds, ev->out[g], 0))) return HQ_ERR_CUDA;
        if (rows > 0) {
            if (do_row && (!ok(cudaMemcpyAsync(row_codes + e0 / 2, base + L.row_codes + e0 / 2, e / 2,
                                               cudaMemcpyDeviceToHost, ds)) ||
                           !ok(cudaMemcpyAsync(row_sf + e0 / 16, base + L.row_sf + e0 / 16, e / 16,
                                               cudaMemcpyDeviceToHost, ds))))
                return HQ_ERR_CUDA;
            if (do_col && (!ok(cudaMemcpyAsync(col_codes + e0 / 2, base + L.col_codes + e0 / 2, e / 2,
                                               cudaMemcpyDeviceToHost, ds)) ||
                           !ok(cudaMemcpyAsync(col_sf + e0 / 16, base + L.col_sf + e0 / 16, e / 16,
                                               cudaMemcpyDeviceToHost, ds))))
                return HQ_ERR_CUDA;
        }
        r0 += rows;
    }
    // the per-section arrays after the last group
    if (do_row && ((!(flags & HQ_AMAX_GIVEN) &&
                    !ok(cudaMemcpyAsync(amax_row, base + L.amax_row, fS, cudaMemcpyDeviceToHost, ds))) ||
                   !ok(cudaMemcpyAsync(sdec_row, base + L.sdec_row, fS, cudaMemcpyDeviceToHost, ds))))
        return HQ_ERR_CUDA;
    if (do_col && ((!(flags & HQ_AMAX_GIVEN) &&
                    !ok(cudaMemcpyAsync(amax_col, base + L.amax_col, fS, cudaMemcpyDeviceToHost, ds))) ||
                   !ok(cudaMemcpyAsync(sdec_col, base + L.sdec_col, fS, cudaMemcpyDeviceToHost, ds))))
        return HQ_ERR_CUDA;
    // work enqueued on `stream` afterwards runs after the last copy back
    if (!ok(cudaEventRecord(ev->end, ds)) || !ok(cudaStreamWaitEvent(st, ev->end, 0))) return HQ_ERR_CUDA;
    return HQ_OK;
}

size_t hq_cat_rotate_fp8_workspace_size(void) { return 0; }
size_t hq_swiglu_fp8_k128_workspace_size(void) { return 0; }

// Both DSA entry points: argument checks, tiling, launch.  fp4: NVFP4 codes
// [M, G*64] in `out`, block scales [M, G*8] in `sf`, per-vector decode
// scales in `scales`; else FP8 codes [M, G*128] and group scales.
static hq_status cat_rotate(const void* a, int64_t a_row_stride, int a_width, const void* b, int64_t b_row_stride,
                            int b_width, int64_t M, int G, int hadamard_n, uint8_t* out, uint8_t* sf, float* scales,
                            int scale_layout, int64_t scale_ld, float* amax_opt, void* stream, bool fp4) {
    if (hadamard_n != 0 && hadamard_n != 128) return HQ_ERR_UNSUPPORTED;
    // the format bit of this call: UE8M0 FP8 scales, or interleaved FP4 block scales
    const int fmt_bit = fp4 ? (int)HQ_SF_SWIZZLED : HQ_FP8_UE8M0;
    const bool fmt = (scale_layout & fmt_bit) != 0;
    scale_layout &= ~fmt_bit;
    if (scale_layout != HQ_SCALE_ROWMAJOR && scale_layout != HQ_SCALE_TRANSPOSED) return HQ_ERR_UNSUPPORTED;
    if (M < 0 || G <= 0 || a_width < 0 || b_width < 0 || a_width + b_width != 128) return HQ_ERR_SHAPE;
    if (M == 0) return HQ_OK;
    if (!a || !out || !scales || (b_width > 0 && !b) || (fp4 && !sf)) return HQ_ERR_NULL;
    if (a_width % 8 || b_width % 8 || a_row_stride % 8 || b_row_stride % 8) return HQ_ERR_ALIGN;
    if (a_row_stride < (int64_t)G * a_width || (b_width > 0 && b_row_stride < (int64_t)G * b_width))
        return HQ_ERR_SHAPE;
    if (scale_layout == HQ_SCALE_TRANSPOSED && scale_ld < M) return HQ_ERR_SHAPE;
    if (fp4 && fmt && M % 128 != 0) return HQ_ERR_ALIGN;  // whole 128-row tiles of block scales
    if (!aligned16(a) || (b_width > 0 && !aligned16(b)) || !aligned16(out) || !aligned4(scales) ||
        !aligned4(amax_opt))
        return HQ_ERR_ALIGN;
    const DeviceInfo* dev = device_info();
    if (!dev) return HQ_ERR_CUDA;

    CatRotateParams p;
    p.a = static_cast<const uint16_t*>(a);
    p.b = static_cast<const uint16_t*>(b);
    p.a_row_stride = a_row_stride;
    p.b_row_stride = b_row_stride;
    p.a_width = a_width;
    p.b_width = b_width;
    p.nvec = M * G;
    p.M = M;
    p.G = G;
    p.rotate = hadamard_n == 128;
    p.out = out;
    p.sf = sf;
    p.scales = scales;
    p.amax = amax_opt;
    p.scale_layout = scale_layout;
    p.scale_ld = scale_ld;
    p.ue8m0 = !fp4 && fmt;
    p.sf_swizzle = fp4 && fmt;
    p.wide32 = a_width % 32 == 0 && b_width % 32 == 0 && a_row_stride % 16 == 0 && b_row_stride % 16 == 0 &&
               (reinterpret_cast<uintptr_t>(a) & 31u) == 0 && (b_width == 0 || (reinterpret_cast<uintptr_t>(b) & 31u) == 0);
    p.ntiles = cat_rotate_tiles(p);
    if (p.nvec >= ((int64_t)1 << 31) || p.ntiles >= ((int64_t)1 << 31)) return HQ_ERR_SHAPE;
    p.g_magic = 0xFFFFFFFFu / (uint32_t)G;
    p.gt_magic = 0xFFFFFFFFu / (uint32_t)cat_rotate_group_tiles(G);
    const int64_t tiles = p.ntiles;
    const int64_t cap = (int64_t)dev->sms * dev->cat_blocks_per_sm[fp4 ? 1 : 0];
    const int grid = (int)(tiles < cap ? tiles : cap);
    launch_cat_rotate(p, grid, (cudaStream_t)stream, fp4);
    return launch_status();
}

hq_status hq_cat_rotate_fp8(const void* a, int64_t a_row_stride, int a_width, const void* b,
                            int64_t b_row_stride, int b_width, int64_t M, int G, int hadamard_n,
                            uint8_t* out_fp8, float* scales, int scale_layout, int64_t scale_ld, float* amax_opt,
                            void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    return cat_rotate(a, a_row_stride, a_width, b, b_row_stride, b_width, M, G, hadamard_n, out_fp8, nullptr,
                      scales, scale_layout, scale_ld, amax_opt, stream, false);
}

size_t hq_cat_rotate_nvfp4_workspace_size(void) { return 0; }

hq_status hq_cat_rotate_nvfp4(const void* a, int64_t a_row_stride, int a_width, const void* b,
                              int64_t b_row_stride, int b_width, int64_t M, int G, int hadamard_n,
                              uint8_t* codes, uint8_t* block_sf, float* sdec, int scale_layout, int64_t scale_ld,
                              float* amax_opt, void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    return cat_rotate(a, a_row_stride, a_width, b, b_row_stride, b_width, M, G, hadamard_n, codes, block_sf, sdec,
                      scale_layout, scale_ld, amax_opt, stream, true);
}

hq_status hq_swiglu_fp8_k128(int mode, const void* in, int64_t M, int64_t K_out, uint8_t* out_fp8,
                             float* scales, float* amax_opt, void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    const bool ue8m0 = (mode & HQ_FP8_UE8M0) != 0;
    mode &= ~HQ_FP8_UE8M0;
    if (mode != HQ_ACT_NONE_BF16 && mode != HQ_ACT_NONE_F32 && mode != HQ_ACT_SWIGLU_F32) return HQ_ERR_UNSUPPORTED;
    if (M < 0 || K_out <= 0) return HQ_ERR_SHAPE;
    if (K_out % 128) return HQ_ERR_ALIGN;
    if (M == 0) return HQ_OK;
    if (!in || !out_fp8 || !scales) return HQ_ERR_NULL;
    if (!aligned16(in) || !aligned16(out_fp8) || !aligned4(scales) || !aligned4(amax_opt)) return HQ_ERR_ALIGN;
    const DeviceInfo* dev = device_info();
    if (!dev) return HQ_ERR_CUDA;
    K128Params p;
    p.in = in;
    p.K_out = K_out;
    p.ngroups = M * (K_out / 128);
    if (p.ngroups >= ((int64_t)1 << 31) || K_out / 128 >= ((int64_t)1 << 31)) return HQ_ERR_SHAPE;
    p.gpr_magic = 0xFFFFFFFFu / (uint32_t)(K_out / 128);
    p.out = out_fp8;
    p.scales = scales;
    p.ue8m0 = ue8m0 ? 1 : 0;
    p.amax = amax_opt;
    constexpr int warps_per_block = K128_THREADS / 32;
    const int64_t pairs = (p.ngroups + 1) / 2;
    const int64_t per_block = (int64_t)warps_per_block * K128_UNROLL;
    const int64_t blocks_needed = (pairs + per_block - 1) / per_block;
    const int64_t cap = (int64_t)dev->sms * 8;
    const int grid = (int)(blocks_needed < cap ? blocks_needed : cap);
    launch_k128(mode, p, grid, (cudaStream_t)stream);
    return launch_status();
}

hq_status hq_convert(int fmt, const float* in, uint8_t* out, int64_t n, void* stream) {
    if (fmt != HQ_FMT_E4M3 && fmt != HQ_FMT_E2M1) return HQ_ERR_UNSUPPORTED;
    if (n < 0) return HQ_ERR_SHAPE;
    if (n == 0) return HQ_OK;
    if (!in || !out) return HQ_ERR_NULL;
    const DeviceInfo* dev = device_info();
    if (!dev) return HQ_ERR_CUDA;
    const int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)dev->sms * 16;
    launch_convert(fmt, in, out, n, (int)(blocks < cap ? blocks : cap), (cudaStream_t)stream);
    return launch_status();
}

hq_status hq_convert_e2m1_sr(const float* in, const uint8_t* rnd, uint8_t* out, int64_t n, void* stream) {
    if (n < 0) return HQ_ERR_SHAPE;
    if (n == 0) return HQ_OK;
    if (!in || !rnd || !out) return HQ_ERR_NULL;
    const DeviceInfo* dev = device_info();
    if (!dev) return HQ_ERR_CUDA;
    const int64_t blocks = ((n + 3) / 4 + 255) / 256;
    const int64_t cap = (int64_t)dev->sms * 16;
    launch_convert_e2m1_sr(in, rnd, out, n, (int)(blocks < cap ? blocks : cap), (cudaStream_t)stream);
    return launch_status();
}

}  // extern "C"
