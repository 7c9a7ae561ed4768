// hq_noalloc.cu -- hq_group_rht_quant_noalloc: the grouped RHT16 + NVFP4
// cast for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they quantize: plugins whose host framework owns all device
// memory, or allocation-free inference runtimes.  For them this entry point keeps the
// grouped kernel's scratch words (tile counter, per-section amax accumulators
// and completion counts) in a fixed array of the library itself instead of a
// caller workspace.  The paper has no counterpart; it is an addition of this
// library.
#include <mutex>

#include "hq_internal.h"

namespace {

// Scratch for up to HQ_MAX_SECTIONS (256) sections: the workspace size the
// grouped call asks for at 256 sections (3088 bytes rounded up to 3328, the
// size the call clears), held on every GPU that
// loads the library until the process exits.
constexpr int kNoallocWords = 3328 / 4;
static_assert(((4 * (hq::NV_WS_HEADER + 3 * HQ_MAX_SECTIONS) + 255) & ~255) <= 3328,
              "scratch too small");
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoallocWords];

constexpr int kMaxDevices = 64;
uint32_t* g_scratch_ptr[kMaxDevices];  // published only after a successful lookup
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// the symbol is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, with that device current.  A successful lookup is
// kept for the device; a failed one (e.g. made during a stream capture) is
// not cached, so a later call tries again, and its error is cleared from the
// runtime so that it is not reported by an unrelated later call.
uint32_t* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) {
            g_scratch_ptr[dev] = static_cast<uint32_t*>(p);
        } else {
            (void)cudaGetLastError();
            return nullptr;
        }
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" hq_status hq_group_rht_quant_noalloc(const void* x, int64_t M, int64_t K, const int64_t* split_rows,
                                                int S, uint16_t sign_mask, unsigned flags, uint8_t* row_codes,
                                                uint8_t* row_sf, uint8_t* col_codes, uint8_t* col_sf,
                                                float* amax_row, float* amax_col, float* sdec_row,
                                                float* sdec_col, void* stream) {
    if (S < 1 || S > HQ_MAX_SECTIONS) return HQ_ERR_SHAPE;  // beyond the scratch array's size
    uint32_t* scratch = scratch_on_current_device();
    if (!scratch) return HQ_ERR_CUDA;
    const size_t bytes = hq_group_rht_quant_workspace_size(S);
    // The array keeps the previous call's contents: start from zero.
    if (cudaMemsetAsync(scratch, 0, bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) return HQ_ERR_CUDA;
    return hq_group_rht_quant(x, M, K, split_rows, S, sign_mask, flags, row_codes, row_sf, col_codes, col_sf,
                              amax_row, amax_col, sdec_row, sdec_col, scratch, bytes, stream);
}
