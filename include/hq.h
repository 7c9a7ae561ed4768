/*
 * hq.h -- C ABI of the hq library: Hadamard rotation fused with block-scaled
 * low-precision quantization (NVFP4 and FP8 E4M3) on NVIDIA B200 (sm_100a).
 *
 * Conventions for every call below:
 *  - Pointers are CUDA device pointers owned by the caller, unless a comment
 *    says "host".  The library allocates no memory, never synchronizes the
 *    stream (hq_get_error excepted) and reads no environment variables.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *  - Every argument is checked before anything is launched; a violation
 *    returns a nonzero hq_status and leaves all outputs untouched.  There is no
 *    fallback path: an unsupported request is an error.
 *  - Calls are asynchronous: a status of HQ_OK means the work was enqueued.
 *  - BF16 tensors are passed as their 16-bit patterns, FP8 E4M3 codes as
 *    bytes, NVFP4 E2M1 codes two per byte (element 2k in the low nibble).
 *
 * Sources for the operations (page titles):
 *  [GRP] TransformerEngine PR #2564 "[NVFP4][MOE] Bug Fix for NVFP4 Grouped
 *        Quant": the grouped row-cast / column-Hadamard-transform-cast kernel
 *        over MoE split sections, and its caller-provided 4-byte tile
 *        scheduler workspace (replacing a per-call cudaMallocAsync), plus the
 *        reviewers' request for a workspace-size query.
 *  [FUS] TransformerEngine PR #2555 review comments: split_section % 128
 *        fusion rule, rht_matrix, rowwise-only output needs no RHT, the RHT'd
 *        columnwise output is the transposed [cols, rows] tensor.
 *  [DSA] TensorRT-LLM PR #15158 "[#13061][bugfix] Add rotate_activation to DSA
 *        fused_cat_fp8 path": cat([pe, nope]) -> Hadamard rotation ->
 *        fp8_quantize_1x128, scales transposed.
 *  [QMOE] onnxruntime PR #33644 (QMoE activation_quantization="dynamic_fp8"),
 *        Description: K128 groups, saturating nearest-even E4M3,
 *        max(amax, 1e-10) * float32(1/448) scales, FP32 SiLU/SwiGLU before
 *        the second quantizer, explicit errors instead of fallbacks.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hq_status {
    HQ_OK = 0,
    HQ_ERR_NULL = 1,        /* a required pointer is NULL */
    HQ_ERR_SHAPE = 2,       /* sizes negative, inconsistent or too large */
    HQ_ERR_ALIGN = 3,       /* pointer/stride not 16-byte aligned, or a size
                               not a multiple of the required block */
    HQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the query */
    HQ_ERR_UNSUPPORTED = 5, /* unknown flag, mode, layout or transform size */
    HQ_ERR_CUDA = 6,        /* the CUDA runtime reported an error */
    HQ_ERR_TIMEOUT = 7      /* a bounded device-side wait gave up */
} hq_status;

/* hq_group_rht_quant flags */
#define HQ_ROWWISE 1u      /* rowwise NVFP4 output (plain cast along K) */
#define HQ_COLWISE 2u      /* columnwise NVFP4 output (RHT16 along M, transposed) */
#define HQ_ROW_RHT 4u      /* with HQ_ROWWISE: the rowwise output casts the RHT16
                              of each 16-column block along K instead of x */
#define HQ_ROW_SR 32u      /* hq_group_rht_quant_sr: rowwise codes round stochastically */
#define HQ_COL_SR 64u      /* hq_group_rht_quant_sr: columnwise codes round stochastically */
#define HQ_AMAX_GIVEN 16u  /* amax_row / amax_col are inputs: the caller's section
                              amax values; one pass, no amax computation */
#define HQ_SF_SWIZZLED 128u /* row_sf and each section's col_sf block in the
                              interleaved 128 x 4 tiles that block-scaled
                              tcgen05 MMAs read (see below) */
#define HQ_TWO_PASS 8u     /* schedule: amax pass and cast pass as two launches
                              (without HQ_ROW_RHT the amax pass is a streaming
                              kernel of its own) instead of one launch in which
                              each section's cast follows its amax while the
                              rows are still in L2.  A call whose only
                              non-empty section fills the grid at least once,
                              without HQ_ROW_RHT, takes two launches without
                              the flag too (its casts wait for the whole amax
                              pass either way).  Results are identical. */

/* hq_cat_rotate_fp8 scale layouts */
#define HQ_SCALE_ROWMAJOR 0   /* scale of group (t, g) at scales[t * G + g] */
#define HQ_SCALE_TRANSPOSED 1 /* scale of group (t, g) at scales[g * scale_ld + t] */

/*
 * Scale formats for GEMMs that consume the outputs directly (the TensorRT-LLM
 * PR #15158 review asks for a use_ue8m0 option of the 1x128 quantizer;
 * DeepGEMM issue #320 discusses the tcgen05 data-path layouts of scales).
 *
 * HQ_FP8_UE8M0, added to scale_layout of hq_cat_rotate_fp8 or to mode of
 * hq_swiglu_fp8_k128: each group's FP32 scale s is rounded up to the smallest
 * power of two not below it, and the codes are E4M3(y / that power of two).
 * The stored scale is that FP32 power of two; its UE8M0 byte is the binary32
 * exponent field (bits 30..23).
 *
 * HQ_SF_SWIZZLED (hq_group_rht_quant* flags; added to scale_layout of
 * hq_cat_rotate_nvfp4): E4M3 block scales in tiles of 128 rows x 4 columns
 * of the [rows, cols] scale matrix, 512 bytes each, stored tile-row major;
 * element (r, c) at byte
 *   ((r / 128) * (cols / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.
 * The grouped cast's row_sf is [M, K/16]; each section's col_sf block is
 * [K, M_s/16] at its usual byte K * r0 / 16 (every dimension a multiple of the
 * tile: a permutation of the plain layout, same size).  The FP4 DSA call's
 * block_sf is [M, G * 8] and needs M % 128 == 0 (HQ_ERR_ALIGN otherwise).
 */
#define HQ_FP8_UE8M0 256

/* hq_swiglu_fp8_k128 modes (+ HQ_FP8_UE8M0) */
#define HQ_ACT_NONE_BF16 0  /* in: BF16 [M, K_out] */
#define HQ_ACT_NONE_F32 1   /* in: FP32 [M, K_out] */
#define HQ_ACT_SWIGLU_F32 2 /* in: FP32 [M, 2*K_out], gate = cols [0, K_out),
                               up = cols [K_out, 2*K_out); value SiLU(gate)*up */

/* hq_convert formats */
#define HQ_FMT_E4M3 0 /* one E4M3 code per output byte */
#define HQ_FMT_E2M1 1 /* one E2M1 code per output byte (low nibble) */

#define HQ_MAX_SECTIONS 256

/* Library version, (major << 16) | minor. */
int hq_version(void);

/* Static description of a status code. */
const char *hq_status_string(hq_status s);

/*
 * Workspace bytes hq_group_rht_quant needs for `num_sections` sections
 * (1 <= num_sections <= HQ_MAX_SECTIONS; 0 otherwise).  The first 4 bytes
 * are the tile-scheduler counter of [GRP]; an exit count, an error word, an
 * abort flag, then per section an amax accumulator per direction and a count
 * of its completed amax tiles follow (16 + 12 * S bytes, rounded up to 256).
 * The size query is the reviewers' proposal in [GRP].
 */
size_t hq_group_rht_quant_workspace_size(int num_sections);

/*
 * Put a workspace into its rest state (all zero).  Call once after
 * allocating it (an enqueued memset on `stream`).  Every hq_group_rht_quant
 * call leaves the workspace in the rest state again, so no per-call memset
 * is needed.  Two calls that share one workspace must not overlap in time
 * (same stream, or ordered by events).
 * Errors: HQ_ERR_NULL, HQ_ERR_ALIGN (ws not 16-byte aligned), HQ_ERR_CUDA.
 */
hq_status hq_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Read and clear the workspace's device error word.  Synchronizes `stream`.
 * *err_out (host) receives 0, or HQ_ERR_TIMEOUT if a bounded device wait of
 * an earlier call gave up (that call's outputs are then incomplete).
 */
hq_status hq_get_error(void *ws, size_t ws_bytes, uint32_t *err_out, void *stream);

/*
 * Grouped random-Hadamard-transform + NVFP4 cast over MoE split sections
 * [GRP], [FUS].
 *
 *  x          BF16 [M, K] row major.  16-byte aligned.
 *  M, K       rows, columns.  K > 0 and K % 128 == 0.
 *  split_rows HOST int64 [S]: rows per section, each >= 0 and a multiple of
 *             128 ([FUS] fusion rule), summing to M.  Empty sections allowed.
 *  S          number of sections, 1 <= S <= HQ_MAX_SECTIONS.
 *  sign_mask  the random sign vector of the 16-point RHT: bit i set means
 *             sigma_i = -1 for position i of each 16-row block (and, with
 *             HQ_ROW_RHT, of each 16-column block of a row).
 *  flags      HQ_ROWWISE | HQ_COLWISE (at least one), optionally HQ_ROW_RHT
 *             (only with HQ_ROWWISE; the grouped-quant pages speak of the RHT
 *             on both outputs, their fused kernel rotates only the columns),
 *             HQ_AMAX_GIVEN, HQ_TWO_PASS (ignored with HQ_AMAX_GIVEN) and
 *             HQ_SF_SWIZZLED.
 *
 * For section s (rows [r0, r0 + M_s)) and each requested direction:
 *   A_s = max |v| over the section's values (v = x rowwise, the RHT16 output
 *   along K with HQ_ROW_RHT; v = RHT16 output columnwise), or with
 *   HQ_AMAX_GIVEN the caller's amax_*[s]; S_enc = 2688 / A_s (1 when A_s is
 *   not positive or the quotient is not finite),
 *   sdec = 1 / S_enc; for each block of 16 values along the quantized
 *   direction: sf = E4M3((a_b / 6) * S_enc), code_i = E2M1(v_i * S_enc / sf)
 *   (0 when sf == 0); saturating round-to-nearest-even conversions.
 *   RHT16 of a block: v = 0.25 * H16 * diag(sigma) * x, H16 the Sylvester
 *   Hadamard matrix.
 *
 * Outputs (device; each 16-byte aligned; amax/sdec 4-byte aligned):
 *  row_codes  uint8 [M, K/2]     rowwise E2M1 codes          (HQ_ROWWISE)
 *  row_sf     uint8 [M, K/16]    rowwise E4M3 block scales   (HQ_ROWWISE)
 *  col_codes  uint8 [M*K/2]      per section s: [K, M_s/2] at byte K*r0/2
 *  col_sf     uint8 [M*K/16]     per section s: [K, M_s/16] at byte K*r0/16
 *  amax_row, sdec_row  float [S] (HQ_ROWWISE)
 *  amax_col, sdec_col  float [S] (HQ_COLWISE)
 *  With HQ_AMAX_GIVEN amax_row / amax_col are inputs (device, read only, set
 *  before the call in stream order) and only sdec_* is written; the call then
 *  reads x once (the cast pass alone).
 *  Pointers of a direction not requested may be NULL, and so may the code
 *  and block-scale buffers when M == 0.
 *
 *  ws, ws_bytes  caller workspace, >= hq_group_rht_quant_workspace_size(S),
 *                16-byte aligned, in the rest state (hq_workspace_init).
 * Errors: HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_ALIGN, HQ_ERR_WORKSPACE,
 *         HQ_ERR_UNSUPPORTED, HQ_ERR_CUDA.
 * Inputs must be finite (NaN/inf are outside the NVFP4 contract).
 */
hq_status hq_group_rht_quant(const void *x, int64_t M, int64_t K,
                             const int64_t *split_rows, int S, uint16_t sign_mask,
                             unsigned flags,
                             uint8_t *row_codes, uint8_t *row_sf,
                             uint8_t *col_codes, uint8_t *col_sf,
                             float *amax_row, float *amax_col,
                             float *sdec_row, float *sdec_col,
                             void *ws, size_t ws_bytes, void *stream);

/*
 * hq_group_rht_quant with stochastic rounding of the E2M1 codes (the grouped
 * pages' review discusses the Philox generator and deterministic offsets of
 * stochastic rounding for this cast; it gives no rounding rule).  flags may
 * add HQ_ROW_SR (with HQ_ROWWISE) and HQ_COL_SR (with HQ_COLWISE); block
 * scales, amax and sdec are as without.  A code rounds |v| (v = value *
 * encode factor, as for nearest-even) up to the next E2M1 value iff its
 * random byte r < floor(256 f), f the fraction of |v| above the E2M1 value
 * below it in grid steps (0.5 below 2, 1 below 4, 2 below 6); |v| >= 6
 * saturates; the sign is kept.  r of output element e (its index in
 * row_codes' [M, K] order, or in col_codes' element order) is byte
 * offset + e of the stream of bytes B_i = byte (i % 4) of word (i / 4) % 4
 * of Philox4x32-10(counter = {i / 16 low 32 bits, i / 16 high 32 bits, 0, 0},
 * key = {k low, k high}), k = seed for rowwise codes and seed + 1 for
 * columnwise codes, so results depend only on (seed, offset), not on the
 * launch.  offset must be a multiple of 16 (HQ_ERR_ALIGN).  Other arguments,
 * outputs and errors as hq_group_rht_quant (which rejects the SR flags).
 */
hq_status hq_group_rht_quant_sr(const void *x, int64_t M, int64_t K,
                                const int64_t *split_rows, int S, uint16_t sign_mask,
                                unsigned flags, uint64_t seed, uint64_t offset,
                                uint8_t *row_codes, uint8_t *row_sf,
                                uint8_t *col_codes, uint8_t *col_sf,
                                float *amax_row, float *amax_col,
                                float *sdec_row, float *sdec_col,
                                void *ws, size_t ws_bytes, void *stream);

/*
 * The grouped cast with x and every output in HOST memory: the rows are
 * copied to the device, cast and copied back in groups of whole sections, so
 * the copies of one group overlap the cast of the next and the copies in the
 * other direction (page-locked host buffers are needed for the overlap;
 * pageable ones give the same results, copied without overlap).  The codes
 * and scales are those of hq_group_rht_quant_sr on the whole tensor (without
 * HQ_ROW_SR / HQ_COL_SR, those of hq_group_rht_quant); a section's amax never
 * crosses groups, and the random byte streams keep their element indices.
 *  x, row_codes, row_sf, col_codes, col_sf, amax_row, amax_col, sdec_row,
 *  sdec_col      host buffers with the layouts of hq_group_rht_quant; with
 *                HQ_AMAX_GIVEN amax_* are read (host) and copied in.
 *  seed, offset  as hq_group_rht_quant_sr (ignored without the SR flags).
 *  dev_buf, dev_buf_bytes  device staging memory, >=
 *                hq_group_rht_quant_host_device_bytes(M, K, S), 256-byte
 *                aligned; it holds x, the outputs and the workspace (kept in
 *                its rest state by the calls; zero it once before the first).
 *  groups        section groups (1..HQ_HOST_MAX_GROUPS); 0 picks 16.  Groups
 *                are cut at section boundaries only (a section's amax needs
 *                all its rows), so S sections give at most S groups and a
 *                single section is copied, cast and copied back in sequence.
 *  stream        the cast runs here; the call is ordered after the work
 *                already on it, and work enqueued on it afterwards runs after
 *                the last copy back (synchronize it before reading outputs).
 *  h2d_stream, d2h_stream  two further streams for the copies (distinct from
 *                stream and from each other).
 * A fixed set of CUDA events per device is created on the first call and
 * kept for the life of the process; calls from several host threads are
 * serialized while they enqueue.
 * Errors: as hq_group_rht_quant_sr, HQ_ERR_WORKSPACE when dev_buf is too
 *         small, HQ_ERR_UNSUPPORTED for a bad group count or stream set.
 *         Argument errors are found before anything is enqueued; a CUDA
 *         error after the first group was enqueued returns HQ_ERR_CUDA with
 *         the earlier groups' copies and casts still in flight.
 */
#define HQ_HOST_MAX_GROUPS 32
size_t hq_group_rht_quant_host_device_bytes(int64_t M, int64_t K, int S);
hq_status hq_group_rht_quant_host(const void *x, int64_t M, int64_t K,
                                  const int64_t *split_rows, int S, uint16_t sign_mask,
                                  unsigned flags, uint64_t seed, uint64_t offset,
                                  uint8_t *row_codes, uint8_t *row_sf,
                                  uint8_t *col_codes, uint8_t *col_sf,
                                  float *amax_row, float *amax_col,
                                  float *sdec_row, float *sdec_col,
                                  void *dev_buf, size_t dev_buf_bytes, int groups,
                                  void *stream, void *h2d_stream, void *d2h_stream);

/*
 * hq_group_rht_quant without a caller workspace, for callers that cannot
 * allocate device memory where they quantize (plugins whose host framework
 * owns all device memory, allocation-free runtimes).  The paper has no
 * counterpart.
 *
 * Arguments, outputs and errors are those of hq_group_rht_quant without
 * ws / ws_bytes.  The scratch words live in a fixed array inside the library
 * (3328 bytes, room for HQ_MAX_SECTIONS = 256 sections; S > 256 returns
 * HQ_ERR_SHAPE), present on every GPU that loads the library until the
 * process exits.  The call allocates nothing: it clears the array with an
 * enqueued memset and launches the kernel.  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress) and so should come
 * before any stream capture; a lookup that fails returns HQ_ERR_CUDA and is
 * tried again by the next call.  All calls on a device share the one array:
 * calls that overlap on the GPU (different streams without ordering) race
 * and give wrong results.  A bounded device wait that gives up is not
 * reported by this entry point (there is no workspace to read it from).
 */
hq_status hq_group_rht_quant_noalloc(const void *x, int64_t M, int64_t K,
                                     const int64_t *split_rows, int S, uint16_t sign_mask,
                                     unsigned flags,
                                     uint8_t *row_codes, uint8_t *row_sf,
                                     uint8_t *col_codes, uint8_t *col_sf,
                                     float *amax_row, float *amax_col,
                                     float *sdec_row, float *sdec_col, void *stream);

/*
 * Concatenate -> 128-point Hadamard rotation -> FP8 E4M3 1x128 quantization
 * [DSA] (the DSA indexer's q/k preparation), with the scale rule of [QMOE].
 *
 *  a          BF16; element j of group g of row t is
 *             a[t * a_row_stride + g * a_width + j], 0 <= j < a_width.
 *  b          BF16 or NULL (when b_width == 0); same indexing with b_*.
 *             The 128-vector of (t, g) is a-part followed by b-part
 *             ([pe, nope]); a_width + b_width == 128, both multiples of 8.
 *  M, G       rows (tokens) and groups (heads) per row.
 *  hadamard_n 128 (rotate by H128 / sqrt(128), Sylvester order) or 0 (none).
 *  out_fp8    uint8 [M, G*128] codes: (t, g, j) at (t * G + g) * 128 + j.
 *  scales     float: group scale s = max(amax, 1e-10) * float32(1/448),
 *             codes = E4M3(y / s) (IEEE division, saturating RNE).
 *             scale_layout HQ_SCALE_ROWMAJOR: [M, G] (scale_ld ignored);
 *             HQ_SCALE_TRANSPOSED: [G, scale_ld], scale_ld >= M; either may
 *             add HQ_FP8_UE8M0.
 *  amax_opt   float, NULL or each group's amax = max |y| (y the rotated
 *             128-vector), in the scales' layout; 4-byte aligned.
 *  ws, ws_bytes  unused: hq_cat_rotate_fp8_workspace_size() is 0 (may be
 *             NULL / 0).
 * Alignment: a, b, out 16 bytes; strides multiples of 8 elements.
 * Errors: HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED,
 *         HQ_ERR_CUDA.
 */
hq_status hq_cat_rotate_fp8(const void *a, int64_t a_row_stride, int a_width,
                            const void *b, int64_t b_row_stride, int b_width,
                            int64_t M, int G, int hadamard_n,
                            uint8_t *out_fp8, float *scales, int scale_layout,
                            int64_t scale_ld, float *amax_opt,
                            void *ws, size_t ws_bytes, void *stream);

/* Workspace bytes hq_cat_rotate_fp8 needs: 0 (none). */
size_t hq_cat_rotate_fp8_workspace_size(void);

/*
 * The DSA indexer prep with an NVFP4 output (the FP4 path [DSA] names as
 * lacking the rotation; the pages give no FP4 format, the reading is the
 * two-level NVFP4 scheme of hq_group_rht_quant with the 128-vector in place
 * of a section): concat and optional rotation exactly as hq_cat_rotate_fp8,
 * then for each vector (t, g) with rotated values y:
 *   A = max |y| over the vector, S_enc = 2688 / A (1 when A is 0 or the
 *   quotient is not finite); per block of 16 consecutive values
 *   sf = E4M3((a_b / 6) * S_enc), code_i = E2M1(y_i * S_enc / sf) (0 when
 *   sf == 0); saturating round-to-nearest-even conversions.
 *
 *  a, b, a_width, b_width, strides, M, G, hadamard_n, scale_layout,
 *  scale_ld   as hq_cat_rotate_fp8.
 *  codes      uint8 [M, G*64]: vector (t, g) at (t * G + g) * 64, two E2M1
 *             codes per byte, element 2k in the low nibble.  16-byte aligned.
 *  block_sf   uint8 [M, G*8] E4M3 block scales.
 *  sdec       float, per vector 1 / S_enc, in the FP8 scales' layouts
 *             ([M, G] or [G, scale_ld]).  4-byte aligned.
 *  amax_opt   float, NULL or A per vector, in the same layout.
 *  ws, ws_bytes  unused: hq_cat_rotate_nvfp4_workspace_size() is 0.
 * Errors: HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED,
 *         HQ_ERR_CUDA.  Inputs must be finite.  scale_layout may add
 *         HQ_SF_SWIZZLED (block_sf in the interleaved tiles, M % 128 == 0).
 */
hq_status hq_cat_rotate_nvfp4(const void *a, int64_t a_row_stride, int a_width,
                              const void *b, int64_t b_row_stride, int b_width,
                              int64_t M, int G, int hadamard_n,
                              uint8_t *codes, uint8_t *block_sf, float *sdec,
                              int scale_layout, int64_t scale_ld, float *amax_opt,
                              void *ws, size_t ws_bytes, void *stream);

/* Workspace bytes hq_cat_rotate_nvfp4 needs: 0 (none). */
size_t hq_cat_rotate_nvfp4_workspace_size(void);

/*
 * QMoE dynamic FP8 activation quantizer [QMOE]: each row of K_out values is
 * split into consecutive groups of 128; each group gets the FP8 rule above.
 *  mode     HQ_ACT_NONE_BF16, HQ_ACT_NONE_F32 or HQ_ACT_SWIGLU_F32 (the value
 *           quantized is SiLU(gate) * up computed in FP32, SiLU(g) =
 *           g / (1 + exp(-g)), with no narrower rounding in between); any
 *           mode may add HQ_FP8_UE8M0.
 *  in       see the modes; row stride K_out (or 2*K_out for SwiGLU).
 *  out_fp8  uint8 [M, K_out];  scales float [M, K_out/128] row major.
 *  amax_opt float [M, K_out/128] or NULL: each group's amax = max |y|.
 *  K_out    multiple of 128.   ws, ws_bytes unused:
 *           hq_swiglu_fp8_k128_workspace_size() is 0 (may be NULL / 0).
 * Alignment: in and out 16 bytes, scales and amax_opt 4 bytes.
 * Errors: HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED,
 *         HQ_ERR_CUDA.
 */
hq_status hq_swiglu_fp8_k128(int mode, const void *in, int64_t M, int64_t K_out,
                             uint8_t *out_fp8, float *scales, float *amax_opt,
                             void *ws, size_t ws_bytes, void *stream);

/* Workspace bytes hq_swiglu_fp8_k128 needs: 0 (none). */
size_t hq_swiglu_fp8_k128_workspace_size(void);

/*
 * Element-wise conversion of FP32 values with the library's own device
 * conversion routines (the ones every kernel above uses): E4M3 (saturating,
 * nearest even) or E2M1 (one nibble per byte).  n >= 0; in and out may have
 * any alignment.
 * Errors: HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_UNSUPPORTED, HQ_ERR_CUDA.
 */
hq_status hq_convert(int fmt, const float *in, uint8_t *out, int64_t n, void *stream);

/*
 * Element-wise stochastic E2M1 conversion with the device routine of
 * hq_group_rht_quant_sr: out[i] (low nibble) is the code of in[i] rounded
 * with random byte rnd[i] by that call's rule (|v| up to the next E2M1 value
 * iff rnd[i] < floor(256 f); |v| >= 6 saturates; sign kept).  n >= 0; any
 * alignment.  Errors: HQ_ERR_NULL, HQ_ERR_SHAPE, HQ_ERR_CUDA.
 */
hq_status hq_convert_e2m1_sr(const float *in, const uint8_t *rnd, uint8_t *out, int64_t n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
