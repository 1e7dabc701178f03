/*
 * gl.h -- C ABI of the B200 grouped linear library (libgl.so).
 *
 * The operation is the grouped (mixture-of-experts) linear layer of
 * TransformerEngine's ``grouped_linear.py`` (ops/basic), ``GroupedLinear``:
 * the input rows are split by ``m_splits`` into G contiguous groups and group
 * i is multiplied by its own weight W_i, y_i = x_i W_i^T + b_i.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensors are row-major and contiguous; pointers named "device" point
 *    to memory of the current CUDA device; the caller owns every buffer.  The
 *    library never allocates device or pinned memory (the one scratch array
 *    of group_quantize_mxfp8_dbias_noalloc is part of the library's device
 *    image, not an allocation).
 *  - Shapes: x [M,K], W_i [N,K], b_i [N], y [y_rows,N], dy [M,N],
 *    dx [dx_rows,K], main_grad_i [N,K] fp32.  Group i owns rows
 *    [o[i], o[i+1]) of x, y, dy and dx, where o = offsets from gl_offsets.
 *  - Floating types: x, W, b, dy, y, dx are bf16 (2 bytes); main_grad is
 *    fp32.  Products accumulate in fp32 on the tensor cores.
 *  - When M == 0 (every group empty) the row operands (x, dy, y, dx) may
 *    be NULL; gl_fwd / gl_dgrad then do nothing and gl_wgrad only zeroes
 *    main_grad when it overwrites.
 *  - Every call is asynchronous on ``stream`` (a cudaStream_t; NULL is the
 *    legacy default stream) and never synchronises the host: split sizes stay
 *    on the device.
 *  - Host-checkable errors (null pointers, non-positive or unaligned sizes,
 *    buffers too small) return GL_ERR_INVALID / GL_ERR_UNSUPPORTED before
 *    anything is launched.  Data-dependent errors (negative split sizes, a
 *    split sum that does not match M, more rows than the output buffer holds)
 *    are detected on the device by gl_offsets, which writes them into the
 *    int32 device status word; every later kernel that is given the status
 *    word reads it first and writes nothing when it is non-zero.  A kernel
 *    that gives up on a bounded internal wait ORs GL_DEV_TIMEOUT into it.
 *    The caller reads the status word whenever it likes (for example with a
 *    device-to-host copy after the step).
 *  - Weights, biases and main_grad are passed as a gl_grouped: either one
 *    stacked [G, rows, cols] tensor (the single grouped parameter of
 *    ``GroupedLinear(single_grouped_weight=True)``) or a host array of G
 *    device pointers, one [rows, cols] tensor per group (``weight0`` ..
 *    ``weight{G-1}``).
 */
#ifndef GL_H_
#define GL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- host return codes -------------------------------------------------- */
typedef int gl_status;
#define GL_OK 0
#define GL_ERR_INVALID 1      /* bad argument; nothing was launched            */
#define GL_ERR_UNSUPPORTED 2  /* valid but outside the kernels' limits (sizes  */
                              /* not multiples of 8 / 32, too many groups ...) */
#define GL_ERR_CUDA 3         /* a CUDA runtime call or a launch failed        */

/* ---- device status word bits (int32, written by gl_offsets) ------------- */
#define GL_DEV_NEG_SPLIT 1    /* some m_splits[i] < 0                          */
#define GL_DEV_SUM_MISMATCH 2 /* sum(m_splits) != expect_rows                  */
#define GL_DEV_OUT_OVERFLOW 4 /* sum(m_splits) > out_rows                      */
#define GL_DEV_TIMEOUT 8      /* a kernel abandoned a bounded wait             */

/* ---- grouped parameter descriptor --------------------------------------- */
#define GL_STACKED 0   /* base -> [G, rows, cols], group stride rows*cols      */
#define GL_PER_GROUP 1 /* ptrs -> host array of G device pointers [rows,cols] */

typedef struct gl_grouped {
  int mode;                /* GL_STACKED or GL_PER_GROUP                      */
  const void* base;        /* GL_STACKED: device pointer                      */
  const void* const* ptrs; /* GL_PER_GROUP: host array of G device pointers   */
} gl_grouped;

/* Largest G accepted by any entry point. */
#define GL_MAX_GROUPS 4096

/* Library version (major*10000 + minor*100 + patch). */
int gl_version(void);

/* Human-readable text of a gl_status value. */
const char* gl_status_string(gl_status s);

/*
 * gl_gemm_opts -- per-call options of the six grouped GEMMs (gl_fwd,
 * gl_dgrad, gl_wgrad and their MXFP8 forms); pass NULL for the defaults.
 * They belong to the one call: the library keeps no mode between calls, so
 * callers on different threads never change each other's kernels.
 *
 *   tiles          GL_TILES_PAIR (0, the default): 256 x 256 output tiles
 *                  on pairs of CTAs (tcgen05 cta_group::2, one CTA per SM).
 *                  GL_TILES_SINGLE: 128 x 256 tiles on single CTAs.  Results
 *                  agree within rounding.
 *   wait_limit_us  bound, in microseconds, on each wait of the kernel's
 *                  load -> MMA -> epilogue pipeline that finds its barrier not
 *                  yet complete; 0 = the default (2 s), at most
 *                  GL_WAIT_LIMIT_MAX_US.  A wait that runs out ORs
 *                  GL_DEV_TIMEOUT into the status word and the kernel stops
 *                  early with its outputs incomplete; the waits that drain a
 *                  CTA's in-flight copies and MMAs before it exits keep their
 *                  2 s bound.
 *   flags          0, or GL_OPT_HOLD_LOADS: the load warp issues no copies,
 *                  so no stage ever lands, every pipeline wait runs out after
 *                  wait_limit_us, the call writes no output and sets
 *                  GL_DEV_TIMEOUT.  It exists to test that failure path
 *                  (status reported, context still usable) without a fault.
 * Values the header does not define give GL_ERR_INVALID.
 */
#define GL_TILES_PAIR 0
#define GL_TILES_SINGLE 1
#define GL_WAIT_LIMIT_MAX_US 2000000u
#define GL_OPT_HOLD_LOADS 1u
typedef struct gl_gemm_opts {
  int tiles;
  uint32_t wait_limit_us;
  uint32_t flags;
} gl_gemm_opts;

/*
 * gl_offsets -- group row offsets from the split sizes, on the device.
 *
 * Computes o[0] = 0 and o[i+1] = o[i] + m_splits[i] (int64, G+1 values),
 * the prefix sum with a leading zero that TransformerEngine's nvte_cumsum
 * produces ("Single parameter for GroupedLinear module", PR #2727), so that the
 * split sizes never travel to the host (``grouped_linear.py`` fuser_forward
 * reads them with ``split_sizes.tolist()``, a host synchronisation).
 *
 *   m_splits    device int64[G], group row counts
 *   G           1 <= G <= GL_MAX_GROUPS
 *   expect_rows rows of the input (M); sum(m) must equal it
 *   out_rows    rows of the output buffers (>= M); sum(m) must not exceed it
 *   offsets     device int64[G+1], written
 *   status      device int32, overwritten with the GL_DEV_* flags (0 = ok)
 * Errors: GL_ERR_INVALID for null pointers, G out of range, negative sizes.
 */
gl_status gl_offsets(const int64_t* m_splits, int G, int64_t expect_rows, int64_t out_rows,
                     int64_t* offsets, int32_t* status, void* stream);

/*
 * gl_fwd -- grouped forward, y_i = x_i W_i^T (+ b_i).
 *
 * ``grouped_linear.py`` (ops/basic) GroupedLinear docstring and fuser_forward
 * ("Perform GEMMs", one output, per-group bias).  The output may be a caller
 * buffer with more rows than M ("Add optional caller-provided output/grad-input
 * buffers", PR #3161): only the packed valid rows [0, M) that belong to a group
 * are written; rows [M, y_rows) are left untouched.
 *
 *   x        device bf16 [M, K]
 *   w        bf16 weights, [G, N, K] stacked or G pointers to [N, K]
 *   bias     NULL (no bias) or bf16 [G, N] stacked / G pointers to [N]
 *   offsets  device int64[G+1] from gl_offsets
 *   status   device int32 status word from gl_offsets (read; may get TIMEOUT)
 *   y        device bf16 [y_rows, N], y_rows >= M
 *   opts     NULL (defaults) or per-call options, see gl_gemm_opts
 * Limits: K % 8 == 0, N % 8 == 0 (16-byte row pitch), G <= GL_MAX_GROUPS.
 * The bias is added to the fp32 accumulator, then one round-to-nearest-even
 * conversion gives the bf16 output.
 */
gl_status gl_fwd(const void* x, gl_grouped w, const gl_grouped* bias, const int64_t* offsets,
                 int32_t* status, int G, int64_t M, int N, int K, void* y, int64_t y_rows,
                 const gl_gemm_opts* opts, void* stream);

/*
 * gl_dgrad -- grouped data gradient, dx_i = dy_i W_i.
 *
 * ``grouped_linear.py`` fuser_backward, "Perform dgrad GEMMs" (layout "NN",
 * one output).  Same caller-buffer rule as gl_fwd: rows [M, dx_rows) are not
 * written.
 *
 *   dy       device bf16 [M, N]
 *   w        bf16 weights as in gl_fwd
 *   dx       device bf16 [dx_rows, K], dx_rows >= M
 * Limits: K % 8 == 0, N % 8 == 0.
 */
gl_status gl_dgrad(const void* dy, gl_grouped w, const int64_t* offsets, int32_t* status, int G,
                   int64_t M, int N, int K, void* dx, int64_t dx_rows, const gl_gemm_opts* opts, void* stream);

/*
 * gl_wgrad -- grouped weight gradient into fp32 main_grad.
 *
 * ``grouped_linear.py`` fuser_backward, "Initialize grad weight buffers" and
 * "Perform wgrad GEMMs" (layout "NT"): dW_i = dy_i^T x_i.  With
 * accumulate != 0 it is added to main_grad (Megatron-style wgrad fusion);
 * with accumulate == 0 it overwrites main_grad (``overwrite_main_grad``), so
 * an empty group gets zeros.  With accumulate != 0 an empty group's
 * main_grad is not touched.
 *
 *   x, dy      device bf16 [M, K] and [M, N]
 *   main_grad  fp32 [G, N, K] stacked or G pointers to [N, K]
 * Limits: K % 8 == 0, N % 8 == 0.
 */
gl_status gl_wgrad(const void* x, const void* dy, const int64_t* offsets, int32_t* status, int G,
                   int64_t M, int N, int K, gl_grouped main_grad, int accumulate, const gl_gemm_opts* opts, void* stream);

/*
 * gl_dbias -- bias gradient: db_i[n] = sum of dy[r, n] over the rows r of
 * group i (``grouped_linear.py`` ops/basic fuser_backward: with a bias, each
 * split of grad_output is summed over its rows).  fp32 accumulation, one
 * round-to-nearest-even to bf16 per output; an empty group gets zeros.
 *
 *   dy       device bf16 [M, N] (rows packed by group)
 *   offsets  device int64[G+1] from gl_offsets
 *   status   device int32 status word (required); non-zero -> nothing written
 *   dbias    bf16 [G, N] stacked or G pointers to [N]; every element written
 * Limits: N % 8 == 0; dy 16-byte aligned.  Asynchronous on `stream`.
 */
gl_status gl_dbias(const void* dy, const int64_t* offsets, int32_t* status, int G, int64_t M, int N,
                   gl_grouped dbias, void* stream);

/*
 * group_quantize_mxfp8 -- MXFP8 (E4M3 codes, E8M0 block scales) cast of a
 * bf16 [rows, cols] tensor whose rows form G groups.
 *
 * ``grouped_linear.py`` (ops/basic): MXFP8 tensors hold E4M3 data and one
 * power-of-two scale per 32 elements, in a rowwise and a columnwise copy
 * (``_quantize_weights_mxfp8``); inputs and output gradients are quantized
 * per split (``split_quantize``); the grouped cast kernel is
 * ``group_quantize_mxfp8`` ("Improve device-init grouped linear module",
 * PR #3224).  For every block of 32 elements: amax = max |v|; the scale is
 * 2^e with e the smallest integer such that amax <= 448 * 2^e (clamped to
 * [-127, 127]; e = 0 when amax = 0), stored as the byte e + 127; each code is
 * v * 2^-e rounded to the nearest E4M3 value (ties to even, saturating).
 *
 *   src         device bf16 [rows, cols]
 *   row_offsets device int64[G+1] group row offsets, or NULL for G equal
 *               groups of rows/G rows (a stacked [G, rows/G, cols] weight)
 *   status      device int32 status word or NULL; non-zero -> nothing
 *               written (so a flag set on the device makes a captured weight
 *               cast a no-op on CUDA-graph replays); a load that never lands
 *               (2 s) sets GL_DEV_TIMEOUT
 *   codes_r     NULL or device u8 [rows, cols]: rowwise codes (blocks of 32
 *               along each row)
 *   scales_r    device u8 (required with codes_r), in scale_layout:
 *               GL_SCALES_ROWMAJOR: a [rows, cols/32] array;
 *               GL_SCALES_MMA (cols % 128 == 0): 512-byte atoms, atom (q, b)
 *               at byte (q * R + b) * 512 with R = ceil(rows/128), holding the
 *               scales of k-blocks 4q..4q+3 of rows 128b..128b+127; the scale
 *               of k-block 4q+j of row 128b+i sits at byte
 *               (i % 32) * 16 + (i / 32) * 4 + j of its atom (the tcgen05
 *               scale-factor layout, so the MXFP8 GEMMs copy atoms to tensor
 *               memory as they are).  R * (cols/128) atoms.
 *   codes_c     NULL or device u8 [rows, cols]: columnwise codes (blocks of 32
 *               rows along each column, restarting at every group's first
 *               row; a group's last block may be partial)
 *   scales_c    device u8 (required with codes_c), in scale_layout:
 *               GL_SCALES_ROWMAJOR: [S, cols], group i's block j in scale
 *               row sum_{l<i} ceil(m_l/32) + j, S <= ceil(rows/32) + G;
 *               GL_SCALES_MMA (cols % 128 == 0): group i owns k-groups
 *               T_i .. T_i + ceil(m_i/128) - 1, T_i = sum_{l<i} ceil(m_l/128);
 *               atom (T_i + t, c) at byte ((T_i + t) * (cols/128) + c) * 512
 *               holds blocks 4t..4t+3 of group i for columns 128c..128c+127,
 *               the scale of block 4t+j of column 128c+n at byte
 *               (n % 32) * 16 + (n / 32) * 4 + j.  At most
 *               (ceil(rows/128) + G) * (cols/128) atoms.
 *               In either MMA layout the bytes of rows (or blocks) that do not
 *               exist are not written.
 * gl_mxfp8_scale_bytes gives the bytes to allocate for a scale array.
 * Limits: cols % 32 == 0; rows/G integral when row_offsets is NULL.
 */
#define GL_SCALES_ROWMAJOR 0
#define GL_SCALES_MMA 1
gl_status group_quantize_mxfp8(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                               int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                               uint8_t* codes_c, uint8_t* scales_c, int scale_layout, void* stream);

/*
 * gl_mxfp8_scale_bytes -- bytes of a scale array written by
 * group_quantize_mxfp8 for a [rows, cols] source in G groups: rowwise
 * (colwise == 0) or columnwise (colwise != 0) scales in scale_layout.  For
 * columnwise scales with row offsets it is the bound that holds for any split
 * sizes.  Host-only, no device access; returns 0 for invalid arguments.
 */
size_t gl_mxfp8_scale_bytes(int64_t rows, int cols, int G, int colwise, int scale_layout);

/*
 * group_quantize_mxfp8_dbias -- group_quantize_mxfp8 of a ragged bf16 dy
 * that also writes its bias gradient from the same read of dy:
 * db_i[n] = sum of dy[r, n] over the rows r of group i (``grouped_linear.py``
 * ops/basic fuser_backward with MXFP8 quantizers: grad_output is quantized per
 * split and, with a bias, each split is summed over its rows; doing both in
 * one pass saves a full read of dy).
 *
 * Each 32-row block of a group adds its rows per column in fp32 in a fixed
 * order and stores one fp32 partial per (block, column) in the workspace; a
 * second kernel adds each group's partials in a fixed order and rounds once
 * to bf16 (round-to-nearest-even).  The result is deterministic; it agrees
 * with gl_dbias to fp32 rounding (the two add in different orders).  An
 * empty group gets zeros.
 *
 *   src .. scale_layout   as for group_quantize_mxfp8; row_offsets required
 *   status      device int32 status word (required); non-zero -> nothing
 *               written
 *   dbias       bf16 [G, cols] stacked or G pointers to [cols]; every element
 *               written
 *   workspace   device scratch of workspace_bytes >= gl_dbias_workspace_bytes
 *               (rows, cols, G), 256-byte aligned, owned by the caller; its
 *               contents on entry do not matter and it may be reused once the
 *               call's work on `stream` has finished
 * Errors: GL_ERR_INVALID for a NULL row_offsets / status / workspace or a
 * workspace that is too small; GL_ERR_UNSUPPORTED for a misaligned
 * workspace; otherwise those of group_quantize_mxfp8.  Asynchronous on
 * `stream` (two launches).
 */
gl_status group_quantize_mxfp8_dbias(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                                     int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                                     uint8_t* codes_c, uint8_t* scales_c, int scale_layout, gl_grouped dbias,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * gl_dbias_workspace_bytes -- workspace bytes for group_quantize_mxfp8_dbias:
 * int64[G+1] block offsets (padded to 256 bytes) + fp32
 * [ceil(rows/32) + G, cols] partials.  Host-only; 0 for invalid arguments.
 */
size_t gl_dbias_workspace_bytes(int64_t rows, int cols, int G);

/*
 * group_quantize_mxfp8_dbias_noalloc -- group_quantize_mxfp8_dbias for
 * callers that cannot allocate device memory where they call it (their
 * memory belongs to another runtime's pool and they are handed no allocator;
 * a cudaMalloc there would also synchronise the device).  This entry point
 * has no counterpart in the pages: it exists for those callers only.
 *
 * It takes no workspace: its scratch is one fixed 16 MiB array in the
 * library's own device memory, which every GPU that loads the library holds
 * until the process exits.  Every other argument, and the results, are those
 * of group_quantize_mxfp8_dbias.
 *   - gl_dbias_workspace_bytes(rows, cols, G), which is
 *     256 * ceil(8 (G + 1) / 256) + 4 * cols * (ceil(rows / 32) + G),
 *     must be at most 16 MiB (16777216): e.g. up to 9088 rows of 14336
 *     columns in 8 groups, or 32000 rows of 4096 columns in at most 23
 *     groups.  Larger calls return GL_ERR_UNSUPPORTED and touch nothing;
 *     argument errors are reported first, as group_quantize_mxfp8_dbias
 *     reports them.
 *   - The first call on each device looks up the array's device address
 *     (with that device current) and may load the library's device code;
 *     make that first call before any stream capture.  The address is kept
 *     with the identity of its CUDA context, so after a device reset the next
 *     call looks it up again.  GL_ERR_CUDA if the address cannot be obtained
 *     (the runtime's last-error state is cleared, so later calls are not
 *     affected).
 *   - Every call on a device uses the same array: calls whose work can
 *     overlap on the GPU (other streams, or other threads' streams) race
 *     and corrupt each other's results; order them on one stream or with
 *     events.  No part of the array needs to start at zero.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
gl_status group_quantize_mxfp8_dbias_noalloc(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                                             int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                                             uint8_t* codes_c, uint8_t* scales_c, int scale_layout,
                                             gl_grouped dbias, void* stream);

/*
 * MXFP8 grouped GEMMs -- the three products of gl_fwd / gl_dgrad / gl_wgrad
 * on MXFP8 operands (E4M3 codes, E8M0 scale per 32 contraction elements, as
 * written by group_quantize_mxfp8), computed as
 *     sum over k of (q_a * 2^(s_a - 127)) * (q_b * 2^(s_b - 127))
 * with fp32 accumulation on the block-scaled tensor cores (``grouped_linear.py``
 * fuser_forward / fuser_backward with MXFP8 quantizers: x and W rowwise for
 * fprop, dy rowwise and W columnwise for dgrad, x and dy columnwise for wgrad).
 * Outputs, offsets, status, caller buffers and main_grad behave exactly as in
 * the bf16 entry points.
 *
 * Operand forms (all device memory, produced by group_quantize_mxfp8; every
 * scale array in the GL_SCALES_MMA layout):
 *   rowwise codes    u8 [rows, cols] (x, dy: [M, K] / [M, N]; W: [G, N, K])
 *   rowwise scales   x: rows M, cols K; dy: rows M, cols N; stacked W: rows
 *                    G*N, cols K; per-group W: rows N, cols K
 *   columnwise codes u8 [rows, cols] (x_c [M, K], dy_c [M, N], W_c [G, N, K])
 *   columnwise scales x_c / dy_c quantized with the group offsets; stacked
 *                    W_c as G equal groups of N rows; per-group W_c as one
 *                    group of N rows
 * Limits: N % 128 == 0, K % 128 == 0, G <= GL_MAX_GROUPS_MXFP8.
 */
#define GL_MAX_GROUPS_MXFP8 2048

gl_status gl_fwd_mxfp8(const uint8_t* x_codes, const uint8_t* x_scales, gl_grouped w_codes,
                       gl_grouped w_scales, const gl_grouped* bias, const int64_t* offsets,
                       int32_t* status, int G, int64_t M, int N, int K, void* y, int64_t y_rows,
                       const gl_gemm_opts* opts, void* stream);

gl_status gl_dgrad_mxfp8(const uint8_t* dy_codes, const uint8_t* dy_scales, gl_grouped w_codes_c,
                         gl_grouped w_scales_c, const int64_t* offsets, int32_t* status, int G,
                         int64_t M, int N, int K, void* dx, int64_t dx_rows, const gl_gemm_opts* opts, void* stream);

gl_status gl_wgrad_mxfp8(const uint8_t* x_codes_c, const uint8_t* x_scales_c, const uint8_t* dy_codes_c,
                         const uint8_t* dy_scales_c, const int64_t* offsets, int32_t* status, int G,
                         int64_t M, int N, int K, gl_grouped main_grad, int accumulate, const gl_gemm_opts* opts, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GL_H_ */
