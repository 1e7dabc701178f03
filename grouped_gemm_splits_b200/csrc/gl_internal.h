// gl_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gl.h"

namespace gl {

// Number of SMs of the current device (cached per device).
int num_sms();

// cuTensorMapEncodeTiled through the runtime's driver entry point.  Returns
// false if the driver rejected the map.  dims/strides are innermost first;
// strides_bytes has rank-1 entries (dims 1..rank-1).
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);

// Opt a kernel into more than 48 KB of dynamic shared memory (once).
cudaError_t set_max_smem(const void* func, int bytes);

enum GemmMode { kFwd = 0, kDgrad = 1, kWgrad = 2 };

struct GemmCall {
  int mode;
  const void* a;           // FWD: x   DGRAD: dy   WGRAD: dy
  const void* b;           // WGRAD: x (unused otherwise)
  gl_grouped w;            // FWD/DGRAD weights
  const gl_grouped* bias;  // FWD bias (nullable)
  gl_grouped out_grouped;  // WGRAD main_grad
  void* out;               // FWD y / DGRAD dx
  int64_t out_rows;
  const int64_t* offsets;
  int32_t* status;
  int G;
  int64_t M;
  int N, K;
  int accumulate;
  int cta_pair;  // 1: 256x256 tiles on CTA pairs (cta_group::2); 0: 128x256 tiles per CTA
  uint64_t wait_ns;  // bound on each pipeline wait inside the kernel
  int hold_loads;    // testing: issue no loads (every pipeline wait runs out)
  cudaStream_t stream;
};

gl_status launch_grouped_gemm(const GemmCall& c);

// MXFP8 grouped GEMM (E4M3 codes, E8M0 scales; see gl_gemm_mx.cu).
struct MxCall {
  int mode;
  const void* a;           // A codes: FWD x, DGRAD dy (rowwise); WGRAD dy (columnwise)
  const void* sa;          // A scale atoms: rowwise (FWD/DGRAD) or columnwise (WGRAD), GL_SCALES_MMA
  const void* b;           // WGRAD: x columnwise codes
  const void* sb;          // WGRAD: x columnwise scale atoms
  gl_grouped w;            // FWD: W rowwise codes; DGRAD: W columnwise codes
  gl_grouped ws;           // FWD: W rowwise scale atoms; DGRAD: W columnwise scale atoms
  const gl_grouped* bias;  // FWD (nullable)
  gl_grouped out_grouped;  // WGRAD main_grad
  void* out;
  int64_t out_rows;
  const int64_t* offsets;
  int32_t* status;
  int G;
  int64_t M;
  int N, K;
  int accumulate;
  int cta_pair;  // 1: 256x256 tiles on CTA pairs; 0: 128x256 tiles on single CTAs
  uint64_t wait_ns;  // bound on each pipeline wait inside the kernel
  int hold_loads;    // testing: issue no loads (every pipeline wait runs out)
  cudaStream_t stream;
};

gl_status launch_grouped_gemm_mx(const MxCall& c);

gl_status launch_dbias(const void* dy, const int64_t* offsets, int32_t* status, int G, int N,
                       gl_grouped dbias, cudaStream_t stream);

gl_status launch_offsets(const int64_t* m, int G, int64_t expect_rows, int64_t out_rows,
                         int64_t* offsets, int32_t* status, cudaStream_t stream);

// part != NULL: also the per-(32-row block, column) fp32 sums of the source
// (part [part_blocks, cols]) and the groups' first blocks (part_prefix
// int64[G+1]); row_offsets required.
gl_status launch_quantize(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                          int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                          uint8_t* codes_c, uint8_t* scales_c, int scale_layout, float* part,
                          int64_t part_blocks, int64_t* part_prefix, cudaStream_t stream);

// Argument checks of group_quantize_mxfp8_dbias other than its workspace
// (GL_OK when the call is valid).
gl_status check_quantize_dbias_args(const void* src, int64_t rows, int cols, const int64_t* row_offsets, int G,
                                    const int32_t* status, const uint8_t* codes_r, const uint8_t* scales_r,
                                    const uint8_t* codes_c, const uint8_t* scales_c, int scale_layout,
                                    const gl_grouped& dbias);

// Bias gradient from the cast's partials: dbias_g[n] = sum over the blocks
// [part_prefix[g], part_prefix[g+1]) of part[b, n], in block order, rounded
// once to bf16.
gl_status launch_dbias_partials(const float* part, const int64_t* part_prefix, int32_t* status, int G, int N,
                                gl_grouped dbias, cudaStream_t stream);

}  // namespace gl
