// gl_noalloc.cu -- group_quantize_mxfp8_dbias_noalloc: the fused MXFP8 cast +
// bias gradient of group_quantize_mxfp8_dbias without a caller workspace.
//
// Some callers cannot allocate device memory where they call this: their
// memory belongs to another runtime's pool and they are handed no allocator
// (and a cudaMalloc there would also synchronise the device).  This entry
// point takes its scratch from one fixed array in the library's own device
// memory instead, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it until the process exits.  Host code cannot use its name
// as a device address, so the first call on each device looks the address
// up (cudaGetSymbolAddress, with that device current) and keeps it.
#include <cuda_runtime.h>

#include <mutex>

#include "gl.h"

namespace {

// Largest scratch one call may use: gl_dbias_workspace_bytes(rows, cols, G)
// must not exceed it.
constexpr size_t kScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per
// device); nullptr if the runtime cannot give it.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) return nullptr;
    g_addr[dev] = p;
  }
  return g_addr[dev];
}

}  // namespace

extern "C" {

gl_status group_quantize_mxfp8_dbias_noalloc(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                                             int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                                             uint8_t* codes_c, uint8_t* scales_c, int scale_layout,
                                             gl_grouped dbias, void* stream) {
  const size_t need = gl_dbias_workspace_bytes(rows, cols, G);
  if (need == 0) return GL_ERR_INVALID;
  if (need > kScratchBytes) return GL_ERR_UNSUPPORTED;  // larger than the fixed scratch
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return GL_ERR_CUDA;
  // Nothing in the scratch needs to start at zero: the cast writes every
  // partial and offset that the reduction reads.
  return group_quantize_mxfp8_dbias(src, rows, cols, row_offsets, G, status, codes_r, scales_r, codes_c, scales_c,
                                    scale_layout, dbias, scratch, kScratchBytes, stream);
}

}  // extern "C"
