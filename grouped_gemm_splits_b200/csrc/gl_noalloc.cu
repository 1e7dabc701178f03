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
// as a device address, so the first call on each device looks the address up
// (cudaGetSymbolAddress, with that device current) and keeps it, together
// with the identity of the context it belongs to; if that context is later
// destroyed and re-created (a device reset), the next call looks it up again.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "gl_internal.h"

namespace {

// Largest scratch one call may use: gl_dbias_workspace_bytes(rows, cols, G)
// must not exceed it.
constexpr size_t kScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

struct ScratchAddr {
  void* addr = nullptr;
  unsigned long long ctx = 0;  // id of the context the address belongs to
};

std::mutex g_mu;
ScratchAddr g_addr[kMaxDevices];

// Unique id of the calling thread's current context (0 when there is none,
// or the driver cannot say).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_scratch on the current device; nullptr (with the
// runtime's sticky last error cleared) if the runtime cannot give it.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchAddr& a = g_addr[dev];
  const unsigned long long ctx = current_context_id();
  if (a.addr != nullptr && ctx != 0 && ctx == a.ctx) return a.addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();  // reported once, by this call; later launches start clean
    a = ScratchAddr{};
    return nullptr;
  }
  a.addr = p;
  a.ctx = current_context_id();  // the lookup made the context current if it was not
  return p;
}

}  // namespace

extern "C" {

gl_status group_quantize_mxfp8_dbias_noalloc(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                                             int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                                             uint8_t* codes_c, uint8_t* scales_c, int scale_layout,
                                             gl_grouped dbias, void* stream) {
  // argument errors first, in the order group_quantize_mxfp8_dbias reports them
  const gl_status st = gl::check_quantize_dbias_args(src, rows, cols, row_offsets, G, status, codes_r, scales_r,
                                                     codes_c, scales_c, scale_layout, dbias);
  if (st != GL_OK) return st;
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
