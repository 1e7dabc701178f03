// gl_offsets.cu -- device prefix scan of the split sizes.
//
// o[0] = 0, o[i+1] = o[i] + m[i] in int64 ("Single parameter for GroupedLinear
// module", TransformerEngine PR #2727: nvte_cumsum, a scan with a leading zero
// replacing cumsum + cat).  One CTA of 1024 threads scans the sizes in chunks
// of 1024 (warp shuffles, then a scan of the 32 warp totals, then a carry into
// the next chunk) and also folds the validity checks of the sizes into the
// status word, so the split sizes never have to reach the host.
#include "gl_internal.h"

namespace gl {
namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
    offsets_kernel(const int64_t* __restrict__ m, int G, int64_t expect_rows, int64_t out_rows,
                   int64_t* __restrict__ offsets, int32_t* __restrict__ status) {
  __shared__ int64_t warp_tot[32];
  __shared__ int64_t carry_s;
  __shared__ int neg_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry_s = 0;
    neg_s = 0;
    offsets[0] = 0;
  }
  __syncthreads();
  int neg = 0;
  for (int base = 0; base < G; base += kScanThreads) {
    const int i = base + tid;
    int64_t v = (i < G) ? m[i] : 0;
    neg |= (v < 0);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int64_t w = warp_tot[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t u = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += u;
      }
      warp_tot[lane] = w;  // inclusive scan of warp totals
    }
    __syncthreads();
    const int64_t carry = carry_s;
    const int64_t incl = v + (warp > 0 ? warp_tot[warp - 1] : 0) + carry;
    if (i < G) offsets[i + 1] = incl;
    __syncthreads();
    if (tid == kScanThreads - 1) carry_s = incl;
    __syncthreads();
  }
  if (neg) atomicOr(&neg_s, 1);
  __syncthreads();
  if (tid == 0) {
    const int64_t total = carry_s;
    int32_t flags = 0;
    if (neg_s) flags |= GL_DEV_NEG_SPLIT;
    if (total != expect_rows) flags |= GL_DEV_SUM_MISMATCH;
    if (total > out_rows) flags |= GL_DEV_OUT_OVERFLOW;
    *status = flags;
  }
}

}  // namespace

gl_status launch_offsets(const int64_t* m, int G, int64_t expect_rows, int64_t out_rows,
                         int64_t* offsets, int32_t* status, cudaStream_t stream) {
  offsets_kernel<<<1, kScanThreads, 0, stream>>>(m, G, expect_rows, out_rows, offsets, status);
  return cudaGetLastError() == cudaSuccess ? GL_OK : GL_ERR_CUDA;
}

}  // namespace gl
