// gl_dbias.cu -- bias gradient of the grouped linear layer: for every group g
// and output feature n, db_g[n] = sum over the group's rows r of dy[r, n].
//
// TransformerEngine ``grouped_linear.py`` (ops/basic, fuser_backward): with a
// bias, each split of grad_output is summed over its rows
// (``dy.reshape(-1, dy.size(-1)).sum(dim=0)`` per split) -- a bf16 tensor
// reduced with fp32 accumulation and rounded once to bf16.
//
// One cluster of 8 CTAs per (group, 128-column strip): the 64 warps of the
// cluster stride over the group's rows (4 rows in flight per warp, 8 bytes per
// lane: a warp covers the strip's 256 bytes of a row) and accumulate in fp32
// registers; each CTA combines its 8 warps through shared memory, and the
// cluster's first CTA adds the 8 CTA sums through distributed shared memory
// and rounds to bf16.  Splitting every group 8 ways keeps the largest group
// of a skewed split from serialising the pass.  HBM-bound: dy is read once;
// the output is [G, N].  An empty group gets zeros.
//
// The same kernel, on fp32 input, finishes the bias gradient that the MXFP8
// cast of dy computes on the way (gl_quantize.cu): its rows are then the
// cast's per-32-row-block column sums and the group offsets count blocks.
// Every level adds in a fixed order, so the result is deterministic.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "gl_internal.h"
#include "gl_ptx.cuh"

namespace gl {
namespace {

constexpr int kDThreads = 256;
constexpr int kDCols = 128;  // columns per CTA (4 per lane)
constexpr int kDWarps = kDThreads / 32;
constexpr int kDUnroll = 4;   // rows in flight per warp
constexpr int kDCluster = 8;  // CTAs sharing one (group, strip)
constexpr int kDPG = 64;      // per-group output pointers carried by one launch

struct DbiasPG {
  __nv_bfloat16* ptr[kDPG];
};

// four consecutive columns of one row as fp32
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                     __uint_as_float(v.y & 0xFFFF0000u));
}
__device__ __forceinline__ float4 load4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }

template <typename T>
__global__ void __cluster_dims__(kDCluster, 1, 1) __launch_bounds__(kDThreads)
    dbias_kernel(const T* __restrict__ dy, const int64_t* __restrict__ offsets,
                 const int32_t* __restrict__ status, int N, int strips, __nv_bfloat16* __restrict__ out,
                 const __grid_constant__ DbiasPG pg, int per_group) {
  __shared__ __align__(16) float part[kDWarps][kDCols];
  if (status != nullptr && *status != 0) return;  // every CTA of the cluster reads the same word
  const int unit = static_cast<int>(blockIdx.x) / kDCluster;
  const uint32_t crank = cluster_ctarank();
  const int g = unit / strips;
  const int strip = unit - g * strips;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = strip * kDCols + lane * 4;  // this lane's 4 columns
  const bool col_ok = col < N;                // N % 8 == 0, so 4 columns are all in or all out
  const int64_t r0 = offsets[g], r1 = offsets[g + 1];
  constexpr int kStride = kDCluster * kDWarps;  // rows between a warp's consecutive rows

  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (col_ok) {
    const T* base = dy + col;
    int64_t r = r0 + static_cast<int>(crank) * kDWarps + warp;
    // kDUnroll independent rows per iteration keep loads in flight
    for (; r + (kDUnroll - 1) * kStride < r1; r += kDUnroll * kStride) {
      float4 v[kDUnroll];
#pragma unroll
      for (int u = 0; u < kDUnroll; ++u) v[u] = load4(base + (r + u * kStride) * N);
#pragma unroll
      for (int u = 0; u < kDUnroll; ++u) {
        acc[0] += v[u].x;
        acc[1] += v[u].y;
        acc[2] += v[u].z;
        acc[3] += v[u].w;
      }
    }
    for (; r < r1; r += kStride) {
      const float4 v = load4(base + r * N);
      acc[0] += v.x;
      acc[1] += v.y;
      acc[2] += v.z;
      acc[3] += v.w;
    }
  }
  *reinterpret_cast<float4*>(&part[warp][lane * 4]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (threadIdx.x < kDCols) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) s += part[w][threadIdx.x];
    part[0][threadIdx.x] = s;  // this CTA's sum (each thread rewrites only its own column)
  }
  cluster_sync();  // every CTA's sum is in its shared memory
  if (crank == 0 && threadIdx.x < kDCols) {
    const int c = strip * kDCols + static_cast<int>(threadIdx.x);
    float s = part[0][threadIdx.x];
    const uint32_t mine = smem_u32(&part[0][threadIdx.x]);
#pragma unroll
    for (uint32_t k = 1; k < kDCluster; ++k) {
      float v;
      asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(mapa_shared(mine, k)) : "memory");
      s += v;
    }
    if (c < N) {
      __nv_bfloat16* dst = per_group ? pg.ptr[g] : out + static_cast<int64_t>(g) * N;
      dst[c] = __float2bfloat16_rn(s);
    }
  }
  cluster_sync();  // the first CTA has read every peer's shared memory
}

template <typename T>
gl_status launch_segmented_colsum(const T* src, const int64_t* offsets, int32_t* status, int G, int N,
                                  gl_grouped dbias, cudaStream_t stream) {
  const int strips = (N + kDCols - 1) / kDCols;
  if (dbias.mode == GL_STACKED) {
    DbiasPG none;
    memset(&none, 0, sizeof(none));
    dbias_kernel<T><<<G * strips * kDCluster, kDThreads, 0, stream>>>(
        src, offsets, status, N, strips, static_cast<__nv_bfloat16*>(const_cast<void*>(dbias.base)), none, 0);
    return cudaGetLastError() == cudaSuccess ? GL_OK : GL_ERR_CUDA;
  }
  DbiasPG pg;
  for (int g0 = 0; g0 < G; g0 += kDPG) {
    const int cg = std::min(kDPG, G - g0);
    memset(&pg, 0, sizeof(pg));
    for (int i = 0; i < cg; ++i) pg.ptr[i] = static_cast<__nv_bfloat16*>(const_cast<void*>(dbias.ptrs[g0 + i]));
    dbias_kernel<T><<<cg * strips * kDCluster, kDThreads, 0, stream>>>(src, offsets + g0, status, N, strips, nullptr,
                                                                       pg, 1);
    if (cudaGetLastError() != cudaSuccess) return GL_ERR_CUDA;
  }
  return GL_OK;
}

}  // namespace

gl_status launch_dbias(const void* dy, const int64_t* offsets, int32_t* status, int G, int N,
                       gl_grouped dbias, cudaStream_t stream) {
  return launch_segmented_colsum(static_cast<const __nv_bfloat16*>(dy), offsets, status, G, N, dbias, stream);
}

gl_status launch_dbias_partials(const float* part, const int64_t* part_prefix, int32_t* status, int G, int N,
                                gl_grouped dbias, cudaStream_t stream) {
  return launch_segmented_colsum(part, part_prefix, status, G, N, dbias, stream);
}

}  // namespace gl
