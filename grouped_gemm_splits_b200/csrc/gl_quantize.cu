// gl_quantize.cu -- grouped MXFP8 cast: E4M3 codes, one E8M0 scale per 32
// elements, rowwise and/or columnwise in one pass over the bf16 source.
//
// TransformerEngine ``grouped_linear.py`` (ops/basic) keeps MXFP8 operands as
// E4M3 data with power-of-two block scales in a rowwise copy (blocks along a
// row) and a columnwise copy (blocks down a column), and quantizes each
// split of the input as its own tensor; the grouped cast kernel is
// ``group_quantize_mxfp8`` ("Improve device-init grouped linear module",
// PR #3224).
//
// Work unit: a 32-row block of one group (the columnwise block) x 256
// columns.  Every element is read once (16-byte loads, a warp covers 512
// contiguous bytes of a row); rowwise amax is a 4-lane shuffle reduction,
// columnwise amax a shared-memory reduction over the block's 32 rows.  The
// kernel is persistent; each CTA first builds the per-group block prefix in
// shared memory.  Memory-bound: 2 bytes read and up to 2 bytes (+1/16 for
// scales) written per element.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "gl_internal.h"

namespace gl {
namespace {

constexpr int kQThreads = 256;
constexpr int kQCols = 256;
constexpr int kQRows = 32;

// Scale exponent: smallest e with amax <= 448 * 2^e, clamped to [-127, 127];
// 448 = 1.75 * 2^8, so for amax = 1.f * 2^E the answer is E - 8, plus one when
// 1.f > 1.75.  amax = 0 gives 0.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int E = static_cast<int>((b >> 23) & 0xFFu);
  const uint32_t mant = b & 0x7FFFFFu;
  int e;
  if (amax == 0.0f) e = 0;
  else if (E == 0) e = -127;  // subnormal amax: below 448 * 2^-127
  else e = (E - 127) - 8 + (mant > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as a float (e in [-127, 126] gives a normal number).
__device__ __forceinline__ float pow2_neg(int e) {
  const int bexp = 127 - e;
  return bexp >= 1 && bexp <= 254 ? __uint_as_float(static_cast<uint32_t>(bexp) << 23) : 0.0f;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(kQThreads, 4)
    quantize_kernel(const __nv_bfloat16* __restrict__ src, int64_t rows, int cols,
                    const int64_t* __restrict__ row_offsets, int G, const int32_t* __restrict__ status,
                    uint8_t* __restrict__ codes_r, uint8_t* __restrict__ scales_r,
                    uint8_t* __restrict__ codes_c, uint8_t* __restrict__ scales_c, int64_t scales_c_bytes,
                    int mma_layout) {
  extern __shared__ int64_t qsmem[];
  int64_t* bprefix = qsmem;        // G+1: first 32-row block of each group (ragged mode)
  int64_t* qprefix = qsmem + G + 1;  // G+1: first 128-row k-group of each group (ragged mode)
  __shared__ float cmax[kQThreads / 32][kQCols];
  __shared__ float csf[kQCols];
  if (status != nullptr && *status != 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int64_t per = (row_offsets == nullptr) ? rows / G : 0;
  const int64_t bpg = (per + kQRows - 1) / kQRows;  // blocks per group (uniform mode)
  const int64_t qpg = (per + 127) / 128;            // k-groups per group (uniform mode)
  const int64_t mma_rb = (rows + 127) / 128;        // 128-row blocks (rowwise MMA layout)
  const int mma_cb = cols / 128;                    // 128-column blocks (columnwise MMA layout)
  int64_t nblocks;
  if (row_offsets != nullptr) {
    if (warp == 0) {
      int64_t carry = 0, qcarry = 0;
      for (int base = 0; base < G; base += 32) {
        const int i = base + lane;
        int64_t cnt = 0, qc = 0;
        if (i < G) {
          const int64_t m = row_offsets[i + 1] - row_offsets[i];
          cnt = m > 0 ? (m + kQRows - 1) / kQRows : 0;
          qc = m > 0 ? (m + 127) / 128 : 0;
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int64_t u = __shfl_up_sync(0xffffffffu, cnt, off);
          const int64_t w = __shfl_up_sync(0xffffffffu, qc, off);
          if (lane >= off) { cnt += u; qc += w; }
        }
        if (i < G) { bprefix[i + 1] = carry + cnt; qprefix[i + 1] = qcarry + qc; }
        carry += __shfl_sync(0xffffffffu, cnt, 31);
        qcarry += __shfl_sync(0xffffffffu, qc, 31);
      }
      if (lane == 0) { bprefix[0] = 0; qprefix[0] = 0; }
    }
    __syncthreads();
    nblocks = bprefix[G];
  } else {
    nblocks = bpg * G;
  }
  const int ncc = (cols + kQCols - 1) / kQCols;
  const int64_t ntiles = nblocks * ncc;
  const int c8 = lane;         // 8-column chunk within the 256-column tile
  const int rbase = warp * 4;  // this thread's 4 rows within the 32-row block

  // Where tile t lives: group g, block j, first row r0 and valid row count.
  auto locate = [&](int64_t t, int& g, int64_t& j, int64_t& r0, int& vrows, int& cc) {
    const int64_t rb = t / ncc;
    cc = static_cast<int>(t - rb * ncc);
    int64_t gstart, gend;
    if (row_offsets != nullptr) {
      int lo = 0, hi = G;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (bprefix[mid] <= rb) lo = mid; else hi = mid;
      }
      g = lo;
      j = rb - bprefix[g];
      gstart = min(max(row_offsets[g], int64_t(0)), rows);  // clamp: never leave [0, rows)
      gend = min(max(row_offsets[g + 1], gstart), rows);
    } else {
      g = static_cast<int>(rb / bpg);
      j = rb - static_cast<int64_t>(g) * bpg;
      gstart = static_cast<int64_t>(g) * per;
      gend = gstart + per;
    }
    r0 = gstart + j * kQRows;
    vrows = static_cast<int>(max(int64_t(0), min(static_cast<int64_t>(kQRows), gend - r0)));
  };
  // 16-byte loads of this thread's 4 rows x 8 columns of tile t (zeros outside)
  auto fetch = [&](int64_t r0, int vrows, int cc, uint4 (&raw)[4]) {
    const int col = cc * kQCols + c8 * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = rbase + i;
      if (col < cols && r < vrows)
        raw[i] = __ldg(reinterpret_cast<const uint4*>(src + (r0 + r) * cols + col));
      else
        raw[i] = make_uint4(0, 0, 0, 0);
    }
  };

  int64_t t = blockIdx.x;
  int g = 0, vrows = 0, cc = 0;
  int64_t j = 0, r0 = 0;
  uint4 raw[4];
  if (t < ntiles) {
    locate(t, g, j, r0, vrows, cc);
    fetch(r0, vrows, cc, raw);
  }
  for (; t < ntiles; t += gridDim.x) {
    // issue the next tile's loads before working on this one
    const int64_t tn = t + gridDim.x;
    int gn = 0, vrows_n = 0, cc_n = 0;
    int64_t jn = 0, r0n = 0;
    uint4 raw_n[4];
    if (tn < ntiles) {
      locate(tn, gn, jn, r0n, vrows_n, cc_n);
      fetch(r0n, vrows_n, cc_n, raw_n);
    }
    const int col = cc * kQCols + c8 * 8;
    const bool col_ok = col < cols;
    float v[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw[i]);
#pragma unroll
      for (int k = 0; k < 8; ++k) v[i][k] = __bfloat162float(h[k]);
    }

    if (codes_r != nullptr) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) a = fmaxf(a, fabsf(v[i][k]));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        const int e = mx_scale_exp(a);
        const float s = pow2_neg(e);
        const int r = rbase + i;
        if (col_ok && r < vrows) {
          const int64_t row = r0 + r;
          uint2 q;
          q.x = e4m3x4(v[i][0] * s, v[i][1] * s, v[i][2] * s, v[i][3] * s);
          q.y = e4m3x4(v[i][4] * s, v[i][5] * s, v[i][6] * s, v[i][7] * s);
          *reinterpret_cast<uint2*>(codes_r + row * cols + col) = q;
          if ((c8 & 3) == 0) {
            // row-major [rows, cols/32], or the tcgen05 scale-factor atoms:
            // 512 bytes per (k-group of 4 blocks, 128 rows), row i of the
            // atom at byte (i%32)*16 + ((i/32)%4)*4 + block
            const int64_t kb = col / 32;
            const int64_t at = mma_layout ? ((kb >> 2) * mma_rb + (row >> 7)) * 512 + (row & 31) * 16 +
                                                ((row >> 5) & 3) * 4 + (kb & 3)
                                          : row * (cols / 32) + kb;
            scales_r[at] = static_cast<uint8_t>(e + 127);
          }
        }
      }
    }

    if (codes_c != nullptr) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) a = fmaxf(a, fabsf(v[i][k]));
        cmax[warp][c8 * 8 + k] = a;
      }
      __syncthreads();
      {
        float a = 0.0f;
#pragma unroll
        for (int w = 0; w < kQThreads / 32; ++w) a = fmaxf(a, cmax[w][tid]);
        const int e = mx_scale_exp(a);
        csf[tid] = pow2_neg(e);
        const int ccol = cc * kQCols + tid;
        if (ccol < cols && vrows > 0) {
          int64_t at;
          if (mma_layout) {
            // atom (k-group of the group's blocks 4t..4t+3, 128 columns)
            const int64_t kq = (row_offsets != nullptr ? qprefix[g] : static_cast<int64_t>(g) * qpg) + (j >> 2);
            at = (kq * mma_cb + (ccol >> 7)) * 512 + (ccol & 31) * 16 + ((ccol >> 5) & 3) * 4 + (j & 3);
          } else {
            at = ((row_offsets != nullptr ? bprefix[g] : static_cast<int64_t>(g) * bpg) + j) * cols + ccol;
          }
          // offsets that overlap (only possible without a status word) must
          // not push a write past the documented allocation
          if (at < scales_c_bytes) scales_c[at] = static_cast<uint8_t>(e + 127);
        }
      }
      __syncthreads();
      float s[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) s[k] = csf[c8 * 8 + k];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rbase + i;
        if (col_ok && r < vrows) {
          uint2 q;
          q.x = e4m3x4(v[i][0] * s[0], v[i][1] * s[1], v[i][2] * s[2], v[i][3] * s[3]);
          q.y = e4m3x4(v[i][4] * s[4], v[i][5] * s[5], v[i][6] * s[6], v[i][7] * s[7]);
          *reinterpret_cast<uint2*>(codes_c + (r0 + r) * cols + col) = q;
        }
      }
      __syncthreads();  // cmax / csf are reused by the next tile
    }
    g = gn;
    j = jn;
    r0 = r0n;
    vrows = vrows_n;
    cc = cc_n;
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = raw_n[i];
  }
}

}  // namespace

gl_status launch_quantize(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                          int G, const int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                          uint8_t* codes_c, uint8_t* scales_c, int scale_layout, cudaStream_t stream) {
  const int smem = row_offsets != nullptr ? 2 * (G + 1) * static_cast<int>(sizeof(int64_t)) : 0;
  if (set_max_smem(reinterpret_cast<const void*>(quantize_kernel), smem + 16 * 1024) != cudaSuccess)
    return GL_ERR_CUDA;
  const int grid = num_sms() * 4;
  quantize_kernel<<<grid, kQThreads, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(src), rows, cols, row_offsets, G, status, codes_r,
      scales_r, codes_c, scales_c,
      static_cast<int64_t>(gl_mxfp8_scale_bytes(rows, cols, G, 1, scale_layout)),
      scale_layout == GL_SCALES_MMA ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? GL_OK : GL_ERR_CUDA;
}

}  // namespace gl
