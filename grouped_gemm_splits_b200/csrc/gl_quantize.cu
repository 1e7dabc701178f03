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
// Work unit (tile): a 32-row block of one group (the columnwise block) x 512
// columns (256 when the rows are narrower), staged in shared memory by TMA.
// The kernel is persistent; a producer warp keeps a ring of tiles loaded
// ahead (full / empty mbarriers) and eight consumer warps share no data: each
// owns whole 32-column blocks of the tile (a lane: 4 rows x 8 columns of a
// block), so both block maxima -- along a row and down a column -- are warp
// shuffles and no block-wide barrier is taken per tile.  Each CTA first
// builds the per-group block prefixes in shared memory.  Memory-bound in
// principle: 2 bytes read and up to 2 bytes (+1/16 for scales) written per
// element; in practice about a fifth below the copy bandwidth, bound by the
// per-element integer and conversion work.
//
// With a bias gradient (the cast of dy; fuser_backward sums each split of
// grad_output over its rows next to quantizing it), the same pass also adds
// every block's 32 rows per column in fp32 -- a lane its 4 rows, then the 8
// row groups of the warp by a butterfly -- and stores one fp32 partial per
// (32-row block, column) in a caller workspace; dbias_partials_kernel
// (gl_dbias.cu) adds each group's partials in block order.  The sums are
// deterministic: no atomics, a fixed order at every level.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "gl_internal.h"
#include "gl_ptx.cuh"

namespace gl {
namespace {

constexpr int kQThreads = 256;
constexpr int kQCols = 256;
constexpr int kQRows = 32;
static_assert(kQThreads == 256 && kQCols == 256, "eight consumer warps, one 32-column block each per box");
// Tiles staged in shared memory by TMA, and CTAs per SM (each CTA: eight
// consumer warps and a producer warp).
constexpr int kQBoxBytes = kQRows * kQCols * 2;  // one TMA box: 32 rows x 256 columns
template <int kCB>
struct QCfg {
  static constexpr int kTileBytes = kCB * kQBoxBytes;
  static constexpr int kStages = kCB == 1 ? 4 : 3;
  static constexpr int kCtasPerSm = 2;
};

// Per 16-bit half: the unsigned maximum.
__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The two bf16 values of a word as fp32 (a bf16 is the high half of an fp32).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Block scale from the bf16 bits `a` of a block's amax (sign clear): the
// smallest e with amax <= 448 * 2^e, clamped to [-127, 127]; e = 0 when
// amax = 0.  448 = 1.75 * 2^8, so for amax = 1.m * 2^(E-127) the answer is
// E - 135, plus one when 1.m > 1.75, i.e. when the 7 mantissa bits exceed
// 0x60: adding 0x1F carries into the exponent field exactly then.  A
// subnormal amax is below 448 * 2^-127.  Returns 2^-e as a float and the
// biased byte e + 127.
__device__ __forceinline__ float mx_scale_bf16(uint32_t a, uint32_t& byte) {
  const uint32_t ec = max((a + 0x1Fu) >> 7, 8u);  // e + 135, at least 8
  byte = a ? ec - 8u : 127u;
  return __uint_as_float(a ? (262u - ec) << 23 : 0x3F800000u);
}

// Four values times their scales (exact: powers of two; two packed fp32
// multiplies), rounded to four E4M3 codes (satfinite), the first value in the
// lowest byte.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d, float sa, float sb, float sc,
                                           float sd) {
  uint32_t q;
  asm("{\n\t.reg .b64 v0, v1, s0, s1, p0, p1;\n\t.reg .f32 x0, y0, x1, y1;\n\t.reg .b16 l, h;\n\t"
      "mov.b64 v0, {%1, %2};\n\t"
      "mov.b64 v1, {%3, %4};\n\t"
      "mov.b64 s0, {%5, %6};\n\t"
      "mov.b64 s1, {%7, %8};\n\t"
      "mul.rn.f32x2 p0, v0, s0;\n\t"
      "mul.rn.f32x2 p1, v1, s1;\n\t"
      "mov.b64 {x0, y0}, p0;\n\t"
      "mov.b64 {x1, y1}, p1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 l, y0, x0;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h, y1, x1;\n\t"
      "mov.b32 %0, {l, h};\n\t}"
      : "=r"(q)
      : "f"(a), "f"(b), "f"(c), "f"(d), "f"(sa), "f"(sb), "f"(sc), "f"(sd));
  return q;
}

// Work unit (tile): a 32-row block of one group x kCB * 256 columns, staged
// in shared memory by TMA (kCB boxes of 32 x 256).  Warp 8 is the producer:
// one thread keeps a ring of kStages tiles in flight (full / empty mbarriers).
// Warps 0-7 are consumers and share no data: warp w owns the 32-column
// blocks w, w + 8, .. of the tile, so that both block maxima of its elements
// -- along a row (32 columns) and down a column (32 rows) -- are reduced
// within the warp by shuffles.  A lane holds rows 4 * (lane / 4) .. + 3 and
// 8 columns (8 * (lane % 4) ..) of each of its blocks.
//
// kDbias: also write the per-block column sums (part: [part_blocks, cols]
// fp32, block b of the launch in row b; part_prefix: the groups' first
// blocks, int64[G+1], written by CTA 0).
template <bool kDbias, int kCB>
__global__ void __launch_bounds__(kQThreads + 32, QCfg<kCB>::kCtasPerSm)
    quantize_kernel(const __grid_constant__ CUtensorMap tm_src, int64_t rows, int cols, int box_rows,
                    int box_bytes, const int64_t* __restrict__ row_offsets, int G, int32_t* status,
                    uint8_t* __restrict__ codes_r, uint8_t* __restrict__ scales_r,
                    uint8_t* __restrict__ codes_c, uint8_t* __restrict__ scales_c, int64_t scales_c_bytes,
                    int mma_layout, float* __restrict__ part, int64_t part_blocks,
                    int64_t* __restrict__ part_prefix) {
  using Q = QCfg<kCB>;
  constexpr int kStages = Q::kStages;
  constexpr int kTileCols = kCB * kQCols;
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* qsmem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_buf = qsmem;                                                      // kStages x kCB boxes
  uint64_t* full = reinterpret_cast<uint64_t*>(qsmem + kStages * Q::kTileBytes);  // tile landed
  uint64_t* empty = full + kStages;                                               // tile consumed (8 warps)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  int64_t* bprefix = reinterpret_cast<int64_t*>(qsmem + kStages * Q::kTileBytes + 128);  // G+1 (ragged)
  int64_t* qprefix = bprefix + G + 1;                                                    // G+1 (ragged)
  if (status != nullptr && *reinterpret_cast<volatile int32_t*>(status) != 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kQThreads / 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }

  const int64_t per = (row_offsets == nullptr) ? rows / G : 0;
  const int64_t bpg = (per + kQRows - 1) / kQRows;  // blocks per group (uniform mode)
  const int64_t qpg = (per + 127) / 128;            // k-groups per group (uniform mode)
  const int64_t mma_rb = (rows + 127) / 128;        // 128-row blocks (rowwise MMA layout)
  const int mma_cb = cols / 128;                    // 128-column blocks (columnwise MMA layout)
  if (row_offsets != nullptr && warp == 0) {
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
  if (kDbias && blockIdx.x == 0 && row_offsets != nullptr)
    for (int i = tid; i <= G; i += blockDim.x) part_prefix[i] = bprefix[i];
  const int64_t nblocks = (row_offsets != nullptr) ? bprefix[G] : bpg * G;
  const int ncc = (cols + kTileCols - 1) / kTileCols;
  const int64_t ntiles = nblocks * ncc;
  const int pitch = box_bytes / box_rows;  // bytes per staged row of a box (2 * min(cols, 256))

  // Tile t = rb * ncc + cc (rb: 32-row block, counted over all groups; cc:
  // column chunk).  A CTA visits t = blockIdx.x + k * gridDim.x; the position
  // advances by (gridDim.x / ncc, gridDim.x % ncc) with a carry and the group
  // index moves forward with it, so the loop does no 64-bit division.
  const bool ragged = row_offsets != nullptr;
  const int step_rb = static_cast<int>(gridDim.x) / ncc, step_cc = static_cast<int>(gridDim.x) % ncc;
  struct Pos {
    int64_t rb;
    int cc, g;
  };
  auto advance_group = [&](Pos& q) {
    if (ragged) {
      while (q.g + 1 < G && bprefix[q.g + 1] <= q.rb) ++q.g;
    } else {
      while (q.g + 1 < G && static_cast<int64_t>(q.g + 1) * bpg <= q.rb) ++q.g;
    }
  };
  auto step = [&](Pos& q) {
    q.cc += step_cc;
    q.rb += step_rb;
    if (q.cc >= ncc) { q.cc -= ncc; ++q.rb; }
    advance_group(q);
  };
  // Block j of group g, its first row r0 and valid row count.
  auto resolve = [&](const Pos& q, int64_t& j, int64_t& r0, int& vrows) {
    int64_t gstart, gend;
    if (ragged) {
      j = q.rb - bprefix[q.g];
      gstart = min(max(row_offsets[q.g], int64_t(0)), rows);  // clamp: never leave [0, rows)
      gend = min(max(row_offsets[q.g + 1], gstart), rows);
    } else {
      j = q.rb - static_cast<int64_t>(q.g) * bpg;
      gstart = static_cast<int64_t>(q.g) * per;
      gend = gstart + per;
    }
    r0 = gstart + j * kQRows;
    vrows = static_cast<int>(max(int64_t(0), min(static_cast<int64_t>(kQRows), gend - r0)));
  };
  Pos pos;
  pos.rb = static_cast<int>(blockIdx.x) / ncc;
  pos.cc = static_cast<int>(blockIdx.x) % ncc;
  pos.g = 0;
  if (ragged) {
    int lo = 0, hi = G;  // last group whose first block is <= rb
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (bprefix[mid] <= pos.rb) lo = mid; else hi = mid;
    }
    pos.g = lo;
  }
  advance_group(pos);

  if (warp == kQThreads / 32) {
    // ===================== producer (one thread) =====================
    if (lane == 0) {
      int issued = 0;
      for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++issued) {
        const int s = issued % kStages;
        // the consumers' release of this stage's previous tile
        if (!mbar_wait(&empty[s], (static_cast<uint32_t>(issued / kStages) & 1u) ^ 1u, abort_flag)) {
          if (!*abort_flag) {
            *abort_flag = 1;
            if (status != nullptr) atomicOr(status, GL_DEV_TIMEOUT);
          }
          break;
        }
        int64_t jq, rq;
        int vq;
        resolve(pos, jq, rq, vq);
        // rows of other groups and past the tensor are masked or zero-filled;
        // the consumers use only the block's valid rows
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kCB * box_bytes));
#pragma unroll
        for (int b = 0; b < kCB; ++b)
          tma_load_2d(stage_buf + s * Q::kTileBytes + b * kQBoxBytes, &tm_src, &full[s],
                      pos.cc * kTileCols + b * kQCols, static_cast<int32_t>(rq));
        step(pos);
      }
      // never leave while a load may still be writing shared memory
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      for (int k = issued - kStages > 0 ? issued - kStages : 0; k < issued; ++k)
        mbar_wait_until(&full[k % kStages], static_cast<uint32_t>(k / kStages) & 1u, deadline);
    }
    return;
  }

  // ===================== consumers (warps 0-7) =====================
  const int rg = lane >> 2;   // row group: rows 4 rg .. 4 rg + 3 of the block
  const int cg = lane & 3;    // 8 columns (16 bytes) of each 32-column block
  const int rbase = rg * 4;
  int consumed = 0;
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++consumed) {
    const int s = consumed % kStages;
    const int g = pos.g, cc = pos.cc;
    int64_t j, r0;
    int vrows;
    resolve(pos, j, r0, vrows);
    if (!mbar_wait(&full[s], static_cast<uint32_t>(consumed / kStages) & 1u, abort_flag)) {
      if (lane == 0 && !*abort_flag) {
        *abort_flag = 1;
        if (status != nullptr) atomicOr(status, GL_DEV_TIMEOUT);
      }
      break;
    }
#pragma unroll
    for (int b = 0; b < kCB; ++b) {
      const int cblk = cc * (kTileCols / 32) + b * 8 + warp;  // 32-column block of the tensor
      const int col = cblk * 32 + cg * 8;                      // this lane's first column
      const bool col_ok = col < cols;
      // this lane's 4 rows x 8 columns, one 16-byte piece per row (rows past
      // the block's valid rows and columns past the tensor read as zero)
      uint4 raw[4];
      {
        const uint8_t* tile = stage_buf + s * Q::kTileBytes + b * kQBoxBytes + (warp * 32 + cg * 8) * 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rbase + i;
          raw[i] = (r < vrows && col_ok) ? *reinterpret_cast<const uint4*>(tile + r * pitch) : make_uint4(0, 0, 0, 0);
        }
      }
      // |v| as pairs of bf16 bit patterns: for non-negative values the
      // unsigned order of the bits is the order of the values, so every
      // block maximum is an integer maximum over 16-bit halves
      uint32_t mag[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mag[i][0] = raw[i].x & 0x7FFF7FFFu;
        mag[i][1] = raw[i].y & 0x7FFF7FFFu;
        mag[i][2] = raw[i].z & 0x7FFF7FFFu;
        mag[i][3] = raw[i].w & 0x7FFF7FFFu;
      }
      const int64_t tile_off = r0 * cols + col;  // element offset of this lane's first value

      // Block maxima.  Rows: over this lane's 8 columns, two rows per word,
      // then over the 4 lanes of the row group (lane bits 0-1).  Columns: over
      // this lane's 4 rows (two columns per word), then over the 8 row groups
      // (lane bits 2-4).  Every lane ends with the maxima of all its rows and
      // columns; it turns one of each into a scale (row rbase + cg, column
      // col + rg) and the others arrive by shuffles.
      float rs[4], cs[8];
      uint32_t rbyte = 0, cbyte = 0;
      if (codes_r != nullptr) {
        uint32_t m[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) m[i] = umax2(umax2(mag[i][0], mag[i][1]), umax2(mag[i][2], mag[i][3]));
        uint32_t p01 = umax2(__byte_perm(m[0], m[1], 0x5410), __byte_perm(m[0], m[1], 0x7632));
        uint32_t p23 = umax2(__byte_perm(m[2], m[3], 0x5410), __byte_perm(m[2], m[3], 0x7632));
        p01 = umax2(p01, __shfl_xor_sync(0xffffffffu, p01, 1));
        p23 = umax2(p23, __shfl_xor_sync(0xffffffffu, p23, 1));
        p01 = umax2(p01, __shfl_xor_sync(0xffffffffu, p01, 2));
        p23 = umax2(p23, __shfl_xor_sync(0xffffffffu, p23, 2));
        const uint32_t pw = (cg & 2) ? p23 : p01;
        const float own = mx_scale_bf16((cg & 1) ? (pw >> 16) : (pw & 0xFFFFu), rbyte);
#pragma unroll
        for (int i = 0; i < 4; ++i) rs[i] = __shfl_sync(0xffffffffu, own, (lane & ~3) | i);
      }
      if (codes_c != nullptr) {
        uint32_t cm[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          cm[k] = umax2(umax2(mag[0][k], mag[1][k]), umax2(mag[2][k], mag[3][k]));
          cm[k] = umax2(cm[k], __shfl_xor_sync(0xffffffffu, cm[k], 4));
          cm[k] = umax2(cm[k], __shfl_xor_sync(0xffffffffu, cm[k], 8));
          cm[k] = umax2(cm[k], __shfl_xor_sync(0xffffffffu, cm[k], 16));
        }
        const uint32_t cw = (rg & 4) ? ((rg & 2) ? cm[3] : cm[2]) : ((rg & 2) ? cm[1] : cm[0]);
        const float own = mx_scale_bf16((rg & 1) ? (cw >> 16) : (cw & 0xFFFFu), cbyte);
#pragma unroll
        for (int k = 0; k < 8; ++k) cs[k] = __shfl_sync(0xffffffffu, own, (k << 2) | cg);
      }

      // codes: each row unpacked once, then scaled and rounded for each copy
      {
        uint8_t* dr = (codes_r != nullptr) ? codes_r + tile_off + static_cast<int64_t>(rbase) * cols : nullptr;
        uint8_t* dc = (codes_c != nullptr) ? codes_c + tile_off + static_cast<int64_t>(rbase) * cols : nullptr;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (!(col_ok && rbase + i < vrows)) continue;
          float f[8];
          f[0] = bf16_lo(raw[i].x); f[1] = bf16_hi(raw[i].x);
          f[2] = bf16_lo(raw[i].y); f[3] = bf16_hi(raw[i].y);
          f[4] = bf16_lo(raw[i].z); f[5] = bf16_hi(raw[i].z);
          f[6] = bf16_lo(raw[i].w); f[7] = bf16_hi(raw[i].w);
          if (codes_r != nullptr)
            *reinterpret_cast<uint2*>(dr + i * cols) =
                make_uint2(e4m3x4(f[0], f[1], f[2], f[3], rs[i], rs[i], rs[i], rs[i]),
                           e4m3x4(f[4], f[5], f[6], f[7], rs[i], rs[i], rs[i], rs[i]));
          if (codes_c != nullptr)
            *reinterpret_cast<uint2*>(dc + i * cols) =
                make_uint2(e4m3x4(f[0], f[1], f[2], f[3], cs[0], cs[1], cs[2], cs[3]),
                           e4m3x4(f[4], f[5], f[6], f[7], cs[4], cs[5], cs[6], cs[7]));
        }
      }

      // scale bytes: this lane's row and column
      if (codes_r != nullptr && (cblk << 5) < cols && rbase + cg < vrows) {
        // row-major [rows, cols/32], or the tcgen05 scale-factor atoms: 512
        // bytes per (k-group of 4 blocks, 128 rows), row i of the atom at
        // byte (i%32)*16 + ((i/32)%4)*4 + block
        const int64_t row = r0 + rbase + cg;
        const int64_t at = mma_layout ? ((cblk >> 2) * mma_rb + (row >> 7)) * 512 +
                                            static_cast<int>(((row & 31) << 4) | (((row >> 5) & 3) << 2) | (cblk & 3))
                                      : row * (cols >> 5) + cblk;
        scales_r[at] = static_cast<uint8_t>(rbyte);
      }
      if (codes_c != nullptr) {
        const int ccol = col + rg;
        if (ccol < cols && vrows > 0) {
          int64_t at;
          if (mma_layout) {
            // atom (k-group of the group's blocks 4t..4t+3, 128 columns)
            const int64_t kq = (ragged ? qprefix[g] : static_cast<int64_t>(g) * qpg) + (j >> 2);
            at = (kq * mma_cb + (ccol >> 7)) * 512 + (((ccol & 31) << 4) | (((ccol >> 5) & 3) << 2) | (j & 3));
          } else {
            at = ((ragged ? bprefix[g] : static_cast<int64_t>(g) * bpg) + j) * cols + ccol;
          }
          // offsets that overlap (only possible without a status word) must
          // not push a write past the documented allocation
          if (at < scales_c_bytes) scales_c[at] = static_cast<uint8_t>(cbyte);
        }
      }

      if (kDbias) {
        // bias gradient: this lane's 4 rows per column (rows past the block's
        // valid rows were loaded as zeros), then the 8 row groups by a
        // butterfly (every lane ends with the same sums); lane rg stores
        // column col + rg
        float cs[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t w0 = (&raw[0].x)[k], w1 = (&raw[1].x)[k], w2 = (&raw[2].x)[k], w3 = (&raw[3].x)[k];
          cs[2 * k] = ((bf16_lo(w0) + bf16_lo(w1)) + bf16_lo(w2)) + bf16_lo(w3);
          cs[2 * k + 1] = ((bf16_hi(w0) + bf16_hi(w1)) + bf16_hi(w2)) + bf16_hi(w3);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          cs[k] += __shfl_xor_sync(0xffffffffu, cs[k], 4);
          cs[k] += __shfl_xor_sync(0xffffffffu, cs[k], 8);
          cs[k] += __shfl_xor_sync(0xffffffffu, cs[k], 16);
        }
        float mine = cs[0];
#pragma unroll
        for (int k = 1; k < 8; ++k)
          if (rg == k) mine = cs[k];
        const int ccol = col + rg;
        if (ccol < cols && pos.rb < part_blocks) part[pos.rb * cols + ccol] = mine;
      }
    }
    // this warp is done with stage s
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    step(pos);
  }
}

}  // namespace

gl_status launch_quantize(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                          int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                          uint8_t* codes_c, uint8_t* scales_c, int scale_layout, float* part,
                          int64_t part_blocks, int64_t* part_prefix, cudaStream_t stream) {
  // the source as a 2D bf16 tensor; box = one work unit (clamped to the tensor)
  const uint32_t box_cols = static_cast<uint32_t>(cols < kQCols ? cols : kQCols);
  const uint32_t box_rows = static_cast<uint32_t>(rows < kQRows ? rows : kQRows);
  CUtensorMap tm;
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(cols) * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  if (!encode_tmap(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, src, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
    return GL_ERR_UNSUPPORTED;
  const int prefix_bytes = row_offsets != nullptr ? 2 * (G + 1) * static_cast<int>(sizeof(int64_t)) : 0;
  const int box_bytes = static_cast<int>(box_cols * box_rows * 2);
  const int64_t sc_bytes = static_cast<int64_t>(gl_mxfp8_scale_bytes(rows, cols, G, 1, scale_layout));
  const int mma = scale_layout == GL_SCALES_MMA ? 1 : 0;
  auto run = [&](auto kern, int stages, int tile_bytes, int ctas_per_sm, float* pt, int64_t pb, int64_t* pp) {
    const int smem = 1024 + stages * tile_bytes + 128 + prefix_bytes;
    if (set_max_smem(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return GL_ERR_CUDA;
    kern<<<num_sms() * ctas_per_sm, kQThreads + 32, smem, stream>>>(
        tm, rows, cols, static_cast<int>(box_rows), box_bytes, row_offsets, G, status, codes_r, scales_r, codes_c,
        scales_c, sc_bytes, mma, pt, pb, pp);
    return GL_OK;
  };
  // two boxes per tile once the rows are wider than one box
  const bool wide = cols > kQCols;
  gl_status st;
  if (part != nullptr) {
    if (wide) st = run(quantize_kernel<true, 2>, QCfg<2>::kStages, QCfg<2>::kTileBytes, QCfg<2>::kCtasPerSm, part, part_blocks, part_prefix);
    else      st = run(quantize_kernel<true, 1>, QCfg<1>::kStages, QCfg<1>::kTileBytes, QCfg<1>::kCtasPerSm, part, part_blocks, part_prefix);
  } else {
    if (wide) st = run(quantize_kernel<false, 2>, QCfg<2>::kStages, QCfg<2>::kTileBytes, QCfg<2>::kCtasPerSm, nullptr, 0, nullptr);
    else      st = run(quantize_kernel<false, 1>, QCfg<1>::kStages, QCfg<1>::kTileBytes, QCfg<1>::kCtasPerSm, nullptr, 0, nullptr);
  }
  if (st != GL_OK) return st;
  return cudaGetLastError() == cudaSuccess ? GL_OK : GL_ERR_CUDA;
}

}  // namespace gl
