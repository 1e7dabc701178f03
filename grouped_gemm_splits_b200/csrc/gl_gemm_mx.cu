// gl_gemm_mx.cu -- persistent ragged grouped GEMM with MXFP8 operands
// (E4M3 codes, one E8M0 scale per 32 contraction elements) on sm_100a.
//
// The same three products as gl_gemm.cu (TransformerEngine ``grouped_linear.py``
// ops/basic fuser_forward / fuser_backward with MXFP8 quantizers: x and W
// rowwise for fprop, dy rowwise and W columnwise for dgrad, x and dy
// columnwise for wgrad), computed as sum_k (q_a 2^sa)(q_b 2^sb) by
// tcgen05.mma kind::mxf8f6f4.block_scale with fp32 accumulation in TMEM.
//
// Output tile 128*CG x 224.  With CG = 2 a cluster pair shares the tile
// (tcgen05 cta_group::2): each CTA loads its own 128 rows of A and 112 rows
// of B; the leader issues the MMAs.  Two 224-column fp32 accumulators
// (448 TMEM columns) leave 64 columns for per-stage scale-factor slots.
//
// Per stage (128 contraction elements = four MMAs of K=32) the producer
// TMA-loads the codes (128-byte swizzle) and the raw scales of the stage.
// A repack warp turns the raw scales into the 32-row x 16-byte blocks that
// tcgen05.cp.32x128b.warpx4 copies to TMEM (row i of a 128-row block at byte
// (i%32)*16 + ((i/32)%4)*4 + kb) -- each CTA packs the scales of its own A
// rows and of all 224 B rows -- and zeroes the rows of a ragged wgrad tail.
// The MMA warp then copies the scales to TMEM and issues the four MMAs,
// selecting scale byte kb of each MMA through the instruction descriptor.
// Rowwise scales arrive k-group-major ([cols/128][rows] words of four
// scales), columnwise scales as [blocks][cols] rows: one TMA box per stage.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "gl_internal.h"
#include "gl_ptx.cuh"

namespace gl {
namespace {

constexpr int BK = 128;  // fp8 contraction elements per stage (128 bytes)
constexpr int TN = 224;  // accumulator columns
constexpr int kThreads = 224;  // warp 0 TMA, 1 MMA, 2-5 epilogue, 6 scale repack
constexpr int kPG = 64;
constexpr int kBand = 8;
constexpr int kSfCol0 = 2 * TN;  // first TMEM column of the scale-factor slots
constexpr int kSfStage = 3072;   // raw A [0,528) | raw B [640,1536) | packed A 512 | packed B 1024
constexpr int kRawB = 640, kPackA = 1536, kPackB = 2048;

template <int MODE, int CG>
struct CfgMX {
  static constexpr int kTileM = 128 * CG;
  static constexpr int kBRows = TN / CG;  // B rows held per CTA (224 or 112)
  static constexpr int kABytes = 128 * BK;  // 16 KB
  // B codes per CTA: K-major kBRows x 128 B, MN-major 128-column chunks
  static constexpr int kBLoad = (MODE == kFwd) ? kBRows * BK : (CG == 1 ? 2 : 1) * 128 * BK;
  static constexpr int kOpStage = kABytes + (CG == 1 ? 2 : 1) * 128 * BK;  // 48 KB / 32 KB
  static constexpr int kStages = CG == 2 ? 5 : ((MODE == kWgrad) ? 3 : 4);
  static constexpr int kSfSlot = CG == 2 ? 12 : 16;  // TMEM columns per stage slot
  // rowwise A scales: 132 words from a 4-aligned row (TMA's first coordinate
  // must be 16-byte aligned); columnwise: 4 rows x 128 bytes
  static constexpr int kRawABytes = (MODE == kWgrad) ? 4 * 128 : (128 + 4) * 4;
  static constexpr int kRawBBytes = TN * 4;  // 896 either way
  static constexpr int kTx = kABytes + kBLoad + kRawABytes + kRawBBytes;
  static constexpr int kSfOffset = kStages * kOpStage;
  static constexpr int kStagingOffset = kSfOffset + kStages * kSfStage;
  static constexpr int kStagingBytes = (MODE == kWgrad) ? 4 * 2 * 32 * 32 * 4 : 0;
  static constexpr int kBarOffset = (kStagingOffset + kStagingBytes + 1023) / 1024 * 1024;
  static constexpr int kPrefixOffset = kBarOffset + 256;
  static_assert((3 * kStages + 5) * 8 + 16 <= 256, "barrier area");
  static_assert(kSfCol0 + kStages * kSfSlot <= 512, "TMEM columns");
  static_assert(kOpStage % 1024 == 0 && kSfOffset % 1024 == 0 && kStagingOffset % 1024 == 0, "alignment");
  // operand majorness in shared memory (1 = MN-major); scale source kind (1 = columnwise)
  static constexpr int kAMN = (MODE == kWgrad) ? 1 : 0;
  static constexpr int kBMN = (MODE == kFwd) ? 0 : 1;
  static constexpr int kSfaCol = (MODE == kWgrad) ? 1 : 0;
  static constexpr int kSfbCol = (MODE == kFwd) ? 0 : 1;
};

struct MxParams {
  CUtensorMap tmA;    // A codes: FWD x{K,M} / DGRAD dy{N,M} box{128,128}; WGRAD dy_c{N,M} box{128,128}
  CUtensorMap tmB;    // stacked B codes: FWD W{K,N,G} box{128,BRows,1}; DGRAD Wc{K,N,G} box{128,128,1}; WGRAD x_c{K,M} box{128,128}
  CUtensorMap tmSA;   // A scales: FWD/DGRAD k-group words {pitchM, Kc/128} box{132,1}; WGRAD dy_sc{N,S} box{128,4}
  CUtensorMap tmSB;   // stacked B scales: FWD {pitchGN, K/128} box{224,1}; DGRAD Wsc{K,G*N32} box{224,4}; WGRAD x_sc{K,S} box{224,4}
  CUtensorMap tmOut;  // WGRAD stacked main_grad{K,N,G} box{32,32,1}
  const int64_t* offsets;
  int32_t* status;
  int64_t out_rows;
  void* out;
  const __nv_bfloat16* bias;
  int G;
  int N, K;
  int n32;  // ceil(N/32): columnwise scale rows per weight group
  int has_bias;
  int accumulate;
};

template <bool PG>
struct MxPG {
  CUtensorMap tm[kPG];   // FWD/DGRAD: B codes of group g; WGRAD: main_grad of group g
  CUtensorMap tms[kPG];  // FWD/DGRAD: B scales of group g
  const __nv_bfloat16* bias[kPG];
  __device__ const CUtensorMap* map(int g) const { return &tm[g]; }
  __device__ const CUtensorMap* smap(int g) const { return &tms[g]; }
  __device__ const __nv_bfloat16* b(int g) const { return bias[g]; }
};
template <>
struct MxPG<false> {
  int unused;
  __device__ const CUtensorMap* map(int) const { return nullptr; }
  __device__ const CUtensorMap* smap(int) const { return nullptr; }
  __device__ const __nv_bfloat16* b(int) const { return nullptr; }
};

struct Tile {
  int g, num_kb, mt, nt;
  int64_t r0, r1;
};

__device__ __forceinline__ int cdiv(int64_t a, int b) { return static_cast<int>((a + b - 1) / b); }

template <int MODE, int CG>
__device__ __forceinline__ int tiles_of_group(int64_t m, const MxParams& p) {
  constexpr int TMt = CfgMX<MODE, CG>::kTileM;
  if (MODE == kFwd) return m > 0 ? cdiv(m, TMt) * cdiv(p.N, TN) : 0;
  if (MODE == kDgrad) return m > 0 ? cdiv(m, TMt) * cdiv(p.K, TN) : 0;
  return (m > 0 || !p.accumulate) ? cdiv(p.N, TMt) * cdiv(p.K, TN) : 0;
}

template <int MODE, int CG>
__device__ __forceinline__ Tile decode(int t, const int* prefix, const MxParams& p) {
  constexpr int TMt = CfgMX<MODE, CG>::kTileM;
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid;
  }
  Tile tl;
  tl.g = lo;
  const int local = t - prefix[lo];
  const int64_t o0 = __ldg(p.offsets + lo), o1 = __ldg(p.offsets + lo + 1);
  const int64_t m = o1 > o0 ? o1 - o0 : 0;
  const int mtg = (MODE == kWgrad) ? cdiv(p.N, TMt) : cdiv(m, TMt);
  const int ntg = cdiv(MODE == kFwd ? p.N : p.K, TN);
  const int band = local / (kBand * ntg);
  const int base_mt = band * kBand;
  const int bh = min(kBand, mtg - base_mt);
  const int within = local - band * kBand * ntg;
  tl.mt = base_mt + within % bh;
  tl.nt = within / bh;
  if (MODE == kWgrad) {
    tl.r0 = o0;
    tl.r1 = o0 + m;
    tl.num_kb = cdiv(m, BK);
  } else {
    tl.r0 = o0 + static_cast<int64_t>(tl.mt) * TMt;
    tl.r1 = o0 + m;
    tl.num_kb = (MODE == kFwd ? p.K : p.N) / BK;
  }
  return tl;
}

__device__ __forceinline__ void report_abort(volatile int* abort_flag, int32_t* status) {
  if (!*abort_flag) {
    *abort_flag = 1;
    if (status) atomicOr(status, GL_DEV_TIMEOUT);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Word offset of row i inside the packed scale blocks (512 bytes per 128 rows).
__device__ __forceinline__ int packed_word(int i) {
  return (i >> 7) * 128 + (i & 31) * 4 + ((i >> 5) & 3);
}

// Repack one operand's raw scales of a stage into the tcgen05.cp layout.
// Rowwise source: words (four scales of row i in word skip + i).  Columnwise
// source: 4 rows of `pitch` bytes (scale of block kb of row i at kb*pitch + i).
template <bool COLWISE>
__device__ __forceinline__ void pack_scales(const uint8_t* raw, uint32_t* packed, int R, int pitch, int skip,
                                            int lane) {
  for (int i = lane; i < R; i += 32) {
    uint32_t w;
    if (COLWISE) {
      w = static_cast<uint32_t>(raw[i]) | (static_cast<uint32_t>(raw[pitch + i]) << 8) |
          (static_cast<uint32_t>(raw[2 * pitch + i]) << 16) | (static_cast<uint32_t>(raw[3 * pitch + i]) << 24);
    } else {
      w = reinterpret_cast<const uint32_t*>(raw)[skip + i];
    }
    packed[packed_word(i)] = w;
  }
}

template <int MODE, int CG, bool PG>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ MxParams p, const __grid_constant__ MxPG<PG> pg) {
  using C = CfgMX<MODE, CG>;
  constexpr int TMt = C::kTileM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;
  uint64_t* ready = empty + C::kStages;  // stage's scales repacked (both CTAs of a pair)
  uint64_t* tfull = ready + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = abort_flag + 1;
  int* prefix = reinterpret_cast<int*>(smem + C::kPrefixOffset);  // tiles before group g
  int* bprefix = prefix + (p.G + 1);                             // 32-row blocks before group g

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    *skip_flag = (p.status != nullptr && *reinterpret_cast<volatile int32_t*>(p.status) != 0) ? 1 : 0;
    *abort_flag = 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], (CG == 2 && leader) ? 2 : 1);  // leader: both CTAs' repack warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4 * CG);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  bool skip;
  if (CG == 2) {
    cluster_sync();
    uint32_t peer_skip;
    asm volatile("ld.shared::cluster.u32 %0, [%1];"
                 : "=r"(peer_skip)
                 : "r"(mapa_shared(smem_u32(const_cast<int*>(skip_flag)), rank ^ 1u))
                 : "memory");
    skip = (*skip_flag != 0) || (peer_skip != 0);
    cluster_sync();
  } else {
    __syncthreads();
    skip = *skip_flag != 0;
  }
  if (skip) return;

  const int pair = (CG == 2) ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int npairs = (CG == 2) ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == 0) {
    int carry = 0, bcarry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int i = base + lane;
      int cnt = 0, bc = 0;
      if (i < p.G) {
        const int64_t m = __ldg(p.offsets + i + 1) - __ldg(p.offsets + i);
        cnt = tiles_of_group<MODE, CG>(m, p);
        bc = m > 0 ? cdiv(m, 32) : 0;
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, cnt, off);
        const int u = __shfl_up_sync(0xffffffffu, bc, off);
        if (lane >= off) { cnt += v; bc += u; }
      }
      if (i < p.G) { prefix[i + 1] = carry + cnt; bprefix[i + 1] = bcarry + bc; }
      carry += __shfl_sync(0xffffffffu, cnt, 31);
      bcarry += __shfl_sync(0xffffffffu, bc, 31);
    }
    if (lane == 0) { prefix[0] = 0; bprefix[0] = 0; }
  } else if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[p.G];
  const int hr = static_cast<int>(rank) * 128;       // this CTA's A rows within the tile
  const int hb = static_cast<int>(rank) * C::kBRows;  // this CTA's B rows within the tile

  if (warp == 0) {
    // ===================== TMA producer (both CTAs) =====================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = pair; t < total && !*abort_flag; t += npairs) {
        const Tile tl = decode<MODE, CG>(t, prefix, p);
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { report_abort(abort_flag, p.status); break; }
          uint8_t* sa = smem + stage * C::kOpStage;
          uint8_t* sb = sa + C::kABytes;
          uint8_t* sf = smem + C::kSfOffset + stage * kSfStage;
          uint64_t* bar = &full[stage];
          mbar_arrive_expect_tx(bar, C::kTx);
          const int n0 = tl.nt * TN;  // first B row (all 224 for the scales)
          const int32_t ra = static_cast<int32_t>(tl.r0 + hr);
          if (MODE == kFwd) {
            tma_load_2d(sa, &p.tmA, bar, kb * BK, ra);
            tma_load_2d(sf, &p.tmSA, bar, ra & ~3, kb);
            if (PG) {
              tma_load_2d(sb, pg.map(tl.g), bar, kb * BK, n0 + hb);
              tma_load_2d(sf + kRawB, pg.smap(tl.g), bar, n0, kb);
            } else {
              tma_load_3d(sb, &p.tmB, bar, kb * BK, n0 + hb, tl.g);
              tma_load_2d(sf + kRawB, &p.tmSB, bar, tl.g * p.N + n0, kb);
            }
          } else if (MODE == kDgrad) {
            tma_load_2d(sa, &p.tmA, bar, kb * BK, ra);
            tma_load_2d(sf, &p.tmSA, bar, ra & ~3, kb);
#pragma unroll
            for (int c = 0; c < (CG == 1 ? 2 : 1); ++c) {
              if (PG) tma_load_2d(sb + c * 16384, pg.map(tl.g), bar, n0 + hb + c * 128, kb * BK);
              else    tma_load_3d(sb + c * 16384, &p.tmB, bar, n0 + hb + c * 128, kb * BK, tl.g);
            }
            if (PG) tma_load_2d(sf + kRawB, pg.smap(tl.g), bar, n0, 4 * kb);
            else    tma_load_2d(sf + kRawB, &p.tmSB, bar, n0, tl.g * p.n32 + 4 * kb);
          } else {
            const int32_t row = static_cast<int32_t>(tl.r0 + kb * BK);
            const int32_t brow = bprefix[tl.g] + 4 * kb;  // scale row of this stage's first block
            const int m0 = tl.mt * TMt + hr;
            tma_load_2d(sa, &p.tmA, bar, m0, row);
#pragma unroll
            for (int c = 0; c < (CG == 1 ? 2 : 1); ++c) tma_load_2d(sb + c * 16384, &p.tmB, bar, n0 + hb + c * 128, row);
            tma_load_2d(sf, &p.tmSA, bar, m0, brow);
            tma_load_2d(sf + kRawB, &p.tmSB, bar, n0, brow);
          }
          ++issued;
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      const int inflight = issued < C::kStages ? issued : C::kStages;
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < inflight; ++i) {
        if (--s < 0) { s = C::kStages - 1; ph ^= 1u; }
        mbar_wait_bounded(&full[s], ph);
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ===================== scale copy + MMA issue =====================
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int t = pair; t < total; t += npairs, ++it) {
        const Tile tl = decode<MODE, CG>(t, prefix, p);
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], tph ^ 1u, abort_flag))) {
          report_abort(abort_flag, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * TN;
        bool ok = true;
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          // stage landed and repacked in this CTA (and, for a pair, in the peer)
          const bool rdy = mbar_wait(&full[stage], phase, abort_flag) &&
                           (CG == 2 ? mbar_wait_acq_cluster(&ready[stage], phase, abort_flag)
                                    : mbar_wait(&ready[stage], phase, abort_flag));
          if (!__all_sync(0xffffffffu, rdy)) {
            report_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + stage * C::kOpStage;
          uint8_t* sb = sa + C::kABytes;
          uint8_t* sf = smem + C::kSfOffset + stage * kSfStage;
          int ksteps = BK / 32;
          if (MODE == kWgrad && kb == tl.num_kb - 1) {
            const int valid = static_cast<int>(tl.r1 - tl.r0) - kb * BK;
            if (valid < BK) ksteps = (valid + 31) >> 5;
          }
          if (lane == 0) {
            const uint32_t sfa = tmem_base + kSfCol0 + stage * C::kSfSlot, sfb = sfa + 4;
            const uint32_t pa = smem_u32(sf + kPackA), pb = smem_u32(sf + kPackB);
            if (CG == 2) {
              tmem_cp_32x128b_x4_pair(sfa, smem_desc_sf(pa));
              tmem_cp_32x128b_x4_pair(sfb, smem_desc_sf(pb));
              tmem_cp_32x128b_x4_pair(sfb + 4, smem_desc_sf(pb + 512));
            } else {
              tmem_cp_32x128b_x4(sfa, smem_desc_sf(pa));
              tmem_cp_32x128b_x4(sfb, smem_desc_sf(pb));
              tmem_cp_32x128b_x4(sfb + 4, smem_desc_sf(pb + 512));
            }
            const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
            for (int ks = 0; ks < ksteps; ++ks) {
              const uint64_t ad = C::kAMN ? smem_desc_sw128(a0 + ks * 4096, 16384, 1024)
                                          : smem_desc_sw128(a0 + ks * 32, 16, 1024);
              const uint64_t bd = C::kBMN ? smem_desc_sw128(b0 + ks * 4096, 16384, 1024)
                                          : smem_desc_sw128(b0 + ks * 32, 16, 1024);
              const uint32_t idesc = idesc_mxf8(TMt, TN, C::kAMN, C::kBMN, ks, ks);
              const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
              if (CG == 2) mma_mxf8_ss_pair(d_tmem, ad, bd, idesc, sfa, sfb, acc);
              else         mma_mxf8_ss(d_tmem, ad, bd, idesc, sfa, sfb, acc);
            }
            if (CG == 2) tc_commit_pair_mc(&empty[stage], 0x3);
            else         tc_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (lane == 0) {
          if (tl.num_kb > 0) {
            if (CG == 2) tc_commit_pair_mc(&tfull[buf], 0x3);
            else         tc_commit(&tfull[buf]);
          } else {
            mbar_arrive(&tfull[buf]);
            if (CG == 2) mbar_arrive_cluster(mapa_shared(smem_u32(&tfull[buf]), 1));
          }
        }
        __syncwarp();
      }
      if (lane == 0) {
        if (CG == 2) tc_commit_pair_mc(mma_done, 0x1);
        else         tc_commit(mma_done);
        mbar_wait_bounded(mma_done, 0);
      }
      __syncwarp();
    }
  } else if (warp == 6) {
    // ===================== scale repack (and wgrad tail zeroing) =====================
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t ready_leader = (CG == 2) ? mapa_shared(smem_u32(ready), 0) : 0u;
    for (int t = pair; t < total; t += npairs) {
      const Tile tl = decode<MODE, CG>(t, prefix, p);
      bool ok = true;
      for (int kb = 0; kb < tl.num_kb; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) {
          report_abort(abort_flag, p.status);
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * C::kOpStage;
        uint8_t* sb = sa + C::kABytes;
        uint8_t* sf = smem + C::kSfOffset + stage * kSfStage;
        if (MODE == kWgrad && kb == tl.num_kb - 1) {
          // ragged contraction: zero the code rows of the last partial 32-row
          // MMA step (A: one 128-column chunk, B: 1 or 2; 128 bytes per row);
          // the MMA warp skips the steps past the group's end
          const int valid = static_cast<int>(tl.r1 - tl.r0) - kb * BK;
          if (valid < BK) {
            constexpr int kChunks = 1 + (CG == 1 ? 2 : 1);
            const int nrows = ((valid + 31) >> 5) * 32 - valid;
            const int per_chunk = nrows * 8;
            for (int idx = lane; idx < kChunks * per_chunk; idx += 32) {
              const int chunk = idx / per_chunk;
              const int rem = idx - chunk * per_chunk;
              const int r = valid + (rem >> 3);
              uint8_t* base = chunk == 0 ? sa : (sb + (chunk - 1) * 16384);
              *reinterpret_cast<uint4*>(base + r * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
          }
        }
        pack_scales<C::kSfaCol != 0>(sf, reinterpret_cast<uint32_t*>(sf + kPackA), 128, 128,
                                     static_cast<int>((tl.r0 + hr) & 3), lane);
        pack_scales<C::kSfbCol != 0>(sf + kRawB, reinterpret_cast<uint32_t*>(sf + kPackB), TN, TN, 0, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // the leader's MMAs read this CTA's zeroed codes and packed scales
          if (CG == 2) mbar_arrive_cluster_release(ready_leader + stage * 8);
          else         mbar_arrive(&ready[stage]);
        }
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else {
    // ===================== epilogue (warps 2..5, both CTAs) =====================
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const uint32_t tempty_leader = (CG == 2) ? mapa_shared(smem_u32(tempty), 0) : 0u;
    int it = 0;
    int chunk_ctr = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const Tile tl = decode<MODE, CG>(t, prefix, p);
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], tph, abort_flag));
      if (!ok) report_abort(abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * TN + (static_cast<uint32_t>(q * 32) << 16);
      auto release_acc = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2) mbar_arrive_cluster(tempty_leader + buf * 8);
          else         mbar_arrive(&tempty[buf]);
        }
      };
      if (MODE != kWgrad) {
        const int Nout = (MODE == kFwd) ? p.N : p.K;
        const int64_t row = tl.r0 + hr + row_in_tile;
        const bool row_ok = row >= 0 && row < tl.r1 && row < p.out_rows;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
        const __nv_bfloat16* bias = nullptr;
        if (MODE == kFwd && p.has_bias) bias = PG ? pg.b(tl.g) : (p.bias + static_cast<int64_t>(tl.g) * p.N);
        const int nchunks = min(TN / 32, cdiv(Nout - tl.nt * TN, 32));
        for (int c = 0; c < nchunks; ++c) {
          const int n = tl.nt * TN + c * 32;
          uint32_t r[32];
          tmem_ld_32x32b_x32(tacc + c * 32, r);
          tmem_ld_wait();
          if (c == nchunks - 1) release_acc();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          if (bias != nullptr) {
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
              if (n + j8 * 8 < Nout) {
                const uint4 bv = __ldg(reinterpret_cast<const uint4*>(bias + n + j8 * 8));
                const __nv_bfloat16* bb = reinterpret_cast<const __nv_bfloat16*>(&bv);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j8 * 8 + j] += __bfloat162float(bb[j]);
              }
            }
          }
          if (row_ok) {
            __nv_bfloat16* dst = out + row * static_cast<int64_t>(Nout) + n;
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
              if (n + j8 * 8 < Nout) {
                uint4 w;
                w.x = pack_bf16x2(v[j8 * 8 + 0], v[j8 * 8 + 1]);
                w.y = pack_bf16x2(v[j8 * 8 + 2], v[j8 * 8 + 3]);
                w.z = pack_bf16x2(v[j8 * 8 + 4], v[j8 * 8 + 5]);
                w.w = pack_bf16x2(v[j8 * 8 + 6], v[j8 * 8 + 7]);
                *reinterpret_cast<uint4*>(dst + j8 * 8) = w;
              }
            }
          }
        }
      } else {
        // main_grad rows n0.. (this warp's 32 TMEM lanes) x cols k0 + 32c: each
        // epilogue warp stages and stores its own [32 x 32] fp32 boxes
        float* wstage = reinterpret_cast<float*>(smem + C::kStagingOffset) + (warp - 2) * (2 * 32 * 32);
        const int n0 = tl.mt * TMt + hr + q * 32;
        const int k0 = tl.nt * TN;
        const int nchunks = min(TN / 32, cdiv(p.K - k0, 32));
        const bool have_acc = tl.num_kb > 0;
        const bool rows_in = n0 < p.N;
        for (int c = 0; c < nchunks; ++c, ++chunk_ctr) {
          float* stg = wstage + (chunk_ctr & 1) * (32 * 32);
          if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
          __syncwarp();
          uint32_t r[32];
          if (have_acc) {
            tmem_ld_32x32b_x32(tacc + c * 32, r);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0u;
          }
          if (c == nchunks - 1) release_acc();
          uint8_t* rowp = reinterpret_cast<uint8_t*>(stg) + lane * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int pj = j ^ (lane & 7);
            *reinterpret_cast<uint4*>(rowp + pj * 16) = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && rows_in) {
            const int kc = k0 + c * 32;
            if (PG) {
              if (p.accumulate) tma_reduce_add_2d(pg.map(tl.g), stg, kc, n0);
              else              tma_store_2d(pg.map(tl.g), stg, kc, n0);
            } else {
              if (p.accumulate) tma_reduce_add_3d(&p.tmOut, stg, kc, n0, tl.g);
              else              tma_store_3d(&p.tmOut, stg, kc, n0, tl.g);
            }
            bulk_commit_group();
          }
        }
      }
    }
    if (MODE == kWgrad && lane == 0) bulk_wait_group<0>();  // stores of this warp done
  }

  tc_fence_before();
  if (CG == 2) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2) tmem_dealloc_pair(tmem_base, 512);
    else         tmem_dealloc(tmem_base, 512);
  }
}

bool map2(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes,
          uint32_t bi, uint32_t bo, CUtensorMapDataType dt, CUtensorMapSwizzle sw) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {pitch_bytes};
  const uint32_t box[2] = {bi, bo};
  return encode_tmap(m, dt, 2, base, dims, strides, box, sw);
}

bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer, int esize,
          uint32_t bi, uint32_t bm, CUtensorMapDataType dt) {
  const uint64_t dims[3] = {inner, mid, outer};
  const uint64_t strides[2] = {inner * esize, inner * mid * esize};
  const uint32_t box[3] = {bi, bm, 1};
  return encode_tmap(m, dt, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int MODE, int CG>
constexpr int mx_smem_bytes(int G) {
  return CfgMX<MODE, CG>::kPrefixOffset + 2 * (G + 1) * 4 + 1024;
}

cudaLaunchConfig_t pair_cfg(int grid, int smem, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <typename Kern>
int pair_grid(Kern kern, int smem) {
  static std::mutex mu;
  static std::unordered_map<const void*, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const void* key = reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(kern) ^ (static_cast<uintptr_t>(dev) << 48));
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_cfg(2 * (num_sms() / 2), smem, nullptr, attr);
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters <= 0)
    nclusters = num_sms() / 2;
  const int grid = 2 * std::min(nclusters, num_sms() / 2);
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = grid;
  return grid;
}

template <int MODE, int CG, bool PG>
gl_status mx_launch(const MxParams& prm, const MxPG<PG>& pga, int G, cudaStream_t stream) {
  const int smem = mx_smem_bytes<MODE, CG>(G);
  auto kern = grouped_gemm_mx_kernel<MODE, CG, PG>;
  if (set_max_smem(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return GL_ERR_CUDA;
  if (CG == 1) {
    kern<<<num_sms(), kThreads, smem, stream>>>(prm, pga);
  } else {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_cfg(pair_grid(kern, smem), smem, stream, attr);
    if (cudaLaunchKernelEx(&cfg, kern, prm, pga) != cudaSuccess) return GL_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? GL_OK : GL_ERR_CUDA;
}

const void* group_ptr(const gl_grouped& g, int i, size_t stride_bytes) {
  return g.mode == GL_STACKED ? static_cast<const uint8_t*>(g.base) + stride_bytes * i : g.ptrs[i];
}

template <int MODE, int CG>
gl_status mx_mode(const MxCall& c) {
  using Cf = CfgMX<MODE, CG>;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const auto U32 = CU_TENSOR_MAP_DATA_TYPE_UINT32;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  const auto NOSW = CU_TENSOR_MAP_SWIZZLE_NONE;
  MxParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.status = c.status;
  prm.out_rows = c.out_rows;
  prm.out = c.out;
  prm.N = c.N;
  prm.K = c.K;
  prm.n32 = (c.N + 31) / 32;
  prm.accumulate = c.accumulate;
  prm.has_bias = (MODE == kFwd && c.bias != nullptr) ? 1 : 0;
  const uint64_t M = c.M > 0 ? static_cast<uint64_t>(c.M) : 1;
  const uint64_t pitchM = (M + 3) / 4 * 4;
  const uint64_t S = (M + 31) / 32 + c.G;  // columnwise scale rows allocated by the caller
  const uint32_t BR = Cf::kBRows;
  bool ok = true;
  if (MODE == kFwd) {
    ok &= map2(&prm.tmA, c.a, c.K, M, c.K, 128, 128, U8, SW);
    ok &= map2(&prm.tmSA, c.sa, pitchM, c.K / 128, pitchM * 4, 128 + 4, 1, U32, NOSW);
  } else if (MODE == kDgrad) {
    ok &= map2(&prm.tmA, c.a, c.N, M, c.N, 128, 128, U8, SW);
    ok &= map2(&prm.tmSA, c.sa, pitchM, c.N / 128, pitchM * 4, 128 + 4, 1, U32, NOSW);
  } else {
    ok &= map2(&prm.tmA, c.a, c.N, M, c.N, 128, 128, U8, SW);
    ok &= map2(&prm.tmB, c.b, c.K, M, c.K, 128, 128, U8, SW);
    ok &= map2(&prm.tmSA, c.sa, c.N, S, c.N, 128, 4, U8, NOSW);
    ok &= map2(&prm.tmSB, c.sb, c.K, S, c.K, TN, 4, U8, NOSW);
  }
  if (!ok) return GL_ERR_UNSUPPORTED;

  const bool stacked = (MODE == kWgrad) ? c.out_grouped.mode == GL_STACKED
                                        : (c.w.mode == GL_STACKED && c.ws.mode == GL_STACKED);
  const bool bias_ok = !prm.has_bias || c.bias->mode == GL_STACKED;
  if (stacked && bias_ok) {
    if (MODE == kFwd) {
      const uint64_t GN = static_cast<uint64_t>(c.G) * c.N, pitchGN = (GN + 3) / 4 * 4;
      ok &= map3(&prm.tmB, c.w.base, c.K, c.N, c.G, 1, 128, BR, U8);
      ok &= map2(&prm.tmSB, c.ws.base, pitchGN, c.K / 128, pitchGN * 4, TN, 1, U32, NOSW);
    } else if (MODE == kDgrad) {
      ok &= map3(&prm.tmB, c.w.base, c.K, c.N, c.G, 1, 128, 128, U8);
      ok &= map2(&prm.tmSB, c.ws.base, c.K, static_cast<uint64_t>(c.G) * prm.n32, c.K, TN, 4, U8, NOSW);
    } else {
      ok &= map3(&prm.tmOut, c.out_grouped.base, c.K, c.N, c.G, 4, 32, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
    }
    if (!ok) return GL_ERR_UNSUPPORTED;
    prm.offsets = c.offsets;
    prm.G = c.G;
    if (prm.has_bias) prm.bias = reinterpret_cast<const __nv_bfloat16*>(c.bias->base);
    MxPG<false> none{0};
    return mx_launch<MODE, CG, false>(prm, none, c.G, c.stream);
  }
  MxPG<true>* pga = new MxPG<true>;
  gl_status st = GL_OK;
  for (int g0 = 0; g0 < c.G && st == GL_OK; g0 += kPG) {
    const int cg = std::min(kPG, c.G - g0);
    memset(pga, 0, sizeof(*pga));
    for (int i = 0; i < cg; ++i) {
      const int g = g0 + i;
      if (MODE == kWgrad) {
        const void* gp = group_ptr(c.out_grouped, g, static_cast<size_t>(c.N) * c.K * 4);
        ok &= map2(&pga->tm[i], gp, c.K, c.N, static_cast<uint64_t>(c.K) * 4, 32, 32,
                   CU_TENSOR_MAP_DATA_TYPE_FLOAT32, SW);
        continue;
      }
      const void* wp = group_ptr(c.w, g, static_cast<size_t>(c.N) * c.K);
      if (MODE == kFwd) {
        const uint64_t pitchN = (static_cast<uint64_t>(c.N) + 3) / 4 * 4;
        const uint64_t GN = static_cast<uint64_t>(c.G) * c.N, pitchGN = (GN + 3) / 4 * 4;
        ok &= map2(&pga->tm[i], wp, c.K, c.N, c.K, 128, BR, U8, SW);
        if (c.ws.mode == GL_STACKED) {
          // group g's rows of the stacked [K/128][pitch(G*N)] scale array
          const void* sp = static_cast<const uint8_t*>(c.ws.base) + static_cast<size_t>(g) * c.N * 4;
          ok &= map2(&pga->tms[i], sp, c.N, c.K / 128, pitchGN * 4, TN, 1, U32, NOSW);
        } else {
          ok &= map2(&pga->tms[i], c.ws.ptrs[g], pitchN, c.K / 128, pitchN * 4, TN, 1, U32, NOSW);
        }
      } else {
        ok &= map2(&pga->tm[i], wp, c.K, c.N, c.K, 128, 128, U8, SW);
        const void* sp = group_ptr(c.ws, g, static_cast<size_t>(prm.n32) * c.K);
        ok &= map2(&pga->tms[i], sp, c.K, prm.n32, c.K, TN, 4, U8, NOSW);
      }
      if (prm.has_bias)
        pga->bias[i] = reinterpret_cast<const __nv_bfloat16*>(group_ptr(*c.bias, g, static_cast<size_t>(c.N) * 2));
    }
    if (!ok) { st = GL_ERR_UNSUPPORTED; break; }
    prm.offsets = c.offsets + g0;
    prm.G = cg;
    st = mx_launch<MODE, CG, true>(prm, *pga, cg, c.stream);
  }
  delete pga;
  return st;
}

template <int MODE>
gl_status mx_cg(const MxCall& c) {
  return c.cta_pair ? mx_mode<MODE, 2>(c) : mx_mode<MODE, 1>(c);
}

}  // namespace

gl_status launch_grouped_gemm_mx(const MxCall& c) {
  switch (c.mode) {
    case kFwd: return mx_cg<kFwd>(c);
    case kDgrad: return mx_cg<kDgrad>(c);
    case kWgrad: return mx_cg<kWgrad>(c);
  }
  return GL_ERR_INVALID;
}

}  // namespace gl
