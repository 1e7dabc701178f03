// gl_gemm.cu -- persistent ragged grouped GEMM on sm_100a tensor cores (bf16).
//
// One kernel template serves the three products of the grouped linear layer
// (TransformerEngine ``grouped_linear.py``, ops/basic: fuser_forward "Perform
// GEMMs" and fuser_backward "Perform dgrad GEMMs" / "Perform wgrad GEMMs"):
//
//   FWD    y[r, n]          = sum_k x[r, k]  W_g[n, k]   (+ b_g[n])   rows r of group g
//   DGRAD  dx[r, k]         = sum_n dy[r, n] W_g[n, k]                rows r of group g
//   WGRAD  main_grad_g[n,k] (+)= sum_{r in g} dy[r, n] x[r, k]
//
// Persistent kernel, one CTA per SM.  With CG = 2 the CTAs of a cluster pair
// compute one 256 x 256 accumulator tile with tcgen05.mma.cta_group::2: each
// CTA streams its own 128 rows of A and its own half of B (no multicast
// loads), the peer CTA relays "stage landed" to the leader with a remote
// mbarrier arrive, the leader issues the MMAs and its tcgen05.commit
// multicasts stage-free / accumulator-full to both CTAs.  With CG = 1 a CTA
// computes a 128 x 256 tile alone.
//
// Roles: warp 0 TMA producer (128-byte swizzled boxes into a ring of
// shared-memory stages), warp 1 TMEM owner and MMA issuer (leader) or stage
// relay (peer), warps 2-5 epilogue (TMEM -> registers; bias + bf16 rounding
// and row-clipped stores for FWD/DGRAD; for WGRAD 32 x 32 fp32 chunks
// transposed through shared memory and added into main_grad with coalesced
// 16-byte vector reductions, or stored; each tile's main_grad rows are first
// pulled into L2 with bulk prefetches while its main loop runs).  Two accumulators in TMEM let a tile's
// epilogue overlap the next tile's main loop.  Tiles are enumerated group by
// group from the device offsets (tile prefix in shared memory): empty groups
// cost nothing and the host never learns the split sizes.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "gl_internal.h"
#include "gl_ptx.cuh"

namespace gl {
namespace {

constexpr int BK = 64;  // contraction elements of a K-major stage (one 128-byte swizzle row)
constexpr int kPG = 64;  // per-group tensor maps carried by one launch
constexpr int kSmemBudget = 212992;  // stage ring (pairs: 3 x 64 KB; single CTAs: 4 x 48 KB) + (wgrad) 16 KB of transposes
// Tile rows per rasterisation band: 16 for fwd (a band's A strips, 16 x 256
// rows of x, stay in L2 while the band sweeps W, which it reads once);
// dgrad's A strips span the whole N contraction (3.5x longer at the
// 14336-wide layer), so it keeps 8, as does wgrad (no measured difference).
template <int MODE>
__host__ __device__ constexpr int band_rows() { return MODE == kFwd ? 16 : 8; }

template <int MODE, int CG>
struct Cfg {
  static constexpr int kTileM = 128 * CG;          // accumulator rows per tile (pair)
  static constexpr int kTileN = 256;               // accumulator columns
  static constexpr int kBRows = kTileN / CG;       // rows of the B operand held per CTA
  // contraction elements per stage.  A K-major box spans one 128-byte row (64
  // elements); on CTA pairs a stage holds 128 (two boxes per K-major operand,
  // three stages of 64 KB): half the barrier round trips per flop, ~10%
  // faster for wgrad (both operands MN-major) and ~2.5% for fwd / dgrad.
  // Single CTAs keep 64, which leaves room for four 48 KB stages.
  static constexpr int kBK = (CG == 2) ? 128 : BK;
  static constexpr int kMNChunk = 128 * kBK;        // bytes of a 64-column MN-major chunk of a stage
  static constexpr int kABytes = 128 * kBK * 2;     // 32 KB (CG 2) or 16 KB (CG 1)
  static constexpr int kBBytes = kBRows * kBK * 2;  // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  // epilogue warps, one per TMEM lane quarter (eight for wgrad measured no
  // faster and cost a pipeline stage of staging space)
  static constexpr int kEpiWarps = 4;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kStagingBytes = (MODE == kWgrad) ? kEpiWarps * 32 * 32 * 4 : 0;  // one 4 KB transpose per epilogue warp
  static constexpr int kStages = (kSmemBudget - kStagingBytes) / kStageBytes;
  static constexpr int kBarOffset = kStages * kStageBytes + kStagingBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kPrefixOffset = kBarOffset + kBarBytes;
  // shared-memory majorness of the operands (1 = MN-major)
  static constexpr int kAMN = (MODE == kWgrad) ? 1 : 0;
  static constexpr int kBMN = (MODE == kFwd) ? 0 : 1;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, kTileN, kAMN, kBMN);
  static_assert(kStages >= 3, "pipeline too shallow");
  // dynamic shared memory at the largest group count (tile prefix), + alignment slack
  static_assert(kBarOffset + kBarBytes + (GL_MAX_GROUPS + 1) * 4 + 1024 <= 232448, "shared memory");
  static_assert(kBarOffset % 1024 == 0, "stage alignment");
};

struct GemmParams {
  CUtensorMap tmA;    // FWD x{K,M} box{64,128}; DGRAD dy{N,M} box{64,128}; WGRAD dy{N,M} box{64,kBK}
  CUtensorMap tmB;    // stacked W{K,N,G}: FWD box{64,BRows,1}, DGRAD box{64,kBK,1}; WGRAD x{K,M} box{64,kBK}
  const int64_t* offsets;  // G+1 entries
  int32_t* status;
  int64_t M;
  int64_t out_rows;
  void* out;                  // FWD y / DGRAD dx (bf16)
  float* mg;                  // WGRAD stacked main_grad [G, N, K]
  const __nv_bfloat16* bias;  // stacked bias [G,N] or null
  int G;
  int N, K;
  int has_bias;
  int accumulate;
  uint64_t wait_ns;  // bound on each pipeline wait
  int hold_loads;    // testing: the producer issues no loads
};

template <bool PG>
struct PGArgs {
  CUtensorMap tm[kPG];  // FWD/DGRAD: W_g{K,N}
  const __nv_bfloat16* bias[kPG];
  float* mg[kPG];       // WGRAD: main_grad_g [N, K]
  __device__ const CUtensorMap* map(int g) const { return &tm[g]; }
  __device__ const __nv_bfloat16* b(int g) const { return bias[g]; }
  __device__ float* m(int g) const { return mg[g]; }
};
template <>
struct PGArgs<false> {
  int unused;
  __device__ const CUtensorMap* map(int) const { return nullptr; }
  __device__ const __nv_bfloat16* b(int) const { return nullptr; }
  __device__ float* m(int) const { return nullptr; }
};

struct Tile {
  int g;
  int num_kb;
  int mt, nt;
  int64_t r0, r1;  // FWD/DGRAD: tile's first row, group end; WGRAD: contraction rows [r0, r1)
};

__device__ __forceinline__ int ceil_div_i(int64_t a, int b) { return static_cast<int>((a + b - 1) / b); }

template <int MODE, int CG>
__device__ __forceinline__ int tiles_of_group(int64_t m, const GemmParams& p) {
  using C = Cfg<MODE, CG>;
  if (MODE == kFwd) return m > 0 ? ceil_div_i(m, C::kTileM) * ceil_div_i(p.N, C::kTileN) : 0;
  if (MODE == kDgrad) return m > 0 ? ceil_div_i(m, C::kTileM) * ceil_div_i(p.K, C::kTileN) : 0;
  return (m > 0 || !p.accumulate) ? ceil_div_i(p.N, C::kTileM) * ceil_div_i(p.K, C::kTileN) : 0;
}

template <int MODE, int CG>
__device__ __forceinline__ Tile decode_tile(int t, const int* prefix, const GemmParams& p) {
  using C = Cfg<MODE, CG>;
  // largest g with prefix[g] <= t (prefix is non-decreasing, prefix[0] = 0)
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
  // Tile grid of the group: mtg x ntg.  Rasterise in bands of kBand tile
  // rows, column-major inside a band, so the ~#SMs tiles in flight cover a
  // near-square block and share operand strips through L2.
  const int mtg = (MODE == kWgrad) ? ceil_div_i(p.N, C::kTileM) : ceil_div_i(m, C::kTileM);
  const int ntg = ceil_div_i(MODE == kFwd ? p.N : p.K, C::kTileN);
  constexpr int kBand = band_rows<MODE>();
  const int band = local / (kBand * ntg);
  const int base_mt = band * kBand;
  const int bh = min(kBand, mtg - base_mt);
  const int within = local - band * kBand * ntg;
  if (MODE == kWgrad) {
    // row-major inside the band: consecutive tiles cover the same 256 main_grad
    // rows across the whole K width, so the fp32 read-modify-write of the
    // tiles in flight reaches DRAM as long contiguous runs
    tl.mt = base_mt + within / ntg;
    tl.nt = within % ntg;
  } else {
    tl.mt = base_mt + within % bh;
    tl.nt = within / bh;
  }
  if (MODE == kWgrad) {
    tl.r0 = o0;
    tl.r1 = o0 + m;
    tl.num_kb = ceil_div_i(m, C::kBK);
  } else {
    tl.r0 = o0 + static_cast<int64_t>(tl.mt) * C::kTileM;
    tl.r1 = o0 + m;
    tl.num_kb = ceil_div_i(MODE == kFwd ? p.K : p.N, C::kBK);
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
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), round to nearest even
  return *reinterpret_cast<uint32_t*>(&v);
}

// Zero rows [r_from, r_to) of this CTA's A and B stage buffers (MN-major,
// kBK rows x 128 bytes per chunk of 64 columns) so rows past a group's end
// add nothing to a wgrad contraction.  Executed by one full warp.
template <int MODE, int CG>
__device__ __forceinline__ void zero_tail_rows(uint8_t* sa, uint8_t* sb, int r_from, int r_to, int lane) {
  using C = Cfg<MODE, CG>;
  constexpr int kChunksA = 2, kChunksB = C::kBRows / 64;
  const int nrows = r_to - r_from;
  if (nrows <= 0) return;
  const int per_chunk = nrows * 8;  // 16-byte pieces per chunk
  for (int idx = lane; idx < (kChunksA + kChunksB) * per_chunk; idx += 32) {
    const int chunk = idx / per_chunk;
    const int rem = idx - chunk * per_chunk;
    const int row = r_from + (rem >> 3);
    uint8_t* base = (chunk < kChunksA) ? (sa + chunk * C::kMNChunk) : (sb + (chunk - kChunksA) * C::kMNChunk);
    *reinterpret_cast<uint4*>(base + row * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
}

template <int MODE, int CG, bool PG>
__global__ void __launch_bounds__(Cfg<MODE, CG>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ PGArgs<PG> pg) {
  using C = Cfg<MODE, CG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = abort_flag + 1;
  int* prefix = reinterpret_cast<int*>(smem + C::kPrefixOffset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    *skip_flag = (p.status != nullptr && *reinterpret_cast<volatile int32_t*>(p.status) != 0) ? 1 : 0;
    *abort_flag = 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], (CG == 2 && leader) ? 2 : 1);  // leader: own TMA + peer's relay
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kEpiWarps * CG);  // one arrival per epilogue warp of the pair
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  bool skip;
  if (CG == 2) {
    cluster_sync();  // barriers of both CTAs initialised; both skip flags written
    uint32_t peer_skip;
    asm volatile("ld.shared::cluster.u32 %0, [%1];"
                 : "=r"(peer_skip)
                 : "r"(mapa_shared(smem_u32(const_cast<int*>(skip_flag)), rank ^ 1u))
                 : "memory");
    skip = (*skip_flag != 0) || (peer_skip != 0);
    cluster_sync();  // nobody leaves before the peer has read its flag
  } else {
    __syncthreads();
    skip = *skip_flag != 0;
  }
  if (skip) return;  // bad split sizes reported by gl_offsets: write nothing

  const int pair = (CG == 2) ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int npairs = (CG == 2) ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == 0) {
    // tile prefix over groups: prefix[g] = number of tiles of groups < g
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int i = base + lane;
      int cnt = 0;
      if (i < p.G) {
        const int64_t m = __ldg(p.offsets + i + 1) - __ldg(p.offsets + i);
        cnt = tiles_of_group<MODE, CG>(m, p);
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, cnt, off);
        if (lane >= off) cnt += v;
      }
      if (i < p.G) prefix[i + 1] = carry + cnt;
      carry += __shfl_sync(0xffffffffu, cnt, 31);
    }
    if (lane == 0) prefix[0] = 0;
  } else if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(tmem_slot, 512);  // two 128 x 256 fp32 accumulators per CTA
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  } else if (warp == 2 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    if (!PG || MODE == kWgrad) tma_prefetch_desc(&p.tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[p.G];
  const int hr = static_cast<int>(rank) * 128;        // this CTA's A rows within the tile
  const int hb = static_cast<int>(rank) * C::kBRows;  // this CTA's B rows within the tile

  if (warp == 0) {
    // ===================== TMA producer (both CTAs) =====================
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = pair; t < total && !*abort_flag; t += npairs) {
        const Tile tl = decode_tile<MODE, CG>(t, prefix, p);
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.wait_ns)) { report_abort(abort_flag, p.status); break; }
          if (p.hold_loads) {  // testing the timeout path: this stage never lands
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            continue;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          if (MODE == kFwd) {
            const int n0 = tl.nt * C::kTileN + hb;
#pragma unroll
            for (int c = 0; c < C::kBK / 64; ++c) {
              tma_load_2d(sa + c * 16384, &p.tmA, &full[stage], kb * C::kBK + c * 64, static_cast<int32_t>(tl.r0 + hr));
              if (PG) tma_load_2d(sb + c * C::kBRows * 128, pg.map(tl.g), &full[stage], kb * C::kBK + c * 64, n0);
              else    tma_load_3d(sb + c * C::kBRows * 128, &p.tmB, &full[stage], kb * C::kBK + c * 64, n0, tl.g);
            }
          } else if (MODE == kDgrad) {
            const int n0 = tl.nt * C::kTileN + hb;
#pragma unroll
            for (int c = 0; c < C::kBK / 64; ++c)
              tma_load_2d(sa + c * 16384, &p.tmA, &full[stage], kb * C::kBK + c * 64, static_cast<int32_t>(tl.r0 + hr));
#pragma unroll
            for (int c = 0; c < C::kBRows / 64; ++c) {
              if (PG) tma_load_2d(sb + c * C::kMNChunk, pg.map(tl.g), &full[stage], n0 + c * 64, kb * C::kBK);
              else    tma_load_3d(sb + c * C::kMNChunk, &p.tmB, &full[stage], n0 + c * 64, kb * C::kBK, tl.g);
            }
          } else {
            // operand strips are read again by the neighbouring tiles of the
            // band: keep them in L2 ahead of the streamed main_grad lines
            const int32_t row = static_cast<int32_t>(tl.r0 + kb * C::kBK);
            const int m0 = tl.mt * C::kTileM + hr;
            const int n0 = tl.nt * C::kTileN + hb;
#pragma unroll
            for (int c = 0; c < 2; ++c) tma_load_2d_hint(sa + c * C::kMNChunk, &p.tmA, &full[stage], m0 + c * 64, row, keep);
#pragma unroll
            for (int c = 0; c < C::kBRows / 64; ++c)
              tma_load_2d_hint(sb + c * C::kMNChunk, &p.tmB, &full[stage], n0 + c * 64, row, keep);
          }
          ++issued;
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // Do not leave while a TMA load may still be writing shared memory: wait
      // for the last stages this thread filled.  On a pair the leader's stage
      // also waits for the peer's relay, which an aborted peer never sends, so
      // one 2 s budget covers the whole drain.
      const int inflight = issued < C::kStages ? issued : C::kStages;
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < inflight; ++i) {
        if (--s < 0) { s = C::kStages - 1; ph ^= 1u; }
        mbar_wait_until(&full[s], ph, deadline);
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ===================== MMA issuer =====================
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int t = pair; t < total; t += npairs, ++it) {
        const Tile tl = decode_tile<MODE, CG>(t, prefix, p);
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        // every lane waits; the warp acts on a unanimous result
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], tph ^ 1u, abort_flag, p.wait_ns))) {
          report_abort(abort_flag, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * C::kTileN;
        bool ok = true;
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          // On a ragged wgrad tail the peer zeroes rows of its stage before
          // relaying; acquire at cluster scope so those writes are visible.
          const bool peer_zeroed = CG == 2 && MODE == kWgrad && kb == tl.num_kb - 1 &&
                                   static_cast<int>(tl.r1 - tl.r0) - kb * C::kBK < C::kBK;
          const bool landed = peer_zeroed ? mbar_wait_acq_cluster(&full[stage], phase, abort_flag, p.wait_ns)
                                          : mbar_wait(&full[stage], phase, abort_flag, p.wait_ns);
          if (!__all_sync(0xffffffffu, landed)) {
            report_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          int ksteps = C::kBK / 16;
          if (MODE == kWgrad && kb == tl.num_kb - 1) {
            // Ragged contraction: skip whole 16-row MMA steps past the group's
            // end and zero the rows of the last partial step.
            const int valid = static_cast<int>(tl.r1 - tl.r0) - kb * C::kBK;
            if (valid < C::kBK) {
              ksteps = (valid + 15) >> 4;
              zero_tail_rows<MODE, CG>(sa, sb, valid, ksteps * 16, lane);
            }
          }
          __syncwarp();
          if (lane == 0) {
            // The single issuing thread is on the critical path: descriptors
            // are formed once per stage and advanced by constants (16-byte
            // units: 16 MN-major rows of 128 bytes, or 16 K-major elements
            // within a 64-element box, then the next box).
            const uint64_t ad0 = C::kAMN ? smem_desc_sw128(smem_u32(sa), C::kMNChunk, 1024)
                                         : smem_desc_sw128(smem_u32(sa), 16, 1024);
            const uint64_t bd0 = C::kBMN ? smem_desc_sw128(smem_u32(sb), C::kMNChunk, 1024)
                                         : smem_desc_sw128(smem_u32(sb), 16, 1024);
            auto issue = [&](int ks) {
              const uint32_t ao = C::kAMN ? ks * 128 : (ks >> 2) * 1024 + (ks & 3) * 2;
              const uint32_t bo = C::kBMN ? ks * 128 : (ks >> 2) * (C::kBRows * 8) + (ks & 3) * 2;
              const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
              if (CG == 2) mma_bf16_ss_pair(d_tmem, desc_add(ad0, ao), desc_add(bd0, bo), C::kIdesc, acc);
              else         mma_bf16_ss(d_tmem, desc_add(ad0, ao), desc_add(bd0, bo), C::kIdesc, acc);
            };
            if (ksteps == C::kBK / 16) {
#pragma unroll
              for (int ks = 0; ks < C::kBK / 16; ++ks) issue(ks);
            } else {
              for (int ks = 0; ks < ksteps; ++ks) issue(ks);
            }
            // free the stage (in both CTAs) once these MMAs have read it
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
          } else if (!p.hold_loads) {
            // nothing accumulated: the epilogues write zeros
            mbar_arrive(&tfull[buf]);
            if (CG == 2) mbar_arrive_cluster(mapa_shared(smem_u32(&tfull[buf]), 1));
          }
        }
        __syncwarp();
      }
      if (lane == 0) {
        if (CG == 2) tc_commit_pair_mc(mma_done, 0x1);
        else         tc_commit(mma_done);
        mbar_wait_bounded(mma_done, 0);  // no MMA in flight past this point
      }
      __syncwarp();
    } else {
      // ===================== peer: stage relay =====================
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < total; t += npairs) {
        const Tile tl = decode_tile<MODE, CG>(t, prefix, p);
        bool ok = true;
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag, p.wait_ns))) {
            report_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          bool zeroed = false;
          if (MODE == kWgrad && kb == tl.num_kb - 1) {
            const int valid = static_cast<int>(tl.r1 - tl.r0) - kb * C::kBK;
            if (valid < C::kBK) {
              uint8_t* sa = smem + stage * C::kStageBytes;
              zero_tail_rows<MODE, CG>(sa, sa + C::kABytes, valid, ((valid + 15) >> 4) * 16, lane);
              zeroed = true;
            }
          }
          __syncwarp();
          if (lane == 0) {
            const uint32_t leader_full = mapa_shared(smem_u32(&full[stage]), 0);
            if (zeroed) mbar_arrive_cluster_release(leader_full);  // the leader's MMA reads our zeroes
            else        mbar_arrive_cluster(leader_full);
          }
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
    }
  } else {
    // ===================== epilogue (warps 2..5, both CTAs) =====================
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    const uint32_t tempty_leader = (CG == 2) ? mapa_shared(smem_u32(tempty), 0) : 0u;
    auto prefetch_mg = [&](const Tile& tn) {
      constexpr int kCols = C::kTileN / (C::kEpiWarps / 4);
      const int n = tn.mt * C::kTileM + hr + q * 32 + lane;
      const int k0 = tn.nt * C::kTileN + ((warp - 2) >> 2) * kCols;
      const int cols = min(kCols, p.K - k0);
      if (n < p.N && cols > 0) {
        const float* gb = PG ? pg.m(tn.g) : p.mg + static_cast<int64_t>(tn.g) * p.N * p.K;
        l2_prefetch_bulk(gb + static_cast<int64_t>(n) * p.K + k0, static_cast<uint32_t>(cols) * 4u);
      }
    };
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const Tile tl = decode_tile<MODE, CG>(t, prefix, p);
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (MODE == kWgrad && p.accumulate) {
        // while the tile's main loop runs, pull this lane's main_grad row
        // segment into L2 with one bulk request, so that the reductions below
        // find their lines there (prefetching one tile further ahead measured
        // slower on small groups)
        prefetch_mg(tl);
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], tph, abort_flag, p.wait_ns));
      if (!ok) report_abort(abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * C::kTileN + (static_cast<uint32_t>(q * 32) << 16);
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
        if (MODE == kFwd && p.has_bias)
          bias = PG ? pg.b(tl.g) : (p.bias + static_cast<int64_t>(tl.g) * p.N);
        const int nchunks = min(C::kTileN / 32, ceil_div_i(Nout - tl.nt * C::kTileN, 32));
        for (int c = 0; c < nchunks; ++c) {
          const int n = tl.nt * C::kTileN + c * 32;
          uint32_t r[32];
          tmem_ld_32x32b_x32(tacc + c * 32, r);
          tmem_ld_wait();
          tmem_reg_fence(r);
          if (c == nchunks - 1) release_acc();  // accumulator fully read
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
        // main_grad rows n0 + 0..31 (this warp's TMEM lanes) x columns k0 + 32c..:
        // each [32 x 32] fp32 chunk goes through a 4 KB per-warp shared-memory
        // transpose (16-byte pieces, XOR-swizzled: conflict-free both ways), so
        // that 8 lanes cover one row's 128 contiguous bytes, then leaves as
        // coalesced 16-byte vector reductions (accumulate) or stores
        // (overwrite): full-line transactions, many in flight, no waits.
        float* stg = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes) + (warp - 2) * (32 * 32);
        constexpr int kCols = C::kTileN / (C::kEpiWarps / 4);  // columns of this warp (its half)
        const int half = (warp - 2) >> 2;
        const int n0 = tl.mt * C::kTileM + hr + q * 32;
        const int k0 = tl.nt * C::kTileN + half * kCols;
        const int nchunks = max(0, min(kCols / 32, ceil_div_i(p.K - k0, 32)));
        const bool have_acc = tl.num_kb > 0;
        float* gbase = PG ? pg.m(tl.g) : p.mg + static_cast<int64_t>(tl.g) * p.N * p.K;
        const int sub = lane >> 3, piece = lane & 7;  // read side: row 4i + sub, 16-byte piece
        for (int c = 0; c < nchunks; ++c) {
          uint32_t r[32];
          if (have_acc) {
            tmem_ld_32x32b_x32(tacc + half * kCols + c * 32, r);
            tmem_ld_wait();
            tmem_reg_fence(r);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0u;
          }
          if (c == nchunks - 1) release_acc();
          float* mine = stg + lane * 32;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(mine + ((j ^ (lane & 7)) << 2)) =
                make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          __syncwarp();
          const int col = k0 + c * 32 + piece * 4;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int row = 4 * i + sub;
            const uint4 v = *reinterpret_cast<const uint4*>(stg + row * 32 + ((piece ^ (row & 7)) << 2));
            if (n0 + row < p.N && col < p.K) {  // K % 8 == 0: four columns are all in or all out
              float* dst = gbase + static_cast<int64_t>(n0 + row) * p.K + col;
              if (p.accumulate) red_add_v4(dst, v.x, v.y, v.z, v.w);
              else *reinterpret_cast<uint4*>(dst) = v;
            }
          }
          __syncwarp();  // the next chunk overwrites the transpose buffer
        }
        if (nchunks == 0) release_acc();  // this warp's half lies past K: nothing to read
      }
    }
  }

  tc_fence_before();
  if (CG == 2) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2) tmem_dealloc_pair(tmem_base, 512);
    else         tmem_dealloc(tmem_base, 512);
  }
}

template <int MODE, int CG>
constexpr int smem_bytes_for(int G) {
  return Cfg<MODE, CG>::kPrefixOffset + (G + 1) * 4 + 1024;  // + alignment slack
}

bool make_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_in,
             uint32_t box_out, CUtensorMapDataType dt, int esize) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {inner * esize};
  const uint32_t box[2] = {box_in, box_out};
  return encode_tmap(m, dt, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
             uint32_t box_in, uint32_t box_mid, CUtensorMapDataType dt, int esize) {
  const uint64_t dims[3] = {inner, mid, outer};
  const uint64_t strides[2] = {inner * esize, inner * mid * esize};
  const uint32_t box[3] = {box_in, box_mid, 1};
  return encode_tmap(m, dt, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaLaunchConfig_t pair_config(int grid, int threads, int smem, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
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

// Persistent grid: one CTA per SM, or as many CTA pairs as can be resident.
template <typename Kern>
int grid_for(Kern kern, int cg, int threads, int smem) {
  if (cg == 1) return num_sms();
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
  cudaLaunchConfig_t cfg = pair_config(2 * (num_sms() / 2), threads, smem, nullptr, attr);
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters <= 0)
    nclusters = num_sms() / 2;
  const int grid = 2 * std::min(nclusters, num_sms() / 2);
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = grid;
  return grid;
}

template <int MODE, int CG, bool PG>
gl_status launch_one(const GemmParams& prm, const PGArgs<PG>& pga, int G, cudaStream_t stream) {
  const int smem = smem_bytes_for<MODE, CG>(G);
  auto kern = grouped_gemm_kernel<MODE, CG, PG>;
  if (set_max_smem(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return GL_ERR_CUDA;
  constexpr int threads = Cfg<MODE, CG>::kThreads;
  const int grid = grid_for(kern, CG, threads, smem);
  if (CG == 1) {
    kern<<<grid, threads, smem, stream>>>(prm, pga);
  } else {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config(grid, threads, smem, stream, attr);
    if (cudaLaunchKernelEx(&cfg, kern, prm, pga) != cudaSuccess) return GL_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? GL_OK : GL_ERR_CUDA;
}

template <int MODE, int CG>
gl_status launch_mode(const GemmCall& c) {
  using Cf = Cfg<MODE, CG>;
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  GemmParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.status = c.status;
  prm.M = c.M;
  prm.out_rows = c.out_rows;
  prm.out = c.out;
  prm.N = c.N;
  prm.K = c.K;
  prm.accumulate = c.accumulate;
  prm.wait_ns = c.wait_ns ? c.wait_ns : kWaitLimitNs;
  prm.hold_loads = c.hold_loads;
  prm.has_bias = (MODE == kFwd && c.bias != nullptr) ? 1 : 0;
  const uint64_t Mrows = c.M > 0 ? static_cast<uint64_t>(c.M) : 1;  // a map needs >= 1 row
  bool ok = true;
  if (MODE == kFwd) {
    ok &= make_2d(&prm.tmA, c.a, c.K, Mrows, BK, 128, BF, 2);
  } else if (MODE == kDgrad) {
    ok &= make_2d(&prm.tmA, c.a, c.N, Mrows, BK, 128, BF, 2);
  } else {
    ok &= make_2d(&prm.tmA, c.a, c.N, Mrows, 64, Cf::kBK, BF, 2);
    ok &= make_2d(&prm.tmB, c.b, c.K, Mrows, 64, Cf::kBK, BF, 2);
  }
  if (!ok) return GL_ERR_UNSUPPORTED;

  const bool stacked = (MODE == kWgrad) ? (c.out_grouped.mode == GL_STACKED) : (c.w.mode == GL_STACKED);
  const bool bias_stacked = prm.has_bias && c.bias->mode == GL_STACKED;
  if (stacked && (!prm.has_bias || bias_stacked)) {
    if (MODE == kFwd) ok &= make_3d(&prm.tmB, c.w.base, c.K, c.N, c.G, BK, Cf::kBRows, BF, 2);
    if (MODE == kDgrad) ok &= make_3d(&prm.tmB, c.w.base, c.K, c.N, c.G, 64, Cf::kBK, BF, 2);
    if (MODE == kWgrad) prm.mg = static_cast<float*>(const_cast<void*>(c.out_grouped.base));
    if (!ok) return GL_ERR_UNSUPPORTED;
    prm.offsets = c.offsets;
    prm.G = c.G;
    if (prm.has_bias) prm.bias = reinterpret_cast<const __nv_bfloat16*>(c.bias->base);
    PGArgs<false> none{0};
    return launch_one<MODE, CG, false>(prm, none, c.G, c.stream);
  }
  // Per-group pointers (weights, biases or main_grad): launches of <= kPG groups.
  PGArgs<true>* pga = new PGArgs<true>;
  gl_status st = GL_OK;
  for (int g0 = 0; g0 < c.G && st == GL_OK; g0 += kPG) {
    const int cg = (c.G - g0) < kPG ? (c.G - g0) : kPG;
    memset(pga, 0, sizeof(*pga));
    for (int i = 0; i < cg; ++i) {
      const int g = g0 + i;
      if (MODE == kFwd || MODE == kDgrad) {
        const void* wp = (c.w.mode == GL_STACKED)
                             ? static_cast<const uint8_t*>(c.w.base) + static_cast<size_t>(g) * c.N * c.K * 2
                             : c.w.ptrs[g];
        if (MODE == kFwd) ok &= make_2d(&pga->tm[i], wp, c.K, c.N, BK, Cf::kBRows, BF, 2);
        else              ok &= make_2d(&pga->tm[i], wp, c.K, c.N, 64, Cf::kBK, BF, 2);
        if (prm.has_bias)
          pga->bias[i] = reinterpret_cast<const __nv_bfloat16*>(
              c.bias->mode == GL_STACKED
                  ? static_cast<const uint8_t*>(c.bias->base) + static_cast<size_t>(g) * c.N * 2
                  : c.bias->ptrs[g]);
      } else {
        const void* gp = (c.out_grouped.mode == GL_STACKED)
                             ? static_cast<const uint8_t*>(c.out_grouped.base) + static_cast<size_t>(g) * c.N * c.K * 4
                             : c.out_grouped.ptrs[g];
        pga->mg[i] = static_cast<float*>(const_cast<void*>(gp));
      }
    }
    if (!ok) { st = GL_ERR_UNSUPPORTED; break; }
    prm.offsets = c.offsets + g0;
    prm.G = cg;
    st = launch_one<MODE, CG, true>(prm, *pga, cg, c.stream);
  }
  delete pga;
  return st;
}

template <int MODE>
gl_status launch_cg(const GemmCall& c) {
  return c.cta_pair ? launch_mode<MODE, 2>(c) : launch_mode<MODE, 1>(c);
}

}  // namespace

gl_status launch_grouped_gemm(const GemmCall& c) {
  switch (c.mode) {
    case kFwd: return launch_cg<kFwd>(c);
    case kDgrad: return launch_cg<kDgrad>(c);
    case kWgrad: return launch_cg<kWgrad>(c);
  }
  return GL_ERR_INVALID;
}

}  // namespace gl
