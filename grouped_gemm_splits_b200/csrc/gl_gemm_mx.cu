// gl_gemm_mx.cu -- persistent ragged grouped GEMM with MXFP8 operands
// (E4M3 codes, one E8M0 scale per 32 contraction elements) on sm_100a.
//
// The same three products as gl_gemm.cu (TransformerEngine ``grouped_linear.py``
// ops/basic fuser_forward / fuser_backward with MXFP8 quantizers: x and W
// rowwise for fprop, dy rowwise and W columnwise for dgrad, x and dy
// columnwise for wgrad), computed as sum_k (q_a 2^sa)(q_b 2^sb) by
// tcgen05.mma kind::mxf8f6f4.block_scale with fp32 accumulation in TMEM.
//
// Output tile 128*CG x 256.  With CG = 2 a cluster pair shares the tile
// (tcgen05 cta_group::2): each CTA loads its own 128 rows of A and 128 rows
// of B; the peer relays "stage landed" to the leader, which issues the MMAs.
// One fp32 accumulator (256 TMEM columns) per tile: eight epilogue warps (two
// per TMEM lane quarter, 128 columns each) copy it to registers and free it
// at once, so the next tile's MMAs overlap the stores -- fprop / dgrad round
// to bf16 (+ bias); wgrad transposes 32 x 16 fp32 pieces through shared
// memory and adds them into main_grad with coalesced 16-byte vector
// reductions (each tile's main_grad rows first pulled into L2 with bulk
// prefetches).  The remaining TMEM columns hold the scale-factor slots.
//
// Per sub-stage (128 contraction elements = four MMAs of K=32; a stage holds
// two on CTA pairs, one on single CTAs) the producer TMA-loads
// the codes (128-byte swizzle) and the scales.  The scales arrive from the
// quantizer in 512-byte atoms that already have the tcgen05 scale-factor
// layout (128 operand rows x 4 blocks; row i at byte (i%32)*16 + ((i/32)%4)*4
// + block), so a sub-stage's scales are two plain boxes: one atom for the
// CTA's 128 A rows and two consecutive atoms (256 rows) covering the tile's B
// rows.  The MMA thread copies them to TMEM with tcgen05.cp.32x128b.warpx4
// and selects scale byte kb of each MMA through the instruction descriptor.  A tiles (fprop / dgrad) start on 128-row
// boundaries of the packed activations: a group's first tile may begin inside
// the previous group, and only the group's own rows are stored.
//
// The only generic shared-memory writes on the main loop are the zeroed rows
// of a ragged wgrad contraction tail (once per tile); on a pair the peer
// publishes them with a cluster-scope release that the leader acquires.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "gl_internal.h"
#include "gl_ptx.cuh"

namespace gl {
namespace {

constexpr int BK = 128;  // fp8 contraction elements per sub-stage (128 bytes: one swizzle row, one scale k-group)
constexpr int kPG = 64;
constexpr int kBand = 16;  // tile rows per rasterisation band
constexpr int kSfSlots = 4;      // slot j: A at +0 (4 columns), B at +4 (8 columns)
constexpr int kSfSlotCols = 16;
constexpr int kSfABytes = 512;   // one atom
constexpr int kAtomsB = 2;       // the 256 B rows of a tile
constexpr int kSfBytes = 2048;   // a sub-stage's A atom + B atoms, padded to keep stages 1 KB aligned
constexpr int kWgradSub = 2;     // sub-stages per wgrad stage on CTA pairs
constexpr int kWgradMaxG = 256;  // groups per wgrad launch (their tile / scale prefixes share the shared memory)
static_assert(kSfABytes + kAtomsB * 512 <= kSfBytes, "scale staging");

template <int MODE, int CG>
struct CfgMX {
  static constexpr int kTN = 256;     // accumulator columns
  static constexpr int kAccBufs = 1;  // drained to registers at once, so the next tile's MMAs overlap the stores
  static constexpr int kEpiWarps = 8;  // two per TMEM lane quarter, half the columns each
  static constexpr int kThreads = 64 + 32 * kEpiWarps;  // warp 0 TMA, 1 MMA / relay, then epilogue
  static constexpr int kSfCol0 = kAccBufs * kTN;        // first TMEM column of the scale-factor slots
  static constexpr int kTileM = 128 * CG;
  static constexpr int kBRows = kTN / CG;  // B rows held per CTA
  // A stage holds kSub sub-stages of 128 contraction elements, each with its
  // own codes and scale atoms: two on CTA pairs (half the barrier round trips
  // per MMA: fprop / dgrad ~8% faster, wgrad's large groups ~9%; wgrad then
  // keeps three stages by taking at most 256 groups a launch and transposing
  // through 2 KB a warp), one on single CTAs.
  static constexpr int kSub = (CG == 2) ? ((MODE == kWgrad) ? kWgradSub : 2) : 1;
  static constexpr int kA1 = 128 * BK;  // A codes of a sub-stage: 16 KB
  // B codes per CTA and sub-stage: K-major kBRows x 128 B, MN-major 128-column chunks
  static constexpr int kBChunks = (kBRows + 127) / 128;
  static constexpr int kB1 = (MODE == kFwd) ? kBRows * BK : kBChunks * 128 * BK;
  static constexpr int kABytes = kSub * kA1;
  static constexpr int kBAlloc = kSub * kB1;
  static_assert(kTN == 128 * kAtomsB, "a B tile is exactly the loaded scale atoms");
  static constexpr int kStageBytes = kABytes + kBAlloc + kSub * kSfBytes;
  static constexpr int kStagingBytes = (MODE == kWgrad) ? kEpiWarps * 32 * 16 * 4 : 0;  // one 2 KB transpose per epilogue warp
  static constexpr int kMaxG = (MODE == kWgrad) ? kWgradMaxG : GL_MAX_GROUPS_MXFP8;  // groups per launch
  // as many stages as fit beside the barriers and the tile / scale prefixes
  // at the largest group count (at most six)
  static constexpr int kFit = (232448 - 1024 - 256 - 2 * (kMaxG + 1) * 4 - kStagingBytes) / kStageBytes;
  static constexpr int kStages = kFit < 6 ? kFit : 6;
  static_assert(kStages >= 2, "pipeline too shallow");
  static constexpr int kTx = kABytes + kBAlloc + kSub * (kSfABytes + kAtomsB * 512);
  static constexpr int kStagingOffset = kStages * kStageBytes;
  static constexpr int kBarOffset = kStagingOffset + kStagingBytes;
  static constexpr int kPrefixOffset = kBarOffset + 256;
  static_assert((2 * kStages + 5) * 8 + 16 <= 256, "barrier area");
  static_assert(kSfCol0 + kSfSlots * kSfSlotCols <= 512, "TMEM columns");
  // dynamic shared memory at the largest group count (tile and scale prefixes), + alignment slack
  static_assert(kPrefixOffset + 2 * (kMaxG + 1) * 4 + 1024 <= 232448, "shared memory");
  static_assert(kPG <= kMaxG, "per-group launches");
  static_assert(kStageBytes % 1024 == 0, "alignment");
  // operand majorness in shared memory (1 = MN-major)
  static constexpr int kAMN = (MODE == kWgrad) ? 1 : 0;
  static constexpr int kBMN = (MODE == kFwd) ? 0 : 1;
};

struct MxParams {
  CUtensorMap tmA;    // A codes: FWD x{K,M} / DGRAD dy{N,M} box{128,128}; WGRAD dy_c{N,M} box{128,128}
  CUtensorMap tmB;    // stacked B codes: FWD W{K,N,G} box{128,BRows,1}; DGRAD Wc{K,N,G} box{128,128,1}; WGRAD x_c{K,M} box{128,128}
  CUtensorMap tmSA;   // A scale atoms (u32 {128, atoms, k-groups}) box{128,1,1}
  CUtensorMap tmSB;   // stacked B scale atoms box{128,2,1}
  const int64_t* offsets;      // this launch's G+1 offsets
  const int64_t* offsets_all;  // every group's offsets (WGRAD scale k-groups of earlier groups)
  int32_t* status;
  int64_t out_rows;
  void* out;
  float* mg;  // WGRAD stacked main_grad [G, N, K]
  const __nv_bfloat16* bias;
  int G;
  int g0;  // index of this launch's first group
  int N, K;
  int has_bias;
  int accumulate;
  uint64_t wait_ns;  // bound on each pipeline wait
  int hold_loads;    // testing: the producer issues no loads
};

template <bool PG>
struct MxPG {
  CUtensorMap tm[kPG];   // FWD/DGRAD: B codes of group g
  CUtensorMap tms[kPG];  // FWD/DGRAD: B scale atoms of group g
  const __nv_bfloat16* bias[kPG];
  float* mg[kPG];        // WGRAD: main_grad of group g [N, K]
  __device__ const CUtensorMap* map(int g) const { return &tm[g]; }
  __device__ const CUtensorMap* smap(int g) const { return &tms[g]; }
  __device__ const __nv_bfloat16* b(int g) const { return bias[g]; }
  __device__ float* m(int g) const { return mg[g]; }
};
template <>
struct MxPG<false> {
  int unused;
  __device__ const CUtensorMap* map(int) const { return nullptr; }
  __device__ const CUtensorMap* smap(int) const { return nullptr; }
  __device__ const __nv_bfloat16* b(int) const { return nullptr; }
  __device__ float* m(int) const { return nullptr; }
};

struct Tile {
  int g, num_kb, mt, nt;
  int64_t r0;   // FWD/DGRAD: first A row of the tile (a multiple of 128); WGRAD: group start
  int64_t rlo;  // group start
  int64_t r1;   // group end
};

__device__ __forceinline__ int cdiv(int64_t a, int b) { return static_cast<int>((a + b - 1) / b); }

// First A row of a group's fprop / dgrad tiles: the group start rounded down
// to the 128-row scale atoms.
__device__ __forceinline__ int64_t atom_floor(int64_t r) { return r & ~int64_t(127); }

template <int MODE, int CG>
__device__ __forceinline__ int tiles_of_group(int64_t o0, int64_t o1, const MxParams& p) {
  constexpr int TMt = CfgMX<MODE, CG>::kTileM, TN = CfgMX<MODE, CG>::kTN;
  const int64_t m = o1 > o0 ? o1 - o0 : 0;
  if (MODE == kWgrad) return (m > 0 || !p.accumulate) ? cdiv(p.N, TMt) * cdiv(p.K, TN) : 0;
  if (m == 0) return 0;
  return cdiv(o1 - atom_floor(o0), TMt) * cdiv(MODE == kFwd ? p.N : p.K, TN);
}

template <int MODE, int CG>
__device__ __forceinline__ Tile decode(int t, const int* prefix, const MxParams& p) {
  constexpr int TMt = CfgMX<MODE, CG>::kTileM, TN = CfgMX<MODE, CG>::kTN;
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
  const int mtg = (MODE == kWgrad) ? cdiv(p.N, TMt) : cdiv(o0 + m - atom_floor(o0), TMt);
  const int ntg = cdiv(MODE == kFwd ? p.N : p.K, TN);
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
  tl.rlo = o0;
  tl.r1 = o0 + m;
  if (MODE == kWgrad) {
    tl.r0 = o0;
    tl.num_kb = cdiv(m, BK * CfgMX<MODE, CG>::kSub);
  } else {
    tl.r0 = atom_floor(o0) + static_cast<int64_t>(tl.mt) * TMt;
    tl.num_kb = cdiv(MODE == kFwd ? p.K : p.N, BK * CfgMX<MODE, CG>::kSub);
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

// Ragged wgrad contraction: zero the code rows [valid, to) of this CTA's stage
// (A: one 128-column chunk; B: kBChunks chunks; 128 bytes per contraction
// row) -- the rows of the last partial 32-row MMA step that belong to the
// next group.  Steps wholly past the group's end are skipped by the MMA.
template <int MODE, int CG>
__device__ __forceinline__ void zero_tail_rows(uint8_t* sa, uint8_t* sb, int valid, int to, int lane) {
  constexpr int kChunks = 1 + CfgMX<MODE, CG>::kBChunks;
  const int nrows = to - valid;
  if (nrows <= 0) return;
  const int per_chunk = nrows * 8;  // 16-byte pieces per chunk
  for (int idx = lane; idx < kChunks * per_chunk; idx += 32) {
    const int chunk = idx / per_chunk;
    const int rem = idx - chunk * per_chunk;
    const int r = valid + (rem >> 3);
    uint8_t* base = chunk == 0 ? sa : (sb + (chunk - 1) * 16384);
    *reinterpret_cast<uint4*>(base + r * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
}

// Contraction elements of stage kb that count (a multiple of 128 except on a
// ragged wgrad tail; 0 for a sub-stage wholly past the end).
template <int MODE, int CG>
__device__ __forceinline__ int stage_valid(const Tile& tl, int kb, const MxParams& p) {
  constexpr int kSpan = CfgMX<MODE, CG>::kSub * BK;
  const int64_t left = (MODE == kWgrad) ? (tl.r1 - tl.r0) - static_cast<int64_t>(kb) * kSpan
                                        : static_cast<int64_t>(MODE == kFwd ? p.K : p.N) - static_cast<int64_t>(kb) * kSpan;
  return left < kSpan ? static_cast<int>(left) : kSpan;
}

// Zero the ragged tail of each partly valid sub-stage of a wgrad stage.
template <int MODE, int CG>
__device__ __forceinline__ void zero_stage_tail(uint8_t* sa, uint8_t* sb, int valid, int lane) {
  using C = CfgMX<MODE, CG>;
#pragma unroll
  for (int u = 0; u < C::kSub; ++u) {
    const int vu = valid - u * BK;
    if (vu > 0 && vu < BK) zero_tail_rows<MODE, CG>(sa + u * C::kA1, sb + u * C::kB1, vu, ((vu + 31) >> 5) * 32, lane);
  }
}

template <int MODE, int CG, bool PG>
__global__ void __launch_bounds__(CfgMX<MODE, CG>::kThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ MxParams p, const __grid_constant__ MxPG<PG> pg) {
  using C = CfgMX<MODE, CG>;
  constexpr int TMt = C::kTileM, TN = C::kTN;
  constexpr int kSpan = C::kSub * BK;  // contraction elements per stage
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
  int* prefix = reinterpret_cast<int*>(smem + C::kPrefixOffset);  // tiles before group g
  int* qprefix = prefix + (p.G + 1);                             // WGRAD: scale k-groups before group g

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    *skip_flag = (p.status != nullptr && *reinterpret_cast<volatile int32_t*>(p.status) != 0) ? 1 : 0;
    *abort_flag = 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], (CG == 2 && leader) ? 2 : 1);  // leader: own TMA + peer's relay
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kEpiWarps * CG);
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
    // WGRAD: scale k-groups of the groups before this launch (per-group
    // main_grad launches cover 64 groups each)
    int qbase = 0;
    if (MODE == kWgrad) {
      for (int base = 0; base < p.g0; base += 32) {
        const int i = base + lane;
        int qc = 0;
        if (i < p.g0) {
          const int64_t m = __ldg(p.offsets_all + i + 1) - __ldg(p.offsets_all + i);
          qc = m > 0 ? cdiv(m, 128) : 0;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) qc += __shfl_xor_sync(0xffffffffu, qc, off);
        qbase += qc;
      }
    }
    int carry = 0, qcarry = qbase;
    for (int base = 0; base < p.G; base += 32) {
      const int i = base + lane;
      int cnt = 0, qc = 0;
      if (i < p.G) {
        const int64_t o0 = __ldg(p.offsets + i), o1 = __ldg(p.offsets + i + 1);
        cnt = tiles_of_group<MODE, CG>(o0, o1, p);
        qc = o1 > o0 ? cdiv(o1 - o0, 128) : 0;
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, cnt, off);
        const int u = __shfl_up_sync(0xffffffffu, qc, off);
        if (lane >= off) { cnt += v; qc += u; }
      }
      if (i < p.G) { prefix[i + 1] = carry + cnt; qprefix[i + 1] = qcarry + qc; }
      carry += __shfl_sync(0xffffffffu, cnt, 31);
      qcarry += __shfl_sync(0xffffffffu, qc, 31);
    }
    if (lane == 0) { prefix[0] = 0; qprefix[0] = qbase; }
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
      const uint64_t keep = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = pair; t < total && !*abort_flag; t += npairs) {
        const Tile tl = decode<MODE, CG>(t, prefix, p);
        const int n0 = tl.nt * TN;  // first B operand row of the tile
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.wait_ns)) { report_abort(abort_flag, p.status); break; }
          if (p.hold_loads) {  // testing the timeout path: this stage never lands
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            continue;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          uint8_t* sf = sb + C::kBAlloc;
          uint64_t* bar = &full[stage];
          mbar_arrive_expect_tx(bar, C::kTx);
          // every sub-stage is loaded; one past the contraction's end is
          // zero-filled (or holds the next group's rows) and its MMAs are skipped
#pragma unroll
          for (int u = 0; u < C::kSub; ++u) {
            const int kk = kb * C::kSub + u;  // 128-element step (scale k-group) within the contraction
            uint8_t* sau = sa + u * C::kA1;
            uint8_t* sbu = sb + u * C::kB1;
            uint8_t* sfu = sf + u * kSfBytes;
            if (MODE == kFwd || MODE == kDgrad) {
              const int32_t ra = static_cast<int32_t>(tl.r0 + hr);  // multiple of 128
              tma_load_2d(sau, &p.tmA, bar, kk * BK, ra);
              tma_load_3d(sfu, &p.tmSA, bar, 0, ra >> 7, kk);
            }
            if (MODE == kFwd) {
              if (PG) {
                tma_load_2d(sbu, pg.map(tl.g), bar, kk * BK, n0 + hb);
                tma_load_3d(sfu + kSfABytes, pg.smap(tl.g), bar, 0, n0 >> 7, kk);
              } else {
                tma_load_3d(sbu, &p.tmB, bar, kk * BK, n0 + hb, tl.g);
                tma_load_3d(sfu + kSfABytes, &p.tmSB, bar, 0, tl.g * (p.N >> 7) + (n0 >> 7), kk);
              }
            } else if (MODE == kDgrad) {
#pragma unroll
              for (int c = 0; c < C::kBChunks; ++c) {
                if (PG) tma_load_2d(sbu + c * 16384, pg.map(tl.g), bar, n0 + hb + c * 128, kk * BK);
                else    tma_load_3d(sbu + c * 16384, &p.tmB, bar, n0 + hb + c * 128, kk * BK, tl.g);
              }
              if (PG) tma_load_3d(sfu + kSfABytes, pg.smap(tl.g), bar, 0, n0 >> 7, kk);
              else    tma_load_3d(sfu + kSfABytes, &p.tmSB, bar, 0, n0 >> 7, tl.g * (p.N >> 7) + kk);
            } else {
              const int32_t row = static_cast<int32_t>(tl.r0 + kk * BK);
              const int kq = qprefix[tl.g] + kk;  // scale k-group of this sub-stage
              const int m0 = tl.mt * TMt + hr;
              // operand strips are read again by the band's neighbouring tiles:
              // keep them in L2 ahead of the streamed main_grad lines
              tma_load_2d_hint(sau, &p.tmA, bar, m0, row, keep);
#pragma unroll
              for (int c = 0; c < C::kBChunks; ++c)
                tma_load_2d_hint(sbu + c * 16384, &p.tmB, bar, n0 + hb + c * 128, row, keep);
              tma_load_3d(sfu, &p.tmSA, bar, 0, m0 >> 7, kq);
              tma_load_3d(sfu + kSfABytes, &p.tmSB, bar, 0, n0 >> 7, kq);
            }
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
      // ===================== scale copy + MMA issue =====================
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      uint32_t kiter = 0;
      for (int t = pair; t < total; t += npairs, ++it) {
        const Tile tl = decode<MODE, CG>(t, prefix, p);
        const int buf = it % C::kAccBufs;
        const uint32_t tph = (it / C::kAccBufs) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], tph ^ 1u, abort_flag, p.wait_ns))) {
          report_abort(abort_flag, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * TN;
        bool ok = true;
        for (int kb = 0; kb < tl.num_kb; ++kb, ++kiter) {
          // contraction elements of this stage that count: fewer on a ragged
          // wgrad tail, or past the end of an fprop / dgrad contraction of
          // 128 * odd elements (only the last stage of a tile can be short)
          const int valid = (kb == tl.num_kb - 1) ? stage_valid<MODE, CG>(tl, kb, p) : kSpan;
          // the peer zeroed rows of its stage before relaying: acquire at
          // cluster scope so those writes are visible to the pair's MMAs
          const bool peer_zeroed = CG == 2 && MODE == kWgrad && valid < kSpan;
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
          uint8_t* sf = sb + C::kBAlloc;
          if (MODE == kWgrad && valid < kSpan) zero_stage_tail<MODE, CG>(sa, sb, valid, lane);
          __syncwarp();
          if (lane == 0) {
            // The single issuing thread is on the critical path: descriptors
            // are formed once per stage and advanced by constants.
            const uint64_t ad0 = C::kAMN ? smem_desc_sw128(smem_u32(sa), 16384, 1024) : smem_desc_sw128(smem_u32(sa), 16, 1024);
            const uint64_t bd0 = C::kBMN ? smem_desc_sw128(smem_u32(sb), 16384, 1024) : smem_desc_sw128(smem_u32(sb), 16, 1024);
            const uint64_t sd0 = smem_desc_sf(smem_u32(sf));
            const uint32_t slot0 = tmem_base + C::kSfCol0 + ((kiter * C::kSub) & (kSfSlots - 1)) * kSfSlotCols;
            // sub-stage u: its scale atoms to a TMEM slot, then its MMAs
            // (K = 32 each, scale byte ks of the slot's columns)
            auto issue_sub = [&](int u, int ksteps) {
              const uint32_t sfa = slot0 + u * kSfSlotCols, sfb = sfa + 4;
              const uint64_t sd = desc_add(sd0, (u * kSfBytes) >> 4);
              if (CG == 2) {
                tmem_cp_32x128b_x4_pair(sfa, sd);
#pragma unroll
                for (int a = 0; a < kAtomsB; ++a) tmem_cp_32x128b_x4_pair(sfb + 4 * a, desc_add(sd, (kSfABytes + 512 * a) >> 4));
              } else {
                tmem_cp_32x128b_x4(sfa, sd);
#pragma unroll
                for (int a = 0; a < kAtomsB; ++a) tmem_cp_32x128b_x4(sfb + 4 * a, desc_add(sd, (kSfABytes + 512 * a) >> 4));
              }
              const uint64_t ad = desc_add(ad0, (u * C::kA1) >> 4);
              const uint64_t bd = desc_add(bd0, (u * C::kB1) >> 4);
#pragma unroll
              for (int ks = 0; ks < BK / 32; ++ks) {
                if (ks >= ksteps) break;
                const uint32_t idesc = idesc_mxf8(TMt, TN, C::kAMN, C::kBMN, ks, ks);
                const uint32_t acc = (kb > 0 || u > 0 || ks > 0) ? 1u : 0u;
                const uint64_t a_ks = desc_add(ad, (C::kAMN ? 256u : 2u) * ks), b_ks = desc_add(bd, (C::kBMN ? 256u : 2u) * ks);
                if (CG == 2) mma_mxf8_ss_pair(d_tmem, a_ks, b_ks, idesc, sfa, sfb, acc);
                else         mma_mxf8_ss(d_tmem, a_ks, b_ks, idesc, sfa, sfb, acc);
              }
            };
            if (valid == kSpan) {
#pragma unroll
              for (int u = 0; u < C::kSub; ++u) issue_sub(u, BK / 32);
            } else {
              for (int u = 0; u < C::kSub; ++u) {
                const int vu = valid - u * BK;
                if (vu <= 0) break;
                issue_sub(u, vu >= BK ? BK / 32 : (vu + 31) >> 5);
              }
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
          } else if (!p.hold_loads) {  // nothing accumulated: the epilogues write zeros
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
    } else {
      // ===================== peer: stage relay =====================
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < total; t += npairs) {
        const Tile tl = decode<MODE, CG>(t, prefix, p);
        bool ok = true;
        for (int kb = 0; kb < tl.num_kb; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag, p.wait_ns))) {
            report_abort(abort_flag, p.status);
            ok = false;
            break;
          }
          bool zeroed = false;
          if (MODE == kWgrad && kb == tl.num_kb - 1) {
            const int valid = stage_valid<MODE, CG>(tl, kb, p);
            if (valid < kSpan) {
              uint8_t* sa = smem + stage * C::kStageBytes;
              zero_stage_tail<MODE, CG>(sa, sa + C::kABytes, valid, lane);
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
    // ===================== epilogue (warps 2.., both CTAs) =====================
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;         // FWD/DGRAD: 128-column half of the tile
    const int row_in_tile = q * 32 + lane;
    const uint32_t tempty_leader = (CG == 2) ? mapa_shared(smem_u32(tempty), 0) : 0u;
    auto prefetch_mg = [&](const Tile& tn) {
      const int n = tn.mt * TMt + hr + q * 32 + lane;
      const int k0 = tn.nt * TN + h * (TN / 2);
      const int cols = min(TN / 2, p.K - k0);
      if (n < p.N && cols > 0) {
        const float* gb = PG ? pg.m(tn.g) : p.mg + static_cast<int64_t>(tn.g) * p.N * p.K;
        l2_prefetch_bulk(gb + static_cast<int64_t>(n) * p.K + k0, static_cast<uint32_t>(cols) * 4u);
      }
    };
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const Tile tl = decode<MODE, CG>(t, prefix, p);
      const int buf = it % C::kAccBufs;
      const uint32_t tph = (it / C::kAccBufs) & 1;
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
        // this warp: rows q*32.. of the CTA's 128, columns h*128 .. h*128+127;
        // copy them to registers, free the accumulator, then round and store
        const int Nout = (MODE == kFwd) ? p.N : p.K;
        const int64_t row = tl.r0 + hr + row_in_tile;
        const bool row_ok = row >= tl.rlo && row < tl.r1 && row < p.out_rows;
        const int ncol0 = tl.nt * TN + h * 128;
        const int nvalid = Nout - ncol0;  // columns of this warp inside the output (may be <= 0)
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c * 32 < nvalid) tmem_ld_32x32b_x32(tacc + h * 128 + c * 32, r[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_reg_fence(r[c]);
        release_acc();
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
        const __nv_bfloat16* bias = nullptr;
        if (MODE == kFwd && p.has_bias) bias = PG ? pg.b(tl.g) : (p.bias + static_cast<int64_t>(tl.g) * p.N);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c * 32 >= nvalid) break;
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            const int n = ncol0 + c * 32 + j8 * 8;  // 8 output columns (16 bytes)
            if (n >= Nout) break;
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = __uint_as_float(r[c][j8 * 8 + j]);
            if (bias != nullptr) {
              const uint4 bv = __ldg(reinterpret_cast<const uint4*>(bias + n));
              const __nv_bfloat16* bb = reinterpret_cast<const __nv_bfloat16*>(&bv);
#pragma unroll
              for (int j = 0; j < 8; ++j) f[j] += __bfloat162float(bb[j]);
            }
            if (row_ok) {
              uint4 w;
              w.x = pack_bf16x2(f[0], f[1]);
              w.y = pack_bf16x2(f[2], f[3]);
              w.z = pack_bf16x2(f[4], f[5]);
              w.w = pack_bf16x2(f[6], f[7]);
              *reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(Nout) + n) = w;
            }
          }
        }
      } else {
        // main_grad rows n0 + 0..31 (this warp's TMEM lanes) x columns k0 .. k0+127
        // (its half of the tile): copy them to registers and free the
        // accumulator, so the next tile's MMAs run while these sums leave.
        // Each [32 x 16] fp32 piece then goes through a 2 KB per-warp
        // shared-memory transpose (16-byte pieces, XOR-swizzled: conflict-free
        // both ways), so that 4 lanes cover 64 contiguous bytes of a row, and
        // leaves as coalesced 16-byte vector reductions (accumulate) or stores
        // (overwrite): full-sector transactions, many in flight, no waits.
        float* stg = reinterpret_cast<float*>(smem + C::kStagingOffset) + (warp - 2) * (32 * 16);
        constexpr int kCols = TN / 2;  // columns of this warp (its half)
        constexpr int kChunks = kCols / 32;
        const int n0 = tl.mt * TMt + hr + q * 32;
        const int k0 = tl.nt * TN + h * kCols;
        const bool in_k = k0 < p.K;  // K % 128 == 0: the half is all inside K or all past it
        uint32_t r[kChunks][32];
        if (tl.num_kb > 0 && in_k) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c) tmem_ld_32x32b_x32(tacc + h * kCols + c * 32, r[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < kChunks; ++c) tmem_reg_fence(r[c]);
        } else {
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j) r[c][j] = 0u;  // an empty group's overwrite: zeros
        }
        release_acc();
        if (in_k) {
          float* gbase = PG ? pg.m(tl.g) : p.mg + static_cast<int64_t>(tl.g) * p.N * p.K;
          const int sub = lane >> 2, piece = lane & 3;  // read side: row 8i + sub, 16-byte piece
          float* mine = stg + lane * 16;
          const int wsw = (lane >> 1) & 3;  // write-side swizzle of this lane's row
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {  // 16 of the chunk's 32 columns at a time
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(mine + ((j ^ wsw) << 2)) =
                    make_uint4(r[c][16 * hh + 4 * j], r[c][16 * hh + 4 * j + 1], r[c][16 * hh + 4 * j + 2],
                               r[c][16 * hh + 4 * j + 3]);
              __syncwarp();
              const int col = k0 + c * 32 + hh * 16 + piece * 4;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int row = 8 * i + sub;
                const uint4 v = *reinterpret_cast<const uint4*>(stg + row * 16 + ((piece ^ ((row >> 1) & 3)) << 2));
                if (n0 + row < p.N) {
                  float* dst = gbase + static_cast<int64_t>(n0 + row) * p.K + col;
                  if (p.accumulate) red_add_v4(dst, v.x, v.y, v.z, v.w);
                  else *reinterpret_cast<uint4*>(dst) = v;
                }
              }
              __syncwarp();  // the next piece overwrites the transpose buffer
            }
          }
        }
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

// Scale atoms as a u32 tensor {128 words, atoms, k-groups}: `atoms` 512-byte
// atoms per k-group, consecutive k-groups `kstride` atoms apart; the box is
// `box_atoms` consecutive atoms of one k-group.
bool map_atoms(CUtensorMap* m, const void* base, uint64_t atoms, uint64_t kgroups, uint64_t kstride,
               uint32_t box_atoms) {
  const uint64_t dims[3] = {128, atoms, kgroups};
  const uint64_t strides[2] = {512, kstride * 512};
  const uint32_t box[3] = {128, box_atoms, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int MODE, int CG>
constexpr int mx_smem_bytes(int G) {
  return CfgMX<MODE, CG>::kPrefixOffset + 2 * (G + 1) * 4 + 1024;
}

cudaLaunchConfig_t pair_cfg(int grid, int threads, int smem, cudaStream_t stream, cudaLaunchAttribute* attr) {
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

template <typename Kern>
int pair_grid(Kern kern, int threads, int smem) {
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
  cudaLaunchConfig_t cfg = pair_cfg(2 * (num_sms() / 2), threads, smem, nullptr, attr);
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
  constexpr int threads = CfgMX<MODE, CG>::kThreads;
  if (CG == 1) {
    kern<<<num_sms(), threads, smem, stream>>>(prm, pga);
  } else {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_cfg(pair_grid(kern, threads, smem), threads, smem, stream, attr);
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
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  MxParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.status = c.status;
  prm.out_rows = c.out_rows;
  prm.out = c.out;
  prm.N = c.N;
  prm.K = c.K;
  prm.accumulate = c.accumulate;
  prm.wait_ns = c.wait_ns ? c.wait_ns : kWaitLimitNs;
  prm.hold_loads = c.hold_loads;
  prm.has_bias = (MODE == kFwd && c.bias != nullptr) ? 1 : 0;
  prm.offsets_all = c.offsets;
  const uint64_t M = c.M > 0 ? static_cast<uint64_t>(c.M) : 1;
  const uint64_t RB = (M + 127) / 128;                  // row atoms of x / dy rowwise scales
  const uint64_t KQ = RB + static_cast<uint64_t>(c.G);  // bound on x_c / dy_c scale k-groups
  const uint64_t NA = c.N / 128, KA = c.K / 128;        // 128-row atoms along N and K
  const uint64_t G = static_cast<uint64_t>(c.G);
  const uint32_t BR = Cf::kBRows;
  bool ok = true;
  if (MODE == kFwd) {
    ok &= map2(&prm.tmA, c.a, c.K, M, c.K, 128, 128, U8, SW);
    ok &= map_atoms(&prm.tmSA, c.sa, RB, KA, RB, 1);
  } else if (MODE == kDgrad) {
    ok &= map2(&prm.tmA, c.a, c.N, M, c.N, 128, 128, U8, SW);
    ok &= map_atoms(&prm.tmSA, c.sa, RB, NA, RB, 1);
  } else {
    ok &= map2(&prm.tmA, c.a, c.N, M, c.N, 128, 128, U8, SW);
    ok &= map2(&prm.tmB, c.b, c.K, M, c.K, 128, 128, U8, SW);
    ok &= map_atoms(&prm.tmSA, c.sa, NA, KQ, NA, 1);
    ok &= map_atoms(&prm.tmSB, c.sb, KA, KQ, KA, kAtomsB);
  }
  if (!ok) return GL_ERR_UNSUPPORTED;

  const bool stacked = (MODE == kWgrad) ? c.out_grouped.mode == GL_STACKED
                                        : (c.w.mode == GL_STACKED && c.ws.mode == GL_STACKED);
  const bool bias_ok = !prm.has_bias || c.bias->mode == GL_STACKED;
  if (stacked && bias_ok) {
    if (MODE == kFwd) {
      ok &= map3(&prm.tmB, c.w.base, c.K, c.N, c.G, 1, 128, BR, U8);
      ok &= map_atoms(&prm.tmSB, c.ws.base, G * NA, KA, G * NA, kAtomsB);  // rows G*N, cols K
    } else if (MODE == kDgrad) {
      ok &= map3(&prm.tmB, c.w.base, c.K, c.N, c.G, 1, 128, 128, U8);
      ok &= map_atoms(&prm.tmSB, c.ws.base, KA, G * NA, KA, kAtomsB);  // G groups of N/128 k-groups
    } else {
      prm.mg = static_cast<float*>(const_cast<void*>(c.out_grouped.base));
    }
    if (!ok) return GL_ERR_UNSUPPORTED;
    if (prm.has_bias) prm.bias = reinterpret_cast<const __nv_bfloat16*>(c.bias->base);
    MxPG<false> none{0};
    // launches of at most kMaxG groups (wgrad: 256; the others take every group at once)
    constexpr int kMaxG = CfgMX<MODE, CG>::kMaxG;
    float* mg0 = prm.mg;
    gl_status st = GL_OK;
    for (int g0 = 0; g0 < c.G && st == GL_OK; g0 += kMaxG) {
      const int cg = std::min(kMaxG, c.G - g0);
      prm.offsets = c.offsets + g0;
      prm.G = cg;
      prm.g0 = g0;
      if (MODE == kWgrad) prm.mg = mg0 + static_cast<int64_t>(g0) * c.N * c.K;
      st = mx_launch<MODE, CG, false>(prm, none, cg, c.stream);
    }
    return st;
  }
  MxPG<true>* pga = new MxPG<true>;
  gl_status st = GL_OK;
  for (int g0 = 0; g0 < c.G && st == GL_OK; g0 += kPG) {
    const int cg = std::min(kPG, c.G - g0);
    memset(pga, 0, sizeof(*pga));
    for (int i = 0; i < cg; ++i) {
      const int g = g0 + i;
      if (MODE == kWgrad) {
        pga->mg[i] = static_cast<float*>(
            const_cast<void*>(group_ptr(c.out_grouped, g, static_cast<size_t>(c.N) * c.K * 4)));
        continue;
      }
      const void* wp = group_ptr(c.w, g, static_cast<size_t>(c.N) * c.K);
      if (MODE == kFwd) {
        ok &= map2(&pga->tm[i], wp, c.K, c.N, c.K, 128, BR, U8, SW);
        if (c.ws.mode == GL_STACKED) {
          // group g's N/128 atoms inside each k-group of the stacked [G*N, K] atoms
          const void* sp = static_cast<const uint8_t*>(c.ws.base) + static_cast<size_t>(g) * NA * 512;
          ok &= map_atoms(&pga->tms[i], sp, NA, KA, G * NA, kAtomsB);
        } else {
          ok &= map_atoms(&pga->tms[i], c.ws.ptrs[g], NA, KA, NA, kAtomsB);
        }
      } else {
        ok &= map2(&pga->tm[i], wp, c.K, c.N, c.K, 128, 128, U8, SW);
        const void* sp = group_ptr(c.ws, g, static_cast<size_t>(NA) * KA * 512);
        ok &= map_atoms(&pga->tms[i], sp, KA, NA, KA, kAtomsB);
      }
      if (prm.has_bias)
        pga->bias[i] = reinterpret_cast<const __nv_bfloat16*>(group_ptr(*c.bias, g, static_cast<size_t>(c.N) * 2));
    }
    if (!ok) { st = GL_ERR_UNSUPPORTED; break; }
    prm.offsets = c.offsets + g0;
    prm.G = cg;
    prm.g0 = g0;
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
