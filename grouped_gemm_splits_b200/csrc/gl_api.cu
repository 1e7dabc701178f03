// gl_api.cu -- the C ABI (include/gl.h): argument checks, then launches.
// Nothing here allocates device memory or synchronises the host.
#include "gl_internal.h"

namespace {

using gl::GemmCall;

// Per-call GEMM options (NULL = defaults: CTA pairs, the kernels' own 2 s
// wait bound).  False for values the header does not define.
bool read_opts(const gl_gemm_opts* o, int* cta_pair, uint64_t* wait_ns, int* hold_loads) {
  *cta_pair = 1;
  *wait_ns = 0;  // 0: the kernel's default bound
  *hold_loads = 0;
  if (o == nullptr) return true;
  if (o->tiles != GL_TILES_PAIR && o->tiles != GL_TILES_SINGLE) return false;
  if (o->wait_limit_us > GL_WAIT_LIMIT_MAX_US) return false;
  if (o->flags & ~GL_OPT_HOLD_LOADS) return false;
  *cta_pair = (o->tiles == GL_TILES_PAIR) ? 1 : 0;
  *wait_ns = static_cast<uint64_t>(o->wait_limit_us) * 1000u;
  *hold_loads = (o->flags & GL_OPT_HOLD_LOADS) ? 1 : 0;
  return true;
}

cudaStream_t to_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool grouped_ok(const gl_grouped& g, int G) {
  if (g.mode == GL_STACKED) return g.base != nullptr;
  if (g.mode == GL_PER_GROUP) {
    if (g.ptrs == nullptr) return false;
    for (int i = 0; i < G; ++i)
      if (g.ptrs[i] == nullptr) return false;
    return true;
  }
  return false;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool grouped_aligned(const gl_grouped& g, int G) {
  if (g.mode == GL_STACKED) return aligned16(g.base);
  for (int i = 0; i < G; ++i)
    if (!aligned16(g.ptrs[i])) return false;
  return true;
}

// Common shape checks for the three GEMMs (grouped_linear.py: in/out features
// and group count must be positive; TMA needs 16-byte row pitches).
gl_status check_gemm_dims(int G, int64_t M, int N, int K) {
  if (G <= 0 || G > GL_MAX_GROUPS || M < 0 || N <= 0 || K <= 0) return GL_ERR_INVALID;
  if ((N % 8) != 0 || (K % 8) != 0) return GL_ERR_UNSUPPORTED;
  if (M >= (int64_t(1) << 31)) return GL_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  // persistent-scheduler tile counts are int32
  const int64_t rt = (M + 127) / 128 + G;
  const int64_t ct = (int64_t(N > K ? N : K) + 127) / 128;
  if (rt * ct >= (int64_t(1) << 31) || int64_t(G) * ct * ct >= (int64_t(1) << 31)) return GL_ERR_UNSUPPORTED;
  return GL_OK;
}

}  // namespace

extern "C" {

int gl_version(void) { return 200; }

const char* gl_status_string(gl_status s) {
  switch (s) {
    case GL_OK: return "ok";
    case GL_ERR_INVALID: return "invalid argument";
    case GL_ERR_UNSUPPORTED: return "unsupported size or alignment";
    case GL_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

gl_status gl_offsets(const int64_t* m_splits, int G, int64_t expect_rows, int64_t out_rows,
                     int64_t* offsets, int32_t* status, void* stream) {
  if (m_splits == nullptr || offsets == nullptr || status == nullptr) return GL_ERR_INVALID;
  if (G <= 0 || G > GL_MAX_GROUPS || expect_rows < 0 || out_rows < 0) return GL_ERR_INVALID;
  return gl::launch_offsets(m_splits, G, expect_rows, out_rows, offsets, status, to_stream(stream));
}

gl_status gl_fwd(const void* x, gl_grouped w, const gl_grouped* bias, const int64_t* offsets,
                 int32_t* status, int G, int64_t M, int N, int K, void* y, int64_t y_rows,
                 const gl_gemm_opts* opts, void* stream) {
  gl_status st = check_gemm_dims(G, M, N, K);
  if (st != GL_OK) return st;
  int pair = 1, hold = 0;
  uint64_t wait_ns = 0;
  if (!read_opts(opts, &pair, &wait_ns, &hold)) return GL_ERR_INVALID;
  if ((x == nullptr && M > 0) || (y == nullptr && M > 0) || offsets == nullptr || status == nullptr)
    return GL_ERR_INVALID;
  if (!grouped_ok(w, G) || (bias != nullptr && !grouped_ok(*bias, G))) return GL_ERR_INVALID;
  if (y_rows < M) return GL_ERR_INVALID;
  if (!aligned16(x) || !aligned16(y) || !grouped_aligned(w, G) || (bias && !grouped_aligned(*bias, G)))
    return GL_ERR_UNSUPPORTED;
  if (M == 0) return GL_OK;  // no rows: nothing to write
  GemmCall c{};
  c.mode = gl::kFwd;
  c.a = x;
  c.w = w;
  c.bias = bias;
  c.out = y;
  c.out_rows = y_rows;
  c.offsets = offsets;
  c.status = status;
  c.G = G;
  c.M = M;
  c.N = N;
  c.K = K;
  c.cta_pair = pair;
  c.wait_ns = wait_ns;
  c.hold_loads = hold;
  c.stream = to_stream(stream);
  return gl::launch_grouped_gemm(c);
}

gl_status gl_dgrad(const void* dy, gl_grouped w, const int64_t* offsets, int32_t* status, int G,
                   int64_t M, int N, int K, void* dx, int64_t dx_rows, const gl_gemm_opts* opts, void* stream) {
  gl_status st = check_gemm_dims(G, M, N, K);
  if (st != GL_OK) return st;
  int pair = 1, hold = 0;
  uint64_t wait_ns = 0;
  if (!read_opts(opts, &pair, &wait_ns, &hold)) return GL_ERR_INVALID;
  if ((dy == nullptr && M > 0) || (dx == nullptr && M > 0) || offsets == nullptr || status == nullptr)
    return GL_ERR_INVALID;
  if (!grouped_ok(w, G)) return GL_ERR_INVALID;
  if (dx_rows < M) return GL_ERR_INVALID;
  if (!aligned16(dy) || !aligned16(dx) || !grouped_aligned(w, G)) return GL_ERR_UNSUPPORTED;
  if (M == 0) return GL_OK;
  GemmCall c{};
  c.mode = gl::kDgrad;
  c.a = dy;
  c.w = w;
  c.out = dx;
  c.out_rows = dx_rows;
  c.offsets = offsets;
  c.status = status;
  c.G = G;
  c.M = M;
  c.N = N;
  c.K = K;
  c.cta_pair = pair;
  c.wait_ns = wait_ns;
  c.hold_loads = hold;
  c.stream = to_stream(stream);
  return gl::launch_grouped_gemm(c);
}

gl_status gl_wgrad(const void* x, const void* dy, const int64_t* offsets, int32_t* status, int G,
                   int64_t M, int N, int K, gl_grouped main_grad, int accumulate, const gl_gemm_opts* opts, void* stream) {
  gl_status st = check_gemm_dims(G, M, N, K);
  if (st != GL_OK) return st;
  int pair = 1, hold = 0;
  uint64_t wait_ns = 0;
  if (!read_opts(opts, &pair, &wait_ns, &hold)) return GL_ERR_INVALID;
  if ((x == nullptr && M > 0) || (dy == nullptr && M > 0) || offsets == nullptr || status == nullptr)
    return GL_ERR_INVALID;
  if (!grouped_ok(main_grad, G)) return GL_ERR_INVALID;
  if (!aligned16(x) || !aligned16(dy) || !grouped_aligned(main_grad, G)) return GL_ERR_UNSUPPORTED;
  if (M == 0) {
    if (accumulate) return GL_OK;  // every group is empty: main_grad unchanged
    // overwrite: the kernel writes zeros and never reads x / dy; give the
    // operand maps any valid base
    const void* any = main_grad.mode == GL_STACKED ? main_grad.base : main_grad.ptrs[0];
    x = any;
    dy = any;
  }
  GemmCall c{};
  c.mode = gl::kWgrad;
  c.a = dy;
  c.b = x;
  c.out_grouped = main_grad;
  c.offsets = offsets;
  c.status = status;
  c.G = G;
  c.M = M;
  c.N = N;
  c.K = K;
  c.accumulate = accumulate ? 1 : 0;
  c.cta_pair = pair;
  c.wait_ns = wait_ns;
  c.hold_loads = hold;
  c.stream = to_stream(stream);
  return gl::launch_grouped_gemm(c);
}

// ---------------------------------------------------------------- MXFP8 GEMMs
static gl_status check_mx_dims(int G, int64_t M, int N, int K) {
  if (G <= 0 || G > GL_MAX_GROUPS_MXFP8 || M < 0 || N <= 0 || K <= 0) return GL_ERR_INVALID;
  if (N % 128 != 0 || K % 128 != 0) return GL_ERR_UNSUPPORTED;
  if (M >= (int64_t(1) << 31)) return GL_ERR_UNSUPPORTED;
  const int64_t rt = (M + 127) / 128 + G;
  const int64_t ct = (int64_t(N > K ? N : K) + 127) / 128;
  if (rt * ct >= (int64_t(1) << 31) || int64_t(G) * ct * ct >= (int64_t(1) << 31)) return GL_ERR_UNSUPPORTED;
  return GL_OK;
}

gl_status gl_fwd_mxfp8(const uint8_t* x_codes, const uint8_t* x_scales, gl_grouped w_codes,
                       gl_grouped w_scales, const gl_grouped* bias, const int64_t* offsets,
                       int32_t* status, int G, int64_t M, int N, int K, void* y, int64_t y_rows,
                       const gl_gemm_opts* opts, void* stream) {
  gl_status st = check_mx_dims(G, M, N, K);
  if (st != GL_OK) return st;
  int pair = 1, hold = 0;
  uint64_t wait_ns = 0;
  if (!read_opts(opts, &pair, &wait_ns, &hold)) return GL_ERR_INVALID;
  if (((x_codes == nullptr || x_scales == nullptr || y == nullptr) && M > 0) || offsets == nullptr ||
      status == nullptr)
    return GL_ERR_INVALID;
  if (!grouped_ok(w_codes, G) || !grouped_ok(w_scales, G) || (bias && !grouped_ok(*bias, G)))
    return GL_ERR_INVALID;
  if (y_rows < M) return GL_ERR_INVALID;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(y) || !grouped_aligned(w_codes, G) ||
      !grouped_aligned(w_scales, G) || (bias && !grouped_aligned(*bias, G)))
    return GL_ERR_UNSUPPORTED;
  if (M == 0) return GL_OK;
  gl::MxCall c{};
  c.mode = gl::kFwd;
  c.a = x_codes;
  c.sa = x_scales;
  c.w = w_codes;
  c.ws = w_scales;
  c.bias = bias;
  c.out = y;
  c.out_rows = y_rows;
  c.offsets = offsets;
  c.status = status;
  c.G = G;
  c.M = M;
  c.N = N;
  c.K = K;
  c.cta_pair = pair;
  c.wait_ns = wait_ns;
  c.hold_loads = hold;
  c.stream = to_stream(stream);
  return gl::launch_grouped_gemm_mx(c);
}

gl_status gl_dgrad_mxfp8(const uint8_t* dy_codes, const uint8_t* dy_scales, gl_grouped w_codes_c,
                         gl_grouped w_scales_c, const int64_t* offsets, int32_t* status, int G,
                         int64_t M, int N, int K, void* dx, int64_t dx_rows, const gl_gemm_opts* opts, void* stream) {
  gl_status st = check_mx_dims(G, M, N, K);
  if (st != GL_OK) return st;
  int pair = 1, hold = 0;
  uint64_t wait_ns = 0;
  if (!read_opts(opts, &pair, &wait_ns, &hold)) return GL_ERR_INVALID;
  if (((dy_codes == nullptr || dy_scales == nullptr || dx == nullptr) && M > 0) || offsets == nullptr ||
      status == nullptr)
    return GL_ERR_INVALID;
  if (!grouped_ok(w_codes_c, G) || !grouped_ok(w_scales_c, G)) return GL_ERR_INVALID;
  if (dx_rows < M) return GL_ERR_INVALID;
  if (!aligned16(dy_codes) || !aligned16(dy_scales) || !aligned16(dx) || !grouped_aligned(w_codes_c, G) ||
      !grouped_aligned(w_scales_c, G))
    return GL_ERR_UNSUPPORTED;
  if (M == 0) return GL_OK;
  gl::MxCall c{};
  c.mode = gl::kDgrad;
  c.a = dy_codes;
  c.sa = dy_scales;
  c.w = w_codes_c;
  c.ws = w_scales_c;
  c.out = dx;
  c.out_rows = dx_rows;
  c.offsets = offsets;
  c.status = status;
  c.G = G;
  c.M = M;
  c.N = N;
  c.K = K;
  c.cta_pair = pair;
  c.wait_ns = wait_ns;
  c.hold_loads = hold;
  c.stream = to_stream(stream);
  return gl::launch_grouped_gemm_mx(c);
}

gl_status gl_wgrad_mxfp8(const uint8_t* x_codes_c, const uint8_t* x_scales_c, const uint8_t* dy_codes_c,
                         const uint8_t* dy_scales_c, const int64_t* offsets, int32_t* status, int G,
                         int64_t M, int N, int K, gl_grouped main_grad, int accumulate, const gl_gemm_opts* opts, void* stream) {
  gl_status st = check_mx_dims(G, M, N, K);
  if (st != GL_OK) return st;
  int pair = 1, hold = 0;
  uint64_t wait_ns = 0;
  if (!read_opts(opts, &pair, &wait_ns, &hold)) return GL_ERR_INVALID;
  if (((x_codes_c == nullptr || x_scales_c == nullptr || dy_codes_c == nullptr || dy_scales_c == nullptr) &&
       M > 0) ||
      offsets == nullptr || status == nullptr)
    return GL_ERR_INVALID;
  if (!grouped_ok(main_grad, G)) return GL_ERR_INVALID;
  if (!aligned16(x_codes_c) || !aligned16(x_scales_c) || !aligned16(dy_codes_c) || !aligned16(dy_scales_c) ||
      !grouped_aligned(main_grad, G))
    return GL_ERR_UNSUPPORTED;
  if (M == 0) {
    if (accumulate) return GL_OK;
    const void* any = main_grad.mode == GL_STACKED ? main_grad.base : main_grad.ptrs[0];
    x_codes_c = x_scales_c = dy_codes_c = dy_scales_c = static_cast<const uint8_t*>(any);
  }
  gl::MxCall c{};
  c.mode = gl::kWgrad;
  c.a = dy_codes_c;
  c.sa = dy_scales_c;
  c.b = x_codes_c;
  c.sb = x_scales_c;
  c.out_grouped = main_grad;
  c.offsets = offsets;
  c.status = status;
  c.G = G;
  c.M = M;
  c.N = N;
  c.K = K;
  c.accumulate = accumulate ? 1 : 0;
  c.cta_pair = pair;
  c.wait_ns = wait_ns;
  c.hold_loads = hold;
  c.stream = to_stream(stream);
  return gl::launch_grouped_gemm_mx(c);
}

gl_status gl_dbias(const void* dy, const int64_t* offsets, int32_t* status, int G, int64_t M, int N,
                   gl_grouped dbias, void* stream) {
  if (G <= 0 || G > GL_MAX_GROUPS || M < 0 || N <= 0) return GL_ERR_INVALID;
  if ((dy == nullptr && M > 0) || offsets == nullptr || status == nullptr) return GL_ERR_INVALID;
  if (!grouped_ok(dbias, G)) return GL_ERR_INVALID;
  if (N % 8 != 0) return GL_ERR_UNSUPPORTED;
  if (M > 0 && !aligned16(dy)) return GL_ERR_UNSUPPORTED;
  if (M == 0) dy = offsets;  // never read: every group is empty
  return gl::launch_dbias(dy, offsets, status, G, N, dbias, to_stream(stream));
}

}  // extern "C"

namespace {

// Argument checks shared by the two cast entry points (GL_OK when valid).
gl_status check_quantize_args(const void* src, int64_t rows, int cols, const int64_t* row_offsets, int G,
                              const uint8_t* codes_r, const uint8_t* scales_r, const uint8_t* codes_c,
                              const uint8_t* scales_c, int scale_layout) {
  if (src == nullptr || rows < 0 || cols <= 0 || G <= 0 || G > GL_MAX_GROUPS) return GL_ERR_INVALID;
  if (codes_r == nullptr && codes_c == nullptr) return GL_ERR_INVALID;
  if (codes_r != nullptr && scales_r == nullptr) return GL_ERR_INVALID;
  if (codes_c != nullptr && scales_c == nullptr) return GL_ERR_INVALID;
  if (cols % 32 != 0) return GL_ERR_UNSUPPORTED;
  if (scale_layout != GL_SCALES_ROWMAJOR && scale_layout != GL_SCALES_MMA) return GL_ERR_INVALID;
  if (scale_layout == GL_SCALES_MMA && cols % 128 != 0) return GL_ERR_UNSUPPORTED;
  if (rows >= (int64_t(1) << 31)) return GL_ERR_UNSUPPORTED;
  if (row_offsets == nullptr && rows % G != 0) return GL_ERR_INVALID;
  if (!aligned16(src) || (codes_r && (reinterpret_cast<uintptr_t>(codes_r) & 7u)) ||
      (codes_c && (reinterpret_cast<uintptr_t>(codes_c) & 7u)))
    return GL_ERR_UNSUPPORTED;
  return GL_OK;
}

}  // namespace

namespace gl {

gl_status check_quantize_dbias_args(const void* src, int64_t rows, int cols, const int64_t* row_offsets, int G,
                                    const int32_t* status, const uint8_t* codes_r, const uint8_t* scales_r,
                                    const uint8_t* codes_c, const uint8_t* scales_c, int scale_layout,
                                    const gl_grouped& dbias) {
  const gl_status st =
      check_quantize_args(src, rows, cols, row_offsets, G, codes_r, scales_r, codes_c, scales_c, scale_layout);
  if (st != GL_OK) return st;
  if (row_offsets == nullptr || status == nullptr) return GL_ERR_INVALID;
  if (!grouped_ok(dbias, G)) return GL_ERR_INVALID;
  return GL_OK;
}

}  // namespace gl

namespace {

// Workspace of the fused cast + bias gradient: the groups' first blocks
// (int64[G+1], padded to 256 bytes), then the per-block column sums.
size_t dbias_ws_head(int G) { return ((static_cast<size_t>(G) + 1) * 8 + 255) / 256 * 256; }
int64_t dbias_ws_blocks(int64_t rows, int G) { return (rows + 31) / 32 + G; }

}  // namespace

extern "C" {

gl_status group_quantize_mxfp8(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                               int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                               uint8_t* codes_c, uint8_t* scales_c, int scale_layout, void* stream) {
  const gl_status st =
      check_quantize_args(src, rows, cols, row_offsets, G, codes_r, scales_r, codes_c, scales_c, scale_layout);
  if (st != GL_OK) return st;
  if (rows == 0) return GL_OK;
  return gl::launch_quantize(src, rows, cols, row_offsets, G, status, codes_r, scales_r, codes_c, scales_c,
                             scale_layout, nullptr, 0, nullptr, to_stream(stream));
}

size_t gl_dbias_workspace_bytes(int64_t rows, int cols, int G) {
  if (rows < 0 || cols <= 0 || G <= 0) return 0;
  return dbias_ws_head(G) + static_cast<size_t>(dbias_ws_blocks(rows, G)) * static_cast<size_t>(cols) * 4;
}

gl_status group_quantize_mxfp8_dbias(const void* src, int64_t rows, int cols, const int64_t* row_offsets,
                                     int G, int32_t* status, uint8_t* codes_r, uint8_t* scales_r,
                                     uint8_t* codes_c, uint8_t* scales_c, int scale_layout, gl_grouped dbias,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  const gl_status st = gl::check_quantize_dbias_args(src, rows, cols, row_offsets, G, status, codes_r, scales_r,
                                                     codes_c, scales_c, scale_layout, dbias);
  if (st != GL_OK) return st;
  if (workspace == nullptr) return GL_ERR_INVALID;
  if (workspace_bytes < gl_dbias_workspace_bytes(rows, cols, G)) return GL_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GL_ERR_UNSUPPORTED;
  cudaStream_t s = to_stream(stream);
  if (rows == 0)  // every group is empty: zeros (the source is never read)
    return gl::launch_dbias(row_offsets, row_offsets, status, G, cols, dbias, s);
  int64_t* prefix = static_cast<int64_t*>(workspace);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + dbias_ws_head(G));
  const gl_status q = gl::launch_quantize(src, rows, cols, row_offsets, G, status, codes_r, scales_r, codes_c,
                                          scales_c, scale_layout, part, dbias_ws_blocks(rows, G), prefix, s);
  if (q != GL_OK) return q;
  return gl::launch_dbias_partials(part, prefix, status, G, cols, dbias, s);
}

size_t gl_mxfp8_scale_bytes(int64_t rows, int cols, int G, int colwise, int scale_layout) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || G <= 0) return 0;
  const size_t r = static_cast<size_t>(rows), c = static_cast<size_t>(cols), g = static_cast<size_t>(G);
  if (scale_layout == GL_SCALES_ROWMAJOR) return colwise ? ((r + 31) / 32 + g) * c : r * (c / 32);
  if (scale_layout != GL_SCALES_MMA || cols % 128 != 0) return 0;
  return (colwise ? (r + 127) / 128 + g : (r + 127) / 128) * (c / 128) * 512;
}

}  // extern "C"
