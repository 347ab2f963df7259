// C ABI entry points that are not tied to one kernel family: status strings, size queries,
// GEMM argument checking and dispatch, device error word.
#include <string.h>

#include "sp24_internal.cuh"

#include <atomic>

namespace sp24 {

static std::atomic<int64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {

bool is16(int f) { return f == SP24_F16 || f == SP24_BF16; }

// Common checks of the x operand; fills the x part of p.
int prep_x(const sp24_operand* x, int64_t M, int64_t K, SkinnyParams* p) {
  if (!x) return SP24_ERR_INVALID_ARG;
  if (x->format == SP24_NVFP4) {
    if (K % 32) return SP24_ERR_SHAPE;
    if (M > 0 && K > 0 && (!x->data || !x->scales || !x->tensor_scale)) return SP24_ERR_INVALID_ARG;
    p->x_fmt = X_Q4;
  } else if (is16(x->format)) {
    if (K % 8) return SP24_ERR_SHAPE;
    if (M > 0 && K > 0 && !x->data) return SP24_ERR_INVALID_ARG;
    if (!aligned(x->data, 16)) return SP24_ERR_ALIGN;
    p->x_fmt = X_16;
  } else {
    return SP24_ERR_DTYPE;
  }
  p->x = x->data;
  p->x_scales = x->scales;
  p->x_ts = x->tensor_scale;
  return SP24_OK;
}

// MMA type: 16-bit x decides; 16-bit w must agree; NVFP4 x with NVFP4 w -> bf16.
int mma_type(int xf, int wf, int* t16) {
  if (is16(xf) && is16(wf) && xf != wf) return SP24_ERR_DTYPE;
  *t16 = is16(xf) ? xf : (is16(wf) ? wf : SP24_BF16);
  return SP24_OK;
}

// Runs the skinny kernel over M in slabs of 64 rows (one launch per slab).
int run_skinny(int wf, int t16, SkinnyParams p, cudaStream_t s) {
  const int64_t M = p.M;
  for (int64_t m0 = 0; m0 < M; m0 += 64) {
    SkinnyParams q = p;
    q.M = M - m0 < 64 ? M - m0 : 64;
    q.y = p.y + m0 * p.N;
    if (p.x_fmt == X_16) {
      q.x = reinterpret_cast<const uint8_t*>(p.x) + m0 * p.K * 2;
    } else {
      q.x = reinterpret_cast<const uint8_t*>(p.x) + m0 * p.K / 2;
      q.x_scales = p.x_scales + m0 * p.K / 16;
    }
    // the decode kernel declines (SP24_ERR_UNSUPPORTED, nothing launched) when the driver
    // refuses its x tensor map
    int st = decode_tile_supported(wf, q) ? decode_tile(wf, t16, q, s)
             : decode_supported(wf, q)    ? decode_gemv(wf, t16, q, s)
                                          : SP24_ERR_UNSUPPORTED;
    if (st == SP24_ERR_UNSUPPORTED)
      st = skinny2_supported(wf, q) ? skinny2_gemm(wf, t16, q, s) : skinny_gemm(wf, t16, q, s);
    if (st) return st;
  }
  return SP24_OK;
}

int64_t round256(int64_t b) { return (b + 255) / 256 * 256; }

// True when a 2:4 weight takes the native sparse tensor-core kernel (16-byte nibble rows).
bool native_sparse(int wf, int64_t K) { return (wf == W_S16 || wf == W_SQ4) && K % 128 == 0; }

// True when NVFP4 x times NVFP4 w takes the native block-scaled FP4 kernel (256-wide K stages,
// 16-byte aligned scale rows).
bool native_nvfp4(int x_fmt, int wf, const SkinnyParams& p) {
  return x_fmt == X_Q4 && wf == W_DQ4 && p.K % 256 == 0 && aligned(p.x, 16) && aligned(p.w, 16) &&
         aligned(p.x_scales, 16) && aligned(p.w_scales, 16);
}

// Workspace of the W4A4 pair kernel: the tile images (codes and scales) of each operand given
// in row order (x_mma / w_mma: that operand already is an image).
int64_t w4a4_image_bytes(int64_t rows, int64_t K) {
  return round256(nvfp4_mma_codes_bytes(rows, K)) + round256(nvfp4_mma_scales_bytes(rows, K));
}
int64_t w4a4_workspace(bool x_mma, bool w_mma, int64_t M, int64_t N, int64_t K) {
  return (x_mma ? 0 : w4a4_image_bytes(M, K)) + (w_mma ? 0 : w4a4_image_bytes(N, K));
}

// Workspace of the tiled path: 16-bit copies of the operands that are not 16-bit already
// (NVFP4 2:4 values decoded to 16 bits for the native sparse kernel; otherwise the weight
// expanded to a dense 16-bit matrix); for W4A4, the relaid block scales.
int64_t tiled_workspace(int x_fmt, int wf, int64_t M, int64_t N, int64_t K) {
  if (x_fmt == X_Q4 && wf == W_DQ4 && K % 256 == 0) return w4a4_workspace(false, false, M, N, K);
  int64_t b = 0;
  if (native_sparse(wf, K)) {
    if (wf == W_SQ4) b += round256(N * K);  // N x K/2 values of 2 bytes
    b += round256(meta_image_bytes(N, K));  // the metadata in the tcgen05 layout
  } else if (wf != W_D16) {
    b += round256(N * K * 2);
  }
  if (x_fmt == X_Q4) b += round256(M * K * 2);
  return b;
}

// W4A4 on the CTA-pair kernel: an operand given in row order (x_mma / w_mma false) is first
// rewritten as its tile images in the workspace.
int run_w4a4_pair(const uint8_t* xc, const uint8_t* xs, bool x_mma, const float* x_ts, const uint8_t* wc,
                  const uint8_t* wsc, bool w_mma, const float* w_ts, int64_t M, int64_t N, int64_t K, float* y,
                  void* ws, int64_t ws_bytes, cudaStream_t s) {
  const int64_t need = w4a4_workspace(x_mma, w_mma, M, N, K);
  if (need > 0 && (!ws || ws_bytes < need)) return SP24_ERR_WORKSPACE;
  if (need > 0 && !aligned(ws, 256)) return SP24_ERR_ALIGN;
  // one launch rewrites whichever operands are in row order
  uint8_t* cur = reinterpret_cast<uint8_t*>(ws);
  const uint8_t *c[2] = {nullptr, nullptr}, *sc[2] = {nullptr, nullptr};
  uint8_t *co[2] = {nullptr, nullptr}, *so[2] = {nullptr, nullptr};
  int64_t rows[2] = {0, 0};
  int n = 0;
  auto add = [&](const uint8_t** codes, const uint8_t** scales, int64_t r) {
    c[n] = *codes;
    sc[n] = *scales;
    rows[n] = r;
    co[n] = cur;
    so[n] = cur + round256(nvfp4_mma_codes_bytes(r, K));
    cur += w4a4_image_bytes(r, K);
    *codes = co[n];
    *scales = so[n];
    ++n;
  };
  if (!x_mma) add(&xc, &xs, M);
  if (!w_mma) add(&wc, &wsc, N);
  if (n > 0) {
    int st = nvfp4_to_mma2(c[0], sc[0], rows[0], co[0], so[0], c[1], sc[1], rows[1], co[1], so[1], K, s);
    if (st) return st;
  }
  return tc_gemm_nvfp4_pair(xc, xs, x_ts, wc, wsc, w_ts, M, N, K, y, s, 0);
}

// Tiled (tcgen05) path: decode what is not plain 16-bit into the workspace, then one GEMM.
int run_tiled(int wf, int t16, const SkinnyParams& p, void* ws, int64_t ws_bytes, cudaStream_t s) {
  // NVFP4 x with NVFP4 w: both stay 4-bit, the tensor core applies the block scales
  if (native_nvfp4(p.x_fmt, wf, p))
    return run_w4a4_pair(reinterpret_cast<const uint8_t*>(p.x), p.x_scales, false, p.x_ts, p.w, p.w_scales, false,
                         p.w_ts, p.M, p.N, p.K, p.y, ws, ws_bytes, s);
  const int64_t need = tiled_workspace(p.x_fmt, wf, p.M, p.N, p.K);
  if (need > 0 && (!ws || ws_bytes < need)) return SP24_ERR_WORKSPACE;
  if (need > 0 && !aligned(ws, 256)) return SP24_ERR_ALIGN;
  const bool bf = t16 == SP24_BF16;
  const bool sp_native = native_sparse(wf, p.K);
  uint8_t* cur = reinterpret_cast<uint8_t*>(ws);
  const void* w16 = p.w;
  if (sp_native && wf == W_SQ4) {
    // kept values only: [N, K/2] NVFP4 -> 16-bit E2M1 * E4M3
    int st = expand_w16(W_DQ4, bf, p.w, p.w_scales, nullptr, p.N, p.K / 2, reinterpret_cast<uint16_t*>(cur), s);
    if (st) return st;
    w16 = cur;
    cur += round256(p.N * p.K);
  } else if (!sp_native && wf != W_D16) {
    int st = expand_w16(wf, bf, p.w, p.w_scales, p.meta, p.N, p.K, reinterpret_cast<uint16_t*>(cur), s);
    if (st) return st;
    w16 = cur;
    cur += round256(p.N * p.K * 2);
  }
  const void* x16 = p.x;
  if (p.x_fmt == X_Q4) {
    int st = expand_w16(W_DQ4, bf, reinterpret_cast<const uint8_t*>(p.x), p.x_scales, nullptr, p.M, p.K,
                        reinterpret_cast<uint16_t*>(cur), s);
    if (st) return st;
    x16 = cur;
    cur += round256(p.M * p.K * 2);
  }
  const float* sa = (wf == W_DQ4 || wf == W_SQ4) ? p.w_ts : nullptr;
  const float* sb = p.x_fmt == X_Q4 ? p.x_ts : nullptr;
  if (sp_native) {
    // the nibble stream rewritten as tcgen05 metadata tiles, then the CTA-pair 2:4 kernel
    int st = meta_to_image(p.meta, p.N, p.K, cur, s);
    if (st) return st;
    return tc_gemm_f16_pair(x16, w16, cur, p.M, p.N, p.K, bf, p.y, sa, sb, s, 0);
  }
  if (p.K % 64 == 0) return tc_gemm_f16_pair(x16, w16, nullptr, p.M, p.N, p.K, bf, p.y, sa, sb, s, 0);
  return tc_gemm_f16(x16, w16, p.M, p.N, p.K, bf, p.y, sa, sb, s);
}

// ALGO_AUTO: the skinny kernels (FP4 decoded in registers, one launch per 64 rows of x) up to
// M = 64, and up to M = 128 for dense NVFP4 weights with 16-bit x, where the tiled path first
// expands the whole weight to 16 bits in HBM (measured at N = K = 5120: 47 / 52 / 67 us against
// 70 / 71 / 71 us at M = 80 / 96 / 128; at M = 192 tiled wins).  2:4 NVFP4 weights go tiled
// above 64 rows: the skinny 2:4 kernel took 72-120 us there against 50 us tiled.
bool auto_skinny(int x_fmt, int wf, int64_t M) {
  return M <= 64 || (M <= 128 && x_fmt == X_16 && wf == W_DQ4);
}

int dispatch(int wf, int t16, const SkinnyParams& p, int algo, void* ws, int64_t ws_bytes, cudaStream_t s) {
  if (algo == SP24_ALGO_SKINNY || (algo == SP24_ALGO_AUTO && auto_skinny(p.x_fmt, wf, p.M)))
    return run_skinny(wf, t16, p, s);
  return run_tiled(wf, t16, p, ws, ws_bytes, s);
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" const char* sp24_status_string(int status) {
  switch (status) {
    case SP24_OK: return "ok";
    case SP24_ERR_INVALID_ARG: return "invalid argument";
    case SP24_ERR_SHAPE: return "shape violates the operation's rule";
    case SP24_ERR_DTYPE: return "element type not accepted";
    case SP24_ERR_ALIGN: return "pointer misaligned";
    case SP24_ERR_UNSUPPORTED: return "unsupported combination";
    case SP24_ERR_CUDA: return "CUDA runtime error";
    case SP24_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case SP24_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

extern "C" int sp24_abi_version(void) { return 1; }

extern "C" int sp24_sizes(int op, int dtype, const int64_t* shape, int ndim, int64_t* groups,
                          int64_t* values_bytes, int64_t* meta_bytes, int64_t* nvfp4_codes_bytes,
                          int64_t* nvfp4_scales_bytes) {
  int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  if (!shape || ndim < 1 || ndim > 4) return SP24_ERR_INVALID_ARG;
  int64_t n = 1;
  for (int d = 0; d < ndim; ++d) {
    if (shape[d] < 0) return SP24_ERR_SHAPE;
    n *= shape[d];
  }
  int64_t G;
  if (op == SP24_OP_MATMUL) {
    if (shape[ndim - 1] % 4) return SP24_ERR_SHAPE;
    G = n / 4;
  } else if (op == SP24_OP_CONV) {
    if (ndim != 4 || shape[1] % 4) return SP24_ERR_SHAPE;
    G = shape[0] * (shape[1] / 4) * shape[2] * shape[3];
  } else {
    return SP24_ERR_INVALID_ARG;
  }
  if (groups) *groups = G;
  if (values_bytes) *values_bytes = 2 * G * eb;
  if (meta_bytes) *meta_bytes = (G + 1) / 2;
  int64_t L = shape[ndim - 1];
  bool q = op == SP24_OP_MATMUL && L % 16 == 0;
  if (nvfp4_codes_bytes) *nvfp4_codes_bytes = q ? n / 2 : 0;
  if (nvfp4_scales_bytes) *nvfp4_scales_bytes = q ? n / 16 : 0;
  return SP24_OK;
}

extern "C" int sp24_gemm_workspace_size(int x_format, int w_format, int sparse, int64_t M,
                                        int64_t N, int64_t K, int algo, int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return SP24_ERR_SHAPE;
  if (algo < SP24_ALGO_AUTO || algo > SP24_ALGO_TILED) return SP24_ERR_INVALID_ARG;
  if (x_format == SP24_NVFP4_MMA || w_format == SP24_NVFP4_MMA) {
    const bool q4 = (x_format == SP24_NVFP4 || x_format == SP24_NVFP4_MMA) &&
                    (w_format == SP24_NVFP4 || w_format == SP24_NVFP4_MMA);
    if (!q4 || sparse) return SP24_ERR_DTYPE;
    *bytes = w4a4_workspace(x_format == SP24_NVFP4_MMA, w_format == SP24_NVFP4_MMA, M, N, K);
    return SP24_OK;
  }
  if (!(is16(x_format) || x_format == SP24_NVFP4) || !(is16(w_format) || w_format == SP24_NVFP4))
    return SP24_ERR_DTYPE;
  const int wf = sparse ? (is16(w_format) ? W_S16 : W_SQ4) : (is16(w_format) ? W_D16 : W_DQ4);
  const int xf = x_format == SP24_NVFP4 ? X_Q4 : X_16;
  const bool tiled = algo == SP24_ALGO_TILED || (algo == SP24_ALGO_AUTO && !auto_skinny(xf, wf, M));
  *bytes = tiled ? tiled_workspace(xf, wf, M, N, K) : 0;
  return SP24_OK;
}

extern "C" int sp24_gemm_dense(const sp24_operand* x, const sp24_operand* w, int64_t M, int64_t N,
                               int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                               int algo, void* stream) {
  if (!x || !w) return SP24_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return SP24_ERR_SHAPE;
  if (algo < SP24_ALGO_AUTO || algo > SP24_ALGO_TILED) return SP24_ERR_INVALID_ARG;
  if (x->format == SP24_NVFP4_MMA || w->format == SP24_NVFP4_MMA) {
    // W4A4 with scales in the tensor cores' tile order: only the CTA-pair kernel reads them
    const bool xq = x->format == SP24_NVFP4 || x->format == SP24_NVFP4_MMA;
    const bool wq = w->format == SP24_NVFP4 || w->format == SP24_NVFP4_MMA;
    if (!xq || !wq) return SP24_ERR_DTYPE;
    if (K % 256) return SP24_ERR_SHAPE;
    if (algo == SP24_ALGO_SKINNY) return SP24_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return SP24_OK;
    if (!y) return SP24_ERR_INVALID_ARG;
    if (!aligned(y, 4)) return SP24_ERR_ALIGN;
    if (K > 0) {
      if (!x->data || !x->scales || !x->tensor_scale || !w->data || !w->scales || !w->tensor_scale)
        return SP24_ERR_INVALID_ARG;
      if (!aligned(x->data, 16) || !aligned(x->scales, 16) || !aligned(w->data, 16) || !aligned(w->scales, 16))
        return SP24_ERR_ALIGN;
    }
    return run_w4a4_pair(static_cast<const uint8_t*>(x->data), x->scales, x->format == SP24_NVFP4_MMA,
                         x->tensor_scale, static_cast<const uint8_t*>(w->data), w->scales,
                         w->format == SP24_NVFP4_MMA, w->tensor_scale, M, N, K, y, workspace, workspace_bytes,
                         as_stream(stream));
  }
  SkinnyParams p;
  memset(&p, 0, sizeof(p));
  int st = prep_x(x, M, K, &p);
  if (st) return st;
  int t16;
  st = mma_type(x->format, w->format, &t16);
  if (st) return st;
  int wf;
  if (is16(w->format)) {
    wf = W_D16;
    p.w_row_bytes = K * 2;
  } else if (w->format == SP24_NVFP4) {
    if (K % 32) return SP24_ERR_SHAPE;
    wf = W_DQ4;
    p.w_row_bytes = K / 2;
    p.scale_row_bytes = K / 16;
    if (N > 0 && K > 0 && (!w->scales || !w->tensor_scale)) return SP24_ERR_INVALID_ARG;
  } else {
    return SP24_ERR_DTYPE;
  }
  if (M == 0 || N == 0) return SP24_OK;
  if (!y) return SP24_ERR_INVALID_ARG;
  if (!aligned(y, 4)) return SP24_ERR_ALIGN;
  if (K > 0 && !w->data) return SP24_ERR_INVALID_ARG;
  if (!aligned(w->data, 16)) return SP24_ERR_ALIGN;
  p.w = reinterpret_cast<const uint8_t*>(w->data);
  p.w_scales = w->scales;
  p.w_ts = w->tensor_scale;
  p.M = M;
  p.N = N;
  p.K = K;
  p.y = y;
  return dispatch(wf, t16, p, algo, workspace, workspace_bytes, as_stream(stream));
}

extern "C" int sp24_gemm_sparse24(const sp24_operand* x, const sp24_sparse_operand* w, int64_t M,
                                  int64_t N, int64_t K, float* y, void* workspace,
                                  int64_t workspace_bytes, int algo, void* stream) {
  if (!x || !w) return SP24_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return SP24_ERR_SHAPE;
  if (algo < SP24_ALGO_AUTO || algo > SP24_ALGO_TILED) return SP24_ERR_INVALID_ARG;
  SkinnyParams p;
  memset(&p, 0, sizeof(p));
  int st = prep_x(x, M, K, &p);
  if (st) return st;
  int t16;
  st = mma_type(x->format, w->format, &t16);
  if (st) return st;
  int wf;
  if (is16(w->format)) {
    if (K % 16) return SP24_ERR_SHAPE;
    wf = W_S16;
    p.w_row_bytes = K;  // K/2 values of 2 bytes
  } else if (w->format == SP24_NVFP4) {
    if (K % 64) return SP24_ERR_SHAPE;
    wf = W_SQ4;
    p.w_row_bytes = K / 4;
    p.scale_row_bytes = K / 32;
    if (N > 0 && K > 0 && (!w->scales || !w->tensor_scale)) return SP24_ERR_INVALID_ARG;
  } else {
    return SP24_ERR_DTYPE;
  }
  p.meta_row_bytes = K / 8;
  if (M == 0 || N == 0) return SP24_OK;
  if (!y) return SP24_ERR_INVALID_ARG;
  if (!aligned(y, 4)) return SP24_ERR_ALIGN;
  if (K > 0 && (!w->values || !w->meta)) return SP24_ERR_INVALID_ARG;
  if (!aligned(w->values, 16) || !aligned(w->meta, 8)) return SP24_ERR_ALIGN;
  p.w = reinterpret_cast<const uint8_t*>(w->values);
  p.w_scales = w->scales;
  p.w_ts = w->tensor_scale;
  p.meta = w->meta;
  p.M = M;
  p.N = N;
  p.K = K;
  p.y = y;
  return dispatch(wf, t16, p, algo, workspace, workspace_bytes, as_stream(stream));
}

extern "C" int sp24_nvfp4_mma_size(int64_t rows, int64_t cols, int64_t* codes_bytes, int64_t* scales_bytes) {
  if (rows < 0 || cols < 0 || cols % 256) return SP24_ERR_SHAPE;
  if (codes_bytes) *codes_bytes = nvfp4_mma_codes_bytes(rows, cols);
  if (scales_bytes) *scales_bytes = nvfp4_mma_scales_bytes(rows, cols);
  return SP24_OK;
}

extern "C" int sp24_nvfp4_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                 uint8_t* codes_out, uint8_t* scales_out, void* stream) {
  if (rows < 0 || cols < 0 || cols % 256) return SP24_ERR_SHAPE;
  if (rows == 0 || cols == 0) return SP24_OK;
  if (!codes || !scales || !codes_out || !scales_out) return SP24_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 4) || !aligned(codes_out, 16) || !aligned(scales_out, 16))
    return SP24_ERR_ALIGN;
  return nvfp4_to_mma(codes, scales, rows, cols, codes_out, scales_out, as_stream(stream));
}

extern "C" int64_t sp24_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" int sp24_last_device_error(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return SP24_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int)) != cudaSuccess) return SP24_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int)) != cudaSuccess) return SP24_ERR_CUDA;
  return v;
}
