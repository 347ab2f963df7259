// a7: routed-expert (MoE) grouped GEMM, dense and 2:4 sparse.
//
// [P1] "NVFP4 vs 2:4 sparse", "Concurrency, not sparsity, is the lever": tokens are routed top-10
// to 512 experts and every touched expert's weights are read once per step; section "Where it
// is supported in software" notes that no 2:4 grouped GEMM existed for such a model.
//
// Y[t, s, n] = sum_k x[t, k] W[e, n, k] with e = routing[t, s].  Steps, all on the device:
//   1. route_count:   histogram of expert ids (atomic adds into counts[E]);
//   2. route_scan:    one CTA turns counts into offsets (exclusive scan) and a table of token
//                     tiles (expert, first index, count <= tile);
//   3. route_scatter: each (t, s) takes a slot of its expert's range (perm = t * topk + s);
//   4. NVFP4 experts (dense or 2:4) with 16-bit tokens: the tensor-core kernel over tiles of up
//      to 128 routed rows, each CTA writing its outputs once; other formats: the staged skinny kernel in
//      grouped mode over tiles of 64 (grid: 64-row weight blocks, K slices, tiles), each CTA
//      gathering its tile's x rows by index and adding into Y[t, s, :].
// The order of tokens inside an expert's range depends on atomic arrival, but every output is a
// complete sum for one (t, s), so the result does not.
#include "sp24_internal.cuh"

namespace sp24 {
namespace {

constexpr int kTile = 64;     // token tile of the skinny kernel (the smallest tile: sizes the table)
constexpr int kTileTc = 128;  // token tile of the tensor-core kernel

__global__ void route_count(const int32_t* __restrict__ routing, int64_t n, int64_t E, int32_t* __restrict__ counts) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t e = routing[i];
    if (e < 0 || e >= E) {
      set_dev_error(SP24_ERR_INVALID_ARG);
      continue;
    }
    atomicAdd(&counts[e], 1);
  }
}

// Single CTA of 1024 threads: block-wide exclusive scans over E experts in chunks of 1024.
__global__ void __launch_bounds__(1024) route_scan(const int32_t* __restrict__ counts, int64_t E,
                                                   int32_t* __restrict__ offsets, int32_t* __restrict__ tiles,
                                                   int64_t max_tiles, int tile, int32_t* __restrict__ n_tiles) {
  __shared__ int32_t warp_sum[2][32];
  __shared__ int32_t carry[2];
  if (threadIdx.x == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t base = 0; base < E; base += 1024) {
    const int64_t e = base + threadIdx.x;
    const int32_t cnt = e < E ? counts[e] : 0;
    const int32_t nt = (cnt + tile - 1) / tile;
    // inclusive warp scans of (cnt, nt)
    int32_t a = cnt, b = nt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t ya = __shfl_up_sync(0xffffffffu, a, d), yb = __shfl_up_sync(0xffffffffu, b, d);
      if (lane >= d) {
        a += ya;
        b += yb;
      }
    }
    if (lane == 31) {
      warp_sum[0][warp] = a;
      warp_sum[1][warp] = b;
    }
    __syncthreads();
    if (warp == 0) {
      int32_t wa = warp_sum[0][lane], wb = warp_sum[1][lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t ya = __shfl_up_sync(0xffffffffu, wa, d), yb = __shfl_up_sync(0xffffffffu, wb, d);
        if (lane >= d) {
          wa += ya;
          wb += yb;
        }
      }
      warp_sum[0][lane] = wa;  // inclusive over warps
      warp_sum[1][lane] = wb;
    }
    __syncthreads();
    const int32_t pre_a = carry[0] + (warp ? warp_sum[0][warp - 1] : 0) + a - cnt;  // exclusive
    const int32_t pre_b = carry[1] + (warp ? warp_sum[1][warp - 1] : 0) + b - nt;
    if (e < E) {
      offsets[e] = pre_a;
      for (int32_t j = 0; j < nt && pre_b + j < max_tiles; ++j) {
        int32_t* t = tiles + 3 * (int64_t)(pre_b + j);
        t[0] = (int32_t)e;
        t[1] = pre_a + tile * j;
        t[2] = cnt - tile * j < tile ? cnt - tile * j : tile;
      }
    }
    __syncthreads();
    if (threadIdx.x == 1023) {
      carry[0] = pre_a + cnt;
      carry[1] = pre_b + nt;
    }
    __syncthreads();
  }
  // unused tile slots get count 0 (those CTAs exit at once); the used ones come first
  for (int64_t i = carry[1] + threadIdx.x; i < max_tiles; i += blockDim.x) tiles[3 * i + 2] = 0;
  if (threadIdx.x == 0) *n_tiles = carry[1] < max_tiles ? carry[1] : (int32_t)max_tiles;
}

// Also zeroes the outputs of routed rows with an invalid expert id when `y_zero` is set (the
// tensor-core path writes every valid output once and clears nothing else beforehand).
__global__ void route_scatter(const int32_t* __restrict__ routing, int64_t n, int64_t E,
                              const int32_t* __restrict__ offsets, int32_t* __restrict__ fill,
                              int32_t* __restrict__ perm, float* __restrict__ y_zero, int64_t N) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t e = routing[i];
    if (e < 0 || e >= E) {
      if (y_zero)
        for (int64_t c = 0; c < N; ++c) y_zero[i * N + c] = 0.0f;
      continue;
    }
    perm[offsets[e] + atomicAdd(&fill[e], 1)] = (int32_t)i;
  }
}

struct MoeWs {
  int32_t *counts, *fill, *offsets, *n_tiles, *tiles, *perm;
  int64_t max_tiles, bytes;
};

MoeWs moe_layout(void* base, int64_t T, int topk, int64_t E) {
  MoeWs w{};
  const int64_t n = T * topk;
  w.max_tiles = (n + kTile - 1) / kTile + E;
  auto r16 = [](int64_t b) { return (b + 15) / 16 * 16; };
  int64_t off = 0;
  uint8_t* p = reinterpret_cast<uint8_t*>(base);
  w.counts = reinterpret_cast<int32_t*>(p + off);
  off += r16(4 * E);
  w.fill = reinterpret_cast<int32_t*>(p + off);
  off += r16(4 * E);
  w.offsets = reinterpret_cast<int32_t*>(p + off);
  off += r16(4 * E);
  w.n_tiles = reinterpret_cast<int32_t*>(p + off);
  off += 16;
  w.tiles = reinterpret_cast<int32_t*>(p + off);
  off += r16(12 * w.max_tiles);
  w.perm = reinterpret_cast<int32_t*>(p + off);
  off += r16(4 * n);
  w.bytes = off;
  return w;
}

bool is16(int f) { return f == SP24_F16 || f == SP24_BF16; }

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_gemm_grouped_workspace_size(int64_t T, int topk, int64_t E, int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  if (T < 0 || topk < 0 || E <= 0) return SP24_ERR_SHAPE;
  *bytes = moe_layout(nullptr, T, topk, E).bytes;
  return SP24_OK;
}

extern "C" int sp24_gemm_grouped(const sp24_operand* x, const int32_t* routing, int64_t T, int topk,
                                 const sp24_operand* w_dense, const sp24_sparse_operand* w_sparse, int64_t E,
                                 int64_t N, int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                                 void* stream) {
  if (!x || (!w_dense == !w_sparse)) return SP24_ERR_INVALID_ARG;
  if (T < 0 || topk < 0 || E <= 0 || N < 0 || K < 0) return SP24_ERR_SHAPE;
  if (E > INT32_MAX || T * topk > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  const int64_t n = T * topk;
  if (n == 0 || N == 0) return SP24_OK;
  if (!routing || !y) return SP24_ERR_INVALID_ARG;
  if (!aligned(y, 4)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (K == 0) return cudaMemsetAsync(y, 0, (size_t)(n * N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;

  SkinnyParams p{};
  // activations
  if (x->format == SP24_NVFP4) {
    if (K % 32 || !x->data || !x->scales || !x->tensor_scale) return SP24_ERR_INVALID_ARG;
    p.x_fmt = X_Q4;
  } else if (is16(x->format)) {
    if (K % 8 || !x->data) return SP24_ERR_INVALID_ARG;
    if (!aligned(x->data, 16)) return SP24_ERR_ALIGN;
    p.x_fmt = X_16;
  } else {
    return SP24_ERR_DTYPE;
  }
  p.x = x->data;
  p.x_scales = x->scales;
  p.x_ts = x->tensor_scale;
  // expert weights, stacked [E * N, K]
  int wf, wformat;
  if (w_dense) {
    wformat = w_dense->format;
    if (is16(wformat)) {
      wf = W_D16;
      p.w_row_bytes = K * 2;
    } else if (wformat == SP24_NVFP4) {
      wf = W_DQ4;
      p.w_row_bytes = K / 2;
      p.scale_row_bytes = K / 16;
      if (!w_dense->scales || !w_dense->tensor_scale) return SP24_ERR_INVALID_ARG;
    } else {
      return SP24_ERR_DTYPE;
    }
    p.w = reinterpret_cast<const uint8_t*>(w_dense->data);
    p.w_scales = w_dense->scales;
    p.w_ts = w_dense->tensor_scale;
  } else {
    wformat = w_sparse->format;
    if (is16(wformat)) {
      wf = W_S16;
      p.w_row_bytes = K;
    } else if (wformat == SP24_NVFP4) {
      wf = W_SQ4;
      p.w_row_bytes = K / 4;
      p.scale_row_bytes = K / 32;
      if (!w_sparse->scales || !w_sparse->tensor_scale) return SP24_ERR_INVALID_ARG;
    } else {
      return SP24_ERR_DTYPE;
    }
    p.w = reinterpret_cast<const uint8_t*>(w_sparse->values);
    p.w_scales = w_sparse->scales;
    p.w_ts = w_sparse->tensor_scale;
    p.meta = w_sparse->meta;
    p.meta_row_bytes = K / 8;
  }
  if (!p.w || (w_sparse && !p.meta)) return SP24_ERR_INVALID_ARG;
  if (is16(x->format) && is16(wformat) && x->format != wformat) return SP24_ERR_DTYPE;
  const int t16 = is16(x->format) ? x->format : (is16(wformat) ? wformat : SP24_BF16);
  p.N = N;
  p.K = K;
  p.y = y;
  const bool tc = moe_tc_supported(wf, p.x_fmt, T, E, N, K, n / kTileTc + E, p.w, p.w_scales, p.meta, p.x);
  const int tile = tc ? kTileTc : kTile;
  p.M = tile;
  if (!tc && !skinny2_supported(wf, p)) return SP24_ERR_UNSUPPORTED;
  // the skinny kernel adds K-slice partial sums into Y; the tensor-core kernel stores each output
  if (!tc && cudaMemsetAsync(y, 0, (size_t)(n * N) * sizeof(float), s) != cudaSuccess) return SP24_ERR_CUDA;

  MoeWs ws = moe_layout(workspace, T, topk, E);
  if (!workspace || workspace_bytes < ws.bytes) return SP24_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return SP24_ERR_ALIGN;
  const size_t zero_bytes = (size_t)(reinterpret_cast<uint8_t*>(ws.offsets) - reinterpret_cast<uint8_t*>(ws.counts));
  if (cudaMemsetAsync(ws.counts, 0, zero_bytes, s) != cudaSuccess) return SP24_ERR_CUDA;  // counts + fill
  const int blocks = (int)((n + 255) / 256 < (int64_t)sm_count() * 4 ? (n + 255) / 256 : (int64_t)sm_count() * 4);
  // tiles of `tile` rows: at most sum_e ceil(c_e / tile) <= n / tile + E of them
  const int64_t n_tiles = n / tile + E < ws.max_tiles ? n / tile + E : ws.max_tiles;
  route_count<<<blocks, 256, 0, s>>>(routing, n, E, ws.counts);
  route_scan<<<1, 1024, 0, s>>>(ws.counts, E, ws.offsets, ws.tiles, ws.max_tiles, tile, ws.n_tiles);
  route_scatter<<<blocks, 256, 0, s>>>(routing, n, E, ws.offsets, ws.fill, ws.perm, tc ? y : nullptr, N);
  int st = launch_status(3);
  if (st) return st;
  p.perm = ws.perm;
  p.tiles = ws.tiles;
  p.topk = topk;
  p.expert_rows = N;
  if (tc) return moe_tc_grouped(wf, t16, p, E, T, n_tiles, ws.n_tiles, s);
  return skinny2_grouped(wf, t16, p, n_tiles, s);
}

// ------------------------------------------------------------------ expert block
//
// y[t] = sum_s r[t, s] * (SiLU(x_t Wg_e^T) * (x_t Wu_e^T)) Wd_e^T,  e = routing[t, s]
// ([P1] "Concurrency, not sparsity, is the lever": the routed experts of a decode step).
// Routing as for sp24_gemm_grouped (tiles of up to 128 routed rows), then the tensor-core
// kernel twice: gate/up (weights packed as 16-row gate / up blocks, SwiGLU in the epilogue, h in
// x's 16-bit type and routed order) and down (h rows read directly, each routed row's output
// stored once), then a streaming kernel sums each token's slots in order with the router weights
// (fp32, deterministic).

namespace sp24 {
namespace {

__global__ void interleave_rows_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, int64_t out_rows,
                                       int64_t vec_per_row, int64_t block_rows, uint4* __restrict__ out) {
  const int64_t n = out_rows * vec_per_row;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec_per_row, v = i - r * vec_per_row;
    const int64_t blk = r / (2 * block_rows), within = r - blk * 2 * block_rows;
    const int64_t src_row = blk * block_rows + (within % block_rows);
    out[i] = (within < block_rows ? a : b)[src_row * vec_per_row + v];
  }
}

int64_t block_h_bytes(int64_t T, int topk, int64_t F) { return (T * topk * F * 2 + 15) / 16 * 16; }
int64_t block_o_bytes(int64_t T, int topk, int64_t H) { return T * topk * H * 4; }

// y[t, n] = sum_s r[t, s] * o[t, s, n], the slots in order (fp32): four outputs per thread.
__global__ void combine_kernel(const float4* __restrict__ o, const float* __restrict__ r, int64_t T, int topk,
                               int64_t H4, float4* __restrict__ y) {
  const int64_t n = T * H4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / H4, c = i - t * H4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < topk; ++s) {
      const float w = r[t * topk + s];
      const float4 v = __ldcs(o + (t * topk + s) * H4 + c);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    y[i] = acc;
  }
}

}  // namespace
}  // namespace sp24

extern "C" int sp24_interleave_rows(const void* a, const void* b, int64_t rows, int64_t row_bytes,
                                    int64_t block_rows, void* out, void* stream) {
  if (rows < 0 || row_bytes < 0 || block_rows <= 0) return SP24_ERR_SHAPE;
  if (rows % block_rows || row_bytes % 16) return SP24_ERR_SHAPE;
  if (rows == 0 || row_bytes == 0) return SP24_OK;
  if (!a || !b || !out) return SP24_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16)) return SP24_ERR_ALIGN;
  const int64_t n = 2 * rows * (row_bytes / 16);
  const int64_t blocks = (n + 255) / 256 < (int64_t)sm_count() * 8 ? (n + 255) / 256 : (int64_t)sm_count() * 8;
  interleave_rows_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(
      reinterpret_cast<const uint4*>(a), reinterpret_cast<const uint4*>(b), 2 * rows, row_bytes / 16, block_rows,
      reinterpret_cast<uint4*>(out));
  return launch_status();
}

extern "C" int sp24_moe_block_workspace_size(int64_t T, int topk, int64_t E, int64_t H, int64_t F, int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  if (T < 0 || topk < 0 || E <= 0 || H < 0 || F < 0) return SP24_ERR_SHAPE;
  *bytes = moe_layout(nullptr, T, topk, E).bytes + block_h_bytes(T, topk, F) + block_o_bytes(T, topk, H);
  return SP24_OK;
}

namespace {

// An NVFP4 expert operand (dense or 2:4) of the block: format, pointers, validation.
struct BlockW {
  int wf;
  const uint8_t *codes, *scales, *meta;
  const float* ts;
};

int block_weights(const sp24_operand* d, const sp24_sparse_operand* s, BlockW* out) {
  if (!d == !s) return SP24_ERR_INVALID_ARG;
  if (d) {
    if (d->format != SP24_NVFP4) return SP24_ERR_DTYPE;
    *out = {W_DQ4, reinterpret_cast<const uint8_t*>(d->data), d->scales, nullptr, d->tensor_scale};
  } else {
    if (s->format != SP24_NVFP4) return SP24_ERR_DTYPE;
    *out = {W_SQ4, reinterpret_cast<const uint8_t*>(s->values), s->scales, s->meta, s->tensor_scale};
    if (!out->meta) return SP24_ERR_INVALID_ARG;
  }
  if (!out->codes || !out->scales || !out->ts) return SP24_ERR_INVALID_ARG;
  return SP24_OK;
}

}  // namespace

extern "C" int sp24_moe_block(const sp24_operand* x, const int32_t* routing, const float* router_w, int64_t T,
                              int topk, const sp24_operand* w_gate_up, const sp24_sparse_operand* w_gate_up_sparse,
                              const sp24_operand* w_down, const sp24_sparse_operand* w_down_sparse, int64_t E,
                              int64_t H, int64_t F, float* y, void* workspace, int64_t workspace_bytes,
                              void* stream) {
  if (!x) return SP24_ERR_INVALID_ARG;
  if (T < 0 || topk < 0 || E <= 0 || H < 0 || F < 0) return SP24_ERR_SHAPE;
  if (E > INT32_MAX || T * topk > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  if (!is16(x->format)) return SP24_ERR_DTYPE;
  BlockW gu, dn;
  int st = block_weights(w_gate_up, w_gate_up_sparse, &gu);
  if (!st) st = block_weights(w_down, w_down_sparse, &dn);
  if (st) return st;
  const int64_t n = T * topk;
  cudaStream_t s = as_stream(stream);
  if (H == 0 || T == 0) return SP24_OK;
  if (!y) return SP24_ERR_INVALID_ARG;
  if (!aligned(y, 16)) return SP24_ERR_ALIGN;  // the combine writes y as float4 rows (H % 4 == 0)
  if (n == 0 || F == 0) return cudaMemsetAsync(y, 0, (size_t)(T * H) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  if (!routing || !router_w || !x->data) return SP24_ERR_INVALID_ARG;
  if (!aligned(x->data, 16)) return SP24_ERR_ALIGN;
  // gate/up: N = 2F rows per expert, K = H; down: N = H rows per expert, K = F
  const int64_t bound = n / kTileTc + E;
  if (!moe_tc_supported(gu.wf, X_16, T, E, 2 * F, H, bound, gu.codes, gu.scales, gu.meta, x->data) ||
      !moe_tc_supported(dn.wf, X_16, T, E, H, F, bound, dn.codes, dn.scales, dn.meta, x->data))
    return SP24_ERR_UNSUPPORTED;
  MoeWs ws = moe_layout(workspace, T, topk, E);
  if (!workspace || workspace_bytes < ws.bytes + block_h_bytes(T, topk, F) + block_o_bytes(T, topk, H))
    return SP24_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return SP24_ERR_ALIGN;
  uint16_t* h = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(workspace) + ws.bytes);
  float* o = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + ws.bytes + block_h_bytes(T, topk, F));
  const size_t zero_bytes = (size_t)(reinterpret_cast<uint8_t*>(ws.offsets) - reinterpret_cast<uint8_t*>(ws.counts));
  if (cudaMemsetAsync(ws.counts, 0, zero_bytes, s) != cudaSuccess) return SP24_ERR_CUDA;
  const int blocks = (int)((n + 255) / 256 < (int64_t)sm_count() * 4 ? (n + 255) / 256 : (int64_t)sm_count() * 4);
  const int64_t n_tiles = bound < ws.max_tiles ? bound : ws.max_tiles;
  route_count<<<blocks, 256, 0, s>>>(routing, n, E, ws.counts);
  route_scan<<<1, 1024, 0, s>>>(ws.counts, E, ws.offsets, ws.tiles, ws.max_tiles, kTileTc, ws.n_tiles);
  route_scatter<<<blocks, 256, 0, s>>>(routing, n, E, ws.offsets, ws.fill, ws.perm, nullptr, 0);
  st = launch_status(3);
  if (st) return st;
  const int t16 = x->format;
  MoeBlockGemm g{};
  g.tiles = ws.tiles;
  g.perm = ws.perm;
  g.n_valid = ws.n_tiles;
  g.topk = topk;
  g.T = T;
  g.E = E;
  g.n_tiles = n_tiles;
  // gate / up -> h
  g.x = reinterpret_cast<const uint16_t*>(x->data);
  g.codes = gu.codes;
  g.scales = gu.scales;
  g.meta = gu.meta;
  g.w_ts = gu.ts;
  g.h = h;
  g.x_direct = 0;
  g.N = 2 * F;
  g.K = H;
  st = moe_tc_block_gemm(1, gu.wf, t16, g, s);
  if (st) return st;
  // down -> o[t, s, :] (every routed row's output stored once), then the slots combined in order
  g.x = h;
  g.codes = dn.codes;
  g.scales = dn.scales;
  g.meta = dn.meta;
  g.w_ts = dn.ts;
  g.h = nullptr;
  g.y = o;
  g.x_direct = 1;
  g.N = H;
  g.K = F;
  st = moe_tc_block_gemm(0, dn.wf, t16, g, s);
  if (st) return st;
  const int64_t nvec = T * (H / 4);
  const int64_t cb = (nvec + 255) / 256 < (int64_t)sm_count() * 8 ? (nvec + 255) / 256 : (int64_t)sm_count() * 8;
  combine_kernel<<<(unsigned)cb, 256, 0, s>>>(reinterpret_cast<const float4*>(o), router_w, T, topk, H / 4,
                                              reinterpret_cast<float4*>(y));
  return launch_status();
}
