// a7 on the tensor cores: routed-expert GEMM with 16-bit tokens and NVFP4 experts (W4A16).
//
// [P1] "NVFP4 vs 2:4 sparse", "Concurrency, not sparsity, is the lever": every touched expert's
// weights are read once per step, and the tokens routed to it share that read.  One CTA computes
// one token tile of one expert (up to 128 routed rows) against 128 of the expert's weight rows
// over the whole K, so every output has one writer and no K slice is reduced through atomics.
//
// Per 64-wide K stage (a ring of S stages in shared memory):
//   * 256 producer threads copy the stage's raw FP4 codes and E4M3 block scales of the 128
//     weight rows, and gather the tile's token rows of x, with 16-byte cp.async (zero-filled
//     past the tile's count) `S - 1` stages ahead;
//   * once a stage's raw bytes have landed they expand the codes to the 16-bit type of x
//     (exact: integer shifts into 16-bit patterns times the folded block scale) straight into
//     the 128-byte-swizzled K-major layout the MMA descriptors read, fence the generic proxy
//     against the async proxy, and arrive on the stage's full barrier;
//   * one thread issues four `tcgen05.mma kind::f16` (M = 128 weight rows, N = the tile's
//     token count rounded up to 16, K = 16) into a TMEM accumulator and commits the stage's
//     empty barrier;
//   * after the last stage, four warps read the accumulator (TMEM lane = weight row, column =
//     token) and store y[token, slot, row] * 256 * tensor scale.
// Every wait is bounded; on a timeout the CTA records SP24_ERR_DEVICE_TIMEOUT, lets its copies
// land, frees its TMEM and returns.
#include "sp24_fp4.cuh"
#include "sp24_internal.cuh"
#include "sp24_tc.cuh"

namespace sp24 {
namespace {

using namespace tc;

constexpr int kMtRows = 128;      // weight rows per CTA (MMA M)
constexpr int kMtTok = 128;       // routed rows per token tile (MMA N <= 128)
constexpr int kMtBK = 64;         // K per stage (one 128-byte swizzle row of 16-bit values)
constexpr int kMtDx = 3;          // stages of x gathered ahead of the one being converted
constexpr int kMtDw = 11;         // stages of raw weights copied ahead
constexpr int kMtSlotsA = 2;      // expanded weight tiles: stage i reuses the slot of MMA i - 2
constexpr int kMtSlotsB = kMtDx + 2;
constexpr int kMtSlotsR = kMtDw + 1;
constexpr int kMtProducers = 256;
constexpr int kMtThreads = kMtProducers + 32;  // + the MMA warp
constexpr int kMtCols = 128;                   // TMEM accumulator columns (one per routed row)
constexpr uint32_t kMtA = kMtRows * kMtBK * 2;   // 16 KB
constexpr uint32_t kMtB = kMtTok * kMtBK * 2;    // 16 KB
constexpr uint32_t kMtRawC = kMtRows * kMtBK / 2;  // 4 KB of codes
constexpr uint32_t kMtRawS = kMtProducers * 4;     // one 4-byte scale word per producer thread
constexpr uint32_t kMtRaw = kMtRawC + kMtRawS;
constexpr size_t kMtSmem = (size_t)kMtSlotsA * kMtA + (size_t)kMtSlotsB * kMtB + (size_t)kMtSlotsR * kMtRaw + 1024;
static_assert(kMtSmem <= 227 * 1024, "shared memory");

// Offset of 16-byte chunk j (K elements 8j .. 8j + 7) of row r in a 128-byte-swizzled K-major
// tile: 8-row atoms of 1024 bytes, chunk j of row r stored at chunk j ^ (r % 8).
__device__ __forceinline__ uint32_t sw128(int r, int j) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

// 16-byte copy that reads `src_bytes` (16 or 0) and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// 4-byte copy (block scales of one row).
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

struct MoeTcParams {
  const uint16_t* x;        // [T, K] 16-bit tokens
  const uint8_t* codes;     // [E * N, K / 2]
  const uint8_t* scales;    // [E * N, K / 16]
  const float* w_ts;        // tensor scale of the stacked experts
  const int32_t* tiles;     // (expert, first permutation index, count) per token tile
  const int32_t* perm;      // flat (token * topk + slot) of each routed row, grouped by expert
  float* y;                 // [T, topk, N]
  int topk;
  int64_t N, K;
};

// One CTA: token tile blockIdx.y (expert e, rows first .. first + count of the permutation) x
// weight rows 128 * blockIdx.x .. + 127 of expert e, over all of K.
template <typename T>
__global__ void __launch_bounds__(kMtThreads, 1) moe_w4a16_tc_kernel(const MoeTcParams p) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;                          // [kMtSlotsA][128 rows x 128 B], swizzled
  uint8_t* sB = sA + kMtSlotsA * kMtA;         // [kMtSlotsB][128 rows x 128 B], swizzled
  uint8_t* sR = sB + kMtSlotsB * kMtB;         // [kMtSlotsR][codes 128 x 32 B | scale words]
  __shared__ uint64_t full_bar[kMtSlotsA], empty_bar[kMtSlotsA], tfull_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int aborted;
  __shared__ int32_t s_perm[kMtTok];

  const int32_t* tile = p.tiles + 3 * (int64_t)blockIdx.y;
  const int count = tile[2];
  if (count <= 0) return;  // unused tile slot: the whole CTA leaves before any shared state
  const int e = tile[0], first = tile[1];
  const int n_mma = (count + 15) & ~15;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = (int64_t)e * p.N + (int64_t)blockIdx.x * kMtRows;  // stacked weight row
  const int KB = (int)(p.K / kMtBK);

  if (tid < count) s_perm[tid] = p.perm[first + tid];
  if (tid == 0) {
    for (int s = 0; s < kMtSlotsA; ++s) {
      mbar_init(&full_bar[s], kMtProducers);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&tfull_bar, 1);
    aborted = 0;
    fence_mbar_init();
  }
  if (warp == 8) tmem_alloc(&tmem_base, kMtCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp < 8) {
    // ---- producers: thread (r, h) owns codes bytes 16h .. 16h + 15 of weight row r per stage
    // and converts them; thread (i0, j) gathers 16-byte chunk j of routed rows i0 + 32u.
    const int r = tid >> 1, h = tid & 1, j = tid & 7;
    const uint8_t* gc = p.codes + (row0 + r) * (p.K / 2) + 16 * h;
    const uint8_t* gs = p.scales + (row0 + r) * (p.K / 16);
    const uint16_t* xrow[4];
    uint32_t xoff[4], xbytes[4];
    int nx = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = (tid >> 3) + 32 * u;
      xoff[u] = sw128(i, j);
      xbytes[u] = i < count ? 16u : 0u;  // rows count .. n_mma - 1 are zero-filled
      xrow[u] = p.x + (i < count ? (int64_t)(s_perm[i] / p.topk) * p.K : 0) + 8 * j;
      nx += i < n_mma;
    }
    const uint32_t a_off = (uint32_t)r;  // row of this thread's expanded chunks
#pragma unroll 1
    for (int i = -kMtDw; i < KB; ++i) {
      if (i >= 2) {  // A slot i % 2 and B slot (i + kMtDx) % kMtSlotsB were last read by MMA i - 2
        if (!mbar_wait(&empty_bar[i & 1], ((i - 2) >> 1) & 1) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
      }
      const int kw = i + kMtDw;
      if (kw < KB) {
        uint8_t* raw = sR + (kw % kMtSlotsR) * kMtRaw;
        cp_async16(raw + 32 * r + 16 * h, gc + (int64_t)kw * (kMtBK / 2));
        cp_async4(raw + kMtRawC + 4 * tid, gs + (int64_t)kw * (kMtBK / 16));
      }
      const int kx = i + kMtDx;
      if (kx >= 0 && kx < KB) {
        uint8_t* b = sB + (kx % kMtSlotsB) * kMtB;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (u < nx) cp_async16_zfill(b + xoff[u], xrow[u] + (int64_t)kx * kMtBK, xbytes[u]);
      }
      cp_async_commit();
      if (i < 0) continue;
      cp_async_wait<kMtDx>();  // this thread's copies of stage i (x and raw weights) have landed
      const uint8_t* raw = sR + (i % kMtSlotsR) * kMtRaw;
      const uint4 cw = *reinterpret_cast<const uint4*>(raw + 32 * r + 16 * h);
      const uint32_t sw = *reinterpret_cast<const uint32_t*>(raw + kMtRawC + 4 * tid);
      uint32_t s0, s1;
      scale_pair<T>(sw >> (16 * h), s0, s1);  // blocks 2h, 2h + 1 of the stage
      uint8_t* a = sA + (i & 1) * kMtA;
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // chunk 4h + c: K elements 8(4h + c) .. + 7
        const uint32_t s = c < 2 ? s0 : s1;
        uint4 o;
        o.x = hmul2u<T>(fp4_pair_byte<T>(words[c], 0), s);
        o.y = hmul2u<T>(fp4_pair_byte<T>(words[c], 1), s);
        o.z = hmul2u<T>(fp4_pair_byte<T>(words[c], 2), s);
        o.w = hmul2u<T>(fp4_pair_byte<T>(words[c], 3), s);
        *reinterpret_cast<uint4*>(a + sw128((int)a_off, 4 * h + c)) = o;
      }
      fence_proxy_async_smem();  // generic writes and landed cp.async data -> MMA operand reads
      mbar_arrive(&full_bar[i & 1]);
    }
    cp_async_wait<0>();  // nothing may land after an early exit

    // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (weight rows), column chunks
    // w / 4, w / 4 + 2 (routed rows), and stores each routed row's 32 outputs with one store.
    if (mbar_wait(&tfull_bar, 0)) {
      tc_fence_after();
      const int q = warp & 3;
      const int64_t orow = (int64_t)blockIdx.x * kMtRows + 32 * q + lane;
      const float scale = 256.0f * *p.w_ts;
#pragma unroll 1
      for (int c = warp >> 2; 32 * c < count; c += 2) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * c, v);
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
          const int i = 32 * c + ii;
          if (i < count) p.y[(int64_t)s_perm[i] * p.N + orow] = v[ii] * scale;
        }
      }
    } else {
      aborted = 1;
    }
  } else if (lane == 0) {
    // ---- MMA issuer: four K = 16 steps per stage into the TMEM accumulator
    const uint32_t idesc = idesc_f16(kMtRows, n_mma, kBf16);
#pragma unroll 1
    for (int i = 0; i < KB; ++i) {
      if (!mbar_wait(&full_bar[i & 1], (i >> 1) & 1) || *(volatile int*)&aborted) {
        aborted = 1;
        break;
      }
      tc_fence_after();
      const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA + (i & 1) * kMtA));
      const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB + (i % kMtSlotsB) * kMtB));
#pragma unroll
      for (int k = 0; k < kMtBK / 16; ++k) umma_f16(tmem, a0 + 2 * k, b0 + 2 * k, idesc, (i | k) != 0);
      umma_commit(&empty_bar[i & 1]);
    }
    umma_commit(&tfull_bar);  // also after an abort, so the epilogue does not wait in vain
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && aborted) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kMtCols);
  }
}

template <typename T>
int launch_moe_tc(const MoeTcParams& p, int64_t n_tiles, cudaStream_t s) {
  auto kern = moe_w4a16_tc_kernel<T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMtSmem) != cudaSuccess)
    return SP24_ERR_CUDA;
  dim3 grid((unsigned)(p.N / kMtRows), (unsigned)n_tiles);
  kern<<<grid, kMtThreads, kMtSmem, s>>>(p);
  return launch_status();
}

}  // namespace

bool moe_tc_supported(int wf, int x_fmt, int64_t N, int64_t K, int64_t max_tiles, const void* codes,
                      const void* scales, const void* x) {
  return wf == W_DQ4 && x_fmt == X_16 && N > 0 && N % kMtRows == 0 && N / kMtRows <= 65535 && K > 0 &&
         K % kMtBK == 0 && K / kMtBK <= INT32_MAX && max_tiles <= 65535 && aligned(codes, 16) &&
         aligned(scales, 4) && aligned(x, 16);
}

int moe_tc_grouped(int t16, const SkinnyParams& sp, int64_t n_tiles, cudaStream_t s) {
  MoeTcParams p{};
  p.x = reinterpret_cast<const uint16_t*>(sp.x);
  p.codes = sp.w;
  p.scales = sp.w_scales;
  p.w_ts = sp.w_ts;
  p.tiles = sp.tiles;
  p.perm = sp.perm;
  p.y = sp.y;
  p.topk = sp.topk;
  p.N = sp.N;
  p.K = sp.K;
  if (n_tiles <= 0) return SP24_OK;
  return t16 == SP24_F16 ? launch_moe_tc<__half>(p, n_tiles, s) : launch_moe_tc<__nv_bfloat16>(p, n_tiles, s);
}

}  // namespace sp24
