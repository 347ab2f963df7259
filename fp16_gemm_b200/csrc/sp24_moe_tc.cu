// a7 on the tensor cores: routed-expert GEMM with 16-bit tokens and NVFP4 experts (W4A16).
//
// [P1] "NVFP4 vs 2:4 sparse", "Concurrency, not sparsity, is the lever": every touched expert's
// weights are read once per step, and the tokens routed to it share that read.  One CTA computes
// one token tile of one expert (up to 128 routed rows) against 128 of the expert's weight rows
// over the whole K, so every output has one writer and no K slice is reduced through atomics.
//
// Roles (K advances in stages of 64; stage i uses slot i % 10 of an x ring in shared memory and
// of an A ring in tensor memory; slots are synchronised in pairs):
//   * TMA warp W loads the raw weights of four stages at a time: the 128 rows' code bytes
//     (128-byte rows, 128-byte swizzle) and their E4M3 block scales (16-byte rows);
//   * eight gather warps copy the tile's token rows of x for each stage with 16-byte cp.async
//     (rows past the tile's count zero-filled) into a 128-byte swizzled K-major tile, the MMA's
//     B operand, three stage pairs ahead; once a pair has landed they fence the generic proxy
//     against the async proxy and arrive on its barrier (TMA row gathers move only 512 bytes per
//     instruction, and the SM issues TMA instructions far too slowly for that);
//   * four groups of four converter warps: group g expands stages g, g + 4, g + 8, ... (thread
//     = weight row): code pairs -> 16-bit values (hardware E2M1 conversion) times the block
//     scale, written with tcgen05.st into the stage's 32-column slot of tensor memory, the MMA's
//     A operand (lane = weight row, two K elements per column), then arrive on its barrier;
//   * one thread issues four `tcgen05.mma kind::f16` per stage (M = 128 weight rows, N = the
//     tile's count rounded up to 16, K = 16, A from TMEM, B from shared memory) into a TMEM
//     accumulator and commits the slot back to its producers.  An MMA instruction costs the
//     same for any N up to 64 and little more up to 128, so at ~80 routed rows this thread's own
//     pace matters: one barrier per stage, tested for the next stage before the current
//     stage's MMAs are issued;
//   * after the last stage the converter warps read the accumulator (lane = weight row, column
//     = routed row) and store y[token, slot, row] * unscale * tensor scale once.
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
constexpr int kMtBK = 64;         // K per stage
constexpr int kMtBoxK = 256;      // K per weight box (four stages)
constexpr int kMtBoxes = 3;       // weight boxes in flight (12 stages)
constexpr int kMtSlots = 10;      // stage slots: x tile in shared memory + A slot in TMEM (i % 10)
constexpr int kMtPairs = kMtSlots / 2;
constexpr int kMtDp = kMtPairs - 2;  // x is copied three stage pairs ahead (the slot pair's MMAs, two pairs back, are done)
constexpr int kMtGroups = 4;      // converter groups
constexpr int kMtConvWarps = 4 * kMtGroups;
constexpr int kMtGatherWarps = 8;
constexpr int kMtWarpMma = kMtConvWarps, kMtWarpW = kMtConvWarps + 1, kMtWarpX0 = kMtConvWarps + 2;
constexpr int kMtThreads = 32 * (kMtWarpX0 + kMtGatherWarps);
constexpr uint32_t kMtCodeBox = kMtRows * kMtBoxK / 2;    // 16 KB: 128 rows x 128 code bytes
constexpr uint32_t kMtScaleBox = kMtRows * kMtBoxK / 16;  // 2 KB: 128 rows x 16 scale bytes
constexpr uint32_t kMtBox = kMtCodeBox + kMtScaleBox;
constexpr uint32_t kMtX = kMtTok * kMtBK * 2;              // 16 KB
constexpr size_t kMtSmem = (size_t)kMtBoxes * kMtBox + (size_t)kMtSlots * kMtX + 1024;
constexpr uint32_t kMtAccCols = 128;                       // fp32 accumulator, one column per routed row
constexpr uint32_t kMtACols = kMtBK / 2;                   // 32 columns: one stage of A (16-bit pairs)
constexpr uint32_t kMtCols = 512;                          // accumulator + kMtSlots A slots
static_assert(kMtAccCols + kMtSlots * kMtACols <= kMtCols, "tensor memory");
static_assert(kMtSmem <= 227 * 1024, "shared memory");

// 16-byte copy that reads `src_bytes` (16 or 0) and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

// Offset of 16-byte chunk j (K elements 8j .. 8j + 7) of row r in a 128-byte-swizzled K-major
// tile: 8-row atoms of 1024 bytes, chunk j of row r stored at chunk j ^ (r % 8).
__device__ __forceinline__ uint32_t sw128(int r, int j) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

struct MoeTcParams {
  const uint16_t* x;     // [T, K] 16-bit tokens
  const float* w_ts;     // tensor scale of the stacked experts
  const int32_t* tiles;  // (expert, first permutation index, count) per token tile
  const int32_t* perm;   // flat (token * topk + slot) of each routed row, grouped by expert
  float* y;              // [T, topk, N]
  int topk;
  int T;
  int N, K;
};

// Four E2M1 code pairs (the bytes of w, low nibble = lower K index) -> four packed 16-bit pairs
// of the code values: exact f16 from the hardware conversion; for bf16 the same bits moved
// into the bf16 fields, E2M1 * 2^-112 (every E2M1 magnitude is a normal f16 with one mantissa
// bit, so the shift drops only zero bits and no neighbour bits cross into a half).
template <typename T>
__device__ __forceinline__ void e2m1x8_to_16(uint32_t w, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
#pragma unroll
    for (int p = 0; p < 4; ++p) h[p] = ((h[p] & 0x7FFF7FFFu) >> 3) | (h[p] & 0x80008000u);
  }
}

// The four block-scale multipliers of one stage (E4M3 codes in the bytes of `sw`), each in both
// halves of a word: E4M3 (f16: the products stay exact, at most 6 significant bits between
// 2^-10 and 2688) or E4M3 * 2^104 (bf16: with the codes at E2M1 * 2^-112 every product is
// E2M1 * E4M3 * 2^-8, a normal bf16).
template <typename T>
__device__ __forceinline__ void block_scales4(uint32_t sw, uint32_t (&m)[4]) {
  uint32_t lo, hi;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(lo) : "h"((uint16_t)(sw & 0xffffu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hi) : "h"((uint16_t)(sw >> 16)));
  const uint32_t h[4] = {lo & 0xffffu, lo >> 16, hi & 0xffffu, hi >> 16};
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint32_t v = h[b];
    if constexpr (std::is_same<T, __nv_bfloat16>::value)
      v = to_bits16<T>(__half2float(__ushort_as_half((unsigned short)v)) * 0x1p104f);
    m[b] = v | (v << 16);
  }
}

// The factor that takes an accumulated product back to x . w: 2^8 for bf16 operands (see
// block_scales4), 1 for f16, times the experts' tensor scale.
template <typename T>
constexpr float kMtUnscale = std::is_same<T, __nv_bfloat16>::value ? 256.0f : 1.0f;

// One CTA: token tile blockIdx.y (expert e, rows first .. first + count of the permutation) x
// weight rows 128 * blockIdx.x .. + 127 of expert e, over all of K.
template <typename T>
__global__ void __launch_bounds__(kMtThreads, 1)
    moe_w4a16_tc_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmS,
                        const MoeTcParams p) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem;                           // [kMtBoxes][codes 128 x 128 B swizzled | scales 128 x 16 B]
  uint8_t* sX = smem + kMtBoxes * kMtBox;       // [kMtSlots][128 rows x 128 B swizzled]
  // Slots are synchronised in pairs (2q, 2q + 1), so the MMA thread waits and commits once per
  // two stages.  st_full[q]: both stages have their A (4 converter warps each) and their x (8
  // gather warps each); st_empty[q]: the MMAs that read the pair have completed (commit).
  __shared__ uint64_t w_full[kMtBoxes], w_empty[kMtBoxes], st_full[kMtPairs], st_empty[kMtPairs], tfull_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int aborted;
  __shared__ int32_t s_perm[kMtTok];

  const int32_t* tile = p.tiles + 3 * (int64_t)blockIdx.y;
  const int count = tile[2];
  if (count <= 0) return;  // unused tile slot: the whole CTA leaves before any shared state
  const int e = tile[0], first = tile[1];
  const int n_mma = (count + 15) & ~15;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = e * p.N + (int)blockIdx.x * kMtRows;  // stacked weight row (< 2^31)
  const int KB = p.K / kMtBK;                           // stages (a multiple of 4)

  if (tid < count) s_perm[tid] = p.perm[first + tid];
  if (tid == 0) {
    for (int s = 0; s < kMtBoxes; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], kMtConvWarps);
    }
    for (int q = 0; q < kMtPairs; ++q) {
      mbar_init(&st_full[q], 2 * 4 + kMtGatherWarps);  // two converter groups, the gather warps once
      mbar_init(&st_empty[q], 1);
    }
    mbar_init(&tfull_bar, 1);
    aborted = 0;
    fence_mbar_init();
  }
  if (warp == kMtWarpMma) tmem_alloc(&tmem_base, kMtCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp < kMtConvWarps) {
    // ---- converters: group g = warp / 4 expands stages g, g + 4, ...; thread = weight row r
    // (lane quarter warp % 4, the TMEM lanes this warp may access).
    const int g = warp >> 2, qd = warp & 3, r = 32 * qd + lane;
    const uint32_t t_lane = static_cast<uint32_t>(32 * qd) << 16;
    const uint32_t a_base = tmem + t_lane + kMtAccCols;
#pragma unroll 1
    for (int i = g, m = 0; i < KB; i += kMtGroups, ++m) {  // stage i = 4m + g: stage g of box m
      const int bs = m % kMtBoxes;
      if (!__all_sync(0xffffffffu, mbar_wait(&w_full[bs], (m / kMtBoxes) & 1) && !*(volatile int*)&aborted)) {
        aborted = 1;
        break;
      }
      const uint8_t* box = sW + bs * kMtBox;
      // this stage's 32 code bytes of row r: 16-byte chunks 2g, 2g + 1 of the swizzled row
      const uint4 c0 = *reinterpret_cast<const uint4*>(box + r * 128 + (((2 * g) ^ (r & 7)) << 4));
      const uint4 c1 = *reinterpret_cast<const uint4*>(box + r * 128 + (((2 * g + 1) ^ (r & 7)) << 4));
      const uint32_t sw = *reinterpret_cast<const uint32_t*>(box + kMtCodeBox + r * 16 + 4 * g);
      __syncwarp();
      if (lane == 0) mbar_arrive(&w_empty[bs]);  // the warp's raw bytes of this box are in registers
      uint32_t sc[4];
      block_scales4<T>(sw, sc);
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint32_t a[32];  // column j = K elements 2j, 2j + 1 of the stage
#pragma unroll
      for (int wi = 0; wi < 8; ++wi) {
        e2m1x8_to_16<T>(words[wi], &a[4 * wi]);
#pragma unroll
        for (int pq = 0; pq < 4; ++pq) a[4 * wi + pq] = hmul2u<T>(a[4 * wi + pq], sc[wi >> 1]);
      }
      const int as = i % kMtSlots;
      if (i >= kMtSlots &&
          !__all_sync(0xffffffffu, mbar_wait(&st_empty[as >> 1], ((i / kMtSlots) - 1) & 1))) {  // MMA i - 10 done
        aborted = 1;
        break;
      }
      tc_fence_after();
      tmem_st32(a_base + kMtACols * as, a);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st_full[as >> 1]);
    }

    // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (weight rows) and accumulator
    // columns 32 (w / 4) .. + 31 (routed rows), storing each routed row's 32 outputs at once.
    if (__all_sync(0xffffffffu, mbar_wait(&tfull_bar, 0))) {
      tc_fence_after();
      const int c = warp >> 2;
      if (32 * c < count) {
        const int orow = (int)blockIdx.x * kMtRows + r;
        const float scale = kMtUnscale<T> * *p.w_ts;
        float v[32];
        tmem_ld32(tmem + t_lane + 32 * c, v);
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
          const int i = 32 * c + ii;
          if (i < count) p.y[(int64_t)s_perm[i] * p.N + orow] = v[ii] * scale;
        }
      }
    } else {
      aborted = 1;
    }
  } else if (warp == kMtWarpMma) {
    if (lane == 0) {
      // ---- MMA issuer: four K = 16 steps per stage, A from TMEM slot i % 8, B from x slot i % 8.
      // The next stage's barrier is tested (without waiting) before this stage's MMAs are
      // issued, so the test's latency overlaps them.
      const uint32_t idesc = idesc_f16(kMtRows, n_mma, kBf16);
      const uint64_t b_first = desc_kmajor_sw128(smem_u32(sX));
      const int KP = KB / 2;  // stage pairs (KB is a multiple of 4)
      bool ready = mbar_wait(&st_full[0], 0);
#pragma unroll 1
      for (int pr = 0; pr < KP; ++pr) {
        if (!ready) {  // a producer gave up (or the wait ran out): stop issuing
          aborted = 1;
          break;
        }
        const int q = pr % kMtPairs, qn = (pr + 1) % kMtPairs;
        const uint32_t pn = ((pr + 1) / kMtPairs) & 1;
        const bool next = pr + 1 < KP && mbar_test_wait(&st_full[qn], pn);
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int s = 2 * q + h;
          const uint64_t b0 = b_first + (uint64_t)(s * (kMtX >> 4));  // descriptor address: 16-byte units
          const uint32_t a0 = tmem + kMtAccCols + kMtACols * s;
#pragma unroll
          for (int k = 0; k < kMtBK / 16; ++k)
            umma_f16_tmem_a(tmem, a0 + 8 * k, b0 + 2 * k, idesc, (pr | h | k) != 0);
        }
        umma_commit(&st_empty[q]);
        ready = pr + 1 >= KP || next || mbar_wait(&st_full[qn], pn);
      }
      umma_commit(&tfull_bar);  // also after an abort, so the epilogue does not wait in vain
    }
  } else if (warp == kMtWarpW) {
    if (lane == 0) {
      // ---- weight boxes: codes and block scales of four stages per copy pair
      int issued = 0;
#pragma unroll 1
      for (int m = 0; m < KB / 4; ++m) {
        const int s = m % kMtBoxes;
        if (!mbar_wait(&w_empty[s], ((m / kMtBoxes) & 1) ^ 1) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
        mbar_arrive_expect_tx(&w_full[s], kMtBox);
        tma_load_2d(sW + s * kMtBox, &tmC, &w_full[s], m * (kMtBoxK / 2), row0);
        tma_load_2d(sW + s * kMtBox + kMtCodeBox, &tmS, &w_full[s], m * (kMtBoxK / 16), row0);
        ++issued;
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int m = issued - kMtBoxes > 0 ? issued - kMtBoxes : 0; m < issued; ++m)
        mbar_wait(&w_full[m % kMtBoxes], (m / kMtBoxes) & 1);
    }
  } else {
    // ---- token rows: gather thread t copies 16-byte chunk t % 8 of routed rows t / 8 + 32u
    // (u = 0 .. 3) of each stage, kMtDp stage pairs ahead (rows count .. n_mma - 1 zero-filled)
    const int t = tid - 32 * kMtWarpX0, j = t & 7;
    const uint16_t* xrow[4];
    uint32_t xoff[4], xbytes[4];
    int nx = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = (t >> 3) + 32 * u;
      xoff[u] = sw128(i, j);
      xbytes[u] = i < count ? 16u : 0u;
      xrow[u] = p.x + (i < count ? (int64_t)(s_perm[i] / p.topk) * p.K : 0) + 8 * j;
      nx += i < n_mma;
    }
    auto issue = [&](int kx) {
      uint8_t* b = sX + (kx % kMtSlots) * kMtX;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (u < nx) cp_async16_zfill(b + xoff[u], xrow[u] + (int64_t)kx * kMtBK, xbytes[u]);
    };
    const int KP = KB / 2;
    for (int pp = 0; pp < kMtDp; ++pp) {  // the first pairs: their slots are fresh
      if (pp < KP) {
        issue(2 * pp);
        issue(2 * pp + 1);
      }
      cp_async_commit();
    }
#pragma unroll 1
    for (int pr = 0; pr < KP; ++pr) {
      cp_async_wait<kMtDp - 1>();  // this thread's chunks of stage pair pr have landed
      fence_proxy_async_smem();    // ... and are visible to the MMA's operand reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&st_full[pr % kMtPairs]);
      const int pn = pr + kMtDp;
      if (pn < KP) {
        if (pn >= kMtPairs) {  // the slot pair's previous pair pn - kMtPairs = pr - 2 is multiplied
          const bool ok = mbar_wait(&st_empty[pn % kMtPairs], ((pn / kMtPairs) - 1) & 1) && !*(volatile int*)&aborted;
          if (!__all_sync(0xffffffffu, ok)) {
            aborted = 1;
            break;
          }
        }
        issue(2 * pn);
        issue(2 * pn + 1);
      }
      cp_async_commit();
    }
    cp_async_wait<0>();  // nothing may land after an early exit
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && aborted) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
  if (warp == kMtWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kMtCols);
  }
}

template <typename T>
int launch_moe_tc(const CUtensorMap& tmC, const CUtensorMap& tmS, const MoeTcParams& p, int64_t n_tiles,
                  cudaStream_t s) {
  auto kern = moe_w4a16_tc_kernel<T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMtSmem) != cudaSuccess)
    return SP24_ERR_CUDA;
  dim3 grid((unsigned)(p.N / kMtRows), (unsigned)n_tiles);
  kern<<<grid, kMtThreads, kMtSmem, s>>>(tmC, tmS, p);
  return launch_status();
}

}  // namespace

bool moe_tc_supported(int wf, int x_fmt, int64_t T, int64_t E, int64_t N, int64_t K, int64_t max_tiles,
                      const void* codes, const void* scales, const void* x) {
  return wf == W_DQ4 && x_fmt == X_16 && T > 0 && T < INT32_MAX && N > 0 && N % kMtRows == 0 &&
         N / kMtRows <= 65535 && K > 0 && K % kMtBoxK == 0 && K <= INT32_MAX / 2 && E * N <= INT32_MAX &&
         max_tiles <= 65535 && aligned(codes, 16) && aligned(scales, 16) && aligned(x, 16);
}

int moe_tc_grouped(int t16, const SkinnyParams& sp, int64_t E, int64_t T, int64_t n_tiles, cudaStream_t s) {
  if (n_tiles <= 0) return SP24_OK;
  MoeTcParams p{};
  p.x = reinterpret_cast<const uint16_t*>(sp.x);
  p.w_ts = sp.w_ts;
  p.tiles = sp.tiles;
  p.perm = sp.perm;
  p.y = sp.y;
  p.topk = sp.topk;
  p.T = (int)T;
  p.N = (int)sp.N;
  p.K = (int)sp.K;
  const uint64_t rows = (uint64_t)(E * sp.N), K = (uint64_t)sp.K;
  CUtensorMap tmC, tmS;
  int st = make_tmap_2d(&tmC, sp.w, 1, rows, K / 2, K / 2, kMtBoxK / 2, kMtRows);  // codes, 128-byte swizzle
  if (!st) st = make_tmap_2d_plain(&tmS, sp.w_scales, rows, K / 16, K / 16, kMtBoxK / 16, kMtRows);
  if (st) return st;
  return t16 == SP24_F16 ? launch_moe_tc<__half>(tmC, tmS, p, n_tiles, s)
                         : launch_moe_tc<__nv_bfloat16>(tmC, tmS, p, n_tiles, s);
}

}  // namespace sp24
