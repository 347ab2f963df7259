// a7 on the tensor cores: routed-expert GEMM with 16-bit tokens and NVFP4 experts (W4A16),
// dense or 2:4-compressed.
//
// [P1] "NVFP4 vs 2:4 sparse", "Concurrency, not sparsity, is the lever": every touched expert's
// weights are read once per step, and the tokens routed to it share that read.  One CTA computes
// one token tile of one expert (up to 128 routed rows) against 128 of the expert's weight rows
// over the whole K, so every output has one writer and no K slice is reduced through atomics.
// [P2] "The mechanism needs both values and their positions": for 2:4 experts the kept values
// are the MMA's A operand and their positions travel as tcgen05 sparse metadata.
//
// The kernel is persistent: each CTA (one per SM) walks a list of items (token tile x 128-row
// block) and every ring below runs across them.  Roles (K advances in stages of 64 logical
// elements; stage i of the CTA's sequence uses slot i % 8 (dense) or i % 10 (2:4) of an x ring
// in shared memory and of an A ring in tensor memory; slots are synchronised in pairs):
//   * TMA warp W loads the raw weights of 4 (dense) or 8 (2:4) stages at a time: the 128 rows'
//     code bytes (128-byte rows, 128-byte swizzle), their E4M3 block scales (16-byte rows) and,
//     for 2:4, their metadata nibbles (64-byte rows);
//   * eight gather warps copy the tile's token rows of x for each stage with 16-byte cp.async
//     (rows past the tile's count zero-filled) into a 128-byte swizzled K-major tile, the MMA's
//     B operand, three stage pairs ahead; once a pair has landed they fence the generic proxy
//     against the async proxy and arrive on its barrier (TMA row gathers move only 512 bytes per
//     instruction, and the SM issues TMA instructions far too slowly for that);
//   * four groups of four converter warps: group g expands stages g, g + 4, g + 8, ... (thread
//     = weight row): code pairs -> 16-bit values (hardware E2M1 conversion) times the block
//     scale, written with tcgen05.st into the stage's slot of tensor memory, the MMA's A operand
//     (lane = weight row, two stored values per column: 32 columns dense, 16 for 2:4).  For 2:4
//     the row's metadata nibbles are regrouped with warp shuffles into the tcgen05 metadata
//     layout (TMEM lane l carries rows m = 16 (l / 16) + l % 8 and m + 8, the nibbles of groups
//     4 ((l / 8) % 2) .. + 3 of each 32-wide K window, one column per window: the low half for
//     row m, the high half for row m + 8) and stored into two columns beside the slot;
//   * one thread issues the stage's MMAs (M = 128 weight rows, N = the tile's count rounded up
//     to 16, A from TMEM, B from shared memory): four `tcgen05.mma kind::f16` (K = 16) dense,
//     two `tcgen05.mma.sp kind::f16` (K = 32 logical) for 2:4, into a TMEM accumulator, and
//     commits each slot pair back to its producers.  An MMA instruction costs about the same for
//     any N up to 128, so at ~80 routed rows the instruction count sets the pace and the 2:4
//     form needs half as many: one barrier per stage pair, tested for the next pair before the
//     current pair's MMAs are issued;
//   * four epilogue warps read a finished item's accumulator (lane = weight row, column = routed
//     row) and store y[token, slot, row] * unscale * tensor scale once, while the MMAs fill the
//     other of two accumulators with the next item.
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
constexpr int kMtBK = 64;         // logical K per stage
constexpr int kMtGroups = 4;      // converter groups
constexpr int kMtConvWarps = 4 * kMtGroups;
constexpr int kMtGatherWarps = 8;
constexpr int kMtEpiWarps = 4;
constexpr int kMtWarpMma = kMtConvWarps, kMtWarpW = kMtConvWarps + 1, kMtWarpX0 = kMtConvWarps + 2;
constexpr int kMtWarpEpi0 = kMtWarpX0 + kMtGatherWarps;
constexpr int kMtThreads = 32 * (kMtWarpEpi0 + kMtEpiWarps);
constexpr int kMtMaxItems = 256;  // items per CTA (the host sizes the grid for it)
constexpr uint32_t kMtX = kMtTok * kMtBK * 2;              // 16 KB
constexpr uint32_t kMtAccCols = 128;                       // fp32 accumulator, one column per routed row (two of them)
constexpr uint32_t kMtCols = 512;
constexpr uint32_t kMtCodeBox = kMtRows * 128;             // 16 KB: 128 rows x 128 code bytes
constexpr uint32_t kMtScaleBox = kMtRows * 16;             // 2 KB: 128 rows x 16 scale bytes

// Geometry of the dense (SP = false) and 2:4 (SP = true) weight streams.
template <bool SP>
struct MtGeom {
  static constexpr int kStagesPerBox = SP ? 8 : 4;                 // 128 code bytes per row per box
  static constexpr int kBoxK = kMtBK * kStagesPerBox;              // logical K per box
  static constexpr uint32_t kMetaBox = SP ? kMtRows * 64 : 0;      // 128 rows x 64 nibble bytes
  static constexpr uint32_t kBox = kMtCodeBox + kMtScaleBox + kMetaBox;
  static constexpr int kBoxes = SP ? 2 : 3;                        // 16 / 12 stages in flight
  static constexpr int kSlots = SP ? 10 : 8;                       // stage slots: x tile + A slot (i % kSlots)
  static constexpr uint32_t kACols = SP ? 16 : 32;                 // A columns per stage
  static constexpr uint32_t kACol0 = 2 * kMtAccCols;               // after the two accumulators
  static constexpr uint32_t kMetaCol0 = kACol0 + kSlots * kACols;  // 2 metadata columns per slot
  static constexpr size_t kSmem = (size_t)kBoxes * kBox + (size_t)kSlots * kMtX + 1024;
  static_assert(kSlots % 2 == 0 && kSlots >= 6, "slot pairs, copies two pairs behind the MMAs");
  static_assert(kMetaCol0 + (SP ? 2 * kSlots : 0) <= kMtCols, "tensor memory");
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kBox % 1024 == 0, "swizzled boxes stay 1024-byte aligned");
};

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

// Sparse (2:4) MMA, kind::f16, with A (the kept values) in tensor memory.
__device__ __forceinline__ void umma_f16_sp_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                   uint32_t e_tmem, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], [%1], %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Stores 16 / 2 consecutive 32-bit columns of this thread's TMEM lane (no wait).
__device__ __forceinline__ void tmem_st16_nowait(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st2_nowait(uint32_t taddr, uint32_t r0, uint32_t r1) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};" ::"r"(taddr), "r"(r0), "r"(r1) : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Epilogues: the routed-expert GEMM's store (also the expert block's down projection) and the
// expert block's gate/up activation.
enum { kEpiStore = 0, kEpiGlu = 1 };

struct MoeTcParams {
  const uint16_t* x;     // [T, K] 16-bit tokens; with x_direct, [routed rows, K] in routed order
  const float* w_ts;     // tensor scale of the stacked experts
  const int32_t* tiles;  // (expert, first permutation index, count) per token tile
  const int32_t* perm;   // flat (token * topk + slot) of each routed row, grouped by expert
  const int32_t* n_valid;  // number of used tiles (they come first in the table)
  float* y;              // store: [T, topk, N]
  uint16_t* h;           // glu: [routed rows, N / 2] in routed order, x's 16-bit type
  int x_direct;          // x row of routed row p is row p (else token perm[p] / topk)
  int topk;
  int T;
  int N, K;
};

// The SwiGLU activation of the expert block: SiLU(g) * u = g / (1 + e^-g) * u, fp32.
__device__ __forceinline__ float swiglu(float g, float u) { return __fdiv_rn(g, 1.0f + expf(-g)) * u; }

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

// The NS (2 or 4) block-scale multipliers of one stage (E4M3 codes in the low bytes of `sw`),
// each in both halves of a word: E4M3 (f16: the products stay exact, at most 6 significant bits
// between 2^-10 and 2688) or E4M3 * 2^104 (bf16: with the codes at E2M1 * 2^-112 every product
// is E2M1 * E4M3 * 2^-8, a normal bf16).
template <typename T, int NS>
__device__ __forceinline__ void block_scales(uint32_t sw, uint32_t (&m)[NS]) {
  uint32_t h[4];
#pragma unroll
  for (int q = 0; q < NS / 2; ++q) {
    uint32_t w;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(w) : "h"((uint16_t)(sw >> (16 * q))));
    h[2 * q] = w & 0xffffu;
    h[2 * q + 1] = w >> 16;
  }
#pragma unroll
  for (int b = 0; b < NS; ++b) {
    uint32_t v = h[b];
    if constexpr (std::is_same<T, __nv_bfloat16>::value)
      v = to_bits16<T>(__half2float(__ushort_as_half((unsigned short)v)) * 0x1p104f);
    m[b] = v | (v << 16);
  }
}

// The factor that takes an accumulated product back to x . w: 2^8 for bf16 operands (see
// block_scales), 1 for f16, times the experts' tensor scale.
template <typename T>
constexpr float kMtUnscale = std::is_same<T, __nv_bfloat16>::value ? 256.0f : 1.0f;

// Persistent: CTA c takes the items c, c + gridDim.x, ... (item = token tile t x row block rb,
// numbered t * (N / 128) + rb; the used tiles come first) and runs every ring across them, so
// the next item's copies and conversions overlap this item's MMAs; two TMEM accumulators let the
// epilogue warps drain one item while the MMAs fill the next.
template <typename T, bool SP, int EPI>
__global__ void __launch_bounds__(kMtThreads, 1)
    moe_w4a16_tc_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmS,
                        const __grid_constant__ CUtensorMap tmE, const MoeTcParams p) {
  using G = MtGeom<SP>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int kSlots = G::kSlots, kPairs = kSlots / 2, kDp = kPairs - 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem;                        // [kBoxes][codes 128 x 128 B swizzled | scales 128 x 16 B | meta 128 x 64 B]
  uint8_t* sX = smem + G::kBoxes * G::kBox;  // [kSlots][128 rows x 128 B swizzled]
  // Slots are synchronised in pairs (2q, 2q + 1), so the MMA thread waits and commits once per
  // two stages.  st_full[q]: both stages have their A (4 converter warps each) and their x (8
  // gather warps, once for the pair); st_empty[q]: the MMAs that read the pair have completed.
  // t_full[a]: accumulator a holds a finished item; t_empty[a]: the epilogue has read it.
  __shared__ uint64_t w_full[G::kBoxes], w_empty[G::kBoxes], st_full[kPairs], st_empty[kPairs];
  __shared__ uint64_t t_full[2], t_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ int aborted;
  __shared__ int32_t s_item[kMtMaxItems][3];  // expert, first permutation index, count

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int RB = p.N / kMtRows;
  const int n_items = *p.n_valid * RB;
  int nj = n_items > (int)blockIdx.x ? (n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  nj = nj < kMtMaxItems ? nj : kMtMaxItems;  // the host sizes the grid so that this never cuts
  if (nj == 0) return;  // the whole CTA leaves before any shared state
  const int KB = p.K / kMtBK;  // stages per item (a multiple of kStagesPerBox)
  const int KP = KB / 2;
  auto item_id = [&](int j) { return (int)blockIdx.x + j * (int)gridDim.x; };

  for (int j = tid; j < nj; j += blockDim.x) {
    const int32_t* t = p.tiles + 3 * (int64_t)(item_id(j) / RB);
    s_item[j][0] = t[0];
    s_item[j][1] = t[1];
    s_item[j][2] = t[2];
  }
  if (tid == 0) {
    for (int s = 0; s < G::kBoxes; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], kMtConvWarps);
    }
    for (int q = 0; q < kPairs; ++q) {
      mbar_init(&st_full[q], 2 * 4 + kMtGatherWarps);  // two converter groups, the gather warps once
      mbar_init(&st_empty[q], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&t_full[a], 1);
      mbar_init(&t_empty[a], kMtEpiWarps);
    }
    aborted = 0;
    fence_mbar_init();
  }
  if (warp == kMtWarpMma) tmem_alloc(&tmem_base, kMtCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp < kMtConvWarps) {
    // ---- converters: group g = warp / 4 expands stages g, g + 4, ... of the CTA's stage
    // sequence (all its items, back to back); thread = weight row r (lane quarter warp % 4, the
    // TMEM lanes this warp may access).
    const int g = warp >> 2, qd = warp & 3, r = 32 * qd + lane;
    const uint32_t t_lane = static_cast<uint32_t>(32 * qd) << 16;
    const uint32_t a_base = tmem + t_lane + G::kACol0;
    const uint32_t e_base = tmem + t_lane + G::kMetaCol0;
    // metadata regrouping: this lane's TMEM lane carries rows m (lane msrc) and m + 8 (msrc + 8)
    // of the warp, bytes 2h, 2h + 1 of each 32-wide window
    const int msrc = 16 * (lane >> 4) + (lane & 7);
    const uint32_t msel = ((lane >> 3) & 1) ? 0x7632u : 0x5410u;
    const int n_stages = nj * KB;
#pragma unroll 1
    for (int i = g; i < n_stages; i += kMtGroups) {
      const int m = i / G::kStagesPerBox, st = i % G::kStagesPerBox, bs = m % G::kBoxes;
      if (!__all_sync(0xffffffffu, mbar_wait(&w_full[bs], (m / G::kBoxes) & 1) && !*(volatile int*)&aborted)) {
        aborted = 1;
        break;
      }
      const uint8_t* box = sW + bs * G::kBox;
      uint32_t a[G::kACols];  // column j = stored values 2j, 2j + 1 of the stage
      uint32_t ecol[2] = {0u, 0u};
      if constexpr (!SP) {
        // this stage's 32 code bytes of row r: 16-byte chunks 2st, 2st + 1 of the swizzled row
        const uint4 c0 = *reinterpret_cast<const uint4*>(box + r * 128 + (((2 * st) ^ (r & 7)) << 4));
        const uint4 c1 = *reinterpret_cast<const uint4*>(box + r * 128 + (((2 * st + 1) ^ (r & 7)) << 4));
        const uint32_t sw = *reinterpret_cast<const uint32_t*>(box + kMtCodeBox + r * 16 + 4 * st);
        if (st + kMtGroups >= G::kStagesPerBox) {  // this group's last stage of the box
          __syncwarp();
          if (lane == 0) mbar_arrive(&w_empty[bs]);
        }
        uint32_t sc[4];
        block_scales<T, 4>(sw, sc);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
          e2m1x8_to_16<T>(words[wi], &a[4 * wi]);
#pragma unroll
          for (int pq = 0; pq < 4; ++pq) a[4 * wi + pq] = hmul2u<T>(a[4 * wi + pq], sc[wi >> 1]);
        }
      } else {
        // 32 kept values (16 code bytes: chunk st of the swizzled row), 2 block scales, 8 bytes
        // of metadata (two 32-wide windows of 4 bytes) of row r
        const uint4 c = *reinterpret_cast<const uint4*>(box + r * 128 + ((st ^ (r & 7)) << 4));
        const uint32_t sw = *reinterpret_cast<const uint16_t*>(box + kMtCodeBox + r * 16 + 2 * st);
        const uint2 mw = *reinterpret_cast<const uint2*>(box + kMtCodeBox + kMtScaleBox + r * 64 + 8 * st);
        if (st + kMtGroups >= G::kStagesPerBox) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&w_empty[bs]);
        }
        uint32_t sc[2];
        block_scales<T, 2>(sw, sc);
        const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          e2m1x8_to_16<T>(words[wi], &a[4 * wi]);
#pragma unroll
          for (int pq = 0; pq < 4; ++pq) a[4 * wi + pq] = hmul2u<T>(a[4 * wi + pq], sc[wi >> 1]);
        }
        const uint32_t mwin[2] = {mw.x, mw.y};
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint32_t lo = __shfl_sync(0xffffffffu, mwin[t], msrc);
          const uint32_t hi = __shfl_sync(0xffffffffu, mwin[t], msrc + 8);
          ecol[t] = __byte_perm(lo, hi, msel);
        }
      }
      const int as = i % kSlots;
      if (i >= kSlots &&
          !__all_sync(0xffffffffu, mbar_wait(&st_empty[as >> 1], ((i / kSlots) - 1) & 1))) {  // MMA i - kSlots done
        aborted = 1;
        break;
      }
      tc_fence_after();
      if constexpr (!SP) {
        tmem_st32(a_base + G::kACols * as, a);
      } else {
        tmem_st16_nowait(a_base + G::kACols * as, a);
        tmem_st2_nowait(e_base + 2 * as, ecol[0], ecol[1]);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st_full[as >> 1]);
    }

  }
  else if (warp == kMtWarpMma) {
    if (lane == 0) {
      // ---- MMA issuer over the CTA's stage pairs.  Little scalar work per pair (this thread
      // shares the SM with thirty busy warps, and the tensor pipe idles while it computes): the
      // pair loop is unrolled over the slot pairs, so barriers and descriptor offsets are
      // constants; item bookkeeping happens only at item ends.  The next pair's barrier is
      // tested (without waiting) before this pair's MMAs are issued, so the test overlaps them.
      const uint64_t b_first = desc_kmajor_sw128(smem_u32(sX));
      const uint32_t a_first = tmem + G::kACol0, e_first = tmem + G::kMetaCol0;
      const int NP = nj * KP;
      int P = 0, j = 0, lp = 0;
      uint32_t idesc = idesc_f16(kMtRows, (s_item[0][2] + 15) & ~15, kBf16, SP), d_tmem = tmem;
      bool ready = mbar_wait(&st_full[0], 0);
#pragma unroll 1
      for (int round = 0; P < NP; ++round) {
#pragma unroll
        for (int q = 0; q < kPairs; ++q) {
          if (P < NP) {
            if (!ready) {  // a producer gave up (or a wait ran out): stop issuing
              aborted = 1;
              P = NP;
              break;
            }
            const int qn = (q + 1) % kPairs;
            const uint32_t pn = (uint32_t)(round + (q + 1 == kPairs)) & 1;  // parity of pair P + 1
            const bool next = P + 1 < NP && mbar_test_wait(&st_full[qn], pn);
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int sl = 2 * q + h;
              const uint64_t b0 = b_first + (uint64_t)(sl * (kMtX >> 4));  // descriptor address: 16-byte units
              const uint32_t a0 = a_first + G::kACols * sl;
              if constexpr (!SP) {
#pragma unroll
                for (int k = 0; k < kMtBK / 16; ++k)  // K = 16: 8 A columns, 32 bytes of B
                  umma_f16_tmem_a(d_tmem, a0 + 8 * k, b0 + 2 * k, idesc, (lp | h | k) != 0);
              } else {
#pragma unroll
                for (int t = 0; t < 2; ++t) {  // K = 32 logical: 8 A columns, 64 bytes of B, one metadata column
                  // an odd metadata column is named by the even one below it plus the sparse-id2 field
                  const uint32_t ecl = e_first + 2 * sl + t;
                  umma_f16_sp_tmem_a(d_tmem, a0 + 8 * t, b0 + 4 * t, ecl & ~1u, idesc | (ecl & 1u),
                                     (lp | h | t) != 0);
                }
              }
            }
            umma_commit(&st_empty[q]);
            if (++lp == KP) {  // the item is done: hand its accumulator over, set up the next one
              umma_commit(&t_full[j & 1]);
              lp = 0;
              if (++j < nj) {
                d_tmem = tmem + kMtAccCols * (j & 1);
                idesc = idesc_f16(kMtRows, (s_item[j][2] + 15) & ~15, kBf16, SP);
                if (j >= 2 && !mbar_wait(&t_empty[j & 1], ((j >> 1) - 1) & 1)) ready = false;
              }
            }
            if (ready) ready = P + 1 >= NP || next || mbar_wait(&st_full[qn], pn);
            ++P;
          }
        }
      }
      if (aborted) {  // let the epilogue warps through (their results are void)
        umma_commit(&t_full[0]);
        umma_commit(&t_full[1]);
      }
    }
  } else if (warp >= kMtWarpEpi0) {
    // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (weight rows) of the item's
    // accumulator, 32 columns (routed rows) at a time, and stores each routed row's 32 outputs
    // with one store; then it hands the accumulator back.
    const int qd = warp & 3;
    const uint32_t t_lane = static_cast<uint32_t>(32 * qd) << 16;
    const float scale = kMtUnscale<T> * *p.w_ts;
#pragma unroll 1
    for (int j = 0; j < nj; ++j) {
      const int acc = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&t_full[acc], (j >> 1) & 1) && !*(volatile int*)&aborted)) {
        aborted = 1;
        break;
      }
      tc_fence_after();
      const int first = s_item[j][1], count = s_item[j][2];
      const int rb = item_id(j) % RB;
      const int orow = rb * kMtRows + 32 * qd + lane;
#pragma unroll 1
      for (int c = 0; 32 * c < count; ++c) {
        float v[32];
        tmem_ld32(tmem + t_lane + kMtAccCols * acc + 32 * c, v);
        if constexpr (EPI == kEpiStore) {
#pragma unroll
          for (int ii = 0; ii < 32; ++ii) {
            const int i = 32 * c + ii;
            if (i < count) p.y[(int64_t)p.perm[first + i] * p.N + orow] = v[ii] * scale;
          }
        } else {
          // gate / up packed in 16-row blocks: lanes 0-15 of this quarter hold gate rows of
          // features f0 .. f0 + 15, lanes 16-31 the up rows of the same features.  Lanes 0-15
          // evaluate even tokens, lanes 16-31 odd ones (one exchange per token pair: each half
          // sends what the other half lacks)
          const int64_t f = (int64_t)rb * (kMtRows / 2) + 16 * qd + (lane & 15);
          const int64_t F = p.N / 2;
          const bool lo = lane < 16;
#pragma unroll
          for (int ii = 0; ii < 32; ii += 2) {
            const float a = v[ii] * scale, b = v[ii + 1] * scale;
            const float got = __shfl_xor_sync(0xffffffffu, lo ? b : a, 16);
            const int i = 32 * c + ii + (lo ? 0 : 1);
            const float hv = lo ? swiglu(a, got) : swiglu(got, b);  // (gate, up) of token i
            if (i < count) p.h[(int64_t)(first + i) * F + f] = to_bits16<T>(hv);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[acc]);
    }
  } else if (warp == kMtWarpW) {
    if (lane == 0) {
      // ---- weight boxes: codes, block scales (and metadata) of kStagesPerBox stages per copy set
      const int BPI = KB / G::kStagesPerBox, NB = nj * BPI;
      int issued = 0;
#pragma unroll 1
      for (int b = 0; b < NB; ++b) {
        const int j = b / BPI, mb = b - j * BPI, s = b % G::kBoxes;
        const int row0 = s_item[j][0] * p.N + (item_id(j) % RB) * kMtRows;  // stacked weight row (< 2^31)
        if (!mbar_wait(&w_empty[s], ((b / G::kBoxes) & 1) ^ 1) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
        uint8_t* box = sW + s * G::kBox;
        mbar_arrive_expect_tx(&w_full[s], G::kBox);
        tma_load_2d(box, &tmC, &w_full[s], mb * 128, row0);
        tma_load_2d(box + kMtCodeBox, &tmS, &w_full[s], mb * 16, row0);
        if constexpr (SP) tma_load_2d(box + kMtCodeBox + kMtScaleBox, &tmE, &w_full[s], mb * 64, row0);
        ++issued;
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int b = issued - G::kBoxes > 0 ? issued - G::kBoxes : 0; b < issued; ++b)
        mbar_wait(&w_full[b % G::kBoxes], (b / G::kBoxes) & 1);
    }
  } else {
    // ---- token rows: gather thread t copies 16-byte chunk t % 8 of routed rows t / 8 + 32u
    // (u = 0 .. 3) of each stage, kDp stage pairs ahead (rows count .. n_mma - 1 zero-filled)
    const int t = tid - 32 * kMtWarpX0, j8 = t & 7;
    const uint16_t* xrow[4];
    uint32_t xoff[4], xbytes[4];
    int nx = 0, cur_j = -1;
#pragma unroll
    for (int u = 0; u < 4; ++u) xoff[u] = sw128((t >> 3) + 32 * u, j8);
    auto issue_pair = [&](int P) {
      const int j = P / KP, lp = P - j * KP;
      if (j != cur_j) {  // a new item: its routed rows' token addresses
        cur_j = j;
        const int first = s_item[j][1], count = s_item[j][2], n_mma = (count + 15) & ~15;
        nx = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = (t >> 3) + 32 * u;
          xbytes[u] = i < count ? 16u : 0u;
          const int64_t xr = p.x_direct ? (int64_t)(first + i) : (int64_t)(p.perm[first + i] / p.topk);
          xrow[u] = p.x + (i < count ? xr * p.K : 0) + 8 * j8;
          nx += i < n_mma;
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint8_t* b = sX + ((2 * P + h) % kSlots) * kMtX;
        const int64_t kofs = (int64_t)(2 * lp + h) * kMtBK;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (u < nx) cp_async16_zfill(b + xoff[u], xrow[u] + kofs, xbytes[u]);
      }
    };
    const int NP = nj * KP;
    for (int pp = 0; pp < kDp; ++pp) {  // the first pairs: their slots are fresh
      if (pp < NP) issue_pair(pp);
      cp_async_commit();
    }
#pragma unroll 1
    for (int P = 0; P < NP; ++P) {
      cp_async_wait<kDp - 1>();  // this thread's chunks of stage pair P have landed
      fence_proxy_async_smem();  // ... and are visible to the MMA's operand reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&st_full[P % kPairs]);
      const int Pn = P + kDp;
      if (Pn < NP) {
        if (Pn >= kPairs) {  // the slot pair's previous pair Pn - kPairs = P - 2 is multiplied
          const bool ok = mbar_wait(&st_empty[Pn % kPairs], ((Pn / kPairs) - 1) & 1) && !*(volatile int*)&aborted;
          if (!__all_sync(0xffffffffu, ok)) {
            aborted = 1;
            break;
          }
        }
        issue_pair(Pn);
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

template <typename T, bool SP, int EPI>
int launch_moe_tc(const CUtensorMap& tmC, const CUtensorMap& tmS, const CUtensorMap& tmE, const MoeTcParams& p,
                  int64_t n_items_max, cudaStream_t s) {
  auto kern = moe_w4a16_tc_kernel<T, SP, EPI>;
  const size_t smem = MtGeom<SP>::kSmem;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  // one CTA per SM, or more when the items would not fit kMtMaxItems per CTA
  int64_t grid = sm_count();
  if ((n_items_max + kMtMaxItems - 1) / kMtMaxItems > grid) grid = (n_items_max + kMtMaxItems - 1) / kMtMaxItems;
  if (grid > n_items_max) grid = n_items_max;
  if (grid > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  kern<<<(unsigned)grid, kMtThreads, smem, s>>>(tmC, tmS, tmE, p);
  return launch_status();
}

template <int EPI>
int launch_moe_tc_any(bool sparse, int t16, const CUtensorMap& tmC, const CUtensorMap& tmS, const CUtensorMap& tmE,
                      const MoeTcParams& p, int64_t n_items_max, cudaStream_t s) {
  if (sparse)
    return t16 == SP24_F16 ? launch_moe_tc<__half, true, EPI>(tmC, tmS, tmE, p, n_items_max, s)
                           : launch_moe_tc<__nv_bfloat16, true, EPI>(tmC, tmS, tmE, p, n_items_max, s);
  return t16 == SP24_F16 ? launch_moe_tc<__half, false, EPI>(tmC, tmS, tmE, p, n_items_max, s)
                         : launch_moe_tc<__nv_bfloat16, false, EPI>(tmC, tmS, tmE, p, n_items_max, s);
}

}  // namespace

bool moe_tc_supported(int wf, int x_fmt, int64_t T, int64_t E, int64_t N, int64_t K, int64_t max_tiles,
                      const void* codes, const void* scales, const void* meta, const void* x) {
  const bool sp = wf == W_SQ4;
  if (!(wf == W_DQ4 || sp) || x_fmt != X_16) return false;
  const int64_t box_k = sp ? MtGeom<true>::kBoxK : MtGeom<false>::kBoxK;
  return T > 0 && T < INT32_MAX && N > 0 && N % kMtRows == 0 && K > 0 && K % box_k == 0 && K <= INT32_MAX / 2 &&
         E * N <= INT32_MAX && max_tiles * (N / kMtRows) <= INT32_MAX && aligned(codes, 16) && aligned(scales, 16) &&
         (!sp || aligned(meta, 16)) && aligned(x, 16);
}

namespace {

// Tensor maps of a stacked weight operand (dense NVFP4 codes + scales, or 2:4 values + scales +
// nibbles) with `rows` rows of K logical entries.
int weight_maps(bool sparse, const uint8_t* codes, const uint8_t* scales, const uint8_t* meta, uint64_t rows,
                uint64_t K, CUtensorMap* tmC, CUtensorMap* tmS, CUtensorMap* tmE) {
  // per row: codes K/2 (dense) or K/4 (2:4) bytes, scales K/16 or K/32, metadata K/8 (2:4)
  const uint64_t cb = sparse ? K / 4 : K / 2, sb = sparse ? K / 32 : K / 16;
  int st = make_tmap_2d(tmC, codes, 1, rows, cb, cb, 128, kMtRows);  // 128-byte swizzle
  if (!st) st = make_tmap_2d_plain(tmS, scales, rows, sb, sb, 16, kMtRows);
  if (!st) st = sparse ? make_tmap_2d_plain(tmE, meta, rows, K / 8, K / 8, 64, kMtRows) : SP24_OK;
  if (!st && !sparse) *tmE = *tmS;  // unused
  return st;
}

}  // namespace

int moe_tc_grouped(int wf, int t16, const SkinnyParams& sp, int64_t E, int64_t T, int64_t n_tiles,
                   const int32_t* n_valid, cudaStream_t s) {
  if (n_tiles <= 0) return SP24_OK;
  const bool sparse = wf == W_SQ4;
  MoeTcParams p{};
  p.x = reinterpret_cast<const uint16_t*>(sp.x);
  p.w_ts = sp.w_ts;
  p.tiles = sp.tiles;
  p.perm = sp.perm;
  p.n_valid = n_valid;
  p.y = sp.y;
  p.topk = sp.topk;
  p.T = (int)T;
  p.N = (int)sp.N;
  p.K = (int)sp.K;
  CUtensorMap tmC, tmS, tmE;
  const int st = weight_maps(sparse, sp.w, sp.w_scales, sp.meta, (uint64_t)(E * sp.N), (uint64_t)sp.K, &tmC, &tmS, &tmE);
  if (st) return st;
  return launch_moe_tc_any<kEpiStore>(sparse, t16, tmC, tmS, tmE, p, n_tiles * (sp.N / kMtRows), s);
}

int moe_tc_block_gemm(int epi, int wf, int t16, const MoeBlockGemm& g, cudaStream_t s) {
  if (g.n_tiles <= 0) return SP24_OK;
  const bool sparse = wf == W_SQ4;
  MoeTcParams p{};
  p.x = g.x;
  p.w_ts = g.w_ts;
  p.tiles = g.tiles;
  p.perm = g.perm;
  p.n_valid = g.n_valid;
  p.y = g.y;
  p.h = g.h;
  p.x_direct = g.x_direct;
  p.topk = g.topk;
  p.T = (int)g.T;
  p.N = (int)g.N;
  p.K = (int)g.K;
  CUtensorMap tmC, tmS, tmE;
  const int st = weight_maps(sparse, g.codes, g.scales, g.meta, (uint64_t)(g.E * g.N), (uint64_t)g.K, &tmC, &tmS, &tmE);
  if (st) return st;
  const int64_t items = g.n_tiles * (g.N / kMtRows);
  if (epi == kEpiGlu) return launch_moe_tc_any<kEpiGlu>(sparse, t16, tmC, tmS, tmE, p, items, s);
  if (epi == kEpiStore) return launch_moe_tc_any<kEpiStore>(sparse, t16, tmC, tmS, tmE, p, items, s);
  return SP24_ERR_INVALID_ARG;
}

}  // namespace sp24
