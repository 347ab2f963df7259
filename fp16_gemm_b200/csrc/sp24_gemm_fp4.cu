// a4 at prefill-sized M for W4A4 (NVFP4 x NVFP4): a persistent tensor-core GEMM in which the
// two CTAs of a cluster work as one pair on 256 weight rows at a time (tcgen05 cta_group::2).
//
// [P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went", "The ladder, top to
// bottom": the dense NVFP4 GEMM at 4096 cubed is the kernel ceiling the pages measure; past the
// ridge of "The roofline is the whole argument" the product is bound by the tensor pipe, so the
// design goal is to keep that pipe busy:
//   * operand bytes per FLOP: the pair's MMA is M = 256 (128 weight rows from each CTA) by
//     N = BN tokens, and each CTA loads only half of the tokens' B tile (the pair's tensor cores
//     share their B halves), so an SM brings in 128 weight rows + BN/2 token rows per K step for
//     128 x BN outputs;
//   * operands arrive as tile images (sp24_nvfp4_to_mma): codes already in the 128-byte
//     swizzled shared-memory order, one TMA box of eight 2 KB rows per 16 KB tile (boxes of
//     128-byte rows cost the TMA unit one request per row and capped an SM near 48 GB/s), block
//     scales already in the 128-row x 4-scale order that tcgen05.cp moves into TMEM;
//   * scale copies off the MMA thread: a tcgen05 instruction costs its issuing thread tens of
//     nanoseconds, and the twelve scale copies of a 256-K stage (4 SFA + 8 SFB tiles) issued by
//     the MMA thread took longer than the stage's four MMAs (measured: 0.80 us per stage against
//     0.42 us without copies); two warps issue them, six each, into two TMEM slots that
//     alternate between stages (0.51 us per stage);
//   * persistent: one CTA per SM, tiles assigned round-robin to the pairs; two TMEM
//     accumulators, so a tile's epilogue (TMEM -> registers -> shared memory -> TMA store of
//     32-token x 128-row fp32 boxes, marked evict-first in L2) overlaps the next tile's main loop.  For BN = 256 the two
//     accumulators overlap in 96 columns (0-255 and 160-415, scale slots in 416-511): the
//     epilogue reads the shared columns first and releases the accumulator, then drains the rest
//     while the next tile's MMAs run.
//
// Warp roles (256 threads per CTA): warp 0 = TMA producer (one lane; both CTAs load their own
// halves and count the bytes on the even CTA's barrier); warp 1 = TMEM allocation (both CTAs)
// and, in the even CTA, the MMA issuer (one lane); warps 2-5 = epilogue (TMEM lane quarter =
// warp % 4), each thread one weight row; warps 6-7 = scale copies (even CTA, one lane each).
// Every wait is bounded: when one runs out the kernel records SP24_ERR_DEVICE_TIMEOUT and
// unwinds.  No TMA load uses cluster multicast.
#include <cudaTypedefs.h>
#include <string.h>

#include "sp24_tc.cuh"

namespace sp24 {

// ------------------------------------------------------------------ operand images
//
// The W4A4 kernel reads each operand as whole 128-row tiles, stored in global memory exactly as
// the tensor cores want them in shared memory, so one TMA box of a few long rows moves a tile
// (a box of 128-byte rows costs the TMA unit one request per row, which at 256 rows per stage
// caps an SM near 48 GB/s):
//   codes: for each 128-row block rb and 256-K chunk kc a 16 KB tile at byte
//          16384 (rb * K/256 + kc): row r at 128 r, its 16-byte piece c at 16 (c ^ (r % 8))
//          (the 128-byte swizzle of a K-major operand, rows 128 bytes apart);
//   scales: for each 128-row block rb and 64-K chunk kc a 512-byte tile at byte
//          512 (rb * K/64 + kc), row r's four E4M3 scales of the chunk at 16 (r % 32) + 4 (r / 32)
//          (the 128-row x 4-scale tile that tcgen05.cp moves into TMEM).
// Rows are padded to a multiple of 128 with zero codes and zero scales.

namespace {

struct ImageJob {
  const uint4* codes;        // [rows, K/2] bytes as 16-byte pieces (K = FP4 entries per row)
  const uint32_t* scales;    // [rows, K/16] (sw = 4) or [rows, K/32] (sw = 2) bytes, as words
  const uint4* meta;         // pairwise-4:8 nibbles [rows, K/8] bytes (K stored = K/8 bytes), or null
  uint4* codes_out;
  uint32_t* scales_out;
  uint4* meta_out;
  int rows, K, sw, tiles;    // sw: scale words per row per 256-entry tile; tiles = row blocks x K/256
};

// One CTA per code tile (128 rows x 256 entries): its 16 KB of codes (8 threads per 128-byte row
// segment, reads coalesced, each 128-byte row written whole), the scale tiles of the same rows
// and range (sw of them) and, for a pairwise-4:8 weight, its two 2 KB metadata tiles (row r's
// 16 bytes at 16 r; padding rows get 0x44, the legal index pair 0, 1).  Row blocks past `rows`
// are padding.  Up to two operands per launch (job b may be empty).
__global__ void __launch_bounds__(256) to_mma_kernel(ImageJob ja, ImageJob jb) {
  int t = blockIdx.x;
  const bool second = t >= ja.tiles;
  const ImageJob& j = second ? jb : ja;
  if (second) t -= ja.tiles;
  const int kc256 = j.K / 256, rb = t / kc256, kc = t - rb * kc256;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < 1024; i += 256) {
    const int rr = i >> 3, c = i & 7, r = rb * 128 + rr;
    const uint4 v = r < j.rows ? j.codes[(int64_t)r * (j.K / 32) + kc * 8 + c] : zero;
    j.codes_out[(int64_t)t * 1024 + rr * 8 + (c ^ (rr & 7))] = v;
  }
  const int spr = kc256 * j.sw;  // scale words per row
  for (int i = threadIdx.x; i < 128 * j.sw; i += 256) {
    const int rr = i / j.sw, w = i - rr * j.sw, r = rb * 128 + rr;
    const uint32_t v = r < j.rows ? j.scales[(int64_t)r * spr + kc * j.sw + w] : 0u;
    j.scales_out[((int64_t)rb * spr + kc * j.sw + w) * 128 + 4 * (rr & 31) + (rr >> 5)] = v;
  }
  if (j.meta) {  // K entries stored = 2K logical; K/8 meta bytes per row, 32 per code tile
    const int rr = threadIdx.x >> 1, h = threadIdx.x & 1, r = rb * 128 + rr;
    const uint4 v = r < j.rows ? j.meta[(int64_t)r * (j.K / 128) + kc * 2 + h]
                               : make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    j.meta_out[((int64_t)rb * kc256 * 2 + kc * 2 + h) * 128 + rr] = v;
  }
}

ImageJob image_job(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, uint8_t* codes_out,
                   uint8_t* scales_out, int sw = 4, int64_t row_blocks = -1, const uint8_t* meta = nullptr,
                   uint8_t* meta_out = nullptr) {
  ImageJob j;
  j.codes = reinterpret_cast<const uint4*>(codes);
  j.scales = reinterpret_cast<const uint32_t*>(scales);
  j.meta = reinterpret_cast<const uint4*>(meta);
  j.codes_out = reinterpret_cast<uint4*>(codes_out);
  j.scales_out = reinterpret_cast<uint32_t*>(scales_out);
  j.meta_out = reinterpret_cast<uint4*>(meta_out);
  j.rows = (int)rows;
  j.K = (int)K;
  j.sw = sw;
  j.tiles = (int)((row_blocks >= 0 ? row_blocks : (rows + 127) / 128) * (K / 256));
  return j;
}

}  // namespace

int64_t nvfp4_mma_codes_bytes(int64_t rows, int64_t K) { return (rows + 127) / 128 * 128 * (K / 2); }
int64_t nvfp4_mma_scales_bytes(int64_t rows, int64_t K) { return (rows + 127) / 128 * 128 * (K / 16); }

// Tile images of one or two NVFP4 operands (rows1 == 0: only the first), one launch.
int nvfp4_to_mma2(const uint8_t* c0, const uint8_t* s0, int64_t rows0, uint8_t* co0, uint8_t* so0,
                  const uint8_t* c1, const uint8_t* s1, int64_t rows1, uint8_t* co1, uint8_t* so1, int64_t K,
                  cudaStream_t s) {
  if (K % 256 || rows0 > INT32_MAX || rows1 > INT32_MAX || K > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  const ImageJob ja = image_job(c0, s0, rows0, K, co0, so0);
  const ImageJob jb = image_job(c1, s1, rows1, K, co1, so1);
  const int64_t blocks = (int64_t)ja.tiles + jb.tiles;
  if (blocks == 0) return SP24_OK;
  if (blocks > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  to_mma_kernel<<<(unsigned)blocks, 256, 0, s>>>(ja, jb);
  return launch_status();
}

int nvfp4_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, uint8_t* codes_out,
                 uint8_t* scales_out, cudaStream_t s) {
  return nvfp4_to_mma2(codes, scales, rows, codes_out, scales_out, nullptr, nullptr, 0, nullptr, nullptr, K, s);
}

// Images for the sparse FP4 pair kernel: activations with one scale per 32 K (scale tiles of
// 128 K), and a pairwise-4:8 weight (kept values [rows, K/2] as codes with one scale per 16
// stored, metadata tiles), rows padded to whole 256-row pair tiles.
int64_t b32_mma_scales_bytes(int64_t rows, int64_t K) { return (rows + 127) / 128 * 128 * (K / 32); }
int64_t sp48_rows_padded(int64_t rows) { return (rows + 255) / 256 * 256; }
int64_t sp48_mma_values_bytes(int64_t rows, int64_t K) { return sp48_rows_padded(rows) * (K / 4); }
int64_t sp48_mma_scales_bytes(int64_t rows, int64_t K) { return sp48_rows_padded(rows) * (K / 32); }
int64_t sp48_mma_meta_bytes(int64_t rows, int64_t K) { return sp48_rows_padded(rows) * (K / 16); }

int nvfp4_b32_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, uint8_t* codes_out,
                     uint8_t* scales_out, cudaStream_t s) {
  if (K % 256 || rows > INT32_MAX || K > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  const ImageJob j = image_job(codes, scales, rows, K, codes_out, scales_out, 2);
  if (j.tiles == 0) return SP24_OK;
  to_mma_kernel<<<(unsigned)j.tiles, 256, 0, s>>>(j, image_job(nullptr, nullptr, 0, 256, nullptr, nullptr));
  return launch_status();
}

int sp48_to_mma(const uint8_t* values, const uint8_t* scales, const uint8_t* meta, int64_t rows, int64_t K,
                uint8_t* values_out, uint8_t* scales_out, uint8_t* meta_out, cudaStream_t s) {
  if (K % 512 || rows > INT32_MAX || K > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  const ImageJob j = image_job(values, scales, rows, K / 2, values_out, scales_out, 4, sp48_rows_padded(rows) / 128,
                               meta, meta_out);
  if (j.tiles == 0) return SP24_OK;
  to_mma_kernel<<<(unsigned)j.tiles, 256, 0, s>>>(j, image_job(nullptr, nullptr, 0, 256, nullptr, nullptr));
  return launch_status();
}

// ------------------------------------------------------------------ the pair GEMM

namespace {

using namespace tc;

// SP: the pairwise-4:8 sparse FP4 MMA (tcgen05.mma.sp kind::mxf4nvf4, K = 128 logical per
// instruction): a stage is 512 logical K (A 256 stored codes per row, B two 256-entry tiles),
// plus two 2 KB metadata tiles per CTA; dense: a stage is 256 K.
template <int BN, bool SP = false>
struct PairCfg {
  static constexpr uint32_t A = 16384;                 // 128 weight rows x 256 FP4: one tile
  static constexpr uint32_t B = (SP ? 2 : 1) * (BN / 2) * 128;  // this CTA's half of the tokens
  static constexpr uint32_t SFA = 2048;                // 4 scale tiles (128 rows x 4 scales)
  static constexpr uint32_t SFB = (BN / 128) * 2048;   // all BN tokens' scale tiles
  static constexpr uint32_t META = SP ? 4096 : 0;      // two metadata tiles (128 rows x 16 bytes)
  static constexpr uint32_t STAGE = A + B + SFA + SFB + META;
  static constexpr int S = SP ? (BN == 256 ? 3 : 4) : (BN == 256 ? 5 : 6);
  static constexpr uint32_t EPI = 32 * 128 * 4;        // one 32-token x 128-row fp32 chunk
  static constexpr size_t SMEM = (size_t)S * STAGE + 2 * EPI + 1024;
  static constexpr int KSTAGE = SP ? 512 : 256;        // logical K per stage
  // TMEM columns: two accumulators (overlapping at BN = 256), then two stages of scale factors
  // (per MMA: SFA 4 columns + SFB BN/32; SP: then 8 metadata columns), so the copies for stage
  // i + 1 run while the MMAs of stage i read theirs
  static constexpr uint32_t ACC1 = BN == 256 ? (SP ? 128 : 160) : BN;
  static constexpr uint32_t SF = ACC1 + BN;
  static constexpr uint32_t SLOT = 4 + BN / 32;     // one MMA's scale columns
  static constexpr uint32_t META_COL = 4 * SLOT;    // SP: metadata columns after the scales
  static constexpr uint32_t SF_STAGE = 4 * SLOT + (SP ? 8 : 0);
  static constexpr uint32_t COLS = 512;
  static constexpr int CHUNKS = BN / 32;
  static constexpr int OVERLAP_CHUNKS = BN == 256 ? (int)((256 - ACC1) / 32) : 0;
  static constexpr int EARLY = OVERLAP_CHUNKS > 3 ? OVERLAP_CHUNKS : 3;  // chunks read before the release
  static_assert(STAGE % 1024 == 0 && SMEM <= 232448, "shared memory layout");
  static_assert(SF + 2 * SF_STAGE <= COLS, "TMEM columns");
  static_assert(EARLY <= CHUNKS, "epilogue buffers");
};

struct PairParams {
  int M, N, K;          // M tokens, N weight rows
  float* y;             // [M, N] fp32
  const float* ts_w;    // tensor scales (device)
  const float* ts_x;
  int tiles_w, tiles_n; // weight tiles of 256 rows, token tiles of BN
  uint64_t wait_ns;
};

// TMA_Y: the epilogue stages each 32-token chunk in shared memory and writes it with one TMA
// store (needs N % 4 == 0 and a 16-byte aligned y); otherwise each warp stores its rows directly.
template <int BN, bool TMA_Y, bool SP>
__global__ void __launch_bounds__(256, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                           const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                           const PairParams p) {
  using C = PairCfg<BN, SP>;
  constexpr int S = C::S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = tc::align1024(smem_raw);
  auto sA = [&](int s) { return smem + s * C::STAGE; };
  auto sB = [&](int s) { return sA(s) + C::A; };
  auto sSA = [&](int s) { return sB(s) + C::B; };
  auto sSB = [&](int s) { return sSA(s) + C::SFA; };
  auto sE = [&](int s) { return sSB(s) + C::SFB; };  // SP: metadata tiles
  float* sY = reinterpret_cast<float*>(smem + S * C::STAGE);  // two epilogue chunks
  __shared__ uint64_t full_bar[S], empty_bar[S], sf_bar[2 * S], tfull_bar, tempty_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int aborted;
  __shared__ int epi_ok[4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)cluster_id_x(), pairs = (int)cluster_count_x();
  const int KB = p.K / C::KSTAGE;
  const int tiles = p.tiles_w * p.tiles_n;
  const uint64_t wait_ns = p.wait_ns ? p.wait_ns : wait_limit();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_bar[s], 1);
      mbar_init(&sf_bar[S + s], 1);
    }
    mbar_init(&tfull_bar, 1);
    mbar_init(&tempty_bar, 8);  // 4 epilogue warps in each CTA
    aborted = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSA);
    prefetch_tmap(&tmSB);
    if (TMA_Y) prefetch_tmap(&tmY);
    if (SP) prefetch_tmap(&tmE);
  }
  if (warp == 1) tmem_alloc_pair(&tmem_base, C::COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or commit names them
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(smem_u32(&full_bar[0]), 0);  // the even CTA's ring
      int it = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += pairs) {
        const int wb = (t % p.tiles_w) * 2 + (int)rank;   // this CTA's 128-row weight block
        const int n0 = (t / p.tiles_w) * BN;               // the pair's first token
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait_for(&empty_bar[s], ph ^ 1, wait_ns) || *(volatile int*)&aborted) {
            aborted = 1;
            ok = false;
            break;
          }
          const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
          if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * C::STAGE);
          // code tiles: 8 rows of 2 KB each; a 64-token half tile is 4 of them.  SP: A holds the
          // kept values (K/2 stored per row, one tile per stage), B two consecutive tiles
          constexpr int TB = SP ? 2 : 1;          // token tiles per stage
          const int kcx = p.K / 256;              // token tiles per row block
          tma_load_2d_pair(sA(s), &tmA, fb, 0, (wb * KB + kb) * 8);
          if (BN == 256) {
            tma_load_2d_pair(sB(s), &tmB, fb, 0, ((n0 / 128 + (int)rank) * kcx + TB * kb) * 8);
          } else {
#pragma unroll
            for (int u = 0; u < TB; ++u)
              tma_load_2d_pair(sB(s) + u * (BN / 2) * 128, &tmB, fb, 0,
                               ((n0 / 128) * kcx + TB * kb + u) * 8 + 4 * (int)rank);
          }
          // four scale tiles per stage (dense: 64 K each; SP: 128 logical K each)
          const int kst = p.K / (SP ? 128 : 64);  // scale tiles per row block
          tma_load_2d_pair(sSA(s), &tmSA, fb, 0, wb * kst + kb * 4);
#pragma unroll
          for (int g = 0; g < BN / 128; ++g)
            tma_load_2d_pair(sSB(s) + 2048 * g, &tmSB, fb, 0, (n0 / 128 + g) * kst + kb * 4);
          if (SP) tma_load_2d_pair(sE(s), &tmE, fb, 0, wb * (p.K / 256) + kb * 2);  // 2 metadata tiles
        }
      }
      // the even CTA's producer armed every stage it counted: wait (bounded) until those copies
      // (its own and the odd CTA's) have landed before the pair may exit
      if (leader)
        for (int i = it - S > 0 ? it - S : 0; i < it; ++i) mbar_wait_for(&full_bar[i % S], (i / S) & 1, wait_ns);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_nvfp4(256, BN, SP);
      int it = 0, j = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += pairs, ++j) {
        const uint32_t d = tmem + ((j & 1) ? C::ACC1 : 0u);
        if (j >= 1 && !mbar_wait_cluster(&tempty_bar, (j - 1) & 1, wait_ns)) {
          aborted = 1;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait_for(&full_bar[s], ph, wait_ns) || *(volatile int*)&aborted) {
            aborted = 1;
            ok = false;
            break;
          }
          const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA(s)));
          const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB(s)));
          const uint32_t sf0 = tmem + C::SF + (uint32_t)(it & 1) * C::SF_STAGE;
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // the scale copies of MMAs 2h, 2h + 1 (warp 6 + h)
            if (!mbar_wait_for(&sf_bar[h * S + s], ph, wait_ns)) {
              aborted = 1;
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int q = 2 * h; q < 2 * h + 2; ++q) {
              if (SP)  // A: 64 stored = 32 bytes; B: 128 entries = 64 bytes of token tile q / 2
                umma_nvfp4_sp_pair(d, a0 + 2 * q, b0 + (uint64_t)((q >> 1) * (BN / 2) * 128 / 16) + 4 * (q & 1),
                                   sf0 + C::META_COL + 2 * q, idesc, sf0 + C::SLOT * q, sf0 + C::SLOT * q + 4,
                                   (kb | q) != 0);
              else  // K = 64 codes = 32 bytes = 2 descriptor units
                umma_nvfp4_pair(d, a0 + 2 * q, b0 + 2 * q, idesc, sf0 + C::SLOT * q, sf0 + C::SLOT * q + 4,
                                (kb | q) != 0);
            }
          }
          if (!ok) break;
          umma_commit_pair(&empty_bar[s], 0x3);
        }
        if (ok) umma_commit_pair(&tfull_bar, 0x3);
      }
    }
  } else if (warp >= 6) {
    // scale-factor copies (smem -> TMEM) for MMAs 2h and 2h + 1 of every stage, issued apart
    // from the MMA thread so that neither stream of tcgen05 instructions waits for the other;
    // a stage's columns alternate between two slots, reused once the MMAs of two stages back
    // have completed
    if (leader && lane == 0) {
      const int h = warp - 6;
      int it = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += pairs) {
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          const int prev = it - 2;  // the stage whose MMAs last read this slot
          if (!mbar_wait_for(&full_bar[s], ph, wait_ns) ||
              (prev >= 0 && !mbar_wait_for(&empty_bar[prev % S], (prev / S) & 1, wait_ns)) ||
              *(volatile int*)&aborted) {
            aborted = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf0 = tmem + C::SF + (uint32_t)(it & 1) * C::SF_STAGE;
#pragma unroll
          for (int q = 2 * h; q < 2 * h + 2; ++q) {
            tmem_cp_32x128b_x4_pair(sf0 + C::SLOT * q, desc_rows16_noswizzle(smem_u32(sSA(s) + 512 * q)));
#pragma unroll
            for (int g = 0; g < BN / 128; ++g)
              tmem_cp_32x128b_x4_pair(sf0 + C::SLOT * q + 4 + 4 * g,
                                      desc_rows16_noswizzle(smem_u32(sSB(s) + 2048 * g + 512 * q)));
          }
          // SP: metadata tile h (256 logical K, MMAs 2h and 2h + 1) -> row m on lane m, 4 columns
          if (SP) tmem_cp_128x128b_pair(sf0 + C::META_COL + 4 * h, desc_rows16_noswizzle(smem_u32(sE(s) + 2048 * h)));
          umma_commit_pair(&sf_bar[h * S + s], 0x1);
        }
      }
    }
  } else {
    // epilogue: thread = one weight row of this CTA, 32 tokens per TMEM load
    const int q = warp & 3;
    const bool epi_leader = warp == 2 && lane == 0;
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty_bar), 0);
    const float scale = __fmul_rn(*p.ts_w, *p.ts_x);
    const uint64_t y_policy = l2_evict_first_policy();
    int j = 0, chunk = 0;
    for (int t = pair; t < tiles; t += pairs, ++j) {
      const int row0 = (t % p.tiles_w) * 256 + (int)rank * 128;
      const int row = row0 + 32 * q + lane;
      const int n0 = (t / p.tiles_w) * BN;
      // the four epilogue warps agree on the outcome of the wait, so that none of them leaves
      // while the others wait for it at a named barrier
      const bool got = mbar_wait_for(&tfull_bar, j & 1, wait_ns);
      if (lane == 0) epi_ok[q] = got;
      named_bar_sync(1, 128);
      const bool all = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3];
      named_bar_sync(1, 128);
      if (!all) {
        aborted = 1;
        break;
      }
      tc_fence_after();
      const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16) + ((j & 1) ? C::ACC1 : 0u);
      // chunk order: the columns shared with the other accumulator first (BN = 256: the last two
      // chunks of accumulator 0, the first two of accumulator 1)
      auto chunk_at = [&](int i) {
        if (BN == 256 && !(j & 1)) return (i + C::CHUNKS - C::OVERLAP_CHUNKS) % C::CHUNKS;
        return i;
      };
      // the chunks shared with the other accumulator are read first (three buffers in flight),
      // then the accumulator is released to the next tile's MMAs
      uint32_t r[3][32];
#pragma unroll
      for (int i = 0; i < 3; ++i) tmem_ld32_async(base + 32 * chunk_at(i), r[i]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader);
#pragma unroll
      for (int i = 0; i < C::CHUNKS; ++i) {
        if (i >= 3) tmem_wait_ld();
        const int c = chunk_at(i);
        const uint32_t(&v)[32] = r[i % 3];
        if (TMA_Y) {
          float* st = sY + (chunk & 1) * (32 * 128);
          if (epi_leader) bulk_wait_read<1>();  // the store that last read this buffer is done
          named_bar_sync(1, 128);
#pragma unroll
          for (int k = 0; k < 32; ++k) st[k * 128 + 32 * q + lane] = __uint_as_float(v[k]) * scale;
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (epi_leader && row0 < p.N && n0 + 32 * c < p.M) {  // boxes wholly outside Y are skipped
            tma_store_2d_evict_first(&tmY, st, row0, n0 + 32 * c, y_policy);
            bulk_commit();
          }
          ++chunk;
        } else if (row < p.N) {
          float* yp = p.y + (int64_t)(n0 + 32 * c) * p.N + row;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (n0 + 32 * c + k < p.M) yp[(int64_t)k * p.N] = __uint_as_float(v[k]) * scale;
        }
        if (i + 3 < C::CHUNKS) tmem_ld32_async(base + 32 * chunk_at(i + 3), r[i % 3]);
      }
    }
    if (TMA_Y && epi_leader) bulk_wait<0>();  // every output written before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA frees TMEM or exits while the pair's MMAs may run
  if (threadIdx.x == 0 && aborted) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::COLS);
  }
}

}  // namespace

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

int tmap_encoder(EncodeFn* out) {
  static EncodeFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return SP24_ERR_CUDA;
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  *out = encode;
  return SP24_OK;
}

// A 2-D map over `rows` rows of `row_bytes` bytes (elements of `elem` bytes), box `box_rows`
// whole rows, no swizzle (the data is already in its shared-memory order).
int make_tmap_rows(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem, uint64_t row_bytes,
                   uint64_t rows, uint32_t box_rows) {
  EncodeFn encode;
  int st = tmap_encoder(&encode);
  if (st) return st;
  if (!aligned(base, 16)) return SP24_ERR_ALIGN;
  cuuint64_t dims[2] = {row_bytes / elem, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(row_bytes / elem), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SP24_OK : SP24_ERR_CUDA;
}

// The fp32 output Y [M, N] as a 2-D map with box 128 rows of N x 32 tokens.
int make_tmap_y(CUtensorMap* map, float* y, int64_t M, int64_t N) {
  EncodeFn encode;
  int st = tmap_encoder(&encode);
  if (st) return st;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)N * 4};
  cuuint32_t box[2] = {128, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SP24_OK : SP24_ERR_CUDA;
}

namespace {

template <int BN, bool TMA_Y, bool SP>
int launch_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& sa, const CUtensorMap& sb,
                const CUtensorMap& te, const CUtensorMap& ty, const PairParams& p, cudaStream_t s) {
  auto kern = gemm_nvfp4_pair_kernel<BN, TMA_Y, SP>;
  const size_t smem = PairCfg<BN, SP>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  const int tiles = p.tiles_w * p.tiles_n;
  int pairs = sm_count() / 2;
  if (pairs > tiles) pairs = tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a, b, sa, sb, te, ty, p) != cudaSuccess) {
    cudaGetLastError();
    return SP24_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace

// W4A4 GEMM on the CTA-pair kernel: y[M, N] = s_w s_x sum_k dec(x) dec(w) with both operands in
// the tile images above (nvfp4_to_mma); K % 256 == 0.  BN = 256 tokens per pair tile above
// M = 128, else 128.
int tc_gemm_nvfp4_pair(const uint8_t* xc_mma, const uint8_t* xs_mma, const float* x_ts, const uint8_t* wc_mma,
                       const uint8_t* ws_mma, const float* w_ts, int64_t M, int64_t N, int64_t K, float* y,
                       cudaStream_t s, uint64_t wait_ns) {
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || K % 256) return SP24_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return SP24_OK;
  if (K == 0)
    return cudaMemsetAsync(y, 0, (size_t)(M * N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  const int BN = M > 128 ? 256 : 128;
  const uint64_t tiles_w = (uint64_t)(N + 127) / 128 * (K / 256), tiles_x = (uint64_t)(M + 127) / 128 * (K / 256);
  if (tiles_w * 8 > INT32_MAX || tiles_x * 8 > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  CUtensorMap ta, tb, tsa, tsb, ty, te;
  int st = make_tmap_rows(&ta, wc_mma, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 2048, tiles_w * 8, 8);
  if (st) return st;
  st = make_tmap_rows(&tb, xc_mma, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 2048, tiles_x * 8, BN == 256 ? 8 : 4);
  if (st) return st;
  st = make_tmap_rows(&tsa, ws_mma, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 512, (uint64_t)(N + 127) / 128 * (K / 64), 4);
  if (st) return st;
  st = make_tmap_rows(&tsb, xs_mma, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 512, (uint64_t)(M + 127) / 128 * (K / 64), 4);
  if (st) return st;
  const bool tma_y = N % 4 == 0 && aligned(y, 16);
  memset(&ty, 0, sizeof(ty));
  memset(&te, 0, sizeof(te));
  if (tma_y && (st = make_tmap_y(&ty, y, M, N))) return st;
  PairParams p{(int)M, (int)N, (int)K, y, w_ts, x_ts, (int)((N + 255) / 256), (int)((M + BN - 1) / BN), wait_ns};
  if (BN == 256)
    return tma_y ? launch_pair<256, true, false>(ta, tb, tsa, tsb, te, ty, p, s)
                 : launch_pair<256, false, false>(ta, tb, tsa, tsb, te, ty, p, s);
  return tma_y ? launch_pair<128, true, false>(ta, tb, tsa, tsb, te, ty, p, s)
               : launch_pair<128, false, false>(ta, tb, tsa, tsb, te, ty, p, s);
}

// W4A4 on the sparse FP4 MMA with a pairwise-4:8 weight, CTA-pair kernel: x as images with one
// scale per 32 K (nvfp4_b32_to_mma), the weight as images (sp48_to_mma: kept values, their
// scales, metadata; rows padded to 256); K % 512 == 0.
int tc_gemm_nvfp4_sp48_pair(const uint8_t* xc_mma, const uint8_t* xs_mma, const float* x_ts, const uint8_t* vc_mma,
                            const uint8_t* vs_mma, const uint8_t* meta_mma, const float* w_ts, int64_t M, int64_t N,
                            int64_t K, float* y, cudaStream_t s, uint64_t wait_ns) {
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || K % 512) return SP24_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return SP24_OK;
  if (K == 0)
    return cudaMemsetAsync(y, 0, (size_t)(M * N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  const int BN = M > 128 ? 256 : 128;
  const uint64_t wblocks = (uint64_t)sp48_rows_padded(N) / 128, xblocks = (uint64_t)(M + 127) / 128;
  if (wblocks * (K / 512) * 8 > INT32_MAX || xblocks * (K / 256) * 8 > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  CUtensorMap ta, tb, tsa, tsb, ty, te;
  int st = make_tmap_rows(&ta, vc_mma, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 2048, wblocks * (K / 512) * 8, 8);
  if (st) return st;
  st = make_tmap_rows(&tb, xc_mma, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 2048, xblocks * (K / 256) * 8,
                      BN == 256 ? 16 : 4);
  if (st) return st;
  st = make_tmap_rows(&tsa, vs_mma, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 512, wblocks * (K / 128), 4);
  if (st) return st;
  st = make_tmap_rows(&tsb, xs_mma, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, 512, xblocks * (K / 128), 4);
  if (st) return st;
  st = make_tmap_rows(&te, meta_mma, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 2048, wblocks * (K / 256), 2);
  if (st) return st;
  const bool tma_y = N % 4 == 0 && aligned(y, 16);
  memset(&ty, 0, sizeof(ty));
  if (tma_y && (st = make_tmap_y(&ty, y, M, N))) return st;
  PairParams p{(int)M, (int)N, (int)K, y, w_ts, x_ts, (int)((N + 255) / 256), (int)((M + BN - 1) / BN), wait_ns};
  if (BN == 256)
    return tma_y ? launch_pair<256, true, true>(ta, tb, tsa, tsb, te, ty, p, s)
                 : launch_pair<256, false, true>(ta, tb, tsa, tsb, te, ty, p, s);
  return tma_y ? launch_pair<128, true, true>(ta, tb, tsa, tsb, te, ty, p, s)
               : launch_pair<128, false, true>(ta, tb, tsa, tsb, te, ty, p, s);
}

}  // namespace sp24
