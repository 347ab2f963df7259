// a4 / a5 at prefill-sized M for 16-bit operands: a persistent tensor-core GEMM in which the two
// CTAs of a cluster work as one pair on 256 weight rows at a time (tcgen05 cta_group::2,
// kind::f16), dense or 2:4 sparse (tcgen05.mma.sp, K = 32 logical per instruction).
//
// [P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went", "The roofline is the
// whole argument": past the ridge the product is bound by the tensor pipe.  [P2] "Sparse GPU
// FLOPS Need the Right Zeros in the Right Places", "The mechanism needs both values and their
// positions": the kept values are the A operand and their 2-bit positions travel beside them as
// metadata, which the hardware uses to pick the matching activations.
//
// Y[m, n] = scale * sum_k x[m, k] w[n, k]: the weight is the A operand (M_mma = 256: 128 rows
// from each CTA), the activations the B operand (N_mma = BN tokens: each CTA loads its half, the
// pair's tensor cores share them), D in TMEM as weight rows on lanes x tokens on columns.
//   * operands straight from the row-major matrices by 2-D TMA boxes of 64 16-bit entries (one
//     128-byte swizzled K atom) per row; per stage and SM 128 weight rows and BN/2 token rows,
//     a third less than a single CTA computing the same 128 x BN outputs alone would load;
//   * 2:4 metadata from a tile image in the tcgen05 layout (sp24_prepare_sparse, or built per
//     call into the workspace): per stage one TMA row of 2 KB per CTA and one tcgen05.cp into a
//     4-column TMEM slot of that stage, issued by the MMA thread before the stage's MMAs, so no
//     warp rewrites nibbles on the way;
//   * persistent, tiles round-robin over the pairs, two TMEM accumulators so that a tile's
//     epilogue (TMEM -> registers -> shared memory -> TMA store of 32-token x 128-row fp32 boxes,
//     marked evict-first in L2 so the output does not push the operands out) overlaps the next
//     tile's main loop (2:4 at BN = 256: the accumulators overlap in 32
//     columns, read first and released, as in the FP4 pair kernel).
//
// Warp roles (192 threads per CTA): warp 0 = TMA producer (one lane; both CTAs load their own
// halves and count the bytes on the even CTA's barrier); warp 1 = TMEM allocation (both CTAs)
// and, in the even CTA, the MMA issuer (one lane); warps 2-5 = epilogue (TMEM lane quarter =
// warp % 4), each thread one weight row.  Every wait is bounded: when one runs out the kernel
// records SP24_ERR_DEVICE_TIMEOUT and unwinds.  No TMA load uses cluster multicast.
#include <cudaTypedefs.h>

#include "sp24_tc.cuh"

namespace sp24 {

// ------------------------------------------------------------------ 2:4 metadata image
//
// The tcgen05 metadata of a 2:4 A operand for 128 rows and 128 logical K (four 32-wide windows)
// is 4 TMEM columns of 128 lanes: lane l holds rows m = 16 (l / 16) + l % 8 and m + 8 of the
// 128-row block, and in column t (window t) the nibbles of groups 4 h .. 4 h + 3 (h = (l / 8) % 2)
// of window t: row m in the low half, row m + 8 in the high half.  The image stores that tile as
// 2 KB (lane l's 16 bytes at 16 l) for each 128-row block rb and 128-K chunk kc at byte
// 2048 (rb * K/128 + kc), rows padded to whole 256-row pair tiles with 0x44 bytes (the index
// pair 0, 1 in every group).
int64_t meta_image_rows(int64_t rows) { return (rows + 255) / 256 * 256; }
int64_t meta_image_bytes(int64_t rows, int64_t K) { return meta_image_rows(rows) / 128 * (K / 128) * 2048; }

namespace {

__global__ void __launch_bounds__(256) meta_image_kernel(const uint8_t* __restrict__ meta, int64_t rows, int64_t K,
                                                         uint8_t* __restrict__ out, int64_t ntiles) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= ntiles * 128) return;
  const int64_t tile = i >> 7;
  const int l = (int)(i & 127);
  const int64_t kcs = K / 128, rb = tile / kcs, kc = tile % kcs;
  const int64_t m = 128 * rb + 16 * (l / 16) + l % 8;
  const int h = (l / 8) % 2;
  const int64_t mb = K / 8;  // nibble bytes per row
  uint32_t w[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int64_t byte = 16 * kc + 4 * t + 2 * h;
    const uint32_t lo = m < rows ? (uint32_t)meta[m * mb + byte] | ((uint32_t)meta[m * mb + byte + 1] << 8) : 0x4444u;
    const uint32_t hi =
        m + 8 < rows ? (uint32_t)meta[(m + 8) * mb + byte] | ((uint32_t)meta[(m + 8) * mb + byte + 1] << 8) : 0x4444u;
    w[t] = lo | (hi << 16);
  }
  *reinterpret_cast<uint4*>(out + tile * 2048 + 16 * l) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

int meta_to_image(const uint8_t* meta, int64_t rows, int64_t K, uint8_t* out, cudaStream_t s) {
  const int64_t ntiles = meta_image_rows(rows) / 128 * (K / 128);
  if (ntiles == 0) return SP24_OK;
  const int64_t threads = ntiles * 128;
  meta_image_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(meta, rows, K, out, ntiles);
  return launch_status();
}

// ------------------------------------------------------------------ the pair GEMM

namespace {

using namespace tc;

template <int BN, bool SP>
struct F16PairCfg {
  static constexpr int KSTAGE = SP ? 128 : 64;                  // logical K per stage
  static constexpr uint32_t A = 128 * 128;                      // 128 rows x 64 stored 16-bit entries
  static constexpr uint32_t B = (SP ? 2 : 1) * (BN / 2) * 128;  // this CTA's token rows x KSTAGE
  static constexpr uint32_t META = SP ? 2048 : 0;               // one metadata tile
  static constexpr uint32_t STAGE = (A + B + META + 1023) / 1024 * 1024;
  static constexpr uint32_t LOADED = A + B + META;               // bytes one CTA's copies deliver
  static constexpr uint32_t EPI = 32 * 128 * 4;                 // one 32-token x 128-row fp32 chunk
  static constexpr int SMAX = (int)((232448 - 1024 - 2 * EPI) / STAGE);
  static constexpr int S = SMAX > 8 ? 8 : SMAX;
  static constexpr size_t SMEM = (size_t)S * STAGE + 2 * EPI + 1024;
  // TMEM columns: accumulator 0 at 0, accumulator 1 at ACC1 (2:4 at BN = 256: overlapping in
  // 32 columns), then (2:4) one 4-column metadata slot per stage
  static constexpr uint32_t ACC1 = SP && BN == 256 ? 224 : BN;
  static constexpr uint32_t META_COL = ACC1 + BN;
  static constexpr uint32_t COLS = 512;
  static constexpr int CHUNKS = BN / 32;
  static constexpr int OVERLAP_CHUNKS = BN == 256 ? (int)((256 - ACC1) / 32) : 0;
  static_assert(STAGE % 1024 == 0 && SMEM <= 232448 && S >= 2, "shared memory layout");
  static_assert(META_COL + (SP ? 4 * S : 0) <= COLS, "TMEM columns");
  static_assert(OVERLAP_CHUNKS <= 3, "epilogue buffers");
};

struct F16PairParams {
  int M, N, K;          // M tokens, N weight rows
  float* y;             // [M, N] fp32
  const float* scale_a;  // optional scales (device)
  const float* scale_b;
  int tiles_w, tiles_n;  // weight tiles of 256 rows, token tiles of BN
  uint64_t wait_ns;
};

// TMA_Y: the epilogue stages each 32-token chunk in shared memory and writes it with one TMA
// store (needs N % 4 == 0 and a 16-byte aligned y); otherwise each warp stores its rows directly.
template <int BN, bool TMA_Y, bool SP, bool BF16>
__global__ void __launch_bounds__(192, 1)
    gemm_f16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                         const F16PairParams p) {
  using C = F16PairCfg<BN, SP>;
  constexpr int S = C::S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = tc::align1024(smem_raw);
  auto sA = [&](int s) { return smem + s * C::STAGE; };
  auto sB = [&](int s) { return sA(s) + C::A; };
  auto sE = [&](int s) { return sB(s) + C::B; };  // 2:4 metadata tile
  float* sY = reinterpret_cast<float*>(smem + S * C::STAGE);  // two epilogue chunks
  // tempty_bar[0]: with overlapping accumulators, one release per tile (early, after the shared
  // columns are read); without, tempty_bar[a]: accumulator a fully read
  __shared__ uint64_t full_bar[S], empty_bar[S], tfull_bar, tempty_bar[2];
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
    }
    mbar_init(&tfull_bar, 1);
    mbar_init(&tempty_bar[0], 8);  // 4 epilogue warps in each CTA
    mbar_init(&tempty_bar[1], 8);
    aborted = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (SP) prefetch_tmap(&tmE);
    if (TMA_Y) prefetch_tmap(&tmY);
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
        const int wb = (t % p.tiles_w) * 2 + (int)rank;  // this CTA's 128-row weight block
        const int nrow = (t / p.tiles_w) * BN + (int)rank * (BN / 2);  // this CTA's first token
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait_for(&empty_bar[s], ph ^ 1, wait_ns) || *(volatile int*)&aborted) {
            aborted = 1;
            ok = false;
            break;
          }
          const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
          if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * C::LOADED);
          tma_load_2d_pair(sA(s), &tmA, fb, kb * 64, wb * 128);  // 64 stored entries of 128 rows
#pragma unroll
          for (int u = 0; u < (SP ? 2 : 1); ++u)
            tma_load_2d_pair(sB(s) + u * (BN / 2) * 128, &tmB, fb, kb * C::KSTAGE + 64 * u, nrow);
          if (SP) tma_load_2d_pair(sE(s), &tmE, fb, 0, wb * (p.K / 128) + kb);
        }
      }
      // the even CTA's producer armed every stage it counted: wait (bounded) until those copies
      // (its own and the odd CTA's) have landed before the pair may exit
      if (leader)
        for (int i = it - S > 0 ? it - S : 0; i < it; ++i) mbar_wait_for(&full_bar[i % S], (i / S) & 1, wait_ns);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_f16(256, BN, BF16, SP);
      int it = 0, j = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += pairs, ++j) {
        const uint32_t d = tmem + ((j & 1) ? C::ACC1 : 0u);
        const bool wait_ok = C::OVERLAP_CHUNKS ? (j < 1 || mbar_wait_cluster(&tempty_bar[0], (j - 1) & 1, wait_ns))
                                               : (j < 2 || mbar_wait_cluster(&tempty_bar[j & 1], ((j - 2) >> 1) & 1, wait_ns));
        if (!wait_ok) {
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
          tc_fence_after();
          const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA(s)));
          if (SP) {
            // the stage's metadata into its own slot (free: the MMAs that last read it belong to
            // the stage this copy's data replaced, which completed before the producer refilled it)
            const uint32_t ecol = tmem + C::META_COL + 4 * (uint32_t)s;
            tmem_cp_128x128b_pair(ecol, desc_rows16_noswizzle(smem_u32(sE(s))));
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // window q: A + 32 B, B atom q / 2 + 64 B * (q % 2)
              const uint64_t b = desc_kmajor_sw128(smem_u32(sB(s) + (q >> 1) * (BN / 2) * 128)) + 4 * (q & 1);
              // the metadata address must be even: an odd column is named by the even one below it
              // plus the instruction descriptor's sparse-id2 field
              const uint32_t e = ecol + q;
              umma_f16_sp_pair(d, a0 + 2 * q, b, e & ~1u, idesc | (e & 1u), (kb | q) != 0);
            }
          } else {
            const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB(s)));
#pragma unroll
            for (int q = 0; q < 4; ++q)  // K = 16 entries = 32 bytes = 2 descriptor units
              umma_f16_pair(d, a0 + 2 * q, b0 + 2 * q, idesc, (kb | q) != 0);
          }
          umma_commit_pair(&empty_bar[s], 0x3);
        }
        if (ok) umma_commit_pair(&tfull_bar, 0x3);
      }
    }
  } else {
    // epilogue: thread = one weight row of this CTA, 32 tokens per TMEM load
    const int q = warp & 3;
    const bool epi_leader = warp == 2 && lane == 0;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty_bar[1]), 0);
    const uint64_t y_policy = l2_evict_first_policy();
    float scale = 1.0f;
    if (p.scale_a) scale *= *p.scale_a;
    if (p.scale_b) scale *= *p.scale_b;
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
      // chunk order: the columns shared with the other accumulator first
      auto chunk_at = [&](int i) {
        if (C::OVERLAP_CHUNKS && !(j & 1)) return (i + C::CHUNKS - C::OVERLAP_CHUNKS) % C::CHUNKS;
        return i;
      };
      // three chunks in flight; with overlapping accumulators, once those are in registers the
      // accumulator goes back to the MMAs (the shared columns come first)
      uint32_t r[3][32];
#pragma unroll
      for (int i = 0; i < 3; ++i) tmem_ld32_async(base + 32 * chunk_at(i), r[i]);
      tmem_wait_ld();
      if (C::OVERLAP_CHUNKS) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader0);
      }
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
        if (!C::OVERLAP_CHUNKS && i == C::CHUNKS - 1) {  // every column is in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster((j & 1) ? tempty_leader1 : tempty_leader0);
        }
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

template <int BN, bool TMA_Y, bool SP, bool BF16>
int launch_f16_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& e, const CUtensorMap& y,
                    const F16PairParams& p, cudaStream_t s) {
  auto kern = gemm_f16_pair_kernel<BN, TMA_Y, SP, BF16>;
  const size_t smem = F16PairCfg<BN, SP>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  const int tiles = p.tiles_w * p.tiles_n;
  int pairs = sm_count() / 2;
  if (pairs > tiles) pairs = tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a, b, e, y, p) != cudaSuccess) {
    cudaGetLastError();
    return SP24_ERR_CUDA;
  }
  return launch_status();
}

template <bool SP, bool BF16>
int dispatch_f16_pair(int BN, bool tma_y, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& e,
                      const CUtensorMap& y, const F16PairParams& p, cudaStream_t s) {
  if (BN == 256)
    return tma_y ? launch_f16_pair<256, true, SP, BF16>(a, b, e, y, p, s) : launch_f16_pair<256, false, SP, BF16>(a, b, e, y, p, s);
  return tma_y ? launch_f16_pair<128, true, SP, BF16>(a, b, e, y, p, s) : launch_f16_pair<128, false, SP, BF16>(a, b, e, y, p, s);
}

}  // namespace

// 16-bit GEMM on the CTA-pair kernel: y[M, N] = scale_a scale_b sum_k x[m, k] w[n, k] (dense:
// w [N, K], K % 64 == 0) or with a 2:4 weight (values [N, K/2] and its metadata image
// meta_img from meta_to_image, K % 128 == 0).  BN = 256 tokens per pair tile above M = 128.
int tc_gemm_f16_pair(const void* x, const void* w, const uint8_t* meta_img, int64_t M, int64_t N, int64_t K,
                     bool bf16, float* y, const float* scale_a, const float* scale_b, cudaStream_t s,
                     uint64_t wait_ns) {
  const bool sp = meta_img != nullptr;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || K % (sp ? 128 : 64)) return SP24_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return SP24_OK;
  if (K == 0)
    return cudaMemsetAsync(y, 0, (size_t)(M * N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  const int BN = M > 128 ? 256 : 128;
  if (meta_image_rows(N) / 128 * (K / 128) > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  CUtensorMap ta, tb, te, ty;
  int st = make_tmap_2d(&ta, w, 2, (uint64_t)N, (uint64_t)(sp ? K / 2 : K), (uint64_t)(sp ? K : 2 * K), 64, 128);
  if (st) return st;
  st = make_tmap_2d(&tb, x, 2, (uint64_t)M, (uint64_t)K, (uint64_t)(2 * K), 64, (uint32_t)(BN / 2));
  if (st) return st;
  memset(&te, 0, sizeof(te));
  memset(&ty, 0, sizeof(ty));
  if (sp && (st = make_tmap_rows(&te, meta_img, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 2048,
                                 (uint64_t)(meta_image_rows(N) / 128 * (K / 128)), 1)))
    return st;
  const bool tma_y = N % 4 == 0 && aligned(y, 16);
  if (tma_y && (st = make_tmap_y(&ty, y, M, N))) return st;
  F16PairParams p{(int)M, (int)N, (int)K, y, scale_a, scale_b, (int)((N + 255) / 256), (int)((M + BN - 1) / BN), wait_ns};
  if (sp)
    return bf16 ? dispatch_f16_pair<true, true>(BN, tma_y, ta, tb, te, ty, p, s)
                : dispatch_f16_pair<true, false>(BN, tma_y, ta, tb, te, ty, p, s);
  return bf16 ? dispatch_f16_pair<false, true>(BN, tma_y, ta, tb, te, ty, p, s)
              : dispatch_f16_pair<false, false>(BN, tma_y, ta, tb, te, ty, p, s);
}

}  // namespace sp24

using namespace sp24;

extern "C" int sp24_prepare_sparse_size(int64_t rows, int64_t K, int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 128) return SP24_ERR_SHAPE;
  *bytes = meta_image_bytes(rows, K);
  return SP24_OK;
}

extern "C" int sp24_prepare_sparse(const uint8_t* meta, int64_t rows, int64_t K, uint8_t* meta_img, void* stream) {
  if (rows < 0 || K < 0 || K % 128) return SP24_ERR_SHAPE;
  if (rows == 0 || K == 0) return SP24_OK;
  if (!meta || !meta_img) return SP24_ERR_INVALID_ARG;
  if (!aligned(meta_img, 16)) return SP24_ERR_ALIGN;
  return meta_to_image(meta, rows, K, meta_img, as_stream(stream));
}
