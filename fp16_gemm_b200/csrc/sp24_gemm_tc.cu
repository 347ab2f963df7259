// a4 at prefill-sized M, single-CTA form: tensor-core GEMM on tcgen05 (kind::f16), TMA-fed, TMEM
// accumulator, for K that is not a multiple of 64 (the CTA-pair kernel of sp24_gemm_f16pair.cu
// takes every other 16-bit shape, dense and 2:4); also the tensor-map helpers, the sparse FP4
// kernel for pairwise-4:8 weights and the NVFP4 -> 16-bit expansion.
//
// [P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went", "The roofline is the
// whole argument": past the ridge point the product is bound by the tensor pipe, so this path
// keeps the tensor cores fed from shared memory staged by TMA.
//
// Y[m, n] = scale * sum_k x[m, k] w[n, k].  The weight is the MMA's A operand (M_mma = 128
// weight rows per CTA), the activations the B operand (N_mma = BN tokens per CTA); D lives in
// TMEM as 128 lanes (weight rows) x BN fp32 columns (tokens), so the epilogue's tcgen05.ld
// gives each thread one weight row and 32 tokens, and each store instruction writes 32
// consecutive floats of one output row.
//
// Warp roles (192 threads): warp 0 = TMA producer (one lane), warp 1 = TMEM owner and MMA
// issuer (one lane), warps 2..5 = epilogue (TMEM lane quarter = warp % 4).  A ring of S stages
// of (A, B) 64-wide K slices, each 128-byte swizzled, is guarded by full/empty mbarriers; the
// MMA warp frees a stage with tcgen05.commit.  Every wait is bounded: when one runs out the
// kernel records SP24_ERR_DEVICE_TIMEOUT and unwinds.
//
// NVFP4 and 2:4-compressed NVFP4 weights reach the 16-bit kernels through an expansion kernel
// that writes the exact 16-bit values E2M1 * E4M3 (and, for a dense expansion, zeros for pruned
// entries) into a workspace; the tensor scales are applied in the epilogue.
#include <cudaTypedefs.h>

#include "sp24_tc.cuh"

namespace sp24 {

int make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                 uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return SP24_ERR_CUDA;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (!aligned(base, 16) || pitch_bytes % 16) return SP24_ERR_ALIGN;
  CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SP24_OK : SP24_ERR_CUDA;
}

// Byte tensor [rows, cols] with row pitch `pitch_bytes`, box (box_cols x box_rows), no swizzle.
int make_tmap_2d_plain(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                       uint32_t box_cols, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return SP24_ERR_CUDA;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (!aligned(base, 16) || pitch_bytes % 16) return SP24_ERR_ALIGN;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SP24_OK : SP24_ERR_CUDA;
}

namespace {

using namespace tc;

constexpr int kBM = 128, kBK = 64;

template <int BN>
struct TcCfg {
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr uint32_t A_BYTES = kBM * kBK * 2;
  static constexpr uint32_t B_BYTES = BN * kBK * 2;
  static constexpr size_t SMEM = (size_t)STAGES * (A_BYTES + B_BYTES) + 1024;
};

struct TcParams {
  int M, N, K;
  float* y;
  const float* scale_a;  // optional device scalars multiplied into the epilogue scale
  const float* scale_b;
};

template <int BN, bool BF16>
__global__ void __launch_bounds__(192, 1)
    gemm_f16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const TcParams p) {
  using C = TcCfg<BN>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = tc::align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * C::A_BYTES;
  __shared__ uint64_t full_bar[S], empty_bar[S], tfull_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int aborted;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;  // weight rows
  const int n0 = blockIdx.y * BN;   // tokens
  const int KB = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&tfull_bar, 1);
    aborted = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(&tmem_base, BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[s], C::A_BYTES + C::B_BYTES);
        tma_load_2d(sA + s * C::A_BYTES, &tmA, &full_bar[s], kb * kBK, m0);
        tma_load_2d(sB + s * C::B_BYTES, &tmB, &full_bar[s], kb * kBK, n0);
        ++issued;
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int kb = issued - S > 0 ? issued - S : 0; kb < issued; ++kb)
        mbar_wait(&full_bar[kb % S], (kb / S) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kBM, BN, BF16);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!mbar_wait(&full_bar[s], ph) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA + s * C::A_BYTES));
        const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB + s * C::B_BYTES));
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)  // K = 16 per MMA: 32 bytes = 2 descriptor units
          umma_f16(tmem, a0 + 2 * k, b0 + 2 * k, idesc, (kb | k) != 0);
        umma_commit(&empty_bar[s]);
      }
      umma_commit(&tfull_bar);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = m0 + 32 * q + lane;
    if (!mbar_wait(&tfull_bar, 0)) {
      aborted = 1;
    } else {
      tc_fence_after();
      float scale = 1.0f;
      if (p.scale_a) scale *= *p.scale_a;
      if (p.scale_b) scale *= *p.scale_b;
#pragma unroll 1
      for (int j = 0; j < BN / 32; ++j) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * j, v);
        if (row < p.N) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = n0 + 32 * j + i;
            if (tok < p.M) p.y[(int64_t)tok * p.N + row] = v[i] * scale;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && aborted) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

template <int BN, bool BF16>
int launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const TcParams& p, cudaStream_t s) {
  auto kern = gemm_f16_tc_kernel<BN, BF16>;
  const size_t smem = TcCfg<BN>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  dim3 grid((p.N + kBM - 1) / kBM, (p.M + BN - 1) / BN);
  kern<<<grid, 192, smem, s>>>(ta, tb, p);
  return launch_status();
}

// ------------------------------------------------------------------ scale tiles for the sparse FP4 MMA

// Rewrites, in place, the scale rows of `groups` 128-row groups (16 bytes per row: 4 MMAs x 4
// scales) into the tiles tcgen05.cp reads: tile (j, g) = MMA j, rows 128 g .. 128 g + 127, the
// word of row r at index 4 * (r % 32) + r / 32.  One warp; every lane loads all it needs before
// any lane stores.
template <int GROUPS>
__device__ __forceinline__ void scale_tiles_in_place(uint8_t* buf, int lane) {
  uint4 w[GROUPS][4];
#pragma unroll
  for (int g = 0; g < GROUPS; ++g)
#pragma unroll
    for (int rq = 0; rq < 4; ++rq) w[g][rq] = *reinterpret_cast<const uint4*>(buf + 16 * (128 * g + 32 * rq + lane));
  __syncwarp();
#pragma unroll
  for (int g = 0; g < GROUPS; ++g) {
    const uint32_t col[4][4] = {{w[g][0].x, w[g][1].x, w[g][2].x, w[g][3].x}, {w[g][0].y, w[g][1].y, w[g][2].y, w[g][3].y},
                                {w[g][0].z, w[g][1].z, w[g][2].z, w[g][3].z}, {w[g][0].w, w[g][1].w, w[g][2].w, w[g][3].w}};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(buf + 512 * (j * GROUPS + g) + 16 * lane) = make_uint4(col[j][0], col[j][1], col[j][2], col[j][3]);
  }
}

// ------------------------------------------------------------------ W4A4 with a pairwise 4:8 weight
//
// The sparse FP4 MMA (tcgen05.mma.sp kind::mxf4nvf4.block_scale, K = 128 logical per
// instruction).  A = the kept values of a pairwise-4:8 weight as packed E2M1 (64 stored per row
// per instruction, the pairs in ascending order) with their 16-value E4M3 scales (one per 32
// logical K) and the metadata nibbles; B = the activations as E2M1 with one E4M3 scale per 32 K.
// Per stage (512 logical K): A one 128-byte swizzled box, B two; 16 scale bytes per row of each
// operand, rewritten in place by warp 6 into the same TMEM tiles as the dense kernel (4 per
// instruction);
// the metadata as two boxes of 128 rows x 16 bytes, copied into TMEM with tcgen05.cp.128x128b
// (row m on lane m, 16 bytes = 256 logical K = 4 columns, chunk 2c in the low nibble of byte
// c).  Rows beyond N arrive as zeros, which is not a legal nibble; warp 6 writes the legal 0x4
// (pairs 0 and 1) there before the copy, and those rows' outputs are never stored.
template <int BN>
struct SCfg {
  static constexpr int S = BN == 256 ? 2 : 4;
  static constexpr uint32_t A = kBM * 128;  // 128 rows x 256 stored FP4 = 512 logical K
  static constexpr uint32_t B = BN * 256;   // BN rows x 512 FP4, two 128-byte boxes
  static constexpr uint32_t SFA = kBM * 16; // scale rows, rewritten in place into tiles
  static constexpr uint32_t SFB = BN * 16;
  static constexpr uint32_t E = kBM * 32;   // two boxes of 128 rows x 16 bytes
  static constexpr uint32_t STAGE = A + B + SFA + SFB + E;
  static constexpr size_t SMEM = (size_t)S * STAGE + 1024;
  static constexpr int E_COLS = 8;
  static constexpr int SFA_COLS = 16;             // 4 MMAs x 4 columns
  static constexpr int SFB_COLS = 4 * (BN / 32);  // 4 MMAs x BN/32 columns
  static constexpr int STAGE_COLS = E_COLS + SFA_COLS + SFB_COLS;
  static constexpr int COLS = BN + S * STAGE_COLS <= 256 ? 256 : 512;
  static_assert(STAGE % 1024 == 0 && SMEM <= 232448, "stage layout");
  static_assert(BN + S * STAGE_COLS <= 512, "TMEM columns");
};

template <int BN>
__global__ void __launch_bounds__(224, 1)
    gemm_nvfp4sp_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                           const __grid_constant__ CUtensorMap tmE, const TcParams p) {
  using C = SCfg<BN>;
  constexpr int S = C::S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = tc::align1024(smem_raw);
  auto sA = [&](int s) { return smem + s * C::STAGE; };
  auto sB = [&](int s) { return sA(s) + C::A; };
  auto sSA = [&](int s) { return sB(s) + C::B; };
  auto sSB = [&](int s) { return sSA(s) + C::SFA; };
  auto sE = [&](int s) { return sSB(s) + C::SFB; };
  __shared__ uint64_t full_bar[S], sf_bar[S], empty_bar[S], tfull_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int aborted;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;  // weight rows
  const int n0 = blockIdx.y * BN;   // activation rows
  const int KB = p.K / 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&sf_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&tfull_bar, 1);
    aborted = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSA);
    prefetch_tmap(&tmSB);
    prefetch_tmap(&tmE);
  }
  if (warp == 1) tmem_alloc(&tmem_base, C::COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[s], C::A + C::B + C::SFA + C::SFB + C::E);
        tma_load_2d(sA(s), &tmA, &full_bar[s], kb * 128, m0);  // 128 bytes = 256 stored codes
        tma_load_2d(sB(s), &tmB, &full_bar[s], kb * 256, n0);  // 2 x 128 bytes = 512 codes
        tma_load_2d(sB(s) + BN * 128, &tmB, &full_bar[s], kb * 256 + 128, n0);
        tma_load_2d(sSA(s), &tmSA, &full_bar[s], kb * 16, m0);  // 16 scales per row
        tma_load_2d(sSB(s), &tmSB, &full_bar[s], kb * 16, n0);
        tma_load_2d(sE(s), &tmE, &full_bar[s], kb * 32, m0);  // 2 x 16 bytes of nibbles per row
        tma_load_2d(sE(s) + 2048, &tmE, &full_bar[s], kb * 32 + 16, m0);
        ++issued;
      }
      for (int kb = issued - S > 0 ? issued - S : 0; kb < issued; ++kb)
        mbar_wait(&full_bar[kb % S], (kb / S) & 1);
    }
  } else if (warp == 6) {
    const int valid = p.N - m0;  // rows of this weight tile that exist (>= 1)
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (kb / S) & 1;
      if (!mbar_wait(&full_bar[s], ph) || *(volatile int*)&aborted) {
        aborted = 1;
        break;
      }
      scale_tiles_in_place<1>(sSA(s), lane);
      scale_tiles_in_place<BN / 128>(sSB(s), lane);
      for (int r = valid + lane; r < kBM; r += 32) {
        const uint4 legal = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
        *reinterpret_cast<uint4*>(sE(s) + 16 * r) = legal;
        *reinterpret_cast<uint4*>(sE(s) + 2048 + 16 * r) = legal;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_bar[s]);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_nvfp4(kBM, BN, true);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!mbar_wait(&full_bar[s], ph) || !mbar_wait(&sf_bar[s], ph) || *(volatile int*)&aborted) {
          aborted = 1;
          break;
        }
        tc_fence_after();
        const uint32_t e0 = tmem + BN + s * C::STAGE_COLS;
        const uint32_t sfa0 = e0 + C::E_COLS;
        const uint32_t sfb0 = sfa0 + C::SFA_COLS;
        tmem_cp_128x128b(e0, desc_rows16_noswizzle(smem_u32(sE(s))));
        tmem_cp_128x128b(e0 + 4, desc_rows16_noswizzle(smem_u32(sE(s) + 2048)));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tmem_cp_32x128b_x4(sfa0 + 4 * j, desc_rows16_noswizzle(smem_u32(sSA(s) + 512 * j)));
#pragma unroll
          for (int g = 0; g < BN / 128; ++g)
            tmem_cp_32x128b_x4(sfb0 + (BN / 32) * j + 4 * g,
                               desc_rows16_noswizzle(smem_u32(sSB(s) + 512 * (j * (BN / 128) + g))));
        }
        const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA(s)));
        const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB(s)));
        const uint64_t b1 = desc_kmajor_sw128(smem_u32(sB(s) + BN * 128));
#pragma unroll
        for (int j = 0; j < 4; ++j)  // A: 32 bytes (2 descriptor units) per MMA; B: 64 bytes (4)
          umma_nvfp4_sp(tmem, a0 + 2 * j, (j < 2 ? b0 : b1) + 4 * (j & 1), e0 + 2 * j, idesc, sfa0 + 4 * j,
                        sfb0 + (BN / 32) * j, (kb | j) != 0);
        umma_commit(&empty_bar[s]);
      }
      umma_commit(&tfull_bar);
    }
  } else if (warp >= 2) {
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
    if (!mbar_wait(&tfull_bar, 0)) {
      aborted = 1;
    } else {
      tc_fence_after();
      float scale = 1.0f;
      if (p.scale_a) scale *= *p.scale_a;
      if (p.scale_b) scale *= *p.scale_b;
#pragma unroll 1
      for (int j = 0; j < BN / 32; ++j) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * j, v);
        if (row < p.N) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = n0 + 32 * j + i;
            if (tok < p.M) p.y[(int64_t)tok * p.N + row] = v[i] * scale;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && aborted) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::COLS);
  }
}

template <int BN>
int launch_nvfp4sp(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& sa, const CUtensorMap& sb,
                   const CUtensorMap& e, const TcParams& p, cudaStream_t s) {
  auto kern = gemm_nvfp4sp_tc_kernel<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SCfg<BN>::SMEM) != cudaSuccess)
    return SP24_ERR_CUDA;
  dim3 grid((unsigned)((p.N + kBM - 1) / kBM), (unsigned)((p.M + BN - 1) / BN));
  kern<<<grid, 224, SCfg<BN>::SMEM, s>>>(a, b, sa, sb, e, p);
  return launch_status();
}

// ------------------------------------------------------------------ weight expansion to 16-bit

// Dense NVFP4 ([rows, K/2] codes, [rows, K/16] scales) or 2:4-compressed weights (16-bit values
// or NVFP4 values + nibbles) -> dense 16-bit [rows, K] holding E2M1 * E4M3 (exact) or the kept
// 16-bit values, zeros at pruned positions.  One group of four outputs per thread.
template <int WF, bool BF16>
__global__ void __launch_bounds__(256) expand_w16_kernel(const uint8_t* __restrict__ w,
                                                         const uint8_t* __restrict__ scales,
                                                         const uint8_t* __restrict__ meta, int64_t rows,
                                                         int64_t K, uint16_t* __restrict__ out) {
  const int64_t groups = rows * (K / 4);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
    uint16_t e[4] = {0, 0, 0, 0};
    auto fp4 = [&](int64_t idx, int64_t scale_idx) -> uint16_t {
      uint32_t c = (w[idx >> 1] >> (4 * (idx & 1))) & 0xf;
      uint32_t mag = c & 7, ex = mag >> 1, m = mag & 1;
      float a = ex == 0 ? 0.5f * m : (float)(1 << (ex - 1)) * (1.0f + 0.5f * m);
      uint32_t h2;
      uint16_t sc = scales[scale_idx];
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(sc));
      float v = a * __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
      v = c & 8 ? -v : v;
      if (BF16) {
        __nv_bfloat16 b = __float2bfloat16_rn(v);
        return *reinterpret_cast<uint16_t*>(&b);
      }
      __half h = __float2half_rn(v);
      return *reinterpret_cast<uint16_t*>(&h);
    };
    if (WF == W_DQ4) {
#pragma unroll
      for (int i = 0; i < 4; ++i) e[i] = fp4(4 * g + i, (4 * g + i) >> 4);
    } else {
      uint32_t nib = (meta[g >> 1] >> (4 * (g & 1))) & 0xf;
      uint32_t i0 = nib & 3, i1 = nib >> 2;
      uint16_t v0, v1;
      if (WF == W_S16) {
        v0 = reinterpret_cast<const uint16_t*>(w)[2 * g];
        v1 = reinterpret_cast<const uint16_t*>(w)[2 * g + 1];
      } else {
        v0 = fp4(2 * g, (2 * g) >> 4);
        v1 = fp4(2 * g + 1, (2 * g + 1) >> 4);
      }
      if (i0 < i1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) e[i] = (i == (int)i0) ? v0 : ((i == (int)i1) ? v1 : (uint16_t)0);
      }
    }
    reinterpret_cast<uint2*>(out)[g] = make_uint2(e[0] | ((uint32_t)e[1] << 16), e[2] | ((uint32_t)e[3] << 16));
  }
}

}  // namespace

// W4A4 GEMM on the sparse FP4 MMA: y = s_w s_x sum_k dec(x) dec(w) with w a pairwise-4:8 weight
// (values codes [N, K/4], their scales [N, K/32], meta [N, K/16]) and x packed E2M1 with one
// scale per 32 K ([M, K/2] codes, [M, K/32] scales); K % 512 == 0 (whole stages, and 16-byte
// scale-row pitches for the tensor maps).
int tc_gemm_nvfp4_sp48(const uint8_t* xc, const uint8_t* xs, const float* x_ts, const uint8_t* vc,
                       const uint8_t* vs, const uint8_t* meta, const float* w_ts, int64_t M, int64_t N, int64_t K,
                       float* y, cudaStream_t s) {
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || K % 512) return SP24_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return SP24_OK;
  if (K == 0)
    return cudaMemsetAsync(y, 0, (size_t)(M * N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  // 256-wide activation tiles from M = 257 on; below that, 128-wide ones give twice the CTAs
  // (measured at N = K = 4096: M = 256 11.8 us with 128-wide tiles, 17.6 us with 256-wide)
  const int BN = M > 256 ? 256 : 128;
  CUtensorMap ta, tb, tsa, tsb, te;
  int st = make_tmap_2d(&ta, vc, 1, N, K / 4, K / 4, 128, kBM);
  if (st) return st;
  st = make_tmap_2d(&tb, xc, 1, M, K / 2, K / 2, 128, BN);
  if (st) return st;
  st = make_tmap_2d_plain(&tsa, vs, N, K / 32, K / 32, 16, kBM);
  if (st) return st;
  st = make_tmap_2d_plain(&tsb, xs, M, K / 32, K / 32, 16, BN);
  if (st) return st;
  st = make_tmap_2d_plain(&te, meta, N, K / 16, K / 16, 16, kBM);
  if (st) return st;
  TcParams p{(int)M, (int)N, (int)K, y, w_ts, x_ts};
  return BN == 256 ? launch_nvfp4sp<256>(ta, tb, tsa, tsb, te, p, s) : launch_nvfp4sp<128>(ta, tb, tsa, tsb, te, p, s);
}

// Expands an NVFP4 / 2:4 operand of `rows` rows into 16-bit [rows, K] at `out` (workspace).
int expand_w16(int wf, bool bf16, const uint8_t* w, const uint8_t* scales, const uint8_t* meta, int64_t rows,
               int64_t K, uint16_t* out, cudaStream_t s) {
  const int64_t groups = rows * (K / 4);
  if (groups == 0) return SP24_OK;
  int64_t blocks = (groups + 255) / 256;
  if (blocks > (int64_t)sm_count() * 16) blocks = (int64_t)sm_count() * 16;
#define SP24_EXP(WFV)                                                                                      \
  (bf16 ? expand_w16_kernel<WFV, true><<<(unsigned)blocks, 256, 0, s>>>(w, scales, meta, rows, K, out)    \
        : expand_w16_kernel<WFV, false><<<(unsigned)blocks, 256, 0, s>>>(w, scales, meta, rows, K, out))
  switch (wf) {
    case W_DQ4: SP24_EXP(W_DQ4); break;
    case W_S16: SP24_EXP(W_S16); break;
    case W_SQ4: SP24_EXP(W_SQ4); break;
    default: return SP24_ERR_UNSUPPORTED;
  }
#undef SP24_EXP
  return launch_status();
}

// Dense 16-bit tensor-core GEMM: y[M, N] = scale * x[M, K] w[N, K]^T (x, w 16-bit, K % 8 == 0).
int tc_gemm_f16(const void* x, const void* w, int64_t M, int64_t N, int64_t K, bool bf16, float* y,
                const float* scale_a, const float* scale_b, cudaStream_t s) {
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return SP24_ERR_UNSUPPORTED;
  if (K == 0)
    return cudaMemsetAsync(y, 0, (size_t)(M * N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  const int BN = M > 128 ? 256 : (M > 64 ? 128 : 64);
  CUtensorMap ta, tb;
  int st = make_tmap_2d(&ta, w, 2, N, K, K * 2, kBK, kBM);
  if (st) return st;
  st = make_tmap_2d(&tb, x, 2, M, K, K * 2, kBK, BN);
  if (st) return st;
  TcParams p{(int)M, (int)N, (int)K, y, scale_a, scale_b};
  if (BN == 256) return bf16 ? launch_tc<256, true>(ta, tb, p, s) : launch_tc<256, false>(ta, tb, p, s);
  if (BN == 128) return bf16 ? launch_tc<128, true>(ta, tb, p, s) : launch_tc<128, false>(ta, tb, p, s);
  return bf16 ? launch_tc<64, true>(ta, tb, p, s) : launch_tc<64, false>(ta, tb, p, s);
}

}  // namespace sp24

using namespace sp24;

extern "C" int sp24_gemm_sparse48(const sp24_operand* x, const sp24_sparse_operand* w, int64_t M, int64_t N,
                                  int64_t K, float* y, void* stream) {
  if (!x || !w) return SP24_ERR_INVALID_ARG;
  const bool images = x->format == SP24_NVFP4_B32_MMA && w->format == SP24_NVFP4_MMA;
  if (!images && (x->format != SP24_NVFP4_B32 || w->format != SP24_NVFP4)) return SP24_ERR_DTYPE;
  if (M < 0 || N < 0 || K < 0 || K % 512) return SP24_ERR_SHAPE;
  if (M == 0 || N == 0) return SP24_OK;
  if (!y) return SP24_ERR_INVALID_ARG;
  if (!aligned(y, 4)) return SP24_ERR_ALIGN;
  if (K > 0) {
    if (!x->data || !x->scales || !x->tensor_scale || !w->values || !w->scales || !w->tensor_scale || !w->meta)
      return SP24_ERR_INVALID_ARG;
    if (!aligned(x->data, 16) || !aligned(x->scales, 16) || !aligned(w->values, 16) || !aligned(w->scales, 16) ||
        !aligned(w->meta, 16))
      return SP24_ERR_ALIGN;
  }
  if (images)
    return tc_gemm_nvfp4_sp48_pair(static_cast<const uint8_t*>(x->data), x->scales, x->tensor_scale,
                                   static_cast<const uint8_t*>(w->values), w->scales, w->meta, w->tensor_scale, M, N,
                                   K, y, as_stream(stream), 0);
  return tc_gemm_nvfp4_sp48(static_cast<const uint8_t*>(x->data), x->scales, x->tensor_scale,
                            static_cast<const uint8_t*>(w->values), w->scales, w->meta, w->tensor_scale, M, N, K, y,
                            as_stream(stream));
}

extern "C" int sp24_nvfp4_b32_mma_size(int64_t rows, int64_t cols, int64_t* codes_bytes, int64_t* scales_bytes) {
  if (rows < 0 || cols < 0 || cols % 256) return SP24_ERR_SHAPE;
  if (codes_bytes) *codes_bytes = nvfp4_mma_codes_bytes(rows, cols);
  if (scales_bytes) *scales_bytes = b32_mma_scales_bytes(rows, cols);
  return SP24_OK;
}

extern "C" int sp24_nvfp4_b32_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                     uint8_t* codes_out, uint8_t* scales_out, void* stream) {
  if (rows < 0 || cols < 0 || cols % 256) return SP24_ERR_SHAPE;
  if (rows == 0 || cols == 0) return SP24_OK;
  if (!codes || !scales || !codes_out || !scales_out) return SP24_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 4) || !aligned(codes_out, 16) || !aligned(scales_out, 16))
    return SP24_ERR_ALIGN;
  return nvfp4_b32_to_mma(codes, scales, rows, cols, codes_out, scales_out, as_stream(stream));
}

extern "C" int sp24_sparse48_mma_size(int64_t rows, int64_t K, int64_t* values_bytes, int64_t* scales_bytes,
                                      int64_t* meta_bytes) {
  if (rows < 0 || K < 0 || K % 512) return SP24_ERR_SHAPE;
  if (values_bytes) *values_bytes = sp48_mma_values_bytes(rows, K);
  if (scales_bytes) *scales_bytes = sp48_mma_scales_bytes(rows, K);
  if (meta_bytes) *meta_bytes = sp48_mma_meta_bytes(rows, K);
  return SP24_OK;
}

extern "C" int sp24_sparse48_to_mma(const uint8_t* values, const uint8_t* scales, const uint8_t* meta,
                                    int64_t rows, int64_t K, uint8_t* values_out, uint8_t* scales_out,
                                    uint8_t* meta_out, void* stream) {
  if (rows < 0 || K < 0 || K % 512) return SP24_ERR_SHAPE;
  if (rows == 0 || K == 0) return SP24_OK;
  if (!values || !scales || !meta || !values_out || !scales_out || !meta_out) return SP24_ERR_INVALID_ARG;
  if (!aligned(values, 16) || !aligned(scales, 4) || !aligned(meta, 16) || !aligned(values_out, 16) ||
      !aligned(scales_out, 16) || !aligned(meta_out, 16))
    return SP24_ERR_ALIGN;
  return sp48_to_mma(values, scales, meta, rows, K, values_out, scales_out, meta_out, as_stream(stream));
}
