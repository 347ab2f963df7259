// a4 / a5 at prefill-sized M: tensor-core GEMM on tcgen05 (kind::f16), TMA-fed, TMEM accumulator.
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
// NVFP4 and 2:4-compressed weights reach this path through an expansion kernel that writes the
// exact 16-bit values E2M1 * E4M3 (and zeros for pruned entries) into a workspace; the tensor
// scales are applied in the epilogue.
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
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
