// a6: skinny (decode-shaped, M <= 64) dense and 2:4-sparse GEMM: Y[m, n] = sum_k x[m,k] w[n,k].
//
// [P5] "NVFP4 Without FP4 Hardware", section "Why NVFP4 helps without FP4 hardware": every
// generated token reads the whole weight set once, so a decode GEMM is bound by the weight
// read; NVFP4 weights are unpacked to 16-bit inside the kernel before the tensor cores see
// them.  [P1] "NVFP4 vs 2:4 sparse", "The byte saving is about a quarter, not a half": the
// compressed operand (values + 2-bit indices + scales) is what must stream from HBM.
//
// Design (HBM-bound; no shared-memory round trip for the weights):
//   - CTA = 4 warps = 64 weight rows (w rows are the MMA's M dimension: "swap AB"), one
//     K-slice of up to 4 chunks.  Every lane issues all of its 16-byte weight loads for the
//     slice up front (streaming, L1 no-allocate), so a warp keeps up to 8 KB in flight.
//   - Lane (g, c) of a warp owns rows g and g+8 of the warp's 16 and one 16-byte piece of each
//     row per chunk; it decodes that piece straight into the A fragments of mma.m16n8k16.
//     The K order inside a chunk is permuted (the same permutation is applied when x is
//     staged), so that each A register pairs the two entries the decode produces together.
//   - x for the slice is staged once per CTA in shared memory in fragment order: each
//     (step, token tile) is one 256-byte row read by the warp with conflict-free 8-byte loads.
//   - NVFP4 codes are decoded with integer shifts into 16-bit patterns whose value is
//     E2M1(code) * 2^-126 (bf16) or * 2^-14 (f16) and multiplied by the block scale times a
//     power of two; the product E2M1 * E4M3 * 2^-8 is exact in both 16-bit types, and the
//     epilogue multiplies the fp32 accumulator by 2^8 * tensor scales.
//   - 2:4 weights: each group's two kept values are expanded to its four k slots with two
//     byte permutes selected by the group's nibble, then the dense MMA runs.
//   - K-slices are summed into y with fp32 atomic adds (y zeroed first) when there is more
//     than one slice, else stored directly.
#include <mma.h>

#include "sp24_internal.cuh"

namespace sp24 {



namespace {

constexpr int kWarps = 4;
constexpr int kCPW = 4;  // chunks per warp (per K-slice)

template <int WF>
struct WT;
template <>
struct WT<W_D16> { static constexpr int LV = 8, STEPS = 2; };
template <>
struct WT<W_S16> { static constexpr int LV = 16, STEPS = 4; };
template <>
struct WT<W_DQ4> { static constexpr int LV = 32, STEPS = 8; };
template <>
struct WT<W_SQ4> { static constexpr int LV = 64, STEPS = 16; };

// Local k (within a lane's LV-wide piece) of A slot j (0,1 -> a_lo, 2,3 -> a_hi) at step s.
template <int WF>
__host__ __device__ __forceinline__ int kslot(int s, int j) {
  if (WF == W_DQ4) {
    int q = s >> 1, i0 = 2 * (s & 1);
    const int off[4] = {0, 4, 1, 5};
    return 8 * q + i0 + off[j];
  }
  return 4 * s + j;
}

// Byte offset of a lane's 16-byte piece of a weight row, from the piece's first logical k.
template <int WF>
__device__ __forceinline__ int64_t w_byte(int64_t k) {
  if (WF == W_D16) return k * 2;
  if (WF == W_S16) return k;      // K/2 kept 16-bit values per row
  if (WF == W_DQ4) return k / 2;
  return k / 4;                    // W_SQ4: K/2 kept 4-bit values per row
}

template <typename T>
struct Pack;
template <>
struct Pack<__nv_bfloat16> {
  // 16-bit pattern of E2M1(code) * 2^-126: magnitude bits to [6,9), sign to 15
  static constexpr uint32_t MAG = 0x01C001C0u, SGN = 0x80008000u;
  static constexpr int MAGPOS = 6;
  static constexpr float FOLD = 0x1p118f;  // block scale * 2^118 -> product E2M1*E4M3*2^-8
};
template <>
struct Pack<__half> {
  // 16-bit pattern of E2M1(code) * 2^-14: magnitude bits to [9,12), sign to 15
  static constexpr uint32_t MAG = 0x0E000E00u, SGN = 0x80008000u;
  static constexpr int MAGPOS = 9;
  static constexpr float FOLD = 0x1p6f;
};

__device__ __forceinline__ uint32_t shl(uint32_t x, int n) { return n >= 0 ? x << n : x >> (-n); }

// Nibbles i and i+4 of word w (entries 8q+i, 8q+i+4 of the piece) -> 16-bit pair (lo, hi).
template <typename T>
__device__ __forceinline__ uint32_t nib_pair_i4(uint32_t w, int i) {
  return (shl(w, Pack<T>::MAGPOS - 4 * i) & Pack<T>::MAG) | (shl(w, 12 - 4 * i) & Pack<T>::SGN);
}

// Byte bb of word w (two consecutive entries) -> 16-bit pair (lo nibble, hi nibble).
template <typename T>
__device__ __forceinline__ uint32_t nib_pair_byte(uint32_t w, int bb) {
  uint32_t x = w >> (8 * bb);
  constexpr int P = Pack<T>::MAGPOS;
  return ((x << P) & (7u << P)) | ((x << 12) & 0x8000u) | ((x << (P + 12)) & (7u << (P + 16))) |
         ((x << 24) & 0x80000000u);
}

template <typename T>
__device__ __forceinline__ uint32_t mul2(uint32_t a, uint32_t s2) {
  if constexpr (sizeof(T) == 2 && std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&s2));
    return *reinterpret_cast<uint32_t*>(&r);
  } else {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&s2));
    return *reinterpret_cast<uint32_t*>(&r);
  }
}

// Block-scale multiplier (both halves) for a 16-bit type: E4M3(code) * FOLD, exact.
template <typename T>
__device__ __forceinline__ uint32_t scale2(uint32_t code) {
  uint32_t h2;
  uint16_t c = (uint16_t)code;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  float f = __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu))) * Pack<T>::FOLD;
  uint16_t b;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat16 v = __float2bfloat16_rn(f);
    b = *reinterpret_cast<uint16_t*>(&v);
  } else {
    __half v = __float2half_rn(f);
    b = *reinterpret_cast<uint16_t*>(&v);
  }
  return (uint32_t)b | ((uint32_t)b << 16);
}

template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

template <typename T>
__device__ __forceinline__ uint16_t f32_to_bits(float f) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat16 v = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&v);
  } else {
    __half v = __float2half_rn(f);
    return *reinterpret_cast<uint16_t*>(&v);
  }
}

// x[n, k] as 16-bit bits of type T (0 outside the matrix).  NVFP4 x is decoded to
// E2M1 * E4M3 (exact in T); its tensor scale is applied in the epilogue.
template <typename T>
__device__ __forceinline__ uint32_t x_bits(const SkinnyParams& p, int64_t n, int64_t k) {
  if (n >= p.M || k >= p.K) return 0;
  if (p.x_fmt == X_16) return reinterpret_cast<const uint16_t*>(p.x)[n * p.K + k];
  const uint8_t* codes = reinterpret_cast<const uint8_t*>(p.x);
  uint32_t c = (codes[(n * p.K + k) >> 1] >> (4 * (k & 1))) & 0xf;
  uint32_t mag = c & 7, e = mag >> 1, m = mag & 1;
  float a = e == 0 ? 0.5f * m : (float)(1 << (e - 1)) * (1.0f + 0.5f * m);
  uint32_t h2;
  uint16_t sc = p.x_scales[(n * p.K + k) >> 4];
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(sc));
  float v = a * __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
  return f32_to_bits<T>(c & 8 ? -v : v);
}

template <int WF, typename T, int NT>
__global__ void __launch_bounds__(kWarps * 32) skinny_kernel(const SkinnyParams p) {
  constexpr int LV = WT<WF>::LV, STEPS = WT<WF>::STEPS, CHUNK = 4 * LV;
  extern __shared__ __align__(16) uint2 xs[];  // [kCPW][STEPS][NT][32] 8-byte fragments
  __shared__ uint32_t lut[16];                  // 2:4 expansion selectors per nibble

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int chunk0 = blockIdx.y * kCPW;
  const int nchunks = min(kCPW, p.chunks_total - chunk0);
  const int64_t kbase = (int64_t)chunk0 * CHUNK;

  if (WF == W_S16 || WF == W_SQ4) {
    if (threadIdx.x < 16) {
      uint32_t i0 = threadIdx.x & 3, i1 = threadIdx.x >> 2;
      auto sel = [&](uint32_t i) -> uint32_t { return i == i0 ? 0x10u : (i == i1 ? 0x32u : 0x54u); };
      uint32_t ok = i0 < i1;
      uint32_t s01 = ok ? (sel(0) | (sel(1) << 8)) : 0x5454u;
      uint32_t s23 = ok ? (sel(2) | (sel(3) << 8)) : 0x5454u;
      lut[threadIdx.x] = s01 | (s23 << 16);
    }
  }

  // ---- issue the weight loads for the whole slice
  const int64_t r0 = (int64_t)blockIdx.x * (kWarps * 16) + warp * 16 + g, r1 = r0 + 8;
  uint4 raw[kCPW][2];
  uint32_t sraw[kCPW][2];   // NVFP4: two scale bytes per row piece
  uint2 mraw[kCPW][2];      // 2:4: nibbles of the row piece (4 or 16 groups)
#pragma unroll
  for (int ci = 0; ci < kCPW; ++ci) {
    const int64_t k = kbase + (int64_t)ci * CHUNK + LV * c;
    const bool kv = ci < nchunks && k < p.K;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t r = h ? r1 : r0;
      const bool v = kv && r < p.N;
      raw[ci][h] = v ? ldg_stream16(p.w + r * p.w_row_bytes + w_byte<WF>(k)) : make_uint4(0, 0, 0, 0);
      if (WF == W_DQ4)
        sraw[ci][h] = v ? *reinterpret_cast<const uint16_t*>(p.w_scales + r * p.scale_row_bytes + k / 16) : 0u;
      if (WF == W_SQ4)
        sraw[ci][h] = v ? *reinterpret_cast<const uint16_t*>(p.w_scales + r * p.scale_row_bytes + k / 32) : 0u;
      if (WF == W_S16) {
        uint32_t m = v ? *reinterpret_cast<const uint16_t*>(p.meta + r * p.meta_row_bytes + k / 8) : 0x4444u;
        mraw[ci][h] = make_uint2(m, 0);
      }
      if (WF == W_SQ4)
        mraw[ci][h] = v ? *reinterpret_cast<const uint2*>(p.meta + r * p.meta_row_bytes + k / 8) : make_uint2(0x44444444u, 0x44444444u);
    }
  }

  // ---- stage x for the slice in fragment order
  const int entries = nchunks * STEPS * NT * 32;
  for (int e = threadIdx.x; e < entries; e += blockDim.x) {
    const int ln = e & 31, t = (e >> 5) % NT, s = (e / (32 * NT)) % STEPS, ci = e / (32 * NT * STEPS);
    const int gg = ln >> 2, cc = ln & 3;
    const int64_t n = 8 * t + gg;
    const int64_t kp = kbase + (int64_t)ci * CHUNK + LV * cc;
    uint32_t v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = x_bits<T>(p, n, kp + kslot<WF>(s, j));
    xs[e] = make_uint2(v[0] | (v[1] << 16), v[2] | (v[3] << 16));
  }
  __syncthreads();

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

#pragma unroll
  for (int ci = 0; ci < kCPW; ++ci) {
    if (ci >= nchunks) break;
    uint32_t sc[2][2];
    if (WF == W_DQ4 || WF == W_SQ4) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        sc[h][0] = scale2<T>(sraw[ci][h] & 0xffu);
        sc[h][1] = scale2<T>((sraw[ci][h] >> 8) & 0xffu);
      }
    }
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
      uint32_t alo[2], ahi[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 rw = raw[ci][h];
        const uint32_t words[4] = {rw.x, rw.y, rw.z, rw.w};
        if (WF == W_D16) {
          alo[h] = words[2 * s];
          ahi[h] = words[2 * s + 1];
        } else if (WF == W_DQ4) {
          const uint32_t wq = words[s >> 1];
          const int i0 = 2 * (s & 1);
          const uint32_t s2 = sc[h][s >> 2];
          alo[h] = mul2<T>(nib_pair_i4<T>(wq, i0), s2);
          ahi[h] = mul2<T>(nib_pair_i4<T>(wq, i0 + 1), s2);
        } else {
          uint32_t kept, nib;
          if (WF == W_S16) {
            kept = words[s];
            nib = (mraw[ci][h].x >> (4 * s)) & 0xf;
          } else {
            kept = mul2<T>(nib_pair_byte<T>(words[s >> 2], s & 3), sc[h][s >> 3]);
            const uint32_t mw = (s < 8) ? mraw[ci][h].x : mraw[ci][h].y;
            nib = (mw >> (4 * (s & 7))) & 0xf;
          }
          const uint32_t sel = lut[nib];
          alo[h] = __byte_perm(kept, 0u, sel & 0xffffu);
          ahi[h] = __byte_perm(kept, 0u, sel >> 16);
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint2 b = xs[((ci * STEPS + s) * NT + t) * 32 + lane];
        mma16816<T>(acc[t], alo[0], alo[1], ahi[0], ahi[1], b.x, b.y);
      }
    }
  }

  // ---- epilogue: rows r0 / r1, tokens 8t + 2c, 8t + 2c + 1
  float scale = 1.0f;
  if (WF == W_DQ4 || WF == W_SQ4) scale = 256.0f * *p.w_ts;
  if (p.x_fmt == X_Q4) scale *= *p.x_ts;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t n = 8 * t + 2 * c + (q & 1);
      const int64_t r = (q & 2) ? r1 : r0;
      if (n < p.M && r < p.N) {
        float* dst = p.y + n * p.N + r;
        const float v = acc[t][q] * scale;
        if (p.accumulate) atomicAdd(dst, v);
        else *dst = v;
      }
    }
  }
}

template <int WF, typename T>
int launch_nt(const SkinnyParams& p, int nt, cudaStream_t s) {
  constexpr int STEPS = WT<WF>::STEPS;
  dim3 grid((unsigned)((p.N + kWarps * 16 - 1) / (kWarps * 16)), (unsigned)((p.chunks_total + kCPW - 1) / kCPW));
  dim3 block(kWarps * 32);
  size_t smem = (size_t)kCPW * STEPS * nt * 32 * sizeof(uint2);
#define SP24_LAUNCH(NTV)                                                                           \
  {                                                                                                \
    auto kern = skinny_kernel<WF, T, NTV>;                                                         \
    if (smem > 48 * 1024 &&                                                                        \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return SP24_ERR_CUDA;                                                                        \
    kern<<<grid, block, smem, s>>>(p);                                                             \
  }
  switch (nt) {
    case 1: SP24_LAUNCH(1) break;
    case 2: SP24_LAUNCH(2) break;
    case 4: SP24_LAUNCH(4) break;
    case 8: SP24_LAUNCH(8) break;
    default: return SP24_ERR_UNSUPPORTED;
  }
#undef SP24_LAUNCH
  return launch_status();
}

}  // namespace

// Host launcher for the skinny path.  wf: one of W_*; t16: SP24_F16 or SP24_BF16 (the MMA type).
int skinny_gemm(int wf, int t16, SkinnyParams p, cudaStream_t s) {
  if (p.M > 64) return SP24_ERR_UNSUPPORTED;
  int lv = wf == W_D16 ? 8 : wf == W_S16 ? 16 : wf == W_DQ4 ? 32 : 64;
  int chunk = 4 * lv;
  p.chunks_total = (int)((p.K + chunk - 1) / chunk);
  const int nt = p.M <= 8 ? 1 : p.M <= 16 ? 2 : p.M <= 32 ? 4 : 8;
  const int slices = (p.chunks_total + kCPW - 1) / kCPW;
  p.accumulate = slices > 1;
  if (p.accumulate && cudaMemsetAsync(p.y, 0, (size_t)(p.M * p.N) * sizeof(float), s) != cudaSuccess)
    return SP24_ERR_CUDA;
  if (p.chunks_total == 0) {
    return cudaMemsetAsync(p.y, 0, (size_t)(p.M * p.N) * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  }
  const bool bf = t16 == SP24_BF16;
  switch (wf) {
    case W_D16: return bf ? launch_nt<W_D16, __nv_bfloat16>(p, nt, s) : launch_nt<W_D16, __half>(p, nt, s);
    case W_S16: return bf ? launch_nt<W_S16, __nv_bfloat16>(p, nt, s) : launch_nt<W_S16, __half>(p, nt, s);
    case W_DQ4: return bf ? launch_nt<W_DQ4, __nv_bfloat16>(p, nt, s) : launch_nt<W_DQ4, __half>(p, nt, s);
    case W_SQ4: return bf ? launch_nt<W_SQ4, __nv_bfloat16>(p, nt, s) : launch_nt<W_SQ4, __half>(p, nt, s);
  }
  return SP24_ERR_UNSUPPORTED;
}

}  // namespace sp24
