// a3: NVFP4 block quantisation and its decode.
//
// [P5] "NVFP4 Without FP4 Hardware", sections "Convert BF16 to NVFP4 yourself" (4-bit E2M1
// values, one E4M3 scale per 16 values, one fp32 global scale per tensor) and "The shared
// global scale" (one scale shared by a group of tensors, taken from the max absolute value).
//
// Two HBM-bound passes: (1) amax of |T| into a scratch word (warp/block max, one atomicMax
// per block on the float's bit pattern, which orders non-negative floats); (2) encode: one
// thread per 16-entry block, 32 bytes (16-bit input) read and 9 bytes written.  Every scale
// and code decision is an IEEE fp32 operation with round-to-nearest-even, written with the
// explicit __fdiv_rn / __fmul_rn intrinsics so no contraction or approximation can change a
// rounding; the E4M3 and E2M1 roundings use the hardware's RNE + satfinite conversions.
#include "sp24_internal.cuh"
#include "sp24_stream.cuh"

namespace sp24 {
namespace {

constexpr int kThreads = 256;

template <int DT>
__device__ __forceinline__ float to_f32(uint32_t bits16) {
  if (DT == SP24_BF16) return __uint_as_float(bits16 << 16);
  return __half2float(__ushort_as_half((unsigned short)bits16));
}

// 16 entries of a block as fp32 (exact: f16 and bf16 embed in fp32).
template <int DT>
__device__ __forceinline__ void load_block(const void* t, int64_t blk, float (&v)[16]) {
  if (DT == SP24_F32) {
    const uint4* p = reinterpret_cast<const uint4*>(t) + blk * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 x = ldg_stream16(p + q);
      v[4 * q + 0] = __uint_as_float(x.x);
      v[4 * q + 1] = __uint_as_float(x.y);
      v[4 * q + 2] = __uint_as_float(x.z);
      v[4 * q + 3] = __uint_as_float(x.w);
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(t) + blk * 2;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint4 x = ldg_stream16(p + q);
      uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * q + 2 * i] = to_f32<DT>(w[i] & 0xffffu);
        v[8 * q + 2 * i + 1] = to_f32<DT>(w[i] >> 16);
      }
    }
  }
}

// E4M3 code of x >= 0: round to nearest even, values beyond 448 saturate to 448.
__device__ __forceinline__ uint32_t e4m3_rne_satfinite(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xffu;  // the second source lands in the low byte
}

// fp32 value of an E4M3 code (exact).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  uint16_t c = (uint16_t)code;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// Two E2M1 magnitude codes (x_lo, x_hi >= 0) packed as lo | hi << 4, RNE, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x2_rne_satfinite(float x_lo, float x_hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(x_hi), "f"(x_lo));
  return r & 0xffu;
}

// Streaming ring: 3 stages of 16 KB per CTA (512 blocks of 16 16-bit entries, or 256 fp32).
constexpr int kChunk = 16384, kStages = 2;  // 32 KB per CTA (+ 8 KB of threshold tables): four CTAs per SM
constexpr size_t kRingBytes = (size_t)kChunk * kStages;

// 16 entries of a block from shared memory as fp32.
template <int DT>
__device__ __forceinline__ void smem_block(const uint8_t* p, float (&v)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  if (DT == SP24_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x = q[i];
      v[4 * i + 0] = __uint_as_float(x.x);
      v[4 * i + 1] = __uint_as_float(x.y);
      v[4 * i + 2] = __uint_as_float(x.z);
      v[4 * i + 3] = __uint_as_float(x.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 x = q[i];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[8 * i + 2 * k] = to_f32<DT>(w[k] & 0xffffu);
        v[8 * i + 2 * k + 1] = to_f32<DT>(w[k] >> 16);
      }
    }
  }
}

template <int DT>
constexpr int block_bytes() { return DT == SP24_F32 ? 64 : 32; }

template <int DT>
__global__ void __launch_bounds__(kThreads, 4) amax_kernel(const void* __restrict__ t, int64_t nblk,
                                                        unsigned int* __restrict__ amax_bits) {
  extern __shared__ __align__(128) uint8_t ring[];
  constexpr int BB = block_bytes<DT>();
  float m = 0.0f;
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(t), nblk * BB, ring, [&](const uint8_t* chunk, int64_t, int bytes) {
        // any 16-byte vector order will do for a max: consecutive threads, consecutive vectors
        const uint4* cv = reinterpret_cast<const uint4*>(chunk);
        const int nvec = bytes / 16;
#pragma unroll
        for (int q = 0; q < kChunk / 16 / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          if (j >= nvec) continue;
          const uint4 x = cv[j];
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (DT == SP24_F32) {
              m = fmaxf(m, fabsf(__uint_as_float(w[k])));
            } else {
              m = fmaxf(m, fabsf(to_f32<DT>(w[k] & 0xffffu)));
              m = fmaxf(m, fabsf(to_f32<DT>(w[k] >> 16)));
            }
          }
        }
      });
  unsigned int u = __float_as_uint(m);
  u = __reduce_max_sync(0xffffffffu, u);
  __shared__ unsigned int wmax[kThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = u;
  __syncthreads();
  if (threadIdx.x < 32) {
    unsigned int x = threadIdx.x < kThreads / 32 ? wmax[threadIdx.x] : 0u;
    x = __reduce_max_sync(0xffffffffu, x);
    if (threadIdx.x == 0 && x) atomicMax(amax_bits, x);
  }
}

// Encodes one 16-entry block given the tensor scale s_t and d = s_t * 6.
//
// The code of an entry is E2M1_rne(fl(|v| / sc)), and only the side of fl(|v| / sc) relative to
// E2M1's rounding boundaries (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) matters.  With the block's
// divisor sc in [2^-100, 2^100], q = RN(|v| * RN(1 / sc)) is within 2.01 ulp of |v| / sc (two
// roundings of 2^-24 each), so q and fl(|v| / sc) give the same code unless q lies within a few
// ulps of a boundary.  Every boundary is a multiple of 0.25: rounding q to the nearest multiple
// of 0.25 (adding and subtracting 2^21 in fp32) and testing |q - that| < q * 2^-21 (a window of
// 4 to 8 ulps of q; never true for q = 0) flags every such q.  A pair with a flagged entry takes
// the IEEE division for both entries.  The codes are therefore exactly those of the per-entry
// division, at a multiply and four FMA-pipe operations per entry.
__device__ __forceinline__ bool near_quarter(float q) {
  const float r = __fadd_rn(__fadd_rn(q, 0x1p21f), -0x1p21f);   // nearest multiple of 0.25
  return __fmaf_rn(q, 0x1p-21f, -fabsf(__fadd_rn(q, -r))) > 0.0f;
}

__device__ __forceinline__ void encode_block(const float (&v)[16], float s_t, float d, uint2* codes,
                                             uint8_t* scales, int64_t b) {
  float bmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
  uint32_t sb = d != 0.0f ? e4m3_rne_satfinite(__fdiv_rn(bmax, d)) : 0u;
  const float sc = __fmul_rn(e4m3_value(sb), s_t);
  const bool fast = sc >= 0x1p-100f && sc <= 0x1p100f;
  const float y = __frcp_rn(sc);
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float a0 = fabsf(v[i]), a1 = fabsf(v[i + 1]);
    float q0, q1;
    if (fast) {
      q0 = __fmul_rn(a0, y);
      q1 = __fmul_rn(a1, y);
      if (near_quarter(q0) || near_quarter(q1)) {
        q0 = __fdiv_rn(a0, sc);  // within 4 ulp of a multiple of 0.25
        q1 = __fdiv_rn(a1, sc);
      }
    } else {
      q0 = sc != 0.0f ? __fdiv_rn(a0, sc) : 0.0f;
      q1 = sc != 0.0f ? __fdiv_rn(a1, sc) : 0.0f;
    }
    uint32_t byte = e2m1x2_rne_satfinite(q0, q1);
    byte |= (__float_as_uint(v[i]) >> 31) << 3;       // sign of the low entry
    byte |= (__float_as_uint(v[i + 1]) >> 31) << 7;   // sign of the high entry
    packed[i / 8] |= byte << (8 * ((i % 8) / 2));
  }
  codes[b] = make_uint2(packed[0], packed[1]);
  scales[b] = (uint8_t)sb;
}

// ---- 16-bit inputs: codes by counting thresholds, no per-entry division.
//
// fl32(a / sc) rounds (RNE, saturating) to an E2M1 code above j exactly when a / sc > T_j, with
// T_j the boundary between codes j and j + 1 moved half an fp32 ulp to the side its tie goes:
// away from the odd code (0.25, 1.25, 2.5 and 5 round down on a tie, 0.75, 1.75 and 3.5 up).
// a / sc never equals T_j (T_j has more significant bits than any ratio of two fp32 values can
// produce), so for a 16-bit a the test is a >= RU16(T_j * sc), where T_j * sc is exact in fp64.
// Each CTA tabulates the seven 16-bit thresholds for every E4M3 block-scale code (a zero
// divisor gets NaN thresholds: every compare fails, code 0), and an entry's code is the number
// of thresholds it reaches, counted two entries at a time with packed compares and adds.
__constant__ double kE2M1Bound[7] = {0.25 + 0x1p-26, 0.75 - 0x1p-25, 1.25 + 0x1p-24, 1.75 - 0x1p-24,
                                     2.5 + 0x1p-23,  3.5 - 0x1p-23,  5.0 + 0x1p-22};

template <int DT>
struct Pack16;
template <>
struct Pack16<SP24_BF16> {
  static constexpr uint32_t BIAS = 0x43004300u;  // 128.0 twice: 128 + k has k in its low byte
  static constexpr uint32_t QNAN = 0x7FC07FC0u;
};
template <>
struct Pack16<SP24_F16> {
  static constexpr uint32_t BIAS = 0x64006400u;  // 1024.0 twice
  static constexpr uint32_t QNAN = 0x7E007E00u;
};

template <int DT>
__device__ __forceinline__ uint32_t ge2(uint32_t a, uint32_t b) {  // 1.0 / 0.0 per half
  uint32_t r;
  if (DT == SP24_BF16) asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else asm("set.ge.f16x2.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <int DT>
__device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
  uint32_t r;
  if (DT == SP24_BF16) asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <int DT>
__device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) {  // NaN loses, as in fmaxf
  uint32_t r;
  if (DT == SP24_BF16) asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// Smallest 16-bit value of type DT at or above x (x exact in fp64; rounding up twice is rounding
// up once).
template <int DT>
__device__ __forceinline__ uint32_t ru16(double x) {
  const float f = __double2float_ru(x);
  if (DT == SP24_BF16) return __bfloat16_as_ushort(__float2bfloat16_ru(f));
  return __half_as_ushort(__float2half_ru(f));
}

// tab[8 c + j] = threshold j of block-scale code c, in both halves (j = 7 unused).
template <int DT>
__device__ void build_thresholds(float s_t, uint32_t* tab) {
  for (int i = threadIdx.x; i < 128 * 8; i += blockDim.x) {
    const int c = i >> 3, j = i & 7;
    uint32_t v = Pack16<DT>::QNAN;
    if (j < 7 && c < 127) {
      const float sc = __fmul_rn(e4m3_value(c), s_t);
      if (sc != 0.0f) {
        const uint32_t h = ru16<DT>(kE2M1Bound[j] * (double)sc);
        v = h | (h << 16);
      }
    }
    tab[i] = v;
  }
}

// Encodes one block of 16 16-bit entries (32 bytes at p) with the thresholds of its scale code.
template <int DT>
__device__ __forceinline__ void encode_block16(const uint8_t* p, const uint32_t* tab, float d, uint2* codes,
                                               uint8_t* scales, int64_t b) {
  const uint4 u0 = reinterpret_cast<const uint4*>(p)[0], u1 = reinterpret_cast<const uint4*>(p)[1];
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
  uint32_t a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = w[i] & 0x7fff7fffu;
  const uint32_t m = max2<DT>(max2<DT>(max2<DT>(a[0], a[1]), max2<DT>(a[2], a[3])),
                              max2<DT>(max2<DT>(a[4], a[5]), max2<DT>(a[6], a[7])));
  const float bmax = fmaxf(to_f32<DT>(m & 0xffffu), to_f32<DT>(m >> 16));
  const uint32_t sb = d != 0.0f ? e4m3_rne_satfinite(__fdiv_rn(bmax, d)) : 0u;
  const uint4 t0 = reinterpret_cast<const uint4*>(tab + 8 * sb)[0];
  const uint4 t1 = reinterpret_cast<const uint4*>(tab + 8 * sb)[1];
  const uint32_t th[7] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z};
  // per pair of entries: the count starts at BIAS plus 8 for a negative entry, so the low byte of
  // each half ends as the entry's 4-bit code (sign << 3 | magnitude code)
  uint32_t nib[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t acc = ((w[i] >> 12) & 0x00080008u) | Pack16<DT>::BIAS;
#pragma unroll
    for (int j = 0; j < 7; ++j) acc = add2<DT>(acc, ge2<DT>(a[i], th[j]));
    nib[i] = acc;
  }
  // four pairs per code word: gather the low bytes of both halves, fold each byte pair into one
  // byte (high entry in the high nibble), gather again
  uint32_t packed[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t p0 = __byte_perm(nib[4 * k], nib[4 * k + 1], 0x6420);
    const uint32_t p1 = __byte_perm(nib[4 * k + 2], nib[4 * k + 3], 0x6420);
    packed[k] = __byte_perm(p0 | (p0 >> 4), p1 | (p1 >> 4), 0x6420);
  }
  codes[b] = make_uint2(packed[0], packed[1]);
  scales[b] = (uint8_t)sb;
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 4) encode_kernel(const void* __restrict__ t, int64_t nblk,
                                                          const float* __restrict__ ts_in,
                                                          const unsigned int* __restrict__ amax_bits,
                                                          uint2* __restrict__ codes,
                                                          uint8_t* __restrict__ scales,
                                                          float* __restrict__ ts_out) {
  extern __shared__ __align__(128) uint8_t ring[];
  constexpr int BB = block_bytes<DT>();
  // tensor scale: supplied, or amax / 2688 (2688 = 6 * 448)
  const float s_t = ts_in ? *ts_in : __fdiv_rn(__uint_as_float(*amax_bits), 2688.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *ts_out = s_t;
  const float d = __fmul_rn(s_t, 6.0f);
  __shared__ __align__(16) uint32_t tab[DT == SP24_F32 ? 4 : 128 * 8];
  if constexpr (DT != SP24_F32) build_thresholds<DT>(s_t, tab);  // published by the ring's first barrier
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(t), nblk * BB, ring, [&](const uint8_t* chunk, int64_t c, int bytes) {
        const int nb = bytes / BB;
        const int64_t b0 = c * (kChunk / BB);
#pragma unroll
        for (int q = 0; q < kChunk / BB / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          if (j >= nb) continue;
          if constexpr (DT == SP24_F32) {
            float v[16];
            smem_block<DT>(chunk + j * BB, v);
            encode_block(v, s_t, d, codes, scales, b0 + j);
          } else {
            encode_block16<DT>(chunk + j * BB, tab, d, codes, scales, b0 + j);
          }
        }
      });
}

// Encode pass over two tensors in one launch, each with its supplied tensor scale.
struct EncodeJob {
  const void* t;
  int64_t nblk;
  const float* ts_in;
  uint2* codes;
  uint8_t* scales;
  float* ts_out;
};

template <int DT>
__global__ void __launch_bounds__(kThreads, 4) encode_pair_kernel(EncodeJob ja, EncodeJob jb) {
  extern __shared__ __align__(128) uint8_t ring[];
  constexpr int BB = block_bytes<DT>();
  const float s_a = *ja.ts_in, s_b = *jb.ts_in;
  __syncthreads();  // every thread has read the scales before ts_out (which may alias) is written
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *ja.ts_out = s_a;
    *jb.ts_out = s_b;
  }
  const float d_a = __fmul_rn(s_a, 6.0f), d_b = __fmul_rn(s_b, 6.0f);
  __shared__ __align__(16) uint32_t tab[2][DT == SP24_F32 ? 4 : 128 * 8];
  if constexpr (DT != SP24_F32) {  // published by the ring's first barrier
    build_thresholds<DT>(s_a, tab[0]);
    build_thresholds<DT>(s_b, tab[1]);
  }
  stream::for_each_chunk2<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(ja.t), ja.nblk * BB, reinterpret_cast<const uint8_t*>(jb.t),
      jb.nblk * BB, ring, [&](const uint8_t* chunk, int seg, int64_t c, int bytes) {
        const int nb = bytes / BB;
        const int64_t b0 = c * (kChunk / BB);
        uint2* codes = seg ? jb.codes : ja.codes;
        uint8_t* scales = seg ? jb.scales : ja.scales;
        const float s_t = seg ? s_b : s_a, d = seg ? d_b : d_a;
#pragma unroll
        for (int q = 0; q < kChunk / BB / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          if (j >= nb) continue;
          if constexpr (DT == SP24_F32) {
            float v[16];
            smem_block<DT>(chunk + j * BB, v);
            encode_block(v, s_t, d, codes, scales, b0 + j);
          } else {
            encode_block16<DT>(chunk + j * BB, tab[seg], d, codes, scales, b0 + j);
          }
        }
      });
}

// One byte (two entries) per thread; value computed in fp64 (exact) and rounded once.
template <int OUT>
__global__ void __launch_bounds__(kThreads) decode_kernel(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ scales,
                                                          const float* __restrict__ ts,
                                                          int64_t nbytes, void* __restrict__ out) {
  const double s_t = (double)*ts;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbytes; i += stride) {
    uint32_t byte = codes[i];
    double sb = (double)e4m3_value(scales[i / 8]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t c = (byte >> (4 * h)) & 0xf;
      uint32_t mag = c & 7, e = mag >> 1, m = mag & 1;
      double a = e == 0 ? 0.5 * m : (double)(1 << (e - 1)) * (1.0 + 0.5 * m);
      double val = (c & 8 ? -a : a) * sb * s_t;
      int64_t idx = 2 * i + h;
      if (OUT == SP24_F32) reinterpret_cast<float*>(out)[idx] = (float)val;
      else if (OUT == SP24_BF16) reinterpret_cast<__nv_bfloat16*>(out)[idx] = __double2bfloat16(val);
      else reinterpret_cast<__half*>(out)[idx] = __double2half(val);
    }
  }
}

int64_t blocks_for(int64_t items) { return (items + kThreads - 1) / kThreads; }

// Grid of a streaming kernel over `bytes` of input: one CTA per chunk, capped at a full wave
// (at least one CTA, so that the encode kernel also writes the tensor scale of an empty tensor).
template <typename Kern>
int ring_grid(Kern k, int64_t bytes) {
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingBytes);
  return full_wave_grid(k, kThreads, (bytes + kChunk - 1) / kChunk, kRingBytes);
}

// ---- 32-entry blocks: the activation form the sparse FP4 MMA reads (one scale per 32 K).
// The same steps as the 16-entry encoder over 32 entries: bmax, sb = E4M3(bmax / (6 s_t)),
// code = E2M1(|t| / (E4M3(sb) s_t)), every step an IEEE fp32 operation (the per-entry division
// is __fdiv_rn, then the hardware's RNE + satfinite conversion).  One thread per block, grid-
// stride; the tensor is an activation (small next to the weights), so the plain division is
// affordable here.
template <int DT>
__global__ void __launch_bounds__(kThreads) encode32_kernel(const void* __restrict__ t, int64_t nblk,
                                                            const float* __restrict__ ts_in,
                                                            const unsigned int* __restrict__ amax_bits,
                                                            uint4* __restrict__ codes, uint8_t* __restrict__ scales,
                                                            float* __restrict__ ts_out) {
  const float s_t = ts_in ? *ts_in : __fdiv_rn(__uint_as_float(*amax_bits), 2688.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *ts_out = s_t;
  const float d = __fmul_rn(s_t, 6.0f);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
    float v[32];
    load_block<DT>(t, 2 * b, *reinterpret_cast<float(*)[16]>(&v[0]));
    load_block<DT>(t, 2 * b + 1, *reinterpret_cast<float(*)[16]>(&v[16]));
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
    const uint32_t sb = d != 0.0f ? e4m3_rne_satfinite(__fdiv_rn(bmax, d)) : 0u;
    const float sc = __fmul_rn(e4m3_value(sb), s_t);
    uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float q0 = sc != 0.0f ? __fdiv_rn(fabsf(v[i]), sc) : 0.0f;
      const float q1 = sc != 0.0f ? __fdiv_rn(fabsf(v[i + 1]), sc) : 0.0f;
      uint32_t byte = e2m1x2_rne_satfinite(q0, q1);
      byte |= (__float_as_uint(v[i]) >> 31) << 3;
      byte |= (__float_as_uint(v[i + 1]) >> 31) << 7;
      packed[i / 8] |= byte << (8 * ((i % 8) / 2));
    }
    codes[b] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    scales[b] = (uint8_t)sb;
  }
}

constexpr int64_t kQuantWorkspace = 256;

}  // namespace

// Shared by the quantisation entry points: validates and launches amax (unless a tensor
// scale is supplied) and encode.  `amax_word` is 4 bytes of zero-initialisable scratch.
int quantize_nvfp4_launch(const void* t, int dtype, int64_t rows, int64_t cols,
                          const float* ts_in, uint8_t* codes, uint8_t* scales, float* ts_out,
                          unsigned int* amax_word, cudaStream_t s) {
  int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  if (rows < 0 || cols < 0 || cols % 16) return SP24_ERR_SHAPE;
  if (!ts_out) return SP24_ERR_INVALID_ARG;
  const int64_t nblk = rows * cols / 16;
  if (nblk > 0 && (!t || !codes || !scales)) return SP24_ERR_INVALID_ARG;
  if (nblk > 0 && (!aligned(t, 16) || !aligned(codes, 8))) return SP24_ERR_ALIGN;
  int nl = 1;  // encode always runs
  if (!ts_in) {
    if (!amax_word) return SP24_ERR_WORKSPACE;
    if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned int), s) != cudaSuccess) return SP24_ERR_CUDA;
    if (nblk > 0) {
      if (dtype == SP24_F32) amax_kernel<SP24_F32><<<ring_grid(amax_kernel<SP24_F32>, nblk * ((SP24_F32) == SP24_F32 ? 64 : 32)), kThreads, kRingBytes, s>>>(t, nblk, amax_word);
      else if (dtype == SP24_BF16) amax_kernel<SP24_BF16><<<ring_grid(amax_kernel<SP24_BF16>, nblk * ((SP24_BF16) == SP24_F32 ? 64 : 32)), kThreads, kRingBytes, s>>>(t, nblk, amax_word);
      else amax_kernel<SP24_F16><<<ring_grid(amax_kernel<SP24_F16>, nblk * ((SP24_F16) == SP24_F32 ? 64 : 32)), kThreads, kRingBytes, s>>>(t, nblk, amax_word);
      ++nl;
    }
  }
  // launched even when nblk == 0 so that tensor_scale_out is written
  if (dtype == SP24_F32)
    encode_kernel<SP24_F32><<<ring_grid(encode_kernel<SP24_F32>, nblk * ((SP24_F32) == SP24_F32 ? 64 : 32)), kThreads, kRingBytes, s>>>(t, nblk, ts_in, amax_word, (uint2*)codes, scales, ts_out);
  else if (dtype == SP24_BF16)
    encode_kernel<SP24_BF16><<<ring_grid(encode_kernel<SP24_BF16>, nblk * ((SP24_BF16) == SP24_F32 ? 64 : 32)), kThreads, kRingBytes, s>>>(t, nblk, ts_in, amax_word, (uint2*)codes, scales, ts_out);
  else
    encode_kernel<SP24_F16><<<ring_grid(encode_kernel<SP24_F16>, nblk * ((SP24_F16) == SP24_F32 ? 64 : 32)), kThreads, kRingBytes, s>>>(t, nblk, ts_in, amax_word, (uint2*)codes, scales, ts_out);
  return launch_status(nl);
}

}  // namespace sp24

using namespace sp24;

extern "C" int sp24_quantize_nvfp4_workspace_size(int64_t rows, int64_t cols, int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || cols % 16) return SP24_ERR_SHAPE;
  *bytes = kQuantWorkspace;
  return SP24_OK;
}

extern "C" int sp24_quantize_nvfp4(const void* t, int dtype, int64_t rows, int64_t cols,
                                   const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                                   float* tensor_scale_out, void* workspace,
                                   int64_t workspace_bytes, void* stream) {
  unsigned int* amax_word = nullptr;
  if (!tensor_scale_in) {
    if (!workspace || workspace_bytes < kQuantWorkspace) return SP24_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return SP24_ERR_ALIGN;
    amax_word = reinterpret_cast<unsigned int*>(workspace);
  }
  return quantize_nvfp4_launch(t, dtype, rows, cols, tensor_scale_in, codes, scales,
                               tensor_scale_out, amax_word, as_stream(stream));
}

extern "C" int sp24_quantize_nvfp4_block32(const void* t, int dtype, int64_t rows, int64_t cols,
                                           const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                                           float* tensor_scale_out, void* workspace, int64_t workspace_bytes,
                                           void* stream) {
  const int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  if (rows < 0 || cols < 0 || cols % 32) return SP24_ERR_SHAPE;
  if (!tensor_scale_out) return SP24_ERR_INVALID_ARG;
  const int64_t nblk = rows * cols / 32;
  if (nblk > 0 && (!t || !codes || !scales)) return SP24_ERR_INVALID_ARG;
  if (nblk > 0 && (!aligned(t, 16) || !aligned(codes, 16))) return SP24_ERR_ALIGN;
  unsigned int* amax_word = nullptr;
  if (!tensor_scale_in) {
    if (!workspace || workspace_bytes < kQuantWorkspace) return SP24_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return SP24_ERR_ALIGN;
    amax_word = reinterpret_cast<unsigned int*>(workspace);
  }
  cudaStream_t s = as_stream(stream);
  int nl = 1;
  if (!tensor_scale_in) {
    if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned int), s) != cudaSuccess) return SP24_ERR_CUDA;
    if (nblk > 0) {
      const int64_t n16 = 2 * nblk, bytes = n16 * (dtype == SP24_F32 ? 64 : 32);
      if (dtype == SP24_F32)
        amax_kernel<SP24_F32><<<ring_grid(amax_kernel<SP24_F32>, bytes), kThreads, kRingBytes, s>>>(t, n16, amax_word);
      else if (dtype == SP24_BF16)
        amax_kernel<SP24_BF16><<<ring_grid(amax_kernel<SP24_BF16>, bytes), kThreads, kRingBytes, s>>>(t, n16, amax_word);
      else
        amax_kernel<SP24_F16><<<ring_grid(amax_kernel<SP24_F16>, bytes), kThreads, kRingBytes, s>>>(t, n16, amax_word);
      ++nl;
    }
  }
  // launched even when nblk == 0 so that tensor_scale_out is written
  if (dtype == SP24_F32)
    encode32_kernel<SP24_F32><<<full_wave_grid(encode32_kernel<SP24_F32>, kThreads, blocks_for(nblk)), kThreads, 0, s>>>(
        t, nblk, tensor_scale_in, amax_word, (uint4*)codes, scales, tensor_scale_out);
  else if (dtype == SP24_BF16)
    encode32_kernel<SP24_BF16><<<full_wave_grid(encode32_kernel<SP24_BF16>, kThreads, blocks_for(nblk)), kThreads, 0, s>>>(
        t, nblk, tensor_scale_in, amax_word, (uint4*)codes, scales, tensor_scale_out);
  else
    encode32_kernel<SP24_F16><<<full_wave_grid(encode32_kernel<SP24_F16>, kThreads, blocks_for(nblk)), kThreads, 0, s>>>(
        t, nblk, tensor_scale_in, amax_word, (uint4*)codes, scales, tensor_scale_out);
  return launch_status(nl);
}

extern "C" int sp24_quantize_nvfp4_pair(const void* t0, int dtype, int64_t rows0, int64_t cols0,
                                        const float* ts0, uint8_t* codes0, uint8_t* scales0, float* ts_out0,
                                        const void* t1, int64_t rows1, int64_t cols1, const float* ts1,
                                        uint8_t* codes1, uint8_t* scales1, float* ts_out1, void* stream) {
  const int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  if (rows0 < 0 || cols0 < 0 || cols0 % 16 || rows1 < 0 || cols1 < 0 || cols1 % 16) return SP24_ERR_SHAPE;
  if (!ts0 || !ts1 || !ts_out0 || !ts_out1) return SP24_ERR_INVALID_ARG;
  const int64_t n0 = rows0 * cols0 / 16, n1 = rows1 * cols1 / 16;
  if ((n0 > 0 && (!t0 || !codes0 || !scales0)) || (n1 > 0 && (!t1 || !codes1 || !scales1))) return SP24_ERR_INVALID_ARG;
  if ((n0 > 0 && (!aligned(t0, 16) || !aligned(codes0, 8))) || (n1 > 0 && (!aligned(t1, 16) || !aligned(codes1, 8))))
    return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  const EncodeJob a{t0, n0, ts0, (uint2*)codes0, scales0, ts_out0};
  const EncodeJob b{t1, n1, ts1, (uint2*)codes1, scales1, ts_out1};
  const int64_t bytes = (n0 + n1) * (dtype == SP24_F32 ? 64 : 32);
  // launched even for empty tensors, so that both tensor scales are written
  if (dtype == SP24_F32)
    encode_pair_kernel<SP24_F32><<<ring_grid(encode_pair_kernel<SP24_F32>, bytes), kThreads, kRingBytes, s>>>(a, b);
  else if (dtype == SP24_BF16)
    encode_pair_kernel<SP24_BF16><<<ring_grid(encode_pair_kernel<SP24_BF16>, bytes), kThreads, kRingBytes, s>>>(a, b);
  else
    encode_pair_kernel<SP24_F16><<<ring_grid(encode_pair_kernel<SP24_F16>, bytes), kThreads, kRingBytes, s>>>(a, b);
  return launch_status();
}

extern "C" int sp24_dequantize_nvfp4(const uint8_t* codes, const uint8_t* scales,
                                     const float* tensor_scale, int64_t rows, int64_t cols,
                                     int out_dtype, void* out, void* stream) {
  if (rows < 0 || cols < 0 || cols % 16) return SP24_ERR_SHAPE;
  if (!elem_bytes(out_dtype)) return SP24_ERR_DTYPE;
  int64_t nbytes = rows * cols / 2;
  if (nbytes == 0) return SP24_OK;
  if (!codes || !scales || !tensor_scale || !out) return SP24_ERR_INVALID_ARG;
  if (!aligned(out, elem_bytes(out_dtype))) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (out_dtype == SP24_F32)
    decode_kernel<SP24_F32><<<full_wave_grid(decode_kernel<SP24_F32>, kThreads, blocks_for(nbytes)), kThreads, 0, s>>>(codes, scales, tensor_scale, nbytes, out);
  else if (out_dtype == SP24_BF16)
    decode_kernel<SP24_BF16><<<full_wave_grid(decode_kernel<SP24_BF16>, kThreads, blocks_for(nbytes)), kThreads, 0, s>>>(codes, scales, tensor_scale, nbytes, out);
  else
    decode_kernel<SP24_F16><<<full_wave_grid(decode_kernel<SP24_F16>, kThreads, blocks_for(nbytes)), kThreads, 0, s>>>(codes, scales, tensor_scale, nbytes, out);
  return launch_status();
}
