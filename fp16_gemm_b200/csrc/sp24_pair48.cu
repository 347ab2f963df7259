// Pairwise 4:8: eligibility check, pruning + compression, decompression (matmul layout).
//
// The sparse unit of the tensor cores' packed-FP4 MMA kind is a pair of consecutive entries:
// along K, every chunk of 8 entries (four pairs) keeps two pairs, named by a 4-bit nibble
// i0 | i1 << 2 (i0 < i1).  The pruning rule carries [P1] "NVFP4 vs 2:4 sparse: where the other
// half of the petaflop went", section "What 2:4 actually is" (the largest magnitudes survive)
// over to pairs:
//   * a chunk is eligible when at most two of its pairs hold a nonzero entry (+0 and -0 are
//     zero, NaN is not);
//   * pruning keeps the two pairs of largest score |a| + |b| (the entries' fp32 magnitudes added
//     with one IEEE fp32 addition), a NaN score above every number, ties to the lower pair;
//   * values [rows, K/2] hold the kept pairs in ascending order; meta is a nibble stream, chunk
//     2c of the flat chunk sequence in the low nibble of byte c (the 2:4 stream's convention).
//
// These are HBM-bound streams like the 2:4 ones: a 16-bit chunk is one 16-byte vector (an fp32
// chunk two), each thread owns whole chunks, the input is staged through the bulk-copy ring,
// and the keep decision is made in registers.  The two chunks of a meta byte belong to
// neighbouring lanes, which meet with one shuffle.  Pointers without the vector alignment take
// a scalar kernel (one thread per meta byte).
#include "sp24_internal.cuh"
#include "sp24_stream.cuh"

#include <cuda_fp16.h>

namespace sp24 {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 16384, kStages = 3;  // 48 KB ring per CTA
constexpr size_t kRingBytes = (size_t)kChunk * kStages;

// Ordering key of a pair score s = |a| + |b| >= 0: its bit pattern (non-negative floats order
// like their bits), every NaN mapped to one key just above +inf (0x7f800000).
__device__ __forceinline__ uint32_t score_key(float s) { return min(__float_as_uint(s), 0x7f800001u); }

// Key of the pair held in one word of two 16-bit entries (lo = first entry).  The entries' fp32
// magnitudes are exact: bf16 is the top half of an fp32, f16 converts exactly.
template <int DT>
__device__ __forceinline__ uint32_t pair_key16(uint32_t w) {
  const uint32_t m = w & 0x7fff7fffu;
  if (DT == SP24_BF16) return score_key(__fadd_rn(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&m));
  return score_key(__fadd_rn(f.x, f.y));
}

__device__ __forceinline__ uint32_t pair_key32(uint32_t a, uint32_t b) {
  return score_key(__fadd_rn(fabsf(__uint_as_float(a)), fabsf(__uint_as_float(b))));
}

// Nibble i0 | i1 << 2 of the two kept pairs in the order (key descending, index ascending), as a
// tournament: 0 against 1 and 2 against 3 (ties to the lower index), then the two winners (ties
// to the 0/1 side, whose indices are lower).  The runner-up is the better of the final's loser
// and the pair the overall winner beat in its first round; in either case the candidate from the
// 0/1 side has the lower index, so it wins a tie.
__device__ __forceinline__ uint32_t keep_nibble(uint32_t k0, uint32_t k1, uint32_t k2, uint32_t k3) {
  const bool c01 = k0 >= k1, c23 = k2 >= k3;
  const uint32_t win01 = max(k0, k1), lose01 = min(k0, k1), win23 = max(k2, k3), lose23 = min(k2, k3);
  const uint32_t iw01 = c01 ? 0u : 1u, il01 = iw01 ^ 1u, iw23 = c23 ? 2u : 3u, il23 = iw23 ^ 1u;
  const bool left = win01 >= win23;
  const uint32_t first = left ? iw01 : iw23;
  const uint32_t second = left ? (lose01 >= win23 ? il01 : iw23) : (win01 >= lose23 ? iw01 : il23);
  return min(first, second) | (max(first, second) << 2);
}

// A chunk as its four pairs: 16-bit types hold a pair in one word (w[j] = e_2j | e_2j+1 << 16);
// fp32 holds it in two words (w[2j], w[2j + 1]).
template <int DT>
struct Chunk {
  uint32_t w[DT == SP24_F32 ? 8 : 4];

  __device__ __forceinline__ uint32_t key(int j) const {
    if (DT == SP24_F32) return pair_key32(w[2 * j], w[2 * j + 1]);
    return pair_key16<DT>(w[j]);
  }
  __device__ __forceinline__ int pair_nonzero(int j) const {
    if (DT == SP24_F32) return ((w[2 * j] | w[2 * j + 1]) & 0x7fffffffu) != 0;
    return (w[j] & 0x7fff7fffu) != 0;
  }
  __device__ __forceinline__ int eligible() const {
    return (pair_nonzero(0) + pair_nonzero(1) + pair_nonzero(2) + pair_nonzero(3)) <= 2;
  }
  __device__ __forceinline__ uint32_t nibble() const { return keep_nibble(key(0), key(1), key(2), key(3)); }
};

template <int DT>
constexpr int chunk_bytes() {
  return DT == SP24_F32 ? 32 : 16;
}

template <int DT>
__device__ __forceinline__ Chunk<DT> load_chunk(const uint4* p) {
  Chunk<DT> c;
  const uint4 a = p[0];
  c.w[0] = a.x, c.w[1] = a.y, c.w[2] = a.z, c.w[3] = a.w;
  if (DT == SP24_F32) {
    const uint4 b = p[1];
    c.w[4] = b.x, c.w[5] = b.y, c.w[6] = b.z, c.w[7] = b.w;
  }
  return c;
}

__device__ __forceinline__ void count_fails(int fails, int32_t* n_fail) {
  if (!n_fail) return;
  const int s = __reduce_add_sync(0xffffffffu, fails);
  if ((threadIdx.x & 31) == 0 && s) atomicAdd(n_fail, s);
}

// ------------------------------------------------------------------ vector path

// Chunk v of the stage is chunk c * kPer + j of the tensor; kPer and kThreads are even, so v has
// the parity of threadIdx.x and the other chunk of v's meta byte is in lane ^ 1.
template <int DT>
__global__ void __launch_bounds__(kThreads, 4) check48_vec(const uint4* __restrict__ w, int64_t n_chunks,
                                                        uint8_t* __restrict__ pass, int32_t* __restrict__ n_fail) {
  extern __shared__ __align__(128) uint8_t ring[];
  constexpr int CB = chunk_bytes<DT>(), kPer = kChunk / CB;
  int fails = 0;
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(w), n_chunks * CB, ring, [&](const uint8_t* stage, int64_t c, int bytes) {
        const int n = bytes / CB;
#pragma unroll
        for (int q = 0; q < kPer / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          if (j >= n) continue;
          const int ok = load_chunk<DT>(reinterpret_cast<const uint4*>(stage + (size_t)j * CB)).eligible();
          fails += 1 - ok;
          pass[c * kPer + j] = (uint8_t)ok;
        }
      });
  count_fails(fails, n_fail);
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 4) prune48_vec(const uint4* __restrict__ w, int64_t n_chunks,
                                                        void* __restrict__ values, uint8_t* __restrict__ meta) {
  extern __shared__ __align__(128) uint8_t ring[];
  constexpr int CB = chunk_bytes<DT>(), kPer = kChunk / CB;
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(w), n_chunks * CB, ring, [&](const uint8_t* stage, int64_t c, int bytes) {
        const int n = bytes / CB;
#pragma unroll
        for (int q = 0; q < kPer / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          const bool live = j < n;
          Chunk<DT> ch;
          if (live) {
            ch = load_chunk<DT>(reinterpret_cast<const uint4*>(stage + (size_t)j * CB));
          } else {
#pragma unroll
            for (int i = 0; i < (DT == SP24_F32 ? 8 : 4); ++i) ch.w[i] = 0;
          }
          const uint32_t nib = ch.nibble();
          const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
          if (!live) continue;
          const int64_t v = c * kPer + j;
          const uint32_t i0 = nib & 3u, i1 = nib >> 2;
          if (DT == SP24_F32) {
            // pair i0 is one of 0..2, pair i1 one of 1..3
            const uint32_t a0 = i0 == 0 ? ch.w[0] : (i0 == 1 ? ch.w[2] : ch.w[4]);
            const uint32_t a1 = i0 == 0 ? ch.w[1] : (i0 == 1 ? ch.w[3] : ch.w[5]);
            const uint32_t b0 = i1 == 3 ? ch.w[6] : (i1 == 2 ? ch.w[4] : ch.w[2]);
            const uint32_t b1 = i1 == 3 ? ch.w[7] : (i1 == 2 ? ch.w[5] : ch.w[3]);
            reinterpret_cast<uint4*>(values)[v] = make_uint4(a0, a1, b0, b1);
          } else {
            const uint32_t a = i0 == 0 ? ch.w[0] : (i0 == 1 ? ch.w[1] : ch.w[2]);
            const uint32_t b = i1 == 3 ? ch.w[3] : (i1 == 2 ? ch.w[2] : ch.w[1]);
            reinterpret_cast<uint2*>(values)[v] = make_uint2(a, b);
          }
          if ((v & 1) == 0) meta[v >> 1] = (uint8_t)(nib | ((j + 1 < n) ? other << 4 : 0u));
        }
      });
}

// One chunk per thread, grid-stride: the kept pairs back at their places, +0 elsewhere.
template <int DT>
__global__ void __launch_bounds__(kThreads) decompress48_vec(const void* __restrict__ values,
                                                             const uint8_t* __restrict__ meta, int64_t n_chunks,
                                                             uint4* __restrict__ w) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n_chunks; v += stride) {
    const uint32_t nib = (meta[v >> 1] >> (4 * (v & 1))) & 0xfu;
    uint32_t i0 = nib & 3u, i1 = nib >> 2;
    const bool legal = i0 < i1;
    if (!legal) {
      set_dev_error(SP24_ERR_INVALID_ARG);
      i0 = i1 = 4;  // no pair matches: the chunk comes back all +0
    }
    if (DT == SP24_F32) {
      const uint4 kv = reinterpret_cast<const uint4*>(values)[v];
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        o[2 * j] = j == (int)i0 ? kv.x : (j == (int)i1 ? kv.z : 0u);
        o[2 * j + 1] = j == (int)i0 ? kv.y : (j == (int)i1 ? kv.w : 0u);
      }
      w[2 * v] = make_uint4(o[0], o[1], o[2], o[3]);
      w[2 * v + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
      const uint2 kv = reinterpret_cast<const uint2*>(values)[v];
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = j == (int)i0 ? kv.x : (j == (int)i1 ? kv.y : 0u);
      w[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ------------------------------------------------------------------ scalar path (any alignment)

enum { kCheck = 0, kPrune = 1, kDecompress = 2 };

template <int DT>
__device__ __forceinline__ uint32_t ld_entry(const void* p, int64_t i) {
  if (DT == SP24_F32) return reinterpret_cast<const uint32_t*>(p)[i];
  return reinterpret_cast<const uint16_t*>(p)[i];
}

template <int DT>
__device__ __forceinline__ void st_entry(void* p, int64_t i, uint32_t v) {
  if (DT == SP24_F32)
    reinterpret_cast<uint32_t*>(p)[i] = v;
  else
    reinterpret_cast<uint16_t*>(p)[i] = (uint16_t)v;
}

// One thread per meta byte b (chunks 2b and 2b + 1 when present).  kCheck: src = w, dst =
// pass; kPrune: src = w, dst = values; kDecompress: src = values, dst = w_out.
template <int DT, int MODE>
__global__ void __launch_bounds__(kThreads) pair48_any(const void* __restrict__ src, uint8_t* __restrict__ meta,
                                                       int64_t n_chunks, void* __restrict__ dst,
                                                       int32_t* __restrict__ n_fail) {
  const int64_t n_bytes = (n_chunks + 1) / 2;
  int fails = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t b_end = (n_bytes + stride - 1) / stride * stride;  // same trip count in every lane
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < b_end; b += stride) {
    if (b >= n_bytes) continue;
    uint32_t mbyte = 0;
    if (MODE == kDecompress) mbyte = meta[b];
    for (int h = 0; h < 2; ++h) {
      const int64_t v = 2 * b + h;
      if (v >= n_chunks) break;
      if constexpr (MODE == kDecompress) {
        const uint32_t nib = (mbyte >> (4 * h)) & 0xfu;
        int i0 = nib & 3, i1 = nib >> 2;
        if (i0 >= i1) {
          set_dev_error(SP24_ERR_INVALID_ARG);
          i0 = i1 = 4;
        }
        for (int j = 0; j < 4; ++j)
          for (int e = 0; e < 2; ++e) {
            const uint32_t x = j == i0 ? ld_entry<DT>(src, 4 * v + e) : (j == i1 ? ld_entry<DT>(src, 4 * v + 2 + e) : 0u);
            st_entry<DT>(dst, 8 * v + 2 * j + e, x);
          }
      } else {
        Chunk<DT> ch;
        for (int j = 0; j < 4; ++j) {
          const uint32_t a = ld_entry<DT>(src, 8 * v + 2 * j), c = ld_entry<DT>(src, 8 * v + 2 * j + 1);
          if (DT == SP24_F32) {
            ch.w[2 * j] = a;
            ch.w[2 * j + 1] = c;
          } else {
            ch.w[j] = a | (c << 16);
          }
        }
        if (MODE == kCheck) {
          const int ok = ch.eligible();
          fails += 1 - ok;
          reinterpret_cast<uint8_t*>(dst)[v] = (uint8_t)ok;
        } else {
          const uint32_t nib = ch.nibble();
          const int i0 = nib & 3, i1 = nib >> 2;
          for (int e = 0; e < 2; ++e) {
            st_entry<DT>(dst, 4 * v + e, ld_entry<DT>(src, 8 * v + 2 * i0 + e));
            st_entry<DT>(dst, 4 * v + 2 + e, ld_entry<DT>(src, 8 * v + 2 * i1 + e));
          }
          mbyte |= nib << (4 * h);
        }
      }
    }
    if (MODE == kPrune) meta[b] = (uint8_t)mbyte;
  }
  if (MODE == kCheck) count_fails(fails, n_fail);
}

// ------------------------------------------------------------------ host side

int64_t blocks_for(int64_t items) { return (items + kThreads - 1) / kThreads; }

template <typename Kern>
int ring_grid(Kern k, int64_t bytes) {
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingBytes);
  return full_wave_grid(k, kThreads, (bytes + kChunk - 1) / kChunk, kRingBytes);
}

// Validates (dtype, rows, K) and returns the chunk count.
int parse48(int dtype, int64_t rows, int64_t K, int64_t* n_chunks) {
  if (!elem_bytes(dtype)) return SP24_ERR_DTYPE;
  if (rows < 0 || K < 0 || K % 8) return SP24_ERR_SHAPE;
  *n_chunks = rows * (K / 8);
  return SP24_OK;
}

template <int DT>
int check48(const void* w, int64_t C, uint8_t* pass, int32_t* n_fail, cudaStream_t s) {
  if (aligned(w, 16)) {
    auto k = check48_vec<DT>;
    k<<<ring_grid(k, C * chunk_bytes<DT>()), kThreads, kRingBytes, s>>>((const uint4*)w, C, pass, n_fail);
  } else {
    auto k = pair48_any<DT, kCheck>;
    k<<<full_wave_grid(k, kThreads, blocks_for((C + 1) / 2)), kThreads, 0, s>>>(w, nullptr, C, pass, n_fail);
  }
  return launch_status(1);
}

template <int DT>
int prune48(const void* w, int64_t C, void* values, uint8_t* meta, cudaStream_t s) {
  if (aligned(w, 16) && aligned(values, DT == SP24_F32 ? 16 : 8)) {
    auto k = prune48_vec<DT>;
    k<<<ring_grid(k, C * chunk_bytes<DT>()), kThreads, kRingBytes, s>>>((const uint4*)w, C, values, meta);
  } else {
    auto k = pair48_any<DT, kPrune>;
    k<<<full_wave_grid(k, kThreads, blocks_for((C + 1) / 2)), kThreads, 0, s>>>(w, meta, C, values, nullptr);
  }
  return launch_status(1);
}

template <int DT>
int decompress48(const void* values, const uint8_t* meta, int64_t C, void* w_out, cudaStream_t s) {
  if (aligned(values, DT == SP24_F32 ? 16 : 8) && aligned(w_out, 16)) {
    auto k = decompress48_vec<DT>;
    k<<<full_wave_grid(k, kThreads, blocks_for(C)), kThreads, 0, s>>>(values, meta, C, (uint4*)w_out);
  } else {
    auto k = pair48_any<DT, kDecompress>;
    k<<<full_wave_grid(k, kThreads, blocks_for((C + 1) / 2)), kThreads, 0, s>>>(values, const_cast<uint8_t*>(meta), C,
                                                                               w_out, nullptr);
  }
  return launch_status(1);
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_check_48(const void* w, int dtype, int64_t rows, int64_t K, uint8_t* pass, int32_t* n_fail,
                             void* stream) {
  int64_t C = 0;
  const int st = parse48(dtype, rows, K, &C);
  if (st) return st;
  if (C > 0 && (!w || !pass)) return SP24_ERR_INVALID_ARG;
  if (C > 0 && !aligned(w, elem_bytes(dtype))) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (n_fail && cudaMemsetAsync(n_fail, 0, sizeof(int32_t), s) != cudaSuccess) return SP24_ERR_CUDA;
  if (C == 0) return launch_status(0);
  if (dtype == SP24_F32) return check48<SP24_F32>(w, C, pass, n_fail, s);
  if (dtype == SP24_BF16) return check48<SP24_BF16>(w, C, pass, n_fail, s);
  return check48<SP24_F16>(w, C, pass, n_fail, s);
}

extern "C" int sp24_prune_compress_48(const void* w, int dtype, int64_t rows, int64_t K, void* values, uint8_t* meta,
                                      void* stream) {
  int64_t C = 0;
  const int st = parse48(dtype, rows, K, &C);
  if (st) return st;
  if (C == 0) return SP24_OK;
  if (!w || !values || !meta) return SP24_ERR_INVALID_ARG;
  const int eb = elem_bytes(dtype);
  if (!aligned(w, eb) || !aligned(values, eb)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (dtype == SP24_F32) return prune48<SP24_F32>(w, C, values, meta, s);
  if (dtype == SP24_BF16) return prune48<SP24_BF16>(w, C, values, meta, s);
  return prune48<SP24_F16>(w, C, values, meta, s);
}

extern "C" int sp24_decompress_48(const void* values, const uint8_t* meta, int dtype, int64_t rows, int64_t K,
                                  void* w_out, void* stream) {
  int64_t C = 0;
  const int st = parse48(dtype, rows, K, &C);
  if (st) return st;
  if (C == 0) return SP24_OK;
  if (!values || !meta || !w_out) return SP24_ERR_INVALID_ARG;
  const int eb = elem_bytes(dtype);
  if (!aligned(values, eb) || !aligned(w_out, eb)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (dtype == SP24_F32) return decompress48<SP24_F32>(values, meta, C, w_out, s);
  if (dtype == SP24_BF16) return decompress48<SP24_BF16>(values, meta, C, w_out, s);
  return decompress48<SP24_F16>(values, meta, C, w_out, s);
}
