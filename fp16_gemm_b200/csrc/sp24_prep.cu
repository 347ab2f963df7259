// a1 / a2: 2:4 eligibility check, magnitude pruning + compression, decompression.
//
// [P2] "Sparse GPU FLOPS Need the Right Zeros in the Right Places", sections "The operation
// determines which four entries belong together" and "Two half-zero vectors produce different
// pattern answers"; [P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went",
// section "What 2:4 actually is".
//
// These kernels are HBM-bound streams.  For the matmul layout (groups of four consecutive
// entries) every thread owns whole groups: one 16-byte load holds two 16-bit groups or one
// fp32 group, consecutive threads take consecutive 16-byte vectors (each warp load is 512
// contiguous bytes), and the top-2 choice is made in registers with six compares, so no
// cross-lane exchange is needed.  Conv weights [K, C, R, S] put the four members of a group
// R*S entries apart; those kernels take one group (or one pair of groups) per thread and
// read through the read-only cache, which still moves each input byte from DRAM once.
#include "sp24_internal.cuh"
#include "sp24_stream.cuh"

namespace sp24 {

__device__ int g_dev_error = 0;
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

namespace {

constexpr int kThreads = 256;

// ------------------------------------------------------------------ group arithmetic

// Bit mask of the two kept members of a group (|w| descending, index ascending): member i is
// kept when fewer than two members precede it.  A lower-index member precedes on >=, a higher
// one only on >.
__device__ __forceinline__ uint32_t keep_mask(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
  uint32_t r0 = (m1 > m0) + (m2 > m0) + (m3 > m0);
  uint32_t r1 = (m0 >= m1) + (m2 > m1) + (m3 > m1);
  uint32_t r2 = (m0 >= m2) + (m1 >= m2) + (m3 > m2);
  uint32_t r3 = (m0 >= m3) + (m1 >= m3) + (m2 >= m3);
  return (r0 < 2) | ((r1 < 2) << 1) | ((r2 < 2) << 2) | ((r3 < 2) << 3);
}

// nibble = i0 | i1 << 2 of a keep mask with exactly two bits set
__device__ __forceinline__ uint32_t mask_nibble(uint32_t mask) {
  uint32_t i0 = __ffs(mask) - 1;
  uint32_t i1 = 31 - __clz(mask);
  return i0 | (i1 << 2);
}

// One 16-bit group held as two words (lo = e0 | e1 << 16, hi = e2 | e3 << 16).
struct Group16 {
  uint32_t nib;   // kept indices
  uint32_t kept;  // v0 | v1 << 16
};

// Sort keys of a group of four 16-bit entries held as lo = e0 | e1 << 16, hi = e2 | e3 << 16:
// key = magnitude bits << 2 | (3 - index), so a larger key means a larger |w|, or an equal |w|
// at a lower index (the pruning order), and the four keys all differ.  A min/max network gives
// the largest three: k1 and k2 are the kept members, and the group has at least two zeros
// exactly when k3 < 4 (a magnitude of 0).
struct Keys4 {
  uint32_t k1, k2, k3, k4;
};

__device__ __forceinline__ Keys4 sort_keys16(uint32_t lo, uint32_t hi) {
  const uint32_t a = ((lo & 0x7fffu) << 2) | 3u, b = ((lo >> 14) & 0x1fffcu) | 2u;
  const uint32_t c = ((hi & 0x7fffu) << 2) | 1u, d = (hi >> 14) & 0x1fffcu;
  const uint32_t m01 = max(a, b), n01 = min(a, b), m23 = max(c, d), n23 = min(c, d);
  const uint32_t x = min(m01, m23), y = max(n01, n23);
  return Keys4{max(m01, m23), max(x, y), min(x, y), min(n01, n23)};
}

// Nibble (i0 | i1 << 2, i0 < i1) and kept pair (ascending index) from the two largest keys.
// With r = 3 - index, i0 = 3 - max(r) and i1 = 3 - min(r); the byte-permute selector of the
// pair is 0x1010 + 0x22 i0 + 0x2200 i1 (bytes 2 i0, 2 i0 + 1, 2 i1, 2 i1 + 1 of lo:hi).
__device__ __forceinline__ Group16 kept16(const Keys4& k, uint32_t lo, uint32_t hi) {
  const uint32_t ra = k.k1 & 3u, rb = k.k2 & 3u;
  const uint32_t rh = max(ra, rb), rl = min(ra, rb);
  Group16 g;
  g.nib = 15u - rh - 4u * rl;
  g.kept = __byte_perm(lo, hi, (0x1010u + 0x66u + 0x6600u) - 0x22u * rh - 0x2200u * rl);
  return g;
}

__device__ __forceinline__ int zeros16(uint32_t lo, uint32_t hi) {
  return (mag16(lo) == 0) + (mag16(lo >> 16) == 0) + (mag16(hi) == 0) + (mag16(hi >> 16) == 0);
}

__device__ __forceinline__ int zeros32(uint4 v) {
  return (mag32(v.x) == 0) + (mag32(v.y) == 0) + (mag32(v.z) == 0) + (mag32(v.w) == 0);
}

// |x| of one 16-bit entry of type DT as fp32 (exact).
template <int DT>
__device__ __forceinline__ float abs16(uint32_t bits) {
  if (DT == SP24_BF16) return __uint_as_float((bits & 0x7fffu) << 16);
  return fabsf(__half2float(__ushort_as_half((unsigned short)(bits & 0xffffu))));
}

// |w| of the 16-bit entry behind a sort key, as fp32 (exact).
template <int DT>
__device__ __forceinline__ float key_to_abs(uint32_t key) {
  return abs16<DT>(key >> 2);
}

// max(m, |entries of a word|): two 16-bit entries or one fp32.  fmaxf never returns a NaN
// operand, so NaN entries take no part in a maximum.
template <int DT>
__device__ __forceinline__ float max_abs_word(float m, uint32_t w) {
  if (DT == SP24_F32) return fmaxf(m, fabsf(__uint_as_float(w)));
  return fmaxf(fmaxf(m, abs16<DT>(w)), abs16<DT>(w >> 16));
}

// Block-wide max of non-negative floats (ordered like their bit patterns) into *dst with one
// atomicMax per CTA.
__device__ __forceinline__ void block_max_to(float m, unsigned int* dst) {
  __shared__ unsigned int wmax[kThreads / 32];
  __syncthreads();  // wmax may still be read by an earlier call
  unsigned int u = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = u;
  __syncthreads();
  if (threadIdx.x < 32) {
    unsigned int x = threadIdx.x < kThreads / 32 ? wmax[threadIdx.x] : 0u;
    x = __reduce_max_sync(0xffffffffu, x);
    if (threadIdx.x == 0 && x) atomicMax(dst, x);
  }
}

__device__ __forceinline__ void count_fails(int fails, int32_t* n_fail) {
  if (!n_fail) return;
  int s = __reduce_add_sync(0xffffffffu, fails);
  if ((threadIdx.x & 31) == 0 && s) atomicAdd(n_fail, s);
}

// ------------------------------------------------------------------ matmul layout, vector path

// Groups 2v, 2v+1 (16-bit) or group v (fp32) per 16-byte vector v.  Every lane of a warp runs
// the same number of iterations so the final warp reduction sees all lanes.
// Streaming ring: 3 stages of 16 KB per CTA (1024 vectors of 16 bytes, 4 per thread).
constexpr int kChunk = 16384, kStages = 3;  // 48 KB per CTA: four CTAs per SM
constexpr size_t kRingBytes = (size_t)kChunk * kStages;

template <int EB>
__global__ void __launch_bounds__(kThreads, 4) check24_vec(const uint4* __restrict__ w, int64_t nv,
                                                        uint8_t* __restrict__ pass,
                                                        int32_t* __restrict__ n_fail) {
  extern __shared__ __align__(128) uint8_t ring[];
  int fails = 0;
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(w), nv * 16, ring, [&](const uint8_t* chunk, int64_t c, int bytes) {
        const uint4* cv = reinterpret_cast<const uint4*>(chunk);
        const int nvec = bytes / 16;
        const int64_t v0 = c * (kChunk / 16);
#pragma unroll
        for (int q = 0; q < kChunk / 16 / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          if (j >= nvec) continue;
          const uint4 x = cv[j];
          if (EB == 2) {
            const int ok0 = zeros16(x.x, x.y) >= 2, ok1 = zeros16(x.z, x.w) >= 2;
            fails += 2 - ok0 - ok1;
            reinterpret_cast<uint16_t*>(pass)[v0 + j] = (uint16_t)(ok0 | (ok1 << 8));
          } else {
            const int ok = zeros32(x) >= 2;
            fails += 1 - ok;
            pass[v0 + j] = (uint8_t)ok;
          }
        }
      });
  count_fails(fails, n_fail);
}

template <int EB>
__global__ void __launch_bounds__(kThreads, 4) prune24_vec(const uint4* __restrict__ w, int64_t nv,
                                                        uint2* __restrict__ values,
                                                        uint8_t* __restrict__ meta) {
  extern __shared__ __align__(128) uint8_t ring[];
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(w), nv * 16, ring, [&](const uint8_t* chunk, int64_t c, int bytes) {
        const uint4* cv = reinterpret_cast<const uint4*>(chunk);
        const int nvec = bytes / 16;
        const int64_t v0 = c * (kChunk / 16);
#pragma unroll
        for (int q = 0; q < kChunk / 16 / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          const bool live = j < nvec;
          const uint4 x = live ? cv[j] : make_uint4(0, 0, 0, 0);
          const int64_t v = v0 + j;
          if (EB == 2) {
            if (live) {
              const Group16 a = kept16(sort_keys16(x.x, x.y), x.x, x.y);
              const Group16 b = kept16(sort_keys16(x.z, x.w), x.z, x.w);
              values[v] = make_uint2(a.kept, b.kept);
              meta[v] = (uint8_t)(a.nib | (b.nib << 4));
            }
          } else {
            const uint32_t nib = mask_nibble(keep_mask(mag32(x.x), mag32(x.y), mag32(x.z), mag32(x.w)));
            const uint32_t i0 = nib & 3, i1 = nib >> 2;
            const uint32_t e0 = i0 == 0 ? x.x : (i0 == 1 ? x.y : x.z);
            const uint32_t e1 = i1 == 3 ? x.w : (i1 == 2 ? x.z : x.y);
            // the partner group (v ^ 1) is in lane ^ 1: j and v have the parity of threadIdx.x
            const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
            if (live) {
              values[v] = make_uint2(e0, e1);
              const bool partner_live = (j ^ 1) < nvec;
              if ((v & 1) == 0) meta[v >> 1] = (uint8_t)(nib | (partner_live ? other << 4 : 0u));
            }
          }
        }
      });
}

// One read of a matmul weight doing the work of check24_vec, prune24_vec and the amax passes of
// the NVFP4 quantiser for both w and its kept values.  Scratch words (zeroed before the launch):
// acc[0] = amax|w| bits, acc[1] = amax|kept values| bits, acc[2] = failing groups, acc[3] = CTAs
// done.  The last CTA to finish writes the fail count and the two NVFP4 tensor scales
// amax / 2688, computed exactly as the quantiser derives them.
template <int DT>
__global__ void __launch_bounds__(kThreads, 4) prepare_vec(const uint4* __restrict__ w, int64_t nv,
                                                        uint8_t* __restrict__ pass, uint2* __restrict__ values,
                                                        uint8_t* __restrict__ meta, unsigned int* __restrict__ acc,
                                                        int32_t* __restrict__ n_fail, float* __restrict__ ts_w,
                                                        float* __restrict__ ts_v) {
  constexpr int EB = DT == SP24_F32 ? 4 : 2;
  // largest key of a non-NaN 16-bit entry: +inf's magnitude, index 0
  constexpr uint32_t kNaNKey = ((DT == SP24_BF16 ? 0x7f80u : 0x7c00u) << 2) | 3u;
  auto below_nan = [&](const Keys4& k) {  // largest non-NaN key of a group whose k1 is NaN
    return k.k2 <= kNaNKey ? k.k2 : (k.k3 <= kNaNKey ? k.k3 : (k.k4 <= kNaNKey ? k.k4 : 0u));
  };
  auto kept_below_nan = [&](const Keys4& k) {
    return k.k1 <= kNaNKey ? k.k1 : (k.k2 <= kNaNKey ? k.k2 : 0u);
  };
  extern __shared__ __align__(128) uint8_t ring[];
  int fails = 0;
  float mw = 0.0f, mv = 0.0f;  // fp32 weights
  uint32_t km = 0, kw = 0, kv = 0;  // 16-bit weights: keys (w and values, w only, values only)
  stream::for_each_chunk<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(w), nv * 16, ring, [&](const uint8_t* chunk, int64_t c, int bytes) {
        const uint4* cv = reinterpret_cast<const uint4*>(chunk);
        const int nvec = bytes / 16;
        const int64_t v0 = c * (kChunk / 16);
#pragma unroll
        for (int q = 0; q < kChunk / 16 / kThreads; ++q) {
          const int j = threadIdx.x + q * kThreads;
          const bool live = j < nvec;
          const uint4 x = live ? cv[j] : make_uint4(0, 0, 0, 0);
          const int64_t v = v0 + j;
          if (EB == 2) {
            if (live) {
              const Keys4 ka = sort_keys16(x.x, x.y), kb = sort_keys16(x.z, x.w);
              const int ok0 = ka.k3 < 4u, ok1 = kb.k3 < 4u;
              fails += 2 - ok0 - ok1;
              if (pass) reinterpret_cast<uint16_t*>(pass)[v] = (uint16_t)(ok0 | (ok1 << 8));
              const Group16 a = kept16(ka, x.x, x.y), b = kept16(kb, x.z, x.w);
              values[v] = make_uint2(a.kept, b.kept);
              meta[v] = (uint8_t)(a.nib | (b.nib << 4));
              // amax over non-NaN entries on keys (magnitude order; NaN sorts highest).  Without
              // a NaN the largest entry of the vector is kept, so one max serves w and values.
              const uint32_t top = max(ka.k1, kb.k1);
              if (top <= kNaNKey) {
                km = max(km, top);
              } else {
                kw = max(kw, max(ka.k1 <= kNaNKey ? ka.k1 : below_nan(ka), kb.k1 <= kNaNKey ? kb.k1 : below_nan(kb)));
                kv = max(kv, max(kept_below_nan(ka), kept_below_nan(kb)));
              }
            }
          } else {
            const uint32_t nib = mask_nibble(keep_mask(mag32(x.x), mag32(x.y), mag32(x.z), mag32(x.w)));
            const uint32_t i0 = nib & 3, i1 = nib >> 2;
            const uint32_t e0 = i0 == 0 ? x.x : (i0 == 1 ? x.y : x.z);
            const uint32_t e1 = i1 == 3 ? x.w : (i1 == 2 ? x.z : x.y);
            // the partner group (v ^ 1) is in lane ^ 1: j and v have the parity of threadIdx.x
            const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
            if (live) {
              const int ok = zeros32(x) >= 2;
              fails += 1 - ok;
              if (pass) pass[v] = (uint8_t)ok;
              values[v] = make_uint2(e0, e1);
              if ((v & 1) == 0) meta[v >> 1] = (uint8_t)(nib | (other << 4));  // nv is even
              mw = max_abs_word<DT>(max_abs_word<DT>(mw, x.x), x.y);
              mw = max_abs_word<DT>(max_abs_word<DT>(mw, x.z), x.w);
              mv = max_abs_word<DT>(max_abs_word<DT>(mv, e0), e1);
            }
          }
        }
      });
  if constexpr (EB == 2) {
    mw = key_to_abs<DT>(max(km, kw));
    mv = key_to_abs<DT>(max(km, kv));
  }
  count_fails(fails, reinterpret_cast<int32_t*>(acc + 2));
  block_max_to(mw, acc);
  block_max_to(mv, acc + 1);
  // last CTA: publish the totals
  __shared__ int is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(acc + 3, 1u) == gridDim.x - 1;
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    __threadfence();
    const volatile unsigned int* a = acc;
    if (n_fail) *n_fail = (int32_t)a[2];
    if (ts_w) *ts_w = __fdiv_rn(__uint_as_float(a[0]), 2688.0f);
    if (ts_v) *ts_v = __fdiv_rn(__uint_as_float(a[1]), 2688.0f);
  }
}

// Conv layout W[K, C, R, S], 16-bit entries: the four channels 4j .. 4j + 3 of output channel k
// form a contiguous block of 4 RS entries holding the RS groups (k, j, rs); group rs takes
// entries rs, RS + rs, 2 RS + rs and 3 RS + rs of the block, and groups are numbered
// (k, j, rs) row-major, i.e. block after block.  Chunks of whole block pairs (ch bytes) stream
// through the ring; thread t takes groups 2m, 2m + 1 of a chunk (m = t, t + blockDim.x, ...), so
// every nibble byte has one writer.  PRUNE: kept values to [K, C/2, R, S] and nibbles, else the
// pass map and fail count.
template <bool PRUNE>
__global__ void __launch_bounds__(kThreads, 4) conv24_vec16(const uint16_t* __restrict__ w, int64_t nbytes, int ch,
                                                             int RS, uint8_t* __restrict__ pass,
                                                             int32_t* __restrict__ n_fail, uint16_t* __restrict__ values,
                                                             uint8_t* __restrict__ meta) {
  extern __shared__ __align__(128) uint8_t ring[];
  int fails = 0;
  stream::for_each_chunk_rt<kChunk, kStages>(
      reinterpret_cast<const uint8_t*>(w), nbytes, ch, ring, [&](const uint8_t* chunk, int64_t c, int bytes) {
        const uint16_t* e = reinterpret_cast<const uint16_t*>(chunk);
        const int64_t g0 = c * (ch / 8);  // groups before this chunk (8 bytes of entries per group)
        const int ng = bytes / 8;         // even: whole block pairs
        for (int m = threadIdx.x; 2 * m < ng; m += kThreads) {
          uint32_t nib[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int gi = 2 * m + u, b = gi / RS, rs = gi - b * RS;
            const uint16_t* blk = e + (int64_t)b * 4 * RS + rs;
            const uint32_t lo = blk[0] | ((uint32_t)blk[RS] << 16), hi = blk[2 * RS] | ((uint32_t)blk[3 * RS] << 16);
            const Keys4 k = sort_keys16(lo, hi);
            if (PRUNE) {
              const Group16 gr = kept16(k, lo, hi);
              nib[u] = gr.nib;
              const int64_t blk_g = g0 / RS + b;  // global block: chunks hold whole blocks
              values[(2 * blk_g) * RS + rs] = (uint16_t)(gr.kept & 0xffffu);
              values[(2 * blk_g + 1) * RS + rs] = (uint16_t)(gr.kept >> 16);
            } else {
              const int ok = k.k3 < 4u;
              fails += 1 - ok;
              pass[g0 + gi] = (uint8_t)ok;
            }
          }
          if (PRUNE) meta[(g0 >> 1) + m] = (uint8_t)(nib[0] | (nib[1] << 4));
        }
      });
  if (!PRUNE) count_fails(fails, n_fail);
}

// Inverse of prune24_vec for 16-bit data: two groups per thread.
__global__ void __launch_bounds__(kThreads) decompress24_vec16(const uint2* __restrict__ values,
                                                               const uint8_t* __restrict__ meta,
                                                               int64_t nv, uint4* __restrict__ w) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nv; v += stride) {
    uint2 kv = values[v];
    uint32_t mb = meta[v];
    uint32_t out[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t nib = (mb >> (4 * h)) & 0xf;
      uint32_t i0 = nib & 3, i1 = nib >> 2;
      uint32_t kept = h ? kv.y : kv.x;
      if (i0 >= i1) {
        set_dev_error(SP24_ERR_INVALID_ARG);
        kept = 0;
      }
      // byte selectors: slot i takes v0 (bytes 0,1), v1 (bytes 2,3) or zero (bytes 4,5)
      auto sel = [&](uint32_t i) -> uint32_t { return i == i0 ? 0x10u : (i == i1 ? 0x32u : 0x54u); };
      out[2 * h] = __byte_perm(kept, 0u, sel(0) | (sel(1) << 8));
      out[2 * h + 1] = __byte_perm(kept, 0u, sel(2) | (sel(3) << 8));
    }
    w[v] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// ------------------------------------------------------------------ generic (any layout) path

struct Layout {
  int op;
  int64_t C, RS;  // conv: channels and R*S
};

// Chunk bytes for conv24_vec16: whole block pairs (16 RS bytes) up to the ring's stage size, or 0
// when that path does not apply (an odd number of blocks, or R*S too large).
int64_t conv_chunk(const Layout& L, int64_t G) {
  const int64_t unit = 16 * L.RS;
  const int64_t blocks = G / L.RS;
  if (L.op != SP24_OP_CONV || unit > kChunk || blocks % 2) return 0;
  return kChunk / unit * unit;
}


// Element index of member i of group g.
__device__ __forceinline__ int64_t member(const Layout& L, int64_t g, int i) {
  if (L.op == SP24_OP_MATMUL) return g * 4 + i;
  int64_t rs = g % L.RS, kj = g / L.RS;
  int64_t j = kj % (L.C / 4), k = kj / (L.C / 4);
  return (k * L.C + 4 * j + i) * L.RS + rs;
}

// Index of stored value t of group g.
__device__ __forceinline__ int64_t slot(const Layout& L, int64_t g, int t) {
  if (L.op == SP24_OP_MATMUL) return g * 2 + t;
  int64_t rs = g % L.RS, kj = g / L.RS;
  int64_t j = kj % (L.C / 4), k = kj / (L.C / 4);
  return (k * (L.C / 2) + 2 * j + t) * L.RS + rs;
}

template <int EB>
__device__ __forceinline__ uint32_t load_elem(const void* p, int64_t i) {
  if (EB == 2) return __ldg(reinterpret_cast<const unsigned short*>(p) + i);
  return __ldg(reinterpret_cast<const unsigned int*>(p) + i);
}

template <int EB>
__device__ __forceinline__ void store_elem(void* p, int64_t i, uint32_t v) {
  if (EB == 2) reinterpret_cast<uint16_t*>(p)[i] = (uint16_t)v;
  else reinterpret_cast<uint32_t*>(p)[i] = v;
}

template <int EB>
__device__ __forceinline__ uint32_t magb(uint32_t x) {
  return EB == 2 ? mag16(x) : mag32(x);
}

template <int EB>
__global__ void __launch_bounds__(kThreads) check24_any(const void* __restrict__ w, Layout L,
                                                        int64_t g0, int64_t G,
                                                        uint8_t* __restrict__ pass,
                                                        int32_t* __restrict__ n_fail) {
  int fails = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t warp0 = g0 + (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) & ~int64_t(31));
  for (int64_t base = warp0; base < G; base += stride) {
    int64_t g = base + (threadIdx.x & 31);
    if (g < G) {
      int z = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) z += magb<EB>(load_elem<EB>(w, member(L, g, i))) == 0;
      pass[g] = (uint8_t)(z >= 2);
      fails += z < 2;
    }
  }
  count_fails(fails, n_fail);
}

// One pair of groups (one meta byte) per thread.
template <int EB>
__global__ void __launch_bounds__(kThreads) prune24_any(const void* __restrict__ w, Layout L,
                                                        int64_t p0, int64_t G,
                                                        void* __restrict__ values,
                                                        uint8_t* __restrict__ meta) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t P = (G + 1) / 2;
  for (int64_t p = p0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < P; p += stride) {
    uint32_t byte = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int64_t g = 2 * p + h;
      if (g >= G) break;
      uint32_t e[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) e[i] = load_elem<EB>(w, member(L, g, i));
      uint32_t nib = mask_nibble(keep_mask(magb<EB>(e[0]), magb<EB>(e[1]), magb<EB>(e[2]), magb<EB>(e[3])));
      uint32_t i0 = nib & 3, i1 = nib >> 2;
      store_elem<EB>(values, slot(L, g, 0), i0 == 0 ? e[0] : (i0 == 1 ? e[1] : e[2]));
      store_elem<EB>(values, slot(L, g, 1), i1 == 3 ? e[3] : (i1 == 2 ? e[2] : e[1]));
      byte |= nib << (4 * h);
    }
    meta[p] = (uint8_t)byte;
  }
}

template <int EB>
__global__ void __launch_bounds__(kThreads) decompress24_any(const void* __restrict__ values,
                                                             const uint8_t* __restrict__ meta,
                                                             Layout L, int64_t g0, int64_t G,
                                                             void* __restrict__ w) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = g0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < G; g += stride) {
    uint32_t nib = (meta[g >> 1] >> (4 * (g & 1))) & 0xf;
    uint32_t i0 = nib & 3, i1 = nib >> 2;
    bool legal = i0 < i1;
    if (!legal) set_dev_error(SP24_ERR_INVALID_ARG);
    uint32_t v0 = load_elem<EB>(values, slot(L, g, 0)), v1 = load_elem<EB>(values, slot(L, g, 1));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t v = 0;
      if (legal && i == (int)i0) v = v0;
      if (legal && i == (int)i1) v = v1;
      store_elem<EB>(w, member(L, g, i), v);
    }
  }
}

// ------------------------------------------------------------------ host side

int64_t blocks_for(int64_t items) { return (items + kThreads - 1) / kThreads; }

// Grid of a streaming kernel over nv 16-byte vectors: one CTA per chunk, capped at a full wave.
template <typename Kern>
int ring_grid(Kern k, int64_t nv) {
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingBytes);
  return full_wave_grid(k, kThreads, (nv * 16 + kChunk - 1) / kChunk, kRingBytes);
}

// Validates (op, shape, ndim) and returns the group count and layout.
int parse_shape(int op, const int64_t* shape, int ndim, int64_t* G, Layout* L) {
  if (!shape || ndim < 1 || ndim > 4) return SP24_ERR_INVALID_ARG;
  for (int d = 0; d < ndim; ++d)
    if (shape[d] < 0) return SP24_ERR_SHAPE;
  L->op = op;
  L->C = 0;
  L->RS = 1;
  if (op == SP24_OP_MATMUL) {
    if (shape[ndim - 1] % 4) return SP24_ERR_SHAPE;
    int64_t n = 1;
    for (int d = 0; d < ndim; ++d) n *= shape[d];
    *G = n / 4;
    return SP24_OK;
  }
  if (op == SP24_OP_CONV) {
    if (ndim != 4 || shape[1] % 4) return SP24_ERR_SHAPE;
    L->C = shape[1];
    L->RS = shape[2] * shape[3];
    *G = shape[0] * (shape[1] / 4) * L->RS;
    return SP24_OK;
  }
  return SP24_ERR_INVALID_ARG;
}

}  // namespace

int sm_count() {
  static int cached = 0;
  if (!cached) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      cached = n;
    else
      return 148;
  }
  return cached;
}

}  // namespace sp24

using namespace sp24;

extern "C" int sp24_check_24(const void* w, int dtype, int op, const int64_t* shape, int ndim,
                             uint8_t* pass, int32_t* n_fail, void* stream) {
  int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  int64_t G;
  Layout L;
  int st = parse_shape(op, shape, ndim, &G, &L);
  if (st) return st;
  if (G > 0 && (!w || !pass)) return SP24_ERR_INVALID_ARG;
  if (G > 0 && !aligned(w, eb)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  if (n_fail && cudaMemsetAsync(n_fail, 0, sizeof(int32_t), s) != cudaSuccess) return SP24_ERR_CUDA;
  if (G == 0) return launch_status(0);
  int nl = 0;
  int64_t g_done = 0;
  if (op == SP24_OP_CONV && eb == 2 && aligned(w, 16) && conv_chunk(L, G) > 0) {
    const int ch = (int)conv_chunk(L, G);
    auto k = conv24_vec16<false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingBytes);
    const int grid = full_wave_grid(k, kThreads, (G * 8 + ch - 1) / ch, kRingBytes);
    k<<<grid, kThreads, kRingBytes, s>>>((const uint16_t*)w, G * 8, ch, (int)L.RS, pass, n_fail, nullptr, nullptr);
    return launch_status(1);
  }
  if (op == SP24_OP_MATMUL && aligned(w, 16) && aligned(pass, eb == 2 ? 2 : 1)) {
    int64_t nv = G * 4 * eb / 16;  // whole 16-byte vectors
    if (nv > 0) {
      if (eb == 2)
        check24_vec<2><<<ring_grid(check24_vec<2>, nv), kThreads, kRingBytes, s>>>((const uint4*)w, nv, pass, n_fail);
      else
        check24_vec<4><<<ring_grid(check24_vec<4>, nv), kThreads, kRingBytes, s>>>((const uint4*)w, nv, pass, n_fail);
      ++nl;
      g_done = nv * 16 / (4 * eb);
    }
  }
  if (g_done < G) {
    if (eb == 2)
      check24_any<2><<<full_wave_grid(check24_any<2>, kThreads, blocks_for(G - g_done)), kThreads, 0, s>>>(w, L, g_done, G, pass, n_fail);
    else
      check24_any<4><<<full_wave_grid(check24_any<4>, kThreads, blocks_for(G - g_done)), kThreads, 0, s>>>(w, L, g_done, G, pass, n_fail);
    ++nl;
  }
  return launch_status(nl);
}

extern "C" int sp24_prune_compress_24(const void* w, int dtype, int op, const int64_t* shape,
                                      int ndim, void* values, uint8_t* meta, void* stream) {
  int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  int64_t G;
  Layout L;
  int st = parse_shape(op, shape, ndim, &G, &L);
  if (st) return st;
  if (G == 0) return SP24_OK;
  if (!w || !values || !meta) return SP24_ERR_INVALID_ARG;
  if (!aligned(w, eb) || !aligned(values, eb)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  int nl = 0;
  int64_t p_done = 0;  // meta bytes (group pairs) already written
  if (op == SP24_OP_CONV && eb == 2 && aligned(w, 16) && aligned(values, 2) && conv_chunk(L, G) > 0) {
    const int ch = (int)conv_chunk(L, G);
    auto k = conv24_vec16<true>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingBytes);
    const int grid = full_wave_grid(k, kThreads, (G * 8 + ch - 1) / ch, kRingBytes);
    k<<<grid, kThreads, kRingBytes, s>>>((const uint16_t*)w, G * 8, ch, (int)L.RS, nullptr, nullptr, (uint16_t*)values, meta);
    return launch_status(1);
  }
  if (op == SP24_OP_MATMUL && aligned(w, 16) && aligned(values, 8)) {
    int64_t nv = G * 4 * eb / 16;
    if (eb == 4) nv &= ~int64_t(1);  // whole meta bytes only
    if (nv > 0) {
      if (eb == 2)
        prune24_vec<2><<<ring_grid(prune24_vec<2>, nv), kThreads, kRingBytes, s>>>((const uint4*)w, nv, (uint2*)values, meta);
      else
        prune24_vec<4><<<ring_grid(prune24_vec<4>, nv), kThreads, kRingBytes, s>>>((const uint4*)w, nv, (uint2*)values, meta);
      ++nl;
      p_done = (nv * 16 / (4 * eb)) / 2;
    }
  }
  if (2 * p_done < G) {
    int64_t rest = (G + 1) / 2 - p_done;
    if (eb == 2)
      prune24_any<2><<<full_wave_grid(prune24_any<2>, kThreads, blocks_for(rest)), kThreads, 0, s>>>(w, L, p_done, G, values, meta);
    else
      prune24_any<4><<<full_wave_grid(prune24_any<4>, kThreads, blocks_for(rest)), kThreads, 0, s>>>(w, L, p_done, G, values, meta);
    ++nl;
  }
  return launch_status(nl);
}

extern "C" int sp24_decompress_24(const void* values, const uint8_t* meta, int dtype, int op,
                                  const int64_t* shape, int ndim, void* w_out, void* stream) {
  int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  int64_t G;
  Layout L;
  int st = parse_shape(op, shape, ndim, &G, &L);
  if (st) return st;
  if (G == 0) return SP24_OK;
  if (!values || !meta || !w_out) return SP24_ERR_INVALID_ARG;
  if (!aligned(values, eb) || !aligned(w_out, eb)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  int nl = 0;
  int64_t g_done = 0;
  if (op == SP24_OP_MATMUL && eb == 2 && aligned(values, 8) && aligned(w_out, 16)) {
    int64_t nv = G / 2;
    if (nv > 0) {
      decompress24_vec16<<<full_wave_grid(decompress24_vec16, kThreads, blocks_for(nv)), kThreads, 0, s>>>((const uint2*)values, meta, nv, (uint4*)w_out);
      ++nl;
    }
    g_done = 2 * nv;
  }
  if (g_done < G) {
    if (eb == 2)
      decompress24_any<2><<<full_wave_grid(decompress24_any<2>, kThreads, blocks_for(G - g_done)), kThreads, 0, s>>>(values, meta, L, g_done, G, w_out);
    else
      decompress24_any<4><<<full_wave_grid(decompress24_any<4>, kThreads, blocks_for(G - g_done)), kThreads, 0, s>>>(values, meta, L, g_done, G, w_out);
    ++nl;
  }
  return launch_status(nl);
}

extern "C" int sp24_prepare_24_workspace_size(int64_t rows, int64_t K, int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 16) return SP24_ERR_SHAPE;
  *bytes = 256;
  return SP24_OK;
}

extern "C" int sp24_prepare_24(const void* w, int dtype, int64_t rows, int64_t K, uint8_t* pass,
                               int32_t* n_fail, void* values, uint8_t* meta, float* w_tensor_scale,
                               float* v_tensor_scale, void* workspace, int64_t workspace_bytes,
                               void* stream) {
  const int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  if (rows < 0 || K < 0 || K % 16) return SP24_ERR_SHAPE;
  const int64_t nv = rows * K * eb / 16;
  if (nv > 0 && (!w || !values || !meta)) return SP24_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < 256) return SP24_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return SP24_ERR_ALIGN;
  if (nv > 0 && (!aligned(w, 16) || !aligned(values, 8) || (pass && !aligned(pass, 2)))) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  unsigned int* acc = reinterpret_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(acc, 0, 4 * sizeof(unsigned int), s) != cudaSuccess) return SP24_ERR_CUDA;
  // launched even for an empty weight, so that the count and the scales are written
  if (dtype == SP24_F32)
    prepare_vec<SP24_F32><<<ring_grid(prepare_vec<SP24_F32>, nv), kThreads, kRingBytes, s>>>(
        (const uint4*)w, nv, pass, (uint2*)values, meta, acc, n_fail, w_tensor_scale, v_tensor_scale);
  else if (dtype == SP24_BF16)
    prepare_vec<SP24_BF16><<<ring_grid(prepare_vec<SP24_BF16>, nv), kThreads, kRingBytes, s>>>(
        (const uint4*)w, nv, pass, (uint2*)values, meta, acc, n_fail, w_tensor_scale, v_tensor_scale);
  else
    prepare_vec<SP24_F16><<<ring_grid(prepare_vec<SP24_F16>, nv), kThreads, kRingBytes, s>>>(
        (const uint4*)w, nv, pass, (uint2*)values, meta, acc, n_fail, w_tensor_scale, v_tensor_scale);
  return launch_status();
}
