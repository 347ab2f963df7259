// a6: skinny (decode-shaped, M <= 64) dense and 2:4-sparse GEMM, shared-memory staged.
//
// [P5] "NVFP4 Without FP4 Hardware", "Why NVFP4 helps without FP4 hardware": a decode step
// reads every weight once, so the GEMV is bound by the weight read and the 4-bit values are
// unpacked inside the kernel.  [P2] "Sparse GPU FLOPS Need the Right Zeros in the Right
// Places", "The mechanism needs both values and their positions": the 2:4 path hands the kept
// values and their 2-bit positions to the sparse tensor-core MMA, which selects the matching
// activations itself.
//
// CTA = 4 warps = 64 weight rows x one K-slice of KC logical entries.
//   1. Lanes issue one cp.async.bulk per weight row (values/codes, NVFP4 block scales, 2:4
//      nibbles) into padded shared-memory rows, all completing on one mbarrier; the whole
//      slice is in flight at once without costing registers.
//   2. Meanwhile the CTA stages x[M, slice] into shared memory in MMA-fragment order with
//      16-byte loads, so every B fragment is one conflict-free shared load.
//   3. Each warp owns 16 rows: it reads its A fragments from shared memory (row pitches chosen
//      so the reads are bank-conflict free), decodes NVFP4 to 16 bits in registers, and issues
//      mma.m16n8k16 (dense) or mma.sp m16n8k32 (2:4, metadata from the nibble stream).
//   4. K-slices are reduced into y with fp32 atomics (y zeroed first) when there are several.
//
// Dense layouts: a lane reads a contiguous 16-byte piece of a row per chunk and the K order
// inside the chunk is permuted (x is staged with the same permutation).  2:4 layouts: the
// hardware wants lane (g, c) to supply the kept pair of MMA groups c and c+4 of rows g, g+8,
// and takes the nibbles of groups 0-3 / 4-7 of rows g | g+8 from lanes c = 0 / 1; with the
// identity group order inside each 32-wide K window those nibbles are the low / high halves of
// one 32-bit word of each row's nibble stream.
#include "sp24_internal.cuh"
#include "sp24_tc.cuh"
#include "sp24_stream.cuh"
#include "sp24_fp4.cuh"

namespace sp24 {
namespace {

using tc::mbar_arrive_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::smem_u32;

constexpr int kWarps = 4;
constexpr int kRows = kWarps * 16;

// Per format: logical K per slice, bytes per row per slice of each array, shared row pitches.
template <int WF>
struct F2;
template <>
struct F2<W_D16> {  // 16-bit dense: 8 values (16 B) per lane piece, chunk = 32 K
  static constexpr int KC = 256, CHUNK = 32, STEPS = 2;
  static constexpr int VB = KC * 2;
  static constexpr int VP = VB + 64, SP = 0, MP = 0;
};
template <>
struct F2<W_DQ4> {  // NVFP4 dense: 32 codes (16 B) per lane piece, chunk = 128 K
  static constexpr int KC = 512, CHUNK = 128, STEPS = 8;
  static constexpr int VB = KC / 2, SB = KC / 16;
  static constexpr int VP = VB + 64, SP = SB + 16, MP = 0;
};
template <>
struct F2<W_S16> {  // 16-bit 2:4: windows of 32 K (8 groups, 32 B of values)
  static constexpr int KC = 512, CHUNK = 32, STEPS = 1;
  static constexpr int VB = KC, MB = KC / 8;
  static constexpr int VP = VB + 16, SP = 0, MP = MB + 16;
};
template <>
struct F2<W_SQ4> {  // NVFP4 2:4: windows of 32 K (8 groups, 8 B of codes, one block scale)
  static constexpr int KC = 1024, CHUNK = 32, STEPS = 1;
  static constexpr int VB = KC / 4, SB = KC / 32, MB = KC / 8;
  static constexpr int VP = VB + 16, SP = SB + 16, MP = MB + 16;
};

template <int WF>
__host__ __device__ constexpr bool sparse_fmt() { return WF == W_S16 || WF == W_SQ4; }

// Bytes of x fragments per (chunk or window, step, token tile): 32 lanes x 8 B (k16 MMA) or
// x 16 B (k32 sparse MMA).
template <int WF>
__host__ __device__ constexpr int frag_bytes() { return sparse_fmt<WF>() ? 512 : 256; }

template <int WF, int NT>
struct Smem2 {
  using C = F2<WF>;
  static constexpr int XB = (C::KC / C::CHUNK) * C::STEPS * NT * frag_bytes<WF>();
  static constexpr int OFF_V = XB;
  static constexpr int OFF_S = OFF_V + kRows * C::VP;
  static constexpr int OFF_M = OFF_S + kRows * C::SP;
  static constexpr int TOTAL = OFF_M + kRows * C::MP;
  static constexpr int WREG = TOTAL - OFF_V;   // one weight buffer
  // x + one weight buffer (one row block per CTA) or two (grouped: row blocks double-buffered)
  static constexpr int bytes(bool two) { return TOTAL + (two ? WREG : 0); }
};

template <typename T>
__device__ __forceinline__ void mma_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint2 b) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

// Sparse m16n8k32 with ordered metadata (kept indices ascending in each group), selector 0.
template <typename T>
__device__ __forceinline__ void mma_sp_k32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint4 b, uint32_t e) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    asm volatile(
        "mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, 0x0;"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(e));
  else
    asm volatile(
        "mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, 0x0;"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "r"(e));
}


// x[n, k] as 16-bit bits of T (0 outside the matrix); NVFP4 x decoded to E2M1 * E4M3.  `n` is
// the x row already mapped (grouped mode: the routed token), `live` says whether the tile row
// exists.
template <typename T>
__device__ __forceinline__ uint32_t xval(const SkinnyParams& p, int64_t n, int64_t k, bool live = true) {
  if (!live || k >= p.K) return 0;
  if (p.x_fmt == X_16) return __ldg(reinterpret_cast<const unsigned short*>(p.x) + n * p.K + k);
  const uint8_t* codes = reinterpret_cast<const uint8_t*>(p.x);
  const uint32_t c = (codes[(n * p.K + k) >> 1] >> (4 * (k & 1))) & 0xf;
  const uint32_t mag = c & 7, e = mag >> 1, m = mag & 1;
  const float a = e == 0 ? 0.5f * m : (float)(1 << (e - 1)) * (1.0f + 0.5f * m);
  uint32_t h2;
  const uint16_t sc = p.x_scales[(n * p.K + k) >> 4];
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(sc));
  const float v = a * __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
  return to_bits16<T>(c & 8 ? -v : v);
}

// Eight consecutive x entries [k, k+8) of token n as four packed 16-bit pairs.
template <typename T>
__device__ __forceinline__ uint4 xoct(const SkinnyParams& p, int64_t n, int64_t k, bool live) {
  if (p.x_fmt == X_16 && live && k + 8 <= p.K)
    return __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.x) + n * p.K + k));
  uint32_t v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = xval<T>(p, n, k + i, live);
  return make_uint4(v[0] | (v[1] << 16), v[2] | (v[3] << 16), v[4] | (v[5] << 16), v[6] | (v[7] << 16));
}

template <int WF, typename T, int NT, bool GROUPED>
__global__ void __launch_bounds__(kWarps * 32) skinny2_kernel(SkinnyParams p) {
  using C = F2<WF>;
  using L = Smem2<WF, NT>;
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int32_t rows_of[GROUPED ? 64 : 1];  // grouped: flat (token, slot) of each tile row

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  if constexpr (GROUPED) {
    // tile = (expert, first perm index, count): rebase w / scales / meta on the expert's rows
    const int32_t* tl = p.tiles + 3 * (int64_t)blockIdx.z;
    const int32_t e = tl[0], first = tl[1], cnt = tl[2];
    if (cnt <= 0) return;
    p.M = cnt;
    p.w += (int64_t)e * p.expert_rows * p.w_row_bytes;
    if (p.w_scales) p.w_scales += (int64_t)e * p.expert_rows * p.scale_row_bytes;
    if (p.meta) p.meta += (int64_t)e * p.expert_rows * p.meta_row_bytes;
    if (threadIdx.x < 64) rows_of[threadIdx.x] = threadIdx.x < cnt ? p.perm[first + threadIdx.x] : 0;
  }
  const int64_t k0 = (int64_t)blockIdx.y * C::KC;
  const int64_t kv = p.K - k0 < C::KC ? p.K - k0 : C::KC;  // valid logical K in this slice
  const int nrb = (int)((p.N + kRows - 1) / kRows);       // 64-row weight blocks

  // ---- 1. weight slices: row block rb into buffer `buf` with 16-byte cp.async, all threads;
  // each row's pieces are consecutive, so a warp's copies cover whole row segments.
  const uint32_t vbytes = (uint32_t)(WF == W_D16 ? kv * 2 : WF == W_DQ4 ? kv / 2 : WF == W_S16 ? kv : kv / 4);
  const uint32_t sbytes = (uint32_t)(WF == W_DQ4 ? kv / 16 : WF == W_SQ4 ? kv / 32 : 0);
  const uint32_t mbytes = (uint32_t)(sparse_fmt<WF>() ? kv / 8 : 0);
  const int64_t voff = WF == W_D16 ? k0 * 2 : WF == W_DQ4 ? k0 / 2 : WF == W_S16 ? k0 : k0 / 4;
  const int64_t soff = WF == W_DQ4 ? k0 / 16 : k0 / 32, moff = k0 / 8;
  constexpr int WREG = L::WREG;  // one buffer: values, scales, nibbles
  auto load_block = [&](int rb, int buf) {
    uint8_t* bv = sm + L::OFF_V + buf * WREG;
    uint8_t* bs = bv + (L::OFF_S - L::OFF_V);
    uint8_t* bm = bv + (L::OFF_M - L::OFF_V);
    const int64_t row0 = (int64_t)rb * kRows;
    const int rows_v = (int)(p.N - row0 < kRows ? p.N - row0 : kRows);
    const int vp = (int)(vbytes / 16), sp = (int)(sbytes / 16), mp = (int)(mbytes / 16);
    for (int i = threadIdx.x; i < rows_v * vp; i += blockDim.x) {
      const int r = i / vp, j = i - r * vp;
      tc::cp_async16(bv + r * C::VP + 16 * j, p.w + (row0 + r) * p.w_row_bytes + voff + 16 * j);
    }
    if constexpr (C::SP > 0) {
      for (int i = threadIdx.x; i < rows_v * sp; i += blockDim.x) {
        const int r = i / sp, j = i - r * sp;
        tc::cp_async16(bs + r * C::SP + 16 * j, p.w_scales + (row0 + r) * p.scale_row_bytes + soff + 16 * j);
      }
    }
    if constexpr (C::MP > 0) {
      for (int i = threadIdx.x; i < rows_v * mp; i += blockDim.x) {
        const int r = i / mp, j = i - r * mp;
        tc::cp_async16(bm + r * C::MP + 16 * j, p.meta + (row0 + r) * p.meta_row_bytes + moff + 16 * j);
      }
    }
    // Fill what no copy writes: the tail of each row when the slice is short, and whole rows
    // past N.  Values become +0 (uninitialised bits could be NaN, and NaN * 0 is NaN) and
    // nibbles the legal pair (0, 1).  The regions are disjoint from the copies' destinations.
    if (kv < C::KC || rows_v < kRows) {
      for (int i = threadIdx.x; i < kRows * (C::VP / 4); i += blockDim.x) {
        const int r = i / (C::VP / 4), off = (i % (C::VP / 4)) * 4;
        if (r >= rows_v || off >= (int)vbytes) *reinterpret_cast<uint32_t*>(bv + r * C::VP + off) = 0u;
      }
      if constexpr (C::SP > 0) {
        for (int i = threadIdx.x; i < kRows * C::SP; i += blockDim.x) {
          if (i / C::SP >= rows_v || i % C::SP >= (int)sbytes) bs[i] = 0;
        }
      }
      if constexpr (C::MP > 0) {
        for (int i = threadIdx.x; i < kRows * C::MP; i += blockDim.x) {
          if (i / C::MP >= rows_v || i % C::MP >= (int)mbytes) bm[i] = 0x44;
        }
      }
    }
  };
  __syncthreads();  // publishes rows_of
  load_block(blockIdx.x, 0);
  tc::cp_async_commit();

  // ---- 2. stage x in fragment order.  Each thread issues XB independent loads before it stores
  // any, so the staging costs a few L2 round trips rather than one per item.
  constexpr int NCH = C::KC / C::CHUNK;
  constexpr int XB = 8;
  if constexpr (!sparse_fmt<WF>()) {
    // entry (ch, s, t, lane): 8 bytes = x[8t+g][k0 + ch*CHUNK + LV*c + kslot(s, 0..3)]
    constexpr int LV = C::CHUNK / 4;
    uint2* xs = reinterpret_cast<uint2*>(sm);
    // one item per (ch, t, lane, octet): 8 consecutive k of the lane piece -> two entries
    const int items = NCH * NT * 32 * (LV / 8);
    for (int base = threadIdx.x; base < items; base += blockDim.x * XB) {
      uint4 v[XB];
#pragma unroll
      for (int b = 0; b < XB; ++b) {
        const int it = base + b * blockDim.x;
        if (it < items) {
          const int oct = it % (LV / 8), ln = (it / (LV / 8)) % 32, t = (it / (LV / 8) / 32) % NT,
                    ch = it / (LV / 8) / 32 / NT;
          const int gg = ln >> 2, cc = ln & 3;
          const int64_t kb = k0 + (int64_t)ch * C::CHUNK + LV * cc + 8 * oct;
          const int nrow = 8 * t + gg;
          const int64_t xr = GROUPED ? (nrow < p.M ? rows_of[nrow] / p.topk : 0) : nrow;
          v[b] = xoct<T>(p, xr, kb, nrow < p.M);
        }
      }
#pragma unroll
      for (int b = 0; b < XB; ++b) {
        const int it = base + b * blockDim.x;
        if (it < items) {
          const int oct = it % (LV / 8), ln = (it / (LV / 8)) % 32, t = (it / (LV / 8) / 32) % NT,
                    ch = it / (LV / 8) / 32 / NT;
          // the octet covers steps 2*oct and 2*oct+1 of this lane piece
          uint2 e0, e1;
          if (WF == W_DQ4) {  // slots (0,4,1,5) and (2,6,3,7) of the octet
            e0 = make_uint2(__byte_perm(v[b].x, v[b].z, 0x5410), __byte_perm(v[b].x, v[b].z, 0x7632));
            e1 = make_uint2(__byte_perm(v[b].y, v[b].w, 0x5410), __byte_perm(v[b].y, v[b].w, 0x7632));
          } else {  // slots 0..3 and 4..7
            e0 = make_uint2(v[b].x, v[b].y);
            e1 = make_uint2(v[b].z, v[b].w);
          }
          const int s0 = 2 * oct;
          xs[((ch * C::STEPS + s0) * NT + t) * 32 + ln] = e0;
          xs[((ch * C::STEPS + s0 + 1) * NT + t) * 32 + ln] = e1;
        }
      }
    }
  } else {
    // entry (win, t, lane): 16 bytes = x[8t+g][k0 + 32*win + 2c + 8i + {0,1}], i = 0..3
    uint4* xs = reinterpret_cast<uint4*>(sm);
    const int items = NCH * NT * 32;
    constexpr int IB = XB / 4;  // items per batch, four loads each
    for (int base = threadIdx.x; base < items; base += blockDim.x * IB) {
      uint32_t w4[IB][4];
#pragma unroll
      for (int b = 0; b < IB; ++b) {
        const int it = base + b * blockDim.x;
        if (it < items) {
          const int ln = it % 32, t = (it / 32) % NT, win = it / 32 / NT;
          const int gg = ln >> 2, cc = ln & 3;
          const int nrow = 8 * t + gg;
          const bool live = nrow < p.M;
          const int64_t n = GROUPED ? (live ? rows_of[nrow] / p.topk : 0) : nrow;
          const int64_t kb = k0 + 32 * win + 2 * cc;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int64_t k = kb + 8 * i;
            if (p.x_fmt == X_16 && live && k + 2 <= p.K)
              w4[b][i] = __ldg(reinterpret_cast<const unsigned int*>(reinterpret_cast<const uint16_t*>(p.x) + n * p.K + k));
            else
              w4[b][i] = xval<T>(p, n, k, live) | (xval<T>(p, n, k + 1, live) << 16);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < IB; ++b) {
        const int it = base + b * blockDim.x;
        if (it < items) xs[it] = make_uint4(w4[b][0], w4[b][1], w4[b][2], w4[b][3]);
      }
    }
  }
  // ---- 3. row blocks blockIdx.x, blockIdx.x + gridDim.x, ...: the next block's weights stream
  // in while this one is multiplied; the staged x serves them all
  const int rg = warp * 16 + g;  // local rows rg, rg + 8
  const int nch = (int)((kv + C::CHUNK - 1) / C::CHUNK);
  const int ntl = (p.M + 7) / 8;  // live token tiles
  for (int it = 0, rb = blockIdx.x; rb < nrb; ++it, rb += gridDim.x) {
    if (GROUPED && rb + (int)gridDim.x < nrb) load_block(rb + gridDim.x, (it + 1) & 1);
    tc::cp_async_commit();
    tc::cp_async_wait<1>();  // this block's copies (and x's stores, after the barrier)
    __syncthreads();
    const int64_t row0 = (int64_t)rb * kRows;
    uint8_t* const bv = sm + L::OFF_V + (GROUPED ? (it & 1) * WREG : 0);
    const uint8_t* vrow0 = bv + rg * C::VP;
    const uint8_t* vrow1 = vrow0 + 8 * C::VP;
    const uint8_t* srow = bv + (L::OFF_S - L::OFF_V);
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  {
    if constexpr (!sparse_fmt<WF>()) {
      const uint2* xs = reinterpret_cast<const uint2*>(sm);
#pragma unroll 2
      for (int ch = 0; ch < nch; ++ch) {
        const uint4 r0 = *reinterpret_cast<const uint4*>(vrow0 + ch * 64 + 16 * c);
        const uint4 r1 = *reinterpret_cast<const uint4*>(vrow1 + ch * 64 + 16 * c);
        uint32_t sc[2][2];
        if (WF == W_DQ4) {
          const uint32_t s0 = *reinterpret_cast<const uint16_t*>(srow + rg * C::SP + ch * 8 + 2 * c);
          const uint32_t s1 = *reinterpret_cast<const uint16_t*>(srow + (rg + 8) * C::SP + ch * 8 + 2 * c);
          scale_pair<T>(s0, sc[0][0], sc[0][1]);
          scale_pair<T>(s1, sc[1][0], sc[1][1]);
        }
        const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int s = 0; s < C::STEPS; ++s) {
          uint32_t a0, a1, a2, a3;
          if (WF == W_D16) {
            a0 = w0[2 * s];
            a2 = w0[2 * s + 1];
            a1 = w1[2 * s];
            a3 = w1[2 * s + 1];
          } else {
            const int q = s >> 1, i0 = 2 * (s & 1), hb = s >> 2;
            a0 = hmul2u<T>(fp4_pair_i4<T>(w0[q], i0), sc[0][hb]);
            a2 = hmul2u<T>(fp4_pair_i4<T>(w0[q], i0 + 1), sc[0][hb]);
            a1 = hmul2u<T>(fp4_pair_i4<T>(w1[q], i0), sc[1][hb]);
            a3 = hmul2u<T>(fp4_pair_i4<T>(w1[q], i0 + 1), sc[1][hb]);
          }
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < ntl) mma_k16<T>(acc[t], a0, a1, a2, a3, xs[((ch * C::STEPS + s) * NT + t) * 32 + lane]);
        }
      }
    } else {
      const uint4* xs = reinterpret_cast<const uint4*>(sm);
      const uint8_t* mrow0 = bv + (L::OFF_M - L::OFF_V) + rg * C::MP;
      const uint8_t* mrow1 = mrow0 + 8 * C::MP;
#pragma unroll 4
      for (int win = 0; win < nch; ++win) {
        // metadata: word `win` of each row's nibble stream; lanes c = 0 / 1 pass the low / high
        // halves (groups 0-3 / 4-7) of rows g | g+8
        const uint32_t m0 = *reinterpret_cast<const uint32_t*>(mrow0 + 4 * win);
        const uint32_t m1 = *reinterpret_cast<const uint32_t*>(mrow1 + 4 * win);
        const uint32_t e = __byte_perm(m0, m1, (c & 1) ? 0x7632 : 0x5410);
        uint32_t a0, a1, a2, a3;
        if (WF == W_S16) {  // kept pair of group c / c+4: 4-byte words 8*win + c (+4)
          a0 = *reinterpret_cast<const uint32_t*>(vrow0 + 32 * win + 4 * c);
          a2 = *reinterpret_cast<const uint32_t*>(vrow0 + 32 * win + 4 * c + 16);
          a1 = *reinterpret_cast<const uint32_t*>(vrow1 + 32 * win + 4 * c);
          a3 = *reinterpret_cast<const uint32_t*>(vrow1 + 32 * win + 4 * c + 16);
        } else {  // codes: bytes 8*win + c (+4); one block scale per window
          const uint2 v0 = *reinterpret_cast<const uint2*>(vrow0 + 8 * win);
          const uint2 v1 = *reinterpret_cast<const uint2*>(vrow1 + 8 * win);
          uint32_t s0, s1, unused;
          scale_pair<T>(srow[rg * C::SP + win], s0, unused);
          scale_pair<T>(srow[(rg + 8) * C::SP + win], s1, unused);
          const uint32_t b0 = __byte_perm(v0.x, v0.y, c | ((c + 4) << 4));  // bytes c, c+4 -> [0], [1]
          const uint32_t b1 = __byte_perm(v1.x, v1.y, c | ((c + 4) << 4));
          a0 = hmul2u<T>(fp4_pair_byte<T>(b0, 0), s0);
          a2 = hmul2u<T>(fp4_pair_byte<T>(b0, 1), s0);
          a1 = hmul2u<T>(fp4_pair_byte<T>(b1, 0), s1);
          a3 = hmul2u<T>(fp4_pair_byte<T>(b1, 1), s1);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t < ntl) mma_sp_k32<T>(acc[t], a0, a1, a2, a3, xs[(win * NT + t) * 32 + lane], e);
      }
    }
  }

  // ---- 4. epilogue: rows row0 + rg (+8), tokens 8t + 2c (+1)
  float scale = 1.0f;
  if (WF == W_DQ4 || WF == W_SQ4) scale = 256.0f * *p.w_ts;
  if (p.x_fmt == X_Q4) scale *= *p.x_ts;
  if (p.accumulate && p.N % 4 == 0 && (reinterpret_cast<uintptr_t>(p.y) & 15) == 0) {
    // partial sums over a K slice: transpose the tile through the (now idle) weight buffer so
    // that each thread adds four consecutive outputs of one token with one vector atomic
    constexpr int OP = kRows + 4;  // padded row of the transposed tile (floats)
    float* ot = reinterpret_cast<float*>(bv);
    __syncthreads();  // every warp is done reading the weight buffer
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (t < ntl) {
        const int n = 8 * t + 2 * c;
        ot[n * OP + rg] = acc[t][0];
        ot[(n + 1) * OP + rg] = acc[t][1];
        ot[n * OP + rg + 8] = acc[t][2];
        ot[(n + 1) * OP + rg + 8] = acc[t][3];
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < p.M * (kRows / 4); i += blockDim.x) {
      const int n = i / (kRows / 4), r = 4 * (i % (kRows / 4));
      if (row0 + r < p.N) {
        const int64_t orow = GROUPED ? (int64_t)rows_of[n] : n;
        const float4 v = *reinterpret_cast<const float4*>(ot + n * OP + r);
        float* dst = p.y + orow * p.N + row0 + r;
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x * scale),
                     "f"(v.y * scale), "f"(v.z * scale), "f"(v.w * scale)
                     : "memory");
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t n = 8 * t + 2 * c + (q & 1);
        const int64_t r = row0 + rg + ((q & 2) ? 8 : 0);
        if (n < p.M && r < p.N) {
          const int64_t orow = GROUPED ? (int64_t)rows_of[n] : n;
          float* dst = p.y + orow * p.N + r;
          const float v = acc[t][q] * scale;
          if (p.accumulate) atomicAdd(dst, v);
          else *dst = v;
        }
      }
    }
  }
    __syncthreads();  // every warp is done with this buffer before it is refilled
  }
  tc::cp_async_wait<0>();
}

template <int WF, typename T, bool GROUPED = false>
int launch2(const SkinnyParams& p, int nt, cudaStream_t s, unsigned tiles = 1) {
  using C = F2<WF>;
  // grouped: one CTA walks all of an expert's row blocks, so its token tile's x is staged once
  const unsigned nrb = (unsigned)((p.N + kRows - 1) / kRows);
  dim3 grid(GROUPED ? 1u : nrb, (unsigned)((p.K + C::KC - 1) / C::KC), tiles);
#define SP24_L2(NTV)                                                                                        \
  {                                                                                                         \
    auto kern = skinny2_kernel<WF, T, NTV, GROUPED>;                                                        \
    constexpr int smem = Smem2<WF, NTV>::bytes(GROUPED);                                                    \
    if (smem > 48 * 1024 && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
      return SP24_ERR_CUDA;                                                                                 \
    kern<<<grid, kWarps * 32, smem, s>>>(p);                                                                \
  }
  switch (nt) {
    case 1: SP24_L2(1) break;
    case 2: SP24_L2(2) break;
    case 4: SP24_L2(4) break;
    case 8: SP24_L2(8) break;
    default: return SP24_ERR_UNSUPPORTED;
  }
#undef SP24_L2
  return launch_status();
}

// ------------------------------------------------------------------ persistent decode GEMV (M <= 8)
//
// One CTA of 16 warps per SM.  All threads first copy x (M <= 8 tokens, whole K) into shared
// memory with 16-byte cp.async (token rows past M are zeroed).  The weight is cut into units of
// 16 rows x UK logical k; each CTA takes a contiguous range of units in tile-major order (so
// every SM streams the same number of bytes) and its warps take the units round-robin.  A warp
// moves its own units with 16-byte cp.async on the load/store path into a private double
// buffer, so every warp keeps two units in flight without a producer: one thread issuing TMA
// requests for a whole SM cannot keep HBM busy when each unit is 16 short rows.  A warp adds its
// partial sums of a 16-row tile into that tile's shared buffer whenever its next unit belongs to
// another tile; when all units are done the CTA adds its buffers into y (zeroed first) with one
// atomic per output, which also joins tiles split between neighbouring CTAs.
//
// Layouts in shared memory: codes of a unit as 16 rows of 128 bytes, 16-byte chunk j of row r
// stored at chunk j ^ (r % 8); x as boxes of 64 k x 8 tokens, chunk j of token g at j ^ g.  In
// every 8-lane phase the B-fragment reads of different tokens fall in different chunks, and
// MMA row m reads tile row prow(m) = (m/2) + 4 (m%2) (+8 for m >= 8), which puts the two rows of
// a phase in disjoint halves of the banks: the shared reads are conflict free.
constexpr int kDecWarps = 16;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecMaxTiles = 32;  // per-CTA tile buffers (16 rows x 8 tokens fp32 each)

template <int WF>
struct U3;
template <>
struct U3<W_DQ4> {  // 256 k per unit: codes 16 x 128 B, scales 16 x 16 B
  static constexpr int UK = 256, CODES = 2048, SCALES = 256, META = 0, SLOT = 2304;
};
template <>
struct U3<W_SQ4> {  // 512 k per unit: codes 16 x 128 B, scales 16 x 16 B, nibbles 16 x 64 B
  static constexpr int UK = 512, CODES = 2048, SCALES = 256, META = 1024, SLOT = 3328;
};

__device__ __forceinline__ int prow(int m) { return (m & 8) + ((m & 7) >> 1) + 4 * (m & 1); }

// Byte offset in the staged x of token g, column k (k % 8 == 0): box k / 64 of 1 KB, token row of
// 128 B, 16-byte chunk (k % 64) / 8 stored at chunk ^ g.
__device__ __forceinline__ uint32_t xoff(int g, int64_t k) {
  return (uint32_t)((k >> 6) * 1024 + g * 128 + ((((int)(k >> 3) & 7) ^ g) << 4));
}

// One warp copies unit (tile, kp) into `slot`: codes (four 16-byte pieces per lane, each four
// consecutive lanes' pieces one 128-byte row segment), block scales and 2:4 nibbles.
template <int WF>
__device__ __forceinline__ void issue_unit(uint8_t* slot, const SkinnyParams& p, int tile, int kp, int lane) {
  using U = U3<WF>;
  const int64_t crow = WF == W_DQ4 ? p.K / 2 : p.K / 4;
  const uint8_t* cbase = p.w + (int64_t)tile * 16 * crow + kp * 128;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int q = lane + 32 * t, r = q >> 3, j = q & 7;
    tc::cp_async16(slot + r * 128 + ((j ^ (r & 7)) << 4), cbase + r * crow + j * 16);
  }
  if (lane < 16) {
    const int64_t srow = WF == W_DQ4 ? p.K / 16 : p.K / 32;
    tc::cp_async16(slot + U::CODES + lane * 16, p.w_scales + ((int64_t)tile * 16 + lane) * srow + kp * 16);
  }
  if constexpr (U::META > 0) {
    const int64_t mrow = p.K / 8;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int q = lane + 32 * t, r = q >> 2, j = q & 3;
      tc::cp_async16(slot + U::CODES + U::SCALES + r * 64 + j * 16,
                     p.meta + ((int64_t)tile * 16 + r) * mrow + kp * 64 + j * 16);
    }
  }
}

// Dynamic shared memory of the decode kernel: the staged x columns (16 bytes per column) and
// every warp's DEPTH unit buffers.
template <int WF>
constexpr size_t decode_smem(int64_t xcols, int depth) {
  return 16 * (size_t)xcols + (size_t)kDecWarps * depth * U3<WF>::SLOT;
}
constexpr size_t kDecSmemMax = 227 * 1024 - sizeof(float) * kDecMaxTiles * 128;

// Work split of the decode kernel: k-groups of G units (G divides the units per tile).  A CTA's
// contiguous unit range must span at most two k-groups and touch at most kDecMaxTiles tiles;
// the smallest G of at least about 1024 k that satisfies this keeps the staged x small.
// Returns 0 when no G works; *xcols receives the x columns a CTA stages.
template <int WF>
int decode_group(const SkinnyParams& p, int64_t* xcols) {
  const int64_t uk = U3<WF>::UK, upr = p.K / uk, T = p.N / 16, grid = sm_count();
  const int64_t per_cta = (T * upr + grid - 1) / grid;
  const int64_t target = (1024 + uk - 1) / uk;
  for (int64_t g = 1; g <= upr; ++g) {
    if (upr % g || (g < target && g < upr)) continue;
    if (per_cta > T * g || per_cta / g + 3 > kDecMaxTiles) continue;
    const int64_t cols = (upr / g >= 2 ? 2 * g : g) * uk;
    if (decode_smem<WF>(cols, 2) > kDecSmemMax) return 0;
    *xcols = cols;
    return (int)g;
  }
  return 0;
}

template <int WF, typename T, int kDecDepth>
__global__ void __launch_bounds__(kDecThreads, 1) decode_gemv_kernel(const SkinnyParams p, int G) {
  using U = U3<WF>;
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float tbuf[kDecMaxTiles][16][8];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int upr = (int)(p.K / U::UK);           // units per 16-row tile
  const int NT16 = (int)(p.N / 16), TG = NT16 * G;  // tiles; units per k-group
  const int64_t U_all = (int64_t)NT16 * upr;         // < 2^31 (host check)
  const int ub = (int)(U_all * blockIdx.x / gridDim.x), ue = (int)(U_all * (blockIdx.x + 1) / gridDim.x);
  const int nunits = ue - ub;
  if (nunits <= 0) return;                      // whole CTA, before any barrier
  // unit u = (k-group kg, tile, kq): kp = kg * G + kq.  A CTA's range spans at most two k-groups
  // (host check); its tiles get shared-buffer slots: [tf, NT16) of kg_lo, then [0, tl] of kg_hi.
  const int kg_lo = ub / TG, kg_hi = (ue - 1) / TG;
  const int tf = (ub - kg_lo * TG) / G, tl = (ue - 1 - kg_hi * TG) / G;
  const int nlo = kg_lo == kg_hi ? tl - tf + 1 : NT16 - tf;
  const int nloc = kg_lo == kg_hi ? nlo : nlo + tl + 1;   // <= kDecMaxTiles (host check)
  const int64_t k0 = (int64_t)kg_lo * G * U::UK;          // x columns staged: [k0, k0 + kx)
  const int kx = (kg_hi - kg_lo + 1) * G * U::UK;
  uint8_t* xs = dsm;                            // 16 * kx bytes
  uint8_t* slots = dsm + 16 * kx;               // kDecWarps x kDecDepth x SLOT
  for (int i = threadIdx.x; i < nloc * 128; i += blockDim.x) (&tbuf[0][0][0])[i] = 0.f;

  // ---- x: one 16-byte piece per (token, 8 k); consecutive threads take consecutive pieces of a row
  const int kp8 = kx / 8;
  const uint16_t* xg = reinterpret_cast<const uint16_t*>(p.x) + k0;
  for (int i = threadIdx.x; i < 8 * kp8; i += blockDim.x) {
    const int g = i / kp8;
    const int k = (i - g * kp8) * 8;
    uint8_t* dst = xs + xoff(g, k);
    if (g < p.M)
      tc::cp_async16(dst, xg + (int64_t)g * p.K + k);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  tc::cp_async_commit();
  auto unit_at = [&](int u, int& slot, int& tile, int& kp) {
    const int kg = u / TG, rem = u - kg * TG;
    tile = rem / G;
    kp = kg * G + (rem - tile * G);
    slot = kg == kg_lo ? tile - tf : nlo + tile;
  };

  // ---- this warp's units: local index warp + kDecWarps * n; the first kDecDepth in flight now
  uint8_t* wslots = slots + warp * kDecDepth * U::SLOT;
#pragma unroll
  for (int d = 0; d < kDecDepth; ++d) {
    const int i = warp + kDecWarps * d;
    if (i < nunits) {
      int sl, tile, kp;
      unit_at(ub + i, sl, tile, kp);
      issue_unit<WF>(wslots + d * U::SLOT, p, tile, kp, lane);
    }
    tc::cp_async_commit();  // possibly empty: keeps the group count uniform
  }
  tc::cp_async_wait<kDecDepth>();  // this thread's x pieces have landed
  __syncthreads();                 // everyone's x pieces and the zeroed buffers are visible

  const int g = lane >> 2, c = lane & 3;
  const int r0 = prow(g), r1 = prow(g + 8);
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
  int cur = -1;
  auto flush = [&]() {
    float* b = &tbuf[cur][0][0];
    atomicAdd(b + r0 * 8 + 2 * c, acc[0] + acc2[0]);
    atomicAdd(b + r0 * 8 + 2 * c + 1, acc[1] + acc2[1]);
    atomicAdd(b + r1 * 8 + 2 * c, acc[2] + acc2[2]);
    atomicAdd(b + r1 * 8 + 2 * c + 1, acc[3] + acc2[3]);
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = acc2[q] = 0.f;
  };
  for (int n = 0, i = warp; i < nunits; ++n, i += kDecWarps) {
    int slt, tile, kp;
    unit_at(ub + i, slt, tile, kp);
    if (slt != cur) {
      if (cur >= 0) flush();
      cur = slt;
    }
    tc::cp_async_wait<kDecDepth - 1>();  // this unit's group (all but the newest) has landed
    __syncwarp();
    uint8_t* slot = wslots + (n % kDecDepth) * U::SLOT;
    const uint8_t* d = slot;
    const uint8_t* sc = d + U::CODES;
    if constexpr (WF == W_DQ4) {
      // the unit's two 128-k chunks feed two independent accumulator chains
      uint32_t w0[2][4], w1[2][4], sa[2][2], sb[2][2];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int j = 4 * ch + c;
        const uint4 v0 = *reinterpret_cast<const uint4*>(d + r0 * 128 + ((j ^ (r0 & 7)) << 4));
        const uint4 v1 = *reinterpret_cast<const uint4*>(d + r1 * 128 + ((j ^ (r1 & 7)) << 4));
        w0[ch][0] = v0.x; w0[ch][1] = v0.y; w0[ch][2] = v0.z; w0[ch][3] = v0.w;
        w1[ch][0] = v1.x; w1[ch][1] = v1.y; w1[ch][2] = v1.z; w1[ch][3] = v1.w;
        scale_pair<T>(*reinterpret_cast<const uint16_t*>(sc + r0 * 16 + 8 * ch + 2 * c), sa[ch][0], sa[ch][1]);
        scale_pair<T>(*reinterpret_cast<const uint16_t*>(sc + r1 * 16 + 8 * ch + 2 * c), sb[ch][0], sb[ch][1]);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          // x[g][P .. P+8), P = chunk base + 32c + 8q: codes at nibbles (i, i+4) of word q pair
          // with x entries (i, i+4)
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + xoff(g, kp * 256 - k0 + ch * 128 + 32 * c + 8 * q));
          const uint32_t s0 = sa[ch][q >> 1], s1 = sb[ch][q >> 1];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t xa = h ? xv.y : xv.x, xb = h ? xv.w : xv.z;
            const uint2 bx = make_uint2(__byte_perm(xa, xb, 0x5410), __byte_perm(xa, xb, 0x7632));
            const uint32_t a0 = hmul2u<T>(fp4_pair_i4<T>(w0[ch][q], 2 * h), s0);
            const uint32_t a2 = hmul2u<T>(fp4_pair_i4<T>(w0[ch][q], 2 * h + 1), s0);
            const uint32_t a1 = hmul2u<T>(fp4_pair_i4<T>(w1[ch][q], 2 * h), s1);
            const uint32_t a3 = hmul2u<T>(fp4_pair_i4<T>(w1[ch][q], 2 * h + 1), s1);
            mma_k16<T>(ch ? acc2 : acc, a0, a1, a2, a3, bx);
          }
        }
      }
    } else {
      // even and odd windows feed two independent accumulator chains
      const uint8_t* me = sc + U::SCALES;
#pragma unroll 4
      for (int w = 0; w < 16; ++w) {
        const uint32_t m0 = *reinterpret_cast<const uint32_t*>(me + r0 * 64 + 4 * w);
        const uint32_t m1 = *reinterpret_cast<const uint32_t*>(me + r1 * 64 + 4 * w);
        const uint32_t e = __byte_perm(m0, m1, (c & 1) ? 0x7632 : 0x5410);
        const uint2 v0 = *reinterpret_cast<const uint2*>(d + r0 * 128 + (((w >> 1) ^ (r0 & 7)) << 4) + 8 * (w & 1));
        const uint2 v1 = *reinterpret_cast<const uint2*>(d + r1 * 128 + (((w >> 1) ^ (r1 & 7)) << 4) + 8 * (w & 1));
        uint32_t s0, s1, unused;
        scale_pair<T>(sc[r0 * 16 + w], s0, unused);
        scale_pair<T>(sc[r1 * 16 + w], s1, unused);
        const uint32_t b0 = __byte_perm(v0.x, v0.y, c | ((c + 4) << 4));
        const uint32_t b1 = __byte_perm(v1.x, v1.y, c | ((c + 4) << 4));
        const uint32_t a0 = hmul2u<T>(fp4_pair_byte<T>(b0, 0), s0);
        const uint32_t a2 = hmul2u<T>(fp4_pair_byte<T>(b0, 1), s0);
        const uint32_t a1 = hmul2u<T>(fp4_pair_byte<T>(b1, 0), s1);
        const uint32_t a3 = hmul2u<T>(fp4_pair_byte<T>(b1, 1), s1);
        // x[g][32w' + 2c + 8i + {0, 1}], i = 0..3: word c of four consecutive 16-byte pieces
        const int64_t kw = (int64_t)kp * 512 - k0 + 32 * w;
        const uint8_t* xr = xs + 4 * c;
        const uint4 bx = make_uint4(*reinterpret_cast<const uint32_t*>(xr + xoff(g, kw)),
                                    *reinterpret_cast<const uint32_t*>(xr + xoff(g, kw + 8)),
                                    *reinterpret_cast<const uint32_t*>(xr + xoff(g, kw + 16)),
                                    *reinterpret_cast<const uint32_t*>(xr + xoff(g, kw + 24)));
        mma_sp_k32<T>((w & 1) ? acc2 : acc, a0, a1, a2, a3, bx, e);
      }
    }
    __syncwarp();  // every lane is done with the slot before it is refilled
    const int inext = i + kDecWarps * kDecDepth;
    if (inext < nunits) {
      int s2, t2, k2;
      unit_at(ub + inext, s2, t2, k2);
      issue_unit<WF>(slot, p, t2, k2, lane);
    }
    tc::cp_async_commit();
  }
  if (cur >= 0) flush();
  tc::cp_async_wait<0>();  // nothing in flight (the trailing groups are empty)
  __syncthreads();
  // ---- the CTA's tile sums into y
  const float scale = 256.0f * *p.w_ts;
  for (int e = threadIdx.x; e < nloc * 128; e += blockDim.x) {
    const int lt = e >> 7, row = (e >> 3) & 15, tok = e & 7;
    const int tile = lt < nlo ? tf + lt : lt - nlo;
    const int64_t gr = (int64_t)tile * 16 + row;
    const float v = (&tbuf[0][0][0])[e];
    if (tok < p.M && gr < p.N && v != 0.0f) atomicAdd(p.y + (int64_t)tok * p.N + gr, v * scale);
  }
}

template <int WF, typename T>
int launch_decode(const SkinnyParams& p, cudaStream_t s) {
  int64_t xcols = 0;
  const int G = decode_group<WF>(p, &xcols);
  if (!G) return SP24_ERR_UNSUPPORTED;
  // three units in flight per warp when they fit beside x, else two
  const bool deep = decode_smem<WF>(xcols, 3) <= kDecSmemMax;
  const size_t smem = decode_smem<WF>(xcols, deep ? 3 : 2);
  auto kern = deep ? decode_gemv_kernel<WF, T, 3> : decode_gemv_kernel<WF, T, 2>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  if (cudaMemsetAsync(p.y, 0, (size_t)(p.M * p.N) * sizeof(float), s) != cudaSuccess) return SP24_ERR_CUDA;
  kern<<<sm_count(), kDecThreads, smem, s>>>(p, G);
  return launch_status();
}

// ------------------------------------------------------------------ decode GEMV, whole tiles per CTA
//
// When there are at least as many 16-row tiles as SMs, each CTA owns a contiguous range of whole
// tiles.  A tile's codes (and block scales, and 2:4 nibbles) over the full K are one contiguous
// block of memory, so thread 0 fetches each with a single bulk copy into a ring of tile slots
// (bulk copies cost ~30 ns each to issue and move large requests at full speed; tensor copies of
// narrow boxes do not), and x arrives first with one bulk copy of its M rows; the tile copies are
// issued once x has landed, so x does not share the SM's inbound bandwidth with them.
//
// Warp w owns the K range [256 w, 256 w + 256) of every tile (K / 256 warps): its x fragments for
// that range are loaded once, into registers, as f16.  bf16 x is converted as is when the warp's
// largest |x| lies in [2^-8, 2^15) (f16 keeps bf16's 8 significant bits there; values below 2^-14
// round to f16 subnormals, an error under 2^-25 against a maximum of at least 2^-8); otherwise it
// is first multiplied by a power of two 2^S that brings the maximum into [2^14, 2^15), and the
// warp's partial sums are multiplied back by 2^-S.  NVFP4 codes become f16 pairs by the sm_100a
// conversion instruction (E2M1 exact in f16) times their E4M3 block scale (exact: at most five
// significant bits, magnitudes at most 2688), and feed mma.m16n8k16 (dense) or mma.sp m16n8k32
// (2:4) with fp32 accumulation; a measured loop of conversions, scale multiplies and MMAs runs as
// fast as the MMAs alone.  Every warp adds its partial sums into the tile's shared buffer and
// releases the slot; the CTA writes its tiles' outputs at the end with plain stores: every output
// has exactly one writer, so y needs no zeroing and no atomics.
//
// Dense fragments: chunk j (128 entries at k0 = 256 w + 128 j): lane (g, c) holds the 32 codes
// k0 + 32c .. +31 (two E4M3 blocks) of rows g and g + 8 in one 16-byte load each; MMA m of the
// chunk takes codes k0 + 32c + 4m .. +3 (bytes 2m, 2m+1) and x[g][the same four entries].  2:4
// fragments: window pair q = 4w + j: lane (g, c) supplies the kept pair of groups c and c+4 of each
// 32-wide window, B = x[g][32v + 2c + 8i .. +1] for i = 0..3, and the nibbles as in the skinny
// kernel above.
constexpr int kTileMaxLocal = 32;
constexpr int kTileMaxBuf = 4;
constexpr int kTileKW = 256;  // K entries per warp

template <int WF>
struct TileGeom {
  int64_t cb, sb, mb;  // bytes per row: codes, block scales, nibbles
  __host__ __device__ explicit TileGeom(int64_t K)
      : cb(WF == W_DQ4 ? K / 2 : K / 4), sb(WF == W_DQ4 ? K / 16 : K / 32), mb(WF == W_SQ4 ? K / 8 : 0) {}
  __host__ __device__ int64_t bytes() const { return 16 * (cb + sb + mb); }
};

// x row pitch in shared memory: 2K bytes plus 32 (dense) or 16 (2:4), so that the fragment loads
// below are bank-conflict free.
template <int WF>
__host__ __device__ int64_t x_pitch(int64_t K) { return 2 * K + (WF == W_DQ4 ? 32 : 16); }

// Dynamic shared memory: nbuf tile buffers, x (M padded rows), per-tile sums.
template <int WF>
size_t tile_smem(int64_t M, int64_t K, int nbuf, int64_t local_tiles) {
  return (size_t)nbuf * TileGeom<WF>(K).bytes() + (size_t)M * (size_t)x_pitch<WF>(K) + (size_t)local_tiles * 512;
}

// f16 pair <- bf16 pair times sf (a power of two), through f32 (the rounding only touches values
// below f16's normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float sf) {
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16) * sf, __uint_as_float(w & 0xffff0000u) * sf);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Scale exponent S for a warp whose largest |x| has the bf16 magnitude bits m: 0 when m is 0,
// infinite, NaN or in [2^-8, 2^15); else the S with max|x| 2^S in [2^14, 2^15).
__device__ __forceinline__ int x_scale_exp(uint32_t m) {
  if (m == 0 || m >= 0x7f80u || (m >= 0x3B80u && m < 0x4700u)) return 0;
  const int e = (int)(m >> 7) - 127;  // subnormal: -127
  const int s = 14 - e;
  return s > 126 ? 126 : s;
}

template <int WF, typename T, int XI>
__global__ void __launch_bounds__(640, 1) decode_tile_kernel(const SkinnyParams p, int nbuf) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ uint64_t full_bar[kTileMaxBuf], empty_bar[kTileMaxBuf], x_bar;
  __shared__ int issued, abort_flag;
  const TileGeom<WF> tg(p.K);
  uint8_t* bufs = dsm;
  const int64_t xp = x_pitch<WF>(p.K);
  const uint8_t* xs = bufs + nbuf * tg.bytes();                                 // x rows [M][xp]
  float* tbuf = reinterpret_cast<float*>(bufs + nbuf * tg.bytes() + p.M * xp);  // [tile][16][8]
  const int W = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT16 = (int)(p.N / 16);
  const int t0 = (int)((int64_t)NT16 * blockIdx.x / gridDim.x), t1 = (int)((int64_t)NT16 * (blockIdx.x + 1) / gridDim.x);
  const int ntiles = t1 - t0;  // >= 1 (host: tiles >= grid), <= kTileMaxLocal
  // ---- copies: x (one row per copy, into padded rows), then each tile's codes / scales /
  // nibbles, one bulk copy apiece, all issued by thread 0 as its first work; tile i goes to slot
  // i % nbuf once the tile that held it has been released by every warp
  auto issue_tile = [&](int i) {
    const int sl = i % nbuf;
    uint8_t* d = bufs + sl * tg.bytes();
    const int64_t row = (int64_t)(t0 + i) * 16;
    tc::mbar_arrive_expect_tx(&full_bar[sl], (uint32_t)tg.bytes());
    stream::bulk_g2s(d, p.w + row * tg.cb, (uint32_t)(16 * tg.cb), &full_bar[sl]);
    stream::bulk_g2s(d + 16 * tg.cb, p.w_scales + row * tg.sb, (uint32_t)(16 * tg.sb), &full_bar[sl]);
    if (WF == W_SQ4) stream::bulk_g2s(d + 16 * (tg.cb + tg.sb), p.meta + row * tg.mb, (uint32_t)(16 * tg.mb), &full_bar[sl]);
    issued = i + 1;
  };
  if (threadIdx.x == 0) {
    tc::mbar_init(&x_bar, 1);
    for (int i = 0; i < nbuf; ++i) {
      tc::mbar_init(&full_bar[i], 1);
      tc::mbar_init(&empty_bar[i], W);
    }
    abort_flag = 0;
    issued = 0;
    tc::fence_mbar_init();
    tc::mbar_arrive_expect_tx(&x_bar, (uint32_t)(p.M * 2 * p.K));
    const uint8_t* xg = reinterpret_cast<const uint8_t*>(p.x);
    for (int r = 0; r < p.M; ++r)
      stream::bulk_g2s(const_cast<uint8_t*>(xs) + r * xp, xg + (int64_t)r * 2 * p.K, (uint32_t)(2 * p.K), &x_bar);
    for (int i = 0; i < ntiles && i < nbuf; ++i) issue_tile(i);
  }
  for (int i = threadIdx.x; i < ntiles * 128; i += blockDim.x) tbuf[i] = 0.f;
  __syncthreads();  // barriers initialised, sums zeroed

  const int g = lane >> 2, c = lane & 3;
  // every wait is decided warp-uniformly (the MMAs need the whole warp)
  bool ok = __all_sync(0xffffffffu, mbar_wait(&x_bar, 0));
  if (!ok && lane == 0) {
    set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
    abort_flag = 1;
  }
  // x fragments of this warp's K range (token rows past M: zeros)
  const int k0 = kTileKW * warp;
  uint32_t xf[XI][16];
  {
    const uint8_t* xg = xs + (int64_t)g * xp;
    const bool live = ok && g < p.M;
#pragma unroll
    for (int j = 0; j < XI; ++j) {
      if constexpr (WF == W_DQ4) {
        // load h takes piece (h + c / 2) % 4 of the lane's four 16-byte pieces: with the row
        // pitch 32 bytes past a multiple of 128, the 8 lanes of each quarter-warp then read 8
        // different bank groups; the pieces are put back in order after
        uint4 v[4];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          v[h] = live ? *reinterpret_cast<const uint4*>(xg + 2 * (k0 + 128 * j + 32 * c) + 16 * ((h + (c >> 1)) & 3))
                      : make_uint4(0u, 0u, 0u, 0u);
        const bool rot = c >= 2;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint4 u = rot ? v[(h + 3) & 3] : v[h];
          xf[j][4 * h] = u.x; xf[j][4 * h + 1] = u.y; xf[j][4 * h + 2] = u.z; xf[j][4 * h + 3] = u.w;
        }
      } else {
        // window pairs 2j, 2j + 1 of the warp (windows 4j .. 4j + 3)
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int t = 0; t < 4; ++t)
            xf[j][4 * u + t] = live ? *reinterpret_cast<const uint32_t*>(xg + 2 * (k0 + 32 * (4 * j + u) + 2 * c + 8 * t)) : 0u;
      }
    }
  }
  float descale = 1.0f;  // 2^-S of x
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat162 mx = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < XI; ++j)
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const uint32_t a = xf[j][t] & 0x7fff7fffu;
        mx = __hmax2(mx, *reinterpret_cast<const __nv_bfloat162*>(&a));
      }
    const uint32_t mb2 = *reinterpret_cast<const uint32_t*>(&mx);
    const uint32_t m = __reduce_max_sync(0xffffffffu, max(mb2 & 0xffffu, mb2 >> 16));
    const int S = x_scale_exp(m);
    const float sf = __int_as_float((127 + S) << 23);
    descale = __int_as_float((127 - S) << 23);
#pragma unroll
    for (int j = 0; j < XI; ++j)
#pragma unroll
      for (int t = 0; t < 16; ++t) xf[j][t] = bf16x2_to_f16x2(xf[j][t], sf);
  }
  const int r0 = g, r1 = g + 8;
  for (int i = 0; ok && i < ntiles; ++i) {
    const int sl = i % nbuf;
    if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[sl], (i / nbuf) & 1))) {
      if (lane == 0) {
        set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
        abort_flag = 1;
      }
      break;
    }
    const uint8_t* d = bufs + sl * tg.bytes();
    const uint8_t* sc = d + 16 * tg.cb;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
    // 2:4: the block scales of the warp's four window pairs in one 8-byte load per row, and below
    // the nibbles of two pairs in one 16-byte load per row, instead of narrow loads per pair
    uint2 sw0, sw1;
    if constexpr (WF == W_SQ4) {
      sw0 = *reinterpret_cast<const uint2*>(sc + r0 * tg.sb + 8 * warp);
      sw1 = *reinterpret_cast<const uint2*>(sc + r1 * tg.sb + 8 * warp);
    }
#pragma unroll
    for (int j = 0; j < XI; ++j) {
      float(&a)[4] = (j & 1) ? acc2 : acc;
      if constexpr (WF == W_DQ4) {
        const int kb = (k0 + 128 * j + 32 * c) / 2;  // byte of the lane's codes in a row
        const uint4 v0 = *reinterpret_cast<const uint4*>(d + r0 * tg.cb + kb);
        const uint4 v1 = *reinterpret_cast<const uint4*>(d + r1 * tg.cb + kb);
        const int sbk = (k0 + 128 * j + 32 * c) / 16;
        const uint32_t h0 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(sc + r0 * tg.sb + sbk));
        const uint32_t h1 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(sc + r1 * tg.sb + sbk));
        const uint32_t w0[4] = {v0.x, v0.y, v0.z, v0.w}, w1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {  // E4M3 block hb: MMAs 4 hb .. 4 hb + 3
          const uint32_t s0 = __byte_perm(h0, 0u, hb ? 0x3232 : 0x1010), s1 = __byte_perm(h1, 0u, hb ? 0x3232 : 0x1010);
#pragma unroll
          for (int ww = 0; ww < 2; ++ww) {  // word 2 hb + ww: MMAs 4 hb + 2 ww, +1
            uint32_t c0[4], c1[4];
            e2m1x8_to_f16x2(w0[2 * hb + ww], c0[0], c0[1], c0[2], c0[3]);
            e2m1x8_to_f16x2(w1[2 * hb + ww], c1[0], c1[1], c1[2], c1[3]);
#pragma unroll
            for (int mm = 0; mm < 2; ++mm) {
              const int m = 4 * hb + 2 * ww + mm;
              mma_k16<__half>(a, hmul2u<__half>(c0[2 * mm], s0), hmul2u<__half>(c1[2 * mm], s1),
                              hmul2u<__half>(c0[2 * mm + 1], s0), hmul2u<__half>(c1[2 * mm + 1], s1),
                              make_uint2(xf[j][2 * m], xf[j][2 * m + 1]));
            }
          }
        }
      } else {
        const uint8_t* me = sc + 16 * tg.sb;
        const uint4 mq0 = *reinterpret_cast<const uint4*>(me + r0 * tg.mb + 8 * (4 * warp + 2 * j));
        const uint4 mq1 = *reinterpret_cast<const uint4*>(me + r1 * tg.mb + 8 * (4 * warp + 2 * j));
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {  // window pair q = 4w + p, p = 2j + pp
          const int p = 2 * j + pp, q = 4 * warp + p;
          const uint4 c0 = *reinterpret_cast<const uint4*>(d + r0 * tg.cb + 16 * q);
          const uint4 c1 = *reinterpret_cast<const uint4*>(d + r1 * tg.cb + 16 * q);
          const uint2 m0 = pp ? make_uint2(mq0.z, mq0.w) : make_uint2(mq0.x, mq0.y);
          const uint2 m1 = pp ? make_uint2(mq1.z, mq1.w) : make_uint2(mq1.x, mq1.y);
          const uint32_t h0 = e4m3x2_to_f16x2(((p >> 1) ? sw0.y : sw0.x) >> (16 * (p & 1)));
          const uint32_t h1 = e4m3x2_to_f16x2(((p >> 1) ? sw1.y : sw1.x) >> (16 * (p & 1)));
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint32_t e = __byte_perm(u ? m0.y : m0.x, u ? m1.y : m1.x, (c & 1) ? 0x7632 : 0x5410);
            const uint32_t s0 = __byte_perm(h0, 0u, u ? 0x3232 : 0x1010), s1 = __byte_perm(h1, 0u, u ? 0x3232 : 0x1010);
            const uint32_t b0 = __byte_perm(u ? c0.z : c0.x, u ? c0.w : c0.y, c | ((c + 4) << 4));
            const uint32_t b1 = __byte_perm(u ? c1.z : c1.x, u ? c1.w : c1.y, c | ((c + 4) << 4));
            uint32_t a0, a2, a1, a3;
            e2m1x4_to_f16x2(b0, a0, a2);
            e2m1x4_to_f16x2(b1, a1, a3);
            const int v = 2 * pp + u;  // window of the j-th group of four
            mma_sp_k32<__half>(a, hmul2u<__half>(a0, s0), hmul2u<__half>(a1, s1), hmul2u<__half>(a2, s0),
                               hmul2u<__half>(a3, s1),
                               make_uint4(xf[j][4 * v], xf[j][4 * v + 1], xf[j][4 * v + 2], xf[j][4 * v + 3]), e);
          }
        }
      }
    }
    float* bt = tbuf + i * 128;
    atomicAdd(bt + r0 * 8 + 2 * c, (acc[0] + acc2[0]) * descale);
    atomicAdd(bt + r0 * 8 + 2 * c + 1, (acc[1] + acc2[1]) * descale);
    atomicAdd(bt + r1 * 8 + 2 * c, (acc[2] + acc2[2]) * descale);
    atomicAdd(bt + r1 * 8 + 2 * c + 1, (acc[3] + acc2[3]) * descale);
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty_bar[sl]);
    if (warp == 0 && i + nbuf < ntiles) {
      int released = 1;
      if (lane == 0) {
        released = mbar_wait(&empty_bar[sl], (i / nbuf) & 1) ? 1 : 0;
        if (released) {
          issue_tile(i + nbuf);
        } else {
          set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
          abort_flag = 1;
        }
      }
      if (!__shfl_sync(0xffffffffu, released, 0)) break;
    }
  }
  __syncthreads();
  // a gave-up wait may leave copies in flight: let them land before the CTA's memory goes away
  if (abort_flag && threadIdx.x == 0) {
    tc::mbar_wait(&x_bar, 0);
    for (int i = issued > nbuf ? issued - nbuf : 0; i < issued; ++i) tc::mbar_wait(&full_bar[i % nbuf], (i / nbuf) & 1);
  }
  // ---- the CTA's tiles into y, one writer per output
  const float scale = *p.w_ts;
  for (int e = threadIdx.x; e < ntiles * 128; e += blockDim.x) {
    const int lt = e >> 7, row = (e >> 3) & 15, tok = e & 7;
    if (tok < p.M) p.y[(int64_t)tok * p.N + (int64_t)(t0 + lt) * 16 + row] = tbuf[e] * scale;
  }
}

// Tile slots: as many as fit beside x and the per-tile sums, up to kTileMaxBuf.
template <int WF>
int tile_buffers(int64_t M, int64_t K, int64_t local) {
  int nbuf = kTileMaxBuf;
  while (nbuf >= 2 && tile_smem<WF>(M, K, nbuf, local) > 227 * 1024 - 1024) --nbuf;
  return nbuf;
}

template <int WF, typename T>
int launch_tile(const SkinnyParams& p, cudaStream_t s) {
  const int grid = sm_count();
  const int64_t T16 = p.N / 16, local = (T16 + grid - 1) / grid;
  const int nbuf = tile_buffers<WF>(p.M, p.K, local);
  const size_t smem = tile_smem<WF>(p.M, p.K, nbuf, local);
  const int warps = (int)(p.K / kTileKW);
  auto kern = decode_tile_kernel<WF, T, 2>;  // two 128-entry chunks (dense) / two window-pair groups (2:4)
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  kern<<<grid, warps * 32, smem, s>>>(p, nbuf);
  return launch_status();
}

}  // namespace

// Grouped launch: grid.z = max_tiles token tiles (<= 64 tokens each, NT = 8); y must be zeroed
// by the caller when K spans several slices (results are accumulated).
int skinny2_grouped(int wf, int t16, SkinnyParams p, int64_t max_tiles, cudaStream_t s) {
  if (max_tiles <= 0) return SP24_OK;
  if (max_tiles > 65535) return SP24_ERR_UNSUPPORTED;
  const int kc = wf == W_D16 ? F2<W_D16>::KC : wf == W_DQ4 ? F2<W_DQ4>::KC : wf == W_S16 ? F2<W_S16>::KC : F2<W_SQ4>::KC;
  p.accumulate = (p.K + kc - 1) / kc > 1;
  p.M = 64;
  const bool bf = t16 == SP24_BF16;
  const unsigned z = (unsigned)max_tiles;
  switch (wf) {
    case W_D16: return bf ? launch2<W_D16, __nv_bfloat16, true>(p, 8, s, z) : launch2<W_D16, __half, true>(p, 8, s, z);
    case W_DQ4: return bf ? launch2<W_DQ4, __nv_bfloat16, true>(p, 8, s, z) : launch2<W_DQ4, __half, true>(p, 8, s, z);
    case W_S16: return bf ? launch2<W_S16, __nv_bfloat16, true>(p, 8, s, z) : launch2<W_S16, __half, true>(p, 8, s, z);
    case W_SQ4: return bf ? launch2<W_SQ4, __nv_bfloat16, true>(p, 8, s, z) : launch2<W_SQ4, __half, true>(p, 8, s, z);
  }
  return SP24_ERR_UNSUPPORTED;
}

// True when the persistent decode kernel takes the problem: 16-bit x of at most 8 tokens
// (16-byte aligned rows), NVFP4 weights (dense or 2:4) in whole 16-row tiles, K a whole number of
// units, and a k-group split that fits (decode_group).
bool decode_supported(int wf, const SkinnyParams& p) {
  if (p.x_fmt != X_16 || p.M > 8 || p.M < 1 || p.N % 16 || p.N == 0 || p.K == 0) return false;
  if (!aligned(p.x, 16) || !aligned(p.w, 16) || !aligned(p.w_scales, 16)) return false;
  if ((p.N / 16) * (p.K / 256) >= (int64_t(1) << 31)) return false;
  int64_t xcols;
  if (wf == W_DQ4) return p.K % U3<W_DQ4>::UK == 0 && decode_group<W_DQ4>(p, &xcols) > 0;
  if (wf == W_SQ4) return aligned(p.meta, 16) && p.K % U3<W_SQ4>::UK == 0 && decode_group<W_SQ4>(p, &xcols) > 0;
  return false;
}

// True when the whole-tile decode kernel takes the problem: 16-bit x of at most 8 tokens,
// NVFP4 weights (dense or 2:4) with K a multiple of 256 up to 5120 (one warp per 256 entries of
// K, at most 20 warps), at least one 16-row tile per SM and at most kTileMaxLocal tiles per CTA,
// 16-byte aligned operands, and x plus two tile buffers in shared memory.
bool decode_tile_supported(int wf, const SkinnyParams& p) {
  if (p.x_fmt != X_16 || p.M > 8 || p.M < 1 || p.N % 16 || p.K == 0 || p.K % kTileKW || p.K > 20 * kTileKW) return false;
  if (!aligned(p.x, 16) || !aligned(p.w, 16) || !aligned(p.w_scales, 16) || !aligned(p.y, 4)) return false;
  const int64_t T16 = p.N / 16, grid = sm_count(), local = (T16 + grid - 1) / grid;
  if (T16 < grid || local > kTileMaxLocal) return false;
  if (wf == W_DQ4) return tile_smem<W_DQ4>(p.M, p.K, 2, local) <= 227 * 1024 - 1024;
  if (wf == W_SQ4) return aligned(p.meta, 16) && tile_smem<W_SQ4>(p.M, p.K, 2, local) <= 227 * 1024 - 1024;
  return false;
}

int decode_tile(int wf, int t16, const SkinnyParams& p, cudaStream_t s) {
  const bool bf = t16 == SP24_BF16;
  if (wf == W_DQ4) return bf ? launch_tile<W_DQ4, __nv_bfloat16>(p, s) : launch_tile<W_DQ4, __half>(p, s);
  if (wf == W_SQ4) return bf ? launch_tile<W_SQ4, __nv_bfloat16>(p, s) : launch_tile<W_SQ4, __half>(p, s);
  return SP24_ERR_UNSUPPORTED;
}

int decode_gemv(int wf, int t16, const SkinnyParams& p, cudaStream_t s) {
  const bool bf = t16 == SP24_BF16;
  if (wf == W_DQ4) return bf ? launch_decode<W_DQ4, __nv_bfloat16>(p, s) : launch_decode<W_DQ4, __half>(p, s);
  if (wf == W_SQ4) return bf ? launch_decode<W_SQ4, __nv_bfloat16>(p, s) : launch_decode<W_SQ4, __half>(p, s);
  return SP24_ERR_UNSUPPORTED;
}

// True when the shared-memory staged skinny kernel can take this problem: every row slice of
// every array starts 16-byte aligned and has a 16-byte multiple length.
bool skinny2_supported(int wf, const SkinnyParams& p) {
  if (p.M > 64 || p.K == 0) return false;
  if (!aligned(p.w, 16)) return false;
  switch (wf) {
    case W_D16: return p.K % 8 == 0;
    case W_DQ4: return p.K % 256 == 0 && aligned(p.w_scales, 16);
    case W_S16: return p.K % 128 == 0 && aligned(p.meta, 16);
    case W_SQ4: return p.K % 512 == 0 && aligned(p.w_scales, 16) && aligned(p.meta, 16);
  }
  return false;
}

int skinny2_gemm(int wf, int t16, SkinnyParams p, cudaStream_t s) {
  const int kc = wf == W_D16 ? F2<W_D16>::KC : wf == W_DQ4 ? F2<W_DQ4>::KC : wf == W_S16 ? F2<W_S16>::KC : F2<W_SQ4>::KC;
  const int64_t slices = (p.K + kc - 1) / kc;
  p.accumulate = slices > 1;
  if (p.accumulate && cudaMemsetAsync(p.y, 0, (size_t)(p.M * p.N) * sizeof(float), s) != cudaSuccess)
    return SP24_ERR_CUDA;
  const int nt = p.M <= 8 ? 1 : p.M <= 16 ? 2 : p.M <= 32 ? 4 : 8;
  const bool bf = t16 == SP24_BF16;
  switch (wf) {
    case W_D16: return bf ? launch2<W_D16, __nv_bfloat16>(p, nt, s) : launch2<W_D16, __half>(p, nt, s);
    case W_DQ4: return bf ? launch2<W_DQ4, __nv_bfloat16>(p, nt, s) : launch2<W_DQ4, __half>(p, nt, s);
    case W_S16: return bf ? launch2<W_S16, __nv_bfloat16>(p, nt, s) : launch2<W_S16, __half>(p, nt, s);
    case W_SQ4: return bf ? launch2<W_SQ4, __nv_bfloat16>(p, nt, s) : launch2<W_SQ4, __half>(p, nt, s);
  }
  return SP24_ERR_UNSUPPORTED;
}

}  // namespace sp24
