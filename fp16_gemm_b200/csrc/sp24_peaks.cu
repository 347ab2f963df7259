// Roofline denominators measured on this device by this library's own instructions.
//
// Tensor pipe: one CTA per SM (or per CTA pair for the pair shape) issues back-to-back tcgen05
// MMAs of M = 128 (256 for the pair), N = 256 from shared-memory operands filled with non-zero
// pseudo-random data (E2M1 codes of every magnitude, 16-bit values of unit range, E4M3 scales
// of 1.0, legal 2:4 / pairwise metadata), accumulating into TMEM, and times the loop with
// %globaltimer between one commit before and one after.  Kinds: 0 kind::f16 (bf16, K = 16),
// 1 .sp kind::f16 (K = 32 logical), 2 kind::mxf4nvf4 block16 (K = 64), 3 .sp kind::mxf4nvf4
// (K = 128 logical), 4 kind::mxf4nvf4 on a CTA pair (cta_group::2, M = 256, K = 64).
// HBM: a grid-stride stream of 16-byte non-caching loads over a buffer, reduced into one word so
// nothing is optimised away.
// Every wait is bounded by the library's wait limit; nothing here reads or writes out of bounds.
#include "sp24_tc.cuh"

namespace sp24 {
namespace {

using namespace tc;

__device__ __forceinline__ uint32_t mix(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352du;
  x ^= x >> 15;
  x *= 0x846ca68bu;
  x ^= x >> 16;
  return x;
}

template <bool PAIR>
__device__ __forceinline__ void sync_all() {
  if (PAIR) cluster_sync_all();
  else __syncthreads();
}

// kind: see the file comment.  out[cta] = nanoseconds for `rounds` x 4 MMAs (written by the
// issuing CTA; the odd CTA of a pair writes 0).
template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int rounds, unsigned long long* out) {
  constexpr bool PAIR = KIND == 4;
  constexpr bool FP4 = KIND >= 2;
  constexpr bool SP = KIND == 1 || KIND == 3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  // A: 128 rows x 128 bytes, B: 256 rows x 128 bytes (PAIR: 128 rows per CTA), 128B swizzle;
  // then 16 KB of copy sources: 8 KB of E4M3 scales 1.0 (0x38), 8 KB of metadata bytes 0x44
  // (every nibble the legal index pair 0, 1)
  uint8_t* sA = smem;
  uint8_t* sB = smem + 16384;
  uint8_t* sX = smem + 16384 + 32768;
  __shared__ uint64_t done_bar;
  __shared__ uint32_t tmem_base;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0;
  const bool issuer = !PAIR || rank == 0;
  for (int i = threadIdx.x; i < (16384 + 32768) / 4; i += blockDim.x) {
    uint32_t r = mix(i * 2654435761u + blockIdx.x);
    if (!FP4) r &= 0xbfffbfffu, r |= 0x3c003c00u;  // bf16 values in [1, 2) x 2^(-7..0), both signs
    reinterpret_cast<uint32_t*>(sA)[i] = r;
  }
  for (int i = threadIdx.x; i < 16384 / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sX)[i] = i < 2048 ? 0x38383838u : 0x44444444u;
  if (threadIdx.x == 0) {
    mbar_init(&done_bar, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    if (PAIR) tmem_alloc_pair(&tmem_base, 512);
    else tmem_alloc(&tmem_base, 512);
  }
  tc_fence_before();
  sync_all<PAIR>();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (issuer && threadIdx.x == 0) {
    const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA));
    const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB));
    const uint64_t x0 = desc_rows16_noswizzle(smem_u32(sX));
    // TMEM columns 256-319 <- scales (source bytes 0 - 8191), 320-383 <- metadata (8192 - 16383),
    // once; SFA at 256 + 4q, SFB at 272 + 8q, metadata at 320 + 2q (even columns)
    for (int c = 0; c < 32; ++c) {
      if (PAIR) tmem_cp_32x128b_x4_pair(tmem + 256 + 4 * c, x0 + 32 * c);
      else if (FP4 || SP) tmem_cp_32x128b_x4(tmem + 256 + 4 * c, x0 + 32 * c);
    }
    const uint32_t sfa = tmem + 256, sfb = tmem + 256 + 16, meta = tmem + 256 + 64;
    const uint32_t idesc = KIND == 0 ? idesc_f16(128, 256, true)
                           : KIND == 1 ? idesc_f16(128, 256, true, true)
                           : KIND == 2 ? idesc_nvfp4(128, 256)
                           : KIND == 3 ? idesc_nvfp4(128, 256, true)
                                       : idesc_nvfp4(256, 256);
    uint64_t t0 = 0;
    for (int r = -1; r < rounds; ++r) {
      if (r == 0) t0 = globaltimer();  // round -1 warms the pipe
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t acc = (r > -1 || q > 0) ? 1u : 0u;
        if (KIND == 0) umma_f16(tmem, a0 + 2 * q, b0 + 2 * q, idesc, acc);
        if (KIND == 1) umma_f16_sp(tmem, a0 + 2 * q, b0 + 4 * (q & 1), meta + 2 * q, idesc, acc);
        if (KIND == 2) umma_nvfp4(tmem, a0 + 2 * q, b0 + 2 * q, idesc, sfa + 4 * q, sfb + 8 * q, acc);
        if (KIND == 3) umma_nvfp4_sp(tmem, a0 + 2 * q, b0 + 4 * (q & 1), meta + 2 * q, idesc, sfa + 4 * q, sfb + 8 * q, acc);
        if (KIND == 4) umma_nvfp4_pair(tmem, a0 + 2 * q, b0 + 2 * q, idesc, sfa + 4 * q, sfb + 8 * q, acc);
      }
    }
    if (PAIR) umma_commit_pair(&done_bar, 0x3);
    else umma_commit(&done_bar);
    const bool ok = mbar_wait(&done_bar, 0);
    const uint64_t t1 = globaltimer();
    if (!ok) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
    out[blockIdx.x] = ok ? t1 - t0 : 0ull;
  } else if (PAIR && !issuer && threadIdx.x == 0) {
    mbar_wait(&done_bar, 0);  // the pair's commit arrives here too
    out[blockIdx.x] = 0ull;
  }
  tc_fence_before();
  sync_all<PAIR>();
  if (threadIdx.x < 32) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}

__global__ void __launch_bounds__(512) read_stream_kernel(const uint4* __restrict__ src, int64_t n16,
                                                          unsigned int* __restrict__ out) {  // out: one word
  uint32_t acc = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
    const uint4 v = ldg_stream16(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  if ((threadIdx.x & 31) == 0) atomicXor(out, acc);
}

template <int KIND>
int launch_peak(int rounds, unsigned long long* out, cudaStream_t s) {
  constexpr bool PAIR = KIND == 4;
  auto kern = mma_peak_kernel<KIND>;
  // 120 KB: more than half of an SM's shared memory, so each SM holds one CTA (one issuer)
  const size_t smem = 120 * 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SP24_ERR_CUDA;
  const int ctas = PAIR ? sm_count() / 2 * 2 : sm_count();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas, 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, rounds, out) != cudaSuccess) {
    cudaGetLastError();
    return SP24_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_peak_ctas(int kind) {
  if (kind < 0 || kind > 4) return 0;
  return kind == 4 ? sm_count() / 2 * 2 : sm_count();
}

extern "C" int sp24_peak_mma(int kind, int rounds, unsigned long long* out_ns, void* stream) {
  if (kind < 0 || kind > 4 || rounds < 1 || !out_ns) return SP24_ERR_INVALID_ARG;
  if (!aligned(out_ns, 8)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  switch (kind) {
    case 0: return launch_peak<0>(rounds, out_ns, s);
    case 1: return launch_peak<1>(rounds, out_ns, s);
    case 2: return launch_peak<2>(rounds, out_ns, s);
    case 3: return launch_peak<3>(rounds, out_ns, s);
    default: return launch_peak<4>(rounds, out_ns, s);
  }
}

extern "C" int sp24_peak_read(const void* src, int64_t bytes, unsigned int* out, void* stream) {
  if (!src || !out || bytes < 16 || bytes % 16) return SP24_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(out, 4)) return SP24_ERR_ALIGN;
  const int grid = sm_count() * 4;
  read_stream_kernel<<<grid, 512, 0, as_stream(stream)>>>(static_cast<const uint4*>(src), bytes / 16, out);
  return launch_status();
}
