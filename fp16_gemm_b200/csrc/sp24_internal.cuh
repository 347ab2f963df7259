// Internal helpers shared by the libsp24 translation units (device code for sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sp24.h"

namespace sp24 {

// Device error word of this library (one per device, across all kernels): a kernel that
// detects a problem it cannot report otherwise (a bounded wait that ran out, an illegal
// nibble) stores a status here; sp24_last_device_error() reads and clears it.
extern __device__ int g_dev_error;

__device__ __forceinline__ void set_dev_error(int code) { atomicCAS(&g_dev_error, 0, code); }

// Time limit of every bounded device-side wait of this library, in nanoseconds of %globaltimer
// (one per device; default 2 s; sp24_set_wait_limit changes it for later launches).
extern __device__ unsigned long long g_wait_limit_ns;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Host-side count of kernels this library has launched (diagnostics: sp24_kernel_launches).
void count_launch(int n = 1);

// Status of the launches just issued; every launch site calls this once per kernel launched.
inline int launch_status(int kernels = 1) {
  count_launch(kernels);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
}

inline int elem_bytes(int dtype) {
  switch (dtype) {
    case SP24_F16:
    case SP24_BF16:
      return 2;
    case SP24_F32:
      return 4;
    default:
      return 0;
  }
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Number of SMs of the current device (cached per process; B200 has 148).
int sm_count();

// Grid for a grid-stride kernel: the blocks needed, capped at one full wave (as many blocks as
// the occupancy calculator says fit on all SMs at once), so no block waits for a second wave.
template <typename Kern>
int full_wave_grid(Kern kernel, int threads, int64_t blocks_needed, size_t dyn_smem = 0) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, dyn_smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t cap = (int64_t)per_sm * sm_count();
  if (blocks_needed < 1) blocks_needed = 1;
  return (int)(blocks_needed < cap ? blocks_needed : cap);
}

// Magnitude bits of a 16- or 32-bit float pattern: monotone in |value| for non-NaN values.
__device__ __forceinline__ uint32_t mag16(uint32_t h) { return h & 0x7fffu; }
__device__ __forceinline__ uint32_t mag32(uint32_t f) { return f & 0x7fffffffu; }

// Streaming 16-byte global load that bypasses L1 allocation (weights are read once).
__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ------------------------------------------------------------------ skinny GEMM interface
enum { W_D16 = 0, W_S16 = 1, W_DQ4 = 2, W_SQ4 = 3 };  // weight formats
enum { X_16 = 0, X_Q4 = 1 };                          // activation formats

struct SkinnyParams {
  const void* x;            // 16-bit [M, K] or NVFP4 codes [M, K/2]
  const uint8_t* x_scales;  // NVFP4 x: [M, K/16]
  const float* x_ts;        // NVFP4 x: tensor scale (device)
  int x_fmt;
  const uint8_t* w;         // values / codes, row-major
  const uint8_t* w_scales;  // NVFP4 block scales
  const float* w_ts;        // NVFP4 tensor scale (device)
  const uint8_t* meta;      // 2:4 nibble stream, K/8 bytes per row
  int64_t M, N, K;
  int64_t w_row_bytes, scale_row_bytes, meta_row_bytes;
  float* y;
  int chunks_total;         // filled by skinny_gemm
  bool accumulate;          // filled by skinny_gemm
  // grouped (routed-expert) mode: blockIdx.z picks a token tile of one expert
  const int32_t* perm;      // [T * topk] flat (token * topk + slot) entries grouped by expert
  const int32_t* tiles;     // [max_tiles][3] = expert, first perm index, token count (<= tile)
  int topk;
  int64_t expert_rows;      // weight rows per expert (N)
};

// Launches the skinny kernel for M <= 64 (wf: W_*, t16: SP24_F16 / SP24_BF16 MMA type).
int skinny_gemm(int wf, int t16, SkinnyParams p, cudaStream_t s);

// Shared-memory staged skinny kernel (bulk copies + native 2:4 MMA); supported() checks the
// alignment its bulk copies need.
bool skinny2_supported(int wf, const SkinnyParams& p);
int skinny2_gemm(int wf, int t16, SkinnyParams p, cudaStream_t s);
// Persistent decode GEMV for NVFP4 weights (dense / 2:4) at M <= 8 (TMA-fed, one CTA per SM).
// Whole-tile decode GEMV (M <= 8, NVFP4 weights, at least one 16-row tile per SM): writes y
// without atomics, so y needs no zeroing.
bool decode_tile_supported(int wf, const SkinnyParams& p);
int decode_tile(int wf, int t16, const SkinnyParams& p, cudaStream_t s);
bool decode_supported(int wf, const SkinnyParams& p);
int decode_gemv(int wf, int t16, const SkinnyParams& p, cudaStream_t s);
// 2-D TMA maps (defined with the tensor-core GEMMs): 128-byte swizzled, and unswizzled bytes.
int make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t rows, uint64_t cols,
                 uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows);
int make_tmap_2d_plain(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                       uint32_t box_cols, uint32_t box_rows);
// Grouped variant: one launch over max_tiles token tiles (tile table and perm on the device).
int skinny2_grouped(int wf, int t16, SkinnyParams p, int64_t max_tiles, cudaStream_t s);
// Routed-expert GEMM on the tensor cores for NVFP4 experts (dense W_DQ4 or 2:4 W_SQ4) and 16-bit
// tokens: token tiles of up to 128 routed rows (p.tiles, p.perm), 128 weight rows per CTA,
// tcgen05.mma (.sp for 2:4) into TMEM.
bool moe_tc_supported(int wf, int x_fmt, int64_t T, int64_t E, int64_t N, int64_t K, int64_t max_tiles,
                      const void* codes, const void* scales, const void* meta, const void* x);
// n_tiles bounds the tile table; *n_valid (device) is the number of used tiles, which come first.
int moe_tc_grouped(int wf, int t16, const SkinnyParams& p, int64_t E, int64_t T, int64_t n_tiles,
                   const int32_t* n_valid, cudaStream_t s);
// One GEMM of the expert block on the same kernel: epi 1 = gate/up (weights packed in 16-row
// gate / up blocks, output h = SiLU(gate) * up in x's 16-bit type, routed order), epi 0 = down
// (x = h rows in routed order, output stored as y[T, topk, N]).
struct MoeBlockGemm {
  const uint16_t* x;
  const uint8_t *codes, *scales, *meta;
  const float* w_ts;
  const int32_t *tiles, *perm, *n_valid;
  float* y;
  uint16_t* h;
  int x_direct, topk;
  int64_t T, E, N, K, n_tiles;
};
int moe_tc_block_gemm(int epi, int wf, int t16, const MoeBlockGemm& g, cudaStream_t s);

// Tensor-core (tcgen05) 16-bit GEMM: y[M, N] = (*scale_a) (*scale_b) x[M, K] w[N, K]^T.
int tc_gemm_f16(const void* x, const void* w, int64_t M, int64_t N, int64_t K, bool bf16, float* y,
                const float* scale_a, const float* scale_b, cudaStream_t s);

// NVFP4 operand images for the W4A4 kernel (K % 256 == 0): codes [rows, K/2] -> 16 KB tiles of
// 128 rows x 256 K in the 128-byte-swizzled shared-memory order; scales [rows, K/16] -> 512-byte
// tiles of 128 rows x 4 scales in tcgen05.cp order.
int64_t nvfp4_mma_codes_bytes(int64_t rows, int64_t K);
int64_t nvfp4_mma_scales_bytes(int64_t rows, int64_t K);
int nvfp4_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, uint8_t* codes_out,
                 uint8_t* scales_out, cudaStream_t s);
// The same for two operands in one launch (rows1 == 0: the first only).
int nvfp4_to_mma2(const uint8_t* c0, const uint8_t* s0, int64_t rows0, uint8_t* co0, uint8_t* so0,
                  const uint8_t* c1, const uint8_t* s1, int64_t rows1, uint8_t* co1, uint8_t* so1, int64_t K,
                  cudaStream_t s);

// Images for the sparse FP4 pair kernel: activations with one scale per 32 K; a pairwise-4:8
// weight (kept values, their scales, metadata tiles), rows padded to 256.
int64_t b32_mma_scales_bytes(int64_t rows, int64_t K);
int64_t sp48_mma_values_bytes(int64_t rows, int64_t K);
int64_t sp48_mma_scales_bytes(int64_t rows, int64_t K);
int64_t sp48_mma_meta_bytes(int64_t rows, int64_t K);
int nvfp4_b32_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, uint8_t* codes_out,
                     uint8_t* scales_out, cudaStream_t s);
int sp48_to_mma(const uint8_t* values, const uint8_t* scales, const uint8_t* meta, int64_t rows, int64_t K,
                uint8_t* values_out, uint8_t* scales_out, uint8_t* meta_out, cudaStream_t s);
int tc_gemm_nvfp4_sp48_pair(const uint8_t* xc_mma, const uint8_t* xs_mma, const float* x_ts, const uint8_t* vc_mma,
                            const uint8_t* vs_mma, const uint8_t* meta_mma, const float* w_ts, int64_t M, int64_t N,
                            int64_t K, float* y, cudaStream_t s, uint64_t wait_ns);

// A 2-D map over rows of row_bytes bytes (elements of elem bytes), box box_rows whole rows, no
// swizzle; and the fp32 output Y [M, N] with box 128 rows of N x 32 tokens.
int make_tmap_rows(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem, uint64_t row_bytes,
                   uint64_t rows, uint32_t box_rows);
int make_tmap_y(CUtensorMap* map, float* y, int64_t M, int64_t N);

// W4A4 GEMM on the persistent CTA-pair kernel (both operands as images above).  wait_ns bounds
// every device-side wait (0: the library's default).
int tc_gemm_nvfp4_pair(const uint8_t* xc_mma, const uint8_t* xs_mma, const float* x_ts, const uint8_t* wc_mma,
                       const uint8_t* ws_mma, const float* w_ts, int64_t M, int64_t N, int64_t K, float* y,
                       cudaStream_t s, uint64_t wait_ns);

// 16-bit GEMM on the persistent CTA-pair kernel (tcgen05 cta_group::2): dense (meta_img null,
// K % 64) or 2:4 with values [N, K/2] and the metadata image of meta_to_image (K % 128).
int tc_gemm_f16_pair(const void* x, const void* w, const uint8_t* meta_img, int64_t M, int64_t N, int64_t K,
                     bool bf16, float* y, const float* scale_a, const float* scale_b, cudaStream_t s,
                     uint64_t wait_ns);
// The 2:4 metadata image of the pair kernel (tcgen05 metadata tiles of 128 rows x 128 K, rows
// padded to 256) and its size in bytes.
int64_t meta_image_bytes(int64_t rows, int64_t K);
int meta_to_image(const uint8_t* meta, int64_t rows, int64_t K, uint8_t* out, cudaStream_t s);

// Expands an NVFP4 (W_DQ4) or 2:4-compressed (W_S16 / W_SQ4) operand into exact 16-bit values.
int expand_w16(int wf, bool bf16, const uint8_t* w, const uint8_t* scales, const uint8_t* meta,
               int64_t rows, int64_t K, uint16_t* out, cudaStream_t s);

}  // namespace sp24
