/*
 * sp24.h -- C ABI of libsp24: 2:4 structured sparsity and NVFP4 against dense GEMM on one
 * NVIDIA B200 (sm_100a).
 *
 * Sources (pages, by title; section names in quotes):
 *   [P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went" (robertz.co)
 *   [P2] "Sparse GPU FLOPS Need the Right Zeros in the Right Places" (leviathansystems.co)
 *   [P5] "NVFP4 Without FP4 Hardware" (ai-muninn.com)
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must point to memory of the current CUDA device;
 *     `shape` arrays and the operand structs are host memory and are read before the call
 *     returns.  The caller owns every buffer; the library never allocates device memory.
 *   - Tensors are dense and row-major (C order).  GEMM operands are K-contiguous.  Every
 *     element pointer needs at least the alignment of its element type (SP24_ERR_ALIGN
 *     otherwise); calls that need more say so.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and returns a status.  Argument errors are detected on the host and return a
 *     status without launching anything.  SP24_ERR_CUDA reports a failed launch.  Kernels
 *     never trap: a device-side wait that runs out of time sets a device error word, which
 *     sp24_last_device_error() reports.
 *   - No call falls back to the CPU.
 */
#ifndef SP24_H_
#define SP24_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ----------------------------------------------------------------------- status codes */
enum {
  SP24_OK = 0,
  SP24_ERR_INVALID_ARG = 1,   /* null pointer, unknown enum value, bad operand struct */
  SP24_ERR_SHAPE = 2,         /* shape violates the operation's rule (e.g. C % 4 != 0) */
  SP24_ERR_DTYPE = 3,         /* element type not accepted by this call */
  SP24_ERR_ALIGN = 4,         /* a pointer is not aligned as the call requires */
  SP24_ERR_UNSUPPORTED = 5,   /* valid request that no kernel of the library serves */
  SP24_ERR_CUDA = 6,          /* a CUDA runtime call or launch failed */
  SP24_ERR_DEVICE_TIMEOUT = 7,/* a bounded device-side wait gave up */
  SP24_ERR_WORKSPACE = 8      /* workspace missing or smaller than the size query says */
};

/* ----------------------------------------------------------------------- enums */
/* element types */
enum { SP24_F16 = 0, SP24_BF16 = 1, SP24_F32 = 2, SP24_NVFP4 = 3, SP24_NVFP4_B32 = 4, SP24_NVFP4_MMA = 5,
       SP24_NVFP4_B32_MMA = 6 };

/* The operation a weight belongs to decides which four entries form a group ([P2] "The
 * operation determines which four entries belong together"). */
enum {
  SP24_OP_MATMUL = 0, /* W[..., K]: groups of four consecutive entries along the last axis K */
  SP24_OP_CONV = 1    /* W[K, C, R, S]: groups along input channels C at fixed (k, r, s);
                         C % 4 == 0 */
};

/* GEMM kernel choice (SP24_ALGO_AUTO picks by shape). */
enum { SP24_ALGO_AUTO = 0, SP24_ALGO_SKINNY = 1, SP24_ALGO_TILED = 2 };

/* ----------------------------------------------------------------------- operands */
/* A dense GEMM operand with `rows` rows of K entries.
 *   format SP24_F16 / SP24_BF16: data -> [rows, K] elements.
 *   format SP24_NVFP4 ([P5] "Convert BF16 to NVFP4 yourself": 4-bit E2M1 values, one E4M3
 *   scale per 16 values, one fp32 tensor scale):
 *       data -> [rows, K/2] bytes of packed E2M1 codes (entry 2i in the low nibble),
 *       scales -> [rows, K/16] E4M3 block scales, tensor_scale -> one fp32 (device).
 *   format SP24_NVFP4_B32: the same encoding with one E4M3 scale per 32 values, scales ->
 *       [rows, K/32] (the activation form read by sp24_gemm_sparse48 only).
 *   format SP24_NVFP4_MMA: SP24_NVFP4 rewritten as tile images (sp24_nvfp4_to_mma): data ->
 *       code tiles, scales -> scale tiles; accepted by sp24_gemm_dense when both operands are
 *       NVFP4 (either layout), K % 256 == 0.
 *   format SP24_NVFP4_B32_MMA: SP24_NVFP4_B32 rewritten as tile images
 *       (sp24_nvfp4_b32_to_mma), the activation form of sp24_gemm_sparse48's pair kernel. 
 * Decoded value = E2M1(code) * E4M3(scale) * tensor_scale. */
typedef struct {
  int32_t format;
  const void* data;
  const uint8_t* scales;
  const float* tensor_scale;
} sp24_operand;

/* A 2:4-compressed weight W[N, K] ([P1] "What 2:4 actually is": two kept values per group of
 * four plus a 2-bit index for each).
 *   meta -> [N, K/8] bytes: one nibble per group, i0 | i1 << 2 with i0 < i1 the kept indices,
 *           groups in natural order, the even group in the low nibble.
 *   format SP24_F16 / SP24_BF16: values -> [N, K/2] kept entries in ascending index order.
 *   format SP24_NVFP4: the kept values [N, K/2] quantised as an NVFP4 tensor:
 *           values -> [N, K/4] packed codes, scales -> [N, K/32] (one per 16 stored values),
 *           tensor_scale -> one fp32 (device). */
typedef struct {
  int32_t format;
  const void* values;
  const uint8_t* scales;
  const float* tensor_scale;
  const uint8_t* meta;
} sp24_sparse_operand;

/* ----------------------------------------------------------------------- host helpers */
const char* sp24_status_string(int status);
int sp24_abi_version(void);

/* [P1] "The byte saving is about a quarter, not a half"; [P5] "Bit-exact check against lyf's
 * ModelOpt output" (packed and scale bytes of real tensors).
 * Sizes of what the pipeline produces for a tensor (host only, no device access).
 * groups: groups of four along the reduction axis; values_bytes / meta_bytes: compressed
 * form; nvfp4_codes_bytes / nvfp4_scales_bytes: dense NVFP4 of the tensor viewed as
 * [numel / L, L] with L its last axis (matmul only; 0 for conv).  Any output may be NULL. */
int sp24_sizes(int op, int dtype, const int64_t* shape, int ndim, int64_t* groups,
               int64_t* values_bytes, int64_t* meta_bytes, int64_t* nvfp4_codes_bytes,
               int64_t* nvfp4_scales_bytes);

/* ----------------------------------------------------------------------- a1: eligibility */
/* [P2] "The operation determines which four entries belong together", "Two half-zero vectors
 * produce different pattern answers": a group passes when at least two of its four entries
 * are zero (+0 or -0; NaN is not zero); groups are judged one by one.
 *   w      device, dtype F16/BF16/F32, shape [rows..., K] (MATMUL, ndim 1..4, K % 4 == 0)
 *          or [K, C, R, S] (CONV, C % 4 == 0).
 *   pass   device uint8, one byte (0/1) per group, group axis replacing K (MATMUL) or laid
 *          out [K, C/4, R, S] (CONV).
 *   n_fail device int32 or NULL: receives the number of failing groups (overwritten). */
int sp24_check_24(const void* w, int dtype, int op, const int64_t* shape, int ndim,
                  uint8_t* pass, int32_t* n_fail, void* stream);

/* ----------------------------------------------------------------------- a2: prune/compress */
/* [P1] "What 2:4 actually is": magnitude pruning to two of four and compression.  Kept = the
 * two entries first in the order (|w| descending, index ascending), |w| compared as the
 * magnitude bit pattern (NaN above +inf).
 *   values device, same dtype as w: [rows, K/2] (MATMUL) or [K, C/2, R, S] (CONV), kept
 *          entries copied bit for bit in ascending index order.
 *   meta   device, ceil(groups / 2) bytes, nibble stream as in sp24_sparse_operand. */
int sp24_prune_compress_24(const void* w, int dtype, int op, const int64_t* shape, int ndim,
                           void* values, uint8_t* meta, void* stream);

/* [P2] "The mechanism needs both values and their positions".
 * Inverse of compression: w_out (device, dtype, `shape`) receives the kept values at their
 * indices and +0 elsewhere.  Nibbles must be legal (i0 < i1); an illegal nibble yields +0 in
 * its group and sets the device error word (SP24_ERR_INVALID_ARG). */
int sp24_decompress_24(const void* values, const uint8_t* meta, int dtype, int op,
                       const int64_t* shape, int ndim, void* w_out, void* stream);

/* The nibble stream of a 2:4 weight [rows, K] (matmul layout, K % 128 == 0) rewritten in the
 * layout the sparse tensor-core MMA reads its metadata in ([P1] "What 2:4 actually is": the
 * positions travel with the kept values), so that a GEMM moves it into tensor memory without
 * touching it.  Not on the source pages: the layout of this library's kernel.
 *   meta_img: for each 128-row block rb and 128-K chunk kc a 2 KB tile at byte
 *             2048 (rb * K/128 + kc); its 16-byte row l (l = 0..127) is TMEM lane l: rows
 *             m = 128 rb + 16 (l / 16) + l % 8 and m + 8, half h = (l / 8) % 2; 32-bit word t
 *             (the 32-wide K window t) = the two nibble bytes 16 kc + 4 t + 2 h, +1 of row m in
 *             the low half and of row m + 8 in the high half.  Rows are padded to a multiple of
 *             256 with bytes 0x44 (index pair 0, 1 in every group).
 *   sp24_prepare_sparse_size gives the bytes (rows rounded up to 256, times K/128 x 2 KB / 128).
 *   meta: device, [rows, K/8] as from sp24_prune_compress_24; meta_img: device, 16-byte aligned,
 *   owned by the caller.  K % 128 != 0 or negative sizes: SP24_ERR_SHAPE.  One launch.
 * sp24_gemm_sparse24 with 16-bit values at M > 64 builds this image in its workspace itself. */
int sp24_prepare_sparse_size(int64_t rows, int64_t K, int64_t* bytes);
int sp24_prepare_sparse(const uint8_t* meta, int64_t rows, int64_t K, uint8_t* meta_img, void* stream);

/* ----------------------------------------------------------------------- pairwise 4:8 */
/* The sparse pattern of the tensor cores' packed-FP4 MMA kind, whose sparse unit is a pair of
 * consecutive entries.  [P1] "What 2:4 actually is" (the largest magnitudes survive), carried
 * over to pairs.  W is [rows, K] row-major (matmul layout), K % 8 == 0; chunk c is entries
 * 8c .. 8c + 7 of the flat tensor, i.e. four pairs along K.
 *   check:     a chunk passes when at most two of its pairs hold a nonzero entry (+0 and -0 are
 *              zero, NaN is not).  pass: device uint8 [rows, K/8]; n_fail: device int32 or
 *              NULL (overwritten with the failing-chunk count).
 *   prune:     keeps the two pairs of largest score |a| + |b| (one IEEE fp32 addition of the
 *              entries' fp32 magnitudes; a NaN score above every number; ties to the lower
 *              pair).  values: device, w's dtype, [rows, K/2], the kept pairs bit for bit in
 *              ascending order; meta: device, ceil(rows * K / 16) bytes, nibble i0 | i1 << 2
 *              per chunk (i0 < i1), chunk 2c in the low nibble of byte c.
 *   decompress: w_out (device, [rows, K]) receives the kept pairs at their places and +0
 *              elsewhere; an illegal nibble (i0 >= i1) yields +0 in its chunk and sets the
 *              device error word (SP24_ERR_INVALID_ARG).
 * Pointers need the alignment of their element type (SP24_ERR_ALIGN otherwise); 16-byte
 * aligned ones take the vector kernels.  K % 8 != 0 or negative sizes: SP24_ERR_SHAPE.  The
 * caller owns every buffer; all calls are asynchronous on `stream`. */
int sp24_check_48(const void* w, int dtype, int64_t rows, int64_t K, uint8_t* pass, int32_t* n_fail,
                  void* stream);
int sp24_prune_compress_48(const void* w, int dtype, int64_t rows, int64_t K, void* values, uint8_t* meta,
                           void* stream);
int sp24_decompress_48(const void* values, const uint8_t* meta, int dtype, int64_t rows, int64_t K,
                       void* w_out, void* stream);

/* W4A4 GEMM on the sparse FP4 MMA (tcgen05.mma.sp kind::mxf4nvf4, K = 128 logical per
 * instruction): y[M, N] = s_x s_w sum_k dec(x[m, k]) dec(w[n, k]), fp32 accumulation, the
 * product of the pages' 2:4-sparse W4A4 path ([P1] "NVFP4 vs 2:4 sparse: where the other half
 * of the petaflop went") in the pattern that MMA reads.
 *   x  format SP24_NVFP4_B32: data [M, K/2] codes, scales [M, K/32] (sp24_quantize_nvfp4_block32).
 *   w  format SP24_NVFP4: a pairwise-4:8 weight W[N, K]: values -> [N, K/4] codes of the kept
 *      values [N, K/2] quantised with sp24_quantize_nvfp4 (scales -> [N, K/32], one per 16
 *      stored = 32 logical K), meta -> [N, K/16] from sp24_prune_compress_48 (every nibble
 *      legal; other metadata gives undefined results for its rows).
 *   y  device fp32 [M, N], written (not accumulated), 4-byte aligned.
 * K % 512 == 0 (SP24_ERR_SHAPE otherwise); every operand pointer 16-byte aligned; M, N, K up to
 * 2^31 - 1.  Wrong formats: SP24_ERR_DTYPE.  One launch; nothing is allocated. */
int sp24_gemm_sparse48(const sp24_operand* x, const sp24_sparse_operand* w, int64_t M, int64_t N,
                       int64_t K, float* y, void* stream);

/* [P1] "The ladder, top to bottom" (the sparse FP4 rate of the tensor cores).
 * The same GEMM on tile images (x format SP24_NVFP4_B32_MMA, w format SP24_NVFP4_MMA; both or
 * neither) runs a persistent kernel on pairs of SMs (tcgen05.mma.sp.cta_group::2, 256 weight
 * rows x 256 tokens per pair tile, 512 logical K per stage).  Not on the source pages: layouts
 * of this library's kernel.
 *   sp24_nvfp4_b32_mma_size / sp24_nvfp4_b32_to_mma: activations [rows, cols] (cols % 256 == 0)
 *       with one scale per 32 entries -> code tiles as sp24_nvfp4_to_mma, scale tiles of 128 rows
 *       x 4 scales (128 entries) at byte 512 * (rb * cols/128 + t), row r at 16 (r % 32) +
 *       4 (r / 32); rows padded to 128.
 *   sp24_sparse48_mma_size / sp24_sparse48_to_mma: a pairwise-4:8 weight [rows, K] (K % 512):
 *       the kept values' codes [rows, K/4] and scales [rows, K/32] as the code and scale tiles of
 *       a [rows, K/2] NVFP4 tensor (scale tiles of 64 stored = 128 logical K), the metadata
 *       [rows, K/16] as 2 KB tiles per 128 rows and 256 logical K (row r's 16 bytes at 16 r);
 *       rows padded to a multiple of 256 with zero codes and scales and metadata 0x44 (a legal
 *       pattern), so every tile the kernel loads exists.
 * Inputs device, codes and metadata 16-byte aligned, scales 4-byte aligned; outputs 16-byte
 * aligned, of the sizes the queries give.  One launch each. */
int sp24_nvfp4_b32_mma_size(int64_t rows, int64_t cols, int64_t* codes_bytes, int64_t* scales_bytes);
int sp24_nvfp4_b32_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                          uint8_t* codes_out, uint8_t* scales_out, void* stream);
int sp24_sparse48_mma_size(int64_t rows, int64_t K, int64_t* values_bytes, int64_t* scales_bytes,
                           int64_t* meta_bytes);
int sp24_sparse48_to_mma(const uint8_t* values, const uint8_t* scales, const uint8_t* meta, int64_t rows,
                         int64_t K, uint8_t* values_out, uint8_t* scales_out, uint8_t* meta_out,
                         void* stream);

/* ----------------------------------------------------------------------- a3: NVFP4 */
/* [P5] "Convert BF16 to NVFP4 yourself", "The shared global scale": quantise T[rows, cols]
 * (cols % 16 == 0) to NVFP4.
 *   s_t  = tensor_scale_in ? *tensor_scale_in : amax(|T|) / 2688   (2688 = 6 * 448)
 *   block scale sb = E4M3_rne_satfinite(bmax / (s_t * 6)) per 16 consecutive entries of a row
 *   code = sign(t) << 3 | E2M1_rne_satfinite(|t| / (E4M3(sb) * s_t))  (0 when that divisor is 0)
 * every step an IEEE fp32 operation; negative zero keeps its sign bit.
 *   t                 device, F16/BF16/F32, [rows, cols]
 *   tensor_scale_in   device fp32 or NULL (NULL: derive from amax; else a shared scale,
 *                     finite and >= 0)
 *   codes             device, [rows, cols/2] bytes;  scales: device, [rows, cols/16] bytes
 *   tensor_scale_out  device fp32 (may equal tensor_scale_in)
 *   workspace         device, >= sp24_quantize_nvfp4_workspace_size() bytes, 16-byte
 *                     aligned; contents are scratch.  Non-finite inputs give unspecified codes. */
int sp24_quantize_nvfp4_workspace_size(int64_t rows, int64_t cols, int64_t* bytes);
int sp24_quantize_nvfp4(const void* t, int dtype, int64_t rows, int64_t cols,
                        const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                        float* tensor_scale_out, void* workspace, int64_t workspace_bytes,
                        void* stream);

/* [P1] "The ladder, top to bottom" (the dense NVFP4 GEMM at 4096^3).
 * An NVFP4 tensor [rows, cols] (cols % 256 == 0) rewritten as the tile images the W4A4 GEMM
 * loads whole (format SP24_NVFP4_MMA): each tile lands in shared memory with one copy.  Not on
 * the source pages: a layout of this library's W4A4 kernel; the values are unchanged.
 *   codes_out:  per 128-row block rb and 256-column chunk kc a 16 KB tile at byte
 *               16384 * (rb * cols/256 + kc); row r of the block at byte 128 * r, its 16-byte
 *               piece c (columns 32c .. 32c+31 of the chunk) at 16 * (c ^ (r % 8)).
 *   scales_out: per 128-row block rb and 64-column chunk kc a 512-byte tile at byte
 *               512 * (rb * cols/64 + kc); row r's four scales of the chunk at byte
 *               16 * (r % 32) + 4 * (r / 32).
 *   Rows are padded to a multiple of 128 with zero codes and zero scales; sizes from
 *   sp24_nvfp4_mma_size.  codes: device [rows, cols/2] (16-byte aligned); scales: device
 *   [rows, cols/16] (4-byte aligned); outputs device, 16-byte aligned.  Two launches;
 *   SP24_ERR_SHAPE when cols % 256 != 0. */
int sp24_nvfp4_mma_size(int64_t rows, int64_t cols, int64_t* codes_bytes, int64_t* scales_bytes);
int sp24_nvfp4_to_mma(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                      uint8_t* codes_out, uint8_t* scales_out, void* stream);

/* ----------------------------------------------------------------------- bounded waits */
/* Every device-side wait of this library (mbarrier phases, TMA and bulk-copy completions) gives
 * up after a time limit: the kernel then records SP24_ERR_DEVICE_TIMEOUT in the device error
 * word (read with sp24_last_device_error), waits (bounded) for its own copies in flight, frees
 * the tensor memory it holds and returns; nothing traps.  Not on the source pages.
 *   sp24_set_wait_limit   the limit in nanoseconds (> 0; default 2e9) for the current device,
 *                         used by kernels launched afterwards.  Synchronous.
 *   sp24_get_wait_limit   reads it back.
 *   sp24_selftest_wait_timeout  runs that unwind on purpose: one CTA allocates TMEM, starts a
 *                         1 KB bulk copy from `src` (device, 16-byte aligned), waits on an
 *                         mbarrier phase that nothing completes until the limit runs out, sets
 *                         SP24_ERR_DEVICE_TIMEOUT, lets the copy land, frees TMEM.  out (device
 *                         int[2]): out[0] = 2 when the wait ran out (1 if it completed),
 *                         out[1] = 1 + the copy's last byte once it landed (0 if not).
 *                         Takes about one wait limit; for tests. */
int sp24_set_wait_limit(unsigned long long ns);
int sp24_get_wait_limit(unsigned long long* ns);
int sp24_selftest_wait_timeout(const void* src, int* out, void* stream);

/* ----------------------------------------------------------------------- roofline peaks */
/* [P1] "The roofline is the whole argument".
 * The denominators of the roofline fractions, measured with this library's own instructions
 * (not on the source pages).
 *   sp24_peak_mma   one CTA per SM (kind 4: per CTA pair) issues 4 * (rounds + 1) back-to-back
 *                   tcgen05 MMAs of N = 256 from shared-memory operands holding non-zero data,
 *                   accumulating in TMEM; out_ns[cta] = nanoseconds of the last 4 * rounds (0 for
 *                   the odd CTA of a pair).  kind 0: kind::f16 bf16, M 128, K 16; 1: .sp
 *                   kind::f16, K 32 logical; 2: kind::mxf4nvf4 block16, K 64; 3: .sp
 *                   kind::mxf4nvf4, K 128 logical (pairwise 4:8 metadata); 4: kind::mxf4nvf4 on
 *                   a CTA pair (cta_group::2), M 256, K 64.  FLOPs per MMA: 2 M N K (logical K).
 *   sp24_peak_ctas  CTAs the launch uses (entries of out_ns) for a kind.
 *   sp24_peak_read  a grid-stride stream of 16-byte loads over src (bytes % 16 == 0, 16-byte
 *                   aligned), reduced into *out (device word) so nothing is optimised away. */
int sp24_peak_mma(int kind, int rounds, unsigned long long* out_ns, void* stream);
int sp24_peak_ctas(int kind);
int sp24_peak_read(const void* src, int64_t bytes, unsigned int* out, void* stream);

/* [P5] "Convert BF16 to NVFP4 yourself".
 * The same quantisation for callers that cannot allocate device memory: runtimes that only hand
 * out a fixed arena of operand buffers, plugins whose host framework owns the device allocator,
 * and host loops that must not call cudaMalloc (it can synchronise the device).  No counterpart
 * on the source pages: it is a property of this library, not of the method.
 *   Arguments as sp24_quantize_nvfp4, without the workspace.  The scratch is a 256-byte
 *   __device__ array inside the library, one per device, kept until the process exits; the
 *   quantiser needs 4 bytes of it (the amax word) for every tensor shape, and a request needing
 *   more than 256 bytes returns SP24_ERR_WORKSPACE.  The first call on each device looks up the
 *   array's device address (cudaGetSymbolAddress) and caches it; make that first call before
 *   any stream capture begins, and do not call this entry point on a device after a
 *   cudaDeviceReset of it in the same process (the cached address is then stale).  The call
 *   allocates nothing (no cudaMalloc/cudaFree, no allocating library routine).  All calls on a
 *   device share the array: each call clears the amax word first, and calls whose GPU work can
 *   overlap (different streams without ordering) race on it. */
int sp24_quantize_nvfp4_noalloc(const void* t, int dtype, int64_t rows, int64_t cols,
                                const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                                float* tensor_scale_out, void* stream);

/* [P5] "Convert BF16 to NVFP4 yourself" (the steps; its blocks hold 16 values).
 * NVFP4 encoding with 32-value blocks: the activation operand of the sparse FP4 MMA, which
 * reads one scale per 32 K (sp24_gemm_sparse48).  The steps of sp24_quantize_nvfp4 over
 * 32 consecutive entries of a row:  s_t = tensor_scale_in ? *tensor_scale_in : amax / 2688;
 * sb = E4M3_rne_satfinite(bmax32 / (s_t * 6));  code = sign << 3 | E2M1_rne_satfinite(|t| /
 * (E4M3(sb) * s_t)), every step IEEE fp32.  cols % 32 == 0; codes [rows, cols/2] (16-byte
 * aligned), scales [rows, cols/32]; workspace as sp24_quantize_nvfp4 (used only when no scale
 * is supplied).  Errors as sp24_quantize_nvfp4. */
int sp24_quantize_nvfp4_block32(const void* t, int dtype, int64_t rows, int64_t cols,
                                const float* tensor_scale_in, uint8_t* codes, uint8_t* scales,
                                float* tensor_scale_out, void* workspace, int64_t workspace_bytes,
                                void* stream);

/* [P5] "Convert BF16 to NVFP4 yourself"; [P1] "The byte saving is about a quarter, not a half".
 * Two quantisations in one launch (a weight and its 2:4 values, with the tensor scales that
 * sp24_prepare_24 derived, say): the results equal those of sp24_quantize_nvfp4(t0, ts0) and
 * sp24_quantize_nvfp4(t1, ts1).  Both tensors have type `dtype`; each tensor scale is required
 * (device fp32) and is copied to its ts_out (which may be the same pointer).  Shapes, layouts
 * and alignment as for sp24_quantize_nvfp4; either tensor may be empty.  No workspace. */
int sp24_quantize_nvfp4_pair(const void* t0, int dtype, int64_t rows0, int64_t cols0,
                             const float* ts0, uint8_t* codes0, uint8_t* scales0, float* ts_out0,
                             const void* t1, int64_t rows1, int64_t cols1, const float* ts1,
                             uint8_t* codes1, uint8_t* scales1, float* ts_out1, void* stream);

/* [P5] "The shared global scale": one tensor scale for a group of tensors that are read
 * together (q / k / v, gate / up):  s = max_i amax(|T_i|) / 2688, one IEEE fp32 division, the
 * scale sp24_quantize_nvfp4 derives for the group's entries taken as one tensor.  Quantise each
 * tensor with sp24_quantize_nvfp4(T_i, tensor_scale_in = s).
 *   tensors    host array of n device pointers (16-byte aligned when the tensor is not empty)
 *   numels     host array of n entry counts; numel * element size a multiple of 16 bytes
 *   dtype      F16, BF16 or F32, shared by the group
 *   tensor_scale_out  device fp32; n == 0 or all-empty tensors give 0
 *   workspace  device, >= sp24_nvfp4_group_tensor_scale_workspace_size() bytes, 16-byte
 *              aligned; scratch.  NaN entries are skipped; an infinity gives an infinite scale.
 * One launch per 16 tensors plus a one-thread kernel; nothing is allocated. */
int sp24_nvfp4_group_tensor_scale_workspace_size(int64_t* bytes);
int sp24_nvfp4_group_tensor_scale(const void* const* tensors, const int64_t* numels, int n,
                                  int dtype, float* tensor_scale_out, void* workspace,
                                  int64_t workspace_bytes, void* stream);

/* [P5] "Convert BF16 to NVFP4 yourself" (the format decoded).
 * Decode: out[r, c] = E2M1(code) * E4M3(scale) * tensor_scale, rounded once to out_dtype
 * (F16/BF16/F32). */
int sp24_dequantize_nvfp4(const uint8_t* codes, const uint8_t* scales,
                          const float* tensor_scale, int64_t rows, int64_t cols, int out_dtype,
                          void* out, void* stream);

/* ----------------------------------------------------------------------- a1-a3 in one read */
/* Prepares a matmul weight W[rows, K] (K % 16 == 0) with a single read of W: the outputs equal,
 * bit for bit, those of
 *   sp24_check_24(W)            -> pass, n_fail
 *   sp24_prune_compress_24(W)   -> values [rows, K/2], meta [rows, K/8]
 * plus the two tensor scales sp24_quantize_nvfp4 derives when given none:
 *   w_tensor_scale = amax|W| / 2688,  v_tensor_scale = amax|values| / 2688.
 * Passing those scales to sp24_quantize_nvfp4 (tensor_scale_in) then gives the NVFP4 encodings
 * of W and of the values without another amax pass, identical to the unscaled calls.  [P1]
 * "What 2:4 actually is" and [P5] "Convert BF16 to NVFP4 yourself" define the steps; the pages
 * run them one after the other, this call fuses their reads of W.
 *   w          device, F16/BF16/F32, 16-byte aligned
 *   pass       device [rows, K/4] bytes (2-byte aligned) or NULL
 *   n_fail     device int32 or NULL
 *   values     device, dtype, [rows, K/2], 8-byte aligned;  meta: device [rows, K/8] bytes
 *   w_tensor_scale, v_tensor_scale   device fp32 or NULL
 *   workspace  device, >= sp24_prepare_24_workspace_size() bytes, 16-byte aligned; scratch.
 * One memset and one streaming kernel; an empty W gives n_fail 0 and scales 0. */
int sp24_prepare_24_workspace_size(int64_t rows, int64_t K, int64_t* bytes);
int sp24_prepare_24(const void* w, int dtype, int64_t rows, int64_t K, uint8_t* pass,
                    int32_t* n_fail, void* values, uint8_t* meta, float* w_tensor_scale,
                    float* v_tensor_scale, void* workspace, int64_t workspace_bytes,
                    void* stream);

/* ----------------------------------------------------------------------- a4-a6: GEMM */
/* [P1] "The roofline is the whole argument" and [P5] "Why NVFP4 helps without FP4 hardware":
 * the dense product whose bytes (decode) or FLOPs (prefill) the sparse form is compared with.
 * Y[m, n] = sum_k x[m, k] * w[n, k] with fp32 accumulation, Y fp32 [M, N] row-major (device).
 * x: M rows (F16, BF16 or NVFP4); w: N rows (F16, BF16 or NVFP4).  16-bit x and 16-bit w
 * must have the same type.  Where NVFP4 meets NVFP4 (W4A4) both stay 4-bit and the tensor core
 * applies the block scales (K % 256 == 0 and M > 64, or either operand SP24_NVFP4_MMA: a
 * persistent kernel on pairs of SMs; the workspace then holds the tile images of each operand
 * given as SP24_NVFP4).  NVFP4 w with 16-bit x is decoded inside the kernel to x's type at
 * M <= 64 (dense w with algo auto: M <= 128, one launch per 64 rows of x); at larger M it is
 * first expanded to x's type in the workspace (exact values).
 * K alignment: 16-bit w K % 8, NVFP4 w K % 32, NVFP4 x K % 32.  Operand pointers 16-byte
 * aligned, y 4-byte aligned (SP24_ERR_ALIGN otherwise; the same holds for every GEMM entry
 * point below).  M == 0 or N == 0 is a no-op; K == 0 writes zeros.
 * workspace: device scratch of sp24_gemm_workspace_size() bytes (may be NULL when 0).
 * Kernels that split K across CTAs or warps combine partial sums with fp32 atomics, so two
 * identical calls may differ in the last bits of an output. */
int sp24_gemm_workspace_size(int x_format, int w_format, int sparse, int64_t M, int64_t N,
                             int64_t K, int algo, int64_t* bytes);
int sp24_gemm_dense(const sp24_operand* x, const sp24_operand* w, int64_t M, int64_t N,
                    int64_t K, float* y, void* workspace, int64_t workspace_bytes, int algo,
                    void* stream);

/* [P2] "The mechanism needs both values and their positions": the same product with w in
 * 2:4-compressed form; only kept entries are multiplied.  K alignment: 16-bit values K % 16,
 * NVFP4 values K % 64.  At M > 64 with K % 128 == 0 the product runs on the sparse tensor-core
 * MMA of a persistent CTA-pair kernel (NVFP4 kept values first expanded to x's 16-bit type, exact),
 * which reads the metadata in the layout of sp24_prepare_sparse: the call builds it in the
 * workspace (sp24_gemm_workspace_size counts it). */
int sp24_gemm_sparse24(const sp24_operand* x, const sp24_sparse_operand* w, int64_t M,
                       int64_t N, int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                       int algo, void* stream);

/* [P2] "Ask which sparse implementations were actually selected": a 2:4-eligible weight runs
 * sparse only where that is faster for the problem size; dense may win.  For one weight held
 * in both forms (w_dense: the pruned weight, 16-bit or NVFP4; w_sparse: its compressed form,
 * same format):
 *   sp24_gemm_select  times sp24_gemm_dense and sp24_gemm_sparse24 (algo auto) on `stream`, one
 *                     warm-up and `reps` timed launches each, writes the faster to *use_sparse
 *                     and the per-launch times (us, may be NULL), and records the decision for
 *                     (device, x format, weight format, M, N, K).  Synchronises with the stream;
 *                     not for use during graph capture.  y receives a result of either form.
 *   sp24_gemm_choice  (host only) the recorded decision, else a rule of crossovers measured on
 *                     B200: weights of fewer than 2^20 entries dense (launch-bound); else
 *                     16-bit weights, and NVFP4 weights with 16-bit x, 2:4 for M >= 128
 *                     and dense below; NVFP4 weights with NVFP4 x dense.
 *                     *measured (may be NULL): 1 if recorded.
 *                     SP24_ERR_DTYPE for format pairs without a 2:4 path.
 *   sp24_gemm_auto    runs the GEMM sp24_gemm_choice names; *used_sparse (may be NULL) says
 *                     which.  Asynchronous.
 *   workspace: at least the larger of the two sp24_gemm_workspace_size() values (algo 0).
 *   sp24_gemm_choice_reset forgets every recorded decision. */
int sp24_gemm_select(const sp24_operand* x, const sp24_operand* w_dense,
                     const sp24_sparse_operand* w_sparse, int64_t M, int64_t N, int64_t K,
                     float* y, void* workspace, int64_t workspace_bytes, int reps,
                     int* use_sparse, float* us_dense, float* us_sparse, void* stream);
int sp24_gemm_choice(int x_format, int w_format, int64_t M, int64_t N, int64_t K,
                     int* use_sparse, int* measured);
int sp24_gemm_auto(const sp24_operand* x, const sp24_operand* w_dense,
                   const sp24_sparse_operand* w_sparse, int64_t M, int64_t N, int64_t K,
                   float* y, void* workspace, int64_t workspace_bytes, int* used_sparse,
                   void* stream);
int sp24_gemm_choice_reset(void);

/* ----------------------------------------------------------------------- a7: routed experts */
/* [P1] "Concurrency, not sparsity, is the lever": tokens routed top-k to E experts.
 *   Y[t, s, n] = sum_k x[t, k] W[e, n, k],  e = routing[t, s]   (fp32 [T, topk, N], device)
 *   x        T rows (F16, BF16 or NVFP4), as for sp24_gemm_dense.
 *   routing  device int32 [T, topk]; ids outside [0, E) set the device error word
 *            (SP24_ERR_INVALID_ARG) and leave their outputs 0.
 *   weights  the E experts stacked as one [E*N, K] operand: exactly one of w_dense
 *            (16-bit or NVFP4; NVFP4 experts share one tensor scale, [P5] "The shared global
 *            scale") or w_sparse (2:4-compressed, stacked [E*N, K/2] values + [E*N, K/8] meta).
 *   K alignment: NVFP4 dense K % 256, NVFP4 2:4 K % 512, 16-bit K % 8 (2:4: K % 128).
 *   NVFP4 experts (dense or 2:4) with 16-bit x and N % 128 == 0 run on the tensor cores and
 *   write every output once (the result does not depend on launch order); other cases add
 *   K-slice partial sums with fp32 atomics.
 *   workspace: sp24_gemm_grouped_workspace_size() bytes, 16-byte aligned (routing histogram,
 *   offsets, token tiles, permutation). */
int sp24_gemm_grouped_workspace_size(int64_t T, int topk, int64_t E, int64_t* bytes);
int sp24_gemm_grouped(const sp24_operand* x, const int32_t* routing, int64_t T, int topk,
                      const sp24_operand* w_dense, const sp24_sparse_operand* w_sparse, int64_t E,
                      int64_t N, int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                      void* stream);

/* Expert block of the routed model ([P1] "Concurrency, not sparsity, is the lever"): for each
 * token t,  y[t] = sum_s r[t, s] * h_ts Wd_e^T  with  h_ts = SiLU(x_t Wg_e^T) * (x_t Wu_e^T),
 * e = routing[t, s]; SiLU(g) = g / (1 + e^-g).  h is held in x's 16-bit type; y is fp32.
 *   x          T rows of H entries, F16 or BF16, 16-byte aligned
 *   routing    device int32 [T, topk];  router_w: device fp32 [T, topk]
 *   w_gate_up  the E experts' gate and up weights [E * 2F, H], NVFP4, packed by
 *              sp24_interleave_rows(gate, up, block_rows = 16): rows 32k .. 32k + 15 are gate
 *              rows 16k .. 16k + 15, rows 32k + 16 .. 32k + 31 the up rows of the same features;
 *              gate and up share one tensor scale (sp24_nvfp4_group_tensor_scale); exactly one
 *              of w_gate_up (dense) or w_gate_up_sparse (2:4 values + nibbles, same packing)
 *   w_down     [E * H, F], NVFP4 dense or 2:4 (w_down_sparse), one of the two
 *   y          device fp32 [T, H], overwritten, 16-byte aligned (written as 4-float vectors)
 *   Shapes: F % 64 and H % 128; dense K (H for gate/up, F for down) % 256, 2:4 K % 512;
 *   SP24_ERR_UNSUPPORTED otherwise.  Each routed row's down output is stored once and a token's
 *   slots are summed in slot order in fp32 (deterministic).
 *   workspace: sp24_moe_block_workspace_size() bytes, 16-byte aligned (routing tables, h in
 *   x's type [T*topk, F], the per-slot outputs fp32 [T, topk, H]). */
int sp24_moe_block_workspace_size(int64_t T, int topk, int64_t E, int64_t H, int64_t F,
                                  int64_t* bytes);
int sp24_moe_block(const sp24_operand* x, const int32_t* routing, const float* router_w, int64_t T,
                   int topk, const sp24_operand* w_gate_up,
                   const sp24_sparse_operand* w_gate_up_sparse, const sp24_operand* w_down,
                   const sp24_sparse_operand* w_down_sparse, int64_t E, int64_t H, int64_t F,
                   float* y, void* workspace, int64_t workspace_bytes, void* stream);

/* [P5] "The shared global scale" (gate and up are read together).
 * Row interleave: out[2 * rows, row_bytes] takes block_rows rows of a, then block_rows rows of
 * b, and so on (the gate / up packing of sp24_moe_block).  rows % block_rows == 0, row_bytes % 16
 * == 0, all pointers device and 16-byte aligned. */
int sp24_interleave_rows(const void* a, const void* b, int64_t rows, int64_t row_bytes,
                         int64_t block_rows, void* out, void* stream);

/* ----------------------------------------------------------------------- diagnostics */
/* Number of kernels this library has launched in this process (host-side counter, all
 * devices and streams).  For accounting in benchmarks; memsets are not counted. */
int64_t sp24_kernel_launches(void);

/* Synchronises `stream`, then returns and clears the device error word of the current device
 * (SP24_OK when no kernel reported a problem). */
int sp24_last_device_error(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SP24_H_ */
