/*
 * sp24_oracle.c -- plain, slow, scalar CPU oracle for the 2:4 sparsity / NVFP4 pipeline.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or calls this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg load it.  It
 * shares no code, header or table with the CUDA path.
 *
 * Pages this follows (titles as published; section names in quotes):
 *   [P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went" (robertz.co)
 *   [P2] "Sparse GPU FLOPS Need the Right Zeros in the Right Places" (leviathansystems.co)
 *   [P5] "NVFP4 Without FP4 Hardware" (ai-muninn.com)
 *
 * Every function is a direct statement of its definition: no blocking, no fusion, no
 * reordering of a sum.  Floating-point work that decides an integer (the NVFP4 scale and
 * code choices) is done in IEEE fp32 with round-to-nearest-even, as the readings below fix;
 * GEMM sums are accumulated in fp64.  Build with -ffp-contract=off (no fused multiply-add
 * contraction) so every fp32 operation rounds exactly once.
 *
 * Readings of points the pages leave open (each is repeated in the design notes):
 *   R1  A value is zero when its magnitude bits are all zero (+0 and -0 both count; NaN is
 *       not zero).  A group passes the check when it holds at least two zeros.
 *   R2  Pruning keeps the two entries that come first in the order (|w| descending, index
 *       ascending), |w| compared as the unsigned magnitude bit pattern.  Kept indices are
 *       stored ascending; the other two entries become +0.
 *   R3  Metadata: one nibble per group, nibble = i0 | (i1 << 2) with i0 < i1; nibbles form
 *       a flat stream over the groups in natural order, the even group in the low nibble.
 *   R4  NVFP4 scales: s_t = amax / 2688 (2688 = 6 * 448, the E2M1 and E4M3 maxima) unless a
 *       tensor scale is supplied; d = s_t * 6; block scale sb = E4M3(bmax / d); element
 *       code = sign | E2M1(|t| / (dec(sb) * s_t)); all in fp32, RNE, saturating to the
 *       largest finite value.  When d == 0 the block scale is 0; when dec(sb)*s_t == 0 the
 *       magnitude code is 0.  Packing: element 2i in the low nibble.
 *   R5  A sparse NVFP4 operand quantises the compressed values [N, K/2]: one block scale per
 *       16 stored values.
 *   R21 Pairwise 4:8 (the sparse unit of the tensor cores' packed-FP4 MMA is a pair of
 *       entries): chunks of 8 along K; a chunk passes when at most two of its four pairs hold
 *       a nonzero; pruning keeps the two pairs of largest fp32 |a| + |b| (NaN highest, ties to
 *       the lower pair); nibble i0 | i1 << 2 per chunk, stored as in R3.
 *   R22 The activations of the pairwise-4:8 FP4 GEMM use the R4 steps over 32-value blocks
 *       (that MMA reads one scale per 32 K for both operands).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element types known to the oracle (its own numbering) */
enum { O_F16 = 0, O_BF16 = 1, O_F32 = 2 };
/* operation kinds */
enum { O_MATMUL = 0, O_CONV = 1 };
/* return codes */
enum { O_OK = 0, O_EARG = 1, O_ESHAPE = 2, O_EDTYPE = 3 };

static int elem_bytes(int dtype) {
  if (dtype == O_F16 || dtype == O_BF16) return 2;
  if (dtype == O_F32) return 4;
  return 0;
}

/* Raw bits of element i. */
static uint32_t raw_bits(const void* p, int dtype, int64_t i) {
  if (dtype == O_F32) return ((const uint32_t*)p)[i];
  return ((const uint16_t*)p)[i];
}

static void put_raw_bits(void* p, int dtype, int64_t i, uint32_t v) {
  if (dtype == O_F32) ((uint32_t*)p)[i] = v;
  else ((uint16_t*)p)[i] = (uint16_t)v;
}

/* Magnitude bits: everything but the sign bit. Monotone in |value| for non-NaN values. */
static uint32_t mag_bits(uint32_t raw, int dtype) {
  return dtype == O_F32 ? (raw & 0x7fffffffu) : (raw & 0x7fffu);
}

/* IEEE binary16 -> double, from the format definition (1 sign, 5 exponent, 10 fraction). */
static double f16_value(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 0x1f, f = h & 0x3ff;
  double v;
  if (e == 0) v = ldexp((double)f, -24);                 /* subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31) v = f ? NAN : INFINITY;
  else v = ldexp(1.0 + f / 1024.0, e - 15);
  return s ? -v : v;
}

/* bfloat16 -> double: the upper 16 bits of an IEEE binary32. */
static double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double elem_value(const void* p, int dtype, int64_t i) {
  if (dtype == O_F16) return f16_value(((const uint16_t*)p)[i]);
  if (dtype == O_BF16) return bf16_value(((const uint16_t*)p)[i]);
  return (double)((const float*)p)[i];
}

/* fp32 value of element i (exact: f16 and bf16 embed in binary32). */
static float elem_f32(const void* p, int dtype, int64_t i) { return (float)elem_value(p, dtype, i); }

/* ---------------------------------------------------------------- group addressing */

/* Validates the shape for an operation and returns the number of groups of four.
 * MATMUL: shape [rows, K] (any ndim >= 1: the last axis is K, the others are flattened).
 * CONV:   shape [K, C, R, S]; groups run along C ([P2] "The operation determines which four
 *         entries belong together": C must be divisible by four). */
static int64_t group_count(int op, const int64_t* shape, int ndim, int* err) {
  *err = O_OK;
  if (!shape || ndim < 1 || ndim > 4) { *err = O_EARG; return 0; }
  for (int d = 0; d < ndim; ++d)
    if (shape[d] < 0) { *err = O_ESHAPE; return 0; }
  if (op == O_MATMUL) {
    int64_t n = 1;
    for (int d = 0; d < ndim; ++d) n *= shape[d];
    if (shape[ndim - 1] % 4) { *err = O_ESHAPE; return 0; }
    return n / 4;
  }
  if (op == O_CONV) {
    if (ndim != 4 || shape[1] % 4) { *err = O_ESHAPE; return 0; }
    return shape[0] * (shape[1] / 4) * shape[2] * shape[3];
  }
  *err = O_EARG;
  return 0;
}

/* Element index of member i (0..3) of group g. */
static int64_t group_member(int op, const int64_t* shape, int ndim, int64_t g, int i) {
  if (op == O_MATMUL) return g * 4 + i;
  (void)ndim;
  /* group g enumerates (k, j, r, s) in row-major order over [K, C/4, R, S] */
  int64_t C = shape[1], R = shape[2], S = shape[3];
  int64_t s = g % S, t = g / S;
  int64_t r = t % R;
  t /= R;
  int64_t j = t % (C / 4), k = t / (C / 4);
  return ((k * C + (4 * j + i)) * R + r) * S + s;
}

/* Index of stored value t (0/1) of group g in the compressed values tensor.
 * MATMUL: values [rows, K/2], group g's values at 2g, 2g+1.
 * CONV:   values [K, C/2, R, S], group (k,j,r,s) -> values[k, 2j+t, r, s]. */
static int64_t value_slot(int op, const int64_t* shape, int64_t g, int t) {
  if (op == O_MATMUL) return g * 2 + t;
  int64_t C = shape[1], R = shape[2], S = shape[3];
  int64_t s = g % S, u = g / S;
  int64_t r = u % R;
  u /= R;
  int64_t j = u % (C / 4), k = u / (C / 4);
  return ((k * (C / 2) + (2 * j + t)) * R + r) * S + s;
}

/* ---------------------------------------------------------------- a1: eligibility check */

/* [P2] "The operation determines which four entries belong together" and "Two half-zero
 * vectors produce different pattern answers": a group of four entries along the reduction
 * axis is eligible when it holds at least two zeros; each group is judged on its own.
 * Writes pass[g] = 1/0 and returns the number of failing groups (negative on error). */
int64_t sp24o_check_24(const void* w, int dtype, int op, const int64_t* shape, int ndim,
                       uint8_t* pass) {
  int err;
  if (!elem_bytes(dtype)) return -O_EDTYPE;
  int64_t G = group_count(op, shape, ndim, &err);
  if (err) return -err;
  int64_t fails = 0;
  for (int64_t g = 0; g < G; ++g) {
    int zeros = 0;
    for (int i = 0; i < 4; ++i) {
      uint32_t m = mag_bits(raw_bits(w, dtype, group_member(op, shape, ndim, g, i)), dtype);
      if (m == 0) zeros++;
    }
    int ok = zeros >= 2;
    if (pass) pass[g] = (uint8_t)ok;
    if (!ok) fails++;
  }
  return fails;
}

/* ---------------------------------------------------------------- a2: prune / compress */

/* The two kept member indices (ascending) of a group, per reading R2 ([P1] "What 2:4
 * actually is": two of every four weights are forced to zero; the largest magnitudes
 * survive).  Ranks every member by how many others precede it in the order
 * (|w| descending, index ascending); the members of rank 0 and 1 are kept. */
static void kept_pair(const uint32_t mag[4], int* i0, int* i1) {
  int kept[2], nk = 0;
  for (int i = 0; i < 4; ++i) {
    int rank = 0;
    for (int j = 0; j < 4; ++j) {
      if (j == i) continue;
      if (mag[j] > mag[i] || (mag[j] == mag[i] && j < i)) rank++;
    }
    if (rank < 2) kept[nk++] = i;
  }
  *i0 = kept[0];
  *i1 = kept[1];
}

static void group_mags(const void* w, int dtype, int op, const int64_t* shape, int ndim,
                       int64_t g, uint32_t mag[4], int64_t idx[4]) {
  for (int i = 0; i < 4; ++i) {
    idx[i] = group_member(op, shape, ndim, g, i);
    mag[i] = mag_bits(raw_bits(w, dtype, idx[i]), dtype);
  }
}

/* Dense pruned copy: kept entries copied bitwise, the other two set to +0. */
int sp24o_prune_24(const void* w, int dtype, int op, const int64_t* shape, int ndim, void* out) {
  int err;
  if (!elem_bytes(dtype)) return O_EDTYPE;
  int64_t G = group_count(op, shape, ndim, &err);
  if (err) return err;
  for (int64_t g = 0; g < G; ++g) {
    uint32_t mag[4];
    int64_t idx[4];
    int i0, i1;
    group_mags(w, dtype, op, shape, ndim, g, mag, idx);
    kept_pair(mag, &i0, &i1);
    for (int i = 0; i < 4; ++i)
      put_raw_bits(out, dtype, idx[i], (i == i0 || i == i1) ? raw_bits(w, dtype, idx[i]) : 0u);
  }
  return O_OK;
}

/* [P1] "What 2:4 actually is": the stored form is the two kept values plus a 2-bit index
 * for each.  values get the kept entries in ascending index order (bit copies); meta gets
 * nibble i0 | i1 << 2 per group (reading R3).  meta must hold ceil(G/2) bytes. */
int sp24o_compress_24(const void* w, int dtype, int op, const int64_t* shape, int ndim,
                      void* values, uint8_t* meta) {
  int err;
  if (!elem_bytes(dtype)) return O_EDTYPE;
  int64_t G = group_count(op, shape, ndim, &err);
  if (err) return err;
  memset(meta, 0, (size_t)((G + 1) / 2));
  for (int64_t g = 0; g < G; ++g) {
    uint32_t mag[4];
    int64_t idx[4];
    int i0, i1;
    group_mags(w, dtype, op, shape, ndim, g, mag, idx);
    kept_pair(mag, &i0, &i1);
    put_raw_bits(values, dtype, value_slot(op, shape, g, 0), raw_bits(w, dtype, idx[i0]));
    put_raw_bits(values, dtype, value_slot(op, shape, g, 1), raw_bits(w, dtype, idx[i1]));
    uint8_t nib = (uint8_t)(i0 | (i1 << 2));
    meta[g / 2] |= (uint8_t)((g % 2) ? (nib << 4) : nib);
  }
  return O_OK;
}

/* Inverse of compress: kept values back at their indices, +0 elsewhere.  A nibble whose two
 * indices are not strictly ascending is invalid and returns O_EARG. */
int sp24o_decompress_24(const void* values, const uint8_t* meta, int dtype, int op,
                        const int64_t* shape, int ndim, void* out) {
  int err;
  if (!elem_bytes(dtype)) return O_EDTYPE;
  int64_t G = group_count(op, shape, ndim, &err);
  if (err) return err;
  for (int64_t g = 0; g < G; ++g) {
    int nib = (meta[g / 2] >> ((g % 2) * 4)) & 0xf;
    int i0 = nib & 3, i1 = nib >> 2;
    if (i0 >= i1) return O_EARG;
    for (int i = 0; i < 4; ++i) {
      int64_t e = group_member(op, shape, ndim, g, i);
      uint32_t v = 0;
      if (i == i0) v = raw_bits(values, dtype, value_slot(op, shape, g, 0));
      if (i == i1) v = raw_bits(values, dtype, value_slot(op, shape, g, 1));
      put_raw_bits(out, dtype, e, v);
    }
  }
  return O_OK;
}

/* ---------------------------------------------------------------- pairwise 4:8 */

/* Pairwise 4:8, the sparse pattern of the tensor cores' packed-FP4 kind, per reading R21: along
 * K, chunks of 8 consecutive entries, each made of four pairs (2j, 2j + 1).  A chunk is eligible
 * when at most two of its pairs hold a nonzero entry (+0 and -0 are zero).  Pruning keeps the two
 * pairs of largest score |a| + |b| (one IEEE fp32 addition of the entries' fp32 magnitudes), NaN
 * scores above every number, ties to the lower pair.  The compressed chunk is its kept pairs in
 * ascending order (values [rows, K/2]) plus a nibble i0 | i1 << 2 (pair indices, i0 < i1), chunk
 * 2c of the flat chunk sequence in the low nibble of byte c. */

/* Does pair a (score sa, index ia) come before pair b in the keep order? */
static int pair_before(float sa, int ia, float sb, int ib) {
  int na = isnan(sa), nb = isnan(sb);
  if (na != nb) return na;
  if (!na && sa != sb) return sa > sb;
  return ia < ib;
}

static void kept_pairs48(const void* w, int dtype, int64_t base, int* i0, int* i1) {
  float sc[4];
  for (int j = 0; j < 4; ++j) {
    volatile float a = fabsf(elem_f32(w, dtype, base + 2 * j));
    volatile float b = fabsf(elem_f32(w, dtype, base + 2 * j + 1));
    volatile float sum = a + b;
    sc[j] = sum;
  }
  int kept[2], nk = 0;
  for (int i = 0; i < 4; ++i) {
    int rank = 0;
    for (int j = 0; j < 4; ++j)
      if (j != i && pair_before(sc[j], j, sc[i], i)) rank++;
    if (rank < 2) kept[nk++] = i;
  }
  *i0 = kept[0];
  *i1 = kept[1];
}

/* Per-chunk pass map [rows, K/8] (may be NULL); returns the failing-chunk count or -code. */
int64_t sp24o_check_48(const void* w, int dtype, int64_t rows, int64_t K, uint8_t* pass) {
  if (!elem_bytes(dtype)) return -O_EDTYPE;
  if (rows < 0 || K < 0 || K % 8) return -O_ESHAPE;
  int64_t fails = 0;
  for (int64_t c = 0; c < rows * (K / 8); ++c) {
    int nonzero_pairs = 0;
    for (int j = 0; j < 4; ++j) {
      uint32_t a = mag_bits(raw_bits(w, dtype, 8 * c + 2 * j), dtype);
      uint32_t b = mag_bits(raw_bits(w, dtype, 8 * c + 2 * j + 1), dtype);
      if (a || b) nonzero_pairs++;
    }
    int ok = nonzero_pairs <= 2;
    if (pass) pass[c] = (uint8_t)ok;
    if (!ok) fails++;
  }
  return fails;
}

int sp24o_compress_48(const void* w, int dtype, int64_t rows, int64_t K, void* values, uint8_t* meta) {
  if (!elem_bytes(dtype)) return O_EDTYPE;
  if (rows < 0 || K < 0 || K % 8) return O_ESHAPE;
  const int64_t C = rows * (K / 8);
  memset(meta, 0, (size_t)((C + 1) / 2));
  for (int64_t c = 0; c < C; ++c) {
    int i0, i1;
    kept_pairs48(w, dtype, 8 * c, &i0, &i1);
    put_raw_bits(values, dtype, 4 * c + 0, raw_bits(w, dtype, 8 * c + 2 * i0));
    put_raw_bits(values, dtype, 4 * c + 1, raw_bits(w, dtype, 8 * c + 2 * i0 + 1));
    put_raw_bits(values, dtype, 4 * c + 2, raw_bits(w, dtype, 8 * c + 2 * i1));
    put_raw_bits(values, dtype, 4 * c + 3, raw_bits(w, dtype, 8 * c + 2 * i1 + 1));
    uint8_t nib = (uint8_t)(i0 | (i1 << 2));
    meta[c / 2] |= (uint8_t)((c % 2) ? (nib << 4) : nib);
  }
  return O_OK;
}

/* Kept pairs back at their places, +0 elsewhere; a nibble whose pair indices are not strictly
 * ascending returns O_EARG. */
int sp24o_decompress_48(const void* values, const uint8_t* meta, int dtype, int64_t rows, int64_t K, void* out) {
  if (!elem_bytes(dtype)) return O_EDTYPE;
  if (rows < 0 || K < 0 || K % 8) return O_ESHAPE;
  for (int64_t c = 0; c < rows * (K / 8); ++c) {
    int nib = (meta[c / 2] >> ((c % 2) * 4)) & 0xf;
    int i0 = nib & 3, i1 = nib >> 2;
    if (i0 >= i1) return O_EARG;
    for (int j = 0; j < 4; ++j) {
      for (int h = 0; h < 2; ++h) {
        uint32_t v = 0;
        if (j == i0) v = raw_bits(values, dtype, 4 * c + h);
        if (j == i1) v = raw_bits(values, dtype, 4 * c + 2 + h);
        put_raw_bits(out, dtype, 8 * c + 2 * j + h, v);
      }
    }
  }
  return O_OK;
}

/* ---------------------------------------------------------------- a3: NVFP4 */

/* E2M1 magnitude codes 0..7 (1 exponent bit pair, 1 mantissa bit, bias 1):
 * 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6. */
double sp24o_e2m1_value(int code) {
  int mag = code & 7;
  int e = mag >> 1, m = mag & 1;
  double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return (code & 8) ? -v : v;
}

/* E4M3 (FN variant: no infinities, 0x7f / 0xff are NaN, largest finite 448), bias 7. */
double sp24o_e4m3_value(int code) {
  int mag = code & 0x7f;
  if (mag == 0x7f) return NAN;
  int e = mag >> 3, m = mag & 7;
  double v = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return (code & 0x80) ? -v : v;
}

/* Round-to-nearest over a finite code table by exhaustive search; a value exactly half way
 * between two neighbours takes the even code; anything above the largest value saturates to
 * it (the search simply finds the largest).  x must be >= 0 and not NaN. */
static int nearest_code(double x, int ncodes, double (*value)(int)) {
  /* saturation first: at or above the largest finite value the distances below would round
   * (|6 - 1e30| == |0 - 1e30| in fp64) */
  int top = ncodes - 1;
  while (isnan(value(top))) --top;
  if (x >= value(top)) return top;
  int best = 0;
  double bestd = fabs(value(0) - x);
  for (int c = 1; c < ncodes; ++c) {
    double v = value(c);
    if (isnan(v)) continue;
    double d = fabs(v - x);
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return best;
}

/* Magnitude code 0..7 of x >= 0 on the E2M1 grid (RNE, saturating at 6). */
int sp24o_e2m1_round(double x) { return nearest_code(x, 8, sp24o_e2m1_value); }

/* Magnitude code 0..126 of x >= 0 on the E4M3 grid (RNE, saturating at 448). */
int sp24o_e4m3_round(double x) { return nearest_code(x, 127, sp24o_e4m3_value); }

/* Largest |t| of the tensor, exact in fp32. */
static float tensor_amax(const void* t, int dtype, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(elem_f32(t, dtype, i));
    if (a > amax) amax = a;
  }
  return amax;
}

/* Tensor scale per reading R4 ([P5] "Convert BF16 to NVFP4 yourself": one FP32 global scale
 * per tensor; "The shared global scale": taken from the max absolute value). */
float sp24o_nvfp4_tensor_scale(const void* t, int dtype, int64_t n) {
  volatile float amax = tensor_amax(t, dtype, n);
  volatile float s = amax / 2688.0f;
  return s;
}

/* NVFP4 encode of T[rows, cols] ([P5] "Convert BF16 to NVFP4 yourself": 4-bit E2M1 values,
 * one FP8 E4M3 scale per block of consecutive values, one FP32 global scale), per reading R4.
 * The pages' block is 16 values; block 32 is the activation form the sparse FP4 MMA reads
 * (one scale per 32 K, reading R22), computed by the same steps over 32 values.
 * codes: [rows, cols/2] bytes, element 2i in the low nibble; scales: [rows, cols/block] E4M3
 * bytes.  ts_in: NULL to derive the tensor scale from amax, else the shared scale to use
 * ([P5] "The shared global scale").  *ts_out receives the scale used. */
int sp24o_nvfp4_encode_blk(const void* t, int dtype, int64_t rows, int64_t cols, int block, const float* ts_in,
                           uint8_t* codes, uint8_t* scales, float* ts_out) {
  if (!elem_bytes(dtype)) return O_EDTYPE;
  if (block != 16 && block != 32) return O_EARG;
  if (rows < 0 || cols < 0 || cols % block) return O_ESHAPE;
  volatile float s_t = ts_in ? *ts_in : sp24o_nvfp4_tensor_scale(t, dtype, rows * cols);
  if (ts_out) *ts_out = s_t;
  volatile float d = s_t * 6.0f;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < cols / block; ++b) {
      int64_t base = r * cols + b * block;
      float bmax = 0.0f;
      for (int i = 0; i < block; ++i) {
        float a = fabsf(elem_f32(t, dtype, base + i));
        if (a > bmax) bmax = a;
      }
      int sb = 0;
      if (d != 0.0f) {
        volatile float q = bmax / d;
        sb = sp24o_e4m3_round((double)q);
      }
      scales[r * (cols / block) + b] = (uint8_t)sb;
      volatile float sc = (float)sp24o_e4m3_value(sb) * s_t;
      for (int i = 0; i < block; ++i) {
        float v = elem_f32(t, dtype, base + i);
        int mag = 0;
        if (sc != 0.0f) {
          volatile float q = fabsf(v) / sc;
          mag = sp24o_e2m1_round((double)q);
        }
        int code = (signbit(v) ? 8 : 0) | mag;
        int64_t e = base + i;
        uint8_t* byte = &codes[e / 2];
        if (e % 2 == 0) *byte = (uint8_t)((*byte & 0xf0) | code);
        else *byte = (uint8_t)((*byte & 0x0f) | (code << 4));
      }
    }
  }
  return O_OK;
}

int sp24o_nvfp4_encode(const void* t, int dtype, int64_t rows, int64_t cols, const float* ts_in,
                       uint8_t* codes, uint8_t* scales, float* ts_out) {
  return sp24o_nvfp4_encode_blk(t, dtype, rows, cols, 16, ts_in, codes, scales, ts_out);
}

/* NVFP4 decode: E2M1(code) * E4M3(scale of the element's block) * s_t, evaluated in fp64. */
int sp24o_nvfp4_decode_blk(const uint8_t* codes, const uint8_t* scales, float s_t, int64_t rows,
                           int64_t cols, int block, double* out) {
  if (block != 16 && block != 32) return O_EARG;
  if (rows < 0 || cols < 0 || cols % block) return O_ESHAPE;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      int64_t e = r * cols + c;
      int code = (codes[e / 2] >> ((e % 2) * 4)) & 0xf;
      double sb = sp24o_e4m3_value(scales[r * (cols / block) + c / block]);
      out[e] = sp24o_e2m1_value(code) * sb * (double)s_t;
    }
  return O_OK;
}

int sp24o_nvfp4_decode(const uint8_t* codes, const uint8_t* scales, float s_t, int64_t rows,
                       int64_t cols, double* out) {
  return sp24o_nvfp4_decode_blk(codes, scales, s_t, rows, cols, 16, out);
}

/* Element values of a real tensor in fp64 (exact). */
int sp24o_to_double(const void* t, int dtype, int64_t n, double* out) {
  if (!elem_bytes(dtype)) return O_EDTYPE;
  for (int64_t i = 0; i < n; ++i) out[i] = elem_value(t, dtype, i);
  return O_OK;
}

/* ---------------------------------------------------------------- a4-a7: GEMM */

/* Y[m,n] = sum_k X[m,k] * W[n,k] in fp64, k ascending; S[m,n] = sum_k |X[m,k]| |W[n,k]| (the
 * tolerance scale).  X [M,K] and W [N,K] are decoded operands. */
int sp24o_gemm(const double* X, const double* W, int64_t M, int64_t N, int64_t K, double* Y,
               double* S, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        acc += X[m * K + k] * W[n * K + k];
        aacc += fabs(X[m * K + k]) * fabs(W[n * K + k]);
      }
      Y[m * N + n] = acc;
      if (S) S[m * N + n] = aacc;
    }
  (void)nthreads;
  return O_OK;
}

/* The same product with W in compressed form: V [N, K/2] decoded kept values and the nibble
 * stream meta of W [N, K] (reading R3).  Only kept entries are multiplied ([P2] "The
 * mechanism needs both values and their positions": the positions select the matching
 * entries of the other operand). */
int sp24o_gemm_sparse(const double* X, const double* V, const uint8_t* meta, int64_t M, int64_t N,
                      int64_t K, double* Y, double* S, int nthreads) {
  if (K % 4) return O_ESHAPE;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t j = 0; j < K / 4; ++j) {
        int64_t g = n * (K / 4) + j;
        int nib = (meta[g / 2] >> ((g % 2) * 4)) & 0xf;
        int i0 = nib & 3, i1 = nib >> 2;
        double x0 = X[m * K + 4 * j + i0], x1 = X[m * K + 4 * j + i1];
        double v0 = V[n * (K / 2) + 2 * j], v1 = V[n * (K / 2) + 2 * j + 1];
        acc += x0 * v0;
        acc += x1 * v1;
        aacc += fabs(x0) * fabs(v0);
        aacc += fabs(x1) * fabs(v1);
      }
      Y[m * N + n] = acc;
      if (S) S[m * N + n] = aacc;
    }
  (void)nthreads;
  return O_OK;
}

/* Routed expert product: Y[t, s, n] = sum_k X[t, k] * W[e, n, k] with e = routing[t, s]
 * ([P1] "Concurrency, not sparsity, is the lever": top-10 routing of tokens to 512 experts).
 * W holds E decoded expert weights [E, N, K]; an out-of-range expert id returns O_EARG. */
int sp24o_moe(const double* X, const int32_t* routing, const double* W, int64_t T, int topk,
              int64_t E, int64_t N, int64_t K, double* Y, double* S, int nthreads) {
  for (int64_t i = 0; i < T * topk; ++i)
    if (routing[i] < 0 || routing[i] >= E) return O_EARG;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
  for (int64_t t = 0; t < T; ++t)
    for (int s = 0; s < topk; ++s) {
      const double* We = W + (int64_t)routing[t * topk + s] * N * K;
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          acc += X[t * K + k] * We[n * K + k];
          aacc += fabs(X[t * K + k]) * fabs(We[n * K + k]);
        }
        Y[(t * topk + s) * N + n] = acc;
        if (S) S[(t * topk + s) * N + n] = aacc;
      }
    }
  (void)nthreads;
  return O_OK;
}

int sp24o_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
