// a3 for a group of tensors: one shared NVFP4 tensor scale.
//
// [P5] "The shared global scale": one FP32 global scale may serve a group of tensors (the q / k /
// v projections, gate / up, the four projections of a block) that a kernel reads together, and
// it comes from the largest absolute value.  The group's scale is that of the group's entries
// taken together:  s = max_i amax(|T_i|) / 2688  (2688 = 6 * 448, one IEEE fp32 division),
// the scale sp24_quantize_nvfp4 derives for a single tensor.  Each tensor is then quantised with
// sp24_quantize_nvfp4(T_i, tensor_scale_in = s).
//
// One launch reads up to 16 tensors back to back as one sequence of 16-byte vectors (grid-
// stride, streaming loads, a block max, one atomicMax per CTA on the float's bit pattern: the
// values are non-negative, so their bit patterns order like the values); a one-thread kernel
// turns the amax word into the scale.  NaN entries are skipped by the max (as a NaN compares
// false); an infinity gives an infinite scale.
#include "sp24_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace sp24 {
namespace {

constexpr int kGroupMax = 16;  // tensors per launch
constexpr int kGThreads = 256;

struct GroupAmax {
  const uint4* p[kGroupMax];
  int64_t start[kGroupMax + 1];  // first 16-byte vector of tensor i in the launch's sequence
  int n;
};

template <int DT>
__device__ __forceinline__ float abs16(uint32_t h) {
  if (DT == SP24_BF16) return fabsf(__uint_as_float(h << 16));
  return fabsf(__half2float(__ushort_as_half((unsigned short)h)));
}

template <int DT>
__global__ void __launch_bounds__(kGThreads) group_amax_kernel(const __grid_constant__ GroupAmax g,
                                                               unsigned int* __restrict__ amax_bits) {
  float m = 0.0f;
  const int64_t total = g.start[g.n];
  int i = 0;
  for (int64_t v = (int64_t)blockIdx.x * kGThreads + threadIdx.x; v < total; v += (int64_t)gridDim.x * kGThreads) {
    while (v >= g.start[i + 1]) ++i;  // v only grows, so the tensor index only moves forward
    const uint4 x = __ldcs(g.p[i] + (v - g.start[i]));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (DT == SP24_F32) {
        m = fmaxf(m, fabsf(__uint_as_float(w[k])));
      } else {
        m = fmaxf(m, abs16<DT>(w[k] & 0xffffu));
        m = fmaxf(m, abs16<DT>(w[k] >> 16));
      }
    }
  }
  unsigned int u = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  __shared__ unsigned int wmax[kGThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = u;
  __syncthreads();
  if (threadIdx.x < 32) {
    unsigned int x = threadIdx.x < kGThreads / 32 ? wmax[threadIdx.x] : 0u;
    x = __reduce_max_sync(0xffffffffu, x);
    if (threadIdx.x == 0 && x) atomicMax(amax_bits, x);
  }
}

__global__ void group_scale_kernel(const unsigned int* __restrict__ amax_bits, float* __restrict__ ts_out) {
  *ts_out = __fdiv_rn(__uint_as_float(*amax_bits), 2688.0f);
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_nvfp4_group_tensor_scale_workspace_size(int64_t* bytes) {
  if (!bytes) return SP24_ERR_INVALID_ARG;
  *bytes = 16;
  return SP24_OK;
}

extern "C" int sp24_nvfp4_group_tensor_scale(const void* const* tensors, const int64_t* numels, int n, int dtype,
                                             float* tensor_scale_out, void* workspace, int64_t workspace_bytes,
                                             void* stream) {
  if (n < 0 || (n > 0 && (!tensors || !numels)) || !tensor_scale_out) return SP24_ERR_INVALID_ARG;
  const int eb = elem_bytes(dtype);
  if (!eb) return SP24_ERR_DTYPE;
  for (int i = 0; i < n; ++i) {
    if (numels[i] < 0 || (numels[i] * eb) % 16) return SP24_ERR_SHAPE;
    if (numels[i] > 0 && !tensors[i]) return SP24_ERR_INVALID_ARG;
    if (numels[i] > 0 && !aligned(tensors[i], 16)) return SP24_ERR_ALIGN;
  }
  if (!workspace || workspace_bytes < 16) return SP24_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return SP24_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  unsigned int* amax = reinterpret_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(amax, 0, 4, s) != cudaSuccess) return SP24_ERR_CUDA;
  int launched = 0;
  for (int base = 0; base < n; base += kGroupMax) {
    GroupAmax g{};
    g.n = n - base < kGroupMax ? n - base : kGroupMax;
    g.start[0] = 0;
    for (int i = 0; i < g.n; ++i) {
      g.p[i] = reinterpret_cast<const uint4*>(tensors[base + i]);
      g.start[i + 1] = g.start[i] + numels[base + i] * eb / 16;
    }
    const int64_t total = g.start[g.n];
    if (total == 0) continue;
    int64_t blocks = (total + kGThreads - 1) / kGThreads;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (dtype == SP24_F32)
      group_amax_kernel<SP24_F32><<<(unsigned)blocks, kGThreads, 0, s>>>(g, amax);
    else if (dtype == SP24_BF16)
      group_amax_kernel<SP24_BF16><<<(unsigned)blocks, kGThreads, 0, s>>>(g, amax);
    else
      group_amax_kernel<SP24_F16><<<(unsigned)blocks, kGThreads, 0, s>>>(g, amax);
    ++launched;
  }
  group_scale_kernel<<<1, 1, 0, s>>>(amax, tensor_scale_out);
  return launch_status(launched + 1);
}
