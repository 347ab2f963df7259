// NVFP4 quantisation for callers that cannot allocate device memory.
//
// sp24_quantize_nvfp4 needs a few bytes of scratch (the running amax of |T|), which the caller
// normally passes as `workspace`.  Some callers have no way to get one: runtimes that hand out
// only a fixed arena of operand buffers and no general-purpose allocator, plugins hosted by a
// framework whose own caching allocator owns the device memory (a direct cudaMalloc would bypass
// its budget), and latency-bound host loops that must not call cudaMalloc at all because it can
// synchronise the device.  For them this entry point keeps its scratch in a file-scope
// __device__ array instead.
//
// The array exists once per device that loads the library and lives until the process exits.
// Every call on a device shares it and it keeps the last call's contents, so the amax word is
// cleared (cudaMemsetAsync, which allocates nothing) at the start of every call, and two calls
// whose work overlaps on the GPU (different streams, no ordering between them) race on it.
// The array's device address is looked up once per device and cached; a cudaDeviceReset in the
// same process invalidates that address, so a process that resets a device must not call this
// entry point on that device afterwards.
#include <mutex>

#include "sp24_internal.cuh"

namespace sp24 {

int quantize_nvfp4_launch(const void* t, int dtype, int64_t rows, int64_t cols, const float* ts_in,
                          uint8_t* codes, uint8_t* scales, float* ts_out, unsigned int* amax_word,
                          cudaStream_t s);

namespace {

// Largest scratch this entry point can offer: 256 bytes per device.  The quantiser needs one
// 4-byte amax word whatever the tensor's shape.
constexpr int64_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once per device; the
// host-side symbol is a stand-in, never a device address).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SP24_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SP24_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SP24_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SP24_OK;
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_quantize_nvfp4_noalloc(const void* t, int dtype, int64_t rows, int64_t cols,
                                           const float* tensor_scale_in, uint8_t* codes,
                                           uint8_t* scales, float* tensor_scale_out, void* stream) {
  int64_t need = 0;
  int st = sp24_quantize_nvfp4_workspace_size(rows, cols, &need);
  if (st) return st;
  if (need > kNoAllocScratchBytes) return SP24_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st) return st;
  return quantize_nvfp4_launch(t, dtype, rows, cols, tensor_scale_in, codes, scales,
                               tensor_scale_out, reinterpret_cast<unsigned int*>(scratch),
                               as_stream(stream));
}
