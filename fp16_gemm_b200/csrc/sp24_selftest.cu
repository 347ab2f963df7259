// The bounded-wait unwind of the tensor-core kernels, exercised on demand.
//
// Every device-side wait of this library (mbarrier phases, TMA and bulk-copy completions) is
// bounded by the wait limit.  When a wait runs out, a kernel records SP24_ERR_DEVICE_TIMEOUT in
// the device error word, waits (bounded) for its own copies still in flight, frees the tensor
// memory it holds and returns, so the context stays usable.  This kernel goes through exactly
// that path with the same helpers: it allocates TMEM, starts a bulk copy that lands, then waits
// on an mbarrier phase that nothing completes (one arrival expected, none made).  Nothing
// faults, traps or spins without bound; the host reads the outcome with sp24_last_device_error.
#include "sp24_internal.cuh"
#include "sp24_stream.cuh"

namespace sp24 {
namespace {

__global__ void __launch_bounds__(64, 1) wait_timeout_kernel(const uint8_t* __restrict__ src, int* __restrict__ out) {
  __shared__ __align__(16) uint8_t buf[1024];
  __shared__ uint64_t landed, never;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    tc::mbar_init(&landed, 1);
    tc::mbar_init(&never, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(&tmem_base, 32);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (threadIdx.x == 32) {
    tc::mbar_arrive_expect_tx(&landed, 1024);
    stream::bulk_g2s(buf, src, 1024, &landed);
    const bool ok = tc::mbar_wait(&never, 0);  // runs out: nothing arrives on `never`
    if (!ok) set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
    // the unwind: a copy in flight lands before the CTA's shared memory goes away
    const bool drained = tc::mbar_wait(&landed, 0);
    out[0] = ok ? 1 : 2;
    out[1] = drained ? (int)buf[1023] + 1 : 0;
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, 32);
  }
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_set_wait_limit(unsigned long long ns) {
  if (ns == 0) return SP24_ERR_INVALID_ARG;
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns)) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
}

extern "C" int sp24_get_wait_limit(unsigned long long* ns) {
  if (!ns) return SP24_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(ns, g_wait_limit_ns, sizeof(*ns)) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
}

extern "C" int sp24_selftest_wait_timeout(const void* src, int* out, void* stream) {
  if (!src || !out) return SP24_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(out, 4)) return SP24_ERR_ALIGN;
  wait_timeout_kernel<<<1, 64, 0, as_stream(stream)>>>(static_cast<const uint8_t*>(src), out);
  return launch_status();
}
