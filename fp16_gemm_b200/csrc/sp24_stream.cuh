// Bulk-copy streaming pipeline for the HBM-bound kernels.
//
// Each CTA walks the chunks c = blockIdx.x, blockIdx.x + gridDim.x, ... of a contiguous input
// (CHUNK bytes each).  Thread 0 keeps S chunks in flight with cp.async.bulk into a ring of
// shared-memory stages (one mbarrier per stage); all threads consume a stage, meet at a
// __syncthreads, and thread 0 refills the stage with the chunk S ahead.  DRAM therefore sees a
// steady S * CHUNK bytes per CTA in flight, independent of registers and of the consumer's
// instruction count.  Waits are bounded: on timeout the CTA records SP24_ERR_DEVICE_TIMEOUT
// and all threads leave the loop together.
#pragma once

#include "sp24_internal.cuh"
#include "sp24_tc.cuh"

namespace sp24 {
namespace stream {

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}

// Runs body(stage_ptr, segment, chunk_index_in_segment, chunk_bytes) over this CTA's chunks of
// two inputs taken as one sequence: the chunks of `a` (abytes), then those of `b` (bbytes, may
// be 0).  Chunks c = blockIdx.x, blockIdx.x + gridDim.x, ... of that sequence.  Sizes are
// multiples of 16, sources 16-byte aligned.  `ring` must hold S * CHUNK bytes of dynamic shared
// memory, 16-byte aligned.
template <int CHUNK, int S, class Body>
__device__ __forceinline__ void for_each_chunk2(const uint8_t* __restrict__ a, int64_t abytes,
                                                const uint8_t* __restrict__ b, int64_t bbytes, uint8_t* ring,
                                                Body&& body) {
  __shared__ uint64_t bars[S];
  __shared__ int abort_flag;
  const int64_t na = (abytes + CHUNK - 1) / CHUNK;
  const int64_t nchunks = na + (bbytes + CHUNK - 1) / CHUNK;
  const int64_t mine = blockIdx.x < nchunks ? (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) tc::mbar_init(&bars[s], 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  // (segment, byte offset in it, size) of sequence chunk c
  auto locate = [&](int64_t c, int& seg, int64_t& off, uint32_t& sz) {
    seg = c >= na;
    off = (seg ? c - na : c) * (int64_t)CHUNK;
    const int64_t n = seg ? bbytes : abytes;
    sz = (uint32_t)(n - off < CHUNK ? n - off : CHUNK);
  };
  auto issue = [&](int64_t i) {
    const int s = (int)(i % S);
    int seg;
    int64_t off;
    uint32_t sz;
    locate(blockIdx.x + i * gridDim.x, seg, off, sz);
    tc::mbar_arrive_expect_tx(&bars[s], sz);
    bulk_g2s(ring + s * CHUNK, (seg ? b : a) + off, sz, &bars[s]);
  };
  if (threadIdx.x == 0)
    for (int64_t i = 0; i < (mine < S ? mine : S); ++i) issue(i);
  int64_t i = 0;
  for (; i < mine; ++i) {
    const int s = (int)(i % S);
    const bool ok = tc::mbar_wait(&bars[s], (uint32_t)((i / S) & 1));
    if (!ok) abort_flag = 1;
    int seg;
    int64_t off;
    uint32_t sz;
    locate(blockIdx.x + i * gridDim.x, seg, off, sz);
    if (ok) body(ring + s * CHUNK, seg, off / CHUNK, (int)sz);
    __syncthreads();
    if (abort_flag) break;
    if (threadIdx.x == 0 && i + S < mine) issue(i + S);
  }
  if (threadIdx.x == 0 && abort_flag) {
    set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
    // copies already issued must land before the CTA's shared memory goes away
    const int64_t last = i + S < mine ? i + S : mine;
    for (int64_t j = i; j < last; ++j) tc::mbar_wait(&bars[j % S], (uint32_t)((j / S) & 1));
  }
}

// As for_each_chunk below, with chunks of `ch` bytes (a multiple of 16, at most CHUNK) chosen at
// run time; stages stay CHUNK bytes apart in `ring`.
template <int CHUNK, int S, class Body>
__device__ __forceinline__ void for_each_chunk_rt(const uint8_t* __restrict__ src, int64_t nbytes, int ch,
                                                  uint8_t* ring, Body&& body) {
  __shared__ uint64_t bars[S];
  __shared__ int abort_flag;
  const int64_t nchunks = (nbytes + ch - 1) / ch;
  const int64_t mine = blockIdx.x < nchunks ? (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) tc::mbar_init(&bars[s], 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  auto size_of = [&](int64_t c) { return (uint32_t)(nbytes - c * ch < ch ? nbytes - c * ch : ch); };
  auto issue = [&](int64_t i) {
    const int s = (int)(i % S);
    const int64_t c = blockIdx.x + i * gridDim.x;
    const uint32_t sz = size_of(c);
    tc::mbar_arrive_expect_tx(&bars[s], sz);
    bulk_g2s(ring + s * CHUNK, src + c * ch, sz, &bars[s]);
  };
  if (threadIdx.x == 0)
    for (int64_t i = 0; i < (mine < S ? mine : S); ++i) issue(i);
  int64_t i = 0;
  for (; i < mine; ++i) {
    const int s = (int)(i % S);
    const bool ok = tc::mbar_wait(&bars[s], (uint32_t)((i / S) & 1));
    if (!ok) abort_flag = 1;
    const int64_t c = blockIdx.x + i * gridDim.x;
    if (ok) body(ring + s * CHUNK, c, (int)size_of(c));
    __syncthreads();
    if (abort_flag) break;
    if (threadIdx.x == 0 && i + S < mine) issue(i + S);
  }
  if (threadIdx.x == 0 && abort_flag) {
    set_dev_error(SP24_ERR_DEVICE_TIMEOUT);
    const int64_t last = i + S < mine ? i + S : mine;
    for (int64_t j = i; j < last; ++j) tc::mbar_wait(&bars[j % S], (uint32_t)((j / S) & 1));
  }
}

// Runs body(stage_ptr, chunk_index, chunk_bytes) over this CTA's chunks of `src` (nbytes, a
// multiple of 16, src 16-byte aligned): chunks c = blockIdx.x, blockIdx.x + gridDim.x, ...
template <int CHUNK, int S, class Body>
__device__ __forceinline__ void for_each_chunk(const uint8_t* __restrict__ src, int64_t nbytes, uint8_t* ring,
                                               Body&& body) {
  for_each_chunk2<CHUNK, S>(src, nbytes, nullptr, 0, ring,
                            [&](const uint8_t* stage, int, int64_t c, int bytes) { body(stage, c, bytes); });
}

}  // namespace stream
}  // namespace sp24
