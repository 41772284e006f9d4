// A plain 16-byte-vector copy kernel for parallax_copy: small per-step
// transfers between device memory and mapped page-locked host memory, where a
// DMA copy's fixed latency dominates.
#pragma once

#include <cstdint>

namespace plx {

constexpr int kCopyThreads = 256;

// dst[i] = src[i] for i < n16 (16-byte units), grid-stride; to_host: fence
// the stores at system scope before the kernel ends.
__global__ void __launch_bounds__(kCopyThreads)
    parallax_copy_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src, long long n16,
                         int to_host) {
  for (long long i = (long long)blockIdx.x * kCopyThreads + threadIdx.x; i < n16;
       i += (long long)gridDim.x * kCopyThreads)
    dst[i] = src[i];
  if (to_host) __threadfence_system();
}

}  // namespace plx
