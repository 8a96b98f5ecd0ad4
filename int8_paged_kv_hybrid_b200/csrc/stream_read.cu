// stream_read.cu -- hyb_stream_read's kernel: one coalesced streaming read of
// a buffer, the byte-count-matched floor that a decode launch's bandwidth is
// read against.  Each thread keeps four 16-byte loads in flight (grid-stride),
// XORs the words it read and the warps fold their XOR into one word.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace hyb {

__global__ void __launch_bounds__(kStreamReadThreads)
    stream_read_kernel(const uint4 *__restrict__ src, size_t n, uint32_t *sink) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 v0 = __ldcs(src + i), v1 = __ldcs(src + i + stride);
    const uint4 v2 = __ldcs(src + i + 2 * stride), v3 = __ldcs(src + i + 3 * stride);
    acc ^= v0.x ^ v0.y ^ v0.z ^ v0.w ^ v1.x ^ v1.y ^ v1.z ^ v1.w;
    acc ^= v2.x ^ v2.y ^ v2.z ^ v2.w ^ v3.x ^ v3.y ^ v3.z ^ v3.w;
  }
  for (; i < n; i += stride) {
    const uint4 v = __ldcs(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0 && acc != 0u) atomicXor(sink, acc);
}

cudaError_t launch_stream_read(const void *src, size_t bytes, uint32_t *sink, int grid, cudaStream_t stream) {
  stream_read_kernel<<<grid, kStreamReadThreads, 0, stream>>>(static_cast<const uint4 *>(src), bytes / 16, sink);
  return cudaGetLastError();
}

}  // namespace hyb
