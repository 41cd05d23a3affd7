// Read-only bandwidth probe.
//
// Decode attention is a read stream: every step reads the K/V rows of each
// head's window once and writes almost nothing.  The library's own roofline
// for it is therefore a plain read of a large buffer with the same access
// pattern as the decode kernel (16-byte loads, every SM busy), reduced to a
// checksum so the loads cannot be dropped.
#include "internal.h"

namespace moa {
namespace {

constexpr int kReadThreads = 512;
constexpr int kReadUnroll = 4;

__global__ void __launch_bounds__(kReadThreads) stream_read_kernel(const uint4* __restrict__ src, size_t n16,
                                                                   unsigned long long* out) {
  const size_t stride = (size_t)gridDim.x * kReadThreads;
  size_t i = (size_t)blockIdx.x * kReadThreads + threadIdx.x;
  uint32_t a = 0, b = 0, c = 0, d = 0;
  // kReadUnroll independent 16-byte loads in flight per thread
  for (; i + (kReadUnroll - 1) * stride < n16; i += kReadUnroll * stride) {
    uint4 v[kReadUnroll];
#pragma unroll
    for (int u = 0; u < kReadUnroll; ++u) v[u] = __ldg(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < kReadUnroll; ++u) { a ^= v[u].x; b ^= v[u].y; c ^= v[u].z; d ^= v[u].w; }
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldg(src + i);
    a ^= v.x; b ^= v.y; c ^= v.z; d ^= v.w;
  }
  unsigned long long x = ((unsigned long long)(a ^ c) << 32) | (unsigned long long)(b ^ d);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x ^= __shfl_xor_sync(0xffffffffu, x, off);
  if ((threadIdx.x & 31) == 0 && x != 0) atomicXor(out, x);
}

}  // namespace

moa_status launch_stream_read(const void* buf, size_t bytes, void* out, cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOA_ERR_CUDA;
  if (cudaMemsetAsync(out, 0, sizeof(unsigned long long), stream) != cudaSuccess) return MOA_ERR_CUDA;
  const size_t n16 = bytes / 16;
  if (n16 > 0) {
    // four 512-thread blocks per SM keep enough loads in flight to cover
    // HBM latency
    stream_read_kernel<<<sms * 4, kReadThreads, 0, stream>>>(static_cast<const uint4*>(buf), n16,
                                                            static_cast<unsigned long long*>(out));
    if (cudaGetLastError() != cudaSuccess) return MOA_ERR_CUDA;
  }
  return MOA_OK;
}

}  // namespace moa
