// probe.cu -- lbq_read_probe: a plain streaming read of a device buffer, the measured
// ceiling for the products' weight streams. Every byte is read once with 16-byte
// loads that do not allocate in L1; the loaded words are folded into one XOR so the
// loads cannot be dropped. Grid: four 512-thread CTAs per SM, grid-stride, four loads
// in flight per thread.
#include "lbq_common.cuh"

namespace {

using namespace lbq;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(512) read_probe_kernel(const uint4* __restrict__ p, int64_t n16,
                                                         unsigned* __restrict__ sink) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = ld_stream(p + i), b = ld_stream(p + i + stride), c = ld_stream(p + i + 2 * stride),
                d = ld_stream(p + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n16; i += stride) {
    const uint4 a = ld_stream(p + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0 && acc) atomicXor(sink, acc);
}

}  // namespace

extern "C" lbq_status lbq_read_probe(const void* p, size_t bytes, uint32_t* sink, void* stream) {
  if (!p || !sink) return LBQ_ERR_ARG;
  if (bytes == 0 || bytes % 16) return LBQ_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(p) & 15) || (reinterpret_cast<uintptr_t>(sink) & 3))
    return LBQ_ERR_ALIGN;
  const int64_t n16 = static_cast<int64_t>(bytes / 16);
  int64_t grid = 4 * static_cast<int64_t>(sm_count());
  const int64_t need = (n16 + 511) / 512;
  if (need < grid) grid = need;
  read_probe_kernel<<<static_cast<unsigned>(grid), 512, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(p), n16, sink);
  return lbq_cuda_status(cudaGetLastError());
}
