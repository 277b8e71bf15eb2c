// hadamard.cu -- standalone block random Hadamard transform of bf16 activations.
// One warp per (row, 512-block), butterfly in registers (rht.cuh).
#include "rht.cuh"

namespace {

using namespace lbq;

__global__ void __launch_bounds__(128) hadamard_kernel(const uint16_t* __restrict__ x,
                                                       const int8_t* __restrict__ D, int64_t M,
                                                       int64_t K, float* __restrict__ out) {
  const int64_t nblk = K / kRhtBlock;
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (unit >= M * nblk) return;  // whole warps exit together
  const int64_t m = unit / nblk, c = unit % nblk;
  float v[16];
  rht512_warp_load(x + m * K + c * kRhtBlock, D + c * kRhtBlock, v);
  float4* o4 = reinterpret_cast<float4*>(out + m * K + c * kRhtBlock + 16 * (threadIdx.x & 31));
#pragma unroll
  for (int q = 0; q < 4; ++q) o4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

}  // namespace

cudaError_t lbq_launch_hadamard(const uint16_t* x, const int8_t* D, int64_t M, int64_t K,
                                float* out, cudaStream_t s) {
  const int64_t units = M * (K / kRhtBlock);
  const int warps = 4;
  hadamard_kernel<<<static_cast<unsigned>((units + warps - 1) / warps), 32 * warps, 0, s>>>(
      x, D, M, K, out);
  return cudaGetLastError();
}
