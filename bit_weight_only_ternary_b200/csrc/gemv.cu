// gemv.cu -- batch-1 low-bit GEMV, y = W_hat x (bf16 in, fp32 accumulate, bf16 out).
//
// Ternary products reduce to adding, subtracting or skipping activations
// (pptc.cn ternary-27B article §1.2; mhpq.cn "27B in 5.9 GB" article §2.2); each
// block's sum is then scaled by its fp16 scale (mhpq.cn §2.1). The 1-bit format
// is the Q1_0 case of the neodrop.ai round-up (part 2); the 2-bit format takes
// the rotated input of the feinterview.poetries.top "27B in 12 GB" article.
//
// This file holds the straightforward kernels: one warp per output row, each lane
// decoding whole blocks in registers.
#include "lbq_common.cuh"

namespace {

using namespace lbq;

__device__ __forceinline__ float x_at(const uint16_t* __restrict__ x, int64_t k) {
  return bf16_bits_to_f32(x[k]);
}

// Ternary: lane handles blocks lane, lane + 32, ...; each block is 7 aligned words.
__global__ void __launch_bounds__(256) gemv_tern_rowwarp(const uint8_t* __restrict__ codes,
                                                         int64_t stride, int64_t K, int64_t N,
                                                         const uint16_t* __restrict__ x,
                                                         uint16_t* __restrict__ y) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (n >= N) return;
  const int lane = threadIdx.x & 31;
  const int64_t nb = K / kTernBlock;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(codes + n * stride);
  float acc = 0.0f;
  for (int64_t b = lane; b < nb; b += 32) {
    uint32_t w[7];
#pragma unroll
    for (int q = 0; q < 7; ++q) w[q] = row[b * 7 + q];
    const float s = f16_bits_to_f32(static_cast<uint16_t>(w[6] >> 16));
    const uint16_t* xb = x + b * kTernBlock;
    float part = 0.0f;
#pragma unroll
    for (int j = 0; j < kTernCodeBytes; ++j) {
      unsigned v = (w[j >> 2] >> (8 * (j & 3))) & 0xffu;
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        if (5 * j + i < kTernBlock) {
          const int t = static_cast<int>(v % 3u) - 1;
          part += static_cast<float>(t) * x_at(xb, 5 * j + i);
        }
        v /= 3u;
      }
    }
    acc += s * part;
  }
  acc = warp_sum(acc);
  if (lane == 0) y[n] = f32_to_bf16_bits(acc);
}

__global__ void __launch_bounds__(256) gemv_sign_rowwarp(const uint8_t* __restrict__ codes,
                                                         int64_t cstride,
                                                         const uint16_t* __restrict__ scales,
                                                         int64_t sstride, int64_t K, int64_t N,
                                                         const uint16_t* __restrict__ x,
                                                         uint16_t* __restrict__ y) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (n >= N) return;
  const int lane = threadIdx.x & 31;
  const int64_t nb = K / kSignBlock;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(codes + n * cstride);
  float acc = 0.0f;
  for (int64_t b = lane; b < nb; b += 32) {
    const float s = f16_bits_to_f32(scales[n * sstride + b]);
    const uint16_t* xb = x + b * kSignBlock;
    float part = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t bits = row[b * 4 + q];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float xv = x_at(xb, 32 * q + i);
        part += ((bits >> i) & 1u) ? xv : -xv;
      }
    }
    acc += s * part;
  }
  acc = warp_sum(acc);
  if (lane == 0) y[n] = f32_to_bf16_bits(acc);
}

// 2-bit: xr is the rotated input in fp32 (computed beforehand into the workspace).
__global__ void __launch_bounds__(256) gemv_q2_rowwarp(const uint8_t* __restrict__ codes,
                                                       int64_t cstride,
                                                       const uint16_t* __restrict__ scales,
                                                       int64_t sstride, int64_t K, int64_t N,
                                                       const float* __restrict__ xr,
                                                       uint16_t* __restrict__ y) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (n >= N) return;
  const int lane = threadIdx.x & 31;
  const int64_t nb = K / kQ2Block;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(codes + n * cstride);
  float acc = 0.0f;
  for (int64_t b = lane; b < nb; b += 32) {
    const float s = f16_bits_to_f32(scales[n * sstride + b]);
    const float* xb = xr + b * kQ2Block;
    float part = 0.0f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t bits = row[b * 2 + q];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float lvl = static_cast<float>((bits >> (2 * i)) & 3u) - 1.5f;
        part += lvl * xb[16 * q + i];
      }
    }
    acc += s * part;
  }
  acc = warp_sum(acc);
  if (lane == 0) y[n] = f32_to_bf16_bits(acc);
}

}  // namespace

size_t lbq_gemv_workspace(const lbq_weights* w) {
  // the 2-bit path keeps the rotated input (fp32, K values) in the workspace
  return w->fmt == LBQ_Q2RHT ? static_cast<size_t>(w->K) * sizeof(float) : 0;
}

cudaError_t lbq_launch_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                            uint16_t* y, void* ws, cudaStream_t s) {
  const int warps = 8;
  const unsigned grid = static_cast<unsigned>((w->N + warps - 1) / warps);
  const uint8_t* codes = static_cast<const uint8_t*>(w->codes);
  const uint16_t* scales = static_cast<const uint16_t*>(w->scales);
  switch (w->fmt) {
    case LBQ_TERN5:
      gemv_tern_rowwarp<<<grid, 32 * warps, 0, s>>>(codes, w->code_stride, w->K, w->N, x, y);
      break;
    case LBQ_SIGN1:
      gemv_sign_rowwarp<<<grid, 32 * warps, 0, s>>>(codes, w->code_stride, scales,
                                                     w->scale_stride, w->K, w->N, x, y);
      break;
    default: {
      float* xr = static_cast<float*>(ws);
      cudaError_t e = lbq_launch_hadamard(x, D, 1, w->K, xr, s);
      if (e != cudaSuccess) return e;
      gemv_q2_rowwarp<<<grid, 32 * warps, 0, s>>>(codes, w->code_stride, scales, w->scale_stride,
                                                   w->K, w->N, xr, y);
      break;
    }
  }
  return cudaGetLastError();
}
