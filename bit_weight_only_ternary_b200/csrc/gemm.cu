// gemm.cu -- batched low-bit product Y[m][n] = sum_k W_hat[n][k] X[m][k].
//
// Same formats and rules as gemv.cu (1-bit Q1_0, neodrop.ai part 2; 2-bit with the
// rotated input, feinterview.poetries.top). The ternary format goes to the
// tensor-core kernel in gemm_tc.cu; this file holds the CUDA-core kernel the 1-bit
// and 2-bit formats use: one warp per (weight row, group of up to eight activation
// rows), each block's packed words read once and decoded in registers.
#include "lbq_common.cuh"

namespace {

using namespace lbq;

// One warp per weight row n and group of at most kRowsPerWarp activation rows: lane l
// takes the row's scale blocks l, l + 32, ..., reads each block's packed words once
// and applies them to every activation row of the group, accumulating in fp32; the
// lanes' sums are then added across the warp.
constexpr int kRowsPerWarp = 8;

template <int FMT>
__global__ void __launch_bounds__(256) gemm_rowwarp(const uint8_t* __restrict__ codes,
                                                    int64_t cstride,
                                                    const uint16_t* __restrict__ scales,
                                                    int64_t sstride, int64_t K, int64_t N,
                                                    const uint16_t* __restrict__ X,
                                                    const float* __restrict__ Xr, int64_t M,
                                                    uint16_t* __restrict__ Y) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (n >= N) return;
  const int lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kRowsPerWarp;
  const int nm = static_cast<int>(M - m0 < kRowsPerWarp ? M - m0 : kRowsPerWarp);
  // word i and scale b of row n in the group-of-four storage order
  auto word = [&](int64_t i) -> uint32_t {
    return __ldg(reinterpret_cast<const uint32_t*>(codes + g4_word_byte(n, i, cstride)));
  };
  auto scale = [&](int64_t b) -> float { return f16_bits_to_f32(scales[g4_scale_elem(n, b, sstride)]); };
  float acc[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) acc[r] = 0.0f;
  if (FMT == LBQ_SIGN1) {
    for (int64_t b = lane; b < K / kSignBlock; b += 32) {
      uint32_t bits[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) bits[q] = word(b * 4 + q);
      const float s = scale(b);
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        if (r >= nm) break;
        const uint4* xr = reinterpret_cast<const uint4*>(X + (m0 + r) * K + b * kSignBlock);
        float part = 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {  // eight activations per 16-byte load
          const uint4 v = __ldg(xr + q);
          const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int k = 8 * q + i;
            const float xv = bf16_bits_to_f32(static_cast<uint16_t>(i & 1 ? xw[i >> 1] >> 16 : xw[i >> 1]));
            part += ((bits[k >> 5] >> (k & 31)) & 1u) ? xv : -xv;
          }
        }
        acc[r] += s * part;
      }
    }
  } else {
    for (int64_t b = lane; b < K / kQ2Block; b += 32) {
      const uint32_t w0 = word(b * 2), w1 = word(b * 2 + 1);
      const float s = scale(b);
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        if (r >= nm) break;
        const float4* xr = reinterpret_cast<const float4*>(Xr + (m0 + r) * K + b * kQ2Block);
        float part = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // four rotated activations per 16-byte load
          const float4 v = __ldg(xr + q);
          const float xv[4] = {v.x, v.y, v.z, v.w};
          const uint32_t bits = q < 4 ? w0 : w1;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            part += (static_cast<float>((bits >> (2 * (4 * (q & 3) + i))) & 3u) - 1.5f) * xv[i];
        }
        acc[r] += s * part;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    if (r >= nm) break;
    const float v = warp_sum(acc[r]);
    if (lane == 0) Y[(m0 + r) * N + n] = f32_to_bf16_bits(v);
  }
}

}  // namespace

size_t lbq_gemm_workspace(const lbq_weights* w, int64_t M) {
  if (w->fmt == LBQ_TERN5) return lbq_gemm_tc_workspace(w, M);
  return w->fmt == LBQ_Q2RHT
             ? kWsCounterBytes + static_cast<size_t>(w->K) * static_cast<size_t>(M) * sizeof(float)
             : 0;
}

cudaError_t lbq_launch_gemm(const lbq_weights* w, const uint16_t* X, int64_t M, const int8_t* D,
                            uint16_t* Y, void* ws, cudaStream_t s) {
  const int warps = 8;
  dim3 grid(static_cast<unsigned>((w->N + warps - 1) / warps),
            static_cast<unsigned>((M + kRowsPerWarp - 1) / kRowsPerWarp));
  const uint8_t* codes = static_cast<const uint8_t*>(w->codes);
  const uint16_t* scales = static_cast<const uint16_t*>(w->scales);
  switch (w->fmt) {
    case LBQ_TERN5:  // tensor-core path (gemm_tc.cu)
      return lbq_launch_gemm_tc(w, X, M, Y, ws, s);
    case LBQ_SIGN1:
      gemm_rowwarp<LBQ_SIGN1><<<grid, 32 * warps, 0, s>>>(
          codes, w->code_stride, scales, w->scale_stride, w->K, w->N, X, nullptr, M, Y);
      break;
    default: {
      float* xr = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes);
      cudaError_t e = lbq_launch_hadamard(X, D, M, w->K, xr, s);
      if (e != cudaSuccess) return e;
      gemm_rowwarp<LBQ_Q2RHT><<<grid, 32 * warps, 0, s>>>(
          codes, w->code_stride, scales, w->scale_stride, w->K, w->N, X, xr, M, Y);
      break;
    }
  }
  return cudaGetLastError();
}
