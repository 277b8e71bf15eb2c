// gemm.cu -- batched low-bit product Y[m][n] = sum_k W_hat[n][k] X[m][k].
//
// Same formats and rules as gemv.cu (ternary add/subtract/skip per block,
// pptc.cn §1.2 and mhpq.cn §2.1-2.2; 1-bit Q1_0, neodrop.ai part 2; 2-bit with the
// rotated input, feinterview.poetries.top). The ternary format goes to the tensor-core
// kernel in gemm_tc.cu; this file holds the straightforward kernel the 1-bit and
// 2-bit formats use for now: one warp per (row, group of activation rows), blocks
// decoded in registers.
#include "lbq_common.cuh"

namespace {

using namespace lbq;

template <int FMT>
__device__ __forceinline__ float row_dot(const uint8_t* __restrict__ codes, int64_t cstride,
                                         const uint16_t* __restrict__ scales, int64_t sstride,
                                         int64_t n, int64_t K,
                                         const uint16_t* __restrict__ xb16,
                                         const float* __restrict__ xf32) {
  const int lane = threadIdx.x & 31;
  float acc = 0.0f;
  // word i and scale b of row n in the group-of-four storage order
  auto word = [&](int64_t i) -> uint32_t {
    return *reinterpret_cast<const uint32_t*>(codes + g4_word_byte(n, i, cstride));
  };
  auto scale = [&](int64_t b) -> float { return f16_bits_to_f32(scales[g4_scale_elem(n, b, sstride)]); };
  if (FMT == LBQ_TERN5) {
    for (int64_t b = lane; b < K / kTernBlock; b += 32) {
      uint32_t w[7];
#pragma unroll
      for (int q = 0; q < 7; ++q) w[q] = word(b * 7 + q);
      const float s = f16_bits_to_f32(static_cast<uint16_t>(w[6] >> 16));
      float part = 0.0f;
#pragma unroll
      for (int j = 0; j < kTernCodeBytes; ++j) {
        unsigned v = (w[j >> 2] >> (8 * (j & 3))) & 0xffu;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          if (5 * j + i < kTernBlock)
            part += static_cast<float>(static_cast<int>(v % 3u) - 1) *
                    bf16_bits_to_f32(xb16[b * kTernBlock + 5 * j + i]);
          v /= 3u;
        }
      }
      acc += s * part;
    }
  } else if (FMT == LBQ_SIGN1) {
    for (int64_t b = lane; b < K / kSignBlock; b += 32) {
      float part = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t bits = word(b * 4 + q);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float xv = bf16_bits_to_f32(xb16[b * kSignBlock + 32 * q + i]);
          part += ((bits >> i) & 1u) ? xv : -xv;
        }
      }
      acc += scale(b) * part;
    }
  } else {
    for (int64_t b = lane; b < K / kQ2Block; b += 32) {
      float part = 0.0f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint32_t bits = word(b * 2 + q);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          part += (static_cast<float>((bits >> (2 * i)) & 3u) - 1.5f) *
                  xf32[b * kQ2Block + 16 * q + i];
      }
      acc += scale(b) * part;
    }
  }
  return warp_sum(acc);
}

template <int FMT>
__global__ void __launch_bounds__(256) gemm_rowwarp(const uint8_t* __restrict__ codes,
                                                    int64_t cstride,
                                                    const uint16_t* __restrict__ scales,
                                                    int64_t sstride, int64_t K, int64_t N,
                                                    const uint16_t* __restrict__ X,
                                                    const float* __restrict__ Xr, int64_t M,
                                                    int64_t m_per_cta, uint16_t* __restrict__ Y) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (n >= N) return;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * m_per_cta;
  const int64_t m1 = m0 + m_per_cta < M ? m0 + m_per_cta : M;
  for (int64_t m = m0; m < m1; ++m) {
    const float v = row_dot<FMT>(codes, cstride, scales, sstride, n, K, X + m * K,
                                 Xr ? Xr + m * K : nullptr);
    if ((threadIdx.x & 31) == 0) Y[m * N + n] = f32_to_bf16_bits(v);
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
  const int64_t m_per_cta = 8;
  dim3 grid(static_cast<unsigned>((w->N + warps - 1) / warps),
            static_cast<unsigned>((M + m_per_cta - 1) / m_per_cta));
  const uint8_t* codes = static_cast<const uint8_t*>(w->codes);
  const uint16_t* scales = static_cast<const uint16_t*>(w->scales);
  switch (w->fmt) {
    case LBQ_TERN5:  // tensor-core path (gemm_tc.cu)
      return lbq_launch_gemm_tc(w, X, M, Y, ws, s);
    case LBQ_SIGN1:
      gemm_rowwarp<LBQ_SIGN1><<<grid, 32 * warps, 0, s>>>(
          codes, w->code_stride, scales, w->scale_stride, w->K, w->N, X, nullptr, M, m_per_cta, Y);
      break;
    default: {
      float* xr = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes);
      cudaError_t e = lbq_launch_hadamard(X, D, M, w->K, xr, s);
      if (e != cudaSuccess) return e;
      gemm_rowwarp<LBQ_Q2RHT><<<grid, 32 * warps, 0, s>>>(
          codes, w->code_stride, scales, w->scale_stride, w->K, w->N, X, xr, M, m_per_cta, Y);
      break;
    }
  }
  return cudaGetLastError();
}
