// pack.cu -- quantise + pack (offline), unpack (test hook) and the rotation's sign vector.
//
// Quantisation rules: pptc.cn ternary-27B article §5.1 (s = mean|w|,
// t = clip(round(w/s), -1, 1)) applied per 128-weight block as in the mhpq.cn
// "27B in 5.9 GB" article §2.1, fp16 scales (§3.2 there); the 1-bit sign rule of
// the neodrop.ai round-up (part 2, Q1_0: weights +1 or -1); 2-bit nearest-level
// codes for the rotated weights of the feinterview.poetries.top "27B in 12 GB"
// article. One thread per block; not tuned (runs once per weight matrix).
#include "lbq_common.cuh"

namespace {

using namespace lbq;

// fp16 scale from an fp64 value: saturate at the largest finite fp16 first, then
// round once to nearest-even.
__device__ __forceinline__ uint16_t scale_to_f16_bits(double m) {
  if (m > 65504.0) m = 65504.0;
  return __half_as_ushort(__double2half(m));
}

// Sum of |w| over a block, in fp64, in increasing k (the order fixes the bits).
template <int kN>
__device__ __forceinline__ double abs_sum(const float* w) {
  double acc = 0.0;
  const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll 4
  for (int i = 0; i < kN / 4; ++i) {
    float4 v = w4[i];
    acc += fabs(static_cast<double>(v.x));
    acc += fabs(static_cast<double>(v.y));
    acc += fabs(static_cast<double>(v.z));
    acc += fabs(static_cast<double>(v.w));
  }
  return acc;
}

// Trit by exact comparison against half the stored scale: |w| > s/2 -> sign(w),
// else 0 (ties go to 0, as round-half-even of w/s does at |w/s| = 1/2).
__device__ __forceinline__ int trit_of(float w, float half_s, bool zero_scale) {
  if (zero_scale) return 0;
  float a = fabsf(w);
  return a > half_s ? (w > 0.0f ? 1 : -1) : 0;
}

// One thread per (row, block) over the rows padded to a multiple of four; padding
// rows are written as zeros. Codes and scales go to their group-of-four places.
__global__ void pack_tern_kernel(const float* __restrict__ W, int64_t K, int64_t N,
                                 uint8_t* __restrict__ codes, int64_t stride) {
  const int64_t nb = K / kTernBlock;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= g4_rows(N) * nb) return;
  const int64_t n = gid / nb, b = gid % nb;
  uint32_t o32[7] = {0, 0, 0, 0, 0, 0, 0};
  if (n < N) {
    const float* w = W + n * K + b * kTernBlock;
    const uint16_t h = scale_to_f16_bits(abs_sum<kTernBlock>(w) / 128.0);
    const float s = f16_bits_to_f32(h);
    const float half_s = 0.5f * s;
    const bool zs = (s == 0.0f);
    uint8_t bytes[kTernBlockBytes];
#pragma unroll
    for (int j = 0; j < kTernCodeBytes; ++j) {
      int v = 0, p = 1;
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int k = 5 * j + i;
        const int d = (k < kTernBlock) ? trit_of(w[k], half_s, zs) + 1 : 1;
        v += d * p;
        p *= 3;
      }
      bytes[j] = static_cast<uint8_t>(v);
    }
    bytes[26] = static_cast<uint8_t>(h & 0xff);
    bytes[27] = static_cast<uint8_t>(h >> 8);
#pragma unroll
    for (int q = 0; q < 7; ++q)
      o32[q] = bytes[4 * q] | (bytes[4 * q + 1] << 8) | (bytes[4 * q + 2] << 16) |
               (static_cast<uint32_t>(bytes[4 * q + 3]) << 24);
  }
  // block b is words 7b .. 7b+6 of the row
#pragma unroll
  for (int q = 0; q < 7; ++q)
    *reinterpret_cast<uint32_t*>(codes + g4_word_byte(n, 7 * b + q, stride)) = o32[q];
  if (b == nb - 1)  // zero the row padding
    for (int64_t q = 7 * nb; q < stride / 4; ++q)
      *reinterpret_cast<uint32_t*>(codes + g4_word_byte(n, q, stride)) = 0u;
}

__global__ void pack_sign_kernel(const float* __restrict__ W, int64_t K, int64_t N,
                                 uint8_t* __restrict__ codes, int64_t cstride,
                                 uint16_t* __restrict__ scales, int64_t sstride) {
  const int64_t nb = K / kSignBlock;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= g4_rows(N) * nb) return;
  const int64_t n = gid / nb, b = gid % nb;
  const bool real = n < N;
  const float* w = W + (real ? n : 0) * K + b * kSignBlock;
  scales[g4_scale_elem(n, b, sstride)] = real ? scale_to_f16_bits(abs_sum<kSignBlock>(w) / 128.0) : 0;
  if (b == nb - 1)  // zero the scale-row padding
    for (int64_t p = nb; p < sstride; ++p) scales[g4_scale_elem(n, p, sstride)] = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t word = 0;
    if (real) {
#pragma unroll
      for (int i = 0; i < 32; ++i) word |= (w[32 * q + i] >= 0.0f ? 1u : 0u) << i;
    }
    *reinterpret_cast<uint32_t*>(codes + g4_word_byte(n, 4 * b + q, cstride)) = word;
  }
  if (b == nb - 1)
    for (int64_t q = 4 * nb; q < cstride / 4; ++q)
      *reinterpret_cast<uint32_t*>(codes + g4_word_byte(n, q, cstride)) = 0u;
}

__global__ void pack_q2_kernel(const float* __restrict__ W, int64_t K, int64_t N,
                               uint8_t* __restrict__ codes, int64_t cstride,
                               uint16_t* __restrict__ scales, int64_t sstride) {
  const int64_t nb = K / kQ2Block;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= g4_rows(N) * nb) return;
  const int64_t n = gid / nb, b = gid % nb;
  const bool real = n < N;
  const float* w = W + (real ? n : 0) * K + b * kQ2Block;
  float mx = 0.0f;
  if (real) {
#pragma unroll
    for (int i = 0; i < kQ2Block; ++i) mx = fmaxf(mx, fabsf(w[i]));
  }
  const uint16_t h = real ? scale_to_f16_bits(static_cast<double>(mx) / 1.5) : 0;
  scales[g4_scale_elem(n, b, sstride)] = h;
  if (b == nb - 1)
    for (int64_t p = nb; p < sstride; ++p) scales[g4_scale_elem(n, p, sstride)] = 0;
  const float s = f16_bits_to_f32(h);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint32_t word = 0;
    if (real) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v = w[16 * q + i];
        // nearest of {-1.5,-0.5,0.5,1.5}*s, ties upward: boundaries at -s, 0, s
        uint32_t c = (s == 0.0f) ? 2u : (v < -s ? 0u : (v < 0.0f ? 1u : (v < s ? 2u : 3u)));
        word |= c << (2 * i);
      }
    }
    *reinterpret_cast<uint32_t*>(codes + g4_word_byte(n, 2 * b + q, cstride)) = word;
  }
  if (b == nb - 1)
    for (int64_t q = 2 * nb; q < cstride / 4; ++q)
      *reinterpret_cast<uint32_t*>(codes + g4_word_byte(n, q, cstride)) = 0u;
}

__global__ void unpack_kernel(int32_t fmt, const uint8_t* __restrict__ codes, int64_t cstride,
                              const uint16_t* __restrict__ scales, int64_t sstride, int64_t K,
                              int64_t N, int64_t blk, int8_t* __restrict__ out,
                              float* __restrict__ sout) {
  const int64_t nb = K / blk;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= N * nb) return;
  const int64_t n = gid / nb, b = gid % nb;
  int8_t* o = out + n * K + b * blk;
  // byte j of row n (group-of-four order)
  auto byte_at = [&](int64_t j) -> unsigned {
    return codes[g4_word_byte(n, j >> 2, cstride) + (j & 3)];
  };
  float s;
  if (fmt == LBQ_TERN5) {
    const int64_t p = b * kTernBlockBytes;
    s = f16_bits_to_f32(static_cast<uint16_t>(byte_at(p + 26) | (byte_at(p + 27) << 8)));
    for (int j = 0; j < kTernCodeBytes; ++j) {
      unsigned v = byte_at(p + j);
      for (int i = 0; i < 5 && 5 * j + i < kTernBlock; ++i) {
        o[5 * j + i] = static_cast<int8_t>(static_cast<int>(v % 3u) - 1);
        v /= 3u;
      }
    }
  } else if (fmt == LBQ_SIGN1) {
    s = f16_bits_to_f32(scales[g4_scale_elem(n, b, sstride)]);
    for (int i = 0; i < kSignBlock; ++i) {
      const int64_t k = b * kSignBlock + i;
      o[i] = ((byte_at(k >> 3) >> (k & 7)) & 1) ? 1 : -1;
    }
  } else {
    s = f16_bits_to_f32(scales[g4_scale_elem(n, b, sstride)]);
    for (int i = 0; i < kQ2Block; ++i) {
      const int64_t k = b * kQ2Block + i;
      o[i] = static_cast<int8_t>((byte_at(k >> 2) >> (2 * (k & 3))) & 3);
    }
  }
  if (sout) sout[n * nb + b] = s;
}

// SplitMix64 in its counter form: output i (1-based) is the finaliser applied to
// seed + i * 0x9e3779b97f4a7c15 (Steele, Lea & Flood 2014).
__global__ void rht_signs_kernel(uint64_t seed, int64_t K, int8_t* __restrict__ D) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  uint64_t z = seed + static_cast<uint64_t>(k + 1) * 0x9e3779b97f4a7c15ULL;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  z ^= z >> 31;
  D[k] = (z >> 63) ? -1 : 1;
}

inline unsigned grid_for(int64_t n, int threads) {
  return static_cast<unsigned>((n + threads - 1) / threads);
}

}  // namespace

cudaError_t lbq_launch_pack(int32_t fmt, const float* W, int64_t K, int64_t N, uint8_t* codes,
                            uint16_t* scales, const lbq::Layout& L, cudaStream_t s) {
  const int T = 128;
  const int64_t units = g4_rows(N) * (K / L.block);
  switch (fmt) {
    case LBQ_TERN5:
      pack_tern_kernel<<<grid_for(units, T), T, 0, s>>>(W, K, N, codes, L.code_stride);
      break;
    case LBQ_SIGN1:
      pack_sign_kernel<<<grid_for(units, T), T, 0, s>>>(W, K, N, codes, L.code_stride, scales,
                                                         L.scale_stride);
      break;
    default:
      pack_q2_kernel<<<grid_for(units, T), T, 0, s>>>(W, K, N, codes, L.code_stride, scales,
                                                       L.scale_stride);
      break;
  }
  return cudaGetLastError();
}

cudaError_t lbq_launch_unpack(const lbq_weights* w, const lbq::Layout& L, int8_t* out,
                              float* scales_out, cudaStream_t s) {
  const int T = 128;
  const int64_t units = w->N * (w->K / L.block);
  unpack_kernel<<<grid_for(units, T), T, 0, s>>>(
      w->fmt, static_cast<const uint8_t*>(w->codes), w->code_stride,
      static_cast<const uint16_t*>(w->scales), w->scale_stride, w->K, w->N, L.block, out,
      scales_out);
  return cudaGetLastError();
}

cudaError_t lbq_launch_rht_signs(uint64_t seed, int64_t K, int8_t* D, cudaStream_t s) {
  const int T = 256;
  rht_signs_kernel<<<grid_for(K, T), T, 0, s>>>(seed, K, D);
  return cudaGetLastError();
}
