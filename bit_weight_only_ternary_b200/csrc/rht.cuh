// rht.cuh -- 512-point fast Walsh-Hadamard transform held by one warp in registers.
//
// The random Hadamard rotation of the feinterview.poetries.top "27B in 12 GB"
// article (random Hadamard rotation before low-bit coding, QuIP#/QTIP line):
// x' = H_512 D x / sqrt(512), H in Sylvester (natural) order, so
// H[i][j] = (-1)^popcount(i & j). The butterfly computes it in 9 stages: the
// first four within a lane's 16 consecutive values, the last five across lanes.
#pragma once

#include "lbq_common.cuh"

namespace lbq {

// v[i] of lane l is element 16*l + i of the block. Unnormalised (scale after).
__device__ __forceinline__ void fwht512_warp(float (&v)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (!(i & h)) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const bool upper = (lane & d) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, v[i], d);
      v[i] = upper ? (p - v[i]) : (v[i] + p);
    }
  }
}

// Loads 16 bf16 activations x[16l .. 16l+15] of a 512-block and the matching
// signs, applies D, transforms and normalises. x and D 16-byte aligned.
__device__ __forceinline__ void rht512_warp_load(const uint16_t* __restrict__ xb,
                                                 const int8_t* __restrict__ Db, float (&v)[16]) {
  const int lane = threadIdx.x & 31;
  const uint4* x4 = reinterpret_cast<const uint4*>(xb + 16 * lane);
  const uint4 a = x4[0], b = x4[1];
  const uint4 d4 = *reinterpret_cast<const uint4*>(Db + 16 * lane);
  const uint32_t xw[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t bits = (i & 1) ? (xw[i >> 1] & 0xffff0000u) : (xw[i >> 1] << 16);
    const int8_t sgn = static_cast<int8_t>((dw[i >> 2] >> (8 * (i & 3))) & 0xff);
    const float xv = __uint_as_float(bits);
    v[i] = sgn < 0 ? -xv : xv;
  }
  fwht512_warp(v);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] *= kRhtNorm;
}

}  // namespace lbq
