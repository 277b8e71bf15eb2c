// lut.cuh -- the lookup-table arithmetic the batch-1 products share (gemv.cu, gemv_batch.cu).
//
// Ternary products reduce to adding, subtracting or skipping activations (pptc.cn
// ternary-27B article §1.2; mhpq.cn "27B in 5.9 GB" article §2.2), each block's sum
// scaled by its fp16 scale (mhpq.cn §2.1); the 1-bit format is the Q1_0 case of the
// neodrop.ai round-up (part 2); the 2-bit format multiplies the rotated input
// x' = H D x / sqrt(512) of the feinterview.poetries.top "27B in 12 GB" article.
//
// Done a byte at a time: a CTA owns one K-slice (ternary: 4 blocks, 512 weights, 28
// words of a row; 1-bit: 1024 weights, 32 words; 2-bit: 512 weights, 32 words) and
// builds in shared memory, for every byte position of the slice, the partial dot
// product of that byte's codes with the slice of x, for all 256 byte values (128 KB,
// two 64 KB pages). Lane l always handles the same word position of a row, and the
// table is laid out [value][lane], so a warp's lookups never collide on a bank; a
// byte costs one PRMT (which forms the table address from the byte and the lane),
// one LDS and an add.
#pragma once

#include "rht.cuh"

namespace lbq {
namespace lut {

constexpr uint32_t kPage = 65536;  // table page: 256 values x 256 bytes
constexpr uint32_t kTableBytes = 2 * kPage;

template <int FMT>
struct Traits;
// kWeights / kWords / kBlocks: one slice of a row; kDigits: codes per byte;
// kGroupBytes: a group of four rows' codes in one slice; kScaleBytes: its scales
// (1-bit and 2-bit; ternary scales sit among the codes).
template <>
struct Traits<LBQ_TERN5> {
  static constexpr int kWeights = 512, kWords = 28, kBlocks = 4, kDigits = 5, kBlockLanes = 8;
  static constexpr uint32_t kGroupBytes = 16 * kWords, kScaleBytes = 0;
};
template <>
struct Traits<LBQ_SIGN1> {
  static constexpr int kWeights = 1024, kWords = 32, kBlocks = 8, kDigits = 8, kBlockLanes = 4;
  static constexpr uint32_t kGroupBytes = 16 * kWords, kScaleBytes = 8 * kBlocks;
};
template <>
struct Traits<LBQ_Q2RHT> {
  static constexpr int kWeights = 512, kWords = 32, kBlocks = 16, kDigits = 4, kBlockLanes = 2;
  static constexpr uint32_t kGroupBytes = 16 * kWords, kScaleBytes = 8 * kBlocks;
};

// Word of the slice that lane l handles (ternary: block l/8, word l%8 of it; lanes
// 7, 15, 23, 31 have none), or -1; nb = blocks present in this slice.
template <int FMT>
__device__ __forceinline__ int lane_word(int l, int nb) {
  if (FMT == LBQ_TERN5) return ((l & 7) < 7 && (l >> 3) < nb) ? 7 * (l >> 3) + (l & 7) : -1;
  if (FMT == LBQ_SIGN1) return l < 4 * nb ? l : -1;
  return l;
}

// Weight index (within the slice) of digit e of byte `slot` of lane l's word, or -1
// if that digit carries no weight (scale bytes, byte-25 padding digits, no word).
template <int FMT>
__device__ __forceinline__ int digit_weight(int slot, int l, int e, int nb) {
  const int w = lane_word<FMT>(l, nb);
  if (w < 0) return -1;
  if (FMT == LBQ_TERN5) {
    // lane l holds word l % 8 of block l / 8 (lane_word), so no division is needed
    const int bb = l >> 3, c = 4 * (l & 7) + slot;  // byte within the 28-byte block
    if (c >= kTernCodeBytes) return -1;              // the block's fp16 scale
    const int kb = 5 * c + e;
    return kb < kTernBlock ? bb * kTernBlock + kb : -1;
  } else if (FMT == LBQ_SIGN1) {
    return 32 * w + 8 * slot + e;
  } else {
    return 16 * w + 4 * slot + e;
  }
}

__device__ __forceinline__ void sts_f2(uint32_t addr, float2 v) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}
template <uint32_t kImm>
__device__ __forceinline__ float lds_imm(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(kImm));
  return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ float2 h2_to_f2(uint32_t h2) {
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Table entries of one row word: the four bytes' partial sums added up.
// Slot i lives on page i/2 at column offset (i%2)*128; `lanereg` = table base | lane*4.
__device__ __forceinline__ float2 lookup_pair(uint32_t w0, uint32_t w1, uint32_t lanereg) {
  const float2 e0 = make_float2(lds_imm<0>(__byte_perm(w0, lanereg, 0x7604)),
                                lds_imm<0>(__byte_perm(w1, lanereg, 0x7604)));
  const float2 e1 = make_float2(lds_imm<128>(__byte_perm(w0, lanereg, 0x7614)),
                                lds_imm<128>(__byte_perm(w1, lanereg, 0x7614)));
  const float2 e2 = make_float2(lds_imm<kPage>(__byte_perm(w0, lanereg, 0x7624)),
                                lds_imm<kPage>(__byte_perm(w1, lanereg, 0x7624)));
  const float2 e3 = make_float2(lds_imm<kPage + 128>(__byte_perm(w0, lanereg, 0x7634)),
                                lds_imm<kPage + 128>(__byte_perm(w1, lanereg, 0x7634)));
  return __fadd2_rn(__fadd2_rn(e0, e1), __fadd2_rn(e2, e3));
}

// Position of weight k of a slice in the shared-memory x buffer: one pad float after
// every 32 (1-bit, 2-bit) or two after every 128 (ternary). The table builders read x
// 32 (1-bit), 16 (2-bit) or about 128 (ternary) weights apart across a warp's lanes;
// unpadded, those reads fall on one bank (16-way conflicts for the 1-bit and 2-bit
// formats, 4-way for ternary), padded on 16 or 32 different banks.
template <int FMT>
__device__ __forceinline__ int xs_pos(int k) {
  return FMT == LBQ_TERN5 ? k + 2 * (k >> 7) : k + (k >> 5);
}
constexpr uint32_t kXsBytes = 4 * (1024 + 32);  // the largest padded slice (1-bit)

// Eight bf16 activations (weights 8c .. 8c + 7 of the slice) stored as fp32.
template <int FMT>
__device__ __forceinline__ void x_store8(uint4 v, float* xs, int c) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    xs[xs_pos<FMT>(8 * c + 2 * q)] = __uint_as_float(w[q] << 16);
    xs[xs_pos<FMT>(8 * c + 2 * q + 1)] = __uint_as_float(w[q] & 0xffff0000u);
  }
}

// The x slice of slice j, loaded by x_issue with plain loads and stored to shared memory
// as fp32 by x_store (the 2-bit format: rotated by one warp on the way).
struct XLoad {
  uint4 v0, v1, d;
};
template <int FMT>
__device__ __forceinline__ XLoad x_issue(const uint16_t* x, const int8_t* D, int nblk, int32_t j,
                                         int tid) {
  using T = Traits<FMT>;
  XLoad r{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  const int64_t k0 = static_cast<int64_t>(j) * T::kWeights;
  if (FMT == LBQ_Q2RHT) {
    if (tid < 32) {  // one warp: 16 activations and 16 signs per lane
      const uint4* x4 = reinterpret_cast<const uint4*>(x + k0 + 16 * tid);
      r.v0 = x4[0];
      r.v1 = x4[1];
      r.d = *reinterpret_cast<const uint4*>(D + k0 + 16 * tid);
    }
  } else {
    const int blk0 = j * T::kBlocks;
    const int nb = nblk - blk0 < T::kBlocks ? nblk - blk0 : T::kBlocks;
    // one 16-byte load of 8 activations per thread (x and the slices are 16-byte aligned)
    if (tid < T::kWeights / 8 && 8 * tid < nb * kTernBlock)
      r.v0 = __ldg(reinterpret_cast<const uint4*>(x + k0) + tid);
  }
  return r;
}
template <int FMT>
__device__ __forceinline__ void x_store(const XLoad& r, float* xs, int tid) {
  using T = Traits<FMT>;
  if (FMT == LBQ_Q2RHT) {
    if (tid < 32) {
      const uint32_t xw[8] = {r.v0.x, r.v0.y, r.v0.z, r.v0.w, r.v1.x, r.v1.y, r.v1.z, r.v1.w};
      const uint32_t dw[4] = {r.d.x, r.d.y, r.d.z, r.d.w};
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t bits = (i & 1) ? (xw[i >> 1] & 0xffff0000u) : (xw[i >> 1] << 16);
        const int8_t sgn = static_cast<int8_t>((dw[i >> 2] >> (8 * (i & 3))) & 0xff);
        const float xv = __uint_as_float(bits);
        v[i] = sgn < 0 ? -xv : xv;
      }
      fwht512_warp(v);
#pragma unroll
      for (int i = 0; i < 16; ++i) xs[xs_pos<FMT>(16 * tid + i)] = v[i] * kRhtNorm;
    }
  } else if (tid < T::kWeights / 8) {
    x_store8<FMT>(r.v0, xs, tid);
  }
}

// Builds the lookup table for a slice with nb blocks from the x slice in shared memory,
// by kThreadsT threads (a multiple of 64; tid < kThreadsT); the caller synchronises
// them afterwards. Thread t owns table column pair t % 64 (lanes 2c, 2c+1 of one byte
// slot) and the values v = lo + R * hi for hi = t / 64, t / 64 + kThreadsT / 64, ...;
// everything that does not depend on hi is computed once.
template <int FMT, int kThreadsT>
__device__ __forceinline__ void build_table(int nb, uint32_t tbase, const float* xs, int tid) {
  using T = Traits<FMT>;
  const int cp = tid & 63;
  const int slot = cp >> 4, l0 = 2 * (cp & 15);
  float2 xv[T::kDigits];
#pragma unroll
  for (int e = 0; e < T::kDigits; ++e) {
    const int ka = digit_weight<FMT>(slot, l0, e, nb);
    const int kb = digit_weight<FMT>(slot, l0 + 1, e, nb);
    xv[e] = make_float2(ka >= 0 ? xs[xs_pos<FMT>(ka)] : 0.0f, kb >= 0 ? xs[xs_pos<FMT>(kb)] : 0.0f);
  }
  const uint32_t col = tbase + (slot >> 1) * kPage + (slot & 1) * 128 + l0 * 4;
  constexpr int kStep = kThreadsT / 64;
  if (FMT == LBQ_TERN5) {
    // v = d0 + 3 d1 + 9 d2 + 27 (d3 + 3 d4); entry = sum_e (d_e - 1) x_e
    float2 ab[9];
#pragma unroll
    for (int m = 0; m < 9; ++m) {
      const float l0f = static_cast<float>(m % 3 - 1), l1f = static_cast<float>(m / 3 - 1);
      ab[m] = __ffma2_rn(make_float2(l0f, l0f), xv[0], __fmul2_rn(make_float2(l1f, l1f), xv[1]));
    }
    // 27 runs of 9 values (digits 2..4 fixed) per column pair, dealt round-robin
    for (int hd = tid >> 6; hd < 27; hd += kStep) {
      const int hi = hd / 3, d2 = hd - 3 * hi;
      const float l3 = static_cast<float>(hi % 3 - 1), l4 = static_cast<float>(hi / 3 - 1);
      const float2 q = __ffma2_rn(make_float2(l3, l3), xv[3], __fmul2_rn(make_float2(l4, l4), xv[4]));
      const float l = static_cast<float>(d2 - 1);
      const float2 qc = __ffma2_rn(make_float2(l, l), xv[2], q);
      const uint32_t row0 = col + static_cast<uint32_t>(9 * d2 + 27 * hi) * 256u;
#pragma unroll
      for (int m = 0; m < 9; ++m) sts_f2(row0 + m * 256u, __fadd2_rn(qc, ab[m]));
    }
    // byte values 243..255 never occur: zero rows keep them harmless
    for (int i = tid; i < 13 * 64; i += kThreadsT) {
      const int v = 243 + i / 64, c = i % 64;
      sts_f2(tbase + (c >> 5) * kPage + static_cast<uint32_t>(v) * 256u + (c & 31) * 8,
             make_float2(0.0f, 0.0f));
    }
  } else {
    // v = lo + 16 hi; the low two digits come from lo & 3 and lo >> 2
    float2 av[4], bv[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      if (FMT == LBQ_SIGN1) {
        const float s0 = (m & 1) ? 1.0f : -1.0f, s1 = (m & 2) ? 1.0f : -1.0f;
        av[m] = __ffma2_rn(make_float2(s0, s0), xv[0], __fmul2_rn(make_float2(s1, s1), xv[1]));
        bv[m] = __ffma2_rn(make_float2(s0, s0), xv[2], __fmul2_rn(make_float2(s1, s1), xv[3]));
      } else {
        const float l = static_cast<float>(m) - 1.5f;
        av[m] = __fmul2_rn(make_float2(l, l), xv[0]);
        bv[m] = __fmul2_rn(make_float2(l, l), xv[1]);
      }
    }
    for (int hi = tid >> 6; hi < 16; hi += kStep) {
      float2 q;
      if (FMT == LBQ_SIGN1) {
        q = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float l = ((hi >> e) & 1) ? 1.0f : -1.0f;
          q = __ffma2_rn(make_float2(l, l), xv[4 + e], q);
        }
      } else {
        const float l2 = static_cast<float>(hi & 3) - 1.5f, l3 = static_cast<float>(hi >> 2) - 1.5f;
        q = __ffma2_rn(make_float2(l2, l2), xv[2], __fmul2_rn(make_float2(l3, l3), xv[3]));
      }
#pragma unroll
      for (int m1 = 0; m1 < 4; ++m1) {
        const float2 qb = __fadd2_rn(q, bv[m1]);
        const uint32_t row0 = col + static_cast<uint32_t>(4 * m1 + 16 * hi) * 256u;
#pragma unroll
        for (int m0 = 0; m0 < 4; ++m0) sts_f2(row0 + m0 * 256u, __fadd2_rn(qb, av[m0]));
      }
    }
  }
}

// One 16-row unit (four groups of four rows) of one slice, as one lane holds it: its
// word of each group's four rows and the block scales it multiplies after the in-block
// stages of the butterfly (see unit_sum).
struct UnitRegs {
  uint4 w[4];   // the lane's word of each group's four rows
  uint2 s[2];   // scales: ternary s[0] = scale words of rows R, R+1; 1-bit s[0] = group
                // G's four scales of the lane's block; 2-bit s[0], s[1] = groups G, G + 1
};

// One transpose-reduce stage: c values -> c / 2; the lane keeps the upper half of the
// row range if its bit d is set, the lower half otherwise, and adds its partner's.
// (Rows are added two at a time with paired adds where a stage has two or more.)
template <int C>
__device__ __forceinline__ void tr_stage(float (&acc)[16], int lane, int d) {
  const bool up = (lane & d) != 0;
  if (C >= 4) {
#pragma unroll
    for (int r = 0; r < C / 2; r += 2) {
      const float2 lo = make_float2(acc[r], acc[r + 1]), hi = make_float2(acc[r + C / 2], acc[r + C / 2 + 1]);
      const float2 send = up ? lo : hi, keep = up ? hi : lo;
      const float2 recv = make_float2(__shfl_xor_sync(0xffffffffu, send.x, d),
                                      __shfl_xor_sync(0xffffffffu, send.y, d));
      const float2 sum = __fadd2_rn(keep, recv);
      acc[r] = sum.x;
      acc[r + 1] = sum.y;
    }
  } else {
    const float send = up ? acc[0] : acc[1];
    const float keep = up ? acc[1] : acc[0];
    acc[0] = keep + __shfl_xor_sync(0xffffffffu, send, d);
  }
}

// A refill that issues nothing (unit_sum's registers are not reused while it runs).
struct NoRefill {
  __device__ __forceinline__ void group(int, UnitRegs&) const {}
  __device__ __forceinline__ void scales(UnitRegs&) const {}
};

// Lookups, block scales and the reduction of one unit; returns the sum of row
// 8 b0 + 4 b1 + 2 b2 + b3 of the unit in every lane (b_k = bit k of the lane).
// refill.group(q, r) may load the next unit's group q into r.w[q] once its words have
// been looked up, refill.scales(r) its scales once they have been used, so that the
// next unit's loads start as early as the registers allow.
template <int FMT, typename Refill = NoRefill>
__device__ __forceinline__ float unit_sum(UnitRegs& r, uint32_t lanereg, int lane,
                                          const Refill& refill = Refill()) {
  float acc[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 p01 = lookup_pair(r.w[q].x, r.w[q].y, lanereg);
    const float2 p23 = lookup_pair(r.w[q].z, r.w[q].w, lanereg);
    acc[4 * q] = p01.x;
    acc[4 * q + 1] = p01.y;
    acc[4 * q + 2] = p23.x;
    acc[4 * q + 3] = p23.y;
    refill.group(q, r);
  }
  tr_stage<16>(acc, lane, 1);
  if (FMT == LBQ_Q2RHT) {  // 2 lanes a block: rows R .. R + 7 (two groups)
    const float2 s0 = h2_to_f2(r.s[0].x), s1 = h2_to_f2(r.s[0].y);
    const float2 s2 = h2_to_f2(r.s[1].x), s3 = h2_to_f2(r.s[1].y);
    acc[0] *= s0.x; acc[1] *= s0.y; acc[2] *= s1.x; acc[3] *= s1.y;
    acc[4] *= s2.x; acc[5] *= s2.y; acc[6] *= s3.x; acc[7] *= s3.y;
  }
  tr_stage<8>(acc, lane, 2);
  if (FMT == LBQ_SIGN1) {  // 4 lanes a block: rows R .. R + 3 (one group)
    const float2 s0 = h2_to_f2(r.s[0].x), s1 = h2_to_f2(r.s[0].y);
    acc[0] *= s0.x; acc[1] *= s0.y; acc[2] *= s1.x; acc[3] *= s1.y;
  }
  tr_stage<4>(acc, lane, 4);
  if (FMT == LBQ_TERN5) {  // 8 lanes a block (7 with words): rows R, R + 1
    const float2 s = h2_to_f2(__byte_perm(r.s[0].x, r.s[0].y, 0x7632));
    acc[0] *= s.x;
    acc[1] *= s.y;
  }
  refill.scales(r);
  tr_stage<2>(acc, lane, 8);
  return acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 16);
}

}  // namespace lut
}  // namespace lbq
