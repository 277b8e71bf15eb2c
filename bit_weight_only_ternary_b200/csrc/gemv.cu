// gemv.cu -- batch-1 low-bit GEMV, y = W_hat x (bf16 in, fp32 accumulate, bf16 out).
//
// Ternary products reduce to adding, subtracting or skipping activations (pptc.cn
// ternary-27B article §1.2; mhpq.cn "27B in 5.9 GB" article §2.2) and each block's
// sum is scaled by its fp16 scale (mhpq.cn §2.1). The 1-bit format is the Q1_0 case
// of the neodrop.ai round-up (part 2); the 2-bit format multiplies the rotated
// input x' = H D x / sqrt(512) of the feinterview.poetries.top "27B in 12 GB"
// article, computed here in shared memory, never in global memory.
//
// Design (HBM-bound: the decode must cost about one instruction per weight):
//  * Lookup of partial sums. A CTA owns one K-slice at a time (ternary: 4 blocks,
//    512 weights, 28 words of a row; 1-bit: 1024 weights, 32 words; 2-bit: 512
//    weights, 32 words) and builds in shared memory, for every byte position of the
//    slice, the partial dot product of that byte's codes with the slice of x, for
//    all 256 byte values. A byte then costs one PRMT (which forms the table address
//    directly), one LDS and one add. The table is laid out [value][lane], lane l
//    always reads word l of a row, so table reads are bank-conflict free.
//  * Warp specialisation. One producer lane streams 32-row x slice tiles of codes
//    (and, for the 1-bit and 2-bit formats, of scales) with 2D TMA into a ring of
//    shared-memory stages guarded by mbarriers; ragged edges arrive zero-filled.
//    Sixteen consumer warps each take one 32-row unit at a time. At step g lane l
//    works on row g ^ l of the unit (rows visited in Gray-code order, so the row
//    address moves by one signed power of two per step); every read stays
//    conflict-free and a select-free butterfly then leaves row l's sum in lane l.
//  * Split-K. Slices are spread over CTAs; each unit's 32 sums go to the workspace,
//    and a small second kernel (launched with programmatic dependent launch, so it
//    starts while the first is finishing) adds each row's slice sums in slice order
//    and writes bf16 y: results are deterministic. (Folding that sum into the main
//    kernel, with the last of a row group's CTAs doing it, measured slightly slower.)
//    A matrix of one slice writes y directly.
//  * Grid of floor(SMs / slices) CTAs per slice, one CTA per SM, each with an equal
//    share of its slice's 32-row chunks, so that no CTA builds a second table.
//    Programmatic dependent launch:
//    the producer streams weights before the previous kernel in the stream has
//    finished; consumers wait for it before touching x, y or the workspace.
#include <cudaTypedefs.h>

#include "rht.cuh"
#include "sm100_async.cuh"

namespace {

using namespace lbq;

constexpr int kMaxConsumers = 16;               // consumer warps (per format, see Traits)
constexpr int kMaxThreads = 32 * (kMaxConsumers + 1);  // + one producer warp
constexpr int kRows = 32;                       // rows per unit
constexpr int kMaxStages = 32;
constexpr uint32_t kPage = 65536;               // table page: 256 values x 256 bytes
constexpr uint32_t kTailBytes = 4096 + 2 * kMaxStages * 8;  // x slice + mbarriers
// Shared memory layout. The table must start on a 64 KB boundary of the shared
// window (its page addressing keeps the base in the upper half of the PRMT
// operand), and the dynamic allocation does not start on one (the first 1 KB of
// the window is reserved). So the whole opt-in maximum is requested: the table
// sits at the first 64 KB boundary, the stages fill the space below it and
// continue above it, followed by the x slice and the mbarriers. There are more
// stages than consumer warps, so each warp's next unit streams in while it works
// on the current one. The request is sized for a window starting at 0 or 1 KB, and
// leaves room on the SM for a CTA of the small split-K sum kernel.
constexpr uint32_t smem_bytes(uint32_t stage, uint32_t stages) {
  // window starting at 1 KB: stages below the table, the rest above it
  const uint32_t below = (kPage - 1024) / stage < stages ? (kPage - 1024) / stage : stages;
  const uint32_t at_1k = (kPage - 1024) + 2 * kPage + (stages - below) * stage + kTailBytes;
  // window starting at 0: everything above the table
  const uint32_t at_0 = 2 * kPage + stages * stage + kTailBytes;
  return at_1k > at_0 ? at_1k : at_0;
}
constexpr unsigned kFaultProducer = 1, kFaultConsumer = 2, kFaultLayout = 3;

template <int FMT>
struct Traits;
template <>
struct Traits<LBQ_TERN5> {
  static constexpr int kWeights = 512, kBlocks = 4, kPitch = 112;
  static constexpr int kHi = 9;                 // value = lo + 27 * hi
  static constexpr int kScaleBox = 0;           // scales live in the blocks
  static constexpr uint32_t kStageCodes = 3584, kStageBytes = 3584;  // 32 x 112 bytes
  static constexpr int kStages = 26;
  static constexpr int kConsumers = 16;
  static constexpr uint32_t kSmem = smem_bytes(kStageBytes, kStages);
};
template <>
struct Traits<LBQ_SIGN1> {
  static constexpr int kWeights = 1024, kBlocks = 8, kPitch = 128;
  static constexpr int kHi = 16;                // value = lo + 16 * hi
  static constexpr int kScaleBox = 8;           // fp16 scales per row per slice
  static constexpr uint32_t kStageCodes = 4096, kStageBytes = 4096 + 512;
  static constexpr int kStages = 20;
  static constexpr int kConsumers = 14;
  static constexpr uint32_t kSmem = smem_bytes(kStageBytes, kStages);
};
template <>
struct Traits<LBQ_Q2RHT> {
  static constexpr int kWeights = 512, kBlocks = 16, kPitch = 128;
  static constexpr int kHi = 16;
  static constexpr int kScaleBox = 16;
  static constexpr uint32_t kStageCodes = 4096, kStageBytes = 4096 + 1024;
  static constexpr int kStages = 18;
  static constexpr int kConsumers = 12;
  static constexpr uint32_t kSmem = smem_bytes(kStageBytes, kStages);
};

template <uint32_t kImm>
__device__ __forceinline__ float lds_imm(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(kImm));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint16_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.b16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_f2(uint32_t addr, float2 v) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}

// Sum of the four table entries addressed by the bytes of w0 (.x) and of w1 (.y),
// two rows at a time so the adds run packed. Slot i lives on page i/2 at column
// offset (i%2)*128; `lanereg` = table base | lane*4.
template <uint32_t kImm, uint32_t kSel>
__device__ __forceinline__ float2 entry2(uint32_t w0, uint32_t w1, uint32_t lanereg) {
  return make_float2(lds_imm<kImm>(__byte_perm(w0, lanereg, kSel)),
                     lds_imm<kImm>(__byte_perm(w1, lanereg, kSel)));
}
__device__ __forceinline__ float2 lookup4x2(uint32_t w0, uint32_t w1, uint32_t lanereg) {
  const float2 e0 = entry2<0, 0x7604>(w0, w1, lanereg);
  const float2 e1 = entry2<128, 0x7614>(w0, w1, lanereg);
  const float2 e2 = entry2<kPage, 0x7624>(w0, w1, lanereg);
  const float2 e3 = entry2<kPage + 128, 0x7634>(w0, w1, lanereg);
  return __fadd2_rn(__fadd2_rn(e0, e1), __fadd2_rn(e2, e3));
}

// Weight index (within the slice) of digit e of the byte in table column (slot, w),
// or -1 if that digit carries no weight (scale bytes, padding, idle lanes).
template <int FMT>
__device__ __forceinline__ int digit_weight(int slot, int w, int e, int nw) {
  if (w >= nw) return -1;
  if (FMT == LBQ_TERN5) {
    const int bb = w / 7, c = 4 * (w % 7) + slot;  // byte within the 28-byte block
    if (c >= kTernCodeBytes) return -1;            // the block's fp16 scale
    const int kb = 5 * c + e;
    return kb < kTernBlock ? bb * kTernBlock + kb : -1;
  } else if (FMT == LBQ_SIGN1) {
    return 32 * w + 8 * slot + e;
  } else {
    return 16 * w + 4 * slot + e;
  }
}

// Address change when bit b of (g ^ lane) is set, for a row pitch p: +-p * 2^b.
// Five named values (not an array) so that unrolled code keeps them in registers.
struct Steps {
  int32_t d0, d1, d2, d3, d4;
  __device__ __forceinline__ Steps(int lane, int p)
      : d0((lane & 1) ? -p : p),
        d1((lane & 2) ? -2 * p : 2 * p),
        d2((lane & 4) ? -4 * p : 4 * p),
        d3((lane & 8) ? -8 * p : 8 * p),
        d4((lane & 16) ? -16 * p : 16 * p) {}
  __device__ __forceinline__ int32_t at(int b) const {
    return b == 0 ? d0 : (b == 1 ? d1 : (b == 2 ? d2 : (b == 3 ? d3 : d4)));
  }
};

template <int FMT>
struct Args {
  int64_t K, N;
  const uint16_t* x;
  const int8_t* D;
  uint16_t* y;
  float* part;    // [KS][N] slice sums (KS > 1)
  int KS;         // number of slices
  int G;          // CTAs per slice
  int nblk;       // scale blocks per row
  unsigned* fault;  // set when a bounded wait gives up
};

// Builds the x slice and the lookup tables for slice j (consumer threads only).
// Thread t owns table column pair t % 64 (two adjacent lanes of one byte slot) and
// the values v = lo + R * hi for hi = t / 64, t / 64 + T/64, ...; everything that
// does not depend on hi is computed once.
template <int FMT>
__device__ __forceinline__ void build_slice(const Args<FMT>& a, int32_t j, uint32_t tbase,
                                            float* xs, int ctid) {
  using T = Traits<FMT>;
  constexpr int kCT = 32 * T::kConsumers;
  const int blk0 = j * T::kBlocks;
  const int nb_here = a.nblk - blk0 < T::kBlocks ? a.nblk - blk0 : T::kBlocks;
  const int nw = FMT == LBQ_TERN5 ? 7 * nb_here : (FMT == LBQ_SIGN1 ? 4 * nb_here : 2 * nb_here);
  const int nx = FMT == LBQ_Q2RHT ? nb_here * kQ2Block : nb_here * kTernBlock;
  const int64_t k0 = static_cast<int64_t>(j) * T::kWeights;
  const int lane = ctid & 31;

  if (FMT == LBQ_Q2RHT) {
    if (ctid < 32) {
      float v[16];
      rht512_warp_load(a.x + k0, a.D + k0, v);
      float4* d = reinterpret_cast<float4*>(xs + 16 * lane);
#pragma unroll
      for (int q = 0; q < 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {
    // one 16-byte load of 8 activations per thread (x is 16-byte aligned, slices too)
    for (int i = ctid; i < T::kWeights / 8; i += kCT) {
      float f[8];
      if (8 * i < nx) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.x + k0) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          f[2 * q] = __uint_as_float(w[q] << 16);
          f[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] = 0.0f;
      }
      float4* d = reinterpret_cast<float4*>(xs + 8 * i);
      d[0] = make_float4(f[0], f[1], f[2], f[3]);
      d[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
  named_bar_sync(1, kCT);

  const int cp = ctid & 63;
  const int slot = cp >> 4, w0 = 2 * (cp & 15);
  constexpr int kDigits = FMT == LBQ_TERN5 ? 5 : (FMT == LBQ_SIGN1 ? 8 : 4);
  float2 xv[kDigits];
#pragma unroll
  for (int e = 0; e < kDigits; ++e) {
    const int ka = digit_weight<FMT>(slot, w0, e, nw);
    const int kb = digit_weight<FMT>(slot, w0 + 1, e, nw);
    xv[e] = make_float2(ka >= 0 ? xs[ka] : 0.0f, kb >= 0 ? xs[kb] : 0.0f);
  }
  const uint32_t col = tbase + (slot >> 1) * kPage + (slot & 1) * 128 + w0 * 4;
  if (FMT == LBQ_TERN5) {
    // v = d0 + 3 d1 + 9 d2 + 27 (d3 + 3 d4); entry = sum_e (d_e - 1) x_e
    float2 ab[9];
#pragma unroll
    for (int m = 0; m < 9; ++m) {
      const float l0 = static_cast<float>(m % 3 - 1), l1 = static_cast<float>(m / 3 - 1);
      ab[m] = __ffma2_rn(make_float2(l0, l0), xv[0], __fmul2_rn(make_float2(l1, l1), xv[1]));
    }
    for (int hi = ctid >> 6; hi < T::kHi; hi += kCT / 64) {
      const float l3 = static_cast<float>(hi % 3 - 1), l4 = static_cast<float>(hi / 3 - 1);
      const float2 q = __ffma2_rn(make_float2(l3, l3), xv[3], __fmul2_rn(make_float2(l4, l4), xv[4]));
#pragma unroll
      for (int d2 = 0; d2 < 3; ++d2) {
        const float l = static_cast<float>(d2 - 1);
        const float2 qc = __ffma2_rn(make_float2(l, l), xv[2], q);
        const uint32_t row0 = col + static_cast<uint32_t>(9 * d2 + 27 * hi) * 256u;
#pragma unroll
        for (int m = 0; m < 9; ++m) sts_f2(row0 + m * 256u, __fadd2_rn(qc, ab[m]));
      }
    }
    // byte values 243..255 never occur: zero rows keep them harmless
    for (int i = ctid; i < 13 * 64; i += kCT) {
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
        const float l0 = (m & 1) ? 1.0f : -1.0f, l1 = (m & 2) ? 1.0f : -1.0f;
        av[m] = __ffma2_rn(make_float2(l0, l0), xv[0], __fmul2_rn(make_float2(l1, l1), xv[1]));
        bv[m] = __ffma2_rn(make_float2(l0, l0), xv[2], __fmul2_rn(make_float2(l1, l1), xv[3]));
      } else {
        const float l = static_cast<float>(m) - 1.5f;
        av[m] = __fmul2_rn(make_float2(l, l), xv[0]);
        bv[m] = __fmul2_rn(make_float2(l, l), xv[1]);
      }
    }
    for (int hi = ctid >> 6; hi < T::kHi; hi += kCT / 64) {
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
  named_bar_sync(1, kCT);
}

template <int FMT>
__global__ void __launch_bounds__(kMaxThreads, 1)
    gemv_lut_kernel(const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_scales, const Args<FMT> a) {
  using T = Traits<FMT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();

  constexpr int kStages = T::kStages;
  constexpr uint32_t kStageBytes = T::kStageBytes, kStageCodes = T::kStageCodes;
  constexpr int kConsumers = T::kConsumers;
  static_assert(kStages <= kMaxStages && kStages > kConsumers && kConsumers <= kMaxConsumers,
                "stage ring");
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  const uint32_t n_low = (tbase - sbase) / kStageBytes < kStages ? (tbase - sbase) / kStageBytes
                                                                 : kStages;
  const uint32_t high = tbase + 2 * kPage;  // first byte above the table
  const uint32_t tail = high + (kStages - n_low) * kStageBytes;
  if (tail + kTailBytes > sbase + T::kSmem) {  // cannot happen with a 0 or 1 KB reserved prefix
    if (tid == 0) atomicExch(a.fault, kFaultLayout);
    return;
  }
  auto stage_addr = [&](int s) -> uint32_t {
    return static_cast<uint32_t>(s) < n_low ? sbase + s * kStageBytes
                                            : high + (s - n_low) * kStageBytes;
  };
  float* xs = reinterpret_cast<float*>(smem + (tail - sbase));
  const uint32_t full0 = tail + 4096, empty0 = full0 + kStages * 8;

  // This CTA: slice j, 32-row chunks [c_lo, c_hi) of it (a.G CTAs share a slice).
  const int32_t NC = static_cast<int32_t>((a.N + kRows - 1) / kRows);
  const int32_t j = static_cast<int32_t>(blockIdx.x) / a.G;
  const int32_t gs = static_cast<int32_t>(blockIdx.x) - j * a.G;
  // (32-bit arithmetic: NC <= 16384 and G <= the SM count, so gs * NC fits; a 64-bit
  // division here costs the kernel most of a microsecond)
  const int32_t c_lo = static_cast<int32_t>(static_cast<uint32_t>(gs * NC) / static_cast<uint32_t>(a.G));
  const int32_t c_hi =
      static_cast<int32_t>(static_cast<uint32_t>((gs + 1) * NC) / static_cast<uint32_t>(a.G));
  const int32_t n_units = c_hi - c_lo;

  if (tid < kStages) {  // one barrier pair per thread; each initialiser fences its own inits
    mbar_init(full0 + 8 * tid, 1);
    mbar_init(empty0 + 8 * tid, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ---------------- producer: one lane streams tiles of codes (and scales)
    if (lane == 0) {
      prefetch_tmap(&tm_codes);
      if (T::kScaleBox) prefetch_tmap(&tm_scales);
      const uint32_t bytes = T::kPitch * kRows + T::kScaleBox * 2 * kRows;
      int32_t issued = 0;
      int s = 0;
      uint32_t phase = 0;
      for (int32_t c = c_lo; c < c_hi; ++c) {
        if (!mbar_wait(empty0 + 8 * s, phase ^ 1, a.fault, kFaultProducer)) break;
        ++issued;
        mbar_arrive_expect_tx(full0 + 8 * s, bytes);
        const uint32_t dst = stage_addr(s);
        tma_load_2d(dst, &tm_codes, j * T::kPitch, c * kRows, full0 + 8 * s);
        if (T::kScaleBox)
          tma_load_2d(dst + kStageCodes, &tm_scales, j * T::kScaleBox, c * kRows, full0 + 8 * s);
        if (++s == kStages) {
          s = 0;
          phase ^= 1;
        }
      }
      // Before this lane exits, every copy it issued must have landed (normally the
      // consumers have already seen them all; this matters only after a fault).
      for (int s2 = 0; s2 < kStages && s2 < issued; ++s2) {
        const int32_t k_last = s2 + (issued - 1 - s2) / kStages * kStages;
        mbar_wait(full0 + 8 * s2, static_cast<uint32_t>(k_last / kStages) & 1, a.fault,
                  kFaultProducer, /*give_up_after_fault=*/false);
      }
    }
    return;
  }

  // ---------------- consumers
  pdl_wait();  // x, y and the workspace may belong to the previous kernel until here
  const uint32_t lanereg = tbase | static_cast<uint32_t>(lane * 4);
  // per-lane address steps: moving row (g ^ lane) by bit b changes the address by +-pitch*2^b
  constexpr int kSPitch = T::kScaleBox ? 2 * T::kScaleBox : T::kPitch;
  const Steps dw(lane, T::kPitch), ds(lane, kSPitch);
  const uint32_t w_off = static_cast<uint32_t>(T::kPitch * lane + 4 * lane);
  const uint32_t s_off =
      // (ternary lanes 28..31 hold no words; they read block 3's scale, which is finite
      // or zero-filled, so that 0 * scale stays 0)
      FMT == LBQ_TERN5 ? static_cast<uint32_t>(T::kPitch * lane + 28 * (lane / 7 < 3 ? lane / 7 : 3) + 26)
                       : static_cast<uint32_t>(kStageCodes + kSPitch * lane +
                                               2 * (lane / (FMT == LBQ_SIGN1 ? 4 : 2)));
  build_slice<FMT>(a, j, tbase, xs, tid);

  bool ok = true;
  // this warp's units: k = warp, warp + kConsumers, ... (stage k % kStages)
  for (int32_t k = warp; k < n_units; k += kConsumers) {
    const int s = k % kStages;
    const uint32_t use = static_cast<uint32_t>(k / kStages);
    const uint32_t stage = stage_addr(s);
    float acc[kRows];
    if (ok) ok = mbar_wait(full0 + 8 * s, use & 1, a.fault, kFaultConsumer);
    if (ok) {
      uint32_t wa = stage + w_off, sa = stage + s_off;
      // Gray-code walk over g; row (g ^ lane); two rows per step pair
#pragma unroll
      for (int t = 0; t < kRows; t += 2) {
        const int g0 = t ^ (t >> 1), g1 = (t + 1) ^ ((t + 1) >> 1);
        const uint32_t wd0 = lds_u32(wa), sc0 = lds_u16(sa);
        // step t -> t+1 flips bit 0 of g
        const int sg0 = (g0 & 1) ? -1 : 1;
        const uint32_t wa1 = wa + sg0 * dw.at(0), sa1 = sa + sg0 * ds.at(0);
        const uint32_t wd1 = lds_u32(wa1), sc1 = lds_u16(sa1);
        const float2 p = lookup4x2(wd0, wd1, lanereg);
        const float2 sc = make_float2(f16_bits_to_f32(sc0), f16_bits_to_f32(sc1));
        const float2 r = __fmul2_rn(p, sc);
        acc[g0] = r.x;
        acc[g1] = r.y;
        if (t + 2 < kRows) {  // step t+1 -> t+2 flips bit ctz(t+2) of g
          const int b = __ffs(t + 2) - 1;
          const int sg = ((g1 >> b) & 1) ? -1 : 1;
          wa = wa1 + sg * dw.at(b);
          sa = sa1 + sg * ds.at(b);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
    } else {
#pragma unroll
      for (int i = 0; i < kRows; ++i) acc[i] = 0.0f;
    }
    // butterfly: acc[i] holds row (i ^ lane); after it, acc[0] is row `lane`
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
      for (int i = 0; i < o; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i + o], o);
    }
    if (!ok) continue;
    const int64_t r = static_cast<int64_t>(c_lo + k) * kRows + lane;
    if (r < a.N) {
      if (a.KS == 1)
        a.y[r] = f32_to_bf16_bits(acc[0]);
      else
        a.part[static_cast<int64_t>(j) * a.N + r] = acc[0];
    }
  }
}

// Sums the slice sums of every row in slice order and writes bf16 y. Launched right
// after the main kernel with programmatic dependent launch: it may start while that
// kernel is finishing and waits for its results before reading them.
__global__ void __launch_bounds__(256) splitk_sum_kernel(const float* __restrict__ part, int KS,
                                                         int64_t N, uint16_t* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= N) return;
  const float* pr = part + r;
  float sum = 0.0f;
  // all of a row's loads are issued before the sum (16 slices per round); the
  // additions then run in slice order
  for (int j = 0; j < KS; j += 16) {
    float v[16];
#pragma unroll
    for (int q = 0; q < 16; ++q)
      v[q] = j + q < KS ? __ldcg(pr + static_cast<int64_t>(j + q) * N) : 0.0f;
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (j + q < KS) sum += v[q];
  }
  y[r] = f32_to_bf16_bits(sum);
}

// The device word the kernels' bounded waits report to (one per device).
__device__ unsigned int g_fault_word = 0;

int slices_of(const lbq_weights* w) {
  const int64_t per = w->fmt == LBQ_SIGN1 ? 1024 : 512;
  return static_cast<int>((w->K + per - 1) / per);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D map over [rows][inner] elements with a row pitch in bytes; box = (box_inner, 32).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
              uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, static_cast<cuuint32_t>(kRows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT>
cudaError_t launch(const lbq_weights* w, const uint16_t* x, const int8_t* D, uint16_t* y, void* ws,
                   cudaStream_t s) {
  using T = Traits<FMT>;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_lut_kernel<FMT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(T::kSmem));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  Args<FMT> a;
  a.K = w->K;
  a.N = w->N;
  a.x = x;
  a.D = D;
  a.y = y;
  a.KS = slices_of(w);
  a.nblk = static_cast<int>(w->K / (FMT == LBQ_Q2RHT ? kQ2Block : kTernBlock));
  a.fault = lbq_fault_word();
  if (!a.fault) return cudaErrorInvalidDevicePointer;
  a.part = ws ? reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes) : nullptr;

  CUtensorMap tc, ts;
  const uint64_t row_bytes = FMT == LBQ_TERN5 ? static_cast<uint64_t>(a.nblk) * kTernBlockBytes
                                              : (FMT == LBQ_SIGN1 ? w->K / 8 : w->K / 4);
  if (!make_map(&tc, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, row_bytes,
                static_cast<uint64_t>(w->N), static_cast<uint64_t>(w->code_stride), T::kPitch))
    return cudaErrorInvalidValue;
  if (T::kScaleBox) {
    if (!make_map(&ts, w->scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, static_cast<uint64_t>(a.nblk),
                  static_cast<uint64_t>(w->N), static_cast<uint64_t>(w->scale_stride) * 2,
                  T::kScaleBox))
      return cudaErrorInvalidValue;
  } else {
    ts = tc;  // unused
  }
  const int64_t NC = (w->N + kRows - 1) / kRows;
  // Each CTA works on one slice only (one table build): floor(SMs / KS) CTAs per slice.
  const int64_t per = sm_count() / a.KS > 1 ? sm_count() / a.KS : 1;
  a.G = static_cast<int>(per < NC ? per : NC);
  const int64_t grid = static_cast<int64_t>(a.KS) * a.G;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(32 * (T::kConsumers + 1));
  cfg.dynamicSmemBytes = T::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_lut_kernel<FMT>, tc, ts, a);
  if (e != cudaSuccess || a.KS == 1) return e;
  cudaLaunchConfig_t cfg2 = cfg;
  cfg2.gridDim = dim3(static_cast<unsigned>((w->N + 255) / 256));
  cfg2.blockDim = dim3(256);
  cfg2.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg2, splitk_sum_kernel, static_cast<const float*>(a.part), a.KS,
                            static_cast<int64_t>(w->N), y);
}

}  // namespace

unsigned* lbq_fault_word() {
  static unsigned* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fault_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned*>(p);
  }
  return addr[dev];
}

size_t lbq_gemv_workspace(const lbq_weights* w) {
  const int KS = slices_of(w);
  if (KS <= 1) return 0;
  return kWsCounterBytes + static_cast<size_t>(KS) * static_cast<size_t>(w->N) * sizeof(float);
}

cudaError_t lbq_launch_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                            uint16_t* y, void* ws, cudaStream_t s) {
  switch (w->fmt) {
    case LBQ_TERN5: return launch<LBQ_TERN5>(w, x, D, y, ws, s);
    case LBQ_SIGN1: return launch<LBQ_SIGN1>(w, x, D, y, ws, s);
    default: return launch<LBQ_Q2RHT>(w, x, D, y, ws, s);
  }
}
