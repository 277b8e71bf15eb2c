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
//  * Split-K. Slices are spread over CTAs; each unit's 32 sums go to the workspace
//    and the last warp to finish a 32-row chunk (a counter per chunk in the fixed
//    counter region) adds the slices in a fixed order and writes bf16 y: results
//    are deterministic, and that warp resets the counter.
//  * Persistent grid, one 544-thread CTA per SM with an equal share of the
//    (slice, chunk) units in slice-major order. Programmatic dependent launch:
//    the producer streams weights before the previous kernel in the stream has
//    finished; consumers wait for it before touching x, y or the workspace.
#include <cudaTypedefs.h>

#include "rht.cuh"
#include "sm100_async.cuh"

namespace {

using namespace lbq;

constexpr int kConsumers = 16;                  // consumer warps
constexpr int kThreads = 32 * (kConsumers + 1); // + one producer warp
constexpr int kRows = 32;                       // rows per unit
constexpr int kStages = 16;                     // units in flight per CTA
constexpr uint32_t kPage = 65536;               // table page: 256 values x 256 bytes
constexpr uint32_t kStageCodes = 4096;          // 32 rows x 128 bytes (ternary uses 112)
constexpr uint32_t kStageBytes = kStageCodes + 1024;  // + 32 rows x 32 bytes of scales
constexpr uint32_t kTailBytes = 4096 + 2 * kStages * 8;  // x slice + mbarriers
// Shared memory layout. The table must start on a 64 KB boundary of the shared
// window (its page addressing keeps the base in the upper half of the PRMT
// operand), and the dynamic allocation does not start on one (the first 1 KB of
// the window is reserved). So the whole opt-in maximum is requested: the table
// sits at the first 64 KB boundary, the stages fill the space below it and
// continue above it, followed by the x slice and the mbarriers.
constexpr size_t kSmem = 232448;
constexpr unsigned kFaultProducer = 1, kFaultConsumer = 2, kFaultLayout = 3;

template <int FMT>
struct Traits;
template <>
struct Traits<LBQ_TERN5> {
  static constexpr int kWeights = 512, kBlocks = 4, kPitch = 112;
  static constexpr int kHi = 9;                 // value = lo + 27 * hi
  static constexpr int kScaleBox = 0;           // scales live in the blocks
};
template <>
struct Traits<LBQ_SIGN1> {
  static constexpr int kWeights = 1024, kBlocks = 8, kPitch = 128;
  static constexpr int kHi = 16;                // value = lo + 16 * hi
  static constexpr int kScaleBox = 8;           // fp16 scales per row per slice
};
template <>
struct Traits<LBQ_Q2RHT> {
  static constexpr int kWeights = 512, kBlocks = 16, kPitch = 128;
  static constexpr int kHi = 16;
  static constexpr int kScaleBox = 16;
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

// The four table entries addressed by the bytes of `word`, as (e0 + e1, e2 + e3).
// Slot i lives on page i/2 at column offset (i%2)*128; `lanereg` = table base | lane*4.
__device__ __forceinline__ void lookup4(uint32_t word, uint32_t lanereg, float& a, float& b) {
  const float e0 = lds_imm<0>(__byte_perm(word, lanereg, 0x7604));
  const float e1 = lds_imm<128>(__byte_perm(word, lanereg, 0x7614));
  const float e2 = lds_imm<kPage>(__byte_perm(word, lanereg, 0x7624));
  const float e3 = lds_imm<kPage + 128>(__byte_perm(word, lanereg, 0x7634));
  a = e0 + e1;
  b = e2 + e3;
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
  uint32_t* cnt;  // [NC] per-chunk arrival counters (KS > 1)
  int KS;         // number of slices
  int nblk;       // scale blocks per row
  unsigned* fault;  // set when a bounded wait gives up
};

// Builds the x slice and the lookup tables for slice j (consumer threads only).
template <int FMT>
__device__ __forceinline__ void build_slice(const Args<FMT>& a, int64_t j, uint32_t tbase,
                                            float* xs, int ctid) {
  using T = Traits<FMT>;
  const int64_t blk0 = j * T::kBlocks;
  const int nb_here = static_cast<int>(a.nblk - blk0 < T::kBlocks ? a.nblk - blk0 : T::kBlocks);
  const int nw = FMT == LBQ_TERN5 ? 7 * nb_here : (FMT == LBQ_SIGN1 ? 4 * nb_here : 2 * nb_here);
  const int nx = FMT == LBQ_Q2RHT ? nb_here * kQ2Block : nb_here * kTernBlock;
  const int64_t k0 = j * T::kWeights;
  const int lane = ctid & 31;

  if (FMT == LBQ_Q2RHT) {
    if (ctid < 32) {
      float v[16];
      rht512_warp_load(a.x + k0, a.D + k0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) xs[16 * lane + i] = v[i];
    }
  } else {
    for (int i = ctid; i < T::kWeights; i += 32 * kConsumers)
      xs[i] = i < nx ? bf16_bits_to_f32(a.x[k0 + i]) : 0.0f;
  }
  named_bar_sync(1, 32 * kConsumers);

  for (int task = ctid; task < 64 * T::kHi; task += 32 * kConsumers) {
    const int cp = task & 63, hi = task >> 6;
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
      const float l3 = static_cast<float>(hi % 3 - 1), l4 = static_cast<float>(hi / 3 - 1);
      const float2 q = __ffma2_rn(make_float2(l3, l3), xv[3], __fmul2_rn(make_float2(l4, l4), xv[4]));
      float2 qc[3], ab[9];
#pragma unroll
      for (int d2 = 0; d2 < 3; ++d2) {
        const float l = static_cast<float>(d2 - 1);
        qc[d2] = __ffma2_rn(make_float2(l, l), xv[2], q);
      }
#pragma unroll
      for (int m = 0; m < 9; ++m) {
        const float l0 = static_cast<float>(m % 3 - 1), l1 = static_cast<float>(m / 3 - 1);
        ab[m] = __ffma2_rn(make_float2(l0, l0), xv[0], __fmul2_rn(make_float2(l1, l1), xv[1]));
      }
#pragma unroll
      for (int lo = 0; lo < 27; ++lo)
        sts_f2(col + static_cast<uint32_t>(lo + 27 * hi) * 256u, __fadd2_rn(qc[lo / 9], ab[lo % 9]));
    } else {
      // v = lo + 16 hi; low two digits from lo & 3 and lo >> 2 (1-bit: bit pairs)
      float2 qb[4], av[4];
      float2 q;
      if (FMT == LBQ_SIGN1) {
        q = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float l = ((hi >> e) & 1) ? 1.0f : -1.0f;
          q = __ffma2_rn(make_float2(l, l), xv[4 + e], q);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float l0 = (m & 1) ? 1.0f : -1.0f, l1 = (m & 2) ? 1.0f : -1.0f;
          av[m] = __ffma2_rn(make_float2(l0, l0), xv[0], __fmul2_rn(make_float2(l1, l1), xv[1]));
          qb[m] = __ffma2_rn(make_float2(l0, l0), xv[2], __ffma2_rn(make_float2(l1, l1), xv[3], q));
        }
      } else {
        const float l2 = static_cast<float>(hi & 3) - 1.5f, l3 = static_cast<float>(hi >> 2) - 1.5f;
        q = __ffma2_rn(make_float2(l2, l2), xv[2], __fmul2_rn(make_float2(l3, l3), xv[3]));
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float l = static_cast<float>(m) - 1.5f;
          av[m] = __fmul2_rn(make_float2(l, l), xv[0]);
          qb[m] = __ffma2_rn(make_float2(l, l), xv[1], q);
        }
      }
#pragma unroll
      for (int lo = 0; lo < 16; ++lo)
        sts_f2(col + static_cast<uint32_t>(lo + 16 * hi) * 256u, __fadd2_rn(qb[lo >> 2], av[lo & 3]));
    }
  }
  if (FMT == LBQ_TERN5) {  // byte values 243..255 never occur: zero rows keep them harmless
    for (int i = ctid; i < 13 * 64; i += 32 * kConsumers) {
      const int v = 243 + i / 64, c = i % 64;
      sts_f2(tbase + (c >> 5) * kPage + static_cast<uint32_t>(v) * 256u + (c & 31) * 8,
             make_float2(0.0f, 0.0f));
    }
  }
  named_bar_sync(1, 32 * kConsumers);
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_lut_kernel(const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_scales, const Args<FMT> a) {
  using T = Traits<FMT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();

  const uint32_t sbase = smem_u32(smem);
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  const uint32_t n_low = (tbase - sbase) / kStageBytes < kStages ? (tbase - sbase) / kStageBytes
                                                                 : kStages;
  const uint32_t high = tbase + 2 * kPage;  // first byte above the table
  const uint32_t tail = high + (kStages - n_low) * kStageBytes;
  if (tail + kTailBytes > sbase + kSmem) {  // cannot happen with a 0 or 1 KB reserved prefix
    if (tid == 0) atomicExch(a.fault, kFaultLayout);
    return;
  }
  auto stage_addr = [&](int s) -> uint32_t {
    return static_cast<uint32_t>(s) < n_low ? sbase + s * kStageBytes
                                            : high + (s - n_low) * kStageBytes;
  };
  float* xs = reinterpret_cast<float*>(smem + (tail - sbase));
  const uint32_t full0 = tail + 4096, empty0 = full0 + kStages * 8;

  const int64_t NC = (a.N + kRows - 1) / kRows;
  const int64_t U = static_cast<int64_t>(a.KS) * NC;
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * U / gridDim.x;
  const int64_t u1 = static_cast<int64_t>(blockIdx.x + 1) * U / gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ---------------- producer: one lane streams tiles of codes (and scales)
    if (lane == 0) {
      prefetch_tmap(&tm_codes);
      if (T::kScaleBox) prefetch_tmap(&tm_scales);
      const uint32_t bytes = T::kPitch * kRows + T::kScaleBox * 2 * kRows;
      int64_t issued = 0;
      for (int64_t k = 0; k < u1 - u0; ++k) {
        const int s = static_cast<int>(k % kStages);
        const uint32_t use = static_cast<uint32_t>(k / kStages);
        if (!mbar_wait(empty0 + 8 * s, (use & 1) ^ 1, a.fault, kFaultProducer)) break;
        ++issued;
        const int64_t u = u0 + k, j = u / NC, c = u % NC;
        mbar_arrive_expect_tx(full0 + 8 * s, bytes);
        const uint32_t dst = stage_addr(s);
        tma_load_2d(dst, &tm_codes, static_cast<int32_t>(j * T::kPitch),
                    static_cast<int32_t>(c * kRows), full0 + 8 * s);
        if (T::kScaleBox)
          tma_load_2d(dst + kStageCodes, &tm_scales, static_cast<int32_t>(j * T::kScaleBox),
                      static_cast<int32_t>(c * kRows), full0 + 8 * s);
      }
      // Before this lane exits, every copy it issued must have landed (normally the
      // consumers have already seen them all; this matters only after a fault).
      for (int s = 0; s < kStages && s < issued; ++s) {
        const int64_t k_last = s + (issued - 1 - s) / kStages * kStages;
        mbar_wait(full0 + 8 * s, static_cast<uint32_t>(k_last / kStages) & 1, a.fault,
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
  bool ok = true;

  for (int64_t j = u0 / NC; j * NC < u1; ++j) {
    named_bar_sync(1, 32 * kConsumers);  // every consumer is done with the previous table
    build_slice<FMT>(a, j, tbase, xs, tid);
    const int64_t kb = (u0 > j * NC ? u0 : j * NC) - u0;
    const int64_t ke = ((j + 1) * NC < u1 ? (j + 1) * NC : u1) - u0;
    int64_t k = kb + ((warp - kb) % kConsumers + kConsumers) % kConsumers;
    for (; k < ke; k += kConsumers) {
      const int s = static_cast<int>(k % kStages);
      const uint32_t use = static_cast<uint32_t>(k / kStages);
      const uint32_t stage = stage_addr(s);
      const int64_t c = u0 + k - j * NC;
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
          float a0, b0, a1, b1;
          lookup4(wd0, lanereg, a0, b0);
          lookup4(wd1, lanereg, a1, b1);
          const float2 p = __fadd2_rn(make_float2(a0, a1), make_float2(b0, b1));
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
      const float v = acc[0];
      const int64_t r = c * kRows + lane;
      if (a.KS == 1) {
        if (r < a.N) a.y[r] = f32_to_bf16_bits(v);
        continue;
      }
      if (r < a.N) a.part[j * a.N + r] = v;
      __threadfence();
      __syncwarp();
      unsigned last = 0;
      if (lane == 0) last = (atomicAdd(a.cnt + c, 1u) == static_cast<unsigned>(a.KS - 1));
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {  // every slice of this chunk is in: sum them in slice order
        __threadfence();
        if (r < a.N) {
          float sum = 0.0f;
          for (int jj = 0; jj < a.KS; ++jj)
            sum += __ldcg(a.part + static_cast<int64_t>(jj) * a.N + r);
          a.y[r] = f32_to_bf16_bits(sum);
        }
        if (lane == 0) a.cnt[c] = 0u;
      }
    }
  }
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
                                         static_cast<int>(kSmem));
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
  a.cnt = static_cast<uint32_t*>(ws);
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
  const int64_t units = static_cast<int64_t>(a.KS) * NC;
  const int64_t grid = units < sm_count() ? units : sm_count();

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_lut_kernel<FMT>, tc, ts, a);
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
