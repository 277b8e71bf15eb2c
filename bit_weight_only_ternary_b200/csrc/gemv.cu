// gemv.cu -- batch-1 low-bit GEMV, y = W_hat x (bf16 in, fp32 accumulate, bf16 out).
//
// Ternary products reduce to adding, subtracting or skipping activations (pptc.cn
// ternary-27B article §1.2; mhpq.cn "27B in 5.9 GB" article §2.2) and each block's
// sum is scaled by its fp16 scale (mhpq.cn §2.1). The 1-bit format is the Q1_0 case
// of the neodrop.ai round-up (part 2); the 2-bit format multiplies the rotated
// input x' = H D x / sqrt(512) of the feinterview.poetries.top "27B in 12 GB"
// article, computed here in shared memory, never in global memory.
//
// Design (HBM-bound; the decode must cost about one instruction per weight):
//  * A CTA owns one K-slice at a time (ternary 4 blocks = 512 weights = 28 words
//    of a row; 1-bit 1024 weights = 32 words; 2-bit 512 weights = 32 words) and
//    builds in shared memory, for every byte position of the slice, a table of
//    the partial dot product of that byte's codes with the slice of x, for all
//    256 byte values (lookup of partial sums). A byte then costs one PRMT (which
//    forms the table address directly), one LDS and one FADD.
//  * Lane l of a warp always reads word l of the slice, so the 32 lanes hit 32
//    different table columns: the table is laid out [value][lane] and the loads
//    are bank-conflict free. A warp streams 32 rows (one coalesced 4-byte load per
//    lane per row, all 32 issued up front), then a transposing butterfly leaves
//    row r0 + l's slice sum in lane l.
//  * Slices are split over CTAs (split-K). Each warp writes its 32 slice sums to
//    the workspace; the last warp to finish a 32-row chunk (a counter per chunk,
//    in the workspace's fixed counter region) adds the slices in a fixed order and
//    writes bf16 y, so results are deterministic. That warp resets the counter.
//  * Persistent grid: one 512-thread CTA per SM (the table takes 128 KB), each
//    with an equal share of the (slice, 32-row chunk) units in slice-major order.
#include "rht.cuh"

namespace {

using namespace lbq;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 32;                   // rows per unit (one warp)
constexpr uint32_t kPage = 65536;           // one table page: 256 values x 256 bytes
constexpr int kXs = 1024;                   // floats of x per slice (max)
// Dynamic shared memory: up to 64 KB of alignment pad (the table must start at a
// 64 KB boundary of the shared window), two table pages, the slice of x.
constexpr size_t kSmem = kPage + 2 * kPage + kXs * sizeof(float);

template <int FMT>
struct Traits;
template <>
struct Traits<LBQ_TERN5> {
  static constexpr int kWords = 28;         // 4 blocks x 7 words
  static constexpr int kWeights = 512;
  static constexpr int kBlocksPerSlice = 4;
  static constexpr int kHi = 9;             // value = lo + 27 * hi, lo < 27, hi < 9
  static constexpr int kLoN = 27;
};
template <>
struct Traits<LBQ_SIGN1> {
  static constexpr int kWords = 32;         // 8 blocks x 4 words
  static constexpr int kWeights = 1024;
  static constexpr int kBlocksPerSlice = 8;
  static constexpr int kHi = 16;            // value = lo + 16 * hi
  static constexpr int kLoN = 16;
};
template <>
struct Traits<LBQ_Q2RHT> {
  static constexpr int kWords = 32;         // 16 blocks x 2 words
  static constexpr int kWeights = 512;
  static constexpr int kBlocksPerSlice = 16;
  static constexpr int kHi = 16;
  static constexpr int kLoN = 16;
};

__device__ __forceinline__ uint32_t ldg_stream(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ldg_stream_u16(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.b16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

template <uint32_t kImm>
__device__ __forceinline__ float lds_imm(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(kImm));
  return v;
}

__device__ __forceinline__ void sts_f2(uint32_t addr, float a, float b) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}

// Partial sum of the four table entries addressed by the bytes of `word`.
// Slot i lives on page i/2, at column offset (i%2)*128; `lanereg` carries the
// table base (bits 16..31) and lane*4 (bits 0..7).
__device__ __forceinline__ float lookup4(uint32_t word, uint32_t lanereg) {
  const uint32_t a0 = __byte_perm(word, lanereg, 0x7604);
  const uint32_t a1 = __byte_perm(word, lanereg, 0x7614);
  const uint32_t a2 = __byte_perm(word, lanereg, 0x7624);
  const uint32_t a3 = __byte_perm(word, lanereg, 0x7634);
  const float e0 = lds_imm<0>(a0);
  const float e1 = lds_imm<128>(a1);
  const float e2 = lds_imm<kPage>(a2);
  const float e3 = lds_imm<kPage + 128>(a3);
  return (e0 + e1) + (e2 + e3);
}

// acc[i] holds lane's contribution to row i of the unit; returns row `lane`'s total.
__device__ __forceinline__ float transpose_reduce(float (&acc)[kRows], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = hi ? acc[i] : acc[i + o];
      const float keep = hi ? acc[i + o] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return acc[0];
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

// Code value (level) of digit e of byte value v.
template <int FMT>
__device__ __forceinline__ float digit_level(int v, int e) {
  if (FMT == LBQ_TERN5) {
    for (int q = 0; q < e; ++q) v /= 3;
    return static_cast<float>(v % 3 - 1);
  } else if (FMT == LBQ_SIGN1) {
    return ((v >> e) & 1) ? 1.0f : -1.0f;
  } else {
    return static_cast<float>((v >> (2 * e)) & 3) - 1.5f;
  }
}

template <int FMT>
struct Args {
  const uint8_t* codes;
  int64_t cstride;
  const uint16_t* scales;
  int64_t sstride;
  int64_t K, N;
  const uint16_t* x;
  const int8_t* D;
  uint16_t* y;
  float* part;     // [KS][N] slice sums (KS > 1)
  uint32_t* cnt;   // [NC] per-chunk arrival counters (KS > 1)
  int KS;          // number of slices
};

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemv_lut_kernel(const Args<FMT> a) {
  using T = Traits<FMT>;
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // Table base: the first 64 KB boundary of the shared window inside smem.
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  float* xs = reinterpret_cast<float*>(smem + (tbase - sbase) + 2 * kPage);
  const uint32_t lanereg = tbase | static_cast<uint32_t>(lane * 4);

  const int64_t NC = (a.N + kRows - 1) / kRows;
  const int64_t U = static_cast<int64_t>(a.KS) * NC;
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * U / gridDim.x;
  const int64_t u1 = static_cast<int64_t>(blockIdx.x + 1) * U / gridDim.x;
  const int64_t nblk = a.K / (FMT == LBQ_Q2RHT ? kQ2Block : kTernBlock);

  for (int64_t j = u0 / NC; j * NC < u1; ++j) {
    const int64_t c_lo = (u0 > j * NC ? u0 : j * NC) - j * NC;
    const int64_t c_hi = ((j + 1) * NC < u1 ? (j + 1) * NC : u1) - j * NC;
    const int64_t blk0 = j * T::kBlocksPerSlice;
    const int nb_here = static_cast<int>(nblk - blk0 < T::kBlocksPerSlice ? nblk - blk0
                                                                          : T::kBlocksPerSlice);
    const int nw = FMT == LBQ_TERN5 ? 7 * nb_here : (FMT == LBQ_SIGN1 ? 4 * nb_here : 2 * nb_here);
    const int nx = FMT == LBQ_Q2RHT ? nb_here * kQ2Block : nb_here * kTernBlock;
    const int64_t k0 = j * T::kWeights;

    __syncthreads();  // every warp is done with the previous slice's table
    // ---- the slice of x (2-bit: rotated) as fp32 in shared memory
    if (FMT == LBQ_Q2RHT) {
      if (warp == 0) {
        float v[16];
        rht512_warp_load(a.x + k0, a.D + k0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) xs[16 * lane + i] = v[i];
      }
    } else {
      for (int i = tid; i < T::kWeights; i += kThreads)
        xs[i] = i < nx ? bf16_bits_to_f32(a.x[k0 + i]) : 0.0f;
    }
    __syncthreads();
    // ---- the tables: entry(v) = P[v % R] + Q[v / R] for two adjacent columns at once
    for (int task = tid; task < 64 * T::kHi; task += kThreads) {
      const int cp = task & 63, hi = task >> 6;
      const int slot = cp >> 4, w0 = 2 * (cp & 15);
      constexpr int kLoDigits = FMT == LBQ_TERN5 ? 3 : (FMT == LBQ_SIGN1 ? 4 : 2);
      constexpr int kDigits = FMT == LBQ_TERN5 ? 5 : (FMT == LBQ_SIGN1 ? 8 : 4);
      float xa[kDigits], xb[kDigits];
#pragma unroll
      for (int e = 0; e < kDigits; ++e) {
        const int ka = digit_weight<FMT>(slot, w0, e, nw);
        const int kb = digit_weight<FMT>(slot, w0 + 1, e, nw);
        xa[e] = ka >= 0 ? xs[ka] : 0.0f;
        xb[e] = kb >= 0 ? xs[kb] : 0.0f;
      }
      float qa = 0.0f, qb = 0.0f;
#pragma unroll
      for (int e = kLoDigits; e < kDigits; ++e) {
        const float lv = digit_level<FMT>(hi, e - kLoDigits);
        qa += lv * xa[e];
        qb += lv * xb[e];
      }
      const uint32_t col = tbase + (slot >> 1) * kPage + (slot & 1) * 128 + w0 * 4;
#pragma unroll
      for (int lo = 0; lo < T::kLoN; ++lo) {
        float pa = qa, pb = qb;
#pragma unroll
        for (int e = 0; e < kLoDigits; ++e) {
          const float lv = digit_level<FMT>(lo, e);
          pa += lv * xa[e];
          pb += lv * xb[e];
        }
        sts_f2(col + static_cast<uint32_t>(lo + T::kLoN * hi) * 256u, pa, pb);
      }
    }
    if (FMT == LBQ_TERN5) {  // byte values 243..255 never occur: zero rows keep them harmless
      for (int i = tid; i < 13 * 64; i += kThreads) {
        const int v = 243 + i / 64, c = i % 64;
        const uint32_t addr = tbase + (c >> 5) * kPage + static_cast<uint32_t>(v) * 256u +
                              (c & 31) * 8;
        sts_f2(addr, 0.0f, 0.0f);
      }
    }
    __syncthreads();

    // ---- stream the rows of this slice, one 32-row unit per warp at a time
    const bool active = lane < nw;
    const int64_t word0 = (FMT == LBQ_TERN5 ? j * 28 : j * 32) + lane;
    const int scale_lane = FMT == LBQ_TERN5 ? (7 * (lane / 7) + 6 < 31 ? 7 * (lane / 7) + 6 : 31)
                                            : 0;
    const int64_t sidx = FMT == LBQ_SIGN1 ? j * 8 + lane / 4 : j * 16 + lane / 2;
    for (int64_t c = c_lo + warp; c < c_hi; c += kWarps) {
      const int64_t r0 = c * kRows;
      uint32_t wv[kRows];
      uint16_t sv[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const bool ok = active && (r0 + i < a.N);
        const uint32_t* p =
            reinterpret_cast<const uint32_t*>(a.codes + (r0 + i) * a.cstride) + word0;
        wv[i] = ok ? ldg_stream(p) : 0u;
        if (FMT != LBQ_TERN5) sv[i] = ok ? ldg_stream_u16(a.scales + (r0 + i) * a.sstride + sidx)
                                         : static_cast<uint16_t>(0);
      }
      float acc[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        float s;
        if (FMT == LBQ_TERN5) {
          const uint32_t sw = __shfl_sync(0xffffffffu, wv[i], scale_lane);
          s = f16_bits_to_f32(static_cast<uint16_t>(sw >> 16));
        } else {
          s = f16_bits_to_f32(sv[i]);
        }
        acc[i] = lookup4(wv[i], lanereg) * s;
      }
      const float v = transpose_reduce(acc, lane);
      const int64_t r = r0 + lane;
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
          for (int jj = 0; jj < a.KS; ++jj) sum += __ldcg(a.part + static_cast<int64_t>(jj) * a.N + r);
          a.y[r] = f32_to_bf16_bits(sum);
        }
        if (lane == 0) a.cnt[c] = 0u;
      }
    }
  }
}

int slices_of(const lbq_weights* w) {
  const int64_t per = w->fmt == LBQ_SIGN1 ? 1024 : 512;
  return static_cast<int>((w->K + per - 1) / per);
}

template <int FMT>
cudaError_t launch(const lbq_weights* w, const uint16_t* x, const int8_t* D, uint16_t* y, void* ws,
                   cudaStream_t s) {
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
  a.codes = static_cast<const uint8_t*>(w->codes);
  a.cstride = w->code_stride;
  a.scales = static_cast<const uint16_t*>(w->scales);
  a.sstride = w->scale_stride;
  a.K = w->K;
  a.N = w->N;
  a.x = x;
  a.D = D;
  a.y = y;
  a.KS = slices_of(w);
  const int64_t NC = (w->N + kRows - 1) / kRows;
  a.cnt = static_cast<uint32_t*>(ws);
  a.part = ws ? reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes) : nullptr;
  const int64_t units = static_cast<int64_t>(a.KS) * NC;
  const int64_t grid = units < sm_count() ? units : sm_count();
  gemv_lut_kernel<FMT><<<static_cast<unsigned>(grid), kThreads, kSmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

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
