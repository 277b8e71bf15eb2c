// gemm_tc.cu -- batched ternary product Y = X * W_hat^T on the 5th-generation tensor cores.
//
// The dense contraction behind a ternary layer applied to a batch of tokens. Weights
// are ternary trits times one fp16 absmean scale per 128-weight block (pptc.cn
// ternary-27B article §5.1; mhpq.cn "27B in 5.9 GB" article §2.1); the kernel
// dequantises tiles of them into shared memory and feeds tcgen05 MMAs with fp32
// accumulation in tensor memory.
//
// Precision: a dequantised weight s16 * t (t in {-1,0,1}, s16 an fp16 scale) is
// exact in fp16 but not in bf16 (rounding s16 to bf16 could by itself use the whole
// 2^-8 * sum|w x| error budget), so the MMA runs kind::f16 with fp16 operands. The
// activations are converted once per call to fp16 after a per-row power-of-two
// scaling (exact) that keeps every row inside fp16's range; the output is scaled
// back exactly before the bf16 rounding.
//
// Tile: 128 weight rows (the MMA's M) x up to 128 tokens (the MMA's N; small batches
// use N = 16 or 32) x 128 K per stage (one ternary block). Weights: fp16 in tensor
// memory; activations: fp16 in shared memory. Warp roles:
//   warp 0   one lane streams fp16 activation tiles with 2D TMA (128-byte swizzle)
//   warp 1   allocates tensor memory; one lane issues the MMAs and commits stages
//   warps 4-11 two threads per weight row, one per 64-weight half of each block:
//            packed words arrive with cp.async (4 blocks in flight), each byte
//            becomes five fp16 trits through small tables, is scaled, and the 64
//            fp16 go straight to tensor memory (tcgen05.st: the weight operand is
//            read by the MMA from tensor memory, so neither the stores nor the
//            MMA's operand reads use shared-memory bandwidth); then the same warps
//            read the accumulator (warp w reads lane quarter w % 4, the two warp
//            groups split the columns) and write bf16 Y.
// Every wait is bounded (see sm100_async.cuh).
#include <cudaTypedefs.h>

#include "sm100_async.cuh"

namespace {

using namespace lbq;

constexpr int kTileN = 128;     // weight rows per tile (MMA M)
constexpr int kTileK = 128;     // K per stage
constexpr int kMaxTileM = 128;  // tokens per tile (MMA N)
constexpr int kStagesTC = 3;
constexpr int kRawDepth = 4;    // packed blocks in flight per decoder thread
constexpr int kDecoders = 2 * kTileN;  // two threads per weight row
constexpr int kThreadsTC = 128 + kDecoders;
constexpr uint32_t kStageB = 2 * kMaxTileM * 128;
// Tensor memory (512 columns): the fp32 accumulator in columns [0, tile_m), the fp16
// weight stages at kTmemA + 64 s (128 rows x 128 K = 64 columns each).
constexpr uint32_t kTmemCols = 512, kTmemA = 256;
constexpr uint32_t kOffB = 0;
constexpr uint32_t kOffRaw = kOffB + kStagesTC * kStageB;
constexpr uint32_t kRawWords = 5;  // words of a block a half-row decoder needs (see below)
constexpr uint32_t kRawPerThread = kRawDepth * kRawWords * 4;
constexpr uint32_t kOffLut = kOffRaw + kDecoders * kRawPerThread;
constexpr uint32_t kLutBytes = 1024;  // the four small trit tables (see build_trit_tables)
constexpr uint32_t kOffBar = (kOffLut + kLutBytes + 7) / 8 * 8;
constexpr uint32_t kOffTmem = kOffBar + (3 * kStagesTC + 1) * 8;
constexpr size_t kSmemTC = kOffTmem + 16 + 1024;  // + slack to align the base to 1024
constexpr unsigned kFaultX = 4, kFaultMma = 5, kFaultDecode = 6, kFaultEpilogue = 7;

struct TcArgs {
  const uint8_t* codes;
  int64_t cstride;
  int64_t K, N, M;
  const int* xexp;  // token row m of X was scaled by 2^-xexp[m]
  uint16_t* Y;
  int tile_m;       // MMA N: tokens per tile
  uint32_t tmem_cols;
  int kb_per_split; // K blocks per CTA along grid z (split-K)
  float* part;      // [splits][M][N] fp32 partial products, or null (no split)
  unsigned* fault;
};

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row groups
// 1024 bytes apart (sm_100 descriptor version 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;            // leading byte offset (unused with swizzle)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;    // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;            // version
  d |= static_cast<uint64_t>(2) << 61;            // 128-byte swizzle
  return d;
}

// Instruction descriptor: fp16 A and B, fp32 D, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16_m128(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_u128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                         uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// A ternary byte v = lo + 27 hi (lo < 27 holds trits 0..2, hi < 9 trits 3..4; hi is
// (v * 1214) >> 15, exact for every byte value) decodes through four small tables of
// fp16 trits (-1, 0, +1), one pair per word, for the two word alignments a byte's
// five weights can take (5 j is even for even j):
//   even: lo -> {(t0, t1), (t2, 0)} at +0     hi -> {(0, t3), (t4, 0)} at +512
//   odd:  lo -> {(0, t0), (t1, t2)} at +256   hi -> (t3, t4)           at +640
// A few hundred bytes, so the warps' random lookups rarely collide on a bank.
constexpr uint32_t kT27e = 0, kT27o = 256, kT9e = 512, kT9o = 640;

__device__ __forceinline__ uint32_t trit_f16(int d) {  // digit 0, 1, 2 -> fp16 -1, 0, +1
  return d == 0 ? 0xBC00u : (d == 1 ? 0u : 0x3C00u);
}

__device__ __forceinline__ void build_trit_tables(uint32_t lut, int tid) {
  if (tid < 27) {
    const uint32_t t0 = trit_f16(tid % 3), t1 = trit_f16(tid / 3 % 3), t2 = trit_f16(tid / 9);
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(lut + kT27e + 8u * tid), "r"(t0 | (t1 << 16)),
                 "r"(t2)
                 : "memory");
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(lut + kT27o + 8u * tid), "r"(t0 << 16),
                 "r"(t1 | (t2 << 16))
                 : "memory");
  } else if (tid >= 32 && tid < 41) {
    const int h = tid - 32;
    const uint32_t t3 = trit_f16(h % 3), t4 = trit_f16(h / 3);
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(lut + kT9e + 8u * h), "r"(t3 << 16), "r"(t4)
                 : "memory");
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(lut + kT9o + 4u * h), "r"(t3 | (t4 << 16)) : "memory");
  }
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Places byte j's five fp16 trits into hv (pair index b0 = the pair holding weight
// 5j, relative to hv[0]); pairs outside [0, kPairs) are skipped.
template <int kPairs>
__device__ __forceinline__ void place_byte(uint32_t (&hv)[kPairs], int j, int b0, uint32_t v,
                                           uint32_t lut) {
  const uint32_t hi = (v * 1214u) >> 15, lo = v - 27u * hi;
  if (!(j & 1)) {
    const uint2 a = lds64(lut + kT27e + 8u * lo), c = lds64(lut + kT9e + 8u * hi);
    if (b0 >= 0 && b0 < kPairs) hv[b0] = a.x;
    if (b0 + 1 >= 0 && b0 + 1 < kPairs) hv[b0 + 1] = a.y | c.x;
    if (b0 + 2 >= 0 && b0 + 2 < kPairs) hv[b0 + 2] = c.y;
  } else {
    const uint2 a = lds64(lut + kT27o + 8u * lo);
    const uint32_t c = lds32(lut + kT9o + 4u * hi);
    if (b0 >= 0 && b0 < kPairs) hv[b0] |= a.x;
    if (b0 + 1 >= 0 && b0 + 1 < kPairs) hv[b0 + 1] = a.y;
    if (b0 + 2 >= 0 && b0 + 2 < kPairs) hv[b0 + 2] = c;
  }
}

__global__ void __launch_bounds__(kThreadsTC, 1)
    gemm_tern_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t s0 = (sraw + 1023u) & ~1023u;  // 1024-aligned: 128-byte swizzle atoms
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kTileN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * a.tile_m;
  // this CTA's K blocks: [kb0, kb0 + nkb) (all of K unless split over grid z)
  const int kb0 = static_cast<int>(blockIdx.z) * a.kb_per_split;
  const int nkb_all = static_cast<int>(a.K / kTileK);
  const int nkb = (nkb_all - kb0 < a.kb_per_split) ? nkb_all - kb0 : a.kb_per_split;
  const uint32_t fullA = s0 + kOffBar, fullB = fullA + 8 * kStagesTC;
  const uint32_t empty = fullB + 8 * kStagesTC, accum = empty + 8 * kStagesTC;
  const uint32_t lut = s0 + kOffLut;

  build_trit_tables(lut, tid);
  if (tid == 0) {
    for (int s = 0; s < kStagesTC; ++s) {
      mbar_init(fullA + 8 * s, kDecoders);  // every decoder thread arrives
      mbar_init(fullB + 8 * s, 1);       // the TMA lane arrives (+ bytes)
      mbar_init(empty + 8 * s, 1);       // the MMA commit arrives
    }
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s0 + kOffTmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + (s0 - sraw) + kOffTmem);

  if (warp == 0) {
    // ---------------- activations: two 64-k boxes per stage, 128-byte swizzled
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      const uint32_t bytes = 2u * static_cast<uint32_t>(a.tile_m) * 128u;
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStagesTC;
        const uint32_t use = static_cast<uint32_t>(kb / kStagesTC);
        if (!mbar_wait(empty + 8 * s, (use & 1) ^ 1, a.fault, kFaultX)) break;
        ++issued;
        mbar_arrive_expect_tx(fullB + 8 * s, bytes);
        const uint32_t dst = s0 + kOffB + s * kStageB;
        tma_load_2d(dst, &tm_x, (kb0 + kb) * kTileK, static_cast<int32_t>(m0), fullB + 8 * s);
        tma_load_2d(dst + static_cast<uint32_t>(a.tile_m) * 128u, &tm_x, (kb0 + kb) * kTileK + 64,
                    static_cast<int32_t>(m0), fullB + 8 * s);
      }
      // every issued copy must land before this CTA can exit (matters after a fault)
      for (int kb = issued - kStagesTC > 0 ? issued - kStagesTC : 0; kb < issued; ++kb)
        mbar_wait(fullB + 8 * (kb % kStagesTC), static_cast<uint32_t>(kb / kStagesTC) & 1,
                  a.fault, kFaultX, /*give_up_after_fault=*/false);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue: 8 instructions of K = 16 per stage
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_m128(a.tile_m);
      const uint32_t slab_b = static_cast<uint32_t>(a.tile_m) * 128u;
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int s = kb % kStagesTC;
        const uint32_t par = static_cast<uint32_t>(kb / kStagesTC) & 1;
        ok = mbar_wait(fullA + 8 * s, par, a.fault, kFaultMma) &&
             mbar_wait(fullB + 8 * s, par, a.fault, kFaultMma);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t ta = tmem + kTmemA + 64u * s, sb = s0 + kOffB + s * kStageB;
#pragma unroll
        for (int ks = 0; ks < kTileK / 16; ++ks) {  // K = 16: 8 tensor-memory columns of A
          const uint32_t slab = ks >> 2, koff = (ks & 3) * 32;
          mma_f16_ts(tmem, ta + 8u * ks, sw128_desc(sb + slab * slab_b + koff), idesc,
                     (kb | ks) != 0 ? 1u : 0u);
        }
        mma_commit(empty + 8 * s);  // the stage is free once these MMAs are done
      }
      mma_commit(accum);  // the accumulator is complete once every MMA is done
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- decode: thread d owns row d % 128, half h = d / 128 of each block.
    // Half 0 = weights 0..63 = bytes 0..12 (byte 12 only up to its 4th trit); half 1 =
    // weights 64..127 = byte 12's 5th trit and bytes 13..25. Half 0 copies words 0..3
    // and 6 (the scale), half 1 words 3..6.
    const int d = tid - 128;
    const int row = d & (kTileN - 1), h = d >> 7;
    const int64_t n = n0 + row;
    const bool rv = n < a.N;
    const uint32_t* src =
        reinterpret_cast<const uint32_t*>(a.codes + (rv ? n : 0) * a.cstride) + 7 * kb0;
    const uint32_t ring = s0 + kOffRaw + static_cast<uint32_t>(d) * kRawPerThread;
    const int wsrc[kRawWords] = {h ? 3 : 0, h ? 4 : 1, h ? 5 : 2, h ? 6 : 3, 6};
#pragma unroll 1
    for (int p = 0; p < kRawDepth; ++p) {
      if (rv && p < nkb)
        for (int q = 0; q < kRawWords; ++q)
          cp_async4(ring + (p * kRawWords + q) * 4, src + p * 7 + wsrc[q]);
      cp_async_commit();
    }
    bool ok = true;
#pragma unroll 1
    for (int kb = 0; kb < nkb; ++kb) {
      cp_async_wait<kRawDepth - 1>();  // block kb has landed in its ring slot
      const uint32_t slot = ring + (kb % kRawDepth) * kRawWords * 4;
      uint32_t w[kRawWords];
#pragma unroll
      for (int q = 0; q < kRawWords; ++q) w[q] = rv ? lds32(slot + 4 * q) : 0u;
      if (rv && kb + kRawDepth < nkb)
        for (int q = 0; q < kRawWords; ++q)
          cp_async4(slot + 4 * q, src + (kb + kRawDepth) * 7 + wsrc[q]);
      cp_async_commit();

      uint32_t hv[32];  // this half's 64 fp16 weights, in pairs
      if (h == 0) {
        // bytes 0..12 = w[0..3]; byte j covers weights 5j..5j+4 (pair 5j/2)
#pragma unroll
        for (int j = 0; j < 13; ++j)
          place_byte<32>(hv, j, (5 * j) >> 1, (w[j >> 2] >> (8 * (j & 3))) & 0xFFu, lut);
      } else {
        // w[0..3] = words 3..6 = bytes 12..27: byte 12 (the low byte of w[0]) gives
        // weight 64 with its 5th trit; bytes 13..25 follow; pairs relative to weight 64
#pragma unroll
        for (int j = 12; j < kTernCodeBytes; ++j) {
          const int jj = j - 12;
          place_byte<32>(hv, j, ((5 * j) >> 1) - 32, (w[jj >> 2] >> (8 * (jj & 3))) & 0xFFu, lut);
        }
      }
      const uint32_t sbits = (h ? w[3] : w[4]) >> 16;
      const __half2 s2 = __halves2half2(__ushort_as_half(static_cast<uint16_t>(sbits)),
                                        __ushort_as_half(static_cast<uint16_t>(sbits)));
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const __half2 t = *reinterpret_cast<const __half2*>(&hv[i]);
        const __half2 p = __hmul2(t, s2);  // exact: t is -1, 0 or +1
        hv[i] = *reinterpret_cast<const uint32_t*>(&p);
      }

      const int s = kb % kStagesTC;
      const uint32_t use = static_cast<uint32_t>(kb / kStagesTC);
      if (ok) ok = mbar_wait(empty + 8 * s, (use & 1) ^ 1, a.fault, kFaultDecode);
      __syncwarp();  // tcgen05.st is warp-collective
      tc_fence_after_sync();
      // this warp's 32 rows (lane quarter warp % 4), columns of this half of the block
      tmem_st32(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + kTmemA + 64u * s + 32u * h, hv);
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(fullA + 8 * s);
    }
    cp_async_wait<0>();

    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its rows);
    // the two warp groups take alternate 16-column chunks
    if (ok) ok = mbar_wait(accum, 0, a.fault, kFaultEpilogue);
    tc_fence_after_sync();
    const int q = warp & 3, grp = (warp - 4) >> 2;
    const int64_t ne = n0 + 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    for (int c0 = 16 * grp; c0 < a.tile_m; c0 += 32) {
      uint32_t v[16];
      tmem_ld16(lane_base + static_cast<uint32_t>(c0), v);
      tmem_ld_wait();
      if (!ok || ne >= a.N) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int64_t m = m0 + c0 + i;
        if (m < a.M) {
          // undo the activation row's power-of-two scaling (exact)
          const float y = ldexpf(__uint_as_float(v[i]), a.xexp[m]);
          if (a.part)
            a.part[(static_cast<int64_t>(blockIdx.z) * a.M + m) * a.N + ne] = y;
          else
            a.Y[m * a.N + ne] = f32_to_bf16_bits(y);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Activations to fp16, one row per CTA: x' = x * 2^-e with e chosen so that max|x'|
// lies in [2^14, 2^15) (an exact power-of-two scaling, up or down, so rows of large
// and of tiny activations both use fp16's full precision), rounded to nearest fp16.
__global__ void __launch_bounds__(256) x_to_f16_kernel(const uint16_t* __restrict__ X, int64_t K,
                                                        uint16_t* __restrict__ Xh,
                                                        int* __restrict__ xexp) {
  __shared__ float red[8];
  const int64_t m = blockIdx.x;
  const uint16_t* xr = X + m * K;
  float mx = 0.0f;
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) mx = fmaxf(mx, fabsf(bf16_bits_to_f32(xr[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) mx = fmaxf(mx, red[i]);
  const int e = mx > 0.0f ? ilogbf(mx) - 14 : 0;  // floor(log2(max|x|)) - 14
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
    Xh[m * K + k] = __half_as_ushort(__float2half_rn(ldexpf(bf16_bits_to_f32(xr[k]), -e)));
  if (threadIdx.x == 0) xexp[m] = e;
}

// Y = bf16(sum over splits of the fp32 partial products), splits in order.
__global__ void __launch_bounds__(256) gemm_split_sum_kernel(const float* __restrict__ part,
                                                             int splits, int64_t MN,
                                                             uint16_t* __restrict__ Y) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= MN) return;
  float v[8];
  float sum = 0.0f;
  for (int z0 = 0; z0 < splits; z0 += 8) {
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = z0 + q < splits ? __ldcg(part + (z0 + q) * MN + i) : 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (z0 + q < splits) sum += v[q];
  }
  Y[i] = f32_to_bf16_bits(sum);
}

struct TcPlan {
  int tile_m, splits, kb_per_split;
};

// Tile and split-K plan: K is split over grid z only when the output tiles alone
// cannot fill the SMs (small batches).
TcPlan plan_for(const lbq_weights* w, int64_t M) {
  TcPlan p;
  p.tile_m = M >= kMaxTileM ? kMaxTileM : static_cast<int>((M + 15) / 16 * 16);
  const int64_t tiles = ((w->N + kTileN - 1) / kTileN) * ((M + p.tile_m - 1) / p.tile_m);
  const int nkb = static_cast<int>(w->K / kTileK);
  int splits = 1;
  if (tiles < sm_count()) splits = static_cast<int>(sm_count() / tiles);
  if (splits > nkb) splits = nkb;
  if (splits < 1) splits = 1;
  p.kb_per_split = (nkb + splits - 1) / splits;
  p.splits = (nkb + p.kb_per_split - 1) / p.kb_per_split;
  return p;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_tc() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

// Workspace of the ternary tensor-core product:
// [64 KB reserved][fp16 X: M*K][exponents: M][fp32 partials: splits*M*N when split].
size_t lbq_gemm_tc_workspace(const lbq_weights* w, int64_t M) {
  const TcPlan p = plan_for(w, M);
  size_t n = kWsCounterBytes + align_up(static_cast<size_t>(M) * w->K * 2, 1024) +
             align_up(static_cast<size_t>(M) * sizeof(int), 256);
  if (p.splits > 1) n += static_cast<size_t>(p.splits) * M * w->N * sizeof(float);
  return n;
}

cudaError_t lbq_launch_gemm_tc(const lbq_weights* w, const uint16_t* X, int64_t M, uint16_t* Y,
                               void* ws, cudaStream_t s) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tern_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemTC));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  char* base = static_cast<char*>(ws) + kWsCounterBytes;
  uint16_t* Xh = reinterpret_cast<uint16_t*>(base);
  int* xexp = reinterpret_cast<int*>(base + align_up(static_cast<size_t>(M) * w->K * 2, 1024));
  x_to_f16_kernel<<<static_cast<unsigned>(M), 256, 0, s>>>(X, w->K, Xh, xexp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  TcArgs a;
  a.codes = static_cast<const uint8_t*>(w->codes);
  a.cstride = w->code_stride;
  a.K = w->K;
  a.N = w->N;
  a.M = M;
  a.xexp = xexp;
  a.Y = Y;
  const TcPlan plan = plan_for(w, M);
  a.tile_m = plan.tile_m;
  a.kb_per_split = plan.kb_per_split;
  a.part = plan.splits > 1
               ? reinterpret_cast<float*>(reinterpret_cast<char*>(xexp) +
                                          align_up(static_cast<size_t>(M) * sizeof(int), 256))
               : nullptr;
  a.tmem_cols = a.tile_m <= 32 ? 32u : (a.tile_m <= 64 ? 64u : 128u);
  a.fault = lbq_fault_word();
  if (!a.fault) return cudaErrorInvalidDevicePointer;

  auto fn = encode_fn_tc();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap tm;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(w->K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(w->K) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(a.tile_m)};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Xh, dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>((w->N + kTileN - 1) / kTileN),
            static_cast<unsigned>((M + a.tile_m - 1) / a.tile_m), static_cast<unsigned>(plan.splits));
  gemm_tern_tc_kernel<<<grid, kThreadsTC, kSmemTC, s>>>(tm, a);
  e = cudaGetLastError();
  if (e != cudaSuccess || plan.splits == 1) return e;
  const int64_t MN = M * w->N;
  gemm_split_sum_kernel<<<static_cast<unsigned>((MN + 255) / 256), 256, 0, s>>>(a.part, plan.splits, MN, Y);
  return cudaGetLastError();
}
