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
// use N = 16 or 32) x 128 K per stage (one ternary block). Warp roles:
//   warp 0   one lane streams fp16 activation tiles with 2D TMA (128-byte swizzle)
//   warp 1   allocates tensor memory; one lane issues the MMAs and commits stages
//   warps 4-7 one thread per weight row: packed blocks arrive with cp.async (6 in
//            flight), each byte becomes five fp16 trits through a small table, is
//            scaled, and stored in the 128-byte-swizzled K-major operand layout;
//            then the same threads read the accumulator from tensor memory
//            (their own 32-lane quarter) and write bf16 Y.
// Every wait is bounded (see sm100_async.cuh).
#include <cudaTypedefs.h>

#include "sm100_async.cuh"

namespace {

using namespace lbq;

constexpr int kTileN = 128;     // weight rows per tile (MMA M)
constexpr int kTileK = 128;     // K per stage
constexpr int kMaxTileM = 128;  // tokens per tile (MMA N)
constexpr int kStagesTC = 3;
constexpr int kRawDepth = 6;    // packed blocks in flight per decoder thread
constexpr int kThreadsTC = 256;
constexpr uint32_t kSlabA = kTileN * 128;          // 128 rows x 64 k fp16
constexpr uint32_t kStageA = 2 * kSlabA;           // two 64-k slabs
constexpr uint32_t kStageB = 2 * kMaxTileM * 128;
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStagesTC * kStageA;
constexpr uint32_t kOffRaw = kOffB + kStagesTC * kStageB;
constexpr uint32_t kRawPerThread = kRawDepth * kTernBlockBytes;
constexpr uint32_t kOffLut = kOffRaw + kTileN * kRawPerThread;
constexpr uint32_t kLutBytes = 2 * 243 * 16;
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

// Five fp16 trits of one ternary byte, in the two word alignments a byte can take
// (5 j is even for even j). Table entry 16 bytes: three words used.
__device__ __forceinline__ void build_trit_table(uint32_t lut, int tid) {
  for (int i = tid; i < 2 * 243; i += kThreadsTC) {
    const int v = i % 243;
    const bool odd = i >= 243;
    uint32_t t[5];
    int r = v;
#pragma unroll
    for (int e = 0; e < 5; ++e) {
      const int d = r % 3;
      r /= 3;
      t[e] = d == 0 ? 0xBC00u : (d == 1 ? 0u : 0x3C00u);  // fp16 -1, 0, +1
    }
    const uint32_t w0 = odd ? (t[0] << 16) : (t[0] | (t[1] << 16));
    const uint32_t w1 = odd ? (t[1] | (t[2] << 16)) : (t[2] | (t[3] << 16));
    const uint32_t w2 = odd ? (t[3] | (t[4] << 16)) : t[4];
    sts_u128(lut + 16u * i, w0, w1, w2, 0u);
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
  const int nkb = static_cast<int>(a.K / kTileK);
  const uint32_t fullA = s0 + kOffBar, fullB = fullA + 8 * kStagesTC;
  const uint32_t empty = fullB + 8 * kStagesTC, accum = empty + 8 * kStagesTC;
  const uint32_t lut = s0 + kOffLut;

  build_trit_table(lut, tid);
  if (tid == 0) {
    for (int s = 0; s < kStagesTC; ++s) {
      mbar_init(fullA + 8 * s, kTileN);  // every decoder thread arrives
      mbar_init(fullB + 8 * s, 1);       // the TMA lane arrives (+ bytes)
      mbar_init(empty + 8 * s, 1);       // the MMA commit arrives
    }
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s0 + kOffTmem, a.tmem_cols);
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
        tma_load_2d(dst, &tm_x, kb * kTileK, static_cast<int32_t>(m0), fullB + 8 * s);
        tma_load_2d(dst + static_cast<uint32_t>(a.tile_m) * 128u, &tm_x, kb * kTileK + 64,
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
        const uint32_t sa = s0 + kOffA + s * kStageA, sb = s0 + kOffB + s * kStageB;
#pragma unroll
        for (int ks = 0; ks < kTileK / 16; ++ks) {
          const uint32_t slab = ks >> 2, koff = (ks & 3) * 32;
          mma_f16_ss(tmem, sw128_desc(sa + slab * kSlabA + koff), sw128_desc(sb + slab * slab_b + koff),
                     idesc, (kb | ks) != 0 ? 1u : 0u);
        }
        mma_commit(empty + 8 * s);  // the stage is free once these MMAs are done
      }
      mma_commit(accum);  // the accumulator is complete once every MMA is done
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- decode one weight row per thread, then the epilogue
    const int d = tid - 4 * 32;
    const int64_t n = n0 + d;
    const bool rv = n < a.N;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(a.codes + (rv ? n : 0) * a.cstride);
    const uint32_t ring = s0 + kOffRaw + static_cast<uint32_t>(d) * kRawPerThread;
#pragma unroll 1
    for (int p = 0; p < kRawDepth; ++p) {
      if (rv && p < nkb)
        for (int q = 0; q < 7; ++q) cp_async4(ring + p * kTernBlockBytes + 4 * q, src + p * 7 + q);
      cp_async_commit();
    }
    bool ok = true;
#pragma unroll 1
    for (int kb = 0; kb < nkb; ++kb) {
      cp_async_wait<kRawDepth - 1>();  // block kb has landed in its ring slot
      const uint32_t slot = ring + (kb % kRawDepth) * kTernBlockBytes;
      uint32_t w[7];
#pragma unroll
      for (int q = 0; q < 7; ++q) w[q] = rv ? lds32(slot + 4 * q) : 0u;
      if (rv && kb + kRawDepth < nkb)
        for (int q = 0; q < 7; ++q) cp_async4(slot + 4 * q, src + (kb + kRawDepth) * 7 + q);
      cp_async_commit();

      uint32_t hv[64];  // 128 fp16 weights of this row's block, in pairs
#pragma unroll
      for (int j = 0; j < kTernCodeBytes; ++j) {
        const uint32_t v = (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
        const uint4 e = lds_u128(lut + ((j & 1) ? 243u * 16u : 0u) + v * 16u);
        if (!(j & 1)) {
          const int b = 5 * j / 2;
          hv[b] = e.x;
          hv[b + 1] = e.y;
          hv[b + 2] = e.z;
        } else {
          const int b = (5 * j - 1) / 2;
          hv[b] |= e.x;
          if (b + 1 < 64) hv[b + 1] = e.y;
          if (b + 2 < 64) hv[b + 2] = e.z;  // byte 25's last two trits are padding
        }
      }
      const uint32_t sbits = w[6] >> 16;
      const __half2 s2 = __halves2half2(__ushort_as_half(static_cast<uint16_t>(sbits)),
                                        __ushort_as_half(static_cast<uint16_t>(sbits)));
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const __half2 t = *reinterpret_cast<const __half2*>(&hv[i]);
        const __half2 p = __hmul2(t, s2);  // exact: t is -1, 0 or +1
        hv[i] = *reinterpret_cast<const uint32_t*>(&p);
      }

      const int s = kb % kStagesTC;
      const uint32_t use = static_cast<uint32_t>(kb / kStagesTC);
      if (ok) ok = mbar_wait(empty + 8 * s, (use & 1) ^ 1, a.fault, kFaultDecode);
      const uint32_t base = s0 + kOffA + s * kStageA + (d >> 3) * 1024u + (d & 7) * 128u;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t addr = base + (c >> 3) * kSlabA + ((static_cast<uint32_t>(c & 7) ^ (d & 7)) << 4);
        sts_u128(addr, hv[4 * c], hv[4 * c + 1], hv[4 * c + 2], hv[4 * c + 3]);
      }
      fence_proxy_async_smem();  // the tensor cores read these through the async proxy
      mbar_arrive(fullA + 8 * s);
    }
    cp_async_wait<0>();

    // ---------------- epilogue: this warp's 32 TMEM lanes are its 32 weight rows
    if (ok) ok = mbar_wait(accum, 0, a.fault, kFaultEpilogue);
    tc_fence_after_sync();
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    for (int c0 = 0; c0 < a.tile_m; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(lane_base + static_cast<uint32_t>(c0), v);
      tmem_ld_wait();
      if (!ok || !rv) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int64_t m = m0 + c0 + i;
        if (m < a.M) {
          // undo the activation row's power-of-two scaling (exact)
          const float y = ldexpf(__uint_as_float(v[i]), a.xexp[m]);
          a.Y[m * a.N + n] = f32_to_bf16_bits(y);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, a.tmem_cols);
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

// Workspace of the ternary tensor-core product: [64 KB reserved][fp16 X: M*K][exponents: M].
size_t lbq_gemm_tc_workspace(const lbq_weights* w, int64_t M) {
  return kWsCounterBytes + align_up(static_cast<size_t>(M) * w->K * 2, 1024) +
         static_cast<size_t>(M) * sizeof(int);
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
  a.tile_m = M >= kMaxTileM ? kMaxTileM : static_cast<int>((M + 15) / 16 * 16);
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
            static_cast<unsigned>((M + a.tile_m - 1) / a.tile_m));
  gemm_tern_tc_kernel<<<grid, kThreadsTC, kSmemTC, s>>>(tm, a);
  return cudaGetLastError();
}
