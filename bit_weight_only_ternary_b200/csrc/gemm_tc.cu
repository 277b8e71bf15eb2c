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
// Tile: 128 weight rows (the MMA's M) x up to 256 tokens (the MMA's N, a multiple of
// 16 chosen by the tile planner) x 128 K per stage (one ternary block). Weights: fp16
// in tensor memory; activations: fp16 in shared memory. Warp roles:
//   warp 0   one lane streams fp16 activation tiles with 2D TMA (128-byte swizzle)
//   warp 1   allocates tensor memory; one lane issues the MMAs and commits stages
//   warp 3   for token tiles of at most 32: one lane issues the second half of each
//            block's MMAs (into accumulators of its own)
//   warp 2   one lane streams the packed weight rows with 2D TMA, four blocks
//            (112 bytes) of 128 rows per copy
//   warps 4-19 four threads per weight row, one per 32-weight quarter of each block.
//            Each byte becomes five fp16 values through one lookup: a table in
//            shared memory maps the byte to the byte-permute selectors that pick
//            +s, -s or 0 out of a register holding the block's scale, so a byte
//            costs one table load (its address is itself one byte permute of the
//            packed word) and one permute per pair of weights. The table is
//            replicated for the 16 lanes of a half warp, so the lookups of a warp
//            never collide on a bank. The 32 fp16 go straight to tensor memory
//            (tcgen05.st: the MMA reads the weight operand from tensor memory;
//            a block's store completes while the next block is decoded); then the
//            same warps read the accumulator (warp w reads lane quarter w % 4, the
//            four warp groups split the columns), undo the activation rows' scaling
//            and stage bf16 Y in shared memory for one TMA store. They also load
//            the selector table, once the first weight copies are in flight.
// Every wait is bounded (see sm100_async.cuh).
#include <cudaTypedefs.h>

#include <type_traits>
#include <utility>

#include "sm100_async.cuh"

namespace {

using namespace lbq;

constexpr int kTileN = 128;     // weight rows per tile (MMA M)
constexpr int kTileK = 128;     // K per stage (one ternary block)
constexpr int kMaxTileM = 256;  // tokens per tile (MMA N)
constexpr int kStagesTC = 4;
constexpr int kDecoders = 4 * kTileN;  // four threads per weight row, a quarter block each
constexpr int kThreadsTC = 128 + kDecoders;
constexpr int kChunkBlocks = 4;        // packed blocks per weight copy: 28 words of each row
constexpr uint32_t kChunkWords = kChunkBlocks * kTernBlockBytes / 4;
// The rows arrive in groups of four (word w of four rows in 16 consecutive bytes).
// A copy takes 32 groups x 116 words: the chunk's 112 words of each group plus the
// next chunk's first four, so that a group's row in shared memory is 464 bytes (29
// 16-byte bank groups, an odd number): the 32 rows a warp decodes then read their
// words from 32 different banks.
constexpr uint32_t kGroupWords = 4 * kChunkWords + 4;
constexpr uint32_t kRawStageBytes = kGroupWords * 4 * (kTileN / 4);
constexpr int kRawStages = 2;
// Activations arrive in slabs of K = 64 (one 128-byte swizzle row per token), a ring
// of kSlabs; an A stage (K = 128, one ternary block) consumes two of them.
constexpr int kSlabs = 4;
constexpr uint32_t kStageB = kMaxTileM * 128;  // one slab
// Tensor memory (512 columns): nacc fp32 accumulators of tile_m columns each in
// [0, 256), the fp16 weight stages at kTmemA + 64 s (128 rows x 128 K = 64 columns
// each). Successive MMAs go to different accumulators: an MMA that depends on the
// previous one's accumulator waits for it to finish, and a K = 16 step with a small
// token count is far shorter than that latency.
constexpr uint32_t kTmemCols = 512, kTmemA = 256, kAccCols = 256;
// Shared memory. The selector table sits at a 64 KB-aligned shared-window address T
// so that a table address is T | byte << 8 | lane slot (one byte permute):
//   [T - kLowBytes, T)   mbarriers + TMEM slot (256 B), raw weight ring, activation stage 0
//   [T, T + 62208)        selector table: [byte 0..242][even/odd][16 lanes] x 8 bytes
//   [T + 0xF400, ...)     activation stages 1..3
// The dynamic window starts 1 KB into shared memory on sm_100 (T = 64 KB); the
// kernel checks the placement and reports a fault rather than run off its end.
constexpr uint32_t kTabBytes = 243 * 256;
constexpr uint32_t kLowBytes = 256 + kRawStages * kRawStageBytes + kStageB;
constexpr uint32_t kHighB = 0xF400;  // first activation stage above the table (1 KB aligned)
constexpr uint32_t kHighBytes = kHighB + (kSlabs - 1) * kStageB;
constexpr size_t kSmemTC = 0x10000 - 0x400 + kHighBytes;
static_assert(kTabBytes <= kHighB, "table overlaps stage 1");
static_assert(0x400 + kLowBytes <= 0x10000, "low region does not fit below 64 KB");
static_assert(kSmemTC <= 232448, "over the shared-memory limit");
constexpr unsigned kFaultX = 4, kFaultMma = 5, kFaultDecode = 6, kFaultEpilogue = 7, kFaultW = 8,
                   kFaultSmem = 9;

struct TcArgs {
  int64_t K, N, M;
  const int* xexp;   // token row m of X was scaled by 2^-xexp[m]
  const int* xflag;  // 1: row m did not convert to fp16 exactly (recomputed on CUDA cores)
  const uint16_t* X; // the bf16 activations (for the flagged rows)
  const uint8_t* codes;  // packed weights (for the flagged rows), group-of-four order
  int64_t code_stride;
  uint16_t* Y;
  int tile_m;       // MMA N: tokens per tile
  int nacc;         // independent accumulators (a power of two, nacc * tile_m <= 256)
  int kb_per_split; // K blocks per CTA along grid z (split-K)
  float* part;      // [splits][M][N] fp32 partial products, or null (no split)
  int y_tma;        // 1: Y written through shared memory with one TMA store per tile
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

// ---------------------------------------------------------------- byte -> fp16 values
// A byte v = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4 holds five digits d = t + 1 (weights
// 5j .. 5j + 4 of the block for byte j). A register V = (s, -s) as two fp16, next
// to a zero register, lets one byte permute build a pair of fp16 weights: the
// selector code of a digit names the two bytes of +s (digit 2), -s (0) or zero (1).
constexpr uint32_t sel_code(uint32_t d) { return d == 2 ? 0x10u : (d == 0 ? 0x32u : 0x54u); }
constexpr uint32_t digit(uint32_t v, int i) {
  return i == 0 ? v % 3 : (i == 1 ? v / 3 % 3 : (i == 2 ? v / 9 % 3 : (i == 3 ? v / 27 % 3 : v / 81)));
}
// Byte j's first weight is the low half of a pair when j is even (5j even):
//   even entry: x = codes of (t0, t1, t2, t3), y = code of t4 (low half of the next pair)
//   odd entry:  x = code of t0 in the high half, y = codes of (t1, t2, t3, t4)
// so an even byte gives pairs (t0,t1) = x, (t2,t3) = x >> 16, and with the odd byte
// after it (t4, u0) = y_even | x_odd, (u1,u2) = y_odd, (u3,u4) = y_odd >> 16.
struct SelTable {
  uint32_t w[243][2][2];
};
constexpr SelTable make_sel_table() {
  SelTable t{};
  for (uint32_t v = 0; v < 243; ++v) {
    uint32_t c[5] = {};
    for (int i = 0; i < 5; ++i) c[i] = sel_code(digit(v, i));
    t.w[v][0][0] = c[0] | c[1] << 8 | c[2] << 16 | c[3] << 24;
    t.w[v][0][1] = c[4];
    t.w[v][1][0] = c[0] << 8;
    t.w[v][1][1] = c[1] | c[2] << 8 | c[3] << 16 | c[4] << 24;
  }
  return t;
}
__device__ const SelTable g_sel_table = make_sel_table();

// Replicates the table into shared memory as [byte][even/odd][16 lane slots] x 8 bytes
// (thread d of n threads).
__device__ __forceinline__ void load_sel_table(uint32_t tab, int d, int n) {
  const uint2* src = reinterpret_cast<const uint2*>(&g_sel_table);
  constexpr int kSlots = 243 * 2 * 16;
#pragma unroll 4
  for (int i = d; i < kSlots; i += n) {
    const uint2 e = __ldg(src + (i >> 4));
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(tab + 8u * i), "r"(e.x), "r"(e.y) : "memory");
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Word i of the block b of a 4-block row chunk held in raw[7] (compile-time indices).
template <int kB, int kI>
__device__ __forceinline__ uint32_t raw_word(const uint4 (&raw)[7]) {
  constexpr int w = 7 * kB + kI;
  const uint4 q = raw[w >> 2];
  return (w & 3) == 0 ? q.x : ((w & 3) == 1 ? q.y : ((w & 3) == 2 ? q.z : q.w));
}

// Sets word kW (0..27) of a 4-block row chunk held in raw[7].
template <int kW>
__device__ __forceinline__ void put_word(uint4 (&raw)[7], uint32_t v) {
  if constexpr ((kW & 3) == 0) raw[kW >> 2].x = v;
  else if constexpr ((kW & 3) == 1) raw[kW >> 2].y = v;
  else if constexpr ((kW & 3) == 2) raw[kW >> 2].z = v;
  else raw[kW >> 2].w = v;
}
// Loads, for the four blocks of a chunk, only the words quarter kQ decodes: quarter
// 0 reads words 0-1 of a block, 1 words 1-3, 2 words 3-4, 3 words 4-5, and all read
// word 6 (the scale). Word w of the row is 16 bytes from word w - 1 (group-of-four
// order) starting at `src`.
template <int kQ, int kB = 0>
__device__ __forceinline__ void load_quarter_words(uint4 (&raw)[7], uint32_t src) {
  constexpr int lo = kQ == 0 ? 0 : (kQ == 1 ? 1 : (kQ == 2 ? 3 : 4));
  constexpr int hi = kQ == 0 ? 1 : (kQ == 1 ? 3 : (kQ == 2 ? 4 : 5));
  [&]<int... I>(std::integer_sequence<int, I...>) {
    ((put_word<7 * kB + lo + I>(raw, lds32(src + 16u * (7 * kB + lo + I)))), ...);
  }(std::make_integer_sequence<int, hi - lo + 1>{});
  put_word<7 * kB + 6>(raw, lds32(src + 16u * (7 * kB + 6)));
  if constexpr (kB < 3) load_quarter_words<kQ, kB + 1>(raw, src);
}

// Decodes bytes [kJ, kJ1] of block kB into pairs hv[p - kP0] (pairs outside
// [kP0, kP0 + 16) are skipped). base_e / base_o: the table address of byte 0 for this
// lane (even / odd entries); V: (s, -s).
template <int kB, int kJ, int kJ1, int kP0>
struct DecodeBytes {
  static __device__ __forceinline__ void run(const uint4 (&raw)[7], uint32_t base_e, uint32_t base_o,
                                             uint32_t V, uint32_t carry, uint32_t (&hv)[16]) {
    const uint32_t word = raw_word<kB, kJ / 4>(raw);
    constexpr uint32_t sel = 0x7604u | ((kJ & 3) << 4);  // lane slot, byte kJ & 3, table base
    if constexpr ((kJ & 1) == 0) {
      const uint2 e = lds64(prmt(word, base_e, sel));
      constexpr int p = 5 * kJ / 2 - kP0;
      if constexpr (p >= 0 && p < 16) hv[p] = prmt(V, 0u, e.x);
      if constexpr (p + 1 >= 0 && p + 1 < 16) hv[p + 1] = prmt(V, 0u, e.x >> 16);
      if constexpr (kJ < kJ1) carry = e.y;
    } else {
      const uint2 o = lds64(prmt(word, base_o, sel));
      constexpr int p = (5 * kJ - 1) / 2 - kP0;
      if constexpr (p >= 0 && p < 16) hv[p] = prmt(V, 0u, carry | o.x);
      if constexpr (p + 1 >= 0 && p + 1 < 16) hv[p + 1] = prmt(V, 0u, o.y);
      if constexpr (p + 2 >= 0 && p + 2 < 16) hv[p + 2] = prmt(V, 0u, o.y >> 16);
    }
    if constexpr (kJ < kJ1) DecodeBytes<kB, kJ + 1, kJ1, kP0>::run(raw, base_e, base_o, V, carry, hv);
  }
};

// The 32 fp16 weights of quarter r of block kB of the chunk, in pairs (pairs 16 r ..
// 16 r + 15 of the block). Quarter 0 = bytes 0..6, 1 = bytes 6..12, 2 = bytes 12..19,
// 3 = bytes 19..25 (the bytes at the seams are decoded by both neighbours; byte 25's
// last two digits are padding).
template <int kB>
__device__ __forceinline__ void decode_quarter(const uint4 (&raw)[7], int r, uint32_t base_e,
                                               uint32_t base_o, uint32_t (&hv)[16]) {
  const uint32_t sw = raw_word<kB, 6>(raw);              // bytes 24..27: scale in the high half
  const uint32_t V = prmt(sw, sw ^ 0x80000000u, 0x7632u);  // (s, -s)
  switch (r) {
    case 0: DecodeBytes<kB, 0, 6, 0>::run(raw, base_e, base_o, V, 0u, hv); break;
    case 1: DecodeBytes<kB, 6, 12, 16>::run(raw, base_e, base_o, V, 0u, hv); break;
    case 2: DecodeBytes<kB, 12, 19, 32>::run(raw, base_e, base_o, V, 0u, hv); break;
    default: DecodeBytes<kB, 19, kTernCodeBytes - 1, 48>::run(raw, base_e, base_o, V, 0u, hv); break;
  }
}

// v * 2^e, exactly as ldexpf (one rounding): a multiply by the power of two when it
// is a normal float, which is every row but those of extreme magnitude.
__device__ __forceinline__ float scale_pow2(float v, int e) {
  return (e >= -126 && e <= 127) ? v * __int_as_float((e + 127) << 23) : ldexpf(v, e);
}

// Named barrier over `count` threads that also ORs a predicate over them: returns
// whether any participating thread passed true.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// Token rows whose values span more than fp16 holds exactly after one power-of-two
// scaling (bf16 keeps fp32's exponent range: a row may hold 2^40 next to 1.0) are
// flagged by the conversion kernel; for them the tile's outputs are recomputed here
// from the bf16 activations in fp32 on the CUDA cores, block by block as the pages
// define the product (sum of +-x per block, times the block's scale). Called by all
// kDecoders decoder threads (d = 0 .. kDecoders - 1) with the tile's flags in shared
// memory (xf, tile_m entries) and 4 * kTileN floats of shared scratch (red); the
// control flow depends on shared data only, so every thread meets every barrier.
// Each flagged token's 128 outputs go to `put(t, row, value)` on threads d < kTileN.
template <typename Put>
__device__ __forceinline__ void fixup_flagged(const TcArgs& a, int64_t n0, int64_t m0, int kb0,
                                              int nkb, const int* xf, float* red, int d,
                                              Put put) {
  const int row = d & (kTileN - 1), qtr = d / kTileN;  // 4 threads a row, blocks dealt round-robin
  const int64_t n = n0 + row;
  for (int t = 0; t < a.tile_m; ++t) {
    if (!xf[t]) continue;  // shared, so uniform across the threads
    const int64_t m = m0 + t;
    const uint16_t* x = a.X + m * a.K;
    float acc = 0.0f;
    if (n < a.N) {
      for (int kb = kb0 + qtr; kb < kb0 + nkb; kb += 4) {
        uint32_t w[7];
#pragma unroll
        for (int i = 0; i < 7; ++i)
          w[i] = __ldg(reinterpret_cast<const uint32_t*>(a.codes + g4_word_byte(n, 7 * kb + i, a.code_stride)));
        const float s = f16_bits_to_f32(static_cast<uint16_t>(w[6] >> 16));
        const uint16_t* xb = x + static_cast<int64_t>(kb) * kTernBlock;
        float part = 0.0f;
        for (int j = 0; j < kTernCodeBytes; ++j) {
          uint32_t v = (w[j >> 2] >> (8 * (j & 3))) & 0xffu;
          for (int i = 0; i < 5 && 5 * j + i < kTernBlock; ++i) {
            const uint32_t dgt = v % 3u;  // digit = trit + 1
            v /= 3u;
            const float xv = bf16_bits_to_f32(xb[5 * j + i]);
            if (dgt == 2u) part += xv;
            else if (dgt == 0u) part -= xv;
          }
        }
        acc += s * part;
      }
    }
    red[qtr * kTileN + row] = acc;
    named_bar_sync(3, kDecoders);
    if (d < kTileN && n < a.N)
      put(t, row, ((red[row] + red[kTileN + row]) + red[2 * kTileN + row]) + red[3 * kTileN + row]);
    named_bar_sync(3, kDecoders);
  }
}

__global__ void __launch_bounds__(kThreadsTC, 1)
    gemm_tern_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_y, const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t tab = (sraw + kLowBytes + 0xFFFFu) & ~0xFFFFu;
  if (tab - kLowBytes < sraw || tab + kHighBytes > sraw + static_cast<uint32_t>(kSmemTC)) {
    if (threadIdx.x == 0) atomicExch(a.fault, kFaultSmem);  // placement assumption broken
    return;
  }
  const uint32_t bstage0 = tab - kStageB;
  const uint32_t rawring = bstage0 - kRawStages * kRawStageBytes;
  const uint32_t bars = rawring - 256;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kTileN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * a.tile_m;
  // this CTA's K blocks: [kb0, kb0 + nkb) (all of K unless split over grid z);
  // kb_per_split is a multiple of the chunk
  const int kb0 = static_cast<int>(blockIdx.z) * a.kb_per_split;
  const int nkb_all = static_cast<int>(a.K / kTileK);
  const int nkb = (nkb_all - kb0 < a.kb_per_split) ? nkb_all - kb0 : a.kb_per_split;
  const int nchunks = (nkb + kChunkBlocks - 1) / kChunkBlocks;
  // fullA / emptyA: tensor-memory weight stages; fullB / emptyB: activation slabs
  const uint32_t fullA = bars, emptyA = fullA + 8 * kStagesTC;
  const uint32_t fullB = emptyA + 8 * kStagesTC, emptyB = fullB + 8 * kSlabs;
  const uint32_t accum = emptyB + 8 * kSlabs;
  const uint32_t fullR = accum + 8, emptyR = fullR + 8 * kRawStages;
  const uint32_t tslot = emptyR + 8 * kRawStages;
  auto bstage = [&](int s) { return s == 0 ? bstage0 : tab + kHighB + (s - 1) * kStageB; };

  // MMA issuers: with eight accumulators (token tiles of at most 32) the eight K steps
  // of a block split into two halves with disjoint accumulators, issued from two
  // warps on different schedulers (warps 1 and 3): a small MMA costs its issuing
  // scheduler ~45 cycles and more while decoder warps share it, about as long as the
  // tensor core needs for it.
  const int nissue = a.nacc == 8 ? 2 : 1;
  if (tid == 0) {
    for (int s = 0; s < kStagesTC; ++s) {
      mbar_init(fullA + 8 * s, kDecoders / 32);  // every decoder warp arrives
      mbar_init(emptyA + 8 * s, nissue);    // every MMA issuer's commit arrives
    }
    for (int s = 0; s < kSlabs; ++s) {
      mbar_init(fullB + 8 * s, 1);          // the activation TMA lane arrives (+ bytes)
      mbar_init(emptyB + 8 * s, 1);         // the MMA commit arrives
    }
    for (int r = 0; r < kRawStages; ++r) {
      mbar_init(fullR + 8 * r, 1);          // the weight TMA lane arrives (+ bytes)
      mbar_init(emptyR + 8 * r, kDecoders / 32); // every decoder warp has read its rows
    }
    mbar_init(accum, nissue);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tslot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  uint32_t tmem;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(tslot));

  if (warp == 0) {
    // ---------------- activations: one 64-k box per slab, 128-byte swizzled
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      const uint32_t bytes = static_cast<uint32_t>(a.tile_m) * 128u;
      const int nsl = 2 * nkb;
      int issued = 0;
      for (int sl = 0; sl < nsl; ++sl) {
        const int s = sl % kSlabs;
        const uint32_t use = static_cast<uint32_t>(sl / kSlabs);
        if (!mbar_wait(emptyB + 8 * s, (use & 1) ^ 1, a.fault, kFaultX)) break;
        ++issued;
        mbar_arrive_expect_tx(fullB + 8 * s, bytes);
        tma_load_2d(bstage(s), &tm_x, kb0 * kTileK + 64 * sl, static_cast<int32_t>(m0), fullB + 8 * s);
      }
      // every issued copy must land before this CTA can exit (matters after a fault)
      for (int sl = issued - kSlabs > 0 ? issued - kSlabs : 0; sl < issued; ++sl)
        mbar_wait(fullB + 8 * (sl % kSlabs), static_cast<uint32_t>(sl / kSlabs) & 1,
                  a.fault, kFaultX, /*give_up_after_fault=*/false);
    }
  } else if (warp == 1 || (warp == 3 && nissue == 2)) {
    // ---------------- MMA issue: 8 instructions of K = 16 per weight stage, four per
    // activation slab, from lane 0 of warp 1 (or slab halves 0 / 1 from warps 1 / 3).
    // The issue path is kept short (an MMA of 128 x 256 x 16 takes 128 cycles; with
    // descriptors rebuilt per instruction the loop took ~140 cycles an MMA whatever
    // its size): the accumulator columns of the eight K steps are fixed (nacc divides
    // 8), a slab's descriptor is built once and advanced by 32 bytes (+2 in its
    // address field) per K step.
    // (the slab range is a compile-time constant of each variant: a runtime loop
    // over it measurably slowed the issue of large MMAs)
    auto issue = [&](auto h_lo_c, auto h_hi_c) {
      constexpr int h_lo = decltype(h_lo_c)::value, h_hi = decltype(h_hi_c)::value;
      const uint32_t idesc = idesc_f16_m128(a.tile_m);
      uint32_t dcol[8];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) dcol[ks] = tmem + static_cast<uint32_t>((ks & (a.nacc - 1)) * a.tile_m);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int s = kb % kStagesTC;
        ok = mbar_wait(fullA + 8 * s, static_cast<uint32_t>(kb / kStagesTC) & 1, a.fault, kFaultMma);
        if (!ok) break;
        const uint32_t ta = tmem + kTmemA + 64u * s;
#pragma unroll
        for (int h = h_lo; h < h_hi; ++h) {
          const int sl = 2 * kb + h, sb_i = sl % kSlabs;
          ok = mbar_wait(fullB + 8 * sb_i, static_cast<uint32_t>(sl / kSlabs) & 1, a.fault, kFaultMma);
          if (!ok) break;
          tc_fence_after_sync();
          const uint64_t bdesc = sw128_desc(bstage(sb_i));
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {  // K = 16: 8 tensor-memory columns of A, 32 bytes of B
            const int ks = 4 * h + k4;
            // the first MMA into each accumulator overwrites it
            mma_f16_ts(dcol[ks], ta + 8u * ks, bdesc + 2u * k4, idesc, (kb > 0 || ks >= a.nacc) ? 1u : 0u);
          }
          mma_commit(emptyB + 8 * sb_i);  // the slab is free once these MMAs are done
        }
        if (!ok) break;
        mma_commit(emptyA + 8 * s);  // and the weight stage once every issuer's are
      }
      mma_commit(accum);  // the accumulator is complete once every MMA is done
    };
    if (lane == 0) {
      using I0 = std::integral_constant<int, 0>;
      using I1 = std::integral_constant<int, 1>;
      using I2 = std::integral_constant<int, 2>;
      if (nissue == 1) issue(I0{}, I2{});
      else if (warp == 1) issue(I0{}, I1{});
      else issue(I1{}, I2{});
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------- packed weights: 128 rows x 4 blocks per copy (rows past N read 0)
    if (lane == 0) {
      prefetch_tmap(&tm_w);
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int r = c % kRawStages;
        const uint32_t use = static_cast<uint32_t>(c / kRawStages);
        if (!mbar_wait(emptyR + 8 * r, (use & 1) ^ 1, a.fault, kFaultW)) break;
        ++issued;
        mbar_arrive_expect_tx(fullR + 8 * r, kRawStageBytes);
        tma_load_2d(rawring + r * kRawStageBytes, &tm_w,
                    static_cast<int32_t>((kb0 / kChunkBlocks + c) * 4 * kChunkWords),
                    static_cast<int32_t>(n0 / 4), fullR + 8 * r);
      }
      for (int c = issued - kRawStages > 0 ? issued - kRawStages : 0; c < issued; ++c)
        mbar_wait(fullR + 8 * (c % kRawStages), static_cast<uint32_t>(c / kRawStages) & 1,
                  a.fault, kFaultW, /*give_up_after_fault=*/false);
    }
  } else if (warp >= 4) {
    // ---------------- decode: thread d owns row d % 128, quarter r = d / 128 of each block
    const int d = tid - 128;
    // the selector table, loaded while the first weight copies are in flight
    load_sel_table(tab, d, kDecoders);
    named_bar_sync(2, kDecoders);
    const int row = d & (kTileN - 1), r4 = d >> 7;
    const uint32_t base_e = tab | (static_cast<uint32_t>(lane & 15) << 3), base_o = base_e + 128u;
    const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + kTmemA + 16u * r4;
    bool ok = true;
    int kb = 0;  // blocks whose store has been issued
    uint32_t hv[16];
    // the previous block's store has landed: hand its stage to the MMA (one arrival
    // per warp: 512 single-thread arrivals on one barrier cost about a microsecond)
    auto publish_prev = [&]() {
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(fullA + 8 * ((kb - 1) % kStagesTC));
    };
    // store block kb once the MMA has released its stage; completes during the next decode
    auto store = [&]() {
      const int s = kb % kStagesTC;
      if (ok) ok = mbar_wait(emptyA + 8 * s, (static_cast<uint32_t>(kb / kStagesTC) & 1) ^ 1, a.fault,
                             kFaultDecode);
      __syncwarp();  // tcgen05.st is warp-collective
      tc_fence_after_sync();
      tmem_st16(tlane + 64u * s, hv);
      ++kb;
    };
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
      const int r = c % kRawStages;
      if (ok) ok = mbar_wait(fullR + 8 * r, static_cast<uint32_t>(c / kRawStages) & 1, a.fault, kFaultDecode);
      uint4 raw[7] = {};
      // word w of this row: group row >> 2, element 4 w + (row & 3) of the group; only
      // the words this thread's quarter decodes are read (r4 is warp-uniform)
      const uint32_t src = rawring + r * kRawStageBytes +
                           4u * (static_cast<uint32_t>(row >> 2) * kGroupWords + (row & 3));
      switch (r4) {
        case 0: load_quarter_words<0>(raw, src); break;
        case 1: load_quarter_words<1>(raw, src); break;
        case 2: load_quarter_words<2>(raw, src); break;
        default: load_quarter_words<3>(raw, src); break;
      }
      __syncwarp();  // the warp's reads of the chunk are done (mbarrier arrive releases them)
      if (lane == 0) mbar_arrive(emptyR + 8 * r);
      decode_quarter<0>(raw, r4, base_e, base_o, hv);
      if (kb > 0) publish_prev();
      store();
      if (kb < nkb) {
        decode_quarter<1>(raw, r4, base_e, base_o, hv);
        publish_prev();
        store();
      }
      if (kb < nkb) {
        decode_quarter<2>(raw, r4, base_e, base_o, hv);
        publish_prev();
        store();
      }
      if (kb < nkb) {
        decode_quarter<3>(raw, r4, base_e, base_o, hv);
        publish_prev();
        store();
      }
    }
    if (kb > 0) publish_prev();

    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its rows);
    // the four warp groups take turns at 16-column chunks
    if (ok) ok = mbar_wait(accum, 0, a.fault, kFaultEpilogue);
    tc_fence_after_sync();
    const int q = warp & 3, grp = (warp - 4) >> 2;
    const int64_t ne = n0 + 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    // every accumulator received at least one MMA: K >= 128 gives 8 per block
    const int nacc_used = a.nacc < 8 * nkb ? a.nacc : 8 * nkb;
    if (a.y_tma) {
      // bf16 tile [tokens][128 rows] staged in shared memory (the activation slabs are
      // free once the accumulator is complete), then one TMA store; the tokens'
      // exponents first go to shared memory (below the table, where slab 0 was)
      const uint32_t ot = tab + kHighB;
      int* xe = reinterpret_cast<int*>(smem_raw + (bstage0 - sraw));
      int* xf = xe + kMaxTileM;  // the tokens' flags (rows recomputed on the CUDA cores)
      bool flagged = false;
      for (int t = tid - 128; t < a.tile_m; t += kDecoders) {
        xe[t] = m0 + t < a.M ? a.xexp[m0 + t] : 0;
        xf[t] = m0 + t < a.M ? a.xflag[m0 + t] : 0;
        flagged = flagged || xf[t] != 0;
      }
      flagged = named_bar_or(3, kDecoders, flagged);  // any flagged token in this tile
      const int rloc = 32 * q + lane;
      for (int c0 = 16 * grp; c0 < a.tile_m; c0 += 64) {
        uint32_t v[16];
        tmem_ld16(lane_base + static_cast<uint32_t>(c0), v);
        tmem_ld_wait();
        for (int j = 1; j < nacc_used; ++j) {  // accumulators summed in order
          uint32_t u[16];
          tmem_ld16(lane_base + static_cast<uint32_t>(j * a.tile_m + c0), u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(u[i]));
        }
        // the 16 tokens' exponents first (four 16-byte loads), then the 16 conversions,
        // then the stores: interleaved, each store's memory clobber held the next
        // exponent load behind it
        int ex[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const int4 e4 = *reinterpret_cast<const int4*>(xe + c0 + i);
          ex[i] = e4.x;
          ex[i + 1] = e4.y;
          ex[i + 2] = e4.z;
          ex[i + 3] = e4.w;
        }
        // undo the activation rows' power-of-two scaling (exact): a multiply by 2^e
        // unless some exponent of the chunk is outside fp32's normal range (a branch
        // on the whole chunk: per element, the compiler evaluated ldexpf every time)
        bool normal = true;
#pragma unroll
        for (int i = 0; i < 16; ++i) normal = normal && ex[i] >= -126 && ex[i] <= 127;
        uint16_t h[16];
        if (normal) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            h[i] = f32_to_bf16_bits(__uint_as_float(v[i]) * __int_as_float((ex[i] + 127) << 23));
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = f32_to_bf16_bits(ldexpf(__uint_as_float(v[i]), ex[i]));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t addr = ot + static_cast<uint32_t>((c0 + i) * 256 + rloc * 2);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(h[i]) : "memory");
        }
      }
      // flagged tokens: their staged outputs are replaced by the exact recomputation
      if (flagged) {
        named_bar_sync(3, kDecoders);
        fixup_flagged(a, n0, m0, kb0, nkb, xf, reinterpret_cast<float*>(xf + kMaxTileM), tid - 128,
                      [&](int t, int rrow, float v) {
                        const uint32_t addr = ot + static_cast<uint32_t>(t * 256 + rrow * 2);
                        asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(f32_to_bf16_bits(v)) : "memory");
                      });
      }
      fence_proxy_async_smem();  // the generic-proxy writes, before the TMA reads them
      named_bar_sync(3, kDecoders);
      if (tid == 128 && ok) {
        tma_store_2d(&tm_y, ot, static_cast<int32_t>(n0), static_cast<int32_t>(m0));
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    } else {
      // the tile's flagged tokens (flags and scratch in the free activation slab 0)
      int* xf = reinterpret_cast<int*>(smem_raw + (bstage0 - sraw));
      bool flagged = false;
      for (int t = tid - 128; t < a.tile_m; t += kDecoders) {
        xf[t] = m0 + t < a.M ? a.xflag[m0 + t] : 0;
        flagged = flagged || xf[t] != 0;
      }
      flagged = named_bar_or(3, kDecoders, flagged);
      for (int c0 = 16 * grp; c0 < a.tile_m; c0 += 64) {
        uint32_t v[16];
        tmem_ld16(lane_base + static_cast<uint32_t>(c0), v);
        tmem_ld_wait();
        for (int j = 1; j < nacc_used; ++j) {  // accumulators summed in order
          uint32_t u[16];
          tmem_ld16(lane_base + static_cast<uint32_t>(j * a.tile_m + c0), u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(u[i]));
        }
        if (!ok || ne >= a.N) continue;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int64_t m = m0 + c0 + i;
          if (m < a.M && !(flagged && a.xflag[m])) {  // flagged tokens: written by the fixup below
            // undo the activation row's power-of-two scaling (exact)
            const float y = scale_pow2(__uint_as_float(v[i]), a.xexp[m]);
            if (a.part)
              a.part[(static_cast<int64_t>(blockIdx.z) * a.M + m) * a.N + ne] = y;
            else
              a.Y[m * a.N + ne] = f32_to_bf16_bits(y);
          }
        }
      }
      if (flagged) {
        named_bar_sync(3, kDecoders);
        fixup_flagged(a, n0, m0, kb0, nkb, xf, reinterpret_cast<float*>(xf + kMaxTileM), tid - 128,
                      [&](int t, int rrow, float v) {
                        if (!ok) return;
                        const int64_t m = m0 + t, n = n0 + rrow;
                        if (a.part)
                          a.part[(static_cast<int64_t>(blockIdx.z) * a.M + m) * a.N + n] = v;
                        else
                          a.Y[m * a.N + n] = f32_to_bf16_bits(v);
                      });
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
// A bf16 value lands in fp16 exactly unless it sits more than about 2^31 below the
// row's largest (fp16's subnormal step is then coarser than its last bit); a row with
// any such value is flagged (xflag[m] = 1) and the product recomputes its outputs
// on the CUDA cores, so every row meets the same bound whatever its spread.
__global__ void __launch_bounds__(256) x_to_f16_kernel(const uint16_t* __restrict__ X, int64_t K,
                                                        uint16_t* __restrict__ Xh,
                                                        int* __restrict__ xexp,
                                                        int* __restrict__ xflag) {
  __shared__ float red[8];
  const int64_t m = blockIdx.x;
  // 16-byte accesses: 8 values a thread (K is a multiple of 128, rows 16-byte aligned)
  const uint4* xr = reinterpret_cast<const uint4*>(X + m * K);
  uint4* hr = reinterpret_cast<uint4*>(Xh + m * K);
  const int64_t K8 = K / 8;
  auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
  auto hi = [](uint32_t w) { return __uint_as_float(w & 0xffff0000u); };
  float mx = 0.0f;
  for (int64_t k = threadIdx.x; k < K8; k += blockDim.x) {
    const uint4 v = xr[k];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) mx = fmaxf(mx, fmaxf(fabsf(lo(w[q])), fabsf(hi(w[q]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) mx = fmaxf(mx, red[i]);
  const int e = mx > 0.0f ? ilogbf(mx) - 14 : 0;  // floor(log2(max|x|)) - 14
  // x * 2^-e to fp16: a multiply by the power of two when it is a normal float (exact,
  // as ldexpf), ldexpf otherwise
  // (two loops: a select per element had the compiler evaluate ldexpf every time)
  // (an inexact conversion sets `inexact`: the value does not come back from fp16)
  bool inexact = false;
  auto pack = [&inexact](float a0, float a1) {
    const __half h0 = __float2half_rn(a0), h1 = __float2half_rn(a1);
    inexact = inexact || __half2float(h0) != a0 || __half2float(h1) != a1;
    return static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
  };
  if (-e >= -126 && -e <= 127) {
    const float f = __int_as_float((127 - e) << 23);
    for (int64_t k = threadIdx.x; k < K8; k += blockDim.x) {
      const uint4 v = xr[k];
      hr[k] = make_uint4(pack(lo(v.x) * f, hi(v.x) * f), pack(lo(v.y) * f, hi(v.y) * f),
                         pack(lo(v.z) * f, hi(v.z) * f), pack(lo(v.w) * f, hi(v.w) * f));
    }
  } else {
    for (int64_t k = threadIdx.x; k < K8; k += blockDim.x) {
      const uint4 v = xr[k];
      auto sc = [&](float x) { return ldexpf(x, -e); };
      hr[k] = make_uint4(pack(sc(lo(v.x)), sc(hi(v.x))), pack(sc(lo(v.y)), sc(hi(v.y))),
                         pack(sc(lo(v.z)), sc(hi(v.z))), pack(sc(lo(v.w)), sc(hi(v.w))));
    }
  }
  const int any = __syncthreads_or(inexact ? 1 : 0);
  if (threadIdx.x == 0) {
    xexp[m] = e;
    xflag[m] = any ? 1 : 0;
  }
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
  const int64_t ntiles = (w->N + kTileN - 1) / kTileN;
  if (M >= 128 && ntiles * ((M + kMaxTileM - 1) / kMaxTileM) >= 3 * sm_count()) {
    p.tile_m = kMaxTileM;  // many waves of full-width tiles: the tail matters little
  } else if (M >= 128) {
    // Few waves: choose the token tile (a multiple of 16, 128..256) that minimises the
    // modelled time: waves of CTAs x (the tile's MMA time, which stops shrinking below
    // ~160 tokens because an MMA then waits on the previous one, + a fixed cost per tile).
    int64_t best = -1;
    for (int t = 128; t <= kMaxTileM; t += 16) {
      const int64_t tiles = ntiles * ((M + t - 1) / t);
      const int64_t waves = (tiles + sm_count() - 1) / sm_count();
      const int64_t cost = waves * ((t > 160 ? t : 160) + 32);
      if (best < 0 || cost < best || (cost == best && t > p.tile_m)) {
        best = cost;
        p.tile_m = t;
      }
    }
  } else {
    p.tile_m = static_cast<int>((M + 15) / 16 * 16);
  }
  const int64_t tiles = ntiles * ((M + p.tile_m - 1) / p.tile_m);
  const int nkb = static_cast<int>(w->K / kTileK);
  const int nchunks = (nkb + kChunkBlocks - 1) / kChunkBlocks;
  int splits = 1;
  if (tiles < sm_count()) splits = static_cast<int>(sm_count() / tiles);
  if (splits > nchunks) splits = nchunks;
  if (splits < 1) splits = 1;
  // whole chunks per split: a weight copy never straddles two splits
  p.kb_per_split = (nchunks + splits - 1) / splits * kChunkBlocks;
  p.splits = (nkb + p.kb_per_split - 1) / p.kb_per_split;
  return p;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

// Workspace of the ternary tensor-core product:
// [64 KB reserved][fp16 X: M*K][exponents: M][flags: M][fp32 partials: splits*M*N when split].
size_t lbq_gemm_tc_workspace(const lbq_weights* w, int64_t M) {
  const TcPlan p = plan_for(w, M);
  size_t n = kWsCounterBytes + align_up(static_cast<size_t>(M) * w->K * 2, 1024) +
             2 * align_up(static_cast<size_t>(M) * sizeof(int), 256);
  if (p.splits > 1) n += static_cast<size_t>(p.splits) * M * w->N * sizeof(float);
  return n;
}

cudaError_t lbq_launch_gemm_tc(const lbq_weights* w, const uint16_t* X, int64_t M, uint16_t* Y,
                               void* ws, cudaStream_t s) {
  static PerDevice<bool> configured;  // the kernel's shared-memory limit, set once per device
  bool done = false;
  cudaError_t ce = configured.get(
      [](int, bool* v) {
        *v = true;
        return cudaFuncSetAttribute(gemm_tern_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kSmemTC));
      },
      &done);
  if (ce != cudaSuccess) return ce;
  char* base = static_cast<char*>(ws) + kWsCounterBytes;
  uint16_t* Xh = reinterpret_cast<uint16_t*>(base);
  int* xexp = reinterpret_cast<int*>(base + align_up(static_cast<size_t>(M) * w->K * 2, 1024));
  int* xflag = reinterpret_cast<int*>(reinterpret_cast<char*>(xexp) +
                                      align_up(static_cast<size_t>(M) * sizeof(int), 256));
  x_to_f16_kernel<<<static_cast<unsigned>(M), 256, 0, s>>>(X, w->K, Xh, xexp, xflag);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  TcArgs a;
  a.K = w->K;
  a.N = w->N;
  a.M = M;
  a.xexp = xexp;
  a.xflag = xflag;
  a.X = X;
  a.codes = static_cast<const uint8_t*>(w->codes);
  a.code_stride = w->code_stride;
  a.Y = Y;
  const TcPlan plan = plan_for(w, M);
  a.tile_m = plan.tile_m;
  a.nacc = 1;
  while (a.nacc < 8 && 2 * a.nacc * a.tile_m <= static_cast<int>(kAccCols)) a.nacc *= 2;
  a.kb_per_split = plan.kb_per_split;
  a.part = plan.splits > 1
               ? reinterpret_cast<float*>(reinterpret_cast<char*>(xflag) +
                                          align_up(static_cast<size_t>(M) * sizeof(int), 256))
               : nullptr;
  a.fault = lbq_fault_word();
  if (!a.fault) return cudaErrorInvalidDevicePointer;

  auto fn = tensor_map_encoder();
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
  // packed weights as 32-bit words, one row of the map per group of four rows
  // (code_stride words); boxes of 116 words x 32 groups; groups past the end and
  // words past the row read as zero
  CUtensorMap tw;
  const cuuint64_t wdims[2] = {static_cast<cuuint64_t>(w->code_stride),
                               static_cast<cuuint64_t>((w->N + 3) / 4)};
  const cuuint64_t wstrides[1] = {static_cast<cuuint64_t>(w->code_stride) * 4};
  const cuuint32_t wbox[2] = {kGroupWords, static_cast<cuuint32_t>(kTileN / 4)};
  if (fn(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(w->codes), wdims, wstrides, wbox, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // Y through shared memory and one TMA store per tile when the tensor map can
  // describe it (16-byte aligned base and row pitch) and K is not split
  CUtensorMap ty;
  a.y_tma = 0;
  if (!a.part && (reinterpret_cast<uintptr_t>(Y) & 15) == 0 && (w->N * 2) % 16 == 0) {
    const cuuint64_t ydims[2] = {static_cast<cuuint64_t>(w->N), static_cast<cuuint64_t>(M)};
    const cuuint64_t ystrides[1] = {static_cast<cuuint64_t>(w->N) * 2};
    const cuuint32_t ybox[2] = {static_cast<cuuint32_t>(kTileN), static_cast<cuuint32_t>(a.tile_m)};
    if (fn(&ty, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, Y, ydims, ystrides, ybox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      a.y_tma = 1;
  }
  if (!a.y_tma) ty = tw;  // unused
  dim3 grid(static_cast<unsigned>((w->N + kTileN - 1) / kTileN),
            static_cast<unsigned>((M + a.tile_m - 1) / a.tile_m), static_cast<unsigned>(plan.splits));
  gemm_tern_tc_kernel<<<grid, kThreadsTC, kSmemTC, s>>>(tm, tw, ty, a);
  e = cudaGetLastError();
  if (e != cudaSuccess || plan.splits == 1) return e;
  const int64_t MN = M * w->N;
  gemm_split_sum_kernel<<<static_cast<unsigned>((MN + 255) / 256), 256, 0, s>>>(a.part, plan.splits, MN, Y);
  return cudaGetLastError();
}
