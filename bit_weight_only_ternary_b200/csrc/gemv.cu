// gemv.cu -- batch-1 low-bit GEMV, y = W_hat x (bf16 in, fp32 accumulate, bf16 out).
//
// Ternary products reduce to adding, subtracting or skipping activations (pptc.cn
// ternary-27B article §1.2; mhpq.cn "27B in 5.9 GB" article §2.2) and each block's
// sum is scaled by its fp16 scale (mhpq.cn §2.1). The 1-bit format is the Q1_0 case
// of the neodrop.ai round-up (part 2); the 2-bit format multiplies the rotated
// input x' = H D x / sqrt(512) of the feinterview.poetries.top "27B in 12 GB"
// article, computed here in shared memory, never in global memory.
//
// Design (HBM-bound: about one issued instruction per weight is all there is):
//  * Lookup of partial sums. A CTA owns one K-slice (ternary: 4 blocks, 512
//    weights, 28 words of a row; 1-bit: 1024 weights, 32 words; 2-bit: 512
//    weights, 32 words) and builds in shared memory, for every byte position of the
//    slice, the partial dot product of that byte's codes with the slice of x, for
//    all 256 byte values (128 KB). A byte then costs one PRMT (which forms the
//    table address from the byte and the lane), one LDS and one add. Lane l always
//    handles the same word position of a row, and the table is laid out
//    [value][lane], so table reads never collide on a bank.
//  * Streaming. The packed rows are stored in groups of four (word w of four rows
//    in 16 consecutive bytes), so a 16-row unit's slice is four runs of 448
//    (ternary) or 512 bytes. One warp issues tensor copies (TMA) of four units at
//    a time (7 to 10 KB) into a ring of shared-memory slots; the 16 compute warps
//    take one unit each and read their lane's word of four rows with one 16-byte
//    shared load per group. (Per-unit copies, 1.8 KB each, streamed at half the
//    rate: the copy engine keeps few copies in flight. Eight-unit ternary copies
//    measured the same as four-unit ones over a 16-layer pass. Loads into registers
//    instead queue in the L1 path ahead of the x slice and the table build.)
//  * Reduction. Each lane holds one word's partial sum for each of 16 rows; a
//    transpose-reduce butterfly (16 shuffles) leaves row l's slice sum in lane l.
//    (Rotating the group order per lane would spare the selects of two stages, but
//    a warp load then touches four groups instead of one, and the extra sectors
//    cost more than the selects: measured.)
//  * Scales. Ternary scales live in word 6 of each 28-byte block: lanes are mapped
//    so that block b is lanes 8b .. 8b+6, and lane 8b+6 hands each pair of rows'
//    scales to its block's lanes with one shuffle. 1-bit and 2-bit scales come in
//    the same tensor copies as the codes (group-of-four scale order): one 8-byte
//    shared load per lane per four rows.
//  * Split-K. Slices are spread over CTAs; slice sums go to the workspace and a
//    small second kernel adds each row's slice sums in a fixed order and writes bf16
//    y: results are deterministic. (Folding that sum into the main kernel, by the
//    last CTA of a row range or after a meeting of the range's CTAs, measured slower:
//    the tail of L2 round trips then runs on a handful of SMs. So did starting the
//    sum of a row range as soon as its CTAs had counted themselves in.)
//  * Programmatic dependent launch: the copy warp never waits for the previous
//    kernel, so its first copies (one slot per warp group) land while it finishes;
//    the other slots are filled once the table is built (their shared-memory writes
//    slowed the build down). Only the batch-1 kernels let their successor start
//    early, and they never write packed weights; any other kernel has completed
//    before this one starts. x, y and the workspace are touched only after the wait.
#include <type_traits>

#include "lut.cuh"
#include "sm100_async.cuh"

namespace {

using namespace lbq;
using namespace lbq::lut;

constexpr int kWarps = 16;                    // consumer warps
constexpr int kThreads = 32 * kWarps;         // consumer threads
constexpr int kBlockThreads = kThreads + 32;  // + the copy-issuing warp
constexpr int kRows = 16;                     // rows per unit (four groups of four)
constexpr int kSub = 4;                       // units per ring slot (one tensor copy)
// Shared memory: the 128 KB table at the first 64 KB boundary of the window (its
// page addressing keeps the base in the upper half of the PRMT operand); below it
// (the dynamic window starts 1 KB into shared memory on sm_100) the x slice, the
// mbarriers and the first ring slots, above it the other ring slots. A window that
// starts at 0 puts everything above the table.
constexpr uint32_t kXBytes = lut::kXsBytes;  // the padded slice of x as fp32
constexpr int kMaxSlots = 32;
// x and the mbarriers, rounded up so that the ring slots after them stay 128-byte
// aligned, as tensor copies into shared memory require
constexpr uint32_t kMisc = (kXBytes + 2 * 8 * kMaxSlots + 8 + 1023) & ~1023u;
// 225 KB: with the 1 KB every CTA reserves, a CTA of the split-K sum kernel still
// fits beside this one in the SM's 228 KB.
constexpr uint32_t kSmem = 225 * 1024;
constexpr unsigned kFaultLayout = 3, kFaultRing = 10;

using lut::Traits;
using lut::kPage;
// A ring slot: kSub 16-row units of a slice, codes first, then scales.
template <int FMT>
constexpr uint32_t kSlotBytes = 4 * kSub * (Traits<FMT>::kGroupBytes + Traits<FMT>::kScaleBytes);

template <int FMT>
// The packed weights reach the kernel as tensor maps (see the launch).
struct Args {
  int64_t K, N;
  const uint16_t* x;
  const int8_t* D;
  uint16_t* y;
  float* y32;       // if set, y is written here as fp32 (no bf16 rounding) instead
  float* part;      // [KS][N] slice sums (KS > 1)
  int KS;           // number of slices
  int G;            // CTAs per slice
  int nblk;         // scale blocks per row
  unsigned* fault;  // the device fault word (layout check, bounded waits)
};

// One CTA: kWarps consumer warps and one warp that issues the weight copies. At most
// 96 registers a thread: the register file is split between the SM's four schedulers,
// and the CTA's 17 warps put five on one of them (5 x 32 x 96 = 15360 of its 16384,
// which also leaves room for a warp of the split-K sum kernel at 32 registers).
// tm_c / tm_s: the codes / scales as tensor maps with a box of kSub units (tm_c1 /
// tm_s1: one unit).
template <int FMT>
__global__ void __maxnreg__(96) gemv_lut_kernel(const __grid_constant__ CUtensorMap tm_c,
                                                 const __grid_constant__ CUtensorMap tm_s,
                                                 const __grid_constant__ CUtensorMap tm_c1,
                                                 const __grid_constant__ CUtensorMap tm_s1,
                                                 const Args<FMT> a) {
  using T = Traits<FMT>;
  constexpr bool kSepScales = FMT != LBQ_TERN5;
  constexpr uint32_t kScaleOff = 4 * kSub * T::kGroupBytes;  // scales within a slot
  static_assert(kWarps % kSub == 0, "whole warp groups");
  static_assert(kSlotBytes<FMT> % 128 == 0 && kScaleOff % 128 == 0 && (4 * T::kGroupBytes) % 128 == 0 &&
                    (4 * T::kScaleBytes) % 128 == 0,
                "tensor copies land on 128-byte boundaries");
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---- shared-memory layout (see the constants)
  const uint32_t sbase = smem_u32(smem);
  const uint32_t send = sbase + kSmem;
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  const uint32_t ttop = tbase + 2 * kPage;
  const bool misc_low = tbase - sbase >= kMisc;
  const uint32_t misc = misc_low ? sbase : ttop;
  const uint32_t lo0 = misc_low ? sbase + kMisc : sbase;  // ring slots below the table
  const uint32_t hi0 = misc_low ? ttop : ttop + kMisc;    // ... and above it
  const int s_lo = static_cast<int>((tbase - lo0) / kSlotBytes<FMT>);
  const int s_hi = hi0 < send ? static_cast<int>((send - hi0) / kSlotBytes<FMT>) : 0;
  // The slot count is a multiple of the kWarps / kSub warp groups: unit sequence
  // number q goes to slot q % S and is taken by group q % (kWarps / kSub), so every
  // slot belongs to one group, which waits for a slot's next fill only after taking
  // the previous one (an mbarrier parity wait never looks two phases ahead).
  constexpr int kGroups = kWarps / kSub;
  const int S = (s_lo + s_hi < kMaxSlots ? s_lo + s_hi : kMaxSlots) / kGroups * kGroups;
  if (ttop > send || misc + kMisc > send || S < 2 * kGroups || ((lo0 | hi0) & 127) != 0) {
    if (tid == 0) atomicExch(a.fault, kFaultLayout);  // cannot happen with a 0 or 1 KB prefix
    return;
  }
  float* xs = reinterpret_cast<float*>(smem + (misc - sbase));
  const uint32_t full0 = misc + kXBytes, empty0 = full0 + 8 * kMaxSlots;
  const uint32_t built = empty0 + 8 * kMaxSlots;  // the table is built (inside kMisc)
  auto slot_addr = [&](int s) {
    return s < s_lo ? lo0 + static_cast<uint32_t>(s) * kSlotBytes<FMT>
                    : hi0 + static_cast<uint32_t>(s - s_lo) * kSlotBytes<FMT>;
  };
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kSub);
    }
    mbar_init(built, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // This CTA: slice j, units [u_lo, u_hi) of kRows rows (a.G CTAs share a slice).
  // 32-bit arithmetic: NU <= 2^15 and G <= the SM count.
  const int32_t NU = static_cast<int32_t>((a.N + kRows - 1) / kRows);
  const int32_t j = static_cast<int32_t>(blockIdx.x) / a.G;
  const int32_t gs = static_cast<int32_t>(blockIdx.x) - j * a.G;
  const int32_t u_lo = static_cast<int32_t>(static_cast<uint32_t>(gs * NU) / static_cast<uint32_t>(a.G));
  const int32_t u_hi =
      static_cast<int32_t>(static_cast<uint32_t>((gs + 1) * NU) / static_cast<uint32_t>(a.G));
  const int32_t n_units = u_hi - u_lo;
  const int blk0 = j * T::kBlocks;
  const int nb = a.nblk - blk0 < T::kBlocks ? a.nblk - blk0 : T::kBlocks;

  if (warp == kWarps) {
    // ---- copies: slot sequence number q holds units kSub q .. kSub q + kSub - 1 of
    // this CTA and goes to slot q % S; one tensor copy of their groups' slice (groups
    // past the last read as zero) and one of their scales; a last, partial slot gets
    // one copy per unit. The packed weights are never written by a kernel that lets
    // this one start early (only the batch-1 kernels do, and they do not write
    // weights), so the copies do not wait for the previous kernel: the ring fills
    // while it finishes.
    if (lane == 0) {
      prefetch_tmap(&tm_c);
      prefetch_tmap(&tm_c1);
      if (kSepScales) {
        prefetch_tmap(&tm_s);
        prefetch_tmap(&tm_s1);
      }
      const int32_t cx = j * 4 * T::kWords, sx = 4 * blk0;
      const int32_t nslots = (n_units + kSub - 1) / kSub;
      int slot = 0;
      uint32_t round = 0;
      int32_t issued = 0;
      for (int32_t q = 0; q < nslots; ++q) {
        const uint32_t full = full0 + 8 * slot;
        if (round > 0 && !mbar_wait(empty0 + 8 * slot, (round - 1) & 1, a.fault, kFaultRing)) break;
        // one slot per warp group up front; the rest once the table is built, so that
        // their shared-memory writes do not slow the build down
        if (q == kGroups && !mbar_wait(built, 0, a.fault, kFaultRing)) break;
        ++issued;
        const uint32_t dst = slot_addr(slot);
        const int32_t u0 = kSub * q;
        const int32_t nu = n_units - u0 < kSub ? n_units - u0 : kSub;
        const int32_t g0 = 4 * (u_lo + u0);
        mbar_arrive_expect_tx(full, static_cast<uint32_t>(nu) * 4 * (T::kGroupBytes + T::kScaleBytes));
        if (nu == kSub) {
          tma_load_2d(dst, &tm_c, cx, g0, full);
          if (kSepScales) tma_load_2d(dst + kScaleOff, &tm_s, sx, g0, full);
        } else {
          for (int32_t i = 0; i < nu; ++i) {
            tma_load_2d(dst + i * 4 * T::kGroupBytes, &tm_c1, cx, g0 + 4 * i, full);
            if (kSepScales)
              tma_load_2d(dst + kScaleOff + i * 4 * T::kScaleBytes, &tm_s1, sx, g0 + 4 * i, full);
          }
        }
        if (++slot == S) {
          slot = 0;
          ++round;
        }
      }
      // Every issued copy lands before the CTA can exit (after a fault the consumers
      // may have stopped taking them): the last fill of each slot, bounded.
      for (int32_t q = issued - S > 0 ? issued - S : 0; q < issued; ++q)
        mbar_wait(full0 + 8 * (q % S), static_cast<uint32_t>(q / S) & 1, a.fault, kFaultRing,
                  /*give_up_after_fault=*/false);
    }
    return;  // the consumers synchronise among themselves from here on
  }

  // ... and the x slice, which the previous kernel of a chain of products may write:
  // a prefetch into L2 is only a hint and cannot return stale data
  if (tid >= 480 && tid - 480 < T::kWeights / 64) {
    const int64_t k = static_cast<int64_t>(j) * T::kWeights + 64 * (tid - 480);
    if (k + 64 <= a.K) prefetch_l2_bulk(a.x + k, 128);
    if (FMT == LBQ_Q2RHT && tid - 480 < T::kWeights / 128)
      prefetch_l2_bulk(a.D + static_cast<int64_t>(j) * T::kWeights + 128 * (tid - 480), 128);
  }

  pdl_wait();  // x, y and the workspace may belong to the previous kernel until here
  x_store<FMT>(x_issue<FMT>(a.x, a.D, a.nblk, j, tid), xs, tid);
  named_bar_sync(1, kThreads);
  build_table<FMT, kThreads>(nb, tbase, xs, tid);
  named_bar_sync(1, kThreads);
  if (tid == 0) mbar_arrive(built);

  // This lane's word of each group, and (1-bit, 2-bit) its block's scales of four
  // rows. Lanes without a word (their table columns are zero) read the word of the
  // first lane of their quarter-warp, which the shared-memory unit then serves in
  // the same wavefront (word 0 would collide with another lane's banks), and the
  // slice's first block.
  const int wl = lane_word<FMT>(lane, nb);
  const int wq = lane_word<FMT>(lane & ~7, nb);
  const uint32_t woff = 16u * static_cast<uint32_t>(wl >= 0 ? wl : (wq >= 0 ? wq : 0));
  const uint32_t lanereg = tbase | static_cast<uint32_t>(lane * 4);
  // The block scales this lane multiplies after the in-block butterfly stages
  // (unit_sum): ternary, the scale words of rows R, R + 1 of its block (word 6 of the
  // block, inside the codes); 1-bit, group G's four scales of its block; 2-bit, groups
  // G and G + 1's. Offsets within a unit's codes / scales in the ring slot.
  uint32_t s_off;
  if (FMT == LBQ_TERN5) {
    const int R = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1);
    const int b = (lane >> 3) < nb ? (lane >> 3) : nb - 1;
    s_off = static_cast<uint32_t>((R >> 2) * T::kGroupBytes + 16 * (7 * b + 6) + 4 * (R & 3));
  } else {
    const int b = FMT == LBQ_SIGN1 ? (lane >> 2) : (lane >> 1);
    const int bb = b < nb ? b : nb - 1;
    const int G = FMT == LBQ_SIGN1 ? 2 * (lane & 1) + ((lane >> 1) & 1) : 2 * (lane & 1);
    s_off = kScaleOff + static_cast<uint32_t>(G * T::kScaleBytes + 8 * bb);
  }
  // the row unit_sum leaves in this lane (lanes < 16 store it)
  const int rloc = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 3) & 1);
  const int64_t NR = a.N;
  float* const part_j = a.part + static_cast<int64_t>(j) * NR;
  uint16_t* const y = a.y;
  const bool direct = a.KS == 1;
  // ---- consumers: warp w takes units w, w + kWarps, ...; unit tg sits in slot
  // sequence number tg / kSub at place tg % kSub (= w % kSub)
  const uint32_t sub = static_cast<uint32_t>(warp % kSub);
  const int32_t nt = n_units > warp ? (n_units - warp + kWarps - 1) / kWarps : 0;
  int slot = warp / kSub;
  uint32_t round = 0;
  for (int32_t t = 0; t < nt; ++t) {
    if (!mbar_wait(full0 + 8 * slot, round & 1, a.fault, kFaultRing)) break;
    const uint32_t src = slot_addr(slot);
    UnitRegs r;
#pragma unroll
    for (int q = 0; q < 4; ++q) r.w[q] = lds_v4(src + (4 * sub + q) * T::kGroupBytes + woff);
    if (FMT == LBQ_TERN5) {
      r.s[0] = lds_v2(src + 4 * sub * T::kGroupBytes + s_off);
    } else {
      r.s[0] = lds_v2(src + 4 * sub * T::kScaleBytes + s_off);
      if (FMT == LBQ_Q2RHT) r.s[1] = lds_v2(src + (4 * sub + 1) * T::kScaleBytes + s_off);
    }
    // The warp has its words: the slot goes back to the copies (the warp barrier and
    // the proxy fence order these reads before the copy engine's next writes).
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive(empty0 + 8 * slot);
    }
    const float v = unit_sum<FMT>(r, lanereg, lane);
    const int64_t row = static_cast<int64_t>(u_lo + warp + kWarps * t) * kRows + rloc;
    if (lane < kRows && row < NR) {
      if (!direct)
        part_j[row] = v;
      else if (a.y32)
        a.y32[row] = v;
      else
        y[row] = f32_to_bf16_bits(v);
    }
    slot += kGroups;
    if (slot >= S) {
      slot -= S;
      ++round;
    }
  }
  // The split-K sum kernel may start once every CTA is past its units (the copy warp
  // has left already): its CTAs then sit beside the last ones for a short wait only.
  pdl_launch_dependents();
}

// Sums the slice sums of every row and writes bf16 y, launched right after the main
// kernel (in plain stream order, see the launch). The tail is bound by L2 round
// trips, so every load of a
// thread is issued before its adds: a thread takes a pair of rows (one row when N
// is odd, where pairs would be misaligned) and a run of at most kSumRun slices; the
// P threads of a row (consecutive lanes) then combine their runs in a fixed tree
// order, so results are deterministic.
constexpr int kSumThreads = 128, kSumRun = 8;
template <bool kPairs>
__global__ void __maxnreg__(32)
    splitk_sum_kernel(const float* __restrict__ part, int KS, int64_t N, int logP,
                      uint16_t* __restrict__ y, float* __restrict__ y32) {
  pdl_launch_dependents();
  pdl_wait();
  using V = typename std::conditional<kPairs, float2, float>::type;
  const int P = 1 << logP;
  const int run = (KS + P - 1) >> logP;
  const int64_t nv = kPairs ? N / 2 : N;  // pairs (or rows) per slice
  const int64_t total = nv << logP;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kSumThreads;
  // warp-uniform trip count: every lane of a CTA runs the same iterations
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kSumThreads; base < total; base += stride) {
    const int64_t idx = base + threadIdx.x;
    const int64_t e = idx >> logP;
    const int sg = static_cast<int>(idx & (P - 1));
    const int j0 = sg * run;
    const int j1 = min(j0 + run, KS);
    float ax = 0.0f, ay = 0.0f;
    if (idx < total) {
      const V* p = reinterpret_cast<const V*>(part) + e;
      V v[kSumRun];
#pragma unroll
      for (int q = 0; q < kSumRun; ++q) {
        if (j0 + q < j1) {
          v[q] = __ldcg(p + (j0 + q) * nv);
        } else {
          v[q] = V{};
        }
      }
#pragma unroll
      for (int q = 0; q < kSumRun; ++q)
        if (j0 + q < j1) {
          if constexpr (kPairs) {
            ax += v[q].x;
            ay += v[q].y;
          } else {
            ax += v[q];
          }
        }
    }
    for (int o = P >> 1; o >= 1; o >>= 1) {
      ax += __shfl_down_sync(0xffffffffu, ax, o, P);
      if (kPairs) ay += __shfl_down_sync(0xffffffffu, ay, o, P);
    }
    if (idx < total && sg == 0) {
      if (y32) {
        if (kPairs) {
          y32[2 * e] = ax;
          y32[2 * e + 1] = ay;
        } else {
          y32[e] = ax;
        }
      } else if (kPairs) {
        y[2 * e] = f32_to_bf16_bits(ax);
        y[2 * e + 1] = f32_to_bf16_bits(ay);
      } else {
        y[e] = f32_to_bf16_bits(ax);
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

template <int FMT>
cudaError_t launch(const lbq_weights* w, const uint16_t* x, const int8_t* D, uint16_t* y, float* y32, void* ws,
                   cudaStream_t s) {
  static PerDevice<bool> configured;  // the kernel's shared-memory limit, set once per device
  bool ok = false;
  cudaError_t ce = configured.get(
      [](int, bool* v) {
        *v = true;
        return cudaFuncSetAttribute(gemv_lut_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kSmem));
      },
      &ok);
  if (ce != cudaSuccess) return ce;
  Args<FMT> a;
  a.K = w->K;
  a.N = w->N;
  a.x = x;
  a.D = D;
  a.y = y;
  a.y32 = y32;
  a.KS = slices_of(w);
  a.nblk = static_cast<int>(w->K / (FMT == LBQ_Q2RHT ? kQ2Block : kTernBlock));
  a.fault = lbq_fault_word();
  if (!a.fault) return cudaErrorInvalidDevicePointer;
  a.part = ws ? reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes) : nullptr;

  const int64_t NU = (w->N + kRows - 1) / kRows;
  // Each CTA works on one slice only (one table build): floor(SMs / KS) CTAs per slice.
  const int64_t per = sm_count() / a.KS > 1 ? sm_count() / a.KS : 1;
  a.G = static_cast<int>(per < NU ? per : NU);
  const int64_t grid = static_cast<int64_t>(a.KS) * a.G;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kBlockThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // The packed weights as tensor maps for the ring's copies: codes as 32-bit words,
  // one row of the map per group of four rows; 1-bit / 2-bit scales as fp16, one row
  // per group. Boxes cover one slice of kSub units (and of one unit, for the tail).
  using T = Traits<FMT>;
  auto fn = tensor_map_encoder();
  if (!fn) return cudaErrorInvalidValue;
  const cuuint64_t NG = static_cast<cuuint64_t>((w->N + 3) / 4);
  auto encode = [&](CUtensorMap* m, CUtensorMapDataType dt, void* base, cuuint64_t cols,
                    cuuint64_t pitch, cuuint32_t bx, cuuint32_t by) {
    const cuuint64_t dims[2] = {cols, NG};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {bx, by};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  CUtensorMap tm_c, tm_c1, tm_s, tm_s1;
  void* codes = const_cast<void*>(w->codes);
  const cuuint64_t cw = static_cast<cuuint64_t>(w->code_stride);  // words per group
  if (!encode(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT32, codes, cw, cw * 4, 4 * T::kWords, 4 * kSub) ||
      !encode(&tm_c1, CU_TENSOR_MAP_DATA_TYPE_UINT32, codes, cw, cw * 4, 4 * T::kWords, 4))
    return cudaErrorInvalidValue;
  tm_s = tm_c;  // ternary: unused
  tm_s1 = tm_c1;
  if (T::kScaleBytes > 0) {
    void* sc = const_cast<void*>(w->scales);
    const cuuint64_t se = static_cast<cuuint64_t>(w->scale_stride) * 4;  // fp16 per group
    if (!encode(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, sc, se, se * 2, T::kScaleBytes / 2, 4 * kSub) ||
        !encode(&tm_s1, CU_TENSOR_MAP_DATA_TYPE_UINT16, sc, se, se * 2, T::kScaleBytes / 2, 4))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_lut_kernel<FMT>, tm_c, tm_s, tm_c1, tm_s1, a);
  if (e != cudaSuccess || a.KS == 1) return e;
  // The sum kernel is launched early too (the main kernel lets it start when its
  // CTAs are past their units; released at the main kernel's start instead, its CTAs
  // came out of the wait up to 3 us apart). It lets the next product's kernel
  // launch early in turn (launch_dependents at its start).
  cudaLaunchConfig_t cfg2 = cfg;
  int logP = 0;
  while ((a.KS + (1 << logP) - 1) >> logP > kSumRun) ++logP;
  const bool pairs = (w->N % 2) == 0;
  const int64_t threads = (pairs ? w->N / 2 : w->N) << logP;
  const int64_t ctas = (threads + kSumThreads - 1) / kSumThreads;
  // one pass per thread: up to two of its 4096-register CTAs an SM once the main
  // kernel has left (the next product's main kernel waits for the space)
  cfg2.gridDim = dim3(static_cast<unsigned>(ctas < 8 * sm_count() ? ctas : 8 * sm_count()));
  cfg2.blockDim = dim3(kSumThreads);
  cfg2.dynamicSmemBytes = 0;
  const float* part = a.part;
  const int64_t N = w->N;
  return pairs ? cudaLaunchKernelEx(&cfg2, splitk_sum_kernel<true>, part, a.KS, N, logP, y, y32)
               : cudaLaunchKernelEx(&cfg2, splitk_sum_kernel<false>, part, a.KS, N, logP, y, y32);
}

}  // namespace

unsigned* lbq_fault_word() {
  static PerDevice<unsigned*> addr;  // looked up once per device, with that device current
  unsigned* a = nullptr;
  const cudaError_t e = addr.get(
      [](int, unsigned** v) {
        void* p = nullptr;
        const cudaError_t r = cudaGetSymbolAddress(&p, g_fault_word);
        if (r != cudaSuccess) return r;
        *v = static_cast<unsigned*>(p);
        return cudaSuccess;
      },
      &a);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return a;
}

size_t lbq_gemv_workspace(const lbq_weights* w) {
  const int KS = slices_of(w);
  if (KS <= 1) return 0;
  return kWsCounterBytes + static_cast<size_t>(KS) * static_cast<size_t>(w->N) * sizeof(float);
}

cudaError_t lbq_launch_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                            uint16_t* y, float* y32, void* ws, cudaStream_t s) {
  switch (w->fmt) {
    case LBQ_TERN5: return launch<LBQ_TERN5>(w, x, D, y, y32, ws, s);
    case LBQ_SIGN1: return launch<LBQ_SIGN1>(w, x, D, y, y32, ws, s);
    default: return launch<LBQ_Q2RHT>(w, x, D, y, y32, ws, s);
  }
}
