// gemv_batch.cu -- many independent batch-1 products in one persistent launch.
//
// The products are those of gemv.cu (ternary add/subtract/skip per block, pptc.cn
// ternary-27B article §1.2 and mhpq.cn "27B in 5.9 GB" article §2.1-2.2; 1-bit Q1_0,
// neodrop.ai round-up part 2; 2-bit with the rotated input, feinterview.poetries.top
// "27B in 12 GB" article), computed with the same byte-lookup tables (lut.cuh). What
// changes is how a list of them is scheduled: one CTA per SM stays resident for the
// whole list, so nothing is paid per product for a launch, a dependency wait or a
// split-K tail kernel, and the weight stream never stops between products.
//
// Per CTA and product: one K-slice and a range of 16-row units (the same split as
// the single-product kernel). Warps 0-14 load the x slice, build the 128 KB table,
// then take units: each lane loads its word of four rows per group with 16-byte
// global loads (no L1 allocation), one unit ahead, looks its bytes up, and the warp
// reduces the unit's 16 rows with a transpose-reduce butterfly whose first stages
// stay inside one scale block, so the block scales multiply 2 (ternary), 4 (1-bit)
// or 8 (2-bit) values a lane instead of 16. Warp 15 (the helper) runs beside them:
// it prefetches the next product's weights and x into L2 (bulk prefetch), so HBM keeps
// streaming while the table is rebuilt, and it adds up the slice sums of the previous
// product for its share of rows (split-K, in a fixed order: deterministic) once
// every CTA has counted itself done with that product.
//
// Synchronisation between CTAs is through counters at the start of the workspace
// (done and reduced per product, and an exit count); the last CTA to leave resets
// them, so every completed launch leaves them zero. The launch is cooperative, so
// all CTAs are resident together, and every wait is bounded (fault code 12).
#include "lut.cuh"
#include "sm100_async.cuh"

namespace {

using namespace lbq;
using namespace lbq::lut;

// 16 warps in all: the SM's register file is split between its four schedulers, so a
// CTA of 16 warps (four per scheduler) may use 128 registers a thread, one of 17 only 96.
constexpr int kCWarps = 15;                  // compute warps
constexpr int kCThreads = 32 * kCWarps;      // compute threads
constexpr int kBuildThreads = 448;           // the table build takes whole column sets of 64
constexpr int kBThreads = kCThreads + 32;    // + the helper warp
constexpr int kRows = 16;                    // rows per unit (four groups of four)
constexpr int kRing = 4;                     // partial-sum buffers in flight
constexpr uint32_t kXBytes = 4096;           // the x slice as fp32 (up to 1024)
constexpr uint32_t kMiscBytes = kXBytes + 1024;
constexpr uint32_t kSmemBatch = 192 * 1024;  // the table needs a 64 KB-aligned 128 KB
constexpr unsigned kFaultBatch = 12, kFaultBatchLayout = 13;
constexpr int kMaxBatch = LBQ_BATCH_MAX;
// counters (32-bit words at the start of the workspace)
constexpr int kCtrDone = 0, kCtrReduced = kMaxBatch, kCtrExit = 2 * kMaxBatch;

// One product as the kernel sees it (64 bytes). The list lives in the workspace, after
// the counters, written there by the install kernel before each launch: the main
// kernel's own parameters stay small.
struct __align__(16) BProd {
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* x;
  const int8_t* D;
  uint16_t* y;
  int32_t cstride;  // code bytes per row
  int32_t sstride;  // fp16 scales per row
  int32_t N;
  int16_t fmt;
  int16_t KS;       // K-slices
  int16_t G;        // CTAs per slice
  int16_t nblk;     // scale blocks per row
};
static_assert(sizeof(BProd) == 64, "descriptor size");
constexpr int kInstallChunk = 56;  // descriptors per install launch (parameters < 4 KB)
constexpr size_t kDescBytes = kMaxBatch * sizeof(BProd);  // the list, after the ring buffers

struct BInstall {
  int32_t first, count;
  BProd* dst;
  BProd p[kInstallChunk];
};

struct BArgs {
  int32_t n;
  int32_t pad;
  int64_t ring_floats;  // floats per partial-sum buffer
  float* ring;          // kRing buffers
  unsigned* ctr;
  unsigned* fault;
  const BProd* p;       // the list (in the workspace)
};

__global__ void install_kernel(const __grid_constant__ BInstall in) {
  const int i = threadIdx.x;
  if (i < in.count) in.dst[in.first + i] = in.p[i];
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spins (sleeping between polls) until *p >= target; gives up after the wait limit,
// recording the fault code, or once another wait has given up.
__device__ __forceinline__ bool wait_count(const unsigned* p, unsigned target, unsigned* fault) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(i < 64 ? 32 : 256);
    if (ld_acquire(p) >= target) return true;
    if ((i & 63) == 0) {
      if (*reinterpret_cast<volatile unsigned*>(fault) != 0) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicExch(fault, kFaultBatch);
        return false;
      }
    }
  }
}

// Weight loads: read once, so they neither allocate in L1 nor stay in L2 for long
// (an evict-first cache policy: the L2 keeps the prefetched weights of the next
// product and the slice sums instead).
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ldg_stream(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ uint2 ldg_stream2(const void* p, uint64_t pol) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p), "l"(pol));
  return v;
}

// The CTA's work on one product: virtual CTA v in [0, KS * G) is slice v / G and the
// v % G-th share of the 16-row units.
struct Part {
  int32_t j, u_lo, u_hi, nb;
};
template <int FMT>
__device__ __forceinline__ Part part_of(const BProd& P, int v) {
  using T = Traits<FMT>;
  Part r;
  const int32_t NU = (P.N + kRows - 1) / kRows;
  r.j = v / P.G;
  const int32_t gs = v - r.j * P.G;
  r.u_lo = static_cast<int32_t>(static_cast<int64_t>(gs) * NU / P.G);
  r.u_hi = static_cast<int32_t>(static_cast<int64_t>(gs + 1) * NU / P.G);
  const int blk0 = r.j * T::kBlocks;
  r.nb = P.nblk - blk0 < T::kBlocks ? P.nblk - blk0 : T::kBlocks;
  return r;
}

// One unit's packed words (and, for 1-bit / 2-bit, its block scales) for this lane.
struct UnitRegs {
  uint4 w[4];   // the lane's word of each group's four rows
  uint2 s[2];   // scales: ternary s[0] = scale words of rows R, R+1; 1-bit s[0] = group
                // G's four scales of the lane's block; 2-bit s[0], s[1] = groups G, G + 1
};

template <int FMT>
__device__ __forceinline__ void load_unit(const BProd& P, const Part& pt, int32_t u, int lane,
                                          uint32_t woff, uint64_t pol, UnitRegs& r) {
  using T = Traits<FMT>;
  const int64_t NG = (static_cast<int64_t>(P.N) + 3) / 4;
  const int64_t gstride = 4 * static_cast<int64_t>(P.cstride);  // bytes per group of four rows
  const uint8_t* base = P.codes + static_cast<int64_t>(pt.j) * T::kGroupBytes + woff;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t g = 4 * static_cast<int64_t>(u) + q;  // warp-uniform
    r.w[q] = g < NG ? ldg_stream(base + g * gstride, pol) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (FMT == LBQ_TERN5) {
    // rows R, R + 1 after three butterfly stages (R = 8 b0 + 4 b1 + 2 b2 of the lane)
    const int R = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1);
    const int64_t g = 4 * static_cast<int64_t>(u) + (R >> 2);
    int b = lane >> 3;
    if (b >= pt.nb) b = pt.nb - 1;  // no block here: any finite scale times a zero sum
    const uint8_t* sp = P.codes + g * gstride + 16 * (static_cast<int64_t>(pt.j) * T::kWords + 7 * b + 6) +
                        4 * (R & 3);
    r.s[0] = g < NG ? ldg_stream2(sp, pol) : make_uint2(0u, 0u);
  } else {
    const int64_t sg = 8 * static_cast<int64_t>(P.sstride);  // scale bytes per group of four rows
    const int b = FMT == LBQ_SIGN1 ? (lane >> 2) : (lane >> 1);
    const int bb = b < pt.nb ? b : pt.nb - 1;
    const uint8_t* sb = reinterpret_cast<const uint8_t*>(P.scales) +
                        8 * (static_cast<int64_t>(pt.j) * T::kBlocks + bb);
    if (FMT == LBQ_SIGN1) {
      const int64_t g = 4 * static_cast<int64_t>(u) + 2 * (lane & 1) + ((lane >> 1) & 1);
      r.s[0] = g < NG ? ldg_stream2(sb + g * sg, pol) : make_uint2(0u, 0u);
    } else {
      const int64_t g = 4 * static_cast<int64_t>(u) + 2 * (lane & 1);
      r.s[0] = g < NG ? ldg_stream2(sb + g * sg, pol) : make_uint2(0u, 0u);
      r.s[1] = g + 1 < NG ? ldg_stream2(sb + (g + 1) * sg, pol) : make_uint2(0u, 0u);
    }
  }
}

// One transpose-reduce stage: c values -> c / 2; the lane keeps the upper half of the
// row range if its bit d is set, the lower half otherwise, and adds its partner's.
template <int C>
__device__ __forceinline__ void tr_stage(float (&acc)[kRows], int lane, int d) {
  const bool up = (lane & d) != 0;
#pragma unroll
  for (int r = 0; r < C / 2; ++r) {
    const float send = up ? acc[r] : acc[r + C / 2];
    const float keep = up ? acc[r + C / 2] : acc[r];
    acc[r] = keep + __shfl_xor_sync(0xffffffffu, send, d);
  }
}

// Lookups, block scales and the reduction of one unit; returns the sum of row
// 8 b0 + 4 b1 + 2 b2 + b3 of the unit in every lane (b_k = bit k of the lane).
template <int FMT>
__device__ __forceinline__ float unit_sum(const UnitRegs& r, uint32_t lanereg, int lane) {
  float acc[kRows];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 p01 = lookup_pair(r.w[q].x, r.w[q].y, lanereg);
    const float2 p23 = lookup_pair(r.w[q].z, r.w[q].w, lanereg);
    acc[4 * q] = p01.x;
    acc[4 * q + 1] = p01.y;
    acc[4 * q + 2] = p23.x;
    acc[4 * q + 3] = p23.y;
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
  tr_stage<2>(acc, lane, 8);
  return acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 16);
}

// The deferred split-K sum of one product for this CTA's share of its rows, done by the
// compute warps two products later (every CTA is then long done with it): the loads
// are issued before the table build, whose shared-memory work hides their latency,
// and finished after it. Row r of the share is summed by P consecutive threads, each
// over a run of at most kRun slices, combined by a fixed shuffle tree (deterministic).
constexpr int kRun = 8;
struct Reduce {
  float v[kRun];
  int64_t row;   // this thread's row, or -1
  int sub, P;    // its place among the row's P threads
  int nv;        // slices in its run
};

__device__ __forceinline__ void reduce_begin(const BArgs& a, int q, int tid, int64_t batch, Reduce& r) {
  const BProd& P = a.p[q];
  r.row = -1;
  r.nv = 0;
  r.P = 1;
  while ((P.KS + r.P - 1) / r.P > kRun) r.P *= 2;  // at most 64 threads a row (KS <= 512)
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * P.N / gridDim.x;
  const int64_t n1 = static_cast<int64_t>(blockIdx.x + 1) * P.N / gridDim.x;
  const int rows_per_batch = kCThreads / r.P;
  const int64_t row = n0 + batch * rows_per_batch + tid / r.P;
  r.sub = tid % r.P;
  if (tid < rows_per_batch * r.P && row < n1) {
    r.row = row;
    const int run = (P.KS + r.P - 1) / r.P;
    const int j0 = r.sub * run;
    r.nv = P.KS - j0 < run ? (P.KS - j0 > 0 ? P.KS - j0 : 0) : run;
    const float* part = a.ring + static_cast<int64_t>(q % kRing) * a.ring_floats + row;
#pragma unroll
    for (int i = 0; i < kRun; ++i)
      r.v[i] = i < r.nv ? __ldcg(part + static_cast<int64_t>(j0 + i) * P.N) : 0.0f;
  }
}

// Returns whether rows remain for another batch.
__device__ __forceinline__ bool reduce_end(const BArgs& a, int q, int tid, int64_t batch, Reduce& r) {
  const BProd& P = a.p[q];
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < kRun; ++i)
    if (i < r.nv) s += r.v[i];
  for (int o = 1; o < r.P; o <<= 1) s += __shfl_down_sync(0xffffffffu, s, o, r.P);
  if (r.row >= 0 && r.sub == 0) P.y[r.row] = f32_to_bf16_bits(s);
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * P.N / gridDim.x;
  const int64_t n1 = static_cast<int64_t>(blockIdx.x + 1) * P.N / gridDim.x;
  return n0 + (batch + 1) * (kCThreads / r.P) < n1;
}

// The whole share of product q at once (no table build to hide behind).
__device__ __forceinline__ void reduce_all(const BArgs& a, int q, int tid) {
  Reduce r;
  for (int64_t batch = 0;; ++batch) {
    reduce_begin(a, q, tid, batch, r);
    if (!reduce_end(a, q, tid, batch, r)) break;
  }
}

template <int FMT>
__device__ __forceinline__ void compute_product(const BArgs& a, int p, uint32_t tbase, float* xs,
                                                int tid, bool& ok) {
  using T = Traits<FMT>;
  const BProd& P = a.p[p];
  const int warp = tid >> 5, lane = tid & 31;
  const int participants = P.KS * P.G;
  float* part = a.ring + static_cast<int64_t>(p % kRing) * a.ring_floats;
  // Product q = p - 2 is summed here: wait (bounded) until every CTA is done with it,
  // and -- before this product writes its slice sums -- until every CTA has summed
  // product p - kRing, the last user of the ring buffer this product writes.
  const int q = p - 2;
  const bool red = q >= 0 && a.p[q].KS > 1;
  if (tid == 0 && ok && red)
    ok = wait_count(a.ctr + kCtrDone + q, static_cast<unsigned>(a.p[q].KS * a.p[q].G), a.fault);
  if (tid == 0 && ok && P.KS > 1 && p >= kRing)
    ok = wait_count(a.ctr + kCtrReduced + (p - kRing), gridDim.x, a.fault);
  named_bar_sync(1, kCThreads);
  Reduce r;
  int64_t rbatch = 0;
  bool rmore = false;
  if (red) reduce_begin(a, q, tid, 0, r);
  bool rpending = red;
  for (int v = blockIdx.x; v < participants; v += gridDim.x) {
    const Part pt = part_of<FMT>(P, v);
    x_store<FMT>(x_issue<FMT>(P.x, P.D, P.nblk, pt.j, tid), xs, tid);
    named_bar_sync(1, kCThreads);
    if (tid < kBuildThreads) build_table<FMT, kBuildThreads>(pt.nb, tbase, xs, tid);
    if (rpending) {  // the sum's loads have landed behind the build
      rmore = reduce_end(a, q, tid, 0, r);
      rpending = false;
    }
    named_bar_sync(1, kCThreads);

    const int wl = lane_word<FMT>(lane, pt.nb);
    const int wq = lane_word<FMT>(lane & ~7, pt.nb);
    const uint32_t woff = 16u * static_cast<uint32_t>(wl >= 0 ? wl : (wq >= 0 ? wq : 0));
    const uint32_t lanereg = tbase | static_cast<uint32_t>(lane * 4);
    const int rloc = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 3) & 1);
    const int32_t n_units = pt.u_hi - pt.u_lo;
    const int32_t nt = n_units > warp ? (n_units - warp + kCWarps - 1) / kCWarps : 0;
    float* const part_j = part + static_cast<int64_t>(pt.j) * P.N;
    UnitRegs cur, nxt;
    const uint64_t pol = evict_first_policy();
    if (nt > 0) load_unit<FMT>(P, pt, pt.u_lo + warp, lane, woff, pol, cur);
    for (int32_t t = 0; t < nt; ++t) {
      const int32_t u = pt.u_lo + warp + kCWarps * t;
      if (t + 1 < nt) load_unit<FMT>(P, pt, u + kCWarps, lane, woff, pol, nxt);
      const float s = unit_sum<FMT>(cur, lanereg, lane);
      const int64_t row = static_cast<int64_t>(u) * kRows + rloc;
      if (lane < 16 && row < P.N) {
        if (P.KS == 1)
          P.y[row] = f32_to_bf16_bits(s);
        else
          part_j[row] = s;
      }
      cur = nxt;
    }
    __threadfence();  // the slice sums, before the count below
    named_bar_sync(1, kCThreads);  // also: every warp is done with the table
    if (tid == 0) atomicAdd(a.ctr + kCtrDone + p, 1u);
  }
  if (rpending) rmore = reduce_end(a, q, tid, 0, r);  // this CTA had no share of product p
  if (red && rmore) {  // a share larger than one batch: the rest, without overlap
    for (rbatch = 1;; ++rbatch) {
      reduce_begin(a, q, tid, rbatch, r);
      if (!reduce_end(a, q, tid, rbatch, r)) break;
    }
  }
  if (q >= 0) {  // product q is summed (or needed no sum): its ring buffer may be reused
    __threadfence();
    named_bar_sync(1, kCThreads);
    if (tid == 0) atomicAdd(a.ctr + kCtrReduced + q, 1u);
  }
}

// The last two products' sums, after the compute warps' final product.
__device__ __forceinline__ void reduce_tail(const BArgs& a, int tid, bool& ok) {
  for (int q = a.n - 2 > 0 ? a.n - 2 : 0; q < a.n; ++q) {
    if (a.p[q].KS > 1) {
      if (tid == 0 && ok)
        ok = wait_count(a.ctr + kCtrDone + q, static_cast<unsigned>(a.p[q].KS * a.p[q].G), a.fault);
      named_bar_sync(1, kCThreads);
      reduce_all(a, q, tid);
    }
  }
}

// The helper's bulk L2 prefetch of this CTA's share of product p (weights, scales, x).
template <int FMT>
__device__ __forceinline__ void prefetch_product(const BArgs& a, int p, int lane) {
  using T = Traits<FMT>;
  const BProd& P = a.p[p];
  const int participants = P.KS * P.G;
  const int64_t NG = (static_cast<int64_t>(P.N) + 3) / 4;
  for (int v = blockIdx.x; v < participants; v += gridDim.x) {
    const Part pt = part_of<FMT>(P, v);
    const uint32_t cbytes = FMT == LBQ_TERN5 ? 112u * pt.nb : (FMT == LBQ_SIGN1 ? 64u * pt.nb : 512u);
    const uint32_t sbytes = (8u * pt.nb + 15u) & ~15u;  // rows of scales are padded to 16 bytes
    const int64_t g0 = 4 * static_cast<int64_t>(pt.u_lo);
    int64_t g1 = 4 * static_cast<int64_t>(pt.u_hi);
    if (g1 > NG) g1 = NG;
    for (int64_t g = g0 + lane; g < g1; g += 32) {
      prefetch_l2_bulk(P.codes + g * 4 * static_cast<int64_t>(P.cstride) + static_cast<int64_t>(pt.j) * T::kGroupBytes,
                       cbytes);
      if (FMT != LBQ_TERN5)
        prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(P.scales) + g * 8 * static_cast<int64_t>(P.sstride) +
                             static_cast<int64_t>(pt.j) * T::kScaleBytes, sbytes);
    }
    if (lane == 0) {
      const int64_t k0 = static_cast<int64_t>(pt.j) * T::kWeights;
      const int nw = FMT == LBQ_TERN5 ? 128 * pt.nb : (FMT == LBQ_SIGN1 ? 128 * pt.nb : 512);
      prefetch_l2_bulk(P.x + k0, 2u * nw);
      if (FMT == LBQ_Q2RHT) prefetch_l2_bulk(P.D + k0, 512u);
    }
  }
}

// Format masks: the kernel is compiled once per set of formats a list holds, so that a
// list of one format gets code (and registers) for that format alone.
__host__ __device__ constexpr int fmt_bit(int fmt) { return 1 << (fmt - 1); }

template <int kFmts>
__device__ __forceinline__ void prefetch_any(const BArgs& a, int p, int lane) {
  const int f = a.p[p].fmt;
  if ((kFmts & fmt_bit(LBQ_TERN5)) && f == LBQ_TERN5) prefetch_product<LBQ_TERN5>(a, p, lane);
  if ((kFmts & fmt_bit(LBQ_SIGN1)) && f == LBQ_SIGN1) prefetch_product<LBQ_SIGN1>(a, p, lane);
  if ((kFmts & fmt_bit(LBQ_Q2RHT)) && f == LBQ_Q2RHT) prefetch_product<LBQ_Q2RHT>(a, p, lane);
}

template <int kFmts>
__global__ void __launch_bounds__(kBThreads, 1) gemv_batch_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  const bool misc_low = tbase - sbase >= kMiscBytes;
  const uint32_t misc = misc_low ? sbase : tbase + kTableBytes;
  volatile int* started = reinterpret_cast<volatile int*>(smem + (misc - sbase) + kXBytes);
  const bool layout_ok = tbase + kTableBytes <= sbase + kSmemBatch && misc + kMiscBytes <= sbase + kSmemBatch;
  if (tid == 0 && layout_ok) *started = 0;  // products the compute warps have started
  __syncthreads();
  if (!layout_ok) {
    if (tid == 0) atomicExch(a.fault, kFaultBatchLayout);  // cannot happen with a 0 or 1 KB prefix
    // still count this CTA out, so that the counters end at zero
  } else if (warp < kCWarps) {
    float* xs = reinterpret_cast<float*>(smem + (misc - sbase));
    bool ok = true;
    for (int p = 0; p < a.n; ++p) {
      if (tid == 0) *started = p + 1;  // paces the helper's prefetch
      const int f = a.p[p].fmt;
      if ((kFmts & fmt_bit(LBQ_TERN5)) && f == LBQ_TERN5) compute_product<LBQ_TERN5>(a, p, tbase, xs, tid, ok);
      if ((kFmts & fmt_bit(LBQ_SIGN1)) && f == LBQ_SIGN1) compute_product<LBQ_SIGN1>(a, p, tbase, xs, tid, ok);
      if ((kFmts & fmt_bit(LBQ_Q2RHT)) && f == LBQ_Q2RHT) compute_product<LBQ_Q2RHT>(a, p, tbase, xs, tid, ok);
    }
    reduce_tail(a, tid, ok);
    if (tid == 0) *started = a.n + 1;
  } else {
    // helper: prefetch one product ahead of the compute warps
    prefetch_any<kFmts>(a, 0, lane);
    for (int p = 0; p < a.n; ++p) {
      // wait (bounded) until the compute warps have started product p
      const uint64_t t0 = global_ns();
      while (*started < p + 1) {
        __nanosleep(200);
        if (global_ns() - t0 > kWaitLimitNs) {
          if (lane == 0) atomicExch(a.fault, kFaultBatch);
          break;
        }
      }
      if (p + 1 < a.n) prefetch_any<kFmts>(a, p + 1, lane);
    }
  }
  // count this CTA out; the last one resets the counters for the next launch
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(a.ctr + kCtrExit, 1u);
    if (prev == gridDim.x - 1) {
      for (int i = 0; i < a.n; ++i) {
        a.ctr[kCtrDone + i] = 0;
        a.ctr[kCtrReduced + i] = 0;
      }
      a.ctr[kCtrExit] = 0;
      __threadfence();
    }
  }
}

int slices_for(int32_t fmt, int64_t K) {
  const int64_t per = fmt == LBQ_SIGN1 ? 1024 : 512;
  return static_cast<int>((K + per - 1) / per);
}

}  // namespace

// Floats per partial-sum buffer: the largest KS * N of the list, 256-byte multiple.
size_t ring_floats_for(const lbq_product* ps, int32_t n) {
  size_t ring = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int KS = slices_for(ps[i].w.fmt, ps[i].w.K);
    if (KS > 1) {
      const size_t f = static_cast<size_t>(KS) * static_cast<size_t>(ps[i].w.N);
      if (f > ring) ring = f;
    }
  }
  return (ring + 63) / 64 * 64;
}

// [64 KB counters][kRing partial-sum buffers][the product list]
size_t lbq_gemv_batch_ws(const lbq_product* ps, int32_t n) {
  return kWsCounterBytes + kRing * ring_floats_for(ps, n) * sizeof(float) + kDescBytes;
}

namespace {

// Sets the kernel's shared-memory limit (once per device) and checks that one CTA fits
// on an SM; the grid is one CTA per SM (the table takes most of the shared memory).
template <int kFmts>
cudaError_t batch_grid(int* grid) {
  static PerDevice<int> cache;
  return cache.get(
      [](int, int* g) {
        cudaError_t r = cudaFuncSetAttribute(gemv_batch_kernel<kFmts>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBatch));
        if (r != cudaSuccess) return r;
        int per_sm = 0;
        r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_batch_kernel<kFmts>, kBThreads,
                                                          kSmemBatch);
        if (r != cudaSuccess) return r;
        if (per_sm < 1) return cudaErrorLaunchOutOfResources;  // one CTA does not fit an SM
        *g = sm_count();
        return cudaSuccess;
      },
      grid);
}

template <int kFmts>
cudaError_t launch_batch(const BArgs& a, int grid, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kBThreads);
  cfg.dynamicSmemBytes = kSmemBatch;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_batch_kernel<kFmts>, a);
}

}  // namespace

cudaError_t lbq_launch_gemv_batch(const lbq_product* ps, int32_t n, void* ws, cudaStream_t s) {
  int mask = 0;
  for (int32_t i = 0; i < n; ++i) mask |= fmt_bit(ps[i].w.fmt);
  int grid = 0;
  cudaError_t e = mask == fmt_bit(LBQ_TERN5)   ? batch_grid<1>(&grid)
                  : mask == fmt_bit(LBQ_SIGN1) ? batch_grid<2>(&grid)
                  : mask == fmt_bit(LBQ_Q2RHT) ? batch_grid<4>(&grid)
                                               : batch_grid<7>(&grid);
  if (e != cudaSuccess) return e;
  unsigned* fault = lbq_fault_word();
  if (!fault) return cudaErrorInvalidDevicePointer;
  const size_t ring_floats = ring_floats_for(ps, n);
  BArgs a;
  a.n = n;
  a.pad = 0;
  a.ring_floats = static_cast<int64_t>(ring_floats);
  a.ring = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes);
  a.ctr = static_cast<unsigned*>(ws);
  a.fault = fault;
  BProd* list = reinterpret_cast<BProd*>(static_cast<char*>(ws) + kWsCounterBytes +
                                         kRing * ring_floats * sizeof(float));
  a.p = list;
  BInstall in;
  in.dst = list;
  for (int32_t i = 0; i < n; ++i) {
    const lbq_weights& w = ps[i].w;
    BProd& P = in.p[i % kInstallChunk];
    P.codes = static_cast<const uint8_t*>(w.codes);
    P.scales = static_cast<const uint16_t*>(w.scales);
    P.x = ps[i].x;
    P.D = ps[i].D;
    P.y = ps[i].y;
    P.cstride = static_cast<int32_t>(w.code_stride);
    P.sstride = static_cast<int32_t>(w.scale_stride);
    P.N = static_cast<int32_t>(w.N);
    P.fmt = static_cast<int16_t>(w.fmt);
    P.KS = static_cast<int16_t>(slices_for(w.fmt, w.K));
    const int64_t NU = (w.N + kRows - 1) / kRows;
    const int64_t per = grid / P.KS > 1 ? grid / P.KS : 1;
    P.G = static_cast<int16_t>(per < NU ? per : NU);
    P.nblk = static_cast<int16_t>(w.K / (w.fmt == LBQ_Q2RHT ? kQ2Block : kTernBlock));
    if (i % kInstallChunk == kInstallChunk - 1 || i == n - 1) {  // a full chunk, or the last
      in.first = i - i % kInstallChunk;
      in.count = i % kInstallChunk + 1;
      install_kernel<<<1, kInstallChunk, 0, s>>>(in);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return mask == fmt_bit(LBQ_TERN5)   ? launch_batch<1>(a, grid, s)
         : mask == fmt_bit(LBQ_SIGN1) ? launch_batch<2>(a, grid, s)
         : mask == fmt_bit(LBQ_Q2RHT) ? launch_batch<4>(a, grid, s)
                                      : launch_batch<7>(a, grid, s);
}
