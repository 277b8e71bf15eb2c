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

// The SM's register file is split between its four schedulers: a CTA of 16 warps (four
// per scheduler) may use 128 registers a thread, one of 17 to 20 warps only 96.
#ifndef LBQ_BATCH_WARPS
#define LBQ_BATCH_WARPS 15
#endif
constexpr int kCWarps = LBQ_BATCH_WARPS;     // compute warps
constexpr int kCThreads = 32 * kCWarps;      // compute threads
constexpr int kBuildThreads = kCThreads / 64 * 64;  // the table build takes whole column sets of 64
constexpr int kMaxRegs = kCWarps + 1 <= 16 ? 128 : 96;
constexpr int kBThreads = kCThreads + 32;    // + the helper warp
constexpr int kRows = 16;                    // rows per unit (four groups of four)
constexpr int kLag = 4;                      // a product's split-K sum waits this many products
// Partial-sum buffers in flight. Product p's buffer was last used by p - kRing, summed
// during p - kRing + kLag; the helper checks that sum while readying p, two products
// ahead of the compute warps, having released its own CTA's sums up to p - 3: so
// p - kRing + kLag <= p - 3 at least; three products more leave slack for CTAs that
// run behind.
#ifndef LBQ_BATCH_RING_SLACK
#define LBQ_BATCH_RING_SLACK 3
#endif
constexpr int kRing = kLag + 3 + LBQ_BATCH_RING_SLACK;
// The helper asks L2 for the first kPrefetchUnits units of each compute warp of a
// product while the warps build its table (the warps' own loads then run a unit ahead:
// prefetches of their own measured no faster).
constexpr int kPrefetchUnits = 4;
#ifndef LBQ_BATCH_HELPER_PREFETCH
#define LBQ_BATCH_HELPER_PREFETCH 0
#endif
constexpr uint32_t kXBytes = lut::kXsBytes;  // one padded x slice as fp32
constexpr int kXBufs = 3;                    // x slices in shared memory (the helper works 2 ahead)
constexpr uint32_t kMiscBytes = kXBufs * kXBytes + 1024;  // x slices, flags
constexpr uint32_t kDescSmem = 16384;        // the product list, copied to shared memory
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
static_assert(LBQ_BATCH_MAX * sizeof(BProd) <= 16384, "the list fits its shared-memory copy");
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

// Adds v to a counter with release semantics at GPU scope: this thread's earlier writes,
// and those of the threads that met it at a barrier just before, are visible to any
// thread that then reads the new count with acquire semantics.
__device__ __forceinline__ void red_release(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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

// Where this lane's loads of one warp's units are: copied into registers once per
// product and slice, so that the stores of the unit loop cannot make the compiler
// re-read the descriptor. Unit t of the warp is unit u0 + kCWarps t; its groups start
// at w + t * ustep (+ q * gstride for group q); `ng` counts its groups that exist (the
// matrix's last unit may reach past N).
struct Stream {
  const uint8_t* w;   // this lane's word in group 0 of the warp's first unit
  const uint8_t* s;   // this lane's scale load for that unit
  const uint8_t* s0;  // the slice's scale run of group 0 of that unit (1-bit, 2-bit)
  uint32_t ustep;     // bytes between the warp's consecutive units (15 units apart)
  uint32_t sustep;    // the same for the scale loads
  uint32_t gstride;   // code bytes per group of four rows
  uint32_t sstep;     // scale bytes between consecutive groups (1-bit, 2-bit)
  int32_t g0;         // the first unit's first group
  int32_t ng;         // groups of the matrix
};

template <int FMT>
__device__ __forceinline__ Stream make_stream(const BProd& P, const Part& pt, int32_t u0, int lane,
                                              uint32_t woff) {
  using T = Traits<FMT>;
  Stream st;
  st.gstride = 4u * static_cast<uint32_t>(P.cstride);
  st.ustep = kCWarps * 4u * st.gstride;
  st.ng = (P.N + 3) / 4;
  st.g0 = 4 * u0;
  st.w = P.codes + static_cast<int64_t>(st.g0) * st.gstride + pt.j * T::kGroupBytes + woff;
  if (FMT == LBQ_TERN5) {
    // rows R, R + 1 after three butterfly stages (R = 8 b0 + 4 b1 + 2 b2 of the lane)
    const int R = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1);
    int b = lane >> 3;
    if (b >= pt.nb) b = pt.nb - 1;  // no block here: any finite scale times a zero sum
    st.s = P.codes + static_cast<int64_t>(st.g0 + (R >> 2)) * st.gstride +
           16 * (pt.j * T::kWords + 7 * b + 6) + 4 * (R & 3);
    st.s0 = st.s;
    st.sstep = 0;
    st.sustep = st.ustep;
  } else {
    st.sstep = 8u * static_cast<uint32_t>(P.sstride);  // scale bytes per group of four rows
    st.sustep = kCWarps * 4u * st.sstep;
    const int b = FMT == LBQ_SIGN1 ? (lane >> 2) : (lane >> 1);
    const int bb = b < pt.nb ? b : pt.nb - 1;
    const int gl = FMT == LBQ_SIGN1 ? 2 * (lane & 1) + ((lane >> 1) & 1) : 2 * (lane & 1);
    st.s0 = reinterpret_cast<const uint8_t*>(P.scales) + static_cast<int64_t>(st.g0) * st.sstep +
            pt.j * T::kScaleBytes;
    st.s = st.s0 + gl * st.sstep + 8 * bb;
  }
  return st;
}

template <int FMT>
__device__ __forceinline__ void load_unit(const Stream& st, int32_t t, int lane, uint64_t pol,
                                          UnitRegs& r) {
  const uint8_t* w = st.w + static_cast<uint64_t>(t) * st.ustep;
  const int32_t left = st.ng - (st.g0 + 4 * kCWarps * t);  // groups of this unit that exist
  if (left >= 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q) r.w[q] = ldg_stream(w + q * st.gstride, pol);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) r.w[q] = q < left ? ldg_stream(w + q * st.gstride, pol) : make_uint4(0u, 0u, 0u, 0u);
  }
  const uint8_t* sp = st.s + static_cast<uint64_t>(t) * st.sustep;
  if (FMT == LBQ_TERN5) {
    const int gl = 2 * (lane & 1) + ((lane >> 1) & 1);
    r.s[0] = gl < left ? ldg_stream2(sp, pol) : make_uint2(0u, 0u);
  } else if (FMT == LBQ_SIGN1) {
    const int gl = 2 * (lane & 1) + ((lane >> 1) & 1);
    r.s[0] = gl < left ? ldg_stream2(sp, pol) : make_uint2(0u, 0u);
  } else {
    const int gl = 2 * (lane & 1);
    r.s[0] = gl < left ? ldg_stream2(sp, pol) : make_uint2(0u, 0u);
    r.s[1] = gl + 1 < left ? ldg_stream2(sp + st.sstep, pol) : make_uint2(0u, 0u);
  }
}

// Asks L2 for a line (a hint: later loads find it in L2 instead of waiting on HBM).
__device__ __forceinline__ void prefetch_line(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}


// The deferred split-K sum of one product for this CTA's share of its rows, done by the
// compute warps two products later (every CTA is then long done with it): the loads
// are issued before the table build, whose shared-memory work hides their latency,
// and finished after it. Row r of the share is summed by P consecutive threads, each
// over a run of at most kRun slices, combined by a fixed shuffle tree (deterministic).
constexpr int kRun = 8;

// This CTA's split-K sum of one product: rows [n0, n1), logP: log2 of the threads a row
// (2^logP runs of at most kRun slices each). Computed once per product (divisions are
// slow) by the helper, or by reduce_plan in the tail.
struct RedPlan {
  int32_t n0, n1, logP, run;
};
__device__ __forceinline__ RedPlan reduce_plan(const BProd& P) {
  RedPlan rp;
  rp.logP = 0;
  while ((P.KS + (1 << rp.logP) - 1) >> rp.logP > kRun) ++rp.logP;  // at most 64 threads a row
  rp.run = (P.KS + (1 << rp.logP) - 1) >> rp.logP;
  rp.n0 = static_cast<int32_t>(static_cast<int64_t>(blockIdx.x) * P.N / gridDim.x);
  rp.n1 = static_cast<int32_t>(static_cast<int64_t>(blockIdx.x + 1) * P.N / gridDim.x);
  return rp;
}

struct Reduce {
  float v[kRun];
  int32_t row;   // this thread's row, or -1
  int32_t nv;    // slices in its run
};

__device__ __forceinline__ void reduce_begin(const BArgs& a, int q, const RedPlan& rp, int tid, int batch,
                                             Reduce& r) {
  const BProd& P = a.p[q];
  const int rows_per_batch = kCThreads >> rp.logP;
  const int32_t row = rp.n0 + batch * rows_per_batch + (tid >> rp.logP);
  const int sub = tid & ((1 << rp.logP) - 1);
  r.row = -1;
  r.nv = 0;
#pragma unroll
  for (int i = 0; i < kRun; ++i) r.v[i] = 0.0f;
  if (tid < (rows_per_batch << rp.logP) && row < rp.n1) {
    r.row = row;
    const int j0 = sub * rp.run;
    r.nv = P.KS - j0 < rp.run ? (P.KS - j0 > 0 ? P.KS - j0 : 0) : rp.run;
    const float* part = a.ring + static_cast<int64_t>(q % kRing) * a.ring_floats + row;
    // predicated loads into zeroed registers: nothing waits for them until reduce_end
#pragma unroll
    for (int i = 0; i < kRun; ++i)
      asm volatile(
          "{\n\t.reg .pred p;\n\tsetp.lt.s32 p, %2, %3;\n\t@p ld.global.cg.f32 %0, [%1];\n\t}"
          : "+f"(r.v[i])
          : "l"(part + static_cast<int64_t>(j0 + i) * P.N), "r"(i), "r"(r.nv));
  }
}

// Adds the loaded runs, combines each row's runs (fixed shuffle tree), stores y; returns
// whether rows remain for another batch.
__device__ __forceinline__ bool reduce_end(const BArgs& a, int q, const RedPlan& rp, int tid, int batch,
                                           Reduce& r) {
  const BProd& P = a.p[q];
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < kRun; ++i)
    if (i < r.nv) s += r.v[i];
  const int np = 1 << rp.logP;
  for (int o = 1; o < np; o <<= 1) s += __shfl_down_sync(0xffffffffu, s, o, np);
  if (r.row >= 0 && (tid & (np - 1)) == 0) P.y[r.row] = f32_to_bf16_bits(s);
  return rp.n0 + (batch + 1) * (kCThreads >> rp.logP) < rp.n1;
}

// The whole share of product q at once (no table build to hide behind).
__device__ __forceinline__ void reduce_all(const BArgs& a, int q, int tid) {
  const RedPlan rp = reduce_plan(a.p[q]);
  Reduce r;
  for (int batch = 0;; ++batch) {
    reduce_begin(a, q, rp, tid, batch, r);
    if (!reduce_end(a, q, rp, tid, batch, r)) break;
  }
}

// What the helper works out for the compute warps while readying product p: the
// first share of p this CTA takes and the split-K sum of p - kLag it adds.
struct Prep {
  Part pt;
  RedPlan rp;
};

// The x slice of this CTA's first share of product p (slice j), converted to fp32 (the
// 2-bit format: rotated) into xs by one warp; the helper does this a product ahead.
template <int FMT>
__device__ __forceinline__ void x_slice_warp(const BProd& P, int32_t j, int nb, float* xs, int lane) {
  using T = Traits<FMT>;
  if (FMT == LBQ_Q2RHT) {
    x_store<FMT>(x_issue<FMT>(P.x, P.D, P.nblk, j, lane), xs, lane);
  } else {
    const uint4* x8 = reinterpret_cast<const uint4*>(P.x + static_cast<int64_t>(j) * T::kWeights);
    constexpr int kChunks = T::kWeights / 8;  // 16-byte chunks of 8 activations
    uint4 v[kChunks / 32];
#pragma unroll
    for (int i = 0; i < kChunks / 32; ++i) {
      const int c = lane + 32 * i;
      v[i] = 8 * c < nb * kTernBlock ? __ldg(x8 + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kChunks / 32; ++i) x_store8<FMT>(v[i], xs, lane + 32 * i);
  }
}

// Shared-memory flags between the compute warps and the helper (CTA scope).
struct Flags {
  int started;    // products the compute warps have started
  int built;      // products whose table the compute warps have built
  int gate;       // products < gate may start: x slice in place, global counters checked
  int unitsdone;  // products whose units (and the sum due with them) the compute warps finished
};
__device__ __forceinline__ void st_release_cta(volatile int* p, int v) {
  asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(smem_u32(const_cast<int*>(p))), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const volatile int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(const_cast<int*>(p))) : "memory");
  return v;
}

// Spins on a shared-memory counter written by another warp of the CTA; gives up after
// the wait limit, recording the fault code, or as soon as any wait has given up.
__device__ __forceinline__ bool wait_smem(const volatile int* c, int target, unsigned* fault) {
  if (ld_acquire_cta(c) >= target) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1; ld_acquire_cta(c) < target; ++i) {
    __nanosleep(32);
    if ((i & 63) == 0) {
      if (*reinterpret_cast<volatile unsigned*>(fault) != 0) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicExch(fault, kFaultBatch);
        return false;
      }
    }
  }
  return true;
}

template <int FMT>
__device__ __forceinline__ void compute_product(const BArgs& a, int p, uint32_t tbase, float* xbuf,
                                                volatile Flags* fl, const Prep* prep, int tid, bool& ok) {
  using T = Traits<FMT>;
  const BProd& P = a.p[p];
  const int warp = tid >> 5, lane = tid & 31;
  const int participants = P.KS * P.G;
  float* part = a.ring + static_cast<int64_t>(p % kRing) * a.ring_floats;
  float* const xs = xbuf + (p % kXBufs) * (kXBytes / 4);
  // The helper opens the gate of product p once its x slice is in xs, every CTA is done
  // with product q = p - kLag (whose split-K sum is added here) and every CTA has summed
  // product p - kRing (the last user of the ring buffer this product writes).
  const int q = p - kLag;
  const bool red = q >= 0 && a.p[q].KS > 1;
  if (tid == 0 && ok) ok = wait_smem(&fl->gate, p + 1, a.fault);
  named_bar_sync(1, kCThreads);
  // a CTA with no share of this product has no table to build: nothing to wait for
  if (tid == 0 && static_cast<int>(blockIdx.x) >= participants) st_release_cta(&fl->built, p + 1);
  const Prep& pr = prep[p % kXBufs];  // written by the helper before it opened the gate
  const RedPlan rp = pr.rp;
  Reduce r;
  bool rmore = false;
  if (red) reduce_begin(a, q, rp, tid, 0, r);
  bool rpending = red;
  bool first = true;
  for (int v = blockIdx.x; v < participants; v += gridDim.x) {
    const Part pt = first ? pr.pt : part_of<FMT>(P, v);
    if (!first) {  // a further share of this product (more slices than CTAs)
      x_store<FMT>(x_issue<FMT>(P.x, P.D, P.nblk, pt.j, tid), xs, tid);
      named_bar_sync(1, kCThreads);
    }
    first = false;
    if (tid < kBuildThreads) build_table<FMT, kBuildThreads>(pt.nb, tbase, xs, tid);
    if (rpending) {  // the sum's loads have landed behind the build
      rmore = reduce_end(a, q, rp, tid, 0, r);
      rpending = false;
    }
    named_bar_sync(1, kCThreads);
    if (tid == 0) st_release_cta(&fl->built, p + 1);

    const int wl = lane_word<FMT>(lane, pt.nb);
    const int wq = lane_word<FMT>(lane & ~7, pt.nb);
    const uint32_t woff = 16u * static_cast<uint32_t>(wl >= 0 ? wl : (wq >= 0 ? wq : 0));
    const uint32_t lanereg = tbase | static_cast<uint32_t>(lane * 4);
    const int rloc = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 3) & 1);
    const int32_t n_units = pt.u_hi - pt.u_lo;
    const int32_t nt = n_units > warp ? (n_units - warp + kCWarps - 1) / kCWarps : 0;
    // the row this lane stores for the warp's unit t: row0 + 16 kCWarps t
    const int32_t N = P.N;
    const int32_t row0 = (pt.u_lo + warp) * kRows + rloc;
    const bool store_lane = lane < 16;
    uint16_t* const yp = P.y;
    float* const part_j = part + static_cast<int64_t>(pt.j) * N;
    const bool direct = P.KS == 1;
    const Stream st = make_stream<FMT>(P, pt, pt.u_lo + warp, lane, woff);
    const uint64_t pol = evict_first_policy();
    auto finish = [&](float val, int32_t t) {
      const int32_t row = row0 + kRows * kCWarps * t;
      if (store_lane && row < N) {
        if (direct) yp[row] = f32_to_bf16_bits(val);
        else part_j[row] = val;
      }
    };
    // two register buffers, one unit's loads in flight while the other is looked up
    // (a third measured no faster); unrolled by two so that they swap without copies
    UnitRegs ra, rb;
    if (nt > 0) load_unit<FMT>(st, 0, lane, pol, ra);
    for (int32_t t = 0; t < nt; t += 2) {
      if (t + 1 < nt) load_unit<FMT>(st, t + 1, lane, pol, rb);
      finish(unit_sum<FMT>(ra, lanereg, lane), t);
      if (t + 1 >= nt) break;
      if (t + 2 < nt) load_unit<FMT>(st, t + 2, lane, pol, ra);
      finish(unit_sum<FMT>(rb, lanereg, lane), t + 1);
    }
    named_bar_sync(1, kCThreads);  // every warp is done with the table
  }
  if (rpending) rmore = reduce_end(a, q, rp, tid, 0, r);  // this CTA had no share of product p
  if (red && rmore) {  // a share larger than one batch: the rest, without overlap
    for (int rbatch = 1;; ++rbatch) {
      reduce_begin(a, q, rp, tid, rbatch, r);
      if (!reduce_end(a, q, rp, tid, rbatch, r)) break;
    }
  }
  // the slice sums of p and the sums of q are stored: the helper releases them
  named_bar_sync(1, kCThreads);
  if (tid == 0) st_release_cta(&fl->unitsdone, p + 1);
}

// The last products' sums, after the compute warps' final product (the helper has
// checked that every CTA is done with them).
__device__ __forceinline__ void reduce_tail(const BArgs& a, volatile Flags* fl, int tid, bool& ok) {
  if (tid == 0 && ok) ok = wait_smem(&fl->gate, a.n + 1, a.fault);
  named_bar_sync(1, kCThreads);
  for (int q = a.n - kLag > 0 ? a.n - kLag : 0; q < a.n; ++q)
    if (a.p[q].KS > 1) reduce_all(a, q, tid);
}

// The helper's L2 prefetch of the first units of each of this CTA's warps for product p
// (kPrefetchUnits of them, as the warps' own prefetch runs that far ahead), so that HBM
// keeps streaming while the compute warps build the product's table.
template <int FMT>
__device__ __forceinline__ void prefetch_product(const BArgs& a, int p, int lane) {
  using T = Traits<FMT>;
  const BProd& P = a.p[p];
  const int participants = P.KS * P.G;
  const int32_t NG = (P.N + 3) / 4;
  for (int v = blockIdx.x; v < participants; v += gridDim.x) {
    const Part pt = part_of<FMT>(P, v);
    const uint32_t cbytes = FMT == LBQ_TERN5 ? 112u * pt.nb : (FMT == LBQ_SIGN1 ? 64u * pt.nb : 512u);
    const int32_t g0 = 4 * pt.u_lo;
    int32_t g1 = 4 * (pt.u_lo + kCWarps * (kPrefetchUnits + 1));
    if (g1 > 4 * pt.u_hi) g1 = 4 * pt.u_hi;
    if (g1 > NG) g1 = NG;
    const uint8_t* base = P.codes + pt.j * T::kGroupBytes;
    const int64_t gstride = 4 * static_cast<int64_t>(P.cstride);
    // each group's run, line by line (128-byte lines; runs of 448 or 512 bytes)
    const int lines = static_cast<int>((cbytes + 127) / 128) + 1;
    for (int32_t i = lane; i < (g1 - g0) * lines; i += 32) {
      const int32_t g = g0 + i / lines;
      const uint32_t off = 128u * static_cast<uint32_t>(i % lines);
      if (off < cbytes + 127) prefetch_line(base + g * gstride + (off < cbytes ? off : cbytes - 1));
    }
    if (FMT != LBQ_TERN5) {
      const uint8_t* sb = reinterpret_cast<const uint8_t*>(P.scales) + pt.j * T::kScaleBytes;
      for (int32_t g = g0 + lane; g < g1; g += 32) prefetch_line(sb + g * 8 * static_cast<int64_t>(P.sstride));
    }
  }
}

// The helper's preload of the x slice of this CTA's first share of product p.
template <int FMT>
__device__ __forceinline__ void xload_product(const BArgs& a, int p, float* xs, int lane) {
  const BProd& P = a.p[p];
  if (static_cast<int>(blockIdx.x) < P.KS * P.G) {
    const Part pt = part_of<FMT>(P, blockIdx.x);
    x_slice_warp<FMT>(P, pt.j, pt.nb, xs, lane);
  }
}

// Format masks: the kernel is compiled once per set of formats a list holds, so that a
// list of one format gets code (and registers) for that format alone.
// The kernel is compiled once per format (kFmts = that format's bit): one kernel that
// chose the format per product needed more registers than a thread has, and ran every
// phase of a pass about twice as slowly (measured on a ternary list, as a function
// call per product and inlined alike), so a list of several formats is run as one
// launch per format (the products are independent).
__host__ __device__ constexpr int fmt_bit(int fmt) { return 1 << (fmt - 1); }

template <int kFmts>
__device__ __forceinline__ void prefetch_any(const BArgs& a, int p, int lane) {
  const int f = a.p[p].fmt;
  if ((kFmts & fmt_bit(LBQ_TERN5)) && f == LBQ_TERN5) prefetch_product<LBQ_TERN5>(a, p, lane);
  if ((kFmts & fmt_bit(LBQ_SIGN1)) && f == LBQ_SIGN1) prefetch_product<LBQ_SIGN1>(a, p, lane);
  if ((kFmts & fmt_bit(LBQ_Q2RHT)) && f == LBQ_Q2RHT) prefetch_product<LBQ_Q2RHT>(a, p, lane);
}
template <int kFmts>
__device__ __forceinline__ void xload_any(const BArgs& a, int p, float* xs, int lane) {
  const int f = a.p[p].fmt;
  if ((kFmts & fmt_bit(LBQ_TERN5)) && f == LBQ_TERN5) xload_product<LBQ_TERN5>(a, p, xs, lane);
  if ((kFmts & fmt_bit(LBQ_SIGN1)) && f == LBQ_SIGN1) xload_product<LBQ_SIGN1>(a, p, xs, lane);
  if ((kFmts & fmt_bit(LBQ_Q2RHT)) && f == LBQ_Q2RHT) xload_product<LBQ_Q2RHT>(a, p, xs, lane);
}

// Shares of product p this CTA works on (virtual CTAs blockIdx.x, + gridDim.x, ...).
__device__ __forceinline__ unsigned shares_of(const BArgs& a, int p) {
  const int participants = a.p[p].KS * a.p[p].G;
  return static_cast<int>(blockIdx.x) < participants
             ? static_cast<unsigned>((participants - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1)
             : 0u;
}

// The helper readies product p: its x slice, the checks on other CTAs' progress, the L2
// prefetch of its first units; then opens its gate.
template <int FMT>
__device__ __forceinline__ Part first_part(const BProd& P) {
  return static_cast<int>(blockIdx.x) < P.KS * P.G ? part_of<FMT>(P, blockIdx.x) : Part{0, 0, 0, 1};
}

template <int kFmts>
__device__ __forceinline__ bool helper_prepare(const BArgs& a, int p, float* xbuf, volatile Flags* fl,
                                               Prep* prep, int lane, bool ok) {
  if (lane == 0) {  // the share and the sum plan, for the compute warps
    Prep pr;
    const int f = a.p[p].fmt;
    pr.pt = (kFmts & fmt_bit(LBQ_TERN5)) && f == LBQ_TERN5   ? first_part<LBQ_TERN5>(a.p[p])
            : (kFmts & fmt_bit(LBQ_SIGN1)) && f == LBQ_SIGN1 ? first_part<LBQ_SIGN1>(a.p[p])
                                                             : first_part<LBQ_Q2RHT>(a.p[p]);
    pr.rp = p - kLag >= 0 ? reduce_plan(a.p[p - kLag]) : RedPlan{0, 0, 0, 1};
    prep[p % kXBufs] = pr;
  }
  // the two counters are read (lane 0) while the x slice loads are in flight
  const int q = p - kLag;
  const bool need_done = q >= 0 && a.p[q].KS > 1, need_red = a.p[p].KS > 1 && p >= kRing;
  const unsigned done_target = need_done ? static_cast<unsigned>(a.p[q].KS * a.p[q].G) : 0u;
  unsigned dv = 0, rv = 0;
  if (lane == 0 && need_done) dv = ld_acquire(a.ctr + kCtrDone + q);
  if (lane == 0 && need_red) rv = ld_acquire(a.ctr + kCtrReduced + (p - kRing));
  xload_any<kFmts>(a, p, xbuf + (p % kXBufs) * (kXBytes / 4), lane);
  if (lane == 0 && ok && need_done && dv < done_target)
    ok = wait_count(a.ctr + kCtrDone + q, done_target, a.fault);
  if (lane == 0 && ok && need_red && rv < gridDim.x)
    ok = wait_count(a.ctr + kCtrReduced + (p - kRing), gridDim.x, a.fault);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  if (lane == 0) st_release_cta(&fl->gate, p + 1);  // (x slice stores released too)
#if LBQ_BATCH_HELPER_PREFETCH == 1
  prefetch_any<kFmts>(a, p + 0, lane);
#endif
  return ok;
}

template <int kFmts>
__global__ void __maxnreg__(kMaxRegs) gemv_batch_kernel(const __grid_constant__ BArgs a0) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  const bool misc_low = tbase - sbase >= kMiscBytes + kDescSmem;
  const uint32_t misc = misc_low ? sbase : tbase + kTableBytes;
  float* xbuf = reinterpret_cast<float*>(smem + (misc - sbase));  // two x slices
  volatile Flags* fl = reinterpret_cast<volatile Flags*>(smem + (misc - sbase) + kXBufs * kXBytes);
  Prep* prep = reinterpret_cast<Prep*>(smem + (misc - sbase) + kXBufs * kXBytes + 64);
  // the product list in shared memory (every product start reads its descriptor)
  const uint32_t dsc = misc + kMiscBytes;  // after the x slices and flags, below or above the table
  const bool layout_ok = tbase + kTableBytes <= sbase + kSmemBatch && dsc + kDescSmem <= sbase + kSmemBatch &&
                         (!misc_low || dsc + kDescSmem <= tbase);
  BProd* dsm = reinterpret_cast<BProd*>(smem + (dsc - sbase));
  if (layout_ok) {
    const uint4* src = reinterpret_cast<const uint4*>(a0.p);
    uint4* dst = reinterpret_cast<uint4*>(dsm);
    for (int i = tid; i < a0.n * static_cast<int>(sizeof(BProd) / 16); i += blockDim.x) dst[i] = src[i];
  }
  if (tid == 0 && layout_ok) {
    fl->started = 0;
    fl->built = 0;
    fl->gate = 0;
    fl->unitsdone = 0;
  }
  __syncthreads();
  BArgs a = a0;
  a.p = dsm;
  if (!layout_ok) {
    if (tid == 0) atomicExch(a.fault, kFaultBatchLayout);  // cannot happen with a 0 or 1 KB prefix
    // still count this CTA out, so that the counters end at zero
  } else if (warp < kCWarps) {
    bool ok = true;
    for (int p = 0; p < a.n; ++p) {
      if (tid == 0) st_release_cta(&fl->started, p + 1);
      compute_product<kFmts == fmt_bit(LBQ_TERN5)   ? LBQ_TERN5
                      : kFmts == fmt_bit(LBQ_SIGN1) ? LBQ_SIGN1
                                                    : LBQ_Q2RHT>(a, p, tbase, xbuf, fl, prep, tid, ok);
    }
    reduce_tail(a, fl, tid, ok);
  } else {
    // The helper runs two products ahead of the compute warps. For each product p: once
    // they have started p, it readies p + 2 (x slice into the buffer p - 1 used, which
    // they are done with; checks on other CTAs; L2 prefetch) and opens its gate; once
    // they have finished p's units, it releases this CTA's count for p (and for the
    // sum of p - kLag done with it) at GPU scope, off their path.
    bool ok = helper_prepare<kFmts>(a, 0, xbuf, fl, prep, lane, true);
    if (a.n > 1) ok = helper_prepare<kFmts>(a, 1, xbuf, fl, prep, lane, ok);
    for (int p = 0; p < a.n; ++p) {
      if (!wait_smem(&fl->started, p + 1, a.fault)) break;
      // product p + 2's x slice goes where p - 1's was: the compute warps are past it
      if (p + 2 < a.n) ok = helper_prepare<kFmts>(a, p + 2, xbuf, fl, prep, lane, ok);
#if LBQ_BATCH_HELPER_PREFETCH == 2
      // the first units of p + 1 into L2, once the compute warps' prologue of p (whose
      // loads would queue behind these requests) is over
      if (p + 1 < a.n && wait_smem(&fl->built, p + 1, a.fault)) prefetch_any<kFmts>(a, p + 1, lane);
#endif
      if (!wait_smem(&fl->unitsdone, p + 1, a.fault)) break;
      if (lane == 0) {
        const unsigned sh = shares_of(a, p);
        if (sh) red_release(a.ctr + kCtrDone + p, sh);
        if (p - kLag >= 0) red_release(a.ctr + kCtrReduced + (p - kLag), 1u);
      }
    }
    // the last products' sums: every CTA must be done with them
    if (lane == 0) {
      for (int q = a.n - kLag > 0 ? a.n - kLag : 0; q < a.n && ok; ++q)
        if (a.p[q].KS > 1) ok = wait_count(a.ctr + kCtrDone + q, static_cast<unsigned>(a.p[q].KS * a.p[q].G), a.fault);
      st_release_cta(&fl->gate, a.n + 1);
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
                                               : cudaErrorInvalidValue;  // one format a launch
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
                                      : launch_batch<4>(a, grid, s);
}
