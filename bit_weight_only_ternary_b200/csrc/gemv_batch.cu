// gemv_batch.cu -- many independent batch-1 products in one launch (stream-K schedule).
//
// The products are those of gemv.cu (ternary add/subtract/skip per block, pptc.cn
// ternary-27B article §1.2 and mhpq.cn "27B in 5.9 GB" article §2.1-2.2; 1-bit Q1_0,
// neodrop.ai round-up part 2; 2-bit with the rotated input, feinterview.poetries.top
// "27B in 12 GB" article), computed with the same byte-lookup tables (lut.cuh). What
// changes is how a list of them is scheduled.
//
// Work is counted in unit-slices: one 16-row unit of one K-slice (512 weights; 1024 for
// the 1-bit format). A product of KS slices and NU units costs KS * NU. The list's
// products are laid end to end, each as NU row-units of full K, and the total is cut
// into one contiguous range per CTA (one CTA per SM), the ranges of equal cost: their
// unit-slices plus a fixed charge per table the range will build (plan_cut, on the
// host). Every CTA computes whole rows of one or a few products, all of K, so its rows
// need nobody else's sums. It
// walks its range slice by slice: for each slice it builds the 128 KB lookup table of
// that slice of x once and runs all its units of that product through it, keeping
// each row's running sum in shared memory (in chunks of up to kAccUnits units), so a
// table build serves hundreds of units. For a 64-layer pass each CTA builds about 20
// tables, where a product-by-product split builds one per product (256).
//
// A product whose row-units are too coarse for that cut (few rows, many slices: a
// CTA's share would be a fraction of one row-unit) is split along K into S pieces
// of consecutive slices; each piece writes its fp32 sums to the workspace and a small
// second kernel adds the S pieces of every row in a fixed order (deterministic). The
// rule is on the host (pieces_for); a 27B-layer pass has no split product.
//
// There is no communication between CTAs at all: no counters, no waits. Inside a CTA,
// 16 warps build the table together (two barriers per slice), then take units: each
// lane loads its word of four rows per group with 16-byte global loads (no L1
// allocation, evict-first in L2), one unit ahead, looks its bytes up, and the warp
// reduces the unit's 16 rows with the butterfly of lut.cuh. The next slice's x comes
// in by cp.async while the units run; the last units of a slice ask L2 for the first
// ones of the next, and each warp's first two units of the next slice are loaded before
// its table is built, so the weight stream runs on through the build.
#include <vector>

#include "lut.cuh"
#include "sm100_async.cuh"

namespace {

using namespace lbq;
using namespace lbq::lut;

// 16 warps (four per scheduler) may use 128 registers a thread. (20 warps at 96
// registers spill and ran 20-35% slower; 12 or 8 warps with three or four unit
// buffers ran 5-30% slower.)
#ifndef LBQ_BATCH_WARPS
#define LBQ_BATCH_WARPS 16
#endif
constexpr int kWarps = LBQ_BATCH_WARPS;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 16;  // rows per unit (four groups of four)
// Units a chunk keeps running sums for in shared memory (a multiple of kWarps): 63 KB,
// the room below a 64 KB-aligned table when the dynamic window starts 1 KB in.
constexpr int32_t kAccUnits = 1008 / kWarps * kWarps;
constexpr uint32_t kAccBytes = kAccUnits * kRows * 4;
// The split rule: one row-unit of a piece may cost at most 1 / kMinUnitsPerTable of a
// CTA's share, so that a table build serves at least that many units.
constexpr int64_t kMinUnitsPerTable = 64;
constexpr uint32_t kXRawBytes = 2048;  // one x slice as bf16 (1024 weights at most)
constexpr uint32_t kDRawBytes = 512;   // its rotation signs (2-bit format)
constexpr uint32_t kMiscBytes = kXRawBytes + kDRawBytes + kXsBytes + 64;  // + the start index
constexpr uint32_t kSmemBatch = 227 * 1024;
constexpr unsigned kFaultBatchLayout = 13;
constexpr int kMaxBatch = LBQ_BATCH_MAX;

static_assert(kAccUnits % kWarps == 0, "chunks are whole rounds of units");
static_assert(kAccBytes <= 63 * 1024, "the sums fit below the table");

// One product as the kernel sees it (80 bytes).
struct __align__(16) BProd {
  const uint8_t* codes;
  const uint16_t* scales;
  const uint16_t* x;
  const int8_t* D;
  uint16_t* y;
  int64_t c0;       // unit-slices of the products before this one
  int64_t poff;     // first float of this product's piece sums (S > 1)
  int32_t cstride;  // code bytes per row
  int32_t sstride;  // fp16 scales per row
  int32_t N;
  int32_t NU;       // 16-row units
  int16_t fmt;
  int16_t KS;       // K-slices
  int16_t S;        // pieces along K (1: rows are whole on one CTA)
  int16_t nblk;     // scale blocks per row
};
static_assert(sizeof(BProd) == 80, "descriptor size");

// The launch's parameters, the product list included (about 20 KB: kernel parameters
// may take up to 32 KB since CUDA 12.1), so nothing is copied before the launch.
constexpr int kMaxGrid = LBQ_BATCH_MAX_CTAS;  // CTAs a launch may use (one per SM)
struct BArgs {
  float* partial;   // piece sums of split products
  unsigned* fault;
  int64_t W;        // unit-slices of the whole list
  int32_t n;
  int32_t pad;
  int64_t bound[kMaxGrid + 1];  // CTA c's range of unit-slices: [bound[c], bound[c + 1])
  BProd p[kMaxBatch];
};
static_assert(sizeof(BArgs) <= 32764, "kernel parameter limit");

// Weight loads: read once, so they neither allocate in L1 nor stay in L2 for long.
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
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// One step of a CTA's walk: slice j of the chunk [c0, c1) of this CTA's units [u0, u1)
// of piece s (slices [j0, j1)) of product p; p < 0 when the walk is over.
struct Seg {
  int32_t p, s;
  int32_t u0, u1;
  int32_t c0, c1;
  int32_t j, j0, j1;
};

// Piece s of a product: slices [KS s / S, KS (s + 1) / S).
__device__ __forceinline__ int32_t piece_start(int32_t KS, int32_t S, int32_t s) {
  return static_cast<int32_t>(static_cast<int64_t>(KS) * s / S);
}

// The first piece at or after (p, s) with units in [lo, hi): unit u of piece s covers
// the unit-slices [base + u len, base + (u + 1) len), base = c0 + NU j0, len = j1 - j0,
// and belongs to the CTA whose range holds its first one.
__device__ Seg find_piece(const BProd* list, int32_t n, int32_t p, int32_t s, int64_t lo, int64_t hi) {
  Seg g;
  g.p = -1;
  for (; p < n; ++p, s = 0) {
    const BProd& P = list[p];
    if (P.c0 >= hi) return g;
    for (; s < P.S; ++s) {
      const int32_t j0 = piece_start(P.KS, P.S, s), j1 = piece_start(P.KS, P.S, s + 1);
      const int64_t len = j1 - j0;
      const int64_t base = P.c0 + static_cast<int64_t>(P.NU) * j0;
      if (base >= hi) return g;
      const int64_t u0 = lo > base ? (lo - base + len - 1) / len : 0;
      int64_t u1 = (hi - base + len - 1) / len;
      if (u1 > P.NU) u1 = P.NU;
      if (u0 < u1) {
        g.p = p;
        g.s = s;
        g.u0 = static_cast<int32_t>(u0);
        g.u1 = static_cast<int32_t>(u1);
        g.c0 = g.u0;
        g.c1 = g.u1 - g.u0 > kAccUnits ? g.u0 + kAccUnits : g.u1;
        g.j = g.j0 = j0;
        g.j1 = j1;
        return g;
      }
    }
  }
  return g;
}

__device__ __forceinline__ Seg advance(const BProd* list, int32_t n, Seg g, int64_t lo, int64_t hi) {
  if (g.j + 1 < g.j1) {
    ++g.j;
    return g;
  }
  if (g.c1 < g.u1) {
    g.c0 = g.c1;
    g.c1 = g.u1 - g.c0 > kAccUnits ? g.c0 + kAccUnits : g.u1;
    g.j = g.j0;
    return g;
  }
  return find_piece(list, n, g.p, g.s + 1, lo, hi);
}

template <int FMT>
__device__ __forceinline__ int blocks_in(const BProd& P, int32_t j) {
  const int left = P.nblk - j * Traits<FMT>::kBlocks;
  return left < Traits<FMT>::kBlocks ? left : Traits<FMT>::kBlocks;
}

// x slice j of P (and its signs) into the staging buffers, 16 bytes a thread by
// cp.async (x and D are 16-byte aligned, slices start at 16-byte multiples).
template <int FMT>
__device__ __forceinline__ void x_fetch(const BProd& P, int32_t j, int nb, uint32_t xraw, uint32_t draw, int tid) {
  using T = Traits<FMT>;
  const int64_t k0 = static_cast<int64_t>(j) * T::kWeights;
  if (FMT == LBQ_Q2RHT) {
    if (tid < 32) {  // 16 activations and 16 signs a lane, as x_store rotates them
      cp_async16(xraw + 32 * tid, P.x + k0 + 16 * tid);
      cp_async16(xraw + 32 * tid + 16, P.x + k0 + 16 * tid + 8);
      cp_async16(draw + 16 * tid, P.D + k0 + 16 * tid);
    }
  } else if (tid < T::kWeights / 8 && 8 * tid < nb * kTernBlock) {
    cp_async16(xraw + 16 * tid, P.x + k0 + 8 * tid);
  }
  cp_async_commit();
}

// The staged slice as padded fp32 in xs (each thread converts what it fetched).
template <int FMT>
__device__ __forceinline__ void x_convert(int nb, uint32_t xraw, uint32_t draw, float* xs, int tid) {
  using T = Traits<FMT>;
  cp_async_wait_all();
  if (FMT == LBQ_Q2RHT) {
    if (tid < 32) {
      XLoad r;
      r.v0 = lds_v4(xraw + 32 * tid);
      r.v1 = lds_v4(xraw + 32 * tid + 16);
      r.d = lds_v4(draw + 16 * tid);
      x_store<FMT>(r, xs, tid);
    }
  } else if (tid < T::kWeights / 8) {
    const uint4 v = 8 * tid < nb * kTernBlock ? lds_v4(xraw + 16 * tid) : make_uint4(0u, 0u, 0u, 0u);
    x_store8<FMT>(v, xs, tid);
  }
}

// Where this lane's loads of one warp's units are, in registers for the unit loop.
// Unit t of the warp is unit u0 + kWarps t; its groups start at w + t * ustep
// (+ q * gstride for group q); `ng` counts the matrix's groups (its last unit may
// reach past N).
struct Stream {
  const uint8_t* w;   // this lane's word in group 0 of the warp's first unit
  const uint8_t* s;   // this lane's scale load for that unit
  uint32_t ustep;     // bytes between the warp's consecutive units (kWarps units apart)
  uint32_t sustep;    // the same for the scale loads
  uint32_t gstride;   // code bytes per group of four rows
  uint32_t sstep;     // scale bytes between consecutive groups (1-bit, 2-bit)
  int32_t g0;         // the first unit's first group
  int32_t ng;         // groups of the matrix
};

template <int FMT>
__device__ __forceinline__ Stream make_stream(const BProd& P, int32_t j, int nb, int32_t u0, int lane,
                                              uint32_t woff) {
  using T = Traits<FMT>;
  Stream st;
  st.gstride = 4u * static_cast<uint32_t>(P.cstride);
  st.ustep = kWarps * 4u * st.gstride;
  st.ng = (P.N + 3) / 4;
  st.g0 = 4 * u0;
  st.w = P.codes + static_cast<int64_t>(st.g0) * st.gstride + j * T::kGroupBytes + woff;
  if (FMT == LBQ_TERN5) {
    // rows R, R + 1 after three butterfly stages (R = 8 b0 + 4 b1 + 2 b2 of the lane)
    const int R = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1);
    int b = lane >> 3;
    if (b >= nb) b = nb - 1;  // no block here: any finite scale times a zero sum
    st.s = P.codes + static_cast<int64_t>(st.g0 + (R >> 2)) * st.gstride + 16 * (j * T::kWords + 7 * b + 6) +
           4 * (R & 3);
    st.sstep = 0;
    st.sustep = st.ustep;
  } else {
    st.sstep = 8u * static_cast<uint32_t>(P.sstride);  // scale bytes per group of four rows
    st.sustep = kWarps * 4u * st.sstep;
    const int b = FMT == LBQ_SIGN1 ? (lane >> 2) : (lane >> 1);
    const int bb = b < nb ? b : nb - 1;
    const int gl = FMT == LBQ_SIGN1 ? 2 * (lane & 1) + ((lane >> 1) & 1) : 2 * (lane & 1);
    st.s = reinterpret_cast<const uint8_t*>(P.scales) + static_cast<int64_t>(st.g0) * st.sstep +
           j * T::kScaleBytes + gl * st.sstep + 8 * bb;
  }
  return st;
}

// Refills a buffer with the warp's unit t, group by group as unit_sum frees it (t < 0:
// nothing left to load).
template <int FMT>
struct UnitRefill {
  const Stream& st;
  int32_t t;
  int lane;
  uint64_t pol;
  __device__ __forceinline__ void group(int q, UnitRegs& r) const {
    if (t < 0) return;
    const int32_t left = st.ng - (st.g0 + 4 * kWarps * t);
    const uint8_t* w = st.w + static_cast<uint64_t>(t) * st.ustep + q * st.gstride;
    r.w[q] = q < left ? ldg_stream(w, pol) : make_uint4(0u, 0u, 0u, 0u);
  }
  __device__ __forceinline__ void scales(UnitRegs& r) const {
    if (t < 0) return;
    const int32_t left = st.ng - (st.g0 + 4 * kWarps * t);
    const uint8_t* sp = st.s + static_cast<uint64_t>(t) * st.sustep;
    if (FMT == LBQ_Q2RHT) {
      const int gl = 2 * (lane & 1);
      r.s[0] = gl < left ? ldg_stream2(sp, pol) : make_uint2(0u, 0u);
      r.s[1] = gl + 1 < left ? ldg_stream2(sp + st.sstep, pol) : make_uint2(0u, 0u);
    } else {
      const int gl = 2 * (lane & 1) + ((lane >> 1) & 1);
      r.s[0] = gl < left ? ldg_stream2(sp, pol) : make_uint2(0u, 0u);
    }
  }
};

template <int FMT>
__device__ __forceinline__ void load_unit(const Stream& st, int32_t t, int lane, uint64_t pol, UnitRegs& r) {
  const uint8_t* w = st.w + static_cast<uint64_t>(t) * st.ustep;
  const int32_t left = st.ng - (st.g0 + 4 * kWarps * t);  // groups of this unit that exist
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

// Units a warp asks L2 for ahead of its register loads (0: none). Four measured about
// 7% faster than none in every format; two to eight alike.
#ifndef LBQ_BATCH_PD
#define LBQ_BATCH_PD 4
#endif
constexpr int kPD = LBQ_BATCH_PD;

__device__ __forceinline__ void prefetch_line(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}
// L2 prefetch of the warp's unit t: one line request per group (32 lanes x 16 bytes)
// and the scale runs of the 1-bit and 2-bit formats; only groups that exist.
template <int FMT>
__device__ __forceinline__ void prefetch_unit(const Stream& st, int32_t t, int lane, uint32_t dw = 0,
                                              uint32_t ds = 0) {
  const uint8_t* w = st.w + static_cast<uint64_t>(t) * st.ustep + dw;
  const int32_t left = st.ng - (st.g0 + 4 * kWarps * t);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q < left) prefetch_line(w + q * st.gstride);
  if (FMT != LBQ_TERN5) {
    const uint8_t* sp = st.s + static_cast<uint64_t>(t) * st.sustep + ds;
    const int gl = FMT == LBQ_SIGN1 ? 2 * (lane & 1) + ((lane >> 1) & 1) : 2 * (lane & 1);
    if (gl < left) prefetch_line(sp);
    if (FMT == LBQ_Q2RHT && gl + 1 < left) prefetch_line(sp + st.sstep);
  }
}

// The lane's word offset within a group's slice run (lanes without a word read a
// neighbour's: their table entries are zero-weight columns).
template <int FMT>
__device__ __forceinline__ uint32_t word_offset(int lane, int nb) {
  const int wl = lane_word<FMT>(lane, nb);
  const int wq = lane_word<FMT>(lane & ~7, nb);
  return 16u * static_cast<uint32_t>(wl >= 0 ? wl : (wq >= 0 ? wq : 0));
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemv_batch_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // shared memory: the 128 KB table at the first 64 KB boundary (its page addressing
  // keeps the base in the upper half of the PRMT operand), the running sums below it
  // when they fit there, the x staging and the padded x slice above it
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tbase = (sbase + kPage - 1) & ~(kPage - 1);
  const bool acc_low = tbase - sbase >= kAccBytes;
  const uint32_t acc = acc_low ? sbase : tbase + kTableBytes;
  const uint32_t misc = acc_low ? tbase + kTableBytes : acc + kAccBytes;
  if (tbase + kTableBytes > sbase + kSmemBatch || misc + kMiscBytes > sbase + kSmemBatch) {
    if (tid == 0) atomicExch(a.fault, kFaultBatchLayout);  // cannot happen with a 0 or 1 KB prefix
    return;
  }
  const uint32_t xraw = misc, draw = misc + kXRawBytes;
  float* const xs = reinterpret_cast<float*>(smem + (draw + kDRawBytes - sbase));
  int* const start = reinterpret_cast<int*>(smem + (draw + kDRawBytes + kXsBytes - sbase));

  // this CTA's range of the list's unit-slices, and the product it starts in
  const int64_t lo = a.bound[blockIdx.x], hi = a.bound[blockIdx.x + 1];
  if (tid == 0) *start = a.n;
  __syncthreads();
  if (tid < a.n) {
    const int64_t c0 = a.p[tid].c0, c1 = tid + 1 < a.n ? a.p[tid + 1].c0 : a.W;
    if (c0 <= lo && lo < c1) *start = tid;
  }
  __syncthreads();
  Seg g = find_piece(a.p, a.n, *start, 0, lo, hi);
  if (g.p < 0) return;

  const uint32_t lanereg = tbase | static_cast<uint32_t>(lane * 4);
  const int rloc = 8 * (lane & 1) + 4 * ((lane >> 1) & 1) + 2 * ((lane >> 2) & 1) + ((lane >> 3) & 1);
  const uint64_t pol = evict_first_policy();
  int nb = blocks_in<FMT>(a.p[g.p], g.j);
  x_fetch<FMT>(a.p[g.p], g.j, nb, xraw, draw, tid);
  Stream st = make_stream<FMT>(a.p[g.p], g.j, nb, g.c0 + warp, lane, word_offset<FMT>(lane, nb));
  int32_t nt = g.c1 - g.c0 > warp ? (g.c1 - g.c0 - warp + kWarps - 1) / kWarps : 0;
  UnitRegs ra, rb;
  if (nt > 0) load_unit<FMT>(st, 0, lane, pol, ra);
  if (nt > 1) load_unit<FMT>(st, 1, lane, pol, rb);
  for (int32_t u = 2; u < 2 + kPD && u < nt; ++u) prefetch_unit<FMT>(st, u, lane);
  for (;;) {
    // the slice's x in place, every warp done with the previous table: build this one
    x_convert<FMT>(nb, xraw, draw, xs, tid);
    __syncthreads();
    build_table<FMT, kThreads>(nb, tbase, xs, tid);
    __syncthreads();
    const Seg nx = advance(a.p, a.n, g, lo, hi);
    int nbx = 0;
    if (nx.p >= 0) {  // the next slice's x comes in behind the units
      nbx = blocks_in<FMT>(a.p[nx.p], nx.j);
      x_fetch<FMT>(a.p[nx.p], nx.j, nbx, xraw, draw, tid);
    }
    // When the next step is the next slice of the same units (and both slices are
    // whole), the last units of this slice ask L2 for the first ones of the next: the
    // same units, one slice further (codes one group run, scales one scale run), so the
    // stream does not restart cold after the next table build.
    // (Not for the 2-bit format, measured 3% slower with it: its stream is the closest
    // to the HBM rate, and the early requests compete with the slice's own.)
    const bool pf_next = FMT != LBQ_Q2RHT && nx.p == g.p && nx.s == g.s && nx.c0 == g.c0 &&
                         nx.j == g.j + 1 && nb == Traits<FMT>::kBlocks && nbx == Traits<FMT>::kBlocks;
    {
      const BProd& P = a.p[g.p];
      const int32_t N = P.N;
      const bool first = g.j == g.j0, last = g.j == g.j1 - 1;
      uint16_t* const yp = P.S == 1 ? P.y : nullptr;
      float* const pp = a.partial + P.poff + static_cast<int64_t>(g.s) * N;
      const int32_t row0 = g.c0 * kRows + rloc;
      const bool store_lane = lane < 16;
      // lane l < 16 keeps the running sum of row rloc of each of the warp's units
      auto finish = [&](float val, int32_t t) {
        const int32_t ul = warp + kWarps * t;  // unit within the chunk
        const int32_t row = row0 + kRows * ul;
        if (store_lane && row < N) {
          const uint32_t sa = acc + 4u * static_cast<uint32_t>(kRows * ul + rloc);
          float v = val;
          if (!first) {
            float prev;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(prev) : "r"(sa));
            v += prev;
          }
          if (!last) {
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(sa), "f"(v) : "memory");
          } else if (yp) {
            yp[row] = f32_to_bf16_bits(v);
          } else {
            pp[row] = v;
          }
        }
      };
      auto prefetch_ahead = [&](int32_t u) {
        if (u < nt) prefetch_unit<FMT>(st, u, lane);
        else if (pf_next && u - nt < nt)
          prefetch_unit<FMT>(st, u - nt, lane, Traits<FMT>::kGroupBytes,
                             FMT == LBQ_TERN5 ? Traits<FMT>::kGroupBytes : Traits<FMT>::kScaleBytes);
      };
      // two register buffers, one unit's loads in flight while the other is looked up
      // (three or four, with fewer warps to hold them, measured slower), each refilled
      // group by group as its words are looked up; unrolled by two so that they swap
      // without copies
      for (int32_t t = 0; t < nt; t += 2) {
        if (kPD > 0) prefetch_ahead(t + 2 + kPD);
        finish(unit_sum<FMT>(ra, lanereg, lane, UnitRefill<FMT>{st, t + 2 < nt ? t + 2 : -1, lane, pol}), t);
        if (t + 1 >= nt) break;
        if (kPD > 0) prefetch_ahead(t + 3 + kPD);
        finish(unit_sum<FMT>(rb, lanereg, lane, UnitRefill<FMT>{st, t + 3 < nt ? t + 3 : -1, lane, pol}), t + 1);
      }
    }
    if (nx.p < 0) break;
    // the next slice's first two units, before its table is built (and the next few
    // asked of L2)
    g = nx;
    nb = nbx;
    st = make_stream<FMT>(a.p[g.p], g.j, nb, g.c0 + warp, lane, word_offset<FMT>(lane, nb));
    nt = g.c1 - g.c0 > warp ? (g.c1 - g.c0 - warp + kWarps - 1) / kWarps : 0;
    if (nt > 0) load_unit<FMT>(st, 0, lane, pol, ra);
    if (nt > 1) load_unit<FMT>(st, 1, lane, pol, rb);
    for (int32_t u = 2; u < 2 + kPD && u < nt; ++u) prefetch_unit<FMT>(st, u, lane);
  }
}

// The rows of split products: y = the sum of the S piece sums, in piece order.
__global__ void piece_sum_kernel(const __grid_constant__ BArgs a) {
  const BProd& P = a.p[blockIdx.y];
  if (P.S <= 1) return;
  const int32_t row = static_cast<int32_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= P.N) return;
  const float* src = a.partial + P.poff + row;
  float s = 0.0f;
  for (int k = 0; k < P.S; ++k) s += src[static_cast<int64_t>(k) * P.N];
  P.y[row] = f32_to_bf16_bits(s);
}

int slices_for(int32_t fmt, int64_t K) {
  const int64_t per = fmt == LBQ_SIGN1 ? 1024 : 512;
  return static_cast<int>((K + per - 1) / per);
}

// The schedule of one launch's list: every product's cost, pieces and piece-sum offset.
struct Plan {
  int64_t W = 0;               // unit-slices
  size_t partial_floats = 0;   // piece sums of split products
  int32_t max_split_rows = 0;  // the largest N among split products (0: none)
};

// Pieces along K for a product of KS slices: enough that one row-unit of a piece costs
// at most 1 / kMinUnitsPerTable of a CTA's share W / G.
int pieces_for(int KS, int64_t W, int G) {
  const int64_t need = (kMinUnitsPerTable * G * static_cast<int64_t>(KS) + W - 1) / W;
  return static_cast<int>(need < 1 ? 1 : (need > KS ? KS : need));
}

Plan plan_list(const lbq_product* ps, int32_t n, int G, BProd* out) {
  Plan pl;
  for (int32_t i = 0; i < n; ++i)
    pl.W += static_cast<int64_t>(slices_for(ps[i].w.fmt, ps[i].w.K)) * ((ps[i].w.N + kRows - 1) / kRows);
  int64_t c0 = 0;
  for (int32_t i = 0; i < n; ++i) {
    const lbq_weights& w = ps[i].w;
    const int KS = slices_for(w.fmt, w.K);
    const int64_t NU = (w.N + kRows - 1) / kRows;
    const int S = pieces_for(KS, pl.W, G);
    if (out) {
      BProd& P = out[i];
      P.codes = static_cast<const uint8_t*>(w.codes);
      P.scales = static_cast<const uint16_t*>(w.scales);
      P.x = ps[i].x;
      P.D = ps[i].D;
      P.y = ps[i].y;
      P.c0 = c0;
      P.poff = S > 1 ? static_cast<int64_t>(pl.partial_floats) : 0;
      P.cstride = static_cast<int32_t>(w.code_stride);
      P.sstride = static_cast<int32_t>(w.scale_stride);
      P.N = static_cast<int32_t>(w.N);
      P.NU = static_cast<int32_t>(NU);
      P.fmt = static_cast<int16_t>(w.fmt);
      P.KS = static_cast<int16_t>(KS);
      P.S = static_cast<int16_t>(S);
      P.nblk = static_cast<int16_t>(w.K / (w.fmt == LBQ_Q2RHT ? kQ2Block : kTernBlock));
    }
    if (S > 1) {
      pl.partial_floats += static_cast<size_t>(S) * static_cast<size_t>(w.N);
      if (w.N > pl.max_split_rows) pl.max_split_rows = static_cast<int32_t>(w.N);
    }
    c0 += KS * NU;
  }
  pl.partial_floats = (pl.partial_floats + 63) / 64 * 64;
  return pl;
}

// A table build (with the stream's restart behind it) costs about as much time as this
// many unit-slices (measured: ternary CTAs ended 4.2 us later per build, at 0.077 us a
// unit-slice, before the next slice's first units were prefetched across the build;
// 32 and 54 measured alike after it, 0 about 3% slower).
#ifndef LBQ_BATCH_BUILD_COST
#define LBQ_BATCH_BUILD_COST 48
#endif
constexpr int64_t kBuildCost = LBQ_BATCH_BUILD_COST;

// One greedy pass of the cut for a target cost T per CTA: each CTA takes the list's
// next units in order while its cost (unit-slices plus kBuildCost per table it will
// build: every chunk of every piece builds one table per slice of the piece) stays
// within T. Fills bound[0..G] (the first unit-slice of each CTA's range; W past the
// last) and returns whether every unit found a CTA.
bool cut_for(const BProd* P, int32_t n, int G, int64_t W, int64_t T, int64_t* bound) {
  int32_t p = 0, s = 0;
  int64_t u = 0;  // the next unassigned unit of piece s of product p
  auto skip_done = [&]() {
    while (p < n && u >= P[p].NU) {
      u = 0;
      if (++s >= P[p].S) { s = 0; ++p; }
    }
  };
  skip_done();
  for (int c = 0; c < G; ++c) {
    if (p >= n) { bound[c] = W; continue; }
    const int32_t j0 = static_cast<int32_t>(static_cast<int64_t>(P[p].KS) * s / P[p].S);
    bound[c] = P[p].c0 + static_cast<int64_t>(P[p].NU) * j0 + u * (static_cast<int64_t>(P[p].KS) * (s + 1) / P[p].S - j0);
    int64_t cost = 0;
    while (p < n) {
      const int64_t a = static_cast<int64_t>(P[p].KS) * s / P[p].S;
      const int64_t len = static_cast<int64_t>(P[p].KS) * (s + 1) / P[p].S - a;
      // chunks of this CTA's units of the piece, from its first one
      int64_t in_piece = 0;
      bool stop = false;
      while (u < P[p].NU) {
        const int64_t chunk_room = kAccUnits - in_piece % kAccUnits;
        const int64_t start_cost = in_piece % kAccUnits == 0 ? kBuildCost * len : 0;
        const int64_t afford = (T - cost - start_cost) / len;
        if (afford <= 0) { stop = true; break; }
        int64_t k = afford < chunk_room ? afford : chunk_room;
        if (k > P[p].NU - u) k = P[p].NU - u;
        cost += start_cost + k * len;
        u += k;
        in_piece += k;
        if (k < chunk_room && u < P[p].NU) { stop = true; break; }
      }
      if (stop) break;
      skip_done();
    }
  }
  bound[G] = W;
  return p >= n;
}

// The cut with the smallest T that places every unit (bisection; each pass is linear
// in the CTAs and the list's chunks).
void plan_cut(const BProd* P, int32_t n, int G, int64_t W, int64_t* bound) {
  int64_t lo = (W + G - 1) / G, hi = lo;
  while (!cut_for(P, n, G, W, hi, bound)) hi *= 2;
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (cut_for(P, n, G, W, mid, bound)) hi = mid;
    else lo = mid + 1;
  }
  cut_for(P, n, G, W, hi, bound);
}

}  // namespace

// The schedule of one launch's list for `ctas` CTAs (host only): pieces per product and
// the CTAs' boundaries, exactly as launch_list computes them.
int64_t lbq_gemv_batch_plan_list(const lbq_product* ps, int32_t n, int ctas, int32_t* pieces,
                                 int64_t* bound) {
  std::vector<BProd> all(static_cast<size_t>(n));
  const Plan pl = plan_list(ps, n, ctas, all.data());
  for (int32_t i = 0; i < n; ++i) pieces[i] = all[static_cast<size_t>(i)].S;
  plan_cut(all.data(), n, ctas, pl.W, bound);
  return pl.W;
}

// [64 KB kept zero (the counter rule of every workspace)][piece sums]
size_t lbq_gemv_batch_ws(const lbq_product* ps, int32_t n) {
  const Plan pl = plan_list(ps, n, sm_count(), nullptr);
  return kWsCounterBytes + pl.partial_floats * sizeof(float);
}

namespace {

// Sets the kernel's shared-memory limit (once per device) and checks that one CTA fits
// on an SM; the grid is one CTA per SM (the table takes most of the shared memory).
template <int FMT>
cudaError_t batch_grid(int* grid) {
  static PerDevice<int> cache;
  return cache.get(
      [](int, int* g) {
        cudaError_t r = cudaFuncSetAttribute(gemv_batch_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBatch));
        if (r != cudaSuccess) return r;
        int per_sm = 0;
        r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_batch_kernel<FMT>, kThreads, kSmemBatch);
        if (r != cudaSuccess) return r;
        if (per_sm < 1) return cudaErrorLaunchOutOfResources;  // one CTA does not fit an SM
        *g = sm_count() < kMaxGrid ? sm_count() : kMaxGrid;
        return cudaSuccess;
      },
      grid);
}

template <int FMT>
cudaError_t launch_list(const lbq_product* ps, int32_t n, void* ws, cudaStream_t s) {
  int grid = 0;
  cudaError_t e = batch_grid<FMT>(&grid);
  if (e != cudaSuccess) return e;
  unsigned* fault = lbq_fault_word();
  if (!fault) return cudaErrorInvalidDevicePointer;
  static thread_local BArgs a;  // 20 KB: off the stack
  const Plan pl = plan_list(ps, n, grid, a.p);
  a.partial = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsCounterBytes);
  a.fault = fault;
  a.W = pl.W;
  a.n = n;
  a.pad = 0;
  plan_cut(a.p, n, grid, pl.W, a.bound);
  gemv_batch_kernel<FMT><<<grid, kThreads, kSmemBatch, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (pl.max_split_rows > 0) {
    piece_sum_kernel<<<dim3((pl.max_split_rows + 255) / 256, n), 256, 0, s>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

cudaError_t lbq_launch_gemv_batch(const lbq_product* ps, int32_t n, void* ws, cudaStream_t s) {
  if (n < 1 || n > kMaxBatch) return cudaErrorInvalidValue;
  for (int32_t i = 1; i < n; ++i)
    if (ps[i].w.fmt != ps[0].w.fmt) return cudaErrorInvalidValue;  // one format a launch
  switch (ps[0].w.fmt) {
    case LBQ_TERN5: return launch_list<LBQ_TERN5>(ps, n, ws, s);
    case LBQ_SIGN1: return launch_list<LBQ_SIGN1>(ps, n, ws, s);
    case LBQ_Q2RHT: return launch_list<LBQ_Q2RHT>(ps, n, ws, s);
    default: return cudaErrorInvalidValue;
  }
}
