// api.cu -- the C ABI (include/lbq.h): host-side validation, then one or more launches.
// Nothing is enqueued unless every argument passes; launch failures map to LBQ_ERR_CUDA.
#include <vector>

#include "lbq_common.cuh"

namespace {

using lbq::Layout;

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline lbq_status from_cuda(cudaError_t e) { return lbq_cuda_status(e); }

// Up to kTernPerTokenMaxM tokens a ternary product runs as one batch-1 product per
// token: on the tensor cores a 16-token tile costs about as much as a 2-token one
// (each N = 16 MMA is bound by its issue, not by its work), ~125 us per 27B-shaped
// layer, while a batch-1 product costs ~38 us per layer and token (measured: at 8
// tokens the per-token products took 2.4 times as long as the tensor cores).
constexpr int64_t kTernPerTokenMaxM = 3;

inline bool per_token(const lbq_weights* w, int64_t M) {
  if (M == 1) return true;
  return w->fmt == LBQ_TERN5 && M <= kTernPerTokenMaxM &&
         !(lbq_gemv_workspace(w) && w->N > lbq::kMaxSplitRows);
}

inline bool fmt_known(int32_t fmt) {
  return fmt == LBQ_TERN5 || fmt == LBQ_SIGN1 || fmt == LBQ_Q2RHT;
}

// Checks a weight descriptor; fills L on success.
lbq_status check_weights(const lbq_weights* w, Layout* L) {
  if (!w) return LBQ_ERR_ARG;
  if (!fmt_known(w->fmt)) return LBQ_ERR_FORMAT;
  if (w->reserved != 0) return LBQ_ERR_ARG;
  if (w->N < 1 || !lbq::layout_of(w->fmt, w->K, L)) return LBQ_ERR_SHAPE;
  if (!w->codes) return LBQ_ERR_ARG;
  if (!aligned(w->codes, 16)) return LBQ_ERR_ALIGN;
  if (w->code_stride < L->code_stride || w->code_stride % 16) return LBQ_ERR_SHAPE;
  if (w->fmt == LBQ_TERN5) {
    if (w->scales || w->scale_stride != 0) return LBQ_ERR_ARG;
  } else {
    if (!w->scales) return LBQ_ERR_ARG;
    if (!aligned(w->scales, 16)) return LBQ_ERR_ALIGN;
    if (w->scale_stride < L->scale_stride || w->scale_stride % 8) return LBQ_ERR_SHAPE;
  }
  return LBQ_OK;
}

// Every check of a product call but the workspace's.
lbq_status check_operands(const lbq_weights* w, const void* x, int64_t M, const int8_t* D,
                          const void* y, Layout* L) {
  lbq_status st = check_weights(w, L);
  if (st != LBQ_OK) return st;
  if (M < 1) return LBQ_ERR_SHAPE;
  if (!x || !y) return LBQ_ERR_ARG;
  if (!aligned(x, 16) || !aligned(y, 2)) return LBQ_ERR_ALIGN;
  if (w->fmt == LBQ_Q2RHT) {
    if (!D) return LBQ_ERR_ARG;
    if (!aligned(D, 16)) return LBQ_ERR_ALIGN;
  }
  if (M == 1 && lbq_gemv_workspace(w) && w->N > lbq::kMaxSplitRows) return LBQ_ERR_SHAPE;
  return LBQ_OK;
}

lbq_status check_product(const lbq_weights* w, const void* x, int64_t M, const int8_t* D,
                         const void* y, void* ws, size_t ws_bytes, Layout* L) {
  lbq_status st = check_operands(w, x, M, D, y, L);
  if (st != LBQ_OK) return st;
  const size_t need = lbq_workspace_bytes(w, M);
  if (need) {
    if (!ws || ws_bytes < need) return LBQ_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return LBQ_ERR_ALIGN;
  }
  return LBQ_OK;
}

}  // namespace

lbq_status lbq_validate_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                             const uint16_t* y) {
  Layout L;
  return check_operands(w, x, 1, D, y, &L);
}

namespace {

// Byte ranges [lo, hi) overlap.
inline bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// A batch list: every product valid on its own (as for lbq_gemv, without its limit on
// split rows, which the batch kernel does not have), and no output overlapping an
// input or another output.
lbq_status check_batch(const lbq_product* ps, int32_t n) {
  if (!ps || n < 1) return LBQ_ERR_ARG;
  for (int32_t i = 0; i < n; ++i) {
    Layout L;
    const lbq_weights* w = &ps[i].w;
    lbq_status st = check_weights(w, &L);
    if (st != LBQ_OK) return st;
    if (w->N > (int64_t{1} << 28)) return LBQ_ERR_SHAPE;
    if (!ps[i].x || !ps[i].y) return LBQ_ERR_ARG;
    if (!aligned(ps[i].x, 16) || !aligned(ps[i].y, 2)) return LBQ_ERR_ALIGN;
    if (w->fmt == LBQ_Q2RHT) {
      if (!ps[i].D) return LBQ_ERR_ARG;
      if (!aligned(ps[i].D, 16)) return LBQ_ERR_ALIGN;
    }
  }
  for (int32_t i = 0; i < n; ++i) {
    const size_t ny = static_cast<size_t>(ps[i].w.N) * 2;
    for (int32_t k = 0; k < n; ++k) {
      const size_t nx = static_cast<size_t>(ps[k].w.K) * 2;
      if (overlap(ps[i].y, ny, ps[k].x, nx)) return LBQ_ERR_ARG;
      if (ps[k].D && overlap(ps[i].y, ny, ps[k].D, static_cast<size_t>(ps[k].w.K))) return LBQ_ERR_ARG;
      if (k != i && overlap(ps[i].y, ny, ps[k].y, static_cast<size_t>(ps[k].w.N) * 2)) return LBQ_ERR_ARG;
    }
  }
  return LBQ_OK;
}

}  // namespace

namespace {
thread_local int g_last_cuda_error = 0;
}  // namespace

lbq_status lbq_cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LBQ_OK;
  g_last_cuda_error = static_cast<int>(e);
  return LBQ_ERR_CUDA;
}

// The launches of a batch: the kernel runs one format a launch, so a list of several
// runs as one launch (or chunk of LBQ_BATCH_MAX) per format present, in the list's
// order within each format. fn(list, count) returns false to stop.
template <typename F>
void for_each_batch_launch(const lbq_product* ps, int32_t n, F fn) {
  bool one_format = true;
  for (int32_t i = 1; i < n; ++i) one_format = one_format && ps[i].w.fmt == ps[0].w.fmt;
  std::vector<lbq_product> sub;
  for (const int32_t fmt : {LBQ_TERN5, LBQ_SIGN1, LBQ_Q2RHT}) {
    const lbq_product* list = ps;
    int32_t count = n;
    if (!one_format) {
      sub.clear();
      for (int32_t i = 0; i < n; ++i)
        if (ps[i].w.fmt == fmt) sub.push_back(ps[i]);
      list = sub.data();
      count = static_cast<int32_t>(sub.size());
    } else if (ps[0].w.fmt != fmt) {
      continue;
    }
    for (int32_t i = 0; i < count; i += LBQ_BATCH_MAX)
      if (!fn(list + i, count - i < LBQ_BATCH_MAX ? count - i : LBQ_BATCH_MAX)) return;
  }
}

extern "C" {

int32_t lbq_last_cuda_error(void) { return g_last_cuda_error; }

const char* lbq_last_cuda_error_string(void) {
  return g_last_cuda_error ? cudaGetErrorString(static_cast<cudaError_t>(g_last_cuda_error)) : "no error";
}

const char* lbq_status_string(lbq_status st) {
  switch (st) {
    case LBQ_OK: return "ok";
    case LBQ_ERR_ARG: return "invalid argument (null pointer or bad value)";
    case LBQ_ERR_SHAPE: return "invalid shape or stride";
    case LBQ_ERR_ALIGN: return "misaligned pointer";
    case LBQ_ERR_FORMAT: return "unknown packed format";
    case LBQ_ERR_CUDA: return "CUDA error";
    case LBQ_ERR_WORKSPACE: return "workspace missing or too small";
    case LBQ_ERR_DEVICE_WAIT: return "a bounded wait inside a kernel gave up";
    default: return "unknown status";
  }
}

lbq_status lbq_packed_layout(int32_t fmt, int64_t K, int64_t N, int64_t* code_stride,
                             int64_t* scale_stride, size_t* code_bytes, size_t* scale_bytes) {
  if (!fmt_known(fmt)) return LBQ_ERR_FORMAT;
  Layout L;
  if (N < 1 || !lbq::layout_of(fmt, K, &L)) return LBQ_ERR_SHAPE;
  if (code_stride) *code_stride = L.code_stride;
  if (scale_stride) *scale_stride = L.scale_stride;
  const size_t rows = static_cast<size_t>(lbq::g4_rows(N));  // padded to whole groups of four
  if (code_bytes) *code_bytes = rows * static_cast<size_t>(L.code_stride);
  if (scale_bytes) *scale_bytes = rows * static_cast<size_t>(L.scale_stride) * 2;
  return LBQ_OK;
}

lbq_status lbq_pack(int32_t fmt, const float* W, int64_t K, int64_t N, void* codes, void* scales,
                    void* stream) {
  if (!fmt_known(fmt)) return LBQ_ERR_FORMAT;
  Layout L;
  if (N < 1 || !lbq::layout_of(fmt, K, &L)) return LBQ_ERR_SHAPE;
  if (!W || !codes) return LBQ_ERR_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16)) return LBQ_ERR_ALIGN;
  if (fmt == LBQ_TERN5) {
    if (scales) return LBQ_ERR_ARG;
  } else {
    if (!scales) return LBQ_ERR_ARG;
    if (!aligned(scales, 16)) return LBQ_ERR_ALIGN;
  }
  return from_cuda(lbq_launch_pack(fmt, W, K, N, static_cast<uint8_t*>(codes),
                                   static_cast<uint16_t*>(scales), L, as_stream(stream)));
}

lbq_status lbq_unpack(const lbq_weights* w, int8_t* out, float* scales_out, void* stream) {
  Layout L;
  lbq_status st = check_weights(w, &L);
  if (st != LBQ_OK) return st;
  if (!out) return LBQ_ERR_ARG;
  if (scales_out && !aligned(scales_out, 4)) return LBQ_ERR_ALIGN;
  return from_cuda(lbq_launch_unpack(w, L, out, scales_out, as_stream(stream)));
}

lbq_status lbq_rht_signs(uint64_t seed, int64_t K, int8_t* D, void* stream) {
  if (!D) return LBQ_ERR_ARG;
  if (K < 1) return LBQ_ERR_SHAPE;
  return from_cuda(lbq_launch_rht_signs(seed, K, D, as_stream(stream)));
}

lbq_status lbq_hadamard(const uint16_t* x, const int8_t* D, int64_t M, int64_t K, float* out,
                        void* stream) {
  if (!x || !D || !out) return LBQ_ERR_ARG;
  if (M < 1 || K < lbq::kRhtBlock || K % lbq::kRhtBlock) return LBQ_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(D, 16) || !aligned(out, 16)) return LBQ_ERR_ALIGN;
  return from_cuda(lbq_launch_hadamard(x, D, M, K, out, as_stream(stream)));
}

lbq_status lbq_device_fault(uint32_t* code) {
  if (!code) return LBQ_ERR_ARG;
  unsigned* word = lbq_fault_word();
  if (!word) return lbq_cuda_status(cudaErrorInvalidDevicePointer);
  unsigned v = 0;
  cudaError_t e = cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return lbq_cuda_status(e);
  if (v && (e = cudaMemset(word, 0, sizeof(v))) != cudaSuccess) return lbq_cuda_status(e);
  *code = v;
  return v ? LBQ_ERR_DEVICE_WAIT : LBQ_OK;
}

lbq_status lbq_selftest_wait(void* stream) { return from_cuda(lbq_launch_wait_selftest(as_stream(stream))); }

size_t lbq_workspace_bytes(const lbq_weights* w, int64_t M) {
  Layout L;
  if (check_weights(w, &L) != LBQ_OK || M < 1) return 0;
  return per_token(w, M) ? lbq_gemv_workspace(w) : lbq_gemm_workspace(w, M);
}

lbq_status lbq_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D, uint16_t* y,
                    void* workspace, size_t workspace_bytes, void* stream) {
  Layout L;
  lbq_status st = check_product(w, x, 1, D, y, workspace, workspace_bytes, &L);
  if (st != LBQ_OK) return st;
  return from_cuda(lbq_launch_gemv(w, x, D, y, nullptr, workspace, as_stream(stream)));
}

lbq_status lbq_gemv_f32(const lbq_weights* w, const uint16_t* x, const int8_t* D, float* y,
                        void* workspace, size_t workspace_bytes, void* stream) {
  Layout L;
  lbq_status st = check_product(w, x, 1, D, y, workspace, workspace_bytes, &L);
  if (st != LBQ_OK) return st;
  if (!aligned(y, 4)) return LBQ_ERR_ALIGN;
  return from_cuda(lbq_launch_gemv(w, x, D, nullptr, y, workspace, as_stream(stream)));
}

size_t lbq_gemv_batch_workspace_bytes(const lbq_product* ps, int32_t n) {
  if (check_batch(ps, n) != LBQ_OK) return 0;
  size_t need = 0;
  for_each_batch_launch(ps, n, [&](const lbq_product* list, int32_t count) {
    const size_t b = lbq_gemv_batch_ws(list, count);
    if (b > need) need = b;
    return true;
  });
  return need;
}

lbq_status lbq_gemv_batch(const lbq_product* ps, int32_t n, void* workspace,
                          size_t workspace_bytes, void* stream) {
  lbq_status st = check_batch(ps, n);
  if (st != LBQ_OK) return st;
  const size_t need = lbq_gemv_batch_workspace_bytes(ps, n);
  if (!workspace || workspace_bytes < need) return LBQ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return LBQ_ERR_ALIGN;
  for_each_batch_launch(ps, n, [&](const lbq_product* list, int32_t count) {
    const cudaError_t e = lbq_launch_gemv_batch(list, count, workspace, as_stream(stream));
    if (e != cudaSuccess) {
      cudaGetLastError();
      st = lbq_cuda_status(e);
      return false;
    }
    return true;
  });
  return st;
}

lbq_status lbq_gemv_batch_plan(const lbq_product* ps, int32_t n, int32_t ctas, int32_t* pieces,
                               int64_t* bound, int64_t* total) {
  if (!pieces || !bound || !total || ctas < 1 || ctas > LBQ_BATCH_MAX_CTAS || n > LBQ_BATCH_MAX)
    return LBQ_ERR_ARG;
  const lbq_status st = check_batch(ps, n);
  if (st != LBQ_OK) return st;
  for (int32_t i = 1; i < n; ++i)
    if (ps[i].w.fmt != ps[0].w.fmt) return LBQ_ERR_ARG;
  *total = lbq_gemv_batch_plan_list(ps, n, ctas, pieces, bound);
  return LBQ_OK;
}

lbq_status lbq_gemm(const lbq_weights* w, const uint16_t* X, int64_t M, const int8_t* D,
                    uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream) {
  Layout L;
  lbq_status st = check_product(w, X, M, D, Y, workspace, workspace_bytes, &L);
  if (st != LBQ_OK) return st;
  if (per_token(w, M)) {
    if (lbq_gemv_workspace(w) && w->N > lbq::kMaxSplitRows) return LBQ_ERR_SHAPE;
    // one batch-1 product per token, in stream order (they share the workspace)
    for (int64_t m = 0; m < M; ++m) {
      const cudaError_t e =
          lbq_launch_gemv(w, X + m * w->K, D, Y + m * w->N, nullptr, workspace, as_stream(stream));
      if (e != cudaSuccess) return lbq_cuda_status(e);
    }
    return LBQ_OK;
  }
  return from_cuda(lbq_launch_gemm(w, X, M, D, Y, workspace, as_stream(stream)));
}

}  // extern "C"
