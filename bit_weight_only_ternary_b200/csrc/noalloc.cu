// noalloc.cu -- lbq_gemv_noalloc: the batch-1 product for callers that cannot allocate
// device memory, with its scratch in a fixed array compiled into the library.
//
// Some callers have no way to hand the library a workspace: a host that embeds the
// library through its C interface and has no device allocator of its own, or one that
// must not call cudaMalloc after start-up (cudaMalloc can synchronise the device and
// stall every stream, and a framework's memory pool does not see memory allocated
// behind its back). This entry point needs no workspace argument: it uses
// g_lbq_scratch below. The array costs LBQ_NOALLOC_SCRATCH_BYTES on every GPU that
// loads the library, for the life of the process.
#include <mutex>

#include "lbq_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_lbq_scratch[LBQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// The array's device address, looked up once per device with that device current.
// Host code must not pass the symbol itself to a kernel: on the host it is only a
// stand-in, not a device address.
lbq_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LBQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lbq_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LBQ_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LBQ_OK;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

}  // namespace

extern "C" lbq_status lbq_gemv_noalloc(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                                       uint16_t* y, void* stream) {
  const size_t need = lbq_workspace_bytes(w, 1);  // 0 for an invalid descriptor
  if (need > LBQ_NOALLOC_SCRATCH_BYTES) return LBQ_ERR_WORKSPACE;
  if (need == 0) return lbq_gemv(w, x, D, y, nullptr, 0, stream);  // validates everything
  // A scratch is needed, so the descriptor is valid; check the remaining arguments now,
  // so that nothing is enqueued on a bad call.
  if (!x || !y || (w->fmt == LBQ_Q2RHT && !D)) return LBQ_ERR_ARG;
  if (!aligned(x, 16) || !aligned(y, 2) || (D && !aligned(D, 16))) return LBQ_ERR_ALIGN;
  void* scratch = nullptr;
  lbq_status st = scratch_for_current_device(&scratch);
  if (st != LBQ_OK) return st;
  // The array keeps whatever the previous call left; the product expects a zeroed
  // workspace, so clear the part this call uses.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) {
    cudaGetLastError();
    return LBQ_ERR_CUDA;
  }
  return lbq_gemv(w, x, D, y, scratch, LBQ_NOALLOC_SCRATCH_BYTES, stream);
}
