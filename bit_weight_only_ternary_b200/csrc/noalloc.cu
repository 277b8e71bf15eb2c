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
#include "lbq_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_lbq_scratch[LBQ_NOALLOC_SCRATCH_BYTES];

// The array's device address, looked up once per device with that device current.
// Host code must not pass the symbol itself to a kernel: on the host it is only a
// stand-in, not a device address.
lbq_status scratch_for_current_device(void** out) {
  static lbq::PerDevice<void*> addr;
  const cudaError_t e = addr.get(
      [](int, void** v) {
        void* p = nullptr;
        const cudaError_t r = cudaGetSymbolAddress(&p, g_lbq_scratch);
        if (r != cudaSuccess) return r;
        if (!p) return cudaErrorInvalidSymbol;
        *v = p;
        return cudaSuccess;
      },
      out);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return lbq_cuda_status(e);
  }
  return LBQ_OK;
}

}  // namespace

extern "C" lbq_status lbq_gemv_noalloc(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                                       uint16_t* y, void* stream) {
  // the same checks, in the same order, as lbq_gemv; then the scratch size
  const lbq_status st = lbq_validate_gemv(w, x, D, y);
  if (st != LBQ_OK) return st;
  const size_t need = lbq_workspace_bytes(w, 1);
  if (need > LBQ_NOALLOC_SCRATCH_BYTES) return LBQ_ERR_WORKSPACE;
  if (need == 0) return lbq_gemv(w, x, D, y, nullptr, 0, stream);
  void* scratch = nullptr;
  const lbq_status sst = scratch_for_current_device(&scratch);
  if (sst != LBQ_OK) return sst;
  // Nothing needs clearing: the batch-1 product writes every slice sum before it reads
  // it, and never touches the arrival counters at the array's start, which are zero
  // since the library was loaded (static device memory starts zeroed).
  return lbq_gemv(w, x, D, y, scratch, LBQ_NOALLOC_SCRATCH_BYTES, stream);
}
