// lbq_common.cuh -- shared device/host helpers of the CUDA library (not of the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "lbq.h"

namespace lbq {

// Layout constants of the packed formats (byte layouts are documented in lbq.h).
constexpr int kTernBlock = 128;       // weights per ternary block
constexpr int kTernBlockBytes = 28;   // 26 code bytes + fp16 scale
constexpr int kTernCodeBytes = 26;
constexpr int kSignBlock = 128;       // weights per sign scale
constexpr int kQ2Block = 32;          // weights per 2-bit scale
constexpr int kRhtBlock = 512;        // Hadamard block size
// Workspace layout shared by every product: [0, kWsCounterBytes) holds arrival
// counters that must be zero when a call starts and are zero again when it ends;
// the scratch data of a call starts at kWsCounterBytes. Keeping the counters at a
// fixed place lets one workspace serve matrices of any shape in turn.
constexpr size_t kWsCounterBytes = 65536;
constexpr int64_t kMaxSplitRows = static_cast<int64_t>(kWsCounterBytes / 4) * 32;
// 2^-4.5 = 1/sqrt(512), rounded to fp32.
constexpr float kRhtNorm = 0.044194173824159216f;

// Storage order shared by every format: rows are interleaved in groups of four. In
// group g (rows 4g .. 4g+3), 32-bit word w of row 4g+q sits at byte 16 w + 4 q of the
// group's 4 * code_stride bytes, and scale e of row 4g+q at element 4 e + q of its
// 4 * scale_stride fp16. One 16-byte load then brings the same word of four rows.
__host__ __device__ __forceinline__ int64_t g4_rows(int64_t N) { return (N + 3) / 4 * 4; }
__host__ __device__ __forceinline__ int64_t g4_word_byte(int64_t n, int64_t w, int64_t stride) {
  return (n >> 2) * 4 * stride + w * 16 + (n & 3) * 4;
}
__host__ __device__ __forceinline__ int64_t g4_scale_elem(int64_t n, int64_t e, int64_t sstride) {
  return (n >> 2) * 4 * sstride + e * 4 + (n & 3);
}

struct Layout {
  int64_t code_stride;   // bytes per row of codes
  int64_t scale_stride;  // fp16 scales per row (0: scales in-block)
  int64_t block;         // weights per scale
};

// Returns false on an unknown format or a K that violates the shape rules.
inline bool layout_of(int32_t fmt, int64_t K, Layout* L) {
  if (K < 128 || K % 128) return false;
  switch (fmt) {
    case LBQ_TERN5:
      L->code_stride = ((K / kTernBlock) * kTernBlockBytes + 15) / 16 * 16;
      L->scale_stride = 0;
      L->block = kTernBlock;
      return true;
    case LBQ_SIGN1:
      L->code_stride = K / 8;
      L->scale_stride = (K / kSignBlock + 7) / 8 * 8;  // 16-byte rows of scales
      L->block = kSignBlock;
      return true;
    case LBQ_Q2RHT:
      if (K % kRhtBlock) return false;
      L->code_stride = K / 4;
      L->scale_stride = K / kQ2Block;
      L->block = kQ2Block;
      return true;
    default:
      return false;
  }
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kMaxDevices = 64;

// A value computed once per device, on first use with that device current, from any
// number of host threads: the first caller for a device runs `make` under a lock; a
// failed `make` is retried on the next call. Later calls read it without the lock.
template <typename T>
class PerDevice {
 public:
  // `make(dev, &value)` returns cudaSuccess once it has stored the value.
  template <typename F>
  cudaError_t get(F&& make, T* out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!ready_[dev].load(std::memory_order_acquire)) {
      std::lock_guard<std::mutex> lock(mu_);
      if (!ready_[dev].load(std::memory_order_relaxed)) {
        e = make(dev, &val_[dev]);
        if (e != cudaSuccess) return e;
        ready_[dev].store(true, std::memory_order_release);
      }
    }
    *out = val_[dev];
    return cudaSuccess;
  }

 private:
  std::mutex mu_;
  std::atomic<bool> ready_[kMaxDevices] = {};
  T val_[kMaxDevices] = {};
};

// SM count of the current device (148 on B200; 148 if the query fails).
inline int sm_count() {
  static PerDevice<int> cache;
  int n = 0;
  const cudaError_t e = cache.get(
      [](int dev, int* v) {
        int c = 0;
        const cudaError_t r = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
        if (r != cudaSuccess || c <= 0) return r != cudaSuccess ? r : cudaErrorInvalidValue;
        *v = c;
        return cudaSuccess;
      },
      &n);
  return e == cudaSuccess ? n : 148;
}

}  // namespace lbq

// LBQ_OK for cudaSuccess; otherwise records e as the calling thread's last CUDA error
// (lbq_last_cuda_error) and returns LBQ_ERR_CUDA (api.cu).
lbq_status lbq_cuda_status(cudaError_t e);

// Launch helpers implemented in the individual .cu files; all return cudaError_t
// from cudaGetLastError() after the launch.
cudaError_t lbq_launch_pack(int32_t fmt, const float* W, int64_t K, int64_t N, uint8_t* codes,
                            uint16_t* scales, const lbq::Layout& L, cudaStream_t s);
cudaError_t lbq_launch_unpack(const lbq_weights* w, const lbq::Layout& L, int8_t* out,
                              float* scales_out, cudaStream_t s);
cudaError_t lbq_launch_rht_signs(uint64_t seed, int64_t K, int8_t* D, cudaStream_t s);
cudaError_t lbq_launch_hadamard(const uint16_t* x, const int8_t* D, int64_t M, int64_t K,
                                float* out, cudaStream_t s);
size_t lbq_gemv_workspace(const lbq_weights* w);
// Every argument check lbq_gemv makes except the workspace's, with the same statuses
// (api.cu).
lbq_status lbq_validate_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                             const uint16_t* y);
// Device address of the word bounded device waits report to (current device), or NULL.
unsigned* lbq_fault_word();
// Launches the kernel whose bounded wait runs out on purpose (selftest.cu).
cudaError_t lbq_launch_wait_selftest(cudaStream_t s);
// y (bf16) or, when y32 is set, y32 (fp32, no rounding) receives the product.
cudaError_t lbq_launch_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                            uint16_t* y, float* y32, void* ws, cudaStream_t s);
size_t lbq_gemm_workspace(const lbq_weights* w, int64_t M);
// The batched batch-1 products (gemv_batch.cu): workspace for a list of at most
// LBQ_BATCH_MAX products, and one launch over such a list.
size_t lbq_gemv_batch_ws(const lbq_product* ps, int32_t n);
int64_t lbq_gemv_batch_plan_list(const lbq_product* ps, int32_t n, int ctas, int32_t* pieces,
                                 int64_t* bound);
cudaError_t lbq_launch_gemv_batch(const lbq_product* ps, int32_t n, void* ws, cudaStream_t s);
size_t lbq_gemm_tc_workspace(const lbq_weights* w, int64_t M);
cudaError_t lbq_launch_gemm_tc(const lbq_weights* w, const uint16_t* X, int64_t M, uint16_t* Y,
                               void* ws, cudaStream_t s);
cudaError_t lbq_launch_gemm(const lbq_weights* w, const uint16_t* X, int64_t M, const int8_t* D,
                            uint16_t* Y, void* ws, cudaStream_t s);
