// noalloc.cu -- w8a8_linear_static_noalloc: the Decode linear without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run a
// Decode step: a plug-in running inside another runtime that owns all device
// memory and hands none out, or a latency-critical step where the
// device-wide synchronization an allocation may cause is not acceptable.
// This entry point needs no memory from them: its scratch (the statically
// quantized activation handed from the quantization kernel to the GEMM)
// lives in one file-scope device array of fixed size, which every GPU that
// loads the library holds until the process exits. It runs the two-kernel
// form of the Decode linear (quantization, then the decode GEMM), which gives
// the same result as the fused kernel of w8a8_linear_static.
#include <mutex>

#include "device.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

// Largest shape served from the static scratch.
constexpr int64_t kNoAllocMaxM = 32;
constexpr int64_t kNoAllocMaxN = 32768;
constexpr int64_t kNoAllocMaxK = 16384;
// the quantized activation, 32 tokens x 16384 bytes = 524,288 bytes.
constexpr size_t kNoAllocScratchBytes = kNoAllocMaxM * kNoAllocMaxK;

// One array per device (each device that loads the library holds its own
// copy). In host code this name is only a stand-in for the symbol, never a
// device address: the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the
// scratch array (zero-filled once, so it never holds stale bytes).
w8a8_status scratch_for_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return W8A8_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return W8A8_ERR_CUDA;
    }
    if (cudaMemset(ptr, 0, kNoAllocScratchBytes) != cudaSuccess) {
      cudaGetLastError();
      return W8A8_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return W8A8_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace w8a8

using namespace w8a8;

extern "C" w8a8_status w8a8_linear_static_noalloc(const void *X, int64_t M, int64_t K, int64_t ldx, const float *S,
                                                  const float *r, const int32_t *Z, const int8_t *Wq,
                                                  const float *s_w, const int32_t *colsum, const float *bias,
                                                  int64_t N, void *out, w8a8_dtype out_dtype, void *stream) {
  if (M < 0 || N < 0 || K <= 0 || ldx < K) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (M > kNoAllocMaxM || N > kNoAllocMaxN || K > kNoAllocMaxK) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (out_dtype != W8A8_BF16 && out_dtype != W8A8_FP32 && out_dtype != W8A8_I32) return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!X || !S || !r || !Z || !Wq || !s_w || !colsum || !out) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(X) || (ldx % 8) != 0 || !aligned16(Wq) || !aligned16(s_w) || !aligned16(colsum) ||
      !aligned16(out) || (bias && !aligned16(bias)))
    return W8A8_ERR_MISALIGNED;
  int sms = 0;
  int32_t *status = nullptr;
  if (w8a8_status s = current_device_info(&sms, &status)) return s;
  void *scratch = nullptr;
  if (w8a8_status s = scratch_for_current_device(&scratch)) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int8_t *Xq = static_cast<int8_t *>(scratch);  // every byte read is written first by this call
  if (launch_quant_per_tensor(static_cast<const uint16_t *>(X), M, K, ldx, r, Z, Xq, sms, st, /*pdl=*/true) !=
      cudaSuccess)
    return W8A8_ERR_CUDA;
  EpilogueArgs ep;
  ep.S_x = S;
  ep.s_x_per_row = 0;
  ep.Z = Z;
  ep.colsum = colsum;
  ep.s_w = s_w;
  ep.bias = bias;
  ep.out = out;
  ep.out_dtype = out_dtype;
  return launch_gemm_decode(Xq, K, Wq, M, N, K, ep, status, st) == cudaSuccess ? W8A8_OK : W8A8_ERR_CUDA;
}
