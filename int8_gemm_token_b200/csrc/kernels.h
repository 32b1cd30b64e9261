// kernels.h -- launchers of libw8a8's kernels (internal; the public ABI is
// include/w8a8.h). Every launcher returns the launch's cudaError_t.
#pragma once

#include <atomic>

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/w8a8.h"

namespace w8a8 {

// Operands of the fused dequant epilogue (see w8a8_gemm_dequant and
// int8_mixed_decomp_gemm in include/w8a8.h for the per-element formula).
struct EpilogueArgs {
  const float *S_x = nullptr;  // [M] or scalar
  int32_t s_x_per_row = 1;
  const int32_t *Z = nullptr;       // scalar or null
  const int32_t *colsum = nullptr;  // [N], needed when Z != null
  const float *s_w = nullptr;       // [N]
  const float *bias = nullptr;      // [N] or null
  // LLM.int8() side path (mixed mode only)
  const uint16_t *Xo = nullptr;       // [M, cap] bf16
  const int32_t *outlier_idx = nullptr;
  const int32_t *n_out = nullptr;     // device scalar
  int32_t cap = 0;
  const uint16_t *W = nullptr;        // [K, N] bf16, row stride ldw
  int64_t ldw = 0;
  // output
  void *out = nullptr;  // [M, N] dense
  int32_t out_dtype = W8A8_BF16;  // a public w8a8_dtype, or kOutRequantI8
  // kOutRequantI8 (Decode-shaped GEMM only): out is int8, the next linear's
  // static code of the bf16 result, clamp(rne(bf16(y) * r_out) + Z_out, -128, 127)
  const float *r_out = nullptr;    // device scalar
  const int32_t *z_out = nullptr;  // device scalar
};
constexpr int32_t kOutRequantI8 = 16;  // internal; not a public dtype code

// Once per kernel and device: raise the kernel's dynamic shared-memory limit to
// at least `bytes` (and ask for the largest shared-memory carveout). Later
// calls with no larger size skip the driver calls.
template <auto Kernel>
cudaError_t ensure_kernel_smem(int bytes, bool max_carveout) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> set_bytes[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && set_bytes[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && max_carveout)
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
    int prev = set_bytes[dev].load(std::memory_order_relaxed);
    while (prev < bytes && !set_bytes[dev].compare_exchange_weak(prev, bytes)) {
    }
  }
  return e;
}

cudaError_t launch_quant_per_token(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   int8_t *Xq, float *S_x, int num_sms, cudaStream_t s);
// pdl = true: may start while the previous kernel runs. It lets its own
// dependents (the decode GEMM) launch at once, then waits for the previous
// kernel before reading or writing anything.
cudaError_t launch_quant_per_tensor(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                    const float *r, const int32_t *Z, int8_t *Xq, int num_sms,
                                    cudaStream_t s, bool pdl = false);
// out [M, K] dense = S * (Xq - Z) as bf16 (bf16_out) or fp32; K a multiple of 16.
cudaError_t launch_dequant_per_tensor(const int8_t *Xq, int64_t M, int64_t K, int64_t ldq, const float *S,
                                      const int32_t *Z, void *out, bool bf16_out, int num_sms, cudaStream_t s);
// The same two conversions for large dense tensors (rows of exactly K
// elements), streamed through shared memory with bulk copies (stream.cu).
cudaError_t launch_quant_per_tensor_stream(const uint16_t *X, int64_t elems, const float *r, const int32_t *Z,
                                           int8_t *Xq, int num_sms, int32_t *status, cudaStream_t s);
cudaError_t launch_dequant_per_tensor_stream(const int8_t *Xq, int64_t elems, const float *S, const int32_t *Z,
                                             void *out, bool bf16_out, int num_sms, int32_t *status,
                                             cudaStream_t s);
cudaError_t launch_calibrate(const void *X, w8a8_dtype dt, int64_t T, int64_t K, int64_t ldx,
                             float *S, float *r, int32_t *Z, int num_sms, cudaStream_t s);
cudaError_t launch_quant_weight(const void *W, w8a8_dtype dt, int64_t K, int64_t N, int64_t ldw,
                                int8_t *Wq, float *s_w, int32_t *colsum, cudaStream_t s);

// tcgen05 GEMM + epilogue (prefill-sized M; any M works). mixed selects the
// LLM.int8() side path in the epilogue.
cudaError_t launch_gemm_tc(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                           const EpilogueArgs &ep, bool mixed, int num_sms, int32_t *status,
                           cudaStream_t s);

// LLM.int8() mixed GEMM with the 16-bit side product on the tensor cores
// (CTA pairs, one int32 and one fp32 TMEM accumulator per tile; any M). A
// gather kernel first writes the side operands, zero-padded to whole 64-column
// k-blocks, into `workspace` (side_workspace_bytes(M, N, cap) bytes).
cudaError_t launch_gemm_side_tc(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                                const EpilogueArgs &ep, void *workspace, int num_sms, int32_t *status,
                                cudaStream_t s);
size_t side_workspace_bytes(int64_t M, int64_t N, int32_t cap);

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t *status, cudaStream_t s);

// Decode-shaped GEMM (M <= 64): one cluster of decode_split(M, N, K) CTAs
// per 128-row weight tile, partial sums reduced through distributed shared
// memory (no workspace). Launched with programmatic dependent launch: it may
// start while the previous kernel in the stream runs, streams its first
// weight tiles at once and waits for that kernel before reading Xq or S_x,
// s_w, colsum, bias and before writing `out` (so a kernel that lets its
// dependents launch early must not write Wq).
cudaError_t launch_gemm_decode(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                               const EpilogueArgs &ep, int32_t *status, cudaStream_t s);
// The Decode linear in one kernel (M <= 32): the same GEMM, with the static
// per-tensor quantization of bf16 X (row stride ldx elements, device scalars
// r and Z) done inside it on each activation k-block before the MMAs read it.
cudaError_t launch_linear_static_decode(const uint16_t *X, int64_t ldx, const float *r, const int32_t *Z,
                                        const int8_t *Wq, int64_t M, int64_t N, int64_t K, const EpilogueArgs &ep,
                                        int32_t *status, cudaStream_t s);
// Cluster size the decode GEMM uses for this shape on the current device.
int decode_split(int64_t M, int64_t N, int64_t K, bool fused_quant);

// LLM.int8() outlier split: column-flag pass into a K-bit bitmap in
// `workspace` (outlier_workspace_bytes(K); zeroed by the launcher), then the
// masked per-row quantization and outlier gather.
cudaError_t launch_outlier_split(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, float threshold, int32_t cap,
                                 int8_t *Xq, float *S_x, int32_t *idx, int32_t *n_out, uint16_t *Xo, void *workspace,
                                 int num_sms, int32_t *status, cudaStream_t s);
size_t outlier_workspace_bytes(int64_t K);

// Per-device set-up of the C ABI (done once per device): SM count and the
// device address of the device status word.
w8a8_status current_device_info(int *sm_count, int32_t **status_word);

// 2-D tensor map (driver entry point resolved once per process): inner and
// outer extents in elements, row stride in bytes, box in elements; swizzle128
// selects the 128-byte swizzle (box inner extent must then be 128 bytes).
enum class TmapType { kU8, kBF16, kF32 };
bool encode_tmap_2d(void *map, const void *base, TmapType type, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);

}  // namespace w8a8
