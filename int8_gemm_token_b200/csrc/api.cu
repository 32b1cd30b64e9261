// api.cu -- the extern "C" entry points of libw8a8 (declared and documented
// in include/w8a8.h): host-side argument checks, per-device set-up and the
// dispatch to the kernels. No entry point allocates device memory.
#include <cudaTypedefs.h>

#include <mutex>

#include "device.cuh"
#include "kernels.h"

namespace w8a8 {

// One status word per device (each device holds its own copy of this
// variable); kernels get its device address from DeviceInfo.
__device__ int32_t g_device_status = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  int32_t *status = nullptr;  // device address of g_device_status on this device
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

// Per-device set-up, done once with the device current: SM count, compute
// capability check, device address of the status word.
w8a8_status device_info(DeviceInfo **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return W8A8_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo &d = g_devices[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return W8A8_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return W8A8_ERR_NO_DEVICE;  // built for sm_100a only
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
      cudaGetLastError();
      return W8A8_ERR_CUDA;
    }
    d.sm_count = sms;
    d.status = static_cast<int32_t *>(p);
    d.ready = true;
  }
  *out = &d;
  return W8A8_OK;
}

}  // namespace

w8a8_status current_device_info(int *sm_count, int32_t **status_word) {
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  *sm_count = d->sm_count;
  *status_word = d->status;
  return W8A8_OK;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

w8a8_status from_cuda(cudaError_t e) { return e == cudaSuccess ? W8A8_OK : W8A8_ERR_CUDA; }

w8a8_status check_k(int64_t K) {
  if (K <= 0) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > 65536) return W8A8_ERR_UNSUPPORTED_SHAPE;
  return W8A8_OK;
}

// bf16 activation [M, K] with row stride ldx (elements).
w8a8_status check_bf16_rows(const void *X, int64_t M, int64_t K, int64_t ldx) {
  if (M < 0) return W8A8_ERR_INVALID_ARG;
  if (w8a8_status s = check_k(K)) return s;
  if (ldx < K) return W8A8_ERR_INVALID_ARG;
  if (M > 0 && !X) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(X) || (ldx % 8) != 0) return W8A8_ERR_MISALIGNED;
  return W8A8_OK;
}

}  // namespace

bool encode_tmap_2d(void *map, const void *base, TmapType type, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
      cudaGetLastError();
  });
  if (!g_encode) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(static_cast<CUtensorMap *>(map),
                        type == TmapType::kU8    ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                        : type == TmapType::kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        2,
                        const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace w8a8

using namespace w8a8;

extern "C" {

const char *w8a8_status_string(w8a8_status s) {
  switch (s) {
    case W8A8_OK: return "W8A8_OK";
    case W8A8_ERR_INVALID_ARG: return "W8A8_ERR_INVALID_ARG";
    case W8A8_ERR_MISALIGNED: return "W8A8_ERR_MISALIGNED";
    case W8A8_ERR_UNSUPPORTED_SHAPE: return "W8A8_ERR_UNSUPPORTED_SHAPE";
    case W8A8_ERR_UNSUPPORTED_DTYPE: return "W8A8_ERR_UNSUPPORTED_DTYPE";
    case W8A8_ERR_CUDA: return "W8A8_ERR_CUDA";
    case W8A8_ERR_DEVICE_TIMEOUT: return "W8A8_ERR_DEVICE_TIMEOUT";
    case W8A8_ERR_OUTLIER_OVERFLOW: return "W8A8_ERR_OUTLIER_OVERFLOW";
    case W8A8_ERR_NOT_IMPLEMENTED: return "W8A8_ERR_NOT_IMPLEMENTED";
    case W8A8_ERR_WORKSPACE: return "W8A8_ERR_WORKSPACE";
    case W8A8_ERR_NO_DEVICE: return "W8A8_ERR_NO_DEVICE";
    default: return "W8A8_ERR_UNKNOWN";
  }
}

w8a8_status w8a8_quant_weight_per_channel(const void *W, w8a8_dtype w_dtype, int64_t K, int64_t N,
                                          int64_t ldw, int8_t *Wq, float *s_w, int32_t *colsum,
                                          void *stream) {
  if (w_dtype != W8A8_BF16 && w_dtype != W8A8_FP32) return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (N < 0) return W8A8_ERR_INVALID_ARG;
  if (w8a8_status s = check_k(K)) return s;
  if (ldw < N) return W8A8_ERR_INVALID_ARG;
  if (N == 0) return W8A8_OK;
  if (!W || !Wq || !s_w || !colsum) return W8A8_ERR_INVALID_ARG;
  const int64_t esz = w_dtype == W8A8_BF16 ? 2 : 4;
  // W is read element by element: element alignment is enough. Wq rows are
  // written in 8-byte pieces (K is a multiple of 16).
  if ((reinterpret_cast<uintptr_t>(W) % esz) != 0 || (reinterpret_cast<uintptr_t>(Wq) & 7u) != 0)
    return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  return from_cuda(launch_quant_weight(W, w_dtype, K, N, ldw, Wq, s_w, colsum,
                                       static_cast<cudaStream_t>(stream)));
}

w8a8_status w8a8_calibrate_static(const void *Xcal, w8a8_dtype x_dtype, int64_t T, int64_t K,
                                  int64_t ldx, float *S, float *r, int32_t *Z, void *stream) {
  if (x_dtype != W8A8_BF16 && x_dtype != W8A8_FP32) return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (T <= 0 || K <= 0 || ldx < K) return W8A8_ERR_INVALID_ARG;
  if (!Xcal || !S || !r || !Z) return W8A8_ERR_INVALID_ARG;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  return from_cuda(launch_calibrate(Xcal, x_dtype, T, K, ldx, S, r, Z, d->sm_count,
                                    static_cast<cudaStream_t>(stream)));
}

// Dense tensors of at least this many elements take the streaming kernels
// (stream.cu); below it a single grid-stride launch finishes sooner.
constexpr int64_t kStreamMinElems = int64_t(1) << 22;

w8a8_status w8a8_quant_per_token(const void *X, int64_t M, int64_t K, int64_t ldx, int8_t *Xq,
                                 float *S_x, void *stream) {
  if (w8a8_status s = check_bf16_rows(X, M, K, ldx)) return s;
  if (M == 0) return W8A8_OK;
  if (!Xq || !S_x) return W8A8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Xq) & 15u) != 0) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  return from_cuda(launch_quant_per_token(static_cast<const uint16_t *>(X), M, K, ldx, Xq, S_x, d->sm_count,
                                          static_cast<cudaStream_t>(stream)));
}

w8a8_status w8a8_quant_per_tensor(const void *X, int64_t M, int64_t K, int64_t ldx, const float *r,
                                  const int32_t *Z, int8_t *Xq, void *stream) {
  if (w8a8_status s = check_bf16_rows(X, M, K, ldx)) return s;
  if (M == 0) return W8A8_OK;
  if (!r || !Z || !Xq) return W8A8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Xq) & 15u) != 0) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  if (ldx == K && M * K >= kStreamMinElems)  // a large dense tensor: streamed through shared memory
    return from_cuda(launch_quant_per_tensor_stream(static_cast<const uint16_t *>(X), M * K, r, Z, Xq, d->sm_count,
                                                    d->status, static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_quant_per_tensor(static_cast<const uint16_t *>(X), M, K, ldx, r, Z, Xq,
                                           d->sm_count, static_cast<cudaStream_t>(stream), /*pdl=*/true));
}

w8a8_status w8a8_dequant_per_tensor(const int8_t *Xq, int64_t M, int64_t K, int64_t ldq, const float *S,
                                    const int32_t *Z, void *out, w8a8_dtype out_dtype, void *stream) {
  if (M < 0) return W8A8_ERR_INVALID_ARG;
  if (w8a8_status s = check_k(K)) return s;
  if (ldq < K) return W8A8_ERR_INVALID_ARG;
  if (out_dtype != W8A8_BF16 && out_dtype != W8A8_FP32) return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (M == 0) return W8A8_OK;
  if (!Xq || !S || !Z || !out) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(Xq) || (ldq % 16) != 0 || !aligned16(out)) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  if (ldq == K && M * K >= kStreamMinElems)
    return from_cuda(launch_dequant_per_tensor_stream(Xq, M * K, S, Z, out, out_dtype == W8A8_BF16, d->sm_count,
                                                      d->status, static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_dequant_per_tensor(Xq, M, K, ldq, S, Z, out, out_dtype == W8A8_BF16, d->sm_count,
                                             static_cast<cudaStream_t>(stream)));
}

// Calls with at most this many tokens take the weight-streaming decode kernel
// (with the int8 activation); the one-kernel Decode linear serves up to 32.
constexpr int64_t kDecodeMaxM = 64;
constexpr int64_t kFusedMaxM = 32;

static size_t align256(int64_t n) { return static_cast<size_t>(((n + 255) / 256) * 256); }

// Whether the Decode linear quantizes its activation inside the GEMM kernel.
// Every 128-channel tile re-quantizes the whole activation, about MP * 10 / 128
// ALU operations per weight byte streamed: hidden behind the weight stream for
// up to 16 tokens, and for N <= 4096 (few tiles, deep K split); beyond that
// the separate quantization kernel (once per call) is faster on B200.
static bool decode_fuses_quant(int64_t M, int64_t N) { return M <= 16 || (M <= kFusedMaxM && N <= 4096); }

size_t w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  // w8a8_linear_static keeps the statically quantized activation here unless
  // its Decode-shaped GEMM kernel quantizes it; the GEMM kernels themselves
  // need no workspace.
  return decode_fuses_quant(M, N) ? 0 : align256(M * K);
}

static w8a8_status check_gemm_common(const int8_t *Xq, const int8_t *Wq, const float *s_w,
                                     const float *bias, const int32_t *colsum, int64_t M,
                                     int64_t N, int64_t K, void *out, w8a8_dtype out_dtype) {
  if (M < 0 || N < 0) return W8A8_ERR_INVALID_ARG;
  if (w8a8_status s = check_k(K)) return s;
  if (out_dtype != W8A8_BF16 && out_dtype != W8A8_FP32 && out_dtype != W8A8_I32)
    return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!Xq || !Wq || !s_w || !out) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(out) ||
      (bias && !aligned16(bias)) || (colsum && !aligned16(colsum)))
    return W8A8_ERR_MISALIGNED;
  return W8A8_OK;
}

w8a8_status w8a8_gemm_dequant(const int8_t *Xq, const float *S_x, int32_t s_x_per_row,
                              const int32_t *Z, const int8_t *Wq, const float *s_w,
                              const int32_t *colsum, const float *bias, int64_t M, int64_t N,
                              int64_t K, void *out, w8a8_dtype out_dtype, void *workspace,
                              size_t workspace_bytes, void *stream) {
  if (w8a8_status s = check_gemm_common(Xq, Wq, s_w, bias, colsum, M, N, K, out, out_dtype)) return s;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!S_x || (Z && !colsum)) return W8A8_ERR_INVALID_ARG;
  (void)workspace;
  (void)workspace_bytes;
  const bool decode = M <= kDecodeMaxM;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  EpilogueArgs ep;
  ep.S_x = S_x;
  ep.s_x_per_row = s_x_per_row ? 1 : 0;
  ep.Z = Z;
  ep.colsum = colsum;
  ep.s_w = s_w;
  ep.bias = bias;
  ep.out = out;
  ep.out_dtype = out_dtype;
  if (decode)
    return from_cuda(launch_gemm_decode(Xq, K, Wq, M, N, K, ep, d->status,
                                        static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_gemm_tc(Xq, Wq, M, N, K, ep, false, d->sm_count, d->status,
                                  static_cast<cudaStream_t>(stream)));
}

w8a8_status w8a8_gemm_requant(const int8_t *Xq, const float *S_x, int32_t s_x_per_row, const int32_t *Z,
                              const int8_t *Wq, const float *s_w, const int32_t *colsum, const float *bias,
                              int64_t M, int64_t N, int64_t K, const float *r_out, const int32_t *Z_out,
                              int8_t *Xq_out, void *stream) {
  if (w8a8_status s = check_gemm_common(Xq, Wq, s_w, bias, colsum, M, N, K, Xq_out, W8A8_BF16)) return s;
  if (M > kDecodeMaxM) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!S_x || (Z && !colsum) || !r_out || !Z_out) return W8A8_ERR_INVALID_ARG;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  EpilogueArgs ep;
  ep.S_x = S_x;
  ep.s_x_per_row = s_x_per_row ? 1 : 0;
  ep.Z = Z;
  ep.colsum = colsum;
  ep.s_w = s_w;
  ep.bias = bias;
  ep.out = Xq_out;
  ep.out_dtype = kOutRequantI8;
  ep.r_out = r_out;
  ep.z_out = Z_out;
  return from_cuda(launch_gemm_decode(Xq, K, Wq, M, N, K, ep, d->status, static_cast<cudaStream_t>(stream)));
}

// Shared by w8a8_linear_static and w8a8_linear_static_requant once their
// arguments are checked: ep carries the epilogue operands and the output.
static w8a8_status run_linear_static(const void *X, int64_t M, int64_t K, int64_t ldx, const float *r,
                                     const int32_t *Z, const int8_t *Wq, int64_t N, const EpilogueArgs &ep,
                                     void *workspace, size_t workspace_bytes, cudaStream_t st) {
  const size_t need = w8a8_gemm_workspace_size(M, N, K);
  if (need > 0 && (!workspace || workspace_bytes < need)) return W8A8_ERR_WORKSPACE;
  if (!aligned16(workspace)) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  if (decode_fuses_quant(M, N))  // one kernel: the GEMM quantizes each k-block
    return from_cuda(launch_linear_static_decode(static_cast<const uint16_t *>(X), ldx, r, Z, Wq, M, N, K, ep,
                                                 d->status, st));
  // Static quantization into the workspace, then the GEMM; both use
  // programmatic dependent launch, so the GEMM's weight stream starts while
  // the quantization (and the previous kernel) run.
  int8_t *Xq = static_cast<int8_t *>(workspace);
  cudaError_t e = launch_quant_per_tensor(static_cast<const uint16_t *>(X), M, K, ldx, r, Z, Xq, d->sm_count, st,
                                          /*pdl=*/true);
  if (e != cudaSuccess) return W8A8_ERR_CUDA;
  if (M <= kDecodeMaxM) return from_cuda(launch_gemm_decode(Xq, K, Wq, M, N, K, ep, d->status, st));
  return from_cuda(launch_gemm_tc(Xq, Wq, M, N, K, ep, false, d->sm_count, d->status, st));
}

w8a8_status w8a8_linear_static(const void *X, int64_t M, int64_t K, int64_t ldx, const float *S,
                               const float *r, const int32_t *Z, const int8_t *Wq,
                               const float *s_w, const int32_t *colsum, const float *bias,
                               int64_t N, void *out, w8a8_dtype out_dtype, void *workspace,
                               size_t workspace_bytes, void *stream) {
  if (w8a8_status s = check_bf16_rows(X, M, K, ldx)) return s;
  if (N < 0) return W8A8_ERR_INVALID_ARG;
  if (out_dtype != W8A8_BF16 && out_dtype != W8A8_FP32 && out_dtype != W8A8_I32)
    return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!S || !r || !Z || !Wq || !s_w || !colsum || !out) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(Wq) || !aligned16(s_w) || !aligned16(colsum) || !aligned16(out) ||
      (bias && !aligned16(bias)))
    return W8A8_ERR_MISALIGNED;
  EpilogueArgs ep;
  ep.S_x = S;
  ep.s_x_per_row = 0;
  ep.Z = Z;
  ep.colsum = colsum;
  ep.s_w = s_w;
  ep.bias = bias;
  ep.out = out;
  ep.out_dtype = out_dtype;
  return run_linear_static(X, M, K, ldx, r, Z, Wq, N, ep, workspace, workspace_bytes,
                           static_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_linear_static_requant(const void *X, int64_t M, int64_t K, int64_t ldx, const float *S,
                                       const float *r, const int32_t *Z, const int8_t *Wq,
                                       const float *s_w, const int32_t *colsum, const float *bias,
                                       int64_t N, const float *r_out, const int32_t *Z_out, int8_t *Xq_out,
                                       void *workspace, size_t workspace_bytes, void *stream) {
  if (w8a8_status s = check_bf16_rows(X, M, K, ldx)) return s;
  if (N < 0) return W8A8_ERR_INVALID_ARG;
  if (M > kDecodeMaxM) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!S || !r || !Z || !Wq || !s_w || !colsum || !r_out || !Z_out || !Xq_out) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(Wq) || !aligned16(s_w) || !aligned16(colsum) || !aligned16(Xq_out) ||
      (bias && !aligned16(bias)))
    return W8A8_ERR_MISALIGNED;
  EpilogueArgs ep;
  ep.S_x = S;
  ep.s_x_per_row = 0;
  ep.Z = Z;
  ep.colsum = colsum;
  ep.s_w = s_w;
  ep.bias = bias;
  ep.out = Xq_out;
  ep.out_dtype = kOutRequantI8;
  ep.r_out = r_out;
  ep.z_out = Z_out;
  return run_linear_static(X, M, K, ldx, r, Z, Wq, N, ep, workspace, workspace_bytes,
                           static_cast<cudaStream_t>(stream));
}

size_t int8_outlier_split_workspace_size(int64_t K) {
  if (K <= 0) return 0;
  return align256(static_cast<int64_t>(outlier_workspace_bytes(K)));
}

w8a8_status int8_outlier_split(const void *X, int64_t M, int64_t K, int64_t ldx, float threshold,
                               int32_t cap, int8_t *Xq, float *S_x, int32_t *outlier_idx,
                               int32_t *n_out, void *Xo, void *workspace, size_t workspace_bytes,
                               void *stream) {
  if (w8a8_status s = check_bf16_rows(X, M, K, ldx)) return s;
  if (cap < 0 || cap > 4096) return W8A8_ERR_INVALID_ARG;
  if (M == 0) return W8A8_OK;
  if (!Xq || !S_x || !n_out || (cap > 0 && (!outlier_idx || !Xo))) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(Xq) || (Xo && (reinterpret_cast<uintptr_t>(Xo) & 1u))) return W8A8_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < int8_outlier_split_workspace_size(K)) return W8A8_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  return from_cuda(launch_outlier_split(static_cast<const uint16_t *>(X), M, K, ldx, threshold, cap, Xq, S_x,
                                        outlier_idx, n_out, static_cast<uint16_t *>(Xo), workspace, d->sm_count,
                                        d->status, static_cast<cudaStream_t>(stream)));
}

// Shared by int8_mixed_decomp_gemm and int8_mixed_decomp_gemm_tc: checks and
// the epilogue operands.
static w8a8_status check_mixed(const int8_t *Xq, const float *S_x, const void *Xo, const int32_t *outlier_idx,
                               const int32_t *n_out, int32_t cap, const int8_t *Wq, const float *s_w, const void *W,
                               int64_t ldw, const float *bias, int64_t M, int64_t N, int64_t K, void *out,
                               w8a8_dtype out_dtype, EpilogueArgs *ep) {
  if (w8a8_status s = check_gemm_common(Xq, Wq, s_w, bias, nullptr, M, N, K, out, out_dtype)) return s;
  if (out_dtype == W8A8_I32) return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!S_x || !n_out || cap < 0 || cap > 4096 || (cap > 0 && (!Xo || !outlier_idx || !W)) ||
      ldw < N)
    return W8A8_ERR_INVALID_ARG;
  if ((Xo && !aligned16(Xo)) || (W && !aligned16(W))) return W8A8_ERR_MISALIGNED;
  ep->S_x = S_x;
  ep->s_x_per_row = 1;
  ep->s_w = s_w;
  ep->bias = bias;
  ep->Xo = static_cast<const uint16_t *>(Xo);
  ep->outlier_idx = outlier_idx;
  ep->n_out = n_out;
  ep->cap = cap;
  ep->W = static_cast<const uint16_t *>(W);
  ep->ldw = ldw;
  ep->out = out;
  ep->out_dtype = out_dtype;
  return W8A8_OK;
}

size_t int8_mixed_decomp_gemm_tc_workspace_size(int64_t M, int64_t N, int32_t cap) {
  if (M <= 0 || N <= 0 || cap < 0 || cap > 4096) return 0;
  return align256(static_cast<int64_t>(side_workspace_bytes(M, N, cap)));
}

w8a8_status int8_mixed_decomp_gemm_tc(const int8_t *Xq, const float *S_x, const void *Xo,
                                      const int32_t *outlier_idx, const int32_t *n_out, int32_t cap,
                                      const int8_t *Wq, const float *s_w, const void *W, int64_t ldw,
                                      const float *bias, int64_t M, int64_t N, int64_t K, void *out,
                                      w8a8_dtype out_dtype, void *workspace, size_t workspace_bytes,
                                      void *stream) {
  EpilogueArgs ep;
  if (w8a8_status s = check_mixed(Xq, S_x, Xo, outlier_idx, n_out, cap, Wq, s_w, W, ldw, bias, M, N, K, out,
                                  out_dtype, &ep))
    return s;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!workspace || workspace_bytes < int8_mixed_decomp_gemm_tc_workspace_size(M, N, cap))
    return W8A8_ERR_WORKSPACE;
  if (!aligned16(workspace)) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  if (d->sm_count < 2) return W8A8_ERR_NO_DEVICE;
  return from_cuda(launch_gemm_side_tc(Xq, Wq, M, N, K, ep, workspace, d->sm_count, d->status,
                                       static_cast<cudaStream_t>(stream)));
}

w8a8_status int8_mixed_decomp_gemm(const int8_t *Xq, const float *S_x, const void *Xo,
                                   const int32_t *outlier_idx, const int32_t *n_out, int32_t cap,
                                   const int8_t *Wq, const float *s_w, const void *W, int64_t ldw,
                                   const float *bias, int64_t M, int64_t N, int64_t K, void *out,
                                   w8a8_dtype out_dtype, void *stream) {
  if (w8a8_status s = check_gemm_common(Xq, Wq, s_w, bias, nullptr, M, N, K, out, out_dtype)) return s;
  if (out_dtype == W8A8_I32) return W8A8_ERR_UNSUPPORTED_DTYPE;
  if (M == 0 || N == 0) return W8A8_OK;
  if (!S_x || !n_out || cap < 0 || cap > 4096 || (cap > 0 && (!Xo || !outlier_idx || !W)) ||
      ldw < N)
    return W8A8_ERR_INVALID_ARG;
  if ((Xo && !aligned16(Xo)) || (W && !aligned16(W))) return W8A8_ERR_MISALIGNED;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  EpilogueArgs ep;
  ep.S_x = S_x;
  ep.s_x_per_row = 1;
  ep.s_w = s_w;
  ep.bias = bias;
  ep.Xo = static_cast<const uint16_t *>(Xo);
  ep.outlier_idx = outlier_idx;
  ep.n_out = n_out;
  ep.cap = cap;
  ep.W = static_cast<const uint16_t *>(W);
  ep.ldw = ldw;
  ep.out = out;
  ep.out_dtype = out_dtype;
  return from_cuda(launch_gemm_tc(Xq, Wq, M, N, K, ep, true, d->sm_count, d->status,
                                  static_cast<cudaStream_t>(stream)));
}

w8a8_status w8a8_check_device_error(void *stream, w8a8_status *device_status) {
  if (!device_status) return W8A8_ERR_INVALID_ARG;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return W8A8_ERR_CUDA;
  }
  int32_t v = 0;
  if (cudaMemcpy(&v, d->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return W8A8_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpy(d->status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
    return W8A8_ERR_CUDA;
  *device_status = v;
  return W8A8_OK;
}

w8a8_status w8a8_debug_wait_timeout_selftest(uint64_t limit_ns, void *stream) {
  if (limit_ns < 1000000ull || limit_ns > 10000000000ull) return W8A8_ERR_INVALID_ARG;
  DeviceInfo *d;
  if (w8a8_status s = device_info(&d)) return s;
  return from_cuda(launch_wait_selftest(limit_ns, d->status, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
