// quant.cu -- activation and weight quantization kernels (HBM-bound).
//
//  * quant_per_token:  PDMIX glossary §2.3 eq. Q_prefill with Z_token = 0
//    (configuration guide: Prefill is per-token symmetric); LLM.int8()
//    summary §一.1 absmax equation. One fused pass: 16-byte loads of the row
//    into registers, absmax by packed bf16 maxima and warp shuffles, one fp32
//    division per row (a row whose 127/absmax overflows fp32 is quantized as
//    zero), quantize from registers, 8-byte int8 stores.
//  * quant_per_tensor: PDMIX glossary §2.3 eq. Q_decode (static S, Z).
//  * dequant_per_tensor: its inverse x = S (q - Z), the read side of an INT8
//    KV cache kept in the Decode scheme.
//  * calibrate_static: MinMax over all calibration elements (configuration
//    guide Step 3: MinMax observer, asymmetric decode parameters).
//  * quant_weight_per_channel: configuration guide Step 2 (int8 per_channel
//    symmetric minmax weight); LLM.int8() summary step (1) C_w per column.
#include "device.cuh"
#include "kernels.h"

namespace w8a8 {

// ------------------------------------------------------------ per token
// G threads per row (32 = one warp, or 256 = the whole block), VPT 16-byte
// chunks (8 bf16) per thread held in registers, so X is read exactly once.
// Warp-per-row blocks hold RB rows (RB warps).
template <int G, int VPT, int RB>
__global__ void __launch_bounds__(256) quant_per_token_kernel(const uint16_t *__restrict__ X,
                                                              int64_t M, int64_t K, int64_t ldx,
                                                              int8_t *__restrict__ Xq,
                                                              float *__restrict__ S_x) {
  constexpr int NT = G == 32 ? 32 * RB : 256;  // threads per block
  constexpr int R = NT / G;                    // rows per block
  __shared__ uint32_t red[8];
  const int tid = threadIdx.x;
  const int g = tid / G;  // row slot in this block
  const int t = tid % G;  // thread within the row group
  const int64_t m = static_cast<int64_t>(blockIdx.x) * R + g;
  const int64_t chunks = K >> 3;
  const bool row_ok = m < M;
  const uint16_t *xrow = X + m * ldx;
  // Launched with programmatic stream serialization, this kernel may start
  // while the previous kernel still runs: let the dependent GEMM launch (it
  // touches nothing this kernel writes before its own wait), ask L2 for this
  // block's rows, then wait for the previous kernel before reading X or
  // writing Xq, S_x.
  pdl_launch_dependents();
  if (t == 0 && row_ok) prefetch_l2_bulk(xrow, static_cast<uint32_t>(K * 2));
  pdl_wait_prerequisite();

  uint4 v[VPT];
  uint32_t m2 = 0;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int64_t c = t + static_cast<int64_t>(j) * G;
    if (row_ok && c < chunks) {
      v[j] = __ldcs(reinterpret_cast<const uint4 *>(xrow) + c);
      m2 = absmax2_bf16(v[j], m2);
    } else {
      v[j] = make_uint4(0, 0, 0, 0);
    }
  }
  uint32_t amax = absmax2_halves(m2);
  amax = __reduce_max_sync(0xFFFFFFFFu, amax);
  if (G > 32) {
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < G / 32; ++w) amax = max(amax, red[w]);
  }
  if (!row_ok) return;
  const float a = __uint_as_float(amax << 16);
  const float r = sym_r(a);
  if (t == 0) S_x[m] = sym_S(a, r);
  int8_t *qrow = Xq + m * K;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int64_t c = t + static_cast<int64_t>(j) * G;
    if (c < chunks) reinterpret_cast<uint2 *>(qrow)[c] = quant8_sym_sat(v[j], r);
  }
}

template <int G, int VPT, int RB = 4>
static cudaError_t launch_per_token_t(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                      int8_t *Xq, float *S_x, cudaStream_t s) {
  constexpr int NT = G == 32 ? 32 * RB : 256;
  constexpr int R = NT / G;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((M + R - 1) / R));
  cfg.blockDim = dim3(NT);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quant_per_token_kernel<G, VPT, RB>, X, M, K, ldx, Xq, S_x);
}

// Rows (warps) per block of the warp-per-row form at 16 chunks per thread.
// The block scheduler fills an SM up to its occupancy (about 22 of these
// warps, by registers) before it moves on, so with small blocks some SMs take
// far more rows than the average. Blocks of 8 rows allow at most 2 per SM, 16
// rows, which is the even share when M is at most 2 x 8 rows per SM; with
// more rows than that (two waves), blocks of 2 rows even out the second wave.
static int per_token_rows_per_block(int64_t M, int num_sms) {
  if (M >= static_cast<int64_t>(8) * num_sms && M <= static_cast<int64_t>(16) * num_sms) return 8;
  return M > static_cast<int64_t>(16) * num_sms ? 2 : 4;
}

cudaError_t launch_quant_per_token(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                   int8_t *Xq, float *S_x, int num_sms, cudaStream_t s) {
  const int64_t chunks = K / 8;
  if (chunks <= 32 * 1) return launch_per_token_t<32, 1>(X, M, K, ldx, Xq, S_x, s);
  if (chunks <= 32 * 2) return launch_per_token_t<32, 2>(X, M, K, ldx, Xq, S_x, s);
  if (chunks <= 32 * 4) return launch_per_token_t<32, 4>(X, M, K, ldx, Xq, S_x, s);
  if (chunks <= 32 * 8) return launch_per_token_t<32, 8>(X, M, K, ldx, Xq, S_x, s);
  if (chunks <= 32 * 16) {
    switch (per_token_rows_per_block(M, num_sms)) {
      case 8: return launch_per_token_t<32, 16, 8>(X, M, K, ldx, Xq, S_x, s);
      case 2: return launch_per_token_t<32, 16, 2>(X, M, K, ldx, Xq, S_x, s);
      default: return launch_per_token_t<32, 16, 4>(X, M, K, ldx, Xq, S_x, s);
    }
  }
  if (chunks <= 256 * 4) return launch_per_token_t<256, 4>(X, M, K, ldx, Xq, S_x, s);
  if (chunks <= 256 * 8) return launch_per_token_t<256, 8>(X, M, K, ldx, Xq, S_x, s);
  if (chunks <= 256 * 16) return launch_per_token_t<256, 16>(X, M, K, ldx, Xq, S_x, s);
  return launch_per_token_t<256, 32>(X, M, K, ldx, Xq, S_x, s);
}

// ------------------------------------------------------------ per tensor
// Grid-stride over 16-byte chunks; r and Z are device scalars.
__global__ void __launch_bounds__(256) quant_per_tensor_kernel(const uint16_t *__restrict__ X,
                                                               int64_t M, int64_t K, int64_t ldx,
                                                               const float *__restrict__ r_ptr,
                                                               const int32_t *__restrict__ Z_ptr,
                                                               int8_t *__restrict__ Xq) {
  // When launched with programmatic stream serialization this kernel may start
  // while the previous kernel still runs. It lets the dependent decode GEMM
  // launch at once (that GEMM streams only the weight before its own wait,
  // which returns after this kernel has completed), then waits for the
  // previous kernel before reading X or writing Xq.
  pdl_launch_dependents();
  const int64_t cpr = K >> 3;  // chunks per row
  const int64_t total = M * cpr;
  // dense rows: the first 4 KiB span of X this block converts, asked of L2
  // before the wait (only the first: asking for more than the block consumes
  // right away lets later spans evict earlier ones)
  if (ldx == K && threadIdx.x * 32 < blockDim.x) {
    const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x * 32;
    if (i < total) prefetch_l2_bulk(X + i * 8, static_cast<uint32_t>((total - i < 32 ? total - i : 32) * 16));
  }
  pdl_wait_prerequisite();
  const float r = *r_ptr;
  const int z = *Z_ptr;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / cpr, c = i - m * cpr;
    const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(X + m * ldx) + c);
    reinterpret_cast<uint2 *>(Xq + m * K)[c] = quant8_asym_sat(v, r, z);
  }
}

cudaError_t launch_quant_per_tensor(const uint16_t *X, int64_t M, int64_t K, int64_t ldx,
                                    const float *r, const int32_t *Z, int8_t *Xq, int num_sms,
                                    cudaStream_t s, bool pdl) {
  const int64_t total = M * (K / 8);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quant_per_tensor_kernel, X, M, K, ldx, r, Z, Xq);
}

// ------------------------------------------------------------ static dequantization
// out[m, k] = S * float(Xq[m, k] - Z): one 16-byte load of 16 codes, one fp32
// product each (q - Z is a small exact integer), 32 or 64 bytes stored.
// Grid-stride over 16-code chunks; rows of Xq have stride ldq bytes.
template <bool BF16_OUT>
__global__ void __launch_bounds__(256) dequant_per_tensor_kernel(const int8_t *__restrict__ Xq, int64_t M,
                                                                 int64_t K, int64_t ldq,
                                                                 const float *__restrict__ S_ptr,
                                                                 const int32_t *__restrict__ Z_ptr,
                                                                 void *__restrict__ out) {
  // Programmatic dependent launch: let the next kernel launch, ask L2 for
  // this block's codes (dense rows), then wait for the previous kernel before
  // reading Xq, S, Z or writing `out`.
  pdl_launch_dependents();
  const int64_t cpr = K >> 4;  // 16-code chunks per row
  const int64_t total = M * cpr;
  if (ldq == K && threadIdx.x * 32 < blockDim.x) {  // the block's first span, as in quant_per_tensor
    const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x * 32;
    if (i < total) prefetch_l2_bulk(Xq + i * 16, static_cast<uint32_t>((total - i < 32 ? total - i : 32) * 16));
  }
  pdl_wait_prerequisite();
  const float S = *S_ptr;
  const int z = *Z_ptr;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / cpr, c = i - m * cpr;
    const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(Xq + m * ldq) + c);
    float y[16];
    dequant16(v, S, z, y);
    if constexpr (BF16_OUT) {
      uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + m * K) + 2 * c;
      o[0] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                        pack_bf16x2(y[6], y[7]));
      o[1] = make_uint4(pack_bf16x2(y[8], y[9]), pack_bf16x2(y[10], y[11]), pack_bf16x2(y[12], y[13]),
                        pack_bf16x2(y[14], y[15]));
    } else {
      float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + m * K) + 4 * c;
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
    }
  }
}

cudaError_t launch_dequant_per_tensor(const int8_t *Xq, int64_t M, int64_t K, int64_t ldq, const float *S,
                                      const int32_t *Z, void *out, bool bf16_out, int num_sms, cudaStream_t s) {
  const int64_t total = M * (K / 16);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16_out) return cudaLaunchKernelEx(&cfg, dequant_per_tensor_kernel<true>, Xq, M, K, ldq, S, Z, out);
  return cudaLaunchKernelEx(&cfg, dequant_per_tensor_kernel<false>, Xq, M, K, ldq, S, Z, out);
}

// ------------------------------------------------------------ calibration
// Pass 1: every block reduces the largest positive value and the largest
// magnitude of a negative value; both are >= +0, so their fp32 bit patterns
// order like unsigned integers and atomicMax on the bits is exact. The two
// cells are the S and r outputs themselves (zeroed by the host first).
template <typename T>
__device__ __forceinline__ float load_f(const T *p);
template <>
__device__ __forceinline__ float load_f<uint16_t>(const uint16_t *p) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(p)) << 16);
}
template <>
__device__ __forceinline__ float load_f<float>(const float *p) {
  return __ldg(p);
}

template <typename T>
__global__ void __launch_bounds__(256) calibrate_minmax_kernel(const T *__restrict__ X, int64_t T_,
                                                               int64_t K, int64_t ldx,
                                                               uint32_t *hi_cell,
                                                               uint32_t *neg_lo_cell) {
  __shared__ uint32_t sh[2][8];
  uint32_t hi = 0, nlo = 0;
  const int64_t total = T_ * K;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / K, k = i - t * K;
    const float v = load_f<T>(X + t * ldx + k);
    if (v > 0.0f) hi = max(hi, __float_as_uint(v));
    if (v < 0.0f) nlo = max(nlo, __float_as_uint(-v));
  }
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  nlo = __reduce_max_sync(0xFFFFFFFFu, nlo);
  if ((threadIdx.x & 31) == 0) {
    sh[0][threadIdx.x >> 5] = hi;
    sh[1][threadIdx.x >> 5] = nlo;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) {
      hi = max(hi, sh[0][w]);
      nlo = max(nlo, sh[1][w]);
    }
    hi = max(hi, sh[0][0]);
    nlo = max(nlo, sh[1][0]);
    if (hi) atomicMax(hi_cell, hi);
    if (nlo) atomicMax(neg_lo_cell, nlo);
  }
}

// Pass 2 (one thread): S = (hi - lo)/255, r = 255/(hi - lo),
// Z = clamp(-128 - rne(lo * r), -128, 127); all-zero data, or a range so
// small that 255/(hi - lo) overflows fp32, gives S = r = 1, Z = 0.
__global__ void calibrate_finalize_kernel(float *S, float *r, int32_t *Z) {
  const float hi = __uint_as_float(*reinterpret_cast<uint32_t *>(S));
  const float nlo = __uint_as_float(*reinterpret_cast<uint32_t *>(r));
  const float lo = nlo > 0.0f ? -nlo : 0.0f;
  const float d = __fsub_rn(hi, lo);
  const float rr = __fdiv_rn(255.0f, d);
  if (hi == lo || isinf(rr)) {
    *S = 1.0f;
    *r = 1.0f;
    *Z = 0;
    return;
  }
  *S = __fdiv_rn(d, 255.0f);
  *r = rr;
  *Z = min(max(-128 - rne_clamped(__fmul_rn(lo, rr)), -128), 127);
}

cudaError_t launch_calibrate(const void *X, w8a8_dtype dt, int64_t T, int64_t K, int64_t ldx,
                             float *S, float *r, int32_t *Z, int num_sms, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(S, 0, sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(r, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t total = T * K;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 4) blocks = static_cast<int64_t>(num_sms) * 4;
  if (dt == W8A8_BF16)
    calibrate_minmax_kernel<uint16_t><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const uint16_t *>(X), T, K, ldx, reinterpret_cast<uint32_t *>(S),
        reinterpret_cast<uint32_t *>(r));
  else
    calibrate_minmax_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const float *>(X), T, K, ldx, reinterpret_cast<uint32_t *>(S),
        reinterpret_cast<uint32_t *>(r));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  calibrate_finalize_kernel<<<1, 1, 0, s>>>(S, r, Z);
  return cudaGetLastError();
}

// ------------------------------------------------------------ weights
// One block per 32 output channels (columns of W [K, N]). Pass 1: column
// absmax. Pass 2: quantize 64-row slabs, transpose through shared memory so
// that Wq [N, K] is written along K, and accumulate colsum.
template <typename T>
__global__ void __launch_bounds__(256) quant_weight_kernel(const T *__restrict__ W, int64_t K,
                                                           int64_t N, int64_t ldw,
                                                           int8_t *__restrict__ Wq,
                                                           float *__restrict__ s_w,
                                                           int32_t *__restrict__ colsum) {
  __shared__ float red[8][32];
  __shared__ int32_t csum[8][32];
  __shared__ __align__(16) int8_t tile[32][64 + 16];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t n = n0 + tx;
  const bool col_ok = n < N;

  float a = 0.0f;
  if (col_ok)
    for (int64_t k = ty; k < K; k += 8) a = fmaxf(a, fabsf(load_f<T>(W + k * ldw + n)));
  red[ty][tx] = a;
  __syncthreads();
  a = red[0][tx];
#pragma unroll
  for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w][tx]);
  const float r = sym_r(a);
  if (ty == 0 && col_ok) s_w[n] = sym_S(a, r);

  int32_t cs = 0;
  const int wr = threadIdx.x >> 3;  // output row (channel) this thread writes, 0..31
  const int wp = threadIdx.x & 7;   // 8-byte piece of the 64-byte slab row
  for (int64_t k0 = 0; k0 < K; k0 += 64) {
    for (int kk = ty; kk < 64; kk += 8) {
      const int64_t k = k0 + kk;
      int q = 0;
      if (col_ok && k < K) q = min(max(rne_clamped(__fmul_rn(load_f<T>(W + k * ldw + n), r)), -127), 127);
      cs += q;
      tile[tx][kk] = static_cast<int8_t>(q);
    }
    __syncthreads();
    const int64_t nw = n0 + wr, kw = k0 + wp * 8;
    if (nw < N && kw < K)
      *reinterpret_cast<uint2 *>(Wq + nw * K + kw) = *reinterpret_cast<const uint2 *>(&tile[wr][wp * 8]);
    __syncthreads();
  }
  csum[ty][tx] = cs;
  __syncthreads();
  if (ty == 0 && col_ok) {
    int32_t s = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += csum[w][tx];
    colsum[n] = s;
  }
}

cudaError_t launch_quant_weight(const void *W, w8a8_dtype dt, int64_t K, int64_t N, int64_t ldw,
                                int8_t *Wq, float *s_w, int32_t *colsum, cudaStream_t s) {
  const unsigned blocks = static_cast<unsigned>((N + 31) / 32);
  if (dt == W8A8_BF16)
    quant_weight_kernel<uint16_t><<<blocks, 256, 0, s>>>(static_cast<const uint16_t *>(W), K, N,
                                                         ldw, Wq, s_w, colsum);
  else
    quant_weight_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float *>(W), K, N, ldw,
                                                      Wq, s_w, colsum);
  return cudaGetLastError();
}

}  // namespace w8a8
