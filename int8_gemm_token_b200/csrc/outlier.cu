// outlier.cu -- LLM.int8() outlier split (HBM-bound, two passes over X).
//
// What it computes: LLM.int8() paper summary, architecture figure, 16-bit
// decomposition step (1) (the feature columns of X whose magnitude exceeds the
// threshold are split off, with the matching rows of W) and the 8-bit
// vector-wise steps (1)-(2) for the remaining columns (row constant C_x,
// X * 127 / C_x, integers in [-127, 127]); mixed-precision decomposition steps
// 1-2 (threshold 6.0). Readings: a column is an outlier when any of its
// entries has |x| > threshold (strict); its entries become 0 in Xq and do not
// enter the row scale; outlier indices are reported in ascending order.
//
// Pass 1 (column flags): each thread owns 8 adjacent columns (one 16-byte
//   load per row) over a band of 16 rows, with all 16 loads in flight at
//   once, keeps the largest magnitude per column and sets the columns' bits
//   in a K-bit workspace bitmap when it exceeds the threshold (atomicOr only
//   for outlier columns, so almost never). X is loaded under an L2
//   evict-last policy, so that pass 2 finds it in L2. The bitmap is cleared
//   by a one-block kernel just before pass 1; both launch with programmatic
//   dependent launch, so pass 1 streams X while the bitmap is cleared and
//   waits for the clearing only before its first flag (a memset between
//   them cost about 3 us per call).
// Pass 2 (rows): a grid sized to fill the SMs once; every CTA turns the
//   bitmap into the ascending index list (block-wide popcount scan) and
//   copies the bitmap into shared memory once, and each thread takes from it
//   the masks of its own columns (the same in every row); CTA 0 publishes
//   the list and the count. The CTA then walks rows with a grid stride: each
//   row is loaded once into registers (16-byte loads), with the next row's
//   loads in flight when two rows fit in registers; the row's first outlier
//   value per thread is requested at the top of the row, outlier columns are
//   masked to zero, the absmax is reduced (packed bf16 maxima, then warp
//   shuffles), the row is quantized from registers, and the row's outlier
//   values are stored into Xo. Pass 2 is launched with programmatic
//   dependent launch and issues its first row loads before it waits for
//   pass 1 (X is not written by pass 1).
#include "device.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

// pass 1: rows per thread band, all of them requested at once (one round trip
// per thread; measured faster than 32 rows in batches of 8, or 8 rows)
constexpr int kRowsPerThread = 16;

// ------------------------------------------------------------------ pass 1
// 16-byte load that asks L2 to keep the line (evict-last policy): pass 2 reads
// X again, and X (67 MB at 4096 x 8192 bf16) fits in the 126 MB L2.
__device__ __forceinline__ uint4 ld_keep_l2(const uint4 *p, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(policy));
  return v;
}

__global__ void __launch_bounds__(256) outlier_colflag_kernel(const uint16_t *__restrict__ X, int64_t M, int64_t K,
                                                              int64_t ldx, float threshold,
                                                              uint32_t *__restrict__ bitmap) {
  pdl_launch_dependents();  // the row pass may start: it reads only X until this pass completes
  const int64_t groups = K >> 3;  // 8-column groups
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= groups) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kRowsPerThread;
  const int64_t r1 = r0 + kRowsPerThread < M ? r0 + kRowsPerThread : M;
  // magnitude bits of the 8 columns, two per word (packed unsigned maxima)
  uint32_t mx0 = 0, mx1 = 0, mx2 = 0, mx3 = 0;
  const uint4 *p = reinterpret_cast<const uint4 *>(X + r0 * ldx) + g;
  const int64_t step = ldx >> 3;
  uint64_t keep;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
  int64_t r = r0;
  for (; r + kRowsPerThread <= r1; r += kRowsPerThread) {
    uint4 v[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) v[i] = ld_keep_l2(p + i * step, keep);
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      mx0 = __vmaxu2(mx0, v[i].x & 0x7FFF7FFFu);
      mx1 = __vmaxu2(mx1, v[i].y & 0x7FFF7FFFu);
      mx2 = __vmaxu2(mx2, v[i].z & 0x7FFF7FFFu);
      mx3 = __vmaxu2(mx3, v[i].w & 0x7FFF7FFFu);
    }
    p += kRowsPerThread * step;
  }
  for (; r < r1; ++r) {
    const uint4 v = ld_keep_l2(p, keep);
    mx0 = __vmaxu2(mx0, v.x & 0x7FFF7FFFu);
    mx1 = __vmaxu2(mx1, v.y & 0x7FFF7FFFu);
    mx2 = __vmaxu2(mx2, v.z & 0x7FFF7FFFu);
    mx3 = __vmaxu2(mx3, v.w & 0x7FFF7FFFu);
    p += step;
  }
  const uint32_t mw[4] = {mx0, mx1, mx2, mx3};
  uint32_t bits = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (__uint_as_float(mw[j] << 16) > threshold) bits |= 1u << (2 * j);
    if (__uint_as_float(mw[j] & 0xFFFF0000u) > threshold) bits |= 2u << (2 * j);
  }
  // the bitmap is cleared by the kernel before this one: wait for it before the first flag
  pdl_wait_prerequisite();
  if (bits) atomicOr(bitmap + ((g * 8) >> 5), bits << ((g * 8) & 31));
}

// Clears the column bitmap for pass 1. Launched with programmatic dependent
// launch: it waits for the previous kernel (the row pass of a previous split
// may still read the bitmap), then lets pass 1 launch -- the input X is final
// by then, so pass 1 streams it at once and waits for this kernel only before
// its first flag -- and then clears the words.
__global__ void __launch_bounds__(256) outlier_clear_kernel(uint32_t *__restrict__ bitmap, int64_t words) {
  pdl_wait_prerequisite();
  pdl_launch_dependents();
  for (int64_t w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0u;
}

// ------------------------------------------------------------------ pass 2
// Ascending outlier index list from the bitmap, into shared memory (first
// `cap` entries); returns the total count. All threads of the block call it.
__device__ int32_t build_outlier_list(const uint32_t *__restrict__ bitmap, int64_t words, int32_t cap,
                                      int32_t *s_idx, int32_t *s_scan) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t per = (words + nt - 1) / nt;
  const int64_t w0 = tid * per, w1 = w0 + per < words ? w0 + per : words;
  int32_t cnt = 0;
  for (int64_t w = w0; w < w1; ++w) cnt += __popc(__ldcg(bitmap + w));
  // block exclusive scan of cnt
  const int lane = tid & 31, warp = tid >> 5;
  int32_t incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int32_t run = 0;
    for (int i = 0; i < nt / 32; ++i) {
      const int32_t c = s_scan[i];
      s_scan[i] = run;
      run += c;
    }
    s_scan[nt / 32] = run;
  }
  __syncthreads();
  int32_t pos = s_scan[warp] + incl - cnt;
  for (int64_t w = w0; w < w1 && pos < cap; ++w) {
    uint32_t bitsw = __ldcg(bitmap + w);
    while (bitsw && pos < cap) {
      const int b = __ffs(bitsw) - 1;
      bitsw &= bitsw - 1;
      s_idx[pos++] = static_cast<int32_t>(w * 32 + b);
    }
  }
  const int32_t total = s_scan[nt / 32];
  __syncthreads();
  return total;
}

// G threads per row (32: one warp per row, 8 rows per block; 256: one row per
// block), VPT 16-byte chunks per thread held in registers. Each block builds
// the outlier list and copies the column bitmap into shared memory once, then
// walks its row groups (blockIdx.x, + gridDim.x, ...) with the next group's
// loads in flight while the current one is reduced and quantized.
template <int G, int VPT>
__device__ __forceinline__ void load_row_chunks(const uint16_t *xrow, int64_t chunks, int t, bool ok, uint4 (&v)[VPT]) {
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int64_t c = t + static_cast<int64_t>(j) * G;
    v[j] = (ok && c < chunks) ? __ldcs(reinterpret_cast<const uint4 *>(xrow) + c) : make_uint4(0, 0, 0, 0);
  }
}

template <int G, int VPT>
__global__ void __launch_bounds__(256) outlier_row_kernel(const uint16_t *__restrict__ X, int64_t M, int64_t K,
                                                          int64_t ldx, const uint32_t *__restrict__ bitmap,
                                                          int32_t cap, int8_t *__restrict__ Xq,
                                                          float *__restrict__ S_x, int32_t *__restrict__ out_idx,
                                                          int32_t *__restrict__ n_out, uint16_t *__restrict__ Xo,
                                                          int32_t *status) {
  constexpr int R = 256 / G;
  extern __shared__ int32_t s_dyn[];  // cap entries of the index list, then the column bitmap
  __shared__ int32_t s_scan[9];
  __shared__ uint32_t red[2][8];
  const int tid = threadIdx.x;
  const int g = tid / G, t = tid % G;
  const int64_t chunks = K >> 3;
  const int64_t groups = (M + R - 1) / R;
  int64_t grp = blockIdx.x;

  // Launched with programmatic dependent launch, this kernel may start while
  // the column-flag pass still runs. X is final by then (that pass started
  // after everything before it completed), so the first rows' loads go out
  // at once; the bitmap is read, and anything written, only after the wait.
  uint4 v[VPT];
  {
    const int64_t m = grp * R + g;
    load_row_chunks<G, VPT>(X + m * ldx, chunks, t, m < M, v);
  }
  pdl_wait_prerequisite();

  const int64_t words = (K + 31) >> 5;
  const int32_t total = build_outlier_list(bitmap, words, cap, s_dyn, s_scan);
  const int32_t nuse = total < cap ? total : cap;
  uint32_t *s_bits = reinterpret_cast<uint32_t *>(s_dyn + (cap > 0 ? cap : 1));
  for (int64_t w = tid; w < words; w += blockDim.x) s_bits[w] = __ldcg(bitmap + w);
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int j = tid; j < nuse; j += blockDim.x) out_idx[j] = s_dyn[j];
    if (tid == 0) {
      *n_out = total;
      if (total > cap) record_error(status, W8A8_ERR_OUTLIER_OVERFLOW);
    }
  }

  // this thread's chunks are the same columns in every row: their outlier
  // masks (one bit per column, one byte per chunk), gathered once
  uint32_t mk[(VPT + 3) / 4];
  uint32_t mk_any = 0;
#pragma unroll
  for (int i = 0; i < (VPT + 3) / 4; ++i) mk[i] = 0;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int64_t c = t + static_cast<int64_t>(j) * G;
    if (G > 32 && c < chunks) mk[j >> 2] |= ((s_bits[c >> 2] >> ((c & 3) * 8)) & 0xFFu) << ((j & 3) * 8);
  }
#pragma unroll
  for (int i = 0; i < (VPT + 3) / 4; ++i) mk_any |= mk[i];

  for (int it = 0; grp < groups; grp += gridDim.x, ++it) {
    const int64_t m = grp * R + g;
    const bool row_ok = m < M;
    // this row's first outlier value of this thread, requested now so that its
    // round trip overlaps the reduction and quantization below
    const uint16_t *xrow = X + m * ldx;
    uint16_t xo_first = 0;
    if (row_ok && t < nuse) xo_first = __ldg(xrow + s_dyn[t]);
    // next group's loads, in flight while this one is processed (when the
    // two rows fit in registers)
    constexpr bool kPrefetch = VPT <= 8;
    const int64_t mn = (grp + gridDim.x) * R + g;
    const bool next_ok = grp + gridDim.x < groups && mn < M;
    uint4 nxt[kPrefetch ? VPT : 1];
    if constexpr (kPrefetch) load_row_chunks<G, VPT>(X + mn * ldx, chunks, t, next_ok, nxt);
    if (G <= 32 || mk_any) {  // zero the outlier columns of this thread's chunks
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int64_t c = t + static_cast<int64_t>(j) * G;
        const uint32_t mask8 = G > 32 ? (mk[j >> 2] >> ((j & 3) * 8)) & 0xFFu
                                      : (c < chunks ? (s_bits[c >> 2] >> ((c & 3) * 8)) & 0xFFu : 0u);
        if (mask8) {
          uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (mask8 & (1u << (2 * h))) w[h] &= 0xFFFF0000u;
            if (mask8 & (2u << (2 * h))) w[h] &= 0x0000FFFFu;
          }
          v[j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    uint32_t amax = 0;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int64_t c = t + static_cast<int64_t>(j) * G;
      if (row_ok && c < chunks) amax = absmax2_bf16(v[j], amax);
    }
    amax = absmax2_halves(amax);
    amax = __reduce_max_sync(0xFFFFFFFFu, amax);
    if (G > 32) {  // one row per block: combine the warps (double-buffered, one barrier per row)
      if ((tid & 31) == 0) red[it & 1][tid >> 5] = amax;
      __syncthreads();
      amax = red[it & 1][0];
#pragma unroll
      for (int w = 1; w < G / 32; ++w) amax = max(amax, red[it & 1][w]);
    }
    if (row_ok) {
      const float a = __uint_as_float(amax << 16);
      const float r = sym_r(a);
      if (t == 0) S_x[m] = sym_S(a, r);
      int8_t *qrow = Xq + m * K;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int64_t c = t + static_cast<int64_t>(j) * G;
        if (c < chunks) reinterpret_cast<uint2 *>(qrow)[c] = quant8_sym_sat(v[j], r);
      }
      // this row's outlier values (the first one per thread loaded above)
      if (t < nuse) Xo[m * cap + t] = xo_first;
      for (int j = t + G; j < nuse; j += G) Xo[m * cap + j] = __ldg(xrow + s_dyn[j]);
    }
    if constexpr (kPrefetch) {
#pragma unroll
      for (int j = 0; j < VPT; ++j) v[j] = nxt[j];
    } else {
      load_row_chunks<G, VPT>(X + mn * ldx, chunks, t, next_ok, v);
    }
  }
}

template <int G, int VPT>
cudaError_t launch_rows_t(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, const uint32_t *bitmap,
                          int32_t cap, int8_t *Xq, float *S_x, int32_t *idx, int32_t *n_out, uint16_t *Xo,
                          int32_t num_sms, int32_t *status, cudaStream_t s) {
  constexpr int R = 256 / G;
  const size_t smem = static_cast<size_t>((cap > 0 ? cap : 1) + (K + 31) / 32) * sizeof(int32_t);
  auto kern = outlier_row_kernel<G, VPT>;
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_kernel_smem<outlier_row_kernel<G, VPT>>(static_cast<int>(smem), false);
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
  if (e != cudaSuccess) return e;
  const int64_t groups = (M + R - 1) / R;
  const int64_t resident = static_cast<int64_t>(num_sms) * (per_sm > 0 ? per_sm : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(groups < resident ? groups : resident));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, status);
}

}  // namespace

size_t outlier_workspace_bytes(int64_t K) { return static_cast<size_t>(((K + 31) / 32) * 4); }

cudaError_t launch_outlier_split(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, float threshold, int32_t cap,
                                 int8_t *Xq, float *S_x, int32_t *idx, int32_t *n_out, uint16_t *Xo, void *workspace,
                                 int num_sms, int32_t *status, cudaStream_t s) {
  uint32_t *bitmap = static_cast<uint32_t *>(workspace);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c0 = {};
  c0.gridDim = dim3(1);
  c0.blockDim = dim3(256);
  c0.stream = s;
  c0.attrs = pdl;
  c0.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&c0, outlier_clear_kernel, bitmap, static_cast<int64_t>((K + 31) / 32));
  if (e != cudaSuccess) return e;
  const int64_t groups = K / 8;
  cudaLaunchConfig_t c1 = {};
  c1.gridDim = dim3(static_cast<unsigned>((groups + 255) / 256), static_cast<unsigned>((M + kRowsPerThread - 1) / kRowsPerThread));
  c1.blockDim = dim3(256);
  c1.stream = s;
  c1.attrs = pdl;
  c1.numAttrs = 1;
  e = cudaLaunchKernelEx(&c1, outlier_colflag_kernel, X, M, K, ldx, threshold, bitmap);
  if (e != cudaSuccess) return e;
  const int64_t chunks = K / 8;
  if (chunks <= 32 * 4) return launch_rows_t<32, 4>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
  if (chunks <= 32 * 8) return launch_rows_t<32, 8>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
  if (chunks <= 32 * 16) return launch_rows_t<32, 16>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
  if (chunks <= 256 * 4) return launch_rows_t<256, 4>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
  if (chunks <= 256 * 8) return launch_rows_t<256, 8>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
  if (chunks <= 256 * 16) return launch_rows_t<256, 16>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
  return launch_rows_t<256, 32>(X, M, K, ldx, bitmap, cap, Xq, S_x, idx, n_out, Xo, num_sms, status, s);
}

}  // namespace w8a8
