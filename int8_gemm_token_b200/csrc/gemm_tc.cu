// gemm_tc.cu -- INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor cores
// (tcgen05.mma kind::i8) with the dequant epilogue fused in.
//
// What it computes: LLM.int8() paper summary, architecture figure steps (3)
// (INT8 matmul with INT32 accumulation) and (4) (rescale by the outer product
// of the row and column constants), §一.2 four-term zero-point expansion
// (with a symmetric weight only the -Z * colsum[n] term survives), and for
// the mixed mode the 16-bit decomposition step (2) and the final sum
// Y = X_outlier W_outlier + Dequant(Q(X_normal) Q(W_normal)).
//
// How (sm_100a): two persistent, warp-specialized kernels.
//   gemm_i8_tc_kernel (fewer than 256 tokens): one CTA per SM walks output
//   tiles of 128 x BN.
//   gemm_i8_tc2_kernel (256 tokens and more): a cluster of two CTAs per pair
//   of SMs walks 256 x 256 tiles; each CTA loads its own 128 rows of Xq and
//   of Wq, the leader issues tcgen05.mma.cta_group::2 (M = 256) and commits
//   to both CTAs' barriers, so each SM streams 2/3 of the operand bytes of a
//   single-CTA tile. No load uses cluster multicast.
// Roles in both:
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles of Xq [M, K]
//               and Wq [N, K] into a STAGES-deep shared-memory ring;
//   warp 1      TMEM allocator and MMA issuer: one thread issues
//               tcgen05.mma (K = 32 bytes per instruction) into one of two
//               TMEM accumulators, tcgen05.commit frees ring slots and hands
//               a finished accumulator to the epilogue;
//   warps 4..7  epilogue: the tile's per-column constants (s_w, 0 + bias,
//               colsum) staged in shared memory while its MMAs run, then
//               tcgen05.ld of the int32 accumulator (each warp its 32-lane
//               quarter, the next 32 columns already in flight), the
//               fixed-order fp32 dequant and bf16 / fp32 / int32 stores
//               (in the CTA-pair kernel, bf16 rows that are whole 16-byte
//               multiples go through a per-warp shared-memory block and TMA
//               tensor stores).
//               The mixed (LLM.int8()) instantiation adds the 16-bit side
//               product per element; the tile's first 16 outlier rows of W
//               are staged in shared memory with the constants, so up to 16
//               outliers the side product reads no global memory.
// Double-buffered accumulators let the epilogue of tile i overlap the MMAs
// of tile i+1. Programmatic dependent launch: the first ring of weight tiles
// is requested before griddepcontrol.wait, everything else after it. Every
// wait is bounded; on a timeout the CTA records W8A8_ERR_DEVICE_TIMEOUT,
// stops, frees its TMEM and returns.
#include "device.cuh"
#include "gemm_pair.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

constexpr int kBM = 128;              // rows of Xq per tile = TMEM lanes
constexpr int kBK = 128;              // bytes of K per stage = one 128B swizzle row
constexpr int kStageA = kBM * kBK;    // 16 KiB
constexpr int kThreads = 256;
constexpr int kEpiWarp0 = 4;
// Mixed CTA-pair kernel: the first kSideRows outlier rows of W, for the
// tile's 256 columns, are staged in shared memory per accumulator slot.
constexpr int kSideRows = 16;
constexpr int kSideStride = 256;  // staged row length (bf16 elements)

template <int BN, int STAGES, bool MIXED = false>
struct TcConfig {
  static constexpr int kStageB = BN * kBK;
  static constexpr int kTmemCols = 2 * BN;  // two accumulators
  static constexpr size_t kRing = static_cast<size_t>(STAGES) * (kStageA + kStageB);
  // mixed: the staged outlier rows of W, [slot][kSideRows][BN] bf16
  static constexpr size_t kSide = MIXED ? static_cast<size_t>(2) * kSideRows * BN * 2 : 0;
  static constexpr size_t kSmem = kRing + 2 * 3 * BN * 4 /*epilogue constants*/ + kSide + 1024 /*alignment slack*/ +
                                  256 /*barriers etc.*/;
  static_assert(!MIXED || BN == kSideStride, "staged side rows are one tile wide");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation must be a power of two");
};

// Staged bf16 output of the CTA-pair kernel: each epilogue warp owns 32 rows x
// 128 bytes of shared memory, laid out as the SWIZZLE_128B box of the output
// tensor map (the 16-byte chunk c of row r at chunk c ^ (r % 8)); two 32-column
// chunks fill it, then one TMA store writes the 32 x 64 block.
constexpr int kStageBytes = 32 * 128;

// This lane's 32 results as bf16 into half `half` (64 bytes) of its row.
__device__ __forceinline__ void stage_bf16_row32(const float (&y)[32], uint8_t *stage, int lane, int half) {
  uint8_t *row = stage + lane * 128;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int cc = 4 * half + c;
    *reinterpret_cast<uint4 *>(row + ((cc ^ (lane & 7)) << 4)) =
        make_uint4(pack_bf16x2(y[8 * c], y[8 * c + 1]), pack_bf16x2(y[8 * c + 2], y[8 * c + 3]),
                   pack_bf16x2(y[8 * c + 4], y[8 * c + 5]), pack_bf16x2(y[8 * c + 6], y[8 * c + 7]));
  }
}

// The warp's staged block to out[y .. y+32, x .. x+64) with one TMA store
// (rows and columns past the tensor's end are clipped by the copy).
__device__ __forceinline__ void flush_stage_bf16(const CUtensorMap *tmOut, uint8_t *stage, int lane, int64_t x,
                                                 int64_t y) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmOut, stage, static_cast<int32_t>(x), static_cast<int32_t>(y));
    bulk_commit_group();
  }
}

// Before the staging rows are written again: the warp's previous TMA store
// has finished reading them.
__device__ __forceinline__ void stage_bf16_free(int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
}

// Fixed-order epilogue of one row segment of 32 columns (see include/w8a8.h):
//   c = acc - Z*colsum[n]; y = fmaf(float(c), S_x*s_w[n], side + bias[n]),
// with the per-column constants already in shared memory (s_sw = s_w[n];
// s_add = 0 + bias[n] without the side path, bias[n] with it;
// s_cs = colsum[n]; zeros past N). With the side path, outliers j < ns come
// from the staged rows s_wo (row j at j * kSideStride, zeros past N) and this
// row's Xo values packed two per word in xo2; outliers ns .. nuse-1 are read
// from W in global memory. The chain runs over j in ascending order either
// way.
template <bool MIXED>
__device__ __forceinline__ void epilogue_chunk_s(const uint32_t (&acc)[32], int64_t m, int64_t n0, int64_t M,
                                                 int64_t N, float sx, int32_t z, const EpilogueArgs &ep,
                                                 int32_t nuse, const float *s_sw, const float *s_add,
                                                 const int32_t *s_cs, const uint16_t *s_wo,
                                                 const uint32_t (&xo2)[kSideRows / 2], int32_t ns,
                                                 uint8_t *stage = nullptr, int half = 0) {
  if (m >= M) return;
  const bool full = n0 + 32 <= N;
  float side[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) side[i] = 0.0f;
  if (MIXED) {
#pragma unroll
    for (int j = 0; j < kSideRows; ++j) {
      if (j < ns) {
        const float xo = (j & 1) ? bf16_hi(xo2[j >> 1]) : bf16_lo(xo2[j >> 1]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = *reinterpret_cast<const uint4 *>(s_wo + j * kSideStride + 8 * i);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            side[8 * i + 2 * h] = __fmaf_rn(xo, bf16_lo(w4[h]), side[8 * i + 2 * h]);
            side[8 * i + 2 * h + 1] = __fmaf_rn(xo, bf16_hi(w4[h]), side[8 * i + 2 * h + 1]);
          }
        }
      }
    }
    for (int32_t j = ns; j < nuse; ++j) {
      const float xo = __uint_as_float(static_cast<uint32_t>(ep.Xo[m * ep.cap + j]) << 16);
      const uint16_t *wrow = ep.W + static_cast<int64_t>(__ldg(ep.outlier_idx + j)) * ep.ldw + n0;
      if (full && (ep.ldw % 8) == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = __ldg(reinterpret_cast<const uint4 *>(wrow) + i);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            side[8 * i + 2 * h] = __fmaf_rn(xo, bf16_lo(w4[h]), side[8 * i + 2 * h]);
            side[8 * i + 2 * h + 1] = __fmaf_rn(xo, bf16_hi(w4[h]), side[8 * i + 2 * h + 1]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (n0 + i < N) {
            const float wv = __uint_as_float(static_cast<uint32_t>(__ldg(wrow + i)) << 16);
            side[i] = __fmaf_rn(xo, wv, side[i]);
          }
        }
      }
    }
  }
  float y[32];
  int32_t craw[32];
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float4 w = *reinterpret_cast<const float4 *>(s_sw + i);
    const float4 a = *reinterpret_cast<const float4 *>(s_add + i);
    const float sw4[4] = {w.x, w.y, w.z, w.w}, ad4[4] = {a.x, a.y, a.z, a.w};
    int4 cs = make_int4(0, 0, 0, 0);
    if (z != 0) cs = *reinterpret_cast<const int4 *>(s_cs + i);
    const int32_t cs4[4] = {cs.x, cs.y, cs.z, cs.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      int32_t c = static_cast<int32_t>(acc[i + h]);
      if (z != 0) c -= z * cs4[h];
      craw[i + h] = c;
      float add = ad4[h];
      if (MIXED) add = ep.bias ? __fadd_rn(side[i + h], add) : side[i + h];
      y[i + h] = __fmaf_rn(__int2float_rn(c), __fmul_rn(sx, sw4[h]), add);
    }
  }
  if (stage) {  // bf16 into this lane's staging row, for the warp's TMA store
    stage_bf16_row32(y, stage, threadIdx.x & 31, half);
    return;
  }
  if (ep.out_dtype == W8A8_BF16) {
    uint16_t *o = static_cast<uint16_t *>(ep.out) + m * N + n0;
    if (full && (N % 8) == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 v;
        v.x = pack_bf16x2(y[8 * i + 0], y[8 * i + 1]);
        v.y = pack_bf16x2(y[8 * i + 2], y[8 * i + 3]);
        v.z = pack_bf16x2(y[8 * i + 4], y[8 * i + 5]);
        v.w = pack_bf16x2(y[8 * i + 6], y[8 * i + 7]);
        reinterpret_cast<uint4 *>(o)[i] = v;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) {
          __nv_bfloat16 b = __float2bfloat16_rn(y[i]);
          o[i] = *reinterpret_cast<uint16_t *>(&b);
        }
    }
  } else if (ep.out_dtype == W8A8_FP32) {
    float *o = static_cast<float *>(ep.out) + m * N + n0;
    if (full && (N % 4) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4 *>(o)[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) o[i] = y[i];
    }
  } else {
    int32_t *o = static_cast<int32_t *>(ep.out) + m * N + n0;
    if (full && (N % 4) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<int4 *>(o)[i] = make_int4(craw[4 * i], craw[4 * i + 1], craw[4 * i + 2], craw[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) o[i] = craw[i];
    }
  }
}

template <int BN, int STAGES, bool MIXED>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      int64_t M, int64_t N, int64_t K, const __grid_constant__ EpilogueArgs ep,
                      int32_t *status, uint64_t limit_ns) {
  using Cfg = TcConfig<BN, STAGES, MIXED>;
  constexpr uint32_t kIdesc = idesc_i8(kBM, BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = base + STAGES * kStageA;
  // per-column epilogue constants of the tile, one slot per accumulator:
  // [slot][s_w | add | colsum][BN]
  float *sConst = reinterpret_cast<float *>(base + Cfg::kRing);
  uint16_t *sSide = reinterpret_cast<uint16_t *>(sConst + 2 * 3 * BN);  // mixed: staged outlier rows of W
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sSide) + Cfg::kSide);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *tfull_bar = empty_bar + STAGES;
  uint64_t *tempty_bar = tfull_bar + 2;
  uint64_t *cready_bar = tempty_bar + 2;  // a slot of sConst is written (one arrival per epilogue warp)
  uint64_t *drain_bar = cready_bar + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 4);  // one arrival per epilogue warp
      mbar_init(&cready_bar[b], 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncwarp();  // bar.sync is warp-aligned: reconverge after the single-thread set-up
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t num_m = (M + kBM - 1) / kBM;
  const int64_t num_n = (N + BN - 1) / BN;
  const int64_t num_tiles = num_m * num_n;
  const int nkb = static_cast<int>((K + kBK - 1) / kBK);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      // The first ring of weight tiles does not depend on the previous kernel
      // in the stream; the activation may, so its tiles follow the wait.
      int pre = 0;
      if (blockIdx.x < num_tiles) {
        pre = nkb < STAGES ? nkb : STAGES;
        const int32_t nrow0 = static_cast<int32_t>((blockIdx.x / num_m) * BN);
        for (int kb = 0; kb < pre; ++kb) {  // the ring starts empty: no waits
          mbar_arrive_expect_tx(&full_bar[kb], kStageA + Cfg::kStageB);
          tma_load_2d(&tmB, &full_bar[kb], sB + kb * Cfg::kStageB, kb * kBK, nrow0);
        }
      }
      pdl_wait_prerequisite();
      if (pre > 0) {
        const int32_t mrow0 = static_cast<int32_t>((blockIdx.x % num_m) * kBM);
        for (int kb = 0; kb < pre; ++kb) tma_load_2d(&tmA, &full_bar[kb], sA + kb * kStageA, kb * kBK, mrow0);
      }
      int stage = pre % STAGES;
      uint32_t phase = pre == STAGES ? 1u : 0u;
      uint32_t issued_mask = pre >= 32 ? 0xFFFFFFFFu : ((1u << pre) - 1u), issued_parity = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int32_t mrow = static_cast<int32_t>((tile % num_m) * kBM);
        const int32_t nrow = static_cast<int32_t>((tile / num_m) * BN);
        for (int kb = tile == blockIdx.x ? pre : 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_bar[stage], kStageA + Cfg::kStageB);
          tma_load_2d(&tmA, &full_bar[stage], sA + stage * kStageA, kb * kBK, mrow);
          tma_load_2d(&tmB, &full_bar[stage], sB + stage * Cfg::kStageB, kb * kBK, nrow);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        // let the copies already issued land before the CTA's shared memory goes away
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full_bar[s], (issued_parity >> s) & 1u, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      pdl_wait_prerequisite();  // bounded waits below count from here, not from an early launch
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sA + stage * kStageA);
          const uint32_t b_addr = smem_addr(sB + stage * Cfg::kStageB);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            mma_i8(d_tmem, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k),
                   kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull_bar[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        mma_commit(drain_bar);  // wait for MMAs in flight before TMEM is freed
        mbar_wait_bounded(drain_bar, 0, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp >= kEpiWarp0) {
    pdl_wait_prerequisite();  // S_x, scales, side inputs and `out` belong to the previous kernel until then
    // -------------------------------------------------- epilogue
    // As in the CTA-pair kernel: the tile's per-column constants (and, mixed,
    // the first kSideRows outlier rows of W and this row's Xo values) are
    // staged while its MMAs run, and the next chunk's tcgen05.ld is in flight
    // while the current one is stored.
    const int q = warp - kEpiWarp0;  // TMEM lane quarter of this warp (warp % 4)
    const int32_t z = ep.Z ? __ldg(ep.Z) : 0;
    int32_t nuse = 0;
    if (MIXED) nuse = min(__ldg(ep.n_out), ep.cap);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (*abort_flag) break;
      const int64_t nbase = (tile / num_m) * BN;
      float *c_sw = sConst + acc * 3 * BN, *c_add = c_sw + BN;
      int32_t *c_cs = reinterpret_cast<int32_t *>(c_add + BN);
#pragma unroll
      for (int j = 0; j < BN / 128; ++j) {
        const int col = q * (BN / 4) + j * 32 + lane;
        const int64_t n = nbase + col;
        float sw = 0.0f, add = 0.0f;
        int32_t cs = 0;
        if (n < N) {
          sw = __ldg(ep.s_w + n);
          if (ep.bias) add = MIXED ? __ldg(ep.bias + n) : __fadd_rn(0.0f, __ldg(ep.bias + n));
          if (z != 0) cs = __ldg(ep.colsum + n);
        }
        c_sw[col] = sw;
        c_add[col] = add;
        c_cs[col] = cs;
      }
      const int64_t m = (tile % num_m) * kBM + q * 32 + lane;
      uint16_t *c_wo = sSide + (MIXED ? acc * kSideRows * BN : 0);
      int32_t ns = 0;
      uint32_t xo2[kSideRows / 2];
#pragma unroll
      for (int j = 0; j < kSideRows / 2; ++j) xo2[j] = 0;
      if constexpr (MIXED) {
        // warp q stages outlier rows q, q + 4, ... of W (lane: 8 columns)
        ns = nuse < kSideRows ? nuse : kSideRows;
        for (int j = q; j < ns; j += 4) {
          const uint16_t *wrow = ep.W + static_cast<int64_t>(__ldg(ep.outlier_idx + j)) * ep.ldw + nbase;
          const int col = lane * 8;
          uint4 v = make_uint4(0, 0, 0, 0);
          if ((ep.ldw % 8) == 0 && nbase + col + 8 <= N) {
            v = __ldg(reinterpret_cast<const uint4 *>(wrow + col));
          } else {
            uint32_t e[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) e[t] = nbase + col + t < N ? __ldg(wrow + col + t) : 0u;
            v = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
          }
          *reinterpret_cast<uint4 *>(c_wo + j * BN + col) = v;
        }
        if (m < M) {
          const uint16_t *xrow = ep.Xo + m * ep.cap;
#pragma unroll
          for (int j = 0; j < kSideRows; ++j)
            if (j < ns) xo2[j >> 1] |= static_cast<uint32_t>(__ldg(xrow + j)) << (16 * (j & 1));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cready_bar[acc]);
      const bool ready =
          __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&cready_bar[acc], acc_phase, abort_flag, limit_ns) &&
                                      mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag, limit_ns));
      if (!ready) {
        if (lane == 0) {
          record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      float sx = 0.0f;
      if (m < M) sx = ep.s_x_per_row ? __ldg(ep.S_x + m) : __ldg(ep.S_x);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      {
        uint32_t ra[32], rb[32];
        tmem_ld_32x32b_x32(taddr, ra);
#pragma unroll
        for (int c = 0; c < BN / 32; c += 2) {
          tmem_ld_wait();  // chunk c in ra
          tmem_ld_32x32b_x32(taddr + (c + 1) * 32, rb);
          epilogue_chunk_s<MIXED>(ra, m, nbase + c * 32, M, N, sx, z, ep, nuse, c_sw + c * 32, c_add + c * 32,
                                  c_cs + c * 32, c_wo + c * 32, xo2, ns);
          tmem_ld_wait();  // chunk c + 1 in rb
          if (c + 2 < BN / 32) tmem_ld_32x32b_x32(taddr + (c + 2) * 32, ra);
          epilogue_chunk_s<MIXED>(rb, m, nbase + (c + 1) * 32, M, N, sx, z, ep, nuse, c_sw + (c + 1) * 32,
                                  c_add + (c + 1) * 32, c_cs + (c + 1) * 32, c_wo + (c + 1) * 32, xo2, ns);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncwarp();  // lanes of the producer and MMA warps reconverge before the CTA barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------- CTA pairs
// The same GEMM with 256 x 256 output tiles computed by a cluster of two CTAs
// (tcgen05.mma cta_group::2): each CTA of the pair loads its own 128 rows of
// Xq and its own 128 rows of Wq per k-block (32 KiB), the leader issues the
// pair MMA (M = 256, N = 256), and each CTA holds its 128 rows of the
// accumulator in its own TMEM. Per SM this moves 2/3 of the operand bytes of a
// single-CTA 128 x 256 tile for the same tensor work.
//   leader (rank 0): full barriers (expect_tx for both CTAs' loads, which
//                    complete_tx on the leader's barrier), MMA issue, commits
//                    to the empty / accumulator-full barriers of both CTAs,
//                    accumulator-empty barrier counting both CTAs' epilogues;
//   both:            TMA loads into their own shared memory, epilogue.
template <int STAGES, bool MIXED>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmOut, int32_t tma_store, int64_t M, int64_t N,
                       int64_t K, const __grid_constant__ EpilogueArgs ep, int32_t *status, uint64_t limit_ns) {
  constexpr int kHalf = 128;                 // rows of A and of B per CTA
  constexpr int kStageA2 = kHalf * kBK;      // 16 KiB
  constexpr int kStageB2 = kHalf * kBK;      // 16 KiB
  constexpr int kTileM = 256, kTileN = 256;  // pair tile
  constexpr uint32_t kTmemCols = 512;        // two 256-column accumulators
  constexpr uint32_t kIdesc = idesc_i8(kTileM, kTileN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = base + STAGES * kStageA2;
  // per-column epilogue constants of the tile, one slot per accumulator:
  // [slot][s_w | add | colsum][kTileN]
  float *sConst = reinterpret_cast<float *>(sB + STAGES * kStageB2);
  // mixed: the tile's first kSideRows outlier rows of W, one slot per
  // accumulator: [slot][row][kTileN] bf16
  constexpr int kSideElems = MIXED ? 2 * kSideRows * kTileN : 0;
  static_assert(kTileN == kSideStride, "staged side rows are one tile wide");
  uint16_t *sSide = reinterpret_cast<uint16_t *>(sConst + 2 * 3 * kTileN);
  // plain: each epilogue warp's bf16 staging block for TMA stores (1 KiB aligned)
  constexpr int kStageAll = MIXED ? 0 : 4 * kStageBytes;
  uint8_t *sStage = reinterpret_cast<uint8_t *>(sSide + kSideElems);
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(sStage + kStageAll);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *tfull_bar = empty_bar + STAGES;
  uint64_t *tempty_bar = tfull_bar + 2;
  uint64_t *cready_bar = tempty_bar + 2;  // a slot of sConst is written (one arrival per epilogue warp)
  uint64_t *drain_bar = cready_bar + 2;
  uint64_t *exit_bar = drain_bar + 1;  // leader: rank 1's producer has published its fill count
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(exit_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *peer_fills = abort_flag + 1;  // leader: k-block loads rank 1 issued
  volatile int *peer_abort = peer_fills + 1;  // leader: rank 1 gave up

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);  // one arrival per epilogue warp of both CTAs
      mbar_init(&cready_bar[b], 4);  // one arrival per epilogue warp of this CTA
    }
    mbar_init(drain_bar, 1);
    mbar_init(exit_bar, 1);
    *abort_flag = 0;
    *peer_fills = 0;
    *peer_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  pdl_launch_dependents();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t num_m = (M + kTileM - 1) / kTileM;
  const int64_t num_n = (N + kTileN - 1) / kTileN;
  const int64_t num_tiles = num_m * num_n;
  const int nkb = static_cast<int>((K + kBK - 1) / kBK);
  const int64_t cluster_id = blockIdx.x >> 1;
  const int64_t num_clusters = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      pair_tma_producer<STAGES>(&tmA, &tmB, sA, sB, full_bar, empty_bar, PairExitWords{exit_bar, peer_fills, peer_abort},
                                abort_flag, num_m, num_tiles, nkb, cluster_id, num_clusters, rank, status, limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ pair MMA issuer (leader)
      pdl_wait_prerequisite();  // bounded waits below count from here, not from an early launch
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kTileN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sA + stage * kStageA2);
          const uint32_t b_addr = smem_addr(sB + stage * kStageB2);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8_pair(d_tmem, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k), kIdesc,
                        (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(map_to_rank(&empty_bar[stage], 0));
          mma_commit_pair(map_to_rank(&empty_bar[stage], 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(map_to_rank(&tfull_bar[acc], 0));
        mma_commit_pair(map_to_rank(&tfull_bar[acc], 1));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        mma_commit_pair(map_to_rank(drain_bar, 0));
        mbar_wait_bounded(drain_bar, 0, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp >= kEpiWarp0) {
    pdl_wait_prerequisite();  // S_x, scales, side inputs and `out` belong to the previous kernel until then
    // -------------------------------------------------- epilogue (both CTAs)
    // Per tile: the 4 epilogue warps stage the tile's per-column constants in
    // shared memory while its MMAs run (64 columns each), then each warp turns
    // its 32 accumulator rows into outputs, 32 columns at a time, with the
    // next chunk's tcgen05.ld in flight while the current one is stored.
    const int q = warp - kEpiWarp0;
    const int32_t z = ep.Z ? __ldg(ep.Z) : 0;
    int32_t nuse = 0;
    if (MIXED) nuse = min(__ldg(ep.n_out), ep.cap);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = cluster_id; tile < num_tiles; tile += num_clusters) {
      if (*abort_flag) break;
      const int64_t nbase = (tile / num_m) * kTileN;
      float *c_sw = sConst + acc * 3 * kTileN, *c_add = c_sw + kTileN;
      int32_t *c_cs = reinterpret_cast<int32_t *>(c_add + kTileN);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int col = q * 64 + j * 32 + lane;
        const int64_t n = nbase + col;
        float sw = 0.0f, add = 0.0f;
        int32_t cs = 0;
        if (n < N) {
          sw = __ldg(ep.s_w + n);
          if (ep.bias) add = MIXED ? __ldg(ep.bias + n) : __fadd_rn(0.0f, __ldg(ep.bias + n));
          if (z != 0) cs = __ldg(ep.colsum + n);
        }
        c_sw[col] = sw;
        c_add[col] = add;
        c_cs[col] = cs;
      }
      const int64_t m = (tile % num_m) * kTileM + rank * kHalf + q * 32 + lane;
      uint16_t *c_wo = sSide + acc * kSideRows * kTileN;
      int32_t ns = 0;
      uint32_t xo2[kSideRows / 2];
#pragma unroll
      for (int j = 0; j < kSideRows / 2; ++j) xo2[j] = 0;
      if constexpr (MIXED) {
        // the side inputs of this tile, while its MMAs run: warp q stages
        // outlier rows q, q + 4, ... of W (lane: 8 columns); every thread
        // keeps its own row's Xo values
        ns = nuse < kSideRows ? nuse : kSideRows;
        for (int j = q; j < ns; j += 4) {
          const uint16_t *wrow = ep.W + static_cast<int64_t>(__ldg(ep.outlier_idx + j)) * ep.ldw + nbase;
          const int col = lane * 8;
          uint4 v = make_uint4(0, 0, 0, 0);
          if ((ep.ldw % 8) == 0 && nbase + col + 8 <= N) {
            v = __ldg(reinterpret_cast<const uint4 *>(wrow + col));
          } else {
            uint32_t e[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) e[t] = nbase + col + t < N ? __ldg(wrow + col + t) : 0u;
            v = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
          }
          *reinterpret_cast<uint4 *>(c_wo + j * kTileN + col) = v;
        }
        if (m < M) {
          const uint16_t *xrow = ep.Xo + m * ep.cap;
#pragma unroll
          for (int j = 0; j < kSideRows; ++j)
            if (j < ns) xo2[j >> 1] |= static_cast<uint32_t>(__ldg(xrow + j)) << (16 * (j & 1));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cready_bar[acc]);
      const bool ready =
          __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&cready_bar[acc], acc_phase, abort_flag, limit_ns) &&
                                      mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag, limit_ns));
      if (!ready) {
        if (lane == 0) {
          record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      float sx = 0.0f;
      if (m < M) sx = ep.s_x_per_row ? __ldg(ep.S_x + m) : __ldg(ep.S_x);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kTileN);
      // bf16 output through this warp's staging block and TMA stores (32 rows x 64 columns each)
      uint8_t *stg = (!MIXED && tma_store) ? sStage + q * kStageBytes : nullptr;
      const int64_t mrow0 = (tile % num_m) * kTileM + rank * kHalf + q * 32;
      {
        uint32_t ra[32], rb[32];
        tmem_ld_32x32b_x32(taddr, ra);
#pragma unroll
        for (int c = 0; c < kTileN / 32; c += 2) {
          tmem_ld_wait();  // chunk c in ra
          tmem_ld_32x32b_x32(taddr + (c + 1) * 32, rb);
          if (stg) stage_bf16_free(lane);
          epilogue_chunk_s<MIXED>(ra, m, nbase + c * 32, M, N, sx, z, ep, nuse, c_sw + c * 32, c_add + c * 32,
                                  c_cs + c * 32, c_wo + c * 32, xo2, ns, stg, 0);
          tmem_ld_wait();  // chunk c + 1 in rb
          if (c + 2 < kTileN / 32) tmem_ld_32x32b_x32(taddr + (c + 2) * 32, ra);
          epilogue_chunk_s<MIXED>(rb, m, nbase + (c + 1) * 32, M, N, sx, z, ep, nuse, c_sw + (c + 1) * 32,
                                  c_add + (c + 1) * 32, c_cs + (c + 1) * 32, c_wo + (c + 1) * 32, xo2, ns, stg, 1);
          if (stg && nbase + c * 32 < N && mrow0 < M) flush_stage_bf16(&tmOut, stg, lane, nbase + c * 32, mrow0);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&tempty_bar[acc]);
        else
          mbar_arrive_remote(map_to_rank(&tempty_bar[acc], 0));
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (!MIXED && tma_store) {
      if (lane == 0) bulk_wait_all();  // every store of this warp has completed before the CTA leaves
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair still reads its memory or barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int STAGES, bool MIXED>
cudaError_t launch_tc2_t(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                         const EpilogueArgs &ep, int num_sms, int32_t *status, cudaStream_t s) {
  // ring + epilogue constants (+ staged side rows, or the epilogue warps'
  // staging blocks) + 1 KiB alignment slack + barriers and flags (< 256 B)
  constexpr size_t kSmem = static_cast<size_t>(STAGES) * 2 * 128 * kBK + 2 * 3 * 256 * 4 +
                           (MIXED ? 2 * kSideRows * 256 * 2 : 4 * kStageBytes) + 1024 + 256;
  static_assert((2 * STAGES + 7) * 8 + 4 * 4 <= 256, "barriers and flags fit their reserve");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  alignas(64) CUtensorMap tmA, tmB;
  if (!encode_tmap_2d(&tmA, Xq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(K), kBK, 128, true))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tmB, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, 128, true))
    return cudaErrorInvalidValue;
  // bf16 output rows that are whole 16-byte multiples go out through TMA stores
  const int32_t tma_store = !MIXED && ep.out_dtype == W8A8_BF16 && (N % 8) == 0;
  alignas(64) CUtensorMap tmOut;
  if (tma_store) {
    if (!encode_tmap_2d(&tmOut, ep.out, TmapType::kBF16, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                        static_cast<uint64_t>(N) * 2, 64, 32, true))
      return cudaErrorInvalidValue;
  } else {
    tmOut = tmA;  // never used: the epilogue stores directly
  }
  auto kern = gemm_i8_tc2_kernel<STAGES, MIXED>;
  cudaError_t e = ensure_kernel_smem<gemm_i8_tc2_kernel<STAGES, MIXED>>(static_cast<int>(kSmem), false);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmOut, tma_store, M, N, K, ep, status, kWaitLimitNs);
}

template <int BN, int STAGES, bool MIXED>
cudaError_t launch_tc_t(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                        const EpilogueArgs &ep, int num_sms, int32_t *status, cudaStream_t s) {
  using Cfg = TcConfig<BN, STAGES, MIXED>;
  alignas(64) CUtensorMap tmA, tmB;
  if (!encode_tmap_2d(&tmA, Xq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(K), kBK, kBM, true))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tmB, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, BN, true))
    return cudaErrorInvalidValue;
  auto kern = gemm_i8_tc_kernel<BN, STAGES, MIXED>;
  // per function and per device; cheap enough to repeat on every launch
  cudaError_t e = ensure_kernel_smem<gemm_i8_tc_kernel<BN, STAGES, MIXED>>(static_cast<int>(Cfg::kSmem), false);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < num_sms ? tiles : num_sms));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, M, N, K, ep, status, kWaitLimitNs);
}

}  // namespace

cudaError_t launch_gemm_tc(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                           const EpilogueArgs &ep, bool mixed, int num_sms, int32_t *status,
                           cudaStream_t s) {
  // CTA pairs (256-row tiles) once there are enough rows to fill them.
  // 6 stages of 32 KiB (a seventh measured no faster) leave room for the
  // epilogue's per-column constants.
  if (M >= 256 && num_sms >= 2) {
    if (mixed) return launch_tc2_t<6, true>(Xq, Wq, M, N, K, ep, num_sms, status, s);
    return launch_tc2_t<6, false>(Xq, Wq, M, N, K, ep, num_sms, status, s);
  }
  if (mixed) return launch_tc_t<256, 4, true>(Xq, Wq, M, N, K, ep, num_sms, status, s);
  return launch_tc_t<256, 4, false>(Xq, Wq, M, N, K, ep, num_sms, status, s);
}

// ---------------------------------------------------------------- self-test
// A barrier that nothing completes: the bounded wait must give up, record
// W8A8_ERR_DEVICE_TIMEOUT and let the kernel return.
__global__ void wait_selftest_kernel(int32_t *status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    if (!mbar_wait_bounded(&bar, 0, nullptr, limit_ns)) record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
  }
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t *status, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace w8a8
