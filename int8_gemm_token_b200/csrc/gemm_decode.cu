// gemm_decode.cu -- Decode-shaped W8A8 linear (1..32 tokens): the GEMM is a
// stream of the INT8 weight from HBM, so the kernel is organised around
// keeping enough of that stream in flight on every SM that takes part.
//
// What it computes: the INT8 GEMM against the shared per-channel weight and
// the zero-point corrected dequant (LLM.int8() summary steps (3)-(4), §一.2
// with zp_b = 0; PDMIX glossary §2.3 eq. Q_decode for the static S, Z). The
// hardware-acceleration chapter's point that decode is bound by memory
// bandwidth sets the design.
//
// How (sm_100a):
//   * swap-AB: 128 rows of Wq [N, K] are the MMA's M dimension (TMEM lanes);
//     the tokens, padded to MP = 16 or 32, are the MMA's N dimension;
//   * one cluster of SPLIT CTAs per 128-row tile; CTA rank r of the cluster
//     owns the k-blocks [r nkb / SPLIT, (r+1) nkb / SPLIT). SPLIT (1..8) is
//     the largest that keeps tiles x SPLIT within one wave of two CTAs per SM,
//     so small N still spreads over the GPU and large N needs no split;
//   * CTAs are small (~100 KiB of shared memory) so that two share an SM:
//     that doubles the copies in flight per SM and lets the next kernel's
//     CTAs start streaming while this kernel's last CTAs finish;
//   * warp 0 streams the weight tile and the matching int8 activation k-block
//     through a TMA ring (5-6 x (16 KiB + MP x 128 B), 128B swizzle); warp 1
//     issues tcgen05.mma kind::i8 (M = 128, N = MP) into one TMEM accumulator;
//   * warps 4-7 fetch the per-channel constants while the weight streams,
//     then read the accumulator (tcgen05.ld) into registers. With SPLIT = 1
//     they store the outputs from there. Otherwise, after a cluster barrier
//     (every ring is free), each CTA stores its partial sums into the shared
//     memory of the CTA that finishes those rows (st.shared::cluster); after
//     a second barrier each CTA adds the SPLIT partials of its rows (exact
//     int32), runs the epilogue and stores. No global workspace, no atomics;
//   * programmatic dependent launch: the kernel lets its dependents launch
//     as soon as it has started, and requests its first ring of weight tiles
//     before it waits for the previous kernel in the stream
//     (griddepcontrol.wait), so the weight stream overlaps the preceding
//     quantization kernel and the tail of the previous decode GEMM. The
//     weight is the one operand read before that wait; the activation, the
//     scales and the output are touched only after it.
#include "device.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

constexpr int kBK = 128;                 // bytes of K per k-block (one swizzle row)
constexpr int kTileN = 128;              // weight rows per tile = MMA M = TMEM lanes
constexpr int kStageW = kTileN * kBK;    // 16 KiB
constexpr int kThreads = 256;            // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
constexpr int kEpiWarp0 = 4;
constexpr int kCtasPerSm = 2;            // two CTAs of ~100 KiB share an SM
constexpr int kMaxSplit = 8;

template <int MP>
struct DecCfg {
  static constexpr int kStageX = MP * kBK;  // int8 activation k-block
  // ring depth: as deep as two CTAs per SM allow (228 KiB per SM, 1 KiB reserved per CTA)
  static constexpr int kStages = MP == 16 ? 6 : 5;
  static constexpr size_t kSmem = static_cast<size_t>(kStages) * (kStageW + kStageX) + 1024 + 256;
  static constexpr int kTmemCols = 32;
  static_assert(kStageX % 1024 == 0, "1 KiB alignment of activation stages");
  static_assert(kCtasPerSm * (kSmem + 1024) <= 228 * 1024, "two CTAs per SM");
};

// Store a 32-bit word to a shared::cluster address (from map_to_rank).
__device__ __forceinline__ void st_shared_cluster(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int MP, int SPLIT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    gemm_i8_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                          int64_t M, int64_t N, int64_t K, const __grid_constant__ EpilogueArgs ep,
                          int32_t *status, uint64_t limit_ns) {
  using Cfg = DecCfg<MP>;
  constexpr uint32_t kIdesc = idesc_i8(kTileN, MP);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sW = base;                            // kStages x 16 KiB weight ring
  uint8_t *sX = sW + Cfg::kStages * kStageW;     // kStages x MP*128 activation ring
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(sX + Cfg::kStages * Cfg::kStageX);
  uint64_t *empty_bar = full_bar + Cfg::kStages;
  uint64_t *tfull_bar = empty_bar + Cfg::kStages;
  uint64_t *drain_bar = tfull_bar + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(tfull_bar, 1);
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

  const int32_t nkb = static_cast<int32_t>((K + kBK - 1) / kBK);
  const uint32_t rank = SPLIT > 1 ? cluster_rank() : 0;
  const int64_t tile = blockIdx.x / SPLIT;
  const int32_t kb0 = static_cast<int32_t>((static_cast<int64_t>(rank) * nkb) / SPLIT);
  const int32_t kb1 = static_cast<int32_t>((static_cast<int64_t>(rank + 1) * nkb) / SPLIT);
  const int32_t nk = kb1 - kb0;  // >= 2 because 2 SPLIT <= nkb
  const int32_t wrow = static_cast<int32_t>(tile * kTileN);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------- TMA producer
      // The first ring of weight tiles does not depend on the previous kernel;
      // the activation may, so its first k-blocks are requested after the wait.
      const int32_t prefetch = nk < Cfg::kStages ? nk : Cfg::kStages;
      for (int32_t i = 0; i < prefetch; ++i) {  // the ring starts empty: no waits
        mbar_arrive_expect_tx(&full_bar[i], kStageW + Cfg::kStageX);
        tma_load_2d(&tmW, &full_bar[i], sW + i * kStageW, (kb0 + i) * kBK, wrow);
      }
      pdl_wait_prerequisite();
      for (int32_t i = 0; i < prefetch; ++i)
        tma_load_2d(&tmX, &full_bar[i], sX + i * Cfg::kStageX, (kb0 + i) * kBK, 0);
      int stage = prefetch % Cfg::kStages;
      uint32_t phase = prefetch == Cfg::kStages ? 1u : 0u;
      // parity of the last fill of every stage, to wait for copies in flight on failure
      uint32_t issued_mask = prefetch >= 32 ? 0xFFFFFFFFu : ((1u << prefetch) - 1u), issued_parity = 0;
      bool ok = true;
      for (int32_t i = prefetch; i < nk; ++i) {
        if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[stage], kStageW + Cfg::kStageX);
        tma_load_2d(&tmW, &full_bar[stage], sW + stage * kStageW, (kb0 + i) * kBK, wrow);
        tma_load_2d(&tmX, &full_bar[stage], sX + stage * Cfg::kStageX, (kb0 + i) * kBK, 0);
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == Cfg::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        for (int s = 0; s < Cfg::kStages; ++s)  // let this CTA's copies land before its memory is reused
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full_bar[s], (issued_parity >> s) & 1u, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------- MMA issuer
      pdl_wait_prerequisite();  // bounded waits below count from here, not from an early launch
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int32_t i = 0; i < nk; ++i) {
        if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_addr(sW + stage * kStageW);
        const uint32_t b_addr = smem_addr(sX + stage * Cfg::kStageX);
#pragma unroll
        for (int k = 0; k < kBK / 32; ++k)
          mma_i8(tmem_base, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k), kIdesc,
                 (i | k) != 0 ? 1u : 0u);
        mma_commit(&empty_bar[stage]);
        if (++stage == Cfg::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        mma_commit(drain_bar);
        mbar_wait_bounded(drain_bar, 0, nullptr, limit_ns / 16 + 1);
      } else {
        mma_commit(tfull_bar);
      }
    }
  }

  // ------------------------------------------------ epilogue warps
  // This CTA finishes rows [r0, r0 + nrows) of the tile: epilogue thread t
  // takes row r0 + t % nrows for tokens t / nrows, + groups, + 2 groups, ...
  const int r0 = static_cast<int>(rank) * kTileN / SPLIT;
  const int nrows = (static_cast<int>(rank) + 1) * kTileN / SPLIT - r0;
  const int groups = kTileN / nrows;
  const int t = threadIdx.x - kEpiWarp0 * 32;  // epilogue thread index (negative elsewhere)
  const int g = t / nrows;
  const int rl = r0 + t % nrows;
  const int64_t n = tile * kTileN + rl;
  const int rows_m = static_cast<int>(M < MP ? M : MP);
  const bool finisher = t >= 0 && g < groups && n < N;
  uint32_t acc[MP];
  int32_t zc = 0;
  float sw = 0.0f, add = 0.0f, sx0 = 0.0f;
  bool ready = true;
  if (warp >= kEpiWarp0) {
    pdl_wait_prerequisite();  // the previous kernel may still read `out` or write S_x, s_w, ...
    // per-channel constants, fetched while the weight still streams
    if (finisher) {
      const int32_t z = ep.Z ? __ldg(ep.Z) : 0;
      if (z != 0) zc = z * __ldg(ep.colsum + n);
      sw = __ldg(ep.s_w + n);
      if (ep.bias) add = __fadd_rn(add, __ldg(ep.bias + n));
      sx0 = __ldg(ep.S_x);
    }
    // tfull also means every MMA has finished reading the weight ring
    ready = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(tfull_bar, 0, abort_flag, limit_ns));
    if (!ready) {
      if (lane == 0) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
    } else {
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>((warp - kEpiWarp0) * 32) << 16);
      if constexpr (MP == 32)
        tmem_ld_32x32b_x32(taddr, acc);
      else
        tmem_ld_32x32b_x16(taddr, acc);
      tmem_ld_wait();
      tc_fence_before();
    }
  }

  // One output element in the fixed order of include/w8a8.h:
  // c = acc - Z*colsum[n]; y = fmaf(float(c), S_x[m]*s_w[n], bias[n]).
  auto store = [&](int m, int32_t a) {
    const int32_t c = a - zc;
    const float sx = ep.s_x_per_row ? __ldg(ep.S_x + m) : sx0;
    const float y = __fmaf_rn(__int2float_rn(c), __fmul_rn(sx, sw), add);
    const int64_t o = static_cast<int64_t>(m) * N + n;
    if (ep.out_dtype == W8A8_BF16)
      static_cast<__nv_bfloat16 *>(ep.out)[o] = __float2bfloat16_rn(y);
    else if (ep.out_dtype == W8A8_FP32)
      static_cast<float *>(ep.out)[o] = y;
    else
      static_cast<int32_t *>(ep.out)[o] = c;
  };

  if constexpr (SPLIT == 1) {
    // thread t holds row t (its TMEM lane) for every token: store directly
    if (finisher && ready && !*abort_flag) {
#pragma unroll
      for (int m = 0; m < MP; ++m)
        if (m < rows_m) store(m, static_cast<int32_t>(acc[m]));
    }
  } else {
    // Partial sums of the cluster, gathered in the owner's shared memory:
    // sRed[s][m][row - r0 of the owner] holds CTA s's sum for token m.
    constexpr int kR = (kTileN + SPLIT - 1) / SPLIT;
    static_assert(SPLIT * MP * kR * 4 <= Cfg::kStages * kStageW, "the partial sums reuse the weight ring");
    int32_t *sRed = reinterpret_cast<int32_t *>(sW);
    __syncwarp();
    cluster_sync_all();  // every MMA of the cluster is done: the weight rings are free
    if (warp >= kEpiWarp0 && ready) {
      const int row = t;  // this thread's TMEM lane
      const uint32_t owner = static_cast<uint32_t>(((row + 1) * SPLIT - 1) / kTileN);
      const int owner_r0 = static_cast<int>(owner) * kTileN / SPLIT;
      const uint32_t dst = map_to_rank(sRed + (static_cast<int>(rank) * MP) * kR + (row - owner_r0), owner);
#pragma unroll
      for (int m = 0; m < MP; ++m)
        if (m < rows_m) st_shared_cluster(dst + 4u * static_cast<uint32_t>(m * kR), acc[m]);
    }
    __syncwarp();
    cluster_sync_all();  // every partial sum has landed (release / acquire)
    if (finisher && !*abort_flag) {
      for (int m = g; m < rows_m; m += groups) {
        int32_t a = 0;
#pragma unroll
        for (int j = 0; j < SPLIT; ++j) a += sRed[(j * MP + m) * kR + (rl - r0)];
        store(m, a);
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int MP, int SPLIT>
cudaError_t launch_decode_t(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                            const EpilogueArgs &ep, int32_t *status, cudaStream_t s) {
  using Cfg = DecCfg<MP>;
  alignas(64) CUtensorMap tmW, tmX;
  if (!encode_tmap_2d(&tmW, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, kTileN, true))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tmX, Xq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(ldx), kBK, MP, true))
    return cudaErrorInvalidValue;
  auto kern = gemm_i8_decode_kernel<MP, SPLIT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Cfg::kSmem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = (N + kTileN - 1) / kTileN;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * SPLIT));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = SPLIT;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, M, N, K, ep, status, kWaitLimitNs);
}

template <int MP>
cudaError_t launch_decode_mp(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                             const EpilogueArgs &ep, int num_sms, int32_t *status, cudaStream_t s) {
  switch (decode_split(N, K, num_sms)) {
    case 8: return launch_decode_t<MP, 8>(Xq, ldx, Wq, M, N, K, ep, status, s);
    case 7: return launch_decode_t<MP, 7>(Xq, ldx, Wq, M, N, K, ep, status, s);
    case 6: return launch_decode_t<MP, 6>(Xq, ldx, Wq, M, N, K, ep, status, s);
    case 5: return launch_decode_t<MP, 5>(Xq, ldx, Wq, M, N, K, ep, status, s);
    case 4: return launch_decode_t<MP, 4>(Xq, ldx, Wq, M, N, K, ep, status, s);
    case 3: return launch_decode_t<MP, 3>(Xq, ldx, Wq, M, N, K, ep, status, s);
    case 2: return launch_decode_t<MP, 2>(Xq, ldx, Wq, M, N, K, ep, status, s);
    default: return launch_decode_t<MP, 1>(Xq, ldx, Wq, M, N, K, ep, status, s);
  }
}

}  // namespace

// Largest cluster size (1..8) with tiles * size within one wave of CTAs (two
// per SM) and at least 2 k-blocks per CTA.
int decode_split(int64_t N, int64_t K, int num_sms) {
  const int64_t tiles = (N + kTileN - 1) / kTileN;
  const int64_t nkb = (K + kBK - 1) / kBK;
  int split = 1;
  for (int s = 2; s <= kMaxSplit; ++s)
    if (tiles * s <= static_cast<int64_t>(kCtasPerSm) * num_sms && nkb >= 2 * s) split = s;
  return split;
}

cudaError_t launch_gemm_decode(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                               const EpilogueArgs &ep, int num_sms, int32_t *status, cudaStream_t s) {
  if (M <= 16) return launch_decode_mp<16>(Xq, ldx, Wq, M, N, K, ep, num_sms, status, s);
  return launch_decode_mp<32>(Xq, ldx, Wq, M, N, K, ep, num_sms, status, s);
}

}  // namespace w8a8
