// gemm_side.cu -- LLM.int8() mixed-precision decomposition GEMM with the
// 16-bit side product on the tensor cores.
//
// What it computes: LLM.int8() paper summary, architecture figure steps (3)
// (INT8 matmul, INT32 accumulation) and (4) (rescale by the outer product of
// the row and column constants), the 16-bit decomposition step (2)
// (X_F16 W_F16 for the outlier columns) and the final sum
// Y = X_outlier W_outlier + Dequant(Q(X_normal) Q(W_normal)). Per element:
//   side[m, n] = sum_{j < n_used} Xo[m, j] * W[idx[j], n]   (bf16 x bf16, fp32 accumulation)
//   y = fmaf((float) acc[m, n], S_x[m] * s_w[n], side[m, n] + bias[n])
// The side sum is formed by the tensor cores (tcgen05.mma kind::f16) in their
// own summation order, not as the fixed ascending fmaf chain of
// int8_mixed_decomp_gemm; the products are exact in fp32, so the two differ
// only by fp32 rounding of the sum.
//
// How (sm_100a): a cluster of two CTAs walks 256 x 256 output tiles, as the
// CTA-pair INT8 GEMM does, with one int32 accumulator (TMEM columns 0..255)
// and one fp32 side accumulator (columns 256..511) per tile: the two fill
// the 512 TMEM columns, so this kernel keeps a single accumulator of each.
//   warp 0      TMA producer of the INT8 operands (gemm_pair.cuh);
//   warp 1      (leader) MMA issuer: the INT8 k-blocks (kind::i8), and,
//               between them as soon as each is ready, the side k-blocks
//               (kind::f16, K = 16 per instruction, 64 outlier columns per
//               k-block) into the side accumulator;
//   warps 4..7  (both CTAs) side-operand builders, then the epilogue. While
//               a tile's INT8 k-blocks stream, they gather the tile's side
//               operands into a double-buffered shared-memory ring in the
//               128-byte-swizzled K-major layout the MMA reads: A = the
//               tile's rows of Xo (outlier index j contiguous), B = the rows
//               W[idx[j], n] of the tile's output columns (n a row, j
//               contiguous), zero past n_used; then tcgen05.ld of both
//               accumulators, the fixed-order fp32 epilogue and the stores.
// Every wait is bounded; on a timeout the CTA records
// W8A8_ERR_DEVICE_TIMEOUT, stops, lets its copies and MMAs in flight finish,
// frees its TMEM and returns.
#include "device.cuh"
#include "gemm_pair.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

constexpr int kThreads = 256;
constexpr int kEpiWarp0 = 4;
constexpr int kBK = 128;             // bytes of K per INT8 k-block
constexpr int kHalf = 128;           // rows of A and of B per CTA
constexpr int kStage2 = kHalf * kBK; // 16 KiB per operand per stage
constexpr int kSideJ = 64;           // outlier columns per side k-block (128 bytes of bf16)
constexpr int kSideOp = kHalf * kSideJ * 2;  // 16 KiB: one side operand of one CTA
constexpr int kSideBuf = 2 * kSideOp;        // A then B
constexpr uint32_t kTmemCols = 512;          // int32 accumulator + fp32 side accumulator
constexpr uint32_t kSideCol = 256;

template <int STAGES>
struct SideCfg {
  static constexpr size_t kRing = static_cast<size_t>(STAGES) * 2 * kStage2;
  static constexpr size_t kSmem = kRing + 2 * kSideBuf + 1024 /*alignment slack*/ + 256 /*barriers, flags*/;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static_assert((2 * STAGES + 9) * 8 + 5 * 4 <= 256, "barriers and flags fit their reserve");
};

// One side k-block of this CTA's operands, built by the 128 epilogue
// threads (thread t: row t of each operand) into the 128B-swizzled K-major
// layout: the 16-byte chunk c of row r lives at chunk c ^ (r % 8) of the
// row's 128 bytes (the buffers are 1024-byte aligned).
//   A row t: Xo[m0 + t, j0 .. j0 + 63]          (0 past n_used or M)
//   B row t: W[idx[j], n0 + t], j = j0 .. j0+63  (0 past n_used or N)
__device__ __forceinline__ void build_side_block(uint8_t *sXo, uint8_t *sWo, int t, int64_t m0, int64_t n0, int j0,
                                                 int nuse, int64_t M, int64_t N, const EpilogueArgs &ep) {
  const int64_t m = m0 + t;
  const int64_t n = n0 + t;
  const bool vec = (ep.cap % 8) == 0;  // rows of Xo 16-byte aligned (the base is)
  // A: the tile rows' outlier values, 16 bytes at a time
  uint8_t *arow = sXo + t * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int j = j0 + 8 * c;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m < M && j < nuse) {
      const uint16_t *src = ep.Xo + m * ep.cap + j;
      if (vec && j + 8 <= nuse) {
        v = __ldg(reinterpret_cast<const uint4 *>(src));
      } else {
        uint32_t h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = j + e < nuse ? __ldg(src + e) : 0u;
        v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
      }
    }
    *reinterpret_cast<uint4 *>(arow + ((c ^ (t & 7)) << 4)) = v;
  }
  // B: the gathered rows of W, 32 outlier columns in flight at a time
  // (consecutive threads read consecutive n, so each warp load is coalesced)
  uint8_t *brow = sWo + t * 128;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = j0 + 32 * half + e;
      w[e] = 0;
      if (j < nuse && n < N) w[e] = __ldg(ep.W + static_cast<int64_t>(__ldg(ep.outlier_idx + j)) * ep.ldw + n);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = make_uint4(w[8 * c] | (w[8 * c + 1] << 16), w[8 * c + 2] | (w[8 * c + 3] << 16),
                                 w[8 * c + 4] | (w[8 * c + 5] << 16), w[8 * c + 6] | (w[8 * c + 7] << 16));
      const int cc = 4 * half + c;
      *reinterpret_cast<uint4 *>(brow + ((cc ^ (t & 7)) << 4)) = v;
    }
  }
}

// The fixed-order epilogue of 32 columns of one row with the side value of
// each element (zero when there is no outlier column):
//   y = fmaf(float(acc), S_x * s_w[n], bias ? side + bias[n] : side),
// in groups of 8 columns (16-byte bf16 or 2 x 16-byte fp32 stores).
__device__ __forceinline__ void epilogue_side_chunk(const uint32_t (&acc)[32], const uint32_t (&sd)[32], bool has_side,
                                                    int64_t m, int64_t n0, int64_t M, int64_t N, float sx,
                                                    const EpilogueArgs &ep) {
  if (m >= M) return;
  const bool bf16 = ep.out_dtype == W8A8_BF16;
  const bool vec = n0 + 32 <= N && (N % 8) == 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int64_t n = n0 + 8 * g;
    float sw[8], bs[8], y[8];
    if (vec) {
      const float4 w0 = __ldg(reinterpret_cast<const float4 *>(ep.s_w + n));
      const float4 w1 = __ldg(reinterpret_cast<const float4 *>(ep.s_w + n) + 1);
      sw[0] = w0.x; sw[1] = w0.y; sw[2] = w0.z; sw[3] = w0.w; sw[4] = w1.x; sw[5] = w1.y; sw[6] = w1.z; sw[7] = w1.w;
      if (ep.bias) {
        const float4 b0 = __ldg(reinterpret_cast<const float4 *>(ep.bias + n));
        const float4 b1 = __ldg(reinterpret_cast<const float4 *>(ep.bias + n) + 1);
        bs[0] = b0.x; bs[1] = b0.y; bs[2] = b0.z; bs[3] = b0.w; bs[4] = b1.x; bs[5] = b1.y; bs[6] = b1.z; bs[7] = b1.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool ok = n + i < N;
        sw[i] = ok ? __ldg(ep.s_w + n + i) : 0.0f;
        bs[i] = (ok && ep.bias) ? __ldg(ep.bias + n + i) : 0.0f;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float side = has_side ? __uint_as_float(sd[8 * g + i]) : 0.0f;
      const float add = ep.bias ? __fadd_rn(side, bs[i]) : side;
      y[i] = __fmaf_rn(__int2float_rn(static_cast<int32_t>(acc[8 * g + i])), __fmul_rn(sx, sw[i]), add);
    }
    if (bf16) {
      uint16_t *o = static_cast<uint16_t *>(ep.out) + m * N + n;
      if (vec) {
        *reinterpret_cast<uint4 *>(o) = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                                                   pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (n + i < N) {
            __nv_bfloat16 b = __float2bfloat16_rn(y[i]);
            o[i] = *reinterpret_cast<uint16_t *>(&b);
          }
      }
    } else {
      float *o = static_cast<float *>(ep.out) + m * N + n;
      if (vec) {
        reinterpret_cast<float4 *>(o)[0] = make_float4(y[0], y[1], y[2], y[3]);
        reinterpret_cast<float4 *>(o)[1] = make_float4(y[4], y[5], y[6], y[7]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (n + i < N) o[i] = y[i];
      }
    }
  }
}

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_tc2_side_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            int64_t M, int64_t N, int64_t K, const __grid_constant__ EpilogueArgs ep,
                            int32_t *status, uint64_t limit_ns) {
  using Cfg = SideCfg<STAGES>;
  constexpr int kTileM = 256, kTileN = 256;
  constexpr uint32_t kIdescI8 = idesc_i8(kTileM, kTileN);
  constexpr uint32_t kIdescSide = idesc_bf16_f32(kTileM, kTileN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = base + STAGES * kStage2;
  uint8_t *sSide = base + Cfg::kRing;  // [2 buffers][Xo rows 16 KiB | W rows 16 KiB]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(sSide + 2 * kSideBuf);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *tfull_bar = empty_bar + STAGES;  // both accumulators of the tile are final
  uint64_t *tempty_bar = tfull_bar + 1;      // leader: both CTAs' epilogues have read them (8 arrivals)
  uint64_t *sfull_bar = tempty_bar + 1;      // leader [2]: both CTAs built the side k-block (8 arrivals)
  uint64_t *sempty_bar = sfull_bar + 2;      // [2]: the side MMAs reading the buffer have completed
  uint64_t *drain_bar = sempty_bar + 2;
  uint64_t *exit_bar = drain_bar + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(exit_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *peer_fills = abort_flag + 1;
  volatile int *peer_abort = peer_fills + 1;

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
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull_bar[b], 8);
      mbar_init(&sempty_bar[b], 1);
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
    if (lane == 0)
      pair_tma_producer<STAGES>(&tmA, &tmB, sA, sB, full_bar, empty_bar, PairExitWords{exit_bar, peer_fills, peer_abort},
                                abort_flag, num_m, num_tiles, nkb, cluster_id, num_clusters, rank, status, limit_ns);
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader)
      pdl_wait_prerequisite();
      const int nuse = min(__ldg(ep.n_out), ep.cap);
      const int nsb = (nuse + kSideJ - 1) / kSideJ;  // side k-blocks per tile
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      int64_t g0 = 0;  // side k-blocks issued before this tile (all tiles)
      bool ok = true;
      // the side k-block g of all tiles: buffer g % 2, its (g / 2)-th use
      auto issue_side = [&](int64_t g, bool first) {
        tc_fence_after();
        const uint8_t *buf = sSide + (g & 1) * kSideBuf;
        const uint32_t a_addr = smem_addr(buf), b_addr = smem_addr(buf + kSideOp);
#pragma unroll
        for (int k = 0; k < kSideJ / 16; ++k)
          mma_bf16_pair(tmem_base + kSideCol, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k),
                        kIdescSide, (first && k == 0) ? 0u : 1u);
        mma_commit_pair(map_to_rank(&sempty_bar[g & 1], 0));
        mma_commit_pair(map_to_rank(&sempty_bar[g & 1], 1));
      };
      for (int64_t tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
        if (!mbar_wait_bounded(tempty_bar, tphase ^ 1u, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        int si = 0;  // side k-blocks of this tile issued
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sA + stage * kStage2);
          const uint32_t b_addr = smem_addr(sB + stage * kStage2);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8_pair(tmem_base, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k), kIdescI8,
                        (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(map_to_rank(&empty_bar[stage], 0));
          mma_commit_pair(map_to_rank(&empty_bar[stage], 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          // side k-blocks whose operands are ready, between the INT8 k-blocks
          while (si < nsb &&
                 mbar_try_wait_cluster(&sfull_bar[(g0 + si) & 1], static_cast<uint32_t>(((g0 + si) >> 1) & 1))) {
            issue_side(g0 + si, si == 0);
            ++si;
          }
        }
        if (!ok) break;
        for (; si < nsb; ++si) {
          const int64_t g = g0 + si;
          if (!mbar_wait_bounded_cluster(&sfull_bar[g & 1], static_cast<uint32_t>((g >> 1) & 1), abort_flag,
                                         limit_ns)) {
            ok = false;
            break;
          }
          issue_side(g, si == 0);
        }
        if (!ok) break;
        g0 += nsb;
        mma_commit_pair(map_to_rank(tfull_bar, 0));
        mma_commit_pair(map_to_rank(tfull_bar, 1));
        tphase ^= 1u;
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        mma_commit_pair(map_to_rank(drain_bar, 0));  // wait for MMAs in flight before TMEM is freed
        mbar_wait_bounded(drain_bar, 0, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // -------------------------------------------------- side builders + epilogue (both CTAs)
    pdl_wait_prerequisite();  // Xo, idx, n_out, S_x, s_w, bias, W and `out` belong to the previous kernel until then
    const int q = warp - kEpiWarp0;
    const int t = threadIdx.x - kEpiWarp0 * 32;  // 0..127: the operand row this thread builds
    const int nuse = min(__ldg(ep.n_out), ep.cap);
    const int nsb = (nuse + kSideJ - 1) / kSideJ;
    uint32_t tphase = 0;
    int64_t g = 0;
    for (int64_t tile = cluster_id; tile < num_tiles; tile += num_clusters) {
      if (*abort_flag) break;
      const int64_t mtile = (tile % num_m) * kTileM, ntile = (tile / num_m) * kTileN;
      bool ok = true;
      for (int b = 0; b < nsb; ++b, ++g) {
        uint8_t *buf = sSide + (g & 1) * kSideBuf;
        // the buffer's previous side MMAs have completed
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&sempty_bar[g & 1], static_cast<uint32_t>(((g >> 1) & 1) ^ 1),
                                                       abort_flag, limit_ns));
        if (!ok) break;
        build_side_block(buf, buf + kSideOp, t, mtile + rank * kHalf, ntile + rank * kHalf, b * kSideJ, nuse, M, N, ep);
        fence_proxy_async_smem();  // the tensor core reads what these generic stores wrote
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(&sfull_bar[g & 1]);
          else
            mbar_arrive_remote(map_to_rank(&sfull_bar[g & 1], 0));
        }
      }
      ok = ok && __all_sync(0xFFFFFFFFu, mbar_wait_bounded(tfull_bar, tphase, abort_flag, limit_ns));
      if (!ok) {
        if (lane == 0) {
          record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t m = mtile + rank * kHalf + q * 32 + lane;
      const float sx = m < M ? __ldg(ep.S_x + m) : 0.0f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < kTileN / 32; ++c) {
        uint32_t ra[32], rs[32];
        tmem_ld_32x32b_x32(taddr + c * 32, ra);
        if (nsb > 0) tmem_ld_32x32b_x32(taddr + kSideCol + c * 32, rs);
        tmem_ld_wait();
        epilogue_side_chunk(ra, rs, nsb > 0, m, ntile + c * 32, M, N, sx, ep);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(tempty_bar);
        else
          mbar_arrive_remote(map_to_rank(tempty_bar, 0));
      }
      tphase ^= 1u;
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

}  // namespace

cudaError_t launch_gemm_side_tc(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                                const EpilogueArgs &ep, int num_sms, int32_t *status, cudaStream_t s) {
  constexpr int STAGES = 5;
  using Cfg = SideCfg<STAGES>;
  alignas(64) CUtensorMap tmA, tmB;
  if (!encode_tmap_2d(&tmA, Xq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(K), kBK, kHalf, true))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tmB, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, kHalf, true))
    return cudaErrorInvalidValue;
  auto kern = gemm_i8_tc2_side_kernel<STAGES>;
  cudaError_t e = ensure_kernel_smem<gemm_i8_tc2_side_kernel<STAGES>>(static_cast<int>(Cfg::kSmem), false);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
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
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, M, N, K, ep, status, kWaitLimitNs);
}

}  // namespace w8a8
