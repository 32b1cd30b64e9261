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
// How (sm_100a), two kernels:
//   side_gather_kernel writes the side operands once per call, K-major and
//   zero-padded to whole k-blocks of 64 outlier columns: XoP [M, KP] (the
//   rows of Xo) and WoT [N, KP] (WoT[n, j] = W[idx[j], n], the gathered rows
//   of W transposed through shared memory).
//   gemm_i8_tc2_side_kernel: a cluster of two CTAs walks 256 x 256 output
//   tiles like the CTA-pair INT8 GEMM, with one int32 accumulator (TMEM
//   columns 0..255) and one fp32 side accumulator (columns 256..511) per
//   tile -- the two fill the 512 TMEM columns, so there is one of each.
//     warp 0      TMA producer of the INT8 k-blocks (gemm_pair.cuh);
//     warp 1      (leader) MMA issuer: the INT8 k-blocks (kind::i8) and,
//                 between them as soon as each has landed, the side k-blocks
//                 (kind::f16, K = 16 per instruction) into the side
//                 accumulator;
//     warp 2      TMA producer of the side k-blocks (XoP and WoT boxes of
//                 64 columns x 128 rows, a two-stage ring);
//     warps 4..11 epilogue, two warps per TMEM lane quarter (warp w reads
//                 lanes 32 (w % 4) ..), each with 128 of the tile's 256
//                 columns: tcgen05.ld of both accumulators, the fixed-order
//                 fp32 epilogue, and the results staged per warp in
//                 128B-swizzled shared memory and written by TMA tensor
//                 stores; the accumulators go back to the MMAs as soon as
//                 every warp has read its part. With the accumulators single
//                 buffered, this phase is not overlapped with the next tile's
//                 MMAs; two warps per SM sub-partition hide each other's
//                 load latencies.
// Every wait is bounded; on a timeout the CTA records
// W8A8_ERR_DEVICE_TIMEOUT, stops, lets its copies and MMAs in flight finish,
// frees its TMEM and returns.
#include "device.cuh"
#include "gemm_pair.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

constexpr int kThreads = 384;
constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter, each with half of the tile's columns
constexpr int kBK = 128;             // bytes of K per INT8 k-block
constexpr int kHalf = 128;           // rows of A and of B per CTA
constexpr int kStage2 = kHalf * kBK; // 16 KiB per operand per stage
constexpr int kSideJ = 64;           // outlier columns per side k-block (128 bytes of bf16)
constexpr int kSideOp = kHalf * kSideJ * 2;  // 16 KiB: one side operand box of one CTA
constexpr int kSideStage = 2 * kSideOp;      // XoP box then WoT box
constexpr int kSideStages = 2;
constexpr int kStaging = 32 * 128;           // per epilogue warp: 32 rows x 128 bytes
constexpr uint32_t kTmemCols = 512;          // int32 accumulator + fp32 side accumulator
constexpr uint32_t kSideCol = 256;
constexpr int kStages = 4;                   // INT8 ring depth

struct SideSmem {
  static constexpr size_t kRing = static_cast<size_t>(kStages) * 2 * kStage2;
  static constexpr size_t kSide = static_cast<size_t>(kSideStages) * kSideStage;
  static constexpr size_t kStage = kEpiWarps * kStaging;
  static constexpr size_t kBytes = kRing + kSide + kStage + 1024 /*alignment slack*/ + 256 /*barriers, flags*/;
  static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
  static_assert((2 * kStages + 2 * kSideStages + 5) * 8 + 7 * 4 <= 256, "barriers and flags fit their reserve");
};

// Columns of the padded side operands: cap rounded up to whole k-blocks
// (at least one, so that the tensor maps always describe a real region).
int64_t side_kpad(int32_t cap) {
  const int64_t c = cap > 0 ? cap : 1;
  return ((c + kSideJ - 1) / kSideJ) * kSideJ;
}

// ------------------------------------------------------------------ gather
// Blocks [0, nblk_w): a 64 (j) x 64 (n) tile of WoT, read as 64 rows of W
// (16-byte loads along n) into shared memory and written transposed (16-byte
// stores along j). Blocks [nblk_w, ...): 8 rows of XoP each, one warp per
// row. Columns j in [n_used, round_up(n_used, 64)) are written as zeros;
// columns past that are neither read nor written.
constexpr int kGatherThreads = 256;

__global__ void __launch_bounds__(kGatherThreads) side_gather_kernel(const uint16_t *__restrict__ W, int64_t ldw,
                                                                     const int32_t *__restrict__ idx,
                                                                     const int32_t *__restrict__ n_out, int32_t cap,
                                                                     const uint16_t *__restrict__ Xo, int64_t M,
                                                                     int64_t N, int64_t KP, uint16_t *__restrict__ XoP,
                                                                     uint16_t *__restrict__ WoT, int64_t ntn,
                                                                     int64_t nblk_w) {
  __shared__ __align__(16) uint16_t tile[64][64 + 8];
  pdl_launch_dependents();
  pdl_wait_prerequisite();  // idx, n_out and Xo come from the split
  const int nuse = min(__ldg(n_out), cap);
  const int64_t kp_used = ((nuse + kSideJ - 1) / kSideJ) * static_cast<int64_t>(kSideJ);
  const int tid = threadIdx.x;
  if (blockIdx.x < nblk_w) {
    const int64_t n0 = (blockIdx.x % ntn) * 64, j0 = (blockIdx.x / ntn) * 64;
    if (j0 >= kp_used) return;
    const bool vec = (ldw % 8) == 0 && n0 + 64 <= N;
    const int c = tid % 8;
    for (int r = tid / 8; r < 64; r += kGatherThreads / 8) {  // row j0 + r of the gathered W, 8 x 16 bytes
      const int64_t j = j0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j < nuse) {
        const uint16_t *src = W + static_cast<int64_t>(__ldg(idx + j)) * ldw + n0 + 8 * c;
        if (vec) {
          v = __ldg(reinterpret_cast<const uint4 *>(src));
        } else {
          uint32_t h[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) h[e] = n0 + 8 * c + e < N ? __ldg(src + e) : 0u;
          v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
        }
      }
      *reinterpret_cast<uint4 *>(&tile[r][8 * c]) = v;
    }
    __syncthreads();
    for (int nn = tid / 8; nn < 64; nn += kGatherThreads / 8) {  // row n0 + nn of WoT, 8 x 16 bytes along j
      if (n0 + nn >= N) continue;
      uint32_t h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = tile[8 * c + e][nn];
      *reinterpret_cast<uint4 *>(WoT + (n0 + nn) * KP + j0 + 8 * c) =
          make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
    }
    return;
  }
  const int64_t m = (blockIdx.x - nblk_w) * 8 + tid / 32;
  if (m >= M) return;
  const bool vec = (cap % 8) == 0;
  for (int64_t c = tid % 32; c * 8 < kp_used; c += 32) {  // 16-byte chunks of row m
    const int64_t j = c * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j < nuse) {
      const uint16_t *src = Xo + m * cap + j;
      if (vec && j + 8 <= nuse) {
        v = __ldg(reinterpret_cast<const uint4 *>(src));
      } else {
        uint32_t h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = j + e < nuse ? __ldg(src + e) : 0u;
        v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
      }
    }
    *reinterpret_cast<uint4 *>(XoP + m * KP + j) = v;
  }
}

// ------------------------------------------------------------------ epilogue
// The fixed-order epilogue of 32 columns of one row: per element
//   y = fmaf(float(acc), S_x * s_w[n], bias ? side + bias[n] : side)
// (side = 0 when there is no outlier column); the constants are read 8 at a
// time (zero past N).
__device__ __forceinline__ void side_epilogue_values(const uint32_t (&acc)[32], const uint32_t (&sd)[32],
                                                     bool has_side, int64_t n0, int64_t N, float sx,
                                                     const EpilogueArgs &ep, float (&y)[32]) {
  const bool vec = n0 + 32 <= N && (N % 4) == 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int64_t n = n0 + 8 * g;
    float sw[8], bs[8];
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
      y[8 * g + i] = __fmaf_rn(__int2float_rn(static_cast<int32_t>(acc[8 * g + i])), __fmul_rn(sx, sw[i]), add);
    }
  }
}

// Direct stores of one row's 32 results (ragged shapes the TMA store cannot
// describe: N not a multiple of 8 for bf16, of 4 for fp32).
__device__ __forceinline__ void store_row32(const float (&y)[32], int64_t m, int64_t n0, int64_t M, int64_t N,
                                            const EpilogueArgs &ep) {
  if (m >= M) return;
  if (ep.out_dtype == W8A8_BF16) {
    uint16_t *o = static_cast<uint16_t *>(ep.out) + m * N + n0;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (n0 + i < N) {
        __nv_bfloat16 b = __float2bfloat16_rn(y[i]);
        o[i] = *reinterpret_cast<uint16_t *>(&b);
      }
  } else {
    float *o = static_cast<float *>(ep.out) + m * N + n0;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (n0 + i < N) o[i] = y[i];
  }
}

// This lane's 32 results into the warp's staging rows (128 bytes a row, the
// 16-byte chunk c of row r at chunk c ^ (r % 8): the SWIZZLE_128B layout of
// the output tensor map). bf16: 64 bytes at byte offset 64 * half of the
// row; fp32: the whole 128 bytes.
__device__ __forceinline__ void stage_row32(const float (&y)[32], uint8_t *stage, int lane, int half, bool bf16) {
  uint8_t *row = stage + lane * 128;
  if (bf16) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int cc = 4 * half + c;
      *reinterpret_cast<uint4 *>(row + ((cc ^ (lane & 7)) << 4)) =
          make_uint4(pack_bf16x2(y[8 * c], y[8 * c + 1]), pack_bf16x2(y[8 * c + 2], y[8 * c + 3]),
                     pack_bf16x2(y[8 * c + 4], y[8 * c + 5]), pack_bf16x2(y[8 * c + 6], y[8 * c + 7]));
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<float4 *>(row + ((c ^ (lane & 7)) << 4)) =
          make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
  }
}

// The warp's staging rows to the output with one TMA store (lane 0 issues it
// after every lane's stores are fenced for the async proxy).
__device__ __forceinline__ void flush_stage(const CUtensorMap *tmOut, uint8_t *stage, int lane, int64_t x, int64_t y) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmOut, stage, static_cast<int32_t>(x), static_cast<int32_t>(y));
    bulk_commit_group();
  }
}

// Before the staging rows are written again: the warp's previous TMA store
// has finished reading them.
__device__ __forceinline__ void stage_free(int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_tc2_side_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
                            const __grid_constant__ CUtensorMap tmOut, int32_t tma_store, int64_t M, int64_t N,
                            int64_t K, const __grid_constant__ EpilogueArgs ep, int32_t *status, uint64_t limit_ns) {
  constexpr int kTileM = 256, kTileN = 256;
  constexpr uint32_t kIdescI8 = idesc_i8(kTileM, kTileN);
  constexpr uint32_t kIdescSide = idesc_bf16_f32(kTileM, kTileN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = base;
  uint8_t *sB = base + kStages * kStage2;
  uint8_t *sSide = base + SideSmem::kRing;         // [stage][XoP box | WoT box]
  uint8_t *sStage = sSide + SideSmem::kSide;       // [epilogue warp][32 rows x 128 bytes]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(sStage + SideSmem::kStage);
  uint64_t *empty_bar = full_bar + kStages;
  uint64_t *sfull_bar = empty_bar + kStages;       // leader: both CTAs' side boxes landed
  uint64_t *sempty_bar = sfull_bar + kSideStages;  // the side MMAs reading the stage completed
  uint64_t *tfull_bar = sempty_bar + kSideStages;  // both accumulators of the tile are final
  uint64_t *tempty_bar = tfull_bar + 1;            // leader: both CTAs' epilogues have read them (16 arrivals)
  uint64_t *drain_bar = tempty_bar + 1;
  uint64_t *exit_bar = drain_bar + 1;              // leader: INT8 producer handshake
  uint64_t *sexit_bar = exit_bar + 1;              // leader: side producer handshake
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sexit_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *peer_fills = abort_flag + 1, *peer_abort = peer_fills + 1;
  volatile int *speer_fills = peer_abort + 1, *speer_abort = speer_fills + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmXo);
    tma_prefetch_desc(&tmWo);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < kSideStages; ++s) {
      mbar_init(&sfull_bar[s], 1);
      mbar_init(&sempty_bar[s], 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 2 * kEpiWarps);  // every epilogue warp of both CTAs
    mbar_init(drain_bar, 1);
    mbar_init(exit_bar, 1);
    mbar_init(sexit_bar, 1);
    *abort_flag = 0;
    *peer_fills = *peer_abort = *speer_fills = *speer_abort = 0;
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
      pair_tma_producer<kStages>(&tmA, &tmB, sA, sB, full_bar, empty_bar, PairExitWords{exit_bar, peer_fills, peer_abort},
                                 abort_flag, num_m, num_tiles, nkb, cluster_id, num_clusters, rank, status, limit_ns);
  } else if (warp == 2) {
    if (lane == 0) {
      // ------------------------------------------------ side TMA producer (both CTAs)
      pdl_wait_prerequisite();  // XoP, WoT and n_out are written by the gather kernel
      const int nuse = min(__ldg(ep.n_out), ep.cap);
      const int nsb = (nuse + kSideJ - 1) / kSideJ;
      int fills = 0;
      bool ok = true;
      for (int64_t tile = cluster_id; tile < num_tiles && ok && nsb > 0; tile += num_clusters) {
        const int32_t arow = static_cast<int32_t>((tile % num_m) * kTileM + rank * kHalf);
        const int32_t brow = static_cast<int32_t>((tile / num_m) * kTileN + rank * kHalf);
        for (int b = 0; b < nsb; ++b) {
          const int st = fills & 1;
          if (!mbar_wait_bounded(&sempty_bar[st], static_cast<uint32_t>(((fills >> 1) & 1) ^ 1), abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t leader_full = map_to_rank(&sfull_bar[st], 0);
          if (leader) mbar_arrive_expect_tx(&sfull_bar[st], 2 * kSideStage);
          tma_load_2d_pair(&tmXo, leader_full, sSide + st * kSideStage, b * kSideJ, arow);
          tma_load_2d_pair(&tmWo, leader_full, sSide + st * kSideStage + kSideOp, b * kSideJ, brow);
          ++fills;
        }
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
      pair_producer_exit<kSideStages>(rank, fills, ok, sfull_bar, PairExitWords{sexit_bar, speer_fills, speer_abort},
                                      abort_flag, kSideStage, status, limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader)
      pdl_wait_prerequisite();
      const int nuse = min(__ldg(ep.n_out), ep.cap);
      const int nsb = (nuse + kSideJ - 1) / kSideJ;  // side k-blocks per tile
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      int g = 0;  // side k-blocks issued before this tile (all tiles)
      bool ok = true;
      auto issue_side = [&](int gi, bool first) {
        tc_fence_after();
        const uint8_t *buf = sSide + (gi & 1) * kSideStage;
        const uint32_t a_addr = smem_addr(buf), b_addr = smem_addr(buf + kSideOp);
#pragma unroll
        for (int k = 0; k < kSideJ / 16; ++k)
          mma_bf16_pair(tmem_base + kSideCol, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k),
                        kIdescSide, (first && k == 0) ? 0u : 1u);
        mma_commit_pair(map_to_rank(&sempty_bar[gi & 1], 0));
        mma_commit_pair(map_to_rank(&sempty_bar[gi & 1], 1));
      };
      for (int64_t tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
        if (!mbar_wait_bounded_cluster(tempty_bar, tphase ^ 1u, abort_flag, limit_ns)) {
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
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
          // side k-blocks that have landed, between the INT8 k-blocks (a test, never a wait)
          while (si < nsb && mbar_test_wait_cluster(&sfull_bar[(g + si) & 1], static_cast<uint32_t>(((g + si) >> 1) & 1))) {
            issue_side(g + si, si == 0);
            ++si;
          }
        }
        if (!ok) break;
        for (; si < nsb; ++si) {
          const int gi = g + si;
          if (!mbar_wait_bounded_cluster(&sfull_bar[gi & 1], static_cast<uint32_t>((gi >> 1) & 1), abort_flag,
                                         limit_ns)) {
            ok = false;
            break;
          }
          issue_side(gi, si == 0);
        }
        if (!ok) break;
        g += nsb;
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
    // -------------------------------------------------- epilogue (both CTAs)
    pdl_wait_prerequisite();  // S_x, s_w, bias, n_out and `out` belong to the previous kernels until then
    const int e = warp - kEpiWarp0;   // 0..7
    const int q = warp & 3;           // TMEM lane quarter this warp may read
    const int h = e >> 2;             // column half: [128 h, 128 h + 128)
    const int nuse = min(__ldg(ep.n_out), ep.cap);
    const bool has_side = nuse > 0;
    const bool bf16 = ep.out_dtype == W8A8_BF16;
    uint8_t *stage = sStage + e * kStaging;
    uint32_t tphase = 0;
    for (int64_t tile = cluster_id; tile < num_tiles; tile += num_clusters) {
      if (*abort_flag) break;
      const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(tfull_bar, tphase, abort_flag, limit_ns));
      if (!ready) {
        if (lane == 0) {
          record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t mrow0 = (tile % num_m) * kTileM + rank * kHalf + q * 32;  // this warp's first row
      const int64_t m = mrow0 + lane;
      const int64_t ncol0 = (tile / num_m) * kTileN + 128 * h;                 // this warp's first column
      const float sx = m < M ? __ldg(ep.S_x + m) : 0.0f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(128 * h);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t ra[32], rs[32];
        tmem_ld_32x32b_x32(taddr + c * 32, ra);
        if (has_side) tmem_ld_32x32b_x32(taddr + kSideCol + c * 32, rs);
        tmem_ld_wait();
        if (c == 3) {  // every accumulator column of this warp is in registers: hand TMEM back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader)
              mbar_arrive(tempty_bar);
            else
              mbar_arrive_remote(map_to_rank(tempty_bar, 0));
          }
        }
        float y[32];
        side_epilogue_values(ra, rs, has_side, ncol0 + c * 32, N, sx, ep, y);
        if (!tma_store) {
          store_row32(y, m, ncol0 + c * 32, M, N, ep);
        } else if (bf16) {  // two chunks (64 bf16 columns) per staged box
          if ((c & 1) == 0) stage_free(lane);
          stage_row32(y, stage, lane, c & 1, true);
          if (c & 1) flush_stage(&tmOut, stage, lane, ncol0 + (c - 1) * 32, mrow0);
        } else {  // fp32: one chunk (32 columns) per staged box
          stage_free(lane);
          stage_row32(y, stage, lane, 0, false);
          flush_stage(&tmOut, stage, lane, ncol0 + c * 32, mrow0);
        }
      }
      tphase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();  // every store of this warp has completed before the CTA leaves
    __syncwarp();
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

size_t side_workspace_bytes(int64_t M, int64_t N, int32_t cap) {
  return static_cast<size_t>((M + N) * side_kpad(cap) * 2);
}

cudaError_t launch_gemm_side_tc(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                                const EpilogueArgs &ep, void *workspace, int num_sms, int32_t *status,
                                cudaStream_t s) {
  const int64_t KP = side_kpad(ep.cap);
  uint16_t *XoP = static_cast<uint16_t *>(workspace);
  uint16_t *WoT = XoP + M * KP;
  // 1. the side operands, zero-padded to whole k-blocks
  const int64_t ntn = (N + 63) / 64;
  const int64_t nblk_w = ntn * (KP / 64);
  const int64_t nblk = nblk_w + (M + 7) / 8;
  cudaLaunchConfig_t gcfg = {};
  gcfg.gridDim = dim3(static_cast<unsigned>(nblk));
  gcfg.blockDim = dim3(kGatherThreads);
  gcfg.stream = s;
  cudaLaunchAttribute gattr[1];
  gattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  gattr[0].val.programmaticStreamSerializationAllowed = 1;
  gcfg.attrs = gattr;
  gcfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&gcfg, side_gather_kernel, ep.W, ep.ldw, ep.outlier_idx, ep.n_out, ep.cap,
                                     ep.Xo, M, N, KP, XoP, WoT, ntn, nblk_w);
  if (e != cudaSuccess) return e;
  // 2. the GEMM
  alignas(64) CUtensorMap tmA, tmB, tmXo, tmWo, tmOut;
  if (!encode_tmap_2d(&tmA, Xq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(K), kBK, kHalf, true) ||
      !encode_tmap_2d(&tmB, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, kHalf, true) ||
      !encode_tmap_2d(&tmXo, XoP, TmapType::kBF16, static_cast<uint64_t>(KP), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(KP) * 2, kSideJ, kHalf, true) ||
      !encode_tmap_2d(&tmWo, WoT, TmapType::kBF16, static_cast<uint64_t>(KP), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(KP) * 2, kSideJ, kHalf, true))
    return cudaErrorInvalidValue;
  // TMA stores of the output where its rows are whole 16-byte multiples
  const bool bf16 = ep.out_dtype == W8A8_BF16;
  const int32_t tma_store = bf16 ? (N % 8) == 0 : (N % 4) == 0;
  if (tma_store) {
    if (!encode_tmap_2d(&tmOut, ep.out, bf16 ? TmapType::kBF16 : TmapType::kF32, static_cast<uint64_t>(N),
                        static_cast<uint64_t>(M), static_cast<uint64_t>(N) * (bf16 ? 2 : 4), bf16 ? 64 : 32, 32,
                        true))
      return cudaErrorInvalidValue;
  } else {
    tmOut = tmA;  // never used: the epilogue stores directly
  }
  e = ensure_kernel_smem<gemm_i8_tc2_side_kernel>(static_cast<int>(SideSmem::kBytes), false);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SideSmem::kBytes;
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
  return cudaLaunchKernelEx(&cfg, gemm_i8_tc2_side_kernel, tmA, tmB, tmXo, tmWo, tmOut, tma_store, M, N, K, ep,
                            status, kWaitLimitNs);
}

}  // namespace w8a8
