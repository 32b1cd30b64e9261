// gemm_pair.cuh -- the TMA producer role shared by the CTA-pair tcgen05 GEMM
// kernels (gemm_tc.cu, gemm_side.cu): 128-byte-swizzled K-major k-blocks of
// Xq [M, K] and Wq [N, K] for 256 x 256 pair tiles, each CTA loading its own
// 128 rows of both into a STAGES-deep ring whose full barriers live in the
// leader (rank 0). No load uses cluster multicast.
#pragma once

#include "device.cuh"

namespace w8a8 {

// Shared-memory words of the producer's exit handshake (one set per CTA; the
// leader's are the ones used).
struct PairExitWords {
  uint64_t *exit_bar;     // leader: rank 1's producer has published its fill count (count 1)
  volatile int *peer_fills;  // leader: k-block loads rank 1 issued
  volatile int *peer_abort;  // leader: rank 1's producer gave up
};

// Exit of a pair producer (one thread per CTA) whose copies all complete on
// the leader's `full_bar` ring of STAGES stages, `half_bytes` per CTA per
// fill; `fills` counts the fills this CTA issued. Rank 1 reports its count
// and whether it gave up; after a failure in either CTA the leader
// reconciles each stage's last fill -- completing the half of a fill that
// rank 1 never issued, or arming the half that only rank 1 issued -- and
// waits (bounded) for it, so that no CTA leaves while a copy into its shared
// memory may still be in flight.
template <int STAGES>
__device__ __forceinline__ void pair_producer_exit(uint32_t rank, int fills, bool ok, uint64_t *full_bar,
                                                   const PairExitWords &xw, volatile int *abort_flag,
                                                   uint32_t half_bytes, int32_t *status, uint64_t limit_ns) {
  if (rank != 0) {
    st_shared_cluster(map_to_rank(const_cast<int *>(xw.peer_fills), 0), static_cast<uint32_t>(fills));
    st_shared_cluster(map_to_rank(const_cast<int *>(xw.peer_abort), 0), ok ? 0u : 1u);
    mbar_arrive_remote(map_to_rank(xw.exit_bar, 0));
    return;
  }
  const bool heard = mbar_wait_bounded_cluster(xw.exit_bar, 0, nullptr, limit_ns);
  if (heard && !*xw.peer_abort && !*abort_flag) return;
  if (!heard) record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
  const int fr = heard ? *xw.peer_fills : fills;  // unheard: assume rank 1 matched the leader
  for (int s = 0; s < STAGES; ++s) {
    // last fill of stage s by each CTA (-1: none); they differ by at most one ring turn
    const int fl = fills > s ? s + ((fills - 1 - s) / STAGES) * STAGES : -1;
    const int fp = fr > s ? s + ((fr - 1 - s) / STAGES) * STAGES : -1;
    const int f = fl > fp ? fl : fp;
    if (f < 0) continue;
    if (fl > fp) mbar_complete_tx(&full_bar[s], half_bytes);      // rank 1's half never comes
    if (fp > fl) mbar_arrive_expect_tx(&full_bar[s], half_bytes);  // only rank 1's half comes
    mbar_wait_bounded(&full_bar[s], static_cast<uint32_t>(f / STAGES) & 1u, nullptr, limit_ns / 16 + 1);
  }
}

// Run by one thread (lane 0 of the producer warp) of each CTA of the pair.
// Tile t covers rows (t % num_m) * 256 + [0, 256) of Xq and rows
// (t / num_m) * 256 + [0, 256) of Wq; CTA `rank` loads the 128 rows
// rank * 128 + [0, 128) of each. The first ring of weight k-blocks is
// requested before griddepcontrol.wait (the weight is not written by the
// previous kernel), the activation after it.
//
// Exit: every copy either CTA issued completes on the leader's full barriers.
// Rank 1 reports how many k-block loads it issued; after a failure in either
// CTA the leader reconciles each stage's last fill (completing the half of a
// fill that the other CTA never issued, or arming the half only rank 1
// issued) and waits (bounded) for it, so that no CTA leaves while a copy into
// its shared memory may still be in flight.
template <int STAGES>
__device__ __forceinline__ void pair_tma_producer(const CUtensorMap *tmA, const CUtensorMap *tmB, uint8_t *sA,
                                                  uint8_t *sB, uint64_t *full_bar, uint64_t *empty_bar,
                                                  const PairExitWords &xw, volatile int *abort_flag, int64_t num_m,
                                                  int64_t num_tiles, int nkb, int64_t cluster_id,
                                                  int64_t num_clusters, uint32_t rank, int32_t *status,
                                                  uint64_t limit_ns) {
  constexpr int kBK = 128, kHalf = 128, kTileM = 256, kTileN = 256;
  constexpr uint32_t kStageA2 = kHalf * kBK, kStageB2 = kHalf * kBK;
  const bool leader = rank == 0;
  int pre = 0;
  if (cluster_id < num_tiles) {
    pre = nkb < STAGES ? nkb : STAGES;
    const int32_t brow0 = static_cast<int32_t>((cluster_id / num_m) * kTileN + rank * kHalf);
    for (int kb = 0; kb < pre; ++kb) {  // the ring starts empty: no waits
      if (leader) mbar_arrive_expect_tx(&full_bar[kb], 2 * (kStageA2 + kStageB2));
      tma_load_2d_pair(tmB, map_to_rank(&full_bar[kb], 0), sB + kb * kStageB2, kb * kBK, brow0);
    }
  }
  pdl_wait_prerequisite();
  if (pre > 0) {
    const int32_t arow0 = static_cast<int32_t>((cluster_id % num_m) * kTileM + rank * kHalf);
    for (int kb = 0; kb < pre; ++kb)
      tma_load_2d_pair(tmA, map_to_rank(&full_bar[kb], 0), sA + kb * kStageA2, kb * kBK, arow0);
  }
  int stage = pre % STAGES;
  uint32_t phase = pre == STAGES ? 1u : 0u;
  int fills = pre;  // k-block loads this CTA has issued (both CTAs walk the same sequence)
  bool ok = true;
  for (int64_t tile = cluster_id; tile < num_tiles && ok; tile += num_clusters) {
    const int32_t arow = static_cast<int32_t>((tile % num_m) * kTileM + rank * kHalf);
    const int32_t brow = static_cast<int32_t>((tile / num_m) * kTileN + rank * kHalf);
    for (int kb = tile == cluster_id ? pre : 0; kb < nkb; ++kb) {
      if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit_ns)) {
        ok = false;
        break;
      }
      const uint32_t leader_full = map_to_rank(&full_bar[stage], 0);
      if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * (kStageA2 + kStageB2));
      tma_load_2d_pair(tmA, leader_full, sA + stage * kStageA2, kb * kBK, arow);
      tma_load_2d_pair(tmB, leader_full, sB + stage * kStageB2, kb * kBK, brow);
      ++fills;
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (!ok) {
    record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
    *abort_flag = 1;
  }
  pair_producer_exit<STAGES>(rank, fills, ok, full_bar, xw, abort_flag, kStageA2 + kStageB2, status, limit_ns);
}

}  // namespace w8a8
