// gemm_decode.cu -- Decode-shaped W8A8 linear (1..32 tokens): the GEMM is a
// stream of the INT8 weight from HBM, so the kernel is organised around
// keeping every SM's share of that stream in flight.
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
//   * stream-K: the (tile of 128 weight rows) x (128-byte k-block) units are
//     cut into gridDim.x equal contiguous runs, one persistent CTA per SM, so
//     every SM streams the same number of weight bytes whatever N and K are;
//     runs are walked with incremental (tile, k-block) counters (no 64-bit
//     division in the loops);
//   * the int8 activation k-blocks a run needs (a window of at most kWindow
//     k-blocks) are TMA-loaded once into shared memory; the weight streams
//     through a STAGES-deep TMA ring (128 x 128 B boxes, 128B swizzle);
//   * programmatic dependent launch: the weight ring starts filling before the
//     kernel waits for the previous kernel in the stream (griddepcontrol.wait),
//     so a preceding quantization kernel or layer overlaps the weight stream;
//   * a run that covers only part of a tile adds its int32 partial sums to the
//     tile's workspace slice with red.global.add (exact, order-free) and counts
//     its k-blocks on a per-tile counter; the CTA that completes the count reads
//     the total back, runs the epilogue and leaves slice and counter zeroed;
//   * warp 0 issues the TMA loads, warp 1 issues tcgen05.mma kind::i8
//     (M = 128, N = MP) into one of two TMEM accumulators, warps 4-7 drain
//     them (tcgen05.ld) and flush partial sums or run the epilogue.
#include "device.cuh"
#include "kernels.h"

// Timeline probes: compiled out unless W8A8_TRACE is defined (a separate
// diagnostic build); each stamps %globaltimer into a per-CTA row of 256 slots.
#ifdef W8A8_TRACE
__device__ unsigned long long w8a8_decode_trace[1024 * 256];
#define DTRACE(slot) (w8a8_decode_trace[blockIdx.x * 256 + (slot)] = ::w8a8::globaltimer_ns())
#define DTRACE_VAL(slot, v) (w8a8_decode_trace[blockIdx.x * 256 + (slot)] = (unsigned long long)(v))
extern "C" int w8a8_debug_read_decode_trace(unsigned long long *host, int n) {
  return (int)cudaMemcpyFromSymbol(host, w8a8_decode_trace, sizeof(unsigned long long) * n);
}
#else
#define DTRACE(slot) ((void)0)
#define DTRACE_VAL(slot, v) ((void)0)
#endif

namespace w8a8 {

namespace {

constexpr int kBK = 128;                 // bytes of K per k-block (one swizzle row)
constexpr int kTileN = 128;              // weight rows per tile = MMA M = TMEM lanes
constexpr int kStageW = kTileN * kBK;    // 16 KiB
constexpr int kThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 4-7 and 8-11 two epilogue sets
constexpr int kEpiWarp0 = 4;

template <int MP, int STAGES>
struct DecCfg {
  static constexpr int kSlot = MP * kBK;              // one k-block of the int8 activation
  static constexpr int kWindow = (96 * 1024) / kSlot; // k-blocks of activation kept resident
  static constexpr int kStageOut = MP * kTileN * 2;  // bf16 output staging per epilogue set
  static constexpr size_t kSmem = static_cast<size_t>(STAGES) * kStageW + static_cast<size_t>(kWindow) * kSlot +
                                  2 * kStageOut + 1024 + 256;
  static constexpr int kTmemCols = 2 * MP < 32 ? 32 : 2 * MP;  // two accumulators
  static_assert(kSlot % 1024 == 0, "1 KiB alignment of activation slots");
  static_assert(kWindow >= STAGES, "the first window must cover the prefetched ring");
};

// Per-row epilogue operands, loaded before the accumulator is ready so that
// their latency hides behind the weight stream.
struct RowParams {
  float sw = 0.0f, add = 0.0f;
  int32_t cs = 0;
};

__device__ __forceinline__ RowParams load_row_params(int64_t n, int64_t N, int32_t z, const EpilogueArgs &ep) {
  RowParams p;
  if (n < N) {
    p.sw = __ldg(ep.s_w + n);
    if (z != 0) p.cs = __ldg(ep.colsum + n);
    if (ep.bias) p.add = __fadd_rn(0.0f, __ldg(ep.bias + n));
  }
  return p;
}

// Epilogue for one weight row n and the first M token columns, in the fixed
// order of include/w8a8.h: c = acc - Z*colsum[n]; y = fmaf(float(c), S*s_w[n], bias[n]).
template <int MP>
__device__ __forceinline__ void decode_epilogue_row(const int32_t (&acc)[MP], const float (&sx)[MP], int64_t M,
                                                    int64_t N, int64_t n, int32_t z, const RowParams &rp,
                                                    const EpilogueArgs &ep) {
  if (n >= N) return;
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    if (m < M) {
      int32_t c = acc[m];
      if (z != 0) c -= z * rp.cs;
      const float y = __fmaf_rn(__int2float_rn(c), __fmul_rn(sx[m], rp.sw), rp.add);
      if (ep.out_dtype == W8A8_BF16)
        static_cast<__nv_bfloat16 *>(ep.out)[m * N + n] = __float2bfloat16_rn(y);
      else if (ep.out_dtype == W8A8_FP32)
        static_cast<float *>(ep.out)[m * N + n] = y;
      else
        static_cast<int32_t *>(ep.out)[m * N + n] = c;
    }
  }
}

// Epilogue of one 128-row tile for one set of four warps (all 128 threads call
// it; `skip` suppresses a failed warp's work but not its barriers). bf16
// outputs go through shared memory so that every token row leaves as 16-byte
// stores; other outputs are written per element.
template <int MP>
__device__ __forceinline__ void decode_epilogue_tile(const int32_t (&acc)[MP], const float (&sx)[MP], int64_t M,
                                                     int64_t N, int64_t tile, int row, int tid_set, int32_t z,
                                                     const RowParams &rp, const EpilogueArgs &ep,
                                                     uint16_t *stage, uint32_t bar_id, bool skip) {
  const int64_t n = tile * kTileN + row;
  if (ep.out_dtype != W8A8_BF16 || (N % 8) != 0) {
    if (!skip) decode_epilogue_row<MP>(acc, sx, M, N, n, z, rp, ep);
    return;
  }
  if (!skip && n < N) {
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      if (m < M) {
        int32_t c = acc[m];
        if (z != 0) c -= z * rp.cs;
        const float y = __fmaf_rn(__int2float_rn(c), __fmul_rn(sx[m], rp.sw), rp.add);
        const __nv_bfloat16 b = __float2bfloat16_rn(y);
        stage[m * kTileN + row] = *reinterpret_cast<const uint16_t *>(&b);
      }
    }
  }
  __syncwarp();
  named_barrier(bar_id, 128);
  const int rows_out = static_cast<int>(M < MP ? M : MP);
  uint16_t *out = static_cast<uint16_t *>(ep.out);
  for (int c = tid_set; c < rows_out * (kTileN / 8); c += 128) {
    const int m = c / (kTileN / 8), ch = c % (kTileN / 8);
    const int64_t nn = tile * kTileN + ch * 8;
    if (nn < N && !skip)
      *reinterpret_cast<uint4 *>(out + m * N + nn) = *reinterpret_cast<const uint4 *>(stage + m * kTileN + ch * 8);
  }
  __syncwarp();
  named_barrier(bar_id, 128);  // the staging buffer is reused by this set's next tile
}

// Position of a CTA in its run of units: the unit u = tile * nkb + kb, and
// the index of kb in the activation window (k-blocks kb0, kb0+1, ... mod nkb).
struct Cursor {
  int64_t u;
  int32_t tile, kb, slot;
  __device__ __forceinline__ void next(int32_t nkb) {
    ++u;
    if (++kb == nkb) {
      kb = 0;
      ++tile;
    }
    if (++slot == nkb) slot = 0;
  }
};

// TMA loads of the activation window [kb0, kb0 + wlen) (mod nkb) into slots 0..wlen-1.
template <int MP>
__device__ __forceinline__ void load_window(const CUtensorMap *tmX, uint64_t *bar, uint8_t *sX, int32_t kb0,
                                            int32_t wlen, int32_t nkb) {
  constexpr int kSlot = MP * kBK;
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(wlen) * kSlot);
  for (int32_t s = 0, kb = kb0; s < wlen; ++s) {
    tma_load_2d(tmX, bar, sX + s * kSlot, kb * kBK, 0);
    kb = (kb + 1 == nkb) ? 0 : kb + 1;
  }
}

template <int MP, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                          int64_t M, int64_t N, int64_t K, const __grid_constant__ EpilogueArgs ep,
                          int32_t *__restrict__ part, uint32_t *__restrict__ counters, int pdl,
                          int32_t *status, uint64_t limit_ns) {
  using Cfg = DecCfg<MP, STAGES>;
  constexpr uint32_t kIdesc = idesc_i8(kTileN, MP);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sW = base;                            // STAGES x 16 KiB weight ring
  uint8_t *sX = sW + STAGES * kStageW;           // kWindow x MP*128 int8 activation, 128B swizzle
  uint16_t *sOut = reinterpret_cast<uint16_t *>(sX + Cfg::kWindow * Cfg::kSlot);  // 2 x MP x 128 bf16
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sOut) + 2 * Cfg::kStageOut);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *xfull_bar = empty_bar + STAGES;      // activation window loaded
  uint64_t *xfree_bar = xfull_bar + 1;           // MMAs reading the window done
  uint64_t *tfull_bar = xfree_bar + 1;
  uint64_t *tempty_bar = tfull_bar + 2;
  uint64_t *drain_bar = tempty_bar + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *last_flag = abort_flag + 1;  // one per epilogue set

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    DTRACE(0);
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(xfull_bar, 1);
    mbar_init(xfree_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 4);
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

  const int32_t nkb = static_cast<int32_t>((K + kBK - 1) / kBK);
  const int64_t tiles = (N + kTileN - 1) / kTileN;
  const int64_t total = tiles * nkb;
  const int64_t u_begin = (total * blockIdx.x) / gridDim.x;
  const int64_t u_end = (total * (blockIdx.x + 1)) / gridDim.x;
  Cursor start;
  start.u = u_begin;
  start.tile = static_cast<int32_t>(u_begin / nkb);
  start.kb = static_cast<int32_t>(u_begin - static_cast<int64_t>(start.tile) * nkb);
  start.slot = 0;
  const int64_t win0_end = u_end < u_begin + Cfg::kWindow ? u_end : u_begin + Cfg::kWindow;
  if (threadIdx.x == 0) {
    DTRACE(1);
    DTRACE_VAL(2, u_begin);
    DTRACE_VAL(3, u_end);
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------- TMA producer
      // The first ring's worth of weight tiles does not depend on the previous
      // kernel; the activation does, so it is requested after the wait.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      int win = 0;
      int64_t win_end = win0_end;
      // without a programmatic dependency the activation is ready: request it first
      const int64_t prefetch_end = !pdl ? u_begin : (u_end < u_begin + STAGES ? u_end : u_begin + STAGES);
      bool x0_requested = false;
      Cursor c = start;
      for (; c.u < u_end; c.next(nkb)) {
        if (c.u == prefetch_end) {
          pdl_wait_prerequisite();
          load_window<MP>(&tmX, xfull_bar, sX, start.kb,
                          static_cast<int32_t>(win_end - u_begin < nkb ? win_end - u_begin : nkb), nkb);
          x0_requested = true;
        }
        if (c.u == win_end) {
          // a later window (long runs only): wait until the MMAs are done with the previous one
          ++win;
          if (!mbar_wait_bounded(xfree_bar, (win - 1) & 1, abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          win_end = u_end < c.u + Cfg::kWindow ? u_end : c.u + Cfg::kWindow;
          load_window<MP>(&tmX, xfull_bar, sX, c.kb,
                          static_cast<int32_t>(win_end - c.u < nkb ? win_end - c.u : nkb), nkb);
        }
        if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[stage], kStageW);
        tma_load_2d(&tmW, &full_bar[stage], sW + stage * kStageW, c.kb * kBK, c.tile * kTileN);
        if (c.u - u_begin < 64) DTRACE(64 + (c.u - u_begin));
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && !x0_requested) {
        // the whole run fit in the prefetch: request the activation now
        pdl_wait_prerequisite();
        load_window<MP>(&tmX, xfull_bar, sX, start.kb,
                        static_cast<int32_t>(win0_end - u_begin < nkb ? win0_end - u_begin : nkb), nkb);
      }
      if (!ok) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full_bar[s], (issued_parity >> s) & 1u, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = mbar_wait_bounded(xfull_bar, 0, abort_flag, limit_ns);
      DTRACE(4);
      int win = 0;
      int64_t win_end = win0_end;
      Cursor c = start;
      while (ok && c.u < u_end) {
        const int64_t seg_end = u_end < static_cast<int64_t>(c.tile + 1) * nkb ? u_end : static_cast<int64_t>(c.tile + 1) * nkb;
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * MP);
        const int64_t seg_begin = c.u;
        for (; c.u < seg_end; c.next(nkb)) {
          if (c.u == win_end) {  // next activation window
            mma_commit(xfree_bar);
            ++win;
            win_end = u_end < c.u + Cfg::kWindow ? u_end : c.u + Cfg::kWindow;
            c.slot = 0;
            if (!mbar_wait_bounded(xfull_bar, win & 1, abort_flag, limit_ns)) {
              ok = false;
              break;
            }
          }
          if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns)) {
            ok = false;
            break;
          }
          if (c.u - u_begin < 64) DTRACE(128 + (c.u - u_begin));
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sW + stage * kStageW);
          const uint32_t b_addr = smem_addr(sX + c.slot * Cfg::kSlot);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8(d_tmem, smem_desc_k_sw128(a_addr + 32 * k), smem_desc_k_sw128(b_addr + 32 * k), kIdesc,
                   (c.u != seg_begin || k != 0) ? 1u : 0u);
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
        mma_commit(drain_bar);
        mbar_wait_bounded(drain_bar, 0, nullptr, limit_ns / 16 + 1);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ drain / epilogue
    // Two sets of four warps: set 0 drains accumulator 0 (even segments of the
    // run), set 1 accumulator 1 (odd segments), so the flush of one segment
    // overlaps the next. The four warps of a set meet at their own named
    // barrier; after a failed wait a warp keeps walking the same segments
    // (skipping the work) and still takes part in every barrier.
    pdl_wait_prerequisite();  // the previous kernel may still use the workspace or `out`
    const int set = (warp - kEpiWarp0) >> 2;
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int tid_set = threadIdx.x - (kEpiWarp0 + 4 * set) * 32;
    const bool set_leader = tid_set == 0;
    const uint32_t bar_id = 1 + set;
    uint16_t *stage = sOut + set * (Cfg::kStageOut / 2);
    const int32_t z = ep.Z ? __ldg(ep.Z) : 0;
    float sx[MP];
#pragma unroll
    for (int m = 0; m < MP; ++m) sx[m] = (m < M) ? (ep.s_x_per_row ? __ldg(ep.S_x + m) : __ldg(ep.S_x)) : 0.0f;
    const int acc = set;
    uint32_t acc_phase = 0;
    bool failed = false;
    int seg_idx = 0;
    for (int64_t u = u_begin, tile = start.tile; u < u_end; ++tile, ++seg_idx) {
      const int64_t seg_end = u_end < (tile + 1) * nkb ? u_end : (tile + 1) * nkb;
      const int64_t seg_len = seg_end - u;
      u = seg_end;
      if ((seg_idx & 1) != set) continue;
      const int row = q * 32 + lane;  // weight row within the tile
      const int64_t n = tile * kTileN + row;
      const RowParams rp = load_row_params(n, N, z, ep);
      if (!failed) {
        const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag, limit_ns));
        if (!ready) {
          failed = true;
          if (lane == 0) {
            record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
          }
        }
      }
      if (set_leader && seg_idx < 4) DTRACE(8 + 4 * seg_idx);
      int32_t v[MP];
#pragma unroll
      for (int i = 0; i < MP; ++i) v[i] = 0;
      if (!failed) {
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * MP);
        if constexpr (MP == 32) {
          uint32_t rr[32];
          tmem_ld_32x32b_x32(taddr, rr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = static_cast<int32_t>(rr[i]);
        } else {
          uint32_t rr[16];
          tmem_ld_32x32b_x16(taddr, rr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = static_cast<int32_t>(rr[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      }
      acc_phase ^= 1u;

      if (seg_len == nkb) {
        // this CTA owns the whole tile
        decode_epilogue_tile<MP>(v, sx, M, N, tile, row, tid_set, z, rp, ep, stage, bar_id, failed);
      } else {
        // Split tile: add this run's partial sums to the tile's workspace slice
        // (red.global.add: exact and order-free); the CTA that brings the tile
        // counter to nkb k-blocks reads the total back, runs the epilogue and
        // leaves slice and counter zeroed for the next call.
        int32_t *p = part + tile * (32 * kTileN);
        if (!failed) {
#pragma unroll
          for (int m = 0; m < MP; ++m)
            if (m < M) atomicAdd(p + m * kTileN + row, v[m]);
        }
        __syncwarp();
        named_barrier(bar_id, 128);
        if (set_leader) {
          int last = 0;
          if (!*abort_flag) {
            // release: the CTA's additions (ordered before by the barrier) are
            // visible before the count is
            const uint32_t before = atomic_add_release_gpu(counters + tile, static_cast<uint32_t>(seg_len));
            last = (static_cast<int64_t>(before) + seg_len == nkb) ? 1 : 0;
            if (last) fence_acquire_gpu();  // ... and the last arriver sees every other CTA's
          }
          last_flag[set] = last;
          if (seg_idx < 4) {
            DTRACE(9 + 4 * seg_idx);
            DTRACE_VAL(10 + 4 * seg_idx, last);
          }
        }
        __syncwarp();
        named_barrier(bar_id, 128);
        const bool last = last_flag[set] != 0;
        if (last) {
          if (!failed) {
#pragma unroll
            for (int m = 0; m < MP; ++m) {
              if (m < M) {
                v[m] = __ldcg(p + m * kTileN + row);
                __stcg(p + m * kTileN + row, 0);  // leave the workspace zeroed for the next call
              }
            }
          }
          if (set_leader) {
            int chk = 0;
#pragma unroll
            for (int m = 0; m < MP; ++m) chk ^= v[m];
            DTRACE(24);  // the read-back has landed (chk depends on every load)
            DTRACE_VAL(25, chk);
          }
          decode_epilogue_tile<MP>(v, sx, M, N, tile, row, tid_set, z, rp, ep, stage, bar_id, failed);
          if (set_leader) {
            DTRACE(26);
            counters[tile] = 0u;  // zero again for the next call
          }
        }
        __syncwarp();
        named_barrier(bar_id, 128);  // last_flag is rewritten by this set's next segment
      }
      if (set_leader && seg_idx < 4) DTRACE(11 + 4 * seg_idx);
    }
  }

  tc_fence_before();
  __syncwarp();  // lanes of the producer and MMA warps reconverge before the CTA barrier
  __syncthreads();
  if (threadIdx.x == 0) DTRACE(6);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int MP, int STAGES>
cudaError_t launch_decode_t(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                            const EpilogueArgs &ep, void *workspace, bool pdl, int num_sms, int32_t *status,
                            cudaStream_t s) {
  using Cfg = DecCfg<MP, STAGES>;
  alignas(64) CUtensorMap tmW, tmX;
  if (!encode_tmap_2d(&tmW, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, kTileN, true))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tmX, Xq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                      static_cast<uint64_t>(ldx), kBK, MP, true))
    return cudaErrorInvalidValue;
  auto kern = gemm_i8_decode_kernel<MP, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Cfg::kSmem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(decode_grid(N, K, num_sms));
  uint32_t *counters = static_cast<uint32_t *>(workspace);
  int32_t *part = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + decode_counters_bytes(N));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, M, N, K, ep, part, counters, pdl ? 1 : 0, status, kWaitLimitNs);
}

}  // namespace

int decode_grid(int64_t N, int64_t K, int num_sms) {
  const int64_t total = ((N + kTileN - 1) / kTileN) * ((K + kBK - 1) / kBK);
  return static_cast<int>(total < num_sms ? total : num_sms);
}

size_t decode_counters_bytes(int64_t N) {
  const int64_t tiles = (N + kTileN - 1) / kTileN;
  return static_cast<size_t>(((tiles * 4 + 255) / 256) * 256);
}

size_t decode_partials_bytes(int64_t N) {
  const int64_t tiles = (N + kTileN - 1) / kTileN;
  return static_cast<size_t>(tiles) * 32 * kTileN * sizeof(int32_t);
}

cudaError_t launch_gemm_decode(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                               const EpilogueArgs &ep, void *workspace, bool pdl, int num_sms, int32_t *status,
                               cudaStream_t s) {
  if (M <= 16) return launch_decode_t<16, 6>(Xq, ldx, Wq, M, N, K, ep, workspace, pdl, num_sms, status, s);
  return launch_decode_t<32, 6>(Xq, ldx, Wq, M, N, K, ep, workspace, pdl, num_sms, status, s);
}

}  // namespace w8a8
