// gemm_decode.cu -- Decode-shaped W8A8 linear (1..64 tokens): the GEMM is a
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
//     the tokens, padded to MP = 16, 32 or 64, are the MMA's N dimension;
//   * one cluster of SPLIT CTAs per 128-row tile; CTA rank r of the cluster
//     owns the k-blocks [r nkb / SPLIT, (r+1) nkb / SPLIT). SPLIT (1..8) is
//     the largest whose clusters are all resident at once (with at least two
//     k-blocks per CTA), so small N still spreads over the GPU and large N
//     needs no split;
//   * CTAs are small (~100 KiB of shared memory) so that two share an SM:
//     that doubles the copies in flight per SM and lets the next kernel's
//     CTAs start streaming while this kernel's last CTAs finish;
//   * warp 0 streams the weight tile and the matching activation k-block
//     through a TMA ring (3-6 stages of 16 KiB + the activation, 128B
//     swizzle); warp 1 issues tcgen05.mma kind::i8 (M = 128, N = MP) into
//     one TMEM accumulator;
//   * FUSEQ (the one-kernel Decode linear): the activation arrives as bf16,
//     two [MP][64] boxes per k-block, and the four epilogue warps -- idle
//     until the last MMA -- quantize it into the 128B-swizzled int8 operand,
//     fence it for the tensor core and signal a per-stage barrier that the
//     MMA issuer also waits on;
//   * when the accumulator is full, each epilogue thread holds one weight row
//     for every token (tcgen05.ld). Rows are owned by cluster ranks in 8-row
//     groups: a CTA keeps the partial sums of its own rows in its idle weight
//     ring and stores the others into the owner's shared memory
//     (st.shared::cluster). After one cluster barrier all 256 threads add the
//     SPLIT partials (exact int32) of chunks of 8 outputs, run the epilogue
//     with the per-channel constants fetched before the barrier, and store 16
//     bytes at a time (8 when the epilogue writes the next linear's int8
//     codes of the bf16 result instead). No global workspace, no atomics;
//   * programmatic dependent launch: the kernel lets its dependents launch
//     as soon as it has started, and requests its first ring of weight tiles
//     before it waits for the previous kernel in the stream
//     (griddepcontrol.wait), so the weight stream overlaps the preceding
//     quantization kernel and the tail of the previous decode GEMM. The
//     weight is the one operand read before that wait; the activation, the
//     scales and the output are touched only after it.
#include <atomic>

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

// First weight row of a tile that cluster rank j finishes (j = SPLIT gives the
// end of the tile): j * 128 / SPLIT rounded down to a multiple of 8, so that
// every owner's rows start on a 16-byte boundary of the output.
template <int SPLIT>
__host__ __device__ constexpr int owner_row0(int j) {
  return j >= SPLIT ? kTileN : ((j * kTileN / SPLIT) & ~7);
}

template <int SPLIT>
constexpr int max_owned_rows() {
  int r = 0;
  for (int j = 0; j < SPLIT; ++j) {
    const int d = owner_row0<SPLIT>(j + 1) - owner_row0<SPLIT>(j);
    if (d > r) r = d;
  }
  return r;
}

template <int MP, int SPLIT, bool FUSEQ>
struct DecCfg {
  static constexpr int kStageX = MP * kBK;  // int8 activation k-block (128B-swizzled MMA operand)
  // FUSEQ: the bf16 activation k-block as loaded, two [MP][64] boxes
  static constexpr int kStageXb = FUSEQ ? 2 * MP * kBK : 0;
  static constexpr int kStage = kStageW + kStageX + kStageXb;
  // weight rows one CTA finishes, at most (a multiple of 8)
  static constexpr int kR = max_owned_rows<SPLIT>();
  // partial sums this CTA receives from the other SPLIT-1 CTAs of its cluster
  static constexpr int kRedBytes = (SPLIT - 1) * MP * kR * 4;
  // two CTAs per SM: 228 KiB per SM, 1 KiB of it reserved per CTA
  static constexpr int kBudget = 228 * 1024 / kCtasPerSm - 1024 - 1024 /*alignment slack*/ - 256 /*barriers*/;
  static constexpr int kStagesFit = (kBudget - kRedBytes) / kStage;
  static constexpr int kStages = kStagesFit < 6 ? kStagesFit : 6;
  static constexpr size_t kSmem = static_cast<size_t>(kStages) * kStage + kRedBytes + 1024 + 256;
  static constexpr int kTmemCols = MP < 32 ? 32 : MP;  // one int32 column per padded token
  static_assert(kR % 8 == 0, "owned rows in 8-row groups");
  static_assert(kStageX % 1024 == 0 && kStageXb % 1024 == 0, "1 KiB alignment of activation stages");
  static_assert(kStages >= 3, "ring depth");
  static_assert(MP * kR * 4 <= kStages * kStageW, "this CTA's own partial sums fit in the weight ring");
  static_assert(kCtasPerSm * (kSmem + 1024) <= 228 * 1024, "two CTAs per SM");
};

// 8 consecutive int32 from this CTA's shared memory (32-byte aligned address).
__device__ __forceinline__ void ld_shared_8(uint32_t addr, int32_t (&v)[8]) {
  asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(addr));
  asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(addr + 16));
}

// Per-channel constants of outputs n0 .. n0+7 (n0 a multiple of 8; zero past N).
struct Consts8 {
  float sw[8], bs[8];
  int32_t cs[8];
};

__device__ __forceinline__ void load_consts8(const EpilogueArgs &ep, int64_t n0, int64_t N, int32_t z, Consts8 &k) {
  if (n0 + 8 <= N) {
    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(ep.s_w + n0));
    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(ep.s_w + n0) + 1);
    k.sw[0] = w0.x; k.sw[1] = w0.y; k.sw[2] = w0.z; k.sw[3] = w0.w;
    k.sw[4] = w1.x; k.sw[5] = w1.y; k.sw[6] = w1.z; k.sw[7] = w1.w;
    if (ep.bias) {
      const float4 b0 = __ldg(reinterpret_cast<const float4 *>(ep.bias + n0));
      const float4 b1 = __ldg(reinterpret_cast<const float4 *>(ep.bias + n0) + 1);
      k.bs[0] = b0.x; k.bs[1] = b0.y; k.bs[2] = b0.z; k.bs[3] = b0.w;
      k.bs[4] = b1.x; k.bs[5] = b1.y; k.bs[6] = b1.z; k.bs[7] = b1.w;
    }
    if (z != 0) {
      const int4 c0 = __ldg(reinterpret_cast<const int4 *>(ep.colsum + n0));
      const int4 c1 = __ldg(reinterpret_cast<const int4 *>(ep.colsum + n0) + 1);
      k.cs[0] = c0.x; k.cs[1] = c0.y; k.cs[2] = c0.z; k.cs[3] = c0.w;
      k.cs[4] = c1.x; k.cs[5] = c1.y; k.cs[6] = c1.z; k.cs[7] = c1.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool ok = n0 + i < N;
      k.sw[i] = ok ? __ldg(ep.s_w + n0 + i) : 0.0f;
      k.bs[i] = (ok && ep.bias) ? __ldg(ep.bias + n0 + i) : 0.0f;
      k.cs[i] = (ok && z != 0) ? __ldg(ep.colsum + n0 + i) : 0;
    }
  }
}

// The epilogue of 8 consecutive outputs out[m, n0 .. n0+7] (n0 a multiple of
// 8), each in the fixed order of include/w8a8.h:
// c = acc - Z*colsum[n]; y = fmaf(float(c), S_x[m]*s_w[n], bias[n]).
// kOutRequantI8 stores the next linear's static code of bf16(y) instead, with
// its scalars rq = r_out and zq = Z_out.
__device__ __forceinline__ void epilogue8(const EpilogueArgs &ep, int64_t m, int64_t n0, int64_t N,
                                          const int32_t (&a)[8], int32_t z, float sx, const Consts8 &k,
                                          float rq, int32_t zq) {
  const bool full = n0 + 8 <= N;
  int32_t c[8];
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = z != 0 ? a[i] - z * k.cs[i] : a[i];
    float add = 0.0f;
    if (ep.bias) add = __fadd_rn(add, k.bs[i]);
    y[i] = __fmaf_rn(__int2float_rn(c[i]), __fmul_rn(sx, k.sw[i]), add);
  }
  const int64_t o = m * N + n0;
  if (ep.out_dtype == W8A8_BF16) {
    uint16_t *out = static_cast<uint16_t *>(ep.out) + o;
    if (full && (o % 8) == 0) {
      uint4 v;
      v.x = pack_bf16x2(y[0], y[1]);
      v.y = pack_bf16x2(y[2], y[3]);
      v.z = pack_bf16x2(y[4], y[5]);
      v.w = pack_bf16x2(y[6], y[7]);
      *reinterpret_cast<uint4 *>(out) = v;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (n0 + i < N) {
          __nv_bfloat16 b = __float2bfloat16_rn(y[i]);
          out[i] = *reinterpret_cast<uint16_t *>(&b);
        }
    }
  } else if (ep.out_dtype == kOutRequantI8) {
    uint4 v;  // bf16(y), exactly as the bf16 output stores it
    v.x = pack_bf16x2(y[0], y[1]);
    v.y = pack_bf16x2(y[2], y[3]);
    v.z = pack_bf16x2(y[4], y[5]);
    v.w = pack_bf16x2(y[6], y[7]);
    const uint2 q = quant8_asym_sat(v, rq, zq);
    int8_t *out = static_cast<int8_t *>(ep.out) + o;
    if (full && (o % 8) == 0) {
      *reinterpret_cast<uint2 *>(out) = q;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (n0 + i < N) out[i] = static_cast<int8_t>(((i < 4 ? q.x : q.y) >> (8 * (i & 3))) & 0xFFu);
    }
  } else if (ep.out_dtype == W8A8_FP32) {
    float *out = static_cast<float *>(ep.out) + o;
    if (full && (o % 4) == 0) {
      reinterpret_cast<float4 *>(out)[0] = make_float4(y[0], y[1], y[2], y[3]);
      reinterpret_cast<float4 *>(out)[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (n0 + i < N) out[i] = y[i];
    }
  } else {
    int32_t *out = static_cast<int32_t *>(ep.out) + o;
    if (full && (o % 4) == 0) {
      reinterpret_cast<int4 *>(out)[0] = make_int4(c[0], c[1], c[2], c[3]);
      reinterpret_cast<int4 *>(out)[1] = make_int4(c[4], c[5], c[6], c[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (n0 + i < N) out[i] = c[i];
    }
  }
}

constexpr int kQuantThreads = 128;       // FUSEQ: the epilogue warps quantize the activation first

// TMA of one activation k-block into ring slot `slot`: the int8 operand
// directly (128B swizzle), or with FUSEQ the bf16 k-block as two [MP][64]
// boxes (no swizzle) for the quantizer warps.
template <int MP, bool FUSEQ>
__device__ __forceinline__ void load_activation(const CUtensorMap *tmX, uint64_t *bar, uint8_t *sX, uint8_t *sXb,
                                                int slot, int32_t kb) {
  if constexpr (FUSEQ) {
    uint8_t *dst = sXb + slot * (2 * MP * kBK);
    tma_load_2d(tmX, bar, dst, kb * kBK, 0);
    tma_load_2d(tmX, bar, dst + MP * kBK, kb * kBK + kBK / 2, 0);
  } else {
    tma_load_2d(tmX, bar, sX + slot * (MP * kBK), kb * kBK, 0);
  }
}

// Static per-tensor quantization of one bf16 k-block [MP][128] (two [MP][64]
// boxes) into the int8 operand layout the MMA reads: K-major, 128-byte rows,
// the 16-byte chunk c of row m stored at chunk c ^ (m % 8). Thread qt of 128
// takes the 8-element groups qt, qt + 128, ...: all its loads first, then the
// arithmetic, then the stores, so the groups overlap; a warp reads 512
// contiguous bytes per load. Source: PDMIX glossary §2.3 eq. Q_decode,
// q = clamp(rne(x * r) + Z).
template <int MP>
__device__ __forceinline__ void quantize_stage(const uint8_t *xb, uint8_t *xq, int qt, float r, int z) {
  constexpr int kPer = 2 * MP * 8 / kQuantThreads;  // groups per thread
  static_assert(kPer * kQuantThreads == 2 * MP * 8, "whole groups per thread");
  uint4 v[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) v[j] = *reinterpret_cast<const uint4 *>(xb + (qt + j * kQuantThreads) * 16);
  uint2 q[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) q[j] = quant8_asym_sat(v[j], r, z);
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int g = qt + j * kQuantThreads;
    const int h = g / (MP * 8);           // box: elements [64 h, 64 h + 64) of the k-block
    const int m = (g >> 3) - h * MP;      // row
    const int e = (g & 7) * 8 + h * 64;   // first of the 8 elements within the k-block
    *reinterpret_cast<uint2 *>(xq + m * kBK + (((e >> 4) ^ (m & 7)) << 4) + (e & 8)) = q[j];
  }
}

template <int MP, int SPLIT, bool FUSEQ>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    gemm_i8_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                          int64_t M, int64_t N, int64_t K, const __grid_constant__ EpilogueArgs ep,
                          const float *q_r, const int32_t *q_z, int32_t *status, uint64_t limit_ns) {
  using Cfg = DecCfg<MP, SPLIT, FUSEQ>;
  constexpr uint32_t kIdesc = idesc_i8(kTileN, MP);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sW = base;                            // kStages x 16 KiB weight ring
  uint8_t *sX = sW + Cfg::kStages * kStageW;     // kStages x MP*128 int8 activation ring
  uint8_t *sXb = sX + Cfg::kStages * Cfg::kStageX;  // FUSEQ: kStages x 2*MP*128 bf16 activation ring
  int32_t *sRed = reinterpret_cast<int32_t *>(sXb + Cfg::kStages * Cfg::kStageXb);  // [SPLIT-1][MP][kR]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sRed) + Cfg::kRedBytes);
  uint64_t *empty_bar = full_bar + Cfg::kStages;
  uint64_t *xq_bar = empty_bar + Cfg::kStages;  // FUSEQ: the int8 operand of a stage is written
  uint64_t *tfull_bar = xq_bar + Cfg::kStages;
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
      mbar_init(&xq_bar[s], kQuantThreads);
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
      constexpr uint32_t kTx = kStageW + (FUSEQ ? Cfg::kStageXb : Cfg::kStageX);
      const int32_t prefetch = nk < Cfg::kStages ? nk : Cfg::kStages;
      for (int32_t i = 0; i < prefetch; ++i) {  // the ring starts empty: no waits
        mbar_arrive_expect_tx(&full_bar[i], kTx);
        tma_load_2d(&tmW, &full_bar[i], sW + i * kStageW, (kb0 + i) * kBK, wrow);
      }
      pdl_wait_prerequisite();
      for (int32_t i = 0; i < prefetch; ++i) load_activation<MP, FUSEQ>(&tmX, &full_bar[i], sX, sXb, i, kb0 + i);
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
        mbar_arrive_expect_tx(&full_bar[stage], kTx);
        tma_load_2d(&tmW, &full_bar[stage], sW + stage * kStageW, (kb0 + i) * kBK, wrow);
        load_activation<MP, FUSEQ>(&tmX, &full_bar[stage], sX, sXb, stage, kb0 + i);
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
        if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns) ||
            (FUSEQ && !mbar_wait_bounded(&xq_bar[stage], phase, abort_flag, limit_ns))) {
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

  if (FUSEQ && warp >= kEpiWarp0) {
    // ------------------------------------------------ activation quantizers (FUSEQ)
    // Per stage: the bf16 k-block [MP][128] -> the int8 operand, fenced for
    // the tensor core, then xq_bar. The epilogue warps are idle until tfull.
    pdl_wait_prerequisite();  // r and Z may be written by the previous kernel
    const float r = __ldg(q_r);
    const int z = __ldg(q_z);
    const int qt = threadIdx.x - kEpiWarp0 * 32;
    int stage = 0;
    uint32_t phase = 0;
    for (int32_t i = 0; i < nk; ++i) {
      if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit_ns)) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      quantize_stage<MP>(sXb + stage * Cfg::kStageXb, sX + stage * Cfg::kStageX, qt, r, z);
      fence_proxy_async_smem();
      mbar_arrive(&xq_bar[stage]);
      if (++stage == Cfg::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }

  // ------------------------------------------------ partial sums -> shared memory
  // Epilogue thread t holds row t of the tile (its TMEM lane). Rows
  // [owner_row0(j), owner_row0(j+1)) are finished by cluster rank j: the
  // owner keeps its own partial sums in its (now idle) weight ring, the other
  // ranks store theirs into the owner's sRed.
  const int t = threadIdx.x - kEpiWarp0 * 32;  // epilogue thread index (negative elsewhere)
  uint32_t owner = 0;
#pragma unroll
  for (int j = 1; j < SPLIT; ++j)
    if (t >= owner_row0<SPLIT>(j)) owner = static_cast<uint32_t>(j);
  const int owner_r0 = owner_row0<SPLIT>(static_cast<int>(owner));
  const int rows_m = static_cast<int>(M < MP ? M : MP);
  int32_t *sOwn = reinterpret_cast<int32_t *>(sW);  // [MP][kR], once this CTA's MMAs are done
  if (warp >= kEpiWarp0) {
    pdl_wait_prerequisite();  // the bounded wait below counts from here, not from an early launch
    // tfull: every MMA of this CTA has completed (the weight ring is idle)
    const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(tfull_bar, 0, abort_flag, limit_ns));
    if (!ready) {
      if (lane == 0) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
    } else {
      tc_fence_after();
      uint32_t acc[MP];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>((warp - kEpiWarp0) * 32) << 16);
      if constexpr (MP == 64) {
        tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&acc[0]));
        tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&acc[32]));
      } else if constexpr (MP == 32) {
        tmem_ld_32x32b_x32(taddr, acc);
      } else {
        tmem_ld_32x32b_x16(taddr, acc);
      }
      tmem_ld_wait();
      tc_fence_before();
      if (owner == rank) {
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < rows_m) sOwn[m * Cfg::kR + (t - owner_r0)] = static_cast<int32_t>(acc[m]);
      } else {
        // sRed[slot][m][row - owner_row0(owner)] of the owner
        const int slot = static_cast<int>(rank < owner ? rank : rank - 1);
        const uint32_t dst = map_to_rank(sRed + slot * MP * Cfg::kR + (t - owner_r0), owner);
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < rows_m) st_shared_cluster(dst + 4u * static_cast<uint32_t>(m * Cfg::kR), acc[m]);
      }
    }
  }
  // Thread i finishes chunks of 8 outputs (token m, 8 consecutive owned rows);
  // the constants of its first chunk are fetched before the barrier.
  pdl_wait_prerequisite();  // the previous kernel may still read `out` or write S_x, s_w, ...
  const int r0 = owner_row0<SPLIT>(static_cast<int>(rank));
  const int per_m = (owner_row0<SPLIT>(static_cast<int>(rank) + 1) - r0) / 8;
  const int32_t z = ep.Z ? __ldg(ep.Z) : 0;
  const float sx0 = ep.s_x_per_row ? 0.0f : __ldg(ep.S_x);
  const bool requant = ep.out_dtype == kOutRequantI8;
  const float rq = requant ? __ldg(ep.r_out) : 0.0f;
  const int32_t zq = requant ? __ldg(ep.z_out) : 0;
  Consts8 k0;
  {
    const int m = static_cast<int>(threadIdx.x) / per_m;
    const int64_t n0 = tile * kTileN + r0 + 8 * (static_cast<int>(threadIdx.x) - m * per_m);
    if (static_cast<int>(threadIdx.x) < rows_m * per_m && n0 < N) load_consts8(ep, n0, N, z, k0);
  }
  __syncwarp();
  if constexpr (SPLIT > 1)
    cluster_sync_all();  // every partial sum has landed (release / acquire); no remote access after this
  else
    __syncthreads();

  // ------------------------------------------------ sum + epilogue, all threads
  if (!*abort_flag) {
    for (int idx = threadIdx.x; idx < rows_m * per_m; idx += kThreads) {
      const int m = idx / per_m;
      const int rl = 8 * (idx - m * per_m);  // first of the 8 rows, within this CTA's rows
      const int64_t n0 = tile * kTileN + r0 + rl;
      if (n0 >= N) continue;
      Consts8 kc;
      if (idx == static_cast<int>(threadIdx.x))
        kc = k0;
      else
        load_consts8(ep, n0, N, z, kc);
      int32_t a[8];
      ld_shared_8(smem_addr(sOwn + m * Cfg::kR + rl), a);
#pragma unroll 2
      for (int j = 0; j < SPLIT - 1; ++j) {
        int32_t p[8];
        ld_shared_8(smem_addr(sRed + (j * MP + m) * Cfg::kR + rl), p);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] += p[i];
      }
      const float sx = ep.s_x_per_row ? __ldg(ep.S_x + m) : sx0;
      epilogue8(ep, m, n0, N, a, z, sx, kc, rq, zq);
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

// Dynamic shared memory of the kernel, and the largest shared-memory carveout:
// without it the driver may size the carveout for one CTA per SM.
template <int MP, int SPLIT, bool FUSEQ>
cudaError_t configure_decode_kernel() {
  return ensure_kernel_smem<gemm_i8_decode_kernel<MP, SPLIT, FUSEQ>>(static_cast<int>(DecCfg<MP, SPLIT, FUSEQ>::kSmem),
                                                                     true);
}

// The activation operand: int8 Xq [M, K] (row stride ldx bytes) or, with
// FUSEQ, bf16 X [M, K] (row stride ldx elements) with the static r and Z.
struct DecodeActivation {
  const void *x;
  int64_t ldx;
  const float *r;
  const int32_t *z;
};

template <int MP, int SPLIT, bool FUSEQ>
cudaError_t launch_decode_t(const DecodeActivation &act, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                            const EpilogueArgs &ep, int32_t *status, cudaStream_t s) {
  using Cfg = DecCfg<MP, SPLIT, FUSEQ>;
  alignas(64) CUtensorMap tmW, tmX;
  if (!encode_tmap_2d(&tmW, Wq, TmapType::kU8, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), kBK, kTileN, true))
    return cudaErrorInvalidValue;
  const bool ok_x = FUSEQ ? encode_tmap_2d(&tmX, act.x, TmapType::kBF16, static_cast<uint64_t>(K),
                                           static_cast<uint64_t>(M), static_cast<uint64_t>(act.ldx) * 2, kBK / 2,
                                           MP, false)
                          : encode_tmap_2d(&tmX, act.x, TmapType::kU8, static_cast<uint64_t>(K),
                                           static_cast<uint64_t>(M), static_cast<uint64_t>(act.ldx), kBK, MP, true);
  if (!ok_x) return cudaErrorInvalidValue;
  auto kern = gemm_i8_decode_kernel<MP, SPLIT, FUSEQ>;
  cudaError_t e = configure_decode_kernel<MP, SPLIT, FUSEQ>();
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
  return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, M, N, K, ep, act.r, act.z, status, kWaitLimitNs);
}

// A kernel with the decode kernel's launch shape and no body. The runtime's
// occupancy answer for the decode kernel itself is one CTA per SM (it
// allocates tensor memory), while the hardware runs two of its CTAs per SM
// (32 TMEM columns each); the answer for this stand-in gives how clusters of a
// CTA of that size pack into the GPCs.
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_occupancy_standin() {}

// Clusters of SPLIT decode CTAs that can be resident at once on the current
// device (cached per device).
template <int MP, int SPLIT, bool FUSEQ>
int max_active_clusters() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 0;
  }
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  using Cfg = DecCfg<MP, SPLIT, FUSEQ>;
  if (cudaFuncSetAttribute(decode_occupancy_standin, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           200 * 1024) != cudaSuccess ||
      cudaFuncSetAttribute(decode_occupancy_standin, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(SPLIT);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = SPLIT;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, decode_occupancy_standin, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int MP, bool FUSEQ>
int max_active_clusters_of(int split) {
  switch (split) {
    case 8: return max_active_clusters<MP, 8, FUSEQ>();
    case 7: return max_active_clusters<MP, 7, FUSEQ>();
    case 6: return max_active_clusters<MP, 6, FUSEQ>();
    case 5: return max_active_clusters<MP, 5, FUSEQ>();
    case 4: return max_active_clusters<MP, 4, FUSEQ>();
    case 3: return max_active_clusters<MP, 3, FUSEQ>();
    case 2: return max_active_clusters<MP, 2, FUSEQ>();
    default: return max_active_clusters<MP, 1, FUSEQ>();
  }
}

// Largest cluster size (1..8) whose clusters, one per 128-row tile, are all
// resident at once, with at least 2 k-blocks per CTA.
template <int MP, bool FUSEQ>
int decode_split_mp(int64_t N, int64_t K) {
  const int64_t tiles = (N + kTileN - 1) / kTileN;
  const int64_t nkb = (K + kBK - 1) / kBK;
  for (int s = kMaxSplit; s >= 2; --s)
    if (nkb >= 2 * s && tiles <= max_active_clusters_of<MP, FUSEQ>(s)) return s;
  return 1;
}

template <int MP, bool FUSEQ>
cudaError_t launch_decode_mp(const DecodeActivation &act, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                             const EpilogueArgs &ep, int32_t *status, cudaStream_t s) {
  switch (decode_split_mp<MP, FUSEQ>(N, K)) {
    case 8: return launch_decode_t<MP, 8, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    case 7: return launch_decode_t<MP, 7, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    case 6: return launch_decode_t<MP, 6, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    case 5: return launch_decode_t<MP, 5, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    case 4: return launch_decode_t<MP, 4, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    case 3: return launch_decode_t<MP, 3, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    case 2: return launch_decode_t<MP, 2, FUSEQ>(act, Wq, M, N, K, ep, status, s);
    default: return launch_decode_t<MP, 1, FUSEQ>(act, Wq, M, N, K, ep, status, s);
  }
}

}  // namespace

int decode_split(int64_t M, int64_t N, int64_t K, bool fused_quant) {
  if (fused_quant) return M <= 16 ? decode_split_mp<16, true>(N, K) : decode_split_mp<32, true>(N, K);
  if (M <= 16) return decode_split_mp<16, false>(N, K);
  return M <= 32 ? decode_split_mp<32, false>(N, K) : decode_split_mp<64, false>(N, K);
}

cudaError_t launch_gemm_decode(const int8_t *Xq, int64_t ldx, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                               const EpilogueArgs &ep, int32_t *status, cudaStream_t s) {
  const DecodeActivation act{Xq, ldx, nullptr, nullptr};
  if (M <= 16) return launch_decode_mp<16, false>(act, Wq, M, N, K, ep, status, s);
  if (M <= 32) return launch_decode_mp<32, false>(act, Wq, M, N, K, ep, status, s);
  return launch_decode_mp<64, false>(act, Wq, M, N, K, ep, status, s);
}

cudaError_t launch_linear_static_decode(const uint16_t *X, int64_t ldx, const float *r, const int32_t *Z,
                                        const int8_t *Wq, int64_t M, int64_t N, int64_t K, const EpilogueArgs &ep,
                                        int32_t *status, cudaStream_t s) {
  const DecodeActivation act{X, ldx, r, Z};
  if (M <= 16) return launch_decode_mp<16, true>(act, Wq, M, N, K, ep, status, s);
  return launch_decode_mp<32, true>(act, Wq, M, N, K, ep, status, s);
}

}  // namespace w8a8
