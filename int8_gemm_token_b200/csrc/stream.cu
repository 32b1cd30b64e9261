// stream.cu -- the static per-tensor quantization and dequantization of
// large dense tensors (an INT8 KV cache written and read in the Decode
// scheme) as a stream through shared memory.
//
// What it computes: PDMIX glossary §2.3 eq. Q_decode,
//   q = clamp(rne(x * r) + Z, -128, 127)            (bf16 -> int8)
// and its inverse x = S * (q - Z)                  (int8 -> bf16 or fp32),
// exactly as quant_per_tensor_kernel and dequant_per_tensor_kernel in
// quant.cu (the same helpers, the same order of operations), which serve
// the strided and the small tensors.
//
// How (sm_100a): these are pure HBM streams, so the design keeps enough
// bytes in flight per SM without spending registers on them. A persistent
// grid of one CTA per SM; in each, one thread (the producer) copies 16 KiB
// tiles of the input with 1-D bulk copies (cp.async.bulk, completion on an
// mbarrier) into an 8-stage shared-memory ring -- 128 KiB in flight per SM
// -- and consumer warps (eight for the quantization, four for the
// dequantization) convert each tile from shared memory and store
// the results to global memory (coalesced 8- to 64-byte stores per thread),
// then release the stage. Tiles are dealt to the CTAs round robin.
// Programmatic dependent launch: the kernel lets its dependents launch at
// once, asks L2 for its first tiles, and waits for the previous kernel
// before its first copy. Every wait is bounded; on a timeout the CTA records
// W8A8_ERR_DEVICE_TIMEOUT, waits (bounded) for its copies in flight and returns.
#include "device.cuh"
#include "kernels.h"

namespace w8a8 {

namespace {

constexpr int kTile = 16384;  // input bytes per stage
constexpr int kStages = 8;
// Consumer warps per CTA: the quantization's per-byte arithmetic needs two
// per SM sub-partition to hide its latency; the dequantization, one.
template <int Cw>
constexpr int threads_for() { return 32 * (1 + Cw); }
constexpr size_t kSmem = static_cast<size_t>(kStages) * kTile + 2 * kStages * 8 + 16 + 128;

enum class Conv { kQuant, kDequantBf16, kDequantF32 };

// One 16-byte piece of input at element offset e (elements of the input).
template <Conv C>
__device__ __forceinline__ void convert_piece(const uint4 &v, int64_t e, void *out, float a, int z) {
  if constexpr (C == Conv::kQuant) {  // 8 bf16 -> 8 codes
    *reinterpret_cast<uint2 *>(static_cast<int8_t *>(out) + e) = quant8_asym_sat(v, a, z);
  } else {  // 16 codes -> 16 values
    float y[16];
    dequant16(v, a, z, y);
    if constexpr (C == Conv::kDequantBf16) {
      uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + e);
      o[0] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                        pack_bf16x2(y[6], y[7]));
      o[1] = make_uint4(pack_bf16x2(y[8], y[9]), pack_bf16x2(y[10], y[11]), pack_bf16x2(y[12], y[13]),
                        pack_bf16x2(y[14], y[15]));
    } else {
      float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + e);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
    }
  }
}

// in: dense input of in_bytes (a multiple of 16); out: dense output, same
// element count. a, z: r and Z (quantization) or S and Z (dequantization),
// device scalars.
template <Conv C>
constexpr int consumers_for() { return C == Conv::kQuant ? 8 : 4; }

template <Conv C>
__global__ void __launch_bounds__(threads_for<consumers_for<C>()>(), 1)
    stream_convert_kernel(const uint8_t *__restrict__ in, int64_t in_bytes, void *__restrict__ out,
                          const float *__restrict__ a_ptr, const int32_t *__restrict__ z_ptr, int32_t *status,
                          uint64_t limit_ns) {
  constexpr int kElem = C == Conv::kQuant ? 2 : 1;  // input bytes per element
  constexpr int kConsumers = consumers_for<C>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *ring = smem_raw;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(ring + static_cast<size_t>(kStages) * kTile);
  uint64_t *empty_bar = full_bar + kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty_bar + kStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_tiles = (in_bytes + kTile - 1) / kTile;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumers);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane != 0) return;
    // ------------------------------------------------ producer
    for (int i = 0; i < kStages; ++i) {  // the first ring of tiles, asked of L2 before the wait
      const int64_t t = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
      if (t >= n_tiles) break;
      const int64_t off = t * kTile;
      prefetch_l2_bulk(in + off, static_cast<uint32_t>(in_bytes - off < kTile ? in_bytes - off : kTile));
    }
    pdl_wait_prerequisite();
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    int i = 0;
    for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int s = i % kStages;
      const uint32_t ph = static_cast<uint32_t>(i / kStages) & 1u;
      if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, abort_flag, limit_ns)) {
        ok = false;
        break;
      }
      const int64_t off = t * kTile;
      const uint32_t bytes = static_cast<uint32_t>(in_bytes - off < kTile ? in_bytes - off : kTile);
      mbar_arrive_expect_tx(&full_bar[s], bytes);
      bulk_load_1d(ring + s * kTile, in + off, bytes, &full_bar[s]);
      issued_mask |= 1u << s;
      issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
    }
    if (!ok) {
      record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
      *abort_flag = 1;
      for (int s = 0; s < kStages; ++s)  // this CTA's copies land before its shared memory goes away
        if (issued_mask & (1u << s))
          mbar_wait_bounded(&full_bar[s], (issued_parity >> s) & 1u, nullptr, limit_ns / 16 + 1);
    }
    return;
  }
  // -------------------------------------------------- consumers
  pdl_wait_prerequisite();  // the scalars (and `out`) belong to the previous kernel until then
  const float a = __ldg(a_ptr);
  const int z = __ldg(z_ptr);
  const int ct = threadIdx.x - 32;  // 0 .. 32 * kConsumers - 1
  int i = 0;
  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
    const int s = i % kStages;
    const uint32_t ph = static_cast<uint32_t>(i / kStages) & 1u;
    const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full_bar[s], ph, abort_flag, limit_ns));
    if (!ready) {
      if (lane == 0) {
        record_error(status, W8A8_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
      }
      break;
    }
    const int64_t off = t * kTile;
    const int pieces = static_cast<int>((in_bytes - off < kTile ? in_bytes - off : kTile) / 16);
    const uint8_t *tile = ring + s * kTile;
#pragma unroll 4
    for (int p = ct; p < pieces; p += 32 * kConsumers)
      convert_piece<C>(*reinterpret_cast<const uint4 *>(tile + p * 16), (off + p * 16) / kElem, out, a, z);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }
}

template <Conv C>
cudaError_t launch_stream_t(const void *in, int64_t in_bytes, void *out, const float *a, const int32_t *z, int num_sms,
                            int32_t *status, cudaStream_t s) {
  cudaError_t e = ensure_kernel_smem<stream_convert_kernel<C>>(static_cast<int>(kSmem), true);
  if (e != cudaSuccess) return e;
  const int64_t n_tiles = (in_bytes + kTile - 1) / kTile;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_tiles < num_sms ? n_tiles : num_sms));
  cfg.blockDim = dim3(threads_for<consumers_for<C>()>());
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stream_convert_kernel<C>, static_cast<const uint8_t *>(in), in_bytes, out, a, z,
                            status, kWaitLimitNs);
}

}  // namespace

cudaError_t launch_quant_per_tensor_stream(const uint16_t *X, int64_t elems, const float *r, const int32_t *Z,
                                           int8_t *Xq, int num_sms, int32_t *status, cudaStream_t s) {
  return launch_stream_t<Conv::kQuant>(X, elems * 2, Xq, r, Z, num_sms, status, s);
}

cudaError_t launch_dequant_per_tensor_stream(const int8_t *Xq, int64_t elems, const float *S, const int32_t *Z,
                                             void *out, bool bf16_out, int num_sms, int32_t *status,
                                             cudaStream_t s) {
  if (bf16_out) return launch_stream_t<Conv::kDequantBf16>(Xq, elems, out, S, Z, num_sms, status, s);
  return launch_stream_t<Conv::kDequantF32>(Xq, elems, out, S, Z, num_sms, status, s);
}

}  // namespace w8a8
