// dispatch_mxfp4.cuh -- step 3: expert-grouped MXFP4 send buffer at one GPU.
//
// MAX "Struct_ep_dispatch_async_mxfp4", execute(): tokens travel as MXFP4
// with their block scales packed alongside the FP4 quants.  At one GPU the
// send buffer is the receive buffer and the destination row of pair p is
// restore_token_order[p] (from moe_create_indices), so no slot claiming is
// needed and the row order is deterministic.
//
// One warp per token: the row is read once (128-bit loads, 8 bf16 per
// lane), encoded once, and the encoded 32-bit words are stored to each of
// the token's routed rows.  A 32-element MX block is 4 lanes; its amax is a
// 2-step xor-shuffle.  Padding tokens (all slots unrouted) are skipped.
#pragma once
#include "common.cuh"

namespace moe {
namespace disp {

constexpr int kWarpsPerBlock = 8;

// E8M0 exponent of a block: floor(log2(amax)) - 2 clamped to [-127, 127];
// amax == 0 gives -127.  Exact integer arithmetic on the fp32 bits.
__device__ __forceinline__ int mx_shared_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ex = (int)((b >> 23) & 0xFFu);
  int fl;
  if (ex != 0) {
    fl = ex - 127;
  } else {
    const uint32_t m = b & 0x7FFFFFu;
    if (m == 0) return -127;
    fl = (31 - __clz((int)m)) - 149;
  }
  int se = fl - 2;
  se = se < -127 ? -127 : (se > 127 ? 127 : se);
  return se;
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    dispatch_mxfp4_kernel(const uint16_t *__restrict__ x, int32_t N, int32_t K, int32_t top_k,
                          int32_t E, const uint32_t *__restrict__ restore,
                          const uint32_t *__restrict__ start,
                          const int32_t *__restrict__ expert_ids,
                          const uint32_t *__restrict__ stats, uint8_t *__restrict__ recv,
                          int64_t capacity, int32_t stride, uint32_t *__restrict__ counts) {
  const unsigned lane = lane_id();
  if (blockIdx.x == 0) {  // recv_counts[e] from the CSR offsets
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0u;
    __syncthreads();
    const uint32_t A = stats[1];
    for (uint32_t a = threadIdx.x; a < A; a += blockDim.x)
      counts[expert_ids[a]] = start[a + 1] - start[a];
  }
  const int warps_total = gridDim.x * kWarpsPerBlock;
  const int half = K / 2;
  const int nscale = K / 32;
  for (int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < N; t += warps_total) {
    // destinations of this token's slots (top_k <= 32 per step)
    for (int j0 = 0; j0 < top_k; j0 += 32) {
      const int j = j0 + (int)lane;
      uint32_t dest = 0xFFFFFFFFu;
      if (j < top_k) dest = restore[(int64_t)t * top_k + j];
      bool ok = dest != 0xFFFFFFFFu;
      if (ok && (int64_t)dest >= capacity) {
        raise_device_error(MOE_DEVERR_RECV_OVERFLOW);
        ok = false;
      }
      const unsigned dmask = __ballot_sync(0xffffffffu, ok);
      if (dmask == 0u) continue;
      const uint16_t *row = x + (int64_t)t * K;
      for (int seg = 0; seg < K; seg += 256) {
        const int k = seg + 8 * (int)lane;
        const bool active = k < K;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (active) v = ldg_nc_v4(row + k);
        float f[8];
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
        f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
        f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int se = mx_shared_exponent(amax);
        const float mult = __uint_as_float((uint32_t)(127 - se) << 23);  // 2^-se, exact
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = f[i] * mult;
        const uint32_t codes = e2m1x8_from_f32(q);
        // store to every routed row of this token
        unsigned m = dmask;
        while (m) {
          const int src = __ffs(m) - 1;
          m &= m - 1;
          const uint32_t d = __shfl_sync(0xffffffffu, dest, src);
          uint8_t *dst = recv + (int64_t)d * stride;
          if (active) {
            *reinterpret_cast<uint32_t *>(dst + k / 2) = codes;
            if ((lane & 3u) == 0u) dst[half + k / 32] = (uint8_t)(se + 127);
          }
        }
      }
      // zero padding after the scales
      const int pad0 = half + nscale;
      unsigned m = dmask;
      while (m) {
        const int src = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t d = __shfl_sync(0xffffffffu, dest, src);
        for (int b = pad0 + (int)lane; b < stride; b += 32) recv[(int64_t)d * stride + b] = 0;
      }
    }
  }
}

}  // namespace disp
}  // namespace moe
