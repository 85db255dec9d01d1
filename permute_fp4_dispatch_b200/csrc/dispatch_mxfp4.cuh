// dispatch_mxfp4.cuh -- step 3: expert-grouped MXFP4 send buffer at one GPU.
//
// MAX "Struct_ep_dispatch_async_mxfp4", execute(): tokens travel as MXFP4
// with their block scales packed alongside the FP4 quants.  At one GPU the
// send buffer is the receive buffer and the destination row of pair p is
// restore_token_order[p] (from moe_create_indices), so no slot claiming is
// needed and the row order is deterministic.
//
// One warp per (token, group of SEG segments of 256 columns): the row is read
// once (128-bit loads, 8 bf16 per lane, all of the group's loads in flight
// together), encoded once, and the encoded 32-bit words are stored to each of
// the token's routed rows.  The host picks SEG (8, 4, 2 or 1) so that even a
// decode batch of a hundred tokens spreads over every SM.  A 32-element MX block is 4 lanes; its
// amax is a 2-step xor-shuffle.  Padding tokens (no routed slot) write
// nothing.
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

template <int SEG>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    dispatch_mxfp4_kernel(const uint16_t *__restrict__ x, int32_t N, int32_t K, int32_t top_k,
                          int32_t E, const uint32_t *__restrict__ restore,
                          const uint32_t *__restrict__ start,
                          const int32_t *__restrict__ expert_ids,
                          const uint32_t *__restrict__ stats, uint8_t *__restrict__ recv,
                          int64_t capacity, int32_t stride, uint32_t *__restrict__ counts) {
  pdl_wait();
  pdl_launch_dependents();
  const unsigned lane = lane_id();
  if (blockIdx.x == 0) {  // recv_counts[e] from the CSR offsets
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0u;
    __syncthreads();
    const uint32_t A = stats[1];
    for (uint32_t a = threadIdx.x; a < A; a += blockDim.x)
      counts[expert_ids[a]] = start[a + 1] - start[a];
  }
  const int64_t warps_total = (int64_t)gridDim.x * kWarpsPerBlock;
  const int half = K / 2;
  const int nscale = K / 32;
  const int segs = (K + 255) / 256;
  const int groups = (segs + SEG - 1) / SEG;
  const int64_t tasks = (int64_t)N * groups;
  for (int64_t task = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); task < tasks;
       task += warps_total) {
    const int t = (int)(task / groups);
    const int grp = (int)(task % groups);
    const uint16_t *row = x + (int64_t)t * K;
    // issue the group's row loads first (independent of the destinations)
    uint4 v[SEG];
#pragma unroll
    for (int q = 0; q < SEG; ++q) {
      const int k = (grp * SEG + q) * 256 + 8 * (int)lane;
      v[q] = k < K ? ldg_nc_v4(row + k) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int j0 = 0; j0 < top_k; j0 += 32) {
      // destinations of this token's slots (32 per step)
      const int j = j0 + (int)lane;
      uint32_t dest = 0xFFFFFFFFu;
      if (j < top_k) dest = restore[(int64_t)t * top_k + j];
      bool ok = dest != 0xFFFFFFFFu;
      if (ok && (int64_t)dest >= capacity) {
        if (grp == 0) raise_device_error(MOE_DEVERR_RECV_OVERFLOW);
        ok = false;
      }
      const unsigned dmask = __ballot_sync(0xffffffffu, ok);
      if (dmask == 0u) continue;
#pragma unroll
      for (int q = 0; q < SEG; ++q) {
        const int k = (grp * SEG + q) * 256 + 8 * (int)lane;
        if ((grp * SEG + q) * 256 >= K) break;  // warp-uniform
        const bool active = k < K;
        float f[8];
        f[0] = bf16_lo(v[q].x); f[1] = bf16_hi(v[q].x);
        f[2] = bf16_lo(v[q].y); f[3] = bf16_hi(v[q].y);
        f[4] = bf16_lo(v[q].z); f[5] = bf16_hi(v[q].z);
        f[6] = bf16_lo(v[q].w); f[7] = bf16_hi(v[q].w);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int se = mx_shared_exponent(amax);
        const float mult = __uint_as_float((uint32_t)(127 - se) << 23);  // 2^-se, exact
        float qv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) qv[i] = f[i] * mult;
        const uint32_t codes = e2m1x8_from_f32(qv);
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
      // zero padding after the scales (written by the group that holds the last segment)
      if (grp == groups - 1) {
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
}

}  // namespace disp
}  // namespace moe
