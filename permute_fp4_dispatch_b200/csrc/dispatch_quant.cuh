// dispatch_quant.cuh -- steps 3 and 4a from one read of the activations.
//
// MAX "Struct_ep_dispatch_async_mxfp4", execute() (MXFP4 send buffer at one
// GPU) and FlashRT "grouped-moe-gemv" card, quantize_activations_nvfp4_bf16
// (the W4A4 GEMV's NVFP4 activations; the card's grouped_w4a4_gemv_from_bf16
// path quantises and multiplies from the same bf16 rows).  Both steps read
// every token row of x; this kernel reads each row once and writes both
// encodings:
//   * NVFP4 for every row (16-element blocks, E4M3 scale from amax / 6 and
//     the global g, IEEE divisions): exactly the bytes of
//     quant_act_nvfp4_kernel;
//   * MXFP4 (32-element blocks, E8M0 scale) into each routed row of the
//     expert-grouped buffer, plus recv_counts: exactly the bytes of
//     dispatch_mxfp4_kernel.
// Work layout as the dispatch: one warp per (token, group of SEG 256-column
// segments), 8 bf16 per lane, all of the group's loads in flight together.
#pragma once
#include "dispatch_mxfp4.cuh"
#include "quant_nvfp4.cuh"

namespace moe {
namespace dq {

template <int SEG>
__global__ void __launch_bounds__(disp::kWarpsPerBlock * 32)
    dispatch_quant_kernel(const uint16_t *__restrict__ x, int32_t N, int32_t K, int32_t top_k,
                          int32_t E, const uint32_t *__restrict__ restore,
                          const uint32_t *__restrict__ start,
                          const int32_t *__restrict__ expert_ids,
                          const uint32_t *__restrict__ stats, uint8_t *__restrict__ recv,
                          int64_t capacity, int32_t stride, uint32_t *__restrict__ counts,
                          float g, uint8_t *__restrict__ xq, uint8_t *__restrict__ sfa) {
  constexpr int kWPB = disp::kWarpsPerBlock;
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
  const int64_t warps_total = (int64_t)gridDim.x * kWPB;
  const int half = K / 2;
  const int nscale = K / 32;
  const int segs = (K + 255) / 256;
  const int groups = (segs + SEG - 1) / SEG;
  const int64_t tasks = (int64_t)N * groups;
  for (int64_t task = (int64_t)blockIdx.x * kWPB + (threadIdx.x >> 5); task < tasks;
       task += warps_total) {
    const int t = (int)(task / groups);
    const int grp = (int)(task % groups);
    const uint16_t *row = x + (int64_t)t * K;
    uint4 v[SEG];
#pragma unroll
    for (int q = 0; q < SEG; ++q) {
      const int k = (grp * SEG + q) * 256 + 8 * (int)lane;
      v[q] = k < K ? ldg_nc_v4(row + k) : make_uint4(0u, 0u, 0u, 0u);
    }
    // ---- NVFP4 of the row (every row)
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
      uint32_t sb;
      const uint32_t codes = nvq::encode_half_block(f, amax, g, sb);
      if (active) {
        *reinterpret_cast<uint32_t *>(xq + (int64_t)t * (K / 2) + k / 2) = codes;
        if ((lane & 1u) == 0u) sfa[(int64_t)t * (K / 16) + k / 16] = (uint8_t)sb;
      }
    }
    // ---- MXFP4 into every routed row of the token
    for (int j0 = 0; j0 < top_k; j0 += 32) {  // destinations, 32 slots at a time
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
        const int se = disp::mx_shared_exponent(amax);
        const float mult = __uint_as_float((uint32_t)(127 - se) << 23);  // 2^-se, exact
        float qv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) qv[i] = f[i] * mult;
        const uint32_t codes = e2m1x8_from_f32(qv);
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

}  // namespace dq
}  // namespace moe
