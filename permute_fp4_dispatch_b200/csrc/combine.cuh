// combine.cuh -- step 5: router-weighted sum of each token's expert outputs.
//
// MAX "Struct_ep_combine_wait", execute(): the weighted sum of the routed
// expert outputs with the router weights, followed by the optional
// elementwise epilogue (has_epilogue_fusion).  At one GPU all expert outputs
// are already local, so there is no wait phase.
//
// One warp per (token, 256-column segment): each lane owns 8 columns, reads
// the token's top_k expert rows with 128-bit loads (unrouted slots are
// skipped, never read), accumulates in fp32 in slot order and writes 8 bf16
// with one 128-bit store.
#pragma once
#include "common.cuh"

namespace moe {
namespace comb {

constexpr int kWarpsPerBlock = 8;

template <int EPI>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    combine_kernel(const uint16_t *__restrict__ y, const float *__restrict__ rw,
                   const int64_t *__restrict__ ids, int32_t M, int32_t top_k, int32_t H,
                   int32_t E, float alpha, uint16_t *__restrict__ out) {
  const unsigned lane = lane_id();
  const int segs = (H + 255) / 256;
  const int64_t total = (int64_t)M * segs;
  for (int64_t w = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); w < total;
       w += (int64_t)gridDim.x * kWarpsPerBlock) {
    const int64_t t = w / segs;
    const int h = (int)(w % segs) * 256 + 8 * (int)lane;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < top_k; ++j) {
      const int64_t id = ids[t * top_k + j];
      if (id < 0 || id >= E) continue;
      const float wt = rw[t * top_k + j];
      if (h < H) {
        const uint4 v = ldg_nc_v4(y + ((t * top_k + j) * H + h));
        acc[0] = fmaf(wt, bf16_lo(v.x), acc[0]);
        acc[1] = fmaf(wt, bf16_hi(v.x), acc[1]);
        acc[2] = fmaf(wt, bf16_lo(v.y), acc[2]);
        acc[3] = fmaf(wt, bf16_hi(v.y), acc[3]);
        acc[4] = fmaf(wt, bf16_lo(v.z), acc[4]);
        acc[5] = fmaf(wt, bf16_hi(v.z), acc[5]);
        acc[6] = fmaf(wt, bf16_lo(v.w), acc[6]);
        acc[7] = fmaf(wt, bf16_hi(v.w), acc[7]);
      }
    }
    if (EPI == MOE_EPI_SCALE) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fmul_rn(acc[i], alpha);
    }
    if (h < H) {
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4 *>(out + t * H + h) = o;
    }
  }
}

}  // namespace comb
}  // namespace moe
