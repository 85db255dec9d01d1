// combine.cuh -- step 5: router-weighted sum of each token's expert outputs.
//
// MAX "Struct_ep_combine_wait", execute(): the weighted sum of the routed
// expert outputs with the router weights, followed by the optional
// elementwise epilogue (has_epilogue_fusion).  At one GPU all expert outputs
// are already local, so there is no wait phase.
//
// One warp per (token, 256-column segment): each lane owns 8 columns.  The
// token's slot ids and weights are read first (one slot per lane); then only
// the routed slots' rows are loaded (128-bit loads, up to eight in flight),
// accumulated in fp32 in slot order and written as 8 bf16 with one 128-bit
// store.  Rows of unrouted slots -- which the GEMV never wrote -- are never
// read, so padding rows of a CUDA-graph bucket cost their metadata only.
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
  pdl_wait();
  pdl_launch_dependents();
  const unsigned lane = lane_id();
  const int segs = (H + 255) / 256;
  const int64_t total = (int64_t)M * segs;
  for (int64_t w = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); w < total;
       w += (int64_t)gridDim.x * kWarpsPerBlock) {
    const int64_t t = w / segs;
    const int h = (int)(w % segs) * 256 + 8 * (int)lane;
    const bool col_ok = h < H;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j0 = 0; j0 < top_k; j0 += 32) {
      const int jl = j0 + (int)lane;
      bool ok = false;
      float wl = 0.f;
      if (jl < top_k) {
        const int64_t id = ids[t * top_k + jl];
        ok = id >= 0 && id < E;
        wl = rw[t * top_k + jl];
      }
      unsigned m = __ballot_sync(0xffffffffu, ok);
      while (m) {
        // a batch of up to 8 routed slots: issue all loads, then accumulate in order
        uint4 v[8];
        int js[8];
        int nb = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (m) {
            js[b] = __ffs(m) - 1;
            m &= m - 1;
            nb = b + 1;
            v[b] = col_ok ? ldg_nc_v4(y + ((t * top_k + j0 + js[b]) * H + h))
                          : make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (b < nb) {
            const float wt = __shfl_sync(0xffffffffu, wl, js[b]);
            acc[0] = fmaf(wt, bf16_lo(v[b].x), acc[0]);
            acc[1] = fmaf(wt, bf16_hi(v[b].x), acc[1]);
            acc[2] = fmaf(wt, bf16_lo(v[b].y), acc[2]);
            acc[3] = fmaf(wt, bf16_hi(v[b].y), acc[3]);
            acc[4] = fmaf(wt, bf16_lo(v[b].z), acc[4]);
            acc[5] = fmaf(wt, bf16_hi(v[b].z), acc[5]);
            acc[6] = fmaf(wt, bf16_lo(v[b].w), acc[6]);
            acc[7] = fmaf(wt, bf16_hi(v[b].w), acc[7]);
          }
        }
      }
    }
    if (EPI == MOE_EPI_SCALE) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fmul_rn(acc[i], alpha);
    }
    if (col_ok) {
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
