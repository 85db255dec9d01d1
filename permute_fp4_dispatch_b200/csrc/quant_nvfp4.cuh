// quant_nvfp4.cuh -- NVFP4 encoders (FlashRT "grouped-moe-gemv" card,
// Available functions: quantize_activations_nvfp4_bf16 and
// quantize_weights_nvfp4_bf16).
//
// One 16-element block with fp32 global scale g:
//   s = E4M3(fl32(fl32(amax / 6) / g)),  sdec = fl32(e4m3(s) * g),
//   q_i = E2M1(fl32(x_i / sdec))  (signed zeros when sdec == 0).
// Divisions are IEEE round-to-nearest (__fdiv_rn) and the product is an
// explicit __fmul_rn, so the codes do not depend on contraction choices.
//
// Layout of the work: one warp per row segment of 256 elements, 8 elements
// per lane (one 128-bit load of bf16, two of fp32); a block is two lanes and
// its amax is one xor-shuffle.
#pragma once
#include "common.cuh"

namespace moe {
namespace nvq {

constexpr int kWarpsPerBlock = 8;

// Encode 8 values (half a block) given the block amax; returns 4 code bytes
// and the scale byte.
__device__ __forceinline__ uint32_t encode_half_block(const float (&f)[8], float amax, float g,
                                                      uint32_t &scale_byte) {
  const float s32 = __fdiv_rn(__fdiv_rn(amax, 6.0f), g);
  const uint32_t sc = e4m3_from_f32(s32);
  const float sdec = __fmul_rn(e4m3_to_f32(sc), g);
  scale_byte = sc;
  if (sdec == 0.0f) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) w |= ((__float_as_uint(f[i]) >> 31) << 3) << (4 * i);
    return w;
  }
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], sdec);
  return e2m1x8_from_f32(q);
}

// Activations: x bf16 [M, K] -> xq [M, K/2], sfa [M, K/16]; K % 16 == 0.
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    quant_act_nvfp4_kernel(const uint16_t *__restrict__ x, int32_t M, int32_t K, float g,
                           uint8_t *__restrict__ xq, uint8_t *__restrict__ sfa) {
  pdl_wait();
  pdl_launch_dependents();
  const unsigned lane = lane_id();
  const int64_t segs = (K + 255) / 256;
  const int64_t total = (int64_t)M * segs;
  for (int64_t w = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); w < total;
       w += (int64_t)gridDim.x * kWarpsPerBlock) {
    const int64_t r = w / segs;
    const int k = (int)(w % segs) * 256 + 8 * (int)lane;
    const bool active = k < K;
    float f[8];
    if (active) {
      const uint4 v = ldg_nc_v4(x + r * K + k);
      f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
      f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    uint32_t sb;
    const uint32_t codes = encode_half_block(f, amax, g, sb);
    if (active) {
      *reinterpret_cast<uint32_t *>(xq + r * (K / 2) + k / 2) = codes;
      if ((lane & 1u) == 0u) sfa[r * (K / 16) + k / 16] = (uint8_t)sb;
    }
  }
}

// Weights, pass 1: per-expert amax (as fp32 bits) into amax_bits[E] (zeroed
// by the caller).  Grid: (chunks per expert, E).
__global__ void __launch_bounds__(256)
    weight_amax_kernel(const float *__restrict__ w, int64_t per_expert,
                       unsigned int *__restrict__ amax_bits) {
  __shared__ float red[8];
  const int e = blockIdx.y;
  const float *we = w + (int64_t)e * per_expert;
  float m = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_expert;
       i += (int64_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(we[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane_id() == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    atomicMax(amax_bits + e, __float_as_uint(m));
  }
}

__device__ __forceinline__ float weight_global_from_amax(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// Weights, pass 2: encode rows of expert e with g = amax / (6 * 448).
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    quant_weight_nvfp4_kernel(const float *__restrict__ w, int32_t E, int32_t N, int32_t K,
                              const unsigned int *__restrict__ amax_bits,
                              uint8_t *__restrict__ wq, uint8_t *__restrict__ sfw) {
  const unsigned lane = lane_id();
  const int64_t segs = (K + 255) / 256;
  const int64_t total = (int64_t)E * N * segs;
  for (int64_t t = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); t < total;
       t += (int64_t)gridDim.x * kWarpsPerBlock) {
    const int64_t r = t / segs;
    const int e = (int)(r / N);
    const int k = (int)(t % segs) * 256 + 8 * (int)lane;
    const bool active = k < K;
    const float g = weight_global_from_amax(__uint_as_float(amax_bits[e]));
    float f[8];
    if (active) {
      const float4 a = *reinterpret_cast<const float4 *>(w + r * K + k);
      const float4 b = *reinterpret_cast<const float4 *>(w + r * K + k + 4);
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    uint32_t sb;
    const uint32_t codes = encode_half_block(f, amax, g, sb);
    if (active) {
      *reinterpret_cast<uint32_t *>(wq + r * (K / 2) + k / 2) = codes;
      if ((lane & 1u) == 0u) sfw[r * (K / 16) + k / 16] = (uint8_t)sb;
    }
  }
}

// Weights, pass 3: amax bits -> w_global[e] (in place).
__global__ void weight_global_kernel(float *w_global, int32_t E) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) w_global[e] = weight_global_from_amax(w_global[e]);
}

}  // namespace nvq
}  // namespace moe
