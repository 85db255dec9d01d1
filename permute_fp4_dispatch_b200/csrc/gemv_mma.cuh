// gemv_mma.cuh -- step 4b, decode variant: grouped expert GEMV on an NVFP4
// expert library for passes of up to 32 tokens per expert.
//
// FlashRT "grouped-moe-gemv" card (Available functions:
// grouped_w4a16_gemv_bf16 / grouped_w4a4_gemv_bf16; token-major routing).
//
// At decode batch sizes the weight stream is the roofline and the
// tensor-core work per weight is tiny (8-32 tokens), so this variant keeps
// the tensor cores fed from registers:
//   * Same work partition as the tensor-memory variant: (active expert, pass,
//     16-row block) units in equal contiguous ranges per persistent CTA,
//     rounds of up to 8 blocks of one (expert, pass).
//   * Warp 8 streams the FP4 rows and E4M3 scales of each round, 256 columns
//     per chunk, into a kStages-deep ring with tiled TMA (16-row x 128-byte
//     boxes, 128-byte swizzle, L2 evict-first).  Warps 0-7 each own 16 rows
//     of a round and release a stage with an mbarrier arrive when done: the
//     warps never wait for one another inside a round.
//   * When a CTA starts a new (expert, pass), the 8 warps convert that pass's
//     activation rows once, for the whole K, into an fp16 tile in shared
//     memory laid out in mma fragment order with an XOR swizzle; every round
//     of the pass reuses it.  W4A16: plain bf16 -> fp16 (exact for
//     2^-14 <= |x| <= 65504, MOE_DEVERR_ACT_RANGE beyond); W4A4: E2M1 x E4M3
//     products, exact in fp16.
//   * Each lane dequantises its two rows' codes in registers (hardware
//     E2M1 -> f16x2 converter, times the block's E4M3 scale: exact in fp16)
//     and issues m16n8k16 MMAs (fp32 accumulation, two independent chains per
//     8-token group) with the tokens on the n side.  Within a 64-column span
//     each lane owns 16 contiguous columns (one scale block); A and B use the
//     same column permutation, so the dot product is unchanged.
//   * The round's accumulators are scaled by g_w * g_a, rounded to bf16,
//     transposed through shared memory and written as 16-byte row segments.
#pragma once
#include "gemv_common.cuh"

namespace moe {
namespace gemv {
namespace mma {

constexpr int kCW = 8;                  // compute warps (16 rows each)
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kKC = 256;                // columns per chunk
constexpr int kMaxTS = 32;              // tokens per pass at most (4 groups of 8)
constexpr int kNG = kMaxTS / 8;
constexpr int kStages = 4;
constexpr int kWStride = kKC / 2;
constexpr int kSFStride = kKC / 16;
constexpr int kBoxW = 16 * kWStride;
constexpr int kBoxSF = 16 * kSFStride;
constexpr int kStageW = 128 * kWStride;
constexpr int kStageBytes = kStageW + 128 * kSFStride;
constexpr int kGroupChunkBytes = 4 * 2 * 32 * 16;  // one 8-token group x one chunk (4 KB)
constexpr int kActBytes = 128 * 1024;              // fp16 activation tile of a pass
constexpr int kStagingBytes = kCW * kMaxTS * 16 * 2;

static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
constexpr size_t kOffAct = (size_t)kStages * kStageBytes;
constexpr size_t kOffStaging = kOffAct + kActBytes;
constexpr size_t kOffPrefix = kOffStaging + kStagingBytes;
constexpr size_t kOffStart = kOffPrefix + (kMaxExperts + 4) * 4;
constexpr size_t kOffEid = kOffStart + (kMaxExperts + 4) * 4;
constexpr size_t kOffPair = kOffEid + (kMaxExperts + 4) * 4;
constexpr size_t kOffBar = kOffPair + kMaxTS * 4;
constexpr size_t kOffMisc = kOffBar + 2 * kStages * 8;
constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;

// Tokens per pass for a hidden size K: as many 8-token groups (up to 4) as
// the activation tile holds for the whole K; 0 when not even one fits.
__host__ __device__ constexpr int tokens_per_pass(int K) {
  const int nchunks = (K + kKC - 1) / kKC;
  const int groups = kActBytes / (nchunks * kGroupChunkBytes);
  return 8 * (groups < kNG ? groups : kNG);
}

// fp16 activation tile index (16-byte units): chunk c, group G (of ng), span s,
// half h, lane (g, t).
__device__ __forceinline__ int act_index(int c, int ng, int G, int s, int h, int g, int t) {
  return ((((c * ng + G) * 4 + s) * 2 + h) * 32) + ((g * 4 + t) ^ (2 * s + h));
}

// One chunk of one warp: dequantise its two rows' 256 codes (lane (g, t):
// rows g and g + 8, columns 64t..64t+63 of the chunk), multiply with the NG
// token groups of the activation tile, accumulate into acc0 / acc1.
template <int NG>
__device__ __forceinline__ void mma_chunk(const uint8_t *sw, const uint8_t *ssf, const uint4 *act,
                                          int c, int wrow, int g, int t, bool lane_k,
                                          float (&acc0)[kNG][4], float (&acc1)[kNG][4]) {
  uint4 wa[2], wb[2];
  uint32_t sfa_w = 0, sfb_w = 0;
  if (lane_k) {
    // 128-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ (r & 7); r & 7 == g
    const uint4 *pa = reinterpret_cast<const uint4 *>(sw + wrow * kWStride);
    const uint4 *pb = reinterpret_cast<const uint4 *>(sw + (wrow + 8) * kWStride);
    wa[0] = pa[(2 * t) ^ g];
    wa[1] = pa[(2 * t + 1) ^ g];
    wb[0] = pb[(2 * t) ^ g];
    wb[1] = pb[(2 * t + 1) ^ g];
    sfa_w = *reinterpret_cast<const uint32_t *>(ssf + wrow * kSFStride + 4 * t);
    sfb_w = *reinterpret_cast<const uint32_t *>(ssf + (wrow + 8) * kSFStride + 4 * t);
  } else {
    wa[0] = wa[1] = wb[0] = wb[1] = make_uint4(0u, 0u, 0u, 0u);
  }
  const uint32_t sa01 = e4m3x2_to_f16x2(sfa_w & 0xFFFFu), sa23 = e4m3x2_to_f16x2(sfa_w >> 16);
  const uint32_t sb01 = e4m3x2_to_f16x2(sfb_w & 0xFFFFu), sb23 = e4m3x2_to_f16x2(sfb_w >> 16);
  const uint4 *tile = act + c * NG * 256;
#pragma unroll
  for (int sp = 0; sp < 4; ++sp) {
    const uint32_t sca = (sp & 1) ? bcast_hi(sp < 2 ? sa01 : sa23) : bcast_lo(sp < 2 ? sa01 : sa23);
    const uint32_t scb = (sp & 1) ? bcast_hi(sp < 2 ? sb01 : sb23) : bcast_lo(sp < 2 ? sb01 : sb23);
    const uint4 &va = wa[sp >> 1];
    const uint4 &vb = wb[sp >> 1];
    const uint32_t ca0 = (sp & 1) ? va.z : va.x, ca1 = (sp & 1) ? va.w : va.y;
    const uint32_t cb0 = (sp & 1) ? vb.z : vb.x, cb1 = (sp & 1) ? vb.w : vb.y;
    uint32_t A0[4], A1[4], B0[4], B1[4];
    e2m1x8_to_f16x2(ca0, A0[0], A0[1], A0[2], A0[3]);  // row g, MMAs 0, 1
    e2m1x8_to_f16x2(ca1, A1[0], A1[1], A1[2], A1[3]);  // row g, MMAs 2, 3
    e2m1x8_to_f16x2(cb0, B0[0], B0[1], B0[2], B0[3]);  // row g + 8
    e2m1x8_to_f16x2(cb1, B1[0], B1[1], B1[2], B1[3]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      A0[q] = hmul2(A0[q], sca);
      A1[q] = hmul2(A1[q], sca);
      B0[q] = hmul2(B0[q], scb);
      B1[q] = hmul2(B1[q], scb);
    }
#pragma unroll
    for (int G = 0; G < NG; ++G) {
      const uint4 bh0 = tile[act_index(0, NG, G, sp, 0, g, t)];
      const uint4 bh1 = tile[act_index(0, NG, G, sp, 1, g, t)];
      mma_16816_f16(acc0[G], A0[0], B0[0], A0[1], B0[1], bh0.x, bh0.y);
      mma_16816_f16(acc1[G], A1[0], B1[0], A1[1], B1[1], bh1.x, bh1.y);
      mma_16816_f16(acc0[G], A0[2], B0[2], A0[3], B0[3], bh0.z, bh0.w);
      mma_16816_f16(acc1[G], A1[2], B1[2], A1[3], B1[3], bh1.z, bh1.w);
    }
  }
}

template <int MODE, bool SF_TMA>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemv_mma_kernel(const Params p, const int ts, const __grid_constant__ CUtensorMap tmap_w,
                            const __grid_constant__ CUtensorMap tmap_sf) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint4 *act = reinterpret_cast<uint4 *>(smem + kOffAct);
  uint16_t *staging = reinterpret_cast<uint16_t *>(smem + kOffStaging);
  uint32_t *prefix = reinterpret_cast<uint32_t *>(smem + kOffPrefix);
  uint32_t *s_start = reinterpret_cast<uint32_t *>(smem + kOffStart);
  int32_t *s_eid = reinterpret_cast<int32_t *>(smem + kOffEid);
  uint32_t *s_pair = reinterpret_cast<uint32_t *>(smem + kOffPair);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint64_t *empty = full + kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc);

  const int warp = threadIdx.x >> 5;
  const int lane = (int)lane_id();
  const int N = p.N, K = p.K;
  const int RB = (N + 15) / 16;
  const uint32_t A = p.stats[1];

  for (uint32_t i = threadIdx.x; i <= A; i += blockDim.x) {
    s_start[i] = p.start[i];
    if (i < A) s_eid[i] = p.eids[i];
  }
  __syncthreads();
  if (warp == 0) build_prefix(prefix, s_start, A, (uint32_t)ts, RB, lane);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], SF_TMA ? 1u : 33u);
      mbar_init(&empty[s], (uint32_t)kCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t U = prefix[A];
  const uint32_t u_begin = (uint32_t)(((uint64_t)U * blockIdx.x) / gridDim.x);
  const uint32_t u_end = (uint32_t)(((uint64_t)U * (blockIdx.x + 1)) / gridDim.x);
  if (u_begin >= u_end) return;
  const int nchunks = (K + kKC - 1) / kKC;
  const int64_t sf_row_bytes = K / 16;
  const Meta meta{prefix, s_start, s_eid, N};

  auto wait = [&](uint64_t *bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait_bounded(bar, parity, kWaitLimitNs)) *abort_flag = 1;
  };

  if (warp == kCW) {
    // ================================================================ TMA producer
    RoundIter iter{u_begin, u_end, 0, (uint32_t)ts};
    Round r;
    uint32_t it = 0;
    const uint64_t policy = l2_evict_first_policy();
    if (lane == 0) {
      prefetch_tmap(&tmap_w);
      if (SF_TMA) prefetch_tmap(&tmap_sf);
    }
    while (iter.next(meta, RB, r)) {
      for (int c = 0; c < nchunks; ++c, ++it) {
        const int s = (int)(it % kStages);
        wait(&empty[s], ((it / kStages) & 1u) ^ 1u);
        if (*abort_flag) continue;
        const int k0 = c * kKC;
        uint8_t *sw = smem + (size_t)s * kStageBytes;
        uint8_t *ssf = sw + kStageW;
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], (uint32_t)r.nblk * (kBoxW + (SF_TMA ? kBoxSF : 0)));
        __syncwarp();
        if (lane < r.nblk) {
          tma_load_3d(sw + lane * kBoxW, &tmap_w, k0 / 2, r.n0 + 16 * lane, r.e, &full[s], policy);
          if (SF_TMA)
            tma_load_3d(ssf + lane * kBoxSF, &tmap_sf, k0 / 16, r.n0 + 16 * lane, r.e, &full[s],
                        policy);
        }
        if (!SF_TMA) {
          const uint32_t sb = (uint32_t)min(kKC, K - k0) / 16;
          const uint8_t *sbase = p.sfw + ((int64_t)r.e * N + r.n0) * sf_row_bytes + k0 / 16;
          for (int row = lane; row < r.nrows; row += 32)
            for (uint32_t q = 0; q < sb; q += 4)
              cp_async4(ssf + row * kSFStride + q, sbase + row * sf_row_bytes + q);
          cp_async_mbar_arrive_noinc(&full[s]);
        }
      }
    }
    return;
  }

  // ================================================================== compute warps
  const int cw = warp;
  const int g = lane >> 2, t = lane & 3;
  const int wrow = cw * 16 + g;  // round-local row of a0 (a1: wrow + 8)
  RoundIter iter{u_begin, u_end, 0, (uint32_t)ts};
  Round r;
  uint32_t it = 0;
  uint32_t pass_key = 0xFFFFFFFFu;
  int ng = 0;
  const int kpad = nchunks * kKC;

  while (iter.next(meta, RB, r)) {
    if (r.tok0 != pass_key) {
      // ---- new (expert, pass): build its fp16 activation tile for the whole K
      named_bar_sync(1, kCW * 32);  // every warp is done with the previous tile
      ng = (r.ntok + 7) / 8;
      for (int i = threadIdx.x; i < r.ntok; i += kCW * 32) s_pair[i] = p.order[r.tok0 + i];
      named_bar_sync(1, kCW * 32);
      unsigned range_bad = 0;
      const int per_tok = kpad / 8;  // 8-column slices per token
      const int ntask = r.ntok * per_tok;
      // each thread converts up to kBatch slices per step with all loads issued first
      constexpr int kBatch = 8;
      for (int base = 0; base < ntask; base += kCW * 32 * kBatch) {
        uint4 v[kBatch];
        uint32_t sv[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int task = base + b * kCW * 32 + threadIdx.x;
          v[b] = make_uint4(0u, 0u, 0u, 0u);
          sv[b] = 0u;
          if (task < ntask) {
            const int tau = task / per_tok;
            const int k = (task % per_tok) * 8;
            const int64_t m = (int64_t)(s_pair[tau] / (uint32_t)p.top_k);
            if (k < K) {
              if (MODE == MOE_W4A16) {
                v[b] = ldg_nc_v4(static_cast<const uint16_t *>(p.act) + m * K + k);
              } else {
                const uint8_t *qp = static_cast<const uint8_t *>(p.act) + m * (K / 2);
                v[b].x = __ldg(reinterpret_cast<const uint32_t *>(qp + k / 2));
                sv[b] = p.sfa[m * (K / 16) + k / 16];
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int task = base + b * kCW * 32 + threadIdx.x;
          if (task >= ntask) continue;
          const int tau = task / per_tok;
          const int k = (task % per_tok) * 8;
          uint4 hv = make_uint4(0u, 0u, 0u, 0u);
          if (k < K) {
            if (MODE == MOE_W4A16) {
              float f[8];
              f[0] = bf16_lo(v[b].x); f[1] = bf16_hi(v[b].x);
              f[2] = bf16_lo(v[b].y); f[3] = bf16_hi(v[b].y);
              f[4] = bf16_lo(v[b].z); f[5] = bf16_hi(v[b].z);
              f[6] = bf16_lo(v[b].w); f[7] = bf16_hi(v[b].w);
#pragma unroll
              for (int e = 0; e < 8; ++e) range_bad |= (fabsf(f[e]) > 65504.0f) ? 1u : 0u;
              hv.x = pack_f16x2(f[0], f[1]);
              hv.y = pack_f16x2(f[2], f[3]);
              hv.z = pack_f16x2(f[4], f[5]);
              hv.w = pack_f16x2(f[6], f[7]);
            } else {
              const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(sv[b]));
              uint32_t q0, q1, q2, q3;
              e2m1x8_to_f16x2(v[b].x, q0, q1, q2, q3);
              hv.x = hmul2(q0, sc);
              hv.y = hmul2(q1, sc);
              hv.z = hmul2(q2, sc);
              hv.w = hmul2(q3, sc);
            }
          }
          // fragment slot of columns [k, k + 8) of token tau
          const int c = k / kKC, kk = k % kKC, L = kk / 8;
          act[act_index(c, ng, tau / 8, (L & 7) >> 1, L & 1, tau & 7, L >> 3)] = hv;
        }
      }
      if (MODE == MOE_W4A16 && range_bad) raise_device_error(MOE_DEVERR_ACT_RANGE);
      named_bar_sync(1, kCW * 32);
      pass_key = r.tok0;
    }

    const bool has_rows = cw < r.nblk;
    float acc0[kNG][4], acc1[kNG][4];
#pragma unroll
    for (int G = 0; G < kNG; ++G)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc0[G][i] = acc1[G][i] = 0.f;

    for (int c = 0; c < nchunks; ++c, ++it) {
      const int s = (int)(it % kStages);
      wait(&full[s], (it / kStages) & 1u);
      if (has_rows && !*abort_flag) {
        const uint8_t *sw = smem + (size_t)s * kStageBytes;
        const uint8_t *ssf = sw + kStageW;
        const bool lane_k = 64 * t < min(kKC, K - c * kKC);
        switch (ng) {
          case 1: mma_chunk<1>(sw, ssf, act, c, wrow, g, t, lane_k, acc0, acc1); break;
          case 2: mma_chunk<2>(sw, ssf, act, c, wrow, g, t, lane_k, acc0, acc1); break;
          case 3: mma_chunk<3>(sw, ssf, act, c, wrow, g, t, lane_k, acc0, acc1); break;
          default: mma_chunk<4>(sw, ssf, act, c, wrow, g, t, lane_k, acc0, acc1); break;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- round epilogue: scale, round to bf16, transpose, 16-byte stores
    if (has_rows && !*abort_flag) {
      const float gw = p.w_global ? p.w_global[r.e] : 1.0f;
      const float f = __fmul_rn(gw, p.g_a);
      uint16_t *st = staging + cw * (kMaxTS * 16);
#pragma unroll
      for (int G = 0; G < kNG; ++G) {
        if (G < ng) {
          const int c0 = G * 8 + 2 * t;
          const uint32_t lo = pack_bf16x2((acc0[G][0] + acc1[G][0]) * f, (acc0[G][1] + acc1[G][1]) * f);
          const uint32_t hi = pack_bf16x2((acc0[G][2] + acc1[G][2]) * f, (acc0[G][3] + acc1[G][3]) * f);
          st[c0 * 16 + g] = (uint16_t)(lo & 0xFFFFu);
          st[(c0 + 1) * 16 + g] = (uint16_t)(lo >> 16);
          st[c0 * 16 + g + 8] = (uint16_t)(hi & 0xFFFFu);
          st[(c0 + 1) * 16 + g + 8] = (uint16_t)(hi >> 16);
        }
      }
      __syncwarp();
      const int nw = r.n0 + cw * 16;
      for (int task = lane; task < r.ntok * 2; task += 32) {
        const int col = task >> 1, half = task & 1;
        const int n = nw + half * 8;
        if (n < N) {
          const uint32_t pair = s_pair[col];
          *reinterpret_cast<uint4 *>(p.out + (int64_t)pair * N + n) =
              *reinterpret_cast<const uint4 *>(st + col * 16 + half * 8);
        }
      }
      __syncwarp();
    }
  }
}

}  // namespace mma
}  // namespace gemv
}  // namespace moe
