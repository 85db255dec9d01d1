// gemv_nvfp4.cuh -- step 4b: grouped expert GEMV on an NVFP4 expert library.
//
// FlashRT "grouped-moe-gemv" card (Available functions:
// grouped_w4a16_gemv_bf16 / grouped_w4a4_gemv_bf16; W4A4 routing is
// token-major: activations [M, K], library [E, N, K/2], output
// [M, top_k, N]).  For each routed pair p with expert e:
//     out[p, n] = bf16( g_w[e] * g_a * sum_k a(p/top_k, k) * w(e, n, k) ).
//
// Design (decode-first, HBM-bound on the weight stream):
//   * Work is expert-major: the pairs of an active expert (CSR from
//     moe_create_indices) are processed in passes of up to kTS = 32 tokens,
//     and each pass sweeps the expert's N rows in 16-row blocks.  The flat
//     list of (expert, pass, row block) units is split into equal contiguous
//     ranges, one per persistent CTA (grid = SM count), so the weight bytes
//     per CTA are balanced to one 16-row block.
//   * A CTA = 1 producer warp + 8 consumer warps.  Consecutive blocks of one
//     (expert, pass) form a round of up to 128 rows.  The producer streams
//     each round's FP4 rows and E4M3 scales in chunks of kKC = 256 columns
//     into a 4-stage shared-memory ring with bulk copies on the TMA engine
//     (cp.async.bulk, mbarrier transaction counts); scale rows that are not
//     16-byte aligned use 4-byte cp.async instead.
//   * Consumers dequantise in registers, exactly: E2M1 -> f16x2 with the
//     hardware converter, times the block's E4M3 scale (a product of at most
//     6 significant bits, exact in fp16), and feed warp-level tensor-core MMAs
//     (m16n8k16, fp32 accumulation) with the tokens on the n = 8 side.
//     Within a 64-column span each lane owns 16 contiguous columns (one scale
//     block); A and B use the same column permutation, so the dot product is
//     unchanged.
//   * Activations are staged per chunk by the consumers themselves into a
//     double-buffered fp16 tile laid out in fragment order with an XOR
//     swizzle (conflict-free 128-bit loads and stores).  W4A16 rows are scaled
//     by a per-(token, chunk) power of two so the chunk maximum lies in
//     [2^14, 2^15) before the fp16 conversion (exact for every value within
//     2^29 of the chunk maximum); the power of two is undone in fp32 after
//     the chunk.  W4A4 activations are dequantised exactly like the weights.
//   * The round's accumulators are scaled by g_w * g_a, rounded to bf16,
//     transposed through shared memory and written as 16-byte row segments.
#pragma once
#include "common.cuh"

namespace moe {
namespace gemv {

constexpr int kCW = 8;                  // consumer warps
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kRows = 16 * kCW;         // rows per round
constexpr int kKC = 256;                // columns (codes) per chunk
constexpr int kTS = 32;                 // tokens per pass
constexpr int kNG = kTS / 8;            // n8 groups per pass
constexpr int kStages = 4;
constexpr int kWStride = kKC / 2 + 16;  // bytes per weight row in a stage (padded)
constexpr int kSFStride = kKC / 16;     // bytes per scale row in a stage
constexpr int kStageW = kRows * kWStride;
constexpr int kStageBytes = kStageW + kRows * kSFStride;
constexpr int kActBytes = kTS * kKC * 2;
constexpr int kStagingBytes = kCW * kTS * 16 * 2;
constexpr int kMaxExperts = 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

constexpr size_t kOffAct = (size_t)kStages * kStageBytes;
constexpr size_t kOffCS = kOffAct + 2 * kActBytes;
constexpr size_t kOffStaging = kOffCS + 2 * kTS * 4;
constexpr size_t kOffPrefix = kOffStaging + kStagingBytes;
constexpr size_t kOffBar = kOffPrefix + (kMaxExperts + 4) * 4;
constexpr size_t kSmemBytes = kOffBar + 2 * kStages * 8 + 16;

struct Params {
  const void *act;          // W4A16: bf16 [M, K]; W4A4: u8 [M, K/2]
  const uint8_t *sfa;       // W4A4: [M, K/16]
  float g_a;
  int32_t top_k;
  const uint8_t *w;         // [E, N, K/2]
  const uint8_t *sfw;       // [E, N, K/16]
  const float *w_global;    // [E] or null
  int32_t N, K;
  const uint32_t *order;
  const uint32_t *start;
  const int32_t *eids;
  const uint32_t *stats;
  uint16_t *out;            // bf16 [M, top_k, N]
};

struct Round {
  int e;
  uint32_t tok0;
  int ntok;
  int n0;
  int nrows;
  int nblk;
};

// Next round of this CTA's unit range; identical in every warp.
__device__ __forceinline__ bool next_round(uint32_t &u, uint32_t u_end, int &a,
                                           const uint32_t *prefix, const Params &p, int RB,
                                           Round &r) {
  if (u >= u_end) return false;
  while (u >= prefix[a + 1]) ++a;
  const uint32_t v = u - prefix[a];
  const uint32_t pass = v / (uint32_t)RB;
  const uint32_t rb = v % (uint32_t)RB;
  uint32_t nblk = (uint32_t)RB - rb;
  if (nblk > (uint32_t)kCW) nblk = kCW;
  if (nblk > u_end - u) nblk = u_end - u;
  const uint32_t s0 = p.start[a];
  const uint32_t c = p.start[a + 1] - s0;
  r.e = p.eids[a];
  r.tok0 = s0 + pass * kTS;
  r.ntok = (int)min((uint32_t)kTS, c - pass * kTS);
  r.n0 = (int)rb * 16;
  r.nrows = min((int)nblk * 16, p.N - r.n0);
  r.nblk = (int)nblk;
  u += nblk;
  return true;
}

__device__ __forceinline__ uint32_t bcast_lo(uint32_t h) { return __byte_perm(h, h, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t h) { return __byte_perm(h, h, 0x3232); }

// fp16 tile index (in 16-byte units) of (group G, span s, half h, lane (g,t)).
__device__ __forceinline__ int act_chunk16(int G, int s, int h, int g, int t) {
  return ((G * 4 + s) * 2 + h) * 32 + ((g * 4 + t) ^ (2 * s + h));
}

template <int MODE, bool SF_BULK>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemv_kernel(const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *act_tile = smem + kOffAct;
  float *cs_tile = reinterpret_cast<float *>(smem + kOffCS);
  uint16_t *staging = reinterpret_cast<uint16_t *>(smem + kOffStaging);
  uint32_t *prefix = reinterpret_cast<uint32_t *>(smem + kOffPrefix);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint64_t *empty = full + kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = (int)lane_id();
  const int N = p.N, K = p.K;
  const int RB = (N + 15) / 16;
  const uint32_t A = p.stats[1];

  // units per active expert = passes * row blocks; prefix over experts
  if (warp == 0) {
    uint32_t run = 0;
    for (uint32_t a0 = 0; a0 < A; a0 += 32) {
      const uint32_t a = a0 + lane;
      uint32_t units = 0;
      if (a < A) {
        const uint32_t c = p.start[a + 1] - p.start[a];
        units = (c + kTS - 1) / kTS * (uint32_t)RB;
      }
      uint32_t x = units;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (a < A) prefix[a + 1] = run + x;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) prefix[0] = 0;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], SF_BULK ? 1u : 33u);
      mbar_init(&empty[s], (uint32_t)kCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t U = prefix[A];
  const uint32_t u_begin = (uint32_t)(((uint64_t)U * blockIdx.x) / gridDim.x);
  const uint32_t u_end = (uint32_t)(((uint64_t)U * (blockIdx.x + 1)) / gridDim.x);
  const int nchunks = (K + kKC - 1) / kKC;
  const int64_t row_bytes = K / 2, sf_row_bytes = K / 16;

  if (warp == kCW) {
    // ---------------------------------------------------------------- producer
    uint32_t u = u_begin, it = 0;
    int a = 0;
    Round r;
    while (next_round(u, u_end, a, prefix, p, RB, r)) {
      const uint8_t *wbase = p.w + ((int64_t)r.e * N + r.n0) * row_bytes;
      const uint8_t *sbase = p.sfw + ((int64_t)r.e * N + r.n0) * sf_row_bytes;
      for (int c = 0; c < nchunks; ++c, ++it) {
        const int s = (int)(it % kStages);
        const uint32_t ph = (it / kStages) & 1u;
        if (!*abort_flag && !mbar_wait_bounded(&empty[s], ph ^ 1u, kWaitLimitNs)) *abort_flag = 1;
        if (*abort_flag) continue;
        const int k0 = c * kKC;
        const int kcb = min(kKC, K - k0);
        const uint32_t wb = (uint32_t)kcb / 2, sb = (uint32_t)kcb / 16;
        uint8_t *sw = smem + (size_t)s * kStageBytes;
        uint8_t *ssf = sw + kStageW;
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], (uint32_t)r.nrows * (wb + (SF_BULK ? sb : 0u)));
        for (int row = lane; row < r.nrows; row += 32) {
          bulk_g2s(sw + row * kWStride, wbase + row * row_bytes + k0 / 2, wb, &full[s]);
          const uint8_t *src = sbase + row * sf_row_bytes + k0 / 16;
          if (SF_BULK) {
            bulk_g2s(ssf + row * kSFStride, src, sb, &full[s]);
          } else {
            for (uint32_t q = 0; q < sb; q += 4) cp_async4(ssf + row * kSFStride + q, src + q);
          }
        }
        if (!SF_BULK) cp_async_mbar_arrive_noinc(&full[s]);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int cw = warp;
  const int g = lane >> 2, t = lane & 3;
  // converter lane mapping: lane L owns chunk columns [8L, 8L+8)
  const int cv_t = lane >> 3, cv_s = (lane & 7) >> 1, cv_h = lane & 1;
  uint32_t u = u_begin, it = 0;
  int a = 0;
  Round r;
  while (next_round(u, u_end, a, prefix, p, RB, r)) {
    const int ngroups = (r.ntok + 7) / 8;
    // rows of the tokens this warp converts: tau = cw + 8 i
    int64_t arow[kNG];
    bool tv[kNG];
#pragma unroll
    for (int i = 0; i < kNG; ++i) {
      const int tau = cw + 8 * i;
      tv[i] = tau < r.ntok;
      arow[i] = tv[i] ? (int64_t)(p.order[r.tok0 + tau] / (uint32_t)p.top_k) : 0;
    }
    // prefetch chunk 0 of the activations
    uint4 raw[kNG];
    auto load_act = [&](int c) {
      const int k0 = c * kKC;
      const int kcb = min(kKC, K - k0);
      const bool kv = 8 * lane < kcb;
#pragma unroll
      for (int i = 0; i < kNG; ++i) {
        raw[i] = make_uint4(0u, 0u, 0u, 0u);
        if (tv[i] && kv) {
          if (MODE == MOE_W4A16) {
            raw[i] = ldg_nc_v4(static_cast<const uint16_t *>(p.act) + arow[i] * K + k0 + 8 * lane);
          } else {
            const uint8_t *q = static_cast<const uint8_t *>(p.act) + arow[i] * (K / 2);
            raw[i].x = __ldg(reinterpret_cast<const uint32_t *>(q + (k0 + 8 * lane) / 2));
            raw[i].y = p.sfa[arow[i] * (K / 16) + (k0 + 8 * lane) / 16];
          }
        }
      }
    };
    load_act(0);

    float acc[kNG][4];
#pragma unroll
    for (int G = 0; G < kNG; ++G)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[G][i] = 0.f;

    const bool has_rows = cw < r.nblk;
    const int wrow = cw * 16 + g;  // row of a0 within the round (row + 8 for a1)

    for (int c = 0; c < nchunks; ++c, ++it) {
      const int buf = (int)(it & 1u);
      const int k0 = c * kKC;
      const int kcb = min(kKC, K - k0);
      uint4 *tile = reinterpret_cast<uint4 *>(act_tile + buf * kActBytes);
      float *cs = cs_tile + buf * kTS;
      // ---- convert this chunk's activations into the fp16 fragment tile
#pragma unroll
      for (int i = 0; i < kNG; ++i) {
        if (!tv[i]) continue;  // warp-uniform
        uint4 h;
        float back = 1.0f;
        if (MODE == MOE_W4A16) {
          float f[8];
          f[0] = bf16_lo(raw[i].x); f[1] = bf16_hi(raw[i].x);
          f[2] = bf16_lo(raw[i].y); f[3] = bf16_hi(raw[i].y);
          f[4] = bf16_lo(raw[i].z); f[5] = bf16_hi(raw[i].z);
          f[6] = bf16_lo(raw[i].w); f[7] = bf16_hi(raw[i].w);
          float m = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q) m = fmaxf(m, fabsf(f[q]));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          float inv = 1.0f;
          if (m > 0.f) {
            const int ex = (int)((__float_as_uint(m) >> 23) & 0xFFu);
            int sig = ex - 141;  // floor(log2 m) - 14 for normal m
            sig = sig < -126 ? -126 : sig;
            inv = __uint_as_float((uint32_t)(127 - sig) << 23);
            back = __uint_as_float((uint32_t)(127 + sig) << 23);
          }
          h.x = pack_f16x2(f[0] * inv, f[1] * inv);
          h.y = pack_f16x2(f[2] * inv, f[3] * inv);
          h.z = pack_f16x2(f[4] * inv, f[5] * inv);
          h.w = pack_f16x2(f[6] * inv, f[7] * inv);
        } else {
          uint32_t q0, q1, q2, q3;
          e2m1x8_to_f16x2(raw[i].x, q0, q1, q2, q3);
          const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(raw[i].y));
          h.x = hmul2(q0, sc);
          h.y = hmul2(q1, sc);
          h.z = hmul2(q2, sc);
          h.w = hmul2(q3, sc);
        }
        tile[act_chunk16(i, cv_s, cv_h, cw, cv_t)] = h;
        if (lane == 0) cs[cw + 8 * i] = back;
      }
      named_bar_sync(1, kCW * 32);
      if (c + 1 < nchunks) load_act(c + 1);

      const int s = (int)(it % kStages);
      const uint32_t ph = (it / kStages) & 1u;
      if (!*abort_flag && !mbar_wait_bounded(&full[s], ph, kWaitLimitNs)) *abort_flag = 1;

      if (!*abort_flag && has_rows) {
        const uint8_t *sw = smem + (size_t)s * kStageBytes;
        const uint8_t *ssf = sw + kStageW;
        const bool lane_k = 64 * t < kcb;
        uint4 wa[2], wb[2];
        uint32_t sfa_w = 0, sfb_w = 0;
        if (lane_k) {
          const uint4 *pa = reinterpret_cast<const uint4 *>(sw + wrow * kWStride + 32 * t);
          const uint4 *pb = reinterpret_cast<const uint4 *>(sw + (wrow + 8) * kWStride + 32 * t);
          wa[0] = pa[0]; wa[1] = pa[1];
          wb[0] = pb[0]; wb[1] = pb[1];
          sfa_w = *reinterpret_cast<const uint32_t *>(ssf + wrow * kSFStride + 4 * t);
          sfb_w = *reinterpret_cast<const uint32_t *>(ssf + (wrow + 8) * kSFStride + 4 * t);
        } else {
          wa[0] = wa[1] = wb[0] = wb[1] = make_uint4(0u, 0u, 0u, 0u);
        }
        const uint32_t sa01 = e4m3x2_to_f16x2(sfa_w & 0xFFFFu), sa23 = e4m3x2_to_f16x2(sfa_w >> 16);
        const uint32_t sb01 = e4m3x2_to_f16x2(sfb_w & 0xFFFFu), sb23 = e4m3x2_to_f16x2(sfb_w >> 16);
        float d[kNG][4];
#pragma unroll
        for (int G = 0; G < kNG; ++G)
#pragma unroll
          for (int i = 0; i < 4; ++i) d[G][i] = 0.f;
#pragma unroll
        for (int sp = 0; sp < 4; ++sp) {
          const uint32_t sca = (sp & 1) ? bcast_hi(sp < 2 ? sa01 : sa23) : bcast_lo(sp < 2 ? sa01 : sa23);
          const uint32_t scb = (sp & 1) ? bcast_hi(sp < 2 ? sb01 : sb23) : bcast_lo(sp < 2 ? sb01 : sb23);
          const uint4 &va = wa[sp >> 1];
          const uint4 &vb = wb[sp >> 1];
          const uint32_t ca0 = (sp & 1) ? va.z : va.x, ca1 = (sp & 1) ? va.w : va.y;
          const uint32_t cb0 = (sp & 1) ? vb.z : vb.x, cb1 = (sp & 1) ? vb.w : vb.y;
          uint32_t A0[4], A1[4], B0[4], B1[4];
          e2m1x8_to_f16x2(ca0, A0[0], A0[1], A0[2], A0[3]);  // row g, MMAs 0,1
          e2m1x8_to_f16x2(ca1, A1[0], A1[1], A1[2], A1[3]);  // row g, MMAs 2,3
          e2m1x8_to_f16x2(cb0, B0[0], B0[1], B0[2], B0[3]);  // row g+8
          e2m1x8_to_f16x2(cb1, B1[0], B1[1], B1[2], B1[3]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            A0[q] = hmul2(A0[q], sca);
            A1[q] = hmul2(A1[q], sca);
            B0[q] = hmul2(B0[q], scb);
            B1[q] = hmul2(B1[q], scb);
          }
#pragma unroll
          for (int G = 0; G < kNG; ++G) {
            if (G < ngroups) {
              const uint4 *tl = tile;
              const uint4 bh0 = tl[act_chunk16(G, sp, 0, g, t)];
              const uint4 bh1 = tl[act_chunk16(G, sp, 1, g, t)];
              // MMA j = 0, 1 from half 0; j = 2, 3 from half 1
              mma_16816_f16(d[G], A0[0], B0[0], A0[1], B0[1], bh0.x, bh0.y);
              mma_16816_f16(d[G], A0[2], B0[2], A0[3], B0[3], bh0.z, bh0.w);
              mma_16816_f16(d[G], A1[0], B1[0], A1[1], B1[1], bh1.x, bh1.y);
              mma_16816_f16(d[G], A1[2], B1[2], A1[3], B1[3], bh1.z, bh1.w);
            }
          }
        }
#pragma unroll
        for (int G = 0; G < kNG; ++G) {
          if (G < ngroups) {
            const float c0 = cs[G * 8 + 2 * t], c1 = cs[G * 8 + 2 * t + 1];
            acc[G][0] = fmaf(d[G][0], c0, acc[G][0]);
            acc[G][1] = fmaf(d[G][1], c1, acc[G][1]);
            acc[G][2] = fmaf(d[G][2], c0, acc[G][2]);
            acc[G][3] = fmaf(d[G][3], c1, acc[G][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- round epilogue: scale, round to bf16, transpose, 16-byte stores
    if (has_rows && !*abort_flag) {
      const float gw = p.w_global ? p.w_global[r.e] : 1.0f;
      const float f = __fmul_rn(gw, p.g_a);
      uint16_t *st = staging + cw * (kTS * 16);
#pragma unroll
      for (int G = 0; G < kNG; ++G) {
        if (G < ngroups) {
          const int c0 = G * 8 + 2 * t;
          const uint32_t lo = pack_bf16x2(acc[G][0] * f, acc[G][1] * f);  // row g, cols c0, c0+1
          const uint32_t hi = pack_bf16x2(acc[G][2] * f, acc[G][3] * f);  // row g+8
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
          const uint32_t pair = p.order[r.tok0 + col];
          *reinterpret_cast<uint4 *>(p.out + (int64_t)pair * N + n) =
              *reinterpret_cast<const uint4 *>(st + col * 16 + half * 8);
        }
      }
      __syncwarp();
    }
  }
}

}  // namespace gemv
}  // namespace moe
