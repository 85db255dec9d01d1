// gemv_common.cuh -- shared pieces of the grouped NVFP4 GEMV kernels: launch
// parameters, the per-CTA work partition over (active expert, token pass,
// 16-row block) units, and small helpers.
#pragma once
#include "common.cuh"

namespace moe {
namespace gemv {

constexpr int kMaxExperts = 1024;
constexpr int kBlocksPerRound = 8;      // 16-row blocks per round (128 rows), unless a
                                        // kernel asks for another round size
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: default limit of every pipeline wait
constexpr uint64_t kDrainLimitNs = 100000000ull;  // 100 ms: waits for copies in flight after an abort

struct Params {
  const void *act;          // W4A16: bf16 [M, K]; W4A4: u8 [M, K/2]
  const uint8_t *sfa;       // W4A4: [M, K/16]
  float g_a;
  int32_t M, top_k;
  const uint8_t *w;         // [E, N, K/2]
  const uint8_t *sfw;       // [E, N, K/16]
  const float *w_global;    // [E] or null
  int32_t N, K;
  const uint32_t *order;
  const uint32_t *start;
  const int32_t *eids;
  const uint32_t *stats;
  uint16_t *out;            // bf16 [M, top_k, N]
  uint64_t wait_limit_ns;   // limit of each pipeline wait (kWaitLimitNs unless a test shortens it)
  const int64_t *indices;   // routing map [M, top_k]: read when order == nullptr (the
  int32_t E;                // kernel then groups the pairs itself)
};

// W4A16 tokens enter the tensor cores as fp16 scaled by a power of two of
// their own: s = floor(log2(amax)) - 14 (clamped to [-126, 127]), so the
// token's largest element lands in [2^14, 2^15) and every bf16 value of the
// token within 2^29 of it is exact in fp16.  amax_bits are the fp32 bits of
// the token's largest magnitude.
__device__ __forceinline__ int token_shift(uint32_t amax_bits) {
  if (amax_bits == 0u) return 0;
  int s = (int)((amax_bits >> 23) & 0xFFu) - 127 - 14;
  return s < -126 ? -126 : (s > 127 ? 127 : s);
}
__device__ __forceinline__ float pow2f(int s) { return __uint_as_float((uint32_t)(s + 127) << 23); }

struct Round {
  int e;
  uint32_t tok0;
  uint32_t first;  // rank of the pass's first pair within its expert (pass * tokens per pass)
  int ntok;
  int n0;
  int nrows;
  int nblk;
};

// Per-expert metadata staged in shared memory at kernel start.
struct Meta {
  const uint32_t *prefix;  // units before active expert a
  const uint32_t *start;   // CSR offsets
  const int32_t *eid;      // expert ids
  int N;
};

// Active expert holding unit u: the a with prefix[a] <= u < prefix[a + 1]
// (binary search; u < prefix[A]).
__device__ __forceinline__ int expert_of_unit(const uint32_t *prefix, uint32_t A, uint32_t u) {
  int lo = 0, hi = (int)A - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Walks a CTA's unit range round by round; identical in every thread.
// Within an active expert the units (16-row blocks) are ordered by pass, then
// block: a pass's activations are gathered once per round of up to
// round_blocks blocks and its blocks follow each other.  (For bf16
// activations a pass's rows cost more to re-read than a round of FP4
// weights, so the weights are the operand re-streamed per pass.)
struct RoundIter {
  uint32_t u, u_end;
  int a;
  uint32_t ts;  // tokens per pass
  uint32_t round_blocks = kBlocksPerRound;
  __device__ __forceinline__ bool next(const Meta &m, int RB, Round &r) {
    if (u >= u_end) return false;
    while (u >= m.prefix[a + 1]) ++a;
    const uint32_t v = u - m.prefix[a];
    const uint32_t pass = v / (uint32_t)RB;
    const uint32_t rb = v % (uint32_t)RB;
    uint32_t nblk = (uint32_t)RB - rb;
    if (nblk > round_blocks) nblk = round_blocks;
    if (nblk > u_end - u) nblk = u_end - u;
    const uint32_t s0 = m.start[a];
    const uint32_t c = m.start[a + 1] - s0;
    r.e = m.eid[a];
    r.first = pass * ts;
    r.tok0 = s0 + r.first;
    r.ntok = (int)min(ts, c - r.first);
    r.n0 = (int)rb * 16;
    r.nrows = min((int)nblk * 16, m.N - r.n0);
    r.nblk = (int)nblk;
    u += nblk;
    return true;
  }
};

// floor(a * b / c) for a quotient below 2^32, dividing in 32 bits whenever the
// product fits (a 64-bit division is a long software sequence, and one
// thread computes the partition while the CTA waits).
__device__ __forceinline__ uint32_t muldiv(uint32_t a, uint32_t b, uint32_t c) {
  const uint64_t ab = (uint64_t)a * b;
  return (ab >> 32) == 0 ? (uint32_t)ab / c : (uint32_t)(ab / c);
}

// This CTA's share [u0, u1) of the U units, cut at round boundaries: every
// pass (RB units) splits into ceil(RB / rbk) rounds of up to rbk blocks, and
// the grid shares the rounds evenly, so no round is split between CTAs and a
// CTA's warps never face a partial round in the middle of a pass.
__device__ __forceinline__ void cta_round_range(uint32_t U, int RB, int rbk, uint32_t &u0,
                                                uint32_t &u1) {
  const uint32_t R = (uint32_t)((RB + rbk - 1) / rbk);
  const uint32_t T = U / (uint32_t)RB * R;  // rounds in all; T <= U
  const uint32_t r0 = muldiv(T, blockIdx.x, gridDim.x);
  const uint32_t r1 = muldiv(T, blockIdx.x + 1, gridDim.x);
  u0 = r0 / R * (uint32_t)RB + r0 % R * (uint32_t)rbk;
  u1 = r1 / R * (uint32_t)RB + r1 % R * (uint32_t)rbk;
}

// As cta_round_range, but when the passes (U / RB of them) are no more than
// the CTAs, every CTA takes part of exactly one pass: pass p gets the CTAs b
// with floor(b * P / G) == p and splits its rounds evenly among them.  Each
// CTA then builds one activation tile and never waits for its warps between
// passes.
__device__ __forceinline__ void cta_pass_range(uint32_t U, int RB, int rbk, uint32_t &u0,
                                               uint32_t &u1) {
  const uint32_t P = U / (uint32_t)RB, G = gridDim.x, b = blockIdx.x;
  if (P == 0 || P > G) {
    cta_round_range(U, RB, rbk, u0, u1);
    return;
  }
  // P <= G, and G (one CTA per SM) is below 2^16, so every product here fits 32 bits
  const uint32_t pass = b * P / G;
  const uint32_t first = (pass * G + P - 1) / P;        // first CTA of the pass
  const uint32_t count = ((pass + 1) * G + P - 1) / P - first;
  const uint32_t i = b - first;
  const uint32_t R = (uint32_t)((RB + rbk - 1) / rbk);
  const uint32_t r0 = muldiv(R, i, count), r1 = muldiv(R, i + 1, count);
  const uint32_t base = pass * (uint32_t)RB;
  u0 = base + (uint32_t)min((uint64_t)RB, (uint64_t)r0 * (uint32_t)rbk);
  u1 = base + (uint32_t)min((uint64_t)RB, (uint64_t)r1 * (uint32_t)rbk);
}

__device__ __forceinline__ uint32_t bcast_lo(uint32_t h) { return __byte_perm(h, h, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t h) { return __byte_perm(h, h, 0x3232); }

// Warp 0 of the CTA: prefix[a] = units before active expert a, where an
// expert with c tokens has ceil(c / ts) passes of RB row blocks.
__device__ __forceinline__ void build_prefix(uint32_t *prefix, const uint32_t *start, uint32_t A,
                                             uint32_t ts, int RB, int lane) {
  uint32_t run = 0;
  for (uint32_t a0 = 0; a0 < A; a0 += 32) {
    const uint32_t a = a0 + lane;
    uint32_t units = 0;
    if (a < A) {
      const uint32_t c = start[a + 1] - start[a];
      units = (c + ts - 1) / ts * (uint32_t)RB;
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

}  // namespace gemv
}  // namespace moe
