// gemv_mma.cuh -- step 4b, decode variant: grouped expert GEMV on an NVFP4
// expert library for passes of up to 16 tokens per expert.
//
// FlashRT "grouped-moe-gemv" card (Available functions:
// grouped_w4a16_gemv_bf16 / grouped_w4a4_gemv_bf16; token-major routing).
//
// At decode batch sizes the weight stream is the roofline and the
// tensor-core work per weight is tiny (8-16 tokens), so this variant keeps
// the tensor cores fed from registers and spends its effort on the stream:
//   * Work partition over (active expert, pass, 16-row block) units: when
//     the passes are no more than the persistent CTAs, every CTA takes part
//     of exactly one pass (cta_pass_range), else equal contiguous ranges cut
//     at round boundaries; rounds of up to 16 blocks of one (expert, pass),
//     warp w owns block w of every round.  The CTA computes its range once,
//     after each CTA has pulled its slice of the bf16 activations into L2
//     while waiting for the previous kernel (programmatic launch).
//   * Handed the routing map without the step-2 grouping (at most 4096
//     slots, 512 experts), every CTA groups the map itself: per-expert counts
//     (shared-memory histogram), the active experts' CSR offsets (block scan),
//     and the token lists of the passes in its own range (a stable block-wide
//     compaction per expert), so no grouping kernel precedes it.
//   * Each pair of warps shares a one-stage pipeline, with no producer warp
//     and no waits beyond the pair inside a pass; sixteen warps (four per
//     scheduler) hide each other's load and dependency latencies.  A stage
//     is the pair's two 16-row blocks x 1024 codes: one 4-D TMA box (32 rows
//     x 4 lines of 128 bytes, 512 contiguous bytes per row, 128-byte
//     swizzle, L2 evict-first) plus one 3-D box of the stage's 32 x 64 E4M3
//     scale bytes, both issued by the even warp's lane 0 and completing on
//     the stage's mbarrier; each warp then releases the stage on a second
//     barrier, and the even warp refills it once both have.  The TMA
//     engine's throughput grows with the size of its boxes: 16 KB boxes
//     stream about 1.6x faster than 8 KB ones at the same bytes in flight.
//   * Lane (g, t) owns line t of rows g and g + 8.  A line index in the box is
//     4 * row + line, so the swizzle key is (row & 1) * 4 + line and the eight
//     lanes of one shared-memory phase (rows g, g + 1) hit eight distinct
//     16-byte bank groups.
//   * The CTA requests its first pass's activation rows as soon as its token
//     lists are compacted, and every pair its first weight stage right
//     after, so the rows do not queue behind the weights' first burst and
//     the weights stream while the CTA converts its first activation tile.
//   * When a CTA starts a new (expert, pass), it builds that pass's fp16
//     activation tile once, for the whole K; every round of the pass reuses
//     it.  The tile is token-major, one row per token: W4A16 rows arrive as
//     one bulk copy each (TMA engine, one mbarrier), then one warp per token
//     takes the row's largest magnitude and converts the row in place, stage
//     by stage, transposing each stage's 4 x 32 units (line t, MMA pair m) to
//     m * 4 + t; with rows 4 units past a multiple of 8, the eight lanes of a
//     quarter-warp read eight different bank groups.  W4A16: each
//     token is scaled by a power of two of its own so that its largest
//     element lands in [2^14, 2^15), then converted to fp16 -- exact for every
//     element within 2^29 of the token's maximum, whatever the token's
//     magnitude (bf16's whole range), and bit-identical to no scaling when the
//     token already fits fp16 (fp32 accumulation rounds alike at any power-of-
//     two scale); the epilogue multiplies each token column back.  W4A4:
//     E2M1 x E4M3 products, exact in fp16.
//   * Each lane dequantises its codes in registers (hardware E2M1 -> f16x2
//     converter, times the block's E4M3 scale: exact in fp16) and issues
//     m16n8k16 MMAs (fp32 accumulation, two independent chains per 8-token
//     group) with the tokens on the n side.  Lane t's MMA i takes the four
//     codes 256 t + 4 i .. + 3 of the stage; the activation tile uses the same
//     column permutation, so the dot product is unchanged.
//   * Each block's accumulators are scaled by g_w * g_a, rounded to bf16,
//     transposed through shared memory and written as 16-byte row segments.
#pragma once
#include "gemv_common.cuh"

namespace moe {
namespace gemv {
namespace mma {

constexpr int kCW = 16;                      // warps, one 16-row block each per round
constexpr int kThreads = kCW * 32;
constexpr int kLines = 4;                    // 128-byte lines (256 codes) per row per stage
constexpr int kKS = kLines * 256;            // codes per row per stage
constexpr int kPairs = kCW / 2;              // warp pairs; a pair shares one 32-row stage
constexpr int kRowW = kLines * 128;          // bytes of codes per row per stage
constexpr int kRowSF = kLines * 16;          // scale bytes per row per stage
constexpr int kStageRows = 32;               // rows per stage: the pair's two blocks
constexpr int kStageW = kStageRows * kRowW;  // 16 KB
constexpr int kStageSF = kStageRows * kRowSF;  // 2 KB
constexpr int kMaxTS = 16;                   // tokens per pass at most (2 groups of 8)
constexpr int kNG = kMaxTS / 8;
// The fp16 activation tile is token-major: one row per token holding K
// (rounded up to whole stages) fp16.  Within a stage the row keeps the 16-byte
// unit of line t, MMA pair m at m * 4 + t, so that the four lanes t of one
// token read four neighbouring units; rows are padded by 64 bytes (a row is
// then 4 units past a multiple of 8), so the two tokens of a quarter-warp
// fall into opposite halves of the eight 16-byte bank groups: the MMA's
// activation loads are conflict-free.
constexpr int kActPad = 64;
constexpr int kActBytes = kMaxTS * (2048 * 2 + kActPad);  // 16 tokens at K = 2048
__host__ __device__ constexpr int act_row_bytes(int K) {
  return (K + kKS - 1) / kKS * kKS * 2 + kActPad;
}
static_assert((kKS * 2 / 16) % 8 == 0 && (kActPad / 16) % 8 == 4, "activation row bank layout");
constexpr int kStagingBytes = kCW * kMaxTS * 16 * 2;
constexpr uint64_t kActPrefetchMax = 8u << 20;     // activations prefetched into L2 up to 8 MiB
// 16-byte activation slices per thread in a W4A4 pass set-up: a tile holds
// ts rows of act_row_bytes(K) <= kActBytes, so ts * kpad <= 16 * 2048
// columns, 8 columns per slice, spread over the CTA.
constexpr int kSetupTasks = kMaxTS * 2048 * 2 / 16 / kThreads;

constexpr size_t kOffW = 0;
constexpr size_t kOffSF = kOffW + (size_t)kPairs * kStageW;
constexpr size_t kOffAct = kOffSF + (size_t)kPairs * kStageSF;
constexpr size_t kOffStaging = kOffAct + kActBytes;
constexpr int kMaxActive = 512;              // active experts this variant takes
constexpr size_t kOffPrefix = kOffStaging + kStagingBytes;
constexpr size_t kOffStart = kOffPrefix + (kMaxActive + 4) * 4;
constexpr size_t kOffEid = kOffStart + (kMaxActive + 4) * 4;
constexpr size_t kOffPair = kOffEid + (kMaxActive + 4) * 4;
// In-kernel grouping (routing map given, no step-2 outputs): every CTA
// histograms the map and compacts the token lists of the passes in its own
// range.  With at most kFusedSlots slots and kMaxActive experts there are at
// most S/16 + E <= 768 passes and a CTA's round-aligned range touches at most
// ceil(768 / 148) + 1 = 7 of them (one when there are no more passes than CTAs).
constexpr int kFusedSlots = 4096;
constexpr int kFusedPer = kFusedSlots / kThreads;  // slots per thread
constexpr int kMaxCtaPasses = 16;
constexpr size_t kOffPasses = kOffPair + kMaxTS * 4;                 // [kMaxCtaPasses][kMaxTS]
constexpr size_t kOffPassMeta = kOffPasses + (size_t)kMaxCtaPasses * kMaxTS * 4;  // [3][kMaxCtaPasses]
constexpr size_t kOffTokMax = kOffPassMeta + (size_t)3 * kMaxCtaPasses * 4 + 8;  // [2][kMaxTS]
constexpr size_t kOffBar = kOffTokMax + (size_t)2 * kMaxTS * 4;
// full[kPairs], empty[kPairs], the activation rows' barrier
constexpr size_t kOffMisc = kOffBar + (size_t)(2 * kPairs + 1) * 8;
constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kStageW % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");
static_assert(kSmemBytes <= 232448, "shared memory per block");
static_assert(kMaxActive <= kThreads && kStagingBytes >= (kMaxActive + 64) * 4,
              "the in-kernel grouping keeps one expert per thread and its counters in staging");

// Tokens per pass for a hidden size K (a multiple of 256): as many 8-token
// groups (up to 2) as the activation tile holds for the whole K; 0 when not
// even one fits.
__host__ __device__ constexpr int tokens_per_pass(int K) {
  const int groups = kActBytes / (8 * act_row_bytes(K));
  return 8 * (groups < kNG ? groups : kNG);
}



__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// One stage of one warp: lane (g, t) dequantises line t of rows g and g + 8
// (256 codes each) and multiplies with the NG token groups of the activation
// tile, accumulating into acc0 / acc1.  act_lane points at the stage's unit
// (line t, pair 0) in token g's row; group G's token is 8 G rows further
// (group_bytes apart).
template <int NG>
__device__ __forceinline__ void mma_stage(const uint8_t *sw, const uint8_t *ssf,
                                          const uint8_t *act_lane, int group_bytes, int g, int t,
                                          bool line_ok, float (&acc0)[kNG][4],
                                          float (&acc1)[kNG][4]) {
  const uint8_t *ra = sw + g * kRowW + t * 128;
  const uint8_t *rb = ra + 8 * kRowW;
  const int key = ((g & 1) << 2) | t;  // rows g and g + 8 share the parity
  uint4 sa = make_uint4(0u, 0u, 0u, 0u), sb = sa;
  if (line_ok) {
    sa = *reinterpret_cast<const uint4 *>(ssf + g * kRowSF + t * 16);
    sb = *reinterpret_cast<const uint4 *>(ssf + (g + 8) * kRowSF + t * 16);
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    // 16-byte chunk q of the line: 32 codes, scale bytes 2q and 2q + 1
    uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa;
    if (line_ok) {
      wa = *reinterpret_cast<const uint4 *>(ra + ((q ^ key) << 4));
      wb = *reinterpret_cast<const uint4 *>(rb + ((q ^ key) << 4));
    }
    const uint32_t swa = word_of(sa, q >> 1), swb = word_of(sb, q >> 1);
    const uint32_t pa = e4m3x2_to_f16x2((q & 1) ? (swa >> 16) : (swa & 0xFFFFu));
    const uint32_t pb = e4m3x2_to_f16x2((q & 1) ? (swb >> 16) : (swb & 0xFFFFu));
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      const uint32_t sca = wd < 2 ? bcast_lo(pa) : bcast_hi(pa);
      const uint32_t scb = wd < 2 ? bcast_lo(pb) : bcast_hi(pb);
      uint32_t A[4], B[4];
      e2m1x8_to_f16x2(word_of(wa, wd), A[0], A[1], A[2], A[3]);  // row g
      e2m1x8_to_f16x2(word_of(wb, wd), B[0], B[1], B[2], B[3]);  // row g + 8
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        A[i] = hmul2(A[i], sca);
        B[i] = hmul2(B[i], scb);
      }
#pragma unroll
      for (int G = 0; G < NG; ++G) {
        // the 8 columns of MMA pair m = 4 q + wd: codes 8 m .. 8 m + 7 of the line
        const uint4 bv =
            *reinterpret_cast<const uint4 *>(act_lane + G * group_bytes + (4 * q + wd) * 64);
        mma_16816_f16(acc0[G], A[0], B[0], A[1], B[1], bv.x, bv.y);
        mma_16816_f16(acc1[G], A[2], B[2], A[3], B[3], bv.z, bv.w);
      }
    }
  }
}

// Walks the rounds of a CTA's range [u, u_end) (round-aligned) in order: the
// first block of the round steps by kCW within a pass, then the pass, then
// the active expert, so only the starting position needs a division.
struct RoundWalk {
  uint32_t u, u_end;
  int a;
  uint32_t pass;
  int rb;
  __device__ __forceinline__ void init(const Meta &m, uint32_t A, int RB, uint32_t u0,
                                       uint32_t u1) {
    u = u0;
    u_end = u1;
    a = expert_of_unit(m.prefix, A, u0);
    const uint32_t v = u0 - m.prefix[a];
    pass = v / (uint32_t)RB;
    rb = (int)(v % (uint32_t)RB);
  }
  __device__ __forceinline__ bool next(const Meta &m, int RB, uint32_t ts, Round &r) {
    if (u >= u_end) return false;
    const uint32_t s0 = m.start[a], c = m.start[a + 1] - s0;
    const uint32_t first = pass * ts;
    int nblk = RB - rb;
    if (nblk > kCW) nblk = kCW;
    if ((uint32_t)nblk > u_end - u) nblk = (int)(u_end - u);
    r.e = m.eid[a];
    r.first = first;
    r.tok0 = s0 + first;
    r.ntok = (int)min(ts, c - first);
    r.n0 = rb * 16;
    r.nrows = min(nblk * 16, m.N - r.n0);
    r.nblk = nblk;
    u += (uint32_t)nblk;
    rb += nblk;
    if (rb == RB) {
      rb = 0;
      if (first + ts >= c) {
        ++a;
        pass = 0;
      } else {
        ++pass;
      }
    }
    return true;
  }
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemv_mma_kernel(const Params p, const int ts, const __grid_constant__ CUtensorMap tmap_w,
                            const __grid_constant__ CUtensorMap tmap_sf) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic (not through an integer), so the
  // compiler still sees shared memory and addresses it as such
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t *act = smem + kOffAct;  // token-major fp16 rows, act_row_bytes(K) apart
  uint16_t *staging = reinterpret_cast<uint16_t *>(smem + kOffStaging);
  uint32_t *prefix = reinterpret_cast<uint32_t *>(smem + kOffPrefix);
  uint32_t *s_start = reinterpret_cast<uint32_t *>(smem + kOffStart);
  int32_t *s_eid = reinterpret_cast<int32_t *>(smem + kOffEid);
  uint32_t *s_pair = reinterpret_cast<uint32_t *>(smem + kOffPair);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint64_t *act_bar = full + 2 * kPairs;  // a pass's activation rows have landed
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc);

  const int warp = threadIdx.x >> 5;
  const int lane = (int)lane_id();
  // set-up that reads no input runs before the wait for the previous grid
  if (threadIdx.x == 0) {
    // one arrival with the byte count of the stage's two TMA boxes
    for (int i = 0; i < kPairs; ++i) {
      mbar_init(&full[i], 1u);              // the leader's expect-tx arrival
      mbar_init(&full[kPairs + i], 2u);     // "empty": both warps of the pair are done
    }
    mbar_init(act_bar, 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 2 * kMaxTS) {
    reinterpret_cast<uint32_t *>(smem + kOffTokMax)[threadIdx.x] = 0u;
  }
  const int arow = act_row_bytes(p.K);  // bytes per token row of the tile
  if (lane == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_sf);
  }
  if (MODE == MOE_W4A16 && threadIdx.x == 32) {
    // The bf16 activations are an input of the step, not of the grid this
    // launch waits for: every CTA pulls its share of them into L2 while it
    // waits, so the pass set-up finds them there.
    const uint32_t bytes = (uint32_t)p.M * (uint32_t)p.K * 2u;  // K % 64 == 0
    if ((uint64_t)p.M * p.K * 2u <= kActPrefetchMax) {
      const uint32_t chunk = ((bytes + gridDim.x - 1) / gridDim.x + 15u) & ~15u;
      const uint32_t end = min(bytes, chunk * (blockIdx.x + 1));
      for (uint32_t off = chunk * blockIdx.x; off < end; off += 16384u)
        prefetch_l2_bulk(static_cast<const uint8_t *>(p.act) + off, min(16384u, end - off));
    }
  }
  if (p.order == nullptr && threadIdx.x == 64 &&
      (reinterpret_cast<uintptr_t>(p.indices) & 15u) == 0u) {
    // the routing map this CTA will group: into L2 while the previous kernel
    // (the mask, which may still write -1 into it) runs; a hint only (16-byte
    // aligned maps; the size rounded down, so nothing past the map is touched)
    const uint32_t bytes = ((uint32_t)p.M * (uint32_t)p.top_k * 8u) & ~15u;
    for (uint32_t off = 0; off < bytes; off += 16384u)
      prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(p.indices) + off, min(16384u, bytes - off));
  }
  const bool fused = p.order == nullptr;
  uint32_t *cnt = reinterpret_cast<uint32_t *>(staging);   // prologue only: expert counters
  uint64_t *scan_scratch = reinterpret_cast<uint64_t *>(cnt + kMaxActive);  // and scan scratch
  if (fused) {  // the counters are this CTA's own: cleared while the previous grid runs
    for (int e = threadIdx.x; e < p.E; e += kThreads) cnt[e] = 0u;
    __syncthreads();
  }
  pdl_wait();
  pdl_launch_dependents();
  const int N = p.N, K = p.K;
  const int RB = (N + 15) / 16;
  int32_t my_ids[kFusedPer];  // in-kernel grouping: experts of this thread's slots (-1: none)
  const int fq = fused ? (p.M * p.top_k + kThreads - 1) / kThreads : 0;
  uint32_t A, U;
  if (fused) {
    // group the routing map here: counts per expert, then the active experts in
    // ascending id with their CSR offsets (the moe_create_indices definition)
    // and the row-block units before each (its passes times RB)
    const int S = p.M * p.top_k;
#pragma unroll
    for (int j = 0; j < kFusedPer; ++j) {
      const int slot = (int)threadIdx.x * fq + j;
      const int64_t id = (j < fq && slot < S) ? __ldg(p.indices + slot) : -1;
      my_ids[j] = (id >= 0 && id < p.E) ? (int32_t)id : -1;
    }
#pragma unroll
    for (int j = 0; j < kFusedPer; ++j)
      if (my_ids[j] >= 0) atomicAdd(&cnt[my_ids[j]], 1u);
    __syncthreads();
    // one scan of (passes << 32 | active flag << 16 | count): counts stay below
    // 2^13 and the active experts below 2^10, so no field carries into the next
    const uint32_t c = (int)threadIdx.x < p.E ? cnt[threadIdx.x] : 0u;
    const uint32_t passes = (c + (uint32_t)ts - 1u) / (uint32_t)ts;
    uint64_t tot;
    const uint64_t sc = block_exclusive_scan64(
        ((uint64_t)passes << 32) | (c > 0u ? 0x10000u : 0u) | c, scan_scratch, &tot);
    const uint32_t pos = ((uint32_t)sc >> 16) & 0xFFFFu, off = (uint32_t)sc & 0xFFFFu;
    const uint32_t n_active = ((uint32_t)tot >> 16) & 0xFFFFu, n_routed = (uint32_t)tot & 0xFFFFu;
    if (c > 0u) {
      s_eid[pos] = (int32_t)threadIdx.x;
      s_start[pos] = off;
      prefix[pos] = (uint32_t)(sc >> 32) * (uint32_t)RB;
    }
    if (threadIdx.x == 0) {
      s_start[n_active] = n_routed;
      prefix[n_active] = (uint32_t)(tot >> 32) * (uint32_t)RB;
    }
    A = n_active;
    U = (uint32_t)(tot >> 32) * (uint32_t)RB;
    __syncthreads();
  } else {
    A = p.stats[1];
    // the grouping of the active experts (at most kMaxActive, checked on the host)
    // stays in shared memory: every round looks it up
    for (uint32_t i = threadIdx.x; i <= A; i += blockDim.x) {
      s_start[i] = p.start[i];
      if (i < A) s_eid[i] = p.eids[i];
    }
    __syncthreads();
    if (warp == 0) build_prefix(prefix, s_start, A, (uint32_t)ts, RB, lane);
    __syncthreads();
    U = prefix[A];
  }
  // the CTA's share of the units (every thread computes the same)
  uint32_t u_begin, u_end;
  cta_pass_range(U, RB, kCW, u_begin, u_end);
  if (u_begin >= u_end) return;
  const int nst = (K + kKS - 1) / kKS;  // stages per block
  const int lines_total = K / 256;
  const Meta meta{prefix, s_start, s_eid, N};
  int pass_idx = -1;  // index of the current pass in s_passes
  uint32_t act_issued = 0;  // passes whose row copies warp 0 has requested (lane 0's count)
  const int pair = warp >> 1, half = warp & 1;
  const bool leader = half == 0;  // the pair's even warp issues the pair's copies
  uint8_t *pw = smem + kOffW + (size_t)pair * kStageW;
  uint8_t *ps = smem + kOffSF + (size_t)pair * kStageSF;
  uint64_t *pfull = full + pair;
  uint64_t *pempty = full + kPairs + pair;

  // ---- producer side of the pair's pipeline (leader warp): the next (round, stage)
  // in which the pair holds a block
  RoundWalk piter;
  piter.init(meta, A, RB, u_begin, u_end);
  Round pr;
  int pc = 0;
  bool pvalid = false;
  auto next_own_round = [&]() {
    pvalid = false;
    pc = 0;
    while (piter.next(meta, RB, (uint32_t)ts, pr))
      if (2 * pair < pr.nblk) {
        pvalid = true;
        break;
      }
  };
  next_own_round();
  uint32_t produced = 0;
  auto produce = [&]() {
    // lane 0's view of the abort flag decides for the whole warp
    if (!leader || !pvalid || __shfl_sync(0xFFFFFFFFu, *abort_flag, 0)) return;
    // the stage is refilled once both warps of the pair have released its previous contents
    if (produced > 0 && !mbar_wait_bounded(pempty, (produced - 1) & 1u, p.wait_limit_ns))
      *abort_flag = 1;
    if (__shfl_sync(0xFFFFFFFFu, *abort_flag, 0)) return;
    const int n0 = pr.n0 + 32 * pair;
    if (lane == 0) {
      const uint64_t policy = l2_evict_first_policy();  // made here: no register holds it between stages
      mbar_arrive_expect_tx(pfull, (uint32_t)(kStageW + kStageSF));
      tma_load_4d(pw, &tmap_w, 0, pc * kLines, n0, pr.e, pfull, policy);
      // scales: 32 rows x 4 words (one 16-byte group per line), rows beyond N and
      // lines beyond K read as zero
      tma_load_3d(ps, &tmap_sf, pc * kLines * 4, n0, pr.e, pfull, policy);
    }
    ++produced;
    if (++pc == nst) next_own_round();
  };

  uint32_t *s_passes = reinterpret_cast<uint32_t *>(smem + kOffPasses);
  int n_passes = 0;
  if (fused) {
    // token lists of the passes in this CTA's range: pass i of expert e holds
    // the pairs of rank [first, first + ntok) among e's pairs in ascending
    // pair order (stable), found with one block scan per distinct expert.
    // First the distinct passes of the range, in order (one thread).
    int32_t *pe = reinterpret_cast<int32_t *>(smem + kOffPassMeta);
    uint32_t *pf = reinterpret_cast<uint32_t *>(pe + kMaxCtaPasses);
    int32_t *pn = reinterpret_cast<int32_t *>(pf + kMaxCtaPasses);
    int32_t *s_np = pn + kMaxCtaPasses;
    if (U / (uint32_t)RB <= gridDim.x) {
      // no more passes than CTAs: the range lies in one pass, which every
      // thread finds by itself (the shared copy serves the pass set-up)
      const int a = expert_of_unit(prefix, A, u_begin);
      const uint32_t pass = (u_begin - prefix[a]) / (uint32_t)RB;
      const uint32_t c = s_start[a + 1] - s_start[a];
      const int32_t e = s_eid[a];
      const uint32_t first = pass * (uint32_t)ts;
      const int ntok = (int)min((uint32_t)ts, c - first);
      uint32_t mine = 0, total;
#pragma unroll
      for (int j = 0; j < kFusedPer; ++j) mine += my_ids[j] == e ? 1u : 0u;
      uint32_t rank = block_exclusive_scan(mine, reinterpret_cast<uint32_t *>(scan_scratch), &total);
#pragma unroll
      for (int j = 0; j < kFusedPer; ++j) {
        if (my_ids[j] != e) continue;
        if (rank - first < (uint32_t)ntok)
          s_passes[rank - first] = (uint32_t)threadIdx.x * (uint32_t)fq + (uint32_t)j;
        ++rank;
      }
      n_passes = 1;
    } else if (threadIdx.x == 0) {
      RoundWalk w;
      w.init(meta, A, RB, u_begin, u_end);
      Round rr;
      int cnt_p = 0, prev_e = -1;
      uint32_t prev_first = 0xFFFFFFFFu;
      while (cnt_p < kMaxCtaPasses && w.next(meta, RB, (uint32_t)ts, rr)) {
        if (rr.e == prev_e && rr.first == prev_first) continue;
        pe[cnt_p] = rr.e;
        pf[cnt_p] = rr.first;
        pn[cnt_p] = rr.ntok;
        ++cnt_p;
        prev_e = rr.e;
        prev_first = rr.first;
      }
      *s_np = cnt_p;
    }
    if (n_passes == 0) {
      __syncthreads();
      const int np = *s_np;
      n_passes = np;
      for (int i = 0; i < np; ++i) {
        if (i > 0 && pe[i] == pe[i - 1]) continue;  // the passes of one expert share a scan
        const int e = pe[i];
        uint32_t mine = 0, total;
#pragma unroll
        for (int j = 0; j < kFusedPer; ++j) mine += my_ids[j] == e ? 1u : 0u;
        uint32_t rank =
            block_exclusive_scan(mine, reinterpret_cast<uint32_t *>(scan_scratch), &total);
#pragma unroll
        for (int j = 0; j < kFusedPer; ++j) {
          if (my_ids[j] != e) continue;
          for (int k = i; k < np && pe[k] == e; ++k)
            if (rank - pf[k] < (uint32_t)pn[k])
              s_passes[k * kMaxTS + (rank - pf[k])] =
                  (uint32_t)threadIdx.x * (uint32_t)fq + (uint32_t)j;
          ++rank;
        }
      }
    }
    __syncthreads();
  }

  // ---- consumer side
  const int g = lane >> 2, t = lane & 3;
  RoundWalk iter;
  iter.init(meta, A, RB, u_begin, u_end);
  Round r;
  // W4A16: the first pass's activation rows are requested before any weight
  // stage, so they do not wait behind the weight stream's first burst
  const bool first_rows_early = MODE == MOE_W4A16;
  if (first_rows_early && warp == 0) {
    RoundWalk peek = iter;
    Round r0;
    if (peek.next(meta, RB, (uint32_t)ts, r0)) {
      uint32_t row0 = 0;
      if (lane < r0.ntok)
        row0 = (fused ? s_passes[lane] : __ldg(p.order + r0.tok0 + lane)) / (uint32_t)p.top_k;
      if (lane == 0) {
        mbar_arrive_expect_tx(act_bar, (uint32_t)r0.ntok * (uint32_t)K * 2u);
        ++act_issued;
      }
      __syncwarp();
      if (lane < r0.ntok)
        bulk_load_g2s(act + lane * arow, static_cast<const uint16_t *>(p.act) + (int64_t)row0 * K,
                      (uint32_t)K * 2u, act_bar);
    }
  }
  __syncthreads();  // the first rows are requested before every pair's first weight stage
  // then the weights stream while the CTA converts its first activation tile
  produce();
  uint32_t consumed = 0;
  uint32_t pass_key = 0xFFFFFFFFu;
  int ng = 0;
  const int kpad = nst * kKS;

  while (iter.next(meta, RB, (uint32_t)ts, r)) {
    if (r.tok0 != pass_key) {
      // ---- new (expert, pass): build its fp16 activation tile for the whole K,
      // one row per token (lane j of every warp holds the pair of token j)
      uint32_t my_pair = 0, my_row = 0;
      ++pass_idx;
      // (the host's limits keep a CTA's passes within the table; should one
      // not be, the call reports it and computes nothing rather than read past)
      const bool listed = !fused || pass_idx < n_passes;
      if (!listed && threadIdx.x == 0) {
        raise_device_error(MOE_DEVERR_LIMIT);
        *abort_flag = 1;
      }
      if (lane < r.ntok && listed) {
        my_pair = fused ? s_passes[pass_idx * kMaxTS + lane] : __ldg(p.order + r.tok0 + lane);
        my_row = my_pair / (uint32_t)p.top_k;
      }
      uint32_t *tokmax = reinterpret_cast<uint32_t *>(smem + kOffTokMax) + (pass_idx & 1) * kMaxTS;
      const int ng_new = (r.ntok + 7) / 8;
      if (MODE == MOE_W4A16) {
        // the previous tile is free once every warp is here
        if (pass_key != 0xFFFFFFFFu) named_bar_sync(1, kThreads);
        // each token's bf16 row, one bulk copy straight into its tile row
        if (warp == 0 && !(pass_idx == 0 && first_rows_early) &&
            !__shfl_sync(0xFFFFFFFFu, *abort_flag, 0)) {
          // the previous pass's plain reads and writes of the tile come before
          // the copies' writes
          fence_proxy_async_smem();
          if (lane == 0) {
            mbar_arrive_expect_tx(act_bar, (uint32_t)r.ntok * (uint32_t)K * 2u);
            ++act_issued;
          }
          __syncwarp();
          if (lane < r.ntok)
            bulk_load_g2s(act + lane * arow, static_cast<const uint16_t *>(p.act) + (int64_t)my_row * K,
                          (uint32_t)K * 2u, act_bar);
        }
        if (!*abort_flag && !mbar_wait_bounded(act_bar, (uint32_t)pass_idx & 1u, p.wait_limit_ns))
          *abort_flag = 1;
        if (warp < r.ntok) {
          // one warp per token row: the row's largest magnitude, then each
          // stage converted in place -- scaled by the token's power of two
          // (exact), fp16 (exact in range) -- and its 4 x 32 units (line t,
          // pair m) transposed to m * 4 + t; columns past K become zeros
          uint8_t *row = act + warp * arow;
          const int units = K / 8;
          uint32_t mx = 0u;
          for (int u = lane; u < units; u += 32) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + u * 16);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              mx = max(mx, max((w4[i] << 16) & 0x7FFF0000u, w4[i] & 0x7FFF0000u));
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) tokmax[warp] = mx;
          const float down = pow2f(-token_shift(mx));
          for (int c = 0; c < nst; ++c) {
            uint4 h[4];
#pragma unroll
            for (int tl = 0; tl < 4; ++tl) {
              const int u = c * (kKS / 8) + tl * 32 + lane;
              h[tl] = make_uint4(0u, 0u, 0u, 0u);
              if (u < units) {
                const uint4 v = *reinterpret_cast<const uint4 *>(row + u * 16);
                float f[8];
                f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
                f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
                f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
                f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], down);
                h[tl] = make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]),
                                   pack_f16x2(f[4], f[5]), pack_f16x2(f[6], f[7]));
              }
            }
            __syncwarp();  // the stage's units are all read before any is rewritten
#pragma unroll
            for (int tl = 0; tl < 4; ++tl)
              *reinterpret_cast<uint4 *>(row + (c * (kKS / 8) + lane * 4 + tl) * 16) = h[tl];
            __syncwarp();
          }
        }
        ng = ng_new;
        if ((int)threadIdx.x < r.ntok) s_pair[threadIdx.x] = my_pair;
      } else {
        // W4A4: the NVFP4 codes and their scales are loaded before the barrier
        // that frees the previous tile, so their latency overlaps it; columns
        // past K (up to the last stage's end) are written as zeros.  Task b of
        // a thread is slice kk of token tau, b * kThreads + tid = tau * per_tok
        // + kk; per_tok is a multiple of 32, so tau is the same across a warp.
        const int per_tok = kpad / 8;  // 8-column slices per token
        const int ntask = r.ntok * per_tok;  // at most kSetupTasks * kThreads
        const int tau0 = (int)threadIdx.x / per_tok, kk0 = (int)threadIdx.x - tau0 * per_tok;
        int tau = tau0, kk = kk0;
        uint4 v[kSetupTasks];
        uint32_t sv[kSetupTasks];
#pragma unroll
        for (int b = 0; b < kSetupTasks; ++b) {
          const int task = b * kThreads + (int)threadIdx.x;
          const int64_t m = (int64_t)__shfl_sync(0xFFFFFFFFu, my_row, tau & 31);
          const int k = kk * 8;
          v[b] = make_uint4(0u, 0u, 0u, 0u);
          sv[b] = 0u;
          if (task < ntask && k < K) {
            const uint8_t *qp = static_cast<const uint8_t *>(p.act) + m * (K / 2);
            v[b].x = __ldg(reinterpret_cast<const uint32_t *>(qp + k / 2));
            sv[b] = p.sfa[m * (K / 16) + k / 16];
          }
          for (kk += kThreads; kk >= per_tok; kk -= per_tok) ++tau;
        }
        if (pass_key != 0xFFFFFFFFu) named_bar_sync(1, kThreads);  // previous tile no longer read
        ng = ng_new;
        if ((int)threadIdx.x < r.ntok) s_pair[threadIdx.x] = my_pair;
        tau = tau0;
        kk = kk0;
#pragma unroll
        for (int b = 0; b < kSetupTasks; ++b) {
          const int task = b * kThreads + (int)threadIdx.x;
          const int tk = tau, k = kk * 8;
          for (kk += kThreads; kk >= per_tok; kk -= per_tok) ++tau;
          if (task >= ntask) continue;
          uint4 hv = make_uint4(0u, 0u, 0u, 0u);
          if (k < K) {
            const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(sv[b]));
            uint32_t q0, q1, q2, q3;
            e2m1x8_to_f16x2(v[b].x, q0, q1, q2, q3);
            hv.x = hmul2(q0, sc);
            hv.y = hmul2(q1, sc);
            hv.z = hmul2(q2, sc);
            hv.w = hmul2(q3, sc);
          }
          // columns [k, k + 8): stage c, line lt, MMA pair m, kept at unit m * 4 + lt
          const int u = k / 8, c = u / (kKS / 8), lt = (u % (kKS / 8)) / 32, m = u % 32;
          *reinterpret_cast<uint4 *>(act + tk * arow + (c * (kKS / 8) + m * 4 + lt) * 16) = hv;
        }
      }
      named_bar_sync(1, kThreads);
      pass_key = r.tok0;
    }

    if (2 * pair >= r.nblk) continue;  // the pair holds no block of this round
    const bool own = warp < r.nblk;     // this warp's block (the odd warp may have none)
    const float gw = p.w_global ? __ldg(p.w_global + r.e) : 1.0f;  // used by the epilogue
    float acc0[kNG][4], acc1[kNG][4];
#pragma unroll
    for (int G = 0; G < kNG; ++G)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc0[G][i] = acc1[G][i] = 0.f;

    for (int c = 0; c < nst; ++c) {
      if (!*abort_flag && !mbar_wait_bounded(pfull, consumed & 1u, p.wait_limit_ns))
        *abort_flag = 1;
      if (!*abort_flag && own) {
        // this warp's 16 rows of the pair's stage
        const uint8_t *sw = pw + (size_t)half * 16 * kRowW;
        const uint8_t *ssf = ps + (size_t)half * 16 * kRowSF;
        const bool line_ok = c * kLines + t < lines_total;
        const uint8_t *act_lane = act + g * arow + c * (kKS * 2) + t * 16;
        if (ng == 1)
          mma_stage<1>(sw, ssf, act_lane, 8 * arow, g, t, line_ok, acc0, acc1);
        else
          mma_stage<2>(sw, ssf, act_lane, 8 * arow, g, t, line_ok, acc0, acc1);
      }
      ++consumed;
      __syncwarp();  // every lane is done with the stage
      if (lane == 0) mbar_arrive(pempty);
      produce();
    }

    // ---- block epilogue: scale, round to bf16, transpose, 16-byte stores
    if (!*abort_flag && own) {
      const float f = __fmul_rn(gw, p.g_a);
      uint16_t *st = staging + warp * (kMaxTS * 16);
      const uint32_t *tokmax = reinterpret_cast<const uint32_t *>(smem + kOffTokMax) +
                               (pass_idx & 1) * kMaxTS;
      float up0 = 1.0f, up1 = 1.0f;  // the power of two of this lane's two token columns
      // g_w * g_a first, the token's power of two last: the product then never
      // overflows early, and it rounds exactly as the unscaled one would
      auto y = [&](int G, int i) {
        return __fmul_rn(__fmul_rn(acc0[G][i] + acc1[G][i], f), (i & 1) ? up1 : up0);
      };
#pragma unroll
      for (int G = 0; G < kNG; ++G) {
        if (G < ng) {
          const int c0 = G * 8 + 2 * t;
          if (MODE == MOE_W4A16) {
            up0 = pow2f(token_shift(tokmax[c0]));
            up1 = pow2f(token_shift(tokmax[c0 + 1]));
          }
          const uint32_t lo = pack_bf16x2(y(G, 0), y(G, 1));
          const uint32_t hi = pack_bf16x2(y(G, 2), y(G, 3));
          st[c0 * 16 + g] = (uint16_t)(lo & 0xFFFFu);
          st[(c0 + 1) * 16 + g] = (uint16_t)(lo >> 16);
          st[c0 * 16 + g + 8] = (uint16_t)(hi & 0xFFFFu);
          st[(c0 + 1) * 16 + g + 8] = (uint16_t)(hi >> 16);
        }
      }
      __syncwarp();
      const int nw = r.n0 + warp * 16;
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

  // After a timed-out wait, let the copies still in flight land before the
  // CTA exits (bounded again).
  if (*abort_flag && leader && lane == 0 && produced > 0)
    mbar_wait_bounded(pfull, (produced - 1) & 1u, kDrainLimitNs);
  if (*abort_flag && warp == 0 && lane == 0 && act_issued > 0)
    mbar_wait_bounded(act_bar, (act_issued - 1) & 1u, kDrainLimitNs);
}

}  // namespace mma
}  // namespace gemv
}  // namespace moe
