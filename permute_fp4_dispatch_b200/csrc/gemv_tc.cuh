// gemv_tc.cuh -- step 4b, tensor-memory variant: grouped expert GEMV on an
// NVFP4 expert library, for passes of many tokens per expert.
//
// FlashRT "grouped-moe-gemv" card (Available functions:
// grouped_w4a16_gemv_bf16 / grouped_w4a4_gemv_bf16; W4A4 routing is
// token-major: activations [M, K], library [E, N, K/2], output
// [M, top_k, N]).  For each routed pair p with expert e:
//     out[p, n] = bf16( g_w[e] * g_a * sum_k a(p/top_k, k) * w(e, n, k) ).
//
// Design (taken when experts hold more tokens than a decode pass; the FP4
// weight stream and its dequantisation bound it):
//   * Work is expert-major: an active expert's pairs (CSR from
//     moe_create_indices) are taken in passes of up to kTS = 64 tokens (128
//     for W4A16 whose activations were converted once per call, when the
//     experts hold more than 64 tokens on average: the token tile then
//     arrives by cp.async straight from the converted rows, one item ahead,
//     and each pass dequantises the weights for twice the tokens) and
//     each pass sweeps the expert's N rows in 16-row blocks.  The flat list of
//     (expert, pass, row block) units is split into equal contiguous ranges
//     cut at round boundaries, one per persistent CTA (grid = SM count).
//     Consecutive blocks of one (expert, pass) form a round of up to 128
//     rows: one tcgen05 MMA tile (M = 128 weight rows, N = tokens rounded up
//     to 16, fp32 in TMEM).
//   * Warp roles (10 warps):
//       warp 8      TMA producer: streams each round's FP4 rows and E4M3
//                   scales in chunks of kKC = 256 columns into a kStages-deep
//                   shared-memory ring (one 16-row x 128-byte box per row
//                   block, 128-byte swizzle, L2 evict-first; rows past N and
//                   columns past K arrive as zeros; scale rows whose stride is
//                   not a multiple of 16 bytes use 4-byte cp.async);
//       warps 0-7   dequantise: each lane owns one weight row (warp w covers
//                   TMEM lanes 32*(w%4).. and columns half w/4 of the chunk),
//                   E2M1 -> f16x2 with the hardware converter, times the
//                   block's E4M3 scale (at most 6 significant bits: exact in
//                   fp16), written to a double-buffered A tile in tensor
//                   memory with tcgen05.st; they also stage the chunk's
//                   activations as fp16 into a double-buffered, 128B-swizzled
//                   K-major B tile, and run the output epilogue;
//       warp 9      allocates TMEM and issues tcgen05.mma kind::f16 (A from
//                   TMEM, B from shared memory) for every chunk, committing to
//                   mbarriers that free the A/B buffers and publish D.
//     D is double-buffered in TMEM, so a round's epilogue (tcgen05.ld, scale
//     by g_w * g_a, round to bf16, store) runs while the next round's first
//     chunk is already being multiplied.
//   * W4A16 activations enter the tensor core as fp16.  Given room in the
//     caller's workspace, act_f16_kernel converts them once per call, each
//     token that does not fit fp16 exactly scaled by a power of two of its
//     own (exact over bf16's whole range, the power multiplied back in the
//     epilogue), and the staging warps only copy them.  Otherwise each chunk
//     is converted as it is staged: exact for 2^-14 <= |x| <= 65504,
//     fp16-subnormal rounding (absolute error <= 2^-25) below; |x| > 65504
//     raises MOE_DEVERR_ACT_RANGE.  W4A4 activations are dequantised
//     exactly like the weights.
#pragma once
#include "gemv_common.cuh"

namespace moe {
namespace gemv {
namespace tc {

constexpr int kDQ = 8;                  // dequant / staging / epilogue warps
constexpr int kTmaWarp = kDQ;
constexpr int kMmaWarp = kDQ + 1;
constexpr int kThreads = (kDQ + 2) * 32;
constexpr int kKC = 256;                // columns (codes) per chunk
constexpr int kWStride = kKC / 2;       // bytes per weight row in a stage (128B-swizzled)
constexpr int kSFStride = kKC / 16;     // bytes per scale row in a stage
constexpr int kBoxW = 16 * kWStride;    // one 16-row weight box
constexpr int kBoxSF = 16 * kSFStride;  // one 16-row scale box
constexpr int kStageW = 128 * kWStride;
constexpr int kStageBytes = kStageW + 128 * kSFStride;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol = 0;           // A tiles: columns [0, 256), 128 per buffer
constexpr uint32_t kDcol = 256;         // D tiles: two buffers of kTS columns from 256
static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");

// Sizes for TS tokens per pass (MMA N <= TS): 64, or 128 for W4A16 whose
// activations were converted once per call (the token tile then arrives by
// cp.async straight from the converted rows, and a pass of 128 tokens
// halves the weight dequantisation per token).
template <int TS>
struct Cfg {
  static constexpr int kTS = TS;
  static constexpr int kStages = TS >= 128 ? 4 : 5;
  static constexpr int kKatomBytes = TS * 128;  // one 64-column slab of the B tile
  static constexpr int kBTile = 4 * kKatomBytes;
  static constexpr size_t kOffB = (size_t)kStages * kStageBytes;
  static constexpr size_t kOffPrefix = kOffB + 2 * kBTile;
  static constexpr size_t kOffStart = kOffPrefix + (kMaxExperts + 4) * 4;
  static constexpr size_t kOffEid = kOffStart + (kMaxExperts + 4) * 4;
  static constexpr size_t kOffPair = kOffEid + (kMaxExperts + 4) * 4;  // [2][kTS] pair ids
  static constexpr size_t kOffShift = kOffPair + 2 * TS * 4;           // [2][kTS] token offsets
  static constexpr size_t kOffBar = kOffShift + 2 * TS * 4;
  static constexpr int kNumBars = 2 * kStages + 9;
  static constexpr size_t kOffMisc = kOffBar + kNumBars * 8;            // tmem slot, abort flag
  static constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;            // + alignment slack
  static_assert(kDcol + 2 * TS <= kTmemCols, "tensor memory columns");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

// W4A16 activations converted once per call for this variant (it stages
// activations for every 128-row round and 256-column chunk, so converting
// them there would repeat the work per round): one warp per row m of act,
// shift[m] = 0 when the row already converts to fp16 exactly (every nonzero
// magnitude within [2^-14, 65504]), else token_shift(its largest magnitude);
// act16 row m = fp16(act row m * 2^-shift[m]) (exact: a power of two).
__global__ void __launch_bounds__(256)
    act_f16_kernel(const uint16_t *__restrict__ act, int32_t M, int32_t K,
                   int32_t *__restrict__ shift, uint16_t *__restrict__ act16) {
  pdl_wait();
  pdl_launch_dependents();
  const int m = (int)blockIdx.x * 8 + (int)(threadIdx.x >> 5);
  const unsigned lane = lane_id();
  if (m >= M) return;
  const uint16_t *row = act + (int64_t)m * K;
  uint32_t mx = 0u, mn = 0xFFFFFFFFu;  // fp32 bits of the largest and smallest nonzero magnitude
  for (int k = 8 * (int)lane; k < K; k += 256) {  // K % 32 == 0: whole 16-byte slices
    const uint4 v = ldg_nc_v4(row + k);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (w4[i] << 16) & 0x7FFF0000u, hi = w4[i] & 0x7FFF0000u;
      mx = max(mx, max(lo, hi));
      mn = min(mn, min(lo ? lo : 0xFFFFFFFFu, hi ? hi : 0xFFFFFFFFu));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  // 0x477FE000 = 65504 (fp16's largest), 0x38800000 = 2^-14 (its smallest normal)
  const bool fits = mx <= 0x477FE000u && (mn == 0xFFFFFFFFu || mn >= 0x38800000u);
  const int sh = fits ? 0 : token_shift(mx);
  if (lane == 0) shift[m] = sh;
  const float down = pow2f(-sh);
  uint16_t *out = act16 + (int64_t)m * K;
  for (int k = 8 * (int)lane; k < K; k += 256) {
    const uint4 v = ldg_nc_v4(row + k);
    float f[8];
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(f[e], down);
    *reinterpret_cast<uint4 *>(out + k) = make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]),
                                                     pack_f16x2(f[4], f[5]), pack_f16x2(f[6], f[7]));
  }
}

template <int MODE, bool SF_TMA, int TS>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemv_kernel(const Params p, const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_sf,
                        const uint16_t *__restrict__ act16, const int32_t *__restrict__ act_shift) {
  using C = Cfg<TS>;
  constexpr int kTS = C::kTS, kStages = C::kStages, kKatomBytes = C::kKatomBytes;
  constexpr int kBTile = C::kBTile;
  constexpr size_t kOffB = C::kOffB, kOffPrefix = C::kOffPrefix, kOffStart = C::kOffStart;
  constexpr size_t kOffEid = C::kOffEid, kOffPair = C::kOffPair, kOffShift = C::kOffShift;
  constexpr size_t kOffBar = C::kOffBar, kOffMisc = C::kOffMisc;
  constexpr int kTPW = TS / 8;  // tokens per staging warp: lane i < kTPW holds token warp + 8 i
  // the 128-token form reads converted activations only (the host picks it so)
  static_assert(TS == 64 || MODE == MOE_W4A16, "128-token passes take converted W4A16 rows");
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic (not through an integer), so the
  // compiler still sees shared memory and addresses it as such
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t *btile = smem + kOffB;
  uint32_t *prefix = reinterpret_cast<uint32_t *>(smem + kOffPrefix);
  uint32_t *s_start = reinterpret_cast<uint32_t *>(smem + kOffStart);
  int32_t *s_eid = reinterpret_cast<int32_t *>(smem + kOffEid);
  uint32_t *s_pair = reinterpret_cast<uint32_t *>(smem + kOffPair);
  int32_t *s_shift = reinterpret_cast<int32_t *>(smem + kOffShift);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint64_t *empty = full + kStages;
  uint64_t *a_full = empty + kStages;   // [2]
  uint64_t *a_empty = a_full + 2;       // [2]
  uint64_t *d_full = a_empty + 2;       // [2]
  uint64_t *d_empty = d_full + 2;       // [2]
  uint64_t *mma_drain = d_empty + 2;    // completes once every MMA issued so far is done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 8);

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
  if (warp == 0) build_prefix(prefix, s_start, A, kTS, RB, lane);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], SF_TMA ? 1u : 33u);
      mbar_init(&empty[s], (uint32_t)kDQ);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], (uint32_t)kDQ);
      mbar_init(&a_empty[b], 1u);
      mbar_init(&d_full[b], 1u);
      mbar_init(&d_empty[b], (uint32_t)kDQ);
    }
    mbar_init(mma_drain, 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const uint32_t U = prefix[A];
  uint32_t u_begin, u_end;
  cta_round_range(U, RB, kBlocksPerRound, u_begin, u_end);
  const int nchunks = (K + kKC - 1) / kKC;
  const int64_t sf_row_bytes = K / 16;
  const Meta meta{prefix, s_start, s_eid, N};

  auto wait = [&](uint64_t *bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait_bounded(bar, parity, p.wait_limit_ns)) *abort_flag = 1;
  };

  if (warp == kTmaWarp) {
    // ================================================================ TMA producer
    RoundIter iter{u_begin, u_end, u_begin < u_end ? expert_of_unit(prefix, A, u_begin) : 0, (uint32_t)kTS};
    Round r;
    uint32_t it = 0;
    const uint64_t policy = l2_evict_first_policy();
    if (lane == 0) {
      prefetch_tmap(&tmap_w);
      if (SF_TMA) prefetch_tmap(&tmap_sf);
    }
    uint32_t issued = 0;  // stages filled so far (a prefix of the sequence: an abort is final)
    while (iter.next(meta, RB, r)) {
      for (int c = 0; c < nchunks; ++c, ++it) {
        const int s = (int)(it % kStages);
        wait(&empty[s], ((it / kStages) & 1u) ^ 1u);
        // lane 0's view of the abort flag decides for the whole warp
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) continue;
        issued = it + 1;
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
          if ((sf_row_bytes & 3) == 0) {
            // 4-byte aligned scale rows (K % 64 == 0): asynchronous copies
            for (int row = lane; row < r.nrows; row += 32)
              for (uint32_t q = 0; q < sb; q += 4)
                cp_async4(ssf + row * kSFStride + q, sbase + row * sf_row_bytes + q);
            cp_async_mbar_arrive_noinc(&full[s]);
          } else {
            // K % 64 == 32: rows are 2-byte aligned; plain loads and stores,
            // published by this lane's arrival (release semantics)
            for (int row = lane; row < r.nrows; row += 32)
              for (uint32_t q = 0; q < sb; q += 2)
                *reinterpret_cast<uint16_t *>(ssf + row * kSFStride + q) =
                    __ldg(reinterpret_cast<const uint16_t *>(sbase + row * sf_row_bytes + q));
            mbar_arrive(&full[s]);
          }
        }
      }
    }
    // After an abort, let the copies still in flight land before the CTA
    // exits (bounded again): stage s was filled ceil((issued - s) / kStages) times.
    if (lane == 0 && *abort_flag) {
      for (int s = 0; s < kStages; ++s) {
        const uint32_t fills =
            issued > (uint32_t)s ? (issued - (uint32_t)s + kStages - 1) / kStages : 0u;
        if (fills) mbar_wait_bounded(&full[s], (fills - 1) & 1u, kDrainLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      RoundIter iter{u_begin, u_end, u_begin < u_end ? expert_of_unit(prefix, A, u_begin) : 0, (uint32_t)kTS};
      Round r;
      uint32_t it = 0, rnd = 0;
      while (iter.next(meta, RB, r)) {
        const uint32_t d = rnd & 1u;
        wait(&d_empty[d], ((rnd >> 1) & 1u) ^ 1u);
        tc_fence_after();
        const int nmma = (r.ntok + 15) / 16 * 16;
        const uint32_t idesc = umma_idesc_f16(128, nmma);
        const uint32_t d_t = tbase + kDcol + d * (uint32_t)kTS;
        for (int c = 0; c < nchunks; ++c, ++it) {
          const uint32_t b = it & 1u;
          wait(&a_full[b], (it >> 1) & 1u);
          tc_fence_after();
          const int ksteps = min(kKC, K - c * kKC) / 16;
          if (!*abort_flag) {
            const uint32_t bbase = smem_addr(btile + b * kBTile);
            for (int j = 0; j < ksteps; ++j) {
              const uint64_t bdesc =
                  umma_desc_sw128(bbase + (uint32_t)(j >> 2) * kKatomBytes + (uint32_t)(j & 3) * 32u,
                                  1024u);
              umma_f16_ts(d_t, tbase + kAcol + b * 128u + 8u * (uint32_t)j, bdesc, idesc,
                          (c > 0 || j > 0) ? 1u : 0u);
            }
          }
          umma_commit(&a_empty[b]);
        }
        umma_commit(&d_full[d]);
        ++rnd;
      }
      // no MMA may still read shared or tensor memory when the CTA releases them
      umma_commit(mma_drain);
      mbar_wait_bounded(mma_drain, 0u, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ================================================================ dequant / staging / epilogue
    const int q = warp & 3;     // TMEM lane quarter
    const int h = warp >> 2;    // column half of a chunk
    const int row = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    RoundIter iter{u_begin, u_end, u_begin < u_end ? expert_of_unit(prefix, A, u_begin) : 0, (uint32_t)kTS};
    Round r, rn, rp;  // current, next, previous (pending epilogue)
    bool have = iter.next(meta, RB, r);
    bool have_n = have && iter.next(meta, RB, rn);
    bool ep_pending = false;
    uint32_t it = 0, rnd = 0, rnd_p = 0;
    // token pair ids of the current / next round, one token per lane (lanes <
    // kTPW): lane i of warp w holds token tau = w + 8 i
    uint32_t pair_cur = 0xFFFFFFFFu, pair_nxt = 0xFFFFFFFFu;
    int32_t sh_cur = 0, sh_nxt = 0;  // the same tokens' W4A16 offsets (0 without act16)
    const bool pre = MODE == MOE_W4A16 && act16 != nullptr;  // activations converted already
    auto fetch_pairs = [&](const Round &q_, uint32_t &dst, int32_t &sh) {
      const int tau = warp + 8 * lane;
      dst = (lane < kTPW && tau < q_.ntok) ? p.order[q_.tok0 + tau] : 0xFFFFFFFFu;
      sh = (pre && dst != 0xFFFFFFFFu) ? act_shift[dst / (uint32_t)p.top_k] : 0;
    };
    if (have) fetch_pairs(r, pair_cur, sh_cur);

    // activations of this warp's tokens for one chunk (8 values per lane per token)
    uint4 raw[8];
    auto load_act = [&](uint32_t pairs, int ntok, int c) {
      const int k0 = c * kKC;
      const int kcb = min(kKC, K - k0);
      const bool kv = 8 * lane < kcb;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        raw[i] = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t pr = __shfl_sync(0xffffffffu, pairs, i);
        if (warp + 8 * i < ntok && kv) {
          const int64_t m = (int64_t)(pr / (uint32_t)p.top_k);
          if (MODE == MOE_W4A16) {
            raw[i] = ldg_nc_v4((pre ? act16 : static_cast<const uint16_t *>(p.act)) + m * K + k0 +
                               8 * lane);
          } else {
            const uint8_t *qp = static_cast<const uint8_t *>(p.act) + m * (K / 2);
            raw[i].x = __ldg(reinterpret_cast<const uint32_t *>(qp + (k0 + 8 * lane) / 2));
            raw[i].y = p.sfa[m * (K / 16) + (k0 + 8 * lane) / 16];
          }
        }
      }
    };
    // (128-token passes) the converted rows of this warp's tokens for one chunk,
    // copied straight into B buffer bb: 16 bytes per lane and token
    auto copy_act = [&](uint32_t pairs, int ntok, int c, uint32_t bb) {
      const int k0 = c * kKC;
      const int kcb = min(kKC, K - k0);
      const bool kv = 8 * lane < kcb;
      uint8_t *bt = btile + bb * kBTile;
      const int katom = lane >> 3, cidx = lane & 7;
#pragma unroll
      for (int i = 0; i < kTPW; ++i) {
        const uint32_t pr = __shfl_sync(0xffffffffu, pairs, i);
        const int tau = warp + 8 * i;
        if (tau < ntok && kv)
          cp_async16_zfill(bt + katom * kKatomBytes + tau * 128 + ((cidx ^ (tau & 7)) * 16),
                           act16 + (int64_t)(pr / (uint32_t)p.top_k) * K + k0 + 8 * lane, 16u);
      }
    };
    if constexpr (TS < 128) {
      if (have) load_act(pair_cur, r.ntok, 0);
    } else {
      if (have) copy_act(pair_cur, r.ntok, 0, 0u);  // buffer 0 has no earlier user
    }

    auto epilogue = [&](const Round &er, uint32_t ernd) {
      const uint32_t d = ernd & 1u;
      wait(&d_full[d], (ernd >> 1) & 1u);
      tc_fence_after();
      constexpr int kCols = kTS / 2;  // this warp's token columns: kCols from kCols * h
      const int c0 = kCols * h;
      uint32_t v[kCols];
      const bool cols = c0 < er.ntok && 32 * q < er.nrows;
      if (cols) {
        uint32_t t[kCols / 16][16];
        const uint32_t ta = tbase + lane_base + kDcol + d * (uint32_t)kTS + (uint32_t)c0;
#pragma unroll
        for (int j = 0; j < kCols / 16; ++j) tmem_ld16(ta + 16u * (uint32_t)j, t[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kCols / 16; ++j)
#pragma unroll
          for (int i = 0; i < 16; ++i) v[16 * j + i] = t[j][i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[d]);
      if (cols && !*abort_flag && row < er.nrows) {
        const float gw = p.w_global ? p.w_global[er.e] : 1.0f;
        const float f = __fmul_rn(gw, p.g_a);
        const int n = er.n0 + row;
        const uint32_t *pairs = s_pair + (ernd & 1u) * kTS;
        const int32_t *shifts = s_shift + (ernd & 1u) * kTS;
        const int ncol = min(kCols, er.ntok - c0);
#pragma unroll
        for (int i = 0; i < kCols; ++i) {
          if (i < ncol) {
            const uint32_t pr = pairs[c0 + i];
            float y = __fmul_rn(__uint_as_float(v[i]), f);
            // the token's power of two last (no early overflow, the same
            // rounding as without the offset)
            const int sh = shifts[c0 + i];
            if (sh != 0) y = __fmul_rn(y, pow2f(sh));  // warp-uniform: one column per i
            const __nv_bfloat16 o = __float2bfloat16_rn(y);
            p.out[(int64_t)pr * N + n] = __bfloat16_as_ushort(o);
          }
        }
      }
    };

    while (have) {
      // ---- round start: publish this round's pair ids, fetch the next round's
      named_bar_sync(1, kDQ * 32);
      if (lane < kTPW && warp + 8 * lane < r.ntok) {
        s_pair[(rnd & 1u) * kTS + warp + 8 * lane] = pair_cur;
        s_shift[(rnd & 1u) * kTS + warp + 8 * lane] = sh_cur;
      }
      if (have_n) fetch_pairs(rn, pair_nxt, sh_nxt);
      named_bar_sync(1, kDQ * 32);
      const bool has_rows = 32 * q < r.nrows;

      for (int c = 0; c < nchunks; ++c, ++it) {
        const int s = (int)(it % kStages);
        const uint32_t b = it & 1u;
        const int k0 = c * kKC;
        const int kcb = min(kKC, K - k0);
        // ---- weights of this chunk: this lane's row, columns [128h, 128h + 128)
        wait(&full[s], (it / kStages) & 1u);
        const uint8_t *sw = smem + (size_t)s * kStageBytes;
        const uint8_t *ssf = sw + kStageW;
        uint4 wv[4];
        uint2 sv = make_uint2(0u, 0u);
        if (has_rows) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int ci = 4 * h + jj;  // logical 16-byte chunk of the 128-byte row
            wv[jj] = (128 * h + 32 * jj < kcb)
                         ? *reinterpret_cast<const uint4 *>(sw + row * kWStride + ((ci ^ (row & 7)) * 16))
                         : make_uint4(0u, 0u, 0u, 0u);
          }
          sv = *reinterpret_cast<const uint2 *>(ssf + row * kSFStride + 8 * h);
        }
        // ---- A/B buffer b is free once the MMAs of item it - 2 completed
        wait(&a_empty[b], ((it >> 1) & 1u) ^ 1u);
        tc_fence_after();
        if (has_rows) {
          const uint32_t sc01 = e4m3x2_to_f16x2(sv.x & 0xFFFFu), sc23 = e4m3x2_to_f16x2(sv.x >> 16);
          const uint32_t sc45 = e4m3x2_to_f16x2(sv.y & 0xFFFFu), sc67 = e4m3x2_to_f16x2(sv.y >> 16);
          const uint32_t scs[4] = {sc01, sc23, sc45, sc67};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint32_t rr[16];
            const uint32_t slo = bcast_lo(scs[jj]), shi = bcast_hi(scs[jj]);
            e2m1x8_to_f16x2(wv[jj].x, rr[0], rr[1], rr[2], rr[3]);
            e2m1x8_to_f16x2(wv[jj].y, rr[4], rr[5], rr[6], rr[7]);
            e2m1x8_to_f16x2(wv[jj].z, rr[8], rr[9], rr[10], rr[11]);
            e2m1x8_to_f16x2(wv[jj].w, rr[12], rr[13], rr[14], rr[15]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              rr[i] = hmul2(rr[i], slo);
              rr[8 + i] = hmul2(rr[8 + i], shi);
            }
            tmem_st16(tbase + lane_base + kAcol + b * 128u + 64u * (uint32_t)h + 16u * (uint32_t)jj, rr);
          }
        }
        // ---- activations of this chunk -> fp16 B tile (K-major, 128B swizzle);
        // with 128-token passes it was copied in during the previous item
        uint8_t *bt = btile + b * kBTile;
        unsigned range_bad = 0;
#pragma unroll
        for (int i = 0; i < (TS < 128 ? 8 : 0); ++i) {
          const int tau = warp + 8 * i;
          if (tau >= r.ntok) continue;  // warp-uniform
          uint4 hv;
          if (pre) {
            hv = raw[i];  // fp16 already, scaled by the token's power of two
          } else if (MODE == MOE_W4A16) {
            float f[8];
            f[0] = bf16_lo(raw[i].x); f[1] = bf16_hi(raw[i].x);
            f[2] = bf16_lo(raw[i].y); f[3] = bf16_hi(raw[i].y);
            f[4] = bf16_lo(raw[i].z); f[5] = bf16_hi(raw[i].z);
            f[6] = bf16_lo(raw[i].w); f[7] = bf16_hi(raw[i].w);
#pragma unroll
            for (int e = 0; e < 8; ++e) range_bad |= (fabsf(f[e]) > 65504.0f) ? 1u : 0u;
            hv.x = pack_f16x2(f[0], f[1]);
            hv.y = pack_f16x2(f[2], f[3]);
            hv.z = pack_f16x2(f[4], f[5]);
            hv.w = pack_f16x2(f[6], f[7]);
          } else {
            uint32_t q0, q1, q2, q3;
            e2m1x8_to_f16x2(raw[i].x, q0, q1, q2, q3);
            const uint32_t sc = bcast_lo(e4m3x2_to_f16x2(raw[i].y));
            hv.x = hmul2(q0, sc);
            hv.y = hmul2(q1, sc);
            hv.z = hmul2(q2, sc);
            hv.w = hmul2(q3, sc);
          }
          const int katom = lane >> 3, cidx = lane & 7;
          *reinterpret_cast<uint4 *>(bt + katom * kKatomBytes + tau * 128 + ((cidx ^ (tau & 7)) * 16)) = hv;
        }
        if (MODE == MOE_W4A16 && range_bad) raise_device_error(MOE_DEVERR_ACT_RANGE);
        if constexpr (TS < 128) {
          // prefetch the next chunk's activations (or the next round's first chunk)
          if (c + 1 < nchunks) {
            load_act(pair_cur, r.ntok, c + 1);
          } else if (have_n) {
            load_act(pair_nxt, rn.ntok, 0);
          }
        } else {
          cp_async_wait_all();  // this item's token tile, copied in during the previous item
        }
        // ---- publish A (TMEM) and B (shared memory) of item it; release stage s
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&empty[s]);
          mbar_arrive(&a_full[b]);
        }
        if constexpr (TS >= 128) {
          // the next item's token tile into the other buffer, once the MMAs of
          // item it - 1, its previous user, are done
          const uint32_t bn = (it + 1) & 1u;
          if (it >= 1) wait(&a_empty[bn], ((it - 1) >> 1) & 1u);
          if (!*abort_flag) {
            if (c + 1 < nchunks)
              copy_act(pair_cur, r.ntok, c + 1, bn);
            else if (have_n)
              copy_act(pair_nxt, rn.ntok, 0, bn);
          }
        }
        // ---- the previous round's epilogue overlaps this round's first chunk
        if (c == 0 && ep_pending) {
          epilogue(rp, rnd_p);
          ep_pending = false;
        }
      }
      rp = r;
      rnd_p = rnd;
      ep_pending = true;
      ++rnd;
      r = rn;
      pair_cur = pair_nxt;
      sh_cur = sh_nxt;
      have = have_n;
      have_n = have && iter.next(meta, RB, rn);
    }
    if (ep_pending) epilogue(rp, rnd_p);
    cp_async_wait_all();  // no token-tile copy may still land after the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace tc
}  // namespace gemv
}  // namespace moe
