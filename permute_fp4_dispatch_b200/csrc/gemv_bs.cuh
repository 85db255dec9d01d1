// gemv_bs.cuh -- step 4b, W4A4 on the block-scaled FP4 tensor core.
//
// FlashRT "grouped-moe-gemv" card (Available functions: grouped_w4a4_gemv_bf16;
// hardware list: block-scaled-MMA W4A4).  For each routed pair p with expert e:
//     out[p, n] = bf16( g_w[e] * g_a * sum_k e2m1(xq[m,k]) e4m3(sfa[m,k/16])
//                                       * e2m1(wq[e,n,k]) e4m3(sfw[e,n,k/16]) ).
// Both operands stay in their NVFP4 encoding all the way into the tensor
// core: tcgen05.mma.kind::mxf4nvf4.block_scale with 16-element E4M3 scale
// vectors multiplies the raw E2M1 codes and applies both scale factors, so
// nothing is dequantised on the CUDA cores.
//
// Design (one persistent CTA per SM, 6 warps):
//   * Work units are (active expert a, 128-row block rb, pass p of up to
//     kTS tokens), in that order, so the passes of one row block follow
//     each other and a block's weights are read from HBM once even when its
//     expert holds more tokens than one pass.  The CTAs take equal contiguous
//     ranges of units.  One unit is one MMA tile: M = 128 weight rows (A),
//     N = the pass's tokens rounded up to 16 (B), fp32 D in tensor memory.
//     kTS = 128 with 5 stages in flight, or -- when the experts hold 64
//     tokens or fewer on average -- kTS = 64, whose smaller token tiles leave
//     room for 7 stages (more weight bytes in flight per SM).
//   * warp 0, lane 0: streams the unit's weight codes, 128 rows x 256 codes
//     per stage, with one TMA box (128B swizzle, L2 evict-first; rows past N
//     and codes past K arrive as zeros) into a kStages-deep ring, and -- when
//     the scale rows are whole 16-byte units (K % 256 == 0) -- the stage's
//     weight scales as a second box, row-major;
//   * warps 2-5 (128 threads): per stage, gather the pass's token rows
//     (128 bytes of codes each) into the 128B-swizzled K-major B tile, and
//     the stage's scale factors of both operands into shared memory in the
//     tensor core's 32-row x 16-byte scale layout (the weight scales, when
//     they came by TMA, moved there from the row-major box: one 16-byte
//     load and four 4-byte stores per row), all with cp.async laid
//     out so one warp instruction covers whole rows (no copies for rows the
//     result does not use), arriving on the stage's barrier when the copies
//     land; they also run the epilogue
//     (tensor memory -> scale by g_w * g_a -> bf16 -> out) of the previous
//     unit while the next one streams;
//   * warp 1, lane 0: owns tensor memory; per stage copies the scale
//     factors into it (tcgen05.cp 32x128b, replicated over the four lane
//     quadrants) and issues four kind::mxf4nvf4 MMAs of K = 64, committing
//     to the barrier that frees the stage; D is double-buffered, so a unit's
//     epilogue overlaps the next unit's MMAs.
//   * Every wait is bounded; an expired wait raises MOE_DEVERR_WAIT_TIMEOUT,
//     the roles stop issuing, wait (bounded) for their copies and MMAs in
//     flight, and the CTA releases tensor memory and returns.
#pragma once
#include "gemv_common.cuh"

namespace moe {
namespace gemv {
namespace bs {

constexpr int kProdWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSW0 = 2;                   // first staging / epilogue warp
constexpr int kSWThreads = 4 * 32;
constexpr int kThreads = 2 * 32 + kSWThreads;
constexpr int kKC = 256;                  // codes per stage: 128 bytes of each row
constexpr int kKSteps = kKC / 64;         // MMAs (K = 64) per stage
constexpr int kATile = 128 * 128;         // weight tile: 128 rows x 128 bytes
constexpr int kSFStep = 512;              // one operand's scales for one MMA: 32 rows x 16 B
constexpr int kSFBytes = kKSteps * kSFStep;
constexpr int kSFRaw = 128 * (kKC / 16);  // one stage's weight scales, row-major
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDcol = 0;             // D: two buffers of kTS columns

// Sizes for TS tokens per pass: 128 (many tokens per expert), or 64 -- a
// smaller token tile leaves room for two more stages, i.e. more weight
// bytes in flight per SM, which experts with few tokens need.
template <int TS, bool SFT>
struct Cfg {
  static constexpr int kTS = TS;                        // tokens per pass (MMA N <= TS)
  static constexpr int kStages = TS >= 128 ? 5 : 7;
  static constexpr int kBTile = TS * 128;               // token tile: TS rows x 128 bytes
  // weight tile, token tile, both operands' scales in the tensor core's layout,
  // and (SFT) the weight scales as the TMA lands them (128 rows x 16 bytes)
  static constexpr int kSFRawBytes = SFT ? kSFRaw : 0;
  static constexpr int kStageBytes = kATile + kBTile + 2 * kSFBytes + kSFRawBytes;
  static constexpr uint32_t kSFcol = 2 * TS;            // per stage: 16 columns of A scales, 16 of B
  static constexpr size_t kOffStart = (size_t)kStages * kStageBytes;
  static constexpr size_t kOffEid = kOffStart + (kMaxExperts + 4) * 4;
  static constexpr size_t kOffPrefix = kOffEid + (kMaxExperts + 4) * 4;
  static constexpr size_t kOffPair = kOffPrefix + (kMaxExperts + 4) * 4;  // [2][kTS] pair ids
  static constexpr size_t kOffBar = kOffPair + 2 * TS * 4;
  static constexpr int kNumBars = 3 * kStages + 5;
  static constexpr size_t kOffMisc = kOffBar + kNumBars * 8;             // tmem slot, abort flag
  static constexpr size_t kSmemBytes = kOffMisc + 16 + 1024;             // + alignment slack
  static_assert(kSFcol + kStages * 32 <= kTmemCols, "tensor memory columns");
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct Unit {
  int e;          // expert id
  uint32_t tok0;  // first position of the pass in token_expert_order
  int ntok;       // tokens of the pass
  int n0;         // first weight row of the block
};

// Walks a CTA's unit range in order; unit u of active expert a with c pairs
// (P = ceil(c / kTS) passes) is block v / P, pass v % P, v = u - prefix[a].
template <int kTS>
struct UnitWalk {
  uint32_t u, u_end;
  int a;
  __device__ __forceinline__ bool next(const uint32_t *prefix, const uint32_t *start,
                                       const int32_t *eid, Unit &r) {
    if (u >= u_end) return false;
    while (u >= prefix[a + 1]) ++a;
    const uint32_t v = u - prefix[a];
    const uint32_t c = start[a + 1] - start[a];
    const uint32_t P = (c + kTS - 1) / kTS;
    const uint32_t pass = v % P;
    r.e = eid[a];
    r.tok0 = start[a] + pass * kTS;
    r.ntok = (int)min((uint32_t)kTS, c - pass * kTS);
    r.n0 = (int)(v / P) * 128;
    ++u;
    return true;
  }
};

// SFT: the weight scales arrive by TMA with the weight tile (row-major) and
// the staging warps move them into the tensor core's scale layout (K % 256
// == 0: 16-byte scale rows); otherwise they are gathered 4 bytes at a time.
template <int TS, bool SFT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemv_bs_kernel(const Params p, const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_sfw) {
  using C = Cfg<TS, SFT>;
  constexpr int kTS = C::kTS, kStages = C::kStages, kBTile = C::kBTile;
  constexpr int kStageBytes = C::kStageBytes;
  constexpr uint32_t kSFcol = C::kSFcol;
  constexpr size_t kOffStart = C::kOffStart, kOffEid = C::kOffEid, kOffPrefix = C::kOffPrefix;
  constexpr size_t kOffPair = C::kOffPair, kOffBar = C::kOffBar, kOffMisc = C::kOffMisc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint32_t *s_start = reinterpret_cast<uint32_t *>(smem + kOffStart);
  int32_t *s_eid = reinterpret_cast<int32_t *>(smem + kOffEid);
  uint32_t *prefix = reinterpret_cast<uint32_t *>(smem + kOffPrefix);
  uint32_t *s_pair = reinterpret_cast<uint32_t *>(smem + kOffPair);
  uint64_t *a_full = reinterpret_cast<uint64_t *>(smem + kOffBar);  // weight tile landed
  uint64_t *b_full = a_full + kStages;   // token tile and scales landed
  uint64_t *empty = b_full + kStages;    // the stage's MMAs are done
  uint64_t *d_full = empty + kStages;    // [2] a unit's D is complete
  uint64_t *d_empty = d_full + 2;        // [2] a unit's D has been read out
  uint64_t *mma_drain = d_empty + 2;     // completes once every MMA issued so far is done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = (int)lane_id();
  // set-up that reads no input runs before the wait for the previous grid
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&a_full[s], 1u);
      mbar_init(&b_full[s], (uint32_t)kSWThreads);
      mbar_init(&empty[s], 1u);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&d_full[b], 1u);
      mbar_init(&d_empty[b], 4u);
    }
    mbar_init(mma_drain, 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProdWarp && lane == 0) {
    prefetch_tmap(&tmap_w);
    if (SFT) prefetch_tmap(&tmap_sfw);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  pdl_wait();
  pdl_launch_dependents();

  const int N = p.N, K = p.K;
  const int RB = (N + 127) / 128;
  const uint32_t A = p.stats[1];
  for (uint32_t i = threadIdx.x; i <= A; i += blockDim.x) {
    s_start[i] = p.start[i];
    if (i < A) s_eid[i] = p.eids[i];
  }
  __syncthreads();
  if (warp == 0) build_prefix(prefix, s_start, A, (uint32_t)kTS, RB, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t U = prefix[A];
  const uint32_t u0 = muldiv(U, blockIdx.x, gridDim.x);
  const uint32_t u1 = muldiv(U, blockIdx.x + 1, gridDim.x);
  const int nst = (K + kKC - 1) / kKC;
  const int a0 = u0 < u1 ? expert_of_unit(prefix, A, u0) : 0;

  auto wait = [&](uint64_t *bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait_bounded(bar, parity, p.wait_limit_ns)) *abort_flag = 1;
  };
  auto stage = [&](int s) { return smem + (size_t)s * kStageBytes; };

  if (warp == kProdWarp) {
    // ================================================================ weight tiles (TMA)
    if (lane == 0) {
      const uint64_t policy = l2_evict_first_policy();
      UnitWalk<kTS> walk{u0, u1, a0};
      Unit r;
      uint32_t it = 0, issued = 0;
      while (!*abort_flag && walk.next(prefix, s_start, s_eid, r)) {
        for (int c = 0; c < nst; ++c, ++it) {
          const int s = (int)(it % kStages);
          wait(&empty[s], ((it / kStages) & 1u) ^ 1u);
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&a_full[s], (uint32_t)(kATile + (SFT ? kSFRaw : 0)));
          tma_load_3d(stage(s), &tmap_w, c * (kKC / 2), r.n0, r.e, &a_full[s], policy);
          if (SFT)  // 128 rows x the stage's 16 scale bytes; rows past N, columns past K: zeros
            tma_load_3d(stage(s) + kStageBytes - kSFRaw, &tmap_sfw, c * (kKC / 16), r.n0, r.e,
                        &a_full[s], policy);
          issued = it + 1;
        }
      }
      // after an abort, let the copies still in flight land (bounded)
      if (*abort_flag) {
        for (int s = 0; s < kStages; ++s) {
          const uint32_t fills =
              issued > (uint32_t)s ? (issued - (uint32_t)s + kStages - 1) / kStages : 0u;
          if (fills) mbar_wait_bounded(&a_full[s], (fills - 1) & 1u, kDrainLimitNs);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      UnitWalk<kTS> walk{u0, u1, a0};
      Unit r;
      uint32_t it = 0, rnd = 0;
      while (walk.next(prefix, s_start, s_eid, r)) {
        const uint32_t d = rnd & 1u;
        wait(&d_empty[d], ((rnd >> 1) & 1u) ^ 1u);
        tc_fence_after();
        const uint32_t idesc = umma_idesc_nvf4(128, (r.ntok + 15) & ~15);
        const uint32_t d_t = tbase + kDcol + d * (uint32_t)kTS;
        for (int c = 0; c < nst; ++c, ++it) {
          const int s = (int)(it % kStages);
          wait(&a_full[s], (it / kStages) & 1u);
          wait(&b_full[s], (it / kStages) & 1u);
          fence_proxy_async_smem();  // token tile and scales were written by cp.async
          tc_fence_after();
          if (!*abort_flag) {
            const uint8_t *st = stage(s);
            const uint32_t a_addr = smem_addr(st), b_addr = a_addr + kATile;
            const uint32_t sfa_addr = b_addr + kBTile, sfb_addr = sfa_addr + kSFBytes;
            const uint32_t sf_t = tbase + kSFcol + (uint32_t)s * 32u;
            const int ksteps = min(kKSteps, (K - c * kKC) / 64);
            for (int kk = 0; kk < ksteps; ++kk) {
              tmem_cp_32x128b_x4(sf_t + 4u * kk, smem_desc_interleave(sfa_addr + kk * kSFStep, 128));
              tmem_cp_32x128b_x4(sf_t + 16u + 4u * kk,
                                 smem_desc_interleave(sfb_addr + kk * kSFStep, 128));
            }
            for (int kk = 0; kk < ksteps; ++kk)
              umma_nvf4_ss(d_t, umma_desc_sw128(a_addr + 32u * kk, 1024u),
                           umma_desc_sw128(b_addr + 32u * kk, 1024u), idesc, sf_t + 4u * kk,
                           sf_t + 16u + 4u * kk, (c > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&d_full[d]);
        ++rnd;
      }
      // no MMA or scale copy may still use shared or tensor memory when the CTA releases them
      umma_commit(mma_drain);
      mbar_wait_bounded(mma_drain, 0u, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ================================================================ token tiles, scales, epilogue
    const int t = (int)threadIdx.x - kSW0 * 32;  // 0 .. 127
    const int q = warp & 3;                       // the TMEM lane quadrant this warp may access
    const int64_t xrow = K / 2, sfrow = K / 16;
    const uint8_t *xq = static_cast<const uint8_t *>(p.act);
    UnitWalk<kTS> walk{u0, u1, a0};
    Unit r, rp;
    bool have = walk.next(prefix, s_start, s_eid, r), pending = false;
    uint32_t it = 0, rnd = 0, rnd_p = 0;

    auto epilogue = [&](const Unit &er, uint32_t ernd) {
      const uint32_t d = ernd & 1u;
      wait(&d_full[d], (ernd >> 1) & 1u);
      tc_fence_after();
      const int n = er.n0 + 32 * q + lane;
      const bool ok = !*abort_flag && n < N;
      const float f = __fmul_rn(p.w_global ? __ldg(p.w_global + er.e) : 1.0f, p.g_a);
      const uint32_t *pairs = s_pair + (ernd & 1u) * kTS;
      for (int c0 = 0; c0 < er.ntok; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tbase + ((uint32_t)(32 * q) << 16) + kDcol + d * (uint32_t)kTS + (uint32_t)c0, v);
        tmem_wait_ld();
        if (ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (c0 + j < er.ntok) {
              const __nv_bfloat16 o = __float2bfloat16_rn(__uint_as_float(v[j]) * f);
              p.out[(int64_t)pairs[c0 + j] * N + n] = __bfloat16_as_ushort(o);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[d]);
    };

    while (have) {
      named_bar_sync(1, kSWThreads);  // earlier readers of this pair buffer are done
      uint32_t *pairs = s_pair + (rnd & 1u) * kTS;
      if (t < r.ntok) pairs[t] = __ldg(p.order + r.tok0 + t);
      named_bar_sync(1, kSWThreads);
      // Copies are laid out so that a warp instruction covers whole rows: 8
      // lanes per 128-byte token row (4 rows per instruction), 4 lanes per
      // row's 16 scale bytes of the stage (8 rows per instruction).  Rows the
      // MMA result does not use -- tokens past the pass, weight rows past N --
      // are not copied: D row i depends only on A row i, column j only on B row j.
      const int bj = t & 7, bt0 = t >> 3;        // B: chunk bj of token bt0 + 16 * i
      const int skk = t & 3, sr0 = t >> 2;       // scales: word skk of row sr0 + 32 * i
      // this thread's source rows for the whole unit (token rows of x, rows of
      // the weight scales); a row the unit does not use gets offset -1
      int64_t brow[kTS / 16], arow[4], srow[4];
#pragma unroll
      for (int i = 0; i < kTS / 16; ++i) {
        const int tok = bt0 + 16 * i;
        brow[i] = tok < r.ntok ? (int64_t)(pairs[tok] / (uint32_t)p.top_k) * xrow : -1;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = sr0 + 32 * i;
        arow[i] = r.n0 + row < N ? ((int64_t)r.e * N + r.n0 + row) * sfrow : -1;
        srow[i] = row < r.ntok ? (int64_t)(pairs[row] / (uint32_t)p.top_k) * sfrow : -1;
      }
      for (int c = 0; c < nst; ++c, ++it) {
        const int s = (int)(it % kStages);
        wait(&empty[s], ((it / kStages) & 1u) ^ 1u);
        if (!*abort_flag) {
          uint8_t *bt = stage(s) + kATile;
          uint8_t *sfa_s = bt + kBTile, *sfb_s = sfa_s + kSFBytes;
          const int kb0 = c * (kKC / 2);
          const bool bchunk = kb0 + 16 * (bj + 1) <= xrow;
#pragma unroll
          for (int i = 0; i < kTS / 16; ++i) {
            const int tok = bt0 + 16 * i;
            if (brow[i] >= 0 && bchunk)
              cp_async16_zfill(bt + tok * 128 + ((bj ^ (tok & 7)) << 4),
                               xq + brow[i] + kb0 + 16 * bj, 16u);
          }
          const int kc = c * (kKC / 16) + 4 * skk;  // first scale byte of MMA skk of the stage
          if (kc + 4 <= sfrow) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int off = skk * kSFStep + sr0 * 16 + i * 4;  // row sr0 + 32 i of the layout
              if (!SFT && arow[i] >= 0) cp_async4_zfill(sfa_s + off, p.sfw + arow[i] + kc, 4u);
              if (srow[i] >= 0) cp_async4_zfill(sfb_s + off, p.sfa + srow[i] + kc, 4u);
            }
          }
          if (SFT) {
            // weight row t's 16 scale bytes (one word per MMA k-step), from the
            // TMA's row-major box into row t of each k-step's 32 x 16-byte atom
            wait(&a_full[s], (it / kStages) & 1u);
            if (!*abort_flag) {
              const uint4 v = *reinterpret_cast<const uint4 *>(stage(s) + kStageBytes - kSFRaw + t * 16);
              const int off = (t & 31) * 16 + (t >> 5) * 4;
              *reinterpret_cast<uint32_t *>(sfa_s + 0 * kSFStep + off) = v.x;
              *reinterpret_cast<uint32_t *>(sfa_s + 1 * kSFStep + off) = v.y;
              *reinterpret_cast<uint32_t *>(sfa_s + 2 * kSFStep + off) = v.z;
              *reinterpret_cast<uint32_t *>(sfa_s + 3 * kSFStep + off) = v.w;
            }
            fence_proxy_async_smem();  // plain stores, read by tcgen05.cp
          }
        }
        cp_async_mbar_arrive_noinc(&b_full[s]);
        // the previous unit's epilogue overlaps this unit's first stage
        if (c == 0 && pending) {
          epilogue(rp, rnd_p);
          pending = false;
        }
      }
      rp = r;
      rnd_p = rnd;
      pending = true;
      ++rnd;
      have = walk.next(prefix, s_start, s_eid, r);
    }
    if (pending) epilogue(rp, rnd_p);
    cp_async_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace bs
}  // namespace gemv
}  // namespace moe
