// create_indices.cuh -- step 2: group (token, slot) pairs by expert.
//
// MAX "moe_create_indices": histogram of expert ids -> CSR offsets ->
// scatter of token_expert_order / restore_token_order, plus the ascending
// list of active experts and {max count, active experts}.  The page's design
// is one CTA with a shared-memory histogram; here the same counting sort is
// built from per-warp histograms so that the scatter is stable (ascending
// pair index within an expert) without any serial pass:
//
//   pass 1  each warp counts its contiguous slice of slots with warp-
//           aggregated increments (__match_any_sync) into a private row of a
//           [32][E] shared histogram;
//   scan    per expert, an exclusive prefix over the 32 warps (so warp w's
//           pairs of expert e come after warps < w), then a block-wide scan
//           over experts gives the CSR base of each expert;
//   pass 2  each warp re-walks its slice in order; a pair's position is
//           base[e] + warp prefix + its rank among equal ids in the 32-slot
//           step (popc of the match mask below the lane).
//
// Up to kSmallSlots slots this runs as one CTA.  Larger inputs are tiled
// (kTileSlots per CTA): a histogram kernel writes per-tile counts, the last
// CTA to finish (ticket from atomicAdd, no waiting) turns them into per-tile
// bases, and a scatter kernel repeats pass 2 per tile.  Nothing spins.
#pragma once
#include "common.cuh"

namespace moe {
namespace idx {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int64_t kSmallSlots = 16384;     // one-CTA path up to this many slots
constexpr int64_t kTileSlots = 8192;       // slots per CTA in the tiled path
constexpr size_t kWsHeader = 256;          // ticket counter (+ padding)

__host__ __device__ inline size_t smem_bytes(int E) {
  // [32][E] u16 warp histograms, cnt[E], off[E], 64 scratch words
  return ((size_t)kWarps * E * 2 + 15) / 16 * 16 + (size_t)E * 8 + 64 * 4;
}

struct Smem {
  uint16_t *whist;
  uint32_t *cnt;
  uint32_t *off;
  uint32_t *scratch;
};

__device__ __forceinline__ Smem carve(uint8_t *base, int E) {
  Smem s;
  s.whist = reinterpret_cast<uint16_t *>(base);
  s.cnt = reinterpret_cast<uint32_t *>(base + ((size_t)kWarps * E * 2 + 15) / 16 * 16);
  s.off = s.cnt + E;
  s.scratch = s.off + E;
  return s;
}

__device__ __forceinline__ int slot_key(const int64_t *ids, int64_t p, int64_t hi, int E) {
  if (p >= hi) return -1;
  const int64_t id = ids[p];
  return (id >= 0 && id < E) ? static_cast<int>(id) : -1;
}

// Zero the warp histograms.
__device__ __forceinline__ void zero_whist(const Smem &s, int E) {
  uint32_t *w = reinterpret_cast<uint32_t *>(s.whist);
  for (int i = threadIdx.x; i < kWarps * E / 2; i += blockDim.x) w[i] = 0u;
  if ((E & 1) && threadIdx.x == 0) s.whist[kWarps * E - 1] = 0;
}

// Pass 1 over slots [lo, hi) of this warp.
__device__ __forceinline__ void warp_count(const int64_t *ids, int64_t lo, int64_t hi, int E,
                                           uint16_t *my_hist) {
  const unsigned lane = lane_id();
  for (int64_t b = lo; b < hi; b += 32) {
    const int key = slot_key(ids, b + lane, hi, E);
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == (unsigned)(__ffs(peers) - 1))
      my_hist[key] = (uint16_t)(my_hist[key] + __popc(peers));
  }
}

// Per expert: exclusive prefix across warps (in place); returns totals in cnt.
__device__ __forceinline__ void warp_prefix(const Smem &s, int E) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    uint32_t run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t c = s.whist[w * E + e];
      s.whist[w * E + e] = (uint16_t)run;
      run += c;
    }
    s.cnt[e] = run;
  }
}

// Pass 2: stable scatter of this warp's slots; base[e] = s.off[e] + warp prefix.
__device__ __forceinline__ void warp_scatter(const int64_t *ids, int64_t lo, int64_t hi, int E,
                                             const Smem &s, uint16_t *my_hist,
                                             uint32_t *order, uint32_t *restore) {
  const unsigned lane = lane_id();
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t b = lo; b < hi; b += 32) {
    const int64_t p = b + lane;
    const int key = slot_key(ids, p, hi, E);
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (key >= 0) {
      const uint32_t dest = s.off[key] + my_hist[key] + __popc(peers & lt);
      order[dest] = static_cast<uint32_t>(p);
      restore[p] = dest;
    } else if (p < hi) {
      restore[p] = 0xFFFFFFFFu;
    }
    __syncwarp();
    if (key >= 0 && lane == (unsigned)(__ffs(peers) - 1))
      my_hist[key] = (uint16_t)(my_hist[key] + __popc(peers));
    __syncwarp();
  }
}

// From dense per-expert totals s.cnt: s.off = dense exclusive offsets, and the
// compacted outputs.  Requires blockDim.x >= E.  Returns R (routed pairs).
__device__ __forceinline__ uint32_t finalize(const Smem &s, int E, uint32_t *start,
                                             int32_t *expert_ids, uint32_t *stats,
                                             uint32_t *scales_offset) {
  const int e = threadIdx.x;
  const uint32_t c = e < E ? s.cnt[e] : 0u;
  uint32_t A, R, P;
  const uint32_t pos = block_exclusive_scan(c > 0 ? 1u : 0u, s.scratch, &A);
  const uint32_t o = block_exclusive_scan(c, s.scratch, &R);
  const uint32_t padded = (c + 127u) / 128u * 128u;
  const uint32_t po = block_exclusive_scan(padded, s.scratch, &P);
  const uint32_t mx = block_max(c, s.scratch);
  if (e < E) {
    s.off[e] = o;
    if (c > 0) {
      expert_ids[pos] = e;
      start[pos] = o;
      if (scales_offset) scales_offset[pos] = po;
    }
  }
  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    if (i >= (int)A) {
      if (i < E) expert_ids[i] = -1;
      start[i] = R;
      if (scales_offset) scales_offset[i] = P;
    }
  }
  if (threadIdx.x == 0) {
    stats[0] = mx;
    stats[1] = A;
  }
  __syncthreads();
  return R;
}

__device__ __forceinline__ void fill_order_tail(uint32_t *order, uint32_t R, int64_t S,
                                                int64_t tid, int64_t nthreads) {
  for (int64_t i = R + tid; i < S; i += nthreads) order[i] = 0xFFFFFFFFu;
}

// ---------------------------------------------------------------- one-CTA path
__global__ void __launch_bounds__(kThreads, 1)
    create_indices_small_kernel(const int64_t *__restrict__ ids, int64_t S, int E,
                                uint32_t *__restrict__ order, uint32_t *__restrict__ start,
                                uint32_t *__restrict__ restore, int32_t *__restrict__ expert_ids,
                                uint32_t *__restrict__ stats, uint32_t *__restrict__ scales_offset) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const Smem s = carve(smem_raw, E);
  const int warp = threadIdx.x >> 5;
  const int64_t per_warp = (S + kWarps - 1) / kWarps;
  const int64_t lo = warp * per_warp;
  const int64_t hi = lo + per_warp < S ? lo + per_warp : S;
  uint16_t *my_hist = s.whist + warp * E;

  zero_whist(s, E);
  __syncthreads();
  warp_count(ids, lo, hi, E, my_hist);
  __syncthreads();
  warp_prefix(s, E);
  __syncthreads();
  const uint32_t R = finalize(s, E, start, expert_ids, stats, scales_offset);
  warp_scatter(ids, lo, hi, E, s, my_hist, order, restore);
  fill_order_tail(order, R, S, threadIdx.x, blockDim.x);
}

// ---------------------------------------------------------------- tiled path
// Kernel 1: per-tile histogram into ws_tiles[t][E]; the last CTA converts the
// tiles into per-tile bases (in place) and writes the compacted outputs.
__global__ void __launch_bounds__(kThreads, 1)
    create_indices_hist_kernel(const int64_t *__restrict__ ids, int64_t S, int E,
                               uint32_t *__restrict__ order, uint32_t *__restrict__ start,
                               int32_t *__restrict__ expert_ids, uint32_t *__restrict__ stats,
                               uint32_t *__restrict__ scales_offset, uint32_t *ws_ticket,
                               uint32_t *ws_tiles) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ uint32_t is_last;
  const Smem s = carve(smem_raw, E);
  const int warp = threadIdx.x >> 5;
  const int T = gridDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * kTileSlots;
  const int64_t t1 = t0 + kTileSlots < S ? t0 + kTileSlots : S;
  const int64_t per_warp = kTileSlots / kWarps;
  const int64_t lo = t0 + warp * per_warp < t1 ? t0 + warp * per_warp : t1;
  const int64_t hi = lo + per_warp < t1 ? lo + per_warp : t1;

  zero_whist(s, E);
  __syncthreads();
  warp_count(ids, lo, hi, E, s.whist + warp * E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    uint32_t c = 0;
    for (int w = 0; w < kWarps; ++w) c += s.whist[w * E + e];
    ws_tiles[(size_t)blockIdx.x * E + e] = c;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(ws_ticket, 1u) == (uint32_t)(T - 1)) ? 1u : 0u;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // last CTA: totals, compaction, per-tile bases
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    uint32_t c = 0;
    for (int t = 0; t < T; ++t) c += __ldcg(ws_tiles + (size_t)t * E + e);
    s.cnt[e] = c;
  }
  __syncthreads();
  const uint32_t R = finalize(s, E, start, expert_ids, stats, scales_offset);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    uint32_t run = s.off[e];
    for (int t = 0; t < T; ++t) {
      const uint32_t c = __ldcg(ws_tiles + (size_t)t * E + e);
      ws_tiles[(size_t)t * E + e] = run;
      run += c;
    }
  }
  fill_order_tail(order, R, S, threadIdx.x, blockDim.x);
  if (threadIdx.x == 0) *ws_ticket = 0u;  // ready for the next call
}

// Kernel 2: per-tile stable scatter from the bases written by kernel 1.
__global__ void __launch_bounds__(kThreads, 1)
    create_indices_scatter_kernel(const int64_t *__restrict__ ids, int64_t S, int E,
                                  uint32_t *__restrict__ order, uint32_t *__restrict__ restore,
                                  const uint32_t *__restrict__ ws_tiles) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const Smem s = carve(smem_raw, E);
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kTileSlots;
  const int64_t t1 = t0 + kTileSlots < S ? t0 + kTileSlots : S;
  const int64_t per_warp = kTileSlots / kWarps;
  const int64_t lo = t0 + warp * per_warp < t1 ? t0 + warp * per_warp : t1;
  const int64_t hi = lo + per_warp < t1 ? lo + per_warp : t1;
  uint16_t *my_hist = s.whist + warp * E;

  zero_whist(s, E);
  __syncthreads();
  warp_count(ids, lo, hi, E, my_hist);
  __syncthreads();
  warp_prefix(s, E);
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    s.off[e] = ws_tiles[(size_t)blockIdx.x * E + e];
  __syncthreads();
  warp_scatter(ids, lo, hi, E, s, my_hist, order, restore);
}

// ---------------------------------------------------------------- steps 1 + 2 fused
// Up to kTinySlots slots: one CTA of kThreads threads, one slot per thread.
// Thread p applies the step-1 mask to its slot (rows with
// row + tp_rank * N >= *real_token_count are written back as -1), keeps the
// resulting id in a register from its single load to the scatter, and the
// grouping then follows the same counting sort as above with the cross-warp
// prefix done by warp shuffles (experts striped over warps, one lane per
// source warp) and the CSR compaction done in one combined block scan.
constexpr int kTinySlots = kThreads;

__host__ __device__ inline int tiny_hist_stride(int E) { return ((E + 1) / 2 | 1) * 2; }

__host__ __device__ inline size_t tiny_smem_bytes(int E) {
  return ((size_t)kWarps * tiny_hist_stride(E) * 2 + 15) / 16 * 16 + (size_t)E * 8;
}

__global__ void __launch_bounds__(kThreads, 1)
    mask_create_indices_tiny_kernel(int64_t *__restrict__ ids, int32_t N, int32_t top_k,
                                    const int32_t *__restrict__ real_count, int32_t tp_rank,
                                    int E, uint32_t *__restrict__ order,
                                    uint32_t *__restrict__ start, uint32_t *__restrict__ restore,
                                    int32_t *__restrict__ expert_ids,
                                    uint32_t *__restrict__ stats,
                                    uint32_t *__restrict__ scales_offset) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int WS = tiny_hist_stride(E);
  uint16_t *whist = reinterpret_cast<uint16_t *>(smem_raw);
  uint32_t *cnt = reinterpret_cast<uint32_t *>(smem_raw +
                                               ((size_t)kWarps * WS * 2 + 15) / 16 * 16);
  uint32_t *off = cnt + E;
  __shared__ uint32_t wsum[4][kWarps];
  __shared__ uint32_t totals[4];
  const int p = threadIdx.x, warp = p >> 5, lane = p & 31;
  const int S = N * top_k;
  const unsigned lt = (1u << lane) - 1u;

  // step 1 + key: one load per slot, issued together with the count's
  int key = -1;
  const int64_t id = p < S ? ids[p] : -1;
  const int64_t real = *real_count;
  if (p < S) {
    const int row = p / top_k;
    if ((int64_t)row + (int64_t)tp_rank * N >= real) {
      ids[p] = -1;
    } else {
      key = (id >= 0 && id < E) ? (int)id : -1;
    }
  }
  for (int i = p; i < kWarps * WS; i += kThreads) whist[i] = 0;
  __syncthreads();
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  if (key >= 0 && lane == __ffs(peers) - 1) whist[warp * WS + key] = (uint16_t)__popc(peers);
  __syncthreads();
  // per expert: exclusive prefix over the 32 warps (lane = source warp)
  for (int e = warp; e < E; e += kWarps) {
    const uint32_t c = whist[lane * WS + e];
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    whist[lane * WS + e] = (uint16_t)(x - c);
    if (lane == 31) cnt[e] = x;
  }
  __syncthreads();
  // CSR over experts: one block scan of (active flag, count, count padded to 128) and a max
  const uint32_t c = p < E ? cnt[p] : 0u;
  uint32_t v0 = c > 0 ? 1u : 0u, v1 = c, v2 = (c + 127u) / 128u * 128u, mx = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y0 = __shfl_up_sync(0xffffffffu, v0, o);
    const uint32_t y1 = __shfl_up_sync(0xffffffffu, v1, o);
    const uint32_t y2 = __shfl_up_sync(0xffffffffu, v2, o);
    if (lane >= o) { v0 += y0; v1 += y1; v2 += y2; }
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 31) {
    wsum[0][warp] = v0;
    wsum[1][warp] = v1;
    wsum[2][warp] = v2;
    wsum[3][warp] = mx;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = wsum[0][lane], r = wsum[1][lane], q = wsum[2][lane], m = wsum[3][lane];
    const uint32_t a0 = a, r0 = r, q0 = q;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ya = __shfl_up_sync(0xffffffffu, a, o);
      const uint32_t yr = __shfl_up_sync(0xffffffffu, r, o);
      const uint32_t yq = __shfl_up_sync(0xffffffffu, q, o);
      if (lane >= o) { a += ya; r += yr; q += yq; }
      m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    wsum[0][lane] = a - a0;
    wsum[1][lane] = r - r0;
    wsum[2][lane] = q - q0;
    if (lane == 31) {
      totals[0] = a;
      totals[1] = r;
      totals[2] = q;
      totals[3] = m;
    }
  }
  __syncthreads();
  const uint32_t A = totals[0], R = totals[1], P = totals[2];
  if (p < E) {
    const uint32_t pos = wsum[0][warp] + v0 - (c > 0 ? 1u : 0u);
    const uint32_t o = wsum[1][warp] + v1 - c;
    off[p] = o;
    if (c > 0) {
      expert_ids[pos] = p;
      start[pos] = o;
      if (scales_offset) scales_offset[pos] = wsum[2][warp] + v2 - (c + 127u) / 128u * 128u;
    }
  }
  for (int i = (int)A + p; i <= E; i += kThreads) {  // entries [A, E] (E may equal kThreads)
    if (i < E) expert_ids[i] = -1;
    start[i] = R;
    if (scales_offset) scales_offset[i] = P;
  }
  if (p == 0) {
    stats[0] = totals[3];
    stats[1] = A;
  }
  __syncthreads();
  // stable scatter
  if (key >= 0) {
    const uint32_t dest = off[key] + whist[warp * WS + key] + __popc(peers & lt);
    order[dest] = (uint32_t)p;
    restore[p] = dest;
  } else if (p < S) {
    restore[p] = 0xFFFFFFFFu;
  }
  if (p >= (int)R && p < S) order[p] = 0xFFFFFFFFu;
}

}  // namespace idx
}  // namespace moe
