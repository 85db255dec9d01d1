// moe_route.cu -- C ABI of the MoE token-routing library (see
// include/moe_route.h for the contract of every entry point).
//
// Host side of each call: validate arguments, check the device is sm_100,
// choose the kernel variant and launch configuration, enqueue on the
// caller's stream.  No allocation, no synchronisation (except in
// moe_get_device_error).
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "combine.cuh"
#include "common.cuh"
#include "create_indices.cuh"
#include "dispatch_mxfp4.cuh"
#include "dispatch_quant.cuh"
#include "gemv_bs.cuh"
#include "gemv_mma.cuh"
#include "gemv_tc.cuh"
#include "mask.cuh"
#include "quant_nvfp4.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int checked = 0;
  int supported = 0;
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Current device must be sm_100 (B200 class).  The forced-architecture
// override exists for host-side tests of the rejection path.
moe_status_t check_device(int *sms = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    const char *force = std::getenv("MOE_FORCE_ARCH");
    if (force && *force) {
      major = std::atoi(force) / 10;
      minor = std::atoi(force) % 10;
    }
    d.supported = (major == 10 && minor == 0);
    d.sms = sms;
    d.checked = 1;
  }
  if (!d.supported) return MOE_ERR_UNSUPPORTED_ARCH;
  if (sms) *sms = d.sms;
  return MOE_OK;
}

moe_status_t launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <typename Kernel>
moe_status_t set_smem(Kernel k, size_t bytes) {
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Launch with programmatic stream serialization: when the previous work in
// the stream is a kernel, this grid may be scheduled before that kernel
// finishes; the kernel's pdl_wait() holds it until the predecessor's writes
// are visible.  Used for the kernels that call pdl_wait() first thing.
template <typename... KArgs, typename... Args>
moe_status_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int64_t tiles_for(int64_t S) { return (S + moe::idx::kTileSlots - 1) / moe::idx::kTileSlots; }

// ---------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 3-D uint8 map over [E][rows][cols] (cols innermost) with a box of
// box_cols x box_rows x 1.
bool encode_u8_3d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t E,
                  uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cols, rows, E};
  const cuuint64_t strides[2] = {cols, cols * rows};
  const cuuint32_t box[3] = {box_cols, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D uint32 map over the codes of [E][N][K/256 lines][32 words of a 128-byte
// line]; box = `rows` rows x `lines` lines, 128-byte swizzle.  Needs K % 256 == 0.
bool encode_lines_4d(CUtensorMap *m, const void *base, uint64_t K, uint64_t N, uint64_t E,
                     uint32_t lines, uint32_t rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[4] = {32, K / 256, N, E};
  const cuuint64_t strides[3] = {128, K / 2, (K / 2) * N};
  const cuuint32_t box[4] = {32, lines, rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D uint32 map over the scales [E][N][K/16 bytes] seen as [E][N][K/64 words];
// box = `rows` rows x `words` words, no swizzle.  Needs K % 256 == 0 (16-byte rows).
bool encode_scale_words_3d(CUtensorMap *m, const void *base, uint64_t K, uint64_t N, uint64_t E,
                           uint32_t words, uint32_t rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[3] = {K / 64, N, E};
  const cuuint64_t strides[2] = {K / 16, (K / 16) * N};
  const cuuint32_t box[3] = {words, rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Descriptors of the expert library, cached by (pointers, shape): encoding
// costs a driver call, and graph replays reuse the captured parameters anyway.
struct LibMaps {
  const void *w = nullptr, *sfw = nullptr;
  int E = 0, N = 0, K = 0;
  bool sf_tma = false;  // K % 256 == 0: scale boxes for the tensor-memory variant,
                        // and the line map of the decode variant
  CUtensorMap tw, tsf, tlines, tsf_lines;
  CUtensorMap tbs;      // block-scaled variant: 128 rows x 128 bytes, 128B swizzle
  CUtensorMap tbs_sf;   // and its weight scales: 128 rows x 16 bytes (K % 256 == 0)
};
constexpr int kMapCache = 8;
LibMaps g_maps[kMapCache];
int g_maps_next = 0;
std::mutex g_maps_mu;

bool library_maps(const uint8_t *w, const uint8_t *sfw, int E, int N, int K, LibMaps *out) {
  std::lock_guard<std::mutex> lock(g_maps_mu);
  for (auto &m : g_maps)
    if (m.w == w && m.sfw == sfw && m.E == E && m.N == N && m.K == K) {
      *out = m;
      return true;
    }
  LibMaps m;
  m.w = w;
  m.sfw = sfw;
  m.E = E;
  m.N = N;
  m.K = K;
  m.sf_tma = (K % 256) == 0;
  std::memset(&m.tsf, 0, sizeof m.tsf);
  std::memset(&m.tlines, 0, sizeof m.tlines);
  std::memset(&m.tsf_lines, 0, sizeof m.tsf_lines);
  std::memset(&m.tbs, 0, sizeof m.tbs);
  std::memset(&m.tbs_sf, 0, sizeof m.tbs_sf);
  // the tensor-memory variant reads 16-row x 128-byte weight boxes and 16-row x 16-byte scale boxes
  static_assert(moe::gemv::tc::kWStride == 128 && moe::gemv::tc::kSFStride == 16, "box width");
  if (!encode_u8_3d(&m.tw, w, (uint64_t)K / 2, (uint64_t)N, (uint64_t)E, 128, 16,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  static_assert(moe::gemv::bs::kATile == 128 * 128, "block-scaled weight box");
  if (!encode_u8_3d(&m.tbs, w, (uint64_t)K / 2, (uint64_t)N, (uint64_t)E, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  if (m.sf_tma && !encode_u8_3d(&m.tsf, sfw, (uint64_t)K / 16, (uint64_t)N, (uint64_t)E, 16, 16,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  if (m.sf_tma && !encode_u8_3d(&m.tbs_sf, sfw, (uint64_t)K / 16, (uint64_t)N, (uint64_t)E, 16, 128,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  if (m.sf_tma && !encode_lines_4d(&m.tlines, w, (uint64_t)K, (uint64_t)N, (uint64_t)E,
                                   (uint32_t)moe::gemv::mma::kLines,
                                   (uint32_t)moe::gemv::mma::kStageRows))
    return false;
  if (m.sf_tma && !encode_scale_words_3d(&m.tsf_lines, sfw, (uint64_t)K, (uint64_t)N, (uint64_t)E,
                                         (uint32_t)moe::gemv::mma::kLines * 4,
                                         (uint32_t)moe::gemv::mma::kStageRows))
    return false;
  g_maps[g_maps_next] = m;
  g_maps_next = (g_maps_next + 1) % kMapCache;
  *out = m;
  return true;
}

}  // namespace

extern "C" {

int32_t moe_version(void) { return 100; }

const char *moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_ARCH: return "unsupported architecture (sm_100 required)";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

moe_status_t moe_get_device_error(uint32_t *host_flags, int32_t clear) {
  if (!host_flags) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyFromSymbol(host_flags, moe::g_device_error, sizeof(uint32_t)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(moe::g_device_error, &zero, sizeof(uint32_t)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// ------------------------------------------------------------------ step 1
moe_status_t moe_mask_padding(int64_t *routing_map, int32_t N, int32_t top_k,
                              const int32_t *real_token_count, int32_t tp_rank, cudaStream_t s) {
  if (N < 0 || top_k < 1 || tp_rank < 0 || !real_token_count) return MOE_ERR_INVALID_ARG;
  if (N > 0 && !routing_map) return MOE_ERR_INVALID_ARG;
  if (!aligned(routing_map, 8) || !aligned(real_token_count, 4)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  if (N == 0) return MOE_OK;
  const int64_t slots = (int64_t)N * top_k;
  int64_t blocks = (slots + 255) / 256;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  return launch_pdl(moe::mask_padding_kernel, dim3((unsigned)blocks), dim3(256), 0, s, routing_map,
                    N, top_k, real_token_count, tp_rank);
}

// ------------------------------------------------------------------ step 2
size_t moe_create_indices_workspace_bytes(int64_t num_slots, int32_t E) {
  if (num_slots <= moe::idx::kSmallSlots || E < 1) return moe::idx::kWsHeader;
  return moe::idx::kWsHeader + (size_t)tiles_for(num_slots) * (size_t)E * sizeof(uint32_t);
}

moe_status_t moe_create_indices(const int64_t *topk_ids, int64_t num_slots, int32_t E,
                                uint32_t *token_expert_order, uint32_t *expert_start_indices,
                                uint32_t *restore_token_order, int32_t *expert_ids,
                                uint32_t *expert_usage_stats, uint32_t *scales_offset,
                                void *workspace, size_t ws_bytes, cudaStream_t s) {
  using namespace moe::idx;
  if (E < 1 || E > 1024 || num_slots < 0 || num_slots >= (int64_t(1) << 31))
    return MOE_ERR_INVALID_ARG;
  if (!expert_start_indices || !expert_ids || !expert_usage_stats) return MOE_ERR_INVALID_ARG;
  if (num_slots > 0 && (!topk_ids || !token_expert_order || !restore_token_order))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(topk_ids, 8) || !aligned(token_expert_order, 4) ||
      !aligned(restore_token_order, 4) || !aligned(expert_start_indices, 4) ||
      !aligned(expert_ids, 4) || !aligned(expert_usage_stats, 4) || !aligned(scales_offset, 4))
    return MOE_ERR_INVALID_ARG;
  const size_t need = moe_create_indices_workspace_bytes(num_slots, E);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return MOE_ERR_WORKSPACE;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  const size_t smem = smem_bytes(E);
  if (num_slots <= kSmallSlots) {
    if ((st = set_smem(create_indices_small_kernel, smem)) != MOE_OK) return st;
    create_indices_small_kernel<<<1, kThreads, smem, s>>>(
        topk_ids, num_slots, E, token_expert_order, expert_start_indices, restore_token_order,
        expert_ids, expert_usage_stats, scales_offset);
    return launch_status();
  }
  const int64_t T = tiles_for(num_slots);
  uint32_t *ticket = static_cast<uint32_t *>(workspace);
  uint32_t *tiles = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kWsHeader);
  if (cudaMemsetAsync(ticket, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  if ((st = set_smem(create_indices_hist_kernel, smem)) != MOE_OK) return st;
  if ((st = set_smem(create_indices_scatter_kernel, smem)) != MOE_OK) return st;
  create_indices_hist_kernel<<<(unsigned)T, kThreads, smem, s>>>(
      topk_ids, num_slots, E, token_expert_order, expert_start_indices, expert_ids,
      expert_usage_stats, scales_offset, ticket, tiles);
  if ((st = launch_status()) != MOE_OK) return st;
  create_indices_scatter_kernel<<<(unsigned)T, kThreads, smem, s>>>(
      topk_ids, num_slots, E, token_expert_order, restore_token_order, tiles);
  return launch_status();
}

moe_status_t moe_mask_and_create_indices(int64_t *routing_map, int32_t N, int32_t top_k,
                                         const int32_t *real_token_count, int32_t tp_rank,
                                         int32_t E, uint32_t *token_expert_order,
                                         uint32_t *expert_start_indices,
                                         uint32_t *restore_token_order, int32_t *expert_ids,
                                         uint32_t *expert_usage_stats, uint32_t *scales_offset,
                                         void *workspace, size_t ws_bytes, cudaStream_t s) {
  using namespace moe::idx;
  if (N < 0 || top_k < 1 || tp_rank < 0 || !real_token_count) return MOE_ERR_INVALID_ARG;
  const int64_t S = (int64_t)N * top_k;
  if (S > kTinySlots) {
    moe_status_t st = moe_mask_padding(routing_map, N, top_k, real_token_count, tp_rank, s);
    if (st != MOE_OK) return st;
    return moe_create_indices(routing_map, S, E, token_expert_order, expert_start_indices,
                              restore_token_order, expert_ids, expert_usage_stats, scales_offset,
                              workspace, ws_bytes, s);
  }
  if (E < 1 || E > 1024) return MOE_ERR_INVALID_ARG;
  if (!expert_start_indices || !expert_ids || !expert_usage_stats) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!routing_map || !token_expert_order || !restore_token_order))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(routing_map, 8) || !aligned(real_token_count, 4) ||
      !aligned(token_expert_order, 4) || !aligned(restore_token_order, 4) ||
      !aligned(expert_start_indices, 4) || !aligned(expert_ids, 4) ||
      !aligned(expert_usage_stats, 4) || !aligned(scales_offset, 4))
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  const size_t smem = tiny_smem_bytes(E);
  if ((st = set_smem(mask_create_indices_tiny_kernel, smem)) != MOE_OK) return st;
  return launch_pdl(mask_create_indices_tiny_kernel, dim3(1), dim3(kThreads), smem, s, routing_map,
                    N, top_k, real_token_count, tp_rank, E, token_expert_order,
                    expert_start_indices, restore_token_order, expert_ids, expert_usage_stats,
                    scales_offset);
}

// ------------------------------------------------------------------ step 3
size_t moe_mxfp4_row_stride(int32_t K) {
  if (K <= 0) return 0;
  const size_t raw = (size_t)K / 2 + (size_t)K / 32;
  return (raw + 15) / 16 * 16;
}

moe_status_t moe_dispatch_mxfp4(const void *input_tokens, int32_t N, int32_t K, int32_t top_k,
                                int32_t E, const uint32_t *restore_token_order,
                                const uint32_t *expert_start_indices, const int32_t *expert_ids,
                                const uint32_t *expert_usage_stats, uint8_t *recv_buf,
                                int64_t recv_capacity, uint32_t *recv_counts, cudaStream_t s) {
  if (N < 0 || K <= 0 || K % 32 != 0 || top_k < 1 || E < 1 || E > 1024 || top_k > E ||
      recv_capacity < 0)
    return MOE_ERR_INVALID_ARG;
  if (!expert_start_indices || !expert_ids || !expert_usage_stats || !recv_counts)
    return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!input_tokens || !restore_token_order)) return MOE_ERR_INVALID_ARG;
  if (recv_capacity > 0 && !recv_buf) return MOE_ERR_INVALID_ARG;
  if (!aligned(input_tokens, 16) || !aligned(recv_buf, 16) || !aligned(recv_counts, 4))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  // segments of 256 columns per warp task: the largest of 8, 4, 2, 1 that
  // still gives every SM about 8 warps
  const int wpb = moe::disp::kWarpsPerBlock;
  const int64_t segs = (K + 255) / 256;
  int seg = 8;
  while (seg > 1 && (int64_t)N * ((segs + seg - 1) / seg) < (int64_t)sms * 8) seg /= 2;
  const int64_t groups = (segs + seg - 1) / seg;
  int64_t blocks = ((int64_t)N * groups + wpb - 1) / wpb;
  if (blocks < 1) blocks = 1;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  void (*kern)(const uint16_t *, int32_t, int32_t, int32_t, int32_t, const uint32_t *,
               const uint32_t *, const int32_t *, const uint32_t *, uint8_t *, int64_t, int32_t,
               uint32_t *) = seg == 8   ? moe::disp::dispatch_mxfp4_kernel<8>
                             : seg == 4 ? moe::disp::dispatch_mxfp4_kernel<4>
                             : seg == 2 ? moe::disp::dispatch_mxfp4_kernel<2>
                                        : moe::disp::dispatch_mxfp4_kernel<1>;
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(wpb * 32), 0, s,
                    static_cast<const uint16_t *>(input_tokens), N, K, top_k, E,
                    restore_token_order, expert_start_indices, expert_ids, expert_usage_stats,
                    recv_buf, recv_capacity, (int32_t)moe_mxfp4_row_stride(K), recv_counts);
}

moe_status_t moe_dispatch_mxfp4_quantize_nvfp4(
    const void *input_tokens, int32_t N, int32_t K, int32_t top_k, int32_t E,
    const uint32_t *restore_token_order, const uint32_t *expert_start_indices,
    const int32_t *expert_ids, const uint32_t *expert_usage_stats, uint8_t *recv_buf,
    int64_t recv_capacity, uint32_t *recv_counts, float act_global, uint8_t *xq, uint8_t *sfa,
    cudaStream_t s) {
  if (N < 0 || K <= 0 || K % 32 != 0 || top_k < 1 || E < 1 || E > 1024 || top_k > E ||
      recv_capacity < 0 || !(act_global > 0.0f))
    return MOE_ERR_INVALID_ARG;
  if (!expert_start_indices || !expert_ids || !expert_usage_stats || !recv_counts)
    return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!input_tokens || !restore_token_order || !xq || !sfa)) return MOE_ERR_INVALID_ARG;
  if (recv_capacity > 0 && !recv_buf) return MOE_ERR_INVALID_ARG;
  if (!aligned(input_tokens, 16) || !aligned(recv_buf, 16) || !aligned(recv_counts, 4) ||
      !aligned(xq, 4))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  // the dispatch's launch shape: segments of 256 columns per warp task, the
  // largest of 8, 4, 2, 1 that still gives every SM about 8 warps
  const int wpb = moe::disp::kWarpsPerBlock;
  const int64_t segs = (K + 255) / 256;
  int seg = 8;
  while (seg > 1 && (int64_t)N * ((segs + seg - 1) / seg) < (int64_t)sms * 8) seg /= 2;
  const int64_t groups = (segs + seg - 1) / seg;
  int64_t blocks = ((int64_t)N * groups + wpb - 1) / wpb;
  if (blocks < 1) blocks = 1;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  void (*kern)(const uint16_t *, int32_t, int32_t, int32_t, int32_t, const uint32_t *,
               const uint32_t *, const int32_t *, const uint32_t *, uint8_t *, int64_t, int32_t,
               uint32_t *, float, uint8_t *, uint8_t *) =
      seg == 8   ? moe::dq::dispatch_quant_kernel<8>
      : seg == 4 ? moe::dq::dispatch_quant_kernel<4>
      : seg == 2 ? moe::dq::dispatch_quant_kernel<2>
                 : moe::dq::dispatch_quant_kernel<1>;
  return launch_pdl(kern, dim3((unsigned)blocks), dim3(wpb * 32), 0, s,
                    static_cast<const uint16_t *>(input_tokens), N, K, top_k, E,
                    restore_token_order, expert_start_indices, expert_ids, expert_usage_stats,
                    recv_buf, recv_capacity, (int32_t)moe_mxfp4_row_stride(K), recv_counts,
                    act_global, xq, sfa);
}

// ------------------------------------------------------------------ step 4a
moe_status_t moe_quantize_activations_nvfp4(const void *x, int32_t M, int32_t K,
                                            float act_global, uint8_t *xq, uint8_t *sfa,
                                            cudaStream_t s) {
  if (M < 0 || K <= 0 || K % 16 != 0 || !(act_global > 0.0f)) return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!x || !xq || !sfa)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(xq, 4)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  const int wpb = moe::nvq::kWarpsPerBlock;
  const int64_t work = (int64_t)M * ((K + 255) / 256);
  int64_t blocks = (work + wpb - 1) / wpb;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  return launch_pdl(moe::nvq::quant_act_nvfp4_kernel, dim3((unsigned)blocks), dim3(wpb * 32), 0,
                    s, static_cast<const uint16_t *>(x), M, K, act_global, xq, sfa);
}

moe_status_t moe_quantize_weights_nvfp4(const float *w, int32_t E, int32_t N, int32_t K,
                                        uint8_t *wq, uint8_t *sfw, float *w_global,
                                        cudaStream_t s) {
  if (E < 1 || N < 1 || K <= 0 || K % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (!w || !wq || !sfw || !w_global) return MOE_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(wq, 4) || !aligned(w_global, 4)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  if (cudaMemsetAsync(w_global, 0, sizeof(float) * (size_t)E, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int64_t per_expert = (int64_t)N * K;
  int64_t cx = (per_expert + 256 * 64 - 1) / (256 * 64);
  if (cx > 1024) cx = 1024;
  moe::nvq::weight_amax_kernel<<<dim3((unsigned)cx, (unsigned)E), 256, 0, s>>>(
      w, per_expert, reinterpret_cast<unsigned int *>(w_global));
  if ((st = launch_status()) != MOE_OK) return st;
  const int wpb = moe::nvq::kWarpsPerBlock;
  const int64_t work = (int64_t)E * N * ((K + 255) / 256);
  int64_t blocks = (work + wpb - 1) / wpb;
  if (blocks > (int64_t)sms * 32) blocks = (int64_t)sms * 32;
  moe::nvq::quant_weight_nvfp4_kernel<<<(unsigned)blocks, wpb * 32, 0, s>>>(
      w, E, N, K, reinterpret_cast<const unsigned int *>(w_global), wq, sfw);
  if ((st = launch_status()) != MOE_OK) return st;
  moe::nvq::weight_global_kernel<<<(E + 255) / 256, 256, 0, s>>>(w_global, E);
  return launch_status();
}

// ------------------------------------------------------------------ step 4b
namespace {
size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The grouping the GEMV computes for itself when the caller passes only the
// routing map: the moe_create_indices outputs plus that call's own workspace,
// carved from the caller's workspace in this order, each 256-byte aligned.
struct GemvGrouping {
  uint32_t *order, *start, *restore, *stats;
  int32_t *eids;
  void *ci_ws;
  size_t ci_bytes, total;
};
GemvGrouping gemv_grouping_layout(int64_t S, int32_t E, void *base) {
  GemvGrouping g{};
  uint8_t *b = static_cast<uint8_t *>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t *q = b ? b + off : nullptr;
    off += round256(bytes);
    return q;
  };
  g.order = reinterpret_cast<uint32_t *>(take((size_t)S * 4));
  g.restore = reinterpret_cast<uint32_t *>(take((size_t)S * 4));
  g.start = reinterpret_cast<uint32_t *>(take((size_t)(E + 1) * 4));
  g.eids = reinterpret_cast<int32_t *>(take((size_t)E * 4));
  g.stats = reinterpret_cast<uint32_t *>(take(2 * 4));
  g.ci_bytes = moe_create_indices_workspace_bytes(S, E);
  g.ci_ws = take(g.ci_bytes);
  g.total = off;
  return g;
}

// The W4A16 activations converted once per call (tensor-memory variant):
// per-token offsets [M] int32, then the fp16 rows [M, K].
struct GemvActF16 {
  int32_t *shift;
  uint16_t *act16;
  size_t total;
};
GemvActF16 gemv_act_f16_layout(int64_t M, int64_t K, void *base) {
  GemvActF16 a{};
  uint8_t *b = static_cast<uint8_t *>(base);
  a.shift = b ? reinterpret_cast<int32_t *>(b) : nullptr;
  const size_t off = round256((size_t)M * 4);
  a.act16 = b ? reinterpret_cast<uint16_t *>(b + off) : nullptr;
  a.total = off + round256((size_t)M * (size_t)K * 2);
  return a;
}
}  // namespace

namespace {
// Which kernel variant a GEMV call runs, and whether it groups the routing map
// itself.  W4A4 with K % 64 == 0 runs on the block-scaled FP4 tensor core (no
// dequantisation).  W4A16 (and W4A4 otherwise): decode-sized passes (no more
// tokens per expert on average than one pass of the register-dequant
// mma.sync variant holds) take that variant; more tokens per expert take the
// tensor-memory variant, whose tcgen05 MMA has a fixed per-instruction cost up
// to N = 64 and whose passes hold 64 tokens.  Only the decode variant groups
// a small routing map in-kernel (every CTA histograms the map and compacts the
// token lists of its own passes); the bound on passes per CTA behind that path
// needs at most kFusedSlots slots, kMaxActive experts and a full grid.
struct GemvPlan {
  moe_gemv_variant_t variant;
  bool groups_in_kernel;
};
GemvPlan plan_gemv(moe_gemv_mode_t mode, int64_t S, int32_t E, int32_t K, bool grouping_given,
                   int sms) {
  namespace mma = moe::gemv::mma;
  const bool bs_ok = mode == MOE_W4A4 && K % 64 == 0;
  const int ts_mma = K % 256 == 0 ? mma::tokens_per_pass(K) : 0;
  const bool mma_ok = ts_mma >= 8 && E <= mma::kMaxActive;
  bool use_bs = bs_ok;
  bool use_mma = !bs_ok && mma_ok && S <= (int64_t)ts_mma * E;
  // test hook: MOE_GEMV_VARIANT=mma|tc|bs forces a variant where it applies
  // (every variant is exact for every input it accepts)
  if (const char *v = std::getenv("MOE_GEMV_VARIANT")) {
    if (v[0] == 'm' && mma_ok) use_mma = true, use_bs = false;
    if (v[0] == 't') use_mma = false, use_bs = false;
    if (v[0] == 'b' && bs_ok) use_bs = true, use_mma = false;
  }
  GemvPlan g;
  g.variant = use_bs ? MOE_GEMV_BLOCK_SCALED : use_mma ? MOE_GEMV_DECODE : MOE_GEMV_TENSOR_MEMORY;
  g.groups_in_kernel = !grouping_given && use_mma && S <= mma::kFusedSlots && sms >= 148;
  return g;
}
}  // namespace

size_t moe_grouped_gemv_workspace_bytes(int32_t M, int32_t top_k, int32_t E, int32_t K) {
  if (M < 0 || top_k < 1 || E < 1 || K < 0) return 0;
  return gemv_grouping_layout((int64_t)M * top_k, E, nullptr).total +
         gemv_act_f16_layout(M, K, nullptr).total;
}

moe_status_t moe_grouped_gemv_nvfp4(moe_gemv_mode_t mode, const void *act, const uint8_t *sfa,
                                    float act_global, const int64_t *indices, int32_t M,
                                    int32_t top_k, const uint8_t *w, const uint8_t *sfw,
                                    const float *w_global, int32_t E, int32_t N, int32_t K,
                                    const uint32_t *token_expert_order,
                                    const uint32_t *expert_start_indices,
                                    const int32_t *expert_ids,
                                    const uint32_t *expert_usage_stats, void *out,
                                    void *workspace, size_t ws_bytes, cudaStream_t s) {
  using namespace moe::gemv;
  if (mode != MOE_W4A16 && mode != MOE_W4A4) return MOE_ERR_INVALID_ARG;
  if (M < 0 || top_k < 1 || E < 1 || E > kMaxExperts || top_k > E || N < 8 || N % 8 != 0 ||
      K < 32 || K % 32 != 0 || !(act_global > 0.0f))
    return MOE_ERR_INVALID_ARG;
  // the step-2 grouping: all four given, or none (then computed from indices)
  const int given = (token_expert_order != nullptr) + (expert_start_indices != nullptr) +
                    (expert_ids != nullptr) + (expert_usage_stats != nullptr);
  if (given != 0 && given != 4) return MOE_ERR_INVALID_ARG;
  if (!w || !sfw) return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!act || !out)) return MOE_ERR_INVALID_ARG;
  if (given == 0 && M > 0 && !indices) return MOE_ERR_INVALID_ARG;
  if (!aligned(indices, 8)) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_W4A4 && M > 0 && !sfa) return MOE_ERR_INVALID_ARG;
  if (!aligned(act, 16) || !aligned(w, 16) || !aligned(sfw, 16) || !aligned(out, 16) ||
      !aligned(w_global, 4) || !aligned(sfa, 4))
    return MOE_ERR_INVALID_ARG;
  // the flat unit count must fit 32 bits: (S / 32 + E) * ceil(N / 16)
  const int64_t S = (int64_t)M * top_k;
  if ((S / 8 + E + 1) * ((N + 15) / 16) >= (int64_t(1) << 32)) return MOE_ERR_INVALID_ARG;
  if (given == 0 && M > 0) {
    const GemvGrouping g0 = gemv_grouping_layout(S, E, nullptr);
    if (!workspace || ws_bytes < g0.total || !aligned(workspace, 256)) return MOE_ERR_WORKSPACE;
  }
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  const GemvPlan plan = plan_gemv(mode, S, E, K, given == 4, sms);
  const bool fused_grouping = plan.groups_in_kernel;
  // W4A16 in the tensor-memory variant converts the activations once, into
  // the workspace after the grouping's sections (at its start when the
  // grouping is given), when the workspace has room for them
  GemvActF16 a16{};
  if (mode == MOE_W4A16 && plan.variant == MOE_GEMV_TENSOR_MEMORY && workspace &&
      aligned(workspace, 256)) {
    const size_t base = given == 0 ? gemv_grouping_layout(S, E, nullptr).total : 0;
    const GemvActF16 need = gemv_act_f16_layout(M, K, nullptr);
    if (ws_bytes >= base + need.total)
      a16 = gemv_act_f16_layout(M, K, static_cast<uint8_t *>(workspace) + base);
  }
  if (given == 0 && !fused_grouping) {
    // group the pairs of the routing map first, into the caller's workspace
    const GemvGrouping g = gemv_grouping_layout(S, E, workspace);
    st = moe_create_indices(indices, S, E, g.order, g.start, g.restore, g.eids, g.stats, nullptr,
                            g.ci_ws, g.ci_bytes, s);
    if (st != MOE_OK) return st;
    token_expert_order = g.order;
    expert_start_indices = g.start;
    expert_ids = g.eids;
    expert_usage_stats = g.stats;
  }
  Params p;
  p.act = act;
  p.sfa = sfa;
  p.g_a = act_global;
  p.M = M;
  p.top_k = top_k;
  p.w = w;
  p.sfw = sfw;
  p.w_global = w_global;
  p.N = N;
  p.K = K;
  p.order = token_expert_order;
  p.start = expert_start_indices;
  p.eids = expert_ids;
  p.stats = expert_usage_stats;
  p.out = static_cast<uint16_t *>(out);
  p.indices = indices;
  p.E = E;
  p.wait_limit_ns = kWaitLimitNs;
  // test hook: MOE_TEST_WAIT_LIMIT_NS shortens every pipeline wait of the GEMV,
  // so a test can make one expire and check MOE_DEVERR_WAIT_TIMEOUT (the kernel
  // then winds down and waits for its copies in flight; no fault, no hang)
  if (const char *v = std::getenv("MOE_TEST_WAIT_LIMIT_NS")) p.wait_limit_ns = std::strtoull(v, nullptr, 10);
  LibMaps maps;
  if (!library_maps(w, sfw, E, N, K, &maps)) return MOE_ERR_CUDA;
  const bool use_bs = plan.variant == MOE_GEMV_BLOCK_SCALED;
  const bool use_mma = plan.variant == MOE_GEMV_DECODE;
  const int ts_mma = use_mma ? mma::tokens_per_pass(K) : 0;
  if (use_bs) {
    // passes of 64 tokens (two more stages in flight) when the experts hold
    // 64 tokens or fewer on average, else 128
    const bool small = S <= (int64_t)64 * E;
    // weight scales by TMA when their rows are whole 16-byte units (K % 256 == 0)
    void (*kern)(const Params, const CUtensorMap, const CUtensorMap) =
        small ? (maps.sf_tma ? bs::grouped_gemv_bs_kernel<64, true>
                             : bs::grouped_gemv_bs_kernel<64, false>)
              : (maps.sf_tma ? bs::grouped_gemv_bs_kernel<128, true>
                             : bs::grouped_gemv_bs_kernel<128, false>);
    const size_t smem = small ? (maps.sf_tma ? bs::Cfg<64, true>::kSmemBytes
                                             : bs::Cfg<64, false>::kSmemBytes)
                              : (maps.sf_tma ? bs::Cfg<128, true>::kSmemBytes
                                             : bs::Cfg<128, false>::kSmemBytes);
    if ((st = set_smem(kern, smem)) != MOE_OK) return st;
    return launch_pdl(kern, dim3((unsigned)sms), dim3(bs::kThreads), smem, s, p, maps.tbs,
                      maps.tbs_sf);
  }
  if (use_mma) {
    void (*kern)(const Params, const int, const CUtensorMap, const CUtensorMap) =
        mode == MOE_W4A16 ? mma::grouped_gemv_mma_kernel<MOE_W4A16>
                          : mma::grouped_gemv_mma_kernel<MOE_W4A4>;
    if ((st = set_smem(kern, mma::kSmemBytes)) != MOE_OK) return st;
    return launch_pdl(kern, dim3((unsigned)sms), dim3(mma::kThreads), mma::kSmemBytes, s, p,
                      ts_mma, maps.tlines, maps.tsf_lines);
  }
  if (a16.act16) {
    st = launch_pdl(tc::act_f16_kernel, dim3((unsigned)((M + 7) / 8)), dim3(256), 0, s,
                    static_cast<const uint16_t *>(act), M, K, a16.shift, a16.act16);
    if (st != MOE_OK) return st;
  }
  void (*kern)(const Params, const CUtensorMap, const CUtensorMap, const uint16_t *,
               const int32_t *);
  // passes of 128 tokens when the activations were converted and the experts
  // hold more than 64 tokens on average, else 64
  const bool wide = a16.act16 != nullptr && S > (int64_t)64 * E;
  if (mode == MOE_W4A16 && wide)
    kern = maps.sf_tma ? tc::grouped_gemv_kernel<MOE_W4A16, true, 128>
                       : tc::grouped_gemv_kernel<MOE_W4A16, false, 128>;
  else if (mode == MOE_W4A16)
    kern = maps.sf_tma ? tc::grouped_gemv_kernel<MOE_W4A16, true, 64>
                       : tc::grouped_gemv_kernel<MOE_W4A16, false, 64>;
  else
    kern = maps.sf_tma ? tc::grouped_gemv_kernel<MOE_W4A4, true, 64>
                       : tc::grouped_gemv_kernel<MOE_W4A4, false, 64>;
  const size_t smem = wide ? tc::Cfg<128>::kSmemBytes : tc::Cfg<64>::kSmemBytes;
  if ((st = set_smem(kern, smem)) != MOE_OK) return st;
  return launch_pdl(kern, dim3((unsigned)sms), dim3(tc::kThreads), smem, s, p, maps.tw,
                    maps.tsf, static_cast<const uint16_t *>(a16.act16),
                    static_cast<const int32_t *>(a16.shift));
}

moe_status_t moe_grouped_gemv_plan(moe_gemv_mode_t mode, int32_t M, int32_t top_k, int32_t E,
                                   int32_t N, int32_t K, int32_t grouping_given,
                                   int32_t *variant, int32_t *groups_in_kernel) {
  if (mode != MOE_W4A16 && mode != MOE_W4A4) return MOE_ERR_INVALID_ARG;
  if (M < 0 || top_k < 1 || E < 1 || E > moe::gemv::kMaxExperts || top_k > E || N < 8 ||
      N % 8 != 0 || K < 32 || K % 32 != 0 || !variant || !groups_in_kernel)
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  const GemvPlan g = plan_gemv(mode, (int64_t)M * top_k, E, K, grouping_given != 0, sms);
  *variant = (int32_t)g.variant;
  *groups_in_kernel = g.groups_in_kernel ? 1 : 0;
  return MOE_OK;
}

// ------------------------------------------------------------------ step 5
moe_status_t moe_combine(const void *expert_out, const float *router_weights,
                         const int64_t *topk_ids, int32_t M, int32_t top_k, int32_t H, int32_t E,
                         moe_epilogue_t epi, float alpha, void *output_tokens, cudaStream_t s) {
  if (M < 0 || top_k < 1 || H < 8 || H % 8 != 0 || E < 1) return MOE_ERR_INVALID_ARG;
  if (epi != MOE_EPI_NONE && epi != MOE_EPI_IDENTITY && epi != MOE_EPI_SCALE)
    return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!expert_out || !router_weights || !topk_ids || !output_tokens))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(expert_out, 16) || !aligned(output_tokens, 16) || !aligned(router_weights, 4) ||
      !aligned(topk_ids, 8))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  moe_status_t st = check_device(&sms);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  const int wpb = moe::comb::kWarpsPerBlock;
  const int64_t work = (int64_t)M * ((H + 255) / 256);
  int64_t blocks = (work + wpb - 1) / wpb;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  const uint16_t *y = static_cast<const uint16_t *>(expert_out);
  uint16_t *o = static_cast<uint16_t *>(output_tokens);
  if (epi == MOE_EPI_SCALE)
    return launch_pdl(moe::comb::combine_kernel<MOE_EPI_SCALE>, dim3((unsigned)blocks),
                      dim3(wpb * 32), 0, s, y, router_weights, topk_ids, M, top_k, H, E, alpha,
                      o);
  return launch_pdl(moe::comb::combine_kernel<MOE_EPI_IDENTITY>, dim3((unsigned)blocks),
                    dim3(wpb * 32), 0, s, y, router_weights, topk_ids, M, top_k, H, E, alpha, o);
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation grouping
// Scratch of moe_create_indices_static: a fixed array in the library's own
// device memory, so callers that cannot allocate still get the tiled path.
// Host code must not pass the symbol itself to a kernel (on the host it only
// names a host-side shadow); the device address is looked up once per device.
namespace {
static __device__ __align__(256) unsigned char g_create_indices_scratch[MOE_CREATE_INDICES_STATIC_SCRATCH];
void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

moe_status_t static_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_create_indices_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}
}  // namespace

extern "C" moe_status_t moe_create_indices_static(const int64_t *topk_ids, int64_t num_slots,
                                                  int32_t E, uint32_t *token_expert_order,
                                                  uint32_t *expert_start_indices,
                                                  uint32_t *restore_token_order,
                                                  int32_t *expert_ids,
                                                  uint32_t *expert_usage_stats,
                                                  uint32_t *scales_offset, cudaStream_t s) {
  if (E < 1 || E > 1024 || num_slots < 0 || num_slots >= (int64_t(1) << 31))
    return MOE_ERR_INVALID_ARG;
  if (moe_create_indices_workspace_bytes(num_slots, E) > MOE_CREATE_INDICES_STATIC_SCRATCH)
    return MOE_ERR_WORKSPACE;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  void *scratch = nullptr;
  if ((st = static_scratch(&scratch)) != MOE_OK) return st;
  return moe_create_indices(topk_ids, num_slots, E, token_expert_order, expert_start_indices,
                            restore_token_order, expert_ids, expert_usage_stats, scales_offset,
                            scratch, MOE_CREATE_INDICES_STATIC_SCRATCH, s);
}
