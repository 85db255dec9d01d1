/*
 * moe_route.h -- C ABI of the B200 (sm_100a) MoE token-routing library.
 *
 * The five steps of the single-GPU routing hot path, in call order:
 *
 *   moe_mask_padding                 mask CUDA-graph padding rows of the routing map
 *   moe_create_indices               group (token, slot) pairs by expert (CSR)
 *   moe_mask_and_create_indices      steps 1 and 2 in one call
 *   moe_dispatch_mxfp4               expert-grouped MXFP4 send buffer (1 GPU)
 *   moe_quantize_activations_nvfp4   W4A4 only: bf16 activations -> NVFP4
 *   moe_grouped_gemv_nvfp4           grouped expert GEMV on an NVFP4 library
 *   moe_combine                      router-weighted sum of expert outputs
 *
 * Conventions (all entry points):
 *   - Every pointer is a DEVICE pointer owned by the caller, unless stated.
 *     The library allocates no memory: every buffer, including workspace,
 *     comes from the caller, so calls can be captured in a CUDA graph.
 *   - Each call enqueues its kernels on stream `s` and returns without
 *     synchronising.  Values behind device pointers (real_token_count, the
 *     routing map, the grouping) may change between graph replays.
 *   - Arguments are validated on the host before any launch; an invalid
 *     call returns an error and launches nothing.
 *   - A device that is not sm_100 (B200 class) is rejected with
 *     MOE_ERR_UNSUPPORTED_ARCH; there is no fallback path.
 *   - Expert ids outside [0, E) -- the -1 padding sentinel included -- mean
 *     "route nowhere"; they are never an error.
 *   - bf16 means IEEE binary32 truncated to its upper 16 bits; FP4 codes are
 *     E2M1 (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), element 2i in the low
 *     nibble of byte i; E4M3 and E8M0 are the OCP 8-bit scale formats.
 *   - Rounding: every FP4 / E4M3 code is round-to-nearest-even with
 *     saturation to the largest finite value, from an fp32 operand.
 *   - Kernels never spin without bound.  A bounded wait that expires sets a
 *     bit in the device error word (moe_get_device_error) and the kernel
 *     returns; outputs of that call are then undefined.
 */
#ifndef MOE_ROUTE_H_
#define MOE_ROUTE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,      /* bad size, null or misaligned pointer        */
  MOE_ERR_UNSUPPORTED_ARCH = 2, /* current device is not sm_100               */
  MOE_ERR_WORKSPACE = 3,        /* workspace missing or too small             */
  MOE_ERR_CUDA = 4              /* a CUDA runtime call or launch failed       */
} moe_status_t;

typedef enum { MOE_W4A16 = 0, MOE_W4A4 = 1 } moe_gemv_mode_t;

/* Kernel variants of the grouped GEMV (moe_grouped_gemv_plan). */
typedef enum {
  MOE_GEMV_DECODE = 0,         /* few tokens per expert: register dequant + mma.sync    */
  MOE_GEMV_TENSOR_MEMORY = 1,  /* many tokens per expert: dequant into TMEM + tcgen05    */
  MOE_GEMV_BLOCK_SCALED = 2    /* W4A4, K % 64 == 0: tcgen05 block-scaled FP4 MMA        */
} moe_gemv_variant_t;

typedef enum {
  MOE_EPI_NONE = 0,     /* no epilogue fused (has_epilogue_fusion = false)    */
  MOE_EPI_IDENTITY = 1, /* fused elementwise epilogue f(v) = v                */
  MOE_EPI_SCALE = 2     /* fused elementwise epilogue f(v) = alpha * v        */
} moe_epilogue_t;

/* Bits of the device error word. */
#define MOE_DEVERR_WAIT_TIMEOUT   0x1u /* a pipeline wait in the GEMV expired           */
#define MOE_DEVERR_RECV_OVERFLOW  0x2u /* dispatch: routed pairs exceed recv_capacity   */
#define MOE_DEVERR_ACT_RANGE      0x4u /* W4A16 GEMV without offsets: |act| > 65504     */
#define MOE_DEVERR_LIMIT          0x8u /* an internal table limit was exceeded; the call
                                          computed nothing (not expected within the
                                          documented limits)                           */

/* --------------------------------------------------------------------- */
/* Step 1 -- Megatron-Core "core.transformer.moe.inference_routing_mask_  */
/* kernel", mask_routing_padding (API, Parameters).                      */
/* In place: every top_k slot of local row r with                        */
/*   r + tp_rank * N >= *real_token_count                                */
/* becomes -1; other rows are untouched.                                 */
/*   routing_map       int64 [N, top_k], row-major, 8-byte aligned       */
/*   real_token_count  DEVICE int32[1], read inside the kernel (so the   */
/*                     boundary moves across graph replays); may be <= 0 */
/*                     (all rows masked) or > N (none masked)            */
/*   tp_rank           >= 0, offset of this rank's rows in the global    */
/*                     (pre-SP-shard) frame                              */
/* Errors: MOE_ERR_INVALID_ARG for N < 0, top_k < 1, null pointers.      */
MOE_API moe_status_t moe_mask_padding(int64_t *routing_map, int32_t N, int32_t top_k,
                              const int32_t *real_token_count, int32_t tp_rank,
                              cudaStream_t s);

/* --------------------------------------------------------------------- */
/* Step 2 -- MAX "moe_create_indices" (description and Args).             */
/* Groups the S = N*top_k flattened (token, slot) pairs p = t*top_k + j   */
/* by expert so that each expert's pairs are contiguous:                 */
/*   token_expert_order   uint32 [S]: pair indices grouped by expert,    */
/*                        experts in ascending id, pairs in ascending p  */
/*                        within an expert (stable); entries >= R (the   */
/*                        number of routed pairs) are 0xFFFFFFFF         */
/*   expert_start_indices uint32 [E+1]: CSR offsets of the A active      */
/*                        experts into token_expert_order; entries       */
/*                        [A+1, E] equal R                               */
/*   restore_token_order  uint32 [S]: position of pair p in              */
/*                        token_expert_order, 0xFFFFFFFF if unrouted     */
/*   expert_ids           int32 [E]: the active experts in ascending id; */
/*                        entries [A, E) are -1                          */
/*   expert_usage_stats   uint32 [2]: {max pairs on one expert, A}        */
/*   scales_offset        optional (NULL allowed) uint32 [E+1]: offset   */
/*                        of each active expert's first row when every   */
/*                        expert's rows are padded to a multiple of 128  */
/*                        (block-scaled grouped matmul scale layout);    */
/*                        entries [A+1, E] equal the padded total        */
/*   topk_ids             int64 [S] (the flattened routing map)          */
/* workspace: moe_create_indices_workspace_bytes(S, E) bytes, 256-byte   */
/* aligned, caller-owned; contents need no initialisation and are        */
/* scratch between calls.  Calls sharing one workspace must not overlap. */
/* Limits: 1 <= E <= 1024, 0 <= S < 2^31.                                */
MOE_API size_t moe_create_indices_workspace_bytes(int64_t num_slots, int32_t E);
MOE_API moe_status_t moe_create_indices(const int64_t *topk_ids, int64_t num_slots, int32_t E,
                                uint32_t *token_expert_order, uint32_t *expert_start_indices,
                                uint32_t *restore_token_order, int32_t *expert_ids,
                                uint32_t *expert_usage_stats, uint32_t *scales_offset,
                                void *workspace, size_t ws_bytes, cudaStream_t s);

/* Steps 1 and 2 in one call: exactly moe_mask_padding(routing_map, N,   */
/* top_k, real_token_count, tp_rank) followed by moe_create_indices on   */
/* the masked map (num_slots = N * top_k), with the same outputs,        */
/* including the -1 written into masked rows of routing_map.  When       */
/* N * top_k <= 1024 both steps run as one single-CTA kernel (one load   */
/* per slot, no second launch); larger maps take the two-call path.      */
/* Arguments, limits, workspace and errors: as the two calls (workspace  */
/* may be NULL when N * top_k <= 1024).                                  */
MOE_API moe_status_t moe_mask_and_create_indices(int64_t *routing_map, int32_t N, int32_t top_k,
                                                 const int32_t *real_token_count,
                                                 int32_t tp_rank, int32_t E,
                                                 uint32_t *token_expert_order,
                                                 uint32_t *expert_start_indices,
                                                 uint32_t *restore_token_order,
                                                 int32_t *expert_ids,
                                                 uint32_t *expert_usage_stats,
                                                 uint32_t *scales_offset, void *workspace,
                                                 size_t ws_bytes, cudaStream_t s);

/* The same grouping for callers that cannot provide a workspace.  (The   */
/* method's pages have no counterpart: this is an interface convenience.) */
/* Some hosts only hand a kernel its input and output tensors -- plugin  */
/* interfaces with no allocator or workspace argument, and serving loops */
/* that freeze their device-memory plan at start-up and forbid any later */
/* cudaMalloc, which can synchronise the device.  This entry point takes */
/* no workspace and allocates nothing: its scratch is a fixed array of   */
/* MOE_CREATE_INDICES_STATIC_SCRATCH bytes inside the library, held by   */
/* every GPU that loads the library until the process exits.            */
/*   - Same arguments and outputs as moe_create_indices, minus workspace. */
/*   - Requires moe_create_indices_workspace_bytes(num_slots, E) <=       */
/*     MOE_CREATE_INDICES_STATIC_SCRATCH, else MOE_ERR_WORKSPACE and no   */
/*     launch (E = 64 allows about 8 million slots, E = 1024 half a      */
/*     million).                                                         */
/*   - All calls on a device share the one scratch array, and it keeps   */
/*     the previous call's contents; calls whose kernels may overlap on  */
/*     the GPU (several streams, several host threads) race on it and    */
/*     must be serialised by the caller.                                 */
/*   - The first call on each device looks up the array's device address */
/*     (cudaGetSymbolAddress, with that device current); make that first */
/*     call before starting any stream capture.  The address is cached   */
/*     per device for the life of the process: do not use this entry     */
/*     point after cudaDeviceReset, nor from a context other than the    */
/*     device's primary context (the cached address belongs to it).      */
#define MOE_CREATE_INDICES_STATIC_SCRATCH ((size_t)262144)
MOE_API moe_status_t moe_create_indices_static(const int64_t *topk_ids, int64_t num_slots,
                                               int32_t E, uint32_t *token_expert_order,
                                               uint32_t *expert_start_indices,
                                               uint32_t *restore_token_order,
                                               int32_t *expert_ids,
                                               uint32_t *expert_usage_stats,
                                               uint32_t *scales_offset, cudaStream_t s);

/* --------------------------------------------------------------------- */
/* Step 3 -- MAX "Struct_ep_dispatch_async_mxfp4", execute(), reduced to */
/* one GPU (n_gpus_per_node = n_nodes = 1: the send buffer is the        */
/* receive buffer).  Row i < R of recv_buf holds token                   */
/* token_expert_order[i] / top_k quantised to MXFP4, with the block      */
/* scales packed next to the quants:                                     */
/*   bytes [0, K/2)        E2M1 codes                                    */
/*   bytes [K/2, K/2+K/32) E8M0 scales, one per 32 elements: 2^(floor(   */
/*                         log2(amax)) - 2), exponent clamped to         */
/*                         [-127, 127]; an all-zero block gets code 0    */
/*   then zero padding up to moe_mxfp4_row_stride(K) (a multiple of 16)  */
/* recv_counts[e] (uint32 [E]) = pairs routed to expert e.               */
/*   input_tokens  bf16 [N, K], 16-byte aligned rows                     */
/*   restore_token_order, expert_start_indices, expert_ids,              */
/*   expert_usage_stats: the outputs of moe_create_indices for this map  */
/*   recv_buf      uint8 [recv_capacity, stride], 16-byte aligned; rows  */
/*                 >= R are untouched.  If R > recv_capacity, rows past  */
/*                 the capacity are dropped and MOE_DEVERR_RECV_OVERFLOW */
/*                 is raised.                                            */
/* Each token row is read and encoded once and written to each of its    */
/* routed rows.  Limits: K % 32 == 0, 1 <= top_k <= E <= 1024.            */
MOE_API size_t moe_mxfp4_row_stride(int32_t K);
MOE_API moe_status_t moe_dispatch_mxfp4(const void *input_tokens, int32_t N, int32_t K, int32_t top_k,
                                int32_t E, const uint32_t *restore_token_order,
                                const uint32_t *expert_start_indices, const int32_t *expert_ids,
                                const uint32_t *expert_usage_stats, uint8_t *recv_buf,
                                int64_t recv_capacity, uint32_t *recv_counts, cudaStream_t s);

/* Steps 3 and 4a from one read of x (the W4A4 path needs both encodings */
/* of the same rows: MAX ep.dispatch_async.mxfp4 execute(), and the       */
/* FlashRT card's quantize_activations_nvfp4_bf16, whose                  */
/* grouped_w4a4_gemv_from_bf16 path starts from the same bf16 rows).      */
/* Writes exactly what moe_dispatch_mxfp4 (recv_buf, recv_counts) and     */
/* moe_quantize_activations_nvfp4(x, N, K, act_global, xq, sfa) write,    */
/* reading each token row once.  Arguments, limits and errors: as those   */
/* two calls (xq uint8 [N, K/2], sfa uint8 [N, K/16]).                    */
MOE_API moe_status_t moe_dispatch_mxfp4_quantize_nvfp4(
    const void *input_tokens, int32_t N, int32_t K, int32_t top_k, int32_t E,
    const uint32_t *restore_token_order, const uint32_t *expert_start_indices,
    const int32_t *expert_ids, const uint32_t *expert_usage_stats, uint8_t *recv_buf,
    int64_t recv_capacity, uint32_t *recv_counts, float act_global, uint8_t *xq, uint8_t *sfa,
    cudaStream_t s);

/* --------------------------------------------------------------------- */
/* Step 4a -- FlashRT "grouped-moe-gemv" card, Available functions:       */
/* quantize_activations_nvfp4_bf16.  For every 16-element block of       */
/* x [M, K] (bf16) with global scale g = act_global > 0:                 */
/*   s = E4M3( fl32(fl32(amax/6) / g) ),  sdec = fl32(e4m3(s) * g)        */
/*   q_i = E2M1( fl32(x_i / sdec) )   (signed zeros when sdec == 0)       */
/* Outputs xq uint8 [M, K/2] and sfa (E4M3) uint8 [M, K/16].              */
/* Limits: K % 16 == 0; x 16-byte aligned rows when K % 8 == 0.           */
MOE_API moe_status_t moe_quantize_activations_nvfp4(const void *x, int32_t M, int32_t K,
                                            float act_global, uint8_t *xq, uint8_t *sfa,
                                            cudaStream_t s);

/* FlashRT card, quantize_weights_nvfp4_bf16 (offline helper, fp32 input).*/
/* w fp32 [E, N, K] -> wq uint8 [E, N, K/2], sfw uint8 [E, N, K/16],     */
/* w_global fp32 [E] = fl32(amax(W_e) / 2688), or 1 when W_e is all zero.*/
/* Blocks are encoded as in step 4a with g = w_global[e].                */
MOE_API moe_status_t moe_quantize_weights_nvfp4(const float *w, int32_t E, int32_t N, int32_t K,
                                        uint8_t *wq, uint8_t *sfw, float *w_global,
                                        cudaStream_t s);

/* --------------------------------------------------------------------- */
/* Step 4b -- FlashRT "grouped-moe-gemv" card: grouped_w4a16_gemv_bf16 /  */
/* grouped_w4a4_gemv_bf16, token-major routing (W4A4 routing paragraph:  */
/* activations [M, K], device indices [M, top_k], library [E, N, K/2],    */
/* output [M, top_k, N]).  For every routed pair p = m*top_k + j with     */
/* expert e = indices[m, j] in [0, E):                                   */
/*   out[p, n] = bf16( g_w[e] * g_a * sum_k a(m,k) * w(e,n,k) )           */
/* accumulated in fp32, where w = e2m1(wq) * e4m3(sfw) and               */
/*   MOE_W4A16: a = act (bf16 [M, K]), sfa = NULL, g_a = act_global;     */
/*   MOE_W4A4 : a = e2m1(act) * e4m3(sfa), act uint8 [M, K/2],           */
/*              sfa uint8 [M, K/16] (from step 4a), g_a = act_global.    */
/* Slots whose id is outside [0, E) are not written.                     */
/*   indices   int64 [M, top_k], device memory (its values may change     */
/*             between CUDA-graph replays)                                */
/*   w_global  fp32 [E] or NULL (all ones)                                */
/*   grouping  token_expert_order, expert_start_indices, expert_ids,      */
/*             expert_usage_stats: EITHER all four, the moe_create_indices */
/*             outputs for this same map (then indices may be NULL), OR   */
/*             all four NULL: the call then groups the pairs of indices   */
/*             itself (one extra launch) into `workspace`                 */
/*   workspace caller-owned device memory, 256-byte aligned, contents need */
/*             no initialisation; moe_grouped_gemv_workspace_bytes(M,     */
/*             top_k, E, K) bytes serve every variant.  Its first part    */
/*             holds the grouping (required when the grouping is not      */
/*             given); the rest holds the W4A16 activations converted     */
/*             once per call for the tensor-memory variant (used when it  */
/*             fits; with the grouping given that part starts at offset   */
/*             0 and workspace may be NULL)                               */
/* "M = routed pairs, top_k = 1" is simply a routing map of shape [R, 1]. */
/* Limits: K % 32 == 0, N % 8 == 0, 1 <= top_k <= E <= 1024; act, w, sfw  */
/* and out 16-byte aligned, sfa 4-byte aligned.  W4A4 with K % 64 == 0    */
/* runs on the block-scaled FP4 tensor core (both operands stay NVFP4).   */
/* Errors: MOE_ERR_INVALID_ARG (shapes, nulls, alignment, a partial       */
/* grouping), MOE_ERR_WORKSPACE (missing or small workspace when the      */
/* grouping is not given); nothing is launched then.                      */
/* W4A16 activations enter the tensor cores as fp16, each token that does */
/* not already fit fp16 exactly scaled by a power of two of its own first */
/* (the epilogue multiplies it back), so any finite bf16 token is exact   */
/* down to 2^-29 of its largest element.  Only a tensor-memory call whose */
/* workspace lacks the room for the converted activations converts them   */
/* chunk by chunk without offsets: exact for 2^-14 <= |x| <= 65504, fp16  */
/* subnormals below (absolute error <= 2^-25), and |x| > 65504 raises     */
/* MOE_DEVERR_ACT_RANGE (the affected outputs are then undefined).        */
MOE_API size_t moe_grouped_gemv_workspace_bytes(int32_t M, int32_t top_k, int32_t E, int32_t K);
MOE_API moe_status_t moe_grouped_gemv_nvfp4(moe_gemv_mode_t mode, const void *act, const uint8_t *sfa,
                                    float act_global, const int64_t *indices, int32_t M,
                                    int32_t top_k, const uint8_t *w, const uint8_t *sfw,
                                    const float *w_global, int32_t E, int32_t N, int32_t K,
                                    const uint32_t *token_expert_order,
                                    const uint32_t *expert_start_indices,
                                    const int32_t *expert_ids,
                                    const uint32_t *expert_usage_stats, void *out,
                                    void *workspace, size_t ws_bytes, cudaStream_t s);

/* Which variant moe_grouped_gemv_nvfp4 runs for these shapes on the       */
/* current device, and whether it groups the routing map inside the GEMV   */
/* kernel when the grouping is not given (*groups_in_kernel = 1: no        */
/* grouping launch precedes it).  Host-only query, launches nothing.       */
/* (An interface aid of this library, no counterpart on the pages.)       */
/* Errors: MOE_ERR_INVALID_ARG as moe_grouped_gemv_nvfp4 for the shapes.   */
MOE_API moe_status_t moe_grouped_gemv_plan(moe_gemv_mode_t mode, int32_t M, int32_t top_k,
                                           int32_t E, int32_t N, int32_t K,
                                           int32_t grouping_given, int32_t *variant,
                                           int32_t *groups_in_kernel);

/* --------------------------------------------------------------------- */
/* Step 5 -- MAX "Struct_ep_combine_wait", execute() (weighted sum with  */
/* the router weights, then the optional elementwise epilogue,           */
/* has_epilogue_fusion).  At one GPU there is nothing to wait for.        */
/*   output_tokens[t, h] = bf16( epi( sum_{j: 0<=id<E} w[t,j]*y[t,j,h] ) ) */
/* fp32 accumulation in slot order; a row with no routed slot gives      */
/* epi(0).  expert_out bf16 [M, top_k, H] (the GEMV output; unrouted     */
/* slots are never used), router_weights fp32 [M, top_k], topk_ids int64 */
/* [M, top_k], output_tokens bf16 [M, H].  H (hidden_size) is the expert */
/* output width.  Limits: H % 8 == 0, 16-byte aligned bf16 buffers.       */
/* output_tokens may be pinned host memory (a device-accessible pointer   */
/* under unified addressing): the result then reaches the host through   */
/* the kernel's own stores, without a separate copy.                     */
MOE_API moe_status_t moe_combine(const void *expert_out, const float *router_weights,
                         const int64_t *topk_ids, int32_t M, int32_t top_k, int32_t H, int32_t E,
                         moe_epilogue_t epi, float alpha, void *output_tokens, cudaStream_t s);

/* --------------------------------------------------------------------- */
/* Diagnostics.                                                          */
MOE_API const char *moe_status_string(moe_status_t st);
/* Copies the current device's error word to *host_flags (host pointer)  */
/* and clears it when clear != 0.  Synchronises the device.              */
MOE_API moe_status_t moe_get_device_error(uint32_t *host_flags, int32_t clear);
/* Library version as major*10000 + minor*100 + patch. */
MOE_API int32_t moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_ROUTE_H_ */
