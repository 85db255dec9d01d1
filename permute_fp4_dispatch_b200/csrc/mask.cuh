// mask.cuh -- step 1: mask CUDA-graph padding rows of the routing map.
//
// Megatron-Core "core.transformer.moe.inference_routing_mask_kernel",
// mask_routing_padding: every top_k slot of local row r with
// r + tp_rank * N >= real_token_count becomes -1.  The count is read from
// device memory inside the kernel, so a captured graph follows the value
// that is current at replay time.
#pragma once
#include "common.cuh"

namespace moe {

// Grid-stride over the masked tail of the flattened [N, top_k] map.  The
// masked region is a contiguous suffix, so each thread writes whole int64
// slots with no per-row test.  The next grid in the stream may be scheduled
// at once: the kernels of this library that follow it run their input-free
// set-up (barriers, descriptor and L2 prefetches) meanwhile and read the map
// only after their own wait for this grid's completion.
__global__ void __launch_bounds__(256) mask_padding_kernel(int64_t *__restrict__ map, int32_t N,
                                                           int32_t top_k,
                                                           const int32_t *__restrict__ real_ptr,
                                                           int32_t tp_rank) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t real = static_cast<int64_t>(*real_ptr);
  int64_t first = real - static_cast<int64_t>(tp_rank) * N;  // first masked local row
  first = first < 0 ? 0 : (first > N ? N : first);
  const int64_t begin = first * top_k;
  const int64_t end = static_cast<int64_t>(N) * top_k;
  for (int64_t i = begin + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < end;
       i += (int64_t)gridDim.x * blockDim.x)
    map[i] = -1;
}

}  // namespace moe
