// Cache update (scatter of new tokens into their slots) and copy-on-write
// block copies.  Both are pure byte movement in 16-byte vectors, so they are
// bit-exact by construction.
#pragma once

#include "pkv_decode.cuh"

namespace pkv {

// New token n goes to slot s = slot_mapping[n]: block s / bs, offset s % bs
// ("Paged Attention Explained", Step 2; a token fills the current block and a
// new block is used only once it is full).  In the [num_blocks][bs][Hkv][D]
// layout the token row of slot s is the s-th row of Hkv*D elements, so the
// copy is one contiguous row of `row_vec` 16-byte vectors per token.
__global__ void __launch_bounds__(256)
    kv_write_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                    uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                    const int64_t* __restrict__ slot_mapping, int64_t row_vec, int64_t num_slots) {
  launch_overlap_entry();
  const int64_t n = blockIdx.x;
  const int64_t s = slot_mapping[n];
  if (s < 0) return;
  if (s >= num_slots) {
    if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(PKV_DEVERR_SLOT);
    return;
  }
  const uint4* ks = k + n * row_vec;
  const uint4* vs = v + n * row_vec;
  uint4* kd = k_cache + s * row_vec;
  uint4* vd = v_cache + s * row_vec;
  for (int64_t i = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; i < row_vec;
       i += (int64_t)gridDim.y * blockDim.x) {
    const uint4 a = __ldg(ks + i);
    const uint4 b = __ldg(vs + i);
    kd[i] = a;
    vd[i] = b;
  }
}

// Pair i copies physical block src to dst in both pools ("PagedAttention:
// paging the KV cache like an OS pages memory", How it works: block-granularity
// copy-on-write).  blockIdx.y strides over the block's vectors.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                       const int64_t* __restrict__ block_mapping, int64_t block_vec,
                       int64_t num_blocks) {
  launch_overlap_entry();
  const int64_t i = blockIdx.x;
  const int64_t src = block_mapping[2 * i];
  const int64_t dst = block_mapping[2 * i + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(PKV_DEVERR_COPY);
    return;
  }
  const uint4* ks = k_cache + src * block_vec;
  const uint4* vs = v_cache + src * block_vec;
  uint4* kd = k_cache + dst * block_vec;
  uint4* vd = v_cache + dst * block_vec;
  for (int64_t j = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; j < block_vec;
       j += (int64_t)gridDim.y * blockDim.x) {
    const uint4 a = ks[j];
    const uint4 b = vs[j];
    kd[j] = a;
    vd[j] = b;
  }
}

}  // namespace pkv
