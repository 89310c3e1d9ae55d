// Weight Page Table kernels (PagedWeight, "Composants Clés" 1 and 3): stream-ordered commits of
// q_i, so a commit lands exactly between two forward calls (a safe boundary).
#pragma once
#include "pw_common.cuh"

namespace pw {

__global__ void commit_bits_kernel(pw_page_table* __restrict__ pt, int num_blocks,
                                   const int32_t* __restrict__ ids, const uint8_t* __restrict__ q,
                                   int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const long long table_blocks = static_cast<long long>(pt->num_layers) * pt->num_experts * 2;
  const int bid = ids[i];
  if (bid < 0 || bid >= num_blocks || bid >= table_blocks) {
    set_status(PW_ERR_BAD_BITS);
    return;
  }
  pw_block* b = pt->blocks + bid;
  const int qq = q[i];
  if (qq < b->min_bits || qq > b->parent_bits || qq < 1 || qq > PW_MAX_BITS ||
      b->lut[qq] == nullptr) {
    set_status(PW_ERR_BAD_BITS);
    return;
  }
  b->committed_bits = static_cast<uint8_t>(qq);
}

}  // namespace pw
