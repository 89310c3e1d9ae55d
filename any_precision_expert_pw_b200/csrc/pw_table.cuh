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
  const int stored = b->stored_bits ? b->stored_bits : b->parent_bits;
  if (qq < b->min_bits || qq > stored || qq < 1 || qq > PW_MAX_BITS ||
      b->lut[qq] == nullptr) {
    set_status(PW_ERR_BAD_BITS);
    return;
  }
  b->committed_bits = static_cast<uint8_t>(qq);
}

// Stream-ordered page-table edits (page movement, PagedWeight "Composants Clés" 1 and 3): each
// update sets, for one block, whichever of state / stored_bits / committed_bits / planes it
// carries (0 or null = unchanged).  An edit that would leave the entry inconsistent is
// skipped and PW_ERR_BAD_BITS recorded.
__global__ void page_update_kernel(pw_page_table* __restrict__ pt, int num_blocks,
                                   const pw_page_update_t* __restrict__ up, int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const pw_page_update_t u = up[i];
  const long long table_blocks = static_cast<long long>(pt->num_layers) * pt->num_experts * 2;
  if (u.block < 0 || u.block >= num_blocks || u.block >= table_blocks) {
    set_status(PW_ERR_BAD_BITS);
    return;
  }
  pw_block* b = pt->blocks + u.block;
  const int state = u.state ? u.state - 1 : b->state;  // state is stored + 1 (0 = unchanged)
  const int stored = u.stored_bits ? u.stored_bits : (b->stored_bits ? b->stored_bits
                                                                     : b->parent_bits);
  const int q = u.committed_bits ? u.committed_bits : b->committed_bits;
  const bool ok = state >= PW_PAGE_GPU && state <= PW_PAGE_XFER && stored >= b->min_bits &&
                  stored <= b->parent_bits && q >= b->min_bits && q <= stored &&
                  b->lut[q] != nullptr && (reinterpret_cast<uintptr_t>(u.planes) & 15) == 0;
  if (!ok) {
    set_status(PW_ERR_BAD_BITS);
    return;
  }
  if (u.planes) b->planes = u.planes;
  b->stored_bits = static_cast<uint8_t>(stored);
  b->committed_bits = static_cast<uint8_t>(q);
  b->state = static_cast<uint8_t>(state);
}

}  // namespace pw
