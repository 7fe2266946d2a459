// One decode step's cache update and context hashing in a single launch: a warp per
// sequence first commits the ids accepted in the previous step to the sequence's N-gram
// cache ring (section 4.2 of "Scaling Embeddings Outperforms Scaling Experts in Language
// Models", the N-gram Cache), then hashes this step's ids (Eq. 2) against the updated
// history. The same results as ngram_cache_commit followed by the hash of
// ngram_embed_fwd, with one launch fewer per step.
#pragma once

#include "hash.cuh"
#include "simt.cuh"

namespace ngram {

__global__ void __launch_bounds__(256) commit_hash_kernel(const __grid_constant__ CacheParams c,
                                                          const __grid_constant__ HashParams h) {
  pdl_launch_dependents();
  pdl_wait();
  const int32_t b = static_cast<int32_t>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= h.num_seqs) return;
  if (c.counts) append_entry(c, b, lane);
  __syncwarp();  // the ring, len and valid_from written above are visible to the whole warp
  const int64_t start = h.offsets[b], end = h.offsets[b + 1];
  if ((b == 0 && start != 0) || start < 0 || end < start || end > h.T || (b + 1 == h.num_seqs && end != h.T)) {
    if (lane == 0) set_status(h.status, NGRAM_STATUS_BAD_OFFSETS);
    return;
  }
  int32_t slot = h.slots ? h.slots[b] : b;
  int64_t hist_len = 0, hist_from = 0;
  if (slot < 0 || slot >= h.max_seqs) {
    if (lane == 0) set_status(h.status, NGRAM_STATUS_BAD_SLOT);
    slot = -1;
  } else {
    hist_len = h.len[slot];
    hist_from = h.valid_from[slot];
  }
  for (int64_t i = start + lane; i < end; i += 32) hash_one(h, i, start, slot, hist_len, hist_from);
}

}  // namespace ngram
