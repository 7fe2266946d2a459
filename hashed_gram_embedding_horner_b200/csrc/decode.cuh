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

// The same step for the dense-A projection, which reads the step's sub-rows from G: one
// launch commits, hashes and gathers. A block per sequence: warp 0 commits the ids accepted
// in the previous step and hashes this step's ids against the updated history, 32 ids at a
// time, keeping their indices in shared memory as well; then all 8 warps copy the sub-rows
// those indices select into G (row i of G: the concatenated sub-rows of token i), each
// thread issuing its loads before its stores. The indices, the ring and G equal those of
// ngram_cache_commit, the hash and the gather kernel launched one after another.
__global__ void __launch_bounds__(256) commit_hash_gather_kernel(const __grid_constant__ CacheParams c,
                                                                 const __grid_constant__ HashParams h,
                                                                 const __grid_constant__ GatherParams g) {
  __shared__ int32_t s_idx[32 * kMaxS];
  __shared__ int64_t s_start, s_end, s_len, s_from;
  __shared__ int32_t s_slot;
  __shared__ int s_ok;
  pdl_launch_dependents();
  pdl_wait();
  const int32_t b = static_cast<int32_t>(blockIdx.x);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == 0) {
    if (c.counts) append_entry(c, b, lane);
    __syncwarp();  // the ring, len and valid_from written above are visible to the whole warp
    if (lane == 0) {
      const int64_t start = h.offsets[b], end = h.offsets[b + 1];
      const bool bad = (b == 0 && start != 0) || start < 0 || end < start || end > h.T ||
                       (b + 1 == h.num_seqs && end != h.T);
      if (bad) set_status(h.status, NGRAM_STATUS_BAD_OFFSETS);
      int32_t slot = h.slots ? h.slots[b] : b;
      int64_t hist_len = 0, hist_from = 0;
      if (slot < 0 || slot >= h.max_seqs) {
        set_status(h.status, NGRAM_STATUS_BAD_SLOT);
        slot = -1;
      } else {
        hist_len = h.len[slot];
        hist_from = h.valid_from[slot];
      }
      s_ok = bad ? 0 : 1;
      s_start = start;
      s_end = end;
      s_slot = slot;
      s_len = hist_len;
      s_from = hist_from;
    }
  }
  __syncthreads();
  if (!s_ok) return;  // block-uniform
  const int64_t start = s_start, end = s_end;
  const int S = h.S;
  const uint32_t vec_per_row = static_cast<uint32_t>(g.row_bytes >> 4);
  for (int64_t c0 = start; c0 < end; c0 += 32) {
    const int ntok = static_cast<int>(end - c0 < 32 ? end - c0 : 32);
    if (warp == 0 && lane < ntok) {
      const int64_t i = c0 + lane;
      hash_one(h, i, start, s_slot, s_len, s_from);
      for (int s = 0; s < S; ++s) s_idx[lane * S + s] = h.idx_out[i * S + s];  // this thread's own writes
    }
    __syncthreads();
    // vectors of the chunk's G rows, numbered row-major: (token, sub-table, 16-byte vector)
    const uint32_t nvec = static_cast<uint32_t>(ntok * S) * vec_per_row;
    uint8_t* dst0 = g.G + c0 * S * static_cast<int64_t>(g.row_bytes);
    for (uint32_t base = threadIdx.x; base < nvec; base += 256u * kGatherUnroll) {
      uint4 v[kGatherUnroll];
#pragma unroll
      for (int j = 0; j < kGatherUnroll; ++j) {
        const uint32_t vi = base + j * 256u;
        if (vi < nvec) {
          uint32_t cv;
          const uint32_t row = split_vec(vi, g.vshift, vec_per_row, cv);  // token * S + sub-table
          const uint32_t s = row % static_cast<uint32_t>(S);
          int32_t r = s_idx[row];
          if (static_cast<uint32_t>(r) >= g.Vs[s]) {
            set_status(g.status, NGRAM_STATUS_BAD_TOKEN);
            r = 0;
          }
          v[j] = ld_stream_v4(g.E[s] + static_cast<int64_t>(r) * g.row_bytes + cv * 16);
        }
      }
#pragma unroll
      for (int j = 0; j < kGatherUnroll; ++j) {
        const uint32_t vi = base + j * 256u;
        if (vi < nvec) *reinterpret_cast<uint4*>(dst0 + static_cast<int64_t>(vi) * 16) = v[j];
      }
    }
    __syncthreads();  // s_idx is rewritten by the next chunk
  }
}

}  // namespace ngram
