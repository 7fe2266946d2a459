// Draft-phase N-gram embedding cache (section 4.2 of "Scaling Embeddings Outperforms
// Scaling Experts in Language Models", optimisations for speculative decoding: cache the
// n-gram embeddings computed while drafting so that verification does not compute them
// again).
//
// An entry per (cache slot, in-step position) holds the N ids of the window its embedding
// was computed for and the embedding row. The layer's output for a token depends only on
// its window (E_0 row of the newest id, sub-table rows of Eq. 2's hashes of the window), so
// a token whose window equals its entry's key takes the stored row: nothing needs to be
// invalidated when drafts are rejected or the history moves on — a changed window is a
// different key. Per call: the hash kernel also writes each token's window and entry; the
// probe kernel copies hits and compacts misses (token, indices, entry) into a list; the
// projection runs on the misses only, with their count read on the device; the scatter
// kernel places the computed rows in the output and in the cache.
#pragma once

#include "common.cuh"

namespace ngram {

struct DraftParams {
  const int32_t* tokens;
  const int32_t* idx;      // [T * S] this call's indices
  const int32_t* win;      // [T * N] windows (oldest first)
  const int32_t* entry;    // [T] cache entry, or -1 (no entry: computed, not cached)
  int32_t* keys;           // [entries * N]; key[0] == -1: empty
  uint8_t* emb;            // [entries * row_bytes]
  int64_t T;
  int N, S;
  int row_bytes;           // D * element size (a multiple of 16)
  uint8_t* out;            // [T * row_bytes]
  // misses, compacted
  int32_t* miss_count;
  int32_t* miss_token;     // [T] token ids (projection input)
  int32_t* miss_idx;       // [T * S] their indices (projection input)
  int32_t* miss_pos;       // [T] their positions in this call
  int32_t* miss_entry;     // [T] their cache entries (or -1)
  const uint8_t* miss_out; // [T * row_bytes] the projection's rows for the misses
  int32_t* hits;           // optional counter of hits
};

__device__ __forceinline__ void copy_row(uint8_t* dst, const uint8_t* src, int row_bytes, int lane) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int v = lane; v < (row_bytes >> 4); v += 32) d[v] = s[v];
}

// One warp per token: compare the window with the entry's key; copy a hit, list a miss.
__global__ void __launch_bounds__(256) draft_probe_kernel(const __grid_constant__ DraftParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= p.T) return;
  const int32_t e = p.entry[i];
  bool same = e >= 0;
  if (same && lane < p.N) same = p.keys[static_cast<int64_t>(e) * p.N + lane] == p.win[i * p.N + lane];
  same = __all_sync(0xffffffffu, same);
  if (same) {
    copy_row(p.out + i * p.row_bytes, p.emb + static_cast<int64_t>(e) * p.row_bytes, p.row_bytes, lane);
    if (lane == 0 && p.hits) atomicAdd(p.hits, 1);
    return;
  }
  int32_t k = 0;
  if (lane == 0) k = atomicAdd(p.miss_count, 1);
  k = __shfl_sync(0xffffffffu, k, 0);
  if (lane == 0) {
    p.miss_token[k] = p.tokens[i];
    p.miss_pos[k] = static_cast<int32_t>(i);
    p.miss_entry[k] = e;
  }
  if (lane < p.S) p.miss_idx[static_cast<int64_t>(k) * p.S + lane] = p.idx[i * p.S + lane];
  if (e >= 0 && lane < p.N) p.keys[static_cast<int64_t>(e) * p.N + lane] = p.win[i * p.N + lane];
}

// One warp per miss: the computed row to its place in the output and to its cache entry.
__global__ void __launch_bounds__(256) draft_scatter_kernel(const __grid_constant__ DraftParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t k = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (k >= *p.miss_count) return;
  const uint8_t* src = p.miss_out + k * p.row_bytes;
  copy_row(p.out + static_cast<int64_t>(p.miss_pos[k]) * p.row_bytes, src, p.row_bytes, lane);
  const int32_t e = p.miss_entry[k];
  if (e >= 0) copy_row(p.emb + static_cast<int64_t>(e) * p.row_bytes, src, p.row_bytes, lane);
}

// Empty the entries of the given slots (key[0] = -1), or of every slot if slots is null.
struct DraftResetParams {
  int32_t* keys;
  const int32_t* slots;
  int32_t n;           // slots to reset
  int32_t positions;
  int N;
  int32_t max_seqs;
  int* status;
};

__global__ void __launch_bounds__(256) draft_reset_kernel(const __grid_constant__ DraftResetParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(p.n) * p.positions) return;
  const int32_t b = static_cast<int32_t>(t / p.positions);
  const int32_t j = static_cast<int32_t>(t - static_cast<int64_t>(b) * p.positions);
  const int32_t slot = p.slots ? p.slots[b] : b;
  if (slot < 0 || slot >= p.max_seqs) {
    set_status(p.status, NGRAM_STATUS_BAD_SLOT);
    return;
  }
  p.keys[(static_cast<int64_t>(slot) * p.positions + j) * p.N] = -1;
}

}  // namespace ngram
