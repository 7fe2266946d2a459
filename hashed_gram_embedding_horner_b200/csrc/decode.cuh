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

// The step for sequence b one dependent load at a time: the commit (append_entry), then the
// hash of each id against the updated ring. Any number of ids.
__device__ __forceinline__ void commit_hash_warp(const CacheParams& c, const HashParams& h, int32_t b, int lane) {
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

// The same step for sequence b with its loads in three rounds: what depends on b alone (slot,
// commit count, offsets); then the history length, the ids to commit and this step's ids;
// then the ring entries the windows reach. The committed ids enter the windows from the
// commit buffer instead of being read back from the ring: a window position either holds one
// of them or lay in the ring before the commit, and the commit overwrites no position a
// window reads (an overwritten one is older than the new valid_from: evicted). Same ring,
// indices and status bits as commit_hash_warp. Returns false, having done nothing, when more
// than 32 ids are to be committed or hashed (one per lane).
__device__ __forceinline__ bool commit_hash_warp_fast(const CacheParams& c, const HashParams& h, int32_t b,
                                                      int lane) {
  constexpr unsigned kAll = 0xffffffffu;
  int32_t v = 0;
  if (lane == 0) v = h.slots ? h.slots[b] : b;
  else if (lane == 1) v = c.counts ? c.counts[b] : 0;
  else if (lane == 2) v = h.offsets[b];
  else if (lane == 3) v = h.offsets[b + 1];
  const int32_t slot = __shfl_sync(kAll, v, 0), m = __shfl_sync(kAll, v, 1);
  const int64_t start = __shfl_sync(kAll, v, 2), end = __shfl_sync(kAll, v, 3);
  if ((c.counts && m > 32) || end - start > 32) return false;
  const bool slot_ok = slot >= 0 && slot < h.max_seqs;
  bool commit = c.counts != nullptr && slot_ok;
  const int32_t cb = b * c.stride;  // entry b's ids in the commit buffer
  if (commit && (cb < 0 || m < 0 || m > c.capacity || m > c.stride)) {
    if (lane == 0) set_status(c.status, (cb < 0 || m < 0) ? NGRAM_STATUS_BAD_OFFSETS : NGRAM_STATUS_BAD_APPEND);
    commit = false;
  }
  const bool offsets_ok = !((b == 0 && start != 0) || start < 0 || end < start || end > h.T ||
                            (b + 1 == h.num_seqs && end != h.T));
  const int ntok = offsets_ok ? static_cast<int>(end - start) : 0;
  // a bad slot is flagged by the commit, and by the hash once the offsets pass
  if (!slot_ok && (c.counts || offsets_ok) && lane == 0) set_status(h.status, NGRAM_STATUS_BAD_SLOT);

  // round 2
  int64_t lv = 0;
  if (slot_ok && lane < 2) lv = lane == 0 ? c.len[slot] : c.valid_from[slot];
  const int32_t ctok = (commit && lane < m) ? c.tokens[cb + lane] : 0;
  const int32_t stok = lane < ntok ? h.tokens[start + lane] : 0;
  const int64_t L = __shfl_sync(kAll, lv, 0), VF = __shfl_sync(kAll, lv, 1);
  if (commit && __any_sync(kAll, lane < m && (ctok < 0 || static_cast<uint32_t>(ctok) >= c.V0))) {
    if (lane == 0) set_status(c.status, NGRAM_STATUS_BAD_TOKEN);
    commit = false;
  }
  const int64_t len_new = commit ? L + m : L;
  const int64_t vf_new = (commit && len_new - c.capacity > VF) ? len_new - c.capacity : VF;

  // round 3: the ring entries (older than the commit, not evicted) this lane's window needs
  const int64_t i = start + lane;
  int32_t rv[kMaxN], sv[kMaxN], cv[kMaxN];
#pragma unroll
  for (int j = 0; j < kMaxN; ++j) {
    if (j >= h.N) break;
    const int64_t pos = len_new + (i - j - start);  // history position of a token before the step
    rv[j] = 0;
    if (lane < ntok && i - j < start && slot_ok && pos >= 0 && pos >= vf_new && pos < L)
      rv[j] = h.ring[static_cast<int64_t>(slot) * h.capacity + (pos % h.capacity)];
    sv[j] = __shfl_up_sync(kAll, stok, j);  // this step's id at i - j (lane - j)
    const int64_t src = pos - L;            // one of the ids committed now
    cv[j] = __shfl_sync(kAll, ctok, (src >= 0 && src < 32) ? static_cast<int>(src) : 0);
  }

  if (commit) {
    if (lane < m) c.ring[static_cast<int64_t>(slot) * c.capacity + ((L + lane) % c.capacity)] = ctok;
    if (lane == 0) {
      c.len[slot] = len_new;
      if (len_new - c.capacity > VF) c.valid_from[slot] = len_new - c.capacity;
    }
  }
  if (!offsets_ok) {
    if (lane == 0) set_status(h.status, NGRAM_STATUS_BAD_OFFSETS);
    return true;
  }
  if (lane < ntok) {
    uint32_t u[kMaxN];
#pragma unroll
    for (int j = 0; j < kMaxN; ++j) {
      if (j >= h.N) break;
      int64_t t = 0;
      if (i - j >= start) {
        t = sv[j];
      } else if (slot_ok) {
        const int64_t pos = len_new + (i - j - start);
        if (pos >= 0) {
          if (pos < vf_new) set_status(h.status, NGRAM_STATUS_EVICTED);
          else t = pos >= L ? cv[j] : rv[j];
        }
      }
      if (t < 0 || t >= h.V0) {
        set_status(h.status, NGRAM_STATUS_BAD_TOKEN);
        t = 0;
      }
      u[j] = static_cast<uint32_t>(t);
    }
    hash_window(h, i, start, slot_ok ? slot : -1, u);
  }
  return true;
}

__global__ void __launch_bounds__(256) commit_hash_kernel(const __grid_constant__ CacheParams c,
                                                          const __grid_constant__ HashParams h) {
  pdl_launch_dependents();
  pdl_wait();
  const int32_t b = static_cast<int32_t>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= h.num_seqs) return;
  if (!commit_hash_warp_fast(c, h, b, lane)) commit_hash_warp(c, h, b, lane);
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
