// Context assembly + n-gram hash (Eq. 2 of "Scaling Embeddings Outperforms Scaling
// Experts in Language Models", section 2):
//   idx[i][s] = (sum_{j=0}^{n-1} t_{i-j} V0^j) mod V_{n,k},   s = (n-2)K + (k-1)
// evaluated exactly by Horner's rule from the oldest id, h <- (h * V0 + t) mod V,
// each step reduced with Barrett's method (P. Barrett, CRYPTO 1986) against a
// per-modulus reciprocal m = floor((2^64 - 1) / V). With h, t, V0 < 2^31 every
// intermediate h * V0 + t < 2^63, so nothing wraps.
//
// Context: ids before a sequence start are the pad id 0 (prefill) or the sequence's
// committed history in the N-gram cache ring (decode, section 4.2 "N-gram Cache").
#pragma once

#include "common.cuh"

namespace ngram {

struct HashParams {
  const int32_t* tokens;   // [T]
  const int32_t* offsets;  // [num_seqs + 1]
  int32_t num_seqs;
  int64_t T;
  uint32_t V0;
  int N, K, S;
  uint32_t V[kMaxS];
  uint64_t barrett[kMaxS];
  // decode context (ring == nullptr: prefill, pad 0)
  const int32_t* ring;
  const int64_t* len;
  const int64_t* valid_from;
  const int32_t* slots;  // nullptr: slot b for sequence b
  int32_t capacity;
  int32_t max_seqs;
  int32_t* idx_out;  // [T * S]
  // draft-phase embedding cache: the window ids (oldest first) of every token, [T * N], and
  // its cache entry slot * positions + (i - sequence start), or -1 past `positions`
  int32_t* win_out;
  int32_t* entry_out;
  int32_t positions;
  int* status;
};

// (h * V0 + t) mod V for h < V < 2^31, V0 < 2^31, t < 2^31.
__device__ __forceinline__ uint32_t horner_step(uint32_t h, uint32_t V0, uint32_t t, uint32_t V,
                                                uint64_t m) {
  const uint64_t x = static_cast<uint64_t>(h) * V0 + t;
  const uint64_t q = __umul64hi(x, m);
  uint64_t r = x - q * V;  // in [0, 2V)
  if (r >= V) r -= V;
  return static_cast<uint32_t>(r);
}

// Eq. 2 for token i from its window u (u[j] = t_{i-j}, newest first, ids already checked),
// and the draft-phase records of the window when asked for.
__device__ __forceinline__ void hash_window(const HashParams& p, int64_t i, int64_t start, int32_t slot,
                                            const uint32_t (&u)[kMaxN]) {
  if (p.win_out) {
    for (int j = 0; j < p.N; ++j) p.win_out[i * p.N + j] = static_cast<int32_t>(u[p.N - 1 - j]);
    const int64_t jpos = i - start;
    p.entry_out[i] = (slot >= 0 && jpos < p.positions) ? static_cast<int32_t>(slot * p.positions + jpos) : -1;
  }
  int32_t* out = p.idx_out + i * p.S;
  for (int n = 2; n <= p.N; ++n) {
    for (int k = 0; k < p.K; ++k) {
      const int s = (n - 2) * p.K + k;
      const uint32_t V = p.V[s];
      const uint64_t m = p.barrett[s];
      uint32_t h = 0;
      for (int j = n - 1; j >= 0; --j) h = horner_step(h, p.V0, u[j], V, m);
      out[s] = static_cast<int32_t>(h);
    }
  }
}

// Eq. 2 for token i of a sequence starting at `start`, with the sequence's committed
// history (slot >= 0: hist_len ids, those before hist_from evicted) before it.
__device__ __forceinline__ void hash_one(const HashParams& p, int64_t i, int64_t start, int32_t slot,
                                         int64_t hist_len, int64_t hist_from) {
  // u[j] = t_{i-j}, newest first.
  uint32_t u[kMaxN];
#pragma unroll
  for (int j = 0; j < kMaxN; ++j) {
    if (j >= p.N) break;
    const int64_t a = i - j;  // absolute token position if inside this call's sequence
    int64_t t = 0;
    if (a >= start && a >= 0) {
      t = p.tokens[a];
    } else if (slot >= 0) {
      const int64_t pos = hist_len + (a - start);  // position in the committed history
      if (pos >= 0) {
        if (pos < hist_from) {
          set_status(p.status, NGRAM_STATUS_EVICTED);
        } else {
          t = p.ring[static_cast<int64_t>(slot) * p.capacity + (pos % p.capacity)];
        }
      }
    }
    if (t < 0 || t >= p.V0) {
      set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
      t = 0;
    }
    u[j] = static_cast<uint32_t>(t);
  }
  hash_window(p, i, start, slot, u);
}

constexpr int kHashSmemOffsets = 4096;  // offsets staged in shared memory when B + 1 fits

__global__ void __launch_bounds__(256) hash_kernel(const __grid_constant__ HashParams p) {
  __shared__ int32_t s_off[kHashSmemOffsets];
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();

  // Offsets check (sticky status; the lookups below stay in bounds regardless).
  if (i <= p.num_seqs) {
    const int32_t o = p.offsets[i];
    const bool bad = (i == 0 && o != 0) || (i == p.num_seqs && o != p.T) ||
                     (i < p.num_seqs && p.offsets[i + 1] < o);
    if (bad) set_status(p.status, NGRAM_STATUS_BAD_OFFSETS);
  }
  // Small batches: one coalesced pass brings every offset into shared memory, so the
  // sequence search below costs no dependent global loads.
  const bool staged = p.num_seqs + 1 <= kHashSmemOffsets;
  if (staged) {
    for (int k = threadIdx.x; k <= p.num_seqs; k += blockDim.x) s_off[k] = p.offsets[k];
    __syncthreads();
  }
  if (i >= p.T) return;

  // Sequence of token i: the largest b with offsets[b] <= i.
  int32_t lo = 0, hi = p.num_seqs;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if ((staged ? s_off[mid] : p.offsets[mid]) <= i) lo = mid; else hi = mid;
  }
  const int64_t start = staged ? s_off[lo] : p.offsets[lo];

  int32_t slot = -1;
  int64_t hist_len = 0, hist_from = 0;
  if (p.ring) {
    slot = p.slots ? p.slots[lo] : lo;
    if (slot < 0 || slot >= p.max_seqs) {
      set_status(p.status, NGRAM_STATUS_BAD_SLOT);
      slot = -1;
    } else {
      hist_len = p.len[slot];
      hist_from = p.valid_from[slot];
    }
  }

  hash_one(p, i, start, slot, hist_len, hist_from);
}

}  // namespace ngram
