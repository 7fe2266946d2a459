// Hash statistics of an n-gram table (section 3.2.2 and Fig. 3 of "Scaling Embeddings
// Outperforms Scaling Experts in Language Models"):
//   hit rate    = (rows of the table hit at least once by the stream) / V
//   collisions  = (distinct n-gram windows in the stream) - (distinct rows they hash to),
// i.e. the unique n-gram representations lost to the modulus. Windows use the layer's
// context rule (pad id 0 before a sequence start) and Eq. 2's hash X_n mod V.
//
// Distinct windows: when V0^n < 2^64, the exact X_n (a bijection of the window when every
// id is < V0) is inserted into an open-addressing set of 64-bit keys (atomicCAS, linear
// probing). Otherwise (n >= 4 at V0 = 2^17) the window itself is the key: its n ids packed
// two to a 64-bit word (at most 4 words), written by one launch; a second launch inserts
// position indices into the set, and a probe that meets an occupied slot compares the
// occupant's packed window with its own word by word (both written by the first launch), so
// equal windows always meet in the same probe chain and exactly one of them is counted.
// Distinct rows, per modulus: one bit per row (atomicOr); a thread whose OR set the bit
// counts it (one atomic add per warp).
#pragma once

#include "hash.cuh"

namespace ngram {

constexpr unsigned long long kSetEmpty = ~0ull;  // never a key: every X_n <= V0^n - 1 < 2^64 - 1,
                                                  // never a position index
constexpr int kWinWords = kMaxN / 2;              // 64-bit words of a packed window

struct StatsParams {
  const int32_t* tokens;
  const int32_t* offsets;
  int32_t num_seqs;
  int64_t T;
  uint32_t V0;
  int n;
  bool exact64;                  // V0^n < 2^64: X_n kept exactly
  unsigned long long* keys;      // [T] exact X_n (exact64), else [T x kWinWords] packed windows
  unsigned long long* set;       // [set_mask + 1]
  uint64_t set_mask;
  unsigned long long* distinct;  // distinct windows
  uint32_t V;                    // modulus of this pass
  uint64_t barrett;
  uint32_t* bitmap;              // [V / 32 + 1]
  unsigned long long* rows_hit;  // this modulus's counter
  int* status;
};

// The n ids of position i's window, oldest first (pad 0 before the sequence start).
__device__ __forceinline__ void stats_window(const StatsParams& p, int64_t i, uint32_t (&w)[kMaxN]) {
  int32_t lo = 0, hi = p.num_seqs;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (p.offsets[mid] <= i) lo = mid; else hi = mid;
  }
  const int64_t start = p.offsets[lo];
  for (int j = 0; j < p.n; ++j) {  // w[0] = t_{i-n+1}, ..., w[n-1] = t_i
    const int64_t pos = i - (p.n - 1) + j;
    uint32_t t = 0;
    if (pos >= start) {
      const int32_t v = p.tokens[pos];
      if (static_cast<uint32_t>(v) >= p.V0) set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
      else t = static_cast<uint32_t>(v);
    }
    w[j] = t;
  }
}

__device__ __forceinline__ uint64_t mix64(uint64_t x) {  // SplitMix64's finaliser
  x ^= x >> 30;
  x *= 0xbf58476d1ce4e5b9ull;
  x ^= x >> 27;
  x *= 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}

// Exact keys of every position, inserted into the set; counts distinct windows.
__global__ void __launch_bounds__(256) stats_keys_kernel(const __grid_constant__ StatsParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  bool fresh = false;
  if (i < p.T) {
    uint32_t w[kMaxN];
    stats_window(p, i, w);
    unsigned long long x = 0;
    for (int j = 0; j < p.n; ++j) x = x * p.V0 + w[j];  // < V0^n < 2^64: exact
    p.keys[i] = x;
    uint64_t h = mix64(x) & p.set_mask;
    for (uint64_t probe = 0; probe <= p.set_mask; ++probe) {  // the set is at least twice T
      const unsigned long long prev = atomicCAS(p.set + h, kSetEmpty, x);
      if (prev == kSetEmpty) { fresh = true; break; }
      if (prev == x) break;
      h = (h + 1) & p.set_mask;
    }
  }
  const unsigned ballot = __ballot_sync(0xffffffffu, fresh);
  if ((threadIdx.x & 31) == 0 && ballot) atomicAdd(p.distinct, static_cast<unsigned long long>(__popc(ballot)));
}

// Packed windows (V0^n >= 2^64): word k holds ids 2k (low half) and 2k + 1 of the window,
// oldest first; unused halves are zero.
__global__ void __launch_bounds__(256) stats_window_keys_kernel(const __grid_constant__ StatsParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= p.T) return;
  uint32_t w[kMaxN];
  stats_window(p, i, w);
#pragma unroll
  for (int k = 0; k < kWinWords; ++k) {
    const uint32_t lo = 2 * k < p.n ? w[2 * k] : 0u;
    const uint32_t hi = 2 * k + 1 < p.n ? w[2 * k + 1] : 0u;
    p.keys[i * kWinWords + k] = static_cast<unsigned long long>(lo) | (static_cast<unsigned long long>(hi) << 32);
  }
}

// Inserts every position into the set of distinct packed windows; counts distinct windows.
__global__ void __launch_bounds__(256) stats_window_insert_kernel(const __grid_constant__ StatsParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  bool fresh = false;
  if (i < p.T) {
    unsigned long long key[kWinWords];
    uint64_t f = 0x9e3779b97f4a7c15ull;
#pragma unroll
    for (int k = 0; k < kWinWords; ++k) {
      key[k] = p.keys[i * kWinWords + k];
      f = mix64(f ^ key[k]);
    }
    uint64_t h = f & p.set_mask;
    for (uint64_t probe = 0; probe <= p.set_mask; ++probe) {  // the set is at least twice T
      const unsigned long long prev = atomicCAS(p.set + h, kSetEmpty, static_cast<unsigned long long>(i));
      if (prev == kSetEmpty) { fresh = true; break; }
      bool same = true;
#pragma unroll
      for (int k = 0; k < kWinWords; ++k) same &= p.keys[static_cast<int64_t>(prev) * kWinWords + k] == key[k];
      if (same) break;
      h = (h + 1) & p.set_mask;
    }
  }
  const unsigned ballot = __ballot_sync(0xffffffffu, fresh);
  if ((threadIdx.x & 31) == 0 && ballot) atomicAdd(p.distinct, static_cast<unsigned long long>(__popc(ballot)));
}

// Row of every position under modulus V; counts distinct rows.
__global__ void __launch_bounds__(256) stats_rows_kernel(const __grid_constant__ StatsParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  bool fresh = false;
  if (i < p.T) {
    uint32_t r;
    if (p.exact64) {
      const unsigned long long x = p.keys[i];
      const uint64_t q = __umul64hi(x, p.barrett);  // floor(x / V) or one less
      uint64_t rr = x - q * p.V;
      if (rr >= p.V) rr -= p.V;
      r = static_cast<uint32_t>(rr);
    } else {
      uint32_t w[kMaxN];
      stats_window(p, i, w);
      r = 0;
      for (int j = 0; j < p.n; ++j) r = horner_step(r, p.V0 % p.V, w[j] % p.V, p.V, p.barrett);
    }
    const uint32_t bit = 1u << (r & 31);
    fresh = (atomicOr(p.bitmap + (r >> 5), bit) & bit) == 0;
  }
  const unsigned ballot = __ballot_sync(0xffffffffu, fresh);
  if ((threadIdx.x & 31) == 0 && ballot) atomicAdd(p.rows_hit, static_cast<unsigned long long>(__popc(ballot)));
}

}  // namespace ngram
