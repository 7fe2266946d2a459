// CUDA-core kernels: the projection for fp32 tables and for shapes the tensor-core
// kernel does not take (N = 1, D % 128 != 0, d % 64 != 0), the stand-alone sub-row
// gather, and the N-gram cache ring updates.
#pragma once

#include "common.cuh"

namespace ngram {

// ------------------------------------------------------------------ element access

template <typename T> struct Elt;
template <> struct Elt<float> {
  static __device__ __forceinline__ float load(const float* p, int64_t i) { return __ldg(p + i); }
  static __device__ __forceinline__ void store(float* p, int64_t i, float v) { p[i] = v; }
};
template <> struct Elt<uint16_t> {  // bf16 bit patterns
  static __device__ __forceinline__ float load(const uint16_t* p, int64_t i) {
    return bf16_bits_to_float(__ldg(p + i));
  }
  static __device__ __forceinline__ void store(uint16_t* p, int64_t i, float v) {
    p[i] = static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
  }
};

// ------------------------------------------------------------------ SIMT projection

template <typename T>
struct SimtParams {
  const int32_t* tokens;
  const int32_t* idx;
  const T* E0;
  const T* E[kMaxS];
  uint32_t Vs[kMaxS];
  const T* W;
  T* out;
  int64_t T_tokens;
  uint32_t V0;
  int D, S, d;
  int tokens_per_block;
  float scale;
  const int32_t* T_dev;  // if set, the token count is min(*T_dev, T_tokens)
  int* status;
};

// Block = 8 warps over `tokens_per_block` tokens. The tokens' gathered rows G (fp32)
// sit in shared memory; each warp takes output columns o and reduces
// sum_k W[o][k] * G[t][k] across its lanes (coalesced reads of W's row o).
template <typename T>
__global__ void __launch_bounds__(256) proj_simt_kernel(const __grid_constant__ SimtParams<T> p) {
  extern __shared__ float g[];  // [tokens_per_block][D]
  pdl_launch_dependents();
  pdl_wait();
  const int TPB = p.tokens_per_block;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * TPB;
  const int64_t T_eff = p.T_dev ? (*p.T_dev < p.T_tokens ? *p.T_dev : p.T_tokens) : p.T_tokens;
  const int64_t left = T_eff - t0;
  const int nt = static_cast<int>(left < TPB ? left : TPB);
  if (nt <= 0) return;

  for (int e = threadIdx.x; e < nt * p.D; e += blockDim.x) {
    const int t = e / p.D, k = e - t * p.D;
    float v = 0.f;
    if (p.S > 0) {
      const int s = k / p.d, c = k - s * p.d;
      int32_t r = p.idx[(t0 + t) * p.S + s];
      if (static_cast<uint32_t>(r) >= p.Vs[s]) {
        set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
        r = 0;
      }
      v = Elt<T>::load(p.E[s], static_cast<int64_t>(r) * p.d + c);
    }
    g[t * p.D + k] = v;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kMaxTPB = 8;
  int32_t tok[kMaxTPB];
#pragma unroll
  for (int t = 0; t < kMaxTPB; ++t) {
    int32_t x = t < nt ? p.tokens[t0 + t] : 0;
    if (x < 0 || static_cast<uint32_t>(x) >= p.V0) x = 0;  // flagged by the hash stage
    tok[t] = x;
  }
  for (int o = warp; o < p.D; o += 8) {
    float acc[kMaxTPB];
#pragma unroll
    for (int t = 0; t < kMaxTPB; ++t) acc[t] = 0.f;
    if (p.S > 0) {
      for (int k = lane; k < p.D; k += 32) {
        const float w = Elt<T>::load(p.W, static_cast<int64_t>(o) * p.D + k);
#pragma unroll
        for (int t = 0; t < kMaxTPB; ++t)
          if (t < nt) acc[t] = fmaf(w, g[t * p.D + k], acc[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < kMaxTPB; ++t) {
      float a = acc[t];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0 && t < nt) {
        const float e0 = Elt<T>::load(p.E0, static_cast<int64_t>(tok[t]) * p.D + o);
        Elt<T>::store(p.out, (t0 + t) * p.D + o, (a + e0) * p.scale);
      }
    }
  }
}

// ------------------------------------------------------------------ gather (stand-alone)

struct GatherParams {
  const int32_t* idx;
  const uint8_t* E[kMaxS];
  uint32_t Vs[kMaxS];
  uint8_t* G;
  int64_t T;
  int S;
  int row_bytes;  // d * element size, a multiple of 16
  // optional E_0 rows: E0_out[i] = E0[tokens[i]] (E0_out == nullptr: none)
  const int32_t* tokens;
  const uint8_t* E0;
  uint8_t* E0_out;
  uint32_t V0;
  int e0_row_bytes;  // D * element size
  int vshift, eshift;  // log2 of the 16-byte vectors per sub-row / per E_0 row, or -1
  int* status;
};

// 16-byte vectors of G, numbered row-major (row = token * S + s), then (optionally) those
// of the E_0 rows: vector v is copied by thread v mod (threads in the grid), so a warp
// covers 512 contiguous bytes of one row and the grid moves threads x 16 bytes per pass.
// Each thread issues the loads of kGatherUnroll passes before any of their stores, so a
// grid of every resident thread has all rows of a decode step (1280 tokens x (8 sub-rows
// of 1 KiB + one E_0 row of 8 KiB) = 20 MiB) in flight at once.
constexpr int kGatherUnroll = 8;

// Vector index -> (row, vector in row): a shift when the row holds a power of two of
// vectors (always, for d and D multiples of 8 that are powers of two), else a division.
__device__ __forceinline__ uint32_t split_vec(uint32_t v, int shift, uint32_t per_row, uint32_t& c) {
  const uint32_t row = shift >= 0 ? v >> shift : v / per_row;
  c = v - row * per_row;
  return row;
}

__global__ void __launch_bounds__(256) gather_kernel(const __grid_constant__ GatherParams p) {
  pdl_launch_dependents();
  pdl_wait();
  // 32-bit vector numbering (the host launches this kernel only when every index fits):
  // the index arithmetic is per vector, and 64-bit division would cost more than the copy.
  const uint32_t nthreads = gridDim.x * blockDim.x;
  const uint32_t vec_per_row = static_cast<uint32_t>(p.row_bytes >> 4);
  const uint32_t vec_per_e0 = static_cast<uint32_t>(p.e0_row_bytes >> 4);
  const uint32_t S = static_cast<uint32_t>(p.S);
  const uint32_t total_g = static_cast<uint32_t>(p.T) * S * vec_per_row;
  const uint32_t total = total_g + (p.E0_out ? static_cast<uint32_t>(p.T) * vec_per_e0 : 0u);
  for (uint32_t base = blockIdx.x * blockDim.x + threadIdx.x; base < total; base += nthreads * kGatherUnroll) {
    uint4 v[kGatherUnroll];
    uint8_t* dst[kGatherUnroll];
#pragma unroll
    for (int j = 0; j < kGatherUnroll; ++j) {
      const uint32_t vi = base + j * nthreads;
      dst[j] = nullptr;
      if (vi < total_g) {
        uint32_t c;
        const uint32_t row = split_vec(vi, p.vshift, vec_per_row, c);
        const uint32_t s = row % S;
        int32_t r = __ldg(p.idx + row);
        if (static_cast<uint32_t>(r) >= p.Vs[s]) {
          set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
          r = 0;
        }
        v[j] = ld_stream_v4(p.E[s] + static_cast<int64_t>(r) * p.row_bytes + c * 16);
        dst[j] = p.G + static_cast<int64_t>(vi) * 16;
      } else if (vi < total) {
        const uint32_t e = vi - total_g;
        uint32_t c;
        const uint32_t i = split_vec(e, p.eshift, vec_per_e0, c);
        int32_t t = __ldg(p.tokens + i);
        if (static_cast<uint32_t>(t) >= p.V0) {
          set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
          t = 0;
        }
        v[j] = ld_stream_v4(p.E0 + static_cast<int64_t>(t) * p.e0_row_bytes + c * 16);
        dst[j] = p.E0_out + static_cast<int64_t>(e) * 16;
      }
    }
#pragma unroll
    for (int j = 0; j < kGatherUnroll; ++j)
      if (dst[j]) *reinterpret_cast<uint4*>(dst[j]) = v[j];
  }
}

// ------------------------------------------------------------------ embedding amplification
// LayerNorm over each output row (section 3.2.4 of "Scaling Embeddings Outperforms
// Scaling Experts in Language Models": normalising the N-gram embedding output before it
// joins the residual stream amplifies it early in training). One warp per row; the row
// is read three times (mean, centred second moment, write), the second and third from
// L1/L2; fp32 arithmetic; y may alias x.

struct LayerNormParams {
  const void* x;
  void* y;
  const float* gamma;  // [D] or nullptr (1)
  const float* beta;   // [D] or nullptr (0)
  float eps;
  int64_t T;
  int D;
};

// 16 bytes of a row: 4 fp32 or 8 bf16 values.
template <bool F32>
__device__ __forceinline__ void ln_load(const LayerNormParams& p, int64_t row, int c, float (&v)[F32 ? 4 : 8]) {
  if constexpr (F32) {
    const float4 a = reinterpret_cast<const float4*>(static_cast<const float*>(p.x) + row * p.D)[c];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const uint4 u = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + row * p.D)[c];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 * h] = __uint_as_float(w[h] << 16);
      v[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
    }
  }
}

// Rows of up to kLnRegVectors x 32 16-byte vectors (bf16: D <= 4096) are read from memory
// once: each lane keeps its vectors in registers (all loads in flight together), and the
// mean, the centred second moment and the output are computed from them.
constexpr int kLnRegVectors = 16;

template <bool F32>
__global__ void __launch_bounds__(256) layernorm_kernel(const __grid_constant__ LayerNormParams p) {
  constexpr int VW = F32 ? 4 : 8;  // values per 16-byte vector
  pdl_launch_dependents();
  pdl_wait();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.T) return;
  const int nv = p.D / VW;  // D * element size is a multiple of 16 for every plan
  if (nv <= 32 * kLnRegVectors) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.x) + row * p.D * (F32 ? 4 : 2));
    uint4 u[kLnRegVectors];
#pragma unroll
    for (int j = 0; j < kLnRegVectors; ++j)
      if (lane + 32 * j < nv) u[j] = src[lane + 32 * j];
    auto values = [&](int j, float (&v)[VW]) {
      const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
      if constexpr (F32) {
#pragma unroll
        for (int h = 0; h < 4; ++h) v[h] = __uint_as_float(w[h]);
      } else {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          v[2 * h] = __uint_as_float(w[h] << 16);
          v[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
        }
      }
    };
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kLnRegVectors; ++j) {
      if (lane + 32 * j >= nv) break;
      float v[VW];
      values(j, v);
#pragma unroll
      for (int k = 0; k < VW; ++k) sum += v[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum / static_cast<float>(p.D);
    float sq = 0.f;
#pragma unroll
    for (int j = 0; j < kLnRegVectors; ++j) {
      if (lane + 32 * j >= nv) break;
      float v[VW];
      values(j, v);
#pragma unroll
      for (int k = 0; k < VW; ++k) sq += (v[k] - mean) * (v[k] - mean);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rstd = rsqrtf(sq / static_cast<float>(p.D) + p.eps);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.y) + row * p.D * (F32 ? 4 : 2));
#pragma unroll
    for (int j = 0; j < kLnRegVectors; ++j) {
      const int c = lane + 32 * j;
      if (c >= nv) break;
      float v[VW];
      values(j, v);
#pragma unroll
      for (int k = 0; k < VW; ++k) {
        const int col = c * VW + k;
        v[k] = (v[k] - mean) * rstd * (p.gamma ? p.gamma[col] : 1.f) + (p.beta ? p.beta[col] : 0.f);
      }
      if constexpr (F32) {
        dst[c] = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
      } else {
        dst[c] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                            pack_bf16x2(v[6], v[7]));
      }
    }
    return;
  }
  float sum = 0.f;
  for (int c = lane; c < nv; c += 32) {
    float v[VW];
    ln_load<F32>(p, row, c, v);
#pragma unroll
    for (int k = 0; k < VW; ++k) sum += v[k];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / static_cast<float>(p.D);
  float sq = 0.f;
  for (int c = lane; c < nv; c += 32) {
    float v[VW];
    ln_load<F32>(p, row, c, v);
#pragma unroll
    for (int k = 0; k < VW; ++k) sq += (v[k] - mean) * (v[k] - mean);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / static_cast<float>(p.D) + p.eps);
  for (int c = lane; c < nv; c += 32) {
    float v[VW];
    ln_load<F32>(p, row, c, v);
#pragma unroll
    for (int k = 0; k < VW; ++k) {
      const int col = c * VW + k;
      v[k] = (v[k] - mean) * rstd * (p.gamma ? p.gamma[col] : 1.f) + (p.beta ? p.beta[col] : 0.f);
    }
    if constexpr (F32) {
      reinterpret_cast<float4*>(static_cast<float*>(p.y) + row * p.D)[c] = make_float4(v[0], v[1], v[2], v[3]);
    } else {
      reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + row * p.D)[c] =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
  }
}

// ------------------------------------------------------------------ N-gram cache ring

struct CacheParams {
  int32_t* ring;
  int64_t* len;
  int64_t* valid_from;
  int32_t capacity, max_seqs;
  int N;
  uint32_t V0;
  const int32_t* slots;       // nullptr: entry i -> slot i
  const int32_t* tokens;      // append
  const int32_t* tok_offsets; // append
  const int32_t* counts;      // rollback; commit (ids per entry)
  int32_t stride;             // commit: entry i's ids start at tokens[i * stride]
  int32_t n;
  int* status;
};

__device__ __forceinline__ int32_t entry_slot(const CacheParams& p, int32_t i) {
  const int32_t s = p.slots ? p.slots[i] : i;
  if (s < 0 || s >= p.max_seqs) {
    set_status(p.status, NGRAM_STATUS_BAD_SLOT);
    return -1;
  }
  return s;
}

__global__ void cache_reset_kernel(const __grid_constant__ CacheParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.n) return;
  const int32_t s = entry_slot(p, i);
  if (s < 0) return;
  p.len[s] = 0;
  p.valid_from[s] = 0;
}

// One warp per entry: write the ids at positions len .. len+m-1 (slot pos % C), then
// len += m and valid_from = max(valid_from, len - C). Rejected entries change nothing.
// One warp appends entry i's ids (CSR entries, or the first counts[i] of a fixed stride)
// to its slot's ring: the N-gram cache update of a commit.
__device__ __forceinline__ void append_entry(const CacheParams& p, int32_t i, int lane) {
  int32_t s = -1;
  if (lane == 0) s = entry_slot(p, i);
  s = __shfl_sync(0xffffffffu, s, 0);
  if (s < 0) return;
  // CSR entries (tok_offsets) or fixed-stride entries with counts (commit of accepted ids)
  const int32_t b = p.tok_offsets ? p.tok_offsets[i] : i * p.stride;
  const int32_t m = p.tok_offsets ? p.tok_offsets[i + 1] - b : p.counts[i];
  if (b < 0 || m < 0 || m > p.capacity || (!p.tok_offsets && m > p.stride)) {
    if (lane == 0) set_status(p.status, (b < 0 || m < 0) ? NGRAM_STATUS_BAD_OFFSETS : NGRAM_STATUS_BAD_APPEND);
    return;
  }
  bool bad = false;
  for (int k = lane; k < m; k += 32) {
    const int32_t t = p.tokens[b + k];
    bad |= (t < 0 || static_cast<uint32_t>(t) >= p.V0);
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
    return;
  }
  const int64_t L = p.len[s];
  int32_t* ring = p.ring + static_cast<int64_t>(s) * p.capacity;
  for (int k = lane; k < m; k += 32) ring[(L + k) % p.capacity] = p.tokens[b + k];
  __syncwarp();
  if (lane == 0) {
    const int64_t nl = L + m;
    p.len[s] = nl;
    const int64_t vf = nl - p.capacity;
    if (vf > p.valid_from[s]) p.valid_from[s] = vf;
  }
}

__global__ void cache_append_kernel(const __grid_constant__ CacheParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int32_t i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (i >= p.n) return;
  append_entry(p, i, lane);
}

// One thread per entry: drop the newest counts[i] ids if the ring still holds the
// newest N-1 positions that remain; otherwise flag and leave the slot unchanged.
__global__ void cache_rollback_kernel(const __grid_constant__ CacheParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.n) return;
  const int32_t s = entry_slot(p, i);
  if (s < 0) return;
  const int64_t r = p.counts[i];
  const int64_t L = p.len[s];
  const int64_t need = L - r - (p.N - 1);
  if (r < 0 || r > L || (need > 0 ? need : 0) < p.valid_from[s]) {
    set_status(p.status, NGRAM_STATUS_BAD_ROLLBACK);
    return;
  }
  p.len[s] = L - r;
}

}  // namespace ngram
