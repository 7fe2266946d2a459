// Backward of the N-gram embedding layer (Eq. 3 of "Scaling Embeddings Outperforms Scaling
// Experts in Language Models", section 2), for training from scratch (section 6).
//
// With c = (output scale) / ((N-1)K + 1) and g = dL/de [T x D]:
//   dE_0[t_i]              += c g_i                                   (scatter over tokens)
//   dG                      = c g W_stacked                 [T x D]   (tcgen05 GEMM, K = D)
//   dE_s[idx_s(i)][j]      += dG[i][s d + j]                          (scatter, fused in the
//                                                                      GEMM's epilogue)
//   dW_stacked             += c g^T G,  G[i][s d + j] = E_s[idx_s(i)][j]   (tcgen05 GEMM, K = T)
// Colliding rows (several tokens, one table row) add up: every scatter is an fp32 atomic
// add, so the summation order (not the set of terms) varies between runs.
//
// Both GEMMs run on one kernel: bf16 A (M x K) and B (N x K) tiles brought in by 2-D TMA
// straight from the tensors as they lie in memory — K-major (K contiguous: g for dG) or
// MN-major (M or N contiguous: W for dG, g and G for dW), the tensor cores reading either
// layout from its shared-memory descriptor — fp32 accumulators in TMEM, work units of
// (tile, k range) handed out round-robin to persistent CTAs or CTA pairs (split-K where
// tiles are few, the units in flight sharing a k range), and an epilogue that atomically
// adds the scaled partial tile into its destination: sub-table gradient rows (dG) or dW.
// Three forms of it: `dense_gemm_pair_kernel` (CTA pairs, 256 x BN tiles, the default),
// `dense_gemm_sm100_kernel` (one CTA per 128 x BN tile) and `dense_gemm_pair_wide_kernel`
// (CTA pairs, 256 x 512 tiles). The only copy is G itself, gathered row by row from the
// sub-tables into the workspace for dW.
#pragma once

#include "proj_sm100.cuh"

namespace ngram {

// ------------------------------------------------------------------ dE_0 scatter
// dE0[v] += c * sum_{i : t_i = v} g_i. Token streams repeat ids heavily (Zipf: the commonest
// id is ~10 % of a batch), so adding each row atomically into dE0 would serialise on the
// hot rows. Instead: a counting sort of the positions by token id (histogram, exclusive scan
// over V0, placement), then each warp sums a run of kSegRows consecutive sorted positions and
// adds one partial row per distinct id in its run — a hot id costs one add per run. The
// histogram and the placement aggregate equal ids within a warp first (one atomic per
// distinct id per warp), which keeps the hot ids' counters from serialising tens of
// thousands of atomics on one address.

constexpr int kSegRows = 16;

struct ScatterE0Params {
  const int32_t* tokens;
  const uint16_t* g;   // [T x D] bf16
  float* dE0;          // [V0 x D] fp32
  int64_t T;
  int D;
  uint32_t V0;
  float scale;
  int32_t* counts;     // [V0 + 1], zero on entry: histogram, then each bin's start within its
                       // 1024-bin block, then (advanced by the placement) its end; counts[V0]
                       // is the scan's block ticket
  int32_t* order;      // [T]: positions sorted by token id
  int32_t* sorted_tok; // [T]: their ids
  int32_t* block_sums; // [num_blocks]: totals of 1024-bin blocks, then their exclusive prefixes
  int num_blocks;
  int* status;
};

__device__ __forceinline__ uint32_t e0_token(const ScatterE0Params& p, int64_t i) {
  const int32_t t = p.tokens[i];
  if (static_cast<uint32_t>(t) >= p.V0) {
    set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
    return 0;
  }
  return static_cast<uint32_t>(t);
}

// Position i's id, or 0xFFFFFFFF past the end (never equal to an id: V0 < 2^31).
__device__ __forceinline__ uint32_t e0_token_or_none(const ScatterE0Params& p, int64_t i) {
  return i < p.T ? e0_token(p, i) : 0xFFFFFFFFu;
}

__global__ void __launch_bounds__(256) e0_hist_kernel(const __grid_constant__ ScatterE0Params p) {
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const uint32_t t = e0_token_or_none(p, i);
  const uint32_t peers = __match_any_sync(0xffffffffu, t);  // lanes holding the same id
  if (i < p.T && lane == __ffs(peers) - 1) atomicAdd(p.counts + t, __popc(peers));
}

// Exclusive scan of a block's values (one per thread, up to 1024 threads).
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t c, int32_t* warp_sums, int32_t& total) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int32_t x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    int32_t t = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_sums[lane] = t;
  }
  __syncthreads();
  total = warp_sums[31];
  const int32_t r = (w > 0 ? warp_sums[w - 1] : 0) + x - c;
  __syncthreads();  // warp_sums may be reused by the caller's next scan
  return r;
}

// Each block of 1024 bins scans itself in place and records its total; the block that
// finishes last (a ticket counter) then scans the totals into exclusive block prefixes, in
// chunks of 1024. No block waits for another.
__global__ void __launch_bounds__(1024) e0_scan_kernel(const __grid_constant__ ScatterE0Params p) {
  pdl_wait();
  __shared__ int32_t warp_sums[32];
  __shared__ int is_last;
  const int64_t b = static_cast<int64_t>(blockIdx.x) * 1024 + threadIdx.x;
  const int32_t c = b < p.V0 ? p.counts[b] : 0;
  int32_t total;
  const int32_t ex = block_exclusive_scan(c, warp_sums, total);
  if (b < p.V0) p.counts[b] = ex;
  if (threadIdx.x == 0) {
    p.block_sums[blockIdx.x] = total;
    __threadfence();  // the total is visible before the ticket is taken
    is_last = atomicAdd(p.counts + p.V0, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  int32_t carry = 0;
  for (int base = 0; base < p.num_blocks; base += 1024) {
    const int k = base + threadIdx.x;
    const int32_t v = k < p.num_blocks ? __ldcg(p.block_sums + k) : 0;
    int32_t chunk_total;
    const int32_t e = block_exclusive_scan(v, warp_sums, chunk_total);
    if (k < p.num_blocks) p.block_sums[k] = carry + e;
    carry += chunk_total;
  }
}

// Sorted slot of position i: its bin's start (block-local start + block prefix) plus the
// count of equal ids placed before it; one atomic per distinct id in the warp advances the
// bin's cursor (the block-local start in counts).
__global__ void __launch_bounds__(256) e0_place_kernel(const __grid_constant__ ScatterE0Params p) {
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const uint32_t t = e0_token_or_none(p, i);
  const uint32_t peers = __match_any_sync(0xffffffffu, t);
  const int leader = __ffs(peers) - 1;
  int32_t base = 0;
  if (i < p.T && lane == leader) base = atomicAdd(p.counts + t, __popc(peers)) + p.block_sums[t >> 10];
  base = __shfl_sync(0xffffffffu, base, leader);
  if (i < p.T) {
    const int32_t at = base + __popc(peers & ((1u << lane) - 1u));
    p.order[at] = static_cast<int32_t>(i);
    p.sorted_tok[at] = static_cast<int32_t>(t);
  }
}

// One warp per (run of kSegRows sorted positions, 256 columns): each lane loads its 8
// columns (16 bytes) of all kSegRows rows first, then sums them in order, adding one
// partial row into dE0 per distinct id in the run.
__global__ void __launch_bounds__(256) e0_reduce_kernel(const __grid_constant__ ScatterE0Params p) {
  pdl_wait();
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int chunks = (p.D + 255) / 256;
  const int64_t seg = item / chunks;
  const int c = static_cast<int>(item - seg * chunks) * 256 + lane * 8;
  const int64_t k0 = seg * kSegRows;
  if (k0 >= p.T || c >= p.D) return;
  const int n = static_cast<int>(p.T - k0 < kSegRows ? p.T - k0 : kSegRows);
  uint4 rows[kSegRows];
#pragma unroll
  for (int r = 0; r < kSegRows; ++r)
    if (r < n) rows[r] = *reinterpret_cast<const uint4*>(p.g + static_cast<int64_t>(p.order[k0 + r]) * p.D + c);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int32_t cur = p.sorted_tok[k0];
  auto flush = [&](int32_t tok) {
    float4* dst = reinterpret_cast<float4*>(p.dE0 + static_cast<int64_t>(tok) * p.D + c);
    atomicAdd(dst, make_float4(acc[0] * p.scale, acc[1] * p.scale, acc[2] * p.scale, acc[3] * p.scale));
    atomicAdd(dst + 1, make_float4(acc[4] * p.scale, acc[5] * p.scale, acc[6] * p.scale, acc[7] * p.scale));
#pragma unroll
    for (int h = 0; h < 8; ++h) acc[h] = 0.f;
  };
#pragma unroll
  for (int r = 0; r < kSegRows; ++r) {
    if (r >= n) break;
    const int32_t tok = p.sorted_tok[k0 + r];
    if (tok != cur) {
      flush(cur);
      cur = tok;
    }
    const uint32_t wds[4] = {rows[r].x, rows[r].y, rows[r].z, rows[r].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      acc[2 * h] += bf16_bits_to_float(wds[h] & 0xFFFFu);
      acc[2 * h + 1] += bf16_bits_to_float(wds[h] >> 16);
    }
  }
  flush(cur);
}

// ------------------------------------------------------------------ dense tcgen05 GEMM

enum GemmEpi : int { kEpiScatterSub = 0, kEpiAccumDense = 1 };

struct DenseMaps {
  // K-major operand: [rows x K] bf16, box {64, 128 (A) or BN (B)}; MN-major operand:
  // [K x rows] bf16 (rows contiguous), box {64, 64}: a tile is rows / 64 such boxes. All
  // with the 128-byte swizzle.
  CUtensorMap A;
  CUtensorMap B;
};

struct DenseParams {
  int M, N;            // rows of A (tokens, or D) and of B (D)
  int num_m_blocks, num_n_blocks, num_k_blocks;
  int splits;          // k ranges per tile (split-K): unit u = k range * tiles + tile, so the
                       // units running at once share their k range (A and B strips reused
                       // from L2 across the tiles)
  int kb_per_split;
  float scale;
  int epi;             // GemmEpi
  // kEpiScatterSub: row i of the tile -> dE_s[idx[i][s]][c - s d] for column c (s = c / d)
  const int32_t* idx;
  float* dE[kMaxS];
  uint32_t Vs[kMaxS];
  int S, d;
  // kEpiAccumDense: out[row][col] (row stride N)
  float* out;
  int* status;
  int a_mn, b_mn;      // 1: the operand is MN-major in memory (see DenseMaps)
};

constexpr int kGemmThreads = 256;

// Shared-memory descriptor of an MN-major bf16 tile in the canonical 128-byte-swizzle layout
// as 2-D TMA writes it from boxes of 64 (M or N) x 64 (K): within a box, K row r holds 64
// consecutive M/N elements at r * 128 bytes (16-byte chunks XOR-swizzled by r mod 8), so
// groups of 8 K rows are 1024 bytes apart (stride byte offset); consecutive boxes, i.e. the
// next 64 M/N elements, are 8192 bytes apart (leading byte offset). Advancing K by 16 rows
// adds 2048 bytes to the start address.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu)     // start address, bits [0,14)
         | (static_cast<uint64_t>(8192 >> 4) << 16)          // leading byte offset: next 64 M/N
         | (static_cast<uint64_t>(1024 >> 4) << 32)          // stride byte offset: next 8 K rows
         | (static_cast<uint64_t>(1) << 46)                  // descriptor version for sm_100
         | (static_cast<uint64_t>(2) << 61);                 // layout: 128-byte swizzle
}  // warp 0: TMA producer, warp 1: MMA + TMEM, warps 4-7: epilogue

template <int BN, int STAGES>
struct DenseSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  // epilogue staging: 32 rows x 32 fp32 columns per epilogue warp (4 warps)
  static constexpr int kEpiOffset = (kBarOffset + kNumBars * 8 + 16 + 127) / 128 * 128;
  static constexpr int kBytes = kEpiOffset + 4 * 32 * 32 * 4;
  static constexpr int kLaunchBytes = kBytes + 1024;
  static constexpr int kTmemCols = 2 * BN;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    dense_gemm_sm100_kernel(const __grid_constant__ DenseMaps maps, const __grid_constant__ DenseParams p) {
  using L = DenseSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOffset;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOffset + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto a_tile = [&](int s) { return sbase + s * L::kStageBytes; };
  auto b_tile = [&](int s) { return sbase + s * L::kStageBytes + L::kABytes; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1u);   // the producer's byte count
      mbar_init(empty_bar(s), 1u);  // one tcgen05.commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1u);
      mbar_init(tempty_bar(a), 128u);
    }
    mbar_init(drain_bar, 1u);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.A);
    tma_prefetch_desc(&maps.B);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int num_units = num_tiles * p.splits;
  auto unit_k = [&](int u, int& kb0, int& kb1) {
    const int ks = u / num_tiles;
    kb0 = ks * p.kb_per_split;
    kb1 = kb0 + p.kb_per_split < p.num_k_blocks ? kb0 + p.kb_per_split : p.num_k_blocks;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (A and B)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int tile = u % num_tiles;
        const int m_blk = tile / p.num_n_blocks, n_blk = tile % p.num_n_blocks;
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), L::kStageBytes);
          if (p.a_mn) {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d(a_tile(stage) + j * 8192, &maps.A, m_blk * kBM + j * 64, kb * kBK, full_bar(stage), pol);
          } else {
            tma_load_2d(a_tile(stage), &maps.A, kb * kBK, m_blk * kBM, full_bar(stage), pol);
          }
          if (p.b_mn) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(b_tile(stage) + j * 8192, &maps.B, n_blk * BN + j * 64, kb * kBK, full_bar(stage), pol);
          } else {
            tma_load_2d(b_tile(stage), &maps.B, kb * kBK, n_blk * BN, full_bar(stage), pol);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // operand majors: bit 15 (A), bit 16 (B) of the instruction descriptor, 1 = MN-major
      const uint32_t idesc = umma_idesc_bf16(kBM, BN) | (p.a_mn ? 1u << 15 : 0u) | (p.b_mn ? 1u << 16 : 0u);
      const uint32_t a_step = p.a_mn ? 2048u >> 4 : 32u >> 4;  // K += 16 in the descriptor's address field
      const uint32_t b_step = p.b_mn ? 2048u >> 4 : 32u >> 4;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = p.a_mn ? sw128_mnmajor_desc(a_tile(stage)) : sw128_kmajor_desc(a_tile(stage));
          const uint64_t bdesc = p.b_mn ? sw128_mnmajor_desc(b_tile(stage)) : sw128_kmajor_desc(b_tile(stage));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, (kb > kb0 || k != 0) ? 1u : 0u);
          umma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(tfull_bar(acc));
      }
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: atomic adds
    // Per 32-column chunk: each lane reads its row's fp32 accumulators from TMEM (row per
    // lane) into the warp's staging area; then eight lanes per row read them back, 16 bytes
    // each, and add the scaled values into the row's destination, so every reduction
    // instruction covers 4 rows x 128 contiguous bytes (whole 32-byte sectors) instead of
    // 32 rows x 16 bytes. Staging layout: row r at r * 128 bytes, 16-byte unit w at
    // ((w ^ (r & 7)) << 4): conflict-free both ways.
    const int q = warp & 3;
    const uint32_t stg = sbase + L::kEpiOffset + static_cast<uint32_t>(q) * 4096u;
    const uint32_t row_w = stg + static_cast<uint32_t>(lane) * 128u;
    const int wv = lane & 7;   // read-back: 16-byte unit of the row
    const int rq = lane >> 3;  // read-back: rows i * 4 + rq
    int local = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++local) {
      const int tile = u % num_tiles;
      const int m_blk = tile / p.num_n_blocks, n_blk = tile % p.num_n_blocks;
      const int acc = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      const int64_t row0 = static_cast<int64_t>(m_blk) * kBM + q * 32;  // this warp's first row
      bool got = false;
      if (lane == 0) got = mbar_wait(tfull_bar(acc), use & 1u, abort_flag, p.status);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      int s_cur = -1;
      int32_t my_target = 0;  // scatter: this lane's row's table row in sub-table s_cur
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c * 32, v);
        tmem_wait_ld();
        if (c + 1 == BN / 32) {
          tc_fence_before();
          mbar_arrive_relaxed(tempty_bar(acc));
        }
        const int col0 = n_blk * BN + c * 32;
        const int s = p.epi == kEpiScatterSub ? col0 / p.d : 0;  // 32 columns never straddle two sub-tables
        if (p.epi == kEpiScatterSub && s != s_cur) {
          s_cur = s;
          my_target = 0;
          if (row0 + lane < p.M) {
            my_target = p.idx[(row0 + lane) * p.S + s];
            if (static_cast<uint32_t>(my_target) >= p.Vs[s]) {
              set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
              my_target = 0;
            }
          }
        }
#pragma unroll
        for (int w = 0; w < 8; ++w)
          st_shared_v4(row_w + (static_cast<uint32_t>(w ^ (lane & 7)) << 4),
                       make_uint4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = i * 4 + rq;  // row of the warp's 32
          const uint4 x = ld_shared_v4(stg + static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(wv ^ (r & 7)) << 4));
          const int32_t target = __shfl_sync(0xffffffffu, my_target, r);
          const int64_t grow = row0 + r;
          if (grow < p.M) {
            float* dst = p.epi == kEpiScatterSub
                             ? p.dE[s] + static_cast<int64_t>(target) * p.d + (col0 - s * p.d) + wv * 4
                             : p.out + grow * p.N + col0 + wv * 4;
            atomicAdd(reinterpret_cast<float4*>(dst),
                      make_float4(__uint_as_float(x.x) * p.scale, __uint_as_float(x.y) * p.scale,
                                  __uint_as_float(x.z) * p.scale, __uint_as_float(x.w) * p.scale));
          }
        }
        __syncwarp();  // the staging area is rewritten by the next chunk
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}


// CTA-pair form of the dense GEMM (tcgen05.mma.cta_group::2, M = 256): the pair computes a
// 256 x BN tile; each CTA loads its 128 rows of A and BN/2 rows of B per k-block (2-D TMA in
// the .cta_group::2 form, byte counts completing on CTA 0's stage barrier), one thread of CTA 0
// issues the MMAs and commits stage releases and "accumulator ready" to both CTAs, and each
// CTA's epilogue drains its 128 accumulator rows as the one-CTA kernel does (CTA 1's warps
// free the accumulator by remote arrivals on CTA 0's barrier). Per SM and k-block it loads
// 16 KB of A + BN/2 x 128 B of B for the same FLOPs the one-CTA kernel needs 16 KB + BN x
// 128 B for. A stage holds KSUB consecutive k-blocks: every stage costs the MMA thread a
// barrier wait and a commit, which hold the tensor pipe up for a while, so fewer, larger
// stages leave more of its time to the MMAs.
template <int BN, int STAGES, int KSUB>
struct DensePairSmem {
  static constexpr int kABytes = kBM * kBK * 2;           // this CTA's 128 rows of A, one k-block
  static constexpr int kBBytes = (BN / 2) * kBK * 2;      // this CTA's BN/2 rows of B, one k-block
  static constexpr int kSubBytes = kABytes + kBBytes;     // one k-block of both
  static constexpr int kStageBytes = KSUB * kSubBytes;    // a stage: KSUB consecutive k-blocks
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kEpiOffset = (kBarOffset + kNumBars * 8 + 16 + 127) / 128 * 128;
  static constexpr int kBytes = kEpiOffset + 4 * 32 * 32 * 4;
  static constexpr int kLaunchBytes = kBytes + 1024;
  static constexpr int kTmemCols = 2 * BN;
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of 128-byte swizzling");
};

template <int BN, int STAGES, int KSUB>
__global__ void __launch_bounds__(kGemmThreads, 1)
    dense_gemm_pair_kernel(const __grid_constant__ DenseMaps maps, const __grid_constant__ DenseParams p) {
  using L = DensePairSmem<BN, STAGES, KSUB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOffset;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOffset + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto a_tile = [&](int s, int j) { return sbase + s * L::kStageBytes + j * L::kSubBytes; };
  auto b_tile = [&](int s, int j) { return sbase + s * L::kStageBytes + j * L::kSubBytes + L::kABytes; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs and owns the stage barriers
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1u);   // CTA 0: its producer's byte count for both CTAs (CTA 1's: unused)
      mbar_init(empty_bar(s), 1u);  // one tcgen05.commit from CTA 0's MMA thread
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1u);
      mbar_init(tempty_bar(a), 128u + 4u);  // CTA 0's epilogue threads + one remote arrive per CTA 1 warp
    }
    mbar_init(drain_bar, 1u);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.A);
    tma_prefetch_desc(&maps.B);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;  // m blocks of 256 rows
  const int num_units = num_tiles * p.splits;
  auto unit_k = [&](int u, int& kb0, int& kb1) {
    const int ks = u / num_tiles;
    kb0 = ks * p.kb_per_split;
    kb1 = kb0 + p.kb_per_split < p.num_k_blocks ? kb0 + p.kb_per_split : p.num_k_blocks;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (own rows)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < num_units && ok; u += num_pairs) {
        const int tile = u % num_tiles;
        const int m_blk = tile / p.num_n_blocks, n_blk = tile % p.num_n_blocks;
        const int row_a = m_blk * (2 * kBM) + static_cast<int>(rank) * kBM;
        const int row_b = n_blk * BN + static_cast<int>(rank) * (BN / 2);
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; kb += KSUB) {
          const int nsub = kb1 - kb < KSUB ? kb1 - kb : KSUB;  // k-blocks in this stage
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          const uint32_t full0 = map_to_cta(full_bar(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2u * nsub * L::kSubBytes);
          for (int i = 0; i < nsub; ++i) {
            const int kx = (kb + i) * kBK;
            if (p.a_mn) {
#pragma unroll
              for (int j = 0; j < kBM / 64; ++j)
                tma_load_2d_pair(a_tile(stage, i) + j * 8192, &maps.A, row_a + j * 64, kx, full0, pol);
            } else {
              tma_load_2d_pair(a_tile(stage, i), &maps.A, kx, row_a, full0, pol);
            }
            if (p.b_mn) {
#pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                tma_load_2d_pair(b_tile(stage, i) + j * 8192, &maps.B, row_b + j * 64, kx, full0, pol);
            } else {
              tma_load_2d_pair(b_tile(stage, i), &maps.B, kx, row_b, full0, pol);
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {  // aborting: the loads in flight land (bounded) before exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000ull * 1000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = umma_idesc_bf16(2 * kBM, BN) | (p.a_mn ? 1u << 15 : 0u) | (p.b_mn ? 1u << 16 : 0u);
      const uint32_t a_step = p.a_mn ? 2048u >> 4 : 32u >> 4;  // K += 16 in the descriptor's address field
      const uint32_t b_step = p.b_mn ? 2048u >> 4 : 32u >> 4;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int u = pair; u < num_units && ok; u += num_pairs, ++local) {
        const int acc = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait_cluster(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; kb += KSUB) {
          const int nsub = kb1 - kb < KSUB ? kb1 - kb : KSUB;
          if (!mbar_wait_cluster(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          for (int i = 0; i < nsub; ++i) {
            const uint64_t adesc = p.a_mn ? sw128_mnmajor_desc(a_tile(stage, i)) : sw128_kmajor_desc(a_tile(stage, i));
            const uint64_t bdesc = p.b_mn ? sw128_mnmajor_desc(b_tile(stage, i)) : sw128_kmajor_desc(b_tile(stage, i));
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_bf16_pair(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, (kb + i > kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit_pair_both(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) {
          umma_commit_pair_both(tfull_bar(acc));
        }
      }
      umma_commit_pair(map_to_cta(drain_bar, 0));
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: atomic adds
    // As in the one-CTA kernel (staged 32 x 32 chunks, eight lanes per row for the fp32
    // reductions), for this CTA's 128 rows of the pair's tile.
    const int q = warp & 3;
    const uint32_t stg = sbase + L::kEpiOffset + static_cast<uint32_t>(q) * 4096u;
    const uint32_t row_w = stg + static_cast<uint32_t>(lane) * 128u;
    const int wv = lane & 7;
    const int rq = lane >> 3;
    const uint32_t tempty_remote0 = map_to_cta(tempty_bar(0), 0);
    const uint32_t tempty_remote1 = map_to_cta(tempty_bar(1), 0);
    int local = 0;
    for (int u = pair; u < num_units; u += num_pairs, ++local) {
      const int tile = u % num_tiles;
      const int m_blk = tile / p.num_n_blocks, n_blk = tile % p.num_n_blocks;
      const int acc = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      const int64_t row0 = static_cast<int64_t>(m_blk) * (2 * kBM) + rank * kBM + q * 32;  // this warp's first row
      bool got = false;
      if (lane == 0) got = mbar_wait_cluster(tfull_bar(acc), use & 1u, abort_flag, p.status);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      int s_cur = -1;
      int32_t my_target = 0;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c * 32, v);
        tmem_wait_ld();
        if (c + 1 == BN / 32) {
          tc_fence_before();
          if (rank == 0) {
            mbar_arrive_relaxed(tempty_bar(acc));
          } else {
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(acc ? tempty_remote1 : tempty_remote0);
          }
        }
        const int col0 = n_blk * BN + c * 32;
        const int s = p.epi == kEpiScatterSub ? col0 / p.d : 0;  // 32 columns never straddle two sub-tables
        if (p.epi == kEpiScatterSub && s != s_cur) {
          s_cur = s;
          my_target = 0;
          if (row0 + lane < p.M) {
            my_target = p.idx[(row0 + lane) * p.S + s];
            if (static_cast<uint32_t>(my_target) >= p.Vs[s]) {
              set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
              my_target = 0;
            }
          }
        }
#pragma unroll
        for (int w = 0; w < 8; ++w)
          st_shared_v4(row_w + (static_cast<uint32_t>(w ^ (lane & 7)) << 4),
                       make_uint4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = i * 4 + rq;
          const uint4 x = ld_shared_v4(stg + static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(wv ^ (r & 7)) << 4));
          const int32_t target = __shfl_sync(0xffffffffu, my_target, r);
          const int64_t grow = row0 + r;
          if (grow < p.M) {
            float* dst = p.epi == kEpiScatterSub
                             ? p.dE[s] + static_cast<int64_t>(target) * p.d + (col0 - s * p.d) + wv * 4
                             : p.out + grow * p.N + col0 + wv * 4;
            atomicAdd(reinterpret_cast<float4*>(dst),
                      make_float4(__uint_as_float(x.x) * p.scale, __uint_as_float(x.y) * p.scale,
                                  __uint_as_float(x.z) * p.scale, __uint_as_float(x.w) * p.scale));
          }
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrive or pair MMA is outstanding past this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}


// Wide CTA-pair form: 256 x 512 tiles, the pair's accumulator split in two halves of
// 256 x 256 (TMEM columns 0-255 and 256-511 of both CTAs), one N = 256 pair MMA per half and
// k-step. Per SM and k-block it loads 16 KB of A and 32 KB of B (its 128 rows of each half)
// for twice the FLOPs of the 256 x 256 pair tile, so each stage covers twice the load latency.
// With one accumulator the next tile's MMAs need the drain out of the way: eight epilogue
// warps drain half 0 first and free it, then half 1; the MMA thread starts a tile with the
// half-0 products of its first STAGES k-blocks while half 1 drains, then catches up on half 1.
template <int STAGES>
struct DenseWideSmem {
  static constexpr int kABytes = kBM * kBK * 2;       // this CTA's 128 rows of A
  static constexpr int kBSubBytes = kBM * kBK * 2;    // this CTA's 128 rows of one half's B
  static constexpr int kStageBytes = kABytes + 2 * kBSubBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kEpiOffset = (kBarOffset + kNumBars * 8 + 16 + 127) / 128 * 128;
  static constexpr int kBytes = kEpiOffset + 8 * 32 * 32 * 4;  // eight epilogue warps' staging
  static constexpr int kLaunchBytes = kBytes + 1024;
  static constexpr int kTmemCols = 512;
};
constexpr int kWideGemmThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 4-11 epilogue

template <int STAGES>
__global__ void __launch_bounds__(kWideGemmThreads, 1)
    dense_gemm_pair_wide_kernel(const __grid_constant__ DenseMaps maps, const __grid_constant__ DenseParams p) {
  using L = DenseWideSmem<STAGES>;
  constexpr int BN = 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOffset;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int h) { return bar0 + 8u * (2 * STAGES + h); };
  auto tempty_bar = [&](int h) { return bar0 + 8u * (2 * STAGES + 2 + h); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOffset + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto a_tile = [&](int s) { return sbase + s * L::kStageBytes; };
  auto b_tile = [&](int s, int h) { return sbase + s * L::kStageBytes + L::kABytes + h * L::kBSubBytes; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1u);
      mbar_init(empty_bar(s), 1u);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(tfull_bar(h), 1u);
      mbar_init(tempty_bar(h), 256u + 8u);  // CTA 0's 8 epilogue warps + one remote arrive per CTA 1 warp
    }
    mbar_init(drain_bar, 1u);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.A);
    tma_prefetch_desc(&maps.B);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;  // 256-row x 512-column tiles
  const int num_units = num_tiles * p.splits;
  auto unit_k = [&](int u, int& kb0, int& kb1) {
    const int ks = u / num_tiles;
    kb0 = ks * p.kb_per_split;
    kb1 = kb0 + p.kb_per_split < p.num_k_blocks ? kb0 + p.kb_per_split : p.num_k_blocks;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (own rows)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < num_units && ok; u += num_pairs) {
        const int tile = u % num_tiles;
        const int m_blk = tile / p.num_n_blocks, n_blk = tile % p.num_n_blocks;
        const int row_a = m_blk * (2 * kBM) + static_cast<int>(rank) * kBM;
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          const uint32_t full0 = map_to_cta(full_bar(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2u * L::kStageBytes);
          if (p.a_mn) {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d_pair(a_tile(stage) + j * 8192, &maps.A, row_a + j * 64, kb * kBK, full0, pol);
          } else {
            tma_load_2d_pair(a_tile(stage), &maps.A, kb * kBK, row_a, full0, pol);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row_b = n_blk * BN + h * 256 + static_cast<int>(rank) * kBM;
            if (p.b_mn) {
#pragma unroll
              for (int j = 0; j < kBM / 64; ++j)
                tma_load_2d_pair(b_tile(stage, h) + j * 8192, &maps.B, row_b + j * 64, kb * kBK, full0, pol);
            } else {
              tma_load_2d_pair(b_tile(stage, h), &maps.B, kb * kBK, row_b, full0, pol);
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {  // aborting: the loads in flight land (bounded) before exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000ull * 1000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = umma_idesc_bf16(2 * kBM, 256) | (p.a_mn ? 1u << 15 : 0u) | (p.b_mn ? 1u << 16 : 0u);
      const uint32_t a_step = p.a_mn ? 2048u >> 4 : 32u >> 4;
      const uint32_t b_step = p.b_mn ? 2048u >> 4 : 32u >> 4;
      auto mma_half = [&](int s, int h, bool first_kb) {
        const uint64_t adesc = p.a_mn ? sw128_mnmajor_desc(a_tile(s)) : sw128_kmajor_desc(a_tile(s));
        const uint64_t bdesc = p.b_mn ? sw128_mnmajor_desc(b_tile(s, h)) : sw128_kmajor_desc(b_tile(s, h));
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(h * 256);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16_pair(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, (!first_kb || k != 0) ? 1u : 0u);
      };
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int u = pair; u < num_units && ok; u += num_pairs, ++local) {
        const uint32_t use = static_cast<uint32_t>(local);
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        const int n = kb1 - kb0;
        const int head = n < STAGES ? n : STAGES;
        // head: half 0 of the first `head` k-blocks (their stages stay held for half 1)
        if (!mbar_wait_cluster(tempty_bar(0), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < head; ++i) {
          if (!mbar_wait_cluster(full_bar(s), ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          mma_half(s, 0, i == 0);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (head == n) umma_commit_pair_both(tfull_bar(0));
        if (!mbar_wait_cluster(tempty_bar(1), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int i = 0; i < head; ++i) {
          mma_half(stage, 1, i == 0);
          umma_commit_pair_both(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        // the rest: both halves per k-block
        for (int i = head; i < n; ++i) {
          if (!mbar_wait_cluster(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          mma_half(stage, 0, false);
          if (i + 1 == n) umma_commit_pair_both(tfull_bar(0));
          mma_half(stage, 1, false);
          umma_commit_pair_both(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit_pair_both(tfull_bar(1));
      }
      umma_commit_pair(map_to_cta(drain_bar, 0));
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: atomic adds
    // Warps 4-7 take columns 0-127 of each half, warps 8-11 columns 128-255; otherwise as in
    // the one-CTA kernel (staged 32 x 32 chunks, eight lanes per row for the reductions).
    const int q = warp & 3;
    const int grp = (warp - 4) >> 2;
    const uint32_t stg = sbase + L::kEpiOffset + static_cast<uint32_t>(warp - 4) * 4096u;
    const uint32_t row_w = stg + static_cast<uint32_t>(lane) * 128u;
    const int wv = lane & 7;
    const int rq = lane >> 3;
    int local = 0;
    bool ok = true;
    for (int u = pair; u < num_units && ok; u += num_pairs, ++local) {
      const int tile = u % num_tiles;
      const int m_blk = tile / p.num_n_blocks, n_blk = tile % p.num_n_blocks;
      const uint32_t use = static_cast<uint32_t>(local);
      const int64_t row0 = static_cast<int64_t>(m_blk) * (2 * kBM) + rank * kBM + q * 32;
      for (int h = 0; h < 2 && ok; ++h) {
        bool got = false;
        if (lane == 0) got = mbar_wait_cluster(tfull_bar(h), use & 1u, abort_flag, p.status);
        if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(h * 256 + grp * 128);
        int s_cur = -1;
        int32_t my_target = 0;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c * 32, v);
          tmem_wait_ld();
          if (c == 3) {
            tc_fence_before();
            if (rank == 0) {
              mbar_arrive_relaxed(tempty_bar(h));
            } else {
              __syncwarp();
              if (lane == 0) mbar_arrive_remote_relaxed(map_to_cta(tempty_bar(h), 0));
            }
          }
          const int col0 = n_blk * BN + h * 256 + grp * 128 + c * 32;
          const int s = p.epi == kEpiScatterSub ? col0 / p.d : 0;
          if (p.epi == kEpiScatterSub && s != s_cur) {
            s_cur = s;
            my_target = 0;
            if (row0 + lane < p.M) {
              my_target = p.idx[(row0 + lane) * p.S + s];
              if (static_cast<uint32_t>(my_target) >= p.Vs[s]) {
                set_status(p.status, NGRAM_STATUS_BAD_TOKEN);
                my_target = 0;
              }
            }
          }
#pragma unroll
          for (int w = 0; w < 8; ++w)
            st_shared_v4(row_w + (static_cast<uint32_t>(w ^ (lane & 7)) << 4),
                         make_uint4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = i * 4 + rq;
            const uint4 x = ld_shared_v4(stg + static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(wv ^ (r & 7)) << 4));
            const int32_t target = __shfl_sync(0xffffffffu, my_target, r);
            const int64_t grow = row0 + r;
            if (grow < p.M) {
              float* dst = p.epi == kEpiScatterSub
                               ? p.dE[s] + static_cast<int64_t>(target) * p.d + (col0 - s * p.d) + wv * 4
                               : p.out + grow * p.N + col0 + wv * 4;
              atomicAdd(reinterpret_cast<float4*>(dst),
                        make_float4(__uint_as_float(x.x) * p.scale, __uint_as_float(x.y) * p.scale,
                                    __uint_as_float(x.z) * p.scale, __uint_as_float(x.w) * p.scale));
            }
          }
          __syncwarp();
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

}  // namespace ngram
