// Fused sub-row gather + projection + epilogue on the sm_100a tensor cores.
//
// Computes, for a tile of 128 tokens x BN outputs (Eq. 3 of "Scaling Embeddings
// Outperforms Scaling Experts in Language Models", section 2):
//   out[i][o] = ( E_0[t_i][o] + sum_s sum_c W_stacked[o][s*d + c] * E_s[idx[i][s]][c] ) / (S + 1)
// The contraction G * W_stacked^T (G[i] = concat_s E_s[idx[i][s]]) runs on tcgen05.mma
// (kind::f16, bf16 in, fp32 accumulate in TMEM). A k-block of 64 columns always lies
// inside one sub-table (d % 64 == 0), so each A tile row is one 128-byte slice of one
// gathered sub-table row: A tiles are gathered straight from HBM into shared memory in
// the 128-byte-swizzled K-major layout, and G never exists in global memory.
//
// Persistent kernel, one CTA per SM, warp-specialised (12 warps):
//   warps 0-3   A producers. Mode kGather4: warp 0 issues TMA tile::gather4 loads (each
//               lane 4 rows of the 128-row tile). Mode kCpAsync: 128 threads each copy
//               one row with 16-byte cp.async into the swizzled slot, then make the
//               writes visible to the tensor core (wait, proxy fence, arrive).
//   warp 4      W producer: one lane issues 2-D TMA loads of W_stacked tiles.
//   warp 5      TMEM allocator; one lane issues the MMAs and commits.
//   warps 8-11  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4) ..+31), + E_0 row slice, * 1/(S+1), bf16 RNE, store.
// Shared memory holds STAGES (A, B) stage pairs; TMEM holds two BN-column fp32
// accumulators so the epilogue of one tile overlaps the main loop of the next.
// Every wait is bounded (see mbar_wait); on a timeout all roles stop, drain what they
// have in flight, free TMEM and return with NGRAM_STATUS_TIMEOUT set.
#pragma once

#include "common.cuh"

namespace ngram {

constexpr int kBM = 128;  // tokens per tile (UMMA M, TMEM lanes)
constexpr int kBK = 64;   // bf16 columns per k-block = one 128-byte swizzle row
constexpr int kProjThreads = 384;
constexpr int kWarpB = 4;
constexpr int kWarpMma = 5;
constexpr int kWarpEpi0 = 8;

enum AMode : int { kGather4 = 0, kCpAsync = 1 };

struct ProjParams {
  const int32_t* tokens;  // [T]
  const int32_t* idx;     // [T * S]
  const uint16_t* E0;     // [V0 * D] bf16 bits
  const uint16_t* E[kMaxS];
  uint32_t Vs[kMaxS];
  uint16_t* out;          // [T * D] bf16 bits
  int64_t T;
  uint32_t V0;
  int D, S, d;
  int num_m_blocks, num_n_blocks, num_k_blocks;
  float scale;
  int* status;
};

struct ProjMaps {
  CUtensorMap W;            // W_stacked, box {64, BN}, 128-byte swizzle
  CUtensorMap E[kMaxS];     // sub-table s, box {64, 1}, 128-byte swizzle (gather4)
};

template <int BN, int STAGES>
struct ProjSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kBytes = kBarOffset + kNumBars * 8 + 16;
  static constexpr int kLaunchBytes = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kTmemCols = 2 * BN;
};

__device__ __forceinline__ uint32_t clamp_row(int32_t r, uint32_t V, int* status) {
  if (static_cast<uint32_t>(r) >= V) {
    set_status(status, NGRAM_STATUS_BAD_TOKEN);
    return 0;
  }
  return static_cast<uint32_t>(r);
}

template <int BN, int STAGES, int AMODE>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_sm100_kernel(const __grid_constant__ ProjMaps maps, const __grid_constant__ ProjParams p) {
  using L = ProjSmem<BN, STAGES>;
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
    const uint32_t a_arrivals = AMODE == kGather4 ? 1u : 128u;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), a_arrivals + 1u);  // A producer(s) + the W producer
      mbar_init(empty_bar(s), 1u);              // one tcgen05.commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1u);
      mbar_init(tempty_bar(a), 128u);  // every epilogue thread
    }
    mbar_init(drain_bar, 1u);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpB && lane == 0) {
    tma_prefetch_desc(&maps.W);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int KB = p.num_k_blocks;
  const int kb_per_sub = p.d / kBK;

  if ((AMODE == kGather4 && warp == 0) || (AMODE == kCpAsync && warp < 4)) {
    // ------------------------------------------------------------ A producer
    const uint64_t pol = l2_policy_evict_normal();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int prev_stage = -1;  // kCpAsync: stage whose arrival is still held back
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m_blk = tile / p.num_n_blocks;
      if constexpr (AMODE == kGather4) {
        const int64_t row0 = static_cast<int64_t>(m_blk) * kBM + lane * 4;
        int32_t r[4];
        for (int kb = 0; kb < KB; ++kb) {
          const int s = kb / kb_per_sub;
          const int c0 = (kb - s * kb_per_sub) * kBK;
          if (kb == s * kb_per_sub) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int64_t gr = row0 + j;
              r[j] = gr < p.T ? static_cast<int32_t>(clamp_row(p.idx[gr * p.S + s], p.Vs[s], p.status)) : 0;
            }
          }
          // lane 0 waits for the slot and posts the byte count; the warp follows it.
          bool got = false;
          if (lane == 0) {
            got = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status);
            if (got) mbar_arrive_expect_tx(full_bar(stage), L::kABytes);
          }
          if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
          tma_gather4(a_tile(stage) + lane * 512, &maps.E[s], c0, r[0], r[1], r[2], r[3],
                      full_bar(stage), pol);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      } else {
        const int row = threadIdx.x;  // 0..127
        const int64_t gr = static_cast<int64_t>(m_blk) * kBM + row;
        const bool valid = gr < p.T;
        const uint16_t* src = nullptr;
        for (int kb = 0; kb < KB; ++kb) {
          const int s = kb / kb_per_sub;
          const int c0 = (kb - s * kb_per_sub) * kBK;
          if (kb == s * kb_per_sub) {
            const uint32_t ix = valid ? clamp_row(p.idx[gr * p.S + s], p.Vs[s], p.status) : 0u;
            src = p.E[s] + static_cast<int64_t>(ix) * p.d;
          }
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          const uint32_t dst = a_tile(stage) + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) cp_async_16(dst + ((c ^ (row & 7)) << 4), src + c0 + c * 8);
          cp_async_commit();
          if (prev_stage >= 0) {
            cp_async_wait<1>();        // the previous stage's copies have landed
            fence_proxy_async_smem();  // make them visible to the tensor core
            mbar_arrive(full_bar(prev_stage));
          }
          prev_stage = stage;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
    if constexpr (AMODE == kCpAsync) {
      cp_async_wait<0>();
      if (ok && prev_stage >= 0) {
        fence_proxy_async_smem();
        mbar_arrive(full_bar(prev_stage));
      }
    } else if (!ok) {
      // Aborting: give the gathers this warp may still have in flight time to land
      // (bounded) before the CTA exits.
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 1000ull * 1000ull) __nanosleep(1000);
    }
  } else if (warp == kWarpB) {
    // ------------------------------------------------------------ W producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int n_blk = tile % p.num_n_blocks;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), L::kBBytes);
          tma_load_2d(b_tile(stage), &maps.W, kb * kBK, n_blk * BN, full_bar(stage), pol);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          if constexpr (AMODE == kCpAsync) fence_proxy_async_smem();
          const uint64_t adesc = sw128_kmajor_desc(a_tile(stage));
          const uint64_t bdesc = sw128_kmajor_desc(b_tile(stage));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // K = 16 per instruction: +32 B = +2 in the address field
            umma_bf16(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(tfull_bar(acc));
      }
      // Everything issued must complete before TMEM is released.
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp >= kWarpEpi0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int row_in_tile = q * 32 + lane;  // == TMEM lane
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int m_blk = tile / p.num_n_blocks;
      const int n_blk = tile % p.num_n_blocks;
      const int acc = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      const int64_t gr = static_cast<int64_t>(m_blk) * kBM + row_in_tile;
      const bool valid = gr < p.T;
      uint32_t t = 0;
      if (valid) {
        const int32_t tok = p.tokens[gr];
        t = (tok >= 0 && static_cast<uint32_t>(tok) < p.V0) ? static_cast<uint32_t>(tok) : 0u;
      }
      const uint4* e0 = reinterpret_cast<const uint4*>(p.E0 + static_cast<int64_t>(t) * p.D + n_blk * BN);
      uint4* dst = reinterpret_cast<uint4*>(p.out + gr * p.D + n_blk * BN);
      // E_0 slice of chunk 0 before waiting on the accumulator.
      uint4 ecur[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) ecur[v] = valid ? __ldg(e0 + v) : make_uint4(0, 0, 0, 0);

      bool got = false;
      if (lane == 0) got = mbar_wait(tfull_bar(acc), use & 1u, abort_flag, p.status);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;  // warp-uniform: tcgen05.ld is .aligned
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c * 32, v);
        uint4 enext[4];
        const bool has_next = c + 1 < BN / 32;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          enext[w] = (valid && has_next) ? __ldg(e0 + (c + 1) * 4 + w) : make_uint4(0, 0, 0, 0);
        tmem_wait_ld();
        if (c + 1 == BN / 32) {
          tc_fence_before();
          mbar_arrive(tempty_bar(acc));  // accumulator fully read: MMA may reuse it
        }
        if (valid) {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t ew[4] = {ecur[w].x, ecur[w].y, ecur[w].z, ecur[w].w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int col = w * 8 + h * 2;
              const float x0 = (__uint_as_float(v[col]) + bf16_bits_to_float(ew[h] & 0xFFFFu)) * p.scale;
              const float x1 = (__uint_as_float(v[col + 1]) + bf16_bits_to_float(ew[h] >> 16)) * p.scale;
              o[h] = pack_bf16x2(x0, x1);
            }
            dst[c * 4 + w] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) ecur[w] = enext[w];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace ngram
