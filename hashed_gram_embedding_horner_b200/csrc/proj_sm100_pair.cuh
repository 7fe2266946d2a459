// Two-CTA (cta_group::2) form of the fused gather + projection + epilogue kernel.
//
// Same arithmetic as proj_sm100_kernel (Eq. 3 of "Scaling Embeddings Outperforms Scaling
// Experts in Language Models", section 2), on 256 x BN tiles computed by a pair of CTAs
// (a cluster of two on neighbouring SMs): CTA r of the pair gathers rows r*128 .. +127 of
// the tile's A rows and loads rows r*BN/2 .. +BN/2-1 of the tile's W block; one thread of
// CTA 0 issues tcgen05.mma.cta_group::2 (M = 256, N = BN), which reads A and B from both
// CTAs' shared memory and writes each CTA's 128 accumulator rows into its own TMEM. Per SM
// and k-block this moves 16 KB of A + BN/2 * 128 B of W instead of 16 KB + BN * 128 B,
// which is what limits the one-CTA kernel (on-chip bytes in flight, not DRAM).
//
// Cross-CTA signalling, all plain (no multicast):
//   - W halves (and, with tma_rows = 128, the default, the A rows: tile::gather4, 32
//     issuing lanes per CTA) are TMA loads in their .cta_group::2 form: the data lands in
//     the issuing CTA's shared memory and the byte count completes on CTA 0's stage barrier;
//   - with tma_rows = 0 (256- and 128-column tiles only) the A rows arrive by 16-byte
//     cp.async, which can only signal the issuing CTA's own barrier: CTA 0's cp.async
//     threads arrive on CTA 0's stage barrier; CTA 1's arrive on CTA 1's, and a relay lane
//     of CTA 1 (one lane per stage, so the slow cluster-scope release of one stage overlaps
//     the others) waits for it, fences generic->async proxy and arrives remotely on CTA 0's
//     stage barrier;
//   - with dense_a (a call whose sub-rows were gathered into G beforehand, small enough for
//     G to stay in L2), each CTA's W producer thread also brings in its 128 A rows as one
//     2-D TMA box of G per stage (.cta_group::2 form, byte count on CTA 0's barrier), and
//     CTA 0's W producer posts the pair's byte count; the A producer warps stay idle;
//   - CTA 0's MMA thread commits stage release and "accumulator ready" to the barriers of
//     both CTAs (two tcgen05.commit, one per CTA address);
//   - CTA 1's epilogue warps arrive remotely on CTA 0's "accumulator free" barrier.
// Waits on barriers that receive remote arrivals use cluster-scope acquire. Every wait is
// bounded; both CTAs meet at cluster barriers after set-up and before teardown.
#pragma once

#include "proj_sm100.cuh"

namespace ngram {

constexpr int kWarpRelay = 10;

// Stages of (16 KB of A + BN/2 x 128 B of W) per CTA, one barrier pair per stage
// (measured ~2 % faster than separate A and W rings of the same bytes, which double the
// barrier traffic of the cluster-scope waits and commits; a 7th stage gained nothing).
constexpr int kPairStages256 = 6;
constexpr int kPairStages128 = 8;
constexpr int kPairStagesWide = 4;  // BN = 512: 16 KB of A + 32 KB of W per stage

// BN <= 256: one MMA of N = BN per k-step, two accumulators (2 x BN TMEM columns) so the
// epilogue of one tile overlaps the main loop of the next.
// BN = 512 ("wide"): two MMAs of N = 256 per k-step (halves h = 0, 1 of the tile's columns)
// on the same A stage, so every gathered A row feeds twice the columns; the accumulator
// takes all 512 TMEM columns. Eight epilogue warps (12-15 and 4-7; the A rows come by
// gather4 from warps 0-3) drain half 0 first and free it on its own barrier, then half 1,
// and the next tile's half-0 MMAs start on the loaded stages as soon as half 0 is free.
// Stream-K: as in the one-CTA kernel, over pairs instead of CTAs; for 256-column tiles on
// request, for 512-column tiles where whole tiles would leave pairs idle (a decode step).
template <int BN, int STAGES>
struct PairSmem {
  static constexpr bool kWide = BN > 256;
  static constexpr int kHalves = kWide ? 2 : 1;
  static constexpr int kMmaN = BN / kHalves;            // N of one MMA
  static constexpr int kABytes = kBM * kBK * 2;         // this CTA's 128 A rows
  static constexpr int kBSubBytes = (kMmaN / 2) * kBK * 2;  // this CTA's rows of one MMA's B
  static constexpr int kBBytes = kHalves * kBSubBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  // epilogue staging: 32 rows x 32 fp32 columns per epilogue warp (8 warps wide, else 4)
  static constexpr int kEpiWarps = kWide ? 8 : 4;
  static constexpr int kEpiWarpBytes = 32 * 32 * 4;
  static constexpr int kEpiOffset = (kBarOffset + kNumBars * 8 + 16 + 127) / 128 * 128;
  static constexpr int kBytes = kEpiOffset + kEpiWarps * kEpiWarpBytes;
  static constexpr int kLaunchBytes = kBytes + 1024;
  static constexpr int kTmemCols = kWide ? 512 : 2 * BN;
  static_assert(kTmemCols <= 512, "accumulators exceed TMEM");
};

// One stream-K piece of a 256-column pair tile (this CTA's 128 rows), as in the one-CTA
// kernel: per (tile, CTA rank, row quarter) an arrival counter counts the pieces published
// so far; the warp whose piece completes the tile sums every piece in pair order (its own
// from TMEM, the others from their owners' partial slots), adds E_0 and scales. A warp
// that finds all other pieces already counted skips publishing its own. Nobody waits for
// anybody. Out of line: the fixup is rare, and inlined its registers press on the
// whole-tile epilogue. Returns false if the accumulator never became ready (abort).
struct PairPiece {
  Seg sg;
  int acc;
  uint32_t use;
  int64_t T, units_total;
  int KB, grid, pair, q, lane;
  uint32_t rank, tmem_base;
  uint32_t tfull, tempty;  // this accumulator's barriers (tempty: CTA 0's, as a cluster address on CTA 1)
  volatile int* abort_flag;
};

template <int BN>
__device__ __noinline__ bool pair_sk_piece(const ProjParams& p, const PairPiece a) {
  const int tile = a.sg.tile;
  const int m_blk = tile / p.num_n_blocks;
  const int n_blk = tile % p.num_n_blocks;
  const int row_in_tile = a.q * 32 + a.lane;
  const int64_t gr = static_cast<int64_t>(m_blk) * (2 * kBM) + a.rank * kBM + row_in_tile;
  const bool valid = gr < a.T;
  uint32_t t = 0;
  if (valid) {
    const int32_t tok = p.tokens[gr];
    t = (tok >= 0 && static_cast<uint32_t>(tok) < p.V0) ? static_cast<uint32_t>(tok) : 0u;
  }
  const uint4* e0 = reinterpret_cast<const uint4*>(p.E0 + static_cast<int64_t>(t) * p.D + n_blk * BN);
  uint4* dst = reinterpret_cast<uint4*>(p.out + gr * p.D + n_blk * BN);
  bool got = false;
  if (a.lane == 0) got = mbar_wait_cluster(a.tfull, a.use & 1u, a.abort_flag, p.status);
  if (!__shfl_sync(0xffffffffu, got, 0)) return false;
  tc_fence_after();
  const uint32_t taddr = a.tmem_base + (static_cast<uint32_t>(a.q * 32) << 16) + static_cast<uint32_t>(a.acc * BN);
  const int64_t u_tile = static_cast<int64_t>(tile) * a.KB;
  const int c_lo = sk_cta_of(u_tile, a.units_total, a.grid), c_hi = sk_cta_of(u_tile + a.KB - 1, a.units_total, a.grid);
  const int others = c_hi - c_lo;  // pieces of the tile besides this one
  int* cnt = p.sk_counters + (tile * 2 + static_cast<int>(a.rank)) * 4 + a.q;
  // partial slots: [pair][rank][slot] x (128 rows x BN columns), column-group major
  auto slot_of = [&](int pr, int sl) {
    return reinterpret_cast<float4*>(p.sk_partials) +
           ((static_cast<size_t>(pr) * 2 + a.rank) * 2 + sl) * (kBM * BN / 4) + row_in_tile;
  };
  int fin = 0;
  if (a.lane == 0) fin = ld_acquire_gpu(cnt) == others;
  fin = __shfl_sync(0xffffffffu, fin, 0);
  if (!fin) {
    // slot 0: the piece that starts this pair's unit range; slot 1: the one that ends it
    float4* mine = slot_of(a.pair, (u_tile + a.sg.i0 == sk_first_unit(a.units_total, a.grid, a.pair)) ? 0 : 1);
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int w = 0; w < 8; ++w)  // a warp's store is 512 contiguous bytes
        mine[(c * 8 + w) * kBM] = make_float4(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1]),
                                              __uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3]));
    }
    __threadfence();
    __syncwarp();
    if (a.lane == 0) fin = atomicAdd(cnt, 1) == others;
    fin = __shfl_sync(0xffffffffu, fin, 0);
    if (fin) __threadfence();
  }
  if (fin) {
    // 16 columns at a time (register pressure): pieces before this pair's, its own
    // (TMEM), those after, in pair order whoever finishes, so the bits do not depend on
    // arrival order
#pragma unroll 1
    for (int c = 0; c < BN / 16; ++c) {
      float sum[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) sum[k] = 0.f;
      auto add_piece = [&](int pr) {
        const float4* part = slot_of(pr, sk_first_unit(a.units_total, a.grid, pr) >= u_tile ? 0 : 1);
        float4 x[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) x[w] = __ldcg(part + (c * 4 + w) * kBM);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          sum[4 * w] += x[w].x;
          sum[4 * w + 1] += x[w].y;
          sum[4 * w + 2] += x[w].z;
          sum[4 * w + 3] += x[w].w;
        }
      };
      for (int pr = c_lo; pr < a.pair; ++pr) add_piece(pr);
      {
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + c * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) sum[k] += __uint_as_float(v[k]);
      }
      for (int pr = a.pair + 1; pr <= c_hi; ++pr) add_piece(pr);
      if (valid) {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const uint4 ev = __ldg(e0 + c * 2 + w);
          const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
          uint32_t o[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int col = w * 8 + h * 2;
            o[h] = pack_bf16x2((sum[col] + bf16_bits_to_float(ew[h] & 0xFFFFu)) * p.scale,
                               (sum[col + 1] + bf16_bits_to_float(ew[h] >> 16)) * p.scale);
          }
          dst[c * 2 + w] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    if (a.lane == 0) *cnt = 0;  // the tile is done: zero again for the next launch
  }
  tc_fence_before();  // accumulator read for the last time: the MMA may reuse it
  if (a.rank == 0) {
    mbar_arrive_relaxed(a.tempty);
  } else {
    __syncwarp();
    if (a.lane == 0) mbar_arrive_remote_relaxed(a.tempty);
  }
  return true;
}

// One stream-K piece of a 256 x 512 pair tile (the 512-column form): this warp's 32 rows
// (TMEM lane quarter q) and its 256 columns (columns g*128 .. +127 of each accumulator half),
// with an arrival counter per (tile, CTA rank, row quarter, column group). As pair_sk_piece,
// but the warp waits for both accumulator halves, and the finished sum of a 32-column chunk
// goes out through the warp's shared-memory staging area like a whole tile's (four lanes per
// row read it back, add E_0, scale and store 64-byte row segments). Partial slots hold
// 128 x 512 fp32. Returns false if the accumulator never became ready (abort).
struct WidePiece {
  Seg sg;
  uint32_t use;
  int64_t T, units_total;
  int KB, grid, pair, q, g, lane;
  uint32_t rank, tmem_base;
  uint32_t tfull0, tfull1, tempty0, tempty1;  // tempty: CTA 0's barriers (cluster addresses on CTA 1)
  uint32_t row_w, rd_lo, rd_hi;                // this warp's staging addresses (see the epilogue)
  volatile int* abort_flag;
};

__device__ __noinline__ bool pair_sk_piece_wide(const ProjParams& p, const WidePiece a) {
  constexpr int kCols = 512;
  const int tile = a.sg.tile;
  const int m_blk = tile / p.num_n_blocks;
  const int n_blk = tile % p.num_n_blocks;
  const int row_in_tile = a.q * 32 + a.lane;
  for (int h = 0; h < 2; ++h) {
    bool got = false;
    if (a.lane == 0) got = mbar_wait_cluster(h ? a.tfull1 : a.tfull0, a.use & 1u, a.abort_flag, p.status);
    if (!__shfl_sync(0xffffffffu, got, 0)) return false;
  }
  tc_fence_after();
  const uint32_t tlane = a.tmem_base + (static_cast<uint32_t>(a.q * 32) << 16);
  // chunk c (0..7) of this warp: tile column (= accumulator column) (c / 4) * 256 + g * 128 + (c % 4) * 32
  auto chunk_col = [&](int c) { return (c >> 2) * 256 + a.g * 128 + (c & 3) * 32; };
  const int64_t u_tile = static_cast<int64_t>(tile) * a.KB;
  const int c_lo = sk_cta_of(u_tile, a.units_total, a.grid), c_hi = sk_cta_of(u_tile + a.KB - 1, a.units_total, a.grid);
  const int others = c_hi - c_lo;  // pieces of the tile besides this one
  int* cnt = p.sk_counters + ((tile * 2 + static_cast<int>(a.rank)) * 4 + a.q) * 2 + a.g;
  // partial slots: [pair][rank][slot] x (128 rows x 512 columns), column-group major
  auto slot_of = [&](int pr, int sl) {
    return reinterpret_cast<float4*>(p.sk_partials) +
           ((static_cast<size_t>(pr) * 2 + a.rank) * 2 + sl) * (kBM * kCols / 4) + row_in_tile;
  };
  int fin = 0;
  if (a.lane == 0) fin = ld_acquire_gpu(cnt) == others;
  fin = __shfl_sync(0xffffffffu, fin, 0);
  if (!fin) {
    // slot 0: the piece that starts this pair's unit range; slot 1: the one that ends it
    float4* mine = slot_of(a.pair, (u_tile + a.sg.i0 == sk_first_unit(a.units_total, a.grid, a.pair)) ? 0 : 1);
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      const int col = chunk_col(c);
      uint32_t v[32];
      tmem_ld_32x32b_x32(tlane + col, v);
      tmem_wait_ld();
#pragma unroll
      for (int w = 0; w < 8; ++w)  // a warp's store is 512 contiguous bytes
        mine[((col >> 5) * 8 + w) * kBM] = make_float4(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1]),
                                                      __uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3]));
    }
    __threadfence();
    __syncwarp();
    if (a.lane == 0) fin = atomicAdd(cnt, 1) == others;
    fin = __shfl_sync(0xffffffffu, fin, 0);
    if (fin) __threadfence();
  }
  if (fin) {
    const int rsub = a.lane >> 2, u2 = a.lane & 3;  // read-back: rows i*8 + rsub, columns u2*8 .. +7
    const int col0 = n_blk * kCols;
    const int64_t row0 = static_cast<int64_t>(m_blk) * (2 * kBM) + a.rank * kBM + a.q * 32;
    const uint16_t* e0row[4];
    bool valid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t gr = row0 + i * 8 + rsub;
      valid[i] = gr < a.T;
      uint32_t t = 0;
      if (valid[i]) {
        const int32_t tok = p.tokens[gr];
        t = (tok >= 0 && static_cast<uint32_t>(tok) < p.V0) ? static_cast<uint32_t>(tok) : 0u;
      }
      e0row[i] = p.E0 + static_cast<int64_t>(t) * p.D + col0 + u2 * 8;
    }
    uint4* dst0 = reinterpret_cast<uint4*>(p.out + (row0 + rsub) * p.D + col0 + u2 * 8);
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      const int col = chunk_col(c);
      // pieces in pair order, whoever finishes: those before this pair's, its own (TMEM),
      // those after, so the bits do not depend on arrival order
      float sum[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) sum[k] = 0.f;
      auto add_piece = [&](int pr) {
        const float4* part = slot_of(pr, sk_first_unit(a.units_total, a.grid, pr) >= u_tile ? 0 : 1);
        float4 x[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) x[w] = __ldcg(part + ((col >> 5) * 8 + w) * kBM);
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          sum[4 * w] += x[w].x;
          sum[4 * w + 1] += x[w].y;
          sum[4 * w + 2] += x[w].z;
          sum[4 * w + 3] += x[w].w;
        }
      };
      for (int pr = c_lo; pr < a.pair; ++pr) add_piece(pr);
      {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tlane + col, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) sum[k] += __uint_as_float(v[k]);
      }
      for (int pr = a.pair + 1; pr <= c_hi; ++pr) add_piece(pr);
      // stage the 32 x 32 chunk (row per lane), read it back four lanes per row
#pragma unroll
      for (int w = 0; w < 8; ++w)
        st_shared_v4(a.row_w + (static_cast<uint32_t>(w ^ (a.lane & 7)) << 4),
                     make_uint4(__float_as_uint(sum[4 * w]), __float_as_uint(sum[4 * w + 1]),
                                __float_as_uint(sum[4 * w + 2]), __float_as_uint(sum[4 * w + 3])));
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 lo = ld_shared_v4(a.rd_lo + i * 8 * 128);
        const uint4 hi = ld_shared_v4(a.rd_hi + i * 8 * 128);
        if (valid[i]) {
          const uint4 ev = __ldg(reinterpret_cast<const uint4*>(e0row[i] + col));
          const float x[8] = {__uint_as_float(lo.x), __uint_as_float(lo.y), __uint_as_float(lo.z), __uint_as_float(lo.w),
                              __uint_as_float(hi.x), __uint_as_float(hi.y), __uint_as_float(hi.z), __uint_as_float(hi.w)};
          const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
          uint32_t o[4];
#pragma unroll
          for (int h = 0; h < 4; ++h)
            o[h] = pack_bf16x2((x[2 * h] + bf16_bits_to_float(ew[h] & 0xFFFFu)) * p.scale,
                               (x[2 * h + 1] + bf16_bits_to_float(ew[h] >> 16)) * p.scale);
          dst0[static_cast<int64_t>(i) * p.D + col / 8] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      __syncwarp();  // the staging area is rewritten by the next chunk
    }
    if (a.lane == 0) *cnt = 0;  // the tile is done: zero again for the next launch
  }
  tc_fence_before();  // both halves read for the last time: the MMA may reuse them
  if (a.rank == 0) {
    mbar_arrive_relaxed(a.tempty0);
    mbar_arrive_relaxed(a.tempty1);
  } else {
    __syncwarp();
    if (a.lane == 0) {
      mbar_arrive_remote_relaxed(a.tempty0);
      mbar_arrive_remote_relaxed(a.tempty1);
    }
  }
  return true;
}

// WSK: 512-column tiles under the stream-K schedule (a separate instance, so that the
// whole-tile kernel of the prefill carries none of the piece code's registers).
template <int BN, int STAGES, bool WSK = false>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_sm100_pair_kernel(const __grid_constant__ ProjMaps maps, const __grid_constant__ ProjParams p) {
  using L = PairSmem<BN, STAGES>;
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
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs and owns the stage barriers
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  constexpr bool kWide = L::kWide;
  constexpr int kMmaN = L::kMmaN;
  // stream-K: the (tile, k-block) units split evenly over the pairs
  const bool sk = (!L::kWide || WSK) && p.stream_k != 0;
  const bool dense = p.dense_a != 0;                                // A by 2-D TMA boxes of G
  const bool cp_rows = !kWide && !sk && !dense && p.tma_rows == 0;  // A rows by cp.async (else all by TMA gather4)
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // CTA 0: thread 0 posts the pair's TMA bytes (+ its 256 cp.async threads + CTA 1's relay);
      // CTA 1: its 256 cp.async threads (unused in TMA-only mode)
      const uint32_t arrivals = rank == 0 ? (cp_rows ? 1u + static_cast<uint32_t>(kAThreads) + 1u : 1u)
                                          : static_cast<uint32_t>(kAThreads);
      mbar_init(full_bar(s), arrivals);
      mbar_init(empty_bar(s), 1u);  // one tcgen05.commit from CTA 0's MMA thread
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1u);
      // CTA 0: the threads of its epilogue warps + one remote arrive per CTA 1 epilogue warp
      mbar_init(tempty_bar(a), kWide ? 256u + 8u : 128u + 4u);
    }
    mbar_init(drain_bar, 1u);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpB && lane == 0) {
    tma_prefetch_desc(&maps.Whalf);
    if (p.dense_a) tma_prefetch_desc(&maps.A);
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();  // nothing above touched global memory

  const int64_t T = p.T_dev ? (*p.T_dev < p.T ? *p.T_dev : p.T) : p.T;
  const int num_tiles = static_cast<int>((T + 2 * kBM - 1) / (2 * kBM)) * p.num_n_blocks;  // m blocks of 256 rows
  const int KB = p.num_k_blocks;
  const int kb_per_sub = p.d / kBK;
  // Work list of this pair: whole tiles pair, pair + num_pairs, ...; or, under stream-K, an
  // equal run of units (pairs past the unit count, known only here, hold none).
  const int64_t units_total = static_cast<int64_t>(num_tiles) * KB;
  WorkPlan wp;
  wp.num_tiles = num_tiles;
  wp.KB = KB;
  wp.grid = (sk && units_total < num_pairs) ? static_cast<int>(units_total) : num_pairs;
  wp.sk = sk ? 1 : 0;
  wp.u_end = sk ? sk_first_unit(units_total, wp.grid, pair + 1) : 0;

  const bool epi_warp = warp >= kWarpEpi0 || (kWide && warp >= kAWarps / 2 && warp < kAWarps);
  if (warp < kAWarps && !epi_warp && !dense) {
    // ------------------------------------------------------------ A producers (own 128 rows)
    const int t = threadIdx.x;
    const int chunk = t & 7, rsub = t >> 3;                         // cp.async mode
    const uint32_t swz = static_cast<uint32_t>((chunk ^ (rsub & 7)) << 4);
    // gather4 mode: 32 issuing lanes x 4 rows (wide: lanes 0-7 of warps 0-3, else 0-3 of 0-7)
    const bool issuer = !cp_rows && lane < (kWide ? 8 : 4);
    const int iss = kWide ? warp * 8 + lane : warp * 4 + lane;
    const uint32_t pair_tx = cp_rows ? 2u * L::kBBytes : 2u * (L::kABytes + L::kBBytes);
    const uint64_t pol = l2_policy_evict_normal();
    // raw row indices (this thread's 4 rows) of the current and the next run
    int32_t raw[4], nraw[4];
    auto load_raw = [&](const SRun& r, int32_t (&dst)[4]) {
      const int64_t row_base = static_cast<int64_t>(r.g.tile / p.num_n_blocks) * (2 * kBM) + rank * kBM;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t gr = row_base + (cp_rows ? rsub + 32 * j : iss * 4 + j);
        dst[j] = ((cp_rows || issuer) && gr < T) ? ld_idx_early(p.idx + gr * p.S + r.s) : 0;
      }
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    const Seg g0 = seg_first(wp, pair);
    SRun cur = srun_at(g0, g0.i0, p.num_n_blocks, KB, kb_per_sub);
    if (cur.g.tile < num_tiles) load_raw(cur, raw);
    SRun nxt = srun_next(wp, cur, p.num_n_blocks, kb_per_sub);
    if (nxt.g.tile < num_tiles) load_raw(nxt, nraw);
    while (cur.g.tile < num_tiles && ok) {
      const uint32_t V = p.Vs[cur.s];
      const uint16_t* src[4];
      int32_t r4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t ix = clamp_row(raw[j], V, p.status);
        src[j] = p.E[cur.s] + static_cast<int64_t>(ix) * p.d + chunk * 8;
        r4[j] = static_cast<int32_t>(ix);
      }
      for (int q = 0; q < cur.len; ++q) {
        const int c0 = (cur.c_first + q) * kBK;
        if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
        const uint32_t a = a_tile(stage);
        if (rank == 0 && t == 0) mbar_arrive_expect_tx(full_bar(stage), pair_tx);
        if (cp_rows) {
#pragma unroll
          for (int j = 0; j < 4; ++j) cp_async_16(a + (rsub + 32 * j) * 128 + swz, src[j] + c0);
          cp_async_arrive_noinc(full_bar(stage));
        } else if (issuer) {
          tma_gather4_pair(a + iss * 512, &maps.E[cur.s], c0, r4[0], r4[1], r4[2], r4[3],
                           map_to_cta(full_bar(stage), 0), pol);
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      cur = nxt;
#pragma unroll
      for (int j = 0; j < 4; ++j) raw[j] = nraw[j];
      nxt = srun_next(wp, nxt, p.num_n_blocks, kb_per_sub);
      if (nxt.g.tile < num_tiles) load_raw(nxt, nraw);
    }
    cp_async_wait_all();
    if (!ok) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 1000ull * 1000ull) __nanosleep(1000);
    }
  } else if (warp == kWarpB) {
    // ------------------------------------------------------------ W producer (own BN/2 rows)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint64_t pol_a = l2_policy_evict_normal();
      for (Seg g = seg_first(wp, pair); g.tile < num_tiles && ok; g = seg_next(wp, g)) {
        const int n_blk = g.tile % p.num_n_blocks;
        const int m_blk = g.tile / p.num_n_blocks;
        const int rot = k_rotation(m_blk, n_blk, KB);
        for (int i = g.i0; i < g.i1; ++i) {
          int kb = i + rot;
          if (kb >= KB) kb -= KB;
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          if (dense) {
            // this CTA's 128 rows of the k-block as one box of G (rows past T read zeros)
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2u * (L::kABytes + L::kBBytes));
            tma_load_2d_pair(a_tile(stage), &maps.A, kb * kBK, m_blk * (2 * kBM) + static_cast<int>(rank) * kBM,
                             map_to_cta(full_bar(stage), 0), pol_a);
          }
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_2d_pair(b_tile(stage) + h * L::kBSubBytes, &maps.Whalf, kb * kBK,
                             n_blk * BN + h * kMmaN + static_cast<int>(rank) * (kMmaN / 2),
                             map_to_cta(full_bar(stage), 0), pol);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(2 * kBM, kMmaN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      auto advance = [&](int& st, uint32_t& ph) { if (++st == STAGES) { st = 0; ph ^= 1u; } };
      // the MMAs of half h (all of the tile when not wide) on stage st: k-block j of a segment
      // of nj k-blocks (a segment starts a fresh sum)
      auto issue = [&](int st, int h, int j, int nj, uint32_t d_tmem) {
        const uint64_t adesc = sw128_kmajor_desc(a_tile(st));
        const uint64_t bdesc = sw128_kmajor_desc(b_tile(st) + h * L::kBSubBytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16_pair(d_tmem + h * kMmaN, adesc + 2u * k, bdesc + 2u * k, idesc, (j | k) != 0 ? 1u : 0u);
        if (kWide && j + 1 == nj) {  // half h complete: its epilogue may start
          umma_commit_pair_both(tfull_bar(h));
        }
      };
      auto release = [&](int st) {
        umma_commit_pair_both(empty_bar(st));
      };
      for (Seg g = seg_first(wp, pair); g.tile < num_tiles && ok; g = seg_next(wp, g), ++local) {
        // one accumulator of both halves (wide), else two alternating ones
        const int acc = kWide ? 0 : (local & 1);
        const uint32_t use = static_cast<uint32_t>(kWide ? local : local >> 1);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const int nj = g.i1 - g.i0;  // k-blocks of this segment (the whole tile unless stream-K)
        int j0 = 0;
        if (kWide) {
          // The epilogue frees half 0 of the previous tile first: the MMAs of half 0 run on
          // the stages already loaded while half 1 is still being drained; those stages'
          // half-1 MMAs (same per-element order) and releases follow once it is free.
          const int pre = nj < STAGES ? nj : STAGES;
          if (!mbar_wait_cluster(tempty_bar(0), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          int st = stage;
          uint32_t ph = phase;
          for (int j = 0; j < pre; ++j) {
            if (!mbar_wait_cluster(full_bar(st), ph, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            issue(st, 0, j, nj, d_tmem);
            advance(st, ph);
          }
          if (!ok) break;
          if (!mbar_wait_cluster(tempty_bar(1), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          for (int j = 0; j < pre; ++j) {
            issue(stage, 1, j, nj, d_tmem);
            release(stage);
            advance(stage, phase);
          }
          j0 = pre;
        } else {
          if (!mbar_wait_cluster(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
        }
        for (int j = j0; j < nj; ++j) {
          if (!mbar_wait_cluster(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          if (cp_rows) fence_proxy_async_smem();  // this CTA's cp.async rows: generic proxy writes
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h) issue(stage, h, j, nj, d_tmem);
          release(stage);
          advance(stage, phase);
        }
        if (ok && !kWide) {
          umma_commit_pair_both(tfull_bar(acc));
        }
      }
      umma_commit_pair(map_to_cta(drain_bar, 0));
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp == kWarpRelay) {
    // ------------------------------------------------------------ relay (CTA 1, cp.async mode)
    // Lane l handles stages l, l + STAGES, ...: waits for CTA 1's cp.async rows of the stage,
    // fences them for the async proxy and arrives on CTA 0's stage barrier.
    if (cp_rows && rank == 1 && lane < STAGES) {
      const int my_tiles = (num_tiles - pair + num_pairs - 1) / num_pairs;
      const int total = my_tiles > 0 ? my_tiles * KB : 0;
      const uint32_t remote = map_to_cta(full_bar(lane), 0);
      uint32_t phase = 0;
      for (int k = lane; k < total; k += STAGES) {
        if (!mbar_wait(full_bar(lane), phase, abort_flag, p.status)) break;
        fence_proxy_async_smem();
        mbar_arrive_remote(remote);
        phase ^= 1u;
      }
    }
  } else if (epi_warp) {
    // ------------------------------------------------------------ epilogue (own 128 rows)
    // Per 32-column chunk: each lane reads its row's fp32 accumulators from TMEM (32x32b
    // shape: lane = row) and writes them to this warp's staging area in shared memory; then
    // four lanes per row read them back 8 columns each, add the E_0 slice, scale, round and
    // store, so each global access instruction covers 8 rows x 64 contiguous bytes instead
    // of 32 rows x 16 bytes (a quarter of the lines through L1 for the E_0 reads and the
    // output writes). Same arithmetic per element: (acc + E_0) * scale, rounded once.
    // Wide tiles: all eight warps drain half 0 first (warps 12-15 its columns 0-127, warps
    // 4-7 columns 128-255), free it, then half 1 the same way, so half 0 is free for the
    // next tile's MMAs after half of the drain. A stream-K segment that covers only part of
    // a tile is handed to pair_sk_piece.
    constexpr int kSegs = kWide ? 2 : 1;                 // accumulator halves, in drain order
    constexpr int kSegChunks = (kWide ? 128 : kMmaN) / 32;
    constexpr int kChunks = kSegs * kSegChunks;
    const int q = warp & 3;  // TMEM lanes q*32 .. q*32+31 (warp w reaches quadrant w % 4)
    const int g = kWide && warp < kWarpEpi0 ? 1 : 0;    // wide: column group of each half
    const uint32_t stg = sbase + L::kEpiOffset + static_cast<uint32_t>(g * 4 + q) * L::kEpiWarpBytes;
    const int rsub = lane >> 2, u2 = lane & 3;  // read-back: rows i*8 + rsub, columns u2*8 .. u2*8+7
    // staging layout: row r at r*128 bytes, 16-byte unit w at ((w ^ (r & 7)) << 4): conflict-free
    // for both the row-per-lane writes and the 4-lanes-per-row reads
    const uint32_t row_w = stg + static_cast<uint32_t>(lane) * 128u;
    const uint32_t rd_lo = stg + static_cast<uint32_t>(rsub) * 128u + (static_cast<uint32_t>((2 * u2) ^ rsub) << 4);
    const uint32_t rd_hi = stg + static_cast<uint32_t>(rsub) * 128u + (static_cast<uint32_t>((2 * u2 + 1) ^ rsub) << 4);
    const uint32_t tempty_remote0 = map_to_cta(tempty_bar(0), 0);
    const uint32_t tempty_remote1 = map_to_cta(tempty_bar(1), 0);
    // chunk cc: its first column relative to col0 (output / E_0) and within the accumulator
    auto chunk_col = [&](int cc) { return (kWide ? (cc / kSegChunks) * kMmaN : 0) + (cc % kSegChunks) * 32; };
    int local = 0;
    for (Seg sg = seg_first(wp, pair); sg.tile < num_tiles; sg = seg_next(wp, sg), ++local) {
      const int tile = sg.tile;
      const int m_blk = tile / p.num_n_blocks;
      const int n_blk = tile % p.num_n_blocks;
      const int acc = kWide ? 0 : (local & 1);
      const uint32_t use = static_cast<uint32_t>(kWide ? local : local >> 1);
      if (WSK && kWide && (sg.i0 != 0 || sg.i1 != KB)) {
        WidePiece pc;
        pc.sg = sg;
        pc.use = use;
        pc.T = T;
        pc.units_total = units_total;
        pc.KB = KB;
        pc.grid = wp.grid;
        pc.pair = pair;
        pc.q = q;
        pc.g = g;
        pc.lane = lane;
        pc.rank = rank;
        pc.tmem_base = tmem_base;
        pc.tfull0 = tfull_bar(0);
        pc.tfull1 = tfull_bar(1);
        pc.tempty0 = rank == 0 ? tempty_bar(0) : tempty_remote0;
        pc.tempty1 = rank == 0 ? tempty_bar(1) : tempty_remote1;
        pc.row_w = row_w;
        pc.rd_lo = rd_lo;
        pc.rd_hi = rd_hi;
        pc.abort_flag = abort_flag;
        if (!pair_sk_piece_wide(p, pc)) break;
        continue;
      }
      if (!kWide && (sg.i0 != 0 || sg.i1 != KB)) {
        PairPiece pc;
        pc.sg = sg;
        pc.acc = acc;
        pc.use = use;
        pc.T = T;
        pc.units_total = units_total;
        pc.KB = KB;
        pc.grid = wp.grid;
        pc.pair = pair;
        pc.q = q;
        pc.lane = lane;
        pc.rank = rank;
        pc.tmem_base = tmem_base;
        pc.tfull = tfull_bar(acc);
        pc.tempty = rank == 0 ? tempty_bar(acc) : (acc ? tempty_remote1 : tempty_remote0);
        pc.abort_flag = abort_flag;
        if (!pair_sk_piece<BN>(p, pc)) break;
        continue;
      }
      const int col0 = n_blk * BN + g * 128;
      const int64_t row0 = static_cast<int64_t>(m_blk) * (2 * kBM) + rank * kBM + q * 32;
      // this lane's four read-back rows: E_0 and output addresses of its 8 columns
      const uint4* e0r[4];
      // output rows i*8 + rsub: row i is i * D / 8 vectors of 8 columns past row 0
      uint4* dst0 = reinterpret_cast<uint4*>(p.out + (row0 + rsub) * p.D + col0 + u2 * 8);
      bool valid[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t gr = row0 + i * 8 + rsub;
        valid[i] = gr < T;
        uint32_t t = 0;
        if (valid[i]) {
          const int32_t tok = p.tokens[gr];
          t = (tok >= 0 && static_cast<uint32_t>(tok) < p.V0) ? static_cast<uint32_t>(tok) : 0u;
        }
        const uint16_t* row_e0 = p.E0 + static_cast<int64_t>(t) * p.D + col0;
        e0r[i] = reinterpret_cast<const uint4*>(row_e0 + u2 * 8);
        // the row's E_0 columns of this warp toward L2 while the tile's main loop runs: line
        // u2 of them (wide: 2 lines in each half, else kMmaN * 2 / 128 lines)
        constexpr int kLines = kWide ? 4 : kMmaN * 2 / 128;
        if (valid[i] && u2 < kLines)
          prefetch_l2(reinterpret_cast<const uint8_t*>(row_e0) +
                      (kWide ? (u2 >> 1) * kMmaN * 2 + (u2 & 1) * 128 : u2 * 128));
      }
      uint4 e[kChunks][4];  // E_0 of chunk c, row i: loaded two chunks ahead
#pragma unroll
      for (int c = 0; c < 2 && c < kChunks; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) e[c][i] = valid[i] ? __ldg(e0r[i] + chunk_col(c) / 8) : make_uint4(0, 0, 0, 0);

      bool alive = true;
#pragma unroll
      for (int cc = 0; cc < kChunks; ++cc) {
        const int seg = cc / kSegChunks;
        const int bar = kWide ? seg : acc;
        if (cc % kSegChunks == 0) {
          bool got = false;
          if (lane == 0) got = mbar_wait_cluster(tfull_bar(bar), use & 1u, abort_flag, p.status);
          if (!__shfl_sync(0xffffffffu, got, 0)) { alive = false; break; }
          tc_fence_after();
        }
        const uint32_t tcol = (kWide ? static_cast<uint32_t>(seg * kMmaN + g * 128) : static_cast<uint32_t>(acc * kMmaN)) +
                              static_cast<uint32_t>((cc % kSegChunks) * 32);
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + tcol, v);
        if (cc + 2 < kChunks) {
#pragma unroll
          for (int i = 0; i < 4; ++i) e[cc + 2][i] = valid[i] ? __ldg(e0r[i] + chunk_col(cc + 2) / 8) : make_uint4(0, 0, 0, 0);
        }
        tmem_wait_ld();
        if (cc % kSegChunks == kSegChunks - 1) {  // this warp's last read of the segment
          tc_fence_before();
          if (rank == 0) {
            mbar_arrive_relaxed(tempty_bar(bar));
          } else {
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(bar ? tempty_remote1 : tempty_remote0);
          }
        }
#pragma unroll
        for (int w = 0; w < 8; ++w)
          st_shared_v4(row_w + (static_cast<uint32_t>(w ^ (lane & 7)) << 4),
                       make_uint4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 lo = ld_shared_v4(rd_lo + i * 8 * 128);
          const uint4 hi = ld_shared_v4(rd_hi + i * 8 * 128);
          if (valid[i]) {
            const float a[8] = {__uint_as_float(lo.x), __uint_as_float(lo.y), __uint_as_float(lo.z), __uint_as_float(lo.w),
                                __uint_as_float(hi.x), __uint_as_float(hi.y), __uint_as_float(hi.z), __uint_as_float(hi.w)};
            const uint32_t ew[4] = {e[cc][i].x, e[cc][i].y, e[cc][i].z, e[cc][i].w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float x0 = (a[2 * h] + bf16_bits_to_float(ew[h] & 0xFFFFu)) * p.scale;
              const float x1 = (a[2 * h + 1] + bf16_bits_to_float(ew[h] >> 16)) * p.scale;
              o[h] = pack_bf16x2(x0, x1);
            }
            dst0[static_cast<int64_t>(i) * p.D + chunk_col(cc) / 8] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        __syncwarp();  // the staging area is rewritten by the next chunk
      }
      if (!alive) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrive or pair MMA is outstanding past this point
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

}  // namespace ngram
