// CTA-pair form of the fused gather + projection + epilogue kernel with the output split
// by column ranges instead of tiles (Eq. 3 of "Scaling Embeddings Outperforms Scaling
// Experts in Language Models", section 2: out = (E_0[t] + G W_stacked^T) / (S + 1)).
//
// When the 256 x 512 tiles of a call are fewer than the CTA pairs (a decode step: 1280
// tokens at D = 4096 make 40 tiles for 74 pairs), whole tiles leave pairs idle and a
// stream-K split pays for fp32 partial sums that one piece writes and another reads back
// at the end of the launch. Here every pair instead computes the full K of a contiguous
// range of columns of one 256-row block: the pairs are spread evenly over the row blocks
// and each block's D columns are cut into as many near-equal ranges (multiples of 64
// columns) as it has pairs. No partial sums, no fix-ups; the pair's cost is its column
// count, which differs between pairs by at most 64 columns.
//
// A range of c columns (a multiple of 64) runs as two MMAs of N = c/2 per k-step on the same
// A stage (M = 256, tcgen05.mma.cta_group::2), the halves' accumulators at TMEM columns
// [0, c/2) and [256, 256 + c/2). Equal halves, because an MMA's time does not shrink below
// that of N = 128 (measured on B200: a k-block of N = 32, 64 or 128 took 453 cycles, one of
// N = 256 518-541), so a small second MMA would cost as much as a 128-column one. Each CTA
// holds its 128 A rows (16-byte cp.async from the sub-tables) and c/4 rows of W per half
// (2-D TMA: one 128-row box for a 256-column half, else boxes of 64 and 16 rows). A range wider
// than 512 columns (fewer pairs than row blocks times D / 512) is cut into segments of at
// most 512 columns, each a full pass over K.
//
// Roles and synchronisation are those of the pair kernel (warps 0-3: A rows by cp.async, 8: W
// by TMA, 9: MMA on CTA 0, 10: CTA 1's stage relay, 4-7 and 12-15: epilogue), all plain loads
// and barriers, no multicast. With dense A (the call's sub-rows already gathered into G by one
// launch over the whole GPU), warp 8 also brings in each CTA's 128 A rows as one 2-D TMA box
// of G per stage and warps 0-3 and 10 stay idle: the rows are gathered at full-GPU rate
// instead of at one SM's. The
// epilogue drains half 0 first and frees it on its own barrier, so a pair with several
// segments starts the next segment's half-0 MMAs while half 1 is still being drained.
#pragma once

#include "proj_sm100_pair.cuh"

namespace ngram {

// Stage: this CTA's 128 A rows (16 KB) and its rows of the two halves of the B tile (up to
// HROWS rows each: a range of up to 4 * HROWS columns).
template <int HROWS, int STAGES>
struct ColsSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBHalfBytes = HROWS * kBK * 2;
  static constexpr int kStageBytes = kABytes + 2 * kBHalfBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kEpiWarpBytes = 32 * 32 * 4;  // a 32 x 32 fp32 chunk per epilogue warp
  static constexpr int kEpiOffset = (kBarOffset + kNumBars * 8 + 16 + 127) / 128 * 128;
  static constexpr int kBytes = kEpiOffset + 8 * kEpiWarpBytes;
  static constexpr int kLaunchBytes = kBytes + 1024;
  static_assert(kBHalfBytes % 1024 == 0, "tiles keep the 1024-byte alignment of 128-byte swizzling");
  static_assert(HROWS % 16 == 0 && HROWS >= 16 && HROWS <= 128, "a half holds 64 .. 512 columns' rows");
};

// This pair's share of the (256-row block, 64-column unit) grid: row blocks [m0, m1), units
// [u_lo, u_hi) of each, cut into nseg near-equal segments of at most 8 units per block.
struct ColWork {
  int m0, m1, u_lo, u_hi, nseg;
};

__host__ __device__ inline ColWork col_work(int pair, int pairs, int64_t mblocks, int units) {
  ColWork w;
  if (pairs >= mblocks) {
    // pairs spread evenly over the row blocks; block m has pairs [first(m), first(m + 1))
    const int m = static_cast<int>(static_cast<int64_t>(pair) * mblocks / pairs);
    const int first = static_cast<int>((static_cast<int64_t>(m) * pairs + mblocks - 1) / mblocks);
    const int next = static_cast<int>((static_cast<int64_t>(m + 1) * pairs + mblocks - 1) / mblocks);
    const int cnt = next - first, j = pair - first;
    w.m0 = m;
    w.m1 = m + 1;
    w.u_lo = static_cast<int>(static_cast<int64_t>(j) * units / cnt);
    w.u_hi = static_cast<int>(static_cast<int64_t>(j + 1) * units / cnt);
  } else {
    // fewer pairs than row blocks: whole blocks, split evenly over the pairs
    w.m0 = static_cast<int>(static_cast<int64_t>(pair) * mblocks / pairs);
    w.m1 = static_cast<int>(static_cast<int64_t>(pair + 1) * mblocks / pairs);
    w.u_lo = 0;
    w.u_hi = units;
  }
  w.nseg = (w.u_hi - w.u_lo + 7) / 8;
  return w;
}

// Segment k of a pair's work (k < (m1 - m0) * nseg): its row block, first column and width.
struct ColSeg {
  int m_blk, col0, ncols;
};

__host__ __device__ inline ColSeg col_seg(const ColWork& w, int k) {
  ColSeg s;
  const int n = w.u_hi - w.u_lo;
  const int b = k / w.nseg, i = k - b * w.nseg;
  const int lo = w.u_lo + static_cast<int>(static_cast<int64_t>(i) * n / w.nseg);
  const int hi = w.u_lo + static_cast<int>(static_cast<int64_t>(i + 1) * n / w.nseg);
  s.m_blk = w.m0 + b;
  s.col0 = lo * 64;
  s.ncols = (hi - lo) * 64;
  return s;
}

template <int HROWS, int STAGES>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_sm100_cols_kernel(const __grid_constant__ ProjMaps maps, const __grid_constant__ ProjParams p) {
  using L = ColsSmem<HROWS, STAGES>;
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
  auto b_tile = [&](int s, int h) { return sbase + s * L::kStageBytes + L::kABytes + h * L::kBHalfBytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs and owns the stage barriers
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int num_pairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // CTA 0: thread 0's W byte count + its 128 cp.async threads + CTA 1's relay; CTA 1: its
      // 128 cp.async threads. Dense A: the W producer's byte count for everything (CTA 0).
      mbar_init(full_bar(s), p.dense_a ? 1u : (rank == 0 ? 130u : 128u));
      mbar_init(empty_bar(s), 1u);  // one tcgen05.commit from CTA 0's MMA thread
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
  if (warp == kWarpB && lane == 0) {
    tma_prefetch_desc(&maps.Whalf);
    tma_prefetch_desc(&maps.W16);
    tma_prefetch_desc(&maps.W64);
    if (p.dense_a) tma_prefetch_desc(&maps.A);
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512u);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();  // nothing above touched global memory

  const int64_t T = p.T;
  const int64_t mblocks = (T + 2 * kBM - 1) / (2 * kBM);
  const int KB = p.num_k_blocks;
  const int kb_per_sub = p.d / kBK;
  const ColWork cw = col_work(pair, num_pairs, mblocks, p.D / 64);
  const int nsegs = (cw.m1 - cw.m0) * cw.nseg;
  const int rot = k_rotation(cw.m0, pair, KB);  // first k-block: differs between pairs side by side
  auto kblock = [&](int i) { const int kb = i + rot; return kb >= KB ? kb - KB : kb; };

  const bool epi_warp = warp >= kWarpEpi0 || (warp >= kAWarps / 2 && warp < kAWarps);
  const bool dense = p.dense_a != 0;  // A rows already gathered into G: one 2-D TMA box per stage
  if (warp < kAWarps / 2) {
    // ------------------------------------------------------------ A producers (own 128 rows)
    // 16-byte cp.async (no TMA: the TMA unit issues about one copy per 30-40 cycles, so 32
    // row gathers per stage would cap the stage rate): thread t copies chunk t % 8 of rows
    // t / 8 + 16 j, j < 8. Its completion arrives on this CTA's stage barrier; CTA 1's
    // stages are relayed to CTA 0's barrier by warp 10.
    const int t = threadIdx.x;  // 0..127
    const int chunk = t & 7, rsub = t >> 3;
    const uint32_t swz = static_cast<uint32_t>((chunk ^ (rsub & 7)) << 4);  // row r: r % 8 == rsub % 8
    // A run: consecutive k-blocks of one segment that read one sub-table. The row indices of
    // the next run are loaded while the current run's rows are copied.
    struct Run {
      int k, i, s, c_first, len;
    };
    auto run_at = [&](int k, int i) {
      Run r;
      r.k = k;
      r.i = i;
      const int kb = kblock(i);
      r.s = kb / kb_per_sub;
      r.c_first = kb - r.s * kb_per_sub;
      r.len = (kb_per_sub - r.c_first) < (KB - i) ? (kb_per_sub - r.c_first) : (KB - i);
      return r;
    };
    auto run_next = [&](const Run& r) { return r.i + r.len < KB ? run_at(r.k, r.i + r.len) : run_at(r.k + 1, 0); };
    auto load_rows = [&](const Run& r, int32_t (&dst)[8]) {
      const int64_t row_base = static_cast<int64_t>(col_seg(cw, r.k).m_blk) * (2 * kBM) + rank * kBM + rsub;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t gr = row_base + 16 * j;
        dst[j] = gr < T ? ld_idx_early(p.idx + gr * p.S + r.s) : 0;
      }
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int32_t raw[8], nraw[8];
    Run cur = run_at(dense ? nsegs : 0, 0);  // dense A: nothing to copy here
    if (cur.k < nsegs) load_rows(cur, raw);
    Run nxt = run_next(cur);
    if (nxt.k < nsegs) load_rows(nxt, nraw);
    while (cur.k < nsegs && ok) {
      const uint32_t w_tx = static_cast<uint32_t>(col_seg(cw, cur.k).ncols * 128);  // both CTAs' W rows
      const uint16_t* src[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        src[j] = p.E[cur.s] + static_cast<int64_t>(clamp_row(raw[j], p.Vs[cur.s], p.status)) * p.d + chunk * 8;
      for (int q = 0; q < cur.len; ++q) {
        const int c0 = (cur.c_first + q) * kBK;
        if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
        if (rank == 0 && t == 0) mbar_arrive_expect_tx(full_bar(stage), w_tx);
        const uint32_t a = a_tile(stage);
#pragma unroll
        for (int j = 0; j < 8; ++j) cp_async_16(a + (rsub + 16 * j) * 128 + swz, src[j] + c0);
        cp_async_arrive_noinc(full_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      cur = nxt;
#pragma unroll
      for (int j = 0; j < 8; ++j) raw[j] = nraw[j];
      nxt = run_next(nxt);
      if (nxt.k < nsegs) load_rows(nxt, nraw);
    }
    cp_async_wait_all();
  } else if (warp == kWarpB) {
    // ------------------------------------------------------------ W producer (own rows of each half)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      const uint64_t pol_a = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int k = 0; k < nsegs && ok; ++k) {
        const ColSeg sg = col_seg(cw, k);
        const int rows = sg.ncols / 4;  // this CTA's rows of each half
        for (int i = 0; i < KB; ++i) {
          const int kb = kblock(i);
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          if (dense) {
            // this CTA's 128 rows of G as one box (rows past T read zeros); CTA 0 posts the
            // pair's bytes of A and W
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2u * static_cast<uint32_t>(L::kABytes + sg.ncols * 64));
            tma_load_2d_pair(a_tile(stage), &maps.A, kb * kBK, sg.m_blk * (2 * kBM) + static_cast<int>(rank) * kBM,
                             map_to_cta(full_bar(stage), 0), pol_a);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row0 = sg.col0 + h * (sg.ncols / 2) + static_cast<int>(rank) * rows;
            if (rows == 128) {
              tma_load_2d_pair(b_tile(stage, h), &maps.Whalf, kb * kBK, row0, map_to_cta(full_bar(stage), 0), pol);
            } else {  // boxes of 64 rows, then of 16
              int r = 0;
              for (; r + 64 <= rows; r += 64)
                tma_load_2d_pair(b_tile(stage, h) + r * 128, &maps.W64, kb * kBK, row0 + r,
                                 map_to_cta(full_bar(stage), 0), pol);
              for (; r < rows; r += 16)
                tma_load_2d_pair(b_tile(stage, h) + r * 128, &maps.W16, kb * kBK, row0 + r,
                                 map_to_cta(full_bar(stage), 0), pol);
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto advance = [&](int& st, uint32_t& ph) { if (++st == STAGES) { st = 0; ph ^= 1u; } };
      auto release = [&](int st) {
        umma_commit_pair_both(empty_bar(st));
      };
      auto done = [&](int h) {  // half h of the segment summed: its epilogue may start
        umma_commit_pair_both(tfull_bar(h));
      };
      for (int k = 0; k < nsegs && ok; ++k) {
        const ColSeg sg = col_seg(cw, k);
        const uint32_t idesc = umma_idesc_bf16(2 * kBM, sg.ncols / 2);
        const uint32_t use = static_cast<uint32_t>(k);
        // the MMAs of half h on stage st (k-block j of KB; j = 0 starts a fresh sum)
        auto issue = [&](int st, int h, int j) {
          const uint64_t adesc = sw128_kmajor_desc(a_tile(st));
          const uint64_t bdesc = sw128_kmajor_desc(b_tile(st, h));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_pair(tmem_base + h * 256, adesc + 2u * kk, bdesc + 2u * kk, idesc, (j | kk) != 0 ? 1u : 0u);
        };
        // Half 0 of the previous segment is drained first: the MMAs of half 0 run on the
        // stages already loaded while half 1 is still being drained; those stages' half-1
        // MMAs (same per-element order) and releases follow once it is free.
        const int pre = KB < STAGES ? KB : STAGES;
        if (!mbar_wait_cluster(tempty_bar(0), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        int st = stage;
        uint32_t ph = phase;
        for (int j = 0; j < pre; ++j) {
          if (!mbar_wait_cluster(full_bar(st), ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          if (!dense) fence_proxy_async_smem();  // CTA 0's cp.async rows: generic-proxy writes
          issue(st, 0, j);
          if (j + 1 == KB) done(0);
          advance(st, ph);
        }
        if (!ok) break;
        if (!mbar_wait_cluster(tempty_bar(1), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; j < pre; ++j) {
          issue(stage, 1, j);
          release(stage);
          if (j + 1 == KB) done(1);
          advance(stage, phase);
        }
        for (int j = pre; j < KB; ++j) {
          if (!mbar_wait_cluster(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          if (!dense) fence_proxy_async_smem();
          issue(stage, 0, j);
          if (j + 1 == KB) done(0);
          issue(stage, 1, j);
          release(stage);
          if (j + 1 == KB) done(1);
          advance(stage, phase);
        }
      }
      umma_commit_pair(map_to_cta(drain_bar, 0));
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp == kWarpRelay) {
    // ------------------------------------------------------------ relay (CTA 1)
    // Lane l takes stages l, l + STAGES, ...: waits for CTA 1's cp.async rows of the stage,
    // fences them for the async proxy and arrives on CTA 0's stage barrier.
    if (!dense && rank == 1 && lane < STAGES) {
      const int total = nsegs * KB;
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
    // Warp group g (warps 12-15: g = 0, warps 4-7: g = 1) takes the 32-column chunks g, g + 2,
    // ... of each half, TMEM lane quarter q = warp % 4. Per chunk: each lane reads its row's
    // fp32 sums from TMEM and writes them to the warp's staging area; four lanes per row read
    // them back 8 columns each, add E_0 (loaded two chunks ahead), scale, round and store,
    // so every global access covers 8 rows x 64 contiguous bytes. Every warp waits for and
    // frees both halves of every segment, also where it has no columns in one.
    const int q = warp & 3;
    const int g = warp < kWarpEpi0 ? 1 : 0;
    const uint32_t stg = sbase + L::kEpiOffset + static_cast<uint32_t>(g * 4 + q) * L::kEpiWarpBytes;
    const int rsub = lane >> 2, u2 = lane & 3;
    const uint32_t row_w = stg + static_cast<uint32_t>(lane) * 128u;
    const uint32_t rd_lo = stg + static_cast<uint32_t>(rsub) * 128u + (static_cast<uint32_t>((2 * u2) ^ rsub) << 4);
    const uint32_t rd_hi = stg + static_cast<uint32_t>(rsub) * 128u + (static_cast<uint32_t>((2 * u2 + 1) ^ rsub) << 4);
    const uint32_t tempty_remote0 = map_to_cta(tempty_bar(0), 0);
    const uint32_t tempty_remote1 = map_to_cta(tempty_bar(1), 0);
    for (int k = 0; k < nsegs; ++k) {
      const ColSeg sg = col_seg(cw, k);
      const int hw = sg.ncols / 2;             // columns per half
      const int nc = (hw / 32 - g + 1) / 2;    // this warp's chunks per half (at most 4)
      const uint32_t use = static_cast<uint32_t>(k);
      const int64_t row0 = static_cast<int64_t>(sg.m_blk) * (2 * kBM) + rank * kBM + q * 32;
      const uint4* e0r[4];
      uint4* dst0 = reinterpret_cast<uint4*>(p.out + (row0 + rsub) * p.D + sg.col0 + u2 * 8);
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
        const uint16_t* row_e0 = p.E0 + static_cast<int64_t>(t) * p.D + sg.col0;
        e0r[i] = reinterpret_cast<const uint4*>(row_e0 + u2 * 8);
        // the row's E_0 columns toward L2 while the main loop runs: lane u2 takes 128-byte
        // line 2g + (u2 & 1) of half u2 / 2 (lines 0-1 by group 0, 2-3 by group 1)
        const int line = 2 * g + (u2 & 1);
        if (valid[i] && line * 64 < hw) prefetch_l2(row_e0 + (u2 >> 1) * hw + line * 64);
      }
      bool alive = true;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        bool got = false;
        if (lane == 0) got = mbar_wait_cluster(tfull_bar(h), use & 1u, abort_flag, p.status);
        if (!__shfl_sync(0xffffffffu, got, 0)) { alive = false; break; }
        tc_fence_after();
        // this warp's chunk c of the half: columns ocol(c) from col0, TMEM columns tcol(c)
        auto ocol = [&](int c) { return h * hw + (2 * c + g) * 32; };
        auto tcol = [&](int c) { return h * 256 + (2 * c + g) * 32; };
        uint4 e[4][4];  // E_0 of chunk c, row i: loaded two chunks ahead
#pragma unroll
        for (int c = 0; c < 2; ++c)
          if (c < nc)
#pragma unroll
            for (int i = 0; i < 4; ++i) e[c][i] = valid[i] ? __ldg(e0r[i] + ocol(c) / 8) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < nc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(tcol(c)), v);
            if (c + 2 < nc) {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                e[c + 2][i] = valid[i] ? __ldg(e0r[i] + ocol(c + 2) / 8) : make_uint4(0, 0, 0, 0);
            }
            tmem_wait_ld();
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
                const uint32_t ew[4] = {e[c][i].x, e[c][i].y, e[c][i].z, e[c][i].w};
                uint32_t o[4];
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                  const float x0 = (a[2 * hh] + bf16_bits_to_float(ew[hh] & 0xFFFFu)) * p.scale;
                  const float x1 = (a[2 * hh + 1] + bf16_bits_to_float(ew[hh] >> 16)) * p.scale;
                  o[hh] = pack_bf16x2(x0, x1);
                }
                dst0[static_cast<int64_t>(i) * p.D + ocol(c) / 8] = make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
            __syncwarp();  // the staging area is rewritten by the next chunk
          }
        }
        tc_fence_before();  // this warp's last read of half h
        if (rank == 0) {
          mbar_arrive_relaxed(tempty_bar(h));
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive_remote_relaxed(h ? tempty_remote1 : tempty_remote0);
        }
      }
      if (!alive) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrive or pair MMA is outstanding past this point
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512u);
  }
}

}  // namespace ngram
