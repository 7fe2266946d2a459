// Fused sub-row gather + projection + epilogue on the sm_100a tensor cores.
//
// Computes, for a tile of 128 tokens x BN outputs (Eq. 3 of "Scaling Embeddings
// Outperforms Scaling Experts in Language Models", section 2):
//   out[i][o] = ( E_0[t_i][o] + sum_s sum_c W_stacked[o][s*d + c] * E_s[idx[i][s]][c] ) / (S + 1)
// The contraction G * W_stacked^T (G[i] = concat_s E_s[idx[i][s]]) runs on tcgen05.mma
// (kind::f16, bf16 in, fp32 accumulate in TMEM). A k-block of 64 columns always lies
// inside one sub-table (d % 64 == 0), so each A tile row is one 128-byte slice of one
// gathered sub-table row: A tiles are gathered straight from HBM/L2 into shared memory
// in the 128-byte-swizzled K-major layout, and G never exists in global memory.
//
// Gathering 128-byte row slices is the expensive part: per SM, a TMA tile::gather4
// (four rows) and the load/store units each sustain only a fraction of the rate the
// tensor core consumes. So the 128 rows of each A tile are split: the first `tma_rows`
// rows arrive by TMA gather4, the rest by 16-byte cp.async, and both engines run in
// parallel. cp.async writes through the generic proxy; their completion is tracked by
// the stage's mbarrier (cp.async.mbarrier.arrive.noinc), and the MMA thread issues a
// generic->async proxy fence after observing the barrier and before its tcgen05.mma.
//
// Persistent kernel, one CTA per SM, warp-specialised (16 warps):
//   warps 0-7   A producers (256 threads): every thread copies its share of the cp.async
//               rows (thread t: 16-byte chunk t % 8 of rows tma_rows + t/8 + 32 j) and
//               arrives; tma_rows/4 lanes spread over the 8 warps each issue one gather4
//               per stage; thread 0 posts the TMA byte count.
//   warp 8      W producer: one lane issues 2-D TMA loads of W_stacked tiles.
//   warp 9      TMEM allocator; one lane issues the MMAs and commits.
//   warps 12-15 epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4) ..+31), + E_0 row slice, * 1/(S+1), bf16 RNE, store.
// Each tile walks its k-blocks starting at a tile-dependent rotation, so CTAs that share
// a W column block (or an A row block) do not read the same lines at the same time.
// Shared memory holds two rings with their own barriers: AST stages of gathered A rows and
// WST stages of W tiles. A rows come from random table rows (often HBM misses, the longest
// latency on the path) and W tiles from L2, so the A ring is the deeper one: decoupling the
// rings lets more A bytes be in flight than a shared (A, W) stage would. Where the A ring is
// at least as deep as the W ring, the two still share one handshake per k-block (the W tile
// completes on the A stage's full barrier; the A stage's empty barrier frees the W stage
// WST k-blocks later): each barrier wait and tcgen05.commit of the MMA thread costs tensor-
// pipe time. TMEM holds two BN-column fp32 accumulators so the epilogue of one tile overlaps
// the main loop of the next.
// Every wait is bounded (see mbar_wait); on a timeout all roles stop, drain what they
// have in flight, free TMEM and return with NGRAM_STATUS_TIMEOUT set.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace ngram {

constexpr int kBM = 128;  // tokens per tile (UMMA M, TMEM lanes)
constexpr int kBK = 64;   // bf16 columns per k-block = one 128-byte swizzle row
constexpr int kProjThreads = 512;
constexpr int kAWarps = 8;
constexpr int kAThreads = kAWarps * 32;
constexpr int kWarpB = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpEpi0 = 12;

// A decode step fused into the one-CTA projection (ngram_embed_fwd_step in one launch): the
// otherwise idle warps 10 and 11 of every CTA commit and hash a share of the sequences
// (commit_hash_warp_fast, section 4.2 N-gram Cache, Eq. 2) into the index buffer, and the
// gather warps start once the count of sequences done reaches num_seqs. The launch is
// cooperative, so every CTA is resident and the wait ends; it is bounded all the same.
struct StepHash {
  int on;
  CacheParams c;
  HashParams h;
  int* ready;   // sequences hashed so far (zero between launches)
  int* passed;  // CTAs past the wait (the last re-arms both counts)
};

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
  int tma_rows;           // rows of each A tile gathered by TMA (multiple of 32, 0..128)
  float scale;
  int* status;
  // stream-K (one-CTA kernel): per-tile arrival counters (zero between launches) and
  // two fp32 partial slots of 128 x BN per CTA
  int stream_k;
  int* sk_counters;
  float* sk_partials;
  // if set, the token count is min(*T_dev, T), read by the kernel (a count produced on the
  // device, e.g. the cache misses of a draft-phase call); num_m_blocks then covers T
  const int32_t* T_dev;
  // CTA-pair kernel: 1 = A tiles are dense 2-D TMA boxes of an already gathered G [T x D]
  // (maps.A), not rows gathered from the sub-tables
  int dense_a;
  StepHash sh;  // one-CTA kernel: the decode step's commit and hashing, when sh.on
};

__device__ __forceinline__ int32_t ld_cg_b32(const int32_t* p) {
  int32_t v;
  asm volatile("ld.global.cg.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

struct ProjMaps {
  CUtensorMap W;            // W_stacked, box {64, BN}, 128-byte swizzle
  CUtensorMap Whalf;        // W_stacked, box {64, BN/2} (CTA-pair kernel: each CTA loads half)
  CUtensorMap E[kMaxS];     // sub-table s, box {64, 1}, 128-byte swizzle (gather4)
  CUtensorMap Out;          // out [T x D], box {64, 32}, 128-byte swizzle (epilogue TMA stores)
  CUtensorMap A;            // gathered G [T x D], box {64, 128}, 128-byte swizzle (dense-A pair form)
  CUtensorMap W16;          // W_stacked, box {64, 16} (column-range pair form: partial halves)
  CUtensorMap W64;          // W_stacked, box {64, 64} (column-range pair form: partial halves)
};

// Shared memory (224 KB): A stages of 16 KB, W stages of BN x 128 B and the epilogue's
// 128 x BN bf16 tile. N = 256: A + W = 2 + 4, 4 + 3 or 6 + 2 stages; N = 128: 6 + 6, 8 + 4
// or 10 + 2. Defaults:
constexpr int kDefaultAStages256 = 4;
constexpr int kDefaultAStages128 = 8;

template <int BN, int AST, int WST>
struct ProjSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kWOffset = AST * kABytes;  // A ring, then the W ring,
  static constexpr int kEOffset = kWOffset + WST * kBBytes;  // then the epilogue's tile
  static constexpr int kEBytes = kBM * BN * 2;  // E_0 slice in, bf16 output out (BN/64 boxes of 128 x 64)
  static constexpr int kBarOffset = kEOffset + kEBytes;
  static constexpr int kNumBars = 2 * AST + 2 * WST + 5 + 4;  // + one per epilogue warp (end fix-up)
  static constexpr int kBytes = kBarOffset + kNumBars * 8 + 16;
  static constexpr int kLaunchBytes = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kTmemCols = 2 * BN;
  // the last stream-K fix-up stages one partial region per epilogue warp in the rings
  static_assert(4 * BN * 128 <= kEOffset, "rings smaller than four partial regions");
};

__device__ __forceinline__ uint32_t clamp_row(int32_t r, uint32_t V, int* status) {
  if (static_cast<uint32_t>(r) >= V) {
    set_status(status, NGRAM_STATUS_BAD_TOKEN);
    return 0;
  }
  return static_cast<uint32_t>(r);
}

// First k-block of a tile: a rotation that differs between tiles running side by side.
__device__ __forceinline__ int k_rotation(int m_blk, int n_blk, int KB) { return (m_blk * 5 + n_blk * 3) % KB; }

// ---- work lists (one-CTA kernel: a worker is a CTA; pair kernel: a CTA pair) ------------
// Data-parallel: worker c takes whole tiles c, c + grid, ... Stream-K: the tiles' k-positions
// form U = tiles * KB units in tile-major order and worker c takes units [c*U/grid,
// (c+1)*U/grid); a tile whose units straddle workers is computed in pieces ("segments")
// whose fp32 partial sums are added by the last piece to finish. Producers walk a worker's
// sequence run by run (a run: consecutive k-blocks of one segment that use one sub-table)
// and load the row indices of the next run while the current one is being copied.
struct WorkPlan {
  int num_tiles, KB, grid;
  int sk;          // 1: stream-K
  int64_t u_end;   // stream-K: end of this CTA's units
};

struct Seg {
  int tile;        // >= num_tiles: past the end
  int i0, i1;      // positions [i0, i1) of the tile's rotated k-block sequence
  int64_t u_next;  // stream-K: first unit after this segment
};

__device__ __forceinline__ int64_t sk_first_unit(int64_t U, int grid, int cta) { return (int64_t(cta) * U) / grid; }
// The CTA whose units contain unit u.
__device__ __forceinline__ int sk_cta_of(int64_t u, int64_t U, int grid) {
  return static_cast<int>(((u + 1) * grid + U - 1) / U) - 1;
}

__device__ __forceinline__ Seg seg_at_unit(const WorkPlan& w, int64_t u) {
  Seg g;
  if (u >= w.u_end) {
    g.tile = w.num_tiles;
    g.i0 = g.i1 = 0;
    g.u_next = u;
    return g;
  }
  g.tile = static_cast<int>(u / w.KB);
  g.i0 = static_cast<int>(u - static_cast<int64_t>(g.tile) * w.KB);
  const int64_t left = w.u_end - u;
  g.i1 = left < w.KB - g.i0 ? g.i0 + static_cast<int>(left) : w.KB;
  g.u_next = u + (g.i1 - g.i0);
  return g;
}

__device__ __forceinline__ Seg seg_first(const WorkPlan& w, int cta) {
  if (w.sk) return seg_at_unit(w, sk_first_unit(static_cast<int64_t>(w.num_tiles) * w.KB, w.grid, cta));
  Seg g;
  g.tile = cta;
  g.i0 = 0;
  g.i1 = w.KB;
  g.u_next = 0;
  return g;
}

__device__ __forceinline__ Seg seg_next(const WorkPlan& w, const Seg& g) {
  if (w.sk) return seg_at_unit(w, g.u_next);
  Seg n;
  n.tile = g.tile + w.grid;
  n.i0 = 0;
  n.i1 = w.KB;
  n.u_next = 0;
  return n;
}

// A run of k-positions of one segment that use one sub-table.
struct SRun {
  Seg g;
  int i, s, c_first, len;
};

__device__ __forceinline__ SRun srun_at(const Seg& g, int i, int num_n_blocks, int KB, int kb_per_sub) {
  SRun r;
  r.g = g;
  r.i = i;
  int kb = i + k_rotation(g.tile / num_n_blocks, g.tile % num_n_blocks, KB);
  if (kb >= KB) kb -= KB;
  r.s = kb / kb_per_sub;
  r.c_first = kb - r.s * kb_per_sub;
  const int rem = kb_per_sub - r.c_first;
  r.len = rem < g.i1 - i ? rem : g.i1 - i;
  return r;
}

__device__ __forceinline__ SRun srun_next(const WorkPlan& w, const SRun& r, int num_n_blocks, int kb_per_sub) {
  const int i = r.i + r.len;
  if (i >= r.g.i1) {
    const Seg g = seg_next(w, r.g);
    return srun_at(g, g.i0, num_n_blocks, w.KB, kb_per_sub);
  }
  return srun_at(r.g, i, num_n_blocks, w.KB, kb_per_sub);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// A load issued where it stands in the program (volatile asm keeps its place among the
// producer's other asm), consumed one run later.
__device__ __forceinline__ int32_t ld_idx_early(const int32_t* p) {
  int32_t v;
  asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued before has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int BN, int AST, int WST>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_sm100_kernel(const __grid_constant__ ProjMaps maps, const __grid_constant__ ProjParams p) {
  using L = ProjSmem<BN, AST, WST>;
  // One stage handshake per k-block for both rings: the W tile of k-block c lands on the A
  // stage's full barrier, and the W producer reuses a W stage once the A stage barrier says
  // that k-block c - WST was consumed (unambiguous while AST >= WST).
  constexpr bool kJoint = AST >= WST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOffset;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };                   // A ring
  auto empty_bar = [&](int s) { return bar0 + 8u * (AST + s); };
  auto wfull_bar = [&](int s) { return bar0 + 8u * (2 * AST + s); };      // W ring
  auto wempty_bar = [&](int s) { return bar0 + 8u * (2 * AST + WST + s); };
  constexpr int kT0 = 2 * AST + 2 * WST;
  auto tfull_bar = [&](int a) { return bar0 + 8u * (kT0 + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (kT0 + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (kT0 + 4);
  auto fix_bar = [&](int q) { return bar0 + 8u * (kT0 + 5 + q); };  // epilogue warp q's last fix-up
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOffset + L::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto a_tile = [&](int s) { return sbase + s * L::kABytes; };
  auto b_tile = [&](int s) { return sbase + L::kWOffset + s * L::kBBytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < AST; ++s) {
      // every A thread (cp.async completion) and thread 0's TMA byte count
      mbar_init(full_bar(s), static_cast<uint32_t>(kAThreads) + 1u + (kJoint ? 1u : 0u));
      mbar_init(empty_bar(s), 1u);  // one tcgen05.commit
    }
    for (int s = 0; s < WST; ++s) {
      mbar_init(wfull_bar(s), 1u);   // the W producer's TMA byte count
      mbar_init(wempty_bar(s), 1u);  // one tcgen05.commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1u);
      mbar_init(tempty_bar(a), 128u);  // every epilogue thread
    }
    mbar_init(drain_bar, 1u);
    for (int q = 0; q < 4; ++q) mbar_init(fix_bar(q), 1u);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpB && lane == 0) tma_prefetch_desc(&maps.W);
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();  // nothing above touched global memory

  const int64_t T = p.T_dev ? (*p.T_dev < p.T ? *p.T_dev : p.T) : p.T;
  const int num_tiles = static_cast<int>((T + kBM - 1) / kBM) * p.num_n_blocks;
  const int KB = p.num_k_blocks;
  const int kb_per_sub = p.d / kBK;
  WorkPlan wp;
  wp.num_tiles = num_tiles;
  wp.KB = KB;
  // stream-K partitions the units over at most as many CTAs as there are units (the count
  // may be known only here, on the device); CTAs past that hold none
  const int64_t units_total = static_cast<int64_t>(num_tiles) * KB;
  wp.grid = (p.stream_k && units_total < gridDim.x) ? static_cast<int>(units_total) : static_cast<int>(gridDim.x);
  wp.sk = p.stream_k;
  wp.u_end = p.stream_k ? sk_first_unit(static_cast<int64_t>(num_tiles) * KB, wp.grid, blockIdx.x + 1) : 0;

  if (warp < kAWarps) {
    // ------------------------------------------------------------ A producers
    const int t = threadIdx.x;                 // 0..255
    const int chunk = t & 7;
    const int rsub = t >> 3;                   // 0..31
    const int n_cp = (kBM - p.tma_rows) >> 5;  // cp.async rows per thread: tma_rows + rsub + 32 j
    const uint32_t swz = static_cast<uint32_t>((chunk ^ (rsub & 7)) << 4);
    // TMA issuers: lanes 0 .. tma_rows/32 - 1 of every producer warp, 4 rows each.
    const int lanes_tma = p.tma_rows >> 5;
    const bool tma_issuer = lane < lanes_tma;
    const int issuer = warp * lanes_tma + lane;  // rows 4*issuer .. +3
    const uint32_t tma_bytes = static_cast<uint32_t>(p.tma_rows) * 128u;
    const uint64_t pol = l2_policy_evict_normal();
    // A fused decode step: the indices are written during this launch (by warps 10-11 of
    // every CTA): wait until all sequences are done, then read them coherently.
    const bool fused = p.sh.on != 0;
    if (fused) {
      int go = 1;
      if (t == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(p.sh.ready) < p.sh.h.num_seqs) {
          if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
            set_status(p.status, NGRAM_STATUS_TIMEOUT);
            *abort_flag = 1;
            go = 0;
            break;
          }
          __nanosleep(64);
        }
        __threadfence();
        if (atomicAdd(p.sh.passed, 1) == static_cast<int>(gridDim.x) - 1) {  // the last CTA re-arms
          *p.sh.ready = 0;
          *p.sh.passed = 0;
        }
        *reinterpret_cast<volatile int*>(tmem_slot + 2) = go;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");  // the gather warps
    }
    const bool go = !fused || *reinterpret_cast<volatile int*>(tmem_slot + 2) != 0;
    auto ld_idx = [&](const int32_t* q) { return fused ? ld_cg_b32(q) : ld_idx_early(q); };
    // raw row indices of the current and the next run: cp.async rows, then TMA rows
    int32_t raw[8], nraw[8];
    auto load_raw = [&](const SRun& r, int32_t (&dst)[8]) {
      const int64_t row_base = static_cast<int64_t>(r.g.tile / p.num_n_blocks) * kBM;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t g1 = row_base + p.tma_rows + rsub + 32 * j;
        dst[j] = (j < n_cp && g1 < T) ? ld_idx(p.idx + g1 * p.S + r.s) : 0;
        const int64_t g2 = row_base + issuer * 4 + j;
        dst[4 + j] = (tma_issuer && g2 < T) ? ld_idx(p.idx + g2 * p.S + r.s) : 0;
      }
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = go;
    const Seg g0 = seg_first(wp, blockIdx.x);
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
        src[j] = p.E[cur.s] + static_cast<int64_t>(clamp_row(raw[j], V, p.status)) * p.d + chunk * 8;
        r4[j] = static_cast<int32_t>(clamp_row(raw[4 + j], V, p.status));
      }
      for (int q = 0; q < cur.len; ++q) {
        const int c0 = (cur.c_first + q) * kBK;
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
        const uint32_t a = a_tile(stage);
        if (t == 0) mbar_arrive_expect_tx(full_bar(stage), tma_bytes);
        if (tma_issuer)
          tma_gather4(a + issuer * 512, &maps.E[cur.s], c0, r4[0], r4[1], r4[2], r4[3], full_bar(stage), pol);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < n_cp) cp_async_16(a + (p.tma_rows + rsub + 32 * j) * 128 + swz, src[j] + c0);
        cp_async_arrive_noinc(full_bar(stage));
        if (++stage == AST) { stage = 0; phase ^= 1u; }
      }
      cur = nxt;
#pragma unroll
      for (int j = 0; j < 8; ++j) raw[j] = nraw[j];
      nxt = srun_next(wp, nxt, p.num_n_blocks, kb_per_sub);
      if (nxt.g.tile < num_tiles) load_raw(nxt, nraw);
    }
    cp_async_wait_all();
    if (!ok) {
      // Aborting: give the TMA gathers still in flight time to land (bounded) before exit.
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 1000ull * 1000ull) __nanosleep(1000);
    }
  } else if (warp == kWarpB) {
    // ------------------------------------------------------------ W producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int c = 0;  // k-blocks produced so far
      bool ok = true;
      for (Seg g = seg_first(wp, blockIdx.x); g.tile < num_tiles && ok; g = seg_next(wp, g)) {
        const int n_blk = g.tile % p.num_n_blocks;
        const int rot = k_rotation(g.tile / p.num_n_blocks, n_blk, KB);
        for (int i = g.i0; i < g.i1; ++i) {
          int kb = i + rot;
          if (kb >= KB) kb -= KB;
          if constexpr (kJoint) {
            if (c >= WST) {
              const int j = c - WST;
              if (!mbar_wait(empty_bar(j % AST), static_cast<uint32_t>((j / AST) & 1), abort_flag, p.status)) { ok = false; break; }
            }
            mbar_arrive_expect_tx(full_bar(c % AST), L::kBBytes);
            tma_load_2d(b_tile(stage), &maps.W, kb * kBK, n_blk * BN, full_bar(c % AST), pol);
            ++c;
          } else {
            if (!mbar_wait(wempty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
            mbar_arrive_expect_tx(wfull_bar(stage), L::kBBytes);
            tma_load_2d(b_tile(stage), &maps.W, kb * kBK, n_blk * BN, wfull_bar(stage), pol);
          }
          if (++stage == WST) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, BN);
      int stage = 0, wstage = 0;
      uint32_t phase = 0, wphase = 0;
      bool ok = true;
      int local = 0;
      for (Seg g = seg_first(wp, blockIdx.x); g.tile < num_tiles && ok; g = seg_next(wp, g), ++local) {
        const int acc = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int i = g.i0; i < g.i1; ++i) {
          if (!kJoint && !mbar_wait(wfull_bar(wstage), wphase, abort_flag, p.status)) { ok = false; break; }
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          fence_proxy_async_smem();  // the stage's cp.async rows were written by the generic proxy
          const uint64_t adesc = sw128_kmajor_desc(a_tile(stage));
          const uint64_t bdesc = sw128_kmajor_desc(b_tile(wstage));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // K = 16 per instruction: +32 B = +2 in the address field
            umma_bf16(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (i > g.i0 || k != 0) ? 1u : 0u);
          umma_commit(empty_bar(stage));
          if (!kJoint) umma_commit(wempty_bar(wstage));
          if (++stage == AST) { stage = 0; phase ^= 1u; }
          if (++wstage == WST) { wstage = 0; wphase ^= 1u; }
        }
        if (ok) umma_commit(tfull_bar(acc));
      }
      // Everything issued must complete before TMEM is released.
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, 100ull * 1000 * 1000);
    }
  } else if (warp < kWarpEpi0) {
    // ------------------------------------------------------------ warps 10-11: a fused
    // decode step's commit and hashing, sequences blockIdx.x * 2 + (warp - 10), + 2 * grid
    if (p.sh.on) {
      int done = 0;
      for (int32_t b = static_cast<int32_t>(blockIdx.x) * 2 + (warp - 10); b < p.sh.h.num_seqs;
           b += 2 * static_cast<int32_t>(gridDim.x)) {
        if (!commit_hash_warp_fast(p.sh.c, p.sh.h, b, lane)) commit_hash_warp(p.sh.c, p.sh.h, b, lane);
        ++done;
      }
      __syncwarp();
      if (lane == 0 && done) {
        __threadfence();
        atomicAdd(p.sh.ready, done);
      }
    }
  } else if (warp >= kWarpEpi0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int row_in_tile = q * 32 + lane;  // == TMEM lane
    const uint32_t stage_q = sbase + L::kEOffset + q * 4096;  // this warp's rows of box 0
    const int64_t U = static_cast<int64_t>(num_tiles) * KB;
    int local = 0;
    for (Seg g = seg_first(wp, blockIdx.x); g.tile < num_tiles; g = seg_next(wp, g), ++local) {
      const int tile = g.tile;
      const int m_blk = tile / p.num_n_blocks;
      const int n_blk = tile % p.num_n_blocks;
      const int acc = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      const bool whole = g.i0 == 0 && g.i1 == KB;
      const int64_t gr = static_cast<int64_t>(m_blk) * kBM + row_in_tile;
      const bool valid = gr < T;
      uint32_t t = 0;
      if (valid) {
        const int32_t tok = p.tokens[gr];
        t = (tok >= 0 && static_cast<uint32_t>(tok) < p.V0) ? static_cast<uint32_t>(tok) : 0u;
      }
      if (!whole && valid) {
        // A stream-K piece may be the one that finishes the tile: its rows' E_0 slice toward
        // L2 while the piece's main loop runs (the fix-up copies it in only once it knows).
        const uint16_t* e0row = p.E0 + static_cast<int64_t>(t) * p.D + n_blk * BN;
#pragma unroll
        for (int l = 0; l < BN / 64; ++l) prefetch_l2(e0row + l * 64);
      }
      if (whole) {
        // Stage this row's E_0 slice now, a whole main loop ahead of its use: once the
        // previous tile's TMA stores have read the rows, cp.async them into the tile buffer
        // (box b holds columns 64b..64b+63; 16-byte chunk c of row r sits at c ^ (r % 8)).
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        if (valid) {
          const uint16_t* e0row = p.E0 + static_cast<int64_t>(t) * p.D + n_blk * BN;
#pragma unroll 8
          for (int c = 0; c < BN / 8; ++c)
            cp_async_16(stage_q + (c >> 3) * 16384 + lane * 128 + (((c & 7) ^ (lane & 7)) << 4), e0row + c * 8);
        }
      }

      bool got = false;
      if (lane == 0) got = mbar_wait(tfull_bar(acc), use & 1u, abort_flag, p.status);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;  // warp-uniform: tcgen05.ld is .aligned
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if (whole) {
        cp_async_wait_all();  // this lane's E_0 row
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c * 32, v);
          tmem_wait_ld();
          if (c + 1 == BN / 32) {
            tc_fence_before();
            mbar_arrive_relaxed(tempty_bar(acc));  // accumulator fully read: MMA may reuse it
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) {  // columns 32c + 8w .. +7: chunk (4c + w) % 8 of box c / 2
            const uint32_t sa = stage_q + (c >> 1) * 16384 + lane * 128 + (((((c & 1) << 2) | w) ^ (lane & 7)) << 4);
            const uint4 e = ld_shared_v4(sa);
            const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int col = w * 8 + h * 2;
              const float x0 = (__uint_as_float(v[col]) + bf16_bits_to_float(ew[h] & 0xFFFFu)) * p.scale;
              const float x1 = (__uint_as_float(v[col + 1]) + bf16_bits_to_float(ew[h] >> 16)) * p.scale;
              o[h] = pack_bf16x2(x0, x1);
            }
            st_shared_v4(sa, make_uint4(o[0], o[1], o[2], o[3]));
          }
        }
        // The warp's 32 output rows go out as BN/64 TMA box stores (rows past T are clipped;
        // a box that starts past T is not issued).
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && static_cast<int64_t>(m_blk) * kBM + q * 32 < T) {
#pragma unroll
          for (int b = 0; b < BN / 64; ++b)
            tma_store_2d(&maps.Out, stage_q + b * 16384, n_blk * BN + b * 64, m_blk * kBM + q * 32);
          bulk_commit_group();
        }
      } else {
        // Stream-K piece of a tile. Per (tile, row quarter) an arrival counter counts the
        // pieces published so far. The warp whose piece completes the tile sums it: its own
        // piece straight from TMEM, every other piece from its owner's partial slot, then
        // E_0 and the scale, and stores the rows as a whole tile does. A warp that finds all
        // other pieces already counted skips publishing its own. Nobody waits for anybody.
        const int64_t u_tile = static_cast<int64_t>(tile) * KB;
        const int c_lo = sk_cta_of(u_tile, U, wp.grid), c_hi = sk_cta_of(u_tile + KB - 1, U, wp.grid);
        const int others = c_hi - c_lo;  // pieces of the tile besides this one
        int* cnt = p.sk_counters + tile * 4 + q;
        int fin = 0;
        if (lane == 0) fin = ld_acquire_gpu(cnt) == others;
        fin = __shfl_sync(0xffffffffu, fin, 0);
        if (!fin) {
          // slot 0: the piece that starts this CTA's unit range; slot 1: the one that ends it
          const int slot = (u_tile + g.i0 == sk_first_unit(U, wp.grid, blockIdx.x)) ? 0 : 1;
          // a slot holds 4 warp regions of 32 rows x BN columns (BN * 128 contiguous bytes
          // each), column group major within a region: a warp's store is 512 contiguous bytes
          float4* mine = reinterpret_cast<float4*>(p.sk_partials) +
                         (static_cast<size_t>(blockIdx.x) * 2 + slot) * (kBM * BN / 4) + q * (BN / 4) * 32 + lane;
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int w = 0; w < 8; ++w)
              mine[(c * 8 + w) * 32] = make_float4(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1]),
                                                   __uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3]));
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) fin = atomicAdd(cnt, 1) == others;
          fin = __shfl_sync(0xffffffffu, fin, 0);
          if (fin) __threadfence();
        }
        if (fin) {
          // As for a whole tile: the rows' E_0 slice into this warp's staging rows (the
          // previous TMA stores have read them), the finished sums written back there in
          // bf16, and the rows leave by TMA box stores (rows past T clipped).
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
          if (valid) {
            const uint16_t* e0row = p.E0 + static_cast<int64_t>(t) * p.D + n_blk * BN;
#pragma unroll 8
            for (int c = 0; c < BN / 8; ++c)
              cp_async_16(stage_q + (c >> 3) * 16384 + lane * 128 + (((c & 7) ^ (lane & 7)) << 4), e0row + c * 8);
          }
          // The CTA's last segment with one other piece: every stage has been consumed and
          // none will be loaded again, so the rings are free, and the other piece's region
          // for this warp comes in as one bulk copy into ring bytes [q * BN * 128, +BN * 128)
          // instead of BN / 32 rounds of dependent loads at the very end of the launch.
          const int self = static_cast<int>(blockIdx.x);
          const bool staged = others == 1 && seg_next(wp, g).tile >= num_tiles;
          const uint32_t ring_q = sbase + static_cast<uint32_t>(q * BN * 128);
          auto region = [&](int cc) {  // this warp's region of CTA cc's piece of the tile
            const int sl = (sk_first_unit(U, wp.grid, cc) >= u_tile) ? 0 : 1;
            return reinterpret_cast<const float4*>(p.sk_partials) +
                   (static_cast<size_t>(cc) * 2 + sl) * (kBM * BN / 4) + q * (BN / 4) * 32;
          };
          if (staged) {
            if (lane == 0) {
              fence_proxy_async_global();  // the acquired partial, read by the async proxy
              mbar_arrive_expect_tx(fix_bar(q), BN * 128);
              bulk_load_g2s(ring_q, region(c_lo == self ? c_hi : c_lo), BN * 128, fix_bar(q));
              mbar_wait(fix_bar(q), 0, abort_flag, p.status);  // a timeout sets the status word
            }
            __syncwarp();
          }
          cp_async_wait_all();  // this lane's E_0 row
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            // Pieces are added in CTA order whoever finishes, so the bits do not depend on
            // arrival order: the pieces before this CTA's, its own (TMEM), those after.
            float sum[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) sum[k] = 0.f;
            auto add_piece = [&](int cc) {
              float4 x[8];
              if (staged) {
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                  const uint4 r = ld_shared_v4(ring_q + static_cast<uint32_t>(((c * 8 + w) * 32 + lane) * 16));
                  x[w] = make_float4(__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z), __uint_as_float(r.w));
                }
              } else {
                const float4* part = region(cc) + lane;
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = __ldcg(part + (c * 8 + w) * 32);
              }
#pragma unroll
              for (int w = 0; w < 8; ++w) {
                sum[4 * w] += x[w].x;
                sum[4 * w + 1] += x[w].y;
                sum[4 * w + 2] += x[w].z;
                sum[4 * w + 3] += x[w].w;
              }
            };
            for (int cc = c_lo; cc < self; ++cc) add_piece(cc);
            {
              uint32_t v[32];
              tmem_ld_32x32b_x32(taddr + c * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) sum[k] += __uint_as_float(v[k]);
            }
            for (int cc = self + 1; cc <= c_hi; ++cc) add_piece(cc);
#pragma unroll
            for (int w = 0; w < 4; ++w) {  // columns 32c + 8w .. +7: chunk (4c + w) % 8 of box c / 2
              const uint32_t sa = stage_q + (c >> 1) * 16384 + lane * 128 + (((((c & 1) << 2) | w) ^ (lane & 7)) << 4);
              const uint4 e = ld_shared_v4(sa);
              const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
              uint32_t o[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int col = w * 8 + h * 2;
                o[h] = pack_bf16x2((sum[col] + bf16_bits_to_float(ew[h] & 0xFFFFu)) * p.scale,
                                   (sum[col + 1] + bf16_bits_to_float(ew[h] >> 16)) * p.scale);
              }
              st_shared_v4(sa, make_uint4(o[0], o[1], o[2], o[3]));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && static_cast<int64_t>(m_blk) * kBM + q * 32 < T) {
#pragma unroll
            for (int b = 0; b < BN / 64; ++b)
              tma_store_2d(&maps.Out, stage_q + b * 16384, n_blk * BN + b * 64, m_blk * kBM + q * 32);
            bulk_commit_group();
          }
          if (lane == 0) *cnt = 0;  // the tile is done: zero again for the next launch
        }
        tc_fence_before();
        mbar_arrive_relaxed(tempty_bar(acc));  // accumulator read for the last time: MMA may reuse it
      }
    }
    cp_async_wait_all();                   // E_0 rows still landing (after an abort)
    if (lane == 0) bulk_wait_group<0>();  // output stores complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace ngram
