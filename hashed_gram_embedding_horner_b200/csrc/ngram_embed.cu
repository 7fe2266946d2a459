// libngram_embed.so — host side of the C ABI declared in include/ngram_embed.h.
//
// Plan creation validates a layer shape (section 2 of "Scaling Embeddings Outperforms
// Scaling Experts in Language Models", Eq. 3) and picks the projection kernel:
//   - bf16, D % 128 == 0, d % 64 == 0, N >= 2: the fused gather + tcgen05 kernel
//     (proj_sm100.cuh), 128 x 256 tiles (128 x 128 when D % 256 != 0);
//   - otherwise the CUDA-core kernel (simt.cuh).
// Every entry point checks its arguments on the host, launches on the caller's
// stream, and returns without synchronising.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>

#include "common.cuh"
#include "hash.cuh"
#include "proj_sm100.cuh"
#include "proj_sm100_pair.cuh"
#include "proj_sm100_cols.cuh"
#include "simt.cuh"
#include "bwd_sm100.cuh"
#include "stats.cuh"
#include "draft.cuh"
#include "decode.cuh"

using namespace ngram;

namespace {

// Workspace: [status word + padding | stream-K arrival counters | T x S indices | stream-K partials]
constexpr size_t kStatusBytes = 256;
constexpr size_t kStepCountOffset = 128;  // in the status header: the fused decode step's two counts
constexpr int kSkMaxTiles = 2048;                          // stream-K only for grids of at most this many tiles
constexpr size_t kSkCounterBytes = size_t(kSkMaxTiles) * 4 * sizeof(int32_t);  // one per (tile, row quarter)
constexpr size_t kHeadBytes = kStatusBytes + kSkCounterBytes;                   // zeroed by clear_status

enum Variant : int { kAuto = 0, kTcTmaRows = 1, kTcSplitRows = 2, kSimt = 3 };

}  // namespace

struct ngram_embed_plan {
  int64_t V0;
  int D, N, K, S, d;
  int dtype;
  int elt;  // bytes per element
  int64_t V[kMaxS];
  uint64_t barrett[kMaxS];
  int device;
  int sms;         // SMs the plan's kernels use (grids, stream-K shares, partial slots)
  int sms_device;  // SMs of the device (0 without one)
  int variant;  // resolved: kTcTmaRows, kTcSplitRows or kSimt
  int tma_rows; // tensor-core kernel: A rows per tile gathered by TMA (multiple of 32; -1 = per form)
  int bn;       // tensor-core tile width (256 or 128)
  bool tc_ok;   // the shape admits the tensor-core kernel
  // tensor-map cache (re-encoded when a table or W pointer changes)
  ProjMaps maps;
  const void* map_W = nullptr;
  const void* map_E[kMaxS] = {};
  bool maps_valid = false;
  const void* map_out = nullptr;  // the out map's pointer and row count
  int64_t map_out_T = -1;
  bool smem_attr_set[17] = {};  // per kernel instance (form, tile width, rings), on `device`
  int a_stages = 0;            // one-CTA kernel: A ring depth (0 = default for the tile width)
  int cta_pair = -1;           // kernel form: 1 CTA pairs (cta_group::2), 0 one CTA per tile, -1 automatic
  int stream_k = 0;            // one-CTA kernel schedule: 0 automatic, 1 stream-K when possible, 2 never
  bool pdl = false;            // launch as programmatic dependent launches
  float out_scale = 1.0f;      // embedding amplification factor folded into the 1/(S+1) scale
  int pair_wide = -1;          // pair form with 512-column tiles: 1 on, 0 off, -1 automatic
  int dense_a = 0;             // sub-rows gathered into G first, A by dense TMA: 1 on, 0 off
  const void* map_A = nullptr;  // the dense-A map's pointer and row count
  int64_t map_A_T = -1;
  int max_clusters[8] = {};    // co-resident CTA pairs, per kernel instance (0 = not queried)
  int pair_cols = 0;           // pair form over column ranges: 1 whenever possible, 0 off
  int fused_step = 0;          // decode step committed and hashed inside the one-CTA projection
  int bwd_pair = 1;            // backward GEMMs: 1 CTA pairs (256-column tiles), 2 pairs with 512-column
                               // tiles where possible, 0 one CTA per 128-row tile
  int bwd_streams = 1;         // backward: 1 the memory-bound kernels on an auxiliary stream, 0 all on the caller's
  cudaStream_t aux = nullptr;  // the auxiliary stream (created by the first backward call that uses it)
  cudaEvent_t aux_ev[3] = {};  // fork, G gathered, join
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t* status_ptr(void* ws) { return static_cast<int32_t*>(ws); }
int32_t* idx_ptr(void* ws) { return reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kHeadBytes); }

// Bytes every call needs: the head and the index buffer.
size_t ws_base(const ngram_embed_plan* p, int64_t T) {
  const size_t idx = static_cast<size_t>(T) * static_cast<size_t>(p->S) * sizeof(int32_t);
  return kHeadBytes + ((idx + 255) & ~size_t(255));
}
// Whether the plan's shape admits the CTA-pair form's 512-column tiles (256-column W halves).
bool wide_capable(const ngram_embed_plan* p) { return p->tc_ok && p->bn == 256 && p->D % 512 == 0; }
// Stream-K fp32 partial tiles: two slots per SM of 128 rows x the widest tile a stream-K
// schedule of the plan can split (512 columns where the 512-column pair tiles apply, else 256).
size_t sk_partial_bytes(const ngram_embed_plan* p) {
  return p->tc_ok ? size_t(2) * static_cast<size_t>(p->sms) * kBM * (wide_capable(p) ? 512 : 256) * sizeof(float) : 0;
}
// The dense-A form: the call's sub-rows gathered into G [T x D] bf16 first (a stand-alone
// gather kernel with every resident thread copying), then the CTA-pair projection reads A as
// dense TMA boxes of G. Only on request: measured on B200 at the 1280-token decode step
// (D = 4096) it took 78 us a step against 70 us for the fused one-CTA stream-K form, because
// the tensor-core kernels there are limited by the rate at which an SM's shared memory fills
// from L2 (about 55 GB/s per SM), not by the latency of the row gather, and the dense form
// moves the same A bytes plus its own copy.
size_t dense_g_bytes(const ngram_embed_plan* p, int64_t T) {
  return (static_cast<size_t>(T) * static_cast<size_t>(p->D) * 2 + 255) & ~size_t(255);
}
// The dense-A form needs 256-column W halves: tile width 256, D % 256 == 0.
bool dense_wanted(const ngram_embed_plan* p) { return p->tc_ok && p->bn == 256 && p->dense_a == 1; }
// Workspace: [head | T x S indices | stream-K partials | G (dense-A form)]
size_t dense_g_offset(const ngram_embed_plan* p, int64_t ws_T) { return ws_base(p, ws_T) + sk_partial_bytes(p); }
// Bytes that let every call of up to T tokens take its fastest schedule.
size_t ws_bytes(const ngram_embed_plan* p, int64_t T) {
  return ws_base(p, T) + sk_partial_bytes(p) + (dense_wanted(p) ? dense_g_bytes(p, T) : 0);
}

int check_launch() { return cudaGetLastError() == cudaSuccess ? NGRAM_OK : NGRAM_ERR_CUDA; }

// Every kernel launch: optionally as a programmatic dependent launch (the kernel may be
// scheduled while the previous kernel on the stream finishes; its pdl_wait() orders
// the memory), optionally in clusters of `cluster` CTAs.
template <typename... KArgs, typename... Args>
int launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, int cluster,
           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = n ? attr : nullptr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) return NGRAM_ERR_CUDA;
  return check_launch();
}

int encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer, CUtensorMapL2promotion promo) {
  auto fn = encode_fn();
  if (!fn) return NGRAM_ERR_CUDA;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NGRAM_OK : NGRAM_ERR_CUDA;
}

int refresh_maps(ngram_embed_plan* p, const void* const* E_nk, const void* W, void* out, int64_t T) {
  if (p->map_out != out || p->map_out_T != T) {
    p->map_out = nullptr;
    int rc = encode_2d(&p->maps.Out, out, p->D, static_cast<uint64_t>(T), static_cast<uint64_t>(p->D) * 2, kBK, 32,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE);
    if (rc) return rc;
    p->map_out = out;
    p->map_out_T = T;
  }
  bool same = p->maps_valid && p->map_W == W;
  for (int s = 0; same && s < p->S; ++s) same = p->map_E[s] == E_nk[s];
  if (same) return NGRAM_OK;
  p->maps_valid = false;
  int rc = encode_2d(&p->maps.W, W, p->D, p->D, static_cast<uint64_t>(p->D) * 2, kBK, p->bn,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (rc) return rc;
  rc = encode_2d(&p->maps.Whalf, W, p->D, p->D, static_cast<uint64_t>(p->D) * 2, kBK, p->bn / 2,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (rc) return rc;
  rc = encode_2d(&p->maps.W16, W, p->D, p->D, static_cast<uint64_t>(p->D) * 2, kBK, 16,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (rc) return rc;
  rc = encode_2d(&p->maps.W64, W, p->D, p->D, static_cast<uint64_t>(p->D) * 2, kBK, 64,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (rc) return rc;
  for (int s = 0; s < p->S; ++s) {
    rc = encode_2d(&p->maps.E[s], E_nk[s], p->d, p->V[s], static_cast<uint64_t>(p->d) * 2, kBK, 1,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
    if (rc) return rc;
    p->map_E[s] = E_nk[s];
  }
  p->map_W = W;
  p->maps_valid = true;
  return NGRAM_OK;
}

// Stream-K (every CTA takes an equal share of the (tile, k-block) units) instead of one
// tile per CTA per wave: when a grid of two or more waves ends in a wave that leaves many
// SMs idle. Measured on B200 at D = 2048 and 4096: a unit costs about 1.3x as much under
// stream-K (fixups, pieces that start mid-tile), and a single wave is never worth splitting.
bool use_stream_k(const ngram_embed_plan* p, const ProjParams& prm, int64_t T, size_t ws_size) {
  const int tiles = prm.num_m_blocks * prm.num_n_blocks;
  const int64_t units = static_cast<int64_t>(tiles) * prm.num_k_blocks;
  if (p->stream_k == 2 || p->sms <= 0 || tiles > kSkMaxTiles || units < p->sms) return false;
  if (ws_size < ws_base(p, T) + sk_partial_bytes(p)) return false;
  if (p->stream_k == 1) return true;
  const int waves = (tiles + p->sms - 1) / p->sms;
  return waves >= 2 && 1.3 * tiles < static_cast<double>(waves) * p->sms;
}

template <int BN, int AST, int WST>
int launch_tc_rings(ngram_embed_plan* p, const ProjParams& prm, cudaStream_t st, int key) {
  using L = ProjSmem<BN, AST, WST>;
  static_assert(L::kLaunchBytes <= 232448, "one-CTA kernel rings exceed 227 KB of shared memory");
  auto kern = proj_sm100_kernel<BN, AST, WST>;
  if (!p->smem_attr_set[key]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kLaunchBytes) != cudaSuccess)
      return NGRAM_ERR_CUDA;
    p->smem_attr_set[key] = true;
  }
  const int tiles = prm.num_m_blocks * prm.num_n_blocks;
  const int grid = (prm.stream_k || tiles > p->sms) ? p->sms : tiles;
  if (prm.sh.on) {
    // a fused decode step: its gather warps wait for the sequences every CTA hashes, so all
    // CTAs must be resident at once (one per SM)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kProjThreads);
    cfg.dynamicSmemBytes = L::kLaunchBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p->maps, prm) != cudaSuccess) return NGRAM_ERR_CUDA;
    return check_launch();
  }
  return launch(kern, dim3(grid), dim3(kProjThreads), L::kLaunchBytes, st, p->pdl, 1, p->maps, prm);
}

template <int BN>
int launch_tc(ngram_embed_plan* p, const ProjParams& prm, cudaStream_t st) {
  if (BN == 256) {
    switch (p->a_stages ? p->a_stages : kDefaultAStages256) {
      case 2: return launch_tc_rings<256, 2, 4>(p, prm, st, 0);
      case 6: return launch_tc_rings<256, 6, 2>(p, prm, st, 1);
      default: return launch_tc_rings<256, 4, 3>(p, prm, st, 2);
    }
  }
  switch (p->a_stages ? p->a_stages : kDefaultAStages128) {
    case 6: return launch_tc_rings<128, 6, 6>(p, prm, st, 3);
    case 10: return launch_tc_rings<128, 10, 2>(p, prm, st, 5);
    default: return launch_tc_rings<128, 8, 4>(p, prm, st, 4);
  }
}

// Stream-K for the CTA-pair kernel's 256 x 256 tiles, over the co-resident pairs (one per
// two SMs); pieces are counted per (tile, CTA, row quarter) in the workspace head, and each
// CTA has two partial slots of 128 x 256 fp32. Only when the plan asks for both the pair
// form and stream-K: at the 1280-token decode step (D = 4096) it measured 69.9 us against
// 56.2 us for the one-CTA form's stream-K, whose cp.async row gather keeps more DRAM misses
// in flight than TMA gather4.
bool use_pair_stream_k(const ngram_embed_plan* p, int64_t T, size_t ws_size, int64_t ws_T) {
  if (p->stream_k != 1 || p->cta_pair != 1 || p->sms < 2 || p->bn != 256) return false;
  const int64_t pairs = p->sms / 2;
  const int64_t tiles = (T + 2 * kBM - 1) / (2 * kBM) * (p->D / p->bn);
  const int64_t units = tiles * (p->D / kBK);
  if (tiles > kSkMaxTiles / 2 || units < pairs) return false;
  return ws_size >= ws_base(p, ws_T) + sk_partial_bytes(p);
}

// CTA-pair kernel: clusters of two CTAs, one 256 x BN tile per pair per step (WSK: the
// 512-column tiles' stream-K instance).
template <int BN, int kStg, bool WSK = false>
int launch_tc_pair_stages(ngram_embed_plan* p, ProjParams prm, int64_t T, cudaStream_t st, int key) {
  using L = PairSmem<BN, kStg>;
  static_assert(L::kLaunchBytes <= 232448, "CTA-pair kernel stages exceed 227 KB of shared memory");
  auto kern = proj_sm100_pair_kernel<BN, kStg, WSK>;
  if (!p->smem_attr_set[key]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kLaunchBytes) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess)
      return NGRAM_ERR_CUDA;
    p->smem_attr_set[key] = true;
  }
  prm.num_m_blocks = static_cast<int>((T + 2 * kBM - 1) / (2 * kBM));
  const int tiles = prm.num_m_blocks * prm.num_n_blocks;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kProjThreads);
  cfg.dynamicSmemBytes = L::kLaunchBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int& max_pairs = p->max_clusters[WSK ? 3 : (BN == 512 ? 2 : (BN == 256 ? 1 : 0))];
  if (max_pairs == 0) {
    cfg.gridDim = dim3(2 * (p->sms / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return NGRAM_ERR_CUDA;
    max_pairs = n;
  }
  // co-resident pairs, within the plan's SM count (which also sizes the stream-K slots)
  const int cap = max_pairs < p->sms / 2 ? max_pairs : p->sms / 2;
  if (cap < 1) return NGRAM_ERR_CUDA;
  const int pairs = (prm.stream_k || tiles > cap) ? cap : tiles;
  return launch(kern, dim3(2 * pairs), dim3(kProjThreads), L::kLaunchBytes, st, p->pdl, 2, p->maps, prm);
}

template <int BN>
int launch_tc_pair(ngram_embed_plan* p, const ProjParams& prm, int64_t T, cudaStream_t st) {
  if (BN == 256) return launch_tc_pair_stages<256, kPairStages256>(p, prm, T, st, 7);
  return launch_tc_pair_stages<128, kPairStages128>(p, prm, T, st, 6);
}

// The pair form's 512-column tiles (two N = 256 MMAs per A stage): needs 256-column W
// halves and D % 512 == 0. Automatic: whichever width finishes its whole waves of tiles
// sooner, a 256-column tile costing 0.57 of a 512-column one (measured on B200 at T = 32768
// and 65536: 0.54 at D = 2048, 0.61 at D = 4096), so small grids keep the narrow tiles
// that occupy more SMs. Not automatic when the token count is known only on the device (a
// draft call's misses: usually a few tiles, for which the narrow tiles keep more SMs busy).
bool use_pair_wide(const ngram_embed_plan* p, int64_t T, bool count_on_device = false) {
  if (p->bn != 256 || p->D % 512 != 0 || p->pair_wide == 0) return false;
  if (p->pair_wide == 1) return true;
  if (p->sms < 2 || count_on_device) return false;  // no device: the SM count is unknown
  const int64_t pairs = p->sms / 2;
  const int64_t wide_tiles = (T + 2 * kBM - 1) / (2 * kBM) * (p->D / 512);
  const int64_t waves_wide = (wide_tiles + pairs - 1) / pairs;
  const int64_t waves_narrow = (2 * wide_tiles + pairs - 1) / pairs;
  return static_cast<double>(waves_wide) <= 0.57 * static_cast<double>(waves_narrow);
}


// Stream-K for the pair form's 512-column tiles: only when the plan asks for both the
// 512-column tiles and stream-K (ngram_embed_plan_set_pair_wide(plan, 1) and
// ngram_embed_plan_set_stream_k(plan, 1)). Measured on B200 at the 1280-token decode step
// (D = 4096, 40 tiles for 74 pairs): 101 us a step against 71 us for the one-CTA form's
// stream-K and 72 us for whole 512-column tiles. With one 512-column accumulator per CTA a
// piece's epilogue (publishing or summing 256 KB of fp32 partials per CTA) cannot overlap
// the MMAs of the pair's next piece, and each pair runs two pieces. Needs the workspace's
// partial tiles and 16 arrival counters per tile (row quarter x column group, per CTA of
// the pair), and at least half a tile per pair.
bool use_wide_stream_k(const ngram_embed_plan* p, int64_t T, size_t ws_size, int64_t ws_T) {
  if (!wide_capable(p) || p->stream_k != 1 || p->pair_wide != 1 || p->cta_pair == 0 || p->sms < 2) return false;
  const int64_t pairs = p->sms / 2;
  const int64_t tiles = (T + 2 * kBM - 1) / (2 * kBM) * (p->D / 512);
  const int64_t units = tiles * (p->D / kBK);
  if (tiles * 16 > static_cast<int64_t>(kSkMaxTiles) * 4 || units < pairs || 2 * tiles < pairs) return false;
  return ws_size >= ws_base(p, ws_T) + sk_partial_bytes(p);
}

// Column ranges for the pair form (proj_sm100_cols.cuh): every pair computes the full K of
// a range of columns of a 256-row block, so pairs a call's tiles would leave idle share the
// work without stream-K's partial sums. Only with the token count known on the host, and only
// on request (ngram_embed_plan_set_pair_columns(plan, 1)): measured on B200 at the 1280-token
// decode step (D = 4096, 74 pairs, ranges of 256-320 columns), 61 us for the projection with
// the rows copied in the kernel and 57 us reading them from G, against 55 us for the one-CTA
// form's stream-K, whose fix-ups it avoids but whose stage rate (0.55 us per 48 KB stage) the
// pairs' stages do not reach (0.8 us).
bool use_pair_cols(const ngram_embed_plan* p, int64_t T, bool count_on_device) {
  if (!p->tc_ok || p->bn != 256 || p->sms < 2 || count_on_device || T <= 0 || p->cta_pair == 0) return false;
  return p->pair_cols == 1;
}

template <int HROWS, int STAGES>
int set_cols_smem(ngram_embed_plan* p, int key) {
  using L = ColsSmem<HROWS, STAGES>;
  static_assert(L::kLaunchBytes <= 232448, "column-range kernel stages exceed 227 KB of shared memory");
  if (!p->smem_attr_set[key]) {
    if (cudaFuncSetAttribute(proj_sm100_cols_kernel<HROWS, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::kLaunchBytes) != cudaSuccess)
      return NGRAM_ERR_CUDA;
    p->smem_attr_set[key] = true;
  }
  return NGRAM_OK;
}

// The pairs are as many as fit (one per two SMs); the ranges are cut for that count. Ranges of
// at most 320 columns (80 W rows per half and CTA) take the instance with 5 stages of 36 KB,
// wider ones the instance with 4 stages of 48 KB.
int launch_cols(ngram_embed_plan* p, const ProjParams& prm, int64_t T, cudaStream_t st) {
  int rc;
  if ((rc = set_cols_smem<128, 4>(p, 13))) return rc;
  int& max_pairs = p->max_clusters[4];
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (p->sms / 2));
    cfg.blockDim = dim3(kProjThreads);
    cfg.dynamicSmemBytes = ColsSmem<128, 4>::kLaunchBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, proj_sm100_cols_kernel<128, 4>, &cfg) != cudaSuccess || n < 1)
      return NGRAM_ERR_CUDA;
    max_pairs = n;
  }
  const int pairs = max_pairs < p->sms / 2 ? max_pairs : p->sms / 2;
  if (pairs < 1) return NGRAM_ERR_CUDA;
  const int64_t mblocks = (T + 2 * kBM - 1) / (2 * kBM);
  int widest = 0;
  for (int pr = 0; pr < pairs; ++pr) {
    const ColWork w = col_work(pr, pairs, mblocks, p->D / 64);
    for (int k = 0; k < (w.m1 - w.m0) * w.nseg; ++k) {
      const ColSeg sg = col_seg(w, k);
      if (sg.ncols > widest) widest = sg.ncols;
    }
  }
  if (widest <= 320) {
    if ((rc = set_cols_smem<80, 5>(p, 12))) return rc;
    return launch(proj_sm100_cols_kernel<80, 5>, dim3(2 * pairs), dim3(kProjThreads), ColsSmem<80, 5>::kLaunchBytes, st,
                  p->pdl, 2, p->maps, prm);
  }
  return launch(proj_sm100_cols_kernel<128, 4>, dim3(2 * pairs), dim3(kProjThreads), ColsSmem<128, 4>::kLaunchBytes, st,
                p->pdl, 2, p->maps, prm);
}

// ---- backward -------------------------------------------------------------------------
// Workspace: the head (status word, ...), then G [T x D] bf16 (the concatenated sub-rows of
// every token, the B operand of dW), then the dE0 sort buffers, each 256-byte aligned.
constexpr int kBwdStages = 4;  // x (16 KB A + BN x 128 B B)

size_t round256(size_t b) { return (b + 255) & ~size_t(255); }
// dE0's counting sort: counts [V0 + 1], order [T], sorted ids [T], block sums (int32).
size_t bwd_sort_bytes(const ngram_embed_plan* p, int64_t T) {
  return round256((static_cast<size_t>(p->V0) + 1) * 4) + 2 * round256(static_cast<size_t>(T) * 4) +
         round256((static_cast<size_t>(p->V0) + 1023) / 1024 * 4);
}
size_t bwd_g_bytes(const ngram_embed_plan* p, int64_t T) {
  return round256(static_cast<size_t>(T) * static_cast<size_t>(p->D) * 2);
}
size_t bwd_ws_bytes(const ngram_embed_plan* p, int64_t T) {
  return kHeadBytes + bwd_g_bytes(p, T) + bwd_sort_bytes(p, T);
}

// Split-K factor for a GEMM of `tiles` output tiles and KB k-blocks: the one, up to KB / 16
// k-blocks per unit, whose units best fill whole waves of the SMs (ties: fewer splits).
int choose_splits(int tiles, int KB, int sms) {
  int best = 1;
  double best_fill = -1.0;
  const int max_s = KB / 16 > 1 ? (KB / 16 < 64 ? KB / 16 : 64) : 1;
  for (int s = 1; s <= max_s; ++s) {
    const int kbps = (KB + s - 1) / s;
    const int units = tiles * ((KB + kbps - 1) / kbps);
    const int waves = (units + sms - 1) / sms;
    const double fill = static_cast<double>(units) / (static_cast<double>(waves) * sms);
    if (fill > best_fill + 0.01) {
      best_fill = fill;
      best = s;
    }
  }
  return best;
}

// A GEMM operand as it lies in memory: K-major ([rows x K], rows K elements apart) or
// MN-major ([K x rows], K rows of `rows` elements).
struct GemmOperand {
  const void* base;
  int64_t rows;  // M (A) or N (B)
  bool mn;
};

template <int BN>
int launch_dense_gemm(ngram_embed_plan* p, DenseParams prm, GemmOperand A, GemmOperand B, int64_t K, bool split,
                      cudaStream_t st) {
  using L = DenseSmem<BN, kBwdStages>;
  auto kern = dense_gemm_sm100_kernel<BN, kBwdStages>;
  const int key = BN == 256 ? 10 : 11;
  if (!p->smem_attr_set[key]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kLaunchBytes) != cudaSuccess)
      return NGRAM_ERR_CUDA;
    p->smem_attr_set[key] = true;
  }
  auto encode = [&](CUtensorMap* m, const GemmOperand& o, uint32_t box_rows) {
    return o.mn ? encode_2d(m, o.base, static_cast<uint64_t>(o.rows), static_cast<uint64_t>(K),
                            static_cast<uint64_t>(o.rows) * 2, 64, 64, CU_TENSOR_MAP_L2_PROMOTION_L2_256B)
                : encode_2d(m, o.base, static_cast<uint64_t>(K), static_cast<uint64_t>(o.rows),
                            static_cast<uint64_t>(K) * 2, kBK, box_rows, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  };
  DenseMaps maps;
  int rc = encode(&maps.A, A, kBM);
  if (rc) return rc;
  if ((rc = encode(&maps.B, B, BN))) return rc;
  prm.a_mn = A.mn ? 1 : 0;
  prm.b_mn = B.mn ? 1 : 0;
  prm.M = static_cast<int>(A.rows);
  prm.N = static_cast<int>(B.rows);
  prm.num_m_blocks = static_cast<int>((A.rows + kBM - 1) / kBM);
  prm.num_n_blocks = static_cast<int>(B.rows / BN);
  prm.num_k_blocks = static_cast<int>((K + kBK - 1) / kBK);
  const int tiles = prm.num_m_blocks * prm.num_n_blocks;
  const int sms = p->sms > 0 ? p->sms : 1;
  const int s = split ? choose_splits(tiles, prm.num_k_blocks, sms) : 1;
  prm.kb_per_split = (prm.num_k_blocks + s - 1) / s;
  prm.splits = (prm.num_k_blocks + prm.kb_per_split - 1) / prm.kb_per_split;  // every split non-empty
  const int units = tiles * prm.splits;
  const int grid = units < sms ? units : sms;
  return launch(kern, dim3(grid), dim3(kGemmThreads), L::kLaunchBytes, st, p->pdl, 1, maps, prm);
}

// CTA-pair form of the same GEMM: 256-row tiles, each CTA of a pair loading its 128 rows of A
// and half of B's BN rows per stage; units (tile, k range) strided over the co-resident pairs.
constexpr int kBwdPairKsub = 2;        // k-blocks per stage
constexpr int kBwdPairStages256 = 3;  // x 2 x (16 KB A + 16 KB B)
constexpr int kBwdPairStages128 = 4;  // x 2 x (16 KB A + 8 KB B)

template <int BN>
int launch_dense_gemm_pair(ngram_embed_plan* p, DenseParams prm, GemmOperand A, GemmOperand B, int64_t K, bool split,
                           cudaStream_t st) {
  constexpr int STAGES = BN == 256 ? kBwdPairStages256 : kBwdPairStages128;
  using L = DensePairSmem<BN, STAGES, kBwdPairKsub>;
  static_assert(L::kLaunchBytes <= 232448, "pair backward GEMM stages exceed 227 KB of shared memory");
  auto kern = dense_gemm_pair_kernel<BN, STAGES, kBwdPairKsub>;
  const int key = BN == 256 ? 14 : 15;
  if (!p->smem_attr_set[key]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kLaunchBytes) != cudaSuccess)
      return NGRAM_ERR_CUDA;
    p->smem_attr_set[key] = true;
  }
  auto encode = [&](CUtensorMap* m, const GemmOperand& o, uint32_t box_rows) {
    return o.mn ? encode_2d(m, o.base, static_cast<uint64_t>(o.rows), static_cast<uint64_t>(K),
                            static_cast<uint64_t>(o.rows) * 2, 64, 64, CU_TENSOR_MAP_L2_PROMOTION_L2_256B)
                : encode_2d(m, o.base, static_cast<uint64_t>(K), static_cast<uint64_t>(o.rows),
                            static_cast<uint64_t>(K) * 2, kBK, box_rows, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  };
  DenseMaps maps;
  int rc = encode(&maps.A, A, kBM);
  if (rc) return rc;
  if ((rc = encode(&maps.B, B, BN / 2))) return rc;
  prm.a_mn = A.mn ? 1 : 0;
  prm.b_mn = B.mn ? 1 : 0;
  prm.M = static_cast<int>(A.rows);
  prm.N = static_cast<int>(B.rows);
  prm.num_m_blocks = static_cast<int>((A.rows + 2 * kBM - 1) / (2 * kBM));
  prm.num_n_blocks = static_cast<int>(B.rows / BN);
  prm.num_k_blocks = static_cast<int>((K + kBK - 1) / kBK);
  int& max_pairs = p->max_clusters[BN == 256 ? 5 : 6];
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (p->sms / 2));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = L::kLaunchBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return NGRAM_ERR_CUDA;
    max_pairs = n;
  }
  const int pairs_avail = max_pairs < p->sms / 2 ? max_pairs : p->sms / 2;
  if (pairs_avail < 1) return NGRAM_ERR_CUDA;
  const int tiles = prm.num_m_blocks * prm.num_n_blocks;
  const int s = split ? choose_splits(tiles, prm.num_k_blocks, pairs_avail) : 1;
  prm.kb_per_split = (prm.num_k_blocks + s - 1) / s;
  prm.splits = (prm.num_k_blocks + prm.kb_per_split - 1) / prm.kb_per_split;  // every split non-empty
  const int units = tiles * prm.splits;
  const int pairs = units < pairs_avail ? units : pairs_avail;
  return launch(kern, dim3(2 * pairs), dim3(kGemmThreads), L::kLaunchBytes, st, p->pdl, 2, maps, prm);
}

// Wide pair form: 256 x 512 tiles (B.rows % 512 == 0).
constexpr int kBwdWideStages = 4;  // x (16 KB A + 32 KB B)

int launch_dense_gemm_pair_wide(ngram_embed_plan* p, DenseParams prm, GemmOperand A, GemmOperand B, int64_t K,
                                bool split, cudaStream_t st) {
  using L = DenseWideSmem<kBwdWideStages>;
  static_assert(L::kLaunchBytes <= 232448, "wide backward GEMM stages exceed 227 KB of shared memory");
  auto kern = dense_gemm_pair_wide_kernel<kBwdWideStages>;
  if (!p->smem_attr_set[16]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kLaunchBytes) != cudaSuccess)
      return NGRAM_ERR_CUDA;
    p->smem_attr_set[16] = true;
  }
  auto encode = [&](CUtensorMap* m, const GemmOperand& o) {
    return o.mn ? encode_2d(m, o.base, static_cast<uint64_t>(o.rows), static_cast<uint64_t>(K),
                            static_cast<uint64_t>(o.rows) * 2, 64, 64, CU_TENSOR_MAP_L2_PROMOTION_L2_256B)
                : encode_2d(m, o.base, static_cast<uint64_t>(K), static_cast<uint64_t>(o.rows),
                            static_cast<uint64_t>(K) * 2, kBK, kBM, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  };
  DenseMaps maps;
  int rc = encode(&maps.A, A);
  if (rc) return rc;
  if ((rc = encode(&maps.B, B))) return rc;
  prm.a_mn = A.mn ? 1 : 0;
  prm.b_mn = B.mn ? 1 : 0;
  prm.M = static_cast<int>(A.rows);
  prm.N = static_cast<int>(B.rows);
  prm.num_m_blocks = static_cast<int>((A.rows + 2 * kBM - 1) / (2 * kBM));
  prm.num_n_blocks = static_cast<int>(B.rows / 512);
  prm.num_k_blocks = static_cast<int>((K + kBK - 1) / kBK);
  int& max_pairs = p->max_clusters[7];
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (p->sms / 2));
    cfg.blockDim = dim3(kWideGemmThreads);
    cfg.dynamicSmemBytes = L::kLaunchBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return NGRAM_ERR_CUDA;
    max_pairs = n;
  }
  const int pairs_avail = max_pairs < p->sms / 2 ? max_pairs : p->sms / 2;
  if (pairs_avail < 1) return NGRAM_ERR_CUDA;
  const int tiles = prm.num_m_blocks * prm.num_n_blocks;
  const int s = split ? choose_splits(tiles, prm.num_k_blocks, pairs_avail) : 1;
  prm.kb_per_split = (prm.num_k_blocks + s - 1) / s;
  prm.splits = (prm.num_k_blocks + prm.kb_per_split - 1) / prm.kb_per_split;
  const int units = tiles * prm.splits;
  const int pairs = units < pairs_avail ? units : pairs_avail;
  return launch(kern, dim3(2 * pairs), dim3(kWideGemmThreads), L::kLaunchBytes, st, p->pdl, 2, maps, prm);
}

// The backward's GEMMs in the plan's form (pairs need an SM budget of at least 2): 1 = pairs
// with BN-column tiles, 2 = pairs with 512-column tiles where B's rows allow, 0 = one CTA.
template <int BN>
int launch_bwd_gemm(ngram_embed_plan* p, const DenseParams& prm, GemmOperand A, GemmOperand B, int64_t K, bool split,
                    cudaStream_t st) {
  if (p->bwd_pair == 2 && p->sms >= 2 && B.rows % 512 == 0)
    return launch_dense_gemm_pair_wide(p, prm, A, B, K, split, st);
  if (p->bwd_pair >= 1 && p->sms >= 2) return launch_dense_gemm_pair<BN>(p, prm, A, B, K, split, st);
  return launch_dense_gemm<BN>(p, prm, A, B, K, split, st);
}

int validate_common(const ngram_embed_plan* p, void* ws, size_t ws_size, int64_t T) {
  if (!p || !ws || T < 0 || T > INT32_MAX) return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(ws)) return NGRAM_ERR_MISALIGNED;
  if (ws_size < ws_base(p, T)) return NGRAM_ERR_WORKSPACE;
  return NGRAM_OK;
}

int set_device(const ngram_embed_plan* p) {
  if (p->device < 0) return NGRAM_ERR_CUDA;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return NGRAM_ERR_CUDA;
  if (cur != p->device && cudaSetDevice(p->device) != cudaSuccess) return NGRAM_ERR_CUDA;
  return NGRAM_OK;
}

int launch_hash(const ngram_embed_plan* p, const int32_t* tokens, const int32_t* offsets, int32_t num_seqs,
                int64_t T, const ngram_cache* cache, const int32_t* slots, int32_t* idx_out, void* ws,
                cudaStream_t st, int32_t* win_out = nullptr, int32_t* entry_out = nullptr, int32_t positions = 0) {
  HashParams h{};
  h.tokens = tokens;
  h.offsets = offsets;
  h.num_seqs = num_seqs;
  h.T = T;
  h.V0 = static_cast<uint32_t>(p->V0);
  h.N = p->N;
  h.K = p->K;
  h.S = p->S;
  for (int s = 0; s < p->S; ++s) {
    h.V[s] = static_cast<uint32_t>(p->V[s]);
    h.barrett[s] = p->barrett[s];
  }
  if (cache) {
    h.ring = cache->ring;
    h.len = cache->len;
    h.valid_from = cache->valid_from;
    h.capacity = cache->capacity;
    h.max_seqs = cache->max_seqs;
    h.slots = slots;
  }
  h.idx_out = idx_out;
  h.win_out = win_out;
  h.entry_out = entry_out;
  h.positions = positions;
  h.status = status_ptr(ws);
  const int64_t work = T > num_seqs + 1 ? T : num_seqs + 1;
  const int64_t blocks = (work + 255) / 256;
  return launch(hash_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, p->pdl, 1, h);
}

int validate_cache(const ngram_embed_plan* p, const ngram_cache* c) {
  if (!c->ring || !c->len || !c->valid_from || c->max_seqs < 0) return NGRAM_ERR_INVALID_ARG;
  if (c->capacity < 1 || c->capacity < p->N - 1) return NGRAM_ERR_INVALID_ARG;
  return NGRAM_OK;
}

template <typename T>
int launch_simt(const ngram_embed_plan* p, const int32_t* tokens, const int32_t* idx, int64_t n_tok,
                const void* E0, const void* const* E_nk, const void* W, void* out, void* ws, cudaStream_t st,
                const int32_t* T_dev = nullptr) {
  SimtParams<T> s{};
  s.T_dev = T_dev;
  s.tokens = tokens;
  s.idx = idx;
  s.E0 = static_cast<const T*>(E0);
  for (int i = 0; i < p->S; ++i) {
    s.E[i] = static_cast<const T*>(E_nk[i]);
    s.Vs[i] = static_cast<uint32_t>(p->V[i]);
  }
  s.W = static_cast<const T*>(W);
  s.out = static_cast<T*>(out);
  s.T_tokens = n_tok;
  s.V0 = static_cast<uint32_t>(p->V0);
  s.D = p->D;
  s.S = p->S;
  s.d = p->d;
  int tpb = static_cast<int>((48 * 1024) / (static_cast<size_t>(p->D) * sizeof(float)));
  if (tpb > 8) tpb = 8;
  if (tpb < 1) tpb = 1;
  s.tokens_per_block = tpb;
  s.scale = p->out_scale / static_cast<float>(p->S + 1);
  s.status = status_ptr(ws);
  const size_t smem = static_cast<size_t>(tpb) * p->D * sizeof(float);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(proj_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return NGRAM_ERR_CUDA;
  }
  const int64_t blocks = (n_tok + tpb - 1) / tpb;
  return launch(proj_simt_kernel<T>, dim3(static_cast<unsigned>(blocks)), dim3(256), smem, st, p->pdl, 1, s);
}

// The projection kernel a call runs (ngram_embed_plan_kernel_form reports the same codes).
enum Form : int {
  kFormSimt = 0,       // CUDA cores
  kFormOne = 1,        // one CTA per 128 x BN tile, fused row gather
  kFormOneSk = 2,      // one CTA per SM, stream-K, fused row gather
  kFormPair = 3,       // CTA pairs, 256 x BN tiles, fused row gather
  kFormPairWide = 4,   // CTA pairs, 256 x 512 tiles, fused row gather
  kFormPairSk = 5,     // CTA pairs, stream-K, fused row gather (opt-in)
  kFormDense = 6,      // rows gathered into G first; CTA pairs, 256 x 256 tiles, A by dense TMA
  kFormDenseSk = 7,    // the same with the pairs' stream-K schedule
  kFormDenseWide = 8,  // the same with 256 x 512 tiles
  kFormPairWideSk = 9, // CTA pairs, 256 x 512 tiles, stream-K, fused row gather
  kFormPairCols = 10,  // CTA pairs, each a range of columns of a 256-row block, fused row gather
  kFormDenseCols = 11, // rows gathered into G first; CTA pairs over column ranges, A by dense TMA
};

// Stream-K for the dense-A pair form: where a grid of whole 256 x 256 tiles would take two or
// more waves of pairs and leave many pairs idle in the last (a decode step of 1280 tokens at
// D = 4096: 80 tiles on 74 pairs), as for the one-CTA form.
bool dense_stream_k(const ngram_embed_plan* p, int64_t T, size_t ws_size, int64_t ws_T) {
  if (p->stream_k == 2 || p->sms < 2 || p->pair_wide == 1) return false;
  const int64_t pairs = p->sms / 2;
  const int64_t tiles = (T + 2 * kBM - 1) / (2 * kBM) * (p->D / 256);
  const int64_t units = tiles * (p->D / kBK);
  if (tiles > kSkMaxTiles / 2 || units < pairs) return false;
  if (ws_size < ws_base(p, ws_T) + sk_partial_bytes(p)) return false;
  if (p->stream_k == 1) return true;
  const int64_t waves = (tiles + pairs - 1) / pairs;
  return waves >= 2 && 1.3 * static_cast<double>(tiles) < static_cast<double>(waves * pairs);
}

// ws_T: the token count the workspace was validated for (its index buffer's length); the
// stream-K partials and the dense-A G buffer, if the workspace holds them, follow that buffer.
// count_on_device: the token count is known only on the device (a draft call's misses).
int choose_form(const ngram_embed_plan* p, int64_t T, size_t ws_size, int64_t ws_T, bool count_on_device) {
  if (p->variant == kSimt) return kFormSimt;
  if (!count_on_device && p->cta_pair != 0 && dense_wanted(p) &&
      ws_size >= dense_g_offset(p, ws_T) + dense_g_bytes(p, T)) {
    if (use_pair_cols(p, T, count_on_device)) return kFormDenseCols;
    if (dense_stream_k(p, T, ws_size, ws_T)) return kFormDenseSk;
    return use_pair_wide(p, T) ? kFormDenseWide : kFormDense;
  }
  // Not stream-K when the count is known only on the device: for the few tiles of a draft
  // call's misses its fix-ups cost more than they balance (measured: 256 misses at D = 4096,
  // 79 us stream-K vs 64 us CTA pairs). Otherwise the one-CTA form's stream-K where its grid
  // ends in a thin wave, else the pair form (512-column tiles where they fill their waves).
  ProjParams prm{};
  prm.num_m_blocks = static_cast<int>((T + kBM - 1) / kBM);
  prm.num_n_blocks = p->D / p->bn;
  prm.num_k_blocks = p->D / kBK;
  if (use_pair_cols(p, T, count_on_device)) return kFormPairCols;
  const bool psk = !count_on_device && p->cta_pair != 0 && p->pair_wide != 1 && use_pair_stream_k(p, T, ws_size, ws_T);
  if (!psk && !count_on_device && use_wide_stream_k(p, T, ws_size, ws_T)) return kFormPairWideSk;
  const bool sk = !psk && !count_on_device && p->cta_pair != 1 && use_stream_k(p, prm, ws_T, ws_size);
  const bool pair = p->cta_pair == 1 || (p->cta_pair == -1 && !sk);
  if (pair) return psk ? kFormPairSk : (use_pair_wide(p, T, count_on_device) ? kFormPairWide : kFormPair);
  return sk ? kFormOneSk : kFormOne;
}

// The stand-alone gather kernel: G[i][s*d + c] = E_s[idx[i][s]][c] and, if E0_out is given,
// E0_out[i] = E_0[tokens[i]]. Arguments already checked.
int launch_gather(const ngram_embed_plan* p, const int32_t* idx, int64_t T, const void* const* E_nk, void* G,
                  const int32_t* tokens, const void* E0, void* E0_out, void* ws, cudaStream_t st) {
  GatherParams g{};
  for (int s = 0; s < p->S; ++s) {
    g.E[s] = static_cast<const uint8_t*>(E_nk[s]);
    g.Vs[s] = static_cast<uint32_t>(p->V[s]);
  }
  g.idx = idx;
  g.G = static_cast<uint8_t*>(G);
  g.T = T;
  g.S = p->S;
  g.row_bytes = p->d * p->elt;
  g.tokens = tokens;
  g.E0 = static_cast<const uint8_t*>(E0);
  g.E0_out = static_cast<uint8_t*>(E0_out);
  g.V0 = static_cast<uint32_t>(p->V0);
  g.e0_row_bytes = p->D * p->elt;
  g.status = status_ptr(ws);
  // every resident thread (8 blocks of 256 per SM, spread evenly over the SMs) takes an
  // equal share of the 16-byte vectors; fewer blocks only when there are fewer vectors
  const int64_t vecs = T * p->S * (g.row_bytes / 16) + (E0_out ? T * (g.e0_row_bytes / 16) : 0);
  // the kernel numbers vectors (and its grid-stride steps) in 32 bits
  if (vecs + static_cast<int64_t>(p->sms > 0 ? p->sms : 1) * 8 * 256 * kGatherUnroll > UINT32_MAX)
    return NGRAM_ERR_UNSUPPORTED;
  auto log2_or_neg = [](int v) {
    int sh = 0;
    while ((1 << sh) < v) ++sh;
    return (1 << sh) == v ? sh : -1;
  };
  g.vshift = log2_or_neg(g.row_bytes / 16);
  g.eshift = log2_or_neg(g.e0_row_bytes / 16);
  int64_t blocks = (vecs + 255) / 256;
  const int64_t cap = static_cast<int64_t>(p->sms > 0 ? p->sms : 1) * 8;
  if (blocks > cap) blocks = cap;
  return launch(gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, p->pdl, 1, g);
}

// T_dev (optional): the kernels take min(*T_dev, T) tokens, a count known only on the device.
// g_ready: in the dense-A form, G already holds the call's sub-rows (the decode step's fused
// commit + hash + gather launch wrote it).
int project(ngram_embed_plan* p, const int32_t* tokens, const int32_t* idx, int64_t T, const void* E0,
            const void* const* E_nk, const void* W, void* out, void* ws, size_t ws_size, int64_t ws_T,
            cudaStream_t st, const int32_t* T_dev = nullptr, bool g_ready = false,
            const StepHash* sh = nullptr) {
  if (p->variant == kSimt) {
    return p->dtype == NGRAM_F32
               ? launch_simt<float>(p, tokens, idx, T, E0, E_nk, W, out, ws, st, T_dev)
               : launch_simt<uint16_t>(p, tokens, idx, T, E0, E_nk, W, out, ws, st, T_dev);
  }
  int rc = refresh_maps(p, E_nk, W, out, T);
  if (rc) return rc;
  ProjParams prm{};
  prm.tokens = tokens;
  prm.idx = idx;
  prm.E0 = static_cast<const uint16_t*>(E0);
  for (int s = 0; s < p->S; ++s) {
    prm.E[s] = static_cast<const uint16_t*>(E_nk[s]);
    prm.Vs[s] = static_cast<uint32_t>(p->V[s]);
  }
  prm.out = static_cast<uint16_t*>(out);
  prm.T = T;
  prm.V0 = static_cast<uint32_t>(p->V0);
  prm.D = p->D;
  prm.S = p->S;
  prm.d = p->d;
  prm.num_m_blocks = static_cast<int>((T + kBM - 1) / kBM);
  prm.num_n_blocks = p->D / p->bn;
  prm.num_k_blocks = p->D / kBK;
  prm.scale = p->out_scale / static_cast<float>(p->S + 1);
  prm.status = status_ptr(ws);
  prm.T_dev = T_dev;
  auto* wsb = static_cast<uint8_t*>(ws);
  auto stream_k_buffers = [&] {
    prm.stream_k = 1;
    prm.sk_counters = reinterpret_cast<int*>(wsb + kStatusBytes);
    prm.sk_partials = reinterpret_cast<float*>(wsb + ws_base(p, ws_T));
  };
  const int form = choose_form(p, T, ws_size, ws_T, T_dev != nullptr);
  if (form == kFormDense || form == kFormDenseSk || form == kFormDenseWide || form == kFormDenseCols) {
    // the call's sub-rows into G (workspace), then A tiles as dense TMA boxes of G
    void* G = wsb + dense_g_offset(p, ws_T);
    if (!g_ready && (rc = launch_gather(p, idx, T, E_nk, G, nullptr, nullptr, nullptr, ws, st))) return rc;
    if (p->map_A != G || p->map_A_T != T) {
      p->map_A = nullptr;
      if ((rc = encode_2d(&p->maps.A, G, p->D, static_cast<uint64_t>(T), static_cast<uint64_t>(p->D) * 2, kBK, kBM,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B)))
        return rc;
      p->map_A = G;
      p->map_A_T = T;
    }
    prm.dense_a = 1;
    prm.tma_rows = 0;
    if (form == kFormDenseCols) return launch_cols(p, prm, T, st);
    if (form == kFormDenseWide) {
      prm.num_n_blocks = p->D / 512;
      return launch_tc_pair_stages<512, kPairStagesWide>(p, prm, T, st, 8);
    }
    if (form == kFormDenseSk) stream_k_buffers();
    return launch_tc_pair<256>(p, prm, T, st);
  }
  if (form == kFormPairCols) return launch_cols(p, prm, T, st);
  if (form == kFormPairWideSk) {
    prm.num_n_blocks = p->D / 512;
    prm.tma_rows = kBM;  // A rows by gather4 only
    stream_k_buffers();
    return launch_tc_pair_stages<512, kPairStagesWide, true>(p, prm, T, st, 9);
  }
  const bool pair = form == kFormPair || form == kFormPairWide || form == kFormPairSk;
  // A rows by TMA gather4 in the pair form, by cp.async in the one-CTA form (measured
  // fastest for each), unless the plan fixes the split.
  prm.tma_rows = p->variant == kTcTmaRows ? kBM : (p->tma_rows >= 0 ? p->tma_rows : (pair ? kBM : 0));
  if (form == kFormPairWide) {
    prm.num_n_blocks = p->D / 512;
    prm.tma_rows = kBM;  // A rows by gather4 only
    return launch_tc_pair_stages<512, kPairStagesWide>(p, prm, T, st, 8);
  }
  if (form == kFormPairSk) {
    stream_k_buffers();
    prm.tma_rows = kBM;  // A rows by gather4 only
    return launch_tc_pair<256>(p, prm, T, st);
  }
  if (pair) return p->bn == 256 ? launch_tc_pair<256>(p, prm, T, st) : launch_tc_pair<128>(p, prm, T, st);
  if (form == kFormOneSk) stream_k_buffers();
  if (sh && (form == kFormOne || form == kFormOneSk)) prm.sh = *sh;  // the decode step's commit and hashing
  return p->bn == 256 ? launch_tc<256>(p, prm, st) : launch_tc<128>(p, prm, st);
}

int check_tables(const ngram_embed_plan* p, const void* E0, const void* const* E_nk, const void* W) {
  if (!E0 || (p->S > 0 && (!E_nk || !W))) return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(E0)) return NGRAM_ERR_MISALIGNED;
  for (int s = 0; s < p->S; ++s) {
    if (!E_nk[s]) return NGRAM_ERR_INVALID_ARG;
    if (!aligned16(E_nk[s])) return NGRAM_ERR_MISALIGNED;
  }
  if (p->S > 0 && !aligned16(W)) return NGRAM_ERR_MISALIGNED;
  return NGRAM_OK;
}

}  // namespace

extern "C" {

const char* ngram_embed_error_string(int code) {
  switch (code) {
    case NGRAM_OK: return "ok";
    case NGRAM_ERR_INVALID_ARG: return "invalid argument";
    case NGRAM_ERR_UNSUPPORTED: return "unsupported configuration";
    case NGRAM_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case NGRAM_ERR_WORKSPACE: return "workspace too small";
    case NGRAM_ERR_CUDA: return "CUDA call or launch failed";
    default: return "unknown error";
  }
}

int ngram_embed_plan_create(const ngram_embed_config* cfg, ngram_embed_plan** out) {
  if (!cfg || !out) return NGRAM_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg->V0 < 1 || cfg->V0 >= (int64_t(1) << 31) || cfg->D < 1 || cfg->N < 1 || cfg->K < 1)
    return NGRAM_ERR_INVALID_ARG;
  if (cfg->dtype != NGRAM_BF16 && cfg->dtype != NGRAM_F32) return NGRAM_ERR_INVALID_ARG;
  if (cfg->N > kMaxN) return NGRAM_ERR_UNSUPPORTED;
  const int64_t S = static_cast<int64_t>(cfg->N - 1) * cfg->K;
  if (S > kMaxS) return NGRAM_ERR_UNSUPPORTED;
  if (S > 0 && (cfg->D % S != 0)) return NGRAM_ERR_INVALID_ARG;
  if (S > 0 && !cfg->V_nk) return NGRAM_ERR_INVALID_ARG;
  const int elt = cfg->dtype == NGRAM_BF16 ? 2 : 4;
  const int d = S ? static_cast<int>(cfg->D / S) : 0;
  if ((static_cast<int64_t>(cfg->D) * elt) % 16 != 0) return NGRAM_ERR_UNSUPPORTED;
  if (S > 0 && (static_cast<int64_t>(d) * elt) % 16 != 0) return NGRAM_ERR_UNSUPPORTED;
  for (int s = 0; s < S; ++s)
    if (cfg->V_nk[s] < 1 || cfg->V_nk[s] >= (int64_t(1) << 31)) return NGRAM_ERR_INVALID_ARG;

  auto* p = new (std::nothrow) ngram_embed_plan();
  if (!p) return NGRAM_ERR_INVALID_ARG;
  p->V0 = cfg->V0;
  p->D = cfg->D;
  p->N = cfg->N;
  p->K = cfg->K;
  p->S = static_cast<int>(S);
  p->d = d;
  p->dtype = cfg->dtype;
  p->elt = elt;
  for (int s = 0; s < S; ++s) {
    p->V[s] = cfg->V_nk[s];
    p->barrett[s] = ~uint64_t(0) / static_cast<uint64_t>(cfg->V_nk[s]);
  }
  // Without a usable device the plan still validates arguments; launches then fail
  // with NGRAM_ERR_CUDA.
  if (cudaGetDevice(&p->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&p->sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess) {
    cudaGetLastError();
    p->device = -1;
    p->sms = 0;
  }
  p->sms_device = p->sms;
  p->tc_ok = cfg->dtype == NGRAM_BF16 && S > 0 && cfg->D % 128 == 0 && d % kBK == 0;
  p->bn = cfg->D % 256 == 0 ? 256 : 128;
  p->variant = p->tc_ok ? kTcSplitRows : kSimt;
  // Defaults from B200 measurements: the CTA pair with every A row gathered by TMA, except
  // where the one-CTA form's stream-K schedule applies (grids that end in a thin last wave,
  // e.g. a 1280-token decode step at D = 4096), with cp.async rows.
  p->cta_pair = -1;
  p->tma_rows = -1;
  *out = p;
  return NGRAM_OK;
}

int ngram_embed_plan_destroy(ngram_embed_plan* plan) {
  if (plan && plan->aux && set_device(plan) == NGRAM_OK) {
    cudaStreamSynchronize(plan->aux);
    for (cudaEvent_t e : plan->aux_ev)
      if (e) cudaEventDestroy(e);
    cudaStreamDestroy(plan->aux);
  }
  delete plan;
  return NGRAM_OK;
}

int ngram_embed_plan_uses_tensor_cores(const ngram_embed_plan* plan) {
  return plan && plan->variant != kSimt ? 1 : 0;
}

// Select the projection kernel: 0 = automatic, 1 = tensor cores with every A row gathered by
// TMA, 2 = tensor cores with the A rows split between TMA and cp.async, 3 = CUDA cores.
int ngram_embed_plan_set_variant(ngram_embed_plan* plan, int variant) {
  if (!plan || variant < kAuto || variant > kSimt) return NGRAM_ERR_INVALID_ARG;
  if ((variant == kTcTmaRows || variant == kTcSplitRows) && !plan->tc_ok) return NGRAM_ERR_UNSUPPORTED;
  plan->variant = variant == kAuto ? (plan->tc_ok ? kTcSplitRows : kSimt) : variant;
  return NGRAM_OK;
}

// Tensor-core kernel, variant 2: how many of the 128 rows of each A tile TMA gathers
// (0, 32, 64, 96 or 128); cp.async gathers the rest.
int ngram_embed_plan_set_tma_rows(ngram_embed_plan* plan, int rows) {
  if (!plan || rows < -1 || rows > kBM || (rows >= 0 && rows % 32 != 0)) return NGRAM_ERR_INVALID_ARG;
  plan->tma_rows = rows;
  return NGRAM_OK;
}

// Tensor-core kernel form: 1 = CTA pairs (cta_group::2, 256-token tiles; default),
// 0 = one CTA per tile (128-token tiles).
int ngram_embed_plan_set_cta_pair(ngram_embed_plan* plan, int on) {
  if (!plan || on < -1 || on > 1) return NGRAM_ERR_INVALID_ARG;
  plan->cta_pair = on;
  return NGRAM_OK;
}

int ngram_embed_plan_kernel_form(const ngram_embed_plan* plan, int64_t num_tokens) {
  if (!plan || num_tokens < 0 || num_tokens > INT32_MAX) return NGRAM_ERR_INVALID_ARG;
  return choose_form(plan, num_tokens, ws_bytes(plan, num_tokens), num_tokens, false);
}

int ngram_embed_plan_set_backward_streams(ngram_embed_plan* plan, int on) {
  if (!plan || on < 0 || on > 1) return NGRAM_ERR_INVALID_ARG;
  plan->bwd_streams = on;
  return NGRAM_OK;
}

int ngram_embed_plan_set_backward_pair(ngram_embed_plan* plan, int on) {
  if (!plan || on < 0 || on > 2) return NGRAM_ERR_INVALID_ARG;
  plan->bwd_pair = on;
  return NGRAM_OK;
}

int ngram_embed_plan_set_fused_step(ngram_embed_plan* plan, int on) {
  if (!plan || on < 0 || on > 1) return NGRAM_ERR_INVALID_ARG;
  plan->fused_step = on;
  return NGRAM_OK;
}

int ngram_embed_plan_set_pair_columns(ngram_embed_plan* plan, int mode) {
  if (!plan || mode < -1 || mode > 1) return NGRAM_ERR_INVALID_ARG;
  plan->pair_cols = mode == 1 ? 1 : 0;
  return NGRAM_OK;
}

int ngram_embed_plan_set_dense_a(ngram_embed_plan* plan, int mode) {
  if (!plan || mode < 0 || mode > 1) return NGRAM_ERR_INVALID_ARG;
  plan->dense_a = mode;
  return NGRAM_OK;
}

int ngram_embed_plan_set_sm_count(ngram_embed_plan* plan, int sms) {
  if (!plan || sms < 0 || sms == 1 || (plan->sms_device > 0 && sms > plan->sms_device)) return NGRAM_ERR_INVALID_ARG;
  plan->sms = sms == 0 ? plan->sms_device : sms;
  return NGRAM_OK;
}

int ngram_embed_plan_set_pair_wide(ngram_embed_plan* plan, int on) {
  if (!plan || on < -1 || on > 1) return NGRAM_ERR_INVALID_ARG;
  plan->pair_wide = on;
  return NGRAM_OK;
}

// Tensor-core tile width: 256 or 128 output columns per tile (D must divide).
int ngram_embed_plan_set_tile_n(ngram_embed_plan* plan, int bn) {
  if (!plan || (bn != 128 && bn != 256) || plan->D % bn != 0) return NGRAM_ERR_INVALID_ARG;
  plan->bn = bn;
  plan->maps_valid = false;
  return NGRAM_OK;
}

int ngram_embed_plan_set_a_stages(ngram_embed_plan* plan, int stages) {
  if (!plan) return NGRAM_ERR_INVALID_ARG;
  // every depth some form takes; a form given a depth it does not take uses its default
  const bool ok = stages == 0 || (stages % 2 == 0 && stages >= 2 && stages <= 12);
  if (!ok) return NGRAM_ERR_INVALID_ARG;
  plan->a_stages = stages;
  return NGRAM_OK;
}

int ngram_embed_plan_set_output_scale(ngram_embed_plan* plan, float scale) {
  if (!plan || !(scale == scale) || scale == 0.0f || scale > 3.0e38f || scale < -3.0e38f) return NGRAM_ERR_INVALID_ARG;
  plan->out_scale = scale;
  return NGRAM_OK;
}

// ---- hash statistics -----------------------------------------------------------------
namespace {
uint64_t stats_set_cap(int64_t T) {
  uint64_t cap = 1024;
  while (cap < 2 * static_cast<uint64_t>(T)) cap <<= 1;
  return cap;
}
size_t stats_ws_bytes(int64_t T, int64_t max_modulus, int num_moduli) {
  return kHeadBytes + round256(static_cast<size_t>(T) * 8 * kWinWords) + round256(stats_set_cap(T) * 8) + 256 +
         round256((static_cast<size_t>(max_modulus) / 32 + 1) * 4) + round256(static_cast<size_t>(num_moduli) * 8);
}
}  // namespace

size_t ngram_hash_stats_workspace_bytes(int64_t max_tokens, int64_t max_modulus, int num_moduli) {
  if (max_tokens < 0 || max_modulus < 1 || num_moduli < 1) return 0;
  return stats_ws_bytes(max_tokens, max_modulus, num_moduli);
}

int ngram_hash_stats(int64_t V0, int n, const int32_t* tokens, const int32_t* seq_offsets, int32_t num_seqs,
                     int64_t num_tokens, const int64_t* moduli, int num_moduli, int64_t* rows_hit,
                     int64_t* distinct_ngrams, void* workspace, size_t workspace_bytes, void* stream) {
  if (V0 < 1 || V0 >= (int64_t(1) << 31) || n < 1 || n > kMaxN || num_tokens < 0 || num_tokens > INT32_MAX ||
      num_seqs < 1 || !moduli || num_moduli < 1 || !rows_hit || !distinct_ngrams || !workspace ||
      (num_tokens > 0 && (!tokens || !seq_offsets)))
    return NGRAM_ERR_INVALID_ARG;
  int64_t max_v = 0;
  for (int j = 0; j < num_moduli; ++j) {
    if (moduli[j] < 1 || moduli[j] >= (int64_t(1) << 31)) return NGRAM_ERR_INVALID_ARG;
    max_v = moduli[j] > max_v ? moduli[j] : max_v;
  }
  if (!aligned16(workspace)) return NGRAM_ERR_MISALIGNED;
  if (workspace_bytes < stats_ws_bytes(num_tokens, max_v, num_moduli)) return NGRAM_ERR_WORKSPACE;
  // V0^n < 2^64: the window's exact integer fits a 64-bit key
  unsigned __int128 pw = 1;
  bool exact64 = true;
  for (int j = 0; j < n && exact64; ++j) {
    pw *= static_cast<unsigned __int128>(V0);
    exact64 = pw < (static_cast<unsigned __int128>(1) << 64);
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return NGRAM_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const uint64_t cap = stats_set_cap(num_tokens);
  auto* keys = reinterpret_cast<unsigned long long*>(base + kHeadBytes);
  auto* set = reinterpret_cast<unsigned long long*>(base + kHeadBytes + round256(size_t(num_tokens) * 8 * kWinWords));
  auto* distinct = reinterpret_cast<unsigned long long*>(reinterpret_cast<uint8_t*>(set) + round256(cap * 8));
  auto* bitmap = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(distinct) + 256);
  auto* hits = reinterpret_cast<unsigned long long*>(reinterpret_cast<uint8_t*>(bitmap) +
                                                     round256((size_t(max_v) / 32 + 1) * 4));
  if (cudaMemsetAsync(distinct, 0, 8, st) != cudaSuccess ||
      cudaMemsetAsync(hits, 0, size_t(num_moduli) * 8, st) != cudaSuccess)
    return NGRAM_ERR_CUDA;
  StatsParams sp{};
  sp.tokens = tokens;
  sp.offsets = seq_offsets;
  sp.num_seqs = num_seqs;
  sp.T = num_tokens;
  sp.V0 = static_cast<uint32_t>(V0);
  sp.n = n;
  sp.exact64 = exact64;
  sp.keys = keys;
  sp.set = set;
  sp.set_mask = cap - 1;
  sp.distinct = distinct;
  sp.status = status_ptr(workspace);
  const unsigned blocks = static_cast<unsigned>((num_tokens + 255) / 256);
  int rc = NGRAM_OK;
  if (num_tokens > 0) {
    if (cudaMemsetAsync(set, 0xFF, cap * 8, st) != cudaSuccess) return NGRAM_ERR_CUDA;
    if (exact64) {
      if ((rc = launch(stats_keys_kernel, dim3(blocks), dim3(256), 0, st, false, 1, sp))) return rc;
    } else {
      if ((rc = launch(stats_window_keys_kernel, dim3(blocks), dim3(256), 0, st, false, 1, sp))) return rc;
      if ((rc = launch(stats_window_insert_kernel, dim3(blocks), dim3(256), 0, st, false, 1, sp))) return rc;
    }
  }
  for (int j = 0; j < num_moduli && num_tokens > 0; ++j) {
    sp.V = static_cast<uint32_t>(moduli[j]);
    sp.barrett = ~uint64_t(0) / static_cast<uint64_t>(moduli[j]);
    sp.bitmap = bitmap;
    sp.rows_hit = hits + j;
    if (cudaMemsetAsync(bitmap, 0, (size_t(moduli[j]) / 32 + 1) * 4, st) != cudaSuccess) return NGRAM_ERR_CUDA;
    if ((rc = launch(stats_rows_kernel, dim3(blocks), dim3(256), 0, st, false, 1, sp))) return rc;
  }
  unsigned long long d_host = 0;
  if (cudaMemcpyAsync(&d_host, distinct, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(rows_hit, hits, size_t(num_moduli) * 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return NGRAM_ERR_CUDA;
  *distinct_ngrams = static_cast<int64_t>(d_host);
  return NGRAM_OK;
}

// ---- draft-phase embedding cache ----------------------------------------------------
namespace {
struct DraftWs {
  int32_t *idx, *win, *entry, *miss_count, *miss_token, *miss_idx, *miss_pos, *miss_entry;
  uint8_t* miss_out;
  size_t bytes;
};
DraftWs draft_ws(const ngram_embed_plan* p, int64_t T, void* ws) {
  DraftWs w{};
  size_t off = kHeadBytes;
  auto take = [&](size_t b) {
    const size_t at = off;
    off += round256(b);
    return at;
  };
  const size_t t = static_cast<size_t>(T);
  const size_t a_idx = take(t * p->S * 4), a_win = take(t * p->N * 4), a_entry = take(t * 4), a_cnt = take(4),
               a_tok = take(t * 4), a_midx = take(t * p->S * 4), a_pos = take(t * 4), a_ment = take(t * 4),
               a_out = take(t * static_cast<size_t>(p->D) * p->elt);
  w.bytes = off;
  if (ws) {
    auto* b = static_cast<uint8_t*>(ws);
    w.idx = reinterpret_cast<int32_t*>(b + a_idx);
    w.win = reinterpret_cast<int32_t*>(b + a_win);
    w.entry = reinterpret_cast<int32_t*>(b + a_entry);
    w.miss_count = reinterpret_cast<int32_t*>(b + a_cnt);
    w.miss_token = reinterpret_cast<int32_t*>(b + a_tok);
    w.miss_idx = reinterpret_cast<int32_t*>(b + a_midx);
    w.miss_pos = reinterpret_cast<int32_t*>(b + a_pos);
    w.miss_entry = reinterpret_cast<int32_t*>(b + a_ment);
    w.miss_out = b + a_out;
  }
  return w;
}
}  // namespace

size_t ngram_embed_draft_workspace_bytes(const ngram_embed_plan* plan, int64_t max_tokens) {
  if (!plan || max_tokens < 0) return 0;
  return draft_ws(plan, max_tokens, nullptr).bytes;
}

int ngram_draft_cache_reset(const ngram_embed_plan* plan, const ngram_draft_cache* dc, const int32_t* slots,
                            int32_t n, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_common(plan, workspace, workspace_bytes, 0);
  if (rc) return rc;
  if (!dc || !dc->keys || !dc->emb || dc->positions < 1 || dc->max_seqs < 0 || n < 0 || n > dc->max_seqs)
    return NGRAM_ERR_INVALID_ARG;
  if (n == 0) return NGRAM_OK;
  if ((rc = set_device(plan))) return rc;
  DraftResetParams r{};
  r.keys = dc->keys;
  r.slots = slots;
  r.n = n;
  r.positions = dc->positions;
  r.N = plan->N;
  r.max_seqs = dc->max_seqs;
  r.status = status_ptr(workspace);
  const int64_t work = static_cast<int64_t>(n) * dc->positions;
  return launch(draft_reset_kernel, dim3(static_cast<unsigned>((work + 255) / 256)), dim3(256), 0,
                static_cast<cudaStream_t>(stream), plan->pdl, 1, r);
}

int ngram_embed_fwd_draft(const ngram_embed_plan* plan_c, const int32_t* tokens, const int32_t* seq_offsets,
                          int32_t num_seqs, int64_t num_tokens, const void* E0, const void* const* E_nk,
                          const void* W_stacked, const ngram_cache* cache, const int32_t* cache_slots,
                          const ngram_draft_cache* dc, void* out, int32_t* hits_out, void* workspace,
                          size_t workspace_bytes, void* stream) {
  auto* plan = const_cast<ngram_embed_plan*>(plan_c);
  if (!plan || !workspace || num_tokens < 0 || num_tokens > INT32_MAX || num_seqs < 0) return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return NGRAM_ERR_MISALIGNED;
  const DraftWs w = draft_ws(plan, num_tokens, workspace);
  if (workspace_bytes < w.bytes) return NGRAM_ERR_WORKSPACE;
  if (num_tokens == 0) return NGRAM_OK;
  if (!tokens || !seq_offsets || num_seqs == 0 || !out || !cache || !dc || !dc->keys || !dc->emb ||
      dc->positions < 1 || dc->max_seqs < cache->max_seqs)
    return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(dc->emb)) return NGRAM_ERR_MISALIGNED;
  int rc;
  if ((rc = check_tables(plan, E0, E_nk, W_stacked))) return rc;
  if ((rc = validate_cache(plan, cache))) return rc;
  if ((rc = set_device(plan))) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(w.miss_count, 0, 4, st) != cudaSuccess) return NGRAM_ERR_CUDA;
  if ((rc = launch_hash(plan, tokens, seq_offsets, num_seqs, num_tokens, cache, cache_slots, w.idx, workspace, st,
                        w.win, w.entry, dc->positions)))
    return rc;
  DraftParams d{};
  d.tokens = tokens;
  d.idx = w.idx;
  d.win = w.win;
  d.entry = w.entry;
  d.keys = dc->keys;
  d.emb = static_cast<uint8_t*>(dc->emb);
  d.T = num_tokens;
  d.N = plan->N;
  d.S = plan->S;
  d.row_bytes = plan->D * plan->elt;
  d.out = static_cast<uint8_t*>(out);
  d.miss_count = w.miss_count;
  d.miss_token = w.miss_token;
  d.miss_idx = w.miss_idx;
  d.miss_pos = w.miss_pos;
  d.miss_entry = w.miss_entry;
  d.miss_out = w.miss_out;
  d.hits = hits_out;
  const unsigned warps_blocks = static_cast<unsigned>((num_tokens + 7) / 8);
  if ((rc = launch(draft_probe_kernel, dim3(warps_blocks), dim3(256), 0, st, plan->pdl, 1, d))) return rc;
  // the misses' rows (at most num_tokens; the kernels read the count)
  if ((rc = project(plan, w.miss_token, w.miss_idx, num_tokens, E0, E_nk, W_stacked, w.miss_out, workspace,
                    workspace_bytes, 0, st, w.miss_count)))
    return rc;
  return launch(draft_scatter_kernel, dim3(warps_blocks), dim3(256), 0, st, plan->pdl, 1, d);
}

size_t ngram_embed_bwd_workspace_bytes(const ngram_embed_plan* plan, int64_t max_tokens) {
  if (!plan || max_tokens < 0) return 0;
  return bwd_ws_bytes(plan, max_tokens);
}

// The plan's auxiliary stream and its three events, created on first use (non-blocking
// stream: no implicit ordering with the legacy default stream; events without timing).
int ensure_aux(ngram_embed_plan* p) {
  if (p->aux) return NGRAM_OK;
  cudaStream_t s = nullptr;
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return NGRAM_ERR_CUDA;
  cudaEvent_t ev[3] = {};
  for (auto& e : ev) {
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (cudaEvent_t x : ev)
        if (x) cudaEventDestroy(x);
      cudaStreamDestroy(s);
      return NGRAM_ERR_CUDA;
    }
  }
  p->aux = s;
  for (int i = 0; i < 3; ++i) p->aux_ev[i] = ev[i];
  return NGRAM_OK;
}

int ngram_embed_bwd(const ngram_embed_plan* plan_c, const int32_t* tokens, const int32_t* idx, int64_t num_tokens,
                    const void* const* E_nk, const void* W_stacked, const void* grad_out, float* dE0,
                    float* const* dE_nk, float* dW, void* workspace, size_t workspace_bytes, void* stream) {
  auto* p = const_cast<ngram_embed_plan*>(plan_c);
  if (!p || !workspace || num_tokens < 0 || num_tokens > INT32_MAX) return NGRAM_ERR_INVALID_ARG;
  if (!p->tc_ok) return NGRAM_ERR_UNSUPPORTED;  // bf16 tensor-core shapes only
  if (!aligned16(workspace)) return NGRAM_ERR_MISALIGNED;
  if (workspace_bytes < bwd_ws_bytes(p, num_tokens)) return NGRAM_ERR_WORKSPACE;
  if (num_tokens == 0 || (!dE0 && !dE_nk && !dW)) return NGRAM_OK;
  if (!tokens || !idx || !grad_out || (dE_nk && !W_stacked) || (dW && !E_nk))
    return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(grad_out) || (dE0 && !aligned16(dE0)) || (dW && !aligned16(dW)) ||
      (W_stacked && !aligned16(W_stacked)))
    return NGRAM_ERR_MISALIGNED;
  for (int s = 0; s < p->S; ++s) {
    if (dE_nk && (!dE_nk[s] || !aligned16(dE_nk[s]))) return dE_nk[s] ? NGRAM_ERR_MISALIGNED : NGRAM_ERR_INVALID_ARG;
    if (dW && (!E_nk[s] || !aligned16(E_nk[s]))) return E_nk[s] ? NGRAM_ERR_MISALIGNED : NGRAM_ERR_INVALID_ARG;
  }
  int rc = set_device(p);
  if (rc) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t T = num_tokens;
  const int D = p->D;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* G = reinterpret_cast<uint16_t*>(base + kHeadBytes);
  const float scale = p->out_scale / static_cast<float>(p->S + 1);
  const auto* g = static_cast<const uint16_t*>(grad_out);

  // The memory-bound kernels (the gather of G for dW, the dE0 sort and sums) run on the plan's
  // auxiliary stream, forked from and joined back to `st`, so that they overlap the dG GEMM
  // (persistent CTAs that leave registers and threads free on every SM); dW waits for G only.
  // dG is launched first so that its CTAs take their places on the SMs before the side
  // stream's blocks fill what is left.
  const bool fork = p->bwd_streams == 1 && dE_nk && (dE0 || dW);
  if (fork && (rc = ensure_aux(p))) return rc;
  const cudaStream_t side = fork ? p->aux : st;
  bool joined = !fork;
  auto join = [&](int code) {
    if (!joined) {
      joined = true;
      if ((cudaEventRecord(p->aux_ev[2], side) != cudaSuccess || cudaStreamWaitEvent(st, p->aux_ev[2], 0) != cudaSuccess) &&
          code == NGRAM_OK)
        code = NGRAM_ERR_CUDA;
    }
    return code;
  };
  if (fork && (cudaEventRecord(p->aux_ev[0], st) != cudaSuccess || cudaStreamWaitEvent(side, p->aux_ev[0], 0) != cudaSuccess)) {
    joined = true;  // nothing was forked
    return NGRAM_ERR_CUDA;
  }
  if (dE_nk) {
    // dG = c g W_stacked: A = g [T x D] (K-major over D), B[n][k] = W_stacked[k][n] (W as it
    // lies: MN-major); the epilogue adds each 32-column piece into its sub-table's gradient row.
    DenseParams dp{};
    dp.scale = scale;
    dp.epi = kEpiScatterSub;
    dp.idx = idx;
    for (int s = 0; s < p->S; ++s) {
      dp.dE[s] = dE_nk[s];
      dp.Vs[s] = static_cast<uint32_t>(p->V[s]);
    }
    dp.S = p->S;
    dp.d = p->d;
    dp.status = status_ptr(workspace);
    const GemmOperand A{g, T, false}, B{W_stacked, D, true};
    if ((rc = p->D % 256 == 0 ? launch_bwd_gemm<256>(p, dp, A, B, D, false, st)
                              : launch_bwd_gemm<128>(p, dp, A, B, D, false, st)))
      return join(rc);
  }
  if (dW) {
    if ((rc = launch_gather(p, idx, T, E_nk, G, nullptr, nullptr, nullptr, workspace, side))) return join(rc);
    if (fork && cudaEventRecord(p->aux_ev[1], side) != cudaSuccess) return join(NGRAM_ERR_CUDA);
  }
  if (dE0) {
    uint8_t* sort = base + kHeadBytes + bwd_g_bytes(p, T);
    ScatterE0Params e{};
    e.tokens = tokens;
    e.g = g;
    e.dE0 = dE0;
    e.T = T;
    e.D = D;
    e.V0 = static_cast<uint32_t>(p->V0);
    e.scale = scale;
    e.counts = reinterpret_cast<int32_t*>(sort);
    e.order = reinterpret_cast<int32_t*>(sort + round256((size_t(p->V0) + 1) * 4));
    e.sorted_tok = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(e.order) + round256(size_t(T) * 4));
    e.block_sums = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(e.sorted_tok) + round256(size_t(T) * 4));
    e.num_blocks = static_cast<int>((p->V0 + 1023) / 1024);
    e.status = status_ptr(workspace);
    const unsigned tb = static_cast<unsigned>((T + 255) / 256);
    if (cudaMemsetAsync(e.counts, 0, (size_t(p->V0) + 1) * 4, side) != cudaSuccess) return join(NGRAM_ERR_CUDA);
    if ((rc = launch(e0_hist_kernel, dim3(tb), dim3(256), 0, side, p->pdl, 1, e))) return join(rc);
    if ((rc = launch(e0_scan_kernel, dim3(e.num_blocks), dim3(1024), 0, side, p->pdl, 1, e))) return join(rc);
    if ((rc = launch(e0_place_kernel, dim3(tb), dim3(256), 0, side, p->pdl, 1, e))) return join(rc);
    const int64_t items = (T + kSegRows - 1) / kSegRows * ((D + 255) / 256);  // one warp each
    if ((rc = launch(e0_reduce_kernel, dim3(static_cast<unsigned>((items + 7) / 8)), dim3(256), 0, side, p->pdl, 1, e)))
      return join(rc);
  }
  if (dW) {
    if (fork && cudaStreamWaitEvent(st, p->aux_ev[1], 0) != cudaSuccess) return join(NGRAM_ERR_CUDA);
    // dW += c g^T G: A[m][t] = g[t][m] and B[n][t] = G[t][n], both MN-major as they lie
    // (G gathered row by row into the workspace, above), K = T with split-K units adding
    // into dW.
    DenseParams dp{};
    dp.scale = scale;
    dp.epi = kEpiAccumDense;
    dp.out = dW;
    dp.status = status_ptr(workspace);
    const GemmOperand A{g, D, true}, B{G, D, true};
    if ((rc = p->D % 256 == 0 ? launch_bwd_gemm<256>(p, dp, A, B, T, true, st)
                              : launch_bwd_gemm<128>(p, dp, A, B, T, true, st)))
      return join(rc);
  }
  return join(NGRAM_OK);
}

int ngram_embed_layernorm(const ngram_embed_plan* plan, const void* x, int64_t num_tokens, const float* gamma,
                          const float* beta, float eps, void* y, void* workspace, size_t workspace_bytes,
                          void* stream) {
  int rc = validate_common(plan, workspace, workspace_bytes, 0);
  if (rc) return rc;
  if (num_tokens < 0 || num_tokens > INT32_MAX || !(eps >= 0.0f) || eps > 1.0f) return NGRAM_ERR_INVALID_ARG;
  if (num_tokens == 0) return NGRAM_OK;
  if (!x || !y) return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return NGRAM_ERR_MISALIGNED;
  if ((rc = set_device(plan))) return rc;
  LayerNormParams l{};
  l.x = x;
  l.y = y;
  l.gamma = gamma;
  l.beta = beta;
  l.eps = eps;
  l.T = num_tokens;
  l.D = plan->D;
  constexpr int kRowsPerBlock = 8;  // one warp per row
  const int64_t blocks = (num_tokens + kRowsPerBlock - 1) / kRowsPerBlock;
  return plan->dtype == NGRAM_F32
             ? launch(layernorm_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(32 * kRowsPerBlock), 0,
                      static_cast<cudaStream_t>(stream), plan->pdl, 1, l)
             : launch(layernorm_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(32 * kRowsPerBlock), 0,
                      static_cast<cudaStream_t>(stream), plan->pdl, 1, l);
}

int ngram_embed_plan_set_pdl(ngram_embed_plan* plan, int on) {
  if (!plan || (on != 0 && on != 1)) return NGRAM_ERR_INVALID_ARG;
  plan->pdl = on != 0;
  return NGRAM_OK;
}

int ngram_embed_plan_set_stream_k(ngram_embed_plan* plan, int mode) {
  if (!plan || mode < 0 || mode > 2) return NGRAM_ERR_INVALID_ARG;
  plan->stream_k = mode;
  return NGRAM_OK;
}

size_t ngram_embed_workspace_bytes(const ngram_embed_plan* plan, int64_t max_tokens) {
  if (!plan || max_tokens < 0) return 0;
  return ws_bytes(plan, max_tokens);
}

int ngram_hash_indices(const ngram_embed_plan* plan, const int32_t* tokens, const int32_t* seq_offsets,
                       int32_t num_seqs, int64_t num_tokens, const ngram_cache* cache,
                       const int32_t* cache_slots, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                       void* stream) {
  int rc = validate_common(plan, workspace, workspace_bytes, 0);
  if (rc) return rc;
  if (num_tokens < 0 || num_tokens > INT32_MAX || num_seqs < 0) return NGRAM_ERR_INVALID_ARG;
  if (num_tokens == 0) return NGRAM_OK;
  if (!tokens || !seq_offsets || num_seqs == 0 || (plan->S > 0 && !idx_out)) return NGRAM_ERR_INVALID_ARG;
  if (cache && (rc = validate_cache(plan, cache))) return rc;
  if (plan->S == 0) return NGRAM_OK;
  if ((rc = set_device(plan))) return rc;
  return launch_hash(plan, tokens, seq_offsets, num_seqs, num_tokens, cache, cache_slots, idx_out, workspace,
                     static_cast<cudaStream_t>(stream));
}

int ngram_embed_project(const ngram_embed_plan* plan_c, const int32_t* tokens, const int32_t* idx,
                        int64_t num_tokens, const void* E0, const void* const* E_nk, const void* W_stacked,
                        void* out, void* workspace, size_t workspace_bytes, void* stream) {
  auto* plan = const_cast<ngram_embed_plan*>(plan_c);
  int rc = validate_common(plan, workspace, workspace_bytes, 0);
  if (rc) return rc;
  if (num_tokens < 0 || num_tokens > INT32_MAX) return NGRAM_ERR_INVALID_ARG;
  if (num_tokens == 0) return NGRAM_OK;
  if (!tokens || !out || (plan->S > 0 && !idx)) return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(out)) return NGRAM_ERR_MISALIGNED;
  if ((rc = check_tables(plan, E0, E_nk, W_stacked))) return rc;
  if ((rc = set_device(plan))) return rc;
  return project(plan, tokens, idx, num_tokens, E0, E_nk, W_stacked, out, workspace, workspace_bytes, 0,
                 static_cast<cudaStream_t>(stream));
}

int ngram_embed_fwd(const ngram_embed_plan* plan_c, const int32_t* tokens, const int32_t* seq_offsets,
                    int32_t num_seqs, int64_t num_tokens, const void* E0, const void* const* E_nk,
                    const void* W_stacked, const ngram_cache* cache, const int32_t* cache_slots, void* out,
                    void* workspace, size_t workspace_bytes, void* stream) {
  auto* plan = const_cast<ngram_embed_plan*>(plan_c);
  int rc = validate_common(plan, workspace, workspace_bytes, num_tokens);
  if (rc) return rc;
  if (num_seqs < 0) return NGRAM_ERR_INVALID_ARG;
  if (num_tokens == 0) return NGRAM_OK;
  if (!tokens || !seq_offsets || num_seqs == 0 || !out) return NGRAM_ERR_INVALID_ARG;
  if (!aligned16(out)) return NGRAM_ERR_MISALIGNED;
  if ((rc = check_tables(plan, E0, E_nk, W_stacked))) return rc;
  if (cache && (rc = validate_cache(plan, cache))) return rc;
  if ((rc = set_device(plan))) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* idx = idx_ptr(workspace);
  if (plan->S > 0) {
    rc = launch_hash(plan, tokens, seq_offsets, num_seqs, num_tokens, cache, cache_slots, idx, workspace, st);
    if (rc) return rc;
  }
  return project(plan, tokens, idx, num_tokens, E0, E_nk, W_stacked, out, workspace, workspace_bytes, num_tokens,
                 st);
}

int ngram_embed_fwd_step(const ngram_embed_plan* plan_c, const int32_t* commit_tokens, int32_t commit_stride,
                         const int32_t* commit_counts, const int32_t* tokens, const int32_t* seq_offsets,
                         int32_t num_seqs, int64_t num_tokens, const void* E0, const void* const* E_nk,
                         const void* W_stacked, const ngram_cache* cache, const int32_t* cache_slots, void* out,
                         void* workspace, size_t workspace_bytes, void* stream) {
  auto* plan = const_cast<ngram_embed_plan*>(plan_c);
  int rc = validate_common(plan, workspace, workspace_bytes, num_tokens);
  if (rc) return rc;
  if (num_seqs < 1 || !cache || !tokens || !seq_offsets || (num_tokens > 0 && !out)) return NGRAM_ERR_INVALID_ARG;
  if (commit_counts && (!commit_tokens || commit_stride < 1)) return NGRAM_ERR_INVALID_ARG;
  if (num_tokens > 0 && !aligned16(out)) return NGRAM_ERR_MISALIGNED;
  if ((rc = check_tables(plan, E0, E_nk, W_stacked))) return rc;
  if ((rc = validate_cache(plan, cache))) return rc;
  if (num_seqs > cache->max_seqs && !cache_slots) return NGRAM_ERR_INVALID_ARG;
  if ((rc = set_device(plan))) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* idx = idx_ptr(workspace);
  CacheParams c{};
  c.ring = cache->ring;
  c.len = cache->len;
  c.valid_from = cache->valid_from;
  c.capacity = cache->capacity;
  c.max_seqs = cache->max_seqs;
  c.N = plan->N;
  c.V0 = static_cast<uint32_t>(plan->V0);
  c.slots = cache_slots;
  c.tokens = commit_tokens;
  c.counts = commit_counts;
  c.stride = commit_stride;
  c.n = num_seqs;
  c.status = status_ptr(workspace);
  HashParams h{};
  h.tokens = tokens;
  h.offsets = seq_offsets;
  h.num_seqs = num_seqs;
  h.T = num_tokens;
  h.V0 = static_cast<uint32_t>(plan->V0);
  h.N = plan->N;
  h.K = plan->K;
  h.S = plan->S;
  for (int s = 0; s < plan->S; ++s) {
    h.V[s] = static_cast<uint32_t>(plan->V[s]);
    h.barrett[s] = plan->barrett[s];
  }
  h.ring = cache->ring;
  h.len = cache->len;
  h.valid_from = cache->valid_from;
  h.capacity = cache->capacity;
  h.max_seqs = cache->max_seqs;
  h.slots = cache_slots;
  h.idx_out = idx;
  h.status = status_ptr(workspace);
  const int form = num_tokens > 0 ? choose_form(plan, num_tokens, workspace_bytes, num_tokens, false) : kFormSimt;
  if (form == kFormDense || form == kFormDenseSk || form == kFormDenseWide || form == kFormDenseCols) {
    // commit + hash + the sub-row gather into G in one launch (a block per sequence), then
    // the dense-A projection
    GatherParams g{};
    for (int s = 0; s < plan->S; ++s) {
      g.E[s] = static_cast<const uint8_t*>(E_nk[s]);
      g.Vs[s] = static_cast<uint32_t>(plan->V[s]);
    }
    g.G = static_cast<uint8_t*>(workspace) + dense_g_offset(plan, num_tokens);
    g.T = num_tokens;
    g.S = plan->S;
    g.row_bytes = plan->d * plan->elt;
    int sh = 0;
    while ((1 << sh) < g.row_bytes / 16) ++sh;
    g.vshift = (1 << sh) == g.row_bytes / 16 ? sh : -1;
    g.eshift = -1;
    g.status = status_ptr(workspace);
    if ((rc = launch(commit_hash_gather_kernel, dim3(static_cast<unsigned>(num_seqs)), dim3(256), 0, st, plan->pdl,
                     1, c, h, g)))
      return rc;
    return project(plan, tokens, idx, num_tokens, E0, E_nk, W_stacked, out, workspace, workspace_bytes, num_tokens,
                   st, nullptr, true);
  }
  if ((form == kFormOne || form == kFormOneSk) && plan->fused_step && plan->S <= 8 && num_tokens > 0) {
    // One launch: warps 10-11 of every CTA of the one-CTA projection commit and hash a share
    // of the sequences; its gather warps start once all are done.
    StepHash sh{};
    sh.on = 1;
    sh.c = c;
    sh.h = h;
    sh.ready = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + kStepCountOffset);
    sh.passed = sh.ready + 1;
    return project(plan, tokens, idx, num_tokens, E0, E_nk, W_stacked, out, workspace, workspace_bytes, num_tokens,
                   st, nullptr, false, &sh);
  }
  if ((rc = launch(commit_hash_kernel, dim3(static_cast<unsigned>((num_seqs + 7) / 8)), dim3(256), 0, st,
                   plan->pdl, 1, c, h)))
    return rc;
  if (num_tokens == 0) return NGRAM_OK;
  return project(plan, tokens, idx, num_tokens, E0, E_nk, W_stacked, out, workspace, workspace_bytes, num_tokens,
                 st);
}

int ngram_embed_gather(const ngram_embed_plan* plan, const int32_t* idx, int64_t num_tokens,
                       const void* const* E_nk, void* G_out, const int32_t* tokens, const void* E0,
                       void* E0_out, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_common(plan, workspace, workspace_bytes, 0);
  if (rc) return rc;
  if (num_tokens < 0 || num_tokens > INT32_MAX) return NGRAM_ERR_INVALID_ARG;
  if (num_tokens == 0 || (plan->S == 0 && !E0_out)) return NGRAM_OK;
  if (plan->S > 0 && (!idx || !E_nk || !G_out)) return NGRAM_ERR_INVALID_ARG;
  if (E0_out && (!tokens || !E0)) return NGRAM_ERR_INVALID_ARG;
  if ((G_out && !aligned16(G_out)) || (E0_out && (!aligned16(E0_out) || !aligned16(E0))))
    return NGRAM_ERR_MISALIGNED;
  for (int s = 0; s < plan->S; ++s) {
    if (!E_nk[s]) return NGRAM_ERR_INVALID_ARG;
    if (!aligned16(E_nk[s])) return NGRAM_ERR_MISALIGNED;
  }
  if ((rc = set_device(plan))) return rc;
  return launch_gather(plan, idx, num_tokens, E_nk, G_out, tokens, E0, E0_out, workspace,
                       static_cast<cudaStream_t>(stream));
}

static int cache_launch(const ngram_embed_plan* plan, const ngram_cache* cache, const int32_t* slots,
                        const int32_t* tokens, const int32_t* tok_offsets, const int32_t* counts, int32_t n,
                        void* workspace, size_t workspace_bytes, void* stream, int which, int32_t stride = 0) {
  int rc = validate_common(plan, workspace, workspace_bytes, 0);
  if (rc) return rc;
  if (!cache || n < 0) return NGRAM_ERR_INVALID_ARG;
  if ((rc = validate_cache(plan, cache))) return rc;
  if (n == 0) return NGRAM_OK;
  if (which == 1 && (!tokens || !tok_offsets)) return NGRAM_ERR_INVALID_ARG;
  if (which == 3 && (!tokens || !counts || stride < 1)) return NGRAM_ERR_INVALID_ARG;
  if (which == 2 && !counts) return NGRAM_ERR_INVALID_ARG;
  if ((rc = set_device(plan))) return rc;
  CacheParams c{};
  c.ring = cache->ring;
  c.len = cache->len;
  c.valid_from = cache->valid_from;
  c.capacity = cache->capacity;
  c.max_seqs = cache->max_seqs;
  c.N = plan->N;
  c.V0 = static_cast<uint32_t>(plan->V0);
  c.slots = slots;
  c.tokens = tokens;
  c.tok_offsets = tok_offsets;
  c.counts = counts;
  c.stride = stride;
  c.n = n;
  c.status = status_ptr(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (which == 0) return launch(cache_reset_kernel, dim3((n + 255) / 256), dim3(256), 0, st, plan->pdl, 1, c);
  if (which == 1 || which == 3)
    return launch(cache_append_kernel, dim3((n + 7) / 8), dim3(256), 0, st, plan->pdl, 1, c);
  return launch(cache_rollback_kernel, dim3((n + 255) / 256), dim3(256), 0, st, plan->pdl, 1, c);
}

int ngram_cache_reset(const ngram_embed_plan* plan, const ngram_cache* cache, const int32_t* slots, int32_t n,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return cache_launch(plan, cache, slots, nullptr, nullptr, nullptr, n, workspace, workspace_bytes, stream, 0);
}

int ngram_cache_append(const ngram_embed_plan* plan, const ngram_cache* cache, const int32_t* slots,
                       const int32_t* tokens, const int32_t* tok_offsets, int32_t n, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return cache_launch(plan, cache, slots, tokens, tok_offsets, nullptr, n, workspace, workspace_bytes, stream, 1);
}

int ngram_cache_commit(const ngram_embed_plan* plan, const ngram_cache* cache, const int32_t* slots,
                       const int32_t* tokens, int32_t stride, const int32_t* counts, int32_t n, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return cache_launch(plan, cache, slots, tokens, nullptr, counts, n, workspace, workspace_bytes, stream, 3, stride);
}

int ngram_cache_rollback(const ngram_embed_plan* plan, const ngram_cache* cache, const int32_t* slots,
                         const int32_t* counts, int32_t n, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return cache_launch(plan, cache, slots, nullptr, nullptr, counts, n, workspace, workspace_bytes, stream, 2);
}

int ngram_embed_selftest_wait_timeout(void* workspace, int64_t limit_ns, void* stream) {
  if (!workspace || limit_ns <= 0 || limit_ns > 2000000000LL) return NGRAM_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return NGRAM_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status_ptr(workspace),
                                                                         static_cast<uint64_t>(limit_ns));
  return check_launch();
}

int ngram_embed_get_status(const void* workspace, void* stream, int32_t* status_out) {
  if (!workspace || !status_out) return NGRAM_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status_out, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return NGRAM_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? NGRAM_OK : NGRAM_ERR_CUDA;
}

int ngram_embed_clear_status(void* workspace, void* stream) {
  if (!workspace) return NGRAM_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, kHeadBytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? NGRAM_OK
             : NGRAM_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Forward pass with library-owned scratch, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: plugin hosts that hand a layer only its input and
// output buffers, and latency-critical loops where cudaMalloc's implicit device-wide
// synchronisation is not allowed. ngram_embed_fwd_static_ws runs the same forward pass as
// ngram_embed_fwd, but its workspace (the head with the status word and the stream-K
// arrival counters, the per-token index buffer and, when they fit, the stream-K partial
// tiles) is the fixed array below, compiled into the library. Every GPU that loads the
// library holds these kNoAllocScratchBytes until the process exits.
//
// In host code `g_noalloc_scratch` names a host-side stand-in, not a device address, so the
// array's device address is looked up with cudaGetSymbolAddress once per device, with that
// device current, by the first call made on that device (that first call should come
// before any stream capture). A failed lookup is not remembered: the next call tries again.
// All calls share the array and it keeps the last call's contents: each call zeroes the
// whole head (status word and arrival counters, which a call that stopped at a bounded-wait
// timeout may leave non-zero) before use, and calls that overlap on the GPU (concurrent
// streams) race on the array.
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// The array's device address on `device` (current), or nullptr if the lookup failed.
void* noalloc_scratch(int device) {
  if (device < 0 || device >= kNoAllocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) {
      g_noalloc_ptr[device] = p;
    } else {
      cudaGetLastError();  // clear the error; a later call retries the lookup
    }
  }
  return g_noalloc_ptr[device];
}

}  // namespace

extern "C" int ngram_embed_fwd_static_ws(const ngram_embed_plan* plan, const int32_t* tokens,
                                         const int32_t* seq_offsets, int32_t num_seqs, int64_t num_tokens,
                                         const void* E0, const void* const* E_nk, const void* W_stacked,
                                         const ngram_cache* cache, const int32_t* cache_slots, void* out,
                                         int32_t* status_out, void* stream) {
  if (!plan || num_tokens < 0 || num_tokens > INT32_MAX) return NGRAM_ERR_INVALID_ARG;
  if (ws_base(plan, num_tokens) > kNoAllocScratchBytes) return NGRAM_ERR_WORKSPACE;  // above the fixed limit
  int rc = set_device(plan);
  if (rc) return rc;
  void* ws = noalloc_scratch(plan->device);
  if (!ws) return NGRAM_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, kHeadBytes, st) != cudaSuccess) return NGRAM_ERR_CUDA;  // status word + counters
  rc = ngram_embed_fwd(plan, tokens, seq_offsets, num_seqs, num_tokens, E0, E_nk, W_stacked, cache, cache_slots,
                       out, ws, kNoAllocScratchBytes, stream);
  if (rc) return rc;
  if (status_out &&
      cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return NGRAM_ERR_CUDA;
  return NGRAM_OK;
}
