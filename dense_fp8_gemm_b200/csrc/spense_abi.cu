// Host side of the Spense C ABI: argument validation, the packed handle,
// launch planning (tile, token padding, stream-K grid, pipeline depth), the
// activation tensor map, and the workspace layout.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include <cudaTypedefs.h>

#include "spense_internal.h"

using namespace spense;

struct spense_packed {
  uint64_t id = 0;  // unique for the life of the process (keys the launch cache)
  int device = -1;
  int64_t N = 0, K = 0, Ks = 0, Kd = 0;
  int n_tiles = 0, nsb = 0, ndb = 0;
  uint8_t* vs_t = nullptr;
  uint8_t* e_t = nullptr;
  uint8_t* wd_t = nullptr;
  float* s_w = nullptr;
  int32_t* perm = nullptr;
  std::vector<int32_t> perm_host;  // same order on the host (empty for the tail)
  uint8_t* vs_c = nullptr;
  uint8_t* e_c = nullptr;
  uint8_t* wd_c = nullptr;
};

namespace {

thread_local std::string g_last_error;

spense_status fail(spense_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

spense_status ok() {
  g_last_error.clear();
  return SPENSE_OK;
}

spense_status cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaErrorMemoryAllocation)
    return fail(SPENSE_ERR_OOM, "%s: %s", what, cudaGetErrorString(e));
  return fail(SPENSE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DeviceInfo {
  int major = 0;
  int sms = 0;
};

// Current device's capability and SM count (cached per device).
spense_status current_device(int* dev, DeviceInfo* info) {
  static std::mutex mu;
  static std::vector<DeviceInfo> cache;
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail(SPENSE_ERR_UNSUPPORTED, "no CUDA device: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(mu);
  if (static_cast<int>(cache.size()) <= *dev) cache.resize(*dev + 1);
  DeviceInfo& d = cache[*dev];
  if (d.sms == 0) {
    if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess) {
      d.sms = 0;
      return fail(SPENSE_ERR_UNSUPPORTED, "cannot query device %d", *dev);
    }
  }
  *info = d;
  if (d.major != 10)
    return fail(SPENSE_ERR_UNSUPPORTED, "device %d has compute capability %d.x; sm_100 is required",
                *dev, d.major);
  return SPENSE_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

void free_handle(spense_packed* h) {
  if (h == nullptr) return;
  for (void* p : {static_cast<void*>(h->vs_t), static_cast<void*>(h->e_t), static_cast<void*>(h->wd_t),
                  static_cast<void*>(h->s_w), static_cast<void*>(h->perm), static_cast<void*>(h->vs_c),
                  static_cast<void*>(h->e_c), static_cast<void*>(h->wd_c)})
    if (p != nullptr) cudaFree(p);
  delete h;
}

// Minimum streamed weight per CTA in 4 KiB units (default 20 = four 2:4 blocks);
// SPENSE_MIN_CTA_WEIGHT overrides it for tuning.
long long min_cta_weight() {
  static const long long v = [] {
    const char* e = std::getenv("SPENSE_MIN_CTA_WEIGHT");
    long long x = e ? std::atoll(e) : 20;
    return x > 0 ? x : 20;
  }();
  return v;
}

// Tuning knobs read once from the environment: CTAs per SM (1, 2 or 0 =
// automatic), weight-loader warps per CTA (1 or 2, default 2; one more warp
// loads the activation tiles) and how many bulk copies move one 16 KiB weight
// block (1, 2 or 4, default 1). One SM's copy engine serves several issue
// streams at once but one stream's copies one after another, so two CTAs
// with two weight loaders each keep four weight streams going per SM; a
// single CTA with a ring twice as deep does as well on long GEMMs.
int env_int(const char* name, int dflt, int lo, int hi) {
  const char* e = std::getenv(name);
  if (e == nullptr) return dflt;
  const int v = std::atoi(e);
  return (v < lo || v > hi) ? dflt : v;
}
// 0 (default) = automatic: one CTA per SM with a deep ring when the launch has
// more row tiles than two-per-SM CTA slots (large GEMMs, stream-K) or more
// than 32 tokens (the activation tile then fills half of every ring stage),
// two per SM otherwise (short decode GEMMs, where a second CTA per SM hides
// the fixed costs).
int ctas_per_sm_knob() {
  static const int v = env_int("SPENSE_CTAS_PER_SM", 0, 0, 2);
  return v;
}
// CTA slots per SM that one grid may fill (default: all of them); 1 leaves
// room for the next grid in the stream to start beside this one.
int grid_per_sm() {
  static const int v = env_int("SPENSE_GRID_PER_SM", 2, 1, 2);
  return v;
}
// Weight blocks per CTA, past the first ring's worth, prefetched into L2 at
// start; -1 (default) = automatic: 4 for cluster-split launches (few tiles;
// the prefetch overlaps the previous grid's tail: attn32b decode step 0.505
// -> 0.524 of HBM), none for stream-K launches (gate+up 33.5 -> 34.5 us with 8).
int l2_prefetch_knob() {
  static const int v = env_int("SPENSE_L2_PREFETCH", -1, -1, 1 << 20);
  return v;
}
// L2 prefetch depth of a planned launch (see l2_prefetch_knob).
int l2_prefetch_for(const GemmPlan& pl) {
  return l2_prefetch_knob() >= 0 ? l2_prefetch_knob() : (pl.cluster > 1 ? 4 : 0);
}
// Tokens per token tile (multiple of 16, at most 256); 0 (default) =
// automatic (see make_plan).
int token_tile_knob() {
  static const int v = [] {
    const int x = env_int("SPENSE_TOKEN_TILE", 0, 0, kMaxTokenTile);
    return x % 16 == 0 ? x : 0;
  }();
  return v;
}
// 1 (default): a warp of its own issues the activation-tile loads; 0: the
// weight loaders issue them after the weight copies.
int x_warp() {
  static const int v = env_int("SPENSE_X_WARP", 1, 0, 1);
  return v;
}
int producers() {
  static const int v = env_int("SPENSE_PRODUCERS", 2, 1, 2);
  return v;
}
// SPENSE_CLUSTER: 0 = stream-K only, 1 = automatic (default), 2/4/8 = that
// cluster size whenever it fits.
int cluster_mode() {
  static const int v = env_int("SPENSE_CLUSTER", 1, 0, 8);
  return v;
}

// SPENSE_W_KEEP: -1 (default) = automatic (weights keep the evict-normal L2
// policy when several token tiles re-read them: down 5120x27648 at 256 tokens
// 65.2 -> 63.9 us), 0 = always stream them evict-first, 1 = always keep.
int w_keep_knob() {
  static const int v = env_int("SPENSE_W_KEEP", -1, -1, 1);
  return v;
}

// SPENSE_PAIR: 0 (default) = never use CTA pairs; 1 = pairs for more than 64
// tokens; 2 = pairs whenever the layout allows. Pairs are correct but were
// measured slower than single CTAs on every shape of the workloads (gate+up
// 55296x5120 at 256 tokens 121 vs 95 us, at 64 tokens 70 vs 40 us): with 256
// tokens only one accumulator fits in tensor memory, so each tile's epilogue
// stalls the MMAs, and at 64 tokens the halved activation boxes (4 KiB) keep
// many small copies in flight (5.5 us from issue to landing vs 1.5 us).
int pair_knob() {
  static const int v = env_int("SPENSE_PAIR", 0, 0, 2);
  return v;
}

// SPENSE_PAIRS_MAX: at most this many CTA pairs per launch (0 = automatic).
int pairs_max_knob() {
  static const int v = env_int("SPENSE_PAIRS_MAX", 0, 0, kMaxGrid);
  return v;
}

int bulk_split() {
  static const int v = [] {
    const int x = env_int("SPENSE_BULK_SPLIT", 1, 1, 4);
    return x == 3 ? 1 : x;
  }();
  return v;
}

// Checks that `count` handles can share one launch and plans it for M tokens
// on a device with `sms` SMs. Members share the device, K and the column order
// of X: either none has a scattered dense set (their Kd may differ, e.g. the
// 2:4 rows and the dense rows of an output-split weight), or all have the
// same one.
// t_force: token tile to plan with (0: automatic; SPENSE_TOKEN_TILE overrides both).
spense_status make_plan_t(const spense_packed* const* hs, int count, int64_t M, int sms, int t_force,
                          GemmPlan* out) {
  if (hs == nullptr || count < 1 || count > kMaxGroup)
    return fail(SPENSE_ERR_ARG, "a launch takes 1 to %d packed weights, got %d", kMaxGroup, count);
  if (M < 1 || M > 65535) return fail(SPENSE_ERR_SHAPE, "M = %lld outside [1, 65535]", (long long)M);
  const spense_packed* h0 = hs[0];
  if (h0 == nullptr) return fail(SPENSE_ERR_ARG, "Wp is NULL");
  GemmPlan pl{};
  long long row_tiles = 0, weight_units = 0;
  for (int i = 0; i < count; ++i) {
    if (hs[i] == nullptr) return fail(SPENSE_ERR_ARG, "packed weight %d is NULL", i);
    row_tiles += hs[i]->n_tiles;
    weight_units += static_cast<long long>(hs[i]->n_tiles) * (kCostSparse * hs[i]->nsb + kCostDense * hs[i]->ndb);
  }
  // Token tile T: all tokens in one tile up to T, else tiles of T tokens. The
  // CTAs of neighbouring token tiles stream the same weight rows at about the
  // same time, so the repeat reads hit L2. 64 tokens while the tiles of 64
  // fit one per SM (they then split over clusters), or two per SM for a
  // weight of at most 32 MB (its repeat reads stay in L2); 128 otherwise,
  // which halves the repeat reads and gives each CTA longer whole tiles.
  const long long tiles64 = row_tiles * ((M + 63) / 64);
  const bool small_weight = weight_units * 4096ll <= (32ll << 20);  // cost units are 4 KiB
  // Pair mode (opt-in, see pair_knob): two CTAs on two SMs share one MMA of
  // 256 weight rows (tcgen05 cta_group::2), each holding half of the token
  // tile, so every activation byte staged in shared memory serves twice the
  // weight rows, and token tiles of up to 256 tokens read each weight once.
  const int pk = pair_knob();
  pl.pair = (x_warp() && (pk == 2 || (pk == 1 && M > 64))) ? 1 : 0;
  int T = token_tile_knob() != 0 ? token_tile_knob()
          : t_force != 0          ? t_force
          : (pl.pair ? kMaxTokenTile
                     : ((tiles64 <= sms || (tiles64 <= 2LL * sms && small_weight)) ? 64 : 128));
  // Tiles of 128 tokens that leave most CTAs straddling two tiles (fewer than
  // 1.5 tiles per SM) while tiles of 96 would give each about two: take 96
  // (q/k/v 12288x5120 at 256 tokens 35.3 -> 28.4 us; weights that stay at
  // fewer than 1.5 tiles per SM either way were slower with 96). Only for a
  // weight of at most 64 MB, whose re-reads by the extra token tile stay in L2.
  if (token_tile_knob() == 0 && !pl.pair && T == 128 && M > 128 && weight_units * 4096ll <= (64ll << 20)) {
    const long long t128 = row_tiles * ((M + 127) / 128), t96 = row_tiles * ((M + 95) / 96);
    if (2 * t128 < 3LL * sms && 2 * t96 >= 3LL * sms) T = 96;
  }
  pl.npad = M > T ? T : static_cast<int>(round_up(static_cast<size_t>(M), 16));
  // rows one activation box loads: the valid rows of the token tile, or in
  // pair mode this CTA's half of it (rows past M read as zeros)
  pl.box_rows = pl.pair ? pl.npad / 2 : static_cast<int>(M > T ? T : M);
  pl.m_tiles = static_cast<int>((M + T - 1) / T);
  pl.count = count;
  long long n_tiles = 0, blocks = 0, cost = 0;
  pl.min_tile_cost = 1 << 30;
  pl.any_sparse = false;
  for (int i = 0; i < count; ++i) {
    const spense_packed* h = hs[i];
    if (h->device != h0->device || h->K != h0->K || h->perm_host != h0->perm_host)
      return fail(SPENSE_ERR_ARG,
                  "packed weights sharing a launch need the same device, K and column order of X (the same "
                  "scattered dense set, or none)");
    // work tiles of member i: its 128-row tiles, or in pair mode pairs of them
    const int ut = pl.pair ? (h->n_tiles + 1) / 2 : h->n_tiles;
    pl.mem_tiles[i] = ut;
    pl.mem_nsb[i] = h->nsb;
    pl.mem_ndb[i] = h->ndb;
    pl.mem_cost[i] = kCostSparse * h->nsb + kCostDense * h->ndb;
    pl.mem_block_begin[i] = static_cast<int>(std::min<long long>(blocks, 1ll << 31));
    pl.mem_cost_begin[i] = cost;
    const long long tiles_i = static_cast<long long>(ut) * pl.m_tiles;
    blocks += tiles_i * (h->nsb + h->ndb);
    cost += tiles_i * pl.mem_cost[i];
    n_tiles += ut;
    pl.min_tile_cost = std::min(pl.min_tile_cost, pl.mem_cost[i]);
    pl.any_sparse = pl.any_sparse || h->nsb > 0;
  }
  pl.mem_cost_begin[count] = cost;
  if (blocks >= (1ll << 31)) return fail(SPENSE_ERR_SHAPE, "too many blocks for one launch (%lld)", blocks);
  pl.n_tiles = static_cast<int>(n_tiles);
  pl.tiles = pl.n_tiles * pl.m_tiles;
  pl.total_cost = cost;
  // Each CTA gets at least min_cta_weight() units of streamed bytes (never less
  // than one maximal block, so no CTA owns an empty range): small matrices are
  // split across fewer CTAs, which keeps the number of partials per tile low.
  long long grid = pl.total_cost / std::max<long long>(kCostSparse, min_cta_weight());
  pl.bulk_split = bulk_split();
  pl.producers = producers();
  pl.b_bytes = static_cast<uint32_t>(pl.pair ? pl.npad / 2 : pl.npad) * (pl.any_sparse ? 256u : 128u);
  pl.stage_bytes = kBlockBytes + pl.b_bytes + (pl.any_sparse ? kMetaBlockBytes : 0);
  const uint32_t reserve = 1024 + kBarrierBytes;  // alignment slack + barrier area
  // Ring and TMEM for `cps` CTAs per SM; false if two stages or the
  // accumulators do not fit.
  auto fit_ring = [&](int cps, uint32_t recv, int* stages, int* nacc, uint32_t* cols) {
    const uint32_t smem_budget = gemm_max_smem() / cps - (cps > 1 ? 1024u : 0u);
    const uint32_t tmem_budget = 512u / cps;
    if (smem_budget < reserve + recv + 2 * pl.stage_bytes) return false;
    *stages = static_cast<int>(std::min<uint32_t>(kMaxStages, (smem_budget - reserve - recv) / pl.stage_bytes));
    *nacc = (2u * pl.npad + 16u <= tmem_budget) ? 2 : 1;
    *cols = 32;
    while (*cols < static_cast<uint32_t>(*nacc * pl.npad + 16)) *cols <<= 1;
    return *cols <= tmem_budget;
  };
  auto slots_for = [&](int cps) {
    if (pl.pair)  // one pair per two SMs
      return std::min<long long>(pairs_max_knob() > 0 ? pairs_max_knob() : sms / 2, kMaxGrid);
    return std::min<long long>(static_cast<long long>(sms) * std::min(cps, grid_per_sm()), kMaxGrid);
  };
  // Few tiles (at most half the CTA slots): the CTAs of a cluster of S split
  // each tile's K range by weight and reduce in shared memory; otherwise
  // stream-K over all tiles with the global fix-up. Cluster sizes are powers
  // of two (a grid of clusters of 7 did not fit in one wave); the cluster
  // grid must fit the CTA slots and fill at least half of them, unless the
  // GEMM is so small that fixed costs dominate anyway, and rank 0's receive
  // area (S - 1 partials of 128 rows x npad floats) comes out of the ring.
  // Returns the largest such S for `cps` CTAs per SM, or 1.
  const int mode = cluster_mode();
  int max_blocks = 0;  // blocks per tile of the member with the longest K
  for (int i = 0; i < count; ++i) max_blocks = std::max(max_blocks, pl.mem_nsb[i] + pl.mem_ndb[i]);
  auto cluster_for = [&](int cps) {
    const long long slots = slots_for(cps);
    if (mode == 0 || pl.tiles * 2 > slots || pl.npad > 64) return 1;
    for (int S = 8; S >= 2; S >>= 1) {
      if (mode > 1 && S != mode) continue;
      if (pl.tiles * S > slots || S > pl.min_tile_cost / kCostSparse) continue;
      const bool fills = pl.tiles * S * 2 >= slots;
      const bool small = pl.total_cost < 40LL * slots;
      if (!(mode > 1 || fills || small)) continue;
      int st, na;
      uint32_t co;
      if (!fit_ring(cps, static_cast<uint32_t>(S - 1) * kTileRows * pl.npad * 4u, &st, &na, &co)) continue;
      // A two-stage ring only pays when each CTA streams few blocks: q_proj
      // 8192x5120 at 128 tokens (about 13 blocks per CTA) 42.5 -> 16.1 us
      // with it, but down 5120x27648 at 128 tokens (about 67 per CTA) took
      // 53.8 us against 40.7 us as stream-K with a deep ring.
      if (st < 3 && max_blocks > 16 * S) continue;
      // Clusters that leave over 40 % of the SMs idle lose to stream-K over
      // all of them when each clustered CTA would stream a long K range:
      // down 5120x27648 (135 blocks per tile, clusters of 2 on 80 SMs) at 32
      // and 64 tokens 30.8 -> 24.5 us and 32.6 -> 27.3 us as stream-K; o_proj
      // 5120x10240 (50 blocks per tile) stays faster in clusters.
      if (10LL * pl.tiles * S < 6LL * sms && max_blocks > 32 * S) continue;
      return S;
    }
    return 1;
  };
  // CTAs per SM: two (two independent copy streams that hide each other's
  // fixed costs) when the launch has at most two row tiles per SM and the
  // token tile is at most 32 tokens, else one with a deeper ring. A launch
  // that cannot split its tiles over clusters at that count but can at the
  // other count takes the other.
  const int knob = ctas_per_sm_knob();
  int cps = knob != 0 ? knob : ((pl.tiles > 2 * sms || pl.npad > 32) ? 1 : 2);
  if (pl.pair) {
    // pairs: one CTA per SM with the whole ring, stream-K over pair tiles
    cps = 1;
    pl.cluster = 1;
  } else {
    pl.cluster = cluster_for(cps);
    if (pl.cluster == 1 && knob == 0 && cluster_for(3 - cps) > 1) {
      cps = 3 - cps;
      pl.cluster = cluster_for(cps);
    }
    // Few long tiles left to stream-K: one CTA per SM with a deeper ring and
    // half the partials (down 5120x27648 at 32 tokens 24.5 us against 25.1 us
    // at two per SM).
    if (pl.cluster == 1 && knob == 0 && 10LL * pl.tiles < 6LL * sms && max_blocks > 64) cps = 1;
  }
  pl.recv_bytes = pl.cluster > 1 ? static_cast<uint32_t>(pl.cluster - 1) * kTileRows * pl.npad * 4u : 0u;
  if (!fit_ring(cps, pl.recv_bytes, &pl.stages, &pl.nacc, &pl.tmem_cols)) {
    // Stream-K (no receive area) and two CTAs per SM that do not fit: one.
    cps = 1;
    if (!fit_ring(cps, 0, &pl.stages, &pl.nacc, &pl.tmem_cols))
      return fail(SPENSE_ERR_SHAPE, "token tile of %d does not fit one CTA", pl.npad);
  }
  pl.ctas_per_sm = cps;
  const long long slots = slots_for(cps);
  // First block of a tile of member i whose start weight is >= c (c within one tile).
  auto block_at = [&](int i, long long c) {
    const long long sp = static_cast<long long>(kCostSparse) * pl.mem_nsb[i];
    return c <= sp ? (c + kCostSparse - 1) / kCostSparse : pl.mem_nsb[i] + (c - sp + kCostDense - 1) / kCostDense;
  };
  // Member of global tile t (tiles of a member are consecutive).
  auto member_of_tile = [&](long long t) {
    int i = 0;
    long long acc = 0;
    for (; i < count - 1; ++i) {
      acc += static_cast<long long>(pl.mem_tiles[i]) * pl.m_tiles;
      if (t < acc) break;
    }
    return i;
  };
  // First linear block of global tile t.
  auto tile_block0 = [&](long long t) {
    const int i = member_of_tile(t);
    long long first_tile = 0;
    for (int k = 0; k < i; ++k) first_tile += static_cast<long long>(pl.mem_tiles[k]) * pl.m_tiles;
    return pl.mem_block_begin[i] + (t - first_tile) * (pl.mem_nsb[i] + pl.mem_ndb[i]);
  };
  if (pl.cluster > 1) {
    pl.grid = pl.tiles * pl.cluster;
    for (int g = 0; g <= pl.grid; ++g) {
      const long long t = g / pl.cluster, r = g % pl.cluster;
      if (t >= pl.tiles) {
        pl.cta_start[g] = static_cast<int>(blocks);
        continue;
      }
      const int i = member_of_tile(t);
      pl.cta_start[g] = static_cast<int>(tile_block0(t) + block_at(i, (r * pl.mem_cost[i] + pl.cluster - 1) /
                                                                             pl.cluster));
    }
  } else {
    grid = std::max<long long>(1, std::min<long long>(grid, slots));
    pl.grid = static_cast<int>(grid);
    // CTA g takes the blocks whose start weight falls in [g T / G, (g+1) T / G).
    for (int g = 0; g <= pl.grid; ++g) {
      const long long c = (static_cast<long long>(g) * pl.total_cost + pl.grid - 1) / pl.grid;
      if (c >= pl.total_cost) {
        pl.cta_start[g] = static_cast<int>(blocks);
        continue;
      }
      int i = 0;
      while (i + 1 < count && c >= pl.mem_cost_begin[i + 1]) ++i;
      const long long ci = c - pl.mem_cost_begin[i];
      const long long tl = ci / pl.mem_cost[i];  // tile within member i
      pl.cta_start[g] = static_cast<int>(pl.mem_block_begin[i] + tl * (pl.mem_nsb[i] + pl.mem_ndb[i]) +
                                         block_at(i, ci - tl * pl.mem_cost[i]));
    }
  }
  // Output staging for the stream-K epilogue's whole tiles (16-byte stores),
  // when the ring leaves room for it.
  {
    const uint32_t budget = gemm_max_smem() / pl.ctas_per_sm - (pl.ctas_per_sm > 1 ? 1024u : 0u);
    const uint32_t used = reserve + static_cast<uint32_t>(pl.stages) * pl.stage_bytes + pl.recv_bytes;
    pl.ystage = (pl.cluster == 1 && used + kYStageBytes <= budget) ? kYStageBytes : 0u;
  }
  pl.smem_bytes = reserve + static_cast<uint32_t>(pl.stages) * pl.stage_bytes + pl.recv_bytes + pl.ystage;
  WorkspaceLayout& w = pl.ws;
  size_t off = 256;  // header: status word
  w.counters_off = off;
  const int ctas_per_unit = pl.pair ? 2 : 1;
  // one arrival counter per CTA tile (in pair mode each CTA of a pair tile counts its own rows)
  w.counters_bytes = round_up(static_cast<size_t>(pl.tiles) * ctas_per_unit * 4, 256);
  off += w.counters_bytes;
  w.partials_off = off;
  // fp32 partials of shared tiles: stream-K only (a cluster reduces in shared memory)
  w.partials_bytes =
      pl.cluster > 1 ? 0 : static_cast<size_t>(pl.grid) * ctas_per_unit * 2 * pl.npad * kTileRows * 4;
  off += w.partials_bytes;
  w.xg_off = off;
  w.xg_bytes = h0->perm ? round_up(static_cast<size_t>(M * h0->K), 256) : 0;
  off += w.xg_bytes;
  w.total_device = off;
  w.stage_x_off = off;
  off += round_up(static_cast<size_t>(M * h0->K), 256);
  w.stage_sx_off = off;
  off += round_up(static_cast<size_t>(M) * 4, 256);
  w.stage_y_off = off;
  for (int i = 0; i < count; ++i) off += round_up(static_cast<size_t>(M * hs[i]->N) * 2, 256);
  w.total_host = off;
  *out = pl;
  return SPENSE_OK;
}

spense_status make_plan(const spense_packed* const* hs, int count, int64_t M, int sms, GemmPlan* out) {
  const spense_status st = make_plan_t(hs, count, M, sms, 0, out);
  if (st != SPENSE_OK) return st;
  // Tiles of 64 tokens are chosen above 64 tokens so that the tiles can split
  // over clusters; when no cluster split fits (long tiles, see cluster_for),
  // tiles of 128 tokens halve the weight re-reads instead: down 5120x27648 at
  // 128 tokens 38.6 -> 30.2 us, o_proj 5120x10240 21.6 -> 21.2 us.
  if (token_tile_knob() == 0 && !out->pair && out->npad == 64 && M > 64 && out->cluster == 1 &&
      static_cast<long long>(out->n_tiles) * ((M + 63) / 64) <= sms)
    return make_plan_t(hs, count, M, sms, 128, out);
  return SPENSE_OK;
}

// Validates the call-level arguments shared by the GEMM entry points.
spense_status check_gemm_args(const spense_packed* const* hs, int count, int64_t M, void* workspace,
                              DeviceInfo* info) {
  if (hs == nullptr || count < 1 || count > kMaxGroup || hs[0] == nullptr)
    return fail(SPENSE_ERR_ARG, "Wp is NULL");
  if (M < 1 || M > 65535) return fail(SPENSE_ERR_SHAPE, "M = %lld outside [1, 65535]", (long long)M);
  if (workspace == nullptr) return fail(SPENSE_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(SPENSE_ERR_ALIGN, "workspace is not 256-byte aligned");
  int dev = 0;
  spense_status st = current_device(&dev, info);
  if (st != SPENSE_OK) return st;
  if (dev != hs[0]->device)
    return fail(SPENSE_ERR_ARG, "handle was packed on device %d, current device is %d", hs[0]->device, dev);
  return SPENSE_OK;
}

// Everything one launch needs, computed once per distinct call (see the
// launch cache in spense_gemm_grouped_ex).
struct PreparedLaunch {
  CUtensorMap map;
  GemmParams p;
  uint32_t smem = 0;
  const uint8_t* gather_src = nullptr;  // SpenseGPT+ gather into gather_dst first, when set
  const int32_t* perm = nullptr;
  uint8_t* gather_dst = nullptr;
  int64_t M = 0, K = 0;
};

// Builds the launch over `count` packed weights sharing X (arguments validated).
spense_status prepare_gemm(const spense_packed* const* hs, int count, const uint8_t* X, const float* x_scale,
                           int64_t M, uint16_t* const* Ys, uint8_t* ws, const GemmPlan& pl, bool x_packed_order,
                           const int64_t* ldy, PreparedLaunch* out) {
  const spense_packed* h0 = hs[0];
  const uint8_t* xsrc = X;
  out->gather_src = nullptr;
  if (h0->perm != nullptr && !x_packed_order) {
    out->gather_src = X;
    out->perm = h0->perm;
    out->gather_dst = ws + pl.ws.xg_off;
    out->M = M;
    out->K = h0->K;
    xsrc = out->gather_dst;
  }
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return fail(SPENSE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap& map = out->map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(h0->K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(h0->K)};
  const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(pl.box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(xsrc), dims, strides,
                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SPENSE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);

  GemmParams& p = out->p;
  p = GemmParams{};
  int tile_begin = 0;
  for (int i = 0; i < count; ++i) {
    GemmMember& m = p.mem[i];
    m.vs_t = hs[i]->vs_t;
    m.e_t = hs[i]->e_t;
    m.wd_t = hs[i]->wd_t;
    m.s_w = hs[i]->s_w;
    m.y = Ys[i];
    m.N = static_cast<int>(hs[i]->N);
    m.tile_begin = tile_begin;
    m.nsb = pl.mem_nsb[i];
    m.ndb = pl.mem_ndb[i];
    m.nblk = m.nsb + m.ndb;
    m.Ks = static_cast<int>(hs[i]->Ks);
    m.block_begin = pl.mem_block_begin[i];
    m.ldy = static_cast<int>(ldy != nullptr ? ldy[i] : hs[i]->N);
    m.row_tiles = hs[i]->n_tiles;
    tile_begin += pl.mem_tiles[i];
  }
  p.n_members = count;
  p.s_x = x_scale;
  p.partials = reinterpret_cast<float*>(ws + pl.ws.partials_off);
  p.counters = reinterpret_cast<unsigned int*>(ws + pl.ws.counters_off);
  p.status = reinterpret_cast<unsigned int*>(ws);
  p.M = static_cast<int>(M);
  p.n_tiles = pl.n_tiles;
  p.m_tiles = pl.m_tiles;
  p.npad = pl.npad;
  p.box_rows = pl.box_rows;
  p.grid = pl.grid;
  p.stages = pl.stages;
  p.nacc = pl.nacc;
  p.stage_bytes = pl.stage_bytes;
  p.b_bytes = pl.b_bytes;
  p.tmem_cols = pl.tmem_cols;
  std::memcpy(p.cta_start, pl.cta_start, sizeof(int) * (pl.grid + 1));
  p.bulk_split = pl.bulk_split;
  p.producers = pl.producers;
  p.cluster = pl.cluster;
  p.recv_bytes = pl.recv_bytes;
  p.l2_prefetch = l2_prefetch_for(pl);
  p.x_warp = x_warp();
  p.w_keep = w_keep_knob() >= 0 ? w_keep_knob() : (pl.m_tiles > 1 ? 1 : 0);
  p.pair = pl.pair;
  p.ystage = pl.ystage;
#ifdef SPENSE_TEST_HOOKS
  // Test build only: with SPENSE_TEST_STALL=1 the loaders wait on header word
  // 16 of the workspace, which nothing sets, so every launch ends by timeout.
  static const bool stall = env_int("SPENSE_TEST_STALL", 0, 0, 1) == 1;
  p.test_gate = stall ? reinterpret_cast<const unsigned int*>(ws + 64) : nullptr;
#else
  p.test_gate = nullptr;
#endif
  out->smem = pl.smem_bytes;
  return SPENSE_OK;
}

spense_status enqueue_gemm(const PreparedLaunch& L, cudaStream_t stream) {
  if (L.gather_src != nullptr) {
    cudaError_t e = launch_gather(L.gather_src, L.perm, L.M, L.K, L.gather_dst, stream);
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  }
  cudaError_t e = launch_gemm(L.map, L.p, L.smem, stream);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return SPENSE_OK;
}

// Enqueue one launch over `count` packed weights sharing X (arguments validated).
spense_status run_gemm(const spense_packed* const* hs, int count, const uint8_t* X, const float* x_scale,
                       int64_t M, uint16_t* const* Ys, uint8_t* ws, const GemmPlan& pl, cudaStream_t stream,
                       bool x_packed_order = false, const int64_t* ldy = nullptr) {
  PreparedLaunch L;
  spense_status st = prepare_gemm(hs, count, X, x_scale, M, Ys, ws, pl, x_packed_order, ldy, &L);
  if (st != SPENSE_OK) return st;
  return enqueue_gemm(L, stream);
}

// Launch cache: repeated calls with the same weights, shapes, pointers and
// workspace (a decode loop, or the layers of a model issued one after
// another) reuse the plan, the parameter block and the tensor map instead of
// building them again. Keyed by the handles' unique ids, so a freed and
// reallocated handle never matches an old entry.
struct LaunchKey {
  int device = -1, count = 0;
  uint64_t ids[kMaxGroup] = {};
  int64_t M = 0;
  const void* X = nullptr;
  const void* x_scale = nullptr;
  const void* Ys[kMaxGroup] = {};
  int64_t ldy[kMaxGroup] = {};
  const void* ws = nullptr;
  unsigned int flags = 0;
  bool operator==(const LaunchKey& o) const {
    if (device != o.device || count != o.count || M != o.M || X != o.X || x_scale != o.x_scale || ws != o.ws ||
        flags != o.flags)
      return false;
    for (int i = 0; i < count; ++i)
      if (ids[i] != o.ids[i] || Ys[i] != o.Ys[i] || ldy[i] != o.ldy[i]) return false;
    return true;
  }
};

struct LaunchKeyHash {
  size_t operator()(const LaunchKey& k) const {
    uint64_t h = 1469598103934665603ull;  // FNV-1a over the fields that identify a call
    auto mix = [&h](uint64_t v) {
      for (int b = 0; b < 8; ++b) {
        h ^= (v >> (8 * b)) & 0xffu;
        h *= 1099511628211ull;
      }
    };
    mix(static_cast<uint64_t>(k.device));
    mix(static_cast<uint64_t>(k.count));
    mix(static_cast<uint64_t>(k.M));
    mix(reinterpret_cast<uintptr_t>(k.X));
    mix(reinterpret_cast<uintptr_t>(k.x_scale));
    mix(reinterpret_cast<uintptr_t>(k.ws));
    mix(k.flags);
    for (int i = 0; i < k.count; ++i) {
      mix(k.ids[i]);
      mix(reinterpret_cast<uintptr_t>(k.Ys[i]));
      mix(static_cast<uint64_t>(k.ldy[i]));
    }
    return static_cast<size_t>(h);
  }
};

struct LaunchCacheEntry {
  size_t ws_needed = 0;
  PreparedLaunch launch;
};

// Room for the distinct launches of a whole decoder stack (64 layers x a few
// GEMMs each, several token counts); when full it starts over.
constexpr size_t kLaunchCacheSize = 4096;
std::mutex g_launch_mu;
auto* g_launch_cache = new std::unordered_map<LaunchKey, LaunchCacheEntry, LaunchKeyHash>();

// Plans (or finds in the cache) and enqueues one grouped launch; arguments
// validated by the caller. Device pointers only.
spense_status launch_grouped(const spense_packed* const* Wps, int count, const uint8_t* X, const float* x_scale,
                             int64_t M, uint16_t* const* Ys, const int64_t* ldy, void* workspace,
                             size_t workspace_bytes, unsigned int flags, int dev, const DeviceInfo& info,
                             cudaStream_t stream) {
  LaunchKey key;
  key.device = dev;
  key.count = count;
  for (int i = 0; i < count; ++i) {
    key.ids[i] = Wps[i]->id;
    key.Ys[i] = Ys[i];
    key.ldy[i] = ldy != nullptr ? ldy[i] : Wps[i]->N;
  }
  key.M = M;
  key.X = X;
  key.x_scale = x_scale;
  key.ws = workspace;
  key.flags = flags;
  {
    std::lock_guard<std::mutex> lk(g_launch_mu);
    auto it = g_launch_cache->find(key);
    if (it != g_launch_cache->end()) {
      if (workspace_bytes < it->second.ws_needed)
        return fail(SPENSE_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", workspace_bytes,
                    it->second.ws_needed);
      return enqueue_gemm(it->second.launch, stream);
    }
  }
  GemmPlan pl;
  spense_status st = make_plan(Wps, count, M, info.sms, &pl);
  if (st != SPENSE_OK) return st;
  if (workspace_bytes < pl.ws.total_device)
    return fail(SPENSE_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", workspace_bytes,
                pl.ws.total_device);
  LaunchCacheEntry entry;
  entry.ws_needed = pl.ws.total_device;
  st = prepare_gemm(Wps, count, X, x_scale, M, Ys, static_cast<uint8_t*>(workspace), pl,
                    (flags & SPENSE_GEMM_X_PACKED_ORDER) != 0u, ldy, &entry.launch);
  if (st != SPENSE_OK) return st;
  st = enqueue_gemm(entry.launch, stream);
  if (st != SPENSE_OK) return st;
  {
    std::lock_guard<std::mutex> lk(g_launch_mu);
    if (g_launch_cache->size() >= kLaunchCacheSize) g_launch_cache->clear();
    g_launch_cache->emplace(key, entry);
  }
  return SPENSE_OK;
}

// Validates the host-side order arguments shared by spense_pack and
// spense_glu_order: dense_idx strictly ascending in [0, K).
spense_status check_dense_idx(const int32_t* dense_idx, int64_t Kd, int64_t K) {
  for (int64_t j = 0; j < Kd; ++j) {
    if (dense_idx[j] < 0 || dense_idx[j] >= K)
      return fail(SPENSE_ERR_DENSE_IDX, "dense_idx[%lld] = %d outside [0, %lld)", (long long)j, dense_idx[j],
                  (long long)K);
    if (j > 0 && dense_idx[j] <= dense_idx[j - 1])
      return fail(SPENSE_ERR_DENSE_IDX, "dense_idx is not strictly ascending at %lld", (long long)j);
  }
  return SPENSE_OK;
}

// The packed column order of a dense set (Technical Summary §2.B: the dense
// indices permuted into one contiguous block after the others): every index
// not in dense_idx, ascending, then dense_idx. dense_idx validated.
void dense_block_order(const int32_t* dense_idx, int64_t Kd, int64_t K, int32_t* order) {
  std::vector<char> dense(static_cast<size_t>(K), 0);
  for (int64_t j = 0; j < Kd; ++j) dense[static_cast<size_t>(dense_idx[j])] = 1;
  int64_t o = 0;
  for (int64_t k = 0; k < K; ++k)
    if (!dense[static_cast<size_t>(k)]) order[o++] = static_cast<int32_t>(k);
  for (int64_t j = 0; j < Kd; ++j) order[o++] = dense_idx[j];
}

// ---------------------------------------------------------------- allocation-free entry point
// Scratch for spense_gemm_noalloc: a fixed array in device memory that every
// GPU loading this library holds until the process exits. In host code the
// symbol is only a stand-in; its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SPENSE_NOALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch array for device `dev` (current), looked up
// once per (device, context) with cudaGetSymbolAddress and cached. A context
// handle that the driver reuses after a cudaDeviceReset would hit a stale
// entry; the cache assumes each device keeps its context for the life of the
// process (the runtime's primary context, as PyTorch uses it).
spense_status noalloc_scratch(int dev, uint8_t** out) {
  struct Slot {
    int dev;
    CUcontext ctx;
    uint8_t* addr;
  };
  static std::mutex mu;
  static std::vector<Slot> slots;
  CUcontext ctx = nullptr;
  if (CtxGetCurrentFn f = ctx_get_current()) f(&ctx);
  std::lock_guard<std::mutex> lk(mu);
  for (const Slot& sl : slots)
    if (sl.dev == dev && sl.ctx == ctx) {
      *out = sl.addr;
      return SPENSE_OK;
    }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
  slots.push_back(Slot{dev, ctx, static_cast<uint8_t*>(p)});
  *out = static_cast<uint8_t*>(p);
  return SPENSE_OK;
}

}  // namespace

extern "C" {

const char* spense_last_error(void) { return g_last_error.c_str(); }

const char* spense_version(void) { return "0.1.0"; }

spense_status spense_pack_rows(const uint8_t* W, const float* w_scale, int64_t N_src, int64_t K,
                               const int32_t* rows, int64_t N, const uint8_t* mask, const int32_t* dense_idx,
                               int64_t Kd, uint32_t flags, void* stream_v, spense_packed** out) {
  if (out == nullptr) return fail(SPENSE_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (W == nullptr || w_scale == nullptr || rows == nullptr) return fail(SPENSE_ERR_ARG, "W, w_scale or rows is NULL");
  if (N_src < 1 || N_src > (1 << 20) || N < 1 || N > (1 << 20))
    return fail(SPENSE_ERR_SHAPE, "N_src = %lld and N = %lld must be in [1, 2^20]", (long long)N_src, (long long)N);
  if (K < 16 || K > (1 << 20) || K % 16 != 0)
    return fail(SPENSE_ERR_SHAPE, "K = %lld must be a multiple of 16 in [16, 2^20]", (long long)K);
  if (!aligned(W, 16) || (mask != nullptr && !aligned(mask, 16)) || !aligned(w_scale, 4))
    return fail(SPENSE_ERR_ALIGN, "W and mask must be 16-byte aligned, w_scale 4-byte aligned");
  for (int64_t r = 0; r < N; ++r)
    if (rows[r] < 0 || rows[r] >= N_src)
      return fail(SPENSE_ERR_ARG, "rows[%lld] = %d outside [0, %lld)", (long long)r, rows[r], (long long)N_src);
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  // Gather the rows into temporaries, pack those, free them (pack synchronizes).
  uint8_t* wt = nullptr;
  uint8_t* mt = nullptr;
  float* st_ = nullptr;
  int32_t* rd = nullptr;
  const size_t bytes = static_cast<size_t>(N) * static_cast<size_t>(K);
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&wt), bytes);
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&st_), static_cast<size_t>(N) * 4);
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&rd), static_cast<size_t>(N) * 4);
  if (e == cudaSuccess && mask != nullptr) e = cudaMalloc(reinterpret_cast<void**>(&mt), bytes);
  if (e == cudaSuccess) e = cudaMemcpyAsync(rd, rows, static_cast<size_t>(N) * 4, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = launch_gather_rows(W, K, rd, N, wt, w_scale, st_, stream);
  if (e == cudaSuccess && mask != nullptr) e = launch_gather_rows(mask, K, rd, N, mt, nullptr, nullptr, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // `rows` may be a host temporary
  if (e != cudaSuccess) {
    for (void* q : {static_cast<void*>(wt), static_cast<void*>(mt), static_cast<void*>(st_), static_cast<void*>(rd)})
      if (q != nullptr) cudaFree(q);
    return cuda_fail(e, "row gather");
  }
  st = spense_pack(wt, st_, N, K, mt, dense_idx, Kd, flags, stream_v, out);
  for (void* q : {static_cast<void*>(wt), static_cast<void*>(mt), static_cast<void*>(st_), static_cast<void*>(rd)})
    if (q != nullptr) cudaFree(q);
  return st;
}

spense_status spense_pack(const uint8_t* W, const float* w_scale, int64_t N, int64_t K,
                          const uint8_t* mask, const int32_t* dense_idx, int64_t Kd, uint32_t flags,
                          void* stream_v, spense_packed** out) {
  if (out == nullptr) return fail(SPENSE_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (W == nullptr || w_scale == nullptr) return fail(SPENSE_ERR_ARG, "W or w_scale is NULL");
  if (flags & ~SPENSE_PACK_KEEP_CANONICAL) return fail(SPENSE_ERR_ARG, "unknown flags 0x%x", flags);
  if (N < 1 || N > (1 << 20)) return fail(SPENSE_ERR_SHAPE, "N = %lld outside [1, 2^20]", (long long)N);
  if (K < 16 || K > (1 << 20) || K % 16 != 0)
    return fail(SPENSE_ERR_SHAPE, "K = %lld must be a multiple of 16 in [16, 2^20]", (long long)K);
  if (Kd < 0 || Kd > K || Kd % 16 != 0)
    return fail(SPENSE_ERR_SHAPE, "Kd = %lld must be a multiple of 16 in [0, K]", (long long)Kd);
  if (!aligned(W, 16) || (mask != nullptr && !aligned(mask, 16)) || !aligned(w_scale, 4))
    return fail(SPENSE_ERR_ALIGN, "W and mask must be 16-byte aligned, w_scale 4-byte aligned");
  if (dense_idx != nullptr) {
    const spense_status sd = check_dense_idx(dense_idx, Kd, K);
    if (sd != SPENSE_OK) return sd;
  }
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);

  spense_packed* h = new (std::nothrow) spense_packed();
  if (h == nullptr) return fail(SPENSE_ERR_OOM, "host allocation failed");
  static std::atomic<uint64_t> next_id{1};
  h->id = next_id.fetch_add(1);
  h->device = dev;
  h->N = N;
  h->K = K;
  h->Kd = Kd;
  h->Ks = K - Kd;
  h->n_tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  h->nsb = static_cast<int>((h->Ks + kSparseBlockCols - 1) / kSparseBlockCols);
  h->ndb = static_cast<int>((Kd + kDenseBlockCols - 1) / kDenseBlockCols);
  const bool keep_canon = (flags & SPENSE_PACK_KEEP_CANONICAL) != 0;

  auto alloc = [&](void** p, size_t bytes) -> cudaError_t {
    if (bytes == 0) return cudaSuccess;
    return cudaMalloc(p, bytes);
  };
  cudaError_t e = cudaSuccess;
  const size_t nt = static_cast<size_t>(h->n_tiles);
  if (e == cudaSuccess) e = alloc(reinterpret_cast<void**>(&h->vs_t), nt * h->nsb * kBlockBytes);
  if (e == cudaSuccess) e = alloc(reinterpret_cast<void**>(&h->e_t), nt * h->nsb * kMetaBlockBytes);
  if (e == cudaSuccess) e = alloc(reinterpret_cast<void**>(&h->wd_t), nt * h->ndb * kBlockBytes);
  if (e == cudaSuccess) e = alloc(reinterpret_cast<void**>(&h->s_w), static_cast<size_t>(N) * 4);
  if (e == cudaSuccess && dense_idx != nullptr)
    e = alloc(reinterpret_cast<void**>(&h->perm), static_cast<size_t>(K) * 4);
  if (e == cudaSuccess && keep_canon) {
    e = alloc(reinterpret_cast<void**>(&h->vs_c), static_cast<size_t>(N * (h->Ks / 2)));
    if (e == cudaSuccess) e = alloc(reinterpret_cast<void**>(&h->e_c), static_cast<size_t>(N * (h->Ks / 8)));
    if (e == cudaSuccess) e = alloc(reinterpret_cast<void**>(&h->wd_c), static_cast<size_t>(N * Kd));
  }
  unsigned int* err_d = nullptr;
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&err_d), sizeof(unsigned int));
  if (e != cudaSuccess) {
    free_handle(h);
    if (err_d) cudaFree(err_d);
    return cuda_fail(e, "pack allocation");
  }
  if (dense_idx != nullptr) {
    std::vector<int32_t> perm(static_cast<size_t>(K));
    dense_block_order(dense_idx, Kd, K, perm.data());
    e = cudaMemcpyAsync(h->perm, perm.data(), perm.size() * 4, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // `perm` is a host temporary
    h->perm_host = perm;
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(err_d, 0, sizeof(unsigned int), stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h->s_w, w_scale, static_cast<size_t>(N) * 4, cudaMemcpyDeviceToDevice, stream);
  if (e == cudaSuccess)
    e = launch_pack(W, mask, h->perm, N, K, Kd, h->vs_t, h->e_t, h->wd_t, h->vs_c, h->e_c, h->wd_c, err_d,
                    stream);
  unsigned int err_h = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&err_h, err_d, sizeof(unsigned int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  cudaFree(err_d);
  if (e != cudaSuccess) {
    free_handle(h);
    return cuda_fail(e, "pack");
  }
  if (err_h & kPackErrNaN) {
    free_handle(h);
    return fail(SPENSE_ERR_NONFINITE, "W holds an e4m3 NaN byte");
  }
  if (err_h & kPackErrMask) {
    free_handle(h);
    return fail(SPENSE_ERR_MASK, "a group of four in the mask keeps more than two entries");
  }
  *out = h;
  return ok();
}

spense_status spense_free(spense_packed* Wp) {
  free_handle(Wp);
  return ok();
}

size_t spense_gemm_workspace_size(const spense_packed* Wp, int64_t M) {
  return spense_gemm_grouped_workspace_size(&Wp, 1, M);
}

size_t spense_gemm_grouped_workspace_size(const spense_packed* const* Wps, int count, int64_t M) {
  int dev = 0;
  DeviceInfo info;
  if (current_device(&dev, &info) != SPENSE_OK) return 0;
  GemmPlan pl;
  if (make_plan(Wps, count, M, info.sms, &pl) != SPENSE_OK) return 0;
  return pl.ws.total_device;
}

static_assert(SPENSE_PLAN_MAX_GRID == kMaxGrid, "plan introspection array size");

spense_status spense_plan_shapes(int count, const int64_t* N, const int64_t* K, const int64_t* Kd, int64_t M,
                                 int sms, spense_plan_info* out) {
  if (out == nullptr || N == nullptr || K == nullptr || Kd == nullptr)
    return fail(SPENSE_ERR_ARG, "out, N, K or Kd is NULL");
  if (count < 1 || count > kMaxGroup)
    return fail(SPENSE_ERR_ARG, "a launch takes 1 to %d packed weights, got %d", kMaxGroup, count);
  if (sms < 1 || sms > 1024) return fail(SPENSE_ERR_ARG, "sms = %d outside [1, 1024]", sms);
  std::vector<spense_packed> hs(static_cast<size_t>(count));
  std::vector<const spense_packed*> ptrs(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    if (N[i] < 1 || N[i] > (1 << 20)) return fail(SPENSE_ERR_SHAPE, "N = %lld outside [1, 2^20]", (long long)N[i]);
    if (K[i] < 16 || K[i] > (1 << 20) || K[i] % 16 != 0)
      return fail(SPENSE_ERR_SHAPE, "K = %lld must be a multiple of 16 in [16, 2^20]", (long long)K[i]);
    if (Kd[i] < 0 || Kd[i] > K[i] || Kd[i] % 16 != 0)
      return fail(SPENSE_ERR_SHAPE, "Kd = %lld must be a multiple of 16 in [0, K]", (long long)Kd[i]);
    spense_packed& h = hs[static_cast<size_t>(i)];
    h.device = 0;
    h.N = N[i];
    h.K = K[i];
    h.Kd = Kd[i];
    h.Ks = K[i] - Kd[i];
    h.n_tiles = static_cast<int>((N[i] + kTileRows - 1) / kTileRows);
    h.nsb = static_cast<int>((h.Ks + kSparseBlockCols - 1) / kSparseBlockCols);
    h.ndb = static_cast<int>((Kd[i] + kDenseBlockCols - 1) / kDenseBlockCols);
    ptrs[static_cast<size_t>(i)] = &h;
  }
  GemmPlan pl{};
  const spense_status st = make_plan(ptrs.data(), count, M, sms, &pl);
  if (st != SPENSE_OK) return st;
  *out = spense_plan_info{};
  out->npad = pl.npad;
  out->box_rows = pl.box_rows;
  out->m_tiles = pl.m_tiles;
  out->n_tiles = pl.n_tiles;
  out->tiles = pl.tiles;
  out->ctas_per_sm = pl.ctas_per_sm;
  out->cluster = pl.cluster;
  out->grid = pl.grid;
  out->stages = pl.stages;
  out->nacc = pl.nacc;
  out->tmem_cols = pl.tmem_cols;
  out->smem_bytes = pl.smem_bytes;
  out->stage_bytes = pl.stage_bytes;
  out->recv_bytes = pl.recv_bytes;
  out->l2_prefetch = l2_prefetch_for(pl);
  out->pair = pl.pair;
  out->y_stage_bytes = pl.ystage;
  out->total_blocks = pl.cta_start[pl.grid];
  out->workspace_bytes = pl.ws.total_device;
  for (int g = 0; g <= pl.grid; ++g) out->cta_start[g] = pl.cta_start[g];
  return ok();
}

size_t spense_gemm_host_workspace_size(const spense_packed* Wp, int64_t M) {
  int dev = 0;
  DeviceInfo info;
  if (current_device(&dev, &info) != SPENSE_OK) return 0;
  GemmPlan pl;
  if (make_plan(&Wp, 1, M, info.sms, &pl) != SPENSE_OK) return 0;
  return pl.ws.total_host;
}

spense_status spense_gemm_grouped(const spense_packed* const* Wps, int count, const uint8_t* X,
                                  const float* x_scale, int64_t M, uint16_t* const* Ys, void* workspace,
                                  size_t workspace_bytes, void* stream_v) {
  return spense_gemm_grouped_ex(Wps, count, X, x_scale, M, Ys, nullptr, workspace, workspace_bytes, 0u, stream_v);
}

spense_status spense_gemm_grouped_ex(const spense_packed* const* Wps, int count, const uint8_t* X,
                                     const float* x_scale, int64_t M, uint16_t* const* Ys, const int64_t* ldy,
                                     void* workspace, size_t workspace_bytes, unsigned int flags, void* stream_v) {
  if ((flags & ~static_cast<unsigned int>(SPENSE_GEMM_X_PACKED_ORDER)) != 0u)
    return fail(SPENSE_ERR_ARG, "unknown flags %#x", flags);
  if (M < 1 || M > 65535) return fail(SPENSE_ERR_SHAPE, "M = %lld outside [1, 65535]", (long long)M);
  if (X == nullptr || x_scale == nullptr || Ys == nullptr) return fail(SPENSE_ERR_ARG, "X, x_scale or Y is NULL");
  if (!aligned(X, 16) || !aligned(x_scale, 4))
    return fail(SPENSE_ERR_ALIGN, "X must be 16-byte aligned, x_scale 4-byte aligned");
  if (count >= 1 && count <= kMaxGroup) {
    for (int i = 0; i < count; ++i) {
      if (Ys[i] == nullptr) return fail(SPENSE_ERR_ARG, "Y[%d] is NULL", i);
      if (!aligned(Ys[i], 16)) return fail(SPENSE_ERR_ALIGN, "Y[%d] must be 16-byte aligned", i);
      if (ldy != nullptr && Wps != nullptr && Wps[i] != nullptr &&
          (ldy[i] < Wps[i]->N || ldy[i] > (1ll << 30)))
        return fail(SPENSE_ERR_SHAPE, "ldy[%d] = %lld is smaller than N or too large", i, (long long)ldy[i]);
    }
  }
  DeviceInfo info;
  spense_status st = check_gemm_args(Wps, count, M, workspace, &info);
  if (st != SPENSE_OK) return st;
  for (int i = 0; i < count; ++i)
    if (Wps[i] == nullptr) return fail(SPENSE_ERR_ARG, "packed weight %d is NULL", i);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(SPENSE_ERR_UNSUPPORTED, "no CUDA device");
  st = launch_grouped(Wps, count, X, x_scale, M, Ys, ldy, workspace, workspace_bytes, flags, dev, info,
                      static_cast<cudaStream_t>(stream_v));
  return st == SPENSE_OK ? ok() : st;
}

spense_status spense_quantize(const uint16_t* X, int64_t M, int64_t K, const spense_packed* order, uint8_t* Xq,
                              float* x_scale, void* stream_v) {
  if (M < 0 || M > 65535) return fail(SPENSE_ERR_SHAPE, "M = %lld outside [0, 65535]", (long long)M);
  if (M > 0 && (X == nullptr || Xq == nullptr || x_scale == nullptr))
    return fail(SPENSE_ERR_ARG, "X, Xq or x_scale is NULL");
  if (K < 16 || K > (1 << 20) || K % 16 != 0)
    return fail(SPENSE_ERR_SHAPE, "K = %lld must be a positive multiple of 16 up to 2^20", (long long)K);
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(x_scale, 4))
    return fail(SPENSE_ERR_ALIGN, "X and Xq must be 16-byte aligned, x_scale 4-byte aligned");
  const int32_t* perm = nullptr;
  if (order != nullptr) {
    if (order->K != K) return fail(SPENSE_ERR_SHAPE, "order was packed with K = %lld, not %lld",
                                   (long long)order->K, (long long)K);
    perm = order->perm;  // NULL for a tail dense set: the packed order is the identity
  }
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  if (order != nullptr && dev != order->device)
    return fail(SPENSE_ERR_ARG, "order was packed on device %d, current device is %d", order->device, dev);
  cudaError_t e = launch_quantize(X, M, K, perm, Xq, x_scale, info.sms, static_cast<cudaStream_t>(stream_v));
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

size_t spense_score_workspace_size(int64_t I, int64_t H) {
  if (I < 16 || I > (1 << 20) || I % 16 != 0 || H < 16 || H > (1 << 20) || H % 16 != 0) return 0;
  return score_workspace_bytes(I);
}

spense_status spense_score_glu(const uint8_t* gate, const float* s_gate, const uint8_t* up, const float* s_up,
                               int64_t I, int64_t H, const uint8_t* down, const float* s_down, const float* h_in,
                               const float* h_mid, float* score, void* workspace, size_t workspace_bytes,
                               void* stream_v) {
  if (down == nullptr || s_down == nullptr || h_in == nullptr || h_mid == nullptr || score == nullptr)
    return fail(SPENSE_ERR_ARG, "down, s_down, h_in, h_mid or score is NULL");
  if ((gate != nullptr && s_gate == nullptr) || (up != nullptr && s_up == nullptr))
    return fail(SPENSE_ERR_ARG, "gate or up given without its row scales");
  if (I < 16 || I > (1 << 20) || I % 16 != 0 || H < 16 || H > (1 << 20) || H % 16 != 0)
    return fail(SPENSE_ERR_SHAPE, "I = %lld and H = %lld must be multiples of 16 in [16, 2^20]", (long long)I,
                (long long)H);
  if (!aligned(down, 16) || (gate && !aligned(gate, 16)) || (up && !aligned(up, 16)) || !aligned(s_down, 4) ||
      (s_gate && !aligned(s_gate, 4)) || (s_up && !aligned(s_up, 4)) || !aligned(h_in, 4) || !aligned(h_mid, 4) ||
      !aligned(score, 4))
    return fail(SPENSE_ERR_ALIGN, "weights must be 16-byte aligned, vectors 4-byte aligned");
  if (workspace == nullptr || workspace_bytes < score_workspace_bytes(I))
    return fail(SPENSE_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", workspace_bytes,
                score_workspace_bytes(I));
  if (!aligned(workspace, 256)) return fail(SPENSE_ERR_ALIGN, "workspace is not 256-byte aligned");
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  cudaError_t e = launch_score_glu(gate, s_gate, up, s_up, I, H, down, s_down, h_in, h_mid, score,
                                   static_cast<float*>(workspace), static_cast<cudaStream_t>(stream_v));
  if (e != cudaSuccess) return cuda_fail(e, "score launch");
  return ok();
}

spense_status spense_select_dense(const float* score, int64_t I, int64_t Kd, int32_t* dense_idx, void* stream_v) {
  if (I < 1 || I > (1 << 20)) return fail(SPENSE_ERR_SHAPE, "I = %lld outside [1, 2^20]", (long long)I);
  if (Kd < 0 || Kd > I) return fail(SPENSE_ERR_SHAPE, "Kd = %lld outside [0, I]", (long long)Kd);
  if (Kd > 0 && (score == nullptr || dense_idx == nullptr)) return fail(SPENSE_ERR_ARG, "score or dense_idx is NULL");
  if (Kd > 0 && (!aligned(score, 4) || !aligned(dense_idx, 4)))
    return fail(SPENSE_ERR_ALIGN, "score and dense_idx must be 4-byte aligned");
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  cudaError_t e = launch_select_top(score, I, Kd, dense_idx, static_cast<cudaStream_t>(stream_v));
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  return ok();
}

spense_status spense_gemm(const spense_packed* Wp, const uint8_t* X, const float* x_scale, int64_t M,
                          uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream_v) {
  if (Y == nullptr) return fail(SPENSE_ERR_ARG, "X, x_scale or Y is NULL");
  if (X != nullptr && !aligned(X, 16)) return fail(SPENSE_ERR_ALIGN, "X and Y must be 16-byte aligned");
  return spense_gemm_grouped(&Wp, 1, X, x_scale, M, &Y, workspace, workspace_bytes, stream_v);
}

spense_status spense_gemm_grouped_host(const spense_packed* const* Wps, int count, const uint8_t* X,
                                       const float* x_scale, int64_t M, uint16_t* const* Ys, void* workspace,
                                       size_t workspace_bytes, unsigned int flags, void* stream_v) {
  const unsigned int known = SPENSE_GEMM_X_PACKED_ORDER | SPENSE_GEMM_HOST_X | SPENSE_GEMM_HOST_Y;
  if ((flags & ~known) != 0u) return fail(SPENSE_ERR_ARG, "unknown flags %#x", flags);
  if (X == nullptr || x_scale == nullptr || Ys == nullptr) return fail(SPENSE_ERR_ARG, "X, x_scale or Y is NULL");
  const bool host_x = (flags & SPENSE_GEMM_HOST_X) != 0u;
  const bool host_y = (flags & SPENSE_GEMM_HOST_Y) != 0u;
  if (!host_x && (!aligned(X, 16) || !aligned(x_scale, 4)))
    return fail(SPENSE_ERR_ALIGN, "X must be 16-byte aligned, x_scale 4-byte aligned");
  DeviceInfo info;
  spense_status st = check_gemm_args(Wps, count, M, workspace, &info);
  if (st != SPENSE_OK) return st;
  for (int i = 0; i < count; ++i) {
    if (Wps[i] == nullptr) return fail(SPENSE_ERR_ARG, "packed weight %d is NULL", i);
    if (Ys[i] == nullptr) return fail(SPENSE_ERR_ARG, "Y[%d] is NULL", i);
    if (!host_y && !aligned(Ys[i], 16)) return fail(SPENSE_ERR_ALIGN, "Y[%d] must be 16-byte aligned", i);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(SPENSE_ERR_UNSUPPORTED, "no CUDA device");
  GemmPlan pl;
  st = make_plan(Wps, count, M, info.sms, &pl);
  if (st != SPENSE_OK) return st;
  const size_t need = (host_x || host_y) ? pl.ws.total_host : pl.ws.total_device;
  if (workspace_bytes < need)
    return fail(SPENSE_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const uint8_t* xd = X;
  const float* sxd = x_scale;
  if (host_x) {
    uint8_t* xs = ws + pl.ws.stage_x_off;
    float* sxs = reinterpret_cast<float*>(ws + pl.ws.stage_sx_off);
    cudaError_t e = cudaMemcpyAsync(xs, X, static_cast<size_t>(M * Wps[0]->K), cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sxs, x_scale, static_cast<size_t>(M) * 4, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    xd = xs;
    sxd = sxs;
  }
  uint16_t* yd[kMaxGroup];
  size_t y_off = pl.ws.stage_y_off;
  for (int i = 0; i < count; ++i) {
    if (host_y) {
      yd[i] = reinterpret_cast<uint16_t*>(ws + y_off);
      y_off += round_up(static_cast<size_t>(M * Wps[i]->N) * 2, 256);
    } else {
      yd[i] = Ys[i];
    }
  }
  st = launch_grouped(Wps, count, xd, sxd, M, yd, nullptr, workspace, workspace_bytes,
                      flags & SPENSE_GEMM_X_PACKED_ORDER, dev, info, stream);
  if (st != SPENSE_OK) return st;
  if (host_y) {
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < count && e == cudaSuccess; ++i)
      e = cudaMemcpyAsync(Ys[i], yd[i], static_cast<size_t>(M * Wps[i]->N) * 2, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  }
  return ok();
}

size_t spense_gemm_grouped_host_workspace_size(const spense_packed* const* Wps, int count, int64_t M) {
  int dev = 0;
  DeviceInfo info;
  if (current_device(&dev, &info) != SPENSE_OK) return 0;
  GemmPlan pl;
  if (make_plan(Wps, count, M, info.sms, &pl) != SPENSE_OK) return 0;
  return pl.ws.total_host;
}

spense_status spense_gemm_host(const spense_packed* Wp, const uint8_t* X_host, const float* x_scale_host,
                               int64_t M, uint16_t* Y_host, void* workspace, size_t workspace_bytes,
                               void* stream_v) {
  if (Wp == nullptr) return fail(SPENSE_ERR_ARG, "Wp is NULL");
  return spense_gemm_grouped_host(&Wp, 1, X_host, x_scale_host, M, &Y_host, workspace, workspace_bytes,
                                  SPENSE_GEMM_HOST_X | SPENSE_GEMM_HOST_Y, stream_v);
}

spense_status spense_glu_order(int64_t I, const int32_t* dense_idx, int64_t Kd, int32_t* order) {
  if (order == nullptr || (Kd > 0 && dense_idx == nullptr)) return fail(SPENSE_ERR_ARG, "order or dense_idx is NULL");
  if (I < 1 || I > (1 << 20)) return fail(SPENSE_ERR_SHAPE, "I = %lld outside [1, 2^20]", (long long)I);
  if (Kd < 0 || Kd > I) return fail(SPENSE_ERR_SHAPE, "Kd = %lld outside [0, I]", (long long)Kd);
  const spense_status st = check_dense_idx(dense_idx, Kd, I);
  if (st != SPENSE_OK) return st;
  dense_block_order(dense_idx, Kd, I, order);
  return ok();
}

spense_status spense_get_info(const spense_packed* Wp, spense_packed_info* info) {
  if (Wp == nullptr || info == nullptr) return fail(SPENSE_ERR_ARG, "NULL argument");
  info->N = Wp->N;
  info->K = Wp->K;
  info->Ks = Wp->Ks;
  info->Kd = Wp->Kd;
  info->n_tiles = Wp->n_tiles;
  info->sparse_blocks = Wp->nsb;
  info->dense_blocks = Wp->ndb;
  info->Vs_t = Wp->vs_t;
  info->E_t = Wp->e_t;
  info->Wd_t = Wp->wd_t;
  info->w_scale = Wp->s_w;
  info->Vs = Wp->vs_c;
  info->E = Wp->e_c;
  info->Wd = Wp->wd_c;
  info->perm = Wp->perm;
  info->weight_bytes = static_cast<uint64_t>(Wp->n_tiles) *
                       (static_cast<uint64_t>(Wp->nsb) * (kBlockBytes + kMetaBlockBytes) +
                        static_cast<uint64_t>(Wp->ndb) * kBlockBytes);
  return ok();
}

spense_status spense_workspace_status(void* workspace, void* stream_v, uint32_t* status_out) {
  if (workspace == nullptr || status_out == nullptr) return fail(SPENSE_ERR_ARG, "NULL argument");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && word != 0) {
    e = cudaMemsetAsync(workspace, 0, 4, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  *status_out = word;
  return ok();
}

spense_status spense_gemm_noalloc(const spense_packed* Wp, const uint8_t* X, const float* x_scale,
                                  int64_t M, uint16_t* Y, void* stream_v) {
  if (X == nullptr || x_scale == nullptr || Y == nullptr) return fail(SPENSE_ERR_ARG, "X, x_scale or Y is NULL");
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(x_scale, 4))
    return fail(SPENSE_ERR_ALIGN, "X and Y must be 16-byte aligned, x_scale 4-byte aligned");
  if (Wp == nullptr) return fail(SPENSE_ERR_ARG, "Wp is NULL");
  if (M < 1 || M > 65535) return fail(SPENSE_ERR_SHAPE, "M = %lld outside [1, 65535]", (long long)M);
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  if (dev != Wp->device)
    return fail(SPENSE_ERR_ARG, "handle was packed on device %d, current device is %d", Wp->device, dev);
  GemmPlan pl;
  st = make_plan(&Wp, 1, M, info.sms, &pl);
  if (st != SPENSE_OK) return st;
  if (pl.ws.total_device > SPENSE_NOALLOC_SCRATCH_BYTES)
    return fail(SPENSE_ERR_WORKSPACE,
                "this GEMM needs %zu bytes of scratch; the built-in scratch holds %zu (use spense_gemm "
                "with a caller workspace, or fewer tokens)",
                pl.ws.total_device, static_cast<size_t>(SPENSE_NOALLOC_SCRATCH_BYTES));
  uint8_t* ws = nullptr;
  st = noalloc_scratch(dev, &ws);
  if (st != SPENSE_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  // The arrival counters (and the rest of the header) must start at zero;
  // the array keeps whatever the previous call left in it. The status word
  // (the first 4 bytes) is left alone: a timeout stays recorded until
  // spense_noalloc_status reads it.
  const cudaError_t e = cudaMemsetAsync(ws + 4, 0, pl.ws.partials_off - 4, stream);
  if (e != cudaSuccess) return cuda_fail(e, "scratch clear");
  st = run_gemm(&Wp, 1, X, x_scale, M, &Y, ws, pl, stream);
  return st == SPENSE_OK ? ok() : st;
}

spense_status spense_noalloc_status(void* stream_v, uint32_t* status_out) {
  if (status_out == nullptr) return fail(SPENSE_ERR_ARG, "status_out is NULL");
  int dev = 0;
  DeviceInfo info;
  spense_status st = current_device(&dev, &info);
  if (st != SPENSE_OK) return st;
  uint8_t* ws = nullptr;
  st = noalloc_scratch(dev, &ws);
  if (st != SPENSE_OK) return st;
  return spense_workspace_status(ws, stream_v, status_out);
}

}  // extern "C"
