// Hybrid 2:4-sparse + dense FP8 weight GEMM for sm_100a:
//   Y[m][n] = bf16(s_x[m] * s_w[n] * (sum over the 2:4 region + sum over the dense region))
//
// Page: "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs
// for LLM Inference" (gist.science technical summary), Technical Summary §2.A:
// the input-split execution runs the sparse GEMM over the first part of the
// input dimension and the dense GEMM over the second, with accumulation. Here
// both phases feed ONE fp32 accumulator in tensor memory inside one kernel:
// tcgen05.mma.sp over the 2:4 blocks, then tcgen05.mma over the dense blocks.
//
// Layout of the work (swap-AB): weight rows are the MMA M dimension (128 per
// tile), tokens are the MMA N dimension (padded to a multiple of 16), K is the
// packed column order (2:4 region first, then the dense region). Up to
// kMaxGroup weight matrices with the same K layout can share one launch and
// one activation tensor (for example q, k and v projections); their row tiles
// are laid end to end.
//
// Roles (up to two CTAs per SM, 192 to 256 threads):
//   warps 0, 6 producers: bulk copies of the packed weight blocks (values,
//            metadata, dense columns) into a ring of shared-memory stages;
//            with two producer warps each issues every other block;
//   warp 7   (warp 6 with one producer) 2-D TMA loads of the activation tile
//            of every block into the same stages (without it, the producers
//            issue them after each stage's weight copies);
//   warp 1   allocates tensor memory; one lane copies the metadata into tensor
//            memory (tcgen05.cp) and issues the MMAs;
//   warps 2-5 epilogue: tensor memory -> registers, scales, bf16 stores, or
//            fp32 partials plus a deterministic fix-up when a tile is shared.
//
// Work split ("stream-K by bytes"): the blocks of all tiles form one sequence,
// each block weighted by the HBM bytes it streams (a 2:4 block 20 KiB, a dense
// block 16 KiB). The host cuts the sequence into one contiguous range per CTA
// (p.cta_start). A CTA handles the tiles it shares with its neighbours first
// and its whole tiles last, so the cross-CTA fix-ups overlap the streaming of
// whole tiles instead of forming the kernel's tail. A shared tile is finished
// by the last contributor to arrive, which sums every contributor's partial in
// CTA order, so the result does not depend on arrival order.
//
// Launches with few tiles use a cluster split instead: the S CTAs of a cluster
// (S = 2, 4 or 8) stream consecutive K ranges of one tile; each peer stages
// its fp32 partial in its idle ring and sends it into rank 0's shared memory
// with one shared-to-shared bulk copy, and rank 0 adds them in rank order.
//
// Every wait is bounded (1.5 s by %globaltimer); on expiry the kernel records a
// code in the workspace status word and all roles leave their loops.
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "spense_internal.h"

namespace spense {
namespace {

constexpr uint64_t kWaitLimitNs = 1500000000ull;

struct alignas(16) Barriers {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t peer_done;  // cluster mode, rank 0: completes when every peer's partial has landed
  uint64_t ack;        // cluster mode, peers: rank 0 has received this CTA's partial
  uint64_t peer_full[kMaxStages];  // pair mode, even CTA: the odd CTA's stage has landed
  uint32_t tmem_base;
  int abort_flag;
  int fix_flag;
  int npend;    // stream-K: fix-ups left for the end of the kernel (0 to 2)
  int pend[2];  // ... their tiles
  alignas(16) float sx[kMaxTokenTile];  // per-token scales of the token tile being finished
};
static_assert(sizeof(Barriers) <= kBarrierBytes, "barrier area too small");

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, unsigned int* status,
                                         unsigned int code, volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  uint32_t it = 0;
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((++it & 63u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - t0 > kWaitLimitNs) {
        atomicOr(status, code);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Bounded wait with acquire at cluster scope (for arrivals from peer CTAs).
__device__ __forceinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity, unsigned int* status,
                                                 unsigned int code, volatile int* abort_flag) {
  const uint64_t t0 = ptx::globaltimer();
  uint32_t it = 0;
  while (true) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    if ((++it & 63u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - t0 > kWaitLimitNs) {
        atomicOr(status, code);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// CTA owning linear block b: the last g with cta_start[g] <= b.
__device__ __forceinline__ int block_owner(const GemmParams& p, int b) {
  int lo = 0, hi = p.grid - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.cta_start[mid] <= b)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Group member holding global row tile n_tile.
__device__ __forceinline__ int member_of(const GemmParams& p, int n_tile) {
  int i = 0;
#pragma unroll
  for (int k = 1; k < kMaxGroup; ++k)
    if (k < p.n_members && p.mem[k].tile_begin <= n_tile) i = k;
  return i;
}

// First linear block of tile t (and, through nb, its number of blocks): a
// member's tiles all have its layout and lie end to end from block_begin.
__device__ __forceinline__ int tile_block0(const GemmParams& p, int t, int* nb) {
  const GemmMember& mb = p.mem[member_of(p, t / p.m_tiles)];
  if (nb != nullptr) *nb = mb.nblk;
  return mb.block_begin + (t - mb.tile_begin * p.m_tiles) * mb.nblk;
}

// Tile t and block j within it of linear block b.
__device__ __forceinline__ void block_tile(const GemmParams& p, int b, int& t, int& j) {
  int i = 0;
#pragma unroll
  for (int k = 1; k < kMaxGroup; ++k)
    if (k < p.n_members && p.mem[k].block_begin <= b) i = k;
  const GemmMember& mb = p.mem[i];
  const int local = b - mb.block_begin;
  const int tl = local / mb.nblk;
  t = mb.tile_begin * p.m_tiles + tl;
  j = local - tl * mb.nblk;
}

// The units (tile, block range) of one CTA's block range, in processing order:
// a partial last unit is moved to the front, so both shared tiles come first.
struct Units {
  const GemmParams* p;
  int t_first, j_first, t_last, j_last_end, count;
  bool move_last;
  __device__ Units(const GemmParams& pp, int b0, int b1) : p(&pp) {
    if (b1 <= b0) {
      count = 0;
      t_first = j_first = t_last = j_last_end = 0;
      move_last = false;
      return;
    }
    block_tile(pp, b0, t_first, j_first);
    int jl;
    block_tile(pp, b1 - 1, t_last, jl);
    j_last_end = jl + 1;
    count = t_last - t_first + 1;
    move_last = count >= 2 && j_last_end < nblk_of(t_last);
  }
  __device__ int nblk_of(int t) const {
    int nb;
    tile_block0(*p, t, &nb);
    return nb;
  }
  // Unit at processing position u: tile t, blocks [j0, j1).
  __device__ void get(int u, int& t, int& j0, int& j1) const {
    const int k = move_last ? (u == 0 ? count - 1 : u - 1) : u;
    t = t_first + k;
    j0 = (k == 0) ? j_first : 0;
    j1 = (k == count - 1) ? j_last_end : nblk_of(t);
  }
};

// Walks the blocks of a CTA in processing order without integer division on
// the per-block path.
struct BlockWalker {
  const Units* units;
  int u, j, j1, m_tile, m_tiles, member, local_tile;
  __device__ BlockWalker(const Units& us, const GemmParams& p) : units(&us), u(0), m_tiles(p.m_tiles) {
    enter(p);
  }
  __device__ void enter(const GemmParams& p) {
    if (u >= units->count) return;
    int t, j0;
    units->get(u, t, j0, j1);
    j = j0;
    const int n_tile = t / m_tiles;
    m_tile = t - n_tile * m_tiles;
    member = member_of(p, n_tile);
    local_tile = n_tile - p.mem[member].tile_begin;
  }
  // Row tile of the member whose weights this CTA streams: the tile itself,
  // or in pair mode tile 2 x (pair tile) + the CTA's rank in the pair (the
  // odd CTA of a member's last pair past its row count re-reads the last
  // tile; its results are not stored).
  __device__ int weight_tile(const GemmParams& p, uint32_t prank) const {
    if (!p.pair) return local_tile;
    return min(2 * local_tile + static_cast<int>(prank), p.mem[member].row_tiles - 1);
  }
  __device__ void advance(const GemmParams& p) {
    if (++j == j1) {
      ++u;
      enter(p);
    }
  }
};

__device__ __forceinline__ uint16_t to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// The token scales sx[0 .. 15] (staged in shared memory, 16-byte aligned) into
// registers ahead of a chunk's stores. Read one at a time between the stores,
// every load waited for the store before it (the compiler cannot tell the
// staged scales from the outputs apart): a 128-token epilogue took about 4x as
// long that way.
__device__ __forceinline__ void load_sx16(const float* sx, float (&s)[16]) {
  const float4* s4 = reinterpret_cast<const float4*>(sx);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = s4[q];
    s[4 * q] = f.x;
    s[4 * q + 1] = f.y;
    s[4 * q + 2] = f.z;
    s[4 * q + 3] = f.w;
  }
}

// Sums the contributors' partials of stream-K tile t in CTA order, applies
// the scales and stores Y (for a CTA pair: rank prank's 128 rows). Every
// contributor after g_lo starts inside tile t, so its partial is in slot 0;
// g_lo uses slot 1 when its range started in an earlier tile. Threads
// [0, nthr) of the CTA take part (nthr a multiple of 32, tid the caller's
// index among them). Partial slots are token-major, [npad tokens][128 rows]:
// lane l sums rows 4l .. 4l + 3 and warp w tokens 4w .. 4w + 3 of every chunk
// of 4 nthr / 32 tokens, so each access is a 16-byte load (a warp covers one
// token's 128 rows) and each output a 4-row 8-byte store. sx: the token tile's
// scales, staged in shared memory.
__device__ __forceinline__ void fixup_tile(const GemmParams& p, int t, int P, uint32_t prank, int tid, int nthr,
                                           const float* sx) {
  const int n_tile = t / p.m_tiles;
  const int m0 = (t - n_tile * p.m_tiles) * p.npad;
  const GemmMember& mb = p.mem[member_of(p, n_tile)];
  const int m_valid = min(p.npad, p.M - m0);
  int nb_t;
  const int tb = tile_block0(p, t, &nb_t);
  const int g_lo = block_owner(p, tb);
  const int g_hi = block_owner(p, tb + nb_t - 1);
  const int lo_slot = (p.cta_start[g_lo] >= tb) ? 0 : 1;
  const size_t slot_elems = static_cast<size_t>(kTileRows) * p.npad;
  const int r0 = (tid & 31) * 4;
  const int tq = (tid >> 5) * 4;
  const int step = 4 * (nthr >> 5);
  const int n0 = (P * (n_tile - mb.tile_begin) + static_cast<int>(prank)) * kTileRows + r0;
  float sw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sw[i] = n0 + i < mb.N ? __ldg(mb.s_w + n0 + i) : 0.0f;
  const bool vec = n0 + 4 <= mb.N && (mb.ldy % 4) == 0;
  const float* lo_part = p.partials + (static_cast<size_t>(g_lo * P + prank) * 2 + lo_slot) * slot_elems + r0;
  const float* next_part = p.partials + (static_cast<size_t>((g_lo + 1) * P + prank) * 2) * slot_elems + r0;
  const size_t stride = static_cast<size_t>(2 * P) * slot_elems;  // from contributor gg to gg + 1 (slot 0)
  const int others = g_hi - g_lo;
  for (int c0 = 0; c0 < m_valid; c0 += step) {
    float4 a[4], b[4], c[4];
    const int mb0 = c0 + tq;  // this warp's first token of the chunk
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (mb0 + j < m_valid)
        a[j] = __ldcg(reinterpret_cast<const float4*>(lo_part + static_cast<size_t>(mb0 + j) * kTileRows));
    int k = 0;
    for (; k + 2 <= others; k += 2) {
      const float* pb = next_part + k * stride;
      const float* pc = pb + stride;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (mb0 + j < m_valid) {
          b[j] = __ldcg(reinterpret_cast<const float4*>(pb + static_cast<size_t>(mb0 + j) * kTileRows));
          c[j] = __ldcg(reinterpret_cast<const float4*>(pc + static_cast<size_t>(mb0 + j) * kTileRows));
        }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (mb0 + j < m_valid) {
          a[j].x += b[j].x; a[j].y += b[j].y; a[j].z += b[j].z; a[j].w += b[j].w;
          a[j].x += c[j].x; a[j].y += c[j].y; a[j].z += c[j].z; a[j].w += c[j].w;
        }
    }
    if (k < others) {
      const float* pb = next_part + k * stride;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (mb0 + j < m_valid) {
          b[j] = __ldcg(reinterpret_cast<const float4*>(pb + static_cast<size_t>(mb0 + j) * kTileRows));
          a[j].x += b[j].x; a[j].y += b[j].y; a[j].z += b[j].z; a[j].w += b[j].w;
        }
    }
    const float4 s4 = *reinterpret_cast<const float4*>(sx + mb0);  // ahead of the stores (see load_sx16)
    const float s_tok[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = mb0 + j;
      if (m >= m_valid) continue;
      const float s = s_tok[j];
      const uint32_t v0 = to_bf16_bits(a[j].x * sw[0] * s), v1 = to_bf16_bits(a[j].y * sw[1] * s);
      const uint32_t v2 = to_bf16_bits(a[j].z * sw[2] * s), v3 = to_bf16_bits(a[j].w * sw[3] * s);
      uint16_t* yrow = mb.y + static_cast<size_t>(m0 + m) * mb.ldy;
      if (vec) {
        *reinterpret_cast<uint2*>(yrow + n0) = make_uint2(v0 | (v1 << 16), v2 | (v3 << 16));
      } else {
        const uint32_t vv[4] = {v0, v1, v2, v3};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (n0 + i < mb.N) yrow[n0 + i] = static_cast<uint16_t>(vv[i]);
      }
    }
  }
  if (tid == 0) p.counters[t * P + prank] = 0u;  // re-arm for the next launch (ordered by the kernel boundary)
}

// Ring position: stage index and the parity of its current use.
struct Ring {
  uint32_t s = 0, ph = 0, n;
  __device__ explicit Ring(uint32_t stages) : n(stages) {}
  __device__ void advance() {
    if (++s == n) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// kPair: the pair-mode instantiation. A kernel holding tcgen05 cta_group::2
// instructions can only be launched as clusters of CTA pairs, so the
// single-CTA modes (stream-K, cluster K-split) use the other instantiation.
template <bool kPair>
__global__ void __launch_bounds__(kGemmThreadsMax, 2)
    spense_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // [stage ring][cluster receive area][barriers]
  const uint32_t recv_off = static_cast<uint32_t>(p.stages) * p.stage_bytes;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + recv_off + p.recv_bytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair mode: CTAs 2u and 2u + 1 (one cluster) are work unit u; the even
  // CTA (rank 0) issues the pair's MMAs. Otherwise every CTA is a work unit.
  constexpr bool pair = kPair;
  const uint32_t prank = pair ? ptx::cluster_ctarank() : 0u;
  const int g = pair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  // This CTA's partial slots (stream-K) and the stride between the CTAs of
  // consecutive work units that contribute to one of its tiles.
  const int P = pair ? 2 : 1;
  // Let the next kernel in the stream start launching: its CTAs take SMs as
  // this grid's CTAs exit and wait (griddepcontrol.wait) before reading
  // anything this grid writes.
  ptx::griddep_launch_dependents();
  const int b0 = p.cta_start[g];
  const int b1 = p.cta_start[g + 1];
  const bool in_cluster = p.cluster > 1 || pair;  // launched as clusters (uses the cluster barrier)

  if (warp >= 2 && warp <= 5) {
    // The epilogue warps are idle during set-up: they touch the whole
    // parameter block once, so the constant-cache misses are taken in one
    // parallel round trip instead of one after another on the producers'
    // path to their first copy.
    const uint32_t* pw = reinterpret_cast<const uint32_t*>(&p);
    uint32_t acc = 0;
    for (uint32_t i = static_cast<uint32_t>(threadIdx.x - 64) * 8u; i < sizeof(GemmParams) / 4; i += 1024u)
      acc ^= pw[i];
    asm volatile("" ::"r"(acc));
  }
  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tmap_x);
    for (int s = 0; s < p.stages; ++s) {
      ptx::mbar_init(ptx::smem_addr(&bars->full[s]), 1 + p.x_warp);
      ptx::mbar_init(ptx::smem_addr(&bars->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(ptx::smem_addr(&bars->acc_full[a]), 1);
      // pair mode: the even CTA's accumulator is free once both epilogues have
      // read their halves (the odd CTA's epilogue arrives once, remotely)
      ptx::mbar_init(ptx::smem_addr(&bars->acc_empty[a]), pair ? 129 : 128);
    }
    ptx::mbar_init(ptx::smem_addr(&bars->peer_done), 1);
    ptx::mbar_init(ptx::smem_addr(&bars->ack), 1);
    if (pair)
      for (int s = 0; s < p.stages; ++s) ptx::mbar_init(ptx::smem_addr(&bars->peer_full[s]), 1);
    if (p.cluster > 1 && ptx::cluster_ctarank() == 0) {
      // Rank 0 expects every peer's partial of its tile (whole 16-token
      // chunks up to the valid tokens) as one bulk copy per peer. This precedes
      // its arrival on the cluster barrier, which every peer waits for
      // before its first store.
      int t, j_unused;
      block_tile(p, b0, t, j_unused);
      const int m_valid = min(p.npad, p.M - (t % p.m_tiles) * p.npad);
      const uint32_t bytes = static_cast<uint32_t>((p.cluster - 1) * ((m_valid + 15) >> 4)) * kTileRows * 64u;
      ptx::mbar_arrive_expect_tx(ptx::smem_addr(&bars->peer_done), bytes);
    }
    bars->abort_flag = 0;
    bars->fix_flag = 0;
    bars->npend = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (pair) {
      ptx::tmem_alloc_pair(ptx::smem_addr(&bars->tmem_base), p.tmem_cols);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(ptx::smem_addr(&bars->tmem_base), p.tmem_cols);
      ptx::tmem_relinquish();
    }
  }
  // Set-up barriers: the producers only need the mbarriers, so warp 0 (which
  // initialised them) releases the second producer warp (named barrier 2)
  // and the MMA and epilogue warps (named barrier 3, which also publishes the
  // tensor-memory address) without waiting for them. Every thread arrives on
  // the cluster barrier once here; a peer waits on it before its first store
  // into rank 0.
  auto setup_wait = [&]() -> uint32_t {
    if (in_cluster) ptx::cluster_arrive_relaxed();
    ptx::tc_fence_before();
    ptx::named_bar_sync(3, kGemmThreads);
    ptx::tc_fence_after();
    return bars->tmem_base;
  };
  volatile int* abort_flag = &bars->abort_flag;
  const Units units(p, b0, b1);
  const uint32_t smem_base = ptx::smem_addr(smem);

  // Loader warps: warp 0 (and warp 6 with two weight loaders) copy the weight
  // blocks; with x_warp the next warp copies the activation tiles.
  const int x_loader = p.x_warp ? 5 + p.producers : -1;
  const uint32_t bar2_threads = 32u * static_cast<uint32_t>(p.producers + p.x_warp);
  // Test build only (SPENSE_TEST_HOOKS): to exercise the failure path, every
  // loader waits (bounded) on a word nothing sets, before any copy is issued,
  // so the timeout leaves no transfer in flight.
  auto test_gate_wait = [&]() {
#ifdef SPENSE_TEST_HOOKS
    if (lane != 0 || p.test_gate == nullptr) return;
    const uint64_t t0 = ptx::globaltimer();
    while (*reinterpret_cast<const volatile unsigned int*>(p.test_gate) == 0u && !*abort_flag) {
      if (ptx::globaltimer() - t0 > kWaitLimitNs) {
        atomicOr(p.status, SPENSE_DEVICE_TIMEOUT_PRODUCER);
        *abort_flag = 1;
        break;
      }
      __nanosleep(1000);
    }
#endif
  };

  if (warp == x_loader) {
    // ------------------------------------------------------------ activation loader
    // The activation tile of every block, in the ring's order, as an issue
    // stream of its own: the copy engine serves each issuing thread's copies
    // one after another, so these small copies (the MMA needs them, and they
    // wait for the previous grid) do not queue behind the weight copies.
    ptx::named_bar_sync(2, bar2_threads);  // the barriers are initialised
    if (in_cluster) ptx::cluster_arrive_relaxed();
    test_gate_wait();
    if (lane == 0 && !*abort_flag) {
      ptx::griddep_wait();  // X may be written by the previous grid
      const uint64_t pol_x = ptx::policy_evict_last();
      // Pair mode: each CTA of the pair holds half of the token tile's rows.
      const int xrows = pair ? p.npad / 2 : p.npad;
      const uint32_t box = static_cast<uint32_t>(xrows) * 128u;        // smem bytes of a K-atom
      const uint32_t xb = static_cast<uint32_t>(p.box_rows) * 128u;    // bytes of one TMA box
      BlockWalker cx(units, p);
      Ring ring(static_cast<uint32_t>(p.stages));
      const int nb = b1 - b0;
      for (int i = 0; i < nb; ++i, ring.advance(), cx.advance(p)) {
        if (i >= p.stages && !wait_bar(ptx::smem_addr(&bars->empty[ring.s]), ring.ph ^ 1u, p.status,
                                       SPENSE_DEVICE_TIMEOUT_PRODUCER, abort_flag))
          break;
        const GemmMember& mb = p.mem[cx.member];
        const int y0 = cx.m_tile * p.npad + static_cast<int>(prank) * xrows;
        const uint32_t b_s = smem_base + ring.s * p.stage_bytes + kBlockBytes;
        const uint32_t full = ptx::smem_addr(&bars->full[ring.s]);
        if (cx.j < mb.nsb) {
          ptx::mbar_arrive_expect_tx(full, 2 * xb);
          ptx::tma_load_2d(b_s, &tmap_x, cx.j * kSparseBlockCols, y0, full, pol_x);
          ptx::tma_load_2d(b_s + box, &tmap_x, cx.j * kSparseBlockCols + 128, y0, full, pol_x);
        } else {
          ptx::mbar_arrive_expect_tx(full, xb);
          ptx::tma_load_2d(b_s, &tmap_x, mb.Ks + (cx.j - mb.nsb) * kDenseBlockCols, y0, full, pol_x);
        }
      }
    }
    __syncwarp();
  } else if (warp == 0 || (warp == 6 && p.producers > 1)) {
    // ------------------------------------------------------------ producer(s)
    // Blocks go through the ring in processing order. The weight copies of
    // the first ring's worth are issued before waiting on the previous grid
    // (the packed weights never depend on it), the activation tiles after
    // (unless the activation loader issues them). With two producer warps
    // (warps 0 and 6) each issues every other block: the copy engine serves
    // the two issue streams concurrently.
    if (warp == 0) {
      __syncwarp();  // lane 0 initialised the barriers
      if (in_cluster) ptx::cluster_arrive_relaxed();
      ptx::named_bar_arrive(3, kGemmThreads);
      if (bar2_threads > 32u) ptx::named_bar_arrive(2, bar2_threads);
    } else {
      ptx::named_bar_sync(2, bar2_threads);
      if (in_cluster) ptx::cluster_arrive_relaxed();
    }
    test_gate_wait();
    if (lane == 0 && !*abort_flag) {
      const int np = p.producers;
      const int me = warp == 0 ? 0 : 1;
      // Weights stream once (evict first), unless neighbouring token tiles
      // re-read them (then they stay in L2 for the second read).
      const uint64_t pol_w = p.w_keep ? ptx::policy_evict_normal() : ptx::policy_evict_first();
      const uint64_t pol_x = ptx::policy_evict_last();
      const uint32_t box = static_cast<uint32_t>(p.npad) * 128u;         // smem bytes of a K-atom
      // bytes one TMA box of activations loads (none here when the activation loader issues them)
      const uint32_t xbytes = p.x_warp ? 0u : static_cast<uint32_t>(p.box_rows) * 128u;
      const int nb = b1 - b0;
      const int pre = nb < p.stages ? nb : p.stages;
      auto issue_w = [&](const BlockWalker& c, uint32_t s) {
        const GemmMember& mb = p.mem[c.member];
        const uint32_t a_s = smem_base + s * p.stage_bytes;
        const uint32_t full = ptx::smem_addr(&bars->full[s]);
        const uint32_t piece = kBlockBytes / static_cast<uint32_t>(p.bulk_split);
        const int wt = c.weight_tile(p, prank);
        if (c.j < mb.nsb) {
          const size_t blk = static_cast<size_t>(wt) * mb.nsb + c.j;
          ptx::mbar_arrive_expect_tx(full, kBlockBytes + kMetaBlockBytes + 2 * xbytes);
          for (int q = 0; q < p.bulk_split; ++q)
            ptx::bulk_g2s(a_s + q * piece, mb.vs_t + blk * kBlockBytes + q * piece, piece, full, pol_w);
          ptx::bulk_g2s(a_s + kBlockBytes + p.b_bytes, mb.e_t + blk * kMetaBlockBytes, kMetaBlockBytes,
                        full, pol_w);
        } else {
          const size_t blk = static_cast<size_t>(wt) * mb.ndb + (c.j - mb.nsb);
          ptx::mbar_arrive_expect_tx(full, kBlockBytes + xbytes);
          for (int q = 0; q < p.bulk_split; ++q)
            ptx::bulk_g2s(a_s + q * piece, mb.wd_t + blk * kBlockBytes + q * piece, piece, full, pol_w);
        }
      };
      auto issue_x = [&](const BlockWalker& c, uint32_t s) {
        const int y0 = c.m_tile * p.npad;  // token tiles are npad tokens apart
        const uint32_t b_s = smem_base + s * p.stage_bytes + kBlockBytes;
        const uint32_t full = ptx::smem_addr(&bars->full[s]);
        const GemmMember& mb = p.mem[c.member];
        if (c.j < mb.nsb) {
          ptx::tma_load_2d(b_s, &tmap_x, c.j * kSparseBlockCols, y0, full, pol_x);
          ptx::tma_load_2d(b_s + box, &tmap_x, c.j * kSparseBlockCols + 128, y0, full, pol_x);
        } else {
          ptx::tma_load_2d(b_s, &tmap_x, mb.Ks + (c.j - mb.nsb) * kDenseBlockCols, y0, full, pol_x);
        }
      };
      BlockWalker cw(units, p);
      for (int i = 0; i < pre; ++i, cw.advance(p))
        if (i % np == me) issue_w(cw, static_cast<uint32_t>(i));
      if (p.l2_prefetch > 0) {
        // The weights past the first ring's worth are pulled into L2 while
        // this grid waits on the previous one, so the HBM keeps streaming
        // through the previous grid's tail; the ring later reads them from L2.
        BlockWalker cp = cw;
        const int last = min(nb, pre + p.l2_prefetch);
        for (int i = pre; i < last; ++i, cp.advance(p)) {
          if (i % np != me) continue;
          const GemmMember& mb = p.mem[cp.member];
          const int wt = cp.weight_tile(p, prank);
          if (cp.j < mb.nsb) {
            const size_t blk = static_cast<size_t>(wt) * mb.nsb + cp.j;
            ptx::prefetch_l2_bulk(mb.vs_t + blk * kBlockBytes, kBlockBytes);
            ptx::prefetch_l2_bulk(mb.e_t + blk * kMetaBlockBytes, kMetaBlockBytes);
          } else {
            const size_t blk = static_cast<size_t>(wt) * mb.ndb + (cp.j - mb.nsb);
            ptx::prefetch_l2_bulk(mb.wd_t + blk * kBlockBytes, kBlockBytes);
          }
        }
      }
      if (!p.x_warp) {
        ptx::griddep_wait();
        BlockWalker cx(units, p);
        for (int i = 0; i < pre; ++i, cx.advance(p))
          if (i % np == me) issue_x(cx, static_cast<uint32_t>(i));
      }
      Ring ring(static_cast<uint32_t>(p.stages));
      for (int i = 0; i < pre; ++i) ring.advance();
      for (int i = pre; i < nb; ++i, ring.advance(), cw.advance(p)) {
        if (i % np != me) continue;
        if (!wait_bar(ptx::smem_addr(&bars->empty[ring.s]), ring.ph ^ 1u, p.status,
                      SPENSE_DEVICE_TIMEOUT_PRODUCER, abort_flag))
          break;
        issue_w(cw, ring.s);
        if (!p.x_warp) issue_x(cw, ring.s);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    const uint32_t tmem_base = setup_wait();
    // Pair mode: before the first signal into the other CTA of the pair, its
    // barriers must be initialised (it arrived on the cluster barrier after).
    if (pair) ptx::cluster_wait();
    if (lane == 0 && pair && prank == 1) {
      // Odd CTA of a pair: relay. Its stages land on its own barriers; the
      // even CTA issues the pair's MMAs once both halves of a stage are in,
      // so each landed stage is announced to it.
      Ring ring(static_cast<uint32_t>(p.stages));
      const uint32_t peer_full0 = ptx::mapa(ptx::smem_addr(&bars->peer_full[0]), 0u);
      for (int i = 0; i < b1 - b0; ++i, ring.advance()) {
        if (!wait_bar(ptx::smem_addr(&bars->full[ring.s]), ring.ph, p.status, SPENSE_DEVICE_TIMEOUT_MMA,
                      abort_flag))
          break;
        ptx::mbar_arrive_remote_release(peer_full0 + 8u * ring.s);
      }
    } else if (lane == 0) {
      const uint32_t mma_m = pair ? 256u : 128u;
      const uint32_t idesc_sp = ptx::idesc_f8(static_cast<uint32_t>(p.npad), true, mma_m);
      const uint32_t idesc_d = ptx::idesc_f8(static_cast<uint32_t>(p.npad), false, mma_m);
      const uint32_t e_col0 = static_cast<uint32_t>(p.nacc * p.npad);
      const uint32_t box = static_cast<uint32_t>(pair ? p.npad / 2 : p.npad) * 128u;
      Ring ring(static_cast<uint32_t>(p.stages));
      uint32_t ebuf = 0;
      bool ok = true;
      // Completion signals: to this CTA, or in pair mode to both CTAs' barriers.
      auto commit = [&](uint32_t bar) {
        if constexpr (pair)
          ptx::mma_commit_pair(bar, 0x3);
        else
          ptx::mma_commit(bar);
      };
      for (int u = 0; ok && u < units.count; ++u) {
        int t, j0, j1;
        units.get(u, t, j0, j1);
        const uint32_t acc = static_cast<uint32_t>(u % p.nacc);
        const uint32_t aph = static_cast<uint32_t>((u / p.nacc) & 1);
        const uint32_t acc_bar = ptx::smem_addr(&bars->acc_empty[acc]);
        if (!(pair ? wait_bar_cluster(acc_bar, aph ^ 1u, p.status, SPENSE_DEVICE_TIMEOUT_MMA, abort_flag)
                   : wait_bar(acc_bar, aph ^ 1u, p.status, SPENSE_DEVICE_TIMEOUT_MMA, abort_flag))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(p.npad);
        const int nsb_u = p.mem[member_of(p, t / p.m_tiles)].nsb;  // 2:4 blocks of this tile
        for (int j = j0; j < j1; ++j, ring.advance()) {
          if (!wait_bar(ptx::smem_addr(&bars->full[ring.s]), ring.ph, p.status, SPENSE_DEVICE_TIMEOUT_MMA,
                        abort_flag) ||
              (pair && !wait_bar_cluster(ptx::smem_addr(&bars->peer_full[ring.s]), ring.ph, p.status,
                                         SPENSE_DEVICE_TIMEOUT_MMA, abort_flag))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_s = smem_base + ring.s * p.stage_bytes;
          const uint32_t b_s = a_s + kBlockBytes;
          const uint32_t e_s = b_s + p.b_bytes;
          if (j < nsb_u) {
            const uint32_t e_tmem = tmem_base + e_col0 + ebuf * 8u;
            if constexpr (pair) {
              ptx::tmem_cp_128x128b_pair(e_tmem, ptx::desc_rows16(e_s));
              ptx::tmem_cp_128x128b_pair(e_tmem + 4u, ptx::desc_rows16(e_s + 2048u));
            } else {
              ptx::tmem_cp_128x128b(e_tmem, ptx::desc_rows16(e_s));
              ptx::tmem_cp_128x128b(e_tmem + 4u, ptx::desc_rows16(e_s + 2048u));
            }
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
              const uint64_t ad = ptx::desc_sw128(a_s + 32u * k);
              const uint64_t bd = ptx::desc_sw128(b_s + (k >> 1) * box + (k & 1u) * 64u);
              const uint32_t accum = (j > j0 || k > 0) ? 1u : 0u;
              if constexpr (pair)
                ptx::mma_sp_f8_pair(d_tmem, ad, bd, e_tmem + 2u * k, idesc_sp, accum);
              else
                ptx::mma_sp_f8(d_tmem, ad, bd, e_tmem + 2u * k, idesc_sp, accum);
            }
            ebuf ^= 1u;
          } else {
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
              const uint64_t ad = ptx::desc_sw128(a_s + 32u * k);
              const uint64_t bd = ptx::desc_sw128(b_s + 32u * k);
              const uint32_t accum = (j > j0 || k > 0) ? 1u : 0u;
              if constexpr (pair)
                ptx::mma_f8_pair(d_tmem, ad, bd, idesc_d, accum);
              else
                ptx::mma_f8(d_tmem, ad, bd, idesc_d, accum);
            }
          }
          commit(ptx::smem_addr(&bars->empty[ring.s]));
        }
        if (!ok) break;
        commit(ptx::smem_addr(&bars->acc_full[acc]));
      }
      if (ok && p.cluster > 1 && ptx::cluster_ctarank() == 0 &&
          wait_bar_cluster(ptx::smem_addr(&bars->peer_done), 0, p.status, SPENSE_DEVICE_TIMEOUT_EPILOGUE,
                           abort_flag)) {
        // Every peer's copy has landed (so every peer is alive, waiting for
        // this): release them. Off the epilogue's path.
        for (int r = 1; r < p.cluster; ++r)
          ptx::mbar_arrive_remote_relaxed(ptx::mapa(ptx::smem_addr(&bars->ack), static_cast<uint32_t>(r)));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t tmem_base = setup_wait();
    ptx::griddep_wait();  // s_x, Y and the workspace may belong to the previous grid
    const int et = threadIdx.x - 64;  // 0..127
    const int quarter = warp & 3;     // tensor-memory lane quarter this warp may read
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const size_t slot_elems = static_cast<size_t>(kTileRows) * p.npad;
    // This warp's 1 KB of output staging (plans with room for it), after the barrier area.
    uint16_t* const wstage =
        p.ystage ? reinterpret_cast<uint16_t*>(smem + recv_off + p.recv_bytes + kBarrierBytes) + quarter * 512 : nullptr;
    // Token scales of the current token tile, staged in shared memory before
    // the accumulator is ready so no global load sits on the epilogue's path.
    int staged_m0 = -1;
    auto stage_sx = [&](int m0) {
      if (m0 == staged_m0) return;
      ptx::named_bar_sync(1, 128);  // earlier readers are done
      for (int i = et; i < p.npad; i += 128) bars->sx[i] = (m0 + i < p.M) ? __ldg(p.s_x + m0 + i) : 0.0f;
      ptx::named_bar_sync(1, 128);
      staged_m0 = m0;
    };

    // Fix-up of a shared tile by the epilogue warps while this CTA's MMAs go on.
    auto finish_tile = [&](int t) {
      stage_sx((t % p.m_tiles) * p.npad);
      fixup_tile(p, t, P, prank, et, 128, bars->sx);
    };

    // Tiles this CTA must finish. Their fix-ups wait until this CTA has
    // published the partials of all its shared tiles (which come first in the
    // processing order), so no other CTA's fix-up waits behind this one's.
    int pending[2];
    int npending = 0;
    if (p.cluster > 1 && units.count == 1) {
      // Cluster split: the S CTAs of a cluster hold consecutive K ranges of one
      // tile. Each peer stages its fp32 partial in its own (idle) ring and
      // sends it to rank 0's receive area with one bulk copy that counts down
      // rank 0's peer_done barrier; rank 0 adds the partials in rank order
      // and stores Y, while its MMA warp acknowledges the copies (a peer's
      // staging must outlive its copy).
      int t, j0, j1;
      units.get(0, t, j0, j1);
      const int n_tile = t / p.m_tiles;
      const int m0 = (t - n_tile * p.m_tiles) * p.npad;
      const GemmMember& mb = p.mem[member_of(p, n_tile)];
      const int m_valid = min(p.npad, p.M - m0);
      const int nchunk = (m_valid + 15) >> 4;
      const int n_base = (n_tile - mb.tile_begin) * kTileRows;
      const int n = n_base + row;
      const bool row_ok = n < mb.N;
      const uint32_t rank = ptx::cluster_ctarank();
      const float sw = (row_ok && rank == 0) ? __ldg(mb.s_w + n) : 0.0f;
      if (rank == 0) stage_sx(m0);
      const bool got = wait_bar(ptx::smem_addr(&bars->acc_full[0]), 0, p.status,
                                SPENSE_DEVICE_TIMEOUT_EPILOGUE, abort_flag);
      // Rank 0 also needs every peer's partial. The 128 threads take one
      // decision (they meet at named barriers below).
      const bool ready = ptx::named_bar_and(
          1, 128,
          got && (rank != 0 || wait_bar_cluster(ptx::smem_addr(&bars->peer_done), 0, p.status,
                                                SPENSE_DEVICE_TIMEOUT_EPILOGUE, abort_flag)));
      if (ready) {
        ptx::tc_fence_after();
        // Receive slot of peer r in rank 0: [r - 1][chunk][row][16 floats]; the
        // four 16-byte pieces of a row are rotated by (row >> 1) & 3 so that
        // eight consecutive rows cover all shared-memory banks.
        const uint32_t slot_bytes = static_cast<uint32_t>(kTileRows * p.npad) * 4u;
        const uint32_t row_off = static_cast<uint32_t>(row) * 64u;
        const uint32_t rot = static_cast<uint32_t>(row >> 1) & 3u;
        if (rank != 0) {
          // Rank 0's peer_done barrier is initialised and expects the bytes
          // once every CTA of the cluster has arrived from its set-up.
          ptx::cluster_wait();
          // Staging: the receive layout, [chunk][row][16 floats] with rotated
          // 16-byte pieces, from the start of this CTA's ring (every copy has
          // landed and every MMA has completed).
          for (int c = 0; c < nchunk; ++c) {
            uint32_t v[16];
            ptx::tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(c * 16), v);
            ptx::tmem_ld_wait();
            const uint32_t dst = smem_base + static_cast<uint32_t>(c) * (kTileRows * 64u) + row_off;
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q)
              ptx::st_smem_v4(dst + ((q ^ rot) << 4),
                              make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                          __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
          }
          ptx::tc_fence_before();
          ptx::fence_proxy_async_smem();
          ptx::named_bar_sync(1, 128);
          if (et == 0) {
            ptx::bulk_s2s_cluster(ptx::mapa(smem_base + recv_off + (rank - 1) * slot_bytes, 0), smem_base,
                                  static_cast<uint32_t>(nchunk) * (kTileRows * 64u),
                                  ptx::mapa(ptx::smem_addr(&bars->peer_done), 0));
          }
        } else {
          // Y tile staged as [16 tokens][128 rows] bf16 in the first ring stage
          // (idle: every copy has landed and every MMA has completed), then
          // written with 16-byte stores when the tile's rows are all in range.
          const bool vec = (n_base + kTileRows <= mb.N) && (mb.ldy % 8 == 0);
          uint16_t* ystage = reinterpret_cast<uint16_t*>(smem);
          for (int c = 0; c < nchunk; ++c) {
            const int c0 = c * 16;
            uint32_t v[16];
            ptx::tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(c0), v);
            ptx::tmem_ld_wait();
            float a[16], s16[16];
            load_sx16(bars->sx + c0, s16);
#pragma unroll
            for (int i = 0; i < 16; ++i) a[i] = __uint_as_float(v[i]);
            for (int r = 1; r < p.cluster; ++r) {
              const uint32_t src = smem_base + recv_off + (r - 1) * slot_bytes +
                                   static_cast<uint32_t>(c) * (kTileRows * 64u) + row_off;
#pragma unroll
              for (uint32_t q = 0; q < 4; ++q) {
                const float4 b = ptx::ld_smem_v4(src + ((q ^ rot) << 4));
                a[4 * q] += b.x;
                a[4 * q + 1] += b.y;
                a[4 * q + 2] += b.z;
                a[4 * q + 3] += b.w;
              }
            }
            if (vec) {
              if (c > 0) ptx::named_bar_sync(1, 128);  // the previous chunk's readers are done
#pragma unroll
              for (int i = 0; i < 16; ++i) ystage[i * kTileRows + row] = to_bf16_bits(a[i] * sw * s16[i]);
              ptx::named_bar_sync(1, 128);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int idx = et + 128 * h;  // 16-byte piece: token idx / 16, rows 8 * (idx % 16) ..
                const int m = c0 + (idx >> 4);
                if (m < m_valid)
                  ptx::st_global_v4(mb.y + static_cast<size_t>(m0 + m) * mb.ldy + n_base + 8 * (idx & 15),
                                    reinterpret_cast<const uint4*>(ystage)[idx]);
              }
            } else if (row_ok) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int m = c0 + i;
                if (m < m_valid)
                  mb.y[static_cast<size_t>(m0 + m) * mb.ldy + n] = to_bf16_bits(a[i] * sw * s16[i]);
              }
            }
          }
          ptx::tc_fence_before();
        }
      }
    }
    for (int u = 0; p.cluster <= 1 && u < units.count; ++u) {
      int t, j0, j1;
      units.get(u, t, j0, j1);
      const uint32_t acc = static_cast<uint32_t>(u % p.nacc);
      const uint32_t aph = static_cast<uint32_t>((u / p.nacc) & 1);
      const int n_tile = t / p.m_tiles;
      const int m0 = (t - n_tile * p.m_tiles) * p.npad;
      const GemmMember& mb = p.mem[member_of(p, n_tile)];
      const int m_valid = min(p.npad, p.M - m0);
      const int n = (P * (n_tile - mb.tile_begin) + static_cast<int>(prank)) * kTileRows + row;
      const bool row_ok = n < mb.N;
      int nb_t;
      const int tb = tile_block0(p, t, &nb_t);
      const bool whole = (j0 == 0 && j1 == nb_t);
      const float sw = (row_ok && whole) ? __ldg(mb.s_w + n) : 0.0f;
      if (whole) stage_sx(m0);
      const bool got = wait_bar(ptx::smem_addr(&bars->acc_full[acc]), aph, p.status,
                                SPENSE_DEVICE_TIMEOUT_EPILOGUE, abort_flag);
      // One decision for the 128 threads: they meet at named barriers below.
      if (!ptx::named_bar_and(1, 128, got)) break;
      ptx::tc_fence_after();
      const uint32_t taddr = lane_base + acc * static_cast<uint32_t>(p.npad);
      // Partials are stored [CTA][slot][npad][row] (token-major): slot 0 for the
      // tile holding the CTA's first block, slot 1 for the tile holding its last block.
      float* part = nullptr;
      if (!whole) {
        const int slot = (b0 >= tb) ? 0 : 1;
        part = p.partials + (static_cast<size_t>(g * P + prank) * 2 + slot) * slot_elems + row;  // token-major
      }
      for (int c0 = 0; c0 < m_valid; c0 += 16) {
        uint32_t v[16];
        ptx::tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(c0), v);
        ptx::tmem_ld_wait();
        if (whole) {
          float s16[16];
          load_sx16(bars->sx + c0, s16);
          const int nw = n - lane;  // the warp's first row
          if (wstage != nullptr && nw + 32 <= mb.N && (mb.ldy % 8) == 0) {
            // The warp's 32 rows of the chunk go out as 16-byte stores through
            // its 1 KB of staging, [16 tokens][32 rows] bf16 (one 2-byte store
            // per row and token took about 5x as long for a 128-token tile).
#pragma unroll
            for (int i = 0; i < 16; ++i)
              wstage[i * 32 + lane] = to_bf16_bits(__uint_as_float(v[i]) * sw * s16[i]);
            __syncwarp();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int q = lane + 32 * h;  // 16-byte piece: token q / 4, rows 8 (q % 4) .. 8 (q % 4) + 7
              const int m = c0 + (q >> 2);
              if (m < m_valid)
                ptx::st_global_v4(mb.y + static_cast<size_t>(m0 + m) * mb.ldy + nw + 8 * (q & 3),
                                  reinterpret_cast<const uint4*>(wstage)[q]);
            }
            __syncwarp();
          } else if (row_ok) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int m = c0 + i;
              if (m < m_valid)
                mb.y[static_cast<size_t>(m0 + m) * mb.ldy + n] = to_bf16_bits(__uint_as_float(v[i]) * sw * s16[i]);
            }
          }
        } else {
          // token-major partial: consecutive threads (rows) store consecutive words
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < m_valid) __stcg(part + static_cast<size_t>(c0 + i) * kTileRows, __uint_as_float(v[i]));
        }
      }
      ptx::tc_fence_before();
      if (pair && prank == 1) {
        // The pair's accumulator barrier lives in the even CTA: one arrival
        // there once all 128 threads of this CTA have read their rows.
        ptx::named_bar_sync(1, 128);
        if (et == 0) ptx::mbar_arrive_remote_release(ptx::mapa(ptx::smem_addr(&bars->acc_empty[acc]), 0u));
      } else {
        ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[acc]));
      }
      if (!whole) {
        // Publish this CTA's partial: the named barrier orders the 128 threads'
        // stores before thread 0's release-acquire ticket at GPU scope.
        ptx::named_bar_sync(1, 128);
        if (et == 0) {
          const int g_lo = block_owner(p, tb);
          const int g_hi = block_owner(p, tb + nb_t - 1);
          const unsigned int old = ptx::atom_add_acq_rel_gpu(p.counters + t * P + prank, 1u);
          bars->fix_flag = (old == static_cast<unsigned int>(g_hi - g_lo)) ? 1 : 0;
        }
        ptx::named_bar_sync(1, 128);
        if (*reinterpret_cast<volatile int*>(&bars->fix_flag) && npending < 2) pending[npending++] = t;
      }
      // Shared tiles come first; once the next unit is whole (or none is left),
      // every ticket of this CTA is out and the pending fix-ups can run.
      bool next_whole = true;
      if (u + 1 < units.count) {
        int t2, a2, b2;
        units.get(u + 1, t2, a2, b2);
        next_whole = (a2 == 0 && b2 == units.nblk_of(t2));
      }
      if (next_whole) {
        if (u + 1 == units.count) {
          // The CTA's last unit: its fix-ups run at the end with every warp.
          if (et == 0) {
            for (int i = 0; i < npending; ++i) bars->pend[i] = pending[i];
            bars->npend = npending;
          }
        } else {
          for (int i = 0; i < npending; ++i) finish_tile(pending[i]);
        }
        npending = 0;
      }
    }
  }

  __syncwarp();
  if (pair && prank == 1 && warp == 0 && lane == 0) {
    // The even CTA's completion signals land in this CTA's stage barriers
    // asynchronously: wait (bounded) for the last one of every stage before
    // this CTA may exit. After a failure they may never come; the wait runs out.
    const int nb = b1 - b0;
    const uint64_t t0 = ptx::globaltimer();
    for (int i = nb > p.stages ? nb - p.stages : 0; i < nb; ++i) {
      const uint32_t bar = ptx::smem_addr(&bars->empty[i % p.stages]);
      const uint32_t parity = static_cast<uint32_t>((i / p.stages) & 1);
      while (!ptx::mbar_try_wait(bar, parity) && ptx::globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  // Tensor memory is released before any cluster-barrier operation: a
  // dealloc issued after an arrival was measured to stall for microseconds,
  // keeping the CTA (and its SM slot) alive.
  if (warp == 1) {
    ptx::tc_fence_after();
    if constexpr (pair)
      ptx::tmem_dealloc_pair(bars->tmem_base, p.tmem_cols);
    else
      ptx::tmem_dealloc(bars->tmem_base, p.tmem_cols);
  }
  // Stream-K fix-ups left from the CTA's last unit, with every warp (the
  // loaders and the MMA warp are done): twice the loads in flight of the
  // epilogue warps alone, on the kernel's tail.
  const int npend = bars->npend;
  if (npend > 0) {
    ptx::griddep_wait();  // s_x and Y may belong to the previous grid (a no-op once it has completed)
    for (int i = 0; i < npend; ++i) {
      const int t = bars->pend[i];
      const int m0 = (t % p.m_tiles) * p.npad;
      if (i > 0) __syncthreads();  // the previous fix-up's readers of the scales are done
      for (int k = threadIdx.x; k < p.npad; k += blockDim.x) bars->sx[k] = m0 + k < p.M ? __ldg(p.s_x + m0 + k) : 0.0f;
      __syncthreads();
      fixup_tile(p, t, P, prank, threadIdx.x, blockDim.x, bars->sx);
    }
  }
  if (pair) {
    // Neither CTA of a pair leaves while the other may still signal into it:
    // every thread has arrived on the cluster barrier once at set-up (only the
    // MMA warp waited on that phase); all wait for it, then meet once more.
    if (warp != 1) ptx::cluster_wait();
    ptx::cluster_arrive();
    ptx::cluster_wait();
  }
  if (p.cluster > 1) {
    if (ptx::cluster_ctarank() != 0) {
      // A peer's staged partial must outlive its bulk copy: wait (bounded)
      // for rank 0's acknowledgement. Rank 0 only acknowledges on its success
      // path; after a failure elsewhere the wait runs out and the peer leaves.
      const uint64_t t0 = ptx::globaltimer();
      while (!ptx::mbar_try_wait_cluster(ptx::smem_addr(&bars->ack), 0) && ptx::globaltimer() - t0 < kWaitLimitNs) {
      }
    } else if (*abort_flag) {
      // Rank 0 never exits while a peer's copy may still write into it.
      const uint64_t t0 = ptx::globaltimer();
      while (!ptx::mbar_try_wait_cluster(ptx::smem_addr(&bars->peer_done), 0) &&
             ptx::globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  }
}

}  // namespace

uint32_t gemm_max_smem() { return 232448u; }

// Clusters may share SMs (two CTAs per SM) rather than spread one CTA per SM.
cudaClusterSchedulingPolicy cluster_policy() {
  static const cudaClusterSchedulingPolicy v = [] {
    const char* e = std::getenv("SPENSE_CLUSTER_POLICY");
    if (e != nullptr && e[0] == 's') return cudaClusterSchedulingPolicySpread;
    if (e != nullptr && e[0] == 'd') return cudaClusterSchedulingPolicyDefault;
    return cudaClusterSchedulingPolicyLoadBalancing;
  }();
  return v;
}

cudaError_t launch_gemm(const CUtensorMap& tmap_x, const GemmParams& p, uint32_t smem_bytes,
                        cudaStream_t stream) {
  static thread_local int configured_for = -1;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  if (configured_for != dev) {
    st = cudaFuncSetAttribute(spense_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(gemm_max_smem()));
    if (st == cudaSuccess)
      st = cudaFuncSetAttribute(spense_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(gemm_max_smem()));
    if (st != cudaSuccess) return st;
    configured_for = dev;
  }
  // Programmatic dependent launch: CTAs of this grid may start on SMs the
  // previous kernel in the stream has released; they prefetch weights and then
  // wait (griddepcontrol.wait) before reading anything that kernel may write.
  static const bool pdl = [] {
    const char* e = std::getenv("SPENSE_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>(p.grid * (p.pair ? 2 : 1)));
  cfg.blockDim = dim3(kGemmThreads + 32 * (p.producers - 1) + 32 * p.x_warp);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned int>(p.pair ? 2 : (p.cluster > 1 ? p.cluster : 1));
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  attr[2].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[2].val.clusterSchedulingPolicyPreference = cluster_policy();
  cfg.attrs = attr;
  cfg.numAttrs = (p.cluster > 1 || p.pair) ? 3 : 2;
  return p.pair ? cudaLaunchKernelEx(&cfg, spense_gemm_kernel<true>, tmap_x, p)
                : cudaLaunchKernelEx(&cfg, spense_gemm_kernel<false>, tmap_x, p);
}

}  // namespace spense
