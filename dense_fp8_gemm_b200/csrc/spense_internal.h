// Internal declarations shared by the host ABI and the kernels of the Spense
// library. Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "spense.h"

namespace spense {

constexpr int kTileRows = 128;          // weight rows per tile (MMA M)
constexpr int kSparseBlockCols = 256;   // compacted sparse columns per block
constexpr int kDenseBlockCols = 128;    // dense columns per block
constexpr int kBlockBytes = 16384;      // 128 rows x 128 bytes (values or dense weights)
constexpr int kMetaBlockBytes = 4096;   // 2 halves x 128 rows x 16 bytes
constexpr int kMaxTokenTile = 256;      // tokens per tile (MMA N upper bound)
constexpr int kCostSparse = 5;          // HBM bytes of a sparse block in 4 KiB units (16 + 4 KiB)
constexpr int kCostDense = 4;           // ... of a dense block (16 KiB)
constexpr int kGemmThreads = 192;       // warp 0 loads, warp 1 issues MMAs, warps 2-5 epilogue
constexpr int kGemmThreadsMax = 256;    // plus a second weight loader and an activation loader
constexpr int kMaxStages = 12;
constexpr uint32_t kBarrierBytes = 2048;  // mbarriers, flags and staged token scales
constexpr uint32_t kYStageBytes = 4096;   // whole-tile output staging: 16 tokens x 32 rows bf16 per epilogue warp

// Workspace layout: [header 256 B][counters][partials][gathered X][host staging]
struct WorkspaceLayout {
  size_t counters_off, counters_bytes;
  size_t partials_off, partials_bytes;
  size_t xg_off, xg_bytes;
  size_t stage_x_off, stage_sx_off, stage_y_off;
  size_t total_device;  // bytes for spense_gemm
  size_t total_host;    // bytes for spense_gemm_host
};

constexpr int kMaxGroup = 4;    // weight matrices sharing one activation tensor in one launch
constexpr int kMaxGrid = 320;   // work units per launch (CTAs, up to two per SM; or CTA pairs)

struct GemmPlan {
  int npad;        // MMA N (tokens per tile, multiple of 16)
  int box_rows;    // activation rows one TMA box loads (<= npad)
  int m_tiles;
  int n_tiles;     // row tiles over all group members
  int tiles;       // n_tiles * m_tiles
  int count;                                // weight matrices in the launch
  int mem_tiles[kMaxGroup];                 // row tiles of member i
  int mem_nsb[kMaxGroup], mem_ndb[kMaxGroup];  // 2:4 / dense blocks per tile of member i
  int mem_cost[kMaxGroup];                  // kCostSparse * nsb + kCostDense * ndb
  int mem_block_begin[kMaxGroup];           // first linear block of member i
  long long mem_cost_begin[kMaxGroup + 1];  // streamed weight before member i's first tile
  int min_tile_cost;
  bool any_sparse;
  long long total_cost;
  int grid;        // CTAs
  int stages;
  uint32_t stage_bytes;
  uint32_t b_bytes;  // bytes of the activation region of a stage
  int nacc;          // accumulator buffers in tensor memory
  uint32_t tmem_cols;
  uint32_t smem_bytes;
  int ctas_per_sm;
  int bulk_split;
  int producers;
  int cluster;
  uint32_t recv_bytes;
  int pair;        // 1: CTA pairs (tcgen05 cta_group::2) share 256-row MMAs; the work units are pairs
  uint32_t ystage; // bytes of output staging after the barrier area (0 or kYStageBytes)
  int cta_start[kMaxGrid + 1];  // first linear block of each work unit (CTA, or pair); [grid] = total blocks
  WorkspaceLayout ws;
};

// One weight matrix of a launch: its packed blocks, scales, output and the
// first global row tile it occupies.
struct GemmMember {
  const uint8_t* vs_t;
  const uint8_t* e_t;
  const uint8_t* wd_t;
  const float* s_w;
  uint16_t* y;       // row m of the output at y + m * ldy
  int N;
  int tile_begin;    // first global row tile
  int nsb, ndb;      // 2:4 blocks and dense blocks per row tile
  int nblk;          // nsb + ndb
  int Ks;            // X column where the dense region starts
  int block_begin;   // first linear block of the member's tiles
  int ldy;           // output row stride in elements (>= N)
  int row_tiles;     // 128-row tiles of the member (pair mode: its tiles above count pairs of them)
};

struct GemmParams {
  GemmMember mem[kMaxGroup];
  int n_members;
  const float* s_x;
  float* partials;
  unsigned int* counters;
  unsigned int* status;
  int M;
  int n_tiles, m_tiles;
  int npad, box_rows, grid, stages, nacc;
  uint32_t stage_bytes, b_bytes;
  uint32_t tmem_cols;
  int cta_start[kMaxGrid + 1];
  int bulk_split;  // weight block copied as this many bulk copies (1, 2 or 4)
  int producers;   // loader warps (1 or 2)
  int cluster;     // > 1: CTAs of a cluster split one tile's K and reduce through shared memory
  const unsigned int* test_gate;  // test only: loaders wait (bounded) until this word is nonzero
  uint32_t recv_bytes;            // cluster mode: rank 0's receive area for the peers' partials
  int l2_prefetch;                // blocks past the first ring's worth prefetched into L2 at start
  int x_warp;                     // 1: a warp of its own issues the activation-tile loads
  int w_keep;                     // 1: weight copies use the evict-normal L2 policy (re-read by token tiles)
  int pair;                       // 1: pair mode (grid = 2 CTAs per work unit, cluster of 2, M = 256 MMAs)
  uint32_t ystage;                // stream-K: 1 KB of output staging per epilogue warp after the barriers, or 0
};

// Kernels (defined in the .cu files).
cudaError_t launch_pack(const uint8_t* W, const uint8_t* mask, const int32_t* perm, int64_t N,
                        int64_t K, int64_t Kd, uint8_t* vs_t, uint8_t* e_t, uint8_t* wd_t,
                        uint8_t* vs_c, uint8_t* e_c, uint8_t* wd_c, unsigned int* err,
                        cudaStream_t stream);
cudaError_t launch_gather(const uint8_t* X, const int32_t* perm, int64_t M, int64_t K, uint8_t* Xg,
                          cudaStream_t stream);
cudaError_t launch_gather_rows(const uint8_t* src, int64_t K, const int32_t* rows, int64_t N, uint8_t* dst,
                               const float* ssrc, float* sdst, cudaStream_t stream);
cudaError_t launch_gemm(const CUtensorMap& tmap_x, const GemmParams& p, uint32_t smem_bytes,
                        cudaStream_t stream);
uint32_t gemm_max_smem();
size_t score_workspace_bytes(int64_t I);
cudaError_t launch_score_glu(const uint8_t* gate, const float* s_gate, const uint8_t* up, const float* s_up,
                             int64_t I, int64_t H, const uint8_t* down, const float* s_down, const float* h_in,
                             const float* h_mid, float* score, float* partial, cudaStream_t stream);
cudaError_t launch_select_top(const float* score, int64_t I, int64_t Kd, int32_t* out, cudaStream_t stream);
cudaError_t launch_quantize(const uint16_t* X, int64_t M, int64_t K, const int32_t* perm, uint8_t* Xq,
                            float* s_x, int sms, cudaStream_t stream);

// Device error bits written by the pack kernel.
constexpr unsigned int kPackErrMask = 1u;
constexpr unsigned int kPackErrNaN = 2u;

}  // namespace spense
