// spense_pack kernels: split an FP8 weight matrix into its 2:4 region and its
// dense region and write both in the tiled, swizzled layout the GEMM streams.
//
// Page: "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs
// for LLM Inference" (gist.science technical summary), Technical Summary §1
// (2:4: two of every four consecutive weights are zero), §2.A (a contiguous 2:4
// region and a contiguous dense region), §2.B (the dense columns are the tail,
// or an index set permuted into one contiguous block).
//
// The work is integer only: selection compares e4m3 magnitudes as the unsigned
// value of (byte & 0x7F), which orders e4m3fn magnitudes exactly.
#include <algorithm>
#include <cstdint>

#include "pdl.cuh"
#include "spense_internal.h"

namespace spense {
namespace {

__device__ __forceinline__ bool e4m3_is_nan(uint8_t b) { return (b & 0x7F) == 0x7F; }

// Swizzled offset of 16-byte chunk `chunk` of row `r` inside a 128 x 128-byte block.
__device__ __forceinline__ int sw128_off(int r, int chunk) {
  return r * 128 + ((chunk ^ (r & 7)) << 4);
}

// One thread per (row, 32 compacted sparse columns = 8 groups of four).
template <bool kTail>
__global__ void __launch_bounds__(256) pack_sparse_kernel(
    const uint8_t* __restrict__ W, const uint8_t* __restrict__ mask,
    const int32_t* __restrict__ perm, int64_t N, int64_t K, int64_t Ks, int nsb,
    uint8_t* __restrict__ vs_t, uint8_t* __restrict__ e_t, uint8_t* __restrict__ vs_c,
    uint8_t* __restrict__ e_c, unsigned int* __restrict__ err) {
  const int64_t chunks = static_cast<int64_t>(nsb) * 8;
  const int64_t n_pad = (N + kTileRows - 1) / kTileRows * kTileRows;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= n_pad * chunks) return;
  const int64_t n = tid / chunks;
  const int c = static_cast<int>(tid % chunks);
  const int r = static_cast<int>(n % kTileRows);
  const int64_t tile = n / kTileRows;

  uint8_t vals[16];
  uint8_t meta[4] = {0, 0, 0, 0};
  unsigned int e = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int64_t g = static_cast<int64_t>(c) * 8 + q;
    uint8_t b[4] = {0, 0, 0, 0};
    uint32_t kept = 0;
    if (n < N && 4 * g < Ks) {
      int64_t col[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) col[i] = kTail ? 4 * g + i : perm[4 * g + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        b[i] = W[n * K + col[i]];
        if (e4m3_is_nan(b[i])) e |= kPackErrNaN;
      }
      if (mask != nullptr) {
#pragma unroll
        for (int i = 0; i < 4; ++i) kept |= (mask[n * K + col[i]] != 0 ? 1u : 0u) << i;
        if (__popc(kept) > 2) e |= kPackErrMask;
      } else {
        // Entry i survives when fewer than two entries beat it on
        // (magnitude descending, index ascending).
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          int beaten = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int mi = b[i] & 0x7F, mj = b[j] & 0x7F;
            beaten += (j != i) && (mj > mi || (mj == mi && j < i));
          }
          kept |= (beaten < 2 ? 1u : 0u) << i;
        }
      }
    }
    // Stored pair: the kept indices, completed by the lowest unkept ones.
    uint32_t sel = kept;
    while (__popc(sel) < 2) sel |= ~sel & (sel + 1);
    const int i0 = __ffs(static_cast<int>(sel)) - 1;
    const int i1 = 31 - __clz(static_cast<int>(sel));
    vals[2 * q + 0] = ((kept >> i0) & 1u) ? b[i0] : 0;
    vals[2 * q + 1] = ((kept >> i1) & 1u) ? b[i1] : 0;
    meta[q >> 1] |= static_cast<uint8_t>((i0 | (i1 << 2)) << (4 * (q & 1)));
  }
  if (e) atomicOr(err, e);

  // Tiled stores: 16 value bytes = one swizzled chunk; 4 metadata bytes.
  const int blk = c >> 3;
  uint4 v;
  v.x = vals[0] | (vals[1] << 8) | (vals[2] << 16) | (static_cast<uint32_t>(vals[3]) << 24);
  v.y = vals[4] | (vals[5] << 8) | (vals[6] << 16) | (static_cast<uint32_t>(vals[7]) << 24);
  v.z = vals[8] | (vals[9] << 8) | (vals[10] << 16) | (static_cast<uint32_t>(vals[11]) << 24);
  v.w = vals[12] | (vals[13] << 8) | (vals[14] << 16) | (static_cast<uint32_t>(vals[15]) << 24);
  uint8_t* vdst = vs_t + (tile * nsb + blk) * kBlockBytes + sw128_off(r, c & 7);
  *reinterpret_cast<uint4*>(vdst) = v;
  const uint32_t m32 =
      meta[0] | (meta[1] << 8) | (meta[2] << 16) | (static_cast<uint32_t>(meta[3]) << 24);
  const int half = (c & 7) >> 2;
  uint8_t* edst = e_t + ((tile * nsb + blk) * 2 + half) * 2048 + r * 16 + 4 * (c & 3);
  *reinterpret_cast<uint32_t*>(edst) = m32;

  if (n < N) {
    if (vs_c != nullptr) {
      for (int j = 0; j < 16; ++j) {
        const int64_t col = static_cast<int64_t>(c) * 16 + j;
        if (col < Ks / 2) vs_c[n * (Ks / 2) + col] = vals[j];
      }
    }
    if (e_c != nullptr) {
      for (int j = 0; j < 4; ++j) {
        const int64_t col = static_cast<int64_t>(c) * 4 + j;
        if (col < Ks / 8) e_c[n * (Ks / 8) + col] = meta[j];
      }
    }
  }
}

// One thread per (row, 16 dense columns).
template <bool kTail>
__global__ void __launch_bounds__(256) pack_dense_kernel(
    const uint8_t* __restrict__ W, const int32_t* __restrict__ perm, int64_t N, int64_t K,
    int64_t Kd, int ndb, uint8_t* __restrict__ wd_t, uint8_t* __restrict__ wd_c,
    unsigned int* __restrict__ err) {
  const int64_t chunks = static_cast<int64_t>(ndb) * 8;
  const int64_t n_pad = (N + kTileRows - 1) / kTileRows * kTileRows;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= n_pad * chunks) return;
  const int64_t n = tid / chunks;
  const int c = static_cast<int>(tid % chunks);
  const int r = static_cast<int>(n % kTileRows);
  const int64_t tile = n / kTileRows;
  const int64_t Ks = K - Kd;

  uint4 v = make_uint4(0, 0, 0, 0);
  const int64_t d0 = static_cast<int64_t>(c) * 16;
  if (n < N && d0 < Kd) {  // Kd % 16 == 0: a chunk is wholly inside or outside
    uint8_t vals[16];
    unsigned int e = 0;
    if (kTail) {
      v = *reinterpret_cast<const uint4*>(W + n * K + Ks + d0);
      const uint8_t* pv = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
      for (int j = 0; j < 16; ++j) vals[j] = pv[j];
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) vals[j] = W[n * K + perm[Ks + d0 + j]];
      v.x = vals[0] | (vals[1] << 8) | (vals[2] << 16) | (static_cast<uint32_t>(vals[3]) << 24);
      v.y = vals[4] | (vals[5] << 8) | (vals[6] << 16) | (static_cast<uint32_t>(vals[7]) << 24);
      v.z = vals[8] | (vals[9] << 8) | (vals[10] << 16) | (static_cast<uint32_t>(vals[11]) << 24);
      v.w = vals[12] | (vals[13] << 8) | (vals[14] << 16) | (static_cast<uint32_t>(vals[15]) << 24);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (e4m3_is_nan(vals[j])) e |= kPackErrNaN;
    if (e) atomicOr(err, e);
    if (wd_c != nullptr) *reinterpret_cast<uint4*>(wd_c + n * Kd + d0) = v;
  }
  *reinterpret_cast<uint4*>(wd_t + (tile * ndb + (c >> 3)) * kBlockBytes + sw128_off(r, c & 7)) = v;
}

// X'[m][j] = X[m][perm[j]]; one thread per 4 output bytes.
// dst row r = src row rows[r] (K bytes each, K % 16 == 0), and the same for
// one float per row when scales are given.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ src, int64_t K,
                                                          const int32_t* __restrict__ rows, int64_t N,
                                                          uint8_t* __restrict__ dst, const float* __restrict__ ssrc,
                                                          float* __restrict__ sdst) {
  const int64_t q = K / 16;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < N * q;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / q, c = t - r * q;
    const int64_t sr = rows[r];
    reinterpret_cast<uint4*>(dst + r * K)[c] = reinterpret_cast<const uint4*>(src + sr * K)[c];
    if (c == 0 && ssrc != nullptr) sdst[r] = ssrc[sr];
  }
}

__global__ void __launch_bounds__(256) gather_kernel(const uint8_t* __restrict__ X,
                                                     const int32_t* __restrict__ perm, int64_t M,
                                                     int64_t K, uint8_t* __restrict__ Xg) {
  pdl_trigger();  // the GEMM that reads Xg may start prefetching its weights
  pdl_wait();     // X may be written by the previous kernel
  const int64_t quads = K / 4;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < M * quads;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = t / quads;
    const int64_t j = (t % quads) * 4;
    const uint8_t* xr = X + m * K;
    const uint32_t w = xr[perm[j]] | (xr[perm[j + 1]] << 8) | (xr[perm[j + 2]] << 16) |
                       (static_cast<uint32_t>(xr[perm[j + 3]]) << 24);
    *reinterpret_cast<uint32_t*>(Xg + m * K + j) = w;
  }
}

inline unsigned int blocks_for(int64_t threads) {
  return static_cast<unsigned int>((threads + 255) / 256);
}

}  // namespace

cudaError_t launch_pack(const uint8_t* W, const uint8_t* mask, const int32_t* perm, int64_t N,
                        int64_t K, int64_t Kd, uint8_t* vs_t, uint8_t* e_t, uint8_t* wd_t,
                        uint8_t* vs_c, uint8_t* e_c, uint8_t* wd_c, unsigned int* err,
                        cudaStream_t stream) {
  const int64_t Ks = K - Kd;
  const int nsb = static_cast<int>((Ks + kSparseBlockCols - 1) / kSparseBlockCols);
  const int ndb = static_cast<int>((Kd + kDenseBlockCols - 1) / kDenseBlockCols);
  const int64_t n_pad = (N + kTileRows - 1) / kTileRows * kTileRows;
  if (nsb > 0) {
    const int64_t threads = n_pad * nsb * 8;
    if (perm == nullptr)
      pack_sparse_kernel<true><<<blocks_for(threads), 256, 0, stream>>>(
          W, mask, perm, N, K, Ks, nsb, vs_t, e_t, vs_c, e_c, err);
    else
      pack_sparse_kernel<false><<<blocks_for(threads), 256, 0, stream>>>(
          W, mask, perm, N, K, Ks, nsb, vs_t, e_t, vs_c, e_c, err);
    cudaError_t st = cudaGetLastError();
    if (st != cudaSuccess) return st;
  }
  if (ndb > 0) {
    const int64_t threads = n_pad * ndb * 8;
    if (perm == nullptr)
      pack_dense_kernel<true><<<blocks_for(threads), 256, 0, stream>>>(W, perm, N, K, Kd, ndb, wd_t,
                                                                       wd_c, err);
    else
      pack_dense_kernel<false><<<blocks_for(threads), 256, 0, stream>>>(W, perm, N, K, Kd, ndb, wd_t,
                                                                        wd_c, err);
    cudaError_t st = cudaGetLastError();
    if (st != cudaSuccess) return st;
  }
  return cudaSuccess;
}

cudaError_t launch_gather_rows(const uint8_t* src, int64_t K, const int32_t* rows, int64_t N, uint8_t* dst,
                               const float* ssrc, float* sdst, cudaStream_t stream) {
  const int64_t threads = N * (K / 16);
  const unsigned int grid = static_cast<unsigned int>(std::min<int64_t>(blocks_for(threads), 4096));
  gather_rows_kernel<<<grid, 256, 0, stream>>>(src, K, rows, N, dst, ssrc, sdst);
  return cudaGetLastError();
}

cudaError_t launch_gather(const uint8_t* X, const int32_t* perm, int64_t M, int64_t K, uint8_t* Xg,
                          cudaStream_t stream) {
  const int64_t threads = M * (K / 4);
  const unsigned int grid = static_cast<unsigned int>(std::min<int64_t>(blocks_for(threads), 4096));
  return launch_pdl(gather_kernel, grid, 256, 0, stream, X, perm, M, K, Xg);
}

}  // namespace spense
