// SpenseGPT+ dense-index selection on the GPU: importance scores of the
// intermediate indices of a GLU MLP, then the top-Kd of them.
//
// Page: "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs
// for LLM Inference" (gist.science technical summary), Technical Summary §2.B:
// SpenseGPT+ scores each intermediate index by aggregating contributions
// across the gate, up and down projections with the Wanda-style score
// S_ij = |W_ij| sqrt(H_jj), and keeps the top-scoring indices dense. This
// library's reading (weights are e4m3 codes times fp32 row scales; h_in and
// h_mid are the diagonals of the input Hessians of gate/up and of down):
//   score[t] = |s_gate[t]| sum_j |gate[t][j]| sqrt(h_in[j])
//            + |s_up[t]|   sum_j |up[t][j]|   sqrt(h_in[j])
//            + sqrt(h_mid[t]) sum_i |s_down[i]| |down[i][t]|
// Sums are fp32 in a fixed order (deterministic). All three weight matrices are
// read once: the work is bound by HBM bandwidth.
#include <cstdint>

#include "spense_internal.h"

namespace spense {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreRowChunks = 64;  // row chunks of down summed separately, then in order
constexpr int kColThreads = 128;

// |value| of an e4m3 code (bias 7, 3 mantissa bits, subnormals m * 2^-9) times
// 2^-120. The seven magnitude bits placed at float bit 20 give a float whose
// exponent field is e and whose top mantissa bits are m: its value is
// 2^(e-127) (1 + m/8), or (m/8) 2^-126 when e = 0 (an fp32 denormal), i.e.
// exactly 2^-120 times the e4m3 value. Sums of such terms stay far from the
// fp32 limits; the factor 2^120 is applied once per sum. (fp32 denormals are
// kept: the library is not built with flush-to-zero.) NaN codes (0x7F, 0xFF)
// are not valid weights here.
__device__ __forceinline__ float e4m3_abs(uint32_t code) { return __uint_as_float((code & 0x7Fu) << 20) * 0x1p120f; }

// sum over the 4 codes of a word of |value| * sq, times 2^-120: the word's
// sign bits are cleared once, then each code is one shift and one mask away
// from float bit 20.
__device__ __forceinline__ float sum4_scaled(uint32_t w, const float* sq, float acc) {
  const uint32_t m = w & 0x7F7F7F7Fu;
  acc = fmaf(__uint_as_float((m << 20) & 0x07F00000u), sq[0], acc);
  acc = fmaf(__uint_as_float((m << 12) & 0x07F00000u), sq[1], acc);
  acc = fmaf(__uint_as_float((m << 4) & 0x07F00000u), sq[2], acc);
  acc = fmaf(__uint_as_float((m >> 4) & 0x07F00000u), sq[3], acc);
  return acc;
}

// sum over 16 codes of |value| * sq, times 2^-120
__device__ __forceinline__ float sum16_scaled(uint4 v, const float* sq) {
  float acc = 0.0f;
  acc = sum4_scaled(v.x, sq, acc);
  acc = sum4_scaled(v.y, sq + 4, acc);
  acc = sum4_scaled(v.z, sq + 8, acc);
  acc = sum4_scaled(v.w, sq + 12, acc);
  return acc;
}

// Largest hidden size whose sqrt(h_in) is staged in shared memory.
constexpr int64_t kScoreStageH = 16384;

// gate/up terms: one warp per intermediate index t (a row of gate and of up),
// the warps of a persistent grid taking rows in turn; sqrt(h_in) is computed
// once per CTA into shared memory (when H fits).
template <bool kStaged>
__global__ void __launch_bounds__(kScoreThreads) score_rows_kernel(const uint8_t* __restrict__ gate,
                                                                   const float* __restrict__ s_gate,
                                                                   const uint8_t* __restrict__ up,
                                                                   const float* __restrict__ s_up, int64_t I,
                                                                   int64_t H, const float* __restrict__ h_in,
                                                                   float* __restrict__ score) {
  extern __shared__ float sq_all[];  // kStaged: sqrt(h_in), H floats
  if (kStaged) {
    for (int64_t j = threadIdx.x; j < H; j += kScoreThreads) sq_all[j] = sqrtf(__ldg(h_in + j));
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kScoreThreads / 32);
  const int64_t nc = H / 16;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kScoreThreads / 32) + (threadIdx.x >> 5); t < I;
       t += nwarps) {
    float ag = 0.0f, au = 0.0f;
    const uint4* gr = gate ? reinterpret_cast<const uint4*>(gate + t * H) : nullptr;
    const uint4* ur = up ? reinterpret_cast<const uint4*>(up + t * H) : nullptr;
    for (int64_t c0 = lane; c0 < nc; c0 += 4 * 32) {
      // four chunks per lane in flight before any is used
      uint4 gv[4], uv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = c0 + 32 * u;
        gv[u] = (gr && c < nc) ? __ldg(gr + c) : make_uint4(0u, 0u, 0u, 0u);
        uv[u] = (ur && c < nc) ? __ldg(ur + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = c0 + 32 * u;
        if (c >= nc) break;
        float sq[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) sq[i] = kStaged ? sq_all[c * 16 + i] : sqrtf(__ldg(h_in + c * 16 + i));
        ag += sum16_scaled(gv[u], sq);
        au += sum16_scaled(uv[u], sq);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ag += __shfl_xor_sync(0xffffffffu, ag, o);
      au += __shfl_xor_sync(0xffffffffu, au, o);
    }
    if (lane == 0) {
      float r = 0.0f;
      if (gr) r += fabsf(__ldg(s_gate + t)) * (ag * 0x1p120f);
      if (ur) r += fabsf(__ldg(s_up + t)) * (au * 0x1p120f);
      score[t] = r;
    }
  }
}

// down term, part 1: columns t .. t+15 per thread, rows of chunk blockIdx.y.
__global__ void __launch_bounds__(kColThreads) score_cols_kernel(const uint8_t* __restrict__ down,
                                                                 const float* __restrict__ s_down, int64_t I,
                                                                 int64_t H, float* __restrict__ partial) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kColThreads + threadIdx.x;  // 16-column chunk
  if (c >= I / 16) return;
  const int64_t i0 = H * blockIdx.y / kScoreRowChunks, i1 = H * (blockIdx.y + 1) / kScoreRowChunks;
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.0f;
#pragma unroll 8
  for (int64_t i = i0; i < i1; ++i) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(down + i * I) + c);
    const float s = fabsf(__ldg(s_down + i));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[4 * h + b] = fmaf(s, e4m3_abs((w[h] >> (8 * b)) & 0xFFu), acc[4 * h + b]);
  }
  float* out = partial + static_cast<int64_t>(blockIdx.y) * I + c * 16;
#pragma unroll
  for (int k = 0; k < 16; k += 4)
    *reinterpret_cast<float4*>(out + k) = make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]);
}

// down term, part 2: the chunks' partial sums in chunk order, times sqrt(h_mid).
__global__ void __launch_bounds__(kScoreThreads) score_finish_kernel(const float* __restrict__ partial, int64_t I,
                                                                     const float* __restrict__ h_mid,
                                                                     float* __restrict__ score) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kScoreThreads + threadIdx.x;
  if (t >= I) return;
  float col = 0.0f;
  for (int r = 0; r < kScoreRowChunks; ++r) col += __ldg(partial + static_cast<int64_t>(r) * I + t);
  score[t] += sqrtf(__ldg(h_mid + t)) * col;
}

// Top-Kd selection in one CTA: a four-pass radix select over the score bits
// (non-negative floats order like their bit patterns, counted in one
// histogram per warp) finds the Kd-th largest value T; then every score above
// T and the lowest indices among the scores equal to T are kept, written in
// ascending index order: each thread owns a contiguous segment of indices,
// one block-wide scan of its (above, equal) counts gives where its kept
// indices go.
constexpr int kSelectThreads = 1024;

// Exclusive block-wide prefix sum of a 64-bit value (all threads call it).
__device__ __forceinline__ uint64_t block_exclusive_scan(uint64_t v, uint64_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint64_t w = lane < kSelectThreads / 32 ? warp_tot[lane] : 0;
    uint64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < kSelectThreads / 32) warp_tot[lane] = wi - w;  // exclusive
  }
  __syncthreads();
  return warp_tot[warp] + inc - v;
}

template <bool kStaged>
__global__ void __launch_bounds__(kSelectThreads) select_top_kernel(const float* __restrict__ score_g, int64_t I,
                                                                    int64_t Kd, int32_t* __restrict__ out) {
  extern __shared__ float score_s[];  // kStaged: the I scores
  if (kStaged) {
    // eight loads in flight per thread: one CTA has to pull the whole array
    for (int64_t t0 = threadIdx.x; t0 < I; t0 += 8 * kSelectThreads) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t t = t0 + static_cast<int64_t>(u) * kSelectThreads;
        v[u] = t < I ? __ldg(score_g + t) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t t = t0 + static_cast<int64_t>(u) * kSelectThreads;
        if (t < I) score_s[t] = v[u];
      }
    }
  }
  const float* score = kStaged ? score_s : score_g;
  __shared__ unsigned int hist[256];
  __shared__ unsigned int whist[kSelectThreads / 32][256];  // one histogram per warp
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int64_t s_need;
  __shared__ uint64_t warp_tot[kSelectThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_need = Kd;  // rank (from the top, 1-based) of T among the scores matching the prefix
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int bb = lane; bb < 256; bb += 32) whist[warp][bb] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int64_t t = threadIdx.x; t < I; t += kSelectThreads) {
      const uint32_t u = __float_as_uint(score[t]);
      if ((u & mask) == prefix) atomicAdd(&whist[warp][(u >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    for (int bb = threadIdx.x; bb < 256; bb += kSelectThreads) {
      unsigned int c = 0;
      for (int w = 0; w < kSelectThreads / 32; ++w) c += whist[w][bb];
      hist[bb] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255 - 8l .. 248 - 8l (from the top); counts above a
      // lane's bins come from an exclusive scan across lanes
      unsigned int h[8];
      unsigned int tot = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        h[k] = hist[255 - 8 * lane - k];
        tot += h[k];
      }
      unsigned int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      int64_t above = static_cast<int64_t>(incl - tot);
      const int64_t need = s_need;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int bin = 255 - 8 * lane - k;
        if (above < need && need <= above + static_cast<int64_t>(h[k])) {
          s_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
          s_mask = mask | (0xFFu << shift);
          s_need = need - above;
        }
        above += h[k];
      }
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int64_t take_eq = s_need;  // how many scores equal to T are kept (lowest indices first)
  const int64_t per = (I + kSelectThreads - 1) / kSelectThreads;
  const int64_t lo = static_cast<int64_t>(threadIdx.x) * per;
  const int64_t hi = lo + per < I ? lo + per : I;
  uint64_t gt = 0, eq = 0;
  for (int64_t t = lo; t < hi; ++t) {
    const uint32_t u = __float_as_uint(score[t]);
    gt += u > T;
    eq += u == T;
  }
  const uint64_t before = block_exclusive_scan((gt << 32) | eq, warp_tot);
  const int64_t before_gt = static_cast<int64_t>(before >> 32), before_eq = static_cast<int64_t>(before & 0xFFFFFFFFu);
  int64_t pos = before_gt + (before_eq < take_eq ? before_eq : take_eq);
  int64_t eq_seen = before_eq;
  for (int64_t t = lo; t < hi; ++t) {
    const uint32_t u = __float_as_uint(score[t]);
    if (u > T) {
      out[pos++] = static_cast<int32_t>(t);
    } else if (u == T) {
      if (eq_seen < take_eq) out[pos++] = static_cast<int32_t>(t);
      ++eq_seen;
    }
  }
}

}  // namespace

size_t score_workspace_bytes(int64_t I) { return static_cast<size_t>(kScoreRowChunks) * static_cast<size_t>(I) * 4; }

cudaError_t launch_score_glu(const uint8_t* gate, const float* s_gate, const uint8_t* up, const float* s_up,
                             int64_t I, int64_t H, const uint8_t* down, const float* s_down, const float* h_in,
                             const float* h_mid, float* score, float* partial, cudaStream_t stream) {
  if (I == 0) return cudaSuccess;
  const int64_t row_ctas = (I + kScoreThreads / 32 - 1) / (kScoreThreads / 32);
  const unsigned int rows_grid = static_cast<unsigned int>(row_ctas < 1184 ? row_ctas : 1184);  // 8 per SM
  cudaError_t e;
  if (H <= kScoreStageH) {
    static thread_local int configured_for = -1;
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_for != dev) {
      e = cudaFuncSetAttribute(score_rows_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kScoreStageH * 4));
      if (e != cudaSuccess) return e;
      configured_for = dev;
    }
    score_rows_kernel<true><<<rows_grid, kScoreThreads, static_cast<size_t>(H) * 4, stream>>>(gate, s_gate, up, s_up,
                                                                                             I, H, h_in, score);
  } else {
    score_rows_kernel<false><<<rows_grid, kScoreThreads, 0, stream>>>(gate, s_gate, up, s_up, I, H, h_in, score);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 cols_grid(static_cast<unsigned int>((I / 16 + kColThreads - 1) / kColThreads), kScoreRowChunks);
  score_cols_kernel<<<cols_grid, kColThreads, 0, stream>>>(down, s_down, I, H, partial);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  score_finish_kernel<<<static_cast<unsigned int>((I + kScoreThreads - 1) / kScoreThreads), kScoreThreads, 0,
                        stream>>>(partial, I, h_mid, score);
  return cudaGetLastError();
}

// Scores staged in shared memory up to this many (the rest read from global).
constexpr int64_t kSelectStage = 48 * 1024;

cudaError_t launch_select_top(const float* score, int64_t I, int64_t Kd, int32_t* out, cudaStream_t stream) {
  if (Kd == 0) return cudaSuccess;
  if (I > kSelectStage) {
    select_top_kernel<false><<<1, kSelectThreads, 0, stream>>>(score, I, Kd, out);
    return cudaGetLastError();
  }
  static thread_local int configured_for = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_for != dev) {
    e = cudaFuncSetAttribute(select_top_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSelectStage * 4));
    if (e != cudaSuccess) return e;
    configured_for = dev;
  }
  select_top_kernel<true><<<1, kSelectThreads, static_cast<size_t>(I) * 4, stream>>>(score, I, Kd, out);
  return cudaGetLastError();
}

}  // namespace spense
