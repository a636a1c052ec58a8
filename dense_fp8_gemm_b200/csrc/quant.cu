// Per-token FP8 quantisation of bf16 activations, with the column order of a
// packed weight fused in.
//
// Pages: "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs
// for LLM Inference" (gist.science technical summary), Technical Summary §2.B:
// SpenseGPT+ keeps a scattered set of input indices dense and permutes them
// into one contiguous block; the GEMM then needs the activations in that
// column order. The SlideSparse page ("Activation Lifting") folds such a
// rearrangement into the per-token quantisation that runs in front of every
// FP8 GEMM anyway, at almost no extra cost. Here:
//   s[m]    = fp32(max_k |x[m][k]| / 448)   (1 for an all-zero row)
//   q[m][j] = e4m3 round-to-nearest-even, saturating, of fp32(x[m][c(j)] / s[m])
// with c(j) = perm[j] (packed position -> original column) or j.
//
// DRAM sees each byte of X once: the repeated reads of a row (several CTAs per
// row, and the quantising pass after the absmax pass) hit L2.
#include <cstdint>
#include <cuda_bf16.h>

#include "pdl.cuh"
#include "spense_internal.h"

namespace spense {
namespace {

constexpr int kQuantThreads = 512;

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Two floats -> two e4m3 bytes (round to nearest even, saturating to +-448):
// the low byte holds `lo`, the high byte `hi`.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = 0.0f;
#pragma unroll
  for (int i = 0; i < kQuantThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

// Sixteen quantised codes of one 16-column output chunk from its 16 source values.
__device__ __forceinline__ uint4 quantize16(const float (&f)[16], float s) {
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const uint32_t lo = cvt_e4m3x2(__fdiv_rn(f[4 * h], s), __fdiv_rn(f[4 * h + 1], s));
    const uint32_t hi = cvt_e4m3x2(__fdiv_rn(f[4 * h + 2], s), __fdiv_rn(f[4 * h + 3], s));
    o[h] = lo | (hi << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Each row is split over C CTAs (C = 1 .. 8; more CTAs per row when there are
// few rows). CTA c writes the 16-column output chunks [K16 c / C, K16 (c + 1) /
// C) of the row, one chunk per thread per round. Every CTA reads the whole row
// to take its absmax itself (the C - 1 extra reads of a row hit L2; no CTA
// waits for another), and with a gather it keeps the row in shared memory and
// gathers from there. Rows too long for shared memory gather from global
// memory instead (the packed order is two ascending runs, so those loads
// mostly share cache lines).
//
// At decode sizes the kernel is a chain of memory latencies, so it is cut to
// as few as possible: the packed order of a thread's first chunk belongs to the
// weight, not to the previous kernel, so it is fetched before waiting for that
// kernel; the row is read in one round (eight 16-byte loads in flight per
// thread, 512 threads: rows up to 32768 columns); then one reduction, and the
// codes are computed from shared memory or L2.
// K % 16 == 0; X rows 16-byte aligned; Xq rows 16-byte aligned.
template <bool kGather, bool kStaged>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(const uint16_t* __restrict__ X, int64_t K,
                                                                 const int32_t* __restrict__ perm,
                                                                 uint8_t* __restrict__ Xq, float* __restrict__ s_out,
                                                                 int C) {
  extern __shared__ uint4 qsmem[];  // kStaged: the row, K bf16
  __shared__ float red[kQuantThreads / 32];
  pdl_trigger();  // the GEMM that reads Xq may start prefetching its weights
  const int64_t m = blockIdx.x / C;
  const int c = static_cast<int>(blockIdx.x % C);
  const int64_t k16 = K / 16;
  const int64_t j0 = k16 * c / C, j1 = k16 * (c + 1) / C;  // this CTA's 16-column chunks
  int4 cs0[4];  // gather: source columns of this thread's first chunk
  if (kGather && j0 + threadIdx.x < j1) {
    const int4* pj = reinterpret_cast<const int4*>(perm + (j0 + threadIdx.x) * 16);
#pragma unroll
    for (int h = 0; h < 4; ++h) cs0[h] = __ldg(pj + h);
  }
  pdl_wait();  // X may be written by the previous kernel
  const uint16_t* xrow = X + m * K;
  const uint4* xr = reinterpret_cast<const uint4*>(xrow);
  float amax = 0.0f;
  // Absmax of the whole row: 16-byte loads, eight in flight per thread.
  const int64_t n8 = K / 8;
  for (int64_t i = threadIdx.x; i < n8; i += 8 * kQuantThreads) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t ii = i + static_cast<int64_t>(u) * kQuantThreads;
      v[u] = ii < n8 ? __ldg(xr + ii) : make_uint4(0u, 0u, 0u, 0u);
      if (kStaged && ii < n8) qsmem[ii] = v[u];
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        amax = fmaxf(amax, fabsf(bf16_bits_to_float(w[h] & 0xFFFFu)));
        amax = fmaxf(amax, fabsf(bf16_bits_to_float(w[h] >> 16)));
      }
    }
  }
  amax = block_max(amax, red);  // its barrier also publishes the staged row
  const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (c == 0 && threadIdx.x == 0) s_out[m] = s;
  const uint16_t* src = kStaged ? reinterpret_cast<const uint16_t*>(qsmem) : xrow;
  uint4* qr = reinterpret_cast<uint4*>(Xq + m * K);
  for (int64_t i = j0 + threadIdx.x; i < j1; i += kQuantThreads) {
    float f[16];
    if (kGather) {
      int4 cs[4];
      if (i == j0 + threadIdx.x) {
#pragma unroll
        for (int h = 0; h < 4; ++h) cs[h] = cs0[h];
      } else {
        const int4* pj = reinterpret_cast<const int4*>(perm + i * 16);
#pragma unroll
        for (int h = 0; h < 4; ++h) cs[h] = __ldg(pj + h);
      }
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        f[4 * h + 0] = bf16_bits_to_float(kStaged ? src[cs[h].x] : __ldg(src + cs[h].x));
        f[4 * h + 1] = bf16_bits_to_float(kStaged ? src[cs[h].y] : __ldg(src + cs[h].y));
        f[4 * h + 2] = bf16_bits_to_float(kStaged ? src[cs[h].z] : __ldg(src + cs[h].z));
        f[4 * h + 3] = bf16_bits_to_float(kStaged ? src[cs[h].w] : __ldg(src + cs[h].w));
      }
    } else {
      const uint4 r0 = __ldg(xr + 2 * i), r1 = __ldg(xr + 2 * i + 1);
      const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        f[2 * h] = bf16_bits_to_float(w[h] & 0xFFFFu);
        f[2 * h + 1] = bf16_bits_to_float(w[h] >> 16);
      }
    }
    qr[i] = quantize16(f, s);
  }
}

// Shared memory for a staged row: at most 56 KB, so four CTAs (of 512 threads) fit per SM.
constexpr int64_t kQuantStageBytes = 56 * 1024;

}  // namespace

cudaError_t launch_quantize(const uint16_t* X, int64_t M, int64_t K, const int32_t* perm, uint8_t* Xq,
                            float* s_x, int sms, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  // CTAs per row: one once the rows alone cover the SMs (every extra CTA of a
  // row reads the row again); otherwise enough for two CTAs per SM, at most 8
  // (16 for a gather at 4 to 16 tokens) and at most one per 16-column chunk.
  // Measured at 25600 columns, back to back: 1, 2, 4, 8, 16 CTAs per row take
  // 7.8, 6.3, 4.7, 3.8, 3.5 us at 16 tokens and 8.5, 6.8, 4.8, 4.0, 6.6 us at
  // 32 tokens; with the gather 16 rather than 8 per row: 3.61 -> 3.40 us at 4
  // tokens, 3.82 -> 3.55 at 16, but 2.96 -> 3.21 at one token, and without the
  // gather no gain (3.28 -> 3.36 at 16).
  int64_t C = M >= sms ? 1 : (2 * static_cast<int64_t>(sms) + M - 1) / M;
  const int64_t cmax = (perm != nullptr && M >= 4 && M <= 16) ? 16 : 8;
  C = C < 1 ? 1 : (C > cmax ? cmax : C);

  while (C > 1 && K / 16 < C) --C;
  const unsigned int grid = static_cast<unsigned int>(M * C);
  const int ci = static_cast<int>(C);
  if (perm == nullptr)
    return launch_pdl(quantize_kernel<false, false>, grid, kQuantThreads, 0, stream, X, K, perm, Xq, s_x, ci);
  const int64_t stage = K * 2;
  if (stage > kQuantStageBytes)
    return launch_pdl(quantize_kernel<true, false>, grid, kQuantThreads, 0, stream, X, K, perm, Xq, s_x, ci);
  static thread_local int configured_for = -1;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  if (configured_for != dev) {
    st = cudaFuncSetAttribute(quantize_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kQuantStageBytes));
    if (st != cudaSuccess) return st;
    configured_for = dev;
  }
  return launch_pdl(quantize_kernel<true, true>, grid, kQuantThreads, static_cast<size_t>(stage), stream, X, K, perm,
                    Xq, s_x, ci);
}

}  // namespace spense
