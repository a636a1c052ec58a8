// Spense oracle: a plain, slow, obviously-correct CPU statement of the hybrid
// 2:4-sparse + dense FP8 weight GEMM  Y = X * W^T.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
// this file; only the tests, the smoke check and the benchmark's CPU-baseline
// leg use it. It shares no code, header, table or helper with the CUDA library.
//
// Source of truth: the page "SpenseGPT: Practical One-shot Pruning Enabling
// Sparse and Dense GEMMs for LLM Inference" (gist.science technical summary):
//   - Technical Summary, 1. Problem Statement: 2:4 sparsity = in every four
//     consecutive weights two are zero.
//   - Technical Summary, 2.A The Spense Format: each weight matrix is split into
//     a contiguous dense region (p% of the weights) and a contiguous 2:4 region;
//     "input-split" runs the sparse GEMM on the first part of the input and the
//     dense GEMM on the second part, accumulating both.
//   - Technical Summary, 2.B Dense Index Selection Strategies: SpenseGPT keeps
//     the last p% of the indices dense; SpenseGPT+ keeps an arbitrary
//     score-selected index set dense and permutes it into one contiguous block,
//     which does not change the result.
//   - Technical Summary, 4. Experimental Results: FP8 precision on B200.
//
// Readings where the pages are silent (each one is listed with its reason in
// the design notes of this repository):
//   R1  FP8 is OCP e4m3fn: bias 7, no infinities, 0x7F/0xFF are NaN,
//       subnormals are m * 2^-9.
//   R2  The sparse region is formed over the sparse columns in ascending
//       original order after the dense columns are removed ("compacted");
//       groups are 4 consecutive compacted columns.
//   R3  Without a mask, a group keeps its two largest magnitudes; ties go to
//       the lower index; magnitude order of e4m3 bytes is the unsigned order
//       of (byte & 0x7F) (both zeros rank equal).
//   R4  With a mask, a group keeping fewer than two entries is padded with the
//       lowest unkept index (stored value 0x00); more than two is an error.
//   R5  Metadata nibble of a group = i0 | (i1 << 2) with i0 < i1; group 2j of a
//       row sits in the low nibble of byte j.
//   R6  The MMA-tiled layouts are the library's own storage format and are
//       restated here from their written definition (128-row tiles, 256
//       compacted sparse columns or 128 dense columns per block, 128-byte
//       swizzle: 16-byte chunk c of row r sits at chunk c ^ (r & 7)).
//   R12 SpenseGPT+ importance of intermediate index t of a GLU MLP (gate and
//       up [I][H], down [H][I]; weights are e4m3 codes times their fp32 row
//       scales; h_in [H] and h_mid [I] are the diagonals of the input Hessians
//       of gate/up and of down): the Wanda terms |W_ij| sqrt(H_jj) of every
//       weight that touches t, summed:
//         score[t] = sum_j |gate[t][j]| sqrt(h_in[j]) + sum_j |up[t][j]| sqrt(h_in[j])
//                  + sqrt(h_mid[t]) sum_i |down[i][t]|
//       The Kd indices with the largest scores stay dense (ties to the lower
//       index), listed in ascending order.
//   R11 Per-token quantisation of the activations (the step in front of the
//       GEMM) is computed in IEEE fp32: s = absmax / 448 (1 for an all-zero
//       row), q = e4m3(x / s) rounded to nearest even and saturated to 448,
//       one rounding per operation.
//
// Arithmetic: FP8 products and sums are accumulated in double precision.
// Every e4m3 value is a dyadic rational with at most 4 significant bits, so
// each product is exact in double; only the summation rounds (relative error
// ~ K * 2^-53, far below the comparison tolerance).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <thread>
#include <vector>

namespace {

enum OracleStatus {
  OR_OK = 0,
  OR_ERR_ARG = 1,
  OR_ERR_SHAPE = 2,
  OR_ERR_MASK = 4,
  OR_ERR_DENSE_IDX = 5,
  OR_ERR_NONFINITE = 6,
};

// OCP 8-bit floating point, E4M3 ("fn" variant): 1 sign bit, 4 exponent bits
// with bias 7, 3 mantissa bits, no infinity, NaN only when all of exponent and
// mantissa bits are ones.
double decode_e4m3(uint8_t b) {
  const int sign = (b >> 7) & 1;
  const int e = (b >> 3) & 0xF;
  const int m = b & 0x7;
  double mag;
  if (e == 0xF && m == 0x7) {
    mag = std::nan("");
  } else if (e == 0) {
    mag = std::ldexp(static_cast<double>(m), -9);  // 2^(1-7) * (m / 8)
  } else {
    mag = std::ldexp(1.0 + m / 8.0, e - 7);
  }
  return sign ? -mag : mag;
}

bool is_nan_e4m3(uint8_t b) { return (b & 0x7F) == 0x7F; }

// Column order pi = sparse columns (ascending) followed by dense columns
// (as given, ascending). With dense_idx == nullptr the dense set is the tail.
int build_order(int64_t K, const int32_t* dense_idx, int64_t Kd,
                std::vector<int64_t>& sparse_cols, std::vector<int64_t>& dense_cols) {
  sparse_cols.clear();
  dense_cols.clear();
  if (Kd < 0 || Kd > K) return OR_ERR_SHAPE;
  if (dense_idx == nullptr) {
    for (int64_t k = 0; k < K - Kd; ++k) sparse_cols.push_back(k);
    for (int64_t k = K - Kd; k < K; ++k) dense_cols.push_back(k);
    return OR_OK;
  }
  std::vector<char> is_dense(static_cast<size_t>(K), 0);
  for (int64_t j = 0; j < Kd; ++j) {
    const int64_t k = dense_idx[j];
    if (k < 0 || k >= K) return OR_ERR_DENSE_IDX;
    if (j > 0 && dense_idx[j] <= dense_idx[j - 1]) return OR_ERR_DENSE_IDX;
    is_dense[static_cast<size_t>(k)] = 1;
    dense_cols.push_back(k);
  }
  for (int64_t k = 0; k < K; ++k)
    if (!is_dense[static_cast<size_t>(k)]) sparse_cols.push_back(k);
  return OR_OK;
}

// E4M3 encoding of a float by its definition: the finite code whose value is
// nearest; on a tie the code with an even last bit (round to nearest, ties to
// even); magnitudes above 448 saturate to 448; NaN gives 0x7F. The sign is
// kept, so a negative value that rounds to zero gives 0x80.
uint8_t encode_e4m3_rne_sat(float v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));
  if (a >= 448.0) return static_cast<uint8_t>(sign | 0x7E);
  int best = 0;
  double best_d = a;  // distance to code 0 (value 0)
  for (int c = 1; c <= 0x7E; ++c) {
    const double d = std::fabs(decode_e4m3(static_cast<uint8_t>(c)) - a);
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return static_cast<uint8_t>(sign | best);
}

// bf16 bit pattern -> float (exact: bf16 is the upper half of a float).
float bf16_to_float(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

}  // namespace

extern "C" {

// Threads the host offers (std::thread::hardware_concurrency), reported beside
// the oracle's timings; 0 when unknown.
int oracle_hardware_concurrency(void) { return static_cast<int>(std::thread::hardware_concurrency()); }

// Decode all 256 e4m3 bytes (R1).
void oracle_e4m3_table(double* out256) {
  for (int b = 0; b < 256; ++b) out256[b] = decode_e4m3(static_cast<uint8_t>(b));
}

// Reference pack in canonical (row-major, untiled) form.
//   W         [N][K] e4m3 bytes, row-major.
//   mask      [N][K] bytes (nonzero = keep), read on sparse columns only, or NULL
//             for top-2-by-magnitude selection (R3).
//   dense_idx [Kd] strictly ascending column indices, or NULL for the tail.
// Outputs (any may be NULL):
//   Vs     [N][Ks/2]  the two stored values of each group, in index order.
//   Ecanon [N][ceil(Ks/8)]  metadata nibbles (R5).
//   Wd     [N][Kd]    dense columns in dense_idx order.
//   keep   [N][K]     1 where the original entry survives (dense columns and
//                     kept sparse entries), else 0.
int oracle_pack(const uint8_t* W, int64_t N, int64_t K, const uint8_t* mask,
                const int32_t* dense_idx, int64_t Kd, uint8_t* Vs, uint8_t* Ecanon,
                uint8_t* Wd, uint8_t* keep) {
  if (W == nullptr || N < 0 || K < 0) return OR_ERR_ARG;
  std::vector<int64_t> sc, dc;
  int st = build_order(K, dense_idx, Kd, sc, dc);
  if (st != OR_OK) return st;
  const int64_t Ks = K - Kd;
  if (Ks % 4 != 0) return OR_ERR_SHAPE;  // whole groups of four
  const int64_t EB = (Ks + 7) / 8;        // metadata bytes per row
  for (int64_t i = 0; i < N * K; ++i)
    if (is_nan_e4m3(W[i])) return OR_ERR_NONFINITE;
  const int64_t G = Ks / 4;
  if (keep) std::memset(keep, 0, static_cast<size_t>(N * K));
  if (Ecanon) std::memset(Ecanon, 0, static_cast<size_t>(N * EB));

  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* wrow = W + n * K;
    for (int64_t g = 0; g < G; ++g) {
      int64_t col[4];
      for (int i = 0; i < 4; ++i) col[i] = sc[static_cast<size_t>(4 * g + i)];
      bool kept[4] = {false, false, false, false};
      if (mask != nullptr) {
        int cnt = 0;
        for (int i = 0; i < 4; ++i) {
          kept[i] = mask[n * K + col[i]] != 0;
          cnt += kept[i] ? 1 : 0;
        }
        if (cnt > 2) return OR_ERR_MASK;
      } else {
        // R3: choose the two best by (magnitude desc, index asc).
        int order[4] = {0, 1, 2, 3};
        std::stable_sort(order, order + 4, [&](int a, int b) {
          return (wrow[col[a]] & 0x7F) > (wrow[col[b]] & 0x7F);
        });
        kept[order[0]] = true;
        kept[order[1]] = true;
      }
      // The stored pair: kept indices ascending, padded with the lowest
      // unkept indices (R4).
      int sel[2];
      int ns = 0;
      for (int i = 0; i < 4 && ns < 2; ++i)
        if (kept[i]) sel[ns++] = i;
      for (int i = 0; i < 4 && ns < 2; ++i) {
        if (!kept[i]) {
          bool used = false;
          for (int j = 0; j < ns; ++j) used = used || (sel[j] == i);
          if (!used) sel[ns++] = i;
        }
      }
      std::sort(sel, sel + 2);
      if (Vs) {
        for (int j = 0; j < 2; ++j)
          Vs[n * (Ks / 2) + 2 * g + j] = kept[sel[j]] ? wrow[col[sel[j]]] : 0x00;
      }
      if (Ecanon) {
        const uint8_t nib = static_cast<uint8_t>(sel[0] | (sel[1] << 2));
        Ecanon[n * EB + g / 2] |= static_cast<uint8_t>(nib << (4 * (g % 2)));
      }
      if (keep) {
        for (int i = 0; i < 4; ++i)
          if (kept[i]) keep[n * K + col[i]] = 1;
      }
    }
    for (int64_t j = 0; j < Kd; ++j) {
      const int64_t k = dc[static_cast<size_t>(j)];
      if (Wd) Wd[n * Kd + j] = wrow[k];
      if (keep) keep[n * K + k] = 1;
    }
  }
  return OR_OK;
}

// Inverse of oracle_pack: rebuild the masked matrix in original column order
// (dropped entries become 0x00) from the canonical packed arrays.
int oracle_unpack(const uint8_t* Vs, const uint8_t* Ecanon, const uint8_t* Wd, int64_t N,
                  int64_t K, const int32_t* dense_idx, int64_t Kd, uint8_t* Wout) {
  if (Wout == nullptr || N < 0 || K < 0) return OR_ERR_ARG;
  std::vector<int64_t> sc, dc;
  int st = build_order(K, dense_idx, Kd, sc, dc);
  if (st != OR_OK) return st;
  const int64_t Ks = K - Kd;
  if (Ks % 4 != 0) return OR_ERR_SHAPE;
  const int64_t EB = (Ks + 7) / 8;
  std::memset(Wout, 0, static_cast<size_t>(N * K));
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < Ks / 4; ++g) {
      const uint8_t nib = (Ecanon[n * EB + g / 2] >> (4 * (g % 2))) & 0xF;
      const int i0 = nib & 3, i1 = (nib >> 2) & 3;
      Wout[n * K + sc[static_cast<size_t>(4 * g + i0)]] = Vs[n * (Ks / 2) + 2 * g + 0];
      Wout[n * K + sc[static_cast<size_t>(4 * g + i1)]] = Vs[n * (Ks / 2) + 2 * g + 1];
    }
    for (int64_t j = 0; j < Kd; ++j) Wout[n * K + dc[static_cast<size_t>(j)]] = Wd[n * Kd + j];
  }
  return OR_OK;
}

// Reference statement of the library's MMA-tiled storage (R6), from the
// canonical arrays.
//   tiles   nt  = ceil(N / 128)                  (rows beyond N are padding)
//   sparse  nsb = ceil(Ks / 256) blocks per tile; block b holds compacted
//           sparse columns [256 b, 256 b + 256), i.e. value bytes
//           [128 b, 128 b + 128) and metadata bytes [32 b, 32 b + 32) of a row.
//   dense   ndb = ceil(Kd / 128) blocks per tile; block b holds dense columns
//           [128 b, 128 b + 128).
//   Vs_t  [nt][nsb][128 rows][128 B] swizzled; padding value 0x00.
//   E_t   [nt][nsb][2 halves][128 rows][16 B] plain; half h holds the row's
//         block metadata bytes [16 h, 16 h + 16); padding byte 0x44 (every
//         padded group selects indices 0 and 1 of four zero values).
//   Wd_t  [nt][ndb][128 rows][128 B] swizzled; padding value 0x00.
// Swizzled: byte c of row r sits at r*128 + ((c/16) ^ (r%8))*16 + c%16.
int oracle_tile(const uint8_t* Vs, const uint8_t* Ecanon, const uint8_t* Wd, int64_t N,
                int64_t Ks, int64_t Kd, uint8_t* Vs_t, uint8_t* E_t, uint8_t* Wd_t) {
  if (N < 0 || Ks < 0 || Kd < 0 || Ks % 16 != 0 || Kd % 16 != 0) return OR_ERR_SHAPE;
  const int64_t nt = (N + 127) / 128;
  const int64_t nsb = (Ks + 255) / 256;
  const int64_t ndb = (Kd + 127) / 128;
  for (int64_t t = 0; t < nt; ++t) {
    for (int64_t r = 0; r < 128; ++r) {
      const int64_t n = t * 128 + r;
      for (int64_t b = 0; b < nsb; ++b) {
        for (int64_t c = 0; c < 128; ++c) {
          const int64_t src = b * 128 + c;  // value byte within the row
          uint8_t v = 0x00;
          if (n < N && src < Ks / 2) v = Vs[n * (Ks / 2) + src];
          const int64_t off = r * 128 + (((c / 16) ^ (r % 8)) * 16) + (c % 16);
          if (Vs_t) Vs_t[(t * nsb + b) * 16384 + off] = v;
        }
        for (int64_t h = 0; h < 2; ++h) {
          for (int64_t c = 0; c < 16; ++c) {
            const int64_t src = b * 32 + h * 16 + c;  // metadata byte within the row
            uint8_t e = 0x44;
            if (n < N && src < Ks / 8) e = Ecanon[n * (Ks / 8) + src];  // Ks % 16 == 0 here
            if (E_t) E_t[((t * nsb + b) * 2 + h) * 2048 + r * 16 + c] = e;
          }
        }
      }
      for (int64_t b = 0; b < ndb; ++b) {
        for (int64_t c = 0; c < 128; ++c) {
          const int64_t src = b * 128 + c;
          uint8_t v = 0x00;
          if (n < N && src < Kd) v = Wd[n * Kd + src];
          const int64_t off = r * 128 + (((c / 16) ^ (r % 8)) * 16) + (c % 16);
          if (Wd_t) Wd_t[(t * ndb + b) * 16384 + off] = v;
        }
      }
    }
  }
  return OR_OK;
}

// The masked GEMM in original column order, in double precision:
//   yref[m][r]  = s_x[m] * s_w[n] * sum_k dec(X[m][k]) * dec(W[n][k]) * keep[n][k]
//   bound[m][r] = |s_x[m] * s_w[n]| * sum_k |dec(X[m][k]) * dec(W[n][k]) * keep[n][k]|
// for the rows n = rows[r] (or all rows, r = n, when rows == NULL).
// keep == NULL keeps every entry (a plain dense GEMM). Outputs are [M][R].
// nthreads > 1 splits the rows across std::threads; the arithmetic per output
// is the same sequential sum over k in every case.
int oracle_gemm(const uint8_t* X, const float* s_x, int64_t M, const uint8_t* W,
                const float* s_w, int64_t N, int64_t K, const uint8_t* keep,
                const int64_t* rows, int64_t R, double* yref, double* bound, int nthreads) {
  if (X == nullptr || s_x == nullptr || W == nullptr || s_w == nullptr || yref == nullptr)
    return OR_ERR_ARG;
  if (M < 0 || N < 0 || K < 0) return OR_ERR_SHAPE;
  if (rows == nullptr) R = N;
  double table[256];
  oracle_e4m3_table(table);
  // X decoded once: [M][K] doubles.
  std::vector<double> xd(static_cast<size_t>(M * K));
  for (int64_t i = 0; i < M * K; ++i) xd[static_cast<size_t>(i)] = table[X[i]];

  auto work = [&](int64_t r0, int64_t r1) {
    std::vector<double> wrow(static_cast<size_t>(K));
    for (int64_t r = r0; r < r1; ++r) {
      const int64_t n = rows ? rows[r] : r;
      for (int64_t k = 0; k < K; ++k) {
        const bool kept = keep == nullptr || keep[n * K + k] != 0;
        wrow[static_cast<size_t>(k)] = kept ? table[W[n * K + k]] : 0.0;
      }
      for (int64_t m = 0; m < M; ++m) {
        const double* xr = xd.data() + m * K;
        double acc = 0.0, accabs = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          const double p = xr[k] * wrow[static_cast<size_t>(k)];
          acc += p;
          accabs += std::fabs(p);
        }
        const double sc = static_cast<double>(s_x[m]) * static_cast<double>(s_w[n]);
        yref[m * R + r] = sc * acc;
        if (bound) bound[m * R + r] = std::fabs(sc) * accabs;
      }
    }
  };
  for (int64_t r = 0; r < R; ++r) {
    const int64_t n = rows ? rows[r] : r;
    if (n < 0 || n >= N) return OR_ERR_ARG;
  }
  if (nthreads <= 1 || R < 2) {
    work(0, R);
  } else {
    const int64_t T = std::min<int64_t>(nthreads, R);
    std::vector<std::thread> th;
    for (int64_t t = 0; t < T; ++t) {
      const int64_t r0 = R * t / T, r1 = R * (t + 1) / T;
      th.emplace_back(work, r0, r1);
    }
    for (auto& x : th) x.join();
  }
  return OR_OK;
}


// Per-token FP8 quantisation of bf16 activations, the step in front of the
// GEMM, with the column rearrangement a scattered dense set needs fused in
// (the SlideSparse page, "Activation Lifting", folds its rearrangement into
// per-token quantisation the same way; the SpenseGPT page, 2.B, permutes the
// dense indices into one contiguous block):
//   s[m]    = fp32(max_k |x[m][k]| / 448), or 1 for an all-zero row
//   q[m][j] = e4m3_rne_sat(fp32(x[m][c(j)] / s[m]))
// where c is the column order sparse columns ascending then dense_idx
// (dense_idx == NULL: the identity). Reading R11: the scale and each quotient
// are single IEEE fp32 operations (one rounding each), the precision in which
// the code of every element is decided.
int oracle_quantize(const uint16_t* X, int64_t M, int64_t K, const int32_t* dense_idx, int64_t Kd,
                    uint8_t* Xq, float* s) {
  if (X == nullptr || Xq == nullptr || s == nullptr) return OR_ERR_ARG;
  if (M < 0 || K < 0) return OR_ERR_SHAPE;
  std::vector<int64_t> order(static_cast<size_t>(K));
  if (dense_idx == nullptr) {
    for (int64_t k = 0; k < K; ++k) order[static_cast<size_t>(k)] = k;
  } else {
    std::vector<int64_t> sp, dn;
    const int st = build_order(K, dense_idx, Kd, sp, dn);
    if (st != OR_OK) return st;
    size_t j = 0;
    for (int64_t k : sp) order[j++] = k;
    for (int64_t k : dn) order[j++] = k;
  }
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t* xr = X + m * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) amax = std::max(amax, std::fabs(bf16_to_float(xr[k])));
    const float sm = amax > 0.0f ? amax / 448.0f : 1.0f;
    s[m] = sm;
    for (int64_t j = 0; j < K; ++j) {
      const float q = bf16_to_float(xr[order[static_cast<size_t>(j)]]) / sm;
      Xq[m * K + j] = encode_e4m3_rne_sat(q);
    }
  }
  return OR_OK;
}


// SpenseGPT+ importance scores (the SpenseGPT page, 2.B: a Wanda-style score
// S_ij = |W_ij| sqrt(H_jj) aggregated over the gate, up and down projections;
// reading R12). gate or up may be NULL (its term is left out). double precision.
int oracle_score_glu(const uint8_t* gate, const float* s_gate, const uint8_t* up, const float* s_up,
                     int64_t I, int64_t H, const uint8_t* down, const float* s_down, const float* h_in,
                     const float* h_mid, double* score) {
  if (down == nullptr || s_down == nullptr || h_in == nullptr || h_mid == nullptr || score == nullptr)
    return OR_ERR_ARG;
  if ((gate != nullptr && s_gate == nullptr) || (up != nullptr && s_up == nullptr)) return OR_ERR_ARG;
  if (I < 0 || H < 0) return OR_ERR_SHAPE;
  double table[256];
  oracle_e4m3_table(table);
  for (int64_t t = 0; t < I; ++t) {
    double total = 0.0;
    for (int w = 0; w < 2; ++w) {
      const uint8_t* Wm = w == 0 ? gate : up;
      const float* sc = w == 0 ? s_gate : s_up;
      if (Wm == nullptr) continue;
      double acc = 0.0;
      for (int64_t j = 0; j < H; ++j)
        acc += std::fabs(static_cast<double>(sc[t]) * table[Wm[t * H + j]]) * std::sqrt(static_cast<double>(h_in[j]));
      total += acc;
    }
    double col = 0.0;
    for (int64_t i = 0; i < H; ++i) col += std::fabs(static_cast<double>(s_down[i]) * table[down[i * I + t]]);
    total += std::sqrt(static_cast<double>(h_mid[t])) * col;
    score[t] = total;
  }
  return OR_OK;
}

// The Kd largest scores (ties to the lower index), written in ascending index
// order: the dense set SpenseGPT+ keeps (the SpenseGPT page, 2.B: "the
// top-scoring indices are selected to remain dense").
int oracle_select_top(const double* score, int64_t I, int64_t Kd, int32_t* out) {
  if (score == nullptr || (Kd > 0 && out == nullptr)) return OR_ERR_ARG;
  if (I < 0 || Kd < 0 || Kd > I) return OR_ERR_SHAPE;
  std::vector<int64_t> idx(static_cast<size_t>(I));
  for (int64_t t = 0; t < I; ++t) idx[static_cast<size_t>(t)] = t;
  std::stable_sort(idx.begin(), idx.end(), [&](int64_t a, int64_t b) { return score[a] > score[b]; });
  std::vector<int64_t> top(idx.begin(), idx.begin() + Kd);
  std::sort(top.begin(), top.end());
  for (int64_t j = 0; j < Kd; ++j) out[j] = static_cast<int32_t>(top[static_cast<size_t>(j)]);
  return OR_OK;
}

}  // extern "C"
