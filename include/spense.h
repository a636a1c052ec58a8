/*
 * spense.h — C ABI of the Spense hybrid 2:4-sparse + dense FP8 weight GEMM for
 * NVIDIA B200 (sm_100a).
 *
 *   Y[m][n] = bf16( s_x[m] * s_w[n] * sum_k X[m][k] * Wm[n][k] )
 *
 * where Wm is the weight matrix W [N x K] (FP8 e4m3) after its sparse region
 * has been pruned to 2:4. The operation is the one stated on the page
 * "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs for
 * LLM Inference" (gist.science technical summary):
 *   - Technical Summary §1 (Problem Statement): 2:4 semi-structured sparsity,
 *     two of every four consecutive weights are zero;
 *   - §2.A (The Spense Format): W is split along its input dimension into a
 *     contiguous 2:4 region and a contiguous dense region; the input-split
 *     execution runs the sparse GEMM on the first part of the input and the
 *     dense GEMM on the second part and accumulates both. Here both parts are
 *     contracted into one fp32 accumulator by one kernel;
 *   - §2.B (Dense Index Selection Strategies): SpenseGPT keeps the last p% of
 *     the input indices dense (dense_idx == NULL); SpenseGPT+ keeps an
 *     arbitrary score-selected set dense and permutes it into one contiguous
 *     block, which leaves Y unchanged (dense_idx != NULL);
 *   - §4 (Experimental Results): FP8 precision on B200.
 * The FP8 format (OCP e4m3fn), the fp32 per-output-channel and per-token
 * scales and the bf16 output are this library's reading of "FP8 precision".
 *
 * Conventions for every call:
 *   - Device pointers are CUDA device addresses on the current device; host
 *     pointers are plain host memory. Nothing is retained after a call returns
 *     except by spense_pack, which copies what it needs into the handle.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Errors are returned as spense_status codes; nothing aborts or throws. On
 *     failure outputs are left untouched and *out handles are set to NULL.
 *     spense_last_error() gives a message for the calling thread.
 *   - Requires a compute capability 10.x device (B200); otherwise
 *     SPENSE_ERR_UNSUPPORTED.
 */
#ifndef SPENSE_H_
#define SPENSE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPENSE_API __attribute__((visibility("default")))
#else
#define SPENSE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum spense_status {
  SPENSE_OK = 0,
  SPENSE_ERR_ARG = 1,          /* NULL pointer, unknown flag, or bad argument */
  SPENSE_ERR_SHAPE = 2,        /* shape outside the supported set (see below) */
  SPENSE_ERR_ALIGN = 3,        /* a device pointer is not 16-byte aligned */
  SPENSE_ERR_MASK = 4,         /* a group of four in the mask keeps more than two */
  SPENSE_ERR_DENSE_IDX = 5,    /* dense_idx not strictly ascending or out of [0, K) */
  SPENSE_ERR_NONFINITE = 6,    /* W holds an e4m3 NaN byte (0x7F or 0xFF) */
  SPENSE_ERR_WORKSPACE = 7,    /* workspace NULL or smaller than required */
  SPENSE_ERR_OOM = 8,          /* device allocation failed */
  SPENSE_ERR_CUDA = 9,         /* a CUDA runtime call failed */
  SPENSE_ERR_TIMEOUT = 10,     /* a kernel gave up waiting (reported via the status word) */
  SPENSE_ERR_UNSUPPORTED = 11  /* no compute capability 10.x device */
} spense_status;

/* Opaque packed weight. Owns its device buffers. */
typedef struct spense_packed spense_packed;

/* spense_pack flags */
#define SPENSE_PACK_KEEP_CANONICAL 1u /* also keep the untiled Vs / E / Wd arrays (for inspection) */

/*
 * spense_pack — split W into its 2:4 region and dense region and store both in
 * the layout the GEMM kernel streams (Technical Summary §2.A, §2.B).
 *
 *   W         device, e4m3 bytes [N][K] row-major (K contiguous). Read only.
 *   w_scale   device, fp32 [N], per-output-channel scale s_w. Copied.
 *   N, K      1 <= N <= 2^20, 16 <= K <= 2^20, K % 16 == 0.
 *   mask      device, bytes [N][K] row-major, nonzero = keep, read on the sparse
 *             columns only; or NULL to keep the two largest magnitudes of every
 *             group of four (ties to the lower index).
 *   dense_idx HOST, int32 [Kd] strictly ascending in [0, K): the dense columns
 *             (SpenseGPT+); or NULL for the last Kd columns (SpenseGPT).
 *   Kd        number of dense columns, 0 <= Kd <= K, Kd % 16 == 0.
 *   flags     0 or SPENSE_PACK_KEEP_CANONICAL.
 *   out       receives the handle.
 *
 * Sparse region: the Ks = K - Kd non-dense columns in ascending order, grouped
 * four by four. A group keeps the mask's entries, or its top two; a mask group
 * keeping fewer than two is padded with its lowest unkept index (stored value
 * 0). More than two kept -> SPENSE_ERR_MASK.
 *
 * Stored format (the "tiled" arrays; rows padded to a multiple of 128, padding
 * values 0, padding metadata 0x44):
 *   Vs_t [ceil(N/128)][ceil(Ks/256)][128 rows][128 B]  kept values, two per
 *        group in index order; byte c of row r at r*128 + ((c/16)^(r%8))*16 + c%16.
 *   E_t  [ceil(N/128)][ceil(Ks/256)][2][128 rows][16 B]  2-bit index pairs,
 *        one nibble per group (i0 | i1 << 2), group 2j in the low nibble of
 *        byte j; half h holds the row's metadata bytes [16h, 16h+16) of the block.
 *   Wd_t [ceil(N/128)][ceil(Kd/128)][128 rows][128 B]  dense columns in
 *        dense_idx order, swizzled like Vs_t.
 * With SPENSE_PACK_KEEP_CANONICAL the untiled Vs [N][Ks/2], E [N][Ks/8] and
 * Wd [N][Kd] are kept as well.
 *
 * Synchronizes `stream` (mask and NaN errors are found on the device).
 * Errors: ARG, SHAPE, ALIGN (W, mask), MASK, DENSE_IDX, NONFINITE, OOM, CUDA,
 * UNSUPPORTED.
 */
SPENSE_API spense_status spense_pack(const uint8_t* W, const float* w_scale, int64_t N, int64_t K,
                          const uint8_t* mask, const int32_t* dense_idx, int64_t Kd,
                          uint32_t flags, void* stream, spense_packed** out);

/*
 * spense_pack_rows — spense_pack of the rows W[rows[r]], r = 0 .. N-1, of a
 * matrix W [N_src][K] (and the same rows of w_scale and of the mask). The
 * rows are gathered on the device into a temporary before packing. Used for
 * the output-split execution (Technical Summary §2.A: the output channels are
 * split into a 2:4 part and a dense part) and to fold the SpenseGPT+
 * permutation of the intermediate indices into the gate and up rows
 * (Technical Summary §2.B: permuting the intermediate indices of a GLU MLP
 * leaves its output unchanged).
 *   rows   HOST int32 [N], each in [0, N_src) (repeats allowed).
 * Other arguments and errors as spense_pack (ARG also for a bad row index).
 */
SPENSE_API spense_status spense_pack_rows(const uint8_t* W, const float* w_scale, int64_t N_src, int64_t K,
                                          const int32_t* rows, int64_t N, const uint8_t* mask,
                                          const int32_t* dense_idx, int64_t Kd, uint32_t flags, void* stream,
                                          spense_packed** out);

/*
 * spense_gemm — Y = X * Wm^T with scales (Technical Summary §2.A input-split,
 * both regions into one fp32 accumulator; §2.B the activations are gathered
 * into the packed column order when dense_idx was given).
 *
 *   Wp         packed weight from spense_pack.
 *   X          device, e4m3 bytes [M][K] row-major, 16-byte aligned.
 *   x_scale    device, fp32 [M], per-token scale s_x.
 *   M          1 <= M <= 65535.
 *   Y          device, bf16 [M][N] row-major (round to nearest even), 16-byte aligned.
 *   workspace  device scratch of at least spense_gemm_workspace_size(Wp, M)
 *              bytes, 256-byte aligned, ZERO-FILLED before its first use. Every
 *              completed call leaves its counter region zero again, so one
 *              workspace can serve any number of calls issued in stream order
 *              (not concurrently). After SPENSE_ERR_TIMEOUT, zero it again.
 *
 * Asynchronous on `stream`. Device-side failures (a wait that gave up) are
 * recorded in the workspace's status word: see spense_workspace_status.
 * Errors: ARG, SHAPE, ALIGN, WORKSPACE, CUDA, UNSUPPORTED.
 */
SPENSE_API spense_status spense_gemm(const spense_packed* Wp, const uint8_t* X, const float* x_scale,
                          int64_t M, uint16_t* Y, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Bytes of workspace spense_gemm needs for this handle and token count; 0 on a
 * bad argument. */
SPENSE_API size_t spense_gemm_workspace_size(const spense_packed* Wp, int64_t M);

/*
 * spense_gemm_grouped — one launch over `count` (1..4) packed weights that share
 * the activations X: Ys[i] [M][N_i] = X * Wp_i^T with scales. The weights must
 * have been packed on the same device with the same K, Kd and dense column set
 * (for example the q, k and v projections of one layer, or gate and up). Their
 * row tiles are streamed as one sequence, so small matrices share the SMs and
 * the launch cost instead of each paying for its own launch. This is a fusion
 * of independent GEMMs over one input; each output is exactly what spense_gemm
 * gives for that weight.
 *   workspace  at least spense_gemm_grouped_workspace_size(Wps, count, M) bytes,
 *              with the same rules as for spense_gemm.
 * Errors: as spense_gemm, plus ARG when the weights cannot share a launch.
 */
SPENSE_API spense_status spense_gemm_grouped(const spense_packed* const* Wps, int count, const uint8_t* X,
                                             const float* x_scale, int64_t M, uint16_t* const* Ys,
                                             void* workspace, size_t workspace_bytes, void* stream);

SPENSE_API size_t spense_gemm_grouped_workspace_size(const spense_packed* const* Wps, int count, int64_t M);

/* Flags of spense_gemm_grouped_ex and spense_gemm_grouped_host. */
enum {
  /* X (and x_scale) are already in the packed column order of the weights
   * (sparse columns ascending, then the dense columns in dense_idx order), as
   * spense_quantize writes them when given one of the weights as `order`; the
   * GEMM then skips its own gather. No effect for a tail dense set. */
  SPENSE_GEMM_X_PACKED_ORDER = 1u,
  /* spense_gemm_grouped_host only: X and x_scale are in HOST memory. */
  SPENSE_GEMM_HOST_X = 2u,
  /* spense_gemm_grouped_host only: the outputs Ys are in HOST memory. */
  SPENSE_GEMM_HOST_Y = 4u
};

/*
 * spense_gemm_grouped_ex — spense_gemm_grouped with output strides and flags.
 * Members need the same device, K and column order of X, but when none has a
 * scattered dense set their Kd may differ: a weight packed with Kd = 0 (all
 * 2:4) and one packed with Kd = K (all dense) can share a launch. That is the
 * output-split execution of Technical Summary §2.A (the output channels split
 * into a 2:4 part and a dense part): pack the two row sets with
 * spense_pack_rows and point their outputs into one Y with ldy = N_total.
 *   ldy    NULL: Ys[i] is [M][N_i] contiguous. Else host int64 [count]: row m
 *          of output i starts at Ys[i] + m * ldy[i], N_i <= ldy[i] <= 2^30
 *          (16-byte stores are used when ldy[i] % 8 == 0).
 *   flags  0 or SPENSE_GEMM_X_PACKED_ORDER; unknown bits are an ARG error.
 * With ldy == NULL and flags == 0 it is spense_gemm_grouped.
 */
SPENSE_API spense_status spense_gemm_grouped_ex(const spense_packed* const* Wps, int count, const uint8_t* X,
                                                const float* x_scale, int64_t M, uint16_t* const* Ys,
                                                const int64_t* ldy, void* workspace, size_t workspace_bytes,
                                                unsigned int flags, void* stream);

/*
 * spense_quantize — per-token FP8 quantisation of bf16 activations, the step in
 * front of every FP8 GEMM, with the column order of a packed weight fused in.
 * The technical summary of "SpenseGPT: Practical One-shot Pruning Enabling
 * Sparse and Dense GEMMs for LLM Inference" (§2.B) permutes SpenseGPT+'s
 * scattered dense indices into one contiguous block, so the GEMM reads the
 * activations in that order; the SlideSparse page ("Activation Lifting") folds
 * such a rearrangement into the per-token quantisation at almost no cost. This
 * does the same, so the GEMM's own gather can be skipped
 * (SPENSE_GEMM_X_PACKED_ORDER).
 *   X        device, bf16 bit patterns [M][K] row-major, 16-byte aligned.
 *   M        0 .. 65535 token rows (0: nothing to do).
 *   K        multiple of 16, 16 .. 2^20.
 *   order    NULL: columns stay in X's order. A packed weight with the same K on
 *            the current device: columns come out in its packed order (the
 *            identity for a tail dense set).
 *   Xq       device, e4m3 [M][K] row-major, 16-byte aligned (caller-owned).
 *   x_scale  device, fp32 [M], 4-byte aligned (caller-owned).
 * Result, in IEEE fp32 with one rounding per operation:
 *   x_scale[m] = max_k |X[m][k]| / 448 (1 for an all-zero row)
 *   Xq[m][j]   = e4m3 round-to-nearest-even of X[m][c(j)] / x_scale[m],
 *                saturated to +-448 (c = the packed order or the identity).
 * X must be finite; a NaN or infinity gives unspecified codes for its row.
 * Asynchronous on `stream`. Errors: ARG (NULL pointer, order from another
 * device), SHAPE, ALIGN, UNSUPPORTED (no sm_100 device), CUDA.
 */
SPENSE_API spense_status spense_quantize(const uint16_t* X, int64_t M, int64_t K, const spense_packed* order,
                                         uint8_t* Xq, float* x_scale, void* stream);

/*
 * spense_score_glu — SpenseGPT+ importance of every intermediate index of a
 * GLU MLP (Technical Summary §2.B: a Wanda-style score S_ij = |W_ij| sqrt(H_jj)
 * aggregated across the gate, up and down projections; the top-scoring indices
 * stay dense). This library's reading of the aggregation, with weights as e4m3
 * codes times fp32 row scales:
 *   score[t] = |s_gate[t]| sum_j |gate[t][j]| sqrt(h_in[j])
 *            + |s_up[t]|   sum_j |up[t][j]|   sqrt(h_in[j])
 *            + sqrt(h_mid[t]) sum_i |s_down[i]| |down[i][t]|
 * computed in fp32 in a fixed order (repeatable bit for bit).
 *   gate, up   device, e4m3 [I][H] row-major, 16-byte aligned; either may be
 *              NULL (its term is left out). s_gate, s_up: device fp32 [I].
 *   down       device, e4m3 [H][I] row-major, 16-byte aligned; s_down fp32 [H].
 *   h_in       device fp32 [H], h_mid device fp32 [I]: the diagonals of the
 *              input Hessians of gate/up and of down (non-negative).
 *   I, H       multiples of 16 in [16, 2^20].
 *   score      device fp32 [I] (caller-owned).
 *   workspace  device, 256-byte aligned, at least spense_score_workspace_size(I, H)
 *              bytes (no zeroing needed).
 * Asynchronous on `stream`. The weights must hold no e4m3 NaN code (0x7F or
 * 0xFF; spense_pack rejects them too): the score of a row or column with one
 * is unspecified. Errors: ARG, SHAPE, ALIGN, WORKSPACE, UNSUPPORTED, CUDA.
 */
SPENSE_API spense_status spense_score_glu(const uint8_t* gate, const float* s_gate, const uint8_t* up,
                                          const float* s_up, int64_t I, int64_t H, const uint8_t* down,
                                          const float* s_down, const float* h_in, const float* h_mid, float* score,
                                          void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes spense_score_glu needs (0 for a bad shape). */
SPENSE_API size_t spense_score_workspace_size(int64_t I, int64_t H);

/*
 * spense_select_dense — the dense set SpenseGPT+ keeps: the Kd indices with
 * the largest scores, ties to the lower index, written in ascending order
 * (ready for spense_pack's dense_idx after a copy to the host).
 *   score      device fp32 [I], non-negative (as spense_score_glu writes).
 *   I          1 .. 2^20;  Kd  0 .. I.
 *   dense_idx  device int32 [Kd] (caller-owned).
 * Asynchronous on `stream`. Errors: ARG, SHAPE, ALIGN, UNSUPPORTED, CUDA.
 */
SPENSE_API spense_status spense_select_dense(const float* score, int64_t I, int64_t Kd, int32_t* dense_idx,
                                             void* stream);

/*
 * spense_gemm_grouped_host — spense_gemm_grouped with its input, its outputs or
 * both in HOST memory; the copies between host and device run inside the call,
 * on `stream`, through staging areas of the workspace. The GEMM itself is the
 * one of Technical Summary §2.A / §2.B described above.
 *   flags  SPENSE_GEMM_HOST_X: X [M][K] and x_scale [M] are host pointers,
 *          copied to the device before the GEMM (a pageable buffer may be
 *          reused when the call returns; a pinned one must stay unchanged
 *          until the stream has passed the call).
 *          SPENSE_GEMM_HOST_Y: Ys[i] [M][N_i] are host pointers; the outputs
 *          are copied back and the call synchronizes `stream` before
 *          returning. Without it the call is asynchronous, like
 *          spense_gemm_grouped.
 *          SPENSE_GEMM_X_PACKED_ORDER as for spense_gemm_grouped_ex.
 *          With neither HOST flag it is spense_gemm_grouped_ex without ldy.
 *   workspace  at least spense_gemm_grouped_host_workspace_size(Wps, count, M)
 *          bytes when a HOST flag is set (else the grouped size), same rules
 *          as spense_gemm. Device-side inputs and outputs keep the alignment
 *          rules of spense_gemm; host ones have none.
 * A typical use is a stack of layers issued in stream order: the first call
 * takes the host input (HOST_X), the middle ones run on device buffers, and
 * the last returns the host output (HOST_Y).
 * Errors: as spense_gemm_grouped, plus ARG for unknown flags.
 */
SPENSE_API spense_status spense_gemm_grouped_host(const spense_packed* const* Wps, int count, const uint8_t* X,
                                                  const float* x_scale, int64_t M, uint16_t* const* Ys,
                                                  void* workspace, size_t workspace_bytes, unsigned int flags,
                                                  void* stream);

SPENSE_API size_t spense_gemm_grouped_host_workspace_size(const spense_packed* const* Wps, int count, int64_t M);

/*
 * spense_gemm_host — the same GEMM on HOST buffers: copies X [M][K] and
 * x_scale [M] from host memory into the workspace, runs spense_gemm, copies Y
 * [M][N] back to host memory and synchronizes `stream` before returning.
 * Host buffers should be pinned for asynchronous copies. workspace must hold
 * spense_gemm_host_workspace_size(Wp, M) bytes (zero-filled before first use).
 * It is spense_gemm_grouped_host over one weight with both HOST flags.
 */
SPENSE_API spense_status spense_gemm_host(const spense_packed* Wp, const uint8_t* X_host,
                               const float* x_scale_host, int64_t M, uint16_t* Y_host,
                               void* workspace, size_t workspace_bytes, void* stream);

SPENSE_API size_t spense_gemm_host_workspace_size(const spense_packed* Wp, int64_t M);

/*
 * spense_glu_order — the order in which SpenseGPT+ lays out the intermediate
 * indices of a GLU MLP once its dense set is chosen (Technical Summary §2.B:
 * the selected dense indices are permuted into one contiguous block; the
 * permutation leaves the MLP's output unchanged): every index in [0, I) that is
 * not in dense_idx, ascending, then dense_idx. It is also the packed column
 * order spense_pack gives a weight packed with this dense set. Pack the gate
 * and up rows with spense_pack_rows(rows = order) to make their outputs arrive
 * in this order, so down (packed with the same dense set) reads them with
 * SPENSE_GEMM_X_PACKED_ORDER and no gather.
 *   I          1 .. 2^20 intermediate indices.
 *   dense_idx  HOST int32 [Kd], strictly ascending in [0, I) (NULL if Kd == 0).
 *   Kd         0 .. I.
 *   order      HOST int32 [I] (caller-owned), written on success.
 * Host only: needs no device. Errors: ARG, SHAPE, DENSE_IDX.
 */
SPENSE_API spense_status spense_glu_order(int64_t I, const int32_t* dense_idx, int64_t Kd, int32_t* order);

/*
 * spense_gemm_noalloc — the same GEMM as spense_gemm, for callers that must not
 * allocate device memory on the call path and so cannot provide a workspace:
 * for example a plugin inside an inference engine that owns every device
 * allocation and hands plugins no allocator, or a serving loop that forbids
 * cudaMalloc after start-up because it can synchronize the device and can fail
 * under memory pressure in the middle of a request. The paper has no
 * counterpart to this entry point; it is a deployment convenience.
 *
 * Instead of a caller workspace it uses one fixed scratch array of
 * SPENSE_NOALLOC_SCRATCH_BYTES (8 MiB + 64 KiB) that the library places in
 * device memory; every GPU that loads the library holds it until the process
 * exits. Calls whose workspace need (spense_gemm_workspace_size) exceeds it
 * are rejected with SPENSE_ERR_WORKSPACE. On a B200 (148 SMs) every weight
 * of the 32B- and 36B-class decoder shapes (K <= 27648, tail dense set) fits
 * for M <= 32 tokens; a SpenseGPT+ weight also stages M x K gathered
 * activation bytes there. The call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 * The first call on a device looks up the array's device address (with that
 * device current), so make that first call before any stream capture; the
 * address is cached per device and context. Every call clears the array's
 * arrival counters on `stream` before the GEMM. A wait that gave up on the
 * device is recorded in the array's status word, which stays set until
 * spense_noalloc_status reads and clears it. All calls share the one array:
 * calls whose execution can overlap on the GPU (different streams without
 * ordering between them) race on it and give wrong results; serialize them.
 * Arguments, layouts and the remaining errors are those of spense_gemm.
 * Asynchronous on `stream`.
 */
#define SPENSE_NOALLOC_SCRATCH_BYTES ((8u << 20) + (64u << 10))
SPENSE_API spense_status spense_gemm_noalloc(const spense_packed* Wp, const uint8_t* X, const float* x_scale,
                                             int64_t M, uint16_t* Y, void* stream);

/* Reads and clears the status word of spense_gemm_noalloc's scratch array on
 * the current device, as spense_workspace_status does for a workspace: 0 when
 * every noalloc GEMM since the last read completed normally, else an OR of
 * SPENSE_DEVICE_* codes. Synchronizes `stream`. Errors: ARG, UNSUPPORTED, CUDA. */
SPENSE_API spense_status spense_noalloc_status(void* stream, uint32_t* status_out);

/* Releases the handle and its device buffers (stream-ordered on the stream the
 * handle was packed on). NULL is accepted. */
SPENSE_API spense_status spense_free(spense_packed* Wp);

/* Shapes and device addresses of a packed weight (for inspection and tests).
 * Canonical pointers are NULL unless packed with SPENSE_PACK_KEEP_CANONICAL. */
typedef struct spense_packed_info {
  int64_t N, K, Ks, Kd;
  int64_t n_tiles, sparse_blocks, dense_blocks;
  const void* Vs_t;       /* n_tiles * sparse_blocks * 16384 bytes */
  const void* E_t;        /* n_tiles * sparse_blocks * 4096 bytes */
  const void* Wd_t;       /* n_tiles * dense_blocks * 16384 bytes */
  const void* w_scale;    /* fp32 [N] */
  const void* Vs;         /* [N][Ks/2] or NULL */
  const void* E;          /* [N][Ks/8] or NULL */
  const void* Wd;         /* [N][Kd] or NULL */
  const int32_t* perm;    /* device int32 [K]: sparse columns then dense columns, or NULL (tail) */
  uint64_t weight_bytes;  /* bytes of Vs_t + E_t + Wd_t */
} spense_packed_info;

SPENSE_API spense_status spense_get_info(const spense_packed* Wp, spense_packed_info* info);

/* The launch plan a grouped GEMM would get, from shapes alone (no device
 * memory, no GPU needed; for inspection and host-side tests of the planner).
 * Member i is an N[i] x K[i] weight with Kd[i] dense columns (tail), all
 * sharing one activation tensor of M tokens, planned for a device with `sms`
 * SMs. Shape rules and errors are those of spense_pack and
 * spense_gemm_grouped (members must share K). Blocks are numbered member by
 * member, row tile by row tile (token tiles of one row tile consecutive),
 * 2:4 blocks before dense blocks within a tile; CTA g of the launch streams
 * blocks [cta_start[g], cta_start[g + 1]). With cluster > 1 the CTAs of one
 * cluster (cluster consecutive CTAs) split the blocks of one tile. */
#define SPENSE_PLAN_MAX_GRID 320
typedef struct spense_plan_info {
  int32_t npad;          /* tokens per token tile, padded to a multiple of 16 (the MMA N) */
  int32_t box_rows;      /* activation rows one tile load covers */
  int32_t m_tiles;       /* token tiles */
  int32_t n_tiles;       /* 128-row weight tiles over all members */
  int32_t tiles;         /* n_tiles * m_tiles */
  int32_t ctas_per_sm;   /* 1 or 2 */
  int32_t cluster;       /* 1 (stream-K) or the cluster size S splitting each tile's K */
  int32_t grid;          /* CTAs */
  int32_t stages;        /* shared-memory ring stages per CTA */
  int32_t nacc;          /* accumulator buffers in tensor memory */
  uint32_t tmem_cols;    /* tensor-memory columns allocated per CTA */
  uint32_t smem_bytes;   /* dynamic shared memory per CTA */
  uint32_t stage_bytes;  /* bytes of one ring stage */
  uint32_t recv_bytes;   /* cluster mode: rank 0's area for the peers' partials */
  int32_t l2_prefetch;   /* weight blocks per CTA prefetched into L2 at start */
  int32_t pair;          /* 1: CTA pairs share 256-row MMAs; grid, n_tiles and cta_start then count pairs */
  uint32_t y_stage_bytes; /* stream-K: shared memory staging whole output tiles for 16-byte stores (0: none) */
  int64_t total_blocks;  /* blocks the launch streams */
  uint64_t workspace_bytes;                    /* spense_gemm_grouped_workspace_size */
  int32_t cta_start[SPENSE_PLAN_MAX_GRID + 1]; /* [grid] = total_blocks */
} spense_plan_info;

SPENSE_API spense_status spense_plan_shapes(int count, const int64_t* N, const int64_t* K, const int64_t* Kd,
                                            int64_t M, int sms, spense_plan_info* out);

/* Reads and clears the status word a workspace carries. *status_out receives 0
 * when every kernel that used the workspace completed normally, else a bitwise
 * OR of SPENSE_DEVICE_* codes. Synchronizes `stream`. */
#define SPENSE_DEVICE_TIMEOUT_PRODUCER 0x1u
#define SPENSE_DEVICE_TIMEOUT_MMA 0x2u
#define SPENSE_DEVICE_TIMEOUT_EPILOGUE 0x4u
SPENSE_API spense_status spense_workspace_status(void* workspace, void* stream, uint32_t* status_out);

/* Message describing the last error on the calling thread ("" if none). */
SPENSE_API const char* spense_last_error(void);

/* Library version, "major.minor.patch". */
SPENSE_API const char* spense_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPENSE_H_ */
