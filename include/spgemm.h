/*
 * spgemm.h -- C ABI of the B200 (sm_100a) library for the pruned-weight linear
 * layer Y = X . W^T with 2:4 fine-grained and tile-wise structured sparsity.
 *
 * Sources:
 *  [GPUSQ]  "Boost Vision Transformer with GPU-Friendly Sparsity and
 *           Quantization", Abstract: weights pruned to the 2:4 pattern for
 *           fp16 2:4 sparse tensor cores, then quantised to integer 2:4.
 *  [TW]     "Accelerating Sparse DNN Models without Hardware-Support via
 *           Tile-Wise Sparsity" (Guo et al.), slides "Tile-Wise Sparsity",
 *           "Re-organize", "Preprocessed", "Run-time" and "Transpose".
 *
 * Conventions (all entry points):
 *  - Matrices are row-major.  W is [N, K] (K contiguous), X is [M, K] (or
 *    [K, M] where stated), Y is [M, N].  ld* are row pitches in ELEMENTS.
 *  - Every pointer argument not described as "host" is a device pointer owned
 *    by the caller.  The library never allocates device memory and never
 *    frees caller memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; 0 = legacy
 *    default stream) and does not synchronise.  Arguments are validated on
 *    the host first: on any error nothing is launched and the status says
 *    why.  SPG_ERR_CUDA means a CUDA runtime call (for example the launch)
 *    failed; cudaGetLastError() has the detail.
 *  - Kernels never wait without bound: a pipeline wait that exceeds about a
 *    second makes the kernel record a code in the library's device error
 *    word and return early.  spg_check_device_error() reads (and clears)
 *    that word.
 *  - Device requirement: compute capability 10.0 (B200, sm_100a); other
 *    devices get SPG_ERR_UNSUPPORTED_DEVICE.
 *  - The library looks up the device addresses of its own device arrays (the
 *    error word, the scratch of spgemm_tw_f16_noalloc) once per device and
 *    keeps them for the life of the process.  Do not use it across
 *    cudaDeviceReset() or any other teardown of a device's primary context:
 *    the kept addresses would no longer be valid.
 *  - An empty batch (M == 0) is valid for every GEMM entry point except
 *    spgemm_tw_f16_noalloc: the other arguments are validated as usual,
 *    nothing is launched, SPG_OK is returned, and X, Y (and the workspace)
 *    may be NULL.
 */
#ifndef SPGEMM_H_
#define SPGEMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* spg_stream_t; /* == cudaStream_t */

typedef enum {
  SPG_OK = 0,
  SPG_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum value */
  SPG_ERR_UNSUPPORTED_SHAPE = 2, /* a size or pitch outside the documented limits */
  SPG_ERR_MISALIGNED = 3,        /* a pointer or pitch breaks the stated alignment */
  SPG_ERR_UNSUPPORTED_DEVICE = 4,/* current device is not compute capability 10.0 */
  SPG_ERR_CUDA = 5,              /* a CUDA runtime call failed */
  SPG_ERR_TIMEOUT = 6            /* a kernel gave up on a bounded wait */
} spg_status;

typedef enum { SPG_F16 = 0, SPG_BF16 = 1, SPG_S8 = 2 } spg_dtype;

enum { SPG_OUT_F16 = 0, SPG_OUT_S32 = 1 };  /* spgemm_24_s8 output modes */
enum { SPG_X_MK = 0, SPG_X_KM = 1 };        /* spgemm_tw_f16 activation layouts */
enum { SPG_ACT_NONE = 0, SPG_ACT_GELU = 1 }; /* spgemm_24_s8_q activations */

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int spg_version(void);

/* Static, human-readable name of a status code. */
const char* spg_status_string(spg_status s);

/* Takes the current device's error word and clears it in one atomic step
 * (a one-thread kernel on `stream`), synchronises `stream` and returns what
 * it took.  Returns SPG_ERR_TIMEOUT if any kernel gave up on a bounded wait
 * since the last check (the bits are stored in *bits if bits != NULL),
 * SPG_ERR_CUDA if the launch or the synchronisation failed, SPG_OK
 * otherwise.  A bit set by a kernel still running on another stream is
 * either taken by this call or left for the next one, never lost. */
spg_status spg_check_device_error(spg_stream_t stream, uint32_t* bits);

/* Self-test of the failure path every kernel uses (no counterpart on the
 * pages): launches one thread that waits, with the library's bounded wait
 * and a limit of limit_ns nanoseconds (0 < limit_ns <= 10 s), on an mbarrier
 * that nothing ever completes.  The wait gives up, records bit 6 in the
 * device error word and the kernel returns; nothing faults and the context
 * stays usable.  A following spg_check_device_error() returns
 * SPG_ERR_TIMEOUT with that bit (and clears it).  Asynchronous on `stream`. */
spg_status spg_selftest_bounded_wait(int64_t limit_ns, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * sparse_prune_24  [GPUSQ, Abstract: "2:4 structured pruning"]
 *
 * Wm = W with, in every group of 4 consecutive elements along K, the 2
 * elements of largest magnitude kept and the other 2 set to +0.  Magnitudes
 * compare exactly (fp16/bf16: bit pattern with the sign cleared; int8: |q|);
 * among equal magnitudes the lower index is kept.  Exactly 2 slots are kept
 * per group.  NaN/Inf inputs are outside the contract.
 *   W    [N, K] of `dtype`, pitch ldw >= K          (read)
 *   Wm   [N, K] of `dtype`, pitch ldwm >= K         (written; may equal W
 *        when ldwm == ldw: in-place is allowed)
 *   K % 4 == 0; N, K >= 0.  W and Wm must be 8-byte aligned with pitches
 *   in bytes a multiple of 8 (16-bit types) or 4 (int8).
 * ------------------------------------------------------------------------- */
spg_status sparse_prune_24(const void* W, int64_t ldw, void* Wm, int64_t ldwm, int64_t N, int64_t K,
                           spg_dtype dtype, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * sparse_compress_24  [GPUSQ, Abstract; storage format of the 2:4 pattern]
 *
 * Same selection rule as sparse_prune_24 (so compress(prune(W)) ==
 * compress(W)), emitted in compressed form:
 *   Wv   [N, K/2] of `dtype`, contiguous (pitch K/2): the kept values of each
 *        group in K order, Wv[n][2g+s] = W[n][4g+i_s], i0 < i1.
 *   meta [N, K/8] bytes, contiguous (pitch K/8): one 4-bit code per group,
 *        code = i0 | i1 << 2; group 2b in bits 0..3 of meta[n][b], group 2b+1
 *        in bits 4..7.
 *   W    [N, K], pitch ldw >= K.  K % 8 == 0.  W 8-byte aligned, ldw in bytes
 *   a multiple of 8; Wv and meta 4-byte aligned.
 * This canonical metadata is what the GEMMs below consume; the arrangement
 * the tensor cores need in tensor memory is produced inside the GEMM kernels.
 * ------------------------------------------------------------------------- */
spg_status sparse_compress_24(const void* W, int64_t ldw, void* Wv, uint8_t* meta, int64_t N, int64_t K,
                              spg_dtype dtype, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_24_f16  [GPUSQ, Abstract: fp16 2:4 sparse tensor-core GEMM]
 *
 * Y[m][n] = round( sum_k X[m][k] * Wm[n][k]  (+ bias[n]) ) with Wm the
 * decompressed (Wv, meta) weight, products accumulated in fp32 on the 2:4
 * sparse tensor cores, bias added in fp32, one round-to-nearest-even to
 * `dtype` (SPG_F16 or SPG_BF16; X, Wv, bias and Y all share it).
 *   X    [M, K], pitch ldx >= K
 *   Wv, meta: as written by sparse_compress_24 for [N, K]
 *   bias [N] or NULL
 *   Y    [M, N], pitch ldy >= N
 * Limits: K % 64 == 0, K >= 64; M >= 0, N >= 1 (any value, ragged tiles are
 * handled); M, N, K < 2^31.  X, Wv, Y 16-byte aligned; ldx and ldy in bytes
 * multiples of 16; meta 16-byte aligned; bias 2-byte aligned.  (K % 128 != 0
 * is served by a last pipeline stage of half depth; its metadata rows of K/8
 * bytes are then read without TMA.)
 * ------------------------------------------------------------------------- */
spg_status spgemm_24_f16(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                         void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, spg_dtype dtype,
                         spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_24_f16_host  [GPUSQ, Abstract; the layer called from host memory]
 *
 * spgemm_24_f16 on activations and outputs in HOST memory: X_host [M, K]
 * (pitch ldx_host >= K elements) is copied into the caller's device buffer
 * X_dev (pitch K), the layer writes Y_dev [M, N] (pitch ldy_dev), and Y_dev
 * is copied to Y_host [M, N] (pitch ldy_host >= N), all asynchronously on
 * `stream` (cudaMemcpy2DAsync; host memory should be page-locked for the
 * copies to be asynchronous).  Nothing is allocated: X_dev needs M*K*2 bytes
 * and Y_dev M*ldy_dev*2 bytes.  Wv, meta, bias and dtype as spgemm_24_f16;
 * X_dev and Y_dev must satisfy its alignment rules (16-byte aligned, ldy_dev
 * in bytes a multiple of 16).  The host buffers must stay valid until the
 * stream reaches the copy-out.
 * ------------------------------------------------------------------------- */
spg_status spgemm_24_f16_host(const void* X_host, int64_t ldx_host, const void* Wv, const uint8_t* meta,
                              const void* bias, void* Y_host, int64_t ldy_host, int64_t M, int64_t N, int64_t K,
                              spg_dtype dtype, void* X_dev, void* Y_dev, int64_t ldy_dev, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_24_f16_gelu  [GPUSQ, Abstract: the 2:4 layers of a vision
 * transformer; the activation between the two layers of its MLP block]
 *
 * spgemm_24_f16 with the activation fused into the epilogue:
 *   Y[m][n] = round( GELU( sum_k X[m][k] * Wm[n][k] (+ bias[n]) ) )
 * with GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt(2))) evaluated in fp32
 * after the fp32 bias add, then one round-to-nearest-even to `dtype`.
 * Same arguments and limits as spgemm_24_f16.
 * ------------------------------------------------------------------------- */
spg_status spgemm_24_f16_gelu(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                              void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, spg_dtype dtype,
                              spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_24_f16_yt  [GPUSQ, Abstract; TW, slide "Transpose": the transpose
 * the next tile-wise layer needs, fused into the producing layer]
 *
 * spgemm_24_f16 writing the transpose of Y: Yt[n][m] = Y[m][n], Yt [N, M]
 * with pitch ldyt >= M.  A tile-wise layer that follows reads Yt directly as
 * its [K, M] activations (spgemm_tw_f16 with SPG_X_KM), with no transpose.
 * Same arithmetic, bit-identical values.  Same limits as spgemm_24_f16 with
 * Y replaced by Yt: Yt 16-byte aligned, ldyt in bytes a multiple of 16.
 * ------------------------------------------------------------------------- */
spg_status spgemm_24_f16_yt(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                            void* Yt, int64_t ldyt, int64_t M, int64_t N, int64_t K, spg_dtype dtype,
                            spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_24_s8  [GPUSQ, Abstract: "2:4 sparse calculation with integer tensors"]
 *
 * acc[m][n] = sum_k X[m][k] * Wm[n][k] in exact int32 on the 2:4 sparse
 * tensor cores (int8 x int8), then
 *   out_mode SPG_OUT_S32: Y (int32) = acc;
 *   out_mode SPG_OUT_F16: Y (fp16)  = fp16_rn( fp32(acc) *rn scale[n]
 *                                              [ +rn fp32(bias[n]) ] )
 * (one fp32 multiply, optionally one fp32 add, then one round to fp16; a
 * per-tensor activation scale is folded into scale[] by the caller).
 *   X int8 [M, K] pitch ldx; Wv int8 [N, K/2] + meta [N, K/8] from
 *   sparse_compress_24 (dtype SPG_S8); scale fp32 [N] (required for F16,
 *   ignored for S32); bias fp16 [N] or NULL; Y [M, N] pitch ldy.
 * Limits: K % 128 == 0, K >= 128; |acc| must fit int32 (K <= 2^17 is always
 * safe); same alignment rules as spgemm_24_f16 (ldy in bytes a multiple of
 * 16); scale 4-byte aligned.
 * ------------------------------------------------------------------------- */
spg_status spgemm_24_s8(const int8_t* X, int64_t ldx, const int8_t* Wv, const uint8_t* meta, const float* scale,
                        const void* bias, void* Y, int64_t ldy, int out_mode, int64_t M, int64_t N, int64_t K,
                        spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_24_s8_q  [GPUSQ, Abstract: the fixed-point (int8) 2:4 model; the
 * int8 activations of the next layer produced by this layer's epilogue]
 *
 * acc as spgemm_24_s8, then per element, in fp32 with one round-to-nearest-
 * even per operation and no fused multiply-add:
 *   v = fp32(acc) * scale[n]  [ + fp32(bias[n]) ]
 *   act SPG_ACT_GELU: v = GELU(v) = (0.5 v) (1 + erf(v * 0.70710677)), with
 *     erf(u) = sign(u) (1 - r) (Abramowitz & Stegun 7.1.28, |error| <= 3e-7):
 *     a = min(|u|, 4); p = ((((((a6 a + a5) a + a4) a + a3) a + a2) a + a1) a)
 *     + 1 with a1..a6 = 0.0705230784, 0.0422820123, 0.0092705272,
 *     0.0001520143, 0.0002765672, 0.0000430638; p^16 by four squarings;
 *     r = 1 / p^16 by three Newton steps r = r (2 - p^16 r) from the fp32
 *     whose bits are 0x7EF00000 - bits(p^16)
 *   Yq[m][n] (int8) = clamp( rne( v * qscale ), -127, 127 )
 * qscale is the reciprocal of the next layer's activation scale (that scale is
 * folded into the next layer's scale[]).  The fixed operation order makes the
 * int8 codes reproducible bit for bit on the host.
 *   X, Wv, meta, scale, bias as spgemm_24_s8; Yq int8 [M, N], pitch ldy
 *   (bytes, a multiple of 16), 16-byte aligned; 0 < qscale < 3e38.
 * ------------------------------------------------------------------------- */
spg_status spgemm_24_s8_q(const int8_t* X, int64_t ldx, const int8_t* Wv, const uint8_t* meta, const float* scale,
                          const void* bias, float qscale, int act, int8_t* Yq, int64_t ldy, int64_t M, int64_t N,
                          int64_t K, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * Tile-wise sparsity  [TW, slides "Tile-Wise Sparsity", "Re-organize",
 * "Preprocessed", "Run-time"]
 *
 * A dense fp16 W [N, K] is condensed offline: the n_pruned columns of
 * B = W^T (rows n of W) with the smallest L2 norm are pruned (ties: lower n
 * pruned first); the kept columns, ascending (offsetn), are cut into tiles
 * of G consecutive kept columns (the last tile may be shorter); tile t keeps
 * the k_per_tile[t] rows k with the largest L2 norm over its own columns
 * (ties: lower k kept), ascending (offsetk).  Norms are compared exactly.
 * Tile t owns output columns [tile_n0[t], tile_n0[t+1]) of Y: its kept
 * columns and the pruned columns between them (tile 0 starts at 0, the last
 * tile ends at N); pruned columns of Y are written as +0.
 *
 * Descriptor buffers (device, caller-allocated with the sizes from
 * tw_query_sizes, filled by tw_reorganize).  With kpad_t = round-up of
 * k_per_tile[t] to a multiple of 64 and tile_kofs the prefix sums of kpad_t:
 *   offsetn    int32 [Nk]        kept columns, ascending (Nk = N - n_pruned)
 *   tile_n0    int32 [T+1]       output column range of each tile
 *   tile_kofs  int32 [T+1]       start of each tile in offsetk (multiples of 64)
 *   k_per_tile int32 [T]         kept rows per tile
 *   offsetk    int32 [tile_kofs[T]]  tile t's kept k ascending at
 *                                [tile_kofs[t], +k_t), then kpad_t - k_t pad
 *                                entries equal to its last kept k
 *   Wc         fp16 [tile_kofs[T]/64][G][64]  condensed values: block b of
 *                                tile t (block index tile_kofs[t]/64 + b)
 *                                holds Wc[j][c] = W[offsetn[tG+j]][offsetk[
 *                                tile_kofs[t] + 64b + c]] for j < G_t and
 *                                64b + c < k_t, and +0 elsewhere.
 * ------------------------------------------------------------------------- */
typedef struct {
  int64_t N, K, Nk;
  int32_t G, T;
  int64_t offsetk_len;    /* tile_kofs[T] */
  int64_t wc_elems;       /* offsetk_len * G */
  int64_t reorg_ws_bytes; /* device workspace tw_reorganize needs (exact column norms) */
} spg_tw_sizes;

typedef struct {
  int64_t N, K, Nk;
  int32_t G, T;
  int64_t offsetk_len;
  int32_t* offsetn;
  int32_t* tile_n0;
  int32_t* tile_kofs;
  int32_t* k_per_tile;
  int32_t* offsetk;
  void* Wc; /* fp16 */
} spg_tw_desc;

/* Sizes of the descriptor buffers and of the reorganisation workspace.
 * k_per_tile is a HOST array of T entries (T = ceil((N - n_pruned) / G)),
 * each in [1, K].  G must be 128; 0 <= n_pruned < N; K % 64 == 0 and
 * K <= 8192; N < 2^31. */
spg_status tw_query_sizes(int64_t N, int64_t K, int32_t G, int64_t n_pruned, const int32_t* k_per_tile,
                          spg_tw_sizes* out);

/* Fill `desc` (whose sizes and device pointers the caller set; sizes must
 * equal tw_query_sizes) from the dense fp16 W [N, K] (pitch ldw >= K,
 * 2-byte aligned).  k_per_tile is a HOST array of T entries; it is copied
 * to the device before the call returns.  `workspace` (device, 16-byte
 * aligned, ws_bytes >= reorg_ws_bytes) holds the exact column norms; its
 * contents are scratch.  The integer outputs are exact (bit-identical to the
 * selection rule above). */
spg_status tw_reorganize(const void* W, int64_t ldw, int64_t n_pruned, const int32_t* k_per_tile,
                         const spg_tw_desc* desc, void* workspace, size_t ws_bytes, spg_stream_t stream);

/* Workspace bytes spgemm_tw_f16 needs: K*M8*2 with M8 = M rounded up to a
 * multiple of 8 (rounded up to 256 bytes) for x_layout SPG_X_MK (the
 * transposed activations, rows padded to 16 bytes), 0 for SPG_X_KM. */
size_t tw_workspace_size(int64_t M, int64_t K, int x_layout);

/* Y = X . Wd^T with Wd the tile-wise weight described by `desc` [TW,
 * "Run-time": A[offsetA + offsetk[k]], B[offsetB], C[offsetC + offsetn[n]]].
 * X is fp16 [M, K] pitch ldx (x_layout SPG_X_MK; it is first transposed into
 * `workspace`, the explicit transpose of the "Transpose" slide) or fp16
 * [K, M] pitch ldx (SPG_X_KM: the transpose is assumed fused upstream).  Y
 * fp16 [M, N] pitch ldy; every element of Y is written (pruned columns +0).
 * fp32 accumulation, one round-to-nearest-even.
 * Limits: any M >= 0 (M < 2^31; a ragged last block of rows is handled);
 * X and workspace 16-byte aligned, ldx a multiple of 8 (for SPG_X_KM with
 * M % 8 != 0 the caller pads the rows of X to a multiple of 8 elements);
 * Y 2-byte aligned, any ldy >= N; ws_bytes >= tw_workspace_size(M, K,
 * x_layout). */
spg_status spgemm_tw_f16(const void* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, void* Y,
                         int64_t ldy, int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream);

/* Tile-wise GEMM writing the transpose of Y [TW, slide "Transpose": with
 * the transposes fused, a chain of tile-wise layers never leaves the [K, M]
 * activation layout].  Yt[n][m] = Y[m][n] with Y as spgemm_tw_f16 computes
 * it (bit-identical values, pruned columns of Y = rows of Yt written as +0).
 * Yt fp16 [N, M], pitch ldyt >= M, 16-byte aligned, ldyt a multiple of 8.
 * Other arguments and limits as spgemm_tw_f16. */
spg_status spgemm_tw_f16_yt(const void* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, void* Yt,
                            int64_t ldyt, int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * Tile-wise sparsity on the CUDA cores in fp32  [TW, library table (the
 * tile-wise CUDA-fp32 library) and results slide (speedup on CUDA cores)]
 *
 * The pattern of a descriptor filled by tw_reorganize (selected exactly on
 * the fp16 copy of the weights) applied to fp32 weights and activations:
 *   tw_condense_f32: Wc32 [tile_kofs[T]/64][64][G] fp32, k-major (the
 *     descriptor's Wc has the same elements with j and c swapped): block b of
 *     tile t at blk = tile_kofs[t]/64 + b holds Wc32[blk][c][j] =
 *     W[offsetn[tG+j]][offsetk[tile_kofs[t] + 64b + c]] for j < G_t and
 *     64b + c < k_t, +0 elsewhere; W fp32 [N, K], pitch ldw >= K, 4-byte
 *     aligned; Wc32 16-byte aligned, as many elements as the descriptor's Wc.
 *   spgemm_tw_f32: Y [M, N] fp32 = X . Wd^T with Wd the fp32 tile-wise weight,
 *     on the fp32 pipes (fused multiply-add, each tile's kept rows in
 *     ascending order); pruned columns of Y are +0.  X fp32 [M, K] pitch ldx
 *     (SPG_X_MK; first transposed into `workspace`, 16-byte aligned,
 *     ws_bytes >= tw_workspace_size_f32) or [K, M] (SPG_X_KM; 16-byte
 *     aligned, ldx a multiple of 4).  Y 4-byte aligned, any ldy >= N.
 *     M < 2^31 and T * ceil(M / 64) < 2^31 (else SPG_ERR_UNSUPPORTED_SHAPE).
 * ------------------------------------------------------------------------- */
spg_status tw_condense_f32(const float* W, int64_t ldw, const spg_tw_desc* desc, float* Wc32, spg_stream_t stream);

size_t tw_workspace_size_f32(int64_t M, int64_t K, int x_layout);

spg_status spgemm_tw_f32(const float* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, const float* Wc32,
                         float* Y, int64_t ldy, int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream);

/* ---------------------------------------------------------------------------
 * spgemm_tw_f16_noalloc  (no counterpart on the pages: an interface addition)
 *
 * spgemm_tw_f16 with x_layout SPG_X_MK for callers that cannot allocate device
 * memory themselves -- for instance a plug-in running inside a host framework
 * that owns every device allocation and forbids extensions from calling
 * cudaMalloc, or a latency-critical caller that must not pay cudaMalloc's
 * implicit device synchronisation.  The transposed activations [K][M] are
 * kept in a fixed 8 MiB device array inside the library instead of a
 * caller-provided workspace; the caller still passes X, the descriptor and Y.
 *   Same arguments, limits and results as spgemm_tw_f16(X, ldx, SPG_X_MK, desc,
 *   Y, ldy, M, ...), and additionally K * M8 * 2 <= 8 MiB with M8 = M rounded
 *   up to a multiple of 8, else SPG_ERR_UNSUPPORTED_SHAPE (nothing is
 *   launched).
 *   The array is allocated when the library is loaded and every GPU that
 *   loads it holds the 8 MiB until the process exits.  No call allocates or
 *   frees memory.  The first call on a device looks up the array's device
 *   address once (cudaGetSymbolAddress); make that first call before any
 *   stream capture.
 *   All calls share the one array and each call overwrites the part it
 *   reads, so nothing needs clearing between calls; calls that overlap on the
 *   GPU (different streams, or different host threads without ordering) race
 *   on it and must be serialised by the caller.
 * ------------------------------------------------------------------------- */
spg_status spgemm_tw_f16_noalloc(const void* X, int64_t ldx, const spg_tw_desc* desc, void* Y, int64_t ldy,
                                 int64_t M, spg_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SPGEMM_H_ */
