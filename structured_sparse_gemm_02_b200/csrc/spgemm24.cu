// 2:4 structured-sparse GEMM on the sm_100a tensor cores: Y = X . W^T with W
// stored as 2:4-compressed values plus 2-bit position metadata ("Boost Vision
// Transformer with GPU-Friendly Sparsity and Quantization", Abstract: fp16
// 2:4 sparse tensor cores, and integer 2:4 tensors for the quantised model).
//
// Mapping: the sparse MMA operand A is a 128-row tile of the compressed
// weight (rows = output columns n), B is a BN-row tile of X (rows = output
// rows m), and the fp32/s32 accumulator D[n][m] lives in tensor memory
// (lane = n, column = m).  A tile of Y^T is 128 x BN.
//
// Persistent kernel on cluster pairs, one CTA per SM, warp roles (384 threads):
//   warp 0     TMA producer: compressed W, X and the canonical metadata of
//              every stage into a STAGES-deep ring that runs across tiles
//   warp 1     fp16/bf16 only: rearranges each stage's metadata into the
//              order the tensor cores read it (permute_meta_f16), then
//              arrives on the leader's barrier of the stage, which completes
//              once both CTAs' operands have landed and both metadata warps
//              have arrived.  When K % 128 != 0 the canonical metadata rows
//              (K/8 bytes) are not 16-byte multiples, which a TMA map needs:
//              this warp then reads them from global memory itself.
// K is a multiple of the MMA pair of a stage (64 for fp16/bf16, 128 for
// int8): a last stage with half the K of the others issues two MMAs instead
// of four, and its out-of-range operand columns are zero-filled by TMA.
//   warp 2     TMEM owner and MMA issuer (one thread of the leader CTA):
//              waits for a stage, then issues it (tcgen05.cp of the
//              metadata into tensor memory, tcgen05.mma.sp into one of two
//              accumulators) and commits the stage's slot
//   warp 3     idle
//   warps 4-11 epilogue, two warps per tensor-memory lane quadrant:
//              tcgen05.ld of a finished accumulator (released as soon as it
//              is read), bias / dequant, convert, TMA store of output boxes;
//              the ragged right edge uses checked stores
// Every wait is bounded (sm100.cuh); on a timeout the CTA drains what it has
// in flight, frees tensor memory and exits with the error word set.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "host.cuh"
#include "sm100.cuh"
#include "spgemm.h"

namespace spg {
namespace gemm24 {

// Output kinds: Y [M][N] in fp16 / bf16 / int32, or the transpose Y^T [N][M]
// in fp16 / bf16 (the layout a following tile-wise layer reads as its
// activations, so that layer needs no transpose).
// GELU kinds: Y [M][N] = GELU(acc + bias) in fp16 / bf16 (the activation
// between the two layers of a transformer MLP block, fused into the first).
// Quantised kinds (int8 inputs only): Y [M][N] int8 = clamp(rne(v * qscale))
// with v the dequantised value, optionally through GELU first: the int8
// activations of the next 2:4 int8 layer.
enum OutKind {
  OUT_F16 = 0, OUT_BF16 = 1, OUT_S32 = 2, OUT_F16_T = 3, OUT_BF16_T = 4, OUT_F16_G = 5, OUT_BF16_G = 6,
  OUT_S8Q = 7, OUT_S8QG = 8
};
__host__ __device__ constexpr bool out_bf16(int k) { return k == OUT_BF16 || k == OUT_BF16_T || k == OUT_BF16_G; }
__host__ __device__ constexpr bool out_gelu(int k) { return k == OUT_F16_G || k == OUT_BF16_G || k == OUT_S8QG; }
__host__ __device__ constexpr bool out_s8(int k) { return k == OUT_S8Q || k == OUT_S8QG; }

// GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)), in fp32, for the 16-bit
// epilogues (checked against the fp64 definition within the output tolerance).
// erfc from Abramowitz & Stegun 7.1.26: for u >= 0,
//   erfc(u) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-u^2),  t = 1 / (1 + p u),
// with |error| <= 1.5e-7, evaluated branch-free with the hardware reciprocal
// and base-2 exponential approximations:
//   Phi(v) = 1 - erfc(|v| / sqrt 2) / 2 for v >= 0, erfc(|v| / sqrt 2) / 2 otherwise.
__device__ __forceinline__ float gelu_f32(float v) {
  const float u = fabsf(v) * 0.70710678118654752f;
  float t, ex;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, u, 1.0f)));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  poly *= t;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ex) : "f"(-(u * u) * 1.4426950408889634f));  // exp(-u^2)
  const float half_erfc = 0.5f * poly * ex;
  return v * (v >= 0.0f ? 1.0f - half_erfc : half_erfc);
}

// GELU for the quantised path, where the rounded result decides an integer
// code and must be reproducible bit for bit on the host: erf from
// Abramowitz & Stegun 7.1.28, erf(a) = 1 - 1 / (1 + a1 a + ... + a6 a^6)^16
// for a >= 0 (|error| <= 3e-7), odd extension.  Every operation is one fp32
// round-to-nearest-even in the order written, no fused multiply-add:
//  * a = min(|u|, 4): at 4 the result is already 1.0f, so p^16 stays finite;
//  * 1 / p^16 by three Newton steps r = r (2 - x r) from the seed whose bits
//    are 0x7EF00000 - bits(x) (exponent flipped, within 6.25 %): relative
//    error about 1.5e-7 and no division.
__device__ __forceinline__ float gelu_as_f32(float v) {
  const float u = __fmul_rn(v, 0.70710677f);
  const float a = fminf(fabsf(u), 4.0f);
  float h = 0.0000430638f;
  h = __fadd_rn(__fmul_rn(h, a), 0.0002765672f);
  h = __fadd_rn(__fmul_rn(h, a), 0.0001520143f);
  h = __fadd_rn(__fmul_rn(h, a), 0.0092705272f);
  h = __fadd_rn(__fmul_rn(h, a), 0.0422820123f);
  h = __fadd_rn(__fmul_rn(h, a), 0.0705230784f);
  const float p = __fadd_rn(__fmul_rn(h, a), 1.0f);
  const float p2 = __fmul_rn(p, p);
  const float p4 = __fmul_rn(p2, p2);
  const float p8 = __fmul_rn(p4, p4);
  const float p16 = __fmul_rn(p8, p8);
  float r = __uint_as_float(0x7EF00000u - __float_as_uint(p16));
#pragma unroll
  for (int it = 0; it < 3; ++it) r = __fmul_rn(r, __fsub_rn(2.0f, __fmul_rn(p16, r)));
  const float e = __fsub_rn(1.0f, r);
  const float erf_u = u < 0.0f ? -e : e;
  return __fmul_rn(__fmul_rn(0.5f, v), __fadd_rn(1.0f, erf_u));
}

// Pair tile: 256 weight rows (128 per CTA of the cluster pair) x BN rows of X
// (BN/2 loaded by each CTA).  STAGES is the deepest operand ring that fits.
// Stages waited for before their MMAs are issued.  A wait between two groups
// of MMAs leaves the tensor pipe idle for a while, which larger groups
// amortise, but waiting for a second stage delays the first one's MMAs while
// the ring is short of loads; on the ViT-Base MLP shapes a group of two was
// slower than one (42.0 / 42.6 against 40.1 / 39.2 us).
constexpr int kIssueGroup = 1;

template <bool kInt8, int BN, int OUT>
struct Cfg {
  static constexpr int BMC = 128;                      // weight rows per CTA (MMA M = 256 per pair)
  static constexpr int BNH = BN / 2;                   // X rows loaded by each CTA
  static constexpr int KSTEP = kInt8 ? 256 : 128;      // logical K per pipeline stage
  static constexpr int A_BYTES = BMC * 128;            // 128 B of compressed row per stage
  static constexpr int B_BYTES = BNH * 256;            // 256 B of X row per stage (two 128 B atoms)
  static constexpr int MSTG_BYTES = kInt8 ? 4096 : 2048;  // canonical metadata of the stage (TMA)
  static constexpr int MCP_BYTES = kInt8 ? 0 : 2048;      // fp16/bf16: metadata in tcgen05.cp order
  static constexpr int MCOLS = kInt8 ? 8 : 4;          // TMEM columns of metadata per stage
  static constexpr int OUT_ES = OUT == OUT_S32 ? 4 : out_s8(OUT) ? 1 : 2;
  static constexpr bool YT = OUT == OUT_F16_T || OUT == OUT_BF16_T;  // Y^T: stored from registers
  static constexpr bool OUT_BF = out_bf16(OUT);
  // staging per epilogue warp: 16-bit outputs double-buffer a 4 KB box per warp
  // pair (2 KB per warp and buffer); int32 outputs one 4 KB box per warp
  static constexpr int EPI_BUF = OUT_ES == 2 ? 2 * 2048 : 4096;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + MSTG_BYTES + MCP_BYTES;
  // full[S], mtma[S], empty[S], acc_full[2], acc_empty[2], mma_done
  static constexpr int EPI_WARPS = 8;                  // two per tensor-memory lane quadrant
  static constexpr int THREADS = 32 * (4 + EPI_WARPS);
  static constexpr int NCH = BN / 32;                  // 32-column chunks of an accumulator
  static constexpr int BAR_BYTES_MAX = (4 * 8 + 5) * 8 + 16;
  static constexpr int FIXED = EPI_WARPS * EPI_BUF + BAR_BYTES_MAX + 1024;
  static constexpr int STAGES_FIT = (232448 - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_MSTG = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_MCP = OFF_MSTG + STAGES * MSTG_BYTES;
  static constexpr int OFF_EPI = OFF_MCP + STAGES * MCP_BYTES;
  static constexpr int OFF_BAR = OFF_EPI + EPI_WARPS * EPI_BUF;
  static constexpr int NUM_BARS = 3 * STAGES + 5;
  static constexpr int SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr uint32_t META_COL = 2 * BN;  // metadata ring after the two accumulators
  static constexpr uint32_t TMEM_NEED = 2 * BN + 2 * MCOLS;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32    ? 32
                                        : TMEM_NEED <= 64  ? 64
                                        : TMEM_NEED <= 128 ? 128
                                        : TMEM_NEED <= 256 ? 256
                                                           : 512;
  // bytes counted on the leader's full barrier per stage: operands of both CTAs
  // (int8 also its metadata; fp16/bf16 metadata completes on a local barrier)
  static constexpr uint32_t TX_PAIR = 2u * (A_BYTES + B_BYTES + (kInt8 ? MSTG_BYTES : 0));
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256 && BNH % 8 == 0, "BN");
  static_assert(STAGES >= 2, "at least two stages");
  static_assert(TMEM_NEED <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert((B_BYTES % 1024) == 0 && ((BNH * 128) % 1024) == 0, "swizzle atoms stay 1024-aligned");
};

// ---- metadata arrangement ------------------------------------------------------------
// The canonical metadata of a stage is a [128 rows][16 B] box (fp16/bf16: 128
// logical K = 4 MMAs of K 32) or two such boxes (int8: 256 logical K = 4 MMAs
// of K 64), loaded by TMA next to the operands.  tcgen05.cp moves a
// [128][16 B] block into 4 TMEM columns, 16-byte row r -> lane r.
//
// int8 (kind::i8): lane = weight row, the 64 metadata bits of an MMA are two
// consecutive columns in K order -> the canonical boxes are copied as they are.
//
// fp16/bf16 (kind::f16, 32 metadata bits per row per MMA): the tensor cores
// read lane L = m0 + 8*h + 16*m2 (m0 < 8, h < 2, m2 < 8) column j as the 16
// bits of row r = m0 + 16*m2 for K half h of MMA j (low half) and the same 16
// bits of row r + 8 (high half).  For every row pair (r, r+8) the 16-bit
// units are therefore exchanged like a 2x2 transpose:
//   lane r     <- { r.unit(2j),   (r+8).unit(2j)   }  j = 0..3
//   lane r + 8 <- { r.unit(2j+1), (r+8).unit(2j+1) }
// where unit u is bits [16u, 16u+16) of a row's 16 canonical bytes.
__device__ __forceinline__ void permute_meta_f16(const uint8_t* stg, uint8_t* out, int lane) {
#pragma unroll
  for (int pp = 0; pp < 2; ++pp) {
    const int p = lane + 32 * pp;
    const int r = (p & 7) + 16 * (p >> 3);
    const uint4 a = *reinterpret_cast<const uint4*>(stg + r * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(stg + (r + 8) * 16);
    uint4 lo, hi;
    lo.x = __byte_perm(a.x, b.x, 0x5410);
    lo.y = __byte_perm(a.y, b.y, 0x5410);
    lo.z = __byte_perm(a.z, b.z, 0x5410);
    lo.w = __byte_perm(a.w, b.w, 0x5410);
    hi.x = __byte_perm(a.x, b.x, 0x7632);
    hi.y = __byte_perm(a.y, b.y, 0x7632);
    hi.z = __byte_perm(a.z, b.z, 0x7632);
    hi.w = __byte_perm(a.w, b.w, 0x7632);
    *reinterpret_cast<uint4*>(out + r * 16) = lo;
    *reinterpret_cast<uint4*>(out + (r + 8) * 16) = hi;
  }
}

// The same arrangement read straight from the canonical metadata in global
// memory (rows of `pitch` bytes, 8-byte aligned): 16 bytes of rows n0 + r,
// starting at byte col0, of which `valid` (8 or 16) are inside the row; rows
// at or past N and bytes past `valid` read as zero.
__device__ __forceinline__ uint4 load_meta_row16(const uint8_t* meta, int64_t pitch, int row, int N, int col0,
                                                 int valid) {
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (row < N) {
    const uint2* src = reinterpret_cast<const uint2*>(meta + int64_t(row) * pitch + col0);
    const uint2 lo = __ldg(src);
    v.x = lo.x;
    v.y = lo.y;
    if (valid > 8) {
      const uint2 hi = __ldg(src + 1);
      v.z = hi.x;
      v.w = hi.y;
    }
  }
  return v;
}

__device__ __forceinline__ void permute_meta_f16_direct(const uint8_t* meta, int64_t pitch, int n0, int N, int col0,
                                                        int valid, uint8_t* out, int lane) {
#pragma unroll
  for (int pp = 0; pp < 2; ++pp) {
    const int p = lane + 32 * pp;
    const int r = (p & 7) + 16 * (p >> 3);
    const uint4 a = load_meta_row16(meta, pitch, n0 + r, N, col0, valid);
    const uint4 b = load_meta_row16(meta, pitch, n0 + r + 8, N, col0, valid);
    uint4 lo, hi;
    lo.x = __byte_perm(a.x, b.x, 0x5410);
    lo.y = __byte_perm(a.y, b.y, 0x5410);
    lo.z = __byte_perm(a.z, b.z, 0x5410);
    lo.w = __byte_perm(a.w, b.w, 0x5410);
    hi.x = __byte_perm(a.x, b.x, 0x7632);
    hi.y = __byte_perm(a.y, b.y, 0x7632);
    hi.z = __byte_perm(a.z, b.z, 0x7632);
    hi.w = __byte_perm(a.w, b.w, 0x7632);
    *reinterpret_cast<uint4*>(out + r * 16) = lo;
    *reinterpret_cast<uint4*>(out + (r + 8) * 16) = hi;
  }
}

// Wait used only while tearing down: ignores the abort flag, still bounded.
__device__ __forceinline__ void tail_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  int never = 0;
  mbar_wait(bar, parity, &never, err, ERR_WAIT_TAIL);
}

// Accumulator -> output bits.  fp16/bf16: one fp32 add of the bias, one
// round-to-nearest-even.  int8 -> fp16: fp32(acc) *rn scale [+rn bias], then
// one round to fp16.  int32: the accumulator itself.
template <int OUT, bool kInt8>
__device__ __forceinline__ uint32_t convert_out(uint32_t acc, float badd, float sc, bool has_bias) {
  if constexpr (OUT == OUT_S32) {
    return acc;
  } else if constexpr (kInt8) {
    float v = __fmul_rn(__int2float_rn(static_cast<int>(acc)), sc);
    if (has_bias) v = __fadd_rn(v, badd);
    return __half_as_ushort(__float2half_rn(v));
  } else {
    float v = __fadd_rn(__uint_as_float(acc), badd);
    if constexpr (out_gelu(OUT)) v = gelu_f32(v);
    if constexpr (out_bf16(OUT))
      return __bfloat16_as_ushort(__float2bfloat16_rn(v));
    else
      return __half_as_ushort(__float2half_rn(v));
  }
}

// Two accumulator values of one output column (rows k and k+1) -> one packed
// 32-bit word of two 16-bit outputs (row k in the low half), with the same
// arithmetic as convert_out: fp32 bias add, then one round to nearest even.
template <int OUT, bool kInt8>
__device__ __forceinline__ uint32_t convert_pair16(uint32_t a0, uint32_t a1, float badd, float sc, bool has_bias) {
  float v0, v1;
  if constexpr (kInt8) {
    v0 = __fmul_rn(__int2float_rn(static_cast<int>(a0)), sc);
    v1 = __fmul_rn(__int2float_rn(static_cast<int>(a1)), sc);
    if (has_bias) {
      v0 = __fadd_rn(v0, badd);
      v1 = __fadd_rn(v1, badd);
    }
  } else {
    v0 = __fadd_rn(__uint_as_float(a0), badd);
    v1 = __fadd_rn(__uint_as_float(a1), badd);
    if constexpr (out_gelu(OUT)) {
      v0 = gelu_f32(v0);
      v1 = gelu_f32(v1);
    }
  }
  uint32_t w;
  if constexpr (out_bf16(OUT))
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(v1), "f"(v0));
  else
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(v1), "f"(v0));
  return w;
}

// Stage this warp's half of a [32 rows m][64 columns n] box of 16-bit outputs
// (128 B rows, 128-byte swizzle: 16-byte chunk c of row r sits at chunk
// c ^ (r % 8); the box starts 1024-byte aligned); `half` selects columns
// 32*half .. 32*half+31.  Lane n holds p[j] = (row 2j, row 2j+1) of column n.
// At step j the even lane 2i stores row 2j and the odd lane 2i+1 row
// 2(j^2)+1 of the column pair (2i, 2i+1), each taking the missing half from
// its neighbour; with the swizzle the two halves of the warp always land in
// disjoint bank groups.
__device__ __forceinline__ void stage_pair_box16(uint32_t box_saddr, const uint32_t (&p)[16], int lane, int half) {
  const bool even = (lane & 1) == 0;
  const int i = lane >> 1;
  // unswizzled byte offset of this lane's word within its row
  const uint32_t base = box_saddr + uint32_t(((4 * half + (i >> 2)) << 4) + (i & 3) * 4);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int jo = j ^ 2;
    // the even lane stores row 2j and needs the odd lane's row 2j; the odd
    // lane stores row 2jo+1 and needs the even lane's row 2jo+1
    const uint32_t send = even ? (p[jo] >> 16) : (p[j] & 0xFFFFu);
    const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const uint32_t w = even ? __byte_perm(p[j], recv, 0x5410) : __byte_perm(recv, p[jo], 0x7610);
    const uint32_t re = 2 * j, ro = 2 * jo + 1;
    const uint32_t ae = (base + re * 128) ^ ((re & 7) << 4);
    const uint32_t ao = (base + ro * 128) ^ ((ro & 7) << 4);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(even ? ae : ao), "r"(w) : "memory");
  }
}

// Tile order: the ceil(N/256) x ceil(M/BN) tile grid is walked in bands of
// `band` consecutive weight-row tiles; inside a band the weight tile varies
// fastest, so the pairs in flight share X tiles through L2, and a band's
// compressed weights stay in L2 while every X tile passes by once.  HBM then
// reads W once and X once per band (the host sizes a band's weights to a
// fraction of L2; shapes with one band keep the plain n-fastest order).
__device__ __forceinline__ void tile_coords(int t, int NT, int MT, int band, int& nt, int& mt) {
  const int per_band = band * MT;
  const int b = t / per_band;
  const int r = t - b * per_band;
  const int w = min(band, NT - b * band);
  mt = r / w;
  nt = b * band + (r - mt * w);
}

// Cluster pairs: pair p = blockIdx.x / 2 computes tiles p, p + gridDim.x/2, ...
// in the order of tile_coords.  CTA rank r of the pair loads weight rows
// [n0 + 128r, +128) and X rows [m0 + r*BN/2, +BN/2); the leader (rank 0)
// issues the 256 x BN MMAs, which read both CTAs' shared memory and write
// each CTA's own tensor memory (its 128 weight rows x BN).
template <bool kInt8, bool kBF16, int BN, int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    spgemm24_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                    void* __restrict__ Yp, int64_t ldy, const void* __restrict__ bias,
                    const float* __restrict__ scale, float qscale, int M, int N, int K, int band,
                    const uint8_t* __restrict__ meta_g, int meta_direct, uint32_t* err) {
  using C = Cfg<kInt8, BN, OUT>;
  constexpr int STAGES = C::STAGES;
  constexpr int BNH = C::BNH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* mtma = full + STAGES;
  uint64_t* empty = mtma + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = (K + C::KSTEP - 1) / C::KSTEP;
  // MMAs of the last stage: 4, or 2 when K ends half-way through a stage
  const int last_mmas = (K % C::KSTEP) ? 2 : 4;
  const int NT = (N + 255) / 256;
  const int MT = (M + BN - 1) / BN;
  const int total = NT * MT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // operand bytes of both CTAs plus, for fp16/bf16, one arrival from each
      // CTA's metadata warp once the stage's metadata is arranged
      mbar_init(&full[s], kInt8 ? 1 : 3);
      mbar_init(&mtma[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * C::EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmE);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_launch_dependents();
  griddep_wait();  // the previous kernel's writes (X, or readers of Y) are complete
  // the leader's barriers as seen from either CTA of the pair
  const uint32_t full_l = mapa_shared(smem_addr(full), 0);
  const uint32_t acc_empty_l = mapa_shared(smem_addr(acc_empty), 0);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int t = pair; ok && t < total; t += npairs) {
        int nt, mt;
        tile_coords(t, NT, MT, band, nt, mt);
        const int n0 = nt * 256 + 128 * int(rank);
        const int m0 = mt * BN + BNH * int(rank);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % STAGES;
          const uint32_t use = g / STAGES;
          if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, abort_flag, err, ERR_WAIT_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* a_s = smem + C::OFF_A + s * C::A_BYTES;
          uint8_t* b_s = smem + C::OFF_B + s * C::B_BYTES;
          uint8_t* e_s = smem + C::OFF_MSTG + s * C::MSTG_BYTES;
          const uint32_t fb = full_l + 8u * s;
          if (leader) mbar_arrive_expect_tx(&full[s], C::TX_PAIR);
          tma_load_2d_pair(a_s, &tmA, kb * (C::KSTEP / 2), n0, fb);
          tma_load_2d_pair(b_s, &tmB, kb * C::KSTEP, m0, fb);
          tma_load_2d_pair(b_s + BNH * 128, &tmB, kb * C::KSTEP + C::KSTEP / 2, m0, fb);
          if constexpr (kInt8) {
            tma_load_2d_pair(e_s, &tmE, kb * 32, n0, fb);
            tma_load_2d_pair(e_s + 2048, &tmE, kb * 32 + 16, n0, fb);
          } else if (!meta_direct) {
            mbar_arrive_expect_tx(&mtma[s], C::MSTG_BYTES);
            tma_load_2d(e_s, &tmE, kb * 16, n0, &mtma[s]);
          }
        }
      }
      // Let every issued copy land before shared memory can be released: the
      // leader's full barriers count both CTAs' operand bytes, the local
      // metadata barriers this CTA's metadata.
      for (uint32_t q = (g > uint32_t(STAGES) ? g - STAGES : 0u); q < g; ++q) {
        if (leader) tail_wait(&full[q % STAGES], (q / STAGES) & 1, err);
        if constexpr (!kInt8)
          if (!meta_direct) tail_wait(&mtma[q % STAGES], (q / STAGES) & 1, err);
      }
    }
  } else if (warp == 1) {
    // ------------- metadata arrangement (fp16/bf16, both CTAs) -------------
    if constexpr (!kInt8) {
      uint32_t g = 0;
      bool ok = true;
      const int64_t mpitch = K / 8;
      for (int t = pair; ok && t < total; t += npairs) {
        int nt, mt;
        tile_coords(t, NT, MT, band, nt, mt);
        const int n0 = nt * 256 + 128 * int(rank);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % STAGES;
          if (meta_direct) {
            // the stage's previous MMAs (and their tcgen05.cp of this slot) are done
            const uint32_t use = g / STAGES;
            if (use > 0 && !mbar_wait_warp(&empty[s], (use - 1) & 1, abort_flag, err, ERR_WAIT_META)) {
              ok = false;
              break;
            }
            const int col0 = kb * 16;
            permute_meta_f16_direct(meta_g, mpitch, n0, N, col0, int(mpitch) - col0 >= 16 ? 16 : 8,
                                    smem + C::OFF_MCP + s * C::MCP_BYTES, lane);
          } else {
            if (!mbar_wait_warp(&mtma[s], (g / STAGES) & 1, abort_flag, err, ERR_WAIT_META)) {
              ok = false;
              break;
            }
            permute_meta_f16(smem + C::OFF_MSTG + s * C::MSTG_BYTES, smem + C::OFF_MCP + s * C::MCP_BYTES, lane);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(full_l + 8u * s);
        }
      }
    }
  } else if (warp == 2) {
    // ---------------- MMA issuer (leader CTA) ----------------
    // One thread runs the whole loop: the waits are single-thread bounded
    // waits, because a warp-wide wait and vote between two groups of MMAs
    // costs more than its share of the tensor pipe's time.
    if (leader && lane == 0) {
      constexpr uint32_t kFmt = kInt8 ? 1u : (kBF16 ? 1u : 0u);
      constexpr uint32_t kCFmt = kInt8 ? 2u : 1u;
      // Shared-memory descriptors of stage 0.  The start address sits in the
      // low 14 bits as address / 16 and every operand stays below 256 KB, so
      // the descriptor of a stage (and of a K step inside it) is the stage-0
      // descriptor plus its byte offset / 16: nothing is rebuilt per stage.
      const uint64_t a_desc0 = smem_desc(smem_addr(smem + C::OFF_A), 16, 1024, LAYOUT_SW128);
      const uint64_t b_desc0 = smem_desc(smem_addr(smem + C::OFF_B), 16, 1024, LAYOUT_SW128);
      const uint64_t e_desc0 =
          smem_desc(smem_addr(smem + (kInt8 ? C::OFF_MSTG : C::OFF_MCP)), 2048, 128, LAYOUT_NONE);
      constexpr uint64_t kAStep = C::A_BYTES >> 4, kBStep = C::B_BYTES >> 4;
      constexpr uint64_t kEStep = (kInt8 ? C::MSTG_BYTES : C::MCP_BYTES) >> 4;
      uint32_t g = 0;
      int s = 0;
      uint32_t ph = 0;
      int i = 0;
      bool ok = true;
      for (int t = pair; ok && t < total; t += npairs, ++i) {
        const int b = i & 1;
        if (i >= 2 && !mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1, abort_flag, err, ERR_WAIT_ACC_FREE)) break;
        tc_fence_after();
        const uint32_t acc = tmem + uint32_t(b * BN);
        // Stages are issued in groups of kIssueGroup: every barrier of the
        // group is waited first, then the group's MMAs follow back to back.
        for (int kb = 0; kb < KB; kb += kIssueGroup) {
          const int nr = KB - kb < kIssueGroup ? KB - kb : kIssueGroup;
          int s2 = s;
          uint32_t ph2 = ph;
          for (int r = 0; r < nr; ++r) {
            if (!mbar_wait(&full[s2], ph2, abort_flag, err, ERR_WAIT_FULL)) {
              ok = false;
              break;
            }
            if (++s2 == STAGES) {
              s2 = 0;
              ph2 ^= 1u;
            }
          }
          if (!ok) break;
          tc_fence_after();
          for (int r = 0; r < nr; ++r, ++g) {
            const uint64_t ad = a_desc0 + uint64_t(s) * kAStep;
            const uint64_t bd = b_desc0 + uint64_t(s) * kBStep;
            const uint64_t ed = e_desc0 + uint64_t(s) * kEStep;
            const uint32_t ecol = tmem + C::META_COL + (g & 1) * C::MCOLS;
            tc_cp_128x128b_pair(ecol, ed);
            if constexpr (kInt8) tc_cp_128x128b_pair(ecol + 4, ed + (2048 >> 4));
            const int nmma = kb + r + 1 == KB ? last_mmas : 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (j >= nmma) break;
              const uint64_t adesc = ad + uint64_t((32 * j) >> 4);
              const uint64_t bdesc = bd + uint64_t(((j >> 1) * (BNH * 128) + (j & 1) * 64) >> 4);
              const uint32_t e = kInt8 ? ecol + 2 * j : ecol + (j & ~1);
              const uint32_t sel = kInt8 ? 0u : uint32_t(j & 1);
              tc_mma_sp_pair<kInt8>(acc, adesc, bdesc, e, instr_desc(kFmt, kCFmt, 256, BN, true, sel),
                                    ((kb + r) | j) != 0 ? 1u : 0u);
            }
            tc_commit_pair(&empty[s], 0x3);
            if (++s == STAGES) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[b], 0x3);
      }
      tc_commit_pair(mma_done, 0x3);
    }
    __syncwarp();
    // both CTAs: every MMA reading this CTA's shared memory or writing its
    // tensor memory has completed once the leader's final commit arrives
    if (lane == 0) tail_wait(mma_done, 0, err);
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- epilogue (both CTAs) ----------------
    // Warp w reads tensor-memory lanes 32*(w%4).. (its quadrant) and every
    // second 32-column chunk of the accumulator, starting at chunk (w-4)/4.
    constexpr int kStride = C::EPI_WARPS / 4;
    const int q = warp & 3;
    const int sub = (warp - 4) >> 2;
    uint8_t* buf = smem + C::OFF_EPI + (warp - 4) * C::EPI_BUF;
    // 16-bit outputs: warps (sub, 2p) and (sub, 2p+1) share two 4 KB pair boxes
    const int pair_idx = (warp - 4) >> 1;
    const uint32_t pbox0 = smem_addr(smem + C::OFF_EPI + pair_idx * 2 * C::EPI_BUF);
    const uint32_t pair_bar = 1 + pair_idx;
    const bool pair_lead = (q & 1) == 0;
    bool staged = false;  // int32: a TMA store from buf may still be reading it
    uint32_t nst = 0;     // 16-bit: pair boxes stored so far
    uint32_t nyt = 0;     // Y^T: boxes this warp stored so far
    int i = 0;
    for (int t = pair; t < total; t += npairs, ++i) {
      int nt, mt;
      tile_coords(t, NT, MT, band, nt, mt);
      const int n0 = nt * 256 + 128 * int(rank), m0 = mt * BN;
      const int b = i & 1;
      // the two warps of a pair take the same branch: they meet at the pair barrier below
      const bool got = mbar_wait_warp(&acc_full[b], (i >> 1) & 1, abort_flag, err, ERR_WAIT_ACC);
      if (!named_bar_all(pair_bar, 64, got)) break;
      tc_fence_after();
      const int nb = n0 + 32 * q;
      const int n = nb + lane;
      float badd = 0.f, sc = 0.f;
      bool has_bias = false;
      if (n < N) {
        if constexpr (OUT == OUT_S32) {
        } else if constexpr (kInt8) {
          sc = scale[n];
          if (bias) {
            badd = __half2float(static_cast<const __half*>(bias)[n]);
            has_bias = true;
          }
        } else if constexpr (kBF16) {
          if (bias) badd = __bfloat162float(static_cast<const __nv_bfloat16*>(bias)[n]);
        } else {
          if (bias) badd = __half2float(static_cast<const __half*>(bias)[n]);
        }
      }
      const bool full_n = nb + 32 <= N;
      const bool pair_full = n0 + 64 * (q >> 1) + 64 <= N;
      const uint32_t tbase = tmem + (uint32_t(32 * q) << 16) + uint32_t(b * BN);
      constexpr bool kPaired = C::OUT_ES == 2 && !C::YT;
      if (kPaired && pair_full && sub < C::NCH) {
        // 16-bit Y (with or without GELU), whole pair box: two chunks per
        // round, so one pair of barriers, one proxy fence and one store issue
        // serve both
#pragma unroll 1
        for (int c = sub; c < C::NCH; c += 2 * kStride) {
          const int c2 = c + kStride;
          const bool two = c2 < C::NCH;
          uint32_t h[32], h2[32];
          tmem_ld_32x32b_x32(tbase + 32 * c, h);
          if (two) tmem_ld_32x32b_x32(tbase + 32 * c2, h2);
          tmem_ld_wait(h);
          if (two) tmem_ld_wait(h2);
          if ((two ? c2 : c) + kStride >= C::NCH) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_l + 8u * b);
          }
          const int mb = m0 + 32 * c, mb2 = m0 + 32 * c2;
          if (mb >= M) continue;
          const bool do2 = two && mb2 < M;
#pragma unroll
          for (int j = 0; j < 16; ++j) h[j] = convert_pair16<OUT, kInt8>(h[2 * j], h[2 * j + 1], badd, sc, has_bias);
          if (do2) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              h2[j] = convert_pair16<OUT, kInt8>(h2[2 * j], h2[2 * j + 1], badd, sc, has_bias);
          }
          const uint32_t boxa = pbox0 + (nst & 1) * 4096, boxb = pbox0 + ((nst + 1) & 1) * 4096;
          if (nst >= 1) {
            if (pair_lead && lane == 0) bulk_wait_read<0>();
            named_bar_sync(pair_bar, 64);
          }
          stage_pair_box16(boxa, reinterpret_cast<const uint32_t(&)[16]>(h), lane, q & 1);
          if (do2) stage_pair_box16(boxb, reinterpret_cast<const uint32_t(&)[16]>(h2), lane, q & 1);
          fence_proxy_async_smem();
          named_bar_sync(pair_bar, 64);
          if (pair_lead && lane == 0) {
            // one bulk group per box, so a single-chunk round that follows
            // (bulk_wait_read<1>) sees the box it reuses finished
            tma_store_2d_saddr(&tmY, boxa, n0 + 64 * (q >> 1), mb);
            bulk_commit();
            if (do2) {
              tma_store_2d_saddr(&tmY, boxb, n0 + 64 * (q >> 1), mb2);
              bulk_commit();
            }
          }
          __syncwarp();
          nst += do2 ? 2 : 1;
        }
      } else
#pragma unroll 1
      for (int c = sub; c < C::NCH; c += kStride) {
        uint32_t h[32];
        tmem_ld_32x32b_x32(tbase + 32 * c, h);
        tmem_ld_wait(h);
        if (c + kStride >= C::NCH) {
          // last chunk of this warp is read: hand the accumulator back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty_l + 8u * b);
        }
        const int mb = m0 + 32 * c;
        if (nb >= N || mb >= M) continue;
        if constexpr (C::OUT_ES == 1) {
          // int8 out: v = fp32(acc) *rn scale (+rn bias) [GELU], q = clamp(rne(v *rn qscale)),
          // staged as [32 rows m][32 bytes n] in this warp's buffer; lane r stores row r
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            float v = __fmul_rn(__int2float_rn(static_cast<int>(h[k])), sc);
            if (has_bias) v = __fadd_rn(v, badd);
            if constexpr (out_gelu(OUT)) v = gelu_as_f32(v);
            const int qv = max(-127, min(127, __float2int_rn(__fmul_rn(v, qscale))));
            buf[k * 32 + lane] = static_cast<uint8_t>(qv & 0xFF);
          }
          __syncwarp();
          const int row = mb + lane;
          if (row < M) {
            uint8_t* yrow = static_cast<uint8_t*>(Yp) + int64_t(row) * ldy + nb;
            const uint8_t* srow = buf + lane * 32;
            if (full_n) {
              reinterpret_cast<uint4*>(yrow)[0] = reinterpret_cast<const uint4*>(srow)[0];
              reinterpret_cast<uint4*>(yrow)[1] = reinterpret_cast<const uint4*>(srow)[1];
            } else {
              for (int e = 0; e < N - nb; ++e) yrow[e] = srow[e];
            }
          }
          __syncwarp();
          continue;
        }
        if constexpr (C::OUT_ES == 4) {
#pragma unroll
          for (int k = 0; k < 32; ++k) h[k] = convert_out<OUT, kInt8>(h[k], badd, sc, has_bias);
        } else {
          // packed pairs (rows 2j, 2j+1) kept in h[0..15]
#pragma unroll
          for (int j = 0; j < 16; ++j) h[j] = convert_pair16<OUT, kInt8>(h[2 * j], h[2 * j + 1], badd, sc, has_bias);
        }
        if constexpr (C::YT) {
          // Y^T [N][M]: lane n holds rows mb..mb+31 of output column n, i.e.
          // 64 contiguous bytes of row n of Y^T.  The warp's [32 n][32 m]
          // block goes to a double-buffered 2 KB box (64-byte swizzle: 16-byte
          // chunk k of row r at chunk k ^ ((r >> 1) & 3)) and out by one TMA
          // store, which clips rows >= N.  A chunk that crosses M (the
          // inner dimension, where the store would not stop at the exact
          // element) is written by element stores instead.
          if (mb + 32 > M) {
            if (n < N) {
              uint16_t* dst = static_cast<uint16_t*>(Yp) + int64_t(n) * ldy + mb;
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (mb + k < M) dst[k] = static_cast<uint16_t>((k & 1) ? (h[k >> 1] >> 16) : (h[k >> 1] & 0xFFFFu));
            }
            continue;
          }
          const uint32_t box = smem_addr(buf) + (nyt & 1) * 2048u;
          if (nyt >= 2) {
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t a = box + uint32_t(lane) * 64u + (uint32_t(k ^ ((lane >> 1) & 3)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(h[4 * k]), "r"(h[4 * k + 1]),
                         "r"(h[4 * k + 2]), "r"(h[4 * k + 3])
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d_saddr(&tmY, box, mb, nb);
            bulk_commit();
          }
          __syncwarp();
          ++nyt;
          continue;
        }
        if (C::OUT_ES == 4 && full_n) {
          // int32: one [32][32] box (128 B rows) per warp
          if (staged) {
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
          }
#pragma unroll
          for (int k = 0; k < 32; ++k) reinterpret_cast<uint32_t*>(buf)[k * 32 + lane] = h[k];
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, buf, nb, mb);
            bulk_commit();
          }
          __syncwarp();
          staged = true;
        } else if (C::OUT_ES == 2 && pair_full) {
          // 16-bit: the warps of quadrants 2p, 2p+1 fill one [32][64] box (128 B
          // rows) of a double-buffered pair; the lead warp stores it
          const uint32_t box = pbox0 + (nst & 1) * 4096;
          if (nst >= 2) {
            if (pair_lead && lane == 0) bulk_wait_read<1>();
            named_bar_sync(pair_bar, 64);
          }
          stage_pair_box16(box, reinterpret_cast<const uint32_t(&)[16]>(h), lane, q & 1);
          fence_proxy_async_smem();
          named_bar_sync(pair_bar, 64);
          if (pair_lead && lane == 0) {
            tma_store_2d_saddr(&tmY, box, n0 + 64 * (q >> 1), mb);
            bulk_commit();
          }
          __syncwarp();
          ++nst;
        } else if (n < N) {
          // ragged right edge: bounds-checked direct stores
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            if (mb + k >= M) continue;
            if constexpr (C::OUT_ES == 4)
              static_cast<uint32_t*>(Yp)[int64_t(mb + k) * ldy + n] = h[k];
            else
              static_cast<uint16_t*>(Yp)[int64_t(mb + k) * ldy + n] =
                  static_cast<uint16_t>((k & 1) ? (h[k >> 1] >> 16) : (h[k >> 1] & 0xFFFFu));
          }
        }
      }
      if (sub >= C::NCH) {  // narrow tiles: this warp has no chunk, only hands the accumulator back
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_l + 8u * b);
      }
    }
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // neither CTA leaves while its peer may still signal or read it
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// Cluster pairs of `kern` that fit on the device at once (cached per kernel and
// device; the cache is shared by every host thread, under a lock).
int resident_pairs(const void* kern, int smem, int threads) {
  struct Entry { const void* k; int dev; int n; };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].k == kern && cache[i].dev == dev) return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  if (used < 64) cache[used++] = Entry{kern, dev, n};
  return n;
}

template <bool kInt8, bool kBF16, int BN, int OUT>
spg_status launch(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                  const float* scale, void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t stream,
                  float qscale) {
  using C = Cfg<kInt8, BN, OUT>;
  const int es = kInt8 ? 1 : 2;
  // metadata rows of K/8 bytes: a TMA map needs a pitch that is a multiple of
  // 16 bytes (K % 128 == 0); otherwise the metadata warp reads them directly
  // (fp16/bf16 only: int8 K is a multiple of 128)
  const int meta_direct = (K / 8) % 16 != 0 ? 1 : 0;
  CUtensorMap tmA, tmB, tmE, tmY;
  if (!make_tmap_2d(&tmA, Wv, es, uint64_t(K / 2), uint64_t(N), uint64_t(K / 2) * es, 128 / es, 128, true) ||
      !make_tmap_2d(&tmB, X, es, uint64_t(K), uint64_t(M), uint64_t(ldx) * es, 128 / es, C::BNH, true))
    return SPG_ERR_CUDA;
  if (meta_direct)
    std::memset(&tmE, 0, sizeof(tmE));
  else if (!make_tmap_2d(&tmE, meta, 1, uint64_t(K / 8), uint64_t(N), uint64_t(K / 8), 16, 128, false))
    return SPG_ERR_CUDA;
  if (kInt8 && meta_direct) return SPG_ERR_UNSUPPORTED_SHAPE;
  // the output map: Y^T boxes [32 n][32 m] with 64-byte swizzle, Y boxes of 64
  // (16-bit) or 32 (32-bit) columns x 32 rows; int8 outputs are stored without TMA
  bool ymap_ok = true;
  if constexpr (C::OUT_ES == 1)
    std::memset(&tmY, 0, sizeof(tmY));
  else if constexpr (C::YT)
    ymap_ok = make_tmap_2d_swz(&tmY, Y, 2, uint64_t(M), uint64_t(N), uint64_t(ldy) * 2, 32, 32, 64);
  else
    ymap_ok = make_tmap_2d(&tmY, Y, C::OUT_ES, uint64_t(N), uint64_t(M), uint64_t(ldy) * C::OUT_ES,
                           C::OUT_ES == 2 ? 64 : 32, 32, C::OUT_ES == 2);
  if (!ymap_ok) return SPG_ERR_CUDA;
  uint32_t* err = device_error_word();
  if (!err) return SPG_ERR_CUDA;
  auto kern = spgemm24_kernel<kInt8, kBF16, BN, OUT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return SPG_ERR_CUDA;
  const int64_t tiles = ((N + 255) / 256) * ((M + BN - 1) / BN);
  const int64_t pairs_max = resident_pairs(reinterpret_cast<const void*>(kern), C::SMEM, C::THREADS);
  if (pairs_max <= 0) return SPG_ERR_CUDA;
  const int pairs = static_cast<int>(tiles < pairs_max ? tiles : pairs_max);
  // weight-row tiles per band: their compressed values and metadata take at
  // most kBandBytes, a fifth of the 126 MB L2 (prefill-sized weights split into
  // bands; the ViT-sized layers fit in one)
  constexpr int64_t kBandBytes = int64_t(24) << 20;
  const int64_t tile_w_bytes = 256 * (K / 2 * es + K / 8);
  const int64_t nt_all = (N + 255) / 256;
  int64_t band = kBandBytes / tile_w_bytes;
  band = band < 1 ? 1 : band > nt_all ? nt_all : band;
  const int64_t nbands = (nt_all + band - 1) / band;
  band = (nt_all + nbands - 1) / nbands;  // equal bands (64 tiles: 4 x 16, not 3 x 21 + 1)
  if (launch_pdl(kern, dim3(2 * pairs), dim3(C::THREADS), C::SMEM, stream, tmA, tmB, tmE, tmY, Y, ldy, bias, scale,
                 qscale, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(band),
                 meta, meta_direct, err) != cudaSuccess)
    return SPG_ERR_CUDA;
  return launch_status();
}

// Estimated cost of a launch with X-tile width bn: the rounds of pair tiles the
// busiest pair runs, each costing its width plus a fixed per-tile share (the
// epilogue's latency and the pipeline's fill), in units of X rows.  The share
// of 160 matches the ViT-Base MLP measurements: 224 is faster for
// 12608 x 3072 x 768 (39.8 against 41.5 us with 192), 192 for
// 12608 x 768 x 3072 (38.2 against 38.9 us), where 224 leaves the last round
// a third full.
int64_t tile_cost(int64_t M, int64_t N, int bn) {
  const int64_t tiles = ((N + 255) / 256) * ((M + bn - 1) / bn);
  const int64_t pairs = sm_count() / 2;
  const int64_t rounds = (tiles + pairs - 1) / pairs;
  return rounds * (bn + 160);
}

// X rows per pair tile: small batches take narrow tiles, large ones the wider
// of 224 (the widest whose two accumulators and metadata ring fit in tensor
// memory) and 192 by the estimated cost.
template <bool kInt8, bool kBF16, int OUT>
spg_status dispatch(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                    const float* scale, void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                    float qscale = 0.f) {
  if (M <= 32) return launch<kInt8, kBF16, 32, OUT>(X, ldx, Wv, meta, bias, scale, Y, ldy, M, N, K, s, qscale);
  if (M <= 128) return launch<kInt8, kBF16, 128, OUT>(X, ldx, Wv, meta, bias, scale, Y, ldy, M, N, K, s, qscale);
  if (tile_cost(M, N, 192) < tile_cost(M, N, 224))
    return launch<kInt8, kBF16, 192, OUT>(X, ldx, Wv, meta, bias, scale, Y, ldy, M, N, K, s, qscale);
  return launch<kInt8, kBF16, 224, OUT>(X, ldx, Wv, meta, bias, scale, Y, ldy, M, N, K, s, qscale);
}

spg_status validate_common(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, void* Y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, int es, int out_es, int kstep, bool y_transposed = false) {
  // M == 0 (an empty batch) is valid: the caller returns SPG_OK without a launch, and X / Y may be NULL
  if (!Wv || !meta || (M != 0 && (!X || !Y))) return SPG_ERR_INVALID_ARG;
  if (M < 0 || N <= 0 || K <= 0 || ldx < K || ldy < (y_transposed ? M : N)) return SPG_ERR_INVALID_ARG;
  if (K % kstep || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return SPG_ERR_UNSUPPORTED_SHAPE;
  if ((N + 127) / 128 * ((M + 31) / 32) >= (int64_t(1) << 31)) return SPG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SPG_OK;  // nothing is read or written: pointers and pitches need no alignment
  if (!aligned(X, 16) || !aligned(Wv, 16) || !aligned(meta, 16) || !aligned(Y, 16)) return SPG_ERR_MISALIGNED;
  if ((ldx * es) % 16 || (ldy * out_es) % 16) return SPG_ERR_MISALIGNED;
  return SPG_OK;
}

}  // namespace gemm24
}  // namespace spg

extern "C" {

spg_status spgemm_24_f16(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                         void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, spg_dtype dtype,
                         spg_stream_t stream) {
  using namespace spg;
  using namespace spg::gemm24;
  if (dtype != SPG_F16 && dtype != SPG_BF16) return SPG_ERR_INVALID_ARG;
  spg_status st = validate_common(X, ldx, Wv, meta, Y, ldy, M, N, K, 2, 2, 64);
  if (st != SPG_OK) return st;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  if (M == 0) return SPG_OK;  // empty batch: nothing to compute
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SPG_F16) return dispatch<false, false, OUT_F16>(X, ldx, Wv, meta, bias, nullptr, Y, ldy, M, N, K, s);
  return dispatch<false, true, OUT_BF16>(X, ldx, Wv, meta, bias, nullptr, Y, ldy, M, N, K, s);
}

// The same layer from and to host memory: X copied in, the GEMM, Y copied out,
// all on `stream`, through caller-provided device buffers.
spg_status spgemm_24_f16_host(const void* X_host, int64_t ldx_host, const void* Wv, const uint8_t* meta,
                              const void* bias, void* Y_host, int64_t ldy_host, int64_t M, int64_t N, int64_t K,
                              spg_dtype dtype, void* X_dev, void* Y_dev, int64_t ldy_dev, spg_stream_t stream) {
  using namespace spg;
  if (M < 0 || N <= 0 || K <= 0 || ldx_host < K || ldy_host < N) return SPG_ERR_INVALID_ARG;
  if (M != 0 && (!X_host || !Y_host)) return SPG_ERR_INVALID_ARG;
  // the device layer's own checks (X_dev with pitch K, Y_dev with pitch ldy_dev)
  spg_status st = gemm24::validate_common(X_dev, K, Wv, meta, Y_dev, ldy_dev, M, N, K, 2, 2, 64);
  if (st != SPG_OK) return st;
  if (dtype != SPG_F16 && dtype != SPG_BF16) return SPG_ERR_INVALID_ARG;
  if (M == 0) return SPG_OK;
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpy2DAsync(X_dev, size_t(K) * 2, X_host, size_t(ldx_host) * 2, size_t(K) * 2, size_t(M),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
    return SPG_ERR_CUDA;
  st = spgemm_24_f16(X_dev, K, Wv, meta, bias, Y_dev, ldy_dev, M, N, K, dtype, stream);
  if (st != SPG_OK) return st;
  if (cudaMemcpy2DAsync(Y_host, size_t(ldy_host) * 2, Y_dev, size_t(ldy_dev) * 2, size_t(N) * 2, size_t(M),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SPG_ERR_CUDA;
  return SPG_OK;
}

spg_status spgemm_24_f16_gelu(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                              void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, spg_dtype dtype,
                              spg_stream_t stream) {
  using namespace spg;
  using namespace spg::gemm24;
  if (dtype != SPG_F16 && dtype != SPG_BF16) return SPG_ERR_INVALID_ARG;
  spg_status st = validate_common(X, ldx, Wv, meta, Y, ldy, M, N, K, 2, 2, 64);
  if (st != SPG_OK) return st;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  if (M == 0) return SPG_OK;  // empty batch: nothing to compute
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SPG_F16)
    return dispatch<false, false, OUT_F16_G>(X, ldx, Wv, meta, bias, nullptr, Y, ldy, M, N, K, s);
  return dispatch<false, true, OUT_BF16_G>(X, ldx, Wv, meta, bias, nullptr, Y, ldy, M, N, K, s);
}

spg_status spgemm_24_f16_yt(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                            void* Yt, int64_t ldyt, int64_t M, int64_t N, int64_t K, spg_dtype dtype,
                            spg_stream_t stream) {
  using namespace spg;
  using namespace spg::gemm24;
  if (dtype != SPG_F16 && dtype != SPG_BF16) return SPG_ERR_INVALID_ARG;
  spg_status st = validate_common(X, ldx, Wv, meta, Yt, ldyt, M, N, K, 2, 2, 64, true);
  if (st != SPG_OK) return st;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  if (M == 0) return SPG_OK;  // empty batch: nothing to compute
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SPG_F16)
    return dispatch<false, false, OUT_F16_T>(X, ldx, Wv, meta, bias, nullptr, Yt, ldyt, M, N, K, s);
  return dispatch<false, true, OUT_BF16_T>(X, ldx, Wv, meta, bias, nullptr, Yt, ldyt, M, N, K, s);
}

spg_status spgemm_24_s8(const int8_t* X, int64_t ldx, const int8_t* Wv, const uint8_t* meta, const float* scale,
                        const void* bias, void* Y, int64_t ldy, int out_mode, int64_t M, int64_t N, int64_t K,
                        spg_stream_t stream) {
  using namespace spg;
  using namespace spg::gemm24;
  if (out_mode != SPG_OUT_F16 && out_mode != SPG_OUT_S32) return SPG_ERR_INVALID_ARG;
  const int out_es = out_mode == SPG_OUT_S32 ? 4 : 2;
  spg_status st = validate_common(X, ldx, Wv, meta, Y, ldy, M, N, K, 1, out_es, 128);
  if (st != SPG_OK) return st;
  if (out_mode == SPG_OUT_F16 && !scale) return SPG_ERR_INVALID_ARG;
  if (scale && !aligned(scale, 4)) return SPG_ERR_MISALIGNED;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  if (M == 0) return SPG_OK;  // empty batch: nothing to compute
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (out_mode == SPG_OUT_S32)
    return dispatch<true, false, OUT_S32>(X, ldx, Wv, meta, nullptr, nullptr, Y, ldy, M, N, K, s);
  return dispatch<true, false, OUT_F16>(X, ldx, Wv, meta, bias, scale, Y, ldy, M, N, K, s);
}

// int8 2:4 layer whose epilogue quantises its output for the next int8 layer
// (optionally through GELU): the fixed-point path of the compressed ViT MLP.
spg_status spgemm_24_s8_q(const int8_t* X, int64_t ldx, const int8_t* Wv, const uint8_t* meta, const float* scale,
                          const void* bias, float qscale, int act, int8_t* Yq, int64_t ldy, int64_t M, int64_t N,
                          int64_t K, spg_stream_t stream) {
  using namespace spg;
  using namespace spg::gemm24;
  if (act != SPG_ACT_NONE && act != SPG_ACT_GELU) return SPG_ERR_INVALID_ARG;
  if (!scale || !(qscale > 0.f) || !(qscale < 3.0e38f)) return SPG_ERR_INVALID_ARG;
  spg_status st = validate_common(X, ldx, Wv, meta, Yq, ldy, M, N, K, 1, 1, 128);
  if (st != SPG_OK) return st;
  if (!aligned(scale, 4)) return SPG_ERR_MISALIGNED;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  if (M == 0) return SPG_OK;  // empty batch: nothing to compute
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (act == SPG_ACT_GELU)
    return dispatch<true, false, OUT_S8QG>(X, ldx, Wv, meta, bias, scale, Yq, ldy, M, N, K, s, qscale);
  return dispatch<true, false, OUT_S8Q>(X, ldx, Wv, meta, bias, scale, Yq, ldy, M, N, K, s, qscale);
}

}  // extern "C"
