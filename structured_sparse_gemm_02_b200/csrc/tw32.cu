// Tile-wise sparsity on the CUDA cores in fp32 ("Accelerating Sparse DNN Models
// without Hardware-Support via Tile-Wise Sparsity", Guo et al.: the library
// table lists a tile-wise CUDA-fp32 library next to the tensor-core fp16 one,
// and the results slide reports the tile-wise speedup on CUDA cores).
//
// The pattern (offsetn, tile spans, per-tile offsetk) is the descriptor that
// tw_reorganize selects; tw_condense_f32 gathers an fp32 weight through it,
// and spgemm_tw_f32 is the run-time GEMM of the "Run-time" slide on the fp32
// pipes: kept rows of A = X gathered through offsetk, the condensed tile read
// densely, C = Y scattered through offsetn.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "host.cuh"
#include "spgemm.h"

namespace spg {
namespace tw32 {

constexpr int kG = 128;      // tile width (kept columns per tile)
constexpr int kKBlock = 64;  // K padding of the descriptor
constexpr int BM = 128;      // X rows per work unit
constexpr int KS = 32;       // kept rows per shared-memory step
constexpr int THREADS = 256;

// Condensed fp32 values, block b of tile t: Wc[blk][j][c] = W[offsetn[tG+j]][offsetk[kofs+64b+c]]
// for j < G_t and 64b + c < k_t, +0 elsewhere (the layout of the descriptor's fp16 Wc).
__global__ void condense_f32_kernel(const float* __restrict__ W, int64_t ldw, int Nk,
                                    const int* __restrict__ offsetn, const int* __restrict__ tile_kofs,
                                    const int* __restrict__ k_per_tile, const int* __restrict__ offsetk,
                                    float* __restrict__ Wc) {
  const int t = blockIdx.x, b = blockIdx.y;
  const int kofs = tile_kofs[t];
  if (b * kKBlock >= tile_kofs[t + 1] - kofs) return;
  const int j0 = t * kG;
  const int Gt = min(kG, Nk - j0);
  const int kt = k_per_tile[t];
  float* out = Wc + (int64_t(kofs / kKBlock + b) * kG) * kKBlock;
  for (int e = threadIdx.x; e < kG * kKBlock; e += blockDim.x) {
    const int j = e / kKBlock, c = e % kKBlock;
    const int i = b * kKBlock + c;
    out[e] = (j < Gt && i < kt) ? W[int64_t(offsetn[j0 + j]) * ldw + offsetk[kofs + i]] : 0.0f;
  }
}

// X [M, K] -> Xt [K, M] in fp32, 32 x 32 tiles through padded shared memory.
__global__ void transpose_f32_kernel(const float* __restrict__ X, int64_t ldx, int M, int K, float* __restrict__ Xt,
                                     int64_t ldt) {
  __shared__ float tile[32][33];
  const int m0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = m0 + ty + 8 * r, k = k0 + tx;
    if (m < M && k < K) tile[ty + 8 * r][tx] = X[int64_t(m) * ldx + k];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int k = k0 + ty + 8 * r, m = m0 + tx;
    if (k < K && m < M) Xt[int64_t(k) * ldt + m] = tile[tx][ty + 8 * r];
  }
}

// One block per unit (tile t, rows [m0, m0 + 128)).  Thread (tj, tm),
// tj = tid % 16, tm = tid / 16, accumulates the 8 kept columns j = tj + 16 r
// and the 8 rows m0 + 8 tm + s in fp32 (fused multiply-add, each tile's kept
// rows in ascending order): 64 multiply-adds per 16 shared-memory loads.
// Each step stages 32 kept rows: As[k][j] from the condensed tile and
// Bs[k][m] gathered from Xt through offsetk; the next step's values are
// loaded into registers while the current step computes.  The epilogue
// writes Y[m][offsetn[tG+j]] (16 consecutive kept columns per half-warp
// store) and +0 in the pruned columns a kept column owns (the gap after it;
// for the tile's first column also the part of the span before it).
__global__ void __launch_bounds__(THREADS) tw_gemm_f32_kernel(
    const float* __restrict__ xt, int64_t ldt, const float* __restrict__ Wc, float* __restrict__ Y, int64_t ldy,
    int M, int Nk, const int* __restrict__ offsetn, const int* __restrict__ tile_n0,
    const int* __restrict__ tile_kofs, const int* __restrict__ k_per_tile, const int* __restrict__ offsetk) {
  __shared__ float As[KS][kG + 1];  // +1: the transposed fill and the reads are free of bank conflicts
  __shared__ __align__(16) float Bs[KS][BM];
  const int t = blockIdx.x, m0 = blockIdx.y * BM;
  const int tid = threadIdx.x, tj = tid & 15, tm = tid >> 4;
  const int kofs = tile_kofs[t];
  const int kt = k_per_tile[t];
  const int j0 = t * kG;
  const int Gt = min(kG, Nk - j0);
  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int s = 0; s < 8; ++s) acc[r][s] = 0.0f;

  // global -> register staging of one step: A 32 x 128 and B 32 x 128 floats, 16 each per thread
  constexpr int AE = (KS * kG) / THREADS, BE = (KS * BM) / THREADS;
  float ra[AE], rb[BE];
  auto load_step = [&](int k0) {
    const float* wblk = Wc + (int64_t((kofs + k0) / kKBlock) * kG) * kKBlock + (k0 % kKBlock);
#pragma unroll
    for (int e = 0; e < AE; ++e) {
      const int idx = tid + THREADS * e;
      ra[e] = wblk[int64_t(idx / KS) * kKBlock + (idx % KS)];
    }
#pragma unroll
    for (int e = 0; e < BE; ++e) {
      const int idx = tid + THREADS * e;
      const int c = idx / BM, m = m0 + idx % BM;
      // padded entries of offsetk repeat the last kept k; rows past k_t are zero
      const int rk = offsetk[kofs + k0 + c];
      rb[e] = (m < M && k0 + c < kt) ? xt[int64_t(rk) * ldt + m] : 0.0f;
    }
  };
  load_step(0);
  for (int k0 = 0; k0 < kt; k0 += KS) {
    __syncthreads();  // the previous step's tiles have been read
#pragma unroll
    for (int e = 0; e < AE; ++e) {
      const int idx = tid + THREADS * e;
      As[idx % KS][idx / KS] = ra[e];
    }
#pragma unroll
    for (int e = 0; e < BE; ++e) {
      const int idx = tid + THREADS * e;
      Bs[idx / BM][idx % BM] = rb[e];
    }
    __syncthreads();
    if (k0 + KS < kt) load_step(k0 + KS);  // in flight while this step computes
#pragma unroll 4
    for (int c = 0; c < KS; ++c) {
      float a[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] = As[c][tj + 16 * r];
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[c][8 * tm]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[c][8 * tm + 4]);
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int s = 0; s < 8; ++s) acc[r][s] = fmaf(a[r], bv[s], acc[r][s]);
    }
  }

  const int n0 = tile_n0[t], n1 = tile_n0[t + 1];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int j = tj + 16 * r;
    if (j >= Gt) continue;
    const int nj = offsetn[j0 + j];
    const int gap_end = j + 1 < Gt ? offsetn[j0 + j + 1] : n1;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int m = m0 + 8 * tm + s;
      if (m >= M) continue;
      float* yrow = Y + int64_t(m) * ldy;
      yrow[nj] = acc[r][s];
      for (int z = nj + 1; z < gap_end; ++z) yrow[z] = 0.0f;
      if (j == 0)
        for (int z = n0; z < nj; ++z) yrow[z] = 0.0f;
    }
  }
}

spg_status check_desc(const spg_tw_desc* desc) {
  if (!desc) return SPG_ERR_INVALID_ARG;
  if (desc->G != kG || desc->T <= 0 || desc->N <= 0 || desc->K <= 0 || desc->Nk <= 0 || desc->offsetk_len <= 0 ||
      desc->offsetk_len % kKBlock)
    return SPG_ERR_INVALID_ARG;
  if (!desc->offsetn || !desc->tile_n0 || !desc->tile_kofs || !desc->k_per_tile || !desc->offsetk)
    return SPG_ERR_INVALID_ARG;
  return SPG_OK;
}

}  // namespace tw32
}  // namespace spg

extern "C" {

spg_status tw_condense_f32(const float* W, int64_t ldw, const spg_tw_desc* desc, float* Wc32, spg_stream_t stream) {
  using namespace spg;
  using namespace spg::tw32;
  spg_status st = check_desc(desc);
  if (st != SPG_OK) return st;
  if (!W || !Wc32 || ldw < desc->K) return SPG_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(Wc32, 16)) return SPG_ERR_MISALIGNED;
  st = check_device();
  if (st != SPG_OK) return st;
  // the widest tile in K-blocks bounds the grid's second dimension
  const int max_blocks = static_cast<int>(desc->K / kKBlock);
  condense_f32_kernel<<<dim3(desc->T, max_blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      W, ldw, int(desc->Nk), desc->offsetn, desc->tile_kofs, desc->k_per_tile, desc->offsetk, Wc32);
  return launch_status();
}

size_t tw_workspace_size_f32(int64_t M, int64_t K, int x_layout) {
  if (x_layout != SPG_X_MK || M <= 0 || K <= 0) return 0;
  return static_cast<size_t>((M * K * 4 + 255) / 256 * 256);
}

spg_status spgemm_tw_f32(const float* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, const float* Wc32,
                         float* Y, int64_t ldy, int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream) {
  using namespace spg;
  using namespace spg::tw32;
  spg_status st = check_desc(desc);
  if (st != SPG_OK) return st;
  if (!X || !Wc32 || !Y) return SPG_ERR_INVALID_ARG;
  if (x_layout != SPG_X_MK && x_layout != SPG_X_KM) return SPG_ERR_INVALID_ARG;
  const int64_t N = desc->N, K = desc->K;
  if (M <= 0 || ldy < N || (x_layout == SPG_X_MK ? ldx < K : ldx < M)) return SPG_ERR_INVALID_ARG;
  if (M >= (int64_t(1) << 31) || (M + BM - 1) / BM > 65535) return SPG_ERR_UNSUPPORTED_SHAPE;  // grid.y
  if (!aligned(X, 4) || !aligned(Wc32, 16) || !aligned(Y, 4)) return SPG_ERR_MISALIGNED;
  const float* xt = X;
  int64_t ldt = ldx;
  if (x_layout == SPG_X_KM) {
    if (!aligned(X, 16) || ldx % 4) return SPG_ERR_MISALIGNED;  // 16-byte row reads of Xt
  } else {
    if (!workspace || ws_bytes < tw_workspace_size_f32(M, K, x_layout)) return SPG_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SPG_ERR_MISALIGNED;
  }
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (x_layout == SPG_X_MK) {
    float* ws = static_cast<float*>(workspace);
    transpose_f32_kernel<<<dim3(unsigned((K + 31) / 32), unsigned((M + 31) / 32)), 256, 0, s>>>(X, ldx, int(M),
                                                                                               int(K), ws, M);
    xt = ws;
    ldt = M;
  }
  tw_gemm_f32_kernel<<<dim3(unsigned(desc->T), unsigned((M + BM - 1) / BM)), THREADS, 0, s>>>(
      xt, ldt, Wc32, Y, ldy, int(M), int(desc->Nk), desc->offsetn, desc->tile_n0, desc->tile_kofs, desc->k_per_tile,
      desc->offsetk);
  return launch_status();
}

}  // extern "C"
