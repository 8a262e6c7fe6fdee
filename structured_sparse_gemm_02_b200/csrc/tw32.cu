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

constexpr int kG = 128;            // tile width (kept columns per tile)
constexpr int kKBlock = 64;        // K padding of the descriptor
constexpr int KS = 32;             // kept rows per pipeline stage
constexpr int kLptMaxTiles = 256;  // largest T whose units are ordered by k_t
constexpr int kSpanMap = 2048;     // widest tile span written through a column map

// Condensed fp32 values, k-major: block b of tile t holds Wc[blk][c][j] =
// W[offsetn[tG+j]][offsetk[kofs+64b+c]] for j < G_t and 64b + c < k_t, +0
// elsewhere (blk = kofs/64 + b), so 32 consecutive kept rows of a tile are one
// contiguous 16 KB run.
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
  float* out = Wc + (int64_t(kofs / kKBlock + b) * kKBlock) * kG;
  for (int e = threadIdx.x; e < kG * kKBlock; e += blockDim.x) {
    const int c = e / kG, j = e % kG;
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

template <int BM>
struct F32Cfg {
  static constexpr int THREADS = 2 * BM;                    // thread (tj, tm): 16 column groups x BM/8 row groups
  static constexpr int A_FLOATS = KS * kG, B_FLOATS = KS * BM;
  static constexpr int STAGE_FLOATS = A_FLOATS + B_FLOATS;
  static constexpr int SMEM = 2 * STAGE_FLOATS * 4;         // two stages; the epilogue tile S [BM][128] reuses them
  static_assert(BM * kG <= 2 * STAGE_FLOATS, "epilogue tile must fit in the stage buffers");
  static constexpr int A_CHUNKS = A_FLOATS / 4 / THREADS;   // 16-byte copies per thread per stage
  static constexpr int B_CHUNKS = B_FLOATS / 4 / THREADS;
  static constexpr int MIN_BLOCKS = 512 / THREADS;          // 128 registers a thread
};

// One block per unit (tile t, rows [m0, m0 + BM)); a unit's index is its
// rank in the order of k_t descending (ties: lower t first), then its row
// block, so that blocks dispatched in index order start with the longest
// units (T <= 256; larger T keep the natural order).  Thread (tj, tm) holds
// the 8 x 8 accumulators of kept columns {4tj + r, 64 + 4tj + r} (r < 4) and
// rows 8tm + s, in fp32 with fused multiply-add over each tile's kept rows in
// ascending order.  Each stage copies 32 kept rows with cp.async: the
// condensed tile's contiguous run, and Xt[offsetk[.]][m0 .. m0 + BM) (rows
// past k_t and columns past M zero-filled); two stages alternate.  The
// epilogue stages the tile in shared memory and writes each row's span
// [tile_n0[t], tile_n0[t+1]) with consecutive lanes on consecutive columns:
// the kept column's value, +0 in a pruned one (span <= 2048, through a
// column map; wider spans write each kept column at Y[m][offsetn[tG+j]] and
// zero the gap after it, and before the first one, lane by lane).
template <int BM>
__global__ void __launch_bounds__(F32Cfg<BM>::THREADS, F32Cfg<BM>::MIN_BLOCKS) tw_gemm_f32_kernel(
    const float* __restrict__ xt, int64_t ldt, const float* __restrict__ Wc, float* __restrict__ Y, int64_t ldy,
    int M, int Nk, int T, int RU, const int* __restrict__ offsetn, const int* __restrict__ tile_n0,
    const int* __restrict__ tile_kofs, const int* __restrict__ k_per_tile, const int* __restrict__ offsetk) {
  using C = F32Cfg<BM>;
  extern __shared__ __align__(16) float smem[];
  __shared__ int kts[kLptMaxTiles];
  __shared__ int sel;
  __shared__ short pos[kSpanMap];
  const int tid = threadIdx.x;
  const int rank = blockIdx.x / RU, m0 = (blockIdx.x % RU) * BM;
  int t = rank;
  if (T <= kLptMaxTiles) {
    for (int i = tid; i < T; i += C::THREADS) kts[i] = k_per_tile[i];
    __syncthreads();
    for (int i = tid; i < T; i += C::THREADS) {
      const int mine = kts[i];
      int r = 0;
      for (int o = 0; o < T; ++o) r += (kts[o] > mine) | ((kts[o] == mine) & (o < i));
      if (r == rank) sel = i;
    }
    __syncthreads();
    t = sel;
  }
  const int tj = tid & 15, tm = tid >> 4;
  const int kofs = tile_kofs[t];
  const int kt = k_per_tile[t];
  const int j0 = t * kG;
  const int Gt = min(kG, Nk - j0);
  const int nsteps = (kt + KS - 1) / KS;

  // this thread's B copies: rows bc0 + (THREADS / (BM/4)) i, the 4 columns at bm (the same in every stage)
  constexpr int BQ = BM / 4, BSTEP = C::THREADS / BQ;
  const int bc0 = tid / BQ;
  const int bm = m0 + 4 * (tid % BQ);
  const int bvalid = min(max(M - bm, 0), 4) * 4;
  const float* xcol = xt + bm;
  const int* krow = offsetk + kofs + bc0;
  auto issue = [&](int step) {
    float* st = smem + (step & 1) * C::STAGE_FLOATS;
    const int k0 = step * KS;
    const float* asrc = Wc + (int64_t((kofs + k0) / kKBlock) * kKBlock + (k0 % kKBlock)) * kG;
#pragma unroll
    for (int i = 0; i < C::A_CHUNKS; ++i) {
      const int q = tid + C::THREADS * i;
      cp_async16(st + 4 * q, asrc + 4 * q, 16);
    }
    float* bdst = st + C::A_FLOATS + 4 * tid;
#pragma unroll
    for (int i = 0; i < C::B_CHUNKS; ++i) {
      const int c = k0 + bc0 + BSTEP * i;
      const int rk = krow[k0 + BSTEP * i];  // padded entries repeat the last kept k
      const int valid = c < kt ? bvalid : 0;
      cp_async16(bdst + 4 * C::THREADS * i, valid ? xcol + int64_t(rk) * ldt : xt, valid);
    }
    cp_async_commit();
  };

  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int s = 0; s < 8; ++s) acc[r][s] = 0.0f;

  issue(0);
  for (int step = 0; step < nsteps; ++step) {
    if (step + 1 < nsteps) {
      issue(step + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float* As = smem + (step & 1) * C::STAGE_FLOATS;
    const float* Bs = As + C::A_FLOATS;
#pragma unroll
    for (int c = 0; c < KS; ++c) {
      const float4 a0 = *reinterpret_cast<const float4*>(As + c * kG + 4 * tj);
      const float4 a1 = *reinterpret_cast<const float4*>(As + c * kG + 64 + 4 * tj);
      const float4 b0 = *reinterpret_cast<const float4*>(Bs + c * BM + 8 * tm);
      const float4 b1 = *reinterpret_cast<const float4*>(Bs + c * BM + 8 * tm + 4);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int s = 0; s < 8; ++s) acc[r][s] = fmaf(av[r], bv[s], acc[r][s]);
    }
    __syncthreads();  // this stage is refilled by the next issue
  }

  // epilogue: S [BM][128] in the stage buffers, then kept columns scattered through offsetn
  float* S = smem;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    float* row = S + (8 * tm + s) * kG;
    *reinterpret_cast<float4*>(row + 4 * tj) = make_float4(acc[0][s], acc[1][s], acc[2][s], acc[3][s]);
    *reinterpret_cast<float4*>(row + 64 + 4 * tj) = make_float4(acc[4][s], acc[5][s], acc[6][s], acc[7][s]);
  }
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int WARPS = C::THREADS / 32;
  const int n0 = tile_n0[t], n1 = tile_n0[t + 1];
  const int span = n1 - n0;
  if (span <= kSpanMap) {
    // position of each output column of the span among the kept columns, -1 for a pruned one
    for (int z = tid; z < span; z += C::THREADS) pos[z] = -1;
    __syncthreads();
    for (int j = tid; j < Gt; j += C::THREADS) pos[offsetn[j0 + j] - n0] = static_cast<short>(j);
    __syncthreads();
    for (int mm = warp; mm < BM; mm += WARPS) {
      const int m = m0 + mm;
      if (m >= M) break;
      float* yrow = Y + int64_t(m) * ldy + n0;
      const float* srow = S + mm * kG;
      for (int z = lane; z < span; z += 32) {
        const int j = pos[z];
        yrow[z] = j >= 0 ? srow[j] : 0.0f;
      }
    }
    return;
  }
  __syncthreads();
  int nj[4], gend[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = lane + 32 * q;
    nj[q] = j < Gt ? offsetn[j0 + j] : -1;
    gend[q] = j + 1 < Gt ? offsetn[j0 + j + 1] : n1;
  }
  const int lead = offsetn[j0];  // pruned columns before the tile's first kept column
  for (int mm = warp; mm < BM; mm += WARPS) {
    const int m = m0 + mm;
    if (m >= M) break;
    float* yrow = Y + int64_t(m) * ldy;
    const float* srow = S + mm * kG;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (nj[q] < 0) continue;
      yrow[nj[q]] = srow[lane + 32 * q];
      for (int z = nj[q] + 1; z < gend[q]; ++z) yrow[z] = 0.0f;
    }
    for (int z = n0 + lane; z < lead; z += 32) yrow[z] = 0.0f;
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

// Both GEMM variants' dynamic shared-memory limits, raised once per device.
bool smem_attr_set() {
  static int done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (__atomic_load_n(&done[dev], __ATOMIC_ACQUIRE)) return true;
  if (cudaFuncSetAttribute(tw_gemm_f32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           F32Cfg<128>::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(tw_gemm_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           F32Cfg<64>::SMEM) != cudaSuccess)
    return false;
  __atomic_store_n(&done[dev], 1, __ATOMIC_RELEASE);
  return true;
}

template <int BM>
void launch_gemm(const float* xt, int64_t ldt, const float* Wc, float* Y, int64_t ldy, int M,
                 const spg_tw_desc* desc, cudaStream_t s) {
  const int RU = (M + BM - 1) / BM;
  tw_gemm_f32_kernel<BM><<<unsigned(int64_t(desc->T) * RU), F32Cfg<BM>::THREADS, F32Cfg<BM>::SMEM, s>>>(
      xt, ldt, Wc, Y, ldy, M, int(desc->Nk), int(desc->T), RU, desc->offsetn, desc->tile_n0, desc->tile_kofs,
      desc->k_per_tile, desc->offsetk);
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
  return static_cast<size_t>(((M + 3) / 4 * 4 * K * 4 + 255) / 256 * 256);  // Xt [K, M] at a pitch of 4-float multiples
}

spg_status spgemm_tw_f32(const float* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, const float* Wc32,
                         float* Y, int64_t ldy, int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream) {
  using namespace spg;
  using namespace spg::tw32;
  spg_status st = check_desc(desc);
  if (st != SPG_OK) return st;
  // M == 0 (an empty batch) is valid: SPG_OK without a launch, and X / Y / workspace may be NULL
  if (!Wc32 || (M != 0 && (!X || !Y))) return SPG_ERR_INVALID_ARG;
  if (x_layout != SPG_X_MK && x_layout != SPG_X_KM) return SPG_ERR_INVALID_ARG;
  const int64_t N = desc->N, K = desc->K;
  if (M < 0 || ldy < N || (x_layout == SPG_X_MK ? ldx < K : ldx < M)) return SPG_ERR_INVALID_ARG;
  if (M >= (int64_t(1) << 31) || int64_t(desc->T) * ((M + 63) / 64) >= (int64_t(1) << 31))
    return SPG_ERR_UNSUPPORTED_SHAPE;  // one block per (tile, row block)
  if (M == 0) return SPG_OK;  // empty batch: nothing is read or written
  if (!aligned(X, 4) || !aligned(Wc32, 16) || !aligned(Y, 4)) return SPG_ERR_MISALIGNED;
  if (x_layout == SPG_X_KM) {
    if (!aligned(X, 16) || ldx % 4) return SPG_ERR_MISALIGNED;  // 16-byte copies of Xt rows
  } else {
    if (!workspace || ws_bytes < tw_workspace_size_f32(M, K, x_layout)) return SPG_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SPG_ERR_MISALIGNED;
  }
  st = check_device();
  if (st != SPG_OK) return st;
  if (!smem_attr_set()) return SPG_ERR_CUDA;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  const float* xt = X;
  int64_t ldt = ldx;
  if (x_layout == SPG_X_MK) {
    ldt = (M + 3) / 4 * 4;
    float* ws = static_cast<float*>(workspace);
    transpose_f32_kernel<<<dim3(unsigned((K + 31) / 32), unsigned((M + 31) / 32)), 256, 0, s>>>(X, ldx, int(M),
                                                                                               int(K), ws, ldt);
    xt = ws;
  }
  // 128-row units when they fill the GPU's block slots about twice (two blocks per SM), else 64-row units
  const int64_t units128 = int64_t(desc->T) * ((M + 127) / 128);
  if (units128 >= 4 * int64_t(sm_count()))
    launch_gemm<128>(xt, ldt, Wc32, Y, ldy, int(M), desc, s);
  else
    launch_gemm<64>(xt, ldt, Wc32, Y, ldy, int(M), desc, s);
  return launch_status();
}

}  // extern "C"
