// Tile-wise sparsity ("Accelerating Sparse DNN Models without Hardware-Support
// via Tile-Wise Sparsity", Guo et al.): the offline reorganisation of a dense
// fp16 W into condensed tiles (slides "Tile-Wise Sparsity", "Re-organize",
// "Preprocessed"), the explicit activation transpose (slide "Transpose") and
// the run-time GEMM that gathers A through offsetk and scatters C through
// offsetn (slide "Run-time").
//
// In C = A x B of the slides, A = X [M, K], B = W^T and C = Y [M, N]: the
// columns of B are the rows n of W, its rows the reduction indices k.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "host.cuh"
#include "sm100.cuh"
#include "spgemm.h"

namespace spg {
namespace tw {

using u128 = unsigned __int128;

constexpr int kG = 128;          // tile width (kept columns per tile)
constexpr int kKBlock = 64;      // K padding / GEMM K block
constexpr int kMaxK = 8192;      // reorganisation keeps a tile's K row norms in shared memory

// ---- exact norms ------------------------------------------------------------------------
// An fp16 value is +-m * 2^e with m = 1024 + frac, e = exp - 25 (normal) or
// m = frac, e = -24 (subnormal), so w*w*2^48 = m*m * 2^(2e+48) is an integer
// with 2e+48 = 2*exp - 2 (normal) or 0 (subnormal).  Sums of these are exact
// in 128 bits (each term < 2^82, at most 2^31 terms) and order independent.
__device__ __forceinline__ u128 sq_units(uint32_t bits) {
  const uint32_t ex = (bits >> 10) & 0x1Fu, fr = bits & 0x3FFu;
  const uint32_t m = ex ? (fr | 0x400u) : fr;
  const uint32_t sh = ex ? 2u * ex - 2u : 0u;
  return static_cast<u128>(static_cast<uint64_t>(m) * m) << sh;
}

__device__ __forceinline__ u128 shfl_xor_u128(u128 v, int mask) {
  const uint64_t lo = static_cast<uint64_t>(v), hi = static_cast<uint64_t>(v >> 64);
  const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, mask), h2 = __shfl_xor_sync(0xffffffffu, hi, mask);
  return (static_cast<u128>(h2) << 64) | l2;
}

// Column keys: key[n] = sum_k w[n][k]^2 (x 2^48), one warp per row n of W.
__global__ void col_keys_kernel(const uint16_t* __restrict__ W, int64_t ldw, int N, int K, u128* __restrict__ keys) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int n = blockIdx.x * wpb + (threadIdx.x >> 5); n < N; n += gridDim.x * wpb) {
    const uint16_t* row = W + int64_t(n) * ldw;
    u128 acc = 0;
    for (int k = lane; k < K; k += 32) acc += sq_units(row[k]);
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += shfl_xor_u128(acc, o);
    if (lane == 0) keys[n] = acc;
  }
}

// Column n is pruned when fewer than P columns precede it in the order
// (key ascending, index ascending), i.e. it is among the P smallest.
__global__ void col_prune_kernel(const u128* __restrict__ keys, int N, int P, int* __restrict__ kept) {
  __shared__ u128 sk[1024];
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const u128 mine = n < N ? keys[n] : 0;
  int before = 0;
  for (int base = 0; base < N; base += 1024) {
    const int cnt = min(1024, N - base);
    __syncthreads();
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) sk[i] = keys[base + i];
    __syncthreads();
    if (n < N)
      for (int i = 0; i < cnt; ++i) {
        const u128 o = sk[i];
        before += (o < mine) || (o == mine && base + i < n);
      }
  }
  if (n < N) kept[n] = before >= P ? 1 : 0;
}

// Block-wide exclusive scan of 0/1 flags in chunks of blockDim.x; calls
// emit(i, position) for every set flag i in ascending order.  One CTA.
template <typename Flag, typename Emit>
__device__ void compact_ascending(Flag flag, int count, int* s_warp, Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  int carry = 0;
  for (int base = 0; base < count; base += blockDim.x) {
    const int i = base + tid;
    const int f = (i < count && flag(i)) ? 1 : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    int warp_off = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
      if (w < warp) warp_off += s_warp[w];
      total += s_warp[w];
    }
    if (f) emit(i, carry + warp_off + in_warp);
    carry += total;
    __syncthreads();
  }
}

// offsetn (kept columns ascending) and tile_n0 (output column range of each tile).
__global__ void col_compact_kernel(const int* __restrict__ kept, int N, int T, int* __restrict__ offsetn,
                                   int* __restrict__ tile_n0) {
  __shared__ int s_warp[32];
  compact_ascending([&](int i) { return kept[i] != 0; }, N, s_warp,
                    [&](int i, int pos) {
                      offsetn[pos] = i;
                      if (pos % kG == 0) tile_n0[pos / kG] = pos == 0 ? 0 : i;
                    });
  if (threadIdx.x == 0) tile_n0[T] = N;
}

// One CTA per tile: exact row keys over the tile's kept columns, the k_t
// largest (ties: lower k first) kept, offsetk written ascending and padded to
// a multiple of 64 with the last kept k.
__global__ void tile_rows_kernel(const uint16_t* __restrict__ W, int64_t ldw, int K, int Nk,
                                 const int* __restrict__ offsetn, const int* __restrict__ tile_kofs,
                                 const int* __restrict__ k_per_tile, int* __restrict__ offsetk) {
  extern __shared__ uint8_t sm_raw[];
  u128* keys = reinterpret_cast<u128*>(sm_raw);
  int* keep = reinterpret_cast<int*>(keys + K);
  __shared__ int s_warp[32];
  __shared__ int s_last;
  const int t = blockIdx.x;
  const int j0 = t * kG;
  const int Gt = min(kG, Nk - j0);
  const int kt = k_per_tile[t];
  const int kofs = tile_kofs[t];
  const int kpad = tile_kofs[t + 1] - kofs;
  for (int k = threadIdx.x; k < K; k += blockDim.x) keys[k] = 0;
  __syncthreads();
  for (int j = 0; j < Gt; ++j) {
    const uint16_t* row = W + int64_t(offsetn[j0 + j]) * ldw;
    for (int k = threadIdx.x; k < K; k += blockDim.x) keys[k] += sq_units(row[k]);
  }
  __syncthreads();
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const u128 mine = keys[k];
    int before = 0;
    for (int o = 0; o < K; ++o) {
      const u128 v = keys[o];
      before += (v > mine) || (v == mine && o < k);
    }
    keep[k] = before < kt ? 1 : 0;
  }
  __syncthreads();
  compact_ascending([&](int i) { return keep[i] != 0; }, K, s_warp, [&](int i, int pos) {
    offsetk[kofs + pos] = i;
    if (pos == kt - 1) s_last = i;
  });
  __syncthreads();
  for (int i = kt + threadIdx.x; i < kpad; i += blockDim.x) offsetk[kofs + i] = s_last;
}

// Condensed values, block b of tile t: Wc[blk][j][c] = W[offsetn[tG+j]][offsetk[kofs+64b+c]].
__global__ void gather_wc_kernel(const uint16_t* __restrict__ W, int64_t ldw, int Nk,
                                 const int* __restrict__ offsetn, const int* __restrict__ tile_kofs,
                                 const int* __restrict__ k_per_tile, const int* __restrict__ offsetk,
                                 uint16_t* __restrict__ Wc) {
  const int t = blockIdx.x, b = blockIdx.y;
  const int kofs = tile_kofs[t];
  if (b * kKBlock >= tile_kofs[t + 1] - kofs) return;
  const int j0 = t * kG;
  const int Gt = min(kG, Nk - j0);
  const int kt = k_per_tile[t];
  uint16_t* out = Wc + (int64_t(kofs / kKBlock + b) * kG) * kKBlock;
  for (int e = threadIdx.x; e < kG * kKBlock; e += blockDim.x) {
    const int j = e / kKBlock, c = e % kKBlock;
    const int i = b * kKBlock + c;
    uint16_t v = 0;
    if (j < Gt && i < kt) v = W[int64_t(offsetn[j0 + j]) * ldw + offsetk[kofs + i]];
    out[e] = v;
  }
}

// ---- explicit activation transpose X [M, K] -> Xt [K, M] ------------------------------------
// One 64 (m) x 64 (k) tile per 256-thread block, 16-byte accesses on both
// sides (K % 64 == 0, 16-byte aligned rows; Xt's pitch ldt is M rounded up
// to a multiple of 8, and the columns past M in the last 8-wide chunk are
// written as zeros).  The tile sits in
// shared memory as 32-bit pairs (k, k+1) with a row pitch of 33 words, so
// both the row-wise stores and the column-wise reads are free of bank
// conflicts.  Reads: thread t takes 8 consecutive k of rows t/8 and t/8 + 32.
// Writes: thread t takes the k pair 2 (t/8) .. +1 and the 8 m of chunk t % 8,
// so 8 consecutive threads write 128 contiguous bytes of one output row.
__global__ void __launch_bounds__(256) transpose_kernel(const uint16_t* __restrict__ X, int64_t ldx, int M, int K,
                                                        uint16_t* __restrict__ Xt, int64_t ldt) {
  __shared__ uint32_t tile[64][33];  // [m][k pair]
  griddep_launch_dependents();
  griddep_wait();
  const int m0 = blockIdx.y * 64, k0 = blockIdx.x * 64;
  const int t = threadIdx.x;
  {
    const int c = t & 7;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = (t >> 3) + 32 * h;
      const uint4 v = m0 + r < M ? __ldg(reinterpret_cast<const uint4*>(X + int64_t(m0 + r) * ldx + k0 + 8 * c))
                                 : make_uint4(0u, 0u, 0u, 0u);
      tile[r][4 * c + 0] = v.x;
      tile[r][4 * c + 1] = v.y;
      tile[r][4 * c + 2] = v.z;
      tile[r][4 * c + 3] = v.w;
    }
  }
  __syncthreads();
  const int kp = t >> 3, j = t & 7;  // k pair (k = 2 kp, 2 kp + 1), m chunk
  if (m0 + 8 * j >= M) return;
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = tile[8 * j + i][kp];
  uint4 lo, hi;  // rows k (low halves) and k + 1 (high halves), 8 m each
  lo.x = __byte_perm(w[0], w[1], 0x5410);
  lo.y = __byte_perm(w[2], w[3], 0x5410);
  lo.z = __byte_perm(w[4], w[5], 0x5410);
  lo.w = __byte_perm(w[6], w[7], 0x5410);
  hi.x = __byte_perm(w[0], w[1], 0x7632);
  hi.y = __byte_perm(w[2], w[3], 0x7632);
  hi.z = __byte_perm(w[4], w[5], 0x7632);
  hi.w = __byte_perm(w[6], w[7], 0x7632);
  const int k = k0 + 2 * kp;
  *reinterpret_cast<uint4*>(Xt + int64_t(k) * ldt + m0 + 8 * j) = lo;
  *reinterpret_cast<uint4*>(Xt + int64_t(k + 1) * ldt + m0 + 8 * j) = hi;
}

// ---- run-time GEMM -------------------------------------------------------------------------
// ---- run-time GEMM -------------------------------------------------------------------------
// Work unit (tile t, 128-row block of X): D[j][m] = sum_i Wc_t[j][i] * X[m][offsetk_t[i]]
// on the dense tensor cores (A = condensed tile, K-major; B = gathered rows of
// Xt, MN-major), then Y[m][offsetn[tG+j]] = D[j][m] and +0 in the tile's
// pruned columns.  Persistent CTAs with warp roles (512 threads):
//   warps 0-3  loads: warp 0 lane 0 issues the TMA of the condensed tile
//              block; each lane of the four warps gathers kept rows of Xt
//              with 16-byte cp.async (warp w takes rows 16w..16w+15 of a
//              block; four warps keep about twice the bytes in flight of
//              two).
//              The 64 row indices of a block are read one block ahead, and
//              the scalars of the next unit one unit ahead, so no copy waits
//              on a dependent index load.
//   warp 4     TMEM owner and MMA issuer (two accumulators)
//   warps 8-15 drain, in two groups of four warps that each own 64 rows of
//              the unit: tcgen05.ld of the accumulator (released at once).  The
//              16-byte-aligned middle of the unit's output span
//              [tile_n0[t], tile_n0[t+1]) is assembled in double-buffered
//              shared memory, 184 columns at a time (zeroed, then each lane
//              places its kept column), and leaves as a few 2-D TMA stores;
//              the ragged ends (at most 7 columns a side) are assembled the
//              same way in a [128][16] edge buffer and leave with one store
//              instruction per two rows for both ends, from the three warps
//              of the group that did not issue the TMA stores.
constexpr int BN = 128;                   // X rows per work unit
constexpr int A_BYTES = kG * kKBlock * 2;  // 16 KB
constexpr int B_BYTES = kKBlock * BN * 2;  // 16 KB: 64 gathered rows x 128 m, two 64-wide atoms
constexpr int STAGES = 4;
constexpr int EPI_GROUPS = 2;              // drain groups of 4 warps, each owning RG rows of a unit
constexpr int RG = BN / EPI_GROUPS;        // 64
constexpr int kGatherWarps = 4;            // warps 0-3
constexpr int kRowsPerWarp = 64 / kGatherWarps;
constexpr int kMmaWarp = 4;
constexpr int kDrainWarp0 = 8;             // a multiple of 4: warp & 3 is the TMEM lane quadrant
constexpr int THREADS = 32 * kDrainWarp0 + 128 * EPI_GROUPS;
constexpr int WIN = 184;                   // output columns staged per window (a multiple of 8)
constexpr int WIN_ELEMS = RG * WIN;        // one staging buffer: [64 rows] x WIN, box-blocked
constexpr int OFF_STG = STAGES * (A_BYTES + B_BYTES);
constexpr int OFF_EDGE = OFF_STG + EPI_GROUPS * 2 * WIN_ELEMS * 2;  // two staging buffers per group
constexpr int OFF_BAR = OFF_EDGE + EPI_GROUPS * RG * 16 * 2;
constexpr int SMEM = OFF_BAR + (2 * STAGES + 5) * 8 + 16 + 1024;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(WIN % 8 == 0 && (WIN_ELEMS * 2) % 1024 == 0 && OFF_STG % 1024 == 0, "staging blocks stay aligned");
constexpr uint32_t TMEM_COLS = 256;
constexpr int kLoadLanes = 32 * kGatherWarps;  // cp.async arrivals per stage

__device__ __forceinline__ void tail_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  int never = 0;
  mbar_wait(bar, parity, &never, err, ERR_WAIT_TAIL);
}

// 16-byte global -> shared copy; src_bytes 0 fills the destination with zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Arrive on `bar` once every cp.async issued so far by this thread has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__global__ void __launch_bounds__(THREADS, 1)
    tw_gemm_kernel(const __grid_constant__ CUtensorMap tmWc, const __grid_constant__ CUtensorMap tmY64,
                   const __grid_constant__ CUtensorMap tmY8, const uint16_t* __restrict__ xt, int64_t ldt,
                   uint16_t* __restrict__ Y, int64_t ldy, int vec_ok, int y_nm, int M, int Nk, int T,
                   const int* __restrict__ offsetn,
                   const int* __restrict__ tile_n0, const int* __restrict__ tile_kofs,
                   const int* __restrict__ offsetk, uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MB = (M + BN - 1) / BN;
  const int units = T * MB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + kLoadLanes);  // TMA of the tile block + one cp.async arrival per gather lane
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * EPI_GROUPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmWc);
    if (vec_ok) {
      tma_prefetch_desc(&tmY64);
      tma_prefetch_desc(&tmY8);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_launch_dependents();
  griddep_wait();  // the previous kernel's writes (Xt, or readers of Y) are complete

  if (warp < kGatherWarps) {
    // ---------------- loads ----------------
    uint32_t g = 0;
    bool ok = true;
    const int rbase = kRowsPerWarp * warp;  // this warp's rows within a block
    const int rlane = lane % kRowsPerWarp;  // the row whose index this lane holds
    const int a = (lane >> 3) & 1, c = lane & 7, hl = lane >> 4;
    int u = blockIdx.x;
    // scalars of the current unit, and the first row indices of its block 0
    int kofs = 0, KB = 0, nxt = 0;
    if (u < units) {
      const int t = u / MB;
      kofs = tile_kofs[t];
      KB = (tile_kofs[t + 1] - kofs) / kKBlock;
      nxt = offsetk[kofs + rbase + rlane];
    }
    while (ok && u < units) {
      const int mb = (u % MB) * BN;
      const int mcol = mb + 64 * a + 8 * c;
      // the chunk of 8 m at mcol: whole, cut at M (the rest zero-filled), or empty
      const uint32_t src_bytes = mcol + 8 <= M ? 16u : mcol < M ? uint32_t(2 * (M - mcol)) : 0u;
      const uint16_t* xcol = xt + (src_bytes ? mcol : 0);
      // scalars of the next unit, loaded while this one is issued
      const int un = u + gridDim.x;
      int kofs_n = 0, KB_n = 0;
      if (un < units) {
        const int tn = un / MB;
        kofs_n = tile_kofs[tn];
        KB_n = (tile_kofs[tn + 1] - kofs_n) / kKBlock;
      }
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int cur = nxt;
        if (kb + 1 < KB)
          nxt = offsetk[kofs + (kb + 1) * kKBlock + rbase + rlane];
        else if (un < units)
          nxt = offsetk[kofs_n + rbase + rlane];
        const int s = g % STAGES;
        const uint32_t use = g / STAGES;
        if (use > 0 && !mbar_wait_warp(&empty[s], (use - 1) & 1, abort_flag, err, ERR_WAIT_EMPTY)) {
          ok = false;
          break;
        }
        uint8_t* a_s = smem + s * (A_BYTES + B_BYTES);
        const uint32_t b_s = smem_addr(a_s + A_BYTES);
        if (warp == 0 && lane == 0) {
          mbar_arrive_expect_tx(&full[s], A_BYTES);
          tma_load_2d(a_s, &tmWc, 0, (kofs / kKBlock + kb) * kG, &full[s]);
        }
        // B: kept rows of Xt, 128 m each, as two MN-major 128-byte-swizzled
        // atoms of 64 m (16-byte chunk c of row r at chunk c ^ (r % 8))
#pragma unroll
        for (int i = 0; i < kRowsPerWarp / 2; ++i) {
          const int rl = 2 * i + hl;
          const int r = rbase + rl;
          const int rk = __shfl_sync(0xffffffffu, cur, rl);
          const uint32_t dst = b_s + a * 8192 + r * 128 + ((c ^ (r & 7)) << 4);
          cp_async16(dst, xcol + int64_t(rk) * ldt, src_bytes);
        }
        cp_async_arrive(&full[s]);
      }
      u = un;
      kofs = kofs_n;
      KB = KB_n;
    }
    cp_async_wait_all();
    if (warp == 0 && lane == 0)
      for (uint32_t q = (g > uint32_t(STAGES) ? g - STAGES : 0u); q < g; ++q)
        tail_wait(&full[q % STAGES], (q / STAGES) & 1, err);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------- MMA ----------------
    // kind::f16 dense, fp16 inputs, fp32 accumulate, A K-major, B MN-major, M=128, N=128.
    // One thread issues, with single-thread bounded waits.
    constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | (1u << 16) | ((BN >> 3) << 17) | ((128 >> 4) << 24);
    if (lane == 0) {
      uint32_t g = 0;
      int i = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
        const int t = u / MB;
        const int KB = (tile_kofs[t + 1] - tile_kofs[t]) / kKBlock;
        const int b = i & 1;
        if (i >= 2 && !mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1, abort_flag, err, ERR_WAIT_ACC_FREE)) break;
        tc_fence_after();
        const uint32_t acc = tmem + uint32_t(b * BN);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(&full[s], (g / STAGES) & 1, abort_flag, err, ERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          fence_proxy_async_smem();  // the gathered rows were written by cp.async (generic proxy)
          const uint32_t a_s = smem_addr(smem + s * (A_BYTES + B_BYTES));
          const uint32_t b_s = a_s + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kKBlock / 16; ++kk) {
            const uint64_t adesc = smem_desc(a_s + 32 * kk, 16, 1024, LAYOUT_SW128);
            const uint64_t bdesc = smem_desc(b_s + 2048 * kk, 8192, 1024, LAYOUT_SW128);
            tc_mma(acc, adesc, bdesc, kIdesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[b]);
      }
      tc_commit(mma_done);
      tail_wait(mma_done, 0, err);
    }
    __syncwarp();
  } else if (warp >= kDrainWarp0) {
    // ---------------- drain and scatter ----------------
    // Group eg (warps 8-11: eg 0, warps 12-15: eg 1) drains rows [64 eg, 64 eg + 64)
    // of every unit: TMEM columns b*BN + 64 eg .. +63 of the lanes of quadrant q.
    const int q = warp & 3;
    const int eg = (warp - kDrainWarp0) >> 2;
    const int gtid = threadIdx.x - 32 * kDrainWarp0 - 128 * eg;  // 0..127 within the group
    const uint32_t bar_win = 1 + eg, bar_vote = 3 + eg;
    uint16_t* stg0 = reinterpret_cast<uint16_t*>(smem + OFF_STG + eg * (2 * WIN_ELEMS * 2));
    uint16_t* edge = reinterpret_cast<uint16_t*>(smem + OFF_EDGE + eg * (RG * 16 * 2));  // [64 rows][16]
    uint32_t wc = 0;  // windows staged so far: window w uses staging buffer w % 2
    int i = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++i) {
      const int t = u / MB;
      const int mb = (u % MB) * BN + RG * eg;  // first row of this group
      const int b = i & 1;
      // tile scalars first: their loads overlap the wait for the accumulator
      const int j0 = t * kG;
      const int Gt = min(kG, Nk - j0);
      const int j = 32 * q + lane;
      const bool valid = j < Gt;
      const int nj = valid ? offsetn[j0 + j] : 0;
      const int n0 = tile_n0[t], n1 = tile_n0[t + 1];
      const int rows = max(0, min(RG, M - mb));
      // Columns [s0, s1) are staged in windows; with 16-byte rows that is the
      // aligned middle of the span (TMA stores) and the ragged ends [n0, a0),
      // [a1, n1) go through the edge buffer; otherwise every column of the
      // span is staged and copied out by element stores.
      int s0, s1, a0 = n0, a1 = n1;
      if (vec_ok) {
        a0 = (n0 + 7) & ~7;
        a1 = max(a0, n1 & ~7);
        s0 = a0;
        s1 = a1;
      } else {
        s0 = n0 & ~7;
        s1 = (n1 + 7) & ~7;
      }
      const int e1 = n0 & ~7;  // edge slots 0-7: columns [e1, e1 + 8); slots 8-15: [a1, a1 + 8)
      // the four warps of the group take the same branch: they meet at named barriers below
      const bool got = mbar_wait_warp(&acc_full[b], (i >> 1) & 1, abort_flag, err, ERR_WAIT_ACC);
      if (!named_bar_all(bar_vote, 128, got)) break;
      tc_fence_after();
      uint32_t r[2][32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
        tmem_ld_32x32b_x32(tmem + (uint32_t(32 * q) << 16) + uint32_t(b * BN + RG * eg + 32 * cc), r[cc]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);

      if (y_nm) {
        // Y^T [N][M]: this lane's kept column nj is row nj of Y^T, and its 64
        // rows m are 128 contiguous bytes of that row, stored from registers;
        // the pruned columns it owns (its gap, and the tile's lead for j = 0)
        // are rows of zeros.  Yt's pitch is a multiple of 8 elements, so
        // whole 8-row chunks are 16-byte stores; a ragged end (M % 8) is
        // written element by element.
        if (valid && rows > 0) {
          uint16_t* yrow = Y + int64_t(nj) * ldy + mb;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t w[16];
#pragma unroll
            for (int p = 0; p < 16; ++p) {
              const float v0 = __uint_as_float(r[cc][2 * p]), v1 = __uint_as_float(r[cc][2 * p + 1]);
              asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w[p]) : "f"(v1), "f"(v0));
            }
            if (32 * cc + 32 <= rows) {
              uint4* d4 = reinterpret_cast<uint4*>(yrow + 32 * cc);
#pragma unroll
              for (int p = 0; p < 4; ++p) d4[p] = make_uint4(w[4 * p], w[4 * p + 1], w[4 * p + 2], w[4 * p + 3]);
            } else if (32 * cc < rows) {
              const int left = rows - 32 * cc;  // 1..31 rows of this half
              uint4* d4 = reinterpret_cast<uint4*>(yrow + 32 * cc);
#pragma unroll
              for (int p = 0; p < 4; ++p)
                if (8 * p + 8 <= left) d4[p] = make_uint4(w[4 * p], w[4 * p + 1], w[4 * p + 2], w[4 * p + 3]);
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e >= (left & ~7) && e < left)
                  yrow[32 * cc + e] = static_cast<uint16_t>((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu));
            }
          }
          const int gap_end = j + 1 < Gt ? offsetn[j0 + j + 1] : n1;
          auto zero_row = [&](int z) {
            uint4* d4 = reinterpret_cast<uint4*>(Y + int64_t(z) * ldy + mb);
            for (int e = 0; e < rows / 8; ++e) d4[e] = make_uint4(0u, 0u, 0u, 0u);
            for (int e = rows & ~7; e < rows; ++e) Y[int64_t(z) * ldy + mb + e] = 0;
          };
          for (int z = nj + 1; z < gap_end; ++z) zero_row(z);
          if (j == 0)
            for (int z = n0; z < nj; ++z) zero_row(z);
        }
        continue;
      }

      // Windows: zero, place kept columns, store.  Layout of a window of ww
      // columns (a multiple of 8): nw blocks [64 rows][64 columns] then nn
      // blocks [64 rows][8 columns], the shapes of the two TMA store boxes.
      // The first pass also zeroes and fills the edge buffer (even with no window).
      for (int x0 = s0, pass = 0; pass == 0 || x0 < s1; x0 += WIN, ++pass) {
        const int ww = max(0, min(WIN, s1 - x0));
        const int nw = ww >> 6, nn = (ww & 63) >> 3;
        uint16_t* stg = stg0 + (wc & 1) * WIN_ELEMS;
        {
          uint4* z = reinterpret_cast<uint4*>(stg);
          const int nz = ww * (RG / 8);
          for (int e = gtid; e < nz; e += 128) z[e] = make_uint4(0u, 0u, 0u, 0u);
          if (pass == 0 && gtid < RG * 2) reinterpret_cast<uint4*>(edge)[gtid] = make_uint4(0u, 0u, 0u, 0u);
        }
        named_bar_sync(bar_win, 128);
        int off = -1, rs = 0;
        if (valid && nj >= x0 && nj < x0 + ww) {
          const int rel = nj - x0;
          if (rel < 64 * nw) {
            off = (rel >> 6) * (RG * 64) + (rel & 63);
            rs = 64;
          } else {
            const int r2 = rel - 64 * nw;
            off = nw * (RG * 64) + (r2 >> 3) * (RG * 8) + (r2 & 7);
            rs = 8;
          }
        }
        uint16_t* dst = stg + off;
        if (pass == 0 && vec_ok && valid && (nj < a0 || nj >= a1)) {
          dst = edge + (nj < a0 ? nj - e1 : 8 + nj - a1);
          rs = 16;
          off = 0;
        }
        if (off >= 0) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              dst[(32 * cc + k) * rs] = __half_as_ushort(__float2half_rn(__uint_as_float(r[cc][k])));
        }
        fence_proxy_async_smem();             // staged rows -> the TMA stores below
        if (gtid == 0) bulk_wait_read<0>();   // the previous window's stores have read their buffer
        named_bar_sync(bar_win, 128);
        if (ww > 0) {
          if (vec_ok) {
            if (gtid == 0 && rows > 0) {
              const uint32_t sb = smem_addr(stg);
              for (int g = 0; g < nw; ++g)
                tma_store_2d_saddr(&tmY64, sb + uint32_t(g * RG * 64 * 2), x0 + 64 * g, mb);
              for (int h = 0; h < nn; ++h)
                tma_store_2d_saddr(&tmY8, sb + uint32_t((nw * RG * 64 + h * RG * 8) * 2), x0 + 64 * nw + 8 * h,
                                   mb);
              bulk_commit();
            }
          } else {
            // element stores, lanes across the columns of a row
            for (int row = q; row < rows; row += 4) {
              uint16_t* yrow = Y + int64_t(mb + row) * ldy;
              for (int rel = lane; rel < ww; rel += 32) {
                const int col = x0 + rel;
                const int so = rel < 64 * nw ? (rel >> 6) * (RG * 64) + row * 64 + (rel & 63)
                                             : nw * (RG * 64) + ((rel - 64 * nw) >> 3) * (RG * 8) + row * 8 +
                                                   ((rel - 64 * nw) & 7);
                if (col >= n0 && col < n1) yrow[col] = stg[so];
              }
            }
            named_bar_sync(bar_win, 128);  // the buffer is read before it is zeroed again
          }
          ++wc;
        }
      }
      // ragged ends (16-byte rows only): one instruction covers both edge
      // sectors of two rows; lanes 0-7 / 16-23 the head chunk, lanes 8-15 /
      // 24-31 the tail chunk, of rows r and r + 1.  The group's first warp
      // has just issued the TMA stores, so the other three share the rows.
      if (vec_ok && (n0 < a0 || a1 < n1) && q != 0) {
        const int l16 = lane & 15;
        const int col = l16 < 8 ? e1 + l16 : a1 + l16 - 8;
        const bool mine = l16 < 8 ? (col >= n0 && col < a0 && col < n1) : (col < n1);
        if (mine)
          for (int row = 2 * (q - 1) + (lane >> 4); row < rows; row += 6)
            Y[int64_t(mb + row) * ldy + col] = edge[row * 16 + l16];
      }
    }
    if (gtid == 0) bulk_wait_all<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// The GEMM's dynamic shared-memory limit, raised once per device.
bool smem_attr_set() {
  static int done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (__atomic_load_n(&done[dev], __ATOMIC_ACQUIRE)) return true;
  if (cudaFuncSetAttribute(tw_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
    return false;
  __atomic_store_n(&done[dev], 1, __ATOMIC_RELEASE);
  return true;
}

spg_status query(int64_t N, int64_t K, int32_t G, int64_t n_pruned, const int32_t* kpt, spg_tw_sizes* out) {
  if (!kpt || !out) return SPG_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || n_pruned < 0 || n_pruned >= N) return SPG_ERR_INVALID_ARG;
  if (G != kG || K % kKBlock || K > kMaxK || N >= (int64_t(1) << 31)) return SPG_ERR_UNSUPPORTED_SHAPE;
  const int64_t Nk = N - n_pruned;
  const int64_t T = (Nk + G - 1) / G;
  int64_t kofs = 0;
  for (int64_t t = 0; t < T; ++t) {
    if (kpt[t] < 1 || kpt[t] > K) return SPG_ERR_INVALID_ARG;
    kofs += (kpt[t] + kKBlock - 1) / kKBlock * kKBlock;
  }
  out->N = N;
  out->K = K;
  out->Nk = Nk;
  out->G = G;
  out->T = static_cast<int32_t>(T);
  out->offsetk_len = kofs;
  out->wc_elems = kofs * G;
  out->reorg_ws_bytes = (N * 16 + N * 4 + 255) / 256 * 256;
  return SPG_OK;
}

// Tensor maps and launch of the run-time GEMM over transposed activations
// xt [K][ldt] (shared by the entry points below).
spg_status launch_gemm(const uint16_t* xt, int64_t ldt, const spg_tw_desc* desc, uint16_t* Y, int64_t ldy,
                       int64_t M, cudaStream_t s, bool y_nm = false) {
  CUtensorMap tmWc, tmY64, tmY8;
  const uint64_t wc_rows = uint64_t(desc->offsetk_len / kKBlock) * kG;
  if (!make_tmap_2d(&tmWc, desc->Wc, 2, kKBlock, wc_rows, kKBlock * 2, kKBlock, kG, true)) return SPG_ERR_CUDA;
  // Y leaves through TMA when its rows are 16-byte aligned; otherwise by element stores only
  const int vec_ok = !y_nm && aligned(Y, 16) && (ldy % 8) == 0;
  if (vec_ok) {
    if (!make_tmap_2d(&tmY64, Y, 2, uint64_t(desc->N), uint64_t(M), uint64_t(ldy) * 2, 64, RG, false) ||
        !make_tmap_2d(&tmY8, Y, 2, uint64_t(desc->N), uint64_t(M), uint64_t(ldy) * 2, 8, RG, false))
      return SPG_ERR_CUDA;
  } else {
    std::memset(&tmY64, 0, sizeof(tmY64));
    std::memset(&tmY8, 0, sizeof(tmY8));
  }
  uint32_t* err = device_error_word();
  if (!err) return SPG_ERR_CUDA;
  if (!smem_attr_set()) return SPG_ERR_CUDA;
  const int64_t units = int64_t(desc->T) * ((M + BN - 1) / BN);
  const int grid = static_cast<int>(units < sm_count() ? units : sm_count());
  if (launch_pdl(tw_gemm_kernel, dim3(grid), dim3(THREADS), SMEM, s, tmWc, tmY64, tmY8, xt, ldt, Y, ldy, vec_ok, y_nm ? 1 : 0, int(M),
                                              int(desc->Nk), desc->T,
                                         desc->offsetn, desc->tile_n0, desc->tile_kofs, desc->offsetk, err) != cudaSuccess)
    return SPG_ERR_CUDA;
  return launch_status();
}

// Row pitch (elements) of the transposed activations [K][M] the explicit
// transpose writes: M rounded up to a multiple of 8, so every row is 16-byte
// aligned for the gather's 16-byte copies.
inline int64_t xt_pitch(int64_t M) { return (M + 7) / 8 * 8; }

// Validation, the optional explicit transpose and the GEMM launch shared by
// spgemm_tw_f16 (Y [M][N], y_nm false) and spgemm_tw_f16_yt (Y^T [N][M]).
spg_status run(const void* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, void* Y, int64_t ldy, int64_t M,
               void* workspace, size_t ws_bytes, spg_stream_t stream, bool y_nm) {
  // M == 0 (an empty batch) is valid: SPG_OK without a launch, and X / Y / workspace may be NULL
  if (!desc || (M != 0 && (!X || !Y))) return SPG_ERR_INVALID_ARG;
  if (x_layout != SPG_X_MK && x_layout != SPG_X_KM) return SPG_ERR_INVALID_ARG;
  const int64_t N = desc->N, K = desc->K;
  if (M < 0 || N <= 0 || K <= 0 || ldy < (y_nm ? M : N)) return SPG_ERR_INVALID_ARG;
  if (desc->G != kG || desc->T <= 0 || desc->offsetk_len <= 0 || desc->offsetk_len % kKBlock) return SPG_ERR_INVALID_ARG;
  if (!desc->offsetn || !desc->tile_n0 || !desc->tile_kofs || !desc->offsetk || !desc->Wc) return SPG_ERR_INVALID_ARG;
  if (x_layout == SPG_X_MK ? ldx < K : ldx < M) return SPG_ERR_INVALID_ARG;
  if (M == 0) return SPG_OK;  // empty batch: nothing is read or written
  if (M >= (int64_t(1) << 31)) return SPG_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || !aligned(Y, 2) || ldx % 8) return SPG_ERR_MISALIGNED;
  if (y_nm && (!aligned(Y, 16) || ldy % 8)) return SPG_ERR_MISALIGNED;
  if (x_layout == SPG_X_MK) {
    if (!workspace || ws_bytes < tw_workspace_size(M, K, x_layout)) return SPG_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SPG_ERR_MISALIGNED;
  }
  spg_status st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* xt = static_cast<const uint16_t*>(X);
  int64_t ldt = ldx;
  if (x_layout == SPG_X_MK) {
    uint16_t* ws = static_cast<uint16_t*>(workspace);
    dim3 grid(static_cast<unsigned>((K + 63) / 64), static_cast<unsigned>((M + 63) / 64));
    ldt = xt_pitch(M);
    if (launch_pdl(transpose_kernel, grid, dim3(256), 0, s, static_cast<const uint16_t*>(X), ldx, int(M), int(K), ws,
                   ldt) != cudaSuccess)
      return SPG_ERR_CUDA;
    xt = ws;
  }
  return launch_gemm(xt, ldt, desc, static_cast<uint16_t*>(Y), ldy, M, s, y_nm);
}

// ---- scratch for the entry point that allocates nothing ------------------------------------
// spgemm_tw_f16_noalloc keeps the transposed activations [K][M] in this
// file-scope device array instead of a caller-provided workspace.  Every GPU
// that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB: M*K*2 bytes at most
static __device__ __align__(256) uint16_t g_noalloc_xt[kNoAllocScratchBytes / 2];

// Device address of g_noalloc_xt on the current device (looked up once per
// device; the name itself is only a host-side stand-in for the symbol).
uint16_t* noalloc_scratch(spg_status* st) {
  static std::mutex mu;
  static uint16_t* ptr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = SPG_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_xt) != cudaSuccess || !p) {
      *st = SPG_ERR_CUDA;
      return nullptr;
    }
    ptr[dev] = static_cast<uint16_t*>(p);
  }
  *st = SPG_OK;
  return ptr[dev];
}

}  // namespace tw
}  // namespace spg

extern "C" {

spg_status tw_query_sizes(int64_t N, int64_t K, int32_t G, int64_t n_pruned, const int32_t* k_per_tile,
                          spg_tw_sizes* out) {
  return spg::tw::query(N, K, G, n_pruned, k_per_tile, out);
}

size_t tw_workspace_size(int64_t M, int64_t K, int x_layout) {
  if (x_layout != SPG_X_MK || M <= 0 || K <= 0) return 0;
  return static_cast<size_t>((spg::tw::xt_pitch(M) * K * 2 + 255) / 256 * 256);
}

spg_status tw_reorganize(const void* W, int64_t ldw, int64_t n_pruned, const int32_t* k_per_tile,
                         const spg_tw_desc* desc, void* workspace, size_t ws_bytes, spg_stream_t stream) {
  using namespace spg;
  using namespace spg::tw;
  if (!W || !desc || !k_per_tile || !workspace) return SPG_ERR_INVALID_ARG;
  spg_tw_sizes sz{};
  spg_status st = query(desc->N, desc->K, desc->G, n_pruned, k_per_tile, &sz);
  if (st != SPG_OK) return st;
  if (desc->Nk != sz.Nk || desc->T != sz.T || desc->offsetk_len != sz.offsetk_len || ldw < desc->K)
    return SPG_ERR_INVALID_ARG;
  if (!desc->offsetn || !desc->tile_n0 || !desc->tile_kofs || !desc->k_per_tile || !desc->offsetk || !desc->Wc)
    return SPG_ERR_INVALID_ARG;
  if (ws_bytes < size_t(sz.reorg_ws_bytes)) return SPG_ERR_INVALID_ARG;
  if (!aligned(W, 2) || !aligned(workspace, 16) || !aligned(desc->Wc, 16)) return SPG_ERR_MISALIGNED;
  st = check_device();
  if (st != SPG_OK) return st;
  const int N = int(sz.N), K = int(sz.K), Nk = int(sz.Nk), T = sz.T;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  // host tables: k per tile and the padded offsets of each tile in offsetk
  std::vector<int32_t> kofs(T + 1, 0);
  for (int t = 0; t < T; ++t) kofs[t + 1] = kofs[t] + (k_per_tile[t] + kKBlock - 1) / kKBlock * kKBlock;
  if (cudaMemcpyAsync(desc->tile_kofs, kofs.data(), sizeof(int32_t) * (T + 1), cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(desc->k_per_tile, k_per_tile, sizeof(int32_t) * T, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return SPG_ERR_CUDA;
  auto* keys = static_cast<u128*>(workspace);
  auto* kept = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + int64_t(N) * 16);
  const auto* W16 = static_cast<const uint16_t*>(W);
  col_keys_kernel<<<(N + 7) / 8, 256, 0, s>>>(W16, ldw, N, K, keys);
  col_prune_kernel<<<(N + 255) / 256, 256, 0, s>>>(keys, N, int(n_pruned), kept);
  col_compact_kernel<<<1, 1024, 0, s>>>(kept, N, T, desc->offsetn, desc->tile_n0);
  const int rows_smem = K * (16 + 4);
  if (cudaFuncSetAttribute(tile_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, rows_smem) != cudaSuccess)
    return SPG_ERR_CUDA;
  tile_rows_kernel<<<T, 256, rows_smem, s>>>(W16, ldw, K, Nk, desc->offsetn, desc->tile_kofs, desc->k_per_tile,
                                             desc->offsetk);
  int max_blocks = 0;
  for (int t = 0; t < T; ++t) max_blocks = std::max(max_blocks, (kofs[t + 1] - kofs[t]) / kKBlock);
  gather_wc_kernel<<<dim3(T, max_blocks), 256, 0, s>>>(W16, ldw, Nk, desc->offsetn, desc->tile_kofs,
                                                       desc->k_per_tile, desc->offsetk,
                                                       static_cast<uint16_t*>(desc->Wc));
  return launch_status();
}

spg_status spgemm_tw_f16(const void* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, void* Y, int64_t ldy,
                         int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream) {
  return spg::tw::run(X, ldx, x_layout, desc, Y, ldy, M, workspace, ws_bytes, stream, false);
}

// Y^T [N][M] output: the transpose a following tile-wise layer needs is fused here.
spg_status spgemm_tw_f16_yt(const void* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, void* Yt,
                            int64_t ldyt, int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream) {
  return spg::tw::run(X, ldx, x_layout, desc, Yt, ldyt, M, workspace, ws_bytes, stream, true);
}

// Tile-wise GEMM on [M, K] activations for callers that cannot allocate
// device memory: the transposed activations go to the library's own 8 MiB
// device array instead of a caller workspace.  Same results as
// spgemm_tw_f16(..., SPG_X_MK, ...).
spg_status spgemm_tw_f16_noalloc(const void* X, int64_t ldx, const spg_tw_desc* desc, void* Y, int64_t ldy,
                                 int64_t M, spg_stream_t stream) {
  using namespace spg;
  using namespace spg::tw;
  if (!X || !desc || !Y) return SPG_ERR_INVALID_ARG;
  const int64_t N = desc->N, K = desc->K;
  if (M <= 0 || N <= 0 || K <= 0 || ldy < N || ldx < K) return SPG_ERR_INVALID_ARG;
  if (desc->G != kG || desc->T <= 0 || desc->offsetk_len <= 0 || desc->offsetk_len % kKBlock) return SPG_ERR_INVALID_ARG;
  if (!desc->offsetn || !desc->tile_n0 || !desc->tile_kofs || !desc->offsetk || !desc->Wc) return SPG_ERR_INVALID_ARG;
  if (M >= (int64_t(1) << 31)) return SPG_ERR_UNSUPPORTED_SHAPE;
  const int64_t ldt = xt_pitch(M);
  if (uint64_t(ldt) * uint64_t(K) * 2u > kNoAllocScratchBytes) return SPG_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || !aligned(Y, 2) || ldx % 8) return SPG_ERR_MISALIGNED;
  spg_status st = check_device();
  if (st != SPG_OK) return st;
  uint16_t* xt = noalloc_scratch(&st);
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  // every element of the [K][M] region the GEMM reads is written here first,
  // so nothing left in the array by an earlier call is ever read
  dim3 tgrid(static_cast<unsigned>((K + 63) / 64), static_cast<unsigned>((M + 63) / 64));
  if (launch_pdl(transpose_kernel, tgrid, dim3(256), 0, s, static_cast<const uint16_t*>(X), ldx, int(M), int(K), xt,
                 ldt) != cudaSuccess)
    return SPG_ERR_CUDA;
  return launch_gemm(xt, ldt, desc, static_cast<uint16_t*>(Y), ldy, M, s);
}

}  // extern "C"
