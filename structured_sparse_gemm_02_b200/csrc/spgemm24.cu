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
// Persistent kernel, one CTA per SM, warp roles (256 threads):
//   warp 0     TMA producer: compressed W, X and the canonical metadata of
//              every stage into a STAGES-deep ring that runs across tiles
//   warp 1     fp16/bf16 only: rearranges each stage's metadata into the
//              order the tensor cores read it (permute_meta_f16)
//   warp 2     TMEM owner and MMA issuer: tcgen05.cp (metadata into tensor
//              memory), tcgen05.mma.sp into one of two accumulators
//   warp 3     idle
//   warps 4-7  epilogue: tcgen05.ld of a finished accumulator (released as
//              soon as it is read), bias / dequant, convert, TMA store of
//              32x32 output boxes; the ragged right edge uses checked stores
// Every wait is bounded (sm100.cuh); on a timeout the CTA drains what it has
// in flight, frees tensor memory and exits with the error word set.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "host.cuh"
#include "sm100.cuh"
#include "spgemm.h"

namespace spg {
namespace gemm24 {

enum OutKind { OUT_F16 = 0, OUT_BF16 = 1, OUT_S32 = 2 };

template <bool kInt8, int BN, int STAGES, int OUT>
struct Cfg {
  static constexpr int BM = 128;                       // weight rows per tile (MMA M)
  static constexpr int KSTEP = kInt8 ? 256 : 128;      // logical K per pipeline stage
  static constexpr int A_BYTES = BM * 128;             // 128 B of compressed row per stage
  static constexpr int B_BYTES = BN * 256;             // 256 B of X row per stage (two 128 B atoms)
  static constexpr int MSTG_BYTES = kInt8 ? 4096 : 2048;  // canonical metadata of the stage (TMA)
  static constexpr int MCP_BYTES = kInt8 ? 0 : 2048;      // fp16/bf16: metadata in tcgen05.cp order
  static constexpr int MCOLS = kInt8 ? 8 : 4;          // TMEM columns of metadata per stage
  static constexpr int OUT_ES = OUT == OUT_S32 ? 4 : 2;
  static constexpr int EPI_BUF = 32 * 32 * OUT_ES;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_MSTG = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_MCP = OFF_MSTG + STAGES * MSTG_BYTES;
  static constexpr int OFF_EPI = OFF_MCP + STAGES * MCP_BYTES;
  static constexpr int OFF_BAR = OFF_EPI + 4 * 2 * EPI_BUF;
  // tma_full[S], meta_full[S], empty[S], acc_full[2], acc_empty[2], mma_done
  static constexpr int NUM_BARS = 3 * STAGES + 5;
  static constexpr int SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr uint32_t META_COL = 2 * BN;  // metadata ring after the two accumulators
  static constexpr uint32_t TMEM_NEED = 2 * BN + 2 * MCOLS;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32    ? 32
                                        : TMEM_NEED <= 64  ? 64
                                        : TMEM_NEED <= 128 ? 128
                                        : TMEM_NEED <= 256 ? 256
                                                           : 512;
  static constexpr uint32_t TX_BYTES = A_BYTES + B_BYTES + MSTG_BYTES;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(TMEM_NEED <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
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
  } else if constexpr (OUT == OUT_BF16) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(__fadd_rn(__uint_as_float(acc), badd)));
  } else {
    return __half_as_ushort(__float2half_rn(__fadd_rn(__uint_as_float(acc), badd)));
  }
}

// CTA b computes tiles b, b + gridDim.x, ... of the ceil(N/128) x ceil(M/BN)
// tile grid (n fastest, so the CTAs in flight share X tiles through L2).
template <bool kInt8, bool kBF16, int BN, int STAGES, int OUT>
__global__ void __launch_bounds__(256, 1)
    spgemm24_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                    void* __restrict__ Yp, int64_t ldy, const void* __restrict__ bias,
                    const float* __restrict__ scale, int M, int N, int K, uint32_t* err) {
  using C = Cfg<kInt8, BN, STAGES, OUT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* tma_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* meta_full = tma_full + STAGES;
  uint64_t* empty = meta_full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = K / C::KSTEP;
  const int NT = (N + C::BM - 1) / C::BM;
  const int total = NT * ((M + BN - 1) / BN);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&meta_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
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
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const int n0 = (t % NT) * C::BM, m0 = (t / NT) * BN;
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
          mbar_arrive_expect_tx(&tma_full[s], C::TX_BYTES);
          tma_load_2d(a_s, &tmA, kb * (C::KSTEP / 2), n0, &tma_full[s]);
          tma_load_2d(b_s, &tmB, kb * C::KSTEP, m0, &tma_full[s]);
          tma_load_2d(b_s + BN * 128, &tmB, kb * C::KSTEP + C::KSTEP / 2, m0, &tma_full[s]);
          if constexpr (kInt8) {
            tma_load_2d(e_s, &tmE, kb * 32, n0, &tma_full[s]);
            tma_load_2d(e_s + 2048, &tmE, kb * 32 + 16, n0, &tma_full[s]);
          } else {
            tma_load_2d(e_s, &tmE, kb * 16, n0, &tma_full[s]);
          }
        }
      }
      // Let every issued copy land before shared memory can be released.
      for (uint32_t q = (g > uint32_t(STAGES) ? g - STAGES : 0u); q < g; ++q)
        tail_wait(&tma_full[q % STAGES], (q / STAGES) & 1, err);
    }
  } else if (warp == 1) {
    // ------------- metadata arrangement (fp16/bf16 only) -------------
    if constexpr (!kInt8) {
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(&tma_full[s], (g / STAGES) & 1, abort_flag, err, ERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          permute_meta_f16(smem + C::OFF_MSTG + s * C::MSTG_BYTES, smem + C::OFF_MCP + s * C::MCP_BYTES, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&meta_full[s]);
        }
      }
    }
  } else if (warp == 2) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t kFmt = kInt8 ? 1u : (kBF16 ? 1u : 0u);
    constexpr uint32_t kCFmt = kInt8 ? 2u : 1u;
    uint32_t g = 0;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++i) {
      const int b = i & 1;
      if (i >= 2 && !mbar_wait(&acc_empty[b], ((i >> 1) - 1) & 1, abort_flag, err, ERR_WAIT_ACC_FREE)) break;
      tc_fence_after();
      const uint32_t acc = tmem + uint32_t(b * BN);
      for (int kb = 0; kb < KB; ++kb, ++g) {
        const int s = g % STAGES;
        const uint32_t ph = (g / STAGES) & 1;
        if (!mbar_wait(&tma_full[s], ph, abort_flag, err, ERR_WAIT_FULL)) {
          ok = false;
          break;
        }
        if constexpr (!kInt8) {
          if (!mbar_wait(&meta_full[s], ph, abort_flag, err, ERR_WAIT_META)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_s = smem_addr(smem + C::OFF_A + s * C::A_BYTES);
          const uint32_t b_s = smem_addr(smem + C::OFF_B + s * C::B_BYTES);
          const uint32_t ecol = tmem + C::META_COL + (g & 1) * C::MCOLS;
          if constexpr (kInt8) {
            const uint32_t e_s = smem_addr(smem + C::OFF_MSTG + s * C::MSTG_BYTES);
            tc_cp_128x128b(ecol, smem_desc(e_s, 2048, 128, LAYOUT_NONE));
            tc_cp_128x128b(ecol + 4, smem_desc(e_s + 2048, 2048, 128, LAYOUT_NONE));
          } else {
            const uint32_t e_s = smem_addr(smem + C::OFF_MCP + s * C::MCP_BYTES);
            tc_cp_128x128b(ecol, smem_desc(e_s, 2048, 128, LAYOUT_NONE));
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t adesc = smem_desc(a_s + 32 * j, 16, 1024, LAYOUT_SW128);
            const uint64_t bdesc =
                smem_desc(b_s + (j >> 1) * (BN * 128) + (j & 1) * 64, 16, 1024, LAYOUT_SW128);
            const uint32_t e = kInt8 ? ecol + 2 * j : ecol + (j & ~1);
            const uint32_t sel = kInt8 ? 0u : uint32_t(j & 1);
            tc_mma_sp<kInt8>(acc, adesc, bdesc, e, instr_desc(kFmt, kCFmt, 128, BN, true, sel),
                             (kb | j) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&acc_full[b]);
      __syncwarp();
    }
    if (lane == 0) {
      tc_commit(mma_done);
      tail_wait(mma_done, 0, err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;  // tensor-memory lane quadrant of this warp
    uint8_t* epi = smem + C::OFF_EPI + q * 2 * C::EPI_BUF;
    uint32_t cc = 0;  // output boxes staged by this warp so far
    int i = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
      const int n0 = (t % NT) * C::BM, m0 = (t / NT) * BN;
      const int b = i & 1;
      if (!mbar_wait(&acc_full[b], (i >> 1) & 1, abort_flag, err, ERR_WAIT_ACC)) break;
      tc_fence_after();
      uint32_t r[BN / 32][32];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld_32x32b_x32(tmem + (uint32_t(32 * q) << 16) + uint32_t(b * BN + 32 * c), r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);

      const int nb = n0 + 32 * q;
      if (nb >= N) continue;
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
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        const int mb = m0 + 32 * c;
        if (mb >= M) continue;
        if (full_n) {
          if (cc >= 2) {
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          uint8_t* buf = epi + (cc & 1) * C::EPI_BUF;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const uint32_t v = convert_out<OUT, kInt8>(r[c][k], badd, sc, has_bias);
            if constexpr (C::OUT_ES == 4)
              reinterpret_cast<uint32_t*>(buf)[k * 32 + lane] = v;
            else
              reinterpret_cast<uint16_t*>(buf)[k * 32 + lane] = static_cast<uint16_t>(v);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, buf, nb, mb);
            bulk_commit();
          }
          __syncwarp();
          ++cc;
        } else if (n < N) {
          // ragged right edge: bounds-checked direct stores
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            if (mb + k >= M) continue;
            const uint32_t v = convert_out<OUT, kInt8>(r[c][k], badd, sc, has_bias);
            if constexpr (C::OUT_ES == 4)
              static_cast<uint32_t*>(Yp)[int64_t(mb + k) * ldy + n] = v;
            else
              static_cast<uint16_t*>(Yp)[int64_t(mb + k) * ldy + n] = static_cast<uint16_t>(v);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int sm_count() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int v = 148;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = v;
  }
  return cached[dev];
}

template <bool kInt8, bool kBF16, int BN, int STAGES, int OUT>
spg_status launch(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, const void* bias,
                  const float* scale, void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  using C = Cfg<kInt8, BN, STAGES, OUT>;
  const int es = kInt8 ? 1 : 2;
  CUtensorMap tmA, tmB, tmE, tmY;
  if (!make_tmap_2d(&tmA, Wv, es, uint64_t(K / 2), uint64_t(N), uint64_t(K / 2) * es, 128 / es, 128, true) ||
      !make_tmap_2d(&tmB, X, es, uint64_t(K), uint64_t(M), uint64_t(ldx) * es, 128 / es, BN, true) ||
      !make_tmap_2d(&tmE, meta, 1, uint64_t(K / 8), uint64_t(N), uint64_t(K / 8), 16, 128, false) ||
      !make_tmap_2d(&tmY, Y, C::OUT_ES, uint64_t(N), uint64_t(M), uint64_t(ldy) * C::OUT_ES, 32, 32, false))
    return SPG_ERR_CUDA;
  uint32_t* err = device_error_word();
  if (!err) return SPG_ERR_CUDA;
  auto kern = spgemm24_kernel<kInt8, kBF16, BN, STAGES, OUT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return SPG_ERR_CUDA;
  const int64_t tiles = ((N + C::BM - 1) / C::BM) * ((M + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  kern<<<grid, 256, C::SMEM, stream>>>(tmA, tmB, tmE, tmY, Y, ldy, bias, scale, static_cast<int>(M),
                                       static_cast<int>(N), static_cast<int>(K), err);
  return launch_status();
}

spg_status validate_common(const void* X, int64_t ldx, const void* Wv, const uint8_t* meta, void* Y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, int es, int out_es, int kstep) {
  if (!X || !Wv || !meta || !Y) return SPG_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || ldx < K || ldy < N) return SPG_ERR_INVALID_ARG;
  if (K % kstep || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return SPG_ERR_UNSUPPORTED_SHAPE;
  if ((N + 127) / 128 * ((M + 31) / 32) >= (int64_t(1) << 31)) return SPG_ERR_UNSUPPORTED_SHAPE;
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
  spg_status st = validate_common(X, ldx, Wv, meta, Y, ldy, M, N, K, 2, 2, 128);
  if (st != SPG_OK) return st;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SPG_F16)
    return launch<false, false, 128, 4, OUT_F16>(X, ldx, Wv, meta, bias, nullptr, Y, ldy, M, N, K, s);
  return launch<false, true, 128, 4, OUT_BF16>(X, ldx, Wv, meta, bias, nullptr, Y, ldy, M, N, K, s);
}

spg_status spgemm_24_s8(const int8_t* X, int64_t ldx, const int8_t* Wv, const uint8_t* meta, const float* scale,
                        const void* bias, void* Y, int64_t ldy, int out_mode, int64_t M, int64_t N, int64_t K,
                        spg_stream_t stream) {
  using namespace spg;
  using namespace spg::gemm24;
  if (out_mode != SPG_OUT_F16 && out_mode != SPG_OUT_S32) return SPG_ERR_INVALID_ARG;
  const int out_es = out_mode == SPG_OUT_S32 ? 4 : 2;
  spg_status st = validate_common(X, ldx, Wv, meta, Y, ldy, M, N, K, 1, out_es, 256);
  if (st != SPG_OK) return st;
  if (out_mode == SPG_OUT_F16 && !scale) return SPG_ERR_INVALID_ARG;
  if (scale && !aligned(scale, 4)) return SPG_ERR_MISALIGNED;
  if (bias && !aligned(bias, 2)) return SPG_ERR_MISALIGNED;
  st = check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (out_mode == SPG_OUT_S32)
    return launch<true, false, 128, 3, OUT_S32>(X, ldx, Wv, meta, nullptr, nullptr, Y, ldy, M, N, K, s);
  return launch<true, false, 128, 4, OUT_F16>(X, ldx, Wv, meta, bias, scale, Y, ldy, M, N, K, s);
}

}  // extern "C"
