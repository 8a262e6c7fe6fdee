// 2:4 magnitude pruning and compression ("Boost Vision Transformer with
// GPU-Friendly Sparsity and Quantization", Abstract: dense weights pruned to
// the 2:4 pattern along the reduction dimension).
//
// Selection rule, per group of 4 consecutive weights along K: position i is
// kept when fewer than two other positions beat it, where j beats i if
// |w_j| > |w_i|, or |w_j| == |w_i| and j < i.  Magnitudes compare exactly as
// integers: the fp16/bf16 bit pattern with the sign cleared, |q| for int8.
// Memory-bound, offline: one thread per group (prune) or per pair of groups
// (compress), grid-stride loops sized to the SM count.
#include <cuda_runtime.h>

#include <cstdint>

#include "host.cuh"
#include "spgemm.h"

namespace spg {
namespace {

template <int ES>
struct Group;  // 4 elements of ES bytes

template <>
struct Group<2> {
  using Raw = uint2;  // 4 x 16-bit
  __device__ static void mags(const Raw& r, int (&m)[4]) {
    m[0] = r.x & 0x7FFF;
    m[1] = (r.x >> 16) & 0x7FFF;
    m[2] = r.y & 0x7FFF;
    m[3] = (r.y >> 16) & 0x7FFF;
  }
  __device__ static uint32_t elem(const Raw& r, int i) {
    const uint32_t w = i < 2 ? r.x : r.y;
    return (w >> (16 * (i & 1))) & 0xFFFFu;
  }
  __device__ static Raw mask(const Raw& r, unsigned keep) {
    Raw o;
    o.x = (keep & 1 ? (r.x & 0xFFFFu) : 0u) | (keep & 2 ? (r.x & 0xFFFF0000u) : 0u);
    o.y = (keep & 4 ? (r.y & 0xFFFFu) : 0u) | (keep & 8 ? (r.y & 0xFFFF0000u) : 0u);
    return o;
  }
};

template <>
struct Group<1> {
  using Raw = uint32_t;  // 4 x int8
  __device__ static void mags(const Raw& r, int (&m)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int v = static_cast<int8_t>((r >> (8 * i)) & 0xFF);
      m[i] = v < 0 ? -v : v;
    }
  }
  __device__ static uint32_t elem(const Raw& r, int i) { return (r >> (8 * i)) & 0xFFu; }
  __device__ static Raw mask(const Raw& r, unsigned keep) {
    Raw o = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (keep & (1u << i)) o |= r & (0xFFu << (8 * i));
    return o;
  }
};

// Bit i of the result is set when position i of the group is kept.
__device__ __forceinline__ unsigned keep_mask(const int (&m)[4]) {
  unsigned keep = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int beaten = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j != i) beaten += (m[j] > m[i]) || (m[j] == m[i] && j < i);
    if (beaten < 2) keep |= 1u << i;
  }
  return keep;
}

template <int ES>
__global__ void prune24_kernel(const uint8_t* __restrict__ W, int64_t ldw_b, uint8_t* __restrict__ Wm,
                               int64_t ldwm_b, int64_t N, int64_t G4) {
  using GT = Group<ES>;
  using Raw = typename GT::Raw;
  const int64_t total = N * G4;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = i / G4, g = i - n * G4;
    const Raw r = *reinterpret_cast<const Raw*>(W + n * ldw_b + g * 4 * ES);
    int m[4];
    GT::mags(r, m);
    *reinterpret_cast<Raw*>(Wm + n * ldwm_b + g * 4 * ES) = GT::mask(r, keep_mask(m));
  }
}

// One thread per pair of groups: 4 kept values and one metadata byte.
template <int ES>
__global__ void compress24_kernel(const uint8_t* __restrict__ W, int64_t ldw_b, uint8_t* __restrict__ Wv,
                                  uint8_t* __restrict__ meta, int64_t N, int64_t K) {
  using GT = Group<ES>;
  using Raw = typename GT::Raw;
  const int64_t pairs = K / 8;
  const int64_t total = N * pairs;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t n = i / pairs, b = i - n * pairs;
    const uint8_t* src = W + n * ldw_b + b * 8 * ES;
    uint32_t vals[4];
    uint32_t byte = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const Raw r = *reinterpret_cast<const Raw*>(src + h * 4 * ES);
      int m[4];
      GT::mags(r, m);
      const unsigned keep = keep_mask(m);
      int i0 = -1, i1 = -1;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (keep & (1u << q)) {
          if (i0 < 0) i0 = q; else i1 = q;
        }
      vals[2 * h] = GT::elem(r, i0);
      vals[2 * h + 1] = GT::elem(r, i1);
      byte |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * h);
    }
    uint8_t* dst = Wv + (n * (K / 2) + b * 4) * ES;
    if constexpr (ES == 2) {
      reinterpret_cast<uint32_t*>(dst)[0] = vals[0] | (vals[1] << 16);
      reinterpret_cast<uint32_t*>(dst)[1] = vals[2] | (vals[3] << 16);
    } else {
      *reinterpret_cast<uint32_t*>(dst) = vals[0] | (vals[1] << 8) | (vals[2] << 16) | (vals[3] << 24);
    }
    meta[n * (K / 8) + b] = static_cast<uint8_t>(byte);
  }
}

int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = int64_t(sms) * 16;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

int esize_of(spg_dtype d) { return d == SPG_S8 ? 1 : 2; }

}  // namespace
}  // namespace spg

extern "C" {

spg_status sparse_prune_24(const void* W, int64_t ldw, void* Wm, int64_t ldwm, int64_t N, int64_t K,
                           spg_dtype dtype, spg_stream_t stream) {
  using namespace spg;
  if (dtype != SPG_F16 && dtype != SPG_BF16 && dtype != SPG_S8) return SPG_ERR_INVALID_ARG;
  if (N < 0 || K < 0 || ldw < K || ldwm < K) return SPG_ERR_INVALID_ARG;
  if (K % 4) return SPG_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return SPG_OK;
  if (!W || !Wm) return SPG_ERR_INVALID_ARG;
  const int es = esize_of(dtype);
  const int al = 4 * es;
  if (!aligned(W, al) || !aligned(Wm, al) || (ldw * es) % al || (ldwm * es) % al) return SPG_ERR_MISALIGNED;
  if (W == Wm && ldw != ldwm) return SPG_ERR_INVALID_ARG;
  spg_status st = check_device();
  if (st != SPG_OK) return st;
  const int64_t work = N * (K / 4);
  const int threads = 256;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (es == 2)
    prune24_kernel<2><<<grid_for(work, threads), threads, 0, s>>>(
        static_cast<const uint8_t*>(W), ldw * 2, static_cast<uint8_t*>(Wm), ldwm * 2, N, K / 4);
  else
    prune24_kernel<1><<<grid_for(work, threads), threads, 0, s>>>(
        static_cast<const uint8_t*>(W), ldw, static_cast<uint8_t*>(Wm), ldwm, N, K / 4);
  return launch_status();
}

spg_status sparse_compress_24(const void* W, int64_t ldw, void* Wv, uint8_t* meta, int64_t N, int64_t K,
                              spg_dtype dtype, spg_stream_t stream) {
  using namespace spg;
  if (dtype != SPG_F16 && dtype != SPG_BF16 && dtype != SPG_S8) return SPG_ERR_INVALID_ARG;
  if (N < 0 || K < 0 || ldw < K) return SPG_ERR_INVALID_ARG;
  if (K % 8) return SPG_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return SPG_OK;
  if (!W || !Wv || !meta) return SPG_ERR_INVALID_ARG;
  const int es = esize_of(dtype);
  if (!aligned(W, 4 * es) || (ldw * es) % (4 * es) || !aligned(Wv, 4) || !aligned(meta, 4))
    return SPG_ERR_MISALIGNED;
  spg_status st = check_device();
  if (st != SPG_OK) return st;
  const int64_t work = N * (K / 8);
  const int threads = 256;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (es == 2)
    compress24_kernel<2><<<grid_for(work, threads), threads, 0, s>>>(
        static_cast<const uint8_t*>(W), ldw * 2, static_cast<uint8_t*>(Wv), meta, N, K);
  else
    compress24_kernel<1><<<grid_for(work, threads), threads, 0, s>>>(
        static_cast<const uint8_t*>(W), ldw, static_cast<uint8_t*>(Wv), meta, N, K);
  return launch_status();
}

}  // extern "C"
