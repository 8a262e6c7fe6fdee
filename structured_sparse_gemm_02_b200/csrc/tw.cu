// Tile-wise sparsity ("Accelerating Sparse DNN Models without Hardware-Support
// via Tile-Wise Sparsity", slides "Tile-Wise Sparsity", "Re-organize",
// "Run-time", "Transpose"): descriptor sizing.
#include <cuda_runtime.h>

#include <cstdint>

#include "host.cuh"
#include "spgemm.h"

namespace spg {
namespace tw {

spg_status query(int64_t N, int64_t K, int32_t G, int64_t n_pruned, const int32_t* kpt, spg_tw_sizes* out) {
  if (!kpt || !out) return SPG_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || n_pruned < 0 || n_pruned >= N) return SPG_ERR_INVALID_ARG;
  if (G != 128 || K % 64 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return SPG_ERR_UNSUPPORTED_SHAPE;
  const int64_t Nk = N - n_pruned;
  const int64_t T = (Nk + G - 1) / G;
  int64_t kofs = 0;
  for (int64_t t = 0; t < T; ++t) {
    if (kpt[t] < 1 || kpt[t] > K) return SPG_ERR_INVALID_ARG;
    kofs += (kpt[t] + 63) / 64 * 64;
  }
  out->N = N;
  out->K = K;
  out->Nk = Nk;
  out->G = G;
  out->T = static_cast<int32_t>(T);
  out->offsetk_len = kofs;
  out->wc_elems = kofs * G;
  return SPG_OK;
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
  return static_cast<size_t>((M * K * 2 + 255) / 256 * 256);
}

spg_status tw_reorganize(const void* W, int64_t ldw, int64_t n_pruned, const int32_t* k_per_tile,
                         const spg_tw_desc* desc, spg_stream_t stream) {
  (void)W; (void)ldw; (void)n_pruned; (void)k_per_tile; (void)desc; (void)stream;
  return SPG_ERR_UNSUPPORTED_SHAPE;
}

spg_status spgemm_tw_f16(const void* X, int64_t ldx, int x_layout, const spg_tw_desc* desc, void* Y, int64_t ldy,
                         int64_t M, void* workspace, size_t ws_bytes, spg_stream_t stream) {
  (void)X; (void)ldx; (void)x_layout; (void)desc; (void)Y; (void)ldy; (void)M; (void)workspace; (void)ws_bytes;
  (void)stream;
  return SPG_ERR_UNSUPPORTED_SHAPE;
}

}  // extern "C"
