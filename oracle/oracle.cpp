// Plain CPU C++ oracle for the pruned-weight linear layer Y = X . W^T.
//
// TEST INFRASTRUCTURE: loaded only by tests/, __graft_entry__.smoke() and the
// CPU-baseline legs of bench.py (through oracle/native.py).  It shares no code
// with the CUDA library and with the numpy oracle beside it; both are checked
// against each other and against the pinned fixtures in tests/.
//
// What it states, each step the plain definition:
//  * 2:4 selection, compression and decompression ("Boost Vision Transformer
//    with GPU-Friendly Sparsity and Quantization", Abstract: 2 of every 4
//    consecutive weights along K are kept).  Reading where the abstract is
//    silent: keep the two largest magnitudes, the lower index first among
//    equal ones.  Here that is done by picking the largest element of the
//    group, then the largest of the other three.
//  * the dense product over the explicitly masked weight in fp64 (fp16 / bf16
//    inputs), and in exact integers (int8 inputs) followed by the fp32
//    dequantisation y = fp16(fp32(acc) * scale[n] [+ fp32(bias[n])]);
//  * the fixed-point epilogue of the int8 chain (GELU in a fixed fp32
//    operation order, then the int8 quantiser) and GELU in fp64;
//  * the tile-wise reorganisation with exact integer norms, and the expansion
//    back to a dense weight ("Accelerating Sparse DNN
//    Models without Hardware-Support via Tile-Wise Sparsity", slides
//    "Re-organize" and "Run-time": C[offsetn[n]] += A[offsetk[k]] * B) and
//    its fp64 product.
//
// Every output element is one sequential sum over k in index order, so the
// result does not depend on the thread count (OpenMP splits output rows).
// Build: g++ -O3 -ffp-contract=off -fopenmp -shared -fPIC (oracle/native.py).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

enum { F16 = 0, BF16 = 1, S8 = 2, F32 = 3 };

// fp16 bits -> exact value: (-1)^s * m * 2^e, m = 1024 + frac and e = exp - 25
// for normal numbers, m = frac and e = -24 for subnormals.
double f16_value(uint16_t h) {
  const int s = h >> 15, ex = (h >> 10) & 0x1F, fr = h & 0x3FF;
  const double m = ex ? double(1024 + fr) : double(fr);
  const int e = ex ? ex - 25 : -24;
  const double v = std::ldexp(m, e);
  return s ? -v : v;
}

// bf16 bits are the upper half of an fp32.
double bf16_value(uint16_t b) {
  const uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

// fp32 -> fp16 bits, round to nearest even (finite inputs; overflow to Inf).
uint16_t f32_to_f16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint16_t sign = uint16_t((u >> 16) & 0x8000u);
  const double a = std::fabs(double(f));
  if (a == 0.0) return sign;
  // the fp16 grid spacing around a: 2^-24 below 2^-14, else 2^(floor(log2 a) - 10)
  int e2;
  std::frexp(a, &e2);  // a = f * 2^e2 with f in [0.5, 1)
  const int step_exp = (e2 - 1) < -14 ? -24 : (e2 - 1) - 10;
  const double q = a / std::ldexp(1.0, step_exp);  // exact: a power-of-two scaling
  double r = std::floor(q);
  const double frac = q - r;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
  const double v = std::ldexp(r, step_exp);  // the rounded magnitude
  if (v > 65504.0) return uint16_t(sign | 0x7C00);  // rounded past the largest finite fp16
  // encode v
  if (v < std::ldexp(1.0, -14)) return uint16_t(sign | uint16_t(v / std::ldexp(1.0, -24)));
  int ev;
  const double mv = std::frexp(v, &ev);  // v = mv * 2^ev, mv in [0.5, 1)
  const int ex = ev - 1 + 15;
  const int fr = int(mv * 2048.0) - 1024;
  return uint16_t(sign | (ex << 10) | fr);
}

double value(const void* A, int dtype, int64_t i) {
  switch (dtype) {
    case F16: return f16_value(static_cast<const uint16_t*>(A)[i]);
    case BF16: return bf16_value(static_cast<const uint16_t*>(A)[i]);
    case S8: return double(static_cast<const int8_t*>(A)[i]);
    default: return double(static_cast<const float*>(A)[i]);
  }
}

// |w| as an integer in the order of |w|: the bit pattern without its sign for
// fp16 / bf16 (finite values), |q| for int8.
int magnitude(const void* W, int dtype, int64_t i) {
  if (dtype == S8) {
    const int q = static_cast<const int8_t*>(W)[i];
    return q < 0 ? -q : q;
  }
  return static_cast<const uint16_t*>(W)[i] & 0x7FFF;
}

int esize(int dtype) { return dtype == S8 ? 1 : dtype == F32 ? 4 : 2; }

// The two kept positions of the group starting at W[base]: the first largest
// magnitude, then the first largest of the remaining three; returned ascending.
void choose2(const void* W, int dtype, int64_t base, int* i0, int* i1) {
  int a = 0;
  for (int j = 1; j < 4; ++j)
    if (magnitude(W, dtype, base + j) > magnitude(W, dtype, base + a)) a = j;
  int b = -1;
  for (int j = 0; j < 4; ++j) {
    if (j == a) continue;
    if (b < 0 || magnitude(W, dtype, base + j) > magnitude(W, dtype, base + b)) b = j;
  }
  *i0 = a < b ? a : b;
  *i1 = a < b ? b : a;
}

void copy_elem(const void* src, int64_t si, void* dst, int64_t di, int es) {
  std::memcpy(static_cast<uint8_t*>(dst) + di * es, static_cast<const uint8_t*>(src) + si * es, es);
}

}  // namespace

extern "C" {

// 2:4 masked weight: Wm = W with the two unselected elements of every group of
// 4 along K set to +0 (bit pattern 0).  W, Wm [N][K] contiguous.
int orc_prune24(const void* W, int64_t N, int64_t K, int dtype, void* Wm) {
  if (K % 4 || dtype < F16 || dtype > S8) return 1;
  const int es = esize(dtype);
  std::memset(Wm, 0, size_t(N * K * es));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < K / 4; ++g) {
      int i0, i1;
      const int64_t base = n * K + 4 * g;
      choose2(W, dtype, base, &i0, &i1);
      copy_elem(W, base + i0, Wm, base + i0, es);
      copy_elem(W, base + i1, Wm, base + i1, es);
    }
  return 0;
}

// 2:4 compressed form: Wv[n][2g + s] = W[n][4g + i_s] (i0 < i1), and the 4-bit
// code i0 | i1 << 2 of group g in meta[n][g / 2] (even g: low nibble).
int orc_compress24(const void* W, int64_t N, int64_t K, int dtype, void* Wv, uint8_t* meta) {
  if (K % 8 || dtype < F16 || dtype > S8) return 1;
  const int es = esize(dtype);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t b = 0; b < K / 8; ++b) meta[n * (K / 8) + b] = 0;
    for (int64_t g = 0; g < K / 4; ++g) {
      int i0, i1;
      choose2(W, dtype, n * K + 4 * g, &i0, &i1);
      copy_elem(W, n * K + 4 * g + i0, Wv, n * (K / 2) + 2 * g, es);
      copy_elem(W, n * K + 4 * g + i1, Wv, n * (K / 2) + 2 * g + 1, es);
      const uint8_t code = uint8_t(i0 | (i1 << 2));
      meta[n * (K / 8) + g / 2] |= uint8_t(g % 2 ? code << 4 : code);
    }
  }
  return 0;
}

// Inverse of orc_compress24: the masked [N][K] weight.
int orc_decompress24(const void* Wv, const uint8_t* meta, int64_t N, int64_t K, int dtype, void* Wm) {
  if (K % 8 || dtype < F16 || dtype > S8) return 1;
  const int es = esize(dtype);
  std::memset(Wm, 0, size_t(N * K * es));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t g = 0; g < K / 4; ++g) {
      const uint8_t byte = meta[n * (K / 8) + g / 2];
      const int code = g % 2 ? byte >> 4 : byte & 0xF;
      copy_elem(Wv, n * (K / 2) + 2 * g, Wm, n * K + 4 * g + (code & 3), es);
      copy_elem(Wv, n * (K / 2) + 2 * g + 1, Wm, n * K + 4 * g + (code >> 2), es);
    }
  return 0;
}

// Y[i][n] = sum_k X[rows[i]][k] * Wd[n][k] (+ bias[n]) in fp64, k ascending.
// X [M][ldx] of xdtype (fp16, bf16 or fp32); Wd [N][K] fp64; bias [N] fp64 or
// NULL; rows NULL means every row (nrows == M).
int orc_gemm_f64(const void* X, int64_t ldx, int xdtype, int64_t M, int64_t K, const double* Wd, int64_t N,
                 const double* bias, const int64_t* rows, int64_t nrows, double* Y) {
  if (xdtype == S8) return 1;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t i = 0; i < nrows; ++i) {
    const int64_t r = rows ? rows[i] : i;
    std::vector<double> x(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) x[size_t(k)] = value(X, xdtype, r * ldx + k);
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      const double* w = Wd + n * K;
      for (int64_t k = 0; k < K; ++k) acc += x[size_t(k)] * w[k];
      Y[i * N + n] = bias ? acc + bias[n] : acc;
    }
  }
  (void)M;
  return 0;
}

// fp16 / bf16 2:4 layer: the dense fp64 product over decompress(Wv, meta).
// bias [N] in the same dtype or NULL.
int orc_gemm24_f64(const void* X, int64_t M, int64_t K, const void* Wv, const uint8_t* meta, int64_t N,
                   const void* bias, int dtype, const int64_t* rows, int64_t nrows, double* Y) {
  if (dtype != F16 && dtype != BF16) return 1;
  std::vector<uint16_t> Wm(size_t(N * K));
  if (orc_decompress24(Wv, meta, N, K, dtype, Wm.data())) return 1;
  std::vector<double> Wd(static_cast<size_t>(N * K)), b(static_cast<size_t>(N));
  for (int64_t i = 0; i < N * K; ++i) Wd[size_t(i)] = value(Wm.data(), dtype, i);
  for (int64_t n = 0; bias && n < N; ++n) b[size_t(n)] = value(bias, dtype, n);
  return orc_gemm_f64(X, K, dtype, M, K, Wd.data(), N, bias ? b.data() : nullptr, rows, nrows, Y);
}

// int8 2:4 layer, exact: acc[i][n] = sum_k X[rows[i]][k] * Wm[n][k] in int64.
int orc_gemm24_s8(const int8_t* X, int64_t M, int64_t K, const int8_t* Wv, const uint8_t* meta, int64_t N,
                  const int64_t* rows, int64_t nrows, int64_t* acc) {
  std::vector<int8_t> Wm(size_t(N * K));
  if (orc_decompress24(Wv, meta, N, K, S8, Wm.data())) return 1;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t i = 0; i < nrows; ++i) {
    const int64_t r = rows ? rows[i] : i;
    for (int64_t n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += int64_t(X[r * K + k]) * int64_t(Wm[size_t(n * K + k)]);
      acc[i * N + n] = s;
    }
  }
  (void)M;
  return 0;
}

// int8 epilogue: Y[i][n] = fp16_rn( fp32(acc) *rn scale[n] [ +rn fp32(bias[n]) ] ),
// each step one IEEE fp32 operation (built without contraction into FMA).
int orc_dequant_s8(const int64_t* acc, int64_t rows, int64_t N, const float* scale, const uint16_t* bias,
                   uint16_t* Y) {
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t n = 0; n < N; ++n) {
      float v = float(acc[i * N + n]) * scale[n];
      if (bias) v = v + float(f16_value(bias[n]));
      Y[i * N + n] = f32_to_f16_rne(v);
    }
  return 0;
}

// The activation between the two layers of a ViT MLP block (the models the
// 2:4 scheme compresses; the pages do not spell it out): GELU(v) = v Phi(v) =
// 0.5 v (1 + erf(v / sqrt 2)), exact form, in fp64 with the C library's erf.
int orc_gelu_f64(const double* v, int64_t n, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = 0.5 * v[i] * (1.0 + std::erf(v[i] / std::sqrt(2.0)));
  return 0;
}

// The fixed-point epilogue that feeds the next int8 layer, every step one IEEE
// fp32 operation in this order (built without FMA contraction):
//   v = fp32(acc) * scale[n]  [ + fp32(bias[n]) ]
//   [ v = GELU(v) with erf from Abramowitz & Stegun 7.1.28:
//       u = v * 0.70710677; a = min(|u|, 4);
//       p = ((((((a6 a + a5) a + a4) a + a3) a + a2) a + a1) a) + 1;
//       p16 = p^16 by four squarings; r = 1 / p16 by three Newton steps
//       r = r (2 - p16 r) from the fp32 whose bits are 0x7EF00000 - bits(p16);
//       erf(u) = sign(u) (1 - r); GELU = (0.5 v) (1 + erf(u)) ]
//   q = clamp(rne(v * qscale), -127, 127)
int orc_quantize_s8(const int64_t* acc, int64_t rows, int64_t N, const float* scale, const uint16_t* bias,
                    float qscale, int gelu, int8_t* Yq) {
  const float a1 = 0.0705230784f, a2 = 0.0422820123f, a3 = 0.0092705272f, a4 = 0.0001520143f,
              a5 = 0.0002765672f, a6 = 0.0000430638f;
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t n = 0; n < N; ++n) {
      float v = float(acc[i * N + n]) * scale[n];
      if (bias) v = v + float(f16_value(bias[n]));
      if (gelu) {
        const float u = v * 0.70710677f;
        const float a = std::fabs(u) < 4.0f ? std::fabs(u) : 4.0f;
        float h = a6;
        h = h * a + a5;
        h = h * a + a4;
        h = h * a + a3;
        h = h * a + a2;
        h = h * a + a1;
        const float p = h * a + 1.0f;
        const float p2 = p * p, p4 = p2 * p2, p8 = p4 * p4, p16 = p8 * p8;
        uint32_t bits;
        std::memcpy(&bits, &p16, 4);
        bits = 0x7EF00000u - bits;
        float r;
        std::memcpy(&r, &bits, 4);
        for (int it = 0; it < 3; ++it) r = r * (2.0f - p16 * r);
        const float e = 1.0f - r;
        v = (0.5f * v) * (1.0f + (u < 0.0f ? -e : e));
      }
      const float t = v * qscale;
      // round to nearest, ties to even, then clamp
      float rq = std::floor(t);
      const float fr = t - rq;
      if (fr > 0.5f || (fr == 0.5f && std::fmod(rq, 2.0f) != 0.0f)) rq += 1.0f;
      Yq[i * N + n] = int8_t(rq > 127.0f ? 127 : rq < -127.0f ? -127 : int(rq));
    }
  return 0;
}

// fp32 -> fp16 bits (round to nearest even), exposed for its own test.
int orc_f32_to_f16(const float* x, int64_t n, uint16_t* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = f32_to_f16_rne(x[i]);
  return 0;
}

// Tile-wise reorganisation ("Accelerating Sparse DNN Models without
// Hardware-Support via Tile-Wise Sparsity", slides "Tile-Wise Sparsity",
// "Re-organize", "Preprocessed"), with the readings where the slides are
// silent: columns of B = W^T (rows n of W) are pruned globally by smallest L2
// norm (equal norms: the lower n is pruned first); the kept columns, ascending
// (offsetn), form tiles of G consecutive kept columns, the last one shorter;
// tile t keeps its k_t rows k of largest L2 norm over its own columns (equal
// norms: the lower k is kept), ascending (offsetk).  Norms are exact: every
// fp16 value is m * 2^e with e >= -24, so w^2 * 2^48 = m^2 * 2^(2e + 48) is an
// integer, and the sums are kept in unsigned 128-bit integers.
// Output in the library's descriptor layout: offsetn [N - n_pruned],
// tile_kofs [T + 1] (prefix sums of k_t rounded up to 64), offsetk
// [tile_kofs[T]] (padded with the tile's last kept k) and Wc fp16 bits
// [tile_kofs[T] / 64][G][64] (block b of tile t, element [j][c] = W[offsetn[t G
// + j]][offsetk[tile_kofs[t] + 64 b + c]], +0 in unused slots).
int orc_tw_reorganize(const uint16_t* W, int64_t N, int64_t K, int G, int64_t n_pruned, const int32_t* k_per_tile,
                      int32_t* offsetn, int32_t* tile_kofs, int32_t* offsetk, uint16_t* Wc) {
  typedef unsigned __int128 u128;
  if (G != 128 || n_pruned < 0 || n_pruned >= N) return 1;
  auto sq = [&](int64_t n, int64_t k) -> u128 {
    const uint16_t h = W[n * K + k];
    const int ex = (h >> 10) & 0x1F, fr = h & 0x3FF;
    if (ex == 0x1F) return 0;  // Inf / NaN are outside the contract
    const u128 m = ex ? u128(1024 + fr) : u128(fr);
    const int e = ex ? ex - 25 : -24;
    return (m * m) << (2 * e + 48);
  };
  // column keys and the global prune
  std::vector<u128> ckey(static_cast<size_t>(N), 0);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) ckey[size_t(n)] += sq(n, k);
  std::vector<int64_t> order(static_cast<size_t>(N));
  for (int64_t n = 0; n < N; ++n) order[size_t(n)] = n;
  std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
    return ckey[size_t(a)] != ckey[size_t(b)] ? ckey[size_t(a)] < ckey[size_t(b)] : a < b;
  });
  std::vector<char> pruned(static_cast<size_t>(N), 0);
  for (int64_t i = 0; i < n_pruned; ++i) pruned[size_t(order[size_t(i)])] = 1;
  int64_t Nk = 0;
  for (int64_t n = 0; n < N; ++n)
    if (!pruned[size_t(n)]) offsetn[Nk++] = int32_t(n);
  const int64_t T = (Nk + G - 1) / G;
  tile_kofs[0] = 0;
  for (int64_t t = 0; t < T; ++t) {
    if (k_per_tile[t] < 1 || k_per_tile[t] > K) return 1;
    tile_kofs[t + 1] = tile_kofs[t] + (k_per_tile[t] + 63) / 64 * 64;
  }
  std::memset(Wc, 0, size_t(tile_kofs[T]) * size_t(G) * 2);
  // per tile: row keys over the tile's columns, top k_t rows, condensed values
  for (int64_t t = 0; t < T; ++t) {
    const int64_t j0 = t * G, Gt = (Nk - j0) < G ? Nk - j0 : G;
    std::vector<u128> rkey(static_cast<size_t>(K), 0);
    for (int64_t j = 0; j < Gt; ++j)
      for (int64_t k = 0; k < K; ++k) rkey[size_t(k)] += sq(offsetn[j0 + j], k);
    std::vector<int64_t> rk(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) rk[size_t(k)] = k;
    std::sort(rk.begin(), rk.end(), [&](int64_t a, int64_t b) {
      return rkey[size_t(a)] != rkey[size_t(b)] ? rkey[size_t(a)] > rkey[size_t(b)] : a < b;
    });
    const int64_t kt = k_per_tile[t];
    std::sort(rk.begin(), rk.begin() + kt);
    const int64_t base = tile_kofs[t];
    for (int64_t i = 0; i < tile_kofs[t + 1] - base; ++i) offsetk[base + i] = int32_t(rk[size_t(i < kt ? i : kt - 1)]);
    for (int64_t j = 0; j < Gt; ++j)
      for (int64_t i = 0; i < kt; ++i) {
        const int64_t blk = base / 64 + i / 64, c = i % 64;
        Wc[(blk * G + j) * 64 + c] = W[int64_t(offsetn[j0 + j]) * K + rk[size_t(i)]];
      }
  }
  return 0;
}

// Tile-wise expansion to a dense fp64 Wd [N][K]: zero except, for tile t,
// kept column j < G_t and kept row i < k_t,
//   Wd[offsetn[t*G + j]][offsetk[tile_kofs[t] + i]] = Wc of (t, j, i),
// with Wc in the library's block layout: block b of tile t (64 kept rows) at
// blk = tile_kofs[t] / 64 + b holds element [j][c] at
// Wc[(blk * G + j) * 64 + c] for kept row i = 64 b + c.  Wc holds fp16 bits
// (wdtype 0) or fp32 (wdtype 3, the fp32 library's k-major blocks
// Wc32[(blk * 64 + c) * G + j]).
int orc_tw_expand(int64_t N, int64_t K, int G, int64_t Nk, int T, const int32_t* offsetn, const int32_t* tile_kofs,
                  const int32_t* k_per_tile, const int32_t* offsetk, const void* Wc, int wdtype, double* Wd) {
  if (G != 128 || (wdtype != F16 && wdtype != F32)) return 1;
  for (int64_t i = 0; i < N * K; ++i) Wd[i] = 0.0;
  for (int t = 0; t < T; ++t) {
    const int64_t Gt = (Nk - int64_t(t) * G) < G ? Nk - int64_t(t) * G : G;
    for (int64_t j = 0; j < Gt; ++j) {
      const int64_t n = offsetn[t * G + j];
      for (int64_t i = 0; i < k_per_tile[t]; ++i) {
        const int64_t k = offsetk[tile_kofs[t] + i];
        const int64_t blk = tile_kofs[t] / 64 + i / 64, c = i % 64;
        const int64_t idx = wdtype == F16 ? (blk * G + j) * 64 + c : (blk * 64 + c) * G + j;
        Wd[n * K + k] = value(Wc, wdtype, idx);
      }
    }
  }
  return 0;
}

}  // extern "C"
