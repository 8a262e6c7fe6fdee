// Library-wide entry points (version, status strings, device error word) and
// the host helpers declared in host.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "host.cuh"
#include "sm100.cuh"
#include "spgemm.h"

namespace spg {

__device__ uint32_t g_error_word;
// The value spg_check_device_error() took out of g_error_word, for the host to read.
__device__ uint32_t g_error_taken;

namespace {
constexpr int kMaxDevices = 64;
int g_dev_ok[kMaxDevices];           // 0 unknown, 1 ok, -1 unsupported
uint32_t* g_err_ptr[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}
}  // namespace

spg_status check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPG_ERR_CUDA;
  if (dev_out) *dev_out = dev;
  if (dev < 0 || dev >= kMaxDevices) return SPG_ERR_UNSUPPORTED_DEVICE;
  int st = __atomic_load_n(&g_dev_ok[dev], __ATOMIC_ACQUIRE);
  if (st == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return SPG_ERR_CUDA;
    st = (major == 10 && minor == 0) ? 1 : -1;
    __atomic_store_n(&g_dev_ok[dev], st, __ATOMIC_RELEASE);
  }
  return st == 1 ? SPG_OK : SPG_ERR_UNSUPPORTED_DEVICE;
}

int sm_count() {
  static int cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = __atomic_load_n(&cached[dev], __ATOMIC_ACQUIRE);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    __atomic_store_n(&cached[dev], v, __ATOMIC_RELEASE);
  }
  return v;
}

uint32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_err_ptr[dev];
}

bool make_tmap_2d(CUtensorMap* map, const void* base, int esize, uint64_t cols, uint64_t rows,
                  uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
  return make_tmap_2d_swz(map, base, esize, cols, rows, pitch_bytes, box_cols, box_rows, swizzle128 ? 128 : 0);
}

bool make_tmap_2d_swz(CUtensorMap* map, const void* base, int esize, uint64_t cols, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return false;
  CUtensorMapDataType dt = esize == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                           : esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                        : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                        : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One thread waits, with the library's bounded wait and the given limit, on
// an mbarrier that nothing ever arrives on: the wait gives up, records
// ERR_WAIT_SELFTEST in the error word and the kernel returns normally.
__global__ void selftest_wait_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, ERR_WAIT_SELFTEST, limit_ns);
}

// Takes the error word and clears it in one atomic step, so a bit that a
// kernel on another stream sets at the same moment is either taken now or
// left for the next check, never lost.
__global__ void take_error_word_kernel() { g_error_taken = atomicExch(&g_error_word, 0u); }

}  // namespace spg

extern "C" {

int spg_version(void) { return 1 * 10000 + 0 * 100 + 0; }

const char* spg_status_string(spg_status s) {
  switch (s) {
    case SPG_OK: return "SPG_OK";
    case SPG_ERR_INVALID_ARG: return "SPG_ERR_INVALID_ARG";
    case SPG_ERR_UNSUPPORTED_SHAPE: return "SPG_ERR_UNSUPPORTED_SHAPE";
    case SPG_ERR_MISALIGNED: return "SPG_ERR_MISALIGNED";
    case SPG_ERR_UNSUPPORTED_DEVICE: return "SPG_ERR_UNSUPPORTED_DEVICE";
    case SPG_ERR_CUDA: return "SPG_ERR_CUDA";
    case SPG_ERR_TIMEOUT: return "SPG_ERR_TIMEOUT";
  }
  return "SPG_ERR_UNKNOWN";
}

spg_status spg_check_device_error(spg_stream_t stream, uint32_t* bits) {
  if (bits) *bits = 0;
  spg_status st = spg::check_device();
  if (st != SPG_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  spg::take_error_word_kernel<<<1, 1, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return SPG_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SPG_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, spg::g_error_taken, sizeof(v)) != cudaSuccess) return SPG_ERR_CUDA;
  if (bits) *bits = v;
  return v ? SPG_ERR_TIMEOUT : SPG_OK;
}

spg_status spg_selftest_bounded_wait(int64_t limit_ns, spg_stream_t stream) {
  if (limit_ns <= 0 || limit_ns > 10ll * 1000 * 1000 * 1000) return SPG_ERR_INVALID_ARG;
  spg_status st = spg::check_device();
  if (st != SPG_OK) return st;
  uint32_t* err = spg::device_error_word();
  if (!err) return SPG_ERR_CUDA;
  spg::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err, uint64_t(limit_ns));
  return spg::launch_status();
}

}  // extern "C"
