// Host-side helpers shared by the entry points: device checks, the device
// error word, tensor-map encoding through the driver entry point, and
// argument validation shorthands.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "spgemm.h"

namespace spg {

// Current device is compute capability 10.0 (result cached per device).
spg_status check_device(int* dev_out = nullptr);

// Device address of the library's error word on the current device.
uint32_t* device_error_word();

// Number of SMs of the current device (cached per device; 148 if the query fails).
int sm_count();

// 2-D tiled tensor map over a row-major matrix of `rows` x `cols` elements of
// `esize` bytes with a row pitch of `pitch_bytes`; the box is box_cols x
// box_rows.  Returns false if the driver rejects the description.
bool make_tmap_2d(CUtensorMap* map, const void* base, int esize, uint64_t cols, uint64_t rows,
                  uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128);

// As make_tmap_2d with the shared-memory swizzle given in bytes (0, 32, 64 or 128).
bool make_tmap_2d_swz(CUtensorMap* map, const void* base, int esize, uint64_t cols, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch `kernel` on `stream` with programmatic stream serialisation allowed
// (the kernel calls griddep_launch_dependents / griddep_wait, sm100.cuh), so
// its launch and prologue overlap the end of the previous kernel.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline spg_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SPG_OK : SPG_ERR_CUDA;
}

}  // namespace spg
