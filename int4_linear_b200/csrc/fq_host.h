// Host-side helpers shared by the library's translation units: error
// reporting, argument checks, the device error word and TMA tensor maps.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "../../include/fq.h"

namespace fq {

// Record a message for fq_last_error() and return `s`.
fq_status fail(fq_status s, const char* fmt, ...);
// Clear the calling thread's message.
void clear_error();

// Device address of the current device's timeout word (nullptr on failure).
unsigned* device_error_word();

// Number of SMs of the current device (cached).
int sm_count();

// cudaGetLastError() -> FQ_ERR_CUDA with the launch name, else FQ_OK.
fq_status check_launch(const char* what);

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 2-D row-major tensor map over uint8/fp16 data (no swizzle, zero fill for
// out-of-range boxes).  inner = elements per row, rows = rows,
// row_bytes = stride, box = {box_inner, box_rows}.
fq_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner,
                       uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE);

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream is still finishing; it must execute
// pdl_wait() (griddepcontrol.wait) before touching global memory that an
// earlier kernel may write or read, and it lets its own successor start
// early with pdl_launch_dependents().
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// launch_pdl as a cooperative launch: every CTA of the grid is resident at
// once (or the launch fails), so CTAs may wait for one another.
template <typename... KArgs, typename... Args>
cudaError_t launch_coop_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// launch_pdl with thread-block clusters of `cluster_x` CTAs along x
// (gridDim.x must be a multiple of cluster_x).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kGroup = 128;
constexpr int kMaxK = 65536;
constexpr int kMaxQuantK = 32768;

}  // namespace fq

#define FQ_CHECK_ARG(cond, ...)                                   \
  do {                                                            \
    if (!(cond)) return ::fq::fail(FQ_ERR_INVALID, __VA_ARGS__); \
  } while (0)
