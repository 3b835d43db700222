// Host-side helpers shared by the hs2 launchers: TMA descriptor encoding (driver entry point
// fetched through the runtime, so the library needs no libcuda link), device checks, and the
// bounded-wait limit.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <utility>

#include "../../include/hs2.h"

namespace hs2 {

// Encodes a 3D tensor map of bf16 (elem_bytes 2) or bytes (1): dims (inner, rows, batch) with
// strides in elements, box (box_inner, box_rows, 1), 128-byte swizzle, out-of-range elements
// read as zero.
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                  uint64_t row_stride_el, uint64_t batch_stride_el, uint32_t box_inner, uint32_t box_rows,
                  bool swizzle128 = true, int elem_bytes = 2);

// 2D variant: dims (inner, rows), row stride in elements.
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_el,
                  uint32_t box_inner, uint32_t box_rows);

long long wait_limit_ns();
int num_sms();
bool device_is_sm100();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launches `kernel` on `stream`; with pdl = true the launch may begin while the previous
// kernel on the stream is still running (the kernel must call griddep_wait() before it reads
// anything that kernel wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch accounting: every kernel launch site wraps its launch in a LaunchScope, which counts
// the launch and, when per-kernel timing is on for `name`, records CUDA events around it.
class LaunchScope {
 public:
  LaunchScope(const char* name, cudaStream_t stream);
  ~LaunchScope();

 private:
  int slot_;
  cudaStream_t stream_;
  const char* name_;
};

}  // namespace hs2
