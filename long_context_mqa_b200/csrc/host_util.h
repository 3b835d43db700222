// Host-side helpers shared by the hs2 launchers: TMA descriptor encoding (driver entry point
// fetched through the runtime, so the library needs no libcuda link), device checks, and the
// bounded-wait limit.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "../../include/hs2.h"

namespace hs2 {

// Encodes a 3D bf16 tensor map: dims (inner, rows, batch) with strides in elements,
// box (box_inner, box_rows, 1), 128-byte swizzle, out-of-range elements read as zero.
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                  uint64_t row_stride_el, uint64_t batch_stride_el, uint32_t box_inner, uint32_t box_rows,
                  bool swizzle128 = true);

// 2D variant: dims (inner, rows), row stride in elements.
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_el,
                  uint32_t box_inner, uint32_t box_rows);

long long wait_limit_ns();
int num_sms();
bool device_is_sm100();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
