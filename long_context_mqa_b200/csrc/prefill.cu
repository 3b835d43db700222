// Prefill full-attention + selection and KV Bridging GEMM (placeholder until the kernels land).
#include "prefill.h"

namespace hs2 {
namespace prefill {
size_t workspace_bytes(int, int, int, int, int, int, int, int, size_t status_bytes) { return status_bytes; }
hs2_status run(const hs2_bf16*, const hs2_bf16*, const hs2_bf16*, int, int, int, int, int, float, int, int, hs2_bf16*,
               float*, int32_t*, void*, size_t, int, size_t, cudaStream_t) {
  return HS2_ERR_UNSUPPORTED_SHAPE;
}
hs2_status run_bridge(const hs2_bf16*, int, int, const hs2_bf16*, int, int, hs2_bf16*, DevStatus*, cudaStream_t) {
  return HS2_ERR_UNSUPPORTED_SHAPE;
}
}  // namespace prefill
}  // namespace hs2
