// Internal interface of the prefill (Lq == Lk) full-attention + selection path and of the
// KV Bridging GEMM.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/hs2.h"

namespace hs2 {
struct DevStatus;
namespace prefill {
size_t workspace_bytes(int B, int Lq, int Lk, int H, int d, int window, int topk, int sms, size_t status_bytes);
hs2_status run(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lq, int Lk, int H, int d, float c,
               int window, int topk, hs2_bf16* out, float* lse, int32_t* idx, void* ws, size_t ws_bytes, int sms,
               size_t status_bytes, cudaStream_t stream);
hs2_status run_bridge(const hs2_bf16* Hs, int T, int hidden, const hs2_bf16* W, int n_layers, int d, hs2_bf16* KV,
                      DevStatus* st, cudaStream_t stream);
}  // namespace prefill
}  // namespace hs2
