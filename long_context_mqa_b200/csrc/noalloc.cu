// hs2_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plugin whose execute/enqueue hook runs
// inside an inference runtime that forbids device allocation on that path and hands the plugin
// no scratch buffer; or a process that fixed its device-memory budget up front and may not call
// cudaMalloc afterwards. They can pass inputs and outputs, but not the workspace hs2_sparse_attn
// asks for. This entry point uses instead a scratch array that lives in the library itself.
//
// The array below is a file-scope __device__ object of kScratchBytes (4 KiB): every GPU on
// which this library's code is loaded holds it until the process exits. The sparse kernels need
// only their 256-byte status word from a workspace (split rows merge in distributed shared
// memory), so every supported shape fits; larger needs are still rejected, not overrun. Host code
// cannot use the array's name as a device address (it is a host-side stand-in), so the first
// call on each device looks the address up with cudaGetSymbolAddress while that device is
// current, and caches it per device together with the device's current context; a call that
// finds another context (the old one was destroyed, e.g. by cudaDeviceReset) looks it up again.
// That first call on a device should therefore happen before any stream capture. All calls share
// the one array and it keeps what the last call left there: each call clears the status word it
// needs at zero, and hs2_sparse_attn_noalloc_status reads what the last call recorded there.
// Calls whose GPU work overlaps (for example on two streams) race on the array. Nothing here calls
// cudaMalloc, cudaFree or an allocating library routine.
#include <cuda.h>

#include <mutex>

#include "../../include/hs2.h"
#include "host_util.h"

namespace {

constexpr size_t kScratchBytes = 4096;  // per device
__device__ __align__(256) unsigned char g_sparse_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// cuCtxGetCurrent through the runtime's driver entry point (the library does not link libcuda).
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<Fn>(nullptr);
    return reinterpret_cast<Fn>(p);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_sparse_scratch on the current device: looked up once per device (again
// only if the device's context has changed since). `setup` false: report HS2_ERR_WORKSPACE
// instead of looking it up (nothing has run there yet).
hs2_status scratch_for_current_device(void** out, bool setup = true) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HS2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != current_context()) {
    if (!setup) return HS2_ERR_WORKSPACE;
    void* p = nullptr;  // the lookup also makes the device's primary context current
    if (cudaGetSymbolAddress(&p, g_sparse_scratch) != cudaSuccess || p == nullptr) return HS2_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_ptr[dev];
  return HS2_OK;
}

}  // namespace

extern "C" hs2_status hs2_sparse_attn_noalloc(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                                              const int32_t* idx, int B, int Lq, int Lk, int H, int d, int S,
                                              float scale, hs2_bf16* out, float* lse, hs2_stream stream) {
  if (!Q || !K || !V || !idx || !out) return HS2_ERR_INVALID_ARG;
  const size_t need = hs2_sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S);
  if (need == 0) return HS2_ERR_INVALID_ARG;
  if (need > kScratchBytes) return HS2_ERR_WORKSPACE;  // shape needs more than the scratch holds
  void* scratch = nullptr;
  const hs2_status st = scratch_for_current_device(&scratch);
  if (st != HS2_OK) return st;
  // the status word at the start of the scratch must start at zero for this call
  if (cudaMemsetAsync(scratch, 0, 16, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HS2_ERR_CUDA;
  return hs2_sparse_attn(Q, K, V, idx, B, Lq, Lk, H, d, S, scale, out, lse, scratch, kScratchBytes, stream);
}

extern "C" hs2_status hs2_sparse_attn_noalloc_status(hs2_stream stream) {
  void* scratch = nullptr;
  const hs2_status st = scratch_for_current_device(&scratch, false);
  if (st != HS2_OK) return st;
  return hs2_read_device_status(scratch, stream);
}
