// Argument marshalling for the per-step calls of the C ABI (include/hs2.h) from torch tensors: the
// dtype, device, rank, contiguity and shape checks of the Python binding, done in C++ so that a
// decode step's calls cost the host a few microseconds. No arithmetic: every entry checks its
// tensors and calls the C function whose address the Python binding passes in once (the functions
// live in libhs2.so, loaded by the binding). Argument errors raise ValueError.
#include <torch/extension.h>

#include <cstdint>

namespace {

using hs2_status = int;
using FullFn = hs2_status (*)(const void*, const void*, const void*, int, int, int, int, int, float, int, int, void*,
                              float*, int32_t*, void*, size_t, void*);
using SparseFn = hs2_status (*)(const void*, const void*, const void*, const int32_t*, int, int, int, int, int, int,
                                float, void*, float*, void*, size_t, void*);

FullFn g_full = nullptr;
SparseFn g_sparse = nullptr;

void set_entries(int64_t full, int64_t sparse) {
  g_full = reinterpret_cast<FullFn>(full);
  g_sparse = reinterpret_cast<SparseFn>(sparse);
}

// argument errors surface in Python as ValueError, as in the binding's other entries
#define HS2_ARG_CHECK(cond, ...) \
  do {                              \
    if (!(cond)) throw pybind11::value_error(c10::str(__VA_ARGS__)); \
  } while (0)

inline void need(const at::Tensor& t, const char* name, at::ScalarType dt, int64_t dim) {
  HS2_ARG_CHECK(t.is_cuda(), name, " must be a CUDA tensor");
  HS2_ARG_CHECK(t.scalar_type() == dt, name, " must be ", c10::toString(dt), ", got ", c10::toString(t.scalar_type()));
  HS2_ARG_CHECK(t.dim() == dim, name, " must have ", dim, " dims, got ", t.sizes());
  HS2_ARG_CHECK(t.is_contiguous(), name, " must be contiguous");
}

// hs2_full_attn_select: q [B,Lq,H,d] bf16; k, v [B,Lk,d] bf16; out [B,Lq,H,d] bf16; lse [B,Lq,H]
// fp32; idx [B,Lq,window+topk] int32; ws uint8. Returns the C status.
int64_t full_attn_select(const at::Tensor& q, const at::Tensor& k, const at::Tensor& v, double scale, int64_t window,
                         int64_t topk, const at::Tensor& out, const at::Tensor& lse, const at::Tensor& idx,
                         const at::Tensor& ws, int64_t stream) {
  HS2_ARG_CHECK(g_full != nullptr, "entry points not set");
  need(q, "q", at::kBFloat16, 4);
  need(k, "k", at::kBFloat16, 3);
  need(v, "v", at::kBFloat16, 3);
  const int64_t B = q.size(0), Lq = q.size(1), H = q.size(2), d = q.size(3), Lk = k.size(1);
  HS2_ARG_CHECK(k.size(0) == B && k.size(2) == d && v.sizes() == k.sizes(), "k and v must be [B, Lk, d] matching q");
  need(out, "out", at::kBFloat16, 4);
  need(lse, "lse", at::kFloat, 3);
  need(idx, "idx", at::kInt, 3);
  HS2_ARG_CHECK(out.sizes() == q.sizes(), "out must be shaped like q");
  HS2_ARG_CHECK(lse.size(0) == B && lse.size(1) == Lq && lse.size(2) == H, "lse must be [B, Lq, H]");
  HS2_ARG_CHECK(idx.size(0) == B && idx.size(1) == Lq && idx.size(2) == window + topk, "idx must be [B, Lq, window + topk]");
  HS2_ARG_CHECK(ws.is_cuda() && ws.is_contiguous(), "workspace must be a contiguous CUDA tensor");
  return g_full(q.data_ptr(), k.data_ptr(), v.data_ptr(), (int)B, (int)Lq, (int)Lk, (int)H, (int)d, (float)scale,
                (int)window, (int)topk, out.data_ptr(), lse.data_ptr<float>(), idx.data_ptr<int32_t>(), ws.data_ptr(),
                (size_t)ws.nbytes(), reinterpret_cast<void*>(stream));
}

// hs2_sparse_attn: q [B,Lq,H,d] bf16; k, v [B,Lk,d] bf16; idx [B,Lq,S] int32; out like q; lse
// [B,Lq,H] fp32 or None; ws uint8. Returns the C status.
int64_t sparse_attn(const at::Tensor& q, const at::Tensor& k, const at::Tensor& v, const at::Tensor& idx, double scale,
                    const at::Tensor& out, const c10::optional<at::Tensor>& lse, const at::Tensor& ws, int64_t stream) {
  HS2_ARG_CHECK(g_sparse != nullptr, "entry points not set");
  need(q, "q", at::kBFloat16, 4);
  need(k, "k", at::kBFloat16, 3);
  need(v, "v", at::kBFloat16, 3);
  need(idx, "idx", at::kInt, 3);
  const int64_t B = q.size(0), Lq = q.size(1), H = q.size(2), d = q.size(3), Lk = k.size(1), S = idx.size(2);
  HS2_ARG_CHECK(k.size(0) == B && k.size(2) == d && v.sizes() == k.sizes(), "k and v must be [B, Lk, d] matching q");
  HS2_ARG_CHECK(idx.size(0) == B && idx.size(1) == Lq, "idx must be [B, Lq, S]");
  need(out, "out", at::kBFloat16, 4);
  HS2_ARG_CHECK(out.sizes() == q.sizes(), "out must be shaped like q");
  float* lse_p = nullptr;
  if (lse.has_value()) {
    need(*lse, "lse", at::kFloat, 3);
    HS2_ARG_CHECK(lse->size(0) == B && lse->size(1) == Lq && lse->size(2) == H, "lse must be [B, Lq, H]");
    lse_p = lse->data_ptr<float>();
  }
  HS2_ARG_CHECK(ws.is_cuda() && ws.is_contiguous(), "workspace must be a contiguous CUDA tensor");
  return g_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr<int32_t>(), (int)B, (int)Lq, (int)Lk, (int)H,
                  (int)d, (int)S, (float)scale, out.data_ptr(), lse_p, ws.data_ptr(), (size_t)ws.nbytes(),
                  reinterpret_cast<void*>(stream));
}

}  // namespace

PYBIND11_MODULE(TORCH_EXTENSION_NAME, m) {
  m.def("set_entries", &set_entries);
  m.def("full_attn_select", &full_attn_select);
  m.def("sparse_attn", &sparse_attn);
}
