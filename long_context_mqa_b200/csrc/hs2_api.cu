// C ABI of the hs2 library (declared in include/hs2.h): argument validation, workspace
// layout, TMA descriptor set-up and dispatch to the kernel files. No allocation, no
// synchronisation and no host fallback on the compute paths.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "decode.h"
#include "host_util.h"
#include "prefill.h"
#include "tc.cuh"

namespace hs2 {

// ------------------------------------------------------------------------------------------
// host utilities
// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The encoded maps of the last few distinct argument sets, per host thread: a decode loop calls
// with the same buffers every step, and an encoding is a pure function of its arguments.
namespace {
struct TmapEntry {
  uint64_t key[12];
  CUtensorMap map;
  bool used;
};
constexpr int kTmapCache = 8;
thread_local TmapEntry t_tmaps[kTmapCache];
thread_local int t_tmap_next = 0;
TmapEntry* tmap_find(const uint64_t (&key)[12]) {
  for (auto& e : t_tmaps)
    if (e.used && memcmp(e.key, key, sizeof(key)) == 0) return &e;
  return nullptr;
}
void tmap_store(const uint64_t (&key)[12], const CUtensorMap& m) {
  TmapEntry& e = t_tmaps[t_tmap_next];
  t_tmap_next = (t_tmap_next + 1) % kTmapCache;
  memcpy(e.key, key, sizeof(key));
  e.map = m;
  e.used = true;
}
}  // namespace

static bool make_tmap_3d_uncached(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                                  uint64_t row_stride_el, uint64_t batch_stride_el, uint32_t box_inner,
                                  uint32_t box_rows, bool swizzle128, int elem_bytes);

bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                  uint64_t row_stride_el, uint64_t batch_stride_el, uint32_t box_inner, uint32_t box_rows,
                  bool swizzle128, int elem_bytes) {
  const uint64_t key[12] = {3, (uint64_t)(uintptr_t)base, inner, rows, batch, row_stride_el, batch_stride_el,
                            box_inner, box_rows, (uint64_t)swizzle128, (uint64_t)elem_bytes, 0};
  if (const TmapEntry* e = tmap_find(key)) {
    *m = e->map;
    return true;
  }
  if (!make_tmap_3d_uncached(m, base, inner, rows, batch, row_stride_el, batch_stride_el, box_inner, box_rows,
                             swizzle128, elem_bytes))
    return false;
  tmap_store(key, *m);
  return true;
}

static bool make_tmap_3d_uncached(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                                  uint64_t row_stride_el, uint64_t batch_stride_el, uint32_t box_inner,
                                  uint32_t box_rows, bool swizzle128, int elem_bytes) {
  auto enc = get_encoder();
  if (!enc || (elem_bytes != 1 && elem_bytes != 2)) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {row_stride_el * elem_bytes, batch_stride_el * elem_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
             const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_el,
                  uint32_t box_inner, uint32_t box_rows) {
  const uint64_t key[12] = {2, (uint64_t)(uintptr_t)base, inner, rows, row_stride_el, box_inner, box_rows, 0, 0, 0, 0, 0};
  if (const TmapEntry* e = tmap_find(key)) {
    *m = e->map;
    return true;
  }
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_el * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS ? (tmap_store(key, *m), true) : false;
}

static long long g_wait_ns = -1;
long long wait_limit_ns() {
  if (g_wait_ns < 0) {
    const char* e = getenv("HS2_WAIT_LIMIT_MS");
    long long ms = e ? atoll(e) : 0;
    g_wait_ns = (ms > 0 ? ms : 2000) * 1000000LL;
  }
  return g_wait_ns;
}

// Per-device attributes, queried once per device (every call needs them on the host)
constexpr int kMaxDevices = 64;
static std::atomic<int> g_sms[kMaxDevices];       // 0: not queried yet
static std::atomic<int> g_is_sm100[kMaxDevices];  // 0: not queried yet, 1: yes, 2: no

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices && (n = g_sms[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices) g_sms[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < kMaxDevices) {
    const int known = g_is_sm100[dev].load(std::memory_order_relaxed);
    if (known) return known == 1;
  }
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  const bool yes = major == 10 && minor == 0;
  if (dev >= 0 && dev < kMaxDevices) g_is_sm100[dev].store(yes ? 1 : 2, std::memory_order_relaxed);
  return yes;
}

// ------------------------------------------------------------------------------------------
// launch accounting / optional per-kernel timing
// ------------------------------------------------------------------------------------------
static std::atomic<unsigned long long> g_launches{0};
static std::atomic<bool> g_prof_on{false};
static std::mutex g_prof_mu;
static std::string g_prof_filter;
static std::map<std::string, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>> g_prof;
static std::vector<cudaEvent_t> g_event_pool;
static thread_local cudaEvent_t t_pending_start = nullptr;

static cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// While a stream is being captured into a CUDA graph the timing events become event-record nodes
// of the graph (they then hold the times of the graph's latest replay).
static unsigned record_flags(cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return cudaEventRecordDefault;
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
}

LaunchScope::LaunchScope(const char* name, cudaStream_t stream) : slot_(-1), stream_(stream), name_(name) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_filter != "*" && g_prof_filter != name) return;
  cudaEvent_t a = take_event();
  if (!a) return;
  cudaEventRecordWithFlags(a, stream, record_flags(stream));
  t_pending_start = a;
  slot_ = 0;
}

LaunchScope::~LaunchScope() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t b = take_event();
  if (!b) return;
  cudaEventRecordWithFlags(b, stream_, record_flags(stream_));
  g_prof[name_].push_back({t_pending_start, b});
  t_pending_start = nullptr;
}

// ------------------------------------------------------------------------------------------
// workspace carving
// ------------------------------------------------------------------------------------------
constexpr size_t kStatusBytes = 256;   // status word (16 bytes) + the decode grid barrier's counter
constexpr size_t kBarrierOffset = 64;
static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Carve {
  uint8_t* base;
  size_t off;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align256(off + count * sizeof(T));
    return p;
  }
};

// decode (Lq == 1) layout
struct DecodeWs {
  dec::DecParams p;
  int* meta;
  unsigned long long* bnd;
  size_t bytes;
  bool ok;  // the schedule's index arithmetic fits (a group of at most 2^32 / G tiles)
};

// Tiles a decode CTA gives up for crossing a sequence boundary (its second segment's drain,
// record and logsumexp cost about this many tiles of streaming; measured on B200: ~6 us).
constexpr int kBoundaryTiles = 4;

static DecodeWs carve_decode(void* ws, int B, const int* lens, int N, int H, int D, int W, int K, int sms) {
  DecodeWs w{};
  dec::DecParams& p = w.p;
  p.B = B; p.N = N; p.W = W; p.K = K;
  w.ok = B <= dec::kMaxSeqs;  // the schedule's per-sequence tables
  if (!w.ok) return w;
  // One flattened range of all sequences' tiles. (Sequences can be taken in groups small enough
  // for a group's K to stay in L2 between the phases; measured on B200 the per-group grid barrier,
  // pipeline drain and refill cost more than the HBM re-reads they save.)
  dec::Sched& s = p.sch;
  long long tiles = 0;
  for (int b = 0; b < B; ++b) tiles += (lens[b] + 127) / 128;
  w.ok = tiles < (1ll << 31);  // 32-bit tile arithmetic
  if (!w.ok) return w;
  s.set_lengths(B, lens);
  if (sms > dec::kMaxCtas) sms = dec::kMaxCtas;  // the schedule's start table
  s.G = (int)(tiles < sms ? tiles : sms);
  s.partition(kBoundaryTiles);
  int cmax = 1;
  for (int b = 0; b < B; ++b) {
    int g, lo, hi;
    s.covering(b, g, lo, hi);
    if (hi - lo + 1 > cmax) cmax = hi - lo + 1;
  }
  s.cmax = cmax;
  const size_t n_slots = (size_t)B * cmax;
  const int stride = N - W > 1 ? N - W : 1;  // room for the longest sequence's older tokens
  Carve c{(uint8_t*)ws, 0};
  p.st = c.take<DevStatus>(kStatusBytes / sizeof(DevStatus));
  // the grid-barrier counter lives in the status block, so clearing the status re-arms it
  p.gbar = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(p.st) + kBarrierOffset);
  p.ml = c.take<float>(n_slots * 2 * H);
  p.opart = c.take<float>(n_slots * H * D);
  p.lp = c.take<float>(n_slots * H);
  p.lsum = c.take<float>((size_t)B * H);
  p.lse2x = c.take<float>((size_t)B * H);
  p.ovf = c.take<int>((size_t)B + 1);
  p.fallback = 0;
  // phase 1 estimates each head's logsumexp from a sample of each sequence's tiles: 64 tiles (8k
  // keys) per sequence up to 8 sequences, then a budget of about 512 sampled tiles in all (at
  // least 16 per sequence), so that phase 1 stays a few tiles per CTA for large batches of
  // shorter caches (the estimate only sets how many keys the exact band re-score sees)
  p.sample_tiles = B <= 8 ? 64 : (512 / B > 16 ? 512 / B : 16);
  p.sc_stride = stride;
  p.sc = c.take<float>((size_t)B * stride);
  p.hist = c.take<unsigned>((size_t)B * sel::NBINS);
  p.seq_done = c.take<int>((size_t)B);
  w.meta = c.take<int>((size_t)B * sel::META);
  p.meta = w.meta;
  p.K_sel = K;
  p.words = ((stride + 31) / 32 + 7) / 8 * 8;  // rows of 32-byte multiples (vector loads)
  p.bitmap = c.take<unsigned>((size_t)B * p.words);
  w.bnd = c.take<unsigned long long>((size_t)B * stride);
  w.bytes = c.off;
  return w;
}

// sparse layout
static size_t carve_sparse(void* ws, int B, int Lq, int H, int D, int S, int sms, sparse::SpParams* p) {
  const long long rows = (long long)B * Lq;
  const int tiles = (S + 127) / 128;
  // few query rows (decode): split each row's index list over a cluster of CTAs (at most 16),
  // which merge their partial results through distributed shared memory
  int nsplit = 1, per = tiles;
  if (rows < sms && tiles > 1) {
    per = (tiles + 15) / 16;
    nsplit = (tiles + per - 1) / per;
  }
  Carve c{(uint8_t*)ws, 0};
  DevStatus* st = c.take<DevStatus>(kStatusBytes / sizeof(DevStatus));
  if (p) {
    p->st = st;
    p->nsplit = nsplit;
    p->split_slots = per * 128;
  }
  return c.off;
}

static bool shape_ok(int H, int d) { return (H == 64 && d == 128) || (H == 16 && d == 64); }

// ------------------------------------------------------------------------------------------
// device-side helpers of the C ABI
// ------------------------------------------------------------------------------------------
__global__ void selftest_wait_kernel(DevStatus* st, long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the bounded wait must give up and report
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns)) report_status(st, kStatusTimeout, 900);
}

// the device conversions of e4m3 codes, one pair per thread (checked against the format's
// definition by the tests)
__global__ void selftest_e4m3_kernel(const uint8_t* x, uint16_t* y_f16, uint16_t* y_bf16, int n_pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  const uint32_t w = (uint32_t)x[2 * i] | ((uint32_t)x[2 * i + 1] << 8);
  const uint32_t h = e4m3x2_to_f16x2(w), bf = e4m3_f16x2_to_bf16x2(h);
  y_f16[2 * i] = (uint16_t)(h & 0xFFFFu);
  y_f16[2 * i + 1] = (uint16_t)(h >> 16);
  y_bf16[2 * i] = (uint16_t)(bf & 0xFFFFu);
  y_bf16[2 * i + 1] = (uint16_t)(bf >> 16);
}

// e4m3 codes times `scale` -> bf16 (exact when the scale is a power of two), 16 codes per thread
// per step; n16 = number of 16-code groups
__global__ void widen_e4m3_kernel(const uint8_t* x, float scale, __nv_bfloat16* y, long long n16) {
  griddep_wait();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n16; i += stride) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(x) + i);
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t h0, h1;
      e4m3x4_to_f16x4(in[j], h0, h1);
      const uint32_t b0 = e4m3_f16x2_to_bf16x2(h0), b1 = e4m3_f16x2_to_bf16x2(h1);
      o[2 * j] = pack_bf16x2(__uint_as_float(b0 << 16) * scale, __uint_as_float(b0 & 0xFFFF0000u) * scale);
      o[2 * j + 1] = pack_bf16x2(__uint_as_float(b1 << 16) * scale, __uint_as_float(b1 & 0xFFFF0000u) * scale);
    }
    uint4* d = reinterpret_cast<uint4*>(y) + 2 * i;
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace hs2

using namespace hs2;

extern "C" {

int hs2_abi_version(void) { return HS2_ABI_VERSION; }

const char* hs2_status_string(hs2_status s) {
  switch (s) {
    case HS2_OK: return "ok";
    case HS2_ERR_INVALID_ARG: return "invalid argument";
    case HS2_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or device";
    case HS2_ERR_WORKSPACE: return "workspace missing or too small";
    case HS2_ERR_CUDA: return "CUDA error";
    case HS2_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case HS2_ERR_DEVICE_BOUNDS: return "device-side index out of range";
  }
  return "unknown status";
}

void hs2_set_wait_limit_ns(long long limit_ns) { g_wait_ns = limit_ns > 0 ? limit_ns : -1; }

size_t hs2_full_attn_select_workspace_bytes(int B, int Lq, int Lk, int H, int d, int window, int topk) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || d <= 0 || window < 1 || topk < 0) return 0;
  const int sms = num_sms() > 0 ? num_sms() : 148;
  if (Lq == 1 && H == 64 && d == 128) {  // the decode kernels
    if (B > dec::kMaxSeqs) return 0;
    std::vector<int> lens((size_t)B, Lk);
    return carve_decode(nullptr, B, lens.data(), Lk, H, d, window, topk, sms).bytes;
  }
  return prefill::workspace_bytes(B, Lq, Lk, H, d, window, topk, sms, kStatusBytes);
}

// The decode path (one query per sequence at the end of its lens[b]-token cache). K, V are
// [B][Lk] rows, or (ptab != NULL) pools of n_pages pages of 128 rows with Lk = max_pages * 128;
// bf16, or (f8) e4m3 codes with c including K's scale and oscale V's.
// The fused decode kernel (and its exact redo) alone; w receives the workspace layout.
static hs2_status launch_decode_fused(DecodeWs& w, const void* Q, const void* K, const void* V, int B,
                                      const int* lens, int Lk, int H, int d, float c, int window, int topk,
                                      float* lse, void* workspace, size_t workspace_bytes, int sms, cudaStream_t st,
                                      const int32_t* ptab, int max_pages, int n_pages, bool f8,
                                      float* blk_part = nullptr, int blk_groups = 0) {
  if (H != 64 || d != 128) return HS2_ERR_UNSUPPORTED_SHAPE;
  w = carve_decode(workspace, B, lens, Lk, H, d, window, topk, sms);
  if (!w.ok) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < w.bytes) return HS2_ERR_WORKSPACE;
  w.p.blk_part = blk_part;
  w.p.blk_groups = blk_groups;
  w.p.c = c;
  w.p.wait_ns = wait_limit_ns();
  w.p.lse_out = lse;
  w.p.ptab = ptab;
  w.p.max_pages = max_pages;
  w.p.n_pages = n_pages;
  // contiguous: (d, Lk rows, B sequences); paged: (d, 128 rows, n_pages pages)
  const uint64_t rows = ptab ? 128 : (uint64_t)Lk, planes = ptab ? (uint64_t)n_pages : (uint64_t)B;
  CUtensorMap tmK, tmV, tmQ;
  // bf16: boxes of 64 elements (128 bytes) x 128 rows; e4m3: the whole 128-byte row in one box
  const uint32_t kbox = f8 ? 128 : 64;
  const int eb = f8 ? 1 : 2;
  if (!make_tmap_3d(&tmK, K, d, rows, planes, d, rows * d, kbox, 128, true, eb) ||
      !make_tmap_3d(&tmV, V, d, rows, planes, d, rows * d, kbox, 128, true, eb) ||
      !make_tmap_3d(&tmQ, Q, d, H, B, d, (uint64_t)H * d, 64, H))
    return HS2_ERR_CUDA;
  if (dec::launch_decode_attn(tmK, tmV, tmQ, w.p, f8, st) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

static hs2_status run_decode(const void* Q, const void* K, const void* V, int B, const int* lens, int Lk,
                             int H, int d, float c, int window, int topk, hs2_bf16* out, float* lse, int32_t* idx,
                             void* workspace, size_t workspace_bytes, int sms, cudaStream_t st,
                             const int32_t* ptab = nullptr, int max_pages = 0, int n_pages = 0, bool f8 = false,
                             float oscale = 1.f) {
  DecodeWs w{};
  const hs2_status rc = launch_decode_fused(w, Q, K, V, B, lens, Lk, H, d, c, window, topk, lse, workspace,
                                            workspace_bytes, sms, st, ptab, max_pages, n_pages, f8);
  if (rc != HS2_OK) return rc;
  sel::SelParams sp;
  sp.opart = w.p.opart;
  sp.out = reinterpret_cast<__nv_bfloat16*>(out);
  sp.H = H; sp.D = d; sp.sch = w.p.sch;
  sp.lsum = w.p.lsum;
  sp.oscale = oscale;
  sp.qry = reinterpret_cast<const __nv_bfloat16*>(Q);
  sp.kc = f8 ? nullptr : reinterpret_cast<const __nv_bfloat16*>(K);
  sp.kc8 = f8 ? reinterpret_cast<const uint8_t*>(K) : nullptr;
  sp.lse2x = w.p.lse2x;
  sp.gbar = w.p.gbar;
  sp.ptab = ptab;
  sp.max_pages = max_pages;
  sp.n_pages = n_pages;
  sp.c = c;
  sp.sms = sms;
  sp.wait_ns = w.p.wait_ns;
  sp.B = B; sp.N = Lk; sp.W = window; sp.K = topk; sp.S = window + topk;
  sp.ncand = w.p.sc_stride;
  sp.sc = w.p.sc; sp.hist = w.p.hist; sp.meta = w.meta; sp.bnd = w.bnd;
  sp.bitmap = w.p.bitmap; sp.words = w.p.words;
  sp.idx = idx; sp.st = w.p.st;
  if (sel::launch_select(sp, st) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

hs2_status hs2_full_attn_select(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lq, int Lk,
                                int H, int d, float scale, int window, int topk, hs2_bf16* out, float* lse,
                                int32_t* idx, void* workspace, size_t workspace_bytes, hs2_stream stream) {
  if (!Q || !K || !V || !out || !lse || !idx) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || !aligned16(lse) || !aligned16(idx))
    return HS2_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || window < 1 || topk < 0 || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (window + topk > 2048) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!shape_ok(H, d)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  const int sms = num_sms();
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float c = scale * 1.4426950408889634f;
  if (Lq == 1 && H == 64 && d == 128) {  // decode: one query per sequence
    if (B > dec::kMaxSeqs) return HS2_ERR_UNSUPPORTED_SHAPE;
    std::vector<int> lens((size_t)B, Lk);
    return run_decode(Q, K, V, B, lens.data(), Lk, H, d, c, window, topk, out, lse, idx, workspace, workspace_bytes,
                      sms, st);
  }
  // a whole prompt (Lq == Lk) or a chunk of Lq queries appended to a cache (Lq < Lk)
  return prefill::run(Q, K, V, B, Lq, Lk, H, d, c, window, topk, out, lse, idx, workspace, workspace_bytes, sms,
                      kStatusBytes, st);
}

static bool ragged_lens_ok(int B, const int32_t* lens, int Lk) {
  if (!lens || B <= 0 || B > dec::kMaxSeqs) return false;
  for (int b = 0; b < B; ++b)
    if (lens[b] < 1 || lens[b] > Lk) return false;
  return true;
}

size_t hs2_full_attn_select_ragged_workspace_bytes(int B, const int32_t* lens, int Lk, int H, int d, int window,
                                                   int topk) {
  if (Lk <= 0 || H <= 0 || d <= 0 || window < 1 || topk < 0 || !ragged_lens_ok(B, lens, Lk)) return 0;
  const int sms = num_sms() > 0 ? num_sms() : 148;
  return carve_decode(nullptr, B, reinterpret_cast<const int*>(lens), Lk, H, d, window, topk, sms).bytes;
}

hs2_status hs2_full_attn_select_ragged(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B,
                                       const int32_t* lens, int Lk, int H, int d, float scale, int window, int topk,
                                       hs2_bf16* out, float* lse, int32_t* idx, void* workspace,
                                       size_t workspace_bytes, hs2_stream stream) {
  if (!Q || !K || !V || !out || !lse || !idx) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || !aligned16(lse) || !aligned16(idx))
    return HS2_ERR_INVALID_ARG;
  if (Lk <= 0 || window < 1 || topk < 0 || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (!lens || B <= 0) return HS2_ERR_INVALID_ARG;
  if (B > dec::kMaxSeqs) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!ragged_lens_ok(B, lens, Lk)) return HS2_ERR_INVALID_ARG;
  if (window + topk > 2048) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!shape_ok(H, d)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  return run_decode(Q, K, V, B, reinterpret_cast<const int*>(lens), Lk, H, d, scale * 1.4426950408889634f, window,
                    topk, out, lse, idx, workspace, workspace_bytes, num_sms(), reinterpret_cast<cudaStream_t>(stream));
}

size_t hs2_full_attn_select_paged_workspace_bytes(int B, const int32_t* lens, int max_pages, int H, int d,
                                                  int window, int topk) {
  if (max_pages <= 0 || max_pages > (1 << 23)) return 0;
  return hs2_full_attn_select_ragged_workspace_bytes(B, lens, max_pages * 128, H, d, window, topk);
}

hs2_status hs2_full_attn_select_paged(const hs2_bf16* Q, const hs2_bf16* K_pages, const hs2_bf16* V_pages,
                                      int n_pages, const int32_t* page_table, int max_pages, int B,
                                      const int32_t* lens, int H, int d, float scale, int window, int topk,
                                      hs2_bf16* out, float* lse, int32_t* idx, void* workspace,
                                      size_t workspace_bytes, hs2_stream stream) {
  if (!Q || !K_pages || !V_pages || !page_table || !out || !lse || !idx) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(idx) || (reinterpret_cast<uintptr_t>(page_table) & 3u) != 0)
    return HS2_ERR_INVALID_ARG;
  if (n_pages <= 0 || max_pages <= 0 || max_pages > (1 << 23) || window < 1 || topk < 0 || !(scale > 0.f))
    return HS2_ERR_INVALID_ARG;
  const int Lk = max_pages * 128;
  if (!lens || B <= 0) return HS2_ERR_INVALID_ARG;
  if (B > dec::kMaxSeqs) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!ragged_lens_ok(B, lens, Lk)) return HS2_ERR_INVALID_ARG;
  if (window + topk > 2048) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (H != 64 || d != 128) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  return run_decode(Q, K_pages, V_pages, B, reinterpret_cast<const int*>(lens), Lk, H, d,
                    scale * 1.4426950408889634f, window, topk, out, lse, idx, workspace, workspace_bytes, num_sms(),
                    reinterpret_cast<cudaStream_t>(stream), page_table, max_pages, n_pages);
}

size_t hs2_sparse_attn_workspace_bytes(int B, int Lq, int Lk, int H, int d, int S) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || d <= 0 || S <= 0) return 0;
  const int sms = num_sms() > 0 ? num_sms() : 148;
  return carve_sparse(nullptr, B, Lq, H, d, S, sms, nullptr);
}

// K, V: bf16 rows, or (f8) e4m3 codes whose scales multiply the logits (k_scale) and the output
static hs2_status run_sparse(const hs2_bf16* Q, const void* K, const void* V, const int32_t* idx, int B,
                             int Lq, int Lk, int H, int d, int S, float scale, hs2_bf16* out, float* lse,
                             void* workspace, size_t workspace_bytes, hs2_stream stream, const int32_t* ptab,
                             int max_pages, int n_pages, bool f8 = false, float k_scale = 1.f, float v_scale = 1.f) {
  if (!Q || !K || !V || !idx || !out) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || (lse && !aligned16(lse)))
    return HS2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) & 3u) != 0) return HS2_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || S <= 0 || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (S > 4096) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!shape_ok(H, d)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * Lq > 2147483647LL / 16) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  const int sms = num_sms();
  sparse::SpParams p{};
  const size_t need = carve_sparse(workspace, B, Lq, H, d, S, sms, &p);
  if (workspace_bytes < need) return HS2_ERR_WORKSPACE;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.K = f8 ? nullptr : reinterpret_cast<const __nv_bfloat16*>(K);
  p.V = f8 ? nullptr : reinterpret_cast<const __nv_bfloat16*>(V);
  p.K8 = f8 ? reinterpret_cast<const uint8_t*>(K) : nullptr;
  p.V8 = f8 ? reinterpret_cast<const uint8_t*>(V) : nullptr;
  p.oscale = v_scale;
  p.idx = idx;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.S = S;
  p.c = scale * k_scale * 1.4426950408889634f;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.wait_ns = wait_limit_ns();
  p.ptab = ptab;
  p.max_pages = max_pages;
  p.n_pages = n_pages;
  if (sparse::launch_sparse(p, H, d, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

hs2_status hs2_sparse_attn(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx, int B,
                           int Lq, int Lk, int H, int d, int S, float scale, hs2_bf16* out, float* lse,
                           void* workspace, size_t workspace_bytes, hs2_stream stream) {
  return run_sparse(Q, K, V, idx, B, Lq, Lk, H, d, S, scale, out, lse, workspace, workspace_bytes, stream, nullptr,
                    0, 0);
}

hs2_status hs2_sparse_attn_paged(const hs2_bf16* Q, const hs2_bf16* K_pages, const hs2_bf16* V_pages, int n_pages,
                                 const int32_t* page_table, int max_pages, const int32_t* idx, int B, int Lq, int H,
                                 int d, int S, float scale, hs2_bf16* out, float* lse, void* workspace,
                                 size_t workspace_bytes, hs2_stream stream) {
  if (!page_table || (reinterpret_cast<uintptr_t>(page_table) & 3u) != 0) return HS2_ERR_INVALID_ARG;
  if (n_pages <= 0 || max_pages <= 0 || max_pages > (1 << 23)) return HS2_ERR_INVALID_ARG;
  return run_sparse(Q, K_pages, V_pages, idx, B, Lq, max_pages * 128, H, d, S, scale, out, lse, workspace,
                    workspace_bytes, stream, page_table, max_pages, n_pages);
}

// ------------------------------------------------------------------------------------------
// HySparse (v1): block-level selection and the gated two-branch sparse layer
// ------------------------------------------------------------------------------------------
struct V1Ws {
  size_t dec_bytes, bytes;
  int max_blocks, groups;
  float* part;
  float* bsc;
};

// the decode workspace, then the decode kernel's per-32-key head sums and the block scores
static V1Ws carve_v1(void* ws, size_t dec_bytes, int B, int Lk, int H, int block) {
  V1Ws v{};
  v.dec_bytes = dec_bytes;
  v.max_blocks = (Lk + block - 1) / block;
  v.groups = 4 * ((Lk + 127) / 128);  // every group of every (possibly partial) 128-key tile
  Carve c{(uint8_t*)ws, dec_bytes};
  v.part = c.take<float>((size_t)B * v.groups * H);
  v.bsc = c.take<float>((size_t)B * v.max_blocks);
  v.bytes = c.off;
  return v;
}

static bool v1_shape_ok(int H, int d, int window, int block, int n_blocks) {
  return H == 64 && d == 128 && block == 64 && n_blocks >= 1 && n_blocks <= 32 && window >= 1 &&
         n_blocks * block + window <= 2048;
}

size_t hs2_full_attn_select_v1_workspace_bytes(int B, int Lk, int H, int d, int window, int block, int n_blocks) {
  if (B <= 0 || B > dec::kMaxSeqs || Lk <= 0 || !v1_shape_ok(H, d, window, block, n_blocks)) return 0;
  const int sms = num_sms() > 0 ? num_sms() : 148;
  std::vector<int> lens((size_t)B, Lk);
  const DecodeWs w = carve_decode(nullptr, B, lens.data(), Lk, H, d, window, n_blocks * block, sms);
  if (!w.ok) return 0;
  return carve_v1(nullptr, w.bytes, B, Lk, H, block).bytes;
}

hs2_status hs2_full_attn_select_v1(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lk, int H,
                                   int d, float scale, int window, int block, int n_blocks, hs2_bf16* out,
                                   float* lse, int32_t* idx, void* workspace, size_t workspace_bytes,
                                   hs2_stream stream) {
  if (!Q || !K || !V || !out || !lse || !idx) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || !aligned16(lse) || !aligned16(idx))
    return HS2_ERR_INVALID_ARG;
  if (B <= 0 || Lk <= 0 || window < 1 || block <= 0 || n_blocks <= 0 || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (B > dec::kMaxSeqs || !v1_shape_ok(H, d, window, block, n_blocks)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  const int sms = num_sms();
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float c = scale * 1.4426950408889634f;
  std::vector<int> lens((size_t)B, Lk);
  // the decode kernel's own bounds are computed for a top-k of n_blocks * block tokens (unused here)
  DecodeWs w{};
  if (workspace_bytes < hs2_full_attn_select_v1_workspace_bytes(B, Lk, H, d, window, block, n_blocks))
    return HS2_ERR_WORKSPACE;
  // the layout of the decode part first (for the offset of the v1 buffers after it)
  const DecodeWs w0 = carve_decode(nullptr, B, lens.data(), Lk, H, d, window, n_blocks * block, sms);
  const V1Ws v = carve_v1(workspace, w0.bytes, B, Lk, H, block);
  const hs2_status rc = launch_decode_fused(w, Q, K, V, B, lens.data(), Lk, H, d, c, window, n_blocks * block, lse,
                                            workspace, workspace_bytes, sms, st, nullptr, 0, 0, false, v.part,
                                            v.groups);
  if (rc != HS2_OK) return rc;
  blk::BlkParams bp{};
  bp.B = B; bp.H = H; bp.D = d; bp.W = window;
  bp.NB = n_blocks; bp.BLK = block; bp.S = n_blocks * block + window;
  bp.sch = w.p.sch;
  bp.blk_part = v.part; bp.blk_groups = v.groups;
  bp.lsum = w.p.lsum;
  bp.max_blocks = v.max_blocks; bp.bsc = v.bsc;
  bp.idx = idx;
  bp.gbar = w.p.gbar;
  bp.opart = w.p.opart; bp.oscale = 1.f;
  bp.out = reinterpret_cast<__nv_bfloat16*>(out);
  bp.st = w.p.st;
  if (blk::launch_block_select(bp, st) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

hs2_status hs2_sparse_attn_v1(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx,
                              const float* gate, int B, int Lq, int Lk, int H, int d, int S, int branch, float scale,
                              hs2_bf16* out, void* workspace, size_t workspace_bytes, hs2_stream stream) {
  if (!Q || !K || !V || !idx || !gate || !out) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return HS2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) & 3u) != 0 || (reinterpret_cast<uintptr_t>(gate) & 3u) != 0)
    return HS2_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || S <= 0 || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (branch <= 0 || branch >= S || branch % 128 != 0) return HS2_ERR_INVALID_ARG;
  if (H != 64 || d != 128 || S > 2048) return HS2_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * Lq > 2147483647LL / 16) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  sparse::SpParams p{};
  const size_t need = carve_sparse(workspace, B, Lq, H, d, S, num_sms(), &p);
  if (workspace_bytes < need) return HS2_ERR_WORKSPACE;
  // one split (CTA of the row's cluster) per 128 slots, so the branch boundary falls between splits
  p.nsplit = (S + 127) / 128;
  p.split_slots = 128;
  p.branch_split = branch / 128;
  p.gate = gate;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.K = reinterpret_cast<const __nv_bfloat16*>(K);
  p.V = reinterpret_cast<const __nv_bfloat16*>(V);
  p.oscale = 1.f;
  p.idx = idx;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.S = S;
  p.c = scale * 1.4426950408889634f;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = nullptr;
  p.wait_ns = wait_limit_ns();
  if (sparse::launch_sparse(p, H, d, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

// ------------------------------------------------------------------------------------------
// backward pass of the full layer and of a sparse layer
// ------------------------------------------------------------------------------------------
struct BwdWs {
  DevStatus* st;
  float* Dv;
  float* lse2;
  size_t bytes;
};

// status block | D per (query, head) row | lse2 per row (both padded by a 128-row tile: the
// key-side kernel copies a whole tile's values with its Q tile)
static BwdWs carve_bwd(void* ws, int B, int Lq, int Lk, int H, int d) {
  BwdWs w{};
  const long long rows = (long long)B * Lq * H;
  Carve c{(uint8_t*)ws, 0};
  w.st = c.take<DevStatus>(kStatusBytes / sizeof(DevStatus));
  w.Dv = c.take<float>((size_t)rows + 128);
  w.lse2 = c.take<float>((size_t)rows + 128);
  w.bytes = c.off;
  return w;
}

size_t hs2_attn_bwd_workspace_bytes(int B, int Lq, int Lk, int H, int d) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || !shape_ok(H, d)) return 0;
  return carve_bwd(nullptr, B, Lq, Lk, H, d).bytes;
}

static hs2_status bwd_args_ok(const void* Q, const void* K, const void* V, const void* out, const float* lse,
                              const void* dO, const void* dQ, const float* dK, const float* dV, int B, int Lq, int Lk,
                              int H, int d, float scale, const void* workspace) {
  if (!Q || !K || !V || !out || !lse || !dO || !dQ || !dK || !dV) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return HS2_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (!shape_ok(H, d)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * Lq * H > 2147483647LL - 256 || (long long)B * Lk > 2147483647LL / 128)
    return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  return HS2_OK;
}

hs2_status hs2_full_attn_bwd(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const hs2_bf16* out,
                             const float* lse, const hs2_bf16* dO, int B, int Lq, int Lk, int H, int d, float scale,
                             hs2_bf16* dQ, float* dK, float* dV, void* workspace, size_t workspace_bytes,
                             hs2_stream stream) {
  const hs2_status rc = bwd_args_ok(Q, K, V, out, lse, dO, dQ, dK, dV, B, Lq, Lk, H, d, scale, workspace);
  if (rc != HS2_OK) return rc;
  const long long rows = (long long)B * Lq * H;
  const BwdWs w = carve_bwd(workspace, B, Lq, Lk, H, d);
  if (workspace_bytes < w.bytes) return HS2_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms();
  CUtensorMap tmQ, tmdO, tmK, tmV;
  if (!make_tmap_2d(&tmQ, Q, d, (uint64_t)rows, d, 64, 128) || !make_tmap_2d(&tmdO, dO, d, (uint64_t)rows, d, 64, 128) ||
      !make_tmap_3d(&tmK, K, d, Lk, B, d, (uint64_t)Lk * d, 64, 128) ||
      !make_tmap_3d(&tmV, V, d, Lk, B, d, (uint64_t)Lk * d, 64, 128))
    return HS2_ERR_CUDA;
  const __nv_bfloat16* bQ = reinterpret_cast<const __nv_bfloat16*>(Q);
  if (bwd::launch_prep(reinterpret_cast<const __nv_bfloat16*>(dO), reinterpret_cast<const __nv_bfloat16*>(out), lse,
                       w.Dv, w.lse2, rows, d, st) != cudaSuccess)
    return HS2_ERR_CUDA;
  bwd::BwdParams p{};
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.H = H; p.D = d;
  p.off = Lk - Lq;
  p.rows_per_batch = Lq * H;
  p.tiles_per_batch = (Lq * H + 127) / 128;
  p.kv_tiles = (Lk + 127) / 128;
  // key-side work items: a key tile and at most `chunk` row tiles, about a dozen per SM at 32k
  p.chunk = p.tiles_per_batch / 16 > 16 ? p.tiles_per_batch / 16 : 16;
  p.n_chunks = (p.tiles_per_batch + p.chunk - 1) / p.chunk;
  p.c = scale * 1.4426950408889634f;
  p.scale = scale;
  p.lse2 = w.lse2; p.Dv = w.Dv;
  p.dQ = reinterpret_cast<__nv_bfloat16*>(dQ);
  p.dK = dK; p.dV = dV;
  p.Q = bQ;
  p.wait_ns = wait_limit_ns();
  p.st = w.st;
  if (bwd::launch_full_bwd(tmQ, tmdO, tmK, tmV, p, sms, st) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

hs2_status hs2_sparse_attn_bwd(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx,
                               const hs2_bf16* out, const float* lse, const hs2_bf16* dO, int B, int Lq, int Lk, int H,
                               int d, int S, float scale, hs2_bf16* dQ, float* dK, float* dV, void* workspace,
                               size_t workspace_bytes, hs2_stream stream) {
  hs2_status rc = bwd_args_ok(Q, K, V, out, lse, dO, dQ, dK, dV, B, Lq, Lk, H, d, scale, workspace);
  if (rc != HS2_OK) return rc;
  if (!idx || (reinterpret_cast<uintptr_t>(idx) & 3u) != 0 || S <= 0) return HS2_ERR_INVALID_ARG;
  if (S > 4096) return HS2_ERR_UNSUPPORTED_SHAPE;
  const long long rows = (long long)B * Lq * H;
  const BwdWs w = carve_bwd(workspace, B, Lq, Lk, H, d);
  if (workspace_bytes < w.bytes) return HS2_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (bwd::launch_prep(reinterpret_cast<const __nv_bfloat16*>(dO), reinterpret_cast<const __nv_bfloat16*>(out), lse,
                       w.Dv, w.lse2, rows, d, st) != cudaSuccess)
    return HS2_ERR_CUDA;
  bwd::BwdParams p{};
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.H = H; p.D = d;
  p.off = Lk - Lq;
  p.S = S;
  p.c = scale * 1.4426950408889634f;
  p.scale = scale;
  p.lse2 = w.lse2; p.Dv = w.Dv;
  p.dQ = reinterpret_cast<__nv_bfloat16*>(dQ);
  p.dK = dK; p.dV = dV;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.K = reinterpret_cast<const __nv_bfloat16*>(K);
  p.V = reinterpret_cast<const __nv_bfloat16*>(V);
  p.dO = reinterpret_cast<const __nv_bfloat16*>(dO);
  p.idx = idx;
  p.wait_ns = wait_limit_ns();
  p.st = w.st;
  if (bwd::launch_sparse_bwd(p, num_sms(), st) != cudaSuccess) return HS2_ERR_CUDA;
  return HS2_OK;
}

static bool kv_scale_ok(float s) { return s > 0.f && s < INFINITY; }

size_t hs2_full_attn_select_fp8kv_workspace_bytes(int B, const int32_t* lens, int Lk, int H, int d, int window,
                                                  int topk) {
  if (B <= 0 || B > dec::kMaxSeqs || Lk <= 0 || H != 64 || d != 128 || window < 1 || topk < 0) return 0;
  if (lens) return hs2_full_attn_select_ragged_workspace_bytes(B, lens, Lk, H, d, window, topk);
  std::vector<int32_t> all((size_t)B, Lk);
  return hs2_full_attn_select_ragged_workspace_bytes(B, all.data(), Lk, H, d, window, topk);
}

hs2_status hs2_full_attn_select_fp8kv(const hs2_bf16* Q, const uint8_t* K8, const uint8_t* V8, float k_scale,
                                      float v_scale, int B, const int32_t* lens, int Lk, const int32_t* page_table,
                                      int max_pages, int n_pages, int H, int d, float scale, int window, int topk,
                                      hs2_bf16* out, float* lse, int32_t* idx, void* workspace,
                                      size_t workspace_bytes, hs2_stream stream) {
  if (!Q || !K8 || !V8 || !out || !lse || !idx) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K8) || !aligned16(V8) || !aligned16(out) || !aligned16(lse) || !aligned16(idx))
    return HS2_ERR_INVALID_ARG;
  if (!kv_scale_ok(k_scale) || !kv_scale_ok(v_scale)) return HS2_ERR_INVALID_ARG;
  if (Lk <= 0 || window < 1 || topk < 0 || !(scale > 0.f) || B <= 0) return HS2_ERR_INVALID_ARG;
  if (page_table) {
    if ((reinterpret_cast<uintptr_t>(page_table) & 3u) != 0 || n_pages <= 0 || max_pages <= 0 ||
        max_pages > (1 << 23) || Lk != max_pages * 128)
      return HS2_ERR_INVALID_ARG;
  }
  if (B > dec::kMaxSeqs) return HS2_ERR_UNSUPPORTED_SHAPE;
  std::vector<int> all;
  const int* ln = reinterpret_cast<const int*>(lens);
  if (!lens) {
    all.assign((size_t)B, Lk);
    ln = all.data();
  } else if (!ragged_lens_ok(B, lens, Lk)) {
    return HS2_ERR_INVALID_ARG;
  }
  if (window + topk > 2048) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (H != 64 || d != 128) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  return run_decode(Q, K8, V8, B, ln, Lk, H, d, scale * k_scale * 1.4426950408889634f, window, topk, out, lse, idx,
                    workspace, workspace_bytes, num_sms(), reinterpret_cast<cudaStream_t>(stream), page_table,
                    page_table ? max_pages : 0, page_table ? n_pages : 0, true, v_scale);
}

hs2_status hs2_sparse_attn_fp8kv(const hs2_bf16* Q, const uint8_t* K8, const uint8_t* V8, float k_scale,
                                 float v_scale, const int32_t* idx, int B, int Lq, int Lk, const int32_t* page_table,
                                 int max_pages, int n_pages, int H, int d, int S, float scale, hs2_bf16* out,
                                 float* lse, void* workspace, size_t workspace_bytes, hs2_stream stream) {
  if (!kv_scale_ok(k_scale) || !kv_scale_ok(v_scale)) return HS2_ERR_INVALID_ARG;
  if (page_table) {
    if ((reinterpret_cast<uintptr_t>(page_table) & 3u) != 0 || n_pages <= 0 || max_pages <= 0 ||
        max_pages > (1 << 23) || Lk != max_pages * 128)
      return HS2_ERR_INVALID_ARG;
  }
  return run_sparse(Q, K8, V8, idx, B, Lq, Lk, H, d, S, scale, out, lse, workspace, workspace_bytes, stream,
                    page_table, page_table ? max_pages : 0, page_table ? n_pages : 0, true, k_scale, v_scale);
}

// The whole-prompt / chunk entry over an e4m3 cache: one query per sequence goes to the FP8
// decode kernels; otherwise the cache is widened once into the workspace and the prefill kernels
// (tensor-bound: the cache is read from L2 many times) run on the bf16 copy.
static size_t fp8_cache_copy_bytes(int B, int Lk, int d) { return align256((size_t)B * Lk * d * 2); }

size_t hs2_full_attn_select_prefill_fp8kv_workspace_bytes(int B, int Lq, int Lk, int H, int d, int window, int topk) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H <= 0 || d <= 0 || window < 1 || topk < 0) return 0;
  if (Lq == 1 && H == 64 && d == 128) return hs2_full_attn_select_fp8kv_workspace_bytes(B, nullptr, Lk, H, d, window, topk);
  const int sms = num_sms() > 0 ? num_sms() : 148;
  return align256(prefill::workspace_bytes(B, Lq, Lk, H, d, window, topk, sms, kStatusBytes)) +
         2 * fp8_cache_copy_bytes(B, Lk, d);
}

hs2_status hs2_full_attn_select_prefill_fp8kv(const hs2_bf16* Q, const uint8_t* K8, const uint8_t* V8, float k_scale,
                                              float v_scale, int B, int Lq, int Lk, int H, int d, float scale,
                                              int window, int topk, hs2_bf16* out, float* lse, int32_t* idx,
                                              void* workspace, size_t workspace_bytes, hs2_stream stream) {
  if (Lq == 1 && H == 64 && d == 128)
    return hs2_full_attn_select_fp8kv(Q, K8, V8, k_scale, v_scale, B, nullptr, Lk, nullptr, 0, 0, H, d, scale, window,
                                      topk, out, lse, idx, workspace, workspace_bytes, stream);
  if (!Q || !K8 || !V8 || !out || !lse || !idx) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K8) || !aligned16(V8) || !aligned16(out) || !aligned16(lse) || !aligned16(idx))
    return HS2_ERR_INVALID_ARG;
  if (!kv_scale_ok(k_scale) || !kv_scale_ok(v_scale)) return HS2_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || window < 1 || topk < 0 || !(scale > 0.f)) return HS2_ERR_INVALID_ARG;
  if (window + topk > 2048) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!shape_ok(H, d)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace)) return HS2_ERR_WORKSPACE;
  const size_t need = hs2_full_attn_select_prefill_fp8kv_workspace_bytes(B, Lq, Lk, H, d, window, topk);
  if (need == 0 || workspace_bytes < need) return HS2_ERR_WORKSPACE;
  const int sms = num_sms();
  const size_t pre = align256(prefill::workspace_bytes(B, Lq, Lk, H, d, window, topk, sms, kStatusBytes));
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* kb = reinterpret_cast<__nv_bfloat16*>(base + pre);
  __nv_bfloat16* vb = reinterpret_cast<__nv_bfloat16*>(base + pre + fp8_cache_copy_bytes(B, Lk, d));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long n16 = (long long)B * Lk * d / 16;
  const int grid = (int)std::min<long long>((n16 + 255) / 256, (long long)sms * 8);
  {
    LaunchScope ls("widen_e4m3", st);
    if (launch_k(widen_e4m3_kernel, dim3(grid), dim3(256), 0, st, true, K8, k_scale, kb, n16) != cudaSuccess)
      return HS2_ERR_CUDA;
  }
  {
    LaunchScope ls("widen_e4m3", st);
    if (launch_k(widen_e4m3_kernel, dim3(grid), dim3(256), 0, st, true, V8, v_scale, vb, n16) != cudaSuccess)
      return HS2_ERR_CUDA;
  }
  return prefill::run(Q, reinterpret_cast<const hs2_bf16*>(kb), reinterpret_cast<const hs2_bf16*>(vb), B, Lq, Lk, H,
                      d, scale * 1.4426950408889634f, window, topk, out, lse, idx, workspace, pre, sms, kStatusBytes,
                      st);
}

hs2_status hs2_selftest_e4m3(const uint8_t* x, uint16_t* y_f16, uint16_t* y_bf16, int n, hs2_stream stream) {
  if (!x || !y_f16 || !y_bf16 || n < 0 || (n & 1)) return HS2_ERR_INVALID_ARG;
  if (n == 0) return HS2_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  selftest_e4m3_kernel<<<(n / 2 + 255) / 256, 256, 0, st>>>(x, y_f16, y_bf16, n / 2);
  return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

size_t hs2_bridge_kv_proj_workspace_bytes(int T, int hidden, int n_layers, int d) {
  if (T <= 0 || hidden <= 0 || n_layers <= 0 || d <= 0) return 0;
  return kStatusBytes;
}

hs2_status hs2_bridge_kv_proj(const hs2_bf16* Hs, int T, int hidden, const hs2_bf16* W, int n_layers, int d,
                              hs2_bf16* KV, void* workspace, size_t workspace_bytes, hs2_stream stream) {
  if (!Hs || !W || !KV) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Hs) || !aligned16(W) || !aligned16(KV)) return HS2_ERR_INVALID_ARG;
  if (T <= 0 || hidden <= 0 || n_layers <= 0 || d <= 0) return HS2_ERR_INVALID_ARG;
  if (hidden % 64 != 0 || (d != 64 && d != 128)) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || !aligned16(workspace) || workspace_bytes < kStatusBytes) return HS2_ERR_WORKSPACE;
  return prefill::run_bridge(Hs, T, hidden, W, n_layers, d, KV, reinterpret_cast<DevStatus*>(workspace),
                             reinterpret_cast<cudaStream_t>(stream));
}

hs2_status hs2_read_device_status(const void* workspace, hs2_stream stream) {
  if (!workspace) return HS2_ERR_WORKSPACE;
  DevStatus h{};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return HS2_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return HS2_ERR_CUDA;
  if (h.flags & kStatusTimeout) return HS2_ERR_DEVICE_TIMEOUT;
  if (h.flags & kStatusBounds) return HS2_ERR_DEVICE_BOUNDS;
  return HS2_OK;
}

hs2_status hs2_clear_device_status(void* workspace, hs2_stream stream) {
  if (!workspace) return HS2_ERR_WORKSPACE;
  // the whole status block: the status word and the decode grid barrier's counters
  if (cudaMemsetAsync(workspace, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HS2_ERR_CUDA;
  return HS2_OK;
}

hs2_status hs2_selftest_wait_timeout(void* workspace, size_t workspace_bytes, long long limit_ns, hs2_stream stream) {
  if (!workspace || workspace_bytes < kStatusBytes) return HS2_ERR_WORKSPACE;
  if (limit_ns <= 0 || limit_ns > 10000000000LL) return HS2_ERR_INVALID_ARG;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  {
    LaunchScope ls("selftest_wait", reinterpret_cast<cudaStream_t>(stream));
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<DevStatus*>(workspace), limit_ns);
  }
  return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

__global__ void selftest_exp2_kernel(const float* x, float* ys, float* ym, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n) return;
  float a = x[i], b = x[i + 1];
  ym[i] = fast_exp2(a);
  ym[i + 1] = fast_exp2(b);
  exp2_fma2(a, b);
  ys[i] = a;
  ys[i + 1] = b;
}

hs2_status hs2_selftest_exp2(const float* x, float* y_soft, float* y_mufu, int n, hs2_stream stream) {
  if (!x || !y_soft || !y_mufu || n <= 0 || (n & 1)) return HS2_ERR_INVALID_ARG;
  if (!device_is_sm100()) return HS2_ERR_UNSUPPORTED_SHAPE;
  {
    LaunchScope ls("selftest_exp2", reinterpret_cast<cudaStream_t>(stream));
    selftest_exp2_kernel<<<(n / 2 + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y_soft, y_mufu, n);
  }
  return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

unsigned long long hs2_kernel_launches(void) { return g_launches.load(); }

void hs2_profile_enable(const char* kernel) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (kernel) {
    g_prof_filter = kernel;
    g_prof_on = true;
  } else {
    g_prof_filter.clear();
    g_prof_on = false;
  }
}

int hs2_profile_read(const char* kernel, double* total_ms, long long* launches) {
  if (!kernel) return -1;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    auto it = g_prof.find(kernel);
    if (it != g_prof.end()) {
      recs.swap(it->second);
      g_prof.erase(it);
    }
  }
  double sum = 0.0;
  int rc = 0;
  for (auto& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.second) != cudaSuccess || cudaEventElapsedTime(&ms, r.first, r.second) != cudaSuccess)
      rc = -1;
    sum += ms;
  }
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : recs) {
      g_event_pool.push_back(r.first);
      g_event_pool.push_back(r.second);
    }
  }
  if (total_ms) *total_ms = sum;
  if (launches) *launches = (long long)recs.size();
  return rc;
}

}  // extern "C"
