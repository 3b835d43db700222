/*
 * hs2.h -- C ABI of the B200 (sm_100a) HySparse2 hot path.
 *
 * Operations, as the pages about "HySparse2: Hybrid Sparse Attention with Two-Level KV
 * Sharing" state the problem:
 *
 *  hs2_full_attn_select  A causal multi-query full-attention layer (64 query heads share
 *                        one K/V head: arex-research.com article "小米 MiMo 负责人罗福利公开
 *                        MiMo-V3 核心架构 HySparse2", section "三套 80B-A3B 对照模型里算出的数字")
 *                        that also acts as the indexer: from its exact attention scores it
 *                        selects, for every query position t, the `window` most recent tokens
 *                        t-window+1..t plus the `topk` highest-scoring older tokens 0..t-window
 *                        (same article, section "外层 KV Bridging，内层 KV Reuse"; toolnavs.com
 *                        HySparse2 article, section "Was HySparse2 tut"; zgeo.com.cn article,
 *                        section "核心技术原理解析": 128 + 1,024 tokens).
 *                        The pages leave open how the heads' scores are combined. This library
 *                        scores token j for query t as the sum over heads of the post-softmax
 *                        probability (softmax over the whole causal row 0..t); equal scores go
 *                        to the lower index.
 *  hs2_sparse_attn       A sparse layer of the same hybrid block: reuses the full layer's K/V
 *                        cache and selection indices unchanged, with its own Q, and attends
 *                        only to the selected tokens (arex-research.com, section "外层 KV
 *                        Bridging，内层 KV Reuse"; toolnavs.com, section "Was HySparse2 tut").
 *  hs2_bridge_kv_proj    KV Bridging: one self-decoder hidden state H is projected by several
 *                        cross-decoder layers' own W_k / W_v (arex-research.com, section
 *                        "外层 KV Bridging，内层 KV Reuse"; toolnavs.com, section "Was HySparse2
 *                        tut"), computed as one batched GEMM.
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers (cudaMalloc / torch memory), row-major,
 *    contiguous, 16-byte aligned, owned by the caller. bf16 values are passed as
 *    hs2_bf16 (the 16-bit pattern). Inputs are read only; outputs must not alias inputs.
 *  - `workspace` is caller-owned device scratch of at least the size the matching
 *    *_workspace_bytes query returns. Its first 256 bytes are the status block: the device
 *    status word (first 16 bytes) and the counters of the decode kernel's grid barrier. Zero-
 *    fill a workspace before its first use (cudaMemset, torch.zeros); every call leaves it
 *    ready for the next one. After a device-side error, hs2_clear_device_status re-arms it.
 *    The library never allocates, frees or synchronises inside the compute calls.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *    Arguments are validated on the host before anything is launched; a non-zero return
 *    means nothing was launched (HS2_ERR_CUDA: a launch failed).
 *  - Device-side problems (a bounded wait that gave up, an index out of range) never trap:
 *    the kernel records them in the status word and returns. Read them with
 *    hs2_read_device_status.
 *  - There is no CPU fallback: a device that is not sm_100 returns
 *    HS2_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HS2_ABI_VERSION 1

#if defined(__GNUC__)
#define HS2_API __attribute__((visibility("default")))
#else
#define HS2_API
#endif

typedef uint16_t hs2_bf16; /* bf16 bit pattern */
typedef void* hs2_stream;  /* cudaStream_t */

typedef enum {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = 1,       /* null / misaligned pointer, negative or inconsistent size */
  HS2_ERR_UNSUPPORTED_SHAPE = 2, /* (H, d) not supported, or the device is not sm_100 */
  HS2_ERR_WORKSPACE = 3,         /* workspace missing or smaller than required */
  HS2_ERR_CUDA = 4,              /* a CUDA runtime call or kernel launch failed */
  HS2_ERR_DEVICE_TIMEOUT = 5,    /* a kernel's bounded wait gave up (status word) */
  HS2_ERR_DEVICE_BOUNDS = 6      /* a kernel saw an index outside [0, Lk) (status word) */
} hs2_status;

/* ABI version of the loaded library (HS2_ABI_VERSION at build time). */
HS2_API int hs2_abi_version(void);

/* Static, human-readable text of a status code. */
HS2_API const char* hs2_status_string(hs2_status s);

/* ---------------------------------------------------------------------------------
 * Full attention + token selection
 * ---------------------------------------------------------------------------------
 * Q    [B, Lq, H, d] bf16  queries; query i sits at position t = Lk - Lq + i
 *                           (Lq == Lk: prefill over the whole sequence; 1 < Lq < Lk: a chunk of
 *                           Lq new tokens appended to an Lk - Lq token cache, whose K/V rows are
 *                           already the last Lq cache rows; Lq == 1: one decode step)
 * K, V [B, Lk, d]    bf16  the single K/V head
 * scale                     softmax scale applied to q.k (e.g. 1/sqrt(d))
 * window, topk              forced recent tokens and number of older tokens chosen by score
 *                           (the pages: 128 and 1,024); window >= 1, topk >= 0
 * out  [B, Lq, H, d] bf16  softmax(scale q K^T) V over the causal row
 * lse  [B, Lq, H]    fp32  natural-log logsumexp of the scaled logits of the causal row
 * idx  [B, Lq, window+topk] int32  selected token indices of each query, ascending;
 *                           exactly min(t+1, window+topk) valid entries, then -1 padding
 * Supported: (H, d) in {(64, 128), (16, 64)}, 1 <= Lq <= Lk (bf16, fp32 accumulate). Lq == 1
 * with (H, d) = (64, 128) runs the decode kernels (B <= 256); every other shape runs the prefill
 * kernels, which support topk <= 1024.
 */
HS2_API size_t hs2_full_attn_select_workspace_bytes(int B, int Lq, int Lk, int H, int d, int window, int topk);
HS2_API hs2_status hs2_full_attn_select(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lq, int Lk,
                                int H, int d, float scale, int window, int topk, hs2_bf16* out, float* lse,
                                int32_t* idx, void* workspace, size_t workspace_bytes, hs2_stream stream);

/* Ragged decode: one query per sequence, sequence b with its own cache length lens[b] (the
 * per-sequence N of multi-turn agent serving, whose short actions and long, accumulating
 * observations the pages take as the setting: arex-research.com, the lead and section
 * "短动作、长观测：prefill、KV cache 与检索同时成为瓶颈").
 * lens is a HOST array of B lengths, 1 <= lens[b] <= Lk, read before the call returns (the
 * work split across SMs is computed from it on the host). K, V are [B, Lk, d]: sequence b's
 * cache is its first lens[b] rows, the rest is never read. Q, out [B, 1, H, d]; lse [B, 1, H];
 * idx [B, 1, window+topk] as above, sequence b's query sitting at t = lens[b] - 1. Every
 * sequence's result equals hs2_full_attn_select on that sequence alone. Supported: (H, d) =
 * (64, 128), 1 <= B <= 256. The workspace size depends on lens (query it with the same lens).
 */
HS2_API size_t hs2_full_attn_select_ragged_workspace_bytes(int B, const int32_t* lens, int Lk, int H, int d,
                                                           int window, int topk);
HS2_API hs2_status hs2_full_attn_select_ragged(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B,
                                               const int32_t* lens, int Lk, int H, int d, float scale, int window,
                                               int topk, hs2_bf16* out, float* lse, int32_t* idx, void* workspace,
                                               size_t workspace_bytes, hs2_stream stream);

/* Paged decode: as the ragged call, with each sequence's cache in pages of 128 tokens of shared
 * pools (a serving system's block-allocated KV cache).
 * K_pages, V_pages [n_pages, 128, d] bf16  the page pools
 * page_table [B, max_pages] int32 (DEVICE)  page of sequence b's tokens 128 i .. 128 i + 127; only
 *                           the first ceil(lens[b] / 128) entries of a row are read; an id outside
 *                           [0, n_pages) is recorded as HS2_ERR_DEVICE_BOUNDS (its rows read as 0)
 * lens [B] int32 (HOST)     1 <= lens[b] <= 128 * max_pages
 * Rows of a sequence's last page past lens[b] are never used. The results equal the ragged call
 * on the same tokens laid out contiguously. Supported: (H, d) = (64, 128), 1 <= B <= 256.
 */
HS2_API size_t hs2_full_attn_select_paged_workspace_bytes(int B, const int32_t* lens, int max_pages, int H, int d,
                                                          int window, int topk);
HS2_API hs2_status hs2_full_attn_select_paged(const hs2_bf16* Q, const hs2_bf16* K_pages, const hs2_bf16* V_pages,
                                              int n_pages, const int32_t* page_table, int max_pages, int B,
                                              const int32_t* lens, int H, int d, float scale, int window, int topk,
                                              hs2_bf16* out, float* lse, int32_t* idx, void* workspace,
                                              size_t workspace_bytes, hs2_stream stream);

/* FP8 cache: the decode step over a K/V cache stored as 8-bit floats (the pages' KV-cache cost
 * figures at 1M tokens are quoted for FP8 storage: arex-research.com, section "三套 80B-A3B
 * 对照模型里算出的数字", the cost paragraph).
 * K8, V8     e4m3 codes (OCP FP8: sign, 4 exponent bits with bias 7, 3 mantissa bits,
 *            subnormals; 0x7F / 0xFF are NaN), [B, Lk, d] rows, or with a page table the pools
 *            [n_pages, 128, d] as for hs2_full_attn_select_paged (then Lk == 128 * max_pages)
 * k_scale, v_scale  per-tensor factors, positive and finite: the cache holds K = k_scale * K8,
 *            V = v_scale * V8 (a power of two keeps every value exact in bf16)
 * lens       HOST array of B lengths (1 <= lens[b] <= Lk), or NULL: every sequence Lk tokens
 * Q, out, lse, idx as for the ragged call; results equal that call on the dequantised bf16 cache
 * (every e4m3 value times a power of two is a bf16 value). The kernels read the codes (half the
 * bytes of bf16) and widen them exactly on chip. Supported: (H, d) = (64, 128), one query per
 * sequence, 1 <= B <= 256. Workspace: hs2_full_attn_select_fp8kv_workspace_bytes with the same
 * B, lens (or NULL) and Lk.
 */
HS2_API size_t hs2_full_attn_select_fp8kv_workspace_bytes(int B, const int32_t* lens, int Lk, int H, int d,
                                                          int window, int topk);
HS2_API hs2_status hs2_full_attn_select_fp8kv(const hs2_bf16* Q, const uint8_t* K8, const uint8_t* V8, float k_scale,
                                              float v_scale, int B, const int32_t* lens, int Lk,
                                              const int32_t* page_table, int max_pages, int n_pages, int H, int d,
                                              float scale, int window, int topk, hs2_bf16* out, float* lse,
                                              int32_t* idx, void* workspace, size_t workspace_bytes,
                                              hs2_stream stream);

/* Whole prompts and chunks over an FP8 cache: the arguments of hs2_full_attn_select with K8, V8
 * [B, Lk, d] e4m3 codes and k_scale, v_scale as above. Lq == 1 with (H, d) = (64, 128) runs the
 * FP8 decode kernels (as hs2_full_attn_select_fp8kv with lens NULL); otherwise the cache is
 * widened once into the workspace as bf16 (k_scale * K8, v_scale * V8, rounded to bf16: exact for
 * power-of-two scales) and the prefill kernels run on it (they are tensor-bound and read the cache
 * from L2 many times). Results equal hs2_full_attn_select on that bf16 cache. Supported: as
 * hs2_full_attn_select. Workspace: hs2_full_attn_select_prefill_fp8kv_workspace_bytes.
 */
HS2_API size_t hs2_full_attn_select_prefill_fp8kv_workspace_bytes(int B, int Lq, int Lk, int H, int d, int window,
                                                                  int topk);
HS2_API hs2_status hs2_full_attn_select_prefill_fp8kv(const hs2_bf16* Q, const uint8_t* K8, const uint8_t* V8,
                                                      float k_scale, float v_scale, int B, int Lq, int Lk, int H,
                                                      int d, float scale, int window, int topk, hs2_bf16* out,
                                                      float* lse, int32_t* idx, void* workspace,
                                                      size_t workspace_bytes, hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * Sparse attention over selected tokens (one sparse layer)
 * ---------------------------------------------------------------------------------
 * Q    [B, Lq, H, d] bf16  this layer's own queries
 * K, V [B, Lk, d]    bf16  the full layer's K/V cache, reused unchanged
 * idx  [B, Lq, S]    int32 the full layer's selection, reused unchanged; -1 slots are skipped,
 *                           any other value must lie in [0, Lk) (else the status word records
 *                           HS2_ERR_DEVICE_BOUNDS and the row's output is unspecified).
 *                           Every row needs at least one valid entry.
 * out  [B, Lq, H, d] bf16  softmax over the selected tokens of scale q.k, times V
 * lse  [B, Lq, H]    fp32  natural-log logsumexp over the selected tokens, or NULL
 * Supported: (H, d) in {(64, 128), (16, 64)}, 1 <= S <= 4096.
 */
HS2_API size_t hs2_sparse_attn_workspace_bytes(int B, int Lq, int Lk, int H, int d, int S);
HS2_API hs2_status hs2_sparse_attn(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx, int B,
                           int Lq, int Lk, int H, int d, int S, float scale, hs2_bf16* out, float* lse,
                           void* workspace, size_t workspace_bytes, hs2_stream stream);
/* Sparse attention over a paged cache: K_pages, V_pages, page_table, max_pages and n_pages as for
 * hs2_full_attn_select_paged; idx [B, Lq, S] holds token positions (< 128 * max_pages) of each
 * sequence, mapped through its page-table row. Workspace: hs2_sparse_attn_workspace_bytes with
 * Lk = 128 * max_pages. An out-of-pool page id is recorded as HS2_ERR_DEVICE_BOUNDS and its token
 * skipped.
 */
HS2_API hs2_status hs2_sparse_attn_paged(const hs2_bf16* Q, const hs2_bf16* K_pages, const hs2_bf16* V_pages,
                                         int n_pages, const int32_t* page_table, int max_pages, const int32_t* idx,
                                         int B, int Lq, int H, int d, int S, float scale, hs2_bf16* out, float* lse,
                                         void* workspace, size_t workspace_bytes, hs2_stream stream);

/* Sparse attention over an FP8 cache: K8, V8, k_scale, v_scale (and the optional page table,
 * with Lk == 128 * max_pages) as for hs2_full_attn_select_fp8kv; every other argument as for
 * hs2_sparse_attn, whose workspace size applies. Results equal hs2_sparse_attn on the
 * dequantised bf16 cache. Supported: (H, d) in {(64, 128), (16, 64)}, 1 <= S <= 4096.
 */
HS2_API hs2_status hs2_sparse_attn_fp8kv(const hs2_bf16* Q, const uint8_t* K8, const uint8_t* V8, float k_scale,
                                         float v_scale, const int32_t* idx, int B, int Lq, int Lk,
                                         const int32_t* page_table, int max_pages, int n_pages, int H, int d, int S,
                                         float scale, hs2_bf16* out, float* lse, void* workspace,
                                         size_t workspace_bytes, hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * Backward pass (training the hybrid block)
 * ---------------------------------------------------------------------------------
 * The full-attention layers are trained natively as the indexer (arex-research.com, section
 * "外层 KV Bridging，内层 KV Reuse"), and the sparse layers train through the selection, which is
 * a constant of the backward pass (it has no gradient). For the upstream gradient dO of a layer's
 * output these calls compute, with p the forward's softmax probabilities over a row's key set
 * (the causal row 0..t for the full layer, the selected slots for a sparse layer):
 *   dQ = scale sum_j dS_j k_j,  dK_j += scale sum dS_j q,  dV_j += sum p_j dO,
 *   dS_j = p_j (dO.v_j - dO.out),
 * the K and V sums running over every head and every row that reads key j.
 * Q, dO, out [B, Lq, H, d] bf16 (out and lse are the forward call's outputs for these Q, K, V:
 *     hs2_full_attn_select's, or hs2_sparse_attn's with its lse); lse [B, Lq, H] fp32 natural log;
 * K, V [B, Lk, d] bf16; idx [B, Lq, S] (sparse: the forward's selection).
 * dQ [B, Lq, H, d] bf16 (written).
 * dK, dV [B, Lk, d] fp32, ACCUMULATED (+=): the full layer and every sparse layer of a block read
 *     the same K/V (KV Reuse), so their backward calls add into one pair of buffers; zero them
 *     before the block's first backward call. The additions use atomics (their order, and so the
 *     last bits of the sums, may vary from run to run).
 * Causal alignment as in the forward (query i at t = Lk - Lq + i). Supported: (H, d) in
 * {(64, 128), (16, 64)}; sparse S <= 4096. Workspace: hs2_attn_bwd_workspace_bytes (status block
 * plus two floats per (query, head) row).
 */
HS2_API size_t hs2_attn_bwd_workspace_bytes(int B, int Lq, int Lk, int H, int d);
HS2_API hs2_status hs2_full_attn_bwd(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const hs2_bf16* out,
                                     const float* lse, const hs2_bf16* dO, int B, int Lq, int Lk, int H, int d,
                                     float scale, hs2_bf16* dQ, float* dK, float* dV, void* workspace,
                                     size_t workspace_bytes, hs2_stream stream);
HS2_API hs2_status hs2_sparse_attn_bwd(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx,
                                       const hs2_bf16* out, const float* lse, const hs2_bf16* dO, int B, int Lq,
                                       int Lk, int H, int d, int S, float scale, hs2_bf16* dQ, float* dK, float* dV,
                                       void* workspace, size_t workspace_bytes, hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * HySparse (v1) variant: block-level selection and a gated sliding-window branch
 * ---------------------------------------------------------------------------------
 * The predecessor design the pages compare HySparse2 against (arex-research.com, section
 * "外层 KV Bridging，内层 KV Reuse", the paragraph on what HySparse2 changes): the full layer picks
 * its 1,024 global tokens as 16 blocks of 64 consecutive tokens, and each sparse layer adds a
 * separate 128-token sliding-window branch fused with the block branch by a gate. The pages do not
 * give the block score or the gate; this library reads them as:
 *  - block score of block J for the query at t: the sum of score(t, j) (the head-summed
 *    probability defined for hs2_full_attn_select) over the block's tokens j <= t; every block
 *    starting at or before t competes; ties go to the lower block. With at most n_blocks blocks
 *    meeting 0..t, every token 0..t is taken.
 *  - gate: a caller-given g in [0, 1] per (query, head), out = g * O_blocks + (1 - g) * O_window,
 *    each branch its own softmax.
 *
 * hs2_full_attn_select_v1: the decode step's full layer (one query per sequence, at t = Lk - 1)
 * Q [B, 1, H, d], K, V [B, Lk, d] bf16; out, lse as for hs2_full_attn_select.
 * idx [B, 1, n_blocks * block + window] int32: slots [0, n_blocks * block) hold the chosen blocks'
 *     tokens <= t in ascending order, then -1; slots [n_blocks * block, +window) hold the window
 *     t - window + 1 .. t (clamped at 0) ascending, then -1.
 * Supported: (H, d) = (64, 128), block = 64, 1 <= n_blocks <= 32, n_blocks * block + window <= 2048,
 * 1 <= B <= 256. The selection is exact: the decode kernel's bounded token scores bound every
 * block's score, and the blocks that can reach the top n_blocks are re-scored exactly.
 * Workspace: hs2_full_attn_select_v1_workspace_bytes (zero-filled before first use).
 *
 * hs2_sparse_attn_v1: one sparse layer of the v1 design, with the full layer's K/V and idx.
 * idx [B, Lq, S]: slots [0, branch) the block branch, [branch, S) the window branch (-1 skipped;
 *     each branch needs one valid entry); gate [B, Lq, H] fp32 in [0, 1] (DEVICE).
 * out [B, Lq, H, d] bf16 = gate * softmax-attention over the block branch + (1 - gate) *
 *     softmax-attention over the window branch. branch % 128 == 0, 0 < branch < S <= 2048,
 *     (H, d) = (64, 128). Workspace: hs2_sparse_attn_workspace_bytes(B, Lq, Lk, H, d, S).
 */
HS2_API size_t hs2_full_attn_select_v1_workspace_bytes(int B, int Lk, int H, int d, int window, int block,
                                                       int n_blocks);
HS2_API hs2_status hs2_full_attn_select_v1(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lk,
                                           int H, int d, float scale, int window, int block, int n_blocks,
                                           hs2_bf16* out, float* lse, int32_t* idx, void* workspace,
                                           size_t workspace_bytes, hs2_stream stream);
HS2_API hs2_status hs2_sparse_attn_v1(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx,
                                      const float* gate, int B, int Lq, int Lk, int H, int d, int S, int branch,
                                      float scale, hs2_bf16* out, void* workspace, size_t workspace_bytes,
                                      hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * Sparse attention without a caller workspace
 * ---------------------------------------------------------------------------------
 * No counterpart in the paper: a library convenience for callers that cannot allocate
 * device memory -- e.g. a plugin's enqueue hook inside an inference runtime that forbids
 * allocation on that path and offers no scratch buffer, or a process whose device-memory
 * budget is fixed up front. Same arguments and results as hs2_sparse_attn, minus the
 * workspace: the scratch is a 4 KiB array inside the library, held by every GPU that loads
 * it until process exit. Returns HS2_ERR_WORKSPACE (nothing launched) when the shape needs
 * more scratch than that (hs2_sparse_attn_workspace_bytes(...) > 4 KiB; with the current
 * kernels every supported shape needs only its 256-byte status word). The first call on
 * each device performs a one-time set-up (it looks up the array's device address) and should
 * come before any stream capture; the address is cached per device with the device's context,
 * and looked up again when a call finds another context (after cudaDeviceReset). All calls
 * share the array: calls whose GPU work overlaps (e.g. on different streams) race. Each call
 * clears the status word in the array before its kernels run.
 * No cudaMalloc / cudaFree is ever called.
 */
HS2_API hs2_status hs2_sparse_attn_noalloc(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                                           const int32_t* idx, int B, int Lq, int Lk, int H, int d, int S,
                                           float scale, hs2_bf16* out, float* lse, hs2_stream stream);
/* Device status of the latest hs2_sparse_attn_noalloc call on the current device: waits for
 * `stream` (the stream of that call) and returns HS2_OK, HS2_ERR_DEVICE_BOUNDS (an idx entry
 * outside [0, Lk): it was skipped, so that row's output is unspecified) or
 * HS2_ERR_DEVICE_TIMEOUT (a bounded wait gave up), as hs2_read_device_status does for a
 * workspace; HS2_ERR_WORKSPACE if no call has set up this device yet. */
HS2_API hs2_status hs2_sparse_attn_noalloc_status(hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * KV Bridging projection
 * ---------------------------------------------------------------------------------
 * Hs   [T, hidden]                bf16  shared hidden state
 * W    [n_layers, 2, hidden, d]   bf16  per layer: W_k (index 0) then W_v (index 1)
 * KV   [n_layers, 2, T, d]        bf16  K_l = Hs W[l,0], V_l = Hs W[l,1] (fp32 accumulate)
 * Supported: hidden % 64 == 0, d in {64, 128}.
 */
HS2_API size_t hs2_bridge_kv_proj_workspace_bytes(int T, int hidden, int n_layers, int d);
HS2_API hs2_status hs2_bridge_kv_proj(const hs2_bf16* Hs, int T, int hidden, const hs2_bf16* W, int n_layers, int d,
                              hs2_bf16* KV, void* workspace, size_t workspace_bytes, hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * Device status
 * ---------------------------------------------------------------------------------
 * hs2_read_device_status: waits for `stream`, reads the status word of `workspace` and
 * returns HS2_OK, HS2_ERR_DEVICE_TIMEOUT or HS2_ERR_DEVICE_BOUNDS (HS2_ERR_CUDA if the
 * read failed). hs2_clear_device_status: zeroes the status block (the word and the grid
 * barrier's counters; asynchronously, on `stream`).
 * hs2_set_wait_limit_ns: wall-time bound of every device-side wait of later launches
 * (default 2 s, or the environment variable HS2_WAIT_LIMIT_MS at first use).
 * hs2_selftest_wait_timeout: launches one kernel whose bounded wait is on a barrier that
 * nothing completes; it gives up after `limit_ns`, records HS2_ERR_DEVICE_TIMEOUT in the
 * status word and returns, leaving the context usable (a failure-detection test hook).
 */
HS2_API hs2_status hs2_read_device_status(const void* workspace, hs2_stream stream);
HS2_API hs2_status hs2_clear_device_status(void* workspace, hs2_stream stream);
HS2_API void hs2_set_wait_limit_ns(long long limit_ns);
HS2_API hs2_status hs2_selftest_wait_timeout(void* workspace, size_t workspace_bytes, long long limit_ns, hs2_stream stream);

/* hs2_selftest_exp2: evaluates, for the n device floats x[i] (n even), the software 2^x the
 * score pass computes on the FMA pipes (into y_soft) and the hardware approximation (MUFU ex2,
 * flushing subnormals) it is mixed with (into y_mufu), so a test can bound their error. No
 * counterpart in the paper: a check of an arithmetic building block. */
HS2_API hs2_status hs2_selftest_exp2(const float* x, float* y_soft, float* y_mufu, int n, hs2_stream stream);
/* hs2_selftest_e4m3: widens the n device e4m3 codes x (n even) with the conversions the FP8-cache
 * kernels use, to f16 bit patterns (y_f16) and bf16 bit patterns (y_bf16), so a test can check
 * them against the format's definition. */
HS2_API hs2_status hs2_selftest_e4m3(const uint8_t* x, uint16_t* y_f16, uint16_t* y_bf16, int n, hs2_stream stream);

/* ---------------------------------------------------------------------------------
 * Diagnostics (never needed on the compute path)
 * ---------------------------------------------------------------------------------
 * hs2_kernel_launches: number of CUDA kernels this library has launched since it was
 * loaded (all devices, all streams).
 * hs2_profile_enable: NULL turns per-kernel timing off; "*" times every kernel; any other
 * string times only the kernel of that name (e.g. "dec_fused", "sparse_attn"). While on,
 * the library records a pair of CUDA events around each matching launch on its stream; on a
 * stream being captured into a CUDA graph they become event-record nodes of the graph (the
 * events then hold the latest replay's times, and must be read before the events are reused).
 * hs2_profile_read: waits for the recorded events of `kernel`, returns their summed
 * duration in milliseconds and the number of launches, and forgets them. Returns 0, or -1
 * if an event could not be read.
 */
HS2_API unsigned long long hs2_kernel_launches(void);
HS2_API void hs2_profile_enable(const char* kernel);
HS2_API int hs2_profile_read(const char* kernel, double* total_ms, long long* launches);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H_ */
