// Internal interfaces between the hs2 C-ABI layer (hs2_api.cu) and the kernel files.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_sched.h"

namespace hs2 {

struct DevStatus;

namespace dec {
// Parameters of the fused decode (one query per sequence) full-attention + selection kernel.
struct DecParams {
  int B, N, W, K;          // sequences, cache rows per sequence in K/V (the longest length), window, top-k
  Sched sch;               // per-sequence lengths and tiles, contiguous tile ranges per CTA
  float c;                 // scale * log2(e) (FP8 cache: times K's scale)
  long long wait_ns;       // bound of every device-side wait
  float* ml;               // [B*cmax][2][H] phase-1 partial (max, sum), log2 domain
  float* lse_out;          // [B][H] natural log (caller's lse)
  float* opart;            // [B*cmax][H][D] phase-2 partial outputs
  float* sc;               // [B][sc_stride] head-summed scores of the older tokens
  int sc_stride;           // max(N - W, 1): room for the longest sequence's older tokens
  unsigned* hist;          // [B][2048] histogram of score bits 30..20
  int* seq_done;           // [B] CTAs done with each sequence's histogram
  unsigned* bitmap;        // [B][words] selection bitmap of the older tokens (cleared here)
  int words;               // ceil(sc_stride / 32) rounded up to a multiple of 8 (32-byte rows)
  int* meta;               // [B][8] selection metadata (threshold bin, above, need, counters)
  int K_sel;               // top-k of the selection (== K)
  unsigned* gbar;          // grid-barrier arrivals: zero when a step starts; the sampled launch
                           // counts to G per group, the redo on from there (the collect kernel re-arms it)
  int sample_tiles;        // phase 1 samples about this many tiles per sequence (0: every tile)
  float* lp;               // [B*cmax][H] per-(sequence, CTA) sums of p' = exp2(s*c - lse2')
  float* lsum;             // [B][H] their totals L'_h (the output is sum(O') / L')
  float* lse2x;            // [B][H] exact lse, log2 units (for the exact re-score of the band)
  int* ovf;                // [B + 1] sequences whose p' overflowed the sampled reference (and a count)
  int fallback;            // 0: the sampled schedule; 1: redo the flagged sequences with every tile
  const int32_t* ptab;     // paged cache: [B][max_pages] page of each 128-token tile (NULL: contiguous)
  int max_pages, n_pages;  // table width, pages in the K/V pools
  float* blk_part;         // bf16 cache only, or NULL: [B][blk_groups][H] sums of p' over each group of
  int blk_groups;          // 32 consecutive keys per head (HySparse v1 block scores); ceil(N / 32)
  DevStatus* st;
};
size_t fused_smem_bytes(int H, int D, bool f8);
// f8: K and V are e4m3 caches (tensor maps of bytes, 128-byte rows); c then includes K's scale
cudaError_t launch_decode_attn(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                               const DecParams& p, bool f8, cudaStream_t stream);
}  // namespace dec

namespace sel {
constexpr int NBINS = 2048;
constexpr int META = 8;  // ints per sequence: bin above which all are in, their count, need, lowest band
                         // bin, band keys collected, band size expected
// Top-k selection over a materialised score vector per sequence (decode path).
struct SelParams {
  int B, N, W, K, S;              // N: cache rows per sequence in K (the longest length)
  int ncand;                     // max(N - W, 1): the stride of the per-sequence score and band
                                 // arrays; sequence b's own count is max(sch.seq_len[b] - W, 0)
  const float* sc;               // [B][ncand]
  const unsigned* hist;          // [B][NBINS]
  int* meta;                     // [B][META]
  unsigned* bitmap;              // [B][words] chosen older tokens, one bit each
  int words;
  unsigned long long* bnd;       // [B][ncand] boundary-bin candidates (score bits << 32 | ~index)
  int32_t* idx;                  // [B][S] output
  DevStatus* st;
  // output records of the decode kernel, summed into out by the collect kernel's extra CTAs
  const float* opart;            // unnormalised output records, at Sched::slot
  const float* lsum;             // [B][H] totals L' dividing them
  float oscale;                  // factor of the output (an e4m3 V cache's scale, else 1)
  __nv_bfloat16* out;            // [B][H][D]
  int H, D;
  dec::Sched sch;
  // exact re-score of the band keys
  const __nv_bfloat16* qry;      // [B][H][D] the decode queries
  const __nv_bfloat16* kc;       // [B][N][D] the K cache (sequence b's first seq_len[b] rows)
  const uint8_t* kc8;            // the same as e4m3 codes (FP8 cache; kc unused), c includes its scale
  const float* lse2x;            // [B][H] exact lse, log2 units
  float c;                       // scale * log2(e) (FP8 cache: times K's scale)
  int sms;
  unsigned* gbar;                // the decode kernel's grid-barrier counters, re-armed here
  const int32_t* ptab;           // paged cache: [B][max_pages] page ids, kc is the page pool (NULL: contiguous)
  int max_pages, n_pages;
  long long wait_ns;             // bound of the re-score kernel's wait for its MMA
};
cudaError_t launch_select(const SelParams& p, cudaStream_t stream);
}  // namespace sel

namespace blk {
// HySparse (v1) block-level selection after the fused decode kernel (blocksel.cu).
struct BlkParams {
  int B, H, D, W;                // sequences, heads, head dim, window
  int NB, BLK, S;                // blocks chosen, tokens per block (64), idx row length NB * BLK + W
  dec::Sched sch;                // per-sequence lengths (query at t = seq_len - 1)
  const float* blk_part;         // [B][blk_groups][H] the decode kernel's per-32-key sums of p'
  int blk_groups;
  const float* lsum;             // [B][H] L'_h (the exact p of a key is p' / L'_h)
  int max_blocks;                // ceil(N / BLK): the stride of bsc
  float* bsc;                    // [B][max_blocks] exact block scores
  int32_t* idx;                  // [B][S] output
  unsigned* gbar;                // the decode kernel's grid-barrier counters, re-armed here
  // decode output (the decode kernel's records / L')
  const float* opart;
  float oscale;
  __nv_bfloat16* out;
  DevStatus* st;
};
cudaError_t launch_block_select(const BlkParams& p, cudaStream_t stream);
}  // namespace blk

namespace bwd {
// Backward pass of the full layer (causal MQA attention) and of a sparse layer (backward.cu).
struct BwdParams {
  int B, Lq, Lk, H, D;
  int off;                    // Lk - Lq: query i sits at position off + i
  int rows_per_batch;         // Lq * H (query, head) rows per sequence
  int tiles_per_batch;        // ceil(rows_per_batch / 128)
  int kv_tiles;               // ceil(Lk / 128)
  int chunk;                  // row tiles per key-side work item
  int n_chunks;               // ceil(tiles_per_batch / chunk)
  float c;                    // scale * log2(e)
  float scale;
  const float* lse2;          // [B * Lq * H] forward logsumexp, log2 units
  const float* Dv;            // [B * Lq * H] <dO, out> per row
  __nv_bfloat16* dQ;          // [B, Lq, H, D]
  float* dK;                  // [B, Lk, D] accumulated (+=)
  float* dV;
  // sparse layer
  const __nv_bfloat16 *Q, *K, *V, *dO;
  const int32_t* idx;         // [B, Lq, S]
  int S;
  long long wait_ns;
  DevStatus* st;
};
cudaError_t launch_prep(const __nv_bfloat16* dO, const __nv_bfloat16* out, const float* lse, float* Dv, float* lse2,
                        long long n_rows, int D, cudaStream_t stream);
cudaError_t launch_full_bwd(const CUtensorMap& tmQ, const CUtensorMap& tmdO, const CUtensorMap& tmK,
                            const CUtensorMap& tmV, const BwdParams& p, int sms, cudaStream_t stream);
cudaError_t launch_sparse_bwd(const BwdParams& p, int sms, cudaStream_t stream);
}  // namespace bwd

namespace sparse {
struct SpParams {
  const __nv_bfloat16 *Q, *K, *V;
  const uint8_t *K8, *V8;     // FP8 cache: e4m3 codes (K, V unused); c includes K's scale
  float oscale;               // factor of the output (the e4m3 V cache's scale, else 1)
  const int32_t* idx;
  int B, Lq, Lk, S;
  int nsplit, split_slots;    // CTAs per query row (a cluster when > 1, at most 16) and the
                              // idx slots each handles (a multiple of 128)
  float c;                    // scale * log2(e) (FP8 cache: times K's scale)
  __nv_bfloat16* out;
  float* lse;                 // may be null
  long long wait_ns;
  const int32_t* ptab;        // paged cache: [B][max_pages] page ids, K/V are the page pools of
  int max_pages, n_pages;     // n_pages x 128 rows (NULL: K/V are [B][Lk] rows)
  // two gated branches (HySparse v1): splits [0, branch_split) attend over the block branch,
  // the rest over the window branch; out = g * (block branch) + (1 - g) * (window branch) with
  // g = gate[row][head]. NULL: one softmax over every slot.
  const float* gate;
  int branch_split;
  DevStatus* st;
};
size_t sparse_smem_bytes(int H, int D, int nsplit);
cudaError_t launch_sparse(const SpParams& p, int H, int D, cudaStream_t stream);
}  // namespace sparse

}  // namespace hs2
