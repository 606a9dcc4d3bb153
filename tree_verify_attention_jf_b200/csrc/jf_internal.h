// jf_internal.h -- declarations shared between the host entry points (jf_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace jf {

// Kernel attributes (dynamic shared memory, cluster size) are per device: each launch function keeps one
// flag per device and sets them the first time it launches on that device.
constexpr int kMaxDevices = 64;
inline int current_device() {
  int d = -1;
  return (cudaGetDevice(&d) == cudaSuccess && d >= 0 && d < kMaxDevices) ? d : -1;
}

// Every kernel of the library is launched with programmatic stream serialisation: it may be scheduled
// while the kernel before it on the stream is still running, does only local set-up (shared memory,
// barriers, TMEM, tensor-map prefetches) until its griddepcontrol.wait, and reads or writes global
// memory only after it.  Each kernel also signals griddepcontrol.launch_dependents early, so the next
// one's set-up overlaps its tail.  With no kernel before it, the wait returns at once.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              cudaLaunchAttribute* extra, Args&&... args) {
  cudaLaunchAttribute attrs[2];
  int n = 0;
  attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (extra != nullptr) attrs[n++] = *extra;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

constexpr int kHeadDim = 128;
constexpr int kPageSize = 16;
constexpr int kMaxTreeNodes = 256;          // nodes per sequence in jf_tree_attention
constexpr int kAncWords = kMaxTreeNodes / 32;
constexpr int kMaxAttnBatch = 1024;
constexpr int kMaxGrid = 256;               // persistent CTAs (one per SM, capped)
constexpr int kAttnRows = 128;              // rows of one M tile
constexpr int kAttnQTiles = 2;              // M tiles per work unit (they share every K/V tile)

struct AttnParams {
  const int32_t* block_table;
  const int32_t* prefix_lens;
  const int32_t* tree_offsets;
  const int32_t* parent;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;    // [2*kMaxGrid*2][32][128] float4 partial outputs (slot, column quad, row)
  float2* part_ml;  // [2*kMaxGrid*2][128] (running max in log2 units, row sum)
  int32_t* part_ok; // [2*kMaxGrid*2][128] 1 = the partial's sequence passed its device checks
  int4* units;      // [kMaxGrid] descriptor of the split unit whose first CTA is i (c1, first node, nodes, kv head)
  int32_t* status;
  int batch, total_nodes, hq, hkv, group, max_pages, num_pages;
  float scale_log2;  // softmax scale (times the K cache's scale for an 8-bit cache) times log2(e)
  float v_scale;     // the V cache's scale (1 for a bf16 cache)
};

// Workspace layout of jf_tree_attention (offsets in bytes, each 256-aligned).
struct AttnWorkspace {
  static constexpr size_t kSlots = 2 * kMaxGrid * kAttnQTiles;  // (CTA, first/last segment, Q tile)
  static constexpr size_t units_off = 0;
  static constexpr size_t units_bytes = sizeof(int4) * kMaxGrid;
  static constexpr size_t ok_off = units_off + ((units_bytes + 255) & ~size_t(255));
  static constexpr size_t ok_bytes = sizeof(int32_t) * kSlots * kAttnRows;
  static constexpr size_t ml_off = ok_off + ok_bytes;
  static constexpr size_t ml_bytes = sizeof(float2) * kSlots * kAttnRows;
  static constexpr size_t o_off = ml_off + ml_bytes;
  static constexpr size_t o_bytes = sizeof(float) * kSlots * kAttnRows * kHeadDim;
  static constexpr size_t total = o_off + o_bytes;
};

size_t attention_smem_bytes();
// fp8_cache: tm_k / tm_v describe 8-bit (E4M3) caches with whole 128-byte rows per box, no swizzle
cudaError_t launch_tree_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                  const AttnParams& p, int grid, bool fp8_cache, cudaStream_t stream);

// ---- tree build
constexpr int kMaxTopk = 8;
constexpr int kMaxDepths = 64;
constexpr int kMaxBudget = 1024;
constexpr int kStatsChunk = 4096;  // vocab entries per row-statistics CTA

struct RowPartial {  // one (row, chunk) of the draft logits
  double sum;        // sum of exp(x - m) over the chunk, float64
  float m;           // chunk max
  int pad;
  float val[kMaxTopk];
  int id[kMaxTopk];
};

size_t build_workspace_bytes(int batch, int depths, int vocab);
cudaError_t launch_build_tree(const float* logits, const int32_t* root_tokens, int batch, int depths, int vocab,
                              int topk, int budget, int max_depth, int32_t* parent, int32_t* token, float* score,
                              int32_t* depth, RowPartial* partials, int32_t* status, cudaStream_t stream);

// row statistics of `rows` logits rows per sequence (row stride `row_stride` rows); with lim_nodes / lim_begin
// only the frontier rows of each sequence whose tree holds fewer than lim_budget nodes are read
cudaError_t launch_row_stats(const float* logits, int batch, int rows, int row_stride, int vocab, int topk,
                             const int32_t* lim_nodes, const int32_t* lim_begin, int lim_budget,
                             RowPartial* partials, cudaStream_t stream);

// ---- frontier expansion from per-node draft logits
constexpr int kMaxFrontierBudget = 256;  // nodes per tree (= the attention's limit)

struct FrontierState {  // caller-owned, carried from one round to the next
  double* node_key;     // [B, budget] float64 key of every node
  double* cand_lp;      // [B, budget, topk] candidate children's log-probabilities
  int32_t* cand_tok;    // [B, budget, topk] their tokens
  int32_t* cand_next;   // [B, budget] first untaken rank per node
};

struct FrontierStateLayout {  // byte offsets in the state buffer, each 256-aligned
  size_t key_off, lp_off, tok_off, next_off, total;
  FrontierStateLayout(int batch, int budget, int topk) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t nodes = static_cast<size_t>(batch) * budget;
    key_off = 0;
    lp_off = up(key_off + nodes * sizeof(double));
    tok_off = up(lp_off + nodes * topk * sizeof(double));
    next_off = up(tok_off + nodes * topk * sizeof(int32_t));
    total = up(next_off + nodes * sizeof(int32_t));
  }
};

cudaError_t launch_expand_frontier(const float* logits, const int32_t* root_tokens, int batch, int rows, int vocab,
                                   int topk, int budget, int max_depth, int width, int32_t* parent, int32_t* token,
                                   float* score, int32_t* depth, int32_t* num_nodes, int32_t* frontier_begin,
                                   const FrontierState& st, RowPartial* partials, int32_t* status,
                                   cudaStream_t stream);

// ---- accept
constexpr int kMaxAcceptNodes = 1024;
cudaError_t launch_accept(const int32_t* token, const int32_t* parent, const float* logits, int batch,
                          int num_nodes, int vocab, int max_depth, int32_t* accepted_len, int32_t* path,
                          int32_t* bonus, int32_t* status, cudaStream_t stream);

// ---- KV commit
constexpr int kMaxCommitKvHeads = 64;
cudaError_t launch_commit_kv(void* k_cache, void* v_cache, const int32_t* block_table, int max_pages,
                             const int32_t* prefix_lens, const int32_t* tree_offsets, const int32_t* path,
                             const int32_t* accepted_len, int batch, int max_depth, int hkv, int num_pages,
                             int32_t* new_prefix_lens, int32_t* status, cudaStream_t stream);

// ---- tree K/V append with rotary positions
cudaError_t launch_tree_kv_append(const void* k_new, const void* v_new, void* q, void* k_cache, void* v_cache,
                                  const int32_t* block_table, int max_pages, const int32_t* prefix_lens,
                                  const int32_t* tree_offsets, const int32_t* depth, int batch, int total_nodes,
                                  int hq, int hkv, int num_pages, double theta, int32_t* status, cudaStream_t stream);

}  // namespace jf
