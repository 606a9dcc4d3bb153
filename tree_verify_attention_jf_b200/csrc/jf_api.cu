// jf_api.cu -- the C ABI of libjf.so (declared in include/jf.h): argument validation, TMA tensor-map
// encoding, workspace carving and kernel launches.  Every check that needs no device data runs
// before the first CUDA call, so a bad argument never launches anything.
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/jf.h"
#include "jf_internal.h"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count() {
  static std::atomic<int> counts[jf::kMaxDevices];
  const int dev = jf::current_device();
  if (dev < 0) return -1;
  int n = counts[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    counts[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// 3-D tensor map, dims innermost first, out-of-range boxes read as zero: bf16 with 128-byte swizzle, or
// 8-bit elements (E4M3 codes) with no swizzle.
bool encode_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
               uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2, bool bytes = false) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            bytes ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// jf_tree_attention and jf_tree_attention_fp8: validation, tensor maps, workspace carving, launch.
jf_status tree_attention_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                              int max_pages_per_seq, const int32_t* prefix_lens, const int32_t* tree_offsets,
                              const int32_t* parent, int batch, int total_nodes, int num_q_heads, int num_kv_heads,
                              int head_dim, int page_size, int num_pages, float sm_scale, bool fp8, float k_scale,
                              float v_scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                              int32_t* dev_status, jf_stream_t stream) {
  using namespace jf;
  if (batch < 0 || total_nodes < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_pages_per_seq <= 0 ||
      num_pages <= 0)
    return JF_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return JF_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale))
    return JF_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale * k_scale)) return JF_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || page_size != kPageSize) return JF_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return JF_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return JF_ERR_UNSUPPORTED;
  if (batch > kMaxAttnBatch) return JF_ERR_UNSUPPORTED;
  if (static_cast<long long>(num_pages) * kPageSize >= (1ll << 31)) return JF_ERR_UNSUPPORTED;
  if (batch == 0 || total_nodes == 0) return JF_OK;
  if (!q || !k_cache || !v_cache || !block_table || !prefix_lens || !tree_offsets || !parent || !out || !workspace)
    return JF_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(workspace, 256))
    return JF_ERR_INVALID_ARG;
  if (workspace_bytes < AttnWorkspace::total) return JF_ERR_INVALID_ARG;

  const int sms = sm_count();
  if (sms <= 0) return JF_ERR_CUDA;
  const int grid = sms < kMaxGrid ? sms : kMaxGrid;

  CUtensorMap tm_q, tm_k, tm_v;
  const uint64_t row = kHeadDim * sizeof(__nv_bfloat16);  // 256 bytes
  if (!encode_3d(&tm_q, q, kHeadDim, num_q_heads, total_nodes, row, row * num_q_heads, 64, group,
                 kAttnRows / group))
    return JF_ERR_CUDA;
  const uint64_t slots = static_cast<uint64_t>(num_pages) * kPageSize;
  if (fp8) {  // one byte per element: whole 128-byte rows, 16 slots a box
    if (!encode_3d(&tm_k, k_cache, kHeadDim, num_kv_heads, slots, kHeadDim, kHeadDim * num_kv_heads, kHeadDim, 1,
                   kPageSize, true))
      return JF_ERR_CUDA;
    if (!encode_3d(&tm_v, v_cache, kHeadDim, num_kv_heads, slots, kHeadDim, kHeadDim * num_kv_heads, kHeadDim, 1,
                   kPageSize, true))
      return JF_ERR_CUDA;
  } else {
    if (!encode_3d(&tm_k, k_cache, kHeadDim, num_kv_heads, slots, row, row * num_kv_heads, 64, 1, kPageSize))
      return JF_ERR_CUDA;
    if (!encode_3d(&tm_v, v_cache, kHeadDim, num_kv_heads, slots, row, row * num_kv_heads, 64, 1, kPageSize))
      return JF_ERR_CUDA;
  }

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  AttnParams p;
  p.block_table = block_table;
  p.prefix_lens = prefix_lens;
  p.tree_offsets = tree_offsets;
  p.parent = parent;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.units = reinterpret_cast<int4*>(ws + AttnWorkspace::units_off);
  p.part_ok = reinterpret_cast<int32_t*>(ws + AttnWorkspace::ok_off);
  p.part_ml = reinterpret_cast<float2*>(ws + AttnWorkspace::ml_off);
  p.part_o = reinterpret_cast<float*>(ws + AttnWorkspace::o_off);
  p.status = dev_status;
  p.batch = batch;
  p.total_nodes = total_nodes;
  p.hq = num_q_heads;
  p.hkv = num_kv_heads;
  p.group = group;
  p.max_pages = max_pages_per_seq;
  p.num_pages = num_pages;
  p.scale_log2 = sm_scale * k_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  if (launch_tree_attention(tm_q, tm_k, tm_v, p, grid, fp8, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JF_ERR_CUDA;
  return JF_OK;
}

}  // namespace

extern "C" {

const char* jf_status_string(int status) {
  switch (status) {
    case JF_OK: return "JF_OK";
    case JF_ERR_INVALID_ARG: return "JF_ERR_INVALID_ARG";
    case JF_ERR_UNSUPPORTED: return "JF_ERR_UNSUPPORTED";
    case JF_ERR_CUDA: return "JF_ERR_CUDA";
    case JF_ERR_DEVICE_CHECK: return "JF_ERR_DEVICE_CHECK";
    case JF_ERR_TIMEOUT: return "JF_ERR_TIMEOUT";
    default: return "JF_ERR_UNKNOWN";
  }
}

int jf_version(void) { return 10000; }

size_t jf_tree_attention_workspace_size(int batch, int num_q_heads, int num_kv_heads, int total_nodes) {
  (void)batch;
  (void)num_q_heads;
  (void)num_kv_heads;
  (void)total_nodes;
  return jf::AttnWorkspace::total;
}

jf_status jf_tree_attention(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                            int max_pages_per_seq, const int32_t* prefix_lens, const int32_t* tree_offsets,
                            const int32_t* parent, int batch, int total_nodes, int num_q_heads, int num_kv_heads,
                            int head_dim, int page_size, int num_pages, float sm_scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream) {
  return tree_attention_call(q, k_cache, v_cache, block_table, max_pages_per_seq, prefix_lens, tree_offsets, parent,
                             batch, total_nodes, num_q_heads, num_kv_heads, head_dim, page_size, num_pages, sm_scale,
                             false, 1.f, 1.f, out, lse, workspace, workspace_bytes, dev_status, stream);
}

jf_status jf_tree_attention_fp8(const void* q, const void* k_cache, const void* v_cache, float k_scale,
                                float v_scale, const int32_t* block_table, int max_pages_per_seq,
                                const int32_t* prefix_lens, const int32_t* tree_offsets, const int32_t* parent,
                                int batch, int total_nodes, int num_q_heads, int num_kv_heads, int head_dim,
                                int page_size, int num_pages, float sm_scale, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream) {
  return tree_attention_call(q, k_cache, v_cache, block_table, max_pages_per_seq, prefix_lens, tree_offsets, parent,
                             batch, total_nodes, num_q_heads, num_kv_heads, head_dim, page_size, num_pages, sm_scale,
                             true, k_scale, v_scale, out, lse, workspace, workspace_bytes, dev_status, stream);
}

size_t jf_build_tree_workspace_size(int batch, int depths, int vocab, int topk) {
  (void)topk;
  if (batch <= 0 || depths <= 0 || vocab <= 0) return 0;
  return jf::build_workspace_bytes(batch, depths, vocab);
}

jf_status jf_build_tree(const float* draft_logits, const int32_t* root_tokens, int batch, int depths, int vocab,
                        int topk, int budget, int max_depth, int32_t* parent, int32_t* token, float* score,
                        int32_t* depth, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                        jf_stream_t stream) {
  using namespace jf;
  if (batch < 0 || depths <= 0 || vocab <= 0 || topk <= 0 || budget <= 0 || max_depth <= 0)
    return JF_ERR_INVALID_ARG;
  if (topk > kMaxTopk || depths > kMaxDepths || budget > kMaxBudget) return JF_ERR_UNSUPPORTED;
  if (topk > vocab || max_depth > depths) return JF_ERR_INVALID_ARG;
  // the full topk-ary tree of depth max_depth must hold `budget` nodes
  long long cap = 1, layer = 1;
  for (int d = 1; d <= max_depth && cap < budget; ++d) {
    layer = layer * topk;
    if (layer > (1ll << 40)) layer = 1ll << 40;
    cap += layer;
  }
  if (cap < budget) return JF_ERR_INVALID_ARG;
  if (batch == 0) return JF_OK;
  if (!draft_logits || !root_tokens || !parent || !token || !score || !workspace) return JF_ERR_INVALID_ARG;
  if (!aligned(draft_logits, 4) || !aligned(workspace, 16)) return JF_ERR_INVALID_ARG;
  if (workspace_bytes < build_workspace_bytes(batch, depths, vocab)) return JF_ERR_INVALID_ARG;
  if (launch_build_tree(draft_logits, root_tokens, batch, depths, vocab, topk, budget, max_depth, parent, token,
                        score, depth, static_cast<RowPartial*>(workspace), dev_status,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JF_ERR_CUDA;
  return JF_OK;
}

size_t jf_expand_frontier_state_size(int batch, int budget, int topk) {
  if (batch <= 0 || budget <= 0 || topk <= 0) return 0;
  return jf::FrontierStateLayout(batch, budget, topk).total;
}

size_t jf_expand_frontier_workspace_size(int batch, int frontier_rows, int vocab) {
  if (batch <= 0 || frontier_rows <= 0 || vocab <= 0) return 0;
  return jf::build_workspace_bytes(batch, frontier_rows, vocab);
}

jf_status jf_expand_frontier(const float* node_logits, const int32_t* root_tokens, int batch, int frontier_rows,
                             int vocab, int topk, int budget, int max_depth, int width, int32_t* parent,
                             int32_t* token, float* score, int32_t* depth, int32_t* num_nodes,
                             int32_t* frontier_begin, void* state, size_t state_bytes, void* workspace,
                             size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream) {
  using namespace jf;
  if (batch < 0 || frontier_rows <= 0 || vocab <= 0 || topk <= 0 || budget <= 0 || max_depth <= 0 || width <= 0)
    return JF_ERR_INVALID_ARG;
  if (topk > kMaxTopk || budget > kMaxFrontierBudget || frontier_rows > kMaxFrontierBudget)
    return JF_ERR_UNSUPPORTED;
  if (topk > vocab) return JF_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * frontier_rows > 65535) return JF_ERR_UNSUPPORTED;
  if (batch == 0) return JF_OK;
  if (!node_logits || !root_tokens || !parent || !token || !score || !depth || !num_nodes || !frontier_begin ||
      !state || !workspace)
    return JF_ERR_INVALID_ARG;
  if (!aligned(node_logits, 4) || !aligned(state, 256) || !aligned(workspace, 16)) return JF_ERR_INVALID_ARG;
  const FrontierStateLayout lay(batch, budget, topk);
  if (state_bytes < lay.total) return JF_ERR_INVALID_ARG;
  if (workspace_bytes < build_workspace_bytes(batch, frontier_rows, vocab)) return JF_ERR_INVALID_ARG;
  uint8_t* sb = static_cast<uint8_t*>(state);
  FrontierState st;
  st.node_key = reinterpret_cast<double*>(sb + lay.key_off);
  st.cand_lp = reinterpret_cast<double*>(sb + lay.lp_off);
  st.cand_tok = reinterpret_cast<int32_t*>(sb + lay.tok_off);
  st.cand_next = reinterpret_cast<int32_t*>(sb + lay.next_off);
  if (launch_expand_frontier(node_logits, root_tokens, batch, frontier_rows, vocab, topk, budget, max_depth, width,
                             parent, token, score, depth, num_nodes, frontier_begin, st,
                             static_cast<RowPartial*>(workspace), dev_status,
                             reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JF_ERR_CUDA;
  return JF_OK;
}

jf_status jf_accept(const int32_t* token, const int32_t* parent, const float* target_logits, int batch,
                    int num_nodes, int vocab, int max_depth, int32_t* accepted_len, int32_t* path,
                    int32_t* bonus_token, int32_t* dev_status, jf_stream_t stream) {
  using namespace jf;
  if (batch < 0 || num_nodes <= 0 || vocab <= 0 || max_depth < 0) return JF_ERR_INVALID_ARG;
  if (num_nodes > kMaxAcceptNodes || max_depth >= kMaxAcceptNodes) return JF_ERR_UNSUPPORTED;
  if (batch == 0) return JF_OK;
  if (!token || !parent || !target_logits || !accepted_len || !path || !bonus_token) return JF_ERR_INVALID_ARG;
  if (!aligned(target_logits, 16)) return JF_ERR_INVALID_ARG;
  if (launch_accept(token, parent, target_logits, batch, num_nodes, vocab, max_depth, accepted_len, path,
                    bonus_token, dev_status, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JF_ERR_CUDA;
  return JF_OK;
}

jf_status jf_commit_kv(void* k_cache, void* v_cache, const int32_t* block_table, int max_pages_per_seq,
                       const int32_t* prefix_lens, const int32_t* tree_offsets, const int32_t* path,
                       const int32_t* accepted_len, int batch, int max_depth, int num_kv_heads, int head_dim,
                       int page_size, int num_pages, int32_t* new_prefix_lens, int32_t* dev_status,
                       jf_stream_t stream) {
  using namespace jf;
  if (batch < 0 || max_depth < 0 || num_kv_heads <= 0 || max_pages_per_seq <= 0 || num_pages <= 0)
    return JF_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || page_size != kPageSize || num_kv_heads > kMaxCommitKvHeads ||
      max_depth >= kMaxAcceptNodes)
    return JF_ERR_UNSUPPORTED;
  if (static_cast<long long>(num_pages) * kPageSize >= (1ll << 31)) return JF_ERR_UNSUPPORTED;
  if (batch == 0) return JF_OK;
  if (!k_cache || !v_cache || !block_table || !prefix_lens || !tree_offsets || !path || !accepted_len ||
      !new_prefix_lens)
    return JF_ERR_INVALID_ARG;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return JF_ERR_INVALID_ARG;
  if (launch_commit_kv(k_cache, v_cache, block_table, max_pages_per_seq, prefix_lens, tree_offsets, path,
                       accepted_len, batch, max_depth, num_kv_heads, num_pages, new_prefix_lens, dev_status,
                       reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JF_ERR_CUDA;
  return JF_OK;
}

jf_status jf_tree_kv_append(const void* k_new, const void* v_new, void* q, void* k_cache, void* v_cache,
                            const int32_t* block_table, int max_pages_per_seq, const int32_t* prefix_lens,
                            const int32_t* tree_offsets, const int32_t* depth, int batch, int total_nodes,
                            int num_q_heads, int num_kv_heads, int head_dim, int page_size, int num_pages,
                            float rope_theta, int32_t* dev_status, jf_stream_t stream) {
  using namespace jf;
  if (batch < 0 || total_nodes < 0 || num_kv_heads <= 0 || max_pages_per_seq <= 0 || num_pages <= 0)
    return JF_ERR_INVALID_ARG;
  if (q != nullptr && num_q_heads <= 0) return JF_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return JF_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || page_size != kPageSize) return JF_ERR_UNSUPPORTED;
  if (batch > kMaxAttnBatch) return JF_ERR_UNSUPPORTED;
  if (static_cast<long long>(num_pages) * kPageSize >= (1ll << 31)) return JF_ERR_UNSUPPORTED;
  if (batch == 0 || total_nodes == 0) return JF_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !prefix_lens || !tree_offsets || !depth)
    return JF_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      (q != nullptr && !aligned(q, 16)))
    return JF_ERR_INVALID_ARG;
  if (launch_tree_kv_append(k_new, v_new, q, k_cache, v_cache, block_table, max_pages_per_seq, prefix_lens,
                            tree_offsets, depth, batch, total_nodes, q != nullptr ? num_q_heads : 0, num_kv_heads,
                            num_pages, static_cast<double>(rope_theta), dev_status,
                            reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JF_ERR_CUDA;
  return JF_OK;
}

}  // extern "C"
