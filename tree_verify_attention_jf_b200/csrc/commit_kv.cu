// commit_kv.cu -- commit the accepted path's K/V into the paged cache (sm_100a, SIMT copy).
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 1: the longest agreeing prefix of the verified tree is kept; section 3:
// the method runs inside a paged-KV serving engine).  The pages leave the cache update open; the reading used:
// tree node j of sequence b sits at slot P + j during verification, and after acceptance of the path
// [0, n_1, .., n_L] slot P + i (i = 1 .. L) takes the K and V of slot P + n_i while the root's slot P stays, so
// the prefix grows to P + L + 1.
//
// Design: one CTA per sequence.  The copies go in passes of up to 32 KB of rows, each pass reading all of its
// source rows into shared memory before writing any destination.  That ordering is enough: the path strictly
// increases, so a later copy's source P + n_j (n_j > n_i >= i) is never an earlier copy's destination P + i,
// while a source of this pass that is also one of its destinations is read before it is overwritten.  Rows are
// moved as 16-byte words, consecutive threads on consecutive words of a row.
#include "jf_device.cuh"
#include "jf_internal.h"

namespace jf {
namespace commit {

constexpr int kThreads = 256;
constexpr int kStageWords = 2048;  // 16-byte words staged per pass (32 KB)

__global__ void __launch_bounds__(kThreads)
    commit_kv_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, const int32_t* __restrict__ block_table,
                     int max_pages, const int32_t* prefix_lens, const int32_t* __restrict__ tree_offsets,
                     const int32_t* __restrict__ path, const int32_t* __restrict__ accepted_len, int max_depth,
                     int hkv, int num_pages, int32_t* new_prefix_lens, int32_t* status) {
  __shared__ uint4 s_stage[kStageWords];
  __shared__ int s_bad;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the kernel before this one (say, the accept walk) is done
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.x, tid = threadIdx.x;
  // every thread reads P before the barrier below; new_prefix_lens may alias prefix_lens
  const int P = prefix_lens[b];
  const int N = tree_offsets[b + 1] - tree_offsets[b];
  const int L = accepted_len[b];
  const int32_t* pth = path + static_cast<long long>(b) * (max_depth + 1);
  const int32_t* bt = block_table + static_cast<long long>(b) * max_pages;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  if (N > 0) {
    if (tid == 0 && (P < 0 || N < 0 || L < 0 || L > max_depth || L > N - 1 ||
                     static_cast<long long>(P) + N > static_cast<long long>(max_pages) * 16 || pth[0] != 0))
      s_bad = 1;
    const int lc = (L >= 0 && L <= max_depth) ? L : 0;
    for (int i = 1 + tid; i <= lc; i += kThreads)
      if (pth[i] <= pth[i - 1] || pth[i] >= N) s_bad = 1;
    if (P >= 0 && static_cast<long long>(P) + N <= static_cast<long long>(max_pages) * 16)
      for (int pg = P / 16 + tid; pg <= (P + N - 1) / 16; pg += kThreads) {
        const int id = bt[pg];
        if (id < 0 || id >= num_pages) s_bad = 1;
      }
  }
  __syncthreads();
  if (N <= 0 || s_bad) {
    if (tid == 0) {
      if (N != 0) report(status, JF_ERR_DEVICE_CHECK);  // a negative node count: malformed tree_offsets
      new_prefix_lens[b] = P;
    }
    return;
  }
  const int row = hkv * 16;     // 16-byte words of one slot of one cache (hkv x 128 bf16)
  const int per = 2 * row;      // K and V words of one copy
  const int ch = kStageWords / per > 0 ? kStageWords / per : 1;
  for (int i0 = 1; i0 <= L; i0 += ch) {
    const int n = (L + 1 - i0) < ch ? (L + 1 - i0) : ch;
    const int words = n * per;
    for (int x = tid; x < words && x < kStageWords; x += kThreads) {
      const int c = x / per, w = x - c * per;
      const bool is_v = w >= row;
      const int s = P + pth[i0 + c];
      const long long at = (static_cast<long long>(bt[s >> 4]) * 16 + (s & 15)) * row + (is_v ? w - row : w);
      s_stage[x] = is_v ? v_cache[at] : k_cache[at];
    }
    __syncthreads();
    for (int x = tid; x < words && x < kStageWords; x += kThreads) {
      const int c = x / per, w = x - c * per;
      const bool is_v = w >= row;
      const int s = P + i0 + c;
      const long long at = (static_cast<long long>(bt[s >> 4]) * 16 + (s & 15)) * row + (is_v ? w - row : w);
      if (is_v) v_cache[at] = s_stage[x];
      else k_cache[at] = s_stage[x];
    }
    __syncthreads();
  }
  if (tid == 0) new_prefix_lens[b] = P + L + 1;
}

}  // namespace commit

cudaError_t launch_commit_kv(void* k_cache, void* v_cache, const int32_t* block_table, int max_pages,
                             const int32_t* prefix_lens, const int32_t* tree_offsets, const int32_t* path,
                             const int32_t* accepted_len, int batch, int max_depth, int hkv, int num_pages,
                             int32_t* new_prefix_lens, int32_t* status, cudaStream_t stream) {
  return launch_pdl(commit::commit_kv_kernel, dim3(batch), dim3(commit::kThreads), 0, stream, nullptr,
                    static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), block_table, max_pages, prefix_lens,
                    tree_offsets, path, accepted_len, max_depth, hkv, num_pages, new_prefix_lens, status);
}

}  // namespace jf
