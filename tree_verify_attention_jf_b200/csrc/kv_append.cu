// kv_append.cu -- write the tree tokens' K/V into the paged cache with rotary positions (sm_100a, SIMT).
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 1: the target verifies the whole tree in one forward pass; section 3: inside
// a paged-KV serving engine).  The pages leave the details open; the readings used: node j of sequence b goes to
// cache slot P + j, where tree attention reads it; its position is P + depth_j (root at depth 0); the rotary
// embedding turns each pair (i, i + 64) of the 128-dim head by pos * theta^(-2i/128); V is stored unrotated and the
// query, when given, is rotated in place.
//
// Design: one CTA per tree node.  The 64 angles of the node's position are formed and turned into cosines and
// sines in float64 (positions reach 10^5 and more, where a float32 angle would already be off by more than a bf16
// step), once per node in shared memory; every pair of K and q is then rotated in float64 and rounded once to
// bf16.  V moves as 16-byte words.  The tree offsets are staged in shared memory to find the node's sequence.
#include "jf_device.cuh"
#include "jf_internal.h"

namespace jf {
namespace append {

constexpr int kThreads = 256;
constexpr int kHalf = kHeadDim / 2;

__device__ __forceinline__ void rotate_pair(__nv_bfloat16* x, int i, double c, double s) {
  const double x1 = static_cast<double>(__bfloat162float(x[i]));
  const double x2 = static_cast<double>(__bfloat162float(x[i + kHalf]));
  x[i] = __double2bfloat16(x1 * c - x2 * s);
  x[i + kHalf] = __double2bfloat16(x2 * c + x1 * s);
}

__global__ void __launch_bounds__(kThreads)
    tree_kv_append_kernel(const __nv_bfloat16* __restrict__ k_new, const uint4* __restrict__ v_new,
                          __nv_bfloat16* q, __nv_bfloat16* k_cache, uint4* v_cache,
                          const int32_t* __restrict__ block_table, int max_pages, const int32_t* __restrict__ prefix_lens,
                          const int32_t* __restrict__ tree_offsets, const int32_t* __restrict__ depth, int batch,
                          int total_nodes, int hq, int hkv, int num_pages, double theta, int32_t* status) {
  __shared__ int s_off[kMaxAttnBatch + 1];
  __shared__ double s_cos[kHalf], s_sin[kHalf];
  __shared__ int s_seq;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // k_new / v_new / q come from the kernel before this one
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t = blockIdx.x, tid = threadIdx.x;
  for (int i = tid; i <= batch; i += kThreads) s_off[i] = tree_offsets[i];
  if (tid == 0) s_seq = -1;
  __syncthreads();
  if (tid == 0) {
    if (s_off[0] != 0 || s_off[batch] != total_nodes) {
      report(status, JF_ERR_DEVICE_CHECK);
    } else {
      int lo = 0, hi = batch - 1;  // the last sequence whose first node is at or before t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= t) lo = mid; else hi = mid - 1;
      }
      if (s_off[lo] <= t && t < s_off[lo + 1]) s_seq = lo;
      else report(status, JF_ERR_DEVICE_CHECK);  // tree_offsets not non-decreasing
    }
  }
  __syncthreads();
  const int b = s_seq;
  if (b < 0) return;
  const int P = prefix_lens[b];
  const int j = t - s_off[b];
  const int d = depth[t];
  const long long slot = static_cast<long long>(P) + j;
  if (P < 0 || d < 0 || slot >= static_cast<long long>(max_pages) * kPageSize) {
    if (tid == 0) report(status, JF_ERR_DEVICE_CHECK);
    return;
  }
  const int page = block_table[static_cast<long long>(b) * max_pages + (slot >> 4)];
  if (page < 0 || page >= num_pages) {
    if (tid == 0) report(status, JF_ERR_DEVICE_CHECK);
    return;
  }
  if (tid < kHalf) {
    const double inv = pow(theta, -2.0 * tid / kHeadDim);
    double sn, cs;
    sincos(static_cast<double>(P + d) * inv, &sn, &cs);
    s_cos[tid] = cs;
    s_sin[tid] = sn;
  }
  __syncthreads();
  const long long row = (static_cast<long long>(page) * kPageSize + (slot & 15)) * hkv;  // (page, offset, head 0)
  // K: rotate from k_new into the cache
  for (int x = tid; x < hkv * kHalf; x += kThreads) {
    const int h = x / kHalf, i = x - h * kHalf;
    const __nv_bfloat16* src = k_new + (static_cast<long long>(t) * hkv + h) * kHeadDim;
    __nv_bfloat16* dst = k_cache + (row + h) * kHeadDim;
    const double c = s_cos[i], s = s_sin[i];
    const double x1 = static_cast<double>(__bfloat162float(src[i]));
    const double x2 = static_cast<double>(__bfloat162float(src[i + kHalf]));
    dst[i] = __double2bfloat16(x1 * c - x2 * s);
    dst[i + kHalf] = __double2bfloat16(x2 * c + x1 * s);
  }
  // V: copied as is, 16-byte words
  for (int x = tid; x < hkv * (kHeadDim / 8); x += kThreads)
    v_cache[row * (kHeadDim / 8) + x] = v_new[static_cast<long long>(t) * hkv * (kHeadDim / 8) + x];
  // q: rotated in place
  if (q != nullptr)
    for (int x = tid; x < hq * kHalf; x += kThreads) {
      const int h = x / kHalf, i = x - h * kHalf;
      rotate_pair(q + (static_cast<long long>(t) * hq + h) * kHeadDim, i, s_cos[i], s_sin[i]);
    }
}

}  // namespace append

cudaError_t launch_tree_kv_append(const void* k_new, const void* v_new, void* q, void* k_cache, void* v_cache,
                                  const int32_t* block_table, int max_pages, const int32_t* prefix_lens,
                                  const int32_t* tree_offsets, const int32_t* depth, int batch, int total_nodes,
                                  int hq, int hkv, int num_pages, double theta, int32_t* status, cudaStream_t stream) {
  return launch_pdl(append::tree_kv_append_kernel, dim3(total_nodes), dim3(append::kThreads), 0, stream, nullptr,
                    static_cast<const __nv_bfloat16*>(k_new), static_cast<const uint4*>(v_new),
                    static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k_cache), static_cast<uint4*>(v_cache),
                    block_table, max_pages, prefix_lens, tree_offsets, depth, batch, total_nodes, hq, hkv, num_pages,
                    theta, status);
}

}  // namespace jf
