// accept.cu -- greedy acceptance walk over the verified draft tree (sm_100a, SIMT + clusters).
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 1 and section 4): starting at the root, repeatedly take the
// target model's argmax at the current node and move to the child carrying that token; the walk's
// length is the number of accepted draft tokens (tau), the last argmax is the bonus token.
//
// Design: the walk is a chain of dependent argmaxes over 151936-entry rows, so latency matters more
// than bandwidth.  Each sequence gets one thread-block cluster (16 CTAs where the GPU allows it,
// else 8); every CTA reduces its slice of the current row with 16-byte loads issued eight deep, the
// partial (value, id) pairs are exchanged through distributed shared memory (st.async into every
// CTA's inbox, completing bytes on the receiver's mbarrier; no cluster-wide barrier per step), and
// every CTA derives the same next node.  The children of every node are listed
// once at the start; while a row is being reduced, the rows of the current node's children (the
// only candidates for the next step) are prefetched into L2 with bulk prefetches, so the next step
// reads from L2.
#include <cooperative_groups.h>

#include "jf_device.cuh"
#include "jf_internal.h"

namespace cg = cooperative_groups;

namespace jf {
namespace acc {

constexpr int kMaxCluster = 16;
constexpr int kThreads = 512;
constexpr int kUnroll = 8;

struct Best {
  float v;
  int id;
};

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
  return v > bv || (v == bv && id < bid);
}

__device__ __forceinline__ void take(float v, int id, float& bv, int& bid) {
  if (better(v, id, bv, bid)) {
    bv = v;
    bid = id;
  }
}

__device__ __forceinline__ void prefetch_l2(const float* p, long long n) {
  // prefetch the 16-byte aligned interior of [p, p + n)
  uintptr_t a = reinterpret_cast<uintptr_t>(p);
  uintptr_t e = reinterpret_cast<uintptr_t>(p + n);
  a = (a + 15) & ~static_cast<uintptr_t>(15);
  e &= ~static_cast<uintptr_t>(15);
  while (a < e) {
    const uintptr_t len = (e - a) > (1u << 20) ? (1u << 20) : (e - a);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(static_cast<uint32_t>(len)) : "memory");
    a += len;
  }
}

// all lanes of the warp wait (bounded) for the phase of `bar` with the given parity
__device__ __forceinline__ bool warp_all_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void warp_best(float& v, int& id) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, id, off);
    take(ov, oi, v, id);
  }
}

constexpr int kWarps = kThreads / 32;

// address of the same shared-memory variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}

// 8-byte store into another CTA's shared memory that completes 8 bytes of transaction on that CTA's
// mbarrier (the receiver learns of the data by waiting on its own barrier)
__device__ __forceinline__ void st_async_best(uint32_t remote, float v, int id, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(remote),
               "r"(__float_as_uint(v)), "r"(id), "r"(remote_bar)
               : "memory");
}

__global__ void __launch_bounds__(kThreads)
    accept_kernel(const int32_t* __restrict__ token, const int32_t* __restrict__ parent,
                  const float* __restrict__ logits, int num_nodes, int vocab, int max_depth,
                  int32_t* __restrict__ accepted_len, int32_t* __restrict__ path, int32_t* __restrict__ bonus,
                  int32_t* __restrict__ status) {
  __shared__ int s_tok[kMaxAcceptNodes];
  __shared__ int s_par[kMaxAcceptNodes];
  __shared__ int s_cur[kMaxAcceptNodes];      // children per node, then the fill cursor
  __shared__ int s_off[kMaxAcceptNodes + 1];  // children of node n: s_kid[s_off[n] .. s_off[n + 1])
  __shared__ int s_kid[kMaxAcceptNodes];
  __shared__ int s_path[kMaxAcceptNodes + 1];
  __shared__ Best s_part[kWarps];               // this step's per-warp partial argmax
  __shared__ __align__(8) Best s_inbox[2][kMaxCluster];  // every CTA's partial argmax, by step parity
  __shared__ __align__(8) uint64_t s_ibar[2];   // completes when all partials of a step have arrived
  __shared__ int2 s_dec[2];                     // (argmax, next node) of the step, by step parity
  __shared__ int s_abort;
  __shared__ int s_wsum[kWarps];
  __shared__ int s_bad;

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* tk = token + static_cast<long long>(b) * num_nodes;
  const int32_t* pr = parent + static_cast<long long>(b) * num_nodes;
  // this CTA's slice of every row (a multiple of 4 entries, so 16-byte loads stay aligned)
  const int per = ((vocab + C - 1) / C + 3) & ~3;
  const int lo = min(vocab, rank * per);
  const int hi = min(vocab, lo + per);
  const float* rows = logits + static_cast<long long>(b) * num_nodes * vocab;
  const bool vec = (vocab % 4) == 0;  // rows then start 16-byte aligned (the base is checked on the host)
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the kernel before this one has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0 && hi > lo) prefetch_l2(rows + lo, hi - lo);  // the root's row, while the tree is read
  // ---- the tree: tokens, parents (validated) and a children list per node
  if (tid == 0) {
    s_bad = 0;
    s_abort = 0;
    mbar_init(&s_ibar[0], 1);
    mbar_init(&s_ibar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < num_nodes; i += kThreads) s_cur[i] = 0;
  __syncthreads();
  for (int i = tid; i < num_nodes; i += kThreads) {
    const int pi = pr[i];
    s_par[i] = pi;
    s_tok[i] = tk[i];
    if (pi < -1 || pi >= i) s_bad = 1;
    else if (pi >= 0) atomicAdd(&s_cur[pi], 1);
  }
  __syncthreads();
  if (s_bad) {  // every CTA of the cluster sees the same data and leaves here together
    if (rank == 0 && tid == 0) report(status, JF_ERR_DEVICE_CHECK);
    return;
  }
  {
    // exclusive prefix sum of the child counts (two entries per thread, num_nodes <= 2 * kThreads)
    const int i0 = 2 * tid, i1 = 2 * tid + 1;
    const int c0 = i0 < num_nodes ? s_cur[i0] : 0;
    const int c1 = i1 < num_nodes ? s_cur[i1] : 0;
    int incl = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += s_wsum[w];
    const int excl = base + incl - (c0 + c1);
    if (i0 < num_nodes) s_off[i0] = excl;
    if (i1 < num_nodes) s_off[i1] = excl + c0;
    if (tid == kThreads - 1) s_off[num_nodes] = base + incl;
    __syncthreads();
    for (int i = tid; i < num_nodes; i += kThreads) s_cur[i] = s_off[i];
    __syncthreads();
    for (int i = tid; i < num_nodes; i += kThreads) {
      const int pi = s_par[i];
      if (pi >= 0) s_kid[atomicAdd(&s_cur[pi], 1)] = i;
    }
    __syncthreads();
  }
  // every CTA's inbox barriers are initialised before the first remote store reaches them
  cluster.sync();
  // ---- the walk.  Per step: a block barrier for the warp partials; the CTA's partial is pushed into
  // every CTA's inbox with st.async (completing bytes on the receiver's mbarrier); one warp waits for
  // its own inbox, decides the next node, and a block barrier hands the decision to the CTA.
  int cur = 0, L = 0, a = 0;
  if (tid == 0) s_path[0] = 0;
  for (int step = 0;; ++step) {
    const float* row = rows + static_cast<long long>(cur) * vocab;
    const int k0 = s_off[cur], nk = s_off[cur + 1] - k0;
    // the children of cur are the only candidates for the next row: prefetch their slices into L2
    if (L < max_depth && tid < nk && hi > lo)
      prefetch_l2(rows + static_cast<long long>(s_kid[k0 + tid]) * vocab + lo, hi - lo);
    // argmax of row cur over [lo, hi): lowest id among equal maxima
    float bv = -INFINITY;
    int bid = INT_MAX;
    if (vec) {
      const float4* row4 = reinterpret_cast<const float4*>(row);
      const int lo4 = lo >> 2, hi4 = hi >> 2;
      for (int base = lo4 + tid; base < hi4; base += kUnroll * kThreads) {
        float4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int idx = base + u * kThreads;
          v[u] = idx < hi4 ? __ldcg(row4 + idx) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int i0 = (base + u * kThreads) * 4;
          take(v[u].x, i0, bv, bid);
          take(v[u].y, i0 + 1, bv, bid);
          take(v[u].z, i0 + 2, bv, bid);
          take(v[u].w, i0 + 3, bv, bid);
        }
      }
    } else {
      for (int base = lo + tid; base < hi; base += kUnroll * kThreads) {
        float v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int idx = base + u * kThreads;
          v[u] = idx < hi ? __ldcg(row + idx) : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) take(v[u], base + u * kThreads, bv, bid);
      }
    }
    warp_best(bv, bid);
    if (lane == 0) s_part[warp] = Best{bv, bid};
    __syncthreads();
    if (warp == 0) {
      const int par = step & 1;
      if (lane == 0) mbar_arrive_expect_tx(&s_ibar[par], static_cast<uint32_t>(C) * sizeof(Best));
      Best m = lane < kWarps ? s_part[lane] : Best{-INFINITY, INT_MAX};
      warp_best(m.v, m.id);  // every lane holds the CTA's partial
      if (lane < C)
        st_async_best(cluster_addr(&s_inbox[par][rank], lane), m.v, m.id, cluster_addr(&s_ibar[par], lane));
      // one warp per CTA waits for the cluster's partials and decides the next node
      if (!warp_all_wait(&s_ibar[par], (step >> 1) & 1, &s_abort)) {
        if (lane == 0) {
          s_abort = 1;
          report(status, JF_ERR_TIMEOUT);
        }
      }
      Best g{-INFINITY, INT_MAX};
      if (lane < C) g = s_inbox[par][lane];
      warp_best(g.v, g.id);
      const int av = (g.id < 0 || g.id >= vocab) ? 0 : g.id;  // out of range only with NaN rows
      // the child of cur carrying token av (the lowest index if several do)
      int mt = INT_MAX;
      if (L < max_depth && !s_abort) {
        for (int k = lane; k < nk; k += 32) {
          const int c = s_kid[k0 + k];
          if (s_tok[c] == av && c < mt) mt = c;
        }
      }
      mt = __reduce_min_sync(0xffffffffu, mt);
      if (lane == 0) s_dec[par] = make_int2(av, mt);
    }
    __syncthreads();
    const int2 dec = s_dec[step & 1];
    a = dec.x;
    const int match = dec.y;
    if (match == INT_MAX) break;
    ++L;
    cur = match;
    if (tid == 0) s_path[L] = cur;
  }
  if (rank == 0) {
    if (tid == 0) {
      accepted_len[b] = L;
      bonus[b] = a;
    }
    __syncthreads();
    int32_t* po = path + static_cast<long long>(b) * (max_depth + 1);
    for (int i = tid; i <= max_depth; i += kThreads) po[i] = (i <= L) ? s_path[i] : -1;
  }
  // no CTA leaves while another may still write into its shared memory
  cluster.sync();
}

}  // namespace acc

cudaError_t launch_accept(const int32_t* token, const int32_t* parent, const float* logits, int batch,
                          int num_nodes, int vocab, int max_depth, int32_t* accepted_len, int32_t* path,
                          int32_t* bonus, int32_t* status, cudaStream_t stream) {
  // cluster size: 16 CTAs when the device can co-schedule them, else the portable 8
  static std::atomic<int> cluster_of[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  int cluster = cluster_of[dev].load(std::memory_order_acquire);
  if (cluster == 0) {
    cluster = 8;
    if (cudaFuncSetAttribute(acc::accept_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t probe = {};
      probe.gridDim = dim3(acc::kMaxCluster);
      probe.blockDim = dim3(acc::kThreads);
      cudaLaunchAttribute at;
      at.id = cudaLaunchAttributeClusterDimension;
      at.val.clusterDim.x = acc::kMaxCluster;
      at.val.clusterDim.y = 1;
      at.val.clusterDim.z = 1;
      probe.attrs = &at;
      probe.numAttrs = 1;
      int nclusters = 0;
      if (cudaOccupancyMaxActiveClusters(&nclusters, acc::accept_kernel, &probe) == cudaSuccess && nclusters > 0)
        cluster = acc::kMaxCluster;
    }
    cudaGetLastError();  // clear a refused attribute / query
    cluster_of[dev].store(cluster, std::memory_order_release);
  }
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cluster;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  return launch_pdl(acc::accept_kernel, dim3(batch * cluster), dim3(acc::kThreads), 0, stream, &attr, token, parent,
                    logits, num_nodes, vocab, max_depth, accepted_len, path, bonus, status);
}

}  // namespace jf
