// frontier.cu -- one round of best-first tree expansion from per-node (path-conditioned) draft logits
// (sm_100a, SIMT).
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 2: the branch factorisation q(pi(v)|x) = prod q(y_u | x, h, pi_<u) and
// best-first tree construction by cumulative draft log-probability up to a budget).  A path-conditioned draft
// head scores a node's children only once that node is in the tree, so the tree grows in rounds: the draft
// head runs on the current frontier, this call turns the frontier's rows into candidate children, and the
// best untaken candidates of every node scored so far join the tree as the next frontier.
//
// Kernel 1 is the per-depth build's row-statistics kernel over the [B, F, V] frontier logits (only the rows
// of each sequence's frontier are read).  Kernel 2 (one CTA per sequence) merges each frontier row's chunk
// partials into its lse and top-k (one warp per row), writes them to the caller's state, gathers every
// untaken candidate (parent u, rank r) of the tree with its float64 key key(u) + lp_u[r], sorts them by
// (key desc, depth asc, parent asc, rank asc) with a bitonic network over order-preserving integer keys, and
// appends the best ones in that order.  A parent's candidates are sorted by rank and their keys do not
// increase with it, so the selected ranks of a parent always continue where the previous round stopped.
#include "build_common.cuh"
#include "jf_device.cuh"
#include "jf_internal.h"

namespace jf {
namespace frontier {

using build::Cand;

constexpr int kThreads = 512;
constexpr int kPool = kMaxFrontierBudget * kMaxTopk;  // candidates of one sequence at most (2048)

struct Smem {  // 45 KB: fits the static shared-memory limit (48 KB)
  double tab[128];
  double key[kMaxFrontierBudget];                // float64 key of every node
  double lp[kMaxFrontierBudget][kMaxTopk];       // candidate log-probabilities (their tokens stay in global memory)
  int depth[kMaxFrontierBudget];
  int next[kMaxFrontierBudget];                  // first untaken rank per node
  unsigned long long ord[kPool];                 // sort keys: order-preserving image of the float64 key
  unsigned int tie[kPool];                       // (depth << 13) | (parent << 3) | rank, ascending
  int scan[kThreads / 32];
  int n0, fb, ok;
};

// a before b in the expansion order: key desc, then (depth, parent, rank) asc
__device__ __forceinline__ bool before(unsigned long long oa, unsigned int ta, unsigned long long ob,
                                       unsigned int tb) {
  return oa > ob || (oa == ob && ta < tb);
}

template <int K>
__global__ void __launch_bounds__(kThreads)
    frontier_expand_kernel(const RowPartial* __restrict__ part, int nchunks, int rows,
                           const int32_t* __restrict__ root_tokens, int topk, int budget, int max_depth, int width,
                           int32_t* __restrict__ parent, int32_t* __restrict__ token, float* __restrict__ score,
                           int32_t* __restrict__ depth, int32_t* __restrict__ num_nodes,
                           int32_t* __restrict__ frontier_begin, FrontierState st, int32_t* status) {
  __shared__ Smem s;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 128) s.tab[tid] = build::g_exp2_frac128[tid];
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the row statistics are complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long nb = static_cast<long long>(b) * budget;
  int32_t* par_o = parent + nb;
  int32_t* tok_o = token + nb;
  float* sc_o = score + nb;
  int32_t* dep_o = depth + nb;
  double* key_g = st.node_key + nb;
  double* lp_g = st.cand_lp + nb * topk;
  int32_t* tok_g = st.cand_tok + nb * topk;
  int32_t* next_g = st.cand_next + nb;
  if (tid == 0) {
    int n0 = num_nodes[b], fb = frontier_begin[b];
    int ok = 1;
    if (n0 == budget) {  // a full tree: nothing to do, its frontier's rows are not read
      ok = 0;
    } else if (n0 == 0) {  // a new tree: its root is the first frontier
      par_o[0] = -1;
      tok_o[0] = root_tokens[b];
      sc_o[0] = 0.f;
      dep_o[0] = 0;
      key_g[0] = 0.0;
      n0 = 1;
      fb = 0;
    } else if (n0 < 0 || n0 > budget || fb < 0 || fb > n0 || n0 - fb > rows) {
      ok = 0;
      report(status, JF_ERR_DEVICE_CHECK);
    }
    s.n0 = n0;
    s.fb = fb;
    s.ok = ok;
  }
  __syncthreads();
  if (!s.ok) return;  // the sequence's tree is left as it was
  const int n0 = s.n0, fb = s.fb;
  // ---- 1. the tree so far: depths, keys, and the candidates of the nodes scored in earlier rounds
  for (int u = tid; u < n0; u += kThreads) {
    s.depth[u] = dep_o[u];
    s.key[u] = key_g[u];
    s.next[u] = u < fb ? next_g[u] : topk;
  }
  for (int i = tid; i < fb * topk; i += kThreads) {
    const int u = i / topk, r = i - u * topk;
    s.lp[u][r] = lp_g[i];
  }
  __syncthreads();
  // ---- 2. score the frontier: one warp per row merges its chunk partials into lse and the top-k
  for (int j = warp; j < n0 - fb; j += kThreads / 32) {
    const int u = fb + j;
    if (s.depth[u] >= max_depth) continue;  // no children below the maximum depth (next stays topk)
    const RowPartial* rp = part + (static_cast<long long>(b) * rows + j) * nchunks;
    Cand t[K];
    const double lse = build::warp_merge_row<K>(rp, nchunks, lane, s.tab, t);
    if (lane < topk) {
      Cand c = t[0];
#pragma unroll
      for (int r = 1; r < K; ++r)
        if (lane == r) c = t[r];
      const double lp = static_cast<double>(c.v) - lse;
      s.lp[u][lane] = lp;
      lp_g[static_cast<long long>(u) * topk + lane] = lp;
      tok_g[static_cast<long long>(u) * topk + lane] = c.id;
    }
    if (lane == 0) s.next[u] = 0;
  }
  __syncthreads();
  // ---- 3. the candidate pool: every untaken rank of every scored node (at most the round's size per node)
  const int want = min(width, budget - n0);
  int mine = 0;
  for (int u = tid; u < n0; u += kThreads) mine += max(0, min(topk - s.next[u], want));
  // block-wide exclusive scan of the per-thread counts (u = tid only, since n0 <= kThreads)
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s.scan[warp] = incl;
  __syncthreads();
  int base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    base += (w < warp) ? s.scan[w] : 0;
    total += s.scan[w];
  }
  base += incl - mine;
  if (tid < n0) {
    const int u = tid;
    const int r0 = s.next[u];
    const int r1 = min(topk, r0 + want);
    for (int r = r0; r < r1; ++r, ++base) {
      s.ord[base] = build::ord_key(s.key[u] + s.lp[u][r]);
      s.tie[base] = (static_cast<unsigned>(s.depth[u] + 1) << 13) | (static_cast<unsigned>(u) << 3) |
                    static_cast<unsigned>(r);
    }
  }
  int n2 = 1;
  while (n2 < total) n2 <<= 1;
  for (int i = total + tid; i < n2; i += kThreads) {  // padding sorts last
    s.ord[i] = 0ull;
    s.tie[i] = 0xffffffffu;
  }
  __syncthreads();
  // ---- 4. bitonic sort of the pool into expansion order
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n2; i += kThreads) {
        const int l = i ^ j;
        if (l > i) {
          const bool up = (i & k) == 0;  // this block ends up in expansion order
          const unsigned long long oi = s.ord[i], ol = s.ord[l];
          const unsigned int ti = s.tie[i], tl = s.tie[l];
          const bool swap = up ? before(ol, tl, oi, ti) : before(oi, ti, ol, tl);
          if (swap) {
            s.ord[i] = ol;
            s.ord[l] = oi;
            s.tie[i] = tl;
            s.tie[l] = ti;
          }
        }
      }
      __syncthreads();
    }
  }
  // ---- 5. append the best candidates as the next frontier
  const int take = min(want, total);
  for (int i = tid; i < take; i += kThreads) {
    const unsigned int t = s.tie[i];
    const int d = static_cast<int>(t >> 13);
    const int u = static_cast<int>((t >> 3) & 1023u);
    const int r = static_cast<int>(t & 7u);
    const double key = s.key[u] + s.lp[u][r];
    const int n = n0 + i;
    par_o[n] = u;
    tok_o[n] = tok_g[u * topk + r];  // written by this block before the barriers above
    sc_o[n] = static_cast<float>(key);
    dep_o[n] = d;
    key_g[n] = key;
    atomicAdd(&s.next[u], 1);
  }
  __syncthreads();
  for (int u = tid; u < n0; u += kThreads) next_g[u] = s.next[u];
  if (tid == 0) {
    num_nodes[b] = n0 + take;
    frontier_begin[b] = n0;
  }
}

}  // namespace frontier

cudaError_t launch_expand_frontier(const float* logits, const int32_t* root_tokens, int batch, int rows, int vocab,
                                   int topk, int budget, int max_depth, int width, int32_t* parent, int32_t* token,
                                   float* score, int32_t* depth, int32_t* num_nodes, int32_t* frontier_begin,
                                   const FrontierState& st, RowPartial* partials, int32_t* status,
                                   cudaStream_t stream) {
  cudaError_t e = launch_row_stats(logits, batch, rows, rows, vocab, topk, num_nodes, frontier_begin, budget,
                                   partials, stream);
  if (e != cudaSuccess) return e;
  const int nchunks = (vocab + kStatsChunk - 1) / kStatsChunk;
  const dim3 g(batch), blk(frontier::kThreads);
#define JF_FRONTIER_LAUNCH(K)                                                                                    \
  return launch_pdl(frontier::frontier_expand_kernel<K>, g, blk, 0, stream, nullptr,                             \
                    static_cast<const RowPartial*>(partials), nchunks, rows, root_tokens, topk, budget, max_depth, \
                    width, parent, token, score, depth, num_nodes, frontier_begin, st, status)
  if (topk <= 1) JF_FRONTIER_LAUNCH(1);
  if (topk <= 2) JF_FRONTIER_LAUNCH(2);
  if (topk <= 4) JF_FRONTIER_LAUNCH(4);
  JF_FRONTIER_LAUNCH(8);
#undef JF_FRONTIER_LAUNCH
}

}  // namespace jf
