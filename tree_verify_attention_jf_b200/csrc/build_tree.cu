// build_tree.cu -- best-first draft-tree construction under a token budget (sm_100a, SIMT).
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 2, tree construction): per-depth draft log-probabilities, then a
// best-first expansion by cumulative log-probability until the tree holds `budget` nodes.
//
// Kernel 1 (row statistics, HBM-bound): one CTA per (row, 4096-entry chunk) of the [B, depths, V]
// logits reads its chunk once (16-byte loads when the rows allow), and writes the chunk max, the
// float64 sum of exp(x - chunk max) and the chunk's top-8 by (logit desc, id asc).  Only elements at
// or above a per-warp bound (the K-th largest lane maximum) enter the sorted top-K insertion.
// Kernel 2 (expansion, one CTA per sequence): merges the chunk partials into lse and the top-k per
// depth (float64), then selects the budget's nodes.  Best-first popping by (key desc, depth asc,
// parent index asc, rank asc) yields the budget-1 first nodes of that total order, so the kernel
// computes them level-parallel instead of one pop at a time: because every depth-(d-1) node shares
// the same top-k children (per-depth logits), the depth-d candidates are k copies of the sorted
// depth-(d-1) list shifted by lp[d][r]; each candidate's rank among them follows from binary
// searches, the best budget-1 of them are merged into the running global order, and the walk stops
// once no deeper node can enter.  If its node pool would overflow (pathological ties), the CTA falls
// back to popping one node at a time from per-(depth, rank) queues.
#include <cfloat>
#include <mutex>

#include "jf_device.cuh"
#include "jf_internal.h"
#include "jf_math.cuh"
#include "build_common.cuh"

namespace jf {
namespace build {

// ------------------------------------------------------------------------------------------------
// Kernel 1: chunk statistics.  grid = (chunks, batch * max_depth)
// ------------------------------------------------------------------------------------------------
// K: the per-chunk list length, the smallest power of two >= topk (only the best topk of a row can
// ever become children, so shorter lists are exact and much cheaper to maintain).
// With lim_nodes / lim_begin (the frontier expansion), row (b, d) is read only if d is below sequence b's frontier
// size: lim_nodes[b] - lim_begin[b] rows, 1 (the root's) for a tree that has no node yet, none for a tree that
// already holds lim_budget nodes.
template <int K>
__global__ void __launch_bounds__(kThreads, stats_ctas_per_sm(K))
    row_stats_kernel(const float* __restrict__ logits, int depths, int vocab, int max_depth,
                     RowPartial* __restrict__ out, const int32_t* __restrict__ lim_nodes,
                     const int32_t* __restrict__ lim_begin, int lim_budget) {
  __shared__ float s_max[kThreads / 32];
  __shared__ double s_sum[kThreads / 32];
  __shared__ Cand s_top[kThreads / 32][K];
  __shared__ double s_tab[128];
  __shared__ Cand s_cand[kCandCap];  // elements that pass their warp's top-K filter
  __shared__ int s_cnt;
  const int chunk = blockIdx.x, row = blockIdx.y;
  const int b = row / max_depth, d = row - b * max_depth;
  const float* x = logits + (static_cast<long long>(b) * depths + d) * vocab;
  const int lo = chunk * kStatsChunk;
  const int n = min(kStatsChunk, vocab - lo);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double tab_entry = g_exp2_frac128[tid & 127];  // stored once the chunk's loads are issued
  if (tid == 0) s_cnt = 0;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the logits' producer has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (lim_nodes != nullptr) {
    const int nodes = lim_nodes[b];
    const int rows = (nodes == 0) ? 1 : (nodes >= lim_budget ? 0 : nodes - lim_begin[b]);
    if (d >= rows) return;  // uniform over the CTA: a row outside the frontier is never read
  }
  float v[kPerThread];
  if (n == kStatsChunk && (reinterpret_cast<uintptr_t>(x + lo) & 15) == 0) {
    // full, 16-byte aligned chunk: thread t reads float4 number t, t + 256, ...
#pragma unroll
    for (int j = 0; j < kPerThread / 4; ++j) {
      const float4 q = __ldg(reinterpret_cast<const float4*>(x + lo) + j * kThreads + tid);
      v[4 * j + 0] = q.x;
      v[4 * j + 1] = q.y;
      v[4 * j + 2] = q.z;
      v[4 * j + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      const int i = (j / 4) * kThreads * 4 + tid * 4 + (j & 3);
      v[j] = (i < n) ? __ldg(x + lo + i) : -INFINITY;
    }
  }
  if (tid < 128) s_tab[tid] = tab_entry;  // visible after the barrier below
  float m_lane = -INFINITY;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) m_lane = fmaxf(m_lane, v[j]);
  // Top-K filter: the K largest lane maxima are K distinct elements of the warp, so an element below
  // the K-th of them cannot be among the warp's (hence the chunk's) best K, whatever the tie-break.
  float m;  // the warp's max, then the chunk's
  const float tau = warp_kth_bound<K>(m_lane, m);
  if (lane == 0) s_max[warp] = m;
  __syncthreads();
  m = s_max[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, s_max[w]);
  const double md = static_cast<double>(m);
  double sum = 0.0;
  const bool full = n == kStatsChunk;
  if (full) {  // no index checks
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) sum += exp_nonpos_f64(static_cast<double>(v[j]) - md, s_tab);
  } else {
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      const int i = (j / 4) * kThreads * 4 + tid * 4 + (j & 3);
      if (i < n) sum += exp_nonpos_f64(static_cast<double>(v[j]) - md, s_tab);
    }
  }
  // The few elements at or above the filter bound go to one shared list (typically K to 2K per warp);
  // warp 0 selects the chunk's best K from it.  The best K under (logit desc, id asc) is unique, so the
  // order of the list does not matter.
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    const int i = (j / 4) * kThreads * 4 + tid * 4 + (j & 3);
    if (v[j] >= tau && (full || i < n)) {
      const int pos = atomicAdd(&s_cnt, 1);
      if (pos < kCandCap) s_cand[pos] = Cand{v[j], lo + i};
    }
  }
  sum = warp_sum_d(sum);
  if (lane == 0) s_sum[warp] = sum;
  __syncthreads();
  const int cnt = s_cnt;  // uniform over the CTA
  Cand t[K];
#pragma unroll
  for (int i = 0; i < K; ++i) t[i] = Cand{-INFINITY, INT_MAX};
  if (cnt > kCandCap) {
    // list overflow (heavy ties under the bound): every warp merges its own elements, read again from
    // memory, then warp 0 merges the warps' lists
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      const int i = (j / 4) * kThreads * 4 + tid * 4 + (j & 3);
      if (i < n) {
        const float xi = __ldg(x + lo + i);
        if (xi >= tau) insert_k<K>(t, Cand{xi, lo + i});
      }
    }
    warp_merge_k<K>(t, 32);
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < K; ++i) s_top[warp][i] = t[i];
    }
    __syncthreads();
  }
  if (warp == 0) {
    double ssum = (lane < kThreads / 32) ? s_sum[lane] : 0.0;
    ssum = warp_sum_d(ssum);
    if (cnt > kCandCap) {
#pragma unroll
      for (int i = 0; i < K; ++i) t[i] = (lane < kThreads / 32) ? s_top[lane][i] : Cand{-INFINITY, INT_MAX};
      warp_merge_k<K>(t, 8);
    } else {
      for (int c = lane; c < cnt; c += 32) insert_k<K>(t, s_cand[c]);
      warp_merge_k<K>(t, 32);
    }
    if (lane == 0) {
      RowPartial& o = out[static_cast<long long>(row) * gridDim.x + chunk];
      o.sum = ssum;
      o.m = m;
      o.pad = 0;
#pragma unroll
      for (int i = 0; i < kMaxTopk; ++i) {
        o.val[i] = i < K ? t[i < K ? i : 0].v : -INFINITY;
        o.id[i] = i < K ? t[i < K ? i : 0].id : INT_MAX;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Kernel 2: merge + best-first expansion.  grid = batch, block = 256
// ------------------------------------------------------------------------------------------------
struct ExpandSmem {
  double tab[128];                      // 2^(j/128) for exp_nonpos_f64
  double lp[kMaxDepths + 1][kMaxTopk];  // lp[d][r], d = 1..max_depth
  int tok[kMaxDepths + 1][kMaxTopk];
  double key[kMaxBudget];  // sequential fallback: node keys
  int nsd[kMaxBudget];     // sequential fallback: next node of the same depth, in pop order
  int tail[kMaxDepths + 1];
};

// Level-parallel selection state (dynamic shared memory).  Nodes are kept in a pool in creation
// order; lists hold pool ids.  The depth lists are double-buffered: the survivors of depth d (a prefix
// of its list) are the parents of depth d + 1.
constexpr int kPool = 2048;
constexpr int kExpandThreads = 512;
struct SelectSmem {
  double pool_key[kPool];
  int pool_par[kPool];  // parent's pool id, -1 = the root
  int pool_dr[kPool];   // (depth << 8) | rank
  int fidx[kPool];      // final node index of a pool entry
  // All ordering decisions compare order-preserving integer images of the float64 keys: integer
  // compares have a short latency, while a search runs a long chain of dependent compares.
  unsigned long long cord[kMaxTopk][kMaxBudget];  // key of candidate (parent position j, rank r) at [r][j]
  double lkey[2][kMaxBudget];              // candidates of a depth in pop order (best first)
  unsigned long long lord[2][kMaxBudget];  // their integer keys
  int ljr[2][kMaxBudget];                  // (parent position << 4) | rank
  unsigned long long gord[2][kMaxBudget];  // global order so far (integer keys)
  int gpid[2][kMaxBudget];
  int n_kept[3], n_surv[3];  // per depth, d % 3 (reset two depths after their last read)
};

size_t expand_dyn_smem() { return sizeof(SelectSmem); }

// One warp pops the budget's nodes one at a time from per-(depth, rank) queues.  Queue (d, r) lists
// the depth-(d-1) nodes in pop order paired with rank r; it is sorted by the pop order, so the best
// candidate overall is the best queue head (found with redux.sync).
__device__ void expand_sequential(ExpandSmem& s, int lane, int max_depth, int topk, int budget, int32_t* par_o,
                                  int32_t* tok_o, float* sc_o, int32_t* dep_o) {
  if (lane == 0) {
    s.key[0] = 0.0;
    s.nsd[0] = -1;
    for (int i = 0; i <= kMaxDepths; ++i) s.tail[i] = -1;
    s.tail[0] = 0;
  }
  __syncwarp();
  const int nq = max_depth * topk;
  const int nslots = (nq + 31) / 32;
  unsigned long long qord[kSlots];
  unsigned int qtie[kSlots];
  int qnode[kSlots];
#pragma unroll
  for (int sl = 0; sl < kSlots; ++sl) {
    const int q = sl * 32 + lane;
    qord[sl] = 0ull;
    qtie[sl] = 0xffffffffu;
    qnode[sl] = -1;
    if (sl < nslots && q < nq && q < topk) {
      qnode[sl] = 0;
      qord[sl] = ord_key(0.0 + s.lp[1][q]);
      qtie[sl] = (1u << 13) | static_cast<unsigned>(q);
    }
  }
  for (int n = 1; n < budget; ++n) {
    unsigned long long best = 0ull;
    unsigned int btie = 0xffffffffu;
#pragma unroll
    for (int sl = 0; sl < kSlots; ++sl) {
      if (sl < nslots && (qord[sl] > best || (qord[sl] == best && qtie[sl] < btie))) {
        best = qord[sl];
        btie = qtie[sl];
      }
    }
    const unsigned int hi = static_cast<unsigned int>(best >> 32);
    const unsigned int mh = __reduce_max_sync(0xffffffffu, hi);
    const unsigned int lo = (hi == mh) ? static_cast<unsigned int>(best) : 0u;
    const unsigned int ml = __reduce_max_sync(0xffffffffu, lo);
    const unsigned int tt = (hi == mh && static_cast<unsigned int>(best) == ml) ? btie : 0xffffffffu;
    const unsigned int wt = __reduce_min_sync(0xffffffffu, tt);
    if (mh == 0u && ml == 0u) break;
    const int d = static_cast<int>(wt >> 13);
    const int p = static_cast<int>((wt >> 3) & 1023u);
    const int r = static_cast<int>(wt & 7u);
    const double k = key_of_ord((static_cast<unsigned long long>(mh) << 32) | ml);
    const int wq = (d - 1) * topk + r;
    if (lane == 0) {
      par_o[n] = p;
      tok_o[n] = s.tok[d][r];
      sc_o[n] = static_cast<float>(k);
      if (dep_o) dep_o[n] = d;
      s.key[n] = k;
      s.nsd[n] = -1;
      if (s.tail[d] >= 0) s.nsd[s.tail[d]] = n;
      s.tail[d] = n;
    }
    __syncwarp();
#pragma unroll
    for (int sl = 0; sl < kSlots; ++sl) {
      if (sl < nslots && sl * 32 + lane == wq) {
        const int nx = s.nsd[p];
        qnode[sl] = nx;
        if (nx >= 0) {
          qord[sl] = ord_key(s.key[nx] + s.lp[d][r]);
          qtie[sl] = (static_cast<unsigned>(d) << 13) | (static_cast<unsigned>(nx) << 3) | static_cast<unsigned>(r);
        } else {
          qord[sl] = 0ull;
          qtie[sl] = 0xffffffffu;
        }
      }
    }
    if (d < max_depth) {
#pragma unroll
      for (int sl = 0; sl < kSlots; ++sl) {
        const int q = sl * 32 + lane;
        if (sl < nslots && q >= d * topk && q < (d + 1) * topk && qnode[sl] < 0) {
          const int rr = q - d * topk;
          qnode[sl] = n;
          qord[sl] = ord_key(k + s.lp[d + 1][rr]);
          qtie[sl] = (static_cast<unsigned>(d + 1) << 13) | (static_cast<unsigned>(n) << 3) | static_cast<unsigned>(rr);
        }
      }
    }
    __syncwarp();
  }
}

// First position in [0, n) (n <= kMaxBudget) at which pred fails, for a pred that holds on a prefix;
// R searches run interleaved.  Branch-free: pred is always evaluated (on a clamped index) and must not
// short-circuit -- divergent branches in these short searches cost several times the compares.
template <int R, class Pred>
__device__ __forceinline__ void prefix_lengths(int n, int (&cnt)[R], Pred pred) {
#pragma unroll
  for (int i = 0; i < R; ++i) cnt[i] = 0;
  for (int step = n > 0 ? (1 << (31 - __clz(n))) : 0; step > 0; step >>= 1) {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int t = cnt[i] + step;
      const int jj = (t <= n ? t : n) - 1;  // in range; the outcome is discarded when t > n
      const bool take = (t <= n) & pred(i, jj);
      cnt[i] = take ? t : cnt[i];
    }
  }
}

template <int K>
__global__ void __launch_bounds__(kExpandThreads)
    expand_kernel(const RowPartial* __restrict__ part, int nchunks, const int32_t* __restrict__ root_tokens,
                  int max_depth, int topk, int budget, int32_t* __restrict__ parent, int32_t* __restrict__ token,
                  float* __restrict__ score, int32_t* __restrict__ depth_out) {
  __shared__ ExpandSmem s;
  extern __shared__ __align__(16) uint8_t dyn[];
  SelectSmem& q = *reinterpret_cast<SelectSmem*>(dyn);
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 128) s.tab[tid] = g_exp2_frac128[tid];
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the row statistics are complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int root_tok = tid == 0 ? root_tokens[b] : 0;  // in flight while the partials are merged
  __syncthreads();
  // ---- 1. per-depth lse (float64) and top-k: one warp per depth, one lane per chunk partial
  for (int d = 1 + warp; d <= max_depth; d += kExpandThreads / 32) {
    const RowPartial* rp = part + (static_cast<long long>(b) * max_depth + (d - 1)) * nchunks;
    Cand t[K];
    const double lse = warp_merge_row<K>(rp, nchunks, lane, s.tab, t);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < K; ++r) {
        s.lp[d][r] = static_cast<double>(t[r].v) - lse;
        s.tok[d][r] = t[r].id;
      }
    }
  }
  int32_t* par_o = parent + static_cast<long long>(b) * budget;
  int32_t* tok_o = token + static_cast<long long>(b) * budget;
  float* sc_o = score + static_cast<long long>(b) * budget;
  int32_t* dep_o = depth_out ? depth_out + static_cast<long long>(b) * budget : nullptr;
  if (tid == 0) {
    par_o[0] = -1;
    tok_o[0] = root_tok;
    sc_o[0] = 0.f;
    if (dep_o) dep_o[0] = 0;
    q.lkey[0][0] = 0.0;  // "depth 0": the root
    q.n_kept[1] = 0;
    q.n_surv[1] = 0;
  }
  const int T = budget - 1;
  if (T == 0) return;
  __syncthreads();
  // ---- 2. level-parallel selection of the T best nodes in pop order.  Depth d reads the survivors of
  // depth d - 1 (list buffer (d - 1) & 1, a prefix of n_prev entries) and writes buffer d & 1.
  int n_prev = 1, g = 0, cur = 0, pool_base = 0, prev_base = -1;
  bool overflow = false;
  for (int d = 1; d <= max_depth; ++d) {
    if (n_prev == 0) break;
    const int pb = (d - 1) & 1, cb = d & 1;
    const double* prevkey = q.lkey[pb];
    const double* lpd = s.lp[d];
    const bool full = (g == T);
    const unsigned long long thr = full ? q.gord[cur][T - 1] : 0ull;
    if (full && !(ord_key(prevkey[0] + lpd[0]) > thr)) break;  // no depth-d node can enter
    const int ci = d % 3;
    if (tid == 0) {  // counters of depth d + 1, last read at depth d - 2 (before this depth's barriers)
      q.n_kept[(d + 1) % 3] = 0;
      q.n_surv[(d + 1) % 3] = 0;
    }
    // (a) the float64 key of every candidate (j, r) = (parent at position j, rank r), as an integer key
    const int nc = n_prev * topk;
    for (int idx = tid; idx < nc; idx += kExpandThreads) {
      const int j = idx / topk;
      const int r = idx - j * topk;
      q.cord[r][j] = ord_key(prevkey[j] + lpd[r]);
    }
    __syncthreads();
    // (b) rank every candidate among depth d's candidates.  Order: key desc, then parent position,
    // then rank.  Candidates of rank r2 that precede it form a prefix of the parents list (keys are
    // non-increasing along it).
    int kept = 0;
    for (int idx = tid; idx < nc; idx += kExpandThreads) {
      const int j = idx / topk;
      const int r = idx - j * topk;
      const unsigned long long kc = q.cord[r][j];
      if (full && !(kc > thr)) continue;  // cannot beat the current T-th node (ties go to shallower)
      ++kept;
      int cnt[K];
      prefix_lengths<K>(n_prev, cnt, [&](int r2, int jj) {
        const unsigned long long a = q.cord[r2][jj];
        return (a > kc) | ((a == kc) & ((jj < j) | ((jj == j) & (r2 < r))));
      });
      int pos = 0;
#pragma unroll
      for (int r2 = 0; r2 < K; ++r2)
        if (r2 < topk) pos += (r2 == r) ? j : cnt[r2];
      if (pos < T) {
        q.lkey[cb][pos] = prevkey[j] + lpd[r];
        q.lord[cb][pos] = kc;
        q.ljr[cb][pos] = (j << 4) | r;
      }
    }
    kept = __reduce_add_sync(0xffffffffu, kept);
    if (lane == 0 && kept) atomicAdd(&q.n_kept[ci], kept);
    __syncthreads();
    const int n_d = min(q.n_kept[ci], T);
    const unsigned long long* lo = q.lord[cb];
    // (c) merge the global order (g entries) with the depth-d list (n_d entries), keeping T; equal keys:
    // the global (shallower) entry first
    for (int i = tid; i < g; i += kExpandThreads) {
      const unsigned long long gk = q.gord[cur][i];
      int c1[1];
      prefix_lengths<1>(n_d, c1, [&](int, int jj) { return lo[jj] > gk; });
      const int pos = i + c1[0];
      if (pos < T) {
        q.gord[cur ^ 1][pos] = gk;
        q.gpid[cur ^ 1][pos] = q.gpid[cur][i];
      }
    }
    int surv = 0;
    for (int j = tid; j < n_d; j += kExpandThreads) {
      const unsigned long long k = lo[j];
      int c1[1];
      prefix_lengths<1>(g, c1, [&](int, int ii) { return q.gord[cur][ii] >= k; });
      const int pos = j + c1[0];
      if (pos < T) {
        const int pid = pool_base + j;
        surv = j + 1;
        if (pid < kPool) {
          const int jr = q.ljr[cb][j];
          q.pool_key[pid] = q.lkey[cb][j];
          q.pool_par[pid] = (d == 1) ? -1 : prev_base + (jr >> 4);
          q.pool_dr[pid] = (d << 8) | (jr & 15);
        }
        q.gord[cur ^ 1][pos] = k;
        q.gpid[cur ^ 1][pos] = pid;
      }
    }
    surv = __reduce_max_sync(0xffffffffu, surv);
    if (lane == 0 && surv) atomicMax(&q.n_surv[ci], surv);
    __syncthreads();
    const int n_surv = q.n_surv[ci];
    if (pool_base + n_surv > kPool) {
      overflow = true;
      break;
    }
    prev_base = pool_base;
    pool_base += n_surv;
    n_prev = n_surv;
    g = min(g + n_d, T);
    cur ^= 1;
  }
  if (overflow || g < T) {
    __syncthreads();
    if (warp == 0) expand_sequential(s, lane, max_depth, topk, budget, par_o, tok_o, sc_o, dep_o);
    return;
  }
  for (int i = tid; i < T; i += kExpandThreads) q.fidx[q.gpid[cur][i]] = i + 1;
  __syncthreads();
  for (int i = tid; i < T; i += kExpandThreads) {
    const int pid = q.gpid[cur][i];
    const int dr = q.pool_dr[pid];
    const int d = dr >> 8, r = dr & 255;
    const int pp = q.pool_par[pid];
    par_o[i + 1] = pp < 0 ? 0 : q.fidx[pp];
    tok_o[i + 1] = s.tok[d][r];
    sc_o[i + 1] = static_cast<float>(q.pool_key[pid]);
    if (dep_o) dep_o[i + 1] = d;
  }
}

}  // namespace build

size_t build_workspace_bytes(int batch, int depths, int vocab) {
  (void)depths;
  const long long nchunks = (static_cast<long long>(vocab) + kStatsChunk - 1) / kStatsChunk;
  // sized for every depth row (max_depth <= depths)
  return static_cast<size_t>(batch) * depths * nchunks * sizeof(RowPartial);
}

cudaError_t launch_row_stats(const float* logits, int batch, int rows, int row_stride, int vocab, int topk,
                             const int32_t* lim_nodes, const int32_t* lim_begin, int lim_budget,
                             RowPartial* partials, cudaStream_t stream) {
  const int nchunks = (vocab + kStatsChunk - 1) / kStatsChunk;
  const dim3 g1(nchunks, batch * rows), b1(build::kThreads);
  if (topk <= 1)
    return launch_pdl(build::row_stats_kernel<1>, g1, b1, 0, stream, nullptr, logits, row_stride, vocab, rows,
                      partials, lim_nodes, lim_begin, lim_budget);
  if (topk <= 2)
    return launch_pdl(build::row_stats_kernel<2>, g1, b1, 0, stream, nullptr, logits, row_stride, vocab, rows,
                      partials, lim_nodes, lim_begin, lim_budget);
  if (topk <= 4)
    return launch_pdl(build::row_stats_kernel<4>, g1, b1, 0, stream, nullptr, logits, row_stride, vocab, rows,
                      partials, lim_nodes, lim_begin, lim_budget);
  return launch_pdl(build::row_stats_kernel<8>, g1, b1, 0, stream, nullptr, logits, row_stride, vocab, rows,
                    partials, lim_nodes, lim_begin, lim_budget);
}

cudaError_t launch_build_tree(const float* logits, const int32_t* root_tokens, int batch, int depths, int vocab,
                              int topk, int budget, int max_depth, int32_t* parent, int32_t* token, float* score,
                              int32_t* depth, RowPartial* partials, int32_t* status, cudaStream_t stream) {
  (void)status;
  const int nchunks = (vocab + kStatsChunk - 1) / kStatsChunk;
  cudaError_t e = launch_row_stats(logits, batch, max_depth, depths, vocab, topk, nullptr, nullptr, 0, partials,
                                   stream);
  if (e != cudaSuccess) return e;
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  const size_t dyn = build::expand_dyn_smem();
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    const void* fns[4] = {reinterpret_cast<const void*>(build::expand_kernel<1>),
                          reinterpret_cast<const void*>(build::expand_kernel<2>),
                          reinterpret_cast<const void*>(build::expand_kernel<4>),
                          reinterpret_cast<const void*>(build::expand_kernel<8>)};
    for (const void* f : fns) {
      e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn));
      if (e != cudaSuccess) return e;
    }
    attr_set[dev].store(true, std::memory_order_release);
  }
  const dim3 g2(batch), b2(build::kExpandThreads);
  const RowPartial* part = partials;
  if (topk <= 1)
    return launch_pdl(build::expand_kernel<1>, g2, b2, dyn, stream, nullptr, part, nchunks, root_tokens, max_depth,
                      topk, budget, parent, token, score, depth);
  if (topk <= 2)
    return launch_pdl(build::expand_kernel<2>, g2, b2, dyn, stream, nullptr, part, nchunks, root_tokens, max_depth,
                      topk, budget, parent, token, score, depth);
  if (topk <= 4)
    return launch_pdl(build::expand_kernel<4>, g2, b2, dyn, stream, nullptr, part, nchunks, root_tokens, max_depth,
                      topk, budget, parent, token, score, depth);
  return launch_pdl(build::expand_kernel<8>, g2, b2, dyn, stream, nullptr, part, nchunks, root_tokens, max_depth,
                    topk, budget, parent, token, score, depth);
}

}  // namespace jf

// ------------------------------------------------------------------------------------------------
// jf_build_tree_noalloc: the row-statistics scratch of jf_build_tree in a fixed device array, for
// callers that cannot allocate device memory when they call the library.
// ------------------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB, held by every GPU that loads the library
static_assert(sizeof(jf::RowPartial) == 80, "the documented limit of jf_build_tree_noalloc counts 80 B per row partial");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64] = {};  // device address of g_noalloc_scratch, per device

}  // namespace

extern "C" JF_API jf_status jf_build_tree_noalloc(const float* draft_logits, const int32_t* root_tokens, int batch,
                                                  int depths, int vocab, int topk, int budget, int max_depth,
                                                  int32_t* parent, int32_t* token, float* score, int32_t* depth,
                                                  int32_t* dev_status, jf_stream_t stream) {
  if (batch < 0 || depths <= 0 || vocab <= 0) return JF_ERR_INVALID_ARG;
  const unsigned long long chunks = (static_cast<unsigned long long>(vocab) + jf::kStatsChunk - 1) / jf::kStatsChunk;
  const unsigned long long need =
      static_cast<unsigned long long>(batch) * static_cast<unsigned long long>(depths) * chunks * sizeof(jf::RowPartial);
  if (need > kNoAllocScratchBytes) return JF_ERR_UNSUPPORTED;
  if (batch == 0)  // nothing to launch; let the common checks decide the status
    return jf_build_tree(draft_logits, root_tokens, batch, depths, vocab, topk, budget, max_depth, parent, token,
                         score, depth, nullptr, 0, dev_status, stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return JF_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* p = nullptr;
      // In host code the array's name is only a stand-in; its device address comes from the runtime,
      // looked up with this device current.
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return JF_ERR_CUDA;
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return jf_build_tree(draft_logits, root_tokens, batch, depths, vocab, topk, budget, max_depth, parent, token, score,
                       depth, scratch, kNoAllocScratchBytes, dev_status, stream);
}
