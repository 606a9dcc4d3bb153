// build_common.cuh -- device helpers shared by the tree-build kernels (per-depth build and per-node
// frontier expansion): ordered (logit, id) candidate lists and their merges, warp reductions, and the
// order-preserving integer image of a float64 key.
#pragma once

#include <climits>

#include "jf_device.cuh"
#include "jf_internal.h"
#include "jf_math.cuh"

namespace jf {
namespace build {

// 2^(j/128) for the float64 exp (each translation unit keeps its own copy)
static __device__ const double g_exp2_frac128[128] = JF_EXP2_FRAC128;

constexpr int kThreads = 256;
constexpr int kPerThread = kStatsChunk / kThreads;  // 16
constexpr int kCandCap = 512;  // row-statistics candidate list per CTA (4 KB)
// row-statistics CTAs resident per SM: 8 (32 registers a thread) for lists of up to 4, 5 (48) for 8, which
// would spill at 32
constexpr int stats_ctas_per_sm(int K) { return K <= 4 ? 8 : 5; }
constexpr int kSlots = kMaxDepths * kMaxTopk / 32;  // queue slots per lane (16)

struct Cand {
  float v;
  int id;
};

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  return a.v > b.v || (a.v == b.v && a.id < b.id);
}

__device__ __forceinline__ void cswap(Cand& a, Cand& b) {  // after: a better-or-equal than b
  if (better(b, a)) {
    const Cand t = a;
    a = b;
    b = t;
  }
}

// keep t[] sorted best-first; insert x if it beats the last entry
template <int K>
__device__ __forceinline__ void insert_k(Cand (&t)[K], Cand x) {
  if (!better(x, t[K - 1])) return;
  t[K - 1] = x;
#pragma unroll
  for (int i = K - 1; i > 0; --i) cswap(t[i - 1], t[i]);
}

// t := best K of t U u (both sorted best-first), via a bitonic merge (K a power of two)
template <int K>
__device__ __forceinline__ void merge_k(Cand (&t)[K], const Cand (&u)[K]) {
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const Cand o = u[K - 1 - i];
    if (better(o, t[i])) t[i] = o;
  }
  // t is now bitonic; sort it best-first
#pragma unroll
  for (int span = K / 2; span > 0; span >>= 1) {
#pragma unroll
    for (int i = 0; i < K; ++i) {
      if ((i & span) == 0) cswap(t[i], t[i + span]);
    }
  }
}

template <int K>
__device__ __forceinline__ void warp_merge_k(Cand (&t)[K], int width) {
  for (int off = width / 2; off > 0; off >>= 1) {
    Cand u[K];
#pragma unroll
    for (int i = 0; i < K; ++i) {
      u[i].v = __shfl_xor_sync(0xffffffffu, t[i].v, off);
      u[i].id = __shfl_xor_sync(0xffffffffu, t[i].id, off);
    }
    merge_k<K>(t, u);
  }
}

__device__ __forceinline__ void merge8(Cand (&t)[kMaxTopk], const Cand (&u)[kMaxTopk]) { merge_k<kMaxTopk>(t, u); }
__device__ __forceinline__ void warp_merge8(Cand (&t)[kMaxTopk], int width) { warp_merge_k<kMaxTopk>(t, width); }

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ float warp_max_f(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

// A lower bound on the K-th largest of the warp's 32 values: K rounds of "take the warp max, drop every
// lane that holds it".  Ties are dropped together, so the result is the K-th largest distinct value
// (or -inf if there are fewer), which never exceeds the K-th largest counted with multiplicity.  The
// first round's maximum (the warp max) is returned in mx.
template <int K>
__device__ __forceinline__ float warp_kth_bound(float x, float& mx) {
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < K; ++r) {
    m = warp_max_f(x);
    if (r == 0) mx = m;
    if (x == m) x = -INFINITY;
  }
  return m;
}

// Order-preserving map of a (non-NaN) double to an unsigned integer: a < b as doubles iff
// ord_key(a) < ord_key(b).  -0 is taken as +0 so that equal doubles give equal keys.
__device__ __forceinline__ unsigned long long ord_key(double k) {
  if (k == 0.0) k = 0.0;
  const unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(k));
  return (bits >> 63) ? ~bits : (bits | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_of_ord(unsigned long long o) {
  const unsigned long long bits = (o >> 63) ? (o & 0x7fffffffffffffffull) : ~o;
  return __longlong_as_double(static_cast<long long>(bits));
}

// One warp merges the chunk partials of one logits row: returns its natural-log LSE (the max, then the float64
// sum of every chunk's sum scaled by exp(chunk max - max)) and leaves the row's best K by (logit desc, id asc)
// in t on every lane.  tab: the 2^(j/128) table in shared memory.
template <int K>
__device__ __forceinline__ double warp_merge_row(const RowPartial* rp, int nchunks, int lane, const double* tab,
                                                 Cand (&t)[K]) {
  float m = -INFINITY;
  for (int c = lane; c < nchunks; c += 32) m = fmaxf(m, rp[c].m);
  m = warp_max_f(m);
  const double md = static_cast<double>(m);
  double sum = 0.0;
#pragma unroll
  for (int i = 0; i < K; ++i) t[i] = Cand{-INFINITY, INT_MAX};
  for (int c = lane; c < nchunks; c += 32) {
    sum += rp[c].sum * exp_nonpos_f64(static_cast<double>(rp[c].m) - md, tab);
    Cand u[K];
#pragma unroll
    for (int i = 0; i < K; ++i) u[i] = Cand{rp[c].val[i], rp[c].id[i]};
    merge_k<K>(t, u);
  }
  sum = warp_sum_d(sum);
  warp_merge_k<K>(t, 32);
  return md + log(sum);
}

}  // namespace build
}  // namespace jf
