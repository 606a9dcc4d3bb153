// tree_attention.cu -- tree-causal attention over a paged bf16 KV cache on sm_100a.
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 2, tree-causal attention mask and branch factorisation): the
// query of every draft-tree node attends to its sequence's whole cached prefix plus the tree slots of
// its own root path (itself included), never to descendants or unrelated branches.
//
// How (B200-specific design, not taken from the pages, which only name an sm_90 paged kernel):
//   * GQA packing: one M tile = 256 rows = (256 / g) tree nodes x g query heads of one kv head.  A work
//     unit is one M tile of one (sequence, kv head).
//   * A CTA pair (a cluster of 2, one CTA per SM) owns an M tile: each CTA holds 128 of its rows in its own
//     tensor memory, and the even CTA issues CTA-pair tcgen05.mma (cta_group::2, M = 256): S = Q K^T with
//     each CTA holding its 128 Q rows and half of the tile's 128 keys, O += P V with P read from each CTA's
//     tensor memory and each CTA holding half of V's 128 head dims.  So every CTA stages 32 KB of K/V per
//     128-key tile for 128 rows of work, and keeps a 3-deep ring of S buffers (S0 | S1 | S2 | O = 512
//     columns): the QK products run up to three tiles ahead of the softmax, which never waits for its own
//     PV and next QK.
//   * Per CTA (12 warps): warp 0 loads Q (double-buffered, once per segment) and gathers this CTA's half of
//     every K tile, warp 2 its half of every V tile -- one TMA box per page and 64-column half, 128-byte
//     swizzled, gathered through the block table, in a 4-deep ring.  The copies are CTA-pair TMA loads: each
//     lands in its own CTA's shared memory and completes its bytes on the even CTA's barrier.  V rows past
//     the sequence end are zeroed (a partial last page lands on a barrier of its own CTA first) before the
//     CTA's arrival on the even CTA's barrier.  Warp 1 allocates the pair's tensor memory and (in the even CTA) issues the
//     MMAs; every commit is multicast to both CTAs' barriers.  Warp 3 validates each segment's metadata.
//     Warps 4-11 are two softmax warpgroups: the thread of warpgroup h for row r owns columns
//     [64 h, 64 h + 64) of that row; the two exchange their row maxima through shared memory once per
//     tile, write P (bf16) over S in tensor memory, and signal the even CTA.  They also build the per-node
//     256-bit ancestor bitsets by pointer jumping at each tree-holding segment start, rescale O lazily
//     (only when the row maximum grows by more than 2^8) and run the epilogue.
//   * The tree mask only touches tiles that hold tree slots; prefix tiles are unmasked.
//   * Work split: the flattened (unit, kv tile) space, in which every unit also carries a fixed cost for
//     the segment start, is cut into equal contiguous ranges, one per CTA pair (stream-K).  A unit cut
//     between pairs writes fp32 partials (O, running max, row sum) and its first pair records the unit in
//     a descriptor slot; combine_kernel, launched right behind on the same stream with a programmatic
//     dependency, merges each recorded unit's partials and stores the bf16 output.  Nothing spins on
//     another CTA pair.
//   * Every wait is bounded (a %globaltimer limit); a role that gives up reports JF_ERR_TIMEOUT, raises
//     its CTA's and the peer CTA's abort flag, and every role then unwinds to the common exit: the copy
//     warps first wait long enough for every copy they issued to land, the MMA warp for its last MMA, and
//     the softmax warps keep meeting their shared barriers with their work skipped, so that the pair's
//     tensor memory is released only when nothing can still write it.
#include "jf_device.cuh"
#include "jf_internal.h"

namespace jf {
namespace attn {

constexpr int kPage = 16;
constexpr int kBM = 128;             // rows per CTA (the pair's M tile is 2 x kBM)
constexpr int kBN = 128;             // keys per KV tile
constexpr int kPagesPerTile = kBN / kPage;
constexpr int kStages = 4;           // K and V ring depth
constexpr int kSBufs = 3;            // S ring depth in tensor memory
constexpr int kThreads = 384;
constexpr int kQHalf = kBM * 128;                 // 128 rows x 64 bf16
constexpr int kQBytes = 2 * kQHalf;               // 32 KB: this CTA's 128 Q rows
constexpr int kKHalf = (kBN / 2) * 128;           // 64 keys x 64 bf16
constexpr int kKBytes = 2 * kKHalf;               // 16 KB: this CTA's 64 keys of a tile, both 64-dim halves
constexpr int kVBytes = kBN * 128;                // 16 KB: 128 keys x this CTA's 64 dims
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmO = 384;                    // O at column 384, S_i at 128 i
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may grow up to 2^8 before O is rescaled
constexpr int kSegCost = 3;  // kv tiles' worth of time that starting a segment in mid-kernel costs
constexpr int kSoftmaxThreads = 2 * kBM;
// P-ready: one arrival per warp of the tile's softmax warpgroup in both CTAs.  The odd CTA's are relaxed cluster-scope arrivals: P sits
// in tensor memory, its stores complete (tcgen05.wait::st) before the arrival, and a release at cluster scope
// would cost each softmax warp a membar per tile.
constexpr uint32_t kPfullCount = 2 * (kSoftmaxThreads / 64);  // the 4 warps of one warpgroup, both CTAs
constexpr uint16_t kPairMask = 0x3;

struct __align__(1024) Smem {
  uint8_t q[2][kQBytes];
  uint8_t k[kStages][kKBytes];
  uint8_t v[kStages][kVBytes];
  uint32_t anc[kMaxTreeNodes][kAncWords];  // ancestor bitsets of the current segment's nodes
  int jmp[kMaxTreeNodes];                   // pointer-jumping links while they are built
  long long cum_work[kMaxAttnBatch + 1];
  int seq_p[kMaxAttnBatch];        // prefix length of every sequence (copied once by the plan)
  int seq_off[kMaxAttnBatch + 1];  // tree_offsets
  long long scan_warp[kThreads / 32];
  float mhand[2][kBM];    // the running maximum decided at a tile, by tile parity, for the next tile's owner
  float lsum[2][2][kBM];  // row sums of the two softmax warpgroups at a segment's end (by segment parity)
  float msum[2][2][kBM];  // the running maximum each warpgroup's row sum is under
  uint64_t qfull[2], qempty[2];
  uint64_t kfull[kStages], kempty[kStages];
  uint64_t vfull[kStages], vempty[kStages];
  // S, P and PV of tile i use entry i % 3: a waiter is never more than one phase behind (tile i - 3 has
  // completed before tile i is waited for), so parity waits are unambiguous
  uint64_t sfull[kSBufs], pfull[kSBufs], pvdone[kSBufs], drain;
  uint64_t vpart;  // this CTA's copy of a partial last page of V
  uint64_t metafull[2], metaempty[2];
  uint32_t tmem_base;
  int meta_valid[2];
  int meta_ctl;
  int abort_flag;
  int bad_meta;
  int k_started;  // the K gather has issued its first tile (the V gather's first tile goes after it)
};

struct Seg {
  int b, kvh, mp, kb, ke;  // kv tiles [kb, ke) of unit (b, kvh, M tile mp)
  int P, N, off, kt;       // prefix length, nodes, first global node, kv tiles of the sequence
  int c0, c1, slot;        // pairs sharing the unit; this pair's partial slot (times 2)
};

__device__ __forceinline__ int pair_of(long long x, long long W, int G) {
  return static_cast<int>(((x + 1) * G - 1) / W);
}

// M tiles of 256 rows of a sequence with N nodes
__device__ __forceinline__ int mtiles_of(int N, int group) { return (N * group + 2 * kBM - 1) / (2 * kBM); }

// Cost space: a unit costs kSegCost + kt, its kv tiles preceded by kSegCost positions that stand for
// the time a pair loses when it starts a segment in mid-kernel (the previous segment's epilogue, the Q
// reload, the refill of the K/V pipeline).  Cutting this space into equal ranges gives a pair that
// crosses a unit boundary correspondingly fewer kv tiles.  A pair whose range ends inside a unit's
// leading positions takes no part in that unit.
struct SegIter {
  long long x, xend, W;
  int G, b, pair;
  __device__ bool next(const Smem& s, const AttnParams& p, Seg& g) {
    while (x < xend) {
      while (s.cum_work[b + 1] <= x) ++b;
      g.b = b;
      g.P = s.seq_p[b];
      g.off = s.seq_off[b];
      g.N = s.seq_off[b + 1] - g.off;
      g.kt = (g.P + g.N + kBN - 1) / kBN;
      const long long span = g.kt + kSegCost;
      const int mpn = mtiles_of(g.N, p.group);
      const long long unit = (x - s.cum_work[b]) / span;
      const long long u0 = s.cum_work[b] + unit * span, u1 = u0 + span;
      const long long e = xend < u1 ? xend : u1;
      const long long t0 = x - u0 - kSegCost, t1 = e - u0 - kSegCost;  // kv tiles [t0, t1) of the unit
      x = e;
      if (t1 <= 0) continue;
      g.kb = t0 < 0 ? 0 : static_cast<int>(t0);
      g.ke = static_cast<int>(t1);
      g.kvh = static_cast<int>(unit / mpn);
      g.mp = static_cast<int>(unit - static_cast<long long>(g.kvh) * mpn);
      g.c0 = pair_of(u0 + kSegCost, W, G);  // owner of the unit's first kv tile
      g.c1 = pair_of(u1 - 1, W, G);         // owner of its last
      g.slot = (pair == g.c0) ? 2 * pair + 1 : 2 * pair;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ int slot_of(int c, int c0) { return (c == c0) ? 2 * c + 1 : 2 * c; }

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait_cluster(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// Raises this CTA's and the peer CTA's abort flags (the peer's roles then stop waiting on this CTA) and
// reports the timeout.
__device__ __forceinline__ void set_abort(Smem& s, const AttnParams& p) {
  *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
  st_cluster_u32(mapa_shared(smem_u32(&s.abort_flag), cluster_ctarank() ^ 1u), 1u);
  report(p.status, JF_ERR_TIMEOUT);
}

// ------------------------------------------------------------------------------------------------
// Plan: per-sequence cost (kv heads x M tiles x (kv tiles + kSegCost)), exclusive prefix sum in shared
// memory, validation of the batch-level metadata.  Every CTA computes the same plan.
// ------------------------------------------------------------------------------------------------
__device__ void build_plan(Smem& s, const AttnParams& p) {
  const int tid = threadIdx.x;
  const int B = p.batch;
  const int per = (B + kThreads - 1) / kThreads;
  const int b0 = tid * per;
  long long local = 0;
  int bad = 0;
  if (tid == 0) s.bad_meta = 0;
  __syncthreads();
  if (tid == 0 && (p.tree_offsets[0] != 0 || p.tree_offsets[B] != p.total_nodes)) bad = 1;
  if (tid == 0) s.seq_off[B] = p.tree_offsets[B];
  for (int b = b0; b < b0 + per && b < B; ++b) {
    const int P = p.prefix_lens[b];
    const int off = p.tree_offsets[b];
    const int N = p.tree_offsets[b + 1] - off;
    s.seq_p[b] = P;
    s.seq_off[b] = off;
    if (P < 0 || N < 0 || N > kMaxTreeNodes) {
      bad = 1;
      continue;
    }
    if (N == 0) continue;
    const long long kt = (static_cast<long long>(P) + N + kBN - 1) / kBN;
    local += static_cast<long long>(p.hkv) * mtiles_of(N, p.group) * (kt + kSegCost);
  }
  if (bad) atomicOr(&s.bad_meta, 1);
  long long incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((tid & 31) >= o) incl += v;
  }
  if ((tid & 31) == 31) s.scan_warp[tid >> 5] = incl;
  __syncthreads();
  long long warp_off = 0;
  for (int w = 0; w < (tid >> 5); ++w) warp_off += s.scan_warp[w];
  long long run = warp_off + incl - local;
  for (int b = b0; b < b0 + per && b < B; ++b) {
    s.cum_work[b] = run;
    const int P = s.seq_p[b];
    const int N = s.seq_off[b + 1] - s.seq_off[b];
    if (P < 0 || N <= 0 || N > kMaxTreeNodes) continue;
    const long long kt = (static_cast<long long>(P) + N + kBN - 1) / kBN;
    run += static_cast<long long>(p.hkv) * mtiles_of(N, p.group) * (kt + kSegCost);
  }
  if (tid == kThreads - 1) s.cum_work[B] = run;
  __syncthreads();
}

// Page id of page j of kv tile t (or -1: past the sequence, past the block table, or out of range), read
// four tiles at a time: lane l reads page l % 8 of tile t0 + l / 8.
__device__ __forceinline__ int batch_page_ids(const AttnParams& p, const int32_t* bt, int npg, int t0, int ke,
                                              int lane) {
  int pid = -1;
  const int t = t0 + (lane >> 3);
  if (t < ke) {
    const int pg = t * kPagesPerTile + (lane & 7);
    if (pg < npg && pg < p.max_pages) {
      const int v = __ldg(bt + pg);
      if (v >= 0 && v < p.num_pages) pid = v;
    }
  }
  return pid;
}

// ------------------------------------------------------------------------------------------------
// Warp 0: Q (double-buffered, one load per segment) and this CTA's 64 keys of every K tile.  Warp 2: this
// CTA's 64 head dims of every V tile.  Every copy is a CTA-pair TMA: it lands in this CTA's shared memory and
// completes its bytes on the even CTA's barrier, which the even CTA's copy warp arms with the bytes of both
// CTAs (one arrival); for V, the odd CTA adds one arrival of its own (vfull counts 2), made after it has
// zeroed its stage's rows past the sequence end.
// ------------------------------------------------------------------------------------------------
// Once a copy warp has given up it waits this long before its CTA may exit, so that every copy it issued
// has landed (copies take microseconds).
constexpr uint64_t kDrainNs = 200000ull;  // 200 us
__device__ __forceinline__ void drain_delay() {
  const uint64_t t0 = globaltimer();
  while (globaltimer() - t0 < kDrainNs) __nanosleep(1000);
}
// Waits up to `ns` for a phase, ignoring the abort flag (used only while unwinding).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > ns) return;
}

__device__ bool kv_producer(Smem& s, const AttnParams& p, SegIter iter, bool is_v, uint32_t rank,
                            const CUtensorMap* tm_q, const CUtensorMap* tm_kv) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  uint64_t* empty = is_v ? s.vempty : s.kempty;
  const uint32_t full0 = mapa_shared(smem_u32(is_v ? s.vfull : s.kfull), 0);  // the even CTA's full barriers
  const uint32_t qfull0 = mapa_shared(smem_u32(s.qfull), 0);
  Seg g;
  uint32_t it = 0, sidx = 0, vpart_uses = 0;
  const int nodes_per_half = kBM / p.group;
  while (iter.next(s, p, g)) {
    const int npg = (g.P + g.N + kPage - 1) / kPage;
    const int32_t* bt = p.block_table + static_cast<long long>(g.b) * p.max_pages;
    int ids_cur = batch_page_ids(p, bt, npg, g.kb, g.ke, lane);
    int ids_next = batch_page_ids(p, bt, npg, g.kb + 4, g.ke, lane);
    if (!is_v) {  // this CTA's 128 Q rows go out while the page ids are on their way
      const int qb = sidx & 1;
      if (!warp_wait(&s.qempty[qb], ((sidx >> 1) & 1) ^ 1, abort)) return false;
      if (rank == 0 && lane == 0) mbar_arrive_expect_tx(&s.qfull[qb], 2 * kQBytes);
      __syncwarp();
      if (lane < 2) {
        const int node0 = g.off + (g.mp * 2 + static_cast<int>(rank)) * nodes_per_half;
        tma_load_3d_pair(s.q[qb] + lane * kQHalf, tm_q, qfull0 + qb * 8, lane * 64, g.kvh * p.group, node0);
      }
    }
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int st = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      const int bi = (t - g.kb) & 3;
      if (bi == 0 && t > g.kb) {
        ids_cur = ids_next;
        ids_next = batch_page_ids(p, bt, npg, t + 4, g.ke, lane);
      }
      const uint32_t bar = full0 + st * 8;
      if (!warp_wait(&empty[st], ph ^ 1, abort)) return false;
      if (is_v && it == 0) {
        // The copy engine serves requests in order and the first S needs Q and K only: the kernel's
        // first V tile is queued behind the first K tile (bounded wait, like every other).
        const uint64_t t0 = globaltimer();
        while (*reinterpret_cast<volatile int*>(&s.k_started) == 0) {
          if (*abort || globaltimer() - t0 > kWaitLimitNs) return false;
        }
      }
      if (!is_v) {
        // lane j < 8 copies page 4 * rank + j / 2 of the tile, 64-dim half j % 2 (this CTA's 64 keys); the even
        // CTA arms the barrier with the bytes of all the tile's pages (both CTAs).  Keys past the sequence
        // are not copied: their S columns are masked before the softmax.
        const int pid_all = __shfl_sync(0xffffffffu, ids_cur, bi * 8 + (lane & 7));
        const uint32_t all = __ballot_sync(0xffffffffu, lane < 8 && pid_all >= 0);
        int pid = __shfl_sync(0xffffffffu, ids_cur, bi * 8 + 4 * static_cast<int>(rank) + ((lane >> 1) & 3));
        if (rank == 0 && lane == 0) mbar_arrive_expect_tx(&s.kfull[st], static_cast<uint32_t>(__popc(all)) * 4096u);
        if (lane < 8 && pid >= 0) {
          const int half = lane & 1;
          tma_load_3d_pair(s.k[st] + half * kKHalf + (lane >> 1) * (kPage * 128), tm_kv, bar, half * 64, g.kvh,
                           pid * kPage);
        }
        if (it == 0) {
          __syncwarp();
          if (lane == 0) *reinterpret_cast<volatile int*>(&s.k_started) = 1;
        }
      } else {
        // V rows of the tile past the sequence end are zeroed so that stale cache contents (even NaN) cannot
        // reach the output through 0 * V.  Full pages are CTA-pair copies; the sequence's last page, if
        // partial, is copied to this CTA alone (a barrier of its own), and the warp waits for it, zeroes the
        // rows past the end and only then arrives on the even CTA's barrier.
        const int nkeys = g.P + g.N - t * kBN;
        const int zf = nkeys < 0 ? 0 : (nkeys > kBN ? kBN : nkeys);
        const int full_pages = zf / kPage, part = zf % kPage;
        const int pid = __shfl_sync(0xffffffffu, ids_cur, bi * 8 + (lane & 7));
        const bool full_ok = lane < full_pages && pid >= 0;  // full_pages <= 8
        const int pid_part = __shfl_sync(0xffffffffu, ids_cur, bi * 8 + (full_pages & 7));
        const bool part_ok = part > 0 && pid_part >= 0;
        const uint32_t nfull = static_cast<uint32_t>(__popc(__ballot_sync(0xffffffffu, full_ok)));
        if (full_ok)
          tma_load_3d_pair(s.v[st] + lane * (kPage * 128), tm_kv, bar, static_cast<int>(rank) * 64, g.kvh,
                           pid * kPage);
        if (part_ok) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&s.vpart, kPage * 128);
            tma_load_3d(s.v[st] + full_pages * (kPage * 128), tm_kv, &s.vpart, static_cast<int>(rank) * 64,
                        g.kvh, pid_part * kPage);
          }
          if (!warp_wait(&s.vpart, vpart_uses & 1, abort)) return false;
          ++vpart_uses;
        }
        if (zf < kBN) {
          uint8_t* vb = s.v[st];
          for (int i = lane; i < (kBN - zf) * 8; i += 32)
            *reinterpret_cast<uint4*>(vb + (zf + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive_expect_tx(&s.vfull[st], 2 * nfull * (kPage * 128u));  // both CTAs' pages
          else if (zf < kBN) mbar_arrive_cluster(bar);  // publishes the zeroed rows (release)
          else mbar_arrive_cluster_relaxed(bar);        // the copies complete on the barrier themselves
        }
      }
    }
    ++sidx;
  }
  return true;
}

// ------------------------------------------------------------------------------------------------
// Warp 1 of the even CTA: CTA-pair tcgen05.mma issuer.  QK of tile i goes into S buffer i % 3 and is issued
// right after PV of tile i - 3 (which read P from that buffer); every commit is multicast to both CTAs.  Its
// waits acquire at CTA scope (a cluster-scope acquire costs hundreds of cycles per wait on this critical
// warp): the odd CTA's P-ready arrivals are relaxed (P is in tensor memory, its stores complete before the
// arrival) and the copies' bytes complete on the barriers themselves.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void issue_qk(const Smem& s, uint32_t tmem, int qb, int st, int sb) {
  constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, kBN, false, false);
  const uint32_t qaddr = smem_u32(s.q[qb]);
  const uint32_t kaddr = smem_u32(s.k[st]);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    mma2_ss(tmem + sb * 128, smem_desc_sw128(qaddr + (kk >> 2) * kQHalf + (kk & 3) * 32, 16, 1024),
            smem_desc_sw128(kaddr + (kk >> 2) * kKHalf + (kk & 3) * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

__device__ __forceinline__ void issue_pv(const Smem& s, uint32_t tmem, int sb, int st, bool first) {
  constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, 128, false, true);
  const uint32_t vaddr = smem_u32(s.v[st]);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    mma2_ts(tmem + kTmO, tmem + sb * 128 + kk * 8, smem_desc_sw128(vaddr + kk * 2048, kVBytes, 1024), idesc,
            (first && kk == 0) ? 0u : 1u);
  }
}

// Only lane 0 runs the issue loop (the other lanes wait at the warp's exit).  Per tile it waits for everything
// the tile's burst needs -- P and V of tile i, K (and at a segment start Q) of tile i + 3 -- and then issues PV(i)
// and QK(i + 3) back to back, so that the tensor pipe is fed 16 MMAs at a time.
__device__ bool mma_issuer(Smem& s, const AttnParams& p, SegIter pv_iter, uint32_t tmem, bool& issued) {
  volatile int* abort = &s.abort_flag;
  issued = false;
  // the QK side runs kSBufs tiles ahead of the PV side on its own copy of the segment iterator
  SegIter qk_iter = pv_iter;
  Seg gq, gp;
  bool qk_live = qk_iter.next(s, p, gq);
  int qk_t = qk_live ? gq.kb : 0;
  uint32_t it_qk = 0, qk_sidx = 0;
  // Waits for the next QK's operands; false on a timeout/abort.  *have = false when no QK is left.
  auto wait_next_qk = [&](bool* have) -> bool {
    *have = false;
    if (!qk_live) return true;
    if (qk_t == gq.ke) {
      ++qk_sidx;
      qk_live = qk_iter.next(s, p, gq);
      if (!qk_live) return true;
      qk_t = gq.kb;
    }
    if (qk_t == gq.kb && !mbar_wait(&s.qfull[qk_sidx & 1], (qk_sidx >> 1) & 1, abort)) return false;
    if (!mbar_wait(&s.kfull[it_qk % kStages], (it_qk / kStages) & 1, abort)) return false;
    *have = true;
    return true;
  };
  auto issue_qk_now = [&]() {
    const int qb = qk_sidx & 1, st = it_qk % kStages;
    issue_qk(s, tmem, qb, st, it_qk % kSBufs);
    mma2_commit_mc(&s.sfull[it_qk % kSBufs], kPairMask);
    mma2_commit_mc(&s.kempty[st], kPairMask);
    if (qk_t == gq.ke - 1) mma2_commit_mc(&s.qempty[qb], kPairMask);
    ++qk_t;
    ++it_qk;
    issued = true;
  };
  for (int i = 0; i < kSBufs; ++i) {
    bool have;
    if (!wait_next_qk(&have)) return false;
    if (!have) break;
    tc_fence_after();
    issue_qk_now();
  }
  uint32_t it = 0;
  while (pv_iter.next(s, p, gp)) {
    for (int t = gp.kb; t < gp.ke; ++t, ++it) {
      const int sb = it % kSBufs, st = it % kStages;
      if (!mbar_wait(&s.pfull[sb], (it / kSBufs) & 1, abort)) return false;
      // Cluster scope only for the tile whose V rows past the sequence end the odd CTA zeroed (its arrival is a
      // release); every other arrival is relaxed or local, and the copies' bytes complete on the barrier.
      const bool zeroed = static_cast<long long>(t + 1) * kBN > static_cast<long long>(gp.P) + gp.N;
      if (!(zeroed ? mbar_wait_cluster(&s.vfull[st], (it / kStages) & 1, abort)
                   : mbar_wait(&s.vfull[st], (it / kStages) & 1, abort)))
        return false;
      bool have;
      if (!wait_next_qk(&have)) return false;
      tc_fence_after();
      issue_pv(s, tmem, sb, st, t == gp.kb);
      mma2_commit_mc(&s.vempty[st], kPairMask);
      mma2_commit_mc(&s.pvdone[sb], kPairMask);
      issued = true;
      if (have) issue_qk_now();
    }
  }
  return true;
}

// ------------------------------------------------------------------------------------------------
// Warp 3: per-segment validation (in both CTAs; each CTA's epilogue reads its own verdict)
// ------------------------------------------------------------------------------------------------
__device__ bool metadata(Smem& s, const AttnParams& p, SegIter iter) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  Seg g;
  uint32_t sidx = 0;
  while (iter.next(s, p, g)) {
    const int buf = sidx & 1;
    if (!warp_wait(&s.metaempty[buf], ((sidx >> 1) & 1) ^ 1, abort)) return false;
    // --- validation: parent indices, capacity, the page ids this segment reads.  Every global load of
    // the segment is issued before any is used, so the whole check costs one memory round trip.
    const int npg = (g.P + g.N + kPage - 1) / kPage;
    const int32_t* par = p.parent + g.off;
    const int32_t* bt = p.block_table + static_cast<long long>(g.b) * p.max_pages;
    int pr[kMaxTreeNodes / 32];
#pragma unroll
    for (int k = 0; k < kMaxTreeNodes / 32; ++k) {
      const int i = lane + 32 * k;
      pr[k] = i < g.N ? __ldg(par + i) : -1;
    }
    int pg1 = g.ke * kPagesPerTile;
    if (pg1 > npg) pg1 = npg;
    if (pg1 > p.max_pages) pg1 = p.max_pages;
    int bad = (static_cast<long long>(g.P) + g.N > static_cast<long long>(p.max_pages) * kPage) ? 1 : 0;
    for (int pg = g.kb * kPagesPerTile + lane; pg < pg1; pg += 4 * 32) {
      int v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = (pg + 32 * u < pg1) ? __ldg(bt + pg + 32 * u) : 0;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v[u] < 0 || v[u] >= p.num_pages) bad = 1;
    }
#pragma unroll
    for (int k = 0; k < kMaxTreeNodes / 32; ++k) {
      const int i = lane + 32 * k;
      if (i < g.N && (pr[k] < -1 || pr[k] >= i)) bad = 1;
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      s.meta_valid[buf] = bad ? 0 : 1;
      if (bad) report(p.status, JF_ERR_DEVICE_CHECK);
    }
    __syncwarp();
    __threadfence_block();
    mbar_arrive(&s.metafull[buf]);
    ++sidx;
  }
  return true;
}

// ------------------------------------------------------------------------------------------------
// Warps 4-11: online softmax (thread of warpgroup h for row r: columns [64 h, 64 h + 64)) and the epilogue
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void store_half_row_bf16(__nv_bfloat16* dst, const uint32_t (&o)[32], float inv_l) {
#pragma unroll
  for (int c = 0; c < 32; c += 8) {
    uint4 v;
    v.x = pack_bf16x2(__uint_as_float(o[c + 0]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
    v.y = pack_bf16x2(__uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
    v.z = pack_bf16x2(__uint_as_float(o[c + 4]) * inv_l, __uint_as_float(o[c + 5]) * inv_l);
    v.w = pack_bf16x2(__uint_as_float(o[c + 6]) * inv_l, __uint_as_float(o[c + 7]) * inv_l);
    *reinterpret_cast<uint4*>(dst + c) = v;
  }
}

// visibility bits of one 32-key word of a tile that holds tree slots: bit i <=> key slot slot0 + i is
// visible to the row (prefix slots always; tree slot P + j iff j is on the row's root path)
__device__ __forceinline__ uint32_t vis_word(int slot0, int P, int N, bool row_valid, const uint32_t* anc) {
  const int np = P - slot0;  // leading prefix slots in this word
  if (np >= 32) return 0xffffffffu;
  uint32_t bits = np > 0 ? (1u << np) - 1u : 0u;
  const int j0 = slot0 - P;  // tree node of bit 0 (may be negative)
  if (row_valid) {
    uint32_t lo = 0, hi = 0;
    const int wi = j0 >> 5;  // floor division
    const int sh = j0 & 31;
    if (wi >= 0 && wi < kAncWords) lo = anc[wi];
    if (wi + 1 >= 0 && wi + 1 < kAncWords) hi = anc[wi + 1];
    uint32_t tb = sh ? ((lo >> sh) | (hi << (32 - sh))) : lo;
    if (np > 0) tb &= ~((1u << np) - 1u);
    const int lim = N - j0;  // bits [0, lim) can be tree nodes
    if (lim <= 0) tb = 0;
    else if (lim < 32) tb &= (1u << lim) - 1u;
    bits |= tb;
  } else {
    // rows past the last node see every existing slot (their output is dropped)
    const int lim = P + N - slot0;
    if (lim >= 32) bits = 0xffffffffu;
    else if (lim > 0) bits = (1u << lim) - 1u;
  }
  return bits;
}

// Partial outputs are stored column-quad-major so that a warp's 32 rows touch 512 contiguous bytes:
// float4 index ((slot * 32 + c4) * 128 + row), slot = 2 * (segment slot) + CTA rank.
__device__ __forceinline__ float4* part_ptr(const AttnParams& p, int slot, int c4, int r) {
  return reinterpret_cast<float4*>(p.part_o) + (static_cast<long long>(slot) * 32 + c4) * kBM + r;
}

// Named barrier 1 joins the 256 softmax threads (warps 4-11).
__device__ __forceinline__ void softmax_bar() { named_bar_sync(1, kSoftmaxThreads); }
__device__ __forceinline__ bool softmax_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(kSoftmaxThreads)
      : "memory");
  return r != 0;
}

// Ancestor bitsets (node itself included) of the segment's sequence, one softmax thread per node, by
// pointer jumping: anc[i] covers the path from i up to (not including) jmp[i]; each round merges the
// set at jmp[i] and jumps there, so a tree of depth D needs ceil(log2 D) + 1 rounds.  Parents outside
// [-1, i) are treated as -1 (the metadata warp flags such a sequence, whose output is not stored).
__device__ bool build_ancestors(Smem& s, const AttnParams& p, const Seg& g) {
  const int i = static_cast<int>(threadIdx.x) - 128;  // 0 .. 255
  softmax_bar();  // every read of the previous segment's bitsets is done
  int pj = -1;
  if (i < g.N) {
    const int pi = __ldg(p.parent + g.off + i);
    pj = (pi >= 0 && pi < i) ? pi : -1;
#pragma unroll
    for (int w = 0; w < kAncWords; ++w) s.anc[i][w] = (w == (i >> 5)) ? (1u << (i & 31)) : 0u;
    s.jmp[i] = pj;
  }
  for (int round = 0; softmax_bar_or(pj >= 0); ++round) {
    if (round > kMaxTreeNodes) return false;  // unreachable for valid input; keeps the loop bounded
    uint32_t add[kAncWords];
    int nj = -1;
    if (pj >= 0) {
#pragma unroll
      for (int w = 0; w < kAncWords; ++w) add[w] = s.anc[pj][w];
      nj = s.jmp[pj];
    }
    softmax_bar();  // all reads of this round before any write
    if (pj >= 0) {
#pragma unroll
      for (int w = 0; w < kAncWords; ++w) s.anc[i][w] |= add[w];
      s.jmp[i] = nj;
      pj = nj;
    }
  }
  return true;
}

// S columns [c0, c0 + 64) of the row into sr, with the tree mask applied (invisible keys -> -inf); returns
// their maximum (raw scores).
__device__ __forceinline__ float load_masked_half(uint32_t taddr, uint32_t (&sr)[64], bool tree_tile, int slot0,
                                                  const Seg& g, bool row_valid, const uint32_t* anc) {
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
  uint32_t vis[2];
#pragma unroll
  for (int w = 0; w < 2; ++w)
    vis[w] = tree_tile ? vis_word(slot0 + 32 * w, g.P, g.N, row_valid, anc) : 0xffffffffu;
  tmem_ld_wait();
  if (tree_tile) {
    // invisible keys become -inf: they drop out of the max and get P = 2^-inf = 0
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (!((vis[c >> 5] >> (c & 31)) & 1u)) sr[c] = 0xff800000u;
  }
  float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 8) {
    a0 = fmax3(a0, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
    a1 = fmax3(a1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
    a2 = fmax3(a2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
    a3 = fmax3(a3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
  }
  return fmax3(a0, a1, fmaxf(a2, a3));
}

// P = 2^(s * scale - m) of 64 keys into their 32 bf16-pair columns at taddr_p; returns their sum.
__device__ __forceinline__ float exp_store_half(uint32_t taddr_p, const uint32_t (&sr)[64], uint64_t sl2x2,
                                                uint64_t nm2) {
  uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const int cc = 32 * q + c;
      const uint64_t y = f2_fma(f2_pack(__uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1])), sl2x2, nm2);
      float y0, y1;
      f2_unpack(y, y0, y1);
      const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
      if ((c >> 1) & 1) acc1 = f2_add(acc1, f2_pack(p0, p1));
      else acc0 = f2_add(acc0, f2_pack(p0, p1));
      pk[c >> 1] = pack_bf16x2_alu(p0, p1);
    }
    tmem_st16(taddr_p + 16 * q, pk);
  }
  float u0, u1, v0, v1;
  f2_unpack(acc0, u0, u1);
  f2_unpack(acc1, v0, v1);
  return (u0 + u1) + (v0 + v1);
}

// The two softmax warpgroups take the kv tiles in turn (tile i of this CTA's sequence: warpgroup i % 2), each
// thread owning one row, so that one warpgroup's exponentials overlap the other's loads and maximum.  The
// online softmax's running maximum is decided tile by tile in order: the thread of tile i takes tile i - 1's
// decision from shared memory (named barrier 2 + (i - 1) % 2: its owner arrives, this thread syncs), raises
// it lazily (only by more than 2^8) with tile i's maximum, publishes it for tile i + 1, rescales O (after
// PV of tile i - 1) when it was raised, and writes P relative to it.  Each thread keeps its own row sum
// relative to the last maximum it saw; the two are merged at the segment's end.
//
// A warp whose wait gives up keeps running the loop structure with its work skipped (ok = false), so that the
// named barriers the softmax threads share are always reached by all of them.
__device__ bool softmax_epilogue(Smem& s, const AttnParams& p, SegIter iter, uint32_t tmem, uint32_t rank) {
  const int h = (static_cast<int>(threadIdx.x) - 128) >> 7;  // warpgroup
  const int r = threadIdx.x & 127;                             // row of this CTA's 128 == TMEM lane
  const int wq = (threadIdx.x >> 5) & 3;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  volatile int* abort = &s.abort_flag;
  const uint32_t pfull0 = mapa_shared(smem_u32(s.pfull), 0);  // the even CTA's P-ready barriers
  const float sl2 = p.scale_log2;
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const int nodes_per_half = kBM / p.group;
  // the CTA's last tile publishes no decision (no tile follows it)
  uint32_t total = 0;
  {
    SegIter cnt = iter;
    Seg gc;
    while (cnt.next(s, p, gc)) total += static_cast<uint32_t>(gc.ke - gc.kb);
  }
  bool ok = true;
  Seg g;
  uint32_t it = 0, sidx = 0;
  while (iter.next(s, p, g)) {
    const int buf = sidx & 1;
    const int node = (g.mp * 2 + static_cast<int>(rank)) * nodes_per_half + r / p.group;
    const int head = g.kvh * p.group + (r % p.group);
    const bool row_valid = node < g.N;
    if (static_cast<long long>(g.ke) * kBN > g.P && !build_ancestors(s, p, g)) ok = false;
    const uint32_t* anc = &s.anc[row_valid ? node : 0][0];
    float m_cur = -INFINITY, l = 0.f;  // this thread's view of the running maximum, its row sum under it
    bool did_last = false;
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      if (static_cast<int>(it & 1) != h) continue;  // the other warpgroup's tile
      const bool tree_tile = (t + 1) * kBN > g.P;
      const int sb = it % kSBufs;
      const uint32_t s_addr = lane_base + sb * 128;
      if (ok && !warp_wait(&s.sfull[sb], (it / kSBufs) & 1, abort)) ok = false;
      // pass 1: the tile's row maximum (raw scores)
      float mraw = -INFINITY;
      if (ok) {
        tc_fence_after();
        uint32_t sr[64];
        mraw = load_masked_half(s_addr, sr, tree_tile, t * kBN, g, row_valid, anc);
        mraw = fmaxf(mraw, load_masked_half(s_addr + 64, sr, tree_tile, t * kBN + 64, g, row_valid, anc));
      }
      const float mx = (mraw == -INFINITY) ? -INFINITY : mraw * sl2;
      // the running maximum after the previous tile (its owner is the other warpgroup)
      float m_prev = -INFINITY;
      if (it > 0) {
        named_bar_sync(2 + ((it - 1) & 1), kSoftmaxThreads);
        if (t > g.kb) m_prev = s.mhand[(it - 1) & 1][r];
      }
      const float m_new = (m_prev == -INFINITY || mx > m_prev + kRescaleThreshold) ? mx : m_prev;
      if (it + 1 < total) {
        s.mhand[it & 1][r] = m_new;
        named_bar_arrive(2 + (it & 1), kSoftmaxThreads);
      }
      if (!ok) continue;
      if (m_cur != m_new) {  // the other warpgroup (or this tile) raised the maximum: rescale this thread's sum
        if (m_cur != -INFINITY) l *= ex2_approx(m_cur - m_new);
        m_cur = m_new;
      }
      const bool resc = m_prev != -INFINITY && m_new != m_prev;
      if (__any_sync(0xffffffffu, resc)) {
        // O holds PV of the segment's tiles so far, under m_prev; the last of them (tile it - 1) may still run
        if (!warp_wait(&s.pvdone[(it - 1) % kSBufs], ((it - 1) / kSBufs) & 1, abort)) {
          ok = false;
          continue;
        }
        tc_fence_after();
        const float a = resc ? ex2_approx(m_prev - m_new) : 1.f;
#pragma unroll
        for (int cc = 0; cc < 128; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kTmO + cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
          tmem_st32(lane_base + kTmO + cc, o);
        }
      }
      // pass 2: P over the keys of each half; keys [64 k, 64 k + 64) go to columns [32 k, 32 k + 32), over S
      // columns this pass has already read
      const float negm = (m_new == -INFINITY) ? 0.f : -m_new;
      const uint64_t nm2 = f2_pack(negm, negm);
      {
        uint32_t sr[64];
        load_masked_half(s_addr, sr, tree_tile, t * kBN, g, row_valid, anc);
        l += exp_store_half(s_addr, sr, sl2x2, nm2);
        load_masked_half(s_addr + 64, sr, tree_tile, t * kBN + 64, g, row_valid, anc);
        l += exp_store_half(s_addr + 32, sr, sl2x2, nm2);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) {
        if (rank == 0) mbar_arrive(&s.pfull[sb]);
        else mbar_arrive_cluster_relaxed(pfull0 + sb * 8);
      }
      did_last = (t == g.ke - 1);
    }
    // ---------------- epilogue of the segment
    bool seg_ok = false;
    if (ok && !warp_wait(&s.metafull[buf], (sidx >> 1) & 1, abort)) ok = false;
    if (ok) seg_ok = s.meta_valid[buf] != 0;
    // The warpgroup of the segment's last tile waits for its PV (every earlier MMA is complete then too); the
    // barrier below tells the other warpgroup.
    if (ok && did_last && !warp_wait(&s.pvdone[(it - 1) % kSBufs], ((it - 1) / kSBufs) & 1, abort)) ok = false;
    s.lsum[buf][h][r] = l;
    s.msum[buf][h][r] = m_cur;
    softmax_bar();
    float l_tot = 0.f, m_fin = -INFINITY;
    {
      const float m0 = s.msum[buf][0][r], m1 = s.msum[buf][1][r];
      m_fin = fmaxf(m0, m1);
      if (m0 != -INFINITY) l_tot += s.lsum[buf][0][r] * ex2_approx(m0 - m_fin);
      if (m1 != -INFINITY) l_tot += s.lsum[buf][1][r] * ex2_approx(m1 - m_fin);
    }
    if (ok) {
      tc_fence_after();
      mbar_arrive(&s.metaempty[buf]);
      const bool split = g.c0 != g.c1;
      const long long grow = static_cast<long long>(g.off + node) * p.hq + head;  // global row
      if (!split) {
        const float inv_l = 1.f / l_tot;
#pragma unroll
        for (int cc = 0; cc < 64; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kTmO + 64 * h + cc, o);
          tmem_ld_wait();
          if (seg_ok && row_valid) store_half_row_bf16(p.out + grow * 128 + 64 * h + cc, o, inv_l);
        }
        if (seg_ok && row_valid && h == 0 && p.lse != nullptr)
          p.lse[grow] = (m_fin + __log2f(l_tot)) * 0.69314718055994531f;
      } else {
        // unit cut between pairs: store this segment's unnormalised O, (m, l) and validity; the combine
        // kernel that runs after this one merges the segments
        const int myslot = g.slot * 2 + static_cast<int>(rank);
#pragma unroll
        for (int cc = 0; cc < 64; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kTmO + 64 * h + cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            __stcg(part_ptr(p, myslot, (64 * h + cc + c) >> 2, r),
                   make_float4(__uint_as_float(o[c]), __uint_as_float(o[c + 1]), __uint_as_float(o[c + 2]),
                               __uint_as_float(o[c + 3])));
        }
        if (h == 0) {
          __stcg(&p.part_ml[static_cast<long long>(myslot) * kBM + r], make_float2(m_fin, l_tot));
          __stcg(&p.part_ok[static_cast<long long>(myslot) * kBM + r], seg_ok ? 1 : 0);
        }
        if (iter.pair == g.c0 && rank == 0 && h == 0 && r == 0) {
          // descriptor of the split unit, indexed by its first pair (unique per split unit)
          int4 d;
          d.x = g.c1;
          d.y = g.off + g.mp * 2 * nodes_per_half;  // first global node of the unit
          d.z = g.N - g.mp * 2 * nodes_per_half;    // nodes of the sequence from there on
          d.w = g.kvh;
          __stcg(&p.units[g.c0], d);
        }
      }
    }
    ++sidx;
  }
  return ok;
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int npairs = static_cast<int>(gridDim.x) >> 1;
  // Let the combine kernel be scheduled now; its griddepcontrol.wait still holds it until this grid
  // has finished, but it no longer pays a launch after the last CTA exits.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Everything that does not depend on the plan is started before it: the barriers, the tensor-map
  // prefetches and the pair's tensor memory.  The cluster barrier below publishes the barriers to the
  // peer CTA before any arrival crosses over.
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.qfull[i], 1);
      mbar_init(&s.qempty[i], 1);
      mbar_init(&s.metafull[i], 32);
      mbar_init(&s.metaempty[i], kSoftmaxThreads);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.kfull[i], 1);  // the even CTA's arrival (with both CTAs' bytes)
      mbar_init(&s.kempty[i], 1);
      mbar_init(&s.vfull[i], 2);  // both CTAs' arrivals (the even CTA's with both CTAs' bytes)
      mbar_init(&s.vempty[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&s.sfull[i], 1);
      mbar_init(&s.pfull[i], kPfullCount);
      mbar_init(&s.pvdone[i], 1);
    }
    mbar_init(&s.drain, 1);
    mbar_init(&s.vpart, 1);
    s.abort_flag = 0;
    s.k_started = 0;
    fence_barrier_init();
  }
  if (warp == 0 && (tid & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc2(&s.tmem_base, kTmemCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();
  // the kernel before this one on the stream (which may produce any input) has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Slot `pair` of the split-unit table is written only by this pair (if it starts a split unit); clear
  // what an earlier call left there.
  if (tid == 0 && rank == 0 && pair < kMaxGrid) p.units[pair] = make_int4(0, 0, 0, 0);
  build_plan(s, p);
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  bool idle = s.bad_meta != 0;
  if (idle && blockIdx.x == 0 && tid == 0) report(p.status, JF_ERR_DEVICE_CHECK);
  const long long W = s.cum_work[p.batch];
  const int G = static_cast<int>(W < static_cast<long long>(npairs) ? W : static_cast<long long>(npairs));
  idle = idle || W <= 0 || pair >= G;  // uniform over the pair
  if (!idle) {
    SegIter iter;
    iter.x = static_cast<long long>(pair) * W / G;
    iter.xend = static_cast<long long>(pair + 1) * W / G;
    iter.W = W;
    iter.G = G;
    iter.pair = pair;
    {
      // first sequence touched by this pair: binary search over cum_work
      int lo = 0, hi = p.batch - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.cum_work[mid] <= iter.x) lo = mid; else hi = mid - 1;
      }
      iter.b = lo;
    }
    if (warp == 0 || warp == 2) {
      if (!kv_producer(s, p, iter, warp == 2, rank, &tm_q, warp == 2 ? &tm_v : &tm_k)) {
        set_abort(s, p);
        drain_delay();
      }
    } else if (warp == 1) {
      if (rank == 0 && (tid & 31) == 0) {
        bool issued = false;
        if (!mma_issuer(s, p, iter, tmem, issued)) {
          set_abort(s, p);
          if (issued) {
            // the pair's tensor memory is released only after the last MMA issued has completed
            mma2_commit_mc(&s.drain, 0x1);
            drain_wait(&s.drain, 0, kDrainNs);
          }
        }
      }
      __syncwarp();
    } else if (warp == 3) {
      if (!metadata(s, p, iter)) set_abort(s, p);
    } else {
      if (!softmax_epilogue(s, p, iter, tmem, rank)) set_abort(s, p);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs are done with the pair's tensor memory and with each other's barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// Combine kernel: merges the partials of every unit that was cut between CTAs.  A fixed grid (two
// blocks per SM) first compacts the split units out of the descriptor table (one slot per attention
// CTA pair) and then takes work items (split unit, 128-row half, 32-row block) in a grid-stride loop.  A thread
// owns one row and four 4-column groups and merges the unit's segments in a single pass with a
// running max, loading kSegBatch segments at a time (one memory round trip per batch).
// Launched right after the attention kernel (programmatic dependent launch), it waits for the
// attention grid before reading.
// ------------------------------------------------------------------------------------------------
constexpr int kCombineThreads = 256;
constexpr int kCombineRows = 32;
constexpr int kCombineQuads = 4;  // 4-column groups per thread (a block covers 32 rows x 32 * kCombineQuads columns)
constexpr int kSegBatch = 4;      // segments whose partials are loaded in one batch
constexpr int kColParts = 128 / (4 * kCombineQuads * (kCombineThreads / 32));  // column parts of a 32-row block
constexpr int kItemsPerUnit = kAttnQTiles * (kBM / kCombineRows) * kColParts;

__global__ void __launch_bounds__(kCombineThreads, 2) combine_kernel(const AttnParams p, int ncta) {
  static_assert(kMaxGrid <= kCombineThreads, "one descriptor slot per thread");
  static_assert(kColParts >= 1 && kColParts * 4 * kCombineQuads * (kCombineThreads / 32) == 128, "column split");
  __shared__ int4 s_desc[kMaxGrid];
  __shared__ int s_c0[kMaxGrid];
  __shared__ int s_wcount[kCombineThreads / 32];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the attention grid has completed
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // Compact the split units in CTA order (the same list in every block, so that work item i means
  // the same unit everywhere): thread c reads slot c.
  int4 dc = make_int4(0, 0, 0, 0);
  if (tid < ncta) dc = __ldcg(&p.units[tid]);
  const bool split_here = tid < ncta && dc.x > tid;  // a split unit starts at CTA tid and ends at dc.x
  const uint32_t bal = __ballot_sync(0xffffffffu, split_here);
  if (lane == 0) s_wcount[warp] = __popc(bal);
  __syncthreads();
  int base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kCombineThreads / 32; ++w) {
    base += (w < warp) ? s_wcount[w] : 0;
    total += s_wcount[w];
  }
  if (split_here) {
    const int k = base + __popc(bal & ((1u << lane) - 1u));
    s_desc[k] = dc;
    s_c0[k] = tid;
  }
  __syncthreads();
  const int s_n = total;
  const int n_items = s_n * kItemsPerUnit;
  const int rl = lane;
  const int nodes_per_tile = kBM / p.group;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int u = item / kItemsPerUnit;
    const int cp = item % kColParts;
    const int qt = (item / (kColParts * (kBM / kCombineRows))) % kAttnQTiles;
    const int rb = (item / kColParts) % (kBM / kCombineRows);
    const int q0 = (cp * (kCombineThreads / 32) + warp) * kCombineQuads;  // first 4-column group of this thread
    const int4 d = s_desc[u];
    const int c0 = s_c0[u], c1 = d.x;
    const int r = rb * kCombineRows + rl;  // row of the M tile
    const int node = qt * nodes_per_tile + r / p.group;
    if (node >= d.z) continue;
    const long long grow = static_cast<long long>(d.y + node) * p.hq + d.w * p.group + (r % p.group);
    float M = -INFINITY, L = 0.f;
    bool ok = true;
    float4 acc[kCombineQuads];
#pragma unroll
    for (int q = 0; q < kCombineQuads; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int cb = c0; cb <= c1; cb += kSegBatch) {
      float2 ml[kSegBatch];
      int okv[kSegBatch];
      float4 v[kSegBatch][kCombineQuads];
#pragma unroll
      for (int j = 0; j < kSegBatch; ++j) {
        const int c = cb + j;
        const bool have = c <= c1;
        const int sl = slot_of(c, c0) * kAttnQTiles + qt;
        ml[j] = have ? __ldcg(&p.part_ml[static_cast<long long>(sl) * kBM + r]) : make_float2(-INFINITY, 0.f);
        okv[j] = have ? __ldcg(&p.part_ok[static_cast<long long>(sl) * kBM + r]) : 1;
#pragma unroll
        for (int q = 0; q < kCombineQuads; ++q)
          v[j][q] = have ? __ldcg(part_ptr(p, sl, q0 + q, r)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float Mb = M;
#pragma unroll
      for (int j = 0; j < kSegBatch; ++j) {
        Mb = fmaxf(Mb, ml[j].x);
        ok = ok && okv[j] != 0;
      }
      if (Mb == -INFINITY) continue;  // nothing visible so far
      const float a = ex2_approx(M - Mb);  // 0 while M is still -inf
      L *= a;
#pragma unroll
      for (int q = 0; q < kCombineQuads; ++q) {
        acc[q].x *= a;
        acc[q].y *= a;
        acc[q].z *= a;
        acc[q].w *= a;
      }
#pragma unroll
      for (int j = 0; j < kSegBatch; ++j) {
        if (ml[j].x == -INFINITY) continue;
        const float w = ex2_approx(ml[j].x - Mb);
        L = fmaf(w, ml[j].y, L);
#pragma unroll
        for (int q = 0; q < kCombineQuads; ++q) {
          acc[q].x = fmaf(w, v[j][q].x, acc[q].x);
          acc[q].y = fmaf(w, v[j][q].y, acc[q].y);
          acc[q].z = fmaf(w, v[j][q].z, acc[q].z);
          acc[q].w = fmaf(w, v[j][q].w, acc[q].w);
        }
      }
      M = Mb;
    }
    if (!ok) continue;
    const float inv = 1.f / L;
    uint2* dst = reinterpret_cast<uint2*>(p.out + grow * 128 + q0 * 4);
#pragma unroll
    for (int q = 0; q < kCombineQuads; ++q)
      dst[q] = make_uint2(pack_bf16x2(acc[q].x * inv, acc[q].y * inv), pack_bf16x2(acc[q].z * inv, acc[q].w * inv));
    if (q0 == 0 && p.lse != nullptr) p.lse[grow] = (M + __log2f(L)) * 0.69314718055994531f;
  }
}

}  // namespace attn

static_assert(sizeof(attn::Smem) + 1024 <= 227 * 1024, "shared memory of one CTA (plus alignment slack)");
size_t attention_smem_bytes() { return sizeof(attn::Smem) + 1024; }

// CTA pairs of the attention grid on the current device: as many 2-CTA clusters as can be resident at once
// (one CTA per SM), at most kMaxGrid.  0 if the device cannot run the kernel.
static int attention_pairs(int dev) {
  static std::atomic<int> pairs_of_dev[kMaxDevices];
  int n = pairs_of_dev[dev].load(std::memory_order_acquire);
  if (n > 0) return n;
  const size_t smem = attention_smem_bytes();
  if (cudaFuncSetAttribute(attn::tree_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * kMaxGrid);
  cfg.blockDim = dim3(attn::kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = 2;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, attn::tree_attention_kernel, &cfg) != cudaSuccess || clusters <= 0) {
    cudaGetLastError();
    return 0;
  }
  n = clusters < kMaxGrid ? clusters : kMaxGrid;
  pairs_of_dev[dev].store(n, std::memory_order_release);
  return n;
}

cudaError_t launch_tree_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                  const AttnParams& p, cudaStream_t stream) {
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  const int pairs = attention_pairs(dev);
  if (pairs <= 0) return cudaErrorNotSupported;
  cudaLaunchAttribute cl;
  cl.id = cudaLaunchAttributeClusterDimension;
  cl.val.clusterDim.x = 2;
  cl.val.clusterDim.y = 1;
  cl.val.clusterDim.z = 1;
  cudaError_t e = launch_pdl(attn::tree_attention_kernel, dim3(2 * pairs), dim3(attn::kThreads),
                             attention_smem_bytes(), stream, &cl, tm_q, tm_k, tm_v, p);
  if (e != cudaSuccess) return e;
  // The combine kernel may start as soon as the attention grid is scheduled; its griddepcontrol.wait
  // holds it until the attention grid has finished and its writes are visible.
  return launch_pdl(attn::combine_kernel, dim3(4 * pairs), dim3(attn::kCombineThreads), 0, stream, nullptr, p,
                    pairs);
}

}  // namespace jf
