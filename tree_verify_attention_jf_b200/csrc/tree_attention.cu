// tree_attention.cu -- tree-causal attention over a paged bf16 KV cache on sm_100a.
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 2, tree-causal attention mask and branch factorisation): the
// query of every draft-tree node attends to its sequence's whole cached prefix plus the tree slots of
// its own root path (itself included), never to descendants or unrelated branches.
//
// How (B200-specific design, not taken from the pages, which only name an sm_90 paged kernel):
//   * GQA packing: one M tile = 128 rows = (128 / g) tree nodes x g query heads of one kv head.  A work
//     unit is a pair of M tiles of the same kv head: both are multiplied against every staged K/V tile,
//     which halves the K/V traffic per unit of tensor-core work.
//   * Per CTA (persistent, one per SM, 12 warps): warp 0 loads both Q tiles with TMA (once per
//     segment) and gathers K, warp 2 gathers V: 128 keys (8 pages of 16 tokens) per tile, one TMA box
//     per page and 64-column half, 128-byte swizzled, gathered through the block table; the 16 boxes of
//     a tile are issued by 16 lanes at once.  Warp 1 allocates all 512 tensor-memory columns
//     (S0 | S1 | O0 | O1) and issues tcgen05.mma: S_i = Q_i K^T (both operands from shared memory,
//     K-major) and O_i += P_i V with P_i read straight from TMEM (aliasing S_i) and V as an MN-major
//     shared-memory operand, in the order PV0(j), QK0(j+1), PV1(j), QK1(j+1) so that each softmax
//     warpgroup works while the tensor core serves the other one.  Warp 3 validates each segment.
//     Warps 4-7 and 8-11 (one thread per row of M tile 0 / 1) build the per-node 256-bit ancestor
//     bitsets by pointer jumping in shared memory at each tree-holding segment start, run the online
//     softmax out of TMEM with a lazy rescale of O, and the epilogue.
//   * The tree mask only touches tiles that hold tree slots; prefix tiles are unmasked.
//   * Work split: the flattened (unit, kv tile) space, in which every unit also carries a fixed cost for
//     the segment start, is cut into equal contiguous ranges, one per CTA (stream-K).  A unit cut
//     between CTAs writes fp32 partials (O, running max, row sum) and its first CTA records the unit
//     in a descriptor slot; combine_kernel, launched right behind on the
//     same stream with a programmatic dependency, merges each recorded unit's partials and stores the
//     bf16 output.  Nothing spins on another CTA.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "jf_device.cuh"
#include "jf_internal.h"

namespace jf {
#ifdef JF_DEBUG
// Debug build only: while g_debug_hold is nonzero, every attention CTA first waits for it to clear.  Nothing
// clears it during a call, so the wait runs out -- before any copy or MMA is issued -- and the call must come
// back with JF_ERR_TIMEOUT in dev_status and the context still usable (set by jf_debug_hold).
__device__ int g_debug_hold;
#endif
namespace attn {

constexpr int kPage = 16;
constexpr int kBM = 128;             // rows per M tile
constexpr int kBN = 128;             // keys per KV tile
constexpr int kPagesPerTile = kBN / kPage;
constexpr int kStages = 2;
constexpr int kThreads = 384;
constexpr int kHalfBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmS = 0;    // S_i at column 128 * i
constexpr uint32_t kTmO = 256;  // O_i at column 256 + 128 * i
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may grow up to 2^8 before O is rescaled
constexpr int kSegCost = 3;  // kv tiles' worth of time that starting a segment in mid-kernel costs

struct __align__(1024) Smem {
  uint8_t q[kAttnQTiles][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint32_t anc[kMaxTreeNodes][kAncWords];  // ancestor bitsets of the current segment's nodes
  int jmp[kMaxTreeNodes];                   // pointer-jumping links while they are built
  long long cum_work[kMaxAttnBatch + 1];
  int seq_p[kMaxAttnBatch];       // prefix length of every sequence (copied once by the plan)
  int seq_off[kMaxAttnBatch + 1]; // tree_offsets
  long long scan_warp[kThreads / 32];
  uint64_t bar_qfull, bar_qempty;
  uint64_t bar_kfull[kStages], bar_kempty[kStages], bar_vfull[kStages], bar_vempty[kStages];
  // 8-bit cache: the copies land on these; the copy warp converts the tile and then arrives on the full barrier
  uint64_t bar_qland, bar_kland[kStages], bar_vland[kStages];
  uint64_t bar_sfull[kAttnQTiles], bar_pfull[kAttnQTiles], bar_pvdone[kAttnQTiles];
  uint64_t bar_metafull[2], bar_metaempty[2];
  uint64_t bar_drain;  // the MMA warp's last MMA, waited for when unwinding after an abort
  uint32_t tmem_base;
  int meta_valid[2];
  int meta_ctl;
  int abort_flag;
  int bad_meta;
  int k_started;  // the K gather has issued its first tile (the V gather's first tile goes after it)
};

struct Seg {
  int b, kvh, mp, kb, ke;  // positions [kb, ke) of unit (b, kvh, M-tile pair mp)
  int P, N, off, kt;       // prefix length, nodes, first global node, kv tiles of the sequence
  int c0, c1, slot;        // CTAs sharing the unit; this CTA's partial slot (times kAttnQTiles)
  int rot;                 // the unit's rotation: position t reads kv tile (t - rot) mod kt
  __device__ __forceinline__ int tile(int t) const {
    const int x = t - rot;
    return x < 0 ? x + kt : x;
  }
};

__device__ __forceinline__ int cta_of(long long x, long long W, int G) {
  return static_cast<int>(((x + 1) * G - 1) / W);
}

__device__ __forceinline__ int pairs_of(int N, int group) {
  const int mtn = (N * group + kBM - 1) / kBM;
  return (mtn + kAttnQTiles - 1) / kAttnQTiles;
}

// Cost space: a unit costs kSegCost + kt, its kt positions preceded by kSegCost that stand for the time a
// CTA loses when it starts a segment in mid-kernel (the previous segment's epilogue, the Q reload, the refill
// of the K/V pipeline).  Cutting this space into equal ranges gives a CTA that crosses a unit boundary
// correspondingly fewer kv tiles.  A CTA whose range ends inside a unit's leading positions takes no part in
// that unit.
//
// Positions map to kv tiles through a rotation per unit, chosen so that the CTA owning the unit's last
// position starts its range on kv tile 0.  Every CTA starts at the same time and moves at about the same
// rate, so at local time x a CTA reads tile x or tile x + (kt - W / G) of its unit: the M-tile pairs of one
// (sequence, kv head), which read the same K and V, do so at two offsets instead of one offset each, and the
// later readers find most of the tiles in L2.  Any rotation keeps the pieces of a unit disjoint.
struct SegIter {
  long long x, xend, W;
  int G, b;
  __device__ bool next(const Smem& s, const AttnParams& p, Seg& g) {
    while (x < xend) {
      while (s.cum_work[b + 1] <= x) ++b;
      g.b = b;
      g.P = s.seq_p[b];
      g.off = s.seq_off[b];
      g.N = s.seq_off[b + 1] - g.off;
      g.kt = (g.P + g.N + kBN - 1) / kBN;
      const long long span = g.kt + kSegCost;
      const int mpn = pairs_of(g.N, p.group);
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
      g.c0 = cta_of(u0 + kSegCost, W, G);  // owner of the unit's first kv tile
      g.c1 = cta_of(u1 - 1, W, G);         // owner of its last
      g.slot = (static_cast<int>(blockIdx.x) == g.c0) ? 2 * blockIdx.x + 1 : 2 * blockIdx.x;
      const long long k1 = static_cast<long long>(g.c1) * W / G - u0 - kSegCost;  // where the owner of the last starts
      g.rot = k1 > 0 ? static_cast<int>(k1) : 0;
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

__device__ __forceinline__ void set_abort(Smem& s, const AttnParams& p) {
  *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
  report(p.status, JF_ERR_TIMEOUT);
}

// While unwinding after an abort: waits up to `ns` for a phase, ignoring the abort flag, so that copies and
// MMAs already issued finish before the CTA releases its tensor memory and exits.
constexpr uint64_t kDrainNs = kWaitLimitNs;
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kDrainNs) return;
}

// ------------------------------------------------------------------------------------------------
// Plan: per-sequence cost (kv heads x M-tile pairs x (kv tiles + kSegCost)), exclusive prefix sum in shared memory,
// validation of the batch-level metadata.  Every CTA computes the same plan.
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
    local += static_cast<long long>(p.hkv) * pairs_of(N, p.group) * (kt + kSegCost);
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
    run += static_cast<long long>(p.hkv) * pairs_of(N, p.group) * (kt + kSegCost);
  }
  if (tid == kThreads - 1) s.cum_work[B] = run;
  __syncthreads();
}

// ------------------------------------------------------------------------------------------------
// 8-bit (E4M3) cache: conversion to f16 in shared memory.  Every E4M3 value is exactly an f16, so the MMAs
// run on f16 operands (Q converted from bf16, which it also represents exactly in the range of attention
// inputs) and see exactly the decoded cache; the caches' scales are applied outside (K's in the softmax
// scale, V's in the normalisation).
// ------------------------------------------------------------------------------------------------
// One K or V stage: the copy put the tile's 8-bit rows (128 keys x 128 dims, one 128-byte row per key) in the
// stage's upper 16 KB; they become f16 in the 128-byte-swizzled [half][128 keys][64 dims] layout of the whole
// stage.  A warp converts 16 rows [r0, r0 + 16) per step (4 chunks of 16 bytes per lane, all read before any is
// written), the steps in order r0 = 0, 16, ..., 112: the writes of a step land in rows [0, 16 KB) and on the 8-bit
// rows the same step has just read, so rows still to be read are never overwritten.
__device__ __forceinline__ void convert_stage_e4m3_step(uint8_t* stage, int lane, int r0) {
  const int c = lane & 7;  // 16-byte chunk of the 8-bit row: dims [16 c, 16 c + 16)
  const int j0 = 2 * (c & 3);  // its f16 bytes are chunks j0, j0 + 1 of half c / 4
  uint4 raw[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    raw[k] = *reinterpret_cast<const uint4*>(stage + kHalfBytes + (r0 + (lane >> 3) + 4 * k) * 128 + c * 16);
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = r0 + (lane >> 3) + 4 * k;
    const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
    uint32_t hv[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2_raw lo =
          __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] & 0xffffu), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
      hv[2 * i] = static_cast<uint32_t>(lo.x) | (static_cast<uint32_t>(lo.y) << 16);
      hv[2 * i + 1] = static_cast<uint32_t>(hi.x) | (static_cast<uint32_t>(hi.y) << 16);
    }
    uint8_t* base = stage + (c >> 2) * kHalfBytes + row * 128;
    *reinterpret_cast<uint4*>(base + ((j0 ^ (row & 7)) * 16)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(base + (((j0 + 1) ^ (row & 7)) * 16)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
  }
  __syncwarp();
}
constexpr int kConvSteps = kBN / 16;  // 16-row steps per stage

// The Q tiles in place, bf16 -> f16, element by element (the swizzle does not matter).
__device__ __forceinline__ void convert_q_bf16_f16(uint8_t* q, int bytes, int lane) {
#pragma unroll 4
  for (int i = lane * 16; i < bytes; i += 32 * 16) {
    uint4 v = *reinterpret_cast<const uint4*>(q + i);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half2 h = __floats2half2_rn(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
      w[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(q + i) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------------------------------------------------
// Warps 0 and 2: K / V gathers (warp 0 also loads the Q tiles).  With an 8-bit cache each tile lands on a
// barrier of its own; while the warp waits for a stage to free it converts the landed tiles in order, 16 rows
// at a time, and arrives on the full barrier the MMA warp waits on once a tile is done (the Q tiles are
// converted right after the segment's first K tile is issued).
// ------------------------------------------------------------------------------------------------
template <bool kFp8>
__device__ void kv_producer(Smem& s, const AttnParams& p, SegIter iter, bool is_v, const CUtensorMap* tm_q,
                            const CUtensorMap* tm_kv) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  uint64_t* full = is_v ? s.bar_vfull : s.bar_kfull;
  uint64_t* empty = is_v ? s.bar_vempty : s.bar_kempty;
  uint64_t* land = kFp8 ? (is_v ? s.bar_vland : s.bar_kland) : full;
  uint64_t* qland = kFp8 ? &s.bar_qland : &s.bar_qfull;
  Seg g;
  uint32_t it = 0, sidx = 0;
  uint32_t cit = 0;  // 8-bit cache: tiles converted so far (tiles [cit, it) are issued and not yet converted)
  int cstep = 0;     // next 16-row step of tile cit
  bool q_pend = false;
  // the latest phase this warp armed on each landing barrier (bit st of armed; its parity in armed_par), and on
  // the Q landing barrier: on an abort the warp waits for them, i.e. for every copy it issued
  uint32_t armed = 0, armed_par = 0, q_armed = 0, q_par = 0;
  auto unwind = [&]() {
    set_abort(s, p);
    for (int st = 0; st < kStages; ++st)
      if (armed & (1u << st)) drain_wait(&land[st], (armed_par >> st) & 1u);
    if (q_armed) drain_wait(qland, q_par);
  };
  // One step of the oldest unconverted tile: 1 = done, 0 = nothing to convert or (block false) not landed yet,
  // -1 = the landing wait ran out.  The tile's last step hands it to the MMA warp.
  auto conv_step = [&](bool block) -> int {
    if (!kFp8 || cit == it) return 0;
    const int cst = cit % kStages;
    const uint32_t cph = (cit / kStages) & 1;
    if (cstep == 0) {
      if (block) {
        if (!warp_wait(&land[cst], cph, abort)) return -1;
      } else if (!__all_sync(0xffffffffu, mbar_test_wait(&land[cst], cph))) {
        return 0;
      }
    }
    convert_stage_e4m3_step(is_v ? s.v[cst] : s.k[cst], lane, cstep * 16);
    if (++cstep == kConvSteps) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[cst]);
      cstep = 0;
      ++cit;
    }
    return 1;
  };
  auto convert_all = [&]() -> bool {
    while (cit != it)
      if (conv_step(true) < 0) return false;
    return true;
  };
  const int nodes_per_tile = kBM / p.group;
  while (iter.next(s, p, g)) {
    const int npg = (g.P + g.N + kPage - 1) / kPage;
    const int32_t* bt = p.block_table + static_cast<long long>(g.b) * p.max_pages;
    // Page ids are fetched four positions at a time (lane l: logical page 8 * tile(t0 + l / 8) + l % 8, -1 = not
    // loaded) and one batch ahead, so the block-table latency stays off the issue path.
    auto batch_ids = [&](int t0) {
      int pid = -1;
      const int t = t0 + (lane >> 3);
      if (t < g.ke) {
        const int pg = g.tile(t) * kPagesPerTile + (lane & 7);
        if (pg < npg && pg < p.max_pages) {
          const int v = __ldg(bt + pg);
          if (v >= 0 && v < p.num_pages) pid = v;
        }
      }
      return pid;
    };
    int ids_cur = batch_ids(g.kb);
    int ids_next = batch_ids(g.kb + 4);
    // 8-bit cache: the previous segment's last K tiles are converted now -- the Q buffer frees only after their
    // QKs have run
    if (!is_v && !convert_all()) return unwind();
    // the Q tiles go out while the page ids are on their way
    if (!is_v) {
      if (!warp_wait(&s.bar_qempty, (sidx & 1) ^ 1, abort)) return unwind();
      if (lane == 0) mbar_arrive_expect_tx(qland, kAttnQTiles * kTileBytes);
      q_armed = 1;
      q_par = sidx & 1;
      __syncwarp();
      if (lane < 2 * kAttnQTiles) {  // lane: Q tile lane / 2, half lane % 2
        const int qt = lane >> 1, half = lane & 1;
        const int node0 = g.off + (g.mp * kAttnQTiles + qt) * nodes_per_tile;
        tma_load_3d(s.q[qt] + half * kHalfBytes, tm_q, qland, half * 64, g.kvh * p.group, node0);
      }
      q_pend = kFp8;
    }
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int st = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      const int bi = (t - g.kb) & 3;
      if (bi == 0 && t > g.kb) {
        ids_cur = ids_next;
        ids_next = batch_ids(t + 4);
      }
      // bf16: lane j < 16 copies page j / 2, 64-column half j % 2; 8-bit: lane j < 8 copies page j (whole rows)
      int pid = __shfl_sync(0xffffffffu, ids_cur, bi * 8 + (kFp8 ? (lane & 7) : ((lane >> 1) & 7)));
      if (lane >= (kFp8 ? 1 : 2) * kPagesPerTile) pid = -1;
      const uint32_t mask = __ballot_sync(0xffffffffu, pid >= 0);
      const uint32_t bytes = static_cast<uint32_t>(__popc(mask)) * (kPage * 128u);
      if (kFp8) {
        // convert landed tiles step by step while the stage is still in use
        const uint64_t t0 = globaltimer();
        uint32_t spins = 0;
        while (!__all_sync(0xffffffffu, mbar_test_wait(&empty[st], ph ^ 1))) {
          const int r = conv_step(false);
          if (r < 0) return unwind();
          if (r == 0) {
            // a short sleep hands the SMSP's issue slots to the softmax warps; a landing or a free stage is
            // still seen within a fraction of a conversion step
            __nanosleep(64);
            if ((++spins & 31u) == 0 && (*abort || globaltimer() - t0 > kWaitLimitNs)) return unwind();
          }
        }
      } else if (!warp_wait(&empty[st], ph ^ 1, abort)) {
        return unwind();
      }
      if (is_v && it == 0) {
        // The copy engine serves requests in order and the first S needs Q and K only: the kernel's
        // first V tile is queued behind the first K tile (bounded wait, like every other).
        const uint64_t t0 = globaltimer();
        while (*reinterpret_cast<volatile int*>(&s.k_started) == 0) {
          if (*abort || globaltimer() - t0 > kWaitLimitNs) return unwind();
        }
      }
      if (lane == 0) mbar_arrive_expect_tx(&land[st], bytes);
      armed |= 1u << st;
      armed_par = (armed_par & ~(1u << st)) | (ph << st);
      __syncwarp();
      if (pid >= 0) {
        uint8_t* stage = is_v ? s.v[st] : s.k[st];
        if (kFp8) {
          tma_load_3d(stage + kHalfBytes + lane * (kPage * 128), tm_kv, &land[st], 0, g.kvh, pid * kPage);
        } else {
          const int half = lane & 1;
          tma_load_3d(stage + half * kHalfBytes + (lane >> 1) * (kPage * 128), tm_kv, &land[st], half * 64, g.kvh,
                      pid * kPage);
        }
      }
      if (!is_v && it == 0) {
        __syncwarp();
        if (lane == 0) *reinterpret_cast<volatile int*>(&s.k_started) = 1;
      }
      if (kFp8) {
        // segment start: the Q tiles, while this K tile is on its way
        if (q_pend) {
          if (!warp_wait(&s.bar_qland, sidx & 1, abort)) return unwind();
          convert_q_bf16_f16(&s.q[0][0], kAttnQTiles * kTileBytes, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.bar_qfull);
          q_pend = false;
        }
      }
    }
    ++sidx;
  }
  if (!convert_all()) return unwind();
}

// ------------------------------------------------------------------------------------------------
// Warp 1: tcgen05.mma issuer
// ------------------------------------------------------------------------------------------------
// Instruction descriptor of kind::f16 with f16 operands (the 8-bit cache path): the bf16 one with both operand
// format fields (bits 7-9, 10-12) set to 0 = f16.
__host__ __device__ constexpr uint32_t idesc_operands(uint32_t bf16_idesc, bool f16) {
  return f16 ? (bf16_idesc & ~((7u << 7) | (7u << 10))) : bf16_idesc;
}

template <bool kFp8>
__device__ __forceinline__ void issue_qk(const Smem& s, uint32_t tmem, int qt, int st) {
  constexpr uint32_t idesc = idesc_operands(idesc_bf16_f32(kBM, kBN, false, false), kFp8);
  const uint32_t qaddr = smem_u32(s.q[qt]);
  const uint32_t kaddr = smem_u32(s.k[st]);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
    mma_ss(tmem + kTmS + qt * 128, smem_desc_sw128(qaddr + off, 16, 1024), smem_desc_sw128(kaddr + off, 16, 1024),
           idesc, kk > 0 ? 1u : 0u);
  }
}

template <bool kFp8>
__device__ __forceinline__ void issue_pv(const Smem& s, uint32_t tmem, int qt, int st, bool first) {
  constexpr uint32_t idesc = idesc_operands(idesc_bf16_f32(kBM, 128, false, true), kFp8);
  const uint32_t vaddr = smem_u32(s.v[st]);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    mma_ts(tmem + kTmO + qt * 128, tmem + kTmS + qt * 128 + kk * 8, smem_desc_sw128(vaddr + kk * 2048, kHalfBytes, 1024),
           idesc, (first && kk == 0) ? 0u : 1u);
  }
}

template <bool kFp8>
__device__ void mma_issuer(Smem& s, const AttnParams& p, SegIter iter, uint32_t tmem) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  Seg g;
  uint32_t it = 0, sidx = 0;
  bool issued = false;
  auto unwind = [&]() {  // the last MMA issued completes before the CTA releases its tensor memory
    set_abort(s, p);
    if (issued) {
      if (lane == 0) mma_commit(&s.bar_drain);
      __syncwarp();
      drain_wait(&s.bar_drain, 0);
    }
  };
  while (iter.next(s, p, g)) {
    if (!warp_wait(&s.bar_qfull, sidx & 1, abort)) return unwind();
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int st = it % kStages;
      if (t == g.kb) {  // S of the segment's first tile for both Q tiles
        if (!warp_wait(&s.bar_kfull[st], (it / kStages) & 1, abort)) return unwind();
        tc_fence_after();
        if (lane == 0) {
          issue_qk<kFp8>(s, tmem, 0, st);
          mma_commit(&s.bar_sfull[0]);
          issue_qk<kFp8>(s, tmem, 1, st);
          mma_commit(&s.bar_sfull[1]);
          mma_commit(&s.bar_kempty[st]);
          if (t == g.ke - 1) mma_commit(&s.bar_qempty);
        }
        __syncwarp();
        issued = true;
      }
      const bool has_next = t + 1 < g.ke;
      const int st1 = (it + 1) % kStages;
      if (has_next && !warp_wait(&s.bar_kfull[st1], ((it + 1) / kStages) & 1, abort)) return unwind();
      if (!warp_wait(&s.bar_vfull[st], (it / kStages) & 1, abort)) return unwind();
      const int zf = g.P + g.N - g.tile(t) * kBN;  // first row of this tile past the sequence
      if (zf < kBN) {
        // Keys beyond the sequence's last slot: clear their V rows so stale cache contents (even NaN)
        // cannot reach the output through 0 * V.  A whole 128-byte row is cleared, so the swizzle does
        // not matter.
        uint8_t* vb = s.v[st];
        const int z0 = zf < 0 ? 0 : zf;
        const int nchunks = (kBN - z0) * 16;
        for (int i = lane; i < nchunks; i += 32) {
          const int row = z0 + (i >> 4);
          const int half = (i >> 3) & 1;
          const int c = i & 7;
          *reinterpret_cast<uint4*>(vb + half * kHalfBytes + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      for (int qt = 0; qt < kAttnQTiles; ++qt) {
        if (!warp_wait(&s.bar_pfull[qt], it & 1, abort)) return unwind();
        tc_fence_after();
        if (lane == 0) {
          issue_pv<kFp8>(s, tmem, qt, st, t == g.kb);
          mma_commit(&s.bar_pvdone[qt]);
          if (qt == kAttnQTiles - 1) mma_commit(&s.bar_vempty[st]);
          if (has_next) {
            issue_qk<kFp8>(s, tmem, qt, st1);
            mma_commit(&s.bar_sfull[qt]);
            if (qt == kAttnQTiles - 1) {
              mma_commit(&s.bar_kempty[st1]);
              if (t + 1 == g.ke - 1) mma_commit(&s.bar_qempty);
            }
          }
        }
        __syncwarp();
        issued = true;
      }
    }
    ++sidx;
  }
}

// ------------------------------------------------------------------------------------------------
// Warp 3: per-segment validation
// ------------------------------------------------------------------------------------------------
__device__ void metadata(Smem& s, const AttnParams& p, SegIter iter) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  Seg g;
  uint32_t sidx = 0;
  while (iter.next(s, p, g)) {
    const int buf = sidx & 1;
    if (lane == 0) {
      const bool ok = mbar_wait(&s.bar_metaempty[buf], ((sidx >> 1) & 1) ^ 1, abort);
      s.meta_ctl = ok ? 1 : 0;
      if (!ok) set_abort(s, p);
    }
    __syncwarp();
    if (s.meta_ctl == 0) return;
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
    int bad = (static_cast<long long>(g.P) + g.N > static_cast<long long>(p.max_pages) * kPage) ? 1 : 0;
    // the segment's tiles: [a, a + len) of the unit, wrapped at kt
    const int a = g.tile(g.kb), len = g.ke - g.kb;
    const int first_end = a + len < g.kt ? a + len : g.kt;
    for (int part = 0; part < 2; ++part) {
      const int t0 = part == 0 ? a : 0, t1 = part == 0 ? first_end : a + len - g.kt;
      int pg1 = t1 * kPagesPerTile;
      if (pg1 > npg) pg1 = npg;
      if (pg1 > p.max_pages) pg1 = p.max_pages;
      for (int pg = t0 * kPagesPerTile + lane; pg < pg1; pg += 4 * 32) {
        int v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = (pg + 32 * u < pg1) ? __ldg(bt + pg + 32 * u) : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (v[u] < 0 || v[u] >= p.num_pages) bad = 1;
      }
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
    mbar_arrive(&s.bar_metafull[buf]);
    ++sidx;
  }
}

// ------------------------------------------------------------------------------------------------
// Warps 4-11: online softmax (one thread per row of M tile 0 or 1) and the epilogue
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const float* o, float inv_l) {
#pragma unroll
  for (int c = 0; c < 32; c += 8) {
    uint4 v;
    v.x = pack_bf16x2(o[c + 0] * inv_l, o[c + 1] * inv_l);
    v.y = pack_bf16x2(o[c + 2] * inv_l, o[c + 3] * inv_l);
    v.z = pack_bf16x2(o[c + 4] * inv_l, o[c + 5] * inv_l);
    v.w = pack_bf16x2(o[c + 6] * inv_l, o[c + 7] * inv_l);
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
// float4 index ((slot * 32 + c4) * 128 + row), slot = 2 * (segment slot) + Q tile.
__device__ __forceinline__ float4* part_ptr(const AttnParams& p, int slot, int c4, int r) {
  return reinterpret_cast<float4*>(p.part_o) + (static_cast<long long>(slot) * 32 + c4) * kBM + r;
}

// Named barrier 1 joins the 256 softmax threads (warps 4-11).
__device__ __forceinline__ void softmax_bar() { named_bar_sync(1, 2 * kBM); }
__device__ __forceinline__ bool softmax_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(2 * kBM)
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

// A warp whose wait gives up (ok = false) keeps walking the segments with its work skipped, so that the
// ancestor build's named barriers are still reached by all 256 softmax threads; it reports the abort once.
template <bool kFp8>
__device__ void softmax_epilogue(Smem& s, const AttnParams& p, SegIter iter, uint32_t tmem, int qt) {
  const int r = threadIdx.x - 128 - qt * kBM;  // row of M tile qt == TMEM lane
  const int wq = (threadIdx.x >> 5) & 3;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t s_col = kTmS + qt * 128, o_col = kTmO + qt * 128;
  volatile int* abort = &s.abort_flag;
  const float sl2 = p.scale_log2;
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const int nodes_per_tile = kBM / p.group;
  Seg g;
  uint32_t it = 0, sidx = 0;
  bool ok = true;
  while (iter.next(s, p, g)) {
    const int buf = sidx & 1;
    const int node = (g.mp * kAttnQTiles + qt) * nodes_per_tile + r / p.group;
    const int head = g.kvh * p.group + (r % p.group);
    const bool row_valid = node < g.N;
    // the segment reads a tile with tree keys (tiles P / kBN .. kt - 1) iff its rotated range reaches P / kBN
    if (g.tile(g.kb) + (g.ke - g.kb) > g.P / kBN && !build_ancestors(s, p, g)) ok = false;
    const uint32_t* anc = &s.anc[row_valid ? node : 0][0];
    float m_use = -INFINITY, l = 0.f;
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int kv = g.tile(t);
      const bool tree_tile = (kv + 1) * kBN > g.P;
      if (!ok) continue;
      if (!warp_wait(&s.bar_sfull[qt], it & 1, abort)) {
        ok = false;
        continue;
      }
      // S_qt(it) ready also means PV_qt(it-1) is complete: its commit tracks every earlier MMA.
      tc_fence_after();
      // The row of S in registers, in two halves: the max of the first half is taken while the
      // second half is still on its way from TMEM.
      uint32_t sr[128];
      tmem_ld32(lane_base + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(lane_base + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      uint32_t vis[4];
#pragma unroll
      for (int w = 0; w < 4; ++w)
        vis[w] = tree_tile ? vis_word(kv * kBN + 32 * w, g.P, g.N, row_valid, anc) : 0xffffffffu;
      tmem_ld_wait();
      tmem_ld32(lane_base + s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(lane_base + s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (hh == 1) tmem_ld_wait();
        if (tree_tile) {
          // invisible keys become -inf: they drop out of the max and get P = 2^-inf = 0
#pragma unroll
          for (int c = 64 * hh; c < 64 * hh + 64; ++c)
            if (!((vis[c >> 5] >> (c & 31)) & 1u)) sr[c] = 0xff800000u;
        }
#pragma unroll
        for (int c = 64 * hh; c < 64 * hh + 64; c += 8) {
          a0 = fmax3(a0, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
          a1 = fmax3(a1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
          a2 = fmax3(a2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
          a3 = fmax3(a3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
        }
      }
      const float mraw = fmax3(a0, a1, fmaxf(a2, a3));
      const float mx = (mraw == -INFINITY) ? -INFINITY : mraw * sl2;
      float alpha = 1.f;
      bool resc = false;
      if (mx > m_use + kRescaleThreshold) {
        if (m_use != -INFINITY) {
          alpha = ex2_approx(m_use - mx);
          l *= alpha;
          resc = (t > g.kb);
        }
        m_use = mx;
      }
      const float negm = (m_use == -INFINITY) ? 0.f : -m_use;
      const uint64_t nm2 = f2_pack(negm, negm);
      // P = 2^(s * scale - m), row sum in packed pairs, bf16 pairs of P written over S's first 64
      // columns, a quarter (16 packed columns) at a time
      uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int cc = 32 * h + c;
          const uint64_t y = f2_fma(f2_pack(__uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1])), sl2x2, nm2);
          float y0, y1;
          f2_unpack(y, y0, y1);
          const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
          if ((c >> 1) & 1) acc1 = f2_add(acc1, f2_pack(p0, p1));
          else acc0 = f2_add(acc0, f2_pack(p0, p1));
          if (kFp8) {
            const __half2 hp = __floats2half2_rn(p0, p1);  // the PV operands are f16 on this path
            pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
          } else {
            pk[c >> 1] = pack_bf16x2_alu(p0, p1);
          }
        }
        tmem_st16(lane_base + s_col + 16 * h, pk);
      }
      {
        float u0, u1, v0, v1;
        f2_unpack(acc0, u0, u1);
        f2_unpack(acc1, v0, v1);
        l += (u0 + u1) + (v0 + v1);
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O_qt already holds PV_qt(it-1) (implied by S_qt(it) being ready)
        const float a = resc ? alpha : 1.f;
#pragma unroll
        for (int cc = 0; cc < 128; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + o_col + cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
          tmem_st32(lane_base + o_col + cc, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.bar_pfull[qt]);
    }
    // ---------------- epilogue of the segment
    if (ok && !warp_wait(&s.bar_metafull[buf], (sidx >> 1) & 1, abort)) ok = false;
    const bool seg_ok = s.meta_valid[buf] != 0;
    if (ok && !warp_wait(&s.bar_pvdone[qt], (it - 1) & 1, abort)) ok = false;
    if (!ok) {
      ++sidx;
      continue;
    }
    tc_fence_after();
    mbar_arrive(&s.bar_metaempty[buf]);
    const bool split = g.c0 != g.c1;
    const long long grow = static_cast<long long>(g.off + node) * p.hq + head;  // global row
    if (!split) {
      const float inv_l = p.v_scale / l;  // the V cache's scale (1 for a bf16 cache)
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + o_col + cc, o);
        tmem_ld_wait();
        if (seg_ok && row_valid)
          store_row_bf16(p.out + grow * 128 + cc, reinterpret_cast<const float*>(o), inv_l);
      }
      if (seg_ok && row_valid && p.lse != nullptr) p.lse[grow] = (m_use + __log2f(l)) * 0.69314718055994531f;
    } else {
      // unit cut between CTAs: store this segment's unnormalised O, (m, l) and validity; the combine
      // kernel that runs after this one merges the segments
      const int myslot = g.slot * kAttnQTiles + qt;
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + o_col + cc, o);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          __stcg(part_ptr(p, myslot, (cc + c) >> 2, r),
                 make_float4(__uint_as_float(o[c]), __uint_as_float(o[c + 1]), __uint_as_float(o[c + 2]),
                             __uint_as_float(o[c + 3])));
      }
      __stcg(&p.part_ml[static_cast<long long>(myslot) * kBM + r], make_float2(m_use, l));
      __stcg(&p.part_ok[static_cast<long long>(myslot) * kBM + r], seg_ok ? 1 : 0);
      if (static_cast<int>(blockIdx.x) == g.c0 && r == 0) {
        // descriptor of the split unit, indexed by its first CTA (unique per split unit)
        int4 d;
        d.x = g.c1;
        d.y = g.off + g.mp * kAttnQTiles * nodes_per_tile;  // first global node of the unit
        d.z = g.N - g.mp * kAttnQTiles * nodes_per_tile;    // nodes of the sequence from there on
        d.w = g.kvh;
        if (qt == 0) __stcg(&p.units[g.c0], d);
      }
    }
    ++sidx;
  }
  if (!ok) set_abort(s, p);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    tree_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  // Let the combine kernel be scheduled now; its griddepcontrol.wait still holds it until this grid
  // has finished, but it no longer pays a launch after the last CTA exits.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Everything that does not depend on the plan is started before it, so that its latency (cold
  // descriptor and tensor-memory setup) hides behind the plan's metadata loads: the barriers, the
  // tensor-map prefetches and the TMEM allocation.  The plan's barriers publish all of it.
  if (tid == 0) {
    mbar_init(&s.bar_qfull, 1);
    mbar_init(&s.bar_qland, 1);
    mbar_init(&s.bar_qempty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.bar_kfull[i], 1);
      mbar_init(&s.bar_kland[i], 1);
      mbar_init(&s.bar_vland[i], 1);
      mbar_init(&s.bar_kempty[i], 1);
      mbar_init(&s.bar_vfull[i], 1);
      mbar_init(&s.bar_vempty[i], 1);
    }
    for (int i = 0; i < kAttnQTiles; ++i) {
      mbar_init(&s.bar_sfull[i], 1);
      mbar_init(&s.bar_pfull[i], kBM);
      mbar_init(&s.bar_pvdone[i], 1);
    }
    mbar_init(&s.bar_drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_metafull[i], 32);
      mbar_init(&s.bar_metaempty[i], kAttnQTiles * kBM);
    }
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
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // the kernel before this one on the stream (which may produce any input) has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Slot blockIdx.x of the split-unit table is written only by this CTA (if it starts a split unit);
  // clear what an earlier call left there.
  if (tid == 0 && blockIdx.x < kMaxGrid) p.units[blockIdx.x] = make_int4(0, 0, 0, 0);
#ifdef JF_DEBUG
  if (tid == 0 && *reinterpret_cast<volatile int*>(&g_debug_hold) != 0) {
    const uint64_t t0 = globaltimer();
    while (*reinterpret_cast<volatile int*>(&g_debug_hold) != 0) {
      if (globaltimer() - t0 > kWaitLimitNs) {
        set_abort(s, p);
        break;
      }
    }
  }
#endif
  build_plan(s, p);
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  bool idle = s.bad_meta != 0 || s.abort_flag != 0;  // abort_flag: set above by the debug build only
  if (idle && blockIdx.x == 0 && tid == 0) report(p.status, JF_ERR_DEVICE_CHECK);
  const long long W = s.cum_work[p.batch];
  const int G = static_cast<int>(W < static_cast<long long>(gridDim.x) ? W : static_cast<long long>(gridDim.x));
  idle = idle || W <= 0 || static_cast<int>(blockIdx.x) >= G;
  if (idle) {  // uniform over the CTA
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  SegIter iter;
  iter.x = static_cast<long long>(blockIdx.x) * W / G;
  iter.xend = static_cast<long long>(blockIdx.x + 1) * W / G;
  iter.W = W;
  iter.G = G;
  {
    // first sequence touched by this CTA: binary search over cum_work
    int lo = 0, hi = p.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s.cum_work[mid] <= iter.x) lo = mid; else hi = mid - 1;
    }
    iter.b = lo;
  }

  // Register split (the launch gives every thread 168): the copy/MMA/metadata warpgroup runs on 80,
  // which lets the two softmax warpgroups hold a whole 128-column row of S in registers (208).
  // 128 * 80 + 256 * 208 = 63488 <= 384 * 168 = 64512 (the launch's register pool).  With an 8-bit cache
  // the copy warps also convert every tile, which spills at 80: there the split is 104 / 200
  // (128 * 104 + 256 * 200 = 64512).
  if (warp < 4) {
    if (kFp8) asm volatile("setmaxnreg.dec.sync.aligned.u32 104;\n" ::: "memory");
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n" ::: "memory");
    if (warp == 0 || warp == 2) {
      kv_producer<kFp8>(s, p, iter, warp == 2, &tm_q, warp == 2 ? &tm_v : &tm_k);
    } else if (warp == 1) {
      mma_issuer<kFp8>(s, p, iter, tmem);
    } else {
      metadata(s, p, iter);
    }
  } else {
    if (kFp8) asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    else asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n" ::: "memory");
    softmax_epilogue<kFp8>(s, p, iter, tmem, warp < 8 ? 0 : 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// Combine kernel: merges the partials of every unit that was cut between CTAs.  A fixed grid (two
// blocks per SM) first compacts the split units out of the descriptor table (one slot per attention
// CTA) and then takes work items (split unit, M tile, 32-row block) in a grid-stride loop.  A thread
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
    const float inv = p.v_scale / L;  // the V cache's scale (1 for a bf16 cache)
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

cudaError_t launch_tree_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                  const AttnParams& p, int grid, bool fp8_cache, cudaStream_t stream) {
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  const size_t smem = attention_smem_bytes();
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(attn::tree_attention_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn::tree_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  cudaError_t e = fp8_cache ? launch_pdl(attn::tree_attention_kernel<true>, dim3(grid), dim3(attn::kThreads), smem,
                                         stream, nullptr, tm_q, tm_k, tm_v, p)
                            : launch_pdl(attn::tree_attention_kernel<false>, dim3(grid), dim3(attn::kThreads), smem,
                                         stream, nullptr, tm_q, tm_k, tm_v, p);
  if (e != cudaSuccess) return e;
  // The combine kernel may start as soon as the attention grid is scheduled; its griddepcontrol.wait
  // holds it until the attention grid has finished and its writes are visible.
  return launch_pdl(attn::combine_kernel, dim3(2 * grid), dim3(attn::kCombineThreads), 0, stream, nullptr, p, grid);
}

}  // namespace jf

#ifdef JF_DEBUG
extern "C" JF_API jf_status jf_debug_hold(int on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(jf::g_debug_hold, &v, sizeof(v)) == cudaSuccess ? JF_OK : JF_ERR_CUDA;
}
#endif
