// tree_attention.cu -- tree-causal attention over a paged bf16 KV cache on sm_100a.
//
// What it computes ("JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree
// Drafting", technical summary section 2, tree-causal attention mask and branch factorisation): the
// query of every draft-tree node attends to its sequence's whole cached prefix plus the tree slots of
// its own root path (itself included), never to descendants or unrelated branches.
//
// How (B200-specific design, not taken from the pages, which only name an sm_90 paged kernel):
//   * GQA packing: one M tile = 128 rows = (128 / g) tree nodes x g query heads of one kv head, so the
//     K/V of that kv head is staged once for all its query heads.
//   * Per CTA (persistent, one per SM): warp 0 loads Q with TMA (once per segment) and gathers K, warp 2
//     gathers V: 128 keys (8 pages of 16 tokens) per tile, one TMA box per page and 64-column half,
//     128-byte swizzled, gathered through the block table.  A box is only 2 KB, so the 16 boxes of a
//     tile are issued by 16 lanes at once and K and V by separate warps.
//     Warp 1 allocates tensor memory and issues tcgen05.mma: S = Q K^T (both operands from shared
//     memory, K-major) into a double-buffered S in TMEM, and O += P V with P read straight from TMEM
//     (aliasing S) and V as an MN-major shared-memory operand.  Warp 3 validates each segment and
//     builds per-node 256-bit ancestor bitsets by pointer jumping.  Warps 4-7 (one thread per row) run
//     the online softmax out of TMEM with a lazy rescale of O.
//   * The tree mask only touches tiles that hold tree slots; prefix tiles are unmasked.
//   * Work split: the flattened (unit, kv tile) space is cut into equal contiguous ranges, one per CTA
//     (stream-K).  A unit cut between CTAs writes fp32 partials; per row, the last CTA to finish (an
//     atomic counter per row, no spinning) merges them and stores the bf16 output.
#include "jf_device.cuh"
#include "jf_internal.h"

namespace jf {
namespace attn {

constexpr int kPage = 16;
constexpr int kBM = 128;             // rows per M tile
constexpr int kBN = 128;             // keys per KV tile
constexpr int kPagesPerTile = kBN / kPage;
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr int kHalfBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmO = 256;  // S buffers at columns 0 and 128, O at 256
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may grow up to 2^8 before O is rescaled

struct __align__(1024) Smem {
  uint8_t q[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint32_t anc[2][kMaxTreeNodes][kAncWords];
  uint32_t anc_tmp[kMaxTreeNodes][kAncWords];
  int32_t jmp[2][kMaxTreeNodes];
  long long cum_work[kMaxAttnBatch + 1];
  long long scan_warp[kThreads / 32];
  uint64_t bar_qfull, bar_qempty;
  uint64_t bar_kfull[kStages], bar_kempty[kStages], bar_vfull[kStages], bar_vempty[kStages];
  uint64_t bar_sfull[2], bar_pfull[2], bar_pvdone[2];  // pvdone[j & 1] completes when PV(j) is done
  uint64_t bar_metafull[2], bar_metaempty[2];
  uint32_t tmem_base;
  int meta_valid[2];
  int meta_tree[2];
  int meta_ctl;
  int abort_flag;
  int bad_meta;
};

struct Seg {
  int b, kvh, mt, kb, ke;  // kv tiles [kb, ke) of unit (b, kvh, mt)
  int P, N, off, kt;       // prefix length, nodes, first global node, kv tiles of the sequence
  int c0, c1, slot;        // CTAs sharing the unit; this CTA's partial slot
};

__device__ __forceinline__ int cta_of(long long x, long long W, int G) {
  return static_cast<int>(((x + 1) * G - 1) / W);
}

struct SegIter {
  long long x, xend, W;
  int G, b;
  __device__ bool next(const Smem& s, const AttnParams& p, Seg& g) {
    if (x >= xend) return false;
    while (s.cum_work[b + 1] <= x) ++b;
    g.b = b;
    g.P = p.prefix_lens[b];
    g.off = p.tree_offsets[b];
    g.N = p.tree_offsets[b + 1] - g.off;
    g.kt = (g.P + g.N + kBN - 1) / kBN;
    const int mtn = (g.N * p.group + kBM - 1) / kBM;
    const long long local = x - s.cum_work[b];
    const long long unit = local / g.kt;
    g.kb = static_cast<int>(local - unit * g.kt);
    g.kvh = static_cast<int>(unit / mtn);
    g.mt = static_cast<int>(unit - static_cast<long long>(g.kvh) * mtn);
    const long long u0 = s.cum_work[b] + unit * g.kt, u1 = u0 + g.kt;
    const long long e = xend < u1 ? xend : u1;
    g.ke = g.kb + static_cast<int>(e - x);
    g.c0 = cta_of(u0, W, G);
    g.c1 = cta_of(u1 - 1, W, G);
    g.slot = (static_cast<int>(blockIdx.x) == g.c0) ? 2 * blockIdx.x + 1 : 2 * blockIdx.x;
    x = e;
    return true;
  }
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void set_abort(Smem& s, const AttnParams& p) {
  *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
  report(p.status, JF_ERR_TIMEOUT);
}

// ------------------------------------------------------------------------------------------------
// Plan: per-sequence work (kv heads x M tiles x kv tiles), exclusive prefix sum in shared memory,
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
  for (int b = b0; b < b0 + per && b < B; ++b) {
    const int P = p.prefix_lens[b];
    const int N = p.tree_offsets[b + 1] - p.tree_offsets[b];
    if (P < 0 || N < 0 || N > kMaxTreeNodes) {
      bad = 1;
      continue;
    }
    if (N == 0) continue;
    const long long kt = (static_cast<long long>(P) + N + kBN - 1) / kBN;
    const long long mtn = (static_cast<long long>(N) * p.group + kBM - 1) / kBM;
    local += static_cast<long long>(p.hkv) * mtn * kt;
  }
  if (bad) atomicOr(&s.bad_meta, 1);
  // block-wide exclusive scan of `local`
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
    const int P = p.prefix_lens[b];
    const int N = p.tree_offsets[b + 1] - p.tree_offsets[b];
    if (P < 0 || N <= 0 || N > kMaxTreeNodes) continue;
    const long long kt = (static_cast<long long>(P) + N + kBN - 1) / kBN;
    const long long mtn = (static_cast<long long>(N) * p.group + kBM - 1) / kBM;
    run += static_cast<long long>(p.hkv) * mtn * kt;
  }
  if (tid == kThreads - 1) s.cum_work[B] = run;
  __syncthreads();
}

// ------------------------------------------------------------------------------------------------
// Warps 0 and 2: K / V gathers (warp 0 also loads Q)
// ------------------------------------------------------------------------------------------------
__device__ void kv_producer(Smem& s, const AttnParams& p, SegIter iter, bool is_v, const CUtensorMap* tm_q,
                            const CUtensorMap* tm_kv) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  uint64_t* full = is_v ? s.bar_vfull : s.bar_kfull;
  uint64_t* empty = is_v ? s.bar_vempty : s.bar_kempty;
  Seg g;
  uint32_t it = 0, sidx = 0;
  const int nodes_per_tile = kBM / p.group;
  while (iter.next(s, p, g)) {
    if (!is_v) {
      if (!warp_wait(&s.bar_qempty, (sidx & 1) ^ 1, abort)) return set_abort(s, p);
      if (lane == 0) {
        const int node0 = g.off + g.mt * nodes_per_tile;
        mbar_arrive_expect_tx(&s.bar_qfull, kTileBytes);
        tma_load_3d(s.q, tm_q, &s.bar_qfull, 0, g.kvh * p.group, node0);
        tma_load_3d(s.q + kHalfBytes, tm_q, &s.bar_qfull, 64, g.kvh * p.group, node0);
      }
    }
    const int npg = (g.P + g.N + kPage - 1) / kPage;
    const int32_t* bt = p.block_table + static_cast<long long>(g.b) * p.max_pages;
    // Page ids are fetched four tiles at a time (lane l: logical page 8 * (t0 + l / 8) + l % 8, -1 = not
    // loaded) and one batch ahead, so the block-table latency stays off the issue path.
    auto batch_ids = [&](int t0) {
      int pid = -1;
      const int t = t0 + (lane >> 3);
      if (t < g.ke) {
        const int pg = t * kPagesPerTile + (lane & 7);
        if (pg < npg && pg < p.max_pages) {
          const int v = __ldg(bt + pg);
          if (v >= 0 && v < p.num_pages) pid = v;
        }
      }
      return pid;
    };
    int ids_cur = batch_ids(g.kb);
    int ids_next = batch_ids(g.kb + 4);
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int st = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      const int bi = (t - g.kb) & 3;
      if (bi == 0 && t > g.kb) {
        ids_cur = ids_next;
        ids_next = batch_ids(t + 4);
      }
      // lane j < 16: page j / 2, 64-column half j % 2
      int pid = __shfl_sync(0xffffffffu, ids_cur, bi * 8 + ((lane >> 1) & 7));
      if (lane >= 2 * kPagesPerTile) pid = -1;
      const uint32_t mask = __ballot_sync(0xffffffffu, pid >= 0);
      const uint32_t bytes = static_cast<uint32_t>(__popc(mask)) * (kPage * 128u);
      if (!warp_wait(&empty[st], ph ^ 1, abort)) return set_abort(s, p);
      if (lane == 0) mbar_arrive_expect_tx(&full[st], bytes);
      __syncwarp();
      if (pid >= 0) {
        const int half = lane & 1;
        uint8_t* dst = (is_v ? s.v[st] : s.k[st]) + half * kHalfBytes + (lane >> 1) * (kPage * 128);
        tma_load_3d(dst, tm_kv, &full[st], half * 64, g.kvh, pid * kPage);
      }
    }
    ++sidx;
  }
}

// ------------------------------------------------------------------------------------------------
// Warp 1: tcgen05.mma issuer
// ------------------------------------------------------------------------------------------------
struct PendingPV {
  uint32_t it;
  int st, first, zero_from;
};

__device__ __forceinline__ bool issue_pv(Smem& s, const AttnParams& p, uint32_t tmem, const PendingPV& pv) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  const int sb = pv.it & 1;
  if (!warp_wait(&s.bar_pfull[sb], (pv.it >> 1) & 1, abort)) return false;
  if (!warp_wait(&s.bar_vfull[pv.st], (pv.it / kStages) & 1, abort)) return false;
  if (pv.zero_from < kBN) {
    // Keys beyond the sequence's last slot: clear their V rows so stale cache contents (even NaN)
    // cannot reach the output through 0 * V.  A whole 128-byte row is cleared, so the swizzle does
    // not matter.
    uint8_t* vb = s.v[pv.st];
    const int nchunks = (kBN - pv.zero_from) * 16;
    for (int i = lane; i < nchunks; i += 32) {
      const int row = pv.zero_from + (i >> 4);
      const int half = (i >> 3) & 1;
      const int c = i & 7;
      *reinterpret_cast<uint4*>(vb + half * kHalfBytes + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  __syncwarp();
  tc_fence_after();
  if (lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, 128, false, true);
    const uint32_t vaddr = smem_u32(s.v[pv.st]);
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
      const uint64_t bdesc = smem_desc_sw128(vaddr + kk * 2048, kHalfBytes, 1024);
      mma_ts(tmem + kTmO, tmem + sb * 128 + kk * 8, bdesc, idesc, (pv.first && kk == 0) ? 0u : 1u);
    }
    mma_commit(&s.bar_pvdone[pv.it & 1]);
    mma_commit(&s.bar_vempty[pv.st]);
  }
  __syncwarp();
  return true;
}

__device__ void mma_issuer(Smem& s, const AttnParams& p, SegIter iter, uint32_t tmem) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  Seg g;
  uint32_t it = 0, sidx = 0;
  bool have_prev = false;
  PendingPV prev{};
  constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
  const uint32_t qaddr = smem_u32(s.q);
  while (iter.next(s, p, g)) {
    if (!warp_wait(&s.bar_qfull, sidx & 1, abort)) return set_abort(s, p);
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int st = it % kStages;
      const int sb = it & 1;
      if (!warp_wait(&s.bar_kfull[st], (it / kStages) & 1, abort)) return set_abort(s, p);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t kaddr = smem_u32(s.k[st]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(qaddr + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(kaddr + off, 16, 1024);
          mma_ss(tmem + sb * 128, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s.bar_sfull[sb]);
        mma_commit(&s.bar_kempty[st]);
        if (t == g.ke - 1) mma_commit(&s.bar_qempty);
      }
      __syncwarp();
      if (have_prev && !issue_pv(s, p, tmem, prev)) return set_abort(s, p);
      const int zf = g.P + g.N - t * kBN;  // first row of this tile past the sequence
      prev.it = it;
      prev.st = st;
      prev.first = (t == g.kb);
      prev.zero_from = zf < 0 ? 0 : zf;
      have_prev = true;
    }
    ++sidx;
  }
  if (have_prev && !issue_pv(s, p, tmem, prev)) return set_abort(s, p);
}

// ------------------------------------------------------------------------------------------------
// Warp 3: per-segment validation and ancestor bitsets (pointer jumping over parent[])
// ------------------------------------------------------------------------------------------------
__device__ void metadata(Smem& s, const AttnParams& p, SegIter iter) {
  const int mt = threadIdx.x & 31;
  volatile int* abort = &s.abort_flag;
  Seg g;
  uint32_t sidx = 0;
  while (iter.next(s, p, g)) {
    const int buf = sidx & 1;
    if (mt == 0) {
      const bool ok = mbar_wait(&s.bar_metaempty[buf], ((sidx >> 1) & 1) ^ 1, abort);
      s.meta_ctl = ok ? 1 : 0;
      if (!ok) set_abort(s, p);
    }
    __syncwarp();
    if (s.meta_ctl == 0) return;
    // --- validation
    int bad = 0;
    const int npg = (g.P + g.N + kPage - 1) / kPage;
    if (static_cast<long long>(g.P) + g.N > static_cast<long long>(p.max_pages) * kPage) bad = 1;
    const int32_t* par = p.parent + g.off;
    for (int i = mt; i < g.N; i += 32) {
      const int pi = par[i];
      if (pi < -1 || pi >= i) bad = 1;
    }
    const int32_t* bt = p.block_table + static_cast<long long>(g.b) * p.max_pages;
    const int pg0 = g.kb * kPagesPerTile;
    int pg1 = g.ke * kPagesPerTile;
    if (pg1 > npg) pg1 = npg;
    if (pg1 > p.max_pages) pg1 = p.max_pages;
    for (int pg = pg0 + mt; pg < pg1; pg += 32) {
      const int v = bt[pg];
      if (v < 0 || v >= p.num_pages) bad = 1;
    }
    if (mt == 0) s.meta_valid[buf] = 1;
    __syncwarp();
    if (bad) {
      s.meta_valid[buf] = 0;
      report(p.status, JF_ERR_DEVICE_CHECK);
    }
    // --- ancestor bitsets, only if the segment reaches the tree slots
    const bool tree = static_cast<long long>(g.ke) * kBN > g.P;
    if (tree) {
      uint32_t(*A)[kAncWords] = s.anc[buf];
      for (int i = mt; i < g.N; i += 32) {
        const int pi = par[i];
        s.jmp[0][i] = (pi >= 0 && pi < i) ? pi : -1;
#pragma unroll
        for (int w = 0; w < kAncWords; ++w) A[i][w] = (w == (i >> 5)) ? (1u << (i & 31)) : 0u;
      }
      __syncwarp();
      // After round r every node holds its ancestors at distance < 2^r; 8 rounds cover 256 levels.
      uint32_t(*src)[kAncWords] = s.anc[buf];
      uint32_t(*dst)[kAncWords] = s.anc_tmp;
      int cur = 0;
      for (int round = 0; round < 8; ++round) {
        for (int i = mt; i < g.N; i += 32) {
          const int j = s.jmp[cur][i];
          uint4 a0 = *reinterpret_cast<const uint4*>(&src[i][0]);
          uint4 a1 = *reinterpret_cast<const uint4*>(&src[i][4]);
          int jj = -1;
          if (j >= 0) {
            const uint4 b0 = *reinterpret_cast<const uint4*>(&src[j][0]);
            const uint4 b1 = *reinterpret_cast<const uint4*>(&src[j][4]);
            a0.x |= b0.x; a0.y |= b0.y; a0.z |= b0.z; a0.w |= b0.w;
            a1.x |= b1.x; a1.y |= b1.y; a1.z |= b1.z; a1.w |= b1.w;
            jj = s.jmp[cur][j];
          }
          *reinterpret_cast<uint4*>(&dst[i][0]) = a0;
          *reinterpret_cast<uint4*>(&dst[i][4]) = a1;
          s.jmp[cur ^ 1][i] = jj;
        }
        __syncwarp();
        uint32_t(*t)[kAncWords] = src;
        src = dst;
        dst = t;
        cur ^= 1;
      }
      // 8 rounds (even): the result is back in s.anc[buf]
    }
    if (mt == 0) s.meta_tree[buf] = tree ? 1 : 0;
    __threadfence_block();
    mbar_arrive(&s.bar_metafull[buf]);
    ++sidx;
  }
}

// ------------------------------------------------------------------------------------------------
// Warps 4-7: online softmax (one thread per row) and the epilogue
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
// float4 index ((slot * 32 + c4) * 128 + row).
__device__ __forceinline__ float4* part_ptr(const AttnParams& p, int slot, int c4, int r) {
  return reinterpret_cast<float4*>(p.part_o) + (static_cast<long long>(slot) * 32 + c4) * kBM + r;
}

__device__ void softmax_epilogue(Smem& s, const AttnParams& p, SegIter iter, uint32_t tmem) {
  const int r = threadIdx.x - 128;  // row of the M tile == TMEM lane
  const int wq = (threadIdx.x >> 5) & 3;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  volatile int* abort = &s.abort_flag;
  const float sl2 = p.scale_log2;
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const int nodes_per_tile = kBM / p.group;
  Seg g;
  uint32_t it = 0, sidx = 0;
  while (iter.next(s, p, g)) {
    const int buf = sidx & 1;
    const int node = g.mt * nodes_per_tile + r / p.group;
    const int head = g.kvh * p.group + (r % p.group);
    const bool row_valid = node < g.N;
    const uint32_t* anc = &s.anc[buf][row_valid ? node : 0][0];
    float m_use = -INFINITY, l = 0.f;
    bool meta_seen = false;
    for (int t = g.kb; t < g.ke; ++t, ++it) {
      const int sb = it & 1;
      const bool tree_tile = (t + 1) * kBN > g.P;
      if (tree_tile && !meta_seen) {
        if (!warp_wait(&s.bar_metafull[buf], (sidx >> 1) & 1, abort)) return set_abort(s, p);
        meta_seen = true;
      }
      if (!warp_wait(&s.bar_sfull[sb], (it >> 1) & 1, abort)) return set_abort(s, p);
      // S(it) ready implies PV(it-2) is complete (the tensor pipe runs in issue order); observing that
      // phase keeps pvdone[it & 1] in step so later waits on it are unambiguous.
      if (it >= 2 && !warp_wait(&s.bar_pvdone[sb], ((it - 2) >> 1) & 1, abort)) return set_abort(s, p);
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(lane_base + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(lane_base + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(lane_base + sb * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(lane_base + sb * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_ld_wait();
      if (tree_tile) {
        // invisible keys become -inf: they drop out of the max and get P = 2^-inf = 0
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t vw = vis_word(t * kBN + 32 * w, g.P, g.N, row_valid, anc);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (!((vw >> i) & 1u)) sr[32 * w + i] = 0xff800000u;
        }
      }
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        a0 = fmax3(a0, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
        a1 = fmax3(a1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
        a2 = fmax3(a2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
        a3 = fmax3(a3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
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
      uint64_t acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const uint64_t y = f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, nm2);
        float y0, y1;
        f2_unpack(y, y0, y1);
        const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
        const uint64_t pp = f2_pack(p0, p1);
        switch ((c >> 1) & 3) {
          case 0: acc0 = f2_add(acc0, pp); break;
          case 1: acc1 = f2_add(acc1, pp); break;
          case 2: acc2 = f2_add(acc2, pp); break;
          default: acc3 = f2_add(acc3, pp); break;
        }
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      {
        const uint64_t t2 = f2_add(f2_add(acc0, acc1), f2_add(acc2, acc3));
        float u0, u1;
        f2_unpack(t2, u0, u1);
        l += u0 + u1;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O must hold PV(it-1) before it is rescaled
        if (!warp_wait(&s.bar_pvdone[(it - 1) & 1], ((it - 1) >> 1) & 1, abort)) return set_abort(s, p);
        tc_fence_after();
        const float a = resc ? alpha : 1.f;
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
      tmem_st32(lane_base + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st32(lane_base + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.bar_pfull[sb]);
    }
    // ---------------- epilogue of the segment
    if (!meta_seen) {
      if (!warp_wait(&s.bar_metafull[buf], (sidx >> 1) & 1, abort)) return set_abort(s, p);
    }
    const bool seg_ok = s.meta_valid[buf] != 0;
    {
      const uint32_t last = it - 1;
      if (!warp_wait(&s.bar_pvdone[last & 1], (last >> 1) & 1, abort)) return set_abort(s, p);
    }
    tc_fence_after();
    mbar_arrive(&s.bar_metaempty[buf]);
    const bool split = g.c0 != g.c1;
    const long long grow = static_cast<long long>(g.off + node) * p.hq + head;  // global row
    if (!split) {
      const float inv_l = 1.f / l;
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + kTmO + cc, o);
        tmem_ld_wait();
        if (seg_ok && row_valid)
          store_row_bf16(p.out + grow * 128 + cc, reinterpret_cast<const float*>(o), inv_l);
      }
      if (seg_ok && row_valid && p.lse != nullptr) p.lse[grow] = (m_use + __log2f(l)) * 0.69314718055994531f;
    } else {
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + kTmO + cc, o);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          __stcg(part_ptr(p, g.slot, (cc + c) >> 2, r),
                 make_float4(__uint_as_float(o[c]), __uint_as_float(o[c + 1]), __uint_as_float(o[c + 2]),
                             __uint_as_float(o[c + 3])));
      }
      __stcg(&p.part_ml[static_cast<long long>(g.slot) * kBM + r], make_float2(m_use, l));
      __stcg(&p.part_ok[static_cast<long long>(g.slot) * kBM + r], seg_ok ? 1 : 0);
      __threadfence();
      int* ctr = p.counters + static_cast<long long>(g.c0) * kBM + r;
      const int prev = atomicAdd(ctr, 1);
      if (prev == g.c1 - g.c0) {
        // last contributor for this row: merge every CTA's partial; loads are issued four segments and
        // 32 columns at a time so each batch is one memory round trip
        __threadfence();
        constexpr int kGrp = 4;
        float M = -INFINITY, L = 0.f;
        bool all_ok = true;
        for (int cb = g.c0; cb <= g.c1; cb += kGrp) {
          float2 ml[kGrp];
          int ok[kGrp];
#pragma unroll
          for (int u = 0; u < kGrp; ++u) {
            const int c = cb + u;
            const int sl = (c == g.c0) ? 2 * c + 1 : 2 * c;
            ml[u] = c <= g.c1 ? __ldcg(&p.part_ml[static_cast<long long>(sl) * kBM + r]) : make_float2(-INFINITY, 0.f);
            ok[u] = c <= g.c1 ? __ldcg(&p.part_ok[static_cast<long long>(sl) * kBM + r]) : 1;
          }
#pragma unroll
          for (int u = 0; u < kGrp; ++u) {
            M = fmaxf(M, ml[u].x);
            all_ok = all_ok && ok[u] != 0;
          }
        }
        for (int cb = g.c0; cb <= g.c1; cb += kGrp) {
#pragma unroll
          for (int u = 0; u < kGrp; ++u) {
            const int c = cb + u;
            const int sl = (c == g.c0) ? 2 * c + 1 : 2 * c;
            if (c <= g.c1) {
              const float2 ml = __ldcg(&p.part_ml[static_cast<long long>(sl) * kBM + r]);
              if (ml.x != -INFINITY) L += ml.y * ex2_approx(ml.x - M);
            }
          }
        }
        const float inv_L = 1.f / L;
        for (int cc = 0; cc < 128; cc += 32) {
          float acc[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) acc[c] = 0.f;
          for (int cb = g.c0; cb <= g.c1; cb += kGrp) {
            float4 v[kGrp][8];
            float w[kGrp];
#pragma unroll
            for (int u = 0; u < kGrp; ++u) {
              const int c = cb + u;
              const int sl = (c == g.c0) ? 2 * c + 1 : 2 * c;
              const bool have = c <= g.c1;
              const float2 ml = have ? __ldcg(&p.part_ml[static_cast<long long>(sl) * kBM + r])
                                     : make_float2(-INFINITY, 0.f);
              w[u] = (ml.x == -INFINITY) ? 0.f : ex2_approx(ml.x - M);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                v[u][q] = have ? __ldcg(part_ptr(p, sl, (cc >> 2) + q, r)) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kGrp; ++u) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                acc[4 * q + 0] = fmaf(w[u], v[u][q].x, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(w[u], v[u][q].y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(w[u], v[u][q].z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(w[u], v[u][q].w, acc[4 * q + 3]);
              }
            }
          }
          if (all_ok && row_valid) store_row_bf16(p.out + grow * 128 + cc, acc, inv_L);
        }
        if (all_ok && row_valid && p.lse != nullptr) p.lse[grow] = (M + __log2f(L)) * 0.69314718055994531f;
        *ctr = 0;  // leave the workspace zeroed for the next call
      }
    }
    ++sidx;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;

  build_plan(s, p);
  if (s.bad_meta) {
    if (blockIdx.x == 0 && tid == 0) report(p.status, JF_ERR_DEVICE_CHECK);
    return;
  }
  const long long W = s.cum_work[p.batch];
  if (W <= 0) return;
  const int G = static_cast<int>(W < static_cast<long long>(gridDim.x) ? W : static_cast<long long>(gridDim.x));
  if (static_cast<int>(blockIdx.x) >= G) return;
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

  if (tid == 0) {
    mbar_init(&s.bar_qfull, 1);
    mbar_init(&s.bar_qempty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.bar_kfull[i], 1);
      mbar_init(&s.bar_kempty[i], 1);
      mbar_init(&s.bar_vfull[i], 1);
      mbar_init(&s.bar_vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_sfull[i], 1);
      mbar_init(&s.bar_pfull[i], 128);
      mbar_init(&s.bar_metafull[i], 32);
      mbar_init(&s.bar_metaempty[i], 128);
      mbar_init(&s.bar_pvdone[i], 1);
    }
    s.abort_flag = 0;
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
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0 || warp == 2) {
    kv_producer(s, p, iter, warp == 2, &tm_q, warp == 2 ? &tm_v : &tm_k);
  } else if (warp == 1) {
    mma_issuer(s, p, iter, tmem);
  } else if (warp == 3) {
    metadata(s, p, iter);
  } else {
    softmax_epilogue(s, p, iter, tmem);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn

size_t attention_smem_bytes() { return sizeof(attn::Smem) + 1024; }

cudaError_t launch_tree_attention(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                  const AttnParams& p, int grid, cudaStream_t stream) {
  static bool attr_set = false;
  const size_t smem = attention_smem_bytes();
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn::tree_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  attn::tree_attention_kernel<<<grid, attn::kThreads, smem, stream>>>(tm_q, tm_k, tm_v, p);
  return cudaGetLastError();
}

}  // namespace jf
