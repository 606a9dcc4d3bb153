/*
 * jf.h -- C ABI of libjf.so: the tree-verify hot path of causal parallel tree drafting
 * (JetFlow / JetSpec) on NVIDIA B200 (sm_100a).
 *
 * Sources (page titles; the pages print no code and define no API):
 *   [JF] "JetFlow: Breaking the Scaling Ceiling of Speculative Decoding with Parallel Tree Drafting",
 *        technical summary: section 1 (verification and acceptance), section 2 (tree-causal attention
 *        mask, branch factorisation, best-first tree construction to a budget), section 3 (paged
 *        attention inside a serving engine), section 4 (budgets 16..256, tau accepted tokens).
 *   [JS] "JetSpec" paper page, abstract.
 *
 * Conventions shared by every call
 *   - Every array argument is DEVICE memory owned by the caller; the library never allocates,
 *     frees or retains a pointer after the call returns.  Scratch space is passed in as
 *     `workspace`, sized by the matching *_workspace_size() query.
 *   - Calls are asynchronous and stream-ordered on `stream` (0 = legacy default stream).  No call
 *     synchronises the host.  Calls on different streams may run concurrently as long as they use
 *     different workspaces and outputs.
 *   - Problems that the host can see (null pointers, unsupported shapes, short workspace,
 *     misaligned pointers) return an error code synchronously and launch nothing.
 *   - Problems that depend on device data (a parent index out of range, a page id out of range,
 *     a sequence longer than its block table, malformed tree_offsets) are detected on the device:
 *     the first such code is written with atomicCAS into `*dev_status` (an int32 the caller zeroes
 *     before the call), and the outputs of the offending sequence are left unwritten.  The device
 *     never traps.  `dev_status` may be NULL, in which case device-detected problems are silent.
 *   - Every device-side wait is bounded; if one runs out (it never should) the kernel writes
 *     JF_ERR_TIMEOUT to `*dev_status` and returns.
 *   - bf16 arrays are passed as `const void*`: IEEE-754 bfloat16, 2 bytes per element.
 */
#ifndef JF_H_
#define JF_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JF_API __attribute__((visibility("default")))
#else
#define JF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* jf_stream_t; /* identical to cudaStream_t */

typedef enum {
  JF_OK = 0,
  JF_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned pointer, short workspace */
  JF_ERR_UNSUPPORTED = 2,  /* head_dim != 128, page_size != 16, bad GQA ratio, sizes above limits */
  JF_ERR_CUDA = 3,         /* a CUDA runtime / driver call failed (launch, attribute, tensor map) */
  JF_ERR_DEVICE_CHECK = 4, /* device-side data check failed (written to *dev_status only) */
  JF_ERR_TIMEOUT = 5       /* a bounded device-side wait ran out (written to *dev_status only) */
} jf_status;

/* Human-readable name of a status code.  Never NULL. */
JF_API const char* jf_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
JF_API int jf_version(void);

/* ------------------------------------------------------------------------------------------
 * jf_tree_attention -- tree-causal attention of every draft-tree node over the paged KV cache.
 *
 * Defines [JF section 2, "tree-causal attention mask"; branch factorisation
 * q(pi(v)|x) = prod_{u in pi(v)} q(y_u | x, h_x, pi_<u)]: the query of tree node n of sequence b
 * attends to all prefix_lens[b] cached prefix tokens and to the tree slots of its own ancestors
 * and itself, never to descendants or unrelated siblings.  For q head h (kv head h / (Hq/Hkv)):
 *     s_t  = sm_scale * <q[n,h,:], K[t]>               for visible logical slots t
 *     out  = sum_t softmax(s)_t V[t]                    (bf16, round-to-nearest-even)
 *     lse  = ln sum_t exp(s_t)                          (fp32, optional)
 * Visible slots of node n (local index within its sequence): t in [0, P) and t = P + j for every
 * j on n's root path (j = n, parent[n], parent[parent[n]], ... until -1).
 *
 * Layouts (row-major, innermost last):
 *   q            bf16  [total_nodes, num_q_heads, head_dim]; sequence b owns rows
 *                      [tree_offsets[b], tree_offsets[b+1])
 *   k_cache,
 *   v_cache      bf16  [num_pages, page_size, num_kv_heads, head_dim]
 *   block_table  int32 [batch, max_pages_per_seq]: logical page p of sequence b is physical page
 *                      block_table[b*max_pages_per_seq + p]; logical slot t is row t % page_size of
 *                      logical page t / page_size.  The tree nodes' K/V must already sit at logical
 *                      slots prefix_lens[b] .. prefix_lens[b] + N_b - 1 (node order).
 *   prefix_lens  int32 [batch], >= 0
 *   tree_offsets int32 [batch+1], tree_offsets[0] = 0, non-decreasing, tree_offsets[batch] =
 *                      total_nodes; N_b = tree_offsets[b+1] - tree_offsets[b] <= 256
 *   parent       int32 [total_nodes], local index of the parent within the sequence, in
 *                      [-1, i-1] for node i (-1 = child of the cached prefix)
 *   out          bf16  [total_nodes, num_q_heads, head_dim]
 *   lse          fp32  [total_nodes, num_q_heads] or NULL
 * Supported: head_dim == 128, page_size == 16, num_q_heads % num_kv_heads == 0 with
 * Hq/Hkv in {1, 2, 4, 8, 16}, batch <= 1024.  q, k_cache, v_cache and out must be 16-byte aligned.
 * Cache slots beyond prefix_lens[b] + N_b in the last used page are never part of the result.
 *
 * workspace: at least jf_tree_attention_workspace_size(...) bytes of device memory, 256-byte
 * aligned; it needs no initialisation and can be reused by consecutive calls on one stream.  A call
 * launches the attention kernel and, right behind it on the same stream, a kernel that merges the
 * partial results of work units the attention kernel split between CTAs.
 * ------------------------------------------------------------------------------------------ */
JF_API size_t jf_tree_attention_workspace_size(int batch, int num_q_heads, int num_kv_heads, int total_nodes);

JF_API jf_status jf_tree_attention(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_table, int max_pages_per_seq,
                            const int32_t* prefix_lens, const int32_t* tree_offsets,
                            const int32_t* parent, int batch, int total_nodes, int num_q_heads,
                            int num_kv_heads, int head_dim, int page_size, int num_pages,
                            float sm_scale, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_tree_attention_fp8 -- jf_tree_attention over a paged KV cache stored in 8 bits (E4M3).
 *
 * The attention of jf_tree_attention [JF section 2 tree-causal mask; section 3 paged attention in the
 * serving engine] over the decoded cache: a stored code c stands for decode(c) * k_scale in k_cache
 * and decode(c) * v_scale in v_cache, where decode is the E4M3 format (1 sign, 4 exponent bits with
 * bias 7, 3 mantissa bits, no infinities; S.1111.111 is NaN; largest magnitude 448).  The pages do not
 * describe 8-bit caches; this is the serving variant for heavy load, where the cache's bytes dominate.
 * The result is the bf16 path's definition applied to the decoded values: the kernel computes on the
 * exact decoded values (every E4M3 value is exact in f16) with q converted to f16, applies k_scale in
 * the softmax scale and v_scale in the final normalisation; tolerances as for jf_tree_attention.
 *
 * Layouts: as jf_tree_attention except k_cache, v_cache: uint8 E4M3 codes [num_pages, page_size,
 * num_kv_heads, head_dim], 16-byte aligned.  k_scale, v_scale: finite and > 0.  q stays bf16
 * (values beyond the f16 range, |q| > 65504, are not supported).  Same workspace, limits, device
 * checks and errors as jf_tree_attention.
 * ------------------------------------------------------------------------------------------ */
JF_API jf_status jf_tree_attention_fp8(const void* q, const void* k_cache, const void* v_cache, float k_scale,
                                       float v_scale, const int32_t* block_table, int max_pages_per_seq,
                                       const int32_t* prefix_lens, const int32_t* tree_offsets,
                                       const int32_t* parent, int batch, int total_nodes, int num_q_heads,
                                       int num_kv_heads, int head_dim, int page_size, int num_pages,
                                       float sm_scale, void* out, float* lse, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_build_tree -- best-first draft-tree construction under a token budget.
 *
 * Defines [JF section 2, "tree construction": the head emits logits for all depths in parallel; the
 * branch score is the cumulative draft log-probability; best-first expansion up to a budget such
 * as 256].  Reading of the per-depth input: row d-1 of draft_logits scores every child at depth d,
 * so all depth-(d-1) nodes share the same top-k children.  Steps:
 *   1. per (b, d): lse_d = m + ln sum_v exp(x_v - m) with m = max_v x_v (float64 accumulation and
 *      float64 exp), the top-k tokens by (logit descending, token id ascending), and
 *      lp[d][r] = x_tok - lse_d in float64;
 *   2. node 0 = root_tokens[b], parent -1, depth 0, score 0; the budget counts the root;
 *   3. candidates (p, r) with key score(p) + lp[depth(p)+1][r] are popped best-first by
 *      (key descending, depth ascending, parent index ascending, rank ascending); the popped
 *      candidate becomes the next node (parent p, token = r-th top token of its depth, score = key
 *      rounded to fp32); its sibling (p, r+1) and its first child (i, 0) (if depth < max_depth) join
 *      the queue; repeat until `budget` nodes exist.
 * The output order is pop order, so parent[i] < i.
 *
 * Layouts: draft_logits fp32 [batch, depths, vocab]; root_tokens int32 [batch];
 *          parent, token int32 [batch, budget]; score fp32 [batch, budget]; depth int32
 *          [batch, budget] or NULL.
 * Limits: 1 <= topk <= 8, topk <= vocab, 1 <= max_depth <= depths <= 64, 1 <= budget <= 1024 and
 *         budget <= 1 + sum_{d=1..max_depth} topk^d, vocab < 2^31.
 * workspace: jf_build_tree_workspace_size(...) bytes (no zero-fill needed).
 * ------------------------------------------------------------------------------------------ */
JF_API size_t jf_build_tree_workspace_size(int batch, int depths, int vocab, int topk);

JF_API jf_status jf_build_tree(const float* draft_logits, const int32_t* root_tokens, int batch, int depths,
                        int vocab, int topk, int budget, int max_depth, int32_t* parent,
                        int32_t* token, float* score, int32_t* depth, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_build_tree_noalloc -- jf_build_tree for callers that cannot allocate device memory.
 *
 * The pages describe no such call; it exists for hosts of this library that must not allocate at
 * call time: for example a serving engine that hands all spare device memory to its KV-cache pool
 * at start-up, or a plugin framework whose per-call hook is not allowed to allocate.  Such callers
 * cannot provide jf_build_tree's workspace.  This variant takes no workspace: its scratch is a fixed
 * 1 MiB array of device memory inside libjf.so, which every GPU that loads the library keeps until
 * the process exits.
 *
 * Limit: batch * depths * ceil(vocab / 4096) * 80 bytes must fit in 1 MiB (for example batch 16 with
 * 16 depths of a 151936-token vocabulary); larger calls return JF_ERR_UNSUPPORTED and launch nothing.
 * The first call on each device looks up the array's device address with that device current
 * (cudaGetSymbolAddress); make that first call before any stream capture.  Every call uses the same
 * array and leaves its contents behind; nothing in it needs zeroing between calls, but two calls
 * whose kernels overlap on the GPU (for example on two streams) corrupt each other's results, so
 * such calls must be serialized.  All other arguments, outputs and errors are those of
 * jf_build_tree.
 * ------------------------------------------------------------------------------------------ */
JF_API jf_status jf_build_tree_noalloc(const float* draft_logits, const int32_t* root_tokens, int batch,
                                       int depths, int vocab, int topk, int budget, int max_depth,
                                       int32_t* parent, int32_t* token, float* score, int32_t* depth,
                                       int32_t* dev_status, jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_expand_frontier -- one round of best-first tree construction from per-node draft logits.
 *
 * Defines [JF section 2: the draft head conditions every node on its own root path, the branch
 * factorisation q(pi(v)|x) = prod_{u in pi(v)} q(y_u | x, h, pi_<u); the tree is built best-first by
 * cumulative draft log-probability up to a budget].  With path-conditioned logits a node's children can
 * be scored only after the draft head has run on that node, so the tree grows in rounds; each call is
 * one round.  At entry, sequence b's tree holds num_nodes[b] nodes and its frontier is the nodes
 * [frontier_begin[b], num_nodes[b]); row j of node_logits[b] is the draft head's next-token logits at
 * frontier node frontier_begin[b] + j.  num_nodes[b] == 0 starts a new tree: node 0 = root_tokens[b]
 * (parent -1, depth 0, score 0) is created and is the whole frontier, scored by row 0.  Steps:
 *   1. every frontier node u below max_depth gets its candidate children: the top-k tokens of its
 *      row by (logit descending, token id ascending), with lp = x_tok - lse (float64 lse and exp,
 *      as jf_build_tree);
 *   2. among the untaken candidates (u, r) of every node scored so far, keyed key(u) + lp_u[r] in
 *      float64, the best min(width, budget - num_nodes[b]) by (key descending, depth ascending,
 *      parent index ascending, rank ascending) are appended in that order (score = key rounded to
 *      fp32);
 *   3. frontier_begin[b] = the old num_nodes[b]; num_nodes[b] grows by the nodes appended (fewer
 *      than width only at the budget or when no candidate is left), which form the next frontier.
 * With width 1 the rounds reproduce jf_build_tree's pop order when every node's row is its depth's
 * row.  Rows past a sequence's frontier are never read; a sequence whose tree already holds `budget`
 * nodes is left as it is and none of its rows is read.
 *
 * Layouts: node_logits fp32 [batch, frontier_rows, vocab]; root_tokens int32 [batch];
 *          parent, token, depth int32 [batch, budget] and score fp32 [batch, budget], in/out (the
 *          tree so far; entries past num_nodes[b] are unspecified); num_nodes, frontier_begin int32
 *          [batch], in/out.
 * state: jf_expand_frontier_state_size(batch, budget, topk) bytes, caller-owned, carried between
 *        the rounds of one tree (each node's float64 key and its candidates); it needs no
 *        initialisation before a tree's first round and must not be modified between rounds.
 * workspace: jf_expand_frontier_workspace_size(batch, frontier_rows, vocab) bytes, reusable.
 * Limits: 1 <= topk <= 8, topk <= vocab, 1 <= budget <= 256, 1 <= max_depth, 1 <= width,
 *         1 <= frontier_rows <= 256, batch * frontier_rows <= 65535.
 * Device checks (JF_ERR_DEVICE_CHECK, sequence left unchanged): num_nodes[b] outside [0, budget],
 * frontier_begin[b] outside [0, num_nodes[b]], or a frontier longer than frontier_rows.
 * ------------------------------------------------------------------------------------------ */
JF_API size_t jf_expand_frontier_state_size(int batch, int budget, int topk);

JF_API size_t jf_expand_frontier_workspace_size(int batch, int frontier_rows, int vocab);

JF_API jf_status jf_expand_frontier(const float* node_logits, const int32_t* root_tokens, int batch,
                                    int frontier_rows, int vocab, int topk, int budget, int max_depth,
                                    int width, int32_t* parent, int32_t* token, float* score,
                                    int32_t* depth, int32_t* num_nodes, int32_t* frontier_begin,
                                    void* state, size_t state_bytes, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_accept -- greedy acceptance walk over the verified tree.
 *
 * Defines [JF section 1: the target verifies the drafted tokens in parallel and keeps the longest
 * agreeing prefix; section 4: tau accepted tokens]: cur = 0 (root), L = 0; loop:
 * a = argmax_v target_logits[b, cur, v] (lowest id on ties); stop if L == max_depth; otherwise look
 * for a child c of cur (parent[c] == cur) with token[c] == a (lowest c if several); if found,
 * L += 1, path[L] = c, cur = c, repeat; else stop.  bonus_token = a from the last iteration.
 *
 * Layouts: token, parent int32 [batch, num_nodes] (node 0 is the root, parent[0] = -1,
 *          parent[i] in [-1, i-1]); target_logits fp32 [batch, num_nodes, vocab], row i = the
 *          target's next-token logits after node i; accepted_len int32 [batch] (root excluded,
 *          0..max_depth); path int32 [batch, max_depth+1] (path[0] = 0, unused entries -1);
 *          bonus_token int32 [batch].
 * Limits: 1 <= num_nodes <= 1024, 0 <= max_depth <= 1023, 1 <= vocab < 2^31.  target_logits must
 *         be 16-byte aligned; NaN logits give an unspecified (but in-range) argmax.
 * ------------------------------------------------------------------------------------------ */
JF_API jf_status jf_accept(const int32_t* token, const int32_t* parent, const float* target_logits,
                    int batch, int num_nodes, int vocab, int max_depth, int32_t* accepted_len,
                    int32_t* path, int32_t* bonus_token, int32_t* dev_status, jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_commit_kv -- commit the accepted path's K/V into the paged cache, in place.
 *
 * The pages run the method inside a paged-KV serving engine [JF section 3] and keep the longest
 * agreeing prefix of the verified tree [JF section 1]; they leave the cache update itself open.
 * Reading used: during verification tree node j of sequence b sits at cache slot P + j, with
 * P = prefix_lens[b] (where jf_tree_attention reads it).  After jf_accept returned path[b] =
 * [0, n_1, .., n_L] with L = accepted_len[b], slot P + i (i = 1 .. L) receives the K and V of slot
 * P + n_i (every kv head, all head_dim values), slot P (the root) keeps its own, and
 * new_prefix_lens[b] = P + L + 1.  Slots from P + L + 1 on are left with unspecified contents.  A
 * sequence whose tree is empty (tree_offsets[b+1] == tree_offsets[b]) is untouched and keeps P.
 * Slot s of sequence b is offset s % 16 of page block_table[b, s / 16].
 *
 * Layouts: k_cache, v_cache bf16 [num_pages, page_size, num_kv_heads, head_dim], modified in place;
 *          block_table int32 [batch, max_pages_per_seq]; prefix_lens int32 [batch]; tree_offsets
 *          int32 [batch+1]; path int32 [batch, max_depth+1] and accepted_len int32 [batch] as
 *          jf_accept writes them; new_prefix_lens int32 [batch] (it may be prefix_lens itself).
 * Limits: head_dim == 128, page_size == 16, 1 <= num_kv_heads <= 64, 0 <= max_depth <= 1023,
 *         num_pages * 16 < 2^31; k_cache and v_cache 16-byte aligned.
 * Device checks (dev_status = JF_ERR_DEVICE_CHECK; that sequence is left untouched and keeps P):
 *         accepted_len outside [0, min(max_depth, nodes - 1)], path[0] != 0, a path that does not
 *         strictly increase or leaves the tree, slots P .. P + nodes - 1 past max_pages_per_seq * 16,
 *         or one of their page ids outside [0, num_pages).
 * Ownership: every pointer is caller-owned device memory; nothing is allocated.  Stream-ordered and
 *         graph-capturable, like the other calls.
 * ------------------------------------------------------------------------------------------ */
JF_API jf_status jf_commit_kv(void* k_cache, void* v_cache, const int32_t* block_table, int max_pages_per_seq,
                       const int32_t* prefix_lens, const int32_t* tree_offsets, const int32_t* path,
                       const int32_t* accepted_len, int batch, int max_depth, int num_kv_heads, int head_dim,
                       int page_size, int num_pages, int32_t* new_prefix_lens, int32_t* dev_status,
                       jf_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * jf_tree_kv_append -- write the tree tokens' K/V into the paged cache with rotary positions.
 *
 * The target verifies the whole tree in one forward pass [JF section 1] inside a paged-KV serving
 * engine [JF section 3]; the pages leave the cache write and the positions open.  Readings used:
 * node j of sequence b (flattened index t = tree_offsets[b] + j) goes to cache slot P + j with
 * P = prefix_lens[b] (where jf_tree_attention reads it); its position is P + depth[t], the root at
 * depth 0; the rotary embedding turns each pair of head elements (i, i + 64), i < 64, by the angle
 * pos * rope_theta^(-2i/128), computed in float64 and rounded once to bf16; V is stored unrotated; q,
 * when not NULL, is rotated in place with the same positions.
 *
 * Layouts: k_new, v_new bf16 [total_nodes, num_kv_heads, head_dim]; q bf16 [total_nodes,
 *          num_q_heads, head_dim] or NULL; k_cache, v_cache bf16 [num_pages, page_size,
 *          num_kv_heads, head_dim]; block_table int32 [batch, max_pages_per_seq]; prefix_lens int32
 *          [batch]; tree_offsets int32 [batch+1]; depth int32 [total_nodes] (jf_build_tree's depth
 *          output, flattened).
 * Limits: head_dim == 128, page_size == 16, 1 <= batch <= 1024, rope_theta > 0 and finite,
 *         num_pages * 16 < 2^31; k_new, v_new, q, k_cache, v_cache 16-byte aligned.
 * Device checks (dev_status = JF_ERR_DEVICE_CHECK; the node is skipped): tree_offsets not starting
 *         at 0, not ending at total_nodes or decreasing; a negative prefix or depth; a slot past
 *         max_pages_per_seq * 16; a page id outside [0, num_pages).
 * Ownership: every pointer is caller-owned device memory; nothing is allocated.
 * ------------------------------------------------------------------------------------------ */
JF_API jf_status jf_tree_kv_append(const void* k_new, const void* v_new, void* q, void* k_cache, void* v_cache,
                            const int32_t* block_table, int max_pages_per_seq, const int32_t* prefix_lens,
                            const int32_t* tree_offsets, const int32_t* depth, int batch, int total_nodes,
                            int num_q_heads, int num_kv_heads, int head_dim, int page_size, int num_pages,
                            float rope_theta, int32_t* dev_status, jf_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* JF_H_ */
