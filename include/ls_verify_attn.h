/*
 * ls_verify_attn — tree-verification attention for long-context speculative decoding,
 * for NVIDIA B200 (sm_100a).
 *
 * The operation (LongSpec: Long-Context Lossless Speculative Decoding with Efficient
 * Drafting and Verification; gist.science summary, section 2C "Schnelle Tree
 * Attention", the "Aufteilung" and "Aggregation" paragraphs): every query token of a
 * speculated token tree attends
 *   - to the whole cached prefix of its sequence, with no mask ("Cached-Teil"), and
 *   - to the tree tokens under the tree mask ("Speculative-Teil"), read here as
 *     ancestor-or-self visibility built from a parent[] array,
 * and the two partial softmax results are merged with a log-sum-exp step so that
 * the output equals one softmax over the union of both key sets. The abstracts
 * (arXiv v1 on mlsanity; ACL record on PaperTrail) call the method lossless: the
 * result is exact attention, not an approximation.
 *
 * For sequence b, tree node i, query head h (kv head kh = h / (H_q / H_kv)):
 *   visible(i) = { prefix keys 0..L_b-1 } U { tree nodes a : a == i or a is an ancestor of i }
 *   s_x  = softmax_scale * <q[b,i,h,:], k_x[kh,:]>
 *   lse  = ln sum_{x in visible(i)} exp(s_x)            (natural log, scale included)
 *   out  = sum_{x in visible(i)} exp(s_x - lse) * v_x[kh,:]
 *
 * All calls are C functions with plain pointers and sizes. Device pointers are CUDA
 * device (or managed) memory of the current device. The calls that take a workspace
 * allocate no memory and keep no state between calls: every buffer, including the
 * workspace, belongs to the caller. The one exception is ls_verify_attn_static (below),
 * whose scratch is a fixed array in the library's own device memory that keeps what the
 * last such call left in it. Nothing in this library traps or aborts: errors come back
 * as status codes.
 */
#ifndef LS_VERIFY_ATTN_H
#define LS_VERIFY_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LS_API __attribute__((visibility("default")))
#else
#define LS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum {
  LS_OK = 0,
  LS_ERR_INVALID_ARG = 1,  /* null pointer, bad dimension, misaligned pointer, bad cu_seqlens_host */
  LS_ERR_UNSUPPORTED = 2,  /* head_dim other than 64/128, tree_size > 128, not an sm_100 device */
  LS_ERR_WORKSPACE = 3,    /* workspace null, misaligned or smaller than ls_verify_attn_workspace_size */
  LS_ERR_CUDA = 4,         /* a CUDA launch or copy failed */
  LS_ERR_BAD_TREE = 5,     /* device found parent[] that is not a rooted tree with parent[i] < i */
  LS_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up (pipeline stalled) */
  LS_ERR_LENGTHS = 7,      /* device cu_seqlens disagrees with cu_seqlens_host / max_prefix_len */
  LS_ERR_INDEX = 8         /* index-checking build (libls_verify_attn_debug.so) only: a kernel formed
                              a TMA coordinate or global index outside the tensor it addresses */
};

/* Problem description, passed by pointer to every call. */
typedef struct ls_verify_dims {
  int32_t batch;          /* B >= 1 sequences */
  int32_t num_q_heads;    /* H_q >= 1, a multiple of num_kv_heads (grouped-query attention) */
  int32_t num_kv_heads;   /* H_kv >= 1 */
  int32_t head_dim;       /* d: 64 or 128 */
  int32_t tree_size;      /* T: tree nodes per sequence, 1..128, the same for every sequence */
  int32_t max_prefix_len; /* an upper bound on every L_b (used when cu_seqlens_host is NULL) */
  const int32_t* cu_seqlens_host; /* optional HOST copy of cu_seqlens [B+1]; when given it must
                                     equal the device array, and the work split is balanced
                                     over the actual lengths. NULL: every sequence is planned
                                     as max_prefix_len long (correct, less balanced). */
  float softmax_scale;    /* <= 0 selects 1/sqrt(head_dim) */
} ls_verify_dims;

/*
 * Bytes of device workspace that ls_verify_attn needs for these dims on the current
 * device (it depends on the SM count and, when cu_seqlens_host is given, on the
 * lengths). Returns 0 if the dims are invalid or unsupported.
 */
LS_API size_t ls_verify_attn_workspace_size(const ls_verify_dims* dims);

/*
 * Tree-verification attention, asynchronous on `stream` (a cudaStream_t; NULL is the
 * legacy default stream). Returns after enqueuing its kernels.
 *
 *   q          bf16 [B*T, H_q, d]      tree queries, token-major (row b*T+i is node i
 *                                      of sequence b), already position-encoded
 *   k_cache    bf16 [sum_b L_b, H_kv, d] prefix keys of all sequences, packed in
 *                                      sequence order by cu_seqlens
 *   v_cache    bf16 [sum_b L_b, H_kv, d]
 *   k_tree     bf16 [B*T, H_kv, d]     keys of the tree tokens
 *   v_tree     bf16 [B*T, H_kv, d]
 *   tree_parent int32 [B*T]            parent of node i of sequence b as a local index:
 *                                      -1 for node 0 (the root), in [0, i) otherwise
 *   cu_seqlens int32 [B+1] (device)    cu_seqlens[0] = 0, L_b = cu[b+1] - cu[b] >= 0
 *   out        bf16 [B*T, H_q, d]      written (round to nearest even)
 *   lse        fp32 [B*T, H_q]         written: natural-log normaliser, scale included
 *   workspace  device scratch of at least ls_verify_attn_workspace_size(dims) bytes,
 *              256-byte aligned; its contents need no initialisation and are
 *              overwritten. Concurrent calls must use different workspaces.
 *
 * Every tensor is dense row-major with the innermost dimension contiguous. The bf16
 * tensors must start on a 16-byte boundary, the int32/fp32 ones on a 4-byte boundary. `out` and `lse` must not alias any input.
 * Host-detectable errors return LS_ERR_INVALID_ARG / LS_ERR_UNSUPPORTED /
 * LS_ERR_WORKSPACE before anything is launched. Errors that only the device can see
 * (bad tree, cu_seqlens mismatch, a wait that timed out) are recorded in the
 * workspace and reported by ls_verify_attn_check; the outputs of such a call are
 * unspecified but no memory outside the given buffers is touched.
 */
LS_API int ls_verify_attn(const void* q, const void* k_cache, const void* v_cache,
                   const void* k_tree, const void* v_tree,
                   const int32_t* tree_parent, const int32_t* cu_seqlens,
                   void* out, float* lse,
                   const ls_verify_dims* dims,
                   void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * The two stages that ls_verify_attn runs, for callers that want to place or time
 * them separately. They must be called in this order, on the same stream (or with
 * the caller ordering them), with the same dims and workspace; together they are
 * exactly ls_verify_attn. Arguments as for ls_verify_attn.
 *
 * ls_verify_attn_partials (the "Cached-Teil" and "Speculative-Teil" of section 2C):
 * the keys of sequence b are its ceil(L_b/128) prefix blocks followed by one block of
 * its T tree keys. They are split into chunks of consecutive blocks, and each chunk
 * leaves, for every query row of one kv head's unit of rows, its partial (out
 * normalised by its own sum, lse) in the workspace. Prefix keys are attended with no
 * mask; a tree key is visible to node i when it is i or one of i's ancestors
 * (tree_parent is checked: a bad tree is reported as LS_ERR_BAD_TREE by
 * ls_verify_attn_check). k_cache and v_cache may be NULL when no sequence has a prefix
 * (cu_seqlens_host all zero, or max_prefix_len = 0).
 *
 * ls_verify_attn_combine (the "Aggregation" of section 2C): merges every row's
 * partials by log-sum-exp and writes `out` and `lse`.
 */
LS_API int ls_verify_attn_partials(const void* q, const void* k_cache, const void* v_cache,
                                   const void* k_tree, const void* v_tree, const int32_t* tree_parent,
                                   const int32_t* cu_seqlens, const ls_verify_dims* dims, void* workspace,
                                   size_t workspace_bytes, void* stream);
LS_API int ls_verify_attn_combine(const int32_t* cu_seqlens, void* out, float* lse,
                                  const ls_verify_dims* dims, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * A paged K/V cache. The LongSpec pages keep each sequence's cache contiguous and have no
 * counterpart; this is the block-table layout of PagedAttention ("Efficient Memory
 * Management for Large Language Model Serving with PagedAttention", which the mlsanity
 * page of LongSpec lists under "Builds on"), the layout serving engines use. The keys
 * of sequence b are still L_b = cu_seqlens[b+1] - cu_seqlens[b] long, but key k of the
 * sequence lives in row (page_table[b * max_pages_per_seq + k / page_size] * page_size
 * + k % page_size) of
 *   k_pages    bf16 [num_pages * page_size, H_kv, d]   (16-byte aligned)
 *   v_pages    bf16 [num_pages * page_size, H_kv, d]
 * cu_seqlens then gives only the lengths (its offsets are not used to address the cache).
 *
 *   page_size          16, 32, 64, or a multiple of 128 up to 2^20; else LS_ERR_UNSUPPORTED
 *   max_pages_per_seq  columns of page_table, >= ceil(L_b / page_size) for every planned L_b
 *   num_pages          pages in k_pages / v_pages; num_pages * page_size < 2^31
 *   page_table         device int32 [batch, max_pages_per_seq]; an entry outside
 *                      [0, num_pages) is not an error: the kernel then reads zeros or
 *                      another page (never memory outside the cache), so the result is
 *                      unspecified but no fault occurs. Entries past a sequence's last
 *                      page are not read.
 */
typedef struct {
  int32_t page_size;
  int32_t max_pages_per_seq;
  int64_t num_pages;
  const int32_t* page_table;
} ls_paged_kv;

/*
 * ls_verify_attn over a paged K/V cache: the same computation, arguments and errors as
 * ls_verify_attn, with k_cache / v_cache replaced by the pages and their table. The same
 * workspace size (ls_verify_attn_workspace_size) applies.
 */
LS_API int ls_verify_attn_paged(const void* q, const void* k_pages, const void* v_pages,
                                const ls_paged_kv* paged, const void* k_tree, const void* v_tree,
                                const int32_t* tree_parent, const int32_t* cu_seqlens, void* out,
                                float* lse, const ls_verify_dims* dims, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * Per-sequence trees, sliding windows and in-kernel tree positions, for ls_verify_attn_ex.
 *
 * cu_tree: trees of different sizes. Sequence b's tree nodes are rows
 *   [cu_tree[b], cu_tree[b+1]) of q, k_tree, v_tree, tree_parent, out and lse (all packed
 *   by cu_tree instead of b * tree_size); dims->tree_size is then the largest tree
 *   allowed (1..128) and the work is planned for it. cu_tree is device int32 [B+1] with
 *   cu_tree[0] = 0, cu_tree[B] = total_nodes and 0 <= cu_tree[b+1] - cu_tree[b] <=
 *   tree_size; a sequence may have no node. tree_parent holds each tree's own local
 *   indices (-1 for its root, node 0). A device cu_tree that breaks these rules is
 *   reported as LS_ERR_LENGTHS by ls_verify_attn_check (its sequences get no output).
 *   NULL: every sequence has tree_size nodes and total_nodes is ignored.
 *
 * window > 0: sliding-window attention (the draft model's self-attention keeps a window
 *   of recent tokens; LongSpec, gist.science summary, section 2A, "Sliding-Window
 *   Self-Attention", e.g. 512). A query at position P sees the keys at positions
 *   P - window + 1 .. P, where prefix key j sits at position j and tree node i at
 *   L_b + depth(i): node i sees the prefix keys j >= L_b + depth(i) + 1 - window and all
 *   its ancestors (window >= tree_size is required, so no tree key falls outside it;
 *   else LS_ERR_INVALID_ARG). The prefix may be the whole cache or just its last keys;
 *   positions count from its first key. window = 0: the whole prefix.
 *
 * rope_theta > 0: q and k_tree arrive without rotary position embedding and the
 *   library applies it (RoFormer, listed under "Builds on" on the mlsanity page): node i
 *   of sequence b sits at position L_b + depth(i) (the root right after the prefix,
 *   siblings at one position), and each pair (x[e], x[e + d/2]) of a head is rotated by
 *   the angle position * rope_theta^(-2e/d) (the half-split pairing of the Llama and Qwen
 *   models; rope_theta is the model's base, e.g. 10000, 500000 or 1000000). The rotated
 *   values are rounded to bf16, as a caller's own rotation would leave them, and held in
 *   the workspace; v_tree and the cached keys (rotated when they were written) are read
 *   as they are. rope_theta = 0: q and k_tree are already rotated.
 *
 * wait_limit_ns > 0: the longest time (nanoseconds, up to 60 s; more is
 *   LS_ERR_INVALID_ARG) that any of the partials kernel's device-side waits (a CTA's
 *   roles hand tiles to one another through shared-memory barriers) may take. A wait
 *   that runs out stops its CTA: every role lets its copies and tensor-core work in
 *   flight finish, the CTA frees its tensor memory and returns, and
 *   ls_verify_attn_check reports LS_ERR_TIMEOUT for the call (its outputs are then
 *   unspecified; the workspace and the device need no cleaning before the next call).
 *   It is the stall detector of the pipeline: a healthy call waits microseconds, so
 *   the default (wait_limit_ns = 0: 4 s) only fires on a stalled GPU. A limit shorter
 *   than a call's normal waits makes healthy calls fail.
 */
typedef struct {
  const int32_t* cu_tree;
  int32_t total_nodes;
  int32_t window;
  double rope_theta;
  uint64_t wait_limit_ns;
} ls_tree_opts;

/*
 * The general entry: ls_verify_attn over a packed (paged == NULL) or paged K/V cache,
 * with per-sequence trees and in-kernel RoPE as `tree` asks (tree == NULL: neither).
 * Arguments, results and errors are those of ls_verify_attn / ls_verify_attn_paged;
 * with cu_tree, the tree tensors, out and lse have total_nodes rows. The workspace
 * must hold ls_verify_attn_ex_workspace_size(dims, tree) bytes (more than
 * ls_verify_attn_workspace_size when rope_theta > 0); ls_verify_attn_check(dims, ...)
 * reads the call's device status.
 */
LS_API size_t ls_verify_attn_ex_workspace_size(const ls_verify_dims* dims, const ls_tree_opts* tree);
LS_API int ls_verify_attn_ex(const void* q, const void* k_cache, const void* v_cache, const ls_paged_kv* paged,
                             const void* k_tree, const void* v_tree, const int32_t* tree_parent,
                             const int32_t* cu_seqlens, const ls_tree_opts* tree, void* out, float* lse,
                             const ls_verify_dims* dims, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Prefix-only attention: the draft model's cross-attention over the target model's KV
 * cache (LongSpec, gist.science summary, section 2A, "Cross-Attention mit geteiltem
 * KV-Cache": the draft reads the target's cache directly, so long contexts cost it no
 * cache of its own). Every query of sequence b attends to all L_b keys of its sequence
 * in k_cache / v_cache with no mask, and to nothing else: there are no tree keys.
 *
 *   q          bf16 [B*T, H_q, d]   T = dims->tree_size queries per sequence (1..128)
 *   k_cache    bf16 [sum_b L_b, H_kv, d], v_cache likewise, packed by cu_seqlens (may be
 *              NULL when every L_b is 0)
 *   out, lse   as for ls_verify_attn; a sequence with L_b = 0 gets out = 0, lse = -inf
 *   workspace  at least ls_cross_attn_workspace_size(dims) bytes (it differs from
 *              ls_verify_attn_workspace_size: the key lists have no tree block)
 * Errors as for ls_verify_attn; ls_verify_attn_check reads its device status.
 * (The draft's sliding-window self-attention is ls_verify_attn_ex with ls_tree_opts.window.)
 */
LS_API size_t ls_cross_attn_workspace_size(const ls_verify_dims* dims);
LS_API int ls_cross_attn(const void* q, const void* k_cache, const void* v_cache, const int32_t* cu_seqlens,
                         void* out, float* lse, const ls_verify_dims* dims, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * ls_verify_attn without a workspace argument, for callers that cannot allocate device
 * memory (the LongSpec pages have no counterpart: this is an interface convenience).
 *
 * ls_verify_attn needs caller-provided scratch for the attention partials. A caller that
 * only ever receives its input and output buffers, such as an operator plugin inside an
 * inference engine that owns the whole device heap and hands its plugins no allocator,
 * has no way to provide it. This call instead uses a fixed 32 MiB array that lives in
 * the library's own device memory (every GPU that loads the library holds it until the
 * process exits) and allocates nothing. Arguments and results are those of
 * ls_verify_attn.
 *
 *   - Returns LS_ERR_WORKSPACE if these dims need more than 32 MiB of scratch (see
 *     ls_verify_attn_workspace_size); use ls_verify_attn with a workspace for those.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and keeps it; make that first call before capturing any
 *     stream. cudaDeviceReset reloads the library's device code, after which the kept
 *     address may be wrong: a process that resets a device must not call
 *     ls_verify_attn_static on it again.
 *   - All calls on a device share the one array, which keeps whatever the last call
 *     left in it. Calls whose kernels overlap on the GPU (different streams without an
 *     ordering between them) race on it and give wrong results; order them.
 *   - Device-detected errors (bad tree, length mismatch, timeout) are recorded in the
 *     shared array and cannot be read back through ls_verify_attn_check; callers that
 *     need them use ls_verify_attn.
 */
LS_API int ls_verify_attn_static(const void* q, const void* k_cache, const void* v_cache,
                                 const void* k_tree, const void* v_tree,
                                 const int32_t* tree_parent, const int32_t* cu_seqlens,
                                 void* out, float* lse, const ls_verify_dims* dims, void* stream);

/*
 * Greedy acceptance of a verified tree (the step after verification; LongSpec,
 * gist.science summary: section 2C verifies the tree in one pass, section 3 reports the
 * mean acceptance length tau). For each sequence, starting at the root (node 0, the last
 * token already accepted), the walk moves to the child whose draft token equals the
 * argmax of the current node's logits (the smallest such child if several do) and stops
 * when none does. This keeps exactly the tokens that greedy decoding of the target model
 * would produce, so it is lossless; the argmax at the last node is the next token, and
 * the step yields accept_len + 1 tokens. The argmax is the first index of the largest
 * logit above -inf (NaN entries are skipped; a row without such a logit gives 0).
 *
 *   logits       [N, vocab] bf16 or fp32 (logits_dtype), row n = tree node n; N = B * T,
 *                or total_nodes with cu_tree. 2-byte (bf16) / 4-byte (fp32) aligned;
 *                rows that start on 16-byte boundaries are read with 16-byte loads.
 *   tree_tokens  device int32 [N]: the draft token of every node (node 0's is not read)
 *   tree_parent  device int32 [N]: local parents as for ls_verify_attn
 *   cu_tree      device int32 [B+1] (per-sequence trees, as in ls_tree_opts) or NULL
 *   accept_len   device int32 [B]: accepted draft nodes (0..T_b-1); -1 if the sequence has
 *                no node, its cu_tree entry is not a packed layout, or its parents are not
 *                a rooted tree with parent[i] < i
 *   accept_path  device int32 [B, T]: local node indices of the path, root first
 *                (accept_len + 1 entries; the rest of the row is not written)
 *   next_token   device int32 [B]: argmax of the last node's logits (-1 when accept_len is -1)
 *   workspace    at least ls_tree_accept_workspace_size(dims, total_nodes) bytes, 256-byte
 *                aligned; holds per-segment maxima between the two kernels
 * Returns LS_OK, LS_ERR_INVALID_ARG, LS_ERR_UNSUPPORTED (tree_size > 128), LS_ERR_WORKSPACE
 * or LS_ERR_CUDA; asynchronous on `stream`. Sampling-based (non-greedy) verification is
 * not offered.
 */
enum { LS_DTYPE_BF16 = 0, LS_DTYPE_F32 = 1 };

typedef struct {
  int32_t batch;         /* B >= 1 */
  int32_t tree_size;     /* T: nodes per tree (the largest, with cu_tree), 1..128 */
  int32_t vocab;         /* logits per node >= 1 */
  int32_t logits_dtype;  /* LS_DTYPE_BF16 or LS_DTYPE_F32 */
} ls_accept_dims;

LS_API size_t ls_tree_accept_workspace_size(const ls_accept_dims* dims, int32_t total_nodes);
LS_API int ls_tree_accept_greedy(const void* logits, const int32_t* tree_tokens, const int32_t* tree_parent,
                                 const int32_t* cu_tree, int32_t total_nodes, int32_t* accept_len,
                                 int32_t* accept_path, int32_t* next_token, const ls_accept_dims* dims,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Waits for `stream`, then reads the device-side status that the last ls_verify_attn
 * call with this workspace and these dims recorded. Returns LS_OK, LS_ERR_BAD_TREE,
 * LS_ERR_LENGTHS, LS_ERR_TIMEOUT, LS_ERR_INDEX (index-checking build only), or
 * LS_ERR_CUDA if the copy itself failed.
 */
LS_API int ls_verify_attn_check(const ls_verify_dims* dims, const void* workspace, void* stream);

/* A static, human-readable name for a status code. */
LS_API const char* ls_status_string(int status);

/*
 * Describes how ls_verify_attn splits the work for these dims on the current device:
 * number of chunks (CTAs of the partials kernel), key blocks per chunk, and CTAs of
 * the combine kernel. Any pointer may be NULL. Returns a status.
 */
LS_API int ls_verify_attn_plan(const ls_verify_dims* dims, int32_t* partials_ctas,
                        int32_t* blocks_per_chunk, int32_t* combine_ctas);

#ifdef __cplusplus
}
#endif

#endif /* LS_VERIFY_ATTN_H */
