/*
 * hswa.h -- hybrid sliding-window attention on NVIDIA B200 (sm_100a): C ABI of libhswa.so.
 *
 * What it computes. For a query at absolute position i the sliding-window layers
 * attend the keys j with max(0, i - W + 1) <= j <= i and the full layers attend
 * 0 <= j <= i, with softmax(q.k / sqrt(head_dim)) weights on the values
 * ("Sliding Window Attention (SWA) no riron to jisso", disassemble-channel.com,
 * section "formal definition", eqs. (1)-(5)). Several query heads share one KV
 * head: query head h reads KV head h / (n_q_heads / n_kv_heads) (same page,
 * section "Mistral: SWA and GQA"). Keys and values of the SWA layers live in a
 * rolling buffer of W slots with slot = position mod W (same page, section
 * "Rolling Buffer KV Cache", eq. (7)); keys and values of the full layers live
 * in a paged pool sized by the sequence length. The two pools together are the
 * dual-pool KV cache of "MiMo v2.5 inference optimisation" (youngju.dev,
 * section "KV cache redesign"), which also defines the window-safe prefix-match
 * length.
 *
 * Conventions for every call.
 *  - Returns HSWA_OK (0) or a negative HSWA_ERR_* code; hswa_last_error()
 *    returns a message for the last failure on the calling thread.
 *    No C++ exception crosses this boundary.
 *  - Tensor arguments are raw device pointers owned by the caller (normally
 *    torch tensors), contiguous in the layouts stated below, 16-byte aligned.
 *    bf16 data is passed as its 16-bit pattern (hswa_bf16).
 *  - Compute calls enqueue work on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and return without synchronising. Argument errors
 *    found on the host return before anything is enqueued. Errors found on the
 *    device (a page id out of range, a context length above the declared
 *    maximum, a wait that ran out) are recorded in the pool's device error word
 *    and read back with hswa_pool_check_error().
 *  - The library never allocates device memory per call. Pool memory and the decode
 *    workspace are passed in by the caller (hybrid_decode_fwd_noalloc instead uses one
 *    fixed scratch array that is reserved when the library's device code is loaded).
 *  - Supported shapes: head_dim 64 or 128, n_q_heads a multiple of n_kv_heads,
 *    n_q_heads / n_kv_heads <= 16, W >= 1, page_size 64. Anything else returns
 *    HSWA_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef HSWA_H
#define HSWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HSWA_API __attribute__((visibility("default")))
#else
#define HSWA_API
#endif

#define HSWA_OK 0
#define HSWA_ERR_INVALID_ARG (-1)
#define HSWA_ERR_UNSUPPORTED_SHAPE (-2)
#define HSWA_ERR_OUT_OF_MEMORY (-3)
#define HSWA_ERR_CUDA (-4)
#define HSWA_ERR_TIMEOUT (-5)
#define HSWA_ERR_DEVICE_BOUNDS (-6)

/* Storage format of a pool's K/V entries (hswa_pool_desc.kv_format). */
#define HSWA_KV_BF16 0     /* bf16, as given */
#define HSWA_KV_FP8_E4M3 1 /* FP8 E4M3 codes with a scale per (layer, KV head) and K/V, see kv_pool_set_scales */

typedef uint16_t hswa_bf16;
typedef struct hswa_pool hswa_pool;

/* Shape of a dual-pool KV cache.
 * Layers 0 .. n_swa_layers-1 of the pool are sliding-window layers with a
 * W-slot ring per (sequence, layer, KV head); layers n_swa_layers ..
 * n_swa_layers+n_full_layers-1 are full layers whose token-slots are pages of
 * page_size tokens, pages_per_full_layer pages per layer, shared by all
 * sequences through a page table. */
typedef struct hswa_pool_desc {
  int32_t n_swa_layers;          /* >= 0 */
  int32_t n_full_layers;         /* >= 0 */
  int32_t window;                /* W >= 1 */
  int32_t n_kv_heads;            /* >= 1 */
  int32_t head_dim;              /* 64 or 128 */
  int32_t page_size;             /* 64 */
  int32_t max_seqs;              /* number of ring rows (sequence ids 0 .. max_seqs-1) */
  int32_t kv_format;             /* HSWA_KV_BF16 or HSWA_KV_FP8_E4M3 */
  int64_t pages_per_full_layer;  /* >= 0 */
} hswa_pool_desc;

/* Dual-pool sizing ("MiMo v2.5 inference optimisation", section "KV cache redesign":
 * the SWA pool holds W tokens, O(W); the full pool is sized by length, O(N)).
 * Device memory layout, from the base pointer (e = 2 bytes per element for bf16, 1 for FP8):
 *   ring  K then V : [2][max_seqs][n_swa_layers][n_kv_heads][W][head_dim] elements
 *   pages K then V : [2][n_full_layers][pages_per_full_layer][n_kv_heads][page_size][head_dim] elements
 *   scales (FP8 only): [4][n_swa_layers + n_full_layers][n_kv_heads] float32: K scale, V scale,
 *                    and their fp32 reciprocals
 *   error word     : 256 bytes (int32 device error code + spare)
 * each region starting on a 256-byte boundary.
 * bytes_swa  = 2 * max_seqs * n_swa_layers * n_kv_heads * W * head_dim * e, rounded up to 256;
 * bytes_full = 2 * n_full_layers * pages * n_kv_heads * page_size * head_dim * e, rounded up to 256;
 * bytes_total = bytes_swa + bytes_full + (FP8: 16 * layers * n_kv_heads rounded up to 256) + 256.
 * An FP8 entry holds code = E4M3(fp32(x) * fp32(1 / s)) (nearest, ties to even, saturating at
 * +-448; OCP 8-bit floating point E4M3) and stands for the value E4M3_value(code) * s, where s is
 * the scale of its layer, KV head and K or V ("MiMo v2.5 inference optimisation", closing
 * section: quantization cuts the bits per cached entry and stacks with the window's cut in
 * entries). Any output pointer may be NULL. */
HSWA_API int kv_pool_layout(const hswa_pool_desc* desc, size_t* bytes_total, size_t* bytes_swa,
                   size_t* bytes_full);

/* Carve a pool out of caller-owned device memory `dev_mem` of `bytes` bytes
 * (>= bytes_total, 256-byte aligned) on the current CUDA device. The library
 * keeps views and TMA descriptors only; it does not initialise the K/V slots,
 * sets every FP8 scale to 1 and clears the error word (synchronous copies). The
 * caller frees dev_mem after kv_pool_destroy(). */
HSWA_API int kv_pool_create(const hswa_pool_desc* desc, void* dev_mem, size_t bytes, hswa_pool** out);

/* FP8 pools: the scales of layer `layer`, k_scale[g] and v_scale[g] for KV head g (host arrays of
 * n_kv_heads finite values > 0). Entries appended afterwards are quantized with them and every
 * read of the layer dequantizes with them, so set them before the layer's first append. The copy
 * is synchronous; no work on the layer may be in flight. HSWA_ERR_INVALID_ARG for a bf16 pool. */
HSWA_API int kv_pool_set_scales(hswa_pool* pool, int layer, const float* k_scale, const float* v_scale);

/* Release the host-side handle (not the device memory). NULL is accepted. */
HSWA_API int kv_pool_destroy(hswa_pool* pool);

/* Commit n_tok new tokens per sequence into layer `layer` (quantized to FP8 in an FP8 pool).
 *  k, v       [n_seqs][n_tok][n_kv_heads][head_dim] bf16, token t of row b sits at
 *             absolute position start_pos[b] + t.
 *  start_pos  device int64[n_seqs], >= 0.
 *  seq_ids    device int32[n_seqs], ring row of each sequence (SWA layers; may be NULL for full layers).
 *  page_table device int32[n_seqs][pt_stride]: row b lists the physical page of logical page
 *             p = position / page_size of sequence b (full layers; may be NULL for SWA layers).
 * SWA layer: only the last min(n_tok, W) tokens are written, each to slot position mod W
 * ("Rolling Buffer KV Cache", eq. (7)); earlier tokens of the chunk would be
 * overwritten within the same chunk. Full layer: every token goes to
 * page_table[b][pos / page_size], row pos mod page_size. A page id outside
 * [0, pages_per_full_layer) or a logical page >= pt_stride is skipped and
 * recorded as HSWA_ERR_DEVICE_BOUNDS. */
HSWA_API int kv_pool_append(hswa_pool* pool, int layer, int n_seqs, const int32_t* seq_ids,
                   const int64_t* start_pos, int n_tok, const hswa_bf16* k, const hswa_bf16* v,
                   const int32_t* page_table, int pt_stride, void* stream);

/* Assemble ring row dst_seq of sliding-window layer `layer` slot by slot (entries are copied as
 * stored, bf16 or FP8): for each slot s with
 * src_seq[s] >= 0, the K and V rows of slot s (all KV heads) are copied from ring row src_seq[s];
 * slots with src_seq[s] = -1 or src_seq[s] = dst_seq are left as they are. Since every ring keeps
 * position p in slot p mod W, this moves cached window positions held by other sequences' rings
 * into the row of a request that resumes from a prefix-cache match (hswa_tree_match_slots gives
 * src_seq). src_seq: device int32[W]. A source row outside [0, max_seqs) is skipped and recorded
 * as HSWA_ERR_DEVICE_BOUNDS. Rows that are both a source and dst_seq must not be passed. */
HSWA_API int kv_pool_gather_ring(hswa_pool* pool, int layer, int32_t dst_seq, const int32_t* src_seq,
                                 void* stream);

/* Causal sliding-window attention for one chunk of n_q new tokens per sequence
 * ("formal definition", eqs. (1)-(5), window W of the pool), on tensor cores.
 *  q, o    [B][n_q][n_q_heads][head_dim] bf16 (o written, rows in the chunk only)
 *  k, v    [B][n_q][n_kv_heads][head_dim] bf16, the chunk's own keys and values
 *  start_pos device int64[B] = absolute position of the chunk's first token, or NULL for 0.
 *  seq_ids   device int32[B] ring rows (needed when start_pos is not NULL).
 * Keys before start_pos[b] are read from the ring of layer `layer` (an SWA layer),
 * which must hold positions [start_pos[b] - W, start_pos[b]) as committed by
 * kv_pool_append: attention reads the ring as it was before this chunk; commit
 * the chunk with kv_pool_append afterwards. Key tiles wholly outside every
 * query's window are skipped, not masked. fp32 accumulation and softmax.
 * W = 1: the window is the diagonal alone, so o_i = v_i of the query head's KV head; the call
 * copies those rows (q, k and the ring are not read). FP8 pools: keys before start_pos come from
 * the ring dequantized (code value times scale, rounded to bf16); the chunk's own k and v are
 * used as given. */
HSWA_API int swa_prefill_fwd(hswa_pool* pool, int layer, const hswa_bf16* q, const hswa_bf16* k,
                    const hswa_bf16* v, hswa_bf16* o, int B, int n_q, const int64_t* start_pos,
                    const int32_t* seq_ids, int n_q_heads, void* stream);

/* Full causal attention for one chunk of n_q tokens per sequence over the paged
 * pool of full layer `layer`: query i = start_pos[b] + t attends positions 0..i,
 * all read through the page table (the chunk itself must already be appended).
 *  q, o      [B][n_q][n_q_heads][head_dim] bf16
 *  start_pos device int64[B] (NULL for 0); page_table device int32[B][pt_stride]. */
HSWA_API int full_prefill_fwd(hswa_pool* pool, int layer, const hswa_bf16* q, hswa_bf16* o, int B,
                     int n_q, const int64_t* start_pos, const int32_t* page_table, int pt_stride,
                     int n_q_heads, void* stream);

/* Bytes of device workspace hybrid_decode_fwd needs for these arguments. */
HSWA_API int hybrid_decode_workspace_size(const hswa_pool* pool, int n_seqs, int n_q_per_seq,
                                 int n_q_heads, int64_t max_ctx_len, size_t* bytes);

/* One decode step: n_q_per_seq (1..8; 4 = one token + three multi-token-prediction
 * drafts) new query tokens per sequence at positions L .. L+n_q_per_seq-1, where
 * L = ctx_len[b] cached tokens. Draft t attends the cached keys in its window
 * plus new tokens 0..t (causal among themselves). SWA layer: the cached keys
 * come from the ring, which must hold positions [L - W, L); full layer: from the
 * page table, positions [0, L). The new keys/values are read from k_new/v_new,
 * not from the pool: commit them with kv_pool_append after acceptance.
 * Split-KV: the cached keys are cut into splits that run in parallel and are
 * merged with their log-sum-exp partials.
 *  q, o          [n_seqs][n_q_per_seq][n_q_heads][head_dim] bf16
 *  k_new, v_new  [n_seqs][n_q_per_seq][n_kv_heads][head_dim] bf16
 *  ctx_len       device int64[n_seqs], 0 <= L <= max_ctx_len (else HSWA_ERR_DEVICE_BOUNDS)
 *  seq_ids       device int32[n_seqs] ring rows (SWA layer)
 *  page_table    device int32[n_seqs][pt_stride] (full layer)
 *  workspace     device scratch of ws_bytes >= hybrid_decode_workspace_size(); its contents
 *                on entry do not matter; calls sharing one workspace must not overlap.
 * FP8 pools with head_dim 128: the environment variable HSWA_DECODE_TC, read once per process,
 * selects a tcgen05 kernel for full layers (1) or for every layer (2) instead of the default
 * mma.sync kernel (0 or unset); both compute the same attention (within the stated tolerance),
 * the default is the faster one as measured. */
HSWA_API int hybrid_decode_fwd(hswa_pool* pool, int layer, const hswa_bf16* q, const hswa_bf16* k_new,
                      const hswa_bf16* v_new, hswa_bf16* o, int n_seqs, int n_q_per_seq,
                      const int64_t* ctx_len, int64_t max_ctx_len, const int32_t* seq_ids,
                      const int32_t* page_table, int pt_stride, int n_q_heads, void* workspace,
                      size_t ws_bytes, void* stream);

/* Largest scratch hybrid_decode_fwd_noalloc can use: 64 MiB. */
#define HSWA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* hybrid_decode_fwd without a workspace argument. The source pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory when they call
 * the library -- for example a plugin inside a host runtime that owns every device
 * allocation, or a serving loop that must not call cudaMalloc (an allocation can
 * synchronise the device). Its scratch is one fixed device array of
 * HSWA_NOALLOC_SCRATCH_BYTES inside this library, which every GPU that loads the library
 * keeps until the process exits; nothing is allocated per call.
 *  - Same arguments, layouts and results as hybrid_decode_fwd, minus workspace/ws_bytes.
 *  - Returns HSWA_ERR_OUT_OF_MEMORY, before launching anything, when the call would need
 *    more scratch than the array holds (hybrid_decode_workspace_size() reports the need).
 *  - The first call on a device looks up the array's device address on the current
 *    device; make that first call before any stream capture.
 *  - All calls on a device share the one array: calls that overlap on the GPU (other
 *    streams, other host threads) race and give wrong results; serialise them. Leftover
 *    contents from an earlier call do not matter (the kernels reset what they read). */
HSWA_API int hybrid_decode_fwd_noalloc(hswa_pool* pool, int layer, const hswa_bf16* q, const hswa_bf16* k_new,
                                       const hswa_bf16* v_new, hswa_bf16* o, int n_seqs, int n_q_per_seq,
                                       const int64_t* ctx_len, int64_t max_ctx_len, const int32_t* seq_ids,
                                       const int32_t* page_table, int pt_stride, int n_q_heads, void* stream);

/* Window-safe prefix-match length ("MiMo v2.5 inference optimisation", section
 * "KV cache redesign": a prefix-cache match may be reused only as far as the
 * last W tokens before the resume point still have valid SWA slots).
 * For request r with match length m = match_len[r] and cached length C = cached_len[r],
 * whose ring holds positions [max(0, C-W), C) with slot s valid iff bit s%32 of
 * slot_valid[r * ((W+31)/32) + s/32] is set:
 *   out_len[r] = max { L in [0, m] : every position in [max(0, L-W), L) is held in a valid slot }.
 * All arrays are device memory; results are exact integers. */
HSWA_API int window_safe_len(const int64_t* match_len, const int64_t* cached_len,
                    const uint32_t* slot_valid, int32_t W, int32_t n_req, int64_t* out_len,
                    void* stream);

/* SWA-aware prefix cache over a token trie (host memory, host code; "MiMo v2.5 inference
 * optimisation", section "KV cache redesign": a prefix-cache match is cut to the window-safe
 * length, since with sliding-window layers only part of a cached sequence's window KV may
 * survive). Each trie node is one cached position. Its full-attention KV is held while the node
 * exists. Each insert names an owner: the ring row (sequence id of the pool) where the caller keeps
 * that sequence's sliding-window KV, or -1. A position's holders are the owners whose window (their
 * last W positions) covers it and whose copy has not been evicted since that insert; the position
 * holds sliding-window KV while it has a holder. With one cached sequence this is window_safe_len
 * with a per-position eviction mask; here cached sequences share prefixes.
 * Token ids are any int32 values. Calls on one tree are not thread-safe; the caller serialises
 * them. Errors: HSWA_ERR_INVALID_ARG for null pointers or negative lengths (nothing changes);
 * HSWA_ERR_OUT_OF_MEMORY when a host allocation fails during an insert, after which the tree
 * may hold part of that insert and should be destroyed. */
typedef struct hswa_prefix_tree hswa_prefix_tree;

/* New empty tree for window W >= 1; *out owns host memory until hswa_tree_destroy. */
HSWA_API int hswa_tree_create(int32_t window, hswa_prefix_tree** out);
HSWA_API int hswa_tree_destroy(hswa_prefix_tree* tree);

/* Cache tokens[0..n) for `owner`: adds the missing positions and makes the owner a holder of this
 * sequence's window [max(0, n-W), n). *new_nodes (may be null) = positions added. */
HSWA_API int hswa_tree_insert(hswa_prefix_tree* tree, const int32_t* tokens, int64_t n, int32_t owner,
                              int64_t* new_nodes);

/* Undo one hswa_tree_insert of the same tokens by the same owner: the owner stops holding that
 * window (other holders keep their positions). HSWA_ERR_INVALID_ARG, with nothing changed, unless
 * such an insert is left to undo (a cached prefix that was never inserted on its own, another
 * owner's insert, or a second release of a single insert is rejected). n = 0 is a no-op. */
HSWA_API int hswa_tree_release(hswa_prefix_tree* tree, const int32_t* tokens, int64_t n, int32_t owner);

/* Drop the sliding-window KV of positions [pos_lo, pos_hi) along the path tokens[0..n) (every
 * holder loses it); *evicted (may be null) = positions that held it. */
HSWA_API int hswa_tree_evict_swa(hswa_prefix_tree* tree, const int32_t* tokens, int64_t n, int64_t pos_lo,
                                 int64_t pos_hi, int64_t* evicted);

/* Match tokens[0..n): *match_len = m = longest cached prefix; *safe_len = max { L in [0, m] :
 * every position in [max(0, L-W), L) holds sliding-window KV }, the length a request can resume
 * from. Exact integers. */
HSWA_API int hswa_tree_match(const hswa_prefix_tree* tree, const int32_t* tokens, int64_t n,
                             int64_t* match_len, int64_t* safe_len);

/* hswa_tree_match plus where the resumed window lives: slot_owner[W] (host memory) gets, for each
 * position p in [max(0, L-W), L), at slot p mod W, the owner of the most recent insert that holds
 * p; every other slot gets -1. kv_pool_gather_ring with these owners as sources assembles the
 * request's ring for a prefill that starts at L. */
HSWA_API int hswa_tree_match_slots(const hswa_prefix_tree* tree, const int32_t* tokens, int64_t n,
                                   int64_t* match_len, int64_t* safe_len, int32_t* slot_owner);

/* hswa_tree_match for n_req requests: request r is tokens[offsets[r] .. offsets[r+1]). */
HSWA_API int hswa_tree_match_batch(const hswa_prefix_tree* tree, const int32_t* tokens, const int64_t* offsets,
                                   int32_t n_req, int64_t* match_len, int64_t* safe_len);

/* Cached positions (trie nodes) and how many of them hold sliding-window KV. */
HSWA_API int hswa_tree_stats(const hswa_prefix_tree* tree, int64_t* n_positions, int64_t* n_swa_held);

/* Multi-GPU partition of the hot path (host code; one process per GPU).
 * Prefill splits by KV head: query head h reads only KV head h / G ("Sliding Window Attention
 * (SWA) no riron to jisso", section "Mistral: SWA and GQA"), so the rank that owns KV heads
 * [head_begin, head_end) and query heads [head_begin * G, head_end * G) keeps that slice of every
 * pool (a pool created with n_kv_heads = head_end - head_begin) and computes those outputs with
 * no exchange. hswa_shard_kv_heads gives rank `rank` of n_ranks its contiguous, equal range;
 * HSWA_ERR_UNSUPPORTED_SHAPE unless n_kv_heads is a multiple of n_ranks. */
HSWA_API int hswa_shard_kv_heads(int32_t n_kv_heads, int32_t n_ranks, int32_t rank, int32_t* head_begin,
                                 int32_t* head_end);

/* Decode splits by sequence: every sequence, with its ring rows and pages, lives on one rank.
 * Sequences are taken longest length bucket first (>= 256K, 64K..256K, < 64K tokens; "MiMo v2.5
 * inference optimisation", section "KV cache redesign"), longest first inside a bucket, and each
 * goes to the rank with the least total context so far (lowest rank on ties).
 * ctx_len[n_seqs] (host, >= 0) -> rank_of_seq[n_seqs] (host) and, when not NULL,
 * load_per_rank[n_ranks] = total context per rank. */
HSWA_API int hswa_shard_sequences(const int64_t* ctx_len, int32_t n_seqs, int32_t n_ranks, int32_t* rank_of_seq,
                                  int64_t* load_per_rank);

/* Diagnostic: run, on `stream`, one wait on a barrier that nothing arrives at, through the same
 * bounded wait every kernel uses, with a limit of limit_ns (1 ms .. 2 s; the kernels themselves
 * use 2 s). The wait gives up, records HSWA_ERR_TIMEOUT in the pool's error word and the kernel
 * returns; hswa_pool_check_error() then reports it. Nothing faults and the context stays usable. */
HSWA_API int hswa_selftest_wait_timeout(hswa_pool* pool, int64_t limit_ns, void* stream);

/* Synchronise the device, return the pool's device error word in *device_code
 * (0 if none, else a negative HSWA_ERR_* code) and clear it. */
HSWA_API int hswa_pool_check_error(hswa_pool* pool, int* device_code);

/* Message for the last failed call on this thread ("" if none). */
HSWA_API const char* hswa_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* HSWA_H */
