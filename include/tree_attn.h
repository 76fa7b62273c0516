/*
 * tree_attn.h — exact split decode attention on one B200 (sm_100a).
 *
 * What it computes.  For every sequence b and query head h, with KV head
 * g = h / (Hq / Hkv) and scores x_t = scale * q[b,h,:] . K_b[g,t,:]:
 *
 *     out[b,h,:] = sum_t softmax(x)_t V_b[g,t,:]         (exact softmax attention)
 *     lse[b,h]   = ln sum_t exp(x_t)                      (natural log)
 *
 * following the self-attention recap S = QK^T/sqrt(d_k), P = softmax(S), O = PV
 * of the "Attention acceleration" concept page (compassingai.com, Technical
 * principles, part 1) for one decode query per (sequence, head).
 *
 * How.  The KV cache is cut into contiguous chunks, one per CTA; each chunk
 * yields the softmax statistics (m, l, o) — running max, sum of exponentials,
 * unnormalised output — with the online-softmax update of the same page
 * (part 2.1, "Tiling and online softmax").  Because max and logsumexp are
 * associative (Tree Attention article, m.srwj168.com.cn, "The energy view of
 * attention"), the chunks' statistics are merged in a fixed log-depth pairwise
 * tree by the last CTA to finish a (sequence, KV head); this is the on-GPU form
 * of the query host combining softmax statistics in Star Attention's phase 2
 * (tiaojiaomugou.com article, "Phase 2: query encoding and token generation").
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers, except `seqlens` and
 *     `suffix_lens`, which are HOST arrays read before the call returns.
 *   - The caller owns every buffer; the library never frees caller memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Nothing synchronises the host except
 *     tree_attn_check().
 *   - q, k, v pointers must be 16-byte aligned (the kernels move K/V with bulk
 *     copies); out and lse 4-byte aligned.  Misalignment -> TA_ERR_INVALID_ARG.
 *   - Supported shapes: head_dim in {64, 128}; G = n_q_heads / n_kv_heads in
 *     {1, 2, 4, 8}.  Others -> TA_ERR_UNSUPPORTED.  n_q_heads % n_kv_heads != 0,
 *     a negative length, a non-finite scale or a NULL pointer ->
 *     TA_ERR_INVALID_ARG (K/V pointers may be NULL only when every length they
 *     serve is 0: nothing is read from them then).  Validation errors return
 *     before anything is launched.
 *   - A sequence of length 0 gives out = 0 and lse = -inf.
 *   - Results are bit-identical across calls with the same shapes, lengths,
 *     options and device (the chunking is a pure function of those; no float
 *     atomics; fixed merge order).
 *   - No exception crosses this interface.
 *
 * Layouts (row-major, no padding):
 *   q    [B][Hq][D]       bf16 (or f32 for the _f32 entry point / TA_F32)
 *   k, v packed per sequence: sequence b is a [Hkv][S_b][D] block; blocks are
 *        stored back to back in batch order, so sequence b starts at element
 *        Hkv * D * (S_0 + ... + S_{b-1}).  64-bit offsets throughout.
 *   out  [B][Hq][D]       f32
 *   lse  [B][Hq]          f32
 */
#ifndef TREE_ATTN_H
#define TREE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TA_OK = 0,
  TA_ERR_INVALID_ARG = 1, /* NULL / misaligned pointer, bad shape, negative length, non-finite scale */
  TA_ERR_UNSUPPORTED = 2, /* head_dim or GQA group size without a kernel */
  TA_ERR_WORKSPACE = 3,   /* workspace NULL, misaligned or smaller than required */
  TA_ERR_CUDA = 4,        /* a CUDA runtime call or a launch failed; see tree_attn_last_cuda_error() */
  TA_ERR_TIMEOUT = 5,     /* a bounded wait inside a kernel ran out (reported by tree_attn_check) */
  TA_ERR_SCRATCH_LIMIT = 6, /* tree_attn_decode_noalloc: the problem needs more scratch than its fixed buffer */
  TA_ERR_BAD_PAGE = 7       /* paged decode: a block-table entry outside [0, num_pages) (reported by
                               tree_attn_check; nothing was read through it, the outputs are NaN) */
} ta_status;

typedef enum { TA_BF16 = 0, TA_F32 = 1 } ta_dtype;

/* Optional tuning and test hooks; pass NULL for the defaults (all fields 0 / -1). */
typedef struct {
  int32_t num_ctas;        /* 0: one CTA per resident slot (SMs x CTAs per SM), at most one per two
                              tiles; else the split grid size */
  int32_t wait_limit_us;   /* 0: 2,000,000 us.  Bound on every wait inside a kernel; on expiry the
                              kernel records TA_ERR_TIMEOUT in the workspace and returns */
  int32_t debug_skip_tile; /* -1: off.  Test hook: CTA 0 never loads this tile of its range, so its
                              consumers' wait runs out (no fault: the data simply never arrives).
                              Tensor-core passes: CTA (0, 0, 0) never loads this K tile */
  int32_t prefix_path;     /* bifurcated, multi-query and decode calls.  Bifurcated: 0 automatic
                              (tensor-core prefix pass when head_dim is 128 and the prefix is not
                              empty); 1 tensor-core pass (TA_ERR_UNSUPPORTED if not possible); 2
                              split-KV pass per sample.  Multi-query: 0 automatic (tensor cores
                              when bf16, head_dim 128 and 8 <= G * n <= 128); 1 tensor cores; 2
                              split-KV passes.  Decode (tree_attn_decode_ex / _decode, bf16, head_dim
                              128): 0 automatic (tensor cores when G = 8, the split kernel otherwise);
                              1 tensor cores; 2 split kernel */
  int32_t split_tiles;     /* split-KV tile configuration.  0: automatic (short tiles when the mean
                              sequence is under 1024 tokens); 1: long tiles; 2: short tiles.
                              Shared-prefix calls with the tensor-core prefix pass: the suffix pass
                              runs on the short-unit kernel (one CTA per sample and KV head) when
                              head_dim is 128, there are at least as many (sample, KV head) units as
                              SMs and no suffix exceeds 2048 tokens, or always with 3 */
  int32_t debug_skip_stage; /* 0: off.  Test hook of the short-unit suffix kernel: s > 0 makes its
                              CTA 0 never load its key stage s - 1, so that stage's wait runs out */
  int32_t reserved[2];     /* must be 0 */
} ta_options;

/*
 * Build identity (no counterpart in the pages): a hash of every library source file and
 * public header, and of the compiler flags, that this binary was built from (static storage).
 * Lets a caller or a test check that the loaded library matches the sources it reads.
 */
const char* tree_attn_build_id(void);

/*
 * Profiling hook (no counterpart in the pages).  While set (non-NULL, on this host thread),
 * every call records `start` (a cudaEvent_t) on its stream immediately before the first launch
 * of its main kernel and `stop` immediately after the last one, so the caller can time that
 * kernel alone with cudaEventElapsedTime.  The main kernel is the split-KV kernel for decode
 * (contiguous or paged; every pass of a multi-query call), the tensor-core kernel for the
 * shared-prefix, multi-query tensor-core and context-encoding calls (the shared-prefix call's
 * suffix pass and every merge launch fall outside the span, except the merges between the
 * tensor-core launches of multi-query calls over more than 128 sequences).  NULL, NULL turns
 * it off.  The library never creates, waits on or destroys the events.
 */
void tree_attn_profile_events(void* start, void* stop);

/* A short English name of a status code (static storage). */
const char* tree_attn_status_string(ta_status status);

/* The cudaError_t of the most recent TA_ERR_CUDA on this host thread (0 if none). */
int32_t tree_attn_last_cuda_error(void);

/*
 * Workspace for tree_attn_decode_ex on the current device: a header (error word),
 * one merge ticket per (sequence, KV head) and the chunk partials
 * (grid + B*Hkv slots of G*(D+2) floats).  Writes the byte count to *bytes.
 * Same argument rules as tree_attn_decode_ex.
 */
ta_status tree_attn_workspace_size(const int64_t* seqlens, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                   int32_t head_dim, ta_dtype dtype, const ta_options* opts, size_t* bytes);

/*
 * Zero-fill a workspace on `stream`.  Required once before its first use and
 * after any call that reported TA_ERR_TIMEOUT; every successful call leaves the
 * tickets at zero again, so no per-call clearing is needed.
 */
ta_status tree_attn_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Exact decode attention, bf16 q/K/V, f32 out and lse.  Allocates its workspace
 * with cudaMallocAsync on `stream`, zero-fills it and frees it with cudaFreeAsync
 * on every call; tree_attn_decode_ex takes a caller-owned workspace instead.
 * `seqlens`: host array of `batch` lengths S_b >= 0.
 */
ta_status tree_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int64_t* seqlens,
                           int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale,
                           float* out, float* lse, void* stream);

/* The same for float32 q/K/V (all arithmetic is float32 on either path). */
ta_status tree_attn_decode_f32(const float* q, const float* k_cache, const float* v_cache, const int64_t* seqlens,
                               int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale,
                               float* out, float* lse, void* stream);

/*
 * Decode attention with a caller-owned workspace (no allocation; one kernel
 * launch per 128 sequences).  `workspace` must be 256-byte aligned, at least
 * tree_attn_workspace_size() bytes, zero-filled before first use, and not used
 * by two calls in flight at once.  `opts` may be NULL.  bf16 calls with head_dim
 * 128 and G = 8 query heads per KV head run on the tensor cores (the several-query
 * form of tree_attn_decode_multi_ex with one query token: a tcgen05 launch and a
 * merge launch per 128 sequences); ta_options.prefix_path selects the path.
 */
ta_status tree_attn_decode_ex(ta_dtype dtype, const void* q, const void* k_cache, const void* v_cache,
                              const int64_t* seqlens, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                              int32_t head_dim, float scale, float* out, float* lse, const ta_options* opts,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Several query tokens per sequence (speculative or multi-token decode), after the Star
 * Attention article (tiaojiaomugou.com, "How Star Attention cuts the cost of inference" and
 * "Phase 2: query encoding and token generation"): a short query of n tokens follows the
 * cached context, with the tokens' keys and values already written as the last n rows of each
 * sequence's cache, and each query token attends to all the context before it and to itself.
 * Query token j (0-based) of sequence b sits at position S_b - n + j and attends to the first
 * S_b - n + j + 1 keys (causal among the n new tokens).  n = 1 is tree_attn_decode.
 *   q    [B][n][Hq][D]  bf16 (or f32 with TA_F32)
 *   k, v packed per sequence as for tree_attn_decode; every S_b >= n, else TA_ERR_INVALID_ARG
 *   out  [B][n][Hq][D]  f32;  lse [B][n][Hq] f32
 * Two forms (ta_options.prefix_path).  Tensor cores (bf16, head_dim 128, G * n <= 128 with
 * G = n_q_heads / n_kv_heads): the G * n rows of a (sequence, KV head) form one matrix that
 * reads the cache once, S = Q K^T and O = P V on tcgen05, chunked over the SMs and merged
 * exactly.  Split-KV: one pass over the cache serves G * n' rows per KV head (n' consecutive
 * query tokens, a power of two, G * n' <= 8); larger n takes several passes, run in turn on
 * `stream` with one workspace.  Other rules as tree_attn_decode / tree_attn_decode_ex.
 */
ta_status tree_attn_multi_workspace_size(const int64_t* seqlens, int32_t batch, int32_t n_queries,
                                         int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, ta_dtype dtype,
                                         const ta_options* opts, size_t* bytes);

/* Multi-query decode with a caller-owned, zero-filled workspace (rules as tree_attn_decode_ex). */
ta_status tree_attn_decode_multi_ex(ta_dtype dtype, const void* q, const void* k_cache, const void* v_cache,
                                    const int64_t* seqlens, int32_t batch, int32_t n_queries, int32_t n_q_heads,
                                    int32_t n_kv_heads, int32_t head_dim, float scale, float* out, float* lse,
                                    const ta_options* opts, void* workspace, size_t workspace_bytes, void* stream);

/* Multi-query decode, bf16, allocating its workspace per call like tree_attn_decode. */
ta_status tree_attn_decode_multi(const void* q, const void* k_cache, const void* v_cache, const int64_t* seqlens,
                                 int32_t batch, int32_t n_queries, int32_t n_q_heads, int32_t n_kv_heads,
                                 int32_t head_dim, float scale, float* out, float* lse, void* stream);

/*
 * Bifurcated (shared-prefix) decode, after the bifurcated-attention summary
 * (briefgpt.xyz, 2403.08845, TL;DR): sample n's query attends over the
 * concatenation [prefix ; suffix_n] — one shared context prefilled once plus the
 * tokens that sample decoded — computed as a prefix part and a suffix part whose
 * softmax statistics are merged exactly.
 *   q        [N][Hq][D] bf16
 *   k_prefix, v_prefix  [Hkv][prefix_len][D] bf16 (one copy, shared by all samples)
 *   k_suffix, v_suffix  packed per sample like k/v above ([Hkv][S_n][D] blocks)
 *   suffix_lens         HOST array of N lengths >= 0
 *   out [N][Hq][D] f32, lse [N][Hq] f32
 * Allocates its workspace like tree_attn_decode.
 */
ta_status tree_attn_decode_bifurcated(const void* q, const void* k_prefix, const void* v_prefix, int64_t prefix_len,
                                      const void* k_suffix, const void* v_suffix, const int64_t* suffix_lens,
                                      int32_t n_samples, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                      float scale, float* out, float* lse, void* stream);

/* Workspace bytes for tree_attn_decode_bifurcated_ex (same argument rules). */
ta_status tree_attn_bifurcated_workspace_size(int64_t prefix_len, const int64_t* suffix_lens, int32_t n_samples,
                                              int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                              const ta_options* opts, size_t* bytes);

/* Bifurcated decode with a caller-owned, zero-filled workspace (rules as tree_attn_decode_ex). */
ta_status tree_attn_decode_bifurcated_ex(const void* q, const void* k_prefix, const void* v_prefix,
                                         int64_t prefix_len, const void* k_suffix, const void* v_suffix,
                                         const int64_t* suffix_lens, int32_t n_samples, int32_t n_q_heads,
                                         int32_t n_kv_heads, int32_t head_dim, float scale, float* out, float* lse,
                                         const ta_options* opts, void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * Decode attention that allocates nothing (no counterpart in the pages: it is a
 * deployment variant of tree_attn_decode, same bf16 inputs, same results).
 *
 * For callers that cannot allocate device memory while they run: serving
 * runtimes that carve all of HBM into their own pools at start-up and forbid
 * other allocations, or latency-critical paths where an allocation call may
 * block in the driver.  tree_attn_decode allocates its workspace per call and
 * tree_attn_decode_ex needs the caller to own one; this entry point instead uses
 * a fixed 4 MiB scratch array that the library keeps in device memory (every GPU
 * that loads the library holds it until the process exits).
 *
 * Each call made outside stream capture looks up that array's device address on
 * the current device (with that device current); a call inside a capture reuses the
 * address of the last uncaptured call on the device, so make one call on each
 * device before any stream capture.  Every call zero-fills the array's merge
 * tickets and error word on `stream` before its kernel runs.  All calls share the
 * one array, so calls that overlap on the GPU (two streams, two host threads) race
 * and must be serialised by the caller.  A problem whose workspace would exceed
 * 4 MiB (grid + B*Hkv partial slots of G*(D+2) floats, plus a ticket per sequence
 * and KV head) returns TA_ERR_SCRATCH_LIMIT before anything is launched.  Other
 * arguments and statuses as tree_attn_decode.  Device-side errors (a bounded wait
 * that ran out: the affected outputs are NaN) are recorded in the array's error
 * word, which tree_attn_noalloc_check reads.
 */
ta_status tree_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int64_t* seqlens,
                                   int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                   float scale, float* out, float* lse, void* stream);

/*
 * Synchronise `stream` and read the error word of tree_attn_decode_noalloc's scratch array
 * on the current device (no counterpart in the pages): TA_OK, TA_ERR_TIMEOUT if a bounded
 * wait inside the last call's kernel ran out (its affected outputs are NaN), or TA_ERR_CUDA.
 * Allocates nothing.  Like the calls themselves, it must not overlap another no-allocation
 * call on the device.
 */
ta_status tree_attn_noalloc_check(void* stream);

/*
 * Decode over a paged KV cache, after the attention-acceleration concept page
 * (compassingai.com, part 3 "PagedAttention (vLLM)"): the cache is cut into blocks of
 * `page_size` tokens, and a table maps each sequence's logical blocks to physical ones, which
 * sequences may share (a common prompt prefix, for example).
 *   k_pages, v_pages  [num_pages][Hkv][page_size][D] (bf16, or f32 with TA_F32): physical block
 *                     p holds page_size consecutive token rows of every KV head
 *   block_table       DEVICE int32 [B][block_table_stride]: sequence b's tokens
 *                     [i * page_size, (i + 1) * page_size) are rows 0.. of physical block
 *                     block_table[b * block_table_stride + i]; stride >= ceil(max S_b / page_size)
 *   page_size         a power of two >= 16 (TA_ERR_INVALID_ARG otherwise)
 * q, out, lse, seqlens, workspace (tree_attn_workspace_size applies unchanged) and the other
 * rules as tree_attn_decode_ex; bf16 calls with head_dim 128 and G = 8 run on the paged
 * tensor-core form (as tree_attn_decode_multi_paged_ex with one query token; prefix_path
 * selects the path).  Every entry a sequence uses is checked against num_pages on
 * the device before anything is read through it: an entry outside [0, num_pages) makes
 * tree_attn_check report TA_ERR_BAD_PAGE and the affected outputs NaN.
 */
ta_status tree_attn_decode_paged_ex(ta_dtype dtype, const void* q, const void* k_pages, const void* v_pages,
                                    int64_t num_pages, int32_t page_size, const int32_t* block_table,
                                    int64_t block_table_stride, const int64_t* seqlens, int32_t batch,
                                    int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale, float* out,
                                    float* lse, const ta_options* opts, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * Several query tokens per sequence (tree_attn_decode_multi_ex) over a paged cache
 * (tree_attn_decode_paged_ex): q, out, lse and the query-token rules of the first, pages,
 * block table and page rules of the second.  Workspace: tree_attn_multi_workspace_size.  The
 * tensor-core form reads each 128-key tile as one TMA box per page segment it spans.
 */
ta_status tree_attn_decode_multi_paged_ex(ta_dtype dtype, const void* q, const void* k_pages, const void* v_pages,
                                          int64_t num_pages, int32_t page_size, const int32_t* block_table,
                                          int64_t block_table_stride, const int64_t* seqlens, int32_t batch,
                                          int32_t n_queries, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          float scale, float* out, float* lse, const ta_options* opts,
                                          void* workspace, size_t workspace_bytes, void* stream);

/* Paged decode, bf16, allocating its workspace per call like tree_attn_decode. */
ta_status tree_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, int64_t num_pages,
                                 int32_t page_size, const int32_t* block_table, int64_t block_table_stride,
                                 const int64_t* seqlens, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                 int32_t head_dim, float scale, float* out, float* lse, void* stream);

/*
 * Merge of sequence-sharded decode results, after the Tree Attention article (m.srwj168.com.cn,
 * "The energy view of attention": max and logsumexp are associative, so the pieces each
 * device computes over its slice of the cache combine exactly, in any order; across devices,
 * a tree all-reduce) and the query host of Star Attention's phase 2.  Given the (out_s, lse_s)
 * that a tree_attn_decode* call computed over shard s of every sequence's cache (the same
 * rows in every shard), writes the result over the whole cache:
 *   out = sum_s w_s out_s / sum_s w_s,  w_s = exp(lse_s - max_s lse_s),  lse = max + ln sum_s w_s
 * with both sums over s in a fixed pairwise tree (bit-identical across calls).  A shard whose
 * lse is -inf (no token) contributes nothing; all shards empty give out = 0, lse = -inf; a NaN
 * lse in any shard gives NaN.
 *   outs  DEVICE f32 [n_shards][rows][head_dim]    lses  DEVICE f32 [n_shards][rows]
 *   out   DEVICE f32 [rows][head_dim]              lse   DEVICE f32 [rows]
 * rows = B * Hq (times n for multi-query results); 1 <= n_shards <= 65536, else
 * TA_ERR_INVALID_ARG.  No workspace; asynchronous on `stream`.
 */
ta_status tree_attn_merge_shards(const float* outs, const float* lses, int32_t n_shards, int64_t rows,
                                 int32_t head_dim, float* out, float* lse, void* stream);

/*
 * Context encoding with anchor blocks, after the Star Attention article (tiaojiaomugou.com,
 * "Two-phase inference under Star Attention", "Phase 1: context encoding"): the context is cut
 * into blocks of `block_size` tokens, every block after the first is prefixed with the first
 * block (the anchor block), and each block attends causally over [anchor ; itself].  Exact
 * softmax attention under that mask, for every position p of one context of `seq_len` tokens:
 * with i = p / block_size, position p attends to keys [0, p] when i = 0 and to keys
 * [0, block_size) and [i * block_size, p] when i > 0 (query head h reads KV head h / G).
 *   q    [seq_len][Hq][D] bf16        k, v  [Hkv][seq_len][D] bf16
 *   out  [seq_len][Hq][D] f32 (16-byte aligned)   lse [seq_len][Hq] f32
 * Supported: head_dim 128, G = Hq / Hkv in {1, 2, 4, 8}, block_size a positive multiple of 128,
 * Hkv * seq_len < 2^31; others -> TA_ERR_UNSUPPORTED.  A block_size >= seq_len is plain causal
 * attention.  Runs on the tensor cores (tcgen05): one CTA per (query tile of 128 / G positions x
 * G heads, KV head), S = Q K^T and O = P V with TMEM accumulators over the tile's anchor and own
 * keys.  `workspace`: at least 256 bytes, 256-byte aligned, zero-filled before first use (its
 * first word is the error word tree_attn_check reads: a bounded wait that ran out makes the
 * affected rows NaN).  Other rules (options, statuses, asynchrony) as tree_attn_decode_ex.
 */
ta_status tree_attn_anchor_prefill(const void* q, const void* k, const void* v, int64_t seq_len, int64_t block_size,
                                   int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale, float* out,
                                   float* lse, const ta_options* opts, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * Synchronise `stream` and read the workspace's error word: TA_OK, or
 * TA_ERR_TIMEOUT if a kernel's bounded wait ran out since the workspace was
 * last initialised (the affected outputs are NaN), TA_ERR_BAD_PAGE (paged decode, above),
 * or TA_ERR_CUDA.
 */
ta_status tree_attn_check(const void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TREE_ATTN_H */
