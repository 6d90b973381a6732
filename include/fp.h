/*
 * fp.h -- C ABI of the B200 (sm_100a) FlashPrefill-style block-sparse causal prefill library
 *         (libfp.so).
 *
 * The method (FlashPrefill, "Instantaneous Pattern Discovery and Thresholding for Ultra-Fast
 * Long-Context Prefilling"):
 *   1. pool     mean-pool Q and K over B-token blocks (skill summary page, "Stage 1: Block-Level
 *               Attention Approximation"; "Architecture Overview": "average-pooled keys/queries");
 *   2. search   pooled block scores s_ij = qbar_i . kbar_j / sqrt(d) (same section), causal softmax
 *               p_ij over j <= i, keep block j iff p_ij >= tau * max_j p_ij ("Core Concept" item 3,
 *               "Dynamic Thresholding": one max reduction, no sorting or cumulative sums); the sink
 *               block 0 and the diagonal block i are always kept; kept blocks are written as
 *               ascending per-(head, query block) index lists ("Physical Index Jumping");
 *   3. attend   block-sparse causal flash attention over exactly the listed blocks, online softmax
 *               (FlashPrefill V2 abstract: block-sparse prefill attention operator).
 * A dense causal kernel built the same way is the baseline (FlashPrefill V2 abstract: "dense
 * baseline").
 *
 * Conventions shared by every call
 *   - Tensors are row-major [tokens, heads, head_dim]; Q has num_q_heads heads, K and V have
 *     num_kv_heads heads; q-head h reads kv-head h / (num_q_heads / num_kv_heads) (GQA).
 *     Q, K, V and O hold bf16 bit patterns (2 bytes per element).
 *   - Several sequences may be packed along tokens (varlen): device cu_seqlens[s]..cu_seqlens[s+1]
 *     is sequence s. Each sequence is causal on its own (query position == key position space, no
 *     cached prefix); blocks, the sink block and block ids restart at every sequence.
 *   - Block b of a sequence of length L spans local tokens [b*B, min((b+1)*B, L)); nb = ceil(L/B).
 *     Global block id of (sequence s, local block i) = sum_{s'<s} nb_{s'} + i.
 *   - Pooled tensors: float32 [total_blocks, heads, head_dim].
 *   - counts: int32 [num_q_heads, total_blocks]: number of kept blocks of row (h, global block).
 *   - indices: int32, triangular-packed: row (s, h, i) starts at
 *         base_s + h * nb_s*(nb_s+1)/2 + i*(i+1)/2,   base_s = sum_{s'<s} Hq * nb_{s'}(nb_{s'}+1)/2,
 *     has room for i+1 entries, and holds the kept LOCAL block ids in ascending order.
 *     fp_problem.index_elems is the buffer length in int32 elements.
 *   - The caller owns every buffer. The library never allocates or frees device memory and never
 *     synchronises: every call only enqueues kernels on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream). Pointers marked "device" must be device-accessible and 16-byte
 *     aligned.
 *   - Host-side checks run before any launch; a non-OK status means nothing was enqueued, and
 *     fp_last_error() describes the problem. FP_ERR_CUDA means a launch failed.
 *   - dev_status (optional, device int32, may be NULL): kernels OR FP_DEV_* bits into it when a
 *     bounded wait gives up or an index entry is out of range (the entry is skipped). Read it
 *     after the stream has completed. Kernels never trap.
 */
#ifndef FP_H_
#define FP_H_

#include <stdint.h>

#if defined(__GNUC__)
#define FP_API __attribute__((visibility("default")))
#else
#define FP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp_status {
  FP_OK = 0,
  FP_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer, non-finite tau, ... */
  FP_ERR_UNSUPPORTED = 2,  /* valid but not implemented here (head_dim != 128, B not 64/128) */
  FP_ERR_CUDA = 3,         /* a CUDA launch or driver call failed */
  FP_ERR_TIMEOUT = 4       /* fp_check_device_status: a kernel's bounded wait gave up (FP_DEV_TIMEOUT) */
} fp_status;

/* Bits written into dev_status by the kernels. */
#define FP_DEV_TIMEOUT 1     /* a bounded mbarrier wait gave up; outputs of that launch are undefined */
#define FP_DEV_BAD_LIST 2    /* an index-list entry or count was out of range and was skipped/clamped */
#define FP_DEV_BAD_PROBLEM 4 /* device cu_seqlens disagree with the sizes in fp_problem */

#define FP_MAX_SEQS 1024     /* maximum number of packed sequences per call */

/* Shared description of one prefill problem. Fill it with fp_problem_init. */
typedef struct fp_problem {
  const int32_t* cu_seqlens; /* device, [num_seqs+1], cu_seqlens[0] = 0, non-decreasing */
  int32_t num_seqs;          /* 1 .. FP_MAX_SEQS */
  int32_t total_tokens;      /* cu_seqlens[num_seqs] */
  int32_t total_blocks;      /* sum_s ceil(L_s / B) */
  int32_t max_seq_blocks;    /* max_s ceil(L_s / B) */
  int64_t index_elems;       /* int32 entries of the triangular index buffer */
  int32_t num_q_heads;       /* Hq, a multiple of num_kv_heads */
  int32_t num_kv_heads;      /* Hkv */
  int32_t head_dim;          /* d; 128 is supported */
  int32_t block_size;        /* B; 64 or 128 */
  int32_t* sched;            /* optional work counter of the attention calls, see below; NULL after init */
  void* key_split;           /* optional search scratch (the pooled keys split for the tensor cores), see
                                below; NULL after init */
  int64_t key_split_bytes;   /* its size in bytes */
} fp_problem;

/* Work counter. fp_problem_init leaves sched NULL: an attention launch then gives each CTA a fixed
 * share of the (q-head pair, 128-row query tile) units, balanced for causal-dense lists. A caller
 * may point sched at FP_SCHED_WORDS device int32 that hold zero: each CTA then takes its next unit
 * from the counter when it is free, so the work stays balanced whatever the lists' lengths. Every
 * launch leaves the words at zero again, so the same words serve any number of launches (and CUDA
 * graph replays) that run one after another; two launches that may run at the same time (other
 * streams, no ordering between them) must not share them. The results are identical either way.
 * fp_sparse_prefill(_noalloc) use words inside their workspace and ignore sched. */
#define FP_SCHED_WORDS 2

/* Key split. The block search scores pooled keys on the tensor cores as bf16 hi + lo halves (step 2
 * below). fp_problem_init leaves key_split NULL: each search tile then splits the pooled keys it reads
 * itself (every tile of a kv-head splits the same keys again). A caller may point key_split at
 * key_split_bytes >= fp_key_split_bytes(p, cache) bytes of device memory (256-byte aligned, contents
 * scratch): fp_block_search (and the fused and paged searches) then split every pooled key once per
 * call, into that buffer, before the search kernel reads them. The lists are the same either way
 * (the split and the error bound of each key are). Calls that may run at the same time must not share
 * the buffer. cache: NULL for the plain problem, or the paged-cache description the search will use
 * (whose pooled keys include the cached prefixes). fp_sparse_prefill(_noalloc) keep theirs in the
 * workspace. Host-only. */
struct fp_paged_cache;
FP_API fp_status fp_key_split_bytes(const fp_problem* p, const struct fp_paged_cache* cache, int64_t* bytes);

/* Length, in int32 entries, of the index buffer of a problem: sum_s Hq * nb_s (nb_s + 1) / 2 with
 * nb_s = ceil(L_s / block_size) (the triangular layout above: query block i of a sequence keeps at
 * most its i + 1 causal blocks). host_seqlens: HOST array of the num_seqs sequence LENGTHS L_s (not
 * cumulative offsets), read only during the call. The same value is stored by fp_problem_init in
 * fp_problem.index_elems; this call gives it to a caller that sizes buffers before it has a device
 * cu_seqlens. Host-only, nothing is enqueued. FP_ERR_INVALID_ARG for a NULL pointer, num_seqs outside
 * [1, FP_MAX_SEQS], a negative length or num_q_heads < 1; FP_ERR_UNSUPPORTED for block_size other
 * than 64 or 128. */
FP_API fp_status fp_index_buffer_elems(const int32_t* host_seqlens, int32_t num_seqs, int32_t block_size,
                                       int32_t num_q_heads, int64_t* out_elems);

/* Status of the device work behind a dev_status word that the caller read back after the stream
 * completed: FP_OK for 0; FP_ERR_TIMEOUT when FP_DEV_TIMEOUT is set (a bounded wait gave up and
 * that launch's outputs are undefined); otherwise FP_ERR_INVALID_ARG when FP_DEV_BAD_LIST or
 * FP_DEV_BAD_PROBLEM is set (device-side inputs disagreed with the problem: index entries out of
 * range, cu_seqlens or prefix lengths that differ from the host copies). fp_last_error() then names
 * every bit that was set. Host-only, nothing is enqueued. */
FP_API fp_status fp_check_device_status(int32_t dev_status_bits);

/* Fill *p from a HOST copy of cu_seqlens (read only during the call) and the device copy that the
 * kernels will read. Checks sizes and the sequence limits. */
FP_API fp_status fp_problem_init(fp_problem* p, const int32_t* host_cu_seqlens, int32_t num_seqs,
                          const int32_t* dev_cu_seqlens, int32_t num_q_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t block_size);

/* Step 1 -- block mean pooling (FlashPrefill skill summary page, "Stage 1").
 * q: device bf16 [total_tokens, Hq, d]; k: device bf16 [total_tokens, Hkv, d].
 * q_pool: device float32 [total_blocks, Hq, d]; k_pool: device float32 [total_blocks, Hkv, d].
 * The mean of a partial last block is over the tokens it holds. */
FP_API fp_status fp_block_pool(const fp_problem* p, const void* q, const void* k, float* q_pool, float* k_pool,
                        void* stream);

/* Step 2 -- pooled block scores, causal softmax, max-based threshold, index emission
 * (FlashPrefill skill summary page, "Stage 1" and "Core Concept" item 3; "Physical Index Jumping").
 * Keeps block j of row (h, i) iff exp(s_ij - max_j s_ij) >= tau (equal to p_ij >= tau * max_j p_ij),
 * plus j = 0 and j = i. tau <= 0 keeps every causal block; tau must be finite.
 * q_pool/k_pool: outputs of fp_block_pool. counts: device int32 [Hq, total_blocks];
 * indices: device int32 [index_elems] (entries past a row's count are left untouched). */
FP_API fp_status fp_block_search(const fp_problem* p, const float* q_pool, const float* k_pool, float tau,
                          int32_t* counts, int32_t* indices, int32_t* dev_status, void* stream);

/* Comparison selector (not the method: the one its threshold replaces). Cumulative top-p block
 * selection on the same pooled scores (FlashPrefill skill summary page, "The Problem": Top-k /
 * Top-p need score computation, sorting and cumulative sums; FlexPrefill abstract,
 * "Cumulative-Attention Based Index Selection"): row (h, i) keeps block j iff the softmax mass of
 * the blocks strictly more probable than j is below gamma (blocks tied at the cut together), plus
 * j = 0 and j = i. gamma <= 0 keeps those two only, gamma >= 1 every causal block; gamma finite.
 * It needs a whole row of scores before any decision: scores is a device float32 scratch of
 * index_elems entries (the pooled score matrix, laid out like the index lists) written and read
 * by the call. counts / indices as for fp_block_search. */
FP_API fp_status fp_block_search_topp(const fp_problem* p, const float* q_pool, const float* k_pool, float gamma,
                                      float* scores, int32_t* counts, int32_t* indices, int32_t* dev_status,
                                      void* stream);

/* Steps 1 + 2 in one call: fp_block_pool followed by fp_block_search on the same stream (two
 * launches: Q and K are streamed once by the pool kernel at HBM bandwidth; the search kernel
 * then computes the block scores, the threshold and the lists without materialising scores).
 * q_pool and k_pool are required outputs (the pooled tensors). */
FP_API fp_status fp_block_pool_search(const fp_problem* p, const void* q, const void* k, float tau, float* q_pool,
                               float* k_pool, int32_t* counts, int32_t* indices, int32_t* dev_status,
                               void* stream);

/* Step 3 -- block-sparse causal attention over the listed blocks (online softmax, bf16 in,
 * fp32 accumulate, bf16 out). counts/indices as written by fp_block_search (any ascending lists
 * of local block ids <= i are accepted; out-of-range entries are skipped and flagged).
 * softmax_scale <= 0 selects 1/sqrt(d). out: device bf16 [total_tokens, Hq, d].
 * lse (optional, may be NULL): device float32 [Hq, total_tokens], natural-log sum of
 * exp(softmax_scale * q.k) over the attended keys.
 * For B = 128 two kernels are launched on `stream`, one per attention schedule (two adjacent query
 * tiles of one head per unit, or one tile per unit); each first sums the list counts, and the one
 * not chosen returns at once (single tiles when fewer than 40% of the causal blocks are kept). The
 * choice depends on the lists alone, so a call is deterministic; the two schedules add the fp32
 * softmax terms in different orders, both within the same tolerance of exact attention. */
FP_API fp_status fp_block_sparse_attn(const fp_problem* p, const void* q, const void* k, const void* v,
                               const int32_t* counts, const int32_t* indices, float softmax_scale, void* out,
                               float* lse, int32_t* dev_status, void* stream);

/* Dense causal attention (every causal block), same kernel design; the baseline for the speedup. */
FP_API fp_status fp_dense_attn(const fp_problem* p, const void* q, const void* k, const void* v, float softmax_scale,
                        void* out, float* lse, int32_t* dev_status, void* stream);

/* FP8 attention (FlashPrefill V2 abstract: FP8 inference). Q and K hold e4m3 codes (OCP E4M3, one
 * byte per element, row-major [tokens, heads, head_dim], dequantised value = q_scale * code value,
 * resp. k_scale; per-tensor scales, finite and positive); V, P and O stay bf16. Q K^T runs on the
 * tensor cores in e4m3 (tcgen05 kind::f8f6f4) with fp32 accumulation; the logits are
 * softmax_scale * q_scale * k_scale * (q . k), softmax_scale <= 0 selecting 1/sqrt(d).
 * counts / indices / out / lse / dev_status as for fp_block_sparse_attn (lists from any search,
 * e.g. fp_block_search on the bf16 Q and K the e4m3 codes were quantised from). Plain prefill
 * only (no paged-cache variant). */
FP_API fp_status fp_block_sparse_attn_fp8(const fp_problem* p, const void* q_e4m3, const void* k_e4m3, const void* v,
                                          float q_scale, float k_scale, const int32_t* counts, const int32_t* indices,
                                          float softmax_scale, void* out, float* lse, int32_t* dev_status,
                                          void* stream);

/* Dense causal FP8 attention (every causal block), the FP8 baseline. */
FP_API fp_status fp_dense_attn_fp8(const fp_problem* p, const void* q_e4m3, const void* k_e4m3, const void* v,
                                   float q_scale, float k_scale, float softmax_scale, void* out, float* lse,
                                   int32_t* dev_status, void* stream);

/* FP8 attention with per-block scales (FlashPrefill V2 abstract: FP8 inference): as
 * fp_block_sparse_attn_fp8, but the dequantised value of q[t, h, :] is 2^q_exp[b, h] * code and of
 * k[t, g, :] is 2^k_exp[b, g] * code, where b is the global block of token t (block_size tokens,
 * restarting at every sequence, numbered as for the pooled tensors). q_exp: device int8
 * [total_blocks, Hq]; k_exp: device int8 [total_blocks, Hkv]; exponents within [-64, 64]. Power-of-
 * two scales, one per block and head (as in the microscaling formats), follow the range of each
 * block's values while every dequantised value stays exact in bf16 and fp32. The logits are
 * softmax_scale * 2^(q_exp + k_exp) * (q_code . k_code). NULL exponent arrays are invalid. */
FP_API fp_status fp_block_sparse_attn_fp8_blockscaled(const fp_problem* p, const void* q_e4m3, const void* k_e4m3,
                                                      const void* v, const int8_t* q_exp, const int8_t* k_exp,
                                                      const int32_t* counts, const int32_t* indices,
                                                      float softmax_scale, void* out, float* lse, int32_t* dev_status,
                                                      void* stream);

/* Dense causal FP8 attention with per-block scales. */
FP_API fp_status fp_dense_attn_fp8_blockscaled(const fp_problem* p, const void* q_e4m3, const void* k_e4m3,
                                               const void* v, const int8_t* q_exp, const int8_t* k_exp,
                                               float softmax_scale, void* out, float* lse, int32_t* dev_status,
                                               void* stream);

/* Bytes of workspace fp_sparse_prefill needs for this problem: the pooled Q and K, the counts, the
 * index lists and the attention's work counter (FP_SCHED_WORDS int32), each 256-byte aligned. */
FP_API fp_status fp_sparse_prefill_workspace(const fp_problem* p, int64_t* bytes);

/* The whole sparse prefill in one call (FlashPrefill: block pooling, max-based block search and
 * block-sparse attention): fp_block_pool, fp_block_search and fp_block_sparse_attn on `stream`,
 * with the intermediate tensors in `workspace` (device, 256-byte aligned, at least
 * fp_sparse_prefill_workspace bytes; its contents are scratch and are overwritten; the work counter
 * inside it is zeroed by an asynchronous memset on `stream` before the attention launch, and
 * p->sched is not used). out / lse / softmax_scale / dev_status as for fp_block_sparse_attn. */
FP_API fp_status fp_sparse_prefill(const fp_problem* p, const void* q, const void* k, const void* v, float tau,
                            float softmax_scale, void* workspace, int64_t workspace_bytes, void* out, float* lse,
                            int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Chunked prefill onto a paged key/value cache (FlashPrefill V2 abstract: paged KV cache and
 * continuous batching in a serving engine). The pages give no interface; this one keeps the method
 * unchanged and only moves where the keys come from:
 *   - fp_problem describes the new query tokens of this call (the chunk): cu_seqlens over the
 *     chunk's queries, L_s of them for sequence s, and Q is [total_tokens, Hq, d] as before.
 *   - Sequence s already holds prefix_lens[s] tokens in the cache (a multiple of block_size), and
 *     the caller has written the chunk's own keys and values into the cache too: the keys of s are
 *     its prefix_lens[s] + L_s cached tokens, and the chunk's query at local position t sits at key
 *     position prefix_lens[s] + t (causal: it attends keys 0 .. prefix_lens[s] + t).
 *   - Blocks restart at every sequence's key position 0: the chunk's query block i is key block
 *     pb_s + i (pb_s = prefix_lens[s] / block_size), and its list keeps key blocks 0 .. pb_s + i
 *     (sink block 0 and its diagonal pb_s + i are always kept). The prefix is therefore attended
 *     block-sparsely like the rest of the sequence, with pooled keys computed from the cache.
 *   - The cache: k_cache and v_cache are device bf16 [num_pages * page_size, Hkv, d] (pages of
 *     page_size consecutive token rows). Key token u of sequence s lives in page
 *     block_table[s * max_pages + u / page_size] at row u % page_size. page_size must be a
 *     multiple of block_size, so a key block never straddles pages. Block-table entries outside
 *     [0, num_pages) make the kernels skip that key block and flag FP_DEV_BAD_PROBLEM.
 *   - Pooled keys: float32 [total_kv_blocks, Hkv, d], key block j of sequence s at global key
 *     block sum_{s'<s}(pb_{s'} + nb_{s'}) + j. Pooled queries, counts: as for fp_block_pool /
 *     fp_block_search (per query block of the chunk).
 *   - indices: row (s, h, i) starts at base_s + h * (nb_s*pb_s + nb_s*(nb_s+1)/2) + i*pb_s + i*(i+1)/2,
 *     base_s = sum_{s'<s} Hq * (nb*pb + nb(nb+1)/2), and has room for pb_s + i + 1 entries (the
 *     triangular layout above when every prefix is 0). fp_paged_cache.index_elems is its length.
 * With every prefix 0 and the pages holding the sequences in order, these calls compute exactly
 * what the plain calls compute. */
typedef struct fp_paged_cache {
  const int32_t* prefix_lens; /* device [num_seqs] */
  const int32_t* block_table; /* device [num_seqs, max_pages] */
  int32_t max_pages;          /* row length of block_table */
  int32_t page_size;          /* token rows per page; a multiple of block_size */
  int32_t num_pages;          /* pages in k_cache / v_cache */
  int32_t total_kv_blocks;    /* sum_s (pb_s + nb_s) */
  int64_t index_elems;        /* int32 entries of the index buffer */
} fp_paged_cache;

/* Fill *c for problem p (the chunk) from HOST copies of cu_seqlens and prefix_lens (read only during
 * the call) and the device arrays the kernels read. Checks alignment of every prefix to block_size,
 * page_size, and that max_pages covers every sequence's prefix + chunk. */
FP_API fp_status fp_paged_cache_init(fp_paged_cache* c, const fp_problem* p, const int32_t* host_cu_seqlens,
                                     const int32_t* host_prefix_lens, const int32_t* dev_prefix_lens,
                                     const int32_t* dev_block_table, int32_t max_pages, int32_t page_size,
                                     int32_t num_pages);

/* Step 1 for a chunk: q_pool [total_blocks, Hq, d] from the chunk's q; k_pool [total_kv_blocks, Hkv, d]
 * from every key block of every sequence in k_cache. */
FP_API fp_status fp_paged_block_pool(const fp_problem* p, const fp_paged_cache* c, const void* q,
                                     const void* k_cache, float* q_pool, float* k_pool, void* stream);

/* Step 2 for a chunk: as fp_block_search, with row (s, h, i) scoring key blocks 0 .. pb_s + i. */
FP_API fp_status fp_paged_block_search(const fp_problem* p, const fp_paged_cache* c, const float* q_pool,
                                       const float* k_pool, float tau, int32_t* counts, int32_t* indices,
                                       int32_t* dev_status, void* stream);

/* Step 3 for a chunk: block-sparse causal attention of the chunk's queries over the listed key
 * blocks of the cache (lists of key block ids <= pb_s + i). out / lse as for fp_block_sparse_attn
 * (over the chunk's tokens). */
FP_API fp_status fp_paged_block_sparse_attn(const fp_problem* p, const fp_paged_cache* c, const void* q,
                                            const void* k_cache, const void* v_cache, const int32_t* counts,
                                            const int32_t* indices, float softmax_scale, void* out, float* lse,
                                            int32_t* dev_status, void* stream);

/* Dense causal attention of the chunk's queries over all their keys in the cache. */
FP_API fp_status fp_paged_dense_attn(const fp_problem* p, const fp_paged_cache* c, const void* q,
                                     const void* k_cache, const void* v_cache, float softmax_scale, void* out,
                                     float* lse, int32_t* dev_status, void* stream);

/* fp_validate_lists for chunk lists: count in [1, pb_s+i+1], ascending entries in [0, pb_s+i],
 * first 0, last pb_s + i. */
FP_API fp_status fp_paged_validate_lists(const fp_problem* p, const fp_paged_cache* c, const int32_t* counts,
                                         const int32_t* indices, int32_t* dev_status, void* stream);

/* Largest intermediate size (bytes) fp_sparse_prefill_noalloc handles: 64 MiB. */
#define FP_NOALLOC_MAX_BYTES (64ll << 20)

/* fp_sparse_prefill for callers that cannot allocate device memory (the method on the pages has no
 * counterpart: this is a library convenience). Serving loops that plan all device memory up front,
 * plugin hosts that give an operator no workspace, and code that cannot afford cudaMalloc's implicit
 * device synchronisation can call this instead: the intermediates live in a static array of
 * FP_NOALLOC_MAX_BYTES in the library's device image, and nothing is allocated by the call.
 * Every GPU that loads the library holds that array until the process exits. All calls on a device
 * share it and it keeps the last call's contents (nothing needs to start at zero); calls that overlap
 * on the GPU (other streams or threads) race on it. The first call on a device looks up the array's
 * address with that device current: make it before any stream capture. The address is cached for the
 * device's current context; after the context is destroyed and created again (cudaDeviceReset), the
 * next call looks it up again and, like the first, belongs outside stream capture. Problems whose intermediates
 * (fp_sparse_prefill_workspace) exceed FP_NOALLOC_MAX_BYTES return FP_ERR_INVALID_ARG.
 * Arguments as for fp_sparse_prefill, without the workspace. */
FP_API fp_status fp_sparse_prefill_noalloc(const fp_problem* p, const void* q, const void* k, const void* v,
                                    float tau, float softmax_scale, void* out, float* lse, int32_t* dev_status,
                                    void* stream);

/* Device-side check of index lists: every row's count in [1, i+1], entries ascending, in [0, i],
 * first entry 0 and last entry i. Violations OR FP_DEV_BAD_LIST into dev_status (required). */
FP_API fp_status fp_validate_lists(const fp_problem* p, const int32_t* counts, const int32_t* indices,
                            int32_t* dev_status, void* stream);

/* Self-test of the attention softmax's two exp2 paths (a repository test hook; the pages have no
 * counterpart): for i < n, y_poly[i] = the FMA-pipe polynomial 2^x[i] (degree-3 minimax on the
 * fractional part, inputs below -126 clamped) and y_mufu[i] = the hardware ex2.approx 2^x[i].
 * x, y_poly, y_mufu: device float32 [n]. */
FP_API fp_status fp_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n, void* stream);

/* Message for the last non-OK status returned on this thread (never NULL). */
FP_API const char* fp_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
FP_API int32_t fp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP_H_ */
