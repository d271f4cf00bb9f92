/*
 * qsa.h -- C ABI of the B200 (sm_100a) Qwen Sparse Attention library (libqsa.so).
 *
 * The method (sources on the pages):
 *   - "Long context became an architecture problem", section "Linear attention carries
 *     the stream; sparse attention retrieves detail": a small indexer scores compressed
 *     key blocks and picks the relevant ones; the budget is 512 blocks (2,048 tokens);
 *     the final incomplete block stays uncompressed.
 *   - axbrief "unsloth Qwen3.8-Flash-Next GGUF", section "Shifting from Tokens to
 *     Micro-Blocks": micro-block processing; 24 query heads paired with 2 KV heads.
 *   - "Qwen3.8-Flash-Next Previews Qwen4.x Architecture", FAQ: 4-token micro-blocks.
 *   - aiany.app "Qwen3.8-Flash-Next", "Key Capabilities": the indexer is MQA.
 *   - aiany.app, "Implementation notes": KV cache sizing for very long contexts.
 * Parameters the pages leave open, fixed here: head_dim 128; a block's compressed key is
 * the fp32 mean of its 4 per-token indexer keys (summed in token order, stored as bf16
 * round-to-nearest-even); 16 indexer query heads of width 64 sharing one key head; score
 * s(t,b) = sum_h w[t,h] * ReLU(q_idx[t,h] . kbar[b]); one block selection per token for all
 * 24 heads; top-k ties go to the lower block index.
 *
 * Per sequence, token t (0-based) may select among the complete blocks 0 .. floor(t/4)-1
 * (strictly before its own block, even when its own block is complete), keeps the
 * min(k, floor(t/4)) best, and attends to their 4k tokens plus its own block's tokens
 * 4*floor(t/4) .. t, with one softmax (scale 1/sqrt(128)); query head h reads KV head h/12.
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers, 16-byte aligned, contiguous, row-major in
 *     the layouts stated, owned by the caller.  The library never allocates device memory;
 *     scratch space is the caller's `workspace` (size from the *_workspace_size query).
 *     The one exception is qsa_decode_noalloc below: its scratch is a static device array
 *     of QSA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 *     library holds until the process exits.
 *   - `h_*` arguments are HOST pointers read synchronously during the call.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and the call returns
 *     without synchronising.  Host-detectable errors are returned before anything is
 *     enqueued.  Device-side failures (a bounded wait that timed out, an index out of
 *     range) are recorded in the first 16 bytes of the workspace and reported by
 *     qsa_last_device_error().
 *   - bf16 means IEEE bfloat16 (raw 16-bit); fp32 is IEEE single.
 *   - Calls are re-entrant; the only global state is the cached driver entry point for
 *     tensor-map encoding, and, for qsa_decode_noalloc, its static scratch array and the
 *     per-device address of that array.  Concurrent calls must not share a workspace.
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

struct CUstream_st;
typedef struct CUstream_st *qsa_stream_t;   /* same object as a cudaStream_t */

#define QSA_NUM_HEADS 24
#define QSA_NUM_KV_HEADS 2
#define QSA_HEAD_DIM 128
#define QSA_IDX_HEADS 16
#define QSA_IDX_DIM 64
#define QSA_BLOCK 4
#define QSA_MAX_TOPK 1024          /* largest supported budget k (the pages use 512) */
#define QSA_MAX_SEQ_LEN 1048576    /* longest supported sequence / cache, in tokens */
#define QSA_WS_HEADER_BYTES 256    /* status words at the start of every workspace */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad lengths */
  QSA_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte aligned */
  QSA_ERR_CAPACITY = 3,      /* an append would exceed the cache capacity */
  QSA_ERR_WORKSPACE = 4,     /* workspace too small */
  QSA_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed (launch, tensor map) */
  QSA_ERR_TIMEOUT = 6,       /* device: a bounded wait gave up */
  QSA_ERR_DEVICE = 7,        /* device: an out-of-range index was found and skipped */
  QSA_ERR_UNSUPPORTED = 8    /* valid request outside this build's limits */
} qsa_status;

typedef struct {
  int32_t topk_blocks;     /* budget k in blocks, 1..QSA_MAX_TOPK (512 on the pages) */
  int32_t rows_per_tile;   /* prefill attention: query tokens packed into one 128-row
                              tensor-core tile (1..10); 0 = library default */
  int32_t decode_splits;   /* decode attention: key splits per (sequence, KV head), 1..64;
                              0 = library default (one wave of CTAs: SMs / (2 x batch)) */
  int32_t score_chunk_rows;/* prefill: query rows scored per pass (bounds the score
                              buffer in the workspace); 0 = library default */
  int32_t debug_fault;     /* testing only; 0 in normal use.  1: in the prefill attention the
                              last tile's KV head 0 posts nothing for its first key chunk and
                              that tile's MMA waits give up after 1 ms, so the call's device
                              status reads QSA_ERR_TIMEOUT (site 23) and that tile's output is
                              undefined.  It exercises the bounded-wait unwind (copies in
                              flight drained, tensor memory freed): a normal call may follow at
                              once.  Other values are refused (QSA_ERR_INVALID_ARG). */
  int32_t select_mode;     /* prefill selection.  0 (default): the indexer writes each score row
                              and the top-k reads it twice (a first-digit histogram, then the
                              candidates).  1: the indexer also counts each row's first-digit
                              histogram in shared memory and finds its threshold bin, so the
                              top-k reads each row once (rows of fewer than 65,536 candidate
                              blocks; longer ones take mode 0).  The same selection either way;
                              mode 1 measured slower (its shared-memory counting slows the
                              indexer's epilogue).  Other values: QSA_ERR_INVALID_ARG. */
} qsa_params;

/* KV cache for decode.  Blocks of 4 tokens are contiguous per (sequence, KV head):
 *   k_blocks, v_blocks : bf16 [batch][2][capacity/4][4][128]   (1 KB per block)
 *   kbar               : bf16 [batch][capacity/4][64]          compressed indexer keys
 *   kbar_partial       : fp32 [batch][64]  running sum of the current incomplete block
 *   len                : int32 [batch]     tokens stored per sequence (device)
 * capacity is a multiple of 4, at most QSA_MAX_SEQ_LEN.  All buffers are caller-owned;
 * zero-initialise len before the first append. */
typedef struct {
  void *k_blocks;
  void *v_blocks;
  void *kbar;
  float *kbar_partial;
  int32_t *len;
  int32_t batch;
  int32_t capacity;
} qsa_cache;

/* Human-readable name of a status code (static string). */
QSA_API const char *qsa_status_string(qsa_status s);

/* Library version (major*10000 + minor*100 + patch). */
QSA_API int32_t qsa_version(void);

/* Number of CUDA kernels this library has launched in this process (all devices). */
QSA_API uint64_t qsa_launch_count(void);

/* Zero the status words at the start of a workspace (enqueued on stream).  Call once
 * after allocating a workspace, before its first use. */
QSA_API qsa_status qsa_workspace_init(void *workspace, size_t ws_bytes, qsa_stream_t stream);

/* Synchronise `stream`, read and clear the device status word of `workspace`.  Returns
 * QSA_OK, QSA_ERR_TIMEOUT or QSA_ERR_DEVICE (the first failure recorded since the last
 * read), or QSA_ERR_CUDA if the synchronisation itself failed.  If site != NULL it receives
 * an internal id of the failing wait / check. */
QSA_API qsa_status qsa_last_device_error(void *workspace, qsa_stream_t stream, uint32_t *site);

/* ---------------------------------------------------------------------------------- */
/* Step a1: block compression ("Long context became an architecture problem": the indexer
 * scores compressed key blocks; the mean is this library's choice of compression).
 *   k_idx         bf16 [T][64]   per-token indexer keys, sequences packed back to back
 *   d_cu_seqlens  int32 [num_seqs+1] device copy of the cumulative lengths (cu[0] = 0)
 *   h_cu_seqlens  int32 [num_seqs+1] host copy of the same values
 *   kbar          bf16 [sum_s floor(L_s/4)][64] output, sequence s starting at block
 *                 sum_{j<s} floor(L_j/4)
 * kbar[b][d] = bf16_rne(((k0 + k1) + k2) + k3) * 0.25) with fp32 sums; only complete
 * blocks are written (a trailing partial block "remains uncompressed").  The workspace
 * (qsa_compress_workspace_size bytes) holds per-sequence offsets. */
QSA_API size_t qsa_compress_workspace_size(int32_t num_seqs);

QSA_API qsa_status qsa_compress(const void *k_idx, const int32_t *d_cu_seqlens,
                        const int32_t *h_cu_seqlens, int32_t num_seqs, void *kbar,
                        void *workspace, size_t ws_bytes, qsa_stream_t stream);

/* Step a2 alone (prefill shape): indexer scores of query rows [row_begin, row_end) against
 * the compressed keys of their own sequence.  workspace: qsa_prefill_workspace_size bytes
 * (only its header and per-sequence metadata are used).
 *   q_idx   bf16 [T][16][64];  w bf16 [T][16];  kbar as written by qsa_compress
 *   scores  fp32 [row_end-row_begin][ld]: scores[t-row_begin][b] = s(t,b) for every
 *           b < floor(pos(t)/4); other entries are left untouched.  ld >= max n_c.
 * row_begin/row_end must fall on 16-token tile boundaries of their sequences (a sequence
 * start, a multiple of 16 tokens into a sequence, or the end of a sequence).
 * Rows whose candidates all fit in topk (floor(pos/4) <= topk) may be skipped when
 * topk > 0; pass topk = 0 to score every row. */
QSA_API qsa_status qsa_index_scores(const void *q_idx, const void *w, const void *kbar,
                            const int32_t *d_cu_seqlens, const int32_t *h_cu_seqlens,
                            int32_t num_seqs, int64_t row_begin, int64_t row_end,
                            float *scores, int64_t ld, int32_t topk, void *workspace,
                            size_t ws_bytes, qsa_stream_t stream);

/* Step a3 alone: per-row top-k ("Long context ...": budget 512 blocks = 2,048 tokens;
 * ties to the lower block index).
 *   scores  fp32 [rows][ld], row r has n_c[r] candidates in columns 0..n_c[r]-1
 *   n_c     int32 [rows] (device)
 *   idx     int32 [rows][topk] output: the min(topk, n_c) selected blocks in ascending
 *           order, padded with -1;  cnt int32 [rows] output: min(topk, n_c). */
QSA_API qsa_status qsa_topk(const float *scores, int64_t ld, const int32_t *n_c, int64_t rows,
                    int32_t topk, int32_t max_n_c, int32_t *idx, int32_t *cnt,
                    qsa_stream_t stream);

/* ---------------------------------------------------------------------------------- */
/* Prefill (steps a1-a4) over a packed varlen batch.
 *   q      bf16 [T][24][128]      k, v   bf16 [T][2][128]
 *   q_idx  bf16 [T][16][64]       k_idx  bf16 [T][64]       w  bf16 [T][16] (w >= 0)
 *   out    bf16 [T][24][128]
 * Sequence lengths >= 1 and <= QSA_MAX_SEQ_LEN. */
QSA_API size_t qsa_prefill_workspace_size(const int32_t *h_cu_seqlens, int32_t num_seqs,
                                  qsa_params params);

QSA_API qsa_status qsa_prefill(const void *q, const void *k, const void *v, const void *q_idx,
                       const void *k_idx, const void *w, const int32_t *d_cu_seqlens,
                       const int32_t *h_cu_seqlens, int32_t num_seqs, void *out,
                       void *workspace, size_t ws_bytes, qsa_params params,
                       qsa_stream_t stream);

/* Steps a1-a3 only: the block selection of every token.
 *   idx int32 [T][topk] (ascending, -1 padded),  cnt int32 [T]. */
QSA_API qsa_status qsa_prefill_select(const void *q_idx, const void *k_idx, const void *w,
                              const int32_t *d_cu_seqlens, const int32_t *h_cu_seqlens,
                              int32_t num_seqs, int32_t *idx, int32_t *cnt, void *workspace,
                              size_t ws_bytes, qsa_params params, qsa_stream_t stream);

/* Step a4 alone: attention of every token over a given selection (idx/cnt as returned by
 * qsa_prefill_select) plus its own block.  Selected blocks must be < floor(pos/4),
 * ascending, without repeats. */
QSA_API qsa_status qsa_sparse_attention(const void *q, const void *k, const void *v, const int32_t *idx,
                                const int32_t *cnt, const int32_t *d_cu_seqlens,
                                const int32_t *h_cu_seqlens, int32_t num_seqs, void *out,
                                void *workspace, size_t ws_bytes, qsa_params params,
                                qsa_stream_t stream);

/* ---------------------------------------------------------------------------------- */
/* Step a5: append tokens to the cache (aiany.app "Implementation notes": KV cache sizing
 * for very long contexts).  For each sequence b, counts[b] (or n_new if counts is NULL)
 * tokens are appended after its current length:
 *   k, v   bf16 [batch][n_new][2][128]     k_idx  bf16 [batch][n_new][64]
 *   counts int32 [batch] device, each 0..n_new, or NULL
 *   h_len  int32 [batch] HOST copy of the current lengths, used to check capacity.
 * Complete blocks get their compressed key with exactly the bits qsa_compress would
 * produce; an incomplete last block keeps its running fp32 sum in kbar_partial.
 * len is advanced on the device. */
QSA_API qsa_status qsa_append_kv(const qsa_cache *cache, const void *k, const void *v,
                         const void *k_idx, int32_t n_new, const int32_t *counts,
                         const int32_t *h_len, qsa_stream_t stream);

/* Decode (steps a2, a3, a6) for one new query token per sequence, at position
 * p = len-1 (its K/V/k_idx must already be appended).
 *   q      bf16 [batch][24][128]    q_idx bf16 [batch][16][64]    w bf16 [batch][16]
 *   out    bf16 [batch][24][128]
 *   h_len  int32 [batch] HOST copy of the lengths after the append (sizes the grids).
 * Optional outputs sel_idx int32 [batch][topk] / sel_cnt int32 [batch] receive the block
 * selection (pass NULL to skip). */
QSA_API size_t qsa_decode_workspace_size(const qsa_cache *cache, qsa_params params);

QSA_API qsa_status qsa_decode(const void *q, const qsa_cache *cache, const void *q_idx, const void *w,
                      void *out, const int32_t *h_len, int32_t *sel_idx, int32_t *sel_cnt,
                      void *workspace, size_t ws_bytes, qsa_params params,
                      qsa_stream_t stream);

/* ---------------------------------------------------------------------------------- */
/* Context-sharded decode ("Long context became an architecture problem", section "Open
 * weights still require a compatible runtime": 262,144 tokens native, extendable to one
 * million; the pages describe no multi-GPU scheme, so the one below is this library's own).
 * A batch's contexts are split over R shards, one per GPU: shard r is an ordinary qsa_cache
 * (contiguous) holding tokens [t0_r, t0_r + capacity) of every sequence, with t0_r a multiple
 * of 512 (block0 = t0_r / 4 is then a multiple of 128), shards back to back in token order.
 * Its len[b] counts the tokens of sequence b stored there (0 .. capacity); every shard before
 * the one holding a sequence's last token must be full.  Appends go with qsa_append_kv to the
 * shard that holds the new token.  One decode step is then:
 *   1. every shard: qsa_decode_shard_select -> its top-k (score, global block) candidates;
 *   2. exchange: every rank gathers all shards' candidates (e.g. an NCCL all-gather);
 *   3. every rank: qsa_merge_candidates -> the selection (identical on every rank, and bit
 *      for bit the selection qsa_decode would make over the whole context);
 *   4. every shard: qsa_decode_shard_attend -> per-(sequence, head) partial softmax over the
 *      selected blocks it holds (plus the query's own block on the shard that holds it);
 *   5. exchange the partials, then qsa_combine_partials -> the output.
 * d_glen: int32 [batch] device, the sequences' whole lengths (after the append).  The
 * workspace of a shard call is qsa_decode_shard_workspace_size(shard) bytes (the decode
 * workspace of that cache). */
QSA_API size_t qsa_decode_shard_workspace_size(const qsa_cache *shard, qsa_params params);

/*   q_idx bf16 [batch][16][64], w bf16 [batch][16]: the decode query's indexer inputs.
 *   h_len int32 [batch] HOST copy of shard->len (sizes the grids).
 *   cand_score fp32 [batch][topk], cand_idx int32 [batch][topk], cand_cnt int32 [batch]:
 *   the shard's min(topk, n) best candidate blocks (global ids, ascending; padded with -1)
 *   and their scores, n = its complete blocks before the query's own block. */
QSA_API qsa_status qsa_decode_shard_select(const void *q_idx, const void *w,
                                           const qsa_cache *shard, int32_t block0,
                                           const int32_t *d_glen, const int32_t *h_len,
                                           float *cand_score, int32_t *cand_idx,
                                           int32_t *cand_cnt, void *workspace, size_t ws_bytes,
                                           qsa_params params, qsa_stream_t stream);

/* cand_score fp32 [shards][batch][topk], cand_idx int32 [shards][batch][topk], cand_cnt int32
 * [shards][batch] (the shards' outputs stacked in shard order); max_blocks > every global
 * block id (the whole capacity / 4).  sel_idx int32 [batch][topk] (ascending, -1 padded) and
 * sel_cnt int32 [batch] receive the selection: the topk best of all candidates, larger score
 * first and the lower block among equal scores.  shards <= 64; the call needs
 * shards * topk * 8 + max_blocks / 4 bytes of shared memory (about 200 KB at most), else
 * QSA_ERR_UNSUPPORTED.  workspace: at least QSA_WS_HEADER_BYTES (device status only). */
QSA_API qsa_status qsa_merge_candidates(const float *cand_score, const int32_t *cand_idx,
                                        const int32_t *cand_cnt, int32_t shards, int32_t batch,
                                        int32_t topk, int32_t max_blocks, int32_t *sel_idx,
                                        int32_t *sel_cnt, void *workspace, size_t ws_bytes,
                                        qsa_stream_t stream);

/*   q bf16 [batch][24][128]; sel_idx/sel_cnt as returned by qsa_merge_candidates.
 *   part_o fp32 [batch][24][128] (unnormalised), part_m fp32 [batch][24] (running max, in
 *   log2 units of the scaled scores), part_l fp32 [batch][24] (sum of exponentials): this
 *   shard's part of the softmax (m = -inf, l = 0, o = 0 when it holds none of the keys). */
QSA_API qsa_status qsa_decode_shard_attend(const void *q, const qsa_cache *shard,
                                           int32_t block0, const int32_t *d_glen,
                                           const int32_t *sel_idx, const int32_t *sel_cnt,
                                           float *part_o, float *part_m, float *part_l,
                                           void *workspace, size_t ws_bytes, qsa_params params,
                                           qsa_stream_t stream);

/* part_o fp32 [shards][batch][24][128], part_m / part_l fp32 [shards][batch][24] (stacked in
 * shard order) -> out bf16 [batch][24][128], merged by log-sum-exp. */
QSA_API qsa_status qsa_combine_partials(const float *part_o, const float *part_m,
                                        const float *part_l, int32_t shards, int32_t batch,
                                        void *out, qsa_stream_t stream);

/* ---------------------------------------------------------------------------------- */
/* Decode without a caller-provided workspace.  The pages have no counterpart of this entry
 * point; it exists for callers that cannot allocate device memory on the call path and have
 * no buffer to lend -- for example a plugin running inside a host framework whose allocator
 * owns all device memory, or a serving loop that must not allocate after start-up.
 *
 * Same inputs, outputs and result as qsa_decode (it runs the same kernels), but the scratch
 * lives in one fixed device array inside the library, QSA_NOALLOC_SCRATCH_BYTES (32 MiB)
 * large, which every GPU that loads the library holds until the process exits.
 *   - Returns QSA_ERR_WORKSPACE, with nothing enqueued, when this cache's batch, capacity
 *     and budget need more scratch than that (compare qsa_decode_workspace_size); batch 64 at
 *     capacity 262,144 with budget 512 needs about 19 MB.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - Every call made outside a stream capture looks up the array's device address on the
 *     current device (so a module reloaded after cudaDeviceReset is followed).  A call made
 *     during a capture reuses the address of the last uncaptured call on that device: make
 *     one call before any stream capture, or the captured call fails with QSA_ERR_CUDA.
 *   - Every call, on every stream, shares the one array and it keeps the last call's
 *     contents; each call clears the status words at its start.  Calls that overlap on the
 *     GPU race on the array and corrupt each other's results: serialise them (one stream,
 *     or events between streams).  Read a call's device-side status with
 *     qsa_noalloc_last_device_error before the next call clears it. */
#define QSA_NOALLOC_SCRATCH_BYTES (32u << 20)

QSA_API qsa_status qsa_decode_noalloc(const void *q, const qsa_cache *cache, const void *q_idx,
                                      const void *w, void *out, const int32_t *h_len,
                                      int32_t *sel_idx, int32_t *sel_cnt, qsa_params params,
                                      qsa_stream_t stream);

/* The device-side status of the last qsa_decode_noalloc call, read from the library's static
 * scratch array: synchronises `stream`, then returns and clears it exactly as
 * qsa_last_device_error does for a workspace (QSA_OK, QSA_ERR_TIMEOUT, QSA_ERR_DEVICE, or
 * QSA_ERR_CUDA when the copy or the synchronisation failed).  Allocates nothing. */
QSA_API qsa_status qsa_noalloc_last_device_error(qsa_stream_t stream, uint32_t *site);

/* ---------------------------------------------------------------------------------- */
/* Paged KV cache (aiany.app "Qwen3.8-Flash-Next", "Implementation notes": the model ships
 * with serving recipes for vLLM and SGLang, and KV cache sizing for very long contexts is
 * an operational concern).  Those frameworks keep their caches in pages; the pages give no
 * page layout, so the one below is this library's own.  Sequences own fixed-size pages of
 * one shared pool, listed in a page table, so that a batch of sequences of very different
 * lengths needs pool memory only for the pages it has reached:
 *   base.k_blocks, base.v_blocks : bf16 [pool_pages][2][page_tokens/4][4][128]
 *   base.kbar                    : bf16 [pool_pages][page_tokens/4][64]
 *   base.kbar_partial, base.len  : per sequence, as in qsa_cache
 *   page_table : int32 [batch][base.capacity/page_tokens] device: logical page j of sequence
 *                b (its tokens j*page_tokens ..) lives in pool page page_table[b][j]
 * base.capacity is the logical capacity per sequence, a multiple of page_tokens; page_tokens
 * is a multiple of 512 (an indexer tile of 128 blocks then never spans two pages), and
 * pool_pages * 2 * page_tokens < 2^31.  Only the entries of pages a sequence has reached are
 * read.  Each must lie in 0 .. pool_pages-1, and live sequences must not share a page.  An
 * entry out of range is never followed: the append skips the writes that would go there
 * (it has no workspace to report in), and the decode reads zeros there and records
 * QSA_ERR_DEVICE.  Same arguments, results and errors as qsa_append_kv, qsa_decode and
 * qsa_decode_workspace_size otherwise (the workspace size is the contiguous cache's); the
 * results are bit-identical to those of a contiguous cache holding the same tokens. */
typedef struct {
  qsa_cache base;
  int32_t *page_table;
  int32_t page_tokens;
  int32_t pool_pages;
} qsa_paged_cache;

QSA_API qsa_status qsa_append_kv_paged(const qsa_paged_cache *cache, const void *k,
                                       const void *v, const void *k_idx, int32_t n_new,
                                       const int32_t *counts, const int32_t *h_len,
                                       qsa_stream_t stream);

QSA_API size_t qsa_decode_paged_workspace_size(const qsa_paged_cache *cache, qsa_params params);

QSA_API qsa_status qsa_decode_paged(const void *q, const qsa_paged_cache *cache,
                                    const void *q_idx, const void *w, void *out,
                                    const int32_t *h_len, int32_t *sel_idx, int32_t *sel_cnt,
                                    void *workspace, size_t ws_bytes, qsa_params params,
                                    qsa_stream_t stream);

/* ---------------------------------------------------------------------------------- */
/* The Gated DeltaNet layer, prefill over packed variable-length sequences ("Long context
 * became an architecture problem", "Linear attention carries the stream; sparse attention
 * retrieves detail": Gated DeltaNet, a gated linear recurrence over a compact state, carries
 * three of every four token-mixing layers; the pages' table of its parameters is lost, so
 * the update is the published gated delta rule).  Per sequence and head, the state S
 * (128 x 128, fp32) starts at zero, and token t updates it and reads it out:
 *     S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,    o_t = S_t q_t
 * with alpha_t = exp(log_alpha_t).  q and k are used as given (any normalisation or scaling
 * happens before the call); log_alpha below -87 counts as -87 (a full reset, to fp32 range).
 * Arithmetic: the chunked products run on the tensor cores with TF32 operands and fp32
 * accumulation; the operands that carry into the state are split into two TF32 parts (about
 * fp32 accuracy); the state is fp32.
 *   q, k, v      bf16 [T][heads][128], 16-byte aligned
 *   log_alpha    fp32 [T][heads] (<= 0 keeps the state bounded), beta fp32 [T][heads]
 *   d_cu_seqlens int32 [num_seqs+1] on the device, h_cu_seqlens the same on the host
 *                (0 = cu[0] <= cu[1] <= ...; sequences may be empty)
 *   out          bf16 [T][heads][128] output, 16-byte aligned (caller-owned)
 *   final_state  fp32 [num_seqs][heads][128 (v)][128 (k)] output: S after each sequence's
 *                last token, or NULL
 * heads 1..256.  No workspace.  Errors: QSA_ERR_INVALID_ARG (null pointer, bad sizes or
 * cu_seqlens), QSA_ERR_ALIGNMENT, QSA_ERR_CUDA (launch failure).  Asynchronous on stream. */
QSA_API qsa_status qsa_gated_deltanet(const void *q, const void *k, const void *v,
                                      const float *log_alpha, const float *beta,
                                      const int32_t *d_cu_seqlens, const int32_t *h_cu_seqlens,
                                      int32_t num_seqs, int32_t heads, void *out,
                                      float *final_state, qsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H_ */
