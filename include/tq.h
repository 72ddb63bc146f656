/*
 * tq.h -- C ABI of libtq.so: TurboQuant paged KV cache on NVIDIA B200 (sm_100a).
 *
 * What it computes.  "xInfer: Pure-Rust LLM Inference Without a Python
 * Runtime", section "What actually sits between the request and the tokens":
 * the KV cache is compressed by a Walsh-Hadamard transform rotation followed
 * by per-head absmax quantisation (a 2-4 bit cache; the --kvcache-dtype flag
 * of section "Getting a server up" also offers turbo8, and no flag means BF16).
 * Section "TurboQuant is a memory trade": reading the cache dequantises on
 * every attention step.  "infero", section "Continuous batching": requests
 * share the GPU over a paged KV cache.
 *
 * Arithmetic (the pages leave it open; this library fixes it):
 *   rotation  y = H_d x / sqrt(d), H_d the Sylvester-ordered Hadamard matrix,
 *             as fp32 butterflies with strides 1, 2, 4, ..., d/2 and then one
 *             fp32 multiply by fp32(1/sqrt(d)); no fused multiply-add.
 *   scale     s = max_i |y_i|, stored as fp32.
 *   codes     L = 2^(b-1) - 1, code_i = clamp(roundf(fp32(y_i * L) / s), -L, L)
 *             (IEEE division, ties away from zero); s == 0 gives all codes 0.
 *   storage   u_i = code_i + L, bit-packed LSB-first: u_i occupies bits
 *             [i*b, (i+1)*b) of a little-endian byte string of d*b/8 bytes.
 *   attention dequantised yhat_i = code_i * s / L; score_j = (H q / sqrt(d)) .
 *             yhat_k,j / sqrt(d); out = H (sum_j softmax_j yhat_v,j) / sqrt(d).
 *             Query position t of q_len sees keys j <= seq_len - q_len + t.
 *             Query head h reads kv head h / (num_q_heads / num_kv_heads).
 *   fp8       (--kvcache-dtype fp8 of "Getting a server up"; 2x, "near-
 *             lossless" in "TurboQuant is a memory trade"; the rest is this
 *             library's reading) no rotation; s = max_i |x_i| as fp32; code_i
 *             = the OCP E4M3 value nearest fl(fl(x_i * 448) / s), ties to the
 *             even mantissa, saturating at 448 (s == 0: codes 0), stored as its
 *             byte; dequantised xhat_i = value(code_i) * s / 448; attention
 *             softmax(q . k / sqrt(d)) v on the dequantised K and V.  Its
 *             blocks have the turbo8 layout below.
 *
 * Cache layout in device memory (one pool per layer):
 *   pool[num_pages][num_kv_heads][2][block], block = tq_page_block_bytes(...):
 *   the K block, then the V block, of each (page, kv head).  K and V of a
 *   page are adjacent so that decode fetches both with one bulk copy.
 *   turbo b-bit K block: page_size token rows of d*b/8 code bytes (row t =
 *   token t's packed vector), then page_size fp32 scales.  For b = 2, 4, 8
 *   the 16-byte chunks of row t are permuted: logical chunk c is stored at
 *   chunk c ^ w(t), with w(t) = (t >> 2) & 1, (t >> 1) & 3, t & 7 for
 *   b = 2, 4, 8 (a bank-conflict-free read pattern); 3-bit rows are stored
 *   in order.
 *   turbo b-bit V block: the same codes dim-major -- d rows of
 *   page_size*b/8 bytes, row i holding every token's code i (token t at bits
 *   [t*b, (t+1)*b) of the row, LSB-first) -- then page_size fp32 scales.
 *   (K rows feed a decode thread per token, V rows a thread per dimension.)
 *   BF16 block (K and V): page_size token rows of d bf16 values.
 *   A token's slot is page * page_size + offset.
 *
 * Ownership.  The library allocates nothing and keeps no state between calls
 * (the one exception is the fixed scratch array of tq_paged_decode_noalloc,
 * described there).  Every buffer is caller-owned device memory unless
 * stated otherwise.  Every call is asynchronous on the given CUDA stream (a
 * cudaStream_t passed as void*, NULL = legacy default stream); calls on
 * different streams are safe when their buffers are disjoint.
 *
 * Errors.  Arguments are checked on the host before anything is launched; a
 * failed check returns a status and launches nothing.  A CUDA launch failure
 * returns TQ_ERR_CUDA.  Problems only visible on the device (a page id or a
 * slot outside the pool, a sequence length outside [q_len, max_seq_len], a
 * bounded wait that expired) skip the affected work and record the first
 * such event in the optional device word cache->dev_error; read it with
 * tq_read_device_error.  The outputs of a call that recorded an event are
 * unspecified for the affected sequences.  No device code traps or asserts.
 *
 * Supported shapes: head_dim 128; page_size 16, 32 or 64; 1 <= q_len and
 * q_len * (num_q_heads / num_kv_heads) <= 4096: one decode token, a verify
 * window of draft tokens, or a chunk of prefill tokens (appended first, then
 * attending causally over the cache).  With a turbo format, 128 or more
 * rows per kv head run on a query-major kernel (128 rows per CTA, each K/V
 * tile dequantised once per 128 rows, no split workspace); fewer rows beyond
 * 16 run as several 16-row groups (8 for a bf16 cache, 16 for fp8), each
 * reading the kv head's pages.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_ABI_VERSION 3

typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, shape or alignment */
    TQ_ERR_UNSUPPORTED = 2,   /* well-formed but outside the supported shapes */
    TQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    TQ_ERR_TIMEOUT = 4,       /* a bounded device wait expired (device word) */
    TQ_ERR_DEVICE_CHECK = 5,  /* a device-side range check failed (device word) */
    TQ_ERR_WORKSPACE = 6,     /* decode workspace missing or too small */
    TQ_ERR_NO_PAGES = 7       /* prefix-block manager: the pool has no page left */
} tq_status;

/* KV cache formats: the --kvcache-dtype choices of the xInfer page (section
 * "Getting a server up"; turbo2 extends its "2 to 4 bit" range downwards). */
typedef enum {
    TQ_TURBO2 = 2,
    TQ_TURBO3 = 3,
    TQ_TURBO4 = 4,
    TQ_TURBO8 = 8,
    TQ_BF16 = 16,
    TQ_FP8 = 17      /* E4M3 codes, no rotation (see "fp8" above) */
} tq_format;

/* Descriptor of one layer's paged K/V pool.  Plain data; the pointed-to
 * device memory is owned by the caller. */
typedef struct {
    int32_t format;        /* tq_format */
    int32_t head_dim;      /* d; must be 128 */
    int32_t num_kv_heads;  /* >= 1 */
    int32_t page_size;     /* tokens per page: 16, 32 or 64 */
    int32_t num_pages;     /* pages in the pool, >= 1 */
    void* pages;           /* device, 16-byte aligned, num_pages*num_kv_heads*2*block bytes:
                              [page][kv head][K block, V block] */
    uint32_t* dev_error;   /* device word, optional (NULL: device findings dropped).
                              0 = no error; else (tq_status) | (detail << 8). */
} tq_cache;

/* ABI version of the loaded library (TQ_ABI_VERSION). */
int32_t tq_abi_version(void);

/* Readable name of a status.  Never NULL; the string is static. */
const char* tq_status_string(tq_status status);

/* Bytes of one K (or V) block of one (page, kv head), per the layout above
 * (the pool holds num_pages * num_kv_heads * 2 of them); 0 when the arguments
 * are not a supported combination. */
size_t tq_page_block_bytes(int32_t format, int32_t head_dim, int32_t page_size);

/*
 * tq_quantize_append -- rotate, absmax-quantise, bit-pack and store new K/V
 * rows into a turbo cache ("What actually sits between the request and the
 * tokens": Walsh-Hadamard rotation followed by per-head absmax quantisation).
 *   k, v          device bf16 [num_tokens][num_kv_heads][head_dim], 16-byte
 *                 aligned; one (token, head) row is one quantised vector.
 *   slot_mapping  device int64 [num_tokens]: slot = page*page_size + offset;
 *                 a negative slot skips the token; a slot past the pool is
 *                 skipped and recorded as TQ_ERR_DEVICE_CHECK.
 *   num_tokens    >= 0 (0 is a no-op).
 *   bits          2, 3, 4 or 8; must equal cache->format.
 * Result: codes and the fp32 scale of every (token, head) of K and of V are
 * written at their slot; nothing else in the pool changes.  Bit-exact with
 * the definition above for every finite input.
 */
tq_status tq_quantize_append(const void* k, const void* v,
                             const int64_t* slot_mapping, int32_t num_tokens,
                             int32_t bits, const tq_cache* cache, void* stream);

/*
 * tq_append_bf16 -- store new K/V rows unchanged into a BF16 cache (the
 * "no flag means BF16" cache of "Getting a server up"), the uncompressed
 * reference point.  Arguments as tq_quantize_append; cache->format must be
 * TQ_BF16.
 */
tq_status tq_append_bf16(const void* k, const void* v,
                         const int64_t* slot_mapping, int32_t num_tokens,
                         const tq_cache* cache, void* stream);

/*
 * tq_decode_workspace_size -- bytes of device workspace tq_paged_decode and
 * tq_paged_decode_bf16 need for these shapes (0 when every sequence fits in
 * one split and none is needed).  The workspace holds per-split softmax
 * partials and one merge counter per (sequence, kv head, row group).
 * Returns 0 for invalid arguments as well; the decode call re-checks.
 */
size_t tq_decode_workspace_size(int32_t batch, int32_t q_len,
                                int32_t num_q_heads, int32_t max_seq_len,
                                const tq_cache* cache);

/*
 * tq_decode_workspace_init -- zero the merge counters of a workspace.  Call
 * once after allocating it; every decode call leaves them zero again, a call
 * whose device word reports TQ_ERR_TIMEOUT included (a split that gives up
 * records an empty partial and still takes its turn in the merge).
 */
tq_status tq_decode_workspace_init(void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * tq_paged_decode -- batched decode / short speculative-verify attention over
 * a turbo cache through per-sequence page tables, dequantising on the fly
 * ("TurboQuant is a memory trade": dequantisation on every attention step;
 * infero "Continuous batching": paged KV shared by a running batch).
 *   q                device bf16 [batch][q_len][num_q_heads][head_dim].
 *   page_table       device int32 [batch][max_pages_per_seq]; entry p is the
 *                    physical page of tokens [p*page_size, (p+1)*page_size).
 *                    Pages may be shared between sequences (prefix sharing).
 *   seq_lens         device int32 [batch]: cached tokens of each sequence,
 *                    the q_len new ones included (they must already be
 *                    appended); q_len <= seq_lens[b] <= max_seq_len.
 *   batch            >= 0 (0 is a no-op), <= 65535.
 *   q_len            1 for decode, >1 for causal verify of draft tokens.
 *   max_seq_len      host bound on seq_lens, sizes the launch and workspace.
 *   out              device fp32 [batch][q_len][num_q_heads][head_dim],
 *                    16-byte aligned; fully written for valid sequences.
 *   workspace        device, tq_decode_workspace_size bytes (may be NULL
 *                    when that size is 0), 16-byte aligned, initialised once
 *                    by tq_decode_workspace_init.  Calls that overlap in
 *                    time must use different workspaces.
 * Each sequence is split into fixed parts of 2048 tokens (1024 for 64-token
 * pages) whatever the batch holds, so a sequence's output does not depend
 * on the other sequences of the batch.
 */
tq_status tq_paged_decode(const void* q, const tq_cache* cache,
                          const int32_t* page_table, int32_t max_pages_per_seq,
                          const int32_t* seq_lens, int32_t batch, int32_t q_len,
                          int32_t num_q_heads, int32_t max_seq_len, float* out,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_paged_decode_bf16 -- the same decode over a BF16 cache (no rotation, no
 * scales): out = softmax(q k / sqrt(d)) v.  Arguments and workspace rules
 * as tq_paged_decode; cache->format must be TQ_BF16.
 */
tq_status tq_paged_decode_bf16(const void* q, const tq_cache* cache,
                               const int32_t* page_table,
                               int32_t max_pages_per_seq,
                               const int32_t* seq_lens, int32_t batch,
                               int32_t q_len, int32_t num_q_heads,
                               int32_t max_seq_len, float* out,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * tq_paged_decode_noalloc -- tq_paged_decode for callers that may not
 * allocate device memory while they run (for example a runtime plugin whose
 * enqueue hook works inside a fixed memory plan).  The pages have no
 * counterpart; this is a convenience of this library.  Arguments as
 * tq_paged_decode without the workspace: the split-KV scratch lives in one
 * 64 MiB array inside libtq.so that every GPU loading the library holds
 * until exit.  Shapes needing more than that return TQ_ERR_WORKSPACE before
 * any launch.  The first call on a device looks the array up (so make it
 * before any stream capture); every call clears the merge counters with a
 * cudaMemsetAsync on `stream` and allocates nothing.  All calls share the
 * array: calls that overlap in time on one GPU race and must be serialised
 * by the caller.
 */
tq_status tq_paged_decode_noalloc(const void* q, const tq_cache* cache,
                                  const int32_t* page_table,
                                  int32_t max_pages_per_seq,
                                  const int32_t* seq_lens, int32_t batch,
                                  int32_t q_len, int32_t num_q_heads,
                                  int32_t max_seq_len, float* out, void* stream);

/*
 * tq_read_device_error -- wait (bounded, ~10 s) for the stream, then copy the
 * device error word of cache->dev_error into *code (0 when no word is set);
 * clear != 0 resets it to zero.  Returns TQ_ERR_TIMEOUT if the stream did
 * not finish in time, TQ_ERR_CUDA on a CUDA failure, else TQ_OK.
 */
tq_status tq_read_device_error(const tq_cache* cache, uint32_t* code,
                               int32_t clear, void* stream);

/*
 * Roofline probes used by the benchmark to measure this GPU's HBM bandwidth
 * in the same run (no counterpart on the pages):
 *   tq_hbm_copy  dst[i] = src[i] over `bytes` bytes (16-byte aligned,
 *                bytes a multiple of 16); moves 2*bytes through HBM.
 *   tq_hbm_read  reads `bytes` bytes and writes one 32-bit checksum to
 *                *sink so the read cannot be elided; moves `bytes`.
 */
tq_status tq_hbm_copy(const void* src, void* dst, size_t bytes, void* stream);
tq_status tq_hbm_read(const void* src, size_t bytes, uint32_t* sink,
                      void* stream);

/*
 * One decode step captured as a CUDA graph: "CUDA Graphs mean the decode step
 * is captured as a graph and replayed, which removes per-token launch
 * overhead" (xInfer review, "What actually sits between the request and the
 * tokens").  The step is the append of num_tokens new tokens (skipped when 0;
 * tq_quantize_append for a turbo cache, tq_append_bf16 for a BF16 one)
 * followed by the paged decode (skipped when batch is 0), with exactly the
 * arguments of those calls.  Every pointer and size is fixed at capture: the
 * caller refreshes the contents of the buffers (new K/V, slots, q, page
 * table, lengths) between launches, keeping q_len, batch and max_seq_len.
 * The decode workspace returns its counters to zero after every step, so a
 * graph can be replayed any number of times.
 */
typedef struct {
    const void* k;                  /* append: as tq_quantize_append */
    const void* v;
    const int64_t* slot_mapping;
    int32_t num_tokens;
    const void* q;                  /* decode: as tq_paged_decode */
    const int32_t* page_table;
    int32_t max_pages_per_seq;
    const int32_t* seq_lens;
    int32_t batch;
    int32_t q_len;
    int32_t num_q_heads;
    int32_t max_seq_len;
    float* out;
    void* workspace;
    size_t workspace_bytes;
} tq_step;

typedef struct tq_step_graph tq_step_graph;

/* Validate the step as the two calls would, then capture it on `stream` (a
 * created stream, not NULL: the legacy stream cannot be captured) and
 * instantiate it.  Nothing runs on the GPU.  *graph is NULL on failure. */
tq_status tq_step_graph_create(const tq_cache* cache, const tq_step* step, void* stream,
                               tq_step_graph** graph);
/* Run the captured step on `stream` (asynchronous). */
tq_status tq_step_graph_launch(tq_step_graph* graph, void* stream);
void tq_step_graph_destroy(tq_step_graph* graph);

/*
 * Prefix-block manager -- block-granular KV reuse across requests, host side.
 * "xinfer-ai" package docs, "Prefix Cache (KV Reuse)": finished sequences give
 * their full KV blocks to a global prefix cache; a new request reuses the
 * longest cached block-aligned prefix and prefills only the rest; a common
 * prefix ending inside a block has that block's tail recomputed; a prompt
 * cached entirely at block boundaries recomputes its last block (the prefill
 * step is never empty); the cache shares the pool with live sequences and is
 * capped at a token count rounded down to whole blocks.
 *
 * A block is one page of page_size tokens.  The manager hands out page ids of
 * a pool of num_pages pages (the pool itself is the caller's device memory,
 * described by a tq_cache with the same page_size and num_pages); a cached
 * page is shared by every sequence whose prompt starts with the same blocks
 * of token ids.  Pages are reference counted (one reference per live
 * sequence holding the page, one while it is cached); when no page is free,
 * or the cache is over its cap, the least recently used cached block that no
 * live sequence holds and that has no cached children is evicted.  All calls
 * are host-only (no device memory is touched) and thread-safe; the caller
 * copies the page tables to the device.  Errors: TQ_ERR_INVALID_ARG for bad
 * arguments, TQ_ERR_NO_PAGES when the pool cannot supply the pages (nothing
 * changes then).
 */
typedef struct tq_prefix_cache tq_prefix_cache;

typedef struct {
    int64_t free_pages;       /* pages no sequence or cached block holds */
    int64_t cached_blocks;    /* blocks in the prefix cache */
    int64_t live_sequences;   /* begun and not finished */
    int64_t hit_tokens;       /* prompt tokens served from the cache, summed over calls */
    int64_t prompt_tokens;    /* prompt tokens admitted, summed over calls */
    int64_t evictions;        /* cached blocks evicted */
} tq_prefix_stats;

/* A manager for num_pages pages of page_size tokens; at most
 * max_cached_tokens / page_size blocks stay cached (<= 0: half the pool).
 * NULL for bad arguments or when host memory runs out. */
tq_prefix_cache* tq_prefix_cache_create(int32_t num_pages, int32_t page_size,
                                        int64_t max_cached_tokens);
void tq_prefix_cache_destroy(tq_prefix_cache* pc);

/*
 * tq_prefix_cache_begin -- admit a sequence whose prompt is the token ids
 * tokens[0 .. num_tokens), num_tokens >= 1.
 *   page_table     host int32 [max_pages]: entries [0, ceil(num_tokens /
 *                  page_size)) are written -- the shared pages of the reused
 *                  prefix blocks, then fresh pages.
 *   cached_tokens  the prompt tokens whose K/V the pool holds already (a
 *                  multiple of page_size): append tokens [cached_tokens,
 *                  num_tokens) before decoding.
 *   seq            a handle for tq_prefix_cache_extend / _finish.
 */
tq_status tq_prefix_cache_begin(tq_prefix_cache* pc, const int32_t* tokens, int32_t num_tokens,
                                int32_t* page_table, int32_t max_pages,
                                int32_t* cached_tokens, int32_t* seq);

/* Grow sequence seq to new_len tokens: fresh pages are added at the end of
 * its table and the whole table is written to page_table (host int32
 * [max_pages]). */
tq_status tq_prefix_cache_extend(tq_prefix_cache* pc, int32_t seq, int32_t new_len,
                                 int32_t* page_table, int32_t max_pages);

/* Finish sequence seq, whose token ids (prompt and generated) are
 * tokens[0 .. num_tokens): each of its full blocks joins the cache (a block
 * already cached keeps its cached page and this sequence's copy is freed),
 * the rest of its pages are freed, and the cache is trimmed to its cap.
 * The handle is invalid afterwards. */
tq_status tq_prefix_cache_finish(tq_prefix_cache* pc, int32_t seq, const int32_t* tokens,
                                 int32_t num_tokens);

/* Counters of the manager. */
tq_status tq_prefix_cache_stats(tq_prefix_cache* pc, tq_prefix_stats* out);

/* References held on one page (sequences + cache), -1 for a bad page id. */
int32_t tq_prefix_cache_page_refs(tq_prefix_cache* pc, int32_t page);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
