/*
 * duo_kv.h -- mixed-head (retrieval / streaming) KV cache and attention
 * for NVIDIA B200 (sm_100a).  C ABI of libduo_kv.so.
 *
 * The method (DuoAttention) splits each layer's KV heads in two:
 *   retrieval heads keep every token in a full, contiguous cache;
 *   streaming heads keep a constant-length cache of the first S tokens
 *   ("attention sinks") plus the most recent W tokens, as a ring buffer.
 * Sources: "DuoAttention: Dual Retrieval & Streaming Heads Guide",
 * section 2 ("Retrieval Heads vs. Streaming Heads", "DuoAttention Cache
 * Partitioning Mechanics" and its memory equation); "Attention Variants and
 * KV-Cache Compression", section "When Is Reuse Exact?" (chunk mask rule,
 * positions kept after eviction); "Attention Variants and Memory
 * Efficiency", sections "Multi-Query and Grouped-Query Attention" and
 * "Sliding-Window and Mixed Attention" (window rule, ring buffer).
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major, on the device of the handle, unless
 *     marked "host".  bf16 tensors are passed as uint16_t bit patterns.
 *   - B = batch, Hq = query heads, n_kv = KV heads, G = Hq / n_kv,
 *     d = head_dim, S = sink, W = window.  Query head h reads KV head h / G.
 *   - The caller owns every device buffer and stream.  The library never
 *     allocates or frees device memory and never synchronises, except
 *     duo_kv_read_status (documented below).  Calls are asynchronous on the
 *     given stream (NULL = the legacy default stream).
 *   - Sequence lengths live on the device and are passed on every call; the
 *     library keeps no per-sequence state besides the cache contents.
 *   - q and K are already position-encoded (e.g. RoPE) by the caller, each
 *     at the token's original position; the library applies no positional
 *     encoding.  Ring slots keep each token's original position.
 *   - Return value: DUO_OK (0) or a negative DUO_ERR_* code.  On an error
 *     nothing was launched.  Errors found by kernels (a length beyond the
 *     capacity, an empty sequence, a pipeline wait that timed out) set bits
 *     of a device status word instead; see duo_kv_read_status.
 */
#ifndef DUO_KV_H
#define DUO_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DUO_API __attribute__((visibility("default")))
#else
#define DUO_API
#endif

/* A cudaStream_t. */
typedef struct CUstream_st* duo_stream_t;

/* Return codes. */
enum {
    DUO_OK = 0,
    DUO_ERR_INVALID_ARG = -1,   /* null pointer, out-of-range index or size   */
    DUO_ERR_UNSUPPORTED = -2,   /* shape the library is not built for:        */
                                /* head_dim not 64 or 128, G not 1/2/4/8,      */
                                /* n_kv > 64                                   */
    DUO_ERR_BUFFER_TOO_SMALL = -3,  /* device buffer smaller than required    */
    DUO_ERR_WORKSPACE = -4,     /* workspace missing or too small              */
    DUO_ERR_CUDA = -5,          /* a CUDA runtime call or launch failed        */
    DUO_ERR_ALIGNMENT = -6      /* a device pointer is not 16-byte aligned     */
                                /* (dev_buf: 256-byte)                         */
};

/* Bits of the device status word (set by kernels, never cleared by them). */
enum {
    DUO_STATUS_OVER_CAPACITY = 1,   /* a retrieval row index >= capacity:     */
                                    /* the row was not written / read          */
    DUO_STATUS_EMPTY_SEQUENCE = 2,  /* decode with len[b] < 1: output zeroed  */
    DUO_STATUS_WAIT_TIMEOUT = 4,    /* a pipeline wait exceeded its limit:     */
                                    /* the output of that launch is invalid    */
    DUO_STATUS_BAD_LENGTH = 8,      /* negative length or append count         */
    DUO_STATUS_NO_PAGE = 16,        /* paged cache: a retrieval row's page is  */
                                    /* missing (-1 or >= num_pages): not       */
                                    /* written / its tile read as zeros        */
    DUO_STATUS_SHARED_PAGE = 32     /* duo_kv_fork: the prefix's partly filled */
                                    /* last page is the same pool page for     */
                                    /* both sequences (both would append into  */
                                    /* it): not copied                         */
};

/* Element type of the K/V caches. */
enum {
    DUO_KV_BF16 = 0,        /* bf16, as given                                  */
    DUO_KV_FP8_E4M3 = 1,    /* FP8 E4M3 codes with per-(layer, KV head) scales  */
    DUO_KV_INT4 = 2         /* INT4 codes, two per byte, same scales            */
};

/* Cache shape.  retrieval_mask is a HOST array [num_layers][num_kv_heads],
 * 1 = retrieval head, 0 = streaming head: the binary head mask of the
 * DuoAttention guide, section 3 item 4 ("Binarization"), given per KV head
 * (with GQA a KV head is retrieval if any query head of its group needs it,
 * the guide's deployment checklist item 2).  It is copied during
 * duo_kv_alloc and not kept.  capacity = rows reserved per retrieval head
 * per sequence (the maximum length).  Constraints: num_layers, batch,
 * num_q_heads, num_kv_heads >= 1; num_q_heads % num_kv_heads == 0;
 * head_dim in {64, 128}; sink >= 0; window >= 1; capacity >= 1.
 *
 * kv_dtype = DUO_KV_FP8_E4M3 stores every cached key and value (retrieval
 * and streaming heads) as one byte, halving the cache (the DuoAttention
 * guide's "Synergies with Low-Bit Quantization": 8 instead of 16 bits per
 * element).  The pages fix neither the format nor the scaling; this library
 * stores code = E4M3(fp32(x) / fp32(scale)) (round to nearest even,
 * saturating at 448) and reads scale * E4M3(code).  k_scale and v_scale are
 * HOST arrays [num_layers][num_kv_heads] of finite positive scales (NULL =
 * all 1.0), copied during duo_kv_alloc.  FP8 needs head_dim 128.
 *
 * kv_dtype = DUO_KV_INT4 stores each element in 4 bits (the same passage: a
 * 4x cut): code c = round-half-to-even(fp32(x) / fp32(scale)) clamped to
 * [-8, 7], two's complement, two codes per byte (element 2i in the low
 * nibble of byte i, 2i + 1 in the high nibble); the cache reads scale * c.
 * Same scale arrays and head_dim 128 requirement as FP8.
 *
 * page_tokens > 0 pages the retrieval caches (paged attention, "Attention
 * Variants and Memory Efficiency", "What the Inference Runtime Can Change":
 * fixed-size blocks, not contiguous in memory): each layer keeps a pool of
 * num_pages pages of [n_retrieval][page_tokens][d] elements, one page = the
 * page_tokens consecutive positions of one sequence for all of the layer's
 * retrieval heads.  Which page holds which positions is a caller-owned
 * device table set with duo_kv_set_page_table and shared by all layers.
 * capacity stays the largest length a sequence may reach (positions are
 * checked against it).  page_tokens must be a multiple of 256; paging needs
 * head_dim 128.  0 = one contiguous [capacity] range per sequence and head. */
typedef struct {
    int32_t num_layers;
    int32_t batch;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t sink;
    int32_t window;
    int64_t capacity;
    const uint8_t* retrieval_mask;
    int32_t kv_dtype;           /* DUO_KV_BF16 (0), DUO_KV_FP8_E4M3 (1) or DUO_KV_INT4 (2) */
    const float* k_scale;       /* FP8 / INT4 only, see above              */
    const float* v_scale;
    int32_t page_tokens;        /* 0 = contiguous retrieval caches        */
    int64_t num_pages;          /* pages per layer pool (page_tokens > 0) */
} duo_kv_desc;

/* Opaque host-side handle (host memory only). */
typedef struct duo_kv duo_kv;

/* Device views of one layer's cache (for verification and for callers that
 * manage the cache themselves).  Layouts, in elements of the cache's
 * kv_dtype (bf16 bit patterns, or one E4M3 byte each -- the pointers then
 * address bytes):
 *   k_retrieval, v_retrieval: [B][n_retrieval][capacity][d], or, paged,
 *                             the pool [num_pages][n_retrieval][page_tokens][d]
 *   k_streaming, v_streaming: [B][n_streaming][S + W][d]
 *   positions:                [B][S + W] int32, original position of the
 *                             token in each streaming slot, -1 = empty
 *                             (shared by all streaming heads of the layer).
 * Streaming slot of token p: p if p < S, else S + (p - S) mod W.
 * head_rank[g] = index of KV head g among the layer's retrieval heads (if
 * retrieval) or among its streaming heads (if streaming); is_retrieval[g]
 * is the mask entry. */
typedef struct {
    uint16_t* k_retrieval;
    uint16_t* v_retrieval;
    uint16_t* k_streaming;
    uint16_t* v_streaming;
    int32_t* positions;
    int32_t n_retrieval;
    int32_t n_streaming;
    int32_t head_rank[64];
    uint8_t is_retrieval[64];
} duo_kv_layer_view;

/* Bytes of device memory a cache of this shape needs (host arithmetic only,
 * no CUDA call).  *cache_bytes (optional) receives the K/V part alone:
 *   sum over layers of 2 * 2 * d * B * (n_r(l) * capacity + n_s(l) * (S+W)),
 * the DuoAttention guide's memory equation (section 2) times the batch,
 * with T = capacity and R = n_r / n_kv per layer.  The rest is the position
 * tables, a status word, one int32 merge counter per (sequence, KV head)
 * for the decode kernel, and 256-byte alignment padding. */
DUO_API int duo_kv_required_bytes(const duo_kv_desc* desc, size_t* total_bytes, size_t* cache_bytes);

/* Lay a cache out in dev_buf (caller-allocated device memory of buf_bytes,
 * 256-byte aligned, on the current device), set every position to -1 and
 * the status word and merge counters to 0 (memsets on `stream`), build the
 * decode kernel's TMA descriptors (head_dim 128), and return a handle.
 * Queries the current device's SM count once.  Errors: INVALID_ARG,
 * UNSUPPORTED, BUFFER_TOO_SMALL, ALIGNMENT, CUDA. */
DUO_API int duo_kv_alloc(const duo_kv_desc* desc, void* dev_buf, size_t buf_bytes,
                 duo_stream_t stream, duo_kv** out);

/* Release the host handle.  dev_buf stays the caller's.  NULL is a no-op. */
DUO_API int duo_kv_free(duo_kv* kv);

/* Fill *out with the device views of `layer`.  Host only.  This is also the
 * way to read the position table (the original position of every ring
 * slot, kept after eviction): out->positions is its device address, which
 * the caller copies or reads with its own stream, so the library needs no
 * separate call that copies it (and stays free of allocation and
 * synchronisation). */
DUO_API int duo_kv_layer_view_get(const duo_kv* kv, int32_t layer, duo_kv_layer_view* out);

/* Append tokens to one layer's cache (append + evict).
 *   k_new, v_new: [B][n_kv][n_new_max][d] bf16, token i of sequence b sits
 *                 at absolute position len_before[b] + i;
 *   len_before:   device int32 [B], tokens already appended to that layer;
 *   n_new:        device int32 [B] tokens to append per sequence
 *                 (<= n_new_max), or NULL = n_new_max for every sequence.
 * Retrieval head: token p goes to row p (p >= capacity sets
 * DUO_STATUS_OVER_CAPACITY and is dropped).  Streaming head: of the appended
 * tokens only those the ring still holds afterwards are written -- p < S or
 * p >= len_before + n_new - W -- to slot p (p < S) or S + (p - S) mod W, and
 * positions[b][slot] = p; when len_before[b] == 0 the slots this call does
 * not fill are reset to -1.  Following the DuoAttention guide's simulation
 * (append_token) and the sliding-window ring of "Attention Variants and
 * Memory Efficiency"; the result equals appending the tokens one at a time.
 * FP8 caches store each value's code (see duo_kv_desc) instead of its bits.
 * Decode order per layer: append the new token, then duo_decode_attn (or
 * both in one call: duo_decode_step).
 * Prefill order per layer: duo_prefill_attn on the chunk, then append it. */
DUO_API int duo_kv_append(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                  const int32_t* len_before, const int32_t* n_new, int32_t n_new_max,
                  duo_stream_t stream);

/* duo_kv_append for a cache whose retrieval rows hold only a slice of each
 * sequence's positions, [r_pos_begin[b], r_pos_end[b]) (device int32 [B]),
 * stored from row 0: position p goes to row p - r_pos_begin[b]; positions
 * outside the slice are not written to retrieval heads.  Streaming heads and
 * the position table are updated exactly as by duo_kv_append (positions are
 * absolute).  This is the storage of a sequence split over devices: each
 * device appends every token, its retrieval heads keep their own slice.  Not
 * on the pages (their plan has one device); see duo_decode_attn_rows. */
DUO_API int duo_kv_append_rows(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                               const int32_t* len_before, const int32_t* n_new, int32_t n_new_max,
                               const int32_t* r_pos_begin, const int32_t* r_pos_end, duo_stream_t stream);

/* Workspace bytes duo_decode_attn needs (host only). */
DUO_API int duo_decode_workspace_bytes(const duo_kv* kv, size_t* bytes);

/* Decode attention for one layer, every sequence and query head at once
 * (the DuoAttention guide, section 2, "Retrieval Heads vs. Streaming
 * Heads": full attention for retrieval heads, attention over the sinks and
 * the recent window for streaming heads; window rule from "Attention
 * Variants and Memory Efficiency", "Sliding-Window and Mixed Attention":
 * keys max(0, t - W + 1) .. t; query head h reads KV head h / G, as in
 * "Multi-Query and Grouped-Query Attention").
 *   q:    [B][Hq][d] bf16, the query of each sequence's newest token;
 *   len:  device int32 [B], tokens held after this step's append (>= 1);
 *         the query sits at position t = len[b] - 1;
 *   scale: softmax scale (typically 1/sqrt(d));
 *   out:  [B][Hq][d] fp32, softmax(scale * q.K^T) V over the head's keys:
 *         retrieval head: all positions 0..t; streaming head: positions
 *         j <= t with j < S or j >= t - W + 1 (the sinks and the window);
 *   lse:  optional [B][Hq] fp32, natural log of the softmax denominator;
 *   workspace: device scratch of >= duo_decode_workspace_bytes bytes
 *         (no initialisation needed; overlapping calls must not share it).
 * Split-K over each head's keys with a log-sum-exp merge; the result does
 * not depend on how the keys are split beyond rounding.  At head_dim 128
 * the merge happens inside the one kernel launch, counted by the handle's
 * per-(sequence, KV head) counters, which return to 0 when the launch ends:
 * decode calls on one handle must therefore be ordered (one stream, or
 * events), as they also share the status word. */
DUO_API int duo_decode_attn(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* len,
                    float scale, float* out, float* lse, void* workspace, size_t workspace_bytes,
                    duo_stream_t stream);

/* One decode step of one layer: append each sequence's new token, then
 * decode attention over the cache that includes it.  The result (cache
 * contents, out, lse, status) is that of
 *   duo_kv_append(kv, layer, k_new, v_new, len_before, NULL, 1, stream);
 *   duo_decode_attn(kv, layer, q, len, scale, out, lse, workspace, ...);
 * with the same arguments, which this call checks before launching
 * anything.  k_new, v_new: [B][n_kv][1][d] bf16; len_before, len: device
 * int32 [B].  The two kernels overlap (head_dim 128): the attention kernel
 * streams every key tile the append does not write while the append runs,
 * and waits for it only before the last tile of each retrieval head and
 * the streaming rings (the tiles that may hold the new token).  This relies
 * on len[b] = len_before[b] + 1 for every sequence, which the kernel
 * checks; if any sequence differs it waits for the append before reading
 * anything, as duo_decode_attn does.  Every input must be in place when the
 * call is made (produced by work already in the stream). */
DUO_API int duo_decode_step(duo_kv* kv, int32_t layer, const uint16_t* k_new, const uint16_t* v_new,
                            const int32_t* len_before, const uint16_t* q, const int32_t* len, float scale,
                            float* out, float* lse, void* workspace, size_t workspace_bytes, duo_stream_t stream);

/* Decode attention over chosen rows.  Like duo_decode_attn, except that
 * the keys come from explicit row ranges instead of the sequence length:
 *   retrieval heads: cache rows [r_begin[b], r_end[b]) (r_begin may be NULL
 *     = 0; both device int32 [B], clamped to [0, capacity]);
 *   streaming heads: ring slots [0, s_len[b]) (device int32 [B], clamped to
 *     S + W; NULL = no slots).
 * A head with no rows gets out = 0 and lse = -inf, so it contributes nothing
 * to duo_lse_merge.  No status bits are set by this call.  Two uses:
 *   - sequence split over devices: each device holds a slice of every
 *     retrieval head (duo_kv_append_rows) and decodes rows [0, slice); one
 *     device also passes s_len for the streaming heads; the partial (out,
 *     lse) are exchanged and combined with duo_lse_merge;
 *   - the streaming part of the gated forward on a full cache: sinks = rows
 *     [0, S) and window = rows [t-W+1, t+1) of each head, merged with
 *     duo_lse_merge (see duo_alpha_blend). */
DUO_API int duo_decode_attn_rows(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* r_begin,
                                 const int32_t* r_end, const int32_t* s_len, float scale, float* out, float* lse,
                                 void* workspace, size_t workspace_bytes, duo_stream_t stream);

/* Combine attention results over disjoint key sets: for each of `rows`
 * rows, out = sum_r exp(lse_r - LSE) part_out[r], LSE = log sum_r exp(lse_r).
 *   part_out: device fp32 [parts][rows][d]; part_lse: [parts][rows] (natural
 *   log of each part's softmax denominator; -inf = the part saw no key);
 *   out: [rows][d]; lse: optional [rows].  Rows where every part is -inf get
 *   out = 0, lse = -inf.  Exact up to rounding (the softmax over a union is
 *   the log-sum-exp weighted mix of the softmaxes over its parts). */
DUO_API int duo_lse_merge(int32_t parts, int32_t rows, int32_t d, const float* part_out, const float* part_lse,
                          float* out, float* lse, duo_stream_t stream);

/* Gated attention of the DuoAttention guide's head identification (section
 * 3, item 2): out = alpha[h] * full_out + (1 - alpha[h]) * stream_out for
 * query head h.  alpha: device fp32 [num_q_heads]; full_out, stream_out,
 * out: [batch][num_q_heads][d] fp32 (out may alias either input). */
DUO_API int duo_alpha_blend(int32_t batch, int32_t num_q_heads, int32_t d, const float* alpha,
                            const float* full_out, const float* stream_out, float* out, duo_stream_t stream);

/* Bytes of device scratch built into the library for
 * duo_decode_attn_static_ws (a file-scope __device__ array). */
#define DUO_STATIC_WS_BYTES (4u << 20)

/* Decode attention exactly as duo_decode_attn, for callers that cannot
 * allocate device memory: a plugin whose host program owns all device
 * memory and passes it only its inputs and outputs, or a serving loop that
 * must not call cudaMalloc (it can synchronise the device and can fail with
 * out-of-memory in the middle of a request).  Instead of a caller workspace
 * the call uses the library's own DUO_STATIC_WS_BYTES (4 MiB) scratch array,
 * which every GPU that loads the library holds until the process exits; the
 * call itself allocates nothing.
 *   - Limit: duo_decode_workspace_bytes(kv) must be <= DUO_STATIC_WS_BYTES,
 *     otherwise DUO_ERR_WORKSPACE is returned and nothing is launched.
 *   - The handle's device must be the current device (else INVALID_ARG).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture begins.
 *   - All calls on a device share the one array: calls whose kernels can
 *     overlap on the GPU (e.g. on unordered streams) race and corrupt each
 *     other's results.  Leftover contents from earlier calls do no harm.
 * The pages describe no counterpart of this entry point; it only changes
 * where the scratch memory comes from. */
DUO_API int duo_decode_attn_static_ws(duo_kv* kv, int32_t layer, const uint16_t* q, const int32_t* len,
                                      float scale, float* out, float* lse, duo_stream_t stream);

/* Workspace bytes duo_prefill_attn needs for chunks of up to `chunk` rows
 * (host only): fp16 copies of the values one call reads -- the retrieval
 * heads' cached rows, the streaming rings and the chunk --, bf16 copies of
 * the cached keys for FP8, INT4 or paged caches, and the partial outputs of
 * query tiles whose keys are shared by two CTAs (2 x B x Hq x chunk x d
 * fp32 plus their log-sum-exps), and each (sequence, KV head)'s value
 * range (a few hundred bytes). */
DUO_API int duo_prefill_workspace_bytes(const duo_kv* kv, int32_t chunk, size_t* bytes);

/* Chunked-prefill attention for one layer (before the chunk is appended).
 *   q:          [B][Hq][chunk][d] bf16, rows at positions prefix[b] + i;
 *   k_chunk, v_chunk: [B][n_kv][chunk][d] bf16, the chunk's own keys/values;
 *   prefix_len: device int32 [B], tokens already in the cache (P);
 *   out:        [B][Hq][chunk][d] fp32;
 *   workspace:  device scratch of >= duo_prefill_workspace_bytes(kv, chunk)
 *               bytes, 256-byte aligned (no initialisation; calls that may
 *               overlap must not share it).
 * Row i reads keys at positions j <= P + i ("Attention Variants and
 * KV-Cache Compression", "When Is Reuse Exact?"): retrieval heads all of
 * them (prefix from the cache, the rest from k_chunk); streaming heads only
 * j < S or j >= P + i - W + 1 (the sinks and the window, read from the ring
 * and from k_chunk).  The DuoAttention guide's "Hardware-Fused Prefill":
 * dense causal attention for retrieval heads, block-sparse sink + local
 * attention for streaming heads.  Products of probabilities and values run
 * in fp16 (fp32 accumulation) on copies of the values scaled per
 * (sequence, KV head) by a power of two 2^-E, E >= 0 the smallest exponent
 * that keeps the head's |v| * 2^-E below 2^15, and the output is multiplied
 * back by 2^E: any finite bf16 value is accepted (E = 0, no scaling, for
 * heads whose values all lie below 2^15).  FP8 caches:
 * the cached prefix is read dequantised (codes times the scales), the
 * chunk's own keys and values exactly as given; the value scales of the
 * layer must lie in [2^-8, 2^7] (else UNSUPPORTED: probabilities are scaled
 * by them in fp16), and the workspace also holds bf16 copies of the cached
 * keys' codes.  Requirements: head_dim 128 (else UNSUPPORTED); chunk >= 1;
 * prefix_len[b] must equal the tokens appended so far (the ring state is
 * derived from it). */
DUO_API int duo_prefill_attn(duo_kv* kv, int32_t layer, const uint16_t* q, const uint16_t* k_chunk,
                     const uint16_t* v_chunk, const int32_t* prefix_len, int32_t chunk,
                     float scale, float* out, void* workspace, size_t workspace_bytes,
                     duo_stream_t stream);

/* Read the device status word into *status (host).  This call
 * synchronises `stream`.  If clear != 0 the word is reset to 0 afterwards,
 * and if DUO_STATUS_WAIT_TIMEOUT was set, the decode merge counters too (a
 * launch that gave up may have left them non-zero). */
DUO_API int duo_kv_read_status(duo_kv* kv, int32_t* status, int32_t clear, duo_stream_t stream);

/* Diagnostic of the bounded waits: launches one warp that waits on an
 * mbarrier nothing completes, with the bounded-wait routine every pipeline
 * wait of the attention kernels uses, limited to limit_ns (0 < limit_ns <= 1 s,
 * the kernels' own limit), after which it sets DUO_STATUS_WAIT_TIMEOUT in the
 * handle's status word exactly as a timed-out kernel does.  No fault, trap or
 * unbounded wait is involved; the stream and context stay usable.  For tests
 * of the timeout reporting (duo_kv_read_status). */
DUO_API int duo_kv_check_wait_timeout(duo_kv* kv, uint64_t limit_ns, duo_stream_t stream);

/* Paged caches: the device table that maps a sequence's positions to pages,
 * int32 [batch][max_pages]: entry [b][i] is the pool page (0 .. num_pages-1,
 * the same index in every layer's pool) holding positions
 * i*page_tokens .. (i+1)*page_tokens - 1 of sequence b, or -1 for none.
 * The table stays the caller's; the library reads it in later calls
 * (stream-ordered), so the caller updates it as sequences grow.  Host only;
 * INVALID_ARG on a contiguous cache or max_pages < 1. */
DUO_API int duo_kv_set_page_table(duo_kv* kv, const int32_t* d_table, int32_t max_pages);

/* Prefix sharing: make sequence dst continue from the first len tokens of
 * sequence src, in every layer (paged attention's block sharing, "Attention
 * Variants and Memory Efficiency", "What the Inference Runtime Can Change":
 * prefix sharing keeps one copy of the blocks of a common prefix).
 *   src, dst: sequence indices (different, < batch);
 *   len:      host int, tokens src holds (0 <= len <= capacity); afterwards
 *             dst holds the same len tokens and appends from position len.
 * Streaming heads (sinks, ring and position table) are copied.  Retrieval
 * heads of a contiguous cache copy rows [0, len).  Paged caches: the caller
 * first sets dst's page-table entries for the prefix's pages; an entry equal
 * to src's shares that pool page (nothing is copied), any other page
 * receives a copy of src's rows.  The page holding the last, partly filled
 * block of the prefix (len not a multiple of page_tokens) must differ
 * between the two (DUO_STATUS_SHARED_PAGE otherwise); shared pages must not
 * be written through either sequence afterwards (they hold positions < len,
 * which appends never revisit).  Sets DUO_STATUS_NO_PAGE for a missing page
 * and DUO_STATUS_BAD_LENGTH when src's newest ring slot does not hold
 * position len - 1 (src holds a different number of tokens).  One launch per
 * layer on `stream`, ordered like appends. */
DUO_API int duo_kv_fork(duo_kv* kv, int32_t src, int32_t dst, int32_t len, duo_stream_t stream);

/* Override the number of CTAs the decode kernel splits the keys over
 * (0 = one persistent wave, the default).  For tests of split invariance;
 * the workspace requirement grows with it. */
DUO_API int duo_kv_set_decode_ctas(duo_kv* kv, int32_t ctas);

/* Static text for a return code. */
DUO_API const char* duo_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* DUO_KV_H */
