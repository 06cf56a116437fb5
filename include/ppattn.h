/*
 * libppattn -- B200 (sm_100a) attention for Parallel Prompting.
 *
 * Source of the method: "Read Once, Answer Many: Parallel Prompting for
 * Shared-Context LLM Inference" (Zhao & Flanigan), project page, section
 * "How it works", and the arXiv abstract of the same paper.  P independent
 * questions about one document are decoded as P answer streams of a single
 * request.  Every decode step reads the document KV once for all P streams,
 * and a stream-id mask evaluated inside the attention kernel (no dense mask
 * tensor) keeps each answer conditioned only on the document and on its own
 * question and answer tokens.  Every stream's positions start right after the
 * document ("shared positions"), and a decode step has a fixed shape so it
 * can be captured in a CUDA graph.
 *
 * Mask rule implemented by every kernel here (same section, item 1): a query
 * of stream s at position p sees key j iff
 *     j is a document key (stream id 0, index < doc_len), or
 *     sid_j == s  and  pos_j <= p        (own stream, causally earlier or
 *                                         the query's own token).
 * The page numbers the document -1; this library numbers it 0 and the answer
 * streams 1..P (stream id -1 marks an inactive query row).
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless their name starts with h_.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   - The caller owns and allocates every buffer (KV cache, tags, q, o, lse,
 *     workspace).  The library allocates no device memory and keeps no
 *     device state between calls.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream), perform no host synchronisation and no allocation,
 *     and may be captured into a CUDA graph -- except pp_get_device_status,
 *     which synchronises.
 *   - A workspace holds one call's intermediate results (document partials,
 *     counters); calls that may run at the same time (on different streams)
 *     need separate workspaces.  Calls ordered on one stream may share one:
 *     each call initialises what it reads.
 *   - Host-side argument checks return an error before anything is
 *     launched.  Errors found on the device set bits of the layer's device
 *     status word (PP_DEV_*), read with pp_get_device_status.
 *   - Inputs q, k, v, sid, pos are never written.
 *   - bf16 device pointers must be 16-byte aligned.
 */
#ifndef PPATTN_H
#define PPATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PP_ABI_VERSION 1

typedef enum pp_status {
    PP_OK = 0,
    PP_ERR_INVALID_ARG = 1,     /* NULL / misaligned pointer, negative size   */
    PP_ERR_UNSUPPORTED = 2,     /* d not in {64,128}, P > P_max, P > 32767    */
    PP_ERR_CAPACITY = 3,        /* doc_len > doc_cap, workspace too small     */
    PP_ERR_CUDA = 4,            /* a CUDA launch or driver call failed        */
    PP_ERR_DEVICE_TIMEOUT = 5   /* pp_get_device_status: PP_DEV_TIMEOUT is set */
} pp_status;

/* Bits of the per-layer device status word (sticky; cleared by pp_kv_reset). */
#define PP_DEV_SEGMENT_OVERFLOW 0x1  /* append: stream segment full, row dropped */
#define PP_DEV_DOC_OUT_OF_RANGE 0x2  /* append: document position outside cache */
#define PP_DEV_BAD_STREAM       0x4  /* stream id > P_max, or a document query   */
#define PP_DEV_TIMEOUT          0x8  /* a bounded in-kernel wait gave up         */

/*
 * One attention layer's KV cache ("How it works": every KV slot carries a
 * stream id; the document KV is shared by all streams).
 *
 *   k_doc, v_doc  bf16 [H][doc_cap][d]   document block, head-major; document
 *                                        token i sits at index i (stream id 0,
 *                                        position i, both implicit).
 *   k_suf, v_suf  bf16 [P_max][H][S_cap][d]   one segment per answer stream:
 *                                        stream s (1..P_max) owns index s-1;
 *                                        its question and answer tokens in
 *                                        append order.
 *   sid           int16 [P_max][S_cap]   stream id of every segment slot.
 *   pos           int32 [P_max][S_cap]   position of every segment slot.
 *   len           int32 [P_max]          slots in use per segment; slots at or
 *                                        beyond len are never read.
 *   status        int32 [1]              device status word (PP_DEV_* bits).
 */
typedef struct pp_kv_layer {
    int32_t H, d, doc_cap, P_max, S_cap;
    int32_t reserved;
    uint16_t *k_doc, *v_doc;
    uint16_t *k_suf, *v_suf;
    int16_t *sid;
    int32_t *pos;
    int32_t *len;
    int32_t *status;
} pp_kv_layer;

/*
 * Options (NULL = all defaults).
 *   splits                  0 = automatic document split; else the number of
 *                           CTAs the document pass runs on (>= 1).
 *   ablation_doc_per_stream 1 = read the document once PER STREAM (one warp
 *                           per stream and head, no tensor cores) instead of
 *                           once per step: the batched-requests baseline of the
 *                           page's "Inside decode step" figure, kept to measure
 *                           the bytes Parallel Prompting saves.
 *   debug_inject_timeout    test only: 1 = the document pass's producer skips
 *                           its first copy, so the consumers' bounded waits
 *                           expire; the call then sets PP_DEV_TIMEOUT and
 *                           returns without hanging.
 *   wait_limit_log2         test only: 0 = default bound on in-kernel waits
 *                           (about 2^31 clock cycles); else 2^value cycles.
 *   events                  NULL, or 3 caller-created cudaEvent_t handles that
 *                           decode/prefill record on `stream` before the
 *                           document pass, after it, and after the suffix
 *                           pass with its merge (per-kernel timing with CUDA
 *                           events; the work done is unchanged).  During a
 *                           stream capture they are recorded as external
 *                           event-record nodes, i.e. at every graph replay.
 *   sibling_scan            1 = the suffix part as the pages' kernel does it:
 *                           every query scans the answer tokens of ALL
 *                           streams and the stream mask rejects the siblings'
 *                           (project page, section "More results"); same
 *                           result, kept to measure what per-stream segments
 *                           save.  Decode and question prefill only.
 *   suffix_slices           decode suffix pass, how its warps share the (row,
 *                           head) items: 0 = automatic (balanced when the
 *                           items would keep fewer than half of the warps
 *                           busy or segments may pass 512 keys),
 *                           1 = equal item counts, 2 = balanced by work (an
 *                           item longer than 8 chunks may be cut between
 *                           warps; needs the tensor-core document pass and
 *                           at most 4096 rows, else 1).  Same result.
 */
typedef struct pp_options {
    int32_t splits;
    int32_t ablation_doc_per_stream;
    int32_t debug_inject_timeout;
    int32_t wait_limit_log2;
    void **events;
    int32_t sibling_scan;
    int32_t suffix_slices;
} pp_options;

/* Human-readable name of a pp_status value. */
const char *pp_status_str(int32_t status);

/* PP_ABI_VERSION of the loaded library. */
int32_t pp_abi_version(void);

/* Zero len[] and the status word of a layer (asynchronous). */
pp_status pp_kv_reset(const pp_kv_layer *layer, void *stream);

/*
 * Free the segments of n streams for new questions (continuous batching:
 * a stream that has finished its answer hands its segment to the next
 * question of the request).  sid: device int16 [n], stream ids 1..P_max;
 * each listed stream's len is set to 0, so its old slots are invisible (a
 * slot is visible only below len) and the next pp_kv_append of that stream
 * writes from slot 0.  Ids outside 1..P_max set PP_DEV_BAD_STREAM and are
 * skipped; -1 entries are ignored, so a fixed-shape list can carry unused
 * places.  Asynchronous, capture-safe.  The pages have no counterpart: their
 * engine starts a new request for new questions.
 */
pp_status pp_kv_reset_streams(const pp_kv_layer *layer, const int16_t *sid, int32_t n,
                              void *stream);

/*
 * Append n rows to the cache ("How it works": each decode step appends one
 * token per stream; the document is written once as stream 0).
 *   k, v  bf16 [n][H][d];  sid int16 [n];  pos int32 [n].
 * Row i with sid 0 is written to document index pos[i] (0 <= pos < doc_cap,
 * else dropped + PP_DEV_DOC_OUT_OF_RANGE).  Row i with sid s in [1, P_max]
 * goes to slot len[s-1] + r of segment s-1, where r counts earlier rows of
 * the same stream in this call; its sid and pos are stored with it, and
 * len[s-1] advances.  A full segment drops the row and sets
 * PP_DEV_SEGMENT_OVERFLOW; sid > P_max sets PP_DEV_BAD_STREAM; sid < 0 rows
 * are skipped.  Two rows of one call at the same document position: which
 * of them lands is unspecified.  Two kernel launches; n = 0 launches
 * nothing.
 */
pp_status pp_kv_append(const pp_kv_layer *layer, const uint16_t *k, const uint16_t *v,
                       const int16_t *sid, const int32_t *pos, int32_t n, void *stream);

/*
 * Workspace bytes pp_decode_attn and pp_decode_step need for P query rows
 * (fp32 partial results of the split document pass; one int per row for
 * the stream lengths of a step whose append runs inside that pass; arrival
 * counters and fp32 partials for suffix items cut between warps; 0 when
 * doc_len is 0).  The split
 * plan depends on the SM count of the CURRENT device: query with the device
 * that will run the call.  Returns 0 on bad arguments or without a device.
 */
size_t pp_decode_workspace_bytes(int32_t P, int32_t H, int32_t d, int32_t doc_len,
                                 const pp_options *opt);

/*
 * Decode-step attention ("How it works": one query per stream per step; the
 * document K/V are read once for all P streams).
 *   q      bf16 [P][H][d]   query of row i (usually stream i+1's new token)
 *   q_sid  int16 [P]        stream of row i: 1..P_max, or -1 for an inactive
 *                           row (its o is 0 and its lse -inf)
 *   q_pos  int32 [P]        position of row i (shared positions: N + tokens
 *                           the stream has before this one)
 *   doc_len (host)          document keys 0..doc_len-1 are visible
 *   scale                   softmax scale (1/sqrt(d) for the usual model)
 *   o      bf16 [P][H][d]   output (round-to-nearest-even from fp32)
 *   lse    fp32 [P][H]      natural-log sum-exp of the scaled scores, or NULL
 *   ws     workspace of at least pp_decode_workspace_bytes(...) bytes
 * The stream's own K/V for this step must already be appended.  Rows with
 * sid 0 (document queries) or sid > P_max get o = 0 and PP_DEV_BAD_STREAM.
 */
pp_status pp_decode_attn(const pp_kv_layer *layer, int32_t doc_len, const uint16_t *q,
                         const int16_t *q_sid, const int32_t *q_pos, int32_t P, float scale,
                         uint16_t *o, float *lse, void *ws, size_t ws_bytes,
                         const pp_options *opt, void *stream);

/*
 * One decode step of a layer in one call: append each row's new token, then
 * attend ("How it works": a decode step appends one token per stream, then
 * every stream's query reads the shared document once and its own segment).
 *   k, v   bf16 [P][H][d]   the new tokens' keys and values; row i is
 *                           appended to stream q_sid[i] at position q_pos[i]
 *   the other arguments and the workspace size are those of pp_decode_attn.
 * The result equals pp_kv_append(k, v, q_sid, q_pos, P) followed by
 * pp_decode_attn(...) -- the same slots, tags, lengths, device flags and
 * outputs -- except that rows of stream 0 are not written to the document
 * (a decode step has no document rows; they are flagged PP_DEV_BAD_STREAM as
 * in pp_decode_attn).  With a document and at most 4096 rows the append runs
 * inside the document pass launch, on a warp that is otherwise idle, and the
 * suffix pass stores the advanced lengths: two kernel launches per layer
 * instead of four.  Otherwise (doc_len 0, more rows, or the ablation and
 * sibling-scan options) the append kernels run first.  k and v: 16-byte
 * aligned.  Asynchronous, capture-safe.
 */
pp_status pp_decode_step(const pp_kv_layer *layer, int32_t doc_len, const uint16_t *k,
                         const uint16_t *v, const uint16_t *q, const int16_t *q_sid,
                         const int32_t *q_pos, int32_t P, float scale, uint16_t *o, float *lse,
                         void *ws, size_t ws_bytes, const pp_options *opt, void *stream);

/*
 * pp_decode_attn for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is a library convenience.
 *
 * Some callers cannot obtain a workspace -- for example a plugin inside a host
 * application that owns all device memory and gives the plugin no allocator,
 * or a serving loop that forbids device allocation after start-up because
 * cudaMalloc can synchronise the device.  This call takes the same arguments
 * as pp_decode_attn minus the workspace; the caller still passes q, the tags,
 * o and lse.  The document pass's partials go to a scratch array built into
 * the library (PP_NOALLOC_SCRATCH_BYTES on every GPU that loads it, held until
 * the process exits).  It allocates nothing.
 *   - Returns PP_ERR_CAPACITY, launching nothing, when the call would need
 *     more than PP_NOALLOC_SCRATCH_BYTES (pp_decode_workspace_bytes tells how
 *     much it needs; 32 MiB covers P = 256, H = 32, d = 128, doc 16384 on a
 *     148-SM B200).
 *   - The first call on each device looks up the scratch address on that
 *     device (make it the current device); make that first call before any
 *     stream capture.
 *   - Every call shares the one scratch array: calls whose kernels overlap on
 *     the GPU (different streams, unordered) corrupt each other's results.
 *   - The looked-up address is kept for the life of the process.  A
 *     cudaDeviceReset frees the array behind it, so this call must not be
 *     used on a device after that device has been reset.
 *   - Invalid arguments get the same status as from pp_decode_attn
 *     (PP_ERR_INVALID_ARG, PP_ERR_UNSUPPORTED), checked before the size.
 */
#define PP_NOALLOC_SCRATCH_BYTES (32u << 20)
pp_status pp_decode_attn_noalloc(const pp_kv_layer *layer, int32_t doc_len, const uint16_t *q,
                                 const int16_t *q_sid, const int32_t *q_pos, int32_t P,
                                 float scale, uint16_t *o, float *lse, const pp_options *opt,
                                 void *stream);

/*
 * Workspace bytes pp_prefill_attn needs for R question rows: the document
 * pass's fp32 partial results (as for decode) and the question runs -- 16
 * bytes a row (whole groups of 256 rows), their count and a task counter
 * (one 256-byte block) -- which are needed with or without a document.
 */
size_t pp_prefill_workspace_bytes(int32_t R, int32_t H, int32_t d, int32_t doc_len,
                                  const pp_options *opt);

/*
 * Question prefill of all P questions in one call (the page's introductory
 * figure: the document and all questions go into one sequence, prefilled
 * once; each question gets its own answer stream that sees only the
 * document and its own question).
 *   q       bf16 [R][H][d]  question rows, any order (a question's rows
 *                           next to each other are read together: its
 *                           segment is copied once for all of them)
 *   q_sid   int16 [R]       stream of each row (1..P_max; -1 = inactive)
 *   q_pos   int32 [R]       position of each row (N + index in its question)
 *   o bf16 [R][H][d], lse fp32 [R][H] or NULL, ws as for decode.
 * The question rows' own K/V must already be appended (pp_kv_append).  Each
 * row sees the document and the rows of its own stream at positions <= its
 * own (causal within the question).  Row errors are flagged as for decode.
 */
pp_status pp_prefill_attn(const pp_kv_layer *layer, int32_t doc_len, const uint16_t *q,
                          const int16_t *q_sid, const int32_t *q_pos, int32_t R, float scale,
                          uint16_t *o, float *lse, void *ws, size_t ws_bytes,
                          const pp_options *opt, void *stream);

/* Workspace bytes pp_doc_prefill_attn needs for a document of doc_len tokens. */
size_t pp_doc_prefill_workspace_bytes(int32_t H, int32_t d, int32_t doc_len,
                                      const pp_options *opt);

/*
 * Document prefill: attention of the document's own tokens, done once for
 * all streams ("Read Once, Answer Many" project page, section "How it
 * works": the document is encoded once and shared; a document token, stream
 * id 0, sees the document tokens at or before its own position, i.e.
 * ordinary causal attention over the document).
 *   q   bf16 [doc_len][H][d]  query of document token i at row i (position i)
 *   o   bf16 [doc_len][H][d], lse fp32 [doc_len][H] or NULL
 *   ws  caller-owned, 256-byte aligned, >= pp_doc_prefill_workspace_bytes
 * The document's K/V rows 0 .. doc_len-1 must already be in the layer
 * (pp_kv_append with stream id 0).  Runs on the same tensor-core document
 * pass as decode, with row i masked to keys 0..i and the key tiles above a
 * row group's diagonal skipped; the per-stream ablation option is refused
 * (PP_ERR_UNSUPPORTED).  Other errors as for pp_decode_attn.  This call has
 * no counterpart in the pages' measurements; their document prefill runs in
 * the serving engine.
 */
pp_status pp_doc_prefill_attn(const pp_kv_layer *layer, int32_t doc_len, const uint16_t *q,
                              float scale, uint16_t *o, float *lse, void *ws, size_t ws_bytes,
                              const pp_options *opt, void *stream);

/*
 * Test aid: evaluate the mask predicate the attention kernels use.
 *   count_out int32 [nq]: number of keys query i sees (document included).
 *   mask_out  uint8 [nq][P_max*S_cap] or NULL: 1 where segment slot
 *             (s-1)*S_cap + t is visible to query i (slots >= len are 0).
 */
pp_status pp_debug_visibility(const pp_kv_layer *layer, int32_t doc_len, const int16_t *q_sid,
                              const int32_t *q_pos, int32_t nq, int32_t *count_out,
                              uint8_t *mask_out, void *stream);

/*
 * Test aid (host only, no device needed): the document split the attention
 * calls use for `rows` query rows, H heads and doc_len keys over `ctas` CTAs.
 * Writes to host array h_out (h_out_len >= 5 + 2*units entries):
 *   h_out[0..4] = T (key tiles per unit), units (row groups * H), W (total
 *   tiles), C (CTAs), max_chunks; then per unit u: h_out[5+2u] = first CTA
 *   and h_out[6+2u] = last CTA whose tile range covers unit u.
 */
pp_status pp_debug_split_plan(int32_t rows, int32_t H, int32_t doc_len, int32_t ctas,
                              int64_t *h_out, int32_t h_out_len);

/*
 * Test aid (host only): the split pp_doc_prefill_attn uses for a document of
 * doc_len tokens (rows = doc_len; unit (head, group g) holds only the key
 * tiles 0 .. min(T, 2g+2)-1).  Same output layout as pp_debug_split_plan,
 * with h_out[0] = T of a full unit.
 */
pp_status pp_debug_split_plan_causal(int32_t doc_len, int32_t H, int32_t ctas, int64_t *h_out,
                                     int32_t h_out_len);

/*
 * Test aid: the document pass's two base-2 exponentials on n device floats:
 * y_poly[i] from the FMA-pipe polynomial (range reduction + degree-3
 * minimax), y_hw[i] from the hardware ex2 instruction.  No counterpart on
 * the pages; it exists so tests can bound the polynomial's error.
 */
pp_status pp_debug_exp2(const float *x, float *y_poly, float *y_hw, int32_t n, void *stream);

/* Copy the layer's device status word to *h_status (synchronises stream).
 * Returns PP_ERR_DEVICE_TIMEOUT when the word has PP_DEV_TIMEOUT set (a
 * bounded in-kernel wait gave up: that call's outputs are not valid), with
 * *h_status written all the same; PP_OK otherwise, whatever the other bits
 * (they report dropped or rejected rows, not failed launches). */
pp_status pp_get_device_status(const pp_kv_layer *layer, int32_t *h_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PPATTN_H */
