/*
 * akv.h -- C ABI of libakv: tiered KV-history decode attention for NVIDIA B200 (sm_100a).
 *
 * One decode step attends a single new query per head over a long key/value history.
 * The history lives in tiers ("Context beyond VRAM", section "What I built": two
 * precision tiers with separate contracts):
 *   - an exact tier, BF16 keys and values, bit-identical to fully resident attention;
 *   - a compact tier for older history: each (token, KV head) vector is rotated by a
 *     Walsh-Hadamard transform, scaled by its L2 norm (stored as binary16) and coded as
 *     4-bit indices into a fixed 16-level Lloyd-Max table for N(0,1).  The GPU reads the
 *     codes directly; the query is rotated instead of the keys ("QuantForge V2
 *     Walkthrough", section 1 "Triton Fused Kernels": rotation preserves dot products).
 * Each tier is attended in fixed-size splits; every split writes a partial output and its
 * log-sum-exp ("Bringing a serving stack up on new silicon", section "What I built": the
 * attention statistic the memory layer needs), and the partials are merged exactly
 * ("Context beyond VRAM", "What I built": merged with exact attention arithmetic).
 * Older history can be staged from pinned host memory through a bounded device region
 * whose buffers are released only after every copy and kernel that touched them has
 * finished ("Context beyond VRAM", sections "My approach" and "What I built").
 *
 * Conventions for every call:
 *   - The caller owns all device memory and pinned host memory.  The library allocates
 *     no device memory; a stager owns only CUDA events and a small host struct.
 *   - Device pointers are plain CUDA device addresses.  Host arrays (lens, slot bases)
 *     are read during the call and not retained.
 *   - Work is enqueued on the caller's stream; no call synchronises the device except
 *     the stager's bounded waits and akv_stager_destroy.
 *   - Arguments are validated before anything is launched.  A refused call launches
 *     nothing and returns a negative akv_status; akv_last_error() (thread-local) then
 *     holds a one-line reason.  Errors found on the device (a page id outside the pool, a
 *     non-finite input) set bits of a caller-provided device int32 error word, which the
 *     caller reads after the stream has reached that point; akv_error_word_status maps
 *     the word to a status.
 *   - Supported shapes: head dim d in {64, 128}; G = Hq / Hkv in {1, 2, 4, 8}; split_tokens
 *     a multiple of 16 in [16, 1024].  Other shapes return AKV_ERR_UNSUPPORTED.
 *   - Not thread-safe per object; independent calls from several threads are safe.
 */
#ifndef AKV_H_
#define AKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define AKV_ABI_VERSION 2

/* Opaque CUDA stream (cudaStream_t); 0 is the legacy default stream. */
typedef struct CUstream_st* akv_stream_t;

typedef enum akv_status {
  AKV_OK = 0,
  AKV_ERR_INVALID = -1,      /* malformed argument (null pointer, negative size, misaligned) */
  AKV_ERR_UNSUPPORTED = -2,  /* valid but not implemented (head dim, group size, split size) */
  AKV_ERR_CUDA = -3,         /* a CUDA runtime call failed; akv_last_error names it */
  AKV_ERR_NOT_PINNED = -4,   /* a staging source is not page-locked host memory */
  AKV_ERR_BUDGET = -5,       /* a chunk does not fit one staging buffer */
  AKV_ERR_TIMEOUT = -6,      /* a staging buffer was still in use when the wait ran out */
  AKV_ERR_NONFINITE = -7,    /* device: an encoded vector held inf or NaN */
  AKV_ERR_RANGE = -8,        /* device: an encoded vector's norm overflows binary16 */
  AKV_ERR_BOUNDS = -9,       /* device: a page id outside [0, n_pages) */
  AKV_ERR_INTERNAL = -10     /* device: a kernel got less shared memory than its layout needs
                                (a library defect); it returned without reading or writing */
} akv_status;

/* Bits of the device error word. */
#define AKV_EFLAG_NONFINITE 0x1
#define AKV_EFLAG_RANGE 0x2
#define AKV_EFLAG_BOUNDS 0x4
#define AKV_EFLAG_TIMEOUT 0x8 /* a kernel's bounded wait for its own copies gave up */
#define AKV_EFLAG_INTERNAL 0x10 /* a kernel's shared-memory layout did not fit its launch */

int akv_abi_version(void);
const char* akv_last_error(void);
const char* akv_status_string(int status);
/* Most severe status encoded in an error word (AKV_OK for 0). */
akv_status akv_error_word_status(int32_t word);

/* The library's binary16 centroid table, ascending (host; 16 entries).  The library
 * solves for the 16-level Lloyd-Max quantiser of N(0,1) on the host at load time, makes
 * it odd-symmetric and rounds every level to binary16 (round to nearest even). */
void akv_centroids_f16(uint16_t out[16]);

/* ------------------------------------------------------------------------------------
 * Tiers
 * ------------------------------------------------------------------------------------ */

enum { AKV_TIER_BF16 = 0, AKV_TIER_CODES4 = 1 };

/* Tokens per page (paged tiers) and per code block (compact tier). */
#define AKV_PAGE_TOKENS 16

/* Bytes of one compact-tier block of 16 tokens for head dim d, then 16 little-endian
 * binary16 scales; 1056 bytes at d = 128.
 *   Key blocks: 16 code rows of d/2 bytes (token order; byte k of a row holds code 2k in
 *   its low nibble and code 2k+1 in its high nibble).
 *   Value blocks: 8 pair rows of d bytes; byte k of pair row r holds code k of token 2r in
 *   its low nibble and code k of token 2r+1 in its high nibble; the d bytes of pair row r
 *   are 8 units of d/8 bytes with unit u stored at position u ^ w(r), w(r) = 2 (r % 4)
 *   for d = 128 and 4 ((r / 2) % 2) for d = 64 (the tensor-core operand order, read
 *   without bank conflicts).
 * akv_encode_history writes both; other producers must follow the same layout. */
#define AKV_CODES4_BLOCK_BYTES(d) (16 * ((d) / 2) + 32)

/*
 * One tier of the history of a batch of B sequences, for one layer.
 *
 * Addressing of token t (0-based within the tier) of sequence b, KV head h:
 *   BF16, contiguous:   k + b*stride_seq + h*stride_head + t*stride_token        (elements)
 *   BF16, paged:        k + P*stride_seq + h*stride_head + (t%16)*stride_token,
 *                       P = page_table[b*page_table_stride + t/16]               (elements)
 *   CODES4, contiguous: block k + b*stride_seq + h*stride_head + (t/16)*stride_token,
 *                       token t%16 of that block                                 (blocks)
 *   CODES4, paged:      block k + P*stride_seq + h*stride_head, token t%16       (blocks)
 * The head dimension is contiguous.  V uses the same layout from base v.
 * BF16 bases must be 16-byte aligned and BF16 strides multiples of 8 elements; CODES4
 * bases must be 16-byte aligned.  Buffers must cover every addressed token: the library
 * cannot see allocation sizes, except that paged tiers check page ids against n_pages.
 *
 * lens[b] (host) is the number of tokens of sequence b in this tier (0 allowed).
 * slot_base[b] (host) is the partial-output slot of the tier's first split for sequence
 * b; split s (tokens [s*split_tokens, (s+1)*split_tokens) of the tier) goes to slot
 * slot_base[b] + s.  Splits are aligned to the start of the tier.
 *
 * rotation_signs (CODES4 only): bit i (word i / 32, bit i % 32) set negates coordinate i
 * before the Walsh-Hadamard transform -- a randomised rotation z = H (s . x) of the
 * compact form, read back as x = s . (H y) / d.  All zero is the plain transform.  The
 * encoder and the attention kernels take the signs from the compact tier, so a tier must
 * be read with the signs it was written with.  Bits at and above d are ignored.  (The
 * pages name only the trade-off between Hadamard and QR rotations; this is the variant
 * that keeps the fast transform.)
 */
typedef struct akv_tier {
  int32_t kind;                  /* AKV_TIER_BF16 or AKV_TIER_CODES4 */
  int32_t paged;                 /* 0 contiguous, 1 paged through page_table */
  const void* k;                 /* device */
  const void* v;                 /* device */
  const int32_t* page_table;     /* device [B][page_table_stride], paged tiers only */
  int64_t page_table_stride;     /* int32 entries between page-table rows */
  int64_t n_pages;               /* pages in the pool (paged tiers) */
  int64_t stride_seq;            /* contiguous: between sequences; paged: between pages */
  int64_t stride_head;           /* between KV heads */
  int64_t stride_token;          /* see the addressing above; ignored for paged CODES4 */
  const int32_t* lens;           /* host [B] */
  const int32_t* slot_base;      /* host [B] */
  uint32_t rotation_signs[4];    /* CODES4: coordinate sign flips before the rotation */
} akv_tier;

/* ------------------------------------------------------------------------------------
 * akv_append_tokens -- write each sequence's new token into a BF16 tier.
 *
 * A decode step first appends the new token's key and value to the history, then attends
 * ("Context beyond VRAM", "What I built": the step appends the new K/V and attends).  For
 * every sequence b < B with pos[b] >= 0, the key row new_k[b][h][:] and value row
 * new_v[b][h][:] of every KV head h go to token pos[b] of `tier`, addressed exactly as
 * attention reads it (contiguous strides, or the page table for paged tiers).
 * tier: kind BF16, paged or contiguous; its lens and slot_base are not used; its k and v
 * rows at the given positions are WRITTEN.  new_k, new_v: device bf16 [B][Hkv][d], 16-byte
 * aligned.  pos: host int32 [B], the tier-relative token index (negative: skip b).  A paged
 * position whose page id is outside the pool sets AKV_EFLAG_BOUNDS in *err_word (device, may
 * be NULL) and writes nothing for that sequence.  Validation errors launch nothing; B = 0
 * or all positions negative is a no-op.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------------------ */
akv_status akv_append_tokens(const akv_tier* tier, const int32_t* pos, int B, int Hkv, int d, const void* new_k,
                             const void* new_v, int32_t* err_word, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * akv_encode_history -- rotate, quantise and pack BF16 history into the compact tier.
 *
 * For every sequence b < B, KV head h < Hkv and token t < dst->lens[b], the BF16 key and
 * value vectors x at token t of src are encoded into token t of dst (the compact form of
 * the hybrid tier of "Context beyond VRAM", "What I built"):
 *   z = H x (unnormalised Sylvester-order Walsh-Hadamard transform, float64 butterflies
 *       h = 1, 2, ..., d/2 mapping (a, b) to (a + b, a - b));
 *   s = binary16(sqrt(sum of x_i^2)), the sum taken in float64 by pairwise halving;
 *   code_i = number of boundaries b_j = (c_j + c_{j+1}) / 2, j < 15, with z_i > s * b_j;
 *   s == 0 gives codes 7.
 * Every block touched is written whole: rows past dst->lens[b] in the last block hold the
 * zero-vector encoding (codes 7, scale 0).  A vector with a non-finite coordinate or a
 * norm that rounds to binary16 infinity is written as the zero-vector encoding and sets
 * AKV_EFLAG_NONFINITE / AKV_EFLAG_RANGE in *err_word (device int32, may be NULL).
 * src: kind BF16 (its lens and slot_base are not used).  dst: kind CODES4; its k and v
 * blocks are WRITTEN.  Codes and scales are bit-exact against the float64 definition.
 * ------------------------------------------------------------------------------------ */
akv_status akv_encode_history(const akv_tier* src, const akv_tier* dst, int B, int Hkv, int d,
                              int32_t* err_word, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * akv_decode_attend -- split-KV GQA decode attention over one or more tiers.
 *
 * q: device BF16 [B][Hq][d], contiguous.  Query head h reads KV head h / G, G = Hq/Hkv.
 * For every tier, sequence b with lens[b] > 0, split s and query head h it writes
 *   o_part[(slot*Hq + h)*d + i]  (float32)   and   lse_part[slot*Hq + h]  (float32)
 * with slot = slot_base[b] + s:  scores_t = softmax_scale * q_h . k_t over the split's
 * tokens, O = sum_t softmax(scores)_t v_t, LSE = ln sum_t exp(scores_t).  A compact tier
 * is attended in the rotated basis (q rotated once per split, outputs rotated back), over
 * the dequantised vectors x_hat = H (s * c[code] / sqrt d) / sqrt d.
 * Every slot must lie in [0, n_slots); slots of different splits must not coincide.
 * variant: AKV_VARIANT_AUTO (the faster path), AKV_VARIANT_SIMT (CUDA cores, float32
 * FMA) or AKV_VARIANT_MMA (tensor-core mma.sync across the GQA group).  For a given
 * variant and split layout the result does not depend on where the tokens are stored, so
 * a staged run equals the resident run bit for bit.  Page ids outside [0, n_pages) set
 * AKV_EFLAG_BOUNDS in *err_word (device, may be NULL) and read page 0 instead.
 * Streams: asynchronous on `stream`; work enqueued on `stream` after the call sees every
 * partial.  With one BF16 and one compact launch (tensor-core variants) and `stream` on the
 * current device, the library may run the BF16 launch on an internal stream of that device,
 * forked from and joined back to `stream` with events, so the two grids share the SMs (same
 * bits as launched in a row).
 * That internal stream serves every such call on the device: a call whose `stream` is being
 * captured into a graph must not run while another host thread enqueues such a call on the
 * same device, and a call captured into a graph must be made with the capturing stream's
 * device current.  The first such call on a device creates the stream and its two events;
 * make it before any capture.  Apart from an error message, no call allocates memory.
 * ------------------------------------------------------------------------------------ */
enum { AKV_VARIANT_AUTO = 0, AKV_VARIANT_SIMT = 1, AKV_VARIANT_MMA = 2 };

akv_status akv_decode_attend(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale,
                             const akv_tier* tiers, int n_tiers, int split_tokens,
                             float* o_part, float* lse_part, int64_t n_slots, int variant,
                             int32_t* err_word, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * akv_merge_lse -- exact log-sum-exp merge of split partials ("Context beyond VRAM",
 * "What I built": the tiers are merged with exact attention arithmetic).
 *
 * For sequence b and head h the partials in slots seq_slot_base[b] .. +seq_n_slots[b]-1
 * (host arrays) are merged in increasing slot order:
 *   M = max_s LSE_s, w_s = exp(LSE_s - M), L = sum_s w_s,
 *   o[(b*Hq + h)*d + i] = sum_s w_s O_s[i] / L,   lse[b*Hq + h] = M + ln L.
 * No finite partial (seq_n_slots[b] == 0, or all -inf) gives O = 0 and LSE = -inf.
 * o, lse: device float32 [B][Hq][d] and [B][Hq].
 * ------------------------------------------------------------------------------------ */
akv_status akv_merge_lse(const float* o_part, const float* lse_part, int64_t n_slots,
                         const int32_t* seq_slot_base, const int32_t* seq_n_slots, int B, int Hq,
                         int d, float* o, float* lse, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * akv_decode -- one whole decode step in one call: the split attention of every tier and
 * the exact log-sum-exp merge ("Context beyond VRAM", "What I built": recent context
 * exact, older history compact, the two merged with exact attention arithmetic).
 *
 * The call plans the akv_plan_slots layout itself (the tiers' slot_base arrays are ignored)
 * and enqueues the launches of akv_decode_attend and akv_merge_lse, so the result is theirs
 * bit for bit; the merge launch overlaps the attention launches' tail.
 *
 * workspace: caller-owned device scratch of at least akv_decode_workspace_size() bytes,
 * 256-byte aligned, holding the LSE and then the O partials; its contents need no
 * initialisation.  Calls that share a workspace must not overlap on the device.  o, lse:
 * device float32 [B][Hq][d], [B][Hq].  A smaller workspace gives AKV_ERR_BUDGET.
 * ------------------------------------------------------------------------------------ */
akv_status akv_decode_workspace_size(int B, int Hq, int Hkv, int d, const akv_tier* tiers, int n_tiers,
                                     int split_tokens, size_t* bytes);
akv_status akv_decode(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale, const akv_tier* tiers,
                      int n_tiers, int split_tokens, void* workspace, size_t workspace_bytes, float* o, float* lse,
                      int variant, int32_t* err_word, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * akv_decode_host -- one decode step with the query and the results in page-locked host
 * memory: the end-to-end form of akv_decode_attend followed by akv_merge_lse.  No
 * counterpart in the pages, which pass device tensors between their operators.
 *
 * q_host: page-locked host BF16 [B][Hq][d], 16-byte aligned.  o_host, lse_host:
 * page-locked host float32 [B][Hq][d] and [B][Hq].  The call plans its own slots (the
 * tiers' slot_base arrays are ignored) and enqueues on `stream`: the query copy into the
 * workspace, the split attention of every tier, the merge, and the results into o_host and
 * lse_host.  They are valid once that work has completed (synchronise the stream or an
 * event recorded after the call); the host must not write q_host or read the outputs before.
 * Transfers: where the driver reports that a host array lies wholly inside one page-locked
 * allocation mapped for the device, the GPU reads the query over PCIe with a small kernel and
 * the merge writes the outputs there directly, so the step's kernels overlap their launches;
 * otherwise, or with flags AKV_HOST_COPY_ENGINE, the copy engine moves them.  Either way the
 * results are the bits of akv_decode_attend + akv_merge_lse on the same inputs.
 * workspace: caller-owned device scratch of at least akv_decode_host_workspace_size() bytes,
 * 256-byte aligned; calls that share it must not overlap on the device.
 * Refusals: a host array that is not page-locked -> AKV_ERR_NOT_PINNED; a small workspace
 * -> AKV_ERR_BUDGET; the rest as akv_decode_attend.
 * ------------------------------------------------------------------------------------ */
#define AKV_HOST_COPY_ENGINE 0x1
akv_status akv_decode_host_workspace_size(int B, int Hq, int Hkv, int d, const akv_tier* tiers, int n_tiers,
                                          int split_tokens, size_t* bytes);
akv_status akv_decode_host(const void* q_host, int B, int Hq, int Hkv, int d, float softmax_scale,
                           const akv_tier* tiers, int n_tiers, int split_tokens, void* workspace,
                           size_t workspace_bytes, float* o_host, float* lse_host, int flags, int variant,
                           int32_t* err_word, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * akv_decode_static -- akv_decode without a workspace argument, for callers that cannot
 * allocate device memory when they decode: a plugin whose process memory pool belongs to
 * another framework, or a serving loop that has frozen allocation so that no call can block
 * on the allocator or synchronise the device.  (It launches kernels, so like every CUDA
 * call it must not be made from a host function enqueued on a stream.)  The pages have no
 * counterpart: their engine always owns its memory.
 *
 * The scratch is a fixed array of AKV_DECODE_STATIC_MAX_BYTES in this library's device
 * memory, held by every GPU that loads the library until the process exits.  The first call
 * on each device looks up the array's device address while that device is current; under
 * CUDA's lazy module loading that lookup also loads the library's device code on the
 * device, which reserves the array and may block.  So make one warm-up call on each device
 * before freezing allocation or starting a stream capture.  After it, a call allocates no
 * memory, on the device or the host (the first call that runs two tiers side by side also
 * creates the internal stream and events akv_decode_attend describes).  A step whose
 * partials do not fit (see akv_decode_workspace_size), or with more than
 * AKV_DECODE_STATIC_MAX_SEQ sequences or 8 tiers, returns AKV_ERR_BUDGET /
 * AKV_ERR_UNSUPPORTED and launches nothing.  Every call shares the array: it keeps the last
 * call's values, and calls whose work overlaps on the GPU race -- order them.  Arguments and
 * results are those of akv_decode, bit for bit.
 * ------------------------------------------------------------------------------------ */
#define AKV_DECODE_STATIC_MAX_BYTES (8u << 20)
#define AKV_DECODE_STATIC_MAX_SEQ 1024
akv_status akv_decode_static(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale,
                             const akv_tier* tiers, int n_tiers, int split_tokens, float* o, float* lse,
                             int variant, int32_t* err_word, akv_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Context checkpoints -- suspend a context to a file and resume it without recomputation
 * ("Context beyond VRAM", "What I built": a checkpointed context lifecycle).  A context is
 * whatever host spans its owner names (the pinned history of every layer, compact code
 * rows, ...) plus n_meta uint64 values that describe them (layer count, lengths, steps).
 *
 * File layout (little-endian): the 8 bytes "AKVCKPT1", uint32 version (1), uint32 n_meta,
 * uint32 n_spans, uint32 0, n_meta uint64 values, then per span uint64 byte count and
 * uint32 CRC-32 (IEEE 802.3, reflected polynomial 0xEDB88320) with uint32 0, then the span
 * bytes in order.
 *
 * akv_checkpoint_write: spans[i] are host pointers (pinned or pageable) of span_bytes[i]
 * bytes.  The file is written to `path` plus ".tmp" and renamed onto `path` once complete,
 * so a failed write never leaves a partial file under `path`.  I/O failures return
 * AKV_ERR_INVALID with the system's message.  Synchronous; the caller orders it after the
 * device work that produced the spans.
 * akv_checkpoint_info: reads the counts, the meta values (up to *n_meta) and the span
 * sizes (up to *n_spans); on return *n_meta and *n_spans hold the file's counts.
 * akv_checkpoint_read: reads every span into caller buffers whose sizes must equal the
 * recorded ones.  A file whose magic, version, counts, sizes or CRC-32 do not match is
 * refused with AKV_ERR_INVALID (the buffers then hold unspecified bytes).
 * ------------------------------------------------------------------------------------ */
akv_status akv_checkpoint_write(const char* path, const uint64_t* meta, int n_meta, const void* const* spans,
                                const uint64_t* span_bytes, int n_spans);
akv_status akv_checkpoint_info(const char* path, uint64_t* meta, int* n_meta, uint64_t* span_bytes, int* n_spans);
akv_status akv_checkpoint_read(const char* path, void* const* spans, const uint64_t* span_bytes, int n_spans);

/* ------------------------------------------------------------------------------------
 * akv_plan_slots -- host helper: the standard slot layout.
 *
 * Sequence-major: sequence b owns a contiguous run of slots holding tier 0's splits,
 * then tier 1's, and so on (ceil(tier_lens[i][b] / split_tokens) splits per tier).
 * Writes tier_slot_base[i][b], seq_slot_base[b], seq_n_slots[b] and *n_slots (all host).
 * ------------------------------------------------------------------------------------ */
akv_status akv_plan_slots(int B, int n_tiers, const int32_t* const* tier_lens, int split_tokens,
                          int32_t* const* tier_slot_base, int32_t* seq_slot_base,
                          int32_t* seq_n_slots, int64_t* n_slots);

/* ------------------------------------------------------------------------------------
 * Staging: pinned host history through a bounded device region ("Context beyond VRAM",
 * "My approach": pinned host memory is the authoritative copy and the GPU a bounded
 * working set; "What I built": a buffer is released only after every copy and kernel
 * that touched it has finished).
 *
 * The region (caller-owned device memory, 256-byte aligned) is cut into n_buffers equal
 * buffers used round-robin.  Each buffer keeps the list of events recorded by the copies
 * and consumers that touched it since it was last filled.
 *
 * akv_stage_chunk: take the next buffer; make sure every event on its list has fired;
 *   copy `bytes` from pinned_src (page-locked host memory, else AKV_ERR_NOT_PINNED) with
 *   cudaMemcpyAsync on copy_stream, ordered after every akv_stage_writeback of this stager
 *   still in flight whose host range overlaps the source (copy_stream waits for it on the
 *   device); record the copy's event.  bytes larger than one
 *   buffer gives AKV_ERR_BUDGET; bytes == 0 acquires the buffer without copying (the
 *   caller fills it on the device).  timeout_ms >= 0: the host polls the events for at most
 *   timeout_ms and returns AKV_ERR_TIMEOUT, leaving the buffer untouched, if one is still
 *   pending.  timeout_ms < 0: the host does not wait; copy_stream waits for the events
 *   on the device instead.  Returns the buffer index and its device address.
 * akv_stager_use: make consumer_stream wait for the buffer's latest copy.
 * akv_stager_release: record on consumer_stream that the consumer's work on the buffer
 *   is enqueued; the buffer is reused only after that event fires.
 * akv_stage_writeback: copy bytes from the buffer at byte offset to pinned host memory on
 *   stream, ordered after the buffer's copy, and add the copy to the buffer's list.
 * akv_stager_destroy: wait (host) for every listed event, then free the stager.
 * All events are created with timing disabled (timing events serialise copies).
 * ------------------------------------------------------------------------------------ */
typedef struct akv_stager akv_stager;

akv_status akv_stager_create(void* dev_region, size_t region_bytes, int n_buffers, akv_stager** out);
akv_status akv_stage_chunk(akv_stager* st, const void* pinned_src, size_t bytes, akv_stream_t copy_stream,
                           int timeout_ms, int* buf_index, void** dev_ptr);
akv_status akv_stager_use(akv_stager* st, int buf_index, akv_stream_t consumer_stream);
akv_status akv_stager_release(akv_stager* st, int buf_index, akv_stream_t consumer_stream);
akv_status akv_stage_writeback(akv_stager* st, int buf_index, size_t offset, void* pinned_dst, size_t bytes,
                               akv_stream_t stream);
akv_status akv_stager_destroy(akv_stager* st);

/* ------------------------------------------------------------------------------------
 * akv_staged_decode -- one decode step of one layer whose history lives in pinned host
 * memory, in one call ("Context beyond VRAM", "What I built": the fence-safe staging
 * pipeline -- the step appends the new K/V, stages the history through the bounded device
 * region, attends and merges, and a buffer is reused only after everything that touched it
 * has finished).
 *
 * hist->host holds the layer's rows from token 0, pinned:
 *   AKV_TIER_BF16:   token rows [n][K | V][Hkv][d] bf16 (2 Hkv d 2 bytes per token);
 *   AKV_TIER_CODES4: 16-token block rows [n / 16][K | V][Hkv][AKV_CODES4_BLOCK_BYTES(d)].
 * The history is cut into chunks of hist->chunk_tokens tokens (a multiple of split_tokens,
 * and for CODES4 of 16); chunk c is staged with akv_stage_chunk on copy_stream, attended on
 * compute_stream into slots [c chunk / split, ...) and released.  new_row (device bf16
 * [2][Hkv][d], BF16 histories only, may be NULL) is the new token: it is appended at
 * position hist->n_tokens -- written into its staged chunk before that chunk is attended --
 * and written back to its host row (so the next step's copy of that chunk waits for it).
 * window (may be NULL): a device BF16 tier of one sequence attended after the history into
 * the following slots (the exact window of a staged hybrid history; the caller appends
 * to it).  The splits of the history, then of the window, are merged in order into o, lse
 * (device float32 [Hq][d], [Hq]).  o_part / lse_part: device scratch of n_slots slots.
 * Results equal akv_decode_attend + akv_merge_lse over the same tokens and split layout, bit
 * for bit (a staged run equals a resident run).  Refusals: as the calls it makes, plus
 * AKV_ERR_BUDGET when n_slots is too small; an error part-way leaves earlier chunks enqueued.
 * ------------------------------------------------------------------------------------ */
typedef struct akv_staged_history {
  int32_t kind;                 /* AKV_TIER_BF16 or AKV_TIER_CODES4 */
  int32_t chunk_tokens;         /* tokens per staged chunk */
  const void* host;             /* pinned host rows from token 0 */
  int64_t n_tokens;             /* tokens in the history before this step's append */
  uint32_t rotation_signs[4];   /* CODES4: the rotation signs the codes were written with */
} akv_staged_history;

akv_status akv_staged_decode(akv_stager* stager, const akv_staged_history* hist, const void* q, int Hq, int Hkv,
                             int d, float softmax_scale, int split_tokens, const void* new_row,
                             const akv_tier* window, float* o_part, float* lse_part, int64_t n_slots, float* o,
                             float* lse, int variant, int32_t* err_word, akv_stream_t copy_stream,
                             akv_stream_t compute_stream);

/* ------------------------------------------------------------------------------------
 * Window aging -- a live hybrid batch whose exact window ages into the compact tier during
 * decode ("Context beyond VRAM", "What I built": recent context exact, older history in
 * the compact form), one call per step.
 *
 * Sequence b keeps compact_len[b] compact tokens (a multiple of 16) and window_len[b] in
 * [W, W + 16) exact tokens, W = window_tokens.  The window is a ring of ring_pages
 * (>= W / 16 + 2) pages of 16 BF16 tokens: window pool page b * ring_pages + (head + j) %
 * ring_pages holds the window's logical page j, where head = ring_head[b] is the ring slot
 * of its first page, and the window tier's page-table row b (ring_pages entries, device)
 * must say so.  The compact tier's page-table row b holds page_lists[b][0 ..
 * compact_len[b] / 16); as the sequence ages it takes page_lists[b][compact_len[b] / 16],
 * then the next.
 *
 * akv_aging_step, for every sequence: appends the new token (k_new, v_new: device bf16
 * [B][Hkv][d]) at window position window_len[b]; a window that reaches W + 16 tokens
 * encodes its oldest page into the sequence's next code page (akv_encode_history), enters
 * that page in the compact page table and rotates its window page-table row (both written
 * on the device by the call) -- then attends both tiers with the standard slot layout
 * (akv_plan_slots) into o_part / lse_part (n_slots slots) and merges into o, lse (device
 * float32 [B][Hq][d], [B][Hq]).  Everything is enqueued on `stream` (on a step that ages
 * no page the append may run on the library's side stream just before the window's launch,
 * joined back to `stream` like that launch); the context keeps the lengths on the host.  lists_dev: device int32 scratch of 2 B entries (the encode's page
 * lists).  A sequence with no code page left is refused (AKV_ERR_BUDGET) before anything is
 * enqueued.  The tiers' lens and slot_base are ignored.  Results equal the same calls made
 * one by one.  akv_aging_state reads the current lengths, ring heads and the number of pages
 * aged so far (host arrays of B entries, each may be NULL).  The context holds copies of
 * every host array of the description; it owns no device memory.
 * ------------------------------------------------------------------------------------ */
typedef struct akv_aging akv_aging;

typedef struct akv_aging_desc {
  int32_t B, Hq, Hkv, d, split_tokens;
  float softmax_scale;
  int32_t window_tokens;             /* W: a positive multiple of 16 */
  int32_t ring_pages;                /* window pages per sequence */
  akv_tier window;                   /* BF16, paged: B * ring_pages pool pages; page_table device [B][ring_pages] */
  akv_tier compact;                  /* CODES4, paged; page_table device [B][page_table_stride] */
  const int32_t* compact_len;        /* host [B] */
  const int32_t* window_len;         /* host [B] */
  const int32_t* ring_head;          /* host [B] */
  const int32_t* const* page_lists;  /* host [B] arrays of code pages, in the order they are taken */
  const int32_t* page_list_len;      /* host [B] */
  int32_t* lists_dev;                /* device int32 [2 B] scratch */
  float* o_part;                     /* device [n_slots][Hq][d] */
  float* lse_part;                   /* device [n_slots][Hq] */
  int64_t n_slots;
} akv_aging_desc;

akv_status akv_aging_create(const akv_aging_desc* desc, akv_aging** out);
akv_status akv_aging_step(akv_aging* ctx, const void* q, const void* k_new, const void* v_new, float* o, float* lse,
                          int variant, int32_t* err_word, akv_stream_t stream);
akv_status akv_aging_state(const akv_aging* ctx, int32_t* compact_len, int32_t* window_len, int32_t* ring_head,
                           int64_t* aged_pages);
akv_status akv_aging_destroy(akv_aging* ctx);

#ifdef __cplusplus
}
#endif

#endif /* AKV_H_ */
