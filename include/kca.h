/*
 * kca.h -- C ABI of the B200 (sm_100a) states-form KV-cache attention library
 *          (libkca.so).
 *
 * The operation (Karume v0.12.0 release notes, "Performance", items 1-3;
 * Karume v0.8.0 release notes, "Features", conversation-window item, and
 * "Breaking Changes", softmax NaN item):
 *
 *   For a query row at absolute position pos of one sequence and query head h,
 *   with KV head g = h / (n_q_heads / n_kv_heads):
 *     visible keys  J(pos) = [lo, pos],  lo = window > 0 ? max(0, pos-window+1) : 0
 *     s_j  = scale * <q[h,:], K[j,g,:]>                         (j in J(pos))
 *     out[h,:] = sum_j exp(s_j - max s) V[j,g,:] / sum_j exp(s_j - max s)
 *   A NaN score makes the row NaN; a row with no visible key is exactly 0.
 *
 * Prefill (attn_prefill): a chunk of chunk_rows <= 768 query rows at positions
 * chunk_start .. chunk_start+chunk_rows-1 of one sequence; every row sees the
 * cached rows before the chunk and the chunk's own rows up to itself
 * ("chunked prefill", 768-row chunks).  Decode (attn_decode): one query row per
 * sequence of a batch, at position ctx_len[b]-1.
 *
 * Fixed geometry: n_q_heads = 8, n_kv_heads = 1, head_dim = 256.  The
 * arguments are still passed so that a mismatch is an error, not a silent
 * misread.
 *
 * MEMORY LAYOUT (all row-major, no padding, device memory):
 *   K cache, V cache : [batch][capacity][n_kv_heads][head_dim], kv_dtype.
 *                      Row p of sequence b starts at element
 *                      ((b*capacity + p)*n_kv_heads)*head_dim.
 *                      attn_prefill works on one sequence: pass the pointers
 *                      of that sequence's row 0.
 *   q (prefill)      : [chunk_rows][n_q_heads][head_dim], q_dtype
 *   q (decode)       : [batch][n_q_heads][head_dim], q_dtype
 *   out              : [rows or batch][n_q_heads][head_dim], float32
 *   All of q, k_cache, v_cache, out must be 16-byte aligned; workspace
 *   256-byte aligned.
 *
 * PRECONDITIONS: the caller has written the K/V rows of every position the
 * call reads (for prefill the chunk's own rows too; for decode the row at
 * ctx_len-1).  Prefill requires ctx_len == chunk_start + chunk_rows.
 * Rows outside the union of the call's visible ranges are never read.
 * V must be finite on the rows of a tensor-core prefill chunk's visible
 * union: that path multiplies the exact zero probability of a masked key by
 * its V row, so an Inf or NaN in V at position p also reaches rows that do
 * not see p -- every output row of a 16-row tile whose work items cover p's
 * 128-key tile (attn_prefill_plan lists them) becomes NaN, where the
 * definition above leaves the rows that do not see p unaffected.  Rows that
 * see a non-finite V value are non-finite on every path.  The same holds
 * for attn_prefill_batch on a 16-bit cache with 2 or more rows per sequence
 * (multi-row units of up to 4 rows, 8 when a call has more than 4 rows per
 * sequence, share each key): V must be finite on
 * the union of a unit's visible ranges, else the unit's rows that do not
 * see the position are NaN too (in the dims where V is not finite).  The rows path (decode, short or
 * mixed-dtype chunks, one row per sequence) reads only the keys each row
 * sees.
 *
 * DTYPES: decode takes any q_dtype with any kv_dtype.  Prefill with
 * q_dtype == kv_dtype in {F16, BF16} and chunk_rows >= 16 runs on the
 * tcgen05 tensor-core path (16-row tiles, f32 accumulation).  Chunks of 3-15
 * such rows take that path too when their first row sees at least 12,288
 * keys (one pass over the keys beats one pass per row there).  Other chunks
 * of 2-15 rows on a 16-bit cache (mixed dtypes, or 2 rows) whose first row
 * sees at least 12,288 keys take multi-row units (the kernel of
 * attn_prefill_batch for one sequence).  The rows path serves every other
 * prefill combination: one unit per query row, mma.sync with
 * split-precision operands for 16-bit caches, CUDA-core f32 for f32 caches.
 * attn_force_path pins any of the three, so that tests can compare the
 * paths on the same inputs.
 *
 * QUERIES: the workspace-size and plan queries come one per operation
 * (attn_prefill_workspace_bytes, attn_decode_workspace_bytes,
 * attn_decode_partial_workspace_bytes; attn_prefill_plan, attn_decode_plan)
 * rather than as one call that takes an operation code, so that each takes
 * exactly the arguments of its operation.
 *
 * OWNERSHIP: every buffer is allocated and owned by the caller.  The library
 * allocates no device memory, keeps no per-call state and never synchronises
 * the stream.  Work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 * default stream) of the current device.
 *
 * WORKSPACE: scratch device memory of at least attn_*_workspace_bytes()
 * bytes for the same arguments on the same device.  Its first
 * KCA_WORKSPACE_HEADER bytes are the header: a device status word in bytes
 * [0, 256) (read it with attn_device_status) and, in the rest, merge
 * counters: one per (row, head) with which the tensor-core rows kernel
 * elects the CTA that merges a row's partials, one per multi-row unit with
 * which the tcgen05 kernel of attn_prefill_batch elects the split that
 * merges a unit's; every call leaves them at zero again.  Zero the
 * header once after allocation (attn_workspace_init), and again after a call
 * that recorded a device error.  Calls that run concurrently must not share a
 * workspace or an output buffer.
 *
 * ERRORS: every entry point validates all of its arguments on the host before
 * touching the GPU and returns a negative KCA_ERR_* without launching
 * anything.  KCA_ERR_CUDA reports a failed CUDA runtime call (launch
 * configuration, driver entry point); device-side faults are not possible by
 * design, and the only device-side error (a bounded wait inside the tensor-core
 * kernel that ran out) is recorded in the workspace status word.
 */
#ifndef KCA_H
#define KCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types */
#define KCA_F32 0
#define KCA_F16 1
#define KCA_BF16 2
/* packed int8 K rows of the quantised-dot calls: 256 int8 codes, the row's
 * f32 scale at byte 256, 12 zero bytes (272 bytes, 16-byte aligned) */
#define KCA_I8 3
#define KCA_I8_ROW_BYTES 272

/* status codes */
#define KCA_OK 0
#define KCA_ERR_NULL (-1)       /* a required pointer is NULL                      */
#define KCA_ERR_GEOMETRY (-2)   /* heads / head_dim other than 8 / 1 / 256         */
#define KCA_ERR_DTYPE (-3)      /* unknown dtype code                              */
#define KCA_ERR_RANGE (-4)      /* rows, positions, capacity, batch or scale       */
#define KCA_ERR_WORKSPACE (-5)  /* workspace too small or misaligned               */
#define KCA_ERR_ALIGN (-6)      /* q / k / v / out not 16-byte aligned             */
#define KCA_ERR_CUDA (-7)       /* a CUDA runtime call failed                      */
#define KCA_ERR_DEVICE (-8)     /* the device recorded an error (attn_device_status) */

/* limits (v0.8.0 release notes: maxChunkLength 768, maxPosition 131072) */
#define KCA_N_Q_HEADS 8
#define KCA_N_KV_HEADS 1
#define KCA_HEAD_DIM 256
#define KCA_MAX_CHUNK_ROWS 768
#define KCA_MAX_POSITION 131072
#define KCA_MAX_BATCH 256
#define KCA_MAX_BATCH_ROWS 15   /* rows per sequence of attn_prefill_batch */
/* status word (256 B) + 768 rows x 8 heads x 4-byte counters */
#define KCA_WORKSPACE_HEADER 24832

/*
 * attn_prefill -- chunked causal prefill of one sequence.
 * Passage: Karume v0.12.0 release notes, "Performance", item 1 (prefill of
 * the states-form attention, chunk plans of 16 or more rows reading each K/V
 * row once per row tile); v0.8.0 release notes, "Features", conversation-window
 * item (chunkLength <= maxChunkLength = 768, capacity <= maxPosition = 131,072,
 * both checked before any work).
 *   q_chunk      [chunk_rows][8][256] q_dtype, device
 *   k_cache/v_cache  the sequence's [capacity][1][256] kv_dtype rows, device
 *   capacity     rows the cache holds, 1..131072
 *   chunk_start  position of the chunk's first row, >= 0
 *   chunk_rows   1..768
 *   ctx_len      must equal chunk_start + chunk_rows, <= capacity
 *   window       <= 0: none; otherwise keys [pos-window+1, pos]
 *   scale        finite score scale > 0 (1/sqrt(256) for Gemma 4)
 *   out          [chunk_rows][8][256] float32, device
 *   workspace    >= attn_prefill_workspace_bytes(...) bytes, device
 * Returns KCA_OK or a negative KCA_ERR_*.
 */
int attn_prefill(const void *q_chunk, int32_t q_dtype,
                 const void *k_cache, const void *v_cache, int32_t kv_dtype,
                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                 int64_t chunk_start, int32_t chunk_rows, int64_t ctx_len, int32_t window,
                 float scale, float *out, void *workspace, size_t workspace_bytes,
                 void *stream);

/*
 * attn_decode -- one query row per sequence (split-context decode + merge).
 * Passage: Karume v0.12.0 release notes, "Performance", items 2-3 (one-row
 * decode plans whose QK and PV reductions are split in parallel, then
 * combined); v0.8.0 release notes, "Breaking Changes", softmax NaN item.
 *   q            [batch][8][256] q_dtype, device
 *   k_cache/v_cache  [batch][capacity][1][256] kv_dtype, device
 *   batch        1..256
 *   ctx_len      HOST array [batch], 0..capacity; the query sits at ctx_len[b]-1
 *                and ctx_len[b] == 0 yields an all-zero output row
 *   window, scale  as in attn_prefill
 *   out          [batch][8][256] float32, device
 *   workspace    >= attn_decode_workspace_bytes(batch, ctx_len, window) bytes, device
 *   stream       cudaStream_t the kernels are enqueued on
 * Returns KCA_OK or a negative KCA_ERR_* (nothing launched on error).
 */
int attn_decode(const void *q, int32_t q_dtype,
                const void *k_cache, const void *v_cache, int32_t kv_dtype,
                int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                int32_t batch, const int64_t *ctx_len, int32_t window,
                float scale, float *out, void *workspace, size_t workspace_bytes,
                void *stream);

/*
 * attn_prefill_batch -- short chunks of several sequences in one call: each
 * sequence b has `rows` query rows, at positions ctx_len[b] - rows ..
 * ctx_len[b] - 1 (speculative or multi-row decode steps), every row seeing
 * its sequence's keys as in attn_prefill.  With a 16-bit cache and rows > 1,
 * one launch of the multi-row tcgen05 kernel (units of up to 4 consecutive
 * rows of a sequence, 8 when rows > 4, so each K/V row crosses to the SM
 * once per unit; the union of the unit's keys cut into splits across the
 * GPU, merged in the same kernel, or by a second launch when a unit has
 * more than 16 splits); otherwise the rows path of decode (one unit per
 * row).  As in
 * tensor-core prefill, V must be finite on the rows of a unit's key union:
 * a masked key's zero probability multiplies its V row.
 * Passage: Karume v0.12.0 release notes, "Docs", ADR 0067 plan-size geometry
 * table (the 2-15-row plans between decode and the >= 16-row tiles), and
 * "Performance", item 3 (the parallel PV reduction serves plans under 16
 * rows).
 *   q            [batch][rows][8][256] q_dtype, device
 *   k_cache/v_cache  [batch][capacity][1][256] kv_dtype, device; each
 *                sequence's rows up to ctx_len[b] - 1 written
 *   batch        1..256;  rows 1..KCA_MAX_BATCH_ROWS
 *   ctx_len      HOST array [batch], rows..capacity
 *   window, scale  as in attn_prefill
 *   out          [batch][rows][8][256] float32, device
 *   workspace    >= attn_prefill_batch_workspace_bytes(batch, rows, ctx_len, window)
 * With rows = 1 this is attn_decode (the same plan and the same bits).
 * Returns KCA_OK or a negative KCA_ERR_* (nothing launched on error).
 */
int attn_prefill_batch(const void *q, int32_t q_dtype,
                       const void *k_cache, const void *v_cache, int32_t kv_dtype,
                       int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                       int32_t batch, int32_t rows, const int64_t *ctx_len, int32_t window,
                       float scale, float *out, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * attn_decode_dev -- attn_decode with the context lengths in DEVICE memory,
 * read by the kernels when they run, so that one captured launch (CUDA graph)
 * serves every decode step while the caller updates ctx_len_dev in place.
 * Passage: the one-row (decode) plan of Karume v0.12.0 release notes,
 * "Performance", items 2-3; the pages have no device-side context length:
 * it serves decode loops replayed from a CUDA graph, step after step.
 *   ctx_len_dev  DEVICE int64 [batch], 8-byte aligned; each value 0..ctx_bound,
 *                written before the call's kernels run (stream order)
 *   ctx_bound    HOST upper bound of every ctx_len_dev[b], 0..capacity.  The
 *                launch (grid, clusters, workspace) is planned for `batch`
 *                sequences at ctx_bound; each sequence then cuts its actual
 *                keys into the planned number of splits on the device.
 *   workspace    >= attn_decode_workspace_bytes(batch, {ctx_bound, ...}, window)
 * Everything else is as in attn_decode.  The host work of a call depends only
 * on the pointers, dtypes, capacity, batch, ctx_bound, window and scale, never
 * on the device values.  A device value outside 0..ctx_bound is never used to
 * address memory: that sequence's row is computed as an empty context (zeros)
 * and the status word records it (attn_device_status returns KCA_ERR_DEVICE,
 * detail = (10 << 24) | sequence).  ctx_len_dev must not be written while
 * the call runs.
 */
int attn_decode_dev(const void *q, int32_t q_dtype,
                    const void *k_cache, const void *v_cache, int32_t kv_dtype,
                    int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                    int32_t batch, const int64_t *ctx_len_dev, int64_t ctx_bound, int32_t window,
                    float scale, float *out, void *workspace, size_t workspace_bytes,
                    void *stream);

/*
 * attn_decode_static -- attn_decode for callers that cannot allocate device
 * memory: code running where cudaMalloc is unavailable or forbidden (inside a
 * host callback, a custom allocator's own path, a memory pool that admits no
 * further allocations, a runtime that only hands out the tensors it owns).
 * The paper has no counterpart to this entry point.
 *
 * Arguments, layouts, semantics and errors are those of attn_decode, minus
 * the workspace: the per-split partials go to a file-scope device array of
 * KCA_STATIC_SCRATCH_BYTES (16 MiB) that every GPU loading the library holds
 * until the process exits.  A call whose plan needs more than that (many
 * sequences next to a very long one) returns KCA_ERR_WORKSPACE without
 * launching.  The first call on a device looks the array's address up
 * (cudaGetSymbolAddress) with that device current; make it before any stream
 * capture.  No call allocates or frees memory.  All calls on a device share
 * the array: calls that may overlap on the GPU race on it, so serialise them.
 * The array keeps the last call's contents.  Its first KCA_WORKSPACE_HEADER
 * bytes (the device status word and the merge counters described above) must
 * be zero when a call starts, so each call that passes validation first
 * clears them with cudaMemsetAsync on `stream` (a memset, no allocation).
 * The device status of a call (a bounded wait that ran out) is therefore
 * readable only until the next call: pass the address that
 * attn_decode_static_scratch returns to attn_device_status after the call.
 * The address is looked up again when the device's context was created anew
 * (after cudaDeviceReset, say).
 */
#define KCA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
int attn_decode_static(const void *q, int32_t q_dtype,
                       const void *k_cache, const void *v_cache, int32_t kv_dtype,
                       int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                       int32_t batch, const int64_t *ctx_len, int32_t window,
                       float scale, float *out, void *stream);

/*
 * attn_decode_static_scratch -- the device address and size of the array
 * attn_decode_static works in, on the current device (looked up as that call
 * does; allocates nothing).  Its first bytes are a workspace header, so
 * attn_device_status(*device_ptr, stream, &detail) reads and clears the
 * status of the last attn_decode_static call on the device.  Writing the
 * array while a call runs races with it.  The paper has no counterpart to
 * this call either.  Returns KCA_OK, KCA_ERR_NULL or KCA_ERR_CUDA.
 */
int attn_decode_static_scratch(void **device_ptr, size_t *bytes);

/*
 * attn_append_kv -- the step before the attention calls: writes n_rows new
 * K/V rows into the cache, K rotated by rotary position embedding with
 * host-generated cos/sin rows (Passage: Karume v0.8.0 release notes,
 * "Features", conversation-window item: the host generates the cos/sin rows
 * per chunk),
 * V converted only.  Rotate-half pairing of dim i with dim i + 128:
 *   k'[i]       = k[i] cos[i] - k[i+128] sin[i]
 *   k'[i + 128] = k[i+128] cos[i+128] + k[i] sin[i+128]        (i < 128)
 * each product and sum rounded to f32 (no fused multiply-add), then to the
 * cache type with round-to-nearest-even: the bytes written depend on the
 * inputs only.
 *   k_new/v_new  [n_rows][256] in_dtype, device, 16-byte aligned
 *   rope_cos/rope_sin  [n_rows][256] f32, device, 16-byte aligned; both NULL
 *                = no rotation (one NULL alone is KCA_ERR_NULL)
 *   k_cache/v_cache  [cache_rows][256] kv_dtype, device (a batched cache is
 *                addressed by absolute row b * capacity + position)
 *   dst_rows_dev DEVICE int64 [n_rows] destination rows, 8-byte aligned, or
 *                NULL: rows dst_row0 .. dst_row0 + n_rows - 1 (checked on the
 *                host against cache_rows)
 *   workspace    optional status word (a workspace, or NULL): a device
 *                destination outside 0..cache_rows-1 is skipped and recorded
 *                there (error bit 3 = value 4, detail (11 << 24) | row)
 * Rows must not share a destination.  Returns KCA_OK or a KCA_ERR_* before
 * launching anything.
 */
int attn_append_kv(const void *k_new, const void *v_new, int32_t in_dtype, int32_t n_rows,
                   const float *rope_cos, const float *rope_sin,
                   void *k_cache, void *v_cache, int32_t kv_dtype, int64_t cache_rows,
                   const int64_t *dst_rows_dev, int64_t dst_row0, void *workspace, void *stream);

/*
 * attn_decode_partial / attn_merge_partials -- decode with the context split
 * into shards (one per GPU, say): each shard yields the partial-softmax state
 * of every (sequence, head) over the keys it holds, and the states of all
 * shards merge into the output by the log-sum-exp identity.  Passage: the
 * decode of Karume v0.12.0 release notes, "Performance", items 2-3 (the same
 * softmax-weighted sum of V, reduced in a different order), restricted to a
 * key range; the pages have no multi-device form.
 *
 * attn_decode_partial: the cache holds, for each sequence b, the rows of
 * positions [key_begin, key_begin + capacity) at rows b * capacity +
 * (position - key_begin).  The query of sequence b sits at ctx_len[b] - 1 as
 * in attn_decode (ctx_len[b] in 0..KCA_MAX_POSITION, and may lie past the
 * shard); it sees the keys of its causal / window range that the shard
 * holds, possibly none.  Output: the partial record `part`, f32, device,
 * 16-byte aligned, KCA_PARTIAL_FLOATS(batch) floats:
 *   part[(b * 8 + h) * 2 + 0]  m: reference score (the largest scaled score
 *                              q.k*scale of the range, or up to 8 ln 2 below it)
 *   part[(b * 8 + h) * 2 + 1]  l = sum_j exp(s_j - m)
 *   part[batch * 16 + (b * 8 + h) * 256 + d]  acc = sum_j exp(s_j - m) v_j[d]
 * An empty range gives (m, l, acc) = (-inf, 0, 0).  A NaN score makes m NaN.
 * Everything else (q, dtypes, window, scale, workspace >=
 * attn_decode_partial_workspace_bytes, errors) is as in attn_decode.
 *
 * attn_merge_partials: n_parts records (part p at parts + p * part_stride
 * floats, part_stride >= KCA_PARTIAL_FLOATS(batch) and a multiple of 4;
 * device, 16-byte aligned) -> out [batch][8][256] f32 with
 *   M = max_p m_p,  out = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p,
 * combined in part order (the same bits on every call); a row whose parts
 * are all empty is exactly 0, as in attn_decode.  The merge of the shards'
 * records equals attn_decode over the whole context up to rounding.
 */
#define KCA_PARTIAL_FLOATS(batch) ((size_t)(batch) * 8u * 258u)
int attn_decode_partial(const void *q, int32_t q_dtype,
                        const void *k_cache, const void *v_cache, int32_t kv_dtype,
                        int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int64_t capacity,
                        int32_t batch, const int64_t *ctx_len, int64_t key_begin, int32_t window,
                        float scale, float *part, void *workspace, size_t workspace_bytes,
                        void *stream);
int attn_merge_partials(int32_t n_parts, int32_t batch, const float *parts, int64_t part_stride,
                        float *out, void *stream);

/*
 * Quantised-dot attention: K stored as int8 codes with one scale per row,
 * the query quantised the same way per head inside the kernel, the QK dot
 * product taken exactly on the codes, softmax and the V sum in f32.
 * Passage: Karume v0.8.0 release notes, "Fixes": the attention dot product on
 * packed int8 pairs (dp4a, behind a device canary that falls back to the
 * emulation or fails loudly), and the activation-quantisation item (per-token
 * scale amax * f32(1/127)).
 *
 * Quantisation of a row x of 256 values: sx = amax(|x|) * f32(1/127) (NaN when
 * x holds a NaN); code = clamp(round_half_even(x / sx), -127, 127), the
 * quotient in f32, when sx is finite and > 0, else 0.  Scores:
 *   s_j = scale * sq_h * sk_j * sum_t q8_h[t] k8_j[t]
 * (the integer sum exact), then the softmax and V sum of attn_decode.
 *
 * attn_quantize_k: k [n_rows][256] k_dtype (device, 16-byte aligned) ->
 *   k8 [n_rows][KCA_I8_ROW_BYTES] packed rows (device, 16-byte aligned): the
 *   256 codes, sx as f32 at byte 256, 12 zero bytes.  Writes a batched cache
 *   row by row (row b * capacity + p of sequence b at position p).
 * attn_decode_q8: attn_decode with a packed int8 K cache k8_cache
 *   [batch][capacity][KCA_I8_ROW_BYTES] and v_cache [batch][capacity][256] of
 *   v_dtype (F32, F16 or BF16); q of any dtype, out f32; the workspace
 *   (attn_decode_q8_workspace_bytes), errors and semantics of attn_decode.
 *   16-bit V runs the tensor-core decode kernel with the QK product on int8
 *   MMAs (the plan of attn_decode for that V dtype); f32 V (or the CUDA-core
 *   kernel pinned by attn_force_path) runs the CUDA-core kernel with dp4a.
 *   The first call on a device runs the canary below (a synchronising
 *   launch): make it, or call attn_dot_canary, before any stream capture.
 * attn_dot_canary: runs, once per device, the dp4a instruction, its
 *   emulation and the int8 MMA on known answers; *variant receives the mask
 *   of the sane ones (1 dp4a, 2 its emulation, 4 int8 MMA).  The decode
 *   takes the int8 MMA only when it is sane (else the CUDA-core kernel), and
 *   the emulation where dp4a is not; with neither dp4a nor its emulation
 *   sane the call returns KCA_ERR_DEVICE and attn_decode_q8 refuses to run.
 *   Synchronises `stream` on its first call per device.
 */
int attn_quantize_k(const void *k, int32_t k_dtype, int64_t n_rows, void *k8, void *stream);
int attn_decode_q8(const void *q, int32_t q_dtype, const void *k8_cache, const void *v_cache,
                   int32_t v_dtype, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                   int64_t capacity, int32_t batch, const int64_t *ctx_len, int32_t window,
                   float scale, float *out, void *workspace, size_t workspace_bytes, void *stream);
size_t attn_decode_q8_workspace_bytes(int32_t batch, const int64_t *ctx_len, int32_t window);
int attn_dot_canary(void *stream, int32_t *variant);

/* Workspace bytes the calls above need on the current device (0 on a bad
 * argument).  Always >= KCA_WORKSPACE_HEADER.  The size depends on the
 * device (its SM count sets the split plan), so it is asked of the device the
 * call will run on rather than guessed.  Passage: Karume v0.8.0 release
 * notes, "Breaking Changes", estimateSessionMemory item (the estimator needs
 * the device's binding limit and refuses to guess without it) and "Features",
 * conversation-window item (what a window costs is reported before it is
 * allocated). */
size_t attn_prefill_workspace_bytes(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start,
                                    int32_t chunk_rows, int32_t window);
size_t attn_decode_workspace_bytes(int32_t batch, const int64_t *ctx_len, int32_t window);
size_t attn_prefill_batch_workspace_bytes(int32_t batch, int32_t rows, const int64_t *ctx_len,
                                          int32_t window);
size_t attn_decode_partial_workspace_bytes(int32_t batch, const int64_t *ctx_len, int64_t key_begin,
                                           int64_t capacity, int32_t window);

/* Zero the workspace header (cudaMemsetAsync on `stream`).  Passage: as for
 * the workspace queries above (Karume v0.8.0 release notes, "Breaking
 * Changes", estimateSessionMemory item). */
int attn_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Reads and clears the workspace status word (synchronises `stream`).
 * Passage: Karume v0.8.0 release notes, "Breaking Changes", BatchScope.finish()
 * item (a failure is reported to the caller instead of a dispatch going
 * silently missing).
 * Error bits: 1 = a bounded wait ran out (detail: (site << 24) | block),
 * 2 = a device context length was out of range (detail: (10 << 24) | sequence),
 * 4 = an append destination was out of range (detail: (11 << 24) | row).
 * Returns KCA_OK when no kernel recorded an error since the last read,
 * KCA_ERR_DEVICE when one did (*detail, if not NULL, receives the record),
 * or KCA_ERR_CUDA when the copy itself failed.
 */
int attn_device_status(void *workspace, void *stream, uint32_t *detail);

/*
 * Integer plans -- the work items a call with the same arguments runs -- for
 * bit-exact tests.  Passage: Karume v0.12.0 release notes, "Docs", ADR 0067
 * plan-size geometry table (which kernel serves the QK / PV stages of 1,
 * 2-15 and >= 16 rows), and "Performance", item 3 (kernels chosen by plan
 * size).  Each work item is 4 int64: (unit, key_begin, key_end, slot):
 *   prefill, tensor-core path: unit = 16-row tile index, [key_begin, key_end)
 *     the absolute key positions the item covers (128-key tiles clipped to the
 *     call's visible union), slot = partial slot or -1 when the tile is not
 *     split;
 *   rows path (decode, and prefill of short or mixed-dtype chunks): one item
 *     per split, unit = query row (prefill) or sequence (decode),
 *     [key_begin, key_end) within J(pos).  With an f32 cache (or the
 *     CUDA-core kernel pinned by attn_force_path) this is the CUDA-core
 *     kernel's plan for num_sms SMs, host only, and slot = the split's partial
 *     slot or -1 when the unit has one split.  With a 16-bit cache it is the
 *     tensor-core kernel's plan, whose splits run as clusters of 2, 4 or 8
 *     CTAs (or of one CTA when every unit has one split) that fit the
 *     clusters resident at once: for a device of num_sms SMs that holds
 *     cluster_capacity[0], [1], [2] clusters of 2, 4, 8 CTAs (host only), or
 *     with cluster_capacity NULL for the CURRENT DEVICE (num_sms is then not
 *     used; KCA_ERR_CUDA without a device).  For each size the split length
 *     is the smallest multiple of 64 keys whose clusters fit the capacity
 *     (one split per unit when none does), and the size with the lowest
 *     estimated time wins: the key stream takes the longer of all K/V bytes
 *     at 6.5 TB/s and waves x split_len x 1 KiB at 50 GB/s per SM; a unit of
 *     several clusters adds 1.5 us + 0.6 us x (1 + (8 / size) x
 *     ceil(clusters / 32)); ties go to the larger size.
 *     slot = the partial that the split's cluster writes (sequence *
 *     clusters-per-sequence + split / cluster size), or -1 when the unit is
 *     one cluster and merges in shared memory.  *cluster, if not NULL,
 *     receives the cluster size (1 on the CUDA-core kernel).
 *   multi-row units (short chunks on 16-bit caches, see DTYPES): one item
 *     per split of a unit of consecutive rows (4, or 8 when the chunk has
 *     more than 4 rows), unit = the unit's index, [key_begin, key_end)
 *     within the union of its rows' visible keys, slot = the split's index,
 *     or -1 when the unit has one split; the plan of the rows kernels for
 *     num_sms SMs (host only).
 * *path receives 0 for the rows path, 1 for the tensor-core path, 2 for
 * multi-row units; it is set once the arguments are valid, before any
 * device query, so it also answers a call that then fails for want of a
 * device.
 * Returns KCA_OK, or KCA_ERR_RANGE when more than max_items items exist
 * (*n_items still receives the count) or a capacity is negative.
 */
int attn_prefill_plan(int32_t q_dtype, int32_t kv_dtype, int64_t chunk_start,
                      int32_t chunk_rows, int32_t window, int32_t num_sms,
                      const int32_t *cluster_capacity, int64_t *items, int32_t max_items,
                      int32_t *n_items, int32_t *path);
int attn_decode_plan(int32_t batch, const int64_t *ctx_len, int32_t window, int32_t kv_dtype,
                     int32_t num_sms, const int32_t *cluster_capacity, int64_t *items,
                     int32_t max_items, int32_t *n_items, int32_t *cluster);

/*
 * attn_decode_cluster_capacity -- the resident-cluster capacity that the
 * plans above use on the CURRENT DEVICE: capacity[0], [1], [2] receive how
 * many clusters of 2, 4, 8 CTAs of the tensor-core rows kernel fit on it at
 * once (cudaOccupancyMaxActiveClusters, measured once per device).  With
 * these and the device's SM count, attn_decode_plan computes on the host the
 * plan a call on the device runs.  Returns KCA_OK, KCA_ERR_NULL, or
 * KCA_ERR_CUDA without a device.  Passage: as for the plans (Karume v0.12.0
 * release notes, "Docs", ADR 0067 plan-size geometry table).
 */
int attn_decode_cluster_capacity(int32_t *capacity);

/*
 * attn_force_path -- pins the kernel family that later calls take,
 * process-wide, so that two paths can be compared on the same inputs (tests,
 * diagnosis).  op 0 (prefill): path 0 = the rows path, 1 = the tensor-core
 * path where eligible (q and cache both F16 or both BF16), 2 = multi-row
 * units where eligible (16-bit cache, 2-15 rows).  op 1 (the rows
 * path: decode, and prefill chunks on the rows path): path 0 = the CUDA-core
 * kernel, 1 = the tensor-core (mma.sync) kernel where eligible (16-bit
 * cache).  op 2 (attn_prefill_batch with 2 or more rows per sequence on a
 * 16-bit cache, multi-row units): path 0 = the mma.sync kernel, 1 = the
 * tcgen05 kernel (the automatic choice).  path -1 restores the automatic
 * choice described under DTYPES.
 * Plans, workspace queries and calls all follow the pinned choice, so pin
 * before sizing a workspace.  Returns KCA_OK or KCA_ERR_RANGE.
 * Passage: Karume v0.12.0 release notes, "Performance", items 2-3 (the
 * stateAttentionReduce seat, one knob that switches the QK and PV stages
 * between the "sequential" and "parallel" kernels).
 */
int attn_force_path(int32_t op, int32_t path);

/* Static description of a status code.  Passage: Karume v0.8.0 release
 * notes, "Breaking Changes", numeric-contracts item (a violated contract is
 * rejected with an error at the call). */
const char *attn_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* KCA_H */
