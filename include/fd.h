/*
 * fd.h -- split-KV decode attention ("Flash-Decoding") for NVIDIA B200, sm_100a.
 *
 * THE OPERATION
 * "Flash-Decoding for long-context inference" (Tri Dao, Daniel Haziza,
 * Francisco Massa, Grigory Sizov), section "Multi-head attention for
 * decoding": while decoding, the query of the one new token of each sequence
 * attends to every cached key/value of that sequence. For sequence b, query
 * head i, key/value head j = i / (Hq / Hkv) and L = seqlens[b] cached tokens:
 *
 *     z_t       = scale * sum_d q[b,i,d] * k_cache[b,j,t,d]        (t < L)
 *     lse[b,i]  = log( sum_t exp(z_t) )                            (natural log)
 *     out[b,i,:]= sum_t exp(z_t - lse[b,i]) * v_cache[b,j,t,:]
 *
 * Section "A faster attention for decoding: Flash-Decoding" reaches that
 * result by splitting the keys/values along the sequence, computing each
 * split's attention together with one log-sum-exp scalar per row and split,
 * and reducing over the splits with each one rescaled through its
 * log-sum-exp. This library does the same on one GPU:
 *   split   -- every (sequence, kv-head) row's cached tokens are laid end to
 *              end in one stream of 64-token tiles, and the stream is cut into
 *              num_splits equal runs of tiles, one per thread block. A run
 *              that holds a whole row writes out/lse directly; a run that
 *              holds part of a row writes that part's normalised output and
 *              log-sum-exp (one "segment") to the workspace.
 *   combine -- for each row cut into several segments, the LSE-weighted
 *              reduction of its segments; rows with no tokens get out = 0,
 *              lse = -inf.
 * fd_decode runs both in ONE kernel: after writing a segment, a block takes a
 * ticket on its row (an atomic counter in the workspace; nothing waits), and
 * the block that completes the row performs its reduction. A row cut into
 * more than 32 segments is reduced in two levels: its segments 8 at a time
 * (each group by the block completing it, through a counter of its own),
 * then the groups' results. fd_split and fd_combine run the two stages as
 * separate kernels (same arithmetic, same grouping, same results bit for
 * bit).
 *
 * LAYOUTS (all row-major, contiguous, device memory unless stated)
 *   q        [B, Hq, D]          bf16 bit patterns (uint16_t), 16-byte aligned
 *   k_cache  [B, Hkv, Lmax, D]   bf16, 16-byte aligned
 *   v_cache  [B, Hkv, Lmax, D]   bf16, 16-byte aligned
 *   seqlens  [B]                 int32 (device); values are clamped to [0, Lmax]
 *   out      [B, Hq, D]          fp32, 16-byte aligned
 *   lse      [B, Hq]             fp32 natural-log log-sum-exp, 4-byte aligned
 *   workspace                    fd_workspace_bytes() bytes, 16-byte aligned; must be
 *                                zero before its first use by fd_decode (fd_workspace_init);
 *                                every completed fd_decode leaves its counters at zero again
 * Supported: D in {64, 128}; 1 <= Hq/Hkv <= 16; positions t >= seqlens[b]
 * are never used (their contents, NaN included, cannot reach the output).
 *
 * OWNERSHIP AND ERRORS
 * Every pointer is owned by the caller; the library allocates nothing and
 * keeps no state between calls except, per device, a cache of the SM count,
 * an error word (see fd_device_status), a cache of the last 32 encoded TMA
 * tensor maps (keyed by address, shape and box, so reusing a buffer skips the
 * encode; a map describes memory, it owns none) and the fixed scratch buffer
 * of fd_decode_static (a file-scope device array, not an allocation). Calls are
 * asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 * and never synchronise, except fd_device_status. Every entry point returns
 * FD_OK (0) or a negative FD_ERR_* code; argument checks run before any CUDA
 * call, so a rejected call launches nothing.
 */
#ifndef FD_H_
#define FD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FD_API __attribute__((visibility("default")))
#else
#define FD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define FD_OK                 0
#define FD_ERR_NULL_POINTER  -1   /* a required pointer is NULL */
#define FD_ERR_SHAPE         -2   /* B, Hq, Hkv < 1, max_len < 0, or sizes beyond the limits below */
#define FD_ERR_GROUP         -3   /* Hq % Hkv != 0 or Hq / Hkv > 16 */
#define FD_ERR_HEAD_DIM      -4   /* D is not 64 or 128 */
#define FD_ERR_ALIGNMENT     -5   /* a pointer breaks the alignment listed above */
#define FD_ERR_WORKSPACE     -6   /* workspace NULL or smaller than fd_workspace_bytes() */
#define FD_ERR_SPLITS        -7   /* num_splits < 1 or > FD_MAX_SPLITS */
#define FD_ERR_DEVICE        -8   /* no usable CUDA device, or not compute capability 10.0 */
#define FD_ERR_LAUNCH        -9   /* a kernel launch (or tensor-map encode) failed */
#define FD_ERR_TIMEOUT      -10   /* a device-side wait gave up (reported by fd_device_status) */
#define FD_ERR_CAPACITY     -11   /* an output array passed to fd_segments is too small */
#define FD_ERR_STATIC_LIMIT -12   /* fd_decode_static: the problem needs more scratch than its fixed buffer */
#define FD_ERR_BOUNDS       -13   /* debug builds only (-DFD_DEBUG): a device-side bounds check failed; the
                                     access was skipped and the call's outputs are invalid */

#define FD_TILE_TOKENS     64     /* tokens per tile; split boundaries are multiples of this */
#define FD_MAX_SPLITS      65535
#define FD_MAX_GROUP       16
#define FD_STATIC_SCRATCH_BYTES (8u << 20)   /* fixed device scratch behind fd_decode_static */
#define FD_KV_HND           0     /* paged pool [num_pages][Hkv][page_size][D] */
#define FD_KV_NHD           1     /* paged pool [num_pages][page_size][Hkv][D] */
#define FD_KV_E4M3          1     /* 8-bit cache codes: OCP FP8 E4M3 (fd_decode_quant) */
#define FD_KV_INT8          2     /* 8-bit cache codes: int8, two's complement (fd_decode_quant) */

/* Number of splits (thread blocks of the split stage) for a problem shape,
 * sized to the current device's SM count: one block per SM while the batch
 * holds at least 4 tiles (256 tokens) per block, fewer for small problems;
 * with at most 16 tiles per SM (and at least 64 SMs) the count is also
 * capped at the SM count rounded down to a multiple of 32 (128 on B200).
 * Pure function of its arguments and the SM count (queried once per device).
 * Returns num_splits >= 1, or a negative FD_ERR_* code.
 * Reading of the page's dispatcher (the library picks Flash-Decoding or a
 * plain single-pass kernel by problem size): num_splits = 1 is the
 * unsplit case. */
FD_API int fd_plan(int B, int Hq, int Hkv, int D, int max_len);

/* fd_plan with the SM count given instead of queried; no CUDA call. */
FD_API int fd_plan_for_sms(int B, int Hq, int Hkv, int D, int max_len, int num_sms);

/* Workspace bytes that fd_decode / fd_split / fd_combine need for
 * num_splits splits: room for (num_splits + B*Hkv - 1) segments of
 * Hq/Hkv rows, each D fp32 outputs plus one fp32 log-sum-exp, one int32
 * counter per (sequence, kv-head) row and one per segment slot (for the
 * chunks of rows reduced in two levels), laid out as (each part 256-byte
 * aligned)
 *     seg_out [num_segments][Hq/Hkv][D]  fp32
 *     seg_lse [num_segments][Hq/Hkv]     fp32
 *     tickets [B*Hkv + num_segments]     int32 (fd_decode only)
 * Returns 0 when num_splits == 1 (no row is ever cut) or the arguments are
 * invalid. */
FD_API size_t fd_workspace_bytes(int B, int Hq, int Hkv, int D, int max_len, int num_splits);

/* Decode attention with num_splits = fd_plan(B, Hq, Hkv, D, max_len).
 * Writes out and lse for every (b, i). Enqueues one kernel on `stream`.
 * Calls that share a workspace must not overlap on the device. After a call
 * that failed on the device (fd_device_status != FD_OK) re-zero the
 * workspace with fd_workspace_init before using it again. */
FD_API int fd_decode(int B, int Hq, int Hkv, int D, int max_len,
              const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
              const int32_t *seqlens, float scale,
              float *out, float *lse,
              void *workspace, size_t workspace_bytes, void *stream);

/* fd_decode with an explicit num_splits in [1, FD_MAX_SPLITS]; every value
 * gives the same result up to fp32 rounding (the split identity). */
FD_API int fd_decode_splits(int B, int Hq, int Hkv, int D, int max_len,
                     const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                     const int32_t *seqlens, float scale,
                     float *out, float *lse,
                     void *workspace, size_t workspace_bytes,
                     int num_splits, void *stream);

/* Several queries per sequence (speculative decoding; the "flash decoding论文"
 * page: with multi-turn dialogue or speculative decoding several query
 * vectors are computed in parallel). q [B, q_len, Hq, D] bf16 (16-byte
 * aligned), out [B, q_len, Hq, D] fp32, lse [B, q_len, Hq] fp32; caches as
 * for fd_decode. seqlens[b] counts the cached tokens INCLUDING the q_len new
 * ones, which are the last q_len positions; query j sees the first
 * seqlens[b] - (q_len - 1 - j) tokens (causal among the new tokens; fewer
 * than one gives out = 0, lse = -inf). Requires q_len * Hq / Hkv <= 16: the
 * q_len x (Hq/Hkv) (query, head) pairs of a kv head are one small dense
 * contraction, so every K/V byte is still read once. Workspace:
 * fd_workspace_bytes(B, Hq * q_len, Hkv, D, max_len, num_splits);
 * num_splits = 0 means fd_plan(B, Hq, Hkv, D, max_len). q_len = 1 is
 * fd_decode_splits. */
FD_API int fd_decode_multi(int B, int q_len, int Hq, int Hkv, int D, int max_len,
                           const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *seqlens, float scale, float *out, float *lse,
                           void *workspace, size_t workspace_bytes, int num_splits, void *stream);

/* fd_decode_multi over an 8-bit key/value cache with one scale per kv head.
 * The "flash decoding论文" page lists INT8/INT4 quantisation among PaddleNLP's
 * inference techniques; one byte per cached element halves the bytes a
 * decode step streams. k_codes / v_codes: [B][Hkv][max_len][D] bytes, device,
 * 16-byte aligned; kv_type FD_KV_E4M3 (OCP 8-bit floating point E4M3: sign,
 * 4 exponent bits with bias 7, 3 mantissa bits, exponent field 0
 * subnormal, S.1111.111 NaN, no infinities) or FD_KV_INT8. k_scale /
 * v_scale: [Hkv] float32, device, 4-byte aligned. The cached key of token t
 * is k_scale[h] * decode(k_codes[b][h][t][:]), the value likewise with
 * v_scale, and the attention is that of fd_decode_multi over those values
 * (q [B][q_len][Hq][D] bf16, out [B][q_len][Hq][D] and lse [B][q_len][Hq]
 * fp32; q_len = 1 is single-query decode; q_len * Hq/Hkv <= 16). Codes past
 * seqlens[b] are never used, whatever they hold. The query must be finite;
 * it enters the tensor-core contraction as f16 after an exact power-of-two
 * prescale per (query, head), so only its elements smaller than 2^-25 of
 * that query head's largest are rounded. Workspace as fd_decode_multi;
 * num_splits = 0 means fd_plan(B, Hq, Hkv, D, max_len).
 * Errors: FD_ERR_SHAPE also for kv_type or q_len out of range;
 * FD_ERR_NULL_POINTER / FD_ERR_ALIGNMENT also for the scales. */
FD_API int fd_decode_quant(int B, int q_len, int Hq, int Hkv, int D, int max_len, int kv_type,
                           const uint16_t *q, const uint8_t *k_codes, const uint8_t *v_codes,
                           const float *k_scale, const float *v_scale, const int32_t *seqlens, float scale,
                           float *out, float *lse, void *workspace, size_t workspace_bytes, int num_splits,
                           void *stream);

/* The final reduction over R partial results per row computed elsewhere,
 * e.g. one per GPU when a long sequence is sharded along its tokens across
 * GPUs (context parallelism; the DISTFLASHATTN abstract on the "Related
 * papers: Glinthawk" page distributes attention over GPUs along the
 * sequence). Part r of row i is (part_out[r][i][0..D), part_lse[r][i]), the
 * normalised output and natural-log log-sum-exp of the row's attention over
 * that part's tokens, as fd_decode writes them. Writes
 *     lse[i] = log sum_r exp(part_lse[r][i]),
 *     out[i] = sum_r exp(part_lse[r][i] - lse[i]) * part_out[r][i]
 * ("Flash-Decoding for long-context inference", section "A faster attention
 * for decoding: Flash-Decoding", the final reduction), parts in increasing r
 * (deterministic). Parts with lse = -inf weigh 0; a row with no non-empty part
 * gets out = 0, lse = -inf. part_out / out: fp32, device, 16-byte aligned;
 * part_lse / lse: fp32, device, 4-byte aligned; out may not overlap the
 * parts. R >= 1, rows >= 0 (0: nothing to do, no CUDA call), D a multiple
 * of 4 in [4, 4096]. Asynchronous on `stream`. */
FD_API int fd_merge_partials(int R, int rows, int D, const float *part_out, const float *part_lse,
                             float *out, float *lse, void *stream);

/* Measurement utility, not part of the attention (the pages have no
 * counterpart): reads `bytes` of device memory at `buf` once, streaming it
 * the way the split kernel does (one block per SM, 32 KiB bulk copies into a
 * 4-stage shared-memory ring, chunks round-robin over the blocks) with no
 * compute. Timing it over a buffer larger than L2 gives the HBM read ceiling
 * the decode kernels are compared with. The first 32-bit word of every
 * 32 KiB chunk is xor-folded into the low half of *sink (device, 8-byte
 * aligned, zero on entry) so the copies cannot be elided; the high half is
 * set to 1 if a bounded wait gave up (2 s). buf 16-byte aligned, bytes a
 * multiple of 16 (0: nothing). Asynchronous on `stream`. */
FD_API int fd_read_probe(const void *buf, size_t bytes, unsigned long long *sink, void *stream);

/* fd_decode_splits over a PAGED key/value cache. The page pools
 * k_pages / v_pages hold num_pages pages of page_size tokens each, laid out
 * head-major (kv_layout = FD_KV_HND: [num_pages][Hkv][page_size][D] bf16) or
 * token-major (FD_KV_NHD: [num_pages][page_size][Hkv][D] bf16), 16-byte
 * aligned. block_table ([B][max_pages_per_seq] int32, device, 16-byte
 * aligned) gives the page that holds logical page p of sequence b: token t
 * of sequence b is slot t % page_size of page block_table[b][t / page_size].
 * Only the first ceil(seqlens[b] / page_size) entries of a row are read, so
 * the rest may hold anything; an entry outside [0, num_pages) reads as a
 * page of zeros. seqlens[b] is clamped to [0, max_pages_per_seq * page_size].
 * page_size: a power of two in [8, 4096]; max_pages_per_seq: a multiple of 4.
 * num_splits = 0 means fd_plan(B, Hq, Hkv, D, max_pages_per_seq * page_size);
 * workspace as for fd_decode with max_len = max_pages_per_seq * page_size.
 * The paged-KV layout is the one the "flash decoding论文" page lists among
 * PaddleNLP's attention optimisations ("PageAttention"). */
FD_API int fd_decode_paged(int B, int Hq, int Hkv, int D, int page_size, int num_pages, int max_pages_per_seq,
                           int kv_layout, const uint16_t *q, const uint16_t *k_pages, const uint16_t *v_pages,
                           const int32_t *block_table, const int32_t *seqlens, float scale,
                           float *out, float *lse, void *workspace, size_t workspace_bytes,
                           int num_splits, void *stream);

/* fd_decode_quant over a PAGED 8-bit cache: the page pools k_pages /
 * v_pages hold codes (one byte per element) in the layouts of
 * fd_decode_paged (kv_layout FD_KV_HND or FD_KV_NHD), found through the
 * block table as there, and each element is dequantised with its kv head's
 * scale as in fd_decode_quant (kv_type FD_KV_E4M3 or FD_KV_INT8). q_len
 * queries per sequence as in fd_decode_multi. Page and block-table rules,
 * alignment and errors: those of fd_decode_paged and fd_decode_quant;
 * workspace: fd_workspace_bytes(B, Hq * q_len, Hkv, D,
 * max_pages_per_seq * page_size, num_splits). */
FD_API int fd_decode_quant_paged(int B, int q_len, int Hq, int Hkv, int D, int page_size, int num_pages,
                                 int max_pages_per_seq, int kv_layout, int kv_type, const uint16_t *q,
                                 const uint8_t *k_pages, const uint8_t *v_pages, const float *k_scale,
                                 const float *v_scale, const int32_t *block_table, const int32_t *seqlens,
                                 float scale, float *out, float *lse, void *workspace, size_t workspace_bytes,
                                 int num_splits, void *stream);

/* Split stage alone (one kernel): for each run of tiles, writes out/lse of
 * the rows it holds whole and the segments of the rows it holds in part.
 * Rows with no tokens and rows cut into several segments are left for
 * fd_combine. Does not use the workspace counters. */
FD_API int fd_split(int B, int Hq, int Hkv, int D, int max_len,
             const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
             const int32_t *seqlens, float scale,
             float *out, float *lse,
             void *workspace, size_t workspace_bytes,
             int num_splits, void *stream);

/* Combine stage alone (one kernel): reads the segments that fd_split wrote
 * for the same (shape, seqlens, num_splits) and writes out/lse of every row
 * cut into several segments (segment order fixed, so the result is
 * deterministic), and out = 0, lse = -inf for rows with no tokens. Launched
 * as a programmatic dependent of the preceding kernel on the stream. */
FD_API int fd_combine(int B, int Hq, int Hkv, int D, int max_len,
               const int32_t *seqlens,
               float *out, float *lse,
               const void *workspace, size_t workspace_bytes,
               int num_splits, void *stream);

/* Host-side description of where the split stage cuts each row, for host
 * seqlens (HOST memory, [B]). For every segment slot s < capacity:
 * seg_row[s] = b*Hkv + j of the row it belongs to, or -1 if the slot is
 * unused; [seg_begin[s], seg_end[s]) = its token range (clipped to the
 * row's length). seg_whole[s] = 1 if the segment is its row's only one
 * (then fd_split writes out/lse directly and the slot stays unused in the
 * workspace). Returns the number of slots (num_splits + B*Hkv - 1), or
 * FD_ERR_CAPACITY if capacity is smaller, or another FD_ERR_* code. */
FD_API int fd_segments(int B, int Hkv, int max_len, const int32_t *seqlens_host, int num_splits,
                int32_t *seg_row, int32_t *seg_begin, int32_t *seg_end, int32_t *seg_whole,
                int capacity);

/* fd_decode for callers that cannot allocate device memory. The paper has
 * no counterpart to this entry point; it exists for code that is handed its
 * input and output buffers but owns no allocator -- for example a plugin
 * inside a serving engine that plans every device byte itself and forbids
 * allocation on its execution path, or a decode loop that must not call
 * cudaMalloc because cudaMalloc can synchronise the device.
 * Same inputs, outputs, layouts and result as fd_decode with the planned
 * split count; there is no workspace argument. Instead the library keeps one
 * file-scope device buffer of FD_STATIC_SCRATCH_BYTES (8 MiB), which every
 * GPU that loads the library holds until the process exits. A problem whose
 * fd_workspace_bytes() exceeds it is rejected with FD_ERR_STATIC_LIMIT
 * before anything is launched. Nothing is allocated: no cudaMalloc, no
 * cudaFree, no allocating library call.
 * The first call on each device looks up the buffer's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. If that lookup fails the call returns
 * FD_ERR_LAUNCH, nothing is remembered, and the next call tries again; the
 * address is kept once a lookup succeeds. Every call clears the buffer's per-row counters
 * (cudaMemsetAsync on `stream`) and then reuses it, so the buffer keeps the
 * last call's segments. All calls on one device share the one buffer: two
 * calls that can overlap on the GPU (different streams, no ordering between
 * them) race on it and give wrong results. */
FD_API int fd_decode_static(int B, int Hq, int Hkv, int D, int max_len,
                            const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                            const int32_t *seqlens, float scale,
                            float *out, float *lse, void *stream);

/* Zero `workspace_bytes` bytes of workspace on `stream` (cudaMemsetAsync).
 * Needed once after allocation, before the first fd_decode. */
FD_API int fd_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Waits for `stream`, then returns and clears this device's error word:
 * FD_OK, or FD_ERR_TIMEOUT if a kernel's bounded wait gave up (the kernel
 * then returned early and its outputs are invalid). FD_ERR_LAUNCH if the
 * stream itself reports an error. */
FD_API int fd_device_status(void *stream);

/* Text for an FD_* code (static storage). */
FD_API const char *fd_strerror(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
FD_API int fd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FD_H_ */
