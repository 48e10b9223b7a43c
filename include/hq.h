/*
 * hq.h -- C ABI of libhq.so: HyQuant hybrid-precision attention on NVIDIA
 * B200 (sm_100a).
 *
 * Method (web pages on HyQuant):
 *   - "HyQuant: Hybrid-Precision Quantization for LLM Attention" (wiki
 *     summary), TL;DR: a small set of vertical-line key columns, found by a
 *     cheap pattern probe, plus a local sliding window stay in high precision;
 *     every other key/value position is quantized to low bit.  In prefill this
 *     is a hybrid-precision attention operator; in decode a hybrid KV cache
 *     whose dequantization is fused into attention.
 *   - "How HyQuant uses hybrid-precision attention to cut decode compute"
 *     (blog), "Why preserve selected positions?": top 5% of key positions plus
 *     a 128-token window; "What the authors tested": Key-4bit / Value-4bit.
 *   - ACL Anthology page, HyQuant abstract: the prefill operator and the
 *     decode KV-cache compression with fused dequantization.
 *
 * Conventions for every call
 *   Layout: row-major, head-major [B, H, T, D], contiguous over D.  bf16 is
 *     IEEE bfloat16, f16 IEEE binary16, both passed as `const void *`.
 *     Query head h reads KV head h / (Hq / Hkv).
 *   Memory: every pointer is a DEVICE pointer owned by the caller, except the
 *     hq_kv_cache struct itself (host memory, read during the call).  The
 *     library never allocates or frees memory, never synchronizes the stream
 *     and keeps no state between calls.  `stream` is a cudaStream_t (NULL is
 *     the legacy default stream); all work is stream-ordered.
 *   Workspace: calls that need scratch take (ws, ws_bytes).  Size it with the
 *     matching hq_*_workspace_size query, allocate it on the device
 *     (16-byte aligned, as cudaMalloc returns it), zero it ONCE before its
 *     first use (cudaMemset), and keep using it; the library leaves it in a
 *     reusable state (the decode's tile counters return to zero at the end
 *     of every call).  After a call
 *     that reported HQ_DEV_TIMEOUT, zero it again.  The first 16 bytes hold a
 *     device status word (see hq_read_device_status).  Calls that share one
 *     workspace must not run concurrently.
 *   Errors: arguments are checked on the host before any launch; a failed
 *     check returns an error and launches nothing.  HQ_ERR_CUDA reports a
 *     launch error (cudaGetLastError).  Checks made on the device (index
 *     lists out of order or out of range; waits that ran out) never trap:
 *     they skip the offending access and set a bit in the device status word.
 *   Supported shapes: D in {64, 128}; Hq % Hkv == 0 with Hq / Hkv in
 *     {1, 2, 4, 8}; KV bits in {4, 8}; quantization group 32; the prefill
 *     attention D = 128 with Hq / Hkv in {2, 4, 8} (hq_prefill_supported).
 *     Others return HQ_ERR_UNSUPPORTED.  There is no CPU path and each
 *     operation has exactly one kernel per shape.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HQ_OK = 0,
    HQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent dims */
    HQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (D, G, bits, group) */
    HQ_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    HQ_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
    HQ_ERR_TIMEOUT = 5,       /* a bounded device wait ran out (status word) */
    HQ_ERR_DEVICE_CHECK = 6,  /* a device-side argument check failed (status word) */
    HQ_ERR_SCRATCH_LIMIT = 7  /* the problem needs more scratch than a fixed-size buffer holds */
} hq_status;

/* Low-bit code formats of a hybrid KV cache (hq_kv_cache.fmt). */
#define HQ_KV_INT 0   /* asymmetric integer codes, 4 or 8 bits: x^ = s * c + z */
#define HQ_KV_FP8 1   /* FP8 E4M3 codes, 8 bits, symmetric: x^ = s * e4m3(c), z stored as 0 */

/* Device status word bits (hq_read_device_status). */
#define HQ_DEV_BAD_INDEX 0x1u   /* an index list was unsorted, repeated or out of range */
#define HQ_DEV_TIMEOUT 0x2u     /* a bounded inter-CTA wait gave up */

/* Human-readable name of a status code (static storage). */
const char *hq_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int hq_version(void);

/*
 * Hybrid KV cache (decode).  Plain struct of caller-owned device buffers.
 * With L cached tokens, window W and k vertical columns per (b, kv head):
 *   n_lo = L - W - k low-bit rows, n_hi = k + W bf16 rows.
 *   k_codes, v_codes : u8  [B, Hkv, C, D * bits / 8], C = the low-row
 *                      capacity (lo_cap, or n_lo when lo_cap is 0); rows
 *                      0..n_lo-1 of each (b, kv head) are in use.  4-bit codes
 *                      are packed two per byte, even channel in the low nibble.
 *   k_sz, v_sz       : f16 [B, Hkv, C, D / group, 2], (scale, zero) of each
 *                      group; dequantized value = scale * code + zero.
 *   k_hi, v_hi       : bf16 [B, Hkv, n_hi, D]; rows 0..k-1 are the vertical
 *                      columns in ascending position order, rows k..k+W-1 the
 *                      window as a ring keyed by position: window position p
 *                      (L-W <= p < L) sits in row k + p mod W.
 *   lo_pos           : i32 [B, Hkv, C] position of each low row (ascending),
 *                      or NULL when not wanted.
 *   lo_cap           : low rows allocated per (b, kv head); 0 means n_lo.
 *                      Spare rows let hq_kv_append grow the low segment in
 *                      place during decode.  Rows n_lo..C-1 are never read.
 *   fmt              : HQ_KV_INT (0) or HQ_KV_FP8 (1, with bits == 8).  The
 *                      FP8 format answers the wiki summary's "Gaps" remark
 *                      that Blackwell offers FP8 as a third precision point;
 *                      the recipe is the library's reading: per token and
 *                      group, s = fp16(amax / 448) (amax = largest |x|, the
 *                      quotient rounded once), c = E4M3 of x / s rounded to
 *                      nearest even and saturated to +-448, z = 0.
 * All pointers must be 16-byte aligned.  The low rows are stored in ascending
 * position order, with no copy of the vertical rows: attention does not depend
 * on key order, and storing a vertical row only once is what gives the
 * pages' "+15% over strict 4-bit at 5% retention" ("Memory and runtime costs").
 */
typedef struct {
    void *k_codes;
    void *v_codes;
    void *k_sz;
    void *v_sz;
    void *k_hi;
    void *v_hi;
    int32_t *lo_pos;
    int n_lo;
    int n_hi;
    int bits;
    int group;
    int lo_cap;
    int fmt;
} hq_kv_cache;

/*
 * Copy the device status word out of a workspace (synchronizes `stream`).
 * *status_out receives the OR of the HQ_DEV_* bits raised since the word was
 * last cleared; `clear` != 0 resets it to zero afterwards.
 */
hq_status hq_read_device_status(const void *ws, int clear, uint32_t *status_out, void *stream);

/* ------------------------------------------------------------------------ */
/* Vertical-line probe (wiki summary, TL;DR: "vertical-line-aware pattern    */
/* probe"; blog, "Why preserve selected positions?": top 5% + window).       */
/* ------------------------------------------------------------------------ */
/*
 * For every (b, kv head), score[j] = sum over the G query heads of the group
 * and the P probe rows of the causal softmax weight of key j; probe row p sits
 * at position L - P + p and sees keys 0 .. L - P + p.  The k_vert columns of
 * [0, L - window) with the largest score are written to idx_out in ascending
 * order; equal scores go to the lower index.
 *   q_probe   : bf16, row p of head h of batch b at
 *               q_probe + (b * Hq + h) * q_head_stride + p * D  (elements);
 *               q_head_stride >= P * D lets the caller pass the last P rows
 *               of a [B, Hq, N, D] prefill Q without a copy (stride N * D).
 *   k         : bf16 [B, Hkv, L, D].
 *   idx_out   : i32 [B, Hkv, k_vert], ascending.
 *   score_out : f32 [B, Hkv, L] or NULL (the column sums; keys never seen 0).
 *   softmax_scale: 0 selects 1 / sqrt(D).
 * Requires 1 <= P <= L, 0 <= window, 0 <= k_vert <= L - window; P <= 64
 * (the method probes with the 64 most recent queries; larger P returns
 * HQ_ERR_UNSUPPORTED).
 */
size_t hq_probe_workspace_size(int B, int Hq, int Hkv, int P, int L, int D);
hq_status hq_probe_vertical(const void *q_probe, int64_t q_head_stride, const void *k, int B,
                            int Hq, int Hkv, int P, int L, int D, int window, int k_vert,
                            float softmax_scale, int32_t *idx_out, float *score_out, void *ws,
                            size_t ws_bytes, void *stream);

/*
 * The same probe with the context's keys split among ranks (a context too
 * long for one GPU): rank r holds keys [key_off, key_off + Ls) of the L-key
 * context, every rank holds the P probe queries (context positions L - P + p).
 * The probe's two passes need every probe row's softmax max and sum over the
 * whole context, and the top-k over all candidate columns; so the exchange is
 * two small gathers (the caller's: e.g. torch.distributed.all_gather):
 *   1. hq_probe_shard_stats on every rank -> (max, Z) per probe row for its keys;
 *      gather the R results, hq_probe_merge_stats -> (max, 1/Z) of the context;
 *   2. hq_probe_shard_topk on every rank -> its best k_vert candidate columns
 *      (context positions, scores); gather, hq_probe_merge_topk -> the context's
 *      k_vert columns, ascending, ties to the lower position, as
 *      hq_probe_vertical would pick them (candidate scores differ from the
 *      single-GPU probe's only by the order of the row-sum merge).
 * Layouts: q_probe, softmax_scale and q_head_stride as for hq_probe_vertical;
 * k_shard bf16 [B, Hkv, Ls, D]; stats f32 pairs [B*Hkv, (Hq/Hkv)*P, 2] in the
 * log2 domain (row max of s*scale*log2(e), then Z = sum of 2^(x - max), or
 * 1/Z after the merge); a row that sees none of a rank's keys gets
 * (-FLT_MAX, 0).  cand_idx i32 / cand_score f32 [B*Hkv, k_vert]: a rank with
 * fewer than k_vert candidates (keys before L - window) pads with -1 / -FLT_MAX.
 * Merge inputs are the R ranks' arrays stacked on a leading axis.
 * Requires 1 <= P <= min(L, 64), 0 <= key_off, key_off + Ls <= L, Ls >= 1,
 * 0 <= k_vert <= L - window.  Errors as for hq_probe_vertical; a candidate
 * position outside [0, L - window) sets HQ_DEV_BAD_INDEX in the merge's status
 * word and is ignored.
 */
size_t hq_probe_shard_workspace_size(int B, int Hq, int Hkv, int P, int Ls, int D, int k_vert);
hq_status hq_probe_shard_stats(const void *q_probe, int64_t q_head_stride, const void *k_shard,
                               int B, int Hq, int Hkv, int P, int Ls, int D, int key_off, int L,
                               float softmax_scale, float *stats_out, void *ws, size_t ws_bytes,
                               void *stream);
hq_status hq_probe_merge_stats(const float *parts, int R, int nrows, float *stats_out,
                               void *stream);
hq_status hq_probe_shard_topk(const void *q_probe, int64_t q_head_stride, const void *k_shard,
                              int B, int Hq, int Hkv, int P, int Ls, int D, int key_off, int L,
                              int window, int k_vert, float softmax_scale, const float *stats,
                              int32_t *cand_idx, float *cand_score, void *ws, size_t ws_bytes,
                              void *stream);
size_t hq_probe_merge_workspace_size(int B, int Hkv, int L, int window);
hq_status hq_probe_merge_topk(const int32_t *cand_idx, const float *cand_score, int R, int B,
                              int Hkv, int L, int window, int k_vert, int32_t *idx_out, void *ws,
                              size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* KV pack: build the hybrid cache (wiki summary, TL;DR: quantize the rest   */
/* hard, no smoothing; blog, "What the authors tested": Key-4bit/Value-4bit). */
/* ------------------------------------------------------------------------ */
/*
 * Splits [0, L) of every (b, kv head) into the window [L - window, L), the
 * vertical columns idx (ascending, distinct, in [0, L - window)) and the low
 * rows (everything else), and writes `out` as described at hq_kv_cache.
 * Quantizer (out->fmt == HQ_KV_INT), per token and group of `group`
 * channels, `bits`-bit asymmetric:
 *   s = f16_rne((max - min) / (2^bits - 1)),  z = f16_rne(min),
 *   code = clamp(rne((x - z) / s), 0, 2^bits - 1), all 0 when s == 0;
 * with out->fmt == HQ_KV_FP8 (bits 8) the FP8 recipe at hq_kv_cache.  Every
 * intermediate is taken in IEEE double so that each rounding decision is
 * exact and reproducible.  out->n_lo / n_hi / bits / group must equal
 * L - window - k_vert, k_vert + window, bits and group.  An idx list that is
 * unsorted, repeated or out of range sets HQ_DEV_BAD_INDEX in the status word
 * of `ws` (if given) and leaves the affected rows unwritten.
 *   k, v: bf16 [B, Hkv, L, D].  ws may be NULL (no status reporting).
 */
hq_status hq_pack_kv(const void *k, const void *v, const int32_t *idx, int B, int Hkv, int L,
                     int D, int window, int k_vert, int bits, int group, const hq_kv_cache *out,
                     void *ws, size_t ws_bytes, void *stream);

/*
 * One part of the hybrid cache, for a context split across GPUs: the rows
 * [lo0, lo0 + out->n_lo) of the low segment and [hi0, hi0 + out->n_hi) of the
 * bf16 segment of the cache hq_pack_kv would build from the same arguments,
 * written to `out` (row lo0 of the cache becomes row 0 of the part, and so
 * on), bit-identical to those rows of the whole cache.  A rank that decodes
 * only its part (hq_decode_attn with lse_out, then hq_decode_merge over the
 * ranks) holds only these rows: attention does not depend on the order of
 * the cached rows (wiki summary, "Key results": one softmax over all cached
 * positions).  Equal shares of both segments give every rank the same bytes
 * to read.  k and v are the whole context's [B, Hkv, L, D] (the rows of a
 * part come from positions spread over the context); idx is the whole list.
 * Requires 0 <= lo0, lo0 + out->n_lo <= L - window - k_vert, 0 <= hi0,
 * hi0 + out->n_hi <= k_vert + window; an empty part (both counts 0) is a
 * no-op.  Other arguments, layouts and errors as for hq_pack_kv.
 */
hq_status hq_pack_kv_part(const void *k, const void *v, const int32_t *idx, int B, int Hkv, int L,
                          int D, int window, int k_vert, int bits, int group, int lo0, int hi0,
                          const hq_kv_cache *out, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* Decode attention with fused dequantization (wiki summary, "Key results":  */
/* KV dequantization fused with attention in the decode kernel; abstract).   */
/* ------------------------------------------------------------------------ */
/*
 * out[b, h, :] = softmax_j(q[b, h] . key_j * scale) . value_j over all
 * n_lo + n_hi cached rows of KV head h / G, the low rows dequantized in
 * registers (scale * code + zero) and never written back.  Split-KV over the
 * cache with one combine; no mask (the cache includes the current token).
 *   q       : bf16 [B, Hq, D].
 *   out     : f32 [B, Hq, D].
 *   lse_out : f32 [B, Hq] natural-log sum of exp of the scaled logits, or NULL.
 */
size_t hq_decode_workspace_size(int B, int Hq, int Hkv, int D, int n_lo, int n_hi, int bits);
hq_status hq_decode_attn(const void *q, const hq_kv_cache *cache, int B, int Hq, int Hkv, int D,
                         float softmax_scale, float *out, float *lse_out, void *ws,
                         size_t ws_bytes, void *stream);

/*
 * Merge of decode results computed over disjoint parts of one cache's rows,
 * for a context split across GPUs (each rank decodes its part with lse_out,
 * the parts are gathered, one rank or all merge).  Attention does not depend
 * on the order of the cached rows (wiki summary, "Key results": one softmax
 * over all cached positions), so with m = max_r lse_r and w_r = exp(lse_r - m)
 *   out = sum_r w_r part_out[r] / sum_r w_r,   lse_out = m + log(sum_r w_r)
 * is the decode over the union of the parts.  A part with lse = -inf has
 * weight 0; if every part has, out is 0 and lse_out -inf.
 *   part_out : f32 [R, B, Hq, D];  part_lse : f32 [R, B, Hq] (natural log).
 *   out      : f32 [B, Hq, D];     lse_out  : f32 [B, Hq] or NULL.
 * part_out and out must be 16-byte aligned; D in {64, 128}.
 */
hq_status hq_decode_merge(const float *part_out, const float *part_lse, int R, int B, int Hq,
                          int D, float *out, float *lse_out, void *stream);

/*
 * hq_decode_attn without a caller-supplied workspace, for callers that cannot
 * allocate device memory at call time: code running under someone else's
 * stream capture (where a cudaMalloc would break the capture), serving runtimes
 * whose device memory is fixed at start-up, and hosts that forbid allocation
 * after initialization.  It computes exactly what hq_decode_attn computes
 * (same kernels, same results); the pages have no counterpart of this call.
 * Its scratch is one file-scope device array of HQ_STATIC_SCRATCH_BYTES that
 * every GPU loading the library holds until the process exits.
 *   - The first call on a device looks up that array's device address (with
 *     that device current) and caches it with the current CUDA context; make
 *     that first call before any stream capture begins.  After a device reset
 *     (cudaDeviceReset) the next call sees a new context and looks the
 *     address up again, so it too must come before any capture.
 *   - Every call shares the one array and leaves its contents behind; each call
 *     first clears (cudaMemsetAsync on `stream`) the part that must start at
 *     zero.  Calls whose work overlaps on the GPU (different streams, or graph
 *     replays that run concurrently) race on the array: serialize them.
 *   - Problems whose scratch would exceed HQ_STATIC_SCRATCH_BYTES (see
 *     hq_decode_workspace_size) return HQ_ERR_SCRATCH_LIMIT and launch nothing.
 *   - No cudaMalloc / cudaFree or allocating library routine is called.
 */
#define HQ_STATIC_SCRATCH_BYTES (16u << 20)
hq_status hq_decode_attn_static(const void *q, const hq_kv_cache *cache, int B, int Hq, int Hkv,
                                int D, float softmax_scale, float *out, float *lse_out,
                                void *stream);

/*
 * The device status word of the fixed scratch array (its first 4 bytes), the
 * counterpart of hq_read_device_status for hq_decode_attn_static: the OR of
 * the HQ_DEV_* bits raised by the last hq_decode_attn_static call on the
 * current device (HQ_DEV_TIMEOUT when a bounded wait ran out and the output
 * is incomplete).  Each hq_decode_attn_static call clears the word before it
 * launches, so read it after the call whose result you check and before the
 * next one.  Synchronizes `stream`; `clear` != 0 resets the word afterwards.
 * Allocates nothing.
 */
hq_status hq_read_static_status(int clear, uint32_t *status_out, void *stream);

/* ------------------------------------------------------------------------ */
/* Decode cache maintenance (wiki summary, TL;DR: in decode the same rule    */
/* is a KV cache compression policy; blog, "What hybrid-precision attention  */
/* changes": the decode cache is mostly low-bit, selected positions high).   */
/* ------------------------------------------------------------------------ */
/*
 * Append token L (the newly decoded position; the cache holds positions
 * 0..L-1) to every (b, kv head) of the cache, before the decode attention of
 * that token.  The pages do not spell the step out; the library's reading:
 * the vertical set chosen at prefill stays fixed, and the window stays the W
 * most recent positions.  So position L - W leaves the window: its bf16 rows
 * (window row k_vert + L mod W) are quantized exactly as hq_pack_kv
 * quantizes a low row and written as low row n_lo with lo_pos = L - W; then
 * token L's bf16 K/V take that window row.  With window == 0 token L itself
 * becomes low row n_lo (lo_pos = L).  A cache packed from L tokens and given
 * tokens L..L+t-1 this way is bit-identical to the cache packed from L + t
 * tokens with the same vertical set.
 *   k_new, v_new : bf16 [B, Hkv, D], token L's key and value.
 *   cache        : must satisfy n_lo == L - window - k_vert, n_hi == k_vert +
 *                  window and n_lo < lo_cap (room for one more low row).
 *                  The struct is only read: after the call the caller sets
 *                  cache->n_lo to n_lo + 1.
 * One launch, no workspace, no device-side checks (everything is checked on
 * the host).  Stream-ordered: a decode attention issued after it on the same
 * stream sees the new token.
 */
hq_status hq_kv_append(const void *k_new, const void *v_new, int B, int Hkv, int D, int L,
                       int window, int k_vert, const hq_kv_cache *cache, void *stream);

/*
 * hq_kv_append on the part of a context-split cache that ends where the whole
 * cache ends (see hq_pack_kv_part): it holds low rows [lo0, L - window -
 * k_vert) and bf16 rows [hi0, k_vert + window) with hi0 <= k_vert, i.e. the
 * last low rows and the whole window.  The appended low row is row lo0 +
 * cache->n_lo of the whole cache, the window ring row k_vert + L mod window
 * is row k_vert - hi0 + L mod window of the part; the result is
 * bit-identical to those rows of hq_kv_append on the whole cache.  The other
 * ranks' parts do not change.  Requires cache->n_lo == L - window - k_vert -
 * lo0, cache->n_hi == k_vert + window - hi0 and a spare low row; otherwise as
 * hq_kv_append (which is this call with lo0 = hi0 = 0).
 */
hq_status hq_kv_append_part(const void *k_new, const void *v_new, int B, int Hkv, int D, int L,
                            int window, int k_vert, int lo0, int hi0, const hq_kv_cache *cache,
                            void *stream);

/* ------------------------------------------------------------------------ */
/* Hybrid-precision prefill (abstract: Prefill stage keeps vertical-line     */
/* tokens and a local window in full precision, quantizes the rest).         */
/* ------------------------------------------------------------------------ */
/*
 * Pre-pass: symmetric INT8 codes for Q, one scale per (b, head, row), and for
 * the remaining keys -- those that are not vertical columns (idx), taken in
 * position order -- one scale per (b, kv head, block of 64 consecutive
 * remaining keys).  Vertical-column keys are never quantized.
 *   s = fl32(amax / 127) (1 when amax == 0),  code = clamp(rne(fl32(x / s)), -127, 127).
 *   q: bf16 [B, Hq, N, D] -> qi8 i8 [B, Hq, N, D], sq f32 [B, Hq, N]
 *   k: bf16 [B, Hkv, N, D], idx i32 [B, Hkv, k_vert] (ascending) ->
 *      ki8 i8 [B, Hkv, N - k_vert, D], sk f32 [B, Hkv, ceil((N - k_vert) / 64)]
 */
hq_status hq_prefill_quant(const void *q, const void *k, const int32_t *idx, int B, int Hq,
                           int Hkv, int N, int D, int k_vert, int8_t *qi8, float *sq,
                           int8_t *ki8, float *sk, void *stream);
/*
 * The same with a choice of low-part format: HQ_KV_INT (the INT8 codes
 * above) or HQ_KV_FP8, the FP8 third precision point the wiki summary's
 * "Gaps" names for Blackwell, taken at the same granularity (library
 * reading): s = fl32(amax / 448) (1 if amax = 0), code = E4M3 of fl32(x / s)
 * rounded to nearest even and saturated to +-448; the code bits go to the
 * same int8 arrays.
 */
hq_status hq_prefill_quant_ex(const void *q, const void *k, const int32_t *idx, int B, int Hq,
                              int Hkv, int N, int D, int k_vert, int low_fmt, int8_t *qi8,
                              float *sq, int8_t *ki8, float *sk, void *stream);

/*
 * Causal attention in which, for query i, key j <= i is "high" when it is in
 * the window (j > i - window) or is a vertical column of idx, else "low".
 * High logits are bf16 q . k (fp32 accumulate); low logits are the exact INT8
 * dot product of the pre-pass codes times sq[i] and the scale of the key's
 * block of remaining keys; one online softmax covers both; P . V uses fp16 P
 * and V with fp32 accumulation.
 *   q: bf16 [B, Hq, N, D];  k, v: bf16 [B, Hkv, N, D];
 *   idx: i32 [B, Hkv, k_vert] ascending (from hq_probe_vertical);
 *   out: f32 [B, Hq, N, D].  The workspace holds the pre-pass output.
 */
size_t hq_prefill_workspace_size(int B, int Hq, int Hkv, int N, int D, int k_vert);
/*
 * The prefill attention runs on one kernel, written for the 5th-generation
 * tensor cores: head_dim 128 and an even number of query heads per KV head
 * (a CTA serves two query heads that share their key and value tiles).
 * Other shapes (D = 64, Hq == Hkv) return HQ_ERR_UNSUPPORTED from
 * hq_prefill_attn / hq_prefill_attn_ex, and so does a device on which the
 * compiled kernel cannot run as built; nothing is launched then.  This query
 * answers HQ_OK exactly when a prefill call of that shape and low-part format
 * (HQ_KV_INT or HQ_KV_FP8) will run that kernel on the current device.  (The
 * pre-pass hq_prefill_quant / _ex also takes D = 64 and any G.)
 */
hq_status hq_prefill_supported(int D, int Hq, int Hkv, int low_fmt);
hq_status hq_prefill_attn(const void *q, const void *k, const void *v, const int32_t *idx, int B,
                          int Hq, int Hkv, int N, int D, int window, int k_vert,
                          float softmax_scale, float *out, void *ws, size_t ws_bytes,
                          void *stream);
/*
 * The same with a choice of low-part format (HQ_KV_INT: the INT8 low part
 * above; HQ_KV_FP8: the E4M3 codes of hq_prefill_quant_ex, whose low logit is
 * the fp32-accumulated dot product of the E4M3 values times sq[i] and the
 * key block's scale).
 */
hq_status hq_prefill_attn_ex(const void *q, const void *k, const void *v, const int32_t *idx,
                             int B, int Hq, int Hkv, int N, int D, int window, int k_vert,
                             float softmax_scale, int low_fmt, float *out, void *ws,
                             size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
