// api.cu -- the C ABI of libhq.so (declared in include/hq.h): host-side
// argument checks, workspace carving and kernel dispatch.  Nothing here
// allocates, frees or synchronizes (except hq_read_device_status, a debug
// helper that says so).
#include <math.h>

#include "hq_internal.cuh"

using namespace hq;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The probe keeps the probe rows of a KV head in shared memory (the method
// probes with the 64 most recent queries).
constexpr int kMaxProbeRows = 64;

bool supported_G(int Hq, int Hkv) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return G == 1 || G == 2 || G == 4 || G == 8;
}

float resolve_scale(float s, int D) { return s == 0.0f ? 1.0f / sqrtf((float)D) : s; }

// Shapes and formats the prefill attention takes: the tcgen05 kernel is
// written for head_dim 128 and a CTA serves two query heads of one KV head.
bool prefill_shape_ok(int D, int Hq, int Hkv, int low_fmt) {
  return D == 128 && supported_G(Hq, Hkv) && (Hq / Hkv) % 2 == 0 &&
         (low_fmt == HQ_KV_INT || low_fmt == HQ_KV_FP8);
}

hq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA; }

uint32_t *status_word(void *ws) { return ws ? reinterpret_cast<uint32_t *>(ws) : nullptr; }

bool lo_cap_ok(const hq_kv_cache &c) { return c.lo_cap == 0 || c.lo_cap >= c.n_lo; }

// HQ_KV_FP8 is an 8-bit format; any other fmt value is not supported.
bool fmt_ok(const hq_kv_cache &c) {
  return c.fmt == HQ_KV_INT || (c.fmt == HQ_KV_FP8 && c.bits == 8);
}

}  // namespace

namespace hq {
// Host checks of a decode call without the workspace (used by the scratch-free
// entry point; no launch happens on failure).
hq_status check_decode_args(const void *q, const hq_kv_cache *cache, int B, int Hq, int Hkv,
                            int D, const float *out) {
  if (!q || !cache || !out) return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || cache->n_lo < 0 || cache->n_hi < 0 ||
      cache->n_lo + cache->n_hi <= 0 || !lo_cap_ok(*cache))
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || !supported_G(Hq, Hkv) || (cache->bits != 4 && cache->bits != 8) ||
      cache->group != 32 || !fmt_ok(*cache))
    return HQ_ERR_UNSUPPORTED;
  if ((cache->n_lo > 0 && (!cache->k_codes || !cache->v_codes || !cache->k_sz || !cache->v_sz)) ||
      (cache->n_hi > 0 && (!cache->k_hi || !cache->v_hi)))
    return HQ_ERR_INVALID_ARG;
  const void *ptrs[] = {q, cache->k_codes, cache->v_codes, cache->k_sz, cache->v_sz,
                        cache->k_hi, cache->v_hi, out};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return HQ_ERR_INVALID_ARG;
  return HQ_OK;
}
float resolve_softmax_scale(float s, int D) { return resolve_scale(s, D); }
}  // namespace hq

extern "C" {

const char *hq_status_string(int status) {
  switch (status) {
    case HQ_OK: return "HQ_OK";
    case HQ_ERR_INVALID_ARG: return "HQ_ERR_INVALID_ARG";
    case HQ_ERR_UNSUPPORTED: return "HQ_ERR_UNSUPPORTED";
    case HQ_ERR_WORKSPACE: return "HQ_ERR_WORKSPACE";
    case HQ_ERR_CUDA: return "HQ_ERR_CUDA";
    case HQ_ERR_TIMEOUT: return "HQ_ERR_TIMEOUT";
    case HQ_ERR_DEVICE_CHECK: return "HQ_ERR_DEVICE_CHECK";
    case HQ_ERR_SCRATCH_LIMIT: return "HQ_ERR_SCRATCH_LIMIT";
    default: return "HQ_ERR_UNKNOWN";
  }
}

int hq_version(void) { return 100; }

hq_status hq_read_device_status(const void *ws, int clear, uint32_t *status_out, void *stream) {
  if (!ws || !status_out) return HQ_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess) return HQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HQ_ERR_CUDA;
  if (clear && cudaMemsetAsync(const_cast<void *>(ws), 0, sizeof v, s) != cudaSuccess) return HQ_ERR_CUDA;
  *status_out = v;
  return HQ_OK;
}

size_t hq_probe_workspace_size(int B, int Hq, int Hkv, int P, int L, int D) {
  if (B <= 0 || !supported_G(Hq, Hkv) || P <= 0 || P > kMaxProbeRows || L <= 0 || (D != 64 && D != 128))
    return 0;
  return probe_ws_bytes(B, Hq, Hkv, P, L, D);
}

hq_status hq_probe_vertical(const void *q_probe, int64_t q_head_stride, const void *k, int B,
                            int Hq, int Hkv, int P, int L, int D, int window, int k_vert,
                            float softmax_scale, int32_t *idx_out, float *score_out, void *ws,
                            size_t ws_bytes, void *stream) {
  if (!q_probe || !k || !idx_out) return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || P <= 0 || P > L || window < 0 ||
      k_vert < 0 || k_vert > L - window || q_head_stride < (int64_t)P * D)
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || !supported_G(Hq, Hkv) || P > kMaxProbeRows) return HQ_ERR_UNSUPPORTED;
  if (!aligned16(q_probe) || !aligned16(k) || (q_head_stride * 2) % 16) return HQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < probe_ws_bytes(B, Hq, Hkv, P, L, D)) return HQ_ERR_WORKSPACE;
  return cuda_status(launch_probe((const __nv_bfloat16 *)q_probe, q_head_stride,
                                  (const __nv_bfloat16 *)k, B, Hq, Hkv, P, L, D, window, k_vert,
                                  resolve_scale(softmax_scale, D), idx_out, score_out,
                                  (uint8_t *)ws, (cudaStream_t)stream));
}

static bool shard_args_ok(const void *q_probe, int64_t q_head_stride, const void *k, int B, int Hq,
                          int Hkv, int P, int Ls, int D, int key_off, int L) {
  return q_probe && k && B > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && P > 0 && P <= L &&
         Ls > 0 && key_off >= 0 && (int64_t)key_off + Ls <= L && q_head_stride >= (int64_t)P * D;
}

size_t hq_probe_shard_workspace_size(int B, int Hq, int Hkv, int P, int Ls, int D, int k_vert) {
  if (B <= 0 || !supported_G(Hq, Hkv) || P <= 0 || P > kMaxProbeRows || Ls <= 0 || k_vert < 0 ||
      (D != 64 && D != 128))
    return 0;
  return probe_shard_ws_bytes(B, Hq, Hkv, P, Ls, D, k_vert);
}

hq_status hq_probe_shard_stats(const void *q_probe, int64_t q_head_stride, const void *k_shard,
                               int B, int Hq, int Hkv, int P, int Ls, int D, int key_off, int L,
                               float softmax_scale, float *stats_out, void *ws, size_t ws_bytes,
                               void *stream) {
  if (!stats_out || !shard_args_ok(q_probe, q_head_stride, k_shard, B, Hq, Hkv, P, Ls, D, key_off, L))
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || !supported_G(Hq, Hkv) || P > kMaxProbeRows) return HQ_ERR_UNSUPPORTED;
  if (!aligned16(q_probe) || !aligned16(k_shard) || !aligned16(stats_out) || (q_head_stride * 2) % 16)
    return HQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < probe_shard_ws_bytes(B, Hq, Hkv, P, Ls, D, 0)) return HQ_ERR_WORKSPACE;
  return cuda_status(launch_probe_shard_stats(
      (const __nv_bfloat16 *)q_probe, q_head_stride, (const __nv_bfloat16 *)k_shard, B, Hq, Hkv, P,
      Ls, D, key_off, L, resolve_scale(softmax_scale, D), reinterpret_cast<float2 *>(stats_out),
      (uint8_t *)ws, (cudaStream_t)stream));
}

hq_status hq_probe_merge_stats(const float *parts, int R, int nrows, float *stats_out,
                               void *stream) {
  if (!parts || !stats_out || R <= 0 || nrows <= 0) return HQ_ERR_INVALID_ARG;
  if (!aligned16(parts) || !aligned16(stats_out)) return HQ_ERR_INVALID_ARG;
  return cuda_status(launch_probe_merge_stats(reinterpret_cast<const float2 *>(parts), R, nrows,
                                              reinterpret_cast<float2 *>(stats_out),
                                              (cudaStream_t)stream));
}

hq_status hq_probe_shard_topk(const void *q_probe, int64_t q_head_stride, const void *k_shard,
                              int B, int Hq, int Hkv, int P, int Ls, int D, int key_off, int L,
                              int window, int k_vert, float softmax_scale, const float *stats,
                              int32_t *cand_idx, float *cand_score, void *ws, size_t ws_bytes,
                              void *stream) {
  if (!shard_args_ok(q_probe, q_head_stride, k_shard, B, Hq, Hkv, P, Ls, D, key_off, L) || !stats ||
      window < 0 || k_vert < 0 || k_vert > L - window || (k_vert > 0 && (!cand_idx || !cand_score)))
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || !supported_G(Hq, Hkv) || P > kMaxProbeRows) return HQ_ERR_UNSUPPORTED;
  if (!aligned16(q_probe) || !aligned16(k_shard) || !aligned16(stats) || (q_head_stride * 2) % 16)
    return HQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < probe_shard_ws_bytes(B, Hq, Hkv, P, Ls, D, k_vert)) return HQ_ERR_WORKSPACE;
  return cuda_status(launch_probe_shard_topk(
      (const __nv_bfloat16 *)q_probe, q_head_stride, (const __nv_bfloat16 *)k_shard, B, Hq, Hkv, P,
      Ls, D, key_off, L, window, k_vert, resolve_scale(softmax_scale, D),
      reinterpret_cast<const float2 *>(stats), cand_idx, cand_score, (uint8_t *)ws,
      (cudaStream_t)stream));
}

size_t hq_probe_merge_workspace_size(int B, int Hkv, int L, int window) {
  if (B <= 0 || Hkv <= 0 || L <= 0 || window < 0) return 0;
  return probe_merge_ws_bytes(B, Hkv, L, window);
}

hq_status hq_probe_merge_topk(const int32_t *cand_idx, const float *cand_score, int R, int B,
                              int Hkv, int L, int window, int k_vert, int32_t *idx_out, void *ws,
                              size_t ws_bytes, void *stream) {
  if (R <= 0 || B <= 0 || Hkv <= 0 || L <= 0 || window < 0 || k_vert < 0 || k_vert > L - window)
    return HQ_ERR_INVALID_ARG;
  if (k_vert == 0) return HQ_OK;
  if (!cand_idx || !cand_score || !idx_out) return HQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < probe_merge_ws_bytes(B, Hkv, L, window)) return HQ_ERR_WORKSPACE;
  return cuda_status(launch_probe_merge_topk(cand_idx, cand_score, R, B, Hkv, L, window, k_vert,
                                             idx_out, (uint8_t *)ws, status_word(ws),
                                             (cudaStream_t)stream));
}

hq_status hq_pack_kv_part(const void *k, const void *v, const int32_t *idx, int B, int Hkv, int L,
                          int D, int window, int k_vert, int bits, int group, int lo0, int hi0,
                          const hq_kv_cache *out, void *ws, size_t ws_bytes, void *stream) {
  if (!k || !v || !out || (k_vert > 0 && !idx)) return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || L <= 0 || window < 0 || k_vert < 0 || k_vert > L - window)
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || (bits != 4 && bits != 8) || group != 32) return HQ_ERR_UNSUPPORTED;
  if (out->bits == bits && !fmt_ok(*out)) return HQ_ERR_UNSUPPORTED;
  const int n_lo = L - window - k_vert, n_hi = k_vert + window;
  if (lo0 < 0 || hi0 < 0 || out->n_lo < 0 || out->n_hi < 0 || lo0 + out->n_lo > n_lo ||
      hi0 + out->n_hi > n_hi || out->bits != bits || out->group != group || !lo_cap_ok(*out))
    return HQ_ERR_INVALID_ARG;
  if ((out->n_lo > 0 && (!out->k_codes || !out->v_codes || !out->k_sz || !out->v_sz)) ||
      (out->n_hi > 0 && (!out->k_hi || !out->v_hi)))
    return HQ_ERR_INVALID_ARG;
  const void *ptrs[] = {k, v, out->k_codes, out->v_codes, out->k_sz, out->v_sz, out->k_hi, out->v_hi};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return HQ_ERR_INVALID_ARG;
  if (ws && ws_bytes < kWsHeader) return HQ_ERR_WORKSPACE;
  if (out->n_lo + out->n_hi == 0) return HQ_OK;            // an empty part: nothing to write
  return cuda_status(launch_pack((const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, idx, B, Hkv,
                                 L, D, window, k_vert, bits, *out, status_word(ws),
                                 (cudaStream_t)stream, lo0, hi0));
}

hq_status hq_pack_kv(const void *k, const void *v, const int32_t *idx, int B, int Hkv, int L,
                     int D, int window, int k_vert, int bits, int group, const hq_kv_cache *out,
                     void *ws, size_t ws_bytes, void *stream) {
  if (out && L - window - k_vert >= 0 &&
      (out->n_lo != L - window - k_vert || out->n_hi != k_vert + window))
    return HQ_ERR_INVALID_ARG;
  return hq_pack_kv_part(k, v, idx, B, Hkv, L, D, window, k_vert, bits, group, 0, 0, out, ws,
                         ws_bytes, stream);
}

hq_status hq_kv_append_part(const void *k_new, const void *v_new, int B, int Hkv, int D, int L,
                            int window, int k_vert, int lo0, int hi0, const hq_kv_cache *cache,
                            void *stream) {
  if (!k_new || !v_new || !cache) return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || window < 0 || k_vert < 0 || L < window + k_vert) return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || (cache->bits != 4 && cache->bits != 8) || cache->group != 32 ||
      !fmt_ok(*cache))
    return HQ_ERR_UNSUPPORTED;
  // the part must end where the cache ends: the last low rows and the window
  if (lo0 < 0 || hi0 < 0 || hi0 > k_vert || cache->n_lo < 0 ||
      lo0 + cache->n_lo != L - window - k_vert || cache->n_hi != k_vert + window - hi0 ||
      lo_rows(*cache) <= cache->n_lo)
    return HQ_ERR_INVALID_ARG;
  if (!cache->k_codes || !cache->v_codes || !cache->k_sz || !cache->v_sz ||
      (window > 0 && (!cache->k_hi || !cache->v_hi)))
    return HQ_ERR_INVALID_ARG;
  const void *ptrs[] = {k_new, v_new, cache->k_codes, cache->v_codes, cache->k_sz, cache->v_sz,
                        cache->k_hi, cache->v_hi};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return HQ_ERR_INVALID_ARG;
  return cuda_status(launch_kv_append((const __nv_bfloat16 *)k_new, (const __nv_bfloat16 *)v_new,
                                      B, Hkv, D, L, window, k_vert - hi0, *cache,
                                      (cudaStream_t)stream));
}

hq_status hq_kv_append(const void *k_new, const void *v_new, int B, int Hkv, int D, int L,
                       int window, int k_vert, const hq_kv_cache *cache, void *stream) {
  return hq_kv_append_part(k_new, v_new, B, Hkv, D, L, window, k_vert, 0, 0, cache, stream);
}

hq_status hq_decode_merge(const float *part_out, const float *part_lse, int R, int B, int Hq,
                          int D, float *out, float *lse_out, void *stream) {
  if (!part_out || !part_lse || !out) return HQ_ERR_INVALID_ARG;
  if (R <= 0 || B <= 0 || Hq <= 0) return HQ_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return HQ_ERR_UNSUPPORTED;
  const void *ptrs[] = {part_out, out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return HQ_ERR_INVALID_ARG;
  return cuda_status(launch_decode_merge(part_out, part_lse, R, B, Hq, D, out, lse_out,
                                         (cudaStream_t)stream));
}

size_t hq_decode_workspace_size(int B, int Hq, int Hkv, int D, int n_lo, int n_hi, int bits) {
  if (B <= 0 || !supported_G(Hq, Hkv) || (D != 64 && D != 128) || n_lo < 0 || n_hi < 0 ||
      n_lo + n_hi <= 0 || (bits != 4 && bits != 8))
    return 0;
  return decode_ws_bytes(B, Hq, Hkv, D, n_lo, n_hi, bits);
}

hq_status hq_decode_attn(const void *q, const hq_kv_cache *cache, int B, int Hq, int Hkv, int D,
                         float softmax_scale, float *out, float *lse_out, void *ws,
                         size_t ws_bytes, void *stream) {
  if (!q || !cache || !out) return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || cache->n_lo < 0 || cache->n_hi < 0 ||
      cache->n_lo + cache->n_hi <= 0 || !lo_cap_ok(*cache))
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || !supported_G(Hq, Hkv) || (cache->bits != 4 && cache->bits != 8) ||
      cache->group != 32 || !fmt_ok(*cache))
    return HQ_ERR_UNSUPPORTED;
  if ((cache->n_lo > 0 && (!cache->k_codes || !cache->v_codes || !cache->k_sz || !cache->v_sz)) ||
      (cache->n_hi > 0 && (!cache->k_hi || !cache->v_hi)))
    return HQ_ERR_INVALID_ARG;
  const void *ptrs[] = {q, cache->k_codes, cache->v_codes, cache->k_sz, cache->v_sz,
                        cache->k_hi, cache->v_hi, out};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return HQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < decode_ws_bytes(B, Hq, Hkv, D, cache->n_lo, cache->n_hi, cache->bits))
    return HQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return HQ_ERR_INVALID_ARG;
  return cuda_status(launch_decode((const __nv_bfloat16 *)q, *cache, B, Hq, Hkv, D,
                                   resolve_scale(softmax_scale, D), out, lse_out, (uint8_t *)ws,
                                   status_word(ws), (cudaStream_t)stream));
}

hq_status hq_prefill_quant_ex(const void *q, const void *k, const int32_t *idx, int B, int Hq,
                              int Hkv, int N, int D, int k_vert, int low_fmt, int8_t *qi8,
                              float *sq, int8_t *ki8, float *sk, void *stream) {
  if (!q || !k || !qi8 || !sq || (k_vert < N && (!ki8 || !sk)) || (k_vert > 0 && !idx))
    return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || k_vert < 0 || k_vert > N)
    return HQ_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || !supported_G(Hq, Hkv) ||
      (low_fmt != HQ_KV_INT && low_fmt != HQ_KV_FP8))
    return HQ_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, qi8, ki8};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return HQ_ERR_INVALID_ARG;
  return cuda_status(launch_prefill_quant((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, idx,
                                          B, Hq, Hkv, N, D, k_vert, low_fmt, qi8, sq, ki8, sk,
                                          (cudaStream_t)stream));
}

hq_status hq_prefill_quant(const void *q, const void *k, const int32_t *idx, int B, int Hq,
                           int Hkv, int N, int D, int k_vert, int8_t *qi8, float *sq,
                           int8_t *ki8, float *sk, void *stream) {
  return hq_prefill_quant_ex(q, k, idx, B, Hq, Hkv, N, D, k_vert, HQ_KV_INT, qi8, sq, ki8, sk,
                             stream);
}

hq_status hq_prefill_supported(int D, int Hq, int Hkv, int low_fmt) {
  if (!prefill_shape_ok(D, Hq, Hkv, low_fmt)) return HQ_ERR_UNSUPPORTED;
  return prefill_tc_supported(D, Hq, Hkv) ? HQ_OK : HQ_ERR_UNSUPPORTED;
}

size_t hq_prefill_workspace_size(int B, int Hq, int Hkv, int N, int D, int k_vert) {
  if (B <= 0 || !supported_G(Hq, Hkv) || N <= 0 || (D != 64 && D != 128) || k_vert < 0) return 0;
  return prefill_ws_bytes(B, Hq, Hkv, N, D, k_vert);
}

hq_status hq_prefill_attn_ex(const void *q, const void *k, const void *v, const int32_t *idx,
                             int B, int Hq, int Hkv, int N, int D, int window, int k_vert,
                             float softmax_scale, int low_fmt, float *out, void *ws,
                             size_t ws_bytes, void *stream) {
  if (!q || !k || !v || !out || (k_vert > 0 && !idx)) return HQ_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || window < 0 || k_vert < 0 ||
      k_vert > N - (window < N ? window : N))
    return HQ_ERR_INVALID_ARG;
  if (!prefill_shape_ok(D, Hq, Hkv, low_fmt)) return HQ_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, v, out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return HQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < prefill_ws_bytes(B, Hq, Hkv, N, D, k_vert)) return HQ_ERR_WORKSPACE;
  // the compiled tensor-core kernel must be usable on this device (register
  // count, shared memory): otherwise nothing is launched
  if (!prefill_tc_supported(D, Hq, Hkv)) return HQ_ERR_UNSUPPORTED;
  return cuda_status(launch_prefill((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                    (const __nv_bfloat16 *)v, idx, B, Hq, Hkv, N, D, window,
                                    k_vert, resolve_scale(softmax_scale, D), low_fmt, out,
                                    (uint8_t *)ws, status_word(ws), (cudaStream_t)stream));
}

hq_status hq_prefill_attn(const void *q, const void *k, const void *v, const int32_t *idx, int B,
                          int Hq, int Hkv, int N, int D, int window, int k_vert,
                          float softmax_scale, float *out, void *ws, size_t ws_bytes,
                          void *stream) {
  return hq_prefill_attn_ex(q, k, v, idx, B, Hq, Hkv, N, D, window, k_vert, softmax_scale,
                            HQ_KV_INT, out, ws, ws_bytes, stream);
}

}  // extern "C"
