// hq_internal.cuh -- shared declarations of the CUDA side of libhq.so.
// (Internal to the library; the public ABI is include/hq.h.)
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"

namespace hq {

// ---------------------------------------------------------------------------
// Workspace: the first 16 bytes hold the device status word (+ padding);
// call-specific scratch starts at kWsHeader.
// ---------------------------------------------------------------------------
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ void raise_status(uint32_t *status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with pdl_launch() may be
// scheduled while the kernel before it in the stream is still finishing; it
// must call pdl_wait() before it touches any memory an earlier kernel writes
// (the wait returns once that kernel has completed and its writes are
// visible; without the launch attribute it returns at once).
// pdl_trigger() lets the next such kernel be scheduled early.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

template <typename... Params, typename... Args>
cudaError_t pdl_launch(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Launchers (one per .cu file).  Arguments are already validated.
// ---------------------------------------------------------------------------
// Low rows allocated per (b, kv head) of a cache (lo_cap, 0 meaning n_lo).
inline int lo_rows(const hq_kv_cache &c) { return c.lo_cap > 0 ? c.lo_cap : c.n_lo; }

// The pack writes the rows [lo0, lo0 + out.n_lo) of the low segment and
// [hi0, hi0 + out.n_hi) of the bf16 segment (the whole cache: lo0 = hi0 = 0).
cudaError_t launch_pack(const __nv_bfloat16 *k, const __nv_bfloat16 *v, const int32_t *idx,
                        int B, int Hkv, int L, int D, int window, int k_vert, int bits,
                        const hq_kv_cache &out, uint32_t *status, cudaStream_t s, int lo0 = 0,
                        int hi0 = 0);
cudaError_t launch_kv_append(const __nv_bfloat16 *k_new, const __nv_bfloat16 *v_new, int B,
                             int Hkv, int D, int L, int window, int k_vert,
                             const hq_kv_cache &c, cudaStream_t s);

size_t probe_ws_bytes(int B, int Hq, int Hkv, int P, int L, int D);
cudaError_t launch_probe(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                         const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int L, int D,
                         int window, int k_vert, float scale, int32_t *idx_out, float *score_out,
                         uint8_t *ws, cudaStream_t s);
// context split of the probe (keys [key_off, key_off + Ls) of an L-key context)
size_t probe_shard_ws_bytes(int B, int Hq, int Hkv, int P, int Ls, int D, int k_vert);
size_t probe_merge_ws_bytes(int B, int Hkv, int L, int window);
cudaError_t launch_probe_shard_stats(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                                     const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls,
                                     int D, int key_off, int L, float scale, float2 *stats_out,
                                     uint8_t *ws, cudaStream_t s);
cudaError_t launch_probe_merge_stats(const float2 *parts, int R, int nrows, float2 *stats,
                                     cudaStream_t s);
cudaError_t launch_probe_shard_topk(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                                    const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls,
                                    int D, int key_off, int L, int window, int k_vert, float scale,
                                    const float2 *stats, int32_t *cand_idx, float *cand_score,
                                    uint8_t *ws, cudaStream_t s);
cudaError_t launch_probe_merge_topk(const int32_t *cand_idx, const float *cand_score, int R, int B,
                                    int Hkv, int L, int window, int k_vert, int32_t *idx_out,
                                    uint8_t *ws, uint32_t *status, cudaStream_t s);

// tcgen05 probe passes (probe_tc.cu) over keys [0, Ls) whose probe rows sit
// at key positions qpos0 + p; D in {64, 128}, G <= 8, P <= 64.
bool probe_tc_supported(int D, int G, int P);
int probe_tc_chunks(int nbh, int Ls);
// `pdl`: launch as a programmatic dependent of the kernel before it.
cudaError_t launch_probe_pass(bool colsum, const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                              const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls, int D,
                              int qpos0, float scale, float2 *partial, int nchunk,
                              const float2 *stats, float *score, uint32_t *status, cudaStream_t s,
                              bool pdl = false);

bool decode_tma_supported(int D, int bits, int G);
size_t decode_tma_ws_bytes(int B, int Hq, int Hkv, int n_lo, int n_hi, int bits);
cudaError_t launch_decode_tma(const __nv_bfloat16 *q, const hq_kv_cache &c, int B, int Hq,
                              int Hkv, float scale, float *out, float *lse, uint8_t *ws,
                              uint32_t *status, cudaStream_t s);
size_t decode_ws_bytes(int B, int Hq, int Hkv, int D, int n_lo, int n_hi, int bits);
// Leading bytes of the decode workspace that must be zero before a call
// (status word and the split counters).
size_t decode_ws_zero_bytes(int B, int Hq, int Hkv, int D, int n_lo, int n_hi, int bits);
size_t decode_tma_ws_zero_bytes(int B, int Hq, int Hkv, int n_lo, int n_hi, int bits);
hq_status check_decode_args(const void *q, const hq_kv_cache *cache, int B, int Hq, int Hkv,
                            int D, const float *out);
float resolve_softmax_scale(float s, int D);
cudaError_t launch_decode(const __nv_bfloat16 *q, const hq_kv_cache &c, int B, int Hq, int Hkv,
                          int D, float scale, float *out, float *lse, uint8_t *ws,
                          uint32_t *status, cudaStream_t s);
cudaError_t launch_decode_merge(const float *part_out, const float *part_lse, int R, int B,
                                int Hq, int D, float *out, float *lse, cudaStream_t s);

cudaError_t launch_prefill_quant(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                 const int32_t *idx, int B, int Hq, int Hkv, int N, int D,
                                 int k_vert, int low_fmt, int8_t *qi8, float *sq, int8_t *ki8,
                                 float *sk, cudaStream_t s);
// tcgen05 prefill (head_dim 128, an even number of query heads per KV head).
struct TcLaunch {
  const __nv_bfloat16 *q, *k;        // bf16 [B,Hq,N,D], [B,Hkv,N,D]
  const int8_t *qi8, *ki8;           // pre-pass codes (ki8 over the remaining keys)
  const float *sq, *sk;              // pre-pass scales (sk per 64 remaining keys)
  const __half *vh;                  // fp16 V in position order [B,Hkv,N,D]
  const __half *vc;                  // fp16 V of the remaining keys [B,Hkv,N-k_vert,D]
  const __nv_bfloat16 *vk;           // compact vertical K [B,Hkv,kpad,D]
  const __half *vv;                  // compact vertical V
  const int32_t *idx;
  float *out;
  uint32_t *status;
  int B, Hq, Hkv, N, window, k_vert, kpad, nblk_r;
  float scale;
  bool f8;                           // low part in FP8 E4M3 (kind::f8f6f4) instead of INT8
};
bool prefill_tc_supported(int D, int Hq, int Hkv);
cudaError_t launch_prefill_tc(const TcLaunch &p, cudaStream_t s);

size_t prefill_ws_bytes(int B, int Hq, int Hkv, int N, int D, int k_vert);
cudaError_t launch_prefill(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                           const __nv_bfloat16 *v, const int32_t *idx, int B, int Hq, int Hkv,
                           int N, int D, int window, int k_vert, float scale, int low_fmt,
                           float *out, uint8_t *ws, uint32_t *status, cudaStream_t s);

// ---------------------------------------------------------------------------
// Small device helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T>
__device__ __forceinline__ T warp_sum(T x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Index of the first element of sorted a[0..n) that is > x.
__device__ __forceinline__ int upper_bound_i32(const int32_t *a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) <= x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Number of entries of the ascending list a[0, n) below x, found by one warp
// with 32-way splits (about three rounds of loads for thousands of entries
// instead of a dozen dependent ones).  Every lane returns the result.
__device__ __forceinline__ int warp_count_below(const int32_t *__restrict__ a, int n, int x,
                                                int lane) {
  int lo = 0, hi = n;                       // the count lies in [lo, hi]
  while (hi - lo > 32) {
    const int len = hi - lo;
    const int si = lo + (int)(((long long)lane * len) >> 5);        // lane 0 samples lo
    const unsigned below = __ballot_sync(0xffffffffu, __ldg(a + si) < x);
    const int m = __popc(below);            // samples 0 .. m-1 are below x
    if (m == 0) return lo;
    const int s_last = lo + (int)(((long long)(m - 1) * len) >> 5);
    const int s_next = m < 32 ? lo + (int)(((long long)m * len) >> 5) : hi;
    lo = s_last + 1;
    hi = s_next;
  }
  const bool in = lane < hi - lo;
  const unsigned below = __ballot_sync(0xffffffffu, in && __ldg(a + lo + (in ? lane : 0)) < x);
  return lo + __popc(below);
}

// The double d rounded to fp32 toward zero, with the last bit set when that
// dropped anything (round to odd).  Rounding this to a format with far fewer
// bits (E4M3 keeps 4) gives the same result as rounding d itself.
__device__ __forceinline__ float f32_round_odd(double d) {
  const float r = __double2float_rz(d);
  return (double)r == d ? r : __uint_as_float(__float_as_uint(r) | 1u);
}

// True when an fp32 estimate q (relative error a few units of 2^-24) of a
// quotient lies so close to a point halfway between two E4M3 neighbours that
// the exact quotient might round the other way.  Normal range: the 20 bits
// below the 3-bit mantissa within 16 units of the halfway pattern; subnormal
// range (|q| < 2^-6, spacing 2^-9): the fraction of q * 2^9 within 2^-12 of 1/2.
__device__ __forceinline__ bool e4m3_near_tie(float q) {
  const float a = fabsf(q);
  if (a >= 0.015625f) {
    const uint32_t low = __float_as_uint(a) & 0xFFFFFu;
    return low >= 0x80000u - 16u && low <= 0x80000u + 16u;
  }
  const float t = a * 512.f;
  return fabsf(t - floorf(t) - 0.5f) < 1.f / 4096.f;
}

}  // namespace hq
