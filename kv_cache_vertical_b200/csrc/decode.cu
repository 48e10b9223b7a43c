// decode.cu -- split-KV decode attention over the hybrid KV cache with the
// dequantization fused in registers.
//
// Method: "HyQuant: Hybrid-Precision Quantization for LLM Attention" (wiki
// summary), TL;DR and "Key results": in decode the cache stays low-bit and KV
// dequantization is fused into the attention kernel, so dequantized values
// never go back to memory; the ACL abstract states the same for the Decode
// stage.
//
// Work split: one CTA per (split of the cached rows, b, kv head); a CTA scores
// its rows for the G query heads of the KV head, keeps an online softmax
// (running max, sum, output) per head, and writes one partial; a combine
// kernel merges the partials with the usual max-rescaled sums.  This simple
// CUDA-core version serves head_dim 64; head_dim 128 goes to the TMA +
// tensor-core kernel of decode_tma.cu.
#include <float.h>

#include <cuda_fp8.h>

#include "hq_internal.cuh"

namespace hq {
namespace {

constexpr int DWARPS = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  const __nv_bfloat16 *q;
  const uint8_t *k_codes, *v_codes;
  const __half2 *k_sz, *v_sz;
  const __nv_bfloat16 *k_hi, *v_hi;
  int Hq, Hkv, G, n_lo, n_hi, lo_cap, nsplit;
  int fp8;           // low rows hold FP8 E4M3 codes (x^ = s * e4m3(c)) instead of integers
  float scale_log2;
  float *part_o;     // [B*Hq, nsplit, D]
  float2 *part_ml;   // [B*Hq, nsplit]
};

// Channels lane*CPL .. lane*CPL+CPL-1 of one cached row, as fp32.
template <int D, int BITS>
__device__ __forceinline__ void load_row(const uint8_t *codes, const __half2 *sz,
                                         const __nv_bfloat16 *hi, int n_lo, int n_hi, int lo_cap,
                                         bool fp8, size_t bh, int t, int lane, float (&x)[D / 32]) {
  constexpr int CPL = D / 32;
  if (t < n_lo) {
    const size_t row = bh * lo_cap + t;
    const float2 s_z = __half22float2(sz[row * (D / 32) + (lane * CPL) / 32]);
    uint32_t c[CPL];
    const uint8_t *cr = codes + row * (D * BITS / 8);
    if (BITS == 4) {
      uint32_t w = CPL == 4 ? (uint32_t)reinterpret_cast<const uint16_t *>(cr)[lane] : (uint32_t)cr[lane];
#pragma unroll
      for (int i = 0; i < CPL; ++i) c[i] = (w >> (4 * i)) & 0xf;
    } else {
      uint32_t w = CPL == 4 ? reinterpret_cast<const uint32_t *>(cr)[lane]
                            : (uint32_t)reinterpret_cast<const uint16_t *>(cr)[lane];
#pragma unroll
      for (int i = 0; i < CPL; ++i) c[i] = (w >> (8 * i)) & 0xff;
    }
    if (BITS == 8 && fp8) {
#pragma unroll
      for (int i = 0; i < CPL; ++i)
        x[i] = s_z.x * __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c[i], __NV_E4M3)));
    } else {
#pragma unroll
      for (int i = 0; i < CPL; ++i) x[i] = fmaf(s_z.x, (float)c[i], s_z.y);
    }
  } else {
    const uint32_t *hr = reinterpret_cast<const uint32_t *>(hi + (bh * n_hi + (t - n_lo)) * D);
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
      const uint32_t w = hr[lane * (CPL / 2) + i];
      x[2 * i] = bf16_lo(w);
      x[2 * i + 1] = bf16_hi(w);
    }
  }
}

template <int D, int BITS, int G>
__global__ void __launch_bounds__(DWARPS * 32) decode_split(DecodeArgs a) {
  constexpr int CPL = D / 32;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.Hkv, kh = bh % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.n_lo + a.n_hi;
  const int t0 = (int)((long long)T * split / a.nsplit);
  const int t1 = (int)((long long)T * (split + 1) / a.nsplit);

  float q[G][CPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t *qr = reinterpret_cast<const uint32_t *>(a.q + ((size_t)b * a.Hq + kh * G + g) * D);
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
      const uint32_t w = qr[lane * (CPL / 2) + i];
      q[g][2 * i] = bf16_lo(w) * a.scale_log2;
      q[g][2 * i + 1] = bf16_hi(w) * a.scale_log2;
    }
  }
  float m[G], l[G], o[G][CPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -FLT_MAX;
    l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) o[g][i] = 0.f;
  }
  for (int t = t0 + warp; t < t1; t += DWARPS) {
    float kx[CPL], vx[CPL];
    load_row<D, BITS>(a.k_codes, a.k_sz, a.k_hi, a.n_lo, a.n_hi, a.lo_cap, a.fp8 != 0, (size_t)bh, t, lane, kx);
    load_row<D, BITS>(a.v_codes, a.v_sz, a.v_hi, a.n_lo, a.n_hi, a.lo_cap, a.fp8 != 0, (size_t)bh, t, lane, vx);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < CPL; ++i) s = fmaf(q[g][i], kx[i], s);
      s = warp_sum(s);
      const float mn = fmaxf(m[g], s);
      const float alpha = exp2f(m[g] - mn), p = exp2f(s - mn);
      l[g] = l[g] * alpha + p;
#pragma unroll
      for (int i = 0; i < CPL; ++i) o[g][i] = fmaf(o[g][i], alpha, p * vx[i]);
      m[g] = mn;
    }
  }
  // Merge the warps of the CTA through shared memory, then write one partial.
  __shared__ float sm_ml[DWARPS][G][2];
  __shared__ float sm_o[DWARPS][G][D];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      sm_ml[warp][g][0] = m[g];
      sm_ml[warp][g][1] = l[g];
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) sm_o[warp][g][lane * CPL + i] = o[g][i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int g = e / D, d = e % D;
    float mm = -FLT_MAX;
#pragma unroll
    for (int w = 0; w < DWARPS; ++w) mm = fmaxf(mm, sm_ml[w][g][0]);
    float ll = 0.f, oo = 0.f;
#pragma unroll
    for (int w = 0; w < DWARPS; ++w) {
      const float f = exp2f(sm_ml[w][g][0] - mm);
      ll += sm_ml[w][g][1] * f;
      oo += sm_o[w][g][d] * f;
    }
    const size_t hq = (size_t)b * a.Hq + kh * G + g;
    a.part_o[(hq * a.nsplit + split) * D + d] = oo;
    if (d == 0) a.part_ml[hq * a.nsplit + split] = make_float2(mm, ll);
  }
}

template <int D>
__global__ void decode_combine(const float *__restrict__ part_o, const float2 *__restrict__ part_ml,
                               int nsplit, float *__restrict__ out, float *__restrict__ lse) {
  const size_t hq = blockIdx.x;
  const float2 *ml = part_ml + hq * nsplit;
  float m = -FLT_MAX;
  for (int s = 0; s < nsplit; ++s) m = fmaxf(m, ml[s].x);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float l = 0.f, o = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float f = exp2f(ml[s].x - m);
      l += ml[s].y * f;
      o += part_o[(hq * nsplit + s) * D + d] * f;
    }
    out[hq * D + d] = o / l;
    if (d == 0 && lse) lse[hq] = (m + log2f(l)) / kLog2e;
  }
}

int choose_nsplit(int nbh, int T) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int ns = (4 * sms + nbh - 1) / nbh;
  const int max_by_rows = (T + 255) / 256;
  if (ns > max_by_rows) ns = max_by_rows;
  if (ns < 1) ns = 1;
  if (ns > 1024) ns = 1024;
  return ns;
}

template <int D, int BITS, int G>
cudaError_t launch_t(const DecodeArgs &a, int nbh, float *out, float *lse, cudaStream_t s) {
  dim3 grid(a.nsplit, nbh);
  decode_split<D, BITS, G><<<grid, DWARPS * 32, 0, s>>>(a);
  decode_combine<D><<<nbh * G, 128, 0, s>>>(a.part_o, a.part_ml, a.nsplit, out, lse);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_g(const DecodeArgs &a, int nbh, float *out, float *lse, cudaStream_t s) {
  switch (a.G) {
    case 1: return launch_t<D, BITS, 1>(a, nbh, out, lse, s);
    case 2: return launch_t<D, BITS, 2>(a, nbh, out, lse, s);
    case 4: return launch_t<D, BITS, 4>(a, nbh, out, lse, s);
    case 8: return launch_t<D, BITS, 8>(a, nbh, out, lse, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_ws_bytes(int B, int Hq, int Hkv, int D, int n_lo, int n_hi, int bits) {
  if (decode_tma_supported(D, bits, Hq / Hkv)) return decode_tma_ws_bytes(B, Hq, Hkv, n_lo, n_hi, bits);
  const int nbh = B * Hkv;
  const int ns = choose_nsplit(nbh, n_lo + n_hi);
  size_t off = kWsHeader;
  off = align_up(off + (size_t)B * Hq * ns * D * sizeof(float), 256);
  off = align_up(off + (size_t)B * Hq * ns * sizeof(float2), 256);
  return off;
}

size_t decode_ws_zero_bytes(int B, int Hq, int Hkv, int D, int n_lo, int n_hi, int bits) {
  if (decode_tma_supported(D, bits, Hq / Hkv)) return decode_tma_ws_zero_bytes(B, Hq, Hkv, n_lo, n_hi, bits);
  return kWsHeader;
}

cudaError_t launch_decode(const __nv_bfloat16 *q, const hq_kv_cache &c, int B, int Hq, int Hkv,
                          int D, float scale, float *out, float *lse, uint8_t *ws,
                          uint32_t *status, cudaStream_t s) {
  if (decode_tma_supported(D, c.bits, Hq / Hkv))
    return launch_decode_tma(q, c, B, Hq, Hkv, scale, out, lse, ws, status, s);
  DecodeArgs a;
  a.q = q;
  a.k_codes = (const uint8_t *)c.k_codes;
  a.v_codes = (const uint8_t *)c.v_codes;
  a.k_sz = (const __half2 *)c.k_sz;
  a.v_sz = (const __half2 *)c.v_sz;
  a.k_hi = (const __nv_bfloat16 *)c.k_hi;
  a.v_hi = (const __nv_bfloat16 *)c.v_hi;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.n_lo = c.n_lo;
  a.n_hi = c.n_hi;
  a.lo_cap = lo_rows(c);
  a.fp8 = c.fmt == HQ_KV_FP8;
  const int nbh = B * Hkv;
  a.nsplit = choose_nsplit(nbh, c.n_lo + c.n_hi);
  a.scale_log2 = scale * kLog2e;
  size_t off = kWsHeader;
  a.part_o = reinterpret_cast<float *>(ws + off);
  off = align_up(off + (size_t)B * Hq * a.nsplit * D * sizeof(float), 256);
  a.part_ml = reinterpret_cast<float2 *>(ws + off);
  if (D == 128 && c.bits == 4) return launch_g<128, 4>(a, nbh, out, lse, s);
  if (D == 128 && c.bits == 8) return launch_g<128, 8>(a, nbh, out, lse, s);
  if (D == 64 && c.bits == 4) return launch_g<64, 4>(a, nbh, out, lse, s);
  if (D == 64 && c.bits == 8) return launch_g<64, 8>(a, nbh, out, lse, s);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Merge of decode results over disjoint parts of one cache (a context split
// across ranks): with m = max_r lse_r and w_r = exp(lse_r - m),
//   out = sum_r w_r out_r / sum_r w_r,   lse = m + log(sum_r w_r),
// the exact softmax over the union of the parts' rows.  One warp per
// (b, query head); a part with lse = -inf (no rows) has weight 0.
// ---------------------------------------------------------------------------
namespace {
template <int D>
__global__ void __launch_bounds__(128)
decode_merge_kernel(const float *__restrict__ part_out, const float *__restrict__ part_lse, int R,
                    int nq, float *__restrict__ out, float *__restrict__ lse) {
  constexpr int CPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int bq = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (bq >= nq) return;
  float m = -INFINITY;
  for (int r = 0; r < R; ++r) m = fmaxf(m, __ldg(part_lse + (size_t)r * nq + bq));
  float acc[CPL] = {};
  float sum = 0.f;
  if (m > -INFINITY) {
    for (int r = 0; r < R; ++r) {
      const float w = expf(__ldg(part_lse + (size_t)r * nq + bq) - m);
      const float *o = part_out + ((size_t)r * nq + bq) * D + lane * CPL;
      sum += w;
#pragma unroll
      for (int i = 0; i < CPL; ++i) acc[i] = fmaf(w, __ldg(o + i), acc[i]);
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) out[(size_t)bq * D + lane * CPL + i] = acc[i] * inv;
  if (lse && lane == 0) lse[bq] = sum > 0.f ? m + logf(sum) : -INFINITY;
}
}  // namespace

cudaError_t launch_decode_merge(const float *part_out, const float *part_lse, int R, int B,
                                int Hq, int D, float *out, float *lse, cudaStream_t s) {
  const int nq = B * Hq;
  const int blocks = (nq + 3) / 4;
  if (D == 128)
    decode_merge_kernel<128><<<blocks, 128, 0, s>>>(part_out, part_lse, R, nq, out, lse);
  else if (D == 64)
    decode_merge_kernel<64><<<blocks, 128, 0, s>>>(part_out, part_lse, R, nq, out, lse);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace hq
