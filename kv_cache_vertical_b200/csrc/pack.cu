// pack.cu -- build the hybrid KV cache: vertical rows and the window stay
// bf16, every other row is quantized to 4 or 8 bits per group of 32 channels.
//
// Method: "HyQuant: Hybrid-Precision Quantization for LLM Attention" (wiki
// summary), TL;DR -- the critical set stays in high precision and the rest is
// quantized hard, with no smoothing; blog "How HyQuant uses hybrid-precision
// attention to cut decode compute", "What the authors tested" -- Key-4bit /
// Value-4bit; "Memory and runtime costs" -- a vertical row is stored once, in
// 16-bit (the +15% figure), so the low segment holds only the low rows.
//
// One warp per (b, kv head, position): it classifies the position with a
// binary search in the sorted index list, then either copies the bf16 rows or
// quantizes them.  Every rounding decision of the quantizer is the one IEEE
// double arithmetic takes (an fp32 estimate settles the codes that are not
// near a tie), so the codes, scales and zeros are exactly the ones the
// library's specification defines.  HBM-bound: read 2 * D * 2 bytes per position, write
// the packed rows.
#include <limits.h>

#include "hq_internal.cuh"

namespace hq {
namespace {

constexpr int kWarps = 8;

// fp16((mx - mn) / qmax) with the quotient first rounded to IEEE double, as
// the specification states.  The fp32 quotient (mx - mn is exact in fp32 for
// bf16 inputs within 2^15 of each other; otherwise one more rounding) lies
// within 2^-22 relative of the exact one, so unless it is that close to a
// point halfway between two fp16 numbers, or below the fp16 normal range,
// rounding it to fp16 gives the same result; those few cases divide in
// double.
__device__ __forceinline__ __half scale_f16(float mx, float mn, int qmax) {
  const float q = __fdiv_rn(mx - mn, (float)qmax);
  const uint32_t low = __float_as_uint(q) & 0x1fffu;       // the 13 bits below fp16 precision
  const bool near_tie = low >= 0x1000u - 8u && low <= 0x1000u + 8u;
  if (near_tie || q < 6.103515625e-05f)                   // 2^-14
    return __double2half(((double)mx - (double)mn) / (double)qmax);
  return __float2half_rn(q);
}

// D / 32 channels per lane; a group of 32 channels spans 32 / (D/32) lanes.
template <int D, int BITS>
__device__ __forceinline__ void quant_store(const uint32_t (&w)[D / 64], uint8_t *codes_row,
                                            __half2 *sz_row, int lane) {
  constexpr int CPL = D / 32;          // channels per lane: 4 (D=128) or 2 (D=64)
  constexpr int LPG = 32 / CPL;        // lanes per group: 8 or 16
  constexpr int QMAX = (1 << BITS) - 1;
  float x[CPL];
#pragma unroll
  for (int i = 0; i < CPL / 2; ++i) {
    x[2 * i] = bf16_lo(w[i]);
    x[2 * i + 1] = bf16_hi(w[i]);
  }
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < CPL; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
#pragma unroll
  for (int o = LPG / 2; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float fmn = mn == 0.f ? 0.f : mn;  // a -0 minimum is stored as +0
  const __half hs = scale_f16(mx, mn, QMAX);
  const __half hz = __float2half_rn(fmn);   // mn is bf16: exact in fp32, one rounding
  // code = clamp(rint((x - z) / s), 0, QMAX) with the quotient in IEEE
  // double.  An fp32 estimate (error below 2^-14 for |q| < 2^9) decides every
  // code whose quotient is not within 2^-12 of a half-integer: there the
  // double quotient rounds to the same integer.  The rest take the double
  // path itself.
  const float sf = __half2float(hs), zf = __half2float(hz);
  const float rs = sf != 0.f ? __frcp_rn(sf) : 0.f;
  uint32_t c[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const float q = (x[i] - zf) * rs;
    float t = rintf(q);
    if (sf == 0.f) {
      t = 0.f;
    } else if (fabsf(q - t) > 0.5f - 1.f / 4096.f) {
      t = (float)rint(((double)x[i] - (double)zf) / (double)sf);
    }
    t = fminf(fmaxf(t, 0.f), (float)QMAX);
    c[i] = (uint32_t)t;
  }
  if (BITS == 4) {
    if (CPL == 4) {
      const uint16_t b = (uint16_t)(c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12));
      reinterpret_cast<uint16_t *>(codes_row)[lane] = b;
    } else {
      codes_row[lane] = (uint8_t)(c[0] | (c[1] << 4));
    }
  } else {
    if (CPL == 4) {
      reinterpret_cast<uint32_t *>(codes_row)[lane] = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
    } else {
      reinterpret_cast<uint16_t *>(codes_row)[lane] = (uint16_t)(c[0] | (c[1] << 8));
    }
  }
  if (lane % LPG == 0) sz_row[lane / LPG] = __halves2half2(hs, hz);
}

template <int D, int BITS>
__global__ void __launch_bounds__(kWarps * 32)
pack_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
            const int32_t *__restrict__ idx, int nbh, int L, int window, int k_vert, int lo_cap,
            uint8_t *__restrict__ k_codes, uint8_t *__restrict__ v_codes,
            __half2 *__restrict__ k_sz, __half2 *__restrict__ v_sz,
            __nv_bfloat16 *__restrict__ k_hi, __nv_bfloat16 *__restrict__ v_hi,
            int32_t *__restrict__ lo_pos, uint32_t *status) {
  constexpr int W32 = D / 64;                 // 32-bit words of bf16 per lane
  constexpr int ROWB = D * BITS / 8;          // packed bytes per low row
  constexpr int NG = D / 32;
  const int lane = threadIdx.x & 31;
  const int n_lo = L - window - k_vert, n_hi = k_vert + window;
  const long long warp0 = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * kWarps;

  // Device-side check of the index list (ascending, distinct, in range).
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < (long long)nbh * k_vert;
       t += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(t % k_vert);
    const int x = idx[t];
    if (x < 0 || x >= L - window || (r > 0 && idx[t - 1] >= x)) raise_status(status, HQ_DEV_BAD_INDEX);
  }

  // Eight consecutive positions of one pair per warp task: one binary search
  // finds the verticals before the chunk, the next (at most eight) index
  // entries say which chunk positions are vertical, and all sixteen row loads
  // are issued before any quantization.
  constexpr int PCH = 8;
  const long long ntask = (long long)nbh * ((L + PCH - 1) / PCH);
  const int cpb = (L + PCH - 1) / PCH;                // chunks per pair
  for (long long task = warp0; task < ntask; task += nwarps) {
    const int bh = (int)(task / cpb);
    const int j0 = (int)(task % cpb) * PCH;
    const int32_t *id = idx + (size_t)bh * k_vert;
    const int cnt0 = j0 > 0 ? upper_bound_i32(id, k_vert, j0 - 1) : 0;   // verticals before j0
    const int e = cnt0 + (lane & (PCH - 1));
    const int ve = (lane < PCH && e < k_vert) ? __ldg(id + e) : INT_MAX;
    const uint32_t vbit = (ve >= j0 && ve < j0 + PCH) ? 1u << (ve - j0) : 0u;
    const uint32_t vbits = __reduce_or_sync(0xffffffffu, vbit);            // vertical positions of the chunk
    uint32_t kw[PCH][W32], vw[PCH][W32];
#pragma unroll
    for (int p = 0; p < PCH; ++p) {
      const int j = j0 + p;
      const size_t src = ((size_t)bh * L + (j < L ? j : L - 1)) * D;
#pragma unroll
      for (int i = 0; i < W32; ++i) {
        kw[p][i] = __ldg(reinterpret_cast<const uint32_t *>(k + src) + lane * W32 + i);
        vw[p][i] = __ldg(reinterpret_cast<const uint32_t *>(v + src) + lane * W32 + i);
      }
    }
#pragma unroll
    for (int p = 0; p < PCH; ++p) {
      const int j = j0 + p;
      if (j >= L) break;
      const int cnt = cnt0 + __popc(vbits & ((1u << p) - 1u));            // verticals before j
      int hi_row = -1, lo_row = -1;
      if (j >= L - window) hi_row = k_vert + j % window;          // the window ring
      else if (vbits & (1u << p)) hi_row = cnt;
      else lo_row = j - cnt;
      if (hi_row >= 0) {
        if (hi_row >= n_hi) {
          if (lane == 0) raise_status(status, HQ_DEV_BAD_INDEX);
          continue;
        }
        const size_t dst = ((size_t)bh * n_hi + hi_row) * D;
#pragma unroll
        for (int i = 0; i < W32; ++i) {
          reinterpret_cast<uint32_t *>(k_hi + dst)[lane * W32 + i] = kw[p][i];
          reinterpret_cast<uint32_t *>(v_hi + dst)[lane * W32 + i] = vw[p][i];
        }
      } else {
        if (lo_row < 0 || lo_row >= n_lo) {
          if (lane == 0) raise_status(status, HQ_DEV_BAD_INDEX);
          continue;
        }
        const size_t r = (size_t)bh * lo_cap + lo_row;
        quant_store<D, BITS>(kw[p], k_codes + r * ROWB, k_sz + r * NG, lane);
        quant_store<D, BITS>(vw[p], v_codes + r * ROWB, v_sz + r * NG, lane);
        if (lo_pos && lane == 0) lo_pos[r] = j;
      }
    }
  }
}

template <int D, int BITS>
cudaError_t launch_pack_t(const __nv_bfloat16 *k, const __nv_bfloat16 *v, const int32_t *idx,
                          int nbh, int L, int window, int k_vert, const hq_kv_cache &o,
                          uint32_t *status, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long warps = (long long)nbh * ((L + 7) / 8);     // one warp task per 8 positions
  long long blocks = (warps + kWarps - 1) / kWarps;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  pack_kernel<D, BITS><<<(unsigned)blocks, kWarps * 32, 0, s>>>(
      k, v, idx, nbh, L, window, k_vert, lo_rows(o), (uint8_t *)o.k_codes, (uint8_t *)o.v_codes,
      (__half2 *)o.k_sz, (__half2 *)o.v_sz, (__nv_bfloat16 *)o.k_hi, (__nv_bfloat16 *)o.v_hi,
      o.lo_pos, status);
  return cudaGetLastError();
}

// Decode cache maintenance: one warp per (b, kv head).  The warp reads the
// window row that position L - W occupies (row k_vert + L mod W of the ring)
// and the new token's rows, quantizes the old occupant into low row n_lo with
// the pack's quantizer, then overwrites the window row with the new token.
// Each lane reads and writes only its own words of the row, so the in-place
// overwrite after the reads needs no barrier.  With no window the new token
// goes straight to the low segment.
template <int D, int BITS>
__global__ void __launch_bounds__(kWarps * 32)
kv_append_kernel(const __nv_bfloat16 *__restrict__ k_new, const __nv_bfloat16 *__restrict__ v_new,
                 int nbh, int L, int window, int k_vert, int n_lo, int lo_cap,
                 uint8_t *__restrict__ k_codes, uint8_t *__restrict__ v_codes,
                 __half2 *__restrict__ k_sz, __half2 *__restrict__ v_sz,
                 __nv_bfloat16 *__restrict__ k_hi, __nv_bfloat16 *__restrict__ v_hi,
                 int32_t *__restrict__ lo_pos) {
  constexpr int W32 = D / 64;
  constexpr int ROWB = D * BITS / 8;
  constexpr int NG = D / 32;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * kWarps + (threadIdx.x >> 5);
  pdl_wait();      // the token's K/V and the cache rows come from earlier kernels
  pdl_trigger();
  if (bh >= nbh) return;
  const uint32_t *kn = reinterpret_cast<const uint32_t *>(k_new + (size_t)bh * D) + lane * W32;
  const uint32_t *vn = reinterpret_cast<const uint32_t *>(v_new + (size_t)bh * D) + lane * W32;
  uint32_t kw[W32], vw[W32], ko[W32], vo[W32];
#pragma unroll
  for (int i = 0; i < W32; ++i) {
    kw[i] = __ldg(kn + i);
    vw[i] = __ldg(vn + i);
  }
  const size_t r = (size_t)bh * lo_cap + n_lo;
  if (window == 0) {
    quant_store<D, BITS>(kw, k_codes + r * ROWB, k_sz + r * NG, lane);
    quant_store<D, BITS>(vw, v_codes + r * ROWB, v_sz + r * NG, lane);
    if (lo_pos && lane == 0) lo_pos[r] = L;
    return;
  }
  const size_t hrow = ((size_t)bh * (k_vert + window) + k_vert + L % window) * D;
  uint32_t *kh = reinterpret_cast<uint32_t *>(k_hi + hrow) + lane * W32;
  uint32_t *vh = reinterpret_cast<uint32_t *>(v_hi + hrow) + lane * W32;
#pragma unroll
  for (int i = 0; i < W32; ++i) {
    ko[i] = kh[i];
    vo[i] = vh[i];
  }
  quant_store<D, BITS>(ko, k_codes + r * ROWB, k_sz + r * NG, lane);
  quant_store<D, BITS>(vo, v_codes + r * ROWB, v_sz + r * NG, lane);
  if (lo_pos && lane == 0) lo_pos[r] = L - window;
#pragma unroll
  for (int i = 0; i < W32; ++i) {
    kh[i] = kw[i];
    vh[i] = vw[i];
  }
}

template <int D, int BITS>
cudaError_t launch_kv_append_t(const __nv_bfloat16 *k_new, const __nv_bfloat16 *v_new, int nbh,
                               int L, int window, int k_vert, const hq_kv_cache &c,
                               cudaStream_t s) {
  const int blocks = (nbh + kWarps - 1) / kWarps;
  return pdl_launch(kv_append_kernel<D, BITS>, dim3(blocks), dim3(kWarps * 32), 0, s, k_new, v_new,
                    nbh, L, window, k_vert, c.n_lo, lo_rows(c), (uint8_t *)c.k_codes,
                    (uint8_t *)c.v_codes, (__half2 *)c.k_sz, (__half2 *)c.v_sz,
                    (__nv_bfloat16 *)c.k_hi, (__nv_bfloat16 *)c.v_hi, c.lo_pos);
}

}  // namespace

cudaError_t launch_pack(const __nv_bfloat16 *k, const __nv_bfloat16 *v, const int32_t *idx,
                        int B, int Hkv, int L, int D, int window, int k_vert, int bits,
                        const hq_kv_cache &out, uint32_t *status, cudaStream_t s) {
  const int nbh = B * Hkv;
  if (D == 128 && bits == 4) return launch_pack_t<128, 4>(k, v, idx, nbh, L, window, k_vert, out, status, s);
  if (D == 128 && bits == 8) return launch_pack_t<128, 8>(k, v, idx, nbh, L, window, k_vert, out, status, s);
  if (D == 64 && bits == 4) return launch_pack_t<64, 4>(k, v, idx, nbh, L, window, k_vert, out, status, s);
  if (D == 64 && bits == 8) return launch_pack_t<64, 8>(k, v, idx, nbh, L, window, k_vert, out, status, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_kv_append(const __nv_bfloat16 *k_new, const __nv_bfloat16 *v_new, int B,
                             int Hkv, int D, int L, int window, int k_vert,
                             const hq_kv_cache &c, cudaStream_t s) {
  const int nbh = B * Hkv;
  if (D == 128 && c.bits == 4) return launch_kv_append_t<128, 4>(k_new, v_new, nbh, L, window, k_vert, c, s);
  if (D == 128 && c.bits == 8) return launch_kv_append_t<128, 8>(k_new, v_new, nbh, L, window, k_vert, c, s);
  if (D == 64 && c.bits == 4) return launch_kv_append_t<64, 4>(k_new, v_new, nbh, L, window, k_vert, c, s);
  if (D == 64 && c.bits == 8) return launch_kv_append_t<64, 8>(k_new, v_new, nbh, L, window, k_vert, c, s);
  return cudaErrorInvalidValue;
}

}  // namespace hq
