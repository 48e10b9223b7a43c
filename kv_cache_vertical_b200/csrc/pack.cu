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
// quantizes them.  Every rounding decision of the quantizer is taken in IEEE
// double, so the codes, scales and zeros are exactly the ones the library's
// specification defines.  HBM-bound: read 2 * D * 2 bytes per position, write
// the packed rows.
#include "hq_internal.cuh"

namespace hq {
namespace {

constexpr int kWarps = 8;

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
  double dmn = (double)mn;
  if (dmn == 0.0) dmn = 0.0;  // a -0 minimum is stored as +0
  const __half hs = __double2half(((double)mx - (double)mn) / (double)QMAX);
  const __half hz = __double2half(dmn);
  const double s = (double)__half2float(hs), z = (double)__half2float(hz);
  uint32_t c[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    double t = s != 0.0 ? rint(((double)x[i] - z) / s) : 0.0;
    t = fmin(fmax(t, 0.0), (double)QMAX);
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
            const int32_t *__restrict__ idx, int nbh, int L, int window, int k_vert,
            uint8_t *__restrict__ k_codes, uint8_t *__restrict__ v_codes,
            __half2 *__restrict__ k_sz, __half2 *__restrict__ v_sz,
            __nv_bfloat16 *__restrict__ k_hi, __nv_bfloat16 *__restrict__ v_hi,
            int32_t *__restrict__ lo_pos, uint32_t *status) {
  constexpr int W32 = D / 64;                 // 32-bit words of bf16 per lane
  constexpr int ROWB = D * BITS / 8;          // packed bytes per low row
  constexpr int NG = D / 32;
  const int lane = threadIdx.x & 31;
  const int n_lo = L - window - k_vert, n_hi = k_vert + window;
  const long long total = (long long)nbh * L;
  const long long warp0 = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const long long nwarps = (long long)gridDim.x * kWarps;

  // Device-side check of the index list (ascending, distinct, in range).
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < (long long)nbh * k_vert;
       t += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(t % k_vert);
    const int x = idx[t];
    if (x < 0 || x >= L - window || (r > 0 && idx[t - 1] >= x)) raise_status(status, HQ_DEV_BAD_INDEX);
  }

  for (long long wi = warp0; wi < total; wi += nwarps) {
    const int bh = (int)(wi / L);
    const int j = (int)(wi % L);
    const size_t src = ((size_t)bh * L + j) * D;
    uint32_t kw[W32], vw[W32];
#pragma unroll
    for (int i = 0; i < W32; ++i) {
      kw[i] = __ldg(reinterpret_cast<const uint32_t *>(k + src) + lane * W32 + i);
      vw[i] = __ldg(reinterpret_cast<const uint32_t *>(v + src) + lane * W32 + i);
    }
    int hi_row = -1, lo_row = -1;
    if (j >= L - window) {
      hi_row = k_vert + (j - (L - window));
    } else {
      const int32_t *id = idx + (size_t)bh * k_vert;
      const int cnt = upper_bound_i32(id, k_vert, j);  // entries <= j
      if (cnt > 0 && __ldg(id + cnt - 1) == j) hi_row = cnt - 1;
      else lo_row = j - cnt;
    }
    if (hi_row >= 0) {
      if (hi_row >= n_hi) { if (lane == 0) raise_status(status, HQ_DEV_BAD_INDEX); continue; }
      const size_t dst = ((size_t)bh * n_hi + hi_row) * D;
#pragma unroll
      for (int i = 0; i < W32; ++i) {
        reinterpret_cast<uint32_t *>(k_hi + dst)[lane * W32 + i] = kw[i];
        reinterpret_cast<uint32_t *>(v_hi + dst)[lane * W32 + i] = vw[i];
      }
    } else {
      if (lo_row < 0 || lo_row >= n_lo) { if (lane == 0) raise_status(status, HQ_DEV_BAD_INDEX); continue; }
      const size_t r = (size_t)bh * n_lo + lo_row;
      quant_store<D, BITS>(kw, k_codes + r * ROWB, k_sz + r * NG, lane);
      quant_store<D, BITS>(vw, v_codes + r * ROWB, v_sz + r * NG, lane);
      if (lo_pos && lane == 0) lo_pos[r] = j;
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
  const long long warps = (long long)nbh * L;
  long long blocks = (warps + kWarps - 1) / kWarps;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  pack_kernel<D, BITS><<<(unsigned)blocks, kWarps * 32, 0, s>>>(
      k, v, idx, nbh, L, window, k_vert, (uint8_t *)o.k_codes, (uint8_t *)o.v_codes,
      (__half2 *)o.k_sz, (__half2 *)o.v_sz, (__nv_bfloat16 *)o.k_hi, (__nv_bfloat16 *)o.v_hi,
      o.lo_pos, status);
  return cudaGetLastError();
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

}  // namespace hq
