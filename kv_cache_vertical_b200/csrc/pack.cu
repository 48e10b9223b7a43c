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
#include <cuda_fp8.h>
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

// FP8 format: per group of 32 channels s = fp16(amax / 448) (the quotient
// rounded once: scale_f16 with range amax - 0), c = E4M3(x / s) rounded to
// nearest even and saturated, z = 0.  The hardware conversion (nearest even,
// saturating) rounds an fp32 estimate of x / s, except where the estimate is
// near an E4M3 tie; there it rounds the double quotient taken to fp32 with
// round to odd.  Bit-exact to the definition.
template <int D>
__device__ __forceinline__ void quant_store_fp8(const uint32_t (&w)[D / 64], uint8_t *codes_row,
                                                __half2 *sz_row, int lane) {
  constexpr int CPL = D / 32;          // channels per lane: 4 (D=128) or 2 (D=64)
  constexpr int LPG = 32 / CPL;        // lanes per group
  float x[CPL];
#pragma unroll
  for (int i = 0; i < CPL / 2; ++i) {
    x[2 * i] = bf16_lo(w[i]);
    x[2 * i + 1] = bf16_hi(w[i]);
  }
  float amax = fabsf(x[0]);
#pragma unroll
  for (int i = 1; i < CPL; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int o = LPG / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half hs = scale_f16(amax, 0.f, 448);
  const float sf = __half2float(hs);
  const float rs = sf != 0.f ? __frcp_rn(sf) : 0.f;
  uint32_t c[CPL];
#pragma unroll
  for (int i = 0; i < CPL; i += 2) {
    float q0 = x[i] * rs, q1 = x[i + 1] * rs;
    if (e4m3_near_tie(q0)) q0 = f32_round_odd((double)x[i] / (double)sf);
    if (e4m3_near_tie(q1)) q1 = f32_round_odd((double)x[i + 1] / (double)sf);
    // one paired hardware conversion, nearest even, saturating (low byte = q0)
    const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3);
    c[i] = sf != 0.f ? two & 0xffu : 0u;
    c[i + 1] = sf != 0.f ? two >> 8 : 0u;
  }
  if (CPL == 4)
    reinterpret_cast<uint32_t *>(codes_row)[lane] = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  else
    reinterpret_cast<uint16_t *>(codes_row)[lane] = (uint16_t)(c[0] | (c[1] << 8));
  if (lane % LPG == 0) sz_row[lane / LPG] = __halves2half2(hs, __ushort_as_half((unsigned short)0));
}

// One row of the low segment in the cache's code format.
template <int D, int BITS, bool F8>
__device__ __forceinline__ void quant_row_store(const uint32_t (&w)[D / 64], uint8_t *codes_row,
                                                __half2 *sz_row, int lane) {
  if (F8)
    quant_store_fp8<D>(w, codes_row, sz_row, lane);
  else
    quant_store<D, BITS>(w, codes_row, sz_row, lane);
}

// ---------------------------------------------------------------------------
// One lane, one group: the pack kernel gives each lane the 32 channels of one
// quantization group of one row (16 words of bf16 pairs), so the group's
// min / max need no shuffles and its scale is computed once.  The arithmetic
// per value is that of quant_store / quant_store_fp8, so the codes, scales
// and zeros are the same bit for bit.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Codes of one group into `codes` (32 * BITS / 8 bytes, 16-byte aligned) and
// its (scale, zero) into *sz.
template <int BITS, bool F8>
__device__ __forceinline__ void quant_group_lane(const uint32_t (&w)[16], uint8_t *codes, __half2 *sz) {
  if (F8) {
    uint32_t am = w[0] & 0x7fff7fffu;                  // |x| of both halves (sign cleared)
#pragma unroll
    for (int i = 1; i < 16; ++i) am = bmax2(am, w[i] & 0x7fff7fffu);
    const float amax = fmaxf(bf16_lo(am), bf16_hi(am));
    const __half hs = scale_f16(amax, 0.f, 448);
    const float sf = __half2float(hs);
    const float rs = sf != 0.f ? __frcp_rn(sf) : 0.f;
    uint32_t out[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float x0 = bf16_lo(w[i]), x1 = bf16_hi(w[i]);
      float q0 = x0 * rs, q1 = x1 * rs;
      if (e4m3_near_tie(q0)) q0 = f32_round_odd((double)x0 / (double)sf);
      if (e4m3_near_tie(q1)) q1 = f32_round_odd((double)x1 / (double)sf);
      const uint32_t two = sf != 0.f
          ? (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3) : 0u;
      if (i & 1) out[i >> 1] |= two << 16;
      else out[i >> 1] = two;
    }
    reinterpret_cast<uint4 *>(codes)[0] = make_uint4(out[0], out[1], out[2], out[3]);
    reinterpret_cast<uint4 *>(codes)[1] = make_uint4(out[4], out[5], out[6], out[7]);
    *sz = __halves2half2(hs, __ushort_as_half((unsigned short)0));
    return;
  }
  constexpr int QMAX = (1 << BITS) - 1;
  uint32_t mnw = w[0], mxw = w[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    mnw = bmin2(mnw, w[i]);
    mxw = bmax2(mxw, w[i]);
  }
  const float mn = fminf(bf16_lo(mnw), bf16_hi(mnw)), mx = fmaxf(bf16_lo(mxw), bf16_hi(mxw));
  const float fmn = mn == 0.f ? 0.f : mn;              // a -0 minimum is stored as +0
  const __half hs = scale_f16(mx, mn, QMAX);
  const __half hz = __float2half_rn(fmn);
  const float sf = __half2float(hs), zf = __half2float(hz);
  const float rs = sf != 0.f ? __frcp_rn(sf) : 0.f;
  uint32_t c[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float x = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
    const float q = (x - zf) * rs;
    float t = rintf(q);
    if (sf == 0.f) {
      t = 0.f;
    } else if (fabsf(q - t) > 0.5f - 1.f / 4096.f) {
      t = (float)rint(((double)x - (double)zf) / (double)sf);
    }
    t = fminf(fmaxf(t, 0.f), (float)QMAX);
    c[i] = (uint32_t)t;
  }
  if (BITS == 4) {
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t v = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) v |= c[8 * k + e] << (4 * e);   // even channel in the low nibble
      out[k] = v;
    }
    reinterpret_cast<uint4 *>(codes)[0] = make_uint4(out[0], out[1], out[2], out[3]);
  } else {
    uint32_t out[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      out[k] = c[4 * k] | (c[4 * k + 1] << 8) | (c[4 * k + 2] << 16) | (c[4 * k + 3] << 24);
    reinterpret_cast<uint4 *>(codes)[0] = make_uint4(out[0], out[1], out[2], out[3]);
    reinterpret_cast<uint4 *>(codes)[1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
  *sz = __halves2half2(hs, hz);
}

// Asynchronous 16-byte copy global -> shared (completion: cp_async_wait).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// Wait until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Positions per CTA: kWarps warps x kChunks chunks x 8 positions.
constexpr int kChunks = 4;
constexpr int kSpan = kWarps * kChunks * 8;   // 256

// One CTA per span of kSpan consecutive positions of one (b, kv head): warp 0
// counts the vertical columns before the span (one search per CTA) and marks
// those inside it in a shared bit mask, while every warp issues the row loads
// of its first chunk; then each warp classifies and writes its four chunks of
// eight positions (copy the bf16 rows, or quantize them into the next low
// rows), each lane one 32-channel group of one row.  A chunk's 16 rows (K and
// V of its eight positions) are copied into the warp's shared-memory stage by
// cp.async while the warp works on the chunk before, so each warp has the
// next chunk's loads in flight during its quantization.  With a part [lo0, lo1) x
// [hi0, hi1) of the cache's rows (a context split across GPUs), only the rows
// inside it are written, at their offsets from lo0 / hi0.  Three CTAs per SM.
template <int D, int BITS, bool F8>
__global__ void __launch_bounds__(kWarps * 32, 3)
pack_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
            const int32_t *__restrict__ idx, int nbh, int L, int window, int k_vert,
            int lo0, int lo1, int hi0, int hi1, int lo_cap,
            uint8_t *__restrict__ k_codes, uint8_t *__restrict__ v_codes,
            __half2 *__restrict__ k_sz, __half2 *__restrict__ v_sz,
            __nv_bfloat16 *__restrict__ k_hi, __nv_bfloat16 *__restrict__ v_hi,
            int32_t *__restrict__ lo_pos, uint32_t *status) {
  constexpr int ROWB = D * BITS / 8;          // packed bytes per low row
  constexpr int NG = D / 32;                  // quantization groups per row
  constexpr int PCH = 8;
  __shared__ uint32_t vmask[kSpan / 32];
  __shared__ int s_lo;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_lo = L - window - k_vert, n_hi = k_vert + window;
  const int part_hi = hi1 - hi0;               // bf16 rows of the part (its row stride)
  const int nspan = (L + kSpan - 1) / kSpan;
  const int bh = (int)(blockIdx.x / nspan);
  const int p0 = (int)(blockIdx.x % nspan) * kSpan;
  const int p1 = min(p0 + kSpan, L);
  const int32_t *id = idx + (size_t)bh * k_vert;

  // Device-side check of the index list (ascending, distinct, in range).
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < (long long)nbh * k_vert;
       t += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(t % k_vert);
    const int x = idx[t];
    if (x < 0 || x >= L - window || (r > 0 && idx[t - 1] >= x)) raise_status(status, HQ_DEV_BAD_INDEX);
  }

  if (threadIdx.x < kSpan / 32) vmask[threadIdx.x] = 0u;
  // A chunk is 16 rows (K and V of eight positions); each lane takes one
  // 32-channel group of one row per pass: lane = row-in-pass * NG + group.
  constexpr int RP = 32 / NG;                 // rows per pass: 8 (D = 128) or 16 (D = 64)
  constexpr int NPASS = 16 / RP;
  const int g = lane % NG, rsub = lane / NG;
  // The warp's stage: 2 buffers x 16 rows (0-7: K of the chunk's positions,
  // 8-15: V), each row D bf16 plus 16 bytes of padding against bank conflicts.
  constexpr int ROWQ = D / 8 + 1;              // 16-byte units per staged row
  extern __shared__ uint4 pack_stage[];
  uint4 *const stg = pack_stage + warp * 2 * 16 * ROWQ;
  auto issue_chunk = [&](int j0, int b) {
#pragma unroll
    for (int u = 0; u < 16 * (D / 8) / 32; ++u) {
      const int qd = lane + 32 * u;
      const int rho = qd / (D / 8), c16 = qd % (D / 8);
      const int j = min(j0 + (rho & 7), L - 1);
      const __nv_bfloat16 *src = (rho < 8 ? k : v) + ((size_t)bh * L + j) * D + c16 * 8;
      cp_async16(stg + (b * 16 + rho) * ROWQ + c16, src);
    }
    cp_async_commit();
  };
  const int jw = p0 + warp * kChunks * PCH;    // this warp's first position
  if (jw < p1) issue_chunk(jw, 0);
  __syncthreads();                             // mask cleared
  if (warp == 0) {
    const int lo = warp_count_below(id, k_vert, p0, lane);
    if (lane == 0) s_lo = lo;
    // mark the span's verticals (at most kSpan entries follow lo)
    for (int t = lo + lane;; t += 32) {
      const int x = t < k_vert ? __ldg(id + t) : INT_MAX;
      if (x >= p0 && x < p1) atomicOr(&vmask[(x - p0) >> 5], 1u << ((x - p0) & 31));
      if (__any_sync(0xffffffffu, x >= p1)) break;
    }
  }
  __syncthreads();                             // mask and count ready
  const int lo = s_lo;

  for (int ci = 0; ci < kChunks; ++ci) {
    const int j0 = jw + ci * PCH;
    if (j0 >= p1) break;
    const bool more = ci + 1 < kChunks && j0 + PCH < p1;
    if (more) {
      issue_chunk(j0 + PCH, (ci + 1) & 1);     // the next chunk streams in meanwhile
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();                              // every lane's copies of this chunk have landed
    const uint4 *cst = stg + (ci & 1) * 16 * ROWQ;
    const int o = j0 - p0;                     // offset in the span, a multiple of 8
    uint32_t before = 0;                       // verticals in the span before j0
    for (int wdx = 0; wdx < (o >> 5); ++wdx) before += __popc(vmask[wdx]);
    const uint32_t word = vmask[o >> 5];
    before += __popc(word & ((1u << (o & 31)) - 1u));
    const uint32_t vbits = (word >> (o & 31)) & 0xffu;   // vertical positions of the chunk
    const int cnt0 = lo + (int)before;
#pragma unroll
    for (int pi = 0; pi < NPASS; ++pi) {
      const int rho = pi * RP + rsub;
      const bool is_v = rho >= 8;
      const int p = rho & 7;
      const int j = j0 + p;
      if (j >= L) continue;
      uint32_t w[16];                          // this lane's 32 channels of row rho
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 t = cst[rho * ROWQ + g * 4 + u];
        w[4 * u] = t.x;
        w[4 * u + 1] = t.y;
        w[4 * u + 2] = t.z;
        w[4 * u + 3] = t.w;
      }
      const int cnt = cnt0 + __popc(vbits & ((1u << p) - 1u));            // verticals before j
      int hi_row = -1, lo_row = -1;
      if (j >= L - window) hi_row = k_vert + j % window;          // the window ring
      else if (vbits & (1u << p)) hi_row = cnt;
      else lo_row = j - cnt;
      if (hi_row >= 0) {
        if (hi_row >= n_hi) {
          raise_status(status, HQ_DEV_BAD_INDEX);
          continue;
        }
        if (hi_row < hi0 || hi_row >= hi1) continue;   // another part's row
        uint4 *dst = reinterpret_cast<uint4 *>((is_v ? v_hi : k_hi) +
                                               ((size_t)bh * part_hi + hi_row - hi0) * D + g * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      } else {
        if (lo_row < 0 || lo_row >= n_lo) {
          raise_status(status, HQ_DEV_BAD_INDEX);
          continue;
        }
        if (lo_row < lo0 || lo_row >= lo1) continue;   // another part's row
        const size_t r = (size_t)bh * lo_cap + lo_row - lo0;
        quant_group_lane<BITS, F8>(w, (is_v ? v_codes : k_codes) + r * ROWB + g * (32 * BITS / 8),
                                   (is_v ? v_sz : k_sz) + r * NG + g);
        if (lo_pos && !is_v && g == 0) lo_pos[r] = j;
      }
    }
    __syncwarp();                              // this buffer is refilled two chunks on
  }
}

template <int D, int BITS, bool F8>
cudaError_t launch_pack_t(const __nv_bfloat16 *k, const __nv_bfloat16 *v, const int32_t *idx,
                          int nbh, int L, int window, int k_vert, int lo0, int hi0,
                          const hq_kv_cache &o, uint32_t *status, cudaStream_t s) {
  const long long blocks = (long long)nbh * ((L + kSpan - 1) / kSpan);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  // the warps' chunk stages: 2 buffers x 16 rows of D bf16 + 16 bytes each
  const size_t smem = (size_t)kWarps * 2 * 16 * (D / 8 + 1) * 16;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(pack_kernel<D, BITS, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return cudaErrorInvalidValue;
    attr = true;
  }
  pack_kernel<D, BITS, F8><<<(unsigned)blocks, kWarps * 32, smem, s>>>(
      k, v, idx, nbh, L, window, k_vert, lo0, lo0 + o.n_lo, hi0, hi0 + o.n_hi, lo_rows(o),
      (uint8_t *)o.k_codes, (uint8_t *)o.v_codes,
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
template <int D, int BITS, bool F8>
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
    quant_row_store<D, BITS, F8>(kw, k_codes + r * ROWB, k_sz + r * NG, lane);
    quant_row_store<D, BITS, F8>(vw, v_codes + r * ROWB, v_sz + r * NG, lane);
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
  quant_row_store<D, BITS, F8>(ko, k_codes + r * ROWB, k_sz + r * NG, lane);
  quant_row_store<D, BITS, F8>(vo, v_codes + r * ROWB, v_sz + r * NG, lane);
  if (lo_pos && lane == 0) lo_pos[r] = L - window;
#pragma unroll
  for (int i = 0; i < W32; ++i) {
    kh[i] = kw[i];
    vh[i] = vw[i];
  }
}

template <int D, int BITS, bool F8>
cudaError_t launch_kv_append_t(const __nv_bfloat16 *k_new, const __nv_bfloat16 *v_new, int nbh,
                               int L, int window, int k_vert, const hq_kv_cache &c,
                               cudaStream_t s) {
  const int blocks = (nbh + kWarps - 1) / kWarps;
  return pdl_launch(kv_append_kernel<D, BITS, F8>, dim3(blocks), dim3(kWarps * 32), 0, s, k_new, v_new,
                    nbh, L, window, k_vert, c.n_lo, lo_rows(c), (uint8_t *)c.k_codes,
                    (uint8_t *)c.v_codes, (__half2 *)c.k_sz, (__half2 *)c.v_sz,
                    (__nv_bfloat16 *)c.k_hi, (__nv_bfloat16 *)c.v_hi, c.lo_pos);
}

}  // namespace

cudaError_t launch_pack(const __nv_bfloat16 *k, const __nv_bfloat16 *v, const int32_t *idx,
                        int B, int Hkv, int L, int D, int window, int k_vert, int bits,
                        const hq_kv_cache &out, uint32_t *status, cudaStream_t s, int lo0, int hi0) {
  const int nbh = B * Hkv;
  const bool f8 = out.fmt == HQ_KV_FP8;
#define HQ_P(DD, BB, FF) \
  if (D == DD && bits == BB && f8 == FF) return launch_pack_t<DD, BB, FF>(k, v, idx, nbh, L, window, k_vert, lo0, hi0, out, status, s);
  HQ_P(128, 4, false) HQ_P(128, 8, false) HQ_P(64, 4, false) HQ_P(64, 8, false)
  HQ_P(128, 8, true) HQ_P(64, 8, true)
#undef HQ_P
  return cudaErrorInvalidValue;
}

cudaError_t launch_kv_append(const __nv_bfloat16 *k_new, const __nv_bfloat16 *v_new, int B,
                             int Hkv, int D, int L, int window, int k_vert,
                             const hq_kv_cache &c, cudaStream_t s) {
  const int nbh = B * Hkv;
  const bool f8 = c.fmt == HQ_KV_FP8;
#define HQ_A(DD, BB, FF) \
  if (D == DD && c.bits == BB && f8 == FF) return launch_kv_append_t<DD, BB, FF>(k_new, v_new, nbh, L, window, k_vert, c, s);
  HQ_A(128, 4, false) HQ_A(128, 8, false) HQ_A(64, 4, false) HQ_A(64, 8, false)
  HQ_A(128, 8, true) HQ_A(64, 8, true)
#undef HQ_A
  return cudaErrorInvalidValue;
}

}  // namespace hq
