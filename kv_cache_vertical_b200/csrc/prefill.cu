// prefill.cu -- hybrid-precision prefill attention.
//
// Method: ACL abstract of HyQuant, Prefill stage: a hybrid-precision attention
// operator keeps the vertical-line tokens and a local sliding window at full
// precision and quantizes the remaining context; "HyQuant: Hybrid-Precision
// Quantization for LLM Attention" (wiki summary), TL;DR: the same rule governs
// prefill and decode.  Per causal pair (i, j <= i): "high" when j is in the
// window (j > i - W) or is a vertical column, else "low".  High logits are bf16
// q.k (fp32 accumulate); low logits are INT8 q.k (exact s32) times the per-row
// Q scale and per-64-key-block K scale; one online softmax covers both; P.V
// takes fp16 P and V (V converted exactly from bf16) with fp32 accumulation.
//
// Pre-pass (P4): INT8 (or E4M3) codes for Q per row and for the remaining
// (non-vertical) keys per 64 of them, fp16 V in position order and compacted
// like the remaining keys, and a compact bf16 K / fp16 V copy of the vertical
// rows with their positions (so vertical tiles are dense TMA loads, not
// gathers).  The attention kernel that consumes them is prefill_tc.cu's
// (tcgen05, head_dim 128, an even number of query heads per KV head); other
// shapes are rejected on the host.
#include <float.h>
#include <limits.h>

#include <cuda_fp8.h>

#include "hq_internal.cuh"

namespace hq {
namespace {

constexpr int TILE = 64;        // queries per CTA, keys per tile, K-scale block
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Pre-pass kernels
// ---------------------------------------------------------------------------

// x / s rounded to the nearest integer (ties to even), with the quotient a
// single IEEE binary32 rounding.  The product with the rounded reciprocal is
// within 2^-16 of the quotient for |x / s| <= 2^7, so it decides every code
// that is not within 2^-12 of a half-integer; the rest divide exactly.
__device__ __forceinline__ float rint_div(float x, float s, float rcp_s) {
  const float q = x * rcp_s;
  const float t = rintf(q);
  return fabsf(q - t) > 0.5f - 1.f / 4096.f ? rintf(__fdiv_rn(x, s)) : t;
}

// FP8 low part: E4M3 codes of fl32(x0 / s), fl32(x1 / s) (nearest even,
// saturating), low byte first.  The paired hardware conversion rounds the
// reciprocal products, which lie within two units of the binary32 quotients;
// where one is near an E4M3 tie the quotient itself is taken.
__device__ __forceinline__ uint32_t f8_pair_div(float x0, float x1, float s, float rcp) {
  float q0 = x0 * rcp, q1 = x1 * rcp;
  if (e4m3_near_tie(q0)) q0 = __fdiv_rn(x0, s);
  if (e4m3_near_tie(q1)) q1 = __fdiv_rn(x1, s);
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(q0, q1), __NV_SATFINITE, __NV_E4M3);
}

// Q rows: s = amax / 127, code = clamp(rne(x / s), -127, 127), both
// divisions single IEEE binary32 roundings.  Each lane takes one 32-channel
// group of a row (D / 32 lanes per row, two or one shuffles for the row's
// maximum), a warp QPASS passes of 32 / (D / 32) rows with every load issued
// first; codes leave in 16-byte stores.
constexpr int QPASS = 2;
// With F8 the codes are E4M3 of fl32(x / s), s = amax / 448 (f8_pair_div).
template <int D, bool F8>
__global__ void __launch_bounds__(256)
quant_q_rows(const __nv_bfloat16 *__restrict__ q, long long nrows, int8_t *__restrict__ qi8,
             float *__restrict__ sq) {
  constexpr int NG = D / 32;                    // lanes per row
  constexpr int RP = 32 / NG;                   // rows per pass
  const int lane = threadIdx.x & 31;
  const int g = lane % NG;
  const long long row0 = ((long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * (RP * QPASS) +
                         lane / NG;
  uint32_t w[QPASS][16];
#pragma unroll
  for (int pi = 0; pi < QPASS; ++pi) {
    const long long row = row0 + pi * RP;
    const uint4 *src = reinterpret_cast<const uint4 *>(q + (row < nrows ? row : nrows - 1) * D + g * 32);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 t = __ldg(src + u);
      w[pi][4 * u] = t.x;
      w[pi][4 * u + 1] = t.y;
      w[pi][4 * u + 2] = t.z;
      w[pi][4 * u + 3] = t.w;
    }
  }
#pragma unroll
  for (int pi = 0; pi < QPASS; ++pi) {
    const long long row = row0 + pi * RP;
    uint32_t am = w[pi][0] & 0x7fff7fffu;       // |x| of both halves
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      uint32_t d;
      asm("max.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(am), "r"(w[pi][i] & 0x7fff7fffu));
      am = d;
    }
    float amax = fmaxf(bf16_lo(am), bf16_hi(am));
#pragma unroll
    for (int o = NG / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (row >= nrows) continue;
    const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, F8 ? 448.f : 127.f);
    const float rcp = __frcp_rn(s);
    uint32_t out[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t packed = 0;
      if (F8) {
        const uint32_t a0 = w[pi][2 * k], a1 = w[pi][2 * k + 1];
        packed = f8_pair_div(bf16_lo(a0), bf16_hi(a0), s, rcp) |
                 (f8_pair_div(bf16_lo(a1), bf16_hi(a1), s, rcp) << 16);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t word = w[pi][2 * k + (e >> 1)];
          const float x = (e & 1) ? bf16_hi(word) : bf16_lo(word);
          const float c = fminf(fmaxf(rint_div(x, s, rcp), -127.f), 127.f);
          packed |= ((uint32_t)(int)c & 0xffu) << (8 * e);
        }
      }
      out[k] = packed;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(qi8 + row * D + g * 32);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    if (g == 0) sq[row] = s;
  }
}

// Position of the c-th remaining (non-vertical) key: c plus the number of
// vertical columns before it, i.e. the count of r with idx[r] - r <= c.
__device__ __forceinline__ int remaining_pos(const int32_t *id, int k_vert, int c) {
  int lo = 0, hi = k_vert;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(id + mid) - mid <= c) lo = mid + 1;
    else hi = mid;
  }
  return c + lo;
}

// One CTA (256 threads) per block of 64 consecutive remaining keys of one
// (b, kv head): INT8 codes with one symmetric scale per block.  The block's
// rows are read once, 16 bytes per load, and held in registers for both the
// maximum and the codes.
template <int D, bool F8>
__global__ void __launch_bounds__(256)
quant_k_remaining(const __nv_bfloat16 *__restrict__ k, const int32_t *__restrict__ idx, int N,
                  int k_vert, int nblk, int8_t *__restrict__ ki8, float *__restrict__ sk) {
  constexpr int U = D / 8;                                      // 16-byte pieces per row
  constexpr int PER = TILE * U / 256;                           // pieces per thread: 4 or 2
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int nr = N - k_vert;
  const int c0 = blk * TILE, n = min(TILE, nr - c0);
  const int32_t *id = idx + (size_t)bh * k_vert;
  __shared__ int pos[TILE];
  __shared__ float red[8];
  if (threadIdx.x < n) pos[threadIdx.x] = remaining_pos(id, k_vert, c0 + threadIdx.x);
  __syncthreads();
  const uint4 *src = reinterpret_cast<const uint4 *>(k + (size_t)bh * N * D);
  uint4 v[PER];
  uint32_t am = 0u;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int e = threadIdx.x + q * 256;                        // piece e % U of row e / U
    v[q] = e < n * U ? __ldg(src + (size_t)pos[e / U] * U + e % U) : make_uint4(0, 0, 0, 0);
    const uint32_t ww[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t d;
      asm("max.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(am), "r"(ww[i] & 0x7fff7fffu));
      am = d;
    }
  }
  float amax = fmaxf(bf16_lo(am), bf16_hi(am));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, F8 ? 448.f : 127.f);
  const float rcp = __frcp_rn(s);
  uint2 *dst = reinterpret_cast<uint2 *>(ki8 + ((size_t)bh * nr + c0) * D);   // 8 codes per piece
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int e = threadIdx.x + q * 256;
    if (e >= n * U) break;
    const uint32_t ww[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t packed = 0;
      if (F8) {
        const uint32_t a0 = ww[2 * h], a1 = ww[2 * h + 1];
        packed = f8_pair_div(bf16_lo(a0), bf16_hi(a0), s, rcp) |
                 (f8_pair_div(bf16_lo(a1), bf16_hi(a1), s, rcp) << 16);
      } else {
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const uint32_t word = ww[2 * h + (e4 >> 1)];
          const float x = (e4 & 1) ? bf16_hi(word) : bf16_lo(word);
          const float c = fminf(fmaxf(rint_div(x, s, rcp), -127.f), 127.f);
          packed |= ((uint32_t)(int)c & 0xffu) << (8 * e4);
        }
      }
      out[h] = packed;
    }
    dst[e] = make_uint2(out[0], out[1]);
  }
  if (threadIdx.x == 0) sk[(size_t)bh * nblk + blk] = s;
}

// bf16 V -> fp16 V (exact for |v| in the fp16 normal range), both in position
// order (window tiles) and compacted to the remaining keys (low-bit tiles).
// One CTA per span of VSPAN consecutive positions of one (b, kv head): warp 0
// counts the verticals before the span (one warp search) and marks those in
// it in a shared bit mask while every warp loads its first rows; each warp
// then converts and stores its 32 positions, 16 bytes per lane and access.
constexpr int VSPAN = 256;
template <int D>
__global__ void __launch_bounds__(256)
v_prep(const __nv_bfloat16 *__restrict__ v, const int32_t *__restrict__ idx, int nbh, int N,
       int k_vert, __half *__restrict__ vh, __half *__restrict__ vc) {
  constexpr int LPR = D / 8;                                     // lanes per row (16 bytes each)
  constexpr int RPI = 32 / LPR;                                  // rows per warp access: 2 or 4
  constexpr int PCH = 8;                                         // positions per chunk
  constexpr int NA = PCH / RPI;                                  // accesses per chunk per lane
  __shared__ uint32_t vmask[VSPAN / 32];
  __shared__ int s_lo;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nspan = (N + VSPAN - 1) / VSPAN;
  const int bh = (int)(blockIdx.x / nspan);
  const int p0 = (int)(blockIdx.x % nspan) * VSPAN;
  const int p1 = min(p0 + VSPAN, N);
  const int nr = N - k_vert;
  const int32_t *id = idx + (size_t)bh * k_vert;
  const int piece = lane % LPR, rsub = lane / LPR;
  if (threadIdx.x < VSPAN / 32) vmask[threadIdx.x] = 0u;
  uint4 w[NA];
  auto load_chunk = [&](int j0) {
#pragma unroll
    for (int a = 0; a < NA; ++a) {
      const int j = min(j0 + a * RPI + rsub, N - 1);
      w[a] = __ldg(reinterpret_cast<const uint4 *>(v + ((size_t)bh * N + j) * D) + piece);
    }
  };
  const int jw = p0 + warp * (VSPAN / 8);                       // this warp's 32 positions
  if (jw < p1) load_chunk(jw);
  __syncthreads();                                               // mask cleared
  if (warp == 0) {
    const int lo = warp_count_below(id, k_vert, p0, lane);
    if (lane == 0) s_lo = lo;
    for (int t = lo + lane;; t += 32) {
      const int x = t < k_vert ? __ldg(id + t) : INT_MAX;
      if (x >= p0 && x < p1) atomicOr(&vmask[(x - p0) >> 5], 1u << ((x - p0) & 31));
      if (__any_sync(0xffffffffu, x >= p1)) break;
    }
  }
  __syncthreads();
  const int lo = s_lo;
  for (int ci = 0; ci < VSPAN / 8 / PCH; ++ci) {
    const int j0 = jw + ci * PCH;
    if (j0 >= p1) break;
    if (ci > 0) load_chunk(j0);
#pragma unroll
    for (int a = 0; a < NA; ++a) {
      const int j = j0 + a * RPI + rsub;
      if (j >= p1) continue;
      const int o = j - p0;
      uint32_t before = 0;                                       // verticals in the span before j
      for (int wdx = 0; wdx < (o >> 5); ++wdx) before += __popc(vmask[wdx]);
      const uint32_t word = vmask[o >> 5];
      before += __popc(word & ((1u << (o & 31)) - 1u));
      const bool vert = (word >> (o & 31)) & 1u;
      const int rank = j - lo - (int)before;                     // among the remaining keys
      const uint32_t ww[4] = {w[a].x, w[a].y, w[a].z, w[a].w};
      uint32_t hh[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 x = __floats2half2_rn(bf16_lo(ww[i]), bf16_hi(ww[i]));
        hh[i] = *reinterpret_cast<const uint32_t *>(&x);
      }
      const uint4 out = make_uint4(hh[0], hh[1], hh[2], hh[3]);
      reinterpret_cast<uint4 *>(vh + ((size_t)bh * N + j) * D)[piece] = out;
      if (!vert && rank >= 0 && rank < nr) reinterpret_cast<uint4 *>(vc + ((size_t)bh * nr + rank) * D)[piece] = out;
    }
  }
}

// Compact copies of the vertical rows (padded to whole 128-row tiles with zero
// rows at position INT_MAX).  Also checks the index list: strictly ascending,
// every column in [0, N - window); a violation sets HQ_DEV_BAD_INDEX (the
// attention that follows stays in bounds but its result is meaningless).
template <int D>
__global__ void gather_vertical(const __nv_bfloat16 *__restrict__ k, const __half *__restrict__ vh,
                                const int32_t *__restrict__ idx, int N, int window, int k_vert,
                                int kpad, __nv_bfloat16 *__restrict__ kv_k, __half *__restrict__ kv_v,
                                int32_t *__restrict__ kv_pos, uint32_t *status) {
  const int r = blockIdx.x, bh = blockIdx.y;  // one CTA (D/8 threads) per padded row
  const int t = threadIdx.x;                  // 16-byte chunk of the row
  const int pos = r < k_vert ? idx[(size_t)bh * k_vert + r] : INT_MAX;
  if (t == 0 && r < k_vert &&
      (pos < 0 || pos >= N - window || (r > 0 && idx[(size_t)bh * k_vert + r - 1] >= pos)))
    raise_status(status, HQ_DEV_BAD_INDEX);
  const size_t dst = ((size_t)bh * kpad + r) * D;
  uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
  if (r < k_vert && pos >= 0 && pos < N) {
    kk = reinterpret_cast<const uint4 *>(k + ((size_t)bh * N + pos) * D)[t];
    vv = reinterpret_cast<const uint4 *>(vh + ((size_t)bh * N + pos) * D)[t];
  }
  reinterpret_cast<uint4 *>(kv_k + dst)[t] = kk;
  reinterpret_cast<uint4 *>(kv_v + dst)[t] = vv;
  if (t == 0) kv_pos[(size_t)bh * kpad + r] = pos;
}

struct PrefillWs {
  int8_t *qi8, *ki8;
  float *sq, *sk;
  __half *vh, *vc, *vv;
  __nv_bfloat16 *vk;
  int32_t *vpos;
  size_t total;
};

PrefillWs carve(uint8_t *base, int B, int Hq, int Hkv, int N, int D, int k_vert) {
  PrefillWs w;
  const size_t nbh = (size_t)B * Hkv, nbq = (size_t)B * Hq;
  const size_t nr = (size_t)(N - k_vert);
  const size_t nblk_r = (nr + TILE - 1) / TILE;
  const size_t kpad = (size_t)((k_vert + 127) / 128) * 128;  // whole 128-row tiles
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    uint8_t *p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  };
  w.qi8 = (int8_t *)take(nbq * N * D);
  w.sq = (float *)take(nbq * N * sizeof(float));
  w.ki8 = (int8_t *)take(nbh * nr * D);
  w.sk = (float *)take(nbh * nblk_r * sizeof(float));
  w.vh = (__half *)take(nbh * N * D * 2);
  w.vc = (__half *)take(nbh * nr * D * 2);
  w.vk = (__nv_bfloat16 *)take(nbh * kpad * D * 2);
  w.vv = (__half *)take(nbh * kpad * D * 2);
  w.vpos = (int32_t *)take(nbh * kpad * sizeof(int32_t));
  w.total = off;
  return w;
}

template <int D, bool F8>
cudaError_t quant_t(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const int32_t *idx, int B,
                    int Hq, int Hkv, int N, int k_vert, int8_t *qi8, float *sq, int8_t *ki8,
                    float *sk, cudaStream_t s) {
  const long long nrows = (long long)B * Hq * N;
  const long long rows_per_block = 8LL * (32 / (D / 32)) * QPASS;        // 8 warps
  quant_q_rows<D, F8><<<(unsigned)((nrows + rows_per_block - 1) / rows_per_block), 256, 0, s>>>(q, nrows, qi8, sq);
  const int nblk_r = (N - k_vert + TILE - 1) / TILE;
  if (nblk_r > 0)
    quant_k_remaining<D, F8><<<dim3(nblk_r, B * Hkv), 256, 0, s>>>(k, idx, N, k_vert, nblk_r, ki8, sk);
  return cudaGetLastError();
}

// The pre-pass kernels, then the tcgen05 attention kernel.  Shapes the
// tensor-core kernel does not take were rejected on the host; if the compiled
// kernel is not usable (see prefill_tc_supported) nothing is launched.
template <int D>
cudaError_t prefill_t(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                      const int32_t *idx, int B, int Hq, int Hkv, int N, int window, int k_vert,
                      float scale, int low_fmt, float *out, uint8_t *ws, uint32_t *status,
                      cudaStream_t s) {
  if (!prefill_tc_supported(D, Hq, Hkv)) return cudaErrorNotSupported;
  const bool f8 = low_fmt == HQ_KV_FP8;
  PrefillWs w = carve(ws, B, Hq, Hkv, N, D, k_vert);
  const int nbh = B * Hkv;
  const int nr = N - k_vert;
  const int nblk_r = (nr + TILE - 1) / TILE;
  const int kpad = (k_vert + 127) / 128 * 128;
  cudaError_t e = f8 ? quant_t<D, true>(q, k, idx, B, Hq, Hkv, N, k_vert, w.qi8, w.sq, w.ki8, w.sk, s)
                     : quant_t<D, false>(q, k, idx, B, Hq, Hkv, N, k_vert, w.qi8, w.sq, w.ki8, w.sk, s);
  if (e != cudaSuccess) return e;
  {
    const long long blocks = (long long)nbh * ((N + VSPAN - 1) / VSPAN);   // one CTA per span
    v_prep<D><<<(unsigned)blocks, 256, 0, s>>>(v, idx, nbh, N, k_vert, w.vh, w.vc);
  }
  if (kpad > 0)
    gather_vertical<D><<<dim3(kpad, nbh), D / 8, 0, s>>>(k, w.vh, idx, N, window, k_vert, kpad,
                                                         w.vk, w.vv, w.vpos, status);
  TcLaunch p;
  p.q = q;
  p.k = k;
  p.qi8 = w.qi8;
  p.ki8 = w.ki8;
  p.sq = w.sq;
  p.sk = w.sk;
  p.vh = w.vh;
  p.vc = w.vc;
  p.vk = w.vk;
  p.vv = w.vv;
  p.idx = idx;
  p.out = out;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.window = window;
  p.k_vert = k_vert;
  p.kpad = kpad;
  p.nblk_r = nblk_r;
  p.scale = scale;
  p.f8 = f8;
  return launch_prefill_tc(p, s);
}

}  // namespace

cudaError_t launch_prefill_quant(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                 const int32_t *idx, int B, int Hq, int Hkv, int N, int D,
                                 int k_vert, int low_fmt, int8_t *qi8, float *sq, int8_t *ki8,
                                 float *sk, cudaStream_t s) {
  const bool f8 = low_fmt == HQ_KV_FP8;
  if (D == 128 && !f8) return quant_t<128, false>(q, k, idx, B, Hq, Hkv, N, k_vert, qi8, sq, ki8, sk, s);
  if (D == 64 && !f8) return quant_t<64, false>(q, k, idx, B, Hq, Hkv, N, k_vert, qi8, sq, ki8, sk, s);
  if (D == 128 && f8) return quant_t<128, true>(q, k, idx, B, Hq, Hkv, N, k_vert, qi8, sq, ki8, sk, s);
  if (D == 64 && f8) return quant_t<64, true>(q, k, idx, B, Hq, Hkv, N, k_vert, qi8, sq, ki8, sk, s);
  return cudaErrorInvalidValue;
}

size_t prefill_ws_bytes(int B, int Hq, int Hkv, int N, int D, int k_vert) {
  return carve(nullptr, B, Hq, Hkv, N, D, k_vert).total;
}

cudaError_t launch_prefill(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                           const __nv_bfloat16 *v, const int32_t *idx, int B, int Hq, int Hkv,
                           int N, int D, int window, int k_vert, float scale, int low_fmt,
                           float *out, uint8_t *ws, uint32_t *status, cudaStream_t s) {
  if (D == 128) return prefill_t<128>(q, k, v, idx, B, Hq, Hkv, N, window, k_vert, scale, low_fmt, out, ws, status, s);
  return cudaErrorNotSupported;
}

}  // namespace hq
