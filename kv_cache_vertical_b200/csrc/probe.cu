// probe.cu -- vertical-line-aware pattern probe and top-k column selection.
//
// Method: "HyQuant: Hybrid-Precision Quantization for LLM Attention" (wiki
// summary), TL;DR and "What problem it solves": vertical-line tokens are the
// key columns that nearly every query row attends to, found by a cheap pattern
// signal; blog "How HyQuant uses hybrid-precision attention to cut decode
// compute", "Why preserve selected positions?": the top 5% of key positions
// (plus a 128-token window, kept separately).
//
// The signal of key j (per batch element and KV head) is the sum of the exact
// causal softmax weights that the P most recent queries of the G query heads of
// that KV head put on j.  Three kernels:
//   1. probe_qk<STATS>: per (key chunk of 128, KV head) CTA, S = Q K^T on
//      tensor cores (bf16 mma.sync, fp32 accumulate) for all G*P rows; writes
//      per-(row, chunk) partial max / sum-of-exp.
//   2. probe_row_stats: merges the partials into the row max m and sum Z.
//   3. probe_qk<COLSUM>: recomputes S, p = exp(s - m) / Z, and sums each
//      column over the G*P rows in a fixed order.
//   4. probe_topk: radix select of the k-th largest score in [0, L - W) with
//      (score desc, index asc) order, then an ordered compaction, so the list
//      comes out ascending and ties go to the lower index.
#include <float.h>

#include "hq_internal.cuh"
#include "warp_mma.cuh"

namespace hq {
namespace {

constexpr int KC = 128;          // keys per CTA
constexpr int PWARPS = 8;
constexpr float kLog2e = 1.4426950408889634f;

struct ProbeArgs {
  const __nv_bfloat16 *qp;
  int64_t q_head_stride;
  const __nv_bfloat16 *k;
  int Hq, Hkv, P, L, G, R, nchunk;
  float scale_log2;              // softmax scale * log2(e)
  float2 *partial;               // [nbh, R, nchunk] (max, sum) in log2 domain
  const float2 *stats;           // [nbh, R] (max, 1/Z) in log2 domain
  float *score;                  // [nbh, L]
};

// Loads the 16-row A fragments of a row tile straight from global memory.
template <int D>
__device__ __forceinline__ void load_q_frag(const ProbeArgs &a, int b, int kh, int row0,
                                            uint32_t (&qa)[D / 16][4]) {
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = row0 + r + half * 8;
    const uint32_t *src = nullptr;
    if (row < a.R) {
      const int g = row / a.P, p = row % a.P;
      const int h = kh * a.G + g;
      src = reinterpret_cast<const uint32_t *>(a.qp + ((int64_t)b * a.Hq + h) * a.q_head_stride +
                                               (int64_t)p * D);
    }
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa[ks][half] = src ? __ldg(src + ks * 8 + c) : 0u;
      qa[ks][half + 2] = src ? __ldg(src + ks * 8 + 4 + c) : 0u;
    }
  }
}

template <int D, bool COLSUM>
__global__ void __launch_bounds__(PWARPS * 32) probe_qk(ProbeArgs a) {
  constexpr int CH = D / 8;                    // 16-byte chunks per key row
  __shared__ __align__(128) uint4 ks[KC * CH];  // K chunk, XOR-swizzled by key
  __shared__ float colacc[PWARPS][KC];
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.Hkv, kh = bh % a.Hkv;
  const int j0 = chunk * KC;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint4 *kg = reinterpret_cast<const uint4 *>(a.k + ((size_t)bh * a.L) * D);
  for (int t = threadIdx.x; t < KC * CH; t += blockDim.x) {
    const int key = t / CH, ch = t % CH;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (j0 + key < a.L) val = __ldg(kg + (size_t)(j0 + key) * CH + ch);
    ks[key * CH + (ch ^ (key & 7))] = val;
  }
  if (COLSUM)
    for (int t = threadIdx.x; t < PWARPS * KC; t += blockDim.x) (&colacc[0][0])[t] = 0.f;
  __syncthreads();

  const int r = lane >> 2, c = lane & 3;
  const int ntile_rows = (a.R + 15) / 16;
  for (int rt = warp; rt < ntile_rows; rt += PWARPS) {
    uint32_t qa[D / 16][4];
    load_q_frag<D>(a, b, kh, rt * 16, qa);
    float acc[KC / 8][4];
#pragma unroll
    for (int nt = 0; nt < KC / 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < KC / 8; ++nt) {
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp) {
        const int key = nt * 8 + (lane & 7);
        const int ch = kp * 4 + (lane >> 3);
        uint32_t bf[4];
        ldsm_x4(bf, smem_u32(&ks[key * CH + (ch ^ (key & 7))]));
        mma_bf16_16816(acc[nt], qa[2 * kp], bf[0], bf[1]);
        mma_bf16_16816(acc[nt], qa[2 * kp + 1], bf[2], bf[3]);
      }
    }
    // Rows of this thread: rt*16 + r (+8).  Visible keys: j <= L - P + p.
    int lastj[2];
    bool valid[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = rt * 16 + r + hf * 8;
      valid[hf] = row < a.R;
      lastj[hf] = valid[hf] ? a.L - a.P + (row % a.P) : -1;
    }
    if (!COLSUM) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float m = -FLT_MAX;
#pragma unroll
        for (int nt = 0; nt < KC / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = j0 + nt * 8 + 2 * c + e;
            if (j <= lastj[hf]) m = fmaxf(m, acc[nt][2 * hf + e] * a.scale_log2);
          }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < KC / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = j0 + nt * 8 + 2 * c + e;
            if (j <= lastj[hf]) sum += exp2f(acc[nt][2 * hf + e] * a.scale_log2 - m);
          }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (c == 0 && valid[hf]) {
          const int row = rt * 16 + r + hf * 8;
          a.partial[((size_t)bh * a.R + row) * a.nchunk + chunk] = make_float2(m, sum);
        }
      }
    } else {
      float2 st[2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = rt * 16 + r + hf * 8;
        st[hf] = valid[hf] ? a.stats[(size_t)bh * a.R + row] : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int nt = 0; nt < KC / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + nt * 8 + 2 * c + e;
          float col = 0.f;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            if (j <= lastj[hf]) col += exp2f(acc[nt][2 * hf + e] * a.scale_log2 - st[hf].x) * st[hf].y;
          col += __shfl_xor_sync(0xffffffffu, col, 4);
          col += __shfl_xor_sync(0xffffffffu, col, 8);
          col += __shfl_xor_sync(0xffffffffu, col, 16);
          if (r == 0) colacc[warp][nt * 8 + 2 * c + e] += col;
        }
      }
    }
  }
  if (COLSUM) {
    __syncthreads();
    for (int t = threadIdx.x; t < KC; t += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < PWARPS; ++w) s += colacc[w][t];
      if (j0 + t < a.L) a.score[(size_t)bh * a.L + j0 + t] = s;
    }
  }
}

// Row max / 1/Z from the per-chunk partials (log2 domain).
__global__ void probe_row_stats(const float2 *__restrict__ partial, float2 *__restrict__ stats,
                                int nrows, int nchunk) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= nrows) return;
  const float2 *pr = partial + (size_t)row * nchunk;
  float m = -FLT_MAX;
  for (int c = 0; c < nchunk; ++c) m = fmaxf(m, pr[c].x);
  float z = 0.f;
  for (int c = 0; c < nchunk; ++c) z += pr[c].y * exp2f(pr[c].x - m);
  stats[row] = make_float2(m, 1.0f / z);
}

// ---------------------------------------------------------------------------
// Top-k: one CTA per (b, kv head).
// ---------------------------------------------------------------------------
constexpr int TK_THREADS = 1024;

__device__ __forceinline__ uint32_t score_key(float x) {
  // Order-preserving map of a float to uint32 (larger float -> larger key).
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum of one int per thread; returns the total.
__device__ int block_exclusive_scan(int v, int *tmp, int &excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (TK_THREADS / 32) ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    tmp[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int warp_base = warp ? tmp[warp - 1] : 0;
  excl = warp_base + x - v;
  const int total = tmp[TK_THREADS / 32 - 1];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(TK_THREADS)
probe_topk(const float *__restrict__ score, int L, int ncand, int k, int32_t *__restrict__ idx) {
  __shared__ int hist[256];
  __shared__ int tmp[32];
  __shared__ uint32_t sel_prefix, sel_mask;
  __shared__ int remain;
  const int bh = blockIdx.x;
  const float *s = score + (size_t)bh * L;
  int32_t *out = idx + (size_t)bh * k;
  if (k == 0) return;
  if (threadIdx.x == 0) {
    sel_prefix = 0;
    sel_mask = 0;
    remain = k;
  }
  // Radix select of the k-th largest key, 8 bits at a time from the top.
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0;
    __syncthreads();
    const uint32_t pre = sel_prefix, msk = sel_mask;
    for (int j = threadIdx.x; j < ncand; j += blockDim.x) {
      const uint32_t key = score_key(s[j]);
      if ((key & msk) == pre) atomicAdd(&hist[(key >> shift) & 0xff], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int need = remain, acc = 0, bin = 255;
      for (; bin > 0; --bin) {
        if (acc + hist[bin] >= need) break;
        acc += hist[bin];
      }
      remain = need - acc;  // how many to take from the selected bin
      sel_prefix = pre | ((uint32_t)bin << shift);
      sel_mask = msk | (0xffu << shift);
    }
    __syncthreads();
  }
  const uint32_t thr = sel_prefix;  // key of the k-th largest score
  const int take_eq = remain;       // equal keys to take, lowest indices first
  int out_base = 0, eq_base = 0;
  for (int base = 0; base < ncand; base += blockDim.x) {
    const int j = base + threadIdx.x;
    uint32_t key = 0;
    if (j < ncand) key = score_key(s[j]);
    const int gt = (j < ncand) && key > thr;
    const int eq = (j < ncand) && key == thr;
    int eq_excl;
    const int eq_tot = block_exclusive_scan(eq, tmp, eq_excl);
    const int take = gt || (eq && (eq_base + eq_excl) < take_eq);
    int pos;
    const int tot = block_exclusive_scan(take, tmp, pos);
    if (take) out[out_base + pos] = j;
    out_base += tot;
    eq_base += eq_tot;
  }
}

template <int D>
cudaError_t launch_probe_t(ProbeArgs a, int nbh, int k_vert, int window, int32_t *idx,
                           cudaStream_t s) {
  dim3 grid(a.nchunk, nbh);
  probe_qk<D, false><<<grid, PWARPS * 32, 0, s>>>(a);
  const int nrows = nbh * a.R;
  probe_row_stats<<<(nrows + 255) / 256, 256, 0, s>>>(a.partial, const_cast<float2 *>(a.stats),
                                                      nrows, a.nchunk);
  probe_qk<D, true><<<grid, PWARPS * 32, 0, s>>>(a);
  probe_topk<<<nbh, TK_THREADS, 0, s>>>(a.score, a.L, a.L - window, k_vert, idx);
  return cudaGetLastError();
}

}  // namespace

size_t probe_ws_bytes(int B, int Hq, int Hkv, int P, int L, int D) {
  (void)D;
  const size_t nbh = (size_t)B * Hkv, R = (size_t)(Hq / Hkv) * P;
  const size_t nchunk = (L + KC - 1) / KC;
  size_t off = kWsHeader;
  off = align_up(off + nbh * R * nchunk * sizeof(float2), 256);  // partials
  off = align_up(off + nbh * R * sizeof(float2), 256);           // stats
  off = align_up(off + nbh * (size_t)L * sizeof(float), 256);    // scores
  return off;
}

cudaError_t launch_probe(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                         const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int L, int D,
                         int window, int k_vert, float scale, int32_t *idx_out, float *score_out,
                         uint8_t *ws, cudaStream_t s) {
  ProbeArgs a;
  a.qp = q_probe;
  a.q_head_stride = q_head_stride;
  a.k = k;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.P = P;
  a.L = L;
  a.G = Hq / Hkv;
  a.R = a.G * P;
  a.nchunk = (L + KC - 1) / KC;
  a.scale_log2 = scale * kLog2e;
  const size_t nbh = (size_t)B * Hkv;
  size_t off = kWsHeader;
  a.partial = reinterpret_cast<float2 *>(ws + off);
  off = align_up(off + nbh * a.R * a.nchunk * sizeof(float2), 256);
  a.stats = reinterpret_cast<float2 *>(ws + off);
  off = align_up(off + nbh * a.R * sizeof(float2), 256);
  a.score = score_out ? score_out : reinterpret_cast<float *>(ws + off);
  if (D == 128) return launch_probe_t<128>(a, (int)nbh, k_vert, window, idx_out, s);
  if (D == 64) return launch_probe_t<64>(a, (int)nbh, k_vert, window, idx_out, s);
  return cudaErrorInvalidValue;
}

}  // namespace hq
