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
//   1. probe_qk<STATS>: per (key chunk of 256, KV head) CTA, S = Q K^T on
//      tensor cores (bf16 mma.sync, fp32 accumulate) for all G*P rows; each
//      warp keeps one 16-row tile's Q fragments while the chunk's two
//      128-key halves stream through a double-buffered shared-memory ring
//      (cp.async); writes per-(row, chunk) partial max / sum-of-exp.
//   2. probe_row_stats: merges the partials into the row max m and sum Z.
//   3. probe_qk<COLSUM>: recomputes S, p = exp(s - m) / Z, and sums each
//      column over the G*P rows in a fixed order.
//   4. probe_topk: radix select of the k-th largest score in [0, L - W) with
//      (score desc, index asc) order (keys staged in shared memory), then an
//      ordered compaction over contiguous per-thread segments, so the list
//      comes out ascending and ties go to the lower index.
#include <float.h>

#include <algorithm>

#include "hq_internal.cuh"
#include "warp_mma.cuh"

namespace hq {
namespace {

constexpr int KSUB = 128;        // keys per shared-memory stage
constexpr int NSUB = 2;          // stages per CTA
constexpr int KC = KSUB * NSUB;  // keys per CTA
constexpr int PWARPS = 16;       // one 16-row tile of the probe rows per warp (more rows: loop)
constexpr float kLog2e = 1.4426950408889634f;

struct ProbeArgs {
  const __nv_bfloat16 *qp;
  int64_t q_head_stride;
  const __nv_bfloat16 *k;
  int Hq, Hkv, P, L, G, R, nchunk;
  int qpos0;                     // position of probe row 0 counted from key 0 (L - P unsplit)
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  // 16-byte global -> shared copy; an invalid source reads as zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

template <int D>
constexpr int probe_smem_bytes() {
  return 2 * KSUB * D * 2 + PWARPS * KSUB * 4;   // K ring + per-warp column sums
}

template <int D, bool COLSUM>
__global__ void __launch_bounds__(PWARPS * 32, 1) probe_qk(ProbeArgs a) {
  constexpr int CH = D / 8;                    // 16-byte chunks per key row
  extern __shared__ __align__(128) uint8_t psm[];
  uint4 *ring = reinterpret_cast<uint4 *>(psm);                         // [2][KSUB * CH], XOR-swizzled by key
  float *colacc = reinterpret_cast<float *>(psm + 2 * KSUB * D * 2);    // [PWARPS][KSUB]
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.Hkv, kh = bh % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
  const uint4 *kg = reinterpret_cast<const uint4 *>(a.k + ((size_t)bh * a.L) * D);
  auto load_sub = [&](int sub) {
    uint4 *dst = ring + (sub & 1) * KSUB * CH;
    const int jb = chunk * KC + sub * KSUB;
    for (int t = threadIdx.x; t < KSUB * CH; t += blockDim.x) {
      const int key = t / CH, ch = t % CH;
      const bool valid = jb + key < a.L;
      cp_async16(smem_u32(&dst[key * CH + (ch ^ (key & 7))]), kg + (size_t)(valid ? jb + key : 0) * CH + ch, valid);
    }
    cp_async_commit();
  };
  load_sub(0);
  if (NSUB > 1) load_sub(1);

  const int ntile_rows = (a.R + 15) / 16;
  // With at most PWARPS row tiles, each warp's tile fragments load once and
  // stay in registers; with more, every tile reloads them per stage.
  const bool resident = ntile_rows <= PWARPS;
  uint32_t qa[D / 16][4];
  if (resident && warp < ntile_rows) load_q_frag<D>(a, b, kh, warp * 16, qa);

  for (int sub = 0; sub < NSUB; ++sub) {
    if (sub + 1 < NSUB) cp_async_wait<1>();
    else cp_async_wait<0>();
    __syncthreads();
    const uint4 *ks = ring + (sub & 1) * KSUB * CH;
    const int j0 = chunk * KC + sub * KSUB;
    if (COLSUM)
      for (int t = lane; t < KSUB; t += 32) colacc[warp * KSUB + t] = 0.f;
    for (int rt = warp; rt < ntile_rows; rt += PWARPS) {
      if (!resident) load_q_frag<D>(a, b, kh, rt * 16, qa);
      const uint32_t(&q)[D / 16][4] = qa;
      // Rows of this thread: rt*16 + r (+8).  Visible keys: j <= qpos0 + p,
      // and j < L (the zero-filled keys past the end never count, which
      // matters when the probe rows lie beyond this key range).
      int lastj[2];
      bool valid[2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = rt * 16 + r + hf * 8;
        valid[hf] = row < a.R;
        lastj[hf] = valid[hf] ? min(a.qpos0 + (row % a.P), a.L - 1) : -1;
      }
      float2 sx[2];                              // COLSUM: (max, 1/Z) of the two rows
      if (COLSUM)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int row = rt * 16 + r + hf * 8;
          sx[hf] = valid[hf] ? a.stats[(size_t)bh * a.R + row] : make_float2(0.f, 0.f);
        }
      float pm[2] = {-FLT_MAX, -FLT_MAX}, ps[2] = {0.f, 0.f};   // STATS over the stage
      // the stage's keys in two halves of 64 (32 accumulators at a time)
#pragma unroll
      for (int kh2 = 0; kh2 < 2; ++kh2) {
        constexpr int NT = KSUB / 16;            // 8-key MMA tiles per half
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int kp = 0; kp < D / 32; ++kp) {
            const int key = kh2 * 64 + nt * 8 + (lane & 7);
            const int ch = kp * 4 + (lane >> 3);
            uint32_t bf[4];
            ldsm_x4(bf, smem_u32(&ks[key * CH + (ch ^ (key & 7))]));
            mma_bf16_16816(acc[nt], q[2 * kp], bf[0], bf[1]);
            mma_bf16_16816(acc[nt], q[2 * kp + 1], bf[2], bf[3]);
          }
        }
        const int jh = j0 + kh2 * 64;
        if (!COLSUM) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            float m = -FLT_MAX;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int j = jh + nt * 8 + 2 * c + e;
                if (j <= lastj[hf]) m = fmaxf(m, acc[nt][2 * hf + e] * a.scale_log2);
              }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int j = jh + nt * 8 + 2 * c + e;
                if (j <= lastj[hf]) sum += exp2f(acc[nt][2 * hf + e] * a.scale_log2 - m);
              }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            // merge with the stage's first half
            const float mn = fmaxf(pm[hf], m);
            ps[hf] = (pm[hf] == -FLT_MAX ? 0.f : ps[hf] * exp2f(pm[hf] - mn)) +
                     (m == -FLT_MAX ? 0.f : sum * exp2f(m - mn));
            pm[hf] = mn;
          }
        } else {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = jh + nt * 8 + 2 * c + e;
              float col = 0.f;
#pragma unroll
              for (int hf = 0; hf < 2; ++hf)
                if (j <= lastj[hf]) col += exp2f(acc[nt][2 * hf + e] * a.scale_log2 - sx[hf].x) * sx[hf].y;
              col += __shfl_xor_sync(0xffffffffu, col, 4);
              col += __shfl_xor_sync(0xffffffffu, col, 8);
              col += __shfl_xor_sync(0xffffffffu, col, 16);
              if (r == 0) colacc[warp * KSUB + kh2 * 64 + nt * 8 + 2 * c + e] += col;
            }
          }
        }
      }
      if (!COLSUM)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          if (c == 0 && valid[hf] && j0 < a.L) {   // one partial per (row, 128-key stage)
            const int row = rt * 16 + r + hf * 8;
            a.partial[((size_t)bh * a.R + row) * a.nchunk + chunk * NSUB + sub] = make_float2(pm[hf], ps[hf]);
          }
    }
    __syncthreads();   // every warp is done with this stage's keys (and column sums)
    if (COLSUM)
      for (int t = threadIdx.x; t < KSUB; t += blockDim.x) {
        float sm = 0.f;
#pragma unroll
        for (int w = 0; w < PWARPS; ++w) sm += colacc[w * KSUB + t];
        if (j0 + t < a.L) a.score[(size_t)bh * a.L + j0 + t] = sm;
      }
    if (sub + 2 < NSUB) load_sub(sub + 2);
    if (COLSUM) __syncthreads();    // column sums read before the next stage clears them
  }
}

// Row max / 1/Z (or max / Z with invert = false) from the per-stage partials
// (log2 domain): one warp per row, lanes over the partials, merged in a fixed
// order.  A row that sees no key keeps max -FLT_MAX and Z = 0.
__global__ void probe_row_stats(const float2 *__restrict__ partial, float2 *__restrict__ stats,
                                int nrows, int nchunk, bool invert = true) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;
  const float2 *pr = partial + (size_t)row * nchunk;
  float m = -FLT_MAX;
  for (int c = lane; c < nchunk; c += 32) m = fmaxf(m, pr[c].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
  for (int c = lane; c < nchunk; c += 32) z += pr[c].y * exp2f(pr[c].x - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane == 0) stats[row] = make_float2(m, invert ? 1.0f / z : z);
}

// Context split: merge the ranks' (max, Z) of every probe row into the
// row's (max, 1/Z) over the whole context, ranks in a fixed order.
__global__ void probe_merge_stats(const float2 *__restrict__ parts, int R, int nrows,
                                  float2 *__restrict__ stats) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= nrows) return;
  float m = -FLT_MAX;
  for (int r = 0; r < R; ++r) m = fmaxf(m, parts[(size_t)r * nrows + row].x);
  float z = 0.f;
  for (int r = 0; r < R; ++r) {
    const float2 p = parts[(size_t)r * nrows + row];
    if (p.y > 0.f) z += p.y * exp2f(p.x - m);
  }
  stats[row] = make_float2(m, 1.0f / z);
}

// Context split: a rank's top-k (local positions, ascending) as candidates in
// context positions with their scores; slots past the rank's count hold -1.
__global__ void probe_shard_candidates(const int32_t *__restrict__ local_idx, int kk, int k_vert,
                                       const float *__restrict__ score, int Ls, int key_off,
                                       int32_t *__restrict__ cand_idx, float *__restrict__ cand_score) {
  const int bh = blockIdx.y, t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= k_vert) return;
  const size_t o = (size_t)bh * k_vert + t;
  if (t < kk) {
    const int j = local_idx[(size_t)bh * kk + t];
    cand_idx[o] = j + key_off;
    cand_score[o] = score[(size_t)bh * Ls + j];
  } else {
    cand_idx[o] = -1;
    cand_score[o] = -FLT_MAX;
  }
}

// Context split: every rank's candidates into one dense score row per
// (b, kv head) over the context's candidate positions (the rest -inf).
__global__ void probe_fill(float *__restrict__ x, size_t n, float v) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    x[i] = v;
}
__global__ void probe_scatter_candidates(const int32_t *__restrict__ cand_idx,
                                         const float *__restrict__ cand_score, int R, int nbh,
                                         int k_vert, int ncand, float *__restrict__ dense,
                                         uint32_t *status) {
  const size_t n = (size_t)R * nbh * k_vert;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int bh = (int)((i / k_vert) % nbh);
    const int j = cand_idx[i];
    if (j < 0) continue;
    if (j >= ncand) {                     // not a candidate position: a caller error
      if (status) atomicOr(status, HQ_DEV_BAD_INDEX);
      continue;
    }
    dense[(size_t)bh * ncand + j] = cand_score[i];
  }
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

constexpr int TK_STAGE = 32768;   // candidates staged in shared memory (more: read from L2)

// Staged key of candidate j: one pad word per 32, so that the per-thread
// segment walks below hit 32 different banks.
__device__ __forceinline__ int tk_slot(int j) { return j + (j >> 5); }

__global__ void __launch_bounds__(TK_THREADS)
probe_topk(const float *__restrict__ score, int L, int ncand, int k, int32_t *__restrict__ idx) {
  extern __shared__ uint32_t skey[];                 // staged keys (tk_slot layout)
  __shared__ int hist[256];
  __shared__ int tmp[32];
  __shared__ uint32_t sel_prefix, sel_mask;
  __shared__ int remain;
  const int bh = blockIdx.x;
  const float *s = score + (size_t)bh * L;
  int32_t *out = idx + (size_t)bh * k;
  if (k == 0) return;
  const bool staged = ncand <= TK_STAGE;
  auto key_of = [&](int j) -> uint32_t { return staged ? skey[tk_slot(j)] : score_key(__ldg(s + j)); };
  if (staged) {
    // eight loads in flight per thread (a lone CTA per pair: latency-bound)
    for (int j0 = threadIdx.x; j0 < ncand; j0 += 8 * blockDim.x) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * blockDim.x;
        v[u] = j < ncand ? __ldg(s + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * blockDim.x;
        if (j < ncand) skey[tk_slot(j)] = score_key(v[u]);
      }
    }
  }
  if (threadIdx.x == 0) {
    sel_prefix = 0;
    sel_mask = 0;
    remain = k;
  }
  // Radix select of the k-th largest key, 8 bits at a time from the top; the
  // histogram atomics are aggregated per warp over lanes with the same bin.
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0;
    __syncthreads();
    const uint32_t pre = sel_prefix, msk = sel_mask;
    const int jend = (ncand + blockDim.x - 1) / blockDim.x * blockDim.x;   // whole warps iterate
    for (int j = threadIdx.x; j < jend; j += blockDim.x) {
      const uint32_t key = j < ncand ? key_of(j) : 0u;
      const bool in = j < ncand && (key & msk) == pre;
      const int bin = in ? (int)((key >> shift) & 0xff) : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
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
  // Ordered compaction over contiguous per-thread segments: the keys equal to
  // the threshold that come before a segment decide how many of its equal
  // keys are taken; a second scan places every taken index.
  const int seg = (ncand + blockDim.x - 1) / blockDim.x;
  const int jb = min((int)threadIdx.x * seg, ncand), je = min(jb + seg, ncand);
  int n_eq = 0;
  for (int j = jb; j < je; ++j) n_eq += key_of(j) == thr;
  int eq_before;
  block_exclusive_scan(n_eq, tmp, eq_before);
  int n_take = 0;
  {
    int e = eq_before;
    for (int j = jb; j < je; ++j) {
      const uint32_t key = key_of(j);
      if (key > thr) ++n_take;
      else if (key == thr) n_take += (e++ < take_eq);
    }
  }
  int pos;
  block_exclusive_scan(n_take, tmp, pos);
  {
    int e = eq_before;
    for (int j = jb; j < je; ++j) {
      const uint32_t key = key_of(j);
      const bool take = key > thr || (key == thr && e++ < take_eq);
      if (take) out[pos++] = j;
    }
  }
}

// Top-k of every (b, kv head) row of `score` (row stride L) over positions
// [0, ncand): k indices, ascending, ties to the lower index.
cudaError_t launch_topk(const float *score, int L, int ncand, int k, int nbh, int32_t *idx,
                        cudaStream_t s) {
  if (k <= 0 || nbh <= 0) return cudaSuccess;
  const size_t tk_smem = ncand <= TK_STAGE ? (size_t)(ncand + (ncand >> 5) + 1) * 4 : 0;
  static bool tk_attr = false;
  if (!tk_attr) {
    if (cudaFuncSetAttribute(probe_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (TK_STAGE + TK_STAGE / 32 + 1) * 4) != cudaSuccess)
      return cudaErrorInvalidValue;
    tk_attr = true;
  }
  probe_topk<<<nbh, TK_THREADS, tk_smem, s>>>(score, L, ncand, k, idx);
  return cudaGetLastError();
}

template <int D>
cudaError_t probe_attr() {
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(probe_qk<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, probe_smem_bytes<D>()) != cudaSuccess ||
        cudaFuncSetAttribute(probe_qk<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, probe_smem_bytes<D>()) != cudaSuccess)
      return cudaErrorInvalidValue;
    attr = true;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_probe_t(ProbeArgs a, int nbh, int k_vert, int window, int32_t *idx,
                           cudaStream_t s) {
  if (probe_attr<D>() != cudaSuccess) return cudaErrorInvalidValue;
  dim3 grid((a.L + KC - 1) / KC, nbh);
  probe_qk<D, false><<<grid, PWARPS * 32, probe_smem_bytes<D>(), s>>>(a);
  const int nrows = nbh * a.R;
  probe_row_stats<<<(nrows + 7) / 8, 256, 0, s>>>(a.partial, const_cast<float2 *>(a.stats),   // a warp per row
                                                      nrows, a.nchunk);
  probe_qk<D, true><<<grid, PWARPS * 32, probe_smem_bytes<D>(), s>>>(a);
  return launch_topk(a.score, a.L, a.L - window, k_vert, nbh, idx, s);
}

}  // namespace

size_t probe_ws_bytes(int B, int Hq, int Hkv, int P, int L, int D) {
  (void)D;
  const size_t nbh = (size_t)B * Hkv, R = (size_t)(Hq / Hkv) * P;
  const size_t nchunk = (L + KSUB - 1) / KSUB;    // partials per row: one per 128-key stage
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
  a.qpos0 = L - P;
  a.G = Hq / Hkv;
  a.R = a.G * P;
  a.nchunk = (L + KSUB - 1) / KSUB;
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

// ---------------------------------------------------------------------------
// Context split: the keys [key_off, key_off + Ls) of an L-key context on one
// rank; the probe rows sit at context positions L - P + p.
// ---------------------------------------------------------------------------
size_t probe_shard_ws_bytes(int B, int Hq, int Hkv, int P, int Ls, int D, int k_vert) {
  return align_up(probe_ws_bytes(B, Hq, Hkv, P, Ls, D) + (size_t)B * Hkv * k_vert * sizeof(int32_t), 256);
}

namespace {
ProbeArgs shard_args(const __nv_bfloat16 *q_probe, int64_t q_head_stride, const __nv_bfloat16 *k,
                     int B, int Hq, int Hkv, int P, int Ls, int key_off, int L, float scale,
                     uint8_t *ws) {
  ProbeArgs a;
  a.qp = q_probe;
  a.q_head_stride = q_head_stride;
  a.k = k;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.P = P;
  a.L = Ls;
  a.qpos0 = L - P - key_off;
  a.G = Hq / Hkv;
  a.R = a.G * P;
  a.nchunk = (Ls + KSUB - 1) / KSUB;
  a.scale_log2 = scale * kLog2e;
  const size_t nbh = (size_t)B * Hkv;
  size_t off = kWsHeader;
  a.partial = reinterpret_cast<float2 *>(ws + off);
  off = align_up(off + nbh * a.R * a.nchunk * sizeof(float2), 256);
  a.stats = reinterpret_cast<float2 *>(ws + off);
  off = align_up(off + nbh * a.R * sizeof(float2), 256);
  a.score = reinterpret_cast<float *>(ws + off);
  return a;
}
}  // namespace

cudaError_t launch_probe_shard_stats(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                                     const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls,
                                     int D, int key_off, int L, float scale, float2 *stats_out,
                                     uint8_t *ws, cudaStream_t s) {
  ProbeArgs a = shard_args(q_probe, q_head_stride, k, B, Hq, Hkv, P, Ls, key_off, L, scale, ws);
  const int nbh = B * Hkv, nrows = nbh * a.R;
  dim3 grid((Ls + KC - 1) / KC, nbh);
  if (D == 128) {
    if (probe_attr<128>() != cudaSuccess) return cudaErrorInvalidValue;
    probe_qk<128, false><<<grid, PWARPS * 32, probe_smem_bytes<128>(), s>>>(a);
  } else if (D == 64) {
    if (probe_attr<64>() != cudaSuccess) return cudaErrorInvalidValue;
    probe_qk<64, false><<<grid, PWARPS * 32, probe_smem_bytes<64>(), s>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  probe_row_stats<<<(nrows + 7) / 8, 256, 0, s>>>(a.partial, stats_out, nrows, a.nchunk, false);
  return cudaGetLastError();
}

cudaError_t launch_probe_merge_stats(const float2 *parts, int R, int nrows, float2 *stats,
                                     cudaStream_t s) {
  probe_merge_stats<<<(nrows + 255) / 256, 256, 0, s>>>(parts, R, nrows, stats);
  return cudaGetLastError();
}

cudaError_t launch_probe_shard_topk(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                                    const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls,
                                    int D, int key_off, int L, int window, int k_vert, float scale,
                                    const float2 *stats, int32_t *cand_idx, float *cand_score,
                                    uint8_t *ws, cudaStream_t s) {
  ProbeArgs a = shard_args(q_probe, q_head_stride, k, B, Hq, Hkv, P, Ls, key_off, L, scale, ws);
  a.stats = stats;                                   // the whole context's (max, 1/Z)
  const int nbh = B * Hkv;
  int32_t *local_idx = reinterpret_cast<int32_t *>(ws + probe_ws_bytes(B, Hq, Hkv, P, Ls, D));
  dim3 grid((Ls + KC - 1) / KC, nbh);
  if (D == 128) {
    if (probe_attr<128>() != cudaSuccess) return cudaErrorInvalidValue;
    probe_qk<128, true><<<grid, PWARPS * 32, probe_smem_bytes<128>(), s>>>(a);
  } else if (D == 64) {
    if (probe_attr<64>() != cudaSuccess) return cudaErrorInvalidValue;
    probe_qk<64, true><<<grid, PWARPS * 32, probe_smem_bytes<64>(), s>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  // candidates of this rank: its keys before the context's window
  const int ncand = std::max(0, std::min(Ls, L - window - key_off));
  const int kk = std::min(k_vert, ncand);
  cudaError_t e = launch_topk(a.score, Ls, ncand, kk, nbh, local_idx, s);
  if (e != cudaSuccess) return e;
  if (k_vert > 0)
    probe_shard_candidates<<<dim3((k_vert + 255) / 256, nbh), 256, 0, s>>>(
        local_idx, kk, k_vert, a.score, Ls, key_off, cand_idx, cand_score);
  return cudaGetLastError();
}

size_t probe_merge_ws_bytes(int B, int Hkv, int L, int window) {
  return align_up(kWsHeader + (size_t)B * Hkv * (size_t)std::max(0, L - window) * sizeof(float), 256);
}

cudaError_t launch_probe_merge_topk(const int32_t *cand_idx, const float *cand_score, int R, int B,
                                    int Hkv, int L, int window, int k_vert, int32_t *idx_out,
                                    uint8_t *ws, uint32_t *status, cudaStream_t s) {
  const int nbh = B * Hkv, ncand = L - window;
  if (k_vert <= 0 || ncand <= 0) return cudaSuccess;
  float *dense = reinterpret_cast<float *>(ws + kWsHeader);
  probe_fill<<<592, 256, 0, s>>>(dense, (size_t)nbh * ncand, -FLT_MAX);
  probe_scatter_candidates<<<148, 256, 0, s>>>(cand_idx, cand_score, R, nbh, k_vert, ncand, dense,
                                               status);
  return launch_topk(dense, ncand, ncand, k_vert, nbh, idx_out, s);
}

}  // namespace hq
