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
// that KV head put on j.  Steps:
//   1. probe_tc ROWS pass (probe_tc.cu): S = Q K^T on the tensor cores, per
//      (row, CTA) partial max / sum of exp;
//   2. probe_row_stats: merges the partials into the row max m and 1 / Z;
//   3. probe_tc COLSUM pass: S^T = K Q^T, each key's sum of exp(s - m) / Z
//      over the G*P rows in a fixed order;
//   4. probe_topk: radix select of the k-th largest score in [0, L - W) with
//      (score desc, index asc) order, then an ordered compaction over
//      contiguous per-thread segments, so the list comes out ascending and
//      ties go to the lower index.
#include <float.h>

#include <algorithm>

#include "hq_internal.cuh"

namespace hq {
namespace {

constexpr int KTILE = 128;       // keys per probe tile (probe_tc.cu)

// Row max / 1/Z (or max / Z with invert = false) from the per-stage partials
// (log2 domain): one warp per row, lanes over the partials, merged in a fixed
// order.  A row that sees no key keeps max -FLT_MAX and Z = 0.
__global__ void probe_row_stats(const float2 *__restrict__ partial, float2 *__restrict__ stats,
                                int nrows, int nchunk, bool invert = true) {
  pdl_wait();                            // the partials come from the kernel before this one
  pdl_trigger();
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
constexpr int TK_BINS = 4096;     // radix digits of 12, 12 and 8 bits

// Staged key of candidate j: one pad word per 32, so that the per-thread
// segment walks below hit 32 different banks.
__device__ __forceinline__ int tk_slot(int j) { return j + (j >> 5); }

// Radix select of the k-th largest key, top digit first (12, 12, 8 bits),
// then an ordered compaction: keys above the threshold are taken, keys equal
// to it are taken lowest index first.  Histograms are plain shared-memory
// atomics; the bin holding the k-th key is found by a block-wide scan over
// the bins (each thread owns TK_BINS / TK_THREADS consecutive bins, taken
// from the top).
__global__ void __launch_bounds__(TK_THREADS)
probe_topk(const float *__restrict__ score, int L, int ncand, int k, int32_t *__restrict__ idx) {
  extern __shared__ uint32_t skey[];                 // staged keys (tk_slot layout)
  __shared__ int hist[TK_BINS];
  __shared__ int tmp[32];
  __shared__ uint32_t sel_prefix, sel_mask;
  __shared__ int remain;
  pdl_wait();                            // the scores come from the kernel before this one
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
  constexpr int PER = TK_BINS / TK_THREADS;          // bins per thread in the scan
  for (int d = 0; d < 3; ++d) {
    const int shift = d == 0 ? 20 : (d == 1 ? 8 : 0);
    const int nb = d == 2 ? 256 : TK_BINS;
    for (int t = threadIdx.x; t < TK_BINS; t += blockDim.x) hist[t] = 0;
    __syncthreads();
    const uint32_t pre = sel_prefix, msk = sel_mask;
    for (int j = threadIdx.x; j < ncand; j += blockDim.x) {
      const uint32_t key = key_of(j);
      if ((key & msk) == pre) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1);
    }
    __syncthreads();
    // thread t owns bins nb-1-PER*t .. nb-PER*(t+1) (top first)
    const int need = remain;
    int local = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int bin = nb - 1 - PER * (int)threadIdx.x - e;
      local += bin >= 0 ? hist[bin] : 0;
    }
    int before;
    block_exclusive_scan(local, tmp, before);
    if (before < need && need <= before + local) {
      int acc = before;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int bin = nb - 1 - PER * (int)threadIdx.x - e;
        const int c = bin >= 0 ? hist[bin] : 0;
        if (acc + c >= need) {
          remain = need - acc;                       // keys of this bin to take
          sel_prefix = pre | ((uint32_t)bin << shift);
          sel_mask = msk | ((uint32_t)(nb - 1) << shift);
          break;
        }
        acc += c;
      }
    }
    __syncthreads();
  }
  const uint32_t thr = sel_prefix;  // key of the k-th largest score
  const int take_eq = remain;       // equal keys to take, lowest indices first
  // Ordered compaction over contiguous per-warp segments, read 32 keys at a
  // time (coalesced): ballots rank the keys equal to the threshold (the
  // lowest take_eq indices are taken) and place every taken index; the
  // warps' counts are offset by a scan over the warps.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;              // lanes below this one
  const int seg = ((ncand + nwarp - 1) / nwarp + 31) / 32 * 32;
  const int jb = min(warp * seg, ncand), je = min(jb + seg, ncand);
  int n_eq = 0, n_gt = 0;
  for (int j0 = jb; j0 < je; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < je ? key_of(j) : 0u;
    n_eq += __popc(__ballot_sync(0xffffffffu, j < je && key == thr));
    n_gt += __popc(__ballot_sync(0xffffffffu, j < je && key > thr));
  }
  // exclusive prefix over the warps of a per-warp count
  auto warp_prefix = [&](int v) {
    if (lane == 0) tmp[warp] = v;
    __syncthreads();
    int before = 0;
    for (int w = lane; w < warp; w += 32) before += tmp[w];
    before = warp_sum(before);
    __syncthreads();
    return before;
  };
  const int eq_before = warp_prefix(n_eq);
  const int n_take = n_gt + max(0, min(take_eq - eq_before, n_eq));
  int pos = warp_prefix(n_take);
  int e = eq_before;
  for (int j0 = jb; j0 < je; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < je ? key_of(j) : 0u;
    const bool eq = j < je && key == thr;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = (j < je && key > thr) || (eq && e + __popc(eqm & lt) < take_eq);
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tm & lt)] = j;
    pos += __popc(tm);
    e += __popc(eqm);
  }
  pdl_trigger();
}

// Top-k of every (b, kv head) row of `score` (row stride L) over positions
// [0, ncand): k indices, ascending, ties to the lower index.
cudaError_t launch_topk(const float *score, int L, int ncand, int k, int nbh, int32_t *idx,
                        cudaStream_t s, bool pdl = false) {
  if (k <= 0 || nbh <= 0) return cudaSuccess;
  const size_t tk_smem = ncand <= TK_STAGE ? (size_t)(ncand + (ncand >> 5) + 1) * 4 : 0;
  static bool tk_attr = false;
  if (!tk_attr) {
    if (cudaFuncSetAttribute(probe_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (TK_STAGE + TK_STAGE / 32 + 1) * 4) != cudaSuccess)
      return cudaErrorInvalidValue;
    tk_attr = true;
  }
  if (pdl) return pdl_launch(probe_topk, dim3(nbh), dim3(TK_THREADS), tk_smem, s, score, L, ncand, k, idx);
  probe_topk<<<nbh, TK_THREADS, tk_smem, s>>>(score, L, ncand, k, idx);
  return cudaGetLastError();
}

// The probe's four kernels are chained by programmatic dependent launch when
// the tensor-core passes are short (at most 64 key tiles per CTA): each
// launch then overlaps the previous kernel's last CTAs, which saves ~6 us of
// a ~120 us probe of the 32K layer (15 tiles per CTA).  With long passes
// there is no launch gap worth hiding, and the chained launches were
// measured slower (batched 128K cache, 512 tiles per CTA: 1975 -> 2023 us;
// 70B-shaped: 7782 -> 7870 us), so those probes launch plainly.
bool probe_chain_pdl(int nbh, int Ls) {
  const int tiles = (Ls + KTILE - 1) / KTILE, nchunk = probe_tc_chunks(nbh, Ls);
  return (tiles + nchunk - 1) / nchunk <= 64;
}

// The probe of keys [key_off, key_off + Ls) of an L-key context whose probe
// rows sit at positions L - P + p: row statistics (max, 1/Z, or max, Z with
// invert = false) into `stats`, and with colsum the keys' scores.
cudaError_t probe_passes(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                         const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls, int D,
                         int key_off, int L, float scale, float2 *partial, float2 *stats,
                         bool invert, float *score, uint32_t *status, cudaStream_t s) {
  const int nbh = B * Hkv, R = (Hq / Hkv) * P;
  const int nchunk = probe_tc_chunks(nbh, Ls);
  const int qpos0 = L - P - key_off;
  const bool pdl = probe_chain_pdl(nbh, Ls);
  cudaError_t e = launch_probe_pass(false, q_probe, q_head_stride, k, B, Hq, Hkv, P, Ls, D, qpos0,
                                    scale, partial, nchunk, nullptr, nullptr, status, s, pdl);
  if (e != cudaSuccess) return e;
  const int nrows = nbh * R;
  const dim3 rs_grid((nrows + 7) / 8), rs_block(256);                 // a warp per row
  if (pdl) {
    e = pdl_launch(probe_row_stats, rs_grid, rs_block, 0, s, (const float2 *)partial, stats, nrows, nchunk,
                   invert);
  } else {
    probe_row_stats<<<rs_grid, rs_block, 0, s>>>(partial, stats, nrows, nchunk, invert);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess || !score) return e;
  return launch_probe_pass(true, q_probe, q_head_stride, k, B, Hq, Hkv, P, Ls, D, qpos0, scale,
                           nullptr, nchunk, stats, score, status, s, pdl);
}

}  // namespace

size_t probe_ws_bytes(int B, int Hq, int Hkv, int P, int L, int D) {
  (void)D;
  const size_t nbh = (size_t)B * Hkv, R = (size_t)(Hq / Hkv) * P;
  const size_t nchunk = (L + KTILE - 1) / KTILE;  // partials per row: at most one per 128-key tile
  size_t off = kWsHeader;
  off = align_up(off + nbh * R * nchunk * sizeof(float2), 256);  // partials
  off = align_up(off + nbh * R * sizeof(float2), 256);           // stats
  off = align_up(off + nbh * (size_t)L * sizeof(float), 256);    // scores
  return off;
}

namespace {
struct ProbeWs {
  float2 *partial, *stats;
  float *score;
};
ProbeWs probe_ws(uint8_t *ws, int B, int Hq, int Hkv, int P, int L) {
  const size_t nbh = (size_t)B * Hkv, R = (size_t)(Hq / Hkv) * P;
  const size_t nchunk = (L + KTILE - 1) / KTILE;
  ProbeWs w;
  size_t off = kWsHeader;
  w.partial = reinterpret_cast<float2 *>(ws + off);
  off = align_up(off + nbh * R * nchunk * sizeof(float2), 256);
  w.stats = reinterpret_cast<float2 *>(ws + off);
  off = align_up(off + nbh * R * sizeof(float2), 256);
  w.score = reinterpret_cast<float *>(ws + off);
  return w;
}
}  // namespace

cudaError_t launch_probe(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                         const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int L, int D,
                         int window, int k_vert, float scale, int32_t *idx_out, float *score_out,
                         uint8_t *ws, cudaStream_t s) {
  const ProbeWs w = probe_ws(ws, B, Hq, Hkv, P, L);
  float *score = score_out ? score_out : w.score;
  cudaError_t e = probe_passes(q_probe, q_head_stride, k, B, Hq, Hkv, P, L, D, 0, L, scale,
                               w.partial, w.stats, true, score, reinterpret_cast<uint32_t *>(ws), s);
  if (e != cudaSuccess) return e;
  return launch_topk(score, L, L - window, k_vert, B * Hkv, idx_out, s, probe_chain_pdl(B * Hkv, L));
}

// ---------------------------------------------------------------------------
// Context split: the keys [key_off, key_off + Ls) of an L-key context on one
// rank; the probe rows sit at context positions L - P + p.
// ---------------------------------------------------------------------------
size_t probe_shard_ws_bytes(int B, int Hq, int Hkv, int P, int Ls, int D, int k_vert) {
  return align_up(probe_ws_bytes(B, Hq, Hkv, P, Ls, D) + (size_t)B * Hkv * k_vert * sizeof(int32_t), 256);
}

cudaError_t launch_probe_shard_stats(const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                                     const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls,
                                     int D, int key_off, int L, float scale, float2 *stats_out,
                                     uint8_t *ws, cudaStream_t s) {
  const ProbeWs w = probe_ws(ws, B, Hq, Hkv, P, Ls);
  return probe_passes(q_probe, q_head_stride, k, B, Hq, Hkv, P, Ls, D, key_off, L, scale,
                      w.partial, stats_out, false, nullptr, reinterpret_cast<uint32_t *>(ws), s);
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
  const ProbeWs w = probe_ws(ws, B, Hq, Hkv, P, Ls);
  const int nbh = B * Hkv;
  int32_t *local_idx = reinterpret_cast<int32_t *>(ws + probe_ws_bytes(B, Hq, Hkv, P, Ls, D));
  // scores of this rank's keys with the whole context's (max, 1/Z)
  const int nchunk = probe_tc_chunks(nbh, Ls);
  cudaError_t e = launch_probe_pass(true, q_probe, q_head_stride, k, B, Hq, Hkv, P, Ls, D,
                                    L - P - key_off, scale, nullptr, nchunk, stats, w.score,
                                    reinterpret_cast<uint32_t *>(ws), s);
  if (e != cudaSuccess) return e;
  // candidates of this rank: its keys before the context's window
  const int ncand = std::max(0, std::min(Ls, L - window - key_off));
  const int kk = std::min(k_vert, ncand);
  e = launch_topk(w.score, Ls, ncand, kk, nbh, local_idx, s);
  if (e != cudaSuccess) return e;
  if (k_vert > 0)
    probe_shard_candidates<<<dim3((k_vert + 255) / 256, nbh), 256, 0, s>>>(
        local_idx, kk, k_vert, w.score, Ls, key_off, cand_idx, cand_score);
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
