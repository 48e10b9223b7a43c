// probe_tc.cu -- the vertical-line probe's two passes over the keys on the
// 5th-generation tensor cores (tcgen05, scores in tensor memory).
//
// Method: "HyQuant: Hybrid-Precision Quantization for LLM Attention" (wiki
// summary), TL;DR and "What problem it solves": vertical-line tokens are the
// key columns that nearly every query row attends to; the signal of key j is
// the sum, over the P most recent queries of the G query heads of its KV head,
// of their exact causal softmax weights on j ("How HyQuant uses
// hybrid-precision attention to cut decode compute", "Why preserve selected
// positions?").  The softmax weight needs each row's max and sum over ALL its
// keys, so the probe reads the keys twice:
//
//   pass 1 (ROWS):   S = Q K^T, rows = probe rows (M = 128 per block), keys the
//                    N dimension; one thread per row keeps the running max and
//                    sum of exp over the CTA's keys and writes them as a
//                    partial (merged over the CTAs by probe_row_stats);
//   pass 2 (COLSUM): S^T = K Q^T, keys = the M dimension (128 per tile), probe
//                    rows the N dimension (up to 256 per MMA); one thread per
//                    key sums exp(s - m_r) / Z_r over the rows in a fixed order
//                    and writes the key's score.
//
// Both layouts put the reduction of each pass inside one thread (a TMEM lane),
// so neither needs a cross-thread reduction per score.  One CTA per (chunk of
// 128-key tiles, KV head of a batch element).  Warp roles: warp 0 issues the
// TMA copies (the G heads' probe rows once, then a ring of K tiles), warp 1
// owns the tensor memory (512 columns) and issues the MMAs, warps 4-11 (two
// warpgroups) read the scores from tensor memory; S is double-buffered so the
// MMA of the next sub-tile overlaps the exps of this one.  The probe rows of
// head g sit at rows g * Ppad .. g * Ppad + P - 1 (Ppad = P rounded up to 8),
// rows that hold no probe query are zero.
#include <cuda.h>
#include <float.h>

#include "hq_internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace hq {
namespace {

constexpr int KT = 128;                  // keys per K tile (one ring stage)
constexpr int NTHR = 384;                // 12 warps
constexpr int EPI0 = 4;                  // first epilogue warp; warps 4..11
constexpr int NEPI = 8 * 32;             // epilogue threads
constexpr int kMaxStages = 8;

struct PtArgs {
  const float2 *stats;     // COLSUM: [nbh, R] (max, 1/Z), log2 domain
  float2 *partial;         // ROWS:   [nbh, R, nchunk] (max, sum), log2 domain
  float *score;            // COLSUM: [nbh, Ls]
  uint32_t *status;
  int Hq, Hkv, G, P, Ppad, R, Rpad, R2, Ls, qpos0, tiles, tpc, nchunk, nst;
  float sl;                // softmax scale * log2(e)
};

// Byte offsets of the shared-memory regions (1024-aligned base).
struct PtSmem {
  uint32_t ring, rp, lim, colbuf, bar, total;
};
__host__ __device__ inline PtSmem pt_smem(int D, int Rpad, int nst) {
  PtSmem s;
  s.ring = (uint32_t)(D / 64) * Rpad * 128;               // Q: D/64 boxes of Rpad rows x 128 B
  s.rp = s.ring + (uint32_t)nst * KT * D * 2;             // after the ring of nst tiles of 128 keys
  s.lim = s.rp + Rpad * 8;                                // rp: per-row -max then per-row 1/Z
                                                          // (COLSUM), or warpgroup 1's (max,
                                                          // sum) per row (ROWS)
  s.colbuf = s.lim + Rpad * 4;                            // lim: per-row last visible key
  s.bar = s.colbuf + 2 * KT * 4;                          // colbuf: [2][KT] column sums of warpgroup 1
  s.total = s.bar + 256;                                  // barriers, TMEM address, abort flag
  return s;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(NEPI) : "memory");
}

template <int D, bool COLSUM>
__global__ void __launch_bounds__(NTHR, 1)
probe_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
         PtArgs a) {
  constexpr int NKB = D / 64;                   // 128-byte boxes per row
  constexpr int KSTAGE = KT * D * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const PtSmem L = pt_smem(D, a.Rpad, a.nst);
  uint8_t *ring = smem + L.ring;
  float2 *rp = reinterpret_cast<float2 *>(smem + L.rp);      // ROWS: [Rpad] (max, sum)
  float *rcm = reinterpret_cast<float *>(smem + L.rp);        // COLSUM: [Rpad] -max
  float *rw = rcm + a.Rpad;                                   // COLSUM: [Rpad] 1/Z
  int *lim = reinterpret_cast<int *>(smem + L.lim);
  float *colbuf = reinterpret_cast<float *>(smem + L.colbuf);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bar);
  uint64_t *q_full = bar;
  uint64_t *kv_full = bar + 1;                  // [kMaxStages]
  uint64_t *kv_free = bar + 1 + kMaxStages;     // [kMaxStages]
  uint64_t *s_full = bar + 1 + 2 * kMaxStages;  // [4] S buffers (ROWS uses 2)
  uint64_t *s_free = s_full + 4;                // [4], one arrival per reading warp
  uint64_t *mma_done = s_free + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.Hkv, kh = bh % a.Hkv;
  const int t0 = chunk * a.tpc;
  const int nt = min(a.tpc, a.tiles - t0);      // >= 1 by construction of the grid
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MB = a.Rpad / 128;                  // row blocks (ROWS)
  const int TN1 = MB <= 2 ? 128 : 64;           // keys per ROWS sub-tile (2 buffers x MB x TN1 <= 512)
  const int SPS = KT / TN1;                     // ROWS sub-tiles per K tile
  const int NG = (a.R2 + 127) / 128;            // COLSUM row groups of up to 128 (the MMA's N)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_free[s], 1);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&s_full[s], 1);
      // ROWS: both warpgroups read every sub-tile; COLSUM: one warpgroup per buffer
      mbar_init(&s_free[s], COLSUM ? NEPI / 64 : NEPI / 32);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // Rows of the Q block that hold no probe query must be zero (they are
  // MMA columns of the COLSUM pass): clear the block before the copies land.
  if (a.P != a.Ppad || (a.G * a.Ppad) % 16 != 0) {
    for (uint32_t i = threadIdx.x; i < L.ring / 16; i += NTHR)
      reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  // Everything above touched only shared and tensor memory; q, k and the row
  // statistics may be written by the kernel before this one.
  pdl_wait();
  if (COLSUM) {
    for (int r = threadIdx.x; r < a.Rpad; r += NTHR) {
      const int g = r / a.Ppad, p = r % a.Ppad;
      float cm = 0.f, w = 0.f;
      int li = -1;
      if (g < a.G && p < a.P) {
        const float2 st = a.stats[(size_t)bh * a.R + g * a.P + p];
        if (st.x > -FLT_MAX && st.y < FLT_MAX) {
          cm = -st.x;
          w = st.y;
        }
        li = min(a.qpos0 + p, a.Ls - 1);
      }
      rcm[r] = cm;
      rw[r] = w;
      lim[r] = li;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(q_full, (uint32_t)(a.G * NKB * a.P * 128));
      for (int g = 0; g < a.G; ++g)
        for (int kb = 0; kb < NKB; ++kb)
          tma_load_3d(smem + kb * a.Rpad * 128 + g * a.Ppad * 128, &tm_q, q_full, kb * 64, 0,
                      b * a.Hq + kh * a.G + g);
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int s = i % a.nst;
        if (i >= a.nst && !mbar_wait(&kv_free[s], ((i / a.nst) & 1) ^ 1)) {
          *abort_flag = 1;
          raise_status(a.status, HQ_DEV_TIMEOUT);
          break;
        }
        if (*abort_flag) break;
        uint8_t *st = ring + s * KSTAGE;
        mbar_arrive_expect_tx(&kv_full[s], KSTAGE);
        for (int kb = 0; kb < NKB; ++kb)
          tma_load_3d(st + kb * KT * 128, &tm_k, &kv_full[s], kb * 64, (t0 + i) * KT, bh);
        issued = i + 1;
      }
      // never leave with copies in flight
      if (!mbar_wait(q_full, 0)) raise_status(a.status, HQ_DEV_TIMEOUT);
      for (int i = issued > a.nst ? issued - a.nst : 0; i < issued; ++i)
        if (!mbar_wait(&kv_full[i % a.nst], (i / a.nst) & 1)) raise_status(a.status, HQ_DEV_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    // ROWS: sub-tile u (TN1 keys of tile u / SPS) goes to S buffer u & 1; both
    // warpgroups read every sub-tile (half of its columns each).  COLSUM: tile
    // i is read by warpgroup i & 1 alone, one group of up to 128 probe rows
    // (128 TMEM columns) at a time, alternating between that warpgroup's two
    // buffers 2 (i & 1) and 2 (i & 1) + 1, so the MMA of its next group runs
    // while it reads this one.  Tiles are issued in pairs, group by group, so
    // that neither warpgroup waits for the other.
    if (lane == 0) {
      const uint32_t sQ = smem_u32(smem), sR = smem_u32(ring);
      bool ok = mbar_wait(q_full, 0);
      tc_fence_after();
      int use[4] = {0, 0, 0, 0};                   // sub-tiles issued into each buffer
      auto claim_buf = [&](int buf) -> bool {
        if (use[buf] >= 1 && !mbar_wait(&s_free[buf], (use[buf] & 1) ^ 1)) return false;
        ++use[buf];
        tc_fence_after();
        return true;
      };
      auto stage_ready = [&](int i) -> bool {
        if (!mbar_wait(&kv_full[i % a.nst], (i / a.nst) & 1)) return false;
        tc_fence_after();
        return true;
      };
      int nsub_wg[2] = {0, 0};                     // COLSUM sub-tiles issued for each warpgroup
      if (!COLSUM) {
        const uint32_t idesc = make_idesc(1, 1, 1, 0, 0, 128, TN1);
        for (int i = 0; ok && i < nt; ++i) {
          if (!(ok = stage_ready(i))) break;
          const uint32_t kst = sR + (i % a.nst) * KSTAGE;
          for (int v = 0; v < SPS; ++v) {
            const int buf = (i * SPS + v) & 1;
            if (!(ok = claim_buf(buf))) break;
            for (int mb = 0; mb < MB; ++mb) {
              const uint32_t dt = tmem + (buf * MB + mb) * TN1;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ko = (kk & 3) * 32;
                const uint64_t ad = make_sdesc_sw128(sQ + (kk >> 2) * a.Rpad * 128 + mb * 128 * 128 + ko, 16, 1024);
                const uint64_t bd = make_sdesc_sw128(kst + (kk >> 2) * KT * 128 + v * TN1 * 128 + ko, 16, 1024);
                mma_f16_ss(dt, ad, bd, idesc, kk > 0);
              }
            }
            tc_commit(&s_full[buf]);
          }
          if (!ok) break;
          tc_commit(&kv_free[i % a.nst]);          // the tile's MMAs have read the stage
        }
      } else {
        for (int i0 = 0; ok && i0 < nt; i0 += 2) {
          const int npair = min(2, nt - i0);
          for (int j = 0; ok && j < npair; ++j) ok = stage_ready(i0 + j);
          for (int v = 0; ok && v < NG; ++v) {
            const int ng = min(128, a.R2 - 128 * v);
            const uint32_t idesc = make_idesc(1, 1, 1, 0, 0, 128, ng);
            for (int j = 0; ok && j < npair; ++j) {
              const int i = i0 + j, wgi = i & 1;
              const int buf = 2 * wgi + (nsub_wg[wgi]++ & 1);
              if (!(ok = claim_buf(buf))) break;
              const uint32_t kst = sR + (i % a.nst) * KSTAGE;
              const uint32_t dt = tmem + buf * 128;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ko = (kk & 3) * 32;
                const uint64_t ad = make_sdesc_sw128(kst + (kk >> 2) * KT * 128 + ko, 16, 1024);
                const uint64_t bd = make_sdesc_sw128(sQ + (kk >> 2) * a.Rpad * 128 + v * 128 * 128 + ko, 16, 1024);
                mma_f16_ss(dt, ad, bd, idesc, kk > 0);
              }
              tc_commit(&s_full[buf]);
              if (v == NG - 1) tc_commit(&kv_free[i % a.nst]);
            }
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(a.status, HQ_DEV_TIMEOUT);
      }
      tc_commit(mma_done);
    }
    __syncwarp();
  } else if (warp >= EPI0) {
    // ------------------------------ epilogue ------------------------------
    const int wg = (warp - EPI0) >> 2;             // warpgroup
    const int q4 = warp & 3;                       // TMEM lane quarter of this warp
    const int lrow = q4 * 32 + lane;               // TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    bool ok = true;
    if (!COLSUM) {
      // One thread per probe row of each row block: running (max, sum) over
      // this warpgroup's half of every sub-tile's keys.
      float m[4], l[4];
      int lastj[4];
      bool warp_live = false;
#pragma unroll
      for (int mb = 0; mb < 4; ++mb) {
        m[mb] = -FLT_MAX;
        l[mb] = 0.f;
        lastj[mb] = -1;
        const int r = mb * 128 + lrow, g = r / a.Ppad, p = r % a.Ppad;
        if (mb < MB && g < a.G && p < a.P) lastj[mb] = min(a.qpos0 + p, a.Ls - 1);
        warp_live |= __any_sync(0xffffffffu, mb < MB && lastj[mb] >= 0);
      }
      const int HC = TN1 / 2;                      // columns per thread per row block
      const float2 sl2 = make_float2(a.sl, a.sl);
      int u = 0;
      for (int i = 0; ok && i < nt; ++i) {
        for (int v = 0; v < SPS; ++v, ++u) {
          const int buf = u & 1;
          if (!mbar_wait(&s_full[buf], (u >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int jb0 = (t0 + i) * KT + v * TN1 + wg * HC;
          if (warp_live) {
#pragma unroll
            for (int mb = 0; mb < 4; ++mb) {
              if (mb >= MB) break;
              for (int c32 = 0; c32 < HC; c32 += 32) {
                uint32_t xs[32];
                __syncwarp();
                tmem_ld32(tl + (buf * MB + mb) * TN1 + wg * HC + c32, xs);
                const int jb = jb0 + c32, lj = lastj[mb];
                const int nvis = min(32, lj - jb + 1);   // visible keys among these columns (<= 0: none)
                if (nvis == 32) {
                  // every key visible: the extreme raw score gives the max
                  float hi3[4], lo3[4];
#pragma unroll
                  for (int u4 = 0; u4 < 4; ++u4) {
                    hi3[u4] = lo3[u4] = __uint_as_float(xs[u4]);
                  }
#pragma unroll
                  for (int e = 4; e < 32; e += 8) {
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {
                      const float x0 = __uint_as_float(xs[e + u4]), x1 = __uint_as_float(xs[e + u4 + 4 < 32 ? e + u4 + 4 : e + u4]);
                      hi3[u4] = fmax3(hi3[u4], x0, x1);
                      lo3[u4] = fminf(lo3[u4], fminf(x0, x1));
                    }
                  }
                  const float hmax = fmax3(fmaxf(hi3[0], hi3[1]), hi3[2], hi3[3]);
                  const float lmin = fminf(fminf(lo3[0], lo3[1]), fminf(lo3[2], lo3[3]));
                  const float mx = a.sl >= 0.f ? hmax * a.sl : lmin * a.sl;
                  const float mn = fmaxf(m[mb], mx);
                  const float2 o2 = make_float2(-mn, -mn);
                  float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
                  for (int e = 0; e < 32; e += 4) {
                    const float2 y0 = ffma2(make_float2(__uint_as_float(xs[e]), __uint_as_float(xs[e + 1])), sl2, o2);
                    const float2 y1 = ffma2(make_float2(__uint_as_float(xs[e + 2]), __uint_as_float(xs[e + 3])), sl2, o2);
                    s0 = fadd2(s0, make_float2(fast_exp2(y0.x), fast_exp2(y0.y)));
                    s1 = fadd2(s1, make_float2(fast_exp2(y1.x), fast_exp2(y1.y)));
                  }
                  l[mb] = l[mb] * fast_exp2(m[mb] - mn) + ((s0.x + s0.y) + (s1.x + s1.y));
                  m[mb] = mn;
                } else if (nvis > 0) {
                  float mx = -INFINITY;
#pragma unroll
                  for (int e = 0; e < 32; ++e)
                    if (e < nvis) mx = fmaxf(mx, __uint_as_float(xs[e]) * a.sl);
                  const float mn = fmaxf(m[mb], mx);
                  float sm = 0.f;
#pragma unroll
                  for (int e = 0; e < 32; ++e) {
                    const float pe = fast_exp2(fmaf(__uint_as_float(xs[e]), a.sl, -mn));
                    sm += e < nvis ? pe : 0.f;
                  }
                  l[mb] = l[mb] * fast_exp2(m[mb] - mn) + sm;
                  m[mb] = mn;
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[buf]);
        }
      }
      // merge the two warpgroups' halves of each row (fixed order) and write
      // the CTA's partial
      float2 *half = rp;                           // [Rpad] (max, sum) of warpgroup 1
      if (wg == 1)
#pragma unroll
        for (int mb = 0; mb < 4; ++mb)
          if (mb < MB) half[mb * 128 + lrow] = make_float2(m[mb], l[mb]);
      epi_sync();
      if (wg == 0)
#pragma unroll
        for (int mb = 0; mb < 4; ++mb) {
          if (mb >= MB || lastj[mb] < 0) continue;
          const float2 o = half[mb * 128 + lrow];
          const float mm = fmaxf(m[mb], o.x);
          const float ll = (l[mb] > 0.f ? l[mb] * exp2f(m[mb] - mm) : 0.f) +
                           (o.y > 0.f ? o.y * exp2f(o.x - mm) : 0.f);
          const int r = mb * 128 + lrow, g = r / a.Ppad, p = r % a.Ppad;
          a.partial[((size_t)bh * a.R + g * a.P + p) * a.nchunk + chunk] = make_float2(mm, ll);
        }
    } else {
      // Warpgroup wg takes the CTA's tiles i = wg, wg + 2, ... whole: one
      // thread per key sums exp(s - m_r) / Z_r over every probe row, in a
      // fixed order, and writes the key's score.
      const float2 sl2 = make_float2(a.sl, a.sl);
      int uw = 0;                                  // groups read by this warpgroup so far
      for (int i = wg; ok && i < nt; i += 2) {
        const int jt = (t0 + i) * KT;
        const int j = jt + lrow;
        const bool nomask = jt + KT - 1 <= a.qpos0;  // every probe row sees every key of the tile
        float2 c0 = make_float2(0.f, 0.f), c1 = make_float2(0.f, 0.f);
        for (int v = 0; v < NG; ++v, ++uw) {
          const int buf = 2 * wg + (uw & 1);
          if (!mbar_wait(&s_full[buf], (uw >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int ng = min(128, a.R2 - 128 * v);   // a multiple of 16
          for (int cc = 0; cc < ng; cc += 32) {
            uint32_t xs[32];
            __syncwarp();
            tmem_ld32(tl + buf * 128 + cc, xs);
            const int r0 = 128 * v + cc;
            const float4 *cm4 = reinterpret_cast<const float4 *>(rcm + r0);
            const float4 *w4 = reinterpret_cast<const float4 *>(rw + r0);
            if (nomask && cc + 32 <= ng) {
#pragma unroll
              for (int e = 0; e < 32; e += 4) {
                const float4 cm = cm4[e >> 2], w = w4[e >> 2];
                const float2 y0 = ffma2(make_float2(__uint_as_float(xs[e]), __uint_as_float(xs[e + 1])), sl2,
                                        make_float2(cm.x, cm.y));
                const float2 y1 = ffma2(make_float2(__uint_as_float(xs[e + 2]), __uint_as_float(xs[e + 3])), sl2,
                                        make_float2(cm.z, cm.w));
                c0 = ffma2(make_float2(fast_exp2(y0.x), fast_exp2(y0.y)), make_float2(w.x, w.y), c0);
                c1 = ffma2(make_float2(fast_exp2(y1.x), fast_exp2(y1.y)), make_float2(w.z, w.w), c1);
              }
            } else {
              const int nvalid = ng - cc;            // columns past it are not rows of this group
              const int *lm = lim + r0;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                if (e < nvalid) {
                  float pe = fast_exp2(fmaf(__uint_as_float(xs[e]), a.sl, rcm[r0 + e]));
                  if (j > lm[e]) pe = 0.f;
                  if (e & 1) c1.x = fmaf(pe, rw[r0 + e], c1.x);
                  else c0.x = fmaf(pe, rw[r0 + e], c0.x);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[buf]);
        }
        if (ok && j < a.Ls) a.score[(size_t)bh * a.Ls + j] = (c0.x + c0.y) + (c1.x + c1.y);
      }
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(a.status, HQ_DEV_TIMEOUT);
    }
  }
  // The next kernel may be scheduled once every CTA is here: not earlier, or
  // its CTAs would take SMs from this grid's later waves.
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    // every MMA has completed once mma_done fired (bounded, in case of an abort)
    if (!mbar_wait(mma_done, 0)) raise_status(a.status, HQ_DEV_TIMEOUT);
    tmem_dealloc(tmem, 512);
  }
}

// 3-D map with explicit strides (bytes) over [outer][rows][inner] bf16.
bool make_map_bf16(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t outer,
                   uint64_t row_stride, uint64_t outer_stride, uint32_t box_rows) {
  memset(m, 0, sizeof *m);
  EncodeTiledFn fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {row_stride, outer_stride};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool COLSUM>
cudaError_t launch_t(const CUtensorMap &mq, const CUtensorMap &mk, const PtArgs &a, int nbh,
                     int nchunk, uint32_t smem, cudaStream_t s, bool pdl) {
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(probe_tc<D, COLSUM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess)
      return cudaErrorInvalidValue;
    attr = true;
  }
  if (pdl) return pdl_launch(probe_tc<D, COLSUM>, dim3(nchunk, nbh), dim3(NTHR), smem, s, mq, mk, a);
  probe_tc<D, COLSUM><<<dim3(nchunk, nbh), NTHR, smem, s>>>(mq, mk, a);
  return cudaGetLastError();
}

}  // namespace

// Chunks of 128-key tiles per (b, kv head): about one CTA per SM in all.
int probe_tc_chunks(int nbh, int Ls) {
  const int tiles = (Ls + KT - 1) / KT;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int c = (sms + nbh - 1) / nbh;
  if (nbh * c > sms && c > 1) c = sms / nbh > 0 ? sms / nbh : 1;
  c = c < 1 ? 1 : (c > tiles ? tiles : c);
  const int tpc = (tiles + c - 1) / c;
  return (tiles + tpc - 1) / tpc;                 // no empty chunk
}

bool probe_tc_supported(int D, int G, int P) { return (D == 64 || D == 128) && G >= 1 && G <= 8 && P >= 1 && P <= 64; }

cudaError_t launch_probe_pass(bool colsum, const __nv_bfloat16 *q_probe, int64_t q_head_stride,
                              const __nv_bfloat16 *k, int B, int Hq, int Hkv, int P, int Ls, int D,
                              int qpos0, float scale, float2 *partial, int nchunk,
                              const float2 *stats, float *score, uint32_t *status, cudaStream_t s,
                              bool pdl) {
  if (!probe_tc_supported(D, Hq / Hkv, P)) return cudaErrorNotSupported;
  PtArgs a;
  a.stats = stats;
  a.partial = partial;
  a.score = score;
  a.status = status;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.P = P;
  a.Ppad = (P + 7) / 8 * 8;
  a.R = a.G * P;
  const int rows = a.G * a.Ppad;
  a.Rpad = (rows + 127) / 128 * 128;
  a.R2 = (rows + 15) / 16 * 16;
  a.Ls = Ls;
  a.qpos0 = qpos0;
  a.tiles = (Ls + KT - 1) / KT;
  a.tpc = (a.tiles + nchunk - 1) / nchunk;
  a.nchunk = nchunk;
  a.sl = scale * 1.4426950408889634f;
  // as many K stages as fit beside the probe rows (227 KB per CTA)
  const uint32_t fixed = pt_smem(D, a.Rpad, 0).total + 1024;
  int nst = (int)((227u * 1024u - fixed) / (uint32_t)(KT * D * 2));
  a.nst = nst > kMaxStages ? kMaxStages : nst;
  if (a.nst < 2) return cudaErrorNotSupported;
  const uint32_t smem = pt_smem(D, a.Rpad, a.nst).total + 1024;
  const int nbh = B * Hkv;
  CUtensorMap mq, mk;
  // probe rows: [B*Hq][P][D] with the caller's head stride
  if (!make_map_bf16(&mq, q_probe, D, P, (uint64_t)B * Hq, (uint64_t)D * 2, (uint64_t)q_head_stride * 2, P) ||
      !make_map_bf16(&mk, k, D, Ls, nbh, (uint64_t)D * 2, (uint64_t)D * 2 * Ls, KT))
    return cudaErrorInvalidValue;
  // nchunk comes from probe_tc_chunks (a count of the form ceil(tiles / t)),
  // so with tpc = ceil(tiles / nchunk) every one of the nchunk CTAs has tiles
  const int nch = nchunk;
  if ((nch - 1) * a.tpc >= a.tiles) return cudaErrorInvalidValue;
  if (D == 128)
    return colsum ? launch_t<128, true>(mq, mk, a, nbh, nch, smem, s, pdl)
                  : launch_t<128, false>(mq, mk, a, nbh, nch, smem, s, pdl);
  return colsum ? launch_t<64, true>(mq, mk, a, nbh, nch, smem, s, pdl)
                : launch_t<64, false>(mq, mk, a, nbh, nch, smem, s, pdl);
}

}  // namespace hq
