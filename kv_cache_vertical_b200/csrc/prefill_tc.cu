// prefill_tc.cu -- hybrid-precision prefill attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory), head_dim 128.
//
// Method: ACL abstract of HyQuant, Prefill stage -- a hybrid-precision attention
// operator keeps the vertical-line tokens and a local sliding window at full
// precision and quantizes the remaining context; "HyQuant: Hybrid-Precision
// Quantization for LLM Attention" (wiki summary), TL;DR.  Per causal pair
// (i, j <= i): window (j > i - W) or vertical column -> bf16 logit; otherwise
// INT8 logit (exact s32 dot product x per-row Q scale x per-64-key K scale);
// one online softmax; P.V with fp16 P and fp16 V, fp32 accumulation.
//
// One CTA per (128-query tile, pair of query heads that share a KV head): the
// two heads ("A" and "B") see exactly the same key tiles, so every K / V tile
// loaded once feeds both.  Warp roles:
//   warp 0      TMA producer: the four Q tiles once, then a 4-stage ring of
//               (K tile, V tile) pairs;
//   warp 1      allocates 512 TMEM columns; lane 0 issues head A's MMAs,
//   warp 2      lane 0 issues head B's MMAs:
//               S_X = Q_X K^T (kind::i8 into s32, kind::f8f6f4 into f32, or
//               kind::f16 bf16 into f32) and O_X += P_X V (kind::f16, P read
//               from tensor memory, in 32-key chunks as the softmax hands
//               them over);
//   warp 3      idle (warps 0-3 keep the softmax warpgroups aligned to TMEM lanes);
//   warps 4-7   softmax of head A, warps 8-11 softmax of head B: one thread per
//               query row (TMEM lane), so row max / sum need no shuffles.
// Key tiles are 64 keys wide.  TMEM per head X (256 columns): two S buffers
// of 64 columns, S(t) in buffer t & 1 (P(t), packed fp16 pairs, overwrites the
// first 32 columns of its buffer), then O_X in the upper 128.  With S double
// buffered, the QK of the next tile runs while the softmax works on this one.
// Low-bit tiles are INT8 (kind::i8, s32 scores) or FP8 E4M3 (kind::f8f6f4,
// fp32 scores), one format per instantiation.
// Key tiles per query tile, each its own iteration of the online softmax:
//   low tiles   64 consecutive REMAINING (non-vertical) keys, compacted in
//               position order by the pre-pass: keep the keys at positions
//               <= i - W (a prefix of the compact order, so only the last
//               tiles need a per-row bound and no tile needs a vertical mask);
//   window      bf16 tiles of positions meeting (i - W, i]: keep i - W < j <= i;
//   vertical    compact bf16 rows (sorted): keep v <= i - W;
// so every causal pair is counted exactly once.
#include <cuda.h>
#include <float.h>
#include <limits.h>

#include "hq_internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"
#include "warp_mma.cuh"

namespace hq {
namespace {

constexpr int BM = 128, BN = 64, D = 128;
constexpr int NWARPS = 12, NTHR = NWARPS * 32;
constexpr int SM_WARP0 = 4;                     // warps 4-7: head A, 8-11: head B
constexpr int kRegsLaunch = 168;                // 65536 / 384, what a 384-thread CTA starts with
constexpr int kRegsLow = 56, kRegsHigh = 224;   // 128 * 56 + 256 * 224 == 384 * 168
constexpr int NCHUNK = 2;                       // P handed to the MMA in 32-key chunks
constexpr int NST = 4;                          // K/V stages
constexpr uint32_t SM_QI8 = 0;                 // [2 heads][128 rows x 128 B]
constexpr uint32_t SM_QBF = 32768;             // [2 heads][2 boxes][128 rows x 128 B]
constexpr uint32_t SM_KV = 98304;              // [NST stages][K 16 KB | V 16 KB]
constexpr uint32_t KV_STAGE = 32768;
constexpr uint32_t KV_VOFF = 16384;            // V within a stage; K and V boxes are 8 KB
constexpr uint32_t SM_BAR = SM_KV + NST * KV_STAGE;
constexpr uint32_t SMEM_BYTES = SM_BAR + 256 + 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;                   // rescale O only when the max grows by > 2^8
constexpr float kMagic = 12582912.0f;           // 2^23 + 2^22
constexpr uint32_t kMagicBits = 0x4B400000u;    // bits of kMagic

constexpr uint32_t IDESC_I8 = make_idesc(2, 1, 1, 0, 0, BM, BN);     // s32 <- s8 x s8
constexpr uint32_t IDESC_BF = make_idesc(1, 1, 1, 0, 0, BM, BN);     // f32 <- bf16 x bf16
constexpr uint32_t IDESC_F8 = make_idesc(1, 0, 0, 0, 0, BM, BN);     // f32 <- e4m3 x e4m3
constexpr uint32_t IDESC_PV = make_idesc(1, 0, 0, 0, 1, BM, D);      // f32 <- f16 x f16 (V MN-major)

enum { IT_I8 = 0, IT_WIN = 1, IT_VERT = 2 };

// Raw INT8-tile score that marks a masked entry: as an int it is below any
// reachable dot product (|s| <= 128 * 127 * 127 < 2^22), and after adding the
// bits of 2^23 + 2^22 it is the bit pattern of -inf.
constexpr uint32_t kMaskRaw = 0xFF800000u - kMagicBits;
constexpr uint32_t kNegInfBits = 0xFF800000u;

// Max of 64 floats given as bits: 21 three-input maxes in 4 independent chains.
__device__ __forceinline__ float max64(const uint32_t (&x)[64]) {
  float c[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) c[u] = fmax3(__uint_as_float(x[u]), __uint_as_float(x[4 + u]), __uint_as_float(x[8 + u]));
#pragma unroll
  for (int e = 12; e + 8 <= 64; e += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (e + u + 4 < 64) c[u] = fmax3(c[u], __uint_as_float(x[e + u]), __uint_as_float(x[e + u + 4]));
  }
  // e = 12, 20, ..., 52 covers 12..59; the last four are 60..63
#pragma unroll
  for (int u = 0; u < 4; ++u) c[u] = fmaxf(c[u], __uint_as_float(x[60 + u]));
  return fmax3(fmaxf(c[0], c[1]), c[2], c[3]);
}

// Max of 64 signed ints: 8 independent chains, then a tree.
__device__ __forceinline__ int imax64(const uint32_t (&x)[64]) {
  int c[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) c[u] = (int)x[u];
#pragma unroll
  for (int e = 8; e < 64; ++e) c[e & 7] = max(c[e & 7], (int)x[e]);
  return max(max(max(c[0], c[1]), max(c[2], c[3])), max(max(c[4], c[5]), max(c[6], c[7])));
}

struct TcArgs {
  const float *sq;                    // [B*Hq, N]
  const float *sk;                    // [B*Hkv, nblk_r] one scale per 64 remaining keys
  const int32_t *idx;                 // [B*Hkv, k_vert] vertical columns, ascending
  float *out;                         // [B*Hq, N, D]
  uint32_t *status;
  int Hq, Hkv, N, window, k_vert, nblk_r;
  float sl;                           // softmax scale * log2(e)
};

// Remaining (non-vertical) keys at positions <= x.
__device__ __forceinline__ int remaining_upto(const int32_t *id, int k_vert, int x) {
  return x < 0 ? 0 : x + 1 - upper_bound_i32(id, k_vert, x);
}

struct Sched {
  int n_i8, n_w, kw0, n;
  __device__ __forceinline__ int type(int it) const {
    return it < n_i8 ? IT_I8 : (it < n_i8 + n_w ? IT_WIN : IT_VERT);
  }
  __device__ __forceinline__ int tile(int it) const {
    return it < n_i8 ? it : (it < n_i8 + n_w ? kw0 + it - n_i8 : it - n_i8 - n_w);
  }
};

__device__ __forceinline__ Sched make_sched(const TcArgs &a, int i0, size_t bh) {
  Sched s;
  const int i_max = min(i0 + BM - 1, a.N - 1);
  const int W = a.window;
  const int32_t *id = a.idx + bh * a.k_vert;
  s.n_i8 = (remaining_upto(id, a.k_vert, i_max - W) + BN - 1) / BN;
  if (W > 0) {
    s.kw0 = max(0, i0 - W + 1) / BN;
    s.n_w = i_max / BN - s.kw0 + 1;
  } else {
    s.kw0 = 0;
    s.n_w = 0;
  }
  const int cnt = i_max - W >= 0 ? upper_bound_i32(id, a.k_vert, i_max - W) : 0;
  s.n = s.n_i8 + s.n_w + (cnt + BN - 1) / BN;
  return s;
}

template <bool F8>
__global__ void __launch_bounds__(NTHR, 1)
prefill_tc(const __grid_constant__ CUtensorMap tm_qi8, const __grid_constant__ CUtensorMap tm_qbf,
           const __grid_constant__ CUtensorMap tm_ki8, const __grid_constant__ CUtensorMap tm_kbf,
           const __grid_constant__ CUtensorMap tm_v16, const __grid_constant__ CUtensorMap tm_vk,
           const __grid_constant__ CUtensorMap tm_vv, const __grid_constant__ CUtensorMap tm_vc,
           TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + SM_BAR);
  uint64_t *q_full = bar;
  uint64_t *kv_full = bar + 1;   // [NST]
  uint64_t *kv_free = bar + 5;   // [NST], one arrival per MMA issuer
  uint64_t *s_full = bar + 9;    // [2 heads][2 S buffers]
  uint64_t *p_full = bar + 13;   // [2 heads][2 S buffers][NCHUNK], one arrival per softmax warp
  uint64_t *pv_done = bar + 21;  // [2 heads]: the head's P.V of its latest tile has completed
  uint64_t *o_final = bar + 23;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 24);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bar + 25);

  const int ntq = (a.N + BM - 1) / BM;
  const int qt = ntq - 1 - (int)blockIdx.x;      // longest rows first
  const int hp = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int hA = 2 * hp;
  const int kh = hA / G;
  const size_t bh = (size_t)b * a.Hkv + kh;
  const int i0 = qt * BM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Sched sc = make_sched(a, i0, bh);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_free[s], 2);
    }
    for (int s = 0; s < 4; ++s) mbar_init(&s_full[s], 1);
    for (int s = 0; s < 4 * NCHUNK; ++s) mbar_init(&p_full[s], 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(o_final, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Each role runs to its own end (named barrier 1, then return), so the code
  // of the register-poor warps and of the softmax warps never merges again.
  if (warp < SM_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsLow));
  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const int bqA = b * a.Hq + hA, bqB = bqA + 1;
      mbar_arrive_expect_tx(q_full, 2 * 16384 + 2 * 32768);
      tma_load_3d(smem + SM_QI8, &tm_qi8, q_full, 0, i0, bqA);
      tma_load_3d(smem + SM_QI8 + 16384, &tm_qi8, q_full, 0, i0, bqB);
      tma_load_3d(smem + SM_QBF, &tm_qbf, q_full, 0, i0, bqA);
      tma_load_3d(smem + SM_QBF + 16384, &tm_qbf, q_full, 64, i0, bqA);
      tma_load_3d(smem + SM_QBF + 32768, &tm_qbf, q_full, 0, i0, bqB);
      tma_load_3d(smem + SM_QBF + 49152, &tm_qbf, q_full, 64, i0, bqB);
      int issued = 0;
      for (int it = 0; it < sc.n; ++it) {
        const int s = it % NST;
        if (it >= NST && !mbar_wait(&kv_free[s], ((it / NST) & 1) ^ 1)) {
          *abort_flag = 1;
          raise_status(a.status, HQ_DEV_TIMEOUT);
          break;
        }
        if (*abort_flag) break;
        uint8_t *ks = smem + SM_KV + s * KV_STAGE;
        uint8_t *vs = ks + KV_VOFF;
        const int ty = sc.type(it), t = sc.tile(it);
        const int row = t * BN;
        if (ty == IT_I8) {
          mbar_arrive_expect_tx(&kv_full[s], BN * 128 + BN * 256);
          tma_load_3d(ks, &tm_ki8, &kv_full[s], 0, row, (int)bh);
        } else {
          mbar_arrive_expect_tx(&kv_full[s], 2 * BN * 256);
          const CUtensorMap *km = ty == IT_WIN ? &tm_kbf : &tm_vk;
          tma_load_3d(ks, km, &kv_full[s], 0, row, (int)bh);
          tma_load_3d(ks + BN * 128, km, &kv_full[s], 64, row, (int)bh);
        }
        const CUtensorMap *vm = ty == IT_VERT ? &tm_vv : (ty == IT_I8 ? &tm_vc : &tm_v16);
        tma_load_3d(vs, vm, &kv_full[s], 0, row, (int)bh);
        tma_load_3d(vs + BN * 128, vm, &kv_full[s], 64, row, (int)bh);
        issued = it + 1;
      }
      // do not leave with copies in flight
      if (!mbar_wait(q_full, 0)) raise_status(a.status, HQ_DEV_TIMEOUT);
      for (int it = issued > NST ? issued - NST : 0; it < issued; ++it)
        if (!mbar_wait(&kv_full[it % NST], (it / NST) & 1)) raise_status(a.status, HQ_DEV_TIMEOUT);
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------------- MMA issuers, one per head ----------------------
    // Warp 1 issues head A's MMAs, warp 2 head B's.  S is double-buffered in
    // TMEM, so QK(t+1) runs while the softmax works on S(t); per tile t the
    // issuer hands P(t).V(t) to the tensor core chunk by chunk as the softmax
    // releases the chunks, then issues QK(t+2) into the buffer of S(t).  P(t)
    // lives in that buffer and the PTX pipelining rule orders two MMAs only
    // when they share the accumulator, so QK(t+2) waits for P(t).V(t) to
    // complete -- by then the softmax of tile t+1 is under way, so the wait
    // costs the softmax nothing.
    if (lane == 0) {
      const int x = warp - 1;
      const uint32_t sQi8 = smem_u32(smem + SM_QI8), sQbf = smem_u32(smem + SM_QBF);
      const uint32_t sKV = smem_u32(smem + SM_KV);
      const uint32_t hx = tmem + x * 256;                 // S buffers [0,64), [64,128); O [128,256)
      bool ok = mbar_wait(q_full, 0);
      auto issue_qk = [&](int it) {
        const uint32_t kslot = sKV + (it % NST) * KV_STAGE;
        const uint32_t dt = hx + (it & 1) * BN;
        if (sc.type(it) == IT_I8) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = make_sdesc_sw128(sQi8 + x * 16384 + ks * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(kslot + ks * 32, 16, 1024);
            if (F8)
              mma_f8_ss(dt, ad, bd, IDESC_F8, ks > 0);
            else
              mma_i8_ss(dt, ad, bd, IDESC_I8, ks > 0);
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t k16 = (ks & 3) * 32;
            const uint64_t ad = make_sdesc_sw128(sQbf + x * 32768 + (ks >> 2) * 16384 + k16, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(kslot + (ks >> 2) * (BN * 128) + k16, 16, 1024);
            mma_f16_ss(dt, ad, bd, IDESC_BF, ks > 0);
          }
        }
        tc_commit(&s_full[x * 2 + (it & 1)]);
      };
      for (int it = 0; ok && it < 2 && it < sc.n; ++it) {
        if (!(ok = mbar_wait(&kv_full[it], 0))) break;
        tc_fence_after();
        issue_qk(it);
      }
      for (int it = 0; ok && it < sc.n; ++it) {
        const int buf = it & 1;
        const uint32_t vslot = sKV + (it % NST) * KV_STAGE + KV_VOFF;
        const uint32_t dO = hx + 128, aP = hx + buf * BN;
#pragma unroll
        for (int c = 0; c < NCHUNK; ++c) {
          if (!(ok = mbar_wait(&p_full[(x * 2 + buf) * NCHUNK + c], (it >> 1) & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int ks = 2 * c + j;                       // 16 keys per MMA
            const uint64_t bd = make_sdesc_sw128(vslot + ks * 2048, BN * 128, 1024);
            mma_f16_ts(dO, aP + ks * 8, bd, IDESC_PV, (it > 0 || ks > 0) ? 1u : 0u);
          }
        }
        if (!ok) break;
        tc_commit(&kv_free[it % NST]);              // one of the two arrivals
        tc_commit(&pv_done[x]);
        if (it + 2 < sc.n) {
          if (!(ok = mbar_wait(&kv_full[(it + 2) % NST], ((it + 2) / NST) & 1))) break;
          if (!(ok = mbar_wait(&pv_done[x], it & 1))) break;
          tc_fence_after();
          issue_qk(it + 2);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(a.status, HQ_DEV_TIMEOUT);
      }
      tc_commit(o_final);
    }
  }
    tc_fence_before();
    asm volatile("bar.sync 1, %0;\n" ::"r"(NTHR) : "memory");
    if (warp == 1) {
      tc_fence_after();
      // every MMA has completed once o_final fired; wait for it (bounded) in
      // case a softmax warp gave up before it did
      if (!mbar_wait(o_final, 0)) raise_status(a.status, HQ_DEV_TIMEOUT);
      tmem_dealloc(tmem, 512);
    }
    return;
  }
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsHigh));
  {
    // ------------------------------ softmax ------------------------------
    // One thread per query row (TMEM lane), the whole 64-key S row of a tile in
    // registers.  INT8 scores stay integers until the exp: their row max is an
    // integer max, and adding the bits of 2^23 + 2^22 turns s into the float
    // 2^23 + 2^22 + s (exact for |s| < 2^22), whose offset is folded into the
    // scaling FMA.
    const int X = (warp - SM_WARP0) >> 2;          // 0: head A, 1: head B
    const int hq = hA + X;
    const int quarter = warp & 3;                  // TMEM lanes 32*quarter ..
    const int r = quarter * 32 + lane;
    const int i = i0 + r;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = tl + X * 256, tO = tS + 128;   // S buffers at tS, tS + BN
    const size_t bhq = (size_t)b * a.Hq + hq;
    const float sqi = (i < a.N) ? a.sq[bhq * a.N + i] * a.sl : 1.f;
    const int W = a.window;
    const int lim = i - W;                         // low-bit and vertical keys need j <= lim
    const int32_t *id = a.idx + bh * a.k_vert;
    const int cnt_i = remaining_upto(id, a.k_vert, lim);        // low-bit keys of this row
    const int cnt_lo = remaining_upto(id, a.k_vert, i0 - W);     // ... of the tile's first row
    const int nvert = lim >= 0 ? upper_bound_i32(id, a.k_vert, lim) : 0;
    const float *skp = a.sk + bh * a.nblk_r;
    // K scale of a low tile (one 64-key block), fetched one tile ahead
    auto fetch_scale = [&](int it) {
      float k = 1.f;
      if (it < sc.n && sc.type(it) == IT_I8) {
        const int t = sc.tile(it);
        if (t < a.nblk_r) k = __ldg(skp + t);
      }
      return k;
    };
    float kn = fetch_scale(0);
    float m = -1e30f;
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};       // independent partial row sums
    bool ok = true;
    for (int it = 0; it < sc.n; ++it) {
      const int buf = it & 1;
      const float k0 = kn;
      kn = fetch_scale(it + 1);
      if (!mbar_wait(&s_full[X * 2 + buf], (it >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int ty = sc.type(it), t = sc.tile(it);
      const int j0 = t * BN;
      const uint32_t tSb = tS + buf * BN;
      uint32_t xa[64];
      tmem_ld64(tSb, xa);                           // the whole 64-key S row
      float sc0, c0, mt;                            // scale and offset (log2 units)
      uint32_t add = 0u;                            // bits added to a raw score before the FMA
      if (F8 && ty == IT_I8) {                     // fp32 scores of FP8 codes
        sc0 = sqi * k0;
        c0 = 0.f;
        if (j0 + BN > cnt_lo) {
          const int nvalid = cnt_i - j0;
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) xa[e] = kNegInfBits;
        }
        mt = max64(xa) * sc0;
      } else if (!F8 && ty == IT_I8) {
        sc0 = sqi * k0;
        if (j0 + BN > cnt_lo) {                     // same for every row of the tile
          const int nvalid = cnt_i - j0;
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) xa[e] = kMaskRaw;
        }
        c0 = -kMagic * sc0;
        add = kMagicBits;
        mt = fmaf(__uint_as_float((uint32_t)imax64(xa) + kMagicBits), sc0, c0);
      } else {
        sc0 = a.sl;
        c0 = 0.f;
        if (ty == IT_WIN) {
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            const int j = j0 + e;
            if (j > i || j <= lim) xa[e] = kNegInfBits;
          }
        } else {
          const int nvalid = nvert - j0;
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) xa[e] = kNegInfBits;
        }
        mt = max64(xa) * a.sl;
      }
      // ---- lazy rescale of the running max, and of O once the P.V of the
      // previous tile has completed ----
      const bool need = mt > m + kLazy;
      if (__any_sync(0xffffffffu, need)) {
        const float mn = fmaxf(m, mt);
        const float al = exp2f(m - mn);
        m = mn;
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = make_float2(acc[u].x * al, acc[u].y * al);
        if (it > 0) {
          if (!mbar_wait(&pv_done[X], (it - 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + ch * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * al);
            tmem_st32(tO + ch * 32, o);
          }
        }
      }
      // ---- P = exp2(x * scale + offset - m) as packed fp16, 32 keys per
      // chunk, each chunk handed to the MMA as soon as it is in TMEM ----
      c0 -= m;
      const float2 s2 = make_float2(sc0, sc0), o2 = make_float2(c0, c0);
#pragma unroll
      for (int q = 0; q < NCHUNK; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 y = ffma2(make_float2(__uint_as_float(xa[q * 32 + 2 * e] + add),
                                             __uint_as_float(xa[q * 32 + 2 * e + 1] + add)), s2, o2);
          const float2 p = make_float2(fast_exp2(y.x), fast_exp2(y.y));
          acc[e & 3] = fadd2(acc[e & 3], p);
          pk[e] = pack_f16x2(p.x, p.y);
        }
        // hand over the previous chunk (its store has had this chunk's exps
        // to complete), then store this one
        if (q > 0) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[(X * 2 + buf) * NCHUNK + q - 1]);
        }
        tmem_st16(tSb + q * 16, pk);               // keys 32*q .. 32*q+31
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[(X * 2 + buf) * NCHUNK + NCHUNK - 1]);
    }
    const float l = (acc[0].x + acc[0].y + acc[1].x + acc[1].y) + (acc[2].x + acc[2].y + acc[3].x + acc[3].y);
    if (ok) ok = mbar_wait(o_final, 0);
    if (!ok) {
      *abort_flag = 1;
      raise_status(a.status, HQ_DEV_TIMEOUT);
    }
    tc_fence_after();
    const float inv = (ok && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t o[32];
      tmem_ld32(tO + ch * 32, o);
      if (ok && i < a.N) {
        float4 *dst = reinterpret_cast<float4 *>(a.out + (bhq * a.N + i) * D + ch * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                               __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
      }
    }
  }
  tc_fence_before();
  asm volatile("bar.sync 1, %0;\n" ::"r"(NTHR) : "memory");
}

}  // namespace

// The kernel redistributes registers with setmaxnreg, which is only valid
// when the CTA starts with exactly kRegsLaunch registers per thread; that is
// checked once from the compiled kernel.  If the check fails the prefill is
// reported unsupported and nothing is launched (there is no other kernel).
template <bool F8>
static bool kernel_ready() {
  cudaFuncAttributes fa;
  return cudaFuncGetAttributes(&fa, prefill_tc<F8>) == cudaSuccess && fa.numRegs == kRegsLaunch &&
         cudaFuncSetAttribute(prefill_tc<F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              SMEM_BYTES) == cudaSuccess;
}

static bool prefill_tc_ready() {
  static int ready = -1;
  if (ready < 0) ready = kernel_ready<false>() && kernel_ready<true>();
  return ready == 1;
}

bool prefill_tc_supported(int D_, int Hq, int Hkv) {
  return D_ == 128 && Hq % Hkv == 0 && (Hq / Hkv) % 2 == 0 && prefill_tc_ready();
}

cudaError_t launch_prefill_tc(const TcLaunch &p, cudaStream_t s) {
  if (!prefill_tc_ready()) return cudaErrorInvalidValue;
  const int nbq = p.B * p.Hq, nbh = p.B * p.Hkv;
  const int nr = p.N - p.k_vert;                      // remaining keys per (b, kv head)
  CUtensorMap m[8];
  bool ok = true;
  ok &= make_map_3d(&m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (void *)p.qi8, D, p.N, nbq, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void *)p.q, D, p.N, nbq, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[2], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (void *)p.ki8, D, nr, nbh, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[3], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void *)p.k, D, p.N, nbh, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[4], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void *)p.vh, D, p.N, nbh, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[5], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void *)p.vk, D, p.kpad, nbh, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[6], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void *)p.vv, D, p.kpad, nbh, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_3d(&m[7], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void *)p.vc, D, nr, nbh, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  TcArgs a;
  a.sq = p.sq;
  a.sk = p.sk;
  a.idx = p.idx;
  a.out = p.out;
  a.status = p.status;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.N = p.N;
  a.window = p.window;
  a.k_vert = p.k_vert;
  a.nblk_r = p.nblk_r;
  a.sl = p.scale * kLog2e;
  dim3 grid((p.N + BM - 1) / BM, p.Hq / 2, p.B);
  if (p.f8)
    prefill_tc<true><<<grid, NTHR, SMEM_BYTES, s>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], a);
  else
    prefill_tc<false><<<grid, NTHR, SMEM_BYTES, s>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], a);
  return cudaGetLastError();
}

}  // namespace hq
