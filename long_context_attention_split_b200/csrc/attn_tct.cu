// (i) Exact cached-token attention for 3-32 query rows per KV head, on the
// tensor cores: Eq. (3.1) of "Nectar: Neural Estimation of Cached-Token
// Attention via Regression" (§2.1), split over n and joined by log-sum-exp.
//
// At a few rows per head the CUDA-core split kernel spends ~10 instructions
// per (key, row, dim) and is bound by the ALU, not by the K/V bytes.  Here
// the products run on tcgen05, taken transposed so that the keys fill the
// 128 rows of the tensor-core tile and the TMEM lanes:
//   S^T = K Q^T   (M = 128 keys of a tile, N = QC = 16 or 32 >= rows, K = d; K, Q
//                  K-major, 128-byte swizzle),
//   O^T = V^T P^T (M = d, N = QC, K = the tile's keys; V read MN-major).
// Each of the 128 softmax threads owns one key of a tile and holds its row
// scores; the online softmax keeps one running maximum per row for the whole
// CTA: a tile's maximum is reduced over the 128 threads, and the maximum
// moves only when the tile's exceeds it by 2^8 (log2 units, as in the split
// kernel), in which case the O^T column is rescaled in TMEM; that decision
// is the same in every thread.  Each thread keeps its own partial sum of the
// row weights; they are reduced at the end of a head's range.
//
// Schedule and output: the split kernel's.  All heads' 128-key tiles are laid
// end to end and CTA c takes [c T / C, (c + 1) T / C) (two CTAs per SM, so
// that one CTA's softmax latency hides under the other's); a CTA leaves one
// partial (m, l, acc) per head it touched in the workspace, and the split
// kernel's combine launch joins them.
//
// Warp roles: 0 TMA producer (K and V tiles, 32 KB each, into one ring in
// the order the MMAs consume them: K0 K1 V0 K2 V1 ...; the head's Q rows
// per head range), 1 MMA issuer (+ TMEM owner), then one softmax and
// epilogue warpgroup per 16 query columns (each thread: one key, 16 rows).
// S^T and P are double-buffered per tile, Q and O^T per head range, so the
// tile after next is scored while this one's weights are formed.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

namespace {

constexpr int kTKeys = kTctTile;                   // keys per tile (TMEM lanes of S^T)
#ifndef NECTAR_TCT_STAGES
#define NECTAR_TCT_STAGES (6 / NECTAR_TCT_CTAS_PER_SM)
#endif
// Per query-column count QC: resident CTAs per SM and K / V ring stages.
// 16 columns: two CTAs of NECTAR_TCT_STAGES stages; 32 columns (Q, P and
// the row state grow with QC): one CTA of six stages.
template <int QC>
struct TCfg {
  static constexpr int wgs = QC / 16;                     // softmax warpgroups
  static constexpr int threads = 64 + 128 * wgs;
  static constexpr int ctas = QC == 16 ? kTctCtasPerSm : 1;
  static constexpr int stages = QC == 16 ? NECTAR_TCT_STAGES : 6;
};
constexpr uint32_t kTHalf = kTKeys * 128;          // 128 keys x 64 dims bf16: 16 KB
constexpr uint32_t kTTile = 2 * kTHalf;
// one softmax warpgroup (128 threads) per 16 query columns

template <int QC>
struct TSmem {
  static constexpr uint32_t kQHalf = QC * 128;                  // QC rows x 64 dims
  static constexpr uint32_t kQ = 2 * kQHalf;
  static constexpr uint32_t kPChunk = QC * 128;                 // QC rows x 64 keys
  static constexpr uint32_t kP = 2 * kPChunk;                   // one tile of P
  static constexpr uint32_t ring = 0;                           // [stages] K or V tiles
  static constexpr uint32_t q = ring + TCfg<QC>::stages * kTTile;   // [2 head ranges]
  static constexpr uint32_t p = q + 2 * kQ;                     // [2 tiles]
  static constexpr uint32_t red = p + 2 * kP;                   // float [2 tiles][4 warps][QC] maxima
  static constexpr uint32_t reds = red + 2 * 4 * QC * 4;        // float [4 warps][QC] sums
  static constexpr uint32_t corrs = reds + 4 * QC * 4;          // float [QC] a tile's rescale factors
  static constexpr uint32_t bars = corrs + QC * 4;
  // 2 x stages ring barriers, 15 more, the TMEM slot (8 bytes each)
  static constexpr uint32_t total = bars + (2 * TCfg<QC>::stages + 16) * 8;
};

// byte offset of P[row][key] in one tile's P buffer (two K-major 64-key
// chunks of QC rows, 128-byte swizzle)
template <int QC>
__device__ __forceinline__ uint32_t tp_off(int row, int key) {
  return static_cast<uint32_t>(((key >> 6) & 1) * TSmem<QC>::kPChunk + row * 128 +
                               ((((key & 63) >> 3) ^ (row & 7)) << 4) + ((key & 7) << 1));
}

// NV per-lane values reduced over the 32 lanes of a warp (max or sum):
// halving steps (a lane keeps one half of its values and sends the other
// half to its partner), then plain butterfly steps.  Lane L ends with value
// L / (32 / NV) reduced over all lanes.
template <int NV, bool kMax>
__device__ __forceinline__ float twarp_reduce(float (&v)[NV], int lane) {
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const int half = n / 2;
      const bool up = lane & off;
#pragma unroll
      for (int j = 0; j < half; ++j) {
        const float lo = v[j], hi = v[j + half];
        const float send = up ? lo : hi, keep = up ? hi : lo;
        const float got = __shfl_xor_sync(0xffffffffu, send, off);
        v[j] = kMax ? fmaxf(keep, got) : keep + got;
      }
      n = half;
    } else {
      const float got = __shfl_xor_sync(0xffffffffu, v[0], off);
      v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
    }
  }
  return v[0];
}

// 16 columns of 32 lanes of TMEM <-> registers (warp-collective)
__device__ __forceinline__ void ttmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

}  // namespace

template <int QC>
__global__ void __launch_bounds__(TCfg<QC>::threads, TCfg<QC>::ctas)
cache_attn_tct_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const DecParams p) {
  using SL = TSmem<QC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (TCfg<QC>::ctas > 1 && smem != smem_raw) {
    // two CTAs per SM request no alignment slack: refuse rather than overrun
    if (threadIdx.x == 0) record_error(p.err, DEVERR_WAIT_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL::bars);
  constexpr int kTStages = TCfg<QC>::stages;
  const uint32_t b_full = smem_u32(bars);                    // [kTStages]
  const uint32_t b_empty = smem_u32(bars + kTStages);        // [kTStages]
  uint64_t* const bx = bars + 2 * kTStages;
  const uint32_t b_qfull = smem_u32(bx + 0);         // [2] per head range
  const uint32_t b_qempty = smem_u32(bx + 2);        // [2]
  const uint32_t b_sfull = smem_u32(bx + 4);         // [2] per tile
  const uint32_t b_sfree = smem_u32(bx + 6);         // [2]
  const uint32_t b_pfull = smem_u32(bx + 8);         // [2]
  const uint32_t b_pfree = smem_u32(bx + 10);        // [2]
  const uint32_t b_ofull = smem_u32(bx + 12);        // one phase per tile's O^T update
  const uint32_t b_ofree = smem_u32(bx + 13);        // [2] per head range
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bx + 15);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(c) * p.total / p.C;
  const int64_t t1 = static_cast<int64_t>(c + 1) * p.total / p.C;
  const int ntiles = static_cast<int>(t1 - t0);
  const int64_t hd0 = t0 / p.tph;
  const int R = static_cast<int>(p.rows_total);
  constexpr uint32_t kTmemCols = 4 * QC < 32 ? 32 : 4 * QC;   // S^T [2][QC], O^T [2][QC]
  constexpr int kWG = TCfg<QC>::wgs;
  constexpr int kThreadsAll = TCfg<QC>::threads;
  static_assert(QC == 16 || QC == 32, "16 or 32 query columns");
  const uint32_t kOCol = 2 * QC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(b_qfull + 8 * x, 1);
      mbar_init(b_qempty + 8 * x, 1);
      mbar_init(b_sfull + 8 * x, 1);
      mbar_init(b_sfree + 8 * x, 128 * kWG);
      mbar_init(b_pfull + 8 * x, 128 * kWG);
      mbar_init(b_pfree + 8 * x, 1);
      mbar_init(b_ofree + 8 * x, 128 * kWG);
    }
    mbar_init(b_ofull, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // Q rows past the R that TMA writes stay 0 (their S^T and O^T columns are unused)
    for (int x = threadIdx.x - 64; x < 2 * 2 * (QC - R) * 8; x += kThreadsAll - 64) {
      const int buf = x / (2 * (QC - R) * 8), rem = x % (2 * (QC - R) * 8);
      const int half = rem / ((QC - R) * 8), rr = rem % ((QC - R) * 8);
      reinterpret_cast<uint4*>(smem + SL::q + buf * SL::kQ + half * SL::kQHalf + R * 128)[rr] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  griddep_wait();                 // inputs and outputs only from here on (launched after another kernel)

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      const uint64_t pol = policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      auto load_tile = [&](const CUtensorMap* map, int64_t t) {
        const uint32_t s = it % kTStages;
        if (it >= kTStages) ok = mbar_wait(b_empty + 8 * s, ((it / kTStages) - 1) & 1, p.err);
        if (!ok) return;
        const int64_t hd = t / p.tph, kt = t % p.tph;
        mbar_arrive_expect_tx(b_full + 8 * s, kTTile);
        tma_load_4d(smem_u32(smem + SL::ring + s * kTTile), map, 0, static_cast<int>(kt * kTKeys), 0,
                    static_cast<int>(hd), b_full + 8 * s, pol);
        ++it;
      };
      for (int i = 0; i <= ntiles && ok; ++i) {
        if (i < ntiles) {
          const int64_t t = t0 + i;
          const int64_t hd = t / p.tph;
          if (i == 0 || t % p.tph == 0) {
            // this head's query rows, one box per 64-column half
            const int seg = static_cast<int>(hd - hd0);
            const uint32_t qb = seg & 1;
            if (seg >= 2 && !(ok = mbar_wait(b_qempty + 8 * qb, ((seg >> 1) - 1) & 1, p.err))) break;
            mbar_arrive_expect_tx(b_qfull + 8 * qb, static_cast<uint32_t>(2 * R * 128));
            const uint32_t qd = smem_u32(smem + SL::q + qb * SL::kQ);
            tma_load_4d(qd, &tmap_q, 0, 0, 0, static_cast<int>(hd), b_qfull + 8 * qb, pol);
            tma_load_4d(qd + SL::kQHalf, &tmap_q, 0, 0, 1, static_cast<int>(hd), b_qfull + 8 * qb, pol);
          }
          load_tile(&tmap_k, t);
        }
        if (i >= 1) load_tile(&tmap_v, t0 + i - 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, QC, 0, 0);   // A = K tile, B = Q
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, QC, 1, 0);   // A = V tile (MN-major), B = P
      bool ok = true;
      uint32_t it = 0;
      for (int i = 0; i <= ntiles && ok; ++i) {
        if (i < ntiles) {
          // S^T of tile i
          const int64_t t = t0 + i;
          const int seg = static_cast<int>(t / p.tph - hd0);
          const uint32_t qb = seg & 1, sb = i & 1;
          if ((i == 0 || t % p.tph == 0) && !(ok = mbar_wait(b_qfull + 8 * qb, (seg >> 1) & 1, p.err))) break;
          if (i >= 2 && !(ok = mbar_wait(b_sfree + 8 * sb, ((i >> 1) - 1) & 1, p.err))) break;
          const uint32_t s = it % kTStages;
          if (!(ok = mbar_wait(b_full + 8 * s, (it / kTStages) & 1, p.err))) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + SL::ring + s * kTTile);
          const uint32_t qa = smem_u32(smem + SL::q + qb * SL::kQ);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + sb * QC, sdesc_sw128(ka + (kk >> 2) * kTHalf + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(qa + (kk >> 2) * SL::kQHalf + (kk & 3) * 32, 16, 1024), idesc_s, kk != 0);
          mma_commit(b_empty + 8 * s);
          ++it;
          mma_commit(b_sfull + 8 * sb);
          if (i == ntiles - 1 || (t + 1) % p.tph == 0) mma_commit(b_qempty + 8 * qb);
        }
        if (i >= 1) {
          // O^T += V^T P^T of tile j = i - 1, once its weights are in P
          const int j = i - 1;
          const int64_t t = t0 + j;
          const int seg = static_cast<int>(t / p.tph - hd0);
          const bool first = (j == 0 || t % p.tph == 0);
          const uint32_t pb = j & 1;
          if (!(ok = mbar_wait(b_pfull + 8 * pb, (j >> 1) & 1, p.err))) break;
          if (first && seg >= 2 && !(ok = mbar_wait(b_ofree + 8 * (seg & 1), ((seg >> 1) - 1) & 1, p.err))) break;
          const uint32_t s = it % kTStages;
          if (!(ok = mbar_wait(b_full + 8 * s, (it / kTStages) & 1, p.err))) break;
          tc_fence_after();
          const uint32_t va = smem_u32(smem + SL::ring + s * kTTile);
          const uint32_t pa = smem_u32(smem + SL::p + pb * SL::kP);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + kOCol + (seg & 1) * QC, sdesc_sw128(va + kk * 2048, kTHalf, 1024),
                        sdesc_sw128(pa + (kk >> 2) * SL::kPChunk + (kk & 3) * 32, 16, 1024), idesc_o,
                        (!first || kk != 0) ? 1u : 0u);
          mma_commit(b_empty + 8 * s);
          ++it;
          mma_commit(b_pfree + 8 * pb);
          mma_commit(b_ofull);
        }
      }
    }
  } else {
    // ------------- softmax + epilogue (one warpgroup per 16 columns) -------------
    const int wg = (warp - 2) >> 2;                  // softmax warpgroup: columns [16 wg, 16 wg + 16)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                // key of a tile (S^T) / dim (O^T)
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int CH = 16;
    const int cb = wg * CH;
    float* red = reinterpret_cast<float*>(smem + SL::red);
    float* reds = reinterpret_cast<float*>(smem + SL::reds);
    float* corrs = reinterpret_cast<float*>(smem + SL::corrs);
    bool ok = true;
    float M[CH], lp[CH];
    for (int i = 0; i < ntiles; ++i) {
      const int64_t t = t0 + i;
      const int64_t hd = t / p.tph, kt = t % p.tph;
      const int seg = static_cast<int>(hd - hd0);
      const bool first = (i == 0 || kt == 0);
      const bool last = (i == ntiles - 1 || (t + 1) % p.tph == 0);
      const uint32_t sb = i & 1;
      if (first) {
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          M[j] = -INFINITY;
          lp[j] = 0.f;
        }
      }
      if (ok) ok = mbar_wait(b_sfull + 8 * sb, (i >> 1) & 1, p.err);
      tc_fence_after();
      const bool valid = kt * kTKeys + r < p.n;
      // pass 1: the tile's maximum per row over its 128 keys
      {
        uint32_t v[CH];
        NECTAR_TMEM_LD16(tmem + sb * QC + cb + lane_base, v);
        tmem_ld_wait();
        float mx[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) mx[j] = (valid && cb + j < R) ? __uint_as_float(v[j]) * p.qmul : -INFINITY;
        const float w = twarp_reduce<CH, true>(mx, lane);
        if ((lane & 1) == 0) red[(sb * 4 + quarter) * QC + cb + (lane >> 1)] = w;
      }
      named_bar_sync(1 + wg, 128);
      bool need = false;
      float my_corr = 1.f;                            // the factor of column cb + r (r < CH)
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const float* rq = red + sb * 4 * QC + cb + j;
        const float mt = fmaxf(fmaxf(rq[0], rq[QC]), fmaxf(rq[2 * QC], rq[3 * QC]));
        float corr = 1.f;
        if (mt > M[j] + kRescaleSlack) {             // also the head's first finite maximum
          corr = exp2_shift(M[j], mt);
          M[j] = mt;
          need = true;
        }
        lp[j] *= corr;
        if (j == r) my_corr = corr;
      }
      if (need && !first) {
        // the running O^T holds the tiles up to i - 1: rescale this
        // warpgroup's columns (the same decision in its every thread)
        if (r < CH) corrs[cb + r] = my_corr;
        named_bar_sync(9 + wg, 128);
        if (ok) ok = mbar_wait(b_ofull, (i - 1) & 1, p.err);
        tc_fence_after();
        const uint32_t oaddr = tmem + kOCol + (seg & 1) * QC + cb + lane_base;
        uint32_t o[CH];
        NECTAR_TMEM_LD16(oaddr, o);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < CH; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * corrs[cb + j]);
        ttmem_st16(oaddr, o);
        tmem_st_wait();
      }
      // pass 2: the weights, bf16 into P (row, key): what the P V product and
      // the row sums both use
      if (i >= 2 && ok) ok = mbar_wait(b_pfree + 8 * sb, ((i >> 1) - 1) & 1, p.err);
      uint8_t* pt = smem + SL::p + sb * SL::kP;
      {
        uint32_t v[CH];
        NECTAR_TMEM_LD16(tmem + sb * QC + cb + lane_base, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const float sc = (valid && cb + j < R) ? __uint_as_float(v[j]) * p.qmul : -INFINITY;
          const __nv_bfloat16 w = __float2bfloat16_rn(exp2_shift(sc, M[j]));
          lp[j] += __bfloat162float(w);
          *reinterpret_cast<__nv_bfloat16*>(pt + tp_off<QC>(cb + j, r)) = w;
        }
      }
      tc_fence_before();
      mbar_arrive(b_sfree + 8 * sb);                  // S^T of this tile read for the last time
      fence_proxy_async_smem();
      // ofull completes one phase per tile's O^T update, in order, and a
      // parity wait only tells the current phase from the one before.  At a
      // head range's last tile this thread waits for O(i), so first for
      // O(i - 1) (issued after S(i), it may still be running: a wait for
      // phase i alone would pass on phase i - 1's parity) -- and that before
      // its P(i) lets O(i) be issued: waited after, O(i) could complete
      // first, and the parity of phase i - 1 would then name phase i + 1,
      // which waits on this thread's next P (seen as a wait that ran out
      // when another kernel ran beside this one).  (The rescale's wait for
      // O(i - 1) needs no such step: S(i), complete by then, was issued
      // after O(i - 2), and P(i) is not written yet.)
      if (last && ok && i >= 1) ok = mbar_wait(b_ofull, (i - 1) & 1, p.err);
      mbar_arrive(b_pfull + 8 * sb);
      if (last) {
        // the head's partial: O^T (this thread: dim r), the row sums, M
        if (ok) ok = mbar_wait(b_ofull, i & 1, p.err);
        tc_fence_after();
        const int slot = c - first_cta_of_tile(hd * p.tph, p.total, p.C);
        uint32_t o[CH];
        NECTAR_TMEM_LD16(tmem + kOCol + (seg & 1) * QC + cb + lane_base, o);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(b_ofree + 8 * (seg & 1));
        float ls[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) ls[j] = lp[j];
        const float w = twarp_reduce<CH, false>(ls, lane);
        if ((lane & 1) == 0) reds[quarter * QC + cb + (lane >> 1)] = w;
        if (ok) {
#pragma unroll
          for (int j = 0; j < CH; ++j) {
            const int q = cb + j;
            if (q < R) p.ws_acc[((hd * p.S_max + slot) * p.rows_total + q) * kD + r] = __uint_as_float(o[j]);
          }
        }
        named_bar_sync(5 + wg, 128);
        if (ok && r < CH && cb + r < R) {
          const int64_t prow = (hd * p.S_max + slot) * p.rows_total + cb + r;
          float mr = -INFINITY;
#pragma unroll
          for (int j = 0; j < CH; ++j)
            if (j == r) mr = M[j];
          const float* rs = reds + cb + r;
          p.ws_ml[prow * 2] = mr;
          p.ws_ml[prow * 2 + 1] = (rs[0] + rs[QC]) + (rs[2 * QC] + rs[3 * QC]);
        }
        named_bar_sync(5 + wg, 128);                // the sums are read before the next head's
      }
    }
  }
  griddep_launch();                 // the combine may start launching

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// N = 16 or 32 query columns (at least the rows): a kind::f16 MMA with
// M = 128 takes N in multiples of 16.
static int tct_qc(int64_t rows) { return rows <= 16 ? 16 : 32; }

int cache_attn_tct_ctas_per_sm(int64_t rows) {
  const int qc = tct_qc(rows);
  return qc == 16 ? TCfg<16>::ctas : TCfg<32>::ctas;
}

size_t cache_attn_tct_smem(int64_t rows) {
  const int qc = tct_qc(rows);
  const size_t slack = 1024;      // the dynamic base is rounded up to 1024 bytes
  if (qc == 16) return TSmem<16>::total + (TCfg<16>::ctas > 1 ? 0 : slack);
  return TSmem<32>::total + slack;
}

template <int QC>
static cudaError_t launch_tct(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const DecParams& p, cudaStream_t stream) {
  const size_t smem = cache_attn_tct_smem(p.rows_total);
  cudaError_t e = cudaFuncSetAttribute(cache_attn_tct_kernel<QC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(cache_attn_tct_kernel<QC>, dim3(p.C), dim3(TCfg<QC>::threads), smem, stream, 1, tq, tk, tv, p);
}

cudaError_t launch_cache_attn_tct(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const DecParams& p, cudaStream_t stream) {
  switch (tct_qc(p.rows_total)) {
    case 16: return launch_tct<16>(tq, tk, tv, p, stream);
    default: return launch_tct<32>(tq, tk, tv, p, stream);
  }
}

}  // namespace nectar
