// (i) Exact cached-token attention with many query rows per KV head, on the
// tensor cores: Eq. (3.1) of "Nectar: Neural Estimation of Cached-Token
// Attention via Regression" (§2.1), for regression-target generation and
// large decode batches, where the query rows of one (l, h) reuse each K / V
// tile often enough that the contraction, not HBM, bounds the time.
//
// Work unit: (KV head, pair of 128-row query tiles); the pair shares every
// K / V tile, so each byte of K and V brought on chip serves 256 query rows.
// Keys come in tiles of 64.  Units are dealt to the CTAs (one per SM) round
// by round, so the CTAs that work on the query tiles of one head at the same
// time walk its K / V in step and the repeats hit L2; the last one or two
// rounds are cut into equal ranges of key tiles (stream-K) so that every CTA
// ends together.  A unit wholly inside one CTA is finished there (alpha, A
// written directly); a unit cut between CTAs leaves one (m, l, acc) partial
// per piece -- at most two per CTA -- joined by log-sum-exp in a second
// launch, so no CTA ever waits on another.
//
// Per key tile and query tile t (tcgen05 kind::f16, cta_group::1, fp32 in
// TMEM):
//   S_t = Q_t K^T    M = 128, N = 64 keys, K = d     A, B K-major SW128
//   O_t += P_t V     M = 128, N = d, K = 64 keys     P K-major, V MN-major
// S_t is double-buffered in TMEM (S_t of the next tile runs while softmax
// warpgroup t turns this one into bf16 P_t in shared memory, also double-
// buffered).  The running row maximum moves only when a tile's maximum
// exceeds it by more than 2^8; O_t is then rescaled in TMEM (warp-uniform
// decision, as TMEM access is warp-collective), and the final division by
// the same 2^m makes the result exact.  The row sum adds the bf16-rounded
// weights that the P V product uses, so A stays a convex combination.
//
// A unit with one query tile (at most 128 rows left for it) would leave the
// second softmax warpgroup idle; its key range is then split between the
// two warpgroups (interleaved in the K / V ring, both reading query tile
// 0), and warpgroup 1 hands its (m, l, O) to warpgroup 0 through shared
// memory at the end of the unit.  With at most 64 rows (kDup), rows 64..127
// of the query tile repeat rows 0..63, and the thread of row r scores only
// the keys [32 h, 32 h + 32) of each key tile, h = r / 64: P row r holds
// that half's weights and zeros elsewhere, so O rows r and r + 64 are two
// partial states of one query row, joined by log-sum-exp at the end of the
// unit.  Each softmax thread then does half the work of a full tile, none
// of it on padding rows.
//
// Warps: 0..3 softmax / epilogue of query tile 0, 4..7 of tile 1 (thread =
// row = TMEM lane), 8 Q and K producer, 9 V producer, 10 S issuer (and
// TMEM owner), 11 P V issuer.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

constexpr int kTcRows = 128;                       // query rows per tile
constexpr int kTcUnitRows = 2 * kTcRows;           // two tiles per unit
constexpr int kTcKeys = 64;                        // keys per tile
#ifndef NECTAR_TC_POLY_PAIRS
#define NECTAR_TC_POLY_PAIRS 0
#endif
// of every 4 pairs of softmax weights, how many use exp2_poly (0..4); 0:
// measured on B200, moving exponentials to the FMA pipe made the softmax
// slower (the special-function unit is not its limit)
constexpr int kTcPolyPairs = NECTAR_TC_POLY_PAIRS;
constexpr int kTcStages = 3;                       // K and V ring depth
#ifndef NECTAR_TC_PINGPONG
#define NECTAR_TC_PINGPONG 1
#endif
constexpr bool kPingPong = NECTAR_TC_PINGPONG != 0;
constexpr int kPingBar = 4;                         // named barriers 4, 5
constexpr int kTcThreads = 12 * 32;
constexpr uint32_t kQBytes = kTcRows * kD * 2;     // 32 KB
constexpr uint32_t kKVBytes = kTcKeys * kD * 2;    // 16 KB
constexpr uint32_t kPBytes = kTcRows * kTcKeys * 2;   // 16 KB

struct TcSmem {
  static constexpr uint32_t q = 0;                                  // 2 x 32 KB
  static constexpr uint32_t k = q + 2 * kQBytes;                    // 3 x 16 KB
  static constexpr uint32_t v = k + kTcStages * kKVBytes;           // 3 x 16 KB
  static constexpr uint32_t p = v + kTcStages * kKVBytes;           // [tile][buf] 4 x 16 KB
  static constexpr uint32_t xml = p + 4 * kPBytes;                  // split units: (m, l) of warpgroup 1
  static constexpr uint32_t bars = xml + 2 * kTcRows * 4;           // 40 barriers
  static constexpr uint32_t tslot = bars + 40 * 8;
  // K / V ring stage s (s < kTcStages: its own area; s = kTcStages: the
  // second query tile's area, free in the one-query-tile instance)
  static __device__ __forceinline__ uint32_t k_at(int s) { return s < kTcStages ? k + s * kKVBytes : q + kQBytes; }
  static __device__ __forceinline__ uint32_t v_at(int s) {
    return s < kTcStages ? v + s * kKVBytes : q + kQBytes + kKVBytes;
  }
  static constexpr uint32_t total = tslot + 16;
};

__host__ __device__ __forceinline__ int tc_first_cta(int64_t t, int64_t total, int C) {
  return static_cast<int>(((t + 1) * static_cast<int64_t>(C) - 1) / total);
}

// One contiguous piece of a unit's key tiles handled by a CTA.
struct TcSeg {
  int64_t unit;     // global unit index
  int64_t k0, k1;   // key tiles [k0, k1)
  bool whole;       // the CTA does every key tile of the unit
  int slot;         // partial slot when not whole (0: first unit of the CTA's range, 1: last)
};

// CTA c's segments: R data-parallel units c + r*C, then its part of the
// rest: a stream-K range, or (sk_parts = S) the items c and c + C of the
// S * sk_units key parts.
__device__ __forceinline__ int tc_num_segs(const TcParams& p, int c) {
  if (p.sk_parts > 0) {
    const int64_t items = p.sk_units * p.sk_parts;
    return p.dp_rounds + (c < items ? static_cast<int>((items - c + p.C - 1) / p.C) : 0);
  }
  const int64_t Tsk = p.sk_units * p.tph;
  if (Tsk == 0) return p.dp_rounds;
  const int64_t s0 = static_cast<int64_t>(c) * Tsk / p.C, s1 = static_cast<int64_t>(c + 1) * Tsk / p.C;
  if (s1 <= s0) return p.dp_rounds;
  return p.dp_rounds + static_cast<int>((s1 - 1) / p.tph - s0 / p.tph + 1);
}
__device__ __forceinline__ TcSeg tc_seg(const TcParams& p, int c, int i) {
  TcSeg sg;
  if (i < p.dp_rounds) {
    sg.unit = c + static_cast<int64_t>(i) * p.C;
    sg.k0 = 0;
    sg.k1 = p.tph;
    sg.whole = true;
    sg.slot = 0;
    return sg;
  }
  if (p.sk_parts > 0) {
    const int j = i - p.dp_rounds;                       // 0 or 1 (at most 2 items per CTA)
    const int64_t item = c + static_cast<int64_t>(j) * p.C;
    const int64_t part = item / p.sk_units, ul = item % p.sk_units;
    sg.unit = static_cast<int64_t>(p.dp_rounds) * p.C + ul;
    sg.k0 = part * p.tph / p.sk_parts;
    sg.k1 = (part + 1) * p.tph / p.sk_parts;
    sg.whole = p.sk_parts == 1;
    sg.slot = j;
    return sg;
  }
  const int64_t Tsk = p.sk_units * p.tph;
  const int64_t s0 = static_cast<int64_t>(c) * Tsk / p.C, s1 = static_cast<int64_t>(c + 1) * Tsk / p.C;
  const int64_t ul = s0 / p.tph + (i - p.dp_rounds);
  const int64_t b = ul * p.tph;
  sg.unit = static_cast<int64_t>(p.dp_rounds) * p.C + ul;
  sg.k0 = (s0 > b ? s0 : b) - b;
  sg.k1 = (s1 < b + p.tph ? s1 : b + p.tph) - b;
  sg.whole = (sg.k0 == 0 && sg.k1 == p.tph);
  sg.slot = (ul == s0 / p.tph) ? 0 : 1;
  return sg;
}

// The key tiles of a segment in ring order.  With two query tiles every
// key tile serves both softmax warpgroups; with one, warpgroup 0 alone --
// unless the segment has two or more key tiles: then the warpgroups take
// the two halves of its range (split), interleaved in the ring, and merge
// their partial states at the end.  All roles walk the same sequence.
struct TcItem {
  int64_t kt;        // key tile
  uint32_t mask;     // bit t: consumed by softmax warpgroup t
  bool first;        // first key tile of this segment for the warpgroup(s)
};
template <bool kSplit>
__device__ __forceinline__ bool tc_split(const TcSeg& sg, bool two) { return kSplit && !two && sg.k1 - sg.k0 >= 2; }
template <bool kSplit>
__device__ __forceinline__ TcItem tc_item(const TcSeg& sg, bool two, int64_t i) {
  TcItem it;
  if (!tc_split<kSplit>(sg, two)) {
    it.kt = sg.k0 + i;
    it.mask = two ? 3u : 1u;
    it.first = i == 0;
    return it;
  }
  const int64_t n0 = (sg.k1 - sg.k0 + 1) / 2;     // warpgroup 0: [k0, k0 + n0), 1: the rest
  const int64_t pair = i >> 1;
  if (i & 1) {
    it.kt = sg.k0 + n0 + pair;
    it.mask = 2u;
  } else {
    it.kt = sg.k0 + pair;
    it.mask = 1u;
  }
  it.first = pair == 0;
  return it;
}

// element (row, key) of a K-major SW128 tile of 128 rows x 64 keys
__device__ __forceinline__ uint32_t p_off(int row, int col) {
  return static_cast<uint32_t>(row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

// End of a unit for softmax warpgroup t, once its last P V is complete:
// the split hand-off (split units) and the output -- alpha and A, or the
// partial (m, l, acc) of a unit cut between CTAs.  tO: this thread's TMEM
// lane of O_t.
template <bool kSplit>
__device__ __forceinline__ void tc_unit_epilogue(const TcParams& p, uint8_t* smem, uint32_t tO, uint32_t b_ofree_t,
                                              const TcSeg& sg, bool split_, int t, int row, float m, float l, bool ok,
                                              int c) {
  const bool split = kSplit && split_;
  // split unit: warpgroup 1 parks its O rows in the P buffers (free once
  // both warpgroups' last P V is done; 16-byte chunks swizzled by row)
  // and its (m, l); warpgroup 0 joins the two states by log-sum-exp
  float4* xo = reinterpret_cast<float4*>(smem + TcSmem::p) + row * (kD / 4);
  float* xml = reinterpret_cast<float*>(smem + TcSmem::xml);
  float w0 = 1.f, w1 = 0.f;
  if (split) {
    named_bar_sync(1, 2 * kTcRows);
    if (t == 1) {
#pragma unroll
      for (int cb = 0; cb < kD; cb += 16) {
        uint32_t v[16];
        NECTAR_TMEM_LD16(tO + cb, v);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          xo[((cb >> 2) + q4) ^ (row & 31)] =
              make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                          __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
      }
      xml[row] = m;
      xml[kTcRows + row] = l;
      tc_fence_before();
      mbar_arrive(b_ofree_t);
      named_bar_sync(1, 2 * kTcRows);   // parked
      named_bar_sync(1, 2 * kTcRows);   // read by warpgroup 0: the P buffers are free again
      return;
    }
    named_bar_sync(1, 2 * kTcRows);     // warpgroup 1's state is parked
    const float m1 = xml[row], l1 = xml[kTcRows + row];
    const float M = fmaxf(m, m1);
    w0 = exp2_shift(m, M);
    w1 = exp2_shift(m1, M);
    l = w0 * l + w1 * l1;
    m = M;
  }
  const int64_t hd = sg.unit / p.qpairs;
  const int64_t qp = sg.unit % p.qpairs;
  const int64_t r = qp * kTcUnitRows + t * kTcRows + row;
  float* dst;
  float inv = 1.f;
  if (sg.whole) {
    dst = p.A + (hd * p.rows_total + r) * kD;
    inv = 1.0f / l;
  } else {
    const int64_t prow = (static_cast<int64_t>(c) * 2 + sg.slot) * kTcUnitRows + t * kTcRows + row;
    dst = p.ws_acc + prow * kD;
    if (r < p.rows_total) {
      p.ws_ml[prow * 2] = m;
      p.ws_ml[prow * 2 + 1] = l;
    }
  }
#pragma unroll
  for (int cb = 0; cb < kD; cb += 16) {
    uint32_t v[16];
    NECTAR_TMEM_LD16(tO + cb, v);
    tmem_ld_wait();
    if (ok && r < p.rows_total) {
#pragma unroll
      for (int e = 0; e < 16; e += 4) {
        float4 o = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                               __uint_as_float(v[e + 3]));
        if (split) {
          const float4 o1 = xo[((cb + e) >> 2) ^ (row & 31)];
          o = make_float4(w0 * o.x + w1 * o1.x, w0 * o.y + w1 * o1.y, w0 * o.z + w1 * o1.z, w0 * o.w + w1 * o1.w);
        }
        *reinterpret_cast<float4*>(dst + cb + e) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      }
    }
  }
  if (sg.whole && ok && r < p.rows_total) p.alpha[hd * p.rows_total + r] = (m + log2f(l)) * kLn2;
  tc_fence_before();
  mbar_arrive(b_ofree_t);
  if (split) named_bar_sync(1, 2 * kTcRows);   // done with the parked state
}

// The split instance out of line: inlined, its hand-off makes the softmax
// loop spill; the other instance inlines it with no spill.
__device__ __noinline__ void tc_unit_epilogue_split(const TcParams& p, uint8_t* smem, uint32_t tO, uint32_t b_ofree_t,
                                                    const TcSeg& sg, bool split, int t, int row, float m, float l,
                                                    bool ok, int c) {
  tc_unit_epilogue<true>(p, smem, tO, b_ofree_t, sg, split, t, row, m, l, ok, c);
}

// kDup, end of a unit for softmax warpgroup t (its last P V complete):
// fold row r + 64's partial state (the keys of the second half) into row
// r -- its O row and (m, l) through this warpgroup's own P buffers (free
// now), then log-sum-exp.  Returns row r's joined (m, l); O rows 0..63 of
// the tile hold the joined state.  Out of line, as the split hand-off: it
// would take registers from the softmax loop.
__device__ __noinline__ float2 tc_dup_fold(uint8_t* smem, uint32_t tO, int t, int row, float m, float l) {
  float4* park = reinterpret_cast<float4*>(smem + TcSmem::p + 2 * t * kPBytes);   // 64 rows x 512 B
  float* xm = reinterpret_cast<float*>(smem + TcSmem::xml) + t * kTcRows;
  const int q = row & 63;
  if (row >= 64) {
#pragma unroll
    for (int cb = 0; cb < kD; cb += 16) {
      uint32_t v[16];
      NECTAR_TMEM_LD16(tO + cb, v);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        park[q * (kD / 4) + (((cb >> 2) + q4) ^ (q & 31))] =
            make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]), __uint_as_float(v[4 * q4 + 2]),
                        __uint_as_float(v[4 * q4 + 3]));
    }
    xm[q] = m;
    xm[64 + q] = l;
  }
  named_bar_sync(2 + t, kTcRows);
  if (row < 64) {
    const float m1 = xm[q], l1 = xm[64 + q];
    const float M = fmaxf(m, m1);
    const float w0 = exp2_shift(m, M), w1 = exp2_shift(m1, M);
    l = w0 * l + w1 * l1;
    m = M;
#pragma unroll
    for (int cb = 0; cb < kD; cb += 32) {
      uint32_t v[32];
      NECTAR_TMEM_LD32(tO + cb, v);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 o1 = park[q * (kD / 4) + (((cb >> 2) + q4) ^ (q & 31))];
        v[4 * q4] = __float_as_uint(w0 * __uint_as_float(v[4 * q4]) + w1 * o1.x);
        v[4 * q4 + 1] = __float_as_uint(w0 * __uint_as_float(v[4 * q4 + 1]) + w1 * o1.y);
        v[4 * q4 + 2] = __float_as_uint(w0 * __uint_as_float(v[4 * q4 + 2]) + w1 * o1.z);
        v[4 * q4 + 3] = __float_as_uint(w0 * __uint_as_float(v[4 * q4 + 3]) + w1 * o1.w);
      }
      NECTAR_TMEM_ST32(tO + cb, v);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  named_bar_sync(2 + t, kTcRows);       // the parked rows are read
  tc_fence_after();
  return make_float2(m, l);
}

// kSplit: units with one query tile split their keys between the two
// softmax warpgroups (compiled only into the instance used when every unit
// has one query tile: the hand-off costs registers)
template <bool kSplit, bool kDup>
__global__ void __launch_bounds__(kTcThreads, 1)
cache_attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TcSmem::bars);
  const uint32_t b_qfull = smem_u32(bars + 0), b_qempty = smem_u32(bars + 1);
  // K / V ring depth: one more stage in the one-query-tile instance, in the
  // unused second query tile (a head of <= 128 rows streams its K / V at
  // HBM speed there, so more bytes in flight)
  constexpr int kSt = kSplit ? kTcStages + 1 : kTcStages;
  const uint32_t b_kfull = smem_u32(bars + 2), b_kempty = smem_u32(bars + 6);     // [4]
  const uint32_t b_vfull = smem_u32(bars + 10), b_vempty = smem_u32(bars + 14);   // [4]
  // [tile t][buf b] at + 8 * (2 t + b)
  const uint32_t b_sfull = smem_u32(bars + 18), b_sfree = smem_u32(bars + 22);
  const uint32_t b_pfull = smem_u32(bars + 26), b_pvdone = smem_u32(bars + 30);
  const uint32_t b_ofree = smem_u32(bars + 34);                                   // [tile]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + TcSmem::tslot);

  static_assert(kSplit || !kDup, "repeated rows only in the one-query-tile instance");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int nseg = tc_num_segs(p, c);

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_qempty, 1);
    for (int s = 0; s < kSt; ++s) {
      mbar_init(b_kfull + 8 * s, 1);
      mbar_init(b_kempty + 8 * s, 1);
      mbar_init(b_vfull + 8 * s, 1);
      mbar_init(b_vempty + 8 * s, 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(b_sfull + 8 * i, 1);
      mbar_init(b_sfree + 8 * i, 128);
      mbar_init(b_pfull + 8 * i, 128);
      mbar_init(b_pvdone + 8 * i, 1);
    }
    mbar_init(b_ofree + 0, 128);
    mbar_init(b_ofree + 8, 128);
    fence_barrier_init();
  }
  if (warp == 10) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // TMEM columns: S[t][b] at 128 t + 64 b, O[t] at 256 + 128 t

  auto two_tiles = [&](int64_t unit) {
    const int64_t qp = unit % p.qpairs;
    return qp * kTcUnitRows + kTcRows < p.rows_total;
  };

  if (warp == 8) {
    // ----------------------- Q and K producer -----------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      const uint64_t pol_kv = policy_evict_normal();
      const uint64_t pol_q = policy_evict_first();
      bool ok = true;
      uint32_t qn = 0, it = 0;
      for (int si = 0; si < nseg && ok; ++si) {
        const TcSeg sg = tc_seg(p, c, si);
        const int64_t hd = sg.unit / p.qpairs;
        const int qp = static_cast<int>(sg.unit % p.qpairs);
        if (qn > 0 && !(ok = mbar_wait(b_qempty, (qn - 1) & 1, p.err))) break;
        const bool two = two_tiles(sg.unit);
        mbar_arrive_expect_tx(b_qfull, (two ? 2 : 1) * kQBytes);
        if constexpr (kDup) {
          // rows 0..63 of each 64-column half, twice (box: 64 rows, one half)
#pragma unroll
          for (int hq = 0; hq < 4; ++hq)
            tma_load_4d(smem_u32(smem + TcSmem::q + hq * (kQBytes / 4)), &tmap_q, 0, qp * kTcUnitRows, hq >> 1,
                        static_cast<int>(hd), b_qfull, pol_q);
        } else {
          tma_load_4d(smem_u32(smem + TcSmem::q), &tmap_q, 0, qp * kTcUnitRows, 0, static_cast<int>(hd), b_qfull,
                      pol_q);
        }
        if (two)
          tma_load_4d(smem_u32(smem + TcSmem::q + kQBytes), &tmap_q, 0, qp * kTcUnitRows + kTcRows, 0,
                      static_cast<int>(hd), b_qfull, pol_q);
        ++qn;
        for (int64_t i = 0; i < sg.k1 - sg.k0; ++i, ++it) {
          const int64_t kt = tc_item<kSplit>(sg, two, i).kt;
          const uint32_t s = it % kSt;
          if (it >= kSt && !(ok = mbar_wait(b_kempty + 8 * s, ((it / kSt) - 1) & 1, p.err))) break;
          mbar_arrive_expect_tx(b_kfull + 8 * s, kKVBytes);
          tma_load_4d(smem_u32(smem + TcSmem::k_at(s)), &tmap_k, 0, static_cast<int>(kt * kTcKeys), 0,
                      static_cast<int>(hd), b_kfull + 8 * s, pol_kv);
        }
      }
    }
  } else if (warp == 9) {
    // --------------------------- V producer ---------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_v);
      const uint64_t pol_kv = policy_evict_normal();
      bool ok = true;
      uint32_t it = 0;
      for (int si = 0; si < nseg && ok; ++si) {
        const TcSeg sg = tc_seg(p, c, si);
        const int64_t hd = sg.unit / p.qpairs;
        const bool two = two_tiles(sg.unit);
        for (int64_t i = 0; i < sg.k1 - sg.k0; ++i, ++it) {
          const int64_t kt = tc_item<kSplit>(sg, two, i).kt;
          const uint32_t s = it % kSt;
          if (it >= kSt && !(ok = mbar_wait(b_vempty + 8 * s, ((it / kSt) - 1) & 1, p.err))) break;
          mbar_arrive_expect_tx(b_vfull + 8 * s, kKVBytes);
          tma_load_4d(smem_u32(smem + TcSmem::v_at(s)), &tmap_v, 0, static_cast<int>(kt * kTcKeys), 0,
                      static_cast<int>(hd), b_vfull + 8 * s, pol_kv);
        }
      }
    }
  } else if (warp == 10) {
    // ---------------------- S issuer (+ TMEM owner) ----------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kTcKeys, 0, 0);
      bool ok = true;
      uint32_t qn = 0, it = 0;
      uint32_t cs[2] = {0, 0};   // S tiles issued per query tile
      for (int si = 0; si < nseg && ok; ++si) {
        const TcSeg sg = tc_seg(p, c, si);
        const bool two = two_tiles(sg.unit);
        ok = mbar_wait(b_qfull, qn & 1, p.err);
        ++qn;
        const int64_t nit = sg.k1 - sg.k0;
        for (int64_t i = 0; i < nit && ok; ++i, ++it) {
          const TcItem itm = tc_item<kSplit>(sg, two, i);
          const uint32_t ks = it % kSt;
          if (!(ok = mbar_wait(b_kfull + 8 * ks, (it / kSt) & 1, p.err))) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (!(itm.mask >> t & 1u)) continue;
            const uint32_t b = cs[t] & 1;
            if (cs[t] >= 2 && !(ok = mbar_wait(b_sfree + 8 * (2 * t + b), ((cs[t] >> 1) - 1) & 1, p.err))) break;
            tc_fence_after();
            // one query tile (split or not): both warpgroups read tile 0
            const uint32_t qa = smem_u32(smem + TcSmem::q + (two ? t : 0) * kQBytes);
            const uint32_t kb = smem_u32(smem + TcSmem::k_at(ks));
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // d 16 kk..: half kk / 4, byte (kk % 4) * 32 inside the 128-B rows
              mma_bf16_ss(tmem + 128 * t + 64 * b,
                          sdesc_sw128(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024),
                          sdesc_sw128(kb + (kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32, 16, 1024), idesc_s, kk != 0);
            }
            mma_commit(b_sfull + 8 * (2 * t + b));
            ++cs[t];
          }
          mma_commit(b_kempty + 8 * ks);
          if (i + 1 == nit) mma_commit(b_qempty);
        }
      }
    }
  } else if (warp == 11) {
    // ----------------------------- P V issuer -----------------------------
    // A thread of its own, so that the S of the next key tiles is issued as
    // soon as its K tile and S buffer are there, not behind a softmax (a
    // per-tile timeline showed the softmax warpgroups waiting 0.95 us of
    // each 1.76 us tile for their S while one thread issued both products).
    if (lane == 0) {
      const uint32_t idesc_o = idesc_bf16_f32(128, kD, 0, 1);
      bool ok = true;
      uint32_t it = 0;
      uint32_t cp[2] = {0, 0};   // P V products issued per query tile
      uint32_t un[2] = {0, 0};   // units whose O was started, per query tile
      for (int si = 0; si < nseg && ok; ++si) {
        const TcSeg sg = tc_seg(p, c, si);
        const bool two = two_tiles(sg.unit);
        for (int64_t i = 0; i < sg.k1 - sg.k0 && ok; ++i, ++it) {
          const TcItem itm = tc_item<kSplit>(sg, two, i);
          const bool first = itm.first;
          // O_t += P_t V for the ring entry `it`, for every warpgroup t in the mask
          const uint32_t vs = it % kSt;
          if (ok) ok = mbar_wait(b_vfull + 8 * vs, (it / kSt) & 1, p.err);
          for (int t = 0; t < 2; ++t) {
            if (!(itm.mask >> t & 1u)) continue;
            const uint32_t b = cp[t] & 1;
            if (ok) ok = mbar_wait(b_pfull + 8 * (2 * t + b), (cp[t] >> 1) & 1, p.err);
            if (ok && first && un[t] > 0) ok = mbar_wait(b_ofree + 8 * t, (un[t] - 1) & 1, p.err);
            if (first) ++un[t];
            ++cp[t];
            if (!ok) continue;
            tc_fence_after();
            const uint32_t pa = smem_u32(smem + TcSmem::p + (2 * t + b) * kPBytes);
            const uint32_t vb = smem_u32(smem + TcSmem::v_at(vs));
#pragma unroll
            for (int kk = 0; kk < kTcKeys / 16; ++kk) {
              // A = P (K-major, one 64-key chunk): keys 16 kk.. at byte 32 kk.
              // B = V (MN-major): 16 keys = two 8-row groups of 128 B; the two
              // 64-wide d halves are kKVBytes / 2 apart
              mma_bf16_ss(tmem + 256 + 128 * t, sdesc_sw128(pa + kk * 32, 16, 1024),
                          sdesc_sw128(vb + kk * 2048, kKVBytes / 2, 1024), idesc_o, (first && kk == 0) ? 0u : 1u);
            }
            mma_commit(b_pvdone + 8 * (2 * t + b));
          }
          mma_commit(b_vempty + 8 * vs);
        }
      }
    }
  } else {
    // --------------------- softmax + epilogue (tile t) ---------------------
    const int t = warp >> 2;
    const int row = (warp & 3) * 32 + lane;               // TMEM lane = row of the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * t, tO = tmem + 256 + 128 * t;
    bool ok = true;
    uint32_t cnt = 0;   // S tiles consumed by this tile
    for (int si = 0; si < nseg; ++si) {
      const TcSeg sg = tc_seg(p, c, si);
      const bool two = two_tiles(sg.unit);
      const bool split = tc_split<kSplit>(sg, two);
      if (t == 1 && !two && !split) continue;
      // two query tiles: the warpgroups take turns at the exponentials of a
      // key tile (warpgroup 0 first), so that one's run on the special-
      // function unit overlaps the other's maximum, stores and waits
      const bool pp = kPingPong && two;
      const int64_t nk = sg.k1 - sg.k0;
      float m = -INFINITY, l = 0.f;
      for (int64_t i = 0; i < sg.k1 - sg.k0; ++i) {
        const TcItem itm = tc_item<kSplit>(sg, two, i);
        if (!(itm.mask >> t & 1u)) continue;
        const int64_t kt = itm.kt;
        const uint32_t ci = cnt++;               // this warpgroup's S tiles so far
        const uint32_t b = ci & 1;
        const int64_t nvalid = p.n - kt * kTcKeys;
        if (ok) ok = mbar_wait(b_sfull + 8 * (2 * t + b), (ci >> 1) & 1, p.err);
        tc_fence_after();
        // a whole tile of valid keys (every tile but a head's last): keep
        // the raw scores, take the max on them and fold the scale into the
        // exponent's FMA; the last tile scales and masks element by element.
        // kDup: this thread's columns are the 32 keys of its half hh.
        constexpr int kCols = kDup ? kTcKeys / 2 : kTcKeys;
        const int hh = kDup ? (row >> 6) : 0;
        const int64_t nv = nvalid - hh * kCols;          // valid keys among this thread's columns
        const bool full = nv >= kCols;
        float sc[kCols];
        {
          // every load of the tile issued before the one wait
          uint32_t v[kCols];
#pragma unroll
          for (int cb = 0; cb < kCols; cb += 32) NECTAR_TMEM_LD32(tS + 64 * b + lane_base + hh * kCols + cb, (v + cb));
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < kCols; ++e) sc[e] = __uint_as_float(v[e]);
        }
        tc_fence_before();
        mbar_arrive(b_sfree + 8 * (2 * t + b));
        float bm = -INFINITY;
        if (full) {
          // two independent chains (a 64-deep dependent chain would expose
          // its latency on every tile)
          float x0 = sc[0], x1 = sc[1];
          if (p.qmul >= 0.f) {
#pragma unroll
            for (int e = 2; e < kCols; e += 2) {
              x0 = fmaxf(x0, sc[e]);
              x1 = fmaxf(x1, sc[e + 1]);
            }
            bm = fmaxf(x0, x1) * p.qmul;
          } else {
#pragma unroll
            for (int e = 2; e < kCols; e += 2) {
              x0 = fminf(x0, sc[e]);
              x1 = fminf(x1, sc[e + 1]);
            }
            bm = fminf(x0, x1) * p.qmul;
          }
        } else {
#pragma unroll
          for (int e = 0; e < kCols; ++e) {
            sc[e] = (e < nv) ? sc[e] * p.qmul : -INFINITY;
            bm = fmaxf(bm, sc[e]);
          }
        }
        const bool need = bm > m + kRescaleSlack;
        const float corr = need ? exp2_shift(m, bm) : 1.0f;
        if (need) {
          l *= corr;
          m = bm;
        }
        if (__any_sync(0xffffffffu, need) && !itm.first) {
          // O_t holds the earlier key tiles of this unit: wait for their
          // last P V, then rescale it in TMEM (warp-collective)
          const uint32_t pc = ci - 1;
          if (ok) ok = mbar_wait(b_pvdone + 8 * (2 * t + (pc & 1)), (pc >> 1) & 1, p.err);
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < kD; cb += 32) {
            uint32_t v[32];
            NECTAR_TMEM_LD32(tO + lane_base + cb, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
            NECTAR_TMEM_ST32(tO + lane_base + cb, v);
          }
          tmem_st_wait();
        }
        // P buffer b was last read by the P V of this warpgroup's S tile ci - 2
        if (ci >= 2 && ok) ok = mbar_wait(b_pvdone + 8 * (2 * t + b), ((ci >> 1) - 1) & 1, p.err);
        uint8_t* pt = smem + TcSmem::p + (2 * t + b) * kPBytes;
        float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if (pp) {
          // warpgroup 0 waits for warpgroup 1's exponentials of the previous
          // key tile, warpgroup 1 for warpgroup 0's of this one
          if (t == 1) named_bar_sync(kPingBar + 1, 2 * kTcRows);
          else if (i > 0) named_bar_sync(kPingBar, 2 * kTcRows);
        }
        // the row sum adds the rounded weights that P V uses; full tiles and
        // the last (masked) tile in separate loops, so that the unrolled
        // loop body carries no per-pair branch
        const int col0 = hh * kCols;
        if (full) {
          const float2 q2 = make_float2(p.qmul, p.qmul), nm2 = make_float2(-m, -m);
#pragma unroll
          for (int c8 = 0; c8 < kCols / 8; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              // 2^(s * scale * log2 e - m) for two keys: one paired FMA; the
              // last kTcPolyPairs of every 4 pairs take the polynomial exp2
              const float2 x = ffma2(make_float2(sc[c8 * 8 + 2 * e], sc[c8 * 8 + 2 * e + 1]), q2, nm2);
              if (e >= 4 - kTcPolyPairs) w[e] = pack_bf16x2(exp2_poly(x.x), exp2_poly(x.y));
              else w[e] = pack_bf16x2(ex2(x.x), ex2(x.y));
              rs2[e & 1] = fadd2(rs2[e & 1], make_float2(bf16lo(w[e]), bf16hi(w[e])));
            }
            *reinterpret_cast<uint4*>(pt + p_off(row, col0 + c8 * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
#pragma unroll
          for (int c8 = 0; c8 < kCols / 8; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              w[e] = pack_bf16x2(exp2_shift(sc[c8 * 8 + 2 * e], m), exp2_shift(sc[c8 * 8 + 2 * e + 1], m));
              rs2[e & 1] = fadd2(rs2[e & 1], make_float2(bf16lo(w[e]), bf16hi(w[e])));
            }
            *reinterpret_cast<uint4*>(pt + p_off(row, col0 + c8 * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        if (pp) {
          if (t == 0) named_bar_arrive(kPingBar + 1, 2 * kTcRows);
          else if (i + 1 < nk) named_bar_arrive(kPingBar, 2 * kTcRows);
        }
        if constexpr (kDup) {
          // the other half's keys carry no weight in this row
#pragma unroll
          for (int c8 = 0; c8 < kCols / 8; ++c8)
            *reinterpret_cast<uint4*>(pt + p_off(row, (kCols - col0) + c8 * 8)) = make_uint4(0, 0, 0, 0);
        }
        l += (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_pfull + 8 * (2 * t + b));
      }
      // ------------- epilogue of this unit for tile t -------------
      const uint32_t pc = cnt - 1;
      if (ok) ok = mbar_wait(b_pvdone + 8 * (2 * t + (pc & 1)), (pc >> 1) & 1, p.err);
      tc_fence_after();
      if constexpr (kDup) {
        const float2 ml = tc_dup_fold(smem, tO + lane_base, t, row, m, l);
        m = ml.x;
        l = ml.y;
      }
      if constexpr (kSplit) {
        tc_unit_epilogue_split(p, smem, tmem + 256 + 128 * t + lane_base, b_ofree + 8 * t, sg, split, t, row, m, l,
                               ok, c);
      } else {
        tc_unit_epilogue<false>(p, smem, tmem + 256 + 128 * t + lane_base, b_ofree + 8 * t, sg, split, t, row, m, l,
                                ok, c);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One warp per (head, row) of a stream-K unit that was cut between CTAs:
// join its partials (every other unit was written by the main kernel).
__global__ void cache_attn_tc_combine_kernel(const TcParams p) {
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<int64_t>(p.heads) * p.rows_total) return;
  const int64_t hd = gw / p.rows_total, r = gw % p.rows_total;
  const int64_t unit = hd * p.qpairs + r / kTcUnitRows;
  const int rr = static_cast<int>(r % kTcUnitRows);
  const int64_t ul = unit - static_cast<int64_t>(p.dp_rounds) * p.C;   // stream-K local unit
  if (ul < 0) return;
  if (p.sk_parts > 0) {
    // the S key parts of the unit: item part * sk_units + ul, on CTA item % C, slot item / C
    if (p.sk_parts == 1) return;
    const int S = p.sk_parts;
    auto prow_at = [&](int part) {
      const int64_t item = part * p.sk_units + ul;
      return ((item % p.C) * 2 + item / p.C) * kTcUnitRows + rr;
    };
    float M = -INFINITY;
    for (int q = 0; q < S; ++q) M = fmaxf(M, p.ws_ml[prow_at(q) * 2]);
    float ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < S; ++q) {
      const int64_t prow = prow_at(q);
      const float w = exp2_shift(p.ws_ml[prow * 2], M);
      ls = fmaf(p.ws_ml[prow * 2 + 1], w, ls);
      const float4 a4 = reinterpret_cast<const float4*>(p.ws_acc + prow * kD)[lane];
      acc.x = fmaf(a4.x, w, acc.x);
      acc.y = fmaf(a4.y, w, acc.y);
      acc.z = fmaf(a4.z, w, acc.z);
      acc.w = fmaf(a4.w, w, acc.w);
    }
    const float inv = 1.0f / ls;
    reinterpret_cast<float4*>(p.A + gw * kD)[lane] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (lane == 0) p.alpha[gw] = (M + log2f(ls)) * kLn2;
    return;
  }
  const int64_t Tsk = p.sk_units * p.tph;
  const int f = tc_first_cta(ul * p.tph, Tsk, p.C);
  const int la = tc_first_cta(ul * p.tph + p.tph - 1, Tsk, p.C);
  if (f == la) return;
  // the piece of CTA cc sits in slot 0 if ul is the first unit of cc's range
  auto prow_of = [&](int cc) {
    const int64_t first = (static_cast<int64_t>(cc) * Tsk / p.C) / p.tph;
    return (static_cast<int64_t>(cc) * 2 + (ul == first ? 0 : 1)) * kTcUnitRows + rr;
  };
  float M = -INFINITY;
  for (int cc = f; cc <= la; ++cc) M = fmaxf(M, p.ws_ml[prow_of(cc) * 2]);
  float ls = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int cc = f; cc <= la; ++cc) {
    const int64_t prow = prow_of(cc);
    const float w = exp2_shift(p.ws_ml[prow * 2], M);
    ls = fmaf(p.ws_ml[prow * 2 + 1], w, ls);
    const float4 a4 = reinterpret_cast<const float4*>(p.ws_acc + prow * kD)[lane];
    acc.x = fmaf(a4.x, w, acc.x);
    acc.y = fmaf(a4.y, w, acc.y);
    acc.z = fmaf(a4.z, w, acc.z);
    acc.w = fmaf(a4.w, w, acc.w);
  }
  const float inv = 1.0f / ls;
  reinterpret_cast<float4*>(p.A + gw * kD)[lane] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lane == 0) p.alpha[gw] = (M + log2f(ls)) * kLn2;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
TcPlan plan_tc(int heads, int64_t n, int64_t rows, int num_sms) {
  TcPlan pl{};
  pl.qpairs = static_cast<int>((rows + kTcUnitRows - 1) / kTcUnitRows);
  pl.tph = (n + kTcKeys - 1) / kTcKeys;
  const int64_t units = static_cast<int64_t>(heads) * pl.qpairs;
  int64_t C = num_sms;
  if (C > units * pl.tph) C = units * pl.tph;
  if (C < 1) C = 1;
  pl.C = static_cast<int>(C);
  // Whole rounds of units first: unit c + r C on CTA c, so the CTAs of a
  // head's query units read its K / V in step and L2 serves all but the
  // first of them.  The rest, two ways:
  //  - lockstep (heads of several query units): every whole round, then
  //    each remaining unit cut into S equal key parts, item p * U + u on CTA
  //    item % C (one or two items per CTA).  The query units of a head then
  //    read each key part at the same time too.  S minimises the longest
  //    CTA's tiles; taken while that is within 10 % of the even cut below.
  //  - stream-K: one round fewer when the units do not divide, and the
  //    rest (C to 2C units) cut into C equal ranges of key tiles.  Each unit
  //    is then read at staggered times by its CTAs, from DRAM each time
  //    (measured on a 4-layer Qwen3-4B target capture: 7.19 GB of DRAM
  //    reads for 1.0 GB of K / V).
  int64_t R = units / C;
  const int64_t rest = units - R * C;
  int best_s = 0;
  if (pl.qpairs > 1 && rest > 0) {
    const int64_t even = (rest * pl.tph + C - 1) / C;
    int64_t best = 0;
    for (int64_t S = 1; S <= pl.tph && S * rest <= 2 * C; ++S) {
      const int64_t cost = ((S * rest + C - 1) / C) * ((pl.tph + S - 1) / S);
      if (best_s == 0 || cost < best) {
        best = cost;
        best_s = static_cast<int>(S);
      }
    }
    if (best_s > 0 && best * 10 > even * 11) best_s = 0;
  }
  if (best_s == 0 && rest != 0 && R > 0) R -= 1;
  pl.dp_rounds = static_cast<int>(R);
  pl.sk_units = units - R * C;
  pl.sk_parts = best_s;
  pl.ws_bytes = static_cast<size_t>(pl.C) * 2 * kTcUnitRows * (kD + 2) * sizeof(float);
  pl.smem = TcSmem::total + 1024;
  return pl;
}

// At most 64 rows per head: the one-query-tile instance with the rows
// repeated and the keys of each tile halved between a row's two threads.
// NECTAR_TC_DUP=0 keeps one thread per row over all 64 keys of a tile.
bool cache_attn_tc_dup(int64_t rows) {
  const char* e = getenv("NECTAR_TC_DUP");
  return rows <= kTcRows / 2 && !(e != nullptr && e[0] == '0');
}

template <bool kSplit, bool kDup>
static cudaError_t launch_tc_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const TcParams& p,
                               size_t smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(cache_attn_tc_kernel<kSplit, kDup>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cache_attn_tc_kernel<kSplit, kDup><<<p.C, kTcThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_cache_attn_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const TcParams& p, cudaStream_t stream) {
  const size_t smem = TcSmem::total + 1024;
  // every unit has one query tile when a head has at most 128 rows; the
  // query tensor map's box is 64 rows when the rows are repeated
  const bool split = p.rows_total <= kTcRows;
  cudaError_t e = !split ? launch_tc_t<false, false>(tq, tk, tv, p, smem, stream)
                  : cache_attn_tc_dup(p.rows_total) ? launch_tc_t<true, true>(tq, tk, tv, p, smem, stream)
                                                    : launch_tc_t<true, false>(tq, tk, tv, p, smem, stream);
  if (e != cudaSuccess) return e;
  if (p.sk_units == 0 || p.sk_parts == 1) return cudaSuccess;
  const int64_t warps = static_cast<int64_t>(p.heads) * p.rows_total;
  const int64_t blocks = (warps * 32 + 255) / 256;
  cache_attn_tc_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace nectar
