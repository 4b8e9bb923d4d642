// (i) Exact cached-token attention with many query rows per KV head, on the
// tensor cores: Eq. (3.1) of "Nectar: Neural Estimation of Cached-Token
// Attention via Regression" (§2.1) for regression-target generation and
// large decode batches, where the query rows of one (l, h) reuse each
// K / V tile enough times that the contraction, not HBM, bounds the time.
//
// Work: a unit is (KV head, tile of 128 query rows); its n keys are cut into
// 128-key tiles and all units' tiles are laid end to end.  CTA c of C (one
// per SM) takes the contiguous range [c*T/C, (c+1)*T/C): a unit wholly
// inside one range is finished by that CTA (alpha, A written directly); a
// unit cut by range boundaries leaves one (m, l, acc) partial per piece, and
// the combine kernel joins them by log-sum-exp (a separate launch).  A CTA
// can cut at most two units (the first and the last of its range), so the
// partials take two slots per CTA whatever the shape.
//
// Per tile, tcgen05 (kind::f16, cta_group::1, fp32 accumulation in TMEM):
//   S = Q K^T   M = 128 rows, N = 128 keys, K = d    (A, B K-major, SW128)
//   O += P V    M = 128 rows, N = d, K = 128 keys    (P K-major from smem,
//                                                     V MN-major, SW128)
// S is double-buffered in TMEM so S_{j+1} runs while the softmax warps turn
// S_j into P_j.  Softmax keeps a per-row running maximum m and moves it only
// when a tile's maximum exceeds it by more than 2^8; O is then rescaled in
// TMEM (rare), and the final normalisation by the same 2^m makes the result
// the exact quantity.  The row sum l adds the bf16-rounded weights that the
// P V product uses, so A stays a convex combination of the v_j.
//
// Warps: 0..3 softmax / epilogue (thread = query row = TMEM lane),
//        4 TMA producer, 5 MMA issuer and TMEM owner.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

constexpr int kTcRows = 128;     // query rows per unit
constexpr int kTcKeys = 128;     // keys per tile
constexpr int kTcThreads = 192;
constexpr uint32_t kTcTileBytes = 128 * 128 * 2;   // 32 KB: 128 x 128 bf16

struct TcSmem {
  static constexpr uint32_t q = 0;                           // 32 KB
  static constexpr uint32_t k = q + kTcTileBytes;            // 2 x 32 KB
  static constexpr uint32_t v = k + 2 * kTcTileBytes;        // 2 x 32 KB
  static constexpr uint32_t p = v + 2 * kTcTileBytes;        // 2 x 32 KB
  static constexpr uint32_t bars = p + 2 * kTcTileBytes;     // 20 barriers
  static constexpr uint32_t tslot = bars + 20 * 8;
  static constexpr uint32_t total = tslot + 16;
};

__host__ __device__ __forceinline__ int tc_first_cta(int64_t t, int64_t total, int C) {
  return static_cast<int>(((t + 1) * static_cast<int64_t>(C) - 1) / total);
}

// element (row, key) of a K-major SW128 128 x 128 bf16 tile stored as two
// 64-column halves of 128 rows x 128 bytes
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * (128 * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                               ((col & 7) << 1));
}

__global__ void __launch_bounds__(kTcThreads, 1)
cache_attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TcSmem::bars);
  const uint32_t b_qfull = smem_u32(bars + 0), b_qempty = smem_u32(bars + 1);
  const uint32_t b_kfull = smem_u32(bars + 2), b_kempty = smem_u32(bars + 4);     // [2] each
  const uint32_t b_vfull = smem_u32(bars + 6), b_vempty = smem_u32(bars + 8);
  const uint32_t b_sfull = smem_u32(bars + 10), b_sfree = smem_u32(bars + 12);
  const uint32_t b_pfull = smem_u32(bars + 14), b_pvdone = smem_u32(bars + 16);
  const uint32_t b_ofree = smem_u32(bars + 18);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + TcSmem::tslot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(c) * p.total / p.C;
  const int64_t t1 = static_cast<int64_t>(c + 1) * p.total / p.C;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_qempty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_kfull + 8 * s, 1);
      mbar_init(b_kempty + 8 * s, 1);
      mbar_init(b_vfull + 8 * s, 1);
      mbar_init(b_vempty + 8 * s, 1);
      mbar_init(b_sfull + 8 * s, 1);
      mbar_init(b_sfree + 8 * s, 128);
      mbar_init(b_pfull + 8 * s, 128);
      mbar_init(b_pvdone + 8 * s, 1);
    }
    mbar_init(b_ofree, 128);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tmem_o = tmem + 256;

  if (warp == 4) {
    // --------------------------- TMA producer ---------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      const uint64_t pol_kv = policy_evict_first();
      const uint64_t pol_q = policy_evict_last();
      int64_t cur = -1;
      uint32_t qn = 0;
      bool ok = true;
      int64_t jj = 0;
      for (int64_t t = t0; t < t1 && ok; ++t, ++jj) {
        const int64_t u = t / p.tph;
        if (u != cur) {
          if (cur >= 0) ok = mbar_wait(b_qempty, (qn - 1) & 1, p.err);
          if (!ok) break;
          const int64_t hd = u / p.qtiles;
          const int qt = static_cast<int>(u % p.qtiles);
          mbar_arrive_expect_tx(b_qfull, kTcTileBytes);
          tma_load_3d(smem_u32(smem + TcSmem::q), &tmap_q, 0, qt * kTcRows, static_cast<int>(hd), b_qfull, pol_q);
          tma_load_3d(smem_u32(smem + TcSmem::q + kTcTileBytes / 2), &tmap_q, 64, qt * kTcRows, static_cast<int>(hd),
                      b_qfull, pol_q);
          ++qn;
          cur = u;
        }
        const int64_t hd = u / p.qtiles;
        const int key0 = static_cast<int>((t - u * p.tph) * kTcKeys);
        const int s = static_cast<int>(jj & 1);
        const uint32_t ph = static_cast<uint32_t>(((jj >> 1) - 1) & 1);
        if (jj >= 2 && !(ok = mbar_wait(b_kempty + 8 * s, ph, p.err))) break;
        mbar_arrive_expect_tx(b_kfull + 8 * s, kTcTileBytes);
        tma_load_3d(smem_u32(smem + TcSmem::k + s * kTcTileBytes), &tmap_k, 0, key0, static_cast<int>(hd),
                    b_kfull + 8 * s, pol_kv);
        tma_load_3d(smem_u32(smem + TcSmem::k + s * kTcTileBytes + kTcTileBytes / 2), &tmap_k, 64, key0,
                    static_cast<int>(hd), b_kfull + 8 * s, pol_kv);
        if (jj >= 2 && !(ok = mbar_wait(b_vempty + 8 * s, ph, p.err))) break;
        mbar_arrive_expect_tx(b_vfull + 8 * s, kTcTileBytes);
        tma_load_3d(smem_u32(smem + TcSmem::v + s * kTcTileBytes), &tmap_v, 0, key0, static_cast<int>(hd),
                    b_vfull + 8 * s, pol_kv);
        tma_load_3d(smem_u32(smem + TcSmem::v + s * kTcTileBytes + kTcTileBytes / 2), &tmap_v, 64, key0,
                    static_cast<int>(hd), b_vfull + 8 * s, pol_kv);
      }
    }
  } else if (warp == 5) {
    // ---------------------------- MMA issuer ----------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t sq = smem_u32(smem + TcSmem::q);
      bool ok = true;
      uint32_t qn = 0;      // units whose Q has been consumed
      uint32_t un = 0;      // units whose first P V has been issued
      // O += P_x V_x for local tile x; the first P V of a unit starts O
      // from zero, after the epilogue has read the previous unit's O.
      auto issue_pv = [&](int64_t x) {
        const int s = static_cast<int>(x & 1);
        const int64_t tx = t0 + x;
        const bool first = (x == 0) || (tx / p.tph != (tx - 1) / p.tph);
        if (ok) ok = mbar_wait(b_pfull + 8 * s, static_cast<uint32_t>((x >> 1) & 1), p.err);
        if (ok) ok = mbar_wait(b_vfull + 8 * s, static_cast<uint32_t>((x >> 1) & 1), p.err);
        if (ok && first && un > 0) ok = mbar_wait(b_ofree, (un - 1) & 1, p.err);
        if (first) ++un;
        if (!ok) return;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + TcSmem::p + s * kTcTileBytes);
        const uint32_t vb = smem_u32(smem + TcSmem::v + s * kTcTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = P, K-major: keys 16kk.. sit in half kk/4 at byte (kk%4)*32
          const uint64_t ad = sdesc_sw128(pa + (kk >> 2) * (kTcTileBytes / 2) + (kk & 3) * 32, 16, 1024);
          // B = V, MN-major: 16 keys = two 8-row groups of 128 B; the two
          // 64-wide d halves are kTcTileBytes / 2 apart
          const uint64_t bd = sdesc_sw128(vb + kk * 2048, kTcTileBytes / 2, 1024);
          mma_bf16_ss(tmem_o, ad, bd, idesc_o, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(b_vempty + 8 * s);
        mma_commit(b_pvdone + 8 * s);
      };
      int64_t jj = 0;
      for (int64_t t = t0; t < t1 && ok; ++t, ++jj) {
        const int64_t u = t / p.tph;
        const bool unit_first = (t == t0) || (t % p.tph == 0);
        const bool unit_last = (t + 1 == t1) || ((t + 1) % p.tph == 0);
        if (unit_first) {
          ok = mbar_wait(b_qfull, qn & 1, p.err);
          ++qn;
          if (!ok) break;
        }
        (void)u;
        const int s = static_cast<int>(jj & 1);
        if (!(ok = mbar_wait(b_kfull + 8 * s, static_cast<uint32_t>((jj >> 1) & 1), p.err))) break;
        if (jj >= 2 && !(ok = mbar_wait(b_sfree + 8 * s, static_cast<uint32_t>(((jj >> 1) - 1) & 1), p.err))) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + TcSmem::k + s * kTcTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTcTileBytes / 2) + (kk & 3) * 32;
          mma_bf16_ss(tmem + s * 128, sdesc_sw128(sq + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idesc_s,
                      kk != 0);
        }
        mma_commit(b_kempty + 8 * s);
        mma_commit(b_sfull + 8 * s);
        if (unit_last) mma_commit(b_qempty);
        if (jj >= 1) issue_pv(jj - 1);
      }
      if (ok && jj >= 1) issue_pv(jj - 1);
    }
  } else {
    // ------------------------ softmax + epilogue ------------------------
    const int row = (warp & 3) * 32 + lane;              // TMEM lane = query row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float m = -INFINITY, l = 0.f;
    int64_t cur = -1;
    bool ok = true;
    uint32_t on = 0;
    int64_t jj = 0;
    auto finalize = [&](int64_t u, int64_t jlast) {
      // wait for the unit's last P V, then write alpha, A (or a partial)
      const int s = static_cast<int>(jlast & 1);
      if (ok) ok = mbar_wait(b_pvdone + 8 * s, static_cast<uint32_t>((jlast >> 1) & 1), p.err);
      tc_fence_after();
      const int64_t hd = u / p.qtiles;
      const int qt = static_cast<int>(u % p.qtiles);
      const int64_t r = static_cast<int64_t>(qt) * kTcRows + row;
      const int f = tc_first_cta(u * p.tph, p.total, p.C);
      const int la = tc_first_cta(u * p.tph + p.tph - 1, p.total, p.C);
      const bool whole = (f == la);
      float* dst;
      float inv = 1.f;
      if (whole) {
        dst = p.A + (hd * p.rows_total + r) * kD;
        inv = 1.0f / l;
      } else {
        const int slot = (u == t0 / p.tph) ? 0 : 1;    // first or last unit of this CTA's range
        const int64_t prow = (static_cast<int64_t>(c) * 2 + slot) * kTcRows + row;
        dst = p.ws_acc + prow * kD;
        if (r < p.rows_total) {
          p.ws_ml[prow * 2] = m;
          p.ws_ml[prow * 2 + 1] = l;
        }
      }
#pragma unroll
      for (int cb = 0; cb < 128; cb += 32) {
        uint32_t v[32];
        NECTAR_TMEM_LD32(tmem_o + lane_base + cb, v);
        tmem_ld_wait();
        if (ok && r < p.rows_total) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + cb + e) =
                make_float4(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv,
                            __uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
        }
      }
      if (whole && ok && r < p.rows_total) p.alpha[hd * p.rows_total + r] = (m + log2f(l)) * kLn2;
      tc_fence_before();
      mbar_arrive(b_ofree);
      ++on;
    };
    for (int64_t t = t0; t < t1; ++t, ++jj) {
      const int64_t u = t / p.tph;
      if (u != cur) {
        if (cur >= 0) finalize(cur, jj - 1);
        cur = u;
        m = -INFINITY;
        l = 0.f;
      }
      const bool unit_first = (t == t0) || (t % p.tph == 0);
      const int s = static_cast<int>(jj & 1);
      const int nvalid = static_cast<int>(p.n - (t - u * p.tph) * kTcKeys);   // keys of this tile < n
      if (ok) ok = mbar_wait(b_sfull + 8 * s, static_cast<uint32_t>((jj >> 1) & 1), p.err);
      tc_fence_after();
      float sc[128];
#pragma unroll
      for (int cb = 0; cb < 128; cb += 32) {
        uint32_t v[32];
        NECTAR_TMEM_LD32(tmem + s * 128 + lane_base + cb, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) sc[cb + e] = __uint_as_float(v[e]) * p.qmul;
      }
      tc_fence_before();
      mbar_arrive(b_sfree + 8 * s);
      float bm = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; ++e) {
        if (e >= nvalid) sc[e] = -INFINITY;
        bm = fmaxf(bm, sc[e]);
      }
      // Moving the maximum is decided per row, but the TMEM load / store of O
      // is warp-collective (.sync.aligned), so the whole warp takes that path
      // and rows that keep their maximum scale by 1.
      const bool need = bm > m + kRescaleSlack;
      const float corr = need ? exp2_shift(m, bm) : 1.0f;
      if (need) {
        l *= corr;
        m = bm;
      }
      if (__any_sync(0xffffffffu, need) && !unit_first) {
        // O holds the previous tiles of this unit: wait for their last P V,
        // then rescale O in TMEM
        const int64_t jp = jj - 1;
        if (ok) ok = mbar_wait(b_pvdone + 8 * (jp & 1), static_cast<uint32_t>((jp >> 1) & 1), p.err);
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < 128; cb += 32) {
          uint32_t v[32];
          NECTAR_TMEM_LD32(tmem_o + lane_base + cb, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
          NECTAR_TMEM_ST32(tmem_o + lane_base + cb, v);
        }
        tmem_st_wait();
      }
      // P buffer s was last read by the P V of tile jj - 2
      if (jj >= 2 && ok) ok = mbar_wait(b_pvdone + 8 * s, static_cast<uint32_t>(((jj >> 1) - 1) & 1), p.err);
      uint8_t* pt = smem + TcSmem::p + s * kTcTileBytes;
      float rs = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = exp2_shift(sc[c8 * 8 + 2 * e], m);
          const float p1 = exp2_shift(sc[c8 * 8 + 2 * e + 1], m);
          w[e] = pack_bf16x2(p0, p1);
          rs += bf16lo(w[e]) + bf16hi(w[e]);
        }
        *reinterpret_cast<uint4*>(pt + tile_off(row, c8 * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(b_pfull + 8 * s);
    }
    if (cur >= 0) finalize(cur, jj - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One warp per (head, row) of a unit that was cut between CTAs: join its
// partials (units inside one CTA were written by the main kernel).
__global__ void cache_attn_tc_combine_kernel(const TcParams p) {
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<int64_t>(p.heads) * p.rows_total) return;
  const int64_t hd = gw / p.rows_total, r = gw % p.rows_total;
  const int64_t u = hd * p.qtiles + r / kTcRows;
  const int rr = static_cast<int>(r % kTcRows);
  const int f = tc_first_cta(u * p.tph, p.total, p.C);
  const int la = tc_first_cta(u * p.tph + p.tph - 1, p.total, p.C);
  if (f == la) return;
  // the piece of CTA cc sits in slot 0 if u is the first unit of cc's range
  auto prow_of = [&](int cc) {
    const int64_t first_unit = (static_cast<int64_t>(cc) * p.total / p.C) / p.tph;
    return (static_cast<int64_t>(cc) * 2 + (u == first_unit ? 0 : 1)) * kTcRows + rr;
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
  pl.qtiles = static_cast<int>((rows + kTcRows - 1) / kTcRows);
  pl.tph = (n + kTcKeys - 1) / kTcKeys;
  const int64_t units = static_cast<int64_t>(heads) * pl.qtiles;
  pl.total = units * pl.tph;
  int64_t C = num_sms;
  if (C > pl.total) C = pl.total;
  if (C < 1) C = 1;
  pl.C = static_cast<int>(C);
  pl.S_max = 2;    // partial slots per CTA
  pl.ws_bytes = static_cast<size_t>(pl.C) * 2 * kTcRows * (kD + 2) * sizeof(float);
  pl.smem = TcSmem::total + 1024;
  return pl;
}

cudaError_t launch_cache_attn_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const TcParams& p, cudaStream_t stream) {
  const size_t smem = TcSmem::total + 1024;
  cudaError_t e = cudaFuncSetAttribute(cache_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cache_attn_tc_kernel<<<p.C, kTcThreads, smem, stream>>>(tq, tk, tv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t warps = static_cast<int64_t>(p.heads) * p.rows_total;
  const int64_t blocks = (warps * 32 + 255) / 256;
  cache_attn_tc_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace nectar
