// Exact causal local attention on the tensor cores, for many query tokens:
// the local half of Eq. (3.4) of "Nectar: Neural Estimation of Cached-Token
// Attention via Regression" (§2.2) -- Z_local, N_local and their running
// maximum for every query row -- optionally merged at once with a document
// term (a, A_doc) as in Eqs. (3.4)-(3.5).
//
// A job is (KV head, query token i): its G query heads see the same keys,
// the visible prefix of the token's local cache.  Per 128-key tile,
//   S = Q K^T   (tcgen05, M = 128 query rows of which the first G are real,
//                N = 128 keys, K = d; Q and K K-major, 128-byte swizzle),
//   P = 2^(S * scale * log2 e - m)   (one thread per query row, TMEM lane),
//   O += P V    (M = 128 rows, N = d, K = 128 keys; V MN-major),
// with S and O in TMEM.  Most of M is idle -- the rows of a job are its G
// heads -- but a tile's tensor time stays far below the time its 64 KB of
// K and V take to arrive from HBM, and the softmax needs no cross-thread
// reduction at all.  Keys past the visible count are masked to -inf; rows
// >= G are computed on stale shared memory and never read.
//
// Persistent CTAs, one per SM, walk the jobs round-robin.  Warp roles: 0 TMA
// producer (Q by a 4-D box of the G heads, K and V tiles by one 4-D box
// per 64-column half), 1 MMA issuer (+ TMEM owner), 2..5 softmax and
// epilogue (only the warps whose TMEM lane quarter holds rows < G work).
// S and O are double-buffered in TMEM so the MMAs of one tile (or job) run
// under the softmax of the previous one.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

namespace {

constexpr int kLKeys = 128;                    // keys per tile
constexpr int kLStages = 2;                    // K/V tile ring
constexpr uint32_t kLQHalf = 64 * 128;         // 64 rows x 128 B: one d half of Q (G <= 64)
constexpr uint32_t kLQBytes = 2 * kLQHalf;
constexpr uint32_t kLPChunk = 64 * 128;        // 64 rows x 64 keys bf16
constexpr uint32_t kLPBytes = 2 * kLPChunk;
constexpr uint32_t kLKVHalf = kLKeys * 128;    // 128 keys x 64 dims bf16
constexpr uint32_t kLKVBytes = 2 * kLKVHalf;
constexpr int kLThreads = 6 * 32;

struct LSmem {
  static constexpr uint32_t q = 0;                              // [2 jobs][2 halves]
  static constexpr uint32_t p = q + 2 * kLQBytes;               // [2 bufs][2 chunks]
  static constexpr uint32_t k = p + 2 * kLPBytes;               // [stage]
  static constexpr uint32_t v = k + kLStages * kLKVBytes;       // [stage]
  static constexpr uint32_t bars = v + kLStages * kLKVBytes;
  static constexpr uint32_t total = bars + 32 * 8 + 16;
};

// byte offset of P[row][key] in a P buffer (K-major, 128-byte swizzle)
__device__ __forceinline__ uint32_t lp_off(int row, int key) {
  return static_cast<uint32_t>((key >> 6) * kLPChunk + row * 128 + ((((key & 63) >> 3) ^ (row & 7)) << 4) +
                               ((key & 7) << 1));
}

struct LJob {
  int64_t hd, i;
  int b, nv, ntiles;
};

__device__ __forceinline__ LJob local_job(const LocalParams& p, int64_t j) {
  LJob J;
  J.hd = j / p.nq;
  J.i = j % p.nq;
  J.nv = visible_local(p.q_seq, p.q_pos, p.local_len, J.i, p.B, p.T, &J.b, p.err);
  J.ntiles = (J.nv + kLKeys - 1) / kLKeys;
  return J;
}

}  // namespace

__global__ void __launch_bounds__(kLThreads, 1)
local_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const LocalParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LSmem::bars);
  // barrier slots
  const uint32_t b_qfull = smem_u32(bars + 0);     // [2]
  const uint32_t b_qempty = smem_u32(bars + 2);    // [2]
  const uint32_t b_kfull = smem_u32(bars + 4);     // [kLStages]
  const uint32_t b_vfull = smem_u32(bars + 6);     // [kLStages]
  const uint32_t b_kvempty = smem_u32(bars + 8);   // [kLStages]
  const uint32_t b_sfull = smem_u32(bars + 10);    // [2]
  const uint32_t b_sfree = smem_u32(bars + 12);    // [2]
  const uint32_t b_pfull = smem_u32(bars + 14);    // [2]
  const uint32_t b_pvdone = smem_u32(bars + 16);   // [2]
  const uint32_t b_ofull = smem_u32(bars + 18);    // [2]
  const uint32_t b_ofree = smem_u32(bars + 20);    // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 24);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;
  const int nact = (G + 31) / 32;                  // softmax warps with real rows
  const uint32_t n_soft = static_cast<uint32_t>(nact) * 32;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(b_qfull + 8 * x, 1);
      mbar_init(b_qempty + 8 * x, 1);
      mbar_init(b_sfull + 8 * x, 1);
      mbar_init(b_sfree + 8 * x, n_soft);
      mbar_init(b_pfull + 8 * x, n_soft);
      mbar_init(b_pvdone + 8 * x, 1);
      mbar_init(b_ofull + 8 * x, 1);
      mbar_init(b_ofree + 8 * x, n_soft);
    }
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(b_kfull + 8 * s, 1);
      mbar_init(b_vfull + 8 * s, 1);
      mbar_init(b_kvempty + 8 * s, 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  if (p.kbox < kLKeys && warp >= 2) {
    // key rows past a short cache's box are never written by TMA: keep them
    // at zero so that 0-weight keys cannot meet a non-finite stale value
    for (int s = 0; s < kLStages; ++s)
      for (int h = 0; h < 2; ++h) {
        uint4* z = reinterpret_cast<uint4*>(smem + LSmem::v + s * kLKVBytes + h * kLKVHalf + p.kbox * 128);
        const int n16 = (kLKeys - p.kbox) * 8;
        for (int x = threadIdx.x - 64; x < n16; x += kLThreads - 64) z[x] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      const uint64_t pol_kv = policy_evict_first();
      const uint64_t pol_q = policy_evict_first();
      const uint32_t kv_tx = 2u * static_cast<uint32_t>(p.kbox) * 128;
      uint32_t it = 0, jn = 0;
      bool ok = true;
      for (int64_t j = blockIdx.x; j < p.njobs && ok; j += gridDim.x) {
        const LJob J = local_job(p, j);
        if (J.ntiles == 0) continue;
        const uint32_t jb = jn & 1;
        if (jn >= 2 && !(ok = mbar_wait(b_qempty + 8 * jb, ((jn >> 1) - 1) & 1, p.err))) break;
        ++jn;
        mbar_arrive_expect_tx(b_qfull + 8 * jb, 2u * G * 128);
        const uint32_t qd = smem_u32(smem + LSmem::q + jb * kLQBytes);
        tma_load_4d(qd, &tmap_q, 0, static_cast<int>(J.i), 0, static_cast<int>(J.hd), b_qfull + 8 * jb, pol_q);
        tma_load_4d(qd + kLQHalf, &tmap_q, 64, static_cast<int>(J.i), 0, static_cast<int>(J.hd), b_qfull + 8 * jb,
                    pol_q);
        const int seq = static_cast<int>(J.hd * p.B + J.b);
        for (int kt = 0; kt < J.ntiles; ++kt, ++it) {
          const uint32_t s = it % kLStages;
          if (it >= kLStages && !(ok = mbar_wait(b_kvempty + 8 * s, ((it / kLStages) - 1) & 1, p.err))) break;
          // one box per 64-column half, each half at a fixed 16 KB offset
          const uint32_t kd = smem_u32(smem + LSmem::k + s * kLKVBytes);
          const uint32_t vd = smem_u32(smem + LSmem::v + s * kLKVBytes);
          mbar_arrive_expect_tx(b_kfull + 8 * s, kv_tx);
          tma_load_4d(kd, &tmap_k, 0, kt * kLKeys, 0, seq, b_kfull + 8 * s, pol_kv);
          tma_load_4d(kd + kLKVHalf, &tmap_k, 0, kt * kLKeys, 1, seq, b_kfull + 8 * s, pol_kv);
          mbar_arrive_expect_tx(b_vfull + 8 * s, kv_tx);
          tma_load_4d(vd, &tmap_v, 0, kt * kLKeys, 0, seq, b_vfull + 8 * s, pol_kv);
          tma_load_4d(vd + kLKVHalf, &tmap_v, 0, kt * kLKeys, 1, seq, b_vfull + 8 * s, pol_kv);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kLKeys, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, kD, 0, 1);
      bool ok = true;
      uint32_t it = 0, jn = 0, cs = 0, cp = 0;
      // the P V of the previous tile, issued after the next S so that the
      // softmax of one tile overlaps the S product of the next
      struct Pend {
        uint32_t it, ob, jn;
        bool first, last;
      } prev{};
      bool have_prev = false;
      auto issue_pv = [&](const Pend& t) {
        const uint32_t vs = t.it % kLStages;
        const uint32_t pb = cp & 1;
        if (ok) ok = mbar_wait(b_vfull + 8 * vs, (t.it / kLStages) & 1, p.err);
        if (ok) ok = mbar_wait(b_pfull + 8 * pb, (cp >> 1) & 1, p.err);
        if (ok && t.first && t.jn >= 2) ok = mbar_wait(b_ofree + 8 * t.ob, ((t.jn >> 1) - 1) & 1, p.err);
        ++cp;
        if (!ok) return;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + LSmem::p + pb * kLPBytes);
        const uint32_t vb = smem_u32(smem + LSmem::v + vs * kLKVBytes);
#pragma unroll
        for (int kk = 0; kk < kLKeys / 16; ++kk)
          mma_bf16_ss(tmem + 256 + 128 * t.ob, sdesc_sw128(pa + (kk >> 2) * kLPChunk + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(vb + kk * 2048, kLKVHalf, 1024), idesc_o, (t.first && kk == 0) ? 0u : 1u);
        mma_commit(b_pvdone + 8 * pb);
        mma_commit(b_kvempty + 8 * vs);
        if (t.last) mma_commit(b_ofull + 8 * t.ob);
      };
      for (int64_t j = blockIdx.x; j < p.njobs && ok; j += gridDim.x) {
        const LJob J = local_job(p, j);
        if (J.ntiles == 0) continue;
        const uint32_t jb = jn & 1;
        ok = mbar_wait(b_qfull + 8 * jb, (jn >> 1) & 1, p.err);
        for (int kt = 0; kt < J.ntiles && ok; ++kt, ++it) {
          const uint32_t ks = it % kLStages;
          const uint32_t sb = cs & 1;
          if (!(ok = mbar_wait(b_kfull + 8 * ks, (it / kLStages) & 1, p.err))) break;
          if (cs >= 2 && !(ok = mbar_wait(b_sfree + 8 * sb, ((cs >> 1) - 1) & 1, p.err))) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(smem + LSmem::q + jb * kLQBytes);
          const uint32_t kb = smem_u32(smem + LSmem::k + ks * kLKVBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + 128 * sb, sdesc_sw128(qa + (kk >> 2) * kLQHalf + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(kb + (kk >> 2) * kLKVHalf + (kk & 3) * 32, 16, 1024), idesc_s, kk != 0);
          mma_commit(b_sfull + 8 * sb);
          ++cs;
          if (kt + 1 == J.ntiles) mma_commit(b_qempty + 8 * jb);
          if (have_prev) issue_pv(prev);
          prev = Pend{it, jn & 1, jn, kt == 0, kt + 1 == J.ntiles};
          have_prev = true;
        }
        ++jn;
      }
      if (ok && have_prev) issue_pv(prev);
    }
  } else if (((warp & 3) * 32) < G) {
    // --------------------- softmax + epilogue ---------------------
    const int row = (warp & 3) * 32 + lane;               // TMEM lane = query head g of the job
    const bool real = row < G;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int64_t rows = static_cast<int64_t>(G) * p.nq;
    bool ok = true;
    uint32_t cnt = 0, jn = 0;
    for (int64_t j = blockIdx.x; j < p.njobs; j += gridDim.x) {
      const LJob J = local_job(p, j);
      const int64_t orow = J.hd * rows + static_cast<int64_t>(row) * p.nq + J.i;
      float m = -INFINITY, l = 0.f;
      if (J.ntiles == 0) {
        // nothing visible: the local sums are empty
        if (real) {
          if (p.out != nullptr) {
            for (int c = 0; c < kD; c += 4)
              *reinterpret_cast<float4*>(p.out + orow * kD + c) =
                  *reinterpret_cast<const float4*>(p.A_doc + orow * kD + c);
          } else {
            float* st = p.ws_loc + orow * (kD + 2);
            for (int c = 0; c < kD; ++c) st[c] = 0.f;
            st[kD] = -INFINITY;
            st[kD + 1] = 0.f;
          }
        }
        continue;
      }
      const uint32_t ob = jn & 1;
      const uint32_t tO = tmem + 256 + 128 * ob + lane_base;
      for (int kt = 0; kt < J.ntiles; ++kt, ++cnt) {
        const uint32_t b = cnt & 1;
        const int nvalid = J.nv - kt * kLKeys;
        if (ok) ok = mbar_wait(b_sfull + 8 * b, (cnt >> 1) & 1, p.err);
        tc_fence_after();
        float sc[kLKeys];
#pragma unroll
        for (int cb = 0; cb < kLKeys; cb += 32) {
          uint32_t v[32];
          NECTAR_TMEM_LD32(tmem + 128 * b + lane_base + cb, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) sc[cb + e] = __uint_as_float(v[e]) * p.qmul;
        }
        tc_fence_before();
        mbar_arrive(b_sfree + 8 * b);
        float bm = -INFINITY;
#pragma unroll
        for (int e = 0; e < kLKeys; ++e) {
          if (e >= nvalid || !real) sc[e] = -INFINITY;
          bm = fmaxf(bm, sc[e]);
        }
        const bool need = bm > m + kRescaleSlack;
        const float corr = need ? exp2_shift(m, bm) : 1.0f;
        if (need) {
          l *= corr;
          m = bm;
        }
        if (__any_sync(0xffffffffu, need) && kt != 0) {
          // O holds the earlier tiles of this job: wait for their last P V,
          // then rescale it in TMEM (warp-collective)
          const uint32_t pc = cnt - 1;
          if (ok) ok = mbar_wait(b_pvdone + 8 * (pc & 1), (pc >> 1) & 1, p.err);
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < kD; cb += 32) {
            uint32_t v[32];
            NECTAR_TMEM_LD32(tO + cb, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
            NECTAR_TMEM_ST32(tO + cb, v);
          }
          tmem_st_wait();
        }
        // P buffer b was last read by the P V of tile cnt - 2
        if (cnt >= 2 && ok) ok = mbar_wait(b_pvdone + 8 * b, ((cnt >> 1) - 1) & 1, p.err);
        uint8_t* pt = smem + LSmem::p + b * kLPBytes;
        float rs = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < kLKeys / 8; ++c8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            w[e] = pack_bf16x2(exp2_shift(sc[c8 * 8 + 2 * e], m), exp2_shift(sc[c8 * 8 + 2 * e + 1], m));
            rs += bf16lo(w[e]) + bf16hi(w[e]);
          }
          if (real) *reinterpret_cast<uint4*>(pt + lp_off(row, c8 * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l += rs;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_pfull + 8 * b);
      }
      // ------------------ epilogue of this job ------------------
      if (ok) ok = mbar_wait(b_ofull + 8 * ob, (jn >> 1) & 1, p.err);
      tc_fence_after();
      float wd = 0.f, wl = 1.f, den = l;
      if (p.out != nullptr && real) {
        const float ad = p.a[orow] * kLog2e;         // document logit, log2 units
        const float M = fmaxf(ad, m);
        wd = exp2_shift(ad, M);
        wl = exp2_shift(m, M);
        den = wd + wl * l;
      }
      const float inv = 1.0f / den;
#pragma unroll
      for (int cb = 0; cb < kD; cb += 32) {
        uint32_t v[32];
        NECTAR_TMEM_LD32(tO + cb, v);
        tmem_ld_wait();
        if (!ok || !real) continue;
        if (p.out != nullptr) {
          const float* ad = p.A_doc + orow * kD + cb;
          float* od = p.out + orow * kD + cb;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 A4 = *reinterpret_cast<const float4*>(ad + e);
            *reinterpret_cast<float4*>(od + e) =
                make_float4((wd * A4.x + wl * __uint_as_float(v[e])) * inv,
                            (wd * A4.y + wl * __uint_as_float(v[e + 1])) * inv,
                            (wd * A4.z + wl * __uint_as_float(v[e + 2])) * inv,
                            (wd * A4.w + wl * __uint_as_float(v[e + 3])) * inv);
          }
        } else {
          float* st = p.ws_loc + orow * (kD + 2) + cb;
#pragma unroll
          for (int e = 0; e < 32; ++e) st[e] = __uint_as_float(v[e]);
        }
      }
      if (ok && real && p.out == nullptr) {
        p.ws_loc[orow * (kD + 2) + kD] = m;
        p.ws_loc[orow * (kD + 2) + kD + 1] = l;
      }
      tc_fence_before();
      mbar_arrive(b_ofree + 8 * ob);
      ++jn;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t local_tc_smem() { return LSmem::total + 1024; }

cudaError_t launch_local_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const LocalParams& p, int grid, cudaStream_t stream) {
  const size_t smem = local_tc_smem();
  cudaError_t e =
      cudaFuncSetAttribute(local_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  local_tc_kernel<<<grid, kLThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace nectar
