// Exact causal local attention on the tensor cores for few query heads per
// KV head (G <= 16): the local half of Eq. (3.4) of "Nectar: Neural
// Estimation of Cached-Token Attention via Regression" (§2.2) -- Z_local,
// N_local and their maximum for every query row -- optionally merged at once
// with a document term (a, A_doc) as in Eqs. (3.4)-(3.5).
//
// A job is (KV head, query token i): the token's G query heads see the same
// visible prefix of its local cache (at most 512 keys here).  The products
// are taken transposed, so that the keys, not the few query heads, fill the
// 128 rows of the tensor-core tile and the TMEM lanes:
//   S^T = K Q^T   (M = 128 keys, N = 16 query heads of which G are real,
//                  K = d; K and Q K-major, 128-byte swizzle),
//   O^T = V^T P^T (M = d, N = 16, K = keys; V read MN-major, P K-major).
// Each of the 128 softmax threads owns one key of a tile (one TMEM lane of
// S^T) and holds its G scores.  All of the job's S^T tiles are in TMEM
// before the softmax starts, so the per-head maximum is exact (two passes:
// max over the keys, then the weights) and nothing is ever rescaled; the
// maximum and the sum over keys are reduced across the 128 threads by warp
// shuffles and shared memory.  In O^T the TMEM lanes are the d dims, so the
// epilogue's stores of a head's 128 values are coalesced.
//
// Persistent CTAs, two per SM.  Warp roles: 0 TMA producer (Q by a 4-D box
// of the G heads, K and V tiles by one 4-D box per 64-column half), 1 MMA
// issuer (+ TMEM owner), 2..5 softmax and epilogue.  K and V tiles share a
// 2-stage ring; S^T, O^T, Q and P are double-buffered per job, and the
// epilogue of a job runs after the softmax of the next one, under its MMAs.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

namespace {

constexpr int kXKeys = 128;                        // keys per tile (TMEM lanes of S^T)
constexpr int kXMaxTiles = 4;                      // visible keys per job <= 512
constexpr int kXN = 16;                            // query columns of S^T and O^T (G <= 16)
constexpr int kXStages = 2;                        // K / V tile ring
constexpr uint32_t kXTileHalf = kXKeys * 128;      // 128 keys x 64 dims bf16: 16 KB
constexpr uint32_t kXTile = 2 * kXTileHalf;
constexpr uint32_t kXQHalf = kXN * 128;            // 16 heads x 64 dims: 2 KB
constexpr uint32_t kXQ = 2 * kXQHalf;
constexpr uint32_t kXPChunk = kXN * 128;           // 16 heads x 64 keys: 2 KB
constexpr uint32_t kXPTile = 2 * kXPChunk;         // one 128-key tile of P
constexpr uint32_t kXP = kXMaxTiles * kXPTile;     // P of one job: 16 KB
constexpr int kXThreads = 6 * 32;
constexpr uint32_t kXTmemCols = 256;               // S^T [2][4 tiles x 16] + O^T [2][16]
constexpr uint32_t kXOCol = 2 * kXMaxTiles * kXN;  // first O^T column

struct XSmem {
  static constexpr uint32_t ring = 0;                          // [kXStages] K or V tiles
  static constexpr uint32_t q = ring + kXStages * kXTile;      // [2 jobs]
  static constexpr uint32_t p = q + 2 * kXQ;                   // [2 jobs]
  static constexpr uint32_t red = p + 2 * kXP;                 // float [2: max, sum][4 warps][16]
  static constexpr uint32_t ml = red + 2 * 4 * kXN * 4;        // float [2 jobs][2: m, l][16]
  static constexpr uint32_t bars = ml + 2 * 2 * kXN * 4;
  static constexpr uint32_t total = bars + 32 * 8 + 16;
};
static_assert(XSmem::q % 1024 == 0 && XSmem::p % 1024 == 0, "operand tiles need 1024-byte alignment");

// byte offset of P[head][key] in one job's P buffer (per 128-key tile two
// K-major 64-key chunks of 16 rows, 128-byte swizzle)
__device__ __forceinline__ uint32_t xp_off(int head, int key) {
  return static_cast<uint32_t>((key >> 7) * kXPTile + ((key >> 6) & 1) * kXPChunk + head * 128 +
                               ((((key & 63) >> 3) ^ (head & 7)) << 4) + ((key & 7) << 1));
}

struct XJob {
  int64_t hd, i;
  int b, nv, ntiles;
};

__device__ __forceinline__ XJob xjob(const LocalParams& p, int64_t j) {
  XJob J;
  J.hd = j / p.nq;
  J.i = j % p.nq;
  J.nv = visible_local(p.q_seq, p.q_pos, p.local_len, J.i, p.B, p.T, &J.b, p.err);
  if (J.nv > kXMaxTiles * kXKeys) {               // the host routes only T <= 512 here
    record_error(p.err, DEVERR_BAD_LEN);
    J.nv = kXMaxTiles * kXKeys;
  }
  J.ntiles = (J.nv + kXKeys - 1) / kXKeys;
  return J;
}

// 8 or 16 columns of 32 lanes of TMEM -> registers (warp-collective)
template <int QC>
__device__ __forceinline__ void xtmem_ld(uint32_t taddr, uint32_t (&r)[QC]) {
  if constexpr (QC == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
  } else {
    NECTAR_TMEM_LD16(taddr, r);
  }
}

// Reduce NV per-lane values over the 32 lanes of a warp (max or sum):
// log2(NV) halving steps (a lane keeps one half of its values and sends the
// other half to its partner), then plain butterfly steps.  Lane L ends with
// value L / (32 / NV) reduced over all lanes.
template <int NV, bool kMax>
__device__ __forceinline__ float xwarp_reduce(float (&v)[NV], int lane) {
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const int half = n / 2;
      const bool up = lane & off;
#pragma unroll
      for (int j = 0; j < half; ++j) {
        // both values read before the selects: a select between two array
        // elements would become a dynamically indexed (local-memory) array
        const float lo = v[j], hi = v[j + half];
        float send, keep;
        asm("{\n\t.reg .pred p;\n\tsetp.ne.s32 p, %4, 0;\n\t"
            "selp.f32 %0, %2, %3, p;\n\tselp.f32 %1, %3, %2, p;\n\t}"
            : "=f"(send), "=f"(keep)
            : "f"(lo), "f"(hi), "r"(static_cast<int>(up)));
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

}  // namespace

template <int QC>
__global__ void __launch_bounds__(kXThreads, 2)
local_tct_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const LocalParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + XSmem::bars);
  const uint32_t b_qfull = smem_u32(bars + 0);     // [2]
  const uint32_t b_qempty = smem_u32(bars + 2);    // [2]
  const uint32_t b_full = smem_u32(bars + 4);      // [kXStages]
  const uint32_t b_empty = smem_u32(bars + 6);     // [kXStages]
  const uint32_t b_sfull = smem_u32(bars + 8);     // [2]
  const uint32_t b_sfree = smem_u32(bars + 10);    // [2]
  const uint32_t b_pfull = smem_u32(bars + 12);    // [2]
  const uint32_t b_ofull = smem_u32(bars + 14);    // [2]
  const uint32_t b_ofree = smem_u32(bars + 16);    // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 24);
  float* red = reinterpret_cast<float*>(smem + XSmem::red);   // [2][4][16]
  float* ml = reinterpret_cast<float*>(smem + XSmem::ml);     // [2][2][16]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(b_qfull + 8 * x, 1);
      mbar_init(b_qempty + 8 * x, 1);
      mbar_init(b_sfull + 8 * x, 1);
      mbar_init(b_sfree + 8 * x, 128);
      mbar_init(b_pfull + 8 * x, 128);
      mbar_init(b_ofull + 8 * x, 1);
      mbar_init(b_ofree + 8 * x, 128);
    }
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), kXTmemCols);
    tmem_relinquish();
  }
  if (p.kbox < kXKeys && warp >= 2) {
    // key rows past a short cache's box are never written by TMA: keep them
    // at zero so that 0-weight keys cannot meet a non-finite stale value
    for (int s = 0; s < kXStages; ++s)
      for (int h = 0; h < 2; ++h) {
        uint4* z = reinterpret_cast<uint4*>(smem + XSmem::ring + s * kXTile + h * kXTileHalf + p.kbox * 128);
        const int n16 = (kXKeys - p.kbox) * 8;
        for (int x = threadIdx.x - 64; x < n16; x += kXThreads - 64) z[x] = make_uint4(0, 0, 0, 0);
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
      const uint64_t pol = policy_evict_first();
      const uint32_t kv_tx = 2u * static_cast<uint32_t>(p.kbox) * 128;
      uint32_t it = 0, jn = 0;
      bool ok = true;
      auto load_tile = [&](const CUtensorMap* map, int kt, int seq) {
        const uint32_t s = it % kXStages;
        if (it >= kXStages) ok = mbar_wait(b_empty + 8 * s, ((it / kXStages) - 1) & 1, p.err);
        if (!ok) return;
        const uint32_t dst = smem_u32(smem + XSmem::ring + s * kXTile);
        mbar_arrive_expect_tx(b_full + 8 * s, kv_tx);
        tma_load_4d(dst, map, 0, kt * kXKeys, 0, seq, b_full + 8 * s, pol);
        tma_load_4d(dst + kXTileHalf, map, 0, kt * kXKeys, 1, seq, b_full + 8 * s, pol);
        ++it;
      };
      for (int64_t j = blockIdx.x; j < p.njobs && ok; j += gridDim.x) {
        const XJob J = xjob(p, j);
        if (J.ntiles == 0) continue;
        const uint32_t jb = jn & 1;
        if (jn >= 2 && !(ok = mbar_wait(b_qempty + 8 * jb, ((jn >> 1) - 1) & 1, p.err))) break;
        ++jn;
        mbar_arrive_expect_tx(b_qfull + 8 * jb, 2u * G * 128);
        const uint32_t qd = smem_u32(smem + XSmem::q + jb * kXQ);
        tma_load_4d(qd, &tmap_q, 0, static_cast<int>(J.i), 0, static_cast<int>(J.hd), b_qfull + 8 * jb, pol);
        tma_load_4d(qd + kXQHalf, &tmap_q, 64, static_cast<int>(J.i), 0, static_cast<int>(J.hd),
                    b_qfull + 8 * jb, pol);
        const int seq = static_cast<int>(J.hd * p.B + J.b);
        for (int kt = 0; kt < J.ntiles && ok; ++kt) load_tile(&tmap_k, kt, seq);
        for (int kt = 0; kt < J.ntiles && ok; ++kt) load_tile(&tmap_v, kt, seq);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kXN, 0, 0);   // A = K tile, B = Q
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, kXN, 1, 0);   // A = V tile (MN-major), B = P
      bool ok = true;
      uint32_t it = 0, jn = 0;
      for (int64_t j = blockIdx.x; j < p.njobs && ok; j += gridDim.x) {
        const XJob J = xjob(p, j);
        if (J.ntiles == 0) continue;
        const uint32_t jb = jn & 1;
        const uint32_t ph = (jn >> 1) & 1, ph_prev = ((jn >> 1) - 1) & 1;
        if (!(ok = mbar_wait(b_qfull + 8 * jb, ph, p.err))) break;
        if (jn >= 2 && !(ok = mbar_wait(b_sfree + 8 * jb, ph_prev, p.err))) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(smem + XSmem::q + jb * kXQ);
        for (int kt = 0; kt < J.ntiles && ok; ++kt, ++it) {
          const uint32_t s = it % kXStages;
          if (!(ok = mbar_wait(b_full + 8 * s, (it / kXStages) & 1, p.err))) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + XSmem::ring + s * kXTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + jb * (kXMaxTiles * kXN) + kt * kXN,
                        sdesc_sw128(ka + (kk >> 2) * kXTileHalf + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(qa + (kk >> 2) * kXQHalf + (kk & 3) * 32, 16, 1024), idesc_s, kk != 0);
          mma_commit(b_empty + 8 * s);
        }
        if (!ok) break;
        mma_commit(b_sfull + 8 * jb);
        mma_commit(b_qempty + 8 * jb);
        // O^T = V^T P^T once the softmax has written P
        if (!(ok = mbar_wait(b_pfull + 8 * jb, ph, p.err))) break;
        if (jn >= 2 && !(ok = mbar_wait(b_ofree + 8 * jb, ph_prev, p.err))) break;
        tc_fence_after();
        const uint32_t pb = smem_u32(smem + XSmem::p + jb * kXP);
        for (int kt = 0; kt < J.ntiles && ok; ++kt, ++it) {
          const uint32_t s = it % kXStages;
          if (!(ok = mbar_wait(b_full + 8 * s, (it / kXStages) & 1, p.err))) break;
          tc_fence_after();
          const uint32_t va = smem_u32(smem + XSmem::ring + s * kXTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + kXOCol + jb * kXN, sdesc_sw128(va + kk * 2048, kXTileHalf, 1024),
                        sdesc_sw128(pb + kt * kXPTile + (kk >> 2) * kXPChunk + (kk & 3) * 32, 16, 1024), idesc_o,
                        (kt != 0 || kk != 0) ? 1u : 0u);
          mma_commit(b_empty + 8 * s);
        }
        if (!ok) break;
        mma_commit(b_ofull + 8 * jb);
        ++jn;
      }
    }
  } else {
    // --------------------- softmax + epilogue (128 threads) ---------------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                // key of a tile (S^T) / dim (O^T)
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t rows = static_cast<int64_t>(G) * p.nq;
    constexpr int kLanesPer = 32 / QC;                // lanes holding one reduced value
    bool ok = true;
    uint32_t jn = 0;
    bool have_prev = false;
    int64_t prev_hd = 0, prev_i = 0;

    // the epilogue of the job held in buffer eb: O^T from TMEM, (m, l) from
    // shared memory; thread r writes dim r of each of the G rows
    auto epilogue = [&](uint32_t ejn, int64_t hd, int64_t i) {
      const uint32_t eb = ejn & 1;
      if (ok) ok = mbar_wait(b_ofull + 8 * eb, (ejn >> 1) & 1, p.err);
      tc_fence_after();
      uint32_t o[QC];
      xtmem_ld<QC>(tmem + kXOCol + eb * kXN + lane_base, o);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(b_ofree + 8 * eb);
      if (!ok) return;
      const float* mlj = ml + eb * 2 * kXN;
#pragma unroll
      for (int q = 0; q < QC; ++q) {
        if (q >= G) break;
        const int64_t orow = hd * rows + static_cast<int64_t>(q) * p.nq + i;
        const float m = mlj[q], l = mlj[kXN + q], ov = __uint_as_float(o[q]);
        if (p.out != nullptr) {
          const float ad = p.a[orow] * kLog2e;        // document logit, log2 units
          const float M = fmaxf(ad, m);
          const float wd = exp2_shift(ad, M), wl = exp2_shift(m, M);
          p.out[orow * kD + r] = (wd * p.A_doc[orow * kD + r] + wl * ov) / (wd + wl * l);
        } else {
          float* st = p.ws_loc + orow * (kD + 2);
          st[r] = ov;
          if (r == 0) {
            st[kD] = m;
            st[kD + 1] = l;
          }
        }
      }
    };

    // one pass more than there are jobs: the last one only runs the final
    // epilogue (a single call site keeps the epilogue inlined)
    for (int64_t j = blockIdx.x;; j += gridDim.x) {
      if (j >= p.njobs) {
        if (have_prev) {
          named_bar_sync(3, 128);                     // (m, l) of the last job written
          epilogue(jn - 1, prev_hd, prev_i);
        }
        break;
      }
      const XJob J = xjob(p, j);
      if (J.ntiles == 0) {
        // nothing visible: the local sums are empty
        for (int q = 0; q < G; ++q) {
          const int64_t orow = J.hd * rows + static_cast<int64_t>(q) * p.nq + J.i;
          if (p.out != nullptr) {
            p.out[orow * kD + r] = p.A_doc[orow * kD + r];
          } else {
            float* st = p.ws_loc + orow * (kD + 2);
            st[r] = 0.f;
            if (r == 0) {
              st[kD] = -INFINITY;
              st[kD + 1] = 0.f;
            }
          }
        }
        continue;
      }
      const uint32_t jb = jn & 1;
      if (ok) ok = mbar_wait(b_sfull + 8 * jb, (jn >> 1) & 1, p.err);
      tc_fence_after();
      // ---- pass 1: this thread's scores and their maximum per head ----
      float s[kXMaxTiles][QC];
#pragma unroll
      for (int t = 0; t < kXMaxTiles; ++t) {
        if (t < J.ntiles) {
          uint32_t v[QC];
          xtmem_ld<QC>(tmem + jb * (kXMaxTiles * kXN) + t * kXN + lane_base, v);
          tmem_ld_wait();
          const bool valid = t * kXKeys + r < J.nv;
#pragma unroll
          for (int q = 0; q < QC; ++q) s[t][q] = valid ? __uint_as_float(v[q]) * p.qmul : -INFINITY;
        } else {
#pragma unroll
          for (int q = 0; q < QC; ++q) s[t][q] = -INFINITY;
        }
      }
      tc_fence_before();
      mbar_arrive(b_sfree + 8 * jb);
      float mx[QC];
#pragma unroll
      for (int q = 0; q < QC; ++q) {
        float m = s[0][q];
#pragma unroll
        for (int t = 1; t < kXMaxTiles; ++t) m = fmaxf(m, s[t][q]);
        mx[q] = m;
      }
      {
        const float w = xwarp_reduce<QC, true>(mx, lane);
        if (lane % kLanesPer == 0) red[quarter * kXN + lane / kLanesPer] = w;
      }
      named_bar_sync(1, 128);
      float M[QC];
#pragma unroll
      for (int q = 0; q < QC; ++q)
        M[q] = fmaxf(fmaxf(red[q], red[kXN + q]), fmaxf(red[2 * kXN + q], red[3 * kXN + q]));
      // ---- pass 2: the weights, bf16 into P (row = head, column = key) ----
      uint8_t* pj = smem + XSmem::p + jb * kXP;
      float ls[QC];
#pragma unroll
      for (int q = 0; q < QC; ++q) ls[q] = 0.f;
#pragma unroll
      for (int t = 0; t < kXMaxTiles; ++t) {
        if (t < J.ntiles) {
#pragma unroll
          for (int q = 0; q < QC; ++q) {
            const __nv_bfloat16 w = __float2bfloat16_rn(exp2_shift(s[t][q], M[q]));
            ls[q] += __bfloat162float(w);
            if (q < G) *reinterpret_cast<__nv_bfloat16*>(pj + xp_off(q, t * kXKeys + r)) = w;
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(b_pfull + 8 * jb);
      {
        const float w = xwarp_reduce<QC, false>(ls, lane);
        if (lane % kLanesPer == 0) red[4 * kXN + quarter * kXN + lane / kLanesPer] = w;
      }
      named_bar_sync(2, 128);
      if (r < QC) {
        float* mlj = ml + jb * 2 * kXN;
        mlj[r] = M[r];
        mlj[kXN + r] = red[4 * kXN + r] + red[5 * kXN + r] + red[6 * kXN + r] + red[7 * kXN + r];
      }
      // ---- the previous job's epilogue, under this job's MMAs ----
      if (have_prev) epilogue(jn - 1, prev_hd, prev_i);
      have_prev = true;
      prev_hd = J.hd;
      prev_i = J.i;
      ++jn;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kXTmemCols);
  }
}

size_t local_tct_smem() { return XSmem::total + 1024; }

cudaError_t launch_local_tct(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const LocalParams& p, int sms, cudaStream_t stream) {
  const size_t smem = local_tct_smem();
  const int64_t cap = static_cast<int64_t>(sms) * 2;
  const int grid = static_cast<int>(p.njobs < cap ? p.njobs : cap);
  if (grid <= 0) return cudaSuccess;
  cudaError_t e;
  if (p.G <= 8) {
    e = cudaFuncSetAttribute(local_tct_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    local_tct_kernel<8><<<grid, kXThreads, smem, stream>>>(tq, tk, tv, p);
  } else {
    e = cudaFuncSetAttribute(local_tct_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    local_tct_kernel<16><<<grid, kXThreads, smem, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

}  // namespace nectar
