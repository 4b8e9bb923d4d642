// Exact causal attention over local tokens, streamed through shared memory:
// the local half of Eq. (3.4) of "Nectar: Neural Estimation of Cached-Token
// Attention via Regression" (§2.2), Z_local and N_local for each query row.
//
// A job is (query token i, block of up to RG of its G query heads); all rows
// of a job see the same local keys (the token's visible set), so the keys
// are read once per job.  One producer thread streams each job's visible
// local K and V rows, kLocTile keys at a time, into a ring of shared-memory
// stages with TMA bulk copies (whole contiguous rows); CW consumer warps
// split every tile's keys, score them on the CUDA cores (common.cuh) and, at
// the end of the job, join their partial states through shared memory.
// Producer and consumers walk the same job list, so they agree on every
// tile without any other signal than the stage barriers.
#pragma once
#include "common.cuh"

namespace nectar {

constexpr int kLocTile = 32;                        // keys per stage
constexpr int kLocStageBytes = 2 * kLocTile * kRowBytes;   // K then V: 16 KB

struct LocalJobs {
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* local_len;
  const __nv_bfloat16* Kloc;
  const __nv_bfloat16* Vloc;
  int B, T, G;
  int* err;
};

// Local rows of the job's sequence for head hd, and its visible count.
__device__ __forceinline__ int job_rows(const LocalJobs& J, int64_t hd, int64_t i, const uint8_t** kb,
                                        const uint8_t** vb) {
  int b;
  const int nv = visible_local(J.q_seq, J.q_pos, J.local_len, i, J.B, J.T, &b, J.err);
  if (nv > 0) {
    *kb = reinterpret_cast<const uint8_t*>(J.Kloc + ((hd * J.B + b) * J.T) * kD);
    *vb = reinterpret_cast<const uint8_t*>(J.Vloc + ((hd * J.B + b) * J.T) * kD);
  }
  return nv;
}

// Producer (one thread): jobs (token t0 + t for t < ntok, g-block gb) in
// order; stage ring of `LS` stages at smem address `ring`, barriers
// full[LS], empty[LS] (8 bytes apart).  Returns false on a wait timeout.
template <int RG>
__device__ __forceinline__ bool local_produce(const LocalJobs& J, int64_t hd, int64_t t0, int ntok, uint32_t ring,
                                              int LS, uint32_t full0, uint32_t empty0) {
  const uint64_t pol = policy_evict_first();
  const int gblocks = (J.G + RG - 1) / RG;
  uint32_t it = 0;
  for (int t = 0; t < ntok; ++t) {
    const uint8_t *kb = nullptr, *vb = nullptr;
    const int nv = job_rows(J, hd, t0 + t, &kb, &vb);
    for (int gb = 0; gb < gblocks; ++gb) {
      for (int j0 = 0; j0 < nv; j0 += kLocTile, ++it) {
        const uint32_t s = it % LS;
        if (it >= static_cast<uint32_t>(LS) && !mbar_wait(empty0 + 8 * s, ((it / LS) - 1) & 1, J.err)) return false;
        const int cnt = (nv - j0 < kLocTile) ? (nv - j0) : kLocTile;
        const uint32_t bytes = static_cast<uint32_t>(cnt) * kRowBytes;
        const uint32_t dst = ring + s * kLocStageBytes;
        mbar_arrive_expect_tx(full0 + 8 * s, 2 * bytes);
        bulk_g2s(dst, kb + static_cast<int64_t>(j0) * kRowBytes, bytes, full0 + 8 * s, pol);
        bulk_g2s(dst + kLocTile * kRowBytes, vb + static_cast<int64_t>(j0) * kRowBytes, bytes, full0 + 8 * s, pol);
      }
    }
  }
  return true;
}

// Consumers (CW warps, warp index cw, named barrier `bar_id` over them).
// For every job calls done(t, g0, nr, M, l, acc_dim) per (row, dim) item
// with the job's joined state: M and l in log2 units, acc relative to 2^M.
// scratch: CW * RG * (kD + 2) floats of shared memory.
template <int RG, int CW, class Done>
__device__ __forceinline__ void local_consume(const LocalJobs& J, int64_t hd, int64_t t0, int ntok,
                                              const __nv_bfloat16* Qrows0, int64_t qstride_g, float qmul,
                                              const uint8_t* ring, int LS, uint32_t full0, uint32_t empty0,
                                              float* scratch, int bar_id, int cw, int lane, Done&& done) {
  constexpr int LPK = 16;
  using St = RowState<RG, LPK>;
  constexpr int NG = St::NG;
  constexpr int KPW = kLocTile / CW;           // keys per warp per tile
  constexpr int KPG = KPW / NG;                // keys per group per tile
  static_assert(KPG >= 1 && KPW * CW == kLocTile, "tile split");
  const int g = lane / LPK, tl = lane % LPK;
  const int gblocks = (J.G + RG - 1) / RG;
  bool ok = true;
  uint32_t it = 0;
  for (int t = 0; t < ntok; ++t) {
    const uint8_t *kb = nullptr, *vb = nullptr;
    const int nv = job_rows(J, hd, t0 + t, &kb, &vb);
    for (int gb = 0; gb < gblocks; ++gb) {
      const int g0 = gb * RG;
      const int nr = (J.G - g0 < RG) ? (J.G - g0) : RG;
      St st;
      st.reset();
      // rows (g0 + r) of token t0 + t: Qrows0 + (g0 + r) * qstride_g + t * kD
      st.load_q(Qrows0 + static_cast<int64_t>(g0) * qstride_g + static_cast<int64_t>(t) * kD, qstride_g, nr, tl,
                qmul);
      for (int j0 = 0; j0 < nv; j0 += kLocTile, ++it) {
        const uint32_t s = it % LS;
        if (ok) ok = mbar_wait(full0 + 8 * s, (it / LS) & 1, J.err);
        if (ok) {
          const int cnt = (nv - j0 < kLocTile) ? (nv - j0) : kLocTile;
          const uint8_t* kt = ring + s * kLocStageBytes;
          const uint8_t* vt = kt + kLocTile * kRowBytes;
          const uint8_t* kr[KPG];
          const uint8_t* vr[KPG];
          bool valid[KPG];
#pragma unroll
          for (int k = 0; k < KPG; ++k) {
            const int key = cw * KPW + k * NG + g;
            valid[k] = key < cnt;
            kr[k] = kt + key * kRowBytes;
            vr[k] = vt + key * kRowBytes;
          }
          st.template step<KPG>(kr, vr, valid, tl, SmemLoader{});
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
      }
      // join the CW warps' states
      st.merge_groups();
      if (g == 0) {
        float* dst = scratch + (cw * RG) * (kD + 2);
#pragma unroll
        for (int r = 0; r < RG; ++r) {
#pragma unroll
          for (int ci = 0; ci < St::CPL; ++ci)
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[r * (kD + 2) + St::dim_of(tl, ci, e)] = st.acc[r][ci * 8 + e];
          if (tl == 0) {
            dst[r * (kD + 2) + kD] = st.m[r];
            dst[r * (kD + 2) + kD + 1] = st.l[r];
          }
        }
      }
      named_bar_sync(bar_id, CW * 32);
      for (int item = cw * 32 + lane; item < nr * kD; item += CW * 32) {
        const int r = item / kD, dim = item % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < CW; ++w) M = fmaxf(M, scratch[(w * RG + r) * (kD + 2) + kD]);
        float ls = 0.f, as = 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) {
          const float* src = scratch + (w * RG + r) * (kD + 2);
          const float wgt = exp2_shift(src[kD], M);
          ls = fmaf(src[kD + 1], wgt, ls);
          as = fmaf(src[dim], wgt, as);
        }
        done(t, g0 + r, dim, M, ls, as);
      }
      named_bar_sync(bar_id, CW * 32);
    }
  }
}

}  // namespace nectar
