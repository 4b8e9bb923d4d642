// Exact causal local attention for many query tokens, one warp per job: the
// local half of Eq. (3.4) of "Nectar: Neural Estimation of Cached-Token
// Attention via Regression" (§2.2), left as a per-row state (acc, m, l) or
// merged at once with a document term (a, A_doc), Eqs. (3.4)-(3.5).
//
// A job is (KV head, query token, block of up to 4 of its query heads).  In
// a decode batch every token has its own short local cache, so jobs share
// nothing and are many: persistent warps take them round-robin and stream
// the token's visible K and V rows straight from global memory into
// registers (16 lanes per 256-byte row, two keys per warp step; the K and V
// rows of the next step are loaded while this step is computed), score them on the CUDA cores
// (common.cuh) and keep the online softmax in registers.  No shared memory
// and no barriers: latency is hidden by the number of warps in flight.
// Blocks of more than 4 heads would cost registers, hence occupancy; the
// blocks of one token run on neighbouring warps, so its rows are read from
// HBM once and from L2 by the others.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

namespace {

constexpr int kLWWarps = 4;
#ifndef NECTAR_LW_PAIRED
#define NECTAR_LW_PAIRED 1
#endif
constexpr bool kLWPaired = NECTAR_LW_PAIRED != 0;   // paired f32x2 FMAs (RowState)
constexpr int kLWThreads = kLWWarps * 32;

template <int RG>
__host__ __device__ constexpr int lw_keys_per_group() { return RG <= 2 ? 4 : 2; }
template <int RG>
__host__ __device__ constexpr int lw_min_blocks() { return RG <= 1 ? 4 : 3; }

}  // namespace

template <int RG>
__global__ void __launch_bounds__(kLWThreads, lw_min_blocks<RG>()) local_warp_kernel(const LocalParams p) {
  constexpr int LPK = 16;
  constexpr int KPG = lw_keys_per_group<RG>();
  using St = RowState<RG, LPK>;
  constexpr int NG = St::NG;
  const int lane = threadIdx.x & 31;
  const int grp = lane / LPK, tl = lane % LPK;
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * kLWWarps + (threadIdx.x >> 5);
  const int64_t nw = static_cast<int64_t>(gridDim.x) * kLWWarps;
  const int G = p.G;
  const int gblocks = (G + RG - 1) / RG;
  const int64_t rows = static_cast<int64_t>(G) * p.nq;
  const int64_t njobs = p.njobs * gblocks;
  for (int64_t job = w0; job < njobs; job += nw) {
    const int gb = static_cast<int>(job % gblocks);
    const int64_t ti = job / gblocks;
    const int64_t hd = ti / p.nq, i = ti % p.nq;
    int b = 0;
    const int nv = visible_local(p.q_seq, p.q_pos, p.local_len, i, p.B, p.T, &b, p.err);
    const int g0 = gb * RG;
    const int nr = (G - g0 < RG) ? (G - g0) : RG;
    St st;
    st.reset();
    st.load_q(p.Q + ((hd * G + g0) * p.nq + i) * kD, p.nq * kD, nr, tl, p.qmul);
    if (nv > 0) {
      const uint8_t* kb = reinterpret_cast<const uint8_t*>(p.Kloc + (hd * p.B + b) * p.T * kD);
      const uint8_t* vb = reinterpret_cast<const uint8_t*>(p.Vloc + (hd * p.B + b) * p.T * kD);
      // two register buffers: the K and V rows of the next step are in
      // flight while this step is scored and accumulated
      constexpr int kStep = NG * KPG;
      uint4 kw[2][KPG][St::CPL], vw[2][KPG][St::CPL];
      bool valid[2][KPG];
      auto issue = [&](int buf, int j0) {
        const uint8_t* kr[KPG];
        const uint8_t* vr[KPG];
#pragma unroll
        for (int k = 0; k < KPG; ++k) {
          const int key = j0 + k * NG + grp;
          valid[buf][k] = key < nv;
          kr[k] = kb + static_cast<int64_t>(key) * kRowBytes;
          vr[k] = vb + static_cast<int64_t>(key) * kRowBytes;
        }
        St::template load_rows<KPG>(kr, valid[buf], tl, GlobalLoader{}, kw[buf]);
        St::template load_rows<KPG>(vr, valid[buf], tl, GlobalLoader{}, vw[buf]);
      };
      issue(0, 0);
      for (int j0 = 0; j0 < nv; j0 += 2 * kStep) {
        if (j0 + kStep < nv) issue(1, j0 + kStep);
        float pw[KPG][RG];
        st.template weigh<KPG, kLWPaired>(kw[0], valid[0], pw);
        st.template accumulate<KPG, kLWPaired>(vw[0], pw);
        if (j0 + kStep >= nv) break;
        if (j0 + 2 * kStep < nv) issue(0, j0 + 2 * kStep);
        st.template weigh<KPG, kLWPaired>(kw[1], valid[1], pw);
        st.template accumulate<KPG, kLWPaired>(vw[1], pw);
      }
    }
    st.merge_groups();
    if (grp != 0) continue;
    // lanes of group 0 hold dims 8 tl .. 8 tl + 7 of every row
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      if (r >= nr) break;
      const int64_t row = hd * rows + static_cast<int64_t>(g0 + r) * p.nq + i;
      const int dim = St::dim_of(tl, 0, 0);
      if (p.out == nullptr) {
        // state rows are d + 2 = 130 floats (520 B) apart: 8-byte aligned
        // for every row, 16-byte aligned only for even ones
        float* s = p.ws_loc + row * (kD + 2);
#pragma unroll
        for (int e = 0; e < 8; e += 2)
          *reinterpret_cast<float2*>(s + dim + e) = make_float2(st.acc[r][e], st.acc[r][e + 1]);
        if (tl == 0) {
          s[kD] = st.m[r];
          s[kD + 1] = st.l[r];
        }
      } else {
        const float ad = p.a[row] * kLog2e;        // document logit, log2 units
        const float M = fmaxf(ad, st.m[r]);
        const float wd = exp2_shift(ad, M), wl = exp2_shift(st.m[r], M);
        const float inv = 1.0f / (wd + wl * st.l[r]);
        const float4 A0 = *reinterpret_cast<const float4*>(p.A_doc + row * kD + dim);
        const float4 A1 = *reinterpret_cast<const float4*>(p.A_doc + row * kD + dim + 4);
        float* o = p.out + row * kD + dim;
        *reinterpret_cast<float4*>(o) =
            make_float4((wd * A0.x + wl * st.acc[r][0]) * inv, (wd * A0.y + wl * st.acc[r][1]) * inv,
                        (wd * A0.z + wl * st.acc[r][2]) * inv, (wd * A0.w + wl * st.acc[r][3]) * inv);
        *reinterpret_cast<float4*>(o + 4) =
            make_float4((wd * A1.x + wl * st.acc[r][4]) * inv, (wd * A1.y + wl * st.acc[r][5]) * inv,
                        (wd * A1.z + wl * st.acc[r][6]) * inv, (wd * A1.w + wl * st.acc[r][7]) * inv);
      }
    }
  }
}

template <int RG>
static cudaError_t launch_lw(const LocalParams& p, int sms, cudaStream_t stream) {
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, local_warp_kernel<RG>, kLWThreads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int gblocks = (p.G + RG - 1) / RG;
  const int64_t warps = p.njobs * gblocks;
  int64_t grid = static_cast<int64_t>(sms) * per_sm;
  const int64_t need = (warps + kLWWarps - 1) / kLWWarps;
  if (grid > need) grid = need;
  local_warp_kernel<RG><<<static_cast<unsigned>(grid), kLWThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_local_warp(const LocalParams& p, int sms, cudaStream_t stream) {
  switch (p.G < 4 ? p.G : 4) {
    case 1: return launch_lw<1>(p, sms, stream);
    case 2: return launch_lw<2>(p, sms, stream);
    case 3: return launch_lw<3>(p, sms, stream);
    default: return launch_lw<4>(p, sms, stream);
  }
}

}  // namespace nectar
