// (iii) Merge of a document term (a, A_doc) with exact causal attention over
// the local tokens: Eqs. (3.4)-(3.5) of "Nectar: Neural Estimation of
// Cached-Token Attention via Regression" (§2.2).  The document term is one
// extra logit a with value A_doc, softmaxed jointly with the visible local
// keys; with the exact (alpha, A) this is full attention (Eq. (3.4) is an
// identity), with (a_theta, A_theta) it is the Nectar output (Eq. (3.5)).
//
// One CTA (4 warps) per (KV head, query token, block of <= 8 query heads):
// the G query heads of a token share the token's local K/V and its causal
// mask, so the local rows are read once for all of them, straight from
// global memory with 16-byte non-coherent loads.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

constexpr int kMergeWarps = 4;

template <int R, int LPK>
__global__ void __launch_bounds__(kMergeWarps * 32)
merge_local_kernel(const MergeParams p) {
  using St = RowState<R, LPK>;
  constexpr int NG = St::NG;
  constexpr int KPG = 2;
  constexpr int kStride = kMergeWarps * NG;   // key slots per CTA step

  __shared__ float sRed[kMergeWarps][R][kD + 2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane / LPK, t = lane % LPK;
  // unit = (head, token, g-block)
  const int64_t unit = blockIdx.x;
  const int gblocks = (p.G + R - 1) / R;
  const int64_t hd = unit / (p.nq * gblocks);
  const int64_t rem = unit % (p.nq * gblocks);
  const int64_t i = rem / gblocks;
  const int g0 = static_cast<int>(rem % gblocks) * R;
  const int nrows = (p.G - g0 < R) ? (p.G - g0) : R;
  const int64_t rows = static_cast<int64_t>(p.G) * p.nq;

  int b;
  const int nv = visible_local(p.q_seq, p.q_pos, p.local_len, i, p.B, p.T, &b, p.err);

  St st;
  st.reset();
  // query rows g0..g0+nrows-1 of token i: row (g0+gg)*nq + i, stride nq rows
  st.load_q(p.Q + (hd * rows + static_cast<int64_t>(g0) * p.nq + i) * kD, p.nq * kD, nrows, t, p.qmul);

  if (nv > 0) {
    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(p.Kloc + ((hd * p.B + b) * p.T) * kD);
    const uint8_t* vbase = reinterpret_cast<const uint8_t*>(p.Vloc + ((hd * p.B + b) * p.T) * kD);
    for (int j0 = 0; j0 < nv; j0 += kStride * KPG) {
      const uint8_t* kr[KPG];
      const uint8_t* vr[KPG];
      bool valid[KPG];
#pragma unroll
      for (int k = 0; k < KPG; ++k) {
        const int j = j0 + k * kStride + warp * NG + g;
        valid[k] = j < nv;
        kr[k] = kbase + static_cast<int64_t>(j) * kRowBytes;
        vr[k] = vbase + static_cast<int64_t>(j) * kRowBytes;
      }
      st.template step<KPG>(kr, vr, valid, t, GlobalLoader{});
    }
  }
  st.merge_groups();
  if (g == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int ci = 0; ci < St::CPL; ++ci)
#pragma unroll
        for (int e = 0; e < 8; ++e) sRed[warp][r][St::dim_of(t, ci, e)] = st.acc[r][ci * 8 + e];
      if (t == 0) {
        sRed[warp][r][kD] = st.m[r];
        sRed[warp][r][kD + 1] = st.l[r];
      }
    }
  }
  __syncthreads();
  for (int it = threadIdx.x; it < nrows * kD; it += kMergeWarps * 32) {
    const int r = it / kD, dim = it % kD;
    const int64_t row = hd * rows + static_cast<int64_t>(g0 + r) * p.nq + i;
    const float ad = p.a[row] * kLog2e;       // document logit in log2 units
    float M = ad;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) M = fmaxf(M, sRed[w][r][kD]);
    const float wd = exp2_shift(ad, M);
    float den = wd;
    float num = wd * p.A_doc[row * kD + dim];
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
      const float wl = exp2_shift(sRed[w][r][kD], M);
      den = fmaf(sRed[w][r][kD + 1], wl, den);
      num = fmaf(sRed[w][r][dim], wl, num);
    }
    p.out[row * kD + dim] = num / den;
  }
}

template <int R, int LPK>
static cudaError_t launch_merge_t(const MergeParams& p, cudaStream_t stream) {
  const int gblocks = (p.G + R - 1) / R;
  const int64_t units = static_cast<int64_t>(p.heads) * p.nq * gblocks;
  if (units == 0) return cudaSuccess;
  merge_local_kernel<R, LPK><<<static_cast<unsigned>(units), kMergeWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_merge_local(const MergeParams& p, cudaStream_t stream) {
  switch (p.G < 8 ? p.G : 8) {
    case 1: return launch_merge_t<1, 8>(p, stream);
    case 2: return launch_merge_t<2, 8>(p, stream);
    case 3: return launch_merge_t<3, 8>(p, stream);
    case 4: return launch_merge_t<4, 8>(p, stream);
    case 5: return launch_merge_t<5, 16>(p, stream);
    case 6: return launch_merge_t<6, 16>(p, stream);
    case 7: return launch_merge_t<7, 16>(p, stream);
    default: return launch_merge_t<8, 16>(p, stream);
  }
}

}  // namespace nectar
