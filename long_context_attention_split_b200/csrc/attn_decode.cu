// (i) Exact cached-token attention, decode regime (few query rows per KV
// head): Eq. (3.1) of "Nectar: Neural Estimation of Cached-Token Attention
// via Regression" (§2.1), split over n and joined by log-sum-exp.
//
// Schedule.  The document of every (l, h) is cut into tiles of 128 keys (up
// to 2 query rows per pass) or 64 (more rows: their register state needs
// the room), and all
// heads' tiles are laid end to end (head-major).  CTA c of C takes the
// contiguous range [c*T/C, (c+1)*T/C) of that list, so every CTA streams the
// same number of bytes whatever n and the head count are; a CTA whose range
// crosses a head boundary emits one partial (m, l, acc) per head it touched.
// The combine kernel then joins, for each head, the partials of the CTAs
// that covered it -- a separate launch, so no CTA ever waits on another.
//
// Data movement.  One producer warp streams K and V tiles (32 or 16 KB each, whole
// contiguous rows) into a 3-stage ring with TMA bulk copies (evict-first L2
// policy: the document is read once); 8 consumer warps score and accumulate
// on the CUDA cores (see common.cuh).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

constexpr int kDecWarps = 8;
constexpr int kDecStages = 3;
constexpr int kDecThreads = (kDecWarps + 1) * 32;


// RW: query rows held by one warp (R rows in NRG groups of RW); TILE keys per tile.
template <int RW, int TILE>
__host__ __device__ constexpr size_t dec_smem_bytes() {
  return size_t(2) * kDecStages * TILE * kRowBytes            // K, V ring
         + size_t(kDecWarps) * RW * (kD + 2) * sizeof(float)  // cross-warp reduction
         + 2 * kDecStages * sizeof(uint64_t);                 // full / empty barriers
}

// R query rows per CTA pass, in NRG row groups: the consumer warps form NRG
// groups of kDecWarps / NRG, each group scores its RW = R / NRG rows against
// every key of a tile (the group's warps split the keys).  A warp's registers
// grow with RW, so 4 rows as 2 groups of 2 keep the 2-row register budget
// and two CTAs per SM, at the cost of reading each tile from shared memory
// twice.  With 64-key tiles, two CTAs per SM for up to 2 rows per warp
// (register cap 113); 128-key tiles fill most of an SM's shared memory with
// one CTA's ring, which then has the register file to itself.
template <int R, int LPK, int NRG>
__global__ void __launch_bounds__(kDecThreads, (dec_tile(R) == 64 && R / NRG <= 2 ? 2 : 1))
cache_attn_split_kernel(const DecParams p) {
  constexpr int TILE = dec_tile(R);
  constexpr int RW = R / NRG;
  constexpr int WPG = kDecWarps / NRG;       // warps per row group
  static_assert(RW * NRG == R && WPG * NRG == kDecWarps, "row groups");
  using St = RowState<RW, LPK>;
  constexpr int NG = St::NG;
  constexpr int KPW = TILE / WPG;            // keys per warp per tile
  constexpr int KPG = KPW / NG;              // keys per group per tile
  static_assert(KPG >= 1, "tile too small");
  static_assert(KPW * WPG == TILE && KPG * NG == KPW, "a tile's keys split evenly over the warps and lane groups");

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = smem + kDecStages * TILE * kRowBytes;
  float* sRed = reinterpret_cast<float*>(smem + 2 * kDecStages * TILE * kRowBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRed + kDecWarps * RW * (kD + 2));
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kDecStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(c) * p.total / p.C;
  const int64_t t1 = static_cast<int64_t>(c + 1) * p.total / p.C;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kDecWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kDecWarps) {
    // ---------------- producer ----------------
    // (no L2 prefetch of the first stages here: with 64-key tiles and two
    // CTAs per SM it made the launch 2x slower, 1.90 -> 3.9 ms on a
    // 32 x 8-head, 65536-key, 4-row document)
    griddep_wait();
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int64_t i = 0;
      for (int64_t tt = t0; tt < t1; ++tt, ++i) {
        const int s = static_cast<int>(i % kDecStages);
        if (i >= kDecStages && !mbar_wait(empty0 + 8 * s, static_cast<uint32_t>(((i / kDecStages) - 1) & 1), p.err))
          break;
        const int64_t hd = tt / p.tph;
        const int64_t j0 = (tt - hd * p.tph) * TILE;
        const int64_t cnt = (p.n - j0 < TILE) ? (p.n - j0) : TILE;
        const uint32_t bytes = static_cast<uint32_t>(cnt) * kRowBytes;
        const size_t off = (static_cast<size_t>(hd) * p.n + j0) * kD;
        mbar_arrive_expect_tx(full0 + 8 * s, 2 * bytes);
        bulk_g2s(smem_u32(sK + s * TILE * kRowBytes), p.K + off, bytes, full0 + 8 * s, pol);
        bulk_g2s(smem_u32(sV + s * TILE * kRowBytes), p.V + off, bytes, full0 + 8 * s, pol);
      }
    }
    griddep_launch();
    return;
  }
  griddep_wait();

  // ---------------- consumers ----------------
  const int g = lane / LPK, t = lane % LPK;
  const int rg = warp / WPG, wk = warp % WPG;   // row group, warp within it
  // rows of this pass (the last pass of a head may have fewer than R)
  const int rows_here = static_cast<int>((p.rows_total - p.row0 < R) ? (p.rows_total - p.row0) : R);
  const int nr_w = (rows_here - rg * RW < RW) ? (rows_here - rg * RW) : RW;   // may be <= 0
  St st;
  int64_t cur = -1;
  bool ok = true;

  auto finalize = [&](int64_t hd) {
    st.merge_groups();
    if (g == 0) {
      float* dst = sRed + (warp * RW) * (kD + 2);
#pragma unroll
      for (int r = 0; r < RW; ++r) {
#pragma unroll
        for (int ci = 0; ci < St::CPL; ++ci)
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[r * (kD + 2) + St::dim_of(t, ci, e)] = st.acc[r][ci * 8 + e];
        if (t == 0) {
          dst[r * (kD + 2) + kD] = st.m[r];
          dst[r * (kD + 2) + kD + 1] = st.l[r];
        }
      }
    }
    named_bar_sync(1, kDecWarps * 32);
    const int slot = c - first_cta_of_tile(hd * p.tph, p.total, p.C);
    for (int it = threadIdx.x; it < (NRG == 1 ? R : rows_here) * kD; it += kDecWarps * 32) {
      const int r = it / kD, dim = it % kD;
      const int wg0 = (r / RW) * WPG, rr = r % RW;   // the row's group: warps wg0 .. wg0 + WPG - 1
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < WPG; ++w) M = fmaxf(M, sRed[((wg0 + w) * RW + rr) * (kD + 2) + kD]);
      float ls = 0.f, as = 0.f;
#pragma unroll
      for (int w = 0; w < WPG; ++w) {
        const float* src = sRed + ((wg0 + w) * RW + rr) * (kD + 2);
        const float wgt = exp2_shift(src[kD], M);
        ls = fmaf(src[kD + 1], wgt, ls);
        as = fmaf(src[dim], wgt, as);
      }
      const int64_t prow = (hd * p.S_max + slot) * p.rows_total + p.row0 + r;
      p.ws_acc[prow * kD + dim] = as;
      if (dim == 0) {
        p.ws_ml[prow * 2] = M;
        p.ws_ml[prow * 2 + 1] = ls;
      }
    }
    named_bar_sync(1, kDecWarps * 32);
  };

  int64_t i = 0;
  for (int64_t tt = t0; tt < t1; ++tt, ++i) {
    const int64_t hd = tt / p.tph;
    if (hd != cur) {
      if (cur >= 0) finalize(cur);
      cur = hd;
      st.reset();
      if constexpr (NRG == 1) st.load_q(p.Q + (hd * p.rows_total + p.row0) * kD, kD, R, t, p.qmul);
      else st.load_q(p.Q + (hd * p.rows_total + p.row0 + rg * RW) * kD, kD, nr_w, t, p.qmul);
    }
    const int s = static_cast<int>(i % kDecStages);
    if (ok) ok = mbar_wait(full0 + 8 * s, static_cast<uint32_t>((i / kDecStages) & 1), p.err);
    if (ok) {
      const int64_t j0 = (tt - hd * p.tph) * TILE;
      const int cnt = static_cast<int>((p.n - j0 < TILE) ? (p.n - j0) : TILE);
      const uint8_t* kt = sK + s * TILE * kRowBytes;
      const uint8_t* vt = sV + s * TILE * kRowBytes;
      if constexpr (NRG == 1) {
        const uint8_t* kr[KPG];
        const uint8_t* vr[KPG];
        bool valid[KPG];
#pragma unroll
        for (int k = 0; k < KPG; ++k) {
          const int key = warp * KPW + k * NG + g;
          valid[k] = key < cnt;
          kr[k] = kt + key * kRowBytes;
          vr[k] = vt + key * kRowBytes;
        }
        st.template step<KPG>(kr, vr, valid, t, SmemLoader{});
      } else {
        // the warp's KPG keys per lane group, at most 2 per step (registers)
        constexpr int KS = KPG > 2 ? 2 : KPG;
#pragma unroll
        for (int k0 = 0; k0 < KPG; k0 += KS) {
          const uint8_t* kr[KS];
          const uint8_t* vr[KS];
          bool valid[KS];
#pragma unroll
          for (int k = 0; k < KS; ++k) {
            const int key = wk * KPW + (k0 + k) * NG + g;
            valid[k] = key < cnt;
            kr[k] = kt + key * kRowBytes;
            vr[k] = vt + key * kRowBytes;
          }
          st.template step<KS>(kr, vr, valid, t, SmemLoader{});
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
  }
  griddep_launch();               // the combine may start launching
  if (cur >= 0) finalize(cur);
}

// One warp per (head, row): join the partials of every CTA that covered the
// head.  alpha = ln2 * (M + log2 sum_s l_s 2^{m_s - M}), A = sum_s acc_s
// 2^{m_s - M} / sum_s l_s 2^{m_s - M}.
__global__ void cache_attn_combine_kernel(const DecParams p, float* __restrict__ alpha,
                                          float* __restrict__ A) {
  griddep_wait();
  griddep_launch();
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<int64_t>(p.heads) * p.rows_total) return;
  const int64_t hd = gw / p.rows_total, r = gw % p.rows_total;
  float4* out = reinterpret_cast<float4*>(A + gw * kD) + lane;
  if (p.tph == 0) {
    if (lane == 0) alpha[gw] = -INFINITY;
    *out = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const int f = first_cta_of_tile(hd * p.tph, p.total, p.C);
  const int la = first_cta_of_tile(hd * p.tph + p.tph - 1, p.total, p.C);
  const int ns = la - f + 1;                    // partials of this head
  const float* ml = p.ws_ml + (hd * p.S_max * p.rows_total + r) * 2;     // partial s at ml[s * rows_total * 2]
  const float* ac = p.ws_acc + (hd * p.S_max * p.rows_total + r) * kD;   // partial s at ac[s * rows_total * d]
  const int64_t sml = static_cast<int64_t>(p.rows_total) * 2, sac = static_cast<int64_t>(p.rows_total) * kD;
  // the first kFirst partials' value sums, this lane's 4 dims, loaded before
  // anything waits on them: with the (m, l) loads below, one round trip to L2
  // for a head of up to kFirst partials (a one-layer call: ~19)
  constexpr int kFirst = 24;
  float4 a4[kFirst];
#pragma unroll
  for (int j = 0; j < kFirst; ++j)
    a4[j] = j < ns ? reinterpret_cast<const float4*>(ac + j * sac)[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
  // the partials' maxima and row sums, one partial per lane
  float mv = -INFINITY, lv = 0.f;
  if (lane < ns) {
    mv = ml[lane * sml];
    lv = ml[lane * sml + 1];
  }
  float M = mv;
  for (int s = lane + 32; s < ns; s += 32) M = fmaxf(M, ml[s * sml]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  // weights 2^(m_s - M), the sum of the row weights, and the weighted sum of
  // the partial value sums
  float w = lane < ns ? exp2_shift(mv, M) : 0.f;
  float ls = lv * w;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < kFirst; ++j) {
    const float wj = __shfl_sync(0xffffffffu, w, j);
    acc.x = fmaf(a4[j].x, wj, acc.x);
    acc.y = fmaf(a4[j].y, wj, acc.y);
    acc.z = fmaf(a4[j].z, wj, acc.z);
    acc.w = fmaf(a4[j].w, wj, acc.w);
  }
  // partials past kFirst (heads cut over more CTAs), 32 at a time
  for (int s0 = kFirst; s0 < ns; s0 += 32) {
    const int sl = s0 + lane;
    const float wlow = __shfl_sync(0xffffffffu, w, sl & 31);   // partials < 32: lane sl holds the weight
    float w2 = 0.f;
    if (sl < ns) {
      if (sl >= 32) {
        w2 = exp2_shift(ml[sl * sml], M);
        ls = fmaf(ml[sl * sml + 1], w2, ls);
      } else {
        w2 = wlow;            // (its row sum was added with the first 32)
      }
    }
    const int cnt = ns - s0 < 32 ? ns - s0 : 32;
    for (int jj = 0; jj < cnt; ++jj) {
      const float wj = __shfl_sync(0xffffffffu, w2, jj);
      const float4 b4 = reinterpret_cast<const float4*>(ac + (s0 + jj) * sac)[lane];
      acc.x = fmaf(b4.x, wj, acc.x);
      acc.y = fmaf(b4.y, wj, acc.y);
      acc.z = fmaf(b4.z, wj, acc.z);
      acc.w = fmaf(b4.w, wj, acc.w);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  const float inv = 1.0f / ls;
  *out = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lane == 0) alpha[gw] = (M + log2f(ls)) * kLn2;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int R, int LPK, int NRG>
static cudaError_t launch_split(const DecParams& p, cudaStream_t stream) {
  if (p.tile != dec_tile(R)) return cudaErrorInvalidValue;   // planned for another tile size
  const size_t smem = dec_smem_bytes<R / NRG, dec_tile(R)>();
  cudaError_t e = cudaFuncSetAttribute(cache_attn_split_kernel<R, LPK, NRG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(cache_attn_split_kernel<R, LPK, NRG>, dim3(p.C), dim3(kDecThreads), smem, stream, 1, p);
}

int dec_max_rows() { return 8; }

// Resident CTAs per SM of the split kernel for R rows (occupancy calculator).
template <int R, int LPK, int NRG>
static int occ_t() {
  const size_t smem = dec_smem_bytes<R / NRG, dec_tile(R)>();
  if (cudaFuncSetAttribute(cache_attn_split_kernel<R, LPK, NRG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, cache_attn_split_kernel<R, LPK, NRG>, kDecThreads, smem) !=
      cudaSuccess)
    return 1;
  return n < 1 ? 1 : n;
}

int dec_ctas_per_sm(int R) {
  switch (R) {
    case 1: return occ_t<1, 8, 1>();
    case 2: return occ_t<2, 8, 1>();
    case 3:
    case 4: return occ_t<4, 8, 2>();
    case 5: return occ_t<5, 16, 1>();
    case 6: return occ_t<6, 16, 1>();
    case 7: return occ_t<7, 16, 1>();
    default: return occ_t<8, 16, 1>();
  }
}

size_t dec_smem_for_rows(int R) {
  switch (R) {
    case 1: return dec_smem_bytes<1, dec_tile(1)>();
    case 2: return dec_smem_bytes<2, dec_tile(2)>();
    case 3:
    case 4: return dec_smem_bytes<2, dec_tile(4)>();
    case 5: return dec_smem_bytes<5, dec_tile(5)>();
    case 6: return dec_smem_bytes<6, dec_tile(6)>();
    case 7: return dec_smem_bytes<7, dec_tile(7)>();
    default: return dec_smem_bytes<8, dec_tile(8)>();
  }
}

// Plan: tiles per head, total tiles, CTA count and partial slots per head.
DecPlan plan_decode(int heads, int64_t n, int num_sms, int ctas_per_sm, int tile) {
  DecPlan pl{};
  pl.tile = tile;
  pl.tph = (n + tile - 1) / tile;
  pl.total = static_cast<int64_t>(heads) * pl.tph;
  int64_t C = static_cast<int64_t>(num_sms) * ctas_per_sm;
  if (C > pl.total) C = pl.total;
  if (C < 1) C = 1;
  pl.C = static_cast<int>(C);
  pl.S_max = 0;
  if (pl.total > 0) {
    for (int64_t hd = 0; hd < heads; ++hd) {
      const int f = first_cta_of_tile(hd * pl.tph, pl.total, pl.C);
      const int la = first_cta_of_tile(hd * pl.tph + pl.tph - 1, pl.total, pl.C);
      if (la - f + 1 > pl.S_max) pl.S_max = la - f + 1;
    }
  }
  return pl;
}

cudaError_t launch_cache_attn_split(const DecParams& p, int R, cudaStream_t stream) {
  switch (R) {
    case 1: return launch_split<1, 8, 1>(p, stream);
    case 2: return launch_split<2, 8, 1>(p, stream);
    case 3:   // 3 rows run as 4, the last one empty
    case 4: return launch_split<4, 8, 2>(p, stream);
    case 5: return launch_split<5, 16, 1>(p, stream);
    case 6: return launch_split<6, 16, 1>(p, stream);
    case 7: return launch_split<7, 16, 1>(p, stream);
    case 8: return launch_split<8, 16, 1>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_cache_attn_combine(const DecParams& p, float* alpha, float* A, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(p.heads) * p.rows_total;
  if (warps == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  return launch_k(cache_attn_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream, 1, p,
                  alpha, A);
}

}  // namespace nectar
