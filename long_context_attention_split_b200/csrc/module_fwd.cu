// (ii) Nectar module forward on the tensor cores, and the fused decode that
// adds (iii): Eq. (3.6) and Eqs. (3.4)-(3.5) of "Nectar: Neural Estimation
// of Cached-Token Attention via Regression" (§2.2, §2.4).
//
// One CTA per (layer l, KV head h, block of TPC query tokens).  Its N
// activation rows are the G query heads of those tokens (row g*TPC + t),
// fetched by one 4-D TMA box, so the rows that share a token -- and in the
// fused decode its local cache and causal mask -- sit in one CTA.
//
// Each layer is a swap-AB GEMM on tcgen05 (kind::f16, cta_group::1):
//   D[hidden unit, row] = W[hidden unit, :] . X[row, :]
// with M = 128 hidden units per tile (A = weight tile streamed by TMA from
// the packed blob, K-major, 128-byte swizzle), N = the CTA's rows (B = the
// activation matrix X = [q | h_{k-1}], resident in shared memory, K-major,
// 128-byte swizzle) and fp32 accumulators in TMEM, all M tiles of a layer
// side by side (mt * N <= 512 columns).  The epilogue warps read TMEM, add
// the bias, apply SiLU and write h_k back into X as bf16 (the re-injected q
// stays in X's first 128 columns).  The score readout is a dot product over
// X after the last hidden layer; the target readout is one more GEMM
// (M = d).
//
// Warp roles: 0 TMA producer, 1 MMA issuer (+ TMEM owner), 2..5 epilogue,
// and in the fused decode 6..9 compute the exact causal local attention of
// the CTA's tokens while the GEMMs run, then all merge in the epilogue.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "module_layout.h"

namespace nectar {

constexpr int kModStages = 4;                 // weight tiles in flight
constexpr int kWTileBytes = 128 * 128;        // 128 rows x 64 bf16
constexpr int kModEpiWarps = 4;
constexpr int kModLocWarps = 4;

struct ModSmem {
  // offsets in bytes from the 1024-aligned dynamic smem base
  uint32_t w, x, loc, sa, bars, tslot, total;
};

__host__ __device__ inline int mod_tmem_cols(int mt, int N) {
  int need = mt * N;
  int c = 32;
  while (c < need) c <<= 1;
  return c;
}

__host__ __device__ inline ModSmem mod_smem_layout(int Hmax, int N, bool fuse) {
  ModSmem s{};
  uint32_t off = 0;
  s.w = off;
  off += kModStages * kWTileBytes;
  s.x = off;
  off += static_cast<uint32_t>(2 + layout::kchunks(Hmax)) * N * 128;
  s.loc = off;
  // local (acc[d], m, l) per row, then the cross-warp scratch of the local warps
  if (fuse) off += static_cast<uint32_t>(N + kModLocWarps * 8) * (kD + 2) * 4;
  s.sa = off;
  off += static_cast<uint32_t>(N) * 4;                          // score a per row
  off = (off + 7) & ~7u;
  s.bars = off;
  off += 16 * 8;
  s.tslot = off;
  off += 16;
  s.total = off;
  return s;
}

// element (row n, column c) of the swizzled K-major activation matrix X
__device__ __forceinline__ uint32_t x_offset(int N, int n, int c) {
  return static_cast<uint32_t>((c >> 6) * (N * 128) + n * 128 + ((((c & 63) >> 3) ^ (n & 7)) << 4) +
                               ((c & 7) << 1));
}

__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.0f + ex2(-v * kLog2e)); }

// Exact causal local attention of the CTA's tokens (fused decode).  The 4
// local warps take one token at a time and split its visible local keys
// between them; the G rows of the token (in blocks of RG) share the loads.
// Result per activation row n: loc[n] = (acc[0..d), m, l) in log2 units.
template <int RG>
__device__ __forceinline__ void local_attention_rows(const ModParams& p, float* loc, int lw, int lane,
                                                     int64_t hd, int t0) {
  constexpr int LPK = RG <= 4 ? 8 : 16;
  using St = RowState<RG, LPK>;
  constexpr int NG = St::NG;
  constexpr int KPG = RG <= 4 ? 4 : 2;
  constexpr int kStride = kModLocWarps * NG;
  const int g = lane / LPK, tl = lane % LPK;
  float* scratch = loc + p.N * (kD + 2);   // [kModLocWarps][RG][kD + 2]
  const int64_t rows_per_head = static_cast<int64_t>(p.G) * p.nq;
  const int ltid = lw * 32 + lane;
  for (int t = 0; t < p.TPC; ++t) {
    const int64_t i = static_cast<int64_t>(t0) + t;
    if (i >= p.nq) break;
    int b;
    const int nv = visible_local(p.q_seq, p.q_pos, p.local_len, i, p.B, p.T, &b, p.err);
    for (int g0 = 0; g0 < p.G; g0 += RG) {
      const int nr = (p.G - g0 < RG) ? (p.G - g0) : RG;
      St st;
      st.reset();
      st.load_q(p.Q + (hd * rows_per_head + static_cast<int64_t>(g0) * p.nq + i) * kD, p.nq * kD, nr, tl, p.qmul);
      if (nv > 0) {
        const uint8_t* kb = reinterpret_cast<const uint8_t*>(p.Kloc + ((hd * p.B + b) * p.T) * kD);
        const uint8_t* vb = reinterpret_cast<const uint8_t*>(p.Vloc + ((hd * p.B + b) * p.T) * kD);
        for (int j0 = 0; j0 < nv; j0 += kStride * KPG) {
          const uint8_t* kr[KPG];
          const uint8_t* vr[KPG];
          bool valid[KPG];
#pragma unroll
          for (int k = 0; k < KPG; ++k) {
            const int j = j0 + k * kStride + lw * NG + g;
            valid[k] = j < nv;
            kr[k] = kb + static_cast<int64_t>(j) * kRowBytes;
            vr[k] = vb + static_cast<int64_t>(j) * kRowBytes;
          }
          st.template step<KPG>(kr, vr, valid, tl, GlobalLoader{});
        }
      }
      st.merge_groups();
      if (g == 0) {
        float* dst = scratch + (lw * RG) * (kD + 2);
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
      named_bar_sync(3, kModLocWarps * 32);
      for (int it = ltid; it < nr * kD; it += kModLocWarps * 32) {
        const int r = it / kD, dim = it % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kModLocWarps; ++w) M = fmaxf(M, scratch[(w * RG + r) * (kD + 2) + kD]);
        float ls = 0.f, as = 0.f;
#pragma unroll
        for (int w = 0; w < kModLocWarps; ++w) {
          const float* src = scratch + (w * RG + r) * (kD + 2);
          const float wgt = exp2_shift(src[kD], M);
          ls = fmaf(src[kD + 1], wgt, ls);
          as = fmaf(src[dim], wgt, as);
        }
        float* row = loc + ((g0 + r) * p.TPC + t) * (kD + 2);
        row[dim] = as;
        if (dim == 0) {
          row[kD] = M;
          row[kD + 1] = ls;
        }
      }
      named_bar_sync(3, kModLocWarps * 32);
    }
  }
}

template <bool kFuse, int RG>
__global__ void __launch_bounds__((6 + (kFuse ? kModLocWarps : 0)) * 32, 1)
module_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_q,
              const ModParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const ModSmem L = mod_smem_layout(p.Hmax, p.N, kFuse);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  const uint32_t b_wfull = smem_u32(bars + 0);          // [kModStages]
  const uint32_t b_wempty = smem_u32(bars + 4);         // [kModStages]
  const uint32_t b_qfull = smem_u32(bars + 8);
  const uint32_t b_acc = smem_u32(bars + 9);
  const uint32_t b_xready = smem_u32(bars + 10);
  const uint32_t b_loc = smem_u32(bars + 11);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.tslot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, TPC = p.TPC;

  // unit -> (layer, head, token block); layers visited widest first
  const int nblk = p.nblk;
  const int unit = blockIdx.x;
  const int li = unit / (p.Hkv * nblk);
  const int h = (unit / nblk) % p.Hkv;
  const int blk = unit % nblk;
  const int l = p.order[li];
  const int H = p.width[l];
  const int mt = (H + 127) / 128;
  const int depth = p.depth;
  const int64_t head_base = p.layer_base[l] + static_cast<int64_t>(h) * layout::head_elems(H, depth);
  const int64_t hd = static_cast<int64_t>(l) * p.Hkv + h;
  const int t0 = blk * TPC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kModStages; ++s) {
      mbar_init(b_wfull + 8 * s, 1);
      mbar_init(b_wempty + 8 * s, 1);
    }
    mbar_init(b_qfull, 1);
    mbar_init(b_acc, 1);
    mbar_init(b_xready, kModEpiWarps * 32);
    mbar_init(b_loc, kModLocWarps * 32);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  // zero the activation part of X (padding columns must read as 0)
  if (warp >= 2 && warp < 2 + kModEpiWarps) {
    uint4* xz = reinterpret_cast<uint4*>(smem + L.x + 2 * N * 128);
    const int n16 = layout::kchunks(p.Hmax) * N * 128 / 16;
    for (int i = threadIdx.x - 64; i < n16; i += kModEpiWarps * 32) xz[i] = make_uint4(0, 0, 0, 0);
    // rows of the q chunks past the G*TPC rows that TMA writes
    for (int i = threadIdx.x - 64; i < 2 * N * 8; i += kModEpiWarps * 32) {
      const int c = i / (N * 8), rem = i % (N * 8), n = rem / 8;
      if (n >= p.G * TPC) reinterpret_cast<uint4*>(smem + L.x + c * N * 128 + n * 128)[rem % 8] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_w);
      prefetch_tmap(&tmap_q);
      const uint64_t pol_w = policy_evict_first();
      mbar_arrive_expect_tx(b_qfull, 2 * p.G * TPC * 128);
      tma_load_4d(smem_u32(smem + L.x), &tmap_q, 0, t0, 0, static_cast<int>(hd), b_qfull, pol_w);
      tma_load_4d(smem_u32(smem + L.x + N * 128), &tmap_q, 64, t0, 0, static_cast<int>(hd), b_qfull, pol_w);
      uint32_t it = 0;
      bool ok = true;
      for (int net = 0; net < 2 && ok; ++net) {
        const int64_t nb = head_base + (net ? layout::net_elems(H, depth, 1) : 0);
        const int nlayers = depth + (net ? 1 : 0);
        for (int k = 0; k < nlayers && ok; ++k) {
          const bool out = (k == depth);
          const int kc = out ? layout::kchunks(H) : layout::kchunks(layout::hidden_k(H, k));
          const int mts = out ? 1 : mt;
          const int rows = out ? kD : H;
          const int64_t wrow = (nb + (out ? layout::out_w_off(H, depth) : layout::hidden_w_off(H, depth, k))) / 64;
          for (int m = 0; m < mts && ok; ++m)
            for (int c = 0; c < kc; ++c, ++it) {
              const uint32_t s = it % kModStages;
              if (it >= kModStages && !mbar_wait(b_wempty + 8 * s, ((it / kModStages) - 1) & 1, p.err)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(b_wfull + 8 * s, kWTileBytes);
              tma_load_2d(smem_u32(smem + L.w + s * kWTileBytes), &tmap_w, 0,
                          static_cast<int>(wrow + static_cast<int64_t>(c) * rows + m * 128), b_wfull + 8 * s,
                          pol_w);
            }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      bool ok = mbar_wait(b_qfull, 0, p.err);
      uint32_t it = 0, xr = 0;
      const uint32_t idesc = idesc_bf16_f32(128, N, 0, 0);
      const uint32_t xbase = smem_u32(smem + L.x);
      for (int net = 0; net < 2 && ok; ++net) {
        const int nlayers = depth + (net ? 1 : 0);
        for (int k = 0; k < nlayers && ok; ++k) {
          const bool out = (k == depth);
          if (net > 0 || k > 0) {
            ok = mbar_wait(b_xready, xr & 1, p.err);
            ++xr;
            if (!ok) break;
          }
          tc_fence_after();
          const int kc = out ? layout::kchunks(H) : layout::kchunks(layout::hidden_k(H, k));
          const int mts = out ? 1 : mt;
          const int cb = out ? 2 : 0;    // first X chunk read by this layer
          for (int m = 0; m < mts && ok; ++m)
            for (int c = 0; c < kc; ++c, ++it) {
              const uint32_t s = it % kModStages;
              if (!mbar_wait(b_wfull + 8 * s, (it / kModStages) & 1, p.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t wa = smem_u32(smem + L.w + s * kWTileBytes);
              const uint32_t xb = xbase + (cb + c) * N * 128;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + m * N, sdesc_sw128(wa + kk * 32, 16, 1024), sdesc_sw128(xb + kk * 32, 16, 1024),
                            idesc, (c | kk) != 0);
              mma_commit(b_wempty + 8 * s);
            }
          mma_commit(b_acc);
        }
      }
    }
  } else if (warp < 2 + kModEpiWarps) {
    // ------------------------------ epilogue ------------------------------
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int u = q4 * 32 + lane;            // accumulator row owned by this thread
    const int et = threadIdx.x - 64;         // 0..127
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const __nv_bfloat16* blob = p.blob;
    bool ok = true;
    uint32_t accp = 0;
    for (int net = 0; net < 2; ++net) {
      const int64_t nb = head_base + (net ? layout::net_elems(H, depth, 1) : 0);
      for (int k = 0; k < depth; ++k) {
        if (ok) ok = mbar_wait(b_acc, accp & 1, p.err);
        ++accp;
        tc_fence_after();
        const __nv_bfloat16* bias = blob + nb + layout::hidden_b_off(H, depth, k);
        for (int m = 0; m < mt; ++m) {
          const int i = m * 128 + u;
          const float bv = (ok && i < H) ? __bfloat162float(bias[i]) : 0.f;
          for (int n0 = 0; n0 < N; n0 += 16) {
            uint32_t v[16];
            NECTAR_TMEM_LD16(trow + m * N + n0, v);
            tmem_ld_wait();
            if (ok && i < H) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float y = silu(__uint_as_float(v[j]) + bv);
                *reinterpret_cast<__nv_bfloat16*>(smem + L.x + x_offset(N, n0 + j, kD + i)) = __float2bfloat16_rn(y);
              }
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (net == 0 && k == depth - 1) {
          // score readout a = w . h_{depth-1} + c from the bf16 activations in X
          named_bar_sync(2, kModEpiWarps * 32);
          const int tpc = 128 / N;          // threads per row
          const int n = et / tpc, part = et % tpc;
          const __nv_bfloat16* w = blob + nb + layout::out_w_off(H, depth);
          float s = 0.f;
          for (int i = part; i < H; i += tpc)
            s = fmaf(__bfloat162float(w[i]),
                     __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(smem + L.x + x_offset(N, n, kD + i))), s);
          for (int off = tpc >> 1; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
          if (part == 0) {
            s += __bfloat162float(blob[nb + layout::out_b_off(H, depth, 1)]);
            reinterpret_cast<float*>(smem + L.sa)[n] = s;
          }
          named_bar_sync(2, kModEpiWarps * 32);
        }
        mbar_arrive(b_xready);
      }
    }
    // target readout A_theta[row][u] = acc[u][row] + c[u], then (fused) the merge
    if (ok) ok = mbar_wait(b_acc, accp & 1, p.err);
    ++accp;
    if (kFuse && ok) ok = mbar_wait(b_loc, 0, p.err);
    tc_fence_after();
    const int64_t nbt = head_base + layout::net_elems(H, depth, 1);
    const float cb = __bfloat162float(blob[nbt + layout::out_b_off(H, depth, kD) + u]);
    const int64_t rows_per_head = static_cast<int64_t>(p.G) * p.nq;
    const float* sa = reinterpret_cast<const float*>(smem + L.sa);
    for (int n0 = 0; n0 < N; n0 += 16) {
      uint32_t v[16];
      NECTAR_TMEM_LD16(trow + n0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n0 + j;
        const int g = n / TPC, t = n % TPC;
        if (!ok || g >= p.G || t0 + t >= p.nq) continue;
        const int64_t row = hd * rows_per_head + static_cast<int64_t>(g) * p.nq + t0 + t;
        const float at = __uint_as_float(v[j]) + cb;
        if (!kFuse) {
          p.A_out[row * kD + u] = at;
          if (u == 0) p.a_out[row] = sa[n];
        } else {
          // merge with the local term of this row, Eqs. (3.4)-(3.5)
          const float* lr = reinterpret_cast<const float*>(smem + L.loc) + n * (kD + 2);
          const float ad = sa[n] * kLog2e;
          const float M = fmaxf(ad, lr[kD]);
          const float wd = exp2_shift(ad, M), wl = exp2_shift(lr[kD], M);
          p.out[row * kD + u] = (wd * at + wl * lr[u]) / (wd + wl * lr[kD + 1]);
        }
      }
    }
    tc_fence_before();
  } else if constexpr (kFuse) {
    // ------------------- local causal attention (fused decode) -------------------
    const int lw = warp - 2 - kModEpiWarps;
    local_attention_rows<RG>(p, reinterpret_cast<float*>(smem + L.loc), lw, lane, hd, t0);
    mbar_arrive(b_loc);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Rows per CTA: as many whole tokens (all G heads each) as fit in N <= 64,
// halved until the shared-memory plan fits.
ModShape mod_shape(int G, int64_t nq, int Hmax, bool fuse) {
  ModShape sh{};
  int tpc = 64 / G;
  if (tpc < 1) tpc = 1;
  if (tpc > nq) tpc = static_cast<int>(nq);
  while (true) {
    int N = (G * tpc + 15) / 16 * 16;
    if (N == 48) N = 64;   // the score readout splits 128 threads evenly over rows
    sh.TPC = tpc;
    sh.N = N;
    sh.smem = mod_smem_layout(Hmax, N, fuse).total + 1024;
    if (sh.smem <= 227 * 1024 || tpc == 1) break;
    tpc = (tpc + 1) / 2;
  }
  sh.nblk = static_cast<int>((nq + sh.TPC - 1) / sh.TPC);
  const int mt = (Hmax + 127) / 128;
  sh.tmem_cols = mod_tmem_cols(mt, sh.N);
  return sh;
}

template <bool kFuse, int RG>
static cudaError_t launch_module_t(const CUtensorMap& tw, const CUtensorMap& tq, const ModParams& p,
                                   int units, size_t smem, cudaStream_t stream) {
  auto kern = module_kernel<kFuse, RG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int threads = (6 + (kFuse ? kModLocWarps : 0)) * 32;
  kern<<<units, threads, smem, stream>>>(tw, tq, p);
  return cudaGetLastError();
}

cudaError_t launch_module(const CUtensorMap& tw, const CUtensorMap& tq, const ModParams& p, int units, size_t smem,
                          bool fuse, cudaStream_t stream) {
  if (!fuse) return launch_module_t<false, 1>(tw, tq, p, units, smem, stream);
  switch (p.G < 8 ? p.G : 8) {
    case 1: return launch_module_t<true, 1>(tw, tq, p, units, smem, stream);
    case 2: return launch_module_t<true, 2>(tw, tq, p, units, smem, stream);
    case 3: return launch_module_t<true, 3>(tw, tq, p, units, smem, stream);
    case 4: return launch_module_t<true, 4>(tw, tq, p, units, smem, stream);
    case 5: return launch_module_t<true, 5>(tw, tq, p, units, smem, stream);
    case 6: return launch_module_t<true, 6>(tw, tq, p, units, smem, stream);
    case 7: return launch_module_t<true, 7>(tw, tq, p, units, smem, stream);
    default: return launch_module_t<true, 8>(tw, tq, p, units, smem, stream);
  }
}

}  // namespace nectar
