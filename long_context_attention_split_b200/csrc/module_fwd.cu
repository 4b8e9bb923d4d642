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
// with M = 128 hidden units per tile (A = weight tile streamed from the
// packed blob, where it is stored pre-swizzled, by one TMA bulk copy per
// tile: K-major, 128-byte swizzle), N = the CTA's rows (B = the
// activation matrix X = [q | h_{k-1}], resident in shared memory, K-major,
// 128-byte swizzle) and fp32 accumulators in TMEM, all M tiles of a layer
// side by side (mt * N <= 512 columns).  The epilogue warps read TMEM, add
// the bias, apply SiLU and write h_k back into X as bf16 (the re-injected q
// stays in X's first 128 columns).  The score readout is reduced from the
// registers of the last hidden layer's epilogue (w . bf16(h) per row, warp
// shuffles, then shared-memory atomics); the target readout is one more
// GEMM (M = d).
//
// Warp roles: 0 TMA producer, 1 MMA issuer (+ TMEM owner), 2..5 epilogue.
// In the fused decode, warp 6 streams the local K/V rows of the CTA's tokens
// into a ring of its own and warps 7.. compute their exact causal attention
// (local_attn.cuh) while the GEMMs run; the epilogue then merges.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "local_attn.cuh"
#include "module_layout.h"

namespace nectar {

constexpr int kModMaxStages = 12;             // weight stages (upper bound)
constexpr int kWTileBytes = 128 * 128;        // one chunk: 128 rows x 64 bf16
constexpr int kModEpiWarps = 4;
// local-attention warps of the fused decode (the local keys are a small part
// of its bytes; the rest of the SM's registers go to the epilogue)
__host__ __device__ constexpr int loc_warps(int RG) { return (void)RG, 4; }
__host__ __device__ constexpr int mod_threads(bool fuse, int RG) { return (6 + (fuse ? 1 + loc_warps(RG) : 0)) * 32; }
constexpr int kModLocStages = 2;              // local K/V ring of the fused decode

struct ModSmem {
  // offsets in bytes from the 1024-aligned dynamic smem base
  uint32_t w, x, lring, loc, scratch, sa, bars, tslot, total;
};

__host__ __device__ inline int mod_tmem_cols(int mt, int N) {
  int need = mt * N;
  int c = 32;
  while (c < need) c <<= 1;
  return c;
}

__host__ __device__ inline ModSmem mod_smem_layout(int Hmax, int N, bool fuse, int RG, int stages, int cps) {
  ModSmem s{};
  uint32_t off = 0;
  s.w = off;
  off += static_cast<uint32_t>(stages) * cps * kWTileBytes;
  s.x = off;
  off += static_cast<uint32_t>(2 + layout::kchunks(Hmax)) * N * 128;
  s.lring = off;
  if (fuse) off += kModLocStages * kLocStageBytes;
  s.loc = off;                                                   // local (acc[d], m, l) per row
  if (fuse) off += static_cast<uint32_t>(N) * (kD + 2) * 4;
  s.scratch = off;                                               // cross-warp join of the local warps
  if (fuse) off += static_cast<uint32_t>(loc_warps(RG) * RG) * (kD + 2) * 4;
  s.sa = off;
  off += static_cast<uint32_t>(N) * 4;                          // score a per row
  off = (off + 15) & ~15u;
  s.bars = off;
  off += 40 * 8;
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

template <bool kFuse, int RG>
__global__ void __launch_bounds__(mod_threads(kFuse, RG), 1)
module_kernel(const __grid_constant__ CUtensorMap tmap_q, const ModParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const ModSmem L = mod_smem_layout(p.Hmax, p.N, kFuse, RG, p.stages, p.cps);
  const uint32_t S = static_cast<uint32_t>(p.stages);
  const int CPS = p.cps;                                         // weight chunks per stage
  const uint32_t kStageBytes = static_cast<uint32_t>(CPS) * kWTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  const uint32_t b_wfull = smem_u32(bars + 0);                   // [kModMaxStages]
  const uint32_t b_wempty = smem_u32(bars + kModMaxStages);      // [kModMaxStages]
  const uint32_t b_qfull = smem_u32(bars + 2 * kModMaxStages);
  const uint32_t b_acc = smem_u32(bars + 2 * kModMaxStages + 1);
  const uint32_t b_xready = smem_u32(bars + 2 * kModMaxStages + 2);
  const uint32_t b_loc = smem_u32(bars + 2 * kModMaxStages + 3);
  const uint32_t b_lfull = smem_u32(bars + 2 * kModMaxStages + 4);                  // [kModLocStages]
  const uint32_t b_lempty = smem_u32(bars + 2 * kModMaxStages + 4 + kModLocStages);  // [kModLocStages]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.tslot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, TPC = p.TPC;

  // unit -> (layer, head, token block); layers visited widest first
  const int unit = blockIdx.x;
  const int nblk = p.nblk;
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
  const int64_t rows_per_head = static_cast<int64_t>(p.G) * p.nq;
  float* sa = reinterpret_cast<float*>(smem + L.sa);

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < S; ++s) {
      mbar_init(b_wfull + 8 * s, 1);
      mbar_init(b_wempty + 8 * s, 1);
    }
    mbar_init(b_qfull, 1);
    mbar_init(b_acc, 1);
    mbar_init(b_xready, kModEpiWarps * 32);
    mbar_init(b_loc, loc_warps(RG) * 32);
    for (int s = 0; s < kModLocStages; ++s) {
      mbar_init(b_lfull + 8 * s, 1);
      mbar_init(b_lempty + 8 * s, loc_warps(RG));
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 2 + kModEpiWarps) {
    // the activation part of X reads as 0 in its padding columns
    uint4* xz = reinterpret_cast<uint4*>(smem + L.x + 2 * N * 128);
    const int n16 = layout::kchunks(p.Hmax) * N * 128 / 16;
    for (int i = threadIdx.x - 64; i < n16; i += kModEpiWarps * 32) xz[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x - 64; i < N; i += kModEpiWarps * 32) sa[i] = 0.f;
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
      prefetch_tmap(&tmap_q);
      const uint64_t pol_w = policy_evict_first();
      mbar_arrive_expect_tx(b_qfull, 2 * p.G * TPC * 128);
      tma_load_4d(smem_u32(smem + L.x), &tmap_q, 0, t0, 0, static_cast<int>(hd), b_qfull, pol_w);
      tma_load_4d(smem_u32(smem + L.x + N * 128), &tmap_q, 64, t0, 0, static_cast<int>(hd), b_qfull, pol_w);
      uint32_t it = 0;
      bool ok = true;
      for (int net = 0; net < 2 && ok; ++net) {
      const int64_t nb = head_base + (net ? layout::net_elems(H, depth, 1) : 0);
      const int nlayers = depth + net;                           // the target net adds its output GEMM
      for (int k = 0; k < nlayers && ok; ++k) {
        const bool out = (k == depth);
        const int Kk = out ? H : layout::hidden_k(H, k);
        const int kc = layout::kchunks(Kk);
        const int mts = out ? 1 : mt;
        const int rows = out ? kD : H;
        const __nv_bfloat16* wbase = p.blob + nb + (out ? layout::out_w_off(H, depth) : layout::hidden_w_off(H, depth, k));
        for (int m = 0; m < mts && ok; ++m) {
          const int trows = layout::tile_rows(rows, m);
          for (int c0 = 0; c0 < kc; c0 += CPS, ++it) {
            const uint32_t s = it % S;
            if (it >= S && !mbar_wait(b_wempty + 8 * s, ((it / S) - 1) & 1, p.err)) {
              ok = false;
              break;
            }
            // chunks c0.. of row tile m: one contiguous, pre-swizzled block
            const int ncs = (kc - c0 < CPS) ? (kc - c0) : CPS;
            const uint32_t bytes = static_cast<uint32_t>(ncs * trows) * 128;
            mbar_arrive_expect_tx(b_wfull + 8 * s, bytes);
            bulk_g2s(smem_u32(smem + L.w + s * kStageBytes), wbase + layout::tile_chunk_off(rows, Kk, m, c0), bytes,
                     b_wfull + 8 * s, pol_w);
          }
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
      const int nlayers = depth + net;
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
        const int rows = out ? kD : H;
        for (int m = 0; m < mts && ok; ++m) {
          const uint32_t trows = static_cast<uint32_t>(layout::tile_rows(rows, m));
          for (int c0 = 0; c0 < kc; c0 += CPS, ++it) {
            const uint32_t s = it % S;
            if (!mbar_wait(b_wfull + 8 * s, (it / S) & 1, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int ncs = (kc - c0 < CPS) ? (kc - c0) : CPS;
            for (int cl = 0; cl < ncs; ++cl) {
              const uint32_t wa = smem_u32(smem + L.w + s * kStageBytes) + cl * trows * 128;
              const uint32_t xb = xbase + (cb + c0 + cl) * N * 128;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + m * N, sdesc_sw128(wa + kk * 32, 16, 1024), sdesc_sw128(xb + kk * 32, 16, 1024),
                            idesc, (c0 + cl + kk) != 0);
            }
            mma_commit(b_wempty + 8 * s);
          }
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
      const __nv_bfloat16* bias = blob + nb + layout::hidden_b_off(H, depth, k);
      const bool readout = (net == 0 && k == depth - 1);   // score net: reduce w . h here
      const __nv_bfloat16* wsc = blob + nb + layout::out_w_off(H, depth);
      // this thread's biases (and readout weights) do not depend on the
      // accumulators: fetch them while the layer's MMAs run
      float bvs[8], wvs[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i = m * 128 + u;
        bvs[m] = (m < mt && i < H) ? __bfloat162float(bias[i]) : 0.f;
        wvs[m] = (readout && m < mt && i < H) ? __bfloat162float(wsc[i]) : 0.f;
      }
      if (ok) ok = mbar_wait(b_acc, accp & 1, p.err);
      ++accp;
      tc_fence_after();
      for (int n0 = 0; n0 < N; n0 += 16) {
        float part[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) part[j] = 0.f;
        for (int m0 = 0; m0 < mt; m0 += 4) {
          const int mc = (mt - m0 < 4) ? (mt - m0) : 4;     // warp-uniform
          uint32_t v[4][16];
#pragma unroll
          for (int mm = 0; mm < 4; ++mm)
            if (mm < mc) NECTAR_TMEM_LD16(trow + (m0 + mm) * N + n0, v[mm]);
          tmem_ld_wait();
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) {
            const int i = (m0 + mm) * 128 + u;
            if (mm < mc && ok && i < H) {
              float bv = 0.f, wv = 0.f;
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (q == m0 + mm) {
                  bv = bvs[q];
                  wv = wvs[q];
                }
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const __nv_bfloat16 hb = __float2bfloat16_rn(silu(__uint_as_float(v[mm][j]) + bv));
                if (readout) part[j] = fmaf(wv, __bfloat162float(hb), part[j]);
                else *reinterpret_cast<__nv_bfloat16*>(smem + L.x + x_offset(N, n0 + j, kD + i)) = hb;
              }
            }
          }
        }
        if (readout) {
          // sum over the hidden units: warp shuffles, then one shared-memory
          // atomic per warp and row
#pragma unroll
          for (int j = 0; j < 16; ++j) {
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], off);
          }
          if (lane == 0) {
#pragma unroll
            for (int j = 0; j < 16; ++j) atomicAdd(sa + n0 + j, part[j]);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (readout) {
        // score readout bias (the target net never touches sa)
        named_bar_sync(2, kModEpiWarps * 32);
        if (et < N) sa[et] += __bfloat162float(blob[nb + layout::out_b_off(H, depth, 1)]);
      }
      mbar_arrive(b_xready);
    }
    }
    // target readout A_theta[row][u] = acc[u][row] + c[u], then (fused) the merge
    const float cb = __bfloat162float(blob[head_base + layout::net_elems(H, depth, 1) + layout::out_b_off(H, depth, kD) + u]);
    if (ok) ok = mbar_wait(b_acc, accp & 1, p.err);
    if (kFuse && ok) ok = mbar_wait(b_loc, 0, p.err);
    named_bar_sync(2, kModEpiWarps * 32);     // sa complete
    tc_fence_after();
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
    {
      const LocalJobs J{p.q_seq, p.q_pos, p.local_len, p.Kloc, p.Vloc, p.B, p.T, p.G, p.err};
      const int ntok = (p.nq - t0 < TPC) ? static_cast<int>(p.nq - t0) : TPC;
      if (warp == 2 + kModEpiWarps) {
        if (lane == 0) local_produce<RG>(J, hd, t0, ntok, smem_u32(smem + L.lring), kModLocStages, b_lfull, b_lempty);
      } else {
        const int cw = warp - 3 - kModEpiWarps;
        float* loc = reinterpret_cast<float*>(smem + L.loc);
        local_consume<RG, loc_warps(RG)>(
            J, hd, t0, ntok, p.Q + (hd * rows_per_head + t0) * kD, p.nq * kD, p.qmul, smem + L.lring,
            kModLocStages, b_lfull, b_lempty, reinterpret_cast<float*>(smem + L.scratch), 3, cw, lane,
            [&](int t, int g, int dim, float M, float ls, float as) {
              float* row = loc + (g * TPC + t) * (kD + 2);
              row[dim] = as;
              if (dim == 0) {
                row[kD] = M;
                row[kD + 1] = ls;
              }
            });
        mbar_arrive(b_loc);
      }
    }
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
  constexpr size_t kBudget = 227 * 1024;
  const int RG = G < 8 ? G : 8;
  int tpc = 64 / G;
  if (tpc < 1) tpc = 1;
  if (tpc > nq) tpc = static_cast<int>(nq);
  while (true) {
    const int N = (G * tpc + 15) / 16 * 16;
    sh.TPC = tpc;
    sh.N = N;
    sh.smem = mod_smem_layout(Hmax, N, fuse, RG, 3, 1).total + 1024;
    if (sh.smem <= kBudget || tpc == 1) break;
    tpc = (tpc + 1) / 2;
  }
  // weight stages: copies of 2 chunks (32 KB) with at least 5 in flight if
  // they fit, else smaller; then as many stages as shared memory takes
  int cps = 2;
  if (mod_smem_layout(Hmax, sh.N, fuse, RG, 4, 2).total + 1024 > kBudget) cps = 1;
  int stages = 3;
  while (stages < kModMaxStages && mod_smem_layout(Hmax, sh.N, fuse, RG, stages + 1, cps).total + 1024 <= kBudget)
    ++stages;
  sh.cps = cps;
  sh.stages = stages;
  sh.smem = mod_smem_layout(Hmax, sh.N, fuse, RG, stages, cps).total + 1024;
  sh.nblk = static_cast<int>((nq + sh.TPC - 1) / sh.TPC);
  const int mt = (Hmax + 127) / 128;
  sh.tmem_cols = mod_tmem_cols(mt, sh.N);
  return sh;
}

template <bool kFuse, int RG>
static cudaError_t launch_module_t(const CUtensorMap& tq, const ModParams& p, int units, size_t smem,
                                   cudaStream_t stream) {
  auto kern = module_kernel<kFuse, RG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units, 1, 1);
  cfg.blockDim = dim3(mod_threads(kFuse, RG), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, p);
}

cudaError_t launch_module(const CUtensorMap& tq, const ModParams& p, int units, size_t smem, bool fuse,
                          cudaStream_t stream) {
  if (!fuse) return launch_module_t<false, 1>(tq, p, units, smem, stream);
  switch (p.G < 8 ? p.G : 8) {
    case 1: return launch_module_t<true, 1>(tq, p, units, smem, stream);
    case 2: return launch_module_t<true, 2>(tq, p, units, smem, stream);
    case 3: return launch_module_t<true, 3>(tq, p, units, smem, stream);
    case 4: return launch_module_t<true, 4>(tq, p, units, smem, stream);
    case 5: return launch_module_t<true, 5>(tq, p, units, smem, stream);
    case 6: return launch_module_t<true, 6>(tq, p, units, smem, stream);
    case 7: return launch_module_t<true, 7>(tq, p, units, smem, stream);
    default: return launch_module_t<true, 8>(tq, p, units, smem, stream);
  }
}

}  // namespace nectar
