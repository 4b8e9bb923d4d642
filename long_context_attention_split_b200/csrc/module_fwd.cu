// (ii) Nectar module forward on the tensor cores, and the Nectar decode that
// adds (iii): Eq. (3.6) and Eqs. (3.4)-(3.5) of "Nectar: Neural Estimation
// of Cached-Token Attention via Regression" (§2.2, §2.4).
//
// Module CTA: one per (layer l, KV head h, block of TPC query tokens), doing
// the score net and then the target net -- or, when every net streams at
// least 1 MB of weights (p.net_split), one per (l, h, block, net), so that
// the two nets' weight streams run side by side on different SMs.  Its N
// activation rows are the G query heads of those tokens (row g*TPC + t),
// fetched by one 4-D TMA box.
//
// Each layer is a swap-AB GEMM on tcgen05 (kind::f16, cta_group::1):
//   D[hidden unit, row] = W[hidden unit, :] . X[row, :]
// with M = 128 hidden units per tile (A = weight tile streamed from the
// packed blob, where it is stored pre-swizzled, by TMA bulk copies of one or
// two chunks: K-major, 128-byte swizzle), N = the CTA's rows (B = the
// activation matrix X = [q | h_{k-1}], resident in shared memory, K-major,
// 128-byte swizzle) and fp32 accumulators in TMEM, all M tiles of a layer
// side by side (mt * N <= 512 columns).  The epilogue warps read TMEM, add
// the bias, apply SiLU and write h_k back into X as bf16 (the re-injected q
// stays in X's first 128 columns).  The score readout is reduced from the
// registers of the last hidden layer's epilogue (w . bf16(h) per row, warp
// shuffles, then shared-memory atomics); the target readout is one more
// GEMM (M = d).  Warp roles: 0 TMA producer, 1 MMA issuer (+ TMEM owner),
// 2..5 epilogue.
//
// Decode: one launch holds two kinds of CTA side by side -- local CTAs, one
// per (KV head, query token), that stream the token's visible local K/V
// through shared memory and leave its exact causal attention state
// (acc[d], m, l) for every query head (local_attn.cuh), and module CTAs as
// above.  The module weights and the local caches are then read at the same
// time over the whole GPU.  A last small launch merges each row's document
// term (a_theta, A_theta) with its local state.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "local_attn.cuh"
#include "module_layout.h"
#include "out_layout.cuh"

namespace nectar {

constexpr int kModMaxStages = 12;             // weight stages (upper bound)
constexpr int kWTileBytes = 128 * 128;        // one chunk: 128 rows x 64 bf16
constexpr int kModEpiWarps = 4;
constexpr int kModThreads = 6 * 32;
constexpr int kDecLocCW = 4;                  // consumer warps of a local CTA
constexpr int kDecLocStages = 4;

struct ModSmem {
  // offsets in bytes from the 1024-aligned dynamic smem base
  uint32_t w, x, sa, bars, tslot, total;
};

__host__ __device__ inline int mod_tmem_cols(int mt, int N) {
  int need = mt * N;
  int c = 32;
  while (c < need) c <<= 1;
  return c;
}

__host__ __device__ inline ModSmem mod_smem_layout(int Hmax, int N, int stages, int cps) {
  ModSmem s{};
  uint32_t off = 0;
  s.w = off;
  off += static_cast<uint32_t>(stages) * cps * kWTileBytes;
  s.x = off;
  off += static_cast<uint32_t>(2 + layout::kchunks(Hmax)) * N * 128;
  s.sa = off;
  off += static_cast<uint32_t>(5 * N) * 4;                      // score partials [4][N], then a [N]
  off = (off + 15) & ~15u;
  s.bars = off;
  off += 32 * 8;
  s.tslot = off;
  off += 16;
  s.total = off;
  return s;
}

// shared memory of a local CTA of the decode launch
__host__ __device__ inline size_t dec_local_smem(int RG) {
  return size_t(kDecLocStages) * kLocStageBytes + size_t(kDecLocCW) * RG * (kD + 2) * 4 + 2 * kDecLocStages * 8;
}

__device__ __forceinline__ float mod_silu(float v) { return __fdividef(v, 1.0f + ex2(-v * kLog2e)); }

// element (row n, column c) of the swizzled K-major activation matrix X
__device__ __forceinline__ uint32_t x_offset(int N, int n, int c) {
  return static_cast<uint32_t>((c >> 6) * (N * 128) + n * 128 + ((((c & 63) >> 3) ^ (n & 7)) << 4) +
                               ((c & 7) << 1));
}

// One module CTA: (a_theta, A_theta) of the rows of `unit`.  smem is the
// 1024-aligned dynamic shared memory.  a goes to p.a_out[hd * rows + row],
// A_theta to p.A_out[(hd * rows + row) * d].
// kNetSplit: one net per CTA (p.net_split); a compile-time choice, so that
// the usual two-net CTA keeps constant loop bounds over the nets.
template <bool kNetSplit>
__device__ __forceinline__ void module_cta(const CUtensorMap* tmap_q, const ModParams& p, int unit, uint8_t* smem) {
  const ModSmem L = mod_smem_layout(p.Hmax, p.N, p.stages, p.cps);
  const uint32_t S = static_cast<uint32_t>(p.stages);
  const int CPS = p.cps;                                         // weight chunks per stage
  const uint32_t kStageBytes = static_cast<uint32_t>(CPS) * kWTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  const uint32_t b_wfull = smem_u32(bars + 0);                   // [kModMaxStages]
  const uint32_t b_wempty = smem_u32(bars + kModMaxStages);      // [kModMaxStages]
  const uint32_t b_qfull = smem_u32(bars + 2 * kModMaxStages);
  const uint32_t b_acc = smem_u32(bars + 2 * kModMaxStages + 1);
  const uint32_t b_xready = smem_u32(bars + 2 * kModMaxStages + 2);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.tslot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, TPC = p.TPC;

  // unit -> (layer, head, token block[, net]); layers visited widest first
  const int nlo = kNetSplit ? (unit & 1) : 0;                  // nets [nlo, nhi]: 0 score, 1 target
  const int nhi = kNetSplit ? (unit & 1) : 1;
  const int hunit = kNetSplit ? (unit >> 1) : unit;
  const int nblk = p.nblk;
  const int li = hunit / (p.Hkv * nblk);
  const int h = (hunit / nblk) % p.Hkv;
  const int blk = hunit % nblk;
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
  griddep_wait();                 // inputs and outputs only from here on (launched after another kernel)

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(tmap_q);
      const uint64_t pol_w = policy_evict_first();
      mbar_arrive_expect_tx(b_qfull, 2 * p.G * TPC * 128);
      tma_load_4d(smem_u32(smem + L.x), tmap_q, 0, t0, 0, static_cast<int>(hd), b_qfull, pol_w);
      tma_load_4d(smem_u32(smem + L.x + N * 128), tmap_q, 64, t0, 0, static_cast<int>(hd), b_qfull, pol_w);
      uint32_t it = 0;
      bool ok = true;
      for (int net = nlo; net <= nhi && ok; ++net) {
        const int64_t nb = head_base + (net ? layout::net_elems(H, depth, 1) : 0);
        const int nlayers = depth + net;                           // the target net adds its output GEMM
        for (int k = 0; k < nlayers && ok; ++k) {
          const bool out = (k == depth);
          const int Kk = out ? H : layout::hidden_k(H, k);
          const int kc = layout::kchunks(Kk);
          const int mts = out ? 1 : mt;
          const int rows = out ? kD : H;
          const __nv_bfloat16* wbase =
              p.blob + nb + (out ? layout::out_w_off(H, depth) : layout::hidden_w_off(H, depth, k));
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
              bulk_g2s(smem_u32(smem + L.w + s * kStageBytes), wbase + layout::tile_chunk_off(rows, Kk, m, c0),
                       bytes, b_wfull + 8 * s, pol_w);
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
      for (int net = nlo; net <= nhi && ok; ++net) {
        const int nlayers = depth + net;
        for (int k = 0; k < nlayers && ok; ++k) {
          const bool out = (k == depth);
          // the accumulators and X are free once the previous layer's
          // epilogue is done (in a CTA with both nets, also at the target's
          // first layer)
          if (net > nlo || k > 0) {
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
    for (int net = nlo; net <= nhi; ++net) {
      const int64_t nb = head_base + (net ? layout::net_elems(H, depth, 1) : 0);
      for (int k = 0; k < depth; ++k) {
        const __nv_bfloat16* bias = blob + nb + layout::hidden_b_off(H, depth, k);
        const bool readout = (net == 0 && k == depth - 1);   // score net: reduce w . h here
        const __nv_bfloat16* wsc = blob + nb + layout::out_w_off(H, depth);
        // this thread's biases (and readout weights) of the first 8 row tiles
        // do not depend on the accumulators: fetch them while the layer's
        // MMAs run (wider layers read the rest when they need them)
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
          for (int m0 = 0; m0 < mt; m0 += 2) {
            const int mc = (mt - m0 < 2) ? (mt - m0) : 2;     // warp-uniform
            uint32_t v[2][16];
#pragma unroll
            for (int mm = 0; mm < 2; ++mm)
              if (mm < mc) NECTAR_TMEM_LD16(trow + (m0 + mm) * N + n0, v[mm]);
            tmem_ld_wait();
#pragma unroll
            for (int mm = 0; mm < 2; ++mm) {
              const int i = (m0 + mm) * 128 + u;
              if (mm < mc && ok && i < H) {
                float bv = 0.f, wv = 0.f;
                if (m0 + mm < 8) {
#pragma unroll
                  for (int q = 0; q < 8; ++q)
                    if (q == m0 + mm) {
                      bv = bvs[q];
                      wv = wvs[q];
                    }
                } else {
                  bv = __bfloat162float(bias[i]);
                  wv = readout ? __bfloat162float(wsc[i]) : 0.f;
                }
                uint32_t ws[8];
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                  // two rows rounded to bf16 by one packed conversion
                  const uint32_t w = pack_bf16x2(mod_silu(__uint_as_float(v[mm][j]) + bv),
                                                 mod_silu(__uint_as_float(v[mm][j + 1]) + bv));
                  part[j] = fmaf(wv, bf16lo(w), part[j]);          // wv = 0 outside the readout layer
                  part[j + 1] = fmaf(wv, bf16hi(w), part[j + 1]);
                  ws[j >> 1] = w;
                }
                if (!readout) {
                  // h back into X (the readout layer's h is reduced, not stored)
#pragma unroll
                  for (int j = 0; j < 16; j += 2) {
                    *reinterpret_cast<uint16_t*>(smem + L.x + x_offset(N, n0 + j, kD + i)) =
                        static_cast<uint16_t>(ws[j >> 1] & 0xFFFFu);
                    *reinterpret_cast<uint16_t*>(smem + L.x + x_offset(N, n0 + j + 1, kD + i)) =
                        static_cast<uint16_t>(ws[j >> 1] >> 16);
                  }
                }
              }
            }
          }
          if (readout) {
            // sum over the hidden units: warp shuffles, then one slot per
            // warp and row, added in a fixed order below (deterministic)
#pragma unroll
            for (int j = 0; j < 16; ++j) {
#pragma unroll
              for (int off = 16; off >= 1; off >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], off);
            }
            if (lane == 0) {
#pragma unroll
              for (int j = 0; j < 16; ++j) sa[q4 * N + n0 + j] = part[j];
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (readout) {
          // score readout bias (the target net never touches sa)
          named_bar_sync(2, kModEpiWarps * 32);
          if (et < N)
            sa[4 * N + et] = ((sa[et] + sa[N + et]) + (sa[2 * N + et] + sa[3 * N + et])) +
                             __bfloat162float(blob[nb + layout::out_b_off(H, depth, 1)]);
        }
        mbar_arrive(b_xready);
      }
    }
    if (nlo == 0) {
      // score net: a[row] = its reduced readout (sa complete once every
      // epilogue thread has passed the readout layer)
      named_bar_sync(2, kModEpiWarps * 32);
      if (et < N && ok) {
        const int g = et / TPC, t = et % TPC;
        if (g < p.G && t0 + t < p.nq)
          p.a_out[hd * rows_per_head + static_cast<int64_t>(g) * p.nq + t0 + t] = sa[4 * N + et];
      }
    }
    if (nhi == 1) {
      // target net: A_theta[row][u] = acc[u][row] + c[u]
      const float cb =
          __bfloat162float(blob[head_base + layout::net_elems(H, depth, 1) + layout::out_b_off(H, depth, kD) + u]);
      if (ok) ok = mbar_wait(b_acc, accp & 1, p.err);
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
          p.A_out[row * kD + u] = __uint_as_float(v[j]) + cb;
        }
      }
    }
    tc_fence_before();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

// Standalone module forward.  Two CTAs per SM where the plan fits half an SM.
template <bool kNetSplit>
__global__ void __launch_bounds__(kModThreads, 2)
module_kernel(const __grid_constant__ CUtensorMap tmap_q, const ModParams p) {
  extern __shared__ uint8_t smem_raw[];
  module_cta<kNetSplit>(&tmap_q, p, blockIdx.x, aligned_smem(smem_raw));
}

// One local CTA of the decode: the exact causal attention state of every
// query head of token i over its visible local keys, left in the workspace
// as loc[(hd * rows + row) * (d + 2) + {acc[0..d), m, l}] (log2 units).
template <int RG>
__device__ __forceinline__ void local_state_cta(const ModParams& p, int64_t lunit, uint8_t* smem) {
  uint8_t* ring = smem;
  float* scratch = reinterpret_cast<float*>(smem + kDecLocStages * kLocStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + kDecLocCW * RG * (kD + 2));
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kDecLocStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t hd = lunit / p.nq, i = lunit % p.nq;
  const int64_t rows = static_cast<int64_t>(p.G) * p.nq;
  const LocalJobs J{p.q_seq, p.q_pos, p.local_len, p.Kloc, p.Vloc, p.B, p.T, p.G, p.err};
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecLocStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kDecLocCW);
    }
    fence_barrier_init();
  }
  __syncthreads();
  griddep_wait();
  if (warp == kDecLocCW) {
    if (lane == 0) local_produce<RG>(J, hd, i, 1, smem_u32(ring), kDecLocStages, full0, empty0);
  } else if (warp < kDecLocCW) {
    local_consume<RG, kDecLocCW>(J, hd, i, 1, p.Q + (hd * rows + i) * kD, p.nq * kD, p.qmul, ring, kDecLocStages,
                                 full0, empty0, scratch, 1, warp, lane,
                                 [&](int /*t*/, int g, int dim, float M, float ls, float as) {
                                   float* st = p.ws_loc + (hd * rows + static_cast<int64_t>(g) * p.nq + i) * (kD + 2);
                                   st[dim] = as;
                                   if (dim == 0) {
                                     st[kD] = M;
                                     st[kD + 1] = ls;
                                   }
                                 });
  }
}

// Decode launch: n_module module CTAs and n_local local CTAs.  When the
// local CTAs are short next to the module CTAs (p.module_first), the module
// CTAs come first in the grid, two per SM where there are enough, and the
// local CTAs fill the slots left, which keeps the bytes each SM streams
// closer to even; when they are long, they come first, so that they do not
// end the launch as a tail.
template <int RG, bool kNetSplit>
__global__ void __launch_bounds__(kModThreads, 2)
decode_kernel(const __grid_constant__ CUtensorMap tmap_q, const ModParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  const int64_t b = blockIdx.x;
  if (p.module_first) {
    if (b < p.n_module) module_cta<kNetSplit>(&tmap_q, p, static_cast<int>(b), smem);
    else local_state_cta<RG>(p, b - p.n_module, smem);
  } else {
    if (b < p.n_local) local_state_cta<RG>(p, b, smem);
    else module_cta<kNetSplit>(&tmap_q, p, static_cast<int>(b - p.n_local), smem);
  }
  griddep_launch();               // the merge may start launching
}

// Merge of every row's document term (a_theta from the workspace, A_theta
// in A_out) with its local state, Eqs. (3.4)-(3.5), into out (in place when
// A_out is out) or, bf16, into out_bf16 in the layer layout.
__global__ void decode_merge_kernel(const ModParams p, int64_t nrows) {
  griddep_wait();
  griddep_launch();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= nrows * kD) return;
  const int64_t row = idx / kD;
  const int dim = static_cast<int>(idx % kD);
  const float* st = p.ws_loc + row * (kD + 2);
  const float ad = p.a_out[row] * kLog2e;       // document logit in log2 units
  const float M = fmaxf(ad, st[kD]);
  const float wd = exp2_shift(ad, M), wl = exp2_shift(st[kD], M);
  const float v = (wd * p.A_out[idx] + wl * st[dim]) / (wd + wl * st[kD + 1]);
  if (p.out_bf16 != nullptr) p.out_bf16[layer_layout_index(row, dim, p.Hkv, p.G, p.nq)] = __float2bfloat16_rn(v);
  else p.out[idx] = v;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Rows per CTA: as many whole tokens (all G heads each) as fit in N <= 64,
// halved until the shared-memory plan fits; weight stages from what is left.
ModShape mod_shape(int G, int64_t nq, int Hmax, bool fuse) {
  ModShape sh{};
  constexpr size_t kFull = 227 * 1024;
  constexpr size_t kHalf = 113 * 1024;      // two CTAs per SM
  const int RG = G < 8 ? G : 8;
  const size_t floor_smem = fuse ? dec_local_smem(RG) + 1024 : 0;
  size_t kBudget = kFull;
  int tpc = 64 / G;
  if (tpc < 1) tpc = 1;
  if (tpc > nq) tpc = static_cast<int>(nq);
  const int mt = (Hmax + 127) / 128;
  while (true) {
    const int N = (G * tpc + 15) / 16 * 16;
    sh.TPC = tpc;
    sh.N = N;
    sh.smem = mod_smem_layout(Hmax, N, 3, 1).total + 1024;
    // the layer's M tiles sit side by side in TMEM: mt * N <= 512 columns
    if ((sh.smem <= kBudget && mt * N <= 512) || tpc == 1) break;
    tpc = (tpc + 1) / 2;
  }
  // plans that fit half an SM run two CTAs per SM
  if (sh.smem <= kHalf) kBudget = kHalf;
  int cps = 2;
  if (mod_smem_layout(Hmax, sh.N, 4, 2).total + 1024 > kBudget) cps = 1;
  int stages = 3;
  while (stages < kModMaxStages && mod_smem_layout(Hmax, sh.N, stages + 1, cps).total + 1024 <= kBudget) ++stages;
  sh.cps = cps;
  sh.stages = stages;
  sh.smem = mod_smem_layout(Hmax, sh.N, stages, cps).total + 1024;
  if (sh.smem < floor_smem) sh.smem = floor_smem;   // the decode's local CTAs share the launch
  sh.nblk = static_cast<int>((nq + sh.TPC - 1) / sh.TPC);
  sh.tmem_cols = mod_tmem_cols(mt, sh.N);
  return sh;
}

cudaError_t launch_module(const CUtensorMap& tq, const ModParams& p, int units, size_t smem, bool fuse,
                          cudaStream_t stream) {
  (void)fuse;
  if (p.net_split) {
    cudaError_t e = cudaFuncSetAttribute(module_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    module_kernel<true><<<units, kModThreads, smem, stream>>>(tq, p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(module_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    module_kernel<false><<<units, kModThreads, smem, stream>>>(tq, p);
  }
  return cudaGetLastError();
}

template <int RG, bool kNetSplit>
static cudaError_t launch_decode_s(const CUtensorMap& tq, const ModParams& q, size_t smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<RG, kNetSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(decode_kernel<RG, kNetSplit>, dim3(static_cast<unsigned>(q.n_local + q.n_module)), dim3(kModThreads),
                  smem, stream, 1, tq, q);
}

template <int RG>
static cudaError_t launch_decode_t(const CUtensorMap& tq, const ModParams& p, int units, size_t smem,
                                   cudaStream_t stream) {
  ModParams q = p;
  q.n_module = units;
  cudaError_t e = p.net_split ? launch_decode_s<RG, true>(tq, q, smem, stream)
                              : launch_decode_s<RG, false>(tq, q, smem, stream);
  if (e != cudaSuccess) return e;
  const int64_t nrows = static_cast<int64_t>(p.n_local / p.nq) * p.G * p.nq;
  const int64_t threads = nrows * kD;
  return launch_k(decode_merge_kernel, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, stream, 1, p,
                  nrows);
}

template <int RG>
static cudaError_t launch_local_t(const ModParams& p, cudaStream_t stream) {
  const size_t smem = dec_local_smem(RG) + 1024;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<RG, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  CUtensorMap unused{};                      // local CTAs read no tensor map
  ModParams q = p;
  q.n_module = 0;                            // every CTA a local CTA
  q.module_first = 0;
  decode_kernel<RG, false><<<static_cast<unsigned>(p.n_local), kModThreads, smem, stream>>>(unused, q);
  return cudaGetLastError();
}

// Local attention states only (every CTA a local CTA), into p.ws_loc.
cudaError_t launch_local_state(const ModParams& p, cudaStream_t stream) {
  switch (p.G < 8 ? p.G : 8) {
    case 1: return launch_local_t<1>(p, stream);
    case 2: return launch_local_t<2>(p, stream);
    case 3: return launch_local_t<3>(p, stream);
    case 4: return launch_local_t<4>(p, stream);
    case 5: return launch_local_t<5>(p, stream);
    case 6: return launch_local_t<6>(p, stream);
    case 7: return launch_local_t<7>(p, stream);
    default: return launch_local_t<8>(p, stream);
  }
}

cudaError_t launch_decode(const CUtensorMap& tq, const ModParams& p, int units, size_t smem, cudaStream_t stream) {
  switch (p.G < 8 ? p.G : 8) {
    case 1: return launch_decode_t<1>(tq, p, units, smem, stream);
    case 2: return launch_decode_t<2>(tq, p, units, smem, stream);
    case 3: return launch_decode_t<3>(tq, p, units, smem, stream);
    case 4: return launch_decode_t<4>(tq, p, units, smem, stream);
    case 5: return launch_decode_t<5>(tq, p, units, smem, stream);
    case 6: return launch_decode_t<6>(tq, p, units, smem, stream);
    case 7: return launch_decode_t<7>(tq, p, units, smem, stream);
    default: return launch_decode_t<8>(tq, p, units, smem, stream);
  }
}

}  // namespace nectar
