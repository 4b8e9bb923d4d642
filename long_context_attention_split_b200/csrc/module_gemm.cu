// (ii) Nectar module forward for many query rows per KV head, layer by
// layer: Eq. (3.6) of "Nectar: Neural Estimation of Cached-Token Attention
// via Regression" (§2.4), with the Eq. (3.5) merge folded into the last
// layer when it serves the decode (§2.2).
//
// When a KV head has many query rows (a decode batch, a prompt), one CTA per
// block of 64 rows holding all hidden activations in shared memory would
// stream the head's weights once per block.  Here each hidden layer of both
// nets is instead one grouped GEMM over all (layer, KV head) pairs:
//   D[hidden unit, row] = W_k[hidden unit, :] . X[row, :],
//   X = q (k = 0) or [q | h_{k-1}] (k >= 1),
// on tcgen05 (kind::f16, cta_group::1): M = 128 hidden units (A = one row
// tile of the packed, pre-swizzled weights, fetched by bulk copies), N = up
// to 256 rows (B = rows of Q and of the previous layer's activations, by 2-D
// TMA boxes with the 128-byte swizzle), fp32 accumulators in TMEM.  The
// epilogue adds the bias, applies SiLU and stores h_k (bf16, row-major
// [rows][Hp]) for the next launch; the score net's last hidden layer is not
// stored but reduced at once against the readout row w (one fp32 partial per
// 128 hidden units and row).  A last launch runs the target readout GEMM
// (M = d), adds the score partials and the biases, and either writes
// (a_theta, A_theta) or merges them with each row's exact local attention
// state (decode).
//
// Module sets with a shared backbone (§2.4, App. A.3: depths D_b, D_s, D_t)
// take one launch per chain layer: launch s < D_b runs the backbone (its h
// in activation slot 0), later launches run layer s - D_b of each branch
// that has one (a branch's first layer reads slot 0, the others their own
// slot); the classic pair of nets is the case D_b = 0.
//
// Persistent CTAs (one per SM) walk a static list of tiles, widest layers
// first; the host gives each launch per-layer tables (head stride, weight
// offsets) so that decoding a tile costs a binary search and a few adds.
// Warp roles: 0 TMA producer, 1 MMA issuer (+ TMEM owner), 2..9 epilogue
// (two per TMEM lane quarter, alternating 32-column batches).  Two TMEM
// accumulators let the epilogue of one tile run under the MMAs of the next.
// Hidden-layer and readout launches are separate instances of the kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "module_layout.h"
#include "out_layout.cuh"

namespace nectar {

constexpr int kGemmEpiWarps = 8;             // two per TMEM lane quarter
constexpr int kGemmThreads = (2 + kGemmEpiWarps) * 32;
constexpr int kGemmWBytes = 128 * 128;        // one weight chunk: 128 rows x 64 bf16

__host__ __device__ inline uint32_t gemm_stage_bytes(int NR) {
  return (static_cast<uint32_t>(kGemmWBytes + NR * 128) + 1023u) & ~1023u;
}

struct GemmSmem {
  uint32_t ring, red, bars, tslot, total;
};

__host__ __device__ inline GemmSmem gemm_smem_layout(int NR, int stages) {
  GemmSmem s{};
  uint32_t off = 0;
  s.ring = off;
  off += static_cast<uint32_t>(stages) * gemm_stage_bytes(NR);
  s.red = off;                                    // score partials [4 warps][NR]
  off += 4u * NR * 4;
  off = (off + 15) & ~15u;
  s.bars = off;
  off += 2 * kGemmMaxStages * 8 + 4 * 8;
  s.tslot = off;
  off += 16;
  s.total = off;
  return s;
}

// SiLU of two pre-activations x = acc + b, packed to bf16x2.  With h = x / 2,
// SiLU(x) = x sigmoid(x) = h (1 + tanh h) = h + h tanh h: one tanh.approx
// (the hardware approximation, relative error ~2^-11) per value instead of
// an exp2 and a reciprocal, and the bias folded into the first (paired)
// FMA as b / 2.  The absolute error, |x| 2^-12 at most, stays below the
// bf16 rounding of the stored activation for |x| < 8.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t gemm_silu2(uint32_t acc0, uint32_t acc1, float half_bias) {
  const float2 h = ffma2(make_float2(__uint_as_float(acc0), __uint_as_float(acc1)), make_float2(0.5f, 0.5f),
                         make_float2(half_bias, half_bias));
  const float2 y = ffma2(h, make_float2(tanh_approx(h.x), tanh_approx(h.y)), h);
  return pack_bf16x2(y.x, y.y);
}

// One tile of the current launch: layer l, KV head hd, output part (0: the
// backbone or the score branch, 1: the target branch; the readout is part
// 1), 128-unit tile m, row tile rt -- and what the part's layer reads and
// where its weights are (offsets from the host's per-layer tables).
struct GemmTile {
  int l, net, m, rt;
  int64_t hd;
  int H;            // output units of this layer (d for the readout)
  int K;            // reduction length: d + the width of the h it reads (readout: the target width)
  int in_slot;      // h slot read for the columns past d
  int64_t w_off;    // blob offset of the layer's tiled weights
  int64_t b_off;    // blob offset of its bias
  int64_t aux_off;  // blob offset of the score readout's w (score_last) or c (readout)
  bool score_last;  // the score branch's last layer: its readout is fused
  int Hs;           // score width (readout: the number of partials per row)
};

template <bool kReadout>
__device__ __forceinline__ GemmTile gemm_tile(const GemmParams& p, int64_t t) {
  // the layer slot holding tile t: the last li with tile_start[li] <= t
  int lo = 0, hi = p.nlayers - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.tile_start[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int li = lo;
  GemmTile g;
  g.l = p.order[li];
  const int Db = p.depth_b, Ds = p.depth_s, Dt = p.depth_t;
  const int Hb = p.width_b[g.l], Hs = p.width_s[g.l], Ht = p.width_t[g.l];
  const int s = p.stage;
  const int j = s - Db;                                   // branch layer (s >= Db)
  int mt0, mt1;
  if (kReadout) {
    mt0 = 0;
    mt1 = 1;
  } else if (s < Db) {
    mt0 = (Hb + 127) / 128;
    mt1 = 0;
  } else {
    mt0 = j < Ds ? (Hs + 127) / 128 : 0;
    mt1 = j < Dt ? (Ht + 127) / 128 : 0;
  }
  int64_t rem = t - p.tile_start[li];
  g.rt = static_cast<int>(rem % p.rtiles);
  rem /= p.rtiles;
  const int mm = static_cast<int>(rem % (mt0 + mt1));
  const int h = static_cast<int>(rem / (mt0 + mt1));
  g.net = mm < mt0 ? 0 : 1;
  g.m = g.net ? mm - mt0 : mm;
  g.hd = static_cast<int64_t>(g.l) * p.Hkv + h;
  const int64_t hb = p.layer_base[g.l] + static_cast<int64_t>(h) * p.hstride[g.l];
  g.Hs = Hs;
  g.score_last = false;
  g.w_off = hb + p.woff[g.l][g.net];
  g.aux_off = hb + p.aux[g.l];
  if (kReadout) {
    g.H = kD;
    g.K = Ht;
    g.in_slot = 1;
  } else if (s < Db) {
    g.H = Hb;
    g.K = kD + (s > 0 ? Hb : 0);
    g.in_slot = 0;
  } else {
    g.H = g.net ? Ht : Hs;
    g.K = kD + layout::branch_prev(Db, Hb, g.H, j);
    g.in_slot = j == 0 ? 0 : g.net;                         // a branch's first layer reads the backbone
    g.score_last = g.net == 0 && j == Ds - 1;
  }
  g.b_off = g.w_off + layout::chunked_elems(g.H, g.K);     // the bias follows the tiled weights
  return g;
}

// Sum over the 32 lanes of v[j] for j = 0..31; lane j returns the total of
// row j (halving exchange: 31 shuffles instead of 160).
__device__ __forceinline__ float warp_transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < off; ++k) {
      const float send = upper ? v[k] : v[k + off];
      const float keep = upper ? v[k + off] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

// kReadout: the readout launch (target GEMM, merge epilogue) or a hidden
// layer; separate instances keep each launch's code to its own epilogue.
template <bool kReadout>
__global__ void __launch_bounds__(kGemmThreads, 1)
module_gemm_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_h,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NR = p.NR;
  const GemmSmem L = gemm_smem_layout(NR, p.stages);
  const uint32_t S = static_cast<uint32_t>(p.stages);
  const uint32_t SB = gemm_stage_bytes(NR);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  const uint32_t b_full = smem_u32(bars);
  const uint32_t b_empty = smem_u32(bars + kGemmMaxStages);
  const uint32_t b_accf = smem_u32(bars + 2 * kGemmMaxStages);       // [2]
  const uint32_t b_acce = smem_u32(bars + 2 * kGemmMaxStages + 2);   // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.tslot);
  float* red = reinterpret_cast<float*>(smem + L.red);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t heads = static_cast<int64_t>(p.L) * p.Hkv;
  const int R = p.R;

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < S; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_accf + 8 * b, 1);
      mbar_init(b_acce + 8 * b, kGemmEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  griddep_wait();                 // inputs and outputs only from here on (launched after another kernel)
  griddep_launch();

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_h);
      const uint64_t pol_w = policy_evict_last();     // weight tiles are re-read by the row tiles
      const uint64_t pol_x = policy_evict_normal();
      uint32_t it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
        const GemmTile g = gemm_tile<kReadout>(p, t);
        const int rows = g.H;
        const int K = g.K;
        const int kc = layout::kchunks(K);
        const __nv_bfloat16* wbase = p.blob + g.w_off;
        const uint32_t wbytes = static_cast<uint32_t>(layout::tile_rows(rows, g.m)) * 128;
        const int qrow = static_cast<int>(g.hd * R + static_cast<int64_t>(g.rt) * NR);
        const int hrow = static_cast<int>((g.in_slot * heads + g.hd) * R + static_cast<int64_t>(g.rt) * NR);
        const int qch = kReadout ? 0 : 2;             // leading chunks taken from q
        for (int c = 0; c < kc; ++c, ++it) {
          const uint32_t s = it % S;
          if (it >= S && !mbar_wait(b_empty + 8 * s, ((it / S) - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + L.ring + s * SB);
          mbar_arrive_expect_tx(b_full + 8 * s, wbytes + static_cast<uint32_t>(NR) * 128);
          bulk_g2s(dst, wbase + layout::tile_chunk_off(rows, K, g.m, c), wbytes, b_full + 8 * s, pol_w);
          if (c < qch) tma_load_2d(dst + kGemmWBytes, &tmap_q, c * 64, qrow, b_full + 8 * s, pol_x);
          else tma_load_2d(dst + kGemmWBytes, &tmap_h, (c - qch) * 64, hrow, b_full + 8 * s, pol_x);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, NR, 0, 0);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++tc) {
        const GemmTile g = gemm_tile<kReadout>(p, t);
        const int kc = layout::kchunks(g.K);
        const uint32_t b = tc & 1;
        if (tc >= 2 && !mbar_wait(b_acce + 8 * b, ((tc >> 1) - 1) & 1, p.err)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + b * static_cast<uint32_t>(NR);
        for (int c = 0; c < kc; ++c, ++it) {
          const uint32_t s = it % S;
          if (!mbar_wait(b_full + 8 * s, (it / S) & 1, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(smem + L.ring + s * SB);
          const uint32_t xb = wa + kGemmWBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(dacc, sdesc_sw128(wa + kk * 32, 16, 1024), sdesc_sw128(xb + kk * 32, 16, 1024), idesc,
                        (c | kk) != 0);
          mma_commit(b_empty + 8 * s);
        }
        if (ok) mma_commit(b_accf + 8 * b);
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int q4 = warp & 3;                  // TMEM lane quarter of this warp
    const int eh = (warp - 2) >> 2;           // which of the quarter's two warps
    const int et = threadIdx.x - 64;          // 0 .. 32 * kGemmEpiWarps - 1
    const int u = q4 * 32 + lane;             // accumulator lane: hidden unit or output dim
    const uint32_t tlane = static_cast<uint32_t>(q4 * 32) << 16;
    uint32_t tc = 0;
    bool ok = true;
    // A tile's decode and its per-thread constants (bias; the score
    // readout's w) are fetched one tile ahead, as raw bf16 bits, so that the
    // search over the per-layer tables and the global loads (~1.3 us a tile
    // on a per-tile timeline of stage 0, where the epilogue bounds the tile
    // rate) run under the previous tile's epilogue.
    const uint16_t* blob16 = reinterpret_cast<const uint16_t*>(p.blob);
    auto fetch = [&](int64_t tt, GemmTile& gg, uint16_t& braw, uint16_t& wraw) {
      gg = gemm_tile<kReadout>(p, tt);
      const int ii = gg.m * 128 + u;
      braw = 0;
      wraw = 0;
      if (kReadout) {
        braw = blob16[gg.b_off + u];
      } else if (ii < gg.H) {
        braw = blob16[gg.b_off + ii];
        if (gg.score_last) wraw = blob16[gg.aux_off + ii];
      }
    };
    GemmTile gnext{};
    uint16_t bnext = 0, wnext = 0;
    if (blockIdx.x < p.ntiles) fetch(blockIdx.x, gnext, bnext, wnext);
    for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++tc) {
      const GemmTile g = gnext;
      const float bias = __uint_as_float(static_cast<uint32_t>(bnext) << 16);
      const float wsc = __uint_as_float(static_cast<uint32_t>(wnext) << 16);
      if (t + gridDim.x < p.ntiles) fetch(t + gridDim.x, gnext, bnext, wnext);
      const uint32_t b = tc & 1;
      const int r0 = g.rt * NR;
      // rows of this tile; a 32-column batch may run 16 columns past NR
      const int rend = (R < r0 + NR) ? R : r0 + NR;
      const int i = g.m * 128 + u;
      const bool score_last = g.score_last;
      const float hbias = 0.5f * bias;
      if (ok) ok = mbar_wait_sleep(b_accf + 8 * b, (tc >> 1) & 1, p.err);   // waits out a main loop
      ok = __all_sync(0xffffffffu, ok);         // keeps the shuffles below warp-uniform
      tc_fence_after();
      const uint32_t dacc = tmem + tlane + b * static_cast<uint32_t>(NR);
      // the two warps of a lane quarter take alternate 32-column batches
      for (int n0 = 32 * eh; n0 < NR; n0 += 64) {
        uint32_t v[32];
        NECTAR_TMEM_LD32(dacc + n0, v);
        tmem_ld_wait();
        if (!ok) continue;
        if constexpr (!kReadout) {
          if (score_last) {
            float part[32];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              // bf16 rounding of two rows at once (one packed conversion)
              const uint32_t w = gemm_silu2(v[j], v[j + 1], hbias);
              part[j] = (i < g.H) ? wsc * bf16lo(w) : 0.f;
              part[j + 1] = (i < g.H) ? wsc * bf16hi(w) : 0.f;
            }
            const float tot = warp_transpose_sum32(part, lane);
            if (n0 + lane < NR) red[q4 * NR + n0 + lane] = tot;
          } else {
            const int Hp = p.Hp;
            const int64_t hrow0 = (g.net * heads + g.hd) * R;
            if (i < layout::round64(g.H)) {
              // column i of rows r0 + n0 .. ; 32-bit offsets from one base
              uint16_t* hb = reinterpret_cast<uint16_t*>(p.h_out) + (hrow0 + r0 + n0) * Hp + i;
              const int nrow = rend - (r0 + n0);       // rows of this batch inside the tile
              const bool live = i < g.H;
              if (nrow >= 32) {
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                  const uint32_t w = live ? gemm_silu2(v[j], v[j + 1], hbias) : 0u;
                  hb[j * Hp] = static_cast<uint16_t>(w & 0xFFFFu);
                  hb[(j + 1) * Hp] = static_cast<uint16_t>(w >> 16);
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                  const uint32_t w = live ? gemm_silu2(v[j], v[j + 1], hbias) : 0u;
                  if (j < nrow) hb[j * Hp] = static_cast<uint16_t>(w & 0xFFFFu);
                  if (j + 1 < nrow) hb[(j + 1) * Hp] = static_cast<uint16_t>(w >> 16);
                }
              }
            }
          }
        } else {
          // readout: u = output dim; a per row from the score partials
          float a_l = 0.f;
          {
            const int r = r0 + n0 + lane;
            if (r < rend) {
              const float* pr = p.part + (g.hd * R + r) * p.MT;
              const int mts = (g.Hs + 127) / 128;
              for (int m = 0; m < mts; ++m) a_l += pr[m];
              a_l += __bfloat162float(p.blob[g.aux_off]);
              if (q4 == 0 && p.a_out != nullptr) p.a_out[g.hd * R + r] = a_l;
            }
          }
          const int nrow = rend - (r0 + n0);          // rows of this batch inside the tile
          float* arow = p.A_out + (g.hd * R + r0 + n0) * kD + u;
          if (p.ws_loc == nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nrow) arow[j * kD] = __uint_as_float(v[j]) + bias;
          } else if (nrow > 0) {
            // merge with the row's local state (decode).  Lane j forms the two
            // weights of row j once (an exp2 pair and a division per row, not
            // per element); then every lane loads its dim of all the batch's
            // local sums at once (row index clamped into the tile), so the 32
            // loads are in flight together, and combines.
            const float* st0 = p.ws_loc + (g.hd * R + r0 + n0) * (kD + 2);
            const float* stl = st0 + (lane < nrow ? lane : 0) * (kD + 2);
            const float ml = stl[kD], ll = stl[kD + 1];
            const float ad = a_l * kLog2e;                  // document logit, log2 units
            const float M = fmaxf(ad, ml);
            const float wd = exp2_shift(ad, M), wl = exp2_shift(ml, M);
            const float inv = 1.0f / (wd + wl * ll);
            const float cd = wd * inv, cl = wl * inv;
            float xs[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) xs[j] = st0[(j < nrow ? j : 0) * (kD + 2) + u];
            float mv[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              mv[j] = __shfl_sync(0xffffffffu, cd, j) * (__uint_as_float(v[j]) + bias) +
                      __shfl_sync(0xffffffffu, cl, j) * xs[j];
            if (p.out_bf16 == nullptr) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nrow) arow[j * kD] = mv[j];
            } else {
              const int64_t row0 = g.hd * R + r0 + n0;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nrow)
                  p.out_bf16[layer_layout_index(row0 + j, u, p.Hkv, p.G, p.nq)] = __float2bfloat16_rn(mv[j]);
            }
          }
        }
      }
      // this tile's accumulator may be overwritten now
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_acce + 8 * b);
      if (score_last) {
        named_bar_sync(2, kGemmEpiWarps * 32);
        for (int n = et; n < NR; n += kGemmEpiWarps * 32) {
          const int r = r0 + n;
          if (ok && r < rend)
            p.part[(g.hd * R + r) * p.MT + g.m] = (red[n] + red[NR + n]) + (red[2 * NR + n] + red[3 * NR + n]);
        }
        named_bar_sync(2, kGemmEpiWarps * 32);
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
// max_rows: rows per tile at most (256 for the hidden layers; the readout
// picks its own, see readout_rows)
GemmShape gemm_shape(int64_t R, int max_rows) {
  GemmShape sh{};
  sh.rtiles = static_cast<int>((R + max_rows - 1) / max_rows);
  const int64_t per = (R + sh.rtiles - 1) / sh.rtiles;
  sh.NR = static_cast<int>((per + 15) / 16 * 16);
  constexpr size_t kBudget = 227 * 1024;
  int stages = 2;
  while (stages < kGemmMaxStages && gemm_smem_layout(sh.NR, stages + 1).total + 1024 <= kBudget) ++stages;
  sh.stages = stages;
  sh.smem = gemm_smem_layout(sh.NR, stages).total + 1024;
  // two accumulators of NR columns; the epilogue reads in 32-column batches,
  // so the second one's last batch may reach NR % 32 columns past 2 NR
  const int need = 2 * sh.NR + (sh.NR % 32 ? 32 - sh.NR % 32 : 0);
  int c = 32;
  while (c < need) c <<= 1;
  sh.tmem_cols = c;
  return sh;
}

cudaError_t launch_module_gemm(const CUtensorMap& tq, const CUtensorMap& th, const GemmParams& p, int grid,
                               size_t smem, cudaStream_t stream) {
  if (p.readout) {
    cudaError_t e = cudaFuncSetAttribute(module_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_k(module_gemm_kernel<true>, dim3(grid), dim3(kGemmThreads), smem, stream, 1, tq, th, p);
  }
  cudaError_t e = cudaFuncSetAttribute(module_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(module_gemm_kernel<false>, dim3(grid), dim3(kGemmThreads), smem, stream, 1, tq, th, p);
}

}  // namespace nectar
