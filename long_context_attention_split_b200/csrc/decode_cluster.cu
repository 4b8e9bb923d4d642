// Nectar decode for few query rows per KV head, one thread-block cluster per
// (layer l, KV head h): the score and target nets of Eq. (3.6) and the merge
// of Eqs. (3.4)-(3.5) with the exact causal attention over the local tokens
// (§2.2, §2.4 of "Nectar: Neural Estimation of Cached-Token Attention via
// Regression"), all in one launch and with no workspace.
//
// Why a cluster.  At a few query rows per KV head the module forward is a
// weight stream: every weight is used once per row.  One CTA per (l, h)
// streams the head's whole module through one SM, which is slow when a call
// has few heads (one layer of a model run layer after layer: 8 heads on 148
// SMs).  Here the hidden units of every layer of each net are cut into 8
// slices of a multiple of 64 units, and the cluster's CTAs share them: with
// 8 CTAs each holds one slice of both nets; with 16 (a non-portable cluster
// size) CTAs 0-7 hold the score net's slices and 8-15 the target net's, so
// that a CTA's weights fit its shared-memory ring whole.
//
// Per CTA (slice si = rank mod 8, units [u0, u0 + slen) of each net it holds):
//  - hidden layer k: the rows of W_k for its units (A, swap-AB: M = 128
//    units -- a 64-unit slice uses the lanes 0-63 of an M = 128 tile whose
//    other rows it ignores --, N = the head's query rows, K = d or d + H),
//    streamed from the packed blob by bulk copies through a ring, times
//    X = [q | h_{k-1}] (B, resident, K-major, 128-byte swizzle) into TMEM;
//    the epilogue adds the bias, applies SiLU, writes its slice of h_k into
//    its own X as bf16 and copies that slice into the X of the other CTAs
//    holding the same net (DSMEM bulk copies that complete on the receiver's
//    mbarrier: point to point, no multicast).  The next layer starts once
//    every slice has landed.  Depth >= 3 alternates two h buffers, so that
//    a buffer is written again only two layers after it was sent, when every
//    receiver has it (and so every copy out of it has read it); the target's
//    last layer writes a region of its own, the readout's input.
//  - last hidden layer: the score net's readout w . h is summed over the
//    CTA's units in the epilogue registers; the target net's readout
//    W_out[:, slice] h_slice is one more MMA (M = d, K = the slice).
//  - local attention: 4 warps score the CTA's share of every query token's
//    visible local keys (the keys cut into one range per CTA) on the CUDA
//    cores, leaving a partial (m, l, acc) per row.
//  - reduction and merge: each CTA owns d / cluster output dims.  Every
//    CTA stores its partials into the owners' shared memory (score partial
//    of each row to all, target and local partials of each dim to that
//    dim's owner), one cluster barrier, and each owner sums the partials in
//    a fixed order (deterministic), joins the local partials by
//    log-sum-exp and merges: out = (2^{a'} A_theta + 2^{m} acc) /
//    (2^{a'} + 2^{m} l) with a' = a_theta log2 e (Eqs. (3.4)-(3.5)).
// Warp roles: 0 TMA producer, 1 MMA issuer (+ TMEM owner), 2-5 and 6-9 the
// epilogues of the CTA's first and second net (with one net per CTA, 6-9
// only join the barriers), 10-13 local attention; all take part in the
// merge.  Every mbarrier wait is bounded; every thread reaches both cluster
// barriers (no early return).
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "module_layout.h"
#include "out_layout.cuh"

namespace nectar {

namespace {

constexpr uint32_t kStage = 32 * 1024;           // weight ring stage
constexpr uint32_t kPad = 8 * 1024;              // read (not used) past the ring by a 64-row tile
constexpr int kEpiWarps = 8;
constexpr int kLocWarps = 4;
constexpr int kThreads = (2 + kEpiWarps + kLocWarps) * 32;
constexpr int kLocKPG = 2;                        // keys per lane group per step
constexpr int kMaxStages = 8;
constexpr int kMaxSliceTiles = 4;                 // 128-unit M tiles of a slice (H <= 2048, 4 slices)

struct ClSmem {
  uint32_t ring, xq, xh, xro, rt, rl, rs, rml, sp, lscr, bars, tslot, total;
};

// Slices of each net's hidden units: one per CTA holding that net, so
// cluster * nets per CTA / 2.  64-unit granules: the h slices exchanged
// between CTAs are whole 64-column chunks of X.
__host__ __device__ constexpr int cl_slices(int kC, int npc) { return kC * npc / 2; }
__host__ __device__ inline int cl_slice(int H, int ksl) {
  const int s = (H + ksl - 1) / ksl;
  return (s + 63) / 64 * 64;
}
__host__ __device__ inline int cl_slice_len(int H, int si, int ksl) {
  const int S = cl_slice(H, ksl);
  const int len = H - si * S;
  return len < 0 ? 0 : (len < S ? len : S);
}
// rows of the partials exchanged in the reduction: R rounded up to 4
__host__ __device__ inline int cl_rp(int R) { return (R + 3) / 4 * 4; }

// byte offsets from the 1024-aligned dynamic shared memory base, for a
// cluster of kC CTAs each holding npc nets
__host__ __device__ inline ClSmem cl_layout(int kC, int npc, int Hmax, int N, int R, int nb, int stages, int rg) {
  ClSmem s{};
  const int own = kD / kC, Rp = cl_rp(R), ksl = cl_slices(kC, npc);
  uint32_t off = 0;
  s.ring = off;
  off += static_cast<uint32_t>(stages) * kStage + kPad;
  s.xq = off;                                                   // q: 2 chunks of [N][128 B]
  off += 2u * N * 128;
  s.xh = off;                                                   // h: [net][buf][chunk][N][128 B]
  off += static_cast<uint32_t>(npc * nb * layout::kchunks(Hmax) * N * 128);
  s.xro = off;                                                  // the target readout's input: own slice
  off += static_cast<uint32_t>(layout::kchunks(cl_slice(Hmax, ksl))) * N * 128;
  s.rt = off;                                                   // target partials [slice][dim][row]
  off += static_cast<uint32_t>(ksl * own * Rp) * 4;
  s.rl = off;                                                   // local acc partials [cta][row][dim]
  off += static_cast<uint32_t>(kC * Rp * own) * 4;
  s.rs = off;                                                   // score partials [slice][row]
  off += static_cast<uint32_t>(ksl * Rp) * 4;
  s.rml = off;                                                  // local (m, l) [cta][row][2]
  off += static_cast<uint32_t>(kC * Rp * 2) * 4;
  s.sp = off;                                                   // score sums by lane quarter [4][N]
  off += static_cast<uint32_t>(4 * N) * 4;
  s.lscr = off;                                                 // local warps' states [warp][rg][d + 2]
  off += static_cast<uint32_t>(kLocWarps * rg * (kD + 2)) * 4;
  off = (off + 15) & ~15u;
  s.bars = off;
  off += 32 * 8;
  s.tslot = off;
  off += 16;
  s.total = off;
  return s;
}

__device__ __forceinline__ uint8_t* cl_aligned(uint8_t* raw) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float cl_silu(float v) { return __fdividef(v, 1.0f + ex2(-v * kLog2e)); }

// element (row n, column c) of a swizzled K-major [N][64]-chunk matrix
__device__ __forceinline__ uint32_t cl_xoff(int N, int n, int c) {
  return static_cast<uint32_t>((c >> 6) * (N * 128) + n * 128 + ((((c & 63) >> 3) ^ (n & 7)) << 4) +
                               ((c & 7) << 1));
}

template <int RG, int kC, int kNPC>
__global__ void __launch_bounds__(kThreads, 1)
decode_cluster_kernel(const ClusterParams p) {
  constexpr int kSl = cl_slices(kC, kNPC);           // slices of each net
  constexpr int kOwn = kD / kC;                      // output dims merged by each CTA
  static_assert((kC == 8 && (kNPC == 1 || kNPC == 2)) || (kC == 16 && kNPC == 1),
                "8 CTAs holding one or both nets, or 16 holding one");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = cl_aligned(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = static_cast<int>(cluster_ctarank());
  const int si = r % kSl;                           // slice of the units
  const int n0 = kNPC == 1 ? r / kSl : 0;           // the CTA's first net (0 score, 1 target)
  const int pbase = kNPC == 1 ? n0 * kSl : 0;       // rank of slice 0 of the CTA's nets
  const bool has_target = n0 + kNPC - 1 == 1;
  const int ci = static_cast<int>(blockIdx.x) / kC;
  const int li = ci / p.Hkv, h = ci % p.Hkv;
  const int l = p.order[li];
  const int H = p.width[l];
  const int depth = p.depth;
  const int N = p.N;
  const int nb = p.nb;
  const int HC = layout::kchunks(p.Hmax);
  const int S_ = p.stages;
  const int R = p.G * static_cast<int>(p.nq);               // query rows of the head (<= N)
  const int Rp = cl_rp(R);
  const ClSmem SL = cl_layout(kC, kNPC, p.Hmax, N, R, nb, S_, RG);
  const int S = cl_slice(H, kSl);
  const int u0 = si * S;
  const int slen = cl_slice_len(H, si, kSl);
  const int MT = (slen + 127) / 128;                       // M tiles of the slice (0: empty slice)
  const int MTmax = (cl_slice(p.Hmax, kSl) + 127) / 128;   // TMEM columns are planned for the widest layer
  const int64_t sbase = p.layer_base[l] + static_cast<int64_t>(h) * layout::head_elems(H, depth);
  const int64_t tbase = sbase + layout::net_elems(H, depth, 1);
  const int64_t hd = static_cast<int64_t>(l) * p.Hkv + h;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL.bars);
  const uint32_t b_full = smem_u32(bars);                   // [kMaxStages]
  const uint32_t b_empty = smem_u32(bars + kMaxStages);     // [kMaxStages]
  const uint32_t b_q = smem_u32(bars + 2 * kMaxStages);
  const uint32_t b_acc = smem_u32(bars + 2 * kMaxStages + 1);   // [2]: one per local net
  const uint32_t b_hr = smem_u32(bars + 2 * kMaxStages + 3);    // [2]: h_k of every slice landed, k parity
  const uint32_t b_ror = smem_u32(bars + 2 * kMaxStages + 5);   // target h_{D-1} slice written
  const uint32_t b_rof = smem_u32(bars + 2 * kMaxStages + 6);   // readout accumulated
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + SL.tslot);
  const uint32_t xq = smem_u32(smem + SL.xq);
  const uint32_t xh = smem_u32(smem + SL.xh);
  const uint32_t ring = smem_u32(smem + SL.ring);
  const uint32_t xro = smem_u32(smem + SL.xro);
  // X chunk c of local net j as layer input: q (c < 2) or chunk c - 2 of h buffer `buf`
  auto xchunk = [&](int j, int buf, int c) -> uint32_t {
    return c < 2 ? xq + static_cast<uint32_t>(c * N * 128)
                 : xh + static_cast<uint32_t>(((j * nb + buf) * HC + (c - 2)) * N * 128);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S_; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, 1);
    }
    mbar_init(b_q, 1);
    mbar_init(b_acc, 1);
    mbar_init(b_acc + 8, 1);
    mbar_init(b_hr, kNPC);         // the nets' epilogue leaders; the peers' slices as transactions
    mbar_init(b_hr + 8, kNPC);
    mbar_init(b_ror, 1);
    mbar_init(b_rof, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  if (warp >= 2) {
    // h buffers start at 0 (their padding columns are read as 0 by the MMA);
    // q rows past the R that TMA writes are 0
    const int t = threadIdx.x - 64, nt = kThreads - 64;
    uint4* xz = reinterpret_cast<uint4*>(smem + SL.xh);
    const int n16 = static_cast<int>((SL.rt - SL.xh) / 16);    // h buffers and the readout input
    for (int i = t; i < n16; i += nt) xz[i] = make_uint4(0, 0, 0, 0);
    for (int i = t; i < 2 * N * 8; i += nt) {
      const int c = i / (N * 8), rem = i % (N * 8), n = rem / 8;
      if (n >= R) reinterpret_cast<uint4*>(smem + SL.xq + c * N * 128 + n * 128)[rem % 8] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();              // every CTA's barriers are initialised before any DSMEM traffic
  tc_fence_after();
  const uint32_t tmem = *tslot;
  griddep_launch();                // the next kernel may take the SMs this call leaves idle

  // (an L2 prefetch of the CTA's weights before the wait measured slower:
  // 17.4 against 15.4 us per Qwen3-1.7B layer in a graph)
  griddep_wait();                  // inputs and outputs are touched only from here on

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; k < depth && ok; ++k) {
        const int K = layout::hidden_k(H, k), kc = layout::kchunks(K);
        for (int j = 0; j < kNPC && ok; ++j) {
          const __nv_bfloat16* W = p.blob + (n0 + j ? tbase : sbase) + layout::hidden_w_off(H, depth, k);
          for (int t = 0; t < MT && ok; ++t) {
            const int gu = u0 + 128 * t, m = gu >> 7, r0 = gu & 127;
            const int rv = (slen - 128 * t < 128) ? (slen - 128 * t) : 128;
            const int rvp = rv <= 64 ? 64 : 128;
            const int cpg = static_cast<int>(kStage / (rvp * 128));
            const bool whole = (r0 == 0 && rv == 128);              // whole 128-row tiles are contiguous
            for (int c0 = 0; c0 < kc; c0 += cpg, ++it) {
              const uint32_t s = it % S_;
              if (it >= static_cast<uint32_t>(S_) && !mbar_wait(b_empty + 8 * s, ((it / S_) - 1) & 1, p.err)) {
                ok = false;
                break;
              }
              const int nc = (kc - c0 < cpg) ? (kc - c0) : cpg;
              mbar_arrive_expect_tx(b_full + 8 * s, static_cast<uint32_t>(nc * rv * 128));
              const uint32_t dst = ring + s * kStage;
              if (whole) {
                bulk_g2s(dst, W + layout::tile_chunk_off(H, K, m, c0), static_cast<uint32_t>(nc * 128 * 128),
                         b_full + 8 * s, pol);
              } else {
                // a slice that starts inside a 128-row tile of the blob takes
                // its first rows from tile m and the rest from tile m + 1
                const int r1 = rv < 128 - r0 ? rv : 128 - r0;
                for (int cl = 0; cl < nc; ++cl) {
                  bulk_g2s(dst + cl * rvp * 128, W + layout::tile_chunk_off(H, K, m, c0 + cl) + r0 * 64,
                           static_cast<uint32_t>(r1 * 128), b_full + 8 * s, pol);
                  if (rv > r1)
                    bulk_g2s(dst + cl * rvp * 128 + r1 * 128, W + layout::tile_chunk_off(H, K, m + 1, c0 + cl),
                             static_cast<uint32_t>((rv - r1) * 128), b_full + 8 * s, pol);
                }
              }
            }
          }
        }
      }
      if (ok && has_target && MT > 0) {
        // the target readout's K range: chunks of the slice of W_out [d][H]
        const __nv_bfloat16* Wo = p.blob + tbase + layout::out_w_off(H, depth);
        const int cb = u0 / 64, nch = (slen + 63) / 64;
        for (int c0 = 0; c0 < nch; c0 += 2, ++it) {
          const uint32_t s = it % S_;
          if (it >= static_cast<uint32_t>(S_) && !mbar_wait(b_empty + 8 * s, ((it / S_) - 1) & 1, p.err)) break;
          const int nc = (nch - c0 < 2) ? (nch - c0) : 2;
          mbar_arrive_expect_tx(b_full + 8 * s, static_cast<uint32_t>(nc * 128 * 128));
          bulk_g2s(ring + s * kStage, Wo + layout::tile_chunk_off(kD, H, 0, cb + c0),
                   static_cast<uint32_t>(nc * 128 * 128), b_full + 8 * s, pol);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      bool ok = mbar_wait(b_q, 0, p.err);
      const uint32_t idesc = idesc_bf16_f32(128, N, 0, 0);
      const uint64_t dK = sdesc_sw128(0, 16, 1024);    // K-major, 128-byte swizzle, at address 0
      int s = 0;                                      // ring stage and its phase
      uint32_t ph = 0;
      auto next_stage = [&]() {
        if (++s == S_) {
          s = 0;
          ph ^= 1u;
        }
      };
      for (int k = 0; k < depth && ok; ++k) {
        if (k > 0) {
          // every slice of h_{k-1} (of the CTA's nets) is in this CTA's X
          ok = mbar_wait_cluster(b_hr + 8 * ((k - 1) & 1), ((k - 1) >> 1) & 1, p.err);
          if (!ok) break;
          fence_proxy_async_smem();    // the peers' stores, to the tensor core's reads
        }
        tc_fence_after();
        const int kc = layout::kchunks(layout::hidden_k(H, k));
        const int buf = (k - 1 + nb) % nb;
        for (int j = 0; j < kNPC && ok; ++j) {
          if (MT == 0) continue;
          for (int t = 0; t < MT && ok; ++t) {
            const int rv = (slen - 128 * t < 128) ? (slen - 128 * t) : 128;
            const int rvp = rv <= 64 ? 64 : 128;
            const int cpg = static_cast<int>(kStage / (rvp * 128));
            const uint32_t dcol = tmem + static_cast<uint32_t>((j * MTmax + t) * N);
            for (int c0 = 0; c0 < kc; c0 += cpg) {
              // (bulk copies into the ring and the MMAs' reads of it are both
              // async-proxy operations ordered by the barrier; no tcgen05
              // fence is needed here, and one per stage costs ~0.1 us)
              if (!mbar_wait(b_full + 8 * s, ph, p.err)) {
                ok = false;
                break;
              }
              const int nc = (kc - c0 < cpg) ? (kc - c0) : cpg;
              for (int cl = 0; cl < nc; ++cl) {
                const uint64_t da = sdesc_at(dK, ring + s * kStage + cl * rvp * 128);
                const uint64_t db = sdesc_at(dK, xchunk(j, buf, c0 + cl));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // 16 columns (32 bytes) of K per MMA
                  mma_bf16_ss(dcol, da + 2 * kk, db + 2 * kk, idesc, (c0 + cl + kk) != 0);
              }
              mma_commit(b_empty + 8 * s);
              next_stage();
            }
          }
          mma_commit(b_acc + 8 * j);
        }
      }
      if (ok && has_target && MT > 0) {
        // target readout: A_theta partial [d][rows] over this CTA's units
        ok = mbar_wait(b_ror, 0, p.err);
        tc_fence_after();
        const int nch = (slen + 63) / 64;
        const uint32_t dcol = tmem + static_cast<uint32_t>(kNPC * MTmax * N);
        for (int c0 = 0; c0 < nch && ok; c0 += 2) {
          if (!mbar_wait(b_full + 8 * s, ph, p.err)) {
            ok = false;
            break;
          }
          const int nc = (nch - c0 < 2) ? (nch - c0) : 2;
          for (int cl = 0; cl < nc; ++cl) {
            const uint64_t da = sdesc_at(dK, ring + s * kStage + cl * 128 * 128);
            const uint64_t db = sdesc_at(dK, xro + static_cast<uint32_t>((c0 + cl) * N * 128));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(dcol, da + 2 * kk, db + 2 * kk, idesc, (c0 + cl + kk) != 0);
          }
          mma_commit(b_empty + 8 * s);
          next_stage();
        }
        mma_commit(b_rof);
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------ epilogues ------------------------------
    const int j = (warp - 2) >> 2;                   // local net of this warp group
    const int q4 = warp & 3;                         // TMEM lane quarter of this warp
    const int et = ((warp - 2) & 3) * 32 + lane;     // 0..127 within the group
    if (j == 0) {
      // the head's R query rows (contiguous, 256 bytes each) into X's q
      // chunks, 16 bytes per load, swizzled as the MMA reads them; a few
      // hundred bytes, so plain loads: the TMA unit keeps to the weights
      const uint4* qg = reinterpret_cast<const uint4*>(p.Q + hd * R * kD);
      for (int i = et; i < R * 16; i += 128) {
        const int n = i >> 4, c16 = i & 15;
        const uint4 v = qg[i];
        *reinterpret_cast<uint4*>(smem + SL.xq + (c16 >> 3) * N * 128 + n * 128 + (((c16 & 7) ^ (n & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (et == 0) mbar_arrive(b_q);
    }
    if (j < kNPC) {
      const int net = n0 + j;                        // 0 score, 1 target
      const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
      const int64_t nbase = net ? tbase : sbase;
      float* sp = reinterpret_cast<float*>(smem + SL.sp);
      bool ok = true;
      uint32_t peer = 0;                             // bytes of h_k the other slices send here
      for (int o = 0; o < kSl; ++o) {
        const int sl = cl_slice_len(H, o, kSl);
        if (o != si && sl > 0) peer += static_cast<uint32_t>((sl + 63) / 64 * N * 128);
      }
      for (int k = 0; k < depth; ++k) {
        const bool last = (k == depth - 1);
        const int buf = k % nb;
        const bool reduce = last && net == 0;           // the score readout: w . h summed here
        if (MT > 0) {
          // this thread's biases (and score readout weights), read while the
          // layer's MMAs run
          const __nv_bfloat16* bias = p.blob + nbase + layout::hidden_b_off(H, depth, k);
          const __nv_bfloat16* wsc = p.blob + sbase + layout::out_w_off(H, depth);
          float bvr[kMaxSliceTiles], wvr[kMaxSliceTiles];
#pragma unroll
          for (int t = 0; t < kMaxSliceTiles; ++t) {
            const int u = t * 128 + q4 * 32 + lane;
            const bool valid = t < MT && u < slen;
            bvr[t] = valid ? __bfloat162float(bias[u0 + u]) : 0.f;
            wvr[t] = (valid && reduce) ? __bfloat162float(wsc[u0 + u]) : 0.f;
          }
          if (ok) ok = mbar_wait(b_acc + 8 * j, k & 1, p.err);
          tc_fence_after();
          for (int n0r = 0; n0r < N; n0r += 16) {
            float part[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) part[jj] = 0.f;
#pragma unroll
            for (int t = 0; t < kMaxSliceTiles; ++t) {
              if (t >= MT) break;
              const int u = t * 128 + q4 * 32 + lane;
              const bool valid = u < slen && ok;
              const int gu = u0 + u;
              const float bv = bvr[t];
              const float wv = wvr[t];
              uint32_t v[16];
              NECTAR_TMEM_LD16(trow + static_cast<uint32_t>((j * MTmax + t) * N + n0r), v);
              tmem_ld_wait();
              if (valid) {
#pragma unroll
                for (int jj = 0; jj < 16; jj += 2) {
                  const uint32_t w = pack_bf16x2(cl_silu(__uint_as_float(v[jj]) + bv),
                                                 cl_silu(__uint_as_float(v[jj + 1]) + bv));
                  if (reduce) {
                    part[jj] = fmaf(wv, bf16lo(w), part[jj]);
                    part[jj + 1] = fmaf(wv, bf16hi(w), part[jj + 1]);
                  } else {
                    // h_k into the h buffer (to be exchanged), or -- the target's
                    // last layer -- into the readout input, columns from the slice start
                    uint8_t* dst = last ? smem + SL.xro : smem + SL.xq + (xchunk(j, buf, 2) - xq);
                    const int col = last ? u : gu;
                    *reinterpret_cast<uint16_t*>(dst + cl_xoff(N, n0r + jj, col)) = static_cast<uint16_t>(w & 0xFFFFu);
                    *reinterpret_cast<uint16_t*>(dst + cl_xoff(N, n0r + jj + 1, col)) = static_cast<uint16_t>(w >> 16);
                  }
                }
              }
            }
            if (reduce) {
              // the warp's 32 units summed for each of the 16 rows by a
              // halving transpose (16 shuffles, not 16 x 5): after it, lanes
              // 2 r and 2 r + 1 hold row r's sum
#pragma unroll
              for (int off = 16, nv = 8; off >= 2; off >>= 1, nv >>= 1) {
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int q = 0; q < nv; ++q) {
                  const float send = upper ? part[q] : part[q + nv];
                  const float keep = upper ? part[q + nv] : part[q];
                  part[q] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
              }
              const float tot = part[0] + __shfl_xor_sync(0xffffffffu, part[0], 1);
              if ((lane & 1) == 0) sp[q4 * N + n0r + (lane >> 1)] = tot;
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(1 + j, 128);
        if (!last) {
          const uint32_t hr = b_hr + 8 * (k & 1);
          // own arrival, expecting the other slices of this net as transactions
          if (et == 0) mbar_arrive_expect_tx(hr, peer);
          if (MT > 0) {
            // this slice of h_k into the same place of every other CTA holding
            // the net: 16-byte stores by the group's threads, each completing
            // its bytes on the receiver's barrier (point to point, no multicast)
            const uint32_t src = xchunk(j, buf, 2 + u0 / 64);
            const int n16 = (slen + 63) / 64 * N * 8;
            for (int i = et; i < n16; i += 128) {
              const uint4 v = ld_shared_v4(src + 16 * i);
#pragma unroll
              for (int o = 0; o < kSl; ++o)
                if (o != si) st_async_v4(mapa_shared(src + 16 * i, pbase + o), v, mapa_shared(hr, pbase + o));
            }
          }
        } else if (net == 0) {
          // score partial of every row, to every CTA
          if (et < Rp) {
            const float v = (MT > 0 && et < R) ? (sp[et] + sp[N + et]) + (sp[2 * N + et] + sp[3 * N + et]) : 0.f;
            const uint32_t dst = smem_u32(smem + SL.rs) + static_cast<uint32_t>((si * Rp + et) * 4);
            for (int o = 0; o < kC; ++o) st_cluster_f32(mapa_shared(dst, o), v);
          }
        } else {
          // target readout partial [dim][row], to the owner of the dim
          const int dim = q4 * 32 + lane;
          const int o = dim / kOwn, dl = dim % kOwn;
          const uint32_t dst =
              mapa_shared(smem_u32(smem + SL.rt) + static_cast<uint32_t>(((si * kOwn + dl) * Rp) * 4), o);
          if (MT > 0) {
            if (et == 0) mbar_arrive(b_ror);
            if (ok) ok = mbar_wait(b_rof, 0, p.err);
            tc_fence_after();
            for (int n0r = 0; n0r < Rp; n0r += 16) {
              uint32_t v[16];
              NECTAR_TMEM_LD16(trow + static_cast<uint32_t>(kNPC * MTmax * N + n0r), v);
              tmem_ld_wait();
#pragma unroll
              for (int jj = 0; jj < 16; jj += 4)
                if (n0r + jj < Rp)
                  st_cluster_v4f(dst + (n0r + jj) * 4, __uint_as_float(v[jj]), __uint_as_float(v[jj + 1]),
                                 __uint_as_float(v[jj + 2]), __uint_as_float(v[jj + 3]));
            }
          } else {
            for (int n = 0; n < Rp; n += 4) st_cluster_v4f(dst + n * 4, 0.f, 0.f, 0.f, 0.f);
          }
        }
      }
      tc_fence_before();
    }
  } else {
    // ------------------------------ local attention ------------------------------
    using St = RowState<RG, 16>;
    constexpr int NG = St::NG;
    constexpr int KPS = kLocWarps * NG * kLocKPG;    // keys per step of the 4 warps
    const int lw = warp - 2 - kEpiWarps;
    const int g = lane / 16, tl = lane % 16;
    float* lscr = reinterpret_cast<float*>(smem + SL.lscr);
    const int gblocks = (p.G + RG - 1) / RG;
    const uint32_t rl0 = smem_u32(smem + SL.rl), rml0 = smem_u32(smem + SL.rml);
    for (int t = 0; t < static_cast<int>(p.nq); ++t) {
      int b = 0;
      const int nv = visible_local(p.q_seq, p.q_pos, p.local_len, t, p.B, p.T, &b, p.err);
      const int lo = static_cast<int>(static_cast<int64_t>(nv) * r / kC);
      const int hi = static_cast<int>(static_cast<int64_t>(nv) * (r + 1) / kC);
      const uint8_t* kb = reinterpret_cast<const uint8_t*>(p.Kloc) + ((hd * p.B + b) * p.T) * kRowBytes;
      const uint8_t* vb = reinterpret_cast<const uint8_t*>(p.Vloc) + ((hd * p.B + b) * p.T) * kRowBytes;
      for (int gb = 0; gb < gblocks; ++gb) {
        const int g0 = gb * RG;
        const int nr = (p.G - g0 < RG) ? (p.G - g0) : RG;
        St st;
        st.reset();
        st.load_q(p.Q + ((hd * p.G + g0) * p.nq + t) * kD, p.nq * kD, nr, tl, p.qmul);
        for (int j0 = lo + lw * NG * kLocKPG; j0 < hi; j0 += KPS) {
          const uint8_t* kr[kLocKPG];
          const uint8_t* vr[kLocKPG];
          bool valid[kLocKPG];
#pragma unroll
          for (int k = 0; k < kLocKPG; ++k) {
            const int key = j0 + k * NG + g;
            valid[k] = key < hi;
            kr[k] = kb + static_cast<int64_t>(key) * kRowBytes;
            vr[k] = vb + static_cast<int64_t>(key) * kRowBytes;
          }
          st.template step<kLocKPG, GlobalLoader, true>(kr, vr, valid, tl, GlobalLoader{});
        }
        st.merge_groups();
        if (g == 0) {
          float* dst = lscr + (lw * RG) * (kD + 2);
#pragma unroll
          for (int rr = 0; rr < RG; ++rr) {
#pragma unroll
            for (int cc = 0; cc < St::CPL; ++cc)
#pragma unroll
              for (int e = 0; e < 8; ++e) dst[rr * (kD + 2) + St::dim_of(tl, cc, e)] = st.acc[rr][cc * 8 + e];
            if (tl == 0) {
              dst[rr * (kD + 2) + kD] = st.m[rr];
              dst[rr * (kD + 2) + kD + 1] = st.l[rr];
            }
          }
        }
        named_bar_sync(3, kLocWarps * 32);
        // join the 4 warps' states of each row; send each dim to its owner
        for (int item = lw * 32 + lane; item < nr * kD; item += kLocWarps * 32) {
          const int rr = item / kD, dim = item % kD;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kLocWarps; ++w) M = fmaxf(M, lscr[(w * RG + rr) * (kD + 2) + kD]);
          float ls = 0.f, as = 0.f;
#pragma unroll
          for (int w = 0; w < kLocWarps; ++w) {
            const float* src = lscr + (w * RG + rr) * (kD + 2);
            const float wgt = exp2_shift(src[kD], M);
            ls = fmaf(src[kD + 1], wgt, ls);
            as = fmaf(src[dim], wgt, as);
          }
          const int n = (g0 + rr) * static_cast<int>(p.nq) + t;
          const int o = dim / kOwn;
          st_cluster_f32(mapa_shared(rl0 + static_cast<uint32_t>(((r * Rp + n) * kOwn + dim % kOwn) * 4), o), as);
          if (dim < kC) {
            const uint32_t d2 = mapa_shared(rml0 + static_cast<uint32_t>((r * Rp + n) * 2 * 4), dim);
            st_cluster_f32(d2, M);
            st_cluster_f32(d2 + 4, ls);
          }
        }
        named_bar_sync(3, kLocWarps * 32);
      }
    }
  }

  // ------------------------------ reduction and merge ------------------------------
  // the readout biases this thread's merge items need, read before the barrier
  constexpr int kMergeThreads = kThreads - 64;
  constexpr int kMaxItems = (64 * kOwn + kMergeThreads - 1) / kMergeThreads;   // R <= 64
  // (raw bits: the loads are in flight across the barrier, converted after it)
  uint16_t csb = 0, ctb[kMaxItems];
#pragma unroll
  for (int q = 0; q < kMaxItems; ++q) ctb[q] = 0;
  if (warp >= 2) {
    const uint16_t* bits = reinterpret_cast<const uint16_t*>(p.blob);
    csb = bits[sbase + layout::out_b_off(H, depth, 1)];
    const uint16_t* ct = bits + tbase + layout::out_b_off(H, depth, kD);
#pragma unroll
    for (int q = 0; q < kMaxItems; ++q) {
      const int item = threadIdx.x - 64 + q * kMergeThreads;
      if (item < R * kOwn) ctb[q] = ct[r * kOwn + item % kOwn];
    }
  }
  __syncwarp();
  cluster_sync_all();              // every partial is in its owner's shared memory
  if (warp >= 2) {
    const float* rs = reinterpret_cast<const float*>(smem + SL.rs);
    const float* rt = reinterpret_cast<const float*>(smem + SL.rt);
    const float* rl = reinterpret_cast<const float*>(smem + SL.rl);
    const float* rml = reinterpret_cast<const float*>(smem + SL.rml);
#pragma unroll
    for (int q = 0; q < kMaxItems; ++q) {
      const int item = threadIdx.x - 64 + q * kMergeThreads;
      if (item >= R * kOwn) break;
      const int n = item / kOwn, dl = item % kOwn;
      const int dim = r * kOwn + dl;
      float a = 0.f, at = 0.f, Ml = -INFINITY;
#pragma unroll
      for (int c = 0; c < kSl; ++c) {
        a += rs[c * Rp + n];
        at += rt[(c * kOwn + dl) * Rp + n];
      }
#pragma unroll
      for (int c = 0; c < kC; ++c) Ml = fmaxf(Ml, rml[(c * Rp + n) * 2]);
      a += __uint_as_float(static_cast<uint32_t>(csb) << 16);
      at += __uint_as_float(static_cast<uint32_t>(ctb[q]) << 16);
      float ll = 0.f, al = 0.f;
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const float wgt = exp2_shift(rml[(c * Rp + n) * 2], Ml);
        ll = fmaf(rml[(c * Rp + n) * 2 + 1], wgt, ll);
        al = fmaf(rl[(c * Rp + n) * kOwn + dl], wgt, al);
      }
      const float ad = a * kLog2e;                     // document logit in log2 units
      const float M = fmaxf(ad, Ml);
      const float wd = exp2_shift(ad, M), wl = exp2_shift(Ml, M);
      const float v = (wd * at + wl * al) / (wd + wl * ll);
      const int64_t row = hd * R + n;
      if (p.out_bf16 != nullptr)
        p.out_bf16[layer_layout_index(row, dim, p.Hkv, p.G, p.nq)] = __float2bfloat16_rn(v);
      else
        p.out[row * kD + dim] = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

template <int RG, int kC, int kNPC>
cudaError_t set_attrs(size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(decode_cluster_kernel<RG, kC, kNPC>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess && kC > 8)
    e = cudaFuncSetAttribute(decode_cluster_kernel<RG, kC, kNPC>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1);
  return e;
}

template <int RG, int kC, int kNPC>
cudaError_t launch_cl(const ClusterParams& p, int heads, size_t smem, cudaStream_t stream) {
  const cudaError_t e = set_attrs<RG, kC, kNPC>(smem);
  if (e != cudaSuccess) return e;
  return launch_k(decode_cluster_kernel<RG, kC, kNPC>, dim3(static_cast<unsigned>(heads * kC)), dim3(kThreads),
                  smem, stream, kC, p);
}

// Clusters of this shape that can be resident at once (0: none, or unknown).
template <int RG, int kC, int kNPC>
int max_clusters(size_t smem) {
  if (set_attrs<RG, kC, kNPC>(smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kC);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kC;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_cluster_kernel<RG, kC, kNPC>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

int cluster_rg(int G) { return G <= 2 ? 2 : 4; }

ClusterShape cluster_shape(int cluster, int npc, int G, int64_t nq, int Hmax, int depth) {
  ClusterShape sh{};
  const int64_t R = static_cast<int64_t>(G) * nq;
  const bool shape_ok = (cluster == 8 && (npc == 1 || npc == 2)) || (cluster == 16 && npc == 1);
  if (!shape_ok || R < 1 || R > 64 || nq > 256 || depth < 1 || depth > 4) return sh;
  const int ksl = cl_slices(cluster, npc);
  const int S = cl_slice(Hmax, ksl);
  if (S > 128 * kMaxSliceTiles) return sh;
  sh.cluster = cluster;
  sh.npc = npc;
  sh.N = static_cast<int>((R + 15) / 16 * 16);
  sh.nb = depth >= 3 ? 2 : 1;
  const int rg = cluster_rg(G);
  constexpr size_t kMax = 227 * 1024;
  for (int st = kMaxStages; st >= 2; --st) {
    const size_t smem = cl_layout(cluster, npc, Hmax, sh.N, static_cast<int>(R), sh.nb, st, rg).total + 1024;
    if (smem <= kMax) {
      sh.stages = st;
      sh.smem = smem;
      break;
    }
  }
  if (sh.stages == 0) return sh;
  // no longer a ring than one CTA's weights of the widest layer need
  {
    int64_t groups = 0;                  // ring stages the producer fills, as it groups the chunks
    const int cpg = S <= 64 ? 4 : 2;
    for (int k = 0; k < depth; ++k)
      groups += npc * ((S + 127) / 128) * ((layout::kchunks(layout::hidden_k(Hmax, k)) + cpg - 1) / cpg);
    groups += (layout::kchunks(S) + 1) / 2;
    if (groups < sh.stages) {
      sh.stages = groups < 2 ? 2 : static_cast<int>(groups);
      sh.smem = cl_layout(cluster, npc, Hmax, sh.N, static_cast<int>(R), sh.nb, sh.stages, rg).total + 1024;
    }
  }
  const int MTmax = (S + 127) / 128;
  const int cols = (npc * MTmax + 1) * sh.N;
  int c = 32;
  while (c < cols) c <<= 1;
  sh.tmem_cols = c;
  sh.ok = c <= 512;
  return sh;
}

int cluster_max_active(const ClusterShape& sh, int G) {
  if (!sh.ok) return 0;
  const bool rg2 = cluster_rg(G) == 2;
  if (sh.cluster == 16) return rg2 ? max_clusters<2, 16, 1>(sh.smem) : max_clusters<4, 16, 1>(sh.smem);
  if (sh.npc == 1) return rg2 ? max_clusters<2, 8, 1>(sh.smem) : max_clusters<4, 8, 1>(sh.smem);
  return rg2 ? max_clusters<2, 8, 2>(sh.smem) : max_clusters<4, 8, 2>(sh.smem);
}

cudaError_t launch_decode_cluster(const ClusterParams& p, const ClusterShape& sh, int heads, cudaStream_t stream) {
  const bool rg2 = cluster_rg(p.G) == 2;
  const size_t smem = sh.smem;
  if (sh.cluster == 16) return rg2 ? launch_cl<2, 16, 1>(p, heads, smem, stream) : launch_cl<4, 16, 1>(p, heads, smem, stream);
  if (sh.npc == 1) return rg2 ? launch_cl<2, 8, 1>(p, heads, smem, stream) : launch_cl<4, 8, 1>(p, heads, smem, stream);
  return rg2 ? launch_cl<2, 8, 2>(p, heads, smem, stream) : launch_cl<4, 8, 2>(p, heads, smem, stream);
}

}  // namespace nectar
