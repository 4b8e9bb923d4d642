// Shared pieces of the CUDA-core attention path.
//
// A group of LPK lanes owns one key at a time: lane t of the group holds the
// 16-byte chunks t, t+LPK, ... of the key's 256-byte row (d = 128 bf16), so
// one group reads a row with conflict-free 16-byte accesses and the lane keeps
// DPL = 128 / LPK dimensions of every query row in registers.  A warp runs
// NG = 32 / LPK key slots side by side.  Scores are reduced across the LPK
// lanes with xor shuffles, so every lane of a group ends with the full score.
//
// Scores are kept in log2 units (q is pre-multiplied by scale * log2 e), so
// exp becomes exp2.  The running maximum is only moved when a block maximum
// exceeds it by more than kRescaleSlack (2^8): until then the weights
// 2^{s - m} stay below 256, and the final normalisation divides numerator
// and denominator by the same 2^m, so the result is the same quantity.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "ptx.cuh"

namespace nectar {

constexpr int kD = 128;                 // head dimension (the only one supported)
constexpr int kRowBytes = kD * 2;       // one bf16 key / value row
constexpr float kRescaleSlack = 8.0f;   // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float neg_inf() { return -INFINITY; }

// exp2(x - m) for a finite or -inf x, 0 for x == -inf (also when m == -inf).
__device__ __forceinline__ float exp2_shift(float x, float m) {
  return (x == -INFINITY) ? 0.0f : ex2(x - m);
}

// 2^x on the FMA and integer pipes instead of the special-function unit,
// for arguments x <= 127 (softmax exponents, <= the lazy-rescale slack).
// Cody-Waite argument reduction x = n + f with n = round(x), done by adding
// and subtracting 1.5 * 2^23 (n lands in the low mantissa bits of j),
// f in [-0.5, 0.5]; 2^f by a degree-3 polynomial fitted by the Remez
// exchange to minimise the relative error on that interval (coefficients
// from fit_exp2_poly.py; max relative error 7.5e-5, far below the 2^-9 of
// the bf16 rounding the softmax weights get next); 2^n is added to the
// exponent field.  Arguments below -126 give ~2^-126 instead of 0.
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float j = x + 12582912.0f;             // 1.5 * 2^23
  const float f = x - (j - 12582912.0f);
  const float pf = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return __int_as_float(__float_as_int(pf) + (__float_as_int(j) << 23));
}

// Load 8 bf16 (one 16-byte chunk) as floats.
__device__ __forceinline__ void unpack8(const uint4 w, float* f) {
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x);
  f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z); f[5] = bf16hi(w.z);
  f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}

struct SmemLoader {
  __device__ __forceinline__ uint4 operator()(const uint8_t* p) const {
    return *reinterpret_cast<const uint4*>(p);
  }
};
struct GlobalLoader {
  __device__ __forceinline__ uint4 operator()(const uint8_t* p) const { return ld_nc_v4(p); }
};

// Online-softmax state of R query rows held by one lane.
template <int R, int LPK>
struct RowState {
  static constexpr int NG = 32 / LPK;     // key slots per warp
  static constexpr int DPL = kD / LPK;    // dims per lane
  static constexpr int CPL = DPL / 8;     // 16-byte chunks per lane

  float q[R][DPL];
  float m[R], l[R];
  float acc[R][DPL];

  // dimension index of acc[.][ci*8 + e] for lane-in-group t
  __device__ __forceinline__ static int dim_of(int t, int ci, int e) { return 8 * (t + LPK * ci) + e; }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      m[r] = -INFINITY;
      l[r] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[r][e] = 0.f;
    }
  }

  // rows: pointer to row 0 of R consecutive bf16 query rows (d = 128 each),
  // row_stride in elements.  qmul = scale * log2 e.  Rows >= nrows read 0.
  __device__ __forceinline__ void load_q(const __nv_bfloat16* rows, int64_t row_stride, int nrows,
                                         int t, float qmul) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int ci = 0; ci < CPL; ++ci) {
        float f[8];
        if (r < nrows) {
          const uint8_t* p = reinterpret_cast<const uint8_t*>(rows + r * row_stride) + 16 * (t + LPK * ci);
          unpack8(ld_nc_v4(p), f);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) q[r][ci * 8 + e] = f[e] * qmul;
      }
    }
  }

  // Load this lane's 16-byte pieces of KPG key (or value) rows; invalid
  // keys read nothing and give zeros.
  template <int KPG, class Loader>
  __device__ __forceinline__ static void load_rows(const uint8_t* const* row, const bool* valid, int t,
                                                   const Loader& ld, uint4 (&w)[KPG][CPL]) {
#pragma unroll
    for (int k = 0; k < KPG; ++k)
#pragma unroll
      for (int ci = 0; ci < CPL; ++ci)
        w[k][ci] = valid[k] ? ld(row[k] + 16 * (t + LPK * ci)) : make_uint4(0, 0, 0, 0);
  }

  // Scores of KPG keys (log2 units, -inf for invalid keys), the lazy
  // rescale of the running state, and the keys' weights pw.
  // kPaired: the dot products as paired f32x2 FMAs (even and odd dims in
  // two accumulators) -- fewer instructions, two more registers per row.
  template <int KPG, bool kPaired = false>
  __device__ __forceinline__ void weigh(const uint4 (&kw)[KPG][CPL], const bool* valid, float (&pw)[KPG][R]) {
    float sc[KPG][R];
#pragma unroll
    for (int k = 0; k < KPG; ++k) {
      float part[R];
#pragma unroll
      for (int r = 0; r < R; ++r) part[r] = 0.f;
      if (kPaired) {
        float2 part2[R];
#pragma unroll
        for (int r = 0; r < R; ++r) part2[r] = make_float2(0.f, 0.f);
#pragma unroll
        for (int ci = 0; ci < CPL; ++ci) {
          float kf[8];
          unpack8(kw[k][ci], kf);
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < 8; e += 2)
              part2[r] = ffma2(make_float2(q[r][ci * 8 + e], q[r][ci * 8 + e + 1]), make_float2(kf[e], kf[e + 1]),
                               part2[r]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) part[r] = part2[r].x + part2[r].y;
      } else {
#pragma unroll
        for (int ci = 0; ci < CPL; ++ci) {
          float kf[8];
          unpack8(kw[k][ci], kf);
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < 8; ++e) part[r] = fmaf(q[r][ci * 8 + e], kf[e], part[r]);
        }
      }
#pragma unroll
      for (int off = LPK / 2; off >= 1; off >>= 1)
#pragma unroll
        for (int r = 0; r < R; ++r) part[r] += __shfl_xor_sync(0xffffffffu, part[r], off);
#pragma unroll
      for (int r = 0; r < R; ++r) sc[k][r] = valid[k] ? part[r] : -INFINITY;
    }
    // block maximum, lazy rescale
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float bm = sc[0][r];
#pragma unroll
      for (int k = 1; k < KPG; ++k) bm = fmaxf(bm, sc[k][r]);
      if (bm > m[r] + kRescaleSlack) {
        const float corr = exp2_shift(m[r], bm);
        l[r] *= corr;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[r][e] *= corr;
        m[r] = bm;
      }
    }
#pragma unroll
    for (int k = 0; k < KPG; ++k)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        pw[k][r] = exp2_shift(sc[k][r], m[r]);
        l[r] += pw[k][r];
      }
  }

  // acc += pw * v over KPG value rows; kPaired as in weigh (it measured
  // slower in the split decode kernel, whose 96-register cap then spills).
  template <int KPG, bool kPaired = false>
  __device__ __forceinline__ void accumulate(const uint4 (&vw)[KPG][CPL], const float (&pw)[KPG][R]) {
#pragma unroll
    for (int k = 0; k < KPG; ++k)
#pragma unroll
      for (int ci = 0; ci < CPL; ++ci) {
        float vf[8];
        unpack8(vw[k][ci], vf);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (kPaired) {
            const float2 w2 = make_float2(pw[k][r], pw[k][r]);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float2 a2 = ffma2(w2, make_float2(vf[e], vf[e + 1]),
                                      make_float2(acc[r][ci * 8 + e], acc[r][ci * 8 + e + 1]));
              acc[r][ci * 8 + e] = a2.x;
              acc[r][ci * 8 + e + 1] = a2.y;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[r][ci * 8 + e] = fmaf(pw[k][r], vf[e], acc[r][ci * 8 + e]);
          }
        }
      }
  }

  // Process KPG keys of this group.  krow[k] / vrow[k] point at the 256-byte
  // rows; invalid keys are skipped (their rows are never read).  kEarlyV
  // issues the V loads together with the K loads (more bytes in flight when
  // the rows come straight from global memory).
  template <int KPG, class Loader, bool kEarlyV = false>
  __device__ __forceinline__ void step(const uint8_t* const* krow, const uint8_t* const* vrow,
                                       const bool* valid, int t, const Loader& ld) {
    uint4 kw[KPG][CPL];
    uint4 vw[KPG][CPL];
    float pw[KPG][R];
    load_rows<KPG>(krow, valid, t, ld, kw);
    if (kEarlyV) load_rows<KPG>(vrow, valid, t, ld, vw);
    weigh<KPG>(kw, valid, pw);
    if (!kEarlyV) load_rows<KPG>(vrow, valid, t, ld, vw);
    accumulate<KPG>(vw, pw);
  }

  // Join the NG groups of the warp (xor over lane bits >= LPK); afterwards
  // every group holds the warp's combined state.
  __device__ __forceinline__ void merge_groups() {
#pragma unroll
    for (int off = LPK; off < 32; off <<= 1) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[r], off);
        const float lo = __shfl_xor_sync(0xffffffffu, l[r], off);
        const float M = fmaxf(m[r], mo);
        const float wa = exp2_shift(m[r], M), wb = exp2_shift(mo, M);
        l[r] = l[r] * wa + lo * wb;
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[r][e], off);
          acc[r][e] = acc[r][e] * wa + ao * wb;
        }
        m[r] = M;
      }
    }
  }
};

// Visible local tokens of a query token; flags bad metadata (reading of
// §2.2: token i sees local j <= q_pos[i], j < local_len[q_seq[i]]).
__device__ __forceinline__ int visible_local(const int32_t* q_seq, const int32_t* q_pos,
                                             const int32_t* local_len, int64_t i, int B, int T,
                                             int* seq_out, int* err) {
  const int b = q_seq[i];
  *seq_out = b;
  if (b < 0 || b >= B) {
    record_error(err, DEVERR_BAD_SEQ);
    return 0;
  }
  int len = local_len[b];
  if (len < 0 || len > T) {
    record_error(err, DEVERR_BAD_LEN);
    len = len < 0 ? 0 : T;
  }
  // in 64 bits, so that q_pos = INT_MAX sees all len keys rather than wrapping
  int64_t nv = static_cast<int64_t>(q_pos[i]) + 1;
  if (nv > len) nv = len;
  if (nv < 0) nv = 0;
  return static_cast<int>(nv);
}

}  // namespace nectar
