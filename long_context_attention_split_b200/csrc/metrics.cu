// Two small kernels around the module forward of "Nectar: Neural Estimation
// of Cached-Token Attention via Regression":
//
//  * fit_metrics_kernel -- how well a module fits the exact targets, per
//    (layer, KV head) (§4 "score / target MSE"; App. C.4, Eq. (C.1)):
//      score_mse  = mean_q (a(q) - alpha(q))^2
//      target_mse = mean_q (1/d) sum_c (A_theta(q)_c - A(q)_c)^2
//      rte        = mean_q log(||A_theta(q) - A(q)||^2 / ||q - A(q)||^2)
//    (the RTE of Eq. (C.1) is the sum of rte over (layer, KV head)).  One
//    CTA of 16 warps per head; each warp loads 2 rows at a time (a lane
//    holding 4 of the d = 128 dims, 16-byte loads) and issues the next 2
//    rows' loads before reducing the current ones; row sums are reduced by
//    a transposing shuffle tree, the head sums kept in double.  Bound by
//    HBM: every input byte is read once.
//
//  * quadrature_init_kernel -- the Quadrature module of §2.4 keeps p learned
//    key / value rows per (layer, KV head), initialised to the first p rows
//    of the cache: W[h] = K[h][0:p], Z[h] = V[h][0:p] (16-byte copies).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nectar {

namespace {
constexpr int kFmWarps = 16;
constexpr int kFmRows = 2;                   // rows per warp in flight
constexpr int kFmLanesPerRow = 32 / kFmRows; // lanes holding one row's sums after the reduction

// The 2R row sums v = (num_0, den_0, ..., num_{R-1}, den_{R-1}) of a warp,
// reduced over its 32 lanes with 2R - 1 + log2(16 / R) shuffles instead of
// 2R x 5: each of the first log2(2R) steps halves the values a lane carries
// (it keeps one half and sends the other to its partner), the rest are plain
// sums.  Lane L ends with v[L / (16 / R)] summed over all lanes: num_k at
// lane k 32 / R, den_k at lane k 32 / R + 16 / R.
template <int R>
__device__ __forceinline__ float fm_transpose_sum(float (&v)[2 * R], int lane) {
  int n = 2 * R;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const int half = n / 2;
      const bool up = lane & off;
#pragma unroll
      for (int j = 0; j < half; ++j) {
        const float send = up ? v[j] : v[j + half], keep = up ? v[j + half] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
      n = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  return v[0];
}
}  // namespace

__global__ void __launch_bounds__(kFmWarps * 32, 2)
fit_metrics_kernel(const float* __restrict__ alpha, const float* __restrict__ A, const float* __restrict__ a,
                   const float* __restrict__ At, const __nv_bfloat16* __restrict__ Q, int64_t rows,
                   double* __restrict__ out) {
  __shared__ double red[kFmWarps][3];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kr = lane / kFmLanesPerRow;      // the row whose scalars (and sums) this lane holds
  const int64_t hd = blockIdx.x;
  constexpr int64_t kStride = static_cast<int64_t>(kFmWarps) * kFmRows;
  double s_sum = 0.0, t_sum = 0.0, r_sum = 0.0;
  float4 av[kFmRows], tv[kFmRows];
  uint2 qw[kFmRows];
  float ai = 0.f, ali = 0.f;
  // rows past the end are clamped to the last one: loaded, never counted
  auto load = [&](int64_t r0) {
#pragma unroll
    for (int k = 0; k < kFmRows; ++k) {
      const int64_t it = hd * rows + (r0 + k < rows ? r0 + k : rows - 1);
      av[k] = reinterpret_cast<const float4*>(A + it * kD)[lane];
      tv[k] = reinterpret_cast<const float4*>(At + it * kD)[lane];
      qw[k] = reinterpret_cast<const uint2*>(Q + it * kD)[lane];
    }
    const int64_t it = hd * rows + (r0 + kr < rows ? r0 + kr : rows - 1);
    ai = a[it];
    ali = alpha[it];
  };
  int64_t r0 = static_cast<int64_t>(warp) * kFmRows;
  if (r0 < rows) load(r0);
  for (; r0 < rows; r0 += kStride) {
    float v[2 * kFmRows];
#pragma unroll
    for (int k = 0; k < kFmRows; ++k) {
      const float q0 = bf16lo(qw[k].x), q1 = bf16hi(qw[k].x), q2 = bf16lo(qw[k].y), q3 = bf16hi(qw[k].y);
      const float e0 = tv[k].x - av[k].x, e1 = tv[k].y - av[k].y, e2 = tv[k].z - av[k].z, e3 = tv[k].w - av[k].w;
      const float b0 = q0 - av[k].x, b1 = q1 - av[k].y, b2 = q2 - av[k].z, b3 = q3 - av[k].w;
      v[2 * k] = fmaf(e0, e0, fmaf(e1, e1, fmaf(e2, e2, e3 * e3)));
      v[2 * k + 1] = fmaf(b0, b0, fmaf(b1, b1, fmaf(b2, b2, b3 * b3)));
    }
    const double ds = static_cast<double>(ai) - static_cast<double>(ali);
    const bool counted = lane % kFmLanesPerRow == 0 && r0 + kr < rows;
    // the next rows' loads go out before this step's reduction and logarithm
    if (r0 + kStride < rows) load(r0 + kStride);
    const float y = fm_transpose_sum<kFmRows>(v, lane);
    const float den = __shfl_down_sync(0xffffffffu, y, kFmLanesPerRow / 2);
    if (counted) {
      s_sum += ds * ds;
      t_sum += static_cast<double>(y) / kD;
      r_sum += static_cast<double>(logf(y / den));
    }
  }
  // lanes 0, 32 / R, ... hold the warp's sums
#pragma unroll
  for (int off = kFmLanesPerRow; off <= 16; off <<= 1) {
    s_sum += __shfl_xor_sync(0xffffffffu, s_sum, off);
    t_sum += __shfl_xor_sync(0xffffffffu, t_sum, off);
    r_sum += __shfl_xor_sync(0xffffffffu, r_sum, off);
  }
  if (lane == 0) {
    red[warp][0] = s_sum;
    red[warp][1] = t_sum;
    red[warp][2] = r_sum;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    double v = 0.0;
    for (int w = 0; w < kFmWarps; ++w) v += red[w][threadIdx.x];
    out[hd * 3 + threadIdx.x] = rows > 0 ? v / static_cast<double>(rows) : 0.0;
  }
}

cudaError_t launch_fit_metrics(const float* alpha, const float* A, const float* a, const float* At,
                               const __nv_bfloat16* Q, int64_t heads, int64_t rows, double* out,
                               cudaStream_t stream) {
  fit_metrics_kernel<<<static_cast<unsigned>(heads), kFmWarps * 32, 0, stream>>>(alpha, A, a, At, Q, rows, out);
  return cudaGetLastError();
}

__global__ void quadrature_init_kernel(const uint4* __restrict__ K, const uint4* __restrict__ V,
                                       uint4* __restrict__ W, uint4* __restrict__ Z, int64_t n, int64_t p,
                                       int64_t heads) {
  constexpr int64_t kRow16 = kD * 2 / 16;    // 16-byte pieces per row
  const int64_t per_head = p * kRow16;
  const int64_t total = heads * per_head;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t hd = i / per_head, j = i % per_head;
    const int64_t src = hd * n * kRow16 + j;
    W[i] = K[src];
    Z[i] = V[src];
  }
}

cudaError_t launch_quadrature_init(const __nv_bfloat16* K, const __nv_bfloat16* V, __nv_bfloat16* W,
                                   __nv_bfloat16* Z, int64_t heads, int64_t n, int64_t p, int sms,
                                   cudaStream_t stream) {
  const int64_t total = heads * p * (kD * 2 / 16);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quadrature_init_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(K), reinterpret_cast<const uint4*>(V), reinterpret_cast<uint4*>(W),
      reinterpret_cast<uint4*>(Z), n, p, heads);
  return cudaGetLastError();
}

}  // namespace nectar
