// (iii) Merge of a document term (a, A_doc) with exact causal attention over
// the local tokens: Eqs. (3.4)-(3.5) of "Nectar: Neural Estimation of
// Cached-Token Attention via Regression" (§2.2).  The document term is one
// extra logit a with value A_doc, softmaxed jointly with the visible local
// keys; with the exact (alpha, A) this is full attention (Eq. (3.4) is an
// identity), with (a_theta, A_theta) it is the Nectar output (Eq. (3.5)).
//
// One CTA per (KV head, query token): the G query heads of the token share
// its local rows and causal mask, so the rows are streamed once (blocks of
// up to 8 heads are jobs of the same CTA) through a 4-stage shared-memory
// ring filled by TMA bulk copies (local_attn.cuh).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "local_attn.cuh"

namespace nectar {

constexpr int kMergeCW = 4;                       // consumer warps
constexpr int kMergeThreads = (kMergeCW + 1) * 32;  // + 1 producer warp
// ring depth: 4 stages for up to 4 query heads (several CTAs share an SM),
// 8 when the heads' registers leave one CTA per SM
template <int RG>
__host__ __device__ constexpr int merge_stages() { return RG <= 4 ? 4 : 8; }

template <int RG>
__host__ __device__ constexpr size_t merge_smem_bytes() {
  return size_t(merge_stages<RG>()) * kLocStageBytes + size_t(kMergeCW) * RG * (kD + 2) * sizeof(float) +
         2 * merge_stages<RG>() * sizeof(uint64_t);
}

template <int RG>
__global__ void __launch_bounds__(kMergeThreads)
merge_local_kernel(const MergeParams p) {
  constexpr int kMergeStages = merge_stages<RG>();
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  float* scratch = reinterpret_cast<float*>(smem + kMergeStages * kLocStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + kMergeCW * RG * (kD + 2));
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kMergeStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t hd = blockIdx.x / p.nq;
  const int64_t i = blockIdx.x % p.nq;
  const int64_t rows = static_cast<int64_t>(p.G) * p.nq;
  const LocalJobs J{p.q_seq, p.q_pos, p.local_len, p.Kloc, p.Vloc, p.B, p.T, p.G, p.err};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMergeStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kMergeCW);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == kMergeCW) {
    if (lane == 0) local_produce<RG>(J, hd, i, 1, smem_u32(ring), kMergeStages, full0, empty0);
    return;
  }
  const __nv_bfloat16* q0 = p.Q + (hd * rows + i) * kD;   // row (g = 0, token i)
  local_consume<RG, kMergeCW>(
      J, hd, i, 1, q0, p.nq * kD, p.qmul, ring, kMergeStages, full0, empty0, scratch, 1, warp, lane,
      [&](int /*t*/, int g, int dim, float M, float ls, float as) {
        // document term as one more logit a with value A_doc, Eqs. (3.4)-(3.5)
        const int64_t row = hd * rows + static_cast<int64_t>(g) * p.nq + i;
        const float ad = p.a[row] * kLog2e;
        const float Mx = fmaxf(ad, M);
        const float wd = exp2_shift(ad, Mx), wl = exp2_shift(M, Mx);
        p.out[row * kD + dim] = (wd * p.A_doc[row * kD + dim] + wl * as) / (wd + wl * ls);
      });
}

template <int RG>
static cudaError_t launch_merge_t(const MergeParams& p, cudaStream_t stream) {
  const int64_t units = static_cast<int64_t>(p.heads) * p.nq;
  if (units == 0) return cudaSuccess;
  const size_t smem = merge_smem_bytes<RG>();
  cudaError_t e = cudaFuncSetAttribute(merge_local_kernel<RG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  merge_local_kernel<RG><<<static_cast<unsigned>(units), kMergeThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_merge_local(const MergeParams& p, cudaStream_t stream) {
  switch (p.G < 8 ? p.G : 8) {
    case 1: return launch_merge_t<1>(p, stream);
    case 2: return launch_merge_t<2>(p, stream);
    case 3: return launch_merge_t<3>(p, stream);
    case 4: return launch_merge_t<4>(p, stream);
    case 5: return launch_merge_t<5>(p, stream);
    case 6: return launch_merge_t<6>(p, stream);
    case 7: return launch_merge_t<7>(p, stream);
    default: return launch_merge_t<8>(p, stream);
  }
}

}  // namespace nectar
