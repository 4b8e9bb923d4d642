// Where the decode writes a Nectar layer's output when it stands in for a
// base-model attention layer: the kernels compute per-KV-head rows
// [L][Hkv][G][nq][d], row = (l Hkv + h) G nq + g nq + i, while the model's
// attention output is token-major [L][nq][Hkv G][d] with query head h G + g
// (grouped-query attention: the G query heads of KV head h are adjacent).
#pragma once
#include <stdint.h>

namespace nectar {

__device__ __forceinline__ int64_t layer_layout_index(int64_t row, int dim, int Hkv, int G, int64_t nq) {
  constexpr int kHeadDim = 128;
  const int64_t rows = static_cast<int64_t>(G) * nq;
  const int64_t hd = row / rows, rr = row % rows;
  const int64_t g = rr / nq, i = rr % nq;
  const int64_t l = hd / Hkv, h = hd % Hkv;
  return (((l * nq + i) * Hkv + h) * G + g) * kHeadDim + dim;
}

}  // namespace nectar
