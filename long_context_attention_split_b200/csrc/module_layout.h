// Packed layout of a Nectar module set (one bf16 blob), shared by the host
// packer (nectar_module_pack) and the module kernels.
//
// Blocks are ordered (layer l, KV head h, net), net 0 = score, 1 = target;
// all blocks of a layer have the same size, so block (l, h, net) starts at
//   layer_base(l) + h * head_elems(H_l) + net * net_elems(H_l, depth, 1).
// Inside a net (every piece a multiple of 64 elements = 128 bytes):
//   for k = 0..depth-1:
//     W_k  K-chunked [ceil(K_k/64)][H][64], K_k = d (k = 0) or d + H (k >= 1),
//          row i = hidden unit, column c = input feature: c < d multiplies q
//          (U_0 for k = 0, V_k for k >= 1), c >= d multiplies h_{k-1} (U_k);
//     b_k  [round64(H)]
//   score:  w [round64(H)], c [64]            (readout W_out row, bias)
//   target: W_out K-chunked [ceil(H/64)][d][64], c [d]
// K-chunked means each 64-wide column block of the matrix is stored as
// rows x 128 bytes, so a TMA box of (64 columns x 128 rows) over the blob
// viewed as [rows][64] lands as one K-major tile.  Padding columns are 0.
#pragma once
#include <stdint.h>

namespace nectar {
namespace layout {

#ifdef __CUDACC__
#define NECTAR_HD __host__ __device__ __forceinline__
#else
#define NECTAR_HD inline
#endif

constexpr int kDm = 128;   // d

NECTAR_HD int round64(int x) { return (x + 63) & ~63; }
NECTAR_HD int kchunks(int K) { return (K + 63) / 64; }
NECTAR_HD int hidden_k(int H, int k) { return k == 0 ? kDm : kDm + H; }
NECTAR_HD int64_t chunked_elems(int rows, int K) { return static_cast<int64_t>(kchunks(K)) * rows * 64; }
// element (row i, column c) of a K-chunked matrix with `rows` rows
NECTAR_HD int64_t chunked_index(int rows, int c, int i) {
  return (static_cast<int64_t>(c / 64) * rows + i) * 64 + (c % 64);
}
NECTAR_HD int64_t hidden_w_off(int H, int depth, int k) {
  (void)depth;
  int64_t off = 0;
  for (int kk = 0; kk < k; ++kk) off += chunked_elems(H, hidden_k(H, kk)) + round64(H);
  return off;
}
NECTAR_HD int64_t hidden_b_off(int H, int depth, int k) {
  return hidden_w_off(H, depth, k) + chunked_elems(H, hidden_k(H, k));
}
NECTAR_HD int64_t out_w_off(int H, int depth) { return hidden_w_off(H, depth, depth); }
NECTAR_HD int64_t out_b_off(int H, int depth, int dout) {
  return out_w_off(H, depth) + (dout == 1 ? round64(H) : chunked_elems(kDm, H));
}
NECTAR_HD int64_t net_elems(int H, int depth, int dout) {
  return out_b_off(H, depth, dout) + (dout == 1 ? 64 : kDm);
}
NECTAR_HD int64_t head_elems(int H, int depth) { return net_elems(H, depth, 1) + net_elems(H, depth, kDm); }

#undef NECTAR_HD
}  // namespace layout
}  // namespace nectar
