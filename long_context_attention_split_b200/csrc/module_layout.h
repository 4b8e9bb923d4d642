// Packed layout of a Nectar module set (one bf16 blob), shared by the host
// packer (nectar_module_pack) and the module kernels.
//
// Blocks are ordered (layer l, KV head h, net), net 0 = score, 1 = target;
// all blocks of a layer have the same size, so block (l, h, net) starts at
//   layer_base(l) + h * head_elems(H_l) + net * net_elems(H_l, depth, 1).
// Inside a net (every piece a multiple of 64 elements = 128 bytes):
//   for k = 0..depth-1:
//     W_k  tiled [ceil(H/128)][ceil(K_k/64)][tr][64], K_k = d (k = 0) or d + H,
//          row i = hidden unit, column c = input feature: c < d multiplies q
//          (U_0 for k = 0, V_k for k >= 1), c >= d multiplies h_{k-1} (U_k);
//     b_k  [round64(H)]
//   score:  w [round64(H)], c [64]            (readout W_out row, bias)
//   target: W_out tiled [1][ceil(H/64)][d][64], c [d]
// Tiled means: the rows are cut into tiles of 128 (the last one holding
// tr = rows - 128 * m rows), and each row tile stores its 64-column chunks
// one after another, tr rows x 128 bytes each.  Inside every row the eight
// 16-byte pieces sit in the order of the 128-byte swizzle (piece j of row i
// at slot j ^ (i % 8)).  Any run of consecutive chunks of one row tile is
// then a single contiguous block, and its bulk copy to a 1024-byte aligned
// shared-memory address yields, chunk after chunk, exactly the K-major,
// 128-byte-swizzled operand tiles the tensor cores read.  Padding columns
// are 0.
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
// rows of row tile m of a matrix with `rows` rows
NECTAR_HD int tile_rows(int rows, int m) { return (rows - 128 * m < 128) ? (rows - 128 * m) : 128; }
// element offset of chunk c of row tile m (matrix with `rows` rows, K columns)
NECTAR_HD int64_t tile_chunk_off(int rows, int K, int m, int c) {
  return (static_cast<int64_t>(m) * kchunks(K) * 128 + static_cast<int64_t>(c) * tile_rows(rows, m)) * 64;
}
// element (row i, column c) of a tiled, swizzled matrix with `rows` rows and K columns
NECTAR_HD int64_t chunked_index(int rows, int K, int c, int i) {
  const int m = i >> 7, r = i & 127;
  return tile_chunk_off(rows, K, m, c / 64) + static_cast<int64_t>(r) * 64 + ((((c % 64) >> 3) ^ (r & 7)) << 3) +
         (c & 7);
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

// ---------------------------------------------------------------------------
// Module sets with a shared backbone (depths Db, Ds, Dt; widths Hb, Hs, Ht
// of one layer l).  Block of one (l, h):
//   backbone: for k = 0..Db-1: W_k tiled [Hb][K], K = d (k = 0) or d + Hb; b_k
//   score:    for j = 0..Ds-1: W_j tiled [Hs][d + P_j]; b_j; then w, c
//   target:   for j = 0..Dt-1: W_j tiled [Ht][d + P_j]; b_j; then W_out, c
// with P_0 = Hb (0 when Db = 0: the first layer then sees only q) and
// P_j = the branch width for j >= 1.  With Db = 0 and equal branches this is
// exactly the block above (head_elems), so either layout reads the other.
// ---------------------------------------------------------------------------
// input width (besides q) of layer j of a branch of width Hn
NECTAR_HD int branch_prev(int Db, int Hb, int Hn, int j) { return j == 0 ? (Db > 0 ? Hb : 0) : Hn; }
NECTAR_HD int64_t layer_elems(int H, int K) { return chunked_elems(H, K) + round64(H); }
NECTAR_HD int64_t backbone_elems(int Db, int Hb) {
  int64_t off = 0;
  for (int k = 0; k < Db; ++k) off += layer_elems(Hb, k == 0 ? kDm : kDm + Hb);
  return off;
}
// offset, inside the backbone, of the weights of layer k
NECTAR_HD int64_t backbone_w_off(int Hb, int k) { return backbone_elems(k, Hb); }
// offset, inside its branch, of the weights of layer j
NECTAR_HD int64_t branch_w_off(int Db, int Hb, int Hn, int j) {
  int64_t off = 0;
  for (int jj = 0; jj < j; ++jj) off += layer_elems(Hn, kDm + branch_prev(Db, Hb, Hn, jj));
  return off;
}
NECTAR_HD int64_t branch_b_off(int Db, int Hb, int Hn, int j) {
  return branch_w_off(Db, Hb, Hn, j) + chunked_elems(Hn, kDm + branch_prev(Db, Hb, Hn, j));
}
// readout weights / bias of a branch with Dn layers (dout 1: score, d: target)
NECTAR_HD int64_t branch_out_w_off(int Db, int Hb, int Hn, int Dn) { return branch_w_off(Db, Hb, Hn, Dn); }
NECTAR_HD int64_t branch_out_b_off(int Db, int Hb, int Hn, int Dn, int dout) {
  return branch_out_w_off(Db, Hb, Hn, Dn) + (dout == 1 ? round64(Hn) : chunked_elems(kDm, Hn));
}
NECTAR_HD int64_t branch_elems(int Db, int Hb, int Hn, int Dn, int dout) {
  return branch_out_b_off(Db, Hb, Hn, Dn, dout) + (dout == 1 ? 64 : kDm);
}
// start of the score (net 0) or target (net 1) branch inside the block
NECTAR_HD int64_t branch_base(int Db, int Hb, int Ds, int Hs, int net) {
  return backbone_elems(Db, Hb) + (net ? branch_elems(Db, Hb, Hs, Ds, 1) : 0);
}
NECTAR_HD int64_t head_elems_arch(int Db, int Hb, int Ds, int Hs, int Dt, int Ht) {
  return branch_base(Db, Hb, Ds, Hs, 1) + branch_elems(Db, Hb, Ht, Dt, kDm);
}

#undef NECTAR_HD
}  // namespace layout
}  // namespace nectar
