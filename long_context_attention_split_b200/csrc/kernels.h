// Internal launch interface between the C ABI (nectar_api.cu) and the
// kernels.  Not part of the public header.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

namespace nectar {

// Sets the thread's nectar_last_error() text (defined with the C ABI).
void set_last_error(const char* msg);
// Id of the CUDA context current on the calling thread (0: none, or the
// driver cannot tell).
unsigned long long current_context_id();

// Launch with programmatic dependent launch allowed (the kernel calls
// griddep_wait before it touches global memory; see ptx.cuh) and, with
// cluster > 1, as clusters of `cluster` CTAs along x.  NECTAR_PDL=0 (read
// once per process) launches without the attribute.
inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("NECTAR_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  unsigned na = 0;
  if (pdl_enabled()) {
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = static_cast<unsigned>(cluster);
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ----- (i) split-n decode attention (CUDA cores) + LSE combine -------------
struct DecParams {
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const __nv_bfloat16* Q;
  int64_t n;
  int heads;
  int64_t rows_total;   // query rows per head (G * nq)
  int row0;             // first row handled by this launch
  int tile;             // keys per tile: dec_tile(rows of a pass)
  int64_t tph;          // tiles per head
  int64_t total;        // heads * tph
  int C;                // CTAs of the split launch
  int S_max;            // partial slots per head
  float qmul;           // scale * log2(e)
  float* ws_ml;         // [heads][S_max][rows_total][2]  (m in log2 units, l)
  float* ws_acc;        // [heads][S_max][rows_total][128]
  int* err;             // device error word
};

struct DecPlan {
  int64_t tph, total;
  int C, S_max, tile;
};

// Keys per tile of the split kernel for R query rows per pass: 128 up to 2
// rows (one CTA per SM streaming 32 KB bulk copies: measured 0.549 against
// 0.683 ms on a 28 x 8-head, 32768-key, 2-row document), 64 above (at 4
// rows the 64-key tiles with two CTAs per SM measured 1 % faster; from 5
// rows the row state needs the registers of a smaller tile).
#ifndef NECTAR_SPLIT_TILE_R4
#define NECTAR_SPLIT_TILE_R4 64
#endif
__host__ __device__ constexpr int dec_tile(int R) { return R <= 2 ? 128 : (R <= 4 ? NECTAR_SPLIT_TILE_R4 : 64); }
DecPlan plan_decode(int heads, int64_t n, int num_sms, int ctas_per_sm, int tile);
// The CTA of a stream-K split whose range [c*total/C, (c+1)*total/C) holds
// tile t: a head's partial slot s is written by CTA first_cta_of_tile(its
// first tile) + s.
__host__ __device__ __forceinline__ int first_cta_of_tile(int64_t t, int64_t total, int C) {
  return static_cast<int>(((t + 1) * static_cast<int64_t>(C) - 1) / total);
}
int dec_max_rows();
int dec_ctas_per_sm(int R);
size_t dec_smem_for_rows(int R);
cudaError_t launch_cache_attn_split(const DecParams& p, int R, cudaStream_t stream);
cudaError_t launch_cache_attn_combine(const DecParams& p, float* alpha, float* A, cudaStream_t stream);

// ----- (i) 3-32 query rows per head: transposed tensor-core split ---------
// Same stream-K plan (128-key tiles), partial layout and combine as the
// split kernel.
constexpr int kTctTile = 128;
// Up to this many rows per head: measured against the M = 128 tensor-core
// kernel on Llama-8B-shaped documents, 32 rows 1.94 vs 2.06 ms, 64 rows
// 2.60 vs 2.07 ms (one CTA per SM with four softmax warpgroups is bound
// by the softmax chain of each tile), so the kernel is built for 16 and 32
// query columns only.
#ifndef NECTAR_TCT_MAX_ROWS
#define NECTAR_TCT_MAX_ROWS 32
#endif
static_assert(NECTAR_TCT_MAX_ROWS >= 2 && NECTAR_TCT_MAX_ROWS <= 32, "transposed kernel: at most 32 rows");
constexpr int kTctMaxRows = NECTAR_TCT_MAX_ROWS;
// Resident CTAs per SM (each with a ring of 6 / this K or V stages): two
// measured 1.29 ms against 1.72 for one on a 32 x 8-head, 65536-key
// document at 4 rows (6.67 against 5.00 TB/s).
#ifndef NECTAR_TCT_CTAS_PER_SM
#define NECTAR_TCT_CTAS_PER_SM 2
#endif
constexpr int kTctCtasPerSm = NECTAR_TCT_CTAS_PER_SM;
size_t cache_attn_tct_smem(int64_t rows);
int cache_attn_tct_ctas_per_sm(int64_t rows);
cudaError_t launch_cache_attn_tct(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const DecParams& p, cudaStream_t stream);

// ----- (i) tensor-core path for many query rows per head -------------------
struct TcParams {
  int64_t n;
  int heads;
  int64_t rows_total;
  int qpairs;           // units (pairs of 128-row query tiles) per head
  int tile;             // keys per tile: dec_tile(rows of a pass)
  int64_t tph;          // tiles per head
  int C;                // CTAs (one per SM)
  int dp_rounds;        // whole-unit rounds before the rest
  int64_t sk_units;     // the rest: units cut by key tiles across the CTAs
  int sk_parts;         // 0: the rest as one stream-K range list; S > 0: each unit of the rest in S
                        // equal key parts, item p * sk_units + u on CTA item % C (the query units of
                        // a head then read each key part at the same time)
  float qmul;           // scale * log2(e)
  float* alpha;
  float* A;
  float* ws_ml;         // [C][2][256][2]
  float* ws_acc;        // [C][2][256][128]
  int* err;
};
struct TcPlan {
  int qpairs;
  int64_t tph;
  int C, dp_rounds;
  int64_t sk_units;
  int sk_parts;
  size_t ws_bytes, smem;
};
TcPlan plan_tc(int heads, int64_t n, int64_t rows, int num_sms);
// the query map's box is {64, 64, 1, 1} when this is true, else {64, 128, 2, 1}
bool cache_attn_tc_dup(int64_t rows);
cudaError_t launch_cache_attn_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const TcParams& p, cudaStream_t stream);

// ----- (iii) merge with exact causal local attention -----------------------
struct MergeParams {
  const float* a;
  const float* A_doc;
  const __nv_bfloat16* Q;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const __nv_bfloat16* Kloc;
  const __nv_bfloat16* Vloc;
  const int32_t* local_len;
  float* out;
  int heads, G;
  int64_t nq;
  int B, T;
  float qmul;           // scale * log2(e)
  int* err;             // device error word
};
cudaError_t launch_merge_local(const MergeParams& p, cudaStream_t stream);

// ----- (ii) module forward and the fused decode (tcgen05) ------------------
constexpr int kModMaxLayers = 256;
struct ModParams {
  int Hkv, G, depth;            // depth: of both nets when the set has no backbone and equal nets
  int depth_b, depth_s, depth_t;
  bool general;                 // a backbone, or unequal nets: layer-by-layer path only
  int net_split;                // one-launch path: one CTA per net (else one per head, both nets)
  int64_t nq;
  int N, TPC, nblk, Hmax, tmem_cols, stages, cps;
  const __nv_bfloat16* blob;
  const __nv_bfloat16* Q;
  float* a_out;         // module forward outputs
  float* A_out;
  // fused decode
  const int32_t* q_seq;
  const int32_t* q_pos;
  const __nv_bfloat16* Kloc;
  const __nv_bfloat16* Vloc;
  const int32_t* local_len;
  int B, T;
  float qmul;
  float* out;
  float* ws_loc;        // decode: local state per row [(hd * rows + row)][d + 2]
  int64_t n_local;      // decode: local CTAs (heads * nq), after the module CTAs
  int64_t n_module;     // decode: module CTAs (set at launch)
  int module_first;     // decode: module CTAs ahead of the local CTAs in the grid
  __nv_bfloat16* out_bf16;   // decode: if set, the output goes here, bf16 [L][nq][Hkv][G][d]
  int* err;
  int32_t width[kModMaxLayers];        // score width (= target width unless general)
  int32_t width_b[kModMaxLayers];
  int32_t width_t[kModMaxLayers];
  int64_t layer_base[kModMaxLayers];   // blob element offset of layer l
  uint8_t order[kModMaxLayers];        // layers by decreasing width
};
// One-launch decode with one thread-block cluster per (l, h) (decode_cluster.cu):
// the hidden units of every layer are sliced over the cluster's CTAs, for
// calls with few heads (a model's decode run layer after layer).
constexpr int kClusterCtas = 8;
struct ClusterParams {
  int Hkv, G, depth;
  int64_t nq;
  int N;                // activation rows: G * nq rounded up to 16 (<= 64)
  int Hmax, stages, tmem_cols;
  int nb;               // hidden-state buffers per net: 2 when depth >= 3
  const __nv_bfloat16* blob;
  const __nv_bfloat16* Q;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const __nv_bfloat16* Kloc;
  const __nv_bfloat16* Vloc;
  const int32_t* local_len;
  int B, T;
  float qmul;           // scale * log2(e)
  float* out;           // fp32 [L][Hkv][G][nq][d], or
  __nv_bfloat16* out_bf16;   // bf16 layer layout [L][nq][Hkv][G][d]
  int* err;
  int32_t width[kModMaxLayers];
  int64_t layer_base[kModMaxLayers];
  uint8_t order[kModMaxLayers];
};
struct ClusterShape {
  bool ok;
  int cluster, npc, N, nb, stages, tmem_cols;   // npc: nets per CTA (1 or 2)
  size_t smem;
};
// Plan of the cluster decode with `cluster` (8 or 16) CTAs per (l, h), each
// holding npc of the two nets (8 CTAs: 1 or 2; 16 CTAs: 1), for G query
// heads x nq tokens per KV head; ok = false when it does not apply
// (more than 64 rows, depth > 4, or the shared memory or TMEM plan does not
// fit).
ClusterShape cluster_shape(int cluster, int npc, int G, int64_t nq, int Hmax, int depth);
// Clusters of that plan that can be resident on the device at once.
int cluster_max_active(const ClusterShape& sh, int G);
cudaError_t launch_decode_cluster(const ClusterParams& p, const ClusterShape& sh, int heads, cudaStream_t stream);

// Layer-by-layer grouped GEMM path of the module forward (module_gemm.cu),
// used when a KV head has at least kGemmMinRows query rows.
constexpr int kGemmMaxStages = 8;
#ifndef NECTAR_GEMM_MIN_ROWS
#define NECTAR_GEMM_MIN_ROWS 64
#endif
constexpr int kGemmMinRows = NECTAR_GEMM_MIN_ROWS;
struct GemmParams {
  int L, Hkv, stage, readout, nlayers;
  int depth_b, depth_s, depth_t;   // backbone, score and target depths (depth_b = 0: separate nets)
  int R, NR, rtiles, Hp, MT, stages, tmem_cols;
  int64_t ntiles;
  const __nv_bfloat16* blob;
  __nv_bfloat16* h_out;     // [2 slots][heads * R][Hp] bf16 (hidden stages; the backbone uses slot 0)
  float* part;              // score partials [heads * R][MT]
  float* a_out;             // readout: [heads * R]
  float* A_out;             // readout: [heads * R][d] (A_theta, or the merged output)
  const float* ws_loc;      // decode: local state per row [(heads * R)][d + 2], else null
  __nv_bfloat16* out_bf16;  // decode: if set, the merged output goes here, bf16 [L][nq][Hkv][G][d]
  int G;
  int64_t nq;
  int* err;
  int32_t width_b[kModMaxLayers];   // backbone width of layer l (unused when depth_b = 0)
  int32_t width_s[kModMaxLayers];   // score branch width
  int32_t width_t[kModMaxLayers];   // target branch width
  int64_t layer_base[kModMaxLayers];
  // per layer l, filled by the host for the current launch: the element
  // stride between the blocks of its KV heads, the offset inside a head's
  // block of the weights each part reads (part 0: the backbone or the score
  // branch, part 1: the target branch; the readout: W_out as part 1), and
  // aux: the score readout's w (the score's last layer) or c (the readout)
  int64_t hstride[kModMaxLayers];
  int64_t woff[kModMaxLayers][2];
  int64_t aux[kModMaxLayers];
  int64_t tile_start[kModMaxLayers + 1];
  uint8_t order[kModMaxLayers];
};
struct GemmShape {
  int NR, rtiles, stages, tmem_cols;
  size_t smem;
};
GemmShape gemm_shape(int64_t R, int max_rows);
cudaError_t launch_module_gemm(const CUtensorMap& tq, const CUtensorMap& th, const GemmParams& p, int grid,
                               size_t smem, cudaStream_t stream);
cudaError_t launch_local_state(const ModParams& p, cudaStream_t stream);

// Local attention for many query tokens: one job per (KV head, token) on the
// tensor cores (local_tc.cu) or per (KV head, token, block of <= 4 heads)
// on one warp (local_warp.cu).
struct LocalParams {
  int64_t njobs;            // heads * nq
  int64_t nq;
  int G, B, T, kbox;        // kbox = keys per TMA box, min(128, T)
  const __nv_bfloat16* Q;   // [heads][G][nq][d]
  const __nv_bfloat16* Kloc;  // [heads][B][T][d]
  const __nv_bfloat16* Vloc;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* local_len;
  float qmul;               // scale * log2 e
  float* ws_loc;            // state per row [(hd * rows + row)][d + 2] (when out is null)
  const float* a;           // merge: document logit per row
  const float* A_doc;       // merge: document term per row [.][d]
  float* out;               // merge output, or null
  int* err;
};
size_t local_tc_smem();
cudaError_t launch_local_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const LocalParams& p, int grid, cudaStream_t stream);
cudaError_t launch_local_warp(const LocalParams& p, int sms, cudaStream_t stream);
size_t local_tct_smem();
cudaError_t launch_local_tct(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const LocalParams& p, int sms, cudaStream_t stream);

// metrics.cu
cudaError_t launch_fit_metrics(const float* alpha, const float* A, const float* a, const float* At,
                               const __nv_bfloat16* Q, int64_t heads, int64_t rows, double* out,
                               cudaStream_t stream);
cudaError_t launch_quadrature_init(const __nv_bfloat16* K, const __nv_bfloat16* V, __nv_bfloat16* W,
                                   __nv_bfloat16* Z, int64_t heads, int64_t n, int64_t p, int sms,
                                   cudaStream_t stream);

struct ModShape {
  int TPC, N, nblk, tmem_cols, stages, cps;
  size_t smem;
};
ModShape mod_shape(int G, int64_t nq, int Hmax, bool fuse);
cudaError_t launch_module(const CUtensorMap& tq, const ModParams& p, int units, size_t smem, bool fuse,
                          cudaStream_t stream);
cudaError_t launch_decode(const CUtensorMap& tq, const ModParams& p, int units, size_t smem, cudaStream_t stream);

}  // namespace nectar
