/*
 * nectar.h -- C ABI of libnectar.so, the B200 (sm_100a) hot path of Nectar.
 *
 * Method: "Nectar: Neural Estimation of Cached-Token Attention via
 * Regression" (Monteiro, Klein, Ablin, Cuturi; arXiv 2605.09778).  For a
 * fixed document cache K, V (RoPE already applied) of one (layer, KV-head),
 * a query q has the document log-normalizer alpha(q) and the
 * document-normalised readout A(q) of Eq. (3.1).  A trained pair of small
 * networks (score a_theta, target A_theta; Eq. (3.6)) replaces them at
 * inference, and the document then acts as ONE virtual logit a_theta with
 * value A_theta, softmaxed jointly with the exact causal local tokens
 * (Eqs. (3.4)-(3.5)).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - d (head dimension) must be 128; any other value returns
 *    NECTAR_ERR_UNSUPPORTED.
 *  - GQA: query head h' = h*G + g belongs to KV head h and uses its cache and
 *    its module pair (§2.1).  All query tensors are laid out
 *    [L][Hkv][G][nq][d] (bf16), so the G*nq query vectors ("rows") of one
 *    (l, h) are contiguous; row r = g*nq + i is token i of query head g.
 *  - Per-query outputs (alpha, a: fp32 [L][Hkv][G][nq]; A, A_theta, out:
 *    fp32 [L][Hkv][G][nq][d]) follow the same row order.  Outputs are fp32
 *    because the paper stores its regression targets in float32 (App. A).
 *  - Pointers marked DEVICE are device memory owned by the caller; HOST
 *    pointers are read during the call only.  Device pointers must be
 *    16-byte aligned and the tensors contiguous.  The library never
 *    allocates, frees or synchronises in these calls: all work is enqueued on
 *    `stream` and the outputs are valid once the stream reaches that point.
 *  - Every call validates its arguments on the host first and returns a
 *    status.  On any error nothing is enqueued.  nectar_last_error() then
 *    gives a one-line reason (thread-local).
 *  - Values that the host cannot see (device arrays q_seq, q_pos,
 *    local_len) are checked in the kernels: an out-of-range q_seq entry is
 *    treated as a sequence with no local tokens, a local_len above T_max is
 *    clamped to T_max, and both raise a bit readable with
 *    nectar_device_error_flags().
 *  - `scale` multiplies q.k; pass 1/sqrt(d) for Eq. (3.1)'s scores.
 */
#ifndef NECTAR_H_
#define NECTAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NECTAR_API __attribute__((visibility("default")))
#else
#define NECTAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t nectar_bf16;            /* raw bfloat16 bit pattern */
typedef struct CUstream_st *nectar_stream_t;   /* same type as cudaStream_t */

typedef enum {
  NECTAR_OK = 0,
  NECTAR_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size */
  NECTAR_ERR_UNSUPPORTED = 2,   /* d != 128, width or depth out of range */
  NECTAR_ERR_WORKSPACE = 3,     /* workspace missing or too small */
  NECTAR_ERR_CUDA = 4           /* a CUDA call failed (see nectar_last_error) */
} nectar_status;

/* Model shape: L layers, Hkv KV heads, G query heads per KV head, head dim d. */
typedef struct {
  int32_t L, Hkv, G, d;
} nectar_dims;

#define NECTAR_MAX_DEPTH 4
#define NECTAR_MAX_LAYERS 256
#define NECTAR_MAX_WIDTH 2048

/* ------------------------------------------------------------------------
 * (i) Exact cached-token attention, Eq. (3.1), §2.1:
 *   s_j = scale * q . k_j,   alpha(q) = log sum_j e^{s_j},
 *   A(q) = sum_j e^{s_j} v_j / sum_j e^{s_j},
 * for every query row of every (l, h) over that head's n document tokens.
 * The sum is split over n and the parts are joined by their log-sum-exp
 * (the grouping of the softmax sum that Eq. (3.4) rests on), so the result
 * does not depend on how the cache is split.
 *
 *   K, V   DEVICE bf16 [L][Hkv][n][d]       document cache
 *   Q      DEVICE bf16 [L][Hkv][G][nq][d]
 *   alpha  DEVICE fp32 [L][Hkv][G][nq]      (-inf when n == 0)
 *   A      DEVICE fp32 [L][Hkv][G][nq][d]   (0 when n == 0)
 *   workspace  DEVICE scratch of at least
 *              nectar_cache_attn_workspace_size(dims, n, nq) bytes (may be
 *              NULL when that size is 0).  Its contents on entry do not
 *              matter; two calls that overlap on the GPU must not share one.
 *              The size depends on the current device's SM count; it is 0
 *              when n == 0 or nq == 0 (no scratch needed), and also for
 *              invalid dims or when no CUDA device is current, cases in
 *              which nectar_cache_attn_lse itself returns an error.
 * n >= 0, nq >= 0 (nq == 0: nothing to do).  Returns NECTAR_ERR_WORKSPACE
 * when the workspace is too small.
 * ------------------------------------------------------------------------ */
NECTAR_API size_t nectar_cache_attn_workspace_size(nectar_dims dims, int64_t n, int64_t nq);

NECTAR_API nectar_status nectar_cache_attn_lse(nectar_dims dims, const nectar_bf16 *K,
                                    const nectar_bf16 *V, int64_t n,
                                    const nectar_bf16 *Q, int64_t nq, float scale,
                                    float *alpha, float *A, void *workspace,
                                    size_t workspace_bytes, nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * nectar_cache_attn_lse_static -- the same computation as
 * nectar_cache_attn_lse (same validation, kernels and outputs) with no
 * workspace argument and no allocation anywhere.  The paper has no
 * counterpart: this is an interface for callers that cannot create device
 * buffers -- code inside a host application or serving runtime whose memory
 * manager owns the whole device pool, plugin interfaces that receive only
 * input and output pointers, and latency-bound decode loops where cudaMalloc
 * (which may synchronise the device) is not acceptable.
 *
 * Scratch comes from a fixed area that is part of the library's device
 * image: NECTAR_STATIC_SCRATCH_BYTES on every GPU that loads the library,
 * held until the process exits.  A call whose scratch need
 * (nectar_cache_attn_workspace_size) exceeds it returns
 * NECTAR_ERR_WORKSPACE with the two sizes in nectar_last_error().
 *  - The first call on a device looks up the area's device address (with
 *    that device current) and remembers it for the current CUDA context;
 *    make that first call before any stream capture.  A later context on
 *    the device (after cudaDeviceReset, or another context made current)
 *    is detected by its id, and its first call looks the address up again,
 *    so that call too belongs before any capture.
 *  - All calls on a device share the one area, and it keeps whatever the
 *    last call left there.  Nothing in it has to start at zero (every value
 *    read is first written by the same call), but two calls that overlap on
 *    the GPU -- on different streams, or on one stream from different host
 *    threads without ordering -- race on it.
 * Arguments and outputs as for nectar_cache_attn_lse.
 * ------------------------------------------------------------------------ */
#define NECTAR_STATIC_SCRATCH_BYTES (48u << 20)

/* Size in bytes of the static scratch area this library was built with
 * (NECTAR_STATIC_SCRATCH_BYTES).  Host only; never fails. */
NECTAR_API size_t nectar_static_scratch_bytes(void);

NECTAR_API nectar_status nectar_cache_attn_lse_static(nectar_dims dims, const nectar_bf16 *K,
                                                      const nectar_bf16 *V, int64_t n,
                                                      const nectar_bf16 *Q, int64_t nq, float scale,
                                                      float *alpha, float *A,
                                                      nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * Module set: one score net a_theta: R^d -> R and one target net
 * A_theta: R^d -> R^d per (l, h), shared by the G query heads of that KV
 * head (§2.1), each an MLP with input re-injection, Eq. (3.6), §2.4:
 *   h_0 = SiLU(U_0 q + b_0),  h_k = SiLU(V_k q + U_k h_{k-1} + b_k),
 *   k = 1..depth-1, followed by a linear readout y = W_out h_{depth-1} + c
 *   (dout = 1 for the score net, d for the target net).
 * Width H_l may differ between layers (App. C.1); both nets of a layer use
 * it.  Weights and biases are bf16.
 *
 * The device copy is one packed blob built by nectar_module_pack.  Its
 * layout is private to the library (tiled for TMA); size it with
 * nectar_module_packed_elems.
 * ------------------------------------------------------------------------ */
/* Module sets with a shared backbone and nets of their own depth and
 * width ("Nectar", §2.4 and App. A.3: depths (D_b, D_s, D_t)).  The
 * backbone is D_b layers of the recursion above (width width_b[l]); the
 * score branch continues it from the backbone's last hidden state with
 * depth_s layers of width width_s[l] (its first layer sees q and that
 * state: g_0 = SiLU(V_0 q + U_0 h_{D_b - 1} + b_0)), then the score
 * readout; the target branch likewise (depth_t, width_t[l]).  With
 * depth_b = 0 each branch starts from q alone, so depth_b = 0 with equal
 * branches is the classic set above. */
typedef struct {
  int32_t depth_b;          /* backbone layers, 0..NECTAR_MAX_DEPTH - 1 */
  int32_t depth_s, depth_t; /* branch layers, >= 1; depth_b + max(depth_s, depth_t) <= NECTAR_MAX_DEPTH */
  const int32_t *width_b;   /* HOST [L], multiples of 16 in [16, 2048]; may be NULL when depth_b = 0 */
  const int32_t *width_s;   /* HOST [L] */
  const int32_t *width_t;   /* HOST [L] */
} nectar_module_arch;

typedef struct {
  int32_t depth;          /* hidden layers per net, 1..NECTAR_MAX_DEPTH (classic sets) */
  const int32_t *width;   /* HOST [L]: H_l, a multiple of 16 in [16, 2048] (classic sets) */
  const nectar_bf16 *weights;   /* DEVICE packed blob */
  int64_t weights_elems;  /* bf16 elements in the blob */
  const nectar_module_arch *arch;   /* HOST; NULL: the classic set (depth, width); else the
                                       architecture, and depth / width are not read.  Sets
                                       with a backbone or unequal branches run layer by layer
                                       (grouped GEMMs) whatever the number of query rows. */
} nectar_module_set;

/* Plain row-major HOST tensors of one net for all Hkv heads of a layer. */
typedef struct {
  const nectar_bf16 *U[NECTAR_MAX_DEPTH]; /* k=0: [Hkv][H][d]; k>=1: [Hkv][H][H] */
  const nectar_bf16 *V[NECTAR_MAX_DEPTH]; /* k>=1: [Hkv][H][d] (V[0] unused) */
  const nectar_bf16 *b[NECTAR_MAX_DEPTH]; /* [Hkv][H] */
  const nectar_bf16 *Wout;                /* [Hkv][dout][H] */
  const nectar_bf16 *c;                   /* [Hkv][dout] */
} nectar_net_host;

/* Elements of the packed blob of an architecture (0 on invalid arguments). */
NECTAR_API int64_t nectar_module_packed_elems_arch(nectar_dims dims, const nectar_module_arch *arch);

/* Pack HOST tensors of an architecture into a HOST blob.  nets: HOST
 * [L][3] -- nets[3*l + 0] the backbone (U, V, b of its depth_b layers;
 * Wout, c unused), nets[3*l + 1] the score branch, nets[3*l + 2] the target
 * branch.  Branch layer j: U[j] [Hkv][H][P] with P the width of the layer
 * before it (the backbone's for j = 0) and V[j] [Hkv][H][d] -- except for a
 * layer that starts a chain (the backbone's layer 0, or a branch's layer 0
 * when depth_b = 0), whose U is [Hkv][H][d] (it multiplies q) and whose V
 * is unused.  Padding in the blob is written as zeros. */
NECTAR_API nectar_status nectar_module_pack_arch(nectar_dims dims, const nectar_module_arch *arch,
                                      const nectar_net_host *nets, nectar_bf16 *blob,
                                      int64_t blob_elems);

/* Elements of the packed blob for these widths (0 on invalid arguments). */
NECTAR_API int64_t nectar_module_packed_elems(nectar_dims dims, int32_t depth, const int32_t *width);

/* Pack HOST tensors into a HOST blob of `blob_elems` elements.
 * nets: HOST [L][2] -- nets[2*l + 0] the score net, nets[2*l + 1] the target
 * net of layer l.  Padding in the blob is written as zeros. */
NECTAR_API nectar_status nectar_module_pack(nectar_dims dims, int32_t depth, const int32_t *width,
                                 const nectar_net_host *nets, nectar_bf16 *blob,
                                 int64_t blob_elems);

/* ------------------------------------------------------------------------
 * (ii) Module forward, Eq. (3.6): for every query row of every (l, h),
 *   a[row]       = a_theta(q)     DEVICE fp32 [L][Hkv][G][nq]
 *   A_theta[row] = A_theta(q)     DEVICE fp32 [L][Hkv][G][nq][d]
 * Runs on the tensor cores (tcgen05, bf16 operands, fp32 accumulation);
 * hidden activations are rounded to bf16 between layers.  Fewer than 64
 * query rows per KV head (classic sets) and ceil(Hmax / 128) *
 * round16(G) <= 512 (Hmax the widest layer: the one-launch kernel keeps a
 * layer's 128-unit tiles side by side in 512 TMEM columns): one launch,
 * each CTA carrying <= 64 rows through all layers in shared memory
 * (workspace unused, may be NULL).  Otherwise, or for a set with a backbone
 * or unequal branches:
 * one grouped-GEMM launch per hidden layer plus one for the readouts, the
 * hidden activations kept in `workspace` (DEVICE, 256-byte aligned, owned
 * by the caller, overwritten; NECTAR_ERR_WORKSPACE when missing or small).
 * ------------------------------------------------------------------------ */
/* Workspace of nectar_module_forward, in bytes: 0 when the one-launch path
 * runs (classic sets, fewer than 64 query rows G * nq per KV head, and the
 * TMEM condition above), else
 * the hidden activations of the layer-by-layer path,
 * (S >= 2 ? 2 : 1) * align256(2 * rows * Hp * 2) + align256(rows * ceil(Hsmax / 128) * 4),
 * with rows = L * Hkv * G * nq, S the hidden layers of the longest chain
 * (depth, or depth_b + max(depth_s, depth_t)), Hp the widest layer of any
 * part rounded up to 64 and Hsmax the widest score net. */
NECTAR_API size_t nectar_module_workspace_size(nectar_dims dims, const nectar_module_set *mods,
                                               int64_t nq);
NECTAR_API nectar_status nectar_module_forward(nectar_dims dims, const nectar_module_set *mods,
                                    const nectar_bf16 *Q, int64_t nq, float *a,
                                    float *A_theta, void *workspace, size_t workspace_bytes,
                                    nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * (iii) Merge with exact causal local attention, Eqs. (3.4)-(3.5), §2.2:
 *   out = (e^{a} A_doc + sum_{i vis} e^{s_i} v_i) / (e^{a} + sum_{i vis} e^{s_i}),
 *   s_i = scale * q . k_i over the visible local tokens of the row's token.
 * With (a, A_doc) = the exact (alpha, A) of nectar_cache_attn_lse this is
 * full attention over document + local tokens (Eq. (3.4) is an identity);
 * with (a_theta, A_theta) it is the Nectar output (Eq. (3.5)).
 *
 *   a       DEVICE fp32 [L][Hkv][G][nq]
 *   A_doc   DEVICE fp32 [L][Hkv][G][nq][d]
 *   Q       DEVICE bf16 [L][Hkv][G][nq][d]
 *   q_seq   DEVICE int32 [nq]   sequence of token i, in [0, B)
 *   q_pos   DEVICE int32 [nq]   local position t of token i
 *   Kloc, Vloc  DEVICE bf16 [L][Hkv][B][T_max][d]   local cache per sequence
 *   local_len   DEVICE int32 [B]   valid local tokens of each sequence
 *   out     DEVICE fp32 [L][Hkv][G][nq][d]
 * Visible set of token i (reading of §2.2, Eq. (3.4) indexes i <= t):
 *   { j : j <= q_pos[i] and j < local_len[q_seq[i]] }  -- the token itself
 * included.  An empty visible set gives out = A_doc.
 * ------------------------------------------------------------------------ */
NECTAR_API nectar_status nectar_merge_local(nectar_dims dims, const float *a, const float *A_doc,
                                 const nectar_bf16 *Q, int64_t nq, const int32_t *q_seq,
                                 const int32_t *q_pos, const nectar_bf16 *Kloc,
                                 const nectar_bf16 *Vloc, int32_t B, int32_t T_max,
                                 const int32_t *local_len, float scale, float *out,
                                 nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * Nectar decode: (ii) and (iii) together -- the module forward of every row
 * and the merge of its (a_theta, A_theta) with its exact causal local
 * attention, Eq. (3.5) (§2.2, §2.4).  Arguments as in nectar_module_forward
 * and nectar_merge_local; out DEVICE fp32 [L][Hkv][G][nq][d].  Equal (up to
 * rounding order) to nectar_module_forward followed by nectar_merge_local.
 *
 * Fewer than 64 query rows per KV head (classic module sets): one launch
 * whose CTAs run the module forward (writing A_theta into out) side by side
 * with CTAs that compute each row's local attention state, then a small
 * merge that rewrites out in place.  More rows, or a set with a backbone or
 * unequal nets: the local states first, then the layer-by-layer module,
 * whose last launch merges and writes out.
 *
 *   workspace  DEVICE scratch, 256-byte aligned, of at least
 *              nectar_decode_workspace_size(dims, mods, nq) bytes: the
 *              local state of every row, align256(rows * (d + 2) * 4) with
 *              rows = L * Hkv * G * nq, plus align256(rows * 4) (the
 *              one-launch path) or nectar_module_workspace_size (the
 *              layer-by-layer path), align256(x) rounding x up to a
 *              multiple of 256;
 *              owned by the caller, overwritten, must not be used by
 *              another call in flight.
 * Returns NECTAR_ERR_WORKSPACE when it is missing or too small.
 * ------------------------------------------------------------------------ */
NECTAR_API size_t nectar_decode_workspace_size(nectar_dims dims, const nectar_module_set *mods,
                                               int64_t nq);
NECTAR_API nectar_status nectar_decode(nectar_dims dims, const nectar_module_set *mods,
                            const nectar_bf16 *Q, int64_t nq, const int32_t *q_seq,
                            const int32_t *q_pos, const nectar_bf16 *Kloc,
                            const nectar_bf16 *Vloc, int32_t B, int32_t T_max,
                            const int32_t *local_len, float scale, float *out,
                            void *workspace, size_t workspace_bytes,
                            nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * The decode as a base-model attention layer ("Nectar layer"): the same
 * computation as nectar_decode, written in bf16 straight into the layer
 * layout of the base model's attention output,
 *   out   DEVICE bf16 [L][nq][Hkv * G][d], query head h * G + g
 * (token-major; one [nq][Hkv * G][d] block per layer), rounded to nearest
 * even from the fp32 value nectar_decode would write.  Works for decode
 * (one token per sequence) and for prompts (several tokens of a sequence,
 * q_pos giving each its causal prefix).
 *   workspace  as nectar_decode, of nectar_decode_layer_out_workspace_size
 *              bytes (below 64 query rows per KV head it adds rows * d * 4
 *              bytes, rounded up to 256, for A_theta in fp32).
 * ------------------------------------------------------------------------ */
NECTAR_API size_t nectar_decode_layer_out_workspace_size(nectar_dims dims,
                                                         const nectar_module_set *mods, int64_t nq);
NECTAR_API nectar_status nectar_decode_layer_out(nectar_dims dims, const nectar_module_set *mods,
                                                 const nectar_bf16 *Q, int64_t nq,
                                                 const int32_t *q_seq, const int32_t *q_pos,
                                                 const nectar_bf16 *Kloc, const nectar_bf16 *Vloc,
                                                 int32_t B, int32_t T_max, const int32_t *local_len,
                                                 float scale, nectar_bf16 *out, void *workspace,
                                                 size_t workspace_bytes, nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * Quadrature module (§2.4): per (l, h), p learned key / value rows W, Z
 * (DEVICE bf16 [L][Hkv][p][d]), initialised to the first p rows of the cache;
 *   a_theta(q) = log sum_j exp((W q)_j * scale),
 *   A_theta(q) = softmax(W q * scale)^T Z,
 * i.e. the exact attention of Eq. (3.1) over (W, Z) -- computed by the same
 * kernels as nectar_cache_attn_lse, with the same arguments, outputs,
 * workspace rules and errors (n replaced by p).
 * nectar_quadrature_init copies W[l][h] = K[l][h][0:p], Z[l][h] = V[l][h][0:p]
 * (K, V: DEVICE bf16 [L][Hkv][n][d]; 1 <= p <= n; W, Z must not overlap K, V).
 * ------------------------------------------------------------------------ */
NECTAR_API nectar_status nectar_quadrature_init(nectar_dims dims, const nectar_bf16 *K,
                                                const nectar_bf16 *V, int64_t n, int64_t p,
                                                nectar_bf16 *W, nectar_bf16 *Z,
                                                nectar_stream_t stream);
NECTAR_API size_t nectar_quadrature_workspace_size(nectar_dims dims, int64_t p, int64_t nq);
NECTAR_API nectar_status nectar_quadrature_forward(nectar_dims dims, const nectar_bf16 *W,
                                                   const nectar_bf16 *Z, int64_t p,
                                                   const nectar_bf16 *Q, int64_t nq, float scale,
                                                   float *a, float *A_theta, void *workspace,
                                                   size_t workspace_bytes, nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * Fitting metrics of a module against the exact targets (notes §4 and
 * App. C.4, Eq. (C.1)), per (l, h):
 *   metrics[l][h][0] = mean_q (a - alpha)^2                         score MSE
 *   metrics[l][h][1] = mean_q (1/d) ||A_theta - A||^2               target MSE
 *   metrics[l][h][2] = mean_q log(||A_theta - A||^2 / ||q - A||^2)  RTE term
 * The RTE of Eq. (C.1) is the sum of the third column over (l, h).
 *   alpha, a      DEVICE fp32 [L][Hkv][G][nq]
 *   A, A_theta    DEVICE fp32 [L][Hkv][G][nq][d]
 *   Q             DEVICE bf16 [L][Hkv][G][nq][d]
 *   metrics       DEVICE double [L][Hkv][3], overwritten
 * A row whose ||A_theta - A|| is 0 adds -inf to its RTE term (log 0), one
 * whose q equals A adds +inf or NaN: the definition, unguarded.
 * ------------------------------------------------------------------------ */
NECTAR_API nectar_status nectar_fit_metrics(nectar_dims dims, int64_t nq, const float *alpha,
                                            const float *A, const float *a, const float *A_theta,
                                            const nectar_bf16 *Q, double *metrics,
                                            nectar_stream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostics
 * ------------------------------------------------------------------------ */
NECTAR_API const char *nectar_status_string(nectar_status s);
/* One-line reason for the last non-OK status returned on this thread. */
NECTAR_API const char *nectar_last_error(void);
/* Reads (and, if `clear` is non-zero, resets) the device error word of the
 * current device: bit 0 = a bounded wait gave up, bit 1 = a q_seq entry out
 * of range, bit 2 = a local_len entry out of range.  SYNCHRONISES the
 * device; meant for tests and debugging, not for the hot path. */
NECTAR_API nectar_status nectar_device_error_flags(int32_t *flags, int32_t clear);
/* Self-check of the failure handling behind bit 0.  Every wait inside the
 * library's kernels is bounded: it gives up after a time limit, sets bit 0
 * of the device error word, and the kernel finishes without touching the
 * data the wait guarded, so a lost arrival never hangs the GPU.  This call
 * enqueues one small kernel whose thread waits, through that same bounded
 * wait, on a barrier that nothing arrives on, with a limit of `limit_us`
 * microseconds (1 .. 1000000): the wait runs out, bit 0 is set, the kernel
 * returns and the context stays usable.  NECTAR_ERR_INVALID_ARG for a limit
 * out of range.  For tests and health checks, not for the hot path. */
NECTAR_API nectar_status nectar_check_wait_timeout(int32_t limit_us, nectar_stream_t stream);
/* Library version, "major.minor.patch". */
NECTAR_API const char *nectar_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NECTAR_H_ */
