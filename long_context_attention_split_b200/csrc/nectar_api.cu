// C ABI of libnectar.so: argument validation, work planning and dispatch.
// Every entry point validates on the host and enqueues nothing on error.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/nectar.h"
#include "common.cuh"
#include "kernels.h"
#include "module_layout.h"

namespace nectar {
// The device error word (see nectar_device_error_flags).  Kernels get its
// address through their parameters.
__device__ int g_error_word = 0;
}

using namespace nectar;

namespace {
thread_local char t_last_error[512] = "";
}

void nectar::set_last_error(const char* msg) { snprintf(t_last_error, sizeof t_last_error, "%s", msg); }

// cuCtxGetCurrent and cuCtxGetId through the runtime's driver entry points
// (no link-time dependency on libcuda).  A context id is unique for the
// life of the process, so a context made after a cudaDeviceReset has a new
// one even where the driver reuses the handle.
unsigned long long nectar::current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(ptr);
    ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(ptr);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

namespace {

nectar_status fail(nectar_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return s;
}

nectar_status cuda_fail(cudaError_t e, const char* where) {
  return fail(NECTAR_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nectar_status check_dims(const nectar_dims& d) {
  if (d.L < 1 || d.Hkv < 1 || d.G < 1) return fail(NECTAR_ERR_INVALID_ARG, "dims: L, Hkv, G must be >= 1");
  if (d.d != kD) return fail(NECTAR_ERR_UNSUPPORTED, "dims: d = %d, only d = 128 is supported", d.d);
  if (static_cast<int64_t>(d.L) * d.Hkv > (1 << 20)) return fail(NECTAR_ERR_INVALID_ARG, "dims: too many heads");
  return NECTAR_OK;
}

nectar_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(NECTAR_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return NECTAR_OK;
}

#define NECTAR_TRY(expr)              \
  do {                                \
    nectar_status _s = (expr);        \
    if (_s != NECTAR_OK) return _s;   \
  } while (0)

struct DeviceInfo {
  int sms = 0;
  int* err = nullptr;   // device address of g_error_word on this device
};

// The SM count and the error word's device address of the current device.
// The address belongs to the CUDA context it was looked up in, so the cache
// is keyed on that context's id: after a cudaDeviceReset (or with another
// context current) the next call looks it up again.
DeviceInfo device_info() {
  struct Entry {
    unsigned long long ctx = 0;
    DeviceInfo info;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DeviceInfo{};
  std::lock_guard<std::mutex> lk(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  Entry& e = cache[dev];
  const unsigned long long ctx = current_context_id();
  if (e.info.sms == 0 || ctx == 0 || e.ctx != ctx) {
    int sms = 0;
    void* err = nullptr;
    // the symbol lookup also makes the device's primary context current
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaGetSymbolAddress(&err, nectar::g_error_word) != cudaSuccess)
      return DeviceInfo{};
    e.info.err = static_cast<int*>(err);
    e.info.sms = sms;
    e.ctx = current_context_id();
  }
  return e.info;
}

// Query rows per KV head up to which exact attention stays on the CUDA-core
// split kernel (capped at dec_max_rows()).
#ifndef NECTAR_TC_ROUTE_ROWS
#define NECTAR_TC_ROUTE_ROWS 8
#endif
// 3 to kTctMaxRows query rows per KV head: the transposed tensor-core split
// kernel (attn_tct.cu), where the CUDA-core split kernel is bound by its ALU
// work (measured on a Llama-8B-shaped document at 4 rows: the CUDA-core
// kernel reaches 68 % of the HBM copy bandwidth).  NECTAR_TCT=0
// keeps those rows on the CUDA-core kernel (up to NECTAR_TC_ROUTE_ROWS).
bool use_tct_attn(int64_t rows) {
  const char* e = getenv("NECTAR_TCT");
  return !(e != nullptr && e[0] == '0') && rows >= 3 && rows <= kTctMaxRows;
}
// More query rows per KV head than those: the tensor-core kernel.
bool use_tc_attn(int64_t rows) {
  if (use_tct_attn(rows)) return false;
  const int64_t lim = NECTAR_TC_ROUTE_ROWS < dec_max_rows() ? NECTAR_TC_ROUTE_ROWS : dec_max_rows();
  return rows > lim;
}

int dec_row_block(int64_t rows) { return rows < dec_max_rows() ? static_cast<int>(rows) : dec_max_rows(); }

DecPlan cache_attn_plan(const nectar_dims& d, int64_t n, int64_t nq, int sms) {
  const int64_t rows = static_cast<int64_t>(d.G) * nq;
  if (use_tct_attn(rows)) return plan_decode(d.L * d.Hkv, n, sms, cache_attn_tct_ctas_per_sm(rows), kTctTile);
  const int R = dec_row_block(rows);
  return plan_decode(d.L * d.Hkv, n, sms, dec_ctas_per_sm(R < 1 ? 1 : R), dec_tile(R < 1 ? 1 : R));
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims / strides innermost first,
// strides in bytes for dims 1..rank-1.
nectar_status make_tmap(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                        const cuuint64_t* strides, const cuuint32_t* box, const char* what) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return fail(NECTAR_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NECTAR_ERR_CUDA, "tensor map for %s: CUresult %d", what, static_cast<int>(r));
  return NECTAR_OK;
}

}  // namespace

// One thread waits, through the library's bounded wait, on an mbarrier
// that nothing arrives on; the wait gives up after limit_ns, records
// DEVERR_WAIT_TIMEOUT and the kernel returns.
__global__ void wait_timeout_kernel(uint64_t limit_ns, int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0, err, limit_ns);
}

extern "C" {

const char* nectar_version(void) { return "0.1.0"; }

nectar_status nectar_check_wait_timeout(int32_t limit_us, nectar_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return fail(NECTAR_ERR_INVALID_ARG, "limit_us = %d: need 1..1000000", limit_us);
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_us) * 1000u,
                                                                           di.err);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "wait timeout check kernel");
}

const char* nectar_status_string(nectar_status s) {
  switch (s) {
    case NECTAR_OK: return "ok";
    case NECTAR_ERR_INVALID_ARG: return "invalid argument";
    case NECTAR_ERR_UNSUPPORTED: return "unsupported";
    case NECTAR_ERR_WORKSPACE: return "workspace too small";
    case NECTAR_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* nectar_last_error(void) { return t_last_error; }

nectar_status nectar_device_error_flags(int32_t* flags, int32_t clear) {
  if (flags == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "flags is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "nectar_device_error_flags");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, nectar::g_error_word, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e, "nectar_device_error_flags");
  *flags = v;
  if (clear) {
    const int z = 0;
    e = cudaMemcpyToSymbol(nectar::g_error_word, &z, sizeof z);
    if (e != cudaSuccess) return cuda_fail(e, "nectar_device_error_flags");
  }
  return NECTAR_OK;
}

// ---------------------------------------------------------------------------
// (i) exact cached-token attention
// ---------------------------------------------------------------------------
size_t nectar_cache_attn_workspace_size(nectar_dims dims, int64_t n, int64_t nq) {
  if (check_dims(dims) != NECTAR_OK || n < 0 || nq < 0) return 0;
  const int64_t rows = static_cast<int64_t>(dims.G) * nq;
  if (rows == 0 || n == 0) return 0;
  const DeviceInfo di = device_info();
  if (di.sms == 0) return 0;
  if (use_tc_attn(rows)) {
    const TcPlan tp = plan_tc(dims.L * dims.Hkv, n, rows, di.sms);
    return tp.ws_bytes + 256;
  }
  const DecPlan pl = cache_attn_plan(dims, n, nq, di.sms);
  const int64_t prow = static_cast<int64_t>(dims.L) * dims.Hkv * pl.S_max * rows;
  return static_cast<size_t>(prow) * (kD + 2) * sizeof(float) + 256;
}

nectar_status nectar_cache_attn_lse(nectar_dims dims, const nectar_bf16* K, const nectar_bf16* V,
                                    int64_t n, const nectar_bf16* Q, int64_t nq, float scale,
                                    float* alpha, float* A, void* workspace, size_t workspace_bytes,
                                    nectar_stream_t stream) {
  NECTAR_TRY(check_dims(dims));
  if (n < 0 || nq < 0) return fail(NECTAR_ERR_INVALID_ARG, "n and nq must be >= 0");
  if (!(scale == scale)) return fail(NECTAR_ERR_INVALID_ARG, "scale is NaN");
  if (nq == 0) return NECTAR_OK;
  const int heads = dims.L * dims.Hkv;
  const int64_t rows = static_cast<int64_t>(dims.G) * nq;
  if (rows > (int64_t(1) << 30)) return fail(NECTAR_ERR_INVALID_ARG, "too many query rows");
  NECTAR_TRY(check_ptr(Q, "Q"));
  if (alpha == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "alpha is NULL");
  NECTAR_TRY(check_ptr(A, "A"));
  if (n > 0) {
    NECTAR_TRY(check_ptr(K, "K"));
    NECTAR_TRY(check_ptr(V, "V"));
  }
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");

  DecParams p{};
  p.K = reinterpret_cast<const __nv_bfloat16*>(K);
  p.V = reinterpret_cast<const __nv_bfloat16*>(V);
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.n = n;
  p.heads = heads;
  p.rows_total = rows;
  p.qmul = scale * kLog2e;
  p.err = di.err;
  const DecPlan pl = cache_attn_plan(dims, n, nq, di.sms);
  p.tile = pl.tile;
  p.tph = pl.tph;
  p.total = pl.total;
  p.C = pl.C;
  p.S_max = pl.S_max;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (n == 0) {
    cudaError_t e = launch_cache_attn_combine(p, alpha, A, st);
    return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "cache_attn (n = 0)");
  }
  const size_t need = nectar_cache_attn_workspace_size(dims, n, nq);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(NECTAR_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(NECTAR_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  if (use_tc_attn(rows)) {
    // many query rows per head: tcgen05 flash-style kernel
    const TcPlan tp = plan_tc(heads, n, rows, di.sms);
    TcParams tpar{};
    tpar.n = n;
    tpar.heads = heads;
    tpar.rows_total = rows;
    tpar.qpairs = tp.qpairs;
    tpar.tph = tp.tph;
    tpar.C = tp.C;
    tpar.dp_rounds = tp.dp_rounds;
    tpar.sk_units = tp.sk_units;
    tpar.sk_parts = tp.sk_parts;
    tpar.qmul = scale * kLog2e;
    tpar.alpha = alpha;
    tpar.A = A;
    tpar.ws_acc = reinterpret_cast<float*>(workspace);
    tpar.ws_ml = tpar.ws_acc + static_cast<int64_t>(tp.C) * 2 * 256 * kD;
    tpar.err = di.err;
    // 4-D views [heads][2 halves of d][rows][64] so that one box brings both
    // 64-column halves of a tile (each then a K-major, 128-byte-swizzled
    // operand of 128-byte rows)
    CUtensorMap tq, tk, tv;
    const cuuint64_t dq[4] = {64, static_cast<cuuint64_t>(rows), 2, static_cast<cuuint64_t>(heads)};
    const cuuint64_t sq[3] = {256, 128, static_cast<cuuint64_t>(rows) * 256};
    const cuuint64_t dk[4] = {64, static_cast<cuuint64_t>(n), 2, static_cast<cuuint64_t>(heads)};
    const cuuint64_t sk[3] = {256, 128, static_cast<cuuint64_t>(n) * 256};
    const bool dup = cache_attn_tc_dup(rows);
    const cuuint32_t boxq[4] = {64, dup ? 64u : 128u, dup ? 1u : 2u, 1};
    const cuuint32_t boxk[4] = {64, 64, 2, 1};
    NECTAR_TRY(make_tmap(&tq, Q, 4, dq, sq, boxq, "Q"));
    NECTAR_TRY(make_tmap(&tk, K, 4, dk, sk, boxk, "K"));
    NECTAR_TRY(make_tmap(&tv, V, 4, dk, sk, boxk, "V"));
    cudaError_t e = launch_cache_attn_tc(tq, tk, tv, tpar, st);
    return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "cache_attn tensor-core kernel");
  }
  const int64_t prow = static_cast<int64_t>(heads) * pl.S_max * rows;
  p.ws_acc = reinterpret_cast<float*>(workspace);
  p.ws_ml = p.ws_acc + prow * kD;
  if (use_tct_attn(rows)) {
    // K, V as [heads][2 halves of d][n][64]: one box = 128 keys, both halves;
    // Q as [heads][2 halves][rows][64]: one box per half
    CUtensorMap tq, tk, tv;
    const cuuint64_t dq[4] = {64, static_cast<cuuint64_t>(rows), 2, static_cast<cuuint64_t>(heads)};
    const cuuint64_t sq[3] = {256, 128, static_cast<cuuint64_t>(rows) * 256};
    const cuuint64_t dk[4] = {64, static_cast<cuuint64_t>(n), 2, static_cast<cuuint64_t>(heads)};
    const cuuint64_t sk[3] = {256, 128, static_cast<cuuint64_t>(n) * 256};
    const cuuint32_t boxq[4] = {64, static_cast<cuuint32_t>(rows), 1, 1};
    const cuuint32_t boxk[4] = {64, static_cast<cuuint32_t>(kTctTile), 2, 1};
    NECTAR_TRY(make_tmap(&tq, Q, 4, dq, sq, boxq, "Q"));
    NECTAR_TRY(make_tmap(&tk, K, 4, dk, sk, boxk, "K"));
    NECTAR_TRY(make_tmap(&tv, V, 4, dk, sk, boxk, "V"));
    cudaError_t e = launch_cache_attn_tct(tq, tk, tv, p, st);
    if (e != cudaSuccess) return cuda_fail(e, "cache_attn transposed tensor-core kernel");
    e = launch_cache_attn_combine(p, alpha, A, st);
    return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "cache_attn combine kernel");
  }

  const int RB = dec_row_block(rows);
  for (int64_t r0 = 0; r0 < rows; r0 += RB) {
    p.row0 = static_cast<int>(r0);
    const int R = static_cast<int>((rows - r0) < RB ? (rows - r0) : RB);
    cudaError_t e = launch_cache_attn_split(p, R, st);
    if (e != cudaSuccess) return cuda_fail(e, "cache_attn split kernel");
  }
  cudaError_t e = launch_cache_attn_combine(p, alpha, A, st);
  if (e != cudaSuccess) return cuda_fail(e, "cache_attn combine kernel");
  return NECTAR_OK;
}

// ---------------------------------------------------------------------------
// (iii) merge with local attention
// ---------------------------------------------------------------------------
static nectar_status check_local(const int32_t* q_seq, const int32_t* q_pos, const nectar_bf16* Kloc,
                                 const nectar_bf16* Vloc, int32_t B, int32_t T_max,
                                 const int32_t* local_len) {
  if (B < 0 || T_max < 0) return fail(NECTAR_ERR_INVALID_ARG, "B and T_max must be >= 0");
  if (q_seq == nullptr || q_pos == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "q_seq / q_pos is NULL");
  if (B > 0) {
    if (local_len == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "local_len is NULL");
    if (T_max > 0) {
      NECTAR_TRY(check_ptr(Kloc, "Kloc"));
      NECTAR_TRY(check_ptr(Vloc, "Vloc"));
    }
  }
  return NECTAR_OK;
}

// Many query tokens: the local attention runs on the tensor cores
// (local_tc.cu), one job per (KV head, token).
static bool use_local_tc(const nectar_dims& dims, int64_t nq, int32_t B, int32_t T_max) {
  return static_cast<int64_t>(dims.G) * nq >= kGemmMinRows && dims.G <= 64 && B > 0 && T_max > 0;
}

// Either leaves each row's local state in ws_loc (out == nullptr) or merges
// it with (a, A_doc) into out.  `transposed` picks local_tct_kernel (keys on
// the TMEM lanes; G <= 16, T_max <= 512) over local_tc_kernel (query heads
// on the TMEM lanes); both take the same parameters and tensor maps.
static nectar_status run_local_tc(bool transposed, const nectar_dims& dims, const nectar_bf16* Q, int64_t nq,
                                  const int32_t* q_seq, const int32_t* q_pos, const nectar_bf16* Kloc,
                                  const nectar_bf16* Vloc, int32_t B, int32_t T_max, const int32_t* local_len,
                                  float scale, float* ws_loc, const float* a, const float* A_doc, float* out,
                                  cudaStream_t st) {
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");
  const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
  if (heads * B > 0x7fffffffLL || heads > 0x7fffffffLL || nq > 0x7fffffffLL)
    return fail(NECTAR_ERR_UNSUPPORTED, "local cache too large for one call");
  LocalParams p{};
  p.njobs = heads * nq;
  p.nq = nq;
  p.G = dims.G;
  p.B = B;
  p.T = T_max;
  p.kbox = T_max < 128 ? T_max : 128;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.Kloc = reinterpret_cast<const __nv_bfloat16*>(Kloc);
  p.Vloc = reinterpret_cast<const __nv_bfloat16*>(Vloc);
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.local_len = local_len;
  p.qmul = scale * kLog2e;
  p.ws_loc = ws_loc;
  p.a = a;
  p.A_doc = A_doc;
  p.out = out;
  p.err = di.err;
  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dq[4] = {128, static_cast<cuuint64_t>(nq), static_cast<cuuint64_t>(dims.G),
                              static_cast<cuuint64_t>(heads)};
    const cuuint64_t sq[3] = {256, static_cast<cuuint64_t>(nq) * 256, static_cast<cuuint64_t>(nq) * 256 * dims.G};
    const cuuint32_t bq[4] = {64, 1, static_cast<cuuint32_t>(dims.G), 1};
    NECTAR_TRY(make_tmap(&tq, Q, 4, dq, sq, bq, "queries (per token)"));
    // local caches as [heads * B][2 halves][T][64]: one box = kbox keys of one half
    const cuuint64_t dk[4] = {64, static_cast<cuuint64_t>(T_max), 2, static_cast<cuuint64_t>(heads * B)};
    const cuuint64_t sk[3] = {256, 128, static_cast<cuuint64_t>(T_max) * 256};
    const cuuint32_t bk[4] = {64, static_cast<cuuint32_t>(p.kbox), 1, 1};
    NECTAR_TRY(make_tmap(&tk, Kloc, 4, dk, sk, bk, "local keys"));
    NECTAR_TRY(make_tmap(&tv, Vloc, 4, dk, sk, bk, "local values"));
  }
  cudaError_t e;
  if (transposed) {
    e = launch_local_tct(tq, tk, tv, p, di.sms, st);
  } else {
    const int grid = static_cast<int>(p.njobs < di.sms ? p.njobs : di.sms);
    e = launch_local_tc(tq, tk, tv, p, grid, st);
  }
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "local attention kernel");
}

// The same result from the warp-per-job CUDA-core kernel (local_warp.cu).
static nectar_status run_local_warp(const nectar_dims& dims, const nectar_bf16* Q, int64_t nq,
                                    const int32_t* q_seq, const int32_t* q_pos, const nectar_bf16* Kloc,
                                    const nectar_bf16* Vloc, int32_t B, int32_t T_max, const int32_t* local_len,
                                    float scale, float* ws_loc, const float* a, const float* A_doc, float* out,
                                    cudaStream_t st) {
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");
  LocalParams p{};
  p.njobs = static_cast<int64_t>(dims.L) * dims.Hkv * nq;
  p.nq = nq;
  p.G = dims.G;
  p.B = B;
  p.T = T_max;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.Kloc = reinterpret_cast<const __nv_bfloat16*>(Kloc);
  p.Vloc = reinterpret_cast<const __nv_bfloat16*>(Vloc);
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.local_len = local_len;
  p.qmul = scale * kLog2e;
  p.ws_loc = ws_loc;
  p.a = a;
  p.A_doc = A_doc;
  p.out = out;
  p.err = di.err;
  cudaError_t e = launch_local_warp(p, di.sms, st);
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "local attention kernel");
}

// Which kernel runs the local attention of many query tokens.  Default: the
// transposed tensor-core kernel where it applies (G <= 16, at most 512 local
// tokens), else warps for G <= 8 and the row-per-head tensor-core kernel
// above.  NECTAR_LOCAL_TCT=0 turns the transposed kernel off.
static bool use_local_tct(const nectar_dims& dims, int32_t T_max) {
  if (dims.G > 16 || T_max > 512) return false;
  const char* env = getenv("NECTAR_LOCAL_TCT");
  return env == nullptr || atoi(env) != 0;
}

static nectar_status run_local_many(const nectar_dims& dims, const nectar_bf16* Q, int64_t nq,
                                    const int32_t* q_seq, const int32_t* q_pos, const nectar_bf16* Kloc,
                                    const nectar_bf16* Vloc, int32_t B, int32_t T_max, const int32_t* local_len,
                                    float scale, float* ws_loc, const float* a, const float* A_doc, float* out,
                                    cudaStream_t st) {
  if (use_local_tct(dims, T_max))
    return run_local_tc(true, dims, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, ws_loc, a, A_doc,
                        out, st);
  if (dims.G <= 8)
    return run_local_warp(dims, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, ws_loc, a, A_doc, out,
                          st);
  return run_local_tc(false, dims, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, ws_loc, a, A_doc,
                      out, st);
}

nectar_status nectar_merge_local(nectar_dims dims, const float* a, const float* A_doc, const nectar_bf16* Q,
                                 int64_t nq, const int32_t* q_seq, const int32_t* q_pos,
                                 const nectar_bf16* Kloc, const nectar_bf16* Vloc, int32_t B, int32_t T_max,
                                 const int32_t* local_len, float scale, float* out, nectar_stream_t stream) {
  NECTAR_TRY(check_dims(dims));
  if (nq < 0) return fail(NECTAR_ERR_INVALID_ARG, "nq must be >= 0");
  if (nq == 0) return NECTAR_OK;
  if (!(scale == scale)) return fail(NECTAR_ERR_INVALID_ARG, "scale is NaN");
  if (a == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "a is NULL");
  NECTAR_TRY(check_ptr(A_doc, "A_doc"));
  NECTAR_TRY(check_ptr(Q, "Q"));
  NECTAR_TRY(check_ptr(out, "out"));
  NECTAR_TRY(check_local(q_seq, q_pos, Kloc, Vloc, B, T_max, local_len));
  if (use_local_tc(dims, nq, B, T_max))
    return run_local_many(dims, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, nullptr, a, A_doc, out,
                          reinterpret_cast<cudaStream_t>(stream));
  if (static_cast<int64_t>(dims.L) * dims.Hkv * nq * ((dims.G + 7) / 8) > 0x7fffffffLL)
    return fail(NECTAR_ERR_INVALID_ARG, "too many (head, token) units");
  MergeParams p{};
  p.a = a;
  p.A_doc = A_doc;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.Kloc = reinterpret_cast<const __nv_bfloat16*>(Kloc);
  p.Vloc = reinterpret_cast<const __nv_bfloat16*>(Vloc);
  p.local_len = local_len;
  p.out = out;
  p.heads = dims.L * dims.Hkv;
  p.G = dims.G;
  p.nq = nq;
  p.B = B;
  p.T = T_max;
  p.qmul = scale * kLog2e;
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");
  p.err = di.err;
  cudaError_t e = launch_merge_local(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "merge_local kernel");
}

// ---------------------------------------------------------------------------
// module packing (host only)
// ---------------------------------------------------------------------------
static nectar_status check_modules_shape(const nectar_dims& dims, int32_t depth, const int32_t* width) {
  NECTAR_TRY(check_dims(dims));
  if (depth < 1 || depth > NECTAR_MAX_DEPTH)
    return fail(NECTAR_ERR_UNSUPPORTED, "depth %d outside [1, %d]", depth, NECTAR_MAX_DEPTH);
  if (width == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "width is NULL");
  if (dims.L > NECTAR_MAX_LAYERS) return fail(NECTAR_ERR_UNSUPPORTED, "L = %d > %d", dims.L, NECTAR_MAX_LAYERS);
  for (int l = 0; l < dims.L; ++l) {
    const int H = width[l];
    if (H < 16 || H > NECTAR_MAX_WIDTH || H % 16 != 0)
      return fail(NECTAR_ERR_UNSUPPORTED, "width[%d] = %d: need a multiple of 16 in [16, %d]", l, H,
                  NECTAR_MAX_WIDTH);
  }
  return NECTAR_OK;
}

// The architecture of a module set: the classic one (both nets `depth`
// layers of width[l], no backbone) or the one mods->arch gives.
struct Arch {
  int Db, Ds, Dt;
  const int32_t* wb;   // null when Db = 0
  const int32_t* ws;
  const int32_t* wt;
  bool general;        // a backbone or unequal nets: layer-by-layer path only
};

static nectar_status check_widths(const nectar_dims& dims, const int32_t* w, const char* what) {
  if (w == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "%s is NULL", what);
  for (int l = 0; l < dims.L; ++l)
    if (w[l] < 16 || w[l] > NECTAR_MAX_WIDTH || w[l] % 16 != 0)
      return fail(NECTAR_ERR_UNSUPPORTED, "%s[%d] = %d: need a multiple of 16 in [16, %d]", what, l, w[l],
                  NECTAR_MAX_WIDTH);
  return NECTAR_OK;
}

static nectar_status arch_check(const nectar_dims& dims, const nectar_module_arch* a, Arch* out) {
  NECTAR_TRY(check_dims(dims));
  if (a == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "arch is NULL");
  if (dims.L > NECTAR_MAX_LAYERS) return fail(NECTAR_ERR_UNSUPPORTED, "L = %d > %d", dims.L, NECTAR_MAX_LAYERS);
  if (a->depth_b < 0 || a->depth_s < 1 || a->depth_t < 1 ||
      a->depth_b + (a->depth_s > a->depth_t ? a->depth_s : a->depth_t) > NECTAR_MAX_DEPTH)
    return fail(NECTAR_ERR_UNSUPPORTED, "depths (%d, %d, %d): need depth_b >= 0, branches >= 1 and chains <= %d",
                a->depth_b, a->depth_s, a->depth_t, NECTAR_MAX_DEPTH);
  if (a->depth_b > 0) NECTAR_TRY(check_widths(dims, a->width_b, "width_b"));
  NECTAR_TRY(check_widths(dims, a->width_s, "width_s"));
  NECTAR_TRY(check_widths(dims, a->width_t, "width_t"));
  out->Db = a->depth_b;
  out->Ds = a->depth_s;
  out->Dt = a->depth_t;
  out->wb = a->depth_b > 0 ? a->width_b : nullptr;
  out->ws = a->width_s;
  out->wt = a->width_t;
  bool eq = a->depth_b == 0 && a->depth_s == a->depth_t;
  for (int l = 0; eq && l < dims.L; ++l) eq = a->width_s[l] == a->width_t[l];
  out->general = !eq;
  return NECTAR_OK;
}

static nectar_status arch_of(const nectar_dims& dims, const nectar_module_set* mods, Arch* out) {
  if (mods == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "mods is NULL");
  if (mods->arch != nullptr) return arch_check(dims, mods->arch, out);
  NECTAR_TRY(check_modules_shape(dims, mods->depth, mods->width));
  *out = Arch{0, mods->depth, mods->depth, nullptr, mods->width, mods->width, false};
  return NECTAR_OK;
}

static int arch_hb(const Arch& a, int l) { return a.Db > 0 ? a.wb[l] : 0; }

static int64_t arch_head_elems(const Arch& a, int l) {
  return layout::head_elems_arch(a.Db, arch_hb(a, l), a.Ds, a.ws[l], a.Dt, a.wt[l]);
}

static int64_t arch_packed_elems(const nectar_dims& dims, const Arch& a) {
  int64_t tot = 0;
  for (int l = 0; l < dims.L; ++l) tot += static_cast<int64_t>(dims.Hkv) * arch_head_elems(a, l);
  return tot;
}

// Writes one hidden layer of Hkv heads' weights into the tiled layout: the
// logical matrix [H][d + P] takes its first d columns from Vq (or, for a
// layer that starts a chain, P = 0, from U) and the rest from U [H][P].
static void pack_hidden(nectar_bf16* W, nectar_bf16* bias, int h, int H, int P, const nectar_bf16* U,
                        const nectar_bf16* Vq, const nectar_bf16* b) {
  const int K = kD + P;
  for (int i = 0; i < H; ++i)
    for (int c = 0; c < K; ++c) {
      nectar_bf16 v;
      if (P == 0) v = U[(static_cast<int64_t>(h) * H + i) * kD + c];
      else if (c < kD) v = Vq[(static_cast<int64_t>(h) * H + i) * kD + c];
      else v = U[(static_cast<int64_t>(h) * H + i) * P + (c - kD)];
      W[layout::chunked_index(H, K, c, i)] = v;
    }
  for (int i = 0; i < H; ++i) bias[i] = b[static_cast<int64_t>(h) * H + i];
}

int64_t nectar_module_packed_elems_arch(nectar_dims dims, const nectar_module_arch* arch) {
  Arch a;
  if (arch_check(dims, arch, &a) != NECTAR_OK) return 0;
  return arch_packed_elems(dims, a);
}

nectar_status nectar_module_pack_arch(nectar_dims dims, const nectar_module_arch* arch, const nectar_net_host* nets,
                                      nectar_bf16* blob, int64_t blob_elems) {
  Arch a;
  NECTAR_TRY(arch_check(dims, arch, &a));
  if (nets == nullptr || blob == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "nets / blob is NULL");
  const int64_t need = arch_packed_elems(dims, a);
  if (blob_elems < need) return fail(NECTAR_ERR_INVALID_ARG, "blob has %lld elements, %lld needed",
                                     (long long)blob_elems, (long long)need);
  for (int l = 0; l < dims.L; ++l) {
    const int depths[3] = {a.Db, a.Ds, a.Dt};
    for (int part = 0; part < 3; ++part) {
      const nectar_net_host& nh = nets[3 * l + part];
      for (int k = 0; k < depths[part]; ++k) {
        const bool starts = (part == 0 && k == 0) || (part > 0 && k == 0 && a.Db == 0);
        if (nh.U[k] == nullptr || nh.b[k] == nullptr || (!starts && nh.V[k] == nullptr))
          return fail(NECTAR_ERR_INVALID_ARG, "layer %d part %d: missing U/V/b[%d]", l, part, k);
      }
      if (part > 0 && (nh.Wout == nullptr || nh.c == nullptr))
        return fail(NECTAR_ERR_INVALID_ARG, "layer %d part %d: missing Wout / c", l, part);
    }
  }
  memset(blob, 0, sizeof(nectar_bf16) * need);
  int64_t base = 0;
  for (int l = 0; l < dims.L; ++l) {
    const int Hb = arch_hb(a, l), Hs = a.ws[l], Ht = a.wt[l];
    const int64_t per_head = arch_head_elems(a, l);
    for (int h = 0; h < dims.Hkv; ++h) {
      const int64_t hb = base + h * per_head;
      const nectar_net_host& bb = nets[3 * l];
      for (int k = 0; k < a.Db; ++k) {
        nectar_bf16* W = blob + hb + layout::backbone_w_off(Hb, k);
        const int P = k == 0 ? 0 : Hb;
        pack_hidden(W, W + layout::chunked_elems(Hb, kD + P), h, Hb, P, bb.U[k], bb.V[k], bb.b[k]);
      }
      for (int net = 0; net < 2; ++net) {
        const nectar_net_host& nh = nets[3 * l + 1 + net];
        const int Hn = net ? Ht : Hs, Dn = net ? a.Dt : a.Ds, dout = net ? kD : 1;
        const int64_t nb = hb + layout::branch_base(a.Db, Hb, a.Ds, Hs, net);
        for (int j = 0; j < Dn; ++j) {
          const int P = layout::branch_prev(a.Db, Hb, Hn, j);
          pack_hidden(blob + nb + layout::branch_w_off(a.Db, Hb, Hn, j), blob + nb + layout::branch_b_off(a.Db, Hb, Hn, j),
                      h, Hn, P, nh.U[j], nh.V[j], nh.b[j]);
        }
        nectar_bf16* Wo = blob + nb + layout::branch_out_w_off(a.Db, Hb, Hn, Dn);
        if (dout == 1) {
          for (int i = 0; i < Hn; ++i) Wo[i] = nh.Wout[static_cast<int64_t>(h) * Hn + i];
        } else {
          for (int o = 0; o < dout; ++o)
            for (int c = 0; c < Hn; ++c)
              Wo[layout::chunked_index(kD, Hn, c, o)] = nh.Wout[(static_cast<int64_t>(h) * dout + o) * Hn + c];
        }
        nectar_bf16* cb = blob + nb + layout::branch_out_b_off(a.Db, Hb, Hn, Dn, dout);
        for (int o = 0; o < dout; ++o) cb[o] = nh.c[static_cast<int64_t>(h) * dout + o];
      }
    }
    base += static_cast<int64_t>(dims.Hkv) * per_head;
  }
  return NECTAR_OK;
}

int64_t nectar_module_packed_elems(nectar_dims dims, int32_t depth, const int32_t* width) {
  if (check_modules_shape(dims, depth, width) != NECTAR_OK) return 0;
  int64_t tot = 0;
  for (int l = 0; l < dims.L; ++l) tot += static_cast<int64_t>(dims.Hkv) * layout::head_elems(width[l], depth);
  return tot;
}

nectar_status nectar_module_pack(nectar_dims dims, int32_t depth, const int32_t* width,
                                 const nectar_net_host* nets, nectar_bf16* blob, int64_t blob_elems) {
  NECTAR_TRY(check_modules_shape(dims, depth, width));
  if (nets == nullptr || blob == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "nets / blob is NULL");
  const int64_t need = nectar_module_packed_elems(dims, depth, width);
  if (blob_elems < need) return fail(NECTAR_ERR_INVALID_ARG, "blob has %lld elements, %lld needed",
                                     (long long)blob_elems, (long long)need);
  for (int l = 0; l < dims.L; ++l)
    for (int net = 0; net < 2; ++net) {
      const nectar_net_host& nh = nets[2 * l + net];
      for (int k = 0; k < depth; ++k) {
        if (nh.U[k] == nullptr || nh.b[k] == nullptr || (k > 0 && nh.V[k] == nullptr))
          return fail(NECTAR_ERR_INVALID_ARG, "layer %d net %d: missing U/V/b[%d]", l, net, k);
      }
      if (nh.Wout == nullptr || nh.c == nullptr)
        return fail(NECTAR_ERR_INVALID_ARG, "layer %d net %d: missing Wout / c", l, net);
    }
  memset(blob, 0, sizeof(nectar_bf16) * need);
  int64_t base = 0;
  for (int l = 0; l < dims.L; ++l) {
    const int H = width[l];
    const int64_t per_head = layout::head_elems(H, depth);
    for (int h = 0; h < dims.Hkv; ++h) {
      for (int net = 0; net < 2; ++net) {
        const nectar_net_host& nh = nets[2 * l + net];
        const int dout = net == 0 ? 1 : kD;
        const int64_t nb = base + h * per_head + (net ? layout::net_elems(H, depth, 1) : 0);
        for (int k = 0; k < depth; ++k) {
          const int Kk = layout::hidden_k(H, k);
          // logical W_k[i][c]: c < d from V_k (k>=1) or U_0 (k=0); c >= d from U_k
          nectar_bf16* W = blob + nb + layout::hidden_w_off(H, depth, k);
          for (int i = 0; i < H; ++i)
            for (int c = 0; c < Kk; ++c) {
              nectar_bf16 v;
              if (k == 0) v = nh.U[0][(static_cast<int64_t>(h) * H + i) * kD + c];
              else if (c < kD) v = nh.V[k][(static_cast<int64_t>(h) * H + i) * kD + c];
              else v = nh.U[k][(static_cast<int64_t>(h) * H + i) * H + (c - kD)];
              W[layout::chunked_index(H, Kk, c, i)] = v;
            }
          nectar_bf16* bb = blob + nb + layout::hidden_b_off(H, depth, k);
          for (int i = 0; i < H; ++i) bb[i] = nh.b[k][static_cast<int64_t>(h) * H + i];
        }
        nectar_bf16* Wo = blob + nb + layout::out_w_off(H, depth);
        if (dout == 1) {
          for (int i = 0; i < H; ++i) Wo[i] = nh.Wout[static_cast<int64_t>(h) * H + i];
        } else {
          for (int o = 0; o < dout; ++o)
            for (int c = 0; c < H; ++c)
              Wo[layout::chunked_index(kD, H, c, o)] = nh.Wout[(static_cast<int64_t>(h) * dout + o) * H + c];
        }
        nectar_bf16* cb = blob + nb + layout::out_b_off(H, depth, dout);
        for (int o = 0; o < dout; ++o) cb[o] = nh.c[static_cast<int64_t>(h) * dout + o];
      }
    }
    base += static_cast<int64_t>(dims.Hkv) * per_head;
  }
  return NECTAR_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// (ii) module forward and the fused decode
// ---------------------------------------------------------------------------
namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// bytes of the decode workspace's a_theta part (rounded so the local states
// that follow start 256-byte aligned)
size_t decode_ws_a_bytes(int64_t rows) { return align256(static_cast<size_t>(rows) * sizeof(float)); }

// Many query rows per KV head, or a set with a backbone or unequal nets:
// the module runs layer by layer as grouped GEMMs (module_gemm.cu) instead
// of one CTA per block of <= 64 rows.  So do widths whose M tiles, side by
// side for the G rows of one token, would need more than 512 TMEM columns
// in the one-CTA kernel.
int arch_hmax(const nectar_dims& dims, const Arch& a);
bool use_gemm_path(const nectar_dims& dims, int64_t nq, bool general, int Hmax) {
  if (general || static_cast<int64_t>(dims.G) * nq >= kGemmMinRows) return true;
  const int mt = (Hmax + 127) / 128;
  return mt * ((dims.G + 15) / 16 * 16) > 512;
}

// widest layer of any part, widest score net, hidden layers of the longest chain
int arch_hmax(const nectar_dims& dims, const Arch& a) {
  int H = 0;
  for (int l = 0; l < dims.L; ++l) {
    H = std::max(H, std::max(a.ws[l], a.wt[l]));
    if (a.Db > 0) H = std::max(H, a.wb[l]);
  }
  return H;
}
int arch_hsmax(const nectar_dims& dims, const Arch& a) {
  int H = 0;
  for (int l = 0; l < dims.L; ++l) H = std::max(H, a.ws[l]);
  return H;
}
int arch_stages(const Arch& a) { return a.Db + std::max(a.Ds, a.Dt); }

// Workspace of the layer-by-layer path: hidden activations (two buffers
// when the longest chain has >= 2 layers, each [2 slots][rows][Hp] bf16),
// then the score partials [rows][MT] fp32.
size_t gemm_h_bytes(const nectar_dims& dims, int Hmax, int64_t nq) {
  const int64_t rows = static_cast<int64_t>(dims.L) * dims.Hkv * dims.G * nq;
  return align256(static_cast<size_t>(2 * rows) * layout::round64(Hmax) * 2);
}
size_t gemm_ws_bytes(const nectar_dims& dims, const Arch& a, int64_t nq) {
  const int64_t rows = static_cast<int64_t>(dims.L) * dims.Hkv * dims.G * nq;
  const int MT = (arch_hsmax(dims, a) + 127) / 128;
  return (arch_stages(a) >= 2 ? 2 : 1) * gemm_h_bytes(dims, arch_hmax(dims, a), nq) +
         align256(static_cast<size_t>(rows) * MT * 4);
}

// Rows per readout tile.  The readout has a single 128-dim M tile per head,
// and every row tile streams the head's whole W_out again, so tiles are as
// tall as possible (up to 256 rows) while there are still at least four
// tiles per SM; with fewer rows per head they shrink (down to 64) so that
// all SMs get work.
int readout_rows(int64_t heads, int64_t R, int sms) {
  for (int mr = 256; mr > 64; mr /= 2)
    if (heads * ((R + mr - 1) / mr) >= 4 * static_cast<int64_t>(sms)) return mr;
  return 64;
}

// The layer-by-layer module forward: depth hidden-layer launches and one
// readout launch.  With ws_loc the readout merges with the local states
// (decode) and writes the output into A_out.
nectar_status run_module_gemm(const nectar_dims& dims, const ModParams& mp, const nectar_bf16* Q, int64_t nq,
                              float* a, float* A_out, const float* ws_loc, void* ws, cudaStream_t st,
                              __nv_bfloat16* out_bf16 = nullptr) {
  const DeviceInfo di = device_info();
  const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
  const int64_t R = static_cast<int64_t>(dims.G) * nq;
  if (heads * R * 2 > 0x7fffffffLL) return fail(NECTAR_ERR_UNSUPPORTED, "too many query rows for one call");
  const GemmShape sh = gemm_shape(R, 256);
  const GemmShape shr = gemm_shape(R, readout_rows(heads, R, di.sms));
  GemmParams g;
  memset(&g, 0, sizeof(g));
  g.L = dims.L;
  g.Hkv = dims.Hkv;
  g.depth_b = mp.depth_b;
  g.depth_s = mp.depth_s;
  g.depth_t = mp.depth_t;
  g.nlayers = dims.L;
  g.R = static_cast<int>(R);
  g.NR = sh.NR;
  g.rtiles = sh.rtiles;
  g.Hp = layout::round64(mp.Hmax);
  int Hsmax = 0;
  for (int l = 0; l < dims.L; ++l) Hsmax = std::max(Hsmax, mp.width[l]);
  g.MT = (Hsmax + 127) / 128;
  g.stages = sh.stages;
  g.tmem_cols = sh.tmem_cols;
  g.blob = mp.blob;
  g.err = mp.err;
  g.G = dims.G;
  g.nq = nq;
  const int Db = mp.depth_b, Ds = mp.depth_s, Dt = mp.depth_t;
  for (int l = 0; l < dims.L; ++l) {
    g.width_b[l] = mp.width_b[l];
    g.width_s[l] = mp.width[l];
    g.width_t[l] = mp.width_t[l];
    g.layer_base[l] = mp.layer_base[l];
    g.order[l] = mp.order[l];
    g.hstride[l] = layout::head_elems_arch(Db, mp.width_b[l], Ds, mp.width[l], Dt, mp.width_t[l]);
  }
  // hidden layers of the longest chain; the launches are stages 0..nst-1
  // (stage s < depth_b: the backbone, else branch layer s - depth_b of the
  // branches that have it), then the readout
  const int nst = mp.depth_b + std::max(mp.depth_s, mp.depth_t);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t hb = gemm_h_bytes(dims, mp.Hmax, nq);
  __nv_bfloat16* hbuf[2] = {reinterpret_cast<__nv_bfloat16*>(base),
                            reinterpret_cast<__nv_bfloat16*>(base + (nst >= 2 ? hb : 0))};
  g.part = reinterpret_cast<float*>(base + (nst >= 2 ? 2 : 1) * hb);
  CUtensorMap tq, th[2], thr;
  {
    const cuuint64_t dq[2] = {128, static_cast<cuuint64_t>(heads * R)};
    const cuuint64_t sq[1] = {256};
    const cuuint32_t bq[2] = {64, static_cast<cuuint32_t>(sh.NR)};
    NECTAR_TRY(make_tmap(&tq, Q, 2, dq, sq, bq, "queries (rows)"));
    for (int b = 0; b < 2; ++b) {
      const cuuint64_t dh[2] = {static_cast<cuuint64_t>(g.Hp), static_cast<cuuint64_t>(2 * heads * R)};
      const cuuint64_t shs[1] = {static_cast<cuuint64_t>(g.Hp) * 2};
      NECTAR_TRY(make_tmap(&th[b], hbuf[b], 2, dh, shs, bq, "hidden activations"));
    }
    // the readout reads the last hidden layer in its own, smaller row tiles
    const cuuint64_t dh[2] = {static_cast<cuuint64_t>(g.Hp), static_cast<cuuint64_t>(2 * heads * R)};
    const cuuint64_t shs[1] = {static_cast<cuuint64_t>(g.Hp) * 2};
    const cuuint32_t br[2] = {64, static_cast<cuuint32_t>(shr.NR)};
    // the target branch's last layer (stage depth_b + depth_t - 1) wrote its buffer
    NECTAR_TRY(make_tmap(&thr, hbuf[(mp.depth_b + mp.depth_t - 1) & 1], 2, dh, shs, br,
                         "hidden activations (readout)"));
  }
  for (int stage = 0; stage <= nst; ++stage) {
    g.stage = stage;
    g.readout = stage == nst;
    g.h_out = g.readout ? nullptr : hbuf[stage & 1];
    g.a_out = g.readout ? a : nullptr;
    g.A_out = g.readout ? A_out : nullptr;
    g.ws_loc = g.readout ? ws_loc : nullptr;
    g.out_bf16 = g.readout ? out_bf16 : nullptr;
    const GemmShape& ss = g.readout ? shr : sh;
    g.NR = ss.NR;
    g.rtiles = ss.rtiles;
    g.stages = ss.stages;
    g.tmem_cols = ss.tmem_cols;
    // per-layer weight offsets inside a head's block for this launch
    for (int l = 0; l < dims.L; ++l) {
      const int Hb = mp.width_b[l], Hs = mp.width[l], Ht = mp.width_t[l];
      const int64_t sb = layout::branch_base(Db, Hb, Ds, Hs, 0), tb = layout::branch_base(Db, Hb, Ds, Hs, 1);
      const int j = stage - Db;
      g.woff[l][0] = g.woff[l][1] = g.aux[l] = 0;
      if (g.readout) {
        g.woff[l][1] = tb + layout::branch_out_w_off(Db, Hb, Ht, Dt);
        g.aux[l] = sb + layout::branch_out_b_off(Db, Hb, Hs, Ds, 1);            // score c
      } else if (j < 0) {
        g.woff[l][0] = layout::backbone_w_off(Hb, stage);
      } else {
        if (j < Ds) g.woff[l][0] = sb + layout::branch_w_off(Db, Hb, Hs, j);
        if (j < Dt) g.woff[l][1] = tb + layout::branch_w_off(Db, Hb, Ht, j);
        if (j == Ds - 1) g.aux[l] = sb + layout::branch_out_w_off(Db, Hb, Hs, Ds);   // score w
      }
    }
    int64_t acc = 0;
    for (int li = 0; li < dims.L; ++li) {
      g.tile_start[li] = acc;
      const int l = g.order[li];
      const int j = stage - mp.depth_b;
      int mt;                                   // 128-unit tiles per head, as gemm_tile counts them
      if (g.readout) mt = 1;
      else if (j < 0) mt = (mp.width_b[l] + 127) / 128;
      else mt = (j < mp.depth_s ? (mp.width[l] + 127) / 128 : 0) + (j < mp.depth_t ? (mp.width_t[l] + 127) / 128 : 0);
      acc += static_cast<int64_t>(dims.Hkv) * mt * ss.rtiles;
    }
    g.tile_start[dims.L] = acc;
    g.ntiles = acc;
    if (acc == 0) continue;
    const int grid = static_cast<int>(acc < di.sms ? acc : di.sms);
    const CUtensorMap& tin = g.readout ? thr : (stage == 0 ? tq : th[(stage - 1) & 1]);
    cudaError_t e = launch_module_gemm(tq, tin, g, grid, ss.smem, st);
    if (e != cudaSuccess) return cuda_fail(e, "module GEMM kernel");
  }
  return NECTAR_OK;
}

nectar_status prepare_modules(const nectar_dims& dims, const nectar_module_set* mods, const nectar_bf16* Q,
                              int64_t nq, bool fuse, ModParams* p, CUtensorMap* tq, ModShape* sh) {
  Arch ar;
  NECTAR_TRY(arch_of(dims, mods, &ar));
  if (dims.G > 64) return fail(NECTAR_ERR_UNSUPPORTED, "G = %d > 64", dims.G);
  NECTAR_TRY(check_ptr(mods->weights, "mods->weights"));
  const int64_t need = arch_packed_elems(dims, ar);
  if (mods->weights_elems < need)
    return fail(NECTAR_ERR_INVALID_ARG, "weights_elems = %lld, the widths need %lld", (long long)mods->weights_elems,
                (long long)need);
  NECTAR_TRY(check_ptr(Q, "Q"));
  if (nq > 0x7fffffffLL) return fail(NECTAR_ERR_INVALID_ARG, "nq too large");
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");
  memset(p, 0, sizeof(*p));
  p->Hkv = dims.Hkv;
  p->G = dims.G;
  p->depth = ar.Ds;
  p->depth_b = ar.Db;
  p->depth_s = ar.Ds;
  p->depth_t = ar.Dt;
  p->general = ar.general;
  p->nq = nq;
  p->blob = reinterpret_cast<const __nv_bfloat16*>(mods->weights);
  p->Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p->err = di.err;
  int64_t base = 0;
  std::vector<int> cost(dims.L);
  for (int l = 0; l < dims.L; ++l) {
    p->width[l] = ar.ws[l];
    p->width_b[l] = arch_hb(ar, l);
    p->width_t[l] = ar.wt[l];
    p->layer_base[l] = base;
    base += static_cast<int64_t>(dims.Hkv) * arch_head_elems(ar, l);
    cost[l] = std::max(std::max(ar.ws[l], ar.wt[l]), arch_hb(ar, l));
  }
  // widest layers first: their CTAs run longest
  std::vector<int> ord(dims.L);
  for (int l = 0; l < dims.L; ++l) ord[l] = l;
  std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  for (int l = 0; l < dims.L; ++l) p->order[l] = static_cast<uint8_t>(ord[l]);
  const int Hmax = arch_hmax(dims, ar);
  p->Hmax = Hmax;
  if (use_gemm_path(dims, nq, ar.general, arch_hmax(dims, ar))) return NECTAR_OK;   // the layer-by-layer path needs no fused shape
  *sh = mod_shape(dims.G, nq, Hmax, fuse);
  if (sh->smem > 227 * 1024) return fail(NECTAR_ERR_UNSUPPORTED, "width %d needs too much shared memory", Hmax);
  if (sh->tmem_cols > 512)
    return fail(NECTAR_ERR_UNSUPPORTED, "width %d with G = %d needs more than 512 TMEM columns", Hmax, dims.G);
  // one CTA per net when every layer's net streams at least 256 KB of
  // weights: the two streams then run side by side on different SMs, and
  // the smaller CTAs even out the bytes per SM (measured with the module
  // CTAs first in the decode grid: Qwen3-1.7B, H = 512, 95.6 -> 89.8 us;
  // Llama-8B b = 1 at rho = 10 %, 185 -> 169 us)
  {
    int64_t min_net = INT64_MAX;
    for (int l = 0; l < dims.L; ++l)
      min_net = std::min(min_net, layout::net_elems(ar.ws[l], ar.Ds, 1) * 2);
    p->net_split = min_net >= (int64_t(256) << 10) ? 1 : 0;
    const char* ns = getenv("NECTAR_NET_SPLIT");   // =0 or =1 overrides the choice
    if (ns != nullptr && (ns[0] == '0' || ns[0] == '1')) p->net_split = ns[0] - '0';
  }
  p->N = sh->N;
  p->TPC = sh->TPC;
  p->nblk = sh->nblk;
  p->tmem_cols = sh->tmem_cols;
  p->stages = sh->stages;
  p->cps = sh->cps;
  // queries: [heads][G][nq][128]; box = 64 columns x TPC tokens x G heads x 1
  {
    const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
    const cuuint64_t dimsq[4] = {128, static_cast<cuuint64_t>(nq), static_cast<cuuint64_t>(dims.G),
                                 static_cast<cuuint64_t>(heads)};
    const cuuint64_t strq[3] = {256, static_cast<cuuint64_t>(nq) * 256, static_cast<cuuint64_t>(nq) * 256 * dims.G};
    const cuuint32_t boxq[4] = {64, static_cast<cuuint32_t>(sh->TPC), static_cast<cuuint32_t>(dims.G), 1};
    NECTAR_TRY(make_tmap(tq, Q, 4, dimsq, strq, boxq, "queries"));
  }
  return NECTAR_OK;
}

}  // namespace

extern "C" {

size_t nectar_module_workspace_size(nectar_dims dims, const nectar_module_set* mods, int64_t nq) {
  if (check_dims(dims) != NECTAR_OK || nq <= 0 || mods == nullptr) return 0;
  Arch ar;
  if (arch_of(dims, mods, &ar) != NECTAR_OK) return 0;
  if (!use_gemm_path(dims, nq, ar.general, arch_hmax(dims, ar))) return 0;
  return gemm_ws_bytes(dims, ar, nq);
}

nectar_status nectar_module_forward(nectar_dims dims, const nectar_module_set* mods, const nectar_bf16* Q, int64_t nq,
                                    float* a, float* A_theta, void* workspace, size_t workspace_bytes,
                                    nectar_stream_t stream) {
  NECTAR_TRY(check_dims(dims));
  if (nq < 0) return fail(NECTAR_ERR_INVALID_ARG, "nq must be >= 0");
  if (nq == 0) return NECTAR_OK;
  if (a == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "a is NULL");
  NECTAR_TRY(check_ptr(A_theta, "A_theta"));
  ModParams p;
  CUtensorMap tq;
  ModShape sh;
  NECTAR_TRY(prepare_modules(dims, mods, Q, nq, false, &p, &tq, &sh));
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (use_gemm_path(dims, nq, p.general, p.Hmax)) {
    const size_t need = nectar_module_workspace_size(dims, mods, nq);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(NECTAR_ERR_WORKSPACE, "module workspace of %zu bytes given, %zu needed",
                  workspace == nullptr ? size_t(0) : workspace_bytes, need);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
      return fail(NECTAR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    return run_module_gemm(dims, p, Q, nq, a, A_theta, nullptr, workspace, st);
  }
  p.a_out = a;
  p.A_out = A_theta;
  const int units = (p.net_split ? 2 : 1) * dims.L * dims.Hkv * sh.nblk;
  cudaError_t e = launch_module(tq, p, units, sh.smem, false, st);
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "module kernel");
}

size_t nectar_decode_workspace_size(nectar_dims dims, const nectar_module_set* mods, int64_t nq) {
  if (check_dims(dims) != NECTAR_OK || nq <= 0 || mods == nullptr) return 0;
  Arch ar;
  if (arch_of(dims, mods, &ar) != NECTAR_OK) return 0;
  const int64_t rows = static_cast<int64_t>(dims.L) * dims.Hkv * dims.G * nq;
  const size_t loc = align256(static_cast<size_t>(rows) * (kD + 2) * sizeof(float));
  if (use_gemm_path(dims, nq, ar.general, arch_hmax(dims, ar))) return loc + gemm_ws_bytes(dims, ar, nq);
  return decode_ws_a_bytes(rows) + loc;
}

size_t nectar_decode_layer_out_workspace_size(nectar_dims dims, const nectar_module_set* mods, int64_t nq) {
  const size_t base = nectar_decode_workspace_size(dims, mods, nq);
  Arch ar;
  if (base == 0 || arch_of(dims, mods, &ar) != NECTAR_OK || use_gemm_path(dims, nq, ar.general, arch_hmax(dims, ar))) return base;
  // the one-launch path keeps A_theta in fp32 until the merge
  const int64_t rows = static_cast<int64_t>(dims.L) * dims.Hkv * dims.G * nq;
  return base + align256(static_cast<size_t>(rows) * kD * sizeof(float));
}

}  // extern "C"

namespace {

// Calls with at most this many (layer, KV head) pairs take the cluster
// decode (decode_cluster.cu) when it applies; more heads keep the one-launch
// kernel with one CTA per (l, h) (or per net), which then fills the GPU.
#ifndef NECTAR_CLUSTER_MAX_HEADS
#define NECTAR_CLUSTER_MAX_HEADS 32
#endif

// Resident clusters of a cluster-decode plan on the current device, cached.
int cached_max_active(const ClusterShape& sh, int G) {
  struct Key {
    int dev, cluster, npc, rg2;
    size_t smem;
    int n;
  };
  static std::mutex mu;
  static std::vector<Key> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int rg2 = G <= 2 ? 1 : 0;
  std::lock_guard<std::mutex> lk(mu);
  for (const Key& k : cache)
    if (k.dev == dev && k.cluster == sh.cluster && k.npc == sh.npc && k.rg2 == rg2 && k.smem == sh.smem) return k.n;
  const int n = cluster_max_active(sh, G);
  cache.push_back(Key{dev, sh.cluster, sh.npc, rg2, sh.smem, n});
  return n;
}

// The cluster plan the decode takes; returns its size (8 or 16), or 0 for
// the one-launch kernel.  NECTAR_DECODE_CLUSTER=0 never takes the cluster
// decode, =8 or =16 takes that size whenever it applies (with
// NECTAR_DECODE_CLUSTER_NETS=1 or 2 nets per CTA for size 8; default 1);
// unset: with at most NECTAR_CLUSTER_MAX_HEADS (l, h) pairs, the first plan
// that applies of: 8 CTAs holding one net each (4 slices per net), 8 CTAs
// holding both nets (8 slices), 16 CTAs holding one net each.  On one
// Qwen3-1.7B layer in a graph: 17.4 us with both nets per CTA against
// 27.4 with 16 CTAs, whose non-portable clusters do not all fit at once.
int cluster_decode_size(const nectar_dims& dims, int64_t nq, const Arch& ar, int Hmax, ClusterShape* out) {
  if (ar.general || static_cast<int64_t>(dims.G) * nq > 64) return 0;
  const char* env = getenv("NECTAR_DECODE_CLUSTER");
  const int mode = (env != nullptr && env[0] != 0) ? atoi(env) : -1;
  if (mode == 0) return 0;
  const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
  if (mode == 8 || mode == 16) {
    const char* envn = getenv("NECTAR_DECODE_CLUSTER_NETS");
    const int npc = mode == 16 ? 1 : ((envn != nullptr && envn[0] == '2') ? 2 : 1);
    *out = cluster_shape(mode, npc, dims.G, nq, Hmax, ar.Ds);
    return out->ok && cached_max_active(*out, dims.G) > 0 ? mode : 0;
  }
  if (heads > NECTAR_CLUSTER_MAX_HEADS) return 0;
  const int plans[3][2] = {{8, 1}, {8, 2}, {16, 1}};
  for (const auto& pl : plans) {
    const ClusterShape sh = cluster_shape(pl[0], pl[1], dims.G, nq, Hmax, ar.Ds);
    if (sh.ok && cached_max_active(sh, dims.G) > 0) {
      *out = sh;
      return pl[0];
    }
  }
  return 0;
}

// The decode, into out (fp32, per KV head) or out_bf16 (bf16, layer layout).
nectar_status decode_impl(nectar_dims dims, const nectar_module_set* mods, const nectar_bf16* Q, int64_t nq,
                          const int32_t* q_seq, const int32_t* q_pos, const nectar_bf16* Kloc,
                          const nectar_bf16* Vloc, int32_t B, int32_t T_max, const int32_t* local_len, float scale,
                          float* out, __nv_bfloat16* out_bf16, void* workspace, size_t workspace_bytes,
                          nectar_stream_t stream) {
  NECTAR_TRY(check_dims(dims));
  if (nq < 0) return fail(NECTAR_ERR_INVALID_ARG, "nq must be >= 0");
  if (nq == 0) return NECTAR_OK;
  if (!(scale == scale)) return fail(NECTAR_ERR_INVALID_ARG, "scale is NaN");
  NECTAR_TRY(check_ptr(out != nullptr ? static_cast<const void*>(out) : static_cast<const void*>(out_bf16), "out"));
  NECTAR_TRY(check_local(q_seq, q_pos, Kloc, Vloc, B, T_max, local_len));
  Arch ar;
  NECTAR_TRY(arch_of(dims, mods, &ar));
  const size_t need = out != nullptr ? nectar_decode_workspace_size(dims, mods, nq)
                                     : nectar_decode_layer_out_workspace_size(dims, mods, nq);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(NECTAR_ERR_WORKSPACE, "decode workspace of %zu bytes given, %zu needed",
                workspace == nullptr ? size_t(0) : workspace_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return fail(NECTAR_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  ModParams p;
  CUtensorMap tq;
  ModShape sh;
  NECTAR_TRY(prepare_modules(dims, mods, Q, nq, true, &p, &tq, &sh));
  const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
  const int64_t rows = heads * dims.G * nq;
  const bool gemm = use_gemm_path(dims, nq, ar.general, arch_hmax(dims, ar));
  if (heads * nq + (gemm ? 0 : (p.net_split ? 2 : 1) * static_cast<int64_t>(dims.L) * dims.Hkv * sh.nblk) >
      0x7fffffffLL)
    return fail(NECTAR_ERR_UNSUPPORTED, "too many CTAs for one launch");
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.Kloc = reinterpret_cast<const __nv_bfloat16*>(Kloc);
  p.Vloc = reinterpret_cast<const __nv_bfloat16*>(Vloc);
  p.local_len = local_len;
  p.B = B;
  p.T = T_max;
  p.qmul = scale * kLog2e;
  p.out = out;
  p.out_bf16 = out_bf16;
  p.n_local = heads * nq;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  if (gemm) {
    // local states first, then the layer-by-layer module whose readout merges
    p.ws_loc = reinterpret_cast<float*>(base);
    if (use_local_tc(dims, nq, B, T_max)) {
      NECTAR_TRY(run_local_many(dims, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, p.ws_loc,
                                nullptr, nullptr, nullptr, st));
    } else {
      cudaError_t e = launch_local_state(p, st);
      if (e != cudaSuccess) return cuda_fail(e, "local attention kernel");
    }
    return run_module_gemm(dims, p, Q, nq, nullptr, out, p.ws_loc,
                           base + align256(static_cast<size_t>(rows) * (kD + 2) * sizeof(float)), st, out_bf16);
  }
  ClusterShape cs{};
  if (const int csize = cluster_decode_size(dims, nq, ar, p.Hmax, &cs)) {
    ClusterParams c;
    memset(&c, 0, sizeof(c));
    c.Hkv = dims.Hkv;
    c.G = dims.G;
    c.depth = ar.Ds;
    c.nq = nq;
    c.N = cs.N;
    c.Hmax = p.Hmax;
    c.stages = cs.stages;
    c.tmem_cols = cs.tmem_cols;
    c.nb = cs.nb;
    c.blob = p.blob;
    c.Q = p.Q;
    c.q_seq = q_seq;
    c.q_pos = q_pos;
    c.Kloc = p.Kloc;
    c.Vloc = p.Vloc;
    c.local_len = local_len;
    c.B = B;
    c.T = T_max;
    c.qmul = p.qmul;
    c.out = out;
    c.out_bf16 = out_bf16;
    c.err = p.err;
    for (int l = 0; l < dims.L; ++l) {
      c.width[l] = p.width[l];
      c.layer_base[l] = p.layer_base[l];
      c.order[l] = p.order[l];
    }
    cudaError_t e = launch_decode_cluster(c, cs, static_cast<int>(heads), st);
    return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "cluster decode kernel");
  }
  p.a_out = reinterpret_cast<float*>(base);
  p.ws_loc = reinterpret_cast<float*>(base + decode_ws_a_bytes(rows));
  // A_theta lands in out and is merged in place; for the bf16 layer output it
  // is kept in fp32 after the local states
  p.A_out = out != nullptr ? out
                           : reinterpret_cast<float*>(base + decode_ws_a_bytes(rows) +
                                                      align256(static_cast<size_t>(rows) * (kD + 2) * sizeof(float)));
  const int units = (p.net_split ? 2 : 1) * dims.L * dims.Hkv * sh.nblk;
  // Module CTAs first in the grid, local CTAs after them.  With the local
  // CTAs first the block scheduler was seen to place one CTA per SM until
  // the first ones ended (a per-CTA timeline of the Qwen3-1.7B decode: 148
  // local CTAs resident for the first 16 us, then the module CTAs), which
  // left the SMs' second slots and most of HBM idle; module CTAs first:
  // 102.5 -> 96.0 us in the bench step.  NECTAR_DECODE_ORDER=local puts the
  // local CTAs first.
  {
    const char* ord = getenv("NECTAR_DECODE_ORDER");
    p.module_first = (ord != nullptr && ord[0] == 'l') ? 0 : 1;
  }
  cudaError_t e = launch_decode(tq, p, units, sh.smem, st);
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "decode kernels");
}

}  // namespace

extern "C" {

nectar_status nectar_decode(nectar_dims dims, const nectar_module_set* mods, const nectar_bf16* Q, int64_t nq,
                            const int32_t* q_seq, const int32_t* q_pos, const nectar_bf16* Kloc,
                            const nectar_bf16* Vloc, int32_t B, int32_t T_max, const int32_t* local_len,
                            float scale, float* out, void* workspace, size_t workspace_bytes,
                            nectar_stream_t stream) {
  if (out == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "out is NULL");
  return decode_impl(dims, mods, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, out, nullptr,
                     workspace, workspace_bytes, stream);
}

nectar_status nectar_decode_layer_out(nectar_dims dims, const nectar_module_set* mods, const nectar_bf16* Q,
                                      int64_t nq, const int32_t* q_seq, const int32_t* q_pos,
                                      const nectar_bf16* Kloc, const nectar_bf16* Vloc, int32_t B, int32_t T_max,
                                      const int32_t* local_len, float scale, nectar_bf16* out, void* workspace,
                                      size_t workspace_bytes, nectar_stream_t stream) {
  if (out == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "out is NULL");
  return decode_impl(dims, mods, Q, nq, q_seq, q_pos, Kloc, Vloc, B, T_max, local_len, scale, nullptr,
                     reinterpret_cast<__nv_bfloat16*>(out), workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// next rows: Quadrature module, fitting metrics
// ---------------------------------------------------------------------------
nectar_status nectar_quadrature_init(nectar_dims dims, const nectar_bf16* K, const nectar_bf16* V, int64_t n,
                                     int64_t p, nectar_bf16* W, nectar_bf16* Z, nectar_stream_t stream) {
  NECTAR_TRY(check_dims(dims));
  if (p < 1 || p > n) return fail(NECTAR_ERR_INVALID_ARG, "p = %lld must be in [1, n = %lld]", (long long)p,
                                  (long long)n);
  NECTAR_TRY(check_ptr(K, "K"));
  NECTAR_TRY(check_ptr(V, "V"));
  NECTAR_TRY(check_ptr(W, "W"));
  NECTAR_TRY(check_ptr(Z, "Z"));
  const DeviceInfo di = device_info();
  if (di.sms == 0) return fail(NECTAR_ERR_CUDA, "no CUDA device");
  const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
  cudaError_t e = launch_quadrature_init(reinterpret_cast<const __nv_bfloat16*>(K),
                                         reinterpret_cast<const __nv_bfloat16*>(V),
                                         reinterpret_cast<__nv_bfloat16*>(W), reinterpret_cast<__nv_bfloat16*>(Z),
                                         heads, n, p, di.sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "quadrature init kernel");
}

size_t nectar_quadrature_workspace_size(nectar_dims dims, int64_t p, int64_t nq) {
  return nectar_cache_attn_workspace_size(dims, p, nq);
}

nectar_status nectar_quadrature_forward(nectar_dims dims, const nectar_bf16* W, const nectar_bf16* Z, int64_t p,
                                        const nectar_bf16* Q, int64_t nq, float scale, float* a, float* A_theta,
                                        void* workspace, size_t workspace_bytes, nectar_stream_t stream) {
  // the exact attention of Eq. (3.1) over the p learned rows
  return nectar_cache_attn_lse(dims, W, Z, p, Q, nq, scale, a, A_theta, workspace, workspace_bytes, stream);
}

nectar_status nectar_fit_metrics(nectar_dims dims, int64_t nq, const float* alpha, const float* A, const float* a,
                                 const float* A_theta, const nectar_bf16* Q, double* metrics,
                                 nectar_stream_t stream) {
  NECTAR_TRY(check_dims(dims));
  if (nq < 0) return fail(NECTAR_ERR_INVALID_ARG, "nq must be >= 0");
  if (alpha == nullptr || a == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "alpha / a is NULL");
  NECTAR_TRY(check_ptr(A, "A"));
  NECTAR_TRY(check_ptr(A_theta, "A_theta"));
  NECTAR_TRY(check_ptr(Q, "Q"));
  if (metrics == nullptr) return fail(NECTAR_ERR_INVALID_ARG, "metrics is NULL");
  const int64_t heads = static_cast<int64_t>(dims.L) * dims.Hkv;
  if (heads > 0x7fffffffLL) return fail(NECTAR_ERR_UNSUPPORTED, "too many heads");
  cudaError_t e = launch_fit_metrics(alpha, A, a, A_theta, reinterpret_cast<const __nv_bfloat16*>(Q), heads,
                                     static_cast<int64_t>(dims.G) * nq, metrics,
                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NECTAR_OK : cuda_fail(e, "fit metrics kernel");
}

}  // extern "C"
