// C ABI entry points: argument checks, workspace layout and launch order of the POET-X layer.
//
// Forward ("POET-X" blog §第一斧/§第五斧, permutations as index maps §第二斧, batched blocks §第三斧):
//   A = X[:, perm_r];  A'_j = A_j G_R^j;  B = A' W0';  C_j = B_j G_P^j;  Y[:, perm_p] = C.
// Backward (exact gradient of the forward):
//   dC = dY[:, perm_p];  dB_j = dC_j G_P^jT;  dG_P^j = B_j^T dC_j;  dA' = dB W0'^T;
//   dA_j = dA'_j G_R^jT;  dG_R^j = A_j^T dA'_j;  dX[:, perm_r] = dA;  dq = CNP chain rule.
#include "internal.h"
#include "gemm.h"

#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

namespace poetx {

// ------------------------------------------------------------------ error text
static thread_local std::string g_last_error;

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

// ------------------------------------------------------------------ tracing
namespace {
struct TraceRec {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool;
std::vector<std::string> g_trace_only;   // empty: every launch

bool traced(const char* name) {
  if (g_trace_only.empty()) return true;
  for (const auto& n : g_trace_only)
    if (n == name) return true;
  return false;
}

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

int trace_begin(const char* name, cudaStream_t s) {
  if (!g_trace_on) return -1;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (!traced(name)) return -1;
  TraceRec r{name, pool_event(), pool_event()};
  cudaEventRecord(r.start, s);
  g_trace.push_back(r);
  return (int)g_trace.size() - 1;
}

void trace_end(int slot, cudaStream_t s) {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (slot < (int)g_trace.size()) cudaEventRecord(g_trace[slot].stop, s);
}

// ------------------------------------------------------------------ programmatic launch
bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("POETX_PDL");
    on = (v && v[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

void set_pdl_attr(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
}

// ------------------------------------------------------------------ device error word
__device__ int g_device_error;

int* device_error_word() {
  static int* p = nullptr;
  if (!p) cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_device_error);
  return p;
}

}  // namespace poetx

using namespace poetx;

namespace {

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int elem_size(int32_t dt) { return dt == POETX_BF16 ? 2 : 4; }

poetx_status fail(poetx_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_error("%s", buf);
  return st;
}

poetx_status cuda_fail(cudaError_t e, const char* where) {
  return fail(POETX_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define CHECK_CUDA(expr, where)                 \
  do {                                          \
    cudaError_t e_ = (expr);                    \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

// The current device must be a compute-capability 10.x part (B200 = sm_100).
poetx_status check_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static int cached_dev = -1, cached_major = -1;
  if (dev != cached_dev) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    cached_dev = dev;
    cached_major = major;
  }
  if (cached_major != 10)
    return fail(POETX_ERR_UNSUPPORTED, "device %d has compute capability %d.x; sm_100 required",
                dev, cached_major);
  return POETX_OK;
}

poetx_status check_layer(const poetx_layer* L, bool need_lp) {
  if (!L) return fail(POETX_ERR_INVALID_ARG, "layer is NULL");
  if (L->dtype != POETX_F32 && L->dtype != POETX_BF16)
    return fail(POETX_ERR_DTYPE, "unknown layer dtype %d", L->dtype);
  const int32_t storage = L->flags & ~POETX_LAYER_FUSED_W0_P;
  if (storage != 0 && storage != POETX_LAYER_W0M_I8 &&
      storage != (POETX_LAYER_W0M_I8 | POETX_LAYER_W0M_STAGED))
    return fail(POETX_ERR_INVALID_ARG, "unknown layer flags %d", L->flags);
  if (L->flags & POETX_LAYER_W0M_I8) {
    if (L->dtype != POETX_BF16)
      return fail(POETX_ERR_DTYPE, "an int8 W0' needs a BF16 layer");
    if (!L->w0m_scale) return fail(POETX_ERR_INVALID_ARG, "int8 W0' without w0m_scale");
    if (!aligned16(L->w0m_scale)) return fail(POETX_ERR_ALIGN, "w0m_scale not 16-byte aligned");
    if (L->m % 16 || L->n % 16)
      return fail(POETX_ERR_SHAPE, "an int8 W0' needs m and n multiples of 16");
  }
  if (L->m <= 0 || L->n <= 0 || L->b < 2)
    return fail(POETX_ERR_SHAPE, "bad layer shape m=%lld n=%lld b=%lld", (long long)L->m,
                (long long)L->n, (long long)L->b);
  if (L->m % L->b || L->n % L->b)
    return fail(POETX_ERR_SHAPE, "b=%lld must divide m=%lld and n=%lld", (long long)L->b,
                (long long)L->m, (long long)L->n);
  if (L->b > 1024) return fail(POETX_ERR_SHAPE, "b=%lld exceeds 1024", (long long)L->b);
  if (L->dtype == POETX_BF16 && (L->m % 8 || L->n % 8 || L->b % 8))
    return fail(POETX_ERR_SHAPE, "bf16 layers need m, n, b multiples of 8");
  if (!L->w0m || !L->perm_r || !L->perm_p || !L->g_r || !L->g_p)
    return fail(POETX_ERR_INVALID_ARG, "layer has a NULL w0m/perm/g pointer");
  if (need_lp && L->dtype == POETX_BF16 && (!L->g_r_lp || !L->g_p_lp))
    return fail(POETX_ERR_INVALID_ARG, "bf16 layer needs g_r_lp and g_p_lp");
  const void* ptrs[] = {L->w0m, L->perm_r, L->perm_p, L->g_r, L->g_p, L->g_r_lp, L->g_p_lp,
                        L->q_r, L->q_p};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(POETX_ERR_ALIGN, "layer pointer %p not 16-byte aligned", p);
  return POETX_OK;
}

poetx_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return POETX_OK;
  if (!ws || have < need)
    return fail(POETX_ERR_WORKSPACE, "workspace %zu bytes < %zu required", ws ? have : 0, need);
  if (!aligned16(ws)) return fail(POETX_ERR_ALIGN, "workspace not 16-byte aligned");
  return POETX_OK;
}

size_t xq_deq_bytes(const poetx_layer* L, int64_t T, bool fwd_product, bool bwd_product);

// ---- workspace layouts (each buffer 256-byte aligned)
struct FwdWs {
  void *A, *A1, *B, *C;
  int32_t* inv;
  void* Wd;   // dequantised W0' (int8 layers whose product shape is not fused)
};
size_t fwd_layout(const poetx_layer* L, int64_t T, void* base, FwdWs* o) {
  Arena a(base, SIZE_MAX);
  const size_t e = (size_t)elem_size(L->dtype);
  FwdWs w;
  w.A = a.take(T * L->m * e);
  w.A1 = a.take(T * L->m * e);
  w.C = a.take(T * L->n * e);
  w.B = a.take(T * L->n * e);  // used only when the caller does not keep B
  w.inv = static_cast<int32_t*>(a.take(L->n * 4));
  const size_t wd = xq_deq_bytes(L, T, true, false);
  w.Wd = wd ? a.take(wd) : nullptr;
  if (o) *o = w;
  return a.used;
}

struct BwdWs {
  void *dC, *dB, *dA1, *A, *dA;
  void* B;               // recomputed forward product when the caller did not keep it
  float* dG;             // [m/b + n/b][b][b]: the R blocks, then the P blocks
  void* chain;
  void *part_r, *part_p;  // split-K partial sums of dG_R, dG_P (separate launches)
  void* part_rp;          // split-K partial sums of the one launch over both (same region)
  int32_t* inv;
  void* Wd;               // dequantised W0' (int8 layers whose product shapes are not fused)
};
size_t bwd_layout(const poetx_layer* L, int64_t T, void* base, BwdWs* o) {
  Arena a(base, SIZE_MAX);
  const size_t e = (size_t)elem_size(L->dtype);
  BwdWs w;
  w.dC = a.take(T * L->n * e);
  w.dB = a.take(T * L->n * e);
  w.dA1 = a.take(T * L->m * e);
  w.A = a.take(T * L->m * e);
  w.dA = a.take(T * L->m * e);
  w.B = a.take(T * L->n * e);
  w.dG = static_cast<float*>(a.take((size_t)((L->m + L->n) * L->b) * sizeof(float)));
  const DT t = L->dtype == POETX_BF16 ? DT::BF16 : DT::F32;
  w.chain = a.take(gemm_dq_ws_bytes(t, L->m / L->b + L->n / L->b, L->b));
  const size_t pr = block_grad_ws_bytes(t, L->m, L->b, T);
  const size_t pp = block_grad_ws_bytes(t, L->n, L->b, T);
  const size_t prp = block_grad2_ws_bytes(t, L->m, L->n, L->b, T);
  uint8_t* parts = static_cast<uint8_t*>(a.take(std::max(prp, pr + pp)));
  w.part_r = parts;
  w.part_p = parts ? parts + pr : nullptr;
  w.part_rp = parts;
  w.inv = static_cast<int32_t*>(a.take(L->m * 4));
  const size_t wd = xq_deq_bytes(L, T, true, true);
  w.Wd = wd ? a.take(wd) : nullptr;
  if (o) *o = w;
  return a.used;
}

struct MergeWs {
  void *N1, *M;
  int32_t *pr_new, *pp_new, *inv, *rho_r, *rho_p;
};
size_t merge_layout(const poetx_layer* L, void* base, MergeWs* o) {
  Arena a(base, SIZE_MAX);
  const size_t e = (size_t)elem_size(L->dtype);
  MergeWs w;
  w.N1 = a.take(L->m * L->n * e);
  w.M = a.take(L->m * L->n * e);
  w.pr_new = static_cast<int32_t*>(a.take(L->m * 4));
  w.pp_new = static_cast<int32_t*>(a.take(L->n * 4));
  w.inv = static_cast<int32_t*>(a.take(std::max(L->m, L->n) * 4));
  w.rho_r = static_cast<int32_t*>(a.take(L->m * 4));
  w.rho_p = static_cast<int32_t*>(a.take(L->n * 4));
  if (o) *o = w;
  return a.used;
}

DT dt_of(int32_t d) { return d == POETX_BF16 ? DT::BF16 : DT::F32; }

bool w0m_i8(const poetx_layer* L) { return (L->flags & POETX_LAYER_W0M_I8) != 0; }
bool w0m_staged(const poetx_layer* L) { return (L->flags & POETX_LAYER_W0M_STAGED) != 0; }

// bf16 scratch for an explicit dequantisation of an int8 W0': staged layers, and product shapes
// the in-kernel dequantisation does not cover
size_t xq_deq_bytes(const poetx_layer* L, int64_t T, bool fwd_product, bool bwd_product) {
  if (!w0m_i8(L)) return 0;
  const bool need = w0m_staged(L) || (fwd_product && !dense_i8_fused(T, L->n)) ||
                    (bwd_product && !dense_i8_fused(T, L->m));
  return need ? (size_t)(L->m * L->n) * 2 : 0;
}

// B = A W0' (trans = false, A [T, m]) or dA' = dB W0'^T (trans = true, dB [T, n])
cudaError_t w0_product(const poetx_layer* L, const void* A, void* C, int64_t T, bool trans,
                       void* deq_ws, cudaStream_t s) {
  const int64_t N = trans ? L->m : L->n, K = trans ? L->n : L->m;
  if (w0m_i8(L) && w0m_staged(L)) {
    if (!deq_ws) return cudaErrorInvalidValue;
    auto* W = static_cast<__nv_bfloat16*>(deq_ws);
    cudaError_t e = dequantize_cols_i8(static_cast<const int8_t*>(L->w0m), L->w0m_scale, L->m,
                                       L->n, W, s);
    if (e != cudaSuccess) return e;
    return gemm_dense(DT::BF16, A, W, C, T, N, K, trans, s);
  }
  if (w0m_i8(L))
    return gemm_dense_i8(A, static_cast<const int8_t*>(L->w0m), L->w0m_scale, C, T, N, K, trans,
                         deq_ws, s);
  return gemm_dense(dt_of(L->dtype), A, L->w0m, C, T, N, K, trans, s);
}

}  // namespace

extern "C" {

int32_t poetx_abi_version(void) { return 2; }

const char* poetx_status_string(int32_t st) {
  switch (st) {
    case POETX_OK: return "ok";
    case POETX_ERR_INVALID_ARG: return "invalid argument";
    case POETX_ERR_SHAPE: return "unsupported shape";
    case POETX_ERR_ALIGN: return "misaligned pointer";
    case POETX_ERR_DTYPE: return "unsupported dtype";
    case POETX_ERR_BAD_INDEX: return "not a permutation";
    case POETX_ERR_CUDA: return "CUDA error";
    case POETX_ERR_UNSUPPORTED: return "unsupported device";
    case POETX_ERR_WORKSPACE: return "workspace too small";
    case POETX_ERR_TIMEOUT: return "kernel wait timed out";
    default: return "unknown status";
  }
}

const char* poetx_last_error_message(void) { return g_last_error.c_str(); }

poetx_status poetx_trace_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_on = on != 0;
  return POETX_OK;
}

poetx_status poetx_trace_select(const char* names) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_only.clear();
  if (!names) return POETX_OK;
  std::string cur;
  for (const char* p = names;; ++p) {
    if (*p == ',' || *p == 0) {
      if (!cur.empty()) g_trace_only.push_back(cur);
      cur.clear();
      if (*p == 0) break;
    } else {
      cur.push_back(*p);
    }
  }
  return POETX_OK;
}

int64_t poetx_trace_read(char* buf, size_t len) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  size_t off = 0;
  if (buf && len) buf[0] = 0;
  for (auto& r : g_trace) {
    float ms = -1.f;
    if (cudaEventSynchronize(r.stop) == cudaSuccess) cudaEventElapsedTime(&ms, r.start, r.stop);
    if (buf && off + 1 < len) {
      int w = snprintf(buf + off, len - off, "%s %.6f\n", r.name, ms);
      if (w > 0) off = std::min(len - 1, off + (size_t)w);
    }
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  const int64_t count = (int64_t)g_trace.size();
  g_trace.clear();
  return count;
}

poetx_status poetx_device_status(void* stream) {
  poetx_status st = check_device();
  if (st != POETX_OK) return st;
  int* w = device_error_word();
  if (!w) return fail(POETX_ERR_CUDA, "device error word unavailable");
  int host = 0;
  CHECK_CUDA(cudaMemcpyAsync(&host, w, sizeof(int), cudaMemcpyDeviceToHost, as_stream(stream)),
             "read error word");
  CHECK_CUDA(cudaStreamSynchronize(as_stream(stream)), "sync");
  if (host != 0) {
    int zero = 0;
    CHECK_CUDA(cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice), "clear error word");
    return fail(POETX_ERR_TIMEOUT, "device error code %d", host);
  }
  return POETX_OK;
}

// ------------------------------------------------------------------ CNP
size_t poetx_cnp_workspace_bytes(int64_t nblocks, int64_t b) {
  if (nblocks <= 0 || b < 2) return 0;
  return gemm_cnp_ws_bytes(nblocks, b);
}

poetx_status poetx_cnp_build(const float* q, int64_t nblocks, int64_t b, float* g, void* g_lp,
                             int32_t lp_dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (nblocks < 0 || b < 2) return fail(POETX_ERR_INVALID_ARG, "nblocks < 0 or b < 2");
  if (b > 1024) return fail(POETX_ERR_SHAPE, "b=%lld exceeds 1024", (long long)b);
  if (nblocks == 0) return POETX_OK;
  if (!q) return fail(POETX_ERR_INVALID_ARG, "q is NULL");
  if (!g && !g_lp) return fail(POETX_ERR_INVALID_ARG, "both outputs are NULL");
  if (g_lp && lp_dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "g_lp must be BF16");
  if (!aligned16(q) || (g && !aligned16(g)) || (g_lp && !aligned16(g_lp)))
    return fail(POETX_ERR_ALIGN, "cnp pointers must be 16-byte aligned");
  poetx_status st = check_ws(workspace, ws_bytes, poetx_cnp_workspace_bytes(nblocks, b));
  if (st != POETX_OK) return st;
  if ((st = check_device()) != POETX_OK) return st;
  CHECK_CUDA(gemm_cnp_build(q, nblocks, b, g, static_cast<__nv_bfloat16*>(g_lp), workspace,
                            as_stream(stream)),
             "cnp_build");
  return POETX_OK;
}

size_t poetx_layer_cnp_workspace_bytes(const poetx_layer* L) {
  if (!L || L->b < 2 || L->m <= 0 || L->n <= 0) return 0;
  return gemm_cnp_ws_bytes(L->m / L->b + L->n / L->b, L->b);
}

poetx_status poetx_layer_cnp_build(const poetx_layer* L, void* workspace, size_t ws_bytes,
                                   void* stream) {
  poetx_status st = check_layer(L, true);
  if (st != POETX_OK) return st;
  if (!L->q_r || !L->q_p) return fail(POETX_ERR_INVALID_ARG, "layer has no q");
  if ((st = check_ws(workspace, ws_bytes, poetx_layer_cnp_workspace_bytes(L))) != POETX_OK)
    return st;
  if ((st = check_device()) != POETX_OK) return st;
  BlockRuns r;
  const bool lp = L->dtype == POETX_BF16;
  r.q[0] = L->q_r; r.g[0] = L->g_r; r.nb[0] = (int)(L->m / L->b);
  r.q[1] = L->q_p; r.g[1] = L->g_p; r.nb[1] = (int)(L->n / L->b);
  if (lp) {
    r.g_lp[0] = static_cast<__nv_bfloat16*>(L->g_r_lp);
    r.g_lp[1] = static_cast<__nv_bfloat16*>(L->g_p_lp);
  }
  CHECK_CUDA(gemm_cnp_build_runs(r, L->b, workspace, as_stream(stream)), "layer_cnp_build");
  return POETX_OK;
}

// Layers whose blocks one launch sequence covers (two runs each: R, then P)
constexpr int kLayersPerBatch = kMaxRuns / 2;

size_t poetx_layers_cnp_workspace_bytes(const poetx_layer* const* layers, int32_t nlayers) {
  if (!layers || nlayers <= 0) return 0;
  size_t need = 0;
  for (int32_t i0 = 0; i0 < nlayers; i0 += kLayersPerBatch) {
    int64_t nb = 0, b = 0;
    for (int32_t i = i0; i < nlayers && i < i0 + kLayersPerBatch; ++i) {
      const poetx_layer* L = layers[i];
      if (!L || L->b < 2 || L->m <= 0 || L->n <= 0) return 0;
      nb += L->m / L->b + L->n / L->b;
      b = L->b;
    }
    need = std::max(need, gemm_cnp_ws_bytes(nb, b));
  }
  return need;
}

poetx_status poetx_layers_cnp_build(const poetx_layer* const* layers, int32_t nlayers,
                                    void* workspace, size_t ws_bytes, void* stream) {
  if (nlayers < 0) return fail(POETX_ERR_INVALID_ARG, "nlayers < 0");
  if (nlayers == 0) return POETX_OK;
  if (!layers) return fail(POETX_ERR_INVALID_ARG, "layers is NULL");
  for (int32_t i = 0; i < nlayers; ++i) {
    const poetx_layer* L = layers[i];
    poetx_status st = check_layer(L, true);
    if (st != POETX_OK) return st;
    if (!L->q_r || !L->q_p) return fail(POETX_ERR_INVALID_ARG, "layer %d has no q", (int)i);
    if (L->b != layers[0]->b)
      return fail(POETX_ERR_SHAPE, "layer %d has b=%lld, layer 0 b=%lld", (int)i, (long long)L->b,
                  (long long)layers[0]->b);
    if (L->dtype != layers[0]->dtype)
      return fail(POETX_ERR_DTYPE, "layer %d has another dtype than layer 0", (int)i);
  }
  poetx_status st = check_ws(workspace, ws_bytes, poetx_layers_cnp_workspace_bytes(layers, nlayers));
  if (st != POETX_OK) return st;
  if ((st = check_device()) != POETX_OK) return st;
  const int64_t b = layers[0]->b;
  const bool lp = layers[0]->dtype == POETX_BF16;
  for (int32_t i0 = 0; i0 < nlayers; i0 += kLayersPerBatch) {
    BlockRuns r;
    for (int32_t i = i0; i < nlayers && i < i0 + kLayersPerBatch; ++i) {
      const poetx_layer* L = layers[i];
      const int k = 2 * (i - i0);
      r.q[k] = L->q_r; r.g[k] = L->g_r; r.nb[k] = (int)(L->m / b);
      r.q[k + 1] = L->q_p; r.g[k + 1] = L->g_p; r.nb[k + 1] = (int)(L->n / b);
      if (lp) {
        r.g_lp[k] = static_cast<__nv_bfloat16*>(L->g_r_lp);
        r.g_lp[k + 1] = static_cast<__nv_bfloat16*>(L->g_p_lp);
      }
    }
    CHECK_CUDA(gemm_cnp_build_runs(r, b, workspace, as_stream(stream)), "layers_cnp_build");
  }
  return POETX_OK;
}

// ------------------------------------------------------------------ forward
size_t poetx_fwd_workspace_bytes(const poetx_layer* L, int64_t T) {
  if (!L || T < 0 || L->m <= 0 || L->n <= 0) return 0;
  return fwd_layout(L, T, nullptr, nullptr);
}

}  // extern "C"

namespace {
poetx_status linear_fwd_impl(const poetx_layer* L, const void* x, int64_t T, void* y,
                             void* saved_b, void* saved_a, void* workspace, size_t ws_bytes,
                             void* stream) {
  poetx_status st = check_layer(L, true);
  if (st != POETX_OK) return st;
  if (T < 0) return fail(POETX_ERR_SHAPE, "T < 0");
  if (T == 0) return POETX_OK;
  if (!x || !y) return fail(POETX_ERR_INVALID_ARG, "x or y is NULL");
  if (!aligned16(x) || !aligned16(y) || (saved_b && !aligned16(saved_b)) ||
      (saved_a && !aligned16(saved_a)))
    return fail(POETX_ERR_ALIGN, "x, y, saved_b, saved_a must be 16-byte aligned");
  if ((st = check_ws(workspace, ws_bytes, poetx_fwd_workspace_bytes(L, T))) != POETX_OK) return st;
  if ((st = check_device()) != POETX_OK) return st;
  cudaStream_t s = as_stream(stream);
  FwdWs w;
  fwd_layout(L, T, workspace, &w);
  void* B = saved_b ? saved_b : w.B;
  void* A = saved_a ? saved_a : w.A;   // A = X[:, perm_r], kept for the backward when given
  const int e = elem_size(L->dtype);
  const DT t = dt_of(L->dtype);
  const int64_t m = L->m, n = L->n, b = L->b;
  const void* Gr = L->dtype == POETX_BF16 ? L->g_r_lp : (const void*)L->g_r;
  const void* Gp = L->dtype == POETX_BF16 ? L->g_p_lp : (const void*)L->g_p;
  CHECK_CUDA(gather_cols(x, A, T, m, nullptr, L->perm_r, e, s, "perm_fwd_gather_X"), "fwd gather");
  CHECK_CUDA(gemm_blockwise(t, A, Gr, w.A1, T, m, b, false, s), "fwd R blocks");
  // B = A' W0' and C = B Diag(G_P): one kernel where the layer asks for it and it applies (B
  // written only when the caller keeps it), else two launches
  const bool fused = (L->flags & POETX_LAYER_FUSED_W0_P) && t == DT::BF16 && !w0m_i8(L) &&
                     w0_p_fused_supported(w.A1, L->w0m, Gp, saved_b, w.C, T, m, n, b);
  if (fused) {
    CHECK_CUDA(gemm_w0_p_fused(w.A1, L->w0m, Gp, saved_b, w.C, T, m, n, b, s),
               "fwd W0' GEMM + P blocks");
  } else {
    CHECK_CUDA(w0_product(L, w.A1, B, T, false, w.Wd, s), "fwd W0' GEMM");
    CHECK_CUDA(gemm_blockwise(t, B, Gp, w.C, T, n, b, false, s), "fwd P blocks");
  }
  CHECK_CUDA(scatter_cols(w.C, y, T, n, L->perm_p, e, w.inv, s, "perm_fwd_scatter_Y"), "fwd scatter");
  return POETX_OK;
}
}  // namespace

extern "C" {

poetx_status poetx_linear_fwd(const poetx_layer* L, const void* x, int64_t T, void* y,
                              void* saved_b, void* workspace, size_t ws_bytes, void* stream) {
  return linear_fwd_impl(L, x, T, y, saved_b, nullptr, workspace, ws_bytes, stream);
}

poetx_status poetx_linear_fwd_ex(const poetx_layer* L, const void* x, int64_t T, void* y,
                                 void* saved_b, void* saved_a, void* workspace, size_t ws_bytes,
                                 void* stream) {
  return linear_fwd_impl(L, x, T, y, saved_b, saved_a, workspace, ws_bytes, stream);
}

// ------------------------------------------------------------------ backward
size_t poetx_bwd_workspace_bytes(const poetx_layer* L, int64_t T) {
  if (!L || T < 0 || L->m <= 0 || L->n <= 0 || L->b < 2) return 0;
  return bwd_layout(L, T, nullptr, nullptr);
}

}  // extern "C"

namespace {
// dG_out: the per-block gradients [m/b + n/b][b][b] are written there (summed over split
// ranges) and no dq is formed; dq_r / dq_p are then ignored.
poetx_status linear_bwd_impl(const poetx_layer* L, const void* x, const void* dy,
                             const void* saved_b, const void* saved_a, int64_t T, void* dx,
                             float* dq_r, float* dq_p, void* workspace, size_t ws_bytes,
                             void* stream, float* dG_out = nullptr) {
  poetx_status st = check_layer(L, true);
  if (st != POETX_OK) return st;
  if (T < 0) return fail(POETX_ERR_SHAPE, "T < 0");
  if (dG_out) dq_r = dq_p = nullptr;
  if ((dq_r && !L->q_r) || (dq_p && !L->q_p))
    return fail(POETX_ERR_INVALID_ARG, "dq requested but the layer has no q");
  if (dG_out && !aligned16(dG_out)) return fail(POETX_ERR_ALIGN, "dG not 16-byte aligned");
  // which sides' block gradients are formed
  const bool want_r = dq_r || dG_out, want_p = dq_p || dG_out;
  if ((!x && !saved_a) || !dy) return fail(POETX_ERR_INVALID_ARG, "x (or saved_a) or dy is NULL");
  if ((x && !aligned16(x)) || !aligned16(dy) || (saved_b && !aligned16(saved_b)) ||
      (saved_a && !aligned16(saved_a)) || (dx && !aligned16(dx)) ||
      (dq_r && !aligned16(dq_r)) || (dq_p && !aligned16(dq_p)))
    return fail(POETX_ERR_ALIGN, "backward pointers must be 16-byte aligned");
  if ((st = check_ws(workspace, ws_bytes, poetx_bwd_workspace_bytes(L, T))) != POETX_OK) return st;
  if ((st = check_device()) != POETX_OK) return st;
  cudaStream_t s = as_stream(stream);
  BwdWs w;
  bwd_layout(L, T, workspace, &w);
  const int e = elem_size(L->dtype);
  const DT t = dt_of(L->dtype);
  const int64_t m = L->m, n = L->n, b = L->b;
  const void* Gr = L->dtype == POETX_BF16 ? L->g_r_lp : (const void*)L->g_r;
  const void* Gp = L->dtype == POETX_BF16 ? L->g_p_lp : (const void*)L->g_p;
  // A = X[:, perm_r]: the forward's saved copy, or gathered again from X (once, when first needed)
  const void* A = saved_a;
  bool have_a = saved_a != nullptr;
  if (!saved_b && (want_p || want_r)) {
    // memory-saving mode: rebuild B = (X[:, perm_r] Diag(G_R)) W0' exactly instead of keeping it
    if (!have_a) {
      CHECK_CUDA(gather_cols(x, w.A, T, m, nullptr, L->perm_r, e, s, "perm_bwd_regather_X"),
                 "bwd recompute gather");
      A = w.A;
      have_a = true;
    }
    CHECK_CUDA(gemm_blockwise(t, A, Gr, w.dA, T, m, b, false, s), "bwd recompute R blocks");
    CHECK_CUDA(w0_product(L, w.dA, w.B, T, false, w.Wd, s), "bwd recompute W0' GEMM");
    saved_b = w.B;
  }
  CHECK_CUDA(gather_cols(dy, w.dC, T, n, nullptr, L->perm_p, e, s, "perm_bwd_gather_dY"), "bwd gather dY");
  CHECK_CUDA(gemm_blockwise(t, w.dC, Gp, w.dB, T, n, b, true, s), "bwd P blocks");
  // the block gradients go straight into dG_out where a launch needs no split partials
  float* dG_all = dG_out ? dG_out : w.dG;
  float* dG_r = dG_all;
  float* dG_p = dG_all + (m / b) * b * b;
  int sp_r = 1, sp_p = 1;
  // with both sides wanted, dG_R and dG_P run as one launch once dA' exists (bf16, b % 256 == 0)
  const bool one_dg = want_r && want_p && t == DT::BF16 && b % 256 == 0 && T > 0;
  if (want_p && !one_dg)
    CHECK_CUDA(gemm_block_grad(t, saved_b, w.dC, dG_p, T, n, b, w.part_p, &sp_p, s), "bwd dG_P");
  CHECK_CUDA(w0_product(L, w.dB, w.dA1, T, true, w.Wd, s), "bwd W0'^T GEMM");
  if (dx) {
    CHECK_CUDA(gemm_blockwise(t, w.dA1, Gr, w.dA, T, m, b, true, s), "bwd R blocks");
    CHECK_CUDA(scatter_cols(w.dA, dx, T, m, L->perm_r, e, w.inv, s, "perm_bwd_scatter_dX"),
               "bwd scatter dX");
  }
  bool merged = false;
  int sp_rp = 1;
  if (want_r) {
    if (!have_a) {
      CHECK_CUDA(gather_cols(x, w.A, T, m, nullptr, L->perm_r, e, s, "perm_bwd_gather_X"),
                 "bwd gather X");
      A = w.A;
      have_a = true;
    }
    if (one_dg) {
      const cudaError_t ce = gemm_block_grad2(t, A, w.dA1, m, saved_b, w.dC, n, dG_all, T, b,
                                              w.part_rp, &sp_rp, s);
      if (ce == cudaSuccess) merged = true;
      else if (ce != cudaErrorNotSupported) CHECK_CUDA(ce, "bwd dG_R + dG_P");
      else CHECK_CUDA(gemm_block_grad(t, saved_b, w.dC, dG_p, T, n, b, w.part_p, &sp_p, s),
                      "bwd dG_P");
    }
    if (!merged)
      CHECK_CUDA(gemm_block_grad(t, A, w.dA1, dG_r, T, m, b, w.part_r, &sp_r, s), "bwd dG_R");
  }
  if (dG_out) {
    // the block gradients themselves: partial sums added in split order where there are any
    const int64_t bb = b * b;
    if (merged) {
      if (sp_rp > 1)
        CHECK_CUDA(sum_partials(static_cast<const float*>(w.part_rp), dG_out,
                                (m / b + n / b) * bb, sp_rp, s), "dG sum");
    } else {
      if (sp_r > 1)
        CHECK_CUDA(sum_partials(static_cast<const float*>(w.part_r), dG_r, (m / b) * bb, sp_r, s),
                   "dG_R sum");
      if (sp_p > 1)
        CHECK_CUDA(sum_partials(static_cast<const float*>(w.part_p), dG_p, (n / b) * bb, sp_p, s),
                   "dG_P sum");
    }
    return POETX_OK;
  }
  if (dq_r || dq_p) {
    // one dq chain over the R blocks and the P blocks
    BlockRuns r;
    int k = 0;
    if (merged) {
      // partials of the one launch: [splits][m/b + n/b][b][b]
      const float* base = static_cast<const float*>(w.part_rp);
      const int64_t stride = (m / b + n / b) * b * b;
      r.q[0] = L->q_r; r.dq[0] = dq_r; r.splits[0] = sp_rp; r.nb[0] = (int)(m / b);
      r.q[1] = L->q_p; r.dq[1] = dq_p; r.splits[1] = sp_rp; r.nb[1] = (int)(n / b);
      r.parts[0] = sp_rp > 1 ? base : dG_r;
      r.parts[1] = sp_rp > 1 ? base + (m / b) * b * b : dG_p;
      if (sp_rp > 1) r.split_stride[0] = r.split_stride[1] = stride;
    } else {
      if (dq_r) {
        r.q[k] = L->q_r; r.dq[k] = dq_r; r.splits[k] = sp_r; r.nb[k] = (int)(m / b);
        r.parts[k] = sp_r > 1 ? static_cast<const float*>(w.part_r) : dG_r;
        ++k;
      }
      if (dq_p) {
        r.q[k] = L->q_p; r.dq[k] = dq_p; r.splits[k] = sp_p; r.nb[k] = (int)(n / b);
        r.parts[k] = sp_p > 1 ? static_cast<const float*>(w.part_p) : dG_p;
      }
    }
    CHECK_CUDA(gemm_dq_from_dg_runs(t, r, b, dq_r ? dG_r : dG_p, w.chain, s), "dq chain");
  }
  return POETX_OK;
}
}  // namespace

extern "C" {

poetx_status poetx_linear_bwd(const poetx_layer* L, const void* x, const void* dy,
                              const void* saved_b, int64_t T, void* dx, float* dq_r, float* dq_p,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (!x) return fail(POETX_ERR_INVALID_ARG, "x or dy is NULL");
  return linear_bwd_impl(L, x, dy, saved_b, nullptr, T, dx, dq_r, dq_p, workspace, ws_bytes,
                         stream);
}

poetx_status poetx_linear_bwd_ex(const poetx_layer* L, const void* x, const void* dy,
                                 const void* saved_b, const void* saved_a, int64_t T, void* dx,
                                 float* dq_r, float* dq_p, void* workspace, size_t ws_bytes,
                                 void* stream) {
  return linear_bwd_impl(L, x, dy, saved_b, saved_a, T, dx, dq_r, dq_p, workspace, ws_bytes,
                         stream);
}

poetx_status poetx_linear_bwd_dg(const poetx_layer* L, const void* x, const void* dy,
                                 const void* saved_b, const void* saved_a, int64_t T, void* dx,
                                 float* dG, void* workspace, size_t ws_bytes, void* stream) {
  if (!dG) return fail(POETX_ERR_INVALID_ARG, "dG is NULL");
  return linear_bwd_impl(L, x, dy, saved_b, saved_a, T, dx, nullptr, nullptr, workspace,
                         ws_bytes, stream, dG);
}

size_t poetx_layers_dq_workspace_bytes(const poetx_layer* const* layers, int32_t nlayers) {
  if (!layers || nlayers <= 0) return 0;
  size_t need = 0;
  for (int32_t i0 = 0; i0 < nlayers; i0 += kLayersPerBatch) {
    int64_t nb = 0, b = 0;
    DT t = DT::BF16;
    for (int32_t i = i0; i < nlayers && i < i0 + kLayersPerBatch; ++i) {
      const poetx_layer* L = layers[i];
      if (!L || L->b < 2 || L->m <= 0 || L->n <= 0) return 0;
      nb += L->m / L->b + L->n / L->b;
      b = L->b;
      t = dt_of(L->dtype);
    }
    // the chain's own buffers, then the summed gradients it reads in place
    need = std::max(need, align_up(gemm_dq_ws_bytes(t, nb, b), 256) +
                              (size_t)(nb * b * b) * sizeof(float));
  }
  return need;
}

poetx_status poetx_layers_dq_from_dg(const poetx_layer* const* layers, const float* const* dG,
                                     float* const* dq_r, float* const* dq_p, int32_t nlayers,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (nlayers < 0) return fail(POETX_ERR_INVALID_ARG, "nlayers < 0");
  if (nlayers == 0) return POETX_OK;
  if (!layers || !dG || !dq_r || !dq_p) return fail(POETX_ERR_INVALID_ARG, "NULL array");
  for (int32_t i = 0; i < nlayers; ++i) {
    const poetx_layer* L = layers[i];
    poetx_status st = check_layer(L, true);
    if (st != POETX_OK) return st;
    if (!L->q_r || !L->q_p) return fail(POETX_ERR_INVALID_ARG, "layer %d has no q", (int)i);
    if (L->b != layers[0]->b)
      return fail(POETX_ERR_SHAPE, "layer %d has b=%lld, layer 0 b=%lld", (int)i, (long long)L->b,
                  (long long)layers[0]->b);
    if (L->dtype != layers[0]->dtype)
      return fail(POETX_ERR_DTYPE, "layer %d has another dtype than layer 0", (int)i);
    if (!dG[i]) return fail(POETX_ERR_INVALID_ARG, "dG of layer %d is NULL", (int)i);
    if (!aligned16(dG[i]) || (dq_r[i] && !aligned16(dq_r[i])) || (dq_p[i] && !aligned16(dq_p[i])))
      return fail(POETX_ERR_ALIGN, "layer %d: dG / dq not 16-byte aligned", (int)i);
  }
  poetx_status st = check_ws(workspace, ws_bytes, poetx_layers_dq_workspace_bytes(layers, nlayers));
  if (st != POETX_OK) return st;
  if ((st = check_device()) != POETX_OK) return st;
  const int64_t b = layers[0]->b;
  const DT t = dt_of(layers[0]->dtype);
  for (int32_t i0 = 0; i0 < nlayers; i0 += kLayersPerBatch) {
    BlockRuns r;
    int64_t nb = 0;
    for (int32_t i = i0; i < nlayers && i < i0 + kLayersPerBatch; ++i) {
      const poetx_layer* L = layers[i];
      const int k = 2 * (i - i0);
      // a side whose dq is not wanted takes no blocks
      if (dq_r[i]) {
        r.q[k] = L->q_r; r.dq[k] = dq_r[i]; r.nb[k] = (int)(L->m / b); r.parts[k] = dG[i];
      }
      if (dq_p[i]) {
        r.q[k + 1] = L->q_p; r.dq[k + 1] = dq_p[i]; r.nb[k + 1] = (int)(L->n / b);
        r.parts[k + 1] = dG[i] + (L->m / b) * b * b;
      }
      nb += r.nb[k] + r.nb[k + 1];
    }
    if (nb == 0) continue;
    char* base = static_cast<char*>(workspace);
    float* scratch = reinterpret_cast<float*>(base + align_up(gemm_dq_ws_bytes(t, nb, b), 256));
    CHECK_CUDA(gemm_dq_from_dg_runs(t, r, b, scratch, workspace, as_stream(stream)),
               "layers_dq_from_dg");
  }
  return POETX_OK;
}

// ------------------------------------------------------------------ permutations
poetx_status poetx_merge_permutations(const void* w0, const int32_t* perm_r,
                                      const int32_t* perm_p, int64_t m, int64_t n, int32_t dtype,
                                      void* w0m, void* stream) {
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (m < 0 || n < 0) return fail(POETX_ERR_SHAPE, "negative size");
  if (m == 0 || n == 0) return POETX_OK;
  if (!w0 || !perm_r || !perm_p || !w0m) return fail(POETX_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(w0) || !aligned16(w0m) || !aligned16(perm_r) || !aligned16(perm_p))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  const size_t bytes = (size_t)(m * n * elem_size(dtype));
  const char* a = static_cast<const char*>(w0);
  const char* c = static_cast<const char*>(w0m);
  if (a < c + bytes && c < a + bytes) return fail(POETX_ERR_INVALID_ARG, "w0m overlaps w0");
  poetx_status st = check_device();
  if (st != POETX_OK) return st;
  CHECK_CUDA(gather_cols(w0, w0m, m, n, perm_r, perm_p, elem_size(dtype), as_stream(stream)),
             "merge_permutations");
  return POETX_OK;
}

// ------------------------------------------------------------------ 8-bit W0'
poetx_status poetx_quantize_w0(const void* w, int64_t m, int64_t n, int32_t dtype, int8_t* wq,
                               float* scale, void* stream) {
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (m < 0 || n < 0) return fail(POETX_ERR_SHAPE, "negative size");
  if (m == 0 || n == 0) return POETX_OK;
  if (!w || !wq || !scale) return fail(POETX_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(w) || !aligned16(wq) || !aligned16(scale))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  poetx_status st = check_device();
  if (st != POETX_OK) return st;
  CHECK_CUDA(quantize_cols_i8(w, dt_of(dtype), m, n, wq, scale, as_stream(stream)), "quantize_w0");
  return POETX_OK;
}

poetx_status poetx_dequantize_w0(const int8_t* wq, const float* scale, int64_t m, int64_t n,
                                 void* w_bf16, void* stream) {
  if (m < 0 || n < 0) return fail(POETX_ERR_SHAPE, "negative size");
  if (m == 0 || n == 0) return POETX_OK;
  if (!wq || !scale || !w_bf16) return fail(POETX_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(wq) || !aligned16(scale) || !aligned16(w_bf16))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  poetx_status st = check_device();
  if (st != POETX_OK) return st;
  CHECK_CUDA(dequantize_cols_i8(wq, scale, m, n, static_cast<__nv_bfloat16*>(w_bf16),
                                as_stream(stream)),
             "dequantize_w0");
  return POETX_OK;
}

poetx_status poetx_resample_permutation(uint64_t seed, int32_t lane, int64_t k, int32_t* perm,
                                        void* stream) {
  if (k < 0 || k > (int64_t)INT32_MAX) return fail(POETX_ERR_SHAPE, "bad length");
  if (k == 0) return POETX_OK;
  if (!perm) return fail(POETX_ERR_INVALID_ARG, "perm is NULL");
  poetx_status st = check_device();
  if (st != POETX_OK) return st;
  CHECK_CUDA(resample_permutation(seed, lane, k, perm, as_stream(stream)), "resample");
  return POETX_OK;
}

poetx_status poetx_validate_permutation(const int32_t* perm, int64_t k, void* workspace,
                                        size_t ws_bytes, void* stream) {
  if (k < 0) return fail(POETX_ERR_SHAPE, "negative length");
  if (k == 0) return POETX_OK;
  if (!perm) return fail(POETX_ERR_INVALID_ARG, "perm is NULL");
  poetx_status st = check_ws(workspace, ws_bytes, (size_t)(k + 1) * 4);
  if (st != POETX_OK) return st;
  if ((st = check_device()) != POETX_OK) return st;
  cudaStream_t s = as_stream(stream);
  int32_t* cnt = static_cast<int32_t*>(workspace);
  CHECK_CUDA(count_permutation(perm, k, cnt, s), "validate");
  int32_t flag = 0;
  CHECK_CUDA(cudaMemcpyAsync(&flag, cnt + k, 4, cudaMemcpyDeviceToHost, s), "validate read");
  CHECK_CUDA(cudaStreamSynchronize(s), "validate sync");
  return flag ? fail(POETX_ERR_BAD_INDEX, "array is not a permutation of 0..%lld",
                     (long long)(k - 1))
              : POETX_OK;
}

// ------------------------------------------------------------------ merge-then-reinitialize
size_t poetx_merge_reinit_workspace_bytes(const poetx_layer* L) {
  if (!L || L->m <= 0 || L->n <= 0) return 0;
  return merge_layout(L, nullptr, nullptr);
}

poetx_status poetx_merge_reinit(poetx_layer* L, uint64_t seed, void* workspace, size_t ws_bytes,
                                void* stream) {
  poetx_status st = check_layer(L, true);
  if (st != POETX_OK) return st;
  if (!L->q_r || !L->q_p) return fail(POETX_ERR_INVALID_ARG, "layer has no q");
  if ((st = check_ws(workspace, ws_bytes, poetx_merge_reinit_workspace_bytes(L))) != POETX_OK)
    return st;
  if ((st = check_device()) != POETX_OK) return st;
  cudaStream_t s = as_stream(stream);
  MergeWs w;
  merge_layout(L, workspace, &w);
  const int e = elem_size(L->dtype);
  const DT t = dt_of(L->dtype);
  const int64_t m = L->m, n = L->n, b = L->b;
  const void* Gr = L->dtype == POETX_BF16 ? L->g_r_lp : (const void*)L->g_r;
  const void* Gp = L->dtype == POETX_BF16 ? L->g_p_lp : (const void*)L->g_p;
  const bool i8 = w0m_i8(L);
  // M = Diag(G_R) W0' Diag(G_P), block by block (an int8 W0' is dequantised into M's buffer
  // first; that buffer is free again once W0' Diag(G_P) is formed)
  const void* W0m = L->w0m;
  if (i8) {
    CHECK_CUDA(dequantize_cols_i8(static_cast<const int8_t*>(L->w0m), L->w0m_scale, m, n,
                                  static_cast<__nv_bfloat16*>(w.M), s),
               "merge dequantise W0'");
    W0m = w.M;
  }
  CHECK_CUDA(gemm_blockwise(t, W0m, Gp, w.N1, m, n, b, false, s), "merge W0' G_P");
  CHECK_CUDA(gemm_blockwise_left(t, Gr, w.N1, w.M, m, n, b, s), "merge G_R (.)");
  // new permutations, composed index maps rho = perm_old^{-1} o perm_new
  CHECK_CUDA(resample_permutation(seed, 0, m, w.pr_new, s), "resample R");
  CHECK_CUDA(resample_permutation(seed, 1, n, w.pp_new, s), "resample P");
  CHECK_CUDA(compose_inverse(L->perm_r, w.pr_new, w.inv, w.rho_r, m, s), "compose R");
  CHECK_CUDA(compose_inverse(L->perm_p, w.pp_new, w.inv, w.rho_p, n, s), "compose P");
  // W0'_new[i, j] = M[rho_r[i], rho_p[j]]; int8 layers store it as codes and column scales
  if (i8) {
    CHECK_CUDA(gather_cols(w.M, w.N1, m, n, w.rho_r, w.rho_p, e, s), "merge regather");
    CHECK_CUDA(quantize_cols_i8(w.N1, DT::BF16, m, n, static_cast<int8_t*>(L->w0m), L->w0m_scale,
                                s),
               "merge quantise W0'");
  } else {
    CHECK_CUDA(gather_cols(w.M, L->w0m, m, n, w.rho_r, w.rho_p, e, s), "merge regather");
  }
  CHECK_CUDA(cudaMemcpyAsync(L->perm_r, w.pr_new, m * 4, cudaMemcpyDeviceToDevice, s), "perm_r");
  CHECK_CUDA(cudaMemcpyAsync(L->perm_p, w.pp_new, n * 4, cudaMemcpyDeviceToDevice, s), "perm_p");
  CHECK_CUDA(fill_zero_f32(L->q_r, m / b * (b * (b - 1) / 2), s), "zero q_r");
  CHECK_CUDA(fill_zero_f32(L->q_p, n / b * (b * (b - 1) / 2), s), "zero q_p");
  return POETX_OK;
}

}  // extern "C"
