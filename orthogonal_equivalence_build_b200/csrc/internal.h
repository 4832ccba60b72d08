// Internal interfaces between the library's translation units (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/poetx.h"

namespace poetx {

// ------------------------------------------------------------------ errors and tracing
void set_error(const char* fmt, ...);
// One launch record per traced kernel; both are no-ops while tracing is off.
int trace_begin(const char* name, cudaStream_t s);
void trace_end(int slot, cudaStream_t s);
// Device error word (bounded waits that expired write a nonzero code here).
int* device_error_word();

// Also an NVTX range of the same name around the launch (a no-op unless a tool such as ncu is
// attached), so profilers can select a kernel by the library's name for it.
struct TraceScope {
  int slot;
  cudaStream_t s;
  TraceScope(const char* name, cudaStream_t st) : slot(trace_begin(name, st)), s(st) {
    nvtxRangePushA(name);
  }
  ~TraceScope() {
    trace_end(slot, s);
    nvtxRangePop();
  }
};

// ------------------------------------------------------------------ programmatic dependent launch
// The hot-path kernels are launched with programmatic stream serialisation: a kernel may be
// scheduled, and run its prologue (barrier set-up, TMEM allocation), while the previous kernel
// of the stream finishes. Every such kernel calls pdl_wait() before its first global-memory
// access; it returns once the previous grid has completed and its writes are visible, so reads
// after writes and writes after reads across kernels keep stream order. pdl_trigger() allows the
// next launch to be scheduled. Both are no-ops in a kernel launched without the attribute.
// POETX_PDL=0 in the environment launches without it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
bool pdl_enabled();
void set_pdl_attr(cudaLaunchAttribute& a);

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  set_pdl_attr(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Runs of b x b blocks one CNP / dq launch sequence handles (a layer's R and P blocks, or those
// of up to eight layers).
constexpr int kMaxRuns = 16;
// element count rounded up to a multiple of 8 (16-byte aligned offsets for 2- and 4-byte types)
__host__ __device__ inline int64_t pad8(int64_t x) { return (x + 7) & ~(int64_t)7; }

// Carves aligned sub-buffers out of a caller workspace.
struct Arena {
  char* base;
  size_t cap;
  size_t used = 0;
  Arena(void* p, size_t c) : base(static_cast<char*>(p)), cap(c) {}
  void* take(size_t bytes) {
    size_t off = align_up(used, 256);
    used = off + bytes;
    return (base && used <= cap) ? base + off : nullptr;
  }
};

// ------------------------------------------------------------------ permutation kernels (perm.cu)
// out[r, c] = in[row_map ? row_map[r] : r, col_map[c]]       (gather)
cudaError_t gather_cols(const void* in, void* out, int64_t rows, int64_t cols,
                        const int32_t* row_map, const int32_t* col_map, int elem_bytes,
                        cudaStream_t s, const char* name = nullptr);
// out[r, col_map[c]] = in[r, c]                              (scatter)
// With inv_tmp (cols ints, 16-byte aligned) it runs as a gather through the inverse map.
cudaError_t scatter_cols(const void* in, void* out, int64_t rows, int64_t cols,
                         const int32_t* col_map, int elem_bytes, int32_t* inv_tmp,
                         cudaStream_t s, const char* name = nullptr);
// rho[i] = inverse(perm_old)[perm_new[i]]; inv_tmp is k ints of scratch
cudaError_t compose_inverse(const int32_t* perm_old, const int32_t* perm_new, int32_t* inv_tmp,
                            int32_t* rho, int64_t k, cudaStream_t s);
cudaError_t resample_permutation(uint64_t seed, int lane, int64_t k, int32_t* perm,
                                 cudaStream_t s);
cudaError_t count_permutation(const int32_t* perm, int64_t k, int32_t* counts_and_flag,
                              cudaStream_t s);

// ------------------------------------------------------------------ SIMT GEMM (simt_gemm.cu)
enum class DT : int { F32 = 0, BF16 = 1 };

// C[z](i, j) = alpha * sum_k A[z](i, k) B[z](k, j) + beta * D[z](i, j) + diag * (i == j)
// with X[z](i, j) = X[z * x_bs + i * x_rs + j * x_cs]. D may alias C (same strides).
struct SimtGemm {
  int64_t M, N, K, batch;
  const void* A; DT a_t; int64_t a_rs, a_cs, a_bs;
  const void* B; DT b_t; int64_t b_rs, b_cs, b_bs;
  void* C; DT c_t; int64_t c_rs, c_bs;
  const float* D; int64_t d_rs, d_bs;
  float alpha, beta, diag;
};
cudaError_t simt_gemm(const SimtGemm& g, cudaStream_t s);

// ------------------------------------------------------------------ 8-bit W0' (quant.cu)
// Per-column symmetric int8 codes of w [m, n] (bf16 or fp32) and their fp32 scales [n].
cudaError_t quantize_cols_i8(const void* w, DT t, int64_t m, int64_t n, int8_t* q, float* scale,
                             cudaStream_t s);
// out [m, n] = bf16(q * scale[col])
cudaError_t dequantize_cols_i8(const int8_t* q, const float* scale, int64_t m, int64_t n,
                               __nv_bfloat16* out, cudaStream_t s);

// ------------------------------------------------------------------ CNP and dq (cnp.cu)
size_t cnp_ws_bytes(int64_t nb, int64_t b);
cudaError_t cnp_build(const float* q, int64_t nb, int64_t b, float* g, __nv_bfloat16* g_lp,
                      void* ws, cudaStream_t s);
size_t dq_ws_bytes(int64_t nb, int64_t b);
// dq = packed skew gradient of G(q) given dG [nb, b, b] fp32
cudaError_t dq_from_dg(const float* q, const float* dG, int64_t nb, int64_t b, float* dq,
                       void* ws, cudaStream_t s);
// elementwise helpers
cudaError_t f32_to_bf16(const float* in, __nv_bfloat16* out, int64_t count, cudaStream_t s);
cudaError_t fill_zero_f32(float* p, int64_t count, cudaStream_t s);

}  // namespace poetx
