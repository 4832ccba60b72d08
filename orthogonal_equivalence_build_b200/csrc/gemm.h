// Contractions of the POET-X layer, routed to the tensor-core (tcgen05) kernel for bf16 operands
// and to the SIMT kernel for fp32 operands.
#pragma once
#include "internal.h"

namespace poetx {

// C_j = A_j G_j (or A_j G_j^T), j = 0..width/b-1: A, C [rows, width] row-major, G [width/b, b, b].
// The batch-wise block-diagonal product ("POET-X" blog §第三斧).
cudaError_t gemm_blockwise(DT t, const void* A, const void* G, void* C, int64_t rows,
                           int64_t width, int64_t b, bool transpose_g, cudaStream_t s);
// C[rb + i, :] = sum_k G_r[i, k] N[rb + k, :] for row block r (C = Diag(G) N), N, C [m, n].
cudaError_t gemm_blockwise_left(DT t, const void* G, const void* N, void* C, int64_t m,
                                int64_t n, int64_t b, cudaStream_t s);
// C [M, N] = A [M, K] W, with W [K, N] (w_trans = false) or W^T for W [N, K] (w_trans = true).
cudaError_t gemm_dense(DT t, const void* A, const void* W, void* C, int64_t M, int64_t N,
                       int64_t K, bool w_trans, cudaStream_t s);
// The same product with an 8-bit W ("POET-XQ"): int8 codes Wq (layout as W above) with fp32
// scales per column of the stored tensor, used as bf16(code * scale). The dequantisation runs
// inside the CTA-pair kernel's operand pipeline when dense_i8_fused(M, N); otherwise Wq is first
// dequantised into deq_ws (K * N bf16) and the bf16 product runs.
bool dense_i8_fused(int64_t M, int64_t N);
cudaError_t gemm_dense_i8(const void* A, const int8_t* Wq, const float* scale, void* C, int64_t M,
                          int64_t N, int64_t K, bool w_trans, void* deq_ws, cudaStream_t s);
// C = (A1 W0') Diag(G_P) in one tensor-core kernel (bf16, b = 512; see umma_gemm.h), B = A1 W0'
// also written to Bout when it is not NULL. Not supported: cudaErrorNotSupported.
bool w0_p_fused_supported(const void* A1, const void* W0, const void* Gp, const void* Bout,
                          const void* Cout, int64_t T, int64_t m, int64_t n, int64_t b);
cudaError_t gemm_w0_p_fused(const void* A1, const void* W0, const void* Gp, void* Bout,
                            void* Cout, int64_t T, int64_t m, int64_t n, int64_t b,
                            cudaStream_t s);
// dG_j = A_j^T B_j (contraction over the rows): A, B [rows, width], dG [width/b, b, b] fp32.
// Tensor-core tiles: 256 x 512 CTA pairs for b % 512 == 0, 256 x 256 for b % 256 == 0.
// bf16 operands split the contraction over `grad_splits` ranges of rows (the count that a time
// model of the launch plus its partial-sum traffic puts lowest). With more than one
// range the fp32 partial products go to `partials` ([splits][width/b][b][b], block_grad_ws_bytes
// bytes), dG is left untouched and *splits_used says how many ranges there are; the consumer
// (gemm_dq_from_dg) adds them in a fixed order. With one range the result is written to dG.
int grad_splits(int64_t nb, int64_t b, int64_t rows);
// out[e] = sum over s < splits of part[s * count + e], in that order (fp32)
cudaError_t sum_partials(const float* part, float* out, int64_t count, int splits,
                         cudaStream_t s);
size_t block_grad_ws_bytes(DT t, int64_t width, int64_t b, int64_t rows);
cudaError_t gemm_block_grad(DT t, const void* A, const void* B, float* dG, int64_t rows,
                            int64_t width, int64_t b, void* partials, int* splits_used,
                            cudaStream_t s);
// The same contraction for two runs of blocks in one launch (bf16, CTA pairs, b % 256 == 0):
// groups 0 .. w1/b - 1 from (A1, B1) [rows, w1], then w2/b groups from (A2, B2) [rows, w2];
// dG [(w1 + w2)/b][b][b]. One launch over all blocks fills the waves with fewer splits. With
// more than one range the partials go to `partials` ([splits][(w1 + w2)/b][b][b],
// block_grad2_ws_bytes bytes). Returns cudaErrorNotSupported where it does not apply.
size_t block_grad2_ws_bytes(DT t, int64_t w1, int64_t w2, int64_t b, int64_t rows);
cudaError_t gemm_block_grad2(DT t, const void* A1, const void* B1, int64_t w1, const void* A2,
                             const void* B2, int64_t w2, float* dG, int64_t rows, int64_t b,
                             void* partials, int* splits_used, cudaStream_t s);
// CNP blocks and the dq chain: tensor cores (cnp_tc.cu) when b is a multiple of 128, SIMT fp32
// (cnp.cu) otherwise; the dq chain of fp32 layers always runs in fp32 SIMT.
bool tc_blocks_supported(int64_t b);
size_t cnp_tc_ws_bytes(int64_t nb, int64_t b);
size_t dq_tc_ws_bytes(int64_t nb, int64_t b);

// Up to kMaxRuns runs of b x b blocks handled by one launch sequence (the R and the P blocks of
// a layer, or of several layers): launch-wide block j is block j - (nb[0] + .. + nb[k-1]) of the
// run k it falls in. Runs with nb = 0 are empty. Kernels take it as a __grid_constant__
// parameter (indexed in place, not copied per thread).
struct BlockRuns {
  const float* q[kMaxRuns] = {};        // packed skew parameters of each run
  float* g[kMaxRuns] = {};              // fp32 CNP blocks (may be null)
  __nv_bfloat16* g_lp[kMaxRuns] = {};   // bf16 copies (may be null)
  float* dq[kMaxRuns] = {};             // packed gradients
  const float* parts[kMaxRuns] = {};    // dG split partials [splits][nb][b][b]
  int splits[kMaxRuns];
  int64_t split_stride[kMaxRuns] = {};  // elements between splits (0: nb[run] * b * b)
  int nb[kMaxRuns] = {};
  BlockRuns() {
    for (int& x : splits) x = 1;
  }
  int total() const {
    int t = 0;
    for (int x : nb) t += x;
    return t;
  }
};
__device__ __forceinline__ int run_of(const BlockRuns& r, int g, int& local) {
  int start = 0;
#pragma unroll 1
  for (int k = 0; k < kMaxRuns - 1; ++k) {
    if (g < start + r.nb[k]) {
      local = g - start;
      return k;
    }
    start += r.nb[k];
  }
  local = g - start;
  return kMaxRuns - 1;
}
cudaError_t cnp_build_tc(const BlockRuns& r, int64_t b, void* ws, cudaStream_t s);
// dG: [total blocks][b][b] fp32, receives the summed gradients (a run whose parts pointer is
// its own slice of dG with one split is read in place).
cudaError_t dq_from_dg_tc(const BlockRuns& r, int64_t b, float* dG, void* ws, cudaStream_t s);

size_t gemm_cnp_ws_bytes(int64_t nb, int64_t b);
cudaError_t gemm_cnp_build(const float* q, int64_t nb, int64_t b, float* g, __nv_bfloat16* g_lp,
                           void* ws, cudaStream_t s);
// every run in one sequence (tensor cores), or one run after the other (SIMT)
cudaError_t gemm_cnp_build_runs(const BlockRuns& r, int64_t b, void* ws, cudaStream_t s);
size_t gemm_dq_ws_bytes(DT t, int64_t nb, int64_t b);
// dq of the runs in r; dG: [total blocks][b][b] fp32 scratch that receives summed gradients
cudaError_t gemm_dq_from_dg_runs(DT t, const BlockRuns& r, int64_t b, float* dG, void* ws,
                                 cudaStream_t s);

}  // namespace poetx
