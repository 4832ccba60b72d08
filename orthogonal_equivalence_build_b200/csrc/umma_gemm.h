// bf16 tensor-core GEMM (tcgen05 / TMEM / TMA) — host interface.
#pragma once
#include "internal.h"

namespace poetx {
namespace umma {

// C[split](g; i, j) = sum_k A(g; i, k) B(g; k, j), i < M, j < N, over the k range of `split`,
// for g = 0..groups-1. Operands are 2-D bf16 tensors [rows][cols] (cols contiguous, row stride
// ld elements):
//   A K-major  (a_mn = false): A(g; i, k) = A[a_gm*g + i][a_gk*g + k]
//   A MN-major (a_mn = true):  A(g; i, k) = A[a_gk*g + k][a_gm*g + i]
//   B K-major  (b_mn = false): B(g; k, j) = B[b_gn*g + j][b_gk*g + k]
//   B MN-major (b_mn = true):  B(g; k, j) = B[b_gk*g + k][b_gn*g + j]
// Reads beyond a tensor's rows/cols are zeros. C is bf16 or fp32 row-major:
//   C[split * c_split + g * c_gs + i * ldc + j].
struct Gemm {
  int64_t M = 0, N = 0, K = 0, groups = 1, splits = 1;
  const void* A = nullptr; int64_t a_rows = 0, a_cols = 0, a_ld = 0; bool a_mn = false;
  int64_t a_gm = 0, a_gk = 0;
  const void* B = nullptr; int64_t b_rows = 0, b_cols = 0, b_ld = 0; bool b_mn = false;
  int64_t b_gn = 0, b_gk = 0;
  void* C = nullptr; bool out_f32 = false; int64_t ldc = 0, c_gs = 0, c_split = 0;
  const char* name = nullptr;
};

bool supported(const Gemm& g);
// The same product on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 pair tiles); needs
// N % 256 == 0 and M >= 256.
bool pair_supported(const Gemm& g);
cudaError_t gemm_pair(const Gemm& g, cudaStream_t s);

// Number of K ranges the kernel actually uses for `splits` requested ranges over K
// (ranges of whole 64-wide K blocks, none empty).
int effective_splits(int64_t K, int64_t splits);
cudaError_t gemm(const Gemm& g, cudaStream_t s);

}  // namespace umma
}  // namespace poetx
