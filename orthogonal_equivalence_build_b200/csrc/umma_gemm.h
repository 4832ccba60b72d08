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
// b_i8: B is an int8 tensor [rows][cols] (row stride ld bytes) with fp32 scales b_scale[cols];
// the product uses B = bf16(code * b_scale[col]) (CTA-pair kernel, one dense product only).
// K segments (nseg > 1): the contraction is nseg equal segments of K / nseg; within segment s
// the k index restarts at 0 and the TMA coordinates of A and B are shifted by (a_dx[s], a_dy[s])
// and (b_dx[s], b_dy[s]) (x = column, y = row of the 2-D tensor). One accumulator sums
// A_s B_s over the segments, e.g. Xhi Yhi + Xhi Ylo + Xlo Yhi from separate hi / lo buffers.
//
// Epilogue modes (fp32 accumulators of grouped b x b products, groups = blocks, M = N = b):
// instead of storing C, the epilogue evaluates the next elementwise step of the Cayley-Neumann
// blocks or of their gradient at each element (g; i, j) and stores its results. Q(g; i, j) is
// qh + ql (bf16 hi / lo parts of the skew block, ql may be null), all arrays [groups][b][b].
enum EpiMode : int {
  kEpiStore = 0,
  kEpiCnpS = 1,   // acc = S = Q Q: o0, o1 = hi / lo of S; o2, o3 = hi / lo of H = 2I + 2Q + S
  kEpiCnpG = 2,   // acc = S H:  G = I + 2Q + acc to g[run] (fp32) and g_lp[run] (bf16); block g
                  // is block g - run_end[run - 1] of the run with run_end[run - 1] <= g <
                  // run_end[run] (run_end[-1] = 0), for runs 0 .. nruns - 1
  kEpiDqS = 3,    // acc = S = Q Q: o0 = bf16(S), o1 = bf16(S - 2Q)
};
struct Epi {
  int mode = kEpiStore;
  int b = 0, nruns = 1;
  const __nv_bfloat16* qh = nullptr;
  const __nv_bfloat16* ql = nullptr;
  __nv_bfloat16* o[4] = {nullptr, nullptr, nullptr, nullptr};
  float* g[kMaxRuns] = {};
  __nv_bfloat16* g_lp[kMaxRuns] = {};
  int run_end[kMaxRuns] = {};
};

struct Gemm {
  int64_t M = 0, N = 0, K = 0, groups = 1, splits = 1;
  const void* A = nullptr; int64_t a_rows = 0, a_cols = 0, a_ld = 0; bool a_mn = false;
  int64_t a_gm = 0, a_gk = 0;
  const void* B = nullptr; int64_t b_rows = 0, b_cols = 0, b_ld = 0; bool b_mn = false;
  int64_t b_gn = 0, b_gk = 0;
  bool b_i8 = false; const float* b_scale = nullptr;
  int nseg = 1;
  int64_t a_dx[3] = {0, 0, 0}, a_dy[3] = {0, 0, 0}, b_dx[3] = {0, 0, 0}, b_dy[3] = {0, 0, 0};
  Epi epi;
  void* C = nullptr; bool out_f32 = false; int64_t ldc = 0, c_gs = 0, c_split = 0;
  const char* name = nullptr;
  int bn = 0;   // single-CTA tile width (64, 128 or 256; N must be a multiple); 0: the widest
  // CTA-pair kernel only: groups >= groups_1 read a second operand pair (A2, B2), laid out like
  // (A, B) with its own extents; group g >= groups_1 is group g - groups_1 of that pair. The
  // output keeps the global group index. 0: every group reads (A, B).
  int64_t groups_1 = 0;
  const void* A2 = nullptr; int64_t a2_rows = 0, a2_cols = 0, a2_ld = 0;
  const void* B2 = nullptr; int64_t b2_rows = 0, b2_cols = 0, b2_ld = 0;
  // Limit of the epilogue warps' wait for a finished accumulator, in ns (0: the kernels'
  // default of a few seconds). Only the kernel-level test hook sets it, to make the wait run out.
  unsigned long long epi_wait_ns = 0;
  // 256 x 512 kernel only: the two MMAs of a K step share A through the collector buffer
  bool wide_collect = true;
  // CTA-pair kernel, with a second operand pair: two dependent products in one launch. Groups
  // >= groups_1 form the second product, with epilogue epi2 (has_epi2) and, with c_rel2,
  // output groups counted from groups_1. With deps (dep_blocks ints, zero at launch, fp32
  // outputs), second-product group g starts loading only after deps[(g - groups_1) % dep_blocks]
  // reached dep_target, which the first product's epilogue warps of group g' = that index
  // raise by one each after their stores (a 256 x 256 tile has 8 such warps). All clusters are
  // resident at once and the first product's tiles come first in every cluster's order, so
  // the waits always end (each is bounded all the same).
  Epi epi2;
  bool has_epi2 = false;
  int* deps = nullptr;
  int dep_target = 0, dep_blocks = 0;
  bool c_rel2 = false;
};

bool supported(const Gemm& g);
// The same product on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 pair tiles); needs
// N % 256 == 0 and M >= 256.
bool pair_supported(const Gemm& g);
cudaError_t gemm_pair(const Gemm& g, cudaStream_t s);
// Products without split K, A K-major, bf16 out (dense, or grouped as above) on 256 x 512 pair
// tiles with one 512-column accumulator in two halves; needs N % 512 == 0 and M >= 256.
bool wide_supported(const Gemm& g);
cudaError_t gemm_wide(const Gemm& g, cudaStream_t s);
// The forward's W0' product and P-block product in one launch (b = 512, bf16): C = (A1 W0')
// Diag(G_P) with A1 [T][m], W0' [m][n], the stacked bf16 G_P blocks Gp [n][512] (block j in rows
// 512 j ..), C [T][n]; Bout, when not NULL, also receives B = A1 W0' [T][n]. T >= 256, m and n
// multiples of 512, 16-byte aligned pointers.
bool w0p_fused_supported(const void* A1, const void* W0, const void* Gp, const void* Bout,
                         const void* Cout, int64_t T, int64_t m, int64_t n, int64_t b);
cudaError_t w0p_fused(const void* A1, const void* W0, const void* Gp, void* Bout, void* Cout,
                      int64_t T, int64_t m, int64_t n, int64_t b, cudaStream_t s);

// Number of K ranges the kernel actually uses for `splits` requested ranges over K
// (ranges of whole 64-wide K blocks, none empty).
int effective_splits(int64_t K, int64_t splits);
// The single-CTA kernel (128 x bn tiles).
cudaError_t gemm(const Gemm& g, cudaStream_t s);
int sm_count();

}  // namespace umma
}  // namespace poetx
