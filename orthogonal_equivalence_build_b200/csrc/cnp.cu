// Cayley-Neumann blocks and their gradient.
//
// G = I + 2(Q + Q^2 + Q^2 Q) + Q^2 Q^2 ("POET-X" blog §第四斧 item 2; "Reparameterized LLM
// Training ..." §2 CNP with k = 3). Evaluated with S = Q^2 as
//     G = (I + 2Q) + S (2I + 2Q + S),
// which uses exactly the two products S = Q Q and S (2I + 2Q + S) and every term from Q and Q^2.
//
// Gradient (chain rule through the same evaluation order; Q^T = -Q and S^T = S):
//     Hbar = S dG,   Sbar = dG (2I - 2Q + S) + Hbar,   Z = Sbar + Sbar^T,
//     U = 2 dG + 2 Hbar - Z Q,   dq_ij = U_ij - U_ji  (i < j).
// (The two S-terms Sbar Q^T + Q^T Sbar reduce to the skew part of Z Q.)
#include "internal.h"

#include <algorithm>

namespace poetx {
namespace {

__device__ __forceinline__ int64_t triu_index(int64_t i, int64_t j, int64_t b) {
  // position of (i, j), i < j, in the row-major strict upper triangle
  return i * b - i * (i + 1) / 2 + (j - i - 1);
}

__device__ __forceinline__ float skew_entry(const float* __restrict__ qb, int64_t i, int64_t j,
                                            int64_t b) {
  if (i < j) return qb[triu_index(i, j, b)];
  if (i > j) return -qb[triu_index(j, i, b)];
  return 0.f;
}

// out = cI*I + cQ*Q(q) + cS*S + cST*S^T + cD*D, per b x b block.
__global__ void combine_kernel(float* __restrict__ out, const float* __restrict__ q,
                               const float* S, const float* __restrict__ D, int64_t nb,
                               int64_t b, float cI, float cQ, float cS, float cST, float cD) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    float v = (i == j) ? cI : 0.f;
    if (q && cQ != 0.f) v += cQ * skew_entry(q + blk * qs, i, j, b);
    if (S && cS != 0.f) v += cS * S[e];
    if (S && cST != 0.f) v += cST * S[blk * bb + j * b + i];
    if (D && cD != 0.f) v += cD * D[e];
    out[e] = v;
  }
}

// dq[blk][(i,j)] = U_ij - U_ji for i < j
__global__ void pack_skew_kernel(const float* __restrict__ U, float* __restrict__ dq, int64_t nb,
                                 int64_t b) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    if (i < j) dq[blk * qs + triu_index(i, j, b)] = U[e] - U[blk * bb + j * b + i];
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                   int64_t count) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = __float2bfloat16_rn(in[e]);
}

int grid_for(int64_t n) { return (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 16)); }

cudaError_t combine(float* out, const float* q, const float* S, const float* D, int64_t nb,
                    int64_t b, float cI, float cQ, float cS, float cST, float cD, cudaStream_t s) {
  TraceScope t("cnp_combine", s);
  combine_kernel<<<grid_for(nb * b * b), 256, 0, s>>>(out, q, S, D, nb, b, cI, cQ, cS, cST, cD);
  return cudaGetLastError();
}

// C = alpha * A B + beta * D over nb independent b x b blocks (all fp32, row-major).
cudaError_t block_mm(const float* A, bool a_trans, const float* B, float* C, const float* D,
                     float alpha, float beta, int64_t nb, int64_t b, cudaStream_t s) {
  SimtGemm g{};
  g.M = g.N = g.K = b;
  g.batch = nb;
  g.A = A; g.a_t = DT::F32; g.a_bs = b * b;
  g.a_rs = a_trans ? 1 : b; g.a_cs = a_trans ? b : 1;
  g.B = B; g.b_t = DT::F32; g.b_rs = b; g.b_cs = 1; g.b_bs = b * b;
  g.C = C; g.c_t = DT::F32; g.c_rs = b; g.c_bs = b * b;
  g.D = D; g.d_rs = b; g.d_bs = b * b;
  g.alpha = alpha; g.beta = beta; g.diag = 0.f;
  return simt_gemm(g, s);
}

#define POETX_TRY(x)                         \
  do {                                       \
    cudaError_t e_ = (x);                    \
    if (e_ != cudaSuccess) return e_;        \
  } while (0)

}  // namespace

size_t cnp_ws_bytes(int64_t nb, int64_t b) {
  const size_t blk = align_up((size_t)(nb * b * b) * sizeof(float), 256);
  return 3 * blk;
}

cudaError_t cnp_build(const float* q, int64_t nb, int64_t b, float* g, __nv_bfloat16* g_lp,
                      void* ws, cudaStream_t s) {
  if (nb == 0) return cudaSuccess;
  Arena a(ws, cnp_ws_bytes(nb, b));
  const size_t bytes = (size_t)(nb * b * b) * sizeof(float);
  float* Qm = static_cast<float*>(a.take(bytes));
  float* Sm = static_cast<float*>(a.take(bytes));
  float* Gt = static_cast<float*>(a.take(bytes));
  float* G = g ? g : Gt;
  POETX_TRY(combine(Qm, q, nullptr, nullptr, nb, b, 0.f, 1.f, 0.f, 0.f, 0.f, s));   // Q
  POETX_TRY(block_mm(Qm, false, Qm, Sm, nullptr, 1.f, 0.f, nb, b, s));              // S = Q Q
  POETX_TRY(combine(G, q, nullptr, nullptr, nb, b, 1.f, 2.f, 0.f, 0.f, 0.f, s));     // I + 2Q
  POETX_TRY(combine(Qm, q, Sm, nullptr, nb, b, 2.f, 2.f, 1.f, 0.f, 0.f, s));         // 2I + 2Q + S
  POETX_TRY(block_mm(Sm, false, Qm, G, G, 1.f, 1.f, nb, b, s));                     // G += S H
  if (g_lp) POETX_TRY(f32_to_bf16(G, g_lp, nb * b * b, s));
  return cudaSuccess;
}

size_t dq_ws_bytes(int64_t nb, int64_t b) {
  const size_t blk = align_up((size_t)(nb * b * b) * sizeof(float), 256);
  return 5 * blk;
}

cudaError_t dq_from_dg(const float* q, const float* dG, int64_t nb, int64_t b, float* dq,
                       void* ws, cudaStream_t s) {
  if (nb == 0) return cudaSuccess;
  Arena a(ws, dq_ws_bytes(nb, b));
  const size_t bytes = (size_t)(nb * b * b) * sizeof(float);
  float* Qm = static_cast<float*>(a.take(bytes));
  float* Sm = static_cast<float*>(a.take(bytes));
  float* Hb = static_cast<float*>(a.take(bytes));
  float* T1 = static_cast<float*>(a.take(bytes));
  float* Sb = static_cast<float*>(a.take(bytes));
  POETX_TRY(combine(Qm, q, nullptr, nullptr, nb, b, 0.f, 1.f, 0.f, 0.f, 0.f, s));   // Q
  POETX_TRY(block_mm(Qm, false, Qm, Sm, nullptr, 1.f, 0.f, nb, b, s));              // S = Q Q
  POETX_TRY(block_mm(Sm, false, dG, Hb, nullptr, 1.f, 0.f, nb, b, s));              // Hbar = S dG
  POETX_TRY(combine(T1, q, Sm, nullptr, nb, b, 2.f, -2.f, 1.f, 0.f, 0.f, s));       // H^T
  POETX_TRY(block_mm(dG, false, T1, Sb, Hb, 1.f, 1.f, nb, b, s));                   // Sbar
  POETX_TRY(combine(T1, nullptr, Sb, nullptr, nb, b, 0.f, 0.f, 1.f, 1.f, 0.f, s));  // Z
  POETX_TRY(combine(Hb, nullptr, Hb, dG, nb, b, 0.f, 0.f, 2.f, 0.f, 2.f, s));       // 2dG + 2Hbar
  POETX_TRY(block_mm(T1, false, Qm, Sb, Hb, -1.f, 1.f, nb, b, s));                  // U
  TraceScope t("cnp_pack_dq", s);
  pack_skew_kernel<<<grid_for(nb * b * b), 256, 0, s>>>(Sb, dq, nb, b);
  return cudaGetLastError();
}

cudaError_t f32_to_bf16(const float* in, __nv_bfloat16* out, int64_t count, cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  TraceScope t("f32_to_bf16", s);
  f32_to_bf16_kernel<<<grid_for(count), 256, 0, s>>>(in, out, count);
  return cudaGetLastError();
}

cudaError_t fill_zero_f32(float* p, int64_t count, cudaStream_t s) {
  return cudaMemsetAsync(p, 0, (size_t)count * sizeof(float), s);
}

}  // namespace poetx
