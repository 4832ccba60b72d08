// Cayley-Neumann blocks and their gradient on the tensor cores (block size b a multiple of 128).
//
// CNP ("POET-X" blog §第四斧 item 2; "Reparameterized LLM Training ..." §2 CNP, k = 3), evaluated
// as G = (I + 2Q) + S H with S = Q Q and H = 2I + 2Q + S: two b x b products per block, on the
// bf16 tcgen05 kernel with fp32 accumulation. Each fp32 operand x is split into
// x_hi = bf16(x) and x_lo = bf16(x - x_hi); x y is taken as x_hi y_hi + x_hi y_lo + x_lo y_hi,
// i.e. ONE GEMM with the contraction tripled over concatenated operands
//     [x_hi | x_hi | x_lo] . [y_hi ; y_lo ; y_hi],
// which keeps about 16 significant bits per product (the dropped x_lo y_lo is ~2^-16 relative):
// fp32-class G for the 1e-5 bar.
//
// Gradient, for bf16 layers (tolerance 1e-2): with Hbar = S dG, Sbar = dG (2I - 2Q + S) + Hbar,
// Z = Sbar + Sbar^T, U = 2 dG + 2 Hbar - Z Q, dq_ij = U_ij - U_ji (i < j). The four products
// S = QQ, S dG, dG (S - 2Q) and Z Q run single-pass bf16 with fp32 accumulation; the exact
// 2 dG terms are added in fp32.
#include "gemm.h"
#include "umma_gemm.h"

#include <algorithm>

namespace poetx {
namespace {

__device__ __forceinline__ int64_t triu_index(int64_t i, int64_t j, int64_t b) {
  return i * b - i * (i + 1) / 2 + (j - i - 1);
}
__device__ __forceinline__ float skew_entry(const float* __restrict__ qb, int64_t i, int64_t j,
                                            int64_t b) {
  if (i < j) return qb[triu_index(i, j, b)];
  if (i > j) return -qb[triu_index(j, i, b)];
  return 0.f;
}
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

int grid_for(int64_t n) {
  return (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 16));
}

// Concatenated split operands of one product X Y per block:
//   Acat [nb*b][3b] row (g, i) = [Xhi(i, :) | Xhi(i, :) | Xlo(i, :)]
//   Bcat [nb*3b][b] rows (g, k') = Yhi (k' < b), Ylo (b <= k' < 2b), Yhi (2b <= k')
// X and Y are given elementwise: mode 0: X = Y = Q(q);  mode 1: X = S, Y = 2I + 2Q(q) + S.
__global__ void split_operands_kernel(const float* __restrict__ q, const float* __restrict__ S,
                                      int64_t nb, int64_t b, int mode,
                                      __nv_bfloat16* __restrict__ Acat,
                                      __nv_bfloat16* __restrict__ Bcat) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = e / bb, r = e - g * bb, i = r / b, j = r - i * b;
    const float qv = skew_entry(q + g * qs, i, j, b);
    float x, y;
    if (mode == 0) {
      x = qv;
      y = qv;
    } else {
      const float s = S[e];
      x = s;
      y = ((i == j) ? 2.f : 0.f) + 2.f * qv + s;
    }
    __nv_bfloat16 xh, xl, yh, yl;
    split_bf16(x, xh, xl);
    split_bf16(y, yh, yl);
    __nv_bfloat16* arow = Acat + (g * b + i) * 3 * b;
    arow[j] = xh;
    arow[b + j] = xh;
    arow[2 * b + j] = xl;
    __nv_bfloat16* bblk = Bcat + g * 3 * bb;
    bblk[i * b + j] = yh;
    bblk[bb + i * b + j] = yl;
    bblk[2 * bb + i * b + j] = yh;
  }
}

// G = I + 2Q + P, and its bf16 copy.
__global__ void cnp_finish_kernel(const float* __restrict__ q, const float* __restrict__ P,
                                  int64_t nb, int64_t b, float* __restrict__ g,
                                  __nv_bfloat16* __restrict__ g_lp) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    const float v = ((i == j) ? 1.f : 0.f) + 2.f * skew_entry(q + blk * qs, i, j, b) + P[e];
    if (g) g[e] = v;
    if (g_lp) g_lp[e] = __float2bfloat16_rn(v);
  }
}

// bf16 Q and dG for the gradient chain.
__global__ void dq_prep_kernel(const float* __restrict__ q, const float* __restrict__ dG,
                               int64_t nb, int64_t b, __nv_bfloat16* __restrict__ Qh,
                               __nv_bfloat16* __restrict__ dGh) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    Qh[e] = __float2bfloat16_rn(skew_entry(q + blk * qs, i, j, b));
    dGh[e] = __float2bfloat16_rn(dG[e]);
  }
}

// Sh = bf16(S), SmQ = bf16(S - 2Q)
__global__ void dq_prep2_kernel(const float* __restrict__ q, const float* __restrict__ S,
                                int64_t nb, int64_t b, __nv_bfloat16* __restrict__ Sh,
                                __nv_bfloat16* __restrict__ SmQ) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    const float s = S[e];
    Sh[e] = __float2bfloat16_rn(s);
    SmQ[e] = __float2bfloat16_rn(s - 2.f * skew_entry(q + blk * qs, i, j, b));
  }
}

// Sbar = 2dG + T1 + Hb;  Zh = bf16(Sbar + Sbar^T);  V = 2dG + 2Hb (written over S)
__global__ void dq_mid_kernel(const float* __restrict__ dG, const float* __restrict__ T1,
                              const float* __restrict__ Hb, int64_t nb, int64_t b,
                              __nv_bfloat16* __restrict__ Zh, float* __restrict__ V) {
  const int64_t bb = b * b, total = nb * bb;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    const int64_t et = blk * bb + j * b + i;
    const float sb = 2.f * dG[e] + T1[e] + Hb[e];
    const float sbt = 2.f * dG[et] + T1[et] + Hb[et];
    Zh[e] = __float2bfloat16_rn(sb + sbt);
    V[e] = 2.f * dG[e] + 2.f * Hb[e];
  }
}

// dq_ij = (V_ij - ZQ_ij) - (V_ji - ZQ_ji), i < j
__global__ void dq_pack_kernel(const float* __restrict__ V, const float* __restrict__ ZQ,
                               int64_t nb, int64_t b, float* __restrict__ dq) {
  const int64_t bb = b * b, total = nb * bb, qs = b * (b - 1) / 2;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blk = e / bb, r = e - blk * bb, i = r / b, j = r - i * b;
    if (i < j) {
      const int64_t et = blk * bb + j * b + i;
      dq[blk * qs + triu_index(i, j, b)] = (V[e] - ZQ[e]) - (V[et] - ZQ[et]);
    }
  }
}

// C_g = X_g Y_g for nb blocks of b x b (fp32 out), X K-major [nb*b][kx] (kx = K), Y MN-major
// [nb*K][b]. K = b (single pass) or 3b (split operands).
cudaError_t block_product(const void* X, const void* Y, float* C, int64_t nb, int64_t b,
                          int64_t K, const char* name, cudaStream_t s) {
  umma::Gemm g;
  g.M = b; g.N = b; g.K = K; g.groups = nb;
  g.A = X; g.a_rows = nb * b; g.a_cols = K; g.a_ld = K; g.a_mn = false; g.a_gm = b; g.a_gk = 0;
  g.B = Y; g.b_rows = nb * K; g.b_cols = b; g.b_ld = b; g.b_mn = true; g.b_gn = 0; g.b_gk = K;
  g.C = C; g.out_f32 = true; g.ldc = b; g.c_gs = b * b;
  g.name = name;
  if (!umma::supported(g)) return cudaErrorNotSupported;
  return umma::gemm(g, s);
}

#define POETX_TRY(x)                  \
  do {                                \
    cudaError_t e_ = (x);             \
    if (e_ != cudaSuccess) return e_; \
  } while (0)

}  // namespace

bool tc_blocks_supported(int64_t b) { return b % 128 == 0 && b >= 128; }

size_t cnp_tc_ws_bytes(int64_t nb, int64_t b) {
  const size_t cat = align_up((size_t)(nb * b * 3 * b) * 2, 256);
  const size_t f = align_up((size_t)(nb * b * b) * 4, 256);
  return 2 * cat + 2 * f;
}

cudaError_t cnp_build_tc(const float* q, int64_t nb, int64_t b, float* g, __nv_bfloat16* g_lp,
                         void* ws, cudaStream_t s) {
  if (nb == 0) return cudaSuccess;
  Arena a(ws, cnp_tc_ws_bytes(nb, b));
  auto* Acat = static_cast<__nv_bfloat16*>(a.take((size_t)(nb * b * 3 * b) * 2));
  auto* Bcat = static_cast<__nv_bfloat16*>(a.take((size_t)(nb * b * 3 * b) * 2));
  auto* S = static_cast<float*>(a.take((size_t)(nb * b * b) * 4));
  auto* P = static_cast<float*>(a.take((size_t)(nb * b * b) * 4));
  const int grid = grid_for(nb * b * b);
  {
    TraceScope t("cnp_split_Q", s);
    split_operands_kernel<<<grid, 256, 0, s>>>(q, nullptr, nb, b, 0, Acat, Bcat);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Acat, Bcat, S, nb, b, 3 * b, "umma_cnp_QQ", s));
  {
    TraceScope t("cnp_split_SH", s);
    split_operands_kernel<<<grid, 256, 0, s>>>(q, S, nb, b, 1, Acat, Bcat);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Acat, Bcat, P, nb, b, 3 * b, "umma_cnp_SH", s));
  TraceScope t("cnp_finish", s);
  cnp_finish_kernel<<<grid, 256, 0, s>>>(q, P, nb, b, g, g_lp);
  return cudaGetLastError();
}

size_t dq_tc_ws_bytes(int64_t nb, int64_t b) {
  const size_t h = align_up((size_t)(nb * b * b) * 2, 256);
  const size_t f = align_up((size_t)(nb * b * b) * 4, 256);
  return 5 * h + 3 * f;
}

cudaError_t dq_from_dg_tc(const float* q, const float* dG, int64_t nb, int64_t b, float* dq,
                          void* ws, cudaStream_t s) {
  if (nb == 0) return cudaSuccess;
  Arena a(ws, dq_tc_ws_bytes(nb, b));
  const size_t hb = (size_t)(nb * b * b) * 2, fb = (size_t)(nb * b * b) * 4;
  auto* Qh = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* dGh = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* Sh = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* SmQ = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* Zh = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* S = static_cast<float*>(a.take(fb));
  auto* Hb = static_cast<float*>(a.take(fb));
  auto* T1 = static_cast<float*>(a.take(fb));
  const int grid = grid_for(nb * b * b);
  {
    TraceScope t("dq_prep", s);
    dq_prep_kernel<<<grid, 256, 0, s>>>(q, dG, nb, b, Qh, dGh);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Qh, Qh, S, nb, b, b, "umma_dq_QQ", s));
  {
    TraceScope t("dq_prep2", s);
    dq_prep2_kernel<<<grid, 256, 0, s>>>(q, S, nb, b, Sh, SmQ);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Sh, dGh, Hb, nb, b, b, "umma_dq_SdG", s));
  POETX_TRY(block_product(dGh, SmQ, T1, nb, b, b, "umma_dq_dGH", s));
  {
    TraceScope t("dq_mid", s);
    dq_mid_kernel<<<grid, 256, 0, s>>>(dG, T1, Hb, nb, b, Zh, S);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Zh, Qh, T1, nb, b, b, "umma_dq_ZQ", s));
  TraceScope t("dq_pack", s);
  dq_pack_kernel<<<grid, 256, 0, s>>>(S, T1, nb, b, dq);
  return cudaGetLastError();
}

}  // namespace poetx
