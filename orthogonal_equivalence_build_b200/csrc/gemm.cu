// Routing of the layer's contractions: bf16 operands go to the tcgen05 kernel (umma_gemm.cu)
// whenever its tiling fits the shape; fp32 operands (and bf16 shapes the tensor-core tiling does
// not cover, e.g. b < 64) go to the SIMT kernel.
#include "gemm.h"

#include <algorithm>

#include "umma_gemm.h"

namespace poetx {
namespace {

int sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

__global__ void sum_partials_kernel(const float* __restrict__ part, float* __restrict__ out,
                                    int64_t count, int splits) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += part[(int64_t)s * count + e];
    out[e] = v;
  }
}

// CTA-pair tiles where the shape allows (256 x 256 per pair), single-CTA tiles otherwise.
cudaError_t run(const umma::Gemm& g, cudaStream_t s) {
  if (umma::pair_supported(g)) return umma::gemm_pair(g, s);
  return umma::gemm(g, s);
}

// The dense W0' products: 256 x 512 pair tiles where N allows (every workload's m and n are
// multiples of 512), else as above.
cudaError_t run_dense(const umma::Gemm& g, cudaStream_t s) {
  if (umma::wide_supported(g)) return umma::gemm_wide(g, s);
  return run(g, s);
}

}  // namespace

namespace {
// The per-block gradients run on 256 x 512 pair tiles where b is a multiple of 512 (one tile per
// 256 rows of a block), on 256 x 256 pair tiles where b % 256 == 0, else on single-CTA tiles.
bool dg_wide(int64_t b) { return b % 512 == 0; }
// CTAs that one split of one block occupies
int64_t dg_ctas_per_block(int64_t b) {
  if (dg_wide(b)) return (b / 256) * (b / 512) * 2;
  return ((b + 127) / 128) * std::max<int64_t>(1, b / 256);
}
}  // namespace

cudaError_t sum_partials(const float* part, float* out, int64_t count, int splits,
                         cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  TraceScope tr("sum_split_partials", s);
  sum_partials_kernel<<<(int)std::min<int64_t>((count + 255) / 256, sms() * 8), 256, 0, s>>>(
      part, out, count, splits);
  return cudaGetLastError();
}

int grad_splits(int64_t nb, int64_t b, int64_t rows) {
  // Split the contraction over tokens (each split keeps >= 512 token rows) where that shortens
  // the launch: a time model over the split count s,
  //   waves(s) x (64-row K blocks per split) x (one K block of one CTA's tile)
  //   + the fp32 partial products' traffic (each split's b x b blocks written, then read back
  //     by the sum; one range writes dG once),
  // at the per-SM share of the bf16 peak and ~6 TB/s. More splits fill more of the last wave
  // but every extra range costs 2 nb b^2 4 bytes of HBM traffic.
  const int64_t ctas = nb * dg_ctas_per_block(b);
  const int64_t n_sm = sms();
  const double kb_us = (double)(b * b / dg_ctas_per_block(b)) * 64.0 * 2.0 / 11.0e6;
  const double part_us = (double)nb * (double)(b * b) * 4.0 / 6.0e6;
  const int64_t max_s = std::max<int64_t>(1, std::min<int64_t>(16, rows / 512));
  int best = 1;
  double best_t = 0.0;
  for (int64_t s = 1; s <= max_s; ++s) {
    const int64_t waves = (ctas * s + n_sm - 1) / n_sm;
    const int64_t kblocks = ((rows + s - 1) / s + 63) / 64;
    const double t = (double)(waves * kblocks) * kb_us + (s == 1 ? 1.0 : 2.0 * (double)s) * part_us;
    if (s == 1 || t < best_t * 0.98) { best_t = t; best = (int)s; }
  }
  return best;
}

cudaError_t gemm_blockwise(DT t, const void* A, const void* G, void* C, int64_t rows,
                           int64_t width, int64_t b, bool transpose_g, cudaStream_t s) {
  if (t == DT::BF16) {
    umma::Gemm g;
    g.M = rows; g.N = b; g.K = b; g.groups = width / b;
    g.A = A; g.a_rows = rows; g.a_cols = width; g.a_ld = width; g.a_mn = false;
    g.a_gm = 0; g.a_gk = b;
    g.B = G; g.b_rows = width; g.b_cols = b; g.b_ld = b;
    if (transpose_g) { g.b_mn = false; g.b_gn = b; g.b_gk = 0; }   // B(k, j) = G[j][k]
    else { g.b_mn = true; g.b_gn = 0; g.b_gk = b; }                // B(k, j) = G[k][j]
    g.C = C; g.ldc = width; g.c_gs = b;
    g.name = transpose_g ? "umma_blockwise_T" : "umma_blockwise";
    if (umma::supported(g)) return run(g, s);
  }
  SimtGemm g{};
  g.M = rows; g.N = b; g.K = b; g.batch = width / b;
  g.A = A; g.a_t = t; g.a_rs = width; g.a_cs = 1; g.a_bs = b;
  g.B = G; g.b_t = t; g.b_bs = b * b;
  g.b_rs = transpose_g ? 1 : b; g.b_cs = transpose_g ? b : 1;
  g.C = C; g.c_t = t; g.c_rs = width; g.c_bs = b;
  g.alpha = 1.f;
  return simt_gemm(g, s);
}

cudaError_t gemm_blockwise_left(DT t, const void* G, const void* N, void* C, int64_t m,
                                int64_t n, int64_t b, cudaStream_t s) {
  if (t == DT::BF16) {
    umma::Gemm g;
    g.M = b; g.N = n; g.K = b; g.groups = m / b;
    g.A = G; g.a_rows = m; g.a_cols = b; g.a_ld = b; g.a_mn = false; g.a_gm = b; g.a_gk = 0;
    g.B = N; g.b_rows = m; g.b_cols = n; g.b_ld = n; g.b_mn = true; g.b_gn = 0; g.b_gk = b;
    g.C = C; g.ldc = n; g.c_gs = b * n;
    g.name = "umma_blockwise_left";
    if (b % 128 == 0 && umma::supported(g)) return run(g, s);
  }
  SimtGemm g{};
  g.M = b; g.N = n; g.K = b; g.batch = m / b;
  g.A = G; g.a_t = t; g.a_rs = b; g.a_cs = 1; g.a_bs = b * b;
  g.B = N; g.b_t = t; g.b_rs = n; g.b_cs = 1; g.b_bs = b * n;
  g.C = C; g.c_t = t; g.c_rs = n; g.c_bs = b * n;
  g.alpha = 1.f;
  return simt_gemm(g, s);
}

cudaError_t gemm_dense(DT t, const void* A, const void* W, void* C, int64_t M, int64_t N,
                       int64_t K, bool w_trans, cudaStream_t s) {
  if (t == DT::BF16) {
    umma::Gemm g;
    g.M = M; g.N = N; g.K = K;
    g.A = A; g.a_rows = M; g.a_cols = K; g.a_ld = K; g.a_mn = false;
    g.B = W;
    if (w_trans) { g.b_rows = N; g.b_cols = K; g.b_ld = K; g.b_mn = false; }
    else { g.b_rows = K; g.b_cols = N; g.b_ld = N; g.b_mn = true; }
    g.C = C; g.ldc = N;
    g.name = w_trans ? "umma_dense_W0T" : "umma_dense_W0";
    if (umma::supported(g)) return run_dense(g, s);
  }
  SimtGemm g{};
  g.M = M; g.N = N; g.K = K; g.batch = 1;
  g.A = A; g.a_t = t; g.a_rs = K; g.a_cs = 1;
  g.B = W; g.b_t = t;
  g.b_rs = w_trans ? 1 : N; g.b_cs = w_trans ? K : 1;
  g.C = C; g.c_t = t; g.c_rs = N;
  g.alpha = 1.f;
  return simt_gemm(g, s);
}

bool dense_i8_fused(int64_t M, int64_t N) { return M >= 256 && N % 256 == 0; }

cudaError_t gemm_dense_i8(const void* A, const int8_t* Wq, const float* scale, void* C, int64_t M,
                          int64_t N, int64_t K, bool w_trans, void* deq_ws, cudaStream_t s) {
  if (dense_i8_fused(M, N)) {
    umma::Gemm g;
    g.M = M; g.N = N; g.K = K;
    g.A = A; g.a_rows = M; g.a_cols = K; g.a_ld = K; g.a_mn = false;
    g.B = Wq; g.b_i8 = true; g.b_scale = scale;
    if (w_trans) { g.b_rows = N; g.b_cols = K; g.b_ld = K; g.b_mn = false; }
    else { g.b_rows = K; g.b_cols = N; g.b_ld = N; g.b_mn = true; }
    g.C = C; g.ldc = N;
    g.name = w_trans ? "umma_dense_W0T_i8" : "umma_dense_W0_i8";
    if (!umma::pair_supported(g)) return cudaErrorNotSupported;
    return umma::gemm_pair(g, s);
  }
  if (!deq_ws) return cudaErrorInvalidValue;
  auto* W = static_cast<__nv_bfloat16*>(deq_ws);
  const int64_t rows = w_trans ? N : K, cols = w_trans ? K : N;
  cudaError_t e = dequantize_cols_i8(Wq, scale, rows, cols, W, s);
  if (e != cudaSuccess) return e;
  return gemm_dense(DT::BF16, A, W, C, M, N, K, w_trans, s);
}

bool w0_p_fused_supported(const void* A1, const void* W0, const void* Gp, const void* Bout,
                          const void* Cout, int64_t T, int64_t m, int64_t n, int64_t b) {
  return umma::w0p_fused_supported(A1, W0, Gp, Bout, Cout, T, m, n, b);
}

cudaError_t gemm_w0_p_fused(const void* A1, const void* W0, const void* Gp, void* Bout,
                            void* Cout, int64_t T, int64_t m, int64_t n, int64_t b,
                            cudaStream_t s) {
  return umma::w0p_fused(A1, W0, Gp, Bout, Cout, T, m, n, b, s);
}

size_t block_grad_ws_bytes(DT t, int64_t width, int64_t b, int64_t rows) {
  if (t != DT::BF16) return 0;
  const int sp = umma::effective_splits(rows, grad_splits(width / b, b, rows));
  return sp > 1 ? (size_t)sp * (size_t)(width * b) * sizeof(float) : 0;
}

cudaError_t gemm_block_grad(DT t, const void* A, const void* B, float* dG, int64_t rows,
                            int64_t width, int64_t b, void* partials, int* splits_used,
                            cudaStream_t s) {
  *splits_used = 1;
  if (rows == 0) return cudaMemsetAsync(dG, 0, (size_t)(width * b) * sizeof(float), s);
  if (t == DT::BF16) {
    const int sp = umma::effective_splits(rows, grad_splits(width / b, b, rows));
    umma::Gemm g;
    g.M = b; g.N = b; g.K = rows; g.groups = width / b; g.splits = sp;
    g.A = A; g.a_rows = rows; g.a_cols = width; g.a_ld = width; g.a_mn = true;
    g.a_gm = b; g.a_gk = 0;
    g.B = B; g.b_rows = rows; g.b_cols = width; g.b_ld = width; g.b_mn = true;
    g.b_gn = b; g.b_gk = 0;
    g.out_f32 = true; g.ldc = b; g.c_gs = b * b; g.c_split = width * b;
    g.C = sp > 1 ? partials : dG;
    g.name = "umma_block_grad";
    if (b % 128 == 0 && umma::supported(g) && (sp == 1 || partials)) {
      *splits_used = sp;
      if (dg_wide(b) && umma::wide_supported(g)) return umma::gemm_wide(g, s);
      return run(g, s);
    }
  }
  SimtGemm g{};
  g.M = b; g.N = b; g.K = rows; g.batch = width / b;
  g.A = A; g.a_t = t; g.a_rs = 1; g.a_cs = width; g.a_bs = b;
  g.B = B; g.b_t = t; g.b_rs = width; g.b_cs = 1; g.b_bs = b;
  g.C = dG; g.c_t = DT::F32; g.c_rs = b; g.c_bs = b * b;
  g.alpha = 1.f;
  return simt_gemm(g, s);
}

namespace {
umma::Gemm block_grad2_gemm(const void* A1, const void* B1, int64_t w1, const void* A2,
                            const void* B2, int64_t w2, int64_t rows, int64_t b, int sp) {
  umma::Gemm g;
  g.M = b; g.N = b; g.K = rows; g.groups = (w1 + w2) / b; g.splits = sp;
  g.groups_1 = w1 / b;
  g.A = A1; g.a_rows = rows; g.a_cols = w1; g.a_ld = w1; g.a_mn = true;
  g.B = B1; g.b_rows = rows; g.b_cols = w1; g.b_ld = w1; g.b_mn = true;
  g.A2 = A2; g.a2_rows = rows; g.a2_cols = w2; g.a2_ld = w2;
  g.B2 = B2; g.b2_rows = rows; g.b2_cols = w2; g.b2_ld = w2;
  g.a_gm = b; g.a_gk = 0; g.b_gn = b; g.b_gk = 0;
  g.out_f32 = true; g.ldc = b; g.c_gs = b * b; g.c_split = (w1 + w2) * b;
  g.name = "umma_block_grad";
  return g;
}
int block_grad2_splits(int64_t w1, int64_t w2, int64_t b, int64_t rows) {
  return umma::effective_splits(rows, grad_splits((w1 + w2) / b, b, rows));
}
}  // namespace

size_t block_grad2_ws_bytes(DT t, int64_t w1, int64_t w2, int64_t b, int64_t rows) {
  if (t != DT::BF16 || b % 256 != 0) return 0;
  const int sp = block_grad2_splits(w1, w2, b, rows);
  return sp > 1 ? (size_t)sp * (size_t)((w1 + w2) * b) * sizeof(float) : 0;
}

cudaError_t gemm_block_grad2(DT t, const void* A1, const void* B1, int64_t w1, const void* A2,
                             const void* B2, int64_t w2, float* dG, int64_t rows, int64_t b,
                             void* partials, int* splits_used, cudaStream_t s) {
  *splits_used = 1;
  if (t != DT::BF16 || rows == 0 || b % 256 != 0) return cudaErrorNotSupported;
  const int sp = block_grad2_splits(w1, w2, b, rows);
  if (sp > 1 && !partials) return cudaErrorNotSupported;
  umma::Gemm g = block_grad2_gemm(A1, B1, w1, A2, B2, w2, rows, b, sp);
  g.C = sp > 1 ? partials : dG;
  if (dg_wide(b) && umma::wide_supported(g)) {
    *splits_used = sp;
    return umma::gemm_wide(g, s);
  }
  if (!umma::pair_supported(g)) return cudaErrorNotSupported;
  *splits_used = sp;
  return umma::gemm_pair(g, s);
}

size_t gemm_cnp_ws_bytes(int64_t nb, int64_t b) {
  return tc_blocks_supported(b) ? cnp_tc_ws_bytes(nb, b) : cnp_ws_bytes(nb, b);
}

cudaError_t gemm_cnp_build(const float* q, int64_t nb, int64_t b, float* g, __nv_bfloat16* g_lp,
                           void* ws, cudaStream_t s) {
  if (tc_blocks_supported(b)) {
    BlockRuns r;
    r.q[0] = q; r.g[0] = g; r.g_lp[0] = g_lp; r.nb[0] = (int)nb;
    return cnp_build_tc(r, b, ws, s);
  }
  return cnp_build(q, nb, b, g, g_lp, ws, s);
}

cudaError_t gemm_cnp_build_runs(const BlockRuns& r, int64_t b, void* ws, cudaStream_t s) {
  if (tc_blocks_supported(b)) return cnp_build_tc(r, b, ws, s);
  for (int k = 0; k < kMaxRuns; ++k) {
    if (!r.nb[k]) continue;
    cudaError_t e = cnp_build(r.q[k], r.nb[k], b, r.g[k], r.g_lp[k], ws, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

size_t gemm_dq_ws_bytes(DT t, int64_t nb, int64_t b) {
  return (t == DT::BF16 && tc_blocks_supported(b)) ? dq_tc_ws_bytes(nb, b) : dq_ws_bytes(nb, b);
}

cudaError_t gemm_dq_from_dg_runs(DT t, const BlockRuns& r, int64_t b, float* dG, void* ws,
                                 cudaStream_t s) {
  if (t == DT::BF16 && tc_blocks_supported(b)) return dq_from_dg_tc(r, b, dG, ws, s);
  // fp32 layers: per run, sum split partials if any, then the fp32 SIMT chain
  float* dGk = dG;
  for (int k = 0; k < kMaxRuns; ++k) {
    if (!r.nb[k]) continue;
    const int64_t count = (int64_t)r.nb[k] * b * b;
    const float* src = r.parts[k];
    if (r.splits[k] > 1 || src != dGk) {
      TraceScope tr("sum_split_partials", s);
      sum_partials_kernel<<<(int)std::min<int64_t>((count + 255) / 256, sms() * 8), 256, 0, s>>>(
          src, dGk, count, r.splits[k]);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    cudaError_t e = dq_from_dg(r.q[k], dGk, r.nb[k], b, r.dq[k], ws, s);
    if (e != cudaSuccess) return e;
    dGk += count;
  }
  return cudaSuccess;
}

}  // namespace poetx
