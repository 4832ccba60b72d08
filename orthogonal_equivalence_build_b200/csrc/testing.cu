// Kernel-level test hook (include/poetx_testing.h): one plain product on the tcgen05 kernel.
#include "../../include/poetx_testing.h"
#include "umma_gemm.h"

extern "C" poetx_status poetx_testing_gemm_bf16(const void* A, int64_t a_rows, int64_t a_cols,
                                                int32_t a_mn, const void* B, int64_t b_rows,
                                                int64_t b_cols, int32_t b_mn, int64_t M,
                                                int64_t N, int64_t K, void* C, int32_t c_f32,
                                                int64_t ldc, int32_t splits, int32_t variant,
                                                uint64_t epi_wait_ns, void* stream) {
  using namespace poetx;
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0 || splits < 1) {
    set_error("testing_gemm: bad arguments");
    return POETX_ERR_INVALID_ARG;
  }
  if (splits > 1 && !c_f32) {
    set_error("testing_gemm: split partials must be fp32");
    return POETX_ERR_INVALID_ARG;
  }
  if (umma::effective_splits(K, splits) != splits) {
    set_error("testing_gemm: %d K ranges do not split %lld K blocks evenly", (int)splits,
              (long long)((K + 63) / 64));
    return POETX_ERR_INVALID_ARG;
  }
  umma::Gemm g;
  g.M = M; g.N = N; g.K = K; g.splits = splits;
  g.A = A; g.a_rows = a_rows; g.a_cols = a_cols; g.a_ld = a_cols; g.a_mn = a_mn != 0;
  g.B = B; g.b_rows = b_rows; g.b_cols = b_cols; g.b_ld = b_cols; g.b_mn = b_mn != 0;
  g.C = C; g.out_f32 = c_f32 != 0; g.ldc = ldc; g.c_split = M * ldc;
  g.name = "umma_testing_gemm";
  g.epi_wait_ns = epi_wait_ns;
  const bool pair = variant == 1;
  const bool wide = variant == 2 || variant == 3;
  g.wide_collect = variant == 2;
  if (!umma::supported(g) || (g.a_mn && g.b_mn && !g.out_f32) || (g.a_mn && !g.b_mn) ||
      (pair && !umma::pair_supported(g)) || (wide && !umma::wide_supported(g)) || variant < 0 ||
      variant > 3) {
    set_error("testing_gemm: shape/layout not covered by the tensor-core kernel");
    return POETX_ERR_UNSUPPORTED;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = wide ? umma::gemm_wide(g, s) : pair ? umma::gemm_pair(g, s) : umma::gemm(g, s);
  if (e != cudaSuccess) {
    set_error("testing_gemm: %s", cudaGetErrorString(e));
    return POETX_ERR_CUDA;
  }
  return POETX_OK;
}
