// Batched, strided SIMT GEMM with fp32 accumulation.
//
// Serves the fp32 layer (fp32 operands: tensor-core tf32 would not hold the fp32 tolerance) and
// small block sizes that the tensor-core path does not tile. Operands may be fp32 or bf16,
// addressed through arbitrary row/column/batch strides so transposed operands cost nothing.
// Tile 64 x 64 x 16, 256 threads, 4 x 4 outputs per thread.
#include "internal.h"

namespace poetx {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <DT T>
__device__ __forceinline__ float ld(const void* p, int64_t idx) {
  if constexpr (T == DT::F32) return static_cast<const float*>(p)[idx];
  else return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[idx]);
}

template <DT TA, DT TB, DT TC>
__global__ void __launch_bounds__(NT) simt_gemm_kernel(SimtGemm g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int64_t z = blockIdx.z;
  const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t a_base = z * g.a_bs, b_base = z * g.b_bs;
  // choose the loop order that walks the unit-stride dimension with consecutive threads
  const bool a_k_fast = (g.a_cs == 1);
  const bool b_n_fast = (g.b_cs == 1);
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < g.K; k0 += BK) {
    for (int e = tid; e < BM * BK; e += NT) {
      int r, kk;
      if (a_k_fast) { r = e / BK; kk = e % BK; } else { r = e % BM; kk = e / BM; }
      const int64_t gi = m0 + r, gk = k0 + kk;
      As[kk][r] = (gi < g.M && gk < g.K) ? ld<TA>(g.A, a_base + gi * g.a_rs + gk * g.a_cs) : 0.f;
    }
    for (int e = tid; e < BN * BK; e += NT) {
      int c, kk;
      if (b_n_fast) { c = e % BN; kk = e / BN; } else { c = e / BK; kk = e % BK; }
      const int64_t gj = n0 + c, gk = k0 + kk;
      Bs[kk][c] = (gj < g.N && gk < g.K) ? ld<TB>(g.B, b_base + gk * g.b_rs + gj * g.b_cs) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gi = m0 + ty * 4 + i;
    if (gi >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t gj = n0 + tx * 4 + j;
      if (gj >= g.N) continue;
      float v = g.alpha * acc[i][j];
      if (g.D) v += g.beta * g.D[z * g.d_bs + gi * g.d_rs + gj];
      if (gi == gj) v += g.diag;
      const int64_t ci = z * g.c_bs + gi * g.c_rs + gj;
      if constexpr (TC == DT::F32) static_cast<float*>(g.C)[ci] = v;
      else static_cast<__nv_bfloat16*>(g.C)[ci] = __float2bfloat16_rn(v);
    }
  }
}

template <DT TA, DT TB, DT TC>
cudaError_t launch(const SimtGemm& g, cudaStream_t s) {
  dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM), (unsigned)g.batch);
  // bf16 operands reach this kernel only for shapes the tensor-core tiling does not cover
  // (b < 64 or not a multiple of 64): a distinct name makes that slower path visible in the
  // library's trace and in profiler ranges.
  TraceScope t(TA == DT::BF16 ? "simt_gemm_bf16_fallback" : "simt_gemm_f32", s);
  simt_gemm_kernel<TA, TB, TC><<<grid, NT, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t simt_gemm(const SimtGemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return cudaSuccess;
  if (g.M > 65535ll * BM || g.batch > 65535) return cudaErrorInvalidValue;
#define POETX_SG(a, b, c)                                                \
  if (g.a_t == DT::a && g.b_t == DT::b && g.c_t == DT::c) return launch<DT::a, DT::b, DT::c>(g, s);
  POETX_SG(F32, F32, F32)
  POETX_SG(BF16, BF16, BF16)
  POETX_SG(BF16, BF16, F32)
  POETX_SG(F32, F32, BF16)
#undef POETX_SG
  return cudaErrorInvalidValue;
}

}  // namespace poetx
