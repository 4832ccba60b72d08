// 8-bit storage of the merged weight ("POET-XQ": only low-precision weights are stored and
// dequantised on demand — "[Project POET-X] Scaling Orthogonal Equivalence ..." §Quantized
// Training (POET-XQ); "POET-X: Memory-efficient LLM Training ..." (gist.science) §Resumo técnico
// 2 Metodologia). The pages give no format; this library stores symmetric int8 codes with one
// fp32 scale per column of W0' [m, n] (one per output feature):
//   s_j = max_i |W0'[i, j]| / 127,  q_ij = round_half_even(W0'[i, j] / s_j) in [-127, 127],
//   s_j = 0 and q_.j = 0 for an all-zero column;
// and computes with bf16(q_ij * s_j). Divisions and the product are IEEE round-to-nearest fp32
// (__fdiv_rn / __fmul_rn), so codes and dequantised values are reproducible bit for bit.
#include "internal.h"

namespace poetx {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int kColThreads = 256;
constexpr int kRowsPerSlab = 64;

// amax_bits[j] = max over a slab of rows of |w[i, j]| as fp32 bits (non-negative floats order
// like their bit patterns, so an integer atomicMax is exact and order-independent).
template <typename T>
__global__ void __launch_bounds__(kColThreads)
col_absmax_kernel(const T* __restrict__ w, int64_t m, int64_t n, unsigned* __restrict__ amax_bits) {
  const int64_t j = (int64_t)blockIdx.x * kColThreads + threadIdx.x;
  if (j >= n) return;
  const int64_t i0 = (int64_t)blockIdx.y * kRowsPerSlab;
  const int64_t i1 = i0 + kRowsPerSlab < m ? i0 + kRowsPerSlab : m;
  float mx = 0.f;
  for (int64_t i = i0; i < i1; ++i) mx = fmaxf(mx, fabsf(to_f(w[i * n + j])));
  atomicMax(amax_bits + j, __float_as_uint(mx));
}

__device__ __forceinline__ int8_t quant_code(float v, float s) {
  if (!(s > 0.f)) return 0;
  const int q = __float2int_rn(__fdiv_rn(v, s));
  return (int8_t)(q > 127 ? 127 : (q < -127 ? -127 : q));
}

// q[i, j] from the column maxima (read as fp32 bits); 4 consecutive elements per thread.
template <typename T>
__global__ void quantize_kernel(const T* __restrict__ w, int64_t m, int64_t n,
                                const unsigned* __restrict__ amax_bits, int8_t* __restrict__ q) {
  const int64_t total = m * n;
  for (int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; e < total;
       e += (int64_t)gridDim.x * blockDim.x * 4) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t idx = e + k;
      if (idx < total) {
        const int64_t j = idx % n;
        const float s = __fdiv_rn(__uint_as_float(amax_bits[j]), 127.f);
        q[idx] = quant_code(to_f(w[idx]), s);
      }
    }
  }
}

// scale[j] = amax[j] / 127, in place over the bits the maxima were gathered in.
__global__ void finalize_scale_kernel(unsigned* __restrict__ bits, int64_t n) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j < n) {
    const float s = __fdiv_rn(__uint_as_float(bits[j]), 127.f);
    bits[j] = __float_as_uint(s);
  }
}

__global__ void dequantize_kernel(const int8_t* __restrict__ q, const float* __restrict__ scale,
                                  int64_t m, int64_t n, __nv_bfloat16* __restrict__ out) {
  const int64_t total = m * n;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = e % n;
    out[e] = __float2bfloat16_rn(__fmul_rn((float)q[e], scale[j]));
  }
}

// The same values, 16 consecutive codes of a row per thread (n % 16 == 0, 16-byte aligned
// pointers): one 16-byte load of codes, the 16 scales as four 16-byte loads, two 16-byte stores.
__global__ void __launch_bounds__(256)
dequantize16_kernel(const int8_t* __restrict__ q, const float* __restrict__ scale, int64_t m,
                    int64_t n, __nv_bfloat16* __restrict__ out) {
  const int64_t units = m * n / 16;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = u * 16;
    const int64_t j = e % n;   // a multiple of 16: the unit lies inside one row
    const int4 codes = __ldg(reinterpret_cast<const int4*>(q + e));
    const float4* sp = reinterpret_cast<const float4*>(scale + j);
    const float4 s4[4] = {__ldg(sp), __ldg(sp + 1), __ldg(sp + 2), __ldg(sp + 3)};
    const float sc[16] = {s4[0].x, s4[0].y, s4[0].z, s4[0].w, s4[1].x, s4[1].y, s4[1].z, s4[1].w,
                          s4[2].x, s4[2].y, s4[2].z, s4[2].w, s4[3].x, s4[3].y, s4[3].z, s4[3].w};
    const int8_t* c = reinterpret_cast<const int8_t*>(&codes);
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn((float)c[2 * k], sc[2 * k]));
      const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn((float)c[2 * k + 1], sc[2 * k + 1]));
      w[k] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    uint4* o = reinterpret_cast<uint4*>(out + e);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

int grid_for(int64_t work, int threads) {
  const int64_t g = (work + threads - 1) / threads;
  return (int)(g < 148 * 16 ? (g < 1 ? 1 : g) : 148 * 16);
}

}  // namespace

cudaError_t quantize_cols_i8(const void* w, DT t, int64_t m, int64_t n, int8_t* q, float* scale,
                             cudaStream_t s) {
  if (m == 0 || n == 0) return cudaSuccess;
  unsigned* bits = reinterpret_cast<unsigned*>(scale);
  cudaError_t e = cudaMemsetAsync(bits, 0, (size_t)n * sizeof(float), s);
  if (e != cudaSuccess) return e;
  const dim3 g1((unsigned)((n + kColThreads - 1) / kColThreads),
                (unsigned)((m + kRowsPerSlab - 1) / kRowsPerSlab));
  const int g2 = grid_for((m * n + 3) / 4, 256);
  {
    TraceScope tr("xq_col_absmax", s);
    if (t == DT::BF16)
      col_absmax_kernel<<<g1, kColThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(w), m, n, bits);
    else
      col_absmax_kernel<<<g1, kColThreads, 0, s>>>(static_cast<const float*>(w), m, n, bits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    TraceScope tr("xq_quantize", s);
    if (t == DT::BF16)
      quantize_kernel<<<g2, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), m, n, bits, q);
    else
      quantize_kernel<<<g2, 256, 0, s>>>(static_cast<const float*>(w), m, n, bits, q);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  finalize_scale_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(bits, n);
  return cudaGetLastError();
}

cudaError_t dequantize_cols_i8(const int8_t* q, const float* scale, int64_t m, int64_t n,
                               __nv_bfloat16* out, cudaStream_t s) {
  if (m == 0 || n == 0) return cudaSuccess;
  TraceScope tr("xq_dequantize", s);
  const bool vec = n % 16 == 0 &&
                   ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(scale) |
                     reinterpret_cast<uintptr_t>(out)) & 15) == 0;
  if (vec)
    dequantize16_kernel<<<grid_for(m * n / 16, 256), 256, 0, s>>>(q, scale, m, n, out);
  else
    dequantize_kernel<<<grid_for(m * n, 256), 256, 0, s>>>(q, scale, m, n, out);
  return cudaGetLastError();
}

}  // namespace poetx
