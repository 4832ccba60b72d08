// Index-array permutations ("POET-X" blog §第二斧: a permutation is an index array, applied as a
// reorder of rows/columns instead of a product with an explicit permutation matrix).
//
// Column gathers/scatters move whole token rows: a CTA stages one row in shared memory with
// coalesced 16-byte loads, then reads (gather) or writes (scatter) the shared copy through the
// index array, and streams the result out with coalesced stores. Every value is copied
// bit-for-bit.
#include "internal.h"

#include <algorithm>

namespace poetx {
namespace {

constexpr int kPermThreads = 512;

template <typename T>
__device__ __forceinline__ void load_row_to_smem(const T* __restrict__ src, T* sm, int64_t cols) {
  // 16-byte vector path when the row is 16-byte aligned and a multiple of 16 bytes long
  const int64_t bytes = cols * (int64_t)sizeof(T);
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (bytes & 15) == 0) {
    const int4* s4 = reinterpret_cast<const int4*>(src);
    int4* d4 = reinterpret_cast<int4*>(sm);
    for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) d4[i] = __ldg(s4 + i);
  } else {
    for (int64_t i = threadIdx.x; i < cols; i += blockDim.x) sm[i] = src[i];
  }
}

template <typename T>
__device__ __forceinline__ void store_row_from_smem(T* __restrict__ dst, const T* sm, int64_t cols) {
  const int64_t bytes = cols * (int64_t)sizeof(T);
  if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0 && (bytes & 15) == 0) {
    const int4* s4 = reinterpret_cast<const int4*>(sm);
    int4* d4 = reinterpret_cast<int4*>(dst);
    for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) d4[i] = s4[i];
  } else {
    for (int64_t i = threadIdx.x; i < cols; i += blockDim.x) dst[i] = sm[i];
  }
}

// out[r, c] = in[rmap(r), cmap[c]]: stage the source row, gather from shared memory.
template <typename T>
__global__ void __launch_bounds__(kPermThreads)
gather_cols_kernel(const T* __restrict__ in, T* __restrict__ out, int64_t rows, int64_t cols,
                   const int32_t* __restrict__ row_map, const int32_t* __restrict__ col_map) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* src = reinterpret_cast<T*>(smem_raw);
  T* dst = src + pad8(cols);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t rs = row_map ? (int64_t)row_map[r] : r;
    load_row_to_smem(in + rs * cols, src, cols);
    __syncthreads();
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) dst[c] = src[col_map[c]];
    __syncthreads();
    store_row_from_smem(out + r * cols, dst, cols);
    __syncthreads();
  }
}

// out[r, cmap[c]] = in[r, c]: stage the source row, scatter into a shared output row.
template <typename T>
__global__ void __launch_bounds__(kPermThreads)
scatter_cols_kernel(const T* __restrict__ in, T* __restrict__ out, int64_t rows, int64_t cols,
                    const int32_t* __restrict__ col_map) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* src = reinterpret_cast<T*>(smem_raw);
  T* dst = src + pad8(cols);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    load_row_to_smem(in + r * cols, src, cols);
    __syncthreads();
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) dst[col_map[c]] = src[c];
    __syncthreads();
    store_row_from_smem(out + r * cols, dst, cols);
    __syncthreads();
  }
}

// Rows too long for shared memory: direct global gather/scatter (still bit-exact).
template <typename T>
__global__ void gather_cols_global(const T* __restrict__ in, T* __restrict__ out, int64_t rows,
                                   int64_t cols, const int32_t* __restrict__ row_map,
                                   const int32_t* __restrict__ col_map) {
  const int64_t total = rows * cols;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    const int64_t rs = row_map ? (int64_t)row_map[r] : r;
    out[e] = in[rs * cols + col_map[c]];
  }
}

template <typename T>
__global__ void scatter_cols_global(const T* __restrict__ in, T* __restrict__ out, int64_t rows,
                                    int64_t cols, const int32_t* __restrict__ col_map) {
  const int64_t total = rows * cols;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    out[r * cols + col_map[c]] = in[e];
  }
}

// out[r, c] = in[rmap(r), cmap[c]] for many rows sharing one column map. Rows are staged through
// shared memory in chunks of R rows with double-buffered cp.async (16-byte pieces, L1 bypassed),
// so the loads of chunk k+1 overlap the gather of chunk k. Each thread owns up to VPT fixed
// 16-byte output vectors (vector v = tid + k * blockDim) and keeps their source indices in
// registers for the whole launch (packed two 16-bit indices per register), so the per-row work
// is shared-memory reads plus one coalesced 16-byte store per vector. Needs cols <= 65536,
// 16-byte aligned rows and index array, and cols / (16 / sizeof(T)) <= VPT * blockDim.
template <typename T, int VPT>
__global__ void __launch_bounds__(256)
gather_cols_pipelined(const T* __restrict__ in, T* __restrict__ out, int64_t rows, int cols,
                      const int32_t* __restrict__ row_map, const int32_t* __restrict__ col_map,
                      int R) {
  pdl_wait();
  pdl_trigger();
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* buf[2] = {reinterpret_cast<T*>(smem_raw),
               reinterpret_cast<T*>(smem_raw) + (int64_t)R * cols};
  const int nvec = cols / VEC;
  const int64_t nchunks = (rows + R - 1) / R;
  int64_t chunk = blockIdx.x;
  if (chunk >= nchunks) return;
  // this thread's source indices, loaded once
  uint32_t ids[VPT][VEC / 2];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int v = threadIdx.x + k * blockDim.x;
#pragma unroll
    for (int h = 0; h < VEC / 2; ++h) ids[k][h] = 0;
    if (v < nvec) {
#pragma unroll
      for (int h = 0; h < VEC / 4; ++h) {
        const int4 t = __ldg(reinterpret_cast<const int4*>(col_map + v * VEC) + h);
        ids[k][2 * h] = (uint32_t)t.x | ((uint32_t)t.y << 16);
        ids[k][2 * h + 1] = (uint32_t)t.z | ((uint32_t)t.w << 16);
      }
    }
  }
  auto issue = [&](int64_t ch, T* dst) {
    for (int idx = threadIdx.x; idx < R * nvec; idx += blockDim.x) {
      const int r = idx / nvec, v = idx - r * nvec;
      const int64_t row = ch * R + r;
      if (row >= rows) continue;
      const int64_t src_row = row_map ? (int64_t)row_map[row] : row;
      const T* g = in + src_row * cols + (int64_t)v * VEC;
      const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(dst + r * cols + v * VEC));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(g) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(chunk, buf[0]);
  int cur = 0;
  for (; chunk < nchunks; chunk += gridDim.x) {
    const int64_t next = chunk + gridDim.x;
    if (next < nchunks) issue(next, buf[cur ^ 1]);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const int64_t left = rows - chunk * R;
    const int nr = left < R ? (int)left : R;
    for (int r = 0; r < nr; ++r) {
      const T* srow = buf[cur] + r * cols;
      T* orow = out + (chunk * R + r) * cols;
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        const int v = threadIdx.x + k * blockDim.x;
        if (v < nvec) {
          union {
            int4 v4;
            T e[VEC];
          } pack;
#pragma unroll
          for (int h = 0; h < VEC / 2; ++h) {
            pack.e[2 * h] = srow[ids[k][h] & 0xFFFFu];
            pack.e[2 * h + 1] = srow[ids[k][h] >> 16];
          }
          *reinterpret_cast<int4*>(orow + v * VEC) = pack.v4;
        }
      }
    }
    __syncthreads();
    cur ^= 1;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// bf16 rows two at a time, interleaved in shared memory: word c holds element c of row r (low
// half) and of row r + 1 (high half), so one random 32-bit shared-memory access moves the
// element of both rows. Random 2-byte accesses cost about 3.6 bank wavefronts per warp
// instruction (random banks); pairing halves the number of such instructions per element. The
// pair is read from global memory into registers (16-byte loads) one pair ahead. Each thread
// owns up to VPT fixed 16-byte vectors of each row and keeps their column indices in registers
// for the whole launch.
//   gather  (SCATTER = false): out[r, c] = in[r, col_map[c]]. The pair is written to shared
//           memory in order; output vector v reads its eight source words at random.
//   scatter (SCATTER = true):  out[r, col_map[c]] = in[r, c]. Input vector v writes its eight
//           words at random positions; the output is read back in order. No inverse map needed.
// Needs cols % 8 == 0, cols <= 65536, 16-byte aligned rows and index array; for the scatter,
// col_map must be a permutation (an output column no input maps to is left unwritten).
template <int VPT, int NT, bool SCATTER>
__global__ void __launch_bounds__(NT)
gather_cols_rowpair(const __nv_bfloat16* __restrict__ in, __nv_bfloat16* __restrict__ out,
                    int64_t rows, int cols, const int32_t* __restrict__ col_map) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint32_t pw[];   // cols words
  const int nvec = cols / 8;
  const int64_t npairs = (rows + 1) / 2;
  int64_t pr = blockIdx.x;
  if (pr >= npairs) return;
  uint32_t ids[VPT][4];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int v = threadIdx.x + k * blockDim.x;
#pragma unroll
    for (int h = 0; h < 4; ++h) ids[k][h] = 0;
    if (v < nvec) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // (indices are used as given: clamping them here measured 148 -> 210 us on 14336-wide
        // rows; the maps are permutations by contract, see poetx_validate_permutation)
        const int4 t = __ldg(reinterpret_cast<const int4*>(col_map + v * 8) + h);
        ids[k][2 * h] = (uint32_t)t.x | ((uint32_t)t.y << 16);
        ids[k][2 * h + 1] = (uint32_t)t.z | ((uint32_t)t.w << 16);
      }
    }
  }
  uint4 ra[VPT], rb[VPT];
  auto load = [&](int64_t p) {
    const int64_t r0 = 2 * p;
    const bool has1 = r0 + 1 < rows;
    const uint4* s0 = reinterpret_cast<const uint4*>(in + r0 * cols);
    const uint4* s1 = reinterpret_cast<const uint4*>(in + (r0 + 1) * cols);
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int v = threadIdx.x + k * blockDim.x;
      if (v < nvec) {
        ra[k] = __ldcs(s0 + v);
        rb[k] = has1 ? __ldcs(s1 + v) : make_uint4(0, 0, 0, 0);
      }
    }
  };
  load(pr);
  for (; pr < npairs; pr += gridDim.x) {
    __syncthreads();   // the previous pair's reads of pw are done
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int v = threadIdx.x + k * blockDim.x;
      if (v < nvec) {
        const uint4 a = ra[k], b = rb[k];
        // word e = element e of row r (low half) | element e of row r + 1 (high half)
        const uint32_t w[8] = {__byte_perm(a.x, b.x, 0x5410), __byte_perm(a.x, b.x, 0x7632),
                               __byte_perm(a.y, b.y, 0x5410), __byte_perm(a.y, b.y, 0x7632),
                               __byte_perm(a.z, b.z, 0x5410), __byte_perm(a.z, b.z, 0x7632),
                               __byte_perm(a.w, b.w, 0x5410), __byte_perm(a.w, b.w, 0x7632)};
        if constexpr (SCATTER) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            pw[ids[k][h] & 0xFFFFu] = w[2 * h];
            pw[ids[k][h] >> 16] = w[2 * h + 1];
          }
        } else {
          uint4* d = reinterpret_cast<uint4*>(pw + 8 * v);
          d[0] = make_uint4(w[0], w[1], w[2], w[3]);
          d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
    }
    __syncthreads();
    const int64_t nxt = pr + gridDim.x;
    if (nxt < npairs) load(nxt);   // lands in registers while this pair is gathered
    const int64_t r0 = 2 * pr;
    const bool has1 = r0 + 1 < rows;
    uint4* o0 = reinterpret_cast<uint4*>(out + r0 * cols);
    uint4* o1 = reinterpret_cast<uint4*>(out + (r0 + 1) * cols);
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int v = threadIdx.x + k * blockDim.x;
      if (v < nvec) {
        uint32_t x[4], y[4];
        if constexpr (SCATTER) {
          const uint4* d = reinterpret_cast<const uint4*>(pw + 8 * v);
          const uint4 d0 = d[0], d1 = d[1];
          const uint32_t w[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            x[h] = __byte_perm(w[2 * h], w[2 * h + 1], 0x5410);
            y[h] = __byte_perm(w[2 * h], w[2 * h + 1], 0x7632);
          }
        } else {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const uint32_t lo = pw[ids[k][h] & 0xFFFFu], hi = pw[ids[k][h] >> 16];
            x[h] = __byte_perm(lo, hi, 0x5410);   // row r:     elements 2h, 2h + 1
            y[h] = __byte_perm(lo, hi, 0x7632);   // row r + 1
          }
        }
        __stcs(o0 + v, make_uint4(x[0], x[1], x[2], x[3]));
        if (has1) __stcs(o1 + v, make_uint4(y[0], y[1], y[2], y[3]));
      }
    }
  }
}

int num_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

constexpr size_t kMaxRowSmem = 200 * 1024;

bool aligned16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// token rows of a bf16 activation: row pairs interleaved in shared memory
bool rowpair_ok(const void* in, const void* out, int64_t cols, const int32_t* col_map) {
  return cols % 8 == 0 && cols <= 65536 && cols / 8 <= 4 * 512 && aligned16p(in) &&
         aligned16p(out) && aligned16p(col_map);
}

template <bool SCATTER>
cudaError_t launch_rowpair(const void* in, void* out, int64_t rows, int64_t cols,
                           const int32_t* col_map, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const size_t smem = (size_t)cols * 4;
  const int64_t npairs = (rows + 1) / 2, nvec = cols / 8;
  auto launch = [&](auto kern, int threads, int per_sm) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    per_sm = std::max(1, std::min(per_sm, (int)((200 * 1024) / smem)));
    const int64_t grid = std::min<int64_t>(npairs, (int64_t)num_sms() * per_sm);
    launch_k(kern, dim3((unsigned)grid), dim3(threads), smem, s,
             static_cast<const __nv_bfloat16*>(in), static_cast<__nv_bfloat16*>(out), rows,
             (int)cols, col_map);
  };
  // CTAs per SM as the registers allow
  if (nvec <= 2 * 256) launch(gather_cols_rowpair<2, 256, SCATTER>, 256, 3);
  else if (nvec <= 4 * 256) launch(gather_cols_rowpair<4, 256, SCATTER>, 256, 2);
  else launch(gather_cols_rowpair<4, 512, SCATTER>, 512, 1);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gather(const void* in, void* out, int64_t rows, int64_t cols,
                          const int32_t* row_map, const int32_t* col_map, cudaStream_t s,
                          const char* name) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const size_t row_bytes = (size_t)cols * sizeof(T);
  constexpr int VEC = 16 / sizeof(T);
  const int64_t nvec = cols / VEC;
  if (sizeof(T) == 2 && !row_map && rowpair_ok(in, out, cols, col_map)) {
    TraceScope t(name ? name : "perm_gather_cols_bf16", s);
    return launch_rowpair<false>(in, out, rows, cols, col_map, s);
  }
  if (row_bytes % 16 == 0 && row_bytes <= 96 * 1024 && cols <= 65536 && nvec <= 8 * 256 &&
      aligned16p(in) && aligned16p(out) && aligned16p(col_map)) {
    // chunks of about 24 KB per buffer, two buffers per CTA
    const int R = (int)std::max<size_t>(1, std::min<size_t>(16, (24 * 1024) / row_bytes));
    const size_t smem = 2 * (size_t)R * row_bytes;
    const int per_sm = std::max(1, std::min(8, (int)((200 * 1024) / smem)));
    const int64_t nchunks = (rows + R - 1) / R;
    const int64_t grid = std::min<int64_t>(nchunks, (int64_t)num_sms() * per_sm);
    TraceScope t(name ? name : (sizeof(T) == 2 ? "perm_gather_cols_bf16" : "perm_gather_cols_f32"),
                 s);
    auto launch = [&](auto kern) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      launch_k(kern, dim3((unsigned)grid), dim3(256), smem, s, static_cast<const T*>(in),
               static_cast<T*>(out), rows, (int)cols, row_map, col_map, R);
    };
    if (nvec <= 2 * 256) launch(gather_cols_pipelined<T, 2>);
    else if (nvec <= 4 * 256) launch(gather_cols_pipelined<T, 4>);
    else launch(gather_cols_pipelined<T, 8>);
    return cudaGetLastError();
  }
  const size_t smem = 2 * (size_t)pad8(cols) * sizeof(T);
  if (smem <= kMaxRowSmem) {
    cudaFuncSetAttribute(gather_cols_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    const int per_sm = std::max(1, (int)(220 * 1024 / std::max<size_t>(smem, 1)));
    const int64_t grid = std::min<int64_t>(rows, (int64_t)num_sms() * std::min(per_sm, 4));
    TraceScope t(sizeof(T) == 2 ? "perm_gather_cols_bf16" : "perm_gather_cols_f32", s);
    gather_cols_kernel<T><<<(unsigned)grid, kPermThreads, smem, s>>>(
        static_cast<const T*>(in), static_cast<T*>(out), rows, cols, row_map, col_map);
  } else {
    TraceScope t("perm_gather_cols_global", s);
    gather_cols_global<T><<<num_sms() * 8, 256, 0, s>>>(static_cast<const T*>(in),
                                                        static_cast<T*>(out), rows, cols,
                                                        row_map, col_map);
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_scatter(const void* in, void* out, int64_t rows, int64_t cols,
                           const int32_t* col_map, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const size_t smem = 2 * (size_t)pad8(cols) * sizeof(T);
  if (smem <= kMaxRowSmem) {
    cudaFuncSetAttribute(scatter_cols_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    const int per_sm = std::max(1, (int)(220 * 1024 / std::max<size_t>(smem, 1)));
    const int64_t grid = std::min<int64_t>(rows, (int64_t)num_sms() * std::min(per_sm, 4));
    TraceScope t(sizeof(T) == 2 ? "perm_scatter_cols_bf16" : "perm_scatter_cols_f32", s);
    scatter_cols_kernel<T><<<(unsigned)grid, kPermThreads, smem, s>>>(
        static_cast<const T*>(in), static_cast<T*>(out), rows, cols, col_map);
  } else {
    TraceScope t("perm_scatter_cols_global", s);
    scatter_cols_global<T><<<num_sms() * 8, 256, 0, s>>>(static_cast<const T*>(in),
                                                         static_cast<T*>(out), rows, cols,
                                                         col_map);
  }
  return cudaGetLastError();
}

__global__ void invert_kernel(const int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                              int64_t k) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < k;
       i += (int64_t)gridDim.x * blockDim.x)
    inv[perm[i]] = (int32_t)i;
}

__global__ void compose_kernel(const int32_t* __restrict__ inv, const int32_t* __restrict__ pn,
                               int32_t* __restrict__ rho, int64_t k) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < k;
       i += (int64_t)gridDim.x * blockDim.x)
    rho[i] = inv[pn[i]];
}

// ---- counter-based SplitMix64 (Steele, Lea & Flood 2014): the i-th output of the stream that
// starts at `state` is mix(state + (i + 1) * gamma).
__host__ __device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t sm64_output(uint64_t state, uint64_t i) {
  return sm64_mix(state + (i + 1) * 0x9E3779B97F4A7C15ull);
}

constexpr int kRankThreads = 256;
constexpr int kRankTile = 2048;

// perm[rank(i)] = i with rank(i) = #{j : (key_j, j) < (key_i, i)}: the stable argsort of the
// keys, computed by counting (k is at most a few tens of thousands; this runs once per merge).
__global__ void __launch_bounds__(kRankThreads)
rank_permutation_kernel(uint64_t stream_state, int64_t k, int32_t* __restrict__ perm) {
  __shared__ uint64_t tile[kRankTile];
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const uint64_t ki = (i < k) ? sm64_output(stream_state, (uint64_t)i) : 0ull;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < k; j0 += kRankTile) {
    const int64_t nj = min((int64_t)kRankTile, k - j0);
    __syncthreads();
    for (int t = threadIdx.x; t < nj; t += blockDim.x) tile[t] = sm64_output(stream_state, j0 + t);
    __syncthreads();
    if (i < k) {
      for (int t = 0; t < nj; ++t) {
        const uint64_t kj = tile[t];
        rank += (kj < ki) || (kj == ki && (j0 + t) < i);
      }
    }
  }
  if (i < k) perm[rank] = (int32_t)i;
}

__global__ void count_kernel(const int32_t* __restrict__ perm, int64_t k,
                             int32_t* __restrict__ counts) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < k;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t v = perm[i];
    if (v < 0 || (int64_t)v >= k) atomicExch(counts + k, 1);
    else atomicAdd(counts + v, 1);
  }
}

__global__ void check_counts_kernel(int32_t* __restrict__ counts, int64_t k) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < k;
       i += (int64_t)gridDim.x * blockDim.x)
    if (counts[i] != 1) atomicExch(counts + k, 1);
}

}  // namespace

cudaError_t gather_cols(const void* in, void* out, int64_t rows, int64_t cols,
                        const int32_t* row_map, const int32_t* col_map, int elem_bytes,
                        cudaStream_t s, const char* name) {
  if (elem_bytes == 2)
    return launch_gather<__nv_bfloat16>(in, out, rows, cols, row_map, col_map, s, name);
  return launch_gather<float>(in, out, rows, cols, row_map, col_map, s, name);
}

cudaError_t scatter_cols(const void* in, void* out, int64_t rows, int64_t cols,
                         const int32_t* col_map, int elem_bytes, int32_t* inv_tmp,
                         cudaStream_t s, const char* name) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  if (elem_bytes == 2 && rowpair_ok(in, out, cols, col_map)) {
    // bf16 token rows: the row-pair kernel in scatter mode, as fast as its gather mode and
    // without the inverse map's extra launch
    TraceScope t(name ? name : "perm_scatter_cols_bf16", s);
    return launch_rowpair<true>(in, out, rows, cols, col_map, s);
  }
  if (inv_tmp && aligned16p(inv_tmp) && ((size_t)cols * elem_bytes) % 16 == 0) {
    // out[r, p] = in[r, inverse(col_map)[p]]: the scatter as a pipelined gather
    const int grid = (int)std::min<int64_t>((cols + 255) / 256, 4096);
    {
      TraceScope t("perm_invert", s);
      cudaError_t e = launch_k(invert_kernel, dim3(grid), dim3(256), 0, s, col_map, inv_tmp, cols);
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    return gather_cols(in, out, rows, cols, nullptr, inv_tmp, elem_bytes, s, name);
  }
  if (elem_bytes == 2) return launch_scatter<__nv_bfloat16>(in, out, rows, cols, col_map, s);
  return launch_scatter<float>(in, out, rows, cols, col_map, s);
}

cudaError_t compose_inverse(const int32_t* perm_old, const int32_t* perm_new, int32_t* inv_tmp,
                            int32_t* rho, int64_t k, cudaStream_t s) {
  if (k == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((k + 255) / 256, 4096);
  {
    TraceScope t("perm_invert", s);
    invert_kernel<<<grid, 256, 0, s>>>(perm_old, inv_tmp, k);
  }
  TraceScope t("perm_compose", s);
  compose_kernel<<<grid, 256, 0, s>>>(inv_tmp, perm_new, rho, k);
  return cudaGetLastError();
}

cudaError_t resample_permutation(uint64_t seed, int lane, int64_t k, int32_t* perm,
                                 cudaStream_t s) {
  if (k == 0) return cudaSuccess;
  const uint64_t stream_state = sm64_output(seed, (uint64_t)lane);
  TraceScope t("perm_resample_rank", s);
  rank_permutation_kernel<<<(unsigned)((k + kRankThreads - 1) / kRankThreads), kRankThreads, 0,
                            s>>>(stream_state, k, perm);
  return cudaGetLastError();
}

cudaError_t count_permutation(const int32_t* perm, int64_t k, int32_t* counts_and_flag,
                              cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(counts_and_flag, 0, (size_t)(k + 1) * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  if (k == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((k + 255) / 256, 4096);
  TraceScope t("perm_validate", s);
  count_kernel<<<grid, 256, 0, s>>>(perm, k, counts_and_flag);
  check_counts_kernel<<<grid, 256, 0, s>>>(counts_and_flag, k);
  return cudaGetLastError();
}

}  // namespace poetx
