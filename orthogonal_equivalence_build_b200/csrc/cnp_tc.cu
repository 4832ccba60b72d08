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

// ---------------------------------------------------------------- 32 x 32 mirrored tile pairs
// Every elementwise pass works on a pair of tiles (I, J), (J, I) with I <= J of one b x b block;
// only those pairs are launched (nt (nt + 1) / 2 per block). A thread owns one row and four
// consecutive columns of each tile: 16-byte loads, 8-byte bf16 stores, rows stay coalesced, and
// the transposes go through shared memory (conflict-free: the padded row stride is 33 floats).
// The packed q of a pair is read once (its upper tile is contiguous along each row).
constexpr int TS = 32;
constexpr int kTileThreads = 256;  // thread (tx, ty): row ty, columns 4 tx .. 4 tx + 3

struct Tile {
  float v[TS][TS + 1];
};

struct PairCtx {
  int g, I, J;      // block, tile row, tile column (I <= J)
  int r, c0;        // this thread's row in a tile and first of its four columns
  bool diag;
  int64_t bb;       // b * b
};

__device__ __forceinline__ void pair_ctx(int b, PairCtx& c) {
  const int nt = b / TS;
  int p = blockIdx.x, I = 0;
  while (p >= nt - I) {  // tile row I holds the pairs (I, I .. nt - 1)
    p -= nt - I;
    ++I;
  }
  c.I = I;
  c.J = I + p;
  c.g = blockIdx.y;
  c.r = threadIdx.x >> 3;
  c.c0 = (threadIdx.x & 7) * 4;
  c.diag = c.I == c.J;
  c.bb = (int64_t)b * b;
}

dim3 pair_grid(int64_t nb, int64_t b) {
  const int nt = (int)(b / TS);
  return dim3((unsigned)(nt * (nt + 1) / 2), (unsigned)nb);
}

// up <- Q tile (I, J), I <= J, from the packed strict upper triangle of one block (qb).
// The mirrored tile (J, I) is -up^T: its entry (r, col) is -up.v[col][r].
__device__ __forceinline__ void load_q_tile(Tile& up, const float* __restrict__ qb, int b,
                                            const PairCtx& c) {
  const int i = c.I * TS + c.r;
  const int64_t rowbase = (int64_t)i * b - (int64_t)i * (i + 1) / 2 - i - 1;  // + j for j > i
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = c.J * TS + c.c0 + k;
    up.v[c.r][c.c0 + k] = (i < j) ? qb[rowbase + j] : 0.f;
  }
  __syncthreads();
  if (c.diag) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (c.r > c.c0 + k) up.v[c.r][c.c0 + k] = -up.v[c.c0 + k][c.r];
    __syncthreads();
  }
}

__device__ __forceinline__ float4 ld4(const float* __restrict__ p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ void st4(float* p, float a, float b2, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b2, c, d);
}
__device__ __forceinline__ uint32_t bf2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void st4h(__nv_bfloat16* p, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(bf2(v[0], v[1]), bf2(v[2], v[3]));
}
__device__ __forceinline__ void split4(const float (&x)[4], float (&hi)[4], float (&lo)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    hi[k] = __bfloat162float(__float2bfloat16_rn(x[k]));
    lo[k] = x[k] - hi[k];
  }
}

// Concatenated split operands of one block product X Y, four consecutive columns j .. j+3:
//   Acat [nb*b][3b]: row (g, i) = [Xhi(i, :) | Xhi(i, :) | Xlo(i, :)]
//   Bcat [nb*3b][b]: rows (g, k') = Yhi (k' < b), Ylo (b <= k' < 2b), Yhi (2b <= k')
__device__ __forceinline__ void put_split4(__nv_bfloat16* __restrict__ Acat,
                                           __nv_bfloat16* __restrict__ Bcat, int b, int g, int i,
                                           int j, const float (&x)[4], const float (&y)[4]) {
  float xh[4], xl[4], yh[4], yl[4];
  split4(x, xh, xl);
  split4(y, yh, yl);
  __nv_bfloat16* arow = Acat + ((int64_t)g * b + i) * (3 * b) + j;
  st4h(arow, xh);
  st4h(arow + b, xh);
  st4h(arow + 2 * b, xl);
  const int64_t bb = (int64_t)b * b;
  __nv_bfloat16* bp = Bcat + (int64_t)g * 3 * bb + (int64_t)i * b + j;
  st4h(bp, yh);
  st4h(bp + bb, yl);
  st4h(bp + 2 * bb, yh);
}

__device__ __forceinline__ const float* run_q(const BlockRuns& r, int g, int b, int& run,
                                              int& local) {
  run = run_of(r, g, local);
  return r.q[run] + (int64_t)local * (b * (b - 1) / 2);
}

// CNP pass 1: X = Y = Q.
__global__ void __launch_bounds__(kTileThreads)
split_q_kernel(const BlockRuns r, int b, __nv_bfloat16* __restrict__ Acat,
               __nv_bfloat16* __restrict__ Bcat) {
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  load_q_tile(up, run_q(r, c.g, b, run, local), b, c);
  float x[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] = up.v[c.r][c.c0 + k];
  put_split4(Acat, Bcat, b, c.g, c.I * TS + c.r, c.J * TS + c.c0, x, x);
  if (!c.diag) {
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = -up.v[c.c0 + k][c.r];
    put_split4(Acat, Bcat, b, c.g, c.J * TS + c.r, c.I * TS + c.c0, x, x);
  }
}

// CNP pass 2: X = S, Y = 2I + 2Q + S.
__global__ void __launch_bounds__(kTileThreads)
split_sh_kernel(const BlockRuns r, const float* __restrict__ S, int b,
                __nv_bfloat16* __restrict__ Acat, __nv_bfloat16* __restrict__ Bcat) {
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  load_q_tile(up, run_q(r, c.g, b, run, local), b, c);
  const float* Sg = S + (int64_t)c.g * c.bb;
  float x[4], y[4];
  {
    const int i = c.I * TS + c.r, j = c.J * TS + c.c0;
    const float4 s4 = ld4(Sg + (int64_t)i * b + j);
    x[0] = s4.x; x[1] = s4.y; x[2] = s4.z; x[3] = s4.w;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      y[k] = ((c.diag && c.r == c.c0 + k) ? 2.f : 0.f) + 2.f * up.v[c.r][c.c0 + k] + x[k];
    put_split4(Acat, Bcat, b, c.g, i, j, x, y);
  }
  if (!c.diag) {
    const int i = c.J * TS + c.r, j = c.I * TS + c.c0;
    const float4 s4 = ld4(Sg + (int64_t)i * b + j);
    x[0] = s4.x; x[1] = s4.y; x[2] = s4.z; x[3] = s4.w;
#pragma unroll
    for (int k = 0; k < 4; ++k) y[k] = -2.f * up.v[c.c0 + k][c.r] + x[k];
    put_split4(Acat, Bcat, b, c.g, i, j, x, y);
  }
}

// CNP finish: G = I + 2Q + P (fp32 and its bf16 copy).
__global__ void __launch_bounds__(kTileThreads)
cnp_finish_kernel(const BlockRuns r, const float* __restrict__ Pall, int b) {
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  load_q_tile(up, run_q(r, c.g, b, run, local), b, c);
  // P is indexed by the launch-wide block, the outputs by the block within its run
  const float* P = Pall + (int64_t)c.g * c.bb;
  float* g = r.g[run] ? r.g[run] + (int64_t)local * c.bb : nullptr;
  __nv_bfloat16* g_lp = r.g_lp[run] ? r.g_lp[run] + (int64_t)local * c.bb : nullptr;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && c.diag) break;
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    const int64_t off = (int64_t)i * b + j;
    const float4 p4 = ld4(P + off);
    const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float qv = h ? -up.v[c.c0 + k][c.r] : up.v[c.r][c.c0 + k];
      v[k] = ((!h && c.diag && c.r == c.c0 + k) ? 1.f : 0.f) + 2.f * qv + pv[k];
    }
    if (g) st4(g + off, v[0], v[1], v[2], v[3]);
    if (g_lp) st4h(g_lp + off, v);
  }
}

// dq pass 1: Qh = bf16(Q); dG = sum of the split partials (fixed order), dGh = bf16(dG).
__global__ void __launch_bounds__(kTileThreads)
dq_prep_kernel(const BlockRuns r, int b, float* __restrict__ dG,
               __nv_bfloat16* __restrict__ Qh, __nv_bfloat16* __restrict__ dGh) {
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  load_q_tile(up, run_q(r, c.g, b, run, local), b, c);
  const int64_t base = (int64_t)c.g * c.bb;
  // this block's partial sums within its run, [splits][nb_run][b][b]
  const float* pr = r.parts[run] + (int64_t)local * c.bb;
  const int splits = r.splits[run];
  const int64_t split_stride = (int64_t)r.nb[run] * c.bb;
  const bool in_place = splits == 1 && pr == dG + base;  // written straight into dG
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && c.diag) break;
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    const int64_t off = (int64_t)i * b + j;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sp = 0; sp < splits; ++sp) {
      const float4 t = ld4(pr + sp * split_stride + off);
      v[0] += t.x; v[1] += t.y; v[2] += t.z; v[3] += t.w;
    }
    if (!in_place) st4(dG + base + off, v[0], v[1], v[2], v[3]);
    st4h(dGh + base + off, v);
    float qv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) qv[k] = h ? -up.v[c.c0 + k][c.r] : up.v[c.r][c.c0 + k];
    st4h(Qh + base + off, qv);
  }
}

// dq pass 2: Sh = bf16(S), SmQ = bf16(S - 2Q).
__global__ void __launch_bounds__(kTileThreads)
dq_prep2_kernel(const BlockRuns r, const float* __restrict__ S, int b,
                __nv_bfloat16* __restrict__ Sh, __nv_bfloat16* __restrict__ SmQ) {
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  load_q_tile(up, run_q(r, c.g, b, run, local), b, c);
  const int64_t base = (int64_t)c.g * c.bb;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && c.diag) break;
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    const int64_t off = base + (int64_t)i * b + j;
    const float4 s4 = ld4(S + off);
    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      m[k] = sv[k] - 2.f * (h ? -up.v[c.c0 + k][c.r] : up.v[c.r][c.c0 + k]);
    st4h(Sh + off, sv);
    st4h(SmQ + off, m);
  }
}

// dq pass 3: Sbar = 2dG + T1 + Hb; Zh = bf16(Sbar + Sbar^T); V = 2dG + 2Hb (written over S).
__global__ void __launch_bounds__(kTileThreads)
dq_mid_kernel(const float* __restrict__ dG, const float* __restrict__ T1,
              const float* __restrict__ Hb, int b, __nv_bfloat16* __restrict__ Zh,
              float* __restrict__ V) {
  __shared__ Tile sa, sb;  // Sbar tiles (I, J) and (J, I)
  PairCtx c;
  pair_ctx(b, c);
  const int64_t base = (int64_t)c.g * c.bb;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && c.diag) break;
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    const int64_t off = base + (int64_t)i * b + j;
    const float4 d = ld4(dG + off), t = ld4(T1 + off), hb = ld4(Hb + off);
    Tile& dst = h ? sb : sa;
    dst.v[c.r][c.c0 + 0] = 2.f * d.x + t.x + hb.x;
    dst.v[c.r][c.c0 + 1] = 2.f * d.y + t.y + hb.y;
    dst.v[c.r][c.c0 + 2] = 2.f * d.z + t.z + hb.z;
    dst.v[c.r][c.c0 + 3] = 2.f * d.w + t.w + hb.w;
    st4(V + off, 2.f * d.x + 2.f * hb.x, 2.f * d.y + 2.f * hb.y, 2.f * d.z + 2.f * hb.z,
        2.f * d.w + 2.f * hb.w);
  }
  __syncthreads();
  const Tile& tb = c.diag ? sa : sb;
  {
    const int i = c.I * TS + c.r, j = c.J * TS + c.c0;
    float z[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) z[k] = sa.v[c.r][c.c0 + k] + tb.v[c.c0 + k][c.r];
    st4h(Zh + base + (int64_t)i * b + j, z);
  }
  if (!c.diag) {
    const int i = c.J * TS + c.r, j = c.I * TS + c.c0;
    float z[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) z[k] = sb.v[c.r][c.c0 + k] + sa.v[c.c0 + k][c.r];
    st4h(Zh + base + (int64_t)i * b + j, z);
  }
}

// dq pass 4: U = V - ZQ; dq_ij = U_ij - U_ji (i < j), written packed.
__global__ void __launch_bounds__(kTileThreads)
dq_pack_kernel(const BlockRuns r, const float* __restrict__ V, const float* __restrict__ ZQ,
               int b) {
  __shared__ Tile ua, ub;  // U tiles (I, J) and (J, I)
  PairCtx c;
  pair_ctx(b, c);
  const int64_t base = (int64_t)c.g * c.bb;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && c.diag) break;
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    const int64_t off = base + (int64_t)i * b + j;
    const float4 v = ld4(V + off), z = ld4(ZQ + off);
    Tile& dst = h ? ub : ua;
    dst.v[c.r][c.c0 + 0] = v.x - z.x;
    dst.v[c.r][c.c0 + 1] = v.y - z.y;
    dst.v[c.r][c.c0 + 2] = v.z - z.z;
    dst.v[c.r][c.c0 + 3] = v.w - z.w;
  }
  __syncthreads();
  const Tile& tb = c.diag ? ua : ub;
  int local;
  const int run = run_of(r, c.g, local);
  float* dqb = r.dq[run] + (int64_t)local * (b * (b - 1) / 2);
  const int i = c.I * TS + c.r;
  const int64_t rowbase = (int64_t)i * b - (int64_t)i * (i + 1) / 2 - i - 1;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = c.J * TS + c.c0 + k;
    if (i < j) dqb[rowbase + j] = ua.v[c.r][c.c0 + k] - tb.v[c.c0 + k][c.r];
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

cudaError_t cnp_build_tc(const BlockRuns& r, int64_t b, void* ws, cudaStream_t s) {
  const int64_t nb = (int64_t)r.nb[0] + r.nb[1];
  if (nb == 0) return cudaSuccess;
  Arena a(ws, cnp_tc_ws_bytes(nb, b));
  auto* Acat = static_cast<__nv_bfloat16*>(a.take((size_t)(nb * b * 3 * b) * 2));
  auto* Bcat = static_cast<__nv_bfloat16*>(a.take((size_t)(nb * b * 3 * b) * 2));
  auto* S = static_cast<float*>(a.take((size_t)(nb * b * b) * 4));
  auto* P = static_cast<float*>(a.take((size_t)(nb * b * b) * 4));
  const dim3 grid = pair_grid(nb, b);
  const int bi = (int)b;
  {
    TraceScope t("cnp_split_Q", s);
    split_q_kernel<<<grid, kTileThreads, 0, s>>>(r, bi, Acat, Bcat);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Acat, Bcat, S, nb, b, 3 * b, "umma_cnp_QQ", s));
  {
    TraceScope t("cnp_split_SH", s);
    split_sh_kernel<<<grid, kTileThreads, 0, s>>>(r, S, bi, Acat, Bcat);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Acat, Bcat, P, nb, b, 3 * b, "umma_cnp_SH", s));
  TraceScope t("cnp_finish", s);
  cnp_finish_kernel<<<grid, kTileThreads, 0, s>>>(r, P, bi);
  return cudaGetLastError();
}

size_t dq_tc_ws_bytes(int64_t nb, int64_t b) {
  const size_t h = align_up((size_t)(nb * b * b) * 2, 256);
  const size_t f = align_up((size_t)(nb * b * b) * 4, 256);
  return 5 * h + 3 * f;
}

cudaError_t dq_from_dg_tc(const BlockRuns& r, int64_t b, float* dG, void* ws, cudaStream_t s) {
  const int64_t nb = (int64_t)r.nb[0] + r.nb[1];
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
  const dim3 grid = pair_grid(nb, b);
  const int bi = (int)b;
  {
    TraceScope t("dq_prep", s);
    dq_prep_kernel<<<grid, kTileThreads, 0, s>>>(r, bi, dG, Qh, dGh);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Qh, Qh, S, nb, b, b, "umma_dq_QQ", s));
  {
    TraceScope t("dq_prep2", s);
    dq_prep2_kernel<<<grid, kTileThreads, 0, s>>>(r, S, bi, Sh, SmQ);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Sh, dGh, Hb, nb, b, b, "umma_dq_SdG", s));
  POETX_TRY(block_product(dGh, SmQ, T1, nb, b, b, "umma_dq_dGH", s));
  {
    TraceScope t("dq_mid", s);
    dq_mid_kernel<<<grid, kTileThreads, 0, s>>>(dG, T1, Hb, bi, Zh, S);
    POETX_TRY(cudaGetLastError());
  }
  POETX_TRY(block_product(Zh, Qh, T1, nb, b, b, "umma_dq_ZQ", s));
  TraceScope t("dq_pack", s);
  dq_pack_kernel<<<grid, kTileThreads, 0, s>>>(r, S, T1, bi);
  return cudaGetLastError();
}

}  // namespace poetx
