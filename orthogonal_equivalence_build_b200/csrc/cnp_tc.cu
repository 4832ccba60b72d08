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
// Every elementwise pass works on a pair of tiles (I, J), (J, I) with I <= J of one b x b block:
// loads and stores stay coalesced along rows, transposes go through shared memory, and the
// packed q of the pair is read once (its upper tile is contiguous along each row).
constexpr int TS = 32;
constexpr int kTileThreads = 256;  // 32 x 8: thread (tx, ty) owns rows ty, ty+8, ty+16, ty+24

struct Tile {
  float v[TS][TS + 1];
};

struct PairCtx {
  int g, I, J;      // block, tile row, tile column (I <= J)
  int tx, ty;
  bool diag;
  int64_t bb;       // b * b
};

__device__ __forceinline__ bool pair_ctx(int b, PairCtx& c) {
  const int nt = b / TS;
  c.I = blockIdx.x / nt;
  c.J = blockIdx.x - c.I * nt;
  if (c.I > c.J) return false;
  c.g = blockIdx.y;
  c.tx = threadIdx.x & 31;
  c.ty = threadIdx.x >> 5;
  c.diag = c.I == c.J;
  c.bb = (int64_t)b * b;
  return true;
}

// up <- Q tile (I, J), I <= J, from the packed strict upper triangle of one block (qb).
__device__ __forceinline__ void load_q_tile(Tile& up, const float* __restrict__ qb, int b,
                                            const PairCtx& c) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    const int i = c.I * TS + r, j = c.J * TS + c.tx;
    up.v[r][c.tx] = (i < j) ? qb[i * b - i * (i + 1) / 2 + (j - i - 1)] : 0.f;
  }
  __syncthreads();
  if (c.diag) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = c.ty + 8 * k;
      if (r > c.tx) up.v[r][c.tx] = -up.v[c.tx][r];
    }
    __syncthreads();
  }
}
// Q tile (J, I) entry (r, col) is -up.v[col][r].

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Concatenated split operands of one block product X Y:
//   Acat [nb*b][3b]: row (g, i) = [Xhi(i, :) | Xhi(i, :) | Xlo(i, :)]
//   Bcat [nb*3b][b]: rows (g, k') = Yhi (k' < b), Ylo (b <= k' < 2b), Yhi (2b <= k')
__device__ __forceinline__ void put_split(__nv_bfloat16* __restrict__ Acat,
                                          __nv_bfloat16* __restrict__ Bcat, int b, int g, int i,
                                          int j, float x, float y) {
  __nv_bfloat16 xh, xl, yh, yl;
  split_bf16(x, xh, xl);
  split_bf16(y, yh, yl);
  __nv_bfloat16* arow = Acat + ((int64_t)g * b + i) * (3 * b);
  arow[j] = xh;
  arow[b + j] = xh;
  arow[2 * b + j] = xl;
  __nv_bfloat16* bblk = Bcat + (int64_t)g * 3 * b * b;
  const int64_t e = (int64_t)i * b + j, bb = (int64_t)b * b;
  bblk[e] = yh;
  bblk[bb + e] = yl;
  bblk[2 * bb + e] = yh;
}

// CNP pass 1: X = Y = Q.
__global__ void __launch_bounds__(kTileThreads)
split_q_kernel(const BlockRuns r, int b, __nv_bfloat16* __restrict__ Acat,
               __nv_bfloat16* __restrict__ Bcat) {
  __shared__ Tile up;
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  int local;
  const int run = run_of(r, c.g, local);
  load_q_tile(up, r.q[run] + (int64_t)local * (b * (b - 1) / 2), b, c);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    const float v = up.v[r][c.tx];
    put_split(Acat, Bcat, b, c.g, c.I * TS + r, c.J * TS + c.tx, v, v);
    if (!c.diag) {
      const float w = -up.v[c.tx][r];
      put_split(Acat, Bcat, b, c.g, c.J * TS + r, c.I * TS + c.tx, w, w);
    }
  }
}

// CNP pass 2: X = S, Y = 2I + 2Q + S.
__global__ void __launch_bounds__(kTileThreads)
split_sh_kernel(const BlockRuns r, const float* __restrict__ S, int b,
                __nv_bfloat16* __restrict__ Acat, __nv_bfloat16* __restrict__ Bcat) {
  __shared__ Tile up;
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  int local;
  const int run = run_of(r, c.g, local);
  load_q_tile(up, r.q[run] + (int64_t)local * (b * (b - 1) / 2), b, c);
  const float* Sg = S + (int64_t)c.g * c.bb;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    {
      const int i = c.I * TS + r, j = c.J * TS + c.tx;
      const float s = Sg[(int64_t)i * b + j];
      put_split(Acat, Bcat, b, c.g, i, j, s, ((i == j) ? 2.f : 0.f) + 2.f * up.v[r][c.tx] + s);
    }
    if (!c.diag) {
      const int i = c.J * TS + r, j = c.I * TS + c.tx;
      const float s = Sg[(int64_t)i * b + j];
      put_split(Acat, Bcat, b, c.g, i, j, s, -2.f * up.v[c.tx][r] + s);
    }
  }
}

// CNP finish: G = I + 2Q + P (fp32 and its bf16 copy).
__global__ void __launch_bounds__(kTileThreads)
cnp_finish_kernel(const BlockRuns r, const float* __restrict__ Pall, int b) {
  __shared__ Tile up;
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  int local;
  const int run = run_of(r, c.g, local);
  load_q_tile(up, r.q[run] + (int64_t)local * (b * (b - 1) / 2), b, c);
  // P is indexed by the launch-wide block, the outputs by the block within its run
  const float* P = Pall + ((int64_t)c.g - local) * c.bb;
  float* g = r.g[run];
  __nv_bfloat16* g_lp = r.g_lp[run];
  const int64_t base = (int64_t)local * c.bb;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    {
      const int i = c.I * TS + r, j = c.J * TS + c.tx;
      const int64_t e = base + (int64_t)i * b + j;
      const float v = ((i == j) ? 1.f : 0.f) + 2.f * up.v[r][c.tx] + P[e];
      if (g) g[e] = v;
      if (g_lp) g_lp[e] = __float2bfloat16_rn(v);
    }
    if (!c.diag) {
      const int i = c.J * TS + r, j = c.I * TS + c.tx;
      const int64_t e = base + (int64_t)i * b + j;
      const float v = -2.f * up.v[c.tx][r] + P[e];
      if (g) g[e] = v;
      if (g_lp) g_lp[e] = __float2bfloat16_rn(v);
    }
  }
}

// dq pass 1: Qh = bf16(Q); dG = sum of the split partials (fixed order), dGh = bf16(dG).
__global__ void __launch_bounds__(kTileThreads)
dq_prep_kernel(const BlockRuns r, int b, float* __restrict__ dG,
               __nv_bfloat16* __restrict__ Qh, __nv_bfloat16* __restrict__ dGh) {
  __shared__ Tile up;
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  int local;
  const int run = run_of(r, c.g, local);
  load_q_tile(up, r.q[run] + (int64_t)local * (b * (b - 1) / 2), b, c);
  const int64_t base = (int64_t)c.g * c.bb;
  // this block's partial sums within its run, [splits][nb_run][b][b]
  const float* pr = r.parts[run] + (int64_t)local * c.bb;
  const int splits = r.splits[run];
  const int64_t split_stride = (int64_t)r.nb[run] * c.bb;
  const bool in_place = splits == 1 && pr == dG + base;  // written straight into dG
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && c.diag) break;
      const int i = (h ? c.J : c.I) * TS + r, j = (h ? c.I : c.J) * TS + c.tx;
      const int64_t off = (int64_t)i * b + j, e = base + off;
      float v = 0.f;
      for (int sp = 0; sp < splits; ++sp) v += pr[sp * split_stride + off];
      if (!in_place) dG[e] = v;
      dGh[e] = __float2bfloat16_rn(v);
      Qh[e] = __float2bfloat16_rn(h ? -up.v[c.tx][r] : up.v[r][c.tx]);
    }
  }
}

// dq pass 2: Sh = bf16(S), SmQ = bf16(S - 2Q).
__global__ void __launch_bounds__(kTileThreads)
dq_prep2_kernel(const BlockRuns r, const float* __restrict__ S, int b,
                __nv_bfloat16* __restrict__ Sh, __nv_bfloat16* __restrict__ SmQ) {
  __shared__ Tile up;
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  int local;
  const int run = run_of(r, c.g, local);
  load_q_tile(up, r.q[run] + (int64_t)local * (b * (b - 1) / 2), b, c);
  const int64_t base = (int64_t)c.g * c.bb;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && c.diag) break;
      const int i = (h ? c.J : c.I) * TS + r, j = (h ? c.I : c.J) * TS + c.tx;
      const int64_t e = base + (int64_t)i * b + j;
      const float s = S[e];
      const float qv = h ? -up.v[c.tx][r] : up.v[r][c.tx];
      Sh[e] = __float2bfloat16_rn(s);
      SmQ[e] = __float2bfloat16_rn(s - 2.f * qv);
    }
  }
}

// dq pass 3: Sbar = 2dG + T1 + Hb; Zh = bf16(Sbar + Sbar^T); V = 2dG + 2Hb (written over S).
__global__ void __launch_bounds__(kTileThreads)
dq_mid_kernel(const float* __restrict__ dG, const float* __restrict__ T1,
              const float* __restrict__ Hb, int b, __nv_bfloat16* __restrict__ Zh,
              float* __restrict__ V) {
  __shared__ Tile sa, sb;  // Sbar tiles (I, J) and (J, I)
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  const int64_t base = (int64_t)c.g * c.bb;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = (h ? c.J : c.I) * TS + r, j = (h ? c.I : c.J) * TS + c.tx;
      const int64_t e = base + (int64_t)i * b + j;
      const float d = dG[e], hb = Hb[e];
      (h ? sb : sa).v[r][c.tx] = 2.f * d + T1[e] + hb;
      if (h == 0 || !c.diag) V[e] = 2.f * d + 2.f * hb;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    {
      const int i = c.I * TS + r, j = c.J * TS + c.tx;
      Zh[base + (int64_t)i * b + j] = __float2bfloat16_rn(sa.v[r][c.tx] + sb.v[c.tx][r]);
    }
    if (!c.diag) {
      const int i = c.J * TS + r, j = c.I * TS + c.tx;
      Zh[base + (int64_t)i * b + j] = __float2bfloat16_rn(sb.v[r][c.tx] + sa.v[c.tx][r]);
    }
  }
}

// dq pass 4: U = V - ZQ; dq_ij = U_ij - U_ji (i < j), written packed.
__global__ void __launch_bounds__(kTileThreads)
dq_pack_kernel(const BlockRuns r, const float* __restrict__ V, const float* __restrict__ ZQ,
               int b) {
  __shared__ Tile ua, ub;  // U tiles (I, J) and (J, I)
  PairCtx c;
  if (!pair_ctx(b, c)) return;
  const int64_t base = (int64_t)c.g * c.bb;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    {
      const int64_t e = base + (int64_t)(c.I * TS + r) * b + c.J * TS + c.tx;
      ua.v[r][c.tx] = V[e] - ZQ[e];
    }
    {
      const int64_t e = base + (int64_t)(c.J * TS + r) * b + c.I * TS + c.tx;
      ub.v[r][c.tx] = V[e] - ZQ[e];
    }
  }
  __syncthreads();
  int local;
  const int run = run_of(r, c.g, local);
  float* dqb = r.dq[run] + (int64_t)local * (b * (b - 1) / 2);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = c.ty + 8 * k;
    const int i = c.I * TS + r, j = c.J * TS + c.tx;
    if (i < j) dqb[i * b - i * (i + 1) / 2 + (j - i - 1)] = ua.v[r][c.tx] - ub.v[c.tx][r];
  }
}

dim3 pair_grid(int64_t nb, int64_t b) { return dim3((unsigned)((b / TS) * (b / TS)), (unsigned)nb); }

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
