// Cayley-Neumann blocks and their gradient on the tensor cores (block size b a multiple of 128).
//
// CNP ("POET-X" blog §第四斧 item 2; "Reparameterized LLM Training ..." §2 CNP, k = 3), evaluated
// as G = (I + 2Q) + S H with S = Q Q and H = 2I + 2Q + S: two b x b products per block, on the
// bf16 tcgen05 kernel with fp32 accumulation. Each fp32 operand x is split into
// x_hi = bf16(x) and x_lo = bf16(x - x_hi); x y is taken as x_hi y_hi + x_hi y_lo + x_lo y_hi,
// one accumulator over three K segments that read the hi and lo halves from their own buffers
// (the dropped x_lo y_lo is ~2^-16 relative): fp32-class G for the 1e-5 bar.
//   pass 1 (elementwise): q -> Q_hi, Q_lo
//   product 1: S = Q Q; its epilogue writes S_hi, S_lo and H_hi, H_lo (H = 2I + 2Q + S)
//   product 2: P = S H; its epilogue writes G = I + 2Q + P (fp32 and bf16)
// Q in the epilogues is Q_hi + Q_lo (within |Q| 2^-17 of Q).
//
// Gradient, for bf16 layers (tolerance 1e-2): with Hbar = S dG, Sbar = dG (2I - 2Q + S) + Hbar,
// Z = Sbar + Sbar^T, U = 2 dG + 2 Hbar - Z Q, dq_ij = U_ij - U_ji (i < j). The products S = QQ,
// S dG and dG (S - 2Q) (the last two in one launch) and Z Q run single-pass bf16 with fp32
// accumulation; the exact 2 dG terms are added in fp32.
//   pass 1: dG = sum of split partials, dG_h = bf16(dG), Q_h, Q_l
//   product 1: S = Q_h Q_h; epilogue writes S_h = bf16(S), SmQ = bf16(S - 2Q)
//   products 2, 3 (one launch over 2 nb groups): Hbar = S_h dG_h, T1 = dG_h SmQ
//   pass 2: Z_h = bf16(Sbar + Sbar^T), V = 2 dG + 2 Hbar
//   product 4: Z_h Q_h;  pass 3: U = V - Z Q, dq packed.
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

__device__ __forceinline__ const float* run_q(const BlockRuns& r, int g, int b, int& run,
                                              int& local) {
  run = run_of(r, g, local);
  return r.q[run] + (int64_t)local * (b * (b - 1) / 2);
}

// hi / lo parts of four values, stored at p_hi + off and p_lo + off
__device__ __forceinline__ void put_hilo4(__nv_bfloat16* __restrict__ p_hi,
                                          __nv_bfloat16* __restrict__ p_lo, int64_t off,
                                          const float (&x)[4]) {
  float h[4], l[4];
  split4(x, h, l);
  st4h(p_hi + off, h);
  st4h(p_lo + off, l);
}

// The per-block counts of a two-product launch (see run_chain) start at zero: the first CTA
// of the pass before it clears them (the launch waits for this grid to finish).
__device__ __forceinline__ void zero_counts(int* deps, int ndeps) {
  if (deps && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < ndeps; i += blockDim.x) deps[i] = 0;
}

// CNP pass 1: Q_hi, Q_lo [nb][b][b] from the packed strict upper triangles.
__global__ void __launch_bounds__(kTileThreads)
split_q_kernel(const __grid_constant__ BlockRuns r, int b, __nv_bfloat16* __restrict__ Qhi,
               __nv_bfloat16* __restrict__ Qlo, int* __restrict__ deps, int ndeps) {
  pdl_wait();
  pdl_trigger();
  zero_counts(deps, ndeps);
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  load_q_tile(up, run_q(r, c.g, b, run, local), b, c);
  const int64_t base = (int64_t)c.g * c.bb;
  float x[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] = up.v[c.r][c.c0 + k];
  put_hilo4(Qhi, Qlo, base + (int64_t)(c.I * TS + c.r) * b + c.J * TS + c.c0, x);
  if (!c.diag) {
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = -up.v[c.c0 + k][c.r];
    put_hilo4(Qhi, Qlo, base + (int64_t)(c.J * TS + c.r) * b + c.I * TS + c.c0, x);
  }
}

// dq pass 1: Qh = bf16(Q), Ql = bf16(Q - Qh); dG = sum of the split partials (fixed order),
// dGh = bf16(dG).
__global__ void __launch_bounds__(kTileThreads)
dq_prep_kernel(const __grid_constant__ BlockRuns r, int b, float* __restrict__ dG,
               __nv_bfloat16* __restrict__ Qh, __nv_bfloat16* __restrict__ Ql,
               __nv_bfloat16* __restrict__ dGh, int* __restrict__ deps, int ndeps) {
  pdl_wait();
  pdl_trigger();
  zero_counts(deps, ndeps);
  __shared__ Tile up;
  PairCtx c;
  pair_ctx(b, c);
  int run, local;
  const float* qb = run_q(r, c.g, b, run, local);
  const int64_t base = (int64_t)c.g * c.bb;
  // this block's partial sums within its run, [splits][nb_run][b][b]
  const float* pr = r.parts[run] + (int64_t)local * c.bb;
  const int splits = r.splits[run];
  const int64_t split_stride =
      r.split_stride[run] ? r.split_stride[run] : (int64_t)r.nb[run] * c.bb;
  const bool in_place = splits == 1 && pr == dG + base;  // written straight into dG
  // the first split's values of both tiles are requested before the q tile, so the two loads'
  // latencies overlap instead of following each other across the q tile's barrier
  float4 first[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    first[h] = (h == 1 && c.diag) ? make_float4(0.f, 0.f, 0.f, 0.f)
                                  : ld4(pr + (int64_t)i * b + j);
  }
  load_q_tile(up, qb, b, c);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && c.diag) break;
    const int i = (h ? c.J : c.I) * TS + c.r, j = (h ? c.I : c.J) * TS + c.c0;
    const int64_t off = (int64_t)i * b + j;
    float v[4] = {first[h].x, first[h].y, first[h].z, first[h].w};
    int sp = 1;
    for (; sp + 4 <= splits; sp += 4) {   // four loads in flight, added in split order
      float4 t[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) t[u] = ld4(pr + (sp + u) * split_stride + off);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[0] += t[u].x; v[1] += t[u].y; v[2] += t[u].z; v[3] += t[u].w;
      }
    }
    for (; sp < splits; ++sp) {
      const float4 t = ld4(pr + sp * split_stride + off);
      v[0] += t.x; v[1] += t.y; v[2] += t.z; v[3] += t.w;
    }
    if (!in_place) st4(dG + base + off, v[0], v[1], v[2], v[3]);
    st4h(dGh + base + off, v);
    float qv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) qv[k] = h ? -up.v[c.c0 + k][c.r] : up.v[c.r][c.c0 + k];
    put_hilo4(Qh, Ql, base + off, qv);
  }
}

// dq pass 3: Sbar = 2dG + T1 + Hb; Zh = bf16(Sbar + Sbar^T); V = 2dG + 2Hb (written over S).
__global__ void __launch_bounds__(kTileThreads)
dq_mid_kernel(const float* __restrict__ dG, const float* __restrict__ T1,
              const float* __restrict__ Hb, int b, __nv_bfloat16* __restrict__ Zh,
              float* __restrict__ V) {
  pdl_wait();
  pdl_trigger();
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
dq_pack_kernel(const __grid_constant__ BlockRuns r, const float* __restrict__ V, const float* __restrict__ ZQ,
               int b) {
  pdl_wait();
  pdl_trigger();
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

// C_g = X_g Y_g for `groups` blocks of b x b (fp32 accumulators), X K-major [groups*b][kx],
// Y MN-major [groups*K][b] (K = b), with an optional epilogue mode and K segments.
umma::Gemm block_gemm(const void* X, int64_t x_rows, const void* Y, int64_t y_rows, int64_t groups,
                      int64_t b, int64_t K, const char* name) {
  umma::Gemm g;
  g.M = b; g.N = b; g.K = K; g.groups = groups;
  g.A = X; g.a_rows = x_rows; g.a_cols = b; g.a_ld = b; g.a_mn = false; g.a_gm = b; g.a_gk = 0;
  g.B = Y; g.b_rows = y_rows; g.b_cols = b; g.b_ld = b; g.b_mn = true; g.b_gn = 0; g.b_gk = b;
  g.out_f32 = true; g.ldc = b; g.c_gs = b * b;
  g.name = name;
  return g;
}

// x_hi y_hi + x_hi y_lo + x_lo y_hi over three K segments: X = [X_hi; X_lo] and
// Y = [Y_hi; Y_lo] stacked as [2 nb b][b] (the lo halves nb*b rows below the hi halves)
void three_pass(umma::Gemm& g, int64_t nb, int64_t b) {
  g.K = 3 * b;
  g.nseg = 3;
  g.a_dy[0] = 0; g.a_dy[1] = 0; g.a_dy[2] = nb * b;
  g.b_dy[0] = 0; g.b_dy[1] = nb * b; g.b_dy[2] = 0;
}

// These launches hold a few tens of b x b products (one wave or two), so their time is that of
// the busiest SM: waves x (tile area + a fixed cost per tile), minimised over 256 x 256 CTA-pair
// tiles (half the operand traffic per MMA) and 128 x 256 / 128 / 64 single-CTA tiles, ties to
// the larger tile. The fixed cost is a 128 x 128 tile's worth for plain stores and a quarter of
// that for the fused epilogues, whose per-element work spreads over more SMs with smaller
// tiles (measured at b = 256 over 16 blocks and b = 512 over 20; b = 512 over 36 blocks keeps
// the pairs).
// 0: CTA-pair tiles; otherwise the single-CTA tile width; -1: not covered
int block_tile_choice(const umma::Gemm& g) {
  if (!umma::supported(g)) return -1;
  const int64_t sms = umma::sm_count();
  const int64_t fixed = g.epi.mode == umma::kEpiStore ? 128 * 128 : 128 * 32;
  int64_t best = -1;
  int best_bn = 0;   // 0: CTA pairs
  if (umma::pair_supported(g)) {
    const int64_t tiles = g.groups * ((g.M + 255) / 256) * (g.N / 256);
    best = (tiles + sms / 2 - 1) / (sms / 2) * (128 * 256 + fixed);
  }
  for (int bn : {256, 128, 64}) {
    if (g.N % bn) continue;
    const int64_t tiles = g.groups * ((g.M + 127) / 128) * (g.N / bn);
    const int64_t cost = (tiles + sms - 1) / sms * (128 * bn + fixed);
    if (best < 0 || cost < best) {
      best = cost;
      best_bn = bn;
    }
  }
  return best_bn;
}

cudaError_t run_block_gemm(const umma::Gemm& g, cudaStream_t s) {
  const int bn = block_tile_choice(g);
  if (bn < 0) return cudaErrorNotSupported;
  if (bn == 0) return umma::gemm_pair(g, s);
  umma::Gemm h = g;
  h.bn = bn;
  return umma::gemm(h, s);
}

// Two dependent products of a chain in one launch of the CTA-pair kernel, where both would run
// on CTA pairs alone: `second`'s groups follow `first`'s, and a tile of second-product group g
// loads its operands only once every tile of block g % nb of the first product has stored its
// results (deps, nb counts cleared by the pass before). The blocks pipeline through the two
// products instead of the second launch waiting for the whole first one. Returns false (nothing
// launched) where it does not apply.
bool run_chain(const umma::Gemm& first, const umma::Gemm& second, int64_t nb, int* deps,
               cudaStream_t s, cudaError_t* err) {
  if (!deps || block_tile_choice(first) != 0 || block_tile_choice(second) != 0) return false;
  umma::Gemm g = first;
  g.groups = first.groups + second.groups;
  g.groups_1 = first.groups;
  g.A2 = second.A; g.a2_rows = second.a_rows; g.a2_cols = second.a_cols; g.a2_ld = second.a_ld;
  g.B2 = second.B; g.b2_rows = second.b_rows; g.b2_cols = second.b_cols; g.b2_ld = second.b_ld;
  g.epi2 = second.epi;
  g.has_epi2 = true;
  g.C = second.C;
  g.c_rel2 = true;
  g.deps = deps;
  g.dep_blocks = (int)nb;
  // first-product epilogue warps per block: its pair tiles x 2 CTAs x 4 warps
  g.dep_target = (int)(((first.M + 255) / 256) * (first.N / 256) * 8);
  if (first.a_mn != second.a_mn || first.b_mn != second.b_mn || first.out_f32 != second.out_f32 ||
      first.nseg != second.nseg || !umma::pair_supported(g))
    return false;
  for (int k = 0; k < 3; ++k)
    if (first.a_dy[k] != second.a_dy[k] || first.b_dy[k] != second.b_dy[k] ||
        first.a_dx[k] != second.a_dx[k] || first.b_dx[k] != second.b_dx[k])
      return false;
  *err = umma::gemm_pair(g, s);
  return true;
}

#define POETX_TRY(x)                  \
  do {                                \
    cudaError_t e_ = (x);             \
    if (e_ != cudaSuccess) return e_; \
  } while (0)

}  // namespace

bool tc_blocks_supported(int64_t b) { return b % 128 == 0 && b >= 128; }

size_t cnp_tc_ws_bytes(int64_t nb, int64_t b) {
  // [Q_hi; Q_lo], [S_hi; S_lo], [H_hi; H_lo], per-block counts of the two-product launch
  return 3 * align_up((size_t)(2 * nb * b * b) * 2, 256) + align_up((size_t)nb * 4, 256);
}

cudaError_t cnp_build_tc(const BlockRuns& r, int64_t b, void* ws, cudaStream_t s) {
  const int64_t nb = r.total();
  if (nb == 0) return cudaSuccess;
  const int64_t bb = b * b;
  Arena a(ws, cnp_tc_ws_bytes(nb, b));
  auto* Qst = static_cast<__nv_bfloat16*>(a.take((size_t)(2 * nb * bb) * 2));
  auto* Sst = static_cast<__nv_bfloat16*>(a.take((size_t)(2 * nb * bb) * 2));
  auto* Hst = static_cast<__nv_bfloat16*>(a.take((size_t)(2 * nb * bb) * 2));
  auto* deps = static_cast<int*>(a.take((size_t)nb * 4));
  const dim3 grid = pair_grid(nb, b);
  {
    TraceScope t("cnp_split_Q", s);
    POETX_TRY(launch_k(split_q_kernel, grid, dim3(kTileThreads), 0, s, r, (int)b, Qst,
                       Qst + nb * bb, deps, (int)nb));
  }
  umma::Gemm qq = block_gemm(Qst, 2 * nb * b, Qst, 2 * nb * b, nb, b, b, "umma_cnp_QQ");
  three_pass(qq, nb, b);
  qq.epi.mode = umma::kEpiCnpS;
  qq.epi.b = (int)b;
  qq.epi.qh = Qst; qq.epi.ql = Qst + nb * bb;
  qq.epi.o[0] = Sst; qq.epi.o[1] = Sst + nb * bb; qq.epi.o[2] = Hst; qq.epi.o[3] = Hst + nb * bb;
  umma::Gemm sh = block_gemm(Sst, 2 * nb * b, Hst, 2 * nb * b, nb, b, b, "umma_cnp_SH");
  three_pass(sh, nb, b);
  sh.epi.mode = umma::kEpiCnpG;
  sh.epi.b = (int)b;
  sh.epi.qh = Qst; sh.epi.ql = Qst + nb * bb;
  sh.epi.nruns = kMaxRuns;
  for (int k = 0, end = 0; k < kMaxRuns; ++k) {
    end += r.nb[k];
    sh.epi.run_end[k] = end;
    sh.epi.g[k] = r.g[k];
    sh.epi.g_lp[k] = r.g_lp[k];
  }
  // S = Q Q, then G = I + 2Q + S H: one launch where both run on CTA pairs
  umma::Gemm chain = qq;
  chain.name = "umma_cnp_QQ_SH";
  cudaError_t ce = cudaSuccess;
  if (run_chain(chain, sh, nb, deps, s, &ce)) return ce;
  POETX_TRY(run_block_gemm(qq, s));
  return run_block_gemm(sh, s);
}

size_t dq_tc_ws_bytes(int64_t nb, int64_t b) {
  const size_t h = align_up((size_t)(nb * b * b) * 2, 256);
  const size_t f = align_up((size_t)(nb * b * b) * 4, 256);
  return 6 * h + 3 * f + align_up((size_t)nb * 4, 256);
}

cudaError_t dq_from_dg_tc(const BlockRuns& r, int64_t b, float* dG, void* ws, cudaStream_t s) {
  const int64_t nb = r.total();
  if (nb == 0) return cudaSuccess;
  const int64_t bb = b * b;
  // element offsets of 256-byte-aligned slices: nb * b * b is a multiple of 128 here
  Arena a(ws, dq_tc_ws_bytes(nb, b));
  const size_t hb = (size_t)(nb * bb) * 2, fb = (size_t)(nb * bb) * 4;
  auto* Qh = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* Ql = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* hst = static_cast<__nv_bfloat16*>(a.take(3 * hb));   // S_h, dG_h, SmQ, contiguous
  __nv_bfloat16* Sh = hst;
  __nv_bfloat16* dGh = hst + nb * bb;
  __nv_bfloat16* SmQ = hst + 2 * nb * bb;
  auto* Zh = static_cast<__nv_bfloat16*>(a.take(hb));
  auto* fst = static_cast<float*>(a.take(2 * fb));            // Hbar, T1, contiguous
  float* Hb = fst;
  float* T1 = fst + nb * bb;
  auto* V = static_cast<float*>(a.take(fb));
  auto* deps = static_cast<int*>(a.take((size_t)nb * 4));
  const dim3 grid = pair_grid(nb, b);
  const int bi = (int)b;
  {
    TraceScope t("dq_prep", s);
    POETX_TRY(launch_k(dq_prep_kernel, grid, dim3(kTileThreads), 0, s, r, bi, dG, Qh, Ql, dGh,
                       deps, (int)nb));
  }
  umma::Gemm qq = block_gemm(Qh, nb * b, Qh, nb * b, nb, b, b, "umma_dq_QQ");
  qq.epi.mode = umma::kEpiDqS;
  qq.epi.b = bi;
  qq.epi.qh = Qh; qq.epi.ql = Ql;
  qq.epi.o[0] = Sh; qq.epi.o[1] = SmQ;
  // Hbar_g = S_g dG_g (groups 0..nb-1) and T1_g = dG_g SmQ_g (groups nb..2nb-1)
  umma::Gemm sdg = block_gemm(Sh, 2 * nb * b, dGh, 2 * nb * b, 2 * nb, b, b, "umma_dq_SdG_dGH");
  sdg.C = fst;
  {
    // S = Q Q, then S dG and dG (S - 2Q): one launch where all run on CTA pairs
    umma::Gemm chain = qq;
    chain.name = "umma_dq_QQ_SdG_dGH";
    cudaError_t ce = cudaSuccess;
    if (run_chain(chain, sdg, nb, deps, s, &ce)) {
      POETX_TRY(ce);
    } else {
      POETX_TRY(run_block_gemm(qq, s));
      POETX_TRY(run_block_gemm(sdg, s));
    }
  }
  {
    TraceScope t("dq_mid", s);
    POETX_TRY(launch_k(dq_mid_kernel, grid, dim3(kTileThreads), 0, s, (const float*)dG,
                       (const float*)T1, (const float*)Hb, bi, Zh, V));
  }
  {
    umma::Gemm g = block_gemm(Zh, nb * b, Qh, nb * b, nb, b, b, "umma_dq_ZQ");
    g.C = T1;
    POETX_TRY(run_block_gemm(g, s));
  }
  TraceScope t("dq_pack", s);
  return launch_k(dq_pack_kernel, grid, dim3(kTileThreads), 0, s, r, (const float*)V,
                  (const float*)T1, bi);
}

}  // namespace poetx
