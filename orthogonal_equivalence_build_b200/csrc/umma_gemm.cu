// bf16 x bf16 -> fp32 GEMM on the 5th-generation tensor cores (tcgen05 / TMEM / TMA), sm_100a.
//
// Two kernels serve every bf16 contraction of the layer: the W0' products (dense), the
// batch-wise block-diagonal products A_j G_j ("POET-X" blog §第三斧: each b x b block is one
// batch element), the per-block gradients dG_j = A_j^T B_j (contraction over tokens, split-K)
// and the b x b products of the Cayley-Neumann blocks and their gradient:
//   umma_gemm_kernel       one CTA per 128 x BN tile (used where the pair tiling does not fit);
//   umma_gemm_pair_kernel  two-CTA clusters on 256 x 256 tiles (tcgen05.mma.cta_group::2), the
//                          main path; variants: int8 B dequantised in shared memory (8-bit
//                          W0'), fused elementwise epilogues (CNP / dq), bf16 outputs through TMA
//                          bulk tensor stores, K segments, band rasters.
//
// Structure (persistent, warp-specialised, 192 threads (320 with the int8 converters), one CTA
// per SM):
//   warp 0      TMA producer: streams 128 x 64 A and BN x 64 B tiles into a STAGES-deep ring of
//               128-byte-swizzled shared-memory stages (mbarrier complete_tx).
//   warp 1      owns the TMEM allocation (2 x BN fp32 columns: two accumulators) and one lane
//               issues tcgen05.mma (M = 128, N = BN, K = 16 per instruction); tcgen05.commit
//               frees a stage when its MMAs retire and publishes a finished accumulator.
//   warps 2..5  epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes 32*(w%4)..+31),
//               convert, store; then hand the accumulator back, so tile i's epilogue overlaps
//               tile i+1's main loop.
// Operands may be K-major (K contiguous) or MN-major (M/N contiguous); the shared-memory matrix
// descriptors follow the canonical SW128 layouts (K-major: 8-row groups 1024 B apart; MN-major:
// 64-element chunks LBO apart, 8-row K groups 1024 B apart).
// Every mbarrier wait is bounded (a few seconds of %globaltimer); on expiry the kernel records
// a code in the device error word, lets the other roles leave their loops, waits (bounded) for
// its own copies and MMAs in flight, frees TMEM and returns.
#include "umma_gemm.h"

#include <cuda.h>

#include <algorithm>
#include <mutex>

namespace poetx {
namespace umma {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s per drain wait

enum : int {
  kErrProducer = 0x101, kErrMma = 0x102, kErrEpilogue = 0x103, kErrConvert = 0x104,
  kErrDependency = 0x105   // a second-product tile's inputs were not published in time
};

struct Params {
  int M, N, K, groups, splits;
  int tiles_m, tiles_n, kblocks_per_split, total_tiles;
  int a_gm, a_gk, b_gn, b_gk;   // per-group coordinate offsets (elements)
  int nseg, kb_per_seg;         // K segments (see umma_gemm.h)
  int a_dx[3], a_dy[3], b_dx[3], b_dy[3];
  void* C;
  long long ldc, c_gs, c_split;
  Epi epi;
  int* err;
  unsigned long long epi_wait_ns;   // limit of the epilogue's accumulator wait
};

// TMA coordinate shifts of K block kb: k restarts at 0 in every segment.
struct KCoord {
  int k, adx, ady, bdx, bdy;
};
template <typename P>
__device__ __forceinline__ KCoord k_coord(const P& p, int kb) {
  KCoord c{kb * BK, 0, 0, 0, 0};
  if (p.nseg > 1) {
    const int s = kb / p.kb_per_seg;
    c.k = (kb - s * p.kb_per_seg) * BK;
    c.adx = p.a_dx[s]; c.ady = p.a_dy[s]; c.bdx = p.b_dx[s]; c.bdy = p.b_dy[s];
  }
  return c;
}

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of a phase (never suspends the thread, unlike try_wait).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// The same test with cluster-scope acquire: for barriers that other CTAs of the cluster
// release into (their arrivals order their own shared-memory writes before this thread's reads).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctl {
  volatile int* abort;
  int* err;
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Wait until *cnt >= target (a count other CTAs of the same launch publish with release adds);
// false if the wait expired (code recorded, CTA aborting).
__device__ __noinline__ bool wait_count(const int* cnt, int target, Ctl c, int code,
                                        uint64_t limit_ns) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(cnt) >= target) return true;
    if ((it & 15) == 0 && global_ns() - t0 > limit_ns) {
      *c.abort = 1;
      if (code) atomicCAS(c.err, 0, code);
      return false;
    }
  }
}

// Wait for `parity` on `bar`; false if the CTA is aborting (unless stop_on_abort is false) or
// the wait expired.
template <bool CLUSTER = false>
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, Ctl c, int code,
                                          uint64_t limit_ns, bool stop_on_abort = true) {
  auto test = [&] { return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (test()) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (test()) return true;
    if ((it & 31) == 0) {
      if (stop_on_abort && *c.abort) return false;
      if (global_ns() - t0 > limit_ns) {
        *c.abort = 1;
        if (code) atomicCAS(c.err, 0, code);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, SW128, sm_100 format (version 1 at bit 46, layout 2 at 61).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, M = 128, N = BN.
template <int BN, bool A_MN, bool B_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
         ((B_MN ? 1u : 0u) << 16) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct TileCoord {
  int g, mb, nb, split;
};

__device__ __forceinline__ TileCoord decode_tile(const Params& p, int tile) {
  constexpr int GROUP_M = 16;
  const int per_group = p.tiles_m * p.tiles_n;
  const int per_split = per_group * p.groups;
  TileCoord t;
  t.split = tile / per_split;
  const int r = tile - t.split * per_split;
  t.g = r / per_group;
  const int local = r - t.g * per_group;
  const int band = local / (GROUP_M * p.tiles_n);
  const int first_m = band * GROUP_M;
  const int gm = min(GROUP_M, p.tiles_m - first_m);
  const int within = local - band * GROUP_M * p.tiles_n;
  t.mb = first_m + within % gm;
  t.nb = within / gm;
  return t;
}

// Epilogue of one warp's 32 accumulator rows: TMEM -> registers -> a swizzled 8 KB stage in
// shared memory -> global memory, 64 columns at a time. Each store instruction of the warp writes
// whole row segments (4 rows x 128 B for bf16, 2 rows x 256 B for fp32) instead of one 16 B piece
// of 32 different rows. tmem_row0: TMEM address of this warp's lane quarter at the tile's first
// column; off0: element offset of the warp's first row in C at the tile's first column.
constexpr int kEpiStageBytes = 8192;

// Elementwise step after a grouped b x b product at (g; i, j..j+7): acc = the eight sums, q = Q.
// off = g*b*b + i*b + j (elements), bb = b*b.
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ void st8_split(__nv_bfloat16* hi, __nv_bfloat16* lo, const float (&x)[8]) {
  float h[8], l[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    h[k] = __bfloat162float(__float2bfloat16_rn(x[k]));
    l[k] = x[k] - h[k];
  }
  *reinterpret_cast<uint4*>(hi) = pack8(h);
  *reinterpret_cast<uint4*>(lo) = pack8(l);
}
// Run of CNP output block g (kEpiCnpG) and the first block of that run: resolved once per tile.
__device__ __forceinline__ int epi_run(const Epi& e, int g, int& first) {
  int run = 0;
  first = 0;
#pragma unroll 1
  while (run + 1 < e.nruns && g >= e.run_end[run]) first = e.run_end[run++];
  return run;
}

__device__ __forceinline__ void epi_apply8(const Epi& e, int g, int i, int j, long long off,
                                           long long bb, const float (&acc)[8],
                                           const float (&q)[8], int run, int first) {
  if (e.mode == kEpiCnpS) {
    float h[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) h[k] = (i == j + k ? 2.f : 0.f) + 2.f * q[k] + acc[k];
    st8_split(e.o[0] + off, e.o[1] + off, acc);
    st8_split(e.o[2] + off, e.o[3] + off, h);
  } else if (e.mode == kEpiCnpG) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = (i == j + k ? 1.f : 0.f) + 2.f * q[k] + acc[k];
    const long long loc = off - (long long)first * bb;
    if (e.g[run]) {
      float4* gp = reinterpret_cast<float4*>(e.g[run] + loc);
      gp[0] = make_float4(v[0], v[1], v[2], v[3]);
      gp[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    if (e.g_lp[run]) *reinterpret_cast<uint4*>(e.g_lp[run] + loc) = pack8(v);
  } else if (e.mode == kEpiDqS) {
    float m[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = acc[k] - 2.f * q[k];
    *reinterpret_cast<uint4*>(e.o[0] + off) = pack8(acc);
    *reinterpret_cast<uint4*>(e.o[1] + off) = pack8(m);
  }
}

template <bool OUT_F32>
__device__ __forceinline__ void epilogue_warp_rows(uint32_t tmem_row0, int ncols,
                                                   uint8_t* __restrict__ stage, void* C,
                                                   long long off0, long long ldc, int nlive,
                                                   int lane) {
  constexpr int ESZ = OUT_F32 ? 4 : 2;
  constexpr int ROWB = 64 * ESZ;      // bytes of one row per 64-column chunk
  constexpr int V16 = ROWB / 16;      // 16-byte pieces per row chunk: 8 (bf16) or 16 (fp32)
  constexpr int RPI = 32 / V16;       // rows per store instruction: 4 or 2
  uint8_t* myrow = stage + lane * ROWB;
  const int sub = lane % V16, rsub = lane / V16;
  char* Cb = static_cast<char*>(C);
#pragma unroll 1
  for (int c = 0; c < ncols; c += 64) {
    uint32_t r0[32], r1[32];
    tmem_ld32(tmem_row0 + (uint32_t)c, r0);
    tmem_ld32(tmem_row0 + (uint32_t)(c + 32), r1);
    if constexpr (OUT_F32) {
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        const uint32_t* src = v < 8 ? &r0[4 * v] : &r1[4 * (v - 8)];
        *reinterpret_cast<uint4*>(myrow + ((v ^ (lane & 15)) * 16)) =
            make_uint4(src[0], src[1], src[2], src[3]);
      }
    } else {
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint32_t* src = v < 4 ? &r0[8 * v] : &r1[8 * (v - 4)];
        *reinterpret_cast<uint4*>(myrow + ((v ^ (lane & 7)) * 16)) = make_uint4(
            pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
            pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
            pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
            pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 32 / RPI; ++i) {
      const int r = i * RPI + rsub;
      if (r < nlive) {
        const uint4 v =
            *reinterpret_cast<const uint4*>(stage + r * ROWB + ((sub ^ (r & (V16 - 1))) * 16));
        *reinterpret_cast<uint4*>(Cb + (off0 + (long long)r * ldc + c) * ESZ + sub * 16) = v;
      }
    }
    __syncwarp();
  }
}

// bf16 epilogue through the tensor-memory accelerator: each 32-row x 64-column chunk of a warp is
// packed into the 128-byte-swizzled layout of one half of the warp's 8 KB stage and written by
// one bulk tensor store (rows beyond the tensor are clipped by the copy). The two halves
// alternate, so a chunk is packed while the previous chunk's store still reads its half.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {   // at most N groups still reading shared
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() {    // every group's writes complete
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void epilogue_tma_bf16(uint32_t tmem_row0, int ncols,
                                                  uint8_t* __restrict__ stage,
                                                  const CUtensorMap* map, int x0, int y0,
                                                  int lane, int& chunk) {
#pragma unroll 1
  for (int c = 0; c < ncols; c += 64, ++chunk) {
    uint8_t* half = stage + (chunk & 1) * 4096;
    if (lane == 0) bulk_wait_read<1>();   // the store that last read this half is done reading
    __syncwarp();
    uint32_t r0[32], r1[32];
    tmem_ld32(tmem_row0 + (uint32_t)c, r0);
    tmem_ld32(tmem_row0 + (uint32_t)(c + 32), r1);
    uint8_t* myrow = half + lane * 128;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint32_t* src = v < 4 ? &r0[8 * v] : &r1[8 * (v - 4)];
      *reinterpret_cast<uint4*>(myrow + ((v ^ (lane & 7)) * 16)) = make_uint4(
          pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
          pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
          pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
          pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the copy
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(map, smem_u32(half), x0 + c, y0);
      bulk_commit();
    }
  }
}

// Fused elementwise epilogue of a grouped b x b product (epilogue modes). Each 32-column chunk of
// the warp's 32 accumulator rows comes out of TMEM one row per lane, goes through one half of the
// warp's shared-memory stage (16-byte units of row r at unit ^ (r & 7): conflict-free both ways)
// and is read back four lanes per row, eight consecutive columns each, so that every Q load and
// output store of a warp covers 8 rows x 64 (bf16) or 128 (fp32) contiguous bytes. Lane l takes
// rows 8i + l/4 (i = 0..3) and columns 8 (l % 4) .. + 7 of the chunk. The Q values of a chunk
// (16-byte loads of the hi and lo parts) are requested one chunk ahead; the caller requests
// chunk 0 (fused_q_load) before it waits for the accumulator, so those loads overlap the main
// loop.
struct FusedQ {
  uint4 h[4], l[4];
};
__device__ __forceinline__ long long fused_base(const Epi& e, int g, int row0, int col0, int lane) {
  return (long long)g * e.b * e.b + (long long)row0 * e.b + col0 + 8 * (lane & 3);
}
__device__ __forceinline__ void fused_q_load(const Epi& e, long long base, int c, int nlive,
                                             int lane, FusedQ& q) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = 8 * i + (lane >> 2);
    const bool live = rr < nlive;
    const long long off = base + (long long)rr * e.b + c;
    q.h[i] = live ? __ldg(reinterpret_cast<const uint4*>(e.qh + off)) : make_uint4(0, 0, 0, 0);
    q.l[i] = (live && e.ql) ? __ldg(reinterpret_cast<const uint4*>(e.ql + off))
                            : make_uint4(0, 0, 0, 0);
  }
}
__device__ __forceinline__ void epilogue_fused(uint32_t tmem_row0, int ncols,
                                               uint8_t* __restrict__ stage, const Epi& e, int g,
                                               int row0, int col0, int nlive, int lane,
                                               FusedQ& q) {
  const long long bb = (long long)e.b * e.b;
  const long long base = fused_base(e, g, row0, col0, lane);
  const int cg = lane & 3;
  int first = 0;
  const int run = e.mode == kEpiCnpG ? epi_run(e, g, first) : 0;
#pragma unroll 1
  for (int cc = 0, half = 0; cc < ncols; cc += 32, half ^= 1) {
    uint32_t r[32];
    tmem_ld32(tmem_row0 + (uint32_t)cc, r);
    uint8_t* buf = stage + half * 4096;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      *reinterpret_cast<uint4*>(buf + lane * 128 + ((u ^ (lane & 7)) << 4)) =
          make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 8 * i + (lane >> 2);
      const uint8_t* row = buf + rr * 128;
      const float4 a0 = *reinterpret_cast<const float4*>(row + (((2 * cg) ^ (rr & 7)) << 4));
      const float4 a1 = *reinterpret_cast<const float4*>(row + (((2 * cg + 1) ^ (rr & 7)) << 4));
      if (rr < nlive) {
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        float qq[8];
        const uint32_t hw[4] = {q.h[i].x, q.h[i].y, q.h[i].z, q.h[i].w};
        const uint32_t lw[4] = {q.l[i].x, q.l[i].y, q.l[i].z, q.l[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&hw[k]);
          const __nv_bfloat162 l2 = *reinterpret_cast<const __nv_bfloat162*>(&lw[k]);
          qq[2 * k] = __low2float(h2) + __low2float(l2);
          qq[2 * k + 1] = __high2float(h2) + __high2float(l2);
        }
        epi_apply8(e, g, row0 + rr, col0 + cc + 8 * cg, base + (long long)rr * e.b + cc, bb, a,
                   qq, run, first);
      }
    }
    if (cc + 32 < ncols) fused_q_load(e, base, cc + 32, nlive, lane, q);
  }
  __syncwarp();   // every lane's reads of the stage are done before it is written again
}

template <int BN, bool A_MN, bool B_MN, bool OUT_F32, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
umma_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                 const __grid_constant__ Params p) {
  constexpr int A_BYTES = BM * BK * 2;
  constexpr int B_BYTES = BN * BK * 2;
  constexpr uint32_t TMEM_COLS = 2 * BN;  // power of two: 128, 256 or 512
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + STAGES * A_BYTES;
  uint8_t* sepi = sb + STAGES * B_BYTES;   // 4 epilogue warps x 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sepi + 4 * kEpiStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctl ctl{abort_flag, p.err};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(tfull + a), 1);
      mbar_init(smem_u32(tempty + a), 4);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_wait();      // operands and outputs may belong to the previous kernel of the stream
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
        const TileCoord tc = decode_tile(p, tile);
        const int kb0 = tc.split * p.kblocks_per_split;
        const int kb1 = min(kb0 + p.kblocks_per_split, (p.K + BK - 1) / BK);
        const int am = tc.g * p.a_gm + tc.mb * BM, ak = tc.g * p.a_gk;
        const int bn = tc.g * p.b_gn + tc.nb * BN, bk = tc.g * p.b_gk;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_bounded(smem_u32(empty + s), ph ^ 1u, ctl, kErrProducer, kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full + s);
          mbar_expect_tx(fb, A_BYTES + B_BYTES);
          const KCoord kc = k_coord(p, kb);
          const int k = kc.k;
          if constexpr (A_MN) {
#pragma unroll
            for (int h = 0; h < BM / 64; ++h)
              tma_load_2d(smem_u32(sa + s * A_BYTES + h * 64 * BK * 2), &tma_a, fb,
                          am + 64 * h + kc.adx, ak + k + kc.ady);
          } else {
            tma_load_2d(smem_u32(sa + s * A_BYTES), &tma_a, fb, ak + k + kc.adx, am + kc.ady);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(smem_u32(sb + s * B_BYTES + h * 64 * BK * 2), &tma_b, fb,
                          bn + 64 * h + kc.bdx, bk + k + kc.bdy);
          } else {
            tma_load_2d(smem_u32(sb + s * B_BYTES), &tma_b, fb, bk + k + kc.bdx, bn + kc.bdy);
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA leaves
        for (int j = max(0, it - STAGES); j < it; ++j)
          wait_bounded(smem_u32(full + j % STAGES), (uint32_t)(j / STAGES) & 1u, ctl, 0,
                       kDrainLimitNs);
      }
    }
    __syncwarp();  // reconverge before the block-wide barriers below
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<BN, A_MN, B_MN>();
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++tcount) {
        const TileCoord tc = decode_tile(p, tile);
        const int kb0 = tc.split * p.kblocks_per_split;
        const int kb1 = min(kb0 + p.kblocks_per_split, (p.K + BK - 1) / BK);
        const int acc = tcount & 1;
        const uint32_t use = (uint32_t)(tcount >> 1);
        if (!wait_bounded(smem_u32(tempty + acc), (use & 1u) ^ 1u, ctl, kErrMma, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_bounded(smem_u32(full + s), ph, ctl, kErrMma, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sa + s * A_BYTES), b0 = smem_u32(sb + s * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc(a0 + kk * 2048, 64 * BK * 2, 1024)
                                     : smem_desc(a0 + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc(b0 + kk * 2048, 64 * BK * 2, 1024)
                                     : smem_desc(b0 + kk * 32, 16, 1024);
            umma_bf16(d, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(empty + s));
        }
        if (!ok) break;
        umma_commit(smem_u32(tfull + acc));
      }
      // every MMA this thread issued has retired once `drain` completes
      umma_commit(smem_u32(drain));
      wait_bounded(smem_u32(drain), 0, ctl, ok ? kErrMma : 0, ok ? kWaitLimitNs : kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    int tcount = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++tcount) {
      const TileCoord tc = decode_tile(p, tile);
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      const int row0 = tc.mb * BM + quarter * 32;   // first row of this warp
      const int nlive = max(0, min(32, p.M - row0));
      const bool fused = OUT_F32 && p.epi.mode != kEpiStore;
      FusedQ q0;
      if (fused)
        fused_q_load(p.epi, fused_base(p.epi, tc.g, row0, tc.nb * BN, lane), 0, nlive, lane, q0);
      if (!wait_bounded(smem_u32(tfull + acc), use & 1u, ctl, kErrEpilogue, p.epi_wait_ns))
        break;
      tc_fence_after();
      const long long off0 = (long long)tc.split * p.c_split + (long long)tc.g * p.c_gs +
                             (long long)row0 * p.ldc + (long long)tc.nb * BN;
      const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      if (fused)
        epilogue_fused(trow, BN, sepi + (warp - 2) * kEpiStageBytes, p.epi, tc.g, row0,
                       tc.nb * BN, nlive, lane, q0);
      else
        epilogue_warp_rows<OUT_F32>(trow, BN, sepi + (warp - 2) * kEpiStageBytes, p.C, off0,
                                    p.ldc, nlive, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(tempty + acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ CTA-pair kernel
// The same GEMM on a cluster of two CTAs on two SMs with tcgen05.mma.cta_group::2: one MMA
// instruction computes a 256 x 256 x 16 product; CTA r of the pair holds rows [128r, 128r+128)
// of the A tile and rows [128r, 128r+128) of the B tile (N) in its own shared memory and receives
// rows [128r, 128r+128) x 256 of the accumulator in its own TMEM. Per CTA and 64-deep stage that
// is 32 KB of operands for 128 x 256 x 64 outputs, two thirds of the single-CTA 128 x 256 tile's
// 48 KB, which is what bounds that tile by L2 bandwidth.
//   Both producers load their halves with TMA; the bytes of both complete the transaction count
//   of the leader's (rank 0) full barrier. The leader's single MMA thread issues the pair MMAs
//   and commits with a multicast to both CTAs' empty / accumulator-full barriers. Epilogue warps
//   of both CTAs read their own TMEM and arrive on the leader's accumulator-empty barrier.
//   No TMA load is multicast.
struct PairParams {
  int M, N, K, groups, splits;
  int tiles_m, tiles_n, kblocks_per_split, total_tiles;   // tiles of 256 x 256
  int a_gm, a_gk, b_gn, b_gk;
  int nseg, kb_per_seg;
  int a_dx[3], a_dy[3], b_dx[3], b_dy[3];
  void* C;
  long long ldc, c_gs, c_split;
  const float* b_scale;   // int8 B only: one scale per column of the stored B tensor
  int g2;                 // first group read from the second operand pair (groups: none)
  int raster, band;       // tile order within a group: 0 = bands of `band` pair-rows, N inner;
                          // 1 = bands of `band` pair-columns, N fastest inside a band
  Epi epi;
  int* err;
  unsigned long long epi_wait_ns;   // limit of the epilogue's accumulator wait
  // 256 x 512 kernel: tiles from narrow_from on are half-width (256 columns): the last partial
  // wave's tiles, each split in two, so that wave takes half as long (see launch_wide_t)
  int narrow_from;
  // Two dependent products in one launch (256 x 256 kernel): groups from g2 on form the second
  // product, with their own epilogue epi2 and, with c_rel2, output groups counted from g2. When
  // deps is set, second-product group g waits, before its operands are loaded, until
  // deps[(g - g2) % dep_blocks] reaches dep_target: the count of first-product epilogue warps of
  // that group whose stores are visible (each warp adds one after its stores).
  Epi epi2;
  int* deps;
  int dep_target, dep_blocks, c_rel2;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
               "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive once on `bar` in every CTA of the pair when this thread's MMAs have retired
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// Arrive on a barrier of a CTA of the cluster, ordering this thread's earlier memory writes
// before it (cluster scope: the consumer may read them from another CTA).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
// The same arrive without ordering earlier memory operations: for an accumulator handed back
// after tcgen05.wait::ld (its TMEM reads are complete), so the epilogue's global stores need not
// be acknowledged before the MMA may reuse the accumulator.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

// Instruction descriptor for the pair MMA: M = 256, N = 256.
template <bool A_MN, bool B_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc_pair() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
         ((B_MN ? 1u : 0u) << 16) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// Tile order (L2 reuse): raster 0 sweeps all N tiles of a band of `band` pair-rows (the band's
// A rows stay in L2 while B streams); raster 1 sweeps all M tiles of a band of `band`
// pair-columns with the band's columns innermost (the band's B stays in L2 while each A row
// tile is shared by the columns of the band at once).
__device__ __forceinline__ TileCoord decode_pair_tile(const PairParams& p, int tile) {
  const int per_group = p.tiles_m * p.tiles_n;
  const int per_split = per_group * p.groups;
  TileCoord t;
  t.split = tile / per_split;
  const int r = tile - t.split * per_split;
  t.g = r / per_group;
  const int local = r - t.g * per_group;
  if (p.raster == 0) {
    const int band = local / (p.band * p.tiles_n);
    const int first_m = band * p.band;
    const int gm = min(p.band, p.tiles_m - first_m);
    const int within = local - band * p.band * p.tiles_n;
    t.mb = first_m + within % gm;
    t.nb = within / gm;
  } else {
    const int band = local / (p.band * p.tiles_m);
    const int first_n = band * p.band;
    const int gn = min(p.band, p.tiles_n - first_n);
    const int within = local - band * p.band * p.tiles_m;
    t.nb = first_n + within % gn;
    t.mb = within / gn;
  }
  return t;
}

// int8 B operand (8-bit weight storage, "POET-XQ"): B is stored as int8 codes with one fp32
// scale per column of the stored tensor. The producer streams the int8 tile (8 KB per CTA and
// stage) into a separate staging ring; converter warps turn it into the bf16 operand
// bf16(code * scale) in the 128-byte-swizzled stage the MMA reads, then arrive on the leader's
// full barrier (which also counts the A bytes of both CTAs). The MMA and epilogue are unchanged.
// The converters form kConvGroups groups of kConvWarpsPerGroup warps that take the K blocks in
// turn: one group converts a block in about three MMA blocks' time (its loads, the arithmetic
// and the swizzled stores follow each other), so three groups keep up with the MMA (two paced
// it at about 1500 cycles per 512-cycle block).
constexpr int kConvGroups = 3;
constexpr int kConvWarpsPerGroup = 2;
constexpr int kPairConvThreads = 32 * kConvWarpsPerGroup * kConvGroups;

// float(q) for a signed byte q without a conversion instruction: q + 128 = byte ^ 0x80 placed in
// the low mantissa bits of 2^23 (0x4B000000) is the float 2^23 + 128 + q; subtracting 2^23 + 128
// is exact. Then the fp32 product with the column scale (round to nearest), as in the reference
// definition bf16(fp32(q) * s). The subtraction and the product run on packed pairs
// (add / mul .rn.f32x2: the IEEE fp32 operation on each lane, half the instructions).
__device__ __forceinline__ uint64_t f32x2_pack(uint32_t lo, uint32_t hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return pack_bf16x2(__uint_as_float(lo), __uint_as_float(hi));
}
__device__ __forceinline__ uint32_t biased_byte(uint32_t flipped_word, int byte) {
  return __byte_perm(flipped_word, 0x4B000000u, 0x7540u | (uint32_t)byte);   // 2^23 + 128 + q
}
// sc2[p]: the scales of elements 2p and 2p + 1, packed
__device__ __forceinline__ uint4 dequant8(uint2 w, const uint64_t (&sc2)[4]) {
  const uint32_t x[2] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u};
  const uint64_t bias = f32x2_pack(__float_as_uint(-8388736.0f), __float_as_uint(-8388736.0f));
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t xw = x[p >> 1];
    const int b0 = 2 * (p & 1);
    const uint64_t q2 = f32x2_add(f32x2_pack(biased_byte(xw, b0), biased_byte(xw, b0 + 1)), bias);
    o[p] = f32x2_to_bf16x2(f32x2_mul(q2, sc2[p]));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void load_scales8(const float* __restrict__ p, uint64_t (&sc2)[4]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  sc2[0] = f32x2_pack(a.x, a.y); sc2[1] = f32x2_pack(a.z, a.w);
  sc2[2] = f32x2_pack(b.x, b.y); sc2[3] = f32x2_pack(b.z, b.w);
}

// EPI_W epilogue warps (4, or 8 = two per TMEM lane quarter, each taking half of the tile's
// columns). Eight measured slower for the fp32-accumulator products (block gradients, the CNP /
// dq blocks: 0.31 -> 0.33 ms and 83 -> 97 us), so every variant uses four.
template <bool B_I8, bool OUT_F32>
struct PairCfg {
  static constexpr int EPI_W = 4;                   // epilogue warps
  static constexpr int STAGES = B_I8 ? 4 : 6;
  static constexpr int RAW = B_I8 ? 8 : 0;          // int8 staging slots
  static constexpr int RAW_AHEAD = RAW > 2 ? RAW - 2 : 0;  // int8 tiles in flight ahead of A
  static constexpr int RAW_BYTES = 128 * BK;        // this CTA's 128 B rows (or columns) x 64
  static constexpr int THREADS = 64 + 32 * EPI_W + (B_I8 ? kPairConvThreads : 0);
  static constexpr size_t SMEM = (size_t)STAGES * (128 * BK * 2 * 2) + (size_t)RAW * RAW_BYTES +
                                 EPI_W * kEpiStageBytes + 1024 + 256;
};

template <bool A_MN, bool B_MN, bool OUT_F32, bool B_I8>
__global__ void __launch_bounds__((PairCfg<B_I8, OUT_F32>::THREADS), 1)
umma_gemm_pair_kernel(const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b,
                      const __grid_constant__ CUtensorMap tma_c,
                      const __grid_constant__ CUtensorMap tma_a2,
                      const __grid_constant__ CUtensorMap tma_b2,
                      const __grid_constant__ PairParams p) {
  using Cfg = PairCfg<B_I8, OUT_F32>;
  constexpr int EPI_W = Cfg::EPI_W;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int RAW = Cfg::RAW;
  constexpr int A_BYTES = 128 * BK * 2;  // this CTA's 128 rows of A, 16 KB
  constexpr int B_BYTES = 128 * BK * 2;  // this CTA's 128 rows (N) of B, 16 KB
  constexpr int ACC_COLS = 256;
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + STAGES * A_BYTES;
  uint8_t* sq = sb + STAGES * B_BYTES;     // int8 staging (B_I8)
  uint8_t* sepi = sq + RAW * Cfg::RAW_BYTES;   // EPI_W epilogue warps x 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sepi + EPI_W * kEpiStageBytes);
  uint64_t* full = bars;                   // used in the leader only
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;            // used in the leader only (2 * EPI_W arrivals)
  uint64_t* drain = tempty + 2;
  uint64_t* qfull = drain + 1;             // int8 staging slot loaded (local)
  uint64_t* qempty = qfull + RAW;          // int8 staging slot read by the converters (local)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qempty + RAW);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const Ctl ctl{abort_flag, p.err};
  const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // B_I8: the producer's arrive plus one per converter warp of a group, in both CTAs
      mbar_init(smem_u32(full + s), B_I8 ? 1 + 2 * kConvWarpsPerGroup : 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(tfull + a), 1);
      mbar_init(smem_u32(tempty + a), 2 * EPI_W);
    }
    mbar_init(smem_u32(drain), 1);
    for (int r = 0; r < RAW; ++r) {
      mbar_init(smem_u32(qfull + r), 1);
      mbar_init(smem_u32(qempty + r), kConvWarpsPerGroup);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_wait();      // operands and outputs may belong to the previous kernel of the stream
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      // int8 B: its own stream of staged tiles, RAW_AHEAD K blocks ahead of the A stream (one
      // split, so every tile of this cluster has the same nk K blocks)
      const int nk = (p.K + BK - 1) / BK;
      const int my_tiles =
          cluster_id < p.total_tiles ? (p.total_tiles - cluster_id + num_clusters - 1) / num_clusters
                                     : 0;
      const int total_it = B_I8 ? my_tiles * nk : 0;
      int rit = 0;
      // position of the int8 stream: K block rkb of the cluster's tile rtile, whose B coordinates
      // are decoded once per tile (this thread issues every load; it must stay cheap per block)
      int rtile = cluster_id, rkb = 0, rbn = 0, rbk = 0;
      auto raw_tile = [&]() {
        if (rtile < p.total_tiles) {
          const TileCoord tj = decode_pair_tile(p, rtile);
          rbn = tj.g * p.b_gn + tj.nb * 256 + (int)rank * 128;
          rbk = tj.g * p.b_gk;
        }
      };
      if constexpr (B_I8) raw_tile();
      constexpr int RAWD = RAW > 0 ? RAW : 1;   // (the bf16 instantiation never calls this)
      auto issue_raw = [&](int j) -> bool {
        const int r = j % RAWD;
        if (!wait_bounded(smem_u32(qempty + r), ((uint32_t)(j / RAWD) & 1u) ^ 1u, ctl,
                          kErrProducer, kWaitLimitNs, /*stop_on_abort=*/false))
          return false;
        const int kj = rkb * BK;
        const uint32_t qb = smem_u32(qfull + r);
        mbar_expect_tx(qb, Cfg::RAW_BYTES);
        if constexpr (B_MN) tma_load_2d(smem_u32(sq + r * Cfg::RAW_BYTES), &tma_b, qb, rbn, rbk + kj);
        else tma_load_2d(smem_u32(sq + r * Cfg::RAW_BYTES), &tma_b, qb, rbk + kj, rbn);
        if (++rkb == nk) {
          rkb = 0;
          rtile += num_clusters;
          raw_tile();
        }
        return true;
      };
      for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters) {
        const TileCoord tc = decode_pair_tile(p, tile);
        const int kb0 = tc.split * p.kblocks_per_split;
        const int kb1 = min(kb0 + p.kblocks_per_split, (p.K + BK - 1) / BK);
        // groups from g2 on come from the second operand pair, counted from its first group
        const bool second = tc.g >= p.g2;
        const CUtensorMap* map_a = second ? &tma_a2 : &tma_a;
        const CUtensorMap* map_b = second ? &tma_b2 : &tma_b;
        const int gl = second ? tc.g - p.g2 : tc.g;
        const int am = gl * p.a_gm + tc.mb * 256 + (int)rank * 128, ak = gl * p.a_gk;
        const int bn = gl * p.b_gn + tc.nb * 256 + (int)rank * 128, bk = gl * p.b_gk;
        if (second && p.deps) {
          // the first product's results for this group must be written before they are read;
          // then order this thread's asynchronous-proxy (TMA) reads after them
          if (!wait_count(p.deps + gl % p.dep_blocks, p.dep_target, ctl, kErrDependency,
                          kWaitLimitNs)) {
            ok = false;
            break;
          }
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if constexpr (B_I8) {
            while (ok && rit < total_it && rit <= it + Cfg::RAW_AHEAD) {
              ok = issue_raw(rit);
              if (ok) ++rit;
            }
            if (!ok) break;
          }
          // The two producers stop only when this wait runs out, not on the CTA's abort flag:
          // both are released by the same multicast commits, so both then have issued the
          // same loads, every one of which the leader armed and drains below. (Stopping on
          // the flag could leave the peer's last load unarmed and still in flight at exit.)
          if (!wait_bounded(smem_u32(empty + s), ph ^ 1u, ctl, kErrProducer, kWaitLimitNs,
                            /*stop_on_abort=*/false)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(smem_u32(full + s), 0);
          if (leader)
            mbar_expect_tx(smem_u32(full + s), B_I8 ? 2 * A_BYTES : 2 * (A_BYTES + B_BYTES));
          const KCoord kc = k_coord(p, kb);
          const int k = kc.k;
          if constexpr (A_MN) {
            tma_load_2d_pair(smem_u32(sa + s * A_BYTES), map_a, fb, am + kc.adx, ak + k + kc.ady);
            tma_load_2d_pair(smem_u32(sa + s * A_BYTES + 64 * BK * 2), map_a, fb,
                             am + 64 + kc.adx, ak + k + kc.ady);
          } else {
            tma_load_2d_pair(smem_u32(sa + s * A_BYTES), map_a, fb, ak + k + kc.adx, am + kc.ady);
          }
          if constexpr (B_I8) {
            // the int8 tile of this K block was issued by issue_raw
          } else if constexpr (B_MN) {
            tma_load_2d_pair(smem_u32(sb + s * B_BYTES), map_b, fb, bn + kc.bdx, bk + k + kc.bdy);
            tma_load_2d_pair(smem_u32(sb + s * B_BYTES + 64 * BK * 2), map_b, fb,
                             bn + 64 + kc.bdx, bk + k + kc.bdy);
          } else {
            tma_load_2d_pair(smem_u32(sb + s * B_BYTES), map_b, fb, bk + k + kc.bdx, bn + kc.bdy);
          }
        }
      }
      if (!ok) {
        // the leader's full barriers count both CTAs' A (and bf16 B) bytes: let them land
        if (leader)
          for (int j = max(0, it - STAGES); j < it; ++j)
            wait_bounded(smem_u32(full + j % STAGES), (uint32_t)(j / STAGES) & 1u, ctl, 0,
                         kDrainLimitNs);
        if constexpr (B_I8)
          for (int j = max(0, rit - RAW); j < rit; ++j)
            wait_bounded(smem_u32(qfull + j % RAW), (uint32_t)(j / RAW) & 1u, ctl, 0,
                         kDrainLimitNs);
      }
    }
    __syncwarp();  // reconverge before the block-wide barriers below
  } else if (warp == 1) {
    if (leader && lane == 0) {
      constexpr uint32_t idesc = instr_desc_pair<A_MN, B_MN>();
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters, ++tcount) {
        const TileCoord tc = decode_pair_tile(p, tile);
        const int kb0 = tc.split * p.kblocks_per_split;
        const int kb1 = min(kb0 + p.kblocks_per_split, (p.K + BK - 1) / BK);
        const int acc = tcount & 1;
        const uint32_t use = (uint32_t)(tcount >> 1);
        if (!wait_bounded(smem_u32(tempty + acc), (use & 1u) ^ 1u, ctl, kErrMma, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!wait_bounded<B_I8>(smem_u32(full + s), ph, ctl, kErrMma, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sa + s * A_BYTES), b0 = smem_u32(sb + s * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc(a0 + kk * 2048, 64 * BK * 2, 1024)
                                     : smem_desc(a0 + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc(b0 + kk * 2048, 64 * BK * 2, 1024)
                                     : smem_desc(b0 + kk * 32, 16, 1024);
            umma_bf16_pair(d, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair_both(smem_u32(empty + s));
        }
        if (!ok) break;
        umma_commit_pair_both(smem_u32(tfull + acc));
      }
      umma_commit_pair_both(smem_u32(drain));
      wait_bounded(smem_u32(drain), 0, ctl, ok ? kErrMma : 0, ok ? kWaitLimitNs : kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp < 2 + EPI_W) {
    // TMEM lanes 32 * (warp % 4) .. + 31; with eight warps, warps 6.. take the second half of
    // the columns
    const int quarter = warp & 3;
    constexpr int COLS = ACC_COLS / (EPI_W / 4);
    const int cbase = ((warp - 2) / 4) * COLS;
    const uint32_t leader_tempty0 = map_to_rank(smem_u32(tempty), 0);
    int tcount = 0, chunk = 0;
    for (int tile = cluster_id; tile < p.total_tiles; tile += num_clusters, ++tcount) {
      const TileCoord tc = decode_pair_tile(p, tile);
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      const int row0 = tc.mb * 256 + (int)rank * 128 + quarter * 32;
      const int nlive = max(0, min(32, p.M - row0));
      // a second product's tiles use epi2 and their group index within that product
      const bool second = tc.g >= p.g2;
      const Epi& ep = second ? p.epi2 : p.epi;
      const int ge = second ? tc.g - p.g2 : tc.g;
      const int gout = (second && p.c_rel2) ? tc.g - p.g2 : tc.g;
      const bool fused = OUT_F32 && ep.mode != kEpiStore;
      FusedQ q0;
      const int col0 = tc.nb * 256 + cbase;
      if (fused) fused_q_load(ep, fused_base(ep, ge, row0, col0, lane), 0, nlive, lane, q0);
      if (!wait_bounded(smem_u32(tfull + acc), use & 1u, ctl, kErrEpilogue, p.epi_wait_ns))
        break;
      tc_fence_after();
      const long long off0 = (long long)tc.split * p.c_split + (long long)gout * p.c_gs +
                             (long long)row0 * p.ldc + (long long)col0;
      const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                            (uint32_t)(acc * ACC_COLS + cbase);
      if (fused)
        epilogue_fused(trow, COLS, sepi + (warp - 2) * kEpiStageBytes, ep, ge, row0, col0,
                       nlive, lane, q0);
      else if constexpr (!OUT_F32)
        epilogue_tma_bf16(trow, COLS, sepi + (warp - 2) * kEpiStageBytes, &tma_c,
                          (int)(((long long)tc.g * p.c_gs) % p.ldc) + col0,
                          (int)(((long long)tc.g * p.c_gs) / p.ldc) + row0, lane, chunk);
      else
        epilogue_warp_rows<OUT_F32>(trow, COLS, sepi + (warp - 2) * kEpiStageBytes, p.C, off0,
                                    p.ldc, nlive, lane);
      if constexpr (OUT_F32) {
        if (p.deps && !second) {
          // publish this warp's part of a first-product tile: its stores (plain stores of the
          // fused or fp32 epilogue) become visible at GPU scope before the count moves
          __threadfence();
          __syncwarp();
          if (lane == 0) red_release_gpu_add(p.deps + tc.g, 1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(leader_tempty0 + (uint32_t)(acc * 8));
    }
    if constexpr (!OUT_F32) {
      if (lane == 0) bulk_wait_all();   // every store written before the CTA leaves
      __syncwarp();
    }
  } else if constexpr (B_I8) {
    // ------------------------------------------------------------ int8 -> bf16 converters
    // kConvGroups groups of two warps take the K blocks in turn (block it goes to group
    // it % kConvGroups), so that many blocks are converted at a time; the staging ring holds
    // RAW blocks ahead. Thread gt of a group owns one 8-element unit column of the staged tile
    // and 16 of its 64 (B_MN) or 128 (K-major) lines: 8-byte conflict-free reads, 16-byte
    // swizzled conflict-free writes.
    static_assert(kConvWarpsPerGroup == 2, "a group's 64 threads own the tile's unit columns");
    const int cw = warp - (2 + EPI_W);
    const int grp = cw / kConvWarpsPerGroup;
    const int gt = (cw % kConvWarpsPerGroup) * 32 + lane;   // 0..63
    const uint32_t leader_full0 = map_to_rank(smem_u32(full), 0);
    int it = 0;
    bool ok = true;
    for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters) {
      const TileCoord tc = decode_pair_tile(p, tile);
      const int kb0 = tc.split * p.kblocks_per_split;
      const int kb1 = min(kb0 + p.kblocks_per_split, (p.K + BK - 1) / BK);
      const int bn = tc.g * p.b_gn + tc.nb * 256 + (int)rank * 128;
      uint64_t sc[4];
      if constexpr (B_MN) load_scales8(p.b_scale + bn + 8 * (gt & 15), sc);   // per N column
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        if (it % kConvGroups != grp) continue;
        const int s = it % STAGES, r = it % RAW;
        if constexpr (!B_MN) {
          // scales along K for this block, requested before the waits so that their latency
          // overlaps them (K is a multiple of 8: a unit of 8 is all inside or all outside)
          const int kq = kb * BK + 8 * (gt & 7);
          if (kq < p.K) {
            load_scales8(p.b_scale + tc.g * p.b_gk + kq, sc);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[e] = 0ull;   // +0.0f pairs
          }
        }
        // like the producer, the converters stop only when a wait runs out (see there)
        bool got = wait_bounded(smem_u32(qfull + r), (uint32_t)(it / RAW) & 1u, ctl, kErrConvert,
                                kWaitLimitNs, /*stop_on_abort=*/false);
        got = got && wait_bounded(smem_u32(empty + s), ((uint32_t)(it / STAGES) & 1u) ^ 1u, ctl,
                                  kErrConvert, kWaitLimitNs, /*stop_on_abort=*/false);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint8_t* q = sq + r * Cfg::RAW_BYTES;
        uint8_t* dst = sb + s * B_BYTES;
        if constexpr (B_MN) {
          // staged int8 tile: 64 K lines of 128 N bytes; bf16 stage: two 64-column chunks of
          // 64 K lines x 128 B, 16-byte unit u of line k at (u ^ (k & 7))
          const int nu = gt & 15, k0 = gt >> 4;   // lines k0 + 4 j, j = 0..15
          uint8_t* d0 = dst + (nu >> 3) * (64 * BK * 2);
          // every staged read before any operand write (the compiler cannot tell the two
          // shared-memory ranges apart, so interleaving them would serialise each unit)
          uint2 w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[j] = *reinterpret_cast<const uint2*>(q + (k0 + 4 * j) * 128 + nu * 8);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int k = k0 + 4 * j;
            *reinterpret_cast<uint4*>(d0 + k * 128 + (((nu & 7) ^ (k & 7)) << 4)) =
                dequant8(w[j], sc);
          }
        } else {
          // staged int8 tile: 128 N lines of 64 K bytes; bf16 stage: 128 lines x 128 B,
          // 16-byte unit u of line j at (u ^ (j & 7)); the scale runs along K
          const int u = gt & 7, j0 = gt >> 3;     // lines j0 + 8 i, i = 0..15
          uint8_t* d0 = dst + ((u ^ (j0 & 7)) << 4);   // j & 7 == j0 & 7 for every i
          uint2 w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = *reinterpret_cast<const uint2*>(q + (j0 + 8 * i) * 64 + u * 8);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            *reinterpret_cast<uint4*>(d0 + (j0 + 8 * i) * 128) = dequant8(w[i], sc);
        }
        // make the generic-proxy stores visible to the tensor core's reads, then publish
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(qempty + r));
          // the leader's own converters order their writes at CTA scope, the peer's at cluster
          if (leader) mbar_arrive(smem_u32(full + s));
          else mbar_arrive_remote(leader_full0 + (uint32_t)(s * 8));
        }
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();   // no remote arrive or copy may target a CTA that has left
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ wide CTA-pair kernel
// The dense W0' products (B = A' W0', dA' = dB W0'^T) on 256 x 512 pair tiles: per 64-deep K
// block each CTA loads 128 rows of A and 2 x 128 rows (N) of B, and the leader issues, for each
// 16-deep K step, two 256 x 256 x 16 pair MMAs that share the A operand (the first may keep A in
// the tensor core's collector buffer for the second). Per CTA and K block that is 48 KB of
// operands for 128 x 512 outputs, against 32 KB for 128 x 256 on the 256 x 256 tiles: a quarter
// less shared-memory traffic (TMA writes plus MMA operand reads) per MMA cycle, which is what
// those tiles spend a fifth of their cycles waiting on.
//   The accumulator is all 512 TMEM columns, as two 256-column halves with their own
// "drained" barriers: the epilogue hands half 0 back first, and the MMA issuer starts the next
// tile on half 0 alone, holding each stage until half 1 is back, then issues the held half-1
// MMAs in K order and releases those stages. So the epilogue still overlaps the next main loop.
//   Everything else (TMA on both CTAs completing the leader's full barrier, commits multicast to
// both CTAs, bounded waits, bf16 epilogue through TMA stores, programmatic launch) is as in the
// 256 x 256 kernel. Operand layouts, groups (per-group coordinate offsets, a second operand
// pair), split K and fp32 outputs are those of the 256 x 256 kernel: the b = 512 blocks take one
// 512-wide tile per block and row tile, the per-block gradients one per block and M half.
struct WideCfg {
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = 128 * BK * 2;   // 16 KB
  static constexpr int B_BYTES = 256 * BK * 2;   // 32 KB: N half 0 rows, then N half 1 rows
  static constexpr int EPI_W = 4;
  static constexpr int THREADS = 64 + 32 * EPI_W;
  static constexpr size_t SMEM =
      (size_t)STAGES * (A_BYTES + B_BYTES) + EPI_W * kEpiStageBytes + 1024 + 256;
};

// collector usage of the A operand: 0 = none, 1 = fill (keep A for the next MMA), 2 = last use
template <int COLL>
__device__ __forceinline__ void umma_bf16_pair_coll(uint32_t d_tmem, uint64_t a_desc,
                                                    uint64_t b_desc, uint32_t idesc,
                                                    uint32_t accumulate) {
  if constexpr (COLL == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16.collector::a::fill [%0], %1, %2, %3, p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else if constexpr (COLL == 2) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    umma_bf16_pair(d_tmem, a_desc, b_desc, idesc, accumulate);
  }
}

template <bool B_MN>
__device__ __forceinline__ uint64_t wide_b_desc(uint32_t b0, int half, int kk) {
  const uint32_t base = b0 + (uint32_t)half * (128 * BK * 2);
  return B_MN ? smem_desc(base + kk * 2048, 64 * BK * 2, 1024) : smem_desc(base + kk * 32, 16, 1024);
}

// Tile `tile` of the 256 x 512 kernel: a full-width tile (half = -1), or half `half` (0 / 1,
// the 256-column halves) of full-width tile narrow_from + (tile - narrow_from) / 2.
__device__ __forceinline__ TileCoord decode_wide_tile(const PairParams& p, int tile, int& half) {
  if (tile < p.narrow_from) {
    half = -1;
    return decode_pair_tile(p, tile);
  }
  const int j = tile - p.narrow_from;
  half = j & 1;
  return decode_pair_tile(p, p.narrow_from + (j >> 1));
}

template <bool A_MN>
__device__ __forceinline__ uint64_t wide_a_desc(uint32_t a0, int kk) {
  return A_MN ? smem_desc(a0 + kk * 2048, 64 * BK * 2, 1024) : smem_desc(a0 + kk * 32, 16, 1024);
}

template <bool A_MN, bool B_MN, bool OUT_F32, bool COLLECT>
__global__ void __launch_bounds__(WideCfg::THREADS, 1)
umma_gemm_wide_kernel(const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b,
                      const __grid_constant__ CUtensorMap tma_c,
                      const __grid_constant__ CUtensorMap tma_a2,
                      const __grid_constant__ CUtensorMap tma_b2,
                      const __grid_constant__ PairParams p) {
  constexpr int STAGES = WideCfg::STAGES;
  constexpr int A_BYTES = WideCfg::A_BYTES;
  constexpr int B_BYTES = WideCfg::B_BYTES;
  constexpr int EPI_W = WideCfg::EPI_W;
  constexpr uint32_t TMEM_COLS = 512;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + STAGES * A_BYTES;
  uint8_t* sepi = sb + STAGES * B_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sepi + EPI_W * kEpiStageBytes);
  uint64_t* full = bars;                   // leader only
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;     // one accumulator
  uint64_t* tempty = tfull + 1;            // [2]: half 0, half 1 drained (leader only)
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const Ctl ctl{abort_flag, p.err};
  const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
  const int nk_all = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    mbar_init(smem_u32(tfull), 1);
    for (int h = 0; h < 2; ++h) mbar_init(smem_u32(tempty + h), 2 * EPI_W);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters) {
        int half;
        const TileCoord tc = decode_wide_tile(p, tile, half);
        const int kb0 = tc.split * p.kblocks_per_split;
        const int kb1 = min(kb0 + p.kblocks_per_split, nk_all);
        // a half-width tile loads only its N half, into the stage's first B slot
        const int h_lo = half < 0 ? 0 : half, h_n = half < 0 ? 2 : 1;
        // groups from g2 on come from the second operand pair, counted from its first group
        const bool second = tc.g >= p.g2;
        const CUtensorMap* map_a = second ? &tma_a2 : &tma_a;
        const CUtensorMap* map_b = second ? &tma_b2 : &tma_b;
        const int gl = second ? tc.g - p.g2 : tc.g;
        const int am = gl * p.a_gm + tc.mb * 256 + (int)rank * 128, ak = gl * p.a_gk;
        // N half h: rows (K-major B) or columns (N-major B) bn + 256 h
        const int bn = gl * p.b_gn + tc.nb * 512 + (int)rank * 128, bk = gl * p.b_gk;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          // stops only when the wait runs out (see the 256 x 256 kernel's producer)
          if (!wait_bounded(smem_u32(empty + s), ph ^ 1u, ctl, kErrProducer, kWaitLimitNs,
                            /*stop_on_abort=*/false)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(smem_u32(full + s), 0);
          if (leader)
            mbar_expect_tx(smem_u32(full + s), 2 * (A_BYTES + (B_BYTES / 2) * h_n));
          const int k = kb * BK;
          const uint32_t da = smem_u32(sa + s * A_BYTES);
          if constexpr (A_MN) {
            tma_load_2d_pair(da, map_a, fb, am, ak + k);
            tma_load_2d_pair(da + 64 * BK * 2, map_a, fb, am + 64, ak + k);
          } else {
            tma_load_2d_pair(da, map_a, fb, ak + k, am);
          }
          for (int i = 0; i < h_n; ++i) {
            const int h = h_lo + i;   // N half of the tile, loaded into slot i
            const uint32_t dst = smem_u32(sb + s * B_BYTES + i * (128 * BK * 2));
            if constexpr (B_MN) {
              tma_load_2d_pair(dst, map_b, fb, bn + 256 * h, bk + k);
              tma_load_2d_pair(dst + 64 * BK * 2, map_b, fb, bn + 256 * h + 64, bk + k);
            } else {
              tma_load_2d_pair(dst, map_b, fb, bk + k, bn + 256 * h);
            }
          }
        }
      }
      if (!ok && leader)
        for (int j = max(0, it - STAGES); j < it; ++j)
          wait_bounded(smem_u32(full + j % STAGES), (uint32_t)(j / STAGES) & 1u, ctl, 0,
                       kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = instr_desc_pair<A_MN, B_MN>();
      int it = 0, tcount = 0;
      bool ok = true;
      // MMAs of one stage (iteration j, i-th K block of the tile): halves h0..h1-1
      auto issue = [&](int j, int i, int h0, int h1) {
        const int s = j % STAGES;
        const uint32_t a0 = smem_u32(sa + s * A_BYTES), b0 = smem_u32(sb + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = wide_a_desc<A_MN>(a0, kk);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          if (h0 == 0 && h1 == 2 && COLLECT) {
            umma_bf16_pair_coll<1>(tmem_base, ad, wide_b_desc<B_MN>(b0, 0, kk), idesc, acc);
            umma_bf16_pair_coll<2>(tmem_base + 256, ad, wide_b_desc<B_MN>(b0, 1, kk), idesc, acc);
          } else {
            for (int h = h0; h < h1; ++h)
              umma_bf16_pair(tmem_base + 256 * h, ad, wide_b_desc<B_MN>(b0, h, kk), idesc, acc);
          }
        }
      };
      for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters, ++tcount) {
        int half;
        const TileCoord tc = decode_wide_tile(p, tile, half);
        const int kb0 = tc.split * p.kblocks_per_split;
        const int nk = min(kb0 + p.kblocks_per_split, nk_all) - kb0;
        const uint32_t par = ((uint32_t)tcount & 1u) ^ 1u;   // previous tile's drain
        if (!wait_bounded(smem_u32(tempty), par, ctl, kErrMma, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (half >= 0) {
          // half-width tile: accumulator half 0 only, from the stage's first B slot
          for (int i = 0; i < nk; ++i, ++it) {
            const int s = it % STAGES;
            if (!wait_bounded<false>(smem_u32(full + s), (uint32_t)(it / STAGES) & 1u, ctl,
                                     kErrMma, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue(it, i, 0, 1);
            umma_commit_pair_both(smem_u32(empty + s));
          }
          if (!ok) break;
          umma_commit_pair_both(smem_u32(tfull));
          continue;
        }
        bool h1_free = false;
        const int first = it;   // iteration of this tile's first K block
        int held = 0;           // the tile's K blocks 0..held-1 have their half-0 MMAs only
        auto release_held = [&]() {
          for (int i = 0; i < held; ++i) {
            issue(first + i, i, 1, 2);
            umma_commit_pair_both(smem_u32(empty + (first + i) % STAGES));
          }
          held = 0;
        };
        for (int i = 0; i < nk; ++i, ++it) {
          const int s = it % STAGES;
          if (!wait_bounded<false>(smem_u32(full + s), (uint32_t)(it / STAGES) & 1u, ctl, kErrMma,
                                   kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (!h1_free && mbar_test_wait(smem_u32(tempty + 1), par)) {
            h1_free = true;
            tc_fence_after();
            release_held();
          }
          if (h1_free) {
            issue(it, i, 0, 2);
            umma_commit_pair_both(smem_u32(empty + s));
          } else {
            issue(it, i, 0, 1);
            if (++held == STAGES) {
              // every stage is held: wait for half 1 of the previous tile
              if (!wait_bounded(smem_u32(tempty + 1), par, ctl, kErrMma, kWaitLimitNs)) {
                ok = false;
                break;
              }
              h1_free = true;
              tc_fence_after();
              release_held();
            }
          }
        }
        if (!ok) break;
        if (!h1_free) {   // K shorter than the ring
          if (!wait_bounded(smem_u32(tempty + 1), par, ctl, kErrMma, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          release_held();
        }
        umma_commit_pair_both(smem_u32(tfull));
      }
      umma_commit_pair_both(smem_u32(drain));
      wait_bounded(smem_u32(drain), 0, ctl, ok ? kErrMma : 0, ok ? kWaitLimitNs : kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const uint32_t leader_tempty0 = map_to_rank(smem_u32(tempty), 0);
    int tcount = 0, chunk = 0;
    for (int tile = cluster_id; tile < p.total_tiles; tile += num_clusters, ++tcount) {
      int half;
      const TileCoord tc = decode_wide_tile(p, tile, half);
      const int row0 = tc.mb * 256 + (int)rank * 128 + quarter * 32;
      if (!wait_bounded(smem_u32(tfull), (uint32_t)tcount & 1u, ctl, kErrEpilogue, p.epi_wait_ns))
        break;
      tc_fence_after();
      const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16);
      // a group's output starts c_gs elements on: a column offset, or whole rows
      const long long goff = (long long)tc.g * p.c_gs;
      const int gx = (int)(goff % p.ldc), gy = (int)(goff / p.ldc);
      const long long off0 = (long long)tc.split * p.c_split + goff + (long long)row0 * p.ldc +
                             (long long)tc.nb * 512;
      const int nlive = max(0, min(32, p.M - row0));
      // a half-width tile's result is in accumulator half 0; its columns start at 256 * half
      const int nh = half < 0 ? 2 : 1, c0 = half < 0 ? 0 : 256 * half;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        if (h < nh) {
          if constexpr (OUT_F32)
            epilogue_warp_rows<true>(trow + (uint32_t)(256 * h), 256,
                                     sepi + (warp - 2) * kEpiStageBytes, p.C,
                                     off0 + c0 + 256 * h, p.ldc, nlive, lane);
          else
            epilogue_tma_bf16(trow + (uint32_t)(256 * h), 256, sepi + (warp - 2) * kEpiStageBytes,
                              &tma_c, gx + tc.nb * 512 + c0 + 256 * h, gy + row0, lane, chunk);
          tc_fence_before();
        }
        __syncwarp();
        // both halves are handed back for every tile (phase accounting of the MMA's waits)
        if (lane == 0) mbar_arrive_remote_relaxed(leader_tempty0 + (uint32_t)(h * 8));
      }
    }
    if constexpr (!OUT_F32) {
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ W0' -> P-block fused kernel
// The forward's W0' product and P-block product in one launch, for b = 512 (back-to-back fusion
// of "POET-X" blog §第四斧 / §第五斧's forward chain): the 256 x 512 pair tile of B = A' W0'
// whose 512 columns are exactly P block j is finished in TMEM, written once as bf16 into shared
// memory in the MMA operand layout (and, when the caller keeps B for the backward, to global
// memory from there), and multiplied by G_P^j right away: C tile = B tile x G_P^j, into the same
// TMEM columns, then stored. B never makes the HBM round trip between the two products.
//   Per tile (mb, j) of a CTA pair:
//     phase 1  B_acc = A'[256 rows] W0'[:, 512 j ..]: the 256 x 512 main loop (4-stage ring)
//     phase 2  epilogue: B_acc -> bf16 B tile, 8 K-slots of 128 rows x 64 in each CTA's shared
//              memory (the ring's first 128 KB, idle now), optionally stored to global B;
//              columns 0-255 (slots 0-3) first, then 256-511
//     phase 3  C_acc = B tile x G_P^j through four 16 KB G slots (the ring's last 64 KB), one
//              256-column half of C after the other: C half 0 starts on B slots 0-3 as soon
//              as B columns 0-255 are out of TMEM (while 256-511 drain), C half 1 writes the
//              TMEM columns of B half 1; the tensor core reads the B tile of both CTAs
//     phase 4  epilogue: C_acc -> bf16 C, half 0 while the MMAs of C half 1 run, half 1 while
//              the next tile's main loop runs on accumulator half 0 (its stages held for half
//              1 until that half is drained, as in the 256 x 512 kernel)
//   The ring is busy with the B tile and the G slots from the end of phase 1 to the end of
//   phase 3: the producer loads G after the main loop's last MMA and the next tile's stages
//   after phase 3. What stays serial per tile is the drain of B half 0 and the refill of the
//   ring's first stages.
struct FusedCfg {
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = 128 * BK * 2;   // 16 KB
  static constexpr int B_BYTES = 256 * BK * 2;   // 32 KB (N half 0 rows, then N half 1 rows)
  static constexpr int RING = STAGES * (A_BYTES + B_BYTES);   // 192 KB
  static constexpr int SLOTS = 8;                              // K slots of the B tile (b = 512)
  static constexpr int SLOT_BYTES = 128 * BK * 2;              // 16 KB
  static constexpr int GSLOTS = 4;                             // G slots of one C half's rows
  static constexpr int G_BYTES = 128 * BK * 2;                 // 16 KB
  static constexpr int G_OFF = SLOTS * SLOT_BYTES;             // 128 KB
  static constexpr int EPI_W = 4;
  static constexpr int THREADS = 64 + 32 * EPI_W;
  static constexpr size_t SMEM = (size_t)RING + EPI_W * kEpiStageBytes + 1024 + 256;
};
static_assert(FusedCfg::G_OFF + FusedCfg::GSLOTS * FusedCfg::G_BYTES <= FusedCfg::RING,
              "the B tile and the G slots overlay the ring");

// A' [T][m] K-major, W0' [m][n] and the stacked G_P blocks [n][512] N-major; B and C [T][n] bf16.
__global__ void __launch_bounds__(FusedCfg::THREADS, 1)
umma_w0p_fused_kernel(const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_w,
                      const __grid_constant__ CUtensorMap tma_g,
                      const __grid_constant__ CUtensorMap tma_bo,
                      const __grid_constant__ CUtensorMap tma_co,
                      const __grid_constant__ PairParams p, int save_b) {
  constexpr int STAGES = FusedCfg::STAGES;
  constexpr int A_BYTES = FusedCfg::A_BYTES;
  constexpr int B_BYTES = FusedCfg::B_BYTES;
  constexpr int SLOTS = FusedCfg::SLOTS;
  constexpr int SLOT_BYTES = FusedCfg::SLOT_BYTES;
  constexpr int GSLOTS = FusedCfg::GSLOTS;
  constexpr int G_BYTES = FusedCfg::G_BYTES;
  constexpr int EPI_W = FusedCfg::EPI_W;
  constexpr uint32_t TMEM_COLS = 512;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sa = smem;                                 // ring: A stages
  uint8_t* sb = smem + STAGES * A_BYTES;              //       B stages
  uint8_t* btile = smem;                              // phases 2-3: B tile, SLOTS K slots
  uint8_t* sg = smem + FusedCfg::G_OFF;               // phase 3: G slots
  uint8_t* sepi = smem + FusedCfg::RING;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sepi + EPI_W * kEpiStageBytes);
  uint64_t* full = bars;                       // [STAGES] leader
  uint64_t* empty = full + STAGES;             // [STAGES] both (multicast commits)
  uint64_t* gfull = empty + STAGES;            // [GSLOTS] leader
  uint64_t* gempty = gfull + GSLOTS;           // [GSLOTS] both
  uint64_t* tfull_b = gempty + GSLOTS;         // B_acc complete, both
  uint64_t* btile_full = tfull_b + 1;          // [2] B half h out of TMEM and in the B tile,
                                               //     leader (2 * EPI_W arrivals)
  uint64_t* tfull_c = btile_full + 2;          // [2] C half h complete, both
  uint64_t* tempty = tfull_c + 2;              // [2] C half h drained, leader (2 * EPI_W)
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const Ctl ctl{abort_flag, p.err};
  const int cluster_id = blockIdx.x >> 1, num_clusters = gridDim.x >> 1;
  const int nk = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int s = 0; s < GSLOTS; ++s) {
      mbar_init(smem_u32(gfull + s), 1);
      mbar_init(smem_u32(gempty + s), 1);
    }
    mbar_init(smem_u32(tfull_b), 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(smem_u32(btile_full + h), 2 * EPI_W);
      mbar_init(smem_u32(tfull_c + h), 1);
      mbar_init(smem_u32(tempty + h), 2 * EPI_W);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0, git = 0, tcount = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters, ++tcount) {
        const TileCoord tc = decode_pair_tile(p, tile);
        const uint32_t tpar = (uint32_t)tcount & 1u;
        const int am = tc.mb * 256 + (int)rank * 128;
        // N half h of P block j: columns 512 j + 256 h + 128 rank .. + 127 of W0', and the same
        // columns (within the block) of G_P^j, whose K rows start at 512 j
        const int wn = tc.nb * 512 + (int)rank * 128, gk = tc.nb * 512;
        // phase 1 (the previous tile's phase 3 has finished with the ring: the wait at the end
        // of the loop body)
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          // the producers stop only when a wait runs out, never on the abort flag, so that
          // both CTAs have issued the same loads (see the 256 x 256 pair kernel)
          if (!wait_bounded(smem_u32(empty + s), ((uint32_t)(it / STAGES) & 1u) ^ 1u, ctl,
                            kErrProducer, kWaitLimitNs, /*stop_on_abort=*/false)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(smem_u32(full + s), 0);
          if (leader) mbar_expect_tx(smem_u32(full + s), 2 * (A_BYTES + B_BYTES));
          const int k = kb * BK;
          tma_load_2d_pair(smem_u32(sa + s * A_BYTES), &tma_a, fb, k, am);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t dst = smem_u32(sb + s * B_BYTES + h * (128 * BK * 2));
            tma_load_2d_pair(dst, &tma_w, fb, wn + 256 * h, k);
            tma_load_2d_pair(dst + 64 * BK * 2, &tma_w, fb, wn + 256 * h + 64, k);
          }
        }
        if (!ok) break;
        // phase 3's G, C half 0's 256 columns then half 1's, K blocks in order: after the main
        // loop's last MMA (the ring's last 64 KB is free then)
        if (!wait_bounded(smem_u32(tfull_b), tpar, ctl, kErrProducer, kWaitLimitNs,
                          /*stop_on_abort=*/false)) {
          ok = false;
          break;
        }
        for (int i = 0; i < 2 * SLOTS; ++i, ++git) {
          const int h = i / SLOTS, kb = i % SLOTS, gs = git % GSLOTS;
          if (!wait_bounded(smem_u32(gempty + gs), ((uint32_t)(git / GSLOTS) & 1u) ^ 1u, ctl,
                            kErrProducer, kWaitLimitNs, /*stop_on_abort=*/false)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(smem_u32(gfull + gs), 0);
          if (leader) mbar_expect_tx(smem_u32(gfull + gs), 2 * G_BYTES);
          const uint32_t dst = smem_u32(sg + gs * G_BYTES);
          const int gx = 256 * h + 128 * (int)rank;
          tma_load_2d_pair(dst, &tma_g, fb, gx, gk + kb * BK);
          tma_load_2d_pair(dst + 64 * BK * 2, &tma_g, fb, gx + 64, gk + kb * BK);
        }
        if (!ok) break;
        // the next tile's stages once phase 3's MMAs are done with the B tile and the G slots
        if (!wait_bounded(smem_u32(tfull_c + 1), tpar, ctl, kErrProducer, kWaitLimitNs,
                          /*stop_on_abort=*/false)) {
          ok = false;
          break;
        }
      }
      if (!ok && leader) {
        // the leader's full barriers count both CTAs' bytes: let the armed loads land
        for (int j = max(0, it - STAGES); j < it; ++j)
          wait_bounded(smem_u32(full + j % STAGES), (uint32_t)(j / STAGES) & 1u, ctl, 0,
                       kDrainLimitNs);
        for (int j = max(0, git - GSLOTS); j < git; ++j)
          wait_bounded(smem_u32(gfull + j % GSLOTS), (uint32_t)(j / GSLOTS) & 1u, ctl, 0,
                       kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = instr_desc_pair<false, true>();
      int it = 0, git = 0, tcount = 0;
      bool ok = true;
      // the phase-1 MMAs of ring iteration j (K block i of the tile) for accumulator halves
      // h0 .. h1 - 1
      auto issue = [&](int j, int i, int h0, int h1) {
        const int s = j % STAGES;
        const uint32_t a0 = smem_u32(sa + s * A_BYTES), b0 = smem_u32(sb + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = smem_desc(a0 + kk * 32, 16, 1024);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          if (h0 == 0 && h1 == 2) {
            umma_bf16_pair_coll<1>(tmem_base, ad, wide_b_desc<true>(b0, 0, kk), idesc, acc);
            umma_bf16_pair_coll<2>(tmem_base + 256, ad, wide_b_desc<true>(b0, 1, kk), idesc, acc);
          } else {
            for (int h = h0; h < h1; ++h)
              umma_bf16_pair(tmem_base + 256 * h, ad, wide_b_desc<true>(b0, h, kk), idesc, acc);
          }
        }
      };
      for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters, ++tcount) {
        const uint32_t tpar = (uint32_t)tcount & 1u;
        // phase 1 on accumulator half 0 once the previous tile's C half 0 is drained; each
        // stage held (its half-1 MMAs not issued) until C half 1 is drained too
        if (!wait_bounded(smem_u32(tempty), tpar ^ 1u, ctl, kErrMma, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool h1_free = false;
        const int first = it;
        int held = 0;
        auto release_held = [&]() {
          for (int i = 0; i < held; ++i) {
            issue(first + i, i, 1, 2);
            umma_commit_pair_both(smem_u32(empty + (first + i) % STAGES));
          }
          held = 0;
        };
        for (int i = 0; i < nk; ++i, ++it) {
          const int s = it % STAGES;
          if (!wait_bounded<false>(smem_u32(full + s), (uint32_t)(it / STAGES) & 1u, ctl, kErrMma,
                                   kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (!h1_free && mbar_test_wait(smem_u32(tempty + 1), tpar ^ 1u)) {
            h1_free = true;
            tc_fence_after();
            release_held();
          }
          if (h1_free) {
            issue(it, i, 0, 2);
            umma_commit_pair_both(smem_u32(empty + s));
          } else {
            issue(it, i, 0, 1);
            if (++held == STAGES) {
              if (!wait_bounded(smem_u32(tempty + 1), tpar ^ 1u, ctl, kErrMma, kWaitLimitNs)) {
                ok = false;
                break;
              }
              h1_free = true;
              tc_fence_after();
              release_held();
            }
          }
        }
        if (!ok) break;
        if (!h1_free) {   // K shorter than the ring
          if (!wait_bounded(smem_u32(tempty + 1), tpar ^ 1u, ctl, kErrMma, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          release_held();
        }
        umma_commit_pair_both(smem_u32(tfull_b));
        // phase 3: C half h = B tile x G_P^j[:, 256 h ..], 16 G slots in order; C half 0
        // needs B half 0 out of TMEM (its columns) and B slots 0-3, then slots 4-7 (B half 1
        // written), which C half 1's columns need too. Acquire at cluster scope: the peer's
        // epilogue wrote its half of the operand.
        for (int i = 0; i < 2 * SLOTS; ++i, ++git) {
          const int h = i / SLOTS, kb = i % SLOTS, gs = git % GSLOTS;
          if (i == 0 || i == SLOTS / 2) {
            if (!wait_bounded<true>(smem_u32(btile_full + (i ? 1 : 0)), tpar, ctl, kErrMma,
                                    kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!wait_bounded<false>(smem_u32(gfull + gs), (uint32_t)(git / GSLOTS) & 1u, ctl,
                                   kErrMma, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(btile + kb * SLOT_BYTES), b0 = smem_u32(sg + gs * G_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(tmem_base + 256 * h, smem_desc(a0 + kk * 32, 16, 1024),
                           wide_b_desc<true>(b0, 0, kk), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair_both(smem_u32(gempty + gs));
          if (kb == SLOTS - 1) umma_commit_pair_both(smem_u32(tfull_c + h));
        }
      }
      umma_commit_pair_both(smem_u32(drain));
      wait_bounded(smem_u32(drain), 0, ctl, ok ? kErrMma : 0, ok ? kWaitLimitNs : kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    // TMEM lanes 32 * (warp % 4) .. + 31: rows quarter * 32 + lane of this CTA's 128
    const int quarter = warp & 3;
    const uint32_t leader_btile = map_to_rank(smem_u32(btile_full), 0);
    const uint32_t leader_tempty = map_to_rank(smem_u32(tempty), 0);
    int tcount = 0, chunk = 0;
    bool ok = true;
    for (int tile = cluster_id; ok && tile < p.total_tiles; tile += num_clusters, ++tcount) {
      const TileCoord tc = decode_pair_tile(p, tile);
      const uint32_t tpar = (uint32_t)tcount & 1u;
      const int row0 = tc.mb * 256 + (int)rank * 128 + quarter * 32;
      const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16);
      // phase 2: B_acc -> the B tile (slot c holds columns 64 c .. 64 c + 63, K-major, 128-byte
      // rows with 16-byte unit v of row r at v ^ (r & 7)), and to global B when it is kept
      if (!wait_bounded(smem_u32(tfull_b), tpar, ctl, kErrEpilogue, p.epi_wait_ns)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < SLOTS; ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld32(trow + (uint32_t)(64 * c), r0);
        tmem_ld32(trow + (uint32_t)(64 * c + 32), r1);
        uint8_t* part = btile + c * SLOT_BYTES + quarter * 32 * 128;   // this warp's 32 rows
        uint8_t* myrow = part + lane * 128;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint32_t* src = v < 4 ? &r0[8 * v] : &r1[8 * (v - 4)];
          *reinterpret_cast<uint4*>(myrow + ((v ^ (lane & 7)) * 16)) = make_uint4(
              pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
              pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
              pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
              pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
        }
        // visible to the tensor core's reads and to the copy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (save_b && lane == 0) {
          tma_store_2d(&tma_bo, smem_u32(part), tc.nb * 512 + 64 * c, row0);
          bulk_commit();
        }
        if (c == SLOTS / 2 - 1 || c == SLOTS - 1) {
          // B half (c == 3 ? 0 : 1) read out of TMEM and in the B tile; before the second
          // arrive the B stores have finished reading the tile (the ring is refilled only
          // after phase 3, which waits for that arrive)
          tc_fence_before();
          if (lane == 0) {
            if (c == SLOTS - 1) bulk_wait_read<0>();
            mbar_arrive_remote(leader_btile + (uint32_t)(c == SLOTS - 1 ? 8 : 0));
          }
          __syncwarp();
        }
      }
      // phase 4: C half h -> C, each half handed back as soon as it is out of TMEM
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        if (!wait_bounded(smem_u32(tfull_c + h), tpar, ctl, kErrEpilogue, p.epi_wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        epilogue_tma_bf16(trow + (uint32_t)(256 * h), 256, sepi + (warp - 2) * kEpiStageBytes,
                          &tma_co, tc.nb * 512 + 256 * h, row0, lane, chunk);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_relaxed(leader_tempty + (uint32_t)(h * 8));
      }
    }
    if (lane == 0) bulk_wait_all();   // every store written before the CTA leaves
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();   // no remote arrive or copy may target a CTA that has left
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous, row stride ld elements), box {64, box_rows}.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
              int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D int8 tensor [rows][cols] (row stride ld bytes), box {box_x, box_y}, no swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                 int box_x, int box_y) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_y};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


template <typename P>
void fill_segments(const Gemm& g, P& p) {
  p.nseg = g.nseg > 1 ? g.nseg : 1;
  p.kb_per_seg = (int)((g.K / p.nseg + BK - 1) / BK);
  for (int s = 0; s < 3; ++s) {
    const bool on = s < p.nseg && p.nseg > 1;
    p.a_dx[s] = on ? (int)g.a_dx[s] : 0; p.a_dy[s] = on ? (int)g.a_dy[s] : 0;
    p.b_dx[s] = on ? (int)g.b_dx[s] : 0; p.b_dy[s] = on ? (int)g.b_dy[s] : 0;
  }
}

template <int BN>
constexpr int stages_for() {
  return BN == 256 ? 4 : (BN == 128 ? 6 : 8);
}

template <int BN, bool A_MN, bool B_MN, bool OUT_F32>
cudaError_t launch_t(const Gemm& g, cudaStream_t s, const char* name) {
  constexpr int STAGES = stages_for<BN>();
  constexpr size_t smem =
      (size_t)STAGES * (BM * BK * 2 + BN * BK * 2) + 4 * kEpiStageBytes + 1024 + 256;
  CUtensorMap ta, tb;
  if (!make_map(&ta, g.A, g.a_rows, g.a_cols, g.a_ld, A_MN ? BK : BM)) return cudaErrorInvalidValue;
  if (!make_map(&tb, g.B, g.b_rows, g.b_cols, g.b_ld, B_MN ? BK : BN)) return cudaErrorInvalidValue;
  Params p;
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K; p.groups = (int)g.groups;
  p.tiles_m = (int)((g.M + BM - 1) / BM);
  p.tiles_n = (int)(g.N / BN);
  const int kblocks = (int)((g.K + BK - 1) / BK);
  p.splits = effective_splits(g.K, g.splits);
  p.kblocks_per_split = (kblocks + p.splits - 1) / p.splits;
  p.total_tiles = p.tiles_m * p.tiles_n * p.groups * p.splits;
  p.a_gm = (int)g.a_gm; p.a_gk = (int)g.a_gk; p.b_gn = (int)g.b_gn; p.b_gk = (int)g.b_gk;
  fill_segments(g, p);
  p.C = g.C; p.ldc = g.ldc; p.c_gs = g.c_gs; p.c_split = g.c_split;
  p.epi = g.epi;
  p.err = device_error_word();
  p.epi_wait_ns = g.epi_wait_ns ? g.epi_wait_ns : kWaitLimitNs;
  auto kern = umma_gemm_kernel<BN, A_MN, B_MN, OUT_F32, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.total_tiles, sm_count());
  TraceScope t(name, s);
  e = launch_k(kern, dim3(grid), dim3(kThreads), smem, s, ta, tb, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool A_MN, bool B_MN, bool OUT_F32, bool B_I8>
cudaError_t launch_pair_t(const Gemm& g, cudaStream_t s, const char* name) {
  using Cfg = PairCfg<B_I8, OUT_F32>;
  constexpr size_t smem = Cfg::SMEM;
  CUtensorMap ta, tb;
  if (!make_map(&ta, g.A, g.a_rows, g.a_cols, g.a_ld, A_MN ? BK : 128)) return cudaErrorInvalidValue;
  if constexpr (B_I8) {
    // B_MN: 64 K lines of 128 N bytes; K-major: 128 N lines of 64 K bytes
    if (!make_map_u8(&tb, g.B, g.b_rows, g.b_cols, g.b_ld, B_MN ? 128 : BK, B_MN ? BK : 128))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map(&tb, g.B, g.b_rows, g.b_cols, g.b_ld, B_MN ? BK : 128)) return cudaErrorInvalidValue;
  }
  // bf16 output through TMA stores: C as a 2-D [M][ldc] tensor, 64 x 32 boxes, 128-byte swizzle
  CUtensorMap tc = ta;   // fp32 outputs keep the thread stores; the map is then unused
  if constexpr (!OUT_F32) {
    // a group offset c_gs is a column offset (< ldc: every group in the same M rows) or whole
    // rows (a multiple of ldc: group g starts g * c_gs / ldc rows down). The map holds exactly
    // the rows the product owns, so the copy clips a ragged last row tile at row M of its group.
    if (g.c_gs % g.ldc != 0 && g.c_gs >= g.ldc) return cudaErrorNotSupported;
    if (g.c_gs % g.ldc != 0 && (g.groups - 1) * g.c_gs + g.N > g.ldc) return cudaErrorNotSupported;
    const int64_t rows = (g.c_gs % g.ldc == 0) ? (g.groups - 1) * (g.c_gs / g.ldc) + g.M : g.M;
    if (!make_map(&tc, g.C, rows, g.ldc, g.ldc, 32)) return cudaErrorInvalidValue;
  }
  // the second operand pair (groups >= groups_1), same box shapes and swizzle
  CUtensorMap ta2 = ta, tb2 = tb;
  if (g.A2) {
    if constexpr (B_I8) return cudaErrorNotSupported;
    if (!make_map(&ta2, g.A2, g.a2_rows, g.a2_cols, g.a2_ld, A_MN ? BK : 128) ||
        !make_map(&tb2, g.B2, g.b2_rows, g.b2_cols, g.b2_ld, B_MN ? BK : 128))
      return cudaErrorInvalidValue;
  }
  PairParams p;
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K; p.groups = (int)g.groups;
  p.g2 = g.A2 ? (int)g.groups_1 : (int)g.groups;
  p.tiles_m = (int)((g.M + 255) / 256);
  p.tiles_n = (int)(g.N / 256);
  const int kblocks = (int)((g.K + BK - 1) / BK);
  p.splits = effective_splits(g.K, g.splits);
  p.kblocks_per_split = (kblocks + p.splits - 1) / p.splits;
  p.total_tiles = p.tiles_m * p.tiles_n * p.groups * p.splits;
  p.narrow_from = p.total_tiles;
  p.a_gm = (int)g.a_gm; p.a_gk = (int)g.a_gk; p.b_gn = (int)g.b_gn; p.b_gk = (int)g.b_gk;
  fill_segments(g, p);
  p.C = g.C; p.ldc = g.ldc; p.c_gs = g.c_gs; p.c_split = g.c_split;
  p.b_scale = g.b_scale;
  // dense products: wide N keeps bands of 16 pair-rows (W0' swept T / 4096 times); narrow N
  // with a long K (dA' = dB W0'^T) sweeps M under bands of 8 pair-columns
  p.raster = 0;
  p.band = 8;
  if (p.groups == 1 && p.splits == 1) {
    if (p.tiles_n <= 16 && p.tiles_m >= 32 && g.K >= 8192) {
      p.raster = 1;   // the band's B columns are shared by every row tile of the band
      p.band = 8;
    } else {
      p.band = 16;    // the band's A rows are shared by every column tile of the band
    }
  }
  p.epi = g.epi;
  p.epi2 = g.has_epi2 ? g.epi2 : g.epi;
  p.deps = g.deps;
  p.dep_target = g.dep_target;
  p.dep_blocks = g.dep_blocks > 0 ? g.dep_blocks : 1;
  p.c_rel2 = g.c_rel2 ? 1 : 0;
  p.err = device_error_word();
  p.epi_wait_ns = g.epi_wait_ns ? g.epi_wait_ns : kWaitLimitNs;
  auto kern = umma_gemm_pair_kernel<A_MN, B_MN, OUT_F32, B_I8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl_attr(attr[1]);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;   // the occupancy query sees the cluster shape only
  static int max_clusters = 0;
  if (!max_clusters) {
    cfg.gridDim = dim3(2 * 74, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
        max_clusters <= 0)
      max_clusters = sm_count() / 2;
  }
  cfg.numAttrs = 2;
  const int clusters = std::min(p.total_tiles, max_clusters);
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  TraceScope t(name, s);
  e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, ta2, tb2, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool A_MN, bool B_MN, bool OUT_F32, bool COLLECT>
cudaError_t launch_wide_t(const Gemm& g, cudaStream_t s, const char* name) {
  constexpr size_t smem = WideCfg::SMEM;
  CUtensorMap ta, tb;
  if (!make_map(&ta, g.A, g.a_rows, g.a_cols, g.a_ld, A_MN ? BK : 128)) return cudaErrorInvalidValue;
  if (!make_map(&tb, g.B, g.b_rows, g.b_cols, g.b_ld, B_MN ? BK : 128)) return cudaErrorInvalidValue;
  // bf16 C as a 2-D [rows][ldc] tensor holding exactly the rows the product owns (see
  // launch_pair_t); fp32 outputs keep the thread stores and the map is unused
  CUtensorMap tc = ta;
  if constexpr (!OUT_F32) {
    const int64_t crows = (g.c_gs % g.ldc == 0) ? (g.groups - 1) * (g.c_gs / g.ldc) + g.M : g.M;
    if (!make_map(&tc, g.C, crows, g.ldc, g.ldc, 32)) return cudaErrorInvalidValue;
  }
  CUtensorMap ta2 = ta, tb2 = tb;
  if (g.A2) {
    if (!make_map(&ta2, g.A2, g.a2_rows, g.a2_cols, g.a2_ld, A_MN ? BK : 128) ||
        !make_map(&tb2, g.B2, g.b2_rows, g.b2_cols, g.b2_ld, B_MN ? BK : 128))
      return cudaErrorInvalidValue;
  }
  PairParams p{};
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K; p.groups = (int)g.groups;
  p.g2 = g.A2 ? (int)g.groups_1 : (int)g.groups;
  p.tiles_m = (int)((g.M + 255) / 256);
  p.tiles_n = (int)(g.N / 512);
  const int kblocks = (int)((g.K + BK - 1) / BK);
  p.splits = effective_splits(g.K, g.splits);
  p.kblocks_per_split = (kblocks + p.splits - 1) / p.splits;
  p.total_tiles = p.tiles_m * p.tiles_n * p.groups * p.splits;
  p.narrow_from = p.total_tiles;
  p.a_gm = (int)g.a_gm; p.a_gk = (int)g.a_gk; p.b_gn = (int)g.b_gn; p.b_gk = (int)g.b_gk;
  p.nseg = 1; p.kb_per_seg = p.kblocks_per_split;
  p.C = g.C; p.ldc = g.ldc; p.c_gs = g.c_gs; p.c_split = g.c_split;
  // as for the 256 x 256 tiles: narrow N with a long K sweeps M under bands of pair-columns
  // (the band's W0' columns stay in L2), otherwise bands of pair-rows sweep N
  p.raster = 0;
  p.band = p.groups == 1 ? 16 : 8;
  if (p.groups == 1 && p.splits == 1 && p.tiles_n <= 8 && p.tiles_m >= 32 && g.K >= 8192) {
    p.raster = 1;
    p.band = 8;
  }
  p.err = device_error_word();
  p.epi_wait_ns = g.epi_wait_ns ? g.epi_wait_ns : kWaitLimitNs;
  auto kern = umma_gemm_wide_kernel<A_MN, B_MN, OUT_F32, COLLECT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl_attr(attr[1]);
  cfg.blockDim = dim3(WideCfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters = 0;
  if (!max_clusters) {
    cfg.gridDim = dim3(2 * 74, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
        max_clusters <= 0)
      max_clusters = sm_count() / 2;
  }
  cfg.numAttrs = 2;
  // Last partial wave: when it holds at most half the clusters, its tiles are split into two
  // half-width tiles each, so that it takes about half a tile's time instead of a whole one.
  const int rem = p.total_tiles % max_clusters;
  if (p.total_tiles > max_clusters && rem > 0 && 2 * rem <= max_clusters) {
    p.narrow_from = p.total_tiles - rem;
    p.total_tiles += rem;
  }
  const int clusters = std::min(p.total_tiles, max_clusters);
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  TraceScope t(name, s);
  e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, ta2, tb2, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_w0p_fused(const void* A1, const void* W0, const void* Gp, void* Bout,
                             void* Cout, int64_t T, int64_t m, int64_t n, cudaStream_t s) {
  constexpr size_t smem = FusedCfg::SMEM;
  CUtensorMap ta, tw, tg, tbo, tco;
  if (!make_map(&ta, A1, T, m, m, 128) || !make_map(&tw, W0, m, n, n, BK) ||
      !make_map(&tg, Gp, n, 512, 512, BK) || !make_map(&tco, Cout, T, n, n, 32))
    return cudaErrorInvalidValue;
  tbo = tco;
  if (Bout && !make_map(&tbo, Bout, T, n, n, 32)) return cudaErrorInvalidValue;
  PairParams p{};
  p.M = (int)T; p.N = (int)n; p.K = (int)m; p.groups = 1; p.g2 = 1;
  p.tiles_m = (int)((T + 255) / 256);
  p.tiles_n = (int)(n / 512);   // one tile column per P block
  p.splits = 1;
  p.kblocks_per_split = (int)((m + BK - 1) / BK);
  p.total_tiles = p.tiles_m * p.tiles_n;
  p.narrow_from = p.total_tiles;
  p.nseg = 1; p.kb_per_seg = p.kblocks_per_split;
  p.C = Cout; p.ldc = n;
  // the W0' product's forward raster: bands of 16 pair-rows sweep the P blocks
  p.raster = 0;
  p.band = 16;
  p.err = device_error_word();
  p.epi_wait_ns = kWaitLimitNs;
  auto kern = umma_w0p_fused_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl_attr(attr[1]);
  cfg.blockDim = dim3(FusedCfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters = 0;
  if (!max_clusters) {
    cfg.gridDim = dim3(2 * 74, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
        max_clusters <= 0)
      max_clusters = sm_count() / 2;
  }
  cfg.numAttrs = 2;
  const int clusters = std::min(p.total_tiles, max_clusters);
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  TraceScope t("umma_w0p_fused", s);
  e = cudaLaunchKernelEx(&cfg, kern, ta, tw, tg, tbo, tco, p, Bout ? 1 : 0);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int BN>
cudaError_t dispatch_majors(const Gemm& g, cudaStream_t s) {
#define POETX_UM(AM, BMJ, F)                                                                   \
  if (g.a_mn == AM && g.b_mn == BMJ && g.out_f32 == F)                                         \
    return launch_t<BN, AM, BMJ, F>(g, s, g.name ? g.name : "umma_gemm");
  POETX_UM(false, false, false)
  POETX_UM(false, true, false)
  POETX_UM(true, true, true)
  POETX_UM(false, false, true)
  POETX_UM(false, true, true)
#undef POETX_UM
  return cudaErrorNotSupported;
}

}  // namespace

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

int effective_splits(int64_t K, int64_t splits) {
  const int64_t kblocks = (K + BK - 1) / BK;
  const int64_t s = std::max<int64_t>(1, std::min<int64_t>(splits, kblocks));
  const int64_t per = (kblocks + s - 1) / s;
  return (int)((kblocks + per - 1) / per);
}

bool supported(const Gemm& g) {
  if (!encode_fn()) return false;
  if (g.b_i8) return false;   // int8 B: CTA-pair kernel only (pair_supported)
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.groups <= 0) return false;
  if (g.K % BK != 0 && g.groups > 1 && g.a_gk + g.b_gk != 0) return false;
  if (g.N % 64 != 0) return false;
  if (g.a_cols % 8 || g.b_cols % 8 || g.a_ld % 8 || g.b_ld % 8) return false;
  if ((reinterpret_cast<uintptr_t>(g.A) | reinterpret_cast<uintptr_t>(g.B) |
       reinterpret_cast<uintptr_t>(g.C)) & 15)
    return false;
  if (g.ldc % (g.out_f32 ? 4 : 8)) return false;
  if (g.a_cols < 64 || g.b_cols < 64) return false;
  // coordinates must fit in int32 and offsets must keep 64-element alignment
  const int64_t lim = (int64_t)1 << 31;
  if (g.a_rows >= lim || g.a_cols >= lim || g.b_rows >= lim || g.b_cols >= lim) return false;
  if ((g.a_gm | g.a_gk | g.b_gn | g.b_gk) % 64) return false;
  if (g.nseg < 1 || g.nseg > 3) return false;
  if (g.nseg > 1) {
    if (g.K % (64 * g.nseg) || g.splits != 1) return false;
    for (int s = 0; s < g.nseg; ++s)
      if ((g.a_dx[s] | g.b_dx[s]) % 64 || g.a_dx[s] < 0 || g.a_dy[s] < 0 || g.b_dx[s] < 0 ||
          g.b_dy[s] < 0)
        return false;
  }
  if (g.epi.mode != kEpiStore) {
    // grouped b x b blocks with fp32 accumulators; 16-byte aligned rows of 4 elements
    if (!g.out_f32 || g.M != g.epi.b || g.N != g.epi.b || g.epi.b % 8 || !g.epi.qh ||
        g.splits != 1)
      return false;
  }
  return true;
}

bool pair_supported(const Gemm& g) {
  if (g.b_i8) {
    // int8 B with per-column scales: one dense product, bf16 A K-major, bf16 out
    Gemm h = g;
    h.b_i8 = false;
    return supported(h) && g.N % 256 == 0 && g.M >= 256 && g.groups == 1 && g.splits == 1 &&
           g.nseg == 1 && g.epi.mode == kEpiStore &&
           !g.a_mn && !g.out_f32 && g.b_scale && g.b_ld % 16 == 0 && g.b_cols % 16 == 0 &&
           (reinterpret_cast<uintptr_t>(g.b_scale) & 15) == 0;
  }
  if (g.A2) {
    // a second operand pair: both sets must be valid operands of the same grouped product
    Gemm h = g;
    h.A = g.A2; h.a_rows = g.a2_rows; h.a_cols = g.a2_cols; h.a_ld = g.a2_ld;
    h.B = g.B2; h.b_rows = g.b2_rows; h.b_cols = g.b2_cols; h.b_ld = g.b2_ld;
    h.A2 = nullptr; h.B2 = nullptr;
    h.groups = g.groups - g.groups_1;
    h.has_epi2 = false; h.deps = nullptr;
    if (g.has_epi2) h.epi = g.epi2;
    Gemm f = g;
    f.A2 = nullptr; f.B2 = nullptr;
    f.groups = g.groups_1;
    f.has_epi2 = false; f.deps = nullptr;
    // epilogue modes per product need fp32 accumulator outputs (the modes' own rule), and a
    // published dependency needs the first product's stores to be plain stores (fp32 out)
    const bool modes_ok = g.has_epi2 ? g.out_f32 : g.epi.mode == kEpiStore;
    return g.B2 && g.groups_1 > 0 && g.groups_1 < g.groups && !g.b_i8 && modes_ok &&
           (!g.deps || (g.out_f32 && g.dep_target > 0)) && pair_supported(f) &&
           pair_supported(h);
  }
  return supported(g) && g.N % 256 == 0 && g.M >= 256 && !(g.a_mn && !g.b_mn) &&
         !(g.a_mn && g.b_mn && !g.out_f32) && (g.groups == 1 || g.a_gm == 0 || g.a_gm % 256 == 0);
}

cudaError_t gemm_pair(const Gemm& g, cudaStream_t s) {
  const char* name = g.name ? g.name : "umma_gemm_pair";
  if (g.b_i8) {
    if (g.a_mn || g.out_f32) return cudaErrorNotSupported;
    return g.b_mn ? launch_pair_t<false, true, false, true>(g, s, name)
                  : launch_pair_t<false, false, false, true>(g, s, name);
  }
#define POETX_UP(AM, BMJ, F) \
  if (g.a_mn == AM && g.b_mn == BMJ && g.out_f32 == F) \
    return launch_pair_t<AM, BMJ, F, false>(g, s, name);
  POETX_UP(false, false, false)
  POETX_UP(false, true, false)
  POETX_UP(true, true, true)
  POETX_UP(false, false, true)
  POETX_UP(false, true, true)
#undef POETX_UP
  return cudaErrorNotSupported;
}

bool wide_supported(const Gemm& g) {
  if (g.b_i8 || g.nseg != 1 || g.epi.mode != kEpiStore || g.N % 512 != 0 || g.M < 256)
    return false;
  if (g.A2) {
    // a second operand pair: both sets valid operands of the same grouped product
    Gemm h = g;
    h.A = g.A2; h.a_rows = g.a2_rows; h.a_cols = g.a2_cols; h.a_ld = g.a2_ld;
    h.B = g.B2; h.b_rows = g.b2_rows; h.b_cols = g.b2_cols; h.b_ld = g.b2_ld;
    h.A2 = nullptr; h.B2 = nullptr;
    h.groups = g.groups - g.groups_1;
    Gemm f = g;
    f.A2 = nullptr; f.B2 = nullptr;
    f.groups = g.groups_1;
    return g.B2 && g.groups_1 > 0 && g.groups_1 < g.groups && wide_supported(f) &&
           wide_supported(h);
  }
  // operand layouts of the 256 x 256 kernel: A M-major only with B N-major and fp32 out
  if (!supported(g) || (g.a_mn && !g.b_mn) || (g.a_mn && g.b_mn && !g.out_f32)) return false;
  if (g.groups == 1) return true;
  // groups: A's row offsets in whole pair tiles; bf16 output groups are column offsets inside
  // one row (the output map's rows are the product's M) or whole rows
  if (g.a_gm % 256) return false;
  if (!g.out_f32 && g.c_gs % g.ldc != 0 &&
      (g.c_gs >= g.ldc || (g.groups - 1) * g.c_gs + g.N > g.ldc))
    return false;
  return true;
}

cudaError_t gemm_wide(const Gemm& g, cudaStream_t s) {
  if (!wide_supported(g)) return cudaErrorNotSupported;
  const char* name = g.name ? g.name : "umma_gemm_wide";
#define POETX_UW(AM, BMJ, F, C)                                        \
  if (g.a_mn == AM && g.b_mn == BMJ && g.out_f32 == F && g.wide_collect == C) \
    return launch_wide_t<AM, BMJ, F, C>(g, s, name);
  POETX_UW(false, false, false, true)
  POETX_UW(false, true, false, true)
  POETX_UW(false, false, false, false)
  POETX_UW(false, true, false, false)
  POETX_UW(true, true, true, true)
#undef POETX_UW
  return cudaErrorNotSupported;
}

bool w0p_fused_supported(const void* A1, const void* W0, const void* Gp, const void* Bout,
                         const void* Cout, int64_t T, int64_t m, int64_t n, int64_t b) {
  if (!encode_fn() || b != 512 || T < 256 || m < 512 || n < 512 || m % 512 || n % 512) return false;
  const int64_t lim = (int64_t)1 << 31;
  if (T >= lim || m >= lim || n >= lim) return false;
  return ((reinterpret_cast<uintptr_t>(A1) | reinterpret_cast<uintptr_t>(W0) |
           reinterpret_cast<uintptr_t>(Gp) | reinterpret_cast<uintptr_t>(Bout) |
           reinterpret_cast<uintptr_t>(Cout)) & 15) == 0;
}

cudaError_t w0p_fused(const void* A1, const void* W0, const void* Gp, void* Bout, void* Cout,
                      int64_t T, int64_t m, int64_t n, int64_t b, cudaStream_t s) {
  if (!w0p_fused_supported(A1, W0, Gp, Bout, Cout, T, m, n, b)) return cudaErrorNotSupported;
  return launch_w0p_fused(A1, W0, Gp, Bout, Cout, T, m, n, s);
}

cudaError_t gemm(const Gemm& g, cudaStream_t s) {
  if (g.A2) return cudaErrorNotSupported;   // the second operand pair is CTA-pair only
  if (g.bn != 0 && g.bn != 64 && g.bn != 128 && g.bn != 256) return cudaErrorInvalidValue;
  const int cap = g.bn ? g.bn : 256;
  if (g.N % 256 == 0 && cap >= 256) return dispatch_majors<256>(g, s);
  if (g.N % 128 == 0 && cap >= 128) return dispatch_majors<128>(g, s);
  return dispatch_majors<64>(g, s);
}

}  // namespace umma
}  // namespace poetx
