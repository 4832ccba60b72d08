/*
 * poetx.h — C ABI of the POET-X linear layer on NVIDIA B200 (sm_100a).
 *
 * The layer is the spectrum-preserving linear map
 *     y = (R W0 P)^T x            (row form, token-major X [T, m]:  Y = X R W0 P)
 * with W0 [m, n] fixed, and R, P block-stochastic orthogonal matrices
 *     R = Psi_R^T Diag(G_R^1 .. G_R^{m/b}) Psi_R,   P = Psi_P^T Diag(G_P^1 .. G_P^{n/b}) Psi_P
 * whose b x b blocks come from the Cayley-Neumann parameterisation
 *     G = I + 2(Q + Q^2 + Q^3) + Q^4  of a skew-symmetric Q stored as its packed strict upper triangle.
 * Sources (web pages):
 *   "Reparameterized LLM Training via Orthogonal Equivalence Transformation" (POET paper notes):
 *       §整体框架 (W_RP = R W0 P, y = W_RP^T x), §1 SPO (block-stochastic form), §2 CNP (k = 3),
 *       §3 Merge-then-Reinitialize.
 *   "在单张 H100 上预训练 13B 模型：POET-X 如何把正交变换的内存开销砍到 1/3" (POET-X blog):
 *       §第一斧 input-centric evaluation, §第二斧 index permutations and merging 2 of 4 into W,
 *       §第三斧 batch-wise block-diagonal products, §第四斧 packed triangle and the Q/Q^2 form of CNP,
 *       §第五斧 forward steps a = G_R^T x, b = W a, z = G_P^T b.
 *
 * Conventions shared by every call:
 *  - All tensor pointers are DEVICE pointers to row-major, contiguous memory owned by the caller.
 *    The library never allocates or frees device memory; calls that need scratch take a caller
 *    workspace whose size the matching *_workspace_bytes query returns.
 *  - A permutation is an int32 array pi of length k with Psi[i, pi[i]] = 1: X Psi^T = X[:, pi]
 *    (column gather) and, for C Psi = Y, Y[:, pi[i]] = C[:, i] (column scatter).
 *  - The merged weight is W0' = Psi_R W0 Psi_P^T, i.e. W0'[i, j] = W0[perm_r[i], perm_p[j]].
 *  - q of one block holds Q[i, j] (i < j) in row-major order of the strict upper triangle;
 *    Q[j, i] = -Q[i, j]; b(b-1)/2 floats per block.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call only enqueues
 *    work on it and returns; nothing synchronises, except where a comment says so.
 *  - Errors found on the host (bad arguments, shapes, alignment, workspace) return before any
 *    launch and leave every output untouched. POETX_ERR_CUDA reports a failed launch or runtime
 *    call; poetx_last_error_message() gives details (per host thread).
 *  - Pointers must be 16-byte aligned (POETX_ERR_ALIGN). Row strides are the logical widths,
 *    which for BF16 must be multiples of 8 elements (m, n, b, T-independent).
 *  - Outputs are overwritten (never accumulated into).
 */
#ifndef POETX_H
#define POETX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  POETX_OK = 0,
  POETX_ERR_INVALID_ARG = 1, /* a required pointer is NULL, a size is negative, an enum is unknown */
  POETX_ERR_SHAPE = 2,       /* b does not divide m or n, or a size is outside the supported range */
  POETX_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  POETX_ERR_DTYPE = 4,       /* dtype not supported by this call */
  POETX_ERR_BAD_INDEX = 5,   /* poetx_validate_permutation: the array is not a permutation */
  POETX_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
  POETX_ERR_UNSUPPORTED = 7, /* the current device is not sm_100 */
  POETX_ERR_WORKSPACE = 8,   /* workspace is NULL or smaller than the query says */
  POETX_ERR_TIMEOUT = 9      /* poetx_device_status: a kernel's bounded wait expired */
} poetx_status;

typedef enum { POETX_F32 = 0, POETX_BF16 = 1 } poetx_dtype;

/* poetx_layer.flags bit: W0' is stored in 8 bits ("POET-XQ": only the low-precision weights are
 * kept and dequantised on demand — "[Project POET-X] Scaling Orthogonal Equivalence ..."
 * §Quantized Training (POET-XQ); "POET-X: Memory-efficient LLM Training ..." (gist.science)
 * §Resumo técnico 2 Metodologia). The pages give no format; this library uses symmetric int8
 * codes with one fp32 scale per column of W0' (poetx_quantize_w0). w0m then points to int8
 * [m, n] codes, w0m_scale to fp32 [n] scales, and the layer computes exactly as the BF16 layer
 * whose W0' is bf16(code * scale) (poetx_dequantize_w0): the W0' products dequantise each int8
 * tile in shared memory inside the tensor-core kernel (T >= 256 and n, m multiples of 256;
 * other shapes dequantise into the workspace first). Requires dtype == POETX_BF16 and m, n
 * multiples of 16. */
#define POETX_LAYER_W0M_I8 1
/* With POETX_LAYER_W0M_I8: dequantise W0' into the workspace (m*n bf16) once per W0' product and
 * run the bf16 product on it, instead of dequantising each tile inside the product. Results are
 * bitwise the same; it needs 2*m*n more workspace bytes and is faster on this part, because
 * the in-kernel conversion is repeated for every row tile of tokens. */
#define POETX_LAYER_W0M_STAGED 2
/* poetx_layer.flags bit (may be combined with the others): the forward runs the W0' product and
 * the P-block product as one kernel wherever that kernel covers the layer (bf16, bf16 W0',
 * b = 512, T >= 256, m and n multiples of 512; other layers take the two launches). Each 256 x
 * 512 tile of B = A' W0' spans one P block: it is finished on chip, multiplied by G_P^j there and
 * only then stored, so B is not read back from HBM, and when saved_b is NULL (POET-Xmem) it is
 * not written at all (back-to-back fusion, "POET-X" blog §第四斧 / §第五斧). Results are bitwise
 * those of the two-launch forward. Off by default: on this part the drain of B into shared
 * memory and the refill of the operand ring after the G_P product stall the tensor core once per
 * tile, and the fused forward measured the same time as the two launches at the 8B shapes. */
#define POETX_LAYER_FUSED_W0_P 4

/* One POET-X linear. Every pointer is a device pointer owned by the caller. */
typedef struct {
  int64_t m;       /* in-features: rows of W0 */
  int64_t n;       /* out-features: columns of W0 */
  int64_t b;       /* block size; must divide m and n */
  int32_t dtype;   /* poetx_dtype of w0m, activations, saved_b, gradients and g_*_lp */
  int32_t flags;   /* 0, POETX_LAYER_W0M_I8, or POETX_LAYER_W0M_I8 | POETX_LAYER_W0M_STAGED;
                      optionally | POETX_LAYER_FUSED_W0_P */
  void* w0m;       /* [m, n] merged weight W0' (see poetx_merge_permutations); int8 codes
                      when flags has POETX_LAYER_W0M_I8 */
  int32_t* perm_r; /* [m] permutation of R: each of 0..m-1 exactly once */
  int32_t* perm_p; /* [n] permutation of P: each of 0..n-1 exactly once. Not checked on the
                      hot path (poetx_validate_permutation checks one): an index outside the
                      range is undefined behaviour and can make a kernel access memory out of
                      bounds. */
  float* q_r;      /* [m/b, b(b-1)/2] packed skew parameters of R */
  float* q_p;      /* [n/b, b(b-1)/2] packed skew parameters of P */
  float* g_r;      /* [m/b, b, b] fp32 CNP blocks of R (written by poetx_cnp_build) */
  float* g_p;      /* [n/b, b, b] fp32 CNP blocks of P */
  void* g_r_lp;    /* [m/b, b, b] bf16 copy of g_r; required when dtype == POETX_BF16 */
  void* g_p_lp;    /* [n/b, b, b] bf16 copy of g_p; required when dtype == POETX_BF16 */
  float* w0m_scale; /* [n] fp32 column scales of the int8 W0' (POETX_LAYER_W0M_I8), else NULL */
} poetx_layer;

/* ---------------------------------------------------------------------------------------------
 * poetx_cnp_build — packed skew parameters -> Cayley-Neumann blocks.
 *   G = I + 2(Q + Q^2 + Q^2 Q) + Q^2 Q^2 per block ("POET-X" blog §第四斧 item 2; the truncated
 *   Neumann series of "Reparameterized LLM Training ..." §2 CNP with k = 3).
 *   q      [nblocks, b(b-1)/2] fp32, read only.
 *   g      [nblocks, b, b] fp32 output, row-major blocks (may be NULL if g_lp is given).
 *   g_lp   [nblocks, b, b] output in lp_dtype (POETX_BF16, round-to-nearest-even), may be NULL.
 *   workspace >= poetx_cnp_workspace_bytes(nblocks, b) bytes of device scratch.
 *   Accuracy: fp32 output within ~1e-6 absolute of the exact polynomial for |Q| entries <= 0.05.
 *   Errors: INVALID_ARG (q NULL, both outputs NULL, nblocks < 0, b < 2), SHAPE (b > 1024),
 *           WORKSPACE, ALIGN, DTYPE (lp_dtype not BF16 while g_lp != NULL).
 * ------------------------------------------------------------------------------------------- */
size_t poetx_cnp_workspace_bytes(int64_t nblocks, int64_t b);
poetx_status poetx_cnp_build(const float* q, int64_t nblocks, int64_t b, float* g, void* g_lp,
                             int32_t lp_dtype, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_layer_cnp_build — poetx_cnp_build of both sides of a layer in one launch sequence:
 *   L->q_r -> L->g_r (and L->g_r_lp for BF16 layers), L->q_p -> L->g_p (L->g_p_lp). The same
 *   arithmetic as two poetx_cnp_build calls; one pass over all m/b + n/b blocks fills the GPU
 *   better than two.
 *   workspace >= poetx_layer_cnp_workspace_bytes(L). Errors: as poetx_cnp_build, plus those of
 *   the layer descriptor (see poetx_linear_fwd) and INVALID_ARG if q_r or q_p is NULL.
 * ------------------------------------------------------------------------------------------- */
size_t poetx_layer_cnp_workspace_bytes(const poetx_layer* L);
poetx_status poetx_layer_cnp_build(const poetx_layer* L, void* workspace, size_t ws_bytes,
                                   void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_layers_cnp_build — poetx_layer_cnp_build for a set of layers (a model's linears): every
 *   layer's R and P blocks, up to eight layers per launch sequence. One layer's blocks fill a
 *   b x b product launch with a wave or two of tiles; a set of layers gives the products many
 *   waves. Same arithmetic and bit-identical results as one poetx_layer_cnp_build per layer.
 *   layers[0 .. nlayers-1]: host array of layer descriptors, all with the same b and dtype
 *   (else SHAPE / DTYPE), each with q_r and q_p. nlayers = 0 does nothing.
 *   workspace >= poetx_layers_cnp_workspace_bytes(layers, nlayers) (0 for a bad layer pointer).
 *   Errors: as poetx_layer_cnp_build for any layer, plus INVALID_ARG for nlayers < 0.
 * ------------------------------------------------------------------------------------------- */
size_t poetx_layers_cnp_workspace_bytes(const poetx_layer* const* layers, int32_t nlayers);
poetx_status poetx_layers_cnp_build(const poetx_layer* const* layers, int32_t nlayers,
                                    void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_cnp_build_noalloc — poetx_cnp_build for callers that cannot allocate device memory.
 *   The pages have no counterpart to this call; it exists for library users only. Some callers
 *   may not allocate device memory when they build the blocks (a host program that hands out all
 *   device memory at start-up and forbids later allocation, or code that must not risk the
 *   device-wide synchronisation of cudaMalloc/cudaFree). This variant takes no workspace: its
 *   scratch is a fixed POETX_CNP_NOALLOC_SCRATCH_BYTES buffer inside the library's own device
 *   memory, which every GPU that loads the library holds until the process exits. It allocates
 *   nothing and calls no allocating routine.
 *   Arguments, outputs and accuracy are those of poetx_cnp_build; any nblocks is accepted (the
 *   blocks are processed in chunks that fit the buffer).
 *   Limit: b must need at most POETX_CNP_NOALLOC_SCRATCH_BYTES of scratch for ONE block
 *   (12*b*b bytes, in slices rounded up to 256 bytes): b <= 836; larger b returns
 *   POETX_ERR_SHAPE with a message.
 *   Set-up: the first call on each device looks up the buffer's device address
 *   (cudaGetSymbolAddress) with that device current. With lazy module loading (the CUDA
 *   default) that lookup is also where the driver loads the library's module holding the
 *   buffer and commits its device memory. So make the first call on each device before the
 *   stretch of the program that must not allocate, and before any stream capture. A call with
 *   nblocks = 0 does exactly this set-up (and its checks) and launches nothing.
 *   All calls on a device share the one buffer and it keeps the last call's contents (nothing in
 *   it needs to start at zero: every byte read is written earlier in the same call). Calls whose
 *   work overlaps on the GPU (e.g. on two streams without ordering) race on the buffer: order
 *   them on one stream or with events.
 * ------------------------------------------------------------------------------------------- */
#define POETX_CNP_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
poetx_status poetx_cnp_build_noalloc(const float* q, int64_t nblocks, int64_t b, float* g,
                                     void* g_lp, int32_t lp_dtype, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_linear_fwd — Y = X Psi_R^T Diag(G_R) W0' Diag(G_P) Psi_P, input-centric
 *   ("POET-X" blog §第一斧 and §第五斧; permutations as index maps, §第二斧; per-block batched
 *   products, §第三斧). R W0 P is never formed. Steps:
 *     A = X[:, perm_r];  A'_j = A_j G_R^j;  B = A' W0';  C_j = B_j G_P^j;  Y[:, perm_p] = C.
 *   x       [T, m] (layer dtype), read only.        y [T, n] output.
 *   saved_b [T, n] output: B, kept for the backward pass (may be NULL when no backward follows).
 *   Uses L->g_r/g_p (F32) or L->g_r_lp/g_p_lp (BF16) as built by poetx_cnp_build.
 *   BF16 layers compute in bf16 x bf16 -> fp32 on tensor cores and round A', B, C, Y to bf16.
 *   workspace >= poetx_fwd_workspace_bytes(L, T).
 *   Errors: INVALID_ARG, SHAPE (T < 0, b does not divide m or n), ALIGN, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------------------------- */
size_t poetx_fwd_workspace_bytes(const poetx_layer* L, int64_t T);
poetx_status poetx_linear_fwd(const poetx_layer* L, const void* x, int64_t T, void* y,
                              void* saved_b, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_linear_bwd — exact gradient of poetx_linear_fwd for upstream dY:
 *     dC = dY[:, perm_p];  dB_j = dC_j (G_P^j)^T;  dG_P^j = B_j^T dC_j;  dA' = dB W0'^T;
 *     dA_j = dA'_j (G_R^j)^T;  dG_R^j = A_j^T dA'_j (A = X[:, perm_r]);  dX[:, perm_r] = dA;
 *     dq = skew-packed gradient of the CNP polynomial at q (chain rule through G(Q)).
 *   x [T, m], dy [T, n], saved_b [T, n] (from the forward on the same x and layer state).
 *   saved_b may be NULL (memory-saving mode, "POET-Xmem" in "POET-X: Memory-efficient LLM
 *   Training ..." §2 Metodologia / the POET-X blog §第五斧): B is then rebuilt exactly as
 *   (X[:, perm_r] Diag(G_R)) W0' inside the call, which costs one more W0' product (2 T m n
 *   FLOP) and needs no [T, n] buffer between forward and backward. (The pages' cheaper
 *   B = C G_P^T is exact only for orthogonal G, which CNP is not, so it is not used.)
 *   dx [T, m] output (may be NULL to skip it);  dq_r [m/b, b(b-1)/2], dq_p [n/b, b(b-1)/2]
 *   fp32 outputs (either may be NULL to skip that side). Uses L->q_r/q_p and the G blocks.
 *   workspace >= poetx_bwd_workspace_bytes(L, T).
 *   Errors: as poetx_linear_fwd; dy must not be NULL.
 * ------------------------------------------------------------------------------------------- */
size_t poetx_bwd_workspace_bytes(const poetx_layer* L, int64_t T);
poetx_status poetx_linear_bwd(const poetx_layer* L, const void* x, const void* dy,
                              const void* saved_b, int64_t T, void* dx, float* dq_r, float* dq_p,
                              void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_linear_fwd_ex / poetx_linear_bwd_ex — the same forward and backward, keeping
 *   A = X[:, perm_r] between them ("POET-Xfast" in "POET-X: Memory-efficient LLM Training ..."
 *   §2 Metodologia: activations are saved rather than recomputed).
 *   saved_a [T, m] (layer dtype): the forward writes A there (instead of into its workspace);
 *   the backward reads it wherever it needs A (the per-block gradients dG_R^j = A_j^T dA'_j and,
 *   with saved_b NULL, the rebuild of B) instead of gathering X again, which saves one
 *   [T, m] gather pass per backward for T*m elements of memory. saved_a may be NULL: the calls
 *   are then poetx_linear_fwd / poetx_linear_bwd. With saved_a given, the backward does not read
 *   x and x may be NULL. saved_a must hold the forward's A for the same x and layer state
 *   (perm_r unchanged since: merge_reinit changes it).
 *   Results are bit-identical to the calls without saved_a. Errors: as those calls, plus ALIGN
 *   for a saved_a not 16-byte aligned.
 * ------------------------------------------------------------------------------------------- */
poetx_status poetx_linear_fwd_ex(const poetx_layer* L, const void* x, int64_t T, void* y,
                                 void* saved_b, void* saved_a, void* workspace, size_t ws_bytes,
                                 void* stream);
poetx_status poetx_linear_bwd_ex(const poetx_layer* L, const void* x, const void* dy,
                                 const void* saved_b, const void* saved_a, int64_t T, void* dx,
                                 float* dq_r, float* dq_p, void* workspace, size_t ws_bytes,
                                 void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_linear_bwd_dg — poetx_linear_bwd_ex up to the per-block gradients: the backward's
 *   dL/dG of every block (dG_R^j = A_j^T dA'_j, dG_P^j = B_j^T dC_j, summed over tokens) goes to
 *   dG [m/b + n/b][b][b] fp32 (the R blocks, then the P blocks) and no dq is formed. dx as in
 *   poetx_linear_bwd (may be NULL); saved_a as in poetx_linear_bwd_ex (may be NULL).
 * poetx_layers_dq_from_dg — dq of a set of layers from their dG, one launch sequence over every
 *   layer's blocks (up to eight layers per sequence): the CNP chain rule of poetx_linear_bwd,
 *   run over many more blocks at once than one layer's. For a model's linears, call
 *   poetx_linear_bwd_dg per layer, then this once. Results equal those of poetx_linear_bwd
 *   (the same chain on the same dG) bit for bit.
 *   layers [nlayers] (same b and dtype, each with q_r and q_p), dG [nlayers] (as written by
 *   poetx_linear_bwd_dg, read only), dq_r [nlayers], dq_p [nlayers] outputs (an entry may be
 *   NULL to skip that side). workspace >= poetx_layers_dq_workspace_bytes(layers, nlayers).
 *   Errors: as poetx_layers_cnp_build; ALIGN for a dG or dq entry not 16-byte aligned.
 * ------------------------------------------------------------------------------------------- */
poetx_status poetx_linear_bwd_dg(const poetx_layer* L, const void* x, const void* dy,
                                 const void* saved_b, const void* saved_a, int64_t T, void* dx,
                                 float* dG, void* workspace, size_t ws_bytes, void* stream);
size_t poetx_layers_dq_workspace_bytes(const poetx_layer* const* layers, int32_t nlayers);
poetx_status poetx_layers_dq_from_dg(const poetx_layer* const* layers, const float* const* dG,
                                     float* const* dq_r, float* const* dq_p, int32_t nlayers,
                                     void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_merge_permutations — W0' = Psi_R W0 Psi_P^T ("POET-X" blog §第二斧: the two permutations
 *   next to the fixed W are folded into it before the inner loop).
 *   w0 [m, n] input, w0m [m, n] output (must not overlap w0), dtype F32 or BF16. Bit-exact copy.
 *   perm_r [m], perm_p [n] must be permutations (not checked; see poetx_validate_permutation).
 * ------------------------------------------------------------------------------------------- */
poetx_status poetx_merge_permutations(const void* w0, const int32_t* perm_r,
                                      const int32_t* perm_p, int64_t m, int64_t n, int32_t dtype,
                                      void* w0m, void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_merge_reinit — merge-then-reinitialize ("Reparameterized LLM Training ..." §3):
 *   W <- R W P using the current L->g_r, L->g_p (call poetx_cnp_build first), new permutations
 *   drawn from `seed`, W0' <- the new merge of W, q <- 0. In place on L->w0m, L->perm_r,
 *   L->perm_p, L->q_r, L->q_p. The G blocks are NOT reset: rebuild them with poetx_cnp_build
 *   (q = 0 gives G = I exactly). The layer function is preserved up to rounding of W0'.
 *   For POETX_LAYER_W0M_I8 layers the new W0' is computed from the dequantised one and stored
 *   again as int8 codes and column scales (poetx_quantize_w0), in L->w0m and L->w0m_scale.
 *   Permutation draw: key_l[i] = SplitMix64 output i of the stream started at
 *   SplitMix64 output l of `seed` (l = 0 for R, 1 for P); pi_l sorts indices by (key, index).
 *   workspace >= poetx_merge_reinit_workspace_bytes(L).
 * ------------------------------------------------------------------------------------------- */
size_t poetx_merge_reinit_workspace_bytes(const poetx_layer* L);
poetx_status poetx_merge_reinit(poetx_layer* L, uint64_t seed, void* workspace, size_t ws_bytes,
                                void* stream);

/* ---------------------------------------------------------------------------------------------
 * poetx_quantize_w0 — 8-bit storage of a weight for POETX_LAYER_W0M_I8 layers:
 *     scale[j] = max_i |w[i, j]| / 127,   wq[i, j] = round_half_even(w[i, j] / scale[j]),
 *   both in IEEE fp32 (|wq| <= 127; an all-zero column gets scale 0 and codes 0).
 *   w [m, n] F32 or BF16 (dtype), read only;  wq [m, n] int8 and scale [n] fp32 outputs.
 *   Deterministic: the column maxima are order-independent.
 *   Errors: INVALID_ARG, SHAPE (m or n < 0), DTYPE, ALIGN.
 * poetx_dequantize_w0 — w [m, n] bf16 = bf16(wq[i, j] * scale[j]) (fp32 product, rounded to
 *   nearest even): the exact operand the int8 layer's products use.
 * ------------------------------------------------------------------------------------------- */
poetx_status poetx_quantize_w0(const void* w, int64_t m, int64_t n, int32_t dtype, int8_t* wq,
                               float* scale, void* stream);
poetx_status poetx_dequantize_w0(const int8_t* wq, const float* scale, int64_t m, int64_t n,
                                 void* w_bf16, void* stream);

/* Draw the permutation that poetx_merge_reinit would use for (seed, lane) into perm [k]. */
poetx_status poetx_resample_permutation(uint64_t seed, int32_t lane, int64_t k, int32_t* perm,
                                        void* stream);

/* Check on the device that perm [k] is a permutation of 0..k-1. SYNCHRONISES `stream`.
 * workspace >= 4*k bytes. Returns POETX_OK or POETX_ERR_BAD_INDEX. */
poetx_status poetx_validate_permutation(const int32_t* perm, int64_t k, void* workspace,
                                        size_t ws_bytes, void* stream);

/* Device error flag set by kernels whose bounded waits expired (POETX_ERR_TIMEOUT), then
 * cleared. SYNCHRONISES `stream`. */
poetx_status poetx_device_status(void* stream);

/* Tracing: when enabled, every kernel the library launches is bracketed by CUDA events on its
 * stream. poetx_trace_read() synchronises those events and writes one line per launch,
 * "<kernel name> <milliseconds>\n", into buf (truncated to len), then clears the record.
 * Returns the number of launches recorded. The same names label NVTX ranges for profilers.
 * A bf16 contraction whose shape the tensor-core tiling does not cover (a block size b that is
 * not a multiple of 64, or b < 64) runs on the fp32-accumulating SIMT kernel and is recorded as
 * "simt_gemm_bf16_fallback"; fp32 layers' products are "simt_gemm_f32". */
poetx_status poetx_trace_enable(int32_t on);
int64_t poetx_trace_read(char* buf, size_t len);
/* Record only launches whose name is one of `names` (comma-separated, exact match); NULL or ""
 * records every launch again. Events between two launches keep the second from starting early
 * (see below), so a selective trace disturbs the timing of the untraced launches less.
 * Kernels on the layer's path are launched with programmatic stream serialisation: a kernel may
 * run its set-up while the previous one finishes and waits for it before touching memory.
 * POETX_PDL=0 in the environment turns that off. */
poetx_status poetx_trace_select(const char* names);

const char* poetx_status_string(int32_t status);
const char* poetx_last_error_message(void);
int32_t poetx_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* POETX_H */
