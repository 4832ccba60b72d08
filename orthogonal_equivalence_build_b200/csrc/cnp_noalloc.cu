// poetx_cnp_build_noalloc: the CNP block build without any caller workspace.
//
// Some callers cannot allocate device memory at the point where they build the blocks: a host
// program that hands out all device memory up front and forbids allocation afterwards, or code
// that must not risk the device-wide synchronisation a cudaMalloc/cudaFree can cause. For them
// this variant takes its scratch from a fixed array that lives in the library's own device
// memory, so the caller passes only q and the outputs.
//
// The array is one file-scope __device__ buffer of POETX_CNP_NOALLOC_SCRATCH_BYTES. Every GPU
// that loads the library holds it until the process exits. Blocks are processed in chunks that
// fit the buffer; a block size whose single-block scratch does not fit is rejected.
#include "../../include/poetx.h"
#include "gemm.h"

#include <algorithm>
#include <mutex>

namespace poetx {
namespace {

static __device__ __align__(256) unsigned char g_cnp_scratch[POETX_CNP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_cnp_scratch on the current device. In host code the symbol itself is only
// a host-side stand-in, so the address is looked up once per device, with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_cnp_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace poetx

extern "C" poetx_status poetx_cnp_build_noalloc(const float* q, int64_t nblocks, int64_t b,
                                                float* g, void* g_lp, int32_t lp_dtype,
                                                void* stream) {
  using namespace poetx;
  if (nblocks < 0 || b < 2) {
    set_error("cnp_build_noalloc: nblocks < 0 or b < 2");
    return POETX_ERR_INVALID_ARG;
  }
  if (b > 1024) {
    set_error("cnp_build_noalloc: b=%lld exceeds 1024", (long long)b);
    return POETX_ERR_SHAPE;
  }
  const size_t per_block = gemm_cnp_ws_bytes(1, b);
  if (per_block > (size_t)POETX_CNP_NOALLOC_SCRATCH_BYTES) {
    set_error("cnp_build_noalloc: one block of b=%lld needs %zu scratch bytes, more than the "
              "fixed %zu-byte buffer; use poetx_cnp_build with a workspace",
              (long long)b, per_block, (size_t)POETX_CNP_NOALLOC_SCRATCH_BYTES);
    return POETX_ERR_SHAPE;
  }
  if (nblocks > 0 && !q) {
    set_error("cnp_build_noalloc: q is NULL");
    return POETX_ERR_INVALID_ARG;
  }
  if (nblocks > 0 && !g && !g_lp) {
    set_error("cnp_build_noalloc: both outputs are NULL");
    return POETX_ERR_INVALID_ARG;
  }
  if (g_lp && lp_dtype != POETX_BF16) {
    set_error("cnp_build_noalloc: g_lp must be BF16");
    return POETX_ERR_DTYPE;
  }
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(g) |
       reinterpret_cast<uintptr_t>(g_lp)) & 15) {
    set_error("cnp_build_noalloc: pointers must be 16-byte aligned");
    return POETX_ERR_ALIGN;
  }
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    set_error("cnp_build_noalloc: no CUDA device");
    return POETX_ERR_CUDA;
  }
  if (major != 10) {
    set_error("cnp_build_noalloc: device %d is not sm_100", dev);
    return POETX_ERR_UNSUPPORTED;
  }
  // per-device set-up (first call on the device): the scratch buffer's device address. Under
  // lazy module loading this is where the module that holds the buffer gets loaded.
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    set_error("cnp_build_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    return POETX_ERR_CUDA;
  }
  if (nblocks == 0) return POETX_OK;   // set-up only
  // largest chunk of blocks whose scratch fits the buffer
  int64_t chunk = (int64_t)(POETX_CNP_NOALLOC_SCRATCH_BYTES / per_block);
  while (chunk > 1 && gemm_cnp_ws_bytes(chunk, b) > (size_t)POETX_CNP_NOALLOC_SCRATCH_BYTES) --chunk;
  const int64_t qs = b * (b - 1) / 2, bb = b * b;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int64_t j0 = 0; j0 < nblocks; j0 += chunk) {
    const int64_t nb = std::min(chunk, nblocks - j0);
    e = gemm_cnp_build(q + j0 * qs, nb, b, g ? g + j0 * bb : nullptr,
                       g_lp ? static_cast<__nv_bfloat16*>(g_lp) + j0 * bb : nullptr, scratch, s);
    if (e != cudaSuccess) {
      set_error("cnp_build_noalloc: %s", cudaGetErrorString(e));
      return POETX_ERR_CUDA;
    }
  }
  return POETX_OK;
}
