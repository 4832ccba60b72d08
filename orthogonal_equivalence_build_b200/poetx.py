"""Thin Python binding of libpoetx (include/poetx.h), one function per C entry point.

Argument marshalling only: tensors become device pointers, the current torch
CUDA stream is passed as the stream, workspaces are caller-owned torch
buffers sized by the library's own queries.  Every step of the layer runs in
the library's CUDA kernels; there is no other code path.  If the shared
library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libpoetx.so")

F32, BF16 = 0, 1
_STATUS = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "ALIGN", 4: "DTYPE", 5: "BAD_INDEX",
           6: "CUDA", 7: "UNSUPPORTED", 8: "WORKSPACE", 9: "TIMEOUT"}


class PoetxError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"poetx status {status} ({_STATUS.get(status, '?')}): {message}")
        self.status = status


class Layer(ctypes.Structure):
    """Mirror of poetx_layer."""
    _fields_ = [("m", ctypes.c_int64), ("n", ctypes.c_int64), ("b", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("w0m", ctypes.c_void_p), ("perm_r", ctypes.c_void_p),
                ("perm_p", ctypes.c_void_p), ("q_r", ctypes.c_void_p), ("q_p", ctypes.c_void_p),
                ("g_r", ctypes.c_void_p), ("g_p", ctypes.c_void_p),
                ("g_r_lp", ctypes.c_void_p), ("g_p_lp", ctypes.c_void_p),
                ("w0m_scale", ctypes.c_void_p)]


LAYER_W0M_I8 = 1
LAYER_W0M_STAGED = 2
LAYER_FUSED_W0_P = 4


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m orthogonal_equivalence_build_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    V, I32, I64, U64, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                            ctypes.c_size_t)
    LP = ctypes.POINTER(Layer)
    sig = {
        "poetx_cnp_workspace_bytes": (SZ, [I64, I64]),
        "poetx_cnp_build": (I32, [V, I64, I64, V, V, I32, V, SZ, V]),
        "poetx_cnp_build_noalloc": (I32, [V, I64, I64, V, V, I32, V]),
        "poetx_layer_cnp_workspace_bytes": (SZ, [LP]),
        "poetx_layer_cnp_build": (I32, [LP, V, SZ, V]),
        "poetx_layers_cnp_workspace_bytes": (SZ, [ctypes.POINTER(LP), I32]),
        "poetx_layers_cnp_build": (I32, [ctypes.POINTER(LP), I32, V, SZ, V]),
        "poetx_linear_bwd_dg": (I32, [LP, V, V, V, V, I64, V, V, V, SZ, V]),
        "poetx_layers_dq_workspace_bytes": (SZ, [ctypes.POINTER(LP), I32]),
        "poetx_layers_dq_from_dg": (I32, [ctypes.POINTER(LP), ctypes.POINTER(V),
                                          ctypes.POINTER(V), ctypes.POINTER(V), I32, V, SZ, V]),
        "poetx_fwd_workspace_bytes": (SZ, [LP, I64]),
        "poetx_linear_fwd": (I32, [LP, V, I64, V, V, V, SZ, V]),
        "poetx_bwd_workspace_bytes": (SZ, [LP, I64]),
        "poetx_linear_bwd": (I32, [LP, V, V, V, I64, V, V, V, V, SZ, V]),
        "poetx_linear_fwd_ex": (I32, [LP, V, I64, V, V, V, V, SZ, V]),
        "poetx_linear_bwd_ex": (I32, [LP, V, V, V, V, I64, V, V, V, V, SZ, V]),
        "poetx_merge_permutations": (I32, [V, V, V, I64, I64, I32, V, V]),
        "poetx_merge_reinit_workspace_bytes": (SZ, [LP]),
        "poetx_merge_reinit": (I32, [LP, U64, V, SZ, V]),
        "poetx_quantize_w0": (I32, [V, I64, I64, I32, V, V, V]),
        "poetx_dequantize_w0": (I32, [V, V, I64, I64, V, V]),
        "poetx_resample_permutation": (I32, [U64, I32, I64, V, V]),
        "poetx_validate_permutation": (I32, [V, I64, V, SZ, V]),
        "poetx_device_status": (I32, [V]),
        "poetx_trace_enable": (I32, [I32]),
        "poetx_trace_read": (I64, [ctypes.c_char_p, SZ]),
        "poetx_trace_select": (I32, [ctypes.c_char_p]),
        "poetx_status_string": (ctypes.c_char_p, [I32]),
        "poetx_last_error_message": (ctypes.c_char_p, []),
        "poetx_abi_version": (I32, []),
        "poetx_testing_gemm_bf16": (I32, [V, I64, I64, I32, V, I64, I64, I32, I64, I64, I64, V,
                                          I32, I64, I32, I32, U64, V]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
EXPORTED = (
    "poetx_cnp_workspace_bytes", "poetx_cnp_build", "poetx_cnp_build_noalloc",
    "poetx_layer_cnp_workspace_bytes", "poetx_layer_cnp_build",
    "poetx_layers_cnp_workspace_bytes", "poetx_layers_cnp_build",
    "poetx_linear_bwd_dg", "poetx_layers_dq_workspace_bytes", "poetx_layers_dq_from_dg",
    "poetx_fwd_workspace_bytes",
    "poetx_linear_fwd", "poetx_bwd_workspace_bytes", "poetx_linear_bwd",
    "poetx_linear_fwd_ex", "poetx_linear_bwd_ex",
    "poetx_merge_permutations", "poetx_merge_reinit_workspace_bytes", "poetx_merge_reinit",
    "poetx_quantize_w0", "poetx_dequantize_w0", "poetx_resample_permutation", "poetx_validate_permutation", "poetx_device_status",
    "poetx_trace_enable", "poetx_trace_read", "poetx_trace_select", "poetx_status_string",
    "poetx_last_error_message", "poetx_abi_version", "poetx_testing_gemm_bf16")


def _check(status: int) -> None:
    if status != 0:
        raise PoetxError(status, lib.poetx_last_error_message().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to poetx must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return workspace
    if workspace is not None and workspace.numel() * workspace.element_size() >= nbytes:
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise ValueError(f"unsupported dtype {t}")


# ----------------------------------------------------------------------------- layer state
class PoetxLinear:
    """Device state of one POET-X linear (caller-owned torch tensors) plus its C descriptor.

    w0m [m, n] (dtype), perm_r [m], perm_p [n] (int32), q_r [m/b, b(b-1)/2], q_p (fp32),
    g_r [m/b, b, b], g_p (fp32) and, for bf16 layers, g_r_lp / g_p_lp (bf16).
    An int8 w0m with its fp32 column scales w0m_scale [n] makes an 8-bit-weight layer
    (POETX_LAYER_W0M_I8; activations and gradients bf16). fused_w0_p sets
    POETX_LAYER_FUSED_W0_P (the forward's W0' and P-block products as one kernel).
    """

    def __init__(self, w0m: torch.Tensor, perm_r: torch.Tensor, perm_p: torch.Tensor,
                 q_r: torch.Tensor, q_p: torch.Tensor, b: int,
                 w0m_scale: Optional[torch.Tensor] = None, staged: bool = False,
                 fused_w0_p: bool = False):
        m, n = w0m.shape
        dev = w0m.device
        self.b = int(b)
        self.w0m, self.perm_r, self.perm_p = w0m, perm_r, perm_p
        self.w0m_scale = w0m_scale
        self.q_r, self.q_p = q_r, q_p
        self.g_r = torch.empty(m // b, b, b, dtype=torch.float32, device=dev)
        self.g_p = torch.empty(n // b, b, b, dtype=torch.float32, device=dev)
        i8 = w0m.dtype == torch.int8
        if i8 and w0m_scale is None:
            raise ValueError("an int8 w0m needs w0m_scale")
        lp = i8 or w0m.dtype == torch.bfloat16
        self.g_r_lp = torch.empty(m // b, b, b, dtype=torch.bfloat16, device=dev) if lp else None
        self.g_p_lp = torch.empty(n // b, b, b, dtype=torch.bfloat16, device=dev) if lp else None
        self.desc = Layer(m=m, n=n, b=self.b, dtype=BF16 if i8 else dtype_code(w0m.dtype),
                          flags=(((LAYER_W0M_I8 | (LAYER_W0M_STAGED if staged else 0)) if i8
                                  else 0) | (LAYER_FUSED_W0_P if fused_w0_p else 0)),
                          w0m=_ptr(w0m), perm_r=_ptr(perm_r), perm_p=_ptr(perm_p),
                          q_r=_ptr(q_r), q_p=_ptr(q_p), g_r=_ptr(self.g_r), g_p=_ptr(self.g_p),
                          g_r_lp=_ptr(self.g_r_lp), g_p_lp=_ptr(self.g_p_lp),
                          w0m_scale=_ptr(w0m_scale) if i8 else None)

    @property
    def m(self) -> int:
        return int(self.desc.m)

    @property
    def n(self) -> int:
        return int(self.desc.n)

    @property
    def dtype(self) -> torch.dtype:
        """Activation / gradient dtype (bf16 for 8-bit-weight layers)."""
        return torch.bfloat16 if self.w0m.dtype == torch.int8 else self.w0m.dtype


# ----------------------------------------------------------------------------- entry points
def cnp_workspace_bytes(nblocks: int, b: int) -> int:
    return int(lib.poetx_cnp_workspace_bytes(nblocks, b))


def cnp_build(q: torch.Tensor, b: int, g: Optional[torch.Tensor] = None,
              g_lp: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
              stream=None) -> None:
    nb = q.shape[0]
    ws = _workspace(cnp_workspace_bytes(nb, b), q.device, workspace)
    _check(lib.poetx_cnp_build(_ptr(q), nb, b, _ptr(g), _ptr(g_lp), BF16, _ptr(ws),
                               0 if ws is None else ws.numel(), _stream(stream)))


def cnp_build_noalloc(q: torch.Tensor, b: int, g: Optional[torch.Tensor] = None,
                      g_lp: Optional[torch.Tensor] = None, stream=None) -> None:
    """poetx_cnp_build without a workspace (fixed library-owned scratch; see include/poetx.h)."""
    _check(lib.poetx_cnp_build_noalloc(_ptr(q), q.shape[0], b, _ptr(g), _ptr(g_lp), BF16,
                                       _stream(stream)))


def layer_cnp_workspace_bytes(layer: PoetxLinear) -> int:
    return int(lib.poetx_layer_cnp_workspace_bytes(ctypes.byref(layer.desc)))


def layer_cnp_build(layer: PoetxLinear, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> None:
    """CNP blocks of both sides of the layer (poetx_layer_cnp_build)."""
    ws = _workspace(layer_cnp_workspace_bytes(layer), layer.w0m.device, workspace)
    _check(lib.poetx_layer_cnp_build(ctypes.byref(layer.desc), _ptr(ws),
                                     0 if ws is None else ws.numel(), _stream(stream)))


def _layer_array(layers):
    arr = (ctypes.POINTER(Layer) * len(layers))()
    for i, layer in enumerate(layers):
        arr[i] = ctypes.pointer(layer.desc)
    return arr


def layers_cnp_workspace_bytes(layers) -> int:
    arr = _layer_array(layers)
    return int(lib.poetx_layers_cnp_workspace_bytes(arr, len(layers)))


def layers_cnp_build(layers, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """CNP blocks of every layer in `layers` (PoetxLinear, same b and dtype) in one call
    (poetx_layers_cnp_build)."""
    if not layers:
        return
    arr = _layer_array(layers)
    ws = _workspace(int(lib.poetx_layers_cnp_workspace_bytes(arr, len(layers))),
                    layers[0].w0m.device, workspace)
    _check(lib.poetx_layers_cnp_build(arr, len(layers), _ptr(ws), 0 if ws is None else ws.numel(),
                                      _stream(stream)))


def fwd_workspace_bytes(layer: PoetxLinear, T: int) -> int:
    return int(lib.poetx_fwd_workspace_bytes(ctypes.byref(layer.desc), T))


def linear_fwd(layer: PoetxLinear, x: torch.Tensor, y: torch.Tensor,
               saved_b: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None, saved_a: Optional[torch.Tensor] = None) -> None:
    """poetx_linear_fwd; with saved_a [T, m] the forward also keeps A = X[:, perm_r] there
    (poetx_linear_fwd_ex)."""
    T = x.shape[0]
    ws = _workspace(fwd_workspace_bytes(layer, T), x.device, workspace)
    args = (ctypes.byref(layer.desc), _ptr(x), T, _ptr(y), _ptr(saved_b))
    tail = (_ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    if saved_a is None:
        _check(lib.poetx_linear_fwd(*args, *tail))
    else:
        _check(lib.poetx_linear_fwd_ex(*args, _ptr(saved_a), *tail))


def bwd_workspace_bytes(layer: PoetxLinear, T: int) -> int:
    return int(lib.poetx_bwd_workspace_bytes(ctypes.byref(layer.desc), T))


def linear_bwd(layer: PoetxLinear, x: torch.Tensor, dy: torch.Tensor, saved_b: torch.Tensor,
               dx: Optional[torch.Tensor], dq_r: Optional[torch.Tensor],
               dq_p: Optional[torch.Tensor], workspace: Optional[torch.Tensor] = None,
               stream=None, saved_a: Optional[torch.Tensor] = None) -> None:
    """poetx_linear_bwd; with saved_a (the forward's A) the backward reads A from it instead of
    gathering X again (poetx_linear_bwd_ex)."""
    T = dy.shape[0]
    ws = _workspace(bwd_workspace_bytes(layer, T), dy.device, workspace)
    tail = (T, _ptr(dx), _ptr(dq_r), _ptr(dq_p), _ptr(ws), 0 if ws is None else ws.numel(),
            _stream(stream))
    if saved_a is None:
        _check(lib.poetx_linear_bwd(ctypes.byref(layer.desc), _ptr(x), _ptr(dy), _ptr(saved_b),
                                    *tail))
    else:
        _check(lib.poetx_linear_bwd_ex(ctypes.byref(layer.desc), _ptr(x), _ptr(dy),
                                       _ptr(saved_b), _ptr(saved_a), *tail))


def linear_bwd_dg(layer: PoetxLinear, x: Optional[torch.Tensor], dy: torch.Tensor,
                  saved_b: Optional[torch.Tensor], dx: Optional[torch.Tensor],
                  dG: torch.Tensor, workspace: Optional[torch.Tensor] = None, stream=None,
                  saved_a: Optional[torch.Tensor] = None) -> None:
    """The backward up to the per-block gradients: dG [m/b + n/b, b, b] fp32 (R blocks, then P
    blocks); no dq (poetx_linear_bwd_dg)."""
    T = dy.shape[0]
    ws = _workspace(bwd_workspace_bytes(layer, T), dy.device, workspace)
    _check(lib.poetx_linear_bwd_dg(ctypes.byref(layer.desc), _ptr(x), _ptr(dy), _ptr(saved_b),
                                   _ptr(saved_a), T, _ptr(dx), _ptr(dG), _ptr(ws),
                                   0 if ws is None else ws.numel(), _stream(stream)))


def layers_dq_workspace_bytes(layers) -> int:
    return int(lib.poetx_layers_dq_workspace_bytes(_layer_array(layers), len(layers)))


def layers_dq_from_dg(layers, dGs, dq_rs, dq_ps, workspace: Optional[torch.Tensor] = None,
                      stream=None) -> None:
    """dq of every layer from its dG in one launch sequence (poetx_layers_dq_from_dg)."""
    if not layers:
        return
    n = len(layers)
    arr = _layer_array(layers)
    ptrs = lambda ts: (ctypes.c_void_p * n)(*[_ptr(t) for t in ts])
    ws = _workspace(int(lib.poetx_layers_dq_workspace_bytes(arr, n)), layers[0].w0m.device,
                    workspace)
    _check(lib.poetx_layers_dq_from_dg(arr, ptrs(dGs), ptrs(dq_rs), ptrs(dq_ps), n, _ptr(ws),
                                       0 if ws is None else ws.numel(), _stream(stream)))


def merge_permutations(w0: torch.Tensor, perm_r: torch.Tensor, perm_p: torch.Tensor,
                       w0m: torch.Tensor, stream=None) -> None:
    m, n = w0.shape
    _check(lib.poetx_merge_permutations(_ptr(w0), _ptr(perm_r), _ptr(perm_p), m, n,
                                        dtype_code(w0.dtype), _ptr(w0m), _stream(stream)))


def merge_reinit_workspace_bytes(layer: PoetxLinear) -> int:
    return int(lib.poetx_merge_reinit_workspace_bytes(ctypes.byref(layer.desc)))


def merge_reinit(layer: PoetxLinear, seed: int, workspace: Optional[torch.Tensor] = None,
                 stream=None) -> None:
    ws = _workspace(merge_reinit_workspace_bytes(layer), layer.w0m.device, workspace)
    _check(lib.poetx_merge_reinit(ctypes.byref(layer.desc), seed & ((1 << 64) - 1), _ptr(ws),
                                  0 if ws is None else ws.numel(), _stream(stream)))


def quantize_w0(w: torch.Tensor, wq: torch.Tensor, scale: torch.Tensor, stream=None) -> None:
    """wq [m, n] int8, scale [n] fp32 <- per-column symmetric 8-bit codes of w (poetx_quantize_w0)."""
    m, n = w.shape
    _check(lib.poetx_quantize_w0(_ptr(w), m, n, dtype_code(w.dtype), _ptr(wq), _ptr(scale),
                                 _stream(stream)))


def dequantize_w0(wq: torch.Tensor, scale: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """out [m, n] bf16 <- bf16(wq * scale[col]) (poetx_dequantize_w0)."""
    m, n = wq.shape
    _check(lib.poetx_dequantize_w0(_ptr(wq), _ptr(scale), m, n, _ptr(out), _stream(stream)))


def resample_permutation(seed: int, lane: int, perm: torch.Tensor, stream=None) -> None:
    _check(lib.poetx_resample_permutation(seed & ((1 << 64) - 1), lane, perm.numel(), _ptr(perm),
                                          _stream(stream)))


def validate_permutation(perm: torch.Tensor, stream=None) -> bool:
    k = perm.numel()
    ws = torch.empty(4 * (k + 1), dtype=torch.uint8, device=perm.device)
    st = lib.poetx_validate_permutation(_ptr(perm), k, _ptr(ws), ws.numel(), _stream(stream))
    if st == 5:
        return False
    _check(st)
    return True


def device_status(stream=None) -> None:
    _check(lib.poetx_device_status(_stream(stream)))


def trace_enable(on: bool = True) -> None:
    _check(lib.poetx_trace_enable(1 if on else 0))


def trace_select(names=None) -> None:
    """Record only the launches named in `names` (iterable of str); None records all."""
    _check(lib.poetx_trace_select(None if not names else ",".join(names).encode()))


def trace_read(maxlen: int = 1 << 20):
    buf = ctypes.create_string_buffer(maxlen)
    lib.poetx_trace_read(buf, maxlen)
    out = []
    for line in buf.value.decode().splitlines():
        name, ms = line.rsplit(" ", 1)
        out.append((name, float(ms)))
    return out


def testing_gemm_bf16(a: torch.Tensor, a_mn: bool, b: torch.Tensor, b_mn: bool, M: int, N: int,
                      K: int, c: torch.Tensor, splits: int = 1, variant: int = 0,
                      epi_wait_ns: int = 0, stream=None) -> None:
    """Kernel-level hook (include/poetx_testing.h): C = A B on the tcgen05 kernel
    (variant 0: single CTA, 1: CTA pair, 2 / 3: 256 x 512 pair tiles with / without the
    collector buffer); epi_wait_ns > 0 bounds the epilogue's accumulator wait (a test of the
    timeout path)."""
    _check(lib.poetx_testing_gemm_bf16(_ptr(a), a.shape[0], a.shape[1], int(a_mn), _ptr(b),
                                       b.shape[0], b.shape[1], int(b_mn), M, N, K, _ptr(c),
                                       int(c.dtype == torch.float32), c.shape[-1], splits,
                                       variant, int(epi_wait_ns), _stream(stream)))


def abi_version() -> int:
    return int(lib.poetx_abi_version())
