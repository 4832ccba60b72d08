"""Seeded synthetic workloads for the POET-X linear layer.

This module only draws random numbers and rounds them to the storage type.
It holds none of the layer's arithmetic, so both the float64 oracle and the
CUDA library can be fed from it without sharing any of the method's code.

Shapes and distributions follow the Llama-shaped layers the POET-X pages
train ("POET-X: Memory-efficient LLM Training by Scaling Orthogonal
Transformation", Resumo tecnico §4 Resultados Experimentais: Llama 3B/8B/13B
on C4, b = 512).  The C4 text and trained weights are not used: every tensor
is synthetic.  Initialisation follows "Reparameterized LLM Training via
Orthogonal Equivalence Transformation", §4 初始化方案 (normalised Gaussian).

Recipe for one linear (m = in-features, n = out-features, block size b):
  W0      [m, n]      each length-n row ~ N(0, I), scaled to unit l2 norm
  q_r     [m/b, b(b-1)/2]  N(0, sigma_q^2), float32 (packed strict upper triangle)
  q_p     [n/b, b(b-1)/2]  N(0, sigma_q^2), float32
  perm_r  [m]         uniform random permutation (int32)
  perm_p  [n]         uniform random permutation (int32)
  X       [T, m]      N(0, 1)
  dY      [T, n]      N(0, 1)
Every tensor t of layer l in workload s comes from
numpy.random.default_rng(SeedSequence([s, l, t])).  For bfloat16 workloads
W0, X and dY are rounded once, on the host, to bfloat16 with
round-to-nearest-even; the identical bits go to the GPU and (upcast) to the
oracle.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

# tensor ids inside one layer's SeedSequence
T_W0, T_QR, T_QP, T_PR, T_PP, T_X, T_DY = range(7)
T_QPERT = 100  # per-step perturbation of q (13B layer-set run)


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    m: int  # in-features  (rows of W0)
    n: int  # out-features (cols of W0)


@dataclasses.dataclass(frozen=True)
class Workload:
    key: str
    description: str
    dtype: str  # "f32" or "bf16": storage/compute type of activations and W0
    b: int
    tokens: int
    sigma_q: float
    linears: Tuple[Linear, ...]
    cnp_in_step: bool = True
    merge_every: int = 0  # merge_reinit period in steps (0: not part of the run)
    q_step_sigma: float = 0.0  # per-step N(0, s^2) perturbation of q
    steps: int = 1

    def layer(self, i: int = 0) -> Linear:
        return self.linears[i]


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload(
        key="tiny_fp32",
        description="single 512x512 linear, fp32, b=64, 256 tokens, fwd+bwd+merge_reinit",
        dtype="f32", b=64, tokens=256, sigma_q=0.01,
        linears=(Linear("w", 512, 512),), merge_every=1),
    "llama1p3b_attn": Workload(
        key="llama1p3b_attn",
        description="Llama-1.3B attention projection 2048x2048, bf16, b=256, 8192 tokens",
        dtype="bf16", b=256, tokens=8192, sigma_q=0.005,
        linears=(Linear("attn", 2048, 2048),), cnp_in_step=False),
    "llama8b_up_proj": Workload(
        key="llama8b_up_proj",
        description="Llama-8B FFN up_proj 4096x14336, bf16, b=512, 16384 tokens, CNP+fwd+bwd",
        dtype="bf16", b=512, tokens=16384, sigma_q=0.005,
        linears=(Linear("up_proj", 4096, 14336),)),
    "llama8b_decoder": Workload(
        key="llama8b_decoder",
        description="Llama-8B decoder layer (q,k,v,o,gate,up,down), bf16, b=512, 8192 tokens",
        dtype="bf16", b=512, tokens=8192, sigma_q=0.005,
        linears=(Linear("q", 4096, 4096), Linear("k", 4096, 1024),
                 Linear("v", 4096, 1024), Linear("o", 4096, 4096),
                 Linear("gate", 4096, 14336), Linear("up", 4096, 14336),
                 Linear("down", 14336, 4096))),
    "llama13b_layers": Workload(
        key="llama13b_layers",
        description="Llama-13B layer set, bf16, b=512, 8192 tokens, 400 steps, merge_reinit at 400",
        dtype="bf16", b=512, tokens=8192, sigma_q=0.005,
        linears=(Linear("q", 5120, 5120), Linear("k", 5120, 5120),
                 Linear("v", 5120, 5120), Linear("o", 5120, 5120),
                 Linear("gate", 5120, 13824), Linear("up", 5120, 13824),
                 Linear("down", 13824, 5120)),
        merge_every=400, q_step_sigma=1e-4, steps=400),
}

# the workload index used as the base seed of each workload
WORKLOAD_SEED = {"tiny_fp32": 1, "llama1p3b_attn": 2, "llama8b_up_proj": 3,
                 "llama8b_decoder": 4, "llama13b_layers": 5}


def rng_for(seed: int, layer: int, tensor: int, extra: int = 0) -> np.random.Generator:
    words = [int(seed), int(layer), int(tensor)]
    if extra:
        words.append(int(extra))
    return np.random.default_rng(np.random.SeedSequence(words))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 value (ties to even), returned as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
         & np.uint32(0xFFFF0000))
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 values that are exactly bfloat16 -> their uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32, copy=False)
    return round_bf16(a) if dtype == "bf16" else a


def gen_w0(m: int, n: int, rng: np.random.Generator, dtype: str) -> np.ndarray:
    w = rng.standard_normal((m, n), dtype=np.float32)
    norms = np.sqrt(np.einsum("ij,ij->i", w.astype(np.float64), w.astype(np.float64)))
    w = (w / norms[:, None].astype(np.float32)).astype(np.float32)
    return _store(w, dtype)


def gen_q(nblocks: int, b: int, sigma: float, rng: np.random.Generator) -> np.ndarray:
    return (rng.standard_normal((nblocks, b * (b - 1) // 2), dtype=np.float32)
            * np.float32(sigma)).astype(np.float32)


def gen_perm(n: int, rng: np.random.Generator) -> np.ndarray:
    return rng.permutation(n).astype(np.int32)


def gen_act(rows: int, cols: int, rng: np.random.Generator, dtype: str) -> np.ndarray:
    return _store(rng.standard_normal((rows, cols), dtype=np.float32), dtype)


def layer_params(wl: Workload, layer: int = 0, *, m: Optional[int] = None,
                 n: Optional[int] = None, b: Optional[int] = None,
                 seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """W0, q_r, q_p, perm_r, perm_p of one linear (shape overrides for tests)."""
    lin = wl.linears[layer]
    m = lin.m if m is None else m
    n = lin.n if n is None else n
    b = wl.b if b is None else b
    s = WORKLOAD_SEED[wl.key] if seed is None else seed
    return {
        "W0": gen_w0(m, n, rng_for(s, layer, T_W0), wl.dtype),
        "q_r": gen_q(m // b, b, wl.sigma_q, rng_for(s, layer, T_QR)),
        "q_p": gen_q(n // b, b, wl.sigma_q, rng_for(s, layer, T_QP)),
        "perm_r": gen_perm(m, rng_for(s, layer, T_PR)),
        "perm_p": gen_perm(n, rng_for(s, layer, T_PP)),
    }


def layer_acts(wl: Workload, layer: int = 0, *, tokens: Optional[int] = None,
               m: Optional[int] = None, n: Optional[int] = None,
               seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """X [T, m] and dY [T, n] of one linear."""
    lin = wl.linears[layer]
    m = lin.m if m is None else m
    n = lin.n if n is None else n
    T = wl.tokens if tokens is None else tokens
    s = WORKLOAD_SEED[wl.key] if seed is None else seed
    return {"X": gen_act(T, m, rng_for(s, layer, T_X), wl.dtype),
            "dY": gen_act(T, n, rng_for(s, layer, T_DY), wl.dtype)}


def q_perturbation(wl: Workload, layer: int, step: int, side: int,
                   shape: Tuple[int, int]) -> np.ndarray:
    """Per-step N(0, q_step_sigma^2) increment of q (side 0 = R, 1 = P)."""
    s = WORKLOAD_SEED[wl.key]
    rng = rng_for(s, layer, T_QPERT + side, extra=step + 1)
    return (rng.standard_normal(shape, dtype=np.float32)
            * np.float32(wl.q_step_sigma)).astype(np.float32)


def list_workloads() -> List[str]:
    return list(WORKLOADS)
