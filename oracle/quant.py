"""Float CPU oracle of the 8-bit weight storage of POET-XQ.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
the CPU-baseline / reference legs of the benchmark may import or run this
file.  The CUDA library never calls it and shares no code with it.

Sources (web pages on POET / POET-X):
  [P3]  "[Project POET-X] Scaling Orthogonal Equivalence: Training 13B LLMs
        with LoRA-level Memory Efficiency", §Quantized Training (POET-XQ):
        custom kernels dequantise on the fly; 8-bit quantised pretraining.
  [P5]  "POET-X: Memory-efficient LLM Training by Scaling Orthogonal
        Transformation" (gist.science), §Resumo técnico 2 Metodologia, item
        on POET-XQ: only the low-precision weights are stored, dequantised on
        demand; §4 Resultados Experimentais (8-bit training).

The pages fix neither the 8-bit format nor its granularity.  Reading used
here (and by the library): symmetric int8 codes with one fp32 scale per
column of the merged weight W0' [m, n] (one per output feature of the layer):
    s_j  = max_i |W0'[i, j]| / 127             (fp32 division)
    q_ij = round_half_even(W0'[i, j] / s_j)    (fp32 division), |q_ij| <= 127
    s_j  = 0 and q_.j = 0 for an all-zero column.
The layer then computes with the dequantised weight
    W_deq[i, j] = bf16(fp32(q_ij) * s_j)        (fp32 product, rounded to
                                                nearest-even bfloat16),
i.e. exactly the bf16 layer of the oracle with W0' replaced by W_deq.

The quantisation decision (the integer code) is taken in fp32, the
precision the kernels take it in, so codes compare bit for bit when both
sides start from the same stored W0'.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

QMAX = 127


def _bf16_round(x32: np.ndarray) -> np.ndarray:
    """fp32 -> nearest-even bfloat16, returned as float32 (finite inputs)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def quantize_w0_int8(W0m: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """W0' [m, n] (any float dtype; taken as fp32) -> (codes int8 [m, n], scales fp32 [n])."""
    w = np.asarray(W0m, dtype=np.float32)
    amax = np.max(np.abs(w), axis=0) if w.shape[0] else np.zeros(w.shape[1], np.float32)
    scale = (amax / np.float32(QMAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    ratio = (w / safe[None, :]).astype(np.float32)
    q = np.clip(np.rint(ratio), -QMAX, QMAX)
    q = np.where(scale[None, :] > 0, q, 0.0)
    return q.astype(np.int8), scale


def dequantize_w0_int8(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """codes [m, n], scales [n] -> W_deq [m, n] as float64 holding bfloat16 values."""
    prod = (np.asarray(q, dtype=np.float32) *
            np.asarray(scale, dtype=np.float32)[None, :]).astype(np.float32)
    return _bf16_round(prod).astype(np.float64)


def requantize_after_merge(W0m_new: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Merge-then-reinitialize of an 8-bit layer stores the new W0' in 8 bits again
    ("Reparameterized LLM Training ..." §3 gives the merge; [P5] keeps only the
    low-precision weights)."""
    return quantize_w0_int8(W0m_new)
