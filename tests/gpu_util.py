"""Shared set-up for the GPU parity tests: seeded inputs from poetx_workloads go both to the
library (through the C ABI binding) and, upcast to float64, to the oracle."""
from __future__ import annotations

import numpy as np
import torch

import poetx_workloads as W

try:
    from orthogonal_equivalence_build_b200 import poetx
except ImportError:  # pragma: no cover - reported by the tests that need it
    poetx = None

TOL_BF16 = 1e-2   # max|gpu - oracle| / max|oracle| for the bf16 path (y, dx, dq)
TOL_F32 = 1e-5    # fp32 CNP build and the fp32 layer


def rel_err(gpu, ref) -> float:
    g = gpu.detach().double().cpu().numpy() if torch.is_tensor(gpu) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300))


def torch_dtype(wl: W.Workload) -> torch.dtype:
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


class LayerCase:
    """One seeded linear on the device plus the host copies the oracle consumes."""

    def __init__(self, key: str, layer: int = 0, *, m=None, n=None, b=None, tokens=None,
                 seed=None, q_zero=False, w0=None, q_scale=1.0):
        wl = W.WORKLOADS[key]
        self.wl = wl
        p = W.layer_params(wl, layer, m=m, n=n, b=b, seed=seed)
        a = W.layer_acts(wl, layer, tokens=tokens, m=m, n=n, seed=seed)
        if w0 is not None:
            p["W0"] = np.asarray(w0, dtype=np.float32)
        if q_zero:
            p["q_r"][:] = 0
            p["q_p"][:] = 0
        elif q_scale != 1.0:
            p["q_r"] *= np.float32(q_scale)
            p["q_p"] *= np.float32(q_scale)
        self.b = wl.b if b is None else b
        self.p, self.a = p, a
        dt = torch_dtype(wl)
        self.dt = dt
        dev = "cuda"
        self.w0 = torch.from_numpy(p["W0"]).to(dt).to(dev)
        self.perm_r = torch.from_numpy(p["perm_r"]).to(dev)
        self.perm_p = torch.from_numpy(p["perm_p"]).to(dev)
        self.q_r = torch.from_numpy(p["q_r"]).to(dev)
        self.q_p = torch.from_numpy(p["q_p"]).to(dev)
        self.x = torch.from_numpy(a["X"]).to(dt).to(dev)
        self.dy = torch.from_numpy(a["dY"]).to(dt).to(dev)
        w0m = torch.empty_like(self.w0)
        poetx.merge_permutations(self.w0, self.perm_r, self.perm_p, w0m)
        self.layer = poetx.PoetxLinear(w0m, self.perm_r, self.perm_p, self.q_r, self.q_p, self.b)
        poetx.layer_cnp_build(self.layer)
        self.T = self.x.shape[0]

    def host(self):
        """Inputs as the oracle sees them (float64 upcasts of the stored values)."""
        d = {k: np.asarray(v) for k, v in self.p.items()}
        d.update({k: np.asarray(v) for k, v in self.a.items()})
        d["W0m"] = d["W0"][d["perm_r"]][:, d["perm_p"]]
        return d

    def forward(self):
        y = torch.empty(self.T, self.layer.n, dtype=self.dt, device="cuda")
        bsave = torch.empty(self.T, self.layer.n, dtype=self.dt, device="cuda")
        poetx.linear_fwd(self.layer, self.x, y, bsave)
        return y, bsave

    def backward(self, bsave, dy=None):
        dy = self.dy if dy is None else dy
        dx = torch.empty(self.T, self.layer.m, dtype=self.dt, device="cuda")
        dq_r = torch.empty_like(self.q_r)
        dq_p = torch.empty_like(self.q_p)
        poetx.linear_bwd(self.layer, self.x, dy, bsave, dx, dq_r, dq_p)
        return dx, dq_r, dq_p
