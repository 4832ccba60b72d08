"""GPU parity of 8-bit W0' layers (POET-XQ storage: int8 codes with one fp32 scale per column).

- The quantiser and dequantiser agree with the oracle bit for bit (the codes are decided in fp32
  on both sides from the same stored bf16 W0').
- An 8-bit layer is the bf16 layer whose W0' is bf16(code * scale): forward and backward outputs
  are bitwise equal to that layer's, both where the tensor-core kernel dequantises in shared
  memory (T >= 256, m and n multiples of 256) and where the library dequantises into its
  workspace first.
- Against the oracle (float64, W0' = the dequantised weight): y, dx, dq within 1e-2, at small
  sizes with ragged token counts and on sampled rows at the full Llama-8B up_proj size.
- Merge-then-reinitialize of an 8-bit layer: permutations bit-exact, q = 0, the new dequantised
  W0' and the layer output within 1e-2."""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.quant as OQ
from tests.gpu_util import TOL_BF16, LayerCase, poetx, rel_err

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _quantize(w: torch.Tensor):
    m, n = w.shape
    wq = torch.empty(m, n, dtype=torch.int8, device="cuda")
    scale = torch.empty(n, dtype=torch.float32, device="cuda")
    poetx.quantize_w0(w, wq, scale)
    return wq, scale


def _dequantize(wq, scale):
    out = torch.empty(wq.shape, dtype=torch.bfloat16, device="cuda")
    poetx.dequantize_w0(wq, scale, out)
    return out


class XqCase:
    """A LayerCase's bf16 layer, its 8-bit twin (codes of the same merged W0') and the bf16
    layer built on the dequantised W0'."""

    def __init__(self, key, **kw):
        self.c = LayerCase(key, **kw)
        c = self.c
        self.wq, self.scale = _quantize(c.layer.w0m)
        self.xq = poetx.PoetxLinear(self.wq, c.perm_r, c.perm_p, c.q_r, c.q_p, c.b,
                                    w0m_scale=self.scale)
        poetx.layer_cnp_build(self.xq)
        self.deq = poetx.PoetxLinear(_dequantize(self.wq, self.scale), c.perm_r, c.perm_p,
                                     c.q_r, c.q_p, c.b)
        poetx.layer_cnp_build(self.deq)

    def run(self, layer, dy=None, saved=True):
        c = self.c
        T, m, n = c.T, c.layer.m, c.layer.n
        y = torch.empty(T, n, dtype=torch.bfloat16, device="cuda")
        bs = torch.empty(T, n, dtype=torch.bfloat16, device="cuda")
        poetx.linear_fwd(layer, c.x, y, bs)
        dx = torch.empty(T, m, dtype=torch.bfloat16, device="cuda")
        dq_r, dq_p = torch.empty_like(c.q_r), torch.empty_like(c.q_p)
        poetx.linear_bwd(layer, c.x, c.dy if dy is None else dy, bs if saved else None, dx,
                         dq_r, dq_p)
        return y, bs, dx, dq_r, dq_p

    def host_w0m_deq(self):
        h = self.c.host()
        q, s = OQ.quantize_w0_int8(h["W0m"])
        return h, q, s, OQ.dequantize_w0_int8(q, s)


# ------------------------------------------------------------------ quantiser
@pytest.mark.parametrize("m,n,dt", [(512, 768, torch.bfloat16), (1000, 48, torch.bfloat16),
                                    (96, 4096, torch.float32), (4096, 1024, torch.bfloat16),
                                    (37, 40, torch.bfloat16)])
def test_quantize_and_dequantize_bit_exact(m, n, dt):
    """Codes, scales and dequantised values bit for bit against the oracle; n % 16 == 0 takes
    the 16-wide dequantisation, n = 40 the element-wise one."""
    rng = np.random.default_rng(m * 7 + n)
    w = rng.standard_normal((m, n)) * rng.uniform(0.01, 2.0, size=n)[None, :]
    w[:, 5] = 0.0                                      # an all-zero column
    w[:8, 6] = [127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 126.5]   # exact ties at scale 1
    w[8:, 6] = 0.0
    wd = torch.from_numpy(w.astype(np.float32)).to(dt).cuda()
    wq, scale = _quantize(wd)
    deq = _dequantize(wq, scale)
    torch.cuda.synchronize()
    q_ref, s_ref = OQ.quantize_w0_int8(wd.float().cpu().numpy())
    assert np.array_equal(wq.cpu().numpy(), q_ref)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(deq.float().cpu().numpy().astype(np.float64),
                          OQ.dequantize_w0_int8(q_ref, s_ref))


# ------------------------------------------------------------------ layer == bf16 layer on W_deq
@pytest.mark.parametrize("key,m,n,b,T", [
    ("llama8b_up_proj", 1024, 3584, 512, 1100),   # both W0' products fused
    ("llama1p3b_attn", 512, 768, 128, 333),       # fused, ragged token tail
    ("llama1p3b_attn", 512, 640, 128, 300),       # forward dequantises first (n % 256 != 0)
    ("llama1p3b_attn", 768, 512, 256, 200),       # T < 256: both dequantise first
])
def test_xq_layer_bitwise_equals_bf16_layer_on_dequantised_weight(key, m, n, b, T):
    x = XqCase(key, m=m, n=n, b=b, tokens=T)
    out_xq = x.run(x.xq)
    out_bf = x.run(x.deq)
    torch.cuda.synchronize()
    for name, a, r in zip(("y", "B", "dx", "dq_r", "dq_p"), out_xq, out_bf):
        assert torch.equal(a, r), name


@pytest.mark.parametrize("key,m,n,b,T", [("llama8b_up_proj", 1024, 3584, 512, 1100),
                                         ("llama1p3b_attn", 512, 640, 128, 300)])
def test_staged_dequantisation_is_bitwise_the_in_kernel_one(key, m, n, b, T):
    x = XqCase(key, m=m, n=n, b=b, tokens=T)
    c = x.c
    staged = poetx.PoetxLinear(x.wq, c.perm_r, c.perm_p, c.q_r, c.q_p, c.b, w0m_scale=x.scale,
                               staged=True)
    poetx.layer_cnp_build(staged)
    a = x.run(x.xq)
    s = x.run(staged)
    torch.cuda.synchronize()
    for name, u, v in zip(("y", "B", "dx", "dq_r", "dq_p"), a, s):
        assert torch.equal(u, v), name


def test_xq_backward_without_saved_b_is_identical():
    x = XqCase("llama8b_up_proj", m=1024, n=2048, b=512, tokens=600)
    a = x.run(x.xq)
    b = x.run(x.xq, saved=False)
    torch.cuda.synchronize()
    for name, u, v in zip(("dx", "dq_r", "dq_p"), a[2:], b[2:]):
        assert torch.equal(u, v), name


# ------------------------------------------------------------------ against the oracle
@pytest.mark.parametrize("key,m,n,b,T", [
    ("llama8b_up_proj", 1024, 3584, 512, 300),
    ("llama1p3b_attn", 1024, 1024, 256, 333),
    ("llama1p3b_attn", 512, 640, 128, 130),
])
def test_xq_layer_matches_oracle(key, m, n, b, T):
    x = XqCase(key, m=m, n=n, b=b, tokens=T)
    h, q, s, W_deq = x.host_w0m_deq()
    assert np.array_equal(x.wq.cpu().numpy(), q)
    y, _, dx, dq_r, dq_p = x.run(x.xq)
    torch.cuda.synchronize()
    c = x.c
    G_r, G_p = O.cnp(h["q_r"], c.b), O.cnp(h["q_p"], c.b)
    ref = O.linear_bwd(h["X"], h["dY"], W_deq, h["perm_r"], h["perm_p"], G_r, G_p, h["q_r"],
                       h["q_p"], c.b)
    errs = {"y": rel_err(y, ref["Y"]), "dx": rel_err(dx, ref["dX"]),
            "dq_r": rel_err(dq_r, ref["dq_r"]), "dq_p": rel_err(dq_p, ref["dq_p"])}
    for k, e in errs.items():
        assert e <= TOL_BF16, (k, errs)


def test_xq_full_size_sampled_llama8b_up_proj():
    """Full Llama-8B up_proj size (T = 16384, 4096 x 14336, b = 512): sampled token rows of Y
    and dX and the dq of those rows against the oracle on the dequantised W0'."""
    x = XqCase("llama8b_up_proj")
    c = x.c
    h, q, s, W_deq = x.host_w0m_deq()
    rows = np.sort(np.random.default_rng(3).choice(c.T, 8, replace=False))
    dy_sparse = torch.zeros_like(c.dy)
    idx = torch.from_numpy(rows).cuda()
    dy_sparse[idx] = c.dy[idx]
    y, _, dx, dq_r, dq_p = x.run(x.xq, dy=dy_sparse)
    torch.cuda.synchronize()
    assert np.array_equal(x.scale.cpu().numpy().view(np.uint32), s.view(np.uint32))
    G_r, G_p = O.cnp(h["q_r"], c.b), O.cnp(h["q_p"], c.b)
    ref = O.linear_bwd(h["X"][rows], h["dY"][rows], W_deq, h["perm_r"], h["perm_p"], G_r, G_p,
                       h["q_r"], h["q_p"], c.b)
    assert rel_err(y[rows], ref["Y"]) <= TOL_BF16
    assert rel_err(dx[rows], ref["dX"]) <= TOL_BF16
    assert rel_err(dq_r, ref["dq_r"]) <= TOL_BF16
    assert rel_err(dq_p, ref["dq_p"]) <= TOL_BF16


# ------------------------------------------------------------------ merge-then-reinitialize
def test_xq_merge_reinit_matches_oracle():
    x = XqCase("llama1p3b_attn", m=512, n=768, b=128, tokens=64, q_scale=4.0)
    c = x.c
    h, q, s, W_deq = x.host_w0m_deq()
    y0 = x.run(x.xq)[0]
    seed = 0xBEEF
    poetx.merge_reinit(x.xq, seed)
    torch.cuda.synchronize()
    ref = O.merge_reinit(W_deq, h["perm_r"], h["perm_p"], h["q_r"], h["q_p"], c.b, seed)
    assert np.array_equal(c.perm_r.cpu().numpy(), ref["perm_r"])
    assert np.array_equal(c.perm_p.cpu().numpy(), ref["perm_p"])
    assert torch.count_nonzero(c.q_r) == 0 and torch.count_nonzero(c.q_p) == 0
    # new codes: compare what they stand for (codes sit on rounding boundaries the bf16 product
    # on the device and the float64 product of the oracle may round apart)
    assert rel_err(_dequantize(x.wq, x.scale), ref["W0m"]) <= TOL_BF16
    poetx.layer_cnp_build(x.xq)
    y1 = x.run(x.xq)[0]
    torch.cuda.synchronize()
    assert rel_err(y1, y0.double().cpu().numpy()) <= TOL_BF16
