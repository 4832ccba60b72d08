"""GPU parity: the CUDA path through the C ABI against the float64 oracle on the same seeded
inputs.  Bit-exact for permutations and index work; max|gpu - oracle| / max|oracle| within
1e-5 for the fp32 CNP build and fp32 layer, within 1e-2 for the bf16 layer (y, dx, dq)."""
import numpy as np
import pytest
import torch

import oracle as O
import poetx_workloads as W
from tests.gpu_util import TOL_BF16, TOL_F32, LayerCase, poetx, rel_err

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


# ------------------------------------------------------------------ CNP
@pytest.mark.parametrize("b,sigma,nb", [(4, 0.2, 3), (16, 0.05, 2), (64, 0.01, 8), (96, 0.01, 2),
                                        (256, 0.005, 3), (512, 0.005, 2),
                                        # Q grown 4x past the workloads' scale (spectral
                                        # norm ~2 sigma sqrt(b) = 0.9 / 0.64, still below the 1
                                        # the Neumann series needs): the split-precision
                                        # products stay inside the fp32 bar
                                        (512, 0.02, 2), (256, 0.02, 2)])
def test_cnp_build_matches_oracle(b, sigma, nb):
    rng = np.random.default_rng(b)
    q = (rng.standard_normal((nb, b * (b - 1) // 2)) * sigma).astype(np.float32)
    qd = torch.from_numpy(q).cuda()
    g = torch.empty(nb, b, b, device="cuda")
    g_lp = torch.empty(nb, b, b, device="cuda", dtype=torch.bfloat16)
    poetx.cnp_build(qd, b, g, g_lp)
    torch.cuda.synchronize()
    assert rel_err(g, O.cnp(q, b)) <= TOL_F32
    # the bf16 copy is the round-to-nearest-even of the fp32 blocks
    assert torch.equal(g_lp, g.to(torch.bfloat16))


def test_cnp_q_zero_is_exact_identity():
    b, nb = 128, 3
    q = torch.zeros(nb, b * (b - 1) // 2, device="cuda")
    g = torch.empty(nb, b, b, device="cuda")
    g_lp = torch.empty(nb, b, b, device="cuda", dtype=torch.bfloat16)
    poetx.cnp_build(q, b, g, g_lp)
    eye = torch.eye(b, device="cuda").expand(nb, b, b)
    assert torch.equal(g, eye) and torch.equal(g_lp, eye.to(torch.bfloat16))


# ------------------------------------------------------------------ permutations
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("m,n", [(512, 512), (256, 1536), (1000, 24)])
def test_merge_permutations_bit_exact(dt, m, n):
    rng = np.random.default_rng(m + n)
    w0 = rng.standard_normal((m, n)).astype(np.float32)
    pr, pp = rng.permutation(m).astype(np.int32), rng.permutation(n).astype(np.int32)
    w0d = torch.from_numpy(w0).to(dt).cuda()
    out = torch.empty_like(w0d)
    poetx.merge_permutations(w0d, torch.from_numpy(pr).cuda(), torch.from_numpy(pp).cuda(), out)
    ref = O.merge_permutations(w0d.cpu().float().numpy(), pr, pp)
    assert np.array_equal(out.cpu().float().numpy(), ref)


@pytest.mark.parametrize("seed,lane,k", [(0, 0, 1), (1, 0, 7), (1, 1, 7), (1234, 0, 512),
                                         (2 ** 64 - 1, 1, 2048), (42, 0, 14336)])
def test_resampled_permutation_matches_oracle(seed, lane, k):
    perm = torch.empty(k, dtype=torch.int32, device="cuda")
    poetx.resample_permutation(seed, lane, perm)
    assert np.array_equal(perm.cpu().numpy(), O.resample_permutation(seed, lane, k))


def test_validate_permutation():
    p = torch.randperm(1000, dtype=torch.int32, device="cuda")
    assert poetx.validate_permutation(p)
    bad = p.clone(); bad[3] = bad[4]
    assert not poetx.validate_permutation(bad)
    bad = p.clone(); bad[0] = 1000
    assert not poetx.validate_permutation(bad)


# ------------------------------------------------------------------ bit-exact layer cases
@pytest.mark.parametrize("key,m,b,T", [("tiny_fp32", 512, 64, 200),
                                       ("llama1p3b_attn", 512, 128, 333),
                                       ("llama1p3b_attn", 1024, 256, 130),
                                       ("llama1p3b_attn", 1024, 256, 777),
                                       ("llama8b_up_proj", 1024, 512, 1100),
                                       ("llama8b_up_proj", 14336, 512, 97),
                                       ("llama1p3b_attn", 2048, 256, 8191),
                                       ("llama8b_up_proj", 4096, 512, 4099)])
def test_identity_layer_is_bit_exact(key, m, b, T):
    """q = 0 and W0 = I: G = I exactly and every product is by 1.0 or 0.0, so Y == X and
    dX == dY bit for bit; this pins the gathers, scatters and operand layouts. The last two
    cases run tens of row tiles per block product, with a ragged last row tile."""
    c = LayerCase(key, m=m, n=m, b=b, tokens=T, q_zero=True, w0=np.eye(m, dtype=np.float32))
    y, bsave = c.forward()
    dx, dq_r, dq_p = c.backward(bsave)
    torch.cuda.synchronize()
    assert torch.equal(y, c.x)
    assert torch.equal(dx, c.dy)


@pytest.mark.parametrize("key,m,b,T", [("tiny_fp32", 256, 64, 77), ("llama1p3b_attn", 512, 128, 260),
                                       ("llama8b_up_proj", 8192, 512, 129)])
def test_permutation_weight_is_bit_exact(key, m, b, T):
    """W0 a permutation matrix with q = 0: Y is X with its columns moved, bit for bit. With the
    identity cases above, bf16 rows of 512 to 14336 columns take every row-pair gather and
    scatter configuration (256 threads x 2 vectors, 256 x 4, 512 x 4), odd token counts
    included."""
    rng = np.random.default_rng(5)
    s = rng.permutation(m)
    w0 = np.zeros((m, m), dtype=np.float32)
    w0[np.arange(m), s] = 1.0
    c = LayerCase(key, m=m, n=m, b=b, tokens=T, q_zero=True, w0=w0)
    y, _ = c.forward()
    ref = torch.empty_like(c.x)
    ref[:, torch.from_numpy(s).cuda()] = c.x
    assert torch.equal(y, ref)


# ------------------------------------------------------------------ layer parity
def _check_layer(c: LayerCase, tol: float, xmem: bool = False):
    """Y, dX, dq_r, dq_p of the library against the oracle on the same inputs. xmem: the
    backward runs without the saved B (memory-saving mode: B is rebuilt inside the call)."""
    h = c.host()
    y, bsave = c.forward()
    dx, dq_r, dq_p = c.backward(None if xmem else bsave)
    torch.cuda.synchronize()
    G_r, G_p = O.cnp(h["q_r"], c.b), O.cnp(h["q_p"], c.b)
    ref = O.linear_bwd(h["X"], h["dY"], h["W0m"], h["perm_r"], h["perm_p"], G_r, G_p,
                       h["q_r"], h["q_p"], c.b)
    errs = {"y": rel_err(y, ref["Y"]), "dx": rel_err(dx, ref["dX"]),
            "dq_r": rel_err(dq_r, ref["dq_r"]), "dq_p": rel_err(dq_p, ref["dq_p"])}
    for k, e in errs.items():
        assert e <= tol, (k, errs)
    return errs


def tile_rows(T: int, seed: int, tile: int = 128) -> np.ndarray:
    """One random token row in every `tile`-row band of the T rows, plus the last row: every
    row tile of the products (and the ragged last band) is represented."""
    rng = np.random.default_rng(seed)
    rows = [t0 + int(rng.integers(0, min(tile, T - t0))) for t0 in range(0, T, tile)]
    return np.unique(np.array(rows + [T - 1]))


def test_fp32_layer_full_tiny_workload():
    """The tiny fp32 workload at its full size: 512x512, b = 64, 256 tokens."""
    _check_layer(LayerCase("tiny_fp32"), TOL_F32)


@pytest.mark.parametrize("m,n,b,T", [(512, 768, 64, 100), (1024, 512, 128, 257)])
def test_fp32_layer_shapes(m, n, b, T):
    _check_layer(LayerCase("tiny_fp32", m=m, n=n, b=b, tokens=T), TOL_F32)


@pytest.mark.parametrize("key,m,n,b,T", [
    ("llama1p3b_attn", 1024, 1024, 256, 333),
    ("llama8b_up_proj", 1024, 3584, 512, 300),
    ("llama8b_decoder", 512, 1536, 256, 129),
    ("llama1p3b_attn", 512, 512, 128, 1),
    ("llama8b_up_proj", 1024, 2048, 512, 1000),
    ("llama1p3b_attn", 768, 512, 256, 2049),
    ("llama8b_up_proj", 1024, 2048, 512, 2305),
    ("llama8b_up_proj", 1024, 2048, 512, 1),     # b = 512 below one row tile: other kernels
    ("llama8b_up_proj", 512, 1024, 512, 255),
])
def test_bf16_layer_parity(key, m, n, b, T):
    _check_layer(LayerCase(key, m=m, n=n, b=b, tokens=T), TOL_BF16)


@pytest.mark.parametrize("key,m,n,b,T", [("llama8b_up_proj", 1024, 2048, 512, 600),
                                         ("llama1p3b_attn", 1024, 512, 256, 333)])
def test_bf16_layer_parity_with_grown_q(key, m, n, b, T):
    """The layer with q four times the workloads' scale (as after many optimizer steps without
    a merge): G further from the identity, larger Q^2..Q^4 terms in the forward and in every
    product of the dq chain."""
    _check_layer(LayerCase(key, m=m, n=n, b=b, tokens=T, q_scale=4.0), TOL_BF16)


@pytest.mark.parametrize("key,m,n,b,T,tol", [
    ("llama8b_up_proj", 1024, 2048, 512, 2305, TOL_BF16),
    ("llama1p3b_attn", 1024, 1024, 256, 333, TOL_BF16),
    ("llama1p3b_attn", 512, 768, 128, 129, TOL_BF16),
    ("tiny_fp32", 512, 768, 64, 100, TOL_F32),
])
def test_memory_saving_backward_matches_oracle(key, m, n, b, T, tol):
    """POET-Xmem: the backward without the saved B (rebuilt inside the call) against the
    oracle's exact gradient, not only against the saved-B backward."""
    _check_layer(LayerCase(key, m=m, n=n, b=b, tokens=T), tol, xmem=True)


# ------------------------------------------------------------------ W0' -> P-block fusion
def _fused_twin(c: LayerCase):
    """The same layer (same device tensors) with POETX_LAYER_FUSED_W0_P set."""
    f = poetx.PoetxLinear(c.layer.w0m, c.perm_r, c.perm_p, c.q_r, c.q_p, c.b, fused_w0_p=True)
    poetx.layer_cnp_build(f)
    return f


@pytest.mark.parametrize("m,n,T", [(1024, 2048, 1000), (512, 1536, 256), (2048, 1024, 300)])
def test_fused_w0_p_forward_matches_oracle_and_two_launch_forward(m, n, T):
    """The forward with the W0' product and the P-block product in one kernel: Y and the saved
    B bit for bit those of the two-launch forward (same MMAs, same K order), Y within the bf16
    bar of the oracle, and with saved_b = NULL (B never written) the same Y."""
    c = LayerCase("llama8b_up_proj", m=m, n=n, b=512, tokens=T, seed=4000 + m + n + T)
    y0, b0 = c.forward()
    f = _fused_twin(c)
    y1 = torch.full_like(y0, float("nan"))
    b1 = torch.full_like(b0, float("nan"))
    poetx.linear_fwd(f, c.x, y1, b1)
    y2 = torch.full_like(y0, float("nan"))
    poetx.linear_fwd(f, c.x, y2, None)
    torch.cuda.synchronize()
    poetx.device_status()
    assert torch.equal(y1, y0) and torch.equal(b1, b0) and torch.equal(y2, y0)
    h = c.host()
    ref = O.linear_fwd(h["X"], h["W0m"], h["perm_r"], h["perm_p"], O.cnp(h["q_r"], c.b),
                       O.cnp(h["q_p"], c.b))
    assert rel_err(y1, ref["Y"]) <= TOL_BF16


def test_fused_w0_p_layer_full_steps_match_two_launch_layer():
    """A whole step of the fused-forward layer, in both activation modes: with the saved A and B
    (POET-Xfast) and with no B kept (POET-Xmem, B rebuilt by the backward), every output (Y, dX,
    dq_r, dq_p) bit for bit that of the same layer without the flag."""
    c = LayerCase("llama8b_up_proj", m=1024, n=2048, b=512, tokens=777, seed=4321)
    f = _fused_twin(c)
    T, m, n = c.T, c.layer.m, c.layer.n

    def step(layer, keep_b):
        y = torch.empty(T, n, dtype=c.dt, device="cuda")
        a = torch.empty(T, m, dtype=c.dt, device="cuda")
        bs = torch.empty(T, n, dtype=c.dt, device="cuda") if keep_b else None
        poetx.linear_fwd(layer, c.x, y, bs, saved_a=a)
        dx = torch.empty(T, m, dtype=c.dt, device="cuda")
        dq_r, dq_p = torch.empty_like(c.q_r), torch.empty_like(c.q_p)
        poetx.linear_bwd(layer, c.x, c.dy, bs, dx, dq_r, dq_p, saved_a=a)
        return y, dx, dq_r, dq_p

    for keep_b in (True, False):
        ref = step(c.layer, keep_b)
        got = step(f, keep_b)
        torch.cuda.synchronize()
        poetx.device_status()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), keep_b


@pytest.mark.slow
def test_fused_w0_p_forward_many_tiles_per_cluster_matches_two_launch_forward():
    """16384 tokens x 8 P blocks: 512 tiles, several per CTA pair, so the ring, the B tile and
    the G slots are handed from tile to tile; bit for bit the two-launch forward, and the
    backward from the fused forward's saved B is the same too."""
    c = LayerCase("llama8b_up_proj", m=1024, n=4096, b=512, tokens=16384, seed=4242)
    y0, b0 = c.forward()
    f = _fused_twin(c)
    y1 = torch.full_like(y0, float("nan"))
    b1 = torch.full_like(b0, float("nan"))
    poetx.linear_fwd(f, c.x, y1, b1)
    torch.cuda.synchronize()
    poetx.device_status()
    assert torch.equal(y1, y0) and torch.equal(b1, b0)


# ------------------------------------------------------------------ merge-then-reinitialize
@pytest.mark.parametrize("key,m,n,b,tol", [("tiny_fp32", None, None, None, TOL_F32),
                                           ("llama1p3b_attn", 512, 768, 128, TOL_BF16)])
def test_merge_reinit_matches_oracle(key, m, n, b, tol):
    c = LayerCase(key, m=m, n=n, b=b, tokens=64, q_scale=4.0)
    h = c.host()
    y0, _ = c.forward()
    seed = 0xC0FFEE
    poetx.merge_reinit(c.layer, seed)
    torch.cuda.synchronize()
    ref = O.merge_reinit(h["W0m"], h["perm_r"], h["perm_p"], h["q_r"], h["q_p"], c.b, seed)
    assert np.array_equal(c.perm_r.cpu().numpy(), ref["perm_r"])
    assert np.array_equal(c.perm_p.cpu().numpy(), ref["perm_p"])
    assert torch.count_nonzero(c.q_r) == 0 and torch.count_nonzero(c.q_p) == 0
    assert rel_err(c.layer.w0m, ref["W0m"]) <= tol
    # the layer function survives the merge (q = 0 now, so G = I)
    poetx.layer_cnp_build(c.layer)
    y1, _ = c.forward()
    torch.cuda.synchronize()
    assert rel_err(y1, y0.double().cpu().numpy()) <= (tol if tol > TOL_F32 else 1e-5)


# ------------------------------------------------------------------ full-size sampled checks
@pytest.mark.parametrize("key", ["llama1p3b_attn", "llama8b_up_proj"])
def test_full_size_sampled(key):
    """Full workload sizes: one token row in every 128-row tile (and the last row) of Y and dX
    against the oracle row by row, and dq against the oracle restricted to those rows (dY is
    zero elsewhere)."""
    c = LayerCase(key)
    h = c.host()
    rows = tile_rows(c.T, 0)
    G_r, G_p = O.cnp(h["q_r"], c.b), O.cnp(h["q_p"], c.b)
    y, bsave = c.forward()
    dx, _, _ = c.backward(bsave)
    torch.cuda.synchronize()
    Xs, dYs = h["X"][rows], h["dY"][rows]
    y_ref = O.linear_fwd_rows(Xs, h["W0m"], h["perm_r"], h["perm_p"], G_r, G_p)
    dx_ref = O.linear_dx_rows(dYs, h["W0m"], h["perm_r"], h["perm_p"], G_r, G_p)
    assert rel_err(y[rows], y_ref) <= TOL_BF16
    assert rel_err(dx[rows], dx_ref) <= TOL_BF16
    dy_sparse = torch.zeros_like(c.dy)
    idx = torch.from_numpy(rows).cuda()
    dy_sparse[idx] = c.dy[idx]
    _, dq_r, dq_p = c.backward(bsave, dy=dy_sparse)
    torch.cuda.synchronize()
    ref = O.linear_bwd(Xs, dYs, h["W0m"], h["perm_r"], h["perm_p"], G_r, G_p, h["q_r"],
                       h["q_p"], c.b)
    assert rel_err(dq_r, ref["dq_r"]) <= TOL_BF16
    assert rel_err(dq_p, ref["dq_p"]) <= TOL_BF16


@pytest.mark.slow
@pytest.mark.parametrize("key", ["llama1p3b_attn", "llama8b_up_proj"])
def test_full_size_dense_every_row_and_dq(key):
    """Full workload size with dense dY: every row of Y and dX, and dq_r / dq_p, against the
    oracle, for the saved-B backward and for the memory-saving one (saved_b = None). The
    oracle streams the tokens in chunks: Y and dX of a token depend on that token only, and
    dG = sum over tokens of A_t^T dA'_t (B_t^T dC_t) is additive over chunks, so the chunks'
    dG are summed and dq is the CNP chain rule of the sum (dq is linear in dG)."""
    c = LayerCase(key)
    h = c.host()
    G_r, G_p = O.cnp(h["q_r"], c.b), O.cnp(h["q_p"], c.b)
    y, bsave = c.forward()
    dx, dq_r, dq_p = c.backward(bsave)
    dx_m, dq_r_m, dq_p_m = c.backward(None)
    torch.cuda.synchronize()
    num = {k: 0.0 for k in ("y", "dx", "dx_xmem")}
    den = {k: 0.0 for k in ("y", "dx")}
    dG_r = dG_p = 0.0
    chunk = 4096
    for t0 in range(0, c.T, chunk):
        sl = slice(t0, min(c.T, t0 + chunk))
        ref = O.linear_bwd(h["X"][sl], h["dY"][sl], h["W0m"], h["perm_r"], h["perm_p"], G_r,
                           G_p, h["q_r"], h["q_p"], c.b)
        dG_r = dG_r + ref["dG_r"]
        dG_p = dG_p + ref["dG_p"]
        # (error name, reference name, device rows, oracle rows)
        for name, rname, gpu, want in (("y", "y", y[sl], ref["Y"]), ("dx", "dx", dx[sl], ref["dX"]),
                                       ("dx_xmem", "dx", dx_m[sl], ref["dX"])):
            g = gpu.double().cpu().numpy()
            num[name] = max(num[name], float(np.max(np.abs(g - want))))
            den[rname] = max(den[rname], float(np.max(np.abs(want))))
        del ref
    errs = {"y": num["y"] / den["y"], "dx": num["dx"] / den["dx"],
            "dx_xmem": num["dx_xmem"] / den["dx"]}
    dq_r_ref = O.dq_from_dG(dG_r, h["q_r"], c.b)
    dq_p_ref = O.dq_from_dG(dG_p, h["q_p"], c.b)
    errs.update({"dq_r": rel_err(dq_r, dq_r_ref), "dq_p": rel_err(dq_p, dq_p_ref),
                 "dq_r_xmem": rel_err(dq_r_m, dq_r_ref), "dq_p_xmem": rel_err(dq_p_m, dq_p_ref)})
    for k, e in errs.items():
        assert e <= TOL_BF16, (k, errs)


# ------------------------------------------------------------------ layer-level CNP and one-sided dq
@pytest.mark.parametrize("key,m,n,b", [("llama8b_up_proj", 1024, 3584, 512),
                                       ("tiny_fp32", 512, 768, 64)])
def test_layer_cnp_build_matches_per_side_builds(key, m, n, b):
    """One launch sequence over the R and P blocks gives the per-side results bit for bit."""
    c = LayerCase(key, m=m, n=n, b=b, tokens=8)
    lay = c.layer
    g_r = torch.empty_like(lay.g_r)
    g_p = torch.empty_like(lay.g_p)
    lp_r = torch.empty_like(lay.g_r_lp) if lay.g_r_lp is not None else None
    lp_p = torch.empty_like(lay.g_p_lp) if lay.g_p_lp is not None else None
    poetx.cnp_build(c.q_r, b, g_r, lp_r)
    poetx.cnp_build(c.q_p, b, g_p, lp_p)
    torch.cuda.synchronize()
    assert torch.equal(g_r, lay.g_r) and torch.equal(g_p, lay.g_p)
    if lp_r is not None:
        assert torch.equal(lp_r, lay.g_r_lp) and torch.equal(lp_p, lay.g_p_lp)


@pytest.mark.parametrize("key,shapes", [
    ("llama8b_up_proj", [(1024, 3584), (2048, 1024), (512, 4096)]),
    ("llama1p3b_attn", [(512, 768)] * 9),          # nine layers: two launch sequences
    ("tiny_fp32", [(256, 512), (512, 256)]),
])
def test_layers_cnp_build_matches_per_layer_builds(key, shapes):
    """One poetx_layers_cnp_build over a set of layers gives every layer's G blocks (fp32 and
    bf16) bit for bit as one poetx_layer_cnp_build per layer."""
    cases = [LayerCase(key, m=m, n=n, tokens=4, seed=1000 + i) for i, (m, n) in enumerate(shapes)]
    ref = [(c.layer.g_r.clone(), c.layer.g_p.clone(),
            None if c.layer.g_r_lp is None else c.layer.g_r_lp.clone(),
            None if c.layer.g_p_lp is None else c.layer.g_p_lp.clone()) for c in cases]
    for c in cases:
        for t in (c.layer.g_r, c.layer.g_p, c.layer.g_r_lp, c.layer.g_p_lp):
            if t is not None:
                t.fill_(float("nan"))
    poetx.layers_cnp_build([c.layer for c in cases])
    torch.cuda.synchronize()
    for c, (gr, gp, lr, lpp) in zip(cases, ref):
        assert torch.equal(c.layer.g_r, gr) and torch.equal(c.layer.g_p, gp)
        if lr is not None:
            assert torch.equal(c.layer.g_r_lp, lr) and torch.equal(c.layer.g_p_lp, lpp)


@pytest.mark.parametrize("key,shapes,T", [
    ("llama8b_up_proj", [(1024, 3584), (2048, 1024), (512, 4096)], 700),
    ("llama8b_up_proj", [(1024, 2048), (1024, 1024)], 2305),   # split token ranges
    ("llama1p3b_attn", [(512, 768)] * 9, 333),                # nine layers: two sequences
    ("tiny_fp32", [(256, 512), (512, 256)], 99),
])
def test_dg_backward_then_layers_dq_matches_per_layer_backward(key, shapes, T):
    """poetx_linear_bwd_dg per layer (dX and dG) followed by one poetx_layers_dq_from_dg gives
    the dX and dq of poetx_linear_bwd per layer (equal values), with the saved B and with B
    rebuilt."""
    cases = [LayerCase(key, m=m, n=n, tokens=T, seed=2000 + i) for i, (m, n) in enumerate(shapes)]
    for rebuilt in (False, True):
        refs, dGs, dxs = [], [], []
        for c in cases:
            y, bsave = c.forward()
            saved = None if rebuilt else bsave
            refs.append(c.backward(saved))
            dx = torch.empty_like(c.x)
            dG = torch.full((c.layer.m // c.b + c.layer.n // c.b, c.b, c.b), float("nan"),
                            device="cuda")
            poetx.linear_bwd_dg(c.layer, c.x, c.dy, saved, dx, dG)
            dGs.append(dG)
            dxs.append(dx)
        dq_rs = [torch.empty_like(c.q_r) for c in cases]
        dq_ps = [torch.empty_like(c.q_p) for c in cases]
        poetx.layers_dq_from_dg([c.layer for c in cases], dGs, dq_rs, dq_ps)
        torch.cuda.synchronize()
        for (dx_ref, dqr_ref, dqp_ref), dx, dqr, dqp in zip(refs, dxs, dq_rs, dq_ps):
            assert torch.equal(dx, dx_ref)
            assert torch.equal(dqr, dqr_ref) and torch.equal(dqp, dqp_ref)


@pytest.mark.parametrize("key,m,n,b,T", [("llama8b_up_proj", 1024, 2048, 512, 700),
                                         ("tiny_fp32", 256, 512, 64, 99)])
def test_one_sided_dq_matches_two_sided(key, m, n, b, T):
    """dq of one side alone (its own dG launch) equals the two-sided dq (bf16, b % 256 == 0: one
    dG launch over both sides) bit for bit. At T = 700 both take one split of the token range,
    so the sums run in the same order; at larger T the split counts differ and the two agree
    within rounding, which the oracle parity cases (T = 2049, 2305: several splits) check."""
    c = LayerCase(key, m=m, n=n, b=b, tokens=T)
    y, bsave = c.forward()
    dx, dq_r, dq_p = c.backward(bsave)
    only_r = torch.empty_like(dq_r)
    only_p = torch.empty_like(dq_p)
    poetx.linear_bwd(c.layer, c.x, c.dy, bsave, None, only_r, None)
    poetx.linear_bwd(c.layer, c.x, c.dy, bsave, None, None, only_p)
    torch.cuda.synchronize()
    assert torch.equal(only_r, dq_r) and torch.equal(only_p, dq_p)


# ------------------------------------------------------------------ memory-saving backward
@pytest.mark.parametrize("key,m,n,b,T", [("llama8b_up_proj", 1024, 2048, 512, 700),
                                         ("tiny_fp32", 256, 512, 64, 99)])
def test_backward_without_saved_b_is_identical(key, m, n, b, T):
    """saved_b = NULL rebuilds B exactly with the same kernels: results equal bit for bit."""
    c = LayerCase(key, m=m, n=n, b=b, tokens=T)
    y, bsave = c.forward()
    dx, dq_r, dq_p = c.backward(bsave)
    dx2 = torch.empty_like(dx)
    dq_r2, dq_p2 = torch.empty_like(dq_r), torch.empty_like(dq_p)
    poetx.linear_bwd(c.layer, c.x, c.dy, None, dx2, dq_r2, dq_p2)
    torch.cuda.synchronize()
    assert torch.equal(dx2, dx) and torch.equal(dq_r2, dq_r) and torch.equal(dq_p2, dq_p)


@pytest.mark.parametrize("key,m,n,b,T", [("llama8b_up_proj", 1024, 2048, 512, 700),
                                         ("llama1p3b_attn", 512, 768, 128, 333),
                                         ("tiny_fp32", 256, 512, 64, 99)])
def test_saved_a_is_the_gather_and_changes_nothing(key, m, n, b, T):
    """poetx_linear_fwd_ex keeps A = X[:, perm_r] (bit for bit); poetx_linear_bwd_ex reading it
    (x passed as None) gives the same dX, dq as the backward that gathers X again, with the
    saved B and with B rebuilt."""
    c = LayerCase(key, m=m, n=n, b=b, tokens=T)
    y, bsave = c.forward()
    a = torch.empty_like(c.x)
    y2 = torch.empty_like(y)
    b2 = torch.empty_like(bsave)
    poetx.linear_fwd(c.layer, c.x, y2, b2, saved_a=a)
    torch.cuda.synchronize()
    assert torch.equal(a, c.x[:, c.perm_r.long()])
    assert torch.equal(y2, y) and torch.equal(b2, bsave)
    for saved in (bsave, None):
        dx, dq_r, dq_p = c.backward(saved)
        dx2 = torch.empty_like(dx)
        dq_r2, dq_p2 = torch.empty_like(dq_r), torch.empty_like(dq_p)
        poetx.linear_bwd(c.layer, None, c.dy, saved, dx2, dq_r2, dq_p2, saved_a=a)
        torch.cuda.synchronize()
        assert torch.equal(dx2, dx) and torch.equal(dq_r2, dq_r) and torch.equal(dq_p2, dq_p)


# ------------------------------------------------------------------ more full-size shapes
@pytest.mark.parametrize("key,layer", [("llama8b_decoder", 1),    # k_proj 4096 x 1024
                                       ("llama8b_decoder", 6),    # down_proj 14336 x 4096
                                       ("llama13b_layers", 4)])   # gate 5120 x 13824
def test_full_size_sampled_other_linears(key, layer):
    c = LayerCase(key, layer)
    h = c.host()
    rows = tile_rows(c.T, layer)
    G_r, G_p = O.cnp(h["q_r"], c.b), O.cnp(h["q_p"], c.b)
    y, bsave = c.forward()
    dy_sparse = torch.zeros_like(c.dy)
    idx = torch.from_numpy(rows).cuda()
    dy_sparse[idx] = c.dy[idx]
    dx, dq_r, dq_p = c.backward(bsave, dy=dy_sparse)
    torch.cuda.synchronize()
    Xs, dYs = h["X"][rows], h["dY"][rows]
    ref = O.linear_bwd(Xs, dYs, h["W0m"], h["perm_r"], h["perm_p"], G_r, G_p, h["q_r"],
                       h["q_p"], c.b)
    assert rel_err(y[rows], ref["Y"]) <= TOL_BF16
    assert rel_err(dx[rows], ref["dX"]) <= TOL_BF16
    assert rel_err(dq_r, ref["dq_r"]) <= TOL_BF16
    assert rel_err(dq_p, ref["dq_p"]) <= TOL_BF16


# ------------------------------------------------------------------ 13B layer: 400 steps + merge
@pytest.mark.slow
def test_llama13b_layer_400_steps_with_merge_reinit():
    """The 13B layer-set schedule on its q/k/v/o shape (5120 x 5120, b = 512, 8192 tokens): 400
    fwd+bwd steps with q += N(0, 1e-4^2) after each, merge_reinit at step 400, one more step.
    The oracle replays the same float32 q sequence and checks sampled rows of Y at steps 1, 2,
    400 and 401 and the merged weight."""
    import poetx_workloads as W
    wl = W.WORKLOADS["llama13b_layers"]
    c = LayerCase("llama13b_layers", 0)
    h = c.host()
    rows = np.sort(np.random.default_rng(13).choice(c.T, 6, replace=False))
    Xs = h["X"][rows]
    q_r, q_p = h["q_r"].astype(np.float32).copy(), h["q_p"].astype(np.float32).copy()
    W0m = h["W0m"].astype(np.float64)
    pr, pp = h["perm_r"], h["perm_p"]
    checks = {1, 2, 400, 401}

    def check(step):
        y, _ = c.forward()
        torch.cuda.synchronize()
        ref = O.linear_fwd_rows(Xs, W0m, pr, pp, O.cnp(q_r, c.b), O.cnp(q_p, c.b))
        assert rel_err(y[rows], ref) <= TOL_BF16, step

    for step in range(1, 402):
        poetx.layer_cnp_build(c.layer)
        if step in checks:
            check(step)
        y, bsave = c.forward()
        poetx.linear_bwd(c.layer, c.x, c.dy, bsave, None, torch.empty_like(c.q_r),
                         torch.empty_like(c.q_p))
        if step == 400:
            seed = 0x13B0400
            poetx.layer_cnp_build(c.layer)
            poetx.merge_reinit(c.layer, seed)
            torch.cuda.synchronize()
            ref = O.merge_reinit(W0m, pr, pp, q_r, q_p, c.b, seed)
            assert rel_err(c.layer.w0m, ref["W0m"]) <= TOL_BF16
            assert np.array_equal(c.perm_r.cpu().numpy(), ref["perm_r"])
            W0m, pr, pp = ref["W0m"], ref["perm_r"], ref["perm_p"]
            q_r[:] = 0
            q_p[:] = 0
        # harness perturbation, identical float32 arithmetic on both sides
        d_r = W.q_perturbation(wl, 0, step, 0, q_r.shape)
        d_p = W.q_perturbation(wl, 0, step, 1, q_p.shape)
        c.q_r += torch.from_numpy(d_r).cuda()
        c.q_p += torch.from_numpy(d_p).cuda()
        q_r += d_r
        q_p += d_p
    assert np.array_equal(c.q_r.cpu().numpy(), q_r)


# ------------------------------------------------------------------ no writes outside the outputs
@pytest.mark.parametrize("key,m,n,b,T", [("llama8b_up_proj", 1024, 2048, 512, 700),
                                         ("llama1p3b_attn", 1024, 1024, 256, 333),
                                         ("llama8b_up_proj", 1024, 2048, 512, 2305)])
def test_no_write_outside_outputs_or_workspace(key, m, n, b, T):
    """Every output (y, saved B, dx, dq_r, dq_p) and both workspaces sit inside larger buffers whose
    slack is filled with a canary; after the forward and the backward (saved B and rebuilt B) at a
    ragged token count, every canary byte is intact."""
    c = LayerCase(key, m=m, n=n, b=b, tokens=T)
    pad = 4096   # elements of slack on each side

    def boxed(numel, dtype):
        buf = torch.full((numel + 2 * pad,), -7.0, dtype=dtype, device="cuda")
        return buf, buf[pad:pad + numel]

    def ws_boxed(nbytes):
        buf = torch.full((nbytes + 2 * pad * 8,), 0xA5, dtype=torch.uint8, device="cuda")
        return buf, buf[pad * 8:pad * 8 + nbytes]

    dt = c.x.dtype
    y_buf, y = boxed(T * n, dt)
    b_buf, bs = boxed(T * n, dt)
    fws_buf, fws = ws_boxed(poetx.fwd_workspace_bytes(c.layer, T))
    poetx.linear_fwd(c.layer, c.x, y.view(T, n), bs.view(T, n), fws)
    dx_buf, dx = boxed(T * m, dt)
    dqr_buf, dqr = boxed(c.q_r.numel(), torch.float32)
    dqp_buf, dqp = boxed(c.q_p.numel(), torch.float32)
    bws_buf, bws = ws_boxed(poetx.bwd_workspace_bytes(c.layer, T))
    for saved in (bs.view(T, n), None):
        poetx.linear_bwd(c.layer, c.x, c.dy, saved, dx.view(T, m), dqr.view_as(c.q_r),
                         dqp.view_as(c.q_p), bws)
    torch.cuda.synchronize()
    for name, buf, fill in (("y", y_buf, -7.0), ("saved_b", b_buf, -7.0), ("dx", dx_buf, -7.0),
                            ("dq_r", dqr_buf, -7.0), ("dq_p", dqp_buf, -7.0)):
        for side in (buf[:pad], buf[-pad:]):
            assert bool((side == fill).all()), name
    for name, buf in (("fwd workspace", fws_buf), ("bwd workspace", bws_buf)):
        for side in (buf[:pad * 8], buf[-pad * 8:]):
            assert bool((side == 0xA5).all()), name
