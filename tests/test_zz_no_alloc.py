"""poetx_cnp_build_noalloc: the CNP build for callers that cannot allocate device memory.

Such callers (a host program that owns all device memory and forbids later allocation, or code
that must avoid the device-wide synchronisation of cudaMalloc/cudaFree) pass no workspace; the
library uses a fixed scratch buffer of its own.  These tests call it through the C ABI on two
calls in a row, so a result that depended on what the previous call left in the shared buffer
would show, and check it three ways: against the float64 oracle (1e-5, the fp32 CNP bar),
bit for bit against poetx_cnp_build (caller workspace) where both take the blocks in one pass,
and its bf16 copy bit for bit against the round-to-nearest-even of its own fp32 blocks.  This
file sorts last so that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import TOL_F32, poetx, rel_err

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _q(nb, b, sigma, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((nb, b * (b - 1) // 2)) * sigma).astype(np.float32)


def _noalloc(qd, nb, b, g, lp):
    st = poetx.lib.poetx_cnp_build_noalloc(qd.data_ptr(), nb, b, g.data_ptr(),
                                           lp.data_ptr() if lp is not None else None,
                                           poetx.BF16, torch.cuda.current_stream().cuda_stream)
    assert st == 0, poetx.lib.poetx_last_error_message()


def test_noalloc_setup_call_launches_nothing():
    """nblocks = 0 performs only the per-device set-up (the buffer's address) and returns OK,
    with NULL q and outputs."""
    st = poetx.lib.poetx_cnp_build_noalloc(None, 0, 512, None, None, poetx.BF16,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 0, poetx.lib.poetx_last_error_message()


# (nb, b, sigma): 28 blocks of 512 take 14 chunks of the fixed buffer (2 blocks of 512 fit);
# 2 blocks of 512 and 8 of 256 fit in one chunk, as in the workspace build
@pytest.mark.parametrize("nb,b,sigma", [(28, 512, 0.005), (2, 512, 0.005), (8, 256, 0.005),
                                        (5, 96, 0.01)])
def test_noalloc_matches_oracle_and_workspace_build_on_two_calls(nb, b, sigma):
    chunk = (8 << 20) // poetx.cnp_workspace_bytes(1, b)
    for call, seed in enumerate((11, 12)):
        q = _q(nb, b, sigma * (1 + call), seed + b)
        qd = torch.from_numpy(q).cuda()
        g_ref = torch.empty(nb, b, b, device="cuda")
        lp_ref = torch.empty(nb, b, b, device="cuda", dtype=torch.bfloat16)
        poetx.cnp_build(qd, b, g_ref, lp_ref)
        g = torch.full((nb, b, b), float("nan"), device="cuda")
        lp = torch.full((nb, b, b), float("nan"), device="cuda", dtype=torch.bfloat16)
        _noalloc(qd, nb, b, g, lp)
        torch.cuda.synchronize()
        assert rel_err(g, O.cnp(q, b)) <= TOL_F32, (call, b)
        assert torch.equal(lp, g.to(torch.bfloat16)), (call, b)   # RNE of its own fp32 blocks
        if nb <= chunk:
            # one chunk: the same launches on the same blocks as the workspace build
            assert torch.equal(g, g_ref) and torch.equal(lp, lp_ref), (call, b)
        else:
            assert rel_err(g, g_ref.double().cpu().numpy()) <= TOL_F32, (call, b)


def test_noalloc_rejects_blocks_beyond_its_buffer():
    b = 1024
    q = torch.zeros(1, b * (b - 1) // 2, device="cuda")
    g = torch.empty(1, b, b, device="cuda")
    with pytest.raises(poetx.PoetxError) as e:
        poetx.cnp_build_noalloc(q, b, g)
    assert e.value.status == 2 and "buffer" in str(e.value)
