"""poetx_cnp_build_noalloc: the CNP build for callers that cannot allocate device memory.

Such callers (a host program that owns all device memory and forbids later allocation, or code
that must avoid the device-wide synchronisation of cudaMalloc/cudaFree) pass no workspace; the
library uses a fixed scratch buffer of its own.  These tests call it through the C ABI and
compare it with poetx_cnp_build (caller workspace) on two calls in a row, so a result that
depended on what the previous call left in the shared buffer would show.  This file sorts last
so that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

from tests.gpu_util import TOL_BF16, TOL_F32, poetx, rel_err

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _q(nb, b, sigma, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy((rng.standard_normal((nb, b * (b - 1) // 2)) * sigma)
                            .astype(np.float32)).cuda()


@pytest.mark.parametrize("nb,b,sigma", [(28, 512, 0.005), (8, 256, 0.005), (5, 96, 0.01)])
def test_noalloc_matches_workspace_build_on_two_calls(nb, b, sigma):
    for call, seed in enumerate((11, 12)):
        q = _q(nb, b, sigma * (1 + call), seed + b)
        g_ref = torch.empty(nb, b, b, device="cuda")
        lp_ref = torch.empty(nb, b, b, device="cuda", dtype=torch.bfloat16)
        poetx.cnp_build(q, b, g_ref, lp_ref)
        g = torch.full((nb, b, b), float("nan"), device="cuda")
        lp = torch.full((nb, b, b), float("nan"), device="cuda", dtype=torch.bfloat16)
        st = poetx.lib.poetx_cnp_build_noalloc(q.data_ptr(), nb, b, g.data_ptr(), lp.data_ptr(),
                                               poetx.BF16, torch.cuda.current_stream().cuda_stream)
        assert st == 0, poetx.lib.poetx_last_error_message()
        torch.cuda.synchronize()
        assert rel_err(g, g_ref.double().cpu().numpy()) <= TOL_F32, (call, b)
        assert rel_err(lp, lp_ref.double().cpu().numpy()) <= TOL_BF16, (call, b)


def test_noalloc_rejects_blocks_beyond_its_buffer():
    b = 1024
    q = torch.zeros(1, b * (b - 1) // 2, device="cuda")
    g = torch.empty(1, b, b, device="cuda")
    with pytest.raises(poetx.PoetxError) as e:
        poetx.cnp_build_noalloc(q, b, g)
    assert e.value.status == 2 and "buffer" in str(e.value)
