"""mmf_bitlinear_fwd_noalloc: the forward for callers that cannot allocate
device memory (a plug-in whose host runtime owns every device allocation, or a
latency-critical caller that must not block in cudaMalloc).  Its workspace is a
static array inside the library, so the caller passes only inputs and outputs.

Checked through the C ABI against mmf_bitlinear_fwd (caller-supplied
workspace) on two calls in a row with different inputs, so the second call
runs on scratch the first one left behind.  This file is collected last so a
run that stops at its first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from bitlinear_rmsnorm_quant_b200 import mmf
from gpu_cases import Y_REL_TOL, bits_np, make_layer, y_rel_error

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _noalloc(x, g, packed, scale, N, y):
    """Direct C-ABI call; y is preallocated so nothing is allocated here."""
    M, K = x.shape
    return mmf.lib().mmf_bitlinear_fwd_noalloc(x.data_ptr(), g.data_ptr(), 1e-6, packed.data_ptr(),
                                               scale.data_ptr(), M, K, N, y.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream)


# (4096, 2048, 512): the persistent streaming quantiser and the 256-token
# tensor-core tile write and read the static scratch
@pytest.mark.parametrize("M,K,N", [(1000, 2048, 512), (300, 384, 300), (4, 2560, 1000), (4096, 2048, 512)])
def test_noalloc_matches_workspace_forward_twice(M, K, N):
    from bitlinear_rmsnorm_quant_b200 import build
    build.build()
    torch.cuda.set_device(0)
    assert mmf.workspace_bytes(M, K, N) <= mmf.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((21, 22)):           # two calls in a row, different inputs
        x, g, W = make_layer(seed, M, K, N)
        xd, gd = x.to(DEV), g.to(DEV)
        packed, scale = mmf.pack_ternary(W.to(DEV), 1e-5)
        y_ref = mmf.bitlinear_fwd(xd, gd, packed, scale, N)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _noalloc(xd, gd, packed, scale, N, y) == mmf.MMF_OK
        torch.cuda.synchronize()
        mmf.check_async()
        err = y_rel_error(bits_np(y), bits_np(y_ref))
        assert err <= Y_REL_TOL, (call, err)
        assert torch.equal(y, y_ref), f"call {call}: the two entry points differ"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    torch.cuda.set_device(0)
    M, K, N = 16384, 8192, 128                        # 128 MiB of codes > 64 MiB of scratch
    assert mmf.workspace_bytes(M, K, N) > mmf.NOALLOC_SCRATCH_BYTES
    small = torch.zeros(4096, dtype=torch.uint8, device=DEV)   # never read: rejected first
    p = small.data_ptr()
    rc = mmf.lib().mmf_bitlinear_fwd_noalloc(p, p, 1e-6, p, p, M, K, N, p, None)
    assert rc == 4   # MMF_ERR_WORKSPACE
    mmf.check_async()
