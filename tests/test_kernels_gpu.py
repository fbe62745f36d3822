"""GPU unit tests of device routines the attention kernels rely on."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_software_exp2_against_cuda_exp2f():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import bwd_causal_sdpa_b200 as A

    # the range the kernels feed it: scores minus a running max (<= 8) down to
    # far below the bf16 resolution
    x = torch.cat([torch.linspace(-126.0, 8.0, 1_000_001), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0]),
                   torch.randn(100_000) * 3]).float().cuda()
    y = torch.empty_like(x)
    assert A.attn_exp2_selftest(x, y, x.numel(), None) == A.ATTN_OK
    ref = torch.exp2(x)  # CUDA's exp2f
    torch.cuda.synchronize()
    rel = ((y.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel < 2e-4, rel   # polynomial fit 1.0e-4 plus float32 rounding
    assert y[x.numel() - 100_005 + 0].item() == 1.0  # 2^0 is exact
