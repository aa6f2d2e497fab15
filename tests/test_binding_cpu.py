"""The Python binding refuses host tensors and malformed buffers before anything reaches the
library (which dereferences every pointer on the GPU).  CPU only."""
import pytest
import torch

import async_rl_b200 as bi


def test_host_tensors_are_refused():
    h = torch.zeros(4, 128, dtype=torch.bfloat16)
    w = torch.zeros(512, 128, dtype=torch.bfloat16)
    y = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bi.logprob_fwd(h, w, y)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bi.gemm_bf16(h, w)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bi.rmsnorm(h, torch.ones(128, dtype=torch.bfloat16), 1e-6)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bi.d3_stats(torch.zeros(4), torch.zeros(4))
    r = torch.zeros(2)
    with pytest.raises(ValueError, match="CUDA tensor"):
        bi.is_loss_fwd_bwd(h, w, y, torch.zeros(4), r, torch.tensor([0, 2, 4]), torch.tensor([0, 2], dtype=torch.int32))
