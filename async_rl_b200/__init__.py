"""B200-native batch-invariant token logprob + unclipped IS REINFORCE loss (sm_100a).

The compute path is the CUDA library ``libbi_isloss.so`` behind the C ABI in
``include/bi_isloss.h`` (the LM head, loss and diagnostics) and ``include/bi_model.h`` (the
batch-invariant GEMM and RMSNorm of the rest of the model); this package only loads it and
marshals tensors.
"""
from .api import (BiError, LossOutputs, check_status, d3_stats, decode_d3, debug_force_timeout_once,  # noqa: F401
                  gemm_bf16, is_loss_fwd_bwd, logprob_fwd, make_workspace, profile_enable, profile_read,
                  profile_reset, rmsnorm, workspace_bytes)
