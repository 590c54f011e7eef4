"""Fused, chunked distillation KL loss over the LM output head for NVIDIA B200.

The loss and its gradients run in hand-written sm_100a CUDA kernels
(tcgen05/TMEM tensor-core tiles fed by TMA) behind a C ABI
(include/chunked_kl.h); this package only marshals torch tensors into it."""
from ._lib import KLError, kl_launch_count, kl_profile_begin, kl_profile_end  # noqa: F401
from .ops import (alloc_workspace, fused_kl_loss, kl_bwd, kl_fwd, kl_fwd_bwd,  # noqa: F401
                  make_problem, status, workspace_bytes)
