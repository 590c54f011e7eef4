"""fp64 CPU oracle for the distillation KL loss (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs import
this package; the CUDA product path never does."""
from .kl_oracle import (HIDDEN, TOPK, dense_reconstruction_loss, kl_loss,  # noqa: F401
                        logsumexp_rows, teacher_support_probs)
