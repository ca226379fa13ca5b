"""fp64 CPU oracle for the fused LoRA-adapted linear layer (test infrastructure only)."""
from .lora_oracle import *  # noqa: F401,F403
from .lora_oracle import (ACTS, ATOL, NORM_TOL, RTOL, act_backward, bf16_to_f64, compare,  # noqa: F401
                          lora_adapter_grads_identity, lora_backward, lora_backward_rows,
                          lora_forward, lora_forward_rows, lora_linear_branch,
                          lora_linear_branch_backward, sigmoid, silu, silu_grad)
