"""fp64 CPU oracle of the nanochat decoder step (forward + backward).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
bench's CPU-baseline leg, never by the library's product path.  It shares no
code with the CUDA kernels; inputs come from the separate `synth` module.
"""
from .model import (EPS, HEAD_DIM, ROPE_THETA, SOFTCAP, attention, attention_bwd,  # noqa: F401
                    block_backward, block_forward, dims, forward_logits, forward_loss,
                    head_backward_row, head_forward_row, head_loss_row,
                    loss_and_grads, param_layout, rmsnorm, rmsnorm_bwd, rope, rope_bwd,
                    rope_tables)
