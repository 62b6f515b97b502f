"""Float64 CPU oracle of the MoE layer, forward and backward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package; the CUDA product path never does.
"""
from .moe_oracle import (  # noqa: F401
    LayerConfig, Routing, Dispatch, Forward, RELU, SWIGLU,
    gate_logits, normalise_logits, softmax, top_k, route, capacity, dispatch,
    expert_hidden, expert_ffn, expert_segments, combine, forward, forward_tokens,
    brute_force, log_partition, z_loss, adaptive_aux_coef, shared_expert, forward_with_shared,
)
from .moe_backward import (  # noqa: F401
    Grads, loss, backward, expert_backward, normalise_backward, silu_grad, gate_weight_backward,
    aux_prob_grad, softmax_backward, z_loss_score_grad,
)
from . import moe_fp8  # noqa: F401  (MX FP8 expert weights: forward oracle)
