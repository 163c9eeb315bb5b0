"""CPU oracle for the decode megakernel — TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct CPU statement of what one transformer decode
step computes (dense and MoE), written from the Event Tensor pages' definition
that a megakernel computes the same function as the ordinary per-op forward
pass, only scheduled differently ("Event Tensor: A Unified Abstraction for
Compiling Dynamic Megakernel", section "Core method": events are
synchronisation objects and never change values; "Lecture 112: Production
Megakernels for Real-World Inference", section "Summary": the whole forward
pass fused into one persistent kernel).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
path (``event_tensor_task_b200``): neither imports the other.  The only common
module is ``workloads``, which draws the seeded inputs and holds none of the
method's arithmetic.

Precision: fp64 everywhere, except (a) tensors the method stores in bf16 (the
weights, the KV cache including the row appended this step, MoE-layer
inputs and outputs), which are rounded to bf16 where they are stored, and (b)
the MoE router logits, which decide an integer (the top-k expert ids) and are
therefore taken in the kernel's precision, fp32, in one fixed summation order
(``moe.router_logits``).
"""
from .dense import (rms_norm, rope_cos_sin, apply_rope, decode_attention, swiglu,
                    bf16_round, DenseOracle)
from .moe import (router_logits, topk_route, expert_histogram, exp_indptr,
                  moe_ffn, moe_layer)
from .tasks import expected_dense_tasks, dense_family_extents, expected_moe_tasks, moe_tiles

__all__ = [
    "rms_norm", "rope_cos_sin", "apply_rope", "decode_attention", "swiglu",
    "bf16_round", "DenseOracle", "router_logits", "topk_route",
    "expert_histogram", "exp_indptr", "moe_ffn", "moe_layer",
    "expected_dense_tasks", "dense_family_extents", "expected_moe_tasks", "moe_tiles",
]
