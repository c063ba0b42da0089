"""CPU oracle for the GLM-5.2 MoE feed-forward layer forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call, link
or execute this package: only the test suite, the smoke check and the timed
CPU baseline of the benchmark use it.  It shares no code with the CUDA path
(no kernels, headers, helpers or constants); the two meet only through the
seeded inputs of ``moe_inputs``.

The oracle is plain numpy: slow, unblocked and written to be checked against
the method's description by eye.  Precision: every routing decision is taken
in fp32, the router's own precision (the fp32 logit is the fp64 dot product
rounded once; the sigmoid is evaluated in fp64 and rounded once to fp32; the
bias add, the renormalising sum, the division and the scaling are single fp32
operations).  The expert MLPs, the shared expert and the merge are evaluated
in fp64 on the bf16 (or fp32) input values.

Pins (the tests under ``tests/`` that hold the oracle to something other than
itself): brute-force top-k over every k-subset, the closed forms of the
renormalised weights (sum equals the scale; the bias changes the selection but
not the weights; a zero router ties every expert and the lowest indices win;
k = E selects all experts), the routed-scale-zero case against torch's CPU
linear/SiLU, identity-weight experts against silu(x)*x, linearity in the
scale, token-permutation and expert-relabelling metamorphic checks, the
counting-sort permutation against a pure-Python bucket loop, and a
hand-derived worked example under ``tests/golden/``.
"""
from .moe_oracle import (  # noqa: F401
    router_logits,
    sigmoid_scores,
    selection_keys,
    select_topk,
    routing_weights,
    route,
    route_grouped,
    group_scores,
    routing_alternatives,
    swiglu_expert,
    e4m3_value,
    dequantize_fp8_blocks,
    group_by_expert,
    combine,
    moe_layer,
    moe_layer_tokens,
    routed_output_given_routing,
)
