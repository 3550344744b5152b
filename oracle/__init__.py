"""fp64 CPU oracle for the sparse MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg
of the benchmark are the only callers.  The product path never imports this
package, and this package imports nothing from the product.
"""
from .oracle import (  # noqa: F401
    ACT_SIGMOID,
    ACT_SILU,
    ENTROPY_TAU,
    ENTROPY_THRESHOLD,
    W_ENTROPY,
    W_SIGMOID,
    W_SOFTMAX_ALL,
    W_SOFTMAX_TOPK,
    build,
    capacity_limit,
    e4m3_to_double,
    ep_plan,
    forward_fp8,
    num_threads,
    route,
    forward,
    swiglu,
)
