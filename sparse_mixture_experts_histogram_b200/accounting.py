"""Parameter, FLOP and byte accounting of the sparse MoE layer.

Closed forms, stated on the pages and used to turn measured times into
throughput and roofline fractions:

* a SwiGLU feed-forward of width d_hidden holds 3 * d * d_hidden parameters
  (2 matrices for GELU): "MoE: ..." (theaiera.top) sec. 10.6 estimator;
* the router holds d * E parameters (same section);
* one MoE layer holds 3 * d * E * d_ff expert parameters and its activation
  ratio is k / E: "万亿 MoE 只激活 4.9%" (m.xxqk.cn), parameter-count paragraph;
* parameters active per token = router + k * (one expert) (sec. 10.6);
* "match dense" shrinks each expert's hidden width so that the MoE holds as
  many parameters as the dense layer (sec. 10.6; its worked example gives
  1792 for d_hidden = 14336, E = 8).

FLOPs count one multiply-add as 2.  The bytes are the algorithmic minimum of
one layer call: bf16 weights of the experts the batch actually hits, the
router matrix, the bf16 input and the fp32 output.
"""
from __future__ import annotations


def ffn_params(d: int, d_hidden: int, matrices: int = 3) -> int:
    """Dense feed-forward parameters: matrices * d * d_hidden (3 for SwiGLU)."""
    return matrices * d * d_hidden


def router_params(d: int, E: int) -> int:
    return d * E


def expert_params(d: int, d_ff: int) -> int:
    """One SwiGLU expert: W1, W3 [d_ff, d] and W2 [d, d_ff]."""
    return 3 * d * d_ff


def moe_expert_params(d: int, E: int, d_ff: int) -> int:
    """All experts of one layer: 3 * d * E * d_ff."""
    return E * expert_params(d, d_ff)


def active_params_per_token(d: int, E: int, d_ff: int, k: int) -> int:
    return router_params(d, E) + k * expert_params(d, d_ff)


def match_dense_hidden(d: int, d_hidden: int, E: int) -> int:
    """Per-expert hidden width that makes E experts plus the router hold as
    many parameters as the dense SwiGLU layer, rounded to the nearest integer
    (the reading that reproduces the worked example's 1792)."""
    return round((ffn_params(d, d_hidden) - router_params(d, E)) / (E * expert_params(d, 1)))


def active_flops(T: int, d: int, E: int, d_ff: int, k: int, d_ff_shared: int = 0) -> int:
    """2*3*d*d_ff*k*T expert FLOPs + 2*T*d*E router FLOPs (+ the shared expert)."""
    return 2 * 3 * d * d_ff * k * T + 2 * T * d * E + 2 * 3 * d * d_ff_shared * T


def fp8_scale_bytes(d: int, d_ff: int) -> int:
    """fp32 row scales of one FP8 expert: W1 and W3 rows (d_ff each), W2 rows (d)."""
    return 4 * (2 * d_ff + d)


def algorithmic_bytes(T: int, d: int, E: int, d_ff: int, k: int, experts_hit: int,
                      d_ff_shared: int = 0, fp8: bool = False) -> int:
    """Minimum HBM bytes of one layer call: hit experts' weights (bf16, or e4m3
    codes plus their fp32 row scales), bf16 Wg, bf16 x read, fp32 out written
    (+ the shared expert's bf16 weights)."""
    wb = (experts_hit * (expert_params(d, d_ff) + fp8_scale_bytes(d, d_ff)) if fp8
          else 2 * experts_hit * expert_params(d, d_ff))
    return (wb + 2 * d * E + 2 * T * d + 4 * T * d + 2 * expert_params(d, d_ff_shared))


def ffn_bytes(T: int, d: int, d_ff: int, k: int, experts_hit: int, d_ff_shared: int = 0,
              fp8: bool = False) -> int:
    """Algorithmic bytes of the routed experts' feed-forward (both
    projections): bf16 W1, W3, W2 of the hit experts, the bf16 token rows
    read once (T rows of d) and the fp32 layer output written once (T rows of
    d).  The k routed copies of each row, the hidden activations H and the
    per-slot expert outputs are implementation bytes and are not counted.  A
    shared expert is its own launch over the T token rows with its own
    weights."""
    if fp8:
        return experts_hit * (3 * d * d_ff + fp8_scale_bytes(d, d_ff)) + 2 * T * d + 4 * T * d
    return 2 * 3 * experts_hit * d * d_ff + 2 * T * d + 4 * T * d


def ffn_flops(T: int, d: int, d_ff: int, k: int) -> int:
    """FLOPs of the expert feed-forward kernel: 2*3*d*d_ff per routed row."""
    return 2 * 3 * T * k * d * d_ff
