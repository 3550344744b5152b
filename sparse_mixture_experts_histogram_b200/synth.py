"""Seeded synthetic inputs for the sparse MoE layer.

This module only draws random numbers: it holds none of the layer's
arithmetic, and both the CUDA path and the CPU oracle are fed from it.

Recipe (the same for every workload):
  * one ``torch.Generator`` seeded with ``seed`` (42 by default), on the
    device the tensors are made on (CPU and CUDA streams differ, so a workload
    is identified by (shapes, seed, device));
  * tensors drawn in the fixed order x, Wg, W1, W3, W2 [, Ws1, Ws3, Ws2];
    each is drawn one leading-index slice at a time (one expert's matrix, or
    a block of rows of x) so that no fp32 temporary larger than one slice
    exists;
  * every value is an fp32 standard normal times sigma, rounded to bf16 with
    round-to-nearest-even;
  * sigma: x 1; Wg, W1, W3, Ws1, Ws3 1/sqrt(d); W2 1/sqrt(d_ff), Ws2
    1/sqrt(d_ff_shared) -- so router logits are close to N(0, 1).

Layouts are those of ``nn.Linear.weight`` ([out, in], row-major):
x [T,d], Wg [E,d], W1/W3 [E,d_ff,d], W2 [E,d,d_ff], Ws1/Ws3 [d_ffs,d],
Ws2 [d,d_ffs].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

#: Rows of x drawn per slice.
_X_ROWS_PER_SLICE = 4096

#: Router bias used for the skewed-load Mixtral prefill workload: this much
#: is added to one expert's logit.  For 8 iid N(0,1) logits a shift of 1.1
#: makes one expert the top-1 choice about 42% of the time (a property of
#: Gaussians, computed by Monte Carlo); the share actually reached is measured
#: from the routing output of each run.
SKEW_BIAS = 1.1
SKEW_EXPERT = 3


@dataclass(frozen=True)
class Workload:
    """Shapes of one MoE layer invocation."""

    name: str
    T: int
    d: int
    E: int
    d_ff: int
    k: int
    d_ff_shared: int = 0
    skew: bool = False
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def S(self) -> int:
        return self.T * self.k


def small() -> Workload:
    """Small layer whose oracle finishes in seconds."""
    return Workload("small_T512_d512_E8_dff4096_k2", 512, 512, 8, 4096, 2)


#: (E, d_ff, k) of the fixed-total-parameter granularity sweep: d = 512,
#: E * d_ff = 32768 (3*d*E*d_ff = 50.3M parameters), T = 512 tokens.
SWEEP = ((8, 4096, 1), (8, 4096, 2), (32, 1024, 1), (32, 1024, 2), (64, 512, 4), (128, 256, 8))


def sweep() -> list[Workload]:
    return [Workload(f"sweep_T512_d512_E{E}_dff{f}_k{k}", 512, 512, E, f, k) for (E, f, k) in SWEEP]


def mixtral_prefill(T: int, skew: bool = False) -> Workload:
    return Workload(f"mixtral_prefill_T{T}{'_skewed' if skew else ''}", T, 4096, 8, 14336, 2,
                    skew=skew)


def mixtral_decode(T: int) -> Workload:
    return Workload(f"mixtral_decode_T{T}", T, 4096, 8, 14336, 2)


def fine_grained(T: int = 8192, E: int = 256) -> Workload:
    """d = 7168, E routed experts of d_ff = 2048, top-8, one shared expert of
    d_ff = 2048.  E = 256 is the configuration; fewer experts with T scaled by
    E/256 keep its rows per expert (for profiling captures that must stay
    small)."""
    return Workload(f"fine_grained_T{T}_E{E}_k8_shared", T, 7168, E, 2048, 8, d_ff_shared=2048)


def router_bias(wl: Workload, device="cpu") -> torch.Tensor | None:
    """fp32 [E] router bias of a workload (None unless it is the skewed one)."""
    if not wl.skew:
        return None
    b = torch.zeros(wl.E, dtype=torch.float32, device=device)
    b[SKEW_EXPERT] = SKEW_BIAS
    return b


def _draw(g: torch.Generator, shape, sigma: float, device, rows_per_slice: int) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    lead = shape[0]
    for s in range(0, lead, rows_per_slice):
        e = min(lead, s + rows_per_slice)
        sl = torch.randn((e - s,) + tuple(shape[1:]), generator=g, dtype=torch.float32,
                         device=device)
        out[s:e] = (sl * sigma).to(torch.bfloat16)
    return out


def make_inputs(wl: Workload, seed: int = 42, device="cpu") -> dict:
    """Draw every input tensor of ``wl`` (bf16), plus the fp32 router bias."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    T, d, E, f = wl.T, wl.d, wl.E, wl.d_ff
    out = {
        "x": _draw(g, (T, d), 1.0, device, _X_ROWS_PER_SLICE),
        "Wg": _draw(g, (E, d), 1.0 / math.sqrt(d), device, E),
        "W1": _draw(g, (E, f, d), 1.0 / math.sqrt(d), device, 1),
        "W3": _draw(g, (E, f, d), 1.0 / math.sqrt(d), device, 1),
        "W2": _draw(g, (E, d, f), 1.0 / math.sqrt(f), device, 1),
    }
    if wl.d_ff_shared:
        fs = wl.d_ff_shared
        out["Ws1"] = _draw(g, (fs, d), 1.0 / math.sqrt(d), device, fs)
        out["Ws3"] = _draw(g, (fs, d), 1.0 / math.sqrt(d), device, fs)
        out["Ws2"] = _draw(g, (d, fs), 1.0 / math.sqrt(fs), device, d)
    out["bias"] = router_bias(wl, device)
    return out


def bits(t: torch.Tensor):
    """Raw bf16 bits of a tensor as a host numpy uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def shard_tokens(T: int, rank: int, world: int) -> tuple[int, int]:
    """[start, end) of the tokens that ``rank`` owns when T tokens are split
    across ``world`` data-parallel ranks as evenly as possible."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, rem = divmod(T, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s independent batch under weak scaling."""
    return seed + 1000003 * rank


def make_fp8_experts(wl: Workload, seed: int = 42, device="cpu", pow2_scales: bool = False) -> dict:
    """Seeded FP8 expert weights of ``wl``'s shapes: the bf16 recipe's normal
    draws (W1, W3 with sigma 1/sqrt(d), W2 with 1/sqrt(d_ff), drawn after x
    and Wg from the same seeded generator), each weight row stored as e4m3
    codes (torch.float8_e4m3fn, round to nearest even) and one fp32 scale,
    scale = max|row| / 448 (rounded up to a power of two when
    ``pow2_scales``), so that no code overflows the format.  Returns x, Wg (bf16, as make_inputs), q1, q3 [E,d_ff,d]
    and q2 [E,d,d_ff] as uint8 code tensors, s1, s3 [E,d_ff] and s2 [E,d]
    fp32, and the router bias."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    T, d, E, f = wl.T, wl.d, wl.E, wl.d_ff
    out = {
        "x": _draw(g, (T, d), 1.0, device, _X_ROWS_PER_SLICE),
        "Wg": _draw(g, (E, d), 1.0 / math.sqrt(d), device, E),
    }
    for name, shape, sigma in (("1", (E, f, d), 1.0 / math.sqrt(d)),
                               ("3", (E, f, d), 1.0 / math.sqrt(d)),
                               ("2", (E, d, f), 1.0 / math.sqrt(f))):
        q = torch.empty(shape, dtype=torch.uint8, device=device)
        sc = torch.empty(shape[:2], dtype=torch.float32, device=device)
        for e in range(shape[0]):
            w = torch.randn(shape[1:], generator=g, dtype=torch.float32, device=device) * sigma
            s = w.abs().amax(dim=1).clamp_min(1e-30) / 448.0
            if pow2_scales:
                s = torch.exp2(torch.ceil(torch.log2(s)))
            q[e] = (w / s[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
            sc[e] = s
        out["q" + name] = q
        out["s" + name] = sc
    out["bias"] = router_bias(wl, device)
    return out


def fp8_dequant_bf16(q: torch.Tensor, s: torch.Tensor) -> torch.Tensor:
    """bf16 tensor of scale * e4m3(code) (exact when the scales are powers of
    two and the products in range), for checks only."""
    v = q.view(torch.float8_e4m3fn).to(torch.float32) * s[..., None]
    return v.to(torch.bfloat16)
