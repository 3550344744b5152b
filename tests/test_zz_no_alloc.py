"""moe_expert_ffn_static -- the expert FFN for callers that cannot allocate
device memory (a plugin given only its tensors, a loop that must stay out of
the allocator) -- must give what moe_expert_ffn gives with a caller-owned
workspace, and what the fp64 oracle gives.  Kept in its own file, collected
last, and written to pass both alone in a fresh process and after every
other test."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import synth
from sparse_mixture_experts_histogram_b200.synth import Workload, bits

from gpu_util import assert_close

DEV = "cuda"


def _segments_inputs(sizes, d, d_ff, seed):
    E, S = len(sizes), int(sum(sizes))
    wl = Workload("no_alloc", S, d, E, d_ff, 1)
    inp = {k: (None if v is None else v.to(DEV)) for k, v in
           synth.make_inputs(wl, seed=seed, device="cpu").items()}
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    return wl, inp, offsets


@pytest.mark.gpu
def test_static_scratch_ffn_matches_workspace_ffn_and_oracle_twice():
    sizes = [37, 0, 128, 1, 200, 64]
    d, d_ff = 384, 640
    wl, inp, offsets = _segments_inputs(sizes, d, d_ff, seed=5)
    S, E = wl.T, wl.E
    d_off = torch.as_tensor(offsets, device=DEV)
    ws = torch.empty(moe.moe_workspace_size(S, d, E, d_ff, 1), dtype=torch.uint8, device=DEV)
    ref = torch.empty(S, d, dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(S, d, E, d_ff, inp["x"], d_off, inp["W1"], inp["W3"], inp["W2"], ref, ws)
    assert moe.moe_get_device_error(ws)[0] == 0
    ref = ref.cpu().numpy()
    xb = bits(inp["x"])
    exact = [oracle.swiglu(xb[offsets[e]:offsets[e + 1]], bits(inp["W1"][e]), bits(inp["W3"][e]),
                           bits(inp["W2"][e])) for e in range(E)]
    for call in range(2):
        y = torch.full((S, d), float("nan"), dtype=torch.float32, device=DEV)
        moe.moe_expert_ffn_static(S, d, E, d_ff, inp["x"], d_off, inp["W1"], inp["W3"],
                                  inp["W2"], y)
        st, code = moe.moe_expert_ffn_static_error()
        assert st == 0, f"call {call}: static error word {code:#x}"
        y = y.cpu().numpy()
        assert_close(y, ref, f"static-scratch call {call} vs moe_expert_ffn")
        for e in range(E):
            if sizes[e]:
                assert_close(y[offsets[e]:offsets[e + 1]], exact[e],
                             f"static-scratch call {call}, expert {e} vs oracle")


@pytest.mark.gpu
def test_static_scratch_largest_size_that_fits():
    # The largest S whose scratch need (error word, counters, H) fits the
    # fixed array runs; one row more is refused before anything is launched.
    d, d_ff, E = 128, 128, 1
    cap = 32 << 20
    S = max(s for s in range(130000, 132000) if moe.moe_expert_ffn_static_bytes(s, E, d_ff) <= cap)
    assert moe.moe_expert_ffn_static_bytes(S + 1, E, d_ff) > cap
    g = torch.Generator(device=DEV).manual_seed(3)
    x = (torch.randn(S + 1, d, generator=g, device=DEV)).to(torch.bfloat16)
    W1 = (torch.randn(1, d_ff, d, generator=g, device=DEV) / d ** 0.5).to(torch.bfloat16)
    W3 = (torch.randn(1, d_ff, d, generator=g, device=DEV) / d ** 0.5).to(torch.bfloat16)
    W2 = (torch.randn(1, d, d_ff, generator=g, device=DEV) / d_ff ** 0.5).to(torch.bfloat16)
    off = torch.tensor([0, S], dtype=torch.int32, device=DEV)
    y = torch.full((S, d), float("nan"), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn_static(S, d, E, d_ff, x, off, W1, W3, W2, y)
    assert moe.moe_expert_ffn_static_error()[0] == 0
    ws = torch.empty(moe.moe_workspace_size(S, d, E, d_ff, 1), dtype=torch.uint8, device=DEV)
    ref = torch.empty(S, d, dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(S, d, E, d_ff, x, off, W1, W3, W2, ref, ws)
    assert moe.moe_get_device_error(ws)[0] == 0
    assert_close(y.cpu().numpy(), ref.cpu().numpy(), "static-scratch at its largest size")
    off1 = torch.tensor([0, S + 1], dtype=torch.int32, device=DEV)
    y1 = torch.empty(S + 1, d, dtype=torch.float32, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_expert_ffn_static(S + 1, d, E, d_ff, x, off1, W1, W3, W2, y1)
    assert ei.value.status == 3
