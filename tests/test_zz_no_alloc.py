"""moe_expert_ffn_static -- the expert FFN for callers that cannot allocate
device memory (a plugin given only its tensors, a loop that must stay out of
the allocator) -- must give what moe_expert_ffn gives with a caller-owned
workspace.  Kept in its own file, collected last, and written to pass both
alone in a fresh process and after every other test."""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import synth
from sparse_mixture_experts_histogram_b200.synth import Workload

from gpu_util import assert_close

DEV = "cuda"


@pytest.mark.gpu
def test_static_scratch_ffn_matches_workspace_ffn_twice():
    sizes = [37, 0, 128, 1, 200, 64]
    E, d, d_ff = len(sizes), 384, 640
    S = sum(sizes)
    wl = Workload("no_alloc", S, d, E, d_ff, 1)
    inp = {k: (None if v is None else v.to(DEV)) for k, v in
           synth.make_inputs(wl, seed=5, device="cpu").items()}
    offsets = torch.as_tensor(np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32),
                              device=DEV)
    ws = torch.empty(moe.moe_workspace_size(S, d, E, d_ff, 1), dtype=torch.uint8, device=DEV)
    ref = torch.empty(S, d, dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(S, d, E, d_ff, inp["x"], offsets, inp["W1"], inp["W3"], inp["W2"], ref, ws)
    assert moe.moe_get_device_error(ws)[0] == 0
    for call in range(2):
        y = torch.full((S, d), float("nan"), dtype=torch.float32, device=DEV)
        moe.moe_expert_ffn_static(S, d, E, d_ff, inp["x"], offsets, inp["W1"], inp["W3"],
                                  inp["W2"], y)
        torch.cuda.synchronize()
        assert_close(y.cpu().numpy(), ref.cpu().numpy(), f"static-scratch call {call}")


@pytest.mark.gpu
def test_static_scratch_rejects_sizes_over_its_limit():
    # 4096 rows x 4096 hidden x 2 bytes = 32 MiB > 32 MiB - 256: refused on
    # the host, before anything is launched.
    lib = moe.load_library()
    fake = 1 << 20
    st = lib.moe_expert_ffn_static(4096, 512, 8, 4096, fake, fake, fake, fake, fake, fake, None)
    assert st == 3
