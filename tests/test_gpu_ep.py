"""GPU parity of the expert-parallel layer (experts split over R ranks), run
as R emulated ranks on one GPU: the same kernels and buffers as the
multi-process layer, with stream order in place of the collectives.

Checked against the oracle: the receive layout (every pair's receive row and
every owner's segment starts, bit-exact against ``oracle.ep_plan`` on the
GPU's routing), the rows that arrive (bit-exact copies of x), and each
rank's output (the layer's oracle output of that rank's tokens, under the
tolerances of tests/gpu_util.py)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import ep, synth
from sparse_mixture_experts_histogram_b200.synth import Workload, bits

from gpu_util import assert_close, check_routing, sample_tokens

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run(name, R, Ts, d, E, d_ff, k, d_ff_shared=0, bias=None, seed=7):
    """Draws one batch of sum(Ts) tokens, splits it over R ranks, runs the
    emulated layer.  Returns (layer, inputs, per-rank x, per-rank out)."""
    wl = Workload(name, sum(Ts), d, E, d_ff, k, d_ff_shared=d_ff_shared)
    inp = {kk: (None if v is None else v.to(DEV))
           for kk, v in synth.make_inputs(wl, seed=seed, device="cpu").items()}
    if bias is not None:
        inp["bias"] = bias.to(DEV)
    starts = np.concatenate([[0], np.cumsum(Ts)])
    xs = [inp["x"][starts[r]:starts[r + 1]] for r in range(R)]
    outs = [torch.full((Ts[r], d), float("nan"), device=DEV) for r in range(R)]
    layer = ep.EmulatedExpertParallel(R, max(Ts), d, E, d_ff, k, d_ff_shared, device=DEV)
    shared = (inp["Ws1"], inp["Ws3"], inp["Ws2"]) if d_ff_shared else None
    layer.forward(xs, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], outs,
                  router_bias=inp["bias"], shared=shared)
    torch.cuda.synchronize()
    assert layer.device_errors() == [0] * R
    return layer, inp, xs, outs


def _check_layout(layer, xs):
    """pos / recv_offsets bit-exact against the oracle's plan on the GPU's
    routing, and every received row a bit-exact copy of its token."""
    p = layer.plan
    idx = [b.idx[:x.shape[0]].cpu().numpy() for b, x in zip(layer.ranks, xs)]
    pos_ref, off_ref = oracle.ep_plan(idx, p.E, p.R)
    for r, b in enumerate(layer.ranks):
        assert np.array_equal(b.pos[:xs[r].shape[0]].cpu().numpy(), pos_ref[r]), f"pos of rank {r}"
        assert np.array_equal(b.recv_offsets.cpu().numpy(), off_ref[r]), f"segments of rank {r}"
    recv = [bits(b.recv_x) for b in layer.ranks]
    for r, x in enumerate(xs):
        xb = bits(x)
        owner = idx[r] // p.El
        for q in range(p.R):
            t, j = np.nonzero(owner == q)
            assert np.array_equal(recv[q][pos_ref[r][t, j]], xb[t]), f"rows {r} -> {q}"
    return idx


def _check_outputs(layer, inp, xs, outs, idx, tokens_per_rank=None, d_ff_shared=0):
    p = layer.plan
    shared = None
    if d_ff_shared:
        shared = (bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"]))
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    res = []
    for r, x in enumerate(xs):
        T = x.shape[0]
        if T == 0:
            continue  # a rank with no tokens: nothing to compare
        wl = Workload(f"rank{r}", T, p.d, p.E, p.d_ff, p.k)
        rin = {"x": x, "Wg": inp["Wg"], "bias": inp["bias"]}
        gidx, rr, near = check_routing(wl, rin)
        assert np.array_equal(gidx, idx[r]), "the layer's routing is moe_route's"
        tok = np.arange(T) if tokens_per_rank is None else sample_tokens(
            T, tokens_per_rank, idx[r], near, seed=r)
        ref = oracle.forward(bits(x), bits(inp["Wg"]), bits(inp["W1"]), bits(inp["W3"]),
                             bits(inp["W2"]), p.k, bias=bias, tokens=tok, shared=shared,
                             forced=idx[r][tok])
        got = outs[r].cpu().numpy().astype(np.float64)[tok]
        res.append(assert_close(got, ref, f"rank {r}"))
    return res


EP_CASES = [
    # name, R, per-rank tokens (ragged), d, E, d_ff, k, d_ff_shared
    ("R1_E8_k2", 1, [200], 512, 8, 1024, 2, 0),
    ("R2_E8_k2", 2, [300, 251], 512, 8, 1024, 2, 0),
    ("R4_E8_k2", 4, [128, 1, 77, 128], 1024, 8, 512, 2, 0),
    ("R8_E8_k1", 8, [33] * 7 + [5], 256, 8, 384, 1, 0),
    ("R8_E64_k8_shared", 8, [96, 95, 64, 1, 96, 30, 96, 50], 1024, 64, 256, 8, 256),
    ("R4_E16_k3", 4, [160, 129, 100, 7], 384, 16, 640, 3, 0),
    # a rank with no tokens this step: it sends nothing and still serves its experts
    ("R4_E8_k2_empty_rank", 4, [100, 0, 57, 80], 512, 8, 512, 2, 0),
]


@pytest.mark.parametrize("case", EP_CASES, ids=lambda c: c[0])
def test_ep_matches_oracle(case):
    name, R, Ts, d, E, d_ff, k, dfs = case
    layer, inp, xs, outs = _run(name, R, Ts, d, E, d_ff, k, dfs)
    idx = _check_layout(layer, xs)
    _check_outputs(layer, inp, xs, outs, idx, d_ff_shared=dfs)


def test_ep_decode_splits_the_down_projection():
    """Decode-sized batches (8 tokens per rank, one expert per rank): the
    owners' expert kernel splits K of W2 and the combine sums the partials."""
    R, Ts, d, E, d_ff, k = 8, [8] * 8, 4096, 8, 4096, 2
    layer, inp, xs, outs = _run("ep_decode", R, Ts, d, E, d_ff, k)
    assert layer.plan.ksplit > 1
    idx = _check_layout(layer, xs)
    _check_outputs(layer, inp, xs, outs, idx, tokens_per_rank=3)


def test_ep_prefill_tiles():
    """Prefill-sized segments (about 1000 rows per expert): the owners run
    the CTA-pair expert kernel and hand back bf16 rows."""
    R, Ts, d, E, d_ff, k = 2, [1024, 1000], 2048, 4, 1024, 2
    layer, inp, xs, outs = _run("ep_prefill", R, Ts, d, E, d_ff, k)
    assert layer.plan.ksplit == 1 and layer.plan.y_bf16   # complete rows come back as bf16
    idx = _check_layout(layer, xs)
    _check_outputs(layer, inp, xs, outs, idx, tokens_per_rank=48)


def test_ep_one_owner_takes_every_row():
    """A router bias sends every token to experts 0 and 1, both owned by rank
    0: its receive buffer fills to exactly its capacity, the others get
    nothing."""
    R, Ts, d, E, d_ff, k = 4, [64, 64, 64, 64], 256, 8, 256, 2
    bias = torch.zeros(E)
    bias[0] = bias[1] = 30.0   # logits are about N(0, 1): 30 decides the top two
    layer, inp, xs, outs = _run("ep_skew", R, Ts, d, E, d_ff, k, bias=bias)
    off = [b.recv_offsets.cpu().numpy() for b in layer.ranks]
    assert off[0][-1] == layer.plan.recv_rows == sum(Ts) * k
    assert all(o[-1] == 0 for o in off[1:])
    idx = _check_layout(layer, xs)
    _check_outputs(layer, inp, xs, outs, idx)


def test_ep_matches_single_gpu_layer():
    """The split layer and moe_forward_ex give the same output on the same
    tokens, up to the order of the fp32 additions."""
    R, Ts, d, E, d_ff, k = 4, [100, 100, 100, 100], 512, 8, 512, 2
    layer, inp, xs, outs = _run("ep_vs_single", R, Ts, d, E, d_ff, k)
    T = sum(Ts)
    full = torch.empty(T, d, device=DEV)
    ws = torch.empty(moe.moe_workspace_size(T, d, E, d_ff, k), dtype=torch.uint8, device=DEV)
    moe.moe_forward_ex(T, d, E, d_ff, k, inp["x"], inp["Wg"], None, inp["W1"], inp["W3"],
                       inp["W2"], 0, None, None, None, full, ws)
    got = torch.cat(outs).cpu().numpy().astype(np.float64)
    assert_close(got, full.cpu().numpy().astype(np.float64), "EP vs single GPU")


def test_ep_repeatable():
    """Every row's place follows from the routing: two calls give the same bits."""
    R, Ts, d, E, d_ff, k = 4, [90, 60, 128, 3], 512, 16, 256, 4
    layer, inp, xs, outs = _run("ep_repeat", R, Ts, d, E, d_ff, k)
    first = [o.clone() for o in outs]
    layer.forward(xs, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], outs)
    torch.cuda.synchronize()
    for a, b in zip(first, outs):
        assert torch.equal(a, b)


def test_ep_dispatch_rejects_inconsistent_counts():
    """A counts table whose own row disagrees with idx: the dispatch sets
    MOE_DEVERR_EP_COUNTS, sends nothing and marks every slot -1."""
    R, T, d, E, k = 2, 64, 256, 8, 2
    layer = ep.EmulatedExpertParallel(R, T, d, E, 256, k, device=DEV)
    p, b = layer.plan, layer.ranks[0]
    wl = Workload("ep_bad_counts", T, d, E, 256, k)
    inp = {kk: (None if v is None else v.to(DEV))
           for kk, v in synth.make_inputs(wl, seed=3, device="cpu").items()}
    moe.moe_route(T, d, E, k, inp["x"], inp["Wg"], None, b.idx, b.w, b.counts, b.route_ws)
    counts_all = torch.stack([b.counts, b.counts])
    counts_all[0, 0] += 1
    b.recv_x.zero_()
    moe.moe_ep_dispatch(T, d, E, k, R, 0, inp["x"], b.idx, counts_all,
                        [r.recv_x for r in layer.ranks], p.recv_rows, b.pos, b.recv_offsets, b.ws)
    st, code = moe.moe_get_device_error(b.ws)
    assert code & 0x40
    assert (b.pos[:T] == -1).all()
    assert not b.recv_x.any()


_ONE_RANK = r'''
import datetime, os, sys
import numpy as np, torch, torch.distributed as dist
sys.path.insert(0, os.environ["REPO"])
from sparse_mixture_experts_histogram_b200 import ep, synth
from sparse_mixture_experts_histogram_b200.synth import Workload
torch.cuda.set_device(0)
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:" + os.environ["PORT"], rank=0,
                        world_size=1, timeout=datetime.timedelta(seconds=60))
try:
    wl = Workload("ep_nccl", 200, 512, 8, 512, 2, d_ff_shared=256)
    inp = {k: (None if v is None else v.cuda()) for k, v in synth.make_inputs(wl, seed=5).items()}
    layer = ep.ExpertParallelLayer(256, 512, 8, 512, 2, inp["Wg"], inp["W1"], inp["W3"], inp["W2"],
                                   shared=(inp["Ws1"], inp["Ws3"], inp["Ws2"]))
    out = torch.empty(200, 512, device="cuda")
    for _ in range(2):
        layer.forward(inp["x"], out)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    np.savez(os.environ["OUT"], out=out.cpu().numpy(), idx=layer.buf.idx[:200].cpu().numpy())
    layer.close()
finally:
    dist.destroy_process_group()
'''


def test_ep_layer_over_nccl_with_one_rank(tmp_path):
    """The multi-process layer (its NCCL all-gather and barriers, a world of
    one GPU) against the oracle, shared expert included."""
    import os
    import socket
    import subprocess
    import sys
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out_file = str(tmp_path / "ep_one_rank.npz")
    env = dict(os.environ, REPO=root, PORT=str(port), OUT=out_file, NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", _ONE_RANK], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.load(out_file)
    wl = Workload("ep_nccl", 200, 512, 8, 512, 2, d_ff_shared=256)
    inp = synth.make_inputs(wl, seed=5)
    ref = oracle.forward(bits(inp["x"]), bits(inp["Wg"]), bits(inp["W1"]), bits(inp["W3"]),
                         bits(inp["W2"]), 2,
                         shared=(bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"])),
                         forced=got["idx"])
    assert_close(got["out"].astype(np.float64), ref, "EP over NCCL, one rank")


_TWO_PROCS = r'''
import datetime, os, sys
import numpy as np, torch, torch.distributed as dist
sys.path.insert(0, os.environ["REPO"])
from sparse_mixture_experts_histogram_b200 import ep, synth
from sparse_mixture_experts_histogram_b200.synth import Workload
rank, R = int(os.environ["RANK"]), 2
torch.cuda.set_device(0)
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:" + os.environ["PORT"], rank=rank,
                        world_size=R, timeout=datetime.timedelta(seconds=60))
try:
    Ts = [150, 97]
    wl = Workload("ep_ipc", sum(Ts), 512, 8, 512, 2, d_ff_shared=256)
    inp = {k: (None if v is None else v.cuda()) for k, v in synth.make_inputs(wl, seed=9).items()}
    lo, hi = ep.expert_block(8, R, rank)
    x = inp["x"][sum(Ts[:rank]):sum(Ts[:rank + 1])]
    layer = ep.ExpertParallelLayer(160, 512, 8, 512, 2, inp["Wg"], inp["W1"][lo:hi],
                                   inp["W3"][lo:hi], inp["W2"][lo:hi],
                                   shared=(inp["Ws1"], inp["Ws3"], inp["Ws2"]))
    assert layer.host_ordered and len(layer._opened) >= 1
    out = torch.empty(x.shape[0], 512, device="cuda")
    for _ in range(3):
        layer.forward(x, out)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    n = x.shape[0]
    np.savez(os.environ["OUT"] + f".{rank}.npz", out=out.cpu().numpy(),
             idx=layer.buf.idx[:n].cpu().numpy(), pos=layer.buf.pos[:n].cpu().numpy(),
             seg=layer.buf.recv_offsets.cpu().numpy())
    layer.close()
finally:
    dist.destroy_process_group()
'''


def test_ep_layer_two_processes_one_gpu_over_ipc(tmp_path):
    """Two processes on one GPU, each one rank of the split layer: the peer
    buffers are mapped across the processes with CUDA IPC (moe_ipc_*), the
    dispatch stores into the other process's receive buffer and the combine
    reads the other's output buffer; a gloo group orders the steps on the
    host (no kernel waits on the other process).  Layout against the
    oracle's plan, outputs against the oracle layer."""
    import os
    import socket
    import subprocess
    import sys
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    base = str(tmp_path / "ep_ipc")
    procs = [subprocess.Popen([sys.executable, "-c", _TWO_PROCS], stdout=subprocess.PIPE,
                              stderr=subprocess.PIPE, text=True,
                              env=dict(os.environ, REPO=root, PORT=str(port), OUT=base,
                                       RANK=str(r)))
             for r in range(2)]
    errs = []
    for p in procs:
        try:
            _, err = p.communicate(timeout=300)
        except subprocess.TimeoutExpired:
            p.kill()
            _, err = p.communicate()
        errs.append((p.returncode, err[-3000:]))
    assert all(rc == 0 for rc, _ in errs), errs
    got = [np.load(f"{base}.{r}.npz") for r in range(2)]
    pos_ref, seg_ref = oracle.ep_plan([g["idx"] for g in got], 8, 2)
    for r in range(2):
        assert np.array_equal(got[r]["pos"], pos_ref[r])
        assert np.array_equal(got[r]["seg"], seg_ref[r])
    Ts = [150, 97]
    wl = Workload("ep_ipc", sum(Ts), 512, 8, 512, 2, d_ff_shared=256)
    inp = synth.make_inputs(wl, seed=9)
    shared = (bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"]))
    for r in range(2):
        x = inp["x"][sum(Ts[:r]):sum(Ts[:r + 1])]
        ref = oracle.forward(bits(x), bits(inp["Wg"]), bits(inp["W1"]), bits(inp["W3"]),
                             bits(inp["W2"]), 2, shared=shared, forced=got[r]["idx"])
        assert_close(got[r]["out"].astype(np.float64), ref, f"rank {r} over IPC")
