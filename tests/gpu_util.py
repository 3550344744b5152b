"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle under the stated tolerances.

Tolerances (floating point): max|gpu - ref| / max|ref| <= 2e-2 and
sum|gpu - ref| / sum|ref| <= 5e-3 over every compared element; routing
indices and per-expert counts bit-exact except for tokens whose k-th and
(k+1)-th oracle logits are closer than 1e-3, which are counted and compared
against the oracle re-evaluated with the GPU's experts.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import synth
from sparse_mixture_experts_histogram_b200.synth import bits

MAX_REL = 2e-2
MEAN_REL = 5e-3
NEAR_TIE = 1e-3


def rel_errors(got: np.ndarray, ref: np.ndarray) -> tuple[float, float]:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(got - ref)
    mx = float(d.max() / max(np.abs(ref).max(), 1e-300))
    mean = float(d.sum() / max(np.abs(ref).sum(), 1e-300))
    return mx, mean


def assert_close(got, ref, what=""):
    mx, mean = rel_errors(got, ref)
    assert np.isfinite(np.asarray(got)).all(), f"{what}: non-finite output"
    assert mx <= MAX_REL and mean <= MEAN_REL, f"{what}: max_rel={mx:.3e} mean_rel={mean:.3e}"
    return mx, mean


def workspace(wl, device="cuda"):
    n = moe.moe_workspace_size_ex(wl.T, wl.d, wl.E, wl.d_ff, wl.k, wl.d_ff_shared)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device=device)


def gpu_route(wl, inp):
    dev = inp["x"].device
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.k, dtype=torch.float32, device=dev)
    counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
    ws = workspace(wl)
    moe.moe_route(wl.T, wl.d, wl.E, wl.k, inp["x"], inp["Wg"], inp["bias"], idx, w, counts, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 0, f"device error word {code:#x}"
    return idx.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()


def gpu_forward(wl, inp, ws=None):
    dev = inp["x"].device
    out = torch.empty(wl.T, wl.d, dtype=torch.float32, device=dev)
    ws = workspace(wl) if ws is None else ws
    moe.moe_forward_ex(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"], inp["bias"],
                       inp["W1"], inp["W3"], inp["W2"], wl.d_ff_shared, inp.get("Ws1"),
                       inp.get("Ws3"), inp.get("Ws2"), out, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 0, f"device error word {code:#x}"
    return out


def oracle_route(wl, inp):
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    return oracle.route(bits(inp["x"]), bits(inp["Wg"]), wl.k, bias=bias)


def check_routing(wl, inp, r=None):
    """GPU routing vs the oracle.  Returns (gpu idx, oracle route, near-tie mask).

    Tokens whose k-th and (k+1)-th oracle logits are closer than 1e-3 are
    near ties: their selected set may differ and is only counted.  For every
    other token the selected SET must equal the oracle's exactly.  The slot
    order must follow the oracle's logits wherever two selected logits differ
    by at least 1e-3; closer pairs may come in either order (fp32 logits
    cannot order them), and the weights are compared expert by expert.
    """
    r = oracle_route(wl, inp) if r is None else r
    idx, w, counts = gpu_route(wl, inp)
    near = r["gap"] < NEAR_TIE
    far = ~near
    gs, os_ = np.sort(idx, 1), np.sort(r["idx"], 1)
    assert np.array_equal(gs[far], os_[far]), (
        f"expert sets differ on {int((gs[far] != os_[far]).any(1).sum())} non-near-tie tokens")
    L = r["logits"]
    lg = np.take_along_axis(L, idx.astype(np.int64), 1)  # oracle logits in GPU slot order
    for a in range(wl.k):
        for b in range(a + 1, wl.k):
            bad = far & (lg[:, b] > lg[:, a] + NEAR_TIE)
            assert not bad.any(), f"slot order contradicts the logits on {int(bad.sum())} tokens"
    if far.any():
        og = np.argsort(idx, 1)
        oo = np.argsort(r["idx"], 1)
        wg = np.take_along_axis(w, og, 1)
        wo = np.take_along_axis(r["w"], oo, 1)
        assert np.max(np.abs(wg[far] - wo[far])) < 2e-4
    assert np.allclose(w.sum(1), 1.0, atol=1e-5)
    # Counts: the GPU histogram is its own idx's histogram, and it equals the
    # oracle's over the tokens that are not near ties.
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=wl.E))
    assert np.array_equal(np.bincount(idx[far].ravel(), minlength=wl.E),
                          np.bincount(r["idx"][far].ravel(), minlength=wl.E))
    assert all(len(set(row)) == wl.k for row in idx)
    return idx, r, near


def check_forward(wl, inp, tokens=None, r=None):
    """Whole layer vs the oracle on ``tokens`` (default: all)."""
    idx, r, near = check_routing(wl, inp, r)
    out = gpu_forward(wl, inp).cpu().numpy().astype(np.float64)
    tok = np.arange(wl.T) if tokens is None else np.asarray(tokens)
    shared = None
    if wl.d_ff_shared:
        shared = (bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"]))
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    forced = idx[tok]
    # Only the experts the compared tokens use travel to the host: the oracle
    # gets those experts' matrices and router rows, with the forced expert
    # indices renumbered accordingly (the softmax still runs over the same
    # logits, so nothing it computes changes).
    used = np.unique(forced)
    remap = np.full(wl.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    sel = torch.as_tensor(used, device=inp["W1"].device)
    ref = oracle.forward(bits(inp["x"]), bits(inp["Wg"][sel]), bits(inp["W1"][sel]),
                         bits(inp["W3"][sel]), bits(inp["W2"][sel]), wl.k,
                         bias=None if bias is None else bias[used], tokens=tok, shared=shared,
                         forced=remap[forced].astype(np.int32))
    mx, mean = assert_close(out[tok], ref, wl.name)
    return {"max_rel": mx, "mean_rel": mean, "near_ties": int(near.sum()), "tokens": len(tok)}


def sample_tokens(T, n, idx=None, near=None, seed=0):
    """A seeded sample of n tokens that also holds every near-tie token and at
    least one token of every expert the batch hits."""
    g = np.random.default_rng(seed)
    chosen = set(g.choice(T, size=min(n, T), replace=False).tolist())
    if near is not None:
        chosen |= set(np.nonzero(near)[0].tolist())
    if idx is not None:
        for e in np.unique(idx):
            if not any(e in idx[t] for t in chosen):
                chosen.add(int(np.nonzero((idx == e).any(1))[0][0]))
    return np.array(sorted(chosen))


def gpu_forward_variant(wl, inp, variant, ws=None):
    dev = inp["x"].device
    out = torch.empty(wl.T, wl.d, dtype=torch.float32, device=dev)
    ws = workspace(wl) if ws is None else ws
    moe.moe_forward_variant(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"], inp["bias"],
                            inp["W1"], inp["W3"], inp["W2"], wl.d_ff_shared, inp.get("Ws1"),
                            inp.get("Ws3"), inp.get("Ws2"), variant, out, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 0, f"device error word {code:#x}"
    return out


def check_forward_variant(wl, inp, variant, tokens=None):
    """Whole layer under a variant (weights, activation, capacity_factor) vs
    the oracle with the same variant.  Routing is checked as for the method;
    the oracle takes the GPU's selection for the compared tokens (identical
    outside near ties) and, for the capacity ranks, for all tokens."""
    weights, act, cf = variant
    idx, r, near = check_routing(wl, inp)
    out = gpu_forward_variant(wl, inp, variant).cpu().numpy().astype(np.float64)
    tok = np.arange(wl.T) if tokens is None else np.asarray(tokens)
    shared = None
    if wl.d_ff_shared:
        shared = (bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"]))
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    cap = oracle.capacity_limit(cf, wl.T, wl.k, wl.E) if cf > 0 else None
    ref = oracle.forward(bits(inp["x"]), bits(inp["Wg"]), bits(inp["W1"]), bits(inp["W3"]),
                         bits(inp["W2"]), wl.k, bias=bias, tokens=tok, shared=shared,
                         forced=idx[tok], w_mode=weights, act_mode=act, capacity=cap,
                         route_all=idx if cap is not None else None)
    mx, mean = assert_close(out[tok], ref, f"{wl.name} variant {variant}")
    return {"max_rel": mx, "mean_rel": mean, "near_ties": int(near.sum()), "cap": cap}
