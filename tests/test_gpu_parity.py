"""GPU parity: the CUDA path, called through the C ABI, against the fp64
oracle on the same seeded inputs (tolerances in tests/gpu_util.py)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import synth
from sparse_mixture_experts_histogram_b200.synth import Workload, bits

from gpu_util import (assert_close, check_forward, check_forward_variant, check_routing,
                      gpu_forward, gpu_route, sample_tokens, workspace)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(wl, seed=42, device=DEV):
    if device == DEV:
        # small workloads are drawn on the CPU (same bits as the CPU tests),
        # large ones on the GPU
        return {k: (None if v is None else v.to(DEV)) for k, v in
                synth.make_inputs(wl, seed=seed, device="cpu").items()}
    return synth.make_inputs(wl, seed=seed, device=device)


# ------------------------------------------------------------------ routing
ROUTE_CASES = [
    synth.small(),
    *synth.sweep(),
    Workload("T1_E8_k2", 1, 512, 8, 128, 2),
    Workload("T129_E64_k4", 129, 256, 64, 128, 4),
    Workload("T300_E256_k8", 300, 384, 256, 128, 8),
    Workload("T257_E5_k5", 257, 128, 5, 128, 5),
    Workload("T200_E3_k1", 200, 128, 3, 128, 1),
    Workload("T640_E17_k3", 640, 640, 17, 128, 3),
]


@pytest.mark.parametrize("wl", ROUTE_CASES, ids=lambda w: w.name)
def test_route_matches_oracle(wl):
    check_routing(wl, _inputs(wl))


# Shapes with T*E*d above 2^30 take the tensor-core router (tcgen05 MMA,
# top-k and softmax in its epilogue): ragged T, k in {1, 2, 4, 8}, E not a
# multiple of 16, with and without a router bias.
TC_ROUTE_CASES = [
    Workload("tc_T1153_d7168_E256_k8", 1153, 7168, 256, 128, 8),
    Workload("tc_T1000_d7168_E200_k1", 1000, 7168, 200, 128, 1),
    Workload("tc_T1153_d4096_E256_k2", 1153, 4096, 256, 128, 2),
    Workload("tc_T1200_d7168_E136_k4", 1200, 7168, 136, 128, 4),
    # long batch of wide rows with few experts (N = 16 on the tensor cores)
    Workload("tc_T4100_d2048_E8_k2", 4100, 2048, 8, 128, 2),
    Workload("tc_T4096_d4096_E6_k3", 4096, 4096, 6, 128, 3),
]


@pytest.mark.parametrize("with_bias", [False, True], ids=["nobias", "bias"])
@pytest.mark.parametrize("wl", TC_ROUTE_CASES, ids=lambda w: w.name)
def test_tensor_core_route_matches_oracle(wl, with_bias):
    assert wl.T * wl.E * wl.d > 2 ** 30 or (wl.T >= 4096 and wl.d >= 2048)
    inp = synth.make_inputs(wl, device=DEV)
    if with_bias:
        inp["bias"] = torch.linspace(-0.5, 0.5, wl.E, dtype=torch.float32, device=DEV)
    check_routing(wl, inp)


def test_route_equal_logits_pick_lowest_indices():
    wl = Workload("ties", 300, 256, 16, 128, 4)
    inp = _inputs(wl)
    inp["Wg"] = torch.zeros_like(inp["Wg"])
    idx, r, near = check_routing(wl, inp)
    assert (idx == np.arange(4)).all()


def test_route_skewed_bias():
    wl = synth.mixtral_prefill(2048, skew=True)
    inp = synth.make_inputs(wl, device=DEV)
    idx, r, near = check_routing(wl, inp)
    share = float((idx[:, 0] == synth.SKEW_EXPERT).mean())
    assert 0.30 < share < 0.55, share


# ------------------------------------------------------------------ permute
def _expected_dispatch(idx, E):
    T, k = idx.shape
    counts = np.bincount(idx.ravel(), minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    row = np.empty_like(idx)
    fill = offsets[:-1].copy()
    for t in range(T):                      # stable: token order within an expert
        for j in range(k):
            e = idx[t, j]
            row[t, j] = fill[e]
            fill[e] += 1
    return offsets, row


PERMUTE_CASES = [
    (Workload("T1_E8_k2", 1, 128, 8, 128, 2), "random"),
    (Workload("T129_E8_k2", 129, 256, 8, 128, 2), "random"),
    (Workload("T1000_E64_k4", 1000, 128, 64, 128, 4), "random"),
    (Workload("T700_E256_k8", 700, 256, 256, 128, 8), "random"),
    (Workload("T513_E8_k1_one_expert", 513, 128, 8, 128, 1), "one"),
    (Workload("T5_E256_k1_mostly_empty", 5, 128, 256, 128, 1), "random"),
]


@pytest.mark.parametrize("wl,mode", PERMUTE_CASES, ids=lambda c: getattr(c, "name", c))
def test_permute_matches_stable_grouping(wl, mode):
    inp = _inputs(wl)
    g = np.random.default_rng(5)
    if mode == "one":
        idx = np.full((wl.T, wl.k), 3, np.int32)
    else:
        idx = np.stack([g.choice(wl.E, size=wl.k, replace=False) for _ in range(wl.T)]).astype(np.int32)
    offsets_ref, row_ref = _expected_dispatch(idx, wl.E)
    S = wl.T * wl.k
    d_idx = torch.as_tensor(idx, device=DEV)
    offsets = torch.empty(wl.E + 1, dtype=torch.int32, device=DEV)
    row = torch.empty(wl.T, wl.k, dtype=torch.int32, device=DEV)
    xp = torch.empty(S, wl.d, dtype=torch.bfloat16, device=DEV)
    ws = workspace(wl)
    moe.moe_permute(wl.T, wl.d, wl.E, wl.k, inp["x"], d_idx, offsets, row, xp, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 0, hex(code)
    assert np.array_equal(offsets.cpu().numpy(), offsets_ref)
    assert np.array_equal(row.cpu().numpy(), row_ref)
    xb = bits(inp["x"])
    xpb = bits(xp)
    for t in range(wl.T):
        for j in range(wl.k):
            assert np.array_equal(xpb[row_ref[t, j]], xb[t])


def test_permute_flags_out_of_range_expert():
    wl = Workload("bad_idx", 64, 128, 8, 128, 2)
    inp = _inputs(wl)
    idx = np.tile(np.array([[0, 1]], np.int32), (64, 1))
    idx[5, 1] = 9  # outside [0, E)
    d_idx = torch.as_tensor(idx, device=DEV)
    offsets = torch.empty(9, dtype=torch.int32, device=DEV)
    row = torch.empty(64, 2, dtype=torch.int32, device=DEV)
    xp = torch.zeros(128, 128, dtype=torch.bfloat16, device=DEV)
    ws = workspace(wl)
    moe.moe_permute(64, 128, 8, 2, inp["x"], d_idx, offsets, row, xp, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 5 and code & 0x10
    assert row.cpu().numpy()[5, 1] == -1


def test_permute_flags_repeated_expert_and_keeps_a_bijection():
    wl = Workload("dup_idx", 40, 128, 8, 128, 3)
    inp = _inputs(wl)
    g = np.random.default_rng(9)
    idx = np.stack([g.choice(8, size=3, replace=False) for _ in range(40)]).astype(np.int32)
    idx[7, 2] = idx[7, 0]  # token 7 names one expert twice
    offsets = torch.empty(9, dtype=torch.int32, device=DEV)
    row = torch.empty(40, 3, dtype=torch.int32, device=DEV)
    xp = torch.zeros(120, 128, dtype=torch.bfloat16, device=DEV)
    ws = workspace(wl)
    moe.moe_permute(40, 128, 8, 3, inp["x"], torch.as_tensor(idx, device=DEV), offsets, row, xp,
                    ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 5 and code & 0x10
    r = row.cpu().numpy()
    assert r[7, 2] == -1
    valid = r[r >= 0]
    assert len(np.unique(valid)) == len(valid) == 119     # no two pairs share a row
    assert offsets.cpu().numpy()[-1] == 119


# ------------------------------------------------------------------ experts
FFN_SEGMENTS = [
    ("ragged", 512, 384, [0, 1, 15, 16, 17, 127, 128, 129, 300, 0, 33]),
    ("one_big", 256, 256, [700]),
    ("tiny", 128, 128, [1, 2, 3]),
    ("wide_ff", 384, 1024, [40, 0, 200, 5]),
    # a few hundred rows per segment: 256-row token tiles with ragged spills
    ("tile256", 256, 256, [300, 257, 511, 0, 256, 200, 12]),
    ("tile256_wide", 1152, 384, [520, 256, 255, 1]),
]


@pytest.mark.parametrize("name,d,d_ff,sizes", FFN_SEGMENTS, ids=lambda c: c if isinstance(c, str) else None)
def test_expert_ffn_matches_oracle(name, d, d_ff, sizes):
    E = len(sizes)
    S = int(sum(sizes))
    wl = Workload(name, S, d, E, d_ff, 1)
    inp = _inputs(wl, seed=11)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    y = torch.empty(S, d, dtype=torch.float32, device=DEV)
    ws = workspace(wl)
    moe.moe_expert_ffn(S, d, E, d_ff, inp["x"], torch.as_tensor(offsets, device=DEV), inp["W1"],
                       inp["W3"], inp["W2"], y, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 0, hex(code)
    y = y.cpu().numpy()
    xb = bits(inp["x"])
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        ref = oracle.swiglu(xb[a:b], bits(inp["W1"][e]), bits(inp["W3"][e]), bits(inp["W2"][e]))
        assert_close(y[a:b], ref, f"{name} expert {e}")


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """Failure detection without a fault: a wait (the pipelines' bounded
    wait) on a barrier phase that nothing completes gives up after its 2 s
    bound, reports MOE_ERR_TIMEOUT through the error word, and the next
    layer call on the same context still matches the oracle."""
    import time
    ws = torch.empty(4096, dtype=torch.uint8, device=DEV)
    t0 = time.time()
    moe.moe_selftest_wait_timeout(ws)
    st, code = moe.moe_get_device_error(ws)
    dt = time.time() - t0
    assert st == 6 and code & 0x2, (st, code)      # MOE_ERR_TIMEOUT, TIMEOUT_MMA
    assert 1.5 < dt < 60
    wl = Workload("after_timeout", 64, 256, 8, 256, 2)
    check_forward(wl, _inputs(wl))


def test_expert_ffn_rejects_inconsistent_offsets():
    wl = Workload("bad_offsets", 64, 128, 4, 128, 1)
    inp = _inputs(wl)
    offsets = torch.tensor([0, 40, 20, 64, 64], dtype=torch.int32, device=DEV)  # decreasing
    y = torch.full((64, 128), 7.0, dtype=torch.float32, device=DEV)
    ws = workspace(wl)
    moe.moe_expert_ffn(64, 128, 4, 128, inp["x"], offsets, inp["W1"], inp["W3"], inp["W2"], y, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 5 and code & 0x8
    assert (y == 7.0).all()  # nothing computed


# ------------------------------------------------------------------ combine
def test_combine_weighted_sum_in_slot_order():
    T, d, k = 77, 256, 3
    g = torch.Generator().manual_seed(3)
    y = torch.randn(T * k, d, generator=g)
    perm = torch.randperm(T * k, generator=g).reshape(T, k).to(torch.int32)
    w = torch.rand(T, k, generator=g)
    ys = torch.randn(T, d, generator=g)
    out = torch.empty(T, d, device=DEV)
    moe.moe_combine(T, d, k, y.to(DEV), perm.to(DEV), w.to(DEV), ys.to(DEV), out)
    torch.cuda.synchronize()
    ref = (w.double().unsqueeze(-1) * y.double()[perm.long()]).sum(1) + ys.double()
    assert_close(out.cpu().numpy(), ref.numpy(), "combine")


# ------------------------------------------------------------------ whole layer
SMALL_FORWARD = [synth.small(), *synth.sweep(),
                 Workload("dense_E1_k1", 300, 256, 1, 512, 1),
                 Workload("k_equals_E", 130, 256, 4, 256, 4),
                 Workload("T1", 1, 512, 8, 1024, 2),
                 Workload("T129_ragged", 129, 384, 16, 640, 3),
                 Workload("E256_k8_small", 200, 256, 256, 128, 8),
                 Workload("shared_small", 150, 256, 32, 256, 4, d_ff_shared=384),
                 # wide layers on the CTA-pair expert kernel with k <= 2: the
                 # down units add the gate-weighted rows into out themselves
                 Workload("wide_pair_T1100_d1152_E8_k2", 1100, 1152, 8, 512, 2),
                 Workload("wide_pair_T1200_d1152_E4_k1", 1200, 1152, 4, 256, 1)]


@pytest.mark.parametrize("wl", SMALL_FORWARD, ids=lambda w: w.name)
def test_forward_matches_oracle_all_tokens(wl):
    check_forward(wl, _inputs(wl))


def test_forward_all_tokens_one_expert():
    # a bias that sends every token to expert 2 first: one segment of T rows
    wl = Workload("one_expert", 600, 256, 8, 256, 2)
    inp = _inputs(wl)
    inp["bias"] = torch.tensor([0, 0, 50.0, 0, 0, 0, 0, 0], dtype=torch.float32, device=DEV)
    check_forward(wl, inp)


def test_forward_equal_logits_mean_of_first_k():
    wl = Workload("ties_forward", 64, 256, 8, 256, 3)
    inp = _inputs(wl)
    inp["Wg"] = torch.zeros_like(inp["Wg"])
    check_forward(wl, inp)


def test_forward_is_deterministic_and_graph_capturable():
    wl = synth.small()
    inp = _inputs(wl)
    ws = workspace(wl)
    a = gpu_forward(wl, inp, ws).clone()
    b = gpu_forward(wl, inp, ws).clone()
    assert torch.equal(a, b)
    out = torch.empty_like(a)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.moe_forward(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"], inp["W1"],
                        inp["W3"], inp["W2"], out, ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(g, stream=s):
        moe.moe_forward(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"], inp["W1"],
                        inp["W3"], inp["W2"], out, ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, a)


SIDE_STREAM_CASES = [Workload("shared_side_narrow", 300, 256, 32, 256, 4, d_ff_shared=384),
                     Workload("shared_side_wide", 300, 1152, 16, 256, 4, d_ff_shared=256)]


@pytest.mark.parametrize("wl", SIDE_STREAM_CASES, ids=lambda w: w.name)
def test_forward_shared_expert_side_stream_graph(wl):
    # The shared expert runs on the library's side stream, forked after the
    # routing and joined before the combine: the output matches the oracle,
    # repeats from call to call, and a CUDA graph captured on another stream
    # (the fork and join captured with it) replays the same bytes.
    inp = _inputs(wl)
    check_forward(wl, inp)
    ws = workspace(wl)
    a = gpu_forward(wl, inp, ws).clone()
    out = torch.empty_like(a)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def call():
        moe.moe_forward_ex(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"], inp["bias"],
                           inp["W1"], inp["W3"], inp["W2"], wl.d_ff_shared, inp["Ws1"], inp["Ws3"],
                           inp["Ws2"], out, ws, stream=s)

    with torch.cuda.stream(s):
        call()
    torch.cuda.synchronize()
    assert torch.equal(out, a)
    g = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(g, stream=s):
        call()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, a)
    assert moe.moe_get_device_error(ws)[0] == 0


@pytest.mark.parametrize("wl", [synth.sweep()[-1], Workload("E64_k4_T1000", 1000, 384, 64, 256, 4),
                                Workload("wide_pair_T1100_d1152_E8_k2", 1100, 1152, 8, 512, 2)],
                         ids=lambda w: w.name)
def test_forward_repeatable_whatever_the_order(wl):
    # Narrow layers place each expert's rows in the order the router's
    # atomics hand out positions, and wide layers with k <= 2 add each
    # token's weighted rows into out in the order their units finish; both
    # orders differ from run to run, the output must not (each row's expert
    # output is independent of its position, narrow slots are summed in
    # order, and two terms added onto zero give one sum in either order).
    inp = _inputs(wl)
    ws = workspace(wl)
    first = gpu_forward(wl, inp, ws).clone()
    for _ in range(4):
        assert torch.equal(gpu_forward(wl, inp, ws), first)
    check_forward(wl, inp)


@pytest.mark.parametrize("wl", [Workload("nonfinite_narrow", 64, 256, 8, 256, 2),
                                Workload("nonfinite_wide", 40, 1152, 8, 256, 3),
                                Workload("nonfinite_tensor_core_router", 700, 7168, 256, 128, 8)],
                         ids=lambda w: w.name)
def test_nonfinite_rows_route_in_bounds(wl):
    # Inputs are finite by construction everywhere else; a NaN or Inf row must
    # still give every slot of its token a distinct expert in [0, E) (NaN ranks
    # like -inf, ties go to the lower index), raise no device error, and leave
    # the other tokens' outputs as they were.  The first two shapes take the
    # CUDA-core router, the last (T*E*d > 2^30) the tensor-core router.
    big = wl.T * wl.E * wl.d > 2 ** 30
    inp = synth.make_inputs(wl, seed=5, device=DEV) if big else _inputs(wl, seed=5)
    bad = inp["x"].clone()
    bad[3] = float("nan")
    bad[17] = float("inf")
    inp_bad = dict(inp, x=bad)
    idx, _, counts = gpu_route(wl, inp_bad)
    assert idx.min() >= 0 and idx.max() < wl.E
    assert all(len(set(r)) == wl.k for r in idx.tolist())
    assert counts.sum() == wl.T * wl.k
    assert idx[3].tolist() == list(range(wl.k))  # every logit NaN: all tied, lowest indices win
    out_bad = gpu_forward(wl, inp_bad).cpu().numpy()
    out = gpu_forward(wl, inp).cpu().numpy()
    keep = [t for t in range(wl.T) if t not in (3, 17)]
    assert_close(out_bad[keep], out[keep], "finite tokens next to non-finite ones")


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_forward_mixtral_decode(T):
    wl = synth.mixtral_decode(T)
    inp = synth.make_inputs(wl, device=DEV)
    idx, r, near = check_routing(wl, inp)
    tok = sample_tokens(T, 12, idx, near)
    check_forward(wl, inp, tokens=tok, r=r)


@pytest.mark.parametrize("T,skew", [(2048, False), (2048, True), (8192, False), (8192, True)])
def test_forward_mixtral_prefill(T, skew):
    wl = synth.mixtral_prefill(T, skew)
    inp = synth.make_inputs(wl, device=DEV)
    idx, r, near = check_routing(wl, inp)
    tok = sample_tokens(T, 12, idx, near)
    check_forward(wl, inp, tokens=tok, r=r)


def test_forward_fine_grained_shared():
    # Sampled output check: 8 seeded tokens, every near-tie token and one
    # token of every hit expert, so each of the 256 experts' segments is
    # compared element by element at least once.
    wl = synth.fine_grained(8192)
    inp = synth.make_inputs(wl, device=DEV)
    idx, r, near = check_routing(wl, inp)
    tok = sample_tokens(wl.T, 8, idx, near)
    assert set(np.unique(idx[tok])) == set(np.unique(idx))
    check_forward(wl, inp, tokens=tok, r=r)


# ------------------------------------------------------------------ variants
# Gate-weight rules, the sigmoid-gated expert and the expert capacity (the
# variants the pages print beside the method), against the oracle with the
# same variant.  Narrow layers (d <= 1024) and wide ones, both routers.
VARIANT_ROUTE_CASES = [
    Workload("var_T300_E16_k4", 300, 256, 16, 128, 4),
    Workload("var_tc_T1153_d7168_E200_k8", 1153, 7168, 200, 128, 8),
]


@pytest.mark.parametrize("weights", [moe.WEIGHTS_SOFTMAX_ALL, moe.WEIGHTS_SIGMOID])
@pytest.mark.parametrize("wl", VARIANT_ROUTE_CASES, ids=lambda w: w.name)
def test_route_variant_weights_match_oracle(wl, weights):
    big = wl.T * wl.E * wl.d > 2 ** 30
    inp = synth.make_inputs(wl, device=DEV) if big else _inputs(wl)
    inp["bias"] = torch.linspace(-0.4, 0.4, wl.E, dtype=torch.float32, device=DEV)
    bias = inp["bias"].double().cpu().numpy()
    r = oracle.route(bits(inp["x"]), bits(inp["Wg"]), wl.k, bias=bias, w_mode=weights)
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=DEV)
    w = torch.empty(wl.T, wl.k, dtype=torch.float32, device=DEV)
    ws = workspace(wl)
    moe.moe_route_variant(wl.T, wl.d, wl.E, wl.k, inp["x"], inp["Wg"], inp["bias"], weights, idx,
                          w, None, ws)
    assert moe.moe_get_device_error(ws)[0] == 0
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    far = r["gap"] >= 1e-3
    assert np.array_equal(np.sort(idx, 1)[far], np.sort(r["idx"], 1)[far])
    wg = np.take_along_axis(w, np.argsort(idx, 1), 1)
    wo = np.take_along_axis(r["w"], np.argsort(r["idx"], 1), 1)
    assert np.max(np.abs(wg[far] - wo[far])) < 2e-4


VARIANT_FORWARD_CASES = [
    (Workload("var_narrow_T300_d256_E16_k2", 300, 256, 16, 384, 2), (1, 0, 0.0)),
    (Workload("var_narrow_T300_d256_E16_k2", 300, 256, 16, 384, 2), (2, 1, 0.0)),
    (Workload("var_narrow_T300_d256_E16_k2_shared", 300, 256, 16, 384, 2, d_ff_shared=256),
     (2, 1, 0.0)),
    (Workload("var_wide_T200_d1152_E8_k2", 200, 1152, 8, 384, 2), (1, 1, 0.0)),
    (Workload("var_wide_T1100_d1152_E8_k2", 1100, 1152, 8, 512, 2), (2, 1, 0.0)),
    # capacity: skewed router bias so that some experts overflow
    (Workload("cap_narrow_T300_d256_E8_k2", 300, 256, 8, 384, 2, skew=True), (0, 0, 1.0)),
    (Workload("cap_narrow_T300_d256_E8_k2_b", 300, 256, 8, 384, 2, skew=True), (2, 1, 1.25)),
    (Workload("cap_wide_T700_d1152_E8_k2", 700, 1152, 8, 512, 2, skew=True), (0, 0, 1.2)),
    (Workload("cap_wide_T2000_d1152_E16_k4", 2000, 1152, 16, 256, 4, skew=True), (1, 0, 0.8)),
]


@pytest.mark.parametrize("wl,variant", VARIANT_FORWARD_CASES,
                         ids=[f"{w.name}-{v}" for w, v in VARIANT_FORWARD_CASES])
def test_forward_variant_matches_oracle(wl, variant):
    inp = _inputs(wl)
    if wl.skew:
        inp["bias"] = torch.zeros(wl.E, dtype=torch.float32, device=DEV)
        inp["bias"][1] = 1.5
        inp["bias"][2] = 1.0
    res = check_forward_variant(wl, inp, variant)
    if variant[2] > 0:
        # the capacity does drop pairs on these inputs
        idx, _, counts = gpu_route(wl, inp)
        assert counts.max() > res["cap"]


# Entropy-controlled k ("Mixtral 8x7B模型架构解析" entropy_aware_routing): the
# router's Wg is scaled so that the tempered softmax's entropy falls on both
# sides of the 0.8 threshold.  Where floating point decides the slot count,
# tokens whose fp64 entropy is within 1e-3 of the threshold may go either way
# and are compared with the oracle forced to the GPU's choice; likewise for
# near ties of the last used logit.
def _entropy_inputs(wl, scale=0.25, big=False):
    inp = synth.make_inputs(wl, device=DEV) if big else _inputs(wl)
    inp["Wg"] = (inp["Wg"].float() * scale).to(torch.bfloat16)
    inp["bias"] = torch.linspace(-0.02, 0.03, wl.E, dtype=torch.float32, device=DEV)
    return inp


def _entropy_route_check(wl, inp, idx, w):
    """GPU routing under the entropy rule vs the oracle.  Returns (oracle
    route, mask of tokens the test cannot decide by fp64)."""
    bias = inp["bias"].double().cpu().numpy()
    r = oracle.route(bits(inp["x"]), bits(inp["Wg"]), wl.k, bias=bias, w_mode=oracle.W_ENTROPY)
    L = r["logits"]
    P = np.exp((L - L.max(1, keepdims=True)) / oracle.ENTROPY_TAU)
    P /= P.sum(1, keepdims=True)
    H = -np.where(P > 0, P * np.log(np.where(P > 0, P, 1.0)), 0.0).sum(1)
    ku_o = (r["idx"] >= 0).sum(1)
    Ls = -np.sort(-L, 1)
    gap = np.array([Ls[t, ku_o[t] - 1] - Ls[t, ku_o[t]] for t in range(wl.T)])
    unsure = (np.abs(H - oracle.ENTROPY_THRESHOLD) < 1e-3) | (gap < 1e-3)
    far = ~unsure
    ku_g = (idx >= 0).sum(1)
    assert (idx[:, :wl.k - 1] >= 0).all() and ((idx >= 0).sum(1) >= wl.k - 1).all()
    assert (w[idx < 0] == 0).all()
    assert np.array_equal(ku_g[far], ku_o[far]), "slot counts differ"
    for t in np.nonzero(far)[0]:
        assert set(idx[t][idx[t] >= 0]) == set(r["idx"][t][r["idx"][t] >= 0]), t
    wg = np.where(idx >= 0, w, 0.0)
    wgs = np.take_along_axis(wg, np.argsort(np.where(idx >= 0, idx, 10**6), 1), 1)
    wos = np.take_along_axis(r["w"], np.argsort(np.where(r["idx"] >= 0, r["idx"], 10**6), 1), 1)
    assert np.max(np.abs(wgs[far] - wos[far])) < 2e-4
    assert 0.1 < (ku_o == wl.k).mean() < 0.9, "both slot counts occur"
    return r, unsure


@pytest.mark.parametrize("wl", [Workload("ent_T300_E16_k3", 300, 256, 16, 128, 3),
                                Workload("ent_tc_T1153_d4608_E256_k4", 1153, 4608, 256, 128, 4)],
                         ids=lambda w: w.name)
def test_route_entropy_controlled_k_matches_oracle(wl):
    big = wl.T * wl.E * wl.d > 2 ** 30
    inp = _entropy_inputs(wl, scale=0.25 if wl.E <= 16 else 0.6, big=big)
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=DEV)
    w = torch.empty(wl.T, wl.k, dtype=torch.float32, device=DEV)
    counts = torch.empty(wl.E, dtype=torch.int32, device=DEV)
    ws = workspace(wl)
    moe.moe_route_variant(wl.T, wl.d, wl.E, wl.k, inp["x"], inp["Wg"], inp["bias"],
                          moe.WEIGHTS_ENTROPY, idx, w, counts, ws)
    assert moe.moe_get_device_error(ws)[0] == 0
    idx, w, counts = idx.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()
    _entropy_route_check(wl, inp, idx, w)
    assert np.array_equal(counts, np.bincount(idx[idx >= 0], minlength=wl.E))


ENTROPY_FORWARD_CASES = [
    Workload("ent_narrow_T300_d256_E8_k3", 300, 256, 8, 384, 3),
    Workload("ent_narrow_T300_d256_E8_k2_shared", 300, 256, 8, 384, 2, d_ff_shared=256),
    Workload("ent_wide_T200_d1152_E8_k3", 200, 1152, 8, 384, 3),
    Workload("ent_wide_pair_T1100_d1152_E8_k2", 1100, 1152, 8, 512, 2),
]


@pytest.mark.parametrize("wl", ENTROPY_FORWARD_CASES, ids=lambda w: w.name)
def test_forward_entropy_controlled_k_matches_oracle(wl):
    from gpu_util import gpu_forward_variant
    inp = _entropy_inputs(wl)
    variant = (moe.WEIGHTS_ENTROPY, 0, 0.0)
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=DEV)
    w = torch.empty(wl.T, wl.k, dtype=torch.float32, device=DEV)
    ws = workspace(wl)
    moe.moe_route_variant(wl.T, wl.d, wl.E, wl.k, inp["x"], inp["Wg"], inp["bias"],
                          moe.WEIGHTS_ENTROPY, idx, w, None, ws)
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    r, unsure = _entropy_route_check(wl, inp, idx, w)
    out = gpu_forward_variant(wl, inp, variant).cpu().numpy().astype(np.float64)
    tok = np.arange(wl.T) if wl.T <= 300 else sample_tokens(wl.T, 96, idx, unsure)
    shared = None
    if wl.d_ff_shared:
        shared = (bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"]))
    ref = oracle.forward(bits(inp["x"]), bits(inp["Wg"]), bits(inp["W1"]), bits(inp["W3"]),
                         bits(inp["W2"]), wl.k, bias=inp["bias"].double().cpu().numpy(),
                         tokens=tok, shared=shared, forced=idx[tok], w_mode=oracle.W_ENTROPY)
    assert_close(out[tok], ref, wl.name)


def test_entropy_controlled_k_argument_checks():
    wl = Workload("ent_args", 16, 256, 8, 128, 1)
    inp = _inputs(wl)
    ws = workspace(wl)
    out = torch.empty(16, 256, device=DEV)
    with pytest.raises(moe.MoEError) as e:   # k = 1 leaves no slot to drop
        moe.moe_forward_variant(16, 256, 8, 128, 1, inp["x"], inp["Wg"], None, inp["W1"],
                                inp["W3"], inp["W2"], 0, None, None, None,
                                (moe.WEIGHTS_ENTROPY, 0, 0.0), out, ws)
    assert e.value.status == 1
    wl2 = Workload("ent_args2", 16, 256, 8, 128, 2)
    ws2 = workspace(wl2)
    with pytest.raises(moe.MoEError) as e:   # not combined with a capacity
        moe.moe_forward_variant(16, 256, 8, 128, 2, inp["x"], inp["Wg"], None, inp["W1"],
                                inp["W3"], inp["W2"], 0, None, None, None,
                                (moe.WEIGHTS_ENTROPY, 0, 1.0), out, ws2)
    assert e.value.status == 2


def test_forward_variant_none_is_the_method():
    wl = Workload("var_none", 200, 256, 8, 256, 2)
    inp = _inputs(wl)
    from gpu_util import gpu_forward_variant
    a = gpu_forward(wl, inp)
    b = gpu_forward_variant(wl, inp, None)
    c = gpu_forward_variant(wl, inp, (0, 0, 0.0))
    assert torch.equal(a, b) and torch.equal(a, c)


# ------------------------------------------------------------------ FP8 experts
FP8_CASES = [
    Workload("fp8_T8_d512_E8_k2", 8, 512, 8, 1024, 2),
    Workload("fp8_T129_d384_E16_k4", 129, 384, 16, 640, 4),
    Workload("fp8_T300_d1152_E8_k2", 300, 1152, 8, 512, 2),
    Workload("fp8_T1000_d256_E8_k2", 1000, 256, 8, 256, 2),
]


def _fp8_forward(wl, inp):
    out = torch.empty(wl.T, wl.d, dtype=torch.float32, device=DEV)
    ws = workspace(wl)
    moe.moe_forward_fp8(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"], inp["bias"],
                        inp["q1"], inp["s1"], inp["q3"], inp["s3"], inp["q2"], inp["s2"], out, ws)
    st, code = moe.moe_get_device_error(ws)
    assert st == 0, f"device error word {code:#x}"
    return out.cpu().numpy().astype(np.float64)


def _fp8_check(wl, inp, tokens=None):
    idx, r, near = check_routing(wl, inp)
    out = _fp8_forward(wl, inp)
    tok = np.arange(wl.T) if tokens is None else np.asarray(tokens)
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    ref = oracle.forward_fp8(bits(inp["x"]), bits(inp["Wg"]), inp["q1"].cpu().numpy(),
                             inp["s1"].double().cpu().numpy(), inp["q3"].cpu().numpy(),
                             inp["s3"].double().cpu().numpy(), inp["q2"].cpu().numpy(),
                             inp["s2"].double().cpu().numpy(), wl.k, bias=bias, tokens=tok,
                             forced=idx[tok])
    return assert_close(out[tok], ref, wl.name)


@pytest.mark.parametrize("wl", FP8_CASES, ids=lambda w: w.name)
def test_forward_fp8_matches_oracle(wl):
    inp = {k: (None if v is None else v.to(DEV)) for k, v in
           synth.make_fp8_experts(wl, seed=7, device="cpu").items()}
    _fp8_check(wl, inp)


@pytest.mark.parametrize("T", [1, 8, 128])
def test_forward_fp8_mixtral_decode(T):
    wl = synth.mixtral_decode(T)
    inp = synth.make_fp8_experts(wl, seed=7, device=DEV)
    idx, _, counts = gpu_route(wl, inp)
    tok = sample_tokens(T, 8, idx)
    _fp8_check(wl, inp, tokens=tok)


@pytest.mark.parametrize("T", [8, 1000])
def test_forward_fp8_every_code(T):
    # Every finite e4m3 code (both zeros, the subnormals, +-448) in every
    # weight row, rotated from row to row, through both operand paths of the
    # FP8 expert kernel: widened rows in tensor memory (token tiles of up to
    # 64 rows, T = 8) and in shared memory (128-row tiles, T = 1000).
    wl = Workload(f"fp8_every_code_T{T}", T, 512, 4, 256, 2)
    inp = synth.make_fp8_experts(wl, seed=11, device="cpu")
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    for name in ("q1", "q3", "q2"):
        q = inp[name].numpy().copy()
        for e in range(q.shape[0]):
            for r in range(q.shape[1]):
                q[e, r] = np.resize(np.roll(codes, 7 * r + 13 * e), q.shape[2])
        inp[name] = torch.from_numpy(q)
    assert all(len(np.unique(inp[n].numpy())) == 254 for n in ("q1", "q3", "q2"))
    inp = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    _fp8_check(wl, inp)
