"""Host-side checks of the C ABI library (no GPU needed, no compute calls):
the library loads, exports exactly the functions include/*.h declares, and
rejects bad arguments before touching the GPU."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def test_every_declared_symbol_is_exported(lib):
    decl = declared_functions()
    assert decl, "no MOE_API declarations found"
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert decl <= exported, f"declared but not exported: {decl - exported}"
    assert {s for s in exported if s.startswith("moe_")} == decl, "exported but not declared"
    assert set(binding.ABI_FUNCTIONS) == decl
    for n in decl:
        getattr(lib, n)


def test_library_needs_no_libcuda_to_load():
    out = subprocess.run(["ldd", build.LIB], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart" not in out


def test_status_strings(lib):
    for s in range(7):
        txt = moe.moe_status_string(s)
        assert txt.startswith(binding.STATUS_NAMES[s])
    assert "unknown" in moe.moe_status_string(99)


def test_workspace_size(lib):
    n = moe.moe_workspace_size(512, 512, 8, 4096, 2)
    S = 1024
    assert n >= S * 512 * 2 + S * 4096 * 2 + S * 512 * 4
    assert moe.moe_workspace_size_ex(512, 512, 8, 4096, 2, 1024) > n
    assert moe.moe_workspace_size(512, 500, 8, 4096, 2) == 0      # d not a multiple of 128
    assert moe.moe_workspace_size(512, 512, 8, 4096, 9) == 0      # k > E
    assert moe.moe_workspace_size(512, 512, 300, 4096, 2) == 0    # E > 256


FAKE = 1 << 20  # a 16-byte aligned, never dereferenced address


@pytest.mark.parametrize("args,expect", [
    ((0, 512, 8, 2), 1),          # T = 0
    ((16, 512, 8, 9), 1),         # k > E
    ((16, 512, 8, 0), 1),         # k = 0
    ((16, 500, 8, 2), 2),         # d % 128
    ((16, 512, 300, 2), 2),       # E > 256
    ((16, 512, 10, 9), 2),        # k > 8
])
def test_route_rejects_bad_sizes(lib, args, expect):
    T, d, E, k = args
    st = lib.moe_route(T, d, E, k, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 40, None)
    assert st == expect


def test_null_misaligned_and_small_workspace(lib):
    assert lib.moe_route(16, 512, 8, 2, None, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == 1
    assert lib.moe_route(16, 512, 8, 2, FAKE + 2, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 40,
                         None) == 1
    assert lib.moe_route(16, 512, 8, 2, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 64, None) == 3
    assert lib.moe_forward(16, 512, 8, 1024, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64,
                           None) == 3
    assert lib.moe_forward(16, 512, 8, 1000, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                           1 << 40, None) == 2
    assert lib.moe_permute(16, 512, 8, 2, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 40, None) == 1
    assert lib.moe_expert_ffn(64, 512, 8, 1024, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64,
                              None) == 3
    assert lib.moe_combine(16, 512, 9, FAKE, FAKE, FAKE, None, FAKE, None) == 2
    assert lib.moe_combine(16, 512, 2, FAKE, FAKE, FAKE, FAKE + 4, FAKE, None) == 1
    # shared expert requested without its weights
    assert lib.moe_forward_ex(16, 512, 8, 1024, 2, FAKE, FAKE, None, FAKE, FAKE, FAKE, 256,
                              None, None, None, FAKE, FAKE, 1 << 40, None) == 1
    # traced forward needs exactly MOE_TRACE_EVENTS events
    evs = (ctypes.c_void_p * binding.TRACE_EVENTS)()
    assert lib.moe_forward_traced(16, 512, 8, 1024, 2, FAKE, FAKE, None, FAKE, FAKE, FAKE, 0,
                                  None, None, None, FAKE, FAKE, 1 << 40, None, evs,
                                  binding.TRACE_EVENTS - 1) == 1
    assert "#define MOE_TRACE_EVENTS %d" % binding.TRACE_EVENTS in open(
        os.path.join(ROOT, "include", "moe.h")).read()
    assert lib.moe_get_device_error(None, None, None) == 1


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        binding.load_library(str(tmp_path / "nope.so"))
    monkeypatch.setattr(binding, "_lib", None)


def _static_need(S, E, d_ff):
    ctr = 4 * (-(-S // 32) + E) * (d_ff // 128)
    return 256 + -(-ctr // 256) * 256 + 2 * S * d_ff


def test_static_scratch_limit_matches_its_documented_formula(lib):
    cap = 32 << 20
    assert "#define MOE_STATIC_SCRATCH_BYTES ((size_t)32 << 20)" in open(
        os.path.join(ROOT, "include", "moe.h")).read()
    for S, E, d_ff in [(1, 1, 128), (37, 6, 640), (4096, 8, 4096), (131000, 1, 128)]:
        assert moe.moe_expert_ffn_static_bytes(S, E, d_ff) == _static_need(S, E, d_ff)
    assert moe.moe_expert_ffn_static_bytes(10, 1, 100) == 0
    # The largest S that fits for (E=1, d_ff=128), and one row more: the
    # larger call is refused on the host before anything is launched.
    S = max(s for s in range(130000, 132000) if _static_need(s, 1, 128) <= cap)
    assert _static_need(S + 1, 1, 128) > cap
    assert lib.moe_expert_ffn_static(S + 1, 128, 1, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     None) == 3
    # 4096 rows x 4096 hidden x 2 bytes alone fill the array: refused too.
    assert lib.moe_expert_ffn_static(4096, 512, 8, 4096, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     None) == 3
    assert lib.moe_expert_ffn_static(S, 128, 1, 128, FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     None) == 1


def test_variant_arguments_are_checked_on_the_host(lib):
    V = binding.MoEVariant
    ws = 1 << 40
    for bad in (V(4, 0, 0.0), V(-1, 0, 0.0), V(0, 2, 0.0), V(0, 0, -1.0), V(0, 0, float("nan")),
                V(0, 0, float("inf"))):
        st = lib.moe_forward_variant(16, 512, 8, 1024, 2, FAKE, FAKE, None, FAKE, FAKE, FAKE, 0,
                                     None, None, None, ctypes.addressof(bad), FAKE, FAKE, ws, None)
        assert st == 1, (bad.weights, bad.activation, bad.capacity_factor)
    assert lib.moe_route_variant(16, 512, 8, 2, FAKE, FAKE, None, 4, FAKE, FAKE, None, FAKE, ws,
                                 None) == 1
    # the entropy rule needs k >= 2 and takes no capacity
    assert lib.moe_route_variant(16, 512, 8, 1, FAKE, FAKE, None, 3, FAKE, FAKE, None, FAKE, ws,
                                 None) == 1
    for bad, want in ((V(3, 0, 0.0), 1), (V(3, 0, 1.2), 2)):
        k = 1 if want == 1 else 2
        st = lib.moe_forward_variant(16, 512, 8, 1024, k, FAKE, FAKE, None, FAKE, FAKE, FAKE, 0,
                                     None, None, None, ctypes.addressof(bad), FAKE, FAKE, ws, None)
        assert st == want
    assert lib.moe_route_variant(16, 512, 8, 9, FAKE, FAKE, None, 1, FAKE, FAKE, None, FAKE, ws,
                                 None) == 1
    h = open(os.path.join(ROOT, "include", "moe.h")).read()
    for name, v in (("MOE_WEIGHTS_SOFTMAX_TOPK", 0), ("MOE_WEIGHTS_SOFTMAX_ALL", 1),
                    ("MOE_WEIGHTS_SIGMOID", 2), ("MOE_WEIGHTS_ENTROPY", 3), ("MOE_ACT_SILU", 0),
                    ("MOE_ACT_SIGMOID", 1)):
        assert f"#define {name} {v}" in h
    assert ctypes.sizeof(V) == 16


def test_selftest_checks_its_workspace(lib):
    assert lib.moe_selftest_wait_timeout(None, 1 << 20, None) == 1
    assert lib.moe_selftest_wait_timeout(FAKE, 16, None) == 1   # smaller than the header
