"""Host side of the expert-parallel layer, on CPU: the sizes and argument
checks of the C entry points (no GPU call is reached), the owner blocks, and
the exchange of buffer handles between two gloo ranks that builds each
rank's table of peer addresses."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import sparse_mixture_experts_histogram_b200 as moe
from sparse_mixture_experts_histogram_b200 import build, ep

FAKE = 1 << 20  # a 16-byte aligned, never dereferenced address


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def test_recv_rows_is_the_worst_case_of_one_owner(lib):
    # every token of every rank may reach min(k, E/R) experts of one owner
    assert moe.moe_ep_recv_rows(8, 8, 2, 8) == 8 * 8 * 1
    assert moe.moe_ep_recv_rows(100, 8, 2, 2) == 2 * 100 * 2
    assert moe.moe_ep_recv_rows(96, 64, 8, 8) == 8 * 96 * 8
    assert moe.moe_ep_recv_rows(10, 6, 2, 4) == 0     # E not a multiple of R
    assert moe.moe_ep_recv_rows(10, 16, 2, 9) == 0    # more ranks than supported
    assert moe.moe_ep_recv_rows(0, 8, 2, 2) == 0


def test_workspace_and_splits(lib):
    n = moe.moe_ep_workspace_size(64, 512, 8, 1024, 2, 4)
    rows = moe.moe_ep_recv_rows(64, 8, 2, 4)
    assert n >= rows * 1024 * 2                       # the hidden activations
    assert moe.moe_ep_workspace_size(64, 500, 8, 1024, 2, 4) == 0   # d % 128
    assert moe.moe_ep_workspace_size(64, 512, 8, 1024, 2, 3) == 0   # E % R
    # decode-sized owners split the down projection, prefill-sized ones do not
    assert moe.moe_ep_ffn_splits(16, 4096, 1, 14336) > 1
    assert moe.moe_ep_ffn_splits(16384, 4096, 1, 14336) == 1


def _dispatch(lib, T=16, d=256, E=8, k=2, R=2, rank=0, recv=2, rows=64, ws_bytes=1 << 30):
    import ctypes
    arr = (ctypes.c_void_p * max(recv, 1))(*([FAKE] * max(recv, 1)))
    return lib.moe_ep_dispatch(T, d, E, k, R, rank, FAKE, FAKE, FAKE, arr if recv else None,
                               rows, FAKE, FAKE, FAKE, ws_bytes, None)


def test_dispatch_checks_its_arguments_on_the_host(lib):
    assert _dispatch(lib, R=9) == 2          # more ranks than supported
    assert _dispatch(lib, E=6, R=4) == 1     # E not a multiple of R
    assert _dispatch(lib, rank=2) == 1       # rank outside [0, R)
    assert _dispatch(lib, rank=-1) == 1
    assert _dispatch(lib, recv=0) == 1       # no receive table
    assert _dispatch(lib, rows=0) == 1
    assert _dispatch(lib, T=-1) == 1
    # no tokens on this rank: combine has nothing to do (no GPU work)
    import ctypes
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert lib.moe_ep_combine(0, 512, 8, 2, 2, 64, 1, 0, None, None, None, ptrs, None, None,
                              None) == 0
    assert _dispatch(lib, d=500) == 2        # d % 128
    assert _dispatch(lib, ws_bytes=16) == 3  # workspace too small


def test_expert_ffn_and_combine_check_their_arguments(lib):
    import ctypes
    ks = moe.moe_ep_ffn_splits(4 * 2, 512, 4, 1024)
    args = lambda ksplit, R=2, bf=0: ((4, 512, 8, 1024, 2, R, 8, ksplit, bf) + (FAKE,) * 7 +
                                      (1 << 40, None))
    assert lib.moe_ep_expert_ffn(*args(ks + 1)) == 1    # ksplit not the library's
    assert lib.moe_ep_expert_ffn(*args(ks, R=3)) == 1   # E % R
    assert moe.moe_ep_output_bf16(8, 512, 4, 1024) == 0  # decode-sized: split K, fp32 partials
    assert lib.moe_ep_expert_ffn(*args(ks, bf=1)) == 1  # bf16 rows not available here
    assert moe.moe_ep_output_bf16(4096, 4096, 1, 14336) == 1
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    comb = lambda R=2, ksplit=1, E=8, bf=0: lib.moe_ep_combine(4, 512, E, 2, R, 64, ksplit, bf,
                                                               FAKE, FAKE, FAKE, ptrs, None, FAKE,
                                                               None)
    assert comb(R=9) == 2
    assert comb(E=6, R=4) == 1
    assert comb(ksplit=0) == 1
    assert comb(ksplit=9) == 2
    assert comb(ksplit=2, bf=1) == 1                    # bf16 rows hold complete sums only


def test_expert_blocks_tile_the_experts():
    E, R = 64, 8
    blocks = [ep.expert_block(E, R, r) for r in range(R)]
    assert blocks[0] == (0, 8) and blocks[-1] == (56, 64)
    assert all(b[1] == c[0] for b, c in zip(blocks, blocks[1:]))
    with pytest.raises(ValueError):
        ep.expert_block(10, 4, 0)


def test_peer_addresses_open_only_the_peers():
    opened = []

    def fake_open(handle):
        opened.append(handle)
        return {b"h0": 1000, b"h2": 3000}[handle]

    entries = [(b"h0", 16), (b"h1", 0), (b"h2", 256)]
    addrs, bases = ep.peer_addresses(1, entries, 0xABC, fake_open)
    assert addrs == [1016, 0xABC, 3256]
    assert bases == {b"h0": 1000, b"h2": 3000}
    assert opened == [b"h0", b"h2"]     # this rank's own handle is never opened
    # A second buffer in the same allocations reuses the mappings.
    addrs2, bases2 = ep.peer_addresses(1, [(b"h0", 64), (b"h1", 8), (b"h2", 512)], 0xDEF,
                                       fake_open, bases)
    assert addrs2 == [1064, 0xDEF, 3512]
    assert opened == [b"h0", b"h2"] and bases2 is bases


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # Each rank publishes (handle, offset) of its two buffers, as
        # ExpertParallelLayer does, and builds its peer tables.
        mine = ((bytes([rank]) * 64, 16 * rank), (bytes([10 + rank]) * 64, 32 * rank))
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        base_of = lambda h: 1_000_000 * (h[0] + 1)
        opened = {}
        xs, _ = ep.peer_addresses(rank, [g[0] for g in gathered], 7 + rank, base_of, opened)
        ys, _ = ep.peer_addresses(rank, [g[1] for g in gathered], 70 + rank, base_of, opened)
        q.put((rank, xs, ys, len(opened)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_build_matching_peer_tables():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, x0, y0, n0), (_, x1, y1, n1) = res
    # rank 0 sees its own buffers and rank 1's mapped ones (base + offset)
    assert x0 == [7, 2_000_000 + 16] and y0 == [70, 12_000_000 + 32]
    assert x1 == [1_000_000 + 0, 8] and y1 == [11_000_000 + 0, 71]
    assert n0 == n1 == 2
