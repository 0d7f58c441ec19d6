"""Host-side logic of the K/V offload (LRQK page, abstract: a mixed GPU-CPU
cache whose hit-and-miss mechanism keeps the rows the selection keeps
hitting on the GPU): the swap planner of libloki and the argument checks of
the swap issuer, both without a GPU."""
import ctypes

import numpy as np
import pytest

from rank_key_top_b200 import loki


def plan(home, spare, touch, max_moves):
    import torch
    h = torch.tensor(home, dtype=torch.int32)
    sp = ctypes.c_int32(spare)
    moves = loki.loki_offload_plan(h, sp, torch.tensor(touch, dtype=torch.int32), max_moves)
    return h.numpy().copy(), sp.value, moves


def random_state(rng, n, n_dev):
    """n blocks, n_dev of them on device pages (a random permutation of
    n_dev + 1 pages, one left spare), the rest on host pages."""
    on_dev = rng.permutation(n)[:n_dev]
    dev_pages = rng.permutation(n_dev + 1)
    host_pages = rng.permutation(n - n_dev)
    home = np.empty(n, np.int32)
    di = hi = 0
    for b in range(n):
        if b in set(on_dev.tolist()):
            home[b] = dev_pages[di]
            di += 1
        else:
            home[b] = -(host_pages[hi] + 1)
            hi += 1
    return home, int(dev_pages[n_dev])


def simulate(home0, spare0, moves):
    """Pools as dicts page -> block whose rows the page holds, driven by the
    moves in order with the issuer's copies: host_page -> device_page, then
    freed_page -> host_page."""
    dev = {int(p): b for b, p in enumerate(home0) if p >= 0}
    host = {int(-p - 1): b for b, p in enumerate(home0) if p < 0}
    for m in moves:
        assert m.device_page not in dev, "the receiving device page must be free"
        dev[m.device_page] = host[m.host_page]
        host[m.host_page] = dev.pop(m.freed_page)
    return dev, host


@pytest.mark.parametrize("seed", range(6))
def test_plan_puts_the_most_touched_blocks_on_the_device(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 300))
    n_dev = int(rng.integers(1, n))
    home0, spare0 = random_state(rng, n, n_dev)
    touch = rng.integers(0, 6 if seed % 2 else 1000, size=n)   # many ties, or few
    home, spare, moves = plan(home0, spare0, touch, 10 ** 6)
    on_dev = home >= 0
    assert on_dev.sum() == n_dev
    if (~on_dev).any():
        assert touch[on_dev].min() >= touch[~on_dev].max()
    # the map stays a bijection onto the same pages, the spare unused
    assert sorted(home[on_dev].tolist() + [spare]) == sorted(home0[home0 >= 0].tolist() + [spare0])
    assert sorted(home[~on_dev].tolist()) == sorted(home0[home0 < 0].tolist())
    # a move only ever swaps a strictly hotter offloaded block in
    for m in moves:
        assert touch[m.block_in] > touch[m.block_out]
    # data follows the blocks: after the copies every page holds the block the map says
    dev, host = simulate(home0, spare0, moves)
    for b in range(n):
        assert (dev[home[b]] if home[b] >= 0 else host[-home[b] - 1]) == b
    # planning again on the same counts moves nothing
    home2, spare2, moves2 = plan(home, spare, touch, 10 ** 6)
    assert moves2 == [] and np.array_equal(home2, home) and spare2 == spare


def test_plan_respects_max_moves_and_takes_the_hottest_first():
    n = 8
    home0 = np.array([0, 1, 2, 3, -1, -2, -3, -4], np.int32)
    touch = np.array([5, 0, 9, 1, 7, 2, 8, 3])
    home, spare, moves = plan(home0, 4, touch, 2)
    assert [(m.block_in, m.block_out) for m in moves] == [(6, 1), (4, 3)]
    assert [(m.host_page, m.device_page, m.freed_page) for m in moves] == [(2, 4, 1), (0, 1, 3)]
    assert spare == 3
    assert home.tolist() == [0, -3, 2, -1, 1, -2, 4, -4]
    # with no limit the third pair (block 7, 3 touches, against block 0, 5) stays put
    _, _, all_moves = plan(home0, 4, touch, 100)
    assert [(m.block_in, m.block_out) for m in all_moves] == [(6, 1), (4, 3)]


def test_plan_ties_go_to_the_lower_block_id():
    home0 = np.array([0, 1, -1, -2], np.int32)
    home, spare, moves = plan(home0, 2, [3, 3, 9, 9], 1)
    assert [(m.block_in, m.block_out) for m in moves] == [(2, 0)]


def test_plan_rejects_bad_arguments():
    import torch
    home = torch.tensor([0, -1], dtype=torch.int32)
    touch = torch.zeros(2, dtype=torch.int32)
    for spare, max_moves in ((0, 4), (-1, 4), (1, -1)):   # spare in use, negative spare, negative limit
        with pytest.raises(loki.LokiError):
            loki.loki_offload_plan(home, ctypes.c_int32(spare), touch, max_moves)
    assert home.tolist() == [0, -1]


def fake_cache(kv_home=True):
    """A loki_cache with aligned placeholder addresses: enough for the host
    checks, which return before any CUDA call."""
    a = 1 << 20
    c = loki.loki_cache(a, 2 * a, 3 * a, 10, 2, 128, 32, loki.LOKI_BF16)
    if kv_home:
        c.kv_home, c.k_host, c.v_host = 4 * a, 5 * a, 6 * a
        c.num_device_pages, c.num_host_pages = 6, 5
    return c


@pytest.mark.parametrize("field,value", [("block_in", 10), ("block_out", -1), ("host_page", 5),
                                         ("device_page", 6), ("freed_page", -2)])
def test_apply_rejects_moves_outside_the_pools(field, value):
    c = fake_cache()
    m = loki.loki_page_move(1, 2, 0, 5, 3)
    setattr(m, field, value)
    home = np.zeros(10, np.int32)
    st = loki._lib.loki_offload_apply(ctypes.byref(c), (loki.loki_page_move * 1)(m), 1,
                                      home.ctypes.data_as(ctypes.c_void_p), None)
    assert st == loki.LOKI_ERR_INVALID_ARG


def test_apply_needs_an_offloaded_cache():
    c = fake_cache(kv_home=False)
    home = np.zeros(10, np.int32)
    st = loki._lib.loki_offload_apply(ctypes.byref(c), (loki.loki_page_move * 1)(), 0,
                                      home.ctypes.data_as(ctypes.c_void_p), None)
    assert st == loki.LOKI_ERR_INVALID_ARG


def test_offloaded_cache_checks():
    """A host pool with pages needs its addresses; unaligned ones are refused
    (the dense workspace query returns 0 for a cache that fails the checks)."""
    bt = loki.loki_batch(1 << 20, 1 << 21, 1, 4, 64)
    ok = fake_cache()
    assert loki._lib.loki_dense_workspace_bytes(ctypes.byref(ok), ctypes.byref(bt), 4) > 0
    for field, value in (("k_host", 0), ("v_host", (1 << 20) + 8), ("num_host_pages", -1)):
        c = fake_cache()
        setattr(c, field, value)
        st = loki._lib.loki_dense_attention(ctypes.byref(c), ctypes.byref(bt), ctypes.c_void_p(1 << 20), 4,
                                            ctypes.c_void_p(1 << 20), 0.0, ctypes.c_void_p(1 << 20),
                                            ctypes.c_void_p(1 << 20), 1 << 20, None)
        assert st == loki.LOKI_ERR_INVALID_ARG, field
        assert loki._lib.loki_dense_workspace_bytes(ctypes.byref(c), ctypes.byref(bt), 4) == 0
