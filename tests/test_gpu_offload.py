"""K/V offload on the GPU (LRQK page, abstract: a mixed GPU-CPU cache where
only the missing rows of the kept tokens are transferred, and attention stays
exact). An offloaded cache must give bit for bit what the all-device cache
gives — outputs, kept sets and the cache rows themselves — for every call,
before and after the planner's swaps; and the touch counts must equal the
kept sets."""
import numpy as np
import pytest
import torch

from rank_key_top_b200 import synth
from tests import harness

pytestmark = pytest.mark.gpu


def spec(**kw):
    base = dict(name="offload", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128, seq_lens=[3000, 1700, 4100],
                dtype="bf16", alpha=0.8, r=32, k=200, recent_window=16, seed=23)
    base.update(kw)
    base["batch"] = len(base["seq_lens"])
    return synth.Spec(**base)


def split_home(num_blocks, host_every):
    """Blocks b with b % host_every == 1 (every block for host_every = 1) on
    host pages, the others on device pages (in block order), plus one spare
    device page."""
    offset = 1 % host_every
    home = np.empty(num_blocks, np.int32)
    d = h = 0
    for b in range(num_blocks):
        if b % host_every == offset:
            home[b] = -(h + 1)
            h += 1
        else:
            home[b] = d
            d += 1
    return home, d + 1, h


def offloaded(loki, wl, index_dims, host_every=2):
    s = wl.spec
    home, dp, hp = split_home(wl.num_blocks, host_every)
    return loki.OffloadCache(wl.num_blocks, s.num_kv_heads, s.head_dim, synth.torch_dtype(s.dtype), home, dp, hp,
                             index_dims=index_dims)


def rows(cache, wl, b, h, L):
    """Key and value rows of one pair read back through the cache's map."""
    s = wl.spec
    dt = synth.torch_dtype(s.dtype)
    D, Hkv = s.head_dim, s.num_kv_heads
    dk, dv = (t.view(dt).view(-1, Hkv, 16, D).cpu() for t in (cache.k, cache.v))
    home = getattr(cache, "home", None)
    if home is not None:
        hk, hv = (t.view(dt).view(-1, Hkv, 16, D) for t in (cache.hk, cache.hv))
    K, V = [], []
    for p in wl.block_table[b][:(L + 15) // 16].tolist():
        if home is None or home[p] >= 0:
            pg = p if home is None else int(home[p])
            K.append(dk[pg, h])
            V.append(dv[pg, h])
        else:
            pg = -int(home[p]) - 1
            K.append(hk[pg, h])
            V.append(hv[pg, h])
    return torch.cat(K)[:L], torch.cat(V)[:L]


def touch_from_sel(wl, sel, num_blocks):
    """Per block: the kept rows a decode gathers from it (all kv heads)."""
    counts = np.zeros(num_blocks, np.int64)
    for b in range(wl.spec.batch):
        for h in range(wl.spec.num_kv_heads):
            for t in sel[b, h].tolist():
                if t >= 0:
                    counts[int(wl.block_table[b, t // 16])] += 1
    return counts


def same_rows(a, b, wl, lens):
    for bb, L in enumerate(lens):
        for h in range(wl.spec.num_kv_heads):
            for x, y in zip(rows(a, wl, bb, h, L), rows(b, wl, bb, h, L)):
                assert torch.equal(x, y), (bb, h)


@pytest.mark.parametrize("dtype,D,group_max,host_every", [("bf16", 128, False, 2), ("bf16", 128, True, 3),
                                                         ("f32", 64, False, 2), ("bf16", 64, False, 1)])
def test_offloaded_decode_is_bit_identical(cuda_lib, dtype, D, group_max, host_every):
    s = spec(dtype=dtype, head_dim=D)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=32)
    full = dev.cache
    off = offloaded(cuda_lib, wl, 32, host_every)
    cuda_lib.loki_prefill_cache(off, dev.batch, wl.Kt.cuda(), wl.V.cuda())
    out_f, sel_f = dev.decode(group_max=group_max)
    dev.cache = off
    out_o, sel_o = dev.decode(group_max=group_max)
    assert cuda_lib.loki_device_error(clear=True) == 0
    assert torch.equal(out_f, out_o) and torch.equal(sel_f, sel_o)
    same_rows(full, off, wl, s.seq_lens)
    assert np.array_equal(off.touch.cpu().numpy()[:wl.num_blocks], touch_from_sel(wl, sel_o, wl.num_blocks))
    harness.check_pair(wl, 2, 1, out_o, sel_o, s.r, s.k, s.recent_window, group_max=group_max)


def test_offloaded_dense_and_scorers_are_bit_identical(cuda_lib):
    s = spec(seq_lens=[2500, 4097])
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=128)
    off = offloaded(cuda_lib, wl, 128)
    cuda_lib.loki_prefill_cache(off, dev.batch, wl.Kt.cuda(), wl.V.cuda())
    results = []
    for cache in (dev.cache, off):
        dev.cache = cache
        got = [dev.dense()]
        for scorer in (cuda_lib.LOKI_SCORER_MAGNITUDE, cuda_lib.LOKI_SCORER_MAGNITUDE_SLABS):
            got.extend(dev.decode(scorer=scorer))
        results.append(got)
    assert cuda_lib.loki_device_error(clear=True) == 0
    for a, b in zip(*results):
        assert torch.equal(a, b)


@pytest.mark.parametrize("W", [0, 8])
def test_offloaded_decode_step_appends_in_place(cuda_lib, W):
    """The step's append writes the new token into its block wherever that
    block lives (lengths chosen so that some new tokens open a block)."""
    s = spec(seq_lens=[1999, 3200, 47], recent_window=W)
    wl = synth.make_workload(s)
    k_new, v_new = synth.draw_new_tokens(s, step=2)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    results, caches = [], []
    for host_every in (None, 2):
        dev = harness.Device(wl, cuda_lib, index_dims=32)
        if host_every:
            dev.cache = offloaded(cuda_lib, wl, 32, host_every)
            cuda_lib.loki_prefill_cache(dev.cache, dev.batch, wl.Kt.cuda(), wl.V.cuda())
        dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
        out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
        sel = torch.full((s.batch, s.num_kv_heads, s.k + W), -7, dtype=torch.int32, device="cuda")
        cuda_lib.loki_decode_step(dev.cache, dev.batch, k_new.cuda(), v_new.cuda(), dev.q, dev.P, s.r, s.k, out,
                                  recent_window=W, selected_idx=sel)
        torch.cuda.synchronize()
        results.append((out.cpu(), sel.cpu()))
        caches.append(dev.cache)
    assert cuda_lib.loki_device_error(clear=True) == 0
    assert torch.equal(results[0][0], results[1][0]) and torch.equal(results[0][1], results[1][1])
    same_rows(caches[0], caches[1], wl, lens.tolist())


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_offloaded_prefill_rotate_is_bit_identical(cuda_lib, dtype, D):
    s = spec(dtype=dtype, head_dim=D, seq_lens=[700, 1300])
    wl = synth.make_workload(s)
    dt = synth.torch_dtype(dtype)
    P = wl.P.cuda().contiguous()
    K = torch.einsum("bhtd,hed->bhte", wl.Kt.cuda().float(), P).to(dt).contiguous()
    batch = cuda_lib.Batch(wl.block_table.cuda(), wl.seq_lens.cuda(), s.max_seq_len)
    full = cuda_lib.Cache(wl.num_blocks, s.num_kv_heads, D, dt, "cuda", index_dims=32)
    off = offloaded(cuda_lib, wl, 32)
    for c in (full, off):
        cuda_lib.loki_prefill_rotate(c, batch, K, wl.V.cuda(), P)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error(clear=True) == 0
    same_rows(full, off, wl, s.seq_lens)
    xf, xo = (c.x.view(dt).view(-1, s.num_kv_heads, 32, 16) for c in (full, off))
    for b, L in enumerate(s.seq_lens):   # the written index entries (tokens < L) only
        blocks = wl.block_table[b][:(L + 15) // 16].long().cuda()
        for h in range(s.num_kv_heads):
            a = xf[blocks, h].permute(0, 2, 1).reshape(-1, 32)[:L]
            c = xo[blocks, h].permute(0, 2, 1).reshape(-1, 32)[:L]
            assert torch.equal(a, c), (b, h)


def test_rebalance_moves_hot_blocks_and_keeps_results(cuda_lib):
    """After a decode, the planner swaps the most-kept offloaded blocks with
    the least-kept device blocks; the rows move with their blocks, the next
    decode is bit-identical and its touch counts are the same."""
    s = spec(seq_lens=[5000, 3333, 4096])
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=32)
    full = dev.cache
    out_f, sel_f = dev.decode()
    off = offloaded(cuda_lib, wl, 32, host_every=2)
    cuda_lib.loki_prefill_cache(off, dev.batch, wl.Kt.cuda(), wl.V.cuda())
    dev.cache = off
    dev.decode()
    touch = off.touch.cpu().numpy()[:wl.num_blocks].copy()
    moves = cuda_lib.offload_rebalance(off, max_moves=10 ** 6)
    torch.cuda.synchronize()
    assert len(moves) > 0
    home = off.home.numpy()
    assert np.array_equal(off.home_dev.cpu().numpy(), home)
    on_dev = home >= 0
    assert touch[on_dev].min() >= touch[~on_dev].max()
    assert not off.touch.cpu().any()
    same_rows(full, off, wl, s.seq_lens)
    out_o, sel_o = dev.decode()
    assert cuda_lib.loki_device_error(clear=True) == 0
    assert torch.equal(out_f, out_o) and torch.equal(sel_f, sel_o)
    assert np.array_equal(off.touch.cpu().numpy()[:wl.num_blocks], touch)
    assert cuda_lib.offload_rebalance(off, max_moves=10 ** 6) == []


def test_offloaded_decode_full_size(cuda_lib):
    """The bench's workload (8 × 32768 tokens, 32 / 8 heads, r 32, k 2048 + 64)
    with every second block's rows on the host, in the bench's launch
    configuration: outputs and kept sets bit-identical to the all-device cache,
    and sampled pairs against the oracle."""
    s = synth.named_spec("gqa32x8-d128-L32768-bf16")
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=s.r)
    out_f, sel_f = dev.decode()
    off = offloaded(cuda_lib, wl, s.r, host_every=2)
    cuda_lib.loki_prefill_cache(off, dev.batch, wl.Kt.cuda(), wl.V.cuda())
    dev.cache = off
    out_o, sel_o = dev.decode()
    assert cuda_lib.loki_device_error(clear=True) == 0
    assert torch.equal(out_f, out_o) and torch.equal(sel_f, sel_o)
    for b, h in [(0, 0), (5, 3)]:
        harness.check_pair(wl, b, h, out_o, sel_o, s.r, s.k, s.recent_window)


def test_home_entry_outside_its_pool_is_flagged(cuda_lib):
    """A map entry past its pool is caught by the kernels' own range check
    (LOKI_DEVERR_BLOCK_ID): the block's rows are neither read nor written."""
    s = spec(seq_lens=[900, 700])
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=32)
    off = offloaded(cuda_lib, wl, 32, host_every=2)
    cuda_lib.loki_prefill_cache(off, dev.batch, wl.Kt.cuda(), wl.V.cuda())
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error(clear=True) == 0
    bad = off.home.clone()
    p = int(wl.block_table[0, 3])
    bad[p] = -(off.struct.num_host_pages + 7)       # past the host pool
    off.home_dev.copy_(bad.cuda())
    dev.cache = off
    out, _ = dev.decode()
    assert cuda_lib.loki_device_error(clear=True) & cuda_lib.LOKI_DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    bad[p] = off.struct.num_device_pages + 3        # past the device pool
    off.home_dev.copy_(bad.cuda())
    dev.dense()
    assert cuda_lib.loki_device_error(clear=True) & cuda_lib.LOKI_DEVERR_BLOCK_ID
