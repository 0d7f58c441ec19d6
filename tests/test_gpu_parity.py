"""Parity of the CUDA path (through the C ABI) with the oracle, on seeded
synthetic inputs: small workloads in full, edge cases, and the full-size
workloads with every (sequence, kv head) pair checked."""
import numpy as np
import pytest
import torch

import oracle
from rank_key_top_b200 import synth
from tests import harness

pytestmark = pytest.mark.gpu


def spec(**kw):
    base = dict(name="edge", batch=1, num_q_heads=4, num_kv_heads=1, head_dim=128, seq_lens=[1000],
                dtype="bf16", alpha=0.8, r=32, k=64, seed=11)
    base.update(kw)
    base["batch"] = len(base["seq_lens"])
    return synth.Spec(**base)


def run_and_check(cuda_lib, s, pairs=None, group_max=False, **dec):
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    out, sel = dev.decode(group_max=group_max, **dec)
    assert cuda_lib.loki_device_error() == 0
    r = dec.get("r", s.r)
    k = dec.get("k", s.k)
    W = dec.get("W", s.recent_window)
    errs = []
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            if pairs is not None and (b, h) not in pairs:
                continue
            errs.append(harness.check_pair(wl, b, h, out, sel, r, k, W, group_max=group_max,
                                           scale=dec.get("scale", 0.0)))
    return wl, dev, out, sel, errs


# ---------------------------------------------------------------------------
# Small named workloads, every pair
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["single-head-d64-L1024-f32", "mha32-d128-L4096-bf16"])
def test_small_workloads(cuda_lib, name):
    run_and_check(cuda_lib, synth.named_spec(name))


# ---------------------------------------------------------------------------
# Edge cases: ragged lengths, empty sequences, windows, k >= L, groups, dims
# ---------------------------------------------------------------------------

EDGE = {
    "ragged-g4": dict(num_q_heads=8, num_kv_heads=2, seq_lens=[0, 1, 15, 16, 17, 100, 1000, 5000],
                      k=50, recent_window=3),
    "g8-d64-f32": dict(num_q_heads=16, num_kv_heads=2, head_dim=64, dtype="f32", alpha=1.0,
                       seq_lens=[33, 2000, 7, 4096], r=16, k=7),
    "g2-r64-window": dict(num_q_heads=4, num_kv_heads=2, seq_lens=[300, 365, 364, 4000], r=64, k=300,
                          recent_window=64),
    "g1-full-rank": dict(num_q_heads=3, num_kv_heads=3, seq_lens=[700, 64], r=128, k=1000),
    "k1": dict(seq_lens=[3000, 17], k=1),
    "window-only": dict(seq_lens=[900, 10], k=0, recent_window=20),
    "d64-bf16-g4": dict(num_q_heads=8, num_kv_heads=2, head_dim=64, seq_lens=[2500, 1], r=48, k=40,
                        recent_window=5),
    "many-pairs": dict(num_q_heads=32, num_kv_heads=8, seq_lens=[1500] * 4, k=100, recent_window=16),
    # more pairs than resident clusters: the sequences go longest first (ties, empty ones)
    "many-waves-ragged": dict(num_q_heads=32, num_kv_heads=32, seq_lens=[5, 3000, 0, 3000, 17, 1200, 3000, 64,
                                                                         2999, 1], k=40, recent_window=2),
}


@pytest.mark.parametrize("case", sorted(EDGE))
def test_edge_cases(cuda_lib, case):
    run_and_check(cuda_lib, spec(**EDGE[case]))


@pytest.mark.parametrize("g", [1, 4, 8])
def test_group_max(cuda_lib, g):
    s = spec(num_q_heads=2 * g, num_kv_heads=2, seq_lens=[2048, 777], k=100, recent_window=4)
    run_and_check(cuda_lib, s, group_max=True)


def test_per_sequence_k(cuda_lib):
    s = spec(seq_lens=[4096, 1000, 33, 5000], k=600, k_per_seq=[512, 125, 4, 600])
    run_and_check(cuda_lib, s)


def test_explicit_scale(cuda_lib):
    s = spec(seq_lens=[1200], k=100)
    run_and_check(cuda_lib, s, scale=0.05)


def test_longest_supported_sequence(cuda_lib):
    n = cuda_lib.loki_decode_max_seq_len(128, cuda_lib.LOKI_BF16)
    s = spec(seq_lens=[n], k=4096, recent_window=64, spare_tokens=0)
    run_and_check(cuda_lib, s)


# ---------------------------------------------------------------------------
# Exact ties: integer-valued keys and queries with P = I make every score an
# exact small integer on both sides, so the kept sets must be identical,
# including which of the tied tokens are kept across the CTAs of a cluster.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1])
def test_exact_ties_across_cluster(cuda_lib, seed):
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[6000, 3001], k=700, recent_window=7, r=16,
             seed=20 + seed)
    wl = synth.make_workload(s)
    g = torch.Generator().manual_seed(seed)
    wl.Kt = torch.randint(-2, 3, wl.Kt.shape, generator=g).to(torch.bfloat16)
    for b, L in enumerate(s.seq_lens):
        wl.Kt[b, :, L:] = 0
    wl.q = torch.randint(-1, 2, wl.q.shape, generator=g).to(torch.bfloat16)
    wl.P = torch.eye(s.head_dim).repeat(s.num_kv_heads, 1, 1).contiguous()
    dev = harness.Device(wl, cuda_lib)
    out, sel = dev.decode()
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            Kt, V, qq, P = harness.pair_inputs(wl, b, h)
            res = oracle.decode_pair(Kt, V, qq, P, r=s.r, k=s.k, W=s.recent_window)
            np.testing.assert_array_equal(sel[b, h].numpy(), res.sel)
            harness.check_pair(wl, b, h, out, sel, s.r, s.k, s.recent_window)


def test_all_scores_equal_keeps_lowest_indices(cuda_lib):
    s = spec(seq_lens=[5000], k=333, recent_window=10)
    wl = synth.make_workload(s)
    wl.Kt[:, :, :, : s.r] = 0.5
    dev = harness.Device(wl, cuda_lib)
    _, sel = dev.decode()
    want = list(range(333)) + list(range(4990, 5000))
    np.testing.assert_array_equal(sel[0, 0, :343].numpy(), want)


# ---------------------------------------------------------------------------
# Invariants of the CUDA path itself
# ---------------------------------------------------------------------------

def test_block_table_shuffle_is_bit_identical(cuda_lib):
    base = dict(num_q_heads=8, num_kv_heads=2, seq_lens=[3000, 4500], k=256, recent_window=8)
    outs = []
    for shuffle in (False, True):
        wl = synth.make_workload(spec(shuffle_blocks=shuffle, **base))
        out, sel = harness.Device(wl, cuda_lib).decode()
        outs.append((out, sel))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_full_rank_full_k_equals_dense(cuda_lib):
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[3000, 129], r=128, k=3000)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    out, _ = dev.decode()
    dense = dev.dense()
    rel = (out - dense).abs().max() / dense.abs().max()
    assert rel < 1e-5, rel


def test_repeat_calls_identical(cuda_lib):
    wl = synth.make_workload(spec(seq_lens=[5000, 3333], k=300))
    dev = harness.Device(wl, cuda_lib)
    a = dev.decode()
    b = dev.decode()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------------------------------------------------
# Append (rotate the new key by P and write it into the paged cache)
# ---------------------------------------------------------------------------

def read_pair(dev, b, h, L):
    """Reads keys, values and the key index of one pair back through the
    documented layout: block p of head h at element (p * Hkv + h) * 16 * D in
    the key and value caches ([16 tokens][D] each) and at (p * Hkv + h) * 16 * I
    in the key index ([I dims][16 tokens])."""
    s = dev.wl.spec
    dt = synth.torch_dtype(s.dtype)
    D, Hkv, I = s.head_dim, s.num_kv_heads, dev.cache.index_dims
    kc = dev.cache.k.view(dt).view(-1, Hkv, 16, D)
    vc = dev.cache.v.view(dt).view(-1, Hkv, 16, D)
    xc = dev.cache.x.view(dt).view(-1, Hkv, I, 16)
    tbl = dev.wl.block_table[b]
    nblk = (L + 15) // 16
    blocks = tbl[:nblk].long().to(kc.device)
    K = kc[blocks, h].reshape(nblk * 16, D)[:L]
    V = vc[blocks, h].reshape(nblk * 16, D)[:L]
    X = xc[blocks, h].permute(0, 2, 1).reshape(nblk * 16, I)[:L]
    return K.cpu(), V.cpu(), X.cpu()


def test_prefill_layout(cuda_lib):
    s = spec(num_q_heads=4, num_kv_heads=2, seq_lens=[100, 37], head_dim=64, dtype="f32")
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    for b, L in enumerate(s.seq_lens):
        for h in range(2):
            K, V, X = read_pair(dev, b, h, L)
            assert torch.equal(K, wl.Kt[b, h, :L]) and torch.equal(V, wl.V[b, h, :L])
            assert torch.equal(X, wl.Kt[b, h, :L, :dev.cache.index_dims])


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64), ("bf16", 64)])
def test_append_matches_oracle(cuda_lib, dtype, D):
    s = spec(num_q_heads=8, num_kv_heads=4, seq_lens=[31, 32, 100, 0], head_dim=D, dtype=dtype)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    k_new, v_new = synth.draw_new_tokens(s, step=0)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
    before_k = dev.cache.k.clone()
    cuda_lib.loki_append_keys(dev.cache, batch, k_new.cuda(), v_new.cuda(), dev.P)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    for b, L in enumerate(lens.tolist()):
        for h in range(s.num_kv_heads):
            K, V, X = read_pair(dev, b, h, L)
            assert torch.equal(X, K[:, :dev.cache.index_dims])
            assert torch.equal(V[L - 1], v_new[b, h])
            if L > 1:
                assert torch.equal(K[: L - 1], wl.Kt[b, h, : L - 1])
            kk = k_new[b, h].double().numpy()[None]
            Ph = wl.P[h].double().numpy()
            want = oracle.append(kk, Ph, dtype)[0]
            got = K[L - 1].double().numpy()
            exact = oracle.rotate(kk, Ph)[0]
            bound = D * 2.0 ** -24 * (np.abs(kk[0][:, None] * Ph)).sum(axis=0)
            mism = got != want
            # a mismatch is allowed only where the exact value is within the
            # fp32 accumulation bound of the rounding midpoint of the two
            assert np.all(np.abs(exact[mism] - (got[mism] + want[mism]) / 2) <= bound[mism]), (b, h)
    assert not torch.equal(before_k, dev.cache.k)


def unrotated_keys(wl):
    """Keys in the original basis whose rotation is the workload's cache rows:
    K = K~ P^T (P orthonormal), rounded to the cache type."""
    K = torch.einsum("bhtd,hed->bhte", wl.Kt.double(), wl.P.double())
    return K.to(synth.torch_dtype(wl.spec.dtype)).contiguous()


@pytest.mark.parametrize("dtype,D,lens", [("bf16", 128, [300, 1000, 0, 1, 129]), ("bf16", 64, [257, 40]),
                                          ("f32", 128, [300, 17, 0]), ("f32", 64, [65]),
                                          # more tiles than CTAs: tile ranges that cross into the next
                                          # (sequence, kv head), with skipped tiles past short sequences
                                          ("bf16", 128, [5000, 1, 2900, 4100]), ("bf16", 64, [3000, 2000, 10])])
def test_prefill_rotate_matches_oracle(cuda_lib, dtype, D, lens):
    """K~ = round(K P) for every prompt token, the value rows copied and the
    key index filled, read back through the documented layout. bf16 uses the
    tensor cores with P split into two bf16 terms: a key may differ from the
    exactly rounded product only where that lies, within the split's error
    (2^-17 of the products' magnitudes) plus fp32 accumulation, at the
    rounding midpoint of the two values."""
    s = spec(num_q_heads=4, num_kv_heads=2, head_dim=D, seq_lens=lens, dtype=dtype, r=16)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=32)
    dev.cache.k.fill_(0xFF)   # every row the call must write starts as a NaN pattern
    dev.cache.v.fill_(0xFF)
    dev.cache.x.fill_(0xFF)
    k_in = unrotated_keys(wl)
    cuda_lib.loki_prefill_rotate(dev.cache, dev.batch, k_in.cuda(), wl.V.cuda(), dev.P)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    split = 2.0 ** -17 if dtype == "bf16" else 0.0
    for b, L in enumerate(lens):
        for h in range(s.num_kv_heads):
            if L == 0:
                continue
            K, V, X = read_pair(dev, b, h, L)
            assert torch.equal(V, wl.V[b, h, :L])
            assert torch.equal(X, K[:, :dev.cache.index_dims])
            kk = k_in[b, h, :L].double().numpy()
            Ph = wl.P[h].double().numpy()
            want = oracle.append(kk, Ph, dtype)
            got = K.double().numpy()
            assert np.all(np.isfinite(got)), (b, h)
            exact = oracle.rotate(kk, Ph)
            mag = np.abs(kk) @ np.abs(Ph)
            bound = (split + D * 2.0 ** -24) * mag
            mism = got != want
            assert np.all(np.abs(exact[mism] - (got[mism] + want[mism]) / 2) <= bound[mism]), (b, h, int(mism.sum()))


def test_prefill_rotate_long_sequence_many_ctas(cuda_lib):
    """One long sequence: several 128-token tiles per CTA and several CTAs per
    (sequence, kv head); a decode on the rotated cache matches the oracle."""
    s = spec(num_q_heads=4, num_kv_heads=1, seq_lens=[40000], k=500, recent_window=16, r=32)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    k_in = unrotated_keys(wl)
    cuda_lib.loki_prefill_rotate(dev.cache, dev.batch, k_in.cuda(), wl.V.cuda(), dev.P)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    K, V, X = read_pair(dev, 0, 0, 40000)
    kk = k_in[0, 0].double().numpy()
    want = oracle.append(kk, wl.P[0].double().numpy(), "bf16")
    assert np.mean(K.double().numpy() == want) > 0.99
    # the oracle's view of the cache is what the kernel wrote
    wl.Kt = K[None, None].clone()
    out, sel = dev.decode()
    harness.check_pair(wl, 0, 0, out, sel, s.r, s.k, s.recent_window)


@pytest.mark.parametrize("dtype,D,n", [("bf16", 128, 4096), ("f32", 128, 1000), ("bf16", 64, 3000)])
def test_pca_basis_matches_oracle(cuda_lib, dtype, D, n):
    """P calibrated on the GPU from sample keys in the original basis against
    the oracle's eigendecomposition of the same keys' centred covariance:
    spectrum, leading subspaces, the well-separated leading directions (with
    the sign convention), orthonormality and reconstruction, within what fp32
    sums over n keys allow."""
    s = spec(num_q_heads=4, num_kv_heads=2, head_dim=D, seq_lens=[n], dtype=dtype, r=16,
             outlier_channels=4)
    wl = synth.make_workload(s)
    keys = unrotated_keys(wl)[0].contiguous()          # [heads][n][D]
    P = torch.full((2, D, D), float("nan"), device="cuda")
    lam = torch.full((2, D), float("nan"), device="cuda")
    cuda_lib.loki_pca_basis(keys.cuda(), P, lam)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    for h in range(2):
        x = keys[h].double().numpy()
        Pr, lr = oracle.pca_basis(x)
        C = oracle.covariance(x)
        Pg, lg = P[h].cpu().double().numpy(), lam[h].cpu().double().numpy()
        top = lr[0]
        assert np.all(np.abs(lg - lr) <= 1e-3 * top), (h, np.abs(lg - lr).max())
        assert np.all(np.diff(lg) <= 0)
        assert np.abs(Pg.T @ Pg - np.eye(D)).max() <= 1e-4
        assert np.abs(Pg @ np.diag(lg) @ Pg.T - C).max() <= 1e-3 * top
        for r in (8, 16, 32):
            gap = (lr[r - 1] - lr[r]) / top
            err = np.linalg.norm(Pg[:, :r] @ Pg[:, :r].T - Pr[:, :r] @ Pr[:, :r].T, 2)
            assert err <= 1e-3 / max(gap, 1e-3), (h, r, err, gap)
        for j in range(4):   # the leading directions are well separated here
            assert np.abs(Pg[:, j] - Pr[:, j]).max() <= 1e-3, (h, j)


@pytest.mark.parametrize("where", ["start", "end", "blocks"])
def test_position_biased_scores(cuda_lib, where):
    """Scores concentrated in one part of the sequence (an attention sink at
    the start, the most recent tokens, or a few scattered blocks): nearly all
    kept tokens fall in one CTA of the cluster and the boundary bins are
    skewed. Set and output parity as everywhere."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[40000, 21000], k=700, recent_window=8, r=32)
    wl = synth.make_workload(s)
    Kt = wl.Kt.float()
    for b, L in enumerate(s.seq_lens):
        if where == "start":
            Kt[b, :, :1500] *= 3.0
        elif where == "end":
            Kt[b, :, L - 2000:L] *= 3.0
        else:
            for blk in range(7, L // 16, 97):
                Kt[b, :, 16 * blk:16 * blk + 16] *= 3.0
    wl.Kt = Kt.to(wl.Kt.dtype)
    dev = harness.Device(wl, cuda_lib)
    out, sel = dev.decode()
    assert cuda_lib.loki_device_error() == 0
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            harness.check_pair(wl, b, h, out, sel, s.r, s.k, s.recent_window)


def test_append_then_decode(cuda_lib):
    """One whole decode step: append the current token, then attend."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[1999, 3000], k=200, recent_window=4)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    k_new, v_new = synth.draw_new_tokens(s, step=3)
    lens = [n + 1 for n in s.seq_lens]
    dev.batch = cuda_lib.Batch(wl.block_table.cuda(), torch.tensor(lens, dtype=torch.int32).cuda(), max(lens))
    cuda_lib.loki_append_keys(dev.cache, dev.batch, k_new.cuda(), v_new.cuda(), dev.P)
    out, sel = dev.decode()
    # the oracle's own view of the cache after the append
    Kt = torch.zeros(s.batch, s.num_kv_heads, max(lens), s.head_dim, dtype=torch.bfloat16)
    V = torch.zeros_like(Kt)
    for b, n in enumerate(s.seq_lens):
        Kt[b, :, :n] = wl.Kt[b, :, :n]
        V[b, :, :n] = wl.V[b, :, :n]
        for h in range(s.num_kv_heads):
            kk = k_new[b, h].double().numpy()[None]
            Kt[b, h, n] = torch.from_numpy(oracle.append(kk, wl.P[h].double().numpy(), "bf16")[0]).to(torch.bfloat16)
            V[b, h, n] = v_new[b, h]
    wl.Kt, wl.V = Kt, V
    wl.spec.seq_lens = lens
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            harness.check_pair(wl, b, h, out, sel, s.r, s.k, s.recent_window)


@pytest.mark.parametrize("dtype,W,group_max", [("bf16", 4, False), ("bf16", 0, False), ("bf16", 16, True),
                                               ("f32", 4, False), ("f32", 0, True)])
def test_decode_step_equals_append_then_decode(cuda_lib, dtype, W, group_max):
    """loki_decode_step (attention launched as a programmatic dependent of the
    append) gives bit for bit what the two separate calls give, cache included."""
    s = spec(num_q_heads=16, num_kv_heads=4, seq_lens=[1999, 37000, 3000], k=300, recent_window=W, dtype=dtype)
    wl = synth.make_workload(s)
    k_new, v_new = synth.draw_new_tokens(s, step=5)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    results = []
    for fused in (False, True):
        dev = harness.Device(wl, cuda_lib)
        dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
        out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
        sel = torch.full((s.batch, s.num_kv_heads, s.k + W), -7, dtype=torch.int32, device="cuda")
        mode = cuda_lib.LOKI_GROUP_MAX if group_max else cuda_lib.LOKI_GROUP_SUM
        if fused:
            cuda_lib.loki_decode_step(dev.cache, dev.batch, k_new.cuda(), v_new.cuda(), dev.q, dev.P, s.r, s.k, out,
                                      recent_window=W, group_reduce=mode, selected_idx=sel)
        else:
            cuda_lib.loki_append_keys(dev.cache, dev.batch, k_new.cuda(), v_new.cuda(), dev.P)
            cuda_lib.loki_decode_attention(dev.cache, dev.batch, dev.q, dev.P, s.r, s.k, out, recent_window=W,
                                           group_reduce=mode, selected_idx=sel)
        torch.cuda.synchronize()
        rows = [t for b in range(s.batch) for h in range(s.num_kv_heads) for t in read_pair(dev, b, h, int(lens[b]))]
        results.append([out.cpu(), sel.cpu()] + rows)   # the written rows only: the rest of the cache is unset
    assert cuda_lib.loki_device_error(clear=True) == 0
    for a, b in zip(*results):
        assert torch.equal(a, b)
    assert not torch.isnan(results[1][0]).any()


def test_decode_step_repeated_in_one_stream(cuda_lib):
    """Steps issued back to back: each step's append must not overtake the
    previous step's attention, nor its attention the append (same token slot
    rewritten every step with a different key)."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[30000, 12000], k=500, recent_window=8)
    wl = synth.make_workload(s)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    steps = [synth.draw_new_tokens(s, step=i) for i in range(6)]
    outs = {}
    for fused in (False, True):
        dev = harness.Device(wl, cuda_lib)
        dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
        kv = [(k.cuda(), v.cuda()) for k, v in steps]
        res = [torch.empty(s.batch, s.num_q_heads, s.head_dim, device="cuda") for _ in steps]
        for (k_new, v_new), out in zip(kv, res):
            if fused:
                cuda_lib.loki_decode_step(dev.cache, dev.batch, k_new, v_new, dev.q, dev.P, s.r, s.k, out,
                                          recent_window=s.recent_window)
            else:
                cuda_lib.loki_append_keys(dev.cache, dev.batch, k_new, v_new, dev.P)
                cuda_lib.loki_decode_attention(dev.cache, dev.batch, dev.q, dev.P, s.r, s.k, out,
                                               recent_window=s.recent_window)
        torch.cuda.synchronize()
        outs[fused] = [o.cpu() for o in res]
    for a, b in zip(outs[False], outs[True]):
        assert torch.equal(a, b)
    for i in range(1, len(steps)):     # every step saw its own token
        assert not torch.equal(outs[True][i], outs[True][i - 1])


def test_decode_step_in_a_cuda_graph(cuda_lib):
    """The bench's form of a step: loki_decode_step captured in a CUDA graph
    (the programmatic dependency between its two kernels becomes a graph
    edge) and replayed gives what the eager calls give, bit for bit."""
    s = spec(num_q_heads=16, num_kv_heads=4, seq_lens=[9000, 33000], k=400, recent_window=32)
    wl = synth.make_workload(s)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    k_new, v_new = synth.draw_new_tokens(s, step=2)
    results = []
    for graphed in (False, True):
        dev = harness.Device(wl, cuda_lib)
        dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
        kd, vd = k_new.cuda(), v_new.cuda()
        out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            def step():
                cuda_lib.loki_decode_step(dev.cache, dev.batch, kd, vd, dev.q, dev.P, s.r, s.k, out,
                                          recent_window=s.recent_window, stream=stream)
            if graphed:
                step()                      # warm-up outside the capture
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    step()
                out.fill_(float("nan"))
                for _ in range(3):
                    g.replay()
            else:
                step()
        torch.cuda.synchronize()
        results.append(out.cpu())
    assert cuda_lib.loki_device_error() == 0
    assert torch.equal(results[0], results[1])


def test_device_checks_flag_bad_lengths_and_blocks(cuda_lib):
    s = spec(num_q_heads=4, num_kv_heads=1, seq_lens=[500, 600], k=20)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    cuda_lib.loki_device_error(clear=True)
    bad_lens = torch.tensor([500, 9999], dtype=torch.int32).cuda()   # above max_seq_len
    dev.batch = cuda_lib.Batch(wl.block_table.cuda(), bad_lens, 600)
    dev.decode()
    assert cuda_lib.loki_device_error(clear=True) & cuda_lib.LOKI_DEVERR_SEQ_LEN
    tbl = wl.block_table.clone()
    tbl[0, 3] = wl.num_blocks + 5                                    # out of range
    dev.batch = cuda_lib.Batch(tbl.cuda(), wl.seq_lens.cuda(), 600)
    dev.decode()
    assert cuda_lib.loki_device_error(clear=True) & cuda_lib.LOKI_DEVERR_BLOCK_ID
    kps = torch.tensor([5, 50], dtype=torch.int32).cuda()            # above k
    dev.batch = cuda_lib.Batch(wl.block_table.cuda(), wl.seq_lens.cuda(), 600)
    dev.k_per_seq = kps
    dev.decode()
    assert cuda_lib.loki_device_error(clear=True) & cuda_lib.LOKI_DEVERR_K


# ---------------------------------------------------------------------------
# Dense comparison path
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["single-head-d64-L1024-f32", "mha32-d128-L4096-bf16"])
def test_dense_small(cuda_lib, name):
    s = synth.named_spec(name)
    wl = synth.make_workload(s)
    out = harness.Device(wl, cuda_lib).dense()
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            harness.check_dense_pair(wl, b, h, out)


def test_dense_edge(cuda_lib):
    s = spec(num_q_heads=16, num_kv_heads=2, seq_lens=[0, 1, 513, 2049], head_dim=64, k=5)
    wl = synth.make_workload(s)
    out = harness.Device(wl, cuda_lib).dense()
    assert torch.all(out[0] == 0)
    for b in range(1, s.batch):
        for h in range(s.num_kv_heads):
            harness.check_dense_pair(wl, b, h, out)


def test_dense_long_splits_ragged(cuda_lib):
    """Enough pairs that the dense path takes its longer splits (2048 tokens:
    160 pairs x 4 splits of the longest sequence fill four waves of CTAs):
    lengths around the split and block edges, one empty sequence."""
    lens = [8191, 0, 1, 2047, 2048, 2049, 4095, 4097, 6144, 16, 17, 3000, 8000, 5555, 2050, 7777] * 2
    lens += [8191, 1024, 1023, 6000, 4096, 2, 8190, 100]
    s = spec(num_q_heads=16, num_kv_heads=4, seq_lens=lens, head_dim=128, k=5, seed=29)
    assert s.batch * s.num_kv_heads * ((max(lens) + 2047) // 2048) >= 4 * 148
    wl = synth.make_workload(s, pairs={(b, h) for b in range(len(lens)) for h in (0, 3)})
    out = harness.Device(wl, cuda_lib).dense()
    assert cuda_lib.loki_device_error() == 0
    assert torch.all(out[1] == 0)
    for b in range(s.batch):
        if lens[b] > 0:
            for h in (0, 3):
                harness.check_dense_pair(wl, b, h, out)


# ---------------------------------------------------------------------------
# Full-size workloads, every pair
# ---------------------------------------------------------------------------

def test_paged_batched_workload(cuda_lib):
    run_and_check(cuda_lib, synth.named_spec("paged-b16-mha32-L4k-16k-bf16"))


def test_gqa_32k_workload(cuda_lib):
    s = synth.named_spec("gqa32x8-d128-L32768-bf16")
    wl, dev, out, sel, errs = run_and_check(cuda_lib, s)
    dense = dev.dense()
    for b, h in [(0, 0), (3, 5), (7, 7)]:
        harness.check_dense_pair(wl, b, h, dense)


def test_long_context_outliers_sweep(cuda_lib):
    s = synth.named_spec("gqa32x8-d128-L131072-bf16-outliers")
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    L = s.seq_lens[0]
    combos = [(r, L // div) for r in (16, 32, 64) for div in (32, 16, 8)]
    results = {c: dev.decode(r=c[0], k=c[1]) for c in combos}
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            inputs = harness.pair_inputs(wl, b, h)
            for (r, k), (out, sel) in results.items():
                harness.check_pair(wl, b, h, out, sel, r, k, 0, inputs=inputs)


# ---------------------------------------------------------------------------
# Magnitude scorers: the scoring dims chosen per step by the query's magnitude
# (single dims, AQUA's algorithm) or energy (whole 16-dim slabs)
# ---------------------------------------------------------------------------

def magnitude_dim_queries(wl, group_max, index_dims, seed):
    """Queries whose rotated dims carry the magnitudes 1.03^i, i = 0 ..
    index_dims - 1, in a shuffled order per (sequence, kv head): the magnitude
    the reduce measures (|sum_j q_hat_j[c]| for SUM, sqrt(sum_j q_hat_j[c]^2)
    for MAX) is set exactly, so the chosen dims have a 3 % margin over the
    dropped ones. Dims past index_dims get magnitude 1. q = q_hat P^T."""
    s = wl.spec
    g, d = s.group, s.head_dim
    gen = torch.Generator().manual_seed(seed)
    q = torch.empty(s.batch, s.num_q_heads, d, dtype=torch.float64)
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            mags = torch.ones(d, dtype=torch.float64)
            mags[:index_dims] = 1.03 ** torch.randperm(index_dims, generator=gen).double()
            z = torch.randn(g, d, generator=gen, dtype=torch.float64)
            if group_max:
                qhat = z * (mags / z.pow(2).sum(0).sqrt())
            else:
                sign = torch.where(torch.rand(d, generator=gen) < 0.5, -1.0, 1.0).double()
                noise = 0.3 * (z - z.mean(0, keepdim=True)) * mags
                qhat = (mags * sign) / g + noise
            q[b, h * g:(h + 1) * g] = qhat @ wl.P[h].double().T
    return q.to(wl.q.dtype)


@pytest.mark.parametrize("dtype,D,Hq,Hkv,index_dims,r,group_max,lens", [
    ("bf16", 128, 8, 2, 128, 32, False, [20000, 3000, 777, 33]),
    ("bf16", 128, 16, 2, 64, 16, True, [3000, 777]),
    ("bf16", 64, 2, 1, 64, 48, False, [3000, 1]),
    ("f32", 128, 4, 1, 128, 64, True, [3000, 0, 500]),
    ("f32", 64, 4, 4, 64, 16, False, [2500, 777]),
    ("bf16", 128, 4, 4, 96, 32, True, [5000, 1200, 16]),
])
def test_magnitude_scorer_matches_oracle(cuda_lib, dtype, D, Hq, Hkv, index_dims, r, group_max, lens):
    """Set and output parity with the oracle's per-dimension selection (AQUA
    page, Algorithm 1 in prose; appendix on complexity, steps 2-4), which
    chooses from the same queries; at least one pair must choose dims other
    than the leading ones, or the case would not test the choice."""
    s = spec(dtype=dtype, head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, seq_lens=lens, r=r, k=150,
             recent_window=5)
    wl = synth.make_workload(s)
    wl.q = magnitude_dim_queries(wl, group_max, index_dims, seed=23)
    dev = harness.Device(wl, cuda_lib, index_dims=index_dims)
    out, sel = dev.decode(group_max=group_max, scorer=cuda_lib.LOKI_SCORER_MAGNITUDE)
    assert cuda_lib.loki_device_error() == 0
    moved = 0
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            harness.check_pair(wl, b, h, out, sel, r, s.k, s.recent_window, group_max=group_max,
                               magnitude_dims=index_dims, magnitude="dims")
            qq, P = harness.pair_inputs(wl, b, h)[2:]
            dims, _ = oracle.magnitude_dims(qq, P, r, index_dims, group_max)
            moved += dims.tolist() != list(range(r))
    assert moved > 0


def magnitude_queries(wl, group_max, seed):
    """Queries whose rotated slabs carry the energies 1.3^(2i), i = 0 .. d/16 - 1,
    in a shuffled order per (sequence, kv head): the energy the chosen reduce
    measures (of the summed query for SUM, summed over heads for MAX) is set
    exactly, so the choice of slabs has a wide margin. q = q_hat P^T."""
    s = wl.spec
    g, d = s.group, s.head_dim
    gen = torch.Generator().manual_seed(seed)
    q = torch.empty(s.batch, s.num_q_heads, d, dtype=torch.float64)
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            qhat = torch.randn(g, d, generator=gen, dtype=torch.float64)
            mags = 1.3 ** torch.randperm(d // 16, generator=gen).double()
            for sl in range(d // 16):
                blk = qhat[:, 16 * sl:16 * sl + 16]
                norm = blk.pow(2).sum().sqrt() if group_max else blk.sum(0).pow(2).sum().sqrt()
                qhat[:, 16 * sl:16 * sl + 16] = blk * (mags[sl] / norm)
            q[b, h * g:(h + 1) * g] = qhat @ wl.P[h].double().T
    return q.to(wl.q.dtype)


@pytest.mark.parametrize("dtype,D,Hq,Hkv,index_dims,r,group_max,lens", [
    ("bf16", 128, 8, 2, 128, 32, False, [20000, 3000, 777, 33]),
    ("bf16", 128, 16, 2, 64, 16, True, [3000, 777]),
    ("bf16", 64, 2, 1, 64, 48, False, [3000, 1]),
    ("f32", 128, 4, 1, 128, 64, True, [3000, 0, 500]),
    ("f32", 64, 4, 4, 64, 16, False, [2500, 777]),
])
def test_slab_scorer_matches_oracle(cuda_lib, dtype, D, Hq, Hkv, index_dims, r, group_max, lens):
    """The slab variant against the oracle's slab choice from the same
    queries; at least one pair must choose slabs other than the leading ones."""
    s = spec(dtype=dtype, head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, seq_lens=lens, r=r, k=150,
             recent_window=5)
    wl = synth.make_workload(s)
    wl.q = magnitude_queries(wl, group_max, seed=21)
    dev = harness.Device(wl, cuda_lib, index_dims=index_dims)
    out, sel = dev.decode(group_max=group_max, scorer=cuda_lib.LOKI_SCORER_MAGNITUDE_SLABS)
    assert cuda_lib.loki_device_error() == 0
    moved = 0
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            harness.check_pair(wl, b, h, out, sel, r, s.k, s.recent_window, group_max=group_max,
                               magnitude_dims=index_dims, magnitude="slabs")
            qq, P = harness.pair_inputs(wl, b, h)[2:]
            slabs, _ = oracle.magnitude_slabs(qq, P, r, index_dims, group_max)
            moved += slabs.tolist() != list(range(r // 16))
    assert moved > 0


def test_scored_entry_with_leading_scorer_is_decode_attention(cuda_lib):
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[5000, 123], k=200, recent_window=4)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib)
    a = dev.decode()
    b = dev.decode(scorer=cuda_lib.LOKI_SCORER_LEADING)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("group_max", [False, True])
@pytest.mark.parametrize("scorer", ["LOKI_SCORER_MAGNITUDE", "LOKI_SCORER_MAGNITUDE_SLABS"])
def test_magnitude_scorer_with_every_dim_is_leading(cuda_lib, group_max, scorer):
    """r = index_dims: every dim (slab) is chosen, in ascending order, so a
    magnitude scorer computes what the leading scorer does, bit for bit."""
    s = spec(num_q_heads=4, num_kv_heads=1, seq_lens=[4000, 900], r=64, k=100, recent_window=2)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=64)
    a = dev.decode(group_max=group_max)
    b = dev.decode(group_max=group_max, scorer=getattr(cuda_lib, scorer))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------------------------------------------------
# Asymmetric score factors: key index k A_k, append, decode with q A_q
# ---------------------------------------------------------------------------

def saki_inputs(wl, index_dims):
    """Keys in the original basis, and per kv head the oracle's closed-form
    factors A_q, A_k [Hkv, d, index_dims] calibrated on the head's cached keys
    plus fresh key draws, and on fresh query batches: at least 4 d samples of
    each, so that both second moments are well conditioned."""
    s = wl.spec
    g, d = s.group, s.head_dim
    K_orig = unrotated_keys(wl)
    need = 4 * d
    qcal = torch.cat([synth.draw_query_batch(s, 100 + i) for i in range(-(-need // (s.batch * g)))])
    kcal = torch.cat([synth.draw_new_tokens(s, 300 + i)[0] for i in range(-(-need // s.batch))])
    Aq = torch.empty(s.num_kv_heads, d, index_dims)
    Ak = torch.empty_like(Aq)
    for h in range(s.num_kv_heads):
        Kcal = torch.cat([K_orig[b, h, :L] for b, L in enumerate(s.seq_lens)] + [kcal[:, h]]).double().numpy()
        Qcal = qcal[:, h * g:(h + 1) * g].reshape(-1, d).double().numpy()
        a, b, _ = oracle.saki_factors(Qcal, Kcal, index_dims)
        Aq[h], Ak[h] = torch.from_numpy(a), torch.from_numpy(b)
    return K_orig, Aq, Ak


def check_index_rows(got, k, A, dtype):
    """Index rows against the oracle's round(k A): equal, except where the
    exact value lies within the fp32 summation bound of the rounding
    midpoint between the two."""
    want = oracle.index_keys(k, A, dtype)
    exact = k @ A
    bound = k.shape[1] * 2.0 ** -24 * (np.abs(k)[:, :, None] * np.abs(A)[None]).sum(axis=1)
    mism = got != want
    assert np.all(np.abs(exact[mism] - (got[mism] + want[mism]) / 2) <= bound[mism])
    return int(mism.sum())


@pytest.mark.parametrize("dtype,D,I,lens", [("bf16", 128, 32, [300, 1000, 0, 1, 129]), ("f32", 64, 64, [257, 40]),
                                            ("bf16", 64, 16, [70])])
def test_index_keys_matches_oracle(cuda_lib, dtype, D, I, lens):
    s = spec(num_q_heads=4, num_kv_heads=2, seq_lens=lens, head_dim=D, dtype=dtype, r=16)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=I)
    K_orig, _, Ak = saki_inputs(wl, I)
    cuda_lib.loki_index_keys(dev.cache, dev.batch, K_orig.cuda(), Ak.cuda().contiguous())
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    for b, L in enumerate(lens):
        for h in range(s.num_kv_heads):
            K, V, X = read_pair(dev, b, h, L)
            assert torch.equal(K, wl.Kt[b, h, :L]) and torch.equal(V, wl.V[b, h, :L])
            check_index_rows(X.double().numpy(), K_orig[b, h, :L].double().numpy(), Ak[h].double().numpy(), dtype)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_append_asym_matches_oracle_and_index_keys(cuda_lib, dtype, D):
    """The appended index row is round(k_new A_k), and bit-identical to the
    row loki_index_keys writes for the same key."""
    s = spec(num_q_heads=8, num_kv_heads=4, seq_lens=[31, 32, 100, 0], head_dim=D, dtype=dtype)
    wl = synth.make_workload(s)
    I = 32
    dev = harness.Device(wl, cuda_lib, index_dims=I)
    K_orig, _, Ak = saki_inputs(wl, I)
    Ak_dev = Ak.cuda().contiguous()
    k_new, v_new = synth.draw_new_tokens(s, step=0)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
    cuda_lib.loki_append_keys_asym(dev.cache, batch, k_new.cuda(), v_new.cuda(), dev.P, Ak_dev)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    appended = {}
    for b, L in enumerate(lens.tolist()):
        for h in range(s.num_kv_heads):
            K, V, X = read_pair(dev, b, h, L)
            assert torch.equal(V[L - 1], v_new[b, h])
            assert torch.equal(K[:L - 1], wl.Kt[b, h, :L - 1])
            check_index_rows(X[L - 1:].double().numpy(), k_new[b, h][None].double().numpy(),
                             Ak[h].double().numpy(), dtype)
            appended[(b, h)] = X[L - 1].clone()
    K_full = torch.zeros(s.batch, s.num_kv_heads, int(lens.max()), D, dtype=K_orig.dtype)
    K_full[:, :, :K_orig.shape[2]] = K_orig[:, :, :int(lens.max())]
    for b, L in enumerate(lens.tolist()):
        K_full[b, :, L - 1] = k_new[b]
    cuda_lib.loki_index_keys(dev.cache, batch, K_full.cuda(), Ak_dev)
    torch.cuda.synchronize()
    for (b, h), row in appended.items():
        assert torch.equal(read_pair(dev, b, h, lens[b].item())[2][-1], row)


@pytest.mark.parametrize("dtype,D,Hq,Hkv,I,r,group_max,lens", [
    ("bf16", 128, 8, 2, 32, 32, False, [20000, 3000, 777, 33]),
    ("bf16", 128, 16, 2, 64, 16, True, [3000, 777]),
    ("f32", 64, 4, 1, 64, 48, False, [3000, 0, 500]),
    ("bf16", 64, 2, 2, 32, 32, True, [2500, 1]),
])
def test_asym_decode_matches_oracle(cuda_lib, dtype, D, Hq, Hkv, I, r, group_max, lens):
    s = spec(dtype=dtype, head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, seq_lens=lens, r=r, k=150,
             recent_window=5)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=I)
    K_orig, Aq, Ak = saki_inputs(wl, I)
    cuda_lib.loki_index_keys(dev.cache, dev.batch, K_orig.cuda(), Ak.cuda().contiguous())
    out = torch.full((s.batch, Hq, D), float("nan"), device="cuda")
    sel = torch.full((s.batch, Hkv, s.k + s.recent_window), -7, dtype=torch.int32, device="cuda")
    cuda_lib.loki_decode_attention_asym(dev.cache, dev.batch, dev.q, dev.P, Aq.cuda().contiguous(), r, s.k, out,
                                        recent_window=s.recent_window,
                                        group_reduce=cuda_lib.LOKI_GROUP_MAX if group_max else cuda_lib.LOKI_GROUP_SUM,
                                        selected_idx=sel)
    torch.cuda.synchronize()
    assert cuda_lib.loki_device_error() == 0
    out, sel = out.cpu(), sel.cpu()
    for b, L in enumerate(lens):
        for h in range(Hkv):
            Kidx = oracle.index_keys(K_orig[b, h, :L].double().numpy(), Ak[h].double().numpy(), dtype)
            harness.check_pair(wl, b, h, out, sel, r, s.k, s.recent_window, group_max=group_max,
                               asym=(Kidx, Aq[h].double().numpy()))


@pytest.mark.parametrize("group_max", [False, True])
def test_asym_decode_with_pca_factor_is_leading(cuda_lib, group_max):
    """A_q = the first index_dims columns of P on an index that holds the
    keys' leading dims: q A_q is summed like q_hat, so the asymmetric decode
    is the leading decode bit for bit."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[6000, 900], r=32, k=200, recent_window=3)
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=64)
    a = dev.decode(group_max=group_max)
    out = torch.full_like(a[0], float("nan")).cuda()
    sel = torch.full_like(a[1], -7).cuda()
    Aq = dev.P[:, :, :64].contiguous()
    cuda_lib.loki_decode_attention_asym(dev.cache, dev.batch, dev.q, dev.P, Aq, s.r, s.k, out,
                                        recent_window=s.recent_window,
                                        group_reduce=cuda_lib.LOKI_GROUP_MAX if group_max else cuda_lib.LOKI_GROUP_SUM,
                                        selected_idx=sel)
    torch.cuda.synchronize()
    assert torch.equal(a[0], out.cpu()) and torch.equal(a[1], sel.cpu())

@pytest.mark.parametrize("dtype,W", [("bf16", 8), ("f32", 0)])
def test_decode_step_host_equals_decode_step(cuda_lib, dtype, W):
    """loki_decode_step_host (inputs and output in pinned host memory, copies
    on the stream) gives bit for bit what loki_decode_step gives."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[1999, 3000], k=200, recent_window=W, dtype=dtype)
    wl = synth.make_workload(s)
    k_new, v_new = synth.draw_new_tokens(s, step=4)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    outs = []
    for host in (False, True):
        dev = harness.Device(wl, cuda_lib)
        dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
        if host:
            out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan")).pin_memory()
            staging = torch.empty(cuda_lib.loki_decode_step_host_bytes(dev.cache, dev.batch, s.num_q_heads),
                                  dtype=torch.uint8, device="cuda")
            cuda_lib.loki_decode_step_host(dev.cache, dev.batch, k_new.pin_memory(), v_new.pin_memory(),
                                           wl.q.pin_memory(), dev.P, s.r, s.k, out, staging, recent_window=W)
            torch.cuda.synchronize()
            outs.append(out.clone())
        else:
            out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device="cuda")
            cuda_lib.loki_decode_step(dev.cache, dev.batch, k_new.cuda(), v_new.cuda(), dev.q, dev.P, s.r, s.k, out,
                                      recent_window=W)
            torch.cuda.synchronize()
            outs.append(out.cpu())
    assert cuda_lib.loki_device_error(clear=True) == 0
    assert not torch.isnan(outs[1]).any()
    assert torch.equal(outs[0], outs[1])


def test_decode_step_host_in_place_and_staged_paths_agree(cuda_lib):
    """The host-buffer step's two paths give what loki_decode_step gives, bit
    for bit: pinned buffers (read and written in place by the kernels, here
    as views at an offset inside larger pinned tensors), pageable buffers
    (staged copies), and pinned buffers with q 2 bytes off 16-byte alignment
    (staged copies as well)."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[1500, 2100], k=150, recent_window=8)
    wl = synth.make_workload(s)
    k_new, v_new = synth.draw_new_tokens(s, step=6)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    shape = (s.batch, s.num_q_heads, s.head_dim)

    def pinned_view(t, shift):
        flat = torch.zeros(t.numel() + 64, dtype=t.dtype).pin_memory()
        v = flat[shift:shift + t.numel()].view(t.shape)
        v.copy_(t)
        return v

    outs = {}
    for mode in ("device", "in_place", "pageable", "unaligned_q"):
        dev = harness.Device(wl, cuda_lib)
        dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
        if mode == "device":
            out = torch.full(shape, float("nan"), device="cuda")
            cuda_lib.loki_decode_step(dev.cache, dev.batch, k_new.cuda(), v_new.cuda(), dev.q, dev.P, s.r, s.k, out,
                                      recent_window=8)
            torch.cuda.synchronize()
            outs[mode] = out.cpu()
            continue
        if mode == "in_place":
            hk, hv, hq = pinned_view(k_new, 8), pinned_view(v_new, 24), pinned_view(wl.q, 16)
            hout = pinned_view(torch.full(shape, float("nan")), 4)
        elif mode == "pageable":
            hk, hv, hq = k_new.clone(), v_new.clone(), wl.q.clone()
            hout = torch.full(shape, float("nan"))
        else:
            hk, hv = k_new.pin_memory(), v_new.pin_memory()
            hq = pinned_view(wl.q, 1)   # 2 bytes past a 16-byte boundary (bf16)
            assert hq.data_ptr() % 16 == 2
            hout = torch.full(shape, float("nan")).pin_memory()
        staging = torch.full((cuda_lib.loki_decode_step_host_bytes(dev.cache, dev.batch, s.num_q_heads),), 0xAB,
                             dtype=torch.uint8, device="cuda")
        cuda_lib.loki_decode_step_host(dev.cache, dev.batch, hk, hv, hq, dev.P, s.r, s.k, hout, staging,
                                       recent_window=8)
        torch.cuda.synchronize()
        outs[mode] = hout.clone()
        # the in-place path leaves the staging buffer alone; the copies go through it
        assert bool((staging == 0xAB).all()) == (mode == "in_place"), mode
    assert cuda_lib.loki_device_error(clear=True) == 0
    assert not torch.isnan(outs["device"]).any()
    for mode in ("in_place", "pageable", "unaligned_q"):
        assert torch.equal(outs[mode], outs["device"]), mode


def test_decode_step_host_in_a_cuda_graph(cuda_lib):
    """The host-buffer step captured once into a CUDA graph and replayed with
    new host inputs written in place gives what an eager call gives."""
    s = spec(num_q_heads=8, num_kv_heads=2, seq_lens=[1200, 2500], k=100, recent_window=4)
    wl = synth.make_workload(s)
    lens = torch.tensor([n + 1 for n in s.seq_lens], dtype=torch.int32)
    dev = harness.Device(wl, cuda_lib)
    dev.batch = cuda_lib.Batch(wl.block_table.cuda(), lens.cuda(), int(lens.max()))
    staging = torch.empty(cuda_lib.loki_decode_step_host_bytes(dev.cache, dev.batch, s.num_q_heads),
                          dtype=torch.uint8, device="cuda")
    hk, hv = (t.pin_memory() for t in synth.draw_new_tokens(s, step=0))
    hq = wl.q.clone().pin_memory()
    hout = torch.empty(s.batch, s.num_q_heads, s.head_dim).pin_memory()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        cuda_lib.loki_decode_step_host(dev.cache, dev.batch, hk, hv, hq, dev.P, s.r, s.k, hout, staging,
                                       recent_window=4, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            cuda_lib.loki_decode_step_host(dev.cache, dev.batch, hk, hv, hq, dev.P, s.r, s.k, hout, staging,
                                           recent_window=4, stream=stream)
    results = []
    for step in (1, 2):
        k_new, v_new = synth.draw_new_tokens(s, step=step)
        hk.copy_(k_new)
        hv.copy_(v_new)
        hq.copy_(synth.draw_query_batch(s, step))
        g.replay()
        torch.cuda.synchronize()
        graph_out = hout.clone()
        eager = torch.empty_like(hout).pin_memory()
        cuda_lib.loki_decode_step_host(dev.cache, dev.batch, hk, hv, hq, dev.P, s.r, s.k, eager, staging,
                                       recent_window=4)
        torch.cuda.synchronize()
        results.append((graph_out, eager.clone()))
    assert cuda_lib.loki_device_error(clear=True) == 0
    for a, b in results:
        assert not torch.isnan(a).any()
        assert torch.equal(a, b)
    assert not torch.equal(results[0][0], results[1][0])   # the replays saw the new inputs


def test_per_dim_scorer_full_size(cuda_lib):
    """The per-dimension magnitude scorer in the bench's configuration (the
    32768-token GQA workload, an index of all 128 dims, r 32, k 2048 + 64):
    sampled pairs whose r-th and (r+1)-th dim magnitudes are apart by more than
    the selection margin, against the oracle's per-dimension decode."""
    import oracle
    s = synth.named_spec("gqa32x8-d128-L32768-bf16")
    wl = synth.make_workload(s)
    dev = harness.Device(wl, cuda_lib, index_dims=s.head_dim)
    out, sel = dev.decode(scorer=cuda_lib.LOKI_SCORER_MAGNITUDE)
    assert cuda_lib.loki_device_error() == 0
    checked = 0
    for b in range(s.batch):
        for h in range(s.num_kv_heads):
            _, _, qq, P = harness.pair_inputs(wl, b, h)
            _, w = oracle.magnitude_dims(qq, P, s.r, s.head_dim)
            w = np.sort(w)[::-1]
            if w[s.r - 1] - w[s.r] <= harness.SLAB_MARGIN * w[s.r - 1]:
                continue
            harness.check_pair(wl, b, h, out, sel, s.r, s.k, s.recent_window, magnitude_dims=s.head_dim,
                               magnitude="dims")
            checked += 1
            if checked == 3:
                return
    assert checked > 0, "no pair with a dim-selection margin"

