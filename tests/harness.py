"""Shared plumbing of the GPU parity tests: upload a synthetic workload, run
the CUDA path through the C ABI, and compare with the oracle on the same
inputs (set parity with the tie band, output parity on the GPU's own set)."""
import numpy as np
import torch

import oracle
from rank_key_top_b200 import synth

BF16_RTOL = 2e-3   # max normwise relative error of outputs, bf16 caches
F32_RTOL = 1e-5    # the same for fp32 caches
TIE_BAND = 1e-3    # selected sets may differ only where |s_t - s_(k)| <= TIE_BAND |s_(k)|
SLAB_MARGIN = 1e-3  # magnitude scorers: the last kept dim (slab) must beat the first dropped one by this much


def tol_for(spec):
    return BF16_RTOL if spec.dtype == "bf16" else F32_RTOL


class Device:
    """A workload's cache and inputs on the GPU."""

    def __init__(self, wl, loki, device="cuda", max_seq_len=None, index_dims=None):
        s = wl.spec
        self.wl, self.loki = wl, loki
        if index_dims is None:
            index_dims = max(s.r, min(64, s.head_dim))
        self.index_dims = index_dims
        self.cache = loki.Cache(wl.num_blocks, s.num_kv_heads, s.head_dim, synth.torch_dtype(s.dtype), device,
                                index_dims=index_dims)
        self.batch = loki.Batch(wl.block_table.to(device), wl.seq_lens.to(device),
                                max_seq_len if max_seq_len is not None else s.max_seq_len)
        self.q = wl.q.to(device)
        self.P = wl.P.to(device).contiguous()
        self.k_per_seq = wl.k_per_seq.to(device) if wl.k_per_seq is not None else None
        if s.max_seq_len > 0:
            loki.loki_prefill_cache(self.cache, self.batch, wl.Kt.to(device), wl.V.to(device))

    def decode(self, r=None, k=None, W=None, group_max=False, q=None, scale=0.0, scorer=None):
        s, loki = self.wl.spec, self.loki
        r = s.r if r is None else r
        k = s.k if k is None else k
        W = s.recent_window if W is None else W
        q = self.q if q is None else q
        out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device=q.device)
        sel = torch.full((s.batch, s.num_kv_heads, k + W), -7, dtype=torch.int32, device=q.device)
        reduce = loki.LOKI_GROUP_MAX if group_max else loki.LOKI_GROUP_SUM
        if scorer is None:
            loki.loki_decode_attention(self.cache, self.batch, q, self.P, r, k, out,
                                       k_per_seq=self.k_per_seq, recent_window=W, group_reduce=reduce,
                                       scale=scale, selected_idx=sel)
        else:
            loki.loki_decode_attention_scored(self.cache, self.batch, q, self.P, r, k, out, scorer=scorer,
                                              k_per_seq=self.k_per_seq, recent_window=W,
                                              group_reduce=reduce, scale=scale, selected_idx=sel)
        torch.cuda.synchronize()
        return out.cpu(), sel.cpu()

    def dense(self, q=None, scale=0.0):
        s, loki = self.wl.spec, self.loki
        q = self.q if q is None else q
        out = torch.full((s.batch, s.num_q_heads, s.head_dim), float("nan"), device=q.device)
        ws = torch.empty(max(loki.loki_dense_workspace_bytes(self.cache, self.batch, s.num_q_heads), 16),
                         dtype=torch.uint8, device=q.device)
        loki.loki_dense_attention(self.cache, self.batch, q, self.P, out, ws, scale=scale)
        torch.cuda.synchronize()
        return out.cpu()


def pair_inputs(wl, b, h, q=None):
    """The exact stored values of one (sequence, kv head) pair, as float64."""
    s = wl.spec
    L = s.seq_lens[b]
    g = s.group
    q = wl.q if q is None else q
    return (wl.Kt[b, h, :L].double().numpy(), wl.V[b, h, :L].double().numpy(),
            q[b, h * g:(h + 1) * g].double().numpy(), wl.P[h].double().numpy())


def check_pair(wl, b, h, out_gpu, sel_gpu, r, k, W, group_max=False, scale=0.0, q=None, rtol=None,
               inputs=None, magnitude_dims=None, asym=None, magnitude="slabs"):
    """Set parity (with the tie band) and output parity for one pair.

    magnitude_dims: the key index's width when a magnitude scorer ran; with
    magnitude="dims" the oracle chooses single dims (AQUA's per-dimension
    selection), with "slabs" whole 16-dim slabs, from the same queries. The
    input must separate the last kept dim (slab) from the first dropped one by
    SLAB_MARGIN, so that both sides' choice is the same whatever their
    precision.
    asym: (Kidx, A_q) of the pair when the asymmetric scorer ran: the
    oracle's own key-index rows round(k A_k) and the query factor.
    Returns (output error on the GPU's set, output error on the oracle's set)."""
    s = wl.spec
    g = s.group
    L = s.seq_lens[b]
    kb = int(wl.k_per_seq[b]) if wl.k_per_seq is not None else k
    Kt, V, qq, P = inputs if inputs is not None else pair_inputs(wl, b, h, q)
    if asym is not None:
        res = oracle.decode_pair_asym(Kt, V, asym[0], qq, P, asym[1], r, kb, W=W, group_max=group_max,
                                      scale=scale)
    elif magnitude_dims is None:
        res = oracle.decode_pair(Kt, V, qq, P, r=r, k=kb, W=W, group_max=group_max, scale=scale)
    elif magnitude == "dims":
        res = oracle.decode_pair_dims(Kt, V, qq, P, r, kb, magnitude_dims, W=W, group_max=group_max, scale=scale)
        w = np.sort(res.weight)[::-1]
        if r < w.size:
            assert w[r - 1] - w[r] > SLAB_MARGIN * w[r - 1], f"pair {(b, h)}: input without a dim-selection margin"
    else:
        res = oracle.decode_pair_magnitude(Kt, V, qq, P, r, kb, magnitude_dims, W=W, group_max=group_max,
                                           scale=scale)
        e = np.sort(res.energy)[::-1]
        if r // 16 < e.size:
            assert e[r // 16 - 1] - e[r // 16] > SLAB_MARGIN * e[r // 16 - 1], (
                f"pair {(b, h)}: input without a slab-selection margin")
    width = k + W
    row = sel_gpu[b, h].numpy()
    n = res.n_sel
    assert row.shape[0] == width
    assert np.all(row[n:] == -1), f"pair {(b, h)}: padding"
    T_gpu = row[:n]
    assert np.all(T_gpu >= 0) and np.all(T_gpu < max(L, 1)), f"pair {(b, h)}: index range"
    assert np.all(np.diff(T_gpu) > 0), f"pair {(b, h)}: not ascending / duplicates"
    T_ref = res.sel[:n]
    w_eff = min(W, L)
    assert set(range(L - w_eff, L)) <= set(T_gpu.tolist()), f"pair {(b, h)}: recent window"
    diff = np.setxor1d(T_gpu, T_ref)
    if diff.size:
        band = TIE_BAND * abs(res.kth)
        assert np.all(np.abs(res.scores[diff] - res.kth) <= band), (
            f"pair {(b, h)}: {diff.size} tokens differ outside the tie band")
    qhat = oracle.rotate(qq, P)
    ref_gpu_set = oracle.attend_set(Kt, V, qhat, T_gpu, scale=scale) if n else np.zeros((g, s.head_dim))
    got = out_gpu[b, h * g:(h + 1) * g].double().numpy()
    rtol = tol_for(s) if rtol is None else rtol
    errs = []
    for ref in (ref_gpu_set, res.out):
        denom = np.abs(ref).max(axis=1)
        denom = np.where(denom > 0, denom, 1.0)
        errs.append(float((np.abs(got - ref).max(axis=1) / denom).max()))
    assert errs[0] <= rtol, f"pair {(b, h)}: output error {errs[0]:.3g} > {rtol}"
    return errs


def check_dense_pair(wl, b, h, out_gpu, scale=0.0, rtol=None):
    s = wl.spec
    g = s.group
    Kt, V, qq, P = pair_inputs(wl, b, h)
    ref = oracle.dense_pair(Kt, V, qq, P, scale=scale)
    got = out_gpu[b, h * g:(h + 1) * g].double().numpy()
    denom = np.abs(ref).max(axis=1)
    denom = np.where(denom > 0, denom, 1.0)
    err = float((np.abs(got - ref).max(axis=1) / denom).max())
    rtol = tol_for(s) if rtol is None else rtol
    assert err <= rtol, f"dense pair {(b, h)}: error {err:.3g} > {rtol}"
    return err
