"""The benchmark's host-side helpers, without a GPU: its calibration of the
asymmetric score factors gives the oracle's rank-r operator, its byte and
token counts follow the per-sequence k, and its recall is the plain set
overlap."""
import importlib.util
import os

import numpy as np
import torch

import oracle
from rank_key_top_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_saki_calibration_gives_the_oracles_operator():
    """A_q A_k^T (the rank-r score operator, unique when the singular values
    are distinct) equals the oracle's closed form."""
    b = bench()
    rng = np.random.default_rng(5)
    d, r = 32, 8
    Q = rng.standard_normal((400, d)) * np.linspace(0.2, 3.0, d)
    K = rng.standard_normal((900, d)) @ np.diag(np.linspace(2.0, 0.3, d)) @ np.linalg.qr(rng.standard_normal((d, d)))[0]
    aq, ak = b.saki_calibration(Q, K, r)
    oq, ok, _ = oracle.saki_factors(Q, K, r)
    W, Wo = aq @ ak.T, oq @ ok.T
    assert np.abs(W - Wo).max() <= 1e-9 * np.abs(Wo).max()


def test_bytes_and_tokens_follow_the_per_sequence_k():
    b = bench()
    s = synth.named_spec("paged-b16-mha32-L4k-16k-bf16")
    want = sum(s.num_kv_heads * (L * s.r + 2 * min(L // 8, L) * s.head_dim) * 2 for L in s.seq_lens)
    want += s.batch * s.num_q_heads * s.head_dim * 6
    assert b.algorithmic_bytes(s) == want
    assert b.attended_tokens(s) == sum(s.num_q_heads * (L // 8) for L in s.seq_lens)
    c4 = synth.named_spec("gqa32x8-d128-L32768-bf16")
    assert b.algorithmic_bytes(c4) == 203620352
    assert b.attended_tokens(c4) == 8 * 32 * 2112


def test_kept_set_recall():
    b = bench()
    a = torch.tensor([[[0, 1, 2, -1]], [[5, 6, 7, 8]]])
    ref = torch.tensor([[[1, 2, 3, -1]], [[5, 6, 7, 8]]])
    assert abs(b.kept_set_recall(a, ref) - (2 / 3 + 1.0) / 2) < 1e-12
