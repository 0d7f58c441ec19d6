"""The seeded input generator: shapes, determinism and value structure."""
import numpy as np
import torch

from rank_key_top_b200 import synth


def tiny_spec(**kw):
    base = dict(name="tiny", batch=2, num_q_heads=4, num_kv_heads=2, head_dim=32,
                seq_lens=[37, 100], dtype="bf16", alpha=0.8, r=8, k=10, seed=5)
    base.update(kw)
    return synth.Spec(**base)


def test_deterministic_and_shaped():
    s = tiny_spec()
    a, b = synth.make_workload(s), synth.make_workload(s)
    for name in ("P", "q", "Kt", "V", "block_table"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert a.Kt.shape == (2, 2, 100, 32) and a.q.shape == (2, 4, 32)
    assert a.Kt.dtype == torch.bfloat16 and a.P.dtype == torch.float32
    assert torch.all(a.Kt[0, :, 37:] == 0)


def test_block_table_is_a_permutation():
    s = tiny_spec(seq_lens=[37, 100, 0, 16])
    s.batch = 4
    w = synth.make_workload(s)
    per = [-(-(n + s.spare_tokens) // 16) for n in s.seq_lens]
    ids = torch.cat([w.block_table[b, :n] for b, n in enumerate(per)])
    assert sorted(ids.tolist()) == list(range(w.num_blocks))


def test_projection_is_orthonormal_and_spectrum_decays():
    s = tiny_spec(seq_lens=[4000, 4000], head_dim=64)
    w = synth.make_workload(s)
    for h in range(s.num_kv_heads):
        P = w.bases[h].P64
        np.testing.assert_allclose(P.T @ P, np.eye(64), atol=1e-12)
    col_std = w.Kt[0, 0, :4000].float().std(dim=0).numpy()
    want = np.sqrt(np.arange(1, 65) ** (-1.6) + 0.05 ** 2)
    np.testing.assert_allclose(col_std, want, rtol=0.08)


def test_outlier_basis_is_the_covariance_eigenbasis():
    s = tiny_spec(outlier_channels=4, head_dim=32)
    hb = synth.head_basis(s, 0)
    D = hb.channel_scale
    assert sorted(np.unique(D).tolist()) == [1.0, 10.0] and (D == 10).sum() == 4
    cov = D[:, None] * ((hb.U * hb.sigma ** 2) @ hb.U.T + 0.0025 * np.eye(32)) * D[None, :]
    lam = hb.pca_std ** 2
    np.testing.assert_allclose(hb.P64.T @ cov @ hb.P64, np.diag(lam), atol=1e-10)
    assert np.all(np.diff(lam) <= 1e-12)


def test_named_workloads_shapes():
    s = synth.named_spec("paged-b16-mha32-L4k-16k-bf16")
    assert len(s.seq_lens) == 16 and all(4096 <= n <= 16384 for n in s.seq_lens)
    assert s.k_per_seq == [n // 8 for n in s.seq_lens]
    s4 = synth.named_spec("gqa32x8-d128-L32768-bf16")
    assert (s4.group, s4.r, s4.k, s4.recent_window) == (4, 32, 2048, 64)
