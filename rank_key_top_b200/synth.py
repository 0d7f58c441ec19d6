"""Seeded synthetic inputs for Loki-style sparse decode attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no projection of keys by P, no scoring, no selection, no
attention). Both the CUDA path and the reference oracle consume what it makes.

Key model (the workloads' recipe): keys K = Z diag(sigma) U^T + 0.05 N with U a
seeded random orthonormal d x d matrix, Z, N ~ N(0, 1), sigma_j = j^-alpha, and
the projection P = U. The cache holds keys in the PCA basis, K P. Because the
rows of N are isotropic, N U is again i.i.d. N(0, 1), so K P has exactly the
distribution of Z diag(sigma) + 0.05 N'. The generator draws the cached keys
directly in that form (no product by P is taken here). Queries are drawn like
a key row in the original basis, q = z diag(sigma) U^T + 0.05 n, which is the
recipe itself.

Long-context workload with outlier channels: four of the d original-basis
channels (a seeded choice per kv head) are scaled by 10, so the key covariance
is S = D (U diag(sigma^2) U^T + 0.05^2 I) D. P is its eigenbasis (columns by
descending eigenvalue lambda; the offline PCA calibration in the limit of many
calibration keys) and cached keys are drawn as z * sqrt(lambda), which is the
distribution of K P. Queries are drawn as (z diag(sigma) U^T + 0.05 n) D.

Values V ~ N(0, 1). Everything is rounded to the cache type (bf16 or fp32)
with torch's round-to-nearest-even conversion.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

BLOCK_TOKENS = 16


@dataclass
class Spec:
    """Shape and value structure of one synthetic decode workload."""
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    seq_lens: List[int]
    dtype: str                 # "bf16" or "f32"
    alpha: float               # sigma_j = j^-alpha
    r: int
    k: int                     # k for every sequence, or the maximum of k_per_seq
    k_per_seq: Optional[List[int]] = None
    recent_window: int = 0
    outlier_channels: int = 0  # original-basis channels scaled by outlier_scale
    outlier_scale: float = 10.0
    seed: int = 0
    spare_tokens: int = BLOCK_TOKENS  # free slots per sequence for appends
    shuffle_blocks: bool = True

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_seq_len(self) -> int:
        return max(self.seq_lens) if self.seq_lens else 0


def named_spec(name: str, **override) -> Spec:
    """The five workloads, by what they are.

    single-head-d64-L1024-f32      batch 1, one head, d 64, L 1024, fp32,
                                   sigma_j = j^-1, r 16, k 128
    mha32-d128-L4096-bf16          Llama-2-7B-shaped layer: batch 1, 32 MHA
                                   heads, d 128, L 4096, r 32, k 512
    paged-b16-mha32-L4k-16k-bf16   batch 16, 32 MHA heads, L_b ~ U[4096, 16384],
                                   paged (16-token blocks, shuffled), r 32,
                                   k = floor(L_b / 8)
    gqa32x8-d128-L32768-bf16       Llama-3-8B-shaped GQA: batch 8, 32 query / 8
                                   kv heads, L 32768, r 32, k 2048, 64 recent
    gqa32x8-d128-L131072-bf16-outliers
                                   batch 2, 32 / 8 heads, L 131072, 4 of 128
                                   channels x10; r and k set per case
                                   (defaults r 32, k L/16)
    """
    if name == "single-head-d64-L1024-f32":
        s = Spec(name, 1, 1, 1, 64, [1024], "f32", 1.0, r=16, k=128, seed=1001)
    elif name == "mha32-d128-L4096-bf16":
        s = Spec(name, 1, 32, 32, 128, [4096], "bf16", 0.8, r=32, k=512, seed=1002)
    elif name == "paged-b16-mha32-L4k-16k-bf16":
        rng = np.random.default_rng(1003)
        lens = [int(x) for x in rng.integers(4096, 16384, size=16, endpoint=True)]
        s = Spec(name, 16, 32, 32, 128, lens, "bf16", 0.8, r=32, k=max(lens) // 8,
                 k_per_seq=[n // 8 for n in lens], seed=1003)
    elif name == "gqa32x8-d128-L32768-bf16":
        s = Spec(name, 8, 32, 8, 128, [32768] * 8, "bf16", 0.8, r=32, k=2048,
                 recent_window=64, seed=1004)
    elif name == "gqa32x8-d128-L131072-bf16-outliers":
        s = Spec(name, 2, 32, 8, 128, [131072] * 2, "bf16", 0.8, r=32, k=131072 // 16,
                 outlier_channels=4, seed=1005)
    else:
        raise KeyError(name)
    for key, val in override.items():
        setattr(s, key, val)
    return s


NAMED = [
    "single-head-d64-L1024-f32",
    "mha32-d128-L4096-bf16",
    "paged-b16-mha32-L4k-16k-bf16",
    "gqa32x8-d128-L32768-bf16",
    "gqa32x8-d128-L131072-bf16-outliers",
]


def torch_dtype(name: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _gen(*seed_parts: int) -> torch.Generator:
    s = 0
    for part in seed_parts:
        s = (s * 1_000_003 + int(part) + 1) % (2 ** 62)
    return torch.Generator().manual_seed(s)


def random_orthonormal(d: int, seed: int) -> np.ndarray:
    """QR of a seeded N(0, 1) d x d matrix, signs fixed so diag(R) > 0."""
    a = torch.randn(d, d, generator=_gen(seed), dtype=torch.float64).numpy()
    qm, rm = np.linalg.qr(a)
    return qm * np.sign(np.diag(rm))[None, :]


@dataclass
class HeadBasis:
    """Per kv head: P (fp64 and fp32), the key-space scales in the PCA basis,
    and what is needed to draw original-basis query rows."""
    P64: np.ndarray            # [d, d], columns = principal directions
    pca_std: np.ndarray        # [d], std-dev of each cached (rotated) key column
    noise_std: np.ndarray      # [d], extra i.i.d. std-dev per rotated column
    U: np.ndarray              # [d, d] generator basis (original-basis structure)
    sigma: np.ndarray          # [d]
    channel_scale: np.ndarray  # [d] original-basis channel multipliers (D)


def head_basis(spec: Spec, h: int) -> HeadBasis:
    d = spec.head_dim
    U = random_orthonormal(d, spec.seed * 1000 + h)
    sigma = np.arange(1, d + 1, dtype=np.float64) ** (-spec.alpha)
    D = np.ones(d)
    if spec.outlier_channels:
        g = _gen(spec.seed, 77, h)
        idx = torch.randperm(d, generator=g)[: spec.outlier_channels].numpy()
        D[idx] = spec.outlier_scale
        cov = (U * sigma ** 2) @ U.T + 0.05 ** 2 * np.eye(d)
        cov = D[:, None] * cov * D[None, :]
        lam, vec = np.linalg.eigh(cov)
        order = np.argsort(lam)[::-1]
        lam, vec = lam[order], vec[:, order]
        # deterministic sign: the largest-magnitude entry of each column positive
        pivot = np.argmax(np.abs(vec), axis=0)
        vec = vec * np.sign(vec[pivot, np.arange(d)])[None, :]
        return HeadBasis(vec, np.sqrt(np.maximum(lam, 0.0)), np.zeros(d), U, sigma, D)
    return HeadBasis(U, sigma, np.full(d, 0.05), U, sigma, D)


@dataclass
class Workload:
    spec: Spec
    P: torch.Tensor            # [Hkv, d, d] float32 (the values passed to the library)
    q: torch.Tensor            # [B, Hq, d] cache dtype, original basis
    Kt: torch.Tensor           # [B, Hkv, Lmax, d] cache dtype, PCA basis, 0 past L_b
    V: torch.Tensor            # [B, Hkv, Lmax, d] cache dtype
    seq_lens: torch.Tensor     # [B] int32
    k_per_seq: Optional[torch.Tensor]  # [B] int32 or None
    block_table: torch.Tensor  # [B, max_blocks_per_seq] int32, physical block ids
    num_blocks: int
    bases: List[HeadBasis] = field(default_factory=list)


def draw_keys(spec: Spec, basis: HeadBasis, n: int, g: torch.Generator) -> torch.Tensor:
    """n cached-key rows in the PCA basis, float32: z * pca_std + noise_std * n'."""
    d = spec.head_dim
    z = torch.randn(n, d, generator=g)
    out = z * torch.from_numpy(basis.pca_std.astype(np.float32))
    if np.any(basis.noise_std):
        out += torch.randn(n, d, generator=g) * torch.from_numpy(basis.noise_std.astype(np.float32))
    return out


def draw_queries(spec: Spec, basis: HeadBasis, n: int, g: torch.Generator) -> np.ndarray:
    """n original-basis rows drawn like a key: (z sigma U^T + 0.05 n) D, fp64."""
    d = spec.head_dim
    z = torch.randn(n, d, generator=g, dtype=torch.float64).numpy()
    e = torch.randn(n, d, generator=g, dtype=torch.float64).numpy()
    return ((z * basis.sigma) @ basis.U.T + 0.05 * e) * basis.channel_scale


def block_layout(spec: Spec):
    """Seeded paged layout: each sequence gets ceil((L_b + spare) / 16) blocks;
    physical ids are a seeded permutation of all blocks (or in order)."""
    per_seq = [-(-(n + spec.spare_tokens) // BLOCK_TOKENS) for n in spec.seq_lens]
    num_blocks = int(sum(per_seq))
    max_blocks = max(per_seq) if per_seq else 0
    if spec.shuffle_blocks:
        phys = torch.randperm(num_blocks, generator=_gen(spec.seed, 99)).to(torch.int32)
    else:
        phys = torch.arange(num_blocks, dtype=torch.int32)
    table = torch.zeros(spec.batch, max(max_blocks, 1), dtype=torch.int32)
    pos = 0
    for b, nb in enumerate(per_seq):
        table[b, :nb] = phys[pos:pos + nb]
        pos += nb
    return table, num_blocks


def make_workload(spec: Spec, pairs=None) -> Workload:
    """Draw the whole workload. `pairs` (optional set of (b, kv_head)) limits
    the key/value draws to those pairs (others stay zero), for CPU-only uses."""
    B, Hq, Hkv, d = spec.batch, spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    g = spec.group
    dt = torch_dtype(spec.dtype)
    Lmax = spec.max_seq_len
    bases = [head_basis(spec, h) for h in range(Hkv)]
    P = torch.stack([torch.from_numpy(bb.P64) for bb in bases]).to(torch.float32)
    q = torch.empty(B, Hq, d, dtype=torch.float64)
    for b in range(B):
        for h in range(Hkv):
            qg = draw_queries(spec, bases[h], g, _gen(spec.seed, 5, b, h))
            q[b, h * g:(h + 1) * g] = torch.from_numpy(qg)
    Kt = torch.zeros(B, Hkv, Lmax, d, dtype=dt)
    V = torch.zeros(B, Hkv, Lmax, d, dtype=dt)
    for b in range(B):
        L = spec.seq_lens[b]
        for h in range(Hkv):
            if pairs is not None and (b, h) not in pairs:
                continue
            gk = _gen(spec.seed, 1, b, h)
            Kt[b, h, :L] = draw_keys(spec, bases[h], L, gk).to(dt)
            gv = _gen(spec.seed, 2, b, h)
            V[b, h, :L] = torch.randn(L, d, generator=gv).to(dt)
    table, num_blocks = block_layout(spec)
    kps = torch.tensor(spec.k_per_seq, dtype=torch.int32) if spec.k_per_seq else None
    return Workload(spec, P, q.to(dt), Kt, V, torch.tensor(spec.seq_lens, dtype=torch.int32),
                    kps, table, num_blocks, bases)


def draw_anisotropic_queries(spec: Spec, h: int, n: int, tag: int) -> np.ndarray:
    """n original-basis query rows of kv head h whose spectrum runs against
    the keys': z diag(tau) U^T with tau the keys' scales sigma in reverse
    order, fp64. These queries weight most the directions that the keys'
    variance ranks lowest, the setting in which asymmetric query/key factors
    and key PCA rank tokens differently (SAKI page, abstract)."""
    basis = head_basis(spec, h)
    z = torch.randn(n, spec.head_dim, generator=_gen(spec.seed, 11, h, tag), dtype=torch.float64).numpy()
    return (z * basis.sigma[::-1]) @ basis.U.T


def draw_new_tokens(spec: Spec, step: int):
    """Unrotated keys and values of one decode step, [B, Hkv, d] in cache type."""
    B, Hkv, d = spec.batch, spec.num_kv_heads, spec.head_dim
    dt = torch_dtype(spec.dtype)
    bases = [head_basis(spec, h) for h in range(Hkv)]
    k = torch.empty(B, Hkv, d, dtype=torch.float64)
    for b in range(B):
        for h in range(Hkv):
            k[b, h] = torch.from_numpy(draw_queries(spec, bases[h], 1, _gen(spec.seed, 7, step, b, h))[0])
    v = torch.randn(B, Hkv, d, generator=_gen(spec.seed, 8, step)).to(dt)
    return k.to(dt), v


def draw_query_batch(spec: Spec, step: int) -> torch.Tensor:
    """A fresh [B, Hq, d] query batch in cache type (another decode step)."""
    B, Hq, Hkv = spec.batch, spec.num_q_heads, spec.num_kv_heads
    g = spec.group
    bases = [head_basis(spec, h) for h in range(Hkv)]
    q = torch.empty(B, Hq, spec.head_dim, dtype=torch.float64)
    for b in range(B):
        for h in range(Hkv):
            q[b, h * g:(h + 1) * g] = torch.from_numpy(
                draw_queries(spec, bases[h], g, _gen(spec.seed, 9, step, b, h)))
    return q.to(torch_dtype(spec.dtype))
