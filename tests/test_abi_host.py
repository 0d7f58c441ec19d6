"""The C-ABI library without a GPU: it loads, exports every entry point that
include/loki.h declares, and rejects bad arguments on the host before any
launch. No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

from rank_key_top_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def loki():
    lib_build.build()
    from rank_key_top_b200 import loki as mod
    return mod


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "loki.h")).read()
    return sorted(set(re.findall(r"LOKI_API\s+[\w\s\*]+?\b(loki_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for must in ("loki_append_keys", "loki_decode_attention", "loki_dense_attention",
                 "loki_prefill_cache", "loki_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(loki):
    lib = ctypes.CDLL(loki.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert sorted(loki.EXPORTED) == declared_symbols()
    assert loki.loki_abi_version() == 5


def test_status_strings(loki):
    for s in range(5):
        assert loki.loki_status_string(s)
    assert loki.loki_status_string(99) == "unknown status"


def test_index_bytes(loki):
    assert loki.loki_index_bytes(10, 8, 32, loki.LOKI_BF16) == 10 * 8 * 16 * 32 * 2
    assert loki.loki_index_bytes(10, 8, 24, loki.LOKI_BF16) == 0
    assert loki.loki_index_bytes(10, 8, 0, loki.LOKI_F32) == 0


def test_cache_bytes(loki):
    assert loki.loki_cache_bytes(10, 8, 128, loki.LOKI_BF16) == 10 * 8 * 16 * 128 * 2
    assert loki.loki_cache_bytes(10, 8, 64, loki.LOKI_F32) == 10 * 8 * 16 * 64 * 4
    assert loki.loki_cache_bytes(10, 8, 96, loki.LOKI_F32) == 0
    assert loki.loki_cache_bytes(-1, 8, 128, loki.LOKI_F32) == 0
    assert loki.loki_decode_max_seq_len(128, loki.LOKI_BF16) == 262144
    assert loki.loki_decode_max_seq_len(96, loki.LOKI_BF16) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def structs(loki, *, D=128, Hkv=8, dtype=1, B=2, max_blocks=4, max_len=64, blocks=8, index_dims=32):
    c = loki.loki_cache(FAKE, FAKE, FAKE, blocks, Hkv, D, index_dims, dtype)
    b = loki.loki_batch(FAKE, FAKE, B, max_blocks, max_len)
    return c, b


def decode(loki, c, b, Hq=32, r=32, k=8, W=0, group=0, scale=0.0, q=FAKE, P=FAKE, out=FAKE):
    return loki.raw().loki_decode_attention(ctypes.byref(c), ctypes.byref(b), q, Hq, P, r, k, None, W,
                                            group, scale, out, None, None, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0, W=0), 1),            # nothing could be kept
    (dict(k=-1), 1),
    (dict(W=-2), 1),
    (dict(r=0), 1),
    (dict(r=129), 1),
    (dict(r=24), 2),                # not a multiple of 16
    (dict(Hq=30), 1),               # not a multiple of Hkv
    (dict(Hq=24), 2),               # group 3
    (dict(Hq=128), 2),              # group 16
    (dict(group=5), 1),
    (dict(scale=-1.0), 1),
    (dict(scale=float("nan")), 1),
    (dict(q=None), 1),
    (dict(P=None), 1),
    (dict(out=None), 1),
    (dict(P=FAKE + 4), 1),          # P must be 16-byte aligned (vector loads)
    (dict(q=FAKE + 8), 1),          # q must be 16-byte aligned (vector loads)
])
def test_decode_rejects(loki, kw, status):
    c, b = structs(loki)
    assert decode(loki, c, b, **kw) == status


def test_decode_rejects_bad_shapes(loki):
    c, b = structs(loki, D=96)
    assert decode(loki, c, b) == 2
    c, b = structs(loki, max_len=65)       # exceeds 16 * max_blocks_per_seq
    assert decode(loki, c, b) == 1
    c, b = structs(loki, max_blocks=20000, max_len=300000)
    assert decode(loki, c, b) == 2         # above loki_decode_max_seq_len
    c, b = structs(loki, B=-1)
    assert decode(loki, c, b) == 1
    c = loki.loki_cache(FAKE + 8, FAKE, FAKE, 8, 8, 128, 32, 1)
    _, b = structs(loki)
    assert decode(loki, c, b) == 1         # misaligned cache
    c = loki.loki_cache(FAKE, FAKE, FAKE + 4, 8, 8, 128, 32, 1)
    assert decode(loki, c, b) == 1         # misaligned index
    c = loki.loki_cache(FAKE, FAKE, FAKE, 8, 8, 128, 32, 7)
    assert decode(loki, c, b) == 1         # unknown dtype
    for bad_index in (0, 8, 24, 144):
        c = loki.loki_cache(FAKE, FAKE, FAKE, 8, 8, 128, bad_index, 1)
        assert decode(loki, c, b) == 1, bad_index
    c, b = structs(loki, index_dims=32)
    assert decode(loki, c, b, r=48) == 1   # r above the index dims
    assert loki.raw().loki_decode_attention(None, ctypes.byref(b), FAKE, 32, FAKE, 32, 8, None, 0, 0, 0.0,
                                            FAKE, None, None, 0, None) == 1


def step(loki, c, b, k_new=FAKE, v_new=FAKE, Hq=32, r=32, k=8, W=0, q=FAKE, P=FAKE, out=FAKE):
    return loki.raw().loki_decode_step(ctypes.byref(c), ctypes.byref(b), k_new, v_new, q, Hq, P, r, k, None, W,
                                       0, 0.0, out, None, None, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(k_new=None), 1),          # append arguments are checked ...
    (dict(v_new=None), 1),
    (dict(P=FAKE + 4), 1),
    (dict(k=0, W=0), 1),            # ... and so are the decode arguments, before any launch
    (dict(r=24), 2),
    (dict(Hq=24), 2),
    (dict(q=None), 1),
    (dict(out=None), 1),
])
def test_decode_step_rejects(loki, kw, status):
    c, b = structs(loki)
    assert step(loki, c, b, **kw) == status


def scored(loki, c, b, scorer, Hq=32, r=32, k=8, W=0, q=FAKE, P=FAKE, out=FAKE):
    return loki.raw().loki_decode_attention_scored(ctypes.byref(c), ctypes.byref(b), q, Hq, P, r, k, None, W,
                                                   0, 0.0, scorer, out, None, None, 0, None)


@pytest.mark.parametrize("scorer,kw,status", [
    (3, {}, 1),                     # unknown scorer
    (-1, {}, 1),
    (1, dict(r=48), 1),             # r above index_dims (32), for every scorer
    (2, dict(r=48), 1),
    (0, dict(r=48), 1),
    (1, dict(k=0, W=0), 1),
    (1, dict(Hq=24), 2),
    (1, dict(out=None), 1),
])
def test_decode_scored_rejects(loki, scorer, kw, status):
    c, b = structs(loki)
    assert scored(loki, c, b, scorer, **kw) == status


def test_asymmetric_entries_reject(loki):
    c, b = structs(loki)
    lib = loki.raw()

    def dec(Aq, r=32):
        return lib.loki_decode_attention_asym(ctypes.byref(c), ctypes.byref(b), FAKE, 32, FAKE, Aq, r, 8, None, 0,
                                              0, 0.0, FAKE, None, None, 0, None)
    assert dec(None) == 1
    assert dec(FAKE + 4) == 1
    assert dec(FAKE, r=48) == 1        # r above index_dims
    assert dec(FAKE, r=24) == 2
    assert lib.loki_append_keys_asym(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, FAKE, None, None) == 1
    assert lib.loki_append_keys_asym(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, FAKE, FAKE + 8, None) == 1
    assert lib.loki_append_keys_asym(ctypes.byref(c), ctypes.byref(b), None, FAKE, FAKE, FAKE, None) == 1
    assert lib.loki_index_keys(ctypes.byref(c), ctypes.byref(b), None, FAKE, 64, None) == 1
    assert lib.loki_index_keys(ctypes.byref(c), ctypes.byref(b), FAKE, None, 64, None) == 1
    assert lib.loki_index_keys(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE + 4, 64, None) == 1
    assert lib.loki_index_keys(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, 32, None) == 1  # max_len short
    c0, b0 = structs(loki, B=0)
    assert lib.loki_index_keys(ctypes.byref(c0), ctypes.byref(b0), None, None, 0, None) == 0
    assert lib.loki_append_keys_asym(ctypes.byref(c0), ctypes.byref(b0), None, None, None, None, None) == 0
    assert lib.loki_decode_attention_asym(ctypes.byref(c0), ctypes.byref(b0), None, 32, None, None, 32, 8, None, 0,
                                          0, 0.0, None, None, None, 0, None) == 0


def test_empty_batch_is_a_no_op(loki):
    c, b = structs(loki, B=0)
    assert decode(loki, c, b, q=None, P=None, out=None) == 0
    assert loki.raw().loki_append_keys(ctypes.byref(c), ctypes.byref(b), None, None, None, None) == 0
    assert loki.raw().loki_prefill_cache(ctypes.byref(c), ctypes.byref(b), None, None, 0, None) == 0
    assert step(loki, c, b, k_new=None, v_new=None, q=None, P=None, out=None) == 0
    assert scored(loki, c, b, 1, q=None, P=None, out=None) == 0


def test_append_and_prefill_reject(loki):
    c, b = structs(loki)
    lib = loki.raw()
    assert lib.loki_append_keys(ctypes.byref(c), ctypes.byref(b), None, FAKE, FAKE, None) == 1
    assert lib.loki_append_keys(ctypes.byref(c), ctypes.byref(b), FAKE, None, FAKE, None) == 1
    assert lib.loki_prefill_cache(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, 32, None) == 1  # max_len < max_seq_len
    assert lib.loki_prefill_cache(ctypes.byref(c), ctypes.byref(b), FAKE + 2, FAKE, 64, None) == 1


def test_prefill_rotate_rejects(loki):
    c, b = structs(loki)
    lib = loki.raw()
    assert lib.loki_prefill_rotate(ctypes.byref(c), ctypes.byref(b), None, FAKE, FAKE, 64, None) == 1
    assert lib.loki_prefill_rotate(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, None, 64, None) == 1
    assert lib.loki_prefill_rotate(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, FAKE + 4, 64, None) == 1
    assert lib.loki_prefill_rotate(ctypes.byref(c), ctypes.byref(b), FAKE, FAKE, FAKE, 32, None) == 1  # max_len short
    c0, b0 = structs(loki, B=0)
    assert lib.loki_prefill_rotate(ctypes.byref(c0), ctypes.byref(b0), None, None, None, 0, None) == 0


def test_pca_basis_rejects(loki):
    lib = loki.raw()
    assert lib.loki_pca_basis(None, 2, 100, 128, 1, FAKE, None, None) == 1
    assert lib.loki_pca_basis(FAKE, 2, 100, 128, 1, None, None, None) == 1
    assert lib.loki_pca_basis(FAKE, 2, 1, 128, 1, FAKE, None, None) == 1       # n < 2
    assert lib.loki_pca_basis(FAKE, 2, 100, 96, 1, FAKE, None, None) == 2      # head dim
    assert lib.loki_pca_basis(FAKE, 2, 100, 128, 7, FAKE, None, None) == 1     # dtype
    assert lib.loki_pca_basis(None, 0, 100, 128, 1, None, None, None) == 0     # no heads: no-op


def test_dense_rejects(loki):
    c, b = structs(loki)
    lib = loki.raw()
    need = lib.loki_dense_workspace_bytes(ctypes.byref(c), ctypes.byref(b), 32)
    assert need > 0
    args = lambda ws, nbytes, Hq=32: lib.loki_dense_attention(ctypes.byref(c), ctypes.byref(b), FAKE, Hq, FAKE,
                                                               0.0, FAKE, ws, nbytes, None)
    assert args(None, 0) == 3
    assert args(FAKE, need - 1) == 3
    assert args(FAKE + 16, need) == 1      # workspace must be 256-byte aligned
    assert args(FAKE, need, Hq=24) == 2



def test_decode_needs_no_workspace(loki):
    """The fused decode kernel keeps every intermediate on chip: the decode
    calls need no workspace (size 0; NULL is accepted)."""
    lib = loki.raw()
    c, b = structs(loki)
    assert lib.loki_decode_workspace_bytes(ctypes.byref(c), ctypes.byref(b), 32, 8, 0) == 0
    assert lib.loki_decode_workspace_bytes(ctypes.byref(c), ctypes.byref(b), 32, 2048, 64) == 0


def step_host(loki, c, b, k_new=FAKE, v_new=FAKE, q=FAKE, Hq=32, r=32, k=8, W=0, P=FAKE, out=FAKE, staging=FAKE,
              staging_bytes=1 << 30):
    return loki.raw().loki_decode_step_host(ctypes.byref(c), ctypes.byref(b), k_new, v_new, q, Hq, P, r, k, None, W,
                                            0, 0.0, out, staging, staging_bytes, None)


def test_decode_step_host_staging_bytes(loki):
    """k_new, v_new, q in the cache dtype and out in fp32, each region rounded up to 256 bytes."""
    c, b = structs(loki, B=2, Hkv=8, D=128, dtype=1)
    raw = loki.raw()
    kv = 2 * 8 * 128 * 2            # 4096 bytes each
    q = 2 * 32 * 128 * 2            # 16384
    o = 2 * 32 * 128 * 4            # 32768
    assert raw.loki_decode_step_host_bytes(ctypes.byref(c), ctypes.byref(b), 32) == 2 * kv + q + o
    c, b = structs(loki, B=1, Hkv=3, D=64, dtype=0)
    up = lambda x: (x + 255) // 256 * 256
    assert raw.loki_decode_step_host_bytes(ctypes.byref(c), ctypes.byref(b), 3) == (
        2 * up(3 * 64 * 4) + up(3 * 64 * 4) + up(3 * 64 * 4))
    assert raw.loki_decode_step_host_bytes(ctypes.byref(c), ctypes.byref(b), 0) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(k_new=None), 1),           # host buffers are required
    (dict(v_new=None), 1),
    (dict(q=None), 1),
    (dict(out=None), 1),
    (dict(staging=None), 3),         # the staging buffer must exist and be large enough
    (dict(staging_bytes=1024), 3),
    (dict(staging=FAKE + 16), 1),    # and 256-byte aligned
    (dict(k=0, W=0), 1),             # the step's own arguments, before any copy
    (dict(r=24), 2),
    (dict(P=FAKE + 4), 1),
])
def test_decode_step_host_rejects(loki, kw, status):
    c, b = structs(loki)
    assert step_host(loki, c, b, **kw) == status
