"""The dense-attention entry point that allocates nothing.

Some callers cannot allocate device memory: a serving engine that gives all
device memory to its own arena at start-up, a plugin host without an
allocator, or code that must not call cudaMalloc because it can synchronise
the device. loki_dense_attention_static serves them with a scratch array
built into the library instead of a caller workspace. These tests call it
through the C ABI and check it against loki_dense_attention (caller
workspace) on two calls in a row (a larger batch, then a smaller one), check
that the calls take no device memory, and that sizes beyond the array are
rejected before any launch. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from rank_key_top_b200 import synth
from tests import harness

pytestmark = pytest.mark.gpu


def static_call(cuda_lib, dev, out):
    return cuda_lib.raw().loki_dense_attention_static(
        ctypes.byref(dev.cache.struct), ctypes.byref(dev.batch.struct), ctypes.c_void_p(dev.q.data_ptr()),
        dev.wl.spec.num_q_heads, ctypes.c_void_p(dev.P.data_ptr()), 0.0, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_matches_caller_workspace(cuda_lib):
    """Two calls in a row, the first on a larger batch than the second (so the
    second must not read anything the first left in the shared array), each
    compared with loki_dense_attention on a caller workspace; the calls take
    no device memory (free memory is unchanged around them)."""
    big = synth.Spec("static-scratch-big", batch=4, num_q_heads=8, num_kv_heads=2, head_dim=128,
                     seq_lens=[9000, 3000, 1777, 5000], dtype="bf16", alpha=0.8, r=32, k=64, seed=37)
    small = synth.Spec("static-scratch", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128,
                       seq_lens=[3000, 1777, 40], dtype="bf16", alpha=0.8, r=32, k=64, seed=31)
    devs = [harness.Device(synth.make_workload(s), cuda_lib) for s in (big, small)]
    refs = [d.dense() for d in devs]
    outs = [torch.full((d.wl.spec.batch, d.wl.spec.num_q_heads, d.wl.spec.head_dim), float("nan"), device="cuda")
            for d in devs]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for d, out in zip(devs, outs):
        status = static_call(cuda_lib, d, out)
        assert status == cuda_lib.LOKI_OK, cuda_lib.loki_status_string(status)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    for call, (out, ref) in enumerate(zip(outs, refs)):
        got = out.cpu()
        assert torch.isfinite(got).all(), call
        rel = float((got - ref).abs().max() / ref.abs().max())
        assert rel <= harness.BF16_RTOL, (call, rel)
    assert cuda_lib.loki_device_error() == 0


def test_static_scratch_rejects_sizes_beyond_the_array(cuda_lib):
    table = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = cuda_lib.Cache(1, 1, 128, torch.bfloat16)
    # one sequence long enough that the split partials exceed the array
    max_len = 16_000_000
    batch = cuda_lib.loki_batch(table.data_ptr(), lens.data_ptr(), 1, max_len // 16, max_len)
    need = cuda_lib.raw().loki_dense_workspace_bytes(ctypes.byref(cache.struct), ctypes.byref(batch), 4)
    assert need > cuda_lib.LOKI_DENSE_STATIC_SCRATCH_BYTES
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    P = torch.zeros(1, 128, 128, device="cuda")
    out = torch.zeros(1, 4, 128, device="cuda")
    status = cuda_lib.raw().loki_dense_attention_static(
        ctypes.byref(cache.struct), ctypes.byref(batch), ctypes.c_void_p(q.data_ptr()), 4,
        ctypes.c_void_p(P.data_ptr()), 0.0, ctypes.c_void_p(out.data_ptr()), None)
    assert status == cuda_lib.LOKI_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 0)
