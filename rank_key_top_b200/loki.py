"""Thin ctypes binding of libloki.so (include/loki.h), with the same names.

Argument marshalling only: torch tensors in, raw device pointers and sizes
out. Every step of the computation runs in the CUDA kernels of libloki.so;
there is no fallback. Importing this module fails loudly if the library is
missing. A non-OK status raises LokiError.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloki.so")

LOKI_OK = 0
LOKI_ERR_INVALID_ARG = 1
LOKI_ERR_UNSUPPORTED = 2
LOKI_ERR_WORKSPACE = 3
LOKI_ERR_CUDA = 4

LOKI_F32 = 0
LOKI_BF16 = 1
LOKI_GROUP_SUM = 0
LOKI_GROUP_MAX = 1
LOKI_SCORER_LEADING = 0
LOKI_SCORER_MAGNITUDE = 1
LOKI_SCORER_MAGNITUDE_SLABS = 2

LOKI_DEVERR_SEQ_LEN = 0x1
LOKI_DEVERR_BLOCK_ID = 0x2
LOKI_DEVERR_K = 0x4
LOKI_DEVERR_TIMEOUT = 0x8

LOKI_DENSE_STATIC_SCRATCH_BYTES = 16 << 20

BLOCK_TOKENS = 16

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libloki.so is not built ({LIB_PATH}); run rank_key_top_b200/build.py")
_lib = ctypes.CDLL(LIB_PATH)


class loki_cache(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("k_index", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("index_dims", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("kv_home", ctypes.c_void_p), ("k_host", ctypes.c_void_p), ("v_host", ctypes.c_void_p),
                ("num_device_pages", ctypes.c_int32), ("num_host_pages", ctypes.c_int32),
                ("kv_touch", ctypes.c_void_p)]


class loki_page_move(ctypes.Structure):
    _fields_ = [("block_in", ctypes.c_int32), ("block_out", ctypes.c_int32), ("host_page", ctypes.c_int32),
                ("device_page", ctypes.c_int32), ("freed_page", ctypes.c_int32)]


class loki_batch(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("max_seq_len", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t
_C = ctypes.POINTER(loki_cache)
_B = ctypes.POINTER(loki_batch)

_SIGS = {
    "loki_cache_bytes": (_SZ, [_I32, _I32, _I32, ctypes.c_int]),
    "loki_index_bytes": (_SZ, [_I32, _I32, _I32, ctypes.c_int]),
    "loki_prefill_cache": (ctypes.c_int, [_C, _B, _P, _P, _I32, _P]),
    "loki_prefill_rotate": (ctypes.c_int, [_C, _B, _P, _P, _P, _I32, _P]),
    "loki_pca_basis": (ctypes.c_int, [_P, _I32, ctypes.c_int64, _I32, ctypes.c_int, _P, _P, _P]),
    "loki_append_keys": (ctypes.c_int, [_C, _B, _P, _P, _P, _P]),
    "loki_decode_workspace_bytes": (_SZ, [_C, _B, _I32, _I32, _I32]),
    "loki_decode_attention": (ctypes.c_int, [_C, _B, _P, _I32, _P, _I32, _I32, _P, _I32,
                                             ctypes.c_int, ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "loki_decode_attention_scored": (ctypes.c_int, [_C, _B, _P, _I32, _P, _I32, _I32, _P, _I32,
                                                    ctypes.c_int, ctypes.c_float, ctypes.c_int, _P, _P,
                                                    _P, _SZ, _P]),
    "loki_decode_attention_asym": (ctypes.c_int, [_C, _B, _P, _I32, _P, _P, _I32, _I32, _P, _I32,
                                                  ctypes.c_int, ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "loki_append_keys_asym": (ctypes.c_int, [_C, _B, _P, _P, _P, _P, _P]),
    "loki_index_keys": (ctypes.c_int, [_C, _B, _P, _P, _I32, _P]),
    "loki_decode_step": (ctypes.c_int, [_C, _B, _P, _P, _P, _I32, _P, _I32, _I32, _P, _I32,
                                        ctypes.c_int, ctypes.c_float, _P, _P, _P, _SZ, _P]),
    "loki_decode_step_host_bytes": (_SZ, [_C, _B, _I32]),
    "loki_decode_step_host": (ctypes.c_int, [_C, _B, _P, _P, _P, _I32, _P, _I32, _I32, _P, _I32,
                                             ctypes.c_int, ctypes.c_float, _P, _P, _SZ, _P]),
    "loki_decode_max_seq_len": (_I32, [_I32, ctypes.c_int]),
    "loki_dense_workspace_bytes": (_SZ, [_C, _B, _I32]),
    "loki_dense_attention": (ctypes.c_int, [_C, _B, _P, _I32, _P, ctypes.c_float, _P, _P, _SZ, _P]),
    "loki_dense_attention_static": (ctypes.c_int, [_C, _B, _P, _I32, _P, ctypes.c_float, _P, _P]),
    "loki_offload_plan": (_I32, [_I32, _P, ctypes.POINTER(ctypes.c_int32), _P, _I32,
                                 ctypes.POINTER(loki_page_move)]),
    "loki_offload_apply": (ctypes.c_int, [_C, ctypes.POINTER(loki_page_move), _I32, _P, _P]),
    "loki_host_device_pointer": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_void_p)]),
    "loki_device_error": (ctypes.c_int, [_I32, ctypes.POINTER(ctypes.c_uint32)]),
    "loki_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "loki_abi_version": (_I32, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class LokiError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {loki_status_string(status)} (status {status})")


def _check(fn, status):
    if status != LOKI_OK:
        raise LokiError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():  # the C ABI takes dense row-major buffers
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(dt) -> int:
    return {torch.bfloat16: LOKI_BF16, torch.float32: LOKI_F32}[dt]


# --------------------------------------------------------------------------
# Struct builders
# --------------------------------------------------------------------------

class Cache:
    """Owns the key, value and key-index buffers (torch uint8) of a paged
    cache and its loki_cache struct."""

    def __init__(self, num_blocks, num_kv_heads, head_dim, dtype, device="cuda", index_dims=64):
        code = dtype_code(dtype)
        nbytes = loki_cache_bytes(num_blocks, num_kv_heads, head_dim, code)
        ibytes = loki_index_bytes(num_blocks, num_kv_heads, index_dims, code)
        if (nbytes == 0 or ibytes == 0) and num_blocks > 0:
            raise ValueError("invalid cache shape")
        self.dtype = dtype
        self.index_dims = index_dims
        self.k = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        self.v = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        self.x = torch.empty(max(ibytes, 16), dtype=torch.uint8, device=device)
        self.struct = loki_cache(self.k.data_ptr(), self.v.data_ptr(), self.x.data_ptr(), num_blocks,
                                 num_kv_heads, head_dim, index_dims, code)


class OffloadCache(Cache):
    """A cache whose key and value rows are split between device pages and
    pinned host pages (the key index stays on the device): block b's rows are
    device page home[b] for home[b] >= 0, host page -(home[b] + 1) otherwise.
    device_pages must leave one device page unused (the planner's spare).

    Keeps the host copy of the map (`home`), the spare page and the per-block
    touch counters (`touch`, device) that the sparse decode fills."""

    def __init__(self, num_blocks, num_kv_heads, head_dim, dtype, home, device_pages, host_pages,
                 device="cuda", index_dims=64):
        home = torch.as_tensor(home, dtype=torch.int32).cpu().contiguous()
        if home.numel() != num_blocks:
            raise ValueError("home needs one entry per block")
        code = dtype_code(dtype)
        dbytes = loki_cache_bytes(device_pages, num_kv_heads, head_dim, code)
        hbytes = loki_cache_bytes(host_pages, num_kv_heads, head_dim, code)
        ibytes = loki_index_bytes(num_blocks, num_kv_heads, index_dims, code)
        used = set(int(e) for e in home.tolist() if e >= 0)
        free = [pg for pg in range(device_pages) if pg not in used]
        if not free:
            raise ValueError("device_pages leaves no spare page")
        self.dtype = dtype
        self.index_dims = index_dims
        self.page_bytes = loki_cache_bytes(1, num_kv_heads, head_dim, code)
        self.k = torch.empty(max(dbytes, 16), dtype=torch.uint8, device=device)
        self.v = torch.empty(max(dbytes, 16), dtype=torch.uint8, device=device)
        self.x = torch.empty(max(ibytes, 16), dtype=torch.uint8, device=device)
        self.hk = torch.empty(max(hbytes, 16), dtype=torch.uint8, pin_memory=True)
        self.hv = torch.empty(max(hbytes, 16), dtype=torch.uint8, pin_memory=True)
        self.home = home
        self.spare = ctypes.c_int32(free[0])
        self.home_dev = home.to(device)
        self.touch = torch.zeros(max(num_blocks, 1), dtype=torch.int32, device=device)
        self.struct = loki_cache(self.k.data_ptr(), self.v.data_ptr(), self.x.data_ptr(), num_blocks,
                                 num_kv_heads, head_dim, index_dims, code,
                                 self.home_dev.data_ptr(), loki_host_device_pointer(self.hk),
                                 loki_host_device_pointer(self.hv), device_pages, host_pages,
                                 self.touch.data_ptr())


class Batch:
    """Keeps the device block table and lengths alive with their struct."""

    def __init__(self, block_table, seq_lens, max_seq_len=None):
        assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
        self.block_table = block_table.contiguous()
        self.seq_lens = seq_lens.contiguous()
        if max_seq_len is None:
            max_seq_len = int(seq_lens.max().item()) if seq_lens.numel() else 0
        B = self.seq_lens.numel()
        self.struct = loki_batch(self.block_table.data_ptr(), self.seq_lens.data_ptr(), B,
                                 self.block_table.shape[1] if B else 0, max_seq_len)


# --------------------------------------------------------------------------
# The C ABI, one Python function per entry point
# --------------------------------------------------------------------------

def loki_cache_bytes(num_blocks, num_kv_heads, head_dim, dtype_code_):
    return _lib.loki_cache_bytes(num_blocks, num_kv_heads, head_dim, dtype_code_)


def loki_index_bytes(num_blocks, num_kv_heads, index_dims, dtype_code_):
    return _lib.loki_index_bytes(num_blocks, num_kv_heads, index_dims, dtype_code_)


def loki_prefill_cache(cache, batch, k_rot, v, max_len=None, stream=None):
    max_len = k_rot.shape[2] if max_len is None else max_len
    _check("loki_prefill_cache", _lib.loki_prefill_cache(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k_rot), _ptr(v), max_len,
        _stream(stream)))


def loki_prefill_rotate(cache, batch, k, v, P, max_len=None, stream=None):
    """Prefill from unrotated keys: the library computes K~ = K P."""
    max_len = k.shape[2] if max_len is None else max_len
    _check("loki_prefill_rotate", _lib.loki_prefill_rotate(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k), _ptr(v), _ptr(P), max_len,
        _stream(stream)))


def loki_pca_basis(keys, P, eigvals=None, stream=None):
    """P[h] from calibration keys [heads][n][d] (device, bf16 or fp32)."""
    H, n, d = keys.shape
    _check("loki_pca_basis", _lib.loki_pca_basis(_ptr(keys), H, n, d, dtype_code(keys.dtype), _ptr(P),
                                                 _ptr(eigvals), _stream(stream)))


def loki_append_keys(cache, batch, k_new, v_new, P, stream=None):
    _check("loki_append_keys", _lib.loki_append_keys(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k_new), _ptr(v_new), _ptr(P),
        _stream(stream)))


def loki_decode_workspace_bytes(cache, batch, num_q_heads, k, recent_window=0):
    return _lib.loki_decode_workspace_bytes(ctypes.byref(cache.struct), ctypes.byref(batch.struct),
                                            num_q_heads, k, recent_window)


def decode_workspace(cache, batch, num_q_heads, k, recent_window=0, device="cuda"):
    """A device buffer of loki_decode_workspace_bytes() bytes for the decode
    calls, or None when they need none."""
    n = loki_decode_workspace_bytes(cache, batch, num_q_heads, k, recent_window)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def _workspace(workspace, cache, batch, q, k, recent_window):
    """The caller's workspace, or one allocated for this call (torch's caching
    allocator) when none is given and the call needs one."""
    if workspace is None:
        workspace = decode_workspace(cache, batch, q.shape[1], k, recent_window, q.device)
    return workspace, (workspace.numel() * workspace.element_size() if workspace is not None else 0)


def loki_decode_attention(cache, batch, q, P, r, k, out, k_per_seq=None, recent_window=0,
                          group_reduce=LOKI_GROUP_SUM, scale=0.0, selected_idx=None,
                          workspace=None, stream=None):
    workspace, ws_bytes = _workspace(workspace, cache, batch, q, k, recent_window)
    _check("loki_decode_attention", _lib.loki_decode_attention(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(q), q.shape[1], _ptr(P), r, k,
        _ptr(k_per_seq), recent_window, group_reduce, scale, _ptr(out), _ptr(selected_idx),
        _ptr(workspace), ws_bytes, _stream(stream)))


def loki_decode_attention_scored(cache, batch, q, P, r, k, out, scorer=LOKI_SCORER_LEADING, k_per_seq=None,
                                 recent_window=0, group_reduce=LOKI_GROUP_SUM, scale=0.0, selected_idx=None,
                                 workspace=None, stream=None):
    workspace, ws_bytes = _workspace(workspace, cache, batch, q, k, recent_window)
    _check("loki_decode_attention_scored", _lib.loki_decode_attention_scored(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(q), q.shape[1], _ptr(P), r, k,
        _ptr(k_per_seq), recent_window, group_reduce, scale, scorer, _ptr(out), _ptr(selected_idx),
        _ptr(workspace), ws_bytes, _stream(stream)))


def loki_decode_attention_asym(cache, batch, q, P, A_q, r, k, out, k_per_seq=None, recent_window=0,
                               group_reduce=LOKI_GROUP_SUM, scale=0.0, selected_idx=None, workspace=None,
                               stream=None):
    workspace, ws_bytes = _workspace(workspace, cache, batch, q, k, recent_window)
    _check("loki_decode_attention_asym", _lib.loki_decode_attention_asym(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(q), q.shape[1], _ptr(P), _ptr(A_q), r, k,
        _ptr(k_per_seq), recent_window, group_reduce, scale, _ptr(out), _ptr(selected_idx),
        _ptr(workspace), ws_bytes, _stream(stream)))


def loki_append_keys_asym(cache, batch, k_new, v_new, P, A_k, stream=None):
    _check("loki_append_keys_asym", _lib.loki_append_keys_asym(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k_new), _ptr(v_new), _ptr(P), _ptr(A_k),
        _stream(stream)))


def loki_index_keys(cache, batch, k, A_k, stream=None):
    """Fill the key index with k A_k; k is [batch, Hkv, max_len, head_dim]."""
    _check("loki_index_keys", _lib.loki_index_keys(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k), _ptr(A_k), k.shape[2], _stream(stream)))


def loki_decode_step_host_bytes(cache, batch, num_q_heads):
    return _lib.loki_decode_step_host_bytes(ctypes.byref(cache.struct), ctypes.byref(batch.struct), num_q_heads)


def loki_decode_step_host(cache, batch, k_new_host, v_new_host, q_host, P, r, k, out_host, staging, k_per_seq=None,
                          recent_window=0, group_reduce=LOKI_GROUP_SUM, scale=0.0, stream=None):
    """The decode step with its inputs and output in (pinned) host tensors;
    staging: a device uint8 tensor of loki_decode_step_host_bytes bytes."""
    _check("loki_decode_step_host", _lib.loki_decode_step_host(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k_new_host), _ptr(v_new_host), _ptr(q_host),
        q_host.shape[1], _ptr(P), r, k, _ptr(k_per_seq), recent_window, group_reduce, scale, _ptr(out_host),
        _ptr(staging), staging.numel() * staging.element_size(), _stream(stream)))


def loki_decode_step(cache, batch, k_new, v_new, q, P, r, k, out, k_per_seq=None, recent_window=0,
                     group_reduce=LOKI_GROUP_SUM, scale=0.0, selected_idx=None, workspace=None, stream=None):
    """Append the step's token, then decode (one call, the attention overlapping the append)."""
    workspace, ws_bytes = _workspace(workspace, cache, batch, q, k, recent_window)
    _check("loki_decode_step", _lib.loki_decode_step(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(k_new), _ptr(v_new), _ptr(q), q.shape[1],
        _ptr(P), r, k, _ptr(k_per_seq), recent_window, group_reduce, scale, _ptr(out), _ptr(selected_idx),
        _ptr(workspace), ws_bytes, _stream(stream)))


def loki_decode_max_seq_len(head_dim, dtype_code_):
    return _lib.loki_decode_max_seq_len(head_dim, dtype_code_)


def loki_dense_workspace_bytes(cache, batch, num_q_heads):
    return _lib.loki_dense_workspace_bytes(ctypes.byref(cache.struct), ctypes.byref(batch.struct),
                                           num_q_heads)


def loki_dense_attention(cache, batch, q, P, out, workspace, scale=0.0, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("loki_dense_attention", _lib.loki_dense_attention(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(q), q.shape[1], _ptr(P), scale,
        _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


def loki_dense_attention_static(cache, batch, q, P, out, scale=0.0, stream=None):
    """Dense attention with the library's built-in scratch (no workspace)."""
    _check("loki_dense_attention_static", _lib.loki_dense_attention_static(
        ctypes.byref(cache.struct), ctypes.byref(batch.struct), _ptr(q), q.shape[1], _ptr(P), scale,
        _ptr(out), _stream(stream)))


def loki_device_error(clear=True):
    bits = ctypes.c_uint32(0)
    _check("loki_device_error", _lib.loki_device_error(1 if clear else 0, ctypes.byref(bits)))
    return bits.value


def loki_status_string(status):
    return _lib.loki_status_string(status).decode()


def loki_abi_version():
    return _lib.loki_abi_version()


def raw():
    """The loaded ctypes library (for ABI tests)."""
    return _lib


# --------------------------------------------------------------------------
# Host offload (OffloadCache)
# --------------------------------------------------------------------------

def loki_host_device_pointer(host_tensor):
    """Device address of a pinned host tensor's memory."""
    out = ctypes.c_void_p()
    _check("loki_host_device_pointer", _lib.loki_host_device_pointer(ctypes.c_void_p(host_tensor.data_ptr()),
                                                                     ctypes.byref(out)))
    return out.value


def loki_offload_plan(home, spare, touch, max_moves):
    """home: int32 CPU tensor (updated in place); spare: ctypes.c_int32
    (updated); touch: CPU tensor of per-block counts. Returns the moves."""
    assert home.dtype == torch.int32 and home.is_contiguous()
    touch = touch.to(torch.int32).contiguous()
    moves = (loki_page_move * max(max_moves, 1))()
    n = _lib.loki_offload_plan(home.numel(), ctypes.c_void_p(home.data_ptr()), ctypes.byref(spare),
                               ctypes.c_void_p(touch.data_ptr()), max_moves, moves)
    if n < 0:
        raise LokiError("loki_offload_plan", LOKI_ERR_INVALID_ARG)
    return [moves[i] for i in range(n)]


def loki_offload_apply(cache, moves, home, stream=None):
    arr = (loki_page_move * max(len(moves), 1))(*moves)
    _check("loki_offload_apply", _lib.loki_offload_apply(ctypes.byref(cache.struct), arr, len(moves),
                                                         ctypes.c_void_p(home.data_ptr()), _stream(stream)))


def offload_rebalance(cache, max_moves, stream=None):
    """Between decode steps: read the touch counts, plan up to max_moves
    swaps, issue them on the stream and clear the counts. Returns the moves."""
    stream = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.stream(stream):
        touch = cache.touch.cpu()
        moves = loki_offload_plan(cache.home, cache.spare, touch, max_moves)
        loki_offload_apply(cache, moves, cache.home, stream=stream)
        cache.touch.zero_()
    return moves
