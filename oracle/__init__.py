"""Reference oracle for Loki-style low-rank-key sparse decode attention.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
CPU-baseline leg import this package. It is a thin numpy/ctypes wrapper around
oracle.c (plain binary64 C); every step of the arithmetic lives there, with
its citation to the pages. It shares no code with the CUDA library.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None
_lib_path = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U16 = ctypes.POINTER(ctypes.c_uint16)


def use_library(path=None):
    """Point the wrapper at another build of oracle.c (None: the default).

    The mutation tests use this to check that the pins reject planted
    mistakes in a modified copy of the oracle."""
    global _lib, _lib_path
    _lib, _lib_path = None, path


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_lib_path or _build.build())
        lib.oracle_round_bf16.restype = ctypes.c_double
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_round_bf16_array.restype = None
        lib.oracle_round_bf16_array.argtypes = [_D, ctypes.c_int64, _D, _U16]
        lib.oracle_rotate.restype = None
        lib.oracle_rotate.argtypes = [_D, _D, ctypes.c_int64, ctypes.c_int, _D]
        lib.oracle_covariance.restype = None
        lib.oracle_covariance.argtypes = [_D, ctypes.c_int64, ctypes.c_int, _D]
        lib.oracle_append.restype = None
        lib.oracle_append.argtypes = [_D, _D, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _D]
        lib.oracle_attend_set.restype = None
        lib.oracle_attend_set.argtypes = [_D, _D, _D, _I32, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_double, _D, _D]
        lib.oracle_decode_pair.restype = ctypes.c_int
        lib.oracle_decode_pair.argtypes = [_D, _D, _D, _D, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           _D, _I32, ctypes.POINTER(ctypes.c_int), _D, _D]
        lib.oracle_dense_pair.restype = None
        lib.oracle_dense_pair.argtypes = [_D, _D, _D, _D, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_double, _D]
        lib.oracle_decode_batch.restype = ctypes.c_int
        lib.oracle_decode_batch.argtypes = [ctypes.c_int, _D, _D, _D, _D, _I32, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, _I32,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, _D, _I32]
        lib.oracle_index_keys.restype = None
        lib.oracle_index_keys.argtypes = [_D, _D, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _D]
        lib.oracle_decode_pair_asym.restype = ctypes.c_int
        lib.oracle_decode_pair_asym.argtypes = [_D, _D, _D, _D, _D, _D, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, _I32,
                                                ctypes.POINTER(ctypes.c_int), _D, _D]
        lib.oracle_magnitude_slabs.restype = ctypes.c_int
        lib.oracle_magnitude_slabs.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, _I32, _D]
        lib.oracle_magnitude_dims.restype = ctypes.c_int
        lib.oracle_magnitude_dims.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, _I32, _D]
        lib.oracle_decode_pair_dims.restype = ctypes.c_int
        lib.oracle_decode_pair_dims.argtypes = [_D, _D, _D, _D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_double, _D, _I32,
                                                ctypes.POINTER(ctypes.c_int), _D, _D, _I32]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, t=_D):
    return a.ctypes.data_as(t) if a is not None else None


def round_bf16(x):
    """Round binary64 values to bfloat16 (nearest, ties to even), one step.

    Returns (values as float64, bit patterns as uint16)."""
    x = _f64(x)
    out = np.empty_like(x)
    bits = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_round_bf16_array(_p(x), x.size, _p(out), _p(bits, _U16))
    return out, bits


def rotate(x, P):
    """x_hat = x P for row vectors x [n, d]."""
    x = _f64(x)
    P = _f64(P)
    n, d = x.shape
    out = np.empty((n, d))
    _load().oracle_rotate(_p(x), _p(P), n, d, _p(out))
    return out


def covariance(x):
    """Centred covariance (1/n) of the rows of x [n, d] (oracle.c)."""
    x = _f64(x)
    n, d = x.shape
    C = np.empty((d, d))
    _load().oracle_covariance(_p(x), n, d, _p(C))
    return C


def pca_basis(keys):
    """P from calibration keys [n, d]: the eigenvectors of their centred
    covariance as columns, in descending eigenvalue order, each column's sign
    fixed so that its entry of largest magnitude is positive. Returns
    (P [d, d], eigenvalues [d]). numpy's symmetric eigensolver is the step
    that diagonalises the covariance."""
    lam, vec = np.linalg.eigh(covariance(keys))
    order = np.argsort(-lam, kind="stable")
    lam, vec = lam[order], vec[:, order]
    idx = np.argmax(np.abs(vec), axis=0)
    vec = vec * np.sign(vec[idx, np.arange(vec.shape[1])])[None, :]
    return vec, lam


def append(k_new, P, dtype):
    """Keys rotated into the PCA basis and rounded to the cache type.

    dtype: 'bf16' or 'f32'."""
    k_new = _f64(k_new)
    P = _f64(P)
    n, d = k_new.shape
    out = np.empty((n, d))
    _load().oracle_append(_p(k_new), _p(P), n, d, 1 if dtype == "bf16" else 0, _p(out))
    return out


def attend_set(Kt, V, qhat, T, scale=0.0, return_weights=False):
    """Exact softmax attention of the rows of qhat [g, d] over token set T."""
    Kt, V, qhat = _f64(Kt), _f64(V), _f64(qhat)
    T = np.ascontiguousarray(T, dtype=np.int32)
    g, d = qhat.shape
    out = np.empty((g, d))
    w = np.empty((g, len(T))) if return_weights else None
    _load().oracle_attend_set(_p(Kt), _p(V), _p(qhat), _p(T, _I32), len(T), d, g,
                              scale, _p(out), _p(w))
    return (out, w) if return_weights else out


class PairResult:
    __slots__ = ("out", "sel", "n_sel", "scores", "kth", "slabs", "energy", "dims", "weight")


def decode_pair(Kt, V, q, P, r, k, W=0, group_max=False, scale=0.0):
    """One (sequence, kv head) decode step; see oracle_decode_pair in oracle.c."""
    Kt, V, q, P = _f64(Kt), _f64(V), _f64(q), _f64(P)
    L, d = Kt.shape
    g = q.shape[0]
    res = PairResult()
    res.out = np.empty((g, d))
    res.sel = np.empty(k + W, dtype=np.int32)
    n_sel = ctypes.c_int(0)
    res.scores = np.empty(L)
    kth = ctypes.c_double(0.0)
    rc = _load().oracle_decode_pair(_p(Kt), _p(V), _p(q), _p(P), L, d, g, r, k, W,
                                    1 if group_max else 0, scale, _p(res.out),
                                    _p(res.sel, _I32), ctypes.byref(n_sel), _p(res.scores),
                                    ctypes.byref(kth))
    if rc != 0:
        raise ValueError("oracle_decode_pair rejected its arguments")
    res.n_sel = n_sel.value
    res.kth = kth.value
    return res


def magnitude_slabs(q, P, r, index_dims, group_max=False):
    """The r/16 slabs of 16 index dims with the most query energy, ascending,
    and every slab's energy; see oracle_magnitude_slabs in oracle.c."""
    q, P = _f64(q), _f64(P)
    g, d = q.shape
    slabs = np.empty(r // 16, dtype=np.int32)
    energy = np.empty(index_dims // 16)
    rc = _load().oracle_magnitude_slabs(_p(q), _p(P), d, g, index_dims, r, 1 if group_max else 0,
                                        _p(slabs, _I32), _p(energy))
    if rc != 0:
        raise ValueError("oracle_magnitude_slabs rejected its arguments")
    return slabs, energy


def decode_pair_magnitude(Kt, V, q, P, r, k, index_dims, W=0, group_max=False, scale=0.0):
    """decode_pair with the scoring dims chosen by query magnitude.

    The chosen slabs' dims are moved to the front of the basis (the columns
    of P and of the stored keys, the same permutation for both) and
    decode_pair scores with the leading r of them: its approximate scores
    then sum over the chosen dims in ascending order, and its exact logits,
    over all dims, are unchanged by the permutation. The result also carries
    `slabs` and `energy`."""
    Kt, P = _f64(Kt), _f64(P)
    d = P.shape[0]
    slabs, energy = magnitude_slabs(q, P, r, index_dims, group_max)
    front = np.concatenate([np.arange(16 * s, 16 * s + 16) for s in slabs])
    perm = np.concatenate([front, np.setdiff1d(np.arange(d), front)])
    res = decode_pair(Kt[:, perm], V, q, P[:, perm], r, k, W=W, group_max=group_max, scale=scale)
    res.slabs, res.energy = slabs, energy
    return res


def magnitude_dims(q, P, r, index_dims, group_max=False):
    """The r index dims of largest projected-query magnitude, ascending, and
    every dim's magnitude; see oracle_magnitude_dims in oracle.c (AQUA page,
    Algorithm 1 in prose and appendix on complexity, step 2)."""
    q, P = _f64(q), _f64(P)
    g, d = q.shape
    dims = np.empty(r, dtype=np.int32)
    weight = np.empty(index_dims)
    rc = _load().oracle_magnitude_dims(_p(q), _p(P), d, g, index_dims, r, 1 if group_max else 0,
                                       _p(dims, _I32), _p(weight))
    if rc != 0:
        raise ValueError("oracle_magnitude_dims rejected its arguments")
    return dims, weight


def decode_pair_dims(Kt, V, q, P, r, k, index_dims, W=0, group_max=False, scale=0.0):
    """One pair's decode step scored with the r dims of largest query
    magnitude; see oracle_decode_pair_dims in oracle.c. The result also
    carries `dims` and `weight`."""
    Kt, V, q, P = _f64(Kt), _f64(V), _f64(q), _f64(P)
    L, d = Kt.shape
    g = q.shape[0]
    res = PairResult()
    res.out = np.empty((g, d))
    res.sel = np.empty(k + W, dtype=np.int32)
    res.dims = np.empty(r, dtype=np.int32)
    n_sel = ctypes.c_int(0)
    res.scores = np.empty(L)
    kth = ctypes.c_double(0.0)
    rc = _load().oracle_decode_pair_dims(_p(Kt), _p(V), _p(q), _p(P), L, d, g, index_dims, r, k, W,
                                         1 if group_max else 0, scale, _p(res.out), _p(res.sel, _I32),
                                         ctypes.byref(n_sel), _p(res.scores), ctypes.byref(kth),
                                         _p(res.dims, _I32))
    if rc != 0:
        raise ValueError("oracle_decode_pair_dims rejected its arguments")
    res.n_sel = n_sel.value
    res.kth = kth.value
    res.weight = magnitude_dims(q, P, r, index_dims, group_max)[1]
    return res


def index_keys(k, Ak, dtype):
    """Key-index rows round(k A_k) of keys k [n, d] in the original basis,
    A_k [d, ri]; see oracle_index_keys in oracle.c. dtype: 'bf16' or 'f32'."""
    k, Ak = _f64(k), _f64(Ak)
    n, d = k.shape
    ri = Ak.shape[1]
    out = np.empty((n, ri))
    _load().oracle_index_keys(_p(k), _p(Ak), n, d, ri, 1 if dtype == "bf16" else 0, _p(out))
    return out


def decode_pair_asym(Kt, V, Kidx, q, P, Aq, r, k, W=0, group_max=False, scale=0.0):
    """One pair's decode with scores from the key index Kidx [L, ri] and the
    query factor q A_q; see oracle_decode_pair_asym in oracle.c."""
    Kt, V, Kidx, q, P, Aq = _f64(Kt), _f64(V), _f64(Kidx), _f64(q), _f64(P), _f64(Aq)
    L, d = Kt.shape
    ri = Aq.shape[1]
    g = q.shape[0]
    res = PairResult()
    res.out = np.empty((g, d))
    res.sel = np.empty(k + W, dtype=np.int32)
    n_sel = ctypes.c_int(0)
    res.scores = np.empty(L)
    kth = ctypes.c_double(0.0)
    rc = _load().oracle_decode_pair_asym(_p(Kt), _p(V), _p(Kidx), _p(q), _p(P), _p(Aq), L, d, ri, g, r, k, W,
                                         1 if group_max else 0, scale, _p(res.out), _p(res.sel, _I32),
                                         ctypes.byref(n_sel), _p(res.scores), ctypes.byref(kth))
    if rc != 0:
        raise ValueError("oracle_decode_pair_asym rejected its arguments")
    res.n_sel = n_sel.value
    res.kth = kth.value
    return res


def _sym_power(S, power):
    lam, vec = np.linalg.eigh(S)
    if lam.min() <= 0:
        raise ValueError("second-moment matrix is not positive definite")
    return (vec * lam ** power) @ vec.T


def saki_factors(Q, K, r):
    """Rank-r asymmetric score factors from calibration queries Q [n_q, d] and
    keys K [n_k, d] (SAKI page, abstract: the expected score distortion of a
    rank-r approximation q W k^T of q k^T is a covariance-weighted low-rank
    objective, solved in closed form by the SVD of the covariance-weighted
    query-key operator).

    Reading: with the second moments S_q = Q^T Q / n_q and S_k = K^T K / n_k
    (uncentred: the score is a raw inner product), the distortion of W is
    E[(q (I - W) k^T)^2] = ||S_q^1/2 (I - W) S_k^1/2||_F^2, minimised over
    rank r by S_q^1/2 W S_k^1/2 = the rank-r SVD truncation U_r s_r V_r^T of
    C = S_q^1/2 S_k^1/2 (Eckart-Young). Factored as W = A_q A_k^T with
    A_q = S_q^-1/2 U_r diag(s_r)^1/2 and A_k = S_k^-1/2 V_r diag(s_r)^1/2;
    the first r' < r columns of the factors are the rank-r' solution.
    The abstract's random-matrix noise correction is not part of this
    reading (the abstract stops before saying how it is done).

    numpy's symmetric eigensolver (matrix square roots) and SVD are the
    library steps. Returns (A_q [d, r], A_k [d, r], all singular values of C)."""
    Q, K = _f64(Q), _f64(K)
    Sq = Q.T @ Q / Q.shape[0]
    Sk = K.T @ K / K.shape[0]
    C = _sym_power(Sq, 0.5) @ _sym_power(Sk, 0.5)
    U, s, Vt = np.linalg.svd(C)
    root = np.sqrt(s[:r])
    Aq = _sym_power(Sq, -0.5) @ (U[:, :r] * root)
    Ak = _sym_power(Sk, -0.5) @ (Vt[:r].T * root)
    return Aq, Ak, s


def dense_pair(K, V, q, P=None, scale=0.0):
    """Dense decode attention; P=None uses K as given (unrotated comparison)."""
    K, V, q = _f64(K), _f64(V), _f64(q)
    Pp = _f64(P) if P is not None else None
    L, d = K.shape
    g = q.shape[0]
    out = np.empty((g, d))
    _load().oracle_dense_pair(_p(K), _p(V), _p(q), _p(Pp), L, d, g, scale, _p(out))
    return out


def decode_batch(Kt, V, q, P, L, r, k_per_pair, W=0, group_max=False, scale=0.0):
    """Many pairs, one per OpenMP thread.

    Kt, V: [n, Lmax, d]; q: [n, g, d]; P: [n, d, d]; L, k_per_pair: [n]."""
    Kt, V, q, P = _f64(Kt), _f64(V), _f64(q), _f64(P)
    n, Lmax, d = Kt.shape
    g = q.shape[1]
    L = np.ascontiguousarray(L, dtype=np.int32)
    kp = np.ascontiguousarray(k_per_pair, dtype=np.int32)
    kmax = int(kp.max()) if n else 0
    out = np.empty((n, g, d))
    sel = np.empty((n, kmax + W), dtype=np.int32)
    rc = _load().oracle_decode_batch(n, _p(Kt), _p(V), _p(q), _p(P), _p(L, _I32), Lmax, d, g,
                                     r, _p(kp, _I32), kmax, W, 1 if group_max else 0, scale,
                                     _p(out), _p(sel, _I32))
    if rc != 0:
        raise ValueError("oracle_decode_batch rejected its arguments")
    return out, sel


def num_threads():
    return _load().oracle_num_threads()
