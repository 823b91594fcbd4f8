"""fp64 CPU oracle for SALS latent-space sparse decode (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does, and nothing here is shared with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, pthreads); this module
only compiles it, converts arrays to contiguous float64 and calls it through
ctypes.  Method: "SALS: Sparse Attention in Latent Space for KV cache
Compression" (arXiv 2510.24273v1), technical-framework stages 1-4 and the
English abstract; softmax(QK^T/sqrt(d)) as printed in the VL-Cache
OpenReview response to reviewer KiPr, "On Weakness 1".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
               "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


class _Desc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("rank", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("seq_offsets", ctypes.POINTER(ctypes.c_int64)),
        ("q_pos", ctypes.POINTER(ctypes.c_int32)),
        ("rope_base", ctypes.c_double),
        ("softmax_scale", ctypes.c_double),
        ("n_threads", ctypes.c_int32),
        ("select_mode", ctypes.c_int32),
        ("select_threshold", ctypes.c_double),
    ]


_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)


def _load():
    global _lib
    if _lib is None:
        # A test may point this at a deliberately broken build of oracle.c to
        # show that the pins catch the mistake (tests/test_oracle_mutants.py).
        override = os.environ.get("SALS_ORACLE_LIB")
        lib = ctypes.CDLL(override if override else build())
        lib.oracle_round_bf16.restype = ctypes.c_double
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_round_array.restype = None
        lib.oracle_round_array.argtypes = [_D, _D, ctypes.c_int64, ctypes.c_int32]
        lib.oracle_compress.restype = ctypes.c_int
        lib.oracle_compress.argtypes = [_D, _D, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _D,
                                        ctypes.c_int32]
        lib.oracle_rope.restype = None
        lib.oracle_rope.argtypes = [_D, ctypes.c_int32, ctypes.c_double, ctypes.c_double, _D]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [ctypes.POINTER(_Desc), _D, _D, _D, _D, _D, _I32, _D, _D, _D]
        lib.oracle_attend_given_idx.restype = ctypes.c_int
        lib.oracle_attend_given_idx.argtypes = [ctypes.POINTER(_Desc), _D, _D, _D, _D, _D, _I32,
                                                _D, _D]
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a CPU torch tensor (any float dtype): exact upcast
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(_D)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def round_storage(x, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage type ('bf16' or 'f32'), nearest-even."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().oracle_round_array(_dp(x), _dp(y), x.size, 1 if dtype == "bf16" else 0)
    return y


def compress(X, P, n_threads: int | None = None) -> np.ndarray:
    """Stage 1, low-rank projection Y = X . P in fp64 (X: n x hid, P: hid x r)."""
    X, P = _f64(X), _f64(P)
    n, hid = X.shape
    assert P.shape[0] == hid
    r = P.shape[1]
    Y = np.empty((n, r), dtype=np.float64)
    st = _load().oracle_compress(_dp(X), _dp(P), n, hid, r, _dp(Y), n_threads or default_threads())
    if st:
        raise ValueError(f"oracle_compress failed ({st})")
    return Y


def rope(x, pos: float, base: float) -> np.ndarray:
    """Rotate-half RoPE of one d-vector at position ``pos``."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().oracle_rope(_dp(x), x.shape[-1], float(pos), float(base), _dp(y))
    return y


@dataclass
class Problem:
    """Shapes of one decode layer-step (no data)."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rank: int
    top_k: int
    seq_offsets: np.ndarray  # int64 [B+1]
    rope_base: float = 10000.0
    softmax_scale: float = 0.0
    q_pos: np.ndarray | None = None  # int32 [B] or None
    select_threshold: float | None = None  # None: top-k; else keep the top-k scores >= it


def _desc(p: Problem, n_threads: int | None, keep: list) -> _Desc:
    offs = np.ascontiguousarray(np.asarray(p.seq_offsets, dtype=np.int64))
    keep.append(offs)
    qp = None
    if p.q_pos is not None:
        qp = np.ascontiguousarray(np.asarray(p.q_pos, dtype=np.int32))
        keep.append(qp)
    return _Desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.rank, p.top_k,
                 offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                 qp.ctypes.data_as(_I32) if qp is not None else None,
                 float(p.rope_base), float(p.softmax_scale), int(n_threads or default_threads()),
                 0 if p.select_threshold is None else 1,
                 0.0 if p.select_threshold is None else float(p.select_threshold))


def decode(p: Problem, q, Kc, Vc, Pk, Pv, n_threads: int | None = None) -> dict:
    """Stages 2-4: scores, top-k, reconstruction, RoPE, attention.

    Returns ``idx`` [B][U][k] int32 (selection order, -1 pads), ``scores``
    (packed per (b,u): offset seq_offsets[b]*U + u*n_b), ``probs`` [B][Hq][k]
    in selection order and ``out`` [B][Hq][d], all fp64 except idx.
    """
    keep: list = []
    D = _desc(p, n_threads, keep)
    q, Kc, Vc, Pk, Pv = (_f64(a) for a in (q, Kc, Vc, Pk, Pv))
    B, Hq, U, d, k = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.top_k
    N = int(p.seq_offsets[-1])
    idx = np.empty((B, U, k), dtype=np.int32)
    scores = np.empty(N * U, dtype=np.float64)
    probs = np.empty((B, Hq, k), dtype=np.float64)
    out = np.empty((B, Hq, d), dtype=np.float64)
    st = _load().oracle_decode(ctypes.byref(D), _dp(q), _dp(Kc), _dp(Vc), _dp(Pk), _dp(Pv),
                               idx.ctypes.data_as(_I32), _dp(scores), _dp(probs), _dp(out))
    if st:
        raise ValueError(f"oracle_decode failed ({st})")
    return {"idx": idx, "scores": scores, "probs": probs, "out": out}


def fit_subspace(X, rank: int) -> np.ndarray:
    """Learned projection (SALS page, key designs: a low-rank projection from the SVD of the
    keys): the top-``rank`` right singular vectors of X [n][hidden] as columns, [hidden][rank],
    fp64.  Any orthonormal basis of the same subspace is an equivalent projection (the decode
    path uses P only through P P^T), so results are compared as projectors."""
    x = _f64(X)
    _, _, vt = np.linalg.svd(x, full_matrices=False)
    return np.ascontiguousarray(vt[:rank].T)


def unit_scores(p: Problem, scores: np.ndarray, b: int, u: int) -> np.ndarray:
    """View of the packed score vector of unit (b, u)."""
    off = int(p.seq_offsets[b])
    nb = int(p.seq_offsets[b + 1]) - off
    base = off * p.n_kv_heads + u * nb
    return scores[base:base + nb]


def attend_given_idx(p: Problem, q, Kc, Vc, Pk, Pv, idx, n_threads: int | None = None) -> dict:
    """Stages 3-4 only, over a supplied index set [B][U][k] (-1 = unused)."""
    keep: list = []
    D = _desc(p, n_threads, keep)
    q, Kc, Vc, Pk, Pv = (_f64(a) for a in (q, Kc, Vc, Pk, Pv))
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    B, Hq, d, k = p.batch, p.n_q_heads, p.head_dim, p.top_k
    probs = np.empty((B, Hq, k), dtype=np.float64)
    out = np.empty((B, Hq, d), dtype=np.float64)
    st = _load().oracle_attend_given_idx(ctypes.byref(D), _dp(q), _dp(Kc), _dp(Vc), _dp(Pk),
                                         _dp(Pv), idx.ctypes.data_as(_I32), _dp(probs), _dp(out))
    if st:
        raise ValueError(f"oracle_attend_given_idx failed ({st})")
    return {"probs": probs, "out": out}
