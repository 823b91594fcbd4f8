"""ctypes binding of libsalsc (include/salsc.h): argument marshalling only.

Every function here passes raw device pointers, sizes and the current CUDA
stream to the C ABI; all arithmetic happens in the library's kernels.  The
library must have been built (``python -m latent_space_sparse_b200.build``);
importing this module without it raises, and nothing falls back to the CPU.
Tensors are torch CUDA tensors (torch supplies device memory and streams).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "csrc", "libsalsc.so")

SALSC_OK, SALSC_ERR_INVALID_ARG, SALSC_ERR_UNSUPPORTED, SALSC_ERR_WORKSPACE, SALSC_ERR_CUDA = range(5)
SALSC_F32, SALSC_BF16 = 0, 1
FLAG_BAD_INDEX, FLAG_WAIT_TIMEOUT = 1, 2
WS_ALIGN = 256

EXPORTS = (
    "salsc_compress", "salsc_decode_workspace_size", "salsc_decode_prepare", "salsc_decode_step",
    "salsc_decode_step_timed", "salsc_decode_step_traced", "salsc_decode_step_static_ws",
    "salsc_static_workspace_bytes",
    "salsc_decode_launch_count", "salsc_append", "salsc_decode_step_append",
    "salsc_fit_workspace_size",
    "salsc_fit_projection", "salsc_shard_candidates", "salsc_shard_select", "salsc_shard_attend",
    "salsc_shard_merge", "salsc_check_wait_timeout", "salsc_decode_read_flags",
    "salsc_status_string", "salsc_last_cuda_error",
    "salsc_version",
)


class SalscError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = f"{what}: {status_string(status)}"
        if status == SALSC_ERR_CUDA:
            msg += f" ({_lib().salsc_last_cuda_error().decode()})"
        super().__init__(msg)
        self.status = status


class DecodeDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("rank", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("seq_offsets_host", ctypes.POINTER(ctypes.c_int64)),
        ("seq_offsets_dev", ctypes.c_void_p),
        ("q_pos_dev", ctypes.c_void_p),
        ("rope_base", ctypes.c_double),
        ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int),
        ("select_mode", ctypes.c_int32),
        ("select_threshold", ctypes.c_float),
    ]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m latent_space_sparse_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        dp = ctypes.POINTER(DecodeDesc)
        lib.salsc_compress.restype = ctypes.c_int
        lib.salsc_compress.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, ctypes.c_int, vp]
        lib.salsc_decode_workspace_size.restype = sz
        lib.salsc_decode_workspace_size.argtypes = [dp]
        lib.salsc_decode_prepare.restype = ctypes.c_int
        lib.salsc_decode_prepare.argtypes = [dp, vp, sz, vp]
        lib.salsc_decode_step.restype = ctypes.c_int
        lib.salsc_decode_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.salsc_decode_step_append.restype = ctypes.c_int
        lib.salsc_decode_step_append.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                                 vp]
        lib.salsc_fit_workspace_size.restype = sz
        lib.salsc_fit_workspace_size.argtypes = [i32, i32]
        lib.salsc_fit_projection.restype = ctypes.c_int
        lib.salsc_fit_projection.argtypes = [vp, i64, i32, i32, vp, i32, vp, ctypes.c_int, vp, sz, vp]
        lib.salsc_shard_candidates.restype = ctypes.c_int
        lib.salsc_shard_candidates.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.salsc_shard_select.restype = ctypes.c_int
        lib.salsc_shard_select.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]
        lib.salsc_shard_attend.restype = ctypes.c_int
        lib.salsc_shard_attend.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.salsc_shard_merge.restype = ctypes.c_int
        lib.salsc_shard_merge.argtypes = [vp, i32, i32, i32, i32, i32, i32, ctypes.c_int, vp, vp,
                                          vp, sz, vp]
        lib.salsc_append.restype = ctypes.c_int
        lib.salsc_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, ctypes.c_int, vp]
        lib.salsc_decode_launch_count.restype = ctypes.c_int32
        lib.salsc_decode_launch_count.argtypes = [dp]
        lib.salsc_decode_step_traced.restype = ctypes.c_int
        lib.salsc_decode_step_traced.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, sz, vp]
        lib.salsc_decode_step_timed.restype = ctypes.c_int
        lib.salsc_decode_step_timed.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                                ctypes.POINTER(ctypes.c_void_p), i32]
        lib.salsc_decode_step_static_ws.restype = ctypes.c_int
        lib.salsc_decode_step_static_ws.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.salsc_static_workspace_bytes.restype = sz
        lib.salsc_static_workspace_bytes.argtypes = []
        lib.salsc_check_wait_timeout.restype = ctypes.c_int
        lib.salsc_check_wait_timeout.argtypes = [ctypes.c_uint64, vp, sz, vp]
        lib.salsc_decode_read_flags.restype = ctypes.c_int
        lib.salsc_decode_read_flags.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_uint32), vp]
        lib.salsc_status_string.restype = ctypes.c_char_p
        lib.salsc_status_string.argtypes = [ctypes.c_int]
        lib.salsc_last_cuda_error.restype = ctypes.c_char_p
        lib.salsc_last_cuda_error.argtypes = []
        lib.salsc_version.restype = ctypes.c_char_p
        lib.salsc_version.argtypes = []
        _LIB = lib
    return _LIB


def load():
    """Load the library (raises ImportError if it was not built)."""
    return _lib()


def status_string(status: int) -> str:
    return _lib().salsc_status_string(status).decode()


def version() -> str:
    return _lib().salsc_version().decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return SALSC_BF16
    if t == torch.float32:
        return SALSC_F32
    raise TypeError(f"unsupported storage dtype {t}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(st: int, what: str):
    if st != SALSC_OK:
        raise SalscError(st, what)


def salsc_compress(K, V, Pk, Pv, Kc, Vc, stream=None):
    """Kc = K . Pk and Vc = V . Pv on the current stream; K or V may be None."""
    x = K if K is not None else V
    n, hid = x.shape
    r = (Pk if K is not None else Pv).shape[1]
    st = _lib().salsc_compress(_ptr(K), _ptr(V), _ptr(Pk), _ptr(Pv), _ptr(Kc), _ptr(Vc), n, hid, r,
                               _dtype_code(x.dtype), _stream(stream))
    _check(st, "salsc_compress")


def salsc_append(K_new, V_new, Pk, Pv, Kc, Vc, rows, stream=None):
    """Kc[rows[b]] = K_new[b] . Pk and Vc[rows[b]] = V_new[b] . Pv (rows: int64
    device tensor); K_new or V_new may be None."""
    x = K_new if K_new is not None else V_new
    batch, hid = x.shape
    r = (Pk if K_new is not None else Pv).shape[1]
    if rows.dtype != torch.int64 or not rows.is_cuda:
        raise ValueError("rows must be an int64 device tensor")
    st = _lib().salsc_append(_ptr(K_new), _ptr(V_new), _ptr(Pk), _ptr(Pv), _ptr(Kc), _ptr(Vc),
                             _ptr(rows), batch, hid, r, _dtype_code(x.dtype), _stream(stream))
    _check(st, "salsc_append")


FLAG_FIT_NOT_SPD = 4


def salsc_fit_projection(X, rank, omega, iters, out=None, stream=None):
    """Orthonormal basis [hidden][rank] of the dominant right-singular subspace of X [n][hidden]
    (subspace iteration from omega, fp32 [hidden][rank]); returns (P, flags)."""
    n, hidden = X.shape
    if omega.dtype != torch.float32 or tuple(omega.shape) != (hidden, rank):
        raise ValueError("omega must be float32 [hidden][rank]")
    nbytes = int(_lib().salsc_fit_workspace_size(hidden, rank))
    if nbytes == 0:
        raise ValueError("salsc_fit_workspace_size: unsupported shape")
    ws = alloc_workspace(nbytes, X.device)
    P = torch.empty((hidden, rank), dtype=X.dtype, device=X.device) if out is None else out
    st = _lib().salsc_fit_projection(_ptr(X), n, hidden, rank, _ptr(omega), iters, _ptr(P),
                                     _dtype_code(X.dtype), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream))
    _check(st, "salsc_fit_projection")
    return P, salsc_decode_read_flags(ws, stream)


def make_desc(batch, n_q_heads, n_kv_heads, head_dim, rank, top_k, seq_offsets_host,
              seq_offsets_dev=None, q_pos_dev=None, rope_base=10000.0, softmax_scale=0.0,
              dtype=torch.bfloat16, select_threshold=None):
    """Build a DecodeDesc; ``seq_offsets_host`` must be a contiguous CPU int64 tensor kept alive
    by the caller (the descriptor points into it).  ``select_threshold``: None for top-k, else
    threshold selection (of the top-k tokens, those with a unit score below it are dropped)."""
    assert seq_offsets_host.dtype == torch.int64 and not seq_offsets_host.is_cuda
    assert seq_offsets_host.is_contiguous()
    return DecodeDesc(
        batch, n_q_heads, n_kv_heads, head_dim, rank, top_k,
        ctypes.cast(seq_offsets_host.data_ptr(), ctypes.POINTER(ctypes.c_int64)),
        None if seq_offsets_dev is None else seq_offsets_dev.data_ptr(),
        None if q_pos_dev is None else q_pos_dev.data_ptr(),
        float(rope_base), float(softmax_scale), _dtype_code(dtype),
        0 if select_threshold is None else 1,
        0.0 if select_threshold is None else float(select_threshold))


def salsc_decode_workspace_size(desc: DecodeDesc) -> int:
    return int(_lib().salsc_decode_workspace_size(ctypes.byref(desc)))


def salsc_decode_prepare(desc: DecodeDesc, ws, stream=None):
    st = _lib().salsc_decode_prepare(ctypes.byref(desc), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream))
    _check(st, "salsc_decode_prepare")


def salsc_decode_step(desc: DecodeDesc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, stream=None):
    st = _lib().salsc_decode_step(ctypes.byref(desc), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Pk),
                                  _ptr(Pv), _ptr(out), _ptr(idx_out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "salsc_decode_step")


def salsc_decode_step_append(desc: DecodeDesc, K_new, V_new, rows, q, Kc, Vc, Pk, Pv, out, idx_out,
                             ws, stream=None):
    """salsc_append then salsc_decode_step in one call (rows: int64 device tensor)."""
    if rows is None or rows.dtype != torch.int64 or not rows.is_cuda:
        raise ValueError("rows must be an int64 device tensor")
    st = _lib().salsc_decode_step_append(ctypes.byref(desc), _ptr(K_new), _ptr(V_new), _ptr(rows),
                                         _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Pk), _ptr(Pv), _ptr(out),
                                         _ptr(idx_out), _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream))
    _check(st, "salsc_decode_step_append")


def salsc_shard_candidates(desc: DecodeDesc, q, Kc, Pk, shard_off, cand_score, cand_idx, ws,
                           stream=None):
    """Token-sharded step 1: this shard's top-k per unit as (score, global index) candidates."""
    st = _lib().salsc_shard_candidates(ctypes.byref(desc), _ptr(q), _ptr(Kc), _ptr(Pk),
                                       _ptr(shard_off), _ptr(cand_score), _ptr(cand_idx), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "salsc_shard_candidates")


def salsc_shard_select(cand_score_all, cand_idx_all, local_offsets, shard_off, idx_local,
                       stream=None):
    """Token-sharded step 3: the global top-k of the gathered candidates [N][B][U][k]; this
    shard's tokens as slice-local indices in idx_local [B][U][k] (-1 elsewhere)."""
    n, b, u, k = cand_score_all.shape
    st = _lib().salsc_shard_select(_ptr(cand_score_all), _ptr(cand_idx_all), n, b, u, k,
                                   _ptr(local_offsets), _ptr(shard_off), _ptr(idx_local),
                                   _stream(stream))
    _check(st, "salsc_shard_select")


def salsc_shard_attend(desc: DecodeDesc, q, Kc, Vc, Pk, idx_local, shard_off, part_out, ws,
                       stream=None):
    """Token-sharded step 4: attention over idx_local; part_out [B][Hq][r+4] fp32 rows
    (m, l, 0, 0, acc[r]) per head, before the projection."""
    st = _lib().salsc_shard_attend(ctypes.byref(desc), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Pk),
                                   _ptr(idx_local), _ptr(shard_off), _ptr(part_out), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "salsc_shard_attend")


def salsc_shard_merge(part_all, n_kv_heads, head_dim, Pv, out, ws, stream=None):
    """Token-sharded step 6: merge the gathered rows part_all [N][B][Hq][r+4] and project."""
    n, b, hq, rowf = part_all.shape
    st = _lib().salsc_shard_merge(_ptr(part_all), n, b, hq, n_kv_heads, head_dim, rowf - 4,
                                  _dtype_code(out.dtype), _ptr(Pv), _ptr(out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "salsc_shard_merge")


DECODE_KERNELS = ("latent_q", "score", "topk", "attend", "combine")


def salsc_decode_launch_count(desc: DecodeDesc) -> int:
    """Kernels one salsc_decode_step launches for this descriptor (4 or 5)."""
    n = _lib().salsc_decode_launch_count(ctypes.byref(desc))
    if n < 0:
        raise ValueError("salsc_decode_launch_count: invalid or unsupported descriptor")
    return n


def salsc_decode_step_timed(desc: DecodeDesc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, events,
                            stream=None):
    """salsc_decode_step plus an event record before each kernel and after the last
    (``events``: len(DECODE_KERNELS)+1 torch.cuda.Event(enable_timing=True))."""
    for e in events:  # torch creates the CUDA event lazily
        if e.cuda_event == 0:
            e.record(stream if stream is not None else torch.cuda.current_stream())
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    st = _lib().salsc_decode_step_timed(ctypes.byref(desc), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Pk),
                                        _ptr(Pv), _ptr(out), _ptr(idx_out), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream), arr,
                                        len(events))
    _check(st, "salsc_decode_step_timed")


TRACE_MAX_CTAS = 8192  # SALSC_TRACE_MAX_CTAS


def trace_buffer(device) -> torch.Tensor:
    """A zeroed int64 timeline buffer for salsc_decode_step_traced: [stage][cta][3]."""
    return torch.zeros((len(DECODE_KERNELS), TRACE_MAX_CTAS, 3), dtype=torch.int64,
                       device=device)


def salsc_decode_step_traced(desc: DecodeDesc, q, Kc, Vc, Pk, Pv, out, idx_out, ws, trace,
                             stream=None):
    """salsc_decode_step that records per-CTA timestamps (start, dependency wait done,
    end; global ns timer) of every stage into ``trace`` (see trace_buffer)."""
    st = _lib().salsc_decode_step_traced(ctypes.byref(desc), _ptr(q), _ptr(Kc), _ptr(Vc),
                                         _ptr(Pk), _ptr(Pv), _ptr(out), _ptr(idx_out), _ptr(ws),
                                         ws.numel() * ws.element_size(), _ptr(trace),
                                         trace.numel() * trace.element_size(), _stream(stream))
    _check(st, "salsc_decode_step_traced")


def static_workspace_bytes() -> int:
    """Size of the library's fixed scratch array (salsc_decode_step_static_ws's limit)."""
    return int(_lib().salsc_static_workspace_bytes())


def salsc_decode_step_static_ws(desc: DecodeDesc, q, Kc, Vc, Pk, Pv, out, idx_out, stream=None):
    """salsc_decode_step with the library's fixed internal scratch: no workspace argument,
    nothing allocated (for callers that cannot allocate device memory)."""
    st = _lib().salsc_decode_step_static_ws(ctypes.byref(desc), _ptr(q), _ptr(Kc), _ptr(Vc),
                                            _ptr(Pk), _ptr(Pv), _ptr(out), _ptr(idx_out),
                                            _stream(stream))
    _check(st, "salsc_decode_step_static_ws")


def salsc_check_wait_timeout(limit_ns: int, ws, stream=None):
    """Run the decode pipelines' bounded wait on a barrier nothing completes (limit in ns);
    the wait gives up and sets the timeout bit of ``ws``'s anomaly word."""
    st = _lib().salsc_check_wait_timeout(int(limit_ns), _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream))
    _check(st, "salsc_check_wait_timeout")


def salsc_decode_read_flags(ws, stream=None) -> int:
    v = ctypes.c_uint32(0)
    st = _lib().salsc_decode_read_flags(_ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(v),
                                        _stream(stream))
    _check(st, "salsc_decode_read_flags")
    return int(v.value)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A uint8 device buffer of ``nbytes`` starting on a 256-byte boundary."""
    buf = torch.empty(nbytes + WS_ALIGN, dtype=torch.uint8, device=device)
    shift = (-buf.data_ptr()) % WS_ALIGN
    return buf[shift:shift + nbytes]


class Decoder:
    """Descriptor + workspace for one decode shape (marshalling only).

    ``seq_lens`` fixes the ragged layout of the latent cache; q/Kc/Vc/Pk/Pv/out
    are passed per call.  q_pos (CUDA int32 [B]) defaults to n_b.
    """

    def __init__(self, batch, n_q_heads, n_kv_heads, head_dim, rank, top_k, seq_lens,
                 rope_base=10000.0, softmax_scale=0.0, dtype=torch.bfloat16, device="cuda",
                 q_pos=None, select_threshold=None):
        lens = [int(x) for x in seq_lens]
        offs = [0]
        for n in lens:
            offs.append(offs[-1] + n)
        self.seq_offsets_host = torch.tensor(offs, dtype=torch.int64)
        self.seq_offsets_dev = self.seq_offsets_host.to(device)
        self.q_pos = None if q_pos is None else q_pos.to(device=device, dtype=torch.int32).contiguous()
        self.shape = dict(batch=batch, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads,
                          head_dim=head_dim, rank=rank, top_k=top_k)
        self.dtype = dtype
        self.desc = make_desc(batch, n_q_heads, n_kv_heads, head_dim, rank, top_k,
                              self.seq_offsets_host, self.seq_offsets_dev, self.q_pos, rope_base,
                              softmax_scale, dtype, select_threshold)
        nbytes = salsc_decode_workspace_size(self.desc)
        if nbytes == 0:
            raise SalscError(SALSC_ERR_INVALID_ARG, "salsc_decode_workspace_size")
        self.ws = alloc_workspace(nbytes, device)
        salsc_decode_prepare(self.desc, self.ws)

    def step(self, q, Kc, Vc, Pk, Pv, out=None, idx_out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        salsc_decode_step(self.desc, q, Kc, Vc, Pk, Pv, out, idx_out, self.ws, stream)
        return out

    def flags(self, stream=None) -> int:
        return salsc_decode_read_flags(self.ws, stream)
