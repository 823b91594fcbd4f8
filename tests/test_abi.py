"""The C-ABI library loads, exports every declared symbol and validates
arguments on the host.  No test here launches a kernel: every call below
returns its error before any CUDA work is enqueued."""
import ctypes
import os
import re

import pytest
import torch

from latent_space_sparse_b200 import salsc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "salsc.h")).read()
    return sorted(set(re.findall(r"\b(salsc_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_the_binding_exports():
    assert declared_symbols() == sorted(salsc.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = salsc.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert salsc.version().startswith("salsc")


def test_header_constants_match_the_binding():
    text = open(os.path.join(ROOT, "include", "salsc.h")).read()
    assert int(re.search(r"#define SALSC_DECODE_KERNELS (\d+)", text).group(1)) == \
        len(salsc.DECODE_KERNELS)
    assert int(re.search(r"#define SALSC_TRACE_MAX_CTAS (\d+)", text).group(1)) == \
        salsc.TRACE_MAX_CTAS


def test_traced_step_checks_its_buffer_before_launch():
    lib = salsc.load()
    vp = ctypes.c_void_p
    d = desc([0, 1000])
    need = 3 * 8 * len(salsc.DECODE_KERNELS) * salsc.TRACE_MAX_CTAS
    a = vp(1 << 20)

    def traced(tr=vp(1 << 24), nb=need):
        return lib.salsc_decode_step_traced(ctypes.byref(d), a, a, a, a, a, a, None, vp(1 << 28),
                                            1 << 30, tr, nb, None)

    assert traced(tr=None) == salsc.SALSC_ERR_INVALID_ARG
    assert traced(tr=vp((1 << 24) + 4)) == salsc.SALSC_ERR_INVALID_ARG  # not 8-byte aligned
    assert traced(nb=need - 8) == salsc.SALSC_ERR_INVALID_ARG


def test_status_strings():
    for code in range(5):
        assert salsc.status_string(code)
    assert salsc.status_string(salsc.SALSC_ERR_WORKSPACE).startswith("workspace")


def desc(offs, **kw):
    a = dict(batch=len(offs) - 1, n_q_heads=32, n_kv_heads=8, head_dim=128, rank=256, top_k=64,
             rope_base=10000.0, softmax_scale=0.0, dtype=torch.bfloat16)
    a.update(kw)
    host = torch.tensor(offs, dtype=torch.int64)
    d = salsc.make_desc(a["batch"], a["n_q_heads"], a["n_kv_heads"], a["head_dim"], a["rank"],
                        a["top_k"], host, None, None, a["rope_base"], a["softmax_scale"], a["dtype"])
    d._keep = host
    return d


def test_workspace_size_valid_shapes_grow_with_tokens():
    small = salsc.salsc_decode_workspace_size(desc([0, 1000]))
    big = salsc.salsc_decode_workspace_size(desc([0, 1000, 40000]))
    assert 0 < small < big
    assert small % 256 == 0


def test_launch_count():
    # 8 units of one tile: clusters of 8 CTAs merge inside the attention kernel
    assert salsc.salsc_decode_launch_count(desc([0, 1000])) == 4
    # r > 256, the CUDA-core path, and 32 units of 16 tiles (the even split
    # over all SMs is wider than 32 clusters of 4): a separate merge kernel
    for kw in (dict(rank=512), dict(dtype=torch.float32)):
        assert salsc.salsc_decode_launch_count(desc([0, 1000], **kw)) == 5
    offs = [0, 4096, 8192, 12288, 16384]
    assert salsc.salsc_decode_launch_count(desc(offs, top_k=2048)) == 5
    with pytest.raises(ValueError):
        salsc.salsc_decode_launch_count(desc([0, 10], top_k=0))


@pytest.mark.parametrize("kw,offs", [
    (dict(n_q_heads=30), [0, 10]),             # Hq not a multiple of Hkv
    (dict(head_dim=127), [0, 10]),             # odd head dim
    (dict(top_k=0), [0, 10]),                  # k < 1
    (dict(rank=2048), [0, 10]),                # r > hidden / unsupported
    (dict(rope_base=1.0), [0, 10]),            # base must exceed 1
    (dict(softmax_scale=-1.0), [0, 10]),       # negative scale
    ({}, [0, 10, 10]),                         # empty sequence
    ({}, [1, 10]),                             # offsets must start at 0
    (dict(head_dim=96, n_kv_heads=8), [0, 10]),  # no kernel for d = 96
    (dict(rank=96), [0, 10]),                  # bf16 rank must be a multiple of 64
])
def test_invalid_descriptors_have_no_workspace(kw, offs):
    assert salsc.salsc_decode_workspace_size(desc(offs, **kw)) == 0


def call_step(d, q=1 << 20, kc=1 << 21, vc=1 << 22, pk=1 << 23, pv=1 << 24, out=1 << 25,
              idx=None, ws=1 << 26, ws_bytes=16):
    lib = salsc.load()
    vp = ctypes.c_void_p
    return lib.salsc_decode_step(ctypes.byref(d), vp(q), vp(kc), vp(vc), vp(pk), vp(pv), vp(out),
                                 vp(idx), vp(ws), ws_bytes, None)


def test_step_rejects_bad_arguments_before_launch():
    d = desc([0, 100])
    # no device offsets
    assert call_step(d) == salsc.SALSC_ERR_INVALID_ARG
    d.seq_offsets_dev = 1 << 27
    assert call_step(d, q=0) == salsc.SALSC_ERR_INVALID_ARG           # null q
    assert call_step(d, out=0) == salsc.SALSC_ERR_INVALID_ARG         # null out
    assert call_step(d, kc=(1 << 21) + 2) == salsc.SALSC_ERR_INVALID_ARG  # misaligned
    assert call_step(d, ws=0) == salsc.SALSC_ERR_WORKSPACE            # no workspace
    assert call_step(d, ws=(1 << 26) + 64) == salsc.SALSC_ERR_WORKSPACE  # misaligned workspace
    assert call_step(d, ws_bytes=16) == salsc.SALSC_ERR_WORKSPACE     # too small
    bad = desc([0, 100], top_k=0)
    bad.seq_offsets_dev = 1 << 27
    assert call_step(bad) == salsc.SALSC_ERR_INVALID_ARG


def test_prepare_rejects_short_workspace():
    lib = salsc.load()
    d = desc([0, 100])
    need = salsc.salsc_decode_workspace_size(d)
    st = lib.salsc_decode_prepare(ctypes.byref(d), ctypes.c_void_p(1 << 26), need - 1, None)
    assert st == salsc.SALSC_ERR_WORKSPACE
    st = lib.salsc_decode_prepare(ctypes.byref(d), None, need, None)
    assert st == salsc.SALSC_ERR_WORKSPACE


def test_append_validation_before_launch():
    lib = salsc.load()
    vp = ctypes.c_void_p
    ok = dict(K=vp(1 << 20), V=vp(1 << 21), Pk=vp(1 << 22), Pv=vp(1 << 23), Kc=vp(1 << 24),
              Vc=vp(1 << 25), rows=vp(1 << 26))

    def call(batch=2, hidden=1024, rank=256, dtype=1, **kw):
        a = dict(ok)
        a.update(kw)
        return lib.salsc_append(a["K"], a["V"], a["Pk"], a["Pv"], a["Kc"], a["Vc"], a["rows"],
                                batch, hidden, rank, dtype, None)

    assert call(K=None, V=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(rows=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(Pk=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(V=vp(1 << 21), Vc=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(batch=-1) == salsc.SALSC_ERR_INVALID_ARG
    assert call(dtype=7) == salsc.SALSC_ERR_INVALID_ARG
    assert call(hidden=16384) == salsc.SALSC_ERR_UNSUPPORTED
    assert call(batch=0) == salsc.SALSC_OK  # nothing to do, nothing launched


def test_fit_validation_before_launch():
    lib = salsc.load()
    vp = ctypes.c_void_p
    assert lib.salsc_fit_workspace_size(512, 64) >= 8 * 512 * 512
    assert lib.salsc_fit_workspace_size(64, 65) == 0     # rank > hidden
    assert lib.salsc_fit_workspace_size(4096, 2048) == 0  # rank > 1024
    ws = vp(1 << 24)

    def call(X=vp(1 << 20), n=1000, hidden=512, rank=64, omega=vp(1 << 21), iters=4,
             P=vp(1 << 22), dtype=1, ws=ws, ws_bytes=1 << 30):
        return lib.salsc_fit_projection(X, n, hidden, rank, omega, iters, P, dtype, ws, ws_bytes,
                                        None)

    assert call(X=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(omega=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(n=10) == salsc.SALSC_ERR_INVALID_ARG      # n < rank
    assert call(iters=-1) == salsc.SALSC_ERR_INVALID_ARG
    assert call(dtype=9) == salsc.SALSC_ERR_INVALID_ARG
    assert call(rank=2048, hidden=4096, n=5000) == salsc.SALSC_ERR_UNSUPPORTED
    assert call(ws=vp((1 << 24) + 8)) == salsc.SALSC_ERR_WORKSPACE  # misaligned
    assert call(ws_bytes=1000) == salsc.SALSC_ERR_WORKSPACE


def test_select_mode_validation():
    d = desc([0, 1000])
    assert salsc.salsc_decode_workspace_size(d) > 0
    d.select_mode = 2
    assert salsc.salsc_decode_workspace_size(d) == 0  # invalid descriptor
    d.select_mode = 1
    d.select_threshold = float("nan")
    assert salsc.salsc_decode_workspace_size(d) == 0
    d.select_threshold = -1e30
    assert salsc.salsc_decode_workspace_size(d) > 0


def test_step_append_validation_before_launch():
    lib = salsc.load()
    vp = ctypes.c_void_p

    class Dev:  # a device address that is never dereferenced
        def data_ptr(self):
            return 1 << 27

    def call(n_kv_heads=8, **kw):
        host = torch.tensor([0, 100, 250], dtype=torch.int64)
        d = salsc.make_desc(2, n_kv_heads * 4 if n_kv_heads <= 8 else n_kv_heads, n_kv_heads, 128,
                            256, 64, host, Dev(), None, 10000.0, 0.0, torch.bfloat16)
        a = dict(K=vp(1 << 20), V=vp(1 << 21), rows=vp(1 << 26))
        a.update(kw)
        buf = [vp(1 << (28 + i)) for i in range(7)]
        return lib.salsc_decode_step_append(ctypes.byref(d), a["K"], a["V"], a["rows"], *buf[:6],
                                            None, buf[6], 1 << 30, None)

    assert call(rows=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(K=None, V=None) == salsc.SALSC_ERR_INVALID_ARG
    assert call(n_kv_heads=128) == salsc.SALSC_ERR_UNSUPPORTED  # Hkv*d = 16384 > 8192


def test_compress_validation_before_launch():
    lib = salsc.load()
    vp = ctypes.c_void_p
    a, b, c = vp(1 << 20), vp(1 << 21), vp(1 << 22)
    # both halves missing
    assert lib.salsc_compress(None, None, a, b, c, c, 10, 64, 16, salsc.SALSC_BF16, None) == 1
    # hidden not a multiple of 16 (bf16)
    assert lib.salsc_compress(a, None, b, None, c, None, 10, 40, 16, salsc.SALSC_BF16, None) == 1
    # negative rows
    assert lib.salsc_compress(a, None, b, None, c, None, -1, 64, 16, salsc.SALSC_BF16, None) == 1
    # missing projection for a present half
    assert lib.salsc_compress(a, None, None, None, c, None, 10, 64, 16, salsc.SALSC_BF16, None) == 1
    # zero rows is a valid no-op (nothing is enqueued)
    assert lib.salsc_compress(a, None, b, None, c, None, 0, 64, 16, salsc.SALSC_BF16, None) == 0


def test_shard_validation_before_launch():
    """Token-sharded entry points: every argument check returns before a launch."""
    lib = salsc.load()
    vp = ctypes.c_void_p
    a, b, c = vp(1 << 20), vp(1 << 21), vp(1 << 22)
    host = torch.tensor([0, 1000, 1800], dtype=torch.int64)

    class FakeDev:  # a device address that is never dereferenced: every call fails a check
        def __init__(self, p):
            self.p = p

        def data_ptr(self):
            return self.p

    d = salsc.make_desc(2, 32, 8, 128, 256, 64, host, FakeDev(1 << 23), None, 10000.0, 0.0,
                        torch.bfloat16)
    need = lib.salsc_decode_workspace_size(ctypes.byref(d))
    ws = vp(1 << 28)

    def cand(dd=d, q=a, kc=b, pk=c, so=a, cs=b, ci=c, w=ws, n=need):
        return lib.salsc_shard_candidates(ctypes.byref(dd), q, kc, pk, so, cs, ci, w, n, None)

    assert cand(q=None) == salsc.SALSC_ERR_INVALID_ARG
    assert cand(so=None) == salsc.SALSC_ERR_INVALID_ARG
    assert cand(q=vp((1 << 20) + 8)) == salsc.SALSC_ERR_INVALID_ARG  # misaligned
    assert cand(n=need - 1) == salsc.SALSC_ERR_WORKSPACE
    dt = salsc.make_desc(2, 32, 8, 128, 256, 64, host, FakeDev(1 << 23), None, 10000.0, 0.0,
                         torch.bfloat16, 0.5)
    # threshold selection is sharded too; its arguments are checked the same way
    assert cand(dd=dt, q=None) == salsc.SALSC_ERR_INVALID_ARG
    assert cand(dd=dt, n=need - 1) == salsc.SALSC_ERR_WORKSPACE

    def sel(cs=a, ci=b, n=2, batch=2, units=8, k=64, lo=c, so=a, out=b):
        return lib.salsc_shard_select(cs, ci, n, batch, units, k, lo, so, out, None)

    assert sel(cs=None) == salsc.SALSC_ERR_INVALID_ARG
    assert sel(n=0) == salsc.SALSC_ERR_INVALID_ARG
    assert sel(n=8, k=4096) == salsc.SALSC_ERR_UNSUPPORTED  # 32768 candidates per unit
    assert sel(units=300) == salsc.SALSC_ERR_UNSUPPORTED

    def att(dd=d, idx=a, so=b, part=c, w=ws, n=need):
        return lib.salsc_shard_attend(ctypes.byref(dd), a, b, c, a, idx, so, part, w, n, None)

    assert att() == salsc.SALSC_ERR_INVALID_ARG  # the descriptor has no q_pos
    dq = salsc.make_desc(2, 32, 8, 128, 256, 64, host, FakeDev(1 << 23), FakeDev(1 << 24),
                         10000.0, 0.0, torch.bfloat16)
    assert att(dd=dq, idx=None) == salsc.SALSC_ERR_INVALID_ARG
    assert att(dd=dq, part=vp((1 << 22) + 4)) == salsc.SALSC_ERR_INVALID_ARG  # part not 16-aligned
    assert att(dd=dq, n=need - 1) == salsc.SALSC_ERR_WORKSPACE

    def merge(part=a, n=2, batch=2, hq=32, hkv=8, dh=128, r=256, dtype=1, pv=b, out=c, w=ws):
        return lib.salsc_shard_merge(part, n, batch, hq, hkv, dh, r, dtype, pv, out, w, 16, None)

    assert merge(dtype=7) == salsc.SALSC_ERR_INVALID_ARG
    assert merge(part=None) == salsc.SALSC_ERR_INVALID_ARG
    assert merge(hq=30) == salsc.SALSC_ERR_INVALID_ARG  # Hq not a multiple of Hkv
    assert merge(dh=96) == salsc.SALSC_ERR_UNSUPPORTED
    assert merge(hq=96, hkv=8) == salsc.SALSC_ERR_UNSUPPORTED  # 12 heads per unit
    assert merge(w=vp((1 << 28) + 8)) == salsc.SALSC_ERR_WORKSPACE
