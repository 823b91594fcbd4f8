"""The allocation-free decode entry point matches the workspace entry point.

salsc_decode_step_static_ws serves callers that cannot allocate device memory
(a plugin whose host application owns every device allocation, a serving
loop that must never call cudaMalloc): its scratch is a fixed array inside
the library.  These tests call it through the C ABI twice in a row, on two
different inputs, and compare each result with salsc_decode_step (which uses
a caller-allocated workspace).  Both entry points launch the same kernels on
the same inputs, so the outputs and the selected indices must be identical,
bit for bit.  This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from latent_space_sparse_b200 import salsc, synth, workloads as W

DEV = "cuda"


def _tensors(x):
    return {n: x[n].to(DEV) for n in ("q", "Kc", "Vc", "Pk", "Pv")}


@pytest.mark.gpu
@pytest.mark.parametrize("w,lens", [(W.TINY_F32, None), (W.MISTRAL_32K_B4, (4096, 2500)),
                                    (W.LLAMA2_4K_B1, (3000,))])
def test_static_workspace_matches_workspace_entry_point(w, lens):
    xs = [synth.decode_inputs(w, seq_lens=lens), synth.decode_inputs(w, seq_lens=lens,
                                                                     seed=w.seed + 17)]
    offs = xs[0]["seq_offsets"]
    lens_ = np.diff(offs.numpy())
    k = w.top_k
    B = len(lens_)
    host = offs.clone()
    dev_offs = host.to(DEV)
    desc = salsc.make_desc(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, k, host, dev_offs,
                           None, w.rope_base, 0.0, synth.torch_dtype(w.dtype))
    ts = [_tensors(x) for x in xs]
    outs = [torch.empty_like(t["q"]) for t in ts]
    idxs = [torch.full((B, w.n_kv_heads, k), -5, dtype=torch.int32, device=DEV) for _ in ts]
    # two calls in a row on the library's shared scratch, no synchronisation between them
    for t, o, i in zip(ts, outs, idxs):
        salsc.salsc_decode_step_static_ws(desc, t["q"], t["Kc"], t["Vc"], t["Pk"], t["Pv"], o, i)
    torch.cuda.synchronize()
    dec = salsc.Decoder(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, k, lens_,
                        rope_base=w.rope_base, dtype=synth.torch_dtype(w.dtype), device=DEV)
    for t, o, i in zip(ts, outs, idxs):
        ref_idx = torch.full_like(i, -5)
        ref = dec.step(t["q"], t["Kc"], t["Vc"], t["Pk"], t["Pv"], idx_out=ref_idx)
        torch.cuda.synchronize()
        assert torch.equal(o, ref), "outputs differ from salsc_decode_step"
        assert torch.equal(i, ref_idx), "selected indices differ from salsc_decode_step"
    assert dec.flags() == 0


@pytest.mark.parametrize("w", [w for w in W.ALL], ids=lambda w: w.name)
def test_every_full_size_workload_fits_the_static_scratch(w):
    # the header promises that every full-size workload of the suite fits the array
    host = torch.tensor(w.seq_offsets(), dtype=torch.int64)
    desc = salsc.make_desc(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, w.top_k, host,
                           None, None, w.rope_base, 0.0, synth.torch_dtype(w.dtype))
    need = salsc.salsc_decode_workspace_size(desc)
    assert 0 < need <= salsc.static_workspace_bytes(), (w.name, need)


class _FakeDev:
    """A device address that is never dereferenced (every call below fails a check)."""

    def __init__(self, p):
        self.p = p

    def data_ptr(self):
        return self.p


def test_shape_beyond_the_static_limit_is_rejected():
    # 32 units x 200000 tokens of fp32 scores alone exceed the 16 MiB array; the call is
    # rejected before anything is enqueued (the pointers are never dereferenced)
    host = torch.tensor([0, 200000], dtype=torch.int64)
    desc = salsc.make_desc(1, 32, 32, 128, 512, 64, host, _FakeDev(1 << 26), None, 10000.0,
                           0.0, torch.bfloat16)
    assert salsc.salsc_decode_workspace_size(desc) > salsc.static_workspace_bytes()
    lib = salsc.load()
    vp = ctypes.c_void_p
    st = lib.salsc_decode_step_static_ws(ctypes.byref(desc), vp(1 << 20), vp(1 << 21),
                                         vp(1 << 22), vp(1 << 23), vp(1 << 24), vp(1 << 25),
                                         None, None)
    assert st == salsc.SALSC_ERR_WORKSPACE


def test_static_size_matches_the_header():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "salsc.h")).read()
    m = re.search(r"#define SALSC_STATIC_WORKSPACE_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m, "SALSC_STATIC_WORKSPACE_BYTES not found in salsc.h"
    assert salsc.static_workspace_bytes() == int(m.group(1)) << int(m.group(2))


def test_rejected_call_enqueues_nothing():
    # a null query is reported before the scratch's anomaly word is cleared: no device
    # pointer of the call is touched, and without a CUDA device nothing could be enqueued
    host = torch.tensor([0, 512], dtype=torch.int64)
    desc = salsc.make_desc(1, 4, 4, 64, 64, 32, host, _FakeDev(1 << 26), None, 10000.0, 0.0,
                           torch.float32)
    lib = salsc.load()
    vp = ctypes.c_void_p
    st = lib.salsc_decode_step_static_ws(ctypes.byref(desc), None, vp(1 << 21), vp(1 << 22),
                                         vp(1 << 23), vp(1 << 24), vp(1 << 25), None, None)
    assert st == salsc.SALSC_ERR_INVALID_ARG
