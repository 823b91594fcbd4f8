"""The decode kernels' bounded waits give up instead of hanging.

Every pipeline wait of the decode kernels (mbarrier phases, the MMA issuer's
event loop) stops after a wall-time limit, records the timeout bit in the
workspace's anomaly word and returns.  salsc_check_wait_timeout runs that
same wait on a barrier that nothing completes, with a short limit and no copy
in flight; the GPU test checks that the kernel returns, that the bit is set,
and that the workspace serves a correct step after salsc_decode_prepare.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from latent_space_sparse_b200 import salsc, synth, workloads as W
from tests.parity import TOL, check_topk, max_rel_err, problem_of


def test_wait_check_arguments_are_validated():
    lib = salsc.load()
    vp = ctypes.c_void_p
    assert lib.salsc_check_wait_timeout(0, vp(1 << 20), 256, None) == salsc.SALSC_ERR_INVALID_ARG
    assert lib.salsc_check_wait_timeout(2_000_000_000, vp(1 << 20), 256, None) == \
        salsc.SALSC_ERR_INVALID_ARG
    assert lib.salsc_check_wait_timeout(1000, None, 256, None) == salsc.SALSC_ERR_WORKSPACE
    assert lib.salsc_check_wait_timeout(1000, vp((1 << 20) + 16), 256, None) == \
        salsc.SALSC_ERR_WORKSPACE
    assert lib.salsc_check_wait_timeout(1000, vp(1 << 20), 8, None) == salsc.SALSC_ERR_WORKSPACE


@pytest.mark.gpu
def test_a_wait_that_runs_out_sets_the_flag_and_the_context_stays_usable():
    w = W.Workload(name="wait_gqa", batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, rank=128,
                   top_k=256, seq_lens=(1500, 700), dtype="bf16", rope_base=10000.0,
                   low_rank=16, seed=71)
    x = synth.decode_inputs(w)
    dec = salsc.Decoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, w.top_k,
                        w.seq_lens, rope_base=w.rope_base, dtype=torch.bfloat16, device="cuda")
    assert dec.flags() == 0
    t0 = time.perf_counter()
    salsc.salsc_check_wait_timeout(2_000_000, dec.ws)  # 2 ms
    flags = dec.flags()  # synchronises: the kernel has returned
    elapsed = time.perf_counter() - t0
    assert flags & salsc.FLAG_WAIT_TIMEOUT
    assert elapsed < 5.0
    # the word is cleared by prepare, and the same workspace then serves a correct step
    salsc.salsc_decode_prepare(dec.desc, dec.ws)
    assert dec.flags() == 0
    t = {n: x[n].to("cuda") for n in ("q", "Kc", "Vc", "Pk", "Pv")}
    idx = torch.empty((w.batch, w.n_kv_heads, w.top_k), dtype=torch.int32, device="cuda")
    out = dec.step(t["q"], t["Kc"], t["Vc"], t["Pk"], t["Pv"], idx_out=idx)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    p = problem_of(w, x["seq_offsets"].numpy())
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    ih = idx.cpu().numpy()
    check_topk(p, ih, ora)
    given = oracle.attend_given_idx(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"], ih)
    assert max_rel_err(out.float().cpu().numpy(), given["out"]) <= TOL["bf16"]
