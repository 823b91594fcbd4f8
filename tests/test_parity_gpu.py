"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Every call goes through the C ABI (libsalsc via the ctypes binding).  Rules
(tests/parity.py): top-k sets identical up to swaps inside the tie band
1e-4*max|s| of the k-th score; outputs within 2e-2 (bf16) / 1e-4 (fp32) of
the oracle output's max-abs, against the oracle's attention over the GPU's
own kept set, and against the plain oracle when the sets are identical.
Full-size workloads run in one launch, as in the benchmark, and every
sequence is compared with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from latent_space_sparse_b200 import salsc, synth, workloads as W
from tests.parity import TOL, check_topk, max_rel_err, problem_of

pytestmark = pytest.mark.gpu

DEV = "cuda"


def gpu_decode(w, x, top_k=None, q_pos=None, threshold=None):
    offs = x["seq_offsets"].numpy()
    lens = np.diff(offs)
    k = top_k or w.top_k
    dec = salsc.Decoder(len(lens), w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, k, lens,
                        rope_base=w.rope_base, dtype=synth.torch_dtype(w.dtype), device=DEV,
                        q_pos=None if q_pos is None else torch.as_tensor(q_pos),
                        select_threshold=threshold)
    t = {n: x[n].to(DEV) for n in ("q", "Kc", "Vc", "Pk", "Pv")}
    idx = torch.full((len(lens), w.n_kv_heads, k), -7, dtype=torch.int32, device=DEV)
    out = dec.step(t["q"], t["Kc"], t["Vc"], t["Pk"], t["Pv"], idx_out=idx)
    torch.cuda.synchronize()
    assert dec.flags() == 0
    return out.float().cpu().numpy(), idx.cpu().numpy()


def sub_inputs(x, seqs):
    """Inputs of the chosen sequences only (for the oracle)."""
    offs = x["seq_offsets"].numpy()
    rows = np.concatenate([np.arange(offs[b], offs[b + 1]) for b in seqs])
    lens = [offs[b + 1] - offs[b] for b in seqs]
    so = np.zeros(len(seqs) + 1, dtype=np.int64)
    so[1:] = np.cumsum(lens)
    return {"q": x["q"][list(seqs)], "Kc": x["Kc"][rows], "Vc": x["Vc"][rows], "Pk": x["Pk"],
            "Pv": x["Pv"], "seq_offsets": torch.from_numpy(so)}


def check(w, x, seqs=None, top_k=None, q_pos=None):
    out, idx = gpu_decode(w, x, top_k, q_pos)
    if seqs is not None:
        x = sub_inputs(x, seqs)
        out, idx = out[list(seqs)], idx[list(seqs)]
        q_pos = None if q_pos is None else np.asarray(q_pos)[list(seqs)]
    p = problem_of(w, x["seq_offsets"].numpy(), q_pos, top_k)
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    swaps = check_topk(p, idx, ora)
    given = oracle.attend_given_idx(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"], idx)
    err = max_rel_err(out, given["out"])
    assert err <= TOL[w.dtype], f"output error {err:.3e} vs oracle on the GPU's kept set"
    if swaps == 0:
        err2 = max_rel_err(out, ora["out"])
        assert err2 <= TOL[w.dtype], f"output error {err2:.3e} vs oracle"
    return swaps, idx, ora


# ------------------------------------------------------------ whole workloads

def test_tiny_f32():
    w = W.TINY_F32
    check(w, synth.decode_inputs(w))


def test_llama2_4k_b1():
    w = W.LLAMA2_4K_B1
    check(w, synth.decode_inputs(w))


def test_llama2_4k_b16_reduced():
    w = W.LLAMA2_4K_B16
    check(w, synth.decode_inputs(w, seq_lens=(1024, 777, 1500)))


def test_mistral_gqa_reduced():
    w = W.MISTRAL_32K_B4
    check(w, synth.decode_inputs(w, seq_lens=(4096, 2500)))


def test_llama31_ragged_reduced():
    # k = 4096 exceeds two of the lengths: k_b = n_b there
    w = W.LLAMA31_RAGGED_128K
    check(w, synth.decode_inputs(w, seq_lens=(1000, 3000, 5000, 8191)))


@pytest.mark.parametrize("w", [W.LLAMA2_4K_B16, W.MISTRAL_32K_B4, W.LLAMA31_RAGGED_128K],
                         ids=lambda w: w.name)
def test_full_size_every_sequence(w):
    # the full-size batch in one launch (the benchmark's configuration); every sequence,
    # including the ragged 32K, 64K and 128K ones, is compared with the oracle
    check(w, synth.decode_inputs(w), seqs=tuple(range(w.batch)))


# ------------------------------------------------------------ edge cases

def test_single_token_sequences_and_k_above_n():
    w = W.MISTRAL_32K_B4
    x = synth.decode_inputs(w, seq_lens=(1, 2, 130, 1))
    check(w, x, top_k=64)


def test_equal_lengths_k_above_n():
    # every sequence has the same length (the kernels' equal-length path),
    # shorter than k: every token is kept and the tail slots are -1
    w = W.Workload(name="equal_short", batch=3, n_q_heads=8, n_kv_heads=2, head_dim=128,
                   rank=256, top_k=300, seq_lens=(100, 100, 100), dtype="bf16",
                   rope_base=10000.0, low_rank=16, seed=91)
    check(w, synth.decode_inputs(w))


def test_k_equals_one():
    w = W.LLAMA2_4K_B1
    check(w, synth.decode_inputs(w, seq_lens=(700,)), top_k=1)


def test_all_equal_scores_take_lowest_indices():
    w = W.MISTRAL_32K_B4
    x = synth.decode_inputs(w, seq_lens=(600, 333))
    x["Kc"][:] = x["Kc"][0]  # every cached latent key identical: every score ties
    swaps, idx, ora = check(w, x, top_k=100)
    for b, nb in enumerate((600, 333)):
        for u in range(w.n_kv_heads):
            np.testing.assert_array_equal(np.sort(idx[b, u, :100]), np.arange(100))


def test_large_query_positions():
    w = W.LLAMA31_RAGGED_128K
    x = synth.decode_inputs(w, seq_lens=(2000, 900))
    check(w, x, top_k=256, q_pos=np.array([131071, 77777], dtype=np.int32))


def test_head_dim_64_gqa_bf16():
    w = W.Workload(name="gqa_d64", batch=2, n_q_heads=8, n_kv_heads=2, head_dim=64, rank=64,
                   top_k=40, seq_lens=(300, 129), dtype="bf16", rope_base=10000.0, low_rank=8,
                   seed=99)
    check(w, synth.decode_inputs(w))


def test_wide_rank_384_gqa():
    # 256 < r <= 512: the attention takes the latent width in two halves of
    # three 64-column blocks each
    w = W.Workload(name="gqa_r384", batch=2, n_q_heads=8, n_kv_heads=4, head_dim=128, rank=384,
                   top_k=200, seq_lens=(700, 300), dtype="bf16", rope_base=10000.0, low_rank=64,
                   seed=97)
    check(w, synth.decode_inputs(w))


def test_wide_rank_512_mha_many_tiles():
    # r = 512 with several tiles per unit and per CTA (tiles run one after another)
    w = W.LLAMA2_4K_B1
    check(w, synth.decode_inputs(w, seq_lens=(4096,)), top_k=1000)


@pytest.mark.parametrize("batch,heads,kv_heads,rank,top_k,lens", [
    (11, 32, 32, 512, 256, (300, 517, 900, 128, 640, 777, 256, 1000, 333, 129, 450)),  # ragged
    (9, 16, 16, 256, 256, (500,) * 9),               # equal lengths, r = 256
    (3, 16, 2, 256, 2048, (2100, 3000, 2500)),       # 8 heads a unit: three full CTAs of heads
    (5, 8, 4, 512, 256, (900, 1200, 64, 2000, 517)),  # 2 heads a unit, r = 512: a CTA part idle
])
def test_merge_one_warp_per_head(batch, heads, kv_heads, rank, top_k, lens):
    # the merge runs one warp per (sequence, query head, 16 output rows),
    # eight heads of one unit per CTA (the last CTA's spare warps idle); the
    # attention kernel leaves the merge to it (too many tiles a unit for the
    # in-kernel merge, or r > 256)
    w = W.Workload(name="merge_per_head", batch=batch, n_q_heads=heads, n_kv_heads=kv_heads,
                   head_dim=128, rank=rank, top_k=top_k, seq_lens=lens, dtype="bf16",
                   rope_base=10000.0, low_rank=32, seed=93 + batch)
    assert launches(w) == len(salsc.DECODE_KERNELS)
    check(w, synth.decode_inputs(w))


def launches(w, top_k=None):
    lens = w.seq_lens
    dec = salsc.Decoder(len(lens), w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                        top_k or w.top_k, lens, rope_base=w.rope_base,
                        dtype=synth.torch_dtype(w.dtype), device=DEV)
    return salsc.salsc_decode_launch_count(dec.desc)


def test_in_kernel_merge_one_tile_per_cta():
    # one sequence, 32 MHA units of 4 tiles: a cluster of 4 CTAs per unit
    # merges its partials and projects them inside the attention kernel
    w = W.Workload(name="mha_merge", batch=1, n_q_heads=32, n_kv_heads=32, head_dim=128,
                   rank=256, top_k=512, seq_lens=(3000,), dtype="bf16", rope_base=10000.0,
                   low_rank=32, seed=95)
    assert launches(w) == len(salsc.DECODE_KERNELS) - 1
    check(w, synth.decode_inputs(w))


def test_in_kernel_merge_ranks_without_tiles():
    # 2 units of 3 tiles on clusters of 8 CTAs: five ranks hold no tile and
    # merge an empty partial
    w = W.Workload(name="gqa_merge", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, rank=192,
                   top_k=300, seq_lens=(900,), dtype="bf16", rope_base=10000.0, low_rank=16,
                   seed=94)
    assert launches(w) == len(salsc.DECODE_KERNELS) - 1
    check(w, synth.decode_inputs(w))


def test_separate_merge_kernel_when_the_split_is_wider():
    # 32 units of 16 tiles: the even split over every SM beats clusters of 4
    w = W.Workload(name="gqa_split", batch=4, n_q_heads=32, n_kv_heads=8, head_dim=128,
                   rank=256, top_k=2048, seq_lens=(2500, 2200, 3000, 2049), dtype="bf16",
                   rope_base=10000.0, low_rank=32, seed=93)
    assert launches(w) == len(salsc.DECODE_KERNELS)
    check(w, synth.decode_inputs(w))


def check_threshold(w, x, tau, top_k=None):
    """Threshold selection: the kept set is the oracle's up to tokens whose score lies within
    the tie band of the k-th score or of the threshold; the output matches the oracle over
    the GPU's kept set."""
    out, idx = gpu_decode(w, x, top_k, threshold=tau)
    p = problem_of(w, x["seq_offsets"].numpy(), None, top_k)
    p.select_threshold = tau
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    k = p.top_k
    n_kept = 0
    for b in range(p.batch):
        for u in range(p.n_kv_heads):
            s = oracle.unit_scores(p, ora["scores"], b, u)
            g = idx[b, u]
            gk = g[g >= 0]
            n_kept += gk.size
            assert (g[gk.size:] == -1).all(), "kept slots are not a prefix"
            assert len(np.unique(gk)) == gk.size
            o = ora["idx"][b, u]
            o = o[o >= 0]
            lim = 1e-4 * np.abs(s).max()
            for t in np.setxor1d(gk, o):
                near_tau = abs(s[t] - tau) <= lim
                kth = np.sort(s)[::-1][min(k, s.size) - 1]
                assert near_tau or abs(s[t] - kth) <= lim, (b, u, t, s[t], tau)
            assert all(s[t] >= tau - lim for t in gk)
    given = oracle.attend_given_idx(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"], idx)
    assert max_rel_err(out, given["out"]) <= TOL[w.dtype] or np.abs(given["out"]).max() == 0
    if np.abs(given["out"]).max() == 0:
        assert np.abs(out).max() == 0
    return n_kept, ora


@pytest.mark.parametrize("wname,frac", [("MISTRAL_32K_B4", 0.5), ("MISTRAL_32K_B4", 0.97),
                                        ("TINY_F32", 0.6)])
def test_threshold_selection(wname, frac):
    # tau at a quantile of the top-k scores: part of the top-k set is dropped
    w = getattr(W, wname)
    x = synth.decode_inputs(w, seq_lens=(3000, 1500)) if w.dtype == "bf16" else synth.decode_inputs(w)
    k = 256 if w.dtype == "bf16" else w.top_k
    p = problem_of(w, x["seq_offsets"].numpy(), None, k)
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    kept = [oracle.unit_scores(p, ora["scores"], b, u)[t] for b in range(p.batch)
            for u in range(p.n_kv_heads) for t in ora["idx"][b, u] if t >= 0]
    tau = float(np.quantile(kept, frac))
    n_kept, ora = check_threshold(w, x, tau, top_k=k)
    assert 0 < n_kept < (ora["idx"] >= 0).size


def test_threshold_above_every_score_keeps_nothing():
    w = W.MISTRAL_32K_B4
    x = synth.decode_inputs(w, seq_lens=(700, 300))
    out, idx = gpu_decode(w, x, top_k=128, threshold=1e30)
    assert (idx == -1).all()
    assert np.abs(out).max() == 0


def test_threshold_minus_infinity_is_top_k():
    w = W.MISTRAL_32K_B4
    x = synth.decode_inputs(w, seq_lens=(900, 450))
    out0, idx0 = gpu_decode(w, x, top_k=200)
    out1, idx1 = gpu_decode(w, x, top_k=200, threshold=-np.inf)
    np.testing.assert_array_equal(np.sort(idx0, axis=-1), np.sort(idx1, axis=-1))
    np.testing.assert_array_equal(out0, out1)


@pytest.mark.parametrize("dt,n,h,r", [("f32", 2048, 512, 64), ("bf16", 3000, 1024, 256),
                                       ("f32", 257, 96, 96)])
def test_fit_projection_spans_the_dominant_subspace(dt, n, h, r):
    # a matrix with a known spectrum and a gap after the r-th singular value;
    # the oracle takes the same stored (rounded) matrix
    rng = np.random.default_rng(n + h + r)
    k = min(n, h)
    sig = np.concatenate([np.geomspace(20.0, 6.0, r), np.geomspace(2.0, 0.05, k - r)])[:k]
    U, _ = np.linalg.qr(rng.standard_normal((n, k)))
    V, _ = np.linalg.qr(rng.standard_normal((h, h)))
    X = (U * sig) @ V[:, :k].T
    Xt = torch.from_numpy(X).to(synth.torch_dtype(dt))
    omega = torch.from_numpy(rng.standard_normal((h, r)).astype(np.float32))
    P, flags = salsc.salsc_fit_projection(Xt.to(DEV), r, omega.to(DEV), iters=12)
    torch.cuda.synchronize()
    assert flags == 0
    Pg = P.double().cpu().numpy()
    ref = oracle.fit_subspace(Xt, r)
    tol = TOL[dt]
    assert np.abs(Pg.T @ Pg - np.eye(r)).max() <= tol
    assert np.abs(Pg @ Pg.T - ref @ ref.T).max() <= tol


def test_small_rank_f32():
    w = W.Workload(name="f32_r16", batch=3, n_q_heads=6, n_kv_heads=3, head_dim=64, rank=16,
                   top_k=9, seq_lens=(50, 17, 200), dtype="f32", rope_base=500000.0, low_rank=4,
                   seed=98)
    check(w, synth.decode_inputs(w))


def test_repeated_steps_are_deterministic():
    w = W.MISTRAL_32K_B4
    x = synth.decode_inputs(w, seq_lens=(3000, 1000))
    a_out, a_idx = gpu_decode(w, x)
    b_out, b_idx = gpu_decode(w, x)
    np.testing.assert_array_equal(a_idx, b_idx)
    np.testing.assert_array_equal(a_out, b_out)


# ------------------------------------------------------------ compression

def test_compress_tiny_f32():
    w = W.TINY_F32
    x = synth.compress_inputs(w, rows=512)
    K, V, Pk, Pv = (x[n].to(DEV) for n in ("K", "V", "Pk", "Pv"))
    Kc = torch.empty(512, w.rank, device=DEV)
    Vc = torch.empty_like(Kc)
    salsc.salsc_compress(K, V, Pk, Pv, Kc, Vc)
    torch.cuda.synchronize()
    for got, X, P in ((Kc, x["K"], x["Pk"]), (Vc, x["V"], x["Pv"])):
        ref = oracle.compress(X, P)
        assert max_rel_err(got.cpu().numpy(), ref) <= TOL["f32"]


def test_compress_llama2_prefill_sampled_rows():
    w = W.LLAMA2_4K_B16
    rows = w.compress_rows
    x = synth.compress_inputs(w, rows=rows)
    K, V, Pk, Pv = (x[n].to(DEV) for n in ("K", "V", "Pk", "Pv"))
    Kc = torch.empty(rows, w.rank, dtype=torch.bfloat16, device=DEV)
    Vc = torch.empty_like(Kc)
    salsc.salsc_compress(K, V, Pk, Pv, Kc, Vc)
    torch.cuda.synchronize()
    sample = np.random.default_rng(0).choice(rows, 256, replace=False)
    sample = np.concatenate([sample, [0, rows - 1]])
    for got, X, P in ((Kc, x["K"], x["Pk"]), (Vc, x["V"], x["Pv"])):
        ref = oracle.compress(X[sample], P)
        g = got[torch.from_numpy(sample).to(DEV)].float().cpu().numpy()
        assert max_rel_err(g, ref) <= TOL["bf16"]
        # one rounding of an fp32 accumulation: almost every entry is the
        # correctly rounded bf16 value or its neighbour
        exact = oracle.round_storage(ref, "bf16")
        assert np.mean(g == exact) > 0.9


def test_compress_one_half_only():
    w = W.TINY_F32
    x = synth.compress_inputs(w, rows=100)
    V, Pv = x["V"].to(DEV), x["Pv"].to(DEV)
    Vc = torch.empty(100, w.rank, device=DEV)
    salsc.salsc_compress(None, V, None, Pv, None, Vc)
    torch.cuda.synchronize()
    assert max_rel_err(Vc.cpu().numpy(), oracle.compress(x["V"], x["Pv"])) <= TOL["f32"]


@pytest.mark.parametrize("rows,hid,r", [
    (100, 256, 256),     # CTA pairs: the second CTA's 128 rows all lie past the last row
    (1000, 1024, 256),   # 256-column tiles, two 128-row sub-tiles, ragged last row block
    (300, 512, 512),     # two latent column tiles
    (130, 256, 128),     # 128-column tiles, one sub-tile
    (77, 128, 64),       # 64-column tiles, fewer rows than one block
    (513, 208, 192),     # hidden not a multiple of 64 (zero-filled K tail), 64-column tiles
])
def test_compress_tensor_core_shapes(rows, hid, r):
    w = W.Workload(name="cmp", batch=1, n_q_heads=1, n_kv_heads=1, head_dim=hid, rank=r,
                   top_k=1, seq_lens=(rows,), dtype="bf16", rope_base=10000.0, low_rank=16,
                   seed=rows + hid + r)
    x = synth.compress_inputs(w, rows=rows)
    K, V, Pk, Pv = (x[n].to(DEV) for n in ("K", "V", "Pk", "Pv"))
    Kc = torch.full((rows, r), float("nan"), dtype=torch.bfloat16, device=DEV)
    Vc = torch.full_like(Kc, float("nan"))
    salsc.salsc_compress(K, V, Pk, Pv, Kc, Vc)
    torch.cuda.synchronize()
    for got, X, P in ((Kc, x["K"], x["Pk"]), (Vc, x["V"], x["Pv"])):
        ref = oracle.compress(X, P)
        g = got.float().cpu().numpy()
        assert np.isfinite(g).all()
        assert max_rel_err(g, ref) <= TOL["bf16"]
        assert np.mean(g == oracle.round_storage(ref, "bf16")) > 0.9


def test_compress_tensor_core_one_half_only():
    w = W.LLAMA2_4K_B1
    rows = 700
    x = synth.compress_inputs(w, rows=rows)
    K, Pk = x["K"].to(DEV), x["Pk"].to(DEV)
    Kc = torch.zeros(rows, w.rank, dtype=torch.bfloat16, device=DEV)
    salsc.salsc_compress(K, None, Pk, None, Kc, None)
    torch.cuda.synchronize()
    ref = oracle.compress(x["K"], x["Pk"])
    assert max_rel_err(Kc.float().cpu().numpy(), ref) <= TOL["bf16"]


# ------------------------------------------------------------ decode-time append

@pytest.mark.parametrize("wname,dt", [("LLAMA2_4K_B16", "bf16"), ("MISTRAL_32K_B4", "bf16"),
                                      ("TINY_F32", "f32")])
def test_append_new_rows_match_the_oracle(wname, dt):
    w = getattr(W, wname)
    B = max(3, w.batch)
    x = synth.compress_inputs(w, rows=B, seed=w.seed + 5)
    K, V, Pk, Pv = (x[n].to(DEV) for n in ("K", "V", "Pk", "Pv"))
    tdt = synth.torch_dtype(dt)
    n_rows = 50 + 7 * B
    Kc = torch.full((n_rows, w.rank), 3.0, dtype=tdt, device=DEV)
    Vc = torch.full_like(Kc, -2.0)
    # destination rows: distinct, not in order
    rows_np = np.random.default_rng(1).choice(n_rows, B, replace=False).astype(np.int64)
    rows = torch.from_numpy(rows_np).to(DEV)
    salsc.salsc_append(K, V, Pk, Pv, Kc, Vc, rows)
    torch.cuda.synchronize()
    for got, X, P, fill in ((Kc, x["K"], x["Pk"], 3.0), (Vc, x["V"], x["Pv"], -2.0)):
        g = got.float().cpu().numpy()
        ref = oracle.compress(X, P)
        assert max_rel_err(g[rows_np], ref) <= TOL[dt]
        others = np.setdiff1d(np.arange(n_rows), rows_np)
        assert (g[others] == fill).all()  # nothing else written


def test_step_append_equals_append_then_step():
    # the new token's rows written at each sequence's last row, then the step
    # over the updated caches with the query at that token's position
    w = W.Workload(name="gqa_app", batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, rank=128,
                   top_k=64, seq_lens=(300, 201), dtype="bf16", rope_base=10000.0, low_rank=16,
                   seed=92)
    x = synth.decode_inputs(w)
    offs = x["seq_offsets"].numpy()
    lens = np.diff(offs)
    new = synth.compress_inputs(w, rows=w.batch, seed=w.seed + 1)
    K_new = new["K"][:, : w.n_kv_heads * w.head_dim].contiguous().to(DEV)
    V_new = new["V"][:, : w.n_kv_heads * w.head_dim].contiguous().to(DEV)
    rows = torch.from_numpy(offs[1:] - 1).to(DEV)
    q_pos = torch.from_numpy((lens - 1).astype(np.int32))
    t = {n: x[n].to(DEV) for n in ("q", "Pk", "Pv")}
    dec = salsc.Decoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, w.top_k, lens,
                        rope_base=w.rope_base, dtype=torch.bfloat16, device=DEV, q_pos=q_pos)
    res = []
    for fused in (False, True):
        Kc, Vc = x["Kc"].to(DEV), x["Vc"].to(DEV)
        out = torch.empty_like(t["q"])
        idx = torch.empty((w.batch, w.n_kv_heads, w.top_k), dtype=torch.int32, device=DEV)
        if fused:
            salsc.salsc_decode_step_append(dec.desc, K_new, V_new, rows, t["q"], Kc, Vc, t["Pk"],
                                           t["Pv"], out, idx, dec.ws)
        else:
            salsc.salsc_append(K_new, V_new, t["Pk"], t["Pv"], Kc, Vc, rows)
            dec.step(t["q"], Kc, Vc, t["Pk"], t["Pv"], out=out, idx_out=idx)
        torch.cuda.synchronize()
        res.append((Kc.cpu(), Vc.cpu(), out.cpu(), idx.cpu()))
    assert dec.flags() == 0
    for a_, b_ in zip(res[0], res[1]):
        assert torch.equal(a_, b_)
    # the oracle on the updated caches
    Kc, Vc, out, idx = res[1]
    x2 = dict(x, Kc=Kc, Vc=Vc)
    p = problem_of(w, offs, q_pos.numpy())
    ora = oracle.decode(p, x2["q"], x2["Kc"], x2["Vc"], x2["Pk"], x2["Pv"])
    check_topk(p, idx.numpy(), ora)
    given = oracle.attend_given_idx(p, x2["q"], x2["Kc"], x2["Vc"], x2["Pk"], x2["Pv"], idx.numpy())
    assert max_rel_err(out.float().numpy(), given["out"]) <= TOL["bf16"]


def test_append_one_half_and_batch_above_one_pass():
    w = W.MISTRAL_32K_B4
    B = 37  # more sequences than one pass of the kernel takes
    x = synth.compress_inputs(w, rows=B, seed=3)
    V, Pv = x["V"].to(DEV), x["Pv"].to(DEV)
    Vc = torch.zeros(B + 5, w.rank, dtype=torch.bfloat16, device=DEV)
    rows = torch.arange(5, B + 5, dtype=torch.int64, device=DEV)
    salsc.salsc_append(None, V, None, Pv, None, Vc, rows)
    torch.cuda.synchronize()
    ref = oracle.compress(x["V"], x["Pv"])
    assert max_rel_err(Vc[5:].float().cpu().numpy(), ref) <= TOL["bf16"]
    assert (Vc[:5] == 0).all()
