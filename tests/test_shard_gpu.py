"""Token-sharded decode on one GPU: the shards run one after another and the
all-gathers are stacks (nothing waits on another shard), through the C ABI.

- salsc_shard_select against a plain sort (score descending, lower global
  index first), bit-exact, on candidates full of ties;
- the six steps over 2 and 3 shards against the oracle's single-sequence
  decode (the rules of tests/parity.py: kept sets up to the tie band, outputs
  within the storage tolerance);
- ShardedDecoder on a one-rank NCCL group (the library ops and the
  all-gather wiring) against the oracle.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from latent_space_sparse_b200 import salsc, sharded, synth, workloads as W
from tests.parity import TOL, check_topk, max_rel_err, problem_of

pytestmark = pytest.mark.gpu

DEV = "cuda"


def ref_select(cs, ci, local_off, shard_off):
    """This shard's slice-local indices among the k best candidates, in candidate order."""
    N, B, U, K = cs.shape
    out = np.full((B, U, K), -1, dtype=np.int32)
    for b in range(B):
        lo, ln = int(shard_off[b]), int(local_off[b + 1] - local_off[b])
        for u in range(U):
            s = cs[:, b, u, :].reshape(-1).astype(np.float64)
            g = ci[:, b, u, :].reshape(-1).astype(np.int64)
            v = g >= 0
            order = np.lexsort((g[v], -s[v]))
            chosen = set(g[v][order[:min(K, int(v.sum()))]].tolist())
            mine = [x - lo for x in g.tolist() if x in chosen and lo <= x < lo + ln]
            out[b, u, :len(mine)] = mine
    return out


def test_shard_select_matches_sort_with_ties():
    rng = np.random.default_rng(5)
    N, B, U, k = 3, 2, 3, 40
    lens = np.array([[70, 50, 60], [30, 90, 45]])  # [b][shard]
    starts = np.concatenate([np.zeros((B, 1), int), np.cumsum(lens, axis=1)[:, :-1]], axis=1)
    cs = np.full((N, B, U, k), -np.inf, dtype=np.float32)
    ci = np.full((N, B, U, k), -1, dtype=np.int32)
    for s in range(N):
        for b in range(B):
            for u in range(U):
                m = min(k, int(lens[b, s]) - 3)  # a few slots empty
                loc = rng.choice(int(lens[b, s]), size=m, replace=False)
                ci[s, b, u, :m] = starts[b, s] + loc
                cs[s, b, u, :m] = rng.integers(-6, 6, size=m) * 0.5  # many equal scores
    cs_d, ci_d = torch.from_numpy(cs).to(DEV), torch.from_numpy(ci).to(DEV)
    for s in range(N):
        local = np.concatenate([[0], np.cumsum(lens[:, s])]).astype(np.int64)
        so = starts[:, s].astype(np.int64)
        out = torch.full((B, U, k), -9, dtype=torch.int32, device=DEV)
        salsc.salsc_shard_select(cs_d, ci_d, torch.from_numpy(local).to(DEV),
                                 torch.from_numpy(so).to(DEV), out)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy(), ref_select(cs, ci, local, so))


def shard_inputs(x, slices):
    """Rows of one shard: its slice [start, start + len) of every sequence."""
    offs = x["seq_offsets"].numpy()
    rows = np.concatenate([np.arange(offs[b] + st, offs[b] + st + ln)
                           for b, (ln, st) in enumerate(zip(*slices))])
    return x["Kc"][rows], x["Vc"][rows]


def run_shards(w, x, n_shards, q_pos, tau=None):
    """The six steps, shard by shard, on this GPU; returns (out, global kept idx).
    ``tau``: threshold selection (None: top-k)."""
    offs = x["seq_offsets"].numpy()
    lens = np.diff(offs)
    B, U, k, Hq, r = len(lens), w.n_kv_heads, w.top_k, w.n_q_heads, w.rank
    dt = synth.torch_dtype(w.dtype)
    parts = sharded.split_lengths(lens, n_shards)
    q, Pk, Pv = (x[n].to(DEV) for n in ("q", "Pk", "Pv"))
    qp = torch.as_tensor(q_pos, dtype=torch.int32)
    shards = []
    for local_lens, starts in parts:
        dec = salsc.Decoder(B, Hq, U, w.head_dim, r, k, local_lens, rope_base=w.rope_base,
                            dtype=dt, device=DEV, q_pos=qp, select_threshold=tau)
        Kc, Vc = (t.to(DEV) for t in shard_inputs(x, (local_lens, starts)))
        lo = torch.tensor(np.concatenate([[0], np.cumsum(local_lens)]), dtype=torch.int64,
                          device=DEV)
        so = torch.tensor(starts, dtype=torch.int64, device=DEV)
        shards.append(dict(dec=dec, Kc=Kc, Vc=Vc, lo=lo, so=so, starts=np.array(starts)))
    cs = torch.empty((n_shards, B, U, k), dtype=torch.float32, device=DEV)
    ci = torch.empty((n_shards, B, U, k), dtype=torch.int32, device=DEV)
    for s, sh in enumerate(shards):
        salsc.salsc_shard_candidates(sh["dec"].desc, q, sh["Kc"], Pk, sh["so"], cs[s], ci[s],
                                     sh["dec"].ws)
    part = torch.empty((n_shards, B, Hq, r + 4), dtype=torch.float32, device=DEV)
    kept = [[[] for _ in range(U)] for _ in range(B)]
    for s, sh in enumerate(shards):
        idx = torch.empty((B, U, k), dtype=torch.int32, device=DEV)
        salsc.salsc_shard_select(cs, ci, sh["lo"], sh["so"], idx)
        salsc.salsc_shard_attend(sh["dec"].desc, q, sh["Kc"], sh["Vc"], Pk, idx, sh["so"],
                                 part[s], sh["dec"].ws)
        ih = idx.cpu().numpy()
        for b in range(B):
            for u in range(U):
                loc = ih[b, u][ih[b, u] >= 0]
                kept[b][u].extend((loc + sh["starts"][b]).tolist())
    out = torch.empty_like(q)
    salsc.salsc_shard_merge(part, U, w.head_dim, Pv, out, shards[0]["dec"].ws)
    torch.cuda.synchronize()
    for sh in shards:
        assert sh["dec"].flags() == 0
    gidx = np.full((B, U, k), -1, dtype=np.int32)
    for b in range(B):
        for u in range(U):
            gidx[b, u, :len(kept[b][u])] = kept[b][u]
    return out.float().cpu().numpy(), gidx


def check_sharded(w, x, n_shards, q_pos):
    out, gidx = run_shards(w, x, n_shards, q_pos)
    p = problem_of(w, x["seq_offsets"].numpy(), q_pos)
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    swaps = check_topk(p, gidx, ora)
    given = oracle.attend_given_idx(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"], gidx)
    err = max_rel_err(out, given["out"])
    assert err <= TOL[w.dtype], f"output error {err:.3e} vs oracle on the kept set"
    if swaps == 0:
        assert max_rel_err(out, ora["out"]) <= TOL[w.dtype]


GQA = W.Workload(name="gqa_shard", batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, rank=128,
                 top_k=300, seq_lens=(1500, 1100), dtype="bf16", rope_base=10000.0, low_rank=16,
                 seed=61)


@pytest.mark.parametrize("n_shards", [2, 3])
def test_sharded_decode_gqa_bf16(n_shards):
    x = synth.decode_inputs(GQA)
    check_sharded(GQA, x, n_shards, np.array([1500, 1100], dtype=np.int32))


def test_sharded_decode_mistral_shape_k_above_a_slice():
    # Mistral-7B layout (8 units, r = 256): k = 2048 exceeds every slice of the
    # second sequence, so its slices keep all their tokens
    w = W.MISTRAL_32K_B4
    x = synth.decode_inputs(w, seq_lens=(6000, 3000))
    check_sharded(w, x, 2, np.array([6000, 3000], dtype=np.int32))


def test_sharded_decode_f32_cuda_cores():
    w = W.TINY_F32
    x = synth.decode_inputs(w)
    n = int(x["seq_offsets"][-1])
    check_sharded(w, x, 3, np.array([n + 5], dtype=np.int32))


@pytest.mark.parametrize("frac", [0.3, 0.9])
def test_sharded_threshold_selection_matches_the_oracle(frac):
    # threshold selection (of the k best tokens, those scoring >= tau) over 2 and 3 shards:
    # the kept set is the oracle's whole-sequence threshold selection up to tokens whose
    # score lies within the tie band of the k-th score or of tau; the output matches the
    # oracle's attention over the kept set
    w = GQA
    x = synth.decode_inputs(w)
    q_pos = np.array([1500, 1100], dtype=np.int32)
    p = problem_of(w, x["seq_offsets"].numpy(), q_pos)
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    kept = [oracle.unit_scores(p, ora["scores"], b, u)[t] for b in range(p.batch)
            for u in range(p.n_kv_heads) for t in ora["idx"][b, u] if t >= 0]
    tau = float(np.quantile(kept, frac))
    p.select_threshold = tau
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    for n_shards in (2, 3):
        out, gidx = run_shards(w, x, n_shards, q_pos, tau)
        n_kept = 0
        for b in range(p.batch):
            for u in range(p.n_kv_heads):
                s = oracle.unit_scores(p, ora["scores"], b, u)
                g = gidx[b, u][gidx[b, u] >= 0]
                n_kept += g.size
                assert len(np.unique(g)) == g.size
                o = ora["idx"][b, u]
                o = o[o >= 0]
                lim = 1e-4 * np.abs(s).max()
                kth = np.sort(s)[::-1][min(p.top_k, s.size) - 1]
                for t in np.setxor1d(g, o):
                    assert abs(s[t] - tau) <= lim or abs(s[t] - kth) <= lim, (b, u, t, s[t], tau)
                assert all(s[t] >= tau - lim for t in g)
        assert n_kept > 0
        given = oracle.attend_given_idx(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"], gidx)
        assert max_rel_err(out, given["out"]) <= TOL[w.dtype]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_decoder_one_rank_nccl_group():
    import torch.distributed as dist
    w = GQA
    x = synth.decode_inputs(w)
    q_pos = np.array([1500, 1100], dtype=np.int32)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device(DEV, 0))
    try:
        sd = sharded.ShardedDecoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                                    w.top_k, w.seq_lens, q_pos, rope_base=w.rope_base,
                                    dtype=synth.torch_dtype(w.dtype), device=DEV)
        t = {n: x[n].to(DEV) for n in ("q", "Kc", "Vc", "Pk", "Pv")}
        out = sd.step(t["q"], t["Kc"], t["Vc"], t["Pk"], t["Pv"]).float().cpu().numpy()
        torch.cuda.synchronize()
        idx = sd.idx_local.cpu().numpy()  # one rank: its slices are the sequences
    finally:
        dist.destroy_process_group()
    p = problem_of(w, x["seq_offsets"].numpy(), q_pos)
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    swaps = check_topk(p, idx, ora)
    given = oracle.attend_given_idx(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"], idx)
    assert max_rel_err(out, given["out"]) <= TOL[w.dtype]
    if swaps == 0:
        assert max_rel_err(out, ora["out"]) <= TOL[w.dtype]
