"""Token-sharded decode across CPU ranks (gloo, world size 2 and 3): the
exchange logic of ShardedDecoder (slicing, the two all-gathers in shard-major
order, the global selection of each rank's tokens, the merge of the partial
rows) with the per-rank compute done here in fp64 numpy, against the
oracle's single-process decode of the whole sequences.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from latent_space_sparse_b200 import sharded, synth, workloads as W
from tests.parity import max_rel_err, problem_of


class NumpyShardOps:
    """The four per-rank steps in fp64 numpy, on this rank's slices."""

    def __init__(self, w, local_lens, starts, q_pos, tau=None):
        self.w = w
        self.tau = tau  # threshold selection: local candidates below it are dropped
        self.lens = list(local_lens)
        self.starts = list(starts)
        self.offs = np.concatenate([[0], np.cumsum(local_lens)]).astype(np.int64)
        self.q_pos = np.asarray(q_pos)

    def _unit(self, b, u):
        return slice(int(self.offs[b]), int(self.offs[b + 1]))

    def candidates(self, q, Kc, Pk, cand_score, cand_idx):
        w, G, d = self.w, self.w.n_q_heads // self.w.n_kv_heads, self.w.head_dim
        q, Kc, Pk = (t.double().numpy() for t in (q, Kc, Pk))
        k = cand_score.shape[-1]
        cand_score.fill_(-np.inf)
        cand_idx.fill_(-1)
        for b in range(len(self.lens)):
            for u in range(w.n_kv_heads):
                ql = q[b, u * G:(u + 1) * G].sum(axis=0) @ Pk[u * d:(u + 1) * d]
                s = Kc[self._unit(b, u)] @ ql
                order = np.lexsort((np.arange(s.size), -s))[:min(k, s.size)]
                if self.tau is not None:
                    order = order[s[order] >= self.tau]
                cand_score[b, u, :order.size] = torch.from_numpy(s[order])
                cand_idx[b, u, :order.size] = torch.from_numpy(order + self.starts[b])

    def select(self, cs, ci, idx_local):
        cs, ci = cs.double().numpy(), ci.numpy().astype(np.int64)
        N, B, U, K = cs.shape
        idx_local.fill_(-1)
        for b in range(B):
            lo, ln = self.starts[b], self.lens[b]
            for u in range(U):
                s, g = cs[:, b, u].reshape(-1), ci[:, b, u].reshape(-1)
                v = g >= 0
                best = np.lexsort((g[v], -s[v]))[:min(K, int(v.sum()))]
                chosen = set(g[v][best].tolist())
                mine = [x - lo for x in g.tolist() if x in chosen and lo <= x < lo + ln]
                idx_local[b, u, :len(mine)] = torch.tensor(mine, dtype=torch.int32)

    def attend(self, q, Kc, Vc, Pk, idx_local, part):
        w, G, d = self.w, self.w.n_q_heads // self.w.n_kv_heads, self.w.head_dim
        q, Kc, Vc, Pk = (t.double().numpy() for t in (q, Kc, Vc, Pk))
        scale = 1.0 / np.sqrt(d)
        part.zero_()
        for b in range(len(self.lens)):
            for u in range(w.n_kv_heads):
                t = idx_local[b, u].numpy()
                t = t[t >= 0]
                rows = Kc[self._unit(b, u)][t]
                K = np.stack([oracle.rope(rows[j] @ Pk[u * d:(u + 1) * d].T,
                                          self.starts[b] + int(t[j]), w.rope_base)
                              for j in range(t.size)]) if t.size else np.zeros((0, d))
                V = Vc[self._unit(b, u)][t]
                for g in range(G):
                    h = u * G + g
                    qr = oracle.rope(q[b, h], float(self.q_pos[b]), w.rope_base)
                    lg = K @ qr * scale
                    m = lg.max() if t.size else -np.inf
                    e = np.exp(lg - m) if t.size else np.zeros(0)
                    part[b, h, 0] = m
                    part[b, h, 1] = e.sum()
                    part[b, h, 4:] = torch.from_numpy(e @ V if t.size else np.zeros(V.shape[1]))

    def merge(self, part_all, Pv, out, n_kv_heads, head_dim):
        P, Pv = part_all.double().numpy(), Pv.double().numpy()
        G = P.shape[2] // n_kv_heads
        for b in range(P.shape[1]):
            for h in range(P.shape[2]):
                m, l, acc = P[:, b, h, 0], P[:, b, h, 1], P[:, b, h, 4:]
                M = m.max()
                wgt = np.where(m == -np.inf, 0.0, np.exp(m - M))
                a = (wgt[:, None] * acc).sum(axis=0) / (wgt * l).sum()
                u = h // G
                out[b, h] = torch.from_numpy(Pv[u * head_dim:(u + 1) * head_dim] @ a)


W_SHARD = W.Workload(name="gqa_shard_f32", batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
                     rank=32, top_k=48, seq_lens=(300, 170), dtype="f32", rope_base=10000.0,
                     low_rank=8, seed=71)
Q_POS = np.array([305, 170], dtype=np.int32)


def _workload(top_k):
    return W.Workload(**{**W_SHARD.__dict__, "top_k": top_k})


def _rank_main(rank, world, port, result_path, top_k, tau=None):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _workload(top_k)
        x = synth.decode_inputs(w)
        local_lens, starts = sharded.split_lengths(w.seq_lens, world)[rank]
        ops = NumpyShardOps(w, local_lens, starts, Q_POS, tau)
        sd = sharded.ShardedDecoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                                    w.top_k, w.seq_lens, Q_POS, rope_base=w.rope_base,
                                    dtype=torch.float32, device="cpu", ops=ops)
        offs = x["seq_offsets"].numpy()
        rows = np.concatenate([np.arange(offs[b] + st, offs[b] + st + ln)
                               for b, (ln, st) in enumerate(zip(local_lens, starts))])
        out = sd.step(x["q"], x["Kc"][rows], x["Vc"][rows], x["Pk"], x["Pv"])
        gathered = [torch.empty_like(out) for _ in range(world)]
        dist.all_gather(gathered, out)
        if rank == 0:
            np.save(result_path, torch.stack(gathered).numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,top_k", [(2, 48), (3, 48), (3, 120)])
def test_sharded_decoder_gloo_matches_oracle(world, top_k, tmp_path):
    # top_k = 120 over 3 ranks: every slice of the second sequence (57 tokens)
    # and of the first (100) is shorter than k, so slices keep all their tokens
    path = str(tmp_path / "out.npy")
    mp.start_processes(_rank_main, args=(world, _free_port(), path, top_k), nprocs=world,
                       join=True, start_method="spawn")
    outs = np.load(path)
    for r in range(1, world):
        np.testing.assert_array_equal(outs[r], outs[0])  # every rank ends with the same output
    w = _workload(top_k)
    x = synth.decode_inputs(w)
    p = problem_of(w, x["seq_offsets"].numpy(), Q_POS)
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    assert max_rel_err(outs[0], ora["out"]) <= 1e-5


def test_split_lengths():
    parts = sharded.split_lengths([10, 7], 3)
    assert [p[0] for p in parts] == [[4, 3], [3, 2], [3, 2]]
    assert [p[1] for p in parts] == [[0, 0], [4, 3], [7, 5]]
    with pytest.raises(ValueError):
        sharded.split_lengths([2], 3)


def test_sharded_decoder_checks_its_shapes(tmp_path):
    # a one-rank gloo group in this process: the checks run before any compute
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        w = W_SHARD
        with pytest.raises(ValueError):  # one length per sequence
            sharded.ShardedDecoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                                   w.top_k, (300,), Q_POS, device="cpu", ops=object())
        sd = sharded.ShardedDecoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                                    w.top_k, w.seq_lens, Q_POS, device="cpu", ops=object())
        assert sd.world == 1 and sd.local_lens == list(w.seq_lens)
        assert sd.shard_off.tolist() == [0, 0]
        assert sd.local_offsets.tolist() == [0, 300, 470]
        assert tuple(sd.cand_score_all.shape) == (1, w.batch, w.n_kv_heads, w.top_k)
        assert tuple(sd.part_all.shape) == (1, w.batch, w.n_q_heads, w.rank + 4)
        assert sd.q_pos.tolist() == [305, 170]
        # the default query position is the whole sequence's length
        sd0 = sharded.ShardedDecoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                                     w.top_k, w.seq_lens, device="cpu", ops=object())
        assert sd0.q_pos.tolist() == list(w.seq_lens)
        with pytest.raises(ValueError):
            sharded.ShardedDecoder(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank,
                                   w.top_k, w.seq_lens, [1, 2, 3], device="cpu", ops=object())
    finally:
        dist.destroy_process_group()


def test_threshold_selection_decomposes_over_slices(tmp_path):
    """Of the top-k tokens keep those scoring >= tau: each slice's top-k filtered by tau, then
    the k best of the candidates, gives the oracle's whole-sequence threshold selection (a kept
    token has fewer than k better tokens anywhere, all of them >= tau)."""
    world, top_k = 3, 48
    w = _workload(top_k)
    x = synth.decode_inputs(w)
    p = problem_of(w, x["seq_offsets"].numpy(), Q_POS)
    full = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    # tau between the 20th and 21st best scores of unit (0, 0): some units keep fewer than k
    s00 = np.sort(oracle.unit_scores(p, full["scores"], 0, 0))[::-1]
    tau = float((s00[19] + s00[20]) / 2)
    path = str(tmp_path / "out.npy")
    mp.start_processes(_rank_main, args=(world, _free_port(), path, top_k, tau), nprocs=world,
                       join=True, start_method="spawn")
    outs = np.load(path)
    p.select_threshold = tau
    ora = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    assert max_rel_err(outs[0], ora["out"]) <= 1e-5
