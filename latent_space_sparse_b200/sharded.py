"""Token-sharded decode over the ranks of a process group (one process per GPU).

Every sequence's tokens are split into contiguous slices, one per rank; a rank
holds the latent caches Kc/Vc of its slices only, and q, Pk, Pv whole.  One
layer-step (SALS technical framework, stages 2-4, exact: a token among a
unit's k best overall has fewer than k better tokens in its own slice, so it
is in that slice's local top-k):

1. local scoring and top-k -> candidates (score, global token index) per unit;
2. all-gather of the candidates (U*k*8 bytes per sequence and rank);
3. every rank selects the same global top-k and keeps the tokens of its slice;
4. attention over them -> one partial row (m, l, acc[r]) per query head;
5. all-gather of the partial rows (Hq*(r+4)*4 bytes per sequence and rank);
6. merge of the ranks' rows and the value projection.

The compute steps run in libsalsc (``salsc_shard_*``); the two exchanges are
``torch.distributed`` all-gathers (NCCL over NVLink between GPUs).  The result
equals a single-GPU ``salsc_decode_step`` over the whole sequences up to
rounding order.  ``ops`` replaces the four compute steps (a test runs the
exchange logic on CPU ranks with its own implementation); by default they are
the library's and need a GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import salsc


def split_lengths(seq_lens, world: int):
    """Contiguous slices of every sequence over ``world`` ranks, as even as
    possible (the first ``n % world`` ranks take one token more).

    Returns, per rank, (local lengths [B], global index of each slice's first
    token [B]).  Every slice must hold a token."""
    out = [([], []) for _ in range(world)]
    for n in (int(x) for x in seq_lens):
        if n < world:
            raise ValueError(f"a sequence of {n} tokens cannot give each of {world} ranks a token")
        start = 0
        for r in range(world):
            ln = n // world + (1 if r < n % world else 0)
            out[r][0].append(ln)
            out[r][1].append(start)
            start += ln
    return out


def all_gather_stacked(out: torch.Tensor, inp: torch.Tensor, group=None) -> None:
    """out[s] = rank s's ``inp`` (out: [world, *inp.shape], contiguous)."""
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, inp, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), inp, group=group)


class CudaShardOps:
    """The four per-rank compute steps on this rank's GPU (libsalsc)."""

    def __init__(self, dec: salsc.Decoder, local_offsets: torch.Tensor, shard_off: torch.Tensor):
        self.dec = dec
        self.local_offsets = local_offsets
        self.shard_off = shard_off

    def candidates(self, q, Kc, Pk, cand_score, cand_idx):
        salsc.salsc_shard_candidates(self.dec.desc, q, Kc, Pk, self.shard_off, cand_score,
                                     cand_idx, self.dec.ws)

    def select(self, cand_score_all, cand_idx_all, idx_local):
        salsc.salsc_shard_select(cand_score_all, cand_idx_all, self.local_offsets, self.shard_off,
                                 idx_local)

    def attend(self, q, Kc, Vc, Pk, idx_local, part):
        salsc.salsc_shard_attend(self.dec.desc, q, Kc, Vc, Pk, idx_local, self.shard_off, part,
                                 self.dec.ws)

    def merge(self, part_all, Pv, out, n_kv_heads, head_dim):
        salsc.salsc_shard_merge(part_all, n_kv_heads, head_dim, Pv, out, self.dec.ws)


class ShardedDecoder:
    """One decode shape on one rank of a token-sharded group.

    ``seq_lens`` are the whole sequences' lengths; this rank's slices follow
    from :func:`split_lengths`.  ``q_pos`` (int32 [B]) is the query's global
    position; None takes the whole sequence's length, as the single-GPU step
    does (a slice alone does not know where its sequence ends).
    ``select_threshold``: None for top-k selection, else threshold selection
    (of the k best tokens of a unit, those scoring below it are dropped); the
    local selections drop their candidates below it, which gives the same set
    as on one GPU.
    """

    def __init__(self, batch, n_q_heads, n_kv_heads, head_dim, rank, top_k, seq_lens, q_pos=None,
                 group=None, rope_base=10000.0, softmax_scale=0.0, dtype=torch.bfloat16,
                 device="cuda", ops=None, select_threshold=None):
        if len(seq_lens) != batch:
            raise ValueError("seq_lens must have one length per sequence")
        if q_pos is None:
            q_pos = [int(n) for n in seq_lens]
        self.q_pos = torch.as_tensor(q_pos, dtype=torch.int32)
        if self.q_pos.shape != (batch,):
            raise ValueError("q_pos must have one position per sequence")
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        local_lens, starts = split_lengths(seq_lens, self.world)[self.rank]
        self.local_lens = local_lens
        self.shard_off = torch.tensor(starts, dtype=torch.int64, device=device)
        offs = [0]
        for n in local_lens:
            offs.append(offs[-1] + n)
        self.local_offsets = torch.tensor(offs, dtype=torch.int64, device=device)
        self.n_kv_heads, self.head_dim = n_kv_heads, head_dim
        if ops is None:
            dec = salsc.Decoder(batch, n_q_heads, n_kv_heads, head_dim, rank, top_k, local_lens,
                                rope_base=rope_base, softmax_scale=softmax_scale, dtype=dtype,
                                device=device, q_pos=self.q_pos,
                                select_threshold=select_threshold)
            ops = CudaShardOps(dec, self.local_offsets, self.shard_off)
        self.ops = ops
        B, U, k, Hq, W = batch, n_kv_heads, top_k, n_q_heads, self.world
        f32, i32 = dict(dtype=torch.float32, device=device), dict(dtype=torch.int32, device=device)
        self.cand_score = torch.empty((B, U, k), **f32)
        self.cand_idx = torch.empty((B, U, k), **i32)
        self.cand_score_all = torch.empty((W, B, U, k), **f32)
        self.cand_idx_all = torch.empty((W, B, U, k), **i32)
        self.idx_local = torch.empty((B, U, k), **i32)
        self.part = torch.empty((B, Hq, rank + 4), **f32)
        self.part_all = torch.empty((W, B, Hq, rank + 4), **f32)

    def step(self, q, Kc, Vc, Pk, Pv, out=None):
        """One layer-step: q [B][Hq][d] and Pk, Pv whole; Kc, Vc this rank's slices
        ([sum of local lengths][r]).  Every rank must call it (two all-gathers)."""
        if out is None:
            out = torch.empty_like(q)
        self.ops.candidates(q, Kc, Pk, self.cand_score, self.cand_idx)
        all_gather_stacked(self.cand_score_all, self.cand_score, self.group)
        all_gather_stacked(self.cand_idx_all, self.cand_idx, self.group)
        self.ops.select(self.cand_score_all, self.cand_idx_all, self.idx_local)
        self.ops.attend(q, Kc, Vc, Pk, self.idx_local, self.part)
        all_gather_stacked(self.part_all, self.part, self.group)
        self.ops.merge(self.part_all, Pv, out, self.n_kv_heads, self.head_dim)
        return out
