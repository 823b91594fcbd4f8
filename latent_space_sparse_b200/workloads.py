"""Decode workloads: shapes of one SALS decode layer-step.

Shapes follow the model families the SALS page evaluates (LLaMA2-7B,
Mistral-7B, LLaMA3.1-8B on RULER-128k; "SALS: Sparse Attention in Latent
Space for KV cache Compression", English abstract).  The latent rank r and
top-k are the values chosen for this library's measurements; the pages state
neither.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rank: int
    top_k: int
    seq_lens: tuple
    dtype: str  # "f32" or "bf16" storage
    rope_base: float
    low_rank: int  # rank of the synthetic key matrix before projection
    seed: int
    compress_rows: int = 0  # rows of the prefill compression GEMM (0 = none)
    notes: str = field(default="", compare=False)

    @property
    def hidden(self) -> int:
        """KV hidden size Hkv*d: rows of Pk and Pv."""
        return self.n_kv_heads * self.head_dim

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_tokens(self) -> int:
        return int(sum(self.seq_lens))

    def seq_offsets(self):
        offs = [0]
        for n in self.seq_lens:
            offs.append(offs[-1] + int(n))
        return offs


TINY_F32 = Workload(
    name="tiny_mha4_d64_r64_n512_k32_f32", batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64,
    rank=64, top_k=32, seq_lens=(512,), dtype="f32", rope_base=10000.0, low_rank=16,
    seed=20261200, notes="fp32 correctness case; positions 0..511")

LLAMA2_4K_B1 = Workload(
    name="llama2_7b_mha32_d128_r512_n4096_b1_k512_bf16", batch=1, n_q_heads=32, n_kv_heads=32,
    head_dim=128, rank=512, top_k=512, seq_lens=(4096,), dtype="bf16", rope_base=10000.0,
    low_rank=256, seed=20261201)

LLAMA2_4K_B16 = Workload(
    name="llama2_7b_mha32_d128_r512_n4096_b16_k256_bf16", batch=16, n_q_heads=32, n_kv_heads=32,
    head_dim=128, rank=512, top_k=256, seq_lens=(4096,) * 16, dtype="bf16", rope_base=10000.0,
    low_rank=256, seed=20261202, compress_rows=16 * 4096,
    notes="also the prefill compression GEMM (65536 x 4096) . (4096 x 512), K and V")

MISTRAL_32K_B4 = Workload(
    name="mistral_7b_gqa32x8_d128_r256_n32768_b4_k2048_bf16", batch=4, n_q_heads=32,
    n_kv_heads=8, head_dim=128, rank=256, top_k=2048, seq_lens=(32768,) * 4, dtype="bf16",
    rope_base=10000.0, low_rank=128, seed=20261203, notes="sliding window disabled")

LLAMA31_RAGGED_128K = Workload(
    name="llama31_8b_gqa32x8_d128_r256_ragged16k-128k_b4_k4096_bf16", batch=4, n_q_heads=32,
    n_kv_heads=8, head_dim=128, rank=256, top_k=4096, seq_lens=(16384, 32768, 65536, 131072),
    dtype="bf16", rope_base=500000.0, low_rank=128, seed=20261204)

ALL = (TINY_F32, LLAMA2_4K_B1, LLAMA2_4K_B16, MISTRAL_32K_B4, LLAMA31_RAGGED_128K)
BY_NAME = {w.name: w for w in ALL}
