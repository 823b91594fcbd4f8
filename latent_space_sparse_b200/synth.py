"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and casts them to the storage type; it
holds none of the method's arithmetic.  Recipe (numpy PCG64, fp32 draws,
one round-to-nearest-even cast to the storage dtype; the cast values are the
canonical inputs for both sides):

* keys before projection: K = Z.Bm + 0.05 E, Z: n x R_low, Bm: R_low x hid,
  E: n x hid, all N(0, 1) (a low-rank key matrix plus noise);
* values and queries: N(0, 1);
* Pk, Pv: the Q factor of a QR decomposition of a seeded hid x r Gaussian
  (orthonormal columns; the "random matrix" projection choice);
* decode latents: Kc = Zl.C + 0.05 El with Zl: n x R_low, C: R_low x r,
  El: n x r, and Vc ~ N(0, 1).  For Pk with orthonormal columns drawn
  independently of Bm, K.Pk has exactly this law (Bm.Pk and E.Pk are again
  iid N(0, 1)), and so does V.Pv, so decode inputs are drawn directly in
  latent space and never come from a compression kernel.
"""
from __future__ import annotations

import numpy as np
import torch

from .workloads import Workload

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(dtype: str) -> torch.dtype:
    return _TORCH_DT[dtype]


def _cast(a: np.ndarray, dtype: str) -> torch.Tensor:
    """fp32 numpy -> CPU tensor in the storage dtype (RNE for bf16)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(_TORCH_DT[dtype]).contiguous()


def orthonormal(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    g = rng.standard_normal((rows, cols))
    q, _ = np.linalg.qr(g)
    return q.astype(np.float32)


def decode_inputs(w: Workload, layer: int = 0, seq_lens=None, seed: int | None = None) -> dict:
    """All inputs of one decode layer-step as CPU tensors in the storage dtype.

    Returns q [B][Hq][d], Kc and Vc [N][r], Pk and Pv [hid][r] and the int64
    seq_offsets [B+1].  ``seq_lens`` overrides the workload's lengths (used for
    reduced-size parity cases with the same per-token distributions).
    """
    lens = tuple(int(n) for n in (seq_lens if seq_lens is not None else w.seq_lens))
    rng = np.random.default_rng((seed if seed is not None else w.seed) + 7919 * layer)
    n = sum(lens)
    hid, r = w.hidden, w.rank
    zl = rng.standard_normal((n, w.low_rank), dtype=np.float32)
    c = rng.standard_normal((w.low_rank, r), dtype=np.float32)
    kc = zl @ c
    kc += np.float32(0.05) * rng.standard_normal((n, r), dtype=np.float32)
    vc = rng.standard_normal((n, r), dtype=np.float32)
    q = rng.standard_normal((len(lens), w.n_q_heads, w.head_dim), dtype=np.float32)
    pk = orthonormal(rng, hid, r)
    pv = orthonormal(rng, hid, r)
    offs = np.zeros(len(lens) + 1, dtype=np.int64)
    offs[1:] = np.cumsum(lens)
    return {
        "q": _cast(q, w.dtype),
        "Kc": _cast(kc, w.dtype),
        "Vc": _cast(vc, w.dtype),
        "Pk": _cast(pk, w.dtype),
        "Pv": _cast(pv, w.dtype),
        "seq_offsets": torch.from_numpy(offs),
    }


def compress_inputs(w: Workload, rows: int, seed: int | None = None) -> dict:
    """K, V [rows][hid] and Pk, Pv [hid][r] for the prefill compression GEMM."""
    rng = np.random.default_rng((seed if seed is not None else w.seed) + 104729)
    hid, r = w.hidden, w.rank
    z = rng.standard_normal((rows, w.low_rank), dtype=np.float32)
    bm = rng.standard_normal((w.low_rank, hid), dtype=np.float32)
    k = z @ bm
    k += np.float32(0.05) * rng.standard_normal((rows, hid), dtype=np.float32)
    v = rng.standard_normal((rows, hid), dtype=np.float32)
    pk = orthonormal(rng, hid, r)
    pv = orthonormal(rng, hid, r)
    return {"K": _cast(k, w.dtype), "V": _cast(v, w.dtype), "Pk": _cast(pk, w.dtype),
            "Pv": _cast(pv, w.dtype)}


def decode_inputs_device(w: Workload, layer: int, device, seq_lens=None) -> dict:
    """The same recipe drawn on the GPU with a seeded torch generator.

    Used for the extra layer buffer sets of the benchmark (fast to draw);
    parity tests use :func:`decode_inputs`, whose values the oracle sees.
    """
    lens = tuple(int(n) for n in (seq_lens if seq_lens is not None else w.seq_lens))
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1000 + layer)
    n = sum(lens)
    hid, r = w.hidden, w.rank
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    dt = _TORCH_DT[w.dtype]
    kc = torch.randn(n, w.low_rank, **f32) @ torch.randn(w.low_rank, r, **f32)
    kc += 0.05 * torch.randn(n, r, **f32)
    out = {
        "Kc": kc.to(dt),
        "Vc": torch.randn(n, r, **f32).to(dt),
        "q": torch.randn(len(lens), w.n_q_heads, w.head_dim, **f32).to(dt),
        "Pk": torch.linalg.qr(torch.randn(hid, r, **f32))[0].to(dt).contiguous(),
        "Pv": torch.linalg.qr(torch.randn(hid, r, **f32))[0].to(dt).contiguous(),
    }
    offs = torch.zeros(len(lens) + 1, dtype=torch.int64)
    offs[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0)
    out["seq_offsets"] = offs
    return out
