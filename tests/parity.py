"""Comparison rules between the CUDA path and the oracle.

Top-k: the index sets must be identical except for swaps between tokens whose
oracle scores lie within ``band * max|s|`` of the k-th oracle score of the
unit (several index sets are then equally correct); slots >= k_b hold -1 and
the kept indices are distinct and inside the sequence.

Outputs: max-abs error at most ``tol * max|oracle output|`` (2e-2 for bf16
storage, 1e-4 for fp32).  Where the kept sets differ by allowed swaps, the
output is compared with the oracle's attention over the GPU's own kept set.
"""
import numpy as np

import oracle

TIE_BAND = 1e-4
TOL = {"bf16": 2e-2, "f32": 1e-4}


def problem_of(w, seq_offsets, q_pos=None, top_k=None):
    return oracle.Problem(w.batch if seq_offsets is None else len(seq_offsets) - 1, w.n_q_heads,
                          w.n_kv_heads, w.head_dim, w.rank, top_k or w.top_k,
                          np.asarray(seq_offsets, dtype=np.int64), w.rope_base, 0.0, q_pos)


def check_topk(p, gpu_idx, ora, band=TIE_BAND):
    """Returns the number of allowed swaps; raises AssertionError otherwise."""
    gpu_idx = np.asarray(gpu_idx)
    swaps = 0
    for b in range(p.batch):
        nb = int(p.seq_offsets[b + 1] - p.seq_offsets[b])
        kb = min(p.top_k, nb)
        for u in range(p.n_kv_heads):
            s = oracle.unit_scores(p, ora["scores"], b, u)
            g = gpu_idx[b, u]
            assert (g[kb:] == -1).all(), f"(b={b},u={u}) pad slots not -1"
            gk = g[:kb]
            assert ((gk >= 0) & (gk < nb)).all(), f"(b={b},u={u}) index out of range"
            assert len(np.unique(gk)) == kb, f"(b={b},u={u}) repeated index"
            o = ora["idx"][b, u, :kb]
            diff = np.setxor1d(gk, o)
            if diff.size:
                kth = s[o[-1]]
                lim = band * np.abs(s).max()
                bad = diff[np.abs(s[diff] - kth) > lim]
                assert bad.size == 0, (f"(b={b},u={u}) {bad.size} swaps outside the tie band: "
                                       f"tokens {bad[:8]} scores {s[bad[:8]]} kth {kth} band {lim}")
                swaps += diff.size // 2
    return swaps


def max_rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))
