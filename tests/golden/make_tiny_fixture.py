"""Write tests/golden/tiny_f32_oracle.json from the oracle alone.

The fixture freezes the oracle's answer on the seeded tiny fp32 workload
(B=1, 4 MHA heads, d=64, r=64, n=512, k=32) so that a later change to the
oracle or to the input generator shows up as a diff.  It calls only
``oracle`` and the seeded generator; nothing here touches the CUDA path.

    python tests/golden/make_tiny_fixture.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from latent_space_sparse_b200 import synth, workloads  # noqa: E402


def compute():
    w = workloads.TINY_F32
    x = synth.decode_inputs(w)
    p = oracle.Problem(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rank, w.top_k,
                       x["seq_offsets"].numpy(), w.rope_base)
    res = oracle.decode(p, x["q"], x["Kc"], x["Vc"], x["Pk"], x["Pv"])
    return w, x, res


def main():
    w, x, res = compute()
    fx = {
        "workload": w.name,
        "source": "oracle.decode on synth.decode_inputs(TINY_F32); written by make_tiny_fixture.py",
        "input_sums": {k: float(np.asarray(v.double().sum())) for k, v in x.items()
                       if k != "seq_offsets"},
        "idx_sorted": np.sort(res["idx"], axis=-1).tolist(),
        "out": res["out"].tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_oracle.json")
    with open(path, "w") as f:
        json.dump(fx, f, indent=None, separators=(",", ":"))
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
