"""Writes tests/golden/tiny_oracle.json and tests/golden/tiny_qk_oracle.json from the oracle alone.

The MapFlow pages print no worked example with numbers, so the stored values here are the
oracle's own result on the tiny workload (one sequence of 256 tokens, B=32, 4 sender heads,
2 receiver heads, 1 KV head, d=64, f32, tau=0.9, 3 heavy columns, seed 0; the recipe of
synth.maps).  The file pins the oracle against silent drift and gives the GPU tests a second,
stored reference.  It calls nothing but `synth` (inputs) and `oracle/`.

The second file is compression straight from Q, K on a small case (two sequences of 150 and
70 tokens, 4 query heads over 2 key heads, d = 128, B = 64, tau = 0.9, the recipe of synth.qk,
seed 0): block masses, kept sets and sampled kept values of the oracle's float64 maps.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from synth import configs, maps as smaps  # noqa: E402


def tiny_case():
    w = configs.TINY
    L = w.lens[0]
    A = smaps.gen_maps(L, w.B, w.h_s, w.n_heavy, seed=w.seed, dtype=w.dtype)
    W = smaps.gen_w(1, w.h_r, w.h_s, seed=w.seed)[0].numpy()
    V = smaps.gen_v(L, w.h_kv, w.d, seed=w.seed, dtype=w.dtype)
    return w, A, W, V


def compute():
    w, A, W, V = tiny_case()
    L = w.lens[0]
    row_ptr, col_idx, values, seqs = oracle.compress_pack([A], [L], w.B, w.tau)
    r = seqs[0]
    bsr = lambda row: (r["kept"][row], r["values"][row])
    O = oracle.retrieve_step(bsr, w.B, W, V, w.h_kv, [(L, L)], [0])
    masses = [r["masses"][qb].tolist() for qb in range(-(-L // w.B))]
    return {
        "workload": "tiny: L=256 B=32 h_s=4 h_r=2 h_kv=1 d=64 f32 tau=0.9 n_heavy=3 seed=0",
        "row_ptr": row_ptr.tolist(),
        "col_idx": col_idx.tolist(),
        "block_mass": masses,
        "O_shape": list(O.shape),
        # every 16th query row in full (12 significant digits) plus sums over all of O
        "O_rows": list(range(0, L, 16)),
        "O_sampled": [float("%.12g" % x) for x in O[::16].reshape(-1)],
        "O_sum": float(O.sum()),
        "O_sumsq": float((O * O).sum()),
    }


QK_LENS, QK_HS, QK_HKV, QK_D, QK_B, QK_TAU = (150, 70), 4, 2, 128, 64, 0.9


def qk_case():
    from synth.qk import gen_qk
    return gen_qk(QK_LENS, QK_HS, QK_HKV, QK_D, 4, 0)


def compute_qk():
    Q, K = qk_case()
    start, rows = 0, []
    for L in QK_LENS:
        Qs, Ks = Q[start:start + L], K[start:start + L]
        for qb in range(-(-L // QK_B)):
            m, kept, info, vals = oracle.compress_qk_row(Qs, Ks, L, QK_B, qb, QK_TAU, QK_D ** -0.5)
            rows.append({"mass": [float("%.15g" % x) for x in m], "kept": kept.tolist(),
                         "vals_sum": float(vals.sum()),
                         "vals_sampled": [float("%.12g" % x) for x in vals.reshape(-1)[::997]]})
        start += L
    return {"workload": "qk: lens=(150, 70) h_s=4 h_kv=2 d=128 B=64 tau=0.9 seed=0 (synth.qk)",
            "rows": rows}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_qk_oracle.json"), "w") as f:
        json.dump(compute_qk(), f, indent=None, separators=(",", ":"))
        f.write("\n")
    out = compute()
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(out, f, indent=None, separators=(",", ":"))
        f.write("\n")
    print("wrote", len(out["col_idx"]), "kept blocks,", len(out["O_sampled"]), "sampled O values")
