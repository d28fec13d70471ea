"""Helpers of the GPU parity tests: run the CUDA path through the binding, run the oracle on
the same input bytes (copied from the device), compare."""
import numpy as np
import torch

import cross_model_attention_mf_b200 as mf
import oracle
from synth import device as sdev


def tol(dtype):
    return (1e-5, 1e-5) if dtype == "f32" else (2e-2, 1e-2)


def bf16_half_ulp(x):
    """Half a bf16 ulp at |x|: the most that rounding an exact value to bf16 can move it."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def assert_O_close(got, want, dtype, what=""):
    """max-abs and relative-L2 bounds: 1e-5 / 1e-5 for float32, 2e-2 / 1e-2 for bf16.
    For bf16 the max-abs bound applies to the error beyond the unavoidable rounding of the
    result to bf16 (half an ulp of the exact value, 2**-8 of it, which alone exceeds 2e-2
    once |O| >= 8); the relative-L2 bound applies to the raw difference."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    amax, rl2 = tol(dtype)
    slack = 0.0 if dtype == "f32" else bf16_half_ulp(want)
    err = float(np.max(np.abs(got - want) - slack)) if got.size else 0.0
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)) if got.size else 0.0
    assert err <= amax and rel <= rl2, f"{what}: max-abs {err:.3e} (<= {amax}), rel-L2 {rel:.3e} (<= {rl2})"
    return err, rel


def run_compress(w, pack, tau=None, capacity=None, with_mass=True):
    tau = w.tau if tau is None else tau
    cap = w.causal_blocks if capacity is None else capacity
    out = mf.alloc_bsr(sum(w.nqb), cap, w.h_s, w.B, pack.maps.dtype, pack.maps.device,
                       n_causal=w.causal_blocks if with_mass else 0)
    mf.mf_compress(pack.maps, pack.map_seq_offset, pack.cu_seqlens, max(w.lens), w.h_s, w.B, tau, out)
    return out


def host_bsr(b):
    return (b.row_ptr.cpu().numpy(), b.col_idx.cpu().numpy(), int(b.nnz.cpu()[0]))


def oracle_row(pack, w, s, qb, tau=None):
    """Oracle masses / kept set / walk info / values of query block qb of sequence s, from the
    exact device bytes of that row's slab."""
    tau = w.tau if tau is None else tau
    B = w.B
    slab = pack.seq_view(s, w.h_s, B)[:, qb * B:(qb + 1) * B, :(qb + 1) * B].cpu()
    L = w.lens[s]
    m = oracle.row_masses(slab, L, B, qb)
    kept, info = oracle.select(m, qb, tau)
    vals = np.stack([oracle.gather_block(slab, L, B, qb, int(kb)) for kb in kept])
    return m, kept, info, vals


def check_rows(w, pack, bsr, rows, tau=None, values=True):
    """Compare GPU and oracle compression on the (sequence, qb) rows.  Returns
    {(s, qb): (kept, values)} from the oracle and the number of boundary rows."""
    tau = w.tau if tau is None else tau
    rp, ci, nnz = host_bsr(bsr)
    qbase = np.concatenate([[0], np.cumsum(w.nqb)[:-1]])
    cb_base = np.concatenate([[0], np.cumsum([n * (n + 1) // 2 for n in w.nqb])[:-1]])
    masses = bsr.block_mass.cpu().numpy() if bsr.block_mass is not None else None
    vals_gpu = bsr.values
    out, nb = {}, 0
    for s, qb in rows:
        m, kept, info, vals = oracle_row(pack, w, s, qb, tau)
        r = qbase[s] + qb
        g = ci[rp[r]:rp[r + 1]]
        if masses is not None:
            gm = masses[cb_base[s] + qb * (qb + 1) // 2:][:qb + 1]
            np.testing.assert_allclose(gm, m, rtol=2e-6, atol=1e-12, err_msg=f"masses s={s} qb={qb}")
        if oracle.is_boundary(info, tau):
            nb += 1
            # several kept sets are correct here: check the GPU's is valid on the oracle's masses
            assert g.tolist() == sorted(g.tolist()) and qb in g.tolist()
            assert m[g].sum() >= tau * m.sum() * (1 - 1e-5)
        else:
            assert g.tolist() == kept.tolist(), f"kept set s={s} qb={qb}: gpu {g} oracle {kept}"
            if values:
                gv = vals_gpu[rp[r]:rp[r + 1]].cpu()
                raw, _ = oracle.as_raw(gv)
                assert raw.tobytes() == vals.tobytes(), f"values s={s} qb={qb}"
        out[(s, qb)] = (kept, vals)
    return out, nb


def oracle_O_rows(w, orows, s, qb, W_l, V_host, q0, k_start=0, block_table=None, page_size=0,
                  row_range=None):
    """Oracle O rows of query block qb of sequence s (positions >= q0 and < len)."""
    kept, vals = orows[(s, qb)]
    B = w.B
    L = w.lens[s]
    lo = max(q0, qb * B) - qb * B
    hi = min(L, (qb + 1) * B) - qb * B
    if row_range is not None:
        lo, hi = max(lo, row_range[0]), min(hi, row_range[1])
    return oracle.retrieve_block(vals, kept, qb, B, W_l, V_host, w.h_kv, (lo, hi), k_start,
                                 block_table, page_size), (lo, hi)
