"""Helpers of the GPU parity tests: run the CUDA path through the binding, run the oracle on
the same input bytes (copied from the device), compare."""
import os
from concurrent.futures import ThreadPoolExecutor

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
    once |O| >= 8); the relative-L2 bound applies to the raw difference.  The raw max-abs
    error and the number of elements whose raw error exceeds the max-abs bound are printed
    and returned beside the checked figures, so the effect of the rounding allowance is
    visible in every run."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    amax, rl2 = tol(dtype)
    slack = 0.0 if dtype == "f32" else bf16_half_ulp(want)
    diff = np.abs(got - want)
    err = float(np.max(diff - slack)) if got.size else 0.0
    raw = float(diff.max()) if got.size else 0.0
    n_raw = int((diff > amax).sum())
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)) if got.size else 0.0
    print(f"[O] {what}: max-abs beyond rounding {err:.3e}, raw max-abs {raw:.3e}, "
          f"raw > {amax}: {n_raw}/{got.size}, rel-L2 {rel:.3e}")
    assert err <= amax and rel <= rl2, f"{what}: max-abs {err:.3e} (<= {amax}), rel-L2 {rel:.3e} (<= {rl2})"
    return err, rel, raw, n_raw


def run_compress(w, pack, tau=None, capacity=None, with_mass=True):
    tau = w.tau if tau is None else tau
    cap = w.causal_blocks if capacity is None else capacity
    out = mf.alloc_bsr(sum(w.nqb), cap, w.h_s, w.B, pack.maps.dtype, pack.maps.device,
                       n_causal=w.causal_blocks if with_mass else 0)
    mf.mf_compress(pack.maps, pack.map_seq_offset, pack.cu_seqlens, max(w.lens), w.h_s, w.B, tau, out)
    return out


def host_bsr(b):
    return (b.row_ptr.cpu().numpy(), b.col_idx.cpu().numpy(), int(b.nnz.cpu()[0]))


def oracle_row(pack, w, s, qb, tau=None, slab=None):
    """Oracle masses / kept set / walk info / values of query block qb of sequence s, from the
    exact device bytes of that row's slab."""
    tau = w.tau if tau is None else tau
    B = w.B
    if slab is None:
        slab = row_slab(pack, w, s, qb)
    L = w.lens[s]
    m = oracle.row_masses(slab, L, B, qb)
    kept, info = oracle.select(m, qb, tau)
    vals = np.stack([oracle.gather_block(slab, L, B, qb, int(kb)) for kb in kept])
    return m, kept, info, vals


def row_slab(pack, w, s, qb):
    """Host copy of the causal part of query block qb's rows of every sender head."""
    B = w.B
    return pack.seq_view(s, w.h_s, B)[:, qb * B:(qb + 1) * B, :(qb + 1) * B].cpu()


def oracle_pool():
    """Threads for oracle calls: the C oracle runs with the GIL released (ctypes), so rows
    are computed in parallel on the host cores."""
    return ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


def compare_rows(w, pack, bsr, rows, tau=None, values=True):
    """Compare GPU and oracle compression on the (sequence, qb) rows.

    Every row's kept set is compared with the oracle's exactly.  A row may differ only when
    the oracle's walk puts it in the near-tie band (oracle.is_boundary: the walk ends within
    1e-5 of tau, or the last kept and first dropped masses lie within 1e-5 of the row total);
    such a row's GPU set must still be valid on the oracle's masses (ascending, diagonal
    present, reaching tau within rounding).  Returns {"orows": {(s, qb): (kept, values)},
    "flagged": rows in the near-tie band, "mismatched": rows whose set differs}."""
    tau = w.tau if tau is None else tau
    rp, ci, nnz = host_bsr(bsr)
    qbase = np.concatenate([[0], np.cumsum(w.nqb)[:-1]])
    cb_base = np.concatenate([[0], np.cumsum([n * (n + 1) // 2 for n in w.nqb])[:-1]])
    masses = bsr.block_mass.cpu().numpy() if bsr.block_mass is not None else None
    vals_gpu = bsr.values
    out, flagged, mismatched = {}, 0, 0
    with oracle_pool() as pool:
        futs = [(s, qb, pool.submit(oracle_row, pack, w, s, qb, tau, row_slab(pack, w, s, qb)))
                for s, qb in rows]
        for s, qb, f in futs:
            m, kept, info, vals = f.result()
            r = qbase[s] + qb
            g = ci[rp[r]:rp[r + 1]]
            if masses is not None:
                gm = masses[cb_base[s] + qb * (qb + 1) // 2:][:qb + 1]
                np.testing.assert_allclose(gm, m, rtol=2e-6, atol=1e-12, err_msg=f"masses s={s} qb={qb}")
            boundary = oracle.is_boundary(info, tau)
            flagged += int(boundary)
            if g.tolist() != kept.tolist():
                assert boundary, f"kept set s={s} qb={qb}: gpu {g} oracle {kept}"
                mismatched += 1
                # several kept sets are correct here: check the GPU's is valid on the oracle's masses
                assert g.tolist() == sorted(set(g.tolist())) and qb in g.tolist()
                assert m[g].sum() >= tau * m.sum() * (1 - 1e-5)
            elif values:
                gv = vals_gpu[rp[r]:rp[r + 1]].cpu()
                raw, _ = oracle.as_raw(gv)
                assert raw.tobytes() == vals.tobytes(), f"values s={s} qb={qb}"
            out[(s, qb)] = (kept, vals)
    return {"orows": out, "flagged": flagged, "mismatched": mismatched}


def check_rows(w, pack, bsr, rows, tau=None, values=True):
    """compare_rows for callers that want (oracle rows, near-tie rows)."""
    r = compare_rows(w, pack, bsr, rows, tau, values)
    return r["orows"], r["flagged"]


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
