#!/usr/bin/env python
"""Benchmark of the MapFlow hot path on B200: one step = mf_compress of a sender layer
followed by mf_map_retrieve of a receiver layer (the whole hot path) on the
Ministral-like pair (L=8192, B=64, h_s=32, h_r=32, h_kv=8, d=128, bf16, tau=0.95).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Prints ONE JSON line (rank 0).  With N > 1 (torchrun) every rank runs an independent
replica of the workload (the path has no exchange step) and the value is the sum over
ranks divided by the slowest rank's time.  `--impl reference` times the CPU oracle on a
bounded sample of the same workload (there is no other implementation of this method
to run).
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mf_map_retrieve GB/s & prefill tokens/s/layer; % of roofline on 1 B200"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "measured (MEASURED_PEAKS.json)")
    return 6650.0, 1590.0, 1400.0, "fallback (MEASURED_PEAKS.json absent: 6.65 TB/s, 1.59 PFLOP/s)"


def measured_traffic(entry, workload):
    """DRAM bytes per launch from the last ncu capture of this entry point's kernels
    (profiles/traffic.txt), or None when the kernel source changed since the capture."""
    import hashlib
    src = {"mf_compress": "compress.cu", "mf_map_retrieve": "retrieve_tc.cu"}[entry]
    path = os.path.join(ROOT, "cross_model_attention_mf_b200", "csrc", src)
    sha = hashlib.sha1(open(path, "rb").read()).hexdigest()[:12]
    tpath = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(tpath):
        return None
    for line in open(tpath):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == entry and f[1] == sha and f[3] == workload:
            return int(f[2])
    return None


# ------------------------------------------------------------------------ clocks
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


def _nvml_handle(dev):
    """NVML handle of a CUDA device, matched by PCI location (CUDA_VISIBLE_DEVICES may renumber
    devices, so the CUDA ordinal is not NVML's)."""
    import pynvml
    pynvml.nvmlInit()
    p = torch.cuda.get_device_properties(dev)
    want = (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    for k in range(pynvml.nvmlDeviceGetCount()):
        h = pynvml.nvmlDeviceGetHandleByIndex(k)
        pi = pynvml.nvmlDeviceGetPciInfo(h)
        if (pi.domain, pi.bus, pi.device) == want:
            return h
    return None


class ClockSampler:
    """SM clock, its maximum and the clock-event reasons of one GPU, read through NVML (the
    library nvidia-smi reports from) every `period` seconds on a background thread.  Start it
    before the warm-up; `mark(True)` / `mark(False)` bracket the timed region, and `sample()`
    takes one extra reading on demand (call it before the closing synchronize, while the GPU
    is still busy), so even a timed region of a few milliseconds has readings of its own."""

    def __init__(self, dev, period=0.005):
        self.period = period
        self.samples = []        # (time, sm_mhz, max_mhz, reason bits)
        self.t_lo = self.t_hi = None
        self.h = None
        self.stop = threading.Event()
        self.err = None
        try:
            self.h = _nvml_handle(dev)
        except Exception as e:  # NVML missing: no clock record (reported as such)
            self.err = f"{type(e).__name__}: {e}"

    def sample(self):
        if self.h is None:
            return
        import pynvml
        try:
            sm = pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception as e:
            self.err = f"{type(e).__name__}: {e}"
            return
        self.samples.append((time.perf_counter(), float(sm), float(mx), int(bits)))

    def _run(self):
        while not self.stop.is_set():
            self.sample()
            self.stop.wait(self.period)

    def __enter__(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.h is not None:
            self.t.join(timeout=2)

    def mark(self, start):
        if start:
            self.t_lo = time.perf_counter()
        else:
            self.t_hi = time.perf_counter()

    def summary(self):
        lo = self.t_lo if self.t_lo is not None else -1e300
        hi = self.t_hi if self.t_hi is not None else 1e300
        timed = [x for x in self.samples if lo <= x[0] <= hi]
        if not timed:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml", "error": self.err or "no reading inside the timed region"}
        reasons = set()
        for x in timed:
            for b, name in REASONS.items():
                if x[3] & b and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[1] for x in timed),
                "sm_max_mhz": max(x[2] for x in timed), "reasons": sorted(reasons),
                "samples": len(timed), "samples_total": len(self.samples),
                "sm_mhz_min": min(x[1] for x in timed), "source": "nvml"}


# ------------------------------------------------------------------------ workload
def workload(name, reading):
    import synth
    w = synth.ALL[name]
    return w.with_(reading=reading) if reading != w.reading else w


def describe(w):
    return (f"{w.name}: lens={list(w.lens) if len(w.lens) <= 4 else f'{len(w.lens)} seqs'} B={w.B} "
            f"h_s={w.h_s} h_r={w.h_r} h_kv={w.h_kv} d={w.d} {w.dtype} tau={w.tau} "
            f"heavy={w.n_heavy} map reading R{w.reading}")


def algorithmic(w, nnz):
    """Algorithmic bytes / FLOPs of one compress and one retrieve launch: what the method must
    move once (every causal block read and the kept blocks written by compression; the kept
    blocks, V, O and the indices read or written by retrieval) and the mixing + P.V products."""
    e = 4 if w.dtype == "f32" else 2
    blk = w.h_s * w.B * w.B * e
    rows = sum(w.nqb)
    comp_bytes = w.causal_blocks * blk + nnz * blk + 4 * nnz + 4 * (rows + 1)
    ret_bytes = (nnz * blk + w.tokens * w.h_kv * w.d * e + w.tokens * w.h_r * w.d * e
                 + 4 * nnz + 4 * (rows + 1) + 4 * w.h_r * w.h_s)
    ret_flops = nnz * (2 * w.h_r * w.h_s * w.B * w.B + 2 * w.h_r * w.B * w.B * w.d)
    return comp_bytes, ret_bytes, ret_flops


# ------------------------------------------------------------------------ our arm
def run_ours(args, rank, world, dev):
    import cross_model_attention_mf_b200 as mf
    from synth import device as sdev

    w = workload(args.workload, args.reading)
    torch.cuda.set_device(dev)
    pack = sdev.fill_maps(sdev.alloc_maps(w, dev), w, 0)
    W = sdev.w_weights(w, dev)
    V = sdev.v_contiguous(w, 0, dev)
    cap = args.capacity if args.capacity > 0 else w.causal_blocks
    bsr = mf.alloc_bsr(sum(w.nqb), cap, w.h_s, w.B, pack.maps.dtype, dev)
    ws = torch.empty(mf.mf_compress_workspace_size(len(w.lens), max(w.lens), w.B, cap),
                     dtype=torch.uint8, device=dev)
    O = torch.empty((1, w.tokens, w.h_r, w.d), dtype=V.dtype, device=dev)
    qbase = sdev.qblock_base(w, dev)
    cu = pack.cu_seqlens
    maxlen = max(w.lens)
    st = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(st)
        mf.mf_compress(pack.maps, pack.map_seq_offset, cu, maxlen, w.h_s, w.B, w.tau, bsr, ws)
        if ev is not None:
            ev[1].record(st)
        mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qbase, maxlen, w.h_r, w.h_kv, O=O)
        if ev is not None:
            ev[2].record(st)

    clk = ClockSampler(dev).__enter__()  # runs from the warm-up to the end of the timed region
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"device status {rc} bits {bits:#x}")
    nnz = int(bsr.nnz.cpu()[0])

    # per-kernel durations (CUDA events on the launching stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(min(args.steps, 200))]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for ev in evs:
        step(ev)
    torch.cuda.synchronize()
    t_comp = statistics.mean(e[0].elapsed_time(e[1]) for e in evs) * 1e-3
    t_ret = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) * 1e-3

    # the timed region: exactly K steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk.mark(True)
    t0.record(st)
    for _ in range(args.steps):
        step()
    t1.record(st)
    clk.sample()  # one more reading while the queued steps still run
    torch.cuda.synchronize()
    clk.mark(False)
    clk.__exit__(None, None, None)
    elapsed = t0.elapsed_time(t1) * 1e-3
    if world > 1:
        from cross_model_attention_mf_b200 import replicas
        elapsed = replicas.max_over_ranks(elapsed, dev)  # the job takes as long as its slowest rank
        torch.distributed.barrier()
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"device status {rc} bits {bits:#x}")

    # end to end through the public API from pinned host buffers
    e2e = None
    if rank == 0 and not args.no_e2e:
        e2e = run_e2e(args, w, mf, pack, W, V, bsr, ws, O, qbase, dev)

    pcache = None
    if rank == 0 and not args.no_cache:
        pcache = run_prefix_cache(w, mf, bsr, nnz, dev)

    cqk = None
    if rank == 0 and not args.no_qk:
        cqk = run_compress_qk(w, mf, dev, qk_len=args.qk_len)

    multi = None
    if rank == 0 and not args.no_multi:
        multi = run_multi(w, mf, bsr, nnz, qbase, dev)

    calib = None
    if rank == 0 and not args.no_calib:
        calib = run_calib(w, mf, pack, dev, args.calib_len)

    cold = None
    if rank == 0 and not args.no_configs:
        hbm, tf_burst, _, _ = peaks()
        cold = run_cold_retrieve(w, mf, bsr, nnz, W, V, O, qbase, dev, hbm, tf_burst)

    return dict(w=w, nnz=nnz, elapsed=elapsed, t_comp=t_comp, t_ret=t_ret, clocks=clk.summary(),
                e2e=e2e, calib=calib, multi=multi, cqk=cqk, pcache=pcache, cold=cold)


def run_calib(w, mf, pack, dev, calib_len=0, reps=5):
    """Head-map calibration of the workload's receiver (h_r heads) on the sender layer: the Gram
    of the stacked maps over the causal positions (tcgen05 kernel), CUDA-event timed; the
    receiver maps are the recipe's maps of another layer.  Algorithmic bytes: every causal
    position of every sender and receiver head read once."""
    from synth import device as sdev
    if calib_len and calib_len < max(w.lens):  # a shorter calibration sequence (small captures)
        w = w.with_(lens=(calib_len,))
        pack = sdev.fill_maps(sdev.alloc_maps(w, dev), w, 0)
    wr = w.with_(h_s=w.h_r)
    rmaps = sdev.fill_maps(sdev.alloc_maps(wr, dev), wr, 1)
    offs = list(zip(pack.offsets, rmaps.offsets))
    F = w.h_s + w.h_r
    gram = torch.zeros((F, F), dtype=torch.float64, device=dev)
    wsb = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    path = mf.mf_calib_path(pack.maps, rmaps.maps, offs, w.lens, w.h_s, w.h_r, w.B)
    mf.mf_calib_gram(pack.maps, rmaps.maps, offs, w.lens, w.h_s, w.h_r, w.B, gram=gram, workspace=wsb)
    ts = []
    for _ in range(reps):
        gram.zero_()
        gpu_lead(torch.cuda.current_stream())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mf.mf_calib_gram(pack.maps, rmaps.maps, offs, w.lens, w.h_s, w.h_r, w.B, gram=gram, workspace=wsb)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e-3)
    Wm, res = mf.mf_calib_solve(gram, w.h_s, w.h_r, 0.0)
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"calibration status {rc} bits {bits:#x}")
    pos = sum(L * (L + 1) // 2 for L in w.lens)
    t = statistics.median(ts)
    del rmaps
    torch.cuda.empty_cache()
    return {"kernel": "mf_calib_gram (" + ("k_calib_gram_tc" if path == 1 else "k_calib_gram_simt") + ")",
            "workload": f"sender {w.h_s} heads, receiver {w.h_r} heads, lens={list(w.lens)}, B={w.B}",
            "ms": t * 1e3, "bytes": pos * F * 2, "GB/s": pos * F * 2 / t / 1e9,
            "TFLOP/s": 2.0 * F * F * pos / t / 1e12, "reps": reps,
            "fit_rel_residual": float(res.sum() / torch.diagonal(gram)[w.h_s:].sum())}


def run_multi(w, mf, bsr, nnz, qbase, dev, reps=20):
    """One sender layer's blocks serving three receivers (the workload's receiver and two more,
    the second with half the heads), once in shared launches (mf_map_retrieve_multi) and once
    receiver by receiver; CUDA events on the launching stream.  Algorithmic bytes of the shared
    launch: the kept blocks once, plus every receiver's V, O and W."""
    from synth import device as sdev
    specs = [(w.h_r, w.h_kv, w.seed), (w.h_r, w.h_kv, w.seed + 101), (w.h_r // 2, w.h_kv // 2, w.seed + 202)]
    rs = []
    for h_r, h_kv, seed in specs:
        wr = w.with_(h_r=h_r, h_kv=h_kv, seed=seed)
        rs.append(mf.Receiver([0], sdev.w_weights(wr, dev), sdev.v_contiguous(wr, 0, dev)[None], h_r, h_kv,
                              O=torch.empty((1, w.tokens, h_r, w.d), dtype=torch.bfloat16, device=dev)))
    cu = torch.tensor([0] + list(np.cumsum(w.lens)), dtype=torch.int32, device=dev)
    maxlen = max(w.lens)
    fused = mf.mf_retrieve_multi_fused([bsr], rs, cu, cu, qbase, maxlen)
    st = torch.cuda.current_stream()

    def shared():
        mf.mf_map_retrieve_multi([bsr], rs, cu, cu, qbase, maxlen)

    def separate():
        for r in rs:
            mf.mf_map_retrieve([bsr], [0], r.W, r.V, cu, cu, qbase, maxlen, r.h_r, r.h_kv, O=r.O)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            gpu_lead(st)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn()
            e1.record(st)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.median(ts)

    t_sh, t_sep = timed(shared), timed(separate)
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"multi-receiver status {rc} bits {bits:#x}")
    blk = w.h_s * w.B * w.B * 2
    per_r = sum(w.tokens * h_kv * w.d * 2 + w.tokens * h_r * w.d * 2 + 4 * h_r * w.h_s
                for h_r, h_kv, _ in specs)
    b_shared = nnz * blk + 4 * nnz + 4 * (sum(w.nqb) + 1) + per_r
    b_sep = len(specs) * (nnz * blk + 4 * nnz + 4 * (sum(w.nqb) + 1)) + per_r
    del rs
    torch.cuda.empty_cache()
    return {"kernel": "mf_map_retrieve_multi (k_retrieve_tc, " + ("one launch" if fused == 1 else "one launch per receiver") + ")",
            "workload": "one sender layer, receivers " + ", ".join(f"{a}/{b} heads" for a, b, _ in specs),
            "ms_shared": t_sh * 1e3, "ms_separate": t_sep * 1e3, "speedup": t_sep / t_sh,
            "bytes_shared": b_shared, "bytes_separate": b_sep,
            "GB/s": b_shared / t_sh / 1e9, "reps": reps}


MUFU_PER_SM_CLK = 16  # exp2 results per SM per clock (special-function units)


def run_compress_qk(w, mf, dev, reps=5, qk_len=0):
    """Compression from the sender's Q, K (no dense map) on the workload's sequence lengths,
    sender heads h_s over h_kv key heads, d = 128, tau of the workload; CUDA events around the
    whole call (stats, reduce, selection, gather).  Work: the Q.K^T products of every causal
    64-key tile (2 d flops per score) and one exponential per causal score; both passes of the
    kept blocks are counted separately."""
    from synth.qk import gen_qk
    if qk_len:
        w = w.with_(lens=(qk_len,))
    Q, K = gen_qk(w.lens, w.h_s, w.h_kv, 128, w.n_heavy, w.seed)
    Q, K = Q.to(dev), K.to(dev)
    cu = torch.tensor([0] + list(np.cumsum(w.lens)), dtype=torch.int32, device=dev)
    out = mf.alloc_bsr(sum(w.nqb), w.causal_blocks, w.h_s, w.B, torch.bfloat16, dev)
    need = mf.mf_compress_qk_workspace_size(len(w.lens), max(w.lens), w.tokens, w.h_s, w.h_kv,
                                            w.causal_blocks)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    for _ in range(2):
        mf.mf_compress_qk(Q, K, cu, max(w.lens), w.B, w.tau, out, workspace=ws)
    ts = []
    for _ in range(reps):
        gpu_lead(st)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        mf.mf_compress_qk(Q, K, cu, max(w.lens), w.B, w.tau, out, workspace=ws)
        e1.record(st)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e-3)
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"compress_qk status {rc} bits {bits:#x}")
    nnz = int(out.nnz.cpu()[0])
    t = statistics.median(ts)
    # causal 64-key tiles of the stats pass: per 128-row query tile qt, key blocks 0 .. 2qt+1
    tiles = 0
    for n in w.nqb:
        for qt in range(-(-n // 2)):
            tiles += min(2 * qt + 2, n)
    flops_stats = tiles * w.h_s * 2.0 * 128 * 64 * 128
    flops_gather = nnz * w.h_s * 2.0 * 64 * 64 * 128 * 2  # the 128-row tile covers two blocks
    scores = w.h_s * sum(L * (L + 1) // 2 for L in w.lens)
    del Q, K, ws, out
    torch.cuda.empty_cache()
    return {"kernel": "mf_compress_qk (k_qk stats + k_qk_reduce + selection + k_qk gather)",
            "workload": f"lens={list(w.lens)} h_s={w.h_s} h_kv={w.h_kv} d=128 B={w.B} tau={w.tau}",
            "ms": t * 1e3, "nnz": nnz, "density": nnz / w.causal_blocks, "reps": reps,
            "tokens_per_s_layer": w.tokens / t,
            "flops": flops_stats + flops_gather, "TFLOP/s": (flops_stats + flops_gather) / t / 1e12,
            "exp": scores + nnz * w.h_s * 64 * 64, "exp/s": (scores + nnz * w.h_s * 64 * 64) / t}


def run_prefix_cache(w, mf, bsr, nnz, dev, reps=20):
    """Prefix-hash block cache: every row of the compressed sender layer cached, then the whole
    request assembled from the cache on a side stream (CUDA events).  `ms` is the device work of
    one get (a captured graph replayed), `call_ms` the API call with its host-side planning.
    Bytes: the kept blocks read from the pool and written to the request's BSR.  Overlap: the assembly beside a bf16
    GEMM standing in for the receiver's own first-layer compute (8192 x 4096 x 4096) on the main
    stream; hidden = (t_gemm + t_get - t_both) / t_get."""
    blk = w.h_s * w.B * w.B * 2
    pool = torch.empty(max(nnz, 1) * blk, dtype=torch.uint8, device=dev)
    cache = mf.BlockCache(pool, w.h_s, w.B)
    toks = np.random.default_rng(w.seed).integers(0, 150000, size=w.tokens).astype(np.int32)
    h = mf.mf_prefix_hashes(toks, w.B)
    cache.put(0, bsr, h)
    out = mf.alloc_bsr(len(h), max(nnz, 1), w.h_s, w.B, torch.bfloat16, dev)
    main, side = torch.cuda.current_stream(), torch.cuda.Stream(device=dev)
    a = torch.randn(8192, 4096, device=dev, dtype=torch.bfloat16)
    b = torch.randn(4096, 4096, device=dev, dtype=torch.bfloat16)
    torch.cuda.synchronize()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(main)
            fn()
            e1.record(main)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.median(ts)

    def get():
        side.wait_stream(main)
        hit = cache.get(0, h, out, stream=side)
        assert hit == len(h)
        main.wait_stream(side)

    def gemm():
        torch.matmul(a, b)

    def both():
        side.wait_stream(main)
        cache.get(0, h, out, stream=side)
        torch.matmul(a, b)
        main.wait_stream(side)

    t_get, t_mm, t_both = timed(get), timed(gemm), timed(both)
    # the device work of one get alone: the call captured once into a CUDA graph (its copy list
    # is fixed at capture) and the graph replayed, so host-side planning is not in the time
    graph = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream(device=dev)
    cap_stream.wait_stream(main)
    with torch.cuda.graph(graph, stream=cap_stream):
        cache.get(0, h, out, stream=cap_stream)
    torch.cuda.synchronize()
    t_dev = timed(graph.replay)
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"prefix cache status {rc} bits {bits:#x}")
    ok = torch.equal(out.values[:nnz], bsr.values[:nnz])
    st = cache.stats()
    cache.close()
    del pool, out, a, b
    torch.cuda.empty_cache()
    moved = 2 * nnz * blk
    del graph
    return {"kernel": "mf_cache_get (k_cache_copy + k_cache_row_ptr)",
            "workload": f"{len(h)} query-block rows, {nnz} kept blocks ({nnz * blk / 1e6:.1f} MB)",
            "ms": t_dev * 1e3, "GB/s": moved / t_dev / 1e9, "bytes": moved,
            "call_ms": t_get * 1e3,
            "gemm_ms": t_mm * 1e3, "both_ms": t_both * 1e3,
            "hidden_frac": (t_mm + t_get - t_both) / t_get, "bitwise_equal": ok, "reps": reps,
            "cache": st}


CAUSAL_COPY_GROUP = 8  # query blocks per copied slab of the dense maps


def causal_slabs(w, pack, group=CAUSAL_COPY_GROUP):
    """The parts of the dense maps that compression reads, as 2-D copies: per sequence, head and
    group of `group` query blocks, the group's rows over the keys up to the group's last block
    (element offset, rows, row width in elements, row pitch in elements).  The upper triangle
    beyond each group is never read, so it never has to cross PCIe."""
    out = []
    for s, L in enumerate(w.lens):
        Lp = -(-L // w.B) * w.B
        nqb = -(-L // w.B)
        for h in range(w.h_s):
            for q0 in range(0, nqb, group):
                q1 = min(nqb, q0 + group)
                rows = min(L, q1 * w.B) - q0 * w.B
                out.append((pack.offsets[s] + h * Lp * Lp + q0 * w.B * Lp, rows, q1 * w.B, Lp))
    return out


def run_e2e(args, w, mf, pack, W, V, bsr, ws, O, qbase, dev):
    from cuda.bindings import runtime as cudart
    h_maps = torch.empty(pack.maps.shape, dtype=pack.maps.dtype, pin_memory=True)
    h_maps.copy_(pack.maps)
    esz = h_maps.element_size()
    slabs = causal_slabs(w, pack)
    kind = cudart.cudaMemcpyKind.cudaMemcpyHostToDevice
    h_V = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    h_V.copy_(V)
    h_W = torch.empty(W.shape, dtype=W.dtype, pin_memory=True)
    h_W.copy_(W)
    h_O = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    st = torch.cuda.current_stream()
    cu = pack.cu_seqlens
    maxlen = max(w.lens)
    n = max(1, min(args.steps, args.e2e_steps))

    def e2e_step():
        # the causal slabs of the dense maps, one pitched copy each, on the current stream
        sh = st.cuda_stream
        for off, rows, width, pitch in slabs:
            err, = cudart.cudaMemcpy2DAsync(pack.maps.data_ptr() + off * esz, pitch * esz,
                                            h_maps.data_ptr() + off * esz, pitch * esz,
                                            width * esz, rows, kind, sh)
            if err != cudart.cudaError_t.cudaSuccess:
                raise RuntimeError(f"cudaMemcpy2DAsync: {err}")
        V.copy_(h_V, non_blocking=True)
        W.copy_(h_W, non_blocking=True)
        mf.mf_compress(pack.maps, pack.map_seq_offset, cu, maxlen, w.h_s, w.B, w.tau, bsr, ws)
        mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qbase, maxlen, w.h_r, w.h_kv, O=O)
        h_O.copy_(O, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    for _ in range(n):
        e2e_step()
    t1.record(st)
    torch.cuda.synchronize()
    dt = t0.elapsed_time(t1) * 1e-3 / n
    h2d = (sum(rows * width for _, rows, width, _ in slabs) * esz + h_V.numel() * h_V.element_size()
           + h_W.numel() * 4)
    d2h = h_O.numel() * h_O.element_size()
    return {"value": w.tokens / dt, "unit": "tokens/s/layer", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n,
            "h2d": f"the dense maps' causal slabs ({len(slabs)} pitched copies of {CAUSAL_COPY_GROUP} "
                   f"query blocks' rows over the keys up to their last block), V and W"}


# ------------------------------------------------------------------------ the other workloads
L2_FLUSH_BYTES = 256 << 20  # written between timed repetitions: twice the 126 MB L2


LEAD_CYCLES = 2_000_000  # ~1 ms of GPU spin at 1965 MHz


def gpu_lead(st):
    """Keep the GPU busy (a spin kernel of ~1 ms) on stream st while the host prepares the next
    timed call, so that the start event fires when that call's kernels are already queued: no
    host time (descriptor building, argument marshalling) falls inside the timed interval."""
    with torch.cuda.stream(st):
        torch.cuda._sleep(LEAD_CYCLES)


def _timed(fn, st, reps, warm=3, flush=None):
    """Median device time of fn over reps repetitions (CUDA events on stream st), after warm
    untimed runs; when flush is given it is overwritten before every repetition, outside the
    timed interval, so no input is still in L2."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        gpu_lead(st)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        fn()
        e1.record(st)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e-3)
    return statistics.median(ts)


def retrieve_algorithmic(w, nnz, rows, T_q, T_k, layers=1):
    """Algorithmic bytes / FLOPs of retrieval over `rows` query blocks holding nnz kept blocks
    (all layers together): kept blocks, V of T_k keys, O of T_q queries and the indices, once;
    mixing and P.V products of every kept block."""
    e = 4 if w.dtype == "f32" else 2
    blk = w.h_s * w.B * w.B * e
    b = (nnz * blk + layers * (T_k * w.h_kv * w.d * e + T_q * w.h_r * w.d * e + 4 * (rows + 1)
                                + 4 * w.h_r * w.h_s) + 4 * nnz)
    f = nnz * (2 * w.h_r * w.h_s * w.B * w.B + 2 * w.h_r * w.B * w.B * w.d)
    return b, f


def _ret_line(w, t, b, f, hbm, tf, tokens, layers=1):
    t_roof = max(b / (hbm * 1e9), f / (tf * 1e12))
    return {"ms": t * 1e3, "GB/s": b / t / 1e9, "TFLOP/s": f / t / 1e12, "bytes": b, "flops": f,
            "tokens_per_s_layer": tokens * layers / t, "roofline_frac": t_roof / t,
            "bound": "hbm" if b / (hbm * 1e9) >= f / (tf * 1e12) else "tensor"}


def _comp_line(w, t, nnz, hbm, causal=None, rows=None):
    e = 4 if w.dtype == "f32" else 2
    blk = w.h_s * w.B * w.B * e
    causal = w.causal_blocks if causal is None else causal
    rows = sum(w.nqb) if rows is None else rows
    b = causal * blk + nnz * blk + 4 * nnz + 4 * (rows + 1)
    return {"ms": t * 1e3, "GB/s": b / t / 1e9, "bytes": b, "roofline_frac": b / (hbm * 1e9) / t,
            "tokens_per_s_layer": w.tokens / t}


def run_long_context(mf, dev, hbm, tf, points, reps=3, oracle_rows=0):
    """Long-context workload (L = 32768, B = 128, 32 -> 24 / 8 heads) at the given
    (tau, heavy columns, map reading) points: compression of the 68.7 GB dense layer (larger
    than L2 by itself) and retrieval of the compressed layer (L2 flushed before each
    repetition)."""
    from synth import device as sdev
    base = synth_all()["long_context"]
    st = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out, pack, key = [], None, None
    for tau, heavy, reading in points:
        w = base.with_(tau=tau, n_heavy=heavy, reading=reading)
        if key != (heavy, reading):
            pack = None
            torch.cuda.empty_cache()
            pack = sdev.fill_maps(sdev.alloc_maps(w, dev), w, 0)
            key = (heavy, reading)
        cap = w.causal_blocks
        bsr = mf.alloc_bsr(sum(w.nqb), cap, w.h_s, w.B, pack.maps.dtype, dev)
        ws = torch.empty(mf.mf_compress_workspace_size(1, w.lens[0], w.B, cap), dtype=torch.uint8,
                         device=dev)
        cu = pack.cu_seqlens
        t_c = _timed(lambda: mf.mf_compress(pack.maps, pack.map_seq_offset, cu, w.lens[0], w.h_s,
                                            w.B, w.tau, bsr, ws), st, reps, warm=1)
        nnz = int(bsr.nnz.cpu()[0])
        W, V = sdev.w_weights(w, dev), sdev.v_contiguous(w, 0, dev)
        O = torch.empty((1, w.tokens, w.h_r, w.d), dtype=V.dtype, device=dev)
        qb = sdev.qblock_base(w, dev)
        t_r = _timed(lambda: mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qb, w.lens[0], w.h_r,
                                                w.h_kv, O=O), st, reps, warm=1, flush=flush)
        _status_or_raise(mf, "long_context")
        b, f = retrieve_algorithmic(w, nnz, sum(w.nqb), w.tokens, w.tokens)
        out.append({"tau": tau, "heavy": heavy, "reading": reading, "nnz": nnz,
                    "density": nnz / w.causal_blocks,
                    "compress": _comp_line(w, t_c, nnz, hbm),
                    "retrieve": _ret_line(w, t_r, b, f, hbm, tf, w.tokens)})
        if oracle_rows > 0 and len(out) == 1:  # the oracle beside the first point
            out[0]["oracle_cpu"] = oracle_config_sample(w, pack, W[0].cpu().numpy(),
                                                        V[:w.lens[0]].cpu(), oracle_rows)
        del bsr, ws, W, V, O
    del pack, flush
    torch.cuda.empty_cache()
    return {"workload": "long_context: L=32768, B=128, h_s=32 -> h_r=24, h_kv=8, d=128, bf16",
            "points": out, "reps": reps, "l2": "retrieval: L2 flushed before every repetition"}


def run_qwen(mf, dev, hbm, tf, reps=3, oracle_rows=0):
    """Qwen-like pair: 40 sender layers compressed one by one (each layer's dense maps, 6 GB,
    generated into one reused buffer; compression timed per layer), then the 36 receiver layers
    retrieved (layer map l_s = round(l_r 39 / 35)): each layer alone, all 36 in one call, and
    the 36 per-layer launches captured once in a CUDA graph and replayed."""
    from synth import device as sdev
    w = synth_all()["qwen_pair"]
    lm = w.layer_map()
    st = torch.cuda.current_stream()
    pack = sdev.alloc_maps(w, dev)
    cap = 2048
    ws = torch.empty(mf.mf_compress_workspace_size(len(w.lens), max(w.lens), w.B, cap),
                     dtype=torch.uint8, device=dev)
    bsrs, t_comp, nnzs = [], [], []
    cu = pack.cu_seqlens
    for l in range(w.n_sender_layers):
        sdev.fill_maps(pack, w, l)
        b = mf.alloc_bsr(sum(w.nqb), cap, w.h_s, w.B, pack.maps.dtype, dev)
        t_comp.append(_timed(lambda: mf.mf_compress(pack.maps, pack.map_seq_offset, cu, max(w.lens),
                                                    w.h_s, w.B, w.tau, b, ws), st, 2, warm=1))
        bsrs.append(b)
        nnzs.append(int(b.nnz.cpu()[0]))
        if l == 0 and oracle_rows > 0:  # receiver layer 0 reads sender layer 0
            ocpu = oracle_config_sample(w, pack, sdev.w_weights(w, dev)[0].cpu().numpy(),
                                        sdev.v_contiguous(w, 0, dev)[:w.lens[0]].cpu(), oracle_rows)
    _status_or_raise(mf, "qwen compress")
    del pack
    torch.cuda.empty_cache()
    W = sdev.w_weights(w, dev)
    T = w.tokens
    V = torch.empty((w.n_receiver_layers, T, w.h_kv, w.d), dtype=torch.bfloat16, device=dev)
    for l in range(w.n_receiver_layers):
        V[l] = sdev.v_contiguous(w, l, dev)
    O = torch.empty((w.n_receiver_layers, T, w.h_r, w.d), dtype=torch.bfloat16, device=dev)
    qb = sdev.qblock_base(w, dev)
    maxlen = max(w.lens)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def layer(l):
        mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qb, maxlen, w.h_r, w.h_kv, O=O[l:l + 1],
                           l_r_range=(l, l + 1), v_layer_stride=V[0].numel())

    def all_layers():
        mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qb, maxlen, w.h_r, w.h_kv, O=O,
                           v_layer_stride=V[0].numel())

    t_layer = [_timed(lambda: layer(l), st, reps, warm=1, flush=flush) for l in range(w.n_receiver_layers)]
    t_all = _timed(all_layers, st, reps, warm=1, flush=flush)
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(device=dev)
    cs.wait_stream(st)
    with torch.cuda.graph(g, stream=cs):
        for l in range(w.n_receiver_layers):
            mf.mf_map_retrieve(bsrs, lm, W, V, cu, cu, qb, maxlen, w.h_r, w.h_kv, O=O[l:l + 1],
                               l_r_range=(l, l + 1), v_layer_stride=V[0].numel(), stream=cs)
    torch.cuda.synchronize()
    t_graph = _timed(g.replay, st, reps, warm=1, flush=flush)
    _status_or_raise(mf, "qwen retrieve")
    nnz_r = [nnzs[lm[l]] for l in range(w.n_receiver_layers)]
    rows = sum(w.nqb)
    per = [_ret_line(w, t, *retrieve_algorithmic(w, n, rows, T, T), hbm, tf, T)
           for t, n in zip(t_layer, nnz_r)]
    b_all, f_all = retrieve_algorithmic(w, sum(nnz_r), rows, T, T, layers=w.n_receiver_layers)
    comp = [_comp_line(w, t, n, hbm) for t, n in zip(t_comp, nnzs)]
    del g, bsrs, V, O, flush
    torch.cuda.empty_cache()

    def summary(lines, key):
        v = sorted(x[key] for x in lines)
        return {"median": v[len(v) // 2], "min": v[0], "max": v[-1]}

    return {"workload": "qwen_pair: 40 sender layers h_s=40 -> 36 receiver layers h_r=32, h_kv=8, "
                        "d=128, varlen 2048/4096/6144/4096, B=64, tau=0.95, bf16",
            "density_per_sender_layer": summary([{"d": n / w.causal_blocks} for n in nnzs], "d"),
            "compress_per_sender_layer": {k: summary(comp, k) for k in ("ms", "GB/s", "roofline_frac")},
            "retrieve_per_receiver_layer": {k: summary(per, k) for k in
                                            ("ms", "GB/s", "TFLOP/s", "tokens_per_s_layer", "roofline_frac")},
            "retrieve_36_layers_one_call": _ret_line(w, t_all, b_all, f_all, hbm, tf, T,
                                                     layers=w.n_receiver_layers),
            "retrieve_36_layers_graph": _ret_line(w, t_graph, b_all, f_all, hbm, tf, T,
                                                  layers=w.n_receiver_layers),
            **({"oracle_cpu": ocpu} if oracle_rows > 0 else {}),
            "reps": reps, "l2": "retrieval: L2 flushed before every repetition"}


def run_routing(mf, dev, hbm, tf, reps=3, oracle_rows=0):
    """Multi-turn routing batch: 16 varlen sequences (1k-8k tokens) compressed in one call, then
    retrieved by chunked prefill (2048-token query chunks against the whole prefix) over a paged
    V (16-token pages, shuffled block table): every chunk step timed, and the sum."""
    from synth import device as sdev
    w = synth_all()["routing_batch"]
    st = torch.cuda.current_stream()
    pack = sdev.fill_maps(sdev.alloc_maps(w, dev), w, 0)
    cap = 8192
    bsr = mf.alloc_bsr(sum(w.nqb), cap, w.h_s, w.B, pack.maps.dtype, dev)
    ws = torch.empty(mf.mf_compress_workspace_size(len(w.lens), max(w.lens), w.B, cap),
                     dtype=torch.uint8, device=dev)
    cu = pack.cu_seqlens
    t_c = _timed(lambda: mf.mf_compress(pack.maps, pack.map_seq_offset, cu, max(w.lens), w.h_s,
                                        w.B, w.tau, bsr, ws), st, reps, warm=1)
    nnz = int(bsr.nnz.cpu()[0])
    rp = bsr.row_ptr.cpu().numpy()
    ocpu = None
    if oracle_rows > 0:
        ocpu = oracle_config_sample(w, pack, sdev.w_weights(w, dev)[0].cpu().numpy(),
                                    sdev.v_contiguous(w, 0, dev)[:w.lens[0]].cpu(), oracle_rows)
    del pack
    torch.cuda.empty_cache()
    W = sdev.w_weights(w, dev)
    V = sdev.v_contiguous(w, 0, dev)
    Vp, table = sdev.v_paged(w, V)
    del V
    qb = sdev.qblock_base(w, dev)
    qbase = np.concatenate([[0], np.cumsum(w.nqb)[:-1]])
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    steps = []
    for step in synth_chunks(w):
        cu_q, cu_k, mq = sdev.step_tensors(step, dev)
        Tq = int(cu_q[-1])
        O = torch.empty((1, Tq, w.h_r, w.d), dtype=torch.bfloat16, device=dev)
        t = _timed(lambda: mf.mf_map_retrieve([bsr], [0], W, Vp, cu_q, cu_k, qb, mq, w.h_r, w.h_kv,
                                              O=O, paged=(table, w.page_size)), st, reps, warm=1,
                   flush=flush)
        rows = n_step = 0
        for s, (q_len, k_len) in enumerate(step):
            if q_len == 0:
                continue
            q0 = k_len - q_len
            r0, r1 = int(qbase[s]) + q0 // w.B, int(qbase[s]) + -(-k_len // w.B)
            rows += r1 - r0
            n_step += int(rp[r1] - rp[r0])
        b, f = retrieve_algorithmic(w, n_step, rows, Tq, sum(k for _, k in step))
        line = _ret_line(w, t, b, f, hbm, tf, Tq)
        line.update({"queries": Tq, "nnz": n_step})
        steps.append(line)
    _status_or_raise(mf, "routing")
    t_tot = sum(x["ms"] for x in steps) * 1e-3
    b_tot = sum(x["bytes"] for x in steps)
    f_tot = sum(x["flops"] for x in steps)
    del bsr, Vp, flush
    torch.cuda.empty_cache()
    return {"workload": "routing_batch: 16 sequences 1k-8k tokens, chunk 2048, paged V (16-token "
                        "pages, shuffled), h_s=32 -> h_r=32, h_kv=8, d=128, B=64, tau=0.95, bf16",
            "nnz": nnz, "density": nnz / w.causal_blocks,
            "compress": _comp_line(w, t_c, nnz, hbm),
            "retrieve_per_chunk_step": steps,
            "retrieve_all_steps": _ret_line(w, t_tot, b_tot, f_tot, hbm, tf, w.tokens),
            **({"oracle_cpu": ocpu} if ocpu is not None else {}),
            "reps": reps, "l2": "retrieval: L2 flushed before every repetition"}


def run_cold_retrieve(w, mf, bsr, nnz, W, V, O, qb, dev, hbm, tf, reps=20):
    """Retrieval of the main workload with L2 flushed (a 256 MB write) before every repetition:
    in the timed step the kept blocks were written by the compression just before and partly sit
    in L2."""
    st = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    cu = torch.tensor([0] + list(np.cumsum(w.lens)), dtype=torch.int32, device=dev)
    t = _timed(lambda: mf.mf_map_retrieve([bsr], [0], W, V, cu, cu, qb, max(w.lens), w.h_r, w.h_kv,
                                          O=O), st, reps, flush=flush)
    del flush
    torch.cuda.empty_cache()
    b, f = retrieve_algorithmic(w, nnz, sum(w.nqb), w.tokens, w.tokens)
    line = _ret_line(w, t, b, f, hbm, tf, w.tokens)
    line["l2"] = "flushed before every repetition"
    return line


def _status_or_raise(mf, what):
    rc, bits = mf.mf_get_status()
    if rc != mf.MF_OK:
        raise RuntimeError(f"{what}: device status {rc} bits {bits:#x}")


def _json_default(o):
    """numpy scalars (and anything else with .item()) as plain numbers"""
    if hasattr(o, "item"):
        return o.item()
    raise TypeError(f"not JSON serialisable: {type(o).__name__}")


def mf_mod():
    import cross_model_attention_mf_b200 as mf
    return mf


def synth_all():
    import synth
    return synth.ALL


def synth_chunks(w):
    import synth
    return synth.chunks(w)


# ------------------------------------------------------------------------ oracle (CPU baseline)
def _oracle_row(w, qb, slab, W_l, V_host):
    """Oracle compression + retrieval of one query block (whole rows of sequence 0); True when
    the row is a near tie (its cumulative-mass boundary within 1e-5 of tau)."""
    import oracle
    m = oracle.row_masses(slab, w.lens[0], w.B, qb)
    kept, info = oracle.select(m, qb, w.tau)
    vals = np.stack([oracle.gather_block(slab, w.lens[0], w.B, qb, int(kb)) for kb in kept])
    lo, hi = 0, min(w.lens[0], (qb + 1) * w.B) - qb * w.B
    oracle.retrieve_block(vals, kept, qb, w.B, W_l, V_host, w.h_kv, (lo, hi))
    return bool(oracle.is_boundary(info, w.tau))


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(w, slabs, W_l, V_host, rows, threads, ties=None):
    """Wall time of the oracle on the sampled query blocks, one block per task on `threads`
    host threads (the C oracle runs with the GIL released); `ties`, a list, receives the number
    of near-tie rows among them."""
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as pool:
        near = list(pool.map(lambda a: _oracle_row(w, a[0], a[1], W_l, V_host), zip(rows, slabs)))
    dt = time.perf_counter() - t0
    if ties is not None:
        ties.append(sum(near))
    return dt


def cpu_sample_inputs(w, n_rows, dev):
    """Host copies of n_rows query-block rows spread over the sequence (first sequence)."""
    from synth import device as sdev
    pack = sdev.fill_maps(sdev.alloc_maps(w, dev), w, 0)
    W = sdev.w_weights(w, dev)
    V = sdev.v_contiguous(w, 0, dev)
    nqb = w.nqb[0]
    rows = sorted(set(np.linspace(0, nqb - 1, n_rows).astype(int).tolist()))
    view = pack.seq_view(0, w.h_s, w.B)
    slabs = [view[:, qb * w.B:(qb + 1) * w.B, :(qb + 1) * w.B].cpu() for qb in rows]
    out = (rows, slabs, W[0].cpu().numpy(), V[:w.lens[0]].cpu())
    del pack
    torch.cuda.empty_cache()
    return out


def cpu_baseline(w, dev, n_rows):
    rows, slabs, W_l, V_host = cpu_sample_inputs(w, n_rows, dev)
    cores = host_cores()
    ties = []
    dt = oracle_sample(w, slabs, W_l, V_host, rows, cores, ties)
    toks = sum(min(w.lens[0], (qb + 1) * w.B) - qb * w.B for qb in rows)
    return {"value": toks / dt, "unit": "tokens/s/layer", "cores": cores, "kind": "oracle",
            "near_tie_rows": ties[0],
            "sample": f"{len(rows)} of {w.nqb[0]} query blocks ({toks} tokens) of sequence 0, "
                      f"compress + retrieve, float64 C oracle on {cores} host threads (one query "
                      f"block per task), {dt:.2f} s wall"}


def oracle_config_sample(w, pack, W_l, V_host, n_rows):
    """The oracle (compress + retrieve) on n_rows query blocks of a config's first sequence,
    spread over it, on all host cores: the CPU figure beside that config's GPU figures.  pack
    holds the config's dense maps on the device; V_host is the first sequence's V rows."""
    nqb = w.nqb[0]
    rows = sorted(set(np.linspace(0, nqb - 1, n_rows).astype(int).tolist()))
    view = pack.seq_view(0, w.h_s, w.B)
    slabs = [view[:, qb * w.B:(qb + 1) * w.B, :(qb + 1) * w.B].cpu() for qb in rows]
    cores = host_cores()
    ties = []
    dt = oracle_sample(w, slabs, W_l, V_host, rows, cores, ties)
    toks = sum(min(w.lens[0], (qb + 1) * w.B) - qb * w.B for qb in rows)
    return {"value": toks / dt, "unit": "tokens/s/layer", "cores": cores, "kind": "oracle",
            "seconds": dt, "near_tie_rows": ties[0], "sample": f"{len(rows)} of {nqb} query blocks ({toks} tokens) of the "
                                    f"first sequence (length {w.lens[0]}), compress + retrieve, "
                                    f"float64 C oracle on {cores} host threads"}


# ------------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="ministral_pair")
    ap.add_argument("--reading", type=int, default=1)
    ap.add_argument("--config-oracle-rows", type=int, default=16,
                    help="query blocks of each config's first sequence that the oracle is timed on "
                         "(0: none)")
    ap.add_argument("--cpu-rows", type=int, default=128,
                    help="query blocks of sequence 0 the CPU oracle runs (default: all of them for the Ministral-like pair)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-cache", action="store_true", help="skip the prefix-cache line")
    ap.add_argument("--no-qk", action="store_true", help="skip the compression-from-Q,K line")
    ap.add_argument("--qk-len", type=int, default=0,
                    help="sequence length of the compression-from-Q,K line (0: the workload's)")
    ap.add_argument("--qk-only", action="store_true",
                    help="print only the compression-from-Q,K measurement (profiling runs)")
    ap.add_argument("--no-multi", action="store_true", help="skip the several-receivers line")
    ap.add_argument("--no-calib", action="store_true", help="skip the head-map calibration line")
    ap.add_argument("--calib-len", type=int, default=0,
                    help="calibrate on a sequence of this many tokens (0: the workload's own)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (long context, Qwen-like, routing batch, cold L2)")
    ap.add_argument("--long-points", default="0.95:8:1,0.8:8:3,0.99:64:3",
                    help="long-context points tau:heavy:reading, comma separated")
    ap.add_argument("--capacity", type=int, default=0,
                    help="BSR capacity in blocks (0: every causal block, which never overflows)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = workload(args.workload, args.reading)

    if args.impl == "reference":
        if rank != 0:
            return
        # each step: the oracle on one batch of query blocks (one per host thread, cycling over
        # blocks spread along the sequence); the run stops early after ~60 s of wall time
        cores = host_cores()
        rows, slabs, W_l, V_host = cpu_sample_inputs(w, max(8, cores), dev)

        def one(t):
            idx = [(t * cores + k) % len(rows) for k in range(cores)]
            dt = oracle_sample(w, [slabs[i] for i in idx], W_l, V_host, [rows[i] for i in idx], cores)
            return dt, sum(min(w.lens[0], (rows[i] + 1) * w.B) - rows[i] * w.B for i in idx)

        # the requested warm-up steps (bounded by ~20 s of wall time)
        warm, t_warm = 0, time.time()
        while warm < args.warmup and time.time() - t_warm < 20.0:
            one(warm)
            warm += 1
        spent, k, toks = 0.0, 0, 0
        while k < max(args.steps, 1) and (spent < 60.0 or k == 0):
            dt, n = one(warm + k)
            spent += dt
            toks += n
            k += 1
        v = toks / spent
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s/layer",
                "n_gpus": args.gpus, "steps": k, "warmup": warm, "ms_per_step": spent / k * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": describe(w)},
                "cpu_baseline": {"value": v, "unit": "tokens/s/layer", "cores": cores, "kind": "oracle",
                                 "sample": f"{k} steps of {cores} query blocks each ({toks} tokens), "
                                           f"compress + retrieve, float64 C oracle on {cores} host threads"},
                "e2e": {"value": v, "unit": "tokens/s/layer", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    if args.qk_only:
        import cross_model_attention_mf_b200 as mf
        print(json.dumps({"compress_qk": run_compress_qk(w, mf, dev, qk_len=args.qk_len)}), flush=True)
        return
    res = run_ours(args, rank, world, dev)
    if rank == 0:
        hbm, tf_burst, tf_sus, src = peaks()
        w = res["w"]
        nnz = res["nnz"]
        comp_b, ret_b, ret_f = algorithmic(w, nnz)
        step_t = res["elapsed"] / args.steps
        value = world * w.tokens / step_t
        comp_gbs = comp_b / res["t_comp"] / 1e9
        ret_gbs = ret_b / res["t_ret"] / 1e9
        ret_tf = ret_f / res["t_ret"] / 1e12
        ret_roof_t = max(ret_b / (hbm * 1e9), ret_f / (tf_burst * 1e12))
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s/layer", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": describe(w), "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (dense maps of 4.3 GB stream through every step)",
                       "step": "mf_compress (sender layer) + mf_map_retrieve (receiver layer)"},
            "density": nnz / w.causal_blocks, "nnz": nnz,
            "compress": {"ms": res["t_comp"] * 1e3, "GB/s": comp_gbs, "bytes": comp_b,
                         "frac_hbm": comp_gbs / hbm},
            "retrieve": {"ms": res["t_ret"] * 1e3, "GB/s": ret_gbs, "TFLOP/s": ret_tf,
                         "bytes": ret_b, "flops": ret_f,
                         "tokens_per_s_layer": w.tokens / res["t_ret"],
                         "roofline_frac": ret_roof_t / res["t_ret"],
                         "bound": "hbm" if ret_b / (hbm * 1e9) >= ret_f / (tf_burst * 1e12) else "tensor"},
            "roofline": {"bound": "hbm", "kernel": "mf_compress (block stats + select + gather)",
                         "achieved": comp_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": comp_gbs / hbm,
                         "traffic": measured_traffic("mf_compress", w.name),
                         "peak_source": f"{src}, hbm_gbs"},
            "roofline_retrieve": {
                "bound": "hbm", "kernel": "mf_map_retrieve (k_retrieve_tc)",
                "achieved": ret_gbs, "peak": hbm, "unit": "GB/s",
                "frac": ret_roof_t / res["t_ret"],
                "tensor_TFLOP/s": ret_tf, "tensor_peak": tf_burst,
                "traffic": measured_traffic("mf_map_retrieve", w.name),
                "peak_source": f"{src}, hbm_gbs; bf16_tflops burst for the tensor side"},
            # per step: k_stats, k_select, k_gather and k_retrieve_tc, plus k_meta where the
            # compression's geometry pass runs on its own (more than 64 sequences or B = 128)
            "gpu_launches": (4 + (0 if len(w.lens) <= 64 and w.B <= 64 else 1)) * args.steps,
            "clocks": res["clocks"],
        }
        if res["e2e"] is not None:
            line["e2e"] = res["e2e"]
        if res["pcache"] is not None:
            c = res["pcache"]
            c.update({"bound": "hbm", "peak": hbm, "unit": "GB/s", "frac": c["GB/s"] / hbm,
                      "peak_source": f"{src}, hbm_gbs"})
            line["prefix_cache"] = c
        if res["cqk"] is not None:
            c = res["cqk"]
            sm_mhz = (res["clocks"] or {}).get("sm_mhz") or 1965.0
            mufu = MUFU_PER_SM_CLK * torch.cuda.get_device_properties(0).multi_processor_count * sm_mhz * 1e6
            c.update({"bound": "alu", "unit": "exp/s", "achieved": c["exp/s"], "peak": mufu,
                      "frac": c["exp/s"] / mufu,
                      "peak_source": f"{MUFU_PER_SM_CLK} exp2 per SM per clock x SMs x median SM clock",
                      "tensor_frac": c["TFLOP/s"] / tf_burst,
                      "tensor_peak_source": f"{src}, bf16_tflops burst"})
            line["compress_qk"] = c
        if res["multi"] is not None:
            m = res["multi"]
            m.update({"bound": "hbm", "peak": hbm, "unit": "GB/s", "frac": m["GB/s"] / hbm,
                      "peak_source": f"{src}, hbm_gbs"})
            line["multi_receiver"] = m
        if res["calib"] is not None:
            c = res["calib"]
            c.update({"bound": "hbm", "peak": hbm, "unit": "GB/s", "frac": c["GB/s"] / hbm,
                      "peak_source": f"{src}, hbm_gbs"})
            line["calibration"] = c
        if res["cold"] is not None:
            line["retrieve_cold_l2"] = res["cold"]
        if not args.no_configs:
            pts = [tuple(float(x) if i == 0 else int(x) for i, x in enumerate(p.split(":")))
                   for p in args.long_points.split(",") if p]
            line["configs"] = {}
            orows = 0 if (args.no_cpu or world > 1) else args.config_oracle_rows
            for name, fn in (("qwen_pair", lambda: run_qwen(mf_mod(), dev, hbm, tf_burst, oracle_rows=orows)),
                             ("long_context", lambda: run_long_context(mf_mod(), dev, hbm, tf_burst, pts,
                                                                       oracle_rows=orows)),
                             ("routing_batch", lambda: run_routing(mf_mod(), dev, hbm, tf_burst,
                                                                   oracle_rows=orows))):
                line["configs"][name] = fn()
                # each workload's figures also go to stderr as soon as they exist
                print(json.dumps({name: line["configs"][name]}, default=_json_default), file=sys.stderr,
                      flush=True)
        if not args.no_cpu and world == 1:
            line["cpu_baseline"] = cpu_baseline(w, dev, args.cpu_rows)
        print(json.dumps(line, default=_json_default), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
