"""Benchmark of the DSA layer step (indexer -> top-k -> sparse MLA attention).

Default workload: decode at 128K context -- 32 sequences, one query each,
ctx_len 131072, index_topk 2048, 64 index heads x 128, 128 attention heads
over a 576-wide latent (value = first 512).  A step is one pass of the whole
path over one batch of synthetic inputs already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload decode128k|decode128k_fp8|decode32k|prefill8k]

Under torchrun (N > 1) every rank runs its own replica of the workload
(decode shards by sequence, no collective): weak scaling, value = queries
of all ranks / max-over-ranks time.  ``--impl reference`` times the CPU
oracle (the only reference that exists for this path) on rank 0.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def _peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix=f"dsa_clocks_rank{self.index}_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        with open(self.path) as f:
            lines = f.read().splitlines()
        os.unlink(self.path)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": smax, "samples": len(sm), "reasons": sorted(reasons)}


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks of the default process group (a
    timing aggregation; every rank calls it at the same point)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _metric_name(wl):
    if wl.n_q == 1:
        return "DSA layer queries/s at 128K ctx" if wl.s_max == 131072 else f"DSA layer queries/s ({wl.name})"
    return f"DSA layer prefill tokens/s ({wl.name})"


def _workload_desc(wl):
    return (f"{wl.name}: B={wl.batch}, n_q={wl.n_q}, ctx={wl.s_max}, index_topk={wl.topk}, "
            f"H_I={wl.idx_heads}x{wl.idx_dim} ({'e4m3' if wl.idx_fp8 else wl.dtype}), "
            f"H={wl.heads}, d_qk={wl.d_qk}, d_v={wl.d_v}")


def _queries(wl):
    return wl.batch * wl.n_q


def _indexer_bytes(wl):
    """Algorithmic HBM bytes of one indexer launch: every causal key row of the
    index-key cache read once per query block (decode: once per query), plus
    the query block, the head weights and the fp32 score row written."""
    row = wl.idx_dim * (1 if wl.idx_fp8 else 2) + (4 if wl.idx_fp8 else 0)
    if wl.n_q == 1:
        keys = sum(wl.lengths())
        return keys * row + wl.batch * (wl.idx_heads * wl.idx_dim * 2 + wl.idx_heads * 4) + keys * 4
    pairs = sum(wl.n_q * (wl.n_q + 1) // 2 for _ in range(wl.batch))
    return pairs * 4 + wl.batch * wl.s_max * row


def _indexer_flops(wl):
    if wl.n_q == 1:
        pairs = sum(wl.lengths())
    else:
        pairs = wl.batch * wl.n_q * (wl.n_q + 1) // 2
    return 2.0 * wl.idx_heads * wl.idx_dim * pairs


def _attn_extra_launches(wl, dsa, shape):
    """The split combine is a second attention launch when the split plan needs scratch."""
    return 1 if dsa.workspace_bytes(shape, dsa.WS_ATTN) > 0 else 0


# DRAM bytes per indexer launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum),
# keyed by workload and by the SHA-256 of the indexer source the counters were taken on;
# a changed kernel reports null.  Filled in from profiles/indexer_tc_decode128k.md.
TRAFFIC = {
    # B=8 capture (268,660,736 read + 4,674,816 written) scaled by 4 to B=32: traffic grows with the key tiles
    "decode128k": ("3092c7447fe712d5", 4 * (268660736 + 4674816)),
}


def _traffic(wl):
    import hashlib
    path = os.path.join(ROOT, "long_context_indexing_lightning_b200", "csrc", "indexer_tc.cu")
    try:
        sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    rec = TRAFFIC.get(wl.name)
    return rec[1] if rec and rec[0] == sha else None


def run_ours(args, wl):
    import long_context_indexing_lightning_b200 as dsa

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    t = workloads.make_inputs(wl, dev, seed=rank)
    shape = dsa.shape_from_workload(wl)
    stream = torch.cuda.current_stream(dev)
    ld = (wl.s_max + 3) // 4 * 4
    out = torch.empty(wl.batch, wl.n_q, wl.heads, wl.d_v, dtype=t["q"].dtype, device=dev)
    k_idx, k_scale, q_idx, q_scale = t["k_idx"], None, t["q_idx"], None
    q8 = qs = None
    k_ref = None
    if wl.idx_fp8:
        k_idx, k_scale = dsa.hadamard_quant_fp8(t["k_idx"])   # the cache as stored (quantise-on-write)
        q8 = torch.empty(q_idx.shape, dtype=torch.uint8, device=dev)
        qs = torch.empty(q_idx.shape[:-1], dtype=torch.float32, device=dev)
        if wl.idx_rescore > 0:
            k_ref = t["k_idx"]       # the bf16 key cache kept beside the FP8 one for re-scoring
        else:
            del t["k_idx"]

    # prefill runs in rounds of `chunk` queries (positions shifted by the
    # round's first query); decode is a single round
    chunk = wl.n_q if wl.n_q <= args.q_chunk else args.q_chunk
    rounds = []
    for t0 in range(0, wl.n_q, chunk):
        c = min(chunk, wl.n_q - t0)
        sh = shape.replace(n_q=c)
        rounds.append((t0, c, sh, (t["q_pos0"] + t0).contiguous()))
    if len(rounds) > 1 and wl.batch != 1:
        raise SystemExit("prefill rounds are cut per sequence: use batch 1")
    scores = torch.empty(wl.batch, chunk, ld, dtype=torch.float32, device=dev)
    idx = torch.empty(wl.batch, chunk, wl.topk, dtype=torch.int32, device=dev)
    kc = wl.topk + wl.idx_rescore if (wl.idx_fp8 and wl.idx_rescore > 0) else 0
    if kc:
        # e4m3 indexer with re-scoring: the FP8 top-(k + margin) candidates, their bf16 scores
        cand = torch.empty(wl.batch, chunk, kc, dtype=torch.int32, device=dev)
        cand_sc = torch.empty(wl.batch, chunk, kc, dtype=torch.float32, device=dev)
    ws_topk = torch.empty(max(1, dsa.workspace_bytes(rounds[0][2], dsa.WS_TOPK)), dtype=torch.uint8, device=dev)
    # the indexer -> top-k handoff (first-digit histograms from the indexer epilogue at decode)
    hist = torch.empty(dsa.workspace_bytes(shape, dsa.WS_HIST), dtype=torch.uint8, device=dev)
    ws_attn = torch.empty(max(1, dsa.workspace_bytes(rounds[0][2], dsa.WS_ATTN)), dtype=torch.uint8, device=dev)

    def step(evr=None):
        """One pass of the whole path; evr = per-round event quadruples or None."""
        if wl.idx_fp8:
            dsa.hadamard_quant_fp8(q_idx, q8, qs, stream=stream)
            qi, qsc = q8, qs
        else:
            qi, qsc = q_idx, None
        for ri, (t0, c, sh, pos0) in enumerate(rounds):
            ev = evr[ri] if evr is not None else None
            sl = slice(t0, t0 + c)
            if ev: ev[0].record(stream)
            dsa.indexer_scores_hist(sh, qi[:, sl], k_idx, t["w"][:, sl], t["ctx_len"], pos0, hist,
                                    scores=scores[:, :c], q_scale=None if qsc is None else qsc[:, sl],
                                    k_scale=k_scale, stream=stream)
            if ev: ev[1].record(stream)
            if kc:
                dsa.topk_hist(sh.replace(topk=kc), scores[:, :c], t["ctx_len"], pos0, hist, idx=cand[:, :c],
                              stream=stream)
                dsa.indexer_rescore(sh, q_idx[:, sl], k_ref, t["w"][:, sl], cand[:, :c], kc, t["ctx_len"], pos0,
                                    scores=cand_sc[:, :c], stream=stream)
                dsa.topk_candidates(sh, cand_sc[:, :c], cand[:, :c], kc, t["ctx_len"], pos0, idx=idx[:, :c],
                                    stream=stream)
            else:
                dsa.topk_hist(sh, scores[:, :c], t["ctx_len"], pos0, hist, idx=idx[:, :c], stream=stream)
            if ev: ev[2].record(stream)
            dsa.sparse_mla_attn(sh, t["q"][:, sl], t["kv"], idx[:, :c], t["ctx_len"], out=out[:, sl],
                                workspace=ws_attn, stream=stream)
            if ev: ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    rc, word = dsa.get_error(clear=True)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x} after warm-up")

    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in rounds] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    # the timed steps run the pipeline as a user does (no events between its
    # kernels, which would keep each launch from overlapping the previous
    # kernel's tail); the per-stage split comes from a second pass below
    start.record(stream)
    for i in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if ws > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    stage_ms = {"indexer": 0.0, "topk": 0.0, "attention": 0.0}
    for per_step in evs:
        for e in per_step:
            stage_ms["indexer"] += e[0].elapsed_time(e[1])
            stage_ms["topk"] += e[1].elapsed_time(e[2])
            stage_ms["attention"] += e[2].elapsed_time(e[3])
    stage_ms = {k: v / args.steps for k, v in stage_ms.items()}
    rc, word = dsa.get_error(clear=True)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x} after timing")
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps

    # end to end through the host-buffer entry point
    e2e = _e2e(args, wl, dsa, dsa.shape_from_workload(wl, q_chunk=chunk if len(rounds) > 1 else 0), t, k_idx,
               k_scale, dev, stream, k_ref)
    e2e["ms"] = max_over_ranks(e2e["ms"], dev)

    res = None
    if rank == 0:
        hbm, tf, tf_sus, src = _peaks()
        idx_ms = stage_ms["indexer"]
        q_total = _queries(wl) * ws
        decode = wl.n_q == 1
        if decode:
            idx_bytes = _indexer_bytes(wl)
            achieved = idx_bytes / (idx_ms * 1e-3) / 1e9
            roof = {"kernel": "indexer", "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "peak_source": f"{src} hbm_gbs (of {src})",
                    "traffic": _traffic(wl), "algorithmic_bytes": idx_bytes,
                    "tensor_tflops": _indexer_flops(wl) / (idx_ms * 1e-3) / 1e12}
            metric = _metric_name(wl)
        else:
            flops = _indexer_flops(wl)
            achieved = flops / (idx_ms * 1e-3) / 1e12
            peak = tf_sus if tf_sus > 0 else tf
            roof = {"kernel": "indexer", "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "peak_source": f"{src} bf16_tflops_sustained (of {src})",
                    "traffic": _traffic(wl), "algorithmic_flops": flops}
            metric = _metric_name(wl)
        res = {
            "metric": metric,
            "value": q_total / (ms_per_step * 1e-3),
            "unit": "queries/s" if decode else "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if not wl.idx_fp8 else "bf16+e4m3-indexer",
            "data": "synthetic (seeded gaussian, bf16)",
            "config": {"workload": _workload_desc(wl), "global_batch": q_total, "seq_len": wl.s_max,
                       "parallelism": f"replicas{ws}" if ws > 1 else "single",
                       "q_chunk": chunk,
                       "l2": "inputs larger than L2 (index-key cache read each step)" if decode
                             else "latent cache fits L2 (9.4 MB at 8K); no flush between steps"},
            "stages_ms": stage_ms,
            "roofline": roof,
            "roofline_bytes": ("indexer launch: index-key rows read + query block + head weights + fp32 score row "
                               "written" if decode else "indexer launch: 2 * 64 * 128 flop per causal (query, key) pair"),
            "gpu_launches": args.steps * (len(rounds) * (3 + (2 if kc else 0)
                                                         + _attn_extra_launches(wl, dsa, rounds[0][2]))
                                          + (1 if wl.idx_fp8 else 0)),
            "clocks": clk,
            "e2e": {"value": q_total / (e2e["ms"] * 1e-3), "unit": "queries/s" if decode else "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "ms_per_step": e2e["ms"],
                    # this box's pinned copy rates: the step cannot run faster than its own copies
                    "copy": e2e["copy"],
                    "copy_bound_per_s": q_total / (max(e2e["copy"]["both_ms_per_step"], ms_per_step) * 1e-3),
                    # host time to enqueue one step (the calls return before the work ends): a step
                    # whose issue time exceeds its device time is bound by the host
                    "host_issue_ms_per_step": e2e["host_issue_ms"],
                    # host buffers pinned after binding to the GPU's nearest CPUs (their count), or null
                    "near_gpu_cpus": e2e["near_cpus"]},
        }
    if ws > 1:
        torch.distributed.destroy_process_group()
    return res


def _bind_near_gpu(dev):
    """Restrict this process to the CPUs nearest the GPU (NVML's affinity set
    for it), so the host buffers pinned afterwards are allocated on the GPU's
    NUMA node: pinned memory on the far socket slows the GPU's reads of it
    (host -> device copies) well below the link rate.  A host-side setting of
    this process only; returns the CPU count bound to, or None if NVML cannot
    tell."""
    try:
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(dev)
        bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        words = pynvml.nvmlDeviceGetCpuAffinity(h, (os.cpu_count() + 63) // 64)
        cpus = {w * 64 + b for w, m in enumerate(words) for b in range(64) if (m >> b) & 1}
        cpus &= set(range(os.cpu_count()))
        if not cpus:
            return None
        os.sched_setaffinity(0, cpus)
        return len(cpus)
    except Exception:
        return None


def _e2e(args, wl, dsa, shape, t, k_idx, k_scale, dev, stream, k_ref=None):
    """dsa_forward_host_async, one call a step: this step's queries copied in
    from pinned memory and the output copied back every step (the copy-back
    runs under the next step's indexer and top-k), caches resident on the
    device.  The timed region ends when the last step's output is in host
    memory."""
    all_cpus = os.sched_getaffinity(0)
    near = _bind_near_gpu(dev)
    pin = lambda x: x.cpu().pin_memory()
    h = {k: pin(t[k]) for k in ("q_idx", "w", "q", "ctx_len", "q_pos0")}
    h_out = torch.empty(wl.batch, wl.n_q, wl.heads, wl.d_v, dtype=t["q"].dtype).pin_memory()
    wsb = torch.empty(dsa.workspace_bytes(shape, dsa.WS_FORWARD_HOST), dtype=torch.uint8, device=dev)
    done = torch.cuda.Event()
    call = lambda: dsa.forward_host_async(shape, h["q_idx"], h["w"], h["q"], h["ctx_len"], h["q_pos0"], k_idx,
                                          t["kv"], h_out, done=done, k_scale=k_scale, workspace=wsb, stream=stream,
                                          k_rescore=k_ref)
    for _ in range(max(1, args.warmup)):
        call()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    s.record(stream)
    t_issue = time.perf_counter()
    for _ in range(args.steps):
        call()
    t_issue = time.perf_counter() - t_issue  # host time to enqueue the steps (diagnostic)
    stream.wait_event(done)  # the last step's output is in host memory
    e.record(stream)
    torch.cuda.synchronize(dev)
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = h_out.numel() * h_out.element_size()
    ms = s.elapsed_time(e) / args.steps
    copy = _copy_rates(h["q"], h_out, dev)
    os.sched_setaffinity(0, all_cpus)  # (the pinned pages stay where they were placed)
    return {"ms": ms, "h2d": h2d, "d2h": d2h, "copy": copy,
            "host_issue_ms": t_issue * 1e3 / args.steps, "near_cpus": near}


def _copy_rates(h_in, h_out, dev, reps=10):
    """Pinned host <-> device copy rates of this machine for the step's two largest
    transfers (the attention queries in, the output back): each direction
    alone, then both at once on two streams (as the asynchronous step
    overlaps them)."""
    d_in = torch.empty_like(h_in, device=dev)
    d_out = torch.empty_like(h_out, device=dev)
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nb_in = h_in.numel() * h_in.element_size()
    nb_out = h_out.numel() * h_out.element_size()

    def timed(fn, stream):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    with torch.cuda.stream(s1):
        h2d_ms = timed(lambda: d_in.copy_(h_in, non_blocking=True), s1)
        d2h_ms = timed(lambda: h_out.copy_(d_out, non_blocking=True), s1)
    # both directions at once: the wall time of `reps` of each, overlapped
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(s1)
    s2.wait_event(a)
    for _ in range(reps):
        with torch.cuda.stream(s1):
            d_in.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(s2):
            h_out.copy_(d_out, non_blocking=True)
    s1.wait_stream(s2)
    b.record(s1)
    torch.cuda.synchronize(dev)
    both_ms = a.elapsed_time(b) / reps
    return {"h2d_gbs": nb_in / (h2d_ms * 1e-3) / 1e9, "d2h_gbs": nb_out / (d2h_ms * 1e-3) / 1e9,
            "both_ms_per_step": both_ms}


def _oracle_sample(wl, n_rows, seed=0):
    """The CPU oracle (as it stands) on `n_rows` query rows of the workload:
    indexer scores -> top-k -> sparse attention.  Decode: `n_rows` sequences
    of the workload's context; prefill: `n_rows` query rows drawn uniformly
    from one sequence.  Returns (seconds, rows)."""
    import numpy as np
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if wl.n_q == 1:
        sub = workloads.get(wl.name, batch=n_rows)
        rows = [(b, 0) for b in range(n_rows)]
    else:
        sub = workloads.get(wl.name, batch=1)
        rows = [(0, r) for r in workloads.sample_rows(wl.n_q, n_rows, seed=seed + 1)]
    t = workloads.make_inputs(sub, dev, seed=seed)
    h = {k: workloads.to_numpy(v) for k, v in t.items()}
    t0 = time.perf_counter()
    sc = oracle.indexer_scores(h["q_idx"], h["k_idx"], h["w"], h["ctx_len"], h["q_pos0"], rows=rows)
    pos = np.array([h["q_pos0"][b] + r for b, r in rows], dtype=np.int32)
    idx = oracle.topk(np.where(np.isfinite(sc), sc, -np.inf).astype(np.float32), pos, sub.topk)
    oracle.sparse_attn(h["q"], h["kv"], idx, sub.sm_scale, v=sub.d_v, rows=rows)
    return time.perf_counter() - t0, len(rows)


def cpu_baseline(wl, n_rows=None):
    import oracle
    cores = oracle.num_threads()
    n_rows = n_rows or (max(1, min(wl.batch, cores)) if wl.n_q == 1 else cores)
    secs, rows = _oracle_sample(wl, n_rows)
    what = (f"{rows} decode queries of the same workload (full {wl.s_max}-key context each)" if wl.n_q == 1
            else f"{rows} query rows drawn uniformly from the {wl.n_q}-token prefill")
    return {"value": rows / secs, "unit": "queries/s" if wl.n_q == 1 else "tokens/s", "cores": cores,
            "kind": "oracle", "sample": f"{what}, {secs:.1f} s on {cores} host threads"}


def run_reference(args, wl):
    """The reference arm: the fp64 CPU oracle, timed on the host cores."""
    ws, rank, _ = _dist()
    if rank != 0:
        return None
    import oracle
    cores = oracle.num_threads()
    n_rows = max(1, min(wl.batch, cores)) if wl.n_q == 1 else cores
    for _ in range(args.warmup and 1):
        _oracle_sample(wl, 1, seed=99)
    secs = 0.0
    rows = 0
    for i in range(args.steps):
        s, r = _oracle_sample(wl, n_rows, seed=i)
        secs += s
        rows += r
    value = rows / secs
    unit = "queries/s" if wl.n_q == 1 else "tokens/s"
    line = {
        "impl": "reference",
        "metric": _metric_name(wl),
        "value": value, "unit": unit, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded gaussian, bf16)",
        "config": {"workload": _workload_desc(wl), "global_batch": n_rows, "seq_len": wl.s_max,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {n_rows} query rows of the workload"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    return line


def run_append(args):
    """Cache append of one prefill chunk (the update before the step scores):
    `--append-tokens` new tokens of one sequence written into a 65536-row cache,
    index keys copied (bf16) or rotated + quantised (e4m3), latent rows copied.
    HBM-bound: per token the key (256 B) and latent row (1152 B) are read and
    written (the e4m3 key as 128 B of codes + a 4-byte scale)."""
    import long_context_indexing_lightning_b200 as dsa

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev).cuda_stream
    n, s_max = args.append_tokens, 65536
    g = torch.Generator(device=dev).manual_seed(0)
    k_new = (torch.randn(1, n, 128, generator=g, device=dev) / 11.3).to(torch.bfloat16)
    kv_new = torch.randn(1, n, 576, generator=g, device=dev).to(torch.bfloat16)
    kv_cache = torch.zeros(1, s_max, 576, dtype=torch.bfloat16, device=dev)
    caches = {"bf16": (torch.zeros(1, s_max, 128, dtype=torch.bfloat16, device=dev), None),
              "e4m3": (torch.zeros(1, s_max, 128, dtype=torch.uint8, device=dev),
                       torch.zeros(1, s_max, dtype=torch.float32, device=dev))}
    pos = torch.zeros(1, dtype=torch.int32, device=dev)
    res = {}
    for name, (k_cache, k_scale) in caches.items():
        shape = dsa.make_shape(1, 1, s_max, idx_dtype=dsa.DSA_E4M3 if name == "e4m3" else dsa.DSA_BF16)
        call = lambda: dsa.cache_append(shape, k_new, kv_new, pos, k_cache, kv_cache, k_scale=k_scale,
                                        stream=stream)
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize(dev)
        clocks = ClockSampler(local)
        clocks.start()
        time.sleep(0.3)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            call()
        e.record()
        torch.cuda.synchronize(dev)
        clk = clocks.stop()
        ms = max_over_ranks(s.elapsed_time(e) / args.steps, dev)
        key_out = 128 + 4 if name == "e4m3" else 256
        res[name] = (ms, n * (256 + 1152 + key_out + 1152), clk)
    rc, word = dsa.get_error(clear=True)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")
    if rank != 0:
        return None
    hbm, _, _, src = _peaks()
    ms, nbytes, clk = res["bf16"]
    achieved = nbytes / (ms * 1e-3) / 1e9
    ms8, nbytes8, _ = res["e4m3"]
    return {
        "metric": f"cache append tokens/s ({n}-token prefill chunk)",
        "value": n * ws / (ms * 1e-3), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded gaussian, bf16)",
        "config": {"workload": f"append: B=1, {n} new tokens into a 65536-row cache, index key 128 + latent 576",
                   "l2": "inputs + outputs larger than L2"},
        "roofline": {"kernel": "cache_append", "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "peak_source": f"{src} hbm_gbs (of {src})", "traffic": None,
                     "algorithmic_bytes": nbytes},
        "e4m3": {"ms_per_step": ms8, "tokens_per_s": n / (ms8 * 1e-3),
                 "achieved_gbs": nbytes8 / (ms8 * 1e-3) / 1e9, "frac": nbytes8 / (ms8 * 1e-3) / 1e9 / hbm},
        "gpu_launches": args.steps, "clocks": clk,
    }


def run_topk_structures(args):
    """Top-k alone at the 128K decode shape (32 rows x 131072 fp32 scores,
    k = 2048) on rows of four structures: gaussian, a planted recent window
    (the last 2048 keys above the rest), one exponent bucket (all in [1, 2))
    and all-equal scores.  Reports each case's launch time and the
    score-read rate against HBM."""
    import long_context_indexing_lightning_b200 as dsa

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, S, k = 32, 131072, 2048
    g = torch.Generator(device=dev).manual_seed(0)
    cases = {
        "gaussian": torch.randn(B, 1, S, generator=g, device=dev),
        "recent_window": torch.randn(B, 1, S, generator=g, device=dev),
        "one_exponent_bucket": 1.0 + torch.rand(B, 1, S, generator=g, device=dev),
        "all_equal": torch.full((B, 1, S), 0.75, device=dev),
    }
    cases["recent_window"][:, :, S - 2048:] = 4.0 + torch.rand(B, 1, 2048, generator=g, device=dev)
    ctx = torch.full((B,), S, dtype=torch.int32, device=dev)
    pos0 = ctx - 1
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
    shape = dsa.make_shape(B, 1, S, topk=k)
    ws_t = torch.empty(max(1, dsa.workspace_bytes(shape, dsa.WS_TOPK)), dtype=torch.uint8, device=dev)
    hbm, _, _, src = _peaks()
    out = {}
    for name, sc in cases.items():
        call = lambda: dsa.topk(shape, sc, ctx, pos0, idx=idx, workspace=ws_t)
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize(dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            call()
        e.record()
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(s.elapsed_time(e) / args.steps, dev)
        nbytes = B * S * 4 + B * k * 4
        out[name] = {"us": ms * 1e3, "rows_per_s": B / (ms * 1e-3),
                     "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm}
    rc, word = dsa.get_error(clear=True)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")
    if rank != 0:
        return None
    gms = out["gaussian"]["us"] * 1e-3
    return {"metric": "top-k rows/s at 128K (gaussian rows)", "value": B * ws / (gms * 1e-3), "unit": "rows/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": gms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic (seeded)", "config": {"workload": "top-k: B=32 rows x 131072 scores, k=2048",
                                                      "l2": "scores resident in L2 (16.8 MB) between launches"},
            "roofline": {"kernel": "topk_cluster", "bound": "hbm", "peak": hbm, "unit": "GB/s",
                         "achieved": (B * S * 4 + B * k * 4) / (gms * 1e-3) / 1e9,
                         "frac": out["gaussian"]["frac_hbm"], "peak_source": f"{src} hbm_gbs (of {src})",
                         "traffic": None},
            "cases": out, "gpu_launches": args.steps * len(cases)}


def run_proj(args):
    """The indexer projections alone (tensor-core GEMMs, synthetic seeded
    weights): wq_b on the query latent (1536 -> 64 x 128) and the fused index-
    key + weights_proj projection of the hidden state (7168 -> 128 + 64), for
    a decode step's 32 tokens and a 4096-token prefill round.  Reports each
    case's time and TFLOP/s against the bf16 tensor peak, and the bytes moved
    against HBM (the weight-bound decode case)."""
    import long_context_indexing_lightning_b200 as dsa

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm, tf, tf_sus, src = _peaks()
    shape = dsa.make_shape(1, 1, 1024)
    g = torch.Generator(device=dev).manual_seed(0)
    rnd = lambda *sh, std=1.0: (torch.randn(*sh, generator=g, device=dev) * std).to(torch.bfloat16)
    wq = rnd(64 * 128, 1536, std=1536 ** -0.5)
    wkw = rnd(192, 7168, std=7168 ** -0.5)
    out = {}
    for T in (32, 4096):
        lat, x = rnd(T, 1536), rnd(T, 7168)
        q_idx = torch.empty(T, 64, 128, dtype=torch.bfloat16, device=dev)
        k_new = torch.empty(T, 128, dtype=torch.bfloat16, device=dev)
        w = torch.empty(T, 64, dtype=torch.float32, device=dev)
        cases = {
            f"wq_b T={T}": (lambda: dsa.indexer_proj_q(shape, lat, wq, q_idx=q_idx),
                           2 * T * 1536 * 8192, (T * 1536 + 8192 * 1536 + T * 8192) * 2),
            f"key+weights T={T}": (lambda: dsa.indexer_proj_kw(shape, x, wkw, k_new=k_new, w=w),
                                  2 * T * 7168 * 192, (T * 7168 + 192 * 7168) * 2 + T * (128 * 2 + 64 * 4)),
        }
        for name, (call, flops, nbytes) in cases.items():
            for _ in range(args.warmup):
                call()
            torch.cuda.synchronize(dev)
            s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s_.record()
            for _ in range(args.steps):
                call()
            e_.record()
            torch.cuda.synchronize(dev)
            ms = max_over_ranks(s_.elapsed_time(e_) / args.steps, dev)
            out[name] = {"us": ms * 1e3, "tflops": flops / (ms * 1e-3) / 1e12,
                         "frac_tensor": flops / (ms * 1e-3) / 1e12 / tf, "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm}
    rc, word = dsa.get_error(clear=True)
    if rc != 0:
        raise RuntimeError(f"device error word {word:#x}")
    if rank != 0:
        return None
    main_case = out["wq_b T=4096"]
    return {"metric": "indexer projection TFLOP/s (wq_b, 4096 tokens)", "value": main_case["tflops"],
            "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": main_case["us"] * 1e-3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded weights and activations)",
            "config": {"workload": "indexer projections: wq_b 1536->8192, key+weights 7168->192; 32 and 4096 tokens"},
            "roofline": {"kernel": "proj_gemm", "bound": "tensor", "peak": tf, "unit": "TFLOP/s",
                         "achieved": main_case["tflops"], "frac": main_case["frac_tensor"],
                         "peak_source": f"{src} bf16_tflops (of {src})", "traffic": None},
            "cases": out, "gpu_launches": args.steps * 4}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode128k", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling runs)")
    ap.add_argument("--ctx", type=int, default=0, help="override the workload's cache length (profiling runs)")
    ap.add_argument("--q-chunk", type=int, default=4096, help="prefill: queries per indexer/top-k/attention round")
    ap.add_argument("--op", default="step", choices=["step", "append", "topk", "proj"],
                    help="step: the layer step (default); append: the cache append of one prefill chunk; "
                         "topk: top-k alone on structured 128K rows; proj: the indexer projections alone")
    ap.add_argument("--append-tokens", type=int, default=65536)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    over = {}
    if args.batch:
        over["batch"] = args.batch
    if args.ctx:
        over["s_max"] = args.ctx
        if workloads.get(args.workload).n_q > 1:
            over["n_q"] = args.ctx
    wl = workloads.get(args.workload, **over)
    if args.op in ("append", "topk", "proj") and args.impl == "ours":
        line = {"append": run_append, "topk": run_topk_structures, "proj": run_proj}[args.op](args)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.impl == "reference":
        line = run_reference(args, wl)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    res = run_ours(args, wl)
    ws, rank, _ = _dist()
    if rank == 0:
        if ws == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
