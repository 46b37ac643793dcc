"""Benchmark of the Adamas decode step on B200: µs per step and effective HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--budget 128]
                    [--shared] [--paged PAGE] [--thresholds fixed|absmax] [--cp W]
                    [--policy auto|cluster|flat] [--no-per-config] [--impl ours|reference]

Default workload: one Llama-3.1-8B-shaped layer, batch 1, 32 query / 8 kv heads,
d = 128, context 32768, bf16 K/V with 4 outlier channels, budget 128.  A "step" is
one adamas_decode_step (query encode, distance scan, top-k, gather attention,
combine: one kernel launch).  The default line also carries `per_config`: every
workload at the budgets it is quoted on, timed the same way.  --shared times the variant with
one selection per kv head shared by its query heads (adamas_decode_step_shared);
its algorithmic bytes count the selected K/V rows once per kv head.

Timing: inputs resident in HBM; R independent replicas of codes + K + V are
rotated so the working set of consecutive steps exceeds 2x L2 (no cache reuse
between steps); K steps are captured in CUDA graphs and timed with CUDA events on
the launching stream, bracketed by barrier + synchronize; max over ranks.
Multi-GPU: `--gpus N` starts N local ranks (torch.distributed.run) unless a launcher
already set WORLD_SIZE; every rank runs its own replica set (weak scaling, no
collective on the data path).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, generate, replicas_for_l2  # noqa: E402

METRIC = "decode µs/step & effective HBM GB/s (% of roofline) at 32K ctx, budget 128"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")


# ------------------------------------------------------------------ helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the sources of the decode kernel whose ncu traffic is recorded (its device code, the
# shared device helpers, and its launch)
DECODE_SOURCES = ("decode.cu", "adamas_internal.cuh")


def csrc_digest() -> str:
    """Digest of the decode kernel's CUDA sources with comments and white space removed:
    editing a comment keeps the recorded ncu traffic valid, changing code does not."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        p = os.path.join(ROOT, "token_level_sparse_fwht_b200", "csrc", name)
        with open(p, encoding="utf-8") as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload_key: str):
    """DRAM bytes per launch of the decode kernel from the committed ncu summary, or
    None if there is none for this workload or the kernel source changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(workload_key)
    if not e or e.get("csrc_sha") != csrc_digest():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms in the background."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings over all ranks (every rank calls it)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def aggregate_gbs(step_bytes: int, seconds_per_step: float, world: int) -> float:
    """Whole-job effective GB/s under weak scaling: every rank runs its own step
    (independent units, no collective on the data path); the job's time per step
    is the slowest rank's."""
    return step_bytes * world / seconds_per_step / 1e9


# ------------------------------------------------------------- our arm
def smi_id(dev) -> str:
    """nvidia-smi id of a torch device (UUID, so CUDA_VISIBLE_DEVICES does not matter)."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index)


def measure(args, config, k, dev, world, per_config=False):
    """One workload at one budget: data on the device, then the timed steps.

    A step is one pass of the whole path over one batch: every layer's
    adamas_decode_step (and, for the batch-8 workload, the adamas_encode_keys of the
    appended tokens first).  K steps run in CUDA graphs on one stream, timed with
    CUDA events and bracketed by barrier + synchronize; W graph replays come first.
    Returns a dict of measurements (times are this rank's)."""
    import token_level_sparse_fwht_b200 as ad

    w = WORKLOADS[config]
    L = w.L
    t = w.t
    absmax = args.thresholds == "absmax" and not per_config
    shared = args.shared and not per_config
    paged = args.paged if not per_config else 0
    cpW = args.cp if not per_config else 0
    ratio = 0.5
    if absmax and (paged or w.append):
        raise SystemExit("--thresholds absmax is measured on contiguous caches without append")
    layer_sets = []
    planted = None   # layer 0's planted key positions [B, Hq, n] (planted workloads)
    append_check = None
    for layer in range(w.layers):
        inp = generate(w, dev, layer=layer)
        if layer == 0 and inp.planted is not None:
            planted = inp.planted.cpu()
        codes = torch.empty(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device=dev)
        if absmax:
            ad.encode_keys_absmax(inp.k_cache, codes, 0, L, ratio)
        else:
            ad.encode_keys(inp.k_cache, codes, 0, L, t)
        if layer == 0 and w.append:
            # the appended keys' codes against the oracle (outside the timed region)
            append_check = (inp.k_cache[:, :, L - w.append:L].cpu(),
                            codes[:, :, L - w.append:L].cpu())
        layer_sets.append((inp.q, inp.k_cache, inp.v_cache, codes))
        del inp
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    append = w.append
    decode = ad.decode_step_shared if shared else ad.decode_step
    step_bytes = w.algorithmic_bytes(k, shared) * w.layers
    if append:
        step_bytes += w.B * w.Hkv * append * (128 * w.elem_bytes + 32)
    pc = None
    if paged:
        # the same caches held in a page pool (shuffled pages, block table, lengths);
        # an append re-encodes the pages that hold the new positions
        from workloads.paging import make_block_table, scatter_to_pages
        ps = paged
        pc = make_block_table([L] * w.B, L, ps, seed=config, spare=0)
        bt = pc.block_table.to(dev)
        lens = pc.seq_lens.to(dev)
        app_ids = (pc.block_table[:, (L - append) // ps:(L + ps - 1) // ps].reshape(-1)
                   .contiguous().to(dev) if append else None)
        paged_sets = []
        while layer_sets:
            q, kc, vc, cd = layer_sets.pop(0)
            paged_sets.append((q, scatter_to_pages(kc, pc), scatter_to_pages(vc, pc),
                               scatter_to_pages(cd, pc)))
            del kc, vc, cd
        layer_sets = paged_sets
    R = args.replicas or replicas_for_l2(step_bytes, l2, 2.0)
    sets = [layer_sets]
    for _ in range(R - 1):
        sets.append([tuple(x.clone() for x in ls) for ls in layer_sets])
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, L, k, dev)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    plan = (ad.decode_plan_shared if shared else ad.decode_plan)(w.B, w.Hq, w.Hkv, L, k)
    launches_per_step = w.layers * (2 if append else 1) * (1 if not cpW else 3)

    if cpW:
        # one rank of a context-parallel step over W GPUs, on one GPU: this rank holds
        # the first L / W positions; both all-gathers are stood in for by a local copy
        # of this rank's own tensor into the gathered buffer (the NCCL transfer itself
        # is not timed)
        if paged or absmax or append or w.layers > 1:
            raise SystemExit("--cp is measured on one contiguous layer without append")
        Ls = L // cpW
        hist_all = torch.empty((cpW,) + ad.cp_hist_shape(w.B, w.Hq, w.Hkv, shared),
                               dtype=torch.int32, device=dev)
        part_all = torch.empty((cpW, w.B, w.Hq, ad.PART_STRIDE), dtype=torch.float32,
                               device=dev)
        ws_cp = ad.cp_workspace(w.B, w.Hq, w.Hkv, Ls, k, shared, dev)
        step_bytes = (w.B * w.Hkv * Ls * 32 + w.B * w.Hq * min(k, L) // cpW * 2 * 128
                      * w.elem_bytes + w.B * w.Hq * 128 * (w.elem_bytes + 4))

    def step(i, s, q_override=None, out_t=None):
        if cpW:
            for (q, kc, vc, cd) in sets[i % R]:
                qq = q if q_override is None else q_override
                o = out if out_t is None else out_t
                ad.cp_histograms(qq, cd, Ls, k, t, ws_cp, shared=shared, hist_out=hist_all[0],
                                 stream=s)
                hist_all[1:].copy_(hist_all[0].expand_as(hist_all[1:]))
                ad.cp_attend(qq, kc, vc, cd, Ls, L, 0, k, t, hist_all, 0, ws_cp, shared=shared,
                             partial_out=part_all[0], stream=s)
                part_all[1:].copy_(part_all[0].expand_as(part_all[1:]))
                ad.cp_combine(part_all, out=o, stream=s)
            return
        for (q, kc, vc, cd) in sets[i % R]:
            qq = q if q_override is None else q_override
            o = out if out_t is None else out_t
            if pc is not None:
                if append:
                    ad.encode_pages(kc, cd, t, page_ids=app_ids, stream=s)
                ad.decode_step_paged(qq, kc, vc, cd, bt, lens, L, k, t, ws, shared=shared, out=o,
                                     stream=s)
                continue
            if append:
                ad.encode_keys(kc, cd, L - append, append, t, stream=s)
            if absmax:
                ad.decode_step_absmax(qq, kc, vc, cd, L, k, ratio, ws, shared=shared, out=o,
                                      stream=s)
                continue
            decode(qq, kc, vc, cd, L, k, t, ws, out=o, stream=s)

    # eager warm-up (also loads the kernels and sets their attributes)
    with torch.cuda.stream(stream):
        for i in range(max(3, min(args.warmup, 3 * R))):
            step(i, stream)
    stream.synchronize()
    ad.check_workspace(ws, stream)

    # The K timed steps are captured in CUDA graphs of `chunk` steps (rotating replicas),
    # the first graph opening with an event-record node and the last closing with one:
    # the events then bracket exactly the K steps on the device, not the host's
    # submission of the graph to an idle GPU.  A second set of graphs without event
    # nodes serves the warm-up and the extra replays behind the median.
    K = args.steps
    chunk = max(1, min(K, 1000 // launches_per_step))
    sizes = [chunk] * (K // chunk) + ([K % chunk] if K % chunk else [])
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    timed, plain = [], []
    use_graph = True
    try:
        done = 0
        for gi, n in enumerate(sizes):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    if gi == 0:
                        e0.record(stream)
                    for i in range(n):
                        step(done + i, stream)
                    if gi == len(sizes) - 1:
                        e1.record(stream)
            timed.append(g)
            done += n
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(chunk):
                    step(i, stream)
        plain.append(g)
    except Exception as e:  # capture unsupported: launch eagerly
        use_graph = False
        timed, plain = [], []
        print(f"# graph capture failed ({e}); eager launches", file=sys.stderr)
    stream.synchronize()

    sampler = ClockSampler(smi_id(dev)) if not per_config else None
    if sampler:
        sampler.start()
    # W warm-up steps (and one untimed run of the timed graphs: a graph's first launch
    # also uploads it), then the timed K steps
    with torch.cuda.stream(stream):
        if use_graph:
            for g in timed:
                g.replay()
        for _ in range(max(1, math.ceil(args.warmup / max(1, chunk)))):
            if use_graph:
                plain[0].replay()
            else:
                step(0, stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        if use_graph:
            for g in timed:
                g.replay()
        else:
            e0.record(stream)
            for i in range(K):
                step(i, stream)
            e1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    # median step time over further replays of the timed graphs (at least 10, and for
    # about 0.6 s, so the clock sampler sees the GPU under this load)
    reps = []
    t_end = time.perf_counter() + (0.6 if sampler else 0.0)
    while len(reps) < 10 or (time.perf_counter() < t_end and len(reps) < 5000):
        with torch.cuda.stream(stream):
            if use_graph:
                for g in timed:
                    g.replay()
            else:
                e0.record(stream)
                for i in range(K):
                    step(i, stream)
                e1.record(stream)
        stream.synchronize()
        reps.append(e0.elapsed_time(e1) * 1e3 / K)
    med_us = statistics.median(reps)
    clocks = sampler.stop() if sampler else None
    ad.check_workspace(ws, stream)
    del timed, plain

    # e2e through the public API with host buffers: every step copies its queries in
    # from pinned host memory and reads the fp32 output back
    q_host = torch.stack([ls[0] for ls in layer_sets]).cpu().pin_memory()
    out_host = torch.empty((w.layers,) + tuple(out.shape), dtype=torch.float32).pin_memory()
    q_dev = torch.empty(q_host.shape, dtype=q_host.dtype, device=dev)
    outs = torch.empty(out_host.shape, dtype=torch.float32, device=dev)
    K2 = max(3, min(K, 2000 // w.layers))

    # per layer one C call: pinned q in, fused decode, fp32 out back to pinned host;
    # the calls are bound to their buffers once, as a serving loop would
    calls = None
    if not cpW:
        def bind(li, kc, vc, cd):
            if pc is not None:
                return ad.PreparedPagedDecodeHost(q_host[li], q_dev[li], kc, vc, cd, bt, lens, L,
                                                  k, t, ws, outs[li], out_host[li], shared=shared,
                                                  stream=stream)
            if absmax:
                return ad.PreparedAbsmaxDecodeHost(q_host[li], q_dev[li], kc, vc, cd, L, k, ratio,
                                                   ws, outs[li], out_host[li], shared=shared,
                                                   stream=stream)
            return ad.PreparedDecodeHost(q_host[li], q_dev[li], kc, vc, cd, L, k, t, ws, outs[li],
                                         out_host[li], stream=stream, shared=shared)
        calls = [[bind(li, kc, vc, cd) for li, (q, kc, vc, cd) in enumerate(sets[r])]
                 for r in range(R)]

    def e2e_step(i):
        if cpW:
            q_dev.copy_(q_host, non_blocking=True)
            step(i, stream, q_override=q_dev[0], out_t=outs[0])
            out_host.copy_(outs, non_blocking=True)
            return
        for li, (q, kc, vc, cd) in enumerate(sets[i % R]):
            if append:
                if pc is not None:
                    ad.encode_pages(kc, cd, t, page_ids=app_ids, stream=stream)
                else:
                    ad.encode_keys(kc, cd, L - append, append, t, stream=stream)
            calls[i % R][li]()

    with torch.cuda.stream(stream):
        for i in range(3):
            e2e_step(i)
    stream.synchronize()
    # pipelined: K2 calls queued back to back between two events
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for i in range(K2):
            e2e_step(i)
        f1.record(stream)
    stream.synchronize()
    ms_e2e = f0.elapsed_time(f1)
    # synchronised: a serving loop that needs each step's output on the host before
    # the next step (host clock from the call to the stream's completion)
    sync_us = []
    with torch.cuda.stream(stream):
        for i in range(max(10, min(K2, 200))):
            h0 = time.perf_counter()
            e2e_step(i)
            stream.synchronize()
            sync_us.append((time.perf_counter() - h0) * 1e6)
    sync_med = statistics.median(sync_us)

    # recall of the planted keys: one more step on layer 0 with its selections read back
    recall = None
    if planted is not None and not cpW and pc is None:
        idx = torch.empty((w.B, w.Hkv if shared else w.Hq, min(k, L)), dtype=torch.int32,
                          device=dev)
        q, kc, vc, cd = sets[0][0]
        with torch.cuda.stream(stream):
            if absmax:
                ad.decode_step_absmax(q, kc, vc, cd, L, k, ratio, ws, shared=shared, out=out,
                                      idx_out=idx, stream=stream)
            else:
                decode(q, kc, vc, cd, L, k, t, ws, out=out, idx_out=idx, stream=stream)
        stream.synchronize()
        sel = idx.cpu().long()
        hits = [torch.isin(planted[b, h], sel[b, h // w.G if shared else h]).double().mean()
                for b in range(w.B) for h in range(w.Hq)]
        recall = round(float(torch.stack(hits).mean()), 4)

    h2d = q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    del sets, layer_sets, calls, ws, out, q_host, out_host, q_dev, outs
    torch.cuda.empty_cache()
    ms, ms_e2e, med_us, sync_med = max_over_ranks([ms, ms_e2e, med_us, sync_med], world, dev)
    flat = plan["cluster"] == 1 and plan["ctas"] > w.B * w.Hkv
    return dict(w=w, k=k, ms=ms, ms_e2e=ms_e2e, K=K, K2=K2, R=R, step_bytes=step_bytes,
                us_median=med_us, sync_us=sync_med, recall=recall, append_check=append_check,
                clocks=clocks, plan=plan, use_graph=use_graph,
                kernel="decode_flat_kernel" if flat else "decode_kernel",
                launches=K * launches_per_step, h2d=h2d, d2h=d2h)


# the bench line's per_config entries: every workload at the budgets it is quoted on
PER_CONFIG = [(1, 64), (2, 64), (2, 128), (2, 256), (2, 1024), (3, 256), (3, 1024), (4, 128),
              (4, 1024), (5, 1024)]


def measure_encoder(args, dev, world):
    """Key encode of the workload's whole cache (one layer): adamas_encode_keys over all
    B x Hkv x L keys, timed alone with CUDA events on the launching stream, the L2
    flushed (a buffer of 4x L2 written) before every run; median of `--steps` runs
    after `--warmup`, max over ranks."""
    import token_level_sparse_fwht_b200 as ad
    w = WORKLOADS[args.config]
    inp = generate(w, dev)
    codes = torch.empty(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(4 * l2, dtype=torch.uint8, device=dev)
    times = []
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 0xff)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        ad.encode_keys(inp.k_cache, codes, 0, w.L, inp.t)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1) * 1e3)
    us = max_over_ranks([statistics.median(times)], world, dev)[0]
    nbytes = inp.k_cache.numel() * inp.k_cache.element_size() + codes.numel()
    peak, peak_kind = peaks()
    gbs = nbytes / us / 1e3
    return {"metric": "key encode of the whole cache (one layer), µs and effective HBM GB/s",
            "value": round(gbs * world, 2), "unit": "GB/s", "n_gpus": world,
            "us": round(us, 3), "bytes": nbytes, "frac": round(gbs / peak, 4),
            "peak": peak, "peak_source": f"{peak_kind} hbm_gbs", "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "data": "synthetic",
            "dtype": str(inp.k_cache.dtype).replace("torch.", ""),
            "config": {"workload": w.name, "keys": int(inp.k_cache.numel() // 128),
                       "l2": "flushed before every run"}}


def per_config_entry(r, peak):
    w, k = r["w"], r["k"]
    per_step_s = r["ms"] / 1e3 / r["K"]
    gbs = aggregate_gbs(r["step_bytes"], per_step_s, 1)
    e = {"workload": w.name, "k": k, "us_per_step": round(per_step_s * 1e6, 3),
         "us_per_step_median_replay": round(r["us_median"], 3),
         "gbs": round(gbs, 2), "frac": round(gbs / peak, 4),
         "algorithmic_bytes_per_step": r["step_bytes"], "ctas": r["plan"]["ctas"],
         "kernel": r["kernel"], "steps": r["K"],
         "e2e_us_per_step": round(r["ms_e2e"] / 1e3 / r["K2"] * 1e6, 3),
         "e2e_sync_us_per_step": round(r["sync_us"], 2)}
    if r["recall"] is not None:
        e["recall_planted_keys"] = r["recall"]
    return e


def cpu_append_baseline(w, keys, gpu_codes):
    """CPU-baseline leg for a workload with an append: the float64 oracle encodes the
    appended keys on one host core (timed), and the GPU encoder's codes of the same
    keys are compared with it (the fraction of coordinates whose code differs; a
    coordinate within rounding distance of a threshold may legitimately differ)."""
    import oracle
    kk = keys.double().numpy()
    t0 = time.perf_counter()
    want = oracle.encode(kk, w.t)
    ms = (time.perf_counter() - t0) * 1e3
    diff = oracle.unpack_codes(gpu_codes.numpy()) != oracle.unpack_codes(want)
    return {"oracle_encode_ms": round(ms, 2), "cores": 1,
            "gpu_code_mismatch_fraction": float(diff.mean()),
            "sample": f"all {kk.shape[0] * kk.shape[1] * kk.shape[2]} appended keys of layer 0"}


# --------------------------------------------------- float64 oracle on host
def oracle_inputs(w, seed_device="cpu"):
    import numpy as np  # noqa: F401
    import oracle
    inp = generate(w, seed_device)
    q = inp.q.double().cpu().numpy()
    K = inp.k_cache.double().cpu().numpy()
    V = inp.v_cache.double().cpu().numpy()
    return inp.t, q, K, V, oracle


def cpu_baseline(w, k, budget_s=12.0, shared=False, absmax=False, max_threads=16):
    """The float64 oracle, as it stands, on the host cores over a bounded, seeded
    sample of the workload.

    A job is one (layer, sequence, kv head) unit, the kv head's G query heads run
    through the oracle's own decode step on that unit's slice.  Key codes are cache
    state and are built before timing; the query encode is timed.  Jobs are drawn in
    a seeded order (two layers sampled for multi-layer workloads) and run on one
    thread for about budget_s seconds; the step time is the mean job time times the
    jobs in a step.  The same jobs are then run over a pool of
    threads (threads over units; numpy releases the GIL in the array work), and, for
    a workload with an append, the oracle's encode of the appended keys is timed on
    its own."""
    import concurrent.futures
    import numpy as np
    import oracle
    rng = np.random.default_rng(7 + w.config)
    G = w.G
    layers = (sorted(int(x) for x in rng.choice(w.layers, size=min(w.layers, 2), replace=False))
              if w.layers > 1 else [0])
    jobs = [(layer, b, kv) for layer in layers for b in range(w.B) for kv in range(w.Hkv)]
    order = rng.permutation(len(jobs))
    jobs = [jobs[i] for i in order]
    jobs_per_step = w.layers * w.B * w.Hkv
    step_bytes = w.algorithmic_bytes(k, shared) * w.layers
    inputs = {}
    cache = {}

    def layer_inputs(layer):
        # the sampled layers (at most two) stay in host memory
        if layer not in inputs:
            inputs[layer] = generate(w, "cpu", layer=layer)
        return inputs[layer]

    def prepared(job, keep=1):
        """(q slice, K, V, key codes) of a job, float64; keeps `keep` jobs' rows."""
        layer, b, kv = job
        if job not in cache:
            while len(cache) >= keep:
                cache.pop(next(iter(cache)))
            inp = layer_inputs(layer)
            K = inp.k_cache[b:b + 1, kv:kv + 1].double().numpy()
            V = inp.v_cache[b:b + 1, kv:kv + 1].double().numpy()
            kc = oracle.encode_absmax(K, 0.5) if absmax else oracle.encode(K, w.t)
            cache[job] = (inp.q[b:b + 1, kv * G:(kv + 1) * G].double().numpy(), K, V, kc)
        return cache[job]

    def run(qs, K, V, kc):
        qc = oracle.encode_absmax(qs, 0.5) if absmax else None
        fn = oracle.decode_step_shared if shared else oracle.decode_step
        fn(qs, K, V, k, w.t, key_codes=kc, query_codes=qc)

    # one thread
    times = []
    i = 0
    wall0 = time.perf_counter()
    while sum(times) < budget_s and (i < len(jobs) or time.perf_counter() - wall0 < 3 * budget_s):
        args_ = prepared(jobs[i % len(jobs)])
        t0 = time.perf_counter()
        run(*args_)
        times.append(time.perf_counter() - t0)
        i += 1
    per_job = sum(times) / len(times)
    per_step = per_job * jobs_per_step
    whole = len(times) >= jobs_per_step and w.layers == 1
    res = {"value": round(step_bytes / per_step / 1e9, 6), "unit": "GB/s", "cores": 1,
           "kind": "oracle",
           "sample": (f"{len(times)} oracle decode jobs (one kv head's {G} query heads each, "
                      "seeded order"
                      + (f", layers {layers}" if w.layers > 1 else "")
                      + f"), {per_job * 1e3:.1f} ms each; step time = mean x {jobs_per_step} "
                      + ("jobs (every job of the step timed)" if whole else "jobs (scaled)")
                      + "; numpy float64, one thread")}

    # threads over units
    nproc = os.cpu_count() or 1
    T = max(1, min(nproc, max_threads, len(jobs)))
    if T > 1:
        # the jobs of the first T kv heads (host memory: T kv heads' float64 rows),
        # cycled to about budget_s / 2 seconds of pool time
        sub = jobs[:T]
        cache.clear()
        work = [prepared(j, keep=len(sub)) for j in sub]
        reps = max(1, math.ceil(T * budget_s / 2 / max(per_job, 1e-6) / len(work)))
        with concurrent.futures.ThreadPoolExecutor(T) as pool:
            t0 = time.perf_counter()
            list(pool.map(lambda a_: run(*a_), work * reps))
            wall = time.perf_counter() - t0
        n_thr = len(work) * reps
        del work
        per_step_thr = wall / n_thr * jobs_per_step
        res["threads"] = {"value": round(step_bytes / per_step_thr / 1e9, 6), "unit": "GB/s",
                          "cores": T, "nproc": nproc,
                          "sample": f"{n_thr} jobs ({len(sub)} distinct) over {T} threads, "
                                    f"{wall:.2f} s wall; step time = wall / jobs x "
                                    f"{jobs_per_step}"}
    cache.clear()

    # the append's key encode, on its own
    if w.append:
        inp = layer_inputs(0)
        Ka = inp.k_cache[:, :, w.L - w.append:w.L].double().numpy()
        t0 = time.perf_counter()
        oracle.encode(Ka, w.t)
        res["append_encode_ms"] = round((time.perf_counter() - t0) * 1e3, 2)
    inputs.clear()
    return res


def run_reference(args):
    """--impl reference: the float64 oracle as the reference arm.  Each of the K steps
    is one query head over a contiguous key slice sized so the whole run takes about
    a minute; GB/s is computed over the sample's own algorithmic bytes."""
    w = WORKLOADS[args.config]
    k = args.budget
    t, q, K, V, oracle = oracle_inputs(w)
    G = w.G
    nsteps = args.steps + args.warmup
    # calibrate: seconds per key of one head's decode
    S0 = min(w.L, 4096)
    kc0 = oracle.encode(K[0, 0, :S0], t)
    t0 = time.perf_counter()
    oracle.decode_head(q[0, 0], K[0, 0, :S0], V[0, 0, :S0], k, t, key_codes_rows=kc0)
    per_key = (time.perf_counter() - t0) / S0
    S = int(max(256, min(w.L, 60.0 / max(1, nsteps) / per_key)))
    kcs = {}
    tot = 0.0
    nbytes = 0
    for i in range(nsteps):
        h = i % w.Hq
        kv = h // G
        lo = (i * 7919) % max(1, w.L - S + 1)
        key = (kv, lo)
        if key not in kcs:
            kcs[key] = oracle.encode(K[0, kv, lo:lo + S], t)
        a = time.perf_counter()
        oracle.decode_head(q[0, h], K[0, kv, lo:lo + S], V[0, kv, lo:lo + S], k, t,
                           key_codes_rows=kcs[key])
        b = time.perf_counter()
        if i >= args.warmup:
            tot += b - a
            nbytes += S * 32 + min(k, S) * 2 * 128 * w.elem_bytes + 128 * (w.elem_bytes + 4)
        if len(kcs) > 64:
            kcs.clear()
    gbs = nbytes / tot / 1e9
    return {
        "metric": METRIC, "value": round(gbs, 6), "unit": "GB/s", "impl": "reference",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot / max(1, args.steps) * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": 128, "L": w.L,
                   "k": k, "sample_keys_per_step": S},
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: one query head over {S} consecutive keys "
                                   f"(budget min({k}, {S})), numpy float64, single thread"},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------- main
def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(n: int) -> int:
    """`bench.py --gpus N` without a launcher: re-run this command under
    torch.distributed.run with N local ranks (one GPU each) and return its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def init_ranks(world, local):
    import datetime
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
    torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return backend


def launcher_check(world, local, rank):
    """--launcher-check: the rank set-up and the max-over-ranks reduction alone (no
    kernel runs; gloo when no GPU is visible)."""
    backend = init_ranks(world, local) if world > 1 else "none"
    dev = torch.device("cuda", local) if torch.cuda.is_available() else None
    got = max_over_ranks([1.0 + rank, 10.0 - rank], world, dev)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps({"launcher_check": True, "n_gpus": world, "backend": backend,
                          "max_over_ranks": got}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2, choices=sorted(WORKLOADS))
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--replicas", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config entries of the default line")
    ap.add_argument("--per-config", action="store_true",
                    help="add per_config entries to a non-default line")
    ap.add_argument("--shared", action="store_true",
                    help="shared GQA selection (one top-k per kv head)")
    ap.add_argument("--thresholds", default="fixed", choices=["fixed", "absmax"],
                    help="bucket thresholds: one fixed t, or per-vector 0.5 x absmax")
    ap.add_argument("--cp", type=int, default=0, metavar="W",
                    help="time one rank of a W-way context-parallel step (its L/W slice)")
    ap.add_argument("--paged", type=int, default=0, metavar="PAGE",
                    help="hold the caches in a pool of PAGE-token pages (block tables)")
    ap.add_argument("--policy", default="auto", choices=["auto", "cluster", "flat"],
                    help="decode kernel: the planner's choice, thread-block clusters only, "
                         "or the grid-wide kernel wherever it applies")
    ap.add_argument("--launcher-check", action="store_true",
                    help="only set up the ranks and reduce over them (no kernels)")
    ap.add_argument("--encoder", action="store_true",
                    help="time adamas_encode_keys over the workload's whole key cache "
                         "(one layer) instead of the decode step")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)
    if args.budget is None:
        args.budget = 128 if 128 in WORKLOADS[args.config].budgets else WORKLOADS[args.config].budgets[0]
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(spawn_ranks(args.gpus))
    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch with "
              f"torch.distributed.run --nproc-per-node {args.gpus}, or omit WORLD_SIZE",
              file=sys.stderr)
        sys.exit(2)
    if args.launcher_check:
        launcher_check(world, local, rank)
        return

    if args.impl == "reference":
        # the oracle on rank 0's host cores; other ranks have nothing to run
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import token_level_sparse_fwht_b200 as ad
    ad.set_decode_policy({"auto": ad.POLICY_AUTO, "cluster": ad.POLICY_CLUSTER,
                          "flat": ad.POLICY_FLAT}[args.policy])
    if world > 1:
        init_ranks(world, local)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.encoder:
        r = measure_encoder(args, dev, world)
        if rank == 0:
            print(json.dumps(r), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    default_line = (args.config == 2 and args.budget == 128 and not args.shared
                    and not args.paged and not args.cp and args.thresholds == "fixed")
    r = measure(args, args.config, args.budget, dev, world)
    w, k = r["w"], r["k"]
    peak, peak_kind = peaks()
    per_step_s = r["ms"] / 1e3 / r["K"]
    gbs_rank = aggregate_gbs(r["step_bytes"], per_step_s, 1)
    value = aggregate_gbs(r["step_bytes"], per_step_s, world)
    e2e_step_s = r["ms_e2e"] / 1e3 / r["K2"]
    key = (f"config{args.config}_k{k}" + ("_shared" if args.shared else "")
           + (f"_paged{args.paged}" if args.paged else "")
           + ("_absmax" if args.thresholds == "absmax" else "")
           + (f"_cp{args.cp}" if args.cp else ""))
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": r["K"],
        "warmup": args.warmup,
        "ms_per_step": round(r["ms"] / r["K"], 6),
        "us_per_step": round(per_step_s * 1e6, 3),
        "us_per_step_median_replay": round(r["us_median"], 3),
        "pct_of_roofline": round(100 * gbs_rank / peak, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8-codes/bf16-kv/f32-acc" if w.elem_bytes == 2 else "u8-codes/f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": 128, "L": w.L,
                   "k": k, "algorithmic_bytes_per_step": r["step_bytes"],
                   "selection": "shared per kv head" if args.shared else "per query head",
                   "cache": f"paged, {args.paged}-token pages" if args.paged else "contiguous",
                   "thresholds": ("per-vector 0.5 x absmax" if args.thresholds == "absmax"
                                  else "fixed t"),
                   "context_parallel": (f"one rank of {args.cp}: L/{args.cp} slice, all-gathers "
                                        "stood in for by local copies" if args.cp else None),
                   "replicas": r["R"], "l2": "rotated replicas, working set >= 2x L2",
                   "layers": w.layers, "append_tokens": w.append,
                   "graph": r["use_graph"], "ctas": r["plan"]["ctas"],
                   "kernel": r["kernel"], "policy": args.policy,
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(gbs_rank, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(gbs_rank / peak, 4),
                     "traffic": ncu_traffic(key),
                     "kernel": f"{r['kernel']} (one launch per step)",
                     "peak_source": f"{peak_kind} hbm_gbs"},
        "e2e": {"value": round(aggregate_gbs(r["step_bytes"], e2e_step_s, world), 2), "unit": "GB/s",
                "us_per_step": round(e2e_step_s * 1e6, 3),
                "sync_us_per_step": round(r["sync_us"], 2),
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if r["recall"] is not None:
        line["recall_planted_keys"] = r["recall"]
    if (default_line and not args.no_per_config) or args.per_config:
        entries = []
        for cfg, kk in PER_CONFIG:
            if cfg == args.config and kk == args.budget and default_line:
                entries.append(per_config_entry(r, peak))
                continue
            rr = measure(args, cfg, kk, dev, world, per_config=True)
            entries.append(per_config_entry(rr, peak))
            if rr["append_check"] is not None and rank == 0 and world == 1 \
                    and not args.no_cpu_baseline:
                entries[-1]["cpu_baseline_append"] = cpu_append_baseline(rr["w"],
                                                                         *rr["append_check"])
        line["per_config"] = entries
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, k, shared=args.shared,
                                            absmax=args.thresholds == "absmax")
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
