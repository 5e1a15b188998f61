#!/usr/bin/env python
"""Benchmark of the CSA lightning-indexer top-k on B200.

One step = one call of the C-ABI entry point over one batch of synthetic
inputs resident in HBM: the fused scoring/candidate-filter kernel and the
exact top-k select over its candidate lists.  Prints ONE JSON line on rank 0.
The roofline figure is the fused kernel's own duration, taken from CUDA
events the library records around its launches (csa_set_launch_events).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own
independent batch (weak scaling, no data-path collective); the time is the
max over ranks.  ``--impl reference`` times the CPU oracle on the host cores
over a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

# The V4-Flash-shaped prefill (S=65,536 queries over T=16,384 compressed keys,
# H_I=64, d=128, top-2048, bf16): the shape the >= 60 % tensor-peak target names,
# in the arithmetic (bf16 x bf16) whose dense peak is the roofline.
DEFAULT_CONFIG = "v4flash_prefill"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


# sources of the consumer kernels, which the indexer step does not build on
CONSUMER_SOURCES = ("sparse_attn_kernel.cuh", "union_kernel.cuh")


def kernel_sources_sha() -> str:
    """Hash of the CUDA sources the indexer step is built from (every file
    under csrc/ but the consumer kernels'): a traffic figure measured on
    other sources is stale."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for path in sorted(glob.glob(os.path.join(ROOT, "lightning_indexer_top_02_b200", "csrc", "*"))):
        if os.path.basename(path) in CONSUMER_SOURCES:
            continue
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(config: str, sha: str):
    """DRAM bytes per fused-kernel launch from profiles/traffic.txt (ncu
    dram__bytes_read.sum + dram__bytes_write.sum), or None when no capture of
    these exact sources and this workload is recorded."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 4 and not line.startswith("#") and parts[0] == config \
                        and parts[2] == sha:
                    return int(parts[3])
    except OSError:
        pass
    return None


def measured_fp8_peak(kind: str):
    """E4M3 x E4M3 dense GEMM TFLOP/s measured on this GPU model ("burst" or
    "sustained"), from profiles/peaks_fp8.txt, or None."""
    path = os.path.join(ROOT, "profiles", "peaks_fp8.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == "e4m3" \
                        and parts[1] == kind:
                    return float(parts[2])
    except OSError:
        pass
    return None


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (the job is as slow as its slowest
    rank); the value itself on a single process."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def check_world(gpus: int, world: int):
    """``--gpus N`` must match the process count the launcher started (one
    process per GPU under torchrun); returns an error message, or None."""
    if gpus != world:
        return (f"--gpus {gpus} but {world} process(es) were launched: run one process per GPU, "
                f"e.g. python -m torch.distributed.run --nproc-per-node {gpus} bench.py --gpus {gpus}")
    return None


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, out_path: str, keep: bool = True):
        self.out_path = out_path
        self.proc = None
        self.gpu_id = gpu_id
        self.keep = keep

    def start(self):
        try:
            self.f = open(self.out_path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.out_path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not self.keep:
            try:
                os.unlink(self.out_path)
            except OSError:
                pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j].lower() == "active"})
        loaded = [x for x in sm if smax and x > 0.3 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle leg
def oracle_sample(wl, inputs_cpu, budget_rows: int):
    """Time the oracle on an evenly spaced sample of query rows; returns a dict
    with queries/s extrapolated to the full workload by visible-pair count."""
    import oracle

    oracle.build()
    q, w, k, ks = inputs_cpu
    rows_total = wl.B * wl.S
    n = min(rows_total, budget_rows)
    rows = np.unique(np.linspace(0, rows_total - 1, n).round().astype(np.int64))
    pairs_sample = sum(wl.visible(int(r) % wl.S) for r in rows)
    pairs_total = wl.visible_pairs()
    t0 = time.perf_counter()
    oracle.topk(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m, topk=wl.topk,
                causal=wl.causal, mode=1 if wl.gated else 0, rows=rows)
    dt = time.perf_counter() - t0
    full_time = dt * (pairs_total / max(1, pairs_sample))
    return {"value": rows_total / full_time, "unit": "queries/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} of {rows_total} query rows evenly spaced in t "
                      f"({pairs_sample} of {pairs_total} visible pairs); {dt:.2f} s measured, "
                      f"full-workload time extrapolated by visible-pair count",
            "seconds": dt}


def inputs_for_oracle(wl, inp):
    return workloads.as_numpy_bits(inp)


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import torch

    inp = workloads.make_inputs(wl, device="cpu")
    cpu = inputs_for_oracle(wl, inp)
    rows_per_step = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(wl, cpu, max(8, rows_per_step // 8))
    vals, secs = [], []
    for _ in range(args.steps):
        r = oracle_sample(wl, cpu, rows_per_step)
        vals.append(r["value"])
        secs.append(r["seconds"])
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": "indexer queries/s", "value": value, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * (wl.B * wl.S) / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl),
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": r["cores"],
                         "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    del torch
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl):
    return {"workload": wl.name, "B": wl.B, "S": wl.S, "T": wl.T, "H_I": wl.H, "d": wl.d,
            "m": wl.m, "topk": wl.topk, "causal": wl.causal,
            "keys": "e4m3+fp32 scale" if wl.key_fp8 else "bf16",
            "mode": "sigmoid-gate" if wl.gated else "relu-topk",
            **({"query_pieces": wl.q_pieces} if wl.key_fp8 and wl.q_pieces else {}),
            "values": wl.values, "l2": "flushed between timed steps (256 MiB write)",
            "parallelism": "replicas"}


# ----------------------------------------------------------------------------- consumer leg
def attention_leg(L, wl, out_idx, dev, stream, steps, warmup, peaks=None, HA=64, Dk=128, Dv=128):
    """Sparse attention over the selection the timed indexer steps produced:
    CUDA-event time per call, algorithmic flops (2 HA (Dk + Dv) per selected
    key) and gathered bytes (each selected key's cache row read once per query,
    plus q and the output).  At HA (Dk + Dv) / (Dk + Dv) / 2 ~ HA / 2 flop
    per gathered byte the kernel sits far below the tensor/HBM ridge, so its
    roofline is the gather: gathered bytes / time over the measured HBM copy
    bandwidth (most gathered rows come from L2, so this can exceed 1)."""
    import torch

    g = torch.Generator(device=dev).manual_seed(7)
    qa = torch.randn((wl.B, wl.S, HA, Dk), generator=g, device=dev).to(torch.bfloat16)
    kc = torch.randn((wl.B, wl.T, Dk), generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn((wl.B, wl.T, Dv), generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((wl.B, wl.S, HA, Dv), dtype=torch.float32, device=dev)
    n_sel = int((out_idx >= 0).sum().item())
    for _ in range(warmup):
        L.sparse_attention(qa, kc, out_idx, scale=Dk ** -0.5, v=vc, out=out, stream=stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e0, e1 in ev:
        e0.record(stream)
        L.sparse_attention(qa, kc, out_idx, scale=Dk ** -0.5, v=vc, out=out, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    if L.csa_last_device_error(None) != L.CSA_OK:
        raise SystemExit("device error in the attention leg")
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    flops = 2.0 * HA * (Dk + Dv) * n_sel
    gathered = n_sel * (Dk + Dv) * 2 + qa.numel() * 2 + out.numel() * 4
    gbs = gathered / (ms * 1e-3) / 1e9
    out = {"kernel": "sparse_attn_kernel", "heads": HA, "Dk": Dk, "Dv": Dv,
           "selected_keys": n_sel, "ms": ms, "tflops": flops / (ms * 1e-3) / 1e12,
           "gathered_gbs": gbs, "queries_per_s": wl.B * wl.S / (ms * 1e-3)}
    if peaks and peaks.get("hbm_gbs"):
        out["roofline"] = {"bound": "gather (hbm)", "achieved": gbs, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                           "bytes_per_launch": gathered, "flops_per_launch": flops}
    return out


def schedules_leg(L, dev, steps, warmup, n_layers=4, HA=64, Dk=128, Dv=128):
    """One decode step of n_layers layers under each cross-layer schedule of
    ``schedule.py`` ("own": every layer runs its own indexer then its sparse
    attention; "mli": a layer's attention reads the previous layer's selection
    while its own indexer runs for the next layer on a second stream;
    "indexcache": the indexer on every second layer).  The indexer shape is
    decode1_fp8's (32 sequences, one query each, 131,072 E4M3 keys); the
    attention reads 128-dim bf16 key and value caches of the same length.
    CUDA-event time of the whole step on the main stream."""
    import torch
    from lightning_indexer_top_02_b200 import schedule as sched

    wl = workloads.CONFIGS["decode1_fp8"]
    layers = []
    for li in range(n_layers):
        inp = workloads.make_inputs(wl, device=dev, seed=wl.seed + 17 * (li + 1))
        g = torch.Generator(device=dev).manual_seed(100 + li)
        layers.append(sched.Layer(
            iq=inp["q"], iw=inp["w"], ik=inp["k"], ik_scale=inp["k_scale"],
            aq=torch.randn((wl.B, wl.S, HA, Dk), generator=g, device=dev).to(torch.bfloat16),
            kc=torch.randn((wl.B, wl.T, Dk), generator=g, device=dev).to(torch.bfloat16),
            vc=torch.randn((wl.B, wl.T, Dv), generator=g, device=dev).to(torch.bfloat16),
            scale=Dk ** -0.5))
    main = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    out = {"layers": n_layers, "indexer": wl.name, "attention": {"heads": HA, "Dk": Dk, "Dv": Dv}}
    for name in ("own", "mli", "indexcache"):
        for _ in range(warmup):
            sched.decode_layers(layers, m=wl.m, topk=wl.topk, schedule=name, main=main, side=side)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for _ in range(steps):
            sched.decode_layers(layers, m=wl.m, topk=wl.topk, schedule=name, main=main, side=side)
        e1.record(main)
        torch.cuda.synchronize(dev)
        if L.csa_last_device_error(None) != L.CSA_OK:
            raise SystemExit(f"device error in the {name} schedule")
        out[name + "_ms_per_step"] = e0.elapsed_time(e1) / steps
    out["mli_speedup_over_own"] = out["own_ms_per_step"] / out["mli_ms_per_step"]
    out["indexcache_speedup_over_own"] = out["own_ms_per_step"] / out["indexcache_ms_per_step"]
    return out


def sharded_leg(L, wl, inp, world, steps, warmup):
    """Key-sharded selection (``sharded.py``) of this workload over ``world``
    contiguous key ranges, one rank's share timed on this GPU: its range's
    selection (k_local keys per query) and the exact merge of all ``world``
    lists, against the unsharded call.  The lists' all-gather crosses NVLink on
    real ranks; its size is reported, not timed.  Recall of the merged
    selection against the unsharded one for exact (k_local = k) and relaxed
    (k / 2, k / 4) local selections."""
    import numpy as np
    import torch
    from lightning_indexer_top_02_b200 import sharded

    q, w, k, ks = inp["q"], inp["w"], inp["k"], inp["k_scale"]
    mode = 1 if wl.gated else 0

    def timed(fn, batches=5):
        # the median over batches of `steps` calls: a sporadic slow call
        # (allocator, another job on the host) does not set the figure
        for _ in range(warmup):
            r = fn()
        torch.cuda.synchronize()
        times = []
        for _ in range(batches):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                r = fn()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / steps)
        return statistics.median(times), r

    full_ms, (full, _) = timed(lambda: L.indexer_topk(q, w, k, k_scale=ks, m=wl.m, topk=wl.topk,
                                                      causal=wl.causal, mode=mode))
    f = full.cpu().numpy().reshape(-1, wl.topk)
    out = {"ranks": world, "unsharded_ms": full_ms, "variants": []}
    for k_local in (wl.topk, wl.topk // 2, wl.topk // 4):
        li, ls, offs, local_ms = [], [], [], []
        for r in range(world):
            a, b = sharded.shard_range(wl.T, world, r)
            kr = k[:, a:b].contiguous()
            ksr = ks[:, a:b].contiguous() if ks is not None else None
            ms, (i, sc) = timed(lambda: sharded.select_local(
                q, w, kr, start=a, T_total=wl.T, m=wl.m, k_local=k_local, k_scale=ksr,
                causal=wl.causal, mode=mode))
            li.append(i)
            ls.append(sc)
            offs.append(a)
            local_ms.append(ms)
        merge_ms, (gi, _) = timed(lambda: sharded.merge_topk(li, ls, offs, wl.topk))
        g = gi.cpu().numpy().reshape(-1, wl.topk)
        rec = np.array([1.0 if np.sum(f[r] >= 0) == 0 and np.sum(g[r] >= 0) == 0 else
                        len(np.intersect1d(g[r][g[r] >= 0], f[r][f[r] >= 0])) / max(1, np.sum(f[r] >= 0))
                        for r in range(g.shape[0])])   # a row empty in both counts as 1
        per_rank_ms = max(local_ms) + merge_ms
        out["variants"].append({
            "k_local": k_local, "local_select_ms_max": max(local_ms), "merge_ms": merge_ms,
            "per_rank_ms_without_exchange": per_rank_ms,
            "speedup_over_unsharded": full_ms / per_rank_ms,
            "exchange_bytes_per_rank": int(li[0].numel() * 8 * (world - 1)),
            "recall_mean": float(rec.mean()), "recall_min": float(rec.min())})
    return out


# ----------------------------------------------------------------------------- GPU leg
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-rows", type=int, default=256,
                    help="query rows the oracle computes per reference step")
    ap.add_argument("--cpu-rows", type=int, default=512,
                    help="query rows of the CPU-baseline sample (rank 0)")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a workload field (B, S, T, H, d, m, topk, seed, causal, "
                         "key_fp8, gated, q_pieces, num_splits), e.g. for a reduced profiling shape; "
                         "the workload name records it")
    ap.add_argument("--clocks-csv", default="",
                    help="keep the raw nvidia-smi clock samples of the timed region here")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attention", action="store_true",
                    help="also time the sparse-attention consumer over the step's selection "
                         "(HA=64 heads by default, Dk=Dv=128, bf16; reported under 'consumer')")
    ap.add_argument("--attention-heads", type=int, default=64,
                    help="heads of the attention consumer (--attention); up to 64 heads split each "
                         "tile's keys over warp pairs, more use one thread per head row")
    ap.add_argument("--schedules", action="store_true",
                    help="also time a 4-layer decode step under the cross-layer schedules "
                         "(own / mli / indexcache; reported under 'schedules')")
    ap.add_argument("--sharded", type=int, default=0, metavar="W",
                    help="also time key-sharded selection over W key ranges, one rank's share on "
                         "this GPU, with the recall of relaxed local selections ('sharded')")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    wl = workloads.CONFIGS[args.config]
    if args.set:
        kw = {}
        for item in args.set:
            field, _, value = item.partition("=")
            if field not in ("B", "S", "T", "H", "d", "m", "topk", "seed", "causal", "key_fp8",
                             "gated", "q_pieces", "num_splits"):
                raise SystemExit(f"--set: unknown field {field!r}")
            flag = field in ("causal", "key_fp8", "gated")
            kw[field] = (value.lower() in ("1", "true")) if flag else int(value)
        wl = wl.replace(name=wl.name + "[" + ",".join(args.set) + "]", **kw)

    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    import torch.distributed as dist

    import lightning_indexer_top_02_b200 as L

    rank, world, local = dist_env()
    err = check_world(args.gpus, world)
    if err:
        raise SystemExit(err)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    L.load_library()
    stream = torch.cuda.current_stream(dev)

    inp = workloads.make_inputs(wl, device=dev, seed=wl.seed + 1000 * rank)
    q, w, k, ks = inp["q"], inp["w"], inp["k"], inp["k_scale"]
    out_idx = torch.empty((wl.B, wl.S, wl.topk), dtype=torch.int32, device=dev)
    out_sc = torch.empty((wl.B, wl.S, wl.topk), dtype=torch.float32, device=dev)
    mode = 1 if wl.gated else 0
    a = L.make_args(q, w, k, k_scale=ks, m=wl.m, topk=wl.topk, causal=wl.causal, mode=mode,
                    query_pieces=wl.q_pieces, num_splits=wl.num_splits, out_idx=out_idx,
                    out_score=out_sc)
    plan = L.csa_indexer_plan(a)
    ws_bytes = plan.workspace_bytes
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    import ctypes
    sptr = ctypes.c_void_p(stream.cuda_stream)
    wsptr = ctypes.c_void_p(ws.data_ptr())

    def step():
        st = L.csa_indexer_topk_ex(a, wsptr, ws_bytes, sptr)
        if st != L.CSA_OK:
            raise L.CsaError(st, "csa_indexer_topk_ex")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if L.csa_last_device_error(sptr) != L.CSA_OK:
        raise SystemExit("device error during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # events around each kernel launch of each step (fused, select, end)
    n_marks = plan.launches + 1
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks)]
             for _ in range(args.steps)]
    for row in marks:
        for e in row:
            e.record(stream)  # creates the event
    torch.cuda.synchronize(dev)
    sampler = None
    if rank == 0:
        props = torch.cuda.get_device_properties(dev)
        gid = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
        clocks_csv = args.clocks_csv
        if not clocks_csv:
            import tempfile
            fd, clocks_csv = tempfile.mkstemp(prefix="bench_clocks_", suffix=".csv")
            os.close(fd)
        sampler = ClockSampler(gid, clocks_csv, keep=bool(args.clocks_csv))
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        L.csa_set_launch_events(marks[i])
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    L.csa_set_launch_events(None)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    if L.csa_last_device_error(sptr) != L.CSA_OK:
        raise SystemExit("device error during the timed region")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    # per launch chunk: fused kernel between marks 2c and 2c+1, select between 2c+1 and 2c+2
    fused_ms = [sum(row[2 * c].elapsed_time(row[2 * c + 1]) for c in range(plan.launches // 2))
                for row in marks]
    select_ms = [sum(row[2 * c + 1].elapsed_time(row[2 * c + 2])
                     for c in range(plan.launches // 2)) for row in marks]
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    queries = wl.B * wl.S
    value = queries * world / (ms_per_step / 1000.0)
    flops = wl.flops()
    tflops = flops / (ms_per_step / 1000.0) / 1e12

    # ---- end to end through the C ABI with host buffers (pinned), copies timed.
    # Every step uploads its inputs from pinned host memory and reads its
    # results back; as in a serving loop, step i+1's upload and step i-1's
    # read-back run on copy streams beside step i's kernels (two device buffer
    # sets, one per step parity; the kernels share the workspace in order).
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hw = w.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hks = ks.cpu().pin_memory() if ks is not None else None
        h2d = hq.numel() * hq.element_size() + hw.numel() * 4 + hk.numel() * hk.element_size() + (
            hks.numel() * 4 if hks is not None else 0)
        bufs = []
        for j in range(2):
            if j == 0:
                dq, dw, dk, dks, doi, dos = q, w, k, ks, out_idx, out_sc
            else:
                dq, dw, dk = torch.empty_like(q), torch.empty_like(w), torch.empty_like(k)
                dks = torch.empty_like(ks) if ks is not None else None
                doi, dos = torch.empty_like(out_idx), torch.empty_like(out_sc)
            aj = L.make_args(dq, dw, dk, k_scale=dks, m=wl.m, topk=wl.topk, causal=wl.causal,
                             mode=mode, query_pieces=wl.q_pieces, out_idx=doi, out_score=dos)
            hidx = torch.empty(out_idx.shape, dtype=torch.int32).pin_memory()
            hsc = torch.empty(out_sc.shape, dtype=torch.float32).pin_memory()
            bufs.append((dq, dw, dk, dks, doi, dos, aj, hidx, hsc))
        d2h = bufs[0][7].numel() * 4 + bufs[0][8].numel() * 4
        up = torch.cuda.Stream(dev)
        down = torch.cuda.Stream(dev)
        k_done = [torch.cuda.Event() for _ in range(2)]
        dn_done = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            dq, dw, dk, dks, doi, dos, aj, hidx, hsc = bufs[i & 1]
            up_done = torch.cuda.Event()
            with torch.cuda.stream(up):
                if used[i & 1]:
                    up.wait_event(k_done[i & 1])      # the last kernel on this set read its inputs
                dq.copy_(hq, non_blocking=True)
                dw.copy_(hw, non_blocking=True)
                dk.copy_(hk, non_blocking=True)
                if hks is not None:
                    dks.copy_(hks, non_blocking=True)
                up_done.record(up)
            stream.wait_event(up_done)
            if used[i & 1]:
                stream.wait_event(dn_done[i & 1])     # its outputs were read back
            st = L.csa_indexer_topk_ex(aj, wsptr, ws_bytes, sptr)
            if st != L.CSA_OK:
                raise L.CsaError(st, "csa_indexer_topk_ex")
            k_done[i & 1].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(k_done[i & 1])
                hidx.copy_(doi, non_blocking=True)
                hsc.copy_(dos, non_blocking=True)
                dn_done[i & 1].record(down)
            used[i & 1] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        for i in range(n_e2e):
            e2e_step(i)
        for j in range(2):
            stream.wait_event(dn_done[j])             # every read-back is inside the region
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dev)

        # The same steps in series on one stream: upload, call, read-back, with
        # nothing overlapped (the latency of one request through the C ABI).
        dq, dw, dk, dks, doi, dos, aj, hidx, hsc = bufs[0]
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        s0.record(stream)
        for i in range(n_e2e):
            dq.copy_(hq, non_blocking=True)
            dw.copy_(hw, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            if hks is not None:
                dks.copy_(hks, non_blocking=True)
            st = L.csa_indexer_topk_ex(aj, wsptr, ws_bytes, sptr)
            if st != L.CSA_OK:
                raise L.CsaError(st, "csa_indexer_topk_ex")
            hidx.copy_(doi, non_blocking=True)
            hsc.copy_(dos, non_blocking=True)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        serial_ms = max_over_ranks(s0.elapsed_time(s1) / n_e2e, dev)
        e2e = {"value": queries * world / (e_ms / 1000.0), "unit": "queries/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_ms,
               "pipelined": "each step's upload and read-back overlap the neighbouring steps' "
                            "kernels on two copy streams (serving loop)",
               "serial": {"value": queries * world / (serial_ms / 1000.0), "unit": "queries/s",
                          "ms_per_step": serial_ms,
                          "what": "upload, call and read-back of each step in series on one stream"}}

    consumer = attention_leg(L, wl, out_idx, dev, stream, args.steps, args.warmup, load_peaks()[0],
                             HA=args.attention_heads) \
        if args.attention else None
    schedules = schedules_leg(L, dev, args.steps, args.warmup) if args.schedules and rank == 0 else None
    sharded_res = sharded_leg(L, wl, inp, args.sharded, args.steps, args.warmup) \
        if args.sharded > 1 and rank == 0 else None

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    timed_s = total_ms / 1000.0
    sustained = timed_s > 0.5
    peak = peaks.get("bf16_tflops_sustained" if sustained else "bf16_tflops")
    peak_name = f"{peak_src} bf16 dense ({'sustained' if sustained else 'burst'})"
    fp8_measured = None
    if wl.key_fp8 and peak:
        # E4M3 x E4M3 MMAs: the FP8 peak is the measured bf16 one times the
        # nominal dense ratio (4.5 / 2.25 PFLOP/s).  A directly measured E4M3
        # GEMM figure (profiles/peaks_fp8.txt) is reported beside it.
        peak = 2.0 * peak
        peak_name += " x 2 (nominal FP8 / bf16 ratio)"
        fp8_measured = measured_fp8_peak("sustained" if sustained else "burst")
    fused_avg = statistics.mean(fused_ms)
    step_avg = statistics.mean([f + s_ for f, s_ in zip(fused_ms, select_ms)])
    k_tflops = flops / (fused_avg / 1000.0) / 1e12
    sha = kernel_sources_sha()
    alg_bytes = wl.input_bytes() + wl.output_bytes()
    ridge = (peak or peaks["bf16_tflops"]) * 1e12 / (peaks["hbm_gbs"] * 1e9)
    common = {"traffic": measured_traffic(wl.name, sha),
              "kernel": "indexer_topk_kernel (fused scoring + candidate cut)",
              "kernel_ms": fused_avg, "select_kernel_ms": statistics.mean(select_ms),
              "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": alg_bytes,
              "tensor_flops_executed_per_launch": (2 if wl.key_fp8 and wl.q_pieces != 1 else 1) * flops,
              "step_kernels_ms": step_avg,
              "sources_sha": sha}
    if flops / alg_bytes < ridge:
        # few queries per key (single-query decode): the key stream bounds it
        gbs = alg_bytes / (fused_avg / 1000.0) / 1e9
        step_gbs = alg_bytes / (step_avg / 1000.0) / 1e9
        roofline = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_src} copy bandwidth",
                    "step_achieved": step_gbs, "step_frac": step_gbs / peaks["hbm_gbs"],
                    **common}
    else:
        step_tflops = flops / (step_avg / 1000.0) / 1e12
        roofline = {"bound": "tensor", "achieved": k_tflops, "peak": peak, "unit": "TFLOP/s",
                    "frac": k_tflops / peak if peak else None, "peak_source": peak_name,
                    "step_achieved": step_tflops,
                    "step_frac": step_tflops / peak if peak else None,
                    **common}
        if fp8_measured:
            roofline["fp8_measured_peak"] = fp8_measured
            roofline["frac_of_fp8_measured"] = k_tflops / fp8_measured
    cpu = None
    if not args.no_cpu_baseline:
        cpu_inputs = inputs_for_oracle(wl, {"q": q, "w": w, "k": k, "k_scale": ks})
        r = oracle_sample(wl, cpu_inputs, args.cpu_rows)
        cpu = {k_: r[k_] for k_ in ("value", "unit", "cores", "kind", "sample")}

    line = {
        "metric": "indexer queries/s", "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3 keys x one e4m3 query piece, fp32 accumulate" if wl.q_pieces == 1 else
                  "e4m3 keys x e4m3 query pieces, fp32 accumulate") if wl.key_fp8 else "bf16",
        "data": "synthetic", "config": config_dict(wl), "tflops": tflops,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": args.steps * plan.launches,
        **({"consumer": consumer} if consumer else {}),
        **({"schedules": schedules} if schedules else {}),
        **({"sharded": sharded_res} if sharded_res else {}),
        "plan": plan.as_dict(),
        # extra device memory of the call: the caller's workspace (candidate lists
        # and per-CTA score buffers, O(S*k)); the library allocates nothing else
        "extra_memory": {"bytes": int(ws_bytes),
                         "materialised_scores_bytes": int(wl.B * wl.S * wl.H * wl.T * 4),
                         "per_query_bytes": ws_bytes / float(wl.B * wl.S)},
        "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms),
                    "max": max(step_ms)},
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
