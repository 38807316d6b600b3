"""Benchmark of the DAM structured-sparse-attention hot path on B200.

The timed step is the prefill call itself, sparse_attn_fwd (stripe gather + tcgen05
attention forward) over one synthetic layer; `value` is its tokens/s.  The whole path
(sparse_pattern_capture of the layer's 32 averaged maps at L = 512, the fill pass of
sparse_pattern_extend, sparse_attn_fwd) is timed as well and reported under "path".
The default workload is the LLaMA-3-8B-shaped layer at S = 65536 (32 Q / 8 KV heads,
d = 128, per head 1024 contiguous diagonals at a random offset + 128 random columns).
The sizing pass of sparse_pattern_extend (an allocation-size query) runs once at set-up.

Prints ONE JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun), each rank
runs an independent replica (weak scaling), time = max over ranks.
`--impl reference` times the CPU oracle instead (on the host cores, bounded sample).
"""

from __future__ import annotations

import argparse
import itertools
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from structured_sparse_attention_b200 import inputs  # noqa: E402

METRIC = "sparse-attn prefill tokens/s & effective TFLOP/s vs roofline, per mask density"
UNIT = "tokens/s"

# Kernels launched per call (the library's own kernels).
LAUNCHES = {"capture": 3, "extend_fill": 9, "attn": 2}  # library kernels per call of each stage

WORKLOADS = {
    # name: (H_q, H_kv, S, d, pattern builder)
    "llama3-8b-layer-64k": (32, 8, 65536, 128, lambda: inputs.patterns_band_random(inputs.SEED_BASE + 4)),
    "llama3.2-1b-layer-16k": (32, 8, 16384, 64, lambda: inputs.patterns_gqa_16k(inputs.SEED_BASE + 3)),
    # small case of the 8B layer (same pattern rule at S = 16384) for profiler captures
    "llama3-8b-layer-16k": (32, 8, 16384, 128,
                            lambda: inputs.patterns_band_random(inputs.SEED_BASE + 6, S=16384)),
    "long-104k-0.5pct": (24, 8, 104000, 128, lambda: inputs.patterns_density(inputs.SEED_BASE + 5, "0.5")),
    "long-104k-2pct": (24, 8, 104000, 128, lambda: inputs.patterns_density(inputs.SEED_BASE + 5, "2")),
    "long-104k-10pct": (24, 8, 104000, 128, lambda: inputs.patterns_density(inputs.SEED_BASE + 5, "10")),
    "long-104k-100pct": (24, 8, 104000, 128, lambda: inputs.patterns_density(inputs.SEED_BASE + 5, "100")),
}
# Decoding step (one new query per sequence at the last position of its cache):
# name: (B, H_q, H_kv, S_cache, d, pattern builder)
DECODE_WORKLOADS = {
    "decode-llama3-8b-16k-b16": (16, 32, 8, 16384, 128,
                                 lambda: inputs.patterns_band_random(inputs.SEED_BASE + 7, S=16384)),
}
SEEDS = {"llama3-8b-layer-64k": inputs.SEED_BASE + 4, "llama3.2-1b-layer-16k": inputs.SEED_BASE + 3,
         "llama3-8b-layer-16k": inputs.SEED_BASE + 6}
CAPTURE_MAPS = 32  # one layer's heads
# Stage-one map production: n_maps (layers x heads), samples B, capture length L, d
MAPS_WORKLOADS = {
    "maps-llama3.2-1b-l512-b16": (512, 16, 512, 64),
}
MUFU_EX2_PER_CLK_SM = 16  # B200: ex2.approx results per clock per SM (microbenchmark: 15.99)


def sm_max_mhz():
    """clocks.max.sm of the machine's B200s (MEASURED_PEAKS.json, else the nominal 1965 MHz)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p)).get("sm_max_mhz", 1965.0))
    return 1965.0
CAPTURE_L = 512


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def profiled_traffic(workload):
    """DRAM bytes per attention launch from the ncu record of this workload
    (profiles/sparse_attn_fwd_<workload>_dram.json), if the attention sources are still
    the ones it was taken on (else None)."""
    path = os.path.join(ROOT, "profiles", f"sparse_attn_fwd_{workload}_dram.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    if rec.get("source_sha256_16") != attn_source_hash():
        return None
    try:
        return float(rec["traffic_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


def attn_source_hash():
    """First 16 hex digits of the sha256 of the attention sources (attn_fwd.cu, common.cuh)."""
    import hashlib
    csrc = os.path.join(ROOT, "structured_sparse_attention_b200", "csrc")
    h = hashlib.sha256()
    for f in ("attn_fwd.cu", "common.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def nnz_per_head(diags, verts, S):
    """Retained pairs per head of the extended mask, from the list form (integer counting)."""
    out = []
    for D, Cc in zip(diags, verts):
        D = np.asarray(D, np.int64)
        Cc = np.asarray(Cc, np.int64)
        D = D[D < S]
        Cc = Cc[Cc < S]
        total = int((S - D).sum()) + int((S - Cc).sum())
        if len(D) and len(Cc):
            # a cell (c + r, c) lies on both a column and a diagonal: count it once
            shared = np.searchsorted(np.sort(D), S - Cc, side="left").sum()
            total -= int(shared)
        out.append(total)
    return np.array(out, np.int64)


# Stage one at full size: the averaged maps of 16 layers x 32 heads at L = 512 (B = 16
# samples averaged), captured with lambda = 0.5, tau = 0.3, mu = 0.8.
CAPTURE_WORKLOADS = {
    "capture-512maps-l512": (512, 512),  # maps, L
}


def run_capture(args):
    """Time sparse_pattern_capture alone on one GPU: maps/s and the achieved HBM bandwidth
    of the causal half of every map (the bytes the capture must read) against the measured
    copy peak.  The maps (537 MB) exceed L2, and L2 is flushed between timed calls."""
    import torch

    import structured_sparse_attention_b200 as ssa
    n, L = CAPTURE_WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    seed = inputs.SEED_BASE + 2
    maps_h = inputs.averaged_maps(seed, n, L=L, n_samples=16)
    h_maps = torch.from_numpy(maps_h).pin_memory()
    maps = h_maps.to(dev)
    ws = torch.empty(max(ssa.load().sparse_pattern_capture_ws_bytes(n, L), 16), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = ssa.capture(maps, ws=ws, status=status)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        ssa.capture(maps, out=out, ws=ws, status=status, check=False)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0")
    sampler.start()
    time.sleep(0.3)
    for e0, e1 in ev:
        flush.fill_(1)  # evict the maps from L2 (not timed)
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    kept = int(out["diag_ptr"][-1].item()) + int(out["vert_ptr"][-1].item())
    # end to end: the maps in from pinned host memory, the four lists back
    outs_h = {k_: torch.empty(out[k_].shape, dtype=out[k_].dtype).pin_memory()
              for k_ in ("diag_ptr", "diag_offsets", "vert_ptr", "vert_cols")}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(3, min(args.steps, 10))
    e0.record()
    for _ in range(e_steps):
        maps.copy_(h_maps, non_blocking=True)
        call()
        for k_, t_ in outs_h.items():
            t_.copy_(out[k_], non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1) / e_steps
    algo_bytes = n * 4 * L * (L + 1) // 2  # the causal half of every map, read once
    hbm_gbs, _, _, peak_kind = load_peaks()
    achieved = algo_bytes / (ms / 1e3) / 1e9
    line = {"metric": "stage-one pattern capture maps/s & achieved HBM GB/s vs roofline", "value": n / (ms / 1e3),
            "unit": "maps/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "n_maps": n, "L": L, "lambda": 0.5, "tau": 0.3, "mu": 0.8,
                       "eps": 1e-8, "kept_patterns": kept,
                       "l2": "maps (%.0f MB) larger than L2, and L2 flushed between timed calls" % (n * L * L * 4 / 1e6)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": None, "peak_source": f"{peak_kind} (copy)",
                         "kernel": "sparse_pattern_capture (hits + select + pack)",
                         "algorithmic": {"bytes": algo_bytes, "what": "the causal half of every map, fp32"}},
            "clocks": clocks,
            "e2e": {"value": n / (e_ms / 1e3), "unit": "maps/s", "h2d_bytes_per_step": int(h_maps.numel() * 4),
                    "d2h_bytes_per_step": int(sum(t_.numel() * 4 for t_ in outs_h.values())), "ms_per_step": e_ms},
            "gpu_launches": LAUNCHES["capture"] * args.steps, "cpu_baseline": None}
    if not args.no_cpu_baseline:
        from oracle import oracle as ora
        ora.build()
        cores = len(os.sched_getaffinity(0))
        n_cpu = min(n, max(16, cores))
        t0 = time.perf_counter()
        ora.capture(maps_h[:n_cpu])
        cpu_s = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n_cpu / cpu_s, "unit": "maps/s", "cores": cores, "kind": "oracle",
                                "sample": f"the first {n_cpu} of the {n} maps, fp64 scalar oracle"}
    print(json.dumps(line), flush=True)


# Sensitivity of stage one to its free parameters (lambda, tau, mu): the referee's
# missing analysis, run with the library's capture and the extension to S.
SWEEP_WORKLOADS = {
    "capture-sweep-128maps-l512": (128, 512, 65536),  # maps, L, S of the extended mask
}
SWEEP_GRID = {"scaling": ("row", "map"), "lam": (0.0, 0.25, 0.5, 1.0, 2.0), "tau": (0.1, 0.2, 0.3, 0.4, 0.5),
              "mu": (0.6, 0.7, 0.8, 0.9)}


def capture_sweep(capture, planted, S, grid=SWEEP_GRID):
    """For every (scaling, lambda, tau, mu) of `grid`: the kept diagonals and columns per map,
    the recall and precision of the planted patterns, and the density of the extended mask
    at S (retained pairs / causal pairs, mean over maps).  `capture(lam, tau, mu, scaling)`
    returns the host CSR lists (diag_ptr, diag_offsets, vert_ptr, vert_cols) of the maps
    whose planted (diagonals, columns) are `planted`; scaling is "row" (each row scaled to
    [0, 1] by its own causal min and max) or "map" (by the map's), default ("row",)."""
    n = len(planted)
    causal = S * (S + 1) / 2
    rows = []
    for scaling, lam, tau, mu in itertools.product(grid.get("scaling", ("row",)), grid["lam"], grid["tau"],
                                                   grid["mu"]):
        dp, do, vp, vc = (np.asarray(a) for a in capture(lam, tau, mu, scaling))
        diags = [do[dp[m]:dp[m + 1]] for m in range(n)]
        verts = [vc[vp[m]:vp[m + 1]] for m in range(n)]
        tp = fp = fn = 0
        for m in range(n):
            pd, pc = set(np.asarray(planted[m][0]).tolist()), set(np.asarray(planted[m][1]).tolist())
            kd, kc = set(diags[m].tolist()), set(verts[m].tolist())
            tp += len(pd & kd) + len(pc & kc)
            fp += len(kd - pd) + len(kc - pc)
            fn += len(pd - kd) + len(pc - kc)
        dens = nnz_per_head(diags, verts, S) / causal
        rows.append({"scaling": scaling, "lam": lam, "tau": tau, "mu": mu,
                     "diags_per_map": float(np.mean([len(x) for x in diags])),
                     "cols_per_map": float(np.mean([len(x) for x in verts])),
                     "recall": tp / max(tp + fn, 1), "precision": tp / max(tp + fp, 1),
                     "density_at_S": float(dens.mean())})
    return rows


def run_capture_sweep(args):
    """Time the library's capture over the (scaling, lambda, tau, mu) grid on synthetic averaged maps
    and report what each setting keeps (one JSON line; the capture kernels are HBM-bound)."""
    import torch

    import structured_sparse_attention_b200 as ssa
    n, L, S = SWEEP_WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    seed = inputs.SEED_BASE + 2
    maps_h = inputs.averaged_maps(seed, n, L=L, n_samples=16)
    planted = inputs.planted_map_patterns(seed, n, L)
    maps = torch.from_numpy(maps_h).to(dev)
    ws = torch.empty(max(ssa.load().sparse_pattern_capture_ws_bytes(n, L), 16), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = ssa.capture(maps, ws=ws, status=status)
    times = []

    def capture(lam, tau, mu, scaling):
        for _ in range(args.warmup):
            ssa.capture(maps, lam=lam, tau=tau, mu=mu, scaling=scaling, out=out, ws=ws, status=status)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            ssa.capture(maps, lam=lam, tau=tau, mu=mu, scaling=scaling, out=out, ws=ws, status=status,
                        check=False)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / args.steps)
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())}")
        return [out[k].cpu().numpy() for k in ("diag_ptr", "diag_offsets", "vert_ptr", "vert_cols")]

    rows = capture_sweep(capture, planted, S)
    ms = float(np.mean(times))
    hbm_gbs, _, _, peak_kind = load_peaks()
    algo_bytes = n * 4 * L * (L + 1) // 2  # the causal half of every map, read once
    line = {"metric": "stage-one sensitivity sweep: kept patterns, planted recall/precision, extended density",
            "value": n / (ms / 1e3), "unit": "maps/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload, "n_maps": n, "L": L, "S": S, "grid": SWEEP_GRID},
            "roofline": {"bound": "hbm", "achieved": algo_bytes / (ms / 1e3) / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": algo_bytes / (ms / 1e3) / 1e9 / hbm_gbs, "traffic": None,
                         "kernel": "capture (hits + select + pack)", "peak_source": peak_kind},
            "sweep": rows, "e2e": None, "gpu_launches": 3 * args.steps * len(rows), "cpu_baseline": None}
    print(json.dumps(line), flush=True)


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.index = gpu_id  # nvidia-smi --id value (PCI bus id of the device in use)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return rank, world, local, dist
    return 0, 1, 0, None


def max_over_ranks(x: float, dist, device):
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------
# CPU oracle leg
# ------------------------------------------------------------------------------------

def oracle_leg(workload, budget_s=15.0, maps=None):
    """Time the oracle as it stands on a bounded sample of the workload: the attention
    rows of randomly drawn query rows (all heads), grown until `budget_s` seconds of
    work; tokens/s is extrapolated to all S rows.  The capture of the layer's maps and
    the extension are timed in full and reported beside it.  Returns (tokens/s,
    description dict)."""
    from oracle import oracle as ora
    Hq, Hkv, S, d, builder = WORKLOADS[workload]
    diags, verts = builder()
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    # capture of the layer's maps, timed in full
    if maps is None:
        maps = inputs.averaged_maps(inputs.SEED_BASE + 2, CAPTURE_MAPS, L=CAPTURE_L, n_samples=16)
    t0 = time.perf_counter()
    ora.capture(maps)
    t_cap = time.perf_counter() - t0
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)
    t0 = time.perf_counter()
    ext = ora.extend(dp, do, vp, vo, S)
    t_ext = time.perf_counter() - t0
    # attention on sampled rows, growing the sample until the budget is spent
    q, k, v = inputs.qkv(SEEDS.get(workload, inputs.SEED_BASE + 5), Hq, Hkv, S, d)
    g = np.random.default_rng(7)
    n_rows, t_rows, done = 8, 0.0, 0
    while t_rows < budget_s and done < S:
        rows = np.sort(g.choice(S, size=min(n_rows, S), replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        ora.attn_rows(q, k, v, ext, d ** -0.5, rows)
        t_rows += time.perf_counter() - t0
        done += len(rows)
        n_rows *= 2
    t_attn = t_rows * (S / done)  # extrapolated to all S rows
    desc = {"kind": "oracle", "cores": int(os.environ.get("OMP_NUM_THREADS", cores)),
            "extrapolated": True, "rows_timed": int(done), "seconds_timed": round(t_rows, 3),
            "sample": f"attention on {done} random query rows x {Hq} heads ({t_rows:.1f} s of oracle work), "
                      f"extrapolated to S={S} rows; capture of {CAPTURE_MAPS} maps at L={CAPTURE_L} "
                      f"({t_cap:.2f} s) and the extension ({t_ext:.2f} s) timed in full, not in the value",
            "path_tokens_per_s_extrapolated": S / (t_cap + t_ext + t_attn)}
    return S / t_attn, desc


# ------------------------------------------------------------------------------------
# GPU leg
# ------------------------------------------------------------------------------------

def run_gpu(args, rank, world, local, dist):
    import torch

    import structured_sparse_attention_b200 as ssa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    Hq, Hkv, S, d, builder = WORKLOADS[args.workload]
    diags, verts = builder()
    seed = SEEDS.get(args.workload, inputs.SEED_BASE + 5)

    # ---------------- inputs (host, then resident in HBM) ----------------
    maps_h = inputs.averaged_maps(inputs.SEED_BASE + 2, CAPTURE_MAPS, L=CAPTURE_L, n_samples=16)
    q_h, k_h, v_h = inputs.qkv(seed, Hq, Hkv, S, d)
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)

    def pinned(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dtype is not None:
            t = t.view(dtype)
        return t.pin_memory()

    h_maps = pinned(maps_h)
    h_q, h_k, h_v = (pinned(a.view(np.int16), torch.bfloat16) for a in (q_h, k_h, v_h))
    h_lists = [pinned(a.astype(np.int32)) for a in (dp, do, vp, vo)]
    maps = h_maps.to(dev)
    q, k, v = h_q.to(dev), h_k.to(dev), h_v.to(dev)
    lists = [t.to(dev) for t in h_lists]
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    cap_out = ssa.capture(maps)  # allocates outputs once
    cap_ws = torch.empty(ssa.load().sparse_pattern_capture_ws_bytes(CAPTURE_MAPS, CAPTURE_L),
                         dtype=torch.uint8, device=dev)
    plan = ssa.extend(*lists, S)  # sizing pass + first fill (allocations)
    O = torch.empty_like(q)
    LSE = torch.empty((Hq, S), dtype=torch.float32, device=dev)
    attn_ws = torch.empty(max(ssa.attn_ws_bytes(plan, d), 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    ev = {n: [torch.cuda.Event(enable_timing=True) for _ in range(2)] for n in ("cap", "ext", "attn")}

    def attn_step():
        """The timed step: the prefill call (stripe gather + attention kernel)."""
        ssa.attn_fwd(q, k, v, plan, out=O, lse=LSE, ws=attn_ws, status=status, check=False)

    def path_step(timed_stage=None):
        """The whole path: capture of the layer's maps, extension fill pass, attention."""
        if timed_stage:
            ev["cap"][0].record(stream)
        ssa.capture(maps, out=cap_out, ws=cap_ws, status=status, check=False)
        if timed_stage:
            ev["cap"][1].record(stream)
            ev["ext"][0].record(stream)
        ssa.refill(plan, *lists, status=status)
        if timed_stage:
            ev["ext"][1].record(stream)
            ev["attn"][0].record(stream)
        attn_step()
        if timed_stage:
            ev["attn"][1].record(stream)

    for _ in range(args.warmup):
        path_step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")

    # ---------------- device-timed region: K prefill calls ----------------
    stage_ms = {"cap": 0.0, "ext": 0.0, "attn": 0.0}
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)  # let the sampler take its first reading
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        attn_step()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dist is not None:
        dist.barrier()
    ms_total = t_start.elapsed_time(t_end)
    ms_step = max_over_ranks(ms_total / args.steps, dist, dev)

    # the whole path, K steps, then its per-stage device times over a second pass
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        path_step()
    p1.record(stream)
    torch.cuda.synchronize()
    path_ms = max_over_ranks(p0.elapsed_time(p1) / args.steps, dist, dev)
    reps = max(5, min(args.steps, 50))
    for _ in range(reps):
        path_step(timed_stage=True)
        torch.cuda.synchronize()
        for n in stage_ms:
            stage_ms[n] += ev[n][0].elapsed_time(ev[n][1]) / reps
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during timing")

    # ---------------- the same path step, captured once into a CUDA graph and replayed ----------------
    # (14 launches per step: the replay removes the host launch overhead between them)
    g_ms_local, g_err = float("nan"), None
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            path_step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            path_step()
        graph.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        g_ms_local = g0.elapsed_time(g1) / args.steps
        del graph
    except RuntimeError as exc:  # capture unsupported here: reported, the rest still runs
        g_err = str(exc).splitlines()[0][:200]
    g_ms = max_over_ranks(g_ms_local, dist, dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during the graph replays")
    path_graph = ({"error": g_err} if g_err is not None else
                  {"what": "the same path step captured once into a CUDA graph and replayed",
                   "ms_per_step": g_ms, "tokens_per_s": world * S / (g_ms / 1e3)})

    # ---------------- end-to-end through the public API with host buffers ----------------
    e2e = None
    if not args.no_e2e:
        h_O = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
        h_L = torch.empty(LSE.shape, dtype=torch.float32).pin_memory()
        e_steps = max(3, min(10, args.steps))

        def e2e_step():
            maps.copy_(h_maps, non_blocking=True)
            q.copy_(h_q, non_blocking=True)
            k.copy_(h_k, non_blocking=True)
            v.copy_(h_v, non_blocking=True)
            for dst, src in zip(lists, h_lists):
                dst.copy_(src, non_blocking=True)
            path_step()
            h_O.copy_(O, non_blocking=True)
            h_L.copy_(LSE, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        seq_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, dist, dev)
        h2d = (h_maps.numel() * 4 + sum(t.numel() * 2 for t in (h_q, h_k, h_v)) +
               sum(t.numel() * 4 for t in h_lists))
        d2h = h_O.numel() * 2 + h_L.numel() * 4

        # Pipelined: the same steps on two streams with a buffer set each, so that one
        # step's host-to-device copies overlap the previous step's path and its
        # device-to-host copies (every step still copies its inputs in and its O, LSE out).
        def make_set():
            m2 = torch.empty_like(maps)
            q2, k2, v2 = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            l2 = [torch.empty_like(t) for t in lists]
            for dst, src in zip((m2, q2, k2, v2, *l2), (maps, q, k, v, *lists)):
                dst.copy_(src)
            c2 = ssa.capture(m2)
            w2 = torch.empty_like(cap_ws)
            p2 = ssa.extend(*l2, S)
            o2, lse2 = torch.empty_like(O), torch.empty_like(LSE)
            aw2 = torch.empty_like(attn_ws)
            ho = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
            hl = torch.empty(LSE.shape, dtype=torch.float32).pin_memory()
            return dict(maps=m2, q=q2, k=k2, v=v2, lists=l2, cap=c2, ws=w2, plan=p2, O=o2, LSE=lse2, aws=aw2,
                        hO=ho, hL=hl)

        sets = [make_set() for _ in range(2)]
        streams = [torch.cuda.Stream(), torch.cuda.Stream()]

        def pipe_step(b):
            st_ = sets[b]
            for dst, src in zip((st_["maps"], st_["q"], st_["k"], st_["v"], *st_["lists"]),
                                (h_maps, h_q, h_k, h_v, *h_lists)):
                dst.copy_(src, non_blocking=True)
            ssa.capture(st_["maps"], out=st_["cap"], ws=st_["ws"], status=status, check=False)
            ssa.refill(st_["plan"], *st_["lists"], status=status)
            ssa.attn_fwd(st_["q"], st_["k"], st_["v"], st_["plan"], out=st_["O"], lse=st_["LSE"], ws=st_["aws"],
                         status=status, check=False)
            st_["hO"].copy_(st_["O"], non_blocking=True)
            st_["hL"].copy_(st_["LSE"], non_blocking=True)

        torch.cuda.synchronize()
        for b in range(2):  # warm each set once
            with torch.cuda.stream(streams[b]):
                pipe_step(b)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        p_steps = max(4, e_steps)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for b in range(2):
            streams[b].wait_event(s0)
        for i in range(p_steps):
            with torch.cuda.stream(streams[i % 2]):
                pipe_step(i % 2)
        for b in range(2):
            stream.wait_stream(streams[b])
        s1.record(stream)
        torch.cuda.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the pipelined end-to-end steps")
        e_ms = max_over_ranks(s0.elapsed_time(s1) / p_steps, dist, dev)
        del sets
        e2e = {"value": world * S / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms,
               "what": "the whole path through the public API per step: maps, pattern lists and Q/K/V in "
                       "from pinned host memory, capture + extend + attention, O and LSE back; steps "
                       "alternate between two streams and buffer sets, so one step's copies overlap "
                       "its neighbours' work",
               "sequential_ms_per_step": seq_ms}

    # ---------------- dense reference point (context, not the target) ----------------
    dense = None
    if args.dense_ref:
        import torch.nn.functional as F
        qd = q.unsqueeze(0)
        kd, vd = k.unsqueeze(0), v.unsqueeze(0)
        scale = d ** -0.5

        def sdpa():
            return F.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=scale, enable_gqa=True)

        for _ in range(3):
            sdpa()
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        d0.record()
        for _ in range(reps):
            sdpa()
        d1.record()
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1) / reps
        dense = {"what": "torch scaled_dot_product_attention, causal, bf16, same Q/K/V (GQA), all causal pairs",
                 "ms": dms, "tokens_per_s": S / (dms / 1e3),
                 "effective_tflops_of_causal_pairs": 4.0 * d * Hq * S * (S + 1) / 2 / (dms / 1e3) / 1e12}

    # ---------------- metrics ----------------
    nnz = nnz_per_head(diags, verts, S)
    flops = 4.0 * d * float(nnz.sum())
    causal_pairs = S * (S + 1) / 2
    density = float(nnz.mean() / causal_pairs)
    hbm_gbs, tf_burst, tf_sust, peak_kind = load_peaks()
    attn_ms = ms_step  # the timed step is the prefill call
    algo_bytes = (2 * Hq * S * d * 2) + (2 * Hkv * S * d * 2) + Hq * S * 4
    t_tensor = flops / (tf_burst * 1e12)
    t_hbm = algo_bytes / (hbm_gbs * 1e9)
    # one ex2 per retained pair on the MUFU: 16 per clock per SM (measured 15.99) at the
    # maximum SM clock; at d = 64 this, not the tensor pipe, bounds the kernel
    n_exp = float(nnz.sum())  # nnz holds one entry per Q head
    mufu_peak = MUFU_EX2_PER_CLK_SM * props.multi_processor_count * sm_max_mhz() * 1e6
    t_mufu = n_exp / mufu_peak
    bound = max((t_tensor, "tensor"), (t_hbm, "hbm"), (t_mufu, "alu"))[1]
    if bound == "alu":
        achieved = n_exp / (attn_ms / 1e3) / 1e9
        roof = {"bound": "alu", "achieved": achieved, "peak": mufu_peak / 1e9, "unit": "Gex2/s",
                "frac": achieved / (mufu_peak / 1e9), "pipe": "MUFU ex2 (one per retained pair)"}
    elif bound == "tensor":
        achieved = flops / (attn_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                "frac": achieved / tf_burst}
    else:
        achieved = algo_bytes / (attn_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs}
    traffic = args.traffic if args.traffic is not None else profiled_traffic(args.workload)
    roof.update({"traffic": traffic, "traffic_source": ("command line" if args.traffic is not None else
                 f"profiles/sparse_attn_fwd_{args.workload}_dram.json (dram__bytes_read.sum + dram__bytes_write.sum "
                 "per launch, ncu)" if traffic else None),
                 "kernel": "sparse_attn_fwd (stripe gather + attention kernel)",
                 "peak_source": f"{peak_kind} ({'burst' if bound == 'tensor' else 'copy'})",
                 "algorithmic": {"flops": flops, "bytes": algo_bytes},
                 "roofline_ms": max(t_tensor, t_hbm, t_mufu) * 1e3,
                 "frac_of_roofline_time": max(t_tensor, t_hbm, t_mufu) * 1e3 / attn_ms,
                 # against the slower of the tensor and HBM bounds alone (no MUFU bound)
                 "frac_of_tensor_hbm_bound": max(t_tensor, t_hbm) * 1e3 / attn_ms,
                 "bounds_ms": {"tensor": t_tensor * 1e3, "hbm": t_hbm * 1e3, "mufu": t_mufu * 1e3}})

    line = {
        "metric": METRIC, "value": world * S / (ms_step / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "H_q": Hq, "H_kv": Hkv, "S": S, "d": d,
                   "density_of_causal": density, "nnz_per_head_mean": float(nnz.mean()),
                   "step": "one sparse_attn_fwd call (stripe gather + attention) over the layer",
                   "path_capture": f"{CAPTURE_MAPS} maps x L={CAPTURE_L} per path step", "batch": 1,
                   "parallelism": f"replicas x{world}" if world > 1 else "single-gpu",
                   "l2": "inputs larger than L2 (Q+K+V+O %.2f GB)" % ((2 * Hq + 2 * Hkv) * S * d * 2 / 1e9)},
        "path": {"what": "capture of the layer's 32 maps + extend fill pass + attention, per step",
                 "ms_per_step": path_ms, "tokens_per_s": world * S / (path_ms / 1e3),
                 "stages_ms": {"capture": stage_ms["cap"], "extend_fill": stage_ms["ext"],
                               "attn_fwd": stage_ms["attn"]},
                 "gpu_launches_per_step": sum(LAUNCHES.values()), "graph": path_graph},
        "effective_tflops": flops / (attn_ms / 1e3) / 1e12,
        "roofline": roof,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": args.steps * LAUNCHES["attn"],
        "dense_reference": dense,
    }
    return line


def run_decode(args):
    """Time sparse_attn_decode on one GPU: tokens/s (B new tokens per step) and the
    achieved HBM bandwidth of the gathered key/value rows against the measured copy peak."""
    import torch

    import structured_sparse_attention_b200 as ssa
    B, Hq, Hkv, S, d, builder = DECODE_WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    diags, verts = builder()
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)
    lists = [torch.from_numpy(a.astype(np.int32)).to(dev) for a in (dp, do, vp, vo)]
    plan = ssa.extend(*lists, S)
    base = inputs.SEED_BASE + 8
    kc = torch.from_numpy(np.stack([inputs.normal_bf16(base + 2 * b, Hkv, S, d) for b in range(B)]).view(np.int16))
    vc = torch.from_numpy(np.stack([inputs.normal_bf16(base + 2 * b + 1, Hkv, S, d) for b in range(B)]).view(np.int16))
    kc, vc = kc.to(dev).view(torch.bfloat16), vc.to(dev).view(torch.bfloat16)
    h_q = torch.from_numpy(inputs.normal_bf16(base - 1, B, Hq, d).view(np.int16)).view(torch.bfloat16).pin_memory()
    q = h_q.to(dev)
    pos_h = np.full(B, S - 1, np.int32)
    pos = torch.from_numpy(pos_h).to(dev)
    O = torch.empty_like(q)
    LSE = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(ssa.load().sparse_attn_decode_ws_bytes(B, Hq, d), 16), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # larger than the 126 MB L2

    def call():
        ssa.attn_decode(q, kc, vc, pos, plan, out=O, lse=LSE, ws=ws, status=status, check=False)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0")
    sampler.start()
    time.sleep(0.3)
    for e0, e1 in ev:
        flush.fill_(1)  # evict the previous step's rows from L2 (not timed)
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    # end to end: the step's queries in from pinned host memory, O and LSE back
    h_O = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
    h_L = torch.empty(LSE.shape, dtype=torch.float32).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        q.copy_(h_q, non_blocking=True)
        call()
        h_O.copy_(O, non_blocking=True)
        h_L.copy_(LSE, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1) / args.steps
    # retained keys of row S-1 per head (integer counting from the lists)
    keys = 0
    for Dh, Ch in zip(diags, verts):
        Dh, Ch = np.asarray(Dh, np.int64), np.asarray(Ch, np.int64)
        band = set((S - 1 - Dh[Dh <= S - 1]).tolist())
        keys += len(band | set(Ch[Ch <= S - 1].tolist()))
    algo_bytes = B * keys * d * 2 * 2 + 2 * B * Hq * d * 2 + B * Hq * 4
    hbm_gbs, _, _, peak_kind = load_peaks()
    achieved = algo_bytes / (ms / 1e3) / 1e9
    line = {"metric": "sparse-attn decode tokens/s & achieved HBM GB/s vs roofline", "value": B / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "B": B, "H_q": Hq, "H_kv": Hkv, "S_cache": S, "d": d,
                       "keys_per_sequence": keys, "l2": "flushed between timed steps (256 MB write)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": None, "kernel": "sparse_attn_decode (partial + combine)",
                         "peak_source": f"{peak_kind} (copy)", "algorithmic": {"bytes": algo_bytes}},
            "clocks": clocks,
            "e2e": {"value": B / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h_q.numel() * 2),
                    "d2h_bytes_per_step": int(h_O.numel() * 2 + h_L.numel() * 4), "ms_per_step": e_ms},
            "gpu_launches": 2 * args.steps, "cpu_baseline": None}
    print(json.dumps(line), flush=True)


def run_maps(args):
    """Time sparse_attn_maps on one GPU: averaged maps per second and the roofline of the
    kernel (HBM bytes, one exponential and 2 d FLOPs per causal pair per sample)."""
    import torch

    import structured_sparse_attention_b200 as ssa
    n, B, L, d = MAPS_WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    q_h, k_h = inputs.qk_samples(inputs.SEED_BASE + 9, n, B, L=L, d=d)
    h_q = torch.from_numpy(q_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_k = torch.from_numpy(k_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    q, k = h_q.to(dev), h_k.to(dev)
    maps = torch.empty((n, L, L), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = d ** -0.5

    def call():
        ssa.attn_maps(q, k, scale, out=maps, status=status, check=False)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0")
    sampler.start()
    time.sleep(0.3)
    for e0, e1 in ev:
        flush.fill_(1)  # inputs (1.07 GB) exceed L2 anyway; flushed for symmetry (not timed)
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    e2e = None
    if not args.no_e2e:
        # end to end: Q and K in from pinned host memory, the maps back
        h_m = torch.empty(maps.shape, dtype=torch.float32).pin_memory()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_steps = max(3, min(args.steps, 10))
        e0.record()
        for _ in range(e_steps):
            q.copy_(h_q, non_blocking=True)
            k.copy_(h_k, non_blocking=True)
            call()
            h_m.copy_(maps, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1) / e_steps
        e2e = {"value": n / (e_ms / 1e3), "unit": "maps/s", "h2d_bytes_per_step": int(2 * h_q.numel() * 2),
               "d2h_bytes_per_step": int(h_m.numel() * 4), "ms_per_step": e_ms}
    pairs = n * B * L * (L + 1) // 2  # causal (i, j) pairs over all samples
    algo_bytes = 2 * n * B * L * d * 2 + n * L * L * 4
    algo_flops = 2 * d * pairs
    hbm_gbs, tflops, _, peak_kind = load_peaks()
    mufu = MUFU_EX2_PER_CLK_SM * props.multi_processor_count * sm_max_mhz() * 1e6
    bounds = {"hbm": algo_bytes / (hbm_gbs * 1e9) * 1e3, "mufu": pairs / mufu * 1e3,
              "tensor": algo_flops / (tflops * 1e12) * 1e3}
    bound = max(bounds, key=bounds.get)
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": algo_bytes / (ms / 1e3) / 1e9, "peak": hbm_gbs, "unit": "GB/s"}
    elif bound == "mufu":
        roof = {"bound": "alu", "achieved": pairs / (ms / 1e3) / 1e9, "peak": mufu / 1e9, "unit": "Gex2/s",
                "pipe": "MUFU ex2 (one per causal pair per sample)"}
    else:
        roof = {"bound": "tensor", "achieved": algo_flops / (ms / 1e3) / 1e12, "peak": tflops, "unit": "TFLOP/s"}
    roof.update({"frac": bounds[bound] / ms, "traffic": None, "kernel": "attn_maps_kernel",
                 "peak_source": f"{peak_kind}", "roofline_ms": bounds[bound], "bounds_ms": bounds,
                 "algorithmic": {"bytes": algo_bytes, "flops": algo_flops, "ex2": pairs}})
    line = {"metric": "stage-one averaged attention maps/s vs roofline", "value": n / (ms / 1e3), "unit": "maps/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "n_maps": n, "B": B, "L": L, "d": d,
                       "l2": "inputs larger than L2 (Q+K 1.07 GB)"},
            "roofline": roof, "clocks": clocks, "e2e": e2e, "gpu_launches": args.steps, "cpu_baseline": None}
    if not args.no_cpu_baseline:
        from oracle import oracle as ora
        ora.build()
        cores = len(os.sched_getaffinity(0))
        n_cpu = min(n, max(2, cores))  # one map per OpenMP thread
        t0 = time.perf_counter()
        ora.attn_maps(q_h[:n_cpu], k_h[:n_cpu], scale)
        cpu_s = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n_cpu / cpu_s, "unit": "maps/s", "cores": min(cores, n_cpu),
                                "kind": "oracle", "sample": f"the first {n_cpu} of the {n} maps, all {B} samples "
                                "each, fp64, one map per thread"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ssa", choices=["ssa", "reference"])
    ap.add_argument("--workload", default="llama3-8b-layer-64k",
                    choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS) + sorted(MAPS_WORKLOADS)
                    + sorted(SWEEP_WORKLOADS) + sorted(CAPTURE_WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle attention work")
    ap.add_argument("--dense-ref", action="store_true",
                    help="also time torch's causal SDPA on the same inputs (dense reference point)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per attention launch from an ncu capture of the same kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.workload in CAPTURE_WORKLOADS:
        if args.impl != "ssa" or args.gpus != 1:
            ap.error("capture workloads run the library on one GPU")
        run_capture(args)
        return
    if args.workload in SWEEP_WORKLOADS:
        if args.impl != "ssa" or args.gpus != 1:
            ap.error("sweep workloads run the library on one GPU")
        run_capture_sweep(args)
        return
    if args.workload in MAPS_WORKLOADS:
        if args.impl != "ssa" or args.gpus != 1:
            ap.error("map workloads run the library on one GPU")
        run_maps(args)
        return
    if args.workload in DECODE_WORKLOADS:
        if args.impl != "ssa" or args.gpus != 1:
            ap.error("decode workloads run the library on one GPU")
        run_decode(args)
        return
    rank, world, local, dist = dist_setup(args.gpus)
    if args.impl == "reference":
        if rank == 0:
            Hq, Hkv, S, d, _ = WORKLOADS[args.workload]
            t0 = time.perf_counter()
            vals, rows, secs = [], 0, 0.0
            desc = None
            maps = inputs.averaged_maps(inputs.SEED_BASE + 2, CAPTURE_MAPS, L=CAPTURE_L, n_samples=16)
            for i in range(args.warmup + args.steps):
                budget = max(1.0, args.cpu_budget / max(1, args.steps))
                v, desc = oracle_leg(args.workload, budget_s=budget, maps=maps)
                if i >= args.warmup:
                    vals.append(v)
                    rows += desc["rows_timed"]
                    secs += desc["seconds_timed"]
            value = float(np.median(vals))
            # Each step is a bounded sample of the layer (a few thousand query rows, not all
            # S): ms_per_step is the extrapolated time of a whole layer, not a measured one.
            line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": S / value * 1e3,
                    "extrapolated": True, "rows_timed": rows, "seconds_timed": round(secs, 3),
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                    "data": "synthetic", "config": {"workload": args.workload, "H_q": Hq, "H_kv": Hkv, "S": S,
                                                    "d": d, "step": "one sparse-attention prefill of the layer"},
                    "cpu_baseline": dict(desc, value=value, unit=UNIT, rows_timed=rows, seconds_timed=round(secs, 3)),
                    "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                    "wall_s": time.perf_counter() - t0}
            print(json.dumps(line), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    line = run_gpu(args, rank, world, local, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc = oracle_leg(args.workload, budget_s=args.cpu_budget)
        line["cpu_baseline"] = dict(desc, value=v, unit=UNIT)
    elif rank == 0:
        line["cpu_baseline"] = None
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
