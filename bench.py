"""Benchmark of the ZeRO partitioned optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config sweep|gpt2_small|toy|stage3_1p3b|owner_7p5b]
                    [--nd ND --bucket-mb MB]                 # one bucket-sweep point
                    [--sweep OUT.jsonl]                      # the whole bucket sweep
                    [--eager]                                # launch every step from the host

One step = the whole hot path over one batch of gradients: for every bucket,
the fused reduce-scatter + owner Adam + all-gather kernel, then the
gradient-norm / overflow reduction (stage 3 workloads add the forward and
backward layer gathers).  The timed steps are replayed as a CUDA graph
(graph.StepGraph: the same kernels, with the step's constants refreshed in
device memory by a captured copy) unless the workload gathers layers or
--eager is given.  The dominant kernel's rate is timed in the same steps: an
event pair around each step's chain of bucket kernels (which start one
another early through programmatic dependent launch) gives the chain's span,
divided by its launches.  The default workload is one point of the
bucket-size sweep: 5e8 parameters, Nd = 16 logical ranks, stage 2, buckets
of 64 MB of one rank's bf16 gradient (2^25 elements; 15 buckets).  Inputs
are resident in HBM when timing starts and one step touches ~44 GB, far more
than the 126 MB L2, so no flush is needed.

The metric is parameters updated per second (Gparams/s); the JSON line also
carries the achieved HBM bandwidth of the dominant kernel against the measured
B200 copy bandwidth, the CPU oracle timed on a bounded sample, an end-to-end
number with host-resident gradients, and the SM clocks seen while timing.

With N > 1 (torchrun), each rank runs the same single-GPU workload on its own
GPU (the simulated ranks are HBM slices; there is no inter-GPU exchange), and
the value is the sum over ranks of parameters over the slowest rank's time.
"""
import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Gparams/s per ZeRO step (RS+Adam+AG); achieved HBM GB/s vs B200 peak"
UNIT = "Gparams/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, nominal
PROFILES = os.path.join(ROOT, "profiles")
K1_SOURCES = [os.path.join(ROOT, "zero_partitioned_optimizer_step_b200", "csrc", f)
              for f in ("zero_step.cu", "zero_tma.cuh", "zero_ring.cuh", "zero_device.cuh")]


def kernel_source_hash():
    """First 16 hex digits of sha256 over the step kernels' sources."""
    h = hashlib.sha256()
    for f in K1_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="sweep",
                    choices=["sweep", "toy", "gpt2_small", "stage3_1p3b", "owner_7p5b"])
    ap.add_argument("--nd", type=int, default=None,
                    help="logical ranks (bucket sweep point: default 16; other workloads: "
                         "override their Nd)")
    ap.add_argument("--bucket-mb", type=int, default=64)
    ap.add_argument("--sweep", default=None, help="write the bucket sweep grid as JSON lines here")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time the step replayed as a CUDA graph (the default where possible; "
                         "for --sweep: add graph-replay numbers)")
    ap.add_argument("--eager", action="store_true",
                    help="time the step launched from the host every time, not as a graph")
    ap.add_argument("--psi", type=int, default=None,
                    help="override the parameter count (flat single-unit workloads only)")
    ap.add_argument("--shard", type=int, default=None,
                    help="one-owner workloads: owner shard size (psi = nd * shard)")
    ap.add_argument("--layers", type=int, default=None,
                    help="stage-3 layer-wise workload: number of transformer blocks")
    ap.add_argument("--guarded", action="store_true",
                    help="time the two-pass guarded step (global-norm clip, skip on overflow)")
    ap.add_argument("--max-grad-norm", type=float, default=1.0,
                    help="--guarded: clip threshold (0 = no clipping)")
    ap.add_argument("--prefetch", type=int, default=None,
                    help="stage-3 workloads: gather the layers with a prefetch window of this "
                         "depth on a side stream (default: one after the other)")
    ap.add_argument("--weight-decay", type=float, default=0.0,
                    help="decoupled weight decay (AdamW) of every step")
    ap.add_argument("--reshard", type=int, default=None, metavar="ND2",
                    help="time resharding the workload's owner-storage state (w, m, v; and the "
                         "parameter shards at stage 3) from its Nd to ND2 ranks")
    ap.add_argument("--peer", action="store_true",
                    help="time the ranks-as-devices step (zero_step_peers): on one GPU the Nd "
                         "ranks as separate allocations; under torchrun Nd = N GPUs, peers "
                         "mapped through CUDA IPC")
    return ap.parse_args()


def get_cfg(args):
    from zero_partitioned_optimizer_step_b200.configs import CONFIGS, sweep_config
    if args.config == "sweep":
        cfg = sweep_config(args.nd or 16, args.bucket_mb)
    else:
        cfg = dict(CONFIGS[args.config])
        if args.nd is not None:
            cfg["nd"] = args.nd
            cfg["workload"] += " (Nd overridden to %d)" % args.nd
    if args.psi is not None:
        if cfg["units"] is not None or cfg["owner_view"] >= 0:
            raise SystemExit("--psi applies to flat all-ranks workloads only")
        cfg["psi"] = args.psi
        cfg["workload"] = "flat vector psi=%d, Nd=%d, stage %d, %d-element buckets" % (
            args.psi, cfg["nd"], cfg["stage"], cfg["bucket_elems"])
    if args.shard is not None:
        if cfg["owner_view"] < 0:
            raise SystemExit("--shard applies to one-owner workloads only")
        cfg["psi"] = cfg["nd"] * args.shard
        cfg["workload"] = "one owner, shard %d, Nd=%d, %d-element buckets" % (
            args.shard, cfg["nd"], cfg["bucket_elems"])
    if args.layers is not None:
        if cfg["units"] is None:
            raise SystemExit("--layers applies to the stage-3 layer-wise workload only")
        from zero_partitioned_optimizer_step_b200.configs import stage3_units
        cfg["units"] = stage3_units(layers=args.layers)
        cfg["psi"] = sum(cfg["units"])
        cfg["workload"] = "stage 3 layer-wise, %d x hidden 2048 (psi=%d), Nd=%d" % (
            args.layers, cfg["psi"], cfg["nd"])
    return cfg


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def k1_traffic_per_elem(kernel, nd, bucket_elems, view):
    """DRAM bytes per element of one bucket launch, from a committed ncu
    summary of the same kernel on a launch of the same shape (kernel, Nd,
    bucket size, view), if it was taken on the current kernel source (else
    None).  A summary states its shape as `shape: <kernel> nd=<Nd>
    bucket_elems=<n> view=<replicas|owner>`."""
    want = "%s nd=%d bucket_elems=%d view=%s" % (kernel, nd, bucket_elems, view)
    src_hash = kernel_source_hash()
    try:
        names = sorted(os.listdir(PROFILES))
    except OSError:
        return None
    for name in names:
        if not name.endswith(".md"):
            continue
        with open(os.path.join(PROFILES, name), encoding="utf-8") as f:
            txt = f.read()
        sh = re.search(r"^shape:\s*(.+?)\s*$", txt, re.M)
        m = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
        b = re.search(r"dram_bytes_per_element:\s*([0-9.eE+-]+)", txt)
        if sh and m and b and sh.group(1) == want and m.group(1) == src_hash:
            return float(b.group(1))
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed loop runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# -------------------------------------------------------- multi-rank timing
def max_over_ranks(seconds, dist, device):
    """The slowest rank's device time (every rank gets the same value)."""
    if dist is None:
        return seconds
    import torch
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, params_per_rank_step, steps, seconds):
    """Whole-job Gparams/s: every rank updates its own replica of the
    workload, so the job processes world x params per step."""
    return world * params_per_rank_step * steps / seconds / 1e9


# ----------------------------------------------------------------- workload
class Workload:
    """Device buffers of one configuration, built from the seeded generators."""

    def __init__(self, cfg, device, prefetch=None, weight_decay=0.0):
        import torch
        import zero_partitioned_optimizer_step_b200 as Z
        from zero_partitioned_optimizer_step_b200 import inputs
        self.Z, self.torch = Z, torch
        self.cfg = cfg
        self.dev = device
        nd, stage, owner = cfg["nd"], cfg["stage"], cfg["owner_view"]
        self.prefetch = prefetch
        self.lp = Z.zero_plan(cfg["psi"], nd, stage, cfg["bucket_elems"], unit_elems=cfg["units"],
                              max_live=1 + (prefetch or 0))
        self.units = self.lp.units()
        self.S, self.psi_pad = self.lp.S, self.lp.psi_pad
        self.adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=1.0 / nd,
                         weight_decay=weight_decay)
        unit_len = [u[0] for u in self.units]
        unit_pad = [u[1] for u in self.units]
        if owner >= 0:
            n = self.S
            real = min(max(cfg["psi"] - owner * n, 0), n)
            self.G = inputs.grads(nd, [real], [n], cfg["sigma"], cfg["seed_id"], 1, device)
            self.w = inputs.master_logical([real], [n], cfg["seed_id"], device)
        else:
            n = nd * self.S
            self.G = inputs.grads(nd, unit_len, unit_pad, cfg["sigma"], cfg["seed_id"], 1, device,
                                  outlier_frac=cfg["outlier_frac"])
            w_log = inputs.master_logical(unit_len, unit_pad, cfg["seed_id"], device)
            self.w = torch.empty(n, dtype=torch.float32, device=device)
            for o in range(nd):
                for (ln, P, s, U, O) in self.units:
                    self.w[o * self.S + O:o * self.S + O + s] = w_log[U + o * s:U + (o + 1) * s]
            del w_log
        self.m = torch.zeros(n, dtype=torch.float32, device=device)
        self.v = torch.zeros(n, dtype=torch.float32, device=device)
        self.replicas = owner < 0 and stage <= 2
        if self.replicas:
            self.params = torch.empty((nd, self.psi_pad), dtype=torch.bfloat16, device=device)
        else:
            self.params = torch.empty(n, dtype=torch.bfloat16, device=device)
        self.norm = torch.zeros(1, dtype=torch.float64, device=device)
        self.ovf = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws = Z.workspace_for(self.lp, device)
        self.layer = None
        if stage == 3 and owner < 0:
            self.layer = torch.empty(max(unit_len), dtype=torch.bfloat16, device=device)
            if prefetch:
                self.ring = [self.layer] + [torch.empty(max(unit_len), dtype=torch.bfloat16, device=device)
                                            for _ in range(prefetch)]
                self.side = torch.cuda.Stream(device)
        self.owner = owner
        flags = Z.ZERO_BYTES_FLAG_OWNER_VIEW if owner >= 0 else 0
        self.step_bytes = Z.zero_bytes_moved(self.lp, Z.ZERO_BYTES_HBM_STEP, flags)
        self.gather_bytes = (Z.zero_bytes_moved(self.lp, Z.ZERO_BYTES_HBM_GATHER_STEP)
                             if self.layer is not None else 0)
        self.elems = self.S if owner >= 0 else self.psi_pad
        self.params_per_step = (min(max(cfg["psi"] - owner * self.S, 0), self.S)
                                if owner >= 0 else cfg["psi"])
        self.nb = self.lp.n_buckets
        self._make_chunks()

    def make_graph(self):
        """The step captured as CUDA graphs (zero_partitioned_optimizer_step_b200.graph)."""
        from zero_partitioned_optimizer_step_b200.graph import StepGraph
        if self.layer is not None:
            raise SystemExit("--graph: the stage-3 layer gathers are not captured")
        return StepGraph(self.lp, self.G, self.w, self.m, self.v, self.params, self.adam,
                         grad_norm_sq=self.norm, overflow=self.ovf, workspace=self.ws,
                         owner_view=self.owner)

    def rebucket(self, bucket_elems):
        """Same buffers, a new plan with another bucket size."""
        cfg = self.cfg
        self.cfg = dict(cfg, bucket_elems=bucket_elems)
        self.lp = self.Z.zero_plan(cfg["psi"], cfg["nd"], cfg["stage"], bucket_elems,
                                   unit_elems=cfg["units"])
        self.nb = self.lp.n_buckets
        self._make_chunks()

    def bucket_elems(self, b):
        """Elements bucket b processes (the owner's part in the owner view)."""
        _, lo, hi = self.lp.query(self.Z.ZERO_Q_BUCKET_UNIT, b), \
            self.lp.query(self.Z.ZERO_Q_BUCKET_BEGIN, b), self.lp.query(self.Z.ZERO_Q_BUCKET_END, b)
        if self.owner < 0:
            return hi - lo
        u = self.lp.query(self.Z.ZERO_Q_BUCKET_UNIT, b)
        ln, P, s, U, O = self.units[u]
        a = U + self.owner * s
        return max(0, min(hi, a + s) - max(lo, a))

    def step(self, t, stream, events=None, span=None):
        """One step; with `events` (list of nb+1 CUDA events) each bucket's
        launch is bracketed so the vector kernel can be timed per launch; with
        `span` (two events) the step's bucket chain is bracketed as a whole
        (the layer gathers of stage 3 come after the second event)."""
        Z = self.Z
        kw = dict(grad_norm_sq=self.norm, overflow=self.ovf, workspace=self.ws,
                  owner_view=self.owner, stream=stream)
        if events is None:
            if span is not None:
                span[0].record(stream)
            Z.zero_step(self.lp, self.G, self.w, self.m, self.v, self.params, self.adam, t, **kw)
            if span is not None:
                span[1].record(stream)
        else:
            for i, (lo, hi, _) in enumerate(self.chunks):
                events[i].record(stream)
                Z.zero_step_buckets(self.lp, self.G, self.w, self.m, self.v, self.params,
                                    self.adam, t, lo, hi - lo, **kw)
            events[len(self.chunks)].record(stream)
        if self.layer is not None:
            self.gathers(stream)

    def gathers(self, stream):
        """Stage 3: every unit materialised in forward order, then in reverse
        (each released at once); with a prefetch window the next `prefetch`
        units are gathered on a side stream meanwhile."""
        Z = self.Z
        n_units = len(self.units)
        fwd, bwd = list(range(n_units)), list(reversed(range(n_units)))
        if self.prefetch:
            from zero_partitioned_optimizer_step_b200.prefetch import walk_layers
            for order in (fwd, bwd):
                walk_layers(self.lp, self.params, order, lambda u, x: None, depth=self.prefetch,
                            buffers=self.ring, stream=stream, side_stream=self.side)
            return
        for u in fwd + bwd:
            Z.zero_gather_layer(self.lp, u, self.params, self.layer[:self.units[u][0]], stream)
            Z.zero_release_layer(self.lp, u)

    def _make_chunks(self):
        """Bucket ranges that each hold exactly one bucket with work for this
        view (the one-owner view skips the buckets its shard is not in), so a
        call per range launches one bucket kernel: [(first, end, elems)]."""
        act = [b for b in range(self.nb) if self.bucket_elems(b) > 0]
        out, lo = [], 0
        for i, b in enumerate(act):
            hi = b + 1 if i < len(act) - 1 else self.nb
            out.append((lo, hi, self.bucket_elems(b)))
            lo = hi
        self.chunks = out

    def launches_per_step(self):
        n = sum(1 for b in range(self.nb) if self.bucket_elems(b) > 0)
        n += 1  # norm / overflow finalize
        if self.layer is not None:
            n += 2 * len(self.units)
        return n


# ----------------------------------------------------------------- arms
def cpu_baseline(wl, budget_s=10.0):
    """The oracle, as it stands, on a bounded sample of the same workload:
    consecutive 2^22-column windows of the step (all Nd gradient rows and the
    state of those columns, wrapping around), until ~budget_s of
    single-threaded CPU time."""
    import numpy as np
    import torch
    from oracle import core
    win = min(1 << 22, wl.elems)
    done, wins, t_compute = 0, 0, 0.0
    n_win = max(1, wl.elems // win)
    while t_compute < budget_s:
        lo = (wins % n_win) * win
        G = wl.G[:, lo:lo + win].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        w = wl.w[lo:lo + win].cpu().numpy()
        m = wl.m[lo:lo + win].cpu().numpy()
        v = wl.v[lo:lo + win].cpu().numpy()
        t1 = time.perf_counter()
        core.update(G, w, m, v, wl.adam, 1)
        t_compute += time.perf_counter() - t1
        done += win
        wins += 1
    return {"value": done / t_compute / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d windows of %d columns x %d gradient rows (%d params, %.1f s of "
                      "single-threaded oracle time; host copies not timed)"
                      % (wins, win, wl.cfg["nd"], done, t_compute)}


def cpu_baseline_threads(wl, budget_s=5.0):
    """The same oracle core, unchanged, on every host core this process may
    use: each round copies one 2^22-column window of the step to the host,
    cuts it into one contiguous column block per core, and runs the oracle's
    update on all blocks at once from a thread pool (the C core runs without
    the interpreter lock).  Columns are independent, so the blocks need no
    coordination.  Timed: the concurrent section of each round, until
    ~budget_s of wall time."""
    import numpy as np
    import torch
    from concurrent.futures import ThreadPoolExecutor
    from oracle import core
    cores = len(os.sched_getaffinity(0))
    win = min(1 << 22, wl.elems)
    n_win = max(1, wl.elems // win)
    done, rounds, t_wall = 0, 0, 0.0
    with ThreadPoolExecutor(max_workers=cores) as ex:
        while t_wall < budget_s:
            lo = (rounds % n_win) * win
            G = wl.G[:, lo:lo + win].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
            state = [x[lo:lo + win].cpu().numpy() for x in (wl.w, wl.m, wl.v)]
            cuts = np.linspace(0, win, cores + 1).astype(np.int64)
            blocks = [(np.ascontiguousarray(G[:, a:b]), *[x[a:b].copy() for x in state])
                      for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
            t1 = time.perf_counter()
            list(ex.map(lambda blk: core.update(blk[0], blk[1], blk[2], blk[3], wl.adam, 1), blocks))
            t_wall += time.perf_counter() - t1
            done += win
            rounds += 1
    return {"value": done / t_wall / 1e9, "unit": UNIT, "cores": cores,
            "kind": "oracle, all cores (threads over disjoint column blocks)",
            "sample": "%d windows of %d columns x %d gradient rows (%d params, %.1f s of wall time "
                      "on %d threads; host copies not timed)"
                      % (rounds, win, wl.cfg["nd"], done, t_wall, cores)}


def run_reference(args, cfg):
    """Reference arm: the CPU oracle timed on the host cores, K steps of a
    bounded sample (2^22 columns of the workload, all Nd gradient rows)."""
    import numpy as np
    import torch
    from oracle import core
    from zero_partitioned_optimizer_step_b200 import inputs
    nd = cfg["nd"]
    n = 1 << 22
    G = inputs.grads(nd, [n], [n], cfg["sigma"], cfg["seed_id"], 1, "cpu",
                     outlier_frac=cfg["outlier_frac"])
    G = G.view(torch.int16).numpy().view(np.uint16)
    w = inputs.master_logical([n], [n], cfg["seed_id"], "cpu").numpy()
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=1.0 / nd)
    for t in range(1, args.warmup + 1):
        core.update(G, w, m, v, adam, t)
    t0 = time.perf_counter()
    for t in range(args.warmup + 1, args.warmup + args.steps + 1):
        core.update(G, w, m, v, adam, t)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt / 1e9
    sample = ("%d columns x %d gradient rows of %s, per step" % (n, nd, cfg["workload"]))
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": cfg["workload"], "sample_columns": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ours(args, cfg, rank, world, dist):
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = Workload(cfg, dev, prefetch=args.prefetch, weight_decay=args.weight_decay)
    stream = torch.cuda.current_stream(dev)
    # warm-up (also builds the per-device launch grid)
    t = 1
    for _ in range(args.warmup):
        wl.step(t, stream)
        t += 1
    sg = None
    if args.graph and args.eager:
        raise SystemExit("--graph and --eager exclude each other")
    if args.graph or (not args.eager and wl.layer is None):
        sg = wl.make_graph()
        for _ in range(args.warmup):
            sg.replay(t)
            t += 1
    torch.cuda.synchronize()

    # one event pair per timed step around its chain of bucket kernels
    spans = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index).start()
    time.sleep(0.2)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    t0 = t
    for k in range(args.steps):
        if sg is not None:
            spans[k][0].record(stream)
            sg.replay(t0 + k)
            spans[k][1].record(stream)
        else:
            wl.step(t0 + k, stream, span=spans[k])
    end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    elapsed = start.elapsed_time(end) / 1e3
    # dominant kernel: the fused bucket kernel, in the timed steps themselves
    k1_time = sum(a.elapsed_time(b) for a, b in spans) / 1e3
    k1_elems = args.steps * sum(n for _, _, n in wl.chunks)
    # for context: the same kernel launched alone (an event around every
    # bucket, which also stops each launch from starting during the last)
    n_iso = min(args.steps, 20)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(wl.chunks) + 1)]
              for _ in range(n_iso)]
    for k in range(n_iso):
        wl.step(t0 + args.steps + k, stream, events[k])
    torch.cuda.synchronize()
    iso_time = sum(events[k][i].elapsed_time(events[k][i + 1]) / 1e3
                   for k in range(n_iso) for i in range(len(wl.chunks)))
    iso = (iso_time, n_iso * sum(n for _, _, n in wl.chunks), n_iso * len(wl.chunks))
    elapsed = max_over_ranks(elapsed, dist, dev)

    # end to end through the public API: gradients from pinned host memory
    # every step, the step, the norm and overflow flag read back every step
    e2e = None
    if not args.no_e2e:
        e2e = _e2e(args, wl, stream, dev, world, dist, t0 + args.steps + n_iso)
    if rank != 0:
        return None
    timing = ("graph-replayed" if sg is not None else "host-launched") + \
        " timed steps: an event pair around each step's chain of bucket kernels (with the " \
        "workspace reset and the one-CTA finalize, and in a graph the constants copy), " \
        "divided by the chain's launches"
    res = _report(args, cfg, wl, world, elapsed, k1_time, k1_elems, clk, e2e, timing=timing,
                  isolated=iso)
    res["config"]["graph"] = sg is not None
    res["config"]["weight_decay"] = args.weight_decay
    if wl.layer is not None:
        Z = wl.Z
        res["config"].update(prefetch=args.prefetch or 0,
                             peak_live_units=wl.lp.query(Z.ZERO_Q_PEAK_LIVE_UNITS),
                             peak_live_bytes=wl.lp.query(Z.ZERO_Q_PEAK_LIVE_BYTES))
    return res


def guarded_launches(lp):
    """Kernels zero_step_guarded launches per step (all-ranks view): per
    bucket an unaligned head, an 8-aligned body and a tail in each pass (one
    scalar launch where the bucket's offsets are not multiples of 8), and the
    one-block finalize between the passes."""
    import zero_partitioned_optimizer_step_b200 as Z
    units = lp.units()
    multi = len(units) > 1
    n = 0
    for b in range(lp.n_buckets):
        u = lp.query(Z.ZERO_Q_BUCKET_UNIT, b)
        _, _, s, U, O = units[u]
        j0, j1 = lp.query(Z.ZERO_Q_BUCKET_BEGIN, b) - U, lp.query(Z.ZERO_Q_BUCKET_END, b) - U
        vec = U % 8 == 0 and O % 8 == 0 and (not multi or (s % 8 == 0 and (lp.S - s) % 8 == 0))
        lo, hi = (j0 + 7) // 8 * 8, j1 // 8 * 8
        n += 1 if (not vec or lo >= hi) else (j0 < lo) + 1 + (hi < j1)
    return 2 * n + 1


def second_pass_kernel(wl):
    """The kernel zero_step_guarded runs its second pass in (aligned bodies):
    the bulk-copy ring where the parameters are written once (stage 3),
    else k_apply_bulk (replica rows as bulk copies from shared memory), or
    k_apply under ZERO_GUARD_APPLY=ldst; ZERO_STEP_KERNEL=tma forces the
    ring."""
    forced = os.environ.get("ZERO_STEP_KERNEL", "")
    if forced == "tma" or (forced != "ldg" and not wl.replicas):
        return "k_step_tma"
    if not wl.replicas:
        return "k_apply"
    return "k_apply" if os.environ.get("ZERO_GUARD_APPLY") == "ldst" else "k_apply_bulk"


def run_guarded(args, cfg, rank, world, dist):
    """--guarded: the two-pass step with global-norm clipping (at
    --max-grad-norm) and skipping on non-finite gradients, zero_step_guarded,
    on the workload's buffers (stage 3 adds the layer gathers, as in the
    plain step).  Its roofline is the whole guarded call: pass 1 reads the Nd
    bf16 rows and writes the fp32 sum, pass 2 reads the sum and w, m, v and
    writes w, m, v and the parameters."""
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = Workload(cfg, dev, prefetch=args.prefetch, weight_decay=args.weight_decay)
    if wl.owner >= 0:
        raise SystemExit("--guarded: the one-owner view has no global norm; pick an all-ranks workload")
    Z = wl.Z
    red = torch.empty(wl.lp.nd * wl.S, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(t, ev=None):
        if ev is not None:
            ev[0].record(stream)
        Z.zero_step_guarded(wl.lp, wl.G, wl.w, wl.m, wl.v, wl.params, wl.adam, t,
                            max_grad_norm=args.max_grad_norm, skip_nonfinite=True,
                            reduced_grad=red, grad_norm_sq=wl.norm, overflow=wl.ovf,
                            workspace=wl.ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if wl.layer is not None:
            wl.gathers(stream)

    t = 1
    for _ in range(args.warmup):
        step(t)
        t += 1
    Z.zero_stream_status()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index).start()
    time.sleep(0.2)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for k in range(args.steps):
        step(t + k, events[k])
    end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    Z.zero_stream_status()
    skipped = int(wl.ovf.item())
    elapsed = max_over_ranks(start.elapsed_time(end) / 1e3, dist, dev)
    g_time = max_over_ranks(sum(a.elapsed_time(b) for a, b in events) / 1e3, dist, dev)
    if rank != 0:
        return None
    peak, peak_kind = measured_peak()
    g_bytes = Z.zero_bytes_moved(wl.lp, Z.ZERO_BYTES_HBM_GUARDED_STEP)
    step_bytes = g_bytes + wl.gather_bytes
    achieved = g_bytes * args.steps / g_time / 1e9
    return {
        "metric": METRIC, "value": job_value(world, wl.params_per_step, args.steps, elapsed),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": cfg["workload"] + ", guarded step (clip at %g, skip on overflow)"
                               % args.max_grad_norm,
                   "psi": cfg["psi"], "nd": cfg["nd"], "stage": cfg["stage"],
                   "bucket_elems": cfg["bucket_elems"], "guarded": True,
                   "max_grad_norm": args.max_grad_norm, "last_step_skipped": bool(skipped),
                   "hbm_bytes_per_step": step_bytes,
                   "l2": "inputs larger than L2 (%.2f GB touched per step); no flush" % (step_bytes / 1e9)},
        "hbm_gbs": step_bytes / (elapsed / args.steps) / 1e9,
        "roofline": {"kernel": "guarded step (k_reduce, k_guard_finalize, %s: the whole call)" % second_pass_kernel(wl),
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind + " (copy bandwidth)",
                     "traffic": None, "algorithmic_bytes_per_call": g_bytes,
                     "avg_call_ms": g_time / args.steps * 1e3},
        "e2e": None,
        "gpu_launches": (guarded_launches(wl.lp) + (2 * len(wl.units) if wl.layer is not None else 0))
                        * args.steps,
        "clocks": clk,
    }


def _e2e(args, wl, stream, dev, world, dist, t_first):
    import torch
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    Gh = torch.empty(wl.G.shape, dtype=wl.G.dtype, pin_memory=True)
    Gh.copy_(wl.G)
    out_h = torch.empty(2, dtype=torch.float64).pin_memory()
    ovf_h = torch.empty(1, dtype=torch.int32).pin_memory()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for k in range(e2e_steps):
        wl.G.copy_(Gh, non_blocking=True)
        wl.step(t_first + k, stream)
        out_h[:1].copy_(wl.norm, non_blocking=True)
        ovf_h.copy_(wl.ovf, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_t = e0.elapsed_time(e1) / 1e3
    e2e_t = max_over_ranks(e2e_t, dist, dev)
    return {"value": job_value(world, wl.params_per_step, e2e_steps, e2e_t), "unit": UNIT,
            "h2d_bytes_per_step": Gh.numel() * Gh.element_size(),
            "d2h_bytes_per_step": 8 + 4, "steps": e2e_steps}


def _report(args, cfg, wl, world, elapsed, k1_time, k1_elems, clk, e2e, timing, isolated=None):
    """The JSON line.  k1_time / k1_elems: the bucket kernels' time and
    elements over the timed steps (`timing` says how they were timed);
    isolated: (time, elements, launches) of the same kernel timed launch by
    launch, for context, or None."""
    peak, peak_kind = measured_peak()
    per_elem = wl.step_bytes / wl.elems
    k1_bytes = per_elem * k1_elems
    achieved = k1_bytes / k1_time / 1e9
    n_launch = args.steps * len(wl.chunks)
    kname = wl.Z.zero_step_kernel(wl.lp, wl.owner)
    view = "owner" if wl.owner >= 0 else "replicas" if wl.replicas else "shards"
    tr = k1_traffic_per_elem(kname, cfg["nd"], cfg["bucket_elems"], view)
    roof = {"kernel": kname + " (fused reduce-scatter + Adam + all-gather, one bucket)",
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": peak_kind + " (copy bandwidth)",
            "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
            "traffic": None if tr is None else tr * k1_elems / n_launch,
            "algorithmic_bytes_per_launch": k1_bytes / n_launch,
            "avg_launch_ms": k1_time / n_launch * 1e3, "timing": timing}
    if isolated is not None:
        it, ie, il = isolated
        a_iso = per_elem * ie / it / 1e9
        roof["isolated"] = {"avg_launch_ms": it / il * 1e3, "achieved": a_iso, "frac": a_iso / peak,
                            "timing": "host-launched steps with an event around every bucket "
                                      "(no launch starts while the previous one drains)"}
    step_bytes = wl.step_bytes + wl.gather_bytes
    value = job_value(world, wl.params_per_step, args.steps, elapsed)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": cfg["workload"], "psi": cfg["psi"], "nd": cfg["nd"],
                   "precision": "bf16 gradients and parameters; fp32 master, m, v and arithmetic",
                   "stage": cfg["stage"], "bucket_elems": cfg["bucket_elems"],
                   "owner_view": cfg["owner_view"], "buckets": wl.nb,
                   "hbm_bytes_per_step": step_bytes,
                   "l2": "inputs larger than L2 (%.2f GB touched per step, L2 126 MB); no flush"
                         % (step_bytes / 1e9)},
        "hbm_gbs": step_bytes / (elapsed / args.steps) / 1e9,
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": wl.launches_per_step() * args.steps,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(wl)
        out["cpu_baseline_all_cores"] = cpu_baseline_threads(wl)
    return out


NVLINK_GBS = 770.0   # measured peer copy per direction per GPU on this kind of node


def run_peer(args, cfg, rank, world, dist):
    """--peer: the ranks-as-devices step.  Each rank's buffers are its own
    allocations: its bf16 gradient [psi_pad], its bf16 replica [psi_pad]
    (stage 3: its shard [S]) and its fp32 shard of w, m, v.  On one GPU the
    workload's Nd ranks all live on it and a step is Nd calls of
    zero_step_peers, one per rank (the kernel then runs at HBM speed).  Under
    torchrun Nd = N and every rank is one GPU: PeerStep maps the peers'
    buffers through CUDA IPC, and the step's reduce-scatter and all-gather
    are the kernel's NVLink loads and stores."""
    import torch
    import zero_partitioned_optimizer_step_b200 as Z
    from zero_partitioned_optimizer_step_b200 import inputs
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    if cfg["owner_view"] >= 0:
        raise SystemExit("--peer: the one-owner view has no counterpart; pick an all-ranks workload")
    if cfg["stage"] == 0:
        raise SystemExit("--peer: stage 0 keeps the full state on every rank")
    if args.graph:
        raise SystemExit("--peer: --graph is not supported")
    nd = world if world > 1 else cfg["nd"]
    lp = Z.zero_plan(cfg["psi"], nd, cfg["stage"], cfg["bucket_elems"], unit_elems=cfg["units"])
    units = lp.units()
    unit_len, unit_pad = [u[0] for u in units], [u[1] for u in units]
    S, psi_pad = lp.S, lp.psi_pad
    adam = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=1.0 / nd,
                weight_decay=args.weight_decay)
    w_log = inputs.master_logical(unit_len, unit_pad, cfg["seed_id"], dev)
    ranks = range(nd) if world == 1 else [rank]
    R = {}
    for r in ranks:
        g = torch.empty(psi_pad, dtype=torch.bfloat16, device=dev)
        inputs.grad_row(g, unit_len, unit_pad, cfg["sigma"], inputs.seed_for(cfg["seed_id"], r, 1),
                        cfg["outlier_frac"])
        w = torch.cat([w_log[U + r * s:U + (r + 1) * s] for (_, _, s, U, _) in units])
        n_p = psi_pad if cfg["stage"] <= 2 else S
        R[r] = dict(g=g, w=w, m=torch.zeros(S, dtype=torch.float32, device=dev),
                    v=torch.zeros(S, dtype=torch.float32, device=dev),
                    p=torch.empty(n_p, dtype=torch.bfloat16, device=dev),
                    norm=torch.zeros(1, dtype=torch.float64, device=dev),
                    ovf=torch.zeros(1, dtype=torch.int32, device=dev), ws=Z.workspace_for(lp, dev))
    del w_log
    ps = None
    if world > 1:
        from zero_partitioned_optimizer_step_b200.peer import PeerStep
        b = R[rank]
        ps = PeerStep(lp, b["g"], b["p"], b["w"], b["m"], b["v"])
    grads = [R[q]["g"] for q in range(nd)] if world == 1 else None
    params = [R[q]["p"] for q in range(nd)] if world == 1 else None

    def one_step(t, ev=None):
        if ps is not None:
            b = R[rank]
            ps.step(adam, t, grad_norm_sq=b["norm"], overflow=b["ovf"], workspace=b["ws"], events=ev)
            return
        if ev is not None:
            ev[0].record()
        for r in ranks:
            b = R[r]
            Z.zero_step_peers(lp, r, grads, params, b["w"], b["m"], b["v"], adam, t,
                              grad_norm_sq=b["norm"], overflow=b["ovf"], workspace=b["ws"])
        if ev is not None:
            ev[1].record()

    t = 1
    for _ in range(args.warmup):
        one_step(t)
        t += 1
    Z.zero_stream_status()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index).start()
    time.sleep(0.2)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for k in range(args.steps):
        one_step(t + k, events[k])
    end.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    Z.zero_stream_status()
    elapsed = max_over_ranks(start.elapsed_time(end) / 1e3, dist, dev)
    k_time = max_over_ranks(sum(a.elapsed_time(b) for a, b in events) / 1e3, dist, dev)
    if ps is not None:
        ps.close()
    if rank != 0:
        return None
    peak, peak_kind = measured_peak()
    hbm_step = Z.zero_bytes_moved(lp, Z.ZERO_BYTES_HBM_STEP)
    n_ring, n_k5 = peer_kernel_mix(lp, ranks)
    kname = ("k_step_tma through the peer table" if n_k5 == 0 else
             "k_step_peer" if n_ring == 0 else
             "k_step_tma through the peer table (%d calls) + k_step_peer (%d calls)" % (n_ring, n_k5))
    if world == 1:
        per_launch_bytes = hbm_step / max(1, nd)
        roof = {"kernel": kname + " (rank r's reduce-scatter + Adam + all-gather over its "
                          "ranks' buffers; %d calls per step)" % nd,
                "bound": "hbm", "achieved": hbm_step * args.steps / k_time / 1e9, "peak": peak,
                "unit": "GB/s", "peak_kind": peak_kind + " (copy bandwidth)", "traffic": None,
                "algorithmic_bytes_per_call": per_launch_bytes,
                "avg_call_ms": k_time / args.steps / nd * 1e3}
    else:
        # per direction: 2(Nd-1)S bytes of peer gradient reads come in and (stages
        # 1-2) as many bytes of replica stores go out; stage-3 stores stay local
        link = 2 * (nd - 1) * S
        roof = {"kernel": kname + " (one rank per GPU, peer loads and stores over NVLink)",
                "bound": "nvlink", "achieved": link * args.steps / k_time / 1e9, "peak": NVLINK_GBS,
                "unit": "GB/s", "peak_kind": "measured peer copy per direction", "traffic": None,
                "algorithmic_nvlink_bytes_per_direction": link}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return {
        "metric": METRIC, "value": cfg["psi"] * args.steps / elapsed / 1e9, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
        "scaling": "strong" if world > 1 else "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": cfg["workload"] + ", ranks as devices (zero_step_peers)",
                   "psi": cfg["psi"], "nd": nd, "stage": cfg["stage"],
                   "bucket_elems": cfg["bucket_elems"], "peer": True,
                   "hbm_bytes_per_step": hbm_step,
                   "l2": "inputs larger than L2 (%.2f GB touched per step); no flush" % (hbm_step / 1e9)},
        "hbm_gbs": hbm_step / (elapsed / args.steps) / 1e9,
        "roofline": roof, "e2e": None,
        "gpu_launches": sum(peer_launches(lp, r) for r in ranks) * args.steps, "clocks": clk,
    }


def peer_kernel_mix(lp, ranks):
    """How many of `ranks`' calls of one step run their aligned bodies in
    the bulk-copy kernel and how many in K5, as the library reports
    (zero_step_peers_kernel)."""
    import zero_partitioned_optimizer_step_b200 as Z
    kinds = [Z.zero_step_peers_kernel(lp, r) for r in ranks]
    return kinds.count("k_step_tma"), kinds.count("k_step_peer")


def peer_launches(lp, r):
    """Kernels zero_step_peers launches for rank r in one step with the norm
    on: per bucket, r's part split into an unaligned head, an 8-aligned body
    and a tail (all scalar when r's storage offset is not a multiple of 8),
    then the finalize."""
    import zero_partitioned_optimizer_step_b200 as Z
    units = lp.units()
    n = 0
    for b in range(lp.n_buckets):
        u = lp.query(Z.ZERO_Q_BUCKET_UNIT, b)
        lo_b, hi_b = lp.query(Z.ZERO_Q_BUCKET_BEGIN, b), lp.query(Z.ZERO_Q_BUCKET_END, b)
        _, _, s, U, O = units[u]
        lo = U + r * s
        p0, p1 = max(lo_b, lo), min(hi_b, lo + s)
        if p0 >= p1:
            continue
        vlo, vhi = (p0 + 7) // 8 * 8, p1 // 8 * 8
        if (O - lo) % 8 or vlo >= vhi:
            n += 1
        else:
            n += (p0 < vlo) + 1 + (vhi < p1)
    return n + 1


def run_reshard(args, cfg, rank, world, dist):
    """--reshard ND2: the checkpoint step that moves the workload's owner
    storage (fp32 w, m, v, and at stage 3 the bf16 parameter shards) from its
    Nd ranks to ND2 ranks (zero_reshard, one call per array), timed over
    --steps repetitions.  Algorithmic bytes: every real element read once
    and every element of the new layout (padding included) written once."""
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = Workload(cfg, dev)
    if wl.owner >= 0:
        raise SystemExit("--reshard: the one-owner view holds one rank's shard only")
    Z = wl.Z
    to = Z.zero_plan(cfg["psi"], args.reshard, cfg["stage"], cfg["bucket_elems"], unit_elems=cfg["units"])
    arrays = [wl.w, wl.m, wl.v] + ([wl.params] if cfg["stage"] == 3 else [])
    outs = [torch.empty(to.nd * to.S, dtype=x.dtype, device=dev) for x in arrays]
    real = sum(u[0] for u in wl.units)
    nbytes = sum((real + to.nd * to.S) * x.element_size() for x in arrays)
    stream = torch.cuda.current_stream(dev)

    def once():
        for x, y in zip(arrays, outs):
            Z.zero_reshard(wl.lp, x, to, y, stream=stream)

    for _ in range(args.warmup):
        once()
    Z.zero_stream_status()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index).start()
    time.sleep(0.2)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(args.steps):
        once()
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    Z.zero_stream_status()
    elapsed = max_over_ranks(start.elapsed_time(end) / 1e3, dist, dev)
    if rank != 0:
        return None
    peak, peak_kind = measured_peak()
    achieved = nbytes * args.steps / elapsed / 1e9
    return {
        "metric": "Gparams/s resharded (owner storage, Nd to ND2)", "unit": UNIT,
        "value": job_value(world, cfg["psi"], args.steps, elapsed), "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": cfg["workload"] + ", reshard Nd=%d -> %d" % (cfg["nd"], args.reshard),
                   "psi": cfg["psi"], "nd": cfg["nd"], "nd_to": args.reshard, "stage": cfg["stage"],
                   "arrays": len(arrays), "hbm_bytes_per_step": nbytes},
        "hbm_gbs": achieved,
        "roofline": {"kernel": "k_reshard (one launch per unit and array)", "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind + " (copy bandwidth)", "traffic": None},
        "e2e": None,
        "gpu_launches": len(arrays) * len(wl.units) * args.steps,
        "clocks": clk,
    }


def run_sweep(args, rank, world, dist):
    """The bucket-size sweep (5e8 params): for each Nd one set of buffers, then
    every bucket size from 1 MB to 512 MB of one rank's bf16 gradient."""
    import torch
    from zero_partitioned_optimizer_step_b200.configs import sweep_config
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    with open(args.sweep, "w") as f:
        for nd in (2, 4, 8, 16, 64):
            wl = Workload(sweep_config(nd, 1), dev)
            for mb in (1, 2, 4, 8, 16, 32, 64, 128, 256, 512):
                wl.rebucket(mb << 19)
                cfg = dict(wl.cfg, workload="bucket sweep psi=5e8, Nd=%d, %d MB buckets" % (nd, mb))
                stream = torch.cuda.current_stream(dev)
                for t in range(1, args.warmup + 1):
                    wl.step(t, stream)
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                spans = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                         for _ in range(args.steps)]
                torch.cuda.synchronize()
                s0.record(stream)
                for k in range(args.steps):          # the step as a user runs it
                    wl.step(args.warmup + 1 + k, stream, span=spans[k])
                s1.record(stream)
                torch.cuda.synchronize()
                elapsed = s0.elapsed_time(s1) / 1e3
                k1_time = sum(a.elapsed_time(b) for a, b in spans) / 1e3
                k1_elems = args.steps * sum(n for _, _, n in wl.chunks)
                # again with an event around every bucket: each launch alone
                events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(wl.chunks) + 1)]
                          for _ in range(args.steps)]
                for k in range(args.steps):
                    wl.step(args.warmup + args.steps + 1 + k, stream, events[k])
                torch.cuda.synchronize()
                iso_time = sum(events[k][i].elapsed_time(events[k][i + 1]) / 1e3
                               for k in range(args.steps) for i in range(len(wl.chunks)))
                iso = (iso_time, k1_elems, args.steps * len(wl.chunks))
                a = argparse.Namespace(**vars(args))
                a.config = "sweep"
                a.no_cpu_baseline = True
                timing = ("host-launched steps: an event pair around each step's chain of bucket "
                          "kernels, divided by the chain's launches")
                res = _report(a, cfg, wl, world, elapsed, k1_time, k1_elems, None, None,
                              timing=timing, isolated=iso)
                res["config"]["bucket_mb"] = mb
                if args.graph:
                    sg = wl.make_graph()
                    tg = 10 ** 6
                    for _ in range(2):
                        sg.replay(tg)
                        tg += 1
                    torch.cuda.synchronize()
                    s0.record(stream)
                    for _ in range(args.steps):
                        sg.replay(tg)
                        tg += 1
                    s1.record(stream)
                    torch.cuda.synchronize()
                    eg = s0.elapsed_time(s1) / 1e3
                    res["graph"] = {"value": job_value(world, wl.params_per_step, args.steps, eg),
                                    "ms_per_step": eg / args.steps * 1e3,
                                    "hbm_gbs": wl.step_bytes / (eg / args.steps) / 1e9}
                    del sg
                f.write(json.dumps(res) + "\n")
                f.flush()
                print(json.dumps({"nd": nd, "mb": mb, "value": res["value"],
                                  "step_gbs": res["hbm_gbs"], "k1_gbs": res["roofline"]["achieved"],
                                  "k1_frac": res["roofline"]["frac"],
                                  "k1_isolated_frac": res["roofline"]["isolated"]["frac"],
                                  "graph_value": (res.get("graph") or {}).get("value")}), flush=True)
            del wl
            torch.cuda.empty_cache()


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    cfg = get_cfg(args)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, cfg)), flush=True)
        return 0
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.sweep:
            run_sweep(args, rank, world, dist)
            return 0
        run = (run_peer if args.peer else run_guarded if args.guarded else
               run_reshard if args.reshard else run_ours)
        res = run(args, cfg, rank, world, dist)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
