#!/usr/bin/env python
"""DSA decode benchmark on B200: query-tokens/s and the HBM roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one full DSA decode step (indexer -> top-k -> sparse MLA [-> LSE
combine], every layer of the workload) over one batch of synthetic inputs
resident in HBM.  Rank 0 prints one JSON line.  Under torchrun each rank runs
its own replica of the workload (independent sequences, no data-path
collective: weak scaling); the timed region is bracketed by barriers and the
slowest rank's device time is reported.
"""
import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA decode query-tokens/s on 1 B200 at 128K ctx; % of HBM roofline"
UNIT = "query-tokens/s"
DEFAULT_WORKLOAD = "decode_b32_ctx128k"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip timing the other synthetic configs after the headline one")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's sequence count (small profiling cases)")
    ap.add_argument("--tier", action="store_true",
                    help="time the two-tier (HiSparse) decode path instead (one GPU)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the sparse MLA over an e4m3 latent cache against bf16 (one GPU)")
    ap.add_argument("--fused", action="store_true",
                    help="time indexer + top-k as two kernels against the histogram-fused form "
                         "on --workload (one GPU)")
    ap.add_argument("--csa", action="store_true",
                    help="time the compressed-sparse (DeepSeek-V4 CSA) decode step instead (one GPU)")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_traffic(kernel_file: str, profile: str):
    """Per-launch DRAM traffic (read + write bytes) recorded from an ncu capture
    in profiles/, or None when the kernel source changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", profile)
    src = os.path.join(ROOT, "sparse_attention_decode_lightning_b200", "csrc", kernel_file)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.split(":")[0].strip() in ("traffic_bytes_per_launch", "source_sha256_16"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if fields.get("source_sha256_16") != sha or "traffic_bytes_per_launch" not in fields:
        return None
    return int(fields["traffic_bytes_per_launch"])


def gpu_local_cpus(dev) -> set:
    """CPUs of the GPU's own NUMA node (the sysfs local_cpulist of its PCI
    function) that this process may run on; empty when unknown."""
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        bdf = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        with open(f"/sys/bus/pci/devices/{bdf}/local_cpulist") as f:
            text = f.read().strip()
        cpus = set()
        for part in text.split(","):
            if "-" in part:
                a, b = part.split("-")
                cpus.update(range(int(a), int(b) + 1))
            elif part:
                cpus.add(int(part))
        return cpus & os.sched_getaffinity(0)
    except (OSError, ValueError, AttributeError, RuntimeError):
        return set()


def reduce_over_ranks(local_ms: float, world: int, dist=None, device=None) -> float:
    """Slowest rank's device time (ms): the job finishes when its last rank does."""
    if world <= 1 or dist is None:
        return local_ms
    import torch
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Units all ranks processed per second over the slowest rank's time."""
    return units_per_rank * world * steps / (total_ms / 1e3)


def algorithmic_bytes(inp):
    """Roofline bytes of one step: indexer FP8 keys read (once per sequence and
    indexer layer) + bf16 latent rows gathered (576 x 2 B per selected token,
    per layer; position-0 reuse gathers one set per sequence)."""
    import numpy as np
    vis = inp.q_vis.cpu().numpy().astype(np.int64)
    qo = inp.q_offsets.cpu().numpy()
    T = inp.T
    keys = 0
    for b in range(inp.B):
        qv = vis[qo[b]:qo[b + 1]]
        keys += int((qv[:1] if inp.mtp_index_share else qv).max()) * 128
    n_groups = (inp.n_layers + inp.index_share - 1) // inp.index_share
    key_bytes = keys * n_groups
    sel = np.minimum(vis, inp.topk)
    if inp.mtp_index_share:
        sel = sel.reshape(inp.B, T)[:, 0]
    gather_bytes = int(sel.sum()) * 576 * 2 * inp.n_layers
    return key_bytes, gather_bytes


class Clocks:
    """Clock and throttle-reason samples for the timed region: NVML polled about
    every millisecond from a thread (the samples taken between region_begin
    and region_end are the ones reported), with nvidia-smi at 200 ms as the
    fallback when NVML is unavailable or saw nothing inside the region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index, device=None):
        import threading
        self.gpu = gpu_index
        self.device = device
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        self.nvml_rows = []          # (time, sm MHz, max sm MHz, power W, reason mask)
        self.stop = threading.Event()
        self.thread = None
        self.nvml = None
        self.t0 = self.t1 = None

    def _nvml_start(self):
        import threading
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            if self.device is not None:
                pr = torch.cuda.get_device_properties(self.device)
                bdf = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bdf)
            else:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            return

        def poll():
            while not self.stop.is_set():
                try:
                    t = time.perf_counter()
                    row = (t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                           pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM),
                           pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons(h)))
                except Exception:
                    return
                self.nvml_rows.append(row)
                self.stop.wait(0.001)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        self._nvml_start()
        time.sleep(0.3)
        return self

    def region_begin(self):
        self.t0 = time.perf_counter()

    def region_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *a):
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.nvml is not None and (self.thread is None or not self.thread.is_alive()):
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def _nvml_summary(self):
        if self.t0 is None or self.t1 is None or self.nvml is None:
            return None
        rows = [r for r in self.nvml_rows if self.t0 <= r[0] <= self.t1]
        if not rows:
            return None
        masks = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
                 "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
                 "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
                 "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}
        seen = 0
        for r in rows:
            seen |= r[4]
        reasons = sorted(n for n, c in masks.items() if seen & int(getattr(self.nvml, c, 0)))
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(r[2] for r in rows), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(r[3] for r in rows),
                "source": "NVML, ~1 ms polling inside the timed region"}

    def summary(self):
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        inside = self._nvml_summary()
        if inside is not None:
            return inside
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        reasons = sorted({n for r in rows for n, v in zip(self.REASONS, r[5:9])
                          if v.lower().startswith("active")})
        loaded = [s for s, p in zip(sm, pw) if p is not None and p > 300] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None,
                "source": "nvidia-smi, 200 ms sampling around the timed region"}


def host_subproblem(inp, b):
    """Host numpy inputs of sequence b alone (for the oracle baseline sample):
    its keys, its queries and a compact pool of its pages."""
    import numpy as np
    from tests._helpers import np_bits
    T = inp.T
    so = inp.seq_offsets.cpu().numpy()
    k0, k1 = int(so[b]), int(so[b + 1])
    pt = inp.page_table[b].cpu().numpy()
    pages = pt[pt >= 0]
    qs = slice(b * T, (b + 1) * T)
    return {
        "B": 1, "T": T, "topk": inp.topk, "scale": inp.scale, "num_splits": inp.num_splits,
        "index_share": inp.index_share, "mtp_index_share": inp.mtp_index_share,
        "n_layers": inp.n_layers, "seq_offsets": np.array([0, k1 - k0]),
        "q_vis": np_bits(inp.q_vis[qs]), "page_table": np.arange(len(pages), dtype=np.int32)[None],
        "indexer": [{"q_idx": np_bits(d["q_idx"][qs]), "w": np_bits(d["w"][qs]),
                     "k_idx": np_bits(d["k_idx"][k0:k1])} for d in inp.indexer],
        "layers": [{"q": np_bits(L["q"][qs]),
                    "pool": np_bits(L["pool"][__import__("torch").from_numpy(pages).long().to(L["pool"].device)])}
                   for L in inp.layers],
    }


def oracle_sample(inp, seconds):
    """Time the oracle as it stands on whole sequences of the workload until
    about `seconds` of CPU work is done; returns (queries/s, sample text, cores)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        cores = 1
    done_q, spent, seqs = 0, 0.0, 0
    for b in range(inp.B):
        sub = host_subproblem(inp, b)
        t0 = time.perf_counter()
        O.decode_step(sub)
        spent += time.perf_counter() - t0
        done_q += inp.T
        seqs += 1
        if spent >= seconds:
            break
    return done_q / spent, f"{seqs} of {inp.B} sequences ({done_q} query tokens, all layers), {spent:.1f} s", cores


# ---------------------------------------------------------------- our arm
# BASELINE's five synthetic configs (MTP verify in both modes), timed one
# after another in the default run: config 1 is the headline `value`
PER_WORKLOAD = ["decode_b1_ctx8k", "decode_b32_ctx128k", "indexshare4_b64_ctx16k_128k",
                "mtp_verify_b16_t8_ctx128k", "mtp_verify_reuse_b16_t8_ctx128k",
                "decode_b4_ctx1m_split16"]


class StepRunner:
    """One workload's device buffers and its decode step through the binding."""

    def __init__(self, inp, dsa, dev, stream):
        import torch
        self.inp, self.dsa, self.stream = inp, dsa, stream
        Q, G, n = inp.Q, inp.index_share, inp.n_layers
        self.ws = dsa.workspace(Q, inp.max_len, inp.topk, inp.num_splits, device=dev)
        self.outs = [torch.empty(Q, inp.heads, 512, device=dev) for _ in range(n)]
        self.lses = [torch.empty(Q, inp.heads, device=dev) for _ in range(n)]
        ng = (n + G - 1) // G
        self.idx = torch.empty(ng, Q, inp.topk, dtype=torch.int32, device=dev)
        self.qi = [inp.indexer[l // G]["q_idx"] if l % G == 0 else None for l in range(n)]
        self.wl = [inp.indexer[l // G]["w"] if l % G == 0 else None for l in range(n)]
        self.kl = [inp.indexer[l // G]["k_idx"] if l % G == 0 else None for l in range(n)]
        self.qs = [L["q"] for L in inp.layers]
        self.pools = [L["pool"] for L in inp.layers]
        self.pts = [inp.page_table] * n

    def step(self, q_layers=None, qi=None, wl=None, out_layers=None, lse_layers=None):
        inp = self.inp
        self.dsa.dsa_decode_step(qi or self.qi, wl or self.wl, self.kl, inp.seq_offsets,
                                 inp.q_offsets, inp.q_vis, inp.B, inp.max_len, inp.topk,
                                 q_layers or self.qs, self.pools, self.pts, inp.scale,
                                 out_layers or self.outs, lse_layers or self.lses, self.idx,
                                 self.ws, index_share=inp.index_share,
                                 mtp_index_share=inp.mtp_index_share,
                                 num_splits=inp.num_splits, stream=self.stream)

    def stage_times(self, flush, steps):
        """The same kernels as the step, decomposed (indexer, top-k, one layer's
        sparse MLA with its merge), each timed live with CUDA events; ms."""
        import torch
        inp, dsa, stream = self.inp, self.dsa, self.stream
        scores = torch.empty(inp.Q, ((inp.max_len + 63) // 64) * 64, device=self.idx.device)
        first = inp.mtp_index_share
        evs = []
        for _ in range(steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(stream)
            dsa.dsa_indexer_scores(self.qi[0], self.wl[0], self.kl[0], inp.seq_offsets,
                                   inp.q_offsets, inp.q_vis, inp.B, inp.max_len, scores, self.ws,
                                   first_only=first, stream=stream)
            e[1].record(stream)
            dsa.dsa_topk_select(scores, inp.q_offsets, inp.q_vis, inp.B, inp.max_len, inp.topk,
                                self.idx[0], self.ws, first_only=first, stream=stream)
            e[2].record(stream)
            dsa.dsa_sparse_mla_decode(self.qs[0], self.pools[0], self.pts[0], inp.q_offsets,
                                      inp.q_vis, self.idx[0], inp.B, inp.scale, self.outs[0],
                                      self.lses[0], self.ws, num_splits=inp.num_splits,
                                      stream=stream)
            e[3].record(stream)
            evs.append(e)
        torch.cuda.synchronize(self.idx.device)
        dsa.dsa_check_error(self.ws, stream)
        return {"indexer": statistics.mean(e[0].elapsed_time(e[1]) for e in evs),
                "topk": statistics.mean(e[1].elapsed_time(e[2]) for e in evs),
                "mla": statistics.mean(e[2].elapsed_time(e[3]) for e in evs)}


def time_steps(runner, flush, steps, warmup, dev):
    """Device time of each of `steps` decode steps (L2 flushed before each step,
    outside the events), after `warmup` untimed steps; ms per step."""
    import torch
    for _ in range(max(3, warmup)):
        flush.zero_()
        runner.step()
    runner.dsa.dsa_check_error(runner.ws, runner.stream)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(runner.stream)
        runner.step()
        evs[i][1].record(runner.stream)
    torch.cuda.synchronize(dev)
    runner.dsa.dsa_check_error(runner.ws, runner.stream)
    return [a.elapsed_time(b) for a, b in evs]


def workload_summary(inp, step_ms, stages, hbm):
    """Per-workload figures of merit: step time, query-tokens/s, the step's
    roofline fraction (indexer keys + gathered latents over the step time)
    and the indexer's fraction of the measured copy bandwidth."""
    key_b, gat_b = algorithmic_bytes(inp)
    ms = statistics.mean(step_ms)
    ng = (inp.n_layers + inp.index_share - 1) // inp.index_share
    idx_gbs = key_b // ng / (stages["indexer"] / 1e3) / 1e9
    return {"step_us": ms * 1e3, "q_tok_s": inp.Q / (ms / 1e3),
            "step_roofline_frac_of_measured": (key_b + gat_b) / (ms / 1e3) / 1e9 / hbm,
            "step_roofline_frac_of_8tbs": (key_b + gat_b) / (ms / 1e3) / 8e12,
            "indexer_frac_of_measured": idx_gbs / hbm,
            "stages_us": {k: v * 1e3 for k, v in stages.items()},
            "bytes_per_step": key_b + gat_b, "queries_per_step": inp.Q}


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import sparse_attention_decode_lightning_b200 as dsa
    from sparse_attention_decode_lightning_b200.build import build
    from synth import get_workload, make_inputs

    build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
    wl = get_workload(args.workload, **({"B": args.batch} if args.batch else {}))
    inp = make_inputs(wl, seed=args.seed + rank, device=dev)
    Q, G, n = inp.Q, inp.index_share, inp.n_layers
    ng = (n + G - 1) // G
    S = inp.num_splits
    stream = torch.cuda.current_stream(dev)
    runner = StepRunner(inp, dsa, dev, stream)
    ws, outs, lses, idx = runner.ws, runner.outs, runner.lses, runner.idx
    qi, wl_, kl, qs, pools, pts = runner.qi, runner.wl, runner.kl, runner.qs, runner.pools, runner.pts
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        runner.step()
    dsa.dsa_check_error(ws, stream)

    # ---- timed region: K steps, L2 flushed between steps (outside the events)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with Clocks(local_rank, dev) as clk:
        barrier()
        clk.region_begin()
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            runner.step()
            evs[i][1].record(stream)
        barrier()
        t_wall = time.perf_counter() - t_wall
        clk.region_end()
    clocks = clk.summary()
    dsa.dsa_check_error(ws, stream)
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = reduce_over_ranks(sum(step_ms), world, dist, dev)

    # ---- per-kernel breakdown of the same step, live (decomposed calls, same kernels)
    stages = runner.stage_times(flush, args.steps)

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs from pinned host memory, runs the decode step and reads
    # its outputs back.  Device buffers are double-buffered and the copies run
    # on their own streams, so step i's H2D and step i-1's D2H overlap step i's
    # compute; the L2 flush stays inside every step, and the timed region runs
    # from the first H2D to the last D2H.
    e2e = None
    if not args.no_e2e:
        nb = 2
        wc_ptrs = []

        def host_input(t):
            # inputs are staged in write-combined pinned memory (the host only
            # writes it; the copy engine reads it at full PCIe speed, where
            # ordinary pinned memory gave 10-30 GB/s for these sizes)
            if t is None:
                return None
            src = t.cpu()
            nbytes = src.numel() * src.element_size()
            try:
                try:
                    from cuda.bindings import runtime as cudart
                except ImportError:
                    from cuda import cudart
                err, ptr = cudart.cudaHostAlloc(nbytes, cudart.cudaHostAllocWriteCombined)
                if int(err) != 0:
                    raise RuntimeError(str(err))
            except Exception:
                return src.pin_memory()
            wc_ptrs.append((cudart, ptr))
            raw = (ctypes.c_uint8 * nbytes).from_address(int(ptr))
            h = torch.frombuffer(raw, dtype=torch.uint8).view(src.dtype).view(src.shape)
            h.copy_(src)
            return h

        # pinned pages land on the NUMA node of the thread that allocates them:
        # allocate from the GPU's own node so the copies do not cross sockets
        saved_cpus = os.sched_getaffinity(0)
        local_cpus = gpu_local_cpus(dev)
        numa_bound = bool(local_cpus) and local_cpus != saved_cpus
        if numa_bound:
            os.sched_setaffinity(0, local_cpus)
        try:
            h_in = [host_input(t) for t in qi + wl_ + qs]
            h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs + lses]
        finally:
            if numa_bound:
                os.sched_setaffinity(0, saved_cpus)
        d_in = [[torch.empty_like(t) if t is not None else None for t in qi + wl_ + qs]
                for _ in range(nb)]
        d_res = [[torch.empty_like(o) for o in outs + lses] for _ in range(nb)]
        h2d = sum(t.numel() * t.element_size() for t in h_in if t is not None)
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        s_h2d = torch.cuda.Stream(dev)
        s_d2h = torch.cuda.Stream(dev)

        def e2e_run(k):
            ev = lambda: torch.cuda.Event()  # noqa: E731
            h2d_ev, comp_ev, d2h_ev = ([ev() for _ in range(k)] for _ in range(3))
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            s_h2d.wait_event(t0)
            for i in range(k):
                b = i % nb
                if i >= nb:
                    s_h2d.wait_event(comp_ev[i - nb])      # buffer b's previous step is done
                with torch.cuda.stream(s_h2d):
                    for d, h in zip(d_in[b], h_in):
                        if h is not None:
                            d.copy_(h, non_blocking=True)
                h2d_ev[i].record(s_h2d)
                stream.wait_event(h2d_ev[i])
                if i >= nb:
                    stream.wait_event(d2h_ev[i - nb])      # result buffer b has been read
                flush.zero_()
                d = d_in[b]
                dsa.dsa_decode_step(d[:n], d[n:2 * n], kl, inp.seq_offsets, inp.q_offsets, inp.q_vis,
                                    inp.B, inp.max_len, inp.topk, d[2 * n:], pools, pts, inp.scale,
                                    d_res[b][:n], d_res[b][n:], idx, ws, index_share=G,
                                    mtp_index_share=inp.mtp_index_share, num_splits=S, stream=stream)
                comp_ev[i].record(stream)
                s_d2h.wait_event(comp_ev[i])
                with torch.cuda.stream(s_d2h):
                    for h, dd in zip(h_out, d_res[b]):
                        h.copy_(dd, non_blocking=True)
                d2h_ev[i].record(s_d2h)
            stream.wait_event(d2h_ev[k - 1])
            t1.record(stream)
            return t0, t1

        e2e_run(2)
        barrier()
        t0, t1 = e2e_run(args.steps)
        barrier()
        e2e_ms = reduce_over_ranks(t0.elapsed_time(t1), world, dist, dev)
        e2e = {"value": job_throughput(Q, world, args.steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": ("inputs from write-combined pinned host memory" if wc_ptrs else
                        "inputs from pinned host memory") +
                       ", outputs to pinned host memory" +
                       (" (allocated from the GPU's NUMA-local CPUs)" if numa_bound else "") +
                       "; copies on two copy streams overlap "
                       "compute (double-buffered); 256 MiB L2 flush inside every step"}
        dsa.dsa_check_error(ws, stream)
        torch.cuda.synchronize(dev)
        del h_in
        for rt, ptr in wc_ptrs:
            rt.cudaFreeHost(ptr)

    key_b, gat_b = algorithmic_bytes(inp)
    hbm, hbm_kind = peaks()
    idx_ms = stages["indexer"]
    idx_bytes = key_b // ((n + G - 1) // G)
    achieved = idx_bytes / (idx_ms / 1e3) / 1e9
    step_mean_ms = total_ms / args.steps
    S_used = dsa.dsa_choose_splits(Q, inp.topk, S)
    launches_per_step = ng * (1 + 1 + (1 if inp.mtp_index_share else 0)) + n * (1 + (1 if S_used > 1 else 0))
    res = {
        "metric": METRIC, "value": job_throughput(Q, world, args.steps, total_ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_mean_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 indexer, bf16 attention, f32 accumulate", "data": "synthetic",
        "config": workload_config(wl, inp.B, S, world),
        "roofline": {"bound": "hbm", "kernel": "indexer_kernel", "achieved": achieved, "peak": hbm,
                     "peak_source": hbm_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": (measured_traffic("indexer_sm100.cu", "indexer_kernel_decode_b8_ctx128k.md")
                                 if wl.name == DEFAULT_WORKLOAD and not args.batch else None),
                     "traffic_note": "ncu dram read+write of a batch-8 capture scaled x4 to the batch-32 launch"},
        "step_roofline": {"bytes_per_step": key_b + gat_b, "key_bytes": key_b, "gather_bytes": gat_b,
                          "achieved_gbs": (key_b + gat_b) / (step_mean_ms / 1e3) / 1e9,
                          "frac_of_measured": (key_b + gat_b) / (step_mean_ms / 1e3) / 1e9 / hbm,
                          "frac_of_8tbs": (key_b + gat_b) / (step_mean_ms / 1e3) / 8e12},
        "stages_ms": stages,
        "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, cores = oracle_sample(inp, args.cpu_seconds)
        res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample}
    if world == 1 and not args.no_per_workload and not args.batch and wl.name == DEFAULT_WORKLOAD:
        # every synthetic config, each timed the same way (its own warm-up,
        # K steps with the L2 flushed before each, the live stage split); the
        # CPU and end-to-end legs stay with the headline config
        per = {}
        own = workload_summary(inp, step_ms, stages, hbm)
        del runner, ws, outs, lses, idx, qi, wl_, kl, qs, pools, pts
        for name in PER_WORKLOAD:
            if name == wl.name:
                per[name] = own
                continue
            w2 = get_workload(name)
            inp2 = make_inputs(w2, seed=args.seed, device=dev)
            r2 = StepRunner(inp2, dsa, dev, stream)
            ms2 = time_steps(r2, flush, args.steps, args.warmup, dev)
            per[name] = workload_summary(inp2, ms2, r2.stage_times(flush, args.steps), hbm)
            del r2, inp2
            torch.cuda.empty_cache()
        res["per_workload"] = per
    return res


def workload_config(wl, B, S, world):
    """The `config` object of both arms' JSON lines: the workload by name and sizes."""
    return {"workload": wl.name, "B": B, "T": wl.T, "L": wl.L,
            "L_range": list(wl.L_range) if wl.L_range else None, "layers": wl.n_layers,
            "index_share": wl.index_share, "mtp_index_share": wl.mtp_index_share,
            "topk": wl.topk, "num_splits": S, "heads": wl.heads, "idx_heads": wl.idx_heads,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (FP8 keys) and a 256 MiB L2 flush before every step"}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 CPU oracle as it stands, on whole sequences of the workload
    drawn on the host (one sequence per step)."""
    import oracle as O
    from synth import get_workload, make_inputs
    wl = get_workload(args.workload)
    one = get_workload(args.workload, B=1)
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        cores = 1
    inp = make_inputs(one, seed=args.seed, device="cpu")
    from tests._helpers import oracle_inputs
    host = oracle_inputs(inp)
    for _ in range(args.warmup):
        O.decode_step(host)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.decode_step(host)
    dt = time.perf_counter() - t0
    v = inp.Q * args.steps / dt
    return {
        "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(wl, wl.B, wl.num_splits, 1),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps x 1 sequence ({inp.Q} query tokens, all layers)"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_tier(args):
    """Two-tier (HiSparse) decode at GLM-5.2 shapes and 1M context, one GPU.

    Per step (the line's value): the upload of the index rows, the device
    planner (miss detection, LRU eviction, page-table update) and the fetch
    kernel that pulls the missing 16-token pages from pinned host memory, then
    the sparse MLA over the device buffer (page size 16).  The same steps are
    then run with the plan on the host (host_plan_path), whose fetch kernel
    time gives the roofline line.  The full latent cache (4 x 1M tokens, 4.8 GB)
    lives in pinned host memory; each sequence has 8192 device slots (host :
    device = 8).  The selected tokens come from a hot set of 1024 pages per
    sequence of which 64 are replaced every step (a synthetic locality model:
    the pages give no miss rates).  The fetch kernel's rate is compared with a
    plain pinned host-to-device copy measured in the same run."""
    import time

    import numpy as np
    import torch

    import sparse_attention_decode_lightning_b200 as dsa

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    B, L, topk, heads, qk = 4, 1 << 20, 2048, 64, 256
    PT, D = dsa.TIER_PAGE, 8192
    P = L // PT
    HOT, CHURN = 1024, 64
    host = torch.empty(B * P, PT, 576, dtype=torch.bfloat16, pin_memory=True)
    g = torch.Generator().manual_seed(args.seed)
    chunk = torch.randn(8192, PT, 576, generator=g).to(torch.bfloat16)
    for i in range(0, B * P, 8192):
        host[i:i + 8192] = chunk
    pool = torch.zeros(B * D, PT, 576, dtype=torch.bfloat16, device=dev)
    q = torch.randn(B, heads, 576, generator=g).to(torch.bfloat16).to(dev)
    q_off_h = torch.arange(B + 1, dtype=torch.int32)
    q_off = q_off_h.to(dev)
    vis = torch.full((B,), L, dtype=torch.int32, device=dev)
    st = dsa.tier_state(B, D, P)
    cp_h = torch.empty(B * D, 3, dtype=torch.int32, pin_memory=True)
    pt_d = torch.full((B, P), -1, dtype=torch.int32, device=dev)   # patched by every fetch
    cp_d = torch.empty(B * D, 3, dtype=torch.int32, device=dev)
    idx_d = torch.empty(B, topk, dtype=torch.int32, device=dev)
    out = torch.empty(B, heads, 512, device=dev)
    lse = torch.empty(B, heads, device=dev)
    ws = dsa.workspace(B, 1, topk, 0, device=dev)
    rng = np.random.default_rng(args.seed)
    hot = [rng.choice(P, HOT, replace=False) for _ in range(B)]
    n_steps = max(3, args.warmup) + args.steps
    idx_steps = []
    for _ in range(n_steps):
        rows = []
        for b in range(B):
            hot[b][rng.integers(0, HOT, CHURN)] = rng.integers(0, P, CHURN)
            pos = np.unique(rng.choice(hot[b], topk) * PT + rng.integers(0, PT, topk))
            row = np.full(topk, -1, dtype=np.int32)
            row[:len(pos)] = pos[:topk]
            rows.append(row)
        idx_steps.append(torch.from_numpy(np.stack(rows)).pin_memory())
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    scale = 1 / qk ** 0.5
    # device path: the planner and the fetch run on the GPU, no host round trip
    pt_dev = torch.empty(B, P, dtype=torch.int32, device=dev)
    dst = dsa.tier_dev_state(B, D, P, pt_dev)
    # steps are enqueued back to back (no host wait inside the loop), so the
    # host-side argument checks overlap the GPU and the events time the GPU
    drec = {"upload": [], "swap_in": [], "mla": []}
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in idx_steps]
    for i, idx_h in enumerate(idx_steps):
        e = evs[i]
        e[0].record(stream)
        idx_d.copy_(idx_h, non_blocking=True)
        e[1].record(stream)
        dsa.dsa_tier_swap_in(dst, B, D, P, idx_d, q_off, pt_dev, host, pool, ws, stream=stream)
        e[2].record(stream)
        dsa.dsa_sparse_mla_decode(q, pool, pt_dev, q_off, vis, idx_d, B, scale, out, lse, ws,
                                  stream=stream)
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    for e in evs[n_steps - args.steps:]:
        drec["upload"].append(e[0].elapsed_time(e[1]) * 1e3)
        drec["swap_in"].append(e[1].elapsed_time(e[2]) * 1e3)
        drec["mla"].append(e[2].elapsed_time(e[3]) * 1e3)
    dev_step_span_us = evs[n_steps - args.steps][0].elapsed_time(evs[-1][3]) * 1e3 / args.steps
    dsa.dsa_check_error(ws)
    # host path: the same steps with the plan on the host (fresh tier state)
    pool.zero_()
    rec = {"plan": [], "upload": [], "fetch": [], "mla": [], "misses": [], "bytes": []}
    for i, idx_h in enumerate(idx_steps):
        t0 = time.perf_counter()
        n, (hits, misses, evictions) = dsa.dsa_tier_plan(st, idx_h, q_off_h, cp_h)
        t_plan = time.perf_counter() - t0
        ev[0].record(stream)
        cp_d[:n].copy_(cp_h[:n], non_blocking=True)
        idx_d.copy_(idx_h, non_blocking=True)
        ev[1].record(stream)
        dsa.dsa_tier_fetch(host, pool, cp_d, n, ws, page_table=pt_d, stream=stream)
        ev[2].record(stream)
        dsa.dsa_sparse_mla_decode(q, pool, pt_d, q_off, vis, idx_d, B, scale, out, lse, ws,
                                  stream=stream)
        ev[3].record(stream)
        torch.cuda.synchronize(dev)
        if i >= n_steps - args.steps:
            rec["plan"].append(t_plan * 1e6)
            rec["upload"].append(ev[0].elapsed_time(ev[1]) * 1e3)
            rec["fetch"].append(ev[1].elapsed_time(ev[2]) * 1e3)
            rec["mla"].append(ev[2].elapsed_time(ev[3]) * 1e3)
            rec["misses"].append(misses)
            rec["bytes"].append(n * PT * 576 * 2)
    dsa.dsa_check_error(ws)
    # reference rate: one plain pinned host-to-device copy of 256 MiB
    src = torch.empty(256 << 20, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    ev[3].record(stream)
    for _ in range(3):
        dst.copy_(src, non_blocking=True)
    ev[4].record(stream)
    torch.cuda.synchronize(dev)
    copy_gbs = 3 * (256 << 20) / (ev[3].elapsed_time(ev[4]) / 1e3) / 1e9
    m = {k: float(np.mean(v)) for k, v in rec.items()}
    dm = {k: float(np.mean(v)) for k, v in drec.items()}
    host_step_us = m["plan"] + m["upload"] + m["fetch"] + m["mla"]
    step_us = dev_step_span_us          # first timed step's start to the last one's end
    fetch_gbs = m["bytes"] / (m["fetch"] / 1e6) / 1e9 if m["fetch"] > 0 else 0.0
    return {
        "metric": "HiSparse two-tier decode step, GLM-5.2 shapes, 1M ctx (device plan + fetch + MLA)",
        "value": B / (step_us / 1e6), "unit": "query-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": step_us / 1e3, "higher_is_better": True,
        "dtype": "bf16 attention, f32 accumulate", "data": "synthetic",
        "config": {"workload": "glm52_tier_b4_ctx1m", "B": B, "L": L, "heads": heads, "topk": topk,
                   "dev_slots_per_seq": D, "host_pages_per_seq": P, "page_tokens": PT,
                   "hot_pages": HOT, "hot_pages_replaced_per_step": CHURN},
        "stages_us": {"upload_idx": dm["upload"], "swap_in": dm["swap_in"], "mla": dm["mla"]},
        "misses_per_step": m["misses"],
        "misses_note": "from the host-plan pass over the same steps (the two plans are equal)",
        "host_plan_path": {"ms_per_step": host_step_us / 1e3,
                           "stages_us": {"plan_host": m["plan"], "upload": m["upload"],
                                         "fetch": m["fetch"], "mla": m["mla"]},
                           "misses_per_step": m["misses"]},
        "roofline": {"bound": "host link", "kernel": "tier_fetch_kernel", "achieved": fetch_gbs,
                     "peak": copy_gbs, "peak_source": "pinned cudaMemcpyAsync H2D in this run",
                     "unit": "GB/s", "frac": fetch_gbs / copy_gbs if copy_gbs else None},
    }


def run_csa(args):
    """DeepSeek-V4 CSA decode step, V4-Flash selection at 1M raw context: the
    lightning indexer scores the 4x-compressed keys (256K per sequence), the
    selector keeps top-512, and sparse MLA attends to the 512 compressed rows
    plus the 128 most recent raw tokens.  32 sequences, DeepSeek-V3.2 head
    counts (the pages give none for V4).  Only the raw pages under the window
    are allocated: nothing else of the raw cache is read.  L2 is flushed
    before every step."""
    import statistics

    import torch

    import sparse_attention_decode_lightning_b200 as dsa

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    B, L_raw, ratio, topk, window = 32, 1 << 20, 4, 512, 128
    Lc = L_raw // ratio
    g = torch.Generator(device=dev).manual_seed(args.seed)
    pc = Lc // 64                                   # compressed pages per sequence
    pr_used = (window + 63) // 64 + 1               # raw pages under the window
    num_pages = B * (pc + pr_used)
    perm = torch.randperm(num_pages, generator=g, device=dev).to(torch.int32)
    ct = perm[:B * pc].view(B, pc).contiguous()
    rt = torch.full((B, L_raw // 64), -1, dtype=torch.int32, device=dev)
    rt[:, -pr_used:] = perm[B * pc:].view(B, pr_used)
    pool = torch.empty(num_pages, 64, 576, dtype=torch.bfloat16, device=dev)
    for i in range(0, num_pages, 4096):
        pool[i:i + 4096] = torch.randn(pool[i:i + 4096].shape, generator=g, device=dev)
    q = torch.randn(B, 128, 576, generator=g, device=dev).to(torch.bfloat16)
    keys = torch.randn(B * Lc, 128, generator=g, device=dev).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    qi = torch.randn(B, 64, 128, generator=g, device=dev).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    w = torch.randn(B, 64, generator=g, device=dev) / 8
    so = torch.arange(B + 1, dtype=torch.int64, device=dev) * Lc
    qo = torch.arange(B + 1, dtype=torch.int32, device=dev)
    vis = torch.full((B,), Lc, dtype=torch.int32, device=dev)
    wvis = torch.full((B,), L_raw, dtype=torch.int32, device=dev)
    idx = torch.empty(B, topk, dtype=torch.int32, device=dev)
    out = torch.empty(B, 128, 512, device=dev)
    lse = torch.empty(B, 128, device=dev)
    ws = dsa.workspace(B, Lc, topk + window, 0, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1 / 192 ** 0.5

    def step():
        dsa.dsa_indexer_topk(qi, w, keys, so, qo, vis, B, Lc, topk, idx, ws, stream=stream)
        dsa.dsa_sparse_mla_decode_window(q, pool, ct, rt, qo, vis, wvis, idx, B, window, scale,
                                         out, lse, ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    times = {"step": [], "indexer_topk": [], "mla_window": []}
    for _ in range(args.steps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        dsa.dsa_indexer_topk(qi, w, keys, so, qo, vis, B, Lc, topk, idx, ws, stream=stream)
        e[1].record(stream)
        dsa.dsa_sparse_mla_decode_window(q, pool, ct, rt, qo, vis, wvis, idx, B, window, scale,
                                         out, lse, ws, stream=stream)
        e[2].record(stream)
        torch.cuda.synchronize(dev)
        times["indexer_topk"].append(e[0].elapsed_time(e[1]))
        times["mla_window"].append(e[1].elapsed_time(e[2]))
        times["step"].append(e[0].elapsed_time(e[2]))
    dsa.dsa_check_error(ws)
    m = {k: statistics.mean(v) for k, v in times.items()}
    key_b = B * Lc * 128
    gat_b = B * (topk + window) * 576 * 2
    hbm, hbm_kind = peaks()
    return {
        "metric": "DeepSeek-V4 CSA decode query-tokens/s (top-512 of 4x-compressed 1M ctx + 128 window)",
        "value": B / (m["step"] / 1e3), "unit": "query-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": m["step"], "higher_is_better": True,
        "dtype": "e4m3 indexer, bf16 attention, f32 accumulate", "data": "synthetic",
        "config": {"workload": "v4flash_csa_b32_ctx1m", "B": B, "L_raw": L_raw, "ratio": ratio,
                   "compressed_entries": Lc, "topk": topk, "window": window, "heads": 128,
                   "l2": "256 MiB flush before every step"},
        "stages_ms": {"indexer_topk": m["indexer_topk"], "mla_window": m["mla_window"]},
        "step_roofline": {"bytes_per_step": key_b + gat_b, "achieved_gbs": (key_b + gat_b) / (m["step"] / 1e3) / 1e9,
                          "peak": hbm, "peak_source": hbm_kind,
                          "frac": (key_b + gat_b) / (m["step"] / 1e3) / 1e9 / hbm},
    }


def run_fp8(args):
    """Sparse MLA over the same selected rows of the batch-32 128K workload,
    with the latent cache in bf16 (1152 B a row) and in e4m3 (576 B a row, one
    per-tensor scale; the kernel widens rows to bf16 on chip).  Indices come
    from the library's indexer and selector; L2 is flushed before each call."""
    import statistics

    import torch

    import sparse_attention_decode_lightning_b200 as dsa
    from synth import get_workload, make_inputs

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    inp = make_inputs(get_workload(DEFAULT_WORKLOAD), seed=args.seed, device=dev, layers_to_make=1)
    Q, ix = inp.Q, inp.indexer[0]
    idx = torch.empty(Q, inp.topk, dtype=torch.int32, device=dev)
    ws = dsa.workspace(Q, inp.max_len, inp.topk, 0, device=dev)
    dsa.dsa_indexer_topk(ix["q_idx"], ix["w"], ix["k_idx"], inp.seq_offsets, inp.q_offsets,
                         inp.q_vis, inp.B, inp.max_len, inp.topk, idx, ws)
    pool = inp.layers[0]["pool"]
    codes = pool.to(torch.float8_e4m3fn).view(torch.uint8)
    out = torch.empty(Q, inp.heads, 512, device=dev)
    lse = torch.empty(Q, inp.heads, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    calls = {
        "bf16": lambda: dsa.dsa_sparse_mla_decode(inp.layers[0]["q"], pool, inp.page_table,
                                                  inp.q_offsets, inp.q_vis, idx, inp.B, inp.scale,
                                                  out, lse, ws, stream=stream),
        "e4m3": lambda: dsa.dsa_sparse_mla_decode_fp8(inp.layers[0]["q"], codes, 1.0, inp.page_table,
                                                      inp.q_offsets, inp.q_vis, idx, inp.B,
                                                      inp.scale, out, lse, ws, stream=stream),
    }
    res = {}
    for name, fn in calls.items():
        ts = []
        for i in range(max(3, args.warmup) + args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            if i >= max(3, args.warmup):
                ts.append(a.elapsed_time(b) * 1e3)
        res[name] = statistics.mean(ts)
    dsa.dsa_check_error(ws)
    rows = Q * inp.topk
    return {
        "metric": "sparse MLA + merge time, batch-32 128K selected rows: bf16 vs e4m3 latent cache",
        "value": res["e4m3"], "unit": "us", "higher_is_better": False, "n_gpus": 1,
        "steps": args.steps, "warmup": max(3, args.warmup), "data": "synthetic",
        "config": {"workload": DEFAULT_WORKLOAD, "rows": rows, "l2": "256 MiB flush before each call"},
        "us": res, "gather_bytes": {"bf16": rows * 1152, "e4m3": rows * 576},
    }


def run_fused(args):
    """Indexer + top-k selection of one layer of --workload, timed as the two
    kernels the decode step uses (dsa_indexer_topk) and in the histogram-fused
    form (dsa_indexer_topk_fused); L2 is flushed before each call."""
    import statistics

    import torch

    import sparse_attention_decode_lightning_b200 as dsa
    from synth import get_workload, make_inputs

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    inp = make_inputs(get_workload(args.workload), seed=args.seed, device=dev, layers_to_make=1)
    Q, ix = inp.Q, inp.indexer[0]
    first = bool(inp.mtp_index_share)
    idx = {k: torch.empty(Q, inp.topk, dtype=torch.int32, device=dev) for k in ("two", "fused")}
    ws = dsa.workspace(Q, inp.max_len, inp.topk, 0, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    fns = {"two_kernel": (dsa.dsa_indexer_topk, idx["two"]),
           "fused": (dsa.dsa_indexer_topk_fused, idx["fused"])}
    res = {}
    for name, (fn, out) in fns.items():
        ts = []
        for i in range(max(3, args.warmup) + args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn(ix["q_idx"], ix["w"], ix["k_idx"], inp.seq_offsets, inp.q_offsets, inp.q_vis,
               inp.B, inp.max_len, inp.topk, out, ws, first_only=first, stream=stream)
            b.record(stream)
            torch.cuda.synchronize(dev)
            if i >= max(3, args.warmup):
                ts.append(a.elapsed_time(b) * 1e3)
        dsa.dsa_check_error(ws)
        res[name] = statistics.mean(ts)
    # both forms select the same sets (rows compared sorted)
    same = bool(torch.equal(idx["two"].sort(dim=1).values, idx["fused"].sort(dim=1).values))
    return {
        "metric": "indexer + top-k time: two kernels vs histogram-fused",
        "value": res["fused"], "unit": "us", "higher_is_better": False, "n_gpus": 1,
        "steps": args.steps, "warmup": max(3, args.warmup), "data": "synthetic",
        "config": {"workload": args.workload, "B": inp.B, "Q": Q, "L": inp.max_len,
                   "topk": inp.topk, "idx_heads": inp.idx_heads,
                   "l2": "256 MiB flush before each call"},
        "us": res, "same_sets": same,
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.tier:
        if rank == 0:
            print(json.dumps(run_tier(args)), flush=True)
        return
    if args.csa:
        if rank == 0:
            print(json.dumps(run_csa(args)), flush=True)
        return
    if args.fp8:
        if rank == 0:
            print(json.dumps(run_fp8(args)), flush=True)
        return
    if args.fused:
        if rank == 0:
            print(json.dumps(run_fused(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
