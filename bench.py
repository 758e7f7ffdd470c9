"""Benchmark of the tree-verify step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ddt,reference}]
                    [--config 2] [--no-cpu-baseline] [--no-e2e]

One step is one pass of the whole verification path over one synthetic batch:
visibility mask -> tree-verify attention (with its split merge when used) ->
greedy accept -> KV compaction.  The default workload is 64 requests x q_len 33
(64 heads) x prefix 4096.  Prints one JSON line (rank 0).

value        verify-attention algorithmic TFLOP/s of the whole job: FLOPs of all
             ranks' steps / the max over ranks of the device-timed step time.
ms_per_step  device time of one step (CUDA events, max over ranks).
roofline     the verify kernel alone: algorithmic FLOPs per launch / its mean
             launch time (CUDA events on its stream) against the measured bf16
             dense peak.
e2e          the same metric through the public API with host buffers: each step
             copies its per-step inputs from pinned host memory, runs the step
             and reads the accepted tokens back.
cpu_baseline the CPU oracle on a bounded sample of the same workload (rank 0).

With N > 1 (torchrun) every rank runs its own batch (replicas, weak scaling);
there is no collective on the data path, only the timing reduction.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tree_speculative_decoding_05_b200 import inputs  # noqa: E402  (seeded generator only)

METRIC = "verify-attn µs/call & TFLOP/s (% bf16 peak), 64 streams × q_len 33 × 4K prefix"
H, DL, DR = 64, 512, 64
L2_BYTES = 126 * 1000 * 1000  # B200 L2 (126 MB)
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


# ---------------------------------------------------------------------------
# Work accounting (host side, from the workload's tree shapes)
# ---------------------------------------------------------------------------

def tree_depths(parents: np.ndarray) -> np.ndarray:
    depth = np.zeros_like(parents)
    for b in range(parents.shape[0]):
        for i in range(1, parents.shape[1]):
            depth[b, i] = depth[b, parents[b, i]] + 1
    return depth


def verify_flops(prefix_lens: np.ndarray, parents: np.ndarray, heads: int = H) -> float:
    """Algorithmic FLOPs of one verify call: every (request, node, head) row does a
    576-wide dot product and a 512-wide accumulation per visible key; masked keys
    are not counted.  Visible keys of node i: P + depth(i) + 1."""
    depth = tree_depths(parents)
    visible = prefix_lens[:, None].astype(np.float64) + depth + 1
    return float(heads * 2 * (DL + DR + DL) * visible.sum())


def verify_bytes(prefix_lens: np.ndarray, q_len: int, out_bytes: int, want_lse: bool) -> float:
    """Algorithmic bytes: queries read once, each request's KV rows read once,
    outputs (and lse) written once."""
    B = prefix_lens.shape[0]
    q = B * q_len * H * (DL + DR) * 2
    kv = float((prefix_lens.astype(np.float64) + q_len).sum()) * (DL + DR) * 2
    out = B * q_len * H * DL * out_bytes + (B * q_len * H * 4 if want_lse else 0)
    return q + kv + out


def flops_rows(prefix_lens, parents, rows, heads=H) -> float:
    """FLOPs of a subset of query rows (flat (b*Q + i)*H + h)."""
    depth = tree_depths(parents)
    Q = parents.shape[1]
    b = rows // (Q * heads)
    i = (rows // heads) % Q
    vis = prefix_lens[b].astype(np.float64) + depth[b, i] + 1
    return float(2 * (DL + DR + DL) * vis.sum())


# ---------------------------------------------------------------------------
# Peaks and clocks
# ---------------------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "verify_attn_config2.json")


def kernel_source_hash() -> str:
    """sha256 of the verify kernel's sources (the kernel file and its PTX header)."""
    import hashlib
    csrc = os.path.join(ROOT, "tree_speculative_decoding_05_b200", "csrc")
    src = b"".join(open(os.path.join(csrc, f), "rb").read() for f in ("verify_attn.cu", "sm100_ptx.cuh"))
    return hashlib.sha256(src).hexdigest()


def measured_traffic(config_idx: int):
    """DRAM bytes per verify launch of the default workload from the machine-written
    record of its ncu capture (see record_traffic), or None when there is no record
    or the kernel source changed since it was taken."""
    if config_idx != 2:
        return None
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return float(rec["traffic_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


_BYTE_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
               "kibyte": 1024.0, "mibyte": 1024.0 ** 2, "gibyte": 1024.0 ** 3}


def record_traffic(csv_path: str, command: str) -> int:
    """Write the traffic record from `ncu -i <capture> --page raw --csv` output of
    the verify kernel: the mean over the captured launches of
    dram__bytes_read.sum + dram__bytes_write.sum, with the current source hash."""
    import csv
    with open(csv_path, newline="") as f:
        rows = [r for r in csv.reader(f) if r]
    head = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    names, units = rows[head], rows[head + 1]
    col = {n: i for i, n in enumerate(names)}
    launches = []
    for r in rows[head + 2:]:
        if len(r) != len(names) or "verify_attn_kernel" not in r[col["Kernel Name"]]:
            continue
        vals = {}
        for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            scale = _BYTE_UNITS[units[col[m]].strip().lower()]
            vals[m] = float(r[col[m]].replace(",", "")) * scale
        launches.append(vals)
    if not launches:
        raise SystemExit(f"no verify_attn_kernel launch with DRAM byte counters in {csv_path}")
    rd = sum(v["dram__bytes_read.sum"] for v in launches) / len(launches)
    wr = sum(v["dram__bytes_write.sum"] for v in launches) / len(launches)
    rec = {"kernel": "verify_attn_kernel",
           "workload": "64 requests x q_len 33 x 64 heads x prefix 4096, bf16 out",
           "command": command, "launches": len(launches),
           "dram_bytes_read_per_launch": rd, "dram_bytes_write_per_launch": wr,
           "traffic_bytes_per_launch": rd + wr,
           "kernel_source_sha256": kernel_source_hash()}
    with open(TRAFFIC_RECORD, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))
    return 0


class ClockSampler:
    """Samples SM clocks and throttle reasons while running: nvidia-smi every
    100 ms, and NVML in-process every ~2 ms.  A timed region of a few tens of ms
    falls between nvidia-smi's samples, so the summary takes the NVML samples
    inside the region marked by begin() / end() when there are at least three,
    else the nvidia-smi samples."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits and the names nvidia-smi gives them
    REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                   0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int, device=None):
        self.gpu = gpu_index
        self.device = device
        self.proc = None
        self.lines: list[str] = []
        self.nvml_samples: list[tuple[float, float, int]] = []  # (time, SM MHz, reasons)
        self.nvml_max = None
        self.region = (None, None)
        self._stop = threading.Event()
        self._nvml_thread = None

    def _nvml_start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            if self.device is not None:
                import torch
                pr = torch.cuda.get_device_properties(self.device)
                bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
                try:
                    h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
                except pynvml.NVMLError:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu))
            self.nvml_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            return

        def poll():
            while not self._stop.is_set():
                try:
                    mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    rs = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
                    self.nvml_samples.append((time.perf_counter(), mhz, rs))
                except Exception:
                    return
                time.sleep(0.002)

        self._nvml_thread = threading.Thread(target=poll, daemon=True)
        self._nvml_thread.start()

    def begin(self):
        self.region = (time.perf_counter(), None)

    def end(self):
        self.region = (self.region[0], time.perf_counter())

    def __enter__(self):
        self._nvml_start()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            # Start the timed region only once sampling is live.
            deadline = time.time() + 5.0
            while not self.lines and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            # One more sample after the region, so a short region is bracketed.
            n = len(self.lines)
            deadline = time.time() + 1.0
            while len(self.lines) == n and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self._stop.set()
        if self._nvml_thread is not None:
            self._nvml_thread.join(timeout=1.0)

    def summary(self):
        t0, t1 = self.region
        inside = [(m, r) for (t, m, r) in self.nvml_samples
                  if t0 is not None and t1 is not None and t0 <= t <= t1]
        if len(inside) >= 3:
            reasons = set()
            for _, r in inside:
                for bit, name in self.REASON_BITS.items():
                    if r & bit:
                        reasons.add(name)
            return {"sm_mhz": statistics.median(m for m, _ in inside),
                    "sm_max_mhz": self.nvml_max, "reasons": sorted(reasons),
                    "samples": len(inside), "source": "NVML every ~2 ms inside the timed region"}
        return self._smi_summary()

    def _smi_summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi every 100 ms around the timed region"}


def choose_peak(peaks: dict, timed_s: float, clk: dict):
    """The roofline's bf16 denominator: the sustained peak (measured under the
    power cap) when the timed region ran power-capped, i.e. lasted over 2 s, or
    its in-region NVML samples show sw_power_cap with the median SM clock below
    95 % of its maximum; else the burst peak.  Returns (peak, sustained?, why)."""
    capped = (str(clk.get("source") or "").startswith("NVML")
              and "sw_power_cap" in (clk.get("reasons") or [])
              and bool(clk.get("sm_mhz")) and bool(clk.get("sm_max_mhz"))
              and clk["sm_mhz"] < 0.95 * clk["sm_max_mhz"])
    sustained = timed_s > 2.0 or capped
    why = ("" if not sustained else
           " (timed region over 2 s)" if timed_s > 2.0 else
           f" (power-capped: median {clk['sm_mhz']:.0f} of {clk['sm_max_mhz']:.0f} MHz with "
           f"sw_power_cap in the timed region)")
    peak = peaks.get("bf16_tflops_sustained" if sustained else "bf16_tflops",
                     FALLBACK_BF16_TFLOPS)
    return peak, sustained, why


def physical_gpu_index(local: int) -> str:
    """nvidia-smi's index of the GPU this process uses."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


# ---------------------------------------------------------------------------
# Distributed plumbing (timing reduction only)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(values: list[float], world: int, device) -> list[float]:
    """Element-wise max over ranks (identity on one rank)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def reduce_sum(values: list[float], world: int, device) -> list[float]:
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()]


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

def oracle_sample_throughput(w, target_seconds: float, seed: int = 0, max_rows: int = 1 << 16):
    """Run the CPU oracle on random query rows of the workload until about
    target_seconds of CPU work; returns (TFLOP/s, rows, seconds, threads)."""
    import oracle
    rng = np.random.RandomState(seed)
    total = w.B * w.q_len * H
    done_rows, flops, secs = 0, 0.0, 0.0
    chunk = max(16, oracle.threads() * 4)
    while secs < target_seconds and done_rows < max_rows:
        rows = np.sort(rng.choice(total, size=min(chunk, total), replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens, w.parents,
                         w.softmax_scale, rows)
        secs += time.perf_counter() - t0
        flops += flops_rows(w.prefix_lens, w.parents, rows)
        done_rows += len(rows)
        chunk = min(chunk * 2, 4096)
    return flops / secs / 1e12, done_rows, secs, oracle.threads()


def run_reference(args, w):
    """--impl reference: the CPU oracle as it stands.  Each step is the whole path
    (mask, every query row of the attention, accept, compaction) for one request
    of the batch, requests taken in turn: a bounded sample with the same mix of
    work as the GPU step."""
    import oracle
    B = w.B
    subs = {}

    def step(k):
        b = k % B
        if b not in subs:
            subs[b] = inputs.subset(w, [b])
        x = subs[b]
        rows = np.arange(x.q_len * H, dtype=np.int64)
        oracle.build_mask(x.parents)
        oracle.attn_rows(x.q_lat, x.q_rope, x.c_kv, x.k_rope, x.prefix_lens, x.parents,
                         x.softmax_scale, rows)
        path, alen, _, _ = oracle.tree_accept(x.node_tokens, x.target_tokens, x.next_token,
                                              x.next_sibling)
        oracle.kv_compact(x.c_kv, x.k_rope, x.prefix_lens, path, alen)
        return verify_flops(x.prefix_lens, x.parents)

    for k in range(args.warmup):
        step(k)
    t0 = time.perf_counter()
    flops = 0.0
    for k in range(args.steps):
        flops += step(args.warmup + k)
    secs = time.perf_counter() - t0
    value = flops / secs / 1e12
    sample = (f"per step one request of the {B}-request batch, in turn: its mask, all "
              f"{w.q_len * H} query rows of its attention, its accept walk and compaction")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "q_len": w.q_len, "heads": H,
                   "prefix": int(w.prefix_lens.max()), "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Main (GPU arm)
# ---------------------------------------------------------------------------

DRAFT_DEPTH, DRAFT_TOPK = 15, 8  # drafter rows (tree depth <= 15) and candidates per row


def l2_flush(buf) -> None:
    """Evict the L2 by READING a buffer larger than it (a reduction over 256 MB).
    A read leaves clean lines behind; a flush that wrote the buffer would leave
    126 MB of dirty lines whose write-back the next, timed call would pay for."""
    buf.view(torch_int64()).sum()


def torch_int64():
    import torch
    return torch.int64


def graph_time_us(fn, n: int, flush=None, reps: int = 5) -> float:
    """Mean device time of one fn() call: n calls back to back captured in one CUDA
    graph (so host launch overhead is not timed), the graph replayed `reps` times
    with events around each replay, median of those.  With `flush` (a buffer larger
    than L2), every call is preceded by a read of it (l2_flush), and a graph of the
    n flushes alone is timed the same way and subtracted."""
    import torch

    def capture(body):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            body()  # untimed warm-up outside the capture
            side.synchronize()
            with torch.cuda.graph(g, stream=side):
                for k in range(n):
                    body(k)
        torch.cuda.current_stream().wait_stream(side)
        return g

    def replay_ms(g):
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        return statistics.median(times)

    def with_flush(k=0):
        if flush is not None:
            l2_flush(flush)
        fn()

    total = replay_ms(capture(with_flush))
    if flush is not None:
        total -= replay_ms(capture(lambda k=0: l2_flush(flush)))
    return max(total, 0.0) / n * 1e3


def time_extras(w, d, host, mask, out, lse, workspace, max_prefix, stream, flush, iters,
                warmup):
    """Mean device time (us) of the calls outside the benchmark step, each timed as
    `iters` calls in one CUDA graph (L2 flushed before every call when the inputs
    fit in it, the flush's own time subtracted):
    the tree build of drafts of the workload's shape; tree_accept then kv_compact
    against the fused accept_compact; and one chained decode step (tree build, block
    write, verify, accept + compaction) replayed from a CUDA graph with its state
    reset by the graph itself."""
    import torch

    from tree_speculative_decoding_05_b200 import ddt

    dev = d["q_lat"].device
    B, Q = w.B, w.q_len

    def timed(fn):
        for _ in range(warmup):
            fn()
        return graph_time_us(fn, iters, flush)

    draft = inputs.draft_batch(w.seed, B, DRAFT_DEPTH, DRAFT_TOPK)
    lp = torch.from_numpy(draft.lp).to(dev)
    tok = torch.from_numpy(draft.tok).to(dev)
    root = torch.from_numpy(draft.root_token).to(dev)
    tb = ddt.tree_build(lp, tok, root, Q)
    res = {"draft": f"{DRAFT_DEPTH} rows x top-{DRAFT_TOPK} per request"}
    res["tree_build_us"] = timed(lambda: ddt.tree_build(lp, tok, root, Q, out=tb))

    i32 = lambda shape: torch.empty(shape, dtype=torch.int32, device=dev)
    path, alen, bonus, ast, newp, cst = i32((B, Q)), i32(B), i32(B), i32(B), i32(B), i32(B)

    def separate():
        ddt.tree_accept(d["node_tokens"], d["target_tokens"], d["next_token"], d["next_sibling"],
                        path=path, accept_len=alen, bonus=bonus, status=ast)
        ddt.kv_compact(d["c_kv"], d["k_rope"], d["prefix"], path, alen, new_prefix_lens=newp,
                       status=cst)

    def fused():
        ddt.accept_compact(d["node_tokens"], d["target_tokens"], d["next_token"],
                           d["next_sibling"], d["c_kv"], d["k_rope"], d["prefix"], path=path,
                           accept_len=alen, bonus=bonus, accept_status=ast,
                           new_prefix_lens=newp, compact_status=cst)

    res["accept_then_compact_us"] = timed(separate)
    res["accept_compact_us"] = timed(fused)

    # Chained decode step: the workload's queries and its own tree-block rows,
    # drafts as above, and a target continuation that follows the drafter's top
    # token with probability 0.7.
    rows = torch.from_numpy(np.stack([np.arange(int(p), int(p) + Q) for p in w.prefix_lens]))
    bidx = torch.arange(B)[:, None]
    u = inputs.uniform(inputs.stream_base(w.seed, 97, 0), 0, B * Q).reshape(B, Q)
    cont = np.where((u < 0.7) & (np.arange(Q)[None, :] < DRAFT_DEPTH),
                    draft.tok[:, np.minimum(np.arange(Q), DRAFT_DEPTH - 1), 0], 31999)
    step = dict(lp=lp, tok=tok, q_lat=d["q_lat"], q_rope=d["q_rope"],
                block_ckv=host["c_kv"][bidx, rows].contiguous().to(dev),
                block_krope=host["k_rope"][bidx, rows].contiguous().to(dev),
                target_continuation=torch.from_numpy(cont.astype(np.int32)).to(dev))
    state = dict(c_kv=d["c_kv"], k_rope=d["k_rope"], prefix_lens=d["prefix"].clone(),
                 root_token=root.clone())
    p0, r0 = d["prefix"].clone(), root.clone()
    bufs = dict(mask=mask, out=out, lse=lse, workspace=workspace, verify_status=i32(B),
                parents=i32((B, Q)), node_tokens=i32((B, Q)), depth=i32((B, Q)),
                next_token=i32((B, Q)), next_sibling=i32((B, Q)), n_nodes=i32(B),
                target_tokens=i32((B, Q)), path=path, accept_len=alen, status=i32((4, B)))
    dargs = ddt.decode_step_args(state, step, bufs, w.softmax_scale, max_prefix)

    def one_step():
        state["prefix_lens"].copy_(p0)
        state["root_token"].copy_(r0)
        ddt.decode_step(dargs)

    one_step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            one_step()
    torch.cuda.current_stream(dev).wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for k, (a, b) in enumerate(evs):
        if flush is not None:
            l2_flush(flush)
        a.record(stream)
        graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    res["decode_step_us"] = sum(a.elapsed_time(b) for a, b in evs) / iters * 1e3
    st = bufs["status"].cpu().numpy()
    res["decode_step_statuses_ok"] = bool((st == 0).all() and
                                          (bufs["verify_status"].cpu().numpy() == 0).all())
    res["decode_step_mean_accept_len"] = float(alen.float().mean().item())
    res["decode_step_kernels"] = 4 + (1 if workspace is not None else 0)
    del graph
    return res


def per_config_report(configs, peaks, device, preloaded=None):
    """Every workload's calls timed on this run's GPU (the bench line's
    `per_config`): for each config the inputs are generated and moved to the
    device, each call runs 5 times untimed, then n calls are captured back to back
    in one CUDA graph and the replay is timed with CUDA events on the launching
    stream, median of 5 replays (n = 100, or 20 for calls over 0.5 ms).  When the
    workload's inputs are under twice the L2, a 256 MB read precedes every call
    and a graph of the writes alone is timed and subtracted; those workloads'
    calls are also timed with a warm L2 (no read between calls), reported beside
    them as `calls_us_warm_l2`.  Reported: µs per
    call of build_mask, verify_attn (with its split merge), tree_accept and
    kv_compact; verify TFLOP/s as a fraction of the burst and the sustained bf16
    peak; the KV stream's and the compaction's GB/s."""
    import torch

    from tree_speculative_decoding_05_b200 import ddt

    peak_b = peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)
    peak_s = peaks.get("bf16_tflops_sustained", peak_b)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    res = {}
    for cfg in configs:
        w = (preloaded or {}).get(cfg) or inputs.config(cfg)
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
            torch.bfloat16).to(device)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
        q_lat, q_rope, c_kv, k_rope = bf(w.q_lat), bf(w.q_rope), bf(w.c_kv), bf(w.k_rope)
        prefix, parents = i32(w.prefix_lens), i32(w.parents)
        nt, tt, fc, ns = (i32(w.node_tokens), i32(w.target_tokens), i32(w.next_token),
                          i32(w.next_sibling))
        B, Q = w.B, w.q_len
        max_prefix = int(w.prefix_lens.max())
        mask, depth, mst = ddt.build_mask(parents)
        od = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
        out = torch.empty((B, Q, H, DL), dtype=od, device=device)
        lse = torch.empty((B, Q, H), dtype=torch.float32, device=device) if w.want_lse else None
        ws, splits = ddt.verify_attn_workspace_size(q_lat, q_rope, c_kv, k_rope, prefix, mask,
                                                    w.softmax_scale, max_prefix)
        wsp = torch.empty(ws, dtype=torch.uint8, device=device) if ws else None
        path = torch.empty((B, Q), dtype=torch.int32, device=device)
        alen = torch.empty((B,), dtype=torch.int32, device=device)
        newp = torch.empty((B,), dtype=torch.int32, device=device)
        vst = torch.empty((B,), dtype=torch.int32, device=device)
        ddt.tree_accept(nt, tt, fc, ns, path=path, accept_len=alen)
        input_bytes = sum(t.numel() * t.element_size() for t in (q_lat, q_rope, c_kv, k_rope))
        fl = flush if input_bytes < 2 * L2_BYTES else None
        calls = {
            "build_mask": lambda: ddt.build_mask(parents, mask=mask, depth=depth, status=mst),
            "verify_attn": lambda: ddt.verify_attn(q_lat, q_rope, c_kv, k_rope, prefix, mask,
                                                   w.softmax_scale, max_prefix=max_prefix,
                                                   out=out, lse=lse, workspace=wsp,
                                                   status=vst),
            "tree_accept": lambda: ddt.tree_accept(nt, tt, fc, ns, path=path, accept_len=alen),
            "kv_compact": lambda: ddt.kv_compact(c_kv, k_rope, prefix, path, alen,
                                                 new_prefix_lens=newp),
        }
        us, us_warm = {}, {}
        for name, fn in calls.items():
            for _ in range(5):
                fn()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            fn()
            torch.cuda.synchronize()
            n = 20 if time.perf_counter() - t0 > 0.5e-3 else 100
            us[name] = graph_time_us(fn, n, fl, reps=5)
            if fl is not None:
                us_warm[name] = graph_time_us(fn, n, None, reps=5)
        torch.cuda.synchronize()
        path_h, alen_h = path.cpu().numpy(), alen.cpu().numpy()
        moved = sum(int((path_h[b, :alen_h[b]] != np.arange(alen_h[b])).sum()) for b in range(B))
        flops = verify_flops(w.prefix_lens, w.parents)
        tflops = flops / (us["verify_attn"] * 1e-6) / 1e12
        res[str(cfg)] = {
            "workload": w.name, "B": B, "q_len": Q, "prefix_max": max_prefix,
            "out": w.out_dtype, "lse": bool(w.want_lse), "kv_splits": splits,
            "calls_us": us,
            **({"calls_us_warm_l2": us_warm} if us_warm else {}),
            "verify_gflop": flops / 1e9,
            "verify_tflops": tflops,
            "verify_frac_burst": tflops / peak_b,
            "verify_frac_sustained": tflops / peak_s,
            "kv_stream_gbs": float((w.prefix_lens.astype(np.float64) + Q).sum()) * (DL + DR) * 2
                             / (us["verify_attn"] * 1e-6) / 1e9,
            "kv_compact_rows_moved": moved,
            "kv_compact_gbs": 2.0 * moved * (DL + DR) * 2 / (us["kv_compact"] * 1e-6) / 1e9,
            "statuses_ok": bool((vst.cpu().numpy() == 0).all() and (mst.cpu().numpy() == 0).all()),
            "l2": "flushed before every call (flush subtracted)" if fl is not None
                  else "inputs over twice the L2: no flush",
        }
        del q_lat, q_rope, c_kv, k_rope, out, lse, wsp, calls
        torch.cuda.empty_cache()
    return res


def per_call_report(args) -> int:
    """Every call of the path timed alone per workload: 10 warm-up calls, then 100
    calls captured back to back in a CUDA graph and the replay timed with events,
    median of 5 replays; with a warm L2, and with a 256 MB read before every call
    (the writes' own time subtracted).  The oracle runs on the same workload (configs
    0 and 1 whole; larger ones on a sample of query rows) with all host threads and
    with one."""
    import torch

    import oracle
    from tree_speculative_decoding_05_b200 import ddt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = measured_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)
    peak_sustained = peaks.get("bf16_tflops_sustained", peak)

    def timed(fn, flushed):
        # 10 untimed calls, then 100 calls per graph, median of 5 replays
        for _ in range(10):
            fn()
        return graph_time_us(fn, 100, flush if flushed else None, reps=5)

    for cfg in [int(c) for c in args.configs.split(",") if c.strip()]:
        w = inputs.config(cfg)
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
            torch.bfloat16).to(dev)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        q_lat, q_rope, c_kv, k_rope = bf(w.q_lat), bf(w.q_rope), bf(w.c_kv), bf(w.k_rope)
        prefix, parents = i32(w.prefix_lens), i32(w.parents)
        nt, tt, fc, ns = (i32(w.node_tokens), i32(w.target_tokens), i32(w.next_token),
                          i32(w.next_sibling))
        B, Q = w.B, w.q_len
        max_prefix = int(w.prefix_lens.max())
        mask, depth, mst = ddt.build_mask(parents)
        od = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
        out = torch.empty((B, Q, H, DL), dtype=od, device=dev)
        lse = torch.empty((B, Q, H), dtype=torch.float32, device=dev) if w.want_lse else None
        ws, splits = ddt.verify_attn_workspace_size(q_lat, q_rope, c_kv, k_rope, prefix, mask,
                                                    w.softmax_scale, max_prefix)
        wsp = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev) if ws else None
        a_st = ddt._attn_args(q_lat, q_rope, c_kv, k_rope, prefix, mask, w.softmax_scale, out,
                              lse, max_prefix, 0, None, None)
        ws_st = int(ddt.load().ddt_verify_attn_split_tail_workspace_size(ctypes.byref(a_st)))
        wsp_st = torch.empty(ws_st, dtype=torch.uint8, device=dev)
        path, alen = torch.empty((B, Q), dtype=torch.int32, device=dev), \
            torch.empty((B,), dtype=torch.int32, device=dev)
        ddt.tree_accept(nt, tt, fc, ns, path=path, accept_len=alen)
        newp = torch.empty((B,), dtype=torch.int32, device=dev)
        draft = inputs.draft_batch(w.seed, B, DRAFT_DEPTH, DRAFT_TOPK)
        lp, tok, root = (torch.from_numpy(draft.lp).to(dev), torch.from_numpy(draft.tok).to(dev),
                         torch.from_numpy(draft.root_token).to(dev))
        tb = ddt.tree_build(lp, tok, root, Q)
        calls = {
            "tree_build": lambda: ddt.tree_build(lp, tok, root, Q, out=tb),
            "build_mask": lambda: ddt.build_mask(parents, mask=mask, depth=depth, status=mst),
            "verify_attn": lambda: ddt.verify_attn(q_lat, q_rope, c_kv, k_rope, prefix, mask,
                                                   w.softmax_scale, max_prefix=max_prefix,
                                                   out=out, lse=lse, workspace=wsp),
            "verify_attn_split_tail": lambda: ddt.verify_attn(
                q_lat, q_rope, c_kv, k_rope, prefix, mask, w.softmax_scale,
                max_prefix=max_prefix, out=out, lse=lse, workspace=wsp_st, split_tail=True),
            "tree_accept": lambda: ddt.tree_accept(nt, tt, fc, ns, path=path, accept_len=alen),
            "kv_compact": lambda: ddt.kv_compact(c_kv, k_rope, prefix, path, alen,
                                                 new_prefix_lens=newp),
            "accept_compact": lambda: ddt.accept_compact(nt, tt, fc, ns, c_kv, k_rope, prefix,
                                                         path=path, accept_len=alen,
                                                         new_prefix_lens=newp),
        }
        res = {}
        for name, fn in calls.items():
            res[name] = {"warm_us": timed(fn, False), "l2_flushed_us": timed(fn, True)}
        flops = verify_flops(w.prefix_lens, w.parents)
        for name in ("verify_attn", "verify_attn_split_tail"):
            us = res[name]["l2_flushed_us"]
            res[name]["tflops"] = flops / (us * 1e-6) / 1e12
            # a replay of 100 back-to-back calls runs long enough to reach the power cap
            res[name]["frac_of_burst_peak"] = res[name]["tflops"] / peak
            res[name]["frac_of_sustained_peak"] = res[name]["tflops"] / peak_sustained
        # the oracle: whole workload for the two small configs, else a row sample
        total = B * Q * H
        rng = np.random.RandomState(cfg)
        rows = np.arange(total, dtype=np.int64) if cfg in (0, 1) else \
            np.sort(rng.choice(total, size=min(total, 4096), replace=False)).astype(np.int64)
        orc = {}
        for label, nth in (("all_threads", 0), ("one_thread", 1)):
            if nth == 1 and cfg not in (0, 1):
                continue
            t0 = time.perf_counter()
            oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens, w.parents,
                             w.softmax_scale, rows, nthreads=nth)
            secs = time.perf_counter() - t0
            orc[label] = {"seconds": secs, "rows": int(len(rows)),
                          "tflops": flops_rows(w.prefix_lens, w.parents, rows) / secs / 1e12}
        orc["threads"] = oracle.threads()
        print(json.dumps({"workload": w.name, "config": cfg, "kv_splits": splits,
                          "peak_tflops": peak, "peak_sustained_tflops": peak_sustained,
                          "peak_source": f"{peak_src} bf16",
                          "calls_us": res, "oracle": orc}), flush=True)
    return 0


def accept_sweep() -> int:
    """tree_accept timed alone on random trees (depth <= 15) for streams {1, 8, 64} x
    draft budget {8, 32} (q_len = budget + 1): 100 calls in a CUDA graph, median of 5."""
    import torch

    from tree_speculative_decoding_05_b200 import ddt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    res = {}
    for streams in (1, 8, 64):
        for budget in (8, 32):
            w = inputs.make_workload("accept", 500 + streams + budget, streams, budget + 1,
                                     [0] * streams, heads=1, d_latent=8, d_rope=8)
            t = {k: torch.from_numpy(np.ascontiguousarray(getattr(w, k))).to(dev)
                 for k in ("node_tokens", "target_tokens", "next_token", "next_sibling")}
            path = torch.empty((streams, budget + 1), dtype=torch.int32, device=dev)
            alen = torch.empty((streams,), dtype=torch.int32, device=dev)
            fn = lambda: ddt.tree_accept(t["node_tokens"], t["target_tokens"], t["next_token"],
                                         t["next_sibling"], path=path, accept_len=alen)
            for _ in range(10):
                fn()
            res[f"streams={streams},budget={budget}"] = graph_time_us(fn, 100)
    print(json.dumps({"tree_accept_us": res, "timing": "100 calls per CUDA graph, median of 5"}),
          flush=True)
    return 0


def compact_scale() -> int:
    """kv_compact on batches large enough to be bound by HBM rather than by launch
    latency: 1024 requests, q_len 128, 256-row prefixes, separate contiguous caches
    (453 MB), with accepted paths that move most rows: the reversed block (alen 128,
    keep[i] = 127 - i: every row moves) and every second node (alen 64, keep[i] = 2 i:
    63 rows move).  Bytes per call = every moved row read once and written once
    (1152 B each).  Two copies of the caches (906 MB) alternate call by call, so a
    call never finds the rows it reads in the L2 and no flush is needed: 20 calls
    per CUDA graph, median of 5 replays, CUDA events.  One JSON line."""
    import torch

    from tree_speculative_decoding_05_b200 import ddt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = measured_peaks()
    B, Q, P = 1024, 128, 256
    cap = P + Q
    gen = torch.Generator(device=dev)
    gen.manual_seed(12)
    bits = lambda d: torch.randint(-32768, 32768, (B, cap, d), dtype=torch.int32, device=dev,
                                   generator=gen).to(torch.int16).view(torch.bfloat16)
    caches = [(bits(DL), bits(DR)) for _ in range(2)]
    prefix = torch.full((B,), P, dtype=torch.int32, device=dev)
    newp = torch.empty_like(prefix)
    status = torch.empty_like(prefix)
    res = {}
    for name, alen_v, keep in (("reversed block", Q, [Q - 1 - i for i in range(Q)]),
                               ("every second node", Q // 2, [2 * i for i in range(Q // 2)])):
        row = np.zeros(Q, dtype=np.int32)
        row[:alen_v] = keep
        path = torch.from_numpy(np.tile(row, (B, 1))).to(dev)
        alen = torch.full((B,), alen_v, dtype=torch.int32, device=dev)
        moved = sum(1 for i, k in enumerate(keep) if k != i)
        calls = [0]

        def fn(k=None):
            c_kv, k_rope = caches[calls[0] % 2]
            calls[0] += 1
            ddt.kv_compact(c_kv, k_rope, prefix, path, alen, new_prefix_lens=newp, status=status)

        for _ in range(4):
            fn()
        torch.cuda.synchronize()
        assert bool((status == 0).all()), "kv_compact status"
        us = graph_time_us(fn, 20)
        nbytes = 2.0 * B * moved * (DL + DR) * 2
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"alen": alen_v, "rows_moved_per_request": moved, "bytes_per_call": nbytes,
                     "us_per_call": us, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"]}
    print(json.dumps({"kv_compact_at_scale": res, "requests": B, "q_len": Q, "prefix": P,
                      "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
                      "timing": "20 calls per CUDA graph alternating between two 453 MB cache "
                                "copies (no L2 flush needed), median of 5 replays"}), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ddt", "reference"], default="ddt")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--per-call", action="store_true",
                    help="instead of the step benchmark: every call of the path timed alone on "
                         "each workload (10 warm-up + 100 timed calls, median of 5 repetitions, "
                         "warm L2 and after a 256 MB L2 flush), plus the oracle on all host "
                         "cores and on one; one JSON line per workload")
    ap.add_argument("--configs", type=str, default="0,1,2,3,4")
    ap.add_argument("--accept-sweep", action="store_true",
                    help="tree_accept alone over streams {1, 8, 64} x budget {8, 32} (the grid "
                         "the pages report), graph-timed; one JSON line")
    ap.add_argument("--compact-scale", action="store_true",
                    help="kv_compact alone on 1024 requests x q_len 128 with paths that move "
                         "most rows (HBM-bound, not latency-bound); one JSON line")
    ap.add_argument("--shard", choices=["replicas", "lpt"], default="replicas",
                    help="with several GPUs: every rank runs its own batch of the workload "
                         "(replicas, weak scaling) or the ranks split one batch by request "
                         "with the longest-first rule (strong scaling)")
    ap.add_argument("--record-traffic", metavar="RAW_CSV",
                    help="write the verify kernel's DRAM traffic record (profiles/"
                         "verify_attn_config2.json) from `ncu -i <capture> --page raw --csv` "
                         "output; no GPU needed")
    ap.add_argument("--capture-command", default="",
                    help="with --record-traffic: the ncu command that made the capture")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-call timings of all five workloads")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the timings of the calls outside the step (tree build, fused "
                         "accept+compaction, chained decode step)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_env()

    if args.record_traffic:
        return record_traffic(args.record_traffic, args.capture_command)
    if args.per_call:
        return per_call_report(args)
    if args.accept_sweep:
        return accept_sweep()
    if args.compact_scale:
        return compact_scale()
    if args.impl == "reference":
        if rank != 0:
            return 0
        run_reference(args, inputs.config(args.config))
        return 0

    import torch

    from tree_speculative_decoding_05_b200 import ddt

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    # Every rank runs its own batch of the same shape (independent requests), or,
    # with --shard lpt, its longest-first share of one batch.
    w = inputs.config(args.config)
    if args.shard == "lpt" and world > 1:
        from tree_speculative_decoding_05_b200.sharding import lpt_partition, request_costs
        part = lpt_partition(request_costs(w.prefix_lens, w.q_len), world)[rank]
        if len(part) == 0:
            raise SystemExit("--shard lpt: more ranks than requests")
        w = inputs.subset(w, part)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32))

    host = {
        "q_lat": bf16(w.q_lat), "q_rope": bf16(w.q_rope), "c_kv": bf16(w.c_kv),
        "k_rope": bf16(w.k_rope), "prefix": i32(w.prefix_lens), "parents": i32(w.parents),
        "node_tokens": i32(w.node_tokens), "target_tokens": i32(w.target_tokens),
        "next_token": i32(w.next_token), "next_sibling": i32(w.next_sibling),
    }
    d = {k: v.to(device) for k, v in host.items()}
    out_dtype = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    B, Q = w.B, w.q_len
    max_prefix = int(w.prefix_lens.max())
    mask = torch.empty((B, Q, (Q + 63) // 64), dtype=torch.int64, device=device)
    depth = torch.empty((B, Q), dtype=torch.int32, device=device)
    mstatus = torch.empty((B,), dtype=torch.int32, device=device)
    out = torch.empty((B, Q, H, DL), dtype=out_dtype, device=device)
    lse = torch.empty((B, Q, H), dtype=torch.float32, device=device) if w.want_lse else None
    vstatus = torch.empty((B,), dtype=torch.int32, device=device)
    ws_bytes, splits = ddt.verify_attn_workspace_size(
        d["q_lat"], d["q_rope"], d["c_kv"], d["k_rope"], d["prefix"], mask, w.softmax_scale,
        max_prefix)
    workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    path = torch.empty((B, Q), dtype=torch.int32, device=device)
    alen = torch.empty((B,), dtype=torch.int32, device=device)
    bonus = torch.empty((B,), dtype=torch.int32, device=device)
    astatus = torch.empty((B,), dtype=torch.int32, device=device)
    newp = torch.empty((B,), dtype=torch.int32, device=device)
    cstatus = torch.empty((B,), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None, src=None):
        # ev: five events bracketing mask | verify | accept | compact; src: the
        # per-step inputs (default: the resident copies in d)
        x = d if src is None else src
        if ev is not None:
            ev[0].record(stream)
        ddt.build_mask(x["parents"], mask=mask, depth=depth, status=mstatus)
        if ev is not None:
            ev[1].record(stream)
        ddt.verify_attn(x["q_lat"], x["q_rope"], d["c_kv"], d["k_rope"], x["prefix"], mask,
                        w.softmax_scale, max_prefix=max_prefix, out=out, lse=lse,
                        workspace=workspace if ws_bytes else None, status=vstatus)
        if ev is not None:
            ev[2].record(stream)
        ddt.tree_accept(x["node_tokens"], x["target_tokens"], x["next_token"],
                        x["next_sibling"], path=path, accept_len=alen, bonus=bonus,
                        status=astatus)
        if ev is not None:
            ev[3].record(stream)
        ddt.kv_compact(d["c_kv"], d["k_rope"], x["prefix"], path, alen, new_prefix_lens=newp,
                       status=cstatus)
        if ev is not None:
            ev[4].record(stream)

    launches_per_step = 4 + (1 if splits > 1 else 0)
    # Inputs smaller than twice the L2 would be served from a warm L2: then the L2 is
    # flushed (a 256 MB read) between timed steps, outside the steps' events.
    input_bytes = sum(v.numel() * v.element_size() for k, v in d.items())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device) \
        if input_bytes < 2 * L2_BYTES else None

    def flush_l2(k):
        if flush is not None:
            l2_flush(flush)
    ddt.fault_flags(reset=True)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(physical_gpu_index(local), device) as clocks:
        torch.cuda.synchronize()
        clocks.begin()
        t_start.record(stream)
        for k in range(args.steps):
            flush_l2(k)
            step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize()
        clocks.end()
    if world > 1:
        dist.barrier()
    if flush is None:
        step_ms = t_start.elapsed_time(t_end) / args.steps
    else:
        step_ms = sum(e[0].elapsed_time(e[4]) for e in evs) / args.steps
    call_ms = [sum(e[k].elapsed_time(e[k + 1]) for e in evs) / args.steps for k in range(4)]
    verify_ms = call_ms[1]
    # Compaction bytes moved: each accepted row that moves is read and written
    # once (latent + rope = 1152 B).
    path_h, alen_h = path.cpu().numpy(), alen.cpu().numpy()
    moved = sum(int((path_h[b, :alen_h[b]] != np.arange(alen_h[b])).sum()) for b in range(B))
    compact_bytes = 2.0 * moved * (DL + DR) * 2
    faults = ddt.fault_flags(reset=True)
    statuses_ok = all(int(s.max()) == 0 for s in (mstatus, vstatus, astatus, cstatus))

    flops_local = verify_flops(w.prefix_lens, w.parents)
    bytes_local = verify_bytes(w.prefix_lens, Q, 4 if out_dtype == torch.float32 else 2,
                               w.want_lse)
    step_ms_max, verify_ms_max, mask_ms_max, accept_ms_max, compact_ms_max = reduce_max(
        [step_ms, verify_ms, call_ms[0], call_ms[2], call_ms[3]], world, device)
    flops_total = reduce_sum([flops_local], world, device)[0]

    # ---- end to end through the public API with host buffers ---------------
    e2e = None
    if not args.no_e2e:
        # Per step: the queries, the tree block's KV rows and the tree arrays come
        # from pinned host memory (a copy stream, double-buffered, so the copies of
        # step k+1 overlap the compute of step k), the tree block is written into
        # the resident cache with ddt_kv_write_block, the step runs, and the
        # accepted path, its length, the bonus token and the new prefix are read back.
        tree_rows = np.stack([np.arange(int(p), int(p) + Q) for p in w.prefix_lens])
        keys = ("q_lat", "q_rope", "parents", "node_tokens", "target_tokens", "next_token",
                "next_sibling", "prefix")
        pin = {k: host[k].pin_memory() for k in keys}
        pin["block_ckv"] = host["c_kv"][torch.arange(B)[:, None],
                                        torch.from_numpy(tree_rows)].contiguous().pin_memory()
        pin["block_krope"] = host["k_rope"][torch.arange(B)[:, None],
                                            torch.from_numpy(tree_rows)].contiguous().pin_memory()
        sets = [{k: torch.empty_like(v, device=device) for k, v in pin.items()} for _ in range(2)]
        res_host = {k: torch.empty_like(v, device="cpu").pin_memory()
                    for k, v in (("path", path), ("alen", alen), ("bonus", bonus), ("newp", newp))}
        d2h = sum(v.numel() * v.element_size() for v in res_host.values())
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        copy_stream = torch.cuda.Stream(device=device)
        ev_copied = [torch.cuda.Event() for _ in range(2)]
        ev_used = [torch.cuda.Event() for _ in range(2)]
        wstatus = torch.empty((B,), dtype=torch.int32, device=device)

        def e2e_run(n):
            copy_stream.wait_stream(stream)  # no copy starts before the region
            for k in range(n):
                x = sets[k % 2]
                with torch.cuda.stream(copy_stream):
                    if k >= 2:
                        copy_stream.wait_event(ev_used[k % 2])
                    for key, v in pin.items():
                        x[key].copy_(v, non_blocking=True)
                    ev_copied[k % 2].record(copy_stream)
                stream.wait_event(ev_copied[k % 2])
                ddt.kv_write_block(d["c_kv"], d["k_rope"], x["prefix"], x["block_ckv"],
                                   x["block_krope"], status=wstatus)
                step(src=x)
                ev_used[k % 2].record(stream)
                for key, src in (("path", path), ("alen", alen), ("bonus", bonus),
                                 ("newp", newp)):
                    res_host[key].copy_(src, non_blocking=True)

        e2e_run(args.warmup)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush_l2(0)
        e0.record(stream)
        e2e_run(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_max([e0.elapsed_time(e1) / args.steps], world, device)[0]
        statuses_ok = statuses_ok and int(wstatus.max()) == 0
        e2e = {"value": flops_total / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "resident": "prefix KV rows stay in HBM (the cache); per step the queries, "
                           "the tree block's KV rows and the tree arrays are copied in "
                           "(double-buffered on a copy stream, overlapping the previous "
                           "step), the block written into the cache, and the accepted path "
                           "read back"}

    # ---- calls outside the step: tree build, fused accept+compaction, decode step
    extras = None
    if not args.no_extras:
        extras = time_extras(w, d, host, mask, out, lse, workspace if ws_bytes else None,
                             max_prefix, stream, flush, max(args.steps, 20), args.warmup)

    # ---- the other workloads' calls, graph-timed on this GPU ---------------
    per_config = None
    if rank == 0 and world == 1 and not args.no_per_config:
        per_config = per_config_report([0, 1, 2, 3, 4], measured_peaks()[0], device,
                                       preloaded={args.config: w})

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1) -------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, rows, secs, cores = oracle_sample_throughput(w, args.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{rows} random query rows of the workload's attention "
                         f"({secs:.1f} s, fp64 C oracle, OpenMP)"}

    if rank == 0:
        peaks, peak_src = measured_peaks()
        timed_s = step_ms * args.steps / 1e3
        clk = clocks.summary()
        peak, use_sustained, sustained_why = choose_peak(peaks, timed_s, clk)
        achieved = flops_local / (verify_ms_max * 1e-3) / 1e12
        line = {
            "metric": METRIC,
            "value": flops_total / (step_ms_max * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": step_ms_max,
            "higher_is_better": True,
            "scaling": "strong" if (args.shard == "lpt" and world > 1) else "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": B, "q_len": Q, "heads": H,
                       "prefix": max_prefix, "out": w.out_dtype, "kv_splits": splits,
                       "parallelism": ("single GPU" if world == 1 else
                                       f"requests split longest-first over {world} GPUs"
                                       if args.shard == "lpt" else f"replicas x{world}"),
                       "l2": ("inputs %.0f MB per GPU, over twice the L2: no flush" % (
                                  input_bytes / 1e6)) if flush is None else
                             ("inputs %.0f MB per GPU: L2 flushed (256 MB read) between "
                              "timed steps, outside the timed events" % (input_bytes / 1e6))},
            "verify_us_per_call": verify_ms_max * 1e3,
            "calls_us": {"build_mask": mask_ms_max * 1e3, "verify_attn": verify_ms_max * 1e3,
                         "tree_accept": accept_ms_max * 1e3, "kv_compact": compact_ms_max * 1e3},
            "kv_compact_gbs": compact_bytes / (compact_ms_max * 1e-3) / 1e9,
            # each request's cache rows (prefix + tree block, 1152 B each) once per call
            "kv_stream_gbs": float((w.prefix_lens.astype(np.float64) + Q).sum()) * (DL + DR) * 2
                             / (verify_ms_max * 1e-3) / 1e9,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} {'sustained' if use_sustained else 'burst'} bf16"
                                        f"{sustained_why}",
                         "traffic": measured_traffic(args.config),
                         "algorithmic_bytes": bytes_local,
                         "kernel": "verify_attn_kernel"},
            "extras": extras,
            "per_config": per_config,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                       "reasons": clk["reasons"], "samples": clk.get("samples"),
                       "source": clk.get("source")},
            "faults": faults,
            "statuses_ok": statuses_ok,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
