"""Benchmark of the fused rotate+int4 quantize / dequantize+inverse path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
                    [--suite PATH]

Workload: the large-batch throughput sweep.  K and V of 64 sequences x 8 kv
heads x 8192 tokens (8,388,608 vectors) for every d in {64, 128, 256}, fp16
N(0, 1) with 4 outlier channels per head x20, groups g in {32, d}.  One step
runs every cell of the sweep once: for each d, each g and each rotation
(SRFT, then the SRHT control) the forward kernel (x -> packed codes + scales)
then the inverse kernel (codes + scales -> x_hat), 24 launches over 7.5 GB of
fp16 inputs, all resident in HBM and larger than L2 (no flush is needed
between launches).  Metric: GB/s of fp16 KV through the kernels (n_vec * d * 2
bytes per launch), device-timed with CUDA events; every cell is also reported
with its best and median launch time and its algorithmic HBM bytes
(2d + d/2 + 4d/g per vector) as a fraction of the measured copy peak.

Under torchrun (or `--gpus N`, which starts torchrun itself) each rank runs
the same sweep on its own GPU (independent shards, no collective on the data
path: weak scaling); rank 0 prints one JSON line with the whole-job value
(bytes of all ranks / max time over ranks).

--impl reference times the CPU oracle (the plain float64 restatement of the
method) on a bounded sample of the same sweep on the host cores.
--suite PATH additionally measures the other code widths, the lambda hook,
the eager decode step and the int4-reading attention, and writes them as
JSON to PATH.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rotated_int4_kv_kvq_b200 import workloads as W  # noqa: E402

METRIC = "fp16 KV GB/s through fused rotate+int4 quant / dequant+inverse; % of HBM peak"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "rotated_int4_kv_kvq_b200", "csrc")

SWEEP_D = (64, 128, 256)
ROTS = ((0, "srft"), (1, "srht"))


def sweep_groups(d):
    return (32, d)


# the sources the tiled forward / inverse kernels are built and launched from
CODEC_SOURCES = ("kvq_api.cu", "kvq_codec.cuh", "kvq_device.cuh", "kvq_inst.cuh", "kvq_rfft.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in CODEC_SOURCES:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def fwd_bytes(d, g):  # algorithmic bytes per vector, forward (inverse: same)
    return 2 * d + d // 2 + 4 * (d // g)


def cell_name(d, g, rot, direction):
    kern = "kvq_fwd_kernel" if direction == "fwd" else "kvq_inv_kernel"
    return f"{kern} d={d} g={g} {ROTS[rot][1]}"


def recorded_traffic(kernel: str):
    """DRAM bytes per full-size launch of `kernel` (a cell name) from the
    committed ncu summary, if it was taken on the current kernel sources
    (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except Exception:
        return None
    e = rec.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------- clocks ---

REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def summarize_clocks(samples, source):
    """samples: (sm_mhz, max_mhz, set of active reason names) per sample."""
    sm = [s[0] for s in samples]
    mx = [s[1] for s in samples]
    reasons = set()
    for s in samples:
        reasons |= s[2]
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_min_mhz": min(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
            "samples": len(sm), "source": source}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms (the
    fallback when NVML cannot be read from Python)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        t0, t1 = (self.marks + [0, 0])[:2] if len(self.marks) >= 2 else (0, 1e30)
        rows = [l for (t, l) in self.lines if t0 - 0.25 <= t <= t1 + 0.25] or \
            [l for (_, l) in self.lines]
        samples = []
        for r in rows:
            f = [c.strip() for c in r.split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            act = {n for n, v in zip(REASON_NAMES, f[5:9]) if v.lower().startswith("active")}
            samples.append((sm, mx, act))
        return summarize_clocks(samples, "nvidia-smi 200 ms")


class NvmlSampler:
    """Read-only NVML polling of the SM clock and the clock-event reasons
    every `period` seconds from a background thread (changes no setting).
    Only samples between the first two mark() calls are summarized."""

    BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
            "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, handle, nvml, period=0.01):
        self.h, self.nvml, self.period = handle, nvml, period
        self.samples = []
        self.marks = []
        self.stop_flag = threading.Event()
        self.thread = None
        self.max_mhz = float(nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM))

    def _reasons(self):
        fn = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nvml.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _loop(self):
        while not self.stop_flag.is_set():
            try:
                sm = float(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                bits = int(self._reasons())
                act = {n for n, b in self.BITS.items() if bits & b}
                self.samples.append((time.time(), sm, act))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        self.stop_flag.set()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        t0, t1 = (self.marks[0], self.marks[1]) if len(self.marks) >= 2 else (0, 1e30)
        rows = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples
        return summarize_clocks([(sm, self.max_mhz, act) for (_, sm, act) in rows],
                                f"nvml {int(self.period * 1000)} ms")


def make_sampler(dev: torch.device):
    """NVML sampler for the CUDA device `dev` (matched by UUID), else the
    nvidia-smi sampler."""
    try:
        import pynvml as nvml
        nvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        h = nvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        return NvmlSampler(h, nvml)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
        idx = dev.index or 0
        gpu = int(vis[idx]) if idx < len(vis) and vis[idx].isdigit() else idx
        return ClockSampler(gpu)


# ------------------------------------------------------------- launching ---

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_command(argv, gpus, port):
    """torchrun command line that runs this script on `gpus` ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            "--nproc-per-node", str(gpus), "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__), *argv]


def maybe_relaunch(args, argv):
    """--gpus N > 1 outside torchrun: start N ranks under torchrun and exit
    with its status.  Inside torchrun, --gpus must equal WORLD_SIZE."""
    world = os.environ.get("WORLD_SIZE")
    if world is not None:
        if int(world) != args.gpus:
            sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
        return
    if args.gpus <= 1:
        return
    if args.impl == "kvq":
        visible = torch.cuda.device_count() if torch.cuda.is_available() else 0
        if visible < args.gpus:
            sys.exit(f"bench.py: --gpus {args.gpus} but {visible} CUDA device(s) are visible")
    r = subprocess.run(relaunch_command(argv, args.gpus, _free_port()))
    sys.exit(r.returncode)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def allreduce_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


# ------------------------------------------------------------- workload ---

def workload_desc():
    return ("large-batch sweep: K,V x 64 seq x 8 kv heads x 8192 tokens (8,388,608 vectors) "
            "for d in {64,128,256}, fp16 N(0,1) + 4 outlier channels/head x20, g in {32, d}, "
            "SRFT and SRHT, forward then inverse: 24 launches per step")


class SweepData:
    """Device tensors of one d of the sweep: x, out, packed and one scales
    tensor per group."""

    def __init__(self, d, dev, seed_offset=0):
        shape = W.config(5, d=d, group=32)
        self.d = d
        self.x = W.make_kv(shape, device=dev, seed=shape.seed + seed_offset)
        self.n = self.x.shape[0]
        self.signs = torch.from_numpy(W.make_signs(d)).to(dev)
        self.packed = torch.empty((self.n, d // 2), dtype=torch.uint8, device=dev)
        self.scales = {g: torch.empty((self.n, d // g), dtype=torch.float32, device=dev)
                       for g in sweep_groups(d)}
        self.out = torch.empty_like(self.x)


def sweep_cells():
    """(d, g, rot) in execution order; each runs forward then inverse."""
    return [(d, g, rot) for d in SWEEP_D for g in sweep_groups(d) for rot, _ in ROTS]


def sweep_fp16_bytes_per_step(n_by_d):
    """fp16 KV bytes one step moves through the kernels (both directions)."""
    return sum(2 * n_by_d[d] * d * 2 for (d, g, rot) in sweep_cells())


def time_sweep(kvq, S, steps, warmup, sampler=None):
    """Device time of `steps` sweep steps; per-launch times of every cell.
    Returns (total_ms, {(d, g, rot, dir): [ms per launch]})."""
    stream = torch.cuda.current_stream()
    cells = sweep_cells()

    def launch(d, g, rot, direction):
        T = S[d]
        if direction == "fwd":
            kvq.kvq_rot_quant_fwd(T.x, T.signs, rot, g, T.packed, T.scales[g], stream)
        else:
            kvq.kvq_dequant_rot_inv(T.packed, T.scales[g], T.signs, rot, g, T.out, stream)

    for _ in range(warmup):
        for (d, g, rot) in cells:
            launch(d, g, rot, "fwd")
            launch(d, g, rot, "inv")
    torch.cuda.synchronize()
    n_launch = 2 * len(cells)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)]
          for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark()
    start.record(stream)
    for k in range(steps):
        i = 0
        ev[k][0].record(stream)
        for (d, g, rot) in cells:
            for direction in ("fwd", "inv"):
                launch(d, g, rot, direction)
                i += 1
                ev[k][i].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    per = {}
    for k in range(steps):
        i = 0
        for (d, g, rot) in cells:
            for direction in ("fwd", "inv"):
                per.setdefault((d, g, rot, direction), []).append(
                    ev[k][i].elapsed_time(ev[k][i + 1]))
                i += 1
    return start.elapsed_time(end), per


def cell_record(d, g, rot, direction, ms_list, n, peak):
    best, med = min(ms_list), statistics.median(ms_list)
    algo = n * fwd_bytes(d, g)
    return {"cell": cell_name(d, g, rot, direction), "d": d, "group": g, "rot": ROTS[rot][1],
            "dir": direction, "us_best": 1e3 * best, "us_median": 1e3 * med,
            "algo_bytes": algo, "algo_gbs_median": algo / (med * 1e-3) / 1e9,
            "frac_median": algo / (med * 1e-3) / 1e9 / peak,
            "frac_best": algo / (best * 1e-3) / 1e9 / peak,
            "fp16_gbs_median": n * d * 2 / (med * 1e-3) / 1e9,
            "vec_per_s_median": n / (med * 1e-3)}


def run_e2e(kvq, S, world, steps, chunks=8):
    """The sweep through the public API with host buffers: every step copies
    each d's inputs in from pinned host memory (chunked) and every cell's
    output back; copies and kernels of consecutive chunks overlap on three
    streams.  Same metric as the device-timed value."""
    cells = [(g, rot) for g in (32, None) for rot, _ in ROTS]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nmax = max(T.n * T.d for T in S.values())
    oh_all = torch.empty(nmax, dtype=torch.float16, pin_memory=True)
    plan = {}
    for d, T in S.items():
        xh = torch.empty(T.x.shape, dtype=torch.float16, pin_memory=True)
        xh.copy_(T.x)
        bounds = [((i * T.n) // chunks) // 32 * 32 for i in range(chunks)] + [T.n]
        plan[d] = (xh, oh_all[: T.n * d].view(T.n, d), bounds,
                   [torch.cuda.Event() for _ in range(chunks)],  # input chunk landed
                   [torch.cuda.Event() for _ in range(chunks)],  # input chunk free again
                   [torch.cuda.Event() for _ in range(chunks)],  # kernels of the chunk done
                   [torch.cuda.Event() for _ in range(chunks)])  # output chunk copied out

    def one_pass():
        for d, T in S.items():
            xh, oh, bounds, ev_in, ev_free, ev_run, ev_out = plan[d]
            for c in range(chunks):
                a, b = bounds[c], bounds[c + 1]
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev_free[c])
                    T.x[a:b].copy_(xh[a:b], non_blocking=True)
                    ev_in[c].record(s_in)
                s_run.wait_event(ev_in[c])
                for i, (g, rot) in enumerate(cells):
                    g = d if g is None else g
                    kvq.kvq_rot_quant_fwd(T.x[a:b], T.signs, rot, g, T.packed[a:b],
                                          T.scales[g][a:b], s_run)
                    if i == len(cells) - 1:
                        ev_free[c].record(s_run)
                    s_run.wait_event(ev_out[c])  # previous cell's output chunk copied
                    kvq.kvq_dequant_rot_inv(T.packed[a:b], T.scales[g][a:b], T.signs, rot, g,
                                            T.out[a:b], s_run)
                    ev_run[c].record(s_run)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(ev_run[c])
                        oh[a:b].copy_(T.out[a:b], non_blocking=True)
                        ev_out[c].record(s_out)

    e2e_steps = max(2, min(steps, 3))
    one_pass()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    for st in (s_in, s_run, s_out):
        st.wait_stream(cur)
    for _ in range(e2e_steps):
        one_pass()
    for st in (s_in, s_run, s_out):
        cur.wait_stream(st)
    e1.record(cur)
    torch.cuda.synchronize()
    last = S[SWEEP_D[-1]]
    if not torch.equal(plan[last.d][1], last.out.cpu()):
        raise RuntimeError("end-to-end output differs from the device result")
    e2e_ms = allreduce_max(e0.elapsed_time(e1), world)
    n_by_d = {d: T.n for d, T in S.items()}
    fp16_in = sum(T.n * T.d * 2 for T in S.values())
    return {"value": world * e2e_steps * sweep_fp16_bytes_per_step(n_by_d) / (e2e_ms * 1e-3) / 1e9,
            "unit": UNIT, "h2d_bytes_per_step": int(fp16_in),
            "d2h_bytes_per_step": int(len(cells) * fp16_in), "chunks_per_d": chunks,
            "steps": e2e_steps, "gpu_launches_per_step": 2 * len(cells) * chunks * len(S)}


# ----------------------------------------------------- CPU oracle legs ---

def oracle_cell(O, xs, signs, rot, g):
    """Oracle forward + inverse of the rows xs; returns (codes, scales, s)."""
    t0 = time.perf_counter()
    p, sc = O.rot_quant_fwd(xs, signs, rot, g)
    O.dequant_rot_inv(p, sc, signs, rot, g)
    return p, sc, time.perf_counter() - t0


def flip_record(O, xs, signs, rot, g, p_ref, s_ref, p_gpu):
    """Codes that differ between the GPU and the oracle, and how many of
    them are not within 1e-4 of a rounding tie (must be 0)."""
    q_ref = O.unpack_nibbles(p_ref)
    q_gpu = O.unpack_nibbles(p_gpu)
    bad = q_ref != q_gpu
    n_bad = int(bad.sum())
    not_tie = 0
    if n_bad:
        y = O.rotated_values(xs, signs, rot)
        dist = O.near_tie_distance(y, s_ref, g)
        not_tie = int((dist[bad] >= 1e-4).sum())
    return {"codes": int(q_ref.size), "flips": n_bad, "flips_not_near_tie": not_tie}


def cpu_legs(kvq, S, dev, peak_unused=None):
    """The oracle on the host cores: (1) a sample of every sweep cell (the
    cpu_baseline value, same weighting as the device step), (2) configs 1
    and 3 and the config-4 decode step at position 256 on their full
    tensors, (3) a sample of config 2; near-tie flip counts against the GPU
    codes for each."""
    import oracle.kvq_oracle as O
    per_step_bytes, total_s, flips = 0, 0.0, {}
    rows_per_d = {64: 262144, 128: 262144, 256: 131072}  # about 10 s on 16 cores
    for d, T in S.items():
        idx = torch.from_numpy(W.sample_rows(T.n, rows_per_d[d], seed=7 + d)).to(dev)
        xg = T.x[idx].contiguous()
        xs = xg.cpu().numpy()
        signs = W.make_signs(d)
        for g in sweep_groups(d):
            for rot, rname in ROTS:
                p_gpu, _ = kvq.kvq_rot_quant_fwd(xg, T.signs, rot, g)
                p, sc, dt = oracle_cell(O, xs, signs, rot, g)
                total_s += dt
                per_step_bytes += 2 * len(xs) * d * 2
                flips[f"5 sweep d={d} g={g} {rname}"] = flip_record(
                    O, xs, signs, rot, g, p, sc, p_gpu.cpu().numpy())
    value = per_step_bytes / total_s / 1e9
    sample = ", ".join(f"d={d}: {rows_per_d[d]} sampled rows" for d in S) + \
        " of the sweep tensors, forward + inverse for every (g, rotation)"

    per_config = {}
    for i in (1, 3):
        shape = W.config(i)
        x = W.make_kv(shape)
        xs = x.numpy()
        xg = x.to(dev)
        d, g = shape.d, shape.group
        signs = W.make_signs(d)
        sd = torch.from_numpy(signs).to(dev)
        for rot, rname in ROTS:
            p_gpu, _ = kvq.kvq_rot_quant_fwd(xg, sd, rot, g)
            p, sc, dt = oracle_cell(O, xs, signs, rot, g)
            per_config[f"{i} {shape.name} {rname}"] = {
                "vectors": len(xs), "seconds": dt, "gbs": 2 * len(xs) * d * 2 / dt / 1e9}
            flips[f"{i} {shape.name} {rname}"] = flip_record(O, xs, signs, rot, g, p, sc,
                                                             p_gpu.cpu().numpy())
    # config 4: one 26-layer decode step at position 256 (52 heads x 257 rows)
    shape = W.scaled(W.config(4), tokens=257)
    seq = W.make_decode_sequence(shape)  # [52, 257, 256]
    d, g, pos = 256, 256, 256
    signs = W.make_signs(d)
    sd = torch.from_numpy(signs).to(dev)
    for rot, rname in ROTS:
        sq = seq.to(dev)
        pk, sk = kvq.kvq_rot_quant_fwd(sq[:, :pos].reshape(-1, d).contiguous(), sd, rot, g)
        packed = torch.zeros((52, pos + 1, d // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((52, pos + 1, 1), dtype=torch.float32, device=dev)
        packed[:, :pos] = pk.reshape(52, pos, -1)
        scales[:, :pos] = sk.reshape(52, pos, -1)
        kvq.kvq_decode_step(sq[:, pos].contiguous(), packed, scales, pos, sd, rot, g)
        xs = seq.reshape(-1, d).numpy()
        p, sc, dt = oracle_cell(O, xs, signs, rot, g)
        per_config[f"4 gemma3-1b decode step pos 256 {rname}"] = {
            "vectors": len(xs), "seconds": dt, "gbs": 2 * len(xs) * d * 2 / dt / 1e9}
        flips[f"4 gemma3-1b decode step pos 256 {rname}"] = flip_record(
            O, xs, signs, rot, g, p, sc, packed.reshape(-1, d // 2).cpu().numpy())
    # config 2: a sample of the SmolLM2-1.7B-shaped cache (same recipe, 4 heads)
    shape = W.scaled(W.config(2), layers=1, heads=4)
    x = W.make_kv(shape)
    xs = x.numpy()
    d, g = shape.d, shape.group
    signs = W.make_signs(d)
    sd = torch.from_numpy(signs).to(dev)
    for rot, rname in ROTS:
        p_gpu, _ = kvq.kvq_rot_quant_fwd(x.to(dev), sd, rot, g)
        p, sc, dt = oracle_cell(O, xs, signs, rot, g)
        per_config[f"2 {shape.name} sample {rname}"] = {
            "vectors": len(xs), "seconds": dt, "gbs": 2 * len(xs) * d * 2 / dt / 1e9}
        flips[f"2 {shape.name} sample {rname}"] = flip_record(O, xs, signs, rot, g, p, sc,
                                                             p_gpu.cpu().numpy())
    return ({"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
             "sample": sample, "seconds": total_s, "per_config": per_config},
            flips)


# -------------------------------------------------- other measurements ---

def time_pair(kvq, x, packed, scales, out, signs, rot, g, steps, warmup):
    """Per-launch device times (ms lists) of forward and inverse."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        kvq.kvq_rot_quant_fwd(x, signs, rot, g, packed, scales, stream)
        kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, out, stream)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record(stream)
        kvq.kvq_rot_quant_fwd(x, signs, rot, g, packed, scales, stream)
        ev[k][1].record(stream)
        kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, out, stream)
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    return ([e[0].elapsed_time(e[1]) for e in ev], [e[1].elapsed_time(e[2]) for e in ev])


def run_smollm2_cache(kvq, dev, peak, steps):
    """Config 2 (SmolLM2-1.7B-shaped cache, d = g = 64): forward + inverse
    of the whole cache per rotation."""
    shape = W.config(2)
    d, g = shape.d, shape.group
    x = W.make_kv(shape, device=dev)
    n = x.shape[0]
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    packed = torch.empty((n, d // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, d // g), dtype=torch.float32, device=dev)
    out = torch.empty_like(x)
    res = []
    for rot, rname in ROTS:
        f, i = time_pair(kvq, x, packed, scales, out, signs, rot, g, steps, 3)
        for direction, ms in (("fwd", f), ("inv", i)):
            rec = cell_record(d, g, rot, direction, ms, n, peak)
            rec["cell"] = rec["cell"] + " (" + shape.name + ")"
            res.append(rec)
    del x, packed, scales, out
    torch.cuda.empty_cache()
    return res


def run_decode_latency(kvq, dev, peak, positions=(256, 1024, 2048, 4095), eager=False):
    """Config 4 (Gemma-3-1B shape: 26 layers x K,V, d = g = 256): one decode
    step = 26 kvq_decode_step calls (K and V of a layer as 2 heads), timed as
    a CUDA graph at each position; the HBM bytes the step must move and the
    time they take at the measured peak."""
    shape = W.config(4)
    d, g, L = 256, 256, 26
    seq = W.make_decode_sequence(shape, device=dev)  # [52, 4096, 256]
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    cap = 4096
    res = []
    for rot, rname in ROTS:
        packed = torch.zeros((2 * L, cap, d // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((2 * L, cap, 1), dtype=torch.float32, device=dev)
        p, s = kvq.kvq_rot_quant_fwd(seq.reshape(-1, d), signs, rot, g)
        packed.copy_(p.reshape(2 * L, cap, -1))
        scales.copy_(s.reshape(2 * L, cap, -1))
        for pos in positions:
            outs = [torch.empty((2, pos + 1, d), dtype=torch.float16, device=dev)
                    for _ in range(L)]
            xs = [seq[2 * l:2 * l + 2, pos].contiguous() for l in range(L)]

            def step():
                for l in range(L):
                    kvq.kvq_decode_step(xs[l], packed[2 * l:2 * l + 2], scales[2 * l:2 * l + 2],
                                        pos, signs, rot, g, outs[l])
            rec = {"rot": rname, "pos": pos}
            if eager:
                for _ in range(3):
                    step()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(20):
                    step()
                e1.record()
                torch.cuda.synchronize()
                rec["eager_us_per_step"] = 1e3 * e0.elapsed_time(e1) / 20
            rec["graph_us_per_step"] = graph_time_us(step)
            # per head: new token in (2d) + its codes/scale out + pos+1 rows of
            # codes/scales in and fp16 out (the new row's codes come from registers)
            byts = L * 2 * ((pos + 1) * fwd_bytes(d, g) + 2 * d)
            rec["algo_bytes_per_step"] = byts
            rec["ideal_us"] = byts / (peak * 1e9) * 1e6
            rec["frac"] = rec["ideal_us"] / rec["graph_us_per_step"]
            res.append(rec)
            del outs
        del packed, scales
    torch.cuda.empty_cache()
    return res, seq, signs


# ------------------------------------------------------------------ main ---

def run_reference(args, world, rank):
    """The CPU oracle, as it stands, on a bounded sample of the same sweep:
    every step runs forward + inverse of `rows` vectors per (d, g, rotation)
    cell, drawn from smaller tensors of the same recipe."""
    if rank != 0:
        return
    import oracle.kvq_oracle as O
    rows = 4096
    data = {}
    for d in SWEEP_D:
        shape = W.scaled(W.config(5, d=d, group=32), heads=1)  # 16384 vectors of the recipe
        data[d] = (W.make_kv(shape).numpy(), W.make_signs(d))
    times, step_bytes = [], 0
    for k in range(args.warmup + args.steps):
        t = 0.0
        step_bytes = 0
        for d, g, rot in sweep_cells():
            x, signs = data[d]
            part = x[(k * rows) % len(x):][:rows]
            _, _, dt = oracle_cell(O, part, signs, rot, g)
            t += dt
            step_bytes += 2 * len(part) * d * 2
        if k >= args.warmup:
            times.append(t)
    total = sum(times)
    value = step_bytes * len(times) / total / 1e9
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc() + f" (CPU oracle: {rows} vectors per cell "
                                                 "per step)",
                   "rows_per_cell_per_step": rows, "d": list(SWEEP_D), "group": "32, d",
                   "rot": "srft, srht"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows} vectors per (d, g, rotation) cell per step, drawn "
                                   "from 16,384-vector tensors of the sweep recipe"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--suite", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="run --reps forward+inverse passes of one shape (for ncu), no timing")
    ap.add_argument("--rot", type=int, default=0)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--group", type=int, default=64)
    ap.add_argument("--n-vec", type=int, default=1 << 21)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--attn-len", type=int, default=0,
                    help="with --profile: decode attention over this many cached rows "
                         "(--d, --group, --rot; --attn-heads KV heads, --attn-nq queries)")
    ap.add_argument("--attn-heads", type=int, default=32)
    ap.add_argument("--attn-nq", type=int, default=1)
    ap.add_argument("--decode-pos", type=int, default=0,
                    help="with --profile: run --reps 26-layer decode steps at this position")
    argv = sys.argv[1:]
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    if args.profile:
        run_profile_case(args)
        return
    maybe_relaunch(args, argv)
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    from rotated_int4_kv_kvq_b200 import kvq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peak, peak_kind = hbm_peak()
    S = {d: SweepData(d, dev, seed_offset=1000 * rank) for d in SWEEP_D}
    n_by_d = {d: T.n for d, T in S.items()}

    sampler = make_sampler(dev)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    total_ms, per = time_sweep(kvq, S, args.steps, args.warmup, sampler)
    barrier(world)
    sampler.stop()
    status = kvq.kvq_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    total_ms = allreduce_max(total_ms, world)
    value = world * args.steps * sweep_fp16_bytes_per_step(n_by_d) / (total_ms * 1e-3) / 1e9

    cells = [cell_record(d, g, rot, direction, per[(d, g, rot, direction)], n_by_d[d], peak)
             for (d, g, rot) in sweep_cells() for direction in ("fwd", "inv")]
    worst = min(cells, key=lambda c: c["frac_median"])
    roofline = {"bound": "hbm", "achieved": worst["algo_gbs_median"], "peak": peak,
                "unit": "GB/s", "frac": worst["frac_median"],
                "traffic": recorded_traffic(worst["cell"]), "kernel": worst["cell"],
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": worst["algo_bytes"],
                "launch_us_median": worst["us_median"]}
    busiest = max(cells, key=lambda c: c["us_median"])
    detail = {
        "sweep": cells,
        "sweep_min_frac": worst["frac_median"],
        "sweep_cells_below_0.70": [c["cell"] for c in cells if c["frac_median"] < 0.70],
        "dominant_cell": busiest["cell"],
        "vec_per_s": world * args.steps * sum(2 * n_by_d[d] for (d, g, rot) in sweep_cells())
        / (total_ms * 1e-3),
        "kernel_source_hash": kernel_source_hash(),
    }

    e2e = run_e2e(kvq, S, world, args.steps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, flips = cpu_legs(kvq, S, dev)
        detail["near_tie_flips"] = flips
    del S
    torch.cuda.empty_cache()

    if rank == 0:
        detail["smollm2_1.7b_cache"] = run_smollm2_cache(kvq, dev, peak, args.steps)
        detail["gemma3_1b_decode_step"], seq, signs = run_decode_latency(kvq, dev, peak)
        detail["gemma3_1b_decode_step_windowed"] = run_window_suite(kvq, dev, seq, signs, peak)
        del seq
        torch.cuda.empty_cache()

    suite = None
    if args.suite and rank == 0:
        suite_clock = make_sampler(dev)
        suite_clock.start()
        suite = run_suite(kvq, dev)
        suite_clock.stop()
        suite["clocks"] = suite_clock.summary()  # over the whole suite
        with open(args.suite, "w") as f:
            json.dump(suite, f, indent=1)

    if rank == 0:
        clocks = sampler.summary()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": workload_desc(), "n_vec_per_launch": n_by_d[64],
                       "d": list(SWEEP_D), "group": "32, d", "rot": "srft, srht",
                       "launches_per_step": 2 * len(sweep_cells()),
                       "l2": "inputs larger than L2 (1.07-4.29 GB of fp16 per launch), no flush",
                       "parallelism": f"independent shards x{world} (no collective)"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 2 * len(sweep_cells()) * args.steps, "clocks": clocks,
            "detail": detail,
            "hbm_frac_of_nominal_8tbs": roofline["achieved"] / 8000.0,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_profile_case(args):
    """`reps` forward then inverse passes over n_vec vectors of the sweep
    recipe at (d, group, rot): the small case ncu captures."""
    from rotated_int4_kv_kvq_b200 import kvq
    dev = torch.device("cuda", 0)
    if args.decode_pos > 0:
        return run_profile_decode(kvq, dev, args)
    if args.attn_len > 0:
        return run_profile_attn(kvq, dev, args)
    d, g = args.d, args.group
    tokens = 8192
    heads = max(1, -(-args.n_vec // (2 * tokens)))
    shape = W.scaled(W.config(5, d=d, group=g), heads=heads, tokens=tokens)
    x = W.make_kv(shape, device=dev)[: args.n_vec].contiguous()
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    packed, scales = kvq.kvq_rot_quant_fwd(x, signs, args.rot, g)
    out = kvq.kvq_dequant_rot_inv(packed, scales, signs, args.rot, g)
    for _ in range(args.reps):
        kvq.kvq_rot_quant_fwd(x, signs, args.rot, g, packed, scales)
        kvq.kvq_dequant_rot_inv(packed, scales, signs, args.rot, g, out)
    torch.cuda.synchronize()
    st = kvq.kvq_device_status()
    print(json.dumps({"profile_case": {"d": d, "group": g, "rot": args.rot,
                                       "n_vec": int(x.shape[0]), "reps": args.reps,
                                       "status": st}}))
    if st != 0:
        sys.exit(1)


def run_profile_attn(kvq, dev, args):
    """`reps` decode-attention calls over `attn_len` cached rows."""
    d, g, h, nq, n = args.d, args.group, args.attn_heads, args.attn_nq, args.attn_len
    gen = torch.Generator(device=dev).manual_seed(5)
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    c = []
    for _ in range(2):
        x = torch.randn((h * n, d), generator=gen, device=dev).half()
        p, s = kvq.kvq_rot_quant_fwd(x, signs, args.rot, g)
        c += [p.reshape(h, n, -1), s.reshape(h, n, -1)]
    q = torch.randn((h, nq, d), generator=gen, device=dev).half()
    for _ in range(args.reps):
        o = kvq.kvq_attend_decode(q, c[0], c[1], c[2], c[3], n, signs, args.rot, g)
    torch.cuda.synchronize()
    st = kvq.kvq_device_status()
    print(json.dumps({"profile_attn": {"d": d, "group": g, "heads": h, "nq": nq, "len": n,
                                       "status": st, "out0": float(o[0, 0, 0])}}))
    if st != 0:
        sys.exit(1)


def run_profile_decode(kvq, dev, args):
    """`reps` Gemma-3-1B-shaped decode steps (26 layers x K,V, d=256,
    g=256, one call per layer) at position decode_pos."""
    shape = W.scaled(W.config(4), tokens=args.decode_pos + 1)
    d, g, L, pos = 256, 256, 26, args.decode_pos
    seq = W.make_decode_sequence(shape, device=dev)
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    cap = pos + 1
    packed = torch.zeros((2 * L, cap, d // 2), dtype=torch.uint8, device=dev)
    scales = torch.zeros((2 * L, cap, 1), dtype=torch.float32, device=dev)
    p, s = kvq.kvq_rot_quant_fwd(seq.reshape(-1, d), signs, args.rot, g)
    packed.copy_(p.reshape(2 * L, cap, -1))
    scales.copy_(s.reshape(2 * L, cap, -1))
    outs = [torch.empty((2, pos + 1, d), dtype=torch.float16, device=dev) for _ in range(L)]
    xs = [seq[2 * l:2 * l + 2, pos].contiguous() for l in range(L)]
    for _ in range(args.reps):
        for l in range(L):
            kvq.kvq_decode_step(xs[l], packed[2 * l:2 * l + 2], scales[2 * l:2 * l + 2], pos,
                                signs, args.rot, g, outs[l])
    torch.cuda.synchronize()
    st = kvq.kvq_device_status()
    print(json.dumps({"profile_decode": {"pos": pos, "rot": args.rot, "reps": args.reps,
                                         "status": st}}))
    if st != 0:
        sys.exit(1)


def run_suite(kvq, dev):
    """Measurements beyond the JSON line: other code widths and the lambda
    hook on the sweep workload (g = d, SRFT), the eager decode step, and the
    int4-reading attention."""
    res = {}
    peak, _ = hbm_peak()
    steps = 20
    for d in SWEEP_D:
        g = d
        shape = W.config(5, d=d, group=g)
        x = W.make_kv(shape, device=dev)
        n = x.shape[0]
        signs = torch.from_numpy(W.make_signs(d)).to(dev)
        packed = torch.empty((n, d // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((n, d // g), dtype=torch.float32, device=dev)
        out = torch.empty_like(x)
        algo = n * fwd_bytes(d, g)
        for rot, rname in ROTS:
            if rot == 0:  # other code widths on the same workload
                for bits in ((3, 6, 8) if d >= 128 else (6, 8)):
                    pb = torch.empty((n, d * bits // 8), dtype=torch.uint8, device=dev)
                    ab = n * (2 * d + d * bits // 8 + 4 * (d // g))
                    for _ in range(3):
                        kvq.kvq_rot_quant_fwd_bits(x, signs, rot, g, bits, pb, scales)
                        kvq.kvq_dequant_rot_inv_bits(pb, scales, signs, rot, g, bits, out)
                    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                    tf = ti = 0.0
                    for _ in range(steps):
                        e[0].record()
                        kvq.kvq_rot_quant_fwd_bits(x, signs, rot, g, bits, pb, scales)
                        e[1].record()
                        kvq.kvq_dequant_rot_inv_bits(pb, scales, signs, rot, g, bits, out)
                        e[2].record()
                        torch.cuda.synchronize()
                        tf += e[0].elapsed_time(e[1])
                        ti += e[1].elapsed_time(e[2])
                    for name, ms in (("fwd", tf), ("inv", ti)):
                        us = 1e3 * ms / steps
                        res.setdefault("bits", []).append({
                            "d": d, "group": g, "rot": rname, "bits": bits, "dir": name,
                            "us": us, "algo_gbs": ab / (us * 1e-6) / 1e9,
                            "frac": ab / (us * 1e-6) / 1e9 / peak})
                    del pb
            # the per-channel lambda hook on the same workload
            lam = torch.exp(0.5 * torch.randn(d, generator=torch.Generator().manual_seed(d)))
            lam = lam.to(dev)
            for _ in range(3):
                kvq.kvq_rot_quant_fwd(x, signs, rot, g, packed, scales, lam=lam)
                kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, out, lam=lam)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            tf = ti = 0.0
            for _ in range(steps):
                e[0].record()
                kvq.kvq_rot_quant_fwd(x, signs, rot, g, packed, scales, lam=lam)
                e[1].record()
                kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, out, lam=lam)
                e[2].record()
                torch.cuda.synchronize()
                tf += e[0].elapsed_time(e[1])
                ti += e[1].elapsed_time(e[2])
            for name, ms in (("fwd", tf), ("inv", ti)):
                us = 1e3 * ms / steps
                res.setdefault("lambda", []).append({
                    "d": d, "group": g, "rot": rname, "dir": name, "us": us,
                    "algo_gbs": algo / (us * 1e-6) / 1e9,
                    "frac": algo / (us * 1e-6) / 1e9 / peak})
        del x, packed, scales, out
        torch.cuda.empty_cache()
    res["decode"], seq, signs = run_decode_latency(kvq, dev, peak, eager=True)
    del seq
    torch.cuda.empty_cache()
    res["attention"] = run_attention_suite(kvq, dev, peak)
    return res


def graph_time_us(fn, reps=20):
    """Per-call device time of fn() replayed as a CUDA graph."""
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    s2 = torch.cuda.Stream()
    s2.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s2):
        fn()
    torch.cuda.current_stream().wait_stream(s2)
    with torch.cuda.graph(gr):
        fn()
    for _ in range(2):
        gr.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        gr.replay()
    e1.record()
    torch.cuda.synchronize()
    del gr
    return 1e3 * e0.elapsed_time(e1) / reps


def run_attention_suite(kvq, dev, peak):
    """Decode attention reading the int4 cache: the Gemma-3-1B step (26
    layers, 1 KV head with 4 queries, d = g = 256) as a graph of 26 calls, one
    SmolLM2-1.7B-shaped layer (32 KV heads, 1 query each, d = g = 64), and the
    same layers batched over several sequences in one call (the KV heads of
    all sequences as the call's heads), for throughput against the HBM
    roofline (codes + scales of K and V)."""
    out = []
    gen = torch.Generator(device=dev).manual_seed(21)
    cases = [("gemma-3-1b step", 26, 1, 4, 256, 256, (256, 1024, 2048, 4096)),
             ("smollm2-1.7b layer", 1, 32, 1, 64, 64, (1024, 4096, 16384)),
             ("gemma-3-1b layer x 16 sequences", 1, 16, 4, 256, 256, (4096,)),
             ("gemma-3-1b layer x 64 sequences", 1, 64, 4, 256, 256, (4096,)),
             ("gemma-3-1b layer x 128 sequences", 1, 128, 4, 256, 256, (4096,)),
             ("smollm2-1.7b layer x 16 sequences", 1, 512, 1, 64, 64, (16384,)),
             ("8 queries per kv head, d = 128, x 16 sequences", 1, 128, 8, 128, 128, (4096,))]
    for name, layers, heads, nq, d, g, lens in cases:
        cap = max(lens)
        signs = torch.from_numpy(W.make_signs(d)).to(dev)
        for rot in (kvq.SRFT, kvq.SRHT):
            caches = []
            for _ in range(layers):
                c = []
                for _kv in range(2):
                    x = (torch.randn((heads * cap, d), generator=gen, device=dev)).half()
                    p, s = kvq.kvq_rot_quant_fwd(x, signs, rot, g)
                    c += [p.reshape(heads, cap, -1), s.reshape(heads, cap, -1)]
                    del x
                q = torch.randn((heads, nq, d), generator=gen, device=dev).half()
                o = torch.empty((heads, nq, d), dtype=torch.float16, device=dev)
                caches.append((q, c, o))
            for n in lens:
                def fn():
                    for q, (kp, ks, vp, vs), o in caches:
                        kvq.kvq_attend_decode(q, kp, ks, vp, vs, n, signs, rot, g, out=o)
                us = graph_time_us(fn)
                byts = layers * heads * n * 2 * fwd_bytes(d, g) - layers * heads * n * 2 * 2 * d
                out.append({"workload": name, "rot": "srft" if rot == 0 else "srht",
                            "len": n, "kv_heads": heads, "graph_us": us, "calls": layers,
                            "algo_bytes": byts, "algo_gbs": byts / (us * 1e-6) / 1e9,
                            "frac": byts / (us * 1e-6) / 1e9 / peak})
            del caches
            torch.cuda.empty_cache()
    return out


def run_window_suite(kvq, dev, seq, signs, peak, window=16):
    """Gemma-3-1B decode steps with the dequantized-prefix cache: 26 calls
    per step (one per layer, K and V as 2 heads), timed over the `window`
    steps of one window (one flush) as a CUDA graph; per-step average."""
    d, g, L, cap = 256, 256, 26, 4096
    out = []
    for rot in (kvq.SRFT, kvq.SRHT):
        packed = torch.zeros((2 * L, cap, d // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((2 * L, cap, 1), dtype=torch.float32, device=dev)
        kv = seq.clone()  # the attention view, [52, 4096, 256]
        for end in (272, 1024, 2048, 4096):
            first = end - window
            xs = [[seq[2 * l:2 * l + 2, p].contiguous() for l in range(L)]
                  for p in range(first, end)]

            def steps():
                for i, p in enumerate(range(first, end)):
                    for l in range(L):
                        kvq.kvq_decode_step_windowed(xs[i][l], packed[2 * l:2 * l + 2],
                                                     scales[2 * l:2 * l + 2], kv[2 * l:2 * l + 2],
                                                     p, signs, rot, g, window)
            for _ in range(2):
                steps()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            gr = torch.cuda.CUDAGraph()
            s2 = torch.cuda.Stream()
            s2.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s2):
                steps()
            torch.cuda.current_stream().wait_stream(s2)
            with torch.cuda.graph(gr):
                steps()
            for _ in range(2):
                gr.replay()
            torch.cuda.synchronize()
            reps = 10
            e0.record()
            for _ in range(reps):
                gr.replay()
            e1.record()
            torch.cuda.synchronize()
            us = 1e3 * e0.elapsed_time(e1) / reps / window
            del gr
            # per window: every step copies the new rows (2d in, 2d out per
            # head); the flush re-reads the window and writes codes, scales and
            # the dequantized rows
            byts = L * 2 * (window * 4 * d + window * (2 * d + fwd_bytes(d, g)))
            out.append({"rot": "srft" if rot == 0 else "srht", "pos": end - 1, "window": window,
                        "graph_us_per_step": us, "algo_bytes_per_step": byts / window,
                        "ideal_us": byts / window / (peak * 1e9) * 1e6})
        del packed, scales, kv
    return out


if __name__ == "__main__":
    main()
