"""Benchmark of the fused rotate+int4 quantize / dequantize+inverse path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
                    [--suite PATH]

One step = the whole hot path over one synthetic SmolLM2-1.7B-shaped KV cache
(24 layers x K,V x 32 kv heads x 4096 tokens x d=64, group 64, SRFT): the
forward kernel (x -> packed codes + scales) then the inverse kernel
(codes + scales -> x_hat).  The cache (805 MB of fp16) is larger than L2, so
no flush is needed between steps.  Metric: GB/s of fp16 KV through the two
kernels (2 * n_vec * d * 2 bytes per step), device-timed with CUDA events.

Under torchrun each rank runs the same workload on its own GPU (independent
shards, no collective on the data path: weak scaling); rank 0 prints one JSON
line with the whole-job value (sum over ranks / max time over ranks).

--impl reference times the CPU oracle (the plain float64 restatement of the
method) on a bounded sample of the same workload on the host cores.
--suite PATH additionally measures every (d, group, rotation, direction) of
the large-batch sweep and the Gemma-3-1B decode-step latency, and writes them
as JSON to PATH.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
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


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on the current kernel sources (else None)."""
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


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

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
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        t0, t1 = (self.marks + [0, 0])[:2] if len(self.marks) >= 2 else (0, 1e30)
        rows = [l for (t, l) in self.lines if t0 - 0.25 <= t <= t1 + 0.25] or \
            [l for (_, l) in self.lines]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [c.strip() for c in r.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


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


def oracle_sample_gbs(x_sample: np.ndarray, signs, rot, group, min_seconds: float,
                      chunk: int = 1 << 16):
    """Oracle fwd + inv over chunks of the sample until `min_seconds` pass.
    Returns (GB/s of fp16 KV, vectors processed, seconds)."""
    import oracle.kvq_oracle as O
    d = x_sample.shape[1]
    done, t0 = 0, time.perf_counter()
    i = 0
    while True:
        part = x_sample[(i * chunk) % len(x_sample):][:chunk]
        p, s = O.rot_quant_fwd(part, signs, rot, group)
        O.dequant_rot_inv(p, s, signs, rot, group)
        done += len(part)
        i += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return 2 * done * d * 2 / el / 1e9, done, el


def headline_shape():
    return W.config(2)


def workload_desc(shape):
    return (f"{shape.name}: {shape.layers} layers x K,V x {shape.heads} kv heads x "
            f"{shape.tokens} tokens x d={shape.d} fp16, group {shape.group}, SRFT, "
            f"forward then inverse over the whole cache")


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle.kvq_oracle as O
    shape = headline_shape()
    d, g = shape.d, shape.group
    small = W.scaled(shape, layers=1, heads=4)  # 32768 vectors of the same recipe
    x = W.make_kv(small).numpy()
    signs = W.make_signs(d)
    per_step = 1 << 14
    times = []
    for k in range(args.warmup + args.steps):
        part = x[(k * per_step) % len(x):][:per_step]
        t0 = time.perf_counter()
        p, s = O.rot_quant_fwd(part, signs, O.SRFT, g)
        O.dequant_rot_inv(p, s, signs, O.SRFT, g)
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = 2 * per_step * d * 2 * len(times) / total / 1e9
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(shape) + f" (CPU oracle: {per_step} vectors per step)",
                   "n_vec_per_step": per_step, "d": d, "group": g, "rot": "srft"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} vectors per step of the {shape.name} recipe"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_kernels(kvq, x, packed, scales, out, signs, rot, g, steps, warmup, sampler=None,
                 lam=None):
    """Device time of `steps` fwd+inv passes; per-kernel sums via events.
    With `lam`, the per-channel lambda entry points."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        kvq.kvq_rot_quant_fwd(x, signs, rot, g, packed, scales, stream, lam=lam)
        kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, out, stream, lam=lam)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark()
    start.record(stream)
    for k in range(steps):
        ev[k][0].record(stream)
        kvq.kvq_rot_quant_fwd(x, signs, rot, g, packed, scales, stream, lam=lam)
        ev[k][1].record(stream)
        kvq.kvq_dequant_rot_inv(packed, scales, signs, rot, g, out, stream, lam=lam)
        ev[k][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    total = start.elapsed_time(end)
    fwd = sum(e[0].elapsed_time(e[1]) for e in ev)
    inv = sum(e[1].elapsed_time(e[2]) for e in ev)
    return total, fwd, inv


def run_e2e(kvq, x, signs, rot, g, packed, scales, out, world, steps, chunks=24):
    n, d = x.shape
    xh = x.cpu().pin_memory()
    oh = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    # chunk bounds on 32-row multiples keep every slice 16-byte aligned
    bounds = [((i * n) // chunks) // 32 * 32 for i in range(chunks)] + [n]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(chunks)]
    ev_run = [torch.cuda.Event() for _ in range(chunks)]
    ev_out = [torch.cuda.Event() for _ in range(chunks)]

    def one_pass():
        for c in range(chunks):
            a, b = bounds[c], bounds[c + 1]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_run[c])  # previous pass done reading x[a:b]
                x[a:b].copy_(xh[a:b], non_blocking=True)
                ev_in[c].record(s_in)
            s_run.wait_event(ev_in[c])
            s_run.wait_event(ev_out[c])  # previous pass done copying out[a:b]
            kvq.kvq_rot_quant_fwd(x[a:b], signs, rot, g, packed[a:b], scales[a:b], s_run)
            kvq.kvq_dequant_rot_inv(packed[a:b], scales[a:b], signs, rot, g, out[a:b], s_run)
            ev_run[c].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run[c])
                oh[a:b].copy_(out[a:b], non_blocking=True)
                ev_out[c].record(s_out)

    e2e_steps = max(3, min(steps, 10))
    for _ in range(2):
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
    if not torch.equal(oh[: bounds[1]], out[: bounds[1]].cpu()):
        raise RuntimeError("end-to-end output differs from the device result")
    e2e_ms = allreduce_max(e0.elapsed_time(e1), world)
    fp16_bytes_step = 2 * n * d * 2
    return {"value": world * e2e_steps * fp16_bytes_step / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
            "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(oh.numel() * 2),
            "chunks": chunks, "gpu_launches_per_step": 2 * chunks}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
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
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.profile:
        run_profile_case(args)
        return
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
    shape = headline_shape()
    d, g, rot = shape.d, shape.group, kvq.SRFT
    x = W.make_kv(shape, device=dev, seed=shape.seed + 1000 * rank)
    n = x.shape[0]
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    packed = torch.empty((n, d // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, d // g), dtype=torch.float32, device=dev)
    out = torch.empty_like(x)

    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                           if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit()
                           else local)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    total_ms, fwd_ms, inv_ms = time_kernels(kvq, x, packed, scales, out, signs, rot, g,
                                            args.steps, args.warmup, sampler)
    barrier(world)
    sampler.stop()
    status = kvq.kvq_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    total_ms = allreduce_max(total_ms, world)

    fp16_bytes_step = 2 * n * d * 2
    value = world * args.steps * fp16_bytes_step / (total_ms * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()
    algo = n * fwd_bytes(d, g)
    dom, dom_ms = ("kvq_fwd_kernel", fwd_ms) if fwd_ms >= inv_ms else ("kvq_inv_kernel", inv_ms)
    achieved = algo / (dom_ms * 1e-3 / args.steps) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": recorded_traffic(dom),
                "kernel": dom, "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": algo}
    detail = {
        "fwd_us": 1e3 * fwd_ms / args.steps, "inv_us": 1e3 * inv_ms / args.steps,
        "fwd_algo_gbs": algo / (fwd_ms * 1e-3 / args.steps) / 1e9,
        "inv_algo_gbs": algo / (inv_ms * 1e-3 / args.steps) / 1e9,
        "n_vec": n,
    }
    detail["fwd_frac"] = detail["fwd_algo_gbs"] / peak
    detail["inv_frac"] = detail["inv_algo_gbs"] / peak
    # vectors per second: each direction alone, and through both per step
    detail["fwd_vec_per_s"] = n / (fwd_ms * 1e-3 / args.steps)
    detail["inv_vec_per_s"] = n / (inv_ms * 1e-3 / args.steps)
    detail["vec_per_s"] = world * args.steps * n / (total_ms * 1e-3)
    # SRHT control on the same cache (context)
    t2, f2, i2 = time_kernels(kvq, x, packed, scales, out, signs, kvq.SRHT, g,
                              max(10, args.steps // 4), 3)
    k2 = max(10, args.steps // 4)
    detail["srht_fwd_algo_gbs"] = algo / (f2 * 1e-3 / k2) / 1e9
    detail["srht_inv_algo_gbs"] = algo / (i2 * 1e-3 / k2) / 1e9
    detail["srht_value_gbs"] = k2 * fp16_bytes_step / (t2 * 1e-3) / 1e9

    # end to end through the public API with host buffers: the cache streams
    # in chunks; host->device copy, forward+inverse and device->host copy of
    # consecutive chunks run on three streams and overlap.
    e2e = run_e2e(kvq, x, signs, rot, g, packed, scales, out, world, args.steps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        idx = W.sample_rows(n, 1 << 18, seed=7)
        xs = x[torch.from_numpy(idx).to(dev)].cpu().numpy()
        v, done, el = oracle_sample_gbs(xs, W.make_signs(d), 0, g, min_seconds=12.0)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{done} vectors (fwd+inv) drawn from {len(idx)} sampled rows of the "
                         f"cache, {el:.1f} s"}

    suite = None
    if args.suite and rank == 0:
        suite_clock = ClockSampler(sampler.gpu)
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
            "config": {"workload": workload_desc(shape), "n_vec": n, "d": d, "group": g,
                       "rot": "srft", "l2": "inputs larger than L2 (805 MB fp16 per pass), no flush",
                       "parallelism": f"independent shards x{world} (no collective)"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": 2 * args.steps, "clocks": clocks, "detail": detail,
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
    """Large-batch sweep (every d, group, rotation, direction) and the
    Gemma-3-1B decode-step latency."""
    res = {"sweep": [], "decode": []}
    peak, _ = hbm_peak()
    for d in (64, 128, 256):
        for g in (32, d):
            shape = W.config(5, d=d, group=g)
            x = W.make_kv(shape, device=dev)
            n = x.shape[0]
            signs = torch.from_numpy(W.make_signs(d)).to(dev)
            packed = torch.empty((n, d // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty((n, d // g), dtype=torch.float32, device=dev)
            out = torch.empty_like(x)
            algo = n * fwd_bytes(d, g)
            for rot in (kvq.SRFT, kvq.SRHT):
                # median of three timed rounds (single rounds move by a few
                # percent between boxes and runs)
                steps = 20
                rounds = [time_kernels(kvq, x, packed, scales, out, signs, rot, g, steps, 3)
                          for _ in range(3)]
                f = statistics.median(r[1] for r in rounds)
                i = statistics.median(r[2] for r in rounds)
                for name, ms in (("fwd", f), ("inv", i)):
                    us = 1e3 * ms / steps
                    res["sweep"].append({
                        "d": d, "group": g, "rot": "srft" if rot == 0 else "srht", "dir": name,
                        "us": us, "algo_gbs": algo / (us * 1e-6) / 1e9,
                        "fp16_gbs": n * d * 2 / (us * 1e-6) / 1e9,
                        "vec_per_s": n / (us * 1e-6), "frac": algo / (us * 1e-6) / 1e9 / peak})
                if g == d and rot == kvq.SRFT:  # other code widths on the same workload
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
                                "d": d, "group": g, "rot": "srft", "bits": bits, "dir": name,
                                "us": us, "algo_gbs": ab / (us * 1e-6) / 1e9,
                                "frac": ab / (us * 1e-6) / 1e9 / peak})
                        del pb
                if g == d:  # the per-channel lambda hook on the same workload
                    lam = torch.exp(0.5 * torch.randn(d, generator=torch.Generator().manual_seed(d)))
                    lam = lam.to(dev)
                    tot, f, i = time_kernels(kvq, x, packed, scales, out, signs, rot, g, steps, 3,
                                             lam=lam)
                    for name, ms in (("fwd", f), ("inv", i)):
                        us = 1e3 * ms / steps
                        res.setdefault("lambda", []).append({
                            "d": d, "group": g, "rot": "srft" if rot == 0 else "srht",
                            "dir": name, "us": us, "algo_gbs": algo / (us * 1e-6) / 1e9,
                            "frac": algo / (us * 1e-6) / 1e9 / peak})
            del x, packed, scales, out
            torch.cuda.empty_cache()
    # decode: 26 layers x (K, V) x d=256, g=256; one call per layer (2 heads)
    shape = W.config(4)
    d, g, L = 256, 256, 26
    seq = W.make_decode_sequence(shape, device=dev)  # [52, 4096, 256]
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    cap = 4096
    for rot in (kvq.SRFT, kvq.SRHT):
        packed = torch.zeros((2 * L, cap, d // 2), dtype=torch.uint8, device=dev)
        scales = torch.zeros((2 * L, cap, 1), dtype=torch.float32, device=dev)
        p, s = kvq.kvq_rot_quant_fwd(seq.reshape(-1, d), signs, rot, g)
        packed.copy_(p.reshape(2 * L, cap, -1))
        scales.copy_(s.reshape(2 * L, cap, -1))
        for pos in (256, 1024, 2048, 4095):
            outs = [torch.empty((2, pos + 1, d), dtype=torch.float16, device=dev)
                    for _ in range(L)]
            xs = [seq[2 * l:2 * l + 2, pos].contiguous() for l in range(L)]

            def step():
                for l in range(L):
                    kvq.kvq_decode_step(xs[l], packed[2 * l:2 * l + 2], scales[2 * l:2 * l + 2],
                                        pos, signs, rot, g, outs[l])
            for _ in range(3):
                step()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 20
            e0.record()
            for _ in range(reps):
                step()
            e1.record()
            torch.cuda.synchronize()
            eager_us = 1e3 * e0.elapsed_time(e1) / reps
            graph_us = None
            try:
                gr = torch.cuda.CUDAGraph()
                s2 = torch.cuda.Stream()
                s2.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(s2):
                    step()
                torch.cuda.current_stream().wait_stream(s2)
                with torch.cuda.graph(gr):
                    step()
                for _ in range(3):
                    gr.replay()
                torch.cuda.synchronize()
                e0.record()
                for _ in range(reps):
                    gr.replay()
                e1.record()
                torch.cuda.synchronize()
                graph_us = 1e3 * e0.elapsed_time(e1) / reps
                del gr
            except Exception as ex:  # capture unsupported: report eager only
                graph_us = f"capture failed: {ex}"
            # per head: new token in (2d) + its codes/scale out + pos+1 rows of
            # codes/scales in and fp16 out (the new row's codes come from registers)
            byts = L * 2 * ((pos + 1) * fwd_bytes(d, g) + 2 * d)
            res["decode"].append({"rot": "srft" if rot == 0 else "srht", "pos": pos,
                                  "eager_us_per_step": eager_us, "graph_us_per_step": graph_us,
                                  "algo_bytes_per_step": byts,
                                  "ideal_us": byts / (peak * 1e9) * 1e6})
    res["decode_windowed"] = run_window_suite(kvq, dev, seq, signs, peak)
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
    layers, 1 KV head with 4 queries, d = g = 256) as a graph of 26 calls, and
    one SmolLM2-1.7B-shaped layer (32 KV heads, 1 query each, d = g = 64) for
    throughput against the HBM roofline (codes + scales of K and V)."""
    out = []
    gen = torch.Generator(device=dev).manual_seed(21)
    cases = [("gemma-3-1b step", 26, 1, 4, 256, 256, (256, 1024, 2048, 4096)),
             ("smollm2-1.7b layer", 1, 32, 1, 64, 64, (1024, 4096, 16384))]
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
                            "len": n, "graph_us": us, "calls": layers,
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
