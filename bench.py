"""Benchmark of the tensor-parallel block on B200 (one JSON line on rank 0).

Headline workload (the decode configuration): one step = the whole decode TP SwiGLU MLP over a
batch of T=64 single-token sequences, d=8192, d_ff=28672, p=8 logical shards, bf16, weights
N(0, 0.02), x N(0, 1): column-parallel up/gate GEMM with the fused SwiGLU, row-parallel down GEMM
giving 8 full-shape partials, in-order partial-sum reduce.  Weight packing is one-time setup.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extras]

For N > 1 launch with torch.distributed.run (one process per GPU).  The path has no exchange
between GPUs (all p shards live on one GPU), so N GPUs run N independent replicas ("weak"
scaling); value = tokens of all ranks / the slowest rank's time.

Also reported (N = 1 only, under "extras"): prefill SwiGLU MLP forward+backward (T=4096),
GQA attention block (s=2048, 64 Q / 8 KV heads), and the 16-layer decode stack.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TP block TFLOP/s (prefill/bwd) and decode tokens/s at 1 B200; % of roofline"
DECODE = dict(T=64, d=8192, F=28672, p=8)
PREFILL = dict(T=4096, d=8192, F=28672, p=8)
ATTN = dict(b=1, s=2048, h=8192, n_q=64, n_kv=8, hd=128, p=8)
STACK = dict(layers=16, h=8192, F=28672, n_q=64, n_kv=8, hd=128, p=8, kv_len=4096)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------------------------ plumbing
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            import torch
            if torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, v):
        if not self.pg:
            return v
        import torch
        t = torch.tensor([float(v)], device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def job_throughput(dist, ms_local, units_per_rank):
    """Whole-job rate of N replicas: every rank processed ``units_per_rank`` units; the job took
    as long as the slowest rank (max over ranks of the device-timed ``ms_local``).  Returns
    (max ms, units of all ranks per second)."""
    ms = dist.max(ms_local)
    return ms, units_per_rank * dist.world / (ms / 1e3)


def smi_id(local):
    """The nvidia-smi -i argument for CUDA device ``local``: with CUDA_VISIBLE_DEVICES set, CUDA
    ordinals are positions in that list, not nvidia-smi indices."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if 0 <= local < len(ids):
            return ids[local]
    return str(local)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while a timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", smi_id(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a moment to write its first row; wait for it (3 s at most) so that
        # a short timed region still falls between samples instead of before the first one
        t_end = time.time() + 3.0
        while time.time() < t_end and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def _cuda_time(fn, steps, stream):
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def _profile(tp, fn, steps):
    import torch
    tp.tp_profile_reset()
    tp.tp_profile_enable(True)
    for _ in range(steps):
        fn()
    torch.cuda.synchronize()
    tp.tp_profile_enable(False)
    prof = tp.tp_profile_read()
    tp.tp_profile_reset()
    return prof


GEMM_SOURCES = ("gemm_tc.cuh", "sm100.cuh", "gemm_launch.cuh", "tp_mlp.cu", "mlp_decode.cuh")


def _gemm_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "tensor_transformer_matmul_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _measured_traffic(label, workload):
    """ncu DRAM bytes per launch for (label, workload), or None if absent or stale."""
    try:
        cur = _gemm_source_hash()
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 4 and not parts[0].startswith("#") and parts[0] == label \
                        and parts[1] == workload:
                    return int(parts[2]) if parts[3] == cur else None
    except Exception:
        pass
    return None


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


# ------------------------------------------------------------------------- workloads
def decode_mlp_bytes():
    c = DECODE
    Fs = c["F"] // c["p"]
    w1 = 2 * c["F"] * c["d"] * 2          # gate + up, bf16
    w2 = c["F"] * c["d"] * 2
    x = c["T"] * c["d"] * 2
    h = c["T"] * c["F"] * 2
    part = c["p"] * c["T"] * c["d"] * 4
    y = c["T"] * c["d"] * 2
    return {"mlp_up_gemm": w1 + x + h, "mlp_down_gemm": w2 + h + part,
            "mlp_decode_gemm": w1 + x + h + w2 + h + part,   # both projections in one launch
            "mlp_down_gemm_fused": w2 + h + y,
            "reduce_partials": part + y, "step": w1 + w2 + x + y, "weights": w1 + w2, "Fs": Fs}


def setup_mlp(tp, inputs, torch, cfg, backward=False, seed=0, reduce_mode=0):
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = inputs.mlp_inputs(cfg["T"], cfg["d"], cfg["F"], "swiglu", "bf16", seed=seed,
                            device=dev, w_std=0.02, backward=backward)
    desc = tp.mlp_desc(cfg["T"], cfg["d"], cfg["F"], cfg["p"], "swiglu", "bf16", reduce_mode)
    st = {"desc": desc, "x": inp["x"], "dy": inp.get("dy")}
    st["w1p"] = torch.empty(tp.tp_mlp_w1_packed_bytes(desc) // 2, dtype=torch.bfloat16, device=dev)
    st["w2p"] = torch.empty(tp.tp_mlp_w2_packed_bytes(desc) // 2, dtype=torch.bfloat16, device=dev)
    tp.tp_mlp_pack(desc, inp["w1"], inp["w_up"], inp["w2"], st["w1p"], st["w2p"])
    st["y"] = torch.empty(cfg["T"], cfg["d"], dtype=torch.bfloat16, device=dev)
    st["ws"] = torch.empty(tp.tp_mlp_fwd_workspace(desc), dtype=torch.uint8, device=dev)
    if backward:
        st["saved"] = torch.empty(tp.tp_mlp_saved_bytes(desc), dtype=torch.uint8, device=dev)
        st["wsb"] = torch.empty(tp.tp_mlp_bwd_workspace(desc), dtype=torch.uint8, device=dev)
        st["dx"] = torch.empty_like(st["y"])
        st["dw1p"] = torch.empty(st["w1p"].numel(), dtype=torch.float32, device=dev)
        st["dw2p"] = torch.empty(st["w2p"].numel(), dtype=torch.float32, device=dev)
    del inp
    return st


def run_ours(args, dist):
    import torch

    from tensor_transformer_matmul_b200 import build, inputs
    from tensor_transformer_matmul_b200 import tpblock as tp

    if not os.path.exists(tp.LIB_PATH):
        build.build()
    tp.load()
    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    stream = torch.cuda.current_stream()
    peaks = _peaks()
    c = DECODE

    mode = tp.TP_REDUCE_FUSED if args.reduce_mode == "fused" else tp.TP_REDUCE_SEPARATE
    st = setup_mlp(tp, inputs, torch, c, seed=dist.rank, reduce_mode=mode)

    def step():
        tp.tp_mlp_fwd(st["desc"], st["x"], st["w1p"], st["w2p"], st["y"], workspace=st["ws"])

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    clk = ClockSampler(dist.local)
    dist.barrier()
    torch.cuda.synchronize()
    clk.start()
    l0 = tp.tp_launch_count()
    ms = _cuda_time(step, args.steps, stream)
    launches = tp.tp_launch_count() - l0
    clocks = clk.stop()
    dist.barrier()
    ms, value = job_throughput(dist, ms, c["T"] * args.steps)
    ms_step = ms / args.steps
    tokens = c["T"] * args.steps * dist.world

    # distribution of single-step times (one event pair per step, 200 steps at most)
    n_q = min(args.steps, 200)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_q)]
    for a_ev, b_ev in evs:
        a_ev.record(stream)
        step()
        b_ev.record(stream)
    torch.cuda.synchronize()
    one = sorted(a_ev.elapsed_time(b_ev) for a_ev, b_ev in evs)
    step_quantiles = {"p10": round(one[int(0.1 * (n_q - 1))], 5),
                      "p50": round(one[int(0.5 * (n_q - 1))], 5),
                      "p90": round(one[int(0.9 * (n_q - 1))], 5), "steps": n_q}

    # per-kernel durations, measured with events on the launching stream over K more steps
    prof = _profile(tp, step, args.steps)
    nbytes = decode_mlp_bytes()
    if mode == tp.TP_REDUCE_FUSED:
        nbytes["mlp_down_gemm"] = nbytes["mlp_down_gemm_fused"]
    dom = max(prof, key=lambda k: prof[k][1])
    dom_ms = prof[dom][1] / prof[dom][0]
    achieved = nbytes.get(dom, 0) / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": _measured_traffic(dom, "decode_mlp"), "peak_source": peaks["source"],
                "algorithmic_bytes_per_launch": nbytes.get(dom, 0),
                "kernel_ms": round(dom_ms, 5)}
    step_gbs = nbytes["step"] / (ms_step / 1e3) / 1e9
    if mode == tp.TP_REDUCE_FUSED:
        nbytes["mlp_down_gemm"] = nbytes["mlp_down_gemm_fused"]
    kernels = {k: {"launches_per_step": v[0] / args.steps, "ms_per_launch": round(v[1] / v[0], 5),
                   "GB_per_s": round(nbytes[k] / (v[1] / v[0] / 1e3) / 1e9, 1) if k in nbytes else None}
               for k, v in prof.items()}

    # end to end through the public API: every step copies its x from pinned host memory to the
    # device, runs the block and copies its y back to pinned host memory.  The copies run on
    # their own streams with two device buffers each, so one step's copies overlap its
    # neighbours' blocks (step i's x lands while step i-1 computes, its y leaves while step i+1
    # computes); the timed region ends when the last y has reached the host.
    xh = st["x"].cpu().pin_memory()
    yh = [torch.empty_like(st["y"], device="cpu").pin_memory() for _ in range(2)]
    xd = [torch.empty_like(st["x"]) for _ in range(2)]
    yd = [torch.empty_like(st["y"]) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    x_in = [torch.cuda.Event() for _ in range(2)]     # x of the buffer's step has landed
    y_out = [torch.cuda.Event() for _ in range(2)]    # the buffer's block is done
    y_home = [torch.cuda.Event() for _ in range(2)]   # its y has reached the host
    step_no = [0]

    def e2e_step():
        b = step_no[0] & 1
        step_no[0] += 1
        with torch.cuda.stream(h2d):
            h2d.wait_event(y_out[b])          # the block two steps back has read xd[b]
            xd[b].copy_(xh, non_blocking=True)
            x_in[b].record(h2d)
        stream.wait_event(x_in[b])
        stream.wait_event(y_home[b])          # yd[b] has been copied out two steps back
        tp.tp_mlp_fwd(st["desc"], xd[b], st["w1p"], st["w2p"], yd[b], workspace=st["ws"])
        y_out[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(y_out[b])
            yh[b].copy_(yd[b], non_blocking=True)
            y_home[b].record(d2h)

    def e2e_time(steps):
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(stream)
        h2d.wait_stream(stream)               # no copy starts before the timed region
        for _ in range(steps):
            e2e_step()
        stream.wait_stream(d2h)               # ... and it ends with the last y on the host
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = dist.max(e2e_time(args.steps))
    e2e = {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": xh.numel() * xh.element_size(),
           "d2h_bytes_per_step": yh[0].numel() * yh[0].element_size(),
           "copies": "own streams, double-buffered, overlapping the neighbouring steps"}

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) activations, drawn on the GPU)",
        "config": {"workload": "decode TP SwiGLU MLP: T=64 (batch 64, s=1), d=8192, d_ff=28672, "
                               "p=8 logical shards, bf16, fp32 accumulate",
                   "reduce_mode": args.reduce_mode,
                   "global_batch": c["T"] * dist.world, "seq_len": 1,
                   "parallelism": f"replicas x{dist.world} (p=8 logical shards per GPU)",
                   "l2": "inputs larger than L2: 1.41 GB of weights streamed per step",
                   "step_GB_per_s": round(step_gbs, 1),
                   "step_frac_of_hbm": round(step_gbs / peaks["hbm_gbs"], 4)},
        "step_ms_quantiles": step_quantiles,
        "roofline": roofline, "e2e": e2e, "gpu_launches": int(launches), "clocks": clocks,
        "kernels": kernels,
    }

    if dist.world == 1 and not args.no_extras:
        del st
        torch.cuda.empty_cache()
        out["extras"] = run_extras(args, tp, inputs, torch, stream, peaks)
    elif dist.world > 1 and not args.no_extras:
        # every rank runs this, in the same order (its collectives must match across ranks)
        del st
        torch.cuda.empty_cache()
        tpm = tp_multi_gpu(args, dist, tp, inputs, torch, stream)
        if dist.rank == 0:
            out["extras"] = {"tp_one_shard_per_gpu": tpm}

    cpu = None
    if dist.world == 1 and dist.rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_config_baselines(seconds=args.cpu_seconds)
        out["cpu_baseline"] = {"value": cpu["2"]["value"], "unit": "tokens/s",
                               "cores": cpu["cores"], "kind": "oracle",
                               "sample": cpu["2"]["sample"] + " (the whole decode MLP), "
                                         f"{args.cpu_seconds:.0f} s"}
    elif dist.rank == 0:
        out["cpu_baseline"] = None
    dist.close()
    if dist.rank == 0:
        # the compact per-configuration summary goes last, so that it survives in the tail of
        # the output even when the line is cut
        out["configs"] = config_summary(out, cpu, peaks)
        print(json.dumps(out), flush=True)


def tp_multi_gpu(args, dist, tp, inputs, torch, stream):
    """The decode MLP (T=64, d=8192, d_ff=28672) with one shard per GPU, p = N: rank r packs and
    holds only shard r (1/N of the weights), computes its partial, and the 1 MiB bf16 partials
    are summed by an NCCL all-reduce over NVLink, one per step (the pages' decode payload).
    Reports the step time (max over ranks) and the latency of every all-reduce."""
    from tensor_transformer_matmul_b200 import tp_dist
    c = DECODE
    dev = torch.device("cuda", torch.cuda.current_device())
    g = tp_dist.TPGroup(timing=False)
    m = tp_dist.ShardedMLP(g, c["T"], c["d"], c["F"], act="swiglu", dtype="bf16",
                           partial_dtype=torch.bfloat16, device=dev)
    # every rank draws the same full weights, packs its own shard, then drops the rest
    inp = inputs.mlp_inputs(c["T"], c["d"], c["F"], "swiglu", "bf16", seed=0, device=dev,
                            w_std=0.02)
    m.pack(inp["w1"], inp["w_up"], inp["w2"])
    x = inp["x"]
    del inp
    torch.cuda.empty_cache()

    def step():
        m.forward(x)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 500))
    dist.barrier()
    torch.cuda.synchronize()
    ms = _cuda_time(step, steps, stream)
    dist.barrier()
    ms = dist.max(ms) / steps
    g.timing = True
    g.count = 0
    n_lat = min(steps, 200)
    for _ in range(n_lat):
        step()
    lat = g.latencies_ms()
    q = _quantiles_us(lat)
    p50_max = dist.max(q["p50"] if q else 0.0)
    return {"workload": f"decode TP SwiGLU MLP: T=64, d=8192, d_ff=28672, one shard per GPU "
                        f"(p={dist.world}), bf16 partials summed by an NCCL all-reduce",
            "ms_per_step": round(ms, 5), "tokens_per_s": round(c["T"] / (ms / 1e3), 1),
            "allreduce_bytes": c["T"] * c["d"] * 2, "allreduces_per_step": g.count // n_lat,
            "allreduce_us": q, "allreduce_us_p50_max_over_ranks": round(p50_max, 2),
            "steps": steps}


def _clocked(gpu, fn, *a, **k):
    """Run one extra workload with the SM clock sampled while it runs; the median under load
    and the throttle reasons go into its result."""
    clk = ClockSampler(gpu)
    clk.start()
    r = fn(*a, **k)
    c = clk.stop()
    if isinstance(r, dict):
        r["clocks"] = c
    return r


def _mhz(d):
    c = (d or {}).get("clocks") or {}
    return c.get("sm_mhz")


def _dom_short(dom):
    if not dom:
        return None
    r = {"k": dom["kernel"]}
    if "frac" in dom:
        r.update({"work": dom["work_per_launch"], "ach": dom["achieved"], "frac": dom["frac"]})
    return r


def config_summary(out, cpu, peaks):
    """Compact per-configuration summary (well under 1.5 KB): value and unit, the dominant
    kernel with its algorithmic work per launch (bytes or flops), achieved rate and fraction of
    the measured peak, the median SM clock while that workload ran, and the oracle's time on the
    host cores for the same configuration."""
    ex = out.get("extras") or {}
    cpu = cpu or {}
    cb = lambda i: [cpu[i]["value"], cpu[i]["unit"]] if i in cpu else None
    r = {"peaks": {"hbm": peaks["hbm_gbs"], "bf16": peaks["bf16_tflops"],
                   "bf16_sust": peaks["bf16_tflops_sustained"], "src": peaks["source"]},
         "cpu_cores": cpu.get("cores")}
    t = ex.get("tiny_mlp")
    if t:
        r["1_tiny"] = {"v": t["us_per_call"], "u": "us/call", "bound": "launch latency",
                       "launches": t["launches_per_call"], "mhz": _mhz(t), "cpu": cb("1")}
    rf = out.get("roofline") or {}
    r["2_decode_mlp"] = {"v": out["value"], "u": "tokens/s",
                         "dom": {"k": rf.get("kernel"),
                                 "work": rf.get("algorithmic_bytes_per_launch"),
                                 "ach": rf.get("achieved"), "frac": rf.get("frac")},
                         "step_frac_hbm": out["config"].get("step_frac_of_hbm"),
                         "mhz": (out.get("clocks") or {}).get("sm_mhz"), "cpu": cb("2")}
    p = ex.get("prefill_mlp_fwd_bwd")
    if p:
        f = p.get("reduce_fused") or p
        r["3_prefill_fwd_bwd"] = {"v": f["TFLOP_per_s"], "u": "TFLOP/s", "mode": "fused",
                                  "frac_burst": f["frac_of_burst_peak"],
                                  "v_separate": p["TFLOP_per_s"],
                                  "dom": _dom_short(f.get("dominant")), "mhz": _mhz(p),
                                  "fwd_vs_cublas": [(p.get("cublas_context") or {}).get(k) for k in
                                                    ("ratio_TFLOP_per_s", "ratio_per_clock")],
                                  "cpu": cb("3"), "cpu_note": "extrapolated" if "3" in cpu else None}
    a = ex.get("attention_block")
    if a:
        f = a.get("reduce_fused") or a
        r["4_attention"] = {"v": f["TFLOP_per_s"], "u": "TFLOP/s", "mode": "fused",
                            "frac_burst": f.get("frac_of_burst_peak"), "v_separate": a["TFLOP_per_s"],
                            "dom": _dom_short(f.get("dominant")), "mhz": _mhz(a), "cpu": cb("4")}
    tpm = ex.get("tp_one_shard_per_gpu")
    if tpm:
        q = tpm.get("allreduce_us") or {}
        r["tp_one_shard_per_gpu"] = {"v": tpm["tokens_per_s"], "u": "tokens/s",
                                     "ms": tpm["ms_per_step"],
                                     "allreduce_us": [q.get("p10"), q.get("p50"), q.get("p90"),
                                                      q.get("max")]}
    st = ex.get("decode_stack")
    if st:
        q = st.get("reduce_us_quantiles") or {}
        r["5_decode_stack"] = {"v": st["tokens_per_s"], "u": "tokens/s",
                               "frac_hbm": st["frac_of_hbm"], "dom": _dom_short(st.get("dominant")),
                               "reduce_us": [q.get("p10"), q.get("p50"), q.get("p90"), q.get("max")],
                               "reduces": st.get("reductions_per_step"), "mhz": _mhz(st),
                               "cpu": cb("5")}
    return r


def run_extras(args, tp, inputs, torch, stream, peaks):
    ex = {}
    which = set(args.extras.split(","))
    steps = max(3, min(args.steps, args.extra_steps))
    gpu = torch.cuda.current_device()
    if "tiny" in which:
        ex["tiny_mlp"] = _clocked(gpu, extra_tiny, tp, inputs, torch, stream)
    # lightest first, with a short idle gap between workloads, so that no extra is timed at the
    # power-capped clocks a previous seconds-long tensor-core run leaves behind
    if "stack" in which:
        ex["decode_stack"] = _clocked(gpu, extra_stack, tp, torch, stream, peaks, steps,
                                      args.reduce_mode)
        time.sleep(1.0)
    if "attention" in which:
        ex["attention_block"] = _clocked(gpu, extra_attention, tp, inputs, torch, stream, peaks,
                                         steps)
        time.sleep(1.0)
        ex["attention_block_bwd"] = _clocked(gpu, extra_attention_bwd, tp, inputs, torch, stream,
                                             peaks, max(3, steps // 4))
        time.sleep(1.0)
    if "prefill" in which:
        ex["prefill_mlp_fwd_bwd"] = _clocked(gpu, extra_prefill, tp, inputs, torch, stream, peaks,
                                             steps)
    if "seqpar" in which:
        time.sleep(1.0)
        ex["seqpar_prefill_mlp_fwd"] = _clocked(gpu, extra_seqpar, tp, inputs, torch, stream,
                                                peaks, steps)
    if "moe" in which:
        time.sleep(1.0)
        ex["moe_layer"] = _clocked(gpu, extra_moe, tp, inputs, torch, stream, peaks, steps)
    return ex


def extra_moe(tp, inputs, torch, stream, peaks, steps):
    """A DeepSeek-V3-shaped MoE layer (hidden 7168, 256 routed experts of width 2048, top-8, one
    shared expert of width 2048; the pages' 7168 hidden size and MoE facts), p=8, bf16 weights
    N(0, 0.02), router N(0, 1/sqrt(d)): the prefill forward at T=4096 and a decode step at T=64."""
    dev = torch.device("cuda", torch.cuda.current_device())
    d, E, k, F, Fs, p = 7168, 256, 8, 2048, 2048, 8
    out = {"workload": "TP MoE layer: d=7168, 256 experts x d_ff 2048, top-8, shared expert "
                       "d_ff 2048, p=8, bf16"}
    desc0 = tp.moe_desc(4096, d, F, Fs, E, k, p)
    w1p = torch.empty(E * tp.tp_moe_expert_w1_bytes(desc0) // 2, dtype=torch.bfloat16, device=dev)
    w2p = torch.empty(E * tp.tp_moe_expert_w2_bytes(desc0) // 2, dtype=torch.bfloat16, device=dev)
    w1s = torch.empty(tp.tp_moe_shared_w1_bytes(desc0) // 2, dtype=torch.bfloat16, device=dev)
    w2s = torch.empty(tp.tp_moe_shared_w2_bytes(desc0) // 2, dtype=torch.bfloat16, device=dev)
    e1, e2 = tp.tp_moe_expert_w1_bytes(desc0) // 2, tp.tp_moe_expert_w2_bytes(desc0) // 2
    # each expert packs like the dense SwiGLU MLP (tp_moe_pack's layout); drawn and packed one at
    # a time so that the unpacked weights never all sit on the device
    ed = tp.mlp_desc(1, d, F, p, "swiglu", "bf16")
    for e in range(E):
        g_, u_, o_ = (inputs.normal(s_, 0.02, 0, 1000 + 3 * e + j, "bf16", dev)
                      for j, s_ in enumerate(((d, F), (d, F), (F, d))))
        tp.tp_mlp_pack(ed, g_, u_, o_, w1p[e * e1:(e + 1) * e1], w2p[e * e2:(e + 1) * e2])
    sg, su, so = (inputs.normal(s_, 0.02, 0, 900 + j, "bf16", dev)
                  for j, s_ in enumerate(((d, Fs), (d, Fs), (Fs, d))))
    tp.tp_mlp_pack(tp.mlp_desc(1, d, Fs, p, "swiglu", "bf16"), sg, su, so, w1s, w2s)
    del sg, su, so
    wr = inputs.normal((d, E), 1.0 / d ** 0.5, 0, 901, "bf16", dev)
    fl_per_row = 2.0 * d * 3 * F
    for T, name in ((4096, "prefill"), (64, "decode")):
        desc = tp.moe_desc(T, d, F, Fs, E, k, p)
        x = inputs.normal((T, d), 1.0, 0, 902, "bf16", dev)
        y = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(tp.tp_moe_fwd_workspace(desc), dtype=torch.uint8, device=dev)

        def fwd():
            tp.tp_moe_fwd(desc, x, wr, w1p, w2p, y, w1p_s=w1s, w2p_s=w2s, residual=x, workspace=ws)

        for _ in range(3):
            fwd()
        ms = _cuda_time(fwd, steps, stream) / steps
        prof = _profile(tp, fwd, steps)
        flops = T * k * fl_per_row + T * 2.0 * d * 3 * Fs + 2.0 * T * d * E
        # the weights every call must stream: the experts the router picks (counted here from the
        # same logits, outside the timed calls) and the shared expert, plus x and y
        with torch.no_grad():
            picked = torch.topk(x.float() @ wr.float(), k, dim=1).indices.unique().numel()
        nbytes = 2 * (picked * (e1 + e2) + w1s.numel() + w2s.numel()) + 2 * 2 * T * d
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3
        t_tc = flops / (peaks["bf16_tflops"] * 1e12) * 1e3
        out[name] = {"T": T, "ms": round(ms, 3),
                     "TFLOP_per_s": round(flops / (ms / 1e3) / 1e12, 1),
                     "frac_of_burst_peak": round(flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"], 3),
                     "experts_hit": picked, "weight_bytes": nbytes,
                     "GB_per_s": round(nbytes / (ms / 1e3) / 1e9, 1),
                     "bound": "hbm" if t_hbm >= t_tc else "tensor",
                     "roofline_ms": round(max(t_hbm, t_tc), 3),
                     "frac_of_roofline": round(max(t_hbm, t_tc) / ms, 3),
                     "tokens_per_s": round(T / (ms / 1e3), 1),
                     "kernels": {kk: {"ms_per_launch": round(v[1] / v[0], 4)} for kk, v in prof.items()}}
        if name == "prefill":
            # the backward: routing and expert activations recomputed, then every chosen expert's
            # MLP backward (expert by expert after one read-back of the row counts), the router's
            # and the shared expert's; fp32 gradients of all 22.7 GB of weights
            del ws
            torch.cuda.empty_cache()
            wsb = torch.empty(tp.tp_moe_bwd_workspace(desc), dtype=torch.uint8, device=dev)
            dy = inputs.normal((T, d), 1.0, 0, 903, "bf16", dev)
            dx = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
            dwr = torch.empty(d, E, dtype=torch.float32, device=dev)
            dw1 = torch.empty(w1p.numel(), dtype=torch.float32, device=dev)
            dw2 = torch.empty(w2p.numel(), dtype=torch.float32, device=dev)
            dws1 = torch.empty(w1s.numel(), dtype=torch.float32, device=dev)
            dws2 = torch.empty(w2s.numel(), dtype=torch.float32, device=dev)

            def bwd():
                tp.tp_moe_bwd(desc, x, wr, w1p, w2p, dy, dx, dwr, dw1, dw2, w1p_s=w1s, w2p_s=w2s,
                              dw1p_s=dws1, dw2p_s=dws2, workspace=wsb)

            bwd()
            nb = 3
            ms_b = _cuda_time(bwd, nb, stream) / nb
            # recomputed forward (without the combine) + the backward GEMMs (2x the forward's)
            out[name]["backward"] = {
                "ms": round(ms_b, 2), "steps": nb,
                "TFLOP_per_s": round(3 * flops / (ms_b / 1e3) / 1e12, 1),
                "grad_bytes_written": 4 * (dw1.numel() + dw2.numel() + dws1.numel() + dws2.numel()),
                "note": "routed experts differentiated expert by expert (host loop over the 256 "
                        "experts, 8 streams side by side)"}
            del wsb, dy, dx, dwr, dw1, dw2, dws1, dws2
        else:
            del ws
        del x, y
        torch.cuda.empty_cache()
    out["steps"] = steps
    del w1p, w2p, w1s, w2s
    torch.cuda.empty_cache()
    return out


def extra_seqpar(tp, inputs, torch, stream, peaks, steps):
    """Sequence-parallel prefill MLP forward (T=4096, d=8192, d_ff=28672, p=8): x arrives as the
    8 shards' token slices and y leaves as slices -- all-gather, the two GEMMs, then the
    reduce-scatter with the residual add and RMSNorm on the slices -- against the plain forward
    with the same residual and norm."""
    c = PREFILL
    st = setup_mlp(tp, inputs, torch, c)
    dev = st["x"].device
    T, d, p = c["T"], c["d"], c["p"]
    R = T // p
    res = inputs.normal((T, d), 1.0, 0, 98, "bf16", dev)
    yn = torch.empty_like(st["y"])
    cut = lambda t: [t[i * R:(i + 1) * R].clone() for i in range(p)]
    xs, rs = cut(st["x"]), cut(res)
    ys = [torch.empty(R, d, dtype=torch.bfloat16, device=dev) for _ in range(p)]
    yns = [torch.empty_like(ys[0]) for _ in range(p)]
    ws = torch.empty(tp.tp_mlp_fwd_sp_workspace(st["desc"]), dtype=torch.uint8, device=dev)

    def plain():
        tp.tp_mlp_fwd(st["desc"], st["x"], st["w1p"], st["w2p"], st["y"], residual=res,
                      workspace=st["ws"], y_norm=yn)

    def spf():
        tp.tp_mlp_fwd_sp(st["desc"], xs, st["w1p"], st["w2p"], ys, residual_slices=rs,
                         y_norm_slices=yns, workspace=ws)

    for _ in range(3):
        plain()
        spf()
    ms_plain = _cuda_time(plain, steps, stream) / steps
    ms_sp = _cuda_time(spf, steps, stream) / steps
    prof = _profile(tp, spf, steps)
    # algorithmic bytes: the reduce-scatter reads the p fp32 partials and the residual slices
    # and writes y and its norm (bf16); the all-gather reads and writes x once
    coll = {"reduce_scatter": p * T * d * 4 + 3 * T * d * 2, "all_gather": 2 * T * d * 2}
    kern = {}
    for k, (n, ms) in prof.items():
        e = {"ms_per_launch": round(ms / n, 4)}
        if k in coll:
            gbs = coll[k] / (ms / n / 1e3) / 1e9
            e.update({"algorithmic_bytes": coll[k], "GB_per_s": round(gbs, 1),
                      "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 3)})
        kern[k] = e
    same = bool(torch.equal(torch.cat(ys), st["y"]) and torch.equal(torch.cat(yns), yn))
    del st
    torch.cuda.empty_cache()
    return {"workload": "sequence-parallel prefill TP SwiGLU MLP forward: T=4096 as 8 slices of "
                        "512 tokens, d=8192, d_ff=28672, p=8, bf16, residual + RMSNorm on slices",
            "ms": round(ms_sp, 3), "ms_plain_forward": round(ms_plain, 3),
            "TFLOP_per_s": round(2.0 * T * d * c["F"] * 3 / (ms_sp / 1e3) / 1e12, 1),
            "slices_equal_plain_rows": same, "kernels": kern, "steps": steps}


def extra_tiny(tp, inputs, torch, stream, calls=2000):
    """The tiny configuration (T=4, d=8, d_ff=32, p=4, GELU, fp32): launch-latency bound, so it
    is reported as microseconds per forward call (every call enqueues the up GEMM, the partial
    GEMM and the reduce)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = inputs.mlp_inputs(4, 8, 32, "gelu", "f32", seed=0, device=dev)
    d = tp.mlp_desc(4, 8, 32, 4, "gelu", "f32")
    w1p = torch.empty(tp.tp_mlp_w1_packed_bytes(d) // 4, dtype=torch.float32, device=dev)
    w2p = torch.empty(tp.tp_mlp_w2_packed_bytes(d) // 4, dtype=torch.float32, device=dev)
    tp.tp_mlp_pack(d, inp["w1"], None, inp["w2"], w1p, w2p)
    ws = torch.empty(tp.tp_mlp_fwd_workspace(d), dtype=torch.uint8, device=dev)
    y = torch.empty(4, 8, dtype=torch.float32, device=dev)

    def fwd():
        tp.tp_mlp_fwd(d, inp["x"], w1p, w2p, y, workspace=ws)

    for _ in range(20):
        fwd()
    ms = _cuda_time(fwd, calls, stream)
    l0 = tp.tp_launch_count()
    fwd()
    launches = tp.tp_launch_count() - l0
    return {"workload": "tiny MLP: T=4, d=8, d_ff=32, p=4 logical shards, GELU, fp32",
            "us_per_call": round(ms / calls * 1e3, 2), "launches_per_call": int(launches),
            "calls": calls}


def _dominant(prof, work, peak, unit):
    """The kernel with the largest summed time in ``prof`` ({label: (launches, ms)}), with its
    algorithmic work per launch (``work``: label -> bytes or flops), achieved rate and fraction of
    ``peak``."""
    if not prof:
        return None
    k = max(prof, key=lambda q: prof[q][1])
    n, ms = prof[k]
    out = {"kernel": k, "ms_per_launch": round(ms / n, 5), "share": round(ms / sum(v[1] for v in prof.values()), 3)}
    if k in work:
        scale = 1e9 if unit == "GB/s" else 1e12
        ach = work[k] / (ms / n / 1e3) / scale
        out.update({"work_per_launch": work[k], "achieved": round(ach, 1), "unit": unit,
                    "frac": round(ach / peak, 4)})
    return out


def _quantiles_us(ms_list):
    """p10 / p50 / p90 / max of a list of durations in ms, in microseconds."""
    if not ms_list:
        return None
    v = sorted(ms_list)
    q = lambda f: round(v[int(f * (len(v) - 1))] * 1e3, 2)
    return {"p10": q(0.1), "p50": q(0.5), "p90": q(0.9), "max": round(v[-1] * 1e3, 2),
            "n": len(v)}


def extra_stack(tp, torch, stream, peaks, steps, reduce_mode="separate"):
    """16 Llama-70B-shaped decode layers, b=1, KV length 4096, replayed as one CUDA graph."""
    from tensor_transformer_matmul_b200.decode_stack import DecodeStack
    c = STACK
    st = DecodeStack(c["layers"], c["h"], c["F"], c["n_q"], c["n_kv"], c["hd"], c["p"],
                     c["kv_len"], b=1, seed=0,
                     reduce_mode=tp.TP_REDUCE_FUSED if reduce_mode == "fused" else tp.TP_REDUCE_SEPARATE)
    dev = torch.device("cuda", torch.cuda.current_device())
    x = torch.randn(1, 1, c["h"], device=dev)   # float32 residual stream
    st.capture(x)
    for _ in range(3):
        st.replay()
    torch.cuda.synchronize()
    ms = _cuda_time(st.replay, steps, stream) / steps
    # eager steps with the event profiler: per-kernel split and the latency of every reduction
    # (the on-device stand-in for the per-collective latency of a replayed iteration)
    tp.tp_reset_reduction_count()
    n_prof = max(3, steps // 4)
    tp.tp_profile_reset()
    tp.tp_profile_enable(True)
    for _ in range(n_prof):
        st.step(x)
    torch.cuda.synchronize()
    tp.tp_profile_enable(False)
    prof = tp.tp_profile_read()
    red_ms = sorted(tp.tp_profile_launch_ms("reduce_partials"))
    tp.tp_profile_reset()
    per_layer_w = (tp.tp_attn_wqkv_packed_bytes(st.adesc) + tp.tp_attn_wo_packed_bytes(st.adesc)
                   + tp.tp_mlp_w1_packed_bytes(st.mdesc) + tp.tp_mlp_w2_packed_bytes(st.mdesc))
    kv = 2 * c["n_kv"] * (c["kv_len"] + 1) * c["hd"] * 2
    nbytes = c["layers"] * (per_layer_w + kv)
    gbs = nbytes / (ms / 1e3) / 1e9
    red = prof.get("reduce_partials", (0, 0.0))
    h, Fsp = c["h"], -(-c["F"] // c["p"] // 128) * 128
    qkv = (c["n_q"] + 2 * c["n_kv"]) * c["hd"]
    work = {"mlp_up_gemm": tp.tp_mlp_w1_packed_bytes(st.mdesc) + 2 * h + 2 * c["p"] * 2 * Fsp,
            "mlp_down_gemm": tp.tp_mlp_w2_packed_bytes(st.mdesc) + 2 * c["p"] * Fsp + 4 * c["p"] * h,
            "mlp_decode_gemm": tp.tp_mlp_w1_packed_bytes(st.mdesc) + tp.tp_mlp_w2_packed_bytes(st.mdesc)
            + 2 * h + 2 * 2 * c["p"] * Fsp + 4 * c["p"] * h,
            "attn_qkv_gemm": tp.tp_attn_wqkv_packed_bytes(st.adesc) + 2 * h + 2 * qkv,
            "attn_out_gemm": tp.tp_attn_wo_packed_bytes(st.adesc) + 2 * c["n_q"] * c["hd"]
            + 4 * c["p"] * h,
            "attn_decode": kv}
    out = {"workload": "decode stack: 16 layers (GQA attention s=1 over KV 4096+1, SwiGLU MLP "
                       "d_ff=28672), b=1, p=8, 2 reductions of 1x8192 per layer, CUDA graph",
           "ms_per_token": round(ms, 4), "tokens_per_s": round(1e3 / ms, 1),
           "GB_per_s": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
           "bytes_per_step": nbytes,
           "reductions_per_step": red[0] // n_prof,
           "reduce_us_mean": round(red[1] / max(1, red[0]) * 1e3, 2),
           "reduce_us_quantiles": _quantiles_us(red_ms),
           "dominant": _dominant(prof, work, peaks["hbm_gbs"], "GB/s"),
           "kernels": {k: {"launches_per_step": v[0] / n_prof,
                           "ms_per_step": round(v[1] / n_prof, 4),
                           "ms_per_launch": round(v[1] / v[0], 5)}
                       for k, v in prof.items()},
           "steps": steps}
    del st
    torch.cuda.empty_cache()
    return out


def extra_prefill(tp, inputs, torch, stream, peaks, steps):
    # prefill SwiGLU MLP forward + backward: 6 T d F flops per direction pair x 3 matmuls
    res = _prefill_mode(tp, inputs, torch, stream, peaks, steps, tp.TP_REDUCE_SEPARATE)
    fused = _prefill_mode(tp, inputs, torch, stream, peaks, steps, tp.TP_REDUCE_FUSED)
    res["reduce_fused"] = {k: fused[k] for k in ("ms_fwd", "ms_bwd", "TFLOP_per_s",
                                                  "frac_of_burst_peak", "frac_of_sustained_peak",
                                                  "tokens_per_s", "dominant", "kernels")}
    res["cublas_context"] = _cublas_context(tp, inputs, torch, stream)
    return res


def _cublas_context(tp, inputs, torch, stream, region_s=1.0):
    """Context only, not this library's path: the prefill forward's two GEMM shapes (all shards at
    once: T x d by d x 2 d_ff with the SwiGLU epilogue, then T x d_ff by d_ff x d with the shard
    sum) run by this library (tp_mlp_fwd, TP_REDUCE_FUSED) and by torch.matmul (cuBLAS), in
    alternating timed regions of about ``region_s`` seconds each, with the SM clock sampled in
    every region.  Both are reported as TFLOP/s and as flop per clock per SM, so that a gap that
    comes from the power-capped clock is told apart from one in the kernels."""
    try:
        c = PREFILL
        dev = torch.device("cuda", torch.cuda.current_device())
        gpu = torch.cuda.current_device()
        nsm = torch.cuda.get_device_properties(dev).multi_processor_count
        st = setup_mlp(tp, inputs, torch, c, reduce_mode=tp.TP_REDUCE_FUSED)
        g = torch.Generator(device=dev)
        g.manual_seed(7)
        a1 = torch.randn(c["T"], c["d"], generator=g, device=dev).to(torch.bfloat16)
        b1 = torch.randn(c["d"], 2 * c["F"], generator=g, device=dev).to(torch.bfloat16)
        a2 = torch.randn(c["T"], c["F"], generator=g, device=dev).to(torch.bfloat16)
        b2 = torch.randn(c["F"], c["d"], generator=g, device=dev).to(torch.bfloat16)
        flops = 2.0 * c["T"] * c["d"] * 2 * c["F"] + 2.0 * c["T"] * c["F"] * c["d"]

        def ours():
            tp.tp_mlp_fwd(st["desc"], st["x"], st["w1p"], st["w2p"], st["y"], workspace=st["ws"])

        def cublas():
            torch.matmul(a1, b1)
            torch.matmul(a2, b2)

        for fn in (ours, cublas):
            for _ in range(3):
                fn()
        torch.cuda.synchronize()
        ms1 = {"ours": _cuda_time(ours, 5, stream) / 5, "cublas": _cuda_time(cublas, 5, stream) / 5}
        reps = {k: max(5, int(region_s * 1e3 / v)) for k, v in ms1.items()}
        rows = {"ours": [], "cublas": []}
        for _ in range(2):
            for name, fn in (("ours", ours), ("cublas", cublas)):
                time.sleep(0.5)
                clk = ClockSampler(gpu)
                clk.start()
                ms = _cuda_time(fn, reps[name], stream) / reps[name]
                ck = clk.stop() or {}
                rows[name].append((ms, ck.get("sm_mhz")))
        out = {"shapes": "T=4096: [4096x8192]x[8192x57344] + [4096x28672]x[28672x8192]",
               "region_s": region_s}
        for name, r in rows.items():
            ms = min(x[0] for x in r)
            mhz = [x[1] for x in r if x[1]]
            mhz_med = statistics.median(mhz) if mhz else None
            tf = flops / (ms / 1e3) / 1e12
            out[name] = {"ms": round(ms, 3), "TFLOP_per_s": round(tf, 1), "sm_mhz": mhz_med,
                         "flop_per_clk_per_sm": round(tf * 1e12 / (mhz_med * 1e6) / nsm, 1)
                         if mhz_med else None}
        if out["ours"]["flop_per_clk_per_sm"] and out["cublas"]["flop_per_clk_per_sm"]:
            out["ratio_TFLOP_per_s"] = round(out["ours"]["TFLOP_per_s"] / out["cublas"]["TFLOP_per_s"], 3)
            out["ratio_per_clock"] = round(out["ours"]["flop_per_clk_per_sm"]
                                           / out["cublas"]["flop_per_clk_per_sm"], 3)
        del st, a1, b1, a2, b2
        torch.cuda.empty_cache()
        return out
    except Exception as e:  # context only: never fail the bench over it
        return {"error": f"{type(e).__name__}: {e}"[:200]}


def _prefill_mode(tp, inputs, torch, stream, peaks, steps, mode):
    """The prefill step with the shard partials summed by a separate reduce (TP_REDUCE_SEPARATE)
    or inside the down and dx GEMMs' accumulators (TP_REDUCE_FUSED)."""
    c = PREFILL
    st = setup_mlp(tp, inputs, torch, c, backward=True, reduce_mode=mode)

    def fwd():
        tp.tp_mlp_fwd(st["desc"], st["x"], st["w1p"], st["w2p"], st["y"], saved=st["saved"],
                      workspace=st["ws"])

    def bwd():
        tp.tp_mlp_bwd(st["desc"], st["dy"], st["x"], st["saved"], st["w1p"], st["w2p"], st["dx"],
                      st["dw1p"], st["dw2p"], workspace=st["wsb"])

    def both():
        fwd()
        bwd()

    for _ in range(3):
        both()
    f_fl = 2.0 * c["T"] * c["d"] * c["F"] * 3
    b_fl = 2 * f_fl
    ms_f = _cuda_time(fwd, steps, stream) / steps
    ms_b = _cuda_time(bwd, steps, stream) / steps
    prof = _profile(tp, both, steps)
    gemm_fl = {"mlp_up_gemm": 2.0 * c["T"] * c["d"] * 2 * c["F"],
               "mlp_down_gemm": 2.0 * c["T"] * c["d"] * c["F"],
               "mlp_dh_gemm": 2.0 * c["T"] * c["d"] * c["F"],
               "mlp_dw2_gemm": 2.0 * c["T"] * c["d"] * c["F"],
               "mlp_dw1_gemm": 2.0 * c["T"] * c["d"] * 2 * c["F"],
               "mlp_dx_gemm": 2.0 * c["T"] * c["d"] * 2 * c["F"]}
    kern = {}
    for k, (n, ms) in prof.items():
        e = {"ms_per_launch": round(ms / n, 4)}
        if k in gemm_fl:
            tf = gemm_fl[k] / (ms / n / 1e3) / 1e12
            e["TFLOP_per_s"] = round(tf, 1)
            e["frac_of_sustained_peak"] = round(tf / peaks["bf16_tflops_sustained"], 3)
        kern[k] = e
    tot = (ms_f + ms_b)
    dom = _dominant(prof, gemm_fl, peaks["bf16_tflops"], "TFLOP/s")
    res = {
        "workload": "prefill TP SwiGLU MLP fwd+bwd: T=4096, d=8192, d_ff=28672, p=8, bf16",
        "ms_fwd": round(ms_f, 3), "ms_bwd": round(ms_b, 3),
        "TFLOP_per_s": round((f_fl + b_fl) / (tot / 1e3) / 1e12, 1),
        "TFLOP_per_s_fwd": round(f_fl / (ms_f / 1e3) / 1e12, 1),
        "TFLOP_per_s_bwd": round(b_fl / (ms_b / 1e3) / 1e12, 1),
        "frac_of_burst_peak": round((f_fl + b_fl) / (tot / 1e3) / 1e12 / peaks["bf16_tflops"], 3),
        "frac_of_sustained_peak": round((f_fl + b_fl) / (tot / 1e3) / 1e12 / peaks["bf16_tflops_sustained"], 3),
        "tokens_per_s": round(c["T"] / (tot / 1e3), 1), "dominant": dom, "kernels": kern,
        "steps": steps}
    del st
    torch.cuda.empty_cache()
    return res


def extra_attention(tp, inputs, torch, stream, peaks, steps):
    """GQA attention block (prefill): QKV + causal local attention + O-proj + reduce."""
    a = ATTN
    dev = torch.device("cuda", torch.cuda.current_device())
    ai = inputs.attn_inputs(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], "bf16", seed=0,
                            device=dev)
    ad = tp.attn_desc(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], a["p"])
    adf = tp.attn_desc(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], a["p"],
                       reduce_mode=tp.TP_REDUCE_FUSED)
    wqkv = torch.empty(tp.tp_attn_wqkv_packed_bytes(ad) // 2, dtype=torch.bfloat16, device=dev)
    wo = torch.empty(tp.tp_attn_wo_packed_bytes(ad) // 2, dtype=torch.bfloat16, device=dev)
    tp.tp_attn_pack(ad, ai["wq"], ai["wk"], ai["wv"], ai["wo"], wqkv, wo)
    ya = torch.empty_like(ai["x"])
    wsa = torch.empty(max(tp.tp_attn_fwd_workspace(ad), tp.tp_attn_fwd_workspace(adf)),
                      dtype=torch.uint8, device=dev)

    def attn():
        tp.tp_attn_fwd(ad, ai["x"], wqkv, wo, ya, workspace=wsa)

    def attn_fused():
        tp.tp_attn_fwd(adf, ai["x"], wqkv, wo, ya, workspace=wsa)

    for _ in range(3):
        attn()
        attn_fused()
    ms_a = _cuda_time(attn, steps, stream) / steps
    ms_af = _cuda_time(attn_fused, steps, stream) / steps
    s, h = a["s"], a["h"]
    fl_qkv = 2.0 * s * h * (a["n_q"] + 2 * a["n_kv"]) * a["hd"]
    fl_att = 2.0 * 2 * a["n_q"] * a["hd"] * s * (s + 1) / 2
    fl_o = 2.0 * s * a["n_q"] * a["hd"] * h
    prof = _profile(tp, attn, steps)
    prof_f = _profile(tp, attn_fused, steps)
    work = {"attn_qkv_gemm": fl_qkv, "attn_prefill": fl_att, "attn_out_gemm": fl_o}
    pk = peaks["bf16_tflops"]
    return {
        "workload": "TP GQA attention: b=1, s=2048, h=8192, 64 Q / 8 KV heads, hd=128, p=8, causal",
        "ms": round(ms_a, 3),
        "TFLOP_per_s": round((fl_qkv + fl_att + fl_o) / (ms_a / 1e3) / 1e12, 1),
        "frac_of_burst_peak": round((fl_qkv + fl_att + fl_o) / (ms_a / 1e3) / 1e12 / peaks["bf16_tflops"], 3),
        "tokens_per_s": round(s / (ms_a / 1e3), 1),
        "dominant": _dominant(prof, work, pk, "TFLOP/s"),
        "kernels": {k: {"ms_per_launch": round(v[1] / v[0], 4)} for k, v in prof.items()},
        "reduce_fused": {"ms": round(ms_af, 3),
                         "TFLOP_per_s": round((fl_qkv + fl_att + fl_o) / (ms_af / 1e3) / 1e12, 1),
                         "frac_of_burst_peak": round((fl_qkv + fl_att + fl_o) / (ms_af / 1e3)
                                                     / 1e12 / pk, 3),
                         "dominant": _dominant(prof_f, work, pk, "TFLOP/s"),
                         "kernels": {k: {"ms_per_launch": round(v[1] / v[0], 4)}
                                     for k, v in prof_f.items()}},
        "steps": steps}


def extra_attention_bwd(tp, inputs, torch, stream, peaks, steps):
    """Backward of the GQA attention block (prefill): recomputed forward, dO and dWo GEMMs,
    dQ/dK/dV, dWqkv and dX GEMMs, dX reduce."""
    a = ATTN
    dev = torch.device("cuda", torch.cuda.current_device())
    ai = inputs.attn_inputs(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], "bf16", seed=0,
                            device=dev)
    ad = tp.attn_desc(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], a["p"])
    wqkv = torch.empty(tp.tp_attn_wqkv_packed_bytes(ad) // 2, dtype=torch.bfloat16, device=dev)
    wo = torch.empty(tp.tp_attn_wo_packed_bytes(ad) // 2, dtype=torch.bfloat16, device=dev)
    tp.tp_attn_pack(ad, ai["wq"], ai["wk"], ai["wv"], ai["wo"], wqkv, wo)
    dy = inputs.normal((a["b"], a["s"], a["h"]), 1.0, 0, 97, "bf16", dev)
    dx = torch.empty_like(ai["x"])
    dwqkv = torch.empty(wqkv.numel(), dtype=torch.float32, device=dev)
    dwo = torch.empty(wo.numel(), dtype=torch.float32, device=dev)
    adf = tp.attn_desc(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], a["p"],
                       reduce_mode=tp.TP_REDUCE_FUSED)
    ws = torch.empty(max(tp.tp_attn_bwd_workspace(ad), tp.tp_attn_bwd_workspace(adf)),
                     dtype=torch.uint8, device=dev)

    def bwd():
        tp.tp_attn_bwd(ad, ai["x"], wqkv, wo, dy, dx, dwqkv, dwo, workspace=ws)

    def bwd_fused():
        tp.tp_attn_bwd(adf, ai["x"], wqkv, wo, dy, dx, dwqkv, dwo, workspace=ws)

    for _ in range(3):
        bwd()
        bwd_fused()
    ms = _cuda_time(bwd, steps, stream) / steps
    ms_f = _cuda_time(bwd_fused, steps, stream) / steps
    s, h = a["s"], a["h"]
    rqkv = (a["n_q"] + 2 * a["n_kv"]) * a["hd"]
    fl_proj = 2.0 * s * h * rqkv            # one projection-sized GEMM (QKV)
    fl_o = 2.0 * s * a["n_q"] * a["hd"] * h  # one O-projection-sized GEMM
    fl_att = 2.0 * 2 * a["n_q"] * a["hd"] * s * (s + 1) / 2
    # recomputed forward (QKV GEMM + attention), dO and dWo, dQ/dK/dV (2.5x the forward's
    # attention matmuls), dWqkv and dX
    flops = fl_proj + fl_att + 2 * fl_o + 2.5 * fl_att + 2 * fl_proj
    prof = _profile(tp, bwd, steps)
    return {
        "workload": "TP GQA attention backward: b=1, s=2048, h=8192, 64 Q / 8 KV heads, hd=128, "
                    "p=8, causal (forward recomputed inside)",
        "ms": round(ms, 3),
        "TFLOP_per_s": round(flops / (ms / 1e3) / 1e12, 1),
        "frac_of_burst_peak": round(flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"], 3),
        "kernels": {k: {"ms_per_launch": round(v[1] / v[0], 4)} for k, v in prof.items()},
        "reduce_fused": {"ms": round(ms_f, 3),
                         "TFLOP_per_s": round(flops / (ms_f / 1e3) / 1e12, 1)},
        "steps": steps}


# -------------------------------------------------------------------------- CPU side
ORACLE_CHUNK = 512   # d_ff features per oracle step


def _oracle_decode_setup():
    """Host float64 copies of the decode workload's weights (drawn on the CPU)."""
    from tensor_transformer_matmul_b200 import inputs
    c = DECODE
    inp = inputs.mlp_inputs(c["T"], c["d"], c["F"], "swiglu", "bf16", seed=0, device="cpu",
                            w_std=0.02)
    return {k: inputs.to_f64(v) for k, v in inp.items() if v is not None}


def _oracle_step(a, i):
    """One bounded sample of the decode MLP on the oracle: all 64 tokens through a 512-feature
    slice of d_ff (its contribution to y).  Worth 64 * 512 / d_ff token-equivalents."""
    from oracle import mlp as omlp
    n = DECODE["F"] // ORACLE_CHUNK
    c = slice((i % n) * ORACLE_CHUNK, (i % n + 1) * ORACLE_CHUNK)
    return omlp.mlp_forward(a["x"], a["w1"][:, c], a["w2"][c, :], "swiglu", a["w_up"][:, c])


TOKENS_PER_ORACLE_STEP = DECODE["T"] * ORACLE_CHUNK / DECODE["F"]


def cpu_baseline(seconds=10.0, arrays=None):
    """The oracle (float64 numpy, as it stands) on the host cores, in decode tokens/s."""
    a = arrays if arrays is not None else _oracle_decode_setup()
    n, t0 = 0, time.perf_counter()
    while True:
        _oracle_step(a, n)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": round(n * TOKENS_PER_ORACLE_STEP / el, 3), "unit": "tokens/s",
            "cores": _threads(), "kind": "oracle",
            "sample": f"{n} oracle calls, each all 64 tokens through a {ORACLE_CHUNK}-feature slice "
                      f"of d_ff ({TOKENS_PER_ORACLE_STEP:.3f} token-equivalents), {el:.1f} s"}


def _timed(fn, seconds, min_calls=1):
    """Call fn until ``seconds`` have passed (at least ``min_calls`` times); (calls, seconds)."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if n >= min_calls and el >= seconds:
            return n, el


def cpu_config_baselines(seconds=10.0):
    """The oracle (float64 numpy, as it stands) on the host cores for every configuration, in the
    unit the GPU number of that configuration is reported in.

    * tiny MLP (T=4, d=8, d_ff=32, GELU): full calls, us per call;
    * decode MLP (T=64, d=8192, d_ff=28672): full calls, tokens/s;
    * prefill MLP forward + backward (T=4096): a 64-token sample of forward + backward (every
      GEMM's flops scale with the tokens), TFLOP/s and the step time extrapolated by the token
      ratio -- labelled "extrapolated";
    * attention block (s=2048, 64/8 heads): full calls, TFLOP/s (causal half counted, as for
      the GPU);
    * decode stack (16 layers, KV 4096): one layer timed in full, x 16 (the layers have the same
      shapes), tokens/s.
    Inputs are the configurations' seeded draws made on the host.  The returned dict maps
    "1".."5" to {value, unit, sample}, plus the thread count."""
    from oracle import attention as oattn
    from oracle import decode as odec
    from oracle import mlp as omlp
    from tensor_transformer_matmul_b200 import inputs
    f64 = inputs.to_f64
    out = {"cores": _threads()}

    tiny = inputs.mlp_inputs(4, 8, 32, "gelu", "f32", seed=0)
    t = {k: f64(v) for k, v in tiny.items() if v is not None}
    n, el = _timed(lambda: omlp.mlp_forward(t["x"], t["w1"], t["w2"], "gelu"), min(1.0, seconds))
    out["1"] = {"value": round(el / n * 1e6, 2), "unit": "us/call", "sample": f"{n} full calls"}

    c = DECODE
    m = inputs.mlp_inputs(c["T"], c["d"], c["F"], "swiglu", "bf16", seed=0, device="cpu",
                          w_std=0.02)
    W = {k: f64(v) for k, v in m.items() if v is not None}
    del m
    n, el = _timed(lambda: omlp.mlp_forward(W["x"], W["w1"], W["w2"], "swiglu", W["w_up"]),
                   seconds)
    out["2"] = {"value": round(n * c["T"] / el, 2), "unit": "tokens/s",
                "sample": f"{n} full calls of T=64"}

    P, S = PREFILL, 64
    x3 = f64(inputs.normal((S, P["d"]), 1.0, 0, inputs.S_X, "bf16"))
    dy3 = f64(inputs.normal((S, P["d"]), 1.0, 0, inputs.S_DY, "bf16"))

    def fb():
        omlp.mlp_forward(x3, W["w1"], W["w2"], "swiglu", W["w_up"])
        omlp.mlp_backward(x3, W["w1"], W["w2"], dy3, "swiglu", W["w_up"])

    n, el = _timed(fb, seconds / 2)
    fl = 6.0 * S * P["d"] * P["F"] * 3
    out["3"] = {"value": round(fl * n / el / 1e12, 4), "unit": "TFLOP/s",
                "ms_per_step": round(el / n * (P["T"] / S) * 1e3, 1),
                "sample": f"{n} forward+backward calls of {S} of the {P['T']} tokens; step time "
                          f"extrapolated by the token ratio"}

    a = ATTN
    ai = inputs.attn_inputs(a["b"], a["s"], a["h"], a["n_q"], a["n_kv"], a["hd"], "bf16", seed=0)
    A = {k: f64(v) for k, v in ai.items()}
    del ai
    n, el = _timed(lambda: oattn.attention_forward(A["x"], A["wq"], A["wk"], A["wv"], A["wo"],
                                                   a["n_q"], a["n_kv"], a["hd"], causal=True), 0.0)
    s_, h_ = a["s"], a["h"]
    fl = (2.0 * s_ * h_ * (a["n_q"] + 2 * a["n_kv"]) * a["hd"] + 2.0 * s_ * a["n_q"] * a["hd"] * h_
          + 4.0 * a["n_q"] * a["hd"] * s_ * (s_ + 1) / 2)
    out["4"] = {"value": round(fl * n / el / 1e12, 4), "unit": "TFLOP/s",
                "sample": f"{n} full calls"}

    k = STACK
    cache = inputs.attn_inputs(1, 1, k["h"], k["n_q"], k["n_kv"], k["hd"], "bf16", seed=0,
                               kv_len=k["kv_len"])
    kc = f64(cache["k_cache"])[:, :, :k["kv_len"]]
    vc = f64(cache["v_cache"])[:, :, :k["kv_len"]]
    xd = f64(cache["x"])[:, 0]
    del cache
    lw = {"wq": A["wq"], "wk": A["wk"], "wv": A["wv"], "wo": A["wo"], "wg": W["w1"],
          "wu": W["w_up"], "w2": W["w2"]}
    n, el = _timed(lambda: odec.decode_layer(xd, lw, kc, vc, k["n_q"], k["n_kv"], k["hd"]),
                   seconds / 2)
    out["5"] = {"value": round(1.0 / (el / n * k["layers"]), 3), "unit": "tokens/s",
                "sample": f"one layer timed over {n} calls, x {k['layers']} layers"}
    return out


def run_reference(args, dist):
    """The oracle as the reference arm: same workload, metric and unit, on the host cores."""
    if dist.rank != 0:
        return
    a = _oracle_decode_setup()
    for i in range(max(1, args.warmup)):
        _oracle_step(a, i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        _oracle_step(a, i)
    el = time.perf_counter() - t0
    value = TOKENS_PER_ORACLE_STEP * args.steps / el
    sample = (f"{args.steps} steps, each all 64 tokens through a {ORACLE_CHUNK}-feature slice of "
              f"d_ff ({TOKENS_PER_ORACLE_STEP:.3f} token-equivalents)")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
           "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "decode TP SwiGLU MLP: T=64 (batch 64, s=1), d=8192, "
                                  "d_ff=28672, p=8 logical shards",
                      "global_batch": 64, "seq_len": 1, "parallelism": "host oracle"},
           "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": _threads(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra-steps", type=int, default=20)
    ap.add_argument("--extras", default="tiny,prefill,attention,stack,seqpar,moe",
                    help="comma list of extra workloads to measure at N=1")
    ap.add_argument("--reduce-mode", choices=["separate", "fused"], default="separate",
                    help="how the p partial sums are added in the decode workloads")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    run_ours(args, dist)


if __name__ == "__main__":
    main()
