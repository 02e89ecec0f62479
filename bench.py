"""Benchmark of the B200 Hymba hybrid-head mixer.

One step = one hymba_mixer_prefill of the Hymba-1.5B-shaped SWA layer (B=1, T=2048
user tokens + 128 meta tokens, window 1024, bf16): the fused projection with RoPE
and K/V write, Delta projection, meta+window GQA attention, conv + selective scan,
fusion epilogue and output projection. The decode step of the KV-sharing layer pair
(B=64, 1024-slot ring + 128 meta, fp32 state [64, 3200, 16]) is timed the same way
and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own replica (weak scaling, no collective on the
data path); rank 0 prints one JSON line. --impl reference times the CPU oracle on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "hymba15_swa1024_b1_t2048"
DECODE_WORKLOAD = "hymba15_decode_pair_b64_p4096"


MUFU_PER_CLK_SM = 16  # exp2 / rcp results per clock per SM (4 per SM sub-partition)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    sm_mhz=d.get("sm_max_mhz", 1965.0), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_mhz=1965.0, src="fallback")


def kernel_traffic(name, workload):
    """DRAM bytes per launch of a kernel from the committed ncu record (profiles/), or
    None when there is none for this workload or the kernel's device code changed since
    (the record hashes the source file up to the kernel's host launcher)."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json"))).get(name)
        if not rec or rec.get("workload") != workload:
            return None
        src = open(os.path.join(ROOT, rec["kernel_source"]), "rb").read()
        end = src.find(rec["device_code_until"].encode())
        if end < 0 or hashlib.sha1(src[:end]).hexdigest() != rec["device_code_sha1"]:
            return None
        return rec["bytes_per_launch"]
    except (OSError, ValueError, KeyError):
        return None


def roofline_entry(name, bound, units, avg_s, pk, sm_count, sm_mhz):
    """Achieved rate of one kernel against the peak of its bound."""
    if bound == "tensor":
        ach = units / avg_s / 1e12
        return {"kernel": name, "bound": "tensor", "achieved": ach, "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                "frac": ach / pk["bf16_sus"], "peak_kind": f"bf16 dense, sustained, {pk['src']}"}
    if bound == "alu":
        ach = units / avg_s / 1e9
        peak = MUFU_PER_CLK_SM * sm_count * sm_mhz * 1e-3
        return {"kernel": name, "bound": "alu", "achieved": ach, "peak": peak, "unit": "G MUFU op/s",
                "frac": ach / peak,
                "peak_kind": f"{MUFU_PER_CLK_SM} MUFU results per clock per SM x {sm_count} SMs x {sm_mhz:.0f} MHz "
                             "(SM clock sampled in the timed region)"}
    ach = units / avg_s / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": ach, "peak": pk["hbm"], "unit": "GB/s",
            "frac": ach / pk["hbm"], "peak_kind": f"HBM copy, {pk['src']}"}


CLOCK_SAMPLER = r"""
import sys, time
import pynvml as nv
nv.nvmlInit()
bus, index, path, stop = sys.argv[1], int(sys.argv[2]), sys.argv[3], sys.argv[4]
try:
    h = nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
except Exception:
    h = nv.nvmlDeviceGetHandleByIndex(index)
import os
with open(path, "w", buffering=1) as f:
    f.write("time,sm_mhz,sm_max_mhz,reasons_mask\n")
    mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
    n = 0
    while True:
        f.write(f"{time.time():.6f},{nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)},{mx},"
                f"{nv.nvmlDeviceGetCurrentClocksEventReasons(h)}\n")
        n += 1
        if n % 64 == 0 and os.path.exists(stop):
            break
        time.sleep(0.0005)
"""


class Clocks:
    """SM clocks and clock-event (throttle) reasons through NVML (read-only queries; no
    setting is touched), polled about every millisecond by a separate process so that
    the polling does not compete with this one; only the samples taken while the timed
    region is open (wall clock) are reported. The samples go to
    <clocks_dir>/clocks_rank<i>.csv (`--clocks-dir`, default the system temp directory)."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, cuda_index: int, clocks_dir: str = ""):
        self.cuda_index = cuda_index
        self.path = os.path.join(clocks_dir or tempfile.gettempdir(), f"clocks_rank{cuda_index}.csv")
        self.stop_path = self.path + ".stop"
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            import pynvml  # noqa: F401
            import torch
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            if os.path.exists(self.stop_path):
                os.remove(self.stop_path)
            pr = torch.cuda.get_device_properties(self.cuda_index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.err = open(self.path + ".err", "w")
            self.proc = subprocess.Popen([sys.executable, "-c", CLOCK_SAMPLER, bus, str(self.cuda_index), self.path,
                                          self.stop_path], stdout=subprocess.DEVNULL, stderr=self.err)
            # wait for the first samples so that the timed region is covered
            for _ in range(400):
                if os.path.exists(self.path) and sum(1 for _ in open(self.path)) > 3:
                    break
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.01)
        open(self.stop_path, "w").close()
        try:
            self.proc.wait(timeout=10)
        except Exception:
            self.proc.kill()
        os.remove(self.stop_path)
        rows = []
        for line in open(self.path).read().splitlines()[1:]:
            try:
                t, sm, mx, rs = line.split(",")
                rows.append((float(t), float(sm), float(mx), int(rs)))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1]
        source = "NVML, separate process polling about every 1 ms, timed region only"
        if not inside and rows and self.t0 is not None:
            # region shorter than the polling interval: the samples just before and after it
            before = [r for r in rows if r[0] < self.t0][-1:]
            after = [r for r in rows if r[0] > self.t1][:1]
            inside = before + after
            source = "NVML, the samples adjacent to a timed region shorter than the polling interval"
        if not inside:
            return None
        reasons = sorted({n for r in inside for n, m in self.REASONS if r[3] & m})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "source": source}


def visible_pairs(Tp, m, W):
    i = np.arange(Tp)[:, None]
    j = np.arange(Tp)[None, :]
    vis = (j <= i) & ((j < m) | (i - j < W) if W > 0 else True)
    return int(vis.sum())


def prefill_work(cfg, B, T):
    """Algorithmic FLOPs / bytes per launch of each prefill kernel."""
    m, Tp = cfg.n_meta, cfg.n_meta + T
    H, G, dh, dv, di, d, r = (cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim,
                              cfg.d_inner, cfg.d_model, cfg.dt_rank)
    rows = B * Tp
    pairs = visible_pairs(Tp, m, cfg.window)
    return {
        "gemm_in_proj": ("tensor", 2.0 * B * T * cfg.n_in * d),
        "gemm_in_proj_meta": ("tensor", 2.0 * m * cfg.n_in * d),
        "gemm_dt_proj": ("tensor", 2.0 * rows * di * r),
        "attn_prefill": ("tensor", 2.0 * B * pairs * H * (dh + dv)),
        "attn_prefill_simt": ("tensor", 2.0 * B * pairs * H * (dh + dv)),
        # MUFU operations: 16 state decays exp2(Delta A), and exp2 + reciprocal of the SiLU,
        # per (row, channel); the kernel's binding limit (its 56 MB of HBM traffic take
        # 8.5 us at the measured copy rate, the MUFU work 27 us)
        "conv_scan_prefill": ("alu", rows * di * 18.0),
        # O, y_pre, z read, U written: 2 B each per (row, channel)
        "fuse": ("hbm", rows * di * 8.0),
        "gemm_out_proj": ("tensor", 2.0 * rows * d * di),
    }


def decode_work(cfg, B, cap):
    """Algorithmic HBM bytes per launch of the decode kernels (2-byte K/V, fp32 state)."""
    G, dh, dv, di, r = cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim, cfg.d_inner, cfg.dt_rank
    return {
        "attn_decode": ("hbm", B * G * cap * (dh + dv) * 2.0),
        # h and conv state read + written (fp32), x read, y_pre written per (sequence,
        # channel); W_dt once and the dt_low rows for the folded Delta projection
        "ssm_decode": ("hbm", B * di * (16 * 4 * 2 + 4 * 4 * 2 + 2 + 2) + di * r * 2.0 + B * r * 2.0),
        "gemm_in_proj_decode": ("hbm", cfg.n_in * cfg.d_model * 2.0),
        "gemm_out_proj_decode": ("hbm", cfg.d_model * di * 2.0),
    }


def rank_inputs_seed(seed: int, rank: int) -> int:
    """Weak scaling: every rank runs its own sequences, drawn from its own stream."""
    return seed + rank


def max_over_ranks(value: float, world: int, device: str) -> float:
    """The slowest rank's time (every rank calls this collectively)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(T_sample: int):
    """Time the CPU oracle on the first T_sample tokens of the workload's sequence."""
    import oracle
    wl = synth.workload(WORKLOAD)
    cfg = wl["cfg"]
    w = synth.layer_weights(cfg, wl["seed"])
    x = synth.layer_input(cfg, wl["B"], wl["T"], wl["seed"])[:, :T_sample]
    t0 = time.perf_counter()
    oracle.mixer_prefill(cfg, w, x)
    dt = time.perf_counter() - t0
    return x.shape[0] * x.shape[1] / dt, dt


def run_reference(args, rank):
    if rank != 0:
        return
    T_sample = 512
    vals = []
    for i in range(args.warmup + args.steps):
        v, _ = oracle_sample(T_sample)
        if i >= args.warmup:
            vals.append(v)
    v = statistics.median(vals)
    wl = synth.workload(WORKLOAD)
    sample = f"first {T_sample} of {wl['T']} user tokens of the B=1 sequence (+128 meta rows)"
    print(json.dumps({
        "impl": "reference", "metric": "hybrid-head mixer prefill tokens/s", "value": v,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * T_sample / v, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": wl["B"], "T": wl["T"], "n_meta": 128, "window": 1024},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-dir", default="",
                    help="where the NVML clock samples are written (default: the system temp directory)")
    ap.add_argument("--no-decode", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, rank)

    import ctypes
    import torch
    import torch.distributed as dist
    import hybrid_head_ssm_b200 as hy
    from hybrid_head_ssm_b200 import runtime as rt

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ranks(v):
        return max_over_ranks(v, world, "cuda")

    pk = peaks()
    wl = synth.workload(WORKLOAD)
    cfg, B, T = wl["cfg"], wl["B"], wl["T"]
    Tp = cfg.n_meta + T
    w = synth.layer_weights(cfg, wl["seed"])
    x_np = synth.layer_input(cfg, B, T, rank_inputs_seed(wl["seed"], rank))
    layer = rt.DeviceLayer(cfg, w)
    x = rt.to_device(x_np, cfg)
    y = torch.empty((B, Tp, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    kv = rt.KV(cfg, B, seq_cap=Tp)
    ws = rt.workspace(cfg, B, T, hy.HYMBA_MODE_PREFILL)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # > 126 MB L2
    stream = torch.cuda.current_stream()

    def step(xin=None, yout=None):
        rt.prefill(layer, x if xin is None else xin, T, kv, y if yout is None else yout, ws, None, 0)

    clocks = Clocks(local, args.clocks_dir)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    work = prefill_work(cfg, B, T)

    def run_steps(n, traced_only=None, timed=False):
        """n steps, L2 flushed before each (outside the step events); returns the step
        times (ms) and the trace records."""
        if traced_only is not False:
            hy.hymba_trace_enable(1)
            hy.check(hy.hymba_trace_only(traced_only.encode() if traced_only else None))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        barrier()
        torch.cuda.synchronize()
        if timed:
            clocks.begin()
        for i in range(n):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        if timed:
            clocks.end()
        barrier()
        trace = hy.trace_collect() if traced_only is not False else []
        hy.hymba_trace_enable(0)
        hy.check(hy.hymba_trace_only(None))
        return [a.elapsed_time(b) for a, b in ev], trace

    # ---- per-kernel breakdown (every launch bracketed by events; outside the timed region,
    # since events between launches serialise the overlap of consecutive kernels)
    _, trace_all = run_steps(args.steps, traced_only=None)
    per = {}
    for name, t in trace_all:
        per.setdefault(name, []).append(t)
    tot_k = max(sum(map(sum, per.values())), 1e-9)
    kern = {n: {"launches": len(v), "avg_us": 1e3 * sum(v) / len(v), "share": sum(v) / tot_k} for n, v in per.items()}
    dom = max(per, key=lambda n: sum(per[n]))

    # ---- timed region: K steps; only the dominant kernel is bracketed by events
    launches0 = hy.hymba_launch_count()
    step_ms, trace_dom = run_steps(args.steps, traced_only=dom, timed=True)
    launches = hy.hymba_launch_count() - launches0
    clk = clocks.stop()
    ms = max_ranks(sum(step_ms) / len(step_ms))
    tokens = B * T * world
    value = tokens / (ms * 1e-3)

    sm_count = torch.cuda.get_device_properties(local).multi_processor_count
    sm_mhz = clk["sm_mhz"] if clk else pk["sm_mhz"]
    dom_t = [t for n, t in trace_dom if n == dom]
    bound, units = work.get(dom, ("hbm", 0.0))
    roof = roofline_entry(dom, bound, units, sum(dom_t) / len(dom_t) * 1e-3, pk, sm_count, sm_mhz)
    roof["launches_timed"] = len(dom_t)
    roof["traffic"] = kernel_traffic(dom, WORKLOAD)
    if roof["traffic"] is not None:
        roof["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    for n, (bd, u) in work.items():
        if n in per:
            r = roofline_entry(n, bd, u, sum(per[n]) / len(per[n]) * 1e-3, pk, sm_count, sm_mhz)
            kern[n]["achieved"], kern[n]["unit"], kern[n]["frac"] = r["achieved"], r["unit"], r["frac"]

    # ---- end to end through the public API with host buffers: each step uploads its
    # input from pinned host memory, runs the layer and downloads the output; uploads,
    # compute and downloads go on three streams with two device buffer sets, so step
    # i+1's upload and step i-1's download overlap step i's compute. Timed with device
    # events from the first upload to the last download.
    x_host = x.cpu().pin_memory()
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    xs, ys = [x, torch.empty_like(x)], [y, torch.empty_like(y)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        t_start, t_end = ev(), ev()
        uploaded = [torch.cuda.Event(), torch.cuda.Event()]
        computed = [torch.cuda.Event(), torch.cuda.Event()]
        downloaded = [torch.cuda.Event(), torch.cuda.Event()]
        used = [False, False]
        torch.cuda.synchronize()
        t_start.record(up)
        for i in range(n):
            k = i & 1
            with torch.cuda.stream(up):
                if used[k]:
                    up.wait_event(computed[k])  # the compute of step i-2 has read xs[k]
                xs[k].copy_(x_host, non_blocking=True)
                uploaded[k].record(up)
            stream.wait_event(uploaded[k])
            if used[k]:
                stream.wait_event(downloaded[k])  # ys[k] of step i-2 is on the host
            step(xs[k], ys[k])
            computed[k].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[k])
                y_host[k].copy_(ys[k], non_blocking=True)
                downloaded[k].record(down)
            used[k] = True
        down.wait_event(computed[(n - 1) & 1])
        t_end.record(down)
        torch.cuda.synchronize()
        return t_start.elapsed_time(t_end) / n

    e2e_run(args.warmup)
    e2e_ms_step = max_ranks(e2e_run(args.steps))

    # ---- decode step of the KV-sharing pair (B=64, ring 1024 + 128 meta)
    dec = None
    if not args.no_decode:
        dec = bench_decode(args, torch, hy, rt, max_ranks, barrier, world, pk, flush)

    out = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, dt = oracle_sample(T)
            cpu = {"value": v, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                   "sample": f"one full sequence of the workload (B=1, T={T} + 128 meta), {dt:.1f} s"}
        out = {
            "metric": "hybrid-head mixer prefill tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "T": T, "n_meta": cfg.n_meta, "window": cfg.window,
                       "d_model": cfg.d_model, "d_inner": cfg.d_inner, "per_rank_batch": B,
                       "l2": "flushed between steps (256 MB write outside the step events)"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": tokens / (e2e_ms_step * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size()},
            "gpu_launches": int(launches),
            "clocks": clk,
            "kernels": kern,
            "decode": dec,
        }
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()
    return out


def bench_decode(args, torch, hy, rt, max_over_ranks, barrier, world, pk, flush):
    wl = synth.workload(DECODE_WORKLOAD)
    ca = wl["cfg"]
    cb = ca.with_(is_kv_producer=0)
    B, T, seed = wl["B"], wl["T"], wl["seed"]
    la = rt.DeviceLayer(ca, synth.layer_weights(ca, seed * 1000))
    lb = rt.DeviceLayer(cb, synth.layer_weights(cb, seed * 1000 + 1))
    cap = ca.n_meta + ca.window
    Tp = ca.n_meta + T
    import ctypes
    kv = rt.KV(ca, B, seq_cap=Tp, cache_cap=cap)
    kvb = hy.hymba_kv()
    hy.check(hy.hymba_kv_share(ctypes.byref(kv.s), ctypes.byref(lb.c), ctypes.byref(kvb)))
    sa, sb = rt.State(ca, B), rt.State(cb, B)
    fl = rt.stream_flags(ca)  # fp32 residual stream between the two bf16 layers
    x = rt.to_device(synth.layer_input(ca, B, T, seed), ca, io_f32=True)
    ya = torch.empty((B, Tp, ca.d_model), dtype=torch.float32, device="cuda")
    yb = torch.empty_like(ya)
    wsp = rt.workspace(ca, B, T, hy.HYMBA_MODE_PREFILL)
    rt.prefill(la, x, T, kv, ya, wsp, sa, fl)
    rt.prefill(lb, ya, T, kv, yb, wsp, sb, hy.HYMBA_X_HAS_META | fl, kv_struct_override=kvb)
    del wsp, ya, yb
    xt = rt.to_device(synth.layer_input(ca, B, 1, seed, tag=1)[:, 0], ca, io_f32=True)
    ha, hb = torch.empty_like(xt), torch.empty_like(xt)
    wda = rt.workspace(ca, B, cap, hy.HYMBA_MODE_DECODE)
    wdb = rt.workspace(cb, B, cap, hy.HYMBA_MODE_DECODE)
    len0 = kv.len.clone()
    stream = torch.cuda.current_stream()

    def step():
        rt.decode(la, xt, kv.s, sa, ha, wda, fl)
        rt.decode(lb, ha, kvb, sb, hb, wdb, fl)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    hy.hymba_trace_enable(1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    trace = hy.trace_collect()
    hy.hymba_trace_enable(0)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps)
    per = {}
    for name, t in trace:
        per.setdefault(name, []).append(t)
    work = decode_work(ca, B, cap)
    kern = {}
    for n, v in per.items():
        kern[n] = {"launches": len(v), "avg_us": 1e3 * sum(v) / len(v)}
        if n in work:
            a = sum(v) / len(v) * 1e-3
            kern[n]["achieved_gbs"] = work[n][1] / a / 1e9
            kern[n]["frac_hbm"] = kern[n]["achieved_gbs"] / pk["hbm"]
    # the whole step's algorithmic bytes: both layers' weights, the shared KV read
    # twice, state read+write twice
    step_bytes = (2 * decode_work(ca, B, cap)["attn_decode"][1]
                  + (ca.n_in + cb.n_in) * ca.d_model * 2.0 + 2 * ca.d_model * ca.d_inner * 2.0
                  + 2 * decode_work(ca, B, cap)["ssm_decode"][1])
    assert kv.len[0].item() >= len0[0].item()
    return {"workload": DECODE_WORKLOAD, "tokens_per_s": B * world / (ms * 1e-3), "ms_per_step": ms,
            "step_bytes": step_bytes, "step_gbs": step_bytes / (ms * 1e-3) / 1e9,
            "step_frac_hbm": step_bytes / (ms * 1e-3) / 1e9 / pk["hbm"], "kernels": kern}


if __name__ == "__main__":
    main()
