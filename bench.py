"""Benchmark of the B200 Hymba hybrid-head mixer.

Headline step: one prefill of the 32-layer mixer stack (Hymba-1.5B layer shape,
d_model 1600, B=8 sequences of T=4096 user tokens + 128 meta tokens, layers 0, 15
and 31 global, the others sliding-window 1024, consecutive layer pairs sharing KV,
fp32 residual stream between the bf16 layers). Every layer runs the fused
projection with RoPE and K/V write, the Delta projection, meta+window GQA attention,
conv + selective scan, the fusion epilogue and the output projection with the
residual add.

Beside it, under extra keys: the global layer (B=4, T=8192 + 128 meta), the SWA
layer (B=1, T=2048 + 128 meta) and the decode step of the KV-sharing layer pair
(B=64, 1024-slot ring + 128 meta, fp32 state [64, 3200, 16]).

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

WORKLOAD = "hymba15_stack32_b8_t4096"
LAYER_WORKLOADS = ("hymba15_global_b4_t8192", "hymba15_swa1024_b1_t2048", "hymba15_ssd_swa1024_b8_t4096")
DECODE_WORKLOAD = "hymba15_decode_pair_b64_p4096"


MUFU_PER_CLK_SM = 16  # nominal exp2 / rcp results per clock per SM (4 per SM sub-partition)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    sm_mhz=d.get("sm_max_mhz", 1965.0), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_mhz=1965.0, src="fallback")


TRAFFIC_HEADERS = ("hybrid_head_ssm_b200/csrc/common.cuh", "hybrid_head_ssm_b200/csrc/tc.cuh",
                   "hybrid_head_ssm_b200/csrc/kernels.h", "hybrid_head_ssm_b200/csrc/epilogue.cuh",
                   "include/hymba.h")


def sources_sha1(sources):
    """sha1 over the kernel's source file and every header it includes."""
    h = hashlib.sha1()
    for rel in sources:
        h.update(rel.encode())
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()


def kernel_traffic(name, workload):
    """DRAM bytes per launch of a kernel from the committed ncu record (profiles/), or
    None when there is none for this workload or the kernel's source (its file and the
    headers it includes) changed since the counters were taken."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json"))).get(name)
        if not rec or rec.get("workload") != workload:
            return None
        if sources_sha1(rec["sources"]) != rec["sources_sha1"]:
            return None
        return rec["bytes_per_launch"]
    except (OSError, ValueError, KeyError):
        return None


def record_traffic(name, workload, source, bytes_per_launch, counters, summary):
    """Write the committed record of a kernel's measured DRAM traffic (ncu
    dram__bytes_read.sum + dram__bytes_write.sum per launch), keyed on its sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    recs = json.load(open(path)) if os.path.exists(path) else {}
    sources = [source] + list(TRAFFIC_HEADERS)
    recs[name] = {"bytes_per_launch": bytes_per_launch, "counters": counters, "workload": workload,
                  "summary": summary, "sources": sources, "sources_sha1": sources_sha1(sources)}
    json.dump(recs, open(path, "w"), indent=2)


def roofline_entry(name, bound, units, avg_s, pk, sm_count, sm_mhz, long_step=False):
    """Achieved rate of one kernel against the peak of its bound. A tensor-bound kernel
    is set against the burst bf16 peak when its launches are timed in a short step, and
    against the sustained one inside a long step (where the power cap sets the clock);
    both fractions are given."""
    if bound == "tensor":
        ach = units / avg_s / 1e12
        peak = pk["bf16_sus"] if long_step else pk["bf16"]
        kind = "sustained" if long_step else "burst"
        return {"kernel": name, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "frac_burst": ach / pk["bf16"], "frac_sustained": ach / pk["bf16_sus"],
                "peak_kind": f"bf16 dense, {kind}, {pk['src']}"}
    if bound == "alu":
        ach = units / avg_s / 1e9
        rate = pk.get("mufu_per_clk_sm") or MUFU_PER_CLK_SM
        src = "measured by hymba_probe_unit_rates" if pk.get("mufu_per_clk_sm") else "nominal"
        peak = rate * sm_count * sm_mhz * 1e-3
        return {"kernel": name, "bound": "alu", "achieved": ach, "peak": peak, "unit": "G MUFU op/s",
                "frac": ach / peak,
                "peak_kind": f"{rate:.2f} exp2 results per clock per SM ({src}) x {sm_count} SMs x {sm_mhz:.0f} MHz "
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


def layer_work(cfg, B, T, has_meta, io_f32):
    """Algorithmic work of each kernel launch of one prefill call, as {name: (bound,
    units)}: FLOPs for the projections and attention, MUFU results for the scan, bytes
    for the HBM-bound kernels."""
    m, Tp = cfg.n_meta, cfg.n_meta + T
    H, dh, dv, di, d, r = (cfg.n_q_heads, cfg.head_dim, cfg.v_head_dim, cfg.d_inner, cfg.d_model, cfg.dt_rank)
    rows = B * Tp
    # the in-projection computes the user rows and the meta rows once (or every row
    # when the input already carries the meta rows)
    in_rows = rows if has_meta else B * T + m
    pairs = visible_pairs(Tp, m, cfg.window)
    nh = getattr(cfg, "ssm_heads", 0)
    w = {
        "gemm_in_proj": ("tensor", 2.0 * in_rows * cfg.n_in * d),
        "gemm_dt_proj": ("tensor", 2.0 * rows * (nh if nh > 0 else di) * r),
        "attn_prefill": ("tensor", 2.0 * B * pairs * H * (dh + dv)),
    }
    if nh > 0:
        # SSD form: x read and y_pre written (2 B each per (row, channel)), B and C (64 B)
        # and the heads' Delta (4 B each) per row
        w["ssd_scan_prefill"] = ("hbm", rows * (4.0 * di + 64.0 + 4.0 * nh))
    else:
        # MUFU results: 16 state decays exp2(Delta A), and exp2 + reciprocal of the SiLU,
        # per (row, channel): the scan's binding limit
        w["conv_scan_prefill"] = ("alu", rows * di * 18.0)
    w.update({
        # O, y_pre, z read, U written: 2 B each per (row, channel)
        "fuse": ("hbm", rows * di * 8.0),
        "gemm_out_proj": ("tensor", 2.0 * rows * d * di),
    })
    if io_f32 and cfg.dtype == synth.BF16:
        # fp16 copies of the stream rows (fp32 read, fp16 written) and of W_in, W_out
        # and the meta rows (bf16 read, fp16 written)
        xrows = rows if has_meta else B * T
        w["pad_copy"] = ("hbm", xrows * d * 6.0 + (cfg.n_in * d + d * di + (0 if has_meta else m * d)) * 4.0)
    return w


def add_work(total, part):
    for n, (bound, u) in part.items():
        total[n] = (bound, total.get(n, (bound, 0.0))[1] + u)
    return total


def decode_work(cfg, B, cap):
    """Algorithmic HBM bytes per launch of the decode kernels (2-byte K/V, fp32 state)."""
    G, dh, dv, di, r = cfg.n_kv_heads, cfg.head_dim, cfg.v_head_dim, cfg.d_inner, cfg.dt_rank
    attn = B * G * cap * (dh + dv) * 2.0
    # h and conv state read + written (fp32), x read, y_pre written per (sequence,
    # channel); W_dt once and the dt_low rows for the folded Delta projection
    ssm = B * di * (16 * 4 * 2 + 4 * 4 * 2 + 2 + 2) + di * r * 2.0 + B * r * 2.0
    return {
        "attn_decode": ("hbm", attn),
        "ssm_decode": ("hbm", ssm),
        # 16-bit layers: both in one launch
        "attn_ssm_decode": ("hbm", attn + ssm),
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


def workload_config(name):
    wl = synth.workload(name)
    cfg = wl["cfg"]
    c = {"workload": name, "B": wl["B"], "T": wl["T"], "n_meta": cfg.n_meta, "d_model": cfg.d_model,
         "d_inner": cfg.d_inner, "n_q_heads": cfg.n_q_heads, "n_kv_heads": cfg.n_kv_heads,
         "window": cfg.window, "per_rank_batch": wl["B"]}
    if wl["kind"] == "stack":
        c["n_layers"] = wl["n_layers"]
        c["global_layers"] = list(wl["global_layers"])
        c["kv_sharing"] = "consecutive layer pairs (2i producer, 2i+1 consumer)"
        c["residual_stream"] = "fp32"
    return c


# ---------------------------------------------------------------------------
# the CPU oracle as a baseline
# ---------------------------------------------------------------------------
ORACLE_T = 512  # user tokens of the oracle's sample sequence


def _stack_cfgs_weights(layers):
    wl = synth.workload(WORKLOAD)
    cfgs = synth.stack_layer_cfgs(wl["cfg"], wl["n_layers"], wl["global_layers"])
    return wl, cfgs, {l: synth.layer_weights(cfgs[l], 1000 * wl["seed"] + l) for l in layers}


def _oracle_layers(cfgs, weights, layers, x, has_meta):
    import oracle
    h, kv = x, None
    for i, l in enumerate(layers):
        c = cfgs[l]
        r = oracle.mixer_prefill(c, weights[l], h, kv_shared=None if c.is_kv_producer else kv, residual=True,
                                 x_has_meta=has_meta or i > 0)
        if c.is_kv_producer:
            kv = (r["k"], r["v"])
        h = r["y"]
    return h


def oracle_stack_sample():
    """The oracle through all 32 layers of the stack on the first ORACLE_T user tokens of
    sequence 0 (weights drawn before the clock starts). Returns (tokens/s, seconds)."""
    wl, cfgs, weights = _stack_cfgs_weights(range(wl_layers()))
    x = synth.layer_input(cfgs[0], 1, wl["T"], wl["seed"])[:, :ORACLE_T]
    t0 = time.perf_counter()
    _oracle_layers(cfgs, weights, list(range(len(cfgs))), x, False)
    dt = time.perf_counter() - t0
    return ORACLE_T / dt, dt


def wl_layers():
    return synth.workload(WORKLOAD)["n_layers"]


def run_reference(args, rank):
    """The oracle as the reference arm: each step runs one KV-sharing layer pair of the
    stack (pairs taken in turn) on one sequence of ORACLE_T user tokens + 128 meta rows;
    tokens/s of the whole stack = ORACLE_T / (pair time x 16)."""
    if rank != 0:
        return
    n_layers = wl_layers()
    wl, cfgs, weights = _stack_cfgs_weights(range(n_layers))
    x = synth.layer_input(cfgs[0], 1, wl["T"], wl["seed"])[:, :ORACLE_T]
    g = np.random.default_rng([wl["seed"], 91])
    xm = (g.standard_normal((1, cfgs[0].n_meta + ORACLE_T, cfgs[0].d_model)) * 2.0).astype(np.float32)
    times = []
    for i in range(args.warmup + args.steps):
        pair = (i % (n_layers // 2)) * 2
        t0 = time.perf_counter()
        _oracle_layers(cfgs, weights, [pair, pair + 1], x if pair == 0 else xm, pair > 0)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    pair_s = statistics.mean(times)
    step_s = pair_s * n_layers / 2
    v = ORACLE_T / step_s
    sample = (f"one sequence of {ORACLE_T} user tokens + 128 meta rows through one KV-sharing layer pair per "
              f"step (the 16 pairs in turn), scaled to the 32-layer stack")
    print(json.dumps({
        "impl": "reference", "metric": "hybrid-head mixer stack prefill tokens/s", "value": v,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * step_s, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": workload_config(WORKLOAD),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ---------------------------------------------------------------------------
# device workloads
# ---------------------------------------------------------------------------
class PrefillWorkload:
    """A prefill workload on the device: one layer (bf16 input and output) or the
    32-layer stack (fp32 residual stream, KV shared by layer pairs, in place after the
    first layer). step(x, y) queues one pass over all its layers on the current stream."""

    def __init__(self, name, rank, torch, hy, rt, shrink=None):
        import ctypes
        self.name, self.torch, self.hy, self.rt = name, torch, hy, rt
        wl = synth.workload(name)
        if shrink:
            wl.update(shrink)  # a profiling-size case of the same workload
        self.wl = wl
        self.B, self.T = wl["B"], wl["T"]
        base = wl["cfg"]
        self.Tp = base.n_meta + self.T
        self.stack = wl["kind"] == "stack"
        if self.stack:
            self.cfgs = synth.stack_layer_cfgs(base, wl["n_layers"], wl["global_layers"])[:wl["n_layers"]]
            seeds = [1000 * wl["seed"] + l for l in range(len(self.cfgs))]
        else:
            self.cfgs, seeds = [base], [wl["seed"]]
        self.layers = [rt.DeviceLayer(c, synth.layer_weights(c, s)) for c, s in zip(self.cfgs, seeds)]
        io_f32 = self.stack
        x_np = synth.layer_input(base, self.B, self.T, rank_inputs_seed(wl["seed"], rank))
        self.x = rt.to_device(x_np, base, io_f32=io_f32)
        del x_np
        self.y = torch.empty((self.B, self.Tp, base.d_model), dtype=self.x.dtype, device="cuda")
        self.kv = rt.KV(base.with_(is_kv_producer=1), self.B, seq_cap=self.Tp)
        self.kvs = []
        for c, lay in zip(self.cfgs, self.layers):
            if c.is_kv_producer:
                self.kvs.append(self.kv.s)
            else:
                s = hy.hymba_kv()
                hy.check(hy.hymba_kv_share(ctypes.byref(self.kv.s), ctypes.byref(lay.c), ctypes.byref(s)))
                self.kvs.append(s)
        self.ws = rt.workspace(base.with_(is_kv_producer=1), self.B, self.T, hy.HYMBA_MODE_PREFILL)
        self.flags = rt.stream_flags(base) if self.stack else 0
        self.work = {}
        for i, c in enumerate(self.cfgs):
            add_work(self.work, layer_work(c, self.B, self.T, has_meta=i > 0, io_f32=io_f32))
        self.tokens = self.B * self.T

    def step(self, xin=None, yout=None):
        x = self.x if xin is None else xin
        y = self.y if yout is None else yout
        for i, (lay, kvs) in enumerate(zip(self.layers, self.kvs)):
            fl = self.flags | (self.hy.HYMBA_X_HAS_META if i > 0 else 0)
            self.rt.prefill(lay, x if i == 0 else y, self.T, None, y, self.ws, None, fl, kv_struct_override=kvs)


def time_prefill(wk, args, torch, hy, barrier, max_ranks, pk, flush, clocks, sm_count, headline):
    """Warm-up, a traced pass for the per-kernel breakdown, the timed steps (only the
    dominant kernel bracketed by events) and the end-to-end run with host buffers."""
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        wk.step()
    torch.cuda.synchronize()

    def run_steps(n, traced_only=None, timed=False):
        if traced_only is not False:
            hy.hymba_trace_enable(1)
            hy.check(hy.hymba_trace_only(traced_only.encode() if traced_only else None))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        barrier()
        torch.cuda.synchronize()
        if timed and clocks:
            clocks.begin()
        for i in range(n):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            wk.step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        if timed and clocks:
            clocks.end()
        barrier()
        trace = hy.trace_collect() if traced_only is not False else []
        hy.hymba_trace_enable(0)
        hy.check(hy.hymba_trace_only(None))
        return [a.elapsed_time(b) for a, b in ev], trace

    # per-kernel breakdown: every launch bracketed by events, outside the timed region
    # (events between launches serialise the overlap of consecutive kernels)
    n_traced = max(1, min(args.steps, 8192 // (12 * len(wk.layers))))
    _, trace_all = run_steps(n_traced, traced_only=None)
    per = {}
    for name, t in trace_all:
        per.setdefault(name, []).append(t)
    tot_k = max(sum(map(sum, per.values())), 1e-9)
    kern = {n: {"launches_per_step": len(v) / n_traced, "us_per_step": 1e3 * sum(v) / n_traced,
                "share": sum(v) / tot_k} for n, v in per.items()}
    dom = max(per, key=lambda n: sum(per[n]))

    # timed region: K steps, only the dominant kernel's launches bracketed by events
    launches0 = hy.hymba_launch_count()
    step_ms, trace_dom = run_steps(args.steps, traced_only=dom, timed=headline)
    launches = (hy.hymba_launch_count() - launches0) / args.steps
    ms = max_ranks(sum(step_ms) / len(step_ms))
    long_step = ms > 20.0
    sm_mhz = pk["sm_mhz"]
    if headline and clocks:
        clk = clocks.stop()
        if clk:
            sm_mhz = clk["sm_mhz"]
    else:
        clk = None
    dom_t = [t for n, t in trace_dom if n == dom]
    bound, units = wk.work.get(dom, ("hbm", 0.0))
    dom_s_per_step = sum(dom_t) / args.steps * 1e-3
    roof = roofline_entry(dom, bound, units, dom_s_per_step, pk, sm_count, sm_mhz, long_step)
    roof["launches_per_step"] = len(dom_t) / args.steps
    roof["units_per_step"] = units
    roof["traffic"] = kernel_traffic(dom, wk.name)
    if roof["traffic"] is not None:
        roof["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    for n, (bd, u) in wk.work.items():
        if n in per:
            r = roofline_entry(n, bd, u, sum(per[n]) / n_traced * 1e-3, pk, sm_count, sm_mhz, long_step)
            kern[n].update({k: r[k] for k in ("achieved", "unit", "frac", "peak_kind")})
            for k in ("frac_burst", "frac_sustained"):
                if k in r:
                    kern[n][k] = r[k]

    # end to end through the public API with host buffers: each step uploads its input
    # from pinned host memory, runs the workload and downloads the output; uploads,
    # compute and downloads go on three streams with two device buffer sets, so step
    # i+1's upload and step i-1's download overlap step i's compute. Timed with device
    # events from the first upload to the last download.
    x_host = wk.x.cpu().pin_memory()
    y_host = [torch.empty(wk.y.shape, dtype=wk.y.dtype).pin_memory() for _ in range(2)]
    xs, ys = [wk.x, torch.empty_like(wk.x)], [wk.y, torch.empty_like(wk.y)]
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
            wk.step(xs[k], ys[k])
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

    e2e_run(min(args.warmup, 3))
    e2e_ms = max_ranks(e2e_run(args.steps))
    del xs, ys, x_host, y_host
    return dict(ms=ms, launches=launches, roof=roof, kern=kern, clk=clk, e2e_ms=e2e_ms,
                h2d=wk.x.numel() * wk.x.element_size(), d2h=wk.y.numel() * wk.y.element_size())


def bench_decode(args, torch, hy, rt, max_ranks, barrier, world, pk, flush):
    """The decode step of the KV-sharing pair: timed without any tracing, then a traced
    pass for the per-kernel figures."""
    import ctypes
    wl = synth.workload(DECODE_WORKLOAD)
    ca = wl["cfg"]
    cb = ca.with_(is_kv_producer=0)
    B, T, seed = wl["B"], wl["T"], wl["seed"]
    if args.decode_prompt > 0:
        T = args.decode_prompt
    la = rt.DeviceLayer(ca, synth.layer_weights(ca, seed * 1000))
    lb = rt.DeviceLayer(cb, synth.layer_weights(cb, seed * 1000 + 1))
    cap = ca.n_meta + ca.window
    Tp = ca.n_meta + T
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
    stream = torch.cuda.current_stream()

    def step():
        rt.decode(la, xt, kv.s, sa, ha, wda, fl)
        rt.decode(lb, ha, kvb, sb, hb, wdb, fl)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
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
    ms = max_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps)
    # per-kernel figures from a separate traced pass
    hy.hymba_trace_enable(1)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step()
    trace = hy.trace_collect()
    hy.hymba_trace_enable(0)
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
    return {"workload": DECODE_WORKLOAD, "tokens_per_s": B * world / (ms * 1e-3), "ms_per_step": ms,
            "step_bytes": step_bytes, "step_gbs": step_bytes / (ms * 1e-3) / 1e9,
            "step_frac_hbm": step_bytes / (ms * 1e-3) / 1e9 / pk["hbm"],
            "timing": "timed steps untraced; per-kernel figures from a separate traced pass", "kernels": kern}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-dir", default="",
                    help="where the NVML clock samples are written (default: the system temp directory)")
    ap.add_argument("--no-extra", action="store_true", help="time only the headline workload")
    ap.add_argument("--only", default="", choices=["", "stack", "global", "swa", "ssd", "decode"],
                    help="run one workload alone and print its figures (for profiling runs)")
    ap.add_argument("--decode-prompt", type=int, default=0,
                    help="prompt length of the decode pair's prefill (default: the workload's 4096)")
    ap.add_argument("--small", action="store_true",
                    help="with --only: the profiling-size case of the workload (stack: 2 layers, T=1024; "
                         "global: B=1; decode: a 1100-token prompt), a few GB on the device at most")
    ap.add_argument("--record-traffic", nargs=6, metavar=("KERNEL", "WORKLOAD", "SOURCE", "BYTES", "COUNTERS",
                                                          "SUMMARY"),
                    help="write the DRAM traffic record of a kernel measured by ncu and exit")
    args = ap.parse_args()
    if args.record_traffic:
        k, wl, src, nb, counters, summary = args.record_traffic
        record_traffic(k, wl, src, int(nb), counters, summary)
        return None
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, rank)

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
    sm_count = torch.cuda.get_device_properties(local).multi_processor_count
    rates = hy.unit_rates()  # exp2 and FMA results per clock per SM, measured on this GPU
    pk["mufu_per_clk_sm"] = rates["ex2_f32"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # > 126 MB L2

    if args.only:
        # one workload alone, for profiling runs: no headline line
        if args.only == "decode":
            if args.small and args.decode_prompt <= 0:
                args.decode_prompt = 1100
            r = bench_decode(args, torch, hy, rt, max_ranks, barrier, world, pk, flush)
        else:
            name = {"stack": WORKLOAD, "global": LAYER_WORKLOADS[0], "swa": LAYER_WORKLOADS[1],
                    "ssd": LAYER_WORKLOADS[2]}[args.only]
            shrink = None
            if args.small:
                shrink = {"stack": dict(T=1024, n_layers=2), "global": dict(B=1), "swa": {},
                          "ssd": dict(T=1024)}[args.only]
            w1 = PrefillWorkload(name, rank, torch, hy, rt, shrink)
            r = time_prefill(w1, args, torch, hy, barrier, max_ranks, pk, flush, None, sm_count, headline=False)
            r = {"workload": name, "ms_per_step": r["ms"], "tokens_per_s": w1.tokens * world / (r["ms"] * 1e-3),
                 "kernels": r["kern"]}
        if rank == 0:
            print(json.dumps({"only": args.only, **r}))
        if world > 1:
            dist.destroy_process_group()
        return r

    clocks = Clocks(local, args.clocks_dir)
    clocks.start()
    wk = PrefillWorkload(WORKLOAD, rank, torch, hy, rt)
    head = time_prefill(wk, args, torch, hy, barrier, max_ranks, pk, flush, clocks, sm_count, headline=True)
    del wk
    torch.cuda.empty_cache()
    tokens = synth.workload(WORKLOAD)["B"] * synth.workload(WORKLOAD)["T"] * world

    extra = {}
    if not args.no_extra:
        for name in LAYER_WORKLOADS:
            w2 = PrefillWorkload(name, rank, torch, hy, rt)
            r = time_prefill(w2, args, torch, hy, barrier, max_ranks, pk, flush, None, sm_count, headline=False)
            extra[name] = {"tokens_per_s": w2.tokens * world / (r["ms"] * 1e-3), "ms_per_step": r["ms"],
                           "e2e_tokens_per_s": w2.tokens * world / (r["e2e_ms"] * 1e-3), "roofline": r["roof"],
                           "kernels": r["kern"], "gpu_launches_per_step": r["launches"]}
            del w2
            torch.cuda.empty_cache()
        extra[DECODE_WORKLOAD] = bench_decode(args, torch, hy, rt, max_ranks, barrier, world, pk, flush)

    out = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, dt = oracle_stack_sample()
            cpu = {"value": v, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                   "sample": f"sequence 0, first {ORACLE_T} user tokens + 128 meta rows through all "
                             f"{wl_layers()} layers, {dt:.1f} s"}
        out = {
            "metric": "hybrid-head mixer stack prefill tokens/s", "value": tokens / (head["ms"] * 1e-3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": head["ms"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(WORKLOAD),
                           l2="inputs larger than L2 (weights 1.3 GB, stream 216 MB); 256 MB written between steps"),
            "roofline": head["roof"],
            "cpu_baseline": cpu,
            "e2e": {"value": tokens / (head["e2e_ms"] * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": head["h2d"], "d2h_bytes_per_step": head["d2h"]},
            "gpu_launches": int(round(head["launches"] * args.steps)),
            "gpu_launches_per_step": head["launches"],
            "clocks": head["clk"],
            "unit_rates_per_clk_sm": rates,
            "kernels": head["kern"],
            "extra": extra,
        }
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()
    return out


if __name__ == "__main__":
    main()
