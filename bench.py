"""Benchmark of the routed-MoE layer (route + expert FFNs + combine) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = moe_route + moe_forward over one batch of synthetic tokens (every hot-path
step).  The default workload is the 1-token decode layer (hidden 7168, 256 routed
experts, top-8, one shared 3-bit expert, 2-bit routed experts), a fresh token per
step.  Device time comes from CUDA events on the launching stream; the L2 cache is
flushed (a 512 MiB write) between timed steps, outside the events, so every step
reads its experts from HBM.  For N > 1 (torchrun) each rank runs an independent
replica on its own token stream (the layer is data-parallel: no collective on the
data path) and the time is the max over ranks.

The roofline object describes the dominant launch.  On the decode path the library
runs the whole forward as one kernel (ffn_fused_kernel) for 5 to 8 tokens: against the
measured HBM copy bandwidth, with algorithmic bytes = the packed gate/up and down bytes
of every selected expert and the shared expert, each read once.  At other decode token
counts (the default workload's one token among them) it runs separate gate/up, down
and combine launches: the gate/up launch against the same peak (its packed gate/up
bytes).  For the tensor-core prefill path, the gate/up launch against the measured
burst bf16 GEMM rate (algorithmic FLOPs = 2 x routed rows x 2*ffn x hidden; the fp16
operands run at the bf16 rate).

--impl reference times the CPU oracle (the only reference that exists for this
layer) on the same workload, a bounded sample per step, on the host cores.
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

METRIC = "routed-MoE layer tokens/s; decode weight-stream GB/s vs HBM peak (1 B200)"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# gate/up kernel of each path and the sources its ncu traffic record is tied to
PATHS = {
    "fused": ("ffn_fused_kernel (the whole decode forward: gate/up + SwiGLU, down and the combine, one "
              "persistent launch; integer MMAs for ternary / 2-bit experts)",
              ["bit_routed_expert_fp32_b200/csrc/decode_fused.cu", "bit_routed_expert_fp32_b200/csrc/dequant.cuh",
               "bit_routed_expert_fp32_b200/csrc/operands.cuh", "bit_routed_expert_fp32_b200/csrc/iqmma.cuh",
               "bit_routed_expert_fp32_b200/csrc/common.cuh"]),
    "decode": ("ffn_decode_kernel<0> (gate/up + SwiGLU; interval includes the K-part reduction when K is "
               "split)",
               ["bit_routed_expert_fp32_b200/csrc/decode_ffn.cu", "bit_routed_expert_fp32_b200/csrc/dequant.cuh",
                "bit_routed_expert_fp32_b200/csrc/iqmma.cuh", "bit_routed_expert_fp32_b200/csrc/operands.cuh",
                "bit_routed_expert_fp32_b200/csrc/common.cuh"]),
    "prefill": ("tc_gemm_kernel<0> (gate/up + SwiGLU, tcgen05; interval includes the token gather)",
                ["bit_routed_expert_fp32_b200/csrc/prefill_tc.cu", "bit_routed_expert_fp32_b200/csrc/common.cuh"]),
}


def forward_plan(cfg) -> dict:
    """The library's own plan for moe_route + moe_forward(MOE_PATH_AUTO) on this workload
    (moe_forward_plan, host-only): which kernels run, how many launches, the K parts."""
    import bit_routed_expert_fp32_b200 as moe
    return moe.moe_forward_plan(cfg, cfg.T, moe.PATH_AUTO)


def path_of(cfg) -> str:
    """The kernels moe_forward(MOE_PATH_AUTO) runs for this workload: "decode" (separate
    launches), "fused" (the fused decode kernel) or "prefill"."""
    return forward_plan(cfg)["path"]


def decode_kparts(cfg):
    """K parts of the separate decode gate/up and down passes (1, 1 on the other paths)."""
    p = forward_plan(cfg)
    return p["kparts_gu"], p["kparts_dn"]


def launches_per_step(cfg) -> int:
    """Kernels one step (moe_route + moe_forward) launches."""
    return forward_plan(cfg)["launches"]


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of x over all ranks (x itself for one rank)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's device time."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), for the CPU baseline's record."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


def kernel_hash(path: str) -> str:
    h = hashlib.sha256()
    for f in PATHS[path][1]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_record(cfg_name: str, path: str):
    """DRAM bytes per launch of the gate/up kernel from the committed ncu summary, if
    it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(cfg_name)
    if not rec or rec.get("kernel_hash") != kernel_hash(path):
        return None
    return rec


def gu_bytes(cfg, fmt: int) -> int:
    """Packed bytes of one expert's fused gate/up matrix (codes + scales [+ third bits])."""
    K, rows = cfg.H, 2 * cfg.I
    b = rows * (K // 4 + 16 * ((K // 64 + 7) // 8))
    if fmt == synth.FMT_Q3:
        b += rows * 4 * 4 * ((K + 127) // 128)
    return b


def dn_bytes(cfg, fmt: int) -> int:
    K, rows = cfg.I, cfg.H
    b = rows * (K // 4 + 16 * ((K // 64 + 7) // 8))
    if fmt == synth.FMT_Q3:
        b += rows * 4 * 4 * ((K + 127) // 128)
    return b


class Clocks:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# --------------------------------------------------------------------------- oracle
def _expert_cache(cfg, layer, xs, threads):
    """Interchange-form weights of every expert the token batches touch (drawn before
    timing: drawing inputs is not oracle work)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    need = set(range(cfg.E, cfg.E + cfg.S))
    for x in xs:
        _, ids, _ = oracle.route(x, layer.router_w, layer.router_b, cfg.k, threads)
        need.update(int(e) for e in np.unique(ids))
    with ThreadPoolExecutor(threads) as ex:
        mats = list(ex.map(layer.expert, sorted(need)))
    return dict(zip(sorted(need), mats))


def oracle_tokens_per_s(cfg, layer, xs, budget_s: float, max_tokens: int, cache=None):
    """Times the CPU oracle (routing + experts + combine) on whole token batches until
    budget_s has elapsed (at least one batch); returns (tokens/s, tokens, seconds,
    threads used).  Each call into the oracle is single-threaded; independent
    experts run concurrently on the host cores."""
    import oracle
    threads = os.cpu_count() or 1
    if cache is None:
        cache = _expert_cache(cfg, layer, xs, threads)
    done, i, t0 = 0, 0, time.perf_counter()
    used = 1
    while True:
        x = xs[i % len(xs)]
        L = oracle.logits(x, layer.router_w, threads)
        ids, gates = oracle.select(L, layer.router_b, cfg.k)
        oracle.forward_tokens(layer, x, ids, gates, range(x.shape[0]), threads, expert_cache=cache)
        used = max(used, min(threads, len(np.unique(ids)) + cfg.S))
        done += x.shape[0]
        i += 1
        if done >= max_tokens or time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt, used


def run_reference(args, cfg):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    layer = synth.Layer(cfg, 0)
    per_step = max(1, min(cfg.T, 4))           # bounded sample of tokens per step
    xs = [synth.tokens(cfg, 0, s, per_step) for s in range(args.warmup + args.steps)]
    cache = _expert_cache(cfg, layer, xs, os.cpu_count() or 1)
    for s in range(args.warmup):
        oracle_tokens_per_s(cfg, layer, [xs[s]], 0.0, per_step, cache)
    t0 = time.perf_counter()
    tok, threads = 0, 1
    for s in range(args.steps):
        _, n, _, used = oracle_tokens_per_s(cfg, layer, [xs[args.warmup + s]], 0.0, per_step, cache)
        tok += n
        threads = max(threads, used)
    dt = time.perf_counter() - t0
    value = tok / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "cpu": cpu_model(),
                             "kind": "oracle", "sample": f"{per_step} token(s) of the workload per step, routed and run through "
                                       f"all selected experts and the shared expert in fp64 (expert weights "
                                       f"drawn before timing)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_dict(cfg, world, launch=None):
    d = {"workload": cfg.name, "tokens_per_step": cfg.T, "hidden": cfg.H, "experts": cfg.E, "top_k": cfg.k,
         "ffn": cfg.I, "shared": cfg.S, "formats": cfg.formats, "layers": cfg.layers,
         "l2": "flushed between timed steps (512 MiB write)", "parallelism": f"replicas x{world}"}
    if launch:
        d["launch"] = launch
    return d


# --------------------------------------------------------------------------- ours
def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    import bit_routed_expert_fp32_b200 as moe

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    T = cfg.T
    n_layers = cfg.layers
    layers, fmts = [], []
    for li in range(n_layers):
        L = synth.Layer(cfg, li)
        buf = np.zeros(moe.moe_packed_size(cfg, L.fmt), dtype=np.uint8)
        from concurrent.futures import ThreadPoolExecutor

        def job(e, L=L, buf=buf):
            moe.moe_pack_experts(cfg, L.fmt, e, [L.expert(e)], buf)

        with ThreadPoolExecutor(os.cpu_count() or 1) as ex:
            list(ex.map(job, range(cfg.E + cfg.S)))
        layers.append(moe.MoeLayer(cfg, buf, L.router_w, L.router_b, T, device=dev))
        fmts.append(L.fmt)
        del buf
    total = args.warmup + args.steps
    # fresh tokens per step; each rank draws its own stream (seeded by rank)
    xs_host = np.stack([synth.tokens(cfg, 0, 1000 * rank + s, T) for s in range(total)])
    x_dev = moe.bf16_to_device(xs_host.reshape(total * T, cfg.H), dev).view(total, T, cfg.H)
    y = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    ids_log = torch.empty((total, T, cfg.k), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(total)]      # step pass
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(total)]     # kernel pass
    for row in ev + evk:         # torch creates the CUDA event on first record: do it here so
        for e in row:            # the handles handed to the library are real events
            e.record(stream)
    torch.cuda.synchronize(dev)

    def step(s, record=None, per_kernel=False):
        """One layer step; record = the step's 6 events (0 and 5 bracket the step; 1-4
        go between the kernels when per_kernel, which serialises the launches)."""
        st = torch.cuda.current_stream(dev)          # the capture stream while capturing
        lay = layers[s % n_layers]
        if record is not None:
            moe.moe_event_record(record[0], st)
        lay.route(x_dev[s], stream=st)
        lay.forward(x_dev[s], y, events=record[1:5] if (record is not None and per_kernel) else None, stream=st)
        if record is not None:
            moe.moe_event_record(record[5], st)
            ids_log[s].copy_(lay.rt["topk_ids"][:T])

    # Each step (route + forward) is captured as one CUDA graph and replayed.  The
    # kernels are launched with programmatic dependent launch, so a kernel's launch
    # overlaps its predecessor's tail; the timed pass records events only around the
    # whole step.  A second pass over the same steps (same flushes) puts an event
    # between the kernels, which serialises them, to give the per-kernel times and the
    # gate/up launch duration for the roofline.  --no-graph launches eagerly instead.
    graphs = gk = None
    if not args.no_graph:
        for s in range(min(2, total)):              # first-call set-up happens outside capture
            step(s)
        torch.cuda.synchronize(dev)
        graphs, gk = [], []
        for s in range(total):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(s, ev[s])
            graphs.append(g)
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                step(s, evk[s], per_kernel=True)
            gk.append(g2)
        torch.cuda.synchronize(dev)

    def run(s, per_kernel=False):
        if graphs is not None:
            (gk if per_kernel else graphs)[s].replay()
        else:
            step(s, evk[s] if per_kernel else ev[s], per_kernel)

    for s in range(args.warmup):
        flush.zero_()
        run(s)
    torch.cuda.synchronize(dev)
    # clocks are sampled (every 100 ms) over a soak of the same steps that runs right
    # before the timed region and over the timed region itself
    clocks = Clocks(local)
    clocks.start()
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak_s:
        for s in range(args.warmup):
            flush.zero_()
            run(s)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.perf_counter()
    for s in range(args.warmup, total):
        flush.zero_()
        run(s)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    # per-kernel pass (not part of the headline number)
    for s in range(args.warmup, total):
        flush.zero_()
        run(s, per_kernel=True)
    torch.cuda.synchronize(dev)
    ck = clocks.stop()
    if ck is not None:
        ck["sampled_over"] = f"{args.soak_s:.1f} s soak of the same steps + the timed region"
    step_ms = [ev[s][0].elapsed_time(ev[s][5]) for s in range(args.warmup, total)]
    gu_ms = [evk[s][1].elapsed_time(evk[s][2]) for s in range(args.warmup, total)]
    dn_ms = [evk[s][2].elapsed_time(evk[s][3]) for s in range(args.warmup, total)]
    cb_ms = [evk[s][3].elapsed_time(evk[s][4]) for s in range(args.warmup, total)]
    rt_ms = [evk[s][0].elapsed_time(evk[s][1]) for s in range(args.warmup, total)]
    step_serial_ms = [evk[s][0].elapsed_time(evk[s][5]) for s in range(args.warmup, total)]
    my_ms = float(sum(step_ms))
    max_ms = max_over_ranks(my_ms, world, dev)
    value = throughput(world, T, args.steps, max_ms)

    # algorithmic bytes of the gate/up launches from the routing each step produced
    ids_h = ids_log.cpu().numpy()
    gu_alg, dn_alg = [], []
    for s in range(args.warmup, total):
        f = fmts[s % n_layers]
        distinct = np.unique(ids_h[s])
        gb = sum(gu_bytes(cfg, int(f[e])) for e in distinct) + sum(gu_bytes(cfg, int(f[cfg.E + j]))
                                                                   for j in range(cfg.S))
        db = sum(dn_bytes(cfg, int(f[e])) for e in distinct) + sum(dn_bytes(cfg, int(f[cfg.E + j]))
                                                                   for j in range(cfg.S))
        gu_alg.append(gb)
        dn_alg.append(db)
    pk, pk_kind = peaks()
    gu_gbs = (sum(gu_alg) / 1e9) / (sum(gu_ms) / 1e3)
    dn_gbs = (sum(dn_alg) / 1e9) / (sum(dn_ms) / 1e3)
    layer_gbs = ((sum(gu_alg) + sum(dn_alg)) / 1e9) / (my_ms / 1e3)
    path = path_of(cfg)
    tr = traffic_record(cfg.name, path)
    traffic = None if tr is None else tr["dram_bytes_per_launch"]
    if path == "fused":
        fused_alg = [a + b for a, b in zip(gu_alg, dn_alg)]
        fused_gbs = (sum(fused_alg) / 1e9) / (sum(gu_ms) / 1e3)
        roofline = {"bound": "hbm", "kernel": PATHS[path][0], "achieved": fused_gbs, "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": fused_gbs / pk["hbm_gbs"], "traffic": traffic,
                    "algorithmic_bytes_per_launch": float(np.mean(fused_alg)),
                    "peak_source": f"{pk_kind} hbm_gbs (copy bandwidth)",
                    "avg_launch_us": 1e3 * float(np.mean(gu_ms))}
    elif path == "decode":
        roofline = {"bound": "hbm", "kernel": PATHS[path][0], "achieved": gu_gbs, "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": gu_gbs / pk["hbm_gbs"], "traffic": traffic,
                    "algorithmic_bytes_per_launch": float(np.mean(gu_alg)),
                    "peak_source": f"{pk_kind} hbm_gbs (copy bandwidth)",
                    "avg_launch_us": 1e3 * float(np.mean(gu_ms))}
    else:
        rows = T * (cfg.k + cfg.S)
        flops = 2.0 * rows * (2 * cfg.I) * cfg.H
        tflops = flops / (float(np.mean(gu_ms)) / 1e3) / 1e12
        peak = pk["bf16_tflops"]
        roofline = {"bound": "tensor", "kernel": PATHS[path][0], "achieved": tflops, "peak": peak,
                    "unit": "TFLOP/s", "frac": tflops / peak, "traffic": traffic,
                    "algorithmic_flops_per_launch": flops,
                    "peak_source": f"{pk_kind} bf16_tflops (cuBLAS bf16 GEMM, burst: a step of a few "
                                   f"milliseconds is not the seconds-long loop the sustained figure is for; "
                                   f"fp16 operands of kind::f16 run at the bf16 rate)",
                    "frac_of_sustained": tflops / pk["bf16_tflops_sustained"],
                    "avg_launch_us": 1e3 * float(np.mean(gu_ms)),
                    "weight_stream_gbs": gu_gbs}

    # end to end through the public API with host buffers (pinned), copies timed
    x_pin = torch.from_numpy(xs_host.view(np.int16)).pin_memory()
    y_pin = torch.empty((total, T, cfg.H), dtype=torch.int16).pin_memory()
    x_stage = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)
    # (eager calls, as a caller without a graph makes them; two more events split off the
    # copies so that the gap to the graph-replayed device time can be attributed)
    e2e_ms = []
    for s in range(total):
        flush.zero_()
        a, c1, c2, b = (torch.cuda.Event(enable_timing=True) for _ in range(4))
        a.record(stream)
        x_stage.view(torch.int16).copy_(x_pin[s], non_blocking=True)
        c1.record(stream)
        lay = layers[s % n_layers]
        lay.route(x_stage)
        lay.forward(x_stage, y)
        c2.record(stream)
        y_pin[s].copy_(y.view(torch.int16), non_blocking=True)
        b.record(stream)
        if s >= args.warmup:
            e2e_ms.append((a, b, c1, c2))
    torch.cuda.synchronize(dev)
    e2e_total = sum(a.elapsed_time(b) for a, b, _, _ in e2e_ms)
    e2e_h2d_us = 1e3 * float(np.mean([a.elapsed_time(c1) for a, _, c1, _ in e2e_ms]))
    e2e_d2h_us = 1e3 * float(np.mean([c2.elapsed_time(b) for _, b, _, c2 in e2e_ms]))
    e2e_calls_us = 1e3 * float(np.mean([c1.elapsed_time(c2) for _, _, c1, c2 in e2e_ms]))
    e2e_value = throughput(world, T, args.steps, max_over_ranks(e2e_total, world, dev))
    st, det = moe.moe_get_error(layers[0].ws)
    if st != 0:
        raise RuntimeError(f"device error {moe.STATUS[st]} {det:#x}")

    line = None
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_dict(cfg, world, "eager launches" if graphs is None else
                                      "one CUDA graph per step (route + forward), replayed"),
                "roofline": roofline,
                "layer_weight_stream_gbs": layer_gbs,
                "kernel_us": ({"route": 1e3 * float(np.mean(rt_ms)), "forward_fused": 1e3 * float(np.mean(gu_ms)),
                               "step_with_events_between_kernels": 1e3 * float(np.mean(step_serial_ms)),
                               "measured": "second pass over the same steps with an event between the router "
                                           "and the forward kernel (which also stops their overlap)"}
                              if path == "fused" else
                              {"route": 1e3 * float(np.mean(rt_ms)), "gate_up": 1e3 * float(np.mean(gu_ms)),
                               "down": 1e3 * float(np.mean(dn_ms)), "combine": 1e3 * float(np.mean(cb_ms)),
                               "down_gbs": dn_gbs,
                               "step_with_events_between_kernels": 1e3 * float(np.mean(step_serial_ms)),
                               "measured": "second pass over the same steps with an event between kernels"}),
                "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * cfg.H * 2,
                        "d2h_bytes_per_step": T * cfg.H * 2, "launch": "eager calls (no graph)",
                        "us_per_step": {"h2d_copy": e2e_h2d_us, "route_and_forward": e2e_calls_us,
                                        "d2h_copy": e2e_d2h_us}},
                "gpu_launches": launches_per_step(cfg) * args.steps,
                "path": path,
                "wall_s_timed_region": wall,
                "clocks": ck}
        if world == 1 and not args.no_cpu_baseline:
            L0 = synth.Layer(cfg, 0)
            sample = [xs_host[i][: max(1, min(T, 4))] for i in range(min(8, total))]
            v, n, dt, cores = oracle_tokens_per_s(cfg, L0, sample, args.cpu_budget, 64)
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "cpu": cpu_model(),
                                    "kind": "oracle",
                                    "sample": f"{n} token(s) of this workload ({dt:.1f} s), routed and run "
                                              f"through every selected expert and the shared expert in fp64 "
                                              f"(expert weights drawn before timing)"}
        print(json.dumps(line), flush=True)
    for lay in layers:
        del lay
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_host_tier(args):
    """--host-tier: loads of experts from page-locked host memory into the device expert
    cache (moe_cache_load), the 2-bit ternary layout against the dense ternary storage
    form (five codes per byte, expanded on the GPU).  Full-size experts (hidden 7168,
    ffn 2048), 32 routed ternary experts + a ternary shared one, 16 slots; every timed
    round loads 8 experts (a one-token step's) into slots that held others, on one
    stream, timed with CUDA events.  One JSON line; not the benchmark's main line."""
    import dataclasses
    import torch
    import bit_routed_expert_fp32_b200 as moe
    from bit_routed_expert_fp32_b200.cache import ExpertCache
    cfg = synth.micro(T=1, H=7168, E=32, k=8, I=2048, S=1, formats="ternary", seed=7)
    cfg = dataclasses.replace(cfg, shared_format=synth.FMT_TERNARY, name="host_tier_H7168_I2048_ternary")
    layer = synth.Layer(cfg, 0)
    fmt_dense = np.full(cfg.E + cfg.S, moe.FMT_TERNARY_DENSE, np.uint8)
    out = {"metric": "host-tier expert load: host bytes and device time per expert", "config": {
        "workload": cfg.name, "experts": cfg.E, "slots": 16, "experts_per_round": 8, "rounds": args.steps}}
    stream = torch.cuda.current_stream()
    for name, fmt in (("ternary_2bit", layer.fmt), ("ternary_dense", fmt_dense)):
        host = moe.pack_layer(cfg, np.asarray(fmt, np.uint8), layer.expert)
        cache = ExpertCache(cfg, host, n_slots=16)
        ms = []
        for r in range(args.warmup + args.steps):
            ids = [(8 * r + j) % cfg.E for j in range(8)]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            cache.ensure(ids)
            b.record(stream)
            if r >= args.warmup:
                ms.append((a, b))
        torch.cuda.synchronize()
        loads = [a.elapsed_time(b) for a, b in ms]
        ent = host[256:256 + 64 * (cfg.E + cfg.S)].view(np.uint64).reshape(-1, 8)
        starts = sorted(int(v) for v in ent[:, 1])
        span = (starts[1] - starts[0]) if len(starts) > 1 else 0        # one expert's host bytes
        us = 1e3 * float(np.mean(loads)) / 8
        out[name] = {"host_bytes_per_expert": span, "us_per_expert": us,
                     "host_gb_per_s": span / (us * 1e-6) / 1e9}
        del cache
    out["bytes_saved"] = 1 - out["ternary_dense"]["host_bytes_per_expert"] / out["ternary_2bit"]["host_bytes_per_expert"]
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--soak-s", type=float, default=1.5)
    ap.add_argument("--tokens", type=int, default=0, help="override the workload's tokens per step (profiling)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the routed expert count (profiling: the same per-step work on a smaller layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every call eagerly instead of replaying graphs")
    ap.add_argument("--host-tier", action="store_true",
                    help="time expert loads from host memory into the expert cache (2-bit vs dense ternary)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    cfg = synth.CONFIGS[args.config]
    if args.tokens:
        import dataclasses
        cfg = dataclasses.replace(cfg, T=args.tokens, name=f"{cfg.name}_T{args.tokens}")
    if args.experts:
        import dataclasses
        cfg = dataclasses.replace(cfg, E=args.experts, name=f"{cfg.name}_E{args.experts}")
    if args.host_tier:
        return run_host_tier(args)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
