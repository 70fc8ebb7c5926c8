#!/usr/bin/env python
"""Benchmark of the QK-RMSNorm sliding-window attention core on B200.

One step = forward + backward of every layer of the 8-layer "SSSL" attention
stack (B=8, T=2048, H=4, D=128; layers 0-2 and 4-6 window 1024, layers 3 and 7
full causal), each layer on its own seeded bf16 inputs, all enqueued back to
back on one stream through the C ABI (libar_attn.so).

Metric: TFLOP/s counted on unmasked (query, key) pairs only, 4*D FLOPs per pair
forward and 2.5x that backward; also reported as a fraction of the measured
dense bf16 tensor-core peak.

  python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

With N > 1 (under torchrun) every rank runs the same workload on its own GPU
(replicas: the core has no cross-GPU data flow); the time is the max over
ranks and the value the sum of all ranks' FLOPs over that time.
--impl reference times the fp64 CPU oracle on a bounded sample instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd+bwd TFLOP/s (unmasked) at T=2048 SSSL; % of B200 BF16 peak"
D = 128  # head dimension of the stated workloads (a workload may set its own)
BWD_FACTOR = 2.5

WORKLOADS = {
    "stack8": dict(config=3, B=8, T=2048, H=4, n_layer=8, pattern="SSSL",
                   name="8-layer SSSL attention stack fwd+bwd, B=8 T=2048 H=4 D=128 (windows 1024/full)"),
    "stack12": dict(config=5, B=8, T=2048, H=6, n_layer=12, pattern="SSSL",
                    name="12-layer SSSL attention stack fwd+bwd, B=8 T=2048 H=6 D=128 (windows 1024/full)"),
    "layer_s": dict(config=2, B=8, T=2048, H=4, n_layer=1, windows=[1024],
                    name="single S layer fwd+bwd, B=8 T=2048 H=4 D=128, window 1024"),
    "layer_l": dict(config=2, B=8, T=2048, H=4, n_layer=1, windows=[2048],
                    name="single L layer fwd+bwd, B=8 T=2048 H=4 D=128, full causal"),
    "long_s": dict(config=4, B=2, T=8192, H=4, n_layer=1, windows=[4096],
                   name="long-context S layer fwd+bwd, B=2 T=8192 H=4 D=128, window 4096"),
    "long_l": dict(config=4, B=2, T=8192, H=4, n_layer=1, windows=[8192],
                   name="long-context L layer fwd+bwd, B=2 T=8192 H=4 D=128, full causal"),
    # the stack with the steps before the core fused in: RoPE on every layer, the
    # value embedding on every other layer (the last included); not a stated workload
    "stack8_rope": dict(config=3, B=8, T=2048, H=4, n_layer=8, pattern="SSSL", rope=True,
                        name="8-layer SSSL attention stack fwd+bwd with fused RoPE and value embeddings, "
                             "B=8 T=2048 H=4 D=128 (windows 1024/full)"),
    "layer_s_rope": dict(config=2, B=8, T=2048, H=4, n_layer=1, windows=[1024], rope=True,
                         name="single S layer fwd+bwd with fused RoPE and value embedding, B=8 T=2048 H=4 D=128, "
                              "window 1024"),
    # head dimension 64 (width 512 in 8 heads of 64): not one of the stated workloads
    "stack8_d64": dict(config=3, B=8, T=2048, H=8, D=64, n_layer=8, pattern="SSSL",
                       name="8-layer SSSL attention stack fwd+bwd, B=8 T=2048 H=8 D=64 (windows 1024/full)"),
    # grouped K/V heads (n_kv_head = n_head / 2): not one of the stated workloads
    "stack8_gqa": dict(config=3, B=8, T=2048, H=4, Hkv=2, n_layer=8, pattern="SSSL",
                       name="8-layer SSSL attention stack fwd+bwd, B=8 T=2048 H=4 Hkv=2 D=128 (windows 1024/full)"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="stack8")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: oracle time budget for the whole run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def windows_for(wl, rule):
    """Per-layer windows of the workload; rule(n_layer, T, pattern) is the
    library's window rule on the product path and the oracle's in its legs."""
    if "windows" in wl:
        return list(wl["windows"])
    return rule(wl["n_layer"], wl["T"], wl["pattern"])


def lib_windows(wl):
    from sliding_window_attention_rmsnorm_b200.stack import layer_windows
    return windows_for(wl, layer_windows)


def oracle_windows(wl):
    from oracle.stack import layer_windows
    return windows_for(wl, layer_windows)


def pairs(T, w):
    w = T if (w < 0 or w >= T - 1) else w
    n1 = min(w + 1, T)
    return n1 * (n1 + 1) // 2 + (T - n1) * (w + 1)


def head_dim(wl):
    return wl.get("D", D)


def step_flops(wl, windows):
    """(forward, backward) counted FLOPs of one step of the workload: 4 D per
    visible (query, key) pair forward, 2.5 times that backward."""
    f = sum(wl["B"] * wl["H"] * pairs(wl["T"], w) * 4 * head_dim(wl) for w in windows)
    return f, BWD_FACTOR * f


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(bf16_burst=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"], hbm=d["hbm_gbs"],
                    source="measured")
    return dict(bf16_burst=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of each kernel on one S layer and one L layer (B=8 T=2048 H=4
# D=128; windows 1024 and full), each record valid while the sha256 of every
# source the kernel is built from still matches:
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum --clock-control none \
#       -k regex:"fwd_kernel|bwd_kernel|dq_kernel|bwd_prep" -s 12 -c 4 --csv \
#       python bench.py --workload layer_s|layer_l --steps 1 --warmup 3 --no-e2e --no-cpu-baseline
# ncu flushes the caches before each launch: these are cold-L2 bytes.
CAPTURED_TRAFFIC = {
    "fwd": {"sources": {"fwd.cuh": "3238025202dbfa4b90f4191cc23f00fee4f82c3a8e466925ab65278e0af5173d", "sm100.cuh": "1111847c6474fba79ab804963ad60d50973f7689121be5d4af96fe31bc24aafe", "ar_attn.cu": "075ecd8e19f33e0c2de012c2325dcc6389ca626a71fc40ce62de70a9912de609"},
           "bytes": {(8, 2048, 4, 1024): 51979264, (8, 2048, 4, 2048): 51943680}},
    "bwd": {"sources": {"bwd.cuh": "7426e2685f4cdc42d91d97bbbef77aabcd18e68298d2d94892f6ff9d81a0ea60", "sm100.cuh": "1111847c6474fba79ab804963ad60d50973f7689121be5d4af96fe31bc24aafe", "ar_attn.cu": "075ecd8e19f33e0c2de012c2325dcc6389ca626a71fc40ce62de70a9912de609"},
           "bytes": {(8, 2048, 4, 1024): 162760704, (8, 2048, 4, 2048): 205586944}},
    "dq": {"sources": {"dq.cuh": "d28931aa90808a8e6071b2cc4d04d4d1900378b57cb50325525353d1fd32d1a1", "sm100.cuh": "1111847c6474fba79ab804963ad60d50973f7689121be5d4af96fe31bc24aafe", "ar_attn.cu": "075ecd8e19f33e0c2de012c2325dcc6389ca626a71fc40ce62de70a9912de609"},
           "bytes": {(8, 2048, 4, 1024): 149263872, (8, 2048, 4, 2048): 181063936}},
    "bwd_prep": {"sources": {"aux.cuh": "f97d4ff35e9bea1000a15d5ce35268bf1b1c1f70a312d9a7af8cda49d85a7df8", "sm100.cuh": "1111847c6474fba79ab804963ad60d50973f7689121be5d4af96fe31bc24aafe", "ar_attn.cu": "075ecd8e19f33e0c2de012c2325dcc6389ca626a71fc40ce62de70a9912de609"},
           "bytes": {(8, 2048, 4, 1024): 50615808, (8, 2048, 4, 2048): 50615808}},
}


def captured_traffic(kind, wl, windows):
    """Mean DRAM bytes per launch of one kernel over the workload's layers, or
    None when a layer shape was not captured or a source changed since."""
    import hashlib
    rec = CAPTURED_TRAFFIC.get(kind)
    # captured: the plain multi-head path at head dimension 128 (the RoPE and
    # value-embedding variants and D = 64 are other instantiations)
    if rec is None or wl.get("rope") or head_dim(wl) != 128:
        return None
    csrc = os.path.join(ROOT, "sliding_window_attention_rmsnorm_b200", "csrc")
    for name, digest in rec["sources"].items():
        try:
            if hashlib.sha256(open(os.path.join(csrc, name), "rb").read()).hexdigest() != digest:
                return None
        except OSError:
            return None
    per_layer = []
    for w in windows:
        key = (wl["B"], wl["T"], wl["H"], w if w < wl["T"] - 1 else wl["T"])
        if key not in rec["bytes"] or wl.get("Hkv", wl["H"]) != wl["H"]:
            return None
        per_layer.append(rec["bytes"][key])
    return sum(per_layer) / len(per_layer)


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the GPU is timed."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_id), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1] or [s for (_, s) in self.samples]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and "Active" == r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ---------------------------------------------------------------- oracle (CPU baseline and reference arm)
_INPUT_CACHE = {}


def layer_host_inputs(wl, layer):
    """Seeded bf16 CPU inputs of one layer: q, dO with H heads, k, v with Hkv
    (and ve, g on the value-embedding layers of a RoPE workload)."""
    from sliding_window_attention_rmsnorm_b200 import synth
    H, Hkv, Dh = wl["H"], wl.get("Hkv", wl["H"]), head_dim(wl)
    if Hkv == H:
        x = synth.layer_inputs(wl["config"], layer, wl["B"], wl["T"], H, Dh)
    else:
        x = synth.layer_inputs(wl["config"], layer, wl["B"], wl["T"], H, Dh, roles=("q", "dO"))
        x.update(synth.layer_inputs(wl["config"], layer, wl["B"], wl["T"], Hkv, Dh, roles=("k", "v")))
    if wl.get("rope") and layer % 2 == (wl["n_layer"] - 1) % 2:
        x["ve"], x["g"] = synth.value_embedding(wl["config"], layer, wl["B"], wl["T"], Hkv, D)
    return x


def _layer_inputs_cached(wl, layer):
    key = (wl["config"], wl.get("Hkv"), layer)
    if key not in _INPUT_CACHE:
        _INPUT_CACHE[key] = layer_host_inputs(wl, layer)
    return _INPUT_CACHE[key]


def oracle_sample(wl, seconds, seed_layer_offset=0):
    """Run the fp64 oracle fwd+bwd on whole heads of the workload's layers,
    cycling through layers, for about `seconds`; returns (flops, secs, desc, threads)."""
    from oracle import oracle as orc
    ws = oracle_windows(wl)
    B, T, H = wl["B"], wl["T"], wl["H"]
    flops, heads_done, t_total, n = 0.0, [], 0.0, 0
    while t_total < seconds or n == 0:
        layer = (n + seed_layer_offset) % wl["n_layer"]
        head = (7 * n + 3) % (B * H)
        b, h = divmod(head, H)
        hk = h // (H // wl.get("Hkv", H))  # the query head's K/V head
        x = _layer_inputs_cached(wl, layer)
        xs = {r: t[b:b + 1, :, (hk if r in ("k", "v", "ve", "g") else h):][:, :, :1].contiguous()
              for r, t in x.items()}
        t0 = time.perf_counter()
        if wl.get("rope"):
            from oracle import rope_ve
            cs, sn = rope_ve.rope_tables(T, D)
            rope_ve.attn_fwd(xs["q"], xs["k"], xs["v"], cs, sn, ws[layer], ve=xs.get("ve"), g=xs.get("g"))
            rope_ve.attn_bwd(xs["q"], xs["k"], xs["v"], xs["dO"], cs, sn, ws[layer], ve=xs.get("ve"), g=xs.get("g"))
        else:
            orc.attn_fwd(xs["q"], xs["k"], xs["v"], ws[layer])
            orc.attn_bwd(xs["q"], xs["k"], xs["v"], xs["dO"], ws[layer])
        t_total += time.perf_counter() - t0
        flops += pairs(T, ws[layer]) * 4 * head_dim(wl) * (1 + BWD_FACTOR)
        heads_done.append((layer, head))
        n += 1
    desc = "%d whole heads (T=%d) of the workload's layers, fwd+bwd in fp64 C/OpenMP" % (n, T)
    return flops, t_total, desc, orc.num_threads()


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    from oracle import oracle as orc
    per_step = max(1.0, args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(wl, 0.0)
    flops, secs, desc, threads = 0.0, 0.0, "", orc.num_threads()
    for s in range(args.steps):
        f, t, desc, threads = oracle_sample(wl, per_step, seed_layer_offset=s)
        flops += f
        secs += t
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl["name"], "global_batch": wl["B"], "seq_len": wl["T"], "heads": wl["H"],
                   "layers": wl["n_layer"], "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": "per step: " + desc, "cpu_model": cpu_model(), "nproc": os.cpu_count()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- multi-rank helpers
def max_over_ranks(dist, x, device):
    """x maximised over all ranks (x itself in a single process)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world, flops_per_rank_step, ms_per_step):
    """Whole-job rate: every rank runs the same step, timed by the slowest rank."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- our CUDA path
def run_ours(args, wl, rank, world, dist):
    import torch
    from sliding_window_attention_rmsnorm_b200 import attn, build, stack, synth

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    build.build()
    B, T, H, L = wl["B"], wl["T"], wl["H"], wl["n_layer"]
    host = [layer_host_inputs(wl, l) for l in range(L)]
    layers = [{r: t.to("cuda", non_blocking=False) for r, t in x.items()} for x in host]
    rope = attn.rope_tables(T, D) if wl.get("rope") else None
    st = stack.Stack(layers, wl.get("pattern", "SSSL"), windows=wl.get("windows"), rope=rope)
    windows = lib_windows(wl)
    fwd_f, bwd_f = step_flops(wl, windows)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        st.step()
    attn.sync_status()

    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    sampler = ClockSampler(visible[dev] if dev < len(visible) else dev) if rank == 0 else None
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        st.step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    attn.sync_status()
    ms = e0.elapsed_time(e1) / args.steps
    # Per-kernel durations come from a second pass of the same steps with an event
    # pair around every launch: events between launches keep the GPU from
    # overlapping one kernel's launch with the previous kernel's tail, so they
    # stay out of the timed region above.
    ksteps = max(1, min(args.steps, 20))
    attn.timing_enable(True)
    for _ in range(ksteps):
        st.step()
    torch.cuda.synchronize()
    attn.timing_enable(False)
    attn.sync_status()
    kern = attn.timing_read()
    ms = max_over_ranks(dist, ms, "cuda")
    clocks = None
    if sampler is not None:
        sampler.stop()
        clocks = sampler.summary(t_wall0, t_wall1)

    value = job_tflops(world, fwd_f + bwd_f, ms)
    peaks = measured_peaks()

    # Roofline of the dominant kernel: the counted FLOPs of its own products per
    # launch over its event-timed mean duration.  The backward's counted work is
    # 2.5x the forward's, five products of the forward's size; the main kernel
    # runs four of them (S, dP, dV, dK) and the dq kernel the fifth (G K).  The
    # per-launch events cover tens of milliseconds, so the burst peak applies.
    per_kind_flops = {"fwd": fwd_f / L, "bwd": bwd_f / L * 4 / 5, "dq": bwd_f / L / 5}
    dom = max(("fwd", "bwd"), key=lambda k: kern[k][0])
    tot_ms, n_launch = kern[dom]
    achieved = (per_kind_flops[dom] * n_launch) / (tot_ms * 1e-3) / 1e12
    roof = {"kernel": dom + "_kernel", "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_burst"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_burst"],
            "traffic": captured_traffic(dom, wl, windows),
            "peak_kind": "bf16 burst (%s)" % peaks["source"],
            "flops_per_launch": per_kind_flops[dom]}
    kernels = {k: {"ms_per_launch": (v[0] / v[1]) if v[1] else None, "launches": v[1],
                   "share": v[0] / max(1e-9, sum(x[0] for x in kern.values()))} for k, v in kern.items()}
    for k in ("fwd", "bwd", "dq"):
        if kern[k][1]:
            kernels[k]["tflops"] = per_kind_flops[k] * kern[k][1] / (kern[k][0] * 1e-3) / 1e12
            kernels[k]["frac_of_burst"] = kernels[k]["tflops"] / peaks["bf16_burst"]
            kernels[k]["traffic"] = captured_traffic(k, wl, windows)
    if kern["bwd"][1] and kern["dq"][1]:  # the whole backward's products over both kernels' time
        t = (kern["bwd"][0] + kern["dq"][0]) * 1e-3
        kernels["bwd+dq"] = {"tflops": bwd_f * kern["bwd"][1] / L / t / 1e12}
        kernels["bwd+dq"]["frac_of_burst"] = kernels["bwd+dq"]["tflops"] / peaks["bf16_burst"]
    # memory-bound helpers: algorithmic bytes per launch
    tok = B * T * H
    # the dq kernel reads one 32 KB G tile per (query tile, key tile) pair of the band
    # (mean over the stack's layers) plus q, and writes dq; its K tile reads hit L2
    nq = -(-T // 128)
    g_pairs = sum(B * H * sum(min(qt + 1, min(nq, (min(w, T) + 127) // 128 + 1)) for qt in range(nq))
                  for w in windows) / L
    Dh = head_dim(wl)
    algo_bytes = {"fwd_prep": tok * Dh * 2 + tok * 4,
                  "bwd_prep": 3 * tok * Dh * 2 + tok * 4 * 4,
                  "dq": g_pairs * 32768 + tok * Dh * 2 * 2}
    for k, by in algo_bytes.items():
        if kern[k][1]:
            kernels[k]["gbs"] = by * kern[k][1] / (kern[k][0] * 1e-3) / 1e9
            kernels[k]["hbm_frac"] = kernels[k]["gbs"] / peaks["hbm"]
    if kern["bwd_prep"][1]:
        kernels["bwd_prep"]["traffic"] = captured_traffic("bwd_prep", wl, windows)

    # End to end: inputs from pinned host memory, results back to host, all inside
    # the timed region.  The copies run on their own streams, layer by layer: the
    # inputs of layer l+1 cross while layer l's forward runs, each layer's o as
    # soon as the forwards are done, and each layer's gradients while the next
    # (lower) layer's backward runs; the step ends when its last result is on the host.
    e2e = None
    if not args.no_e2e:
        pinned = [{r: t.pin_memory() for r, t in x.items()} for x in host]
        out_names = [[n for n in ("o", "dq", "dk", "dv", "dve", "dg") if n in st.out[l]] for l in range(L)]
        outs_h = [{n: torch.empty(st.out[l][n].shape, dtype=st.out[l][n].dtype, pin_memory=True)
                   for n in out_names[l]} for l in range(L)]
        h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
        # Two stacks (inputs, outputs, scratch), alternating steps: while step i
        # computes on one and its results cross back to the host, step i+1's
        # inputs cross into the other, so the two directions of the host link
        # overlap.  Within a step the forward operands of layer l cross before
        # layer l+1's, dO last (last layer first, the backward's order), each
        # layer's o goes back as soon as its forward is done and its gradients
        # as soon as its backward is.
        layers2 = [{r: torch.empty_like(t) for r, t in x.items()} for x in layers]
        st2 = stack.Stack(layers2, wl.get("pattern", "SSSL"), windows=wl.get("windows"), rope=rope)
        bufs = [(st, layers), (st2, layers2)]
        inputs_free = [None, None]  # per stack: its previous step's last kernel
        outputs_read = [None, None]  # per stack: its previous step's last copy to the host

        def mark(strm):
            ev = torch.cuda.Event()
            ev.record(strm)
            return ev

        def issue_h2d(i):
            _, lay = bufs[i % 2]
            with torch.cuda.stream(h2d_stream):
                if inputs_free[i % 2] is not None:
                    h2d_stream.wait_event(inputs_free[i % 2])
                fwd_in = []
                for l in range(L):
                    for r, t in pinned[l].items():
                        if r != "dO":
                            lay[l][r].copy_(t, non_blocking=True)
                    fwd_in.append(mark(h2d_stream))
                bwd_in = [None] * L
                for l in reversed(range(L)):
                    lay[l]["dO"].copy_(pinned[l]["dO"], non_blocking=True)
                    bwd_in[l] = mark(h2d_stream)
            return fwd_in, bwd_in

        def compute(i, fwd_in, bwd_in):
            s = bufs[i % 2][0]
            if outputs_read[i % 2] is not None:
                stream.wait_event(outputs_read[i % 2])
            for l in range(L):
                stream.wait_event(fwd_in[l])
                s.forward_layer(l)
                d2h_stream.wait_event(mark(stream))
                with torch.cuda.stream(d2h_stream):
                    outs_h[l]["o"].copy_(s.out[l]["o"], non_blocking=True)
            for l in reversed(range(L)):
                stream.wait_event(bwd_in[l])
                s.backward_layer(l)
                d2h_stream.wait_event(mark(stream))
                with torch.cuda.stream(d2h_stream):
                    for n in out_names[l]:
                        if n != "o":
                            outs_h[l][n].copy_(s.out[l][n], non_blocking=True)
            inputs_free[i % 2] = mark(stream)
            outputs_read[i % 2] = mark(d2h_stream)

        def run_steps(n):
            h2d_stream.wait_stream(stream)
            ins = issue_h2d(0)
            for i in range(n):
                nxt = issue_h2d(i + 1) if i + 1 < n else None
                compute(i, *ins)
                ins = nxt
            stream.wait_stream(d2h_stream)

        run_steps(2)
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        run_steps(args.e2e_steps)
        a1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = a0.elapsed_time(a1) / args.e2e_steps
        # the pipelined copies must not change a result: the last step's outputs on
        # the host equal, bit for bit, an ordinary step's on the device (the kernels
        # are deterministic and both buffer sets hold the same inputs)
        st.step()
        torch.cuda.synchronize()
        for l in range(L):
            for n in out_names[l]:
                if not torch.equal(outs_h[l][n], st.out[l][n].cpu()):
                    raise RuntimeError("e2e: layer %d %s differs from an ordinary step" % (l, n))
        ms_e2e = max_over_ranks(dist, ms_e2e, "cuda")
        h2d = sum(t.numel() * t.element_size() for x in pinned for t in x.values())
        d2h = sum(t.numel() * t.element_size() for x in outs_h for t in x.values())
        e2e = {"value": job_tflops(world, fwd_f + bwd_f, ms_e2e), "unit": "TFLOP/s",
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "every step's inputs from pinned host memory and all its outputs back, inside the timed "
                         "region; two device buffer sets, so step i+1's uploads overlap step i's compute and "
                         "downloads; outputs checked bitwise against an ordinary step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, secs, desc, threads = oracle_sample(wl, args.cpu_seconds)
        cpu = {"value": f / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "cpu_model": cpu_model(), "nproc": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl["name"], "global_batch": B * world, "seq_len": T, "heads": H,
                       "head_dim": head_dim(wl),
                       **({"kv_heads": wl["Hkv"]} if wl.get("Hkv", H) != H else {}),
                       "layers": L, "windows": windows, "parallelism": "replicas x%d" % world,
                       "l2": "inputs larger than L2 (%.0f MB of q,k,v,dO per step)"
                             % (sum(t.numel() * t.element_size() for x in host for t in x.values()) / 1e6)},
            "pct_of_bf16_peak": {"sustained": value / world / peaks["bf16_sustained"],
                                 "burst": value / world / peaks["bf16_burst"], "source": peaks["source"]},
            "roofline": roof,
            "kernels": kernels,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(round(sum(v[1] for v in kern.values()) * args.steps / ksteps)),
            "kernels_pass": {"steps": ksteps, "note": "per-launch CUDA events, separate pass after the timed region"},
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    wl = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        if args.impl == "reference":
            run_reference(args, wl, rank, world)
        else:
            run_ours(args, wl, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
