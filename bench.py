"""Window-step benchmark: tokens/s of the DualParal window step and attention TFLOP/s.

One step = the whole hot path on one window: per-block adaLN lookup (host), K/V
modulation prepass, tensor-core window attention over [cache ; window] with the fused Q
prologue and gate epilogue, and the queue/cache advance (head block -> cache, fresh noise
block pushed).  Default workload: the largest window that runs on one GPU, the shape
sweep's 131,072-token window (4 blocks x 32,768 tokens, 32,768-token cache, 16 x 128
heads, bf16).  The default run also times, each in its own timed region with its own clock
record, the Wan-like window (8 x 6,240 tokens, 12 x 128 heads), the long run's steady-state
window (8 x 2,700 tokens, 24 x 64 heads) and the whole 850-step long run, under
"target_configs" (--no-extra skips them).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

The roofline peak is the measured dense bf16 GEMM peak that matches the timed region's
clocks: the sustained figure (measured back to back for seconds under the power cap) when
sw_power_cap was active during a timed region of a second or more, else the burst figure;
both fractions are reported.

N > 1 runs under torch.distributed.run, one process per GPU; every rank runs an
independent replica (the step needs no exchange between GPUs), the timed region is
bracketed by barriers and synchronizes, and the slowest rank's time sets the value.
--impl reference times the CPU oracle (float64 NumPy) on a bounded sample of the same
workload.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "window-step tokens/s and attention TFLOP/s (fraction of bf16 peak) at 1 B200"

# DRAM bytes (read + write) of one attention launch from an ncu capture (summaries under
# profiles/), valid only for the kernel source they were captured on (md5 over
# csrc/dp_attn_tc.cu and csrc/dp_device.cuh); any other source reports null.
TRAFFIC_SOURCE_MD5 = "0f4d0a643530e059790321993f0188af"
TRAFFIC_BYTES = {"cogvideo_bf16": 233.596416e6 + 50.829312e6, "wan_bf16": 633.475072e6 + 142.530048e6,
                 "sweep_16384": 236.308736e6 + 51.109632e6, "sweep_131072": 9532.882944e6 + 564.817408e6}
L2_BYTES = 126 * 1024 * 1024


def attention_traffic(config_name: str):
    import hashlib
    h = hashlib.md5()
    for name in ("dp_attn_tc.cu", "dp_device.cuh"):
        try:
            with open(os.path.join(ROOT, "long_video_diffusion_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        except OSError:
            return None
    return TRAFFIC_BYTES.get(config_name) if h.hexdigest() == TRAFFIC_SOURCE_MD5 else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def choose_peak(peaks, clocks, timed_s: float):
    """The bf16 peak that matches how the timed region ran: the sustained figure was measured
    as a seconds-long GEMM loop under the 1 kW power cap, the burst one as short runs at full
    clock.  The sustained one applies when sw_power_cap was active during a timed region of at
    least a second; otherwise the burst one."""
    reasons = (clocks or {}).get("reasons") or []
    capped = "sw_power_cap" in reasons
    if capped and timed_s >= 1.0:
        kind, why = "bf16_tflops_sustained", f"sw_power_cap active over a {timed_s:.1f} s timed region"
    else:
        kind = "bf16_tflops"
        why = ("no power cap in the clock record" if not capped
               else f"sw_power_cap active but the timed region is only {timed_s:.2f} s")
    return {"peak": peaks[kind], "kind": f"{kind} ({peaks['source']})", "why": why,
            "burst": peaks["bf16_tflops"], "sustained": peaks["bf16_tflops_sustained"]}


def roofline_fracs(achieved, pk):
    if not achieved:
        return {"frac": None, "frac_of_burst": None, "frac_of_sustained": None}
    return {"frac": achieved / pk["peak"], "frac_of_burst": achieved / pk["burst"],
            "frac_of_sustained": achieved / pk["sustained"]}


DEFAULT_CONFIG = "sweep_131072"
# timed steps when --steps is not given: about a few seconds of timed work per workload
DEFAULT_STEPS = {"sweep_131072": 30, "wan_bf16": 80, "longrun_steady_bf16": 300}
EXTRA_CONFIGS = ["wan_bf16", "longrun_steady_bf16", "long_run"]


def workload(name: str):
    from workloads import step_config
    if name.startswith("sublayer_fresh_"):
        return step_config(name[len("sublayer_fresh_"):])
    if name.startswith("sublayer_"):
        return step_config(name[len("sublayer_"):])
    if name.startswith("long_run"):
        # the oracle arms time a steady-state step of the run (same shapes as its 8-block window)
        return step_config("longrun_steady_bf16")
    if name.startswith("sweep_"):
        parts = name.split("_")
        return step_config("sweep", int(parts[1]), ragged=len(parts) > 2 and parts[2] == "ragged")
    return step_config(name)


def describe(cfg) -> str:
    return (f"{cfg.name}: {cfg.n_blocks} blocks x {cfg.block_rows[0]} tokens (window {cfg.n_win}), "
            f"cache {cfg.cache_len}, {cfg.n_heads}x{cfg.head_dim} heads, {cfg.dtype}")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.out = os.path.join("/tmp", f"dp_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.out, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.out) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == len(self.FIELDS):
                    rows.append(parts)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, nme in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(nme)
        load = [s for s in sm if s > 0]
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------------------- GPU arm

def gpu_arm(args, rank: int, world: int, local_rank: int, config: str = None, steps: int = None,
            with_e2e: bool = True):
    import torch
    import torch.distributed as dist

    import long_video_diffusion_b200 as dp
    from workloads import as_features, make_step_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    config = config or args.config
    steps = steps or args.steps
    cfg = workload(config)
    if cfg.dtype != "bf16":
        raise SystemExit("bench workloads are bf16")
    x = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    eb = 2
    table = x["table"].to(dev)
    blk = dp.blocks_from_table(table, x["timesteps"], cfg.block_rows)
    q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    noise = x["noise"].to(dev)
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float16,
                       k=as_features(x["cache_k"], cfg.dtype).to(dev).view(1, -1, D),
                       v=as_features(x["cache_v"], cfg.dtype).to(dev).view(1, -1, D), length=cfg.cache_len)
    slot_rows = max(cfg.block_rows)
    queue = dp.Queue(cfg.n_blocks, slot_rows, D, device=dev)
    for _ in range(cfg.n_blocks):
        dp.queue_push(queue, noise)
    kv = torch.empty(2, n, D, dtype=torch.float16, device=dev)
    out = torch.empty(n, D, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        dp.window_step(q, k, v, blk, cache, kv, out, H, hd, pop=True, queue=queue, push_noise=noise)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dp.device_status()

    # ---- timed region: K window steps; each stage is timed live by the library's events
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(_smi_index(local_rank)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    dp.profile_begin(steps)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    mod_ms, attn_ms, adv_ms, n_prof = dp.profile_end()
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    dp.device_status()
    ms = t0.elapsed_time(t1)
    attn_ms, mod_ms, adv_ms = attn_ms / n_prof, mod_ms / n_prof, adv_ms / n_prof
    if not with_e2e:
        ms, attn_ms, mod_ms, adv_ms = max_over_ranks([ms, attn_ms, mod_ms, adv_ms], dev)
        return cfg, dict(ms=ms, steps=steps, attn_ms=attn_ms, mod_ms=mod_ms, adv_ms=adv_ms, clocks=clocks)

    # ---- the two HBM-bound kernels timed alone, back to back on the same bytes (the stage
    # events above hold each launch's gap and run at the SM clock the attention leaves behind,
    # power-capped on the large workloads)
    def t_alone(fn, iters=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(iters):
            fn()
        a1.record(stream)
        torch.cuda.synchronize()
        return a0.elapsed_time(a1) / iters

    n0 = cfg.block_rows[0]
    mod_alone_ms = t_alone(lambda: (dp.adaln_modulate(k, kv[0], blk), dp.adaln_modulate(v, kv[1], blk)))
    adv_alone_ms = t_alone(lambda: dp.kvcache_advance(cache, kv[0][:n0], kv[1][:n0], n0))
    dp.device_status()

    # ---- e2e: the same step through the public API from pinned host buffers, every step's
    # inputs copied in and its output read back inside the timed region (the library's
    # StepPipeline overlaps step i's copies with step i - 1's compute on three streams)
    hq, hk, hv = (x[key].pin_memory() for key in ("q", "k", "v"))
    hnoise = x["noise"].pin_memory()
    hout = torch.empty(n, D, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(steps, 50))
    pipe = dp.StepPipeline(n, D, noise.shape[0], device=dev)

    def e2e_step():
        pipe.submit(hq, hk, hv, hnoise, hout, blk, cache, kv, H, hd, pop=True, queue=queue)

    for _ in range(3):
        e2e_step()
    pipe.finish()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.h2d)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(pipe.d2h)
    pipe.finish()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    dp.device_status()

    # slowest rank sets the time
    ms, e2e_ms, attn_ms, mod_ms, adv_ms, mod_alone_ms, adv_alone_ms = max_over_ranks(
        [ms, e2e_ms, attn_ms, mod_ms, adv_ms, mod_alone_ms, adv_alone_ms], dev)
    return cfg, dict(ms=ms, steps=steps, e2e_ms=e2e_ms, e2e_steps=e2e_steps, attn_ms=attn_ms, mod_ms=mod_ms,
                     adv_ms=adv_ms, mod_alone_ms=mod_alone_ms, adv_alone_ms=adv_alone_ms, clocks=clocks,
                     h2d=(hq.numel() + hk.numel() + hv.numel() + hnoise.numel()) * eb, d2h=hout.numel() * eb)


def long_run_arm(args, rank: int, world: int, local_rank: int, config: str = None, steps: int = None,
                 with_e2e: bool = True):
    """The whole long-video queue run (257 latent frames, 8-block window, 50 staggered
    timesteps per block): every schedule step is one window step of the library, with the
    window growing from 1 to 8 blocks, the head block exiting into the cache and fresh noise
    blocks pushed.  W warm-up steps run on a separate queue; then the first K schedule steps
    (all 850 by default) of a fresh run are timed.  long_run_ctx4: the cache holds the last
    four exited blocks (8 latent frames, the pages' NumC = 8) and every step attends to all
    of them.  long_run_coord: blocks are pushed with the coordinated noise initialisation
    (frames of a pool holding the first window's noise, in a fresh random order per block).
    long_run_fresh: before every step the context K/V are recomputed from the exited block's
    latent rows (conditioned on timestep 0, where its last evaluation ran) instead of reused."""
    import torch
    import torch.distributed as dist

    import long_video_diffusion_b200 as dp
    from workloads import make_noise_permutations, make_run_noise, make_run_pool, make_run_table, run_config

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    config = config or args.config
    steps = steps or args.steps
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    noise_cpu = make_run_noise(rc)
    table = make_run_table(rc).to(dev)
    noise = [b.to(dev) for b in noise_cpu]
    tau = [int(round(999.0 * (T - 1 - i) / (T - 1))) for i in range(T)]
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device=dev)
    out = torch.empty(n_max, D, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    n_ctx = 4 if config == "long_run_ctx4" else 1
    fresh_t = 0 if config == "long_run_fresh" else None
    frame_pool = None
    if config == "long_run_coord":
        pool = make_run_pool(rc).to(dev)
        nf = [r // rc.frame_rows for r in rc.block_rows]
        perms = make_noise_permutations(len(nf), pool.shape[0], seed=rc.seed + 2000)
        frame_pool = (pool, dp.coordinated_schedule(nf, W, perms))

    def new_state():
        return (dp.KVCache(rc.slot_rows, D, torch.float16, n_slots=n_ctx, device=dev),
                dp.Queue(W + (1 if fresh_t is not None else 0), rc.slot_rows, D, device=dev))

    def cache_rows_read(c):
        return sum(c.desc.len[i] for i in range(n_ctx)) if n_ctx > 1 else c.length

    cache, queue = new_state()
    dp.run_fifo(noise, table, tau, W, cache, queue, kv, out, H, hd, max_steps=args.warmup,
                cache_all_slots=n_ctx > 1, frame_pool=frame_pool, fresh_t=fresh_t)
    torch.cuda.synchronize()
    dp.device_status()

    # per-step attention work: 4 n (L_c + n) hd H with L_c the cache length before the step
    steps_n, steps_lc = [], []
    cache, queue = new_state()
    state = {"lc": 0, "exited": False}

    launches = [0]

    step_ev = []

    def on_step(step, n, popped, pushed):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        step_ev.append(ev)
        steps_n.append(n)
        steps_lc.append(state["lc"])
        state["lc"] = cache_rows_read(cache)
        if fresh_t is not None and state["exited"]:
            launches[0] += 1     # the context recompute before the step
        state["exited"] = state["exited"] or popped
        if frame_pool is None:   # modulate, attention (+ one copy for the pop and the push)
            launches[0] += 2 + (1 if (popped or pushed is not None) else 0)
        else:                    # modulate, attention (+ the pop's copy) (+ the push's gather)
            launches[0] += 2 + (1 if popped else 0) + (1 if pushed is not None else 0)

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(_smi_index(local_rank)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    dp.profile_begin(steps)
    t0.record(stream)
    n_steps = dp.run_fifo(noise, table, tau, W, cache, queue, kv, out, H, hd, on_step=on_step, max_steps=steps,
                          cache_all_slots=n_ctx > 1, frame_pool=frame_pool, fresh_t=fresh_t)
    t1.record(stream)
    torch.cuda.synchronize()
    mod_ms, attn_ms, adv_ms, n_prof = dp.profile_end()
    clocks = sampler.stop() if sampler else None
    # per-step times of the full-window (steady-state) steps, early and late in the run: the
    # step's work depends on the block size, not on how much video came before
    step_ms = [(step_ev[i - 1] if i else t0).elapsed_time(step_ev[i]) for i in range(len(step_ev))]
    full = [i for i, nn in enumerate(steps_n) if nn == max(steps_n)]
    steady = {}
    if len(full) >= 6:
        third = len(full) // 3
        pick = lambda idx: sorted(step_ms[i] for i in idx)
        allv = pick(full)
        steady = {"steps": len(full), "median_ms": statistics.median(allv),
                  "p05_ms": allv[len(allv) // 20], "p95_ms": allv[(19 * len(allv)) // 20],
                  "first_third_median_ms": statistics.median(pick(full[:third])),
                  "last_third_median_ms": statistics.median(pick(full[-third:]))}
    if world > 1:
        dist.barrier()
    dp.device_status()
    ms = t0.elapsed_time(t1)
    tokens = sum(steps_n)
    flop = sum(4 * n * (lc + n) * hd * H for n, lc in zip(steps_n, steps_lc))
    if not with_e2e:
        ms, attn_ms = max_over_ranks([ms, attn_ms], dev)
        return dict(ms=ms, steps=n_steps, tokens=tokens, flop=flop, attn_ms=attn_ms, mod_ms=mod_ms, adv_ms=adv_ms,
                    clocks=clocks, rc=rc, launches=launches[0], n_ctx=n_ctx, fresh=fresh_t is not None,
                    steady=steady)

    # e2e: the same run through the public API with every pushed noise block copied from
    # pinned host memory right before its push and every step's output read back to the host
    class _HostBlocks:
        def __init__(self, blocks):
            self.host = [b.pin_memory() for b in blocks]
            self.dev = torch.empty(rc.slot_rows, D, dtype=torch.bfloat16, device=dev)
            self.h2d = 0

        def __len__(self):
            return len(self.host)

        def __getitem__(self, i):
            h = self.host[i]
            self.dev[:h.shape[0]].copy_(h, non_blocking=True)
            self.h2d += h.numel() * 2
            return self.dev[:h.shape[0]]

    hb = _HostBlocks(noise_cpu)
    # each step's output is read back on a copy stream while the next step computes: the
    # steps alternate between two output buffers, and a step waits for the readback of the
    # buffer it is about to overwrite
    outs = [out, torch.empty_like(out)]
    houts = [torch.empty(n_max, D, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    d2h_stream = torch.cuda.Stream(dev)
    read_done = [None, None]
    d2h = [0]

    def on_step_e2e(step, n, popped, pushed):
        slot = step % 2
        done = torch.cuda.Event()
        done.record(stream)
        d2h_stream.wait_event(done)
        with torch.cuda.stream(d2h_stream):
            houts[slot][:n].copy_(outs[slot][:n], non_blocking=True)
        ev = torch.cuda.Event()
        ev.record(d2h_stream)
        read_done[slot] = ev
        if read_done[1 - slot] is not None:
            stream.wait_event(read_done[1 - slot])
        d2h[0] += n * D * 2

    cache, queue = new_state()
    e2e_pool = None
    if frame_pool is not None:   # the pool is the run's input: copied from pinned host memory once
        hpool = frame_pool[0].cpu().pin_memory()
        dpool = torch.empty_like(frame_pool[0])
        hb.h2d = hpool.numel() * 2
        e2e_pool = (dpool, frame_pool[1])
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if e2e_pool is not None:
        e2e_pool[0].copy_(hpool, non_blocking=True)
    n_e2e = dp.run_fifo(hb, table, tau, W, cache, queue, kv, outs, H, hd, on_step=on_step_e2e,
                        max_steps=steps, cache_all_slots=n_ctx > 1, frame_pool=e2e_pool, fresh_t=fresh_t)
    for ev in read_done:
        if ev is not None:
            stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    dp.device_status()
    ms, e2e_ms, attn_ms = max_over_ranks([ms, e2e_ms, attn_ms], dev)
    return dict(ms=ms, steps=n_steps, tokens=tokens, flop=flop, attn_ms=attn_ms, mod_ms=mod_ms, adv_ms=adv_ms,
                e2e_ms=e2e_ms, e2e_steps=n_e2e, h2d=hb.h2d / max(n_e2e, 1), d2h=d2h[0] / max(n_e2e, 1),
                clocks=clocks, rc=rc, launches=launches[0], n_ctx=n_ctx, fresh=fresh_t is not None, steady=steady)


def long_run_line(args, world, r, config: str = None):
    peaks = load_peaks()
    config = config or args.config
    rc = r["rc"]
    achieved = r["flop"] / (r["attn_ms"] / 1e3) / 1e12
    pk = choose_peak(peaks, r["clocks"], r["ms"] / 1e3)
    steady_flop = 4 * 21600 * (21600 + r["n_ctx"] * 2700) * rc.head_dim * rc.n_heads
    return {
        "metric": METRIC, "value": world * r["tokens"] / (r["ms"] / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": r["steps"], "warmup": args.warmup, "ms_per_step": r["ms"] / r["steps"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": (f"{config}: {rc.n_frames} latent frames x {rc.frame_rows} tokens in "
                                f"{rc.frames_per_block}-frame blocks, window of {rc.window_blocks} blocks, "
                                f"{rc.n_timesteps} staggered timesteps per block, {rc.n_heads}x{rc.head_dim} heads, "
                                f"bf16, cache of the last {r['n_ctx']} exited block(s)"
                                + ("; context K/V recomputed before every step (timestep 0)" if r["fresh"] else "")
                                + f"; first {r['steps']} schedule steps"),
                   "parallelism": f"replicas x{world} (no exchange)",
                   "l2": "steady-state window q = k = v 66 MiB plus k', v', cache and out: 265 MiB per step > 126 MiB"},
        "window_tokens": r["tokens"],
        "full_window_step_ms": r["steady"],
        "attn_tflops": achieved,
        "stage_ms": {"modulate": r["mod_ms"] / r["steps"], "attention": r["attn_ms"] / r["steps"],
                     "advance": r["adv_ms"] / r["steps"],
                     "outside_stages": (r["ms"] - r["mod_ms"] - r["attn_ms"] - r["adv_ms"]) / r["steps"]},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["peak"], "unit": "TFLOP/s",
                     **roofline_fracs(achieved, pk), "traffic": None,
                     "traffic_unit": "bytes per launch (not captured for the run: window sizes vary per step)",
                     "kernel": "window_attn_tc_kernel", "peak_kind": pk["kind"], "peak_why": pk["why"],
                     "algorithmic_flop_per_run": r["flop"], "steady_state_flop_per_launch": steady_flop},
        "clocks": r["clocks"],
        "e2e": ({"value": world * r["tokens"] / (r["e2e_ms"] / 1e3), "unit": "tokens/s",
                 "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]} if "e2e_ms" in r else None),
        "gpu_launches": r["launches"],
    }


def sublayer_arm(args, rank: int, world: int, local_rank: int):
    """The DiT attention sublayer step on the window: pre-LN with adaLN modulation, q/k/v
    projection (tensor cores), window attention over [cache ; window], out projection with
    the gated residual, and the advance (head block's k, v -> cache, noise pushed).  The
    ``sublayer_fresh_*`` workloads recompute the context's k, v before every step (pre-LN of
    the context rows conditioned on timestep 0, then the k/v projection) instead of reusing
    the cached ones: the cost side of the cache's staleness ablation."""
    import torch
    import torch.distributed as dist

    import long_video_diffusion_b200 as dp
    from workloads import as_features, make_step_inputs, make_sublayer_weights

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = workload(args.config)
    x_in = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    wts = {k: t.to(dev) for k, t in make_sublayer_weights(D, cfg.seed + 100).items()}
    blk = dp.blocks_from_table(x_in["table"].to(dev), x_in["timesteps"], cfg.block_rows)
    x = x_in["q"].to(dev)
    noise = x_in["noise"].to(dev)
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float16,
                       k=as_features(x_in["cache_k"], cfg.dtype).to(dev).view(1, -1, D),
                       v=as_features(x_in["cache_v"], cfg.dtype).to(dev).view(1, -1, D), length=cfg.cache_len)
    queue = dp.Queue(cfg.n_blocks, max(cfg.block_rows), D, device=dev)
    for _ in range(cfg.n_blocks):
        dp.queue_push(queue, noise)
    work = dp.sublayer_work(n, D, device=dev)
    out = torch.empty(n, D, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    fresh = args.config.startswith("sublayer_fresh_")
    n_ctx = cfg.cache_len
    x_ctx = x[:n_ctx].clone()                 # the context block's rows, resident like the cache
    ctx_blk = dp.blocks_from_table(x_in["table"].to(dev), [0], [n_ctx])
    ref_ev = []

    def refresh(strm=None, timed=False):
        if timed:
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            e[0].record(stream)
        dp.context_refresh_sublayer(x_ctx, ctx_blk, wts["w_qkv"], wts["b_qkv"], cache, work, stream=strm)
        if timed:
            e[1].record(stream)
            ref_ev.append(e)

    def step(xx=x, nz=noise, timed=False):
        if fresh:
            refresh(timed=timed)
        dp.sublayer_step(xx, blk, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], cache, work, out, H, hd,
                         pop=True, queue=queue, push_noise=nz)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dp.device_status()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(_smi_index(local_rank)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    dp.profile_begin(args.steps)
    t0.record(stream)
    for _ in range(args.steps):
        step(timed=True)
    t1.record(stream)
    torch.cuda.synchronize()
    stages, _, n_prof = dp.profile_end_stages(5)
    refresh_ms = sum(a.elapsed_time(b) for a, b in ref_ev) / len(ref_ev) if ref_ev else None
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    dp.device_status()
    ms = t0.elapsed_time(t1)
    stages = [v / n_prof for v in stages]

    # e2e through the public API from pinned host memory, copies overlapped with the
    # previous step's compute (StepPipeline)
    hx, hnoise = x_in["q"].pin_memory(), x_in["noise"].pin_memory()
    hout = torch.empty(n, D, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    pipe = dp.StepPipeline(n, D, noise.shape[0], device=dev, shapes=[(n, D), tuple(noise.shape)])

    def run(d, dout, strm):
        if fresh:
            refresh(strm)
        dp.sublayer_step(d[0], blk, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], cache, work, dout, H, hd,
                         pop=True, queue=queue, push_noise=d[1], stream=strm)

    def e2e_step():
        pipe.submit_with([hx, hnoise], hout, run)

    for _ in range(3):
        e2e_step()
    pipe.finish()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.h2d)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(pipe.d2h)
    pipe.finish()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    dp.device_status()
    vals = max_over_ranks([ms, e2e_ms] + stages + [refresh_ms or 0.0], dev)
    refresh_ms = vals[-1] if fresh else None
    vals = vals[:-1]
    return cfg, dict(ms=vals[0], e2e_ms=vals[1], e2e_steps=e2e_steps, stages=vals[2:], clocks=clocks,
                     h2d=(hx.numel() + hnoise.numel()) * 2, d2h=hout.numel() * 2,
                     refresh_ms=refresh_ms, n_ctx=n_ctx if fresh else 0)


def sublayer_line(args, world, cfg, r):
    peaks = load_peaks()
    n, D, H, hd = cfg.n_win, cfg.hidden, cfg.n_heads, cfg.head_dim
    ln_ms, qkv_ms, attn_ms, out_ms, adv_ms = r["stages"]
    attn_flop = cfg.attn_flop()
    qkv_flop = 2 * n * D * 3 * D
    out_flop = 2 * n * D * D
    pk = choose_peak(peaks, r["clocks"], r["ms"] / 1e3)
    peak = pk["peak"]
    tf = lambda flop, ms: flop / (ms / 1e3) / 1e12 if ms > 0 else None
    achieved = tf(attn_flop, attn_ms)
    ln_bytes = 2 * n * D * 2
    adv_bytes = (4 * cfg.block_rows[0] + 2 * cfg.push_rows) * D * 2
    gbs = lambda b, ms: b / (ms / 1e3) / 1e9 if ms > 0 else None
    ms_step = r["ms"] / args.steps
    n_ctx = r["n_ctx"]
    fresh_text = (f"; context k, v recomputed before every step (pre-LN + k/v projection of {n_ctx} context rows)"
                  if n_ctx else "")
    line = {
        "metric": METRIC, "value": job_throughput(world, n, args.steps, r["ms"]), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "DiT attention sublayer step (pre-LN + adaLN, q/k/v projection, window attention, "
                               "out projection with gated residual, advance; synthetic weights) on " + describe(cfg)
                               + fresh_text,
                   "parallelism": f"replicas x{world} (no exchange)",
                   "l2": f"inputs larger than L2 (x, W_qkv, W_o {(n * D + 4 * D * D) * 2 / 2**20:.0f} MiB "
                         f"> {L2_BYTES / 2**20:.0f} MiB)"},
        "attn_tflops": achieved,
        "stage_ms": {"ln_modulate": ln_ms, "qkv_projection": qkv_ms, "attention": attn_ms,
                     "out_projection": out_ms, "advance": adv_ms},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     **roofline_fracs(achieved, pk), "traffic": None,
                     "traffic_unit": "bytes per launch (see the window-step configurations)",
                     "kernel": "window_attn_tc_kernel", "peak_kind": pk["kind"], "peak_why": pk["why"],
                     "algorithmic_flop_per_launch": attn_flop},
        "stage_tensor": {
            "qkv_projection": {"flop": qkv_flop, "ms": qkv_ms, "achieved_tflops": tf(qkv_flop, qkv_ms),
                               "frac": (tf(qkv_flop, qkv_ms) or 0) / peak},
            "out_projection": {"flop": out_flop, "ms": out_ms, "achieved_tflops": tf(out_flop, out_ms),
                               "frac": (tf(out_flop, out_ms) or 0) / peak}},
        "stage_hbm": {
            "ln_modulate": {"bytes": ln_bytes, "ms": ln_ms, "achieved_gbs": gbs(ln_bytes, ln_ms),
                            "frac": (gbs(ln_bytes, ln_ms) or 0) / peaks["hbm_gbs"]},
            "advance": {"bytes": adv_bytes, "ms": adv_ms, "achieved_gbs": gbs(adv_bytes, adv_ms),
                        "frac": (gbs(adv_bytes, adv_ms) or 0) / peaks["hbm_gbs"],
                        "mirror_write_bytes": cfg.push_rows * D * 2,
                        "note": "bytes = 4 n_exit D e + 2 n_push D e (algorithmic); the push's second write into "
                                "the mirrored latent ring (mirror_write_bytes) is overhead, not counted"}},
        "clocks": r["clocks"],
        "e2e": {"value": world * n / (r["e2e_ms"] / r["e2e_steps"] / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": (7 if n_ctx else 5) * args.steps,
    }
    if n_ctx:
        kv_flop = 2 * n_ctx * D * 2 * D
        ref_ms = r["refresh_ms"]
        line["stage_ms"]["context_refresh"] = ref_ms
        line["stage_tensor"]["context_refresh"] = {
            "flop": kv_flop, "ms": ref_ms, "achieved_tflops": tf(kv_flop, ref_ms),
            "frac": (tf(kv_flop, ref_ms) or 0) / peak,
            "note": "pre-LN of the context rows plus their k/v projection, timed together"}
    return line


def oracle_sublayer_sample(cfg, x, wts, n_rows: int, head: int, seed: int, fresh: bool = False):
    """One oracle sublayer step on a bounded sample: the pre-norm of all rows, the q/k/v
    projection of all rows for one head's columns, that head's attention for n_rows random
    query rows, and the out projection of those rows.  Returns (seconds, seconds
    extrapolated to the whole step): per-head parts times the head count, per-row parts
    times n_win / n_rows.  ``fresh``: the context's k, v are first recomputed whole (pre-norm
    and k/v projection of the context rows, conditioned on timestep 0) and the attention
    reads them."""
    import numpy as np

    import oracle as O
    from workloads import as_features
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(cfg.n_win, size=min(n_rows, cfg.n_win), replace=False))
    D, hd, H = cfg.hidden, cfg.head_dim, cfg.n_heads
    c0, c1 = head * hd, (head + 1) * hd
    mod = O.lookup(x["table"], x["timesteps"])
    ck = as_features(x["cache_k"], cfg.dtype)[:, c0:c1]
    cv = as_features(x["cache_v"], cfg.dtype)[:, c0:c1]
    wq = O.as_f64(wts["w_qkv"])
    t_ctx = 0.0
    if fresh:
        tc = time.perf_counter()
        n_ctx = cfg.cache_len
        fk, fv = O.fresh_context_sublayer(x["q"][:n_ctx], [0, n_ctx], O.lookup(x["table"], [0]), wts["w_qkv"],
                                          wts["b_qkv"], 1e-6)
        ck, cv = fk[:, c0:c1], fv[:, c0:c1]
        t_ctx = time.perf_counter() - tc
    t0 = time.perf_counter()
    h = O.round_to(O.ln_modulate(x["q"], cfg.row_offset, mod, 1e-6), "bf16")
    t1 = time.perf_counter()
    cols = np.concatenate([np.arange(c0, c1), D + np.arange(c0, c1), 2 * D + np.arange(c0, c1)])
    qkv = O.linear(h, wq[cols], O.as_f64(wts["b_qkv"])[cols])
    q, k, v = qkv[:, :hd], qkv[:, hd:2 * hd], qkv[:, 2 * hd:]
    t2 = time.perf_counter()
    o = O.window_attention(q, k, v, ck, cv, cfg.cache_len, cfg.row_offset, mod[:, :, c0:c1], 1, hd,
                           mod_q=False, gate_out=False, rows=rows)
    t3 = time.perf_counter()
    o_all = np.tile(o, (1, H))
    O.linear(o_all, wts["w_o"], wts["b_o"])
    t4 = time.perf_counter()
    full = (t1 - t0) + (t2 - t1) * H + (t3 - t2) * H * cfg.n_win / len(rows) + (t4 - t3) * cfg.n_win / len(rows)
    return t4 - t0 + t_ctx, full + t_ctx


def sublayer_cpu_baseline(cfg, budget_s: float = 12.0, fresh: bool = False):
    from workloads import make_step_inputs, make_sublayer_weights
    x = make_step_inputs(cfg)
    wts = make_sublayer_weights(cfg.hidden, cfg.seed + 100)
    spent, fulls, i = 0.0, [], 0
    n_rows = 64
    while (spent < budget_s or i < 2) and i < 2 * cfg.n_heads:
        s, full = oracle_sublayer_sample(cfg, x, wts, n_rows, head=i % cfg.n_heads, seed=i, fresh=fresh)
        spent += s
        fulls.append(full)
        i += 1
    t = statistics.median(fulls)
    return {"value": cfg.n_win / t, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": (f"{i} oracle sublayer steps, each: the pre-norm of all {cfg.n_win} rows, the q/k/v projection "
                       f"of all rows for one head's columns (scaled by {cfg.n_heads} heads), that head's attention for "
                       f"{n_rows} random rows over all {cfg.cache_len + cfg.n_win} keys and the out projection of those "
                       f"rows (scaled linearly to all rows)"
                       + (f", after recomputing the {cfg.cache_len} context rows' k, v whole" if fresh else "")
                       + f"; {spent:.1f} s of CPU work")}


def stage_hbm(cfg, r, peaks):
    """Achieved HBM bandwidth of the two copy-like stages (algorithmic bytes / event time):
    modulation reads k, v and writes k', v' (4 N_w D e bytes); the advance copies the head
    block's k'/v' into the cache (4 n_exit D e) and pushes the noise block (read and write,
    2 n_push D e).  The push also writes the block a second time, into the mirror half of the
    latent ring (n_push D e): overhead of the layout, reported apart and not counted."""
    eb = cfg.elem_bytes
    mod_b = 4 * cfg.n_win * cfg.hidden * eb
    adv_b = (4 * cfg.block_rows[0] + 2 * cfg.push_rows) * cfg.hidden * eb
    out = {}
    for name, b, ms in (("modulate", mod_b, r["mod_ms"]), ("advance", adv_b, r["adv_ms"])):
        gbs = b / (ms / 1e3) / 1e9 if ms > 0 else None
        out[name] = {"bytes": b, "ms": ms, "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
                     "frac": (gbs / peaks["hbm_gbs"]) if gbs else None}
    out["advance"]["mirror_write_bytes"] = cfg.push_rows * cfg.hidden * eb
    # the same kernels alone (no launch gap, no power-capped clock inherited from the attention):
    # the prepass over k and v, and the advance's cache write (the head block's k', v')
    for name, b, key in (("modulate_alone", mod_b, "mod_alone_ms"),
                         ("advance_cache_alone", 4 * cfg.block_rows[0] * cfg.hidden * eb, "adv_alone_ms")):
        if key in r and r[key] > 0:
            gbs = b / (r[key] / 1e3) / 1e9
            out[name] = {"bytes": b, "ms": r[key], "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
                         "frac": gbs / peaks["hbm_gbs"]}
    return out


def max_over_ranks(values, device=None):
    """Element-wise maximum of per-rank timings (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor(values, dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world: int, n_win: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own window per step (weak scaling)."""
    return world * n_win * steps / (max_ms / 1e3)


def _smi_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [s.strip() for s in vis.split(",") if s.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ----------------------------------------------------------------------------- CPU oracle

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_step(cfg, x, n_rows: int, head: int, seed: int):
    """One oracle window step on a bounded sample: head `head` only (heads are independent:
    its K/V modulation over all window rows, its attention for n_rows random query rows over
    all keys).  Returns (seconds, seconds extrapolated to the whole step: attention scaled
    linearly to all rows, everything scaled by the head count)."""
    import numpy as np

    import oracle as O
    from workloads import as_features
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(cfg.n_win, size=min(n_rows, cfg.n_win), replace=False))
    c0, c1 = head * cfg.head_dim, (head + 1) * cfg.head_dim
    sl = lambda t: t[:, c0:c1].contiguous()
    x = dict(x, cache_k=as_features(x["cache_k"], cfg.dtype), cache_v=as_features(x["cache_v"], cfg.dtype))
    mod = O.lookup(x["table"][:, :, c0:c1].contiguous(), x["timesteps"])
    q, k, v, ck, cv = sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["cache_k"]), sl(x["cache_v"])
    t0 = time.perf_counter()
    kp = O.modulate(k, cfg.row_offset, mod)
    vp = O.modulate(v, cfg.row_offset, mod)
    t1 = time.perf_counter()
    O.window_attention(q, kp, vp, ck, cv, cfg.cache_len, cfg.row_offset, mod, 1, cfg.head_dim, rows=rows)
    t2 = time.perf_counter()
    full = ((t1 - t0) + (t2 - t1) * cfg.n_win / len(rows)) * cfg.n_heads
    return t2 - t0, full, len(rows)


def _sample_text(cfg, n_rows):
    return (f"one head of {cfg.n_heads} per oracle step (heads are independent): its K/V modulation over all "
            f"{cfg.n_win} window rows and its attention for {n_rows} random query rows over all "
            f"{cfg.cache_len + cfg.n_win} keys; attention time scaled linearly to all rows, the step's time "
            f"scaled by the head count")


def cpu_baseline(cfg, budget_s: float = 12.0):
    from workloads import make_step_inputs
    x = make_step_inputs(cfg)
    spent, fulls, i = 0.0, [], 0
    n_rows = 64
    while (spent < budget_s or i < 3) and i < 4 * cfg.n_heads:
        s, full, _ = oracle_sample_step(cfg, x, n_rows, head=i % cfg.n_heads, seed=i)
        spent += s
        fulls.append(full)
        i += 1
    t = statistics.median(fulls)
    return {"value": cfg.n_win / t, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{i} oracle steps; " + _sample_text(cfg, n_rows) + f"; {spent:.1f} s of CPU work"}


def reference_arm(args):
    """The oracle as the reference arm: W untimed + K timed bounded-sample steps."""
    from workloads import make_step_inputs, make_sublayer_weights
    cfg = workload(args.config)
    x = make_step_inputs(cfg)
    n_rows = 16
    if args.config.startswith("sublayer_"):
        wts = make_sublayer_weights(cfg.hidden, cfg.seed + 100)
        fresh = args.config.startswith("sublayer_fresh_")
        sample = lambda i, seed: oracle_sublayer_sample(cfg, x, wts, n_rows, head=i % cfg.n_heads, seed=seed,
                                                        fresh=fresh)[1]
        text = "each step: one head's share of an oracle sublayer step (see cpu_baseline of the ours arm)"
    else:
        sample = lambda i, seed: oracle_sample_step(cfg, x, n_rows, head=i % cfg.n_heads, seed=seed)[1]
        text = "each step: " + _sample_text(cfg, n_rows)
    for i in range(args.warmup):
        sample(i, 1000 + i)
    fulls = []
    for i in range(args.steps):
        fulls.append(sample(i, i))
    ms = 1e3 * statistics.mean(fulls)
    value = cfg.n_win / (ms / 1e3)
    cores = _blas_threads()
    sample = text
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": describe(cfg) + ("; context k, v recomputed before every step"
                                                    if args.config.startswith("sublayer_fresh_") else "")},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def step_line(args, world, cfg, r, config: str):
    """The JSON record of a window-step workload (the main line, or one of target_configs)."""
    peaks = load_peaks()
    flop = cfg.attn_flop()
    steps = r["steps"]
    achieved = flop / (r["attn_ms"] / 1e3) / 1e12
    pk = choose_peak(peaks, r["clocks"], r["ms"] / 1e3)
    line = {
        "metric": METRIC, "value": job_throughput(world, cfg.n_win, steps, r["ms"]), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": r["ms"] / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(cfg), "parallelism": f"replicas x{world} (no exchange)",
                   "l2": f"inputs larger than L2 (q, k, v {3 * cfg.n_win * cfg.hidden * 2 / 2**20:.0f} MiB "
                         f"> {L2_BYTES / 2**20:.0f} MiB)"},
        "attn_tflops": achieved,
        "stage_ms": {"modulate": r["mod_ms"], "attention": r["attn_ms"], "advance": r["adv_ms"]},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["peak"], "unit": "TFLOP/s",
                     **roofline_fracs(achieved, pk), "traffic": attention_traffic(config),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "kernel": "window_attn_tc_kernel", "peak_kind": pk["kind"], "peak_why": pk["why"],
                     "algorithmic_flop_per_launch": flop},
        "stage_hbm": stage_hbm(cfg, r, peaks),
        "clocks": r["clocks"],
        "gpu_launches": 3 * steps,
    }
    if "e2e_ms" in r:
        line["e2e"] = {"value": world * cfg.n_win / (r["e2e_ms"] / r["e2e_steps"] / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]}
    return line


def compact(line):
    """The figures of a target_configs entry."""
    rf = line["roofline"]
    out = {"workload": line["config"]["workload"], "value": line["value"], "unit": line["unit"],
           "steps": line["steps"], "ms_per_step": line["ms_per_step"], "attn_tflops": line["attn_tflops"],
           "attention_ms_per_step": line["stage_ms"]["attention"],
           "roofline": {k: rf[k] for k in ("achieved", "peak", "frac", "frac_of_burst", "frac_of_sustained",
                                           "peak_kind", "peak_why", "traffic") if k in rf},
           "clocks": line["clocks"]}
    if "full_window_step_ms" in line:
        out["full_window_step_ms"] = line["full_window_step_ms"]
    if "stage_hbm" in line:
        out["stage_hbm"] = {k: {"achieved_gbs": v["achieved_gbs"], "frac": v["frac"]}
                            for k, v in line["stage_hbm"].items()}
    return out


def extra_lines(args, rank: int, world: int, local_rank: int):
    """The other target workloads, each timed in its own region: the Wan-like window, the long
    run's steady-state window and the whole long run (no e2e or CPU baseline for these)."""
    out = {}
    for name in EXTRA_CONFIGS:
        if name == "long_run":
            r = long_run_arm(args, rank, world, local_rank, config=name, steps=850, with_e2e=False)
            if rank == 0:
                out[name] = compact(long_run_line(args, world, r, config=name))
        else:
            cfg, r = gpu_arm(args, rank, world, local_rank, config=name, steps=DEFAULT_STEPS[name], with_e2e=False)
            if rank == 0:
                out[name] = compact(step_line(args, world, cfg, r, name))
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the target_configs timings of the default run")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    default_run = args.config is None
    if args.config is None:
        args.config = DEFAULT_CONFIG
    if args.steps is None:
        args.steps = 850 if args.config.startswith("long_run") else DEFAULT_STEPS.get(args.config, 300)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    if args.config in ("long_run", "long_run_ctx4", "long_run_coord", "long_run_fresh"):
        r = long_run_arm(args, rank, world, local_rank)
        if rank == 0:
            line = long_run_line(args, world, r)
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(workload("long_run"))
                line["cpu_baseline"]["sample"] = "steady-state step of the run: " + line["cpu_baseline"]["sample"]
            print(json.dumps(line), flush=True)
    elif args.config.startswith("sublayer_"):
        cfg, r = sublayer_arm(args, rank, world, local_rank)
        if rank == 0:
            line = sublayer_line(args, world, cfg, r)
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = sublayer_cpu_baseline(cfg, fresh=args.config.startswith("sublayer_fresh_"))
            print(json.dumps(line), flush=True)
    else:
        cfg, r = gpu_arm(args, rank, world, local_rank)
        line = step_line(args, world, cfg, r, args.config) if rank == 0 else None
        extras = extra_lines(args, rank, world, local_rank) if default_run and not args.no_extra else None
        if rank == 0:
            if extras:
                line["target_configs"] = extras
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(cfg)
            print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
