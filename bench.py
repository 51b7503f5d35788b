"""Batch-1 decode benchmark: µs/token and achieved HBM GB/s of the persistent
decode megakernel on B200, next to the fp64 CPU oracle.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference]

One "step" = one decode step of the whole forward pass (one cooperative
launch), greedy, token chained on the device.  The default workload is the
Llama-7B-shaped bf16 decoder decoding at KV context 2048 (13.2 GB of weights
+ 1.07 GB of KV read per token: larger than L2, so no flush is needed).
Every step decodes at position = context (the row is rewritten each step).

The timing is printed only beside a PASS parity verdict from the same run
(the first step's logits against the oracle), after the honesty rule of
"RightNow-AI/AutoMegaKernel" README, "Honesty rules": no latency without a
paired correctness verdict.

Multi-GPU: batch-1 decode does not shard; N GPUs run N independent replicas
(one rank per GPU, no data-path collective).  value = whole-job time per
token = max-over-ranks elapsed / (N * K).

--impl reference times the fp64 oracle (the only reference implementation
this path has) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth_inputs as si  # noqa: E402

METRIC = "batch-1 decode us/token"
UNIT = "us/token"

# name -> (model config, KV context)
WORKLOADS = {
    "llama7b-ctx2048": ("llama7b", 2048),
    "llama7b-ctx0": ("llama7b", 0),
    "llama7b_w8-ctx2048": ("llama7b_w8", 2048),
    "llama7b_w8-ctx0": ("llama7b_w8", 0),
    "tinyllama-ctx0": ("tinyllama", 0),
    "tinyllama-ctx1024": ("tinyllama", 1024),
    "llama1b_w8-ctx0": ("llama1b_w8", 0),
    "llama1b_w8-ctx512": ("llama1b_w8", 512),
    "smol135_w4-ctx0": ("smol135_w4", 0),
    "llama7b_w4-ctx2048": ("llama7b_w4", 2048),
    "smol135-ctx0": ("smol135", 0),
    "smol135-ctx128": ("smol135", 128),
    "tiny-ctx4": ("tiny", 4),
}
DEFAULT_WORKLOAD = "llama7b-ctx2048"
KERNEL_SOURCES = ["persistent_megakernel_decode_cta_b200/csrc/amk_kernel_body.cuh",
                  "persistent_megakernel_decode_cta_b200/csrc/amk_internal.h"]


def algorithmic_bytes(cfg, ctx: int) -> int:
    """Bytes one decode step must move: every weight byte once (int8 scales,
    norm gains, one embedding row and the LM head -- the embedding table when
    tied -- included), the KV rows 0..ctx-1 of every layer, the new K/V row,
    and the logits."""
    kv_row = 2 * cfg.n_layers * cfg.n_kv_heads * cfg.head_dim * 2
    return si.streamed_weight_bytes(cfg) + kv_row * ctx + kv_row + cfg.vocab * 4


def kernel_hash(sources=None) -> str:
    """Hash of the kernel's code: the sources with their comments and blank
    space removed, so that a profile stays attached to the code it measured
    when only the commentary changes."""
    h = hashlib.sha256()
    for p in (sources or [os.path.join(ROOT, q) for q in KERNEL_SOURCES]):
        text = open(p, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on this workload with the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_hash():
        return None
    return e.get("dram_bytes_per_launch")


def measured_peak():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            try:
                gid = "GPU-" + str(torch.cuda.get_device_properties(self.gpu).uuid)
            except Exception:
                gid = str(self.gpu)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for ln in (self.out or "").strip().splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5], f[6], f[7], f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, v in zip(names, r[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "reasons": sorted(reasons), "samples": len(rows)}


def dist_env(n_gpus: int):
    """(world, rank, local rank) from the launcher's environment; the world
    size must equal --gpus."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One rank per GPU.  The process group carries only the barriers and the
    max-over-ranks reductions of the timing (replicas share no data)."""
    world, rank, local = dist_env(n_gpus)
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_token(elapsed_ms: float, steps: int, world: int) -> float:
    """Whole-job time per token: `world` replicas each decode `steps` tokens
    within the slowest rank's `elapsed_ms`."""
    return elapsed_ms * 1e3 / (steps * world)


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_steps(cfg, weights, ctx, kv_fill, budget_s: float, max_steps: int, threads: int = 0):
    """Times full fp64 oracle decode steps at position ctx (as many as fit the
    budget, at least one) on `threads` OpenMP threads (0: all host cores).
    Returns (us per token, steps, threads, logits of the first step)."""
    import oracle
    m = oracle.OracleModel(cfg, weights)
    threads = oracle.set_threads(threads if threads > 0 else (os.cpu_count() or 1))
    if kv_fill is not None:
        m.fill_kv(kv_fill)
    tok = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
    times, first = [], None
    t_all = time.perf_counter()
    while len(times) < max_steps:
        t0 = time.perf_counter()
        logits, am, _ = m.step(tok, ctx)
        times.append(time.perf_counter() - t0)
        if first is None:
            first = logits
        tok = am
        if time.perf_counter() - t_all > budget_s:
            break
    return statistics.median(times) * 1e6, len(times), threads, first


KINDS = {1: "qkv", 2: "attn", 3: "oproj", 4: "gateup", 5: "down", 6: "lmhead", 7: "ffn"}


def phase_shares(P):
    """Where the consumers' time goes, from the kernel's phase timers of one
    step (uint64 [n_sms, kinds, fields]; amk_get_profile): shares of the
    consumer warpgroups' time from kernel start to their end, summed over
    SMs, and the producer lane's share of time stalled on a full ring or the
    in-flight cap."""
    P = P.astype(np.float64)
    total = float((P[:, 0, 1] - P[:, 0, 0]).sum())
    prod = float((P[:, 0, 3] - P[:, 0, 0]).sum())
    # waits for a task's inputs: counter polls (field 1) or, with flagged
    # waits, thread 0's polls of the flagged words (field 3)
    wait = float(P[:, 1:, 1].sum()) + float(P[:, 1:, 3].sum())
    prologue = float(P[:, 1:, 2].sum())
    ring = float(P[:, 1:, 6].sum()) / 8.0
    compute = float(P[:, 1:, 7].sum()) / 8.0
    run = float(P[:, 1:, 4].sum())
    epi = float(P[:, 1:, 5].sum())
    per_kind = {}
    for k, name in KINDS.items():
        n = float(P[:, k, 0].sum())
        if n == 0:
            continue
        f = P[:, k, :].sum(axis=0) / n / 1e3
        per_kind[name] = {"tasks": int(n), "counter_wait_us": f[1] + f[3], "prologue_us": f[2],
                          "ring_wait_us": f[6] / 8.0, "gemv_or_attention_us": f[7] / 8.0,
                          "epilogue_release_us": f[5], "run_us": f[4]}
    return {
        "counter_wait": wait / total, "prologue": prologue / total,
        "ring_wait": ring / total, "gemv_or_attention": compute / total,
        "epilogue_release": epi / total,
        "other": max(0.0, 1.0 - (float(P[:, 1:, 1].sum()) + run) / total),
        "producer_stalled": float(P[:, 0, 2].sum()) / prod if prod > 0 else None,
        "per_task_kind_us": per_kind,
        "how": "phase timers (globaltimer) of one profiled step after the timed region; "
               "shares of the consumer warpgroups' time, summed over SMs",
    }


def run_reference(args):
    # rank 0 alone times the oracle; no process group is needed for that
    world, rank, _ = dist_env(args.gpus)
    if rank != 0:
        return
    name = args.workload
    mname, ctx = WORKLOADS[name]
    cfg = si.get_config(mname)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = si.make_model(cfg, seed=0, device=dev)
    kv = si.make_kv_fill(cfg, ctx, device=dev) if ctx else None
    budget = float(os.environ.get("AMK_REF_BUDGET_S", "120"))
    us, n, threads, _ = oracle_steps(cfg, w, ctx, kv, budget, args.steps + args.warmup)
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(name, cfg, ctx),
        "cpu_baseline": {"value": us, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{n} full fp64 decode steps of {name} (of "
                                   f"{args.steps + args.warmup} requested; {budget:.0f} s cap)"},
        "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(name, cfg, ctx):
    return {"workload": f"{name}: random-init {cfg.name}-shaped decoder, batch 1, "
                        f"greedy decode at KV context {ctx}",
            "hidden": cfg.hidden, "layers": cfg.n_layers, "heads": cfg.n_heads,
            "kv_heads": cfg.n_kv_heads, "head_dim": cfg.head_dim, "ffn": cfg.ffn,
            "vocab": cfg.vocab, "kv_context": ctx, "weights": cfg.quant,
            "tied_embeddings": cfg.tied, "global_batch": 1,
            "l2": "inputs larger than L2 (weights streamed every step)"
            if si.model_bytes(cfg)["linear"] > 126e6 else "weights fit in L2"}


def run_ours(args):
    import persistent_megakernel_decode_cta_b200 as amk
    from persistent_megakernel_decode_cta_b200 import build as amk_build
    world, rank, local = dist_setup(args.gpus)
    if rank == 0:
        amk_build.build()
    barrier(world)
    name = args.workload
    mname, ctx = WORKLOADS[name]
    cfg = si.get_config(mname)
    if ctx + 2 > cfg.max_ctx:
        raise SystemExit("context too large for the config")
    w = si.make_model(cfg, seed=0, device="cuda")
    kv = si.make_kv_fill(cfg, ctx, device="cuda") if ctx else None
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    opts = amk.default_options()
    with torch.cuda.stream(stream):
        dec = amk.Decoder(cfg, w, opts, stream=stream.cuda_stream)

    def fill():
        if kv is None:
            return
        for l in range(cfg.n_layers):
            k, v = dec.kv(l)
            k[:, :ctx].copy_(kv[l, 0])
            v[:, :ctx].copy_(kv[l, 1])
        torch.cuda.synchronize()

    fill()
    tok0 = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")

    # ---- parity gate on the first step (rank 0 also times the oracle) -------
    dec.step(tok0, ctx, logits=logits)
    g = logits.double().cpu().numpy()
    parity, cpu_base = None, None
    if rank == 0:
        budget = float(os.environ.get("AMK_CPU_BUDGET_S", "20"))
        us, n, threads, ref = oracle_steps(cfg, w, ctx, kv, budget, 64)
        scale = float(np.abs(ref).max())
        err = float(np.abs(g - ref).max())
        tol = (2e-2 if cfg.quant in ("w8a16", "w4a16") else 1e-2) * scale
        parity = {"verdict": "PASS" if err <= tol else "FAIL", "max_abs_dlogit": err,
                  "tolerance": tol, "max_abs_logit": scale,
                  "argmax_match": int(np.argmax(g)) == int(np.argmax(ref))}
        us1, n1, _, _ = oracle_steps(cfg, w, ctx, kv, 0.0, 1, threads=1)
        cpu_base = {"value": us, "unit": UNIT, "cores": threads, "kind": "oracle",
                    "sample": f"{n} full fp64 decode steps of {name} at position {ctx} "
                              f"(~{budget:.0f} s budget), median",
                    "cpu_model": cpu_model(), "host_cores": os.cpu_count(),
                    "one_core": {"value": us1, "unit": UNIT, "cores": 1,
                                 "sample": f"{n1} full fp64 decode step on one thread"}}

    # ---- device timing --------------------------------------------------------
    def step():
        dec.step(-1, ctx, want_argmax=False)

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            step()
    torch.cuda.synchronize()
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            t_begin.record(stream)
            for i in range(K):
                starts[i].record(stream)
                step()
                ends[i].record(stream)
            t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    # a step that timed out surfaces here
    dec.step(-1, ctx, logits=logits)
    elapsed_ms = t_begin.elapsed_time(t_end)
    per_launch = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    elapsed_ms = max_over_ranks(world, elapsed_ms)
    kernel_ms = max_over_ranks(world, statistics.mean(per_launch))
    qs = np.percentile(np.array(per_launch) * 1e3, [10, 50, 90])

    # ---- end to end: host token in, host logits + token out, every step ------
    host_logits = torch.empty(cfg.vocab, dtype=torch.float32).pin_memory()
    hl = host_logits.numpy()
    tok = tok0
    with torch.cuda.stream(stream):
        for _ in range(3):
            tok = dec.step_host(tok, ctx, hl)
    K_e2e = max(10, min(K, 200))
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for _ in range(K_e2e):
            tok = dec.step_host(tok, ctx, hl)
    e2e_s = max_over_ranks(world, time.perf_counter() - t0)

    # ---- phase timers of one profiled step (outside the timed region) -------
    phases = None
    if rank == 0 and not args.no_phases:
        popts = amk.default_options()
        popts.profile = 1
        with torch.cuda.stream(stream):
            pdec = amk.Decoder(cfg, w, popts, stream=stream.cuda_stream)
            if kv is not None:
                for l in range(cfg.n_layers):
                    k, v = pdec.kv(l)
                    k[:, :ctx].copy_(kv[l, 0])
                    v[:, :ctx].copy_(kv[l, 1])
            pdec.step(tok0, ctx, want_argmax=False)
            for _ in range(3):
                pdec.step(-1, ctx, want_argmax=False)
        torch.cuda.synchronize()
        phases = phase_shares(pdec.profile())
        pdec.close()

    # ---- the weight stream's read ceiling (outside the timed region) ---------
    # The kernel's own bulk copies into the shared-memory ring, one CTA per
    # SM, nothing consuming them, over 4 GiB (amk_read_ceiling): the decode
    # step only reads weights and KV, so its fraction of this read rate is
    # reported beside the fraction of the copy peak (read + write bytes).
    st = dec.stats()
    read_gbs, read_cfg = None, None
    if rank == 0:
        buf = torch.empty(4 << 30, dtype=torch.uint8, device="cuda").fill_(1)
        torch.cuda.synchronize()
        best = 0.0
        for sb, ns in ((32768, 3), (65536, 3), (49152, 4)):
            g = amk.read_ceiling(buf, st.n_sms, sb, ns, reps=3, stream=stream.cuda_stream)
            if g > best:
                best, read_cfg = g, f"{ns} x {sb // 1024} KiB in flight per SM"
        read_gbs = best
        del buf
        torch.cuda.empty_cache()

    nbytes = algorithmic_bytes(cfg, ctx)
    peak, peak_kind = measured_peak()
    achieved = nbytes / (kernel_ms * 1e-3) / 1e9
    value = job_us_per_token(elapsed_ms, K, world)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None,
            "dtype": {"w8a16": "int8 weights x int16 activations, i32 then f32 accumulate",
                      "w4a16": "int4 weights (fp16 group scales) x int16 activations, "
                               "i32 then f32 accumulate"}.get(
                          cfg.quant, "bf16 weights x f32 activations (the SwiGLU vector "
                          "handed over at 15 mantissa bits), f32 accumulate"),
            "data": "synthetic (seeded random-init weights and KV cache)",
            "config": dict(workload_config(name, cfg, ctx),
                           parallelism=f"replicas{world}" if world > 1 else "single"),
            "parity": parity,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": load_traffic(name),
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
                         "algorithmic_bytes_per_launch": nbytes,
                         "kernel_us_per_launch": kernel_ms * 1e3,
                         "read_ceiling_gbs": read_gbs,
                         "frac_of_read_ceiling": achieved / read_gbs if read_gbs else None,
                         "read_ceiling_how": "amk_read_ceiling: the kernel's bulk-copy ring "
                                             f"({read_cfg}, {st.n_sms} CTAs) streaming 4 GiB "
                                             "with no consumer, best of 3 launches"},
            "achieved_gbs": achieved,
            "cpu_baseline": cpu_base,
            "e2e": {"value": job_us_per_token(e2e_s * 1e3, K_e2e, world), "unit": UNIT,
                    "h2d_bytes_per_step": 4, "d2h_bytes_per_step": cfg.vocab * 4 + 8 + 32,
                    "steps": K_e2e},
            "per_step_us": {"p10": float(qs[0]), "p50": float(qs[1]), "p90": float(qs[2]),
                            "mean": kernel_ms * 1e3, "steps": K},
            "phases": phases,
            "gpu_launches": K,
            "clocks": clocks.summary(),
            "schedule": {"tasks": st.n_tasks, "ctas": st.n_sms, "ring_stages": st.ring_stages,
                         "stage_bytes": st.stage_bytes, "attn_splits": st.attn_splits,
                         "smem_bytes": st.smem_bytes, "threads_per_cta": st.threads_per_cta,
                         "waits": "flagged words" if st.flagged_waits else "level counters",
                         "ffn_fused": bool(st.ffn_fused)},
        }
        if parity["verdict"] != "PASS":
            line["value"] = None
            line["error"] = "parity FAIL: timing withheld"
        print(json.dumps(line), flush=True)
    dec.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_noalloc(args):
    """Times amk_decode_step_noalloc on the workload (one GPU): device time
    per call (CUDA events on the stream) and host time per call (the task
    table is resolved on the host and uploaded into the static array on
    every call), next to amk_decode_step on the same weights.  Prints one
    JSON line; not part of the driver's contract."""
    import persistent_megakernel_decode_cta_b200 as amk
    from persistent_megakernel_decode_cta_b200 import build as amk_build
    amk_build.build()
    torch.cuda.set_device(0)
    name = args.workload
    mname, ctx = WORKLOADS[name]
    cfg = si.get_config(mname)
    w = si.make_model(cfg, seed=0, device="cuda")
    kv_fill = si.make_kv_fill(cfg, ctx, device="cuda") if ctx else None
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    owner = amk.Plan(cfg, sms)
    # at position 0 the caller runs the position-0 schedule, as amk_decode_step does
    plan = (owner.pos0() or owner) if ctx == 0 else owner
    ws, keep = amk.weights_struct(cfg, w)
    kv = torch.zeros((cfg.n_layers, 2, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim),
                     dtype=torch.bfloat16, device="cuda")
    if kv_fill is not None:
        kv[:, :, :, :ctx].copy_(kv_fill)
    logits = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    tok = si.make_prompt(cfg, 1, seed=10 + ctx)[0]
    st = plan.stats()
    for _ in range(max(args.warmup, 3)):
        amk.decode_step_noalloc(plan, ws, kv, tok, ctx, logits)
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    host = []
    ev[0].record()
    for i in range(K):
        t0 = time.perf_counter()
        amk.decode_step_noalloc(plan, ws, kv, tok, ctx, logits)
        host.append(time.perf_counter() - t0)
        ev[i + 1].record()
    torch.cuda.synchronize()
    dev = [ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(K)]
    dec = amk.Decoder(cfg, w)
    if kv_fill is not None:
        for l in range(cfg.n_layers):
            k, v = dec.kv(l)
            k[:, :ctx].copy_(kv_fill[l, 0])
            v[:, :ctx].copy_(kv_fill[l, 1])
    dec.step(tok, ctx, want_argmax=False)
    for _ in range(3):
        dec.step(tok, ctx, want_argmax=False)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(K):
        dec.step(tok, ctx, want_argmax=False)
    b.record()
    torch.cuda.synchronize()
    alloc_us = a.elapsed_time(b) * 1e3 / K
    dec.close()
    table = st.n_tasks * 96 + (sms + 1) * 4
    print(json.dumps({
        "metric": "amk_decode_step_noalloc us/token", "workload": name, "steps": K,
        "device_us_per_call": {"p10": float(np.percentile(dev, 10)),
                               "p50": float(np.percentile(dev, 50)),
                               "p90": float(np.percentile(dev, 90))},
        "host_us_per_call": {"p50": float(np.percentile(host, 50) * 1e6),
                             "p90": float(np.percentile(host, 90) * 1e6)},
        "amk_decode_step_us_per_call": alloc_us,
        "schedule_table_bytes": table,  # uploaded when the plan, weights or KV change "tasks": st.n_tasks,
    }), flush=True)
    plan.close()
    owner.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-phases", action="store_true",
                    help="skip the profiled step that reports the phase-timer shares")
    ap.add_argument("--noalloc", action="store_true",
                    help="time amk_decode_step_noalloc (schedule upload per call included) "
                         "instead of the bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.noalloc:
        run_noalloc(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
