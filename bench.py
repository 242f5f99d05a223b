#!/usr/bin/env python
"""Benchmark of the Domino draft-block hot path on B200.

One step = one whole draft block (stage 1 base logits + W1_h h terms, stage 2
16-position correction loop, verification fused into its tail) for B requests
of the Qwen3-8B-shaped workload (d=4096, V=151936, GRU hidden 1024, rank 256,
block 16, bf16 weights, greedy).  Inputs are seeded synthetic tensors already
resident in HBM; L2 is flushed (512 MiB write) before every step and the flush
is outside the step timing.  Metric: draft blocks per second over all GPUs
(µs per block = 1e6 / value per GPU).

Multi-GPU: replicas (requests are independent; each rank drafts its own share,
no collective on the data path).  Launch with torch.distributed.run; the
timed region is bracketed by a barrier and device synchronisation and the
reported time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only baseline this path has)
on the host cores, one sixteenth of a draft block per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "draft_blocks_per_s"
UNIT = "blocks/s"
WORKLOAD = ("qwen3-8b-shaped draft block: d=4096, V=151936, GRU hidden 1024, rank 256, block 16, "
            "bf16, greedy, {B} request(s) per GPU")
LOOP_SOURCES = ["draft_model_b200/csrc/correct_loop.cu", "draft_model_b200/csrc/common.cuh",
                "draft_model_b200/csrc/domino_internal.h"]


# ---------------------------------------------------------------- distributed plumbing (CPU-testable)

def dist_env():
    """(rank, local_rank, world) from the torch.distributed.run environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init_dist(world: int, backend: str):
    """Join the process group.  Its timeout (DOMINO_PG_TIMEOUT_S, default 300 s)
    bounds every collective: when a rank dies, the others' next barrier or
    all-reduce ends with an error instead of waiting for good."""
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        timeout = float(os.environ.get("DOMINO_PG_TIMEOUT_S", "300"))
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout))


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (all-reduce MAX)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(step_seconds: list[float], units_per_step_per_rank: int, world: int, device=None):
    """Whole-job throughput: units all ranks processed / max-over-ranks time."""
    total = sum(step_seconds)
    t = max_over_ranks(total, world, device)
    units = units_per_step_per_rank * len(step_seconds) * world
    return units / t, t


# ---------------------------------------------------------------- byte / flop models

def loop_bytes(cfg, B: int) -> int:
    """Algorithmic HBM bytes of one 16-step correction loop.

    Per step, read once for the batch: W2 (V r), W1 (r (d+H)), W_ih (3H E), W_hh
    (3H H) in bf16; per request per step: the base-logit row (V fp32), h_i and
    the fed embedding row (bf16).
    """
    wb = 2
    per_step = (cfg.V * cfg.r + cfg.r * (cfg.d + cfg.H) + 3 * cfg.H * cfg.E + 3 * cfg.H * cfg.H) * wb
    per_req = cfg.V * 4 + cfg.d * wb + cfg.E * wb
    return cfg.K * (per_step + B * per_req)


def lm_head_bytes(cfg, B: int) -> int:
    """W_lm once + hidden states + base-logit writes (fp32)."""
    return cfg.V * cfg.d * 2 + B * cfg.K * cfg.d * 2 + B * cfg.K * cfg.V * 4


def lm_head_flops(cfg, B: int) -> int:
    return 2 * B * cfg.K * cfg.V * cfg.d


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def source_digest(paths) -> str:
    h = hashlib.sha1()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """ncu DRAM bytes per launch recorded in profiles/traffic.json, if still current."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_digest") != source_digest(LOOP_SOURCES):
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks during the timed region

CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle timing

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_block_rate(cfg, w, hidden, anchor, target, budget_s: float = 15.0, max_blocks: int = 4):
    """Full oracle draft blocks until ~budget_s of CPU work.

    Each block is timed in two stages: the LM head, then the loop and tau given
    its base logits (the same work as one draft_block call).  Returns
    (blocks/s, blocks, seconds, LM-head seconds per block, loop seconds per block).
    """
    import oracle
    model = oracle.Model.from_storage(w)      # weight widening: outside the timed sample
    n, t_lm, t_loop = 0, 0.0, 0.0
    while n < max_blocks and (n == 0 or t_lm + t_loop < budget_s):
        t0 = time.perf_counter()
        base = oracle.lm_head(oracle.widen_f64(hidden, cfg.dtype), model.w_lm, cfg.dtype)
        t1 = time.perf_counter()
        oracle.draft_block(model, hidden, anchor, mode=cfg.mode, temperature=cfg.temperature, seed=cfg.seed,
                           target=target, want_logits=False, base=base)
        t2 = time.perf_counter()
        t_lm += t1 - t0
        t_loop += t2 - t1
        n += 1
    t = t_lm + t_loop
    return n / t, n, t, t_lm / n, t_loop / n


class OracleFraction:
    """One sixteenth of a draft block per call: one vocabulary chunk of the LM
    head (all positions) and one position of the correction loop."""

    def __init__(self, cfg, w, hidden, anchor):
        import oracle
        self.o = oracle
        self.cfg = cfg
        self.model = oracle.Model.from_storage(w)
        self.h64 = oracle.widen_f64(hidden, cfg.dtype)
        self.anchor = anchor
        self.base = oracle.lm_head(self.h64, self.model.w_lm, cfg.dtype)
        self.parts = cfg.K
        self.chunk = (cfg.V + self.parts - 1) // self.parts
        self.it = None
        self.j = 0

    def step(self):
        c = self.j % self.parts
        v0 = c * self.chunk
        self.base[:, :, v0:v0 + self.chunk] = self.o.lm_head(self.h64, self.model.w_lm[v0:v0 + self.chunk],
                                                             self.cfg.dtype)
        if self.it is None:
            self.it = self.o.positions(self.model, self.h64, self.anchor, self.base, mode=self.cfg.mode,
                                       temperature=self.cfg.temperature, seed=self.cfg.seed)
        try:
            next(self.it)
        except StopIteration:
            self.it = None
            return self.step()
        self.j += 1


# ---------------------------------------------------------------- arms

def workload_config(B: int):
    import synth
    return synth.sweep_config(B) if B != 1 else synth.CONFIGS["qwen3_8b_b1"]


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    import synth
    cfg = workload_config(args.batch)
    w = synth.make_weights(cfg)
    hidden, anchor = synth.make_hidden(cfg, args.batch), synth.make_anchor(cfg, args.batch)
    frac = OracleFraction(cfg, w, hidden, anchor)
    for _ in range(args.warmup):
        frac.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        frac.step()
    dt = time.perf_counter() - t0
    blocks = args.steps / frac.parts * args.batch
    value = blocks / dt
    cores = blas_threads()
    sample = f"{args.steps} sixteenths of a draft block (1/16 of the LM head + one loop position), fp64 oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD.format(B=args.batch), "global_batch": args.batch, "block_size": cfg.K,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import numpy as np
    import torch

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    init_dist(world, "nccl")

    import draft_model_b200 as dm
    import synth
    from draft_model_b200.tensors import device_weights, to_dev, workspace_for

    dm.load_library()
    B = args.batch
    cfg = workload_config(B)
    w = synth.make_weights(cfg)
    dw = device_weights(w, dev)
    if args.gate_table:
        # variant: token -> gate table built once per weight set (not timed)
        from draft_model_b200.tensors import aligned_workspace
        table = torch.empty((cfg.V, 3 * cfg.H), dtype=torch.float32, device=dev)
        dm.domino_build_gate_table(dw, table, workspace=aligned_workspace(1024))
        dw.set_gate_table(table)
    first = rank * B
    hidden_np = synth.make_hidden(cfg, B, first)
    anchor_np = synth.make_anchor(cfg, B, first)
    hidden = to_dev(hidden_np, cfg.dtype, dev)
    anchor = torch.from_numpy(anchor_np).to(dev)
    ws = workspace_for(dw, B, cfg.K)
    draft = torch.empty((B, cfg.K), dtype=torch.int32, device=dev)
    tau = torch.empty((B,), dtype=torch.int32, device=dev)
    # targets from a prior draft of the same inputs (synthetic acceptance prefix)
    dm.domino_draft_block(dw, hidden, anchor, draft_out=draft, workspace=ws)
    torch.cuda.synchronize()
    target_np = synth.make_targets(cfg, draft.cpu().numpy())
    target = torch.from_numpy(target_np).to(dev)
    scrub = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for row in ev:          # create the CUDA events up front (torch creates them lazily)
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()

    def one_step(events):
        dm.domino_draft_block_events(dw, hidden, anchor, target=target, draft_out=draft, tau_out=tau,
                                     workspace=ws, events=events)

    for k in range(args.warmup):
        scrub.fill_(float(k))
        one_step(ev[0])
    torch.cuda.synchronize()
    if dm.domino_poll(ws) != 0:
        raise RuntimeError("device error during warm-up")

    clocks = ClockSampler() if rank == 0 else None
    if clocks:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for k in range(args.steps):
        scrub.fill_(float(k))
        one_step(ev[k])
    torch.cuda.synchronize()
    barrier(world)
    clock_rec = clocks.stop() if clocks else None
    status = dm.domino_poll(ws)
    if status != 0:
        raise RuntimeError(f"device error in the timed region: {dm.domino_status_str(status)}")

    step_s = [ev[k][0].elapsed_time(ev[k][2]) * 1e-3 for k in range(args.steps)]
    lm_s = [ev[k][0].elapsed_time(ev[k][1]) * 1e-3 for k in range(args.steps)]
    loop_s = [ev[k][1].elapsed_time(ev[k][2]) * 1e-3 for k in range(args.steps)]
    value, t_max = aggregate(step_s, B, world, dev)
    loop_avg = statistics.mean(loop_s)
    lm_avg = statistics.mean(lm_s)

    # warm-L2 figures beside the cold ones: the same steps back to back, no flush
    n_warm = min(args.steps, 100)
    for k in range(n_warm):
        one_step(ev[k])
    torch.cuda.synchronize()
    if dm.domino_poll(ws) != 0:
        raise RuntimeError("device error in the warm-L2 steps")
    warm = {"us_per_block": statistics.mean(ev[k][0].elapsed_time(ev[k][2]) for k in range(n_warm)) * 1e3 / B,
            "stages_us": {"lm_head_and_w1h": statistics.mean(ev[k][0].elapsed_time(ev[k][1])
                                                             for k in range(n_warm)) * 1e3,
                          "correct_loop": statistics.mean(ev[k][1].elapsed_time(ev[k][2])
                                                          for k in range(n_warm)) * 1e3},
            "steps": n_warm, "note": "L2 not flushed; outside the timed region, rank-local"}

    # end to end through the host-buffer entry point: H2D of the inputs, D2H of the results
    hid_h = torch.from_numpy(hidden_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    anc_h = torch.from_numpy(anchor_np).pin_memory()
    tgt_h = torch.from_numpy(target_np).pin_memory()
    draft_h = torch.empty((B, cfg.K), dtype=torch.int32).pin_memory()
    tau_h = torch.empty((B,), dtype=torch.int32).pin_memory()
    ws_h = workspace_for(dw, B, cfg.K, host=True)
    n_e2e = max(10, min(args.steps, 100))
    e2e_s = []
    for k in range(args.warmup + n_e2e):
        scrub.fill_(float(k))
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        dm.domino_draft_block_host(dw, hid_h, anc_h, target_host=tgt_h, draft_out_host=draft_h, tau_out_host=tau_h,
                                   workspace=ws_h)
        if k >= args.warmup:
            e2e_s.append(time.perf_counter() - t0)
    e2e_value, _ = aggregate(e2e_s, B, world, dev)
    h2d = hid_h.numel() * 2 + anc_h.numel() * 4 + tgt_h.numel() * 4
    d2h = draft_h.numel() * 4 + tau_h.numel() * 4

    peaks, peak_kind = measured_peaks()
    lbytes = loop_bytes(cfg, B)
    achieved = lbytes / loop_avg / 1e9
    # recorded for the standard B=1 loop only (the gate-table variant reads no W_ih)
    traffic = recorded_traffic("correct_loop_kernel") if B == 1 and not args.gate_table else None
    lm_frac_hbm = lm_head_bytes(cfg, B) / lm_avg / 1e9 / peaks["hbm_gbs"]
    lm_tflops = lm_head_flops(cfg, B) / lm_avg / 1e12
    # the LM head runs inside a long back-to-back step: the sustained (power-capped)
    # GEMM peak is its denominator; the burst figure is reported beside it
    lm_frac_tc = lm_tflops / peaks["bf16_tflops_sustained"]
    lm_frac_tc_burst = lm_tflops / peaks["bf16_tflops"]
    launches = dm.domino_launches_per_block(dw, B, cfg.K)
    persistent = launches == 1 + -(-B // min(8, 1 << (B.bit_length() - 1)))

    if rank != 0:
        barrier(world)
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, nblk, tcpu, t_lm, t_loop = oracle_block_rate(cfg, w, hidden_np, anchor_np, target_np)
        cpu = {"value": rate * B, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{nblk} full draft block(s) of this workload (LM head + 16-step loop + tau), "
                         f"fp64 numpy, {tcpu:.1f} s", "host_cpus": os.cpu_count(), "cpu_model": cpu_model(),
               "stages_s": {"lm_head": t_lm, "loop_and_tau": t_loop}}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD.format(B=B) + (", token->gate table variant" if args.gate_table else ""),
                   "global_batch": B * world, "block_size": cfg.K,
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": "flushed before every step (512 MiB write, outside the step timing)"},
        "us_per_block": t_max / args.steps / B * 1e6,
        "draft_tokens_per_s": value * cfg.K,
        "stages_us": {"lm_head_and_w1h": lm_avg * 1e6, "correct_loop": loop_avg * 1e6},
        "warm_l2": warm,
        "roofline": {"kernel": "correct_loop_kernel" if persistent else
                     f"correct_loop stage: per-step tensor-core path, {launches - 1} launches per block",
                     "bound": "hbm", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic, "algorithmic_bytes": lbytes, "peak_source": peak_kind},
        "lm_head_roofline": {"bound": "hbm" if B < 32 else "tensor", "frac_of_hbm": lm_frac_hbm,
                             "achieved_tflops": lm_tflops,
                             "frac_of_bf16_tensor": lm_frac_tc, "tensor_peak": "bf16_tflops_sustained",
                             "frac_of_bf16_tensor_burst": lm_frac_tc_burst, "peak_source": peak_kind},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * launches,
        "clocks": clock_rec,
    }
    print(json.dumps(line), flush=True)
    barrier(world)


def run_loss(args):
    """Training forward (teacher-forced block + base-anchored curriculum loss) on one GPU.

    Times domino_draft_loss per step (L2 flushed between steps) and, on its own,
    the curriculum-loss kernels over [B, K, V] final and base logits against the
    HBM roofline (both tensors read once).
    """
    import numpy as np
    import torch

    import draft_model_b200 as dm
    import synth
    from draft_model_b200.tensors import aligned_workspace, device_weights, to_dev

    dm.load_library()
    B = args.batch
    cfg = workload_config(B)
    dw = device_weights(synth.make_weights(cfg))
    hidden = to_dev(synth.make_hidden(cfg, B), cfg.dtype)
    anchor = torch.from_numpy(synth.make_anchor(cfg, B)).cuda()
    labels = torch.from_numpy(np.random.default_rng([7, B]).integers(0, cfg.V, size=(B, cfg.K)).astype(np.int32)).cuda()
    ws = aligned_workspace(dm.domino_draft_loss_workspace_bytes(dw, B, cfg.K))
    loss = torch.zeros(4, dtype=torch.float32, device="cuda")
    scrub = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    def step(k):
        scrub.fill_(float(k))
        e = ev[min(k, args.steps - 1)]
        e[0].record()
        dm.domino_draft_loss(dw, hidden, anchor, labels, lam=0.5, gamma=0.9, loss_out=loss, workspace=ws)
        e[1].record()

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    for k in range(args.steps):
        step(k)
    torch.cuda.synchronize()
    if dm.domino_poll(ws) != 0:
        raise RuntimeError("device error in the training forward")
    t = statistics.mean(e[0].elapsed_time(e[1]) * 1e-3 for e in ev)

    # the loss kernels alone on resident logits
    fin = torch.randn((B, cfg.K, cfg.V), device="cuda") * 4
    bas = torch.randn((B, cfg.K, cfg.V), device="cuda") * 4
    lws = aligned_workspace(dm.domino_curriculum_loss_workspace_bytes(B, cfg.K, cfg.V))
    lt = []
    for k in range(args.warmup + 20):
        scrub.fill_(float(k))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dm.domino_curriculum_loss(fin, bas, labels, lam=0.5, gamma=0.9, loss_out=loss, workspace=lws)
        e1.record()
        torch.cuda.synchronize()
        if k >= args.warmup:
            lt.append(e0.elapsed_time(e1) * 1e-3)
    lt_avg = statistics.mean(lt)
    peaks, peak_kind = measured_peaks()
    ce_bytes = 2 * B * cfg.K * cfg.V * 4
    achieved = ce_bytes / lt_avg / 1e9
    print(json.dumps({
        "metric": "training_forward_blocks_per_s", "value": B / t, "unit": "blocks/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD.format(B=B) + ", teacher-forced, curriculum loss lambda 0.5 gamma 0.9",
                   "l2": "flushed before every step"},
        "curriculum_loss_kernels": {"us": lt_avg * 1e6, "bound": "hbm", "achieved": achieved,
                                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                                    "algorithmic_bytes": ce_bytes, "peak_source": peak_kind},
        "loss": float(loss[0].item()),
    }), flush=True)


def run_verify(args):
    """Stochastic verification (speculative sampling) of a block of the workload's shape.

    Times domino_verify_sample on resident synthetic draft logits [B, K, V] and
    target logits [B, K+1, V] (L2 flushed between launches) against the HBM
    roofline: every row read once plus the resampled row pair read again.
    """
    import numpy as np
    import torch

    import draft_model_b200 as dm
    from draft_model_b200.tensors import aligned_workspace

    dm.load_library()
    B = args.batch
    cfg = workload_config(B)
    K, V = cfg.K, cfg.V
    g = torch.Generator(device="cuda").manual_seed(5)
    dl = torch.randn((B, K, V), device="cuda", generator=g) * 2
    tl = torch.cat([dl + 0.5 * torch.randn((B, K, V), device="cuda", generator=g),
                    2 * torch.randn((B, 1, V), device="cuda", generator=g)], dim=1)
    draft = torch.from_numpy(np.random.default_rng(5).integers(0, V, size=(B, K)).astype(np.int32)).cuda()
    ws = aligned_workspace(dm.domino_verify_sample_workspace_bytes(B, K, V))
    tau = torch.zeros(B, dtype=torch.int32, device="cuda")
    tok = torch.zeros(B, dtype=torch.int32, device="cuda")
    scrub = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    ts = []
    for k in range(args.warmup + args.steps):
        scrub.fill_(float(k))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dm.domino_verify_sample(dl, tl, draft, temperature=1.0, seed=k, tau_out=tau, token_out=tok, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        if k >= args.warmup:
            ts.append(e0.elapsed_time(e1) * 1e-3)
    if dm.domino_poll(ws) != 0:
        raise RuntimeError("device error in verification")
    t = statistics.mean(ts)
    peaks, peak_kind = measured_peaks()
    vbytes = (2 * K + 3) * B * V * 4
    achieved = vbytes / t / 1e9
    print(json.dumps({
        "metric": "verified_blocks_per_s", "value": B / t, "unit": "blocks/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"speculative-sampling verification, {B} request(s), block {K}, V={V}, T=1",
                   "l2": "flushed before every step"},
        "roofline": {"kernel": "verify_sample (4 launches)", "bound": "hbm", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "algorithmic_bytes": vbytes, "peak_source": peak_kind},
        "mean_tau": float(tau.float().mean().item()),
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--batch", type=int, default=1, help="requests per GPU per draft block")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gate-table", action="store_true",
                    help="variant: precomputed token->gate table (G = W_ih E + b_ih) in the batched loop")
    ap.add_argument("--mode", choices=["draft", "loss", "verify"], default="draft",
                    help="draft: the draft block (default); loss: the teacher-forced training forward; "
                         "verify: stochastic verification")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "loss":
        run_loss(args)
    elif args.mode == "verify":
        run_verify(args)
    else:
        run_ours(args)
    _, _, world = dist_env()
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
