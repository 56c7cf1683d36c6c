"""Throughput of the batched RLT transition engine on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic
sequences: reset to H_0, encode the prompt (causal encoder + memory), the
recurrent prefill (one transition per position per row), then -- for
workloads with a decode phase -- sampled generation (readout, sample, encode
the token, one transition), and the final readout.  Inputs are resident on
the device when the timed region starts.  The metric is transitions per
second: rows x positions processed, summed over ranks.

With N > 1 (torchrun) every rank runs its own shard of rows (the same
per-GPU batch: weak scaling); there is no collective on the data path, only
the barrier and the max-over-ranks reduction of the timing.

--impl reference times the CPU oracle (test infrastructure, float64 numpy)
on all host cores, one process per core over rows, on a bounded sample of
the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import rlt_inputs as ri  # noqa: E402

METRIC = "decoder transition tokens/s (batch x steps) at 1 B200"
DEFAULT_CONFIG = "parity_bf16"


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


def kernel_traffic(alg_bytes_per_launch: float, record: str | None = None):
    """DRAM bytes per launch of the dominant kernel from its committed ncu
    capture (profiles/dominant_kernel_traffic.json), scaled from the captured
    launch to the average launch by the algorithmic bytes.  None when there is
    no capture or the kernel's source changed since it was taken."""
    import hashlib
    try:
        path = record or os.path.join(ROOT, "profiles", "dominant_kernel_traffic.json")
        rec = json.load(open(path))
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
        if hashlib.sha256(src).hexdigest() != rec["source_sha256"]:
            return None
        return rec["dram_bytes"] * alg_bytes_per_launch / rec["alg_bytes"]
    except Exception:
        return None


def encoder_flops(cfg, rows: int, T: int) -> float:
    """Algorithmic FLOPs of encoding T positions of `rows` rows from empty
    caches: per position and encoder layer 2 (4 d^2 + 3 d f) for the
    projections and the SwiGLU FFN, per layer the causal attention
    2 * 2 d * t summed over t = 1..T, and 2 * 2 d^2 per memory group."""
    d, f = cfg.d, cfg.ffn
    per_pos = cfg.n_enc * 2 * (4 * d * d + 3 * d * f)
    if cfg.n_dec > 0:
        per_pos += cfg.groups * 2 * 2 * d * d
    attn = cfg.n_enc * 2 * d * T * (T + 1)
    return float(rows) * (per_pos * T + attn)


def workload_desc(cfg) -> dict:
    kind = {0: "RLT-0", 1: "RLT-1", 2: f"RLT-2 (feedback chunk {cfg.chunk})"}[cfg.variant]
    dt = "bf16" if cfg.dtype == ri.DT_BF16 else "fp32"
    return {
        "workload": f"{cfg.name}: {kind} {dt}, vocab {cfg.vocab}, d={cfg.d}, {cfg.heads} heads, "
                    f"{cfg.n_enc}+{cfg.n_dec} layers{' tied' if cfg.tied else ''}, W={cfg.window}, "
                    f"G={cfg.groups}, {cfg.token_recipe} tokens, random N(0,0.02) weights",
        "batch_per_gpu": cfg.batch, "prompt": cfg.prompt, "decode": cfg.decode,
    }


# ----------------------------------------------------------------------------
# CPU oracle leg
# ----------------------------------------------------------------------------
def _oracle_worker(job):
    """One host process of the CPU baseline: run the oracle (float64, as it
    stands, one BLAS thread) on whole rows of the workload until the budget
    is spent; returns (transitions, rows, seconds)."""
    fields, row0, stride, T, budget_s = job
    try:
        import threadpoolctl
        threadpoolctl.threadpool_limits(1)
    except Exception:
        pass
    from oracle import RLTOracle
    cfg = ri.RLTConfig(**fields)
    orc = RLTOracle(cfg, ri.generate_weights(cfg, threads=1), "fp64")
    done, rows, row = 0, 0, row0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        st = orc.new_state()
        orc.encode(st, ri.make_tokens(cfg, 1, T, row0=row)[0])
        for _ in range(T):
            orc.transition(st)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        orc.readout(st)
        rows += 1
        row += stride
    return done, rows, time.perf_counter() - t0


def oracle_processes(cfg) -> int:
    """Host processes for the CPU baseline: one per core, fewer when the
    oracle's float64 copy of the weights would not fit in host memory."""
    cores = os.cpu_count() or 1
    wbytes = 8.0 * ri.param_count(cfg) * 2.2          # float64 copy + generation buffers
    try:
        avail = os.sysconf("SC_AVPHYS_PAGES") * os.sysconf("SC_PAGE_SIZE")
        cores = max(1, min(cores, int(0.6 * avail // wbytes)))
    except (ValueError, OSError, AttributeError):
        pass
    return cores


def oracle_sample(cfg, budget_s: float = 15.0):
    """The CPU baseline: the oracle as it stands (float64 numpy, one row at a
    time) on all host cores, one process per core over independent rows of
    the workload (spawned, so no process inherits a CUDA context).  Returns
    (tokens/s, description, processes)."""
    import multiprocessing as mp
    procs = oracle_processes(cfg)
    T = min(cfg.prompt, 256)
    import dataclasses
    fields = dataclasses.asdict(cfg)
    jobs = [(fields, p, procs, T, budget_s) for p in range(procs)]
    t0 = time.perf_counter()
    with mp.get_context("spawn").Pool(procs) as pool:
        res = pool.map(_oracle_worker, jobs)
    wall = time.perf_counter() - t0
    done = sum(r[0] for r in res)
    rows = sum(r[1] for r in res)
    busy = max(r[2] for r in res)
    desc = (f"{rows} row(s) of the same workload, prompt {T} (encode + transitions + readout; "
            f"the last row of each process cut at the budget), float64 numpy oracle, one "
            f"process per core with one BLAS thread each: {done} transitions in {busy:.1f} s "
            f"({wall:.1f} s with process start-up and weight generation)")
    return done / busy, desc, procs


# ----------------------------------------------------------------------------
# rank bookkeeping (weak scaling: every rank runs its own rows, no collective
# on the data path)
# ----------------------------------------------------------------------------
def shard_tokens(cfg, rank: int, batch: int, length: int) -> np.ndarray:
    """This rank's prompts: rows rank*batch .. rank*batch+batch-1 of the one
    global token stream (each row has its own substream)."""
    return ri.make_tokens(cfg, batch, length, row0=rank * batch)


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: the job's time."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(batch: int, positions: int, world: int, ms_per_step: float) -> float:
    """Transitions of all ranks in one step over the slowest rank's time."""
    return batch * positions * world / (ms_per_step / 1e3)


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    vals = []
    # every sample starts its own processes; their start-up and weight
    # generation stay outside the timed part
    for _ in range(args.warmup):
        oracle_sample(cfg, budget_s=1.0)
    for _ in range(args.steps):
        v, desc, threads = oracle_sample(cfg, budget_s=max(5.0, 60.0 / max(1, args.steps)))
        vals.append(v)
    value = statistics.median(vals)
    # the line of the run it is compared with (same N, workload and global
    # batch); the work itself ran on rank 0's host cores, as cpu_baseline says
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(workload_desc(cfg), global_batch=cfg.batch * args.gpus),
            "hardware": "host CPU cores of rank 0 (the float64 oracle, one process per core; "
                        "no GPU work)",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0 or world == 1:
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "rlt_build", os.path.join(ROOT, "stateful_decoding_b200", "build.py"))
        builder = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(builder)
        builder.build()
    if world > 1:
        dist.barrier()
    import stateful_decoding_b200 as sd

    B, T, D = cfg.batch, cfg.prompt, cfg.decode
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W), device=local)
    st = sd.State(model, B, T + D)
    # each rank runs its own rows: the token substreams start at rank * B
    toks_h = shard_tokens(cfg, rank, B, T)
    toks = torch.from_numpy(toks_h).to(dev)
    logits = torch.empty(B, cfg.vocab, device=dev)
    ids = torch.empty(B, dtype=torch.int32, device=dev)
    am = torch.empty(B, dtype=torch.int32, device=dev)
    # a stream of our own: the library replays transition blocks as CUDA
    # graphs, which cannot be captured on the legacy default stream
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    def step(tok_in, out_logits, out_ids, out_am):
        st.reset(stream=stream)
        st.encode(tok_in, stream=stream)
        st.prefill(T, stream=stream)
        for k in range(D):
            st.readout(sampled=out_ids, seed=ri.SAMPLE_SEED, step=k, stream=stream)
            st.encode(out_ids.view(B, 1) if hasattr(out_ids, "view") else out_ids.reshape(B, 1),
                      stream=stream)
            st.step(stream=stream)
        st.readout(logits=out_logits, argmax=out_am, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(3, args.warmup)):
        step(toks, logits, ids, am)
    barrier()

    # ---- device-resident timed region ----
    launches0 = sd.rlt_kernel_launches()
    st.profile(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.nvtx.range_push("timed")
        e0.record(stream)
        for _ in range(args.steps):
            step(toks, logits, ids, am)
        e1.record(stream)
        torch.cuda.nvtx.range_pop()
        barrier()
    ms_total = e0.elapsed_time(e1)
    launches = sd.rlt_kernel_launches() - launches0
    prof = {name: st.profile_query(cls, stream) for name, cls in
            (("xattn", sd.PROF_XATTN), ("swa", sd.PROF_SWA), ("step", sd.PROF_STEP),
             ("enc", sd.PROF_ENC), ("enc1", sd.PROF_ENC1))}
    st.profile(False)
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / args.steps
    tokens_step = B * (T + D) * world
    value = job_tokens_per_s(B, T + D, world, ms_step)

    # ---- end to end through the C ABI with host buffers ----
    toks_pin = torch.from_numpy(toks_h).pin_memory()
    lg_pin = torch.empty(B, cfg.vocab, dtype=torch.float32).pin_memory()
    am_pin = torch.empty(B, dtype=torch.int32).pin_memory()
    ids_pin = np.zeros(B, np.int32)
    barrier()
    t0 = time.perf_counter()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        step(toks_pin, lg_pin, ids, am_pin)
    f1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev) / args.steps
    e2e_wall = (time.perf_counter() - t0) * 1e3 / args.steps
    h2d = B * T * 4
    d2h = B * cfg.vocab * 4 + B * 4

    # ---- per-launch timing of the attention kernels: one more, untimed step
    # whose graphs carry event nodes around each attention launch ----
    barrier()
    st.profile(2)
    step(toks, logits, ids, am)
    kprof = {name: st.profile_query(cls, stream) for name, cls in
             (("xattn", sd.PROF_XATTN), ("swa", sd.PROF_SWA))}
    per_layer = {}
    for name, cls in (("xattn", sd.PROF_XATTN), ("swa", sd.PROF_SWA)):
        rows = []
        for lyr in range(cfg.n_dec):
            n_l, ms_l, by_l = st.profile_query(cls + sd.PROF_NCLS * (lyr + 1), stream)
            rows.append({"layer": lyr, "avg_us": ms_l / n_l * 1e3 if n_l else None,
                         "alg_GBps": by_l / ms_l * 1e3 / 1e9 if ms_l else None})
        per_layer[name] = rows
    st.profile(0)

    pk, pk_kind = peaks()
    n_s, ms_s, by_s = prof["step"]
    step_gbs = (by_s / ms_s * 1e3 / 1e9) if ms_s else 0.0
    enc_ms = prof["enc"][1] / args.steps
    enc_tf = encoder_flops(cfg, B, T) / (enc_ms / 1e3) / 1e12 if enc_ms else 0.0
    # the one-position encoder calls of the generation loop: HBM-bound reads
    # of the cached keys and values (weights not counted)
    n_e1, ms_e1, by_e1 = prof["enc1"]
    enc1_gbs = (by_e1 / ms_e1 * 1e3 / 1e9) if ms_e1 else 0.0
    tc_peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    n, ms, by = kprof["xattn"]
    kname = ("decoder cross-attention (one warp per (row, head), q from the projection slabs: "
             + ("k_attn_sq, keys staged in shared memory by cp.async" if cfg.d // cfg.heads == 64
                else "k_attn_xsplit, keys split over four warps") + ")")
    xattn_timed = bool(n)
    if not n:       # no per-launch records: fall back to whole transition blocks
        n, ms, by = prof["step"]
        kname = "decoder transition block (graph of the block's kernels)"
    achieved = (by / n) / ((ms / n) / 1e3) / 1e9 if n else 0.0
    n_w, ms_w, by_w = kprof["swa"]
    swa_gbs = (by_w / n_w) / ((ms_w / n_w) / 1e3) / 1e9 if n_w else 0.0

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == ri.DT_BF16 else "f32", "data": "synthetic",
        "config": dict(workload_desc(cfg), global_batch=B * world,
                       parallelism=f"replicas x{world} (rows sharded, no collective)",
                       l2="no flush: each step writes and reads > 126 MB "
                          "(encoder cache, memory, rings of all rows)"),
        "gpu_launches": launches,
        "e2e": {"value": job_tokens_per_s(B, T + D, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "wall_ms_per_step": e2e_wall},
        "roofline": {"bound": "hbm", "kernel": kname,
                     "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"],
                     "traffic": kernel_traffic(by / n) if xattn_timed else None,
                     "peak_kind": f"{pk_kind} hbm_gbs", "launches": n,
                     "avg_launch_us": (ms / n * 1e3) if n else None,
                     "alg_bytes_per_launch": (by / n) if n else None},
        # the whole decoder step (every kernel of the transition blocks)
        # against its HBM roofline, and the encoder against the tensor peak
        "roofline_decoder_step": {
            "bound": "hbm", "achieved": step_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": step_gbs / pk["hbm_gbs"], "peak_kind": f"{pk_kind} hbm_gbs",
            "alg_bytes_per_step": by_s / args.steps, "ms_per_step": ms_s / args.steps},
        "roofline_encoder": {
            "bound": "tensor", "achieved": enc_tf, "peak": tc_peak, "unit": "TFLOP/s",
            "frac": enc_tf / tc_peak if tc_peak else None,
            "peak_kind": f"{pk_kind} bf16_tflops_sustained",
            "flops_per_step": encoder_flops(cfg, B, T), "ms_per_step": enc_ms},
        "breakdown": {
            "decoder_step": {"launches": n_s, "avg_us": (ms_s / n_s * 1e3) if n_s else None,
                             "alg_GBps": step_gbs, "frac_hbm": step_gbs / pk["hbm_gbs"]},
            "swa": {"launches": n_w, "avg_us": (ms_w / n_w * 1e3) if n_w else None,
                    "alg_GBps": swa_gbs, "frac_hbm": swa_gbs / pk["hbm_gbs"]},
            "attention_by_layer": per_layer,
            "encoder_ms_per_step": (prof["enc"][1] + ms_e1) / args.steps,
            "encoder_prompt_ms_per_step": enc_ms,
            "encoder_generation_ms_per_step": ms_e1 / args.steps,
            "decoder_ms_per_step": ms_s / args.steps,
        },
    }
    if n_e1:
        line["roofline_encoder_generation"] = {
            "bound": "hbm", "achieved": enc1_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": enc1_gbs / pk["hbm_gbs"], "peak_kind": f"{pk_kind} hbm_gbs",
            "blocks": n_e1, "alg_bytes_per_step": by_e1 / args.steps,
            "ms_per_step": ms_e1 / args.steps}
    clk_s = clk.summary()
    if clk_s:
        line["clocks"] = clk_s
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, threads = oracle_sample(cfg, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line))
    st.close()
    model.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(ri.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the rows per GPU (small profiling cases only)")
    ap.add_argument("--prompt", type=int, default=None,
                    help="override the prompt length (small profiling cases only)")
    ap.add_argument("--decode", type=int, default=None,
                    help="override the sampled tokens per row (small profiling cases only)")
    ap.add_argument("--variant", type=int, default=None, choices=[0, 1, 2],
                    help="run the workload's model as RLT-0, RLT-1 or RLT-2 (feedback variants)")
    ap.add_argument("--chunk", type=int, default=None,
                    help="RLT-2 feedback chunk B_c (with --variant 2)")
    args = ap.parse_args()
    cfg = ri.CONFIGS[args.config]
    if args.batch or args.prompt or args.decode is not None:
        cfg = cfg.replace(batch=args.batch or cfg.batch, prompt=args.prompt or cfg.prompt,
                          decode=cfg.decode if args.decode is None else args.decode)
    if args.variant is not None:
        v = args.variant
        chunk = (args.chunk or cfg.chunk) if v == 2 else 1
        cfg = cfg.replace(name=f"{cfg.name} as RLT-{v}" + (f" B_c={chunk}" if v == 2 else ""),
                          variant=v, chunk=chunk)
    elif args.chunk is not None:
        ap.error("--chunk needs --variant 2")
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
