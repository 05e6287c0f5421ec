"""Benchmark: one ARMT-1B-shaped forward over 131072 tokens (128 segments of
1024), Diagonal Batching schedule, on the library's own kernels.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 1b|3b|small|tiny] [--segments S]

Prints ONE JSON line on rank 0.  `value` = tokens/s of the whole job (all
ranks; each rank runs its own independent forward: the path does not shard,
multi-GPU runs are replicas).  Inputs are resident in HBM before the timed
region; the 512 MB input embeddings and 2 GB of weights exceed the 126 MB L2,
so no flush is needed between steps.

--impl reference times the CPU oracle (fp64, numpy) on the host cores on a
bounded sample of the same workload (the first segment), rank 0 only.
"""
from __future__ import annotations

import argparse
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

METRIC = "tokens/s, one 131072-token ARMT-1B forward; grouped-GEMM tensor-pipe % peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "of measured"
    return dict(FALLBACK_PEAKS), "of fallback"


def workload_name(cfg, S, schedule):
    return (f"ARMT-{cfg.name} forward, {S * cfg.seg_len} tokens = {S} segments x {cfg.seg_len} "
            f"(+{cfg.n_mem} memory tokens), L={cfg.n_layers}, d={cfg.d_model}, batch 1, {schedule} schedule")


# ---------------------------------------------------------------------------- algorithmic work

def kind_flops(cfg, n_nodes: int, T: int):
    """Algorithmic flops of every kernel kind over n_nodes nodes of T' = T + M rows."""
    Tp = T + cfg.n_mem
    d, H, KV, hd, F, dk, P, M = (cfg.d_model, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.d_ffn,
                                 cfg.d_key, cfg.phi_dim, cfg.n_mem)
    nqkv = (H + 2 * KV) * hd
    per = {
        "tc_qmem": 2 * Tp * dk * d,
        "tc_read": 2 * Tp * P * d,
        "tc_qkv_rope": 2 * Tp * nqkv * d,
        "tc_o": 2 * Tp * d * H * hd,
        "tc_gateup_swiglu": 2 * Tp * 2 * F * d,
        "tc_down": 2 * Tp * d * F,
        "attention": 4 * hd * H * Tp * (Tp + 1) // 2,
        "tc_kvmem": 2 * M * (dk + d) * d,
    }
    return {k: v * n_nodes for k, v in per.items()}


def weight_bytes(cfg) -> int:
    """Bytes of the stacked 16-bit layer weights (attention, MLP, memory projections)."""
    d, hd = cfg.d_model, cfg.head_dim
    per_layer = ((cfg.n_heads + 2 * cfg.n_kv_heads) * hd * d + d * cfg.n_heads * hd + 3 * cfg.d_ffn * d
                 + (cfg.d_key + cfg.d_key + d) * d)
    return 2 * cfg.n_layers * per_layer


def kind_bytes(cfg, n_nodes: int, T: int):
    """Algorithmic HBM bytes of the memory-bound kinds over n_nodes nodes."""
    Tp = T + cfg.n_mem
    d, P, M, dk = cfg.d_model, cfg.phi_dim, cfg.n_mem, cfg.d_key
    per = {
        "memw_update": d * P * (4 + 4),              # read A, write A (fp32 state)
        "memw_phi": M * P * 4 + P * 8,
        "dpfp_read": Tp * dk * 4 + Tp * P * 4,       # q in, phi out (fp32, tf32-rounded)
        "tc_kvmem": (dk + d) * d * 2 + M * d * 2 + M * (dk + d) * 4,   # weight-read bound (M = 16 rows)
    }
    return {k: v * n_nodes for k, v in per.items()}


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, pw, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                    pw.append(float(parts[3]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of x over all ranks (the timed region's duration of the
    slowest replica); x itself on one rank."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, ms_max: float, world: int) -> float:
    """Whole-job tokens/s of `world` independent replicas, each processing
    tokens_per_rank tokens, timed by the slowest one (ms_max)."""
    return world * tokens_per_rank / (ms_max / 1e3)


# ---------------------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, weights, emb, threads_note=True):
    """Time the oracle on the first segment of the workload; returns (tokens/s, seconds, cores)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max((p.get("num_threads", 1) for p in threadpool_info()), default=os.cpu_count())
    except Exception:
        cores = os.cpu_count()
    T = cfg.seg_len
    t0 = time.perf_counter()
    oracle.forward(cfg, weights, emb[:T])
    dt = time.perf_counter() - t0
    return T / dt, dt, cores


def run_reference(args, cfg, S):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from recurrent_memory_transformer_diag_b200.inputs import make_embeddings, make_weights
    weights = make_weights(cfg)
    emb = make_embeddings(cfg, 1)
    for _ in range(args.warmup):
        oracle_sample(cfg, weights, emb)
    times = []
    cores = os.cpu_count()
    for _ in range(args.steps):
        _, dt, cores = oracle_sample(cfg, weights, emb)
        times.append(dt)
    t = sum(times) / len(times)
    value = cfg.seg_len / t
    sample = (f"first segment only ({cfg.seg_len} tokens + {cfg.n_mem} memory tokens through all "
              f"{cfg.n_layers} layers) of the {S * cfg.seg_len}-token workload, fp64 numpy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(cfg, S, "sequential (oracle)"), "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- our arm

def run_ours(args, cfg, S):
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    from recurrent_memory_transformer_diag_b200.inputs import make_embeddings, make_weights

    world, rank, local = dist_setup(args.gpus)
    peaks, peak_note = load_peaks()
    T, L, d, P = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    esz = 2 if cfg.dtype == "bf16" else 4

    weights = make_weights(cfg)
    emb_host = make_embeddings(cfg, S)
    m = Armt(cfg, max_segments=S, schedule=args.schedule)
    m.load_weights(weights)
    emb = torch.from_numpy(emb_host).to("cuda").to(dt)
    out = torch.empty(S * T, d, dtype=dt, device="cuda")
    A = torch.empty(L, d, P, dtype=torch.float32, device="cuda")
    z = torch.empty(L, P, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def timed(n_steps, schedule):
        m.set_schedule(schedule)
        for _ in range(args.warmup):
            m.forward(emb, S, T, out, A, z)
        m.device_status()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push(f"timed_{schedule}")
        e0.record(stream)
        for _ in range(n_steps):
            m.forward(emb, S, T, out, A, z)
        e1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        barrier(world)
        m.device_status()
        return e0.elapsed_time(e1) / n_steps

    # ---- timed region: the diagonal (or requested) schedule
    clocks = ClockSampler(local)
    clocks.start()
    ms = timed(args.steps, args.schedule)
    clk = clocks.stop()
    ms = max_over_ranks(ms, world)
    tokens = S * T
    value = replica_throughput(tokens, ms, world)
    launches_per_step = m.launch_count(S)

    extra = {}
    # ---- the library's own sequential schedule on the same kernels
    if not args.no_seq and args.schedule == "diagonal":
        ms_seq = max_over_ranks(timed(max(2, args.steps // 2), "sequential"), world)
        extra["sequential_tokens_per_s"] = replica_throughput(tokens, ms_seq, world)
        extra["sequential_ms_per_step"] = ms_seq
        extra["speedup_vs_sequential"] = ms_seq / ms
        m.set_schedule(args.schedule)

    # ---- sequence-length sweep at this shape (same context, same kernels): the
    # diagonal and sequential schedules at S segments each; and the "ideal even
    # load" throughput, every node run at the per-node cost of a full wave (the
    # marginal cost of one more segment once S >= L, measured between the two
    # largest S of the sweep)
    if world == 1 and not args.no_sweep:
        extra["sweep"] = seq_len_sweep(args, m, emb, out, A, z, S, T, L, stream)
        m.set_schedule(args.schedule)

    # ---- per-kernel device times (un-graphed forward, CUDA events around each launch)
    prof = m.profile_forward(emb, S, T, out, A, z)
    n_nodes = S * L
    flops = kind_flops(cfg, n_nodes, T)
    byts = kind_bytes(cfg, n_nodes, T)
    peak_tf = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    kernels = {}
    for k, (kms, cnt) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
        row = {"ms": round(kms, 3), "launches": cnt, "share": None}
        if k in flops and k.startswith(("tc_", "attention")) and k != "tc_kvmem":
            row["tflops"] = round(flops[k] / (kms / 1e3) / 1e12, 1)
        if k in byts:
            row["gbs"] = round(byts[k] / (kms / 1e3) / 1e9, 1)
        kernels[k] = row
    tot = sum(v["ms"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = round(v["ms"] / tot, 4) if tot else None
    gemm_kinds = [k for k in prof if k.startswith("tc_") and k != "tc_kvmem"]   # tensor-bound grouped GEMMs
    gemm_ms = sum(prof[k][0] for k in gemm_kinds)
    gemm_fl = sum(flops[k] for k in gemm_kinds)
    dominant = max(gemm_kinds, key=lambda k: prof[k][0]) if gemm_kinds else max(prof, key=lambda k: prof[k][0])
    dms, dcnt = prof[dominant]
    d_flops_launch = flops.get(dominant, 0) / max(dcnt, 1)
    achieved = d_flops_launch / (dms / dcnt / 1e3) / 1e12
    traffic = read_traffic(dominant, cfg.name, T)
    if traffic is not None:
        traffic = round(traffic * n_nodes / dcnt)   # bytes per node x nodes per launch (average over launches)
    roofline = {"bound": "tensor", "kernel": dominant, "achieved": round(achieved, 1), "peak": peak_tf,
                "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                "peak_note": f"dense bf16 sustained {peak_note}",
                "flops_per_launch": d_flops_launch, "launches": dcnt,
                "traffic": traffic,
                "all_grouped_gemms": {"achieved": round(gemm_fl / (gemm_ms / 1e3) / 1e12, 1) if gemm_ms else None,
                                      "frac": round(gemm_fl / (gemm_ms / 1e3) / 1e12 / peak_tf, 4) if gemm_ms else None,
                                      "ms": round(gemm_ms, 3)}}

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        he = torch.from_numpy(emb_host).to(dt).pin_memory()
        ho = torch.empty(S * T, d, dtype=dt).pin_memory()
        hA = torch.empty(L, d, P, dtype=torch.float32).pin_memory()
        hz = torch.empty(L, P, dtype=torch.float32).pin_memory()
        m.forward_host(he, S, T, ho, hA, hz)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(2, args.steps // 2)
        e0.record(stream)
        for _ in range(n_e2e):
            m.forward_host(he, S, T, ho, hA, hz)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        e2e = {"value": replica_throughput(tokens, ms_e2e, world), "unit": "tokens/s",
               "h2d_bytes_per_step": tokens * d * esz,
               "d2h_bytes_per_step": tokens * d * esz + L * d * P * 4 + L * P * 4,
               "ms_per_step": ms_e2e}

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, secs, cores = oracle_sample(cfg, weights, emb_host[:T])
        cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first segment ({T} tokens + {cfg.n_mem} memory tokens, all {L} layers) of the "
                         f"workload, fp64 numpy oracle, {secs:.1f} s"}

    # ---- segment-length sweep: the same token count split into segments of
    # 512 and 2048 tokens (a context per length; skill page, "Practical
    # Guidance", segment length tuning)
    if world == 1 and not args.no_sweep and extra.get("sweep") is not None:
        extra["sweep"]["seg_len"] = seg_len_sweep(args, cfg, weights, emb, S * T, T, ms, extra, stream)

    # ---- the full-attention decoder over the same tokens on the same kernels
    # (no memory tokens, one segment): the baseline the pages compare with
    if world == 1 and not args.no_sweep:
        extra["full_attention"] = full_attention(cfg, weights, emb, S * T, ms, stream)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": workload_name(cfg, S, args.schedule), "segments": S, "seg_len": T,
                   "batch": 1, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": (f"inputs (emb {S * T * cfg.d_model * 2 / 1e6:.0f} MB) and weights "
                          f"({weight_bytes(cfg) / 1e9:.1f} GB) exceed the 126 MB L2; no flush needed"),
                   "weights": "random init N(0,0.02) (bf16-rounded), embeddings N(0,1)",
                   "precision": ("bf16 weights held exactly in fp16, fp16 MMA operands, fp32 accumulate, "
                                 "fp32 residual stream and memory state; bf16 embeddings in, bf16 hidden out"
                                 if cfg.dtype == "bf16" else "fp32 throughout")},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps, "launches_per_step": launches_per_step,
        "clocks": clk, "kernels": kernels, **extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    m.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _time_forward(m, emb, out, A, z, S, T, schedule, n_steps, n_warm, stream):
    """Mean ms of n_steps graph-launched forwards of S segments after n_warm warm-ups."""
    import torch
    m.set_schedule(schedule)
    for _ in range(n_warm):
        m.forward(emb, S, T, out, A, z)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_steps):
        m.forward(emb, S, T, out, A, z)
    e1.record(stream)
    torch.cuda.synchronize()
    m.device_status()
    return e0.elapsed_time(e1) / n_steps


SWEEP_SEGMENTS = (4, 16, 32, 64, 128)


def seq_len_sweep(args, m, emb, out, A, z, S_max, T, L, stream):
    rows = []
    for S in [s for s in SWEEP_SEGMENTS if s <= S_max]:
        md = _time_forward(m, emb, out, A, z, S, T, "diagonal", 3, 2, stream)
        mq = _time_forward(m, emb, out, A, z, S, T, "sequential", 2, 1, stream)
        rows.append({"segments": S, "tokens": S * T, "diagonal_tokens_per_s": S * T / (md / 1e3),
                     "sequential_tokens_per_s": S * T / (mq / 1e3), "diagonal_ms": md, "sequential_ms": mq,
                     "speedup": mq / md})
    res = {"rows": rows}
    big = [r for r in rows if r["segments"] >= L]
    if len(big) >= 2:
        a, b = big[-2], big[-1]
        per_seg = (b["diagonal_ms"] - a["diagonal_ms"]) / (b["segments"] - a["segments"])
        res["ideal_even_load"] = {
            "tokens_per_s": T / (per_seg / 1e3), "ms_per_full_wave": per_seg,
            "how": (f"every node at the per-node cost of a full {L}-node wave: the marginal diagonal time of one "
                    f"more segment between S={a['segments']} and S={b['segments']} (each adds one full wave)"),
        }
        for r in rows:
            r["frac_of_ideal"] = r["diagonal_tokens_per_s"] / res["ideal_even_load"]["tokens_per_s"]
    return res


def seg_len_sweep(args, cfg, weights, emb, tokens, T0, ms0, extra, stream):
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    rows = [{"seg_len": T0, "segments": tokens // T0, "diagonal_tokens_per_s": tokens / (ms0 / 1e3),
             "sequential_tokens_per_s": extra.get("sequential_tokens_per_s"),
             "speedup": extra.get("speedup_vs_sequential")}]
    for Tx in (512, 2048):
        if Tx == T0 or tokens % Tx:
            continue
        Sx = tokens // Tx
        c2 = cfg.with_(seg_len=Tx, n_segments=Sx)
        m2 = Armt(c2, max_segments=Sx)
        try:
            m2.load_weights(weights)
            out2 = torch.empty(tokens, cfg.d_model, dtype=emb.dtype, device="cuda")
            A2 = torch.empty(cfg.n_layers, cfg.d_model, cfg.phi_dim, dtype=torch.float32, device="cuda")
            z2 = torch.empty(cfg.n_layers, cfg.phi_dim, dtype=torch.float32, device="cuda")
            md = _time_forward(m2, emb, out2, A2, z2, Sx, Tx, "diagonal", 3, 2, stream)
            mq = _time_forward(m2, emb, out2, A2, z2, Sx, Tx, "sequential", 2, 1, stream)
            rows.append({"seg_len": Tx, "segments": Sx, "diagonal_tokens_per_s": tokens / (md / 1e3),
                         "sequential_tokens_per_s": tokens / (mq / 1e3), "speedup": mq / md})
            del out2, A2, z2
        finally:
            m2.close()
    return rows


def full_attention(cfg, weights, emb, tokens, ms_armt, stream):
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    c2 = cfg.with_(n_mem=0, seg_len=tokens, n_segments=1)
    m2 = Armt(c2, max_segments=1)
    try:
        m2.load_weights(weights)
        out2 = torch.empty(tokens, cfg.d_model, dtype=emb.dtype, device="cuda")
        A2 = torch.empty(cfg.n_layers, cfg.d_model, cfg.phi_dim, dtype=torch.float32, device="cuda")
        z2 = torch.empty(cfg.n_layers, cfg.phi_dim, dtype=torch.float32, device="cuda")
        msf = _time_forward(m2, emb, out2, A2, z2, 1, tokens, "diagonal", 3, 2, stream)
        del out2, A2, z2
    finally:
        m2.close()
    return {"tokens_per_s": tokens / (msf / 1e3), "ms": msf, "armt_diagonal_speedup": msf / ms_armt,
            "workload": f"LLaMA-{cfg.name}-shaped decoder, full causal attention over {tokens} tokens "
                        f"(no memory tokens, one segment), same kernels"}


def read_traffic(kernel: str, config: str, seg_len: int):
    """DRAM bytes per node of `kernel` from the committed ncu summary
    (profiles/traffic.txt: dram__bytes_read.sum + dram__bytes_write.sum of one
    captured full wave, divided by its nodes), if it was taken on the current
    kernel source (the source hash is recorded there) and on this model shape
    and segment length; else None."""
    import hashlib
    summ = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "recurrent_memory_transformer_diag_b200", "csrc", "tc_gemm.cu")
    if not (os.path.exists(summ) and os.path.exists(src)):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for line in open(summ):
        parts = line.split()
        if (len(parts) >= 5 and parts[0] == kernel and parts[2] == h and parts[3] == config
                and parts[4] == str(seg_len)):
            return float(parts[1])
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="1b")
    ap.add_argument("--segments", type=int, default=None)
    ap.add_argument("--schedule", default="diagonal", choices=["diagonal", "sequential"])
    ap.add_argument("--no-seq", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    args = ap.parse_args()
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS
    cfg = CONFIGS[args.config]
    S = args.segments or cfg.n_segments
    if args.impl == "reference":
        run_reference(args, cfg, S)
    else:
        run_ours(args, cfg, S)


if __name__ == "__main__":
    main()
