"""Benchmark of the TurboQuant decode step on B200.

Workload (the decode-s configuration): batch 1 per GPU, 12 query heads on 2 KV heads,
d = 128, a 32768-token packed cache (keys 3-bit prod = 2-bit Lloyd-Max MSE + 1-bit QJL,
values 2-bit groups of 32, fp16 norms and group parameters), bf16 synthetic inputs
(keys N(0,1) x U[2,20] per row, values and queries N(0,1)). One step = append one new
token per KV head (quantize its key and value and write them at len) + fused decode
attention of one query token over the whole cache. Metric: keys scored per second
(query heads x cached tokens / step time) and the decode kernel's HBM GB/s; the line
also carries the key-quantize throughput (2^24 bf16 rows, 3-bit prod, 4 layers) under
"key_quantize".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]

L2 is flushed (a 256 MiB write) before every timed step, outside its events. Multi-GPU runs
are independent replicas (weak scaling): each rank holds its own batch, no collective on
the data path; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# decode workloads (synthetic, seeded): keys N(0,1) x per-row U[2,20], values N(0,1), bf16
DECODE_WORKLOADS = {
    "decode-s": dict(batch=1, n_q_heads=12, n_kv_heads=2, ctx=32768, key_bits=3, value_bits=2,
                     group=32, qseed=0),
    "decode-l": dict(batch=8, n_q_heads=28, n_kv_heads=4, ctx=32768, key_bits=3, value_bits=2,
                     group=32, qseed=0),
    "decode-stream": dict(batch=1, n_q_heads=64, n_kv_heads=8, ctx=131072, key_bits=4,
                          value_bits=4, group=32, qseed=0),
}
CFG = DECODE_WORKLOADS["decode-s"]
KEY_BYTES = 52            # 3-bit prod: 32 B indices + 16 B QJL signs + 4 B fp16 norms
VAL_BYTES = 48            # 2-bit values: 32 B codes + 4 groups x (fp16 min, fp16 scale)


def key_bytes(bits):      # prod mode: (bits - 1)-bit indices (3-bit stored in 4) + signs + norms
    w = {1: 1, 2: 2, 3: 4}[bits - 1]
    return 128 * w // 8 + 16 + 4


def value_bytes(vb):
    return 128 * vb // 8 + 16


WL_DESC = {"decode-s": "decode-s: batch 1, 12 q heads / 2 kv heads, d 128, ctx 32768, "
                       "keys 3-bit prod, values 2-bit g32",
           "decode-l": "decode-l: batch 8, 28 q heads / 4 kv heads, d 128, ctx 32768, "
                       "keys 3-bit prod, values 2-bit g32",
           "decode-stream": "decode-stream: batch 1, 64 q heads / 8 kv heads, d 128, "
                            "ctx 131072, keys 4-bit prod, values 4-bit g32"}


def decode_config(name: str, world: int) -> dict:
    """The `config` of a decode workload's JSON line (both arms)."""
    wl = DECODE_WORKLOADS[name]
    return {"workload": WL_DESC[name], "global_batch": wl["batch"] * world, "seq_len": wl["ctx"],
            "parallelism": f"replicas x{world}",
            "data_types": "bf16 query and new K/V rows, u8 packed cache, fp16 norms and value "
                          "params (the arithmetic type is the line's dtype)"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-quantize", action="store_true", help="skip the key-quantize leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "decode", "quantize"],
                    help="run one leg only (small cases for profiling)")
    ap.add_argument("--quantize-rows", type=int, default=1 << 22, help="rows per layer")
    ap.add_argument("--decode-workload", default="decode-s", choices=sorted(DECODE_WORKLOADS),
                    help="decode workload of the timed step (the headline line is decode-s)")
    ap.add_argument("--quantize-sweep", action="store_true",
                    help="with --only quantize: every mode and width of the key-quantize sweep")
    ap.add_argument("--quantize-mode", default="prod3",
                    choices=["mse1", "mse2", "mse3", "mse4", "prod2", "prod3", "prod4",
                             "grouped1", "grouped2", "grouped3"],
                    help="with --only quantize: the mode and width of the single timed pass")
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        sms.sort()
        med = sms[len(sms) // 2] if sms else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sms)}


def dist_setup(n_gpus, backend=None):
    """One process per GPU (torchrun env). NCCL on GPUs; gloo when asked (CPU tests)."""
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def _sync_device():
    import torch
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    _sync_device()


def _all_reduce(x: float, world: int, op: str) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    return _all_reduce(x, world, "max")


def sum_over_ranks(x: float, world: int) -> float:
    return _all_reduce(x, world, "sum")


def replica_throughput(units: float, ms: float, world: int):
    """Whole-job throughput of independent replicas: the units all ranks processed over the
    slowest rank's time. Returns (units per second, max ms over ranks)."""
    ms_max = max_over_ranks(ms, world)
    return sum_over_ranks(units, world) / (ms_max / 1e3), ms_max


# ------------------------------------------------------------------------------ tq arm
def run_tq(args):
    import torch

    import kv_cache_vector_fwht_b200 as tq

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    peak, peak_kind = load_peaks()
    if args.only == "quantize":
        if args.quantize_sweep:
            out = {}
            for mode, bits in [("mse", 1), ("mse", 2), ("mse", 3), ("mse", 4), ("prod", 2),
                               ("prod", 3), ("prod", 4), ("grouped", 1), ("grouped", 2),
                               ("grouped", 3)]:
                out[f"{mode}{bits}"] = bench_quantize(tq, torch, dev, world, peak, peak_kind,
                                                      rows=args.quantize_rows, mode=mode,
                                                      bits=bits)
            if rank == 0:
                print(json.dumps({"key_quantize_sweep": out}))
            return
        qm = args.quantize_mode
        r = bench_quantize(tq, torch, dev, world, peak, peak_kind, rows=args.quantize_rows,
                           mode=qm[:-1], bits=int(qm[-1]))
        if rank == 0:
            print(json.dumps({"key_quantize": r}))
        return
    WL = DECODE_WORKLOADS[args.decode_workload]
    B, Hq, Hkv, N = WL["batch"], WL["n_q_heads"], WL["n_kv_heads"], WL["ctx"]
    steps, warm = args.steps, args.warmup
    extra = warm + steps + 8
    # seeded synthetic inputs: context + one fresh token per step (per rank: its own batch)
    g = torch.Generator(device=dev).manual_seed(2 + 1000 * rank)
    K = torch.randn((B, Hkv, N, 128), generator=g, device=dev)
    K *= torch.empty((B, Hkv, N, 1), device=dev).uniform_(2.0, 20.0, generator=g)
    K = K.to(torch.bfloat16)
    V = torch.randn((B, Hkv, N, 128), generator=g, device=dev).to(torch.bfloat16)
    Kn = (torch.randn((extra, B, Hkv, 1, 128), generator=g, device=dev) *
          torch.empty((extra, B, Hkv, 1, 1), device=dev).uniform_(2.0, 20.0, generator=g)).to(torch.bfloat16)
    Vn = torch.randn((extra, B, Hkv, 1, 128), generator=g, device=dev).to(torch.bfloat16)
    Qs = torch.randn((extra, B, Hq, 128), generator=g, device=dev).to(torch.bfloat16)

    qz = tq.tq_build_codebook(128, WL["key_bits"], "prod", WL["qseed"])
    cap = ((N + extra + 2 * extra + 15) // 16) * 16
    cache = tq.KVCache(qz, B, Hkv, cap, value_bits=WL["value_bits"], device=dev)
    tq.tq_append(qz, cache, K.contiguous(), V.contiguous())       # prefill (untimed)
    ws = tq.alloc_decode_workspace(cache, Hq, dev)
    out = torch.empty((B, Hq, 128), device=dev, dtype=torch.bfloat16)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):   # one decode step: append this step's token per KV head, then decode
        tq.tq_append_decode(qz, cache, Kn[i], Vn[i], Qs[i], out, ws)

    for i in range(warm):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()

    # Timed region: `steps` decode steps, each one tq_append_decode call (the append and the
    # decode are launched back to back, so the decode's query prologue overlaps the append);
    # L2 flushed before each step, outside its events.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    lens = []
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    t_wall = time.perf_counter()
    for s in range(steps):
        flush.zero_()
        e0, e2 = ev[s]
        e0.record(stream)
        tq.tq_append_decode(qz, cache, Kn[warm + s], Vn[warm + s], Qs[warm + s], out, ws)
        e2.record(stream)
        lens.append(cache.lengths[0])
    barrier(world)
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    step_ms = [a.elapsed_time(c) for a, c in ev]
    tot_ms = sum(step_ms)
    keys_scored = float(sum(Hq * L for L in lens) * B)
    value, tot_ms_max = replica_throughput(keys_scored, tot_ms, world)
    # The decode kernel's own duration for the roofline: the same decode launches on the
    # final cache, an event on each side of every launch (an event between the append and
    # the decode would hold the decode back until the append ends), L2 flushed before each.
    k_launches = min(steps, 200)
    evk = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(k_launches)]
    for s in range(k_launches):
        flush.zero_()
        evk[s][0].record(stream)
        tq.tq_decode_attention(qz, cache, Qs[warm + s], out, ws)
        evk[s][1].record(stream)
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(c) for a, c in evk]
    dec_avg_ms = sum(dec_ms) / len(dec_ms)
    mean_len = float(cache.lengths[0])
    dec_bytes = (B * Hkv * mean_len * (key_bytes(WL["key_bits"]) + value_bytes(WL["value_bits"]))
                 + B * Hq * 128 * 2 * 2)
    achieved = dec_bytes / (dec_avg_ms / 1e3) / 1e9

    # ---- end to end through the public API: host (pinned) inputs in, result out, per step
    # each step's new keys, new values and query sit in one pinned host row (bf16, in that
    # order) and reach the device with one copy; the API reads views of the device row
    e2e_steps = 0 if args.no_e2e else min(steps, 500)
    nk, nv, nq = Kn[0].numel(), Vn[0].numel(), Qs[0].numel()
    stage_h = torch.empty((max(e2e_steps, 1), nk + nv + nq), dtype=Kn.dtype).pin_memory()
    if e2e_steps:
        stage_h[:, :nk] = Kn[:e2e_steps].reshape(e2e_steps, nk).cpu()
        stage_h[:, nk:nk + nv] = Vn[:e2e_steps].reshape(e2e_steps, nv).cpu()
        stage_h[:, nk + nv:] = Qs[:e2e_steps].reshape(e2e_steps, nq).cpu()
    oh = torch.empty((B, Hq, 128), dtype=torch.bfloat16).pin_memory()
    stage_d = torch.empty((nk + nv + nq,), dtype=Kn.dtype, device=dev)
    kd = stage_d[:nk].view(Kn[0].shape)
    vd = stage_d[nk:nk + nv].view(Vn[0].shape)
    qd = stage_d[nk + nv:].view(Qs[0].shape)
    cache.set_lengths([N] * B)
    e2e_ms = 0.0
    for s in range(e2e_steps):
        flush.zero_()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        stage_d.copy_(stage_h[s], non_blocking=True)
        tq.tq_append_decode(qz, cache, kd, vd, qd, out, ws)
        oh.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        e2e_ms += (time.perf_counter() - t0) * 1e3
    e2e_keys = float(sum(Hq * (N + s + 1) for s in range(e2e_steps)) * B)
    e2e_ms_max = max_over_ranks(e2e_ms, world)
    e2e_value = sum_over_ranks(e2e_keys, world) / (e2e_ms_max / 1e3) if e2e_steps else None

    # the block shape the library picks (tq.h, tq_set_decode_policy): up to 8 query heads per
    # block (two table sets) when a KV head has more than 4 and there are >= 4 x 384 (token,
    # KV head) units per SM (all SMs but 4), else up to 4
    heads_per_kv = Hq // Hkv
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    two_sets = heads_per_kv > 4 and B * Hkv * N >= 4 * 384 * max(1, n_sms - 4)
    cap = 8 if two_sets else 4
    nh_cta = -(-heads_per_kv // -(-heads_per_kv // cap))   # query heads per block
    nh_tpl = (2 if nh_cta <= 2 else nh_cta) if not two_sets else (6 if nh_cta <= 6 else 8)
    n_sets = 2 if two_sets else 1
    result = {
        "metric": f"fused-decode keys scored/s ({args.decode_workload} step: append 1 token per "
                  "KV head + decode)",
        "value": value, "unit": "keys/s", "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": tot_ms_max / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded torch CUDA generator; N(0,1) x U[2,20] keys)",
        "config": dict(decode_config(args.decode_workload, world),
                       l2="flushed (256 MiB write) before each step, outside its events"),
        "decode_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": f"k_decode<{WL['key_bits'] - 1},{WL['value_bits']},{nh_tpl},prod,"
                               f"{n_sets} table set{'s' if n_sets > 1 else ''}>",
                     "bytes_per_launch": dec_bytes, "avg_launch_us": dec_avg_ms * 1e3,
                     "peak_kind": f"{peak_kind} (hbm_gbs, burst)"},
        "e2e": {"value": e2e_value, "unit": "keys/s", "h2d_bytes_per_step": int(
            kd.numel() * 2 + vd.numel() * 2 + qd.numel() * 2),
                "d2h_bytes_per_step": int(oh.numel() * 2), "steps": e2e_steps},
        "gpu_launches": steps * 2,   # fused append + decode per step
        "clocks": clk,
        "wall_s_timed_region": t_wall,
    }
    if not args.no_quantize and args.only == "all":
        result["key_quantize"] = bench_quantize(tq, torch, dev, world, peak, peak_kind,
                                                rows=args.quantize_rows)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.decode_workload == "decode-s":
        result["cpu_baseline"] = cpu_baseline(sample_keys=4096)
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_quantize(tq, torch, dev, world, peak, peak_kind, rows=1 << 22, reps=5, mode="prod",
                   bits=3):
    """Key-quantize throughput: 4 layers x 2^22 bf16 rows (2^24 rows), 3-bit prod by default,
    quantizer seed = layer, 32 channels at 4x std. Inputs (4 GiB) exceed L2; no flush needed."""
    import workloads as W
    ch = torch.from_numpy(W.outlier_channels(4)).long().to(dev)
    g = torch.Generator(device=dev).manual_seed(4)
    xs, qs, planes = [], [], []
    for layer in range(4):
        x = torch.randn((rows, 128), generator=g, device=dev)
        x[:, ch] *= 4.0
        xs.append(x.to(torch.bfloat16))
        del x
        qs.append(tq.tq_build_codebook(128, bits, mode, layer,
                                       W.outlier_channels(4) if mode == "grouped" else None))
        planes.append(qs[-1].alloc_key_planes(rows, dev))
    st = torch.cuda.current_stream()
    for layer in range(4):
        tq.tq_quantize_keys(qs[layer], xs[layer], planes[layer])
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for layer in range(4):
            tq.tq_quantize_keys(qs[layer], xs[layer], planes[layer])
        e1.record(st)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    tq.tq_sync_status()
    ms = sum(times) / len(times)
    n = 4 * rows
    lay = qs[0].layout
    out_bytes = lay["idx_bytes"] + lay["sign_bytes"] + 2 * lay["n_norms"]
    gbs = n * (256 + out_bytes) / (ms / 1e3) / 1e9
    kernel = {"prod": f"k_keys_tc<prod,{bits - 1}>", "mse": f"k_keys_tc<mse,{bits}>",
              "grouped": f"k_keys_grp_tc<{bits}>"}[mode]
    del xs, planes
    torch.cuda.empty_cache()
    return {"rows_per_s": n / (ms / 1e3), "ms_per_pass": ms, "rows_per_pass": n,
            "mode": f"{mode} b={bits}",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": None,
                         "bytes_per_row": 256 + out_bytes, "kernel": kernel,
                         "peak_kind": f"{peak_kind} (hbm_gbs, burst)"}}


# ------------------------------------------------------------------------------ oracle
def _oracle_setup(sample_keys):
    import numpy as np

    import oracle as O
    import workloads as W
    g = W.rng(2)
    K = W.round_bf16(W.scaled_gaussian_rows(g, CFG["n_kv_heads"] * sample_keys))
    V = W.round_bf16(W.gaussian(g, (CFG["n_kv_heads"] * sample_keys, 128)))
    Q = W.round_bf16(W.gaussian(g, (1, CFG["n_q_heads"], 128)))
    qo = O.build_quantizer(128, CFG["key_bits"], "prod", CFG["qseed"])
    p = O.quantize_keys(qo, K.astype(np.float64))
    v = O.quantize_values(V.astype(np.float64), 2)
    H = CFG["n_kv_heads"]
    cache = dict(k_idx=p["idx"].reshape(1, H, sample_keys, -1),
                 k_signs=p["signs"].reshape(1, H, sample_keys, -1),
                 k_norms=p["norms"].reshape(1, H, sample_keys, -1),
                 v_q=v["q"].reshape(1, H, sample_keys, -1),
                 v_params=v["params"].reshape(1, H, sample_keys, 4, 2),
                 len=np.array([sample_keys]))
    return O, qo, cache, Q, K, V


def _oracle_step(O, qo, cache, Q, K, V):
    # the step's new token (quantize key + value), then decode over the cached sample
    O.quantize_keys(qo, K[:2].astype("float64"))
    O.quantize_values(V[:2].astype("float64"), 2)
    O.decode_attention(qo, cache, Q.astype("float64"), value_bits=2)


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(sample_keys=4096, seconds=10.0):
    """The oracle (fp64 numpy, as it stands) on the host cores: decode steps over a
    sample_keys-token context, repeated for about `seconds`."""
    O, qo, cache, Q, K, V = _oracle_setup(sample_keys)
    _oracle_step(O, qo, cache, Q, K, V)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        _oracle_step(O, qo, cache, Q, K, V)
        n += 1
    dt = time.perf_counter() - t0
    value = CFG["n_q_heads"] * sample_keys * n / dt
    return {"value": value, "unit": "keys/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{n} decode steps (append 1 token + 12 heads over {sample_keys} "
                      f"cached tokens of the decode-s workload), {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sample_keys = 2048
    O, qo, cache, Q, K, V = _oracle_setup(sample_keys)
    t0 = time.perf_counter()
    _oracle_step(O, qo, cache, Q, K, V)
    one = time.perf_counter() - t0
    # bound the whole run to about two minutes
    budget = 120.0
    per_step = budget / max(1, args.steps + args.warmup)
    if one > per_step:
        sample_keys = max(64, int(sample_keys * per_step / one) // 16 * 16)
        O, qo, cache, Q, K, V = _oracle_setup(sample_keys)
    for _ in range(args.warmup):
        _oracle_step(O, qo, cache, Q, K, V)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(O, qo, cache, Q, K, V)
    dt = time.perf_counter() - t0
    value = CFG["n_q_heads"] * sample_keys * args.steps / dt
    sample = (f"each step: append 1 token per KV head + decode of 12 heads over {sample_keys} "
              f"cached tokens (bounded sample of the 32768-token decode-s workload)")
    print(json.dumps({
        "impl": "reference", "metric": "fused-decode keys scored/s (decode-s step: append 1 "
        "token per KV head + decode)", "value": value, "unit": "keys/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": decode_config("decode-s", args.gpus),
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": _cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}))


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_tq(a)
