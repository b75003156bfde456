"""Benchmark of the TurboQuant hot path on B200: one JSON line.

Headline workload (decode-stream): batch 1 per GPU, 64 query heads on 8 KV heads, d = 128, a
131072-token packed cache (keys 4-bit prod = 3-bit Lloyd-Max MSE in 4-bit fields + 1-bit QJL,
values 4-bit groups of 32, fp16 norms and group parameters), bf16 synthetic inputs (keys
N(0,1) x U[2,20] per row, values and queries N(0,1)). One step = append one new token per KV
head (quantize its key and value, write them at len, advance len) + fused decode attention of
one query token over the whole cache. Metric: keys scored per second (query heads x cached
tokens / step time).

The same line carries every other configuration, each timed the same way:
  decode_s       batch 1, 12/2 heads, 32768 tokens, 3-bit prod keys, 2-bit values
  decode_l       batch 8, 28/4 heads, 32768 tokens, 16 planted keys per (sequence, KV head)
  score          4096 fp32 keys quantized (3-bit prod) then scored by 8 queries (key-only cache)
  key_quantize   2^24 bf16 rows (4 layers x 2^22, quantizer seed = layer), every mode and
                 width: mse b=1..4, prod b=2..4, grouped b=1..3

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]

L2 is flushed (a 256 MiB write) before every timed decode step, outside its events; the
key-quantize inputs (4 GiB) exceed L2. Multi-GPU runs are independent replicas (weak scaling):
each rank holds its own batch, no collective on the data path; times are the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# decode workloads (synthetic, seeded): keys N(0,1) x per-row U[2,20], values N(0,1), bf16
DECODE_WORKLOADS = {
    "decode-s": dict(batch=1, n_q_heads=12, n_kv_heads=2, ctx=32768, key_bits=3, value_bits=2,
                     group=32, qseed=0, planted=0, data_seed=2),
    "decode-l": dict(batch=8, n_q_heads=28, n_kv_heads=4, ctx=32768, key_bits=3, value_bits=2,
                     group=32, qseed=0, planted=16, data_seed=3),
    "decode-stream": dict(batch=1, n_q_heads=64, n_kv_heads=8, ctx=131072, key_bits=4,
                          value_bits=4, group=32, qseed=0, planted=0, data_seed=5),
}
HEADLINE = "decode-stream"
WL_DESC = {
    "decode-s": "decode-s: batch 1, 12 q heads / 2 kv heads, d 128, ctx 32768, keys 3-bit prod, "
                "values 2-bit g32",
    "decode-l": "decode-l: batch 8, 28 q heads / 4 kv heads, d 128, ctx 32768 + 16 planted keys "
                "per (sequence, kv head), keys 3-bit prod, values 2-bit g32",
    "decode-stream": "decode-stream: batch 1, 64 q heads / 8 kv heads, d 128, ctx 131072 + "
                     "streaming append, keys 4-bit prod, values 4-bit g32",
}
QUANT_MODES = [("mse", 1), ("mse", 2), ("mse", 3), ("mse", 4), ("prod", 2), ("prod", 3),
               ("prod", 4), ("grouped", 1), ("grouped", 2), ("grouped", 3)]
# kernel launches of one tq_append_decode step: the fused append and the fused decode
LAUNCHES_PER_STEP = 2
DECODE_SOURCES = ["decode_kernel.cuh", "decode.cu", "decode_prod.cu", "decode_mse.cu",
                  "decode_grp.cu", "tq_device.cuh", "tq_internal.h"]


def key_bytes(bits):      # prod mode: (bits - 1)-bit indices (3-bit stored in 4) + signs + norms
    w = {1: 1, 2: 2, 3: 4}[bits - 1]
    return 128 * w // 8 + 16 + 4


def value_bytes(vb):
    return 128 * vb // 8 + 16


def decode_config(name: str, world: int) -> dict:
    """The `config` of a decode workload's JSON line (both arms)."""
    wl = DECODE_WORKLOADS[name]
    return {"workload": WL_DESC[name], "global_batch": wl["batch"] * world, "seq_len": wl["ctx"],
            "parallelism": f"replicas x{world}",
            "l2": "flushed (256 MiB write) before each timed step, outside its events",
            "data_types": "bf16 query and new K/V rows, u8 packed cache, fp16 norms and value "
                          "params (the arithmetic type is the line's dtype)"}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-extras", action="store_true",
                    help="headline workload only (no decode-s / decode-l / score / quantize)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "decode", "quantize"],
                    help="one leg only, no JSON contract (small cases for profiling)")
    ap.add_argument("--quantize-rows", type=int, default=1 << 22, help="rows per layer")
    ap.add_argument("--decode-workload", default=HEADLINE, choices=sorted(DECODE_WORKLOADS),
                    help="with --only decode: the decode workload to time")
    ap.add_argument("--quantize-mode", default="all",
                    choices=["all"] + [f"{m}{b}" for m, b in QUANT_MODES],
                    help="with --only quantize: one mode and width, or all")
    ap.add_argument("--extra-steps", type=int, default=200,
                    help="timed steps of each non-headline decode workload")
    ap.add_argument("--key-only", action="store_true",
                    help="with --only decode: a key-only cache decoded without outputs (the "
                         "table lookups alone)")
    return ap.parse_args(argv)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _code_only(text: str) -> str:
    """C/CUDA source without its comments and trailing blanks: what the compiler sees, so that
    editing a comment does not orphan the traffic recorded for the code. (The kernel sources
    put no comment markers inside string literals.)"""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_sha(files) -> str:
    """Short hash of the kernel sources' code (the key under which ncu DRAM traffic was
    recorded)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "kv_cache_vector_fwht_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, sha: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the ncu summaries in
    profiles/dram_traffic.txt, or None when absent or recorded for other kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split("#", 1)[0].split()
                if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload:
                    return float(parts[3]) if parts[2] == sha else None
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs (read-only query)."""
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
class DecodeBench:
    """A decode workload on the device: the prefilled packed cache, fresh tokens and queries
    for every step, the decode workspace and the L2 flush buffer."""

    def __init__(self, tq, torch, dev, name: str, n_steps: int, rank: int, key_only=False):
        wl = DECODE_WORKLOADS[name]
        self.name, self.wl, self.tq, self.torch, self.dev = name, wl, tq, torch, dev
        B, Hq, Hkv, N = wl["batch"], wl["n_q_heads"], wl["n_kv_heads"], wl["ctx"]
        self.B, self.Hq, self.Hkv, self.N = B, Hq, Hkv, N
        extra = n_steps + 8
        g = torch.Generator(device=dev).manual_seed(wl["data_seed"] + 1000 * rank)
        K = torch.randn((B, Hkv, N, 128), generator=g, device=dev)
        K *= torch.empty((B, Hkv, N, 1), device=dev).uniform_(2.0, 20.0, generator=g)
        V = torch.randn((B, Hkv, N, 128), generator=g, device=dev).to(torch.bfloat16)
        self.Kn = (torch.randn((extra, B, Hkv, 1, 128), generator=g, device=dev) *
                   torch.empty((extra, B, Hkv, 1, 1), device=dev).uniform_(2.0, 20.0, generator=g)
                   ).to(torch.bfloat16)
        self.Vn = torch.randn((extra, B, Hkv, 1, 128), generator=g, device=dev).to(torch.bfloat16)
        self.Qs = torch.randn((extra, B, Hq, 128), generator=g, device=dev).to(torch.bfloat16)
        if wl["planted"]:
            # 16 seeded positions per (sequence, KV head): 0.9 q + 0.1 N(0,1), q = the first
            # query head of that KV head's group; every step of this workload uses that query
            grp = Hq // Hkv
            self.Qs[:] = self.Qs[0:1].clone()
            q0 = self.Qs[0].float()
            for b in range(B):
                for h in range(Hkv):
                    pos = torch.randperm(N, generator=g, device=dev)[:wl["planted"]]
                    noise = torch.randn((wl["planted"], 128), generator=g, device=dev)
                    K[b, h, pos] = 0.9 * q0[b, h * grp][None, :] + 0.1 * noise
        K = K.to(torch.bfloat16)
        self.qz = tq.tq_build_codebook(128, wl["key_bits"], "prod", wl["qseed"])
        cap = ((N + extra + 15) // 16) * 16
        self.key_only = key_only
        vb = 0 if key_only else wl["value_bits"]
        self.cache = tq.KVCache(self.qz, B, Hkv, cap, value_bits=vb, device=dev)
        tq.tq_append(self.qz, self.cache, K.contiguous(), None if key_only else V.contiguous())
        del K, V
        self.ws = tq.alloc_decode_workspace(self.cache, Hq, dev)
        self.out = None if key_only else torch.empty((B, Hq, 128), device=dev, dtype=torch.bfloat16)
        self.flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.i = 0

    def step(self):
        """One decode step through the public API: append this step's token per KV head,
        then decode (one tq_append_decode call)."""
        i = self.i
        if self.key_only:   # the decode's table lookups alone (no values, no outputs)
            self.tq.tq_decode_attention(self.qz, self.cache, self.Qs[i], None, self.ws)
        else:
            self.tq.tq_append_decode(self.qz, self.cache, self.Kn[i], self.Vn[i], self.Qs[i],
                                     self.out, self.ws)
        self.i += 1

    def bytes_per_step(self, mean_len: float) -> float:
        """Algorithmic HBM bytes of one step: the cache read by the decode, the appended rows
        (bf16 in, packed out), the query and the output."""
        wl = self.wl
        if self.key_only:   # keys read, the query; no append, no values, no output
            return self.B * self.Hkv * mean_len * key_bytes(wl["key_bits"]) + self.B * self.Hq * 256
        per = key_bytes(wl["key_bits"]) + value_bytes(wl["value_bits"])
        return (self.B * self.Hkv * mean_len * per
                + self.B * self.Hkv * (2 * 256 + per)
                + self.B * self.Hq * 128 * 2 * 2)

    def run(self, steps: int, warm: int, world: int, clocks=None):
        """Warm-up steps, then `steps` timed steps (events on the launching stream around each
        step, L2 flushed before each, outside the events). Returns a result dict."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        for _ in range(warm):
            self.flush.zero_()
            self.step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        lens = []
        if clocks:
            clocks.start()
        barrier(world)
        t_wall = time.perf_counter()
        for s in range(steps):
            self.flush.zero_()
            e0, e1 = ev[s]
            e0.record(stream)
            self.step()
            e1.record(stream)
            lens.append(self.cache.lengths[0])
        barrier(world)
        t_wall = time.perf_counter() - t_wall
        clk = clocks.stop() if clocks else None
        self.tq.tq_sync_status()
        step_ms = [a.elapsed_time(c) for a, c in ev]
        tot_ms = sum(step_ms)
        keys_scored = float(sum(self.Hq * L for L in lens) * self.B)
        value, tot_ms_max = replica_throughput(keys_scored, tot_ms, world)
        ms_step = tot_ms_max / steps
        mean_len = sum(lens) / len(lens)
        nbytes = self.bytes_per_step(mean_len)
        peak, peak_kind = load_peaks()
        achieved = nbytes / (ms_step / 1e3) / 1e9
        sha = source_sha(DECODE_SOURCES)
        return {
            "value": value, "unit": "keys/s", "ms_per_step": ms_step, "steps": steps,
            "warmup": warm, "mean_len": mean_len, "wall_s_timed_region": t_wall,
            "clocks": clk,
            "roofline": {
                "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": recorded_traffic("k_decode", self.name, sha),
                "kernel": "k_decode (with the k_append it follows in each step)",
                "bytes_per_launch": nbytes, "avg_launch_us": ms_step * 1e3,
                "time_basis": "whole step (append + decode, one tq_append_decode call): an "
                              "upper bound of the decode kernel's own time",
                "peak_kind": f"{peak_kind} (hbm_gbs, burst)", "source_sha": sha},
        }

    def e2e(self, steps: int, world: int):
        """The same step end to end through the public API with host buffers: each step's new
        keys, values and query sit in one pinned host row and reach the device in one copy;
        the output is read back to pinned host memory; synchronize; host wall clock."""
        torch, tq = self.torch, self.tq
        Kn, Vn, Qs = self.Kn, self.Vn, self.Qs
        nk, nv, nq = Kn[0].numel(), Vn[0].numel(), Qs[0].numel()
        stage_h = torch.empty((steps, nk + nv + nq), dtype=Kn.dtype).pin_memory()
        stage_h[:, :nk] = Kn[:steps].reshape(steps, nk).cpu()
        stage_h[:, nk:nk + nv] = Vn[:steps].reshape(steps, nv).cpu()
        stage_h[:, nk + nv:] = Qs[:steps].reshape(steps, nq).cpu()
        oh = torch.empty((self.B, self.Hq, 128), dtype=torch.bfloat16).pin_memory()
        stage_d = torch.empty((nk + nv + nq,), dtype=Kn.dtype, device=self.dev)
        kd = stage_d[:nk].view(Kn[0].shape)
        vd = stage_d[nk:nk + nv].view(Vn[0].shape)
        qd = stage_d[nk + nv:].view(Qs[0].shape)
        self.cache.set_lengths([self.N] * self.B)
        e2e_ms = 0.0
        for s in range(steps):
            self.flush.zero_()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            stage_d.copy_(stage_h[s], non_blocking=True)
            tq.tq_append_decode(self.qz, self.cache, kd, vd, qd, self.out, self.ws)
            oh.copy_(self.out, non_blocking=True)
            torch.cuda.synchronize()
            e2e_ms += (time.perf_counter() - t0) * 1e3
        keys = float(sum(self.Hq * (self.N + s + 1) for s in range(steps)) * self.B)
        ms_max = max_over_ranks(e2e_ms, world)
        return {"value": sum_over_ranks(keys, world) / (ms_max / 1e3), "unit": "keys/s",
                "h2d_bytes_per_step": int((kd.numel() + vd.numel() + qd.numel()) * 2),
                "d2h_bytes_per_step": int(oh.numel() * 2), "steps": steps,
                "ms_per_step": ms_max / steps}


def bench_score(tq, torch, dev, world, steps=200, warm=10):
    """The score workload: 4096 fp32 keys (N(0,1) x U[2,20] per row) quantized to 3-bit prod
    into a key-only cache, then scored by 8 fp32 queries on one KV head (raw estimates written
    to a 8 x 4096 fp32 matrix). One step = tq_quantize_keys + tq_decode_attention."""
    g = torch.Generator(device=dev).manual_seed(1)
    n, nq = 4096, 8
    keys = torch.randn((n, 128), generator=g, device=dev)
    keys *= torch.empty((n, 1), device=dev).uniform_(2.0, 20.0, generator=g)
    qv = torch.randn((1, nq, 128), generator=g, device=dev)
    qz = tq.tq_build_codebook(128, 3, "prod", 0)
    cache = tq.KVCache(qz, 1, 1, n, value_bits=0, device=dev)
    cache.set_lengths([n])
    planes = cache.key_planes()
    scores = torch.empty((1, nq, n), device=dev)
    ws = tq.alloc_decode_workspace(cache, nq, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        tq.tq_quantize_keys(qz, keys, planes)
        tq.tq_decode_attention(qz, cache, qv, None, ws, scores=scores)

    for _ in range(warm):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s in range(steps):
        flush.zero_()
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    tq.tq_sync_status()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    ms_max = max_over_ranks(ms, world)
    return {"workload": "score: 4096 fp32 keys (N(0,1) x U[2,20]) -> 3-bit prod, 8 fp32 queries "
                        "-> 8 x 4096 raw scores", "us_per_step": ms_max * 1e3,
            "keys_per_s": world * n / (ms_max / 1e3),
            "scores_per_s": world * n * nq / (ms_max / 1e3),
            "note": "latency-bound (2.5 MB per step); no HBM fraction target"}


def bench_quantize(tq, torch, dev, world, rows=1 << 22, reps=5, modes=QUANT_MODES):
    """Key-quantize throughput over the quantize workload: 4 layers x `rows` bf16 rows, N(0,1)
    with 32 fixed channels at 4x std, quantizer seed = layer; one timed pass = all 4 layers
    (tq_quantize_keys per layer). Inputs (4 GiB at 2^22 rows per layer) exceed L2."""
    import workloads as W
    ch_np = W.outlier_channels(4)
    ch = torch.from_numpy(ch_np).long().to(dev)
    g = torch.Generator(device=dev).manual_seed(4)
    xs = []
    for _ in range(4):
        x = torch.randn((rows, 128), generator=g, device=dev)
        x[:, ch] *= 4.0
        xs.append(x.to(torch.bfloat16))
        del x
    # output planes sized for the widest layout (64 index bytes, 16 sign bytes, 2 norms)
    bufs = [dict(idx=torch.empty((rows, 64), dtype=torch.uint8, device=dev),
                 signs=torch.empty((rows, 16), dtype=torch.uint8, device=dev),
                 norms=torch.empty((rows, 2), dtype=torch.int16, device=dev)) for _ in range(4)]
    peak, peak_kind = load_peaks()
    st = torch.cuda.current_stream()
    out = {}
    for mode, bits in modes:
        qs = [tq.tq_build_codebook(128, bits, mode, layer, ch_np if mode == "grouped" else None)
              for layer in range(4)]
        lay = qs[0].layout
        # contiguous per-layout views: the library writes idx_bytes per row at that stride
        planes = [dict(idx=bf["idx"].view(-1)[:rows * lay["idx_bytes"]].view(rows, lay["idx_bytes"]),
                       signs=(bf["signs"] if lay["sign_bytes"] else None),
                       norms=bf["norms"].view(-1)[:rows * lay["n_norms"]].view(rows, lay["n_norms"]))
                  for bf in bufs]
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
        ms = max_over_ranks(sum(times) / len(times), world)
        n = 4 * rows
        out_bytes = lay["idx_bytes"] + lay["sign_bytes"] + 2 * lay["n_norms"]
        gbs = world * n * (256 + out_bytes) / (ms / 1e3) / 1e9
        kernel = {"prod": f"k_keys_tc<prod,{bits - 1}>", "mse": f"k_keys_tc<mse,{bits}>",
                  "grouped": f"k_keys_grp_tc<{bits}>"}[mode]
        out[f"{mode}{bits}"] = {
            "rows_per_s": world * n / (ms / 1e3), "ms_per_pass": ms, "rows_per_pass": n,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": None, "bytes_per_row": 256 + out_bytes,
                         "kernel": kernel, "peak_kind": f"{peak_kind} (hbm_gbs, burst)"}}
        del qs
    del xs, bufs
    torch.cuda.empty_cache()
    return out


def run_tq(args):
    import torch

    import kv_cache_vector_fwht_b200 as tq

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    steps, warm = args.steps, max(3, args.warmup)

    if args.only == "quantize":
        modes = QUANT_MODES if args.quantize_mode == "all" else \
            [(args.quantize_mode[:-1], int(args.quantize_mode[-1]))]
        r = bench_quantize(tq, torch, dev, world, rows=args.quantize_rows, modes=modes)
        if rank == 0:
            print(json.dumps({"key_quantize": r}))
        return _finish(world)
    if args.only == "decode":
        d = DecodeBench(tq, torch, dev, args.decode_workload, warm + steps, rank,
                        key_only=args.key_only)
        r = d.run(steps, warm, world)
        if rank == 0:
            print(json.dumps({args.decode_workload: r}))
        return _finish(world)

    # ---- headline: decode-stream steps (append 1 token per KV head + decode)
    head = DecodeBench(tq, torch, dev, HEADLINE, warm + steps + 1024, rank)
    r = head.run(steps, warm, world, clocks=ClockSampler(local))
    e2e = None if args.no_e2e else head.e2e(min(steps, 500), world)
    del head
    torch.cuda.empty_cache()
    wl = DECODE_WORKLOADS[HEADLINE]
    result = {
        "metric": "fused-decode keys scored/s (decode-stream step: append 1 token per KV head + "
                  "decode over the packed cache)",
        "value": r["value"], "unit": "keys/s", "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded torch CUDA generator; keys N(0,1) x U[2,20] per row, values "
                "and queries N(0,1))",
        "config": decode_config(HEADLINE, world),
        "decode_gbs": r["roofline"]["achieved"],
        "roofline": r["roofline"],
        "e2e": e2e,
        "gpu_launches": steps * LAUNCHES_PER_STEP,
        "clocks": r["clocks"],
        "wall_s_timed_region": r["wall_s_timed_region"],
        "mean_context": r["mean_len"],
        "keys_per_step": wl["n_q_heads"] * r["mean_len"] * wl["batch"],
    }
    if not args.no_extras:
        es = max(3, min(steps, args.extra_steps))
        for name, key in (("decode-s", "decode_s"), ("decode-l", "decode_l")):
            d = DecodeBench(tq, torch, dev, name, warm + es, rank)
            x = d.run(es, warm, world)
            x.pop("clocks", None)
            x["config"] = decode_config(name, world)
            result[key] = x
            del d
            torch.cuda.empty_cache()
        result["score"] = bench_score(tq, torch, dev, world)
        result["key_quantize"] = bench_quantize(tq, torch, dev, world, rows=args.quantize_rows)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(HEADLINE)
    if rank == 0:
        print(json.dumps(result))
    return _finish(world)


def _finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ oracle
def _oracle_worker(job):
    """One KV head of a decode workload on the oracle, in a spawned single-threaded process:
    quantize a sample context once, then `iters` steps of (quantize one new key and value,
    decode the KV head's query heads over the sample). Returns (iters done, seconds)."""
    name, kv, sample, seconds, max_iters = job
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"
    import numpy as np
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    import oracle as O
    import workloads as W
    wl = DECODE_WORKLOADS[name]
    G = wl["n_q_heads"] // wl["n_kv_heads"]
    g = W.rng(wl["data_seed"] * 100 + kv)
    K = W.round_bf16(W.scaled_gaussian_rows(g, sample + 1))
    V = W.round_bf16(W.gaussian(g, (sample + 1, 128)))
    Q = W.round_bf16(W.gaussian(g, (1, G, 128)))
    qo = O.build_quantizer(128, wl["key_bits"], "prod", wl["qseed"])
    p = O.quantize_keys(qo, K[:sample].astype(np.float64))
    v = O.quantize_values(V[:sample].astype(np.float64), wl["value_bits"])
    cache = dict(k_idx=p["idx"][None, None], k_signs=p["signs"][None, None],
                 k_norms=p["norms"][None, None], v_q=v["q"][None, None],
                 v_params=v["params"][None, None], len=np.array([sample]))

    def step():
        O.quantize_keys(qo, K[sample:].astype(np.float64))
        O.quantize_values(V[sample:].astype(np.float64), wl["value_bits"])
        O.decode_attention(qo, cache, Q.astype(np.float64), value_bits=wl["value_bits"])

    step()
    n, t0 = 0, time.perf_counter()
    while n < max_iters and (time.perf_counter() - t0 < seconds or n == 0):
        step()
        n += 1
    return n, time.perf_counter() - t0


def oracle_decode_rate(name: str, sample: int, seconds: float, max_iters: int = 1 << 30):
    """The oracle (fp64 numpy, as it stands) on the host cores: one spawned single-threaded
    process per KV head of the workload (at most the host's core count), each timing decode
    steps of its query heads over a `sample`-token context. Returns (keys scored/s, cores,
    steps per KV head, seconds)."""
    import multiprocessing as mp
    wl = DECODE_WORKLOADS[name]
    cores = max(1, min(os.cpu_count() or 1, wl["n_kv_heads"]))
    jobs = [(name, kv, sample, seconds, max_iters) for kv in range(wl["n_kv_heads"])]
    ctx = mp.get_context("spawn")
    with ctx.Pool(cores) as pool:
        res = pool.map(_oracle_worker, jobs, chunksize=1)
    G = wl["n_q_heads"] // wl["n_kv_heads"]
    # every KV head's worker ran concurrently with the others (or in waves of `cores`)
    waves = -(-wl["n_kv_heads"] // cores)
    wall = max(t for _, t in res) * waves
    keys = sum(n * G * sample for n, _ in res) * wl["batch"]
    return keys / wall, cores, min(n for n, _ in res), wall


def cpu_baseline(name: str, sample: int = 4096, seconds: float = 12.0):
    value, cores, n, wall = oracle_decode_rate(name, sample, seconds)
    wl = DECODE_WORKLOADS[name]
    return {"value": value, "unit": "keys/s", "cores": cores, "kind": "oracle",
            "sample": f"{name}: {wl['n_kv_heads']} KV heads x {wl['n_q_heads'] // wl['n_kv_heads']}"
                      f" query heads over a {sample}-token sample context (of {wl['ctx']}), "
                      f">= {n} steps of (append 1 token + decode) per KV head, one "
                      f"single-threaded process per KV head, {wall:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = HEADLINE
    sample = 2048
    # about two minutes in all: warm-up and timed steps as the arguments ask
    t_one = oracle_decode_rate(name, sample, 0.0, max_iters=1)[3]
    per_step = 100.0 / max(1, args.steps + args.warmup)
    if t_one > per_step:
        sample = max(64, int(sample * per_step / t_one) // 16 * 16)
    oracle_decode_rate(name, sample, 0.0, max_iters=max(1, args.warmup))
    value, cores, n, wall = oracle_decode_rate(name, sample, 0.0, max_iters=args.steps)
    wl = DECODE_WORKLOADS[name]
    sample_txt = (f"each step: append 1 token per KV head + decode of {wl['n_q_heads']} heads over "
                  f"a {sample}-token sample context (bounded sample of the {wl['ctx']}-token "
                  f"{name} workload), one single-threaded process per KV head")
    print(json.dumps({
        "impl": "reference",
        "metric": "fused-decode keys scored/s (decode-stream step: append 1 token per KV head + "
                  "decode over the packed cache)",
        "value": value, "unit": "keys/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": wall * 1e3 / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": decode_config(name, args.gpus),
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": cores, "kind": "oracle",
                         "sample": sample_txt},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}))


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_tq(a)
