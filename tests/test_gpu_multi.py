"""GPU tests of the multi-GPU decode paths on the one GPU this run has.

- KV-head-parallel decode: three "ranks" each hold a KV-head range of the cache and decode
  their query heads (kv_head_parallel_decode, local head map); reassembled, the outputs match
  the oracle and the single-cache decode.
- Context-parallel decode through a real process group: context_parallel_decode (CUDA
  partial records, all-gather over NCCL, CUDA merge) in a world-size-1 NCCL group.
- Two gloo ranks (two processes on cuda:0, no kernel of one waits on the other): each
  computes its context slice's records with the CUDA partial kernel, the records are staged
  to the CPU and all-gathered over gloo, and each rank merges them with the CUDA merge kernel;
  both match the oracle's decode over the whole context.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import oracle_cache, require_cuda, to_device, upload_cache
from parity import check_attention

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402
from kv_cache_vector_fwht_b200.context_parallel import context_parallel_decode, context_slice  # noqa: E402
from kv_cache_vector_fwht_b200.kv_head_parallel import (default_head_map, kv_head_parallel_decode,  # noqa: E402
                                                        kv_head_slice)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(seed, B, Hq, Hkv, lengths, bits=3, vbits=2):
    g = W.rng(seed)
    N = max(lengths)
    K = W.round_bf16(W.scaled_gaussian_rows(g, B * Hkv * N).reshape(B, Hkv, N, 128))
    V = W.round_bf16(W.gaussian(g, (B, Hkv, N, 128)))
    Q = W.round_bf16(W.gaussian(g, (B, Hq, 128)))
    qo = O.build_quantizer(128, bits, "prod", seed)
    oc = oracle_cache(qo, K, V, vbits, lengths)
    return qo, oc, Q


def test_kv_head_parallel_reassembles_single_gpu_output():
    dev = require_cuda()
    B, Hq, Hkv, lengths, cap = 2, 24, 6, [700, 333], 704
    qo, oc, Q = _case(31, B, Hq, Hkv, lengths)
    qg = tq.tq_build_codebook(128, 3, "prod", 31)
    full = tq.KVCache(qg, B, Hkv, cap, value_bits=2, device=dev)
    upload_cache(full, oc)
    qt = to_device(Q, torch.bfloat16)
    out_full = torch.empty((B, Hq, 128), device=dev)
    tq.tq_decode_attention(qg, full, qt, out_full, tq.alloc_decode_workspace(full, Hq))
    hm = default_head_map(Hq, Hkv)
    got = torch.full((B, Hq, 128), float("nan"), device=dev)
    world = 4   # 6 KV heads over 4 ranks: 2, 2, 1, 1
    for r in range(world):
        a, b = kv_head_slice(Hkv, r, world)
        local = {k: (v[:, a:b] if k != "len" else v) for k, v in oc.items() if v is not None}
        c = tq.KVCache(qg, B, b - a, cap, value_bits=2, device=dev)
        upload_cache(c, local)
        n_local = sum(1 for h in range(Hq) if a <= hm[h] < b)
        out = torch.empty((B, n_local, 128), device=dev)
        ws = tq.alloc_decode_workspace(c, n_local)
        qs = kv_head_parallel_decode(qg, c, qt, out, ws, a, b, head_map=hm)
        assert len(qs) == n_local
        got[:, qs] = out
    torch.cuda.synchronize()
    g = got.cpu().numpy()
    assert not np.isnan(g).any()
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=2)
    check_attention(g, ref, False)
    # the same heads, decoded by the same kernel over a smaller cache: equal up to the
    # rounding order of the context splits
    assert np.max(np.abs(g - out_full.cpu().numpy())) < 1e-5


def test_context_parallel_decode_world_size_one_nccl():
    import torch.distributed as dist
    dev = require_cuda()
    B, Hq, Hkv, lengths, cap = 2, 8, 2, [900, 450], 912
    qo, oc, Q = _case(33, B, Hq, Hkv, lengths)
    qg = tq.tq_build_codebook(128, 3, "prod", 33)
    cache = tq.KVCache(qg, B, Hkv, cap, value_bits=2, device=dev)
    upload_cache(cache, oc)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=dev)
    try:
        out = torch.empty((B, Hq, 128), device=dev)
        parts = context_parallel_decode(qg, cache, to_device(Q, torch.bfloat16), out,
                                        tq.alloc_decode_workspace(cache, Hq))
        torch.cuda.synchronize()
        assert tuple(parts.shape) == (1, B, Hq, tq.TQ_PART_FLOATS)
    finally:
        dist.destroy_process_group()
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=2)
    check_attention(out.cpu().numpy(), ref, False)


def _gloo_rank(rank: int, world: int, port: int, q_out):
    try:
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                          MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import torch
        import torch.distributed as dist

        import kv_cache_vector_fwht_b200 as tqm
        from gpu_util import upload_cache as up
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        B, Hq, Hkv, lengths = 2, 8, 2, [1000, 610]
        qo, oc, Q = _case(35, B, Hq, Hkv, lengths)
        qg = tqm.tq_build_codebook(128, 3, "prod", 35)
        a, b = context_slice(max(lengths), rank, world)
        sl = {k: v[:, :, a:b] for k, v in oc.items() if k != "len" and v is not None}
        sl["len"] = np.clip(np.asarray(oc["len"]) - a, 0, b - a)
        c = tqm.KVCache(qg, B, Hkv, ((b - a) + 15) // 16 * 16, value_bits=2, device=dev)
        up(c, sl)
        part = torch.empty((B, Hq, tqm.TQ_PART_FLOATS), device=dev)
        tqm.tq_decode_attention_partial(qg, c, to_device(Q, torch.bfloat16), part,
                                        tqm.alloc_decode_workspace(c, Hq))
        torch.cuda.synchronize()
        rec = part.cpu()                      # staged to the host for the gloo exchange
        parts = [torch.empty_like(rec) for _ in range(world)]
        dist.all_gather(parts, rec)
        out = torch.empty((B, Hq, 128), device=dev)
        tqm.tq_merge_partials(torch.stack(parts).to(dev).contiguous(), out)
        torch.cuda.synchronize()
        ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=2)
        err = check_attention(out.cpu().numpy(), ref, False)
        dist.destroy_process_group()
        q_out.put((rank, float(err)))
    except Exception as e:  # report instead of hanging the parent
        q_out.put((rank, "error: " + repr(e)))


def test_two_gloo_ranks_merge_cuda_partial_records():
    require_cuda()
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=600) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, err in results:
        assert not isinstance(err, str), err
