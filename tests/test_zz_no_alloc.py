"""The decode entry point that allocates nothing (tq_decode_attention_noalloc).

It serves callers that cannot allocate device memory -- for example a plain C host with no
device allocator of its own, or a serving loop that must not call cudaMalloc on its hot
path. It must give the same results as tq_decode_attention, which takes a caller-allocated
workspace, on consecutive calls (the built-in scratch keeps the previous call's contents,
so the second call checks that nothing stale leaks into it). This file sorts last so a
run that stops at the first failure has run every other test before it."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_util import require_cuda, to_device
from parity import check_attention

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402


def _cache(dev, B, Hq, Hkv, N, cap, bits=3, vbits=2, seed=91):
    g = W.rng(seed)
    qg = tq.tq_build_codebook(128, bits, "prod", seed)
    cache = tq.KVCache(qg, B, Hkv, cap, value_bits=vbits, device=dev)
    k = W.round_bf16(W.scaled_gaussian_rows(g, B * Hkv * N).reshape(B, Hkv, N, 128))
    v = W.round_bf16(W.gaussian(g, (B, Hkv, N, 128)))
    tq.tq_append(qg, cache, to_device(k, torch.bfloat16), to_device(v, torch.bfloat16))
    return qg, cache, g


def test_noalloc_decode_matches_workspace_decode_twice():
    dev = require_cuda()
    qg, cache, g = _cache(dev, 2, 12, 2, 3000, 3008)
    ws = tq.alloc_decode_workspace(cache, 12, dev)
    for call in range(2):
        q = to_device(W.round_bf16(W.gaussian(g, (2, 12, 128))), torch.bfloat16)
        ref = torch.empty((2, 12, 128), device=dev, dtype=torch.float32)
        got = torch.full((2, 12, 128), float("nan"), device=dev, dtype=torch.float32)
        tq.tq_decode_attention(qg, cache, q, ref, ws)
        tq.tq_decode_attention_noalloc(qg, cache, q, got)
        torch.cuda.synchronize()
        check_attention(got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64),
                        bf16=False)
        assert torch.equal(got, ref), f"call {call}: results differ from the workspace entry point"


def test_noalloc_rejects_problems_beyond_its_scratch():
    dev = require_cuda()
    qg, cache, g = _cache(dev, 8, 512, 8, 16, 65536, seed=3)
    assert tq.tq_decode_workspace_bytes(cache, 512) > tq.TQ_NOALLOC_SCRATCH_BYTES
    q = to_device(W.gaussian(g, (8, 512, 128)), torch.float32)
    out = torch.empty((8, 512, 128), device=dev, dtype=torch.float32)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention_noalloc(qg, cache, q, out)
    assert e.value.status == tq.TQ_ETOOLARGE
