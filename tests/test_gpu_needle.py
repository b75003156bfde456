"""Needle retrieval through the GPU path (validate_paper.py test_needle_retrieval_depths and the
chunked 8192-token needle test): a large key ("needle", x3.0) hidden among small keys (x0.02)
is found by its own query at every depth and for every KV head, both from the fused decode
scores and from <q, x_hat> over tq_dequantize_keys, and attention then returns the needle's
dequantized value. Keys and values enter the cache through tq_append; the expected value
row comes from the oracle's value quantizer on the same fp32 input."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import require_cuda

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402

D = 128


def _haystack(g, n_kv, n, positions):
    keys = (g.standard_normal((1, n_kv, n, D)) * 0.02).astype(np.float32)
    vals = g.standard_normal((1, n_kv, n, D)).astype(np.float32)
    needles = (g.standard_normal((n_kv, D)) * 3.0).astype(np.float32)
    for h in range(n_kv):
        keys[0, h, positions[h]] = needles[h]
    return keys, vals, needles


def _check_retrieval(qz, cache, needles, positions, vals, n, value_bits):
    dev = needles.device
    n_kv = needles.shape[0]
    scores = torch.empty((1, n_kv, cache.capacity), device=dev)
    ws = tq.alloc_decode_workspace(cache, n_kv)
    out = torch.empty((1, n_kv, D), device=dev)
    tq.tq_decode_attention(qz, cache, needles.reshape(1, n_kv, D), out, ws,
                           head_map=list(range(n_kv)), scores=scores)
    xhat = torch.empty((cache.capacity, D), device=dev)
    found_dec, found_deq = [], []
    for h in range(n_kv):
        planes = {k: (v[cache.rows(0, h)] if v is not None else None)
                  for k, v in cache.key_planes().items()}
        tq.tq_dequantize_keys(qz, planes, xhat)
        found_deq.append(int(torch.argmax(xhat[:n] @ needles[h])))
        found_dec.append(int(torch.argmax(scores[0, h, :n])))
    torch.cuda.synchronize()
    assert found_dec == list(positions), (found_dec, positions)
    assert found_deq == list(positions), (found_deq, positions)
    # the needle's logit exceeds every other by ~100 (x3.0 vs x0.02 at d = 128): the output is
    # its dequantized value row up to fp32 rounding
    for h in range(n_kv):
        row = vals[0, h, positions[h]][None].astype(np.float64)
        pv = O.quantize_values(row, value_bits)
        want = O.dequantize_values(pv["q"], pv["params"], value_bits, D)[0]
        np.testing.assert_allclose(out[0, h].cpu().numpy(), want, rtol=0, atol=2e-4)


@pytest.mark.parametrize("mode,bits", [("prod", 3), ("prod", 4), ("mse", 3)])
def test_needle_at_five_depths(mode, bits):
    """H_kv = 4, N = 4096, value 2-bit group 32; one append of the whole context."""
    dev = require_cuda()
    n_kv, n = 4, 4096
    qz = tq.tq_build_codebook(D, bits, mode, 42)
    for d_i, depth in enumerate((0.05, 0.25, 0.5, 0.75, 0.95)):
        g = np.random.default_rng(1000 * bits + d_i)
        pos = [int(n * depth) + 7 * h for h in range(n_kv)]
        keys, vals, needles = _haystack(g, n_kv, n, pos)
        cache = tq.KVCache(qz, 1, n_kv, n, value_bits=2, device=dev)
        tq.tq_append(qz, cache, torch.from_numpy(keys).to(dev), torch.from_numpy(vals).to(dev))
        _check_retrieval(qz, cache, torch.from_numpy(needles).to(dev), pos, vals, n, 2)


def test_needle_in_chunked_8192():
    """8192 tokens appended in chunks of 1024 (the pages' chunked store), needle at 5555."""
    dev = require_cuda()
    n_kv, n, chunk = 2, 8192, 1024
    qz = tq.tq_build_codebook(D, 3, "prod", 42)
    g = np.random.default_rng(5555)
    pos = [5555, 5555]
    keys, vals, needles = _haystack(g, n_kv, n, pos)
    cache = tq.KVCache(qz, 1, n_kv, n, value_bits=2, device=dev)
    kd, vd = torch.from_numpy(keys).to(dev), torch.from_numpy(vals).to(dev)
    for c0 in range(0, n, chunk):
        tq.tq_append(qz, cache, kd[:, :, c0:c0 + chunk].contiguous(),
                     vd[:, :, c0:c0 + chunk].contiguous())
    assert cache.lengths == [n]
    _check_retrieval(qz, cache, torch.from_numpy(needles).to(dev), pos, vals, n, 2)
