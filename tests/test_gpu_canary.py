"""Writes stay inside their rows: canary bytes around every output the hot calls produce.

tq_quantize_keys and tq_quantize_values write n_rows rows of planes that are allocated with
extra rows filled with a canary byte; tq_append writes rows [len, len + n) of each (sequence,
KV head) of a cache whose every other row holds the canary (both the fused path for up to 64
new rows and the separate quantize kernels beyond it). The prefix test runs a contiguous
2^20-row block of the quantize workload's first layer (quantizer seed 0) through prod b=3 and
checks every row against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import require_cuda, to_device, to_np_planes
from parity import check_key_parity

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402

CANARY = 0xA5


def _fill(t):
    t.view(torch.uint8).fill_(CANARY)


def _untouched(t, rows):
    a = t.view(torch.uint8).cpu().numpy().reshape(t.shape[0], -1)
    return bool(np.all(a[rows] == CANARY))


@pytest.mark.parametrize("mode,bits", [("prod", 3), ("mse", 1), ("mse", 4), ("grouped", 1),
                                       ("grouped", 3)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_keys_leaves_rows_past_n(mode, bits, dtype):
    dev = require_cuda()
    ch = W.outlier_channels(4)
    outl = ch if mode == "grouped" else None
    qg = tq.tq_build_codebook(128, bits, mode, 5, outl)
    for n in (1, 129, 1000):
        extra = 40
        planes = qg.alloc_key_planes(n + extra, dev)
        for t in planes.values():
            if t is not None:
                _fill(t)
        x = to_device(W.outlier_rows(W.rng(n), n, ch), dtype)
        view = {k: (v[:n] if v is not None else None) for k, v in planes.items()}
        tq.tq_quantize_keys(qg, x, view)
        torch.cuda.synchronize()
        for name, t in planes.items():
            if t is not None:
                assert _untouched(t, slice(n, n + extra)), (mode, bits, n, name)


@pytest.mark.parametrize("bits", [2, 4])
def test_quantize_values_leaves_rows_past_n(bits):
    dev = require_cuda()
    for n in (1, 33, 777):
        planes = tq.alloc_value_planes(n + 16, bits, device=dev)
        for t in planes.values():
            _fill(t)
        v = to_device(W.gaussian(W.rng(n), (n, 128)), torch.bfloat16)
        tq.tq_quantize_values(v, {k: t[:n] for k, t in planes.items()}, bits)
        torch.cuda.synchronize()
        for name, t in planes.items():
            assert _untouched(t, slice(n, n + 16)), (bits, n, name)


@pytest.mark.parametrize("mode,bits,vbits", [("prod", 3, 2), ("prod", 4, 4), ("mse", 2, 4)])
@pytest.mark.parametrize("n_new", [1, 5, 100])   # 100 rows: the separate quantize kernels
def test_append_writes_only_its_rows(mode, bits, vbits, n_new):
    dev = require_cuda()
    qg = tq.tq_build_codebook(128, bits, mode, 6)
    B, H, cap = 2, 3, 320
    cache = tq.KVCache(qg, B, H, cap, value_bits=vbits, device=dev)
    planes = [cache.k_idx, cache.k_signs, cache.k_norms, cache.v_q, cache.v_params]
    for t in planes:
        if t is not None:
            _fill(t)
    lens = [17, 200]
    cache.set_lengths(lens)
    k = to_device(W.scaled_gaussian_rows(W.rng(3), B * H * n_new).reshape(B, H, n_new, 128),
                  torch.bfloat16)
    v = to_device(W.gaussian(W.rng(4), (B, H, n_new, 128)), torch.bfloat16)
    tq.tq_append(qg, cache, k, v)
    torch.cuda.synchronize()
    assert cache.lengths == [L + n_new for L in lens]
    assert cache.len_dev.cpu().tolist() == [L + n_new for L in lens]
    for t in planes:
        if t is None:
            continue
        a = t.view(torch.uint8).cpu().numpy().reshape(B * H, cap, -1)
        for b in range(B):
            for h in range(H):
                r = a[b * H + h]
                lo, hi = lens[b], lens[b] + n_new
                assert np.all(r[:lo] == CANARY), (b, h, "below len")
                assert np.all(r[hi:] == CANARY), (b, h, "past len + n")
                assert not np.all(r[lo:hi] == CANARY), (b, h, "not written")


def test_quantize_workload_prefix_2_20_rows_prod3():
    """A contiguous 2^20-row block of the quantize workload's layer 0 (rows N(0,1) with the
    32 fixed channels at 4x std, bf16; quantizer seed 0), 3-bit prod: every row against the
    oracle."""
    dev = require_cuda()
    n = 1 << 20
    ch = W.outlier_channels(4)
    x = W.quantize_rows_numpy(0, n, ch)
    qg = tq.tq_build_codebook(128, 3, "prod", 0)
    qo = O.build_quantizer(128, 3, "prod", 0)
    planes = qg.alloc_key_planes(n, dev)
    tq.tq_quantize_keys(qg, to_device(x, torch.bfloat16), planes)
    torch.cuda.synchronize()
    got = to_np_planes(planes)
    step = 1 << 18
    for s in range(0, n, step):
        part = {k: v[s:s + step] for k, v in got.items()}
        stats = check_key_parity(qo, x[s:s + step].astype(np.float64), part)
        print("prefix", s, stats)
