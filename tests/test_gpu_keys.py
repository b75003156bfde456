"""GPU parity of key quantization (tq_quantize_keys) against the oracle, every mode and
width, both input dtypes, edge cases, and the full 2^24-row quantize workload (sampled)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import require_cuda, to_device, to_np_planes
from parity import check_key_parity

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402

MODES = [("mse", 1), ("mse", 2), ("mse", 3), ("mse", 4), ("prod", 2), ("prod", 3), ("prod", 4),
         ("grouped", 1), ("grouped", 2), ("grouped", 3)]


def edge_rows(qo, n):
    """Rows that stress the decisions: zero, the rotation's own sign vector (its transform
    has exact zeros), a one-hot row, tiny and large scales, constant rows."""
    g = W.rng(77)
    x = W.gaussian(g, (n, 128)) * 3.0
    x[0] = 0.0
    if qo.mode != "grouped":
        x[1] = qo.signs
    x[2] = 0.0
    x[2, 5] = 2.5
    x[3] *= 1e-3
    x[4] *= 300.0
    x[5] = 1.0
    x[6] = -0.5
    return x


@pytest.mark.parametrize("mode,bits", MODES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_keys_parity(mode, bits, dtype):
    dev = require_cuda()
    ch = W.outlier_channels(4)
    outl = ch if mode == "grouped" else None
    seed = 1000 + 17 * bits
    qo = O.build_quantizer(128, bits, mode, seed, outl)
    n = 4096 + 37                                   # many warps plus a ragged tail
    x = W.outlier_rows(W.rng(bits), n, ch)
    x[:16] = edge_rows(qo, 16)
    if dtype == torch.bfloat16:
        x = W.round_bf16(x)
    qg = tq.tq_build_codebook(128, bits, mode, seed, outl)
    planes = qg.alloc_key_planes(n, dev)
    tq.tq_quantize_keys(qg, to_device(x, dtype), planes)
    torch.cuda.synchronize()
    stats = check_key_parity(qo, x.astype(np.float64), to_np_planes(planes))
    print(mode, bits, dtype, stats)


@pytest.mark.parametrize("mode,bits", [("prod", 3), ("grouped", 2), ("mse", 4)])
def test_keys_strided_rows_and_tiny_batches(mode, bits):
    dev = require_cuda()
    ch = W.outlier_channels(4)
    outl = ch if mode == "grouped" else None
    qo = O.build_quantizer(128, bits, mode, 5, outl)
    qg = tq.tq_build_codebook(128, bits, mode, 5, outl)
    full = W.round_bf16(W.gaussian(W.rng(9), (333, 136)) * 2)
    xt = to_device(full, torch.bfloat16)[:, :128]          # ld = 136 elements
    assert xt.stride(0) == 136
    planes = qg.alloc_key_planes(333, dev)
    tq.tq_quantize_keys(qg, xt, planes)
    torch.cuda.synchronize()
    check_key_parity(qo, full[:, :128].astype(np.float64), to_np_planes(planes))
    for n in (1, 2, 15, 17):
        planes = qg.alloc_key_planes(n, dev)
        tq.tq_quantize_keys(qg, to_device(full[:n, :128], torch.bfloat16), planes)
        torch.cuda.synchronize()
        check_key_parity(qo, full[:n, :128].astype(np.float64), to_np_planes(planes))
    # zero rows: a no-op that touches nothing
    planes = qg.alloc_key_planes(1, dev)
    tq.tq_quantize_keys(qg, to_device(full[:0, :128], torch.bfloat16), planes)


def test_keys_score_workload():
    """Keys of the score workload: 4096 fp32 rows (N(0,1) x U[2,20]), 3-bit prod, seed 0."""
    dev = require_cuda()
    keys, _ = W.score_inputs()
    qo = O.build_quantizer(128, 3, "prod", 0)
    qg = tq.tq_build_codebook(128, 3, "prod", 0)
    planes = qg.alloc_key_planes(4096, dev)
    tq.tq_quantize_keys(qg, to_device(keys, torch.float32), planes)
    torch.cuda.synchronize()
    stats = check_key_parity(qo, keys.astype(np.float64), to_np_planes(planes))
    print(stats)


@pytest.mark.parametrize("mode,bits", MODES)
def test_keys_full_quantize_workload_sampled(mode, bits):
    """The 2^24-row quantize workload exactly as the benchmark launches it (4 layers of 2^22
    bf16 rows, quantizer seed = layer); every 4099th row of each layer plus its last 64
    rows are checked against the oracle."""
    dev = require_cuda()
    ch = W.outlier_channels(4)
    outl = ch if mode == "grouped" else None
    rows = 1 << 22
    gen = torch.Generator(device=dev).manual_seed(4)
    total = {"idx_exempt": 0, "coords": 0}
    for layer in range(4):
        x = torch.randn((rows, 128), generator=gen, device=dev, dtype=torch.float32)
        x[:, torch.from_numpy(ch).long().to(dev)] *= 4.0
        x = x.to(torch.bfloat16)
        qg = tq.tq_build_codebook(128, bits, mode, layer, outl)
        planes = qg.alloc_key_planes(rows, dev)
        tq.tq_quantize_keys(qg, x, planes)
        torch.cuda.synchronize()
        sel = torch.cat([torch.arange(0, rows, 4099, device=dev),
                         torch.arange(rows - 64, rows, device=dev)])
        xs = x[sel].float().cpu().numpy().astype(np.float64)
        gp = to_np_planes({k: (v[sel] if v is not None else None) for k, v in planes.items()})
        qo = O.build_quantizer(128, bits, mode, layer, outl)
        st = check_key_parity(qo, xs, gp)
        total["idx_exempt"] += st["idx_exempt"]
        total["coords"] += st["coords"]
        del x, planes
    print(mode, bits, total)
