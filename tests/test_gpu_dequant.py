"""GPU parity of key dequantization (tq_dequantize_keys) against the oracle's
reconstruct_keys, on packed planes produced by the oracle (every mode and width), and the
identity <q, x_hat> = decode estimate on the GPU path."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import require_cuda

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402

MODES = [("mse", 1), ("mse", 2), ("mse", 3), ("mse", 4), ("prod", 2), ("prod", 3), ("prod", 4),
         ("grouped", 1), ("grouped", 2), ("grouped", 3)]


def planes_to_device(p, dev):
    def t(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)
    return dict(idx=t(p["idx"], np.uint8),
                signs=t(p["signs"], np.uint8) if p.get("signs") is not None else None,
                norms=t(p["norms"].astype(np.uint16), np.int16))


@pytest.mark.parametrize("mode,bits", MODES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_dequantize_keys(mode, bits, out_dtype):
    dev = require_cuda()
    ch = W.outlier_channels(4)
    qo = O.build_quantizer(128, bits, mode, 300 + bits, ch if mode == "grouped" else None)
    qg = tq.tq_build_codebook(128, bits, mode, 300 + bits, ch if mode == "grouped" else None)
    n = 1000 + 37
    x = W.outlier_rows(W.rng(bits + 11), n, ch)
    p = O.quantize_keys(qo, x)
    ref = O.reconstruct_keys(qo, p)
    out = torch.full((n, 136), float("nan"), device=dev, dtype=out_dtype)   # ld 136 > d
    tq.tq_dequantize_keys(qg, planes_to_device(p, dev), out)
    torch.cuda.synchronize()
    got = out[:, :128].float().cpu().numpy().astype(np.float64)
    scale = np.linalg.norm(ref, axis=1, keepdims=True) + 1e-30
    if out_dtype == torch.float32:
        assert np.max(np.abs(got - ref) / scale) < 2e-6
    else:
        rb = O.bf16_rn(ref)
        _, e = np.frexp(rb)
        ulp = np.where(rb != 0, np.ldexp(1.0, e - 8), 2.0 ** -133)
        assert np.all(np.abs(got - rb) <= ulp + 2e-6 * scale)


def test_dequantized_keys_reproduce_decode_scores():
    """<q, x_hat> from the GPU dequantizer equals the GPU decode estimate (prod, 3-bit)."""
    dev = require_cuda()
    qz = tq.tq_build_codebook(128, 3, "prod", 9)
    g = torch.Generator(device=dev).manual_seed(3)
    n = 777
    k = (torch.randn((1, 1, n, 128), generator=g, device=dev) * 4).to(torch.bfloat16)
    cache = tq.KVCache(qz, 1, 1, 784, value_bits=0, device=dev)
    tq.tq_append(qz, cache, k, None)
    q = torch.randn((1, 4, 128), generator=g, device=dev)
    scores = torch.empty((1, 4, 784), device=dev)
    ws = tq.alloc_decode_workspace(cache, 4)
    tq.tq_decode_attention(qz, cache, q, None, ws, head_map=[0] * 4, scores=scores)
    planes = dict(idx=cache.k_idx[:n], signs=cache.k_signs[:n], norms=cache.k_norms[:n])
    xh = torch.empty((n, 128), device=dev)
    tq.tq_dequantize_keys(qz, planes, xh)
    torch.cuda.synchronize()
    est = (q[0].double() @ xh.double().T).cpu().numpy()
    sc = scores[0, :, :n].double().cpu().numpy()
    floor = np.linalg.norm(q[0].cpu().numpy(), axis=1)[:, None] * np.linalg.norm(xh.cpu().numpy(), axis=1)[None, :] / 128 ** 0.5
    assert np.max(np.abs(est - sc) / np.maximum(np.abs(sc), floor)) < 1e-3
