"""GPU parity of value quantization (bit-exact: the code decision is fp32 IEEE on both
sides) and of tq_append (writes at len[b], advances len, refuses overflow)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import require_cuda, to_device, to_np_planes
from parity import check_key_parity

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_values_bit_exact(bits, dtype):
    dev = require_cuda()
    g = W.rng(21 + bits)
    n = 5000 + 3
    v = W.gaussian(g, (n, 128)) * g.uniform(0.01, 8.0, (n, 1)).astype(np.float32)
    v[0] = 0.0
    v[1] = 1.5                           # constant groups: scale 0, codes 0
    v[2, :32] = np.linspace(-1, 1, 32)
    v[3] = np.float32(1e-4) * W.gaussian(g, (128,))
    if dtype == torch.bfloat16:
        v = W.round_bf16(v)
    planes = tq.alloc_value_planes(n, bits, device=dev)
    tq.tq_quantize_values(to_device(v, dtype), planes, bits)
    torch.cuda.synchronize()
    got = to_np_planes(planes)
    ref = O.quantize_values(v.astype(np.float64), bits)
    assert np.array_equal(got["q"], ref["q"])
    assert np.array_equal(got["params"].reshape(n, 4, 2), ref["params"])


def test_values_reject_bad_arguments():
    dev = require_cuda()
    v = torch.zeros((4, 128), device=dev)
    planes = tq.alloc_value_planes(4, 2, device=dev)
    for bits, group in ((3, 32), (2, 16)):
        with pytest.raises(tq.TQError) as e:
            tq.tq_quantize_values(v, planes, bits, group)
        assert e.value.status == tq.TQ_EUNSUPPORTED
    with pytest.raises(tq.TQError):
        tq.tq_quantize_values(v.to(torch.float16), planes, 2)


@pytest.mark.parametrize("mode,bits,vbits", [("prod", 3, 2), ("prod", 4, 4), ("mse", 2, 2),
                                             ("grouped", 2, 4)])
def test_append_writes_at_len_and_advances(mode, bits, vbits):
    dev = require_cuda()
    ch = W.outlier_channels(4)
    outl = ch if mode == "grouped" else None
    qg = tq.tq_build_codebook(128, bits, mode, 3, outl)
    qo = O.build_quantizer(128, bits, mode, 3, outl)
    B, H, cap = 3, 2, 64
    cache = tq.KVCache(qg, B, H, cap, value_bits=vbits, device=dev)
    cache.set_lengths([0, 5, 62])
    g = W.rng(31)
    for n_tok in (1, 3):
        before = cache.lengths
        k = W.round_bf16(W.scaled_gaussian_rows(g, B * H * n_tok).reshape(B, H, n_tok, 128))
        v = W.round_bf16(W.gaussian(g, (B, H, n_tok, 128)))
        if max(before) + n_tok > cap:
            with pytest.raises(tq.TQError) as e:
                tq.tq_append(qg, cache, to_device(k, torch.bfloat16), to_device(v, torch.bfloat16))
            assert e.value.status == tq.TQ_ECAPACITY
            assert cache.lengths == before
            cache.set_lengths([before[0], before[1], 0])
            before = cache.lengths
        tq.tq_append(qg, cache, to_device(k, torch.bfloat16), to_device(v, torch.bfloat16))
        torch.cuda.synchronize()
        assert cache.lengths == [n + n_tok for n in before]
        assert cache.len_dev.cpu().tolist() == cache.lengths
        for b in range(B):
            for h in range(H):
                rows = slice((b * H + h) * cap + before[b], (b * H + h) * cap + before[b] + n_tok)
                gp = to_np_planes({"idx": cache.k_idx[rows], "signs": None if cache.k_signs is None
                                   else cache.k_signs[rows], "norms": cache.k_norms[rows]})
                check_key_parity(qo, k[b, h].astype(np.float64), gp)
                ref = O.quantize_values(v[b, h].astype(np.float64), vbits)
                assert np.array_equal(cache.v_q[rows].cpu().numpy(), ref["q"])
                assert np.array_equal(cache.v_params[rows].cpu().numpy().view(np.uint16), ref["params"])


def test_append_key_only_cache_and_errors():
    dev = require_cuda()
    qg = tq.tq_build_codebook(128, 3, "prod", 0)
    cache = tq.KVCache(qg, 1, 1, 16, value_bits=0, device=dev)
    k = torch.zeros((1, 1, 16, 128), device=dev, dtype=torch.bfloat16)
    tq.tq_append(qg, cache, k)
    assert cache.lengths == [16]
    with pytest.raises(tq.TQError) as e:
        tq.tq_append(qg, cache, k[:, :, :1].contiguous())
    assert e.value.status == tq.TQ_ECAPACITY
    with pytest.raises(tq.TQError) as e:   # values given to a key-only cache
        tq.tq_append(qg, cache, k[:, :, :1].contiguous(), k[:, :, :1].contiguous())
    assert e.value.status == tq.TQ_EINVAL
    with pytest.raises(ValueError):
        tq.KVCache(qg, 1, 1, 20, device=dev)


@pytest.mark.parametrize("mode,bits,vbits,dtype", [("prod", 3, 2, torch.bfloat16),
                                                   ("prod", 2, 4, torch.float32),
                                                   ("mse", 4, 2, torch.bfloat16),
                                                   ("grouped", 3, 2, torch.bfloat16)])
def test_append_multi_token_chunks(mode, bits, vbits, dtype):
    """Prefill in ragged chunks (store.py append_chunk): chunk sizes on both sides of the
    64-token switch between the fused append kernel and the separate quantize kernels, ragged
    starting lengths, bf16 and fp32 inputs. Every cached row matches the oracle's quantization
    of the whole prefix, so chunk boundaries leave no trace."""
    dev = require_cuda()
    ch = W.outlier_channels(6)
    outl = ch if mode == "grouped" else None
    qg = tq.tq_build_codebook(128, bits, mode, 8, outl)
    qo = O.build_quantizer(128, bits, mode, 8, outl)
    B, H, cap = 2, 3, 544
    start = [0, 17]
    chunks = [1, 63, 64, 65, 130, 200]
    total = sum(chunks)
    cache = tq.KVCache(qg, B, H, cap, value_bits=vbits, device=dev)
    cache.set_lengths(start)
    g = W.rng(77)
    k = W.scaled_gaussian_rows(g, B * H * total).reshape(B, H, total, 128)
    if dtype == torch.bfloat16:
        k = W.round_bf16(k)
    v = W.gaussian(g, (B, H, total, 128))
    v = W.round_bf16(v) if dtype == torch.bfloat16 else v.astype(np.float32).astype(np.float64)
    k = k if dtype == torch.bfloat16 else k.astype(np.float32).astype(np.float64)
    t0 = 0
    for n_tok in chunks:
        tq.tq_append(qg, cache, to_device(k[:, :, t0:t0 + n_tok], dtype).contiguous(),
                     to_device(v[:, :, t0:t0 + n_tok], dtype).contiguous())
        t0 += n_tok
    torch.cuda.synchronize()
    assert cache.lengths == [s + total for s in start]
    assert cache.len_dev.cpu().tolist() == cache.lengths
    for b in range(B):
        for h in range(H):
            base = (b * H + h) * cap + start[b]
            rows = slice(base, base + total)
            gp = to_np_planes({"idx": cache.k_idx[rows], "signs": None if cache.k_signs is None
                               else cache.k_signs[rows], "norms": cache.k_norms[rows]})
            check_key_parity(qo, k[b, h].astype(np.float64), gp)
            ref = O.quantize_values(v[b, h].astype(np.float64), vbits)
            assert np.array_equal(cache.v_q[rows].cpu().numpy(), ref["q"])
            assert np.array_equal(cache.v_params[rows].cpu().numpy().view(np.uint16), ref["params"])


def test_append_decode_equals_append_then_decode():
    """tq_append_decode (one call, both kernels launched back to back) leaves the same cache
    and gives the same outputs and scores, bit for bit, as tq_append followed by
    tq_decode_attention; a decode argument error launches nothing (lengths unchanged)."""
    dev = require_cuda()
    qg = tq.tq_build_codebook(128, 3, "prod", 11)
    B, H, Hq, cap = 2, 2, 6, 272
    g = W.rng(12)
    pre_k = to_device(W.round_bf16(W.scaled_gaussian_rows(g, B * H * 200).reshape(B, H, 200, 128)), torch.bfloat16)
    pre_v = to_device(W.round_bf16(W.gaussian(g, (B, H, 200, 128))), torch.bfloat16)
    k_new = to_device(W.round_bf16(W.scaled_gaussian_rows(g, B * H).reshape(B, H, 1, 128)), torch.bfloat16)
    v_new = to_device(W.round_bf16(W.gaussian(g, (B, H, 1, 128))), torch.bfloat16)
    q = to_device(W.round_bf16(W.gaussian(g, (B, Hq, 128))), torch.bfloat16)
    res = []
    for fused in (False, True):
        cache = tq.KVCache(qg, B, H, cap, value_bits=2, device=dev)
        tq.tq_append(qg, cache, pre_k, pre_v)
        ws = tq.alloc_decode_workspace(cache, Hq)
        out = torch.empty((B, Hq, 128), device=dev)
        sc = torch.full((B, Hq, 256), float("nan"), device=dev)
        if fused:
            tq.tq_append_decode(qg, cache, k_new, v_new, q, out, ws, scores=sc)
        else:
            tq.tq_append(qg, cache, k_new, v_new)
            tq.tq_decode_attention(qg, cache, q, out, ws, scores=sc)
        torch.cuda.synchronize()
        # the written rows only (rows past each length are uninitialised memory)
        written = lambda t: t.reshape(B * H, cap, -1)[:, :201].cpu()
        res.append((out.cpu(), sc.cpu(), cache.lengths, written(cache.k_idx), written(cache.v_q)))
        if fused:
            with pytest.raises(tq.TQError) as e:   # scores_ld below the post-append length
                tq.tq_append_decode(qg, cache, k_new, v_new, q, out, ws, scores=sc[:, :, :201])
            assert e.value.status == tq.TQ_EINVAL
            assert cache.lengths == [201, 201]
    (o0, s0, l0, k0, v0), (o1, s1, l1, k1, v1) = res
    assert l0 == l1 == [201, 201]
    assert torch.equal(o0, o1) and torch.equal(k0, k1) and torch.equal(v0, v1)
    assert torch.equal(torch.nan_to_num(s0, nan=-7.0), torch.nan_to_num(s1, nan=-7.0))
