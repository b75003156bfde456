"""GPU parity of fused decode attention (tq_decode_attention) against the oracle.

The packed caches are produced by the oracle's quantizer (never by the CUDA path) and
uploaded, so these tests isolate the decode kernel; key-quantize parity is tested apart."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import download_pair, oracle_cache, require_cuda, to_device, to_np_planes, upload_cache
from parity import check_attention, check_key_parity, check_scores

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402


def run_decode(qg, cache, Q, q_dtype, out_dtype, head_map=None, sm_scale=0.0, scores_ld=0):
    dev = cache.len_dev.device
    B, Hq, d = Q.shape
    qt = to_device(Q, q_dtype)
    out = torch.full((B, Hq, d), float("nan"), device=dev, dtype=out_dtype) if cache.value_bits else None
    scores = torch.full((B, Hq, scores_ld), float("nan"), device=dev) if scores_ld else None
    ws = tq.alloc_decode_workspace(cache, Hq)
    tq.tq_decode_attention(qg, cache, qt, out, ws, head_map=head_map, sm_scale=sm_scale,
                           scores=scores)
    torch.cuda.synchronize()
    return (out.float().cpu().numpy() if out is not None else None,
            scores.cpu().numpy() if scores is not None else None, ws)


def small_case(seed, B, Hq, Hkv, lengths, cap, bits, vbits, mode="prod"):
    g = W.rng(seed)
    N = max(lengths)
    K = W.round_bf16(W.scaled_gaussian_rows(g, B * Hkv * N).reshape(B, Hkv, N, 128))
    V = W.round_bf16(W.gaussian(g, (B, Hkv, N, 128)))
    Q = W.round_bf16(W.gaussian(g, (B, Hq, 128)))
    qo = O.build_quantizer(128, bits, mode, seed)
    qg = tq.tq_build_codebook(128, bits, mode, seed)
    oc = oracle_cache(qo, K, V if vbits else None, vbits, lengths)
    cache = tq.KVCache(qg, B, Hkv, cap, value_bits=vbits, device="cuda:0")
    upload_cache(cache, oc)
    return qo, qg, oc, cache, Q


@pytest.mark.parametrize("bits,vbits", [(2, 2), (3, 2), (3, 4), (4, 4), (4, 2), (2, 4)])
@pytest.mark.parametrize("q_dtype,out_dtype", [(torch.bfloat16, torch.float32),
                                               (torch.float32, torch.bfloat16)])
def test_decode_small_ragged(bits, vbits, q_dtype, out_dtype):
    """Several context splits, a ragged tail and sequences of different lengths."""
    require_cuda()
    qo, qg, oc, cache, Q = small_case(40 + bits + vbits, 2, 6, 2, [1000, 777], 1024, bits, vbits)
    if q_dtype == torch.float32:
        Q = W.gaussian(W.rng(5), Q.shape)
    out, _, _ = run_decode(qg, cache, Q, q_dtype, out_dtype)
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=vbits)
    err = check_attention(out, ref, out_dtype == torch.bfloat16)
    print(bits, vbits, err)


@pytest.mark.parametrize("bits,vbits", [(1, 2), (2, 2), (3, 4), (4, 4), (4, 2)])
def test_decode_mse_keys(bits, vbits):
    """mse caches: s = n16 <Pi q, c[idx]> (no QJL term), 1..4-bit indices."""
    require_cuda()
    qo, qg, oc, cache, Q = small_case(60 + bits, 2, 7, 2, [1100, 613], 1152, bits, vbits, "mse")
    hm = [0, 0, 0, 0, 1, 1, 1]   # groups of 4 and 3 query heads
    out, _, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32, head_map=hm)
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), head_map=hm, value_bits=vbits)
    err = check_attention(out, ref, False)
    print("mse", bits, vbits, err)


@pytest.mark.parametrize("bits", [1, 3, 4])
def test_decode_mse_scores(bits):
    require_cuda()
    qo, qg, oc, cache, Q = small_case(70 + bits, 1, 8, 1, [777], 784, bits, 0, "mse")
    _, sc, _ = run_decode(qg, cache, Q, torch.float32, torch.float32, scores_ld=784)
    _, ref = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=0, want_scores=True)
    for h in range(8):
        check_scores(sc[0, h, :777], ref[0][h], np.linalg.norm(Q[0, h]),
                     O.fp16_from_bits(oc["k_norms"][0, 0, :777, 0]))


def grouped_case(seed, B, Hq, Hkv, lengths, cap, bits, vbits):
    """Keys with 32 fixed high-variance channels (4x std), as in the key-quantize workload."""
    g = W.rng(seed)
    N = max(lengths)
    ch = W.outlier_channels(seed)
    K = W.round_bf16(W.outlier_rows(g, B * Hkv * N, ch).reshape(B, Hkv, N, 128))
    V = W.round_bf16(W.gaussian(g, (B, Hkv, N, 128)))
    Q = W.round_bf16(W.gaussian(g, (B, Hq, 128)))
    qo = O.build_quantizer(128, bits, "grouped", seed, ch)
    qg = tq.tq_build_codebook(128, bits, "grouped", seed, ch)
    oc = oracle_cache(qo, K, V if vbits else None, vbits, lengths)
    cache = tq.KVCache(qg, B, Hkv, cap, value_bits=vbits, device="cuda:0")
    upload_cache(cache, oc)
    return qo, qg, oc, cache, Q


@pytest.mark.parametrize("bits,vbits", [(1, 2), (2, 2), (2, 4), (3, 4), (3, 2)])
def test_decode_grouped_keys(bits, vbits):
    """grouped caches: s = n_o <Pi_o q_o, c_o[idx_o]> + n_n <Pi_n q_n, c_n[idx_n]> (outlier
    group at b + 1 bits, normal group at b bits; 20 / 40 / 64 index bytes per key)."""
    require_cuda()
    qo, qg, oc, cache, Q = grouped_case(80 + bits, 2, 7, 2, [1100, 613], 1152, bits, vbits)
    hm = [0, 0, 0, 0, 1, 1, 1]
    out, _, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32, head_map=hm)
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), head_map=hm, value_bits=vbits)
    err = check_attention(out, ref, False)
    print("grouped", bits, vbits, err)


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_decode_grouped_scores(bits):
    require_cuda()
    qo, qg, oc, cache, Q = grouped_case(90 + bits, 1, 6, 1, [745], 752, bits, 0)
    _, sc, _ = run_decode(qg, cache, Q, torch.float32, torch.float32, scores_ld=752)
    _, ref = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=0, want_scores=True)
    nrm = O.fp16_from_bits(oc["k_norms"][0, 0, :745])
    for h in range(6):
        check_scores(sc[0, h, :745], ref[0][h], np.linalg.norm(Q[0, h]),
                     np.sqrt(nrm[:, 0] ** 2 + nrm[:, 1] ** 2))


def test_decode_head_map_scale_and_scores():
    require_cuda()
    qo, qg, oc, cache, Q = small_case(7, 1, 5, 3, [600], 608, 3, 2)
    hm = np.array([2, 0, 2, 1, 2])
    out, sc, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32, head_map=hm,
                            sm_scale=0.05, scores_ld=608)
    ref, rs = O.decode_attention(qo, oc, Q.astype(np.float64), head_map=hm, sm_scale=0.05,
                                 value_bits=2, want_scores=True)
    check_attention(out, ref, False)
    n16 = O.fp16_from_bits(oc["k_norms"][0, :, :600, 0])
    for h in range(5):
        check_scores(sc[0, h, :600], rs[0][h], np.linalg.norm(Q[0, h]), n16[hm[h]])
    assert np.all(np.isnan(sc[0, :, 600:]))      # nothing written beyond len


def test_decode_empty_and_single_token_sequences():
    require_cuda()
    qo, qg, oc, cache, Q = small_case(8, 3, 4, 2, [0, 1, 300], 304, 3, 2)
    out, _, ws = run_decode(qg, cache, Q, torch.bfloat16, torch.float32)
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=2)
    assert np.all(out[0] == 0.0)                 # len 0 -> zeros
    check_attention(out, ref, False)
    vh = O.dequantize_values(oc["v_q"][1, 0, :1], oc["v_params"][1, 0, :1], 2, 128)[0]
    assert np.allclose(out[1, 0], vh, atol=1e-6)  # one key -> its value
    # the workspace is left reusable: a second call gives the same result
    out2, _, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32)
    assert np.array_equal(out, out2)


def test_score_workload():
    """Score workload: 4096 fp32 keys (3-bit prod, seed 0), 8 fp32 queries as 8 query heads
    on one KV head, key-only cache; outputs the 4096 x 8 estimate matrix. Also checks the
    keys the GPU quantized against the oracle (end to end)."""
    dev = require_cuda()
    keys, queries = W.score_inputs()
    qo = O.build_quantizer(128, 3, "prod", 0)
    qg = tq.tq_build_codebook(128, 3, "prod", 0)
    oc = oracle_cache(qo, keys[None, None], None, 0, [4096])
    cache = tq.KVCache(qg, 1, 1, 4096, value_bits=0, device=dev)
    upload_cache(cache, oc)
    _, sc, _ = run_decode(qg, cache, queries[None], torch.float32, None, scores_ld=4096)
    _, rs = O.decode_attention(qo, oc, queries[None].astype(np.float64), want_scores=True)
    n16 = O.fp16_from_bits(oc["k_norms"][0, 0, :, 0])
    worst = max(check_scores(sc[0, h], rs[0][h], np.linalg.norm(queries[h]), n16)
                for h in range(8))
    print("score rel err", worst)
    # end to end: GPU-quantized keys scored on the GPU
    cache2 = tq.KVCache(qg, 1, 1, 4096, value_bits=0, device=dev)
    tq.tq_append(qg, cache2, to_device(keys[None, None], torch.float32))
    gp = to_np_planes(cache2.key_planes())
    check_key_parity(qo, keys.astype(np.float64), gp)
    _, sc2, _ = run_decode(qg, cache2, queries[None], torch.float32, None, scores_ld=4096)
    same = np.all(gp["idx"] == oc["k_idx"][0, 0], axis=1) & np.all(gp["signs"] == oc["k_signs"][0, 0], axis=1)
    for h in range(8):
        check_scores(sc2[0, h][same], rs[0][h][same], np.linalg.norm(queries[h]), n16[same])


def _full_decode(cfg_id, sample_pairs, out_dtype):
    require_cuda()
    cfg = W.WORKLOADS[cfg_id]
    B, Hq, Hkv, N = cfg["batch"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["ctx"]
    K, V, Q, _ = W.decode_inputs(cfg_id, B, Hq, Hkv, N, planted=cfg.get("planted", 0))
    qo = O.build_quantizer(128, cfg["key_bits"], "prod", cfg["qseed"])
    qg = tq.tq_build_codebook(128, cfg["key_bits"], "prod", cfg["qseed"])
    G = Hq // Hkv
    vb = cfg["value_bits"]
    # the oracle quantizes only the (b, kv) pairs that are checked; the rest of the cache
    # holds the same data quantized on the GPU, which only feeds outputs not compared here
    cap = N + 256
    cache = tq.KVCache(qg, B, Hkv, cap, value_bits=vb, device="cuda:0")
    tq.tq_append(qg, cache, to_device(K, torch.bfloat16), to_device(V, torch.bfloat16))
    for b, kv in sample_pairs:
        oc = oracle_cache(qo, K[b:b + 1, kv:kv + 1], V[b:b + 1, kv:kv + 1], vb, [N])
        rows = cache.rows(b, kv)
        for name, key in (("k_idx", "k_idx"), ("k_signs", "k_signs"), ("k_norms", "k_norms"),
                          ("v_q", "v_q"), ("v_params", "v_params")):
            src = oc[key][0, 0]
            if src.dtype == np.uint16:
                src = src.view(np.int16)
            getattr(cache, name)[rows][:N].copy_(torch.from_numpy(np.ascontiguousarray(src)).reshape(
                getattr(cache, name)[rows][:N].shape))
        pairs_oc = oc
        pairs_oc["len"] = np.array([N])
        heads = list(range(kv * G, (kv + 1) * G))
        out, _, _ = run_decode(qg, cache, Q, torch.bfloat16, out_dtype)
        ref, _ = O.decode_attention(qo, pairs_oc, Q[b:b + 1, heads].astype(np.float64),
                                    head_map=np.zeros(G, dtype=int), value_bits=vb)
        err = check_attention(out[b, heads], ref[0], out_dtype == torch.bfloat16)
        print(cfg["name"], b, kv, err)
    return out


def test_decode_full_config_decode_s():
    """Batch 1, 12/2 GQA, context 32768, 3-bit prod keys, 2-bit values: every head."""
    _full_decode(2, [(0, 0), (0, 1)], torch.float32)


def test_decode_full_config_decode_l():
    """Batch 8, 28/4 GQA, context 32768 with planted keys; sampled (sequence, KV head) pairs
    quantized by the oracle, all 7 heads of each against the oracle's decode."""
    out = _full_decode(3, [(0, 0), (7, 3), (3, 1)], torch.bfloat16)
    assert np.all(np.isfinite(out))


def test_decode_l_every_pair_and_planted_scores():
    """decode-l at full size on the GPU-quantized cache (batch 8, 28/4 GQA, 32768 tokens with
    16 planted keys 0.9 q + 0.1 noise per pair): every (sequence, KV head) pair's 7 heads
    against the oracle's decode of the same packed rows (bf16 output), and the scores of the
    planted keys for the query head they were planted for against the oracle's scores. With
    row scales up to 20 the planted keys do not dominate attention; their softmax mass is
    printed."""
    require_cuda()
    cfg = W.WORKLOADS[3]
    B, Hq, Hkv, N = cfg["batch"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["ctx"]
    K, V, Q, pos = W.decode_inputs(3, B, Hq, Hkv, N, planted=cfg["planted"])
    qo = O.build_quantizer(128, cfg["key_bits"], "prod", cfg["qseed"])
    qg = tq.tq_build_codebook(128, cfg["key_bits"], "prod", cfg["qseed"])
    G, vb = Hq // Hkv, cfg["value_bits"]
    cache = tq.KVCache(qg, B, Hkv, N, value_bits=vb, device="cuda:0")
    tq.tq_append(qg, cache, to_device(K, torch.bfloat16), to_device(V, torch.bfloat16))
    out, sc, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.bfloat16, scores_ld=N)
    worst = 0.0
    for b in range(B):
        for kv in range(Hkv):
            oc = download_pair(cache, b, kv, N)
            heads = list(range(kv * G, (kv + 1) * G))
            ref, rs = O.decode_attention(qo, oc, Q[b:b + 1, heads].astype(np.float64),
                                         head_map=np.zeros(G, dtype=int), value_bits=vb,
                                         want_scores=True)
            worst = max(worst, check_attention(out[b, heads], ref[0], True))
            h = kv * G
            p = pos[b, kv]
            n16 = O.fp16_from_bits(oc["k_norms"][0, 0, :, 0])
            check_scores(sc[b, h][p], rs[0][0][p], np.linalg.norm(Q[b, h]), n16[p])
            s = rs[0][0] / np.sqrt(128.0)
            w = np.exp(s - s.max())
            if b == 0:
                print("pair", b, kv, "planted softmax mass", float(w[p].sum() / w.sum()))
    print("decode-l every pair: worst", worst)


def test_decode_stream_steps():
    """Streaming decode: context 131072, 64/8 GQA, 4-bit prod keys, 4-bit values; each step
    appends one token per KV head on the GPU, then decodes. Appended rows are checked
    against the oracle, the decode after each step against the oracle's cache (one KV head),
    and after the last step every KV head against the oracle's decode of the GPU's rows."""
    require_cuda()
    cfg = W.WORKLOADS[5]
    B, Hq, Hkv, N = 1, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["ctx"]
    steps = 3
    K, V, Q, _ = W.decode_inputs(5, B, Hq, Hkv, N, extra_tokens=steps)
    qo = O.build_quantizer(128, 4, "prod", 0)
    qg = tq.tq_build_codebook(128, 4, "prod", 0)
    cap = N + 256
    cache = tq.KVCache(qg, B, Hkv, cap, value_bits=4, device="cuda:0")
    tq.tq_append(qg, cache, to_device(K[:, :, :N], torch.bfloat16),
                 to_device(V[:, :, :N], torch.bfloat16))
    kv = 5
    G = Hq // Hkv
    heads = list(range(kv * G, (kv + 1) * G))
    oc = oracle_cache(qo, K[:, kv:kv + 1], V[:, kv:kv + 1], 4, [N + steps])
    rows = cache.rows(0, kv)
    for name in ("k_idx", "k_signs", "k_norms", "v_q", "v_params"):
        src = oc[name][0, 0][:N]
        if src.dtype == np.uint16:
            src = src.view(np.int16)
        dst = getattr(cache, name)[rows][:N]
        dst.copy_(torch.from_numpy(np.ascontiguousarray(src)).reshape(dst.shape))
    for s in range(steps):
        tq.tq_append(qg, cache, to_device(K[:, :, N + s:N + s + 1], torch.bfloat16),
                     to_device(V[:, :, N + s:N + s + 1], torch.bfloat16))
        r = slice(rows.start + N + s, rows.start + N + s + 1)
        gp = to_np_planes({"idx": cache.k_idx[r], "signs": cache.k_signs[r], "norms": cache.k_norms[r]})
        check_key_parity(qo, K[0, kv, N + s:N + s + 1].astype(np.float64), gp)
        out, _, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32)
        step_oc = dict(oc, len=np.array([N + s + 1]))
        ref, _ = O.decode_attention(qo, step_oc, Q[:, heads].astype(np.float64),
                                    head_map=np.zeros(G, dtype=int), value_bits=4)
        check_attention(out[0, heads], ref[0], False)
    # after the last step, every KV head's 8 query heads against the oracle's decode of the
    # GPU's own packed rows (the appended token included)
    n = N + steps
    for kvh in range(Hkv):
        oc_h = download_pair(cache, 0, kvh, n)
        hs = list(range(kvh * G, (kvh + 1) * G))
        ref, _ = O.decode_attention(qo, oc_h, Q[:, hs].astype(np.float64),
                                    head_map=np.zeros(G, dtype=int), value_bits=4)
        check_attention(out[0, hs], ref[0], False)


def _slice_oracle_cache(oc, start, stop):
    out = {k: v[:, :, start:stop] for k, v in oc.items() if k != "len" and v is not None}
    out["len"] = np.clip(np.asarray(oc["len"]) - start, 0, stop - start)
    return out


@pytest.mark.parametrize("mode,bits,vbits", [("prod", 3, 2), ("mse", 4, 4), ("grouped", 2, 2)])
def test_decode_context_split_partials_and_merge(mode, bits, vbits):
    """Context-parallel decode on one GPU: each sequence's context is cut into three ragged
    slices held by three caches (the shorter sequence leaves the last slice empty).
    tq_decode_attention_partial on each slice and tq_merge_partials over the three record
    sets match the oracle's decode over the whole context; each slice's normalised record
    matches the oracle's attention over that slice; an empty slice gives (-inf, 0, 0); and
    one slice merged alone reproduces tq_decode_attention bit for bit."""
    dev = require_cuda()
    lengths, cap = [1000, 700], 1024
    if mode == "grouped":
        qo, qg, oc, cache, Q = grouped_case(120 + bits, 2, 6, 2, lengths, cap, bits, vbits)
    else:
        qo, qg, oc, cache, Q = small_case(110 + bits, 2, 6, 2, lengths, cap, bits, vbits, mode)
    B, Hq = Q.shape[:2]
    qt = to_device(Q, torch.bfloat16)
    cuts = (0, 333, 800, 1000)
    parts = torch.empty((len(cuts) - 1, B, Hq, tq.TQ_PART_FLOATS), device=dev)
    for i, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        sl = _slice_oracle_cache(oc, a, b)
        c = tq.KVCache(qg, B, 2, ((b - a) + 15) // 16 * 16, value_bits=vbits, device=dev)
        upload_cache(c, sl)
        ws = tq.alloc_decode_workspace(c, Hq)
        tq.tq_decode_attention_partial(qg, c, qt, parts[i], ws)
        torch.cuda.synchronize()
        rec = parts[i].cpu().numpy().astype(np.float64)
        m_ref, l_ref, o_ref = O.decode_partial(qo, sl, Q.astype(np.float64), value_bits=vbits)
        for bb in range(B):
            if sl["len"][bb] == 0:
                assert np.all(rec[bb, :, 0] == -np.inf) and np.all(rec[bb, :, 1:] == 0)
                continue
            assert np.allclose(rec[bb, :, 0], m_ref[bb], rtol=1e-3, atol=1e-3)
            check_attention(rec[bb, :, 4:] / rec[bb, :, 1:2], o_ref[bb] / l_ref[bb][:, None], False)
    out = torch.empty((B, Hq, 128), device=dev)
    tq.tq_merge_partials(parts, out)
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=vbits)
    check_attention(out.cpu().numpy(), ref, False)
    # a single slice: the merge of its one record set is the decode's own output
    whole = torch.empty((1, B, Hq, tq.TQ_PART_FLOATS), device=dev)
    ws = tq.alloc_decode_workspace(cache, Hq)
    tq.tq_decode_attention_partial(qg, cache, qt, whole[0], ws)
    tq.tq_merge_partials(whole, out)
    direct, _, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32)
    assert np.array_equal(out.cpu().numpy(), direct)


@pytest.fixture(params=["two_sets", "one_set"])
def decode_shape(request):
    """Force the two-set (up to 8 heads per block) or the one-set decode shape."""
    pol = tq.TQ_DECODE_TWO_SETS if request.param == "two_sets" else tq.TQ_DECODE_ONE_SET
    prev = tq.tq_set_decode_policy(pol)
    yield request.param
    tq.tq_set_decode_policy(prev)


@pytest.fixture
def two_sets():
    prev = tq.tq_set_decode_policy(tq.TQ_DECODE_TWO_SETS)
    yield
    tq.tq_set_decode_policy(prev)


@pytest.mark.parametrize("mode,bits,vbits,hq,hm", [
    ("prod", 3, 2, 12, None),                                   # 6 heads per KV head
    ("prod", 3, 2, 14, None),                                   # 7
    ("prod", 4, 4, 16, None),                                   # 8, 3-bit indices in nibbles
    ("prod", 2, 4, 10, None),                                   # 5
    ("mse", 2, 2, 12, None),
    ("mse", 3, 4, 16, None),
    ("prod", 3, 2, 11, [0] * 8 + [1] * 3),                      # 8 and 3: one CTA with nh < NH
])
def test_decode_eight_heads_per_cta(mode, bits, vbits, hq, hm, decode_shape):
    """More than 4 query heads per KV head, in both block shapes: one block serving up to 8
    of them with two table sets (8 warps, byte tables for both lookup segments, P.V over
    every head of the block), and blocks of at most 4 (one set, 16 warps)."""
    require_cuda()
    qo, qg, oc, cache, Q = small_case(150 + bits + hq, 2, hq, 2, [1000, 613], 1024, bits, vbits, mode)
    out, sc, _ = run_decode(qg, cache, Q, torch.bfloat16, torch.float32, head_map=hm,
                            scores_ld=1024)
    ref, rs = O.decode_attention(qo, oc, Q.astype(np.float64), head_map=hm, value_bits=vbits,
                                 want_scores=True)
    err = check_attention(out, ref, False)
    hmap = hm if hm is not None else O.default_head_map(hq, 2)
    for b, L in enumerate([1000, 613]):
        n16 = O.fp16_from_bits(oc["k_norms"][b, :, :L, 0])
        for h in range(hq):
            check_scores(sc[b, h, :L], rs[b][h], np.linalg.norm(Q[b, h]), n16[hmap[h]])
    print(mode, bits, vbits, hq, decode_shape, err)


@pytest.mark.parametrize("bits", [2, 3])
def test_decode_eight_heads_scores_only(bits, two_sets):
    """Key-only cache (scores, no values) with 8 query heads per KV head."""
    require_cuda()
    qo, qg, oc, cache, Q = small_case(170 + bits, 1, 8, 1, [777], 784, bits, 0)
    _, sc, _ = run_decode(qg, cache, Q, torch.float32, torch.float32, scores_ld=784)
    _, ref = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=0, want_scores=True)
    n16 = O.fp16_from_bits(oc["k_norms"][0, 0, :777, 0])
    for h in range(8):
        check_scores(sc[0, h, :777], ref[0][h], np.linalg.norm(Q[0, h]), n16)


def test_decode_eight_heads_partials_and_merge(two_sets):
    """The context-split partial records with two table sets per CTA."""
    dev = require_cuda()
    qo, qg, oc, cache, Q = small_case(190, 2, 14, 2, [900, 640], 912, 3, 2)
    B, Hq = Q.shape[:2]
    qt = to_device(Q, torch.bfloat16)
    cuts = (0, 300, 900)
    parts = torch.empty((2, B, Hq, tq.TQ_PART_FLOATS), device=dev)
    for i, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        sl = _slice_oracle_cache(oc, a, b)
        c = tq.KVCache(qg, B, 2, ((b - a) + 15) // 16 * 16, value_bits=2, device=dev)
        upload_cache(c, sl)
        tq.tq_decode_attention_partial(qg, c, qt, parts[i], tq.alloc_decode_workspace(c, Hq))
    out = torch.empty((B, Hq, 128), device=dev)
    tq.tq_merge_partials(parts, out)
    ref, _ = O.decode_attention(qo, oc, Q.astype(np.float64), value_bits=2)
    check_attention(out.cpu().numpy(), ref, False)
