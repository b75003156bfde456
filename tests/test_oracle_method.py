"""Pins of the oracle's quantizers, estimator, value quantizer and decode attention against
what the pages and the mathematics fix (validate_paper.py's theorem checks, closed forms,
brute force on small inputs)."""
import math

import numpy as np
import pytest
from scipy import stats

import oracle as O
from conftest import read_golden

D = 128


def unit_rows(seed, n, d=D):
    x = np.random.default_rng(seed).standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


# ---------------------------------------------------------------- Theorem 1 (MSE)
def test_theorem1_mse_within_table1_bound():
    """validate_paper.py test_mse_distortion_bounds (Theorem 1): d=128, seed 42, b=1..4,
    MSE <= 1.15 x {0.360, 0.117, 0.030, 0.009}. Reading: the MSE is measured per coordinate
    of the sqrt(d)-scaled vector, ||x - x_hat||^2 / ||x||^2 (the page's unit-norm mean over
    coordinates is d times smaller and could never fail)."""
    bounds = {int(b): float(v) for b, v in read_golden("table1_mse.txt")}
    x = unit_rows(42, 40000)
    for bits, bound in bounds.items():
        q = O.build_quantizer(D, bits, "mse", 42)
        xh = O.reconstruct_keys(q, O.quantize_keys(q, x))
        mse = np.mean(np.sum((x - xh) ** 2, axis=1))
        assert mse <= 1.15 * bound, (bits, mse)
        # and close to the Gaussian Lloyd-Max distortion (sphere coordinates are slightly
        # lighter-tailed than the Gaussian, so a little below it)
        c, t = O.lloyd_max_gaussian(bits)
        dist = O.gaussian_distortion(c, t)
        assert 0.95 * dist < mse < 1.01 * dist, (bits, mse, dist)


def test_mse_indices_are_nearest_centroid():
    """Brute force: every coordinate's code is the nearest centroid of u = Pi x / ||x||."""
    q = O.build_quantizer(D, 3, "mse", 9)
    x = np.random.default_rng(2).standard_normal((300, D)) * 3.0
    p = O.quantize_keys(q, x)
    u = (x @ q.Pi.T) / np.linalg.norm(x, axis=1, keepdims=True)
    nearest = np.argmin(np.abs(u[:, :, None] - q.cent[None, None, :]), axis=2)
    assert np.array_equal(p["idx_codes"], nearest)
    n16 = O.fp16_from_bits(p["norms"][:, 0])
    assert np.allclose(n16, np.linalg.norm(x, axis=1), rtol=2.0 ** -11)


# ---------------------------------------------------------------- Theorem 2 (unbiasedness)
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_theorem2_prod_estimator_unbiased(bits):
    """validate_paper.py test_prod_unbiased: d=128, N=5000, 20 trials with quantizer seed
    trial*100; the mean bias over trials must be within 3 standard errors of 0 (and under
    the page's 0.05)."""
    biases = []
    for trial in range(20):
        q = O.build_quantizer(D, bits, "prod", trial * 100)
        g = np.random.default_rng(1000 + trial)
        x = g.standard_normal((5000, D))
        y = g.standard_normal(D)
        est = O.key_scores(q, O.quantize_keys(q, x), y)
        biases.append(np.mean(est - x @ y))
    biases = np.array(biases)
    se = biases.std(ddof=1) / math.sqrt(len(biases))
    assert abs(biases.mean()) < 3.0 * se + 1e-12, (biases.mean(), se)
    assert abs(biases.mean()) < 0.05


def test_qjl_identity_expectation():
    """E[<s,y> sign<s,r>] = sqrt(2/pi) <y,r>/||r|| for s ~ N(0, I): the identity that makes
    r16 sqrt(pi/2)/d <S y, sign(S r)> unbiased. Checked by Monte Carlo over many Gaussian
    rows, independently of the quantizer code."""
    g = np.random.default_rng(3)
    y = g.standard_normal(16)
    r = g.standard_normal(16)
    s = g.standard_normal((2_000_000, 16))
    lhs = np.mean((s @ y) * np.sign(s @ r))
    rhs = math.sqrt(2 / math.pi) * (y @ r) / np.linalg.norm(r)
    assert abs(lhs - rhs) < 4.0 * np.linalg.norm(y) / math.sqrt(2e6)


def test_prod_estimator_without_residual_term_is_biased():
    """Sanity of the tests above: the MSE part alone shrinks <y,x> by about the codebook
    distortion (1-bit MSE: D = 0.36); the full prod estimate, averaged over quantizer seeds
    (the expectation Theorem 2 takes), does not."""
    g = np.random.default_rng(4)
    y = g.standard_normal(D)
    x = g.standard_normal((2000, D)) + 2.0 * y / np.linalg.norm(y)
    true = x @ y
    b_mse, b_full = [], []
    for seed in range(12):
        q = O.build_quantizer(D, 2, "prod", 7 * seed + 1)
        p = O.quantize_keys(q, x)
        mse_only = dict(p, signs=np.zeros_like(p["signs"]),
                        norms=np.stack([p["norms"][:, 0], np.zeros(2000, dtype=np.uint16)], 1))
        b_mse.append(np.mean(O.key_scores(q, mse_only, y) - true))
        b_full.append(np.mean(O.key_scores(q, p, y) - true))
    c, t = O.lloyd_max_gaussian(1)
    shrink = O.gaussian_distortion(c, t)
    assert abs(np.mean(b_mse) / np.mean(true) + shrink) < 0.1
    assert abs(np.mean(b_full)) < 0.1 * abs(np.mean(b_mse))


# ---------------------------------------------------------------- Theorem 3 and quality
def test_theorem3_distortion_scaling():
    """validate_paper.py test_prod_distortion_scaling: N=2000, b=2,3,4; each extra bit cuts
    the inner-product distortion by more than 2x; and D_prod <= sqrt(3) pi^2 ||y||^2/d 4^-b."""
    g = np.random.default_rng(42)
    x = g.standard_normal((2000, D))
    y = g.standard_normal(D)
    dist = {}
    for bits in (2, 3, 4):
        q = O.build_quantizer(D, bits, "prod", 42)
        est = O.key_scores(q, O.quantize_keys(q, x), y)
        # per unit-norm key: the theorem is stated for ||x|| = 1
        nx = np.linalg.norm(x, axis=1)
        dist[bits] = np.mean(((est - x @ y) / nx) ** 2)
        assert dist[bits] <= math.sqrt(3) * math.pi ** 2 * (y @ y) / D * 4.0 ** -bits
    assert dist[2] / dist[3] > 2.0 and dist[3] / dist[4] > 2.0


def test_recall_at_8():
    """validate_paper.py test_recall_at_scale: d=128, N=4096, 32 queries, x0.1 scale;
    recall@8 >= 0.40 (3-bit), >= 0.55 (4-bit), 4-bit > 3-bit."""
    g = np.random.default_rng(42)
    keys = g.standard_normal((4096, D)) * 0.1
    queries = g.standard_normal((32, D)) * 0.1
    true = np.argsort(-(queries @ keys.T), axis=1)[:, :8]
    rec = {}
    for bits in (3, 4):
        q = O.build_quantizer(D, bits, "prod", 42)
        p = O.quantize_keys(q, keys)
        est = np.stack([O.key_scores(q, p, y) for y in queries])
        top = np.argsort(-est, axis=1)[:, :8]
        rec[bits] = np.mean([len(set(a) & set(b)) / 8 for a, b in zip(true, top)])
    assert rec[3] >= 0.40 and rec[4] >= 0.55 and rec[4] > rec[3], rec


def test_rank_correlation():
    """validate_paper.py test_rank_correlation_scale: N=2048; Spearman > 0.75 (3-bit),
    > 0.90 (4-bit)."""
    g = np.random.default_rng(42)
    keys = g.standard_normal((2048, D)) * 0.1
    y = g.standard_normal(D) * 0.1
    for bits, floor in ((3, 0.75), (4, 0.90)):
        q = O.build_quantizer(D, bits, "prod", 42)
        est = O.key_scores(q, O.quantize_keys(q, keys), y)
        assert stats.spearmanr(est, keys @ y).statistic > floor


# ---------------------------------------------------------------- estimator structure
@pytest.mark.parametrize("mode,bits", [("mse", 2), ("prod", 3), ("prod", 4), ("grouped", 2)])
def test_score_equals_inner_product_with_reconstruction(mode, bits):
    """The rotated-domain score (Pi y, S y) equals <y, x_tilde> with x_tilde rebuilt in the
    original coordinates (Pi^T c[idx], S^T signs): pins Pi against Pi^T and the sign map."""
    q = O.build_quantizer(D, bits, mode, 17, np.arange(3, 128, 4))
    g = np.random.default_rng(8)
    x = g.standard_normal((200, D)) * 4
    y = g.standard_normal(D)
    p = O.quantize_keys(q, x)
    assert np.allclose(O.key_scores(q, p, y), O.reconstruct_keys(q, p) @ y, atol=1e-9)


def test_prod_residual_and_signs_definition():
    """r = x - x_mse with x_mse from the stored fp16 norm; sigma_j = [(S r)_j >= 0];
    S = S_rot Pi has i.i.d. N(0,1)-like rows (orthogonal mixing of a Gaussian matrix)."""
    q = O.build_quantizer(D, 3, "prod", 1)
    g = np.random.default_rng(12)
    x = g.standard_normal((64, D)) * 7
    p = O.quantize_keys(q, x)
    # rebuild the MSE part by hand from the packed bytes
    idx = O.unpack_bits(p["idx"], 2, D)
    n16 = O.fp16_from_bits(p["norms"][:, 0])
    xm = n16[:, None] * (q.cent[idx] @ q.Pi)
    r = x - xm
    assert np.array_equal(O.unpack_bits(p["signs"], 1, D), ((r @ q.S.T) >= 0).astype(int))
    assert np.allclose(O.fp16_from_bits(p["norms"][:, 1]), np.linalg.norm(r, axis=1),
                       rtol=2.0 ** -11)
    assert np.allclose(q.S @ q.S.T / D, np.eye(D), atol=0.5)


def test_zero_row_is_defined():
    """A zero key: norm 0, u = 0 (idx = number of negative thresholds), residual 0, all
    signs +1, and every score 0."""
    q = O.build_quantizer(D, 4, "prod", 0)
    p = O.quantize_keys(q, np.zeros((1, D)))
    assert np.all(p["idx_codes"] == 3)                    # 3-bit MSE: 3 negative thresholds
    assert p["norms"].tolist() == [[0, 0]]
    assert np.all(p["signs"] == 255)
    assert O.key_scores(q, p, np.ones(D))[0] == 0.0


def test_grouped_mode_layout_and_independence():
    outl = np.sort(np.random.default_rng(0).choice(128, 32, replace=False))
    q = O.build_quantizer(D, 2, "grouped", 3, outl)
    x = np.random.default_rng(5).standard_normal((500, D))
    x[:, outl] *= 4
    p = O.quantize_keys(q, x)
    assert p["idx"].shape == (500, 16 + 24)
    n = O.fp16_from_bits(p["norms"])
    assert np.allclose(n[:, 0], np.linalg.norm(x[:, outl], axis=1), rtol=2.0 ** -11)
    normals = np.setdiff1d(np.arange(128), outl)
    assert np.allclose(n[:, 1], np.linalg.norm(x[:, normals], axis=1), rtol=2.0 ** -11)
    # the outlier channels alone decide the first 16 bytes
    x2 = x.copy()
    x2[:, normals] = np.random.default_rng(6).standard_normal((500, 96))
    p2 = O.quantize_keys(q, x2)
    assert np.array_equal(p["idx"][:, :16], p2["idx"][:, :16])
    # grouped beats plain mse at the same base width on outlier-heavy rows
    qm = O.build_quantizer(D, 2, "mse", 3)
    e_g = np.mean(np.sum((x - O.reconstruct_keys(q, p)) ** 2, 1) / np.sum(x * x, 1))
    e_m = np.mean(np.sum((x - O.reconstruct_keys(qm, O.quantize_keys(qm, x))) ** 2, 1)
                  / np.sum(x * x, 1))
    assert e_g < e_m


# ---------------------------------------------------------------- values
@pytest.mark.parametrize("bits", [2, 4])
def test_value_quantization_brute_force(bits):
    g = np.random.default_rng(bits)
    v = (g.standard_normal((400, D)) * g.uniform(0.1, 5, (400, 1))).astype(np.float32)
    out = O.quantize_values(v, bits)
    vh = O.dequantize_values(out["q"], out["params"], bits, D)
    mn = O.fp16_from_bits(out["params"][..., 0])
    sc = O.fp16_from_bits(out["params"][..., 1])
    gi = np.repeat(np.arange(4), 32)
    # codes in range; each value within half a step of its reconstruction, up to the fp16
    # rounding of min and scale (mn16 off by <= 2^-11 |mn|, the top code off by the scale's
    # rounding times the code)
    assert out["codes"].min() >= 0 and out["codes"].max() <= (1 << bits) - 1
    slack = 2.0 ** -11 * (np.abs(mn[:, gi]) + ((1 << bits) - 1) * sc[:, gi]) + 1e-12
    assert np.all(np.abs(v - vh) <= 0.5 * sc[:, gi] + slack)
    # brute force: the code is the nearest level mn16 + k s16 (ties either way)
    levels = mn[:, gi, None] + np.arange(1 << bits)[None, None, :] * sc[:, gi, None]
    best = np.min(np.abs(v[:, :, None] - levels), axis=2)
    got = np.abs(v - vh)
    # (fp32 rounding of the quotient can flip a near-tie: up to a few ulp of 15 steps)
    assert np.all(got <= best + 4e-6 * sc[:, gi] + 1e-12)


def test_value_constant_group_is_exact():
    v = np.full((3, D), 0.75)
    v[1, 32:64] = -2.0
    out = O.quantize_values(v, 2)
    assert np.array_equal(O.dequantize_values(out["q"], out["params"], 2, D), v)
    assert np.all(out["codes"] == 0)


def test_value_layout_and_bytes():
    out2 = O.quantize_values(np.zeros((5, D)), 2)
    out4 = O.quantize_values(np.zeros((5, D)), 4)
    assert out2["q"].shape == (5, 32) and out4["q"].shape == (5, 64)
    assert out2["params"].shape == (5, 4, 2)


# ---------------------------------------------------------------- decode attention
def _cache_from(q, keys, vals, vbits=2):
    """keys, vals: (B, H, N, d) -> oracle cache dict."""
    B, H, N, d = keys.shape
    p = O.quantize_keys(q, keys.reshape(-1, d))
    v = O.quantize_values(vals.reshape(-1, d), vbits)
    c = dict(k_idx=p["idx"].reshape(B, H, N, -1), k_norms=p["norms"].reshape(B, H, N, -1),
             v_q=v["q"].reshape(B, H, N, -1), v_params=v["params"].reshape(B, H, N, 4, 2),
             len=np.full(B, N))
    if q.mode == "prod":
        c["k_signs"] = p["signs"].reshape(B, H, N, -1)
    return c


def test_decode_single_key_returns_its_value():
    q = O.build_quantizer(D, 3, "prod", 0)
    g = np.random.default_rng(1)
    k = g.standard_normal((1, 1, 1, D))
    v = g.standard_normal((1, 1, 1, D))
    c = _cache_from(q, k, v)
    out, _ = O.decode_attention(q, c, g.standard_normal((1, 2, D)))
    vh = O.dequantize_values(c["v_q"][0, 0], c["v_params"][0, 0], 2, D)[0]
    assert np.allclose(out[0, 0], vh, atol=1e-15) and np.allclose(out[0, 1], vh, atol=1e-15)


def test_decode_equal_scores_average_values_and_two_key_closed_form():
    q = O.build_quantizer(D, 3, "prod", 0)
    g = np.random.default_rng(2)
    k1 = g.standard_normal(D)
    k = np.stack([k1, k1, k1])[None, None]
    v = g.standard_normal((1, 1, 3, D))
    c = _cache_from(q, k, v)
    out, _ = O.decode_attention(q, c, g.standard_normal((1, 1, D)))
    vh = O.dequantize_values(c["v_q"][0, 0], c["v_params"][0, 0], 2, D)
    assert np.allclose(out[0, 0], vh.mean(axis=0), atol=1e-14)
    # two keys: weight of key 0 is the logistic of the logit gap
    k = g.standard_normal((1, 1, 2, D)) * 3
    c = _cache_from(q, k, v[:, :, :2])
    y = g.standard_normal((1, 1, D))
    out, sc = O.decode_attention(q, c, y, want_scores=True)
    s = sc[0][0]
    w0 = 1.0 / (1.0 + math.exp((s[1] - s[0]) / math.sqrt(D)))
    vh = O.dequantize_values(c["v_q"][0, 0], c["v_params"][0, 0], 2, D)
    assert np.allclose(out[0, 0], w0 * vh[0] + (1 - w0) * vh[1], atol=1e-13)


def test_decode_head_map_and_lengths():
    """GQA: query head h reads KV head head_map[h]; tokens at or beyond len[b] are ignored."""
    q = O.build_quantizer(D, 3, "prod", 0)
    g = np.random.default_rng(3)
    k = g.standard_normal((2, 2, 6, D))
    v = g.standard_normal((2, 2, 6, D))
    c = _cache_from(q, k, v)
    c["len"] = np.array([6, 4])
    Q = g.standard_normal((2, 4, D))
    out, _ = O.decode_attention(q, c, Q)
    # head 3 -> kv 1 under the default map; compare to a cache holding only kv 1's first 4
    c1 = {key: (val[1:2, 1:2, :4] if key != "len" else np.array([4])) for key, val in c.items()}
    out1, _ = O.decode_attention(q, c1, Q[1:2, 3:4])
    assert np.allclose(out[1, 3], out1[0, 0], atol=1e-15)
    hm = np.array([1, 1, 0, 0])
    out2, _ = O.decode_attention(q, c, Q, head_map=hm)
    c2 = {key: (val[0:1, 1:2] if key != "len" else np.array([6])) for key, val in c.items()}
    out3, _ = O.decode_attention(q, c2, Q[0:1, 0:1])
    assert np.allclose(out2[0, 0], out3[0, 0], atol=1e-15)


def test_needle_retrieval_small():
    """validate_paper.py test_needle_retrieval_depths, reduced: H_kv=2, N=1024, keys x0.02,
    needle x3.0; the needle has the top estimated score for its own query."""
    for bits in (3, 4):
        q = O.build_quantizer(D, bits, "prod", 0)
        g = np.random.default_rng(bits)
        for depth in (0.1, 0.5, 0.9):
            k = g.standard_normal((1, 2, 1024, D)) * 0.02
            pos = int(1024 * depth)
            needle = g.standard_normal((2, D)) * 3.0
            k[0, :, pos] = needle
            c = _cache_from(q, k, g.standard_normal((1, 2, 1024, D)))
            _, sc = O.decode_attention(q, c, needle[None], want_scores=True)
            for h in range(2):
                assert int(np.argmax(sc[0][h])) == pos


def _slice_cache(c, start, stop):
    """Tokens [start, stop) of every sequence (clipped to its length) as a cache of their own."""
    out = {k: v[:, :, start:stop] for k, v in c.items() if k != "len"}
    out["len"] = np.clip(c["len"] - start, 0, stop - start)
    return out


def test_context_split_merge_equals_full_decode():
    """Softmax over a union of disjoint token sets is the log-sum-exp merge of per-set records:
    decode_partial over ragged slices of the context (one slice empty for the shorter
    sequence) merged by merge_partials reproduces decode_attention over the whole context,
    for prod and mse keys, a GQA head map and a non-default scale."""
    g = np.random.default_rng(17)
    for mode, bits in (("prod", 3), ("mse", 2)):
        q = O.build_quantizer(D, bits, mode, 3)
        k = g.standard_normal((2, 2, 300, D)) * g.uniform(2, 20, (2, 2, 300, 1))
        c = _cache_from(q, k, g.standard_normal((2, 2, 300, D)))
        c["len"] = np.array([300, 120])
        Q = g.standard_normal((2, 4, D))
        hm = np.array([0, 1, 1, 0])
        full, _ = O.decode_attention(q, c, Q, head_map=hm, sm_scale=0.07)
        for cuts in ((0, 300), (0, 100, 300), (0, 37, 150, 299, 300)):
            parts = [O.decode_partial(q, _slice_cache(c, a, b), Q, head_map=hm, sm_scale=0.07)
                     for a, b in zip(cuts[:-1], cuts[1:])]
            merged = O.merge_partials(*zip(*parts))
            assert np.allclose(merged, full, rtol=0, atol=1e-12), (mode, cuts)
        # an empty slice: (-inf, 0, 0), and merging it changes nothing
        m, l, o = O.decode_partial(q, _slice_cache(c, 300, 300), Q, head_map=hm)
        assert np.all(m == -np.inf) and np.all(l == 0) and np.all(o == 0)
