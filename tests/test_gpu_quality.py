"""Quality gates of the GPU path on synthetic data (validate_paper.py test_recall_at_scale and
test_rank_correlation_scale): keys quantized by tq_append on the GPU, inner-product estimates
read from tq_decode_attention's scores on the GPU, compared with the exact dot products."""
import numpy as np
import pytest
import torch
from scipy import stats

from gpu_util import require_cuda

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402

D = 128


def gpu_scores(keys: np.ndarray, queries: np.ndarray, bits: int, mode: str = "prod"):
    dev = require_cuda()
    n, nq = keys.shape[0], queries.shape[0]
    qz = tq.tq_build_codebook(D, bits, mode, 42)
    cap = ((n + 15) // 16) * 16
    cache = tq.KVCache(qz, 1, 1, cap, value_bits=0, device=dev)
    tq.tq_append(qz, cache, torch.from_numpy(keys).float().to(dev).reshape(1, 1, n, D), None)
    scores = torch.empty((1, nq, cap), device=dev)
    ws = tq.alloc_decode_workspace(cache, nq)
    q = torch.from_numpy(queries).float().to(dev).reshape(1, nq, D)
    tq.tq_decode_attention(qz, cache, q, None, ws, head_map=[0] * nq, scores=scores)
    torch.cuda.synchronize()
    return scores[0, :, :n].cpu().numpy().astype(np.float64)


def test_gpu_recall_at_8():
    g = np.random.default_rng(42)
    keys = (g.standard_normal((4096, D)) * 0.1).astype(np.float32)
    queries = (g.standard_normal((32, D)) * 0.1).astype(np.float32)
    true = np.argsort(-(queries.astype(np.float64) @ keys.T.astype(np.float64)), axis=1)[:, :8]
    rec = {}
    for bits in (3, 4):
        est = gpu_scores(keys, queries, bits)
        top = np.argsort(-est, axis=1)[:, :8]
        rec[bits] = np.mean([len(set(a) & set(b)) / 8 for a, b in zip(true, top)])
    print("recall@8", rec)
    assert rec[3] >= 0.40 and rec[4] >= 0.55 and rec[4] > rec[3], rec


def test_gpu_rank_correlation():
    g = np.random.default_rng(42)
    keys = (g.standard_normal((2048, D)) * 0.1).astype(np.float32)
    y = (g.standard_normal((4, D)) * 0.1).astype(np.float32)
    for bits, floor in ((3, 0.75), (4, 0.90)):
        est = gpu_scores(keys, y, bits)
        exact = y.astype(np.float64) @ keys.T.astype(np.float64)
        rho = [stats.spearmanr(est[i], exact[i]).statistic for i in range(y.shape[0])]
        print("spearman", bits, rho)
        assert min(rho) > floor


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gpu_mse_keys_track_exact_scores(bits):
    """mse caches: more bits, closer estimates (the bits-per-coordinate trade-off)."""
    g = np.random.default_rng(7)
    keys = (g.standard_normal((2048, D))).astype(np.float32)
    y = (g.standard_normal((2, D))).astype(np.float32)
    est = gpu_scores(keys, y, bits, "mse")
    exact = y.astype(np.float64) @ keys.T.astype(np.float64)
    rho = min(stats.spearmanr(est[i], exact[i]).statistic for i in range(2))
    assert rho > {2: 0.90, 3: 0.96, 4: 0.985}[bits], rho
