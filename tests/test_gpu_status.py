"""Bounded device waits report instead of hanging: a diagnostic kernel whose mbarrier wait
can never complete gives up after its limit, and tq_sync_status returns TQ_ETIMEOUT once
(the flag is then clear). No device fault is involved."""
import pytest
import torch

from gpu_util import require_cuda

pytestmark = pytest.mark.gpu

import kv_cache_vector_fwht_b200 as tq  # noqa: E402


def test_bounded_wait_timeout_is_reported_once():
    dev = require_cuda()
    tq.tq_sync_status()                       # start from a clear flag
    tq.tq_selftest_bounded_wait(20000)        # 20 ms
    with pytest.raises(tq.TQError) as e:
        tq.tq_sync_status()
    assert e.value.status == tq.TQ_ETIMEOUT
    tq.tq_sync_status()                       # cleared
    # the context stays usable: a normal key quantization afterwards reports no error
    qz = tq.tq_build_codebook(128, 3, "prod", 1)
    x = torch.randn((300, 128), device=dev).to(torch.bfloat16)
    planes = qz.alloc_key_planes(300, dev)
    tq.tq_quantize_keys(qz, x, planes)
    tq.tq_sync_status()
