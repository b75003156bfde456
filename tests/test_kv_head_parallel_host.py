"""Host logic of KV-head-parallel decode on CPU: the KV-head partition (kv_head_slice), the
rank-local query heads and head map (local_heads), and two gloo ranks that each decode their
KV heads with the oracle under the local map; gathered on rank 0 in query-head order, the
outputs equal the oracle's decode over all KV heads (no exchange is needed in between)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
D = 128


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _helpers():
    """The pure host functions (the package module imports the library binding)."""
    sys.path.insert(0, ROOT)
    from kv_cache_vector_fwht_b200.kv_head_parallel import (default_head_map, kv_head_slice,
                                                            local_heads)
    return kv_head_slice, default_head_map, local_heads


@pytest.mark.parametrize("n,world", [(1, 1), (8, 1), (8, 2), (8, 3), (4, 8), (64, 7)])
def test_kv_head_slice_partition(n, world):
    kv_head_slice, _, _ = _helpers()
    sl = [kv_head_slice(n, r, world) for r in range(world)]
    assert sl[0][0] == 0 and sl[-1][1] == n
    for (a0, b0), (a1, b1) in zip(sl[:-1], sl[1:]):
        assert b0 == a1
    sizes = [b - a for a, b in sl]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        kv_head_slice(n, world, world)


def test_local_heads_cover_every_query_head_once():
    kv_head_slice, default_head_map, local_heads = _helpers()
    hm = default_head_map(64, 8)
    assert hm[:9] == [0] * 8 + [1]
    seen = []
    for r in range(3):
        a, b = kv_head_slice(8, r, 3)
        qs, lmap = local_heads(hm, a, b)
        assert all(0 <= v < b - a for v in lmap)
        assert [hm[h] - a for h in qs] == lmap
        seen += qs
    assert sorted(seen) == list(range(64))
    # an uneven map: some KV heads carry no query head
    qs, lmap = local_heads([2, 2, 0, 5], 1, 4)
    assert qs == [0, 1] and lmap == [1, 1]
    with pytest.raises(ValueError):
        default_head_map(10, 4)


def _rank_main(rank: int, world: int, port: int, q_out):
    try:
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                          MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import torch
        import torch.distributed as dist

        import oracle as O
        kv_head_slice, default_head_map, local_heads = _helpers()
        dist.init_process_group("gloo", rank=rank, world_size=world)
        g = np.random.default_rng(9)
        q = O.build_quantizer(D, 3, "prod", 2)
        B, H, N, Hq = 2, 5, 150, 10
        keys = g.standard_normal((B, H, N, D)) * g.uniform(2, 20, (B, H, N, 1))
        vals = g.standard_normal((B, H, N, D))
        p = O.quantize_keys(q, keys.reshape(-1, D))
        v = O.quantize_values(vals.reshape(-1, D), 2)
        full = dict(k_idx=p["idx"].reshape(B, H, N, -1), k_norms=p["norms"].reshape(B, H, N, -1),
                    k_signs=p["signs"].reshape(B, H, N, -1), v_q=v["q"].reshape(B, H, N, -1),
                    v_params=v["params"].reshape(B, H, N, 4, 2), len=np.array([150, 77]))
        Q = g.standard_normal((B, Hq, D))
        hm = default_head_map(Hq, H)
        a, b = kv_head_slice(H, rank, world)
        qs, lmap = local_heads(hm, a, b)
        mine = {k: val[:, a:b] for k, val in full.items() if k != "len"}
        mine["len"] = full["len"]
        out, _ = O.decode_attention(q, mine, Q[:, qs], head_map=np.array(lmap))
        # gather every rank's (query heads, outputs); sizes differ, so pad to the largest
        pad = np.zeros((B, Hq, D))
        pad[:, :len(qs)] = out
        idx = np.full(Hq, -1)
        idx[:len(qs)] = qs
        outs = [torch.zeros((B, Hq, D), dtype=torch.float64) for _ in range(world)]
        idxs = [torch.zeros(Hq, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(outs, torch.from_numpy(pad))
        dist.all_gather(idxs, torch.from_numpy(idx))
        err = None
        if rank == 0:
            got = np.zeros((B, Hq, D))
            hit = np.zeros(Hq, dtype=int)
            for r in range(world):
                for i, h in enumerate(idxs[r].numpy()):
                    if h >= 0:
                        got[:, h] = outs[r].numpy()[:, i]
                        hit[h] += 1
            assert np.all(hit == 1)
            ref, _ = O.decode_attention(q, full, Q, head_map=np.array(hm))
            err = float(np.max(np.abs(got - ref)))
        dist.destroy_process_group()
        q_out.put((rank, err))
    except Exception as e:  # report instead of hanging the parent
        q_out.put((rank, "error: " + repr(e)))


def test_two_gloo_ranks_decode_their_kv_heads():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err in results:
        assert not isinstance(err, str), err
        if rank == 0:
            assert err == 0.0, err   # the same per-head arithmetic: identical outputs
