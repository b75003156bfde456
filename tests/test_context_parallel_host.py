"""Host logic of context-parallel decode on CPU: the context partition (context_slice) and
the all-gather of partial records (gather_partials) over two gloo ranks, one process each.
Each rank's records come from the oracle (decode_partial over its context slice); after the
gather every rank holds all ranks' records in rank order, and their log-sum-exp merge equals
the oracle's decode over the whole context."""
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


@pytest.mark.parametrize("n,world", [(0, 1), (1, 2), (7, 3), (100, 8), (32768, 8), (131073, 7)])
def test_context_slice_partition(n, world):
    sys.path.insert(0, ROOT)
    from kv_cache_vector_fwht_b200.context_parallel import context_slice
    sl = [context_slice(n, r, world) for r in range(world)]
    assert sl[0][0] == 0 and sl[-1][1] == n
    for (a0, b0), (a1, b1) in zip(sl[:-1], sl[1:]):
        assert b0 == a1
    sizes = [b - a for a, b in sl]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        context_slice(n, world, world)


def _records(O, q, cache, Q, hm):
    """Oracle records in the library's layout: m, l, 0, 0, o[128] per (sequence, head)."""
    m, l, o = O.decode_partial(q, cache, Q, head_map=hm)
    rec = np.zeros(m.shape + (132,))
    rec[..., 0], rec[..., 1], rec[..., 4:] = m, l, o
    return rec


def _rank_main(rank: int, world: int, port: int, q_out):
    try:
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                          MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        import torch
        import torch.distributed as dist

        import oracle as O
        from kv_cache_vector_fwht_b200.context_parallel import context_slice, gather_partials
        dist.init_process_group("gloo", rank=rank, world_size=world)
        g = np.random.default_rng(5)
        q = O.build_quantizer(D, 3, "prod", 1)
        B, H, N = 2, 2, 200
        keys = g.standard_normal((B, H, N, D)) * g.uniform(2, 20, (B, H, N, 1))
        vals = g.standard_normal((B, H, N, D))
        p = O.quantize_keys(q, keys.reshape(-1, D))
        v = O.quantize_values(vals.reshape(-1, D), 2)
        full = dict(k_idx=p["idx"].reshape(B, H, N, -1), k_norms=p["norms"].reshape(B, H, N, -1),
                    k_signs=p["signs"].reshape(B, H, N, -1), v_q=v["q"].reshape(B, H, N, -1),
                    v_params=v["params"].reshape(B, H, N, 4, 2), len=np.array([200, 90]))
        Q = g.standard_normal((B, 4, D))
        hm = np.array([0, 0, 1, 1])
        # this rank's slice of each sequence's context (the shorter one may leave it empty)
        a, b = context_slice(N, rank, world)
        mine = {k: val[:, :, a:b] for k, val in full.items() if k != "len"}
        mine["len"] = np.clip(full["len"] - a, 0, b - a)
        rec = torch.from_numpy(_records(O, q, mine, Q, hm))
        parts = gather_partials(rec.contiguous())
        assert tuple(parts.shape) == (world,) + tuple(rec.shape)
        assert torch.equal(parts[rank], rec)
        arr = parts.numpy()
        merged = O.merge_partials([arr[r][..., 0] for r in range(world)],
                                  [arr[r][..., 1] for r in range(world)],
                                  [arr[r][..., 4:] for r in range(world)])
        ref, _ = O.decode_attention(q, full, Q, head_map=hm)
        err = float(np.max(np.abs(merged - ref)))
        dist.destroy_process_group()
        q_out.put((rank, err))
    except Exception as e:  # report instead of hanging the parent
        q_out.put((rank, "error: " + repr(e)))


def test_two_gloo_ranks_gather_records_and_merge():
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
        assert err < 1e-12, (rank, err)
