"""CPU-only checks of the C-ABI library: it loads, exports every entry point include/tq.h
declares, its host-side tables agree with the oracle's (computed independently), and host
argument checks reject bad input before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

tq = pytest.importorskip("kv_cache_vector_fwht_b200")


def declared_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tq.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(tq.EXPORTED) <= set(names)
    assert tq.tq_abi_version() == 1


def test_status_strings():
    assert tq.tq_status_string(0) == "ok"
    assert "capacity" in tq.tq_status_string(tq.TQ_ECAPACITY)


@pytest.mark.parametrize("mode,bits", [("mse", 1), ("mse", 2), ("mse", 3), ("mse", 4),
                                       ("prod", 2), ("prod", 3), ("prod", 4),
                                       ("grouped", 1), ("grouped", 2), ("grouped", 3)])
def test_host_tables_match_oracle(mode, bits):
    outl = np.sort(np.random.default_rng(4).choice(128, 32, replace=False)) if mode == "grouped" else None
    seed = 12345 + bits
    t = tq.tq_host_tables(128, bits, mode, seed, outl)
    q = O.build_quantizer(128, bits, mode, seed, outl)
    if mode == "grouped":
        groups = q.groups
        for gi, g in enumerate(groups):
            c, th = O.lloyd_max_gaussian(g.bits)
            n = len(c)
            # fp64 agreement to rounding; fp32 (what the kernels use) identical
            assert np.allclose(t["centroids"][gi][:n], c, rtol=0, atol=1e-13)
            assert np.array_equal(t["centroids"][gi][:n].astype(np.float32), c.astype(np.float32))
            assert np.array_equal(t["thresholds"][gi][:n - 1].astype(np.float32), th.astype(np.float32))
        assert np.array_equal(t["signs"][:32], groups[0].signs.astype(np.int8))
        assert np.array_equal(t["signs"][32:], groups[1].signs.astype(np.int8))
        assert np.array_equal(t["channels"][:32], q.outliers)
        assert np.array_equal(t["channels"][32:], q.normals)
    else:
        mb = bits if mode == "mse" else bits - 1
        c, th = O.lloyd_max_gaussian(mb)
        n = len(c)
        assert np.array_equal(t["centroids"][0][:n].astype(np.float32), c.astype(np.float32))
        assert np.array_equal(t["thresholds"][0][:n - 1].astype(np.float32), th.astype(np.float32))
        assert t["thresholds"][0][n // 2 - 1] == 0.0
        assert np.array_equal(t["signs"], q.signs.astype(np.int8))
        if mode == "prod":
            assert np.array_equal(O.fp16_from_bits(t["s_rot_fp16"]), q.S_rot)


@pytest.mark.parametrize("args,status", [
    ((64, 3, "prod", 0, None), tq.TQ_EUNSUPPORTED),    # d != 128 on the GPU path
    ((100, 3, "prod", 0, None), tq.TQ_EINVAL),         # not a power of two
    ((128, 5, "mse", 0, None), tq.TQ_EUNSUPPORTED),
    ((128, 1, "prod", 0, None), tq.TQ_EUNSUPPORTED),
    ((128, 4, "grouped", 0, list(range(32))), tq.TQ_EUNSUPPORTED),
    ((128, 2, "grouped", 0, None), tq.TQ_EINVAL),      # outliers missing
    ((128, 2, "grouped", 0, list(range(31)) + [30]), tq.TQ_EINVAL),   # duplicate
    ((128, 2, "grouped", 0, list(range(31)) + [128]), tq.TQ_EINVAL),  # out of range
    ((128, 2, "mse", 0, list(range(32))), tq.TQ_EINVAL),              # outliers on mse
])
def test_build_rejects_bad_arguments_on_host(args, status):
    with pytest.raises(tq.TQError) as e:
        tq.tq_host_tables(*args)
    assert e.value.status == status
    with pytest.raises(tq.TQError) as e:
        tq.tq_build_codebook(*args)
    assert e.value.status == status


def test_workspace_size_is_host_only():
    desc = tq.KVCacheDesc()
    desc.batch, desc.n_kv_heads, desc.capacity, desc.d = 8, 4, 32768 + 256, 128
    n = ctypes.c_size_t()
    assert tq._lib.tq_decode_workspace_bytes(ctypes.byref(desc), 28, ctypes.byref(n)) == 0
    assert n.value > 8 * 28 * 132 * 4
    assert tq._lib.tq_decode_workspace_bytes(ctypes.byref(desc), 0, ctypes.byref(n)) == tq.TQ_EINVAL


@pytest.mark.parametrize("limit_us", [0, 2_000_001])
def test_selftest_wait_limit_checked_on_host(limit_us):
    with pytest.raises(tq.TQError) as e:
        tq.tq_selftest_bounded_wait(limit_us)
    assert e.value.status == tq.TQ_EINVAL


def test_merge_partials_checks_arguments_on_host():
    """tq_merge_partials rejects bad arguments before any device work (no GPU needed)."""
    lib = tq._lib
    buf = (ctypes.c_float * (4 * 132 + 4))()
    aligned = (ctypes.addressof(buf) + 15) // 16 * 16
    ok = dict(parts=aligned, n=1, b=1, h=1, out=aligned, dt=tq.TQ_F32)
    cases = [(dict(n=0), tq.TQ_EINVAL), (dict(n=65537), tq.TQ_EINVAL), (dict(b=0), tq.TQ_EINVAL),
             (dict(h=513), tq.TQ_EINVAL), (dict(parts=None), tq.TQ_EINVAL),
             (dict(parts=aligned + 4), tq.TQ_EINVAL), (dict(out=None), tq.TQ_EINVAL),
             (dict(dt=7), tq.TQ_EUNSUPPORTED)]
    for change, status in cases:
        a = dict(ok, **change)
        assert lib.tq_merge_partials(a["parts"], a["n"], a["b"], a["h"], a["out"], a["dt"],
                                     None) == status, change


def test_decode_policy_setter_on_host():
    prev = tq.tq_set_decode_policy(tq.TQ_DECODE_ONE_SET)
    try:
        assert tq.tq_set_decode_policy(tq.TQ_DECODE_TWO_SETS) == tq.TQ_DECODE_ONE_SET
        with pytest.raises(tq.TQError) as e:
            tq.tq_set_decode_policy(3)
        assert e.value.status == tq.TQ_EINVAL
        assert tq.tq_set_decode_policy(tq.TQ_DECODE_AUTO) == tq.TQ_DECODE_TWO_SETS
    finally:
        tq.tq_set_decode_policy(prev)
