"""Host argument checks of every hot-path entry point, on CPU (no GPU, nothing launched).

A quantizer built with tq_build_codebook_host has no device tables: each call below runs its
argument checks and returns their error; a call whose arguments are all valid returns
TQ_ECUDA ("no device copy") without launching. So for every case, a specific error status
(rather than TQ_ECUDA) shows that the check fired on the host. Device pointers are fake but
16-byte aligned numbers: the library never dereferences device memory on the host.
"""
import ctypes

import pytest

tq = pytest.importorskip("kv_cache_vector_fwht_b200")

lib = tq._lib
EINVAL, EUNSUP, ECAP, ECUDA = tq.TQ_EINVAL, tq.TQ_EUNSUPPORTED, tq.TQ_ECAPACITY, tq.TQ_ECUDA
BASE = 1 << 32          # a fake, 256-byte aligned device address
F32, BF16, F16 = tq.TQ_F32, tq.TQ_BF16, tq.TQ_F16


def dev(i):
    """Distinct fake device buffers, 1 MiB apart (16-byte aligned)."""
    return BASE + i * (1 << 20)


@pytest.fixture(scope="module")
def qp():
    return tq.tq_build_codebook_host(128, 3, "prod", 0)


@pytest.fixture(scope="module")
def qm():
    return tq.tq_build_codebook_host(128, 2, "mse", 0)


def planes(prod=True, idx=dev(1), signs=dev(2), norms=dev(3)):
    return tq.KeyPlanes(idx, signs if prod else None, norms)


class Cache:
    """A cache descriptor over fake device planes (host lengths are real)."""

    def __init__(self, batch=2, n_kv=2, cap=64, vbits=2, lens=(10, 20), prod=True):
        self.len_host = (ctypes.c_int32 * batch)(*lens)
        self.desc = tq.KVCacheDesc(batch, n_kv, cap, 128, vbits, 32, planes(prod),
                                   tq.ValuePlanes(dev(4) if vbits else None,
                                                  dev(5) if vbits else None),
                                   dev(6), self.len_host)

    def ref(self):
        return ctypes.byref(self.desc)

    def lengths(self):
        return list(self.len_host)


def ws_bytes(c, hq):
    """Workspace bytes for hq query heads (1 MiB where hq itself is invalid)."""
    n = ctypes.c_size_t()
    if lib.tq_decode_workspace_bytes(c.ref(), hq, ctypes.byref(n)) != 0:
        return 1 << 20
    return n.value


def test_host_quantizer_layout_and_free():
    q = tq.tq_build_codebook_host(128, 4, "prod", 7)
    assert q.layout["bytes_per_key"] == 84
    g = tq.tq_build_codebook_host(128, 2, "grouped", 1, list(range(0, 128, 4)))
    assert g.layout["bytes_per_key"] == 44
    del q, g   # tq_free of host-only quantizers


# ------------------------------------------------------------------ tq_quantize_keys
@pytest.mark.parametrize("change,status", [
    ({}, ECUDA),                                   # all valid: checks pass, nothing launched
    (dict(n=0), tq.TQ_OK),                         # no rows: a no-op
    (dict(n=-1), EINVAL),
    (dict(x=None), EINVAL),
    (dict(x=dev(0) + 8), EINVAL),                  # misaligned rows
    (dict(dt=F16), EUNSUP),
    (dict(dt=9), EUNSUP),
    (dict(ld=64), EINVAL),                         # ld < d
    (dict(ld=132), EINVAL),                        # bf16 row stride not a multiple of 16 B
    (dict(p=planes(idx=None)), EINVAL),
    (dict(p=planes(idx=dev(1) + 4)), EINVAL),
    (dict(p=planes(signs=None)), EINVAL),          # prod needs sign bytes
    (dict(p=planes(norms=dev(3) + 2)), EINVAL),    # norms of prod keys are 4-byte pairs
])
def test_quantize_keys_checks(qp, change, status):
    a = dict(x=dev(0), dt=BF16, n=100, ld=128, p=planes())
    a.update(change)
    assert lib.tq_quantize_keys(qp.handle, a["x"], a["dt"], a["n"], a["ld"], a["p"], None) == status
    assert lib.tq_quantize_keys(None, a["x"], a["dt"], 100, a["ld"], a["p"], None) == EINVAL


def test_dequantize_keys_checks(qp):
    ok = lib.tq_dequantize_keys(qp.handle, planes(), 10, dev(0), F32, 128, None)
    assert ok == ECUDA
    assert lib.tq_dequantize_keys(qp.handle, planes(), 10, dev(0) + 4, F32, 128, None) == EINVAL
    assert lib.tq_dequantize_keys(qp.handle, planes(), 10, dev(0), F16, 128, None) == EUNSUP
    assert lib.tq_dequantize_keys(qp.handle, planes(signs=None), 10, dev(0), F32, 128, None) == EINVAL


# ------------------------------------------------------------------ tq_quantize_values
@pytest.mark.parametrize("change,status", [
    (dict(n=0), tq.TQ_OK),
    (dict(d=64), EUNSUP),
    (dict(bits=3), EUNSUP),
    (dict(group=16), EUNSUP),
    (dict(dt=F16), EUNSUP),
    (dict(v=dev(0) + 2), EINVAL),
    (dict(n=-3), EINVAL),
    (dict(ld=100), EINVAL),
    (dict(q=None), EINVAL),
    (dict(par=None), EINVAL),
    (dict(par=dev(5) + 2), EINVAL),
])
def test_quantize_values_checks(change, status):
    a = dict(v=dev(0), dt=BF16, n=10, ld=128, d=128, bits=2, group=32, q=dev(4), par=dev(5))
    a.update(change)
    st = lib.tq_quantize_values(a["v"], a["dt"], a["n"], a["ld"], a["d"], a["bits"], a["group"],
                                tq.ValuePlanes(a["q"], a["par"]), None)
    assert st == status


# ------------------------------------------------------------------ tq_append
def append(q, c, k=dev(7), v=dev(8), dt=BF16, n=1):
    return lib.tq_append(q.handle, c.ref(), k, v, dt, n, None)


def test_append_checks_leave_lengths(qp):
    c = Cache(cap=32, lens=(10, 31))
    assert append(qp, c) == ECUDA and c.lengths() == [10, 31]       # valid: nothing launched
    assert append(qp, c, n=2) == ECAP and c.lengths() == [10, 31]   # 31 + 2 > 32
    assert append(qp, c, n=0) == tq.TQ_OK
    assert append(qp, c, n=-1) == EINVAL
    assert append(qp, c, k=None) == EINVAL
    assert append(qp, c, k=dev(7) + 8) == EINVAL
    assert append(qp, c, v=None) == EINVAL                         # a cache with values
    assert append(qp, c, dt=F16) == EUNSUP
    ko = Cache(vbits=0)
    assert append(qp, ko, v=dev(8)) == EINVAL                      # key-only cache: no values
    assert append(qp, ko, v=None) == ECUDA
    assert lib.tq_append(None, c.ref(), dev(7), dev(8), BF16, 1, None) == EINVAL


@pytest.mark.parametrize("field,value,status", [
    ("batch", 0, EINVAL), ("n_kv_heads", 0, EINVAL), ("capacity", 40, EINVAL),   # not % 16
    ("capacity", 0, EINVAL), ("d", 64, EUNSUP), ("value_bits", 3, EUNSUP),
    ("value_group", 16, EUNSUP), ("len_dev", None, EINVAL),
])
def test_cache_descriptor_checks(qp, field, value, status):
    c = Cache()
    setattr(c.desc, field, value)
    assert append(qp, c) == status
    hq = 4
    assert lib.tq_decode_attention(qp.handle, c.ref(), dev(9), BF16, hq, None, 0.0, dev(10), F32,
                                   None, 0, dev(11), 1 << 20, None) == status


def test_cache_plane_checks(qp):
    for kp, status in ((planes(idx=None), EINVAL), (planes(signs=None), EINVAL),
                       (planes(norms=dev(3) + 4), EINVAL)):
        c = Cache()
        c.desc.keys = kp
        assert append(qp, c) == status
    c = Cache()
    c.desc.values = tq.ValuePlanes(dev(4) + 1, dev(5))
    assert append(qp, c) == EINVAL
    c = Cache(lens=(10, 65))   # a length beyond the capacity
    assert append(qp, c) == EINVAL


# ------------------------------------------------------------------ tq_decode_attention
def decode(q, c, hq=4, qv=dev(9), qdt=BF16, hm=None, out=dev(10), odt=F32, scores=None,
           sld=0, ws=dev(11), wsb=None):
    wsb = ws_bytes(c, hq) if wsb is None else wsb
    hm_arr = (ctypes.c_int32 * len(hm))(*hm) if hm is not None else None
    return lib.tq_decode_attention(q.handle, c.ref(), qv, qdt, hq, hm_arr, 0.0, out, odt, scores,
                                   sld, ws, wsb, None)


@pytest.mark.parametrize("change,status", [
    ({}, ECUDA),
    (dict(hq=0), EINVAL), (dict(hq=513), EINVAL),
    (dict(hq=3), EINVAL),                           # 3 query heads on 2 KV heads, no map
    (dict(hq=3, hm=[0, 1, 1]), ECUDA),              # with a map
    (dict(hq=3, hm=[0, 2, 1]), EINVAL),             # KV head out of range
    (dict(hq=3, hm=[0, -1, 1]), EINVAL),
    (dict(qv=None), EINVAL), (dict(qv=dev(9) + 4), EINVAL),
    (dict(qdt=F16), EUNSUP),
    (dict(out=None), EINVAL), (dict(out=dev(10) + 8), EINVAL),
    (dict(odt=F16), EUNSUP),
    (dict(scores=dev(12), sld=19), EINVAL),          # scores_ld below the longest length
    (dict(scores=dev(12), sld=20), ECUDA),
    (dict(ws=None), EINVAL), (dict(ws=dev(11) + 4), EINVAL),
    (dict(wsb=1024), EINVAL),                        # workspace too small
])
def test_decode_attention_checks(qp, change, status):
    assert decode(qp, Cache(), **change) == status


def test_decode_key_only_cache(qp):
    ko = Cache(vbits=0)
    assert decode(qp, ko, out=None, scores=dev(12), sld=32) == ECUDA
    assert decode(qp, ko, out=dev(10), scores=dev(12), sld=32) == EINVAL   # no values: no out


def test_decode_partial_checks(qp):
    c = Cache()
    wsb = ws_bytes(c, 4)

    def partial(cache=c, part=dev(13), ws=dev(11), nbytes=wsb, q=qp):
        return lib.tq_decode_attention_partial(q.handle, cache.ref(), dev(9), BF16, 4, None, 0.0,
                                               part, ws, nbytes, None)
    assert partial() == ECUDA
    assert partial(part=None) == EINVAL
    assert partial(part=dev(13) + 4) == EINVAL
    assert partial(cache=Cache(vbits=0)) == EINVAL   # records carry o: values required
    assert partial(ws=None) == EINVAL
    assert partial(nbytes=16) == EINVAL


def test_decode_noalloc_checks(qp):
    c = Cache()

    def na(**kw):
        a = dict(qv=dev(9), hq=4, out=dev(10), odt=F32)
        a.update(kw)
        return lib.tq_decode_attention_noalloc(qp.handle, c.ref(), a["qv"], BF16, a["hq"], None,
                                               0.0, a["out"], a["odt"], None, 0, None)
    assert na() == ECUDA
    assert na(qv=None) == EINVAL
    assert na(hq=5) == EINVAL
    assert na(odt=F16) == EUNSUP


# ------------------------------------------------------------------ tq_append_decode
def append_decode(q, c, hq=4, n=1, hm=None, sld=0, scores=None, wsb=None, k=dev(7)):
    wsb = ws_bytes(c, hq) if wsb is None else wsb
    hm_arr = (ctypes.c_int32 * len(hm))(*hm) if hm is not None else None
    return lib.tq_append_decode(q.handle, c.ref(), k, dev(8), BF16, n, dev(9), BF16, hq, hm_arr,
                                0.0, dev(10), F32, scores, sld, dev(11), wsb, None)


def test_append_decode_rejects_without_side_effects(qp):
    c = Cache(cap=32, lens=(10, 31))
    assert append_decode(qp, c) == ECUDA and c.lengths() == [10, 31]
    assert append_decode(qp, c, n=2) == ECAP
    assert append_decode(qp, c, hq=3) == EINVAL                    # decode argument
    assert append_decode(qp, c, scores=dev(12), sld=31) == EINVAL  # 31 + 1 > scores_ld
    assert append_decode(qp, c, scores=dev(12), sld=32) == ECUDA
    assert append_decode(qp, c, wsb=64) == EINVAL
    assert append_decode(qp, c, k=None) == EINVAL
    assert c.lengths() == [10, 31]


def test_append_decode_too_many_head_groups(qp):
    """More head groups than one decode launch holds (300 KV heads, one query head each):
    refused before the append, so the cache lengths do not move."""
    c = Cache(batch=1, n_kv=300, cap=64, lens=(5,))
    hq = 300
    assert decode(qp, c, hq=hq) == EUNSUP
    assert append_decode(qp, c, hq=hq) == EUNSUP
    assert c.lengths() == [5]


def test_mse_cache_checks(qm):
    c = Cache(prod=False)
    assert append(qm, c) == ECUDA
    assert decode(qm, c) == ECUDA
    c.desc.keys = planes(prod=False, norms=dev(3) + 2)   # norms rows 16-byte aligned in a cache
    assert decode(qm, c) == EINVAL
