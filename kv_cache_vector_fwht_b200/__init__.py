"""B200 TurboQuant KV-cache quantization and fused decode attention.

A thin ctypes binding over libtq.so (include/tq.h). Every step of the hot path runs in the
library's CUDA kernels; this module only marshals arguments, and uses PyTorch for device
memory and streams. The functions keep the C names (tq_build_codebook, tq_quantize_keys,
tq_quantize_values, tq_append, tq_decode_attention, ...). If libtq.so is missing the import
fails: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int, c_int8, c_int32, c_int64, c_size_t, \
    c_uint16, c_uint64, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python kv_cache_vector_fwht_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ECAPACITY, TQ_ENOMEM, TQ_ECUDA, TQ_ETIMEOUT, TQ_ETOOLARGE = \
    0, -1, -2, -3, -4, -5, -6, -7
TQ_NOALLOC_SCRATCH_BYTES = 16 << 20
MODES = {"mse": 0, "prod": 1, "grouped": 2}
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2
D = 128

EXPORTED = ["tq_build_codebook", "tq_build_codebook_host", "tq_free", "tq_key_layout", "tq_host_tables",
            "tq_quantize_keys", "tq_dequantize_keys", "tq_quantize_values", "tq_append", "tq_decode_workspace_bytes",
            "tq_decode_attention", "tq_decode_attention_noalloc", "tq_append_decode",
            "tq_decode_attention_partial",
            "tq_merge_partials", "tq_set_decode_policy", "tq_sync_status",
            "tq_selftest_bounded_wait", "tq_status_string", "tq_abi_version"]


class KeyLayout(ctypes.Structure):
    _fields_ = [("d", c_int32), ("bits", c_int32), ("mode", c_int32), ("idx_bytes", c_int32),
                ("sign_bytes", c_int32), ("n_norms", c_int32), ("bytes_per_key", c_int32)]


class KeyPlanes(ctypes.Structure):
    _fields_ = [("idx", c_void_p), ("signs", c_void_p), ("norms", c_void_p)]


class ValuePlanes(ctypes.Structure):
    _fields_ = [("q", c_void_p), ("params", c_void_p)]


class KVCacheDesc(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("n_kv_heads", c_int32), ("capacity", c_int32),
                ("d", c_int32), ("value_bits", c_int32), ("value_group", c_int32),
                ("keys", KeyPlanes), ("values", ValuePlanes), ("len_dev", c_void_p),
                ("len_host", POINTER(c_int32))]


_lib.tq_build_codebook.argtypes = [c_int, c_int, c_int, c_uint64, POINTER(c_int32), c_int,
                                   POINTER(c_void_p)]
_lib.tq_build_codebook.restype = c_int
_lib.tq_build_codebook_host.argtypes = [c_int, c_int, c_int, c_uint64, POINTER(c_int32), c_int,
                                        POINTER(c_void_p)]
_lib.tq_build_codebook_host.restype = c_int
_lib.tq_free.argtypes = [c_void_p]
_lib.tq_free.restype = None
_lib.tq_key_layout.argtypes = [c_void_p, POINTER(KeyLayout)]
_lib.tq_key_layout.restype = c_int
_lib.tq_host_tables.argtypes = [c_int, c_int, c_int, c_uint64, POINTER(c_int32), c_int,
                                POINTER(c_double), POINTER(c_double), POINTER(c_int8),
                                POINTER(c_int32), POINTER(c_uint16)]
_lib.tq_host_tables.restype = c_int
_lib.tq_quantize_keys.argtypes = [c_void_p, c_void_p, c_int, c_int64, c_int64, KeyPlanes,
                                  c_void_p]
_lib.tq_quantize_keys.restype = c_int
_lib.tq_dequantize_keys.argtypes = [c_void_p, KeyPlanes, c_int64, c_void_p, c_int, c_int64,
                                    c_void_p]
_lib.tq_dequantize_keys.restype = c_int
_lib.tq_quantize_values.argtypes = [c_void_p, c_int, c_int64, c_int64, c_int, c_int, c_int,
                                    ValuePlanes, c_void_p]
_lib.tq_quantize_values.restype = c_int
_lib.tq_append.argtypes = [c_void_p, POINTER(KVCacheDesc), c_void_p, c_void_p, c_int, c_int,
                           c_void_p]
_lib.tq_append.restype = c_int
_lib.tq_decode_workspace_bytes.argtypes = [POINTER(KVCacheDesc), c_int, POINTER(c_size_t)]
_lib.tq_decode_workspace_bytes.restype = c_int
_lib.tq_decode_attention.argtypes = [c_void_p, POINTER(KVCacheDesc), c_void_p, c_int, c_int,
                                     POINTER(c_int32), c_float, c_void_p, c_int, c_void_p,
                                     c_int64, c_void_p, c_size_t, c_void_p]
_lib.tq_decode_attention.restype = c_int
_lib.tq_decode_attention_noalloc.argtypes = [c_void_p, POINTER(KVCacheDesc), c_void_p, c_int,
                                             c_int, POINTER(c_int32), c_float, c_void_p, c_int,
                                             c_void_p, c_int64, c_void_p]
_lib.tq_decode_attention_noalloc.restype = c_int
_lib.tq_append_decode.argtypes = [c_void_p, POINTER(KVCacheDesc), c_void_p, c_void_p, c_int, c_int,
                                  c_void_p, c_int, c_int, POINTER(c_int32), c_float, c_void_p,
                                  c_int, c_void_p, c_int64, c_void_p, c_size_t, c_void_p]
_lib.tq_append_decode.restype = c_int
_lib.tq_decode_attention_partial.argtypes = [c_void_p, POINTER(KVCacheDesc), c_void_p, c_int,
                                             c_int, POINTER(c_int32), c_float, c_void_p,
                                             c_void_p, c_size_t, c_void_p]
_lib.tq_decode_attention_partial.restype = c_int
_lib.tq_merge_partials.argtypes = [c_void_p, c_int, c_int, c_int, c_void_p, c_int, c_void_p]
_lib.tq_merge_partials.restype = c_int
_lib.tq_set_decode_policy.argtypes = [c_int, POINTER(c_int)]
_lib.tq_set_decode_policy.restype = c_int
_lib.tq_status_string.argtypes = [c_int]
_lib.tq_status_string.restype = ctypes.c_char_p
_lib.tq_abi_version.argtypes = []
_lib.tq_abi_version.restype = c_int
_lib.tq_sync_status.argtypes = [c_void_p]
_lib.tq_sync_status.restype = c_int
_lib.tq_selftest_bounded_wait.argtypes = [ctypes.c_uint32, c_void_p]
_lib.tq_selftest_bounded_wait.restype = c_int


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {tq_status_string(status)} ({status})")


def _check(status: int, where: str) -> None:
    if status != TQ_OK:
        raise TQError(status, where)


def tq_status_string(status: int) -> str:
    return _lib.tq_status_string(status).decode()


def tq_abi_version() -> int:
    return _lib.tq_abi_version()


def tq_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    """Launch the diagnostic kernel whose bounded wait runs out after limit_us microseconds;
    the next tq_sync_status raises TQError(TQ_ETIMEOUT)."""
    in_range = 0 < limit_us <= 2_000_000   # out-of-range limits are rejected on the host
    _check(_lib.tq_selftest_bounded_wait(limit_us, _stream(stream) if in_range else None),
           "tq_selftest_bounded_wait")


def tq_sync_status(stream=None) -> None:
    """Wait for `stream` and raise TQError(TQ_ETIMEOUT) if a library kernel gave up a bounded
    device wait since the previous call (TQ_ECUDA on a CUDA error)."""
    _check(_lib.tq_sync_status(_stream(stream)), "tq_sync_status")


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    if t.dtype == torch.float16:
        return TQ_F16
    return 99


def _stream(stream) -> int | None:
    import torch
    if stream is None:
        try:   # raw handle of the current stream without building a Stream object
            return torch._C._cuda_getCurrentRawStream(torch.cuda.current_device())
        except AttributeError:
            return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


# ------------------------------------------------------------------------ host tables

def tq_host_tables(d: int, bits: int, mode: str, seed: int, outliers=None) -> dict:
    """The library's host-side codebook, signs, channel order and S_rot (no GPU needed)."""
    import numpy as np
    cent = (c_double * 32)()
    thr = (c_double * 32)()
    signs = (c_int8 * 128)()
    chan = (c_int32 * 128)()
    srot = (c_uint16 * (d * d))() if d <= 128 else None
    out_arr, n_out = _outlier_arg(outliers)
    st = _lib.tq_host_tables(d, bits, MODES[mode], seed, out_arr, n_out, cent, thr, signs, chan,
                             srot)
    _check(st, "tq_host_tables")
    return dict(centroids=np.array(cent[:]).reshape(2, 16), thresholds=np.array(thr[:]).reshape(2, 16),
                signs=np.array(signs[:], dtype=np.int8), channels=np.array(chan[:], dtype=np.int32),
                s_rot_fp16=np.array(srot[:], dtype=np.uint16).reshape(d, d) if srot else None)


def _outlier_arg(outliers):
    if outliers is None:
        return None, 0
    vals = [int(v) for v in outliers]
    return (c_int32 * len(vals))(*vals), len(vals)


# ------------------------------------------------------------------------ quantizer

class Quantizer:
    """Owns a tq_quantizer* (tables on the current CUDA device)."""

    def __init__(self, handle: int, d: int, bits: int, mode: str, seed: int):
        self.handle = handle
        self.d, self.bits, self.mode, self.seed = d, bits, mode, seed
        lay = KeyLayout()
        _check(_lib.tq_key_layout(handle, ctypes.byref(lay)), "tq_key_layout")
        self.layout = {f: getattr(lay, f) for f, _ in KeyLayout._fields_}

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h:
            _lib.tq_free(h)

    def alloc_key_planes(self, n_rows: int, device="cuda"):
        import torch
        lay = self.layout
        idx = torch.empty((n_rows, lay["idx_bytes"]), dtype=torch.uint8, device=device)
        sig = (torch.empty((n_rows, lay["sign_bytes"]), dtype=torch.uint8, device=device)
               if lay["sign_bytes"] else None)
        nrm = torch.empty((n_rows, lay["n_norms"]), dtype=torch.int16, device=device)
        return dict(idx=idx, signs=sig, norms=nrm)


def tq_build_codebook(d: int, bits: int, mode: str, seed: int, outliers=None) -> Quantizer:
    h = c_void_p()
    out_arr, n_out = _outlier_arg(outliers)
    _check(_lib.tq_build_codebook(d, bits, MODES[mode], seed, out_arr, n_out, ctypes.byref(h)),
           "tq_build_codebook")
    return Quantizer(h.value, d, bits, mode, seed)


def tq_build_codebook_host(d: int, bits: int, mode: str, seed: int, outliers=None) -> Quantizer:
    """A quantizer without device tables (no GPU needed): plane sizes and argument checks;
    device entry points given it return TQ_ECUDA after their checks (see tq.h)."""
    h = c_void_p()
    out_arr, n_out = _outlier_arg(outliers)
    _check(_lib.tq_build_codebook_host(d, bits, MODES[mode], seed, out_arr, n_out,
                                       ctypes.byref(h)), "tq_build_codebook_host")
    return Quantizer(h.value, d, bits, mode, seed)


def _key_planes(planes: dict) -> KeyPlanes:
    return KeyPlanes(_ptr(planes["idx"]), _ptr(planes.get("signs")), _ptr(planes["norms"]))


def tq_quantize_keys(q: Quantizer, x, planes: dict, stream=None) -> None:
    """x: (n_rows, ld>=128) fp32/bf16 CUDA tensor (row-major, unit stride in columns)."""
    assert x.dim() == 2 and x.stride(1) == 1
    _check(_lib.tq_quantize_keys(q.handle, _ptr(x), _dtype_code(x), x.shape[0], x.stride(0),
                                 _key_planes(planes), _stream(stream)), "tq_quantize_keys")


def tq_dequantize_keys(q: Quantizer, planes: dict, out, stream=None) -> None:
    """planes: key planes of out.shape[0] rows; out: (n_rows, ld>=128) fp32/bf16 CUDA tensor."""
    assert out.dim() == 2 and out.stride(1) == 1
    _check(_lib.tq_dequantize_keys(q.handle, _key_planes(planes), out.shape[0],
                                   _ptr(out), _dtype_code(out), out.stride(0), _stream(stream)),
           "tq_dequantize_keys")


def alloc_value_planes(n_rows: int, bits: int, d: int = D, group: int = 32, device="cuda"):
    import torch
    return dict(q=torch.empty((n_rows, d * bits // 8), dtype=torch.uint8, device=device),
                params=torch.empty((n_rows, d // group, 2), dtype=torch.int16, device=device))


def tq_quantize_values(v, planes: dict, bits: int, group: int = 32, stream=None) -> None:
    assert v.dim() == 2 and v.stride(1) == 1
    _check(_lib.tq_quantize_values(_ptr(v), _dtype_code(v), v.shape[0], v.stride(0), v.shape[1],
                                   bits, group, ValuePlanes(_ptr(planes["q"]), _ptr(planes["params"])),
                                   _stream(stream)), "tq_quantize_values")


# ------------------------------------------------------------------------ cache + decode

class KVCache:
    """A packed KV cache in caller-owned (torch) device memory; see tq_kv_cache in tq.h."""

    def __init__(self, q: Quantizer, batch: int, n_kv_heads: int, capacity: int,
                 value_bits: int = 2, group: int = 32, device="cuda"):
        import torch
        if capacity % 16:
            raise ValueError("capacity must be a multiple of 16")
        self.q = q
        self.batch, self.n_kv_heads, self.capacity = batch, n_kv_heads, capacity
        self.value_bits, self.group = value_bits, group
        rows = batch * n_kv_heads * capacity
        kp = q.alloc_key_planes(rows, device)
        self.k_idx, self.k_signs, self.k_norms = kp["idx"], kp["signs"], kp["norms"]
        if value_bits:
            vp = alloc_value_planes(rows, value_bits, q.d, group, device)
            self.v_q, self.v_params = vp["q"], vp["params"]
        else:
            self.v_q = self.v_params = None
        self.len_dev = torch.zeros(batch, dtype=torch.int32, device=device)
        self.len_host = (c_int32 * batch)()
        self.desc = KVCacheDesc(batch, n_kv_heads, capacity, q.d, value_bits, group,
                                _key_planes(kp),
                                ValuePlanes(_ptr(self.v_q), _ptr(self.v_params)),
                                _ptr(self.len_dev), self.len_host)

    def rows(self, b: int, h: int):
        """Row range of (sequence b, KV head h) in every plane."""
        start = (b * self.n_kv_heads + h) * self.capacity
        return slice(start, start + self.capacity)

    def set_lengths(self, lengths) -> None:
        import torch
        for b, n in enumerate(lengths):
            self.len_host[b] = int(n)
        self.len_dev.copy_(torch.tensor([int(n) for n in lengths], dtype=torch.int32))

    @property
    def lengths(self):
        return [self.len_host[b] for b in range(self.batch)]

    def key_planes(self) -> dict:
        return dict(idx=self.k_idx, signs=self.k_signs, norms=self.k_norms)

    def value_planes(self) -> dict:
        return dict(q=self.v_q, params=self.v_params)


def tq_append(q: Quantizer, cache: KVCache, k_new, v_new=None, stream=None) -> None:
    """k_new / v_new: (batch, n_kv_heads, n_tokens, d) contiguous fp32/bf16 CUDA tensors."""
    assert k_new.is_contiguous() and k_new.dim() == 4
    _check(_lib.tq_append(q.handle, ctypes.byref(cache.desc), _ptr(k_new), _ptr(v_new),
                          _dtype_code(k_new), k_new.shape[2], _stream(stream)), "tq_append")


def tq_decode_workspace_bytes(cache: KVCache, n_q_heads: int) -> int:
    n = c_size_t()
    _check(_lib.tq_decode_workspace_bytes(ctypes.byref(cache.desc), n_q_heads, ctypes.byref(n)),
           "tq_decode_workspace_bytes")
    return n.value


def alloc_decode_workspace(cache: KVCache, n_q_heads: int, device="cuda"):
    import torch
    return torch.zeros(tq_decode_workspace_bytes(cache, n_q_heads), dtype=torch.uint8,
                       device=device)


def tq_decode_attention(q: Quantizer, cache: KVCache, query, out=None, workspace=None,
                        head_map=None, sm_scale: float = 0.0, scores=None, stream=None) -> None:
    """query: (batch, n_q_heads, d) fp32/bf16; out: same shape, fp32/bf16 (None for a
    key-only cache); scores: optional (batch, n_q_heads, scores_ld) fp32."""
    assert query.is_contiguous() and query.dim() == 3
    hq = query.shape[1]
    hm = (c_int32 * hq)(*[int(v) for v in head_map]) if head_map is not None else None
    sld = scores.shape[2] if scores is not None else 0
    wbytes = workspace.numel() if workspace is not None else 0
    _check(_lib.tq_decode_attention(q.handle, ctypes.byref(cache.desc), _ptr(query),
                                    _dtype_code(query), hq, hm, sm_scale, _ptr(out),
                                    _dtype_code(out) if out is not None else TQ_F32,
                                    _ptr(scores), sld, _ptr(workspace), wbytes, _stream(stream)),
           "tq_decode_attention")


def tq_append_decode(q: Quantizer, cache: KVCache, k_new, v_new, query, out=None, workspace=None,
                     head_map=None, sm_scale: float = 0.0, scores=None, stream=None) -> None:
    """One decode step: tq_append(k_new, v_new) then tq_decode_attention(query), launched back
    to back (see tq.h); arguments as for the two calls."""
    assert k_new.is_contiguous() and k_new.dim() == 4
    assert query.is_contiguous() and query.dim() == 3
    hq = query.shape[1]
    hm = (c_int32 * hq)(*[int(v) for v in head_map]) if head_map is not None else None
    sld = scores.shape[2] if scores is not None else 0
    wbytes = workspace.numel() if workspace is not None else 0
    _check(_lib.tq_append_decode(q.handle, ctypes.byref(cache.desc), _ptr(k_new), _ptr(v_new),
                                 _dtype_code(k_new), k_new.shape[2], _ptr(query),
                                 _dtype_code(query), hq, hm, sm_scale, _ptr(out),
                                 _dtype_code(out) if out is not None else TQ_F32, _ptr(scores),
                                 sld, _ptr(workspace), wbytes, _stream(stream)),
           "tq_append_decode")


TQ_DECODE_AUTO, TQ_DECODE_ONE_SET, TQ_DECODE_TWO_SETS = 0, 1, 2


def tq_set_decode_policy(policy: int) -> int:
    """Process-wide decode block shape (see tq.h); returns the previous policy."""
    prev = c_int(0)
    _check(_lib.tq_set_decode_policy(int(policy), ctypes.byref(prev)), "tq_set_decode_policy")
    return prev.value


TQ_PART_FLOATS = 132   # floats per partial record: m, l, 0, 0, o[128]


def tq_decode_attention_partial(q: Quantizer, cache: KVCache, query, part, workspace,
                                head_map=None, sm_scale: float = 0.0, stream=None) -> None:
    """One context slice of a context-parallel decode: part (batch, n_q_heads, TQ_PART_FLOATS)
    fp32 receives this cache's (m, l, o) records (see tq.h)."""
    assert query.is_contiguous() and query.dim() == 3
    assert part.is_contiguous() and part.shape[-1] == TQ_PART_FLOATS
    hq = query.shape[1]
    hm = (c_int32 * hq)(*[int(v) for v in head_map]) if head_map is not None else None
    _check(_lib.tq_decode_attention_partial(q.handle, ctypes.byref(cache.desc), _ptr(query),
                                            _dtype_code(query), hq, hm, sm_scale, _ptr(part),
                                            _ptr(workspace), workspace.numel(), _stream(stream)),
           "tq_decode_attention_partial")


def tq_merge_partials(parts, out, stream=None) -> None:
    """parts: (n_parts, batch, n_q_heads, TQ_PART_FLOATS) fp32, contiguous; out: (batch,
    n_q_heads, d) fp32/bf16 receives the LSE merge of the slices."""
    assert parts.is_contiguous() and parts.dim() == 4 and parts.shape[-1] == TQ_PART_FLOATS
    assert out.is_contiguous() and tuple(out.shape[:2]) == tuple(parts.shape[1:3])
    _check(_lib.tq_merge_partials(_ptr(parts), parts.shape[0], parts.shape[1], parts.shape[2],
                                  _ptr(out), _dtype_code(out), _stream(stream)),
           "tq_merge_partials")


def tq_decode_attention_noalloc(q: Quantizer, cache: KVCache, query, out=None, head_map=None,
                                sm_scale: float = 0.0, scores=None, stream=None) -> None:
    """tq_decode_attention without a workspace: for callers that cannot allocate device
    memory (the library's built-in scratch array is used instead; see tq.h). Raises
    TQError(TQ_ETOOLARGE) when the problem needs more scratch than the array holds."""
    assert query.is_contiguous() and query.dim() == 3
    hq = query.shape[1]
    hm = (c_int32 * hq)(*[int(v) for v in head_map]) if head_map is not None else None
    sld = scores.shape[2] if scores is not None else 0
    _check(_lib.tq_decode_attention_noalloc(q.handle, ctypes.byref(cache.desc), _ptr(query),
                                            _dtype_code(query), hq, hm, sm_scale, _ptr(out),
                                            _dtype_code(out) if out is not None else TQ_F32,
                                            _ptr(scores), sld, _stream(stream)),
           "tq_decode_attention_noalloc")
