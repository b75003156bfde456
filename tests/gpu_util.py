"""Shared helpers of the GPU parity tests: device checks, plane download, oracle caches."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O


def require_cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    return torch.device("cuda:0")


def to_np_planes(planes: dict) -> dict:
    out = {}
    for k, v in planes.items():
        if v is None:
            continue
        a = v.cpu().numpy()
        out[k] = a.view(np.uint16) if a.dtype == np.int16 else a
    return out


def to_device(x: np.ndarray, dtype, device="cuda:0"):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device=device, dtype=dtype)


def oracle_cache(qo, K: np.ndarray, V: np.ndarray | None, value_bits: int, lengths,
                 chunk: int = 32768) -> dict:
    """Quantize K (B, H, N, d) and V with the oracle into the oracle's cache dict."""
    B, H, N, d = K.shape
    lay = O.key_layout(qo)
    k_idx = np.zeros((B, H, N, lay["idx_bytes"]), np.uint8)
    k_nrm = np.zeros((B, H, N, lay["n_norms"]), np.uint16)
    k_sgn = np.zeros((B, H, N, lay["sign_bytes"]), np.uint8) if lay["sign_bytes"] else None
    v_q = np.zeros((B, H, N, d * value_bits // 8), np.uint8) if V is not None else None
    v_p = np.zeros((B, H, N, d // 32, 2), np.uint16) if V is not None else None
    for b in range(B):
        for h in range(H):
            for s in range(0, N, chunk):
                e = min(N, s + chunk)
                p = O.quantize_keys(qo, K[b, h, s:e].astype(np.float64))
                k_idx[b, h, s:e] = p["idx"]
                k_nrm[b, h, s:e] = p["norms"]
                if k_sgn is not None:
                    k_sgn[b, h, s:e] = p["signs"]
                if V is not None:
                    vq = O.quantize_values(V[b, h, s:e].astype(np.float64), value_bits)
                    v_q[b, h, s:e] = vq["q"]
                    v_p[b, h, s:e] = vq["params"]
    return dict(k_idx=k_idx, k_norms=k_nrm, k_signs=k_sgn, v_q=v_q, v_params=v_p,
                len=np.array(lengths, dtype=np.int64))


def upload_cache(cache, oc: dict) -> None:
    """Copy an oracle cache dict into a KVCache's device planes (row (b,h,t) layout)."""
    B, H, N = oc["k_idx"].shape[:3]
    cap = cache.capacity

    def put(dst, src):
        flat = src.reshape(B * H, N, -1)
        full = np.zeros((B * H, cap, flat.shape[2]), dtype=flat.dtype)
        full[:, :N] = flat
        t = torch.from_numpy(full.reshape(B * H * cap, -1).view(np.int16 if full.dtype == np.uint16 else full.dtype))
        dst.copy_(t.reshape(dst.shape))

    put(cache.k_idx, oc["k_idx"])
    put(cache.k_norms, oc["k_norms"])
    if oc.get("k_signs") is not None:
        put(cache.k_signs, oc["k_signs"])
    if oc.get("v_q") is not None:
        put(cache.v_q, oc["v_q"])
        put(cache.v_params, oc["v_params"])
    cache.set_lengths(oc["len"])


def download_pair(cache, b: int, h: int, n: int) -> dict:
    """The first n rows of (sequence b, KV head h) of a KVCache as an oracle cache dict with
    one sequence and one KV head (the reverse of upload_cache for one pair)."""
    rows = cache.rows(b, h)
    lay_shape = {"k_norms": None, "v_params": (4, 2)}
    out = {}
    for name in ("k_idx", "k_norms", "k_signs", "v_q", "v_params"):
        t = getattr(cache, name, None)
        if t is None:
            out[name] = None
            continue
        a = t[rows][:n].cpu().numpy()
        if a.dtype == np.int16:
            a = a.view(np.uint16)
        shape = lay_shape.get(name)
        a = a.reshape((n,) + shape) if shape else a.reshape(n, -1)
        out[name] = a[None, None]
    out["len"] = np.array([n], dtype=np.int64)
    return out
