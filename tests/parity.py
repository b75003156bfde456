"""Acceptance rules for CUDA-vs-oracle parity.

Packed index and sign bits must equal the oracle's, except at coordinates whose decision
value lies within 1e-4 of a threshold (indices; sqrt(d_g) |u_j - t_k|) or of zero (signs;
|(S r)_j| / ||r||). Such exempt mismatches are counted and must stay under 1e-4 of all
coordinates. An exempt index flip may only move to the neighbouring code. fp16 norms may
differ by one ulp only where the exact norm sits at an fp16 rounding midpoint (to fp32
noise). Where a row took an exempt alternative (a neighbouring code or norm), its QJL
signs are checked against the oracle's signs for that alternative: the alternative is one
of the two values the oracle itself accepts, so it is a valid result, not a new input.
Scores: |ds| <= 1e-3 max(|s_ref|, ||q|| n16 / sqrt(d)). Attention: fp32 output within
2e-3 max-abs; bf16 output within 2e-3 of the oracle's bf16-rounded value, or within one bf16
ulp of it where that ulp is larger (|out| >= 0.25: a half-ulp of bf16 there already exceeds
what an fp32 result can be held to).
"""
from __future__ import annotations

import math

import numpy as np

import oracle as O

MARGIN = 1e-4
MAX_EXEMPT_FRAC = 1e-4


def unpack_codes(qo, idx_bytes: np.ndarray) -> np.ndarray:
    if qo.mode == "grouped":
        out, off = [], 0
        for g in qo.groups:
            w = O.storage_width(g.bits)
            nb = g.channels.size * w // 8
            out.append(O.unpack_bits(idx_bytes[:, off:off + nb], w, g.channels.size))
            off += nb
        return np.concatenate(out, axis=1)
    mb = qo.bits if qo.mode == "mse" else qo.bits - 1
    return O.unpack_bits(idx_bytes, O.storage_width(mb), qo.d)


def _check_norm_pair(gpu_bits, ref_bits, exact, what):
    """gpu/ref fp16 bit patterns (1-D), exact fp64 norms. Returns mismatch mask."""
    g = gpu_bits.astype(np.int64)
    r = ref_bits.astype(np.int64)
    mism = g != r
    if mism.any():
        assert np.all(np.abs(g[mism] - r[mism]) == 1), f"{what}: norm off by more than one ulp"
        a = O.fp16_from_bits(gpu_bits[mism].astype(np.uint16))
        b = O.fp16_from_bits(ref_bits[mism].astype(np.uint16))
        mid = 0.5 * (a + b)
        ex = exact[mism]
        assert np.all(np.abs(ex - mid) <= 2e-6 * np.maximum(ex, 1e-30)), \
            f"{what}: norm differs away from an fp16 rounding midpoint"
    return mism


def check_key_parity(qo, X: np.ndarray, gpu: dict) -> dict:
    """X: (n, d) fp64 inputs (exact values of what the GPU read). gpu: numpy planes
    idx (uint8), norms (uint16 bits), signs (uint8, prod). Asserts the acceptance rules and
    returns the exempt counts."""
    ref = O.quantize_keys(qo, X)
    n, d = X.shape
    stats = dict(rows=n, coords=n * d)
    cg = unpack_codes(qo, gpu["idx"])
    cr = ref["idx_codes"]
    mism = cg != cr
    if mism.any():
        assert np.all(ref["idx_margin"][mism] < MARGIN), \
            f"index mismatch away from a threshold: margins {np.sort(ref['idx_margin'][mism])[-5:]}"
        assert np.all(np.abs(cg[mism] - cr[mism]) == 1)
    stats["idx_exempt"] = int(mism.sum())
    clean = ~mism.any(axis=1)
    assert np.array_equal(gpu["idx"][clean], ref["idx"][clean]), "packed index bytes differ"

    gn = gpu["norms"].astype(np.uint16)
    rn = ref["norms"]
    norm_mism = np.zeros(n, dtype=bool)
    for k in range(rn.shape[1]):
        if qo.mode == "prod" and k == 1:
            continue  # residual norm checked below, under the row's chosen alternative
        m = _check_norm_pair(gn[:, k], rn[:, k], ref["n_exact"][k], f"norm[{k}]")
        norm_mism |= m
    stats["norm_exempt"] = int(norm_mism.sum())

    if qo.mode == "prod":
        sg = O.unpack_bits(gpu["signs"], 1, d)
        sr = ref["sigma"].copy()
        smargin = ref["sign_margin"].copy()
        r16_ref = rn[:, 1].copy()
        r_exact = ref["n_exact"][1].copy()
        alt = ~clean | norm_mism
        if alt.any():
            # the oracle's result for the neighbouring alternative the row took
            rows = np.nonzero(alt)[0]
            n16_alt = O.fp16_from_bits(gn[rows, 0])
            sig_a, mar_a, r16_a, rn_a = O.prod_residual_signs(qo, X[rows], cg[rows], n16_alt)
            sr[rows] = sig_a
            smargin[rows] = mar_a
            r16_ref[rows] = O.fp16_bits(r16_a)
            r_exact[rows] = rn_a
        _check_norm_pair(gn[:, 1], r16_ref, r_exact, "residual norm")
        sm = sg != sr
        if sm.any():
            assert np.all(smargin[sm] < MARGIN), \
                f"QJL sign mismatch away from zero: margins {np.sort(smargin[sm])[-5:]}"
        stats["sign_exempt"] = int(sm.sum())
        assert stats["sign_exempt"] < MAX_EXEMPT_FRAC * n * d + 1
        clean_s = ~sm.any(axis=1)
        assert np.array_equal(gpu["signs"][clean_s], O.pack_bits(sr[clean_s], 1))
    assert stats["idx_exempt"] < MAX_EXEMPT_FRAC * n * d + 1, stats
    return stats


def check_scores(gpu: np.ndarray, ref: np.ndarray, qnorm: float, n16: np.ndarray, d: int = 128):
    floor = qnorm * n16 / math.sqrt(d)
    err = np.abs(gpu - ref)
    tol = 1e-3 * np.maximum(np.abs(ref), floor)
    assert np.all(err <= tol), f"score error {np.max(err / np.maximum(tol, 1e-30))} x tolerance"
    return float(np.max(err / np.maximum(np.abs(ref), floor)))


def check_attention(gpu: np.ndarray, ref: np.ndarray, bf16: bool):
    if bf16:
        rb = O.bf16_rn(ref)
        _, e = np.frexp(rb)
        ulp = np.where(rb != 0, np.ldexp(1.0, e - 8), 2.0 ** -133)   # 8 significant bits
        err = np.abs(gpu - rb)
        tol = np.maximum(ulp, 2e-3)
        assert np.all(err <= tol), f"bf16 output error {np.max(err / tol)} x tolerance"
        return float(np.max(np.abs(gpu - ref)))
    err = float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0
    assert err <= 2e-3, f"attention max-abs error {err}"
    return err
