"""Plain fp64 CPU oracle of TurboQuant KV-cache quantization and decode attention.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg
(and its reference arm) may import this module. The CUDA library never calls it and shares
no code, tables or constants with it: both sides are written from the pages separately and
meet only through the seeded inputs of workloads.py.

Everything is computed in fp64 with dense matrices, in the order the pages describe the
method. Where a floating-point value decides an integer code (a codebook index, a QJL sign,
an fp16 norm, a value code) the decision is taken in fp32, the precision of the pages' own
PyTorch code (torch's default dtype) and of the CUDA kernels; the fp64 value is rounded to
fp32 first.

Sources (page title, section):
  [tqlite]   "tqlite" README: directory layout (rotation.py = Hadamard x random signs,
             codebook.py = Lloyd-Max Gaussian codebook), "three quantization modes" table
             (mse / prod / grouped bit budgets), design notes (per-row L2 normalisation,
             per-layer seeds).
  [tutorial] "Implementing TurboQuant (part 5)" (difai.kr): algorithm overview (residual,
             QJL sign(S @ residual), estimator <q,k_hat> + sqrt(pi/2) (Sq)^T sign_bits).
  [packing]  TurboQuant bit-packing article (m.lqnn.cn): section 2 (2-bit a|b<<2|c<<4|d<<6),
             section 3 (4-bit a|b<<4; 3-bit indices stored as 4-bit), section 4 (8 signs per
             byte with weights 1..128; fp16 norms; 52 bytes per d=128 3-bit key).
  [validate] electron-rare/turboquant validate_paper.py: Theorem 1 (MSE bounds), Table 1
             (codebook MSE), Theorem 2 (unbiasedness), Theorem 3 (distortion), recall,
             rank correlation, needle and compression checks; value_bits / group_size 32.

Readings where the pages are silent are stated at each function.
Parity pins: every public function here is pinned by tests/test_oracle_*.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

MODES = ("mse", "prod", "grouped")

# --------------------------------------------------------------------------------------------
# Random numbers: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014; the reference C code splitmix64.c by S. Vigna).
# The pages draw with torch.manual_seed, which cannot be reproduced without torch; a
# published counter-based generator is used instead, implemented separately on each side.
# --------------------------------------------------------------------------------------------
_MASK64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15

# stream tags: which draws of a quantizer seed feed which table
TAG_ROT_SIGNS = 1      # d rotation signs of the full-width rotation
TAG_QJL_GAUSS = 2      # S_rot entries (two draws per entry)
TAG_OUT_SIGNS = 3      # 32 rotation signs of the outlier group (grouped mode)
TAG_NORM_SIGNS = 4     # 96 rotation signs of the normal group (grouped mode)


def splitmix64(seed: int, n: int) -> list[int]:
    """The first n outputs of SplitMix64 seeded with `seed`: state_k = seed + (k+1)*gamma
    (mod 2^64), output_k = mix(state_k) with the two xor-shift-multiply rounds of the paper."""
    out = []
    s = seed & _MASK64
    for _ in range(n):
        s = (s + _GAMMA) & _MASK64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def stream_seed(seed: int, tag: int) -> int:
    """Seed of the independent stream `tag` of a quantizer seed: seed xor (tag << 56)."""
    return (seed ^ (tag << 56)) & _MASK64


def random_signs(seed: int, tag: int, n: int) -> np.ndarray:
    """n Rademacher signs: +1 when bit 63 of the draw is 0, else -1."""
    return np.array([-1.0 if (z >> 63) else 1.0 for z in splitmix64(stream_seed(seed, tag), n)])


def gaussian_fp16_matrix(seed: int, rows: int, cols: int) -> np.ndarray:
    """The QJL projection S_rot (rows x cols, row-major draw order).

    Entry k uses draws 2k and 2k+1: u1 = ((a >> 11) + 1) * 2^-53 in (0, 1],
    u2 = (b >> 11) * 2^-53 in [0, 1), z = sqrt(-2 ln u1) * cos(2 pi u2) (Box & Muller 1958),
    then z is rounded to fp16 (RNE); that fp16 value *is* the matrix entry.
    libm's log/cos/sqrt are called through Python's math module."""
    draws = splitmix64(stream_seed(seed, TAG_QJL_GAUSS), 2 * rows * cols)
    z = np.empty(rows * cols)
    scale = 2.0 ** -53
    for k in range(rows * cols):
        u1 = ((draws[2 * k] >> 11) + 1) * scale
        u2 = (draws[2 * k + 1] >> 11) * scale
        z[k] = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
    return fp16_rn(z).reshape(rows, cols)


# --------------------------------------------------------------------------------------------
# fp16 / fp32 rounding
# --------------------------------------------------------------------------------------------
def fp16_rn(x) -> np.ndarray:
    """Round to the nearest fp16 value, ties to even (overflow to +-inf); returned as fp64."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def fp16_bits(x) -> np.ndarray:
    """IEEE binary16 bit patterns of fp16-exact values."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def fp16_from_bits(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def fp32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# --------------------------------------------------------------------------------------------
# Lloyd-Max codebook for a standard Gaussian coordinate ([tqlite] codebook.py;
# [validate] Table 1 / get_codebook). Reading: the codebook is the optimal scalar quantizer of
# N(0,1) with 2^bits levels (Max 1960, Lloyd 1982), found by the fixed-point iteration
# "centroid = conditional mean of its cell, threshold = midpoint of adjacent centroids".
# It is symmetric; the positive half is iterated and mirrored, so the middle threshold is 0.
# --------------------------------------------------------------------------------------------
def _phi(x: float) -> float:
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _upper_tail(x: float) -> float:
    return 0.5 * math.erfc(x / math.sqrt(2.0))


def lloyd_max_gaussian(bits: int, tol: float = 1e-14, max_iter: int = 100000):
    """(centroids, thresholds) of the N(0,1) Lloyd-Max quantizer with 2^bits levels,
    ascending; index 0 is the most negative centroid."""
    half = (1 << bits) // 2
    c = [(k + 0.5) * 3.0 / half for k in range(half)]
    for _ in range(max_iter):
        t = [0.0] + [0.5 * (c[k] + c[k + 1]) for k in range(half - 1)]
        new = []
        for k in range(half):
            a = t[k]
            if k + 1 < half:
                b = t[k + 1]
                new.append((_phi(a) - _phi(b)) / (_upper_tail(a) - _upper_tail(b)))
            else:
                new.append(_phi(a) / _upper_tail(a))
        delta = max(abs(x - y) for x, y in zip(new, c))
        c = new
        if delta < tol:
            break
    pos = np.array(c)
    cent = np.concatenate([-pos[::-1], pos])
    thr = 0.5 * (cent[:-1] + cent[1:])
    thr[len(thr) // 2] = 0.0
    return cent, thr


def gaussian_distortion(cent: np.ndarray, thr: np.ndarray) -> float:
    """E[(X - Q(X))^2] for X ~ N(0,1), integrated cell by cell in closed form:
    int_a^b (x - c)^2 phi(x) dx = M2 - 2 c M1 + c^2 M0 with M0 = P(a < X < b),
    M1 = phi(a) - phi(b), M2 = M0 + a phi(a) - b phi(b)."""
    edges = [-math.inf] + list(thr) + [math.inf]
    total = 0.0
    for k, ck in enumerate(cent):
        a, b = edges[k], edges[k + 1]
        pa = 0.0 if a == -math.inf else _phi(a)
        pb = 0.0 if b == math.inf else _phi(b)
        Pa = 1.0 if a == -math.inf else _upper_tail(a)
        Pb = 0.0 if b == math.inf else _upper_tail(b)
        mass = Pa - Pb                                   # P(a < X < b)
        m1 = pa - pb                                     # int_a^b x phi(x) dx
        aa = 0.0 if a == -math.inf else a * pa
        bb = 0.0 if b == math.inf else b * pb
        m2 = mass + aa - bb                              # int_a^b x^2 phi(x) dx
        total += m2 - 2.0 * ck * m1 + ck * ck * mass
    return total


# --------------------------------------------------------------------------------------------
# Rotation Pi = Hadamard x random signs ([tqlite] rotation.py; [tutorial] algorithm overview).
# Reading: Pi = (1/sqrt(d)) H_d diag(s) with H_d the Sylvester Hadamard matrix, so the
# signs are applied first and Pi is orthonormal.
# --------------------------------------------------------------------------------------------
def sylvester_hadamard(n: int) -> np.ndarray:
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation_matrix(signs: np.ndarray) -> np.ndarray:
    d = signs.shape[0]
    return sylvester_hadamard(d) @ np.diag(signs) / math.sqrt(d)


def block_rotation_matrix(signs: np.ndarray, block: int) -> np.ndarray:
    """Block-diagonal rotation: one (1/sqrt(block)) H_block per consecutive block of
    channels, after the sign flips."""
    n = signs.shape[0]
    hb = sylvester_hadamard(block) / math.sqrt(block)
    m = np.zeros((n, n))
    for s in range(0, n, block):
        m[s:s + block, s:s + block] = hb
    return m @ np.diag(signs)


# --------------------------------------------------------------------------------------------
# Bit packing ([packing] sections 2-4). Element j of a row lands in byte (j*w)//8 at bit
# offset (j*w) % 8, lowest bits first: 2-bit a|b<<2|c<<4|d<<6, 4-bit a|b<<4, 1-bit signs
# with weights 1,2,4,...,128. 3-bit indices are stored in 4-bit fields.
# --------------------------------------------------------------------------------------------
def storage_width(bits: int) -> int:
    return {1: 1, 2: 2, 3: 4, 4: 4}[bits]


def pack_bits(codes: np.ndarray, width: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    n, m = codes.shape
    if (m * width) % 8:
        raise ValueError("row does not fill whole bytes")
    if codes.min(initial=0) < 0 or codes.max(initial=0) >= (1 << width):
        raise ValueError("code out of range for width")
    per = 8 // width
    c = codes.reshape(n, m // per, per)
    out = np.zeros((n, m // per), dtype=np.int64)
    for f in range(per):
        out |= c[:, :, f] << (f * width)
    return out.astype(np.uint8)


def unpack_bits(packed: np.ndarray, width: int, m: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.int64)
    per = 8 // width
    fields = [(packed >> (f * width)) & ((1 << width) - 1) for f in range(per)]
    return np.stack(fields, axis=-1).reshape(packed.shape[0], -1)[:, :m]


# --------------------------------------------------------------------------------------------
# Quantizer definition
# --------------------------------------------------------------------------------------------
@dataclass
class Quantizer:
    """Tables of one TurboQuant key quantizer ([tqlite] factory.py build_quantizer(d, bits,
    mode, seed); [validate] TurboQuantMSE / TurboQuantProd(dim, bits, seed)).

    bits is the total bit count per coordinate: mse uses a bits-wide codebook; prod uses a
    (bits-1)-wide MSE codebook plus one QJL sign bit ([tutorial] "PolarQuant (b-1 bit) +
    QJL (1 bit)"; [packing] "3-bit key = 2-bit MSE index + 1-bit QJL sign"); grouped is the
    base width b of the normal channels, the outlier channels take b+1.
    """
    d: int
    bits: int
    mode: str
    seed: int
    outliers: np.ndarray | None = None
    # filled by build()
    cent: np.ndarray = field(default=None, repr=False)        # unit-vector centroids
    thr: np.ndarray = field(default=None, repr=False)
    signs: np.ndarray = field(default=None, repr=False)
    Pi: np.ndarray = field(default=None, repr=False)
    S_rot: np.ndarray = field(default=None, repr=False)
    S: np.ndarray = field(default=None, repr=False)
    # grouped mode
    normals: np.ndarray = field(default=None, repr=False)
    groups: list = field(default=None, repr=False)


@dataclass
class _Group:
    channels: np.ndarray
    bits: int
    cent: np.ndarray
    thr: np.ndarray
    signs: np.ndarray
    Pi: np.ndarray


def build_quantizer(d: int, bits: int, mode: str, seed: int, outliers=None) -> Quantizer:
    if mode not in MODES:
        raise ValueError(mode)
    if d < 2 or d & (d - 1):
        raise ValueError("d must be a power of two")
    q = Quantizer(d=d, bits=bits, mode=mode, seed=seed)
    if mode == "mse":
        if not 1 <= bits <= 4:
            raise ValueError("mse bits must be 1..4")
        mse_bits = bits
    elif mode == "prod":
        if not 2 <= bits <= 4:
            raise ValueError("prod bits must be 2..4")
        mse_bits = bits - 1
    else:
        if not 1 <= bits <= 3 or d != 128:
            raise ValueError("grouped needs d=128 and base bits 1..3")
        out = np.sort(np.asarray(outliers, dtype=np.int64))
        if out.shape != (32,) or len(np.unique(out)) != 32 or out.min() < 0 or out.max() >= d:
            raise ValueError("grouped needs 32 distinct outlier channels in [0, d)")
        normals = np.setdiff1d(np.arange(d), out)
        q.outliers, q.normals = out, normals
        q.groups = []
        for ch, b, tag, block in ((out, bits + 1, TAG_OUT_SIGNS, 32),
                                  (normals, bits, TAG_NORM_SIGNS, 32)):
            dg = ch.shape[0]
            c, t = lloyd_max_gaussian(b)
            s = random_signs(seed, tag, dg)
            q.groups.append(_Group(ch, b, c / math.sqrt(dg), t / math.sqrt(dg), s,
                                   block_rotation_matrix(s, block)))
        return q
    c, t = lloyd_max_gaussian(mse_bits)
    q.cent, q.thr = c / math.sqrt(d), t / math.sqrt(d)
    q.signs = random_signs(seed, TAG_ROT_SIGNS, d)
    q.Pi = rotation_matrix(q.signs)
    if mode == "prod":
        q.S_rot = gaussian_fp16_matrix(seed, d, d)
        q.S = q.S_rot @ q.Pi                      # S = S_rot Pi, an i.i.d. Gaussian matrix
    return q


def key_layout(q: Quantizer) -> dict:
    """Bytes per key in each plane ([packing] section 4 ledger)."""
    if q.mode == "grouped":
        o, n = q.groups
        idx = (o.channels.size * storage_width(o.bits) + n.channels.size *
               storage_width(n.bits)) // 8
        return dict(idx_bytes=idx, sign_bytes=0, n_norms=2, bytes_per_key=idx + 4)
    mse_bits = q.bits if q.mode == "mse" else q.bits - 1
    idx = q.d * storage_width(mse_bits) // 8
    sign = q.d // 8 if q.mode == "prod" else 0
    nn = 2 if q.mode == "prod" else 1
    return dict(idx_bytes=idx, sign_bytes=sign, n_norms=nn, bytes_per_key=idx + sign + 2 * nn)


# --------------------------------------------------------------------------------------------
# Key quantization
# --------------------------------------------------------------------------------------------
def _mse_encode(X: np.ndarray, Pi: np.ndarray, cent: np.ndarray, thr: np.ndarray):
    """TurboQuantMSE on the rows of X ([tqlite] mse.py; [validate] Theorem 1 test).

    n = ||x|| is stored as n16 = fp16(fp32(n)) ([tqlite] design notes: normalise each key,
    restore the norm after; [packing] section 4: fp16 norms). The unit vector is rotated,
    u = Pi x / n (u = 0 when n = 0), and each coordinate takes the index of its cell,
    idx_j = #{k : u_j > t_k}, compared in fp32 (ties go to the lower index).
    Reconstruction: x_hat = n16 Pi^T c[idx]."""
    dg = X.shape[1]
    n = np.sqrt(np.sum(X * X, axis=1))
    n16 = fp16_rn(fp32(n))
    Y = X @ Pi.T
    U = np.zeros_like(Y)
    nz = n > 0
    U[nz] = Y[nz] / n[nz, None]
    idx = np.sum(fp32(U)[:, :, None] > fp32(thr)[None, None, :], axis=2)
    margin = math.sqrt(dg) * np.min(np.abs(U[:, :, None] - thr[None, None, :]), axis=2)
    x_hat = n16[:, None] * (cent[idx] @ Pi)
    return idx, n16, x_hat, margin


def quantize_keys(q: Quantizer, X) -> dict:
    """Quantize key rows X (n x d, any float dtype, read exactly) into packed planes.

    Returns idx (n x idx_bytes uint8), signs (n x d/8 uint8, prod), norms (n x n_norms uint16
    fp16 bits) and the decision margins used by the parity tests:
      idx_margin  sqrt(d_g) |u_j - t_k| to the nearest threshold, per coordinate;
      sign_margin |(S r)_j| / ||r|| per coordinate (prod);
      n_exact     the fp64 norms (and residual norms) before fp16 rounding.
    """
    X = np.asarray(X, dtype=np.float64)
    n_rows = X.shape[0]
    out = {}
    if q.mode in ("mse", "prod"):
        idx, n16, x_hat, margin = _mse_encode(X, q.Pi, q.cent, q.thr)
        mse_bits = q.bits if q.mode == "mse" else q.bits - 1
        out["idx_codes"] = idx
        out["idx"] = pack_bits(idx, storage_width(mse_bits))
        out["idx_margin"] = margin
        norms = [n16]
        out["n_exact"] = [np.sqrt(np.sum(X * X, axis=1))]
        if q.mode == "prod":
            sigma, margin_s, r16, rn = prod_residual_signs(q, X, idx, n16)
            out["sigma"] = sigma
            out["signs"] = pack_bits(sigma, 1)
            out["sign_margin"] = margin_s
            norms.append(r16)
            out["n_exact"].append(rn)
        out["norms"] = fp16_bits(np.stack(norms, axis=1))
        return out
    # grouped ([tqlite] grouped.py, "three quantization modes" table: d_out*b_out + d_n*b_n)
    packed, norms, margins, codes, exact = [], [], [], [], []
    for g in q.groups:
        Xg = X[:, g.channels]
        idx, n16, _, margin = _mse_encode(Xg, g.Pi, g.cent, g.thr)
        packed.append(pack_bits(idx, storage_width(g.bits)))
        norms.append(n16)
        margins.append(margin)
        codes.append(idx)
        exact.append(np.sqrt(np.sum(Xg * Xg, axis=1)))
    out["idx"] = np.concatenate(packed, axis=1)
    out["idx_codes"] = np.concatenate(codes, axis=1)
    out["idx_margin"] = np.concatenate(margins, axis=1)
    out["norms"] = fp16_bits(np.stack(norms, axis=1))
    out["n_exact"] = exact
    assert out["idx"].shape == (n_rows, key_layout(q)["idx_bytes"])
    return out


def prod_residual_signs(q: Quantizer, X: np.ndarray, idx: np.ndarray, n16: np.ndarray):
    """QJL part of TurboQuantProd for given MSE codes and stored norms ([tutorial] algorithm
    overview: residual = k - decompress(codes); sign(S @ residual)).

    r = x - n16 Pi^T c[idx]; r16 = fp16(fp32(||r||)); sigma_j = [fp32((S r)_j) >= 0]
    (sign(0) counts as +1). Returns (sigma, |S r| / ||r||, r16, ||r||)."""
    X = np.asarray(X, dtype=np.float64)
    x_hat = np.asarray(n16, dtype=np.float64)[:, None] * (q.cent[idx] @ q.Pi)
    R = X - x_hat
    rn = np.sqrt(np.sum(R * R, axis=1))
    r16 = fp16_rn(fp32(rn))
    SR = R @ q.S.T
    sigma = (fp32(SR) >= 0).astype(np.int64)
    with np.errstate(divide="ignore", invalid="ignore"):
        margin = np.where(rn[:, None] > 0, np.abs(SR) / rn[:, None], np.inf)
    return sigma, margin, r16, rn


def reconstruct_keys(q: Quantizer, planes: dict) -> np.ndarray:
    """Dequantized keys in the original coordinates. For prod this is the MSE part plus
    the QJL residual reconstruction r16 sqrt(pi/2)/d S^T (2 sigma - 1), whose inner product
    with q equals the QJL term of the estimator."""
    lay = key_layout(q)
    norms = fp16_from_bits(planes["norms"])
    if q.mode == "grouped":
        n = planes["idx"].shape[0]
        x = np.zeros((n, q.d))
        off = 0
        for gi, g in enumerate(q.groups):
            w = storage_width(g.bits)
            nb = g.channels.size * w // 8
            idx = unpack_bits(planes["idx"][:, off:off + nb], w, g.channels.size)
            off += nb
            x[:, g.channels] = norms[:, gi:gi + 1] * (g.cent[idx] @ g.Pi)
        return x
    mse_bits = q.bits if q.mode == "mse" else q.bits - 1
    idx = unpack_bits(planes["idx"], storage_width(mse_bits), q.d)
    x = norms[:, :1] * (q.cent[idx] @ q.Pi)
    if q.mode == "prod":
        sig = unpack_bits(planes["signs"], 1, q.d)
        coef = norms[:, 1:2] * math.sqrt(math.pi / 2.0) / q.d
        x = x + coef * ((2.0 * sig - 1.0) @ q.S)
    assert lay["idx_bytes"] == planes["idx"].shape[1]
    return x


def key_scores(q: Quantizer, planes: dict, y: np.ndarray) -> np.ndarray:
    """Inner-product estimates <y, x_i> for every packed key i ([validate] attention_score;
    [tutorial] estimator).

    mse:     n16 <Pi y, c[idx]>
    prod:    n16 <Pi y, c[idx]> + r16 sqrt(pi/2)/d <S y, 2 sigma - 1>
             (reading: the page prints sqrt(pi/2) (Sq)^T sign_bits; the residual norm and the
             1/d make it unbiased, E[<s,y> sign<s,r>] = sqrt(2/pi) <y,r>/||r|| for s ~ N(0,I))
    grouped: the sum of the two sub-quantizers' mse estimates over their channels.
    """
    y = np.asarray(y, dtype=np.float64)
    norms = fp16_from_bits(planes["norms"])
    if q.mode == "grouped":
        off = 0
        s = np.zeros(planes["idx"].shape[0])
        for gi, g in enumerate(q.groups):
            w = storage_width(g.bits)
            nb = g.channels.size * w // 8
            idx = unpack_bits(planes["idx"][:, off:off + nb], w, g.channels.size)
            off += nb
            s += norms[:, gi] * (g.cent[idx] @ (g.Pi @ y[g.channels]))
        return s
    mse_bits = q.bits if q.mode == "mse" else q.bits - 1
    idx = unpack_bits(planes["idx"], storage_width(mse_bits), q.d)
    s = norms[:, 0] * (q.cent[idx] @ (q.Pi @ y))
    if q.mode == "prod":
        sig = unpack_bits(planes["signs"], 1, q.d)
        s = s + norms[:, 1] * math.sqrt(math.pi / 2.0) / q.d * ((2.0 * sig - 1.0) @ (q.S @ y))
    return s


# --------------------------------------------------------------------------------------------
# Values: asymmetric group quantization ([packing] section 2: turboquant/kv_cache.py packs 2-bit
# values four to a byte; section 3: 4-bit two to a byte; [validate] value_bits=2,
# value_group_size=32). Reading: per group of 32 contiguous channels, mn = min, mx = max,
# scale = (mx - mn)/(2^b - 1), stored as fp16 mn16 and s16; code = clamp(rint((v - mn16)/s16),
# 0, 2^b - 1), 0 when s16 = 0; every step of the code decision in fp32 IEEE arithmetic.
# --------------------------------------------------------------------------------------------
def quantize_values(V, bits: int, group: int = 32) -> dict:
    if bits not in (2, 4):
        raise ValueError("value bits must be 2 or 4")
    V = np.asarray(V, dtype=np.float64)
    n, d = V.shape
    if d % group:
        raise ValueError("d must be a multiple of the group size")
    Vg = fp32(V).reshape(n, d // group, group)             # inputs are fp32-exact
    mn = Vg.min(axis=2)
    mx = Vg.max(axis=2)
    levels = np.float32((1 << bits) - 1)
    scale32 = (mx - mn) / levels                            # fp32 subtract, fp32 divide
    s16 = fp32(fp16_rn(scale32))
    mn16 = fp32(fp16_rn(mn))
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (Vg - mn16[:, :, None]) / s16[:, :, None]      # fp32 subtract, fp32 divide
    codes = np.clip(np.rint(t), 0, (1 << bits) - 1)
    codes = np.where(s16[:, :, None] > 0, codes, 0).astype(np.int64).reshape(n, d)
    params = np.stack([fp16_bits(mn16), fp16_bits(s16)], axis=2)   # (n, groups, 2)
    return dict(q=pack_bits(codes, bits), params=params, codes=codes)


def dequantize_values(packed: np.ndarray, params: np.ndarray, bits: int, d: int,
                      group: int = 32) -> np.ndarray:
    """v_hat = mn16 + code * s16 (fp64, exact)."""
    codes = unpack_bits(packed, bits, d).astype(np.float64)
    mn = fp16_from_bits(params[..., 0])
    sc = fp16_from_bits(params[..., 1])
    g = np.repeat(np.arange(d // group), group)
    return mn[:, g] + codes * sc[:, g]


# --------------------------------------------------------------------------------------------
# Decode attention over the packed cache ([packing] section 5: fused decode kernels read the
# packed bytes; estimator as in key_scores). Reading: logits = s_i * sm_scale (default
# 1/sqrt(d)) over every cached token i < len[b]; no mask; out = softmax(logits) @ v_hat.
# --------------------------------------------------------------------------------------------
def default_head_map(n_q_heads: int, n_kv_heads: int) -> np.ndarray:
    g = n_q_heads // n_kv_heads
    return np.arange(n_q_heads) // g


def decode_attention(q: Quantizer, cache: dict, Q: np.ndarray, head_map=None,
                     sm_scale: float | None = None, value_bits: int = 2, group: int = 32,
                     want_scores: bool = False):
    """cache: dict of numpy planes indexed [b, h_kv, t, ...]:
         k_idx, k_signs (prod), k_norms, v_q, v_params (absent for score-only), len (B,).
       Q: (B, H_q, d). Returns (out (B, H_q, d) fp64 or None, scores list or None)."""
    Q = np.asarray(Q, dtype=np.float64)
    B, Hq, d = Q.shape
    Hkv = cache["k_idx"].shape[1]
    if head_map is None:
        head_map = default_head_map(Hq, Hkv)
    if sm_scale is None or sm_scale == 0.0:
        sm_scale = 1.0 / math.sqrt(d)
    has_v = cache.get("v_q") is not None
    out = np.zeros((B, Hq, d)) if has_v else None
    scores = [[None] * Hq for _ in range(B)] if want_scores else None
    for b in range(B):
        L = int(cache["len"][b])
        for kv in range(Hkv):
            heads = [h for h in range(Hq) if head_map[h] == kv]
            if not heads or L == 0:
                continue
            planes = dict(idx=cache["k_idx"][b, kv, :L], norms=cache["k_norms"][b, kv, :L])
            if q.mode == "prod":
                planes["signs"] = cache["k_signs"][b, kv, :L]
            v_hat = (dequantize_values(cache["v_q"][b, kv, :L], cache["v_params"][b, kv, :L],
                                       value_bits, d, group) if has_v else None)
            for h in heads:
                s = key_scores(q, planes, Q[b, h])
                if want_scores:
                    scores[b][h] = s
                if has_v:
                    z = s * sm_scale
                    p = np.exp(z - z.max())
                    out[b, h] = (p / p.sum()) @ v_hat
    return out, scores


# --------------------------------------------------------------------------------------------
# Context-split decode. Softmax over the union of disjoint token sets is the log-sum-exp merge
# of per-set results (an identity of the softmax, nothing the pages add): a set's record is
# m = max_i x_i, l = sum_i 2^(x_i - m), o = sum_i 2^(x_i - m) v_hat_i with the base-2 logits
# x_i = sm_scale log2(e) s_i of decode_attention; an empty set gives (-inf, 0, 0).
# --------------------------------------------------------------------------------------------
def decode_partial(q: Quantizer, cache: dict, Q: np.ndarray, head_map=None,
                   sm_scale: float | None = None, value_bits: int = 2, group: int = 32):
    """Records (m (B, H_q), l (B, H_q), o (B, H_q, d)) of this cache's tokens."""
    Q = np.asarray(Q, dtype=np.float64)
    B, Hq, d = Q.shape
    Hkv = cache["k_idx"].shape[1]
    if head_map is None:
        head_map = default_head_map(Hq, Hkv)
    if sm_scale is None or sm_scale == 0.0:
        sm_scale = 1.0 / math.sqrt(d)
    m = np.full((B, Hq), -np.inf)
    l = np.zeros((B, Hq))
    o = np.zeros((B, Hq, d))
    for b in range(B):
        L = int(cache["len"][b])
        if L == 0:
            continue
        for h in range(Hq):
            kv = head_map[h]
            planes = dict(idx=cache["k_idx"][b, kv, :L], norms=cache["k_norms"][b, kv, :L])
            if q.mode == "prod":
                planes["signs"] = cache["k_signs"][b, kv, :L]
            v_hat = dequantize_values(cache["v_q"][b, kv, :L], cache["v_params"][b, kv, :L],
                                      value_bits, d, group)
            x = key_scores(q, planes, Q[b, h]) * (sm_scale / math.log(2.0))
            m[b, h] = x.max()
            w = np.exp2(x - m[b, h])
            l[b, h] = w.sum()
            o[b, h] = w @ v_hat
    return m, l, o


def merge_partials(ms, ls, os) -> np.ndarray:
    """LSE merge of records of disjoint token sets (lists over the sets): sum_r 2^(m_r - M) o_r
    / sum_r 2^(m_r - M) l_r with M = max_r m_r; zeros where every set is empty."""
    M = np.max(np.stack(ms), axis=0)
    Mf = np.where(np.isfinite(M), M, 0.0)
    num = np.zeros(os[0].shape)
    den = np.zeros(ls[0].shape)
    for m, l, o in zip(ms, ls, os):
        w = np.where(np.isfinite(m), np.exp2(np.where(np.isfinite(m), m, Mf) - Mf), 0.0)
        num += w[..., None] * o
        den += w * l
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)


def bf16_rn(x) -> np.ndarray:
    """Round fp64 values to bf16 (RNE) and return them as fp64 (for the bf16 output check)."""
    f = fp32(x)
    u = f.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    r = ((u + rounding) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)
