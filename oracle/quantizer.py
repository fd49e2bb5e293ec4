"""TurboQuant encode and dequant (oracle side; test infrastructure).

TurboQuant_mse ("TurboQuant của Google: nén KV cache 6 lần", sections "Trick
đầu tiên" and "Lloyd-Max quantizer"; "内存厂商的噩梦来了", section 4.1):
keep the norm of x (HN thread on TurboQuant: the radius is one value per
vector and can be kept as is), rotate x/||x||, replace each rotated coordinate
by the index of its nearest Lloyd-Max centroid and store only the indices,
with no per-block scale or zero-point.

TurboQuant_prod (same omelet.tech page, section "Vấn đề của inner product:
bias không phải MSE", the (b-1)-bit + 1-bit recipe; "内存厂商的噩梦来了",
sections 4.2-4.3): a (b-1)-bit MSE code, the residual r, and one QJL sign bit
per projected coordinate, sign(S r), plus ||r||.

Canonical fp32 arithmetic (the reading every encoder reproduces bit for bit;
NumPy float32 element-wise ops round to nearest even and never fuse):
  x_f  = fp32(x)                      (bf16 / fp16 widen exactly)
  s    = fold-halves sum of fl(x_i^2): for h = d/2, d/4, ..., 1,
         a_i <- fl(a_i + a_{i+h}) for i < h;    n = sqrt_rn(s)
         (a d that is not a power of two is zero-padded to one first)
  y    = FWHT_f32(sigma * x_f)        (oracle.rotation.fwht_f32)
  w    = fl(n * fp32(sqrt(d)));  inv = fl(1/w) if w > 0 else 0
  u_i  = fl(y_i * inv)                (= (Pi x / ||x||)_i up to rounding)
  idx_i = #{j : u_i > t_j}            (a tie goes to the lower index)
  prod: r_i = fl(u_i - c[idx_i]); gamma = sqrt_rn(fold-halves sum fl(r_i^2));
        z = S r in float64; bit_k = [z_k >= 0]; with b = 1 there is no MSE
        code and r = u.
Readings (the pages are silent): the residual is taken in the rotated basis
(the norm and the law of S Pi are unchanged, so the estimator is the same in
distribution); sign(0) = +1; n = 0 gives inv = 0.

Dense rotation (the Haar-random Pi of oracle.rotation.haar_matrix, stored in
fp32): the norm is the same canonical fp32 value, and the rotation is the plain
definition evaluated in float64, u = (Pi_f32 x_f) / n (0 when n = 0); indices
and residual follow from that u.  Any d that is a multiple of 8 works.

Layout: codes are an LSB-first bitstream per vector, index i's bit k at
stream bit i*b_m + k (byte p >> 3, bit p & 7); the QJL sketch puts bit k at
byte k >> 3, bit k & 7; norms and residual norms are separate fp32 arrays.
"""

import math
from dataclasses import dataclass, field

import numpy as np

from . import codebook as _cb
from . import prng as _prng
from . import rotation as _rot

SQRT_HALF_PI = math.sqrt(math.pi / 2.0)


@dataclass
class Quantizer:
    """All parameters of one TurboQuant quantizer, built by the oracle itself."""
    d: int
    bits: int
    variant: str = "mse"          # "mse" or "prod"
    seed_rot: int = 0
    seed_qjl: int = 1
    dist: str = "gauss"
    rotation: str = "hadamard"    # "hadamard" (sign flips + FWHT) or "dense" (Haar)
    centroids: np.ndarray = field(init=False)
    thresholds: np.ndarray = field(init=False)
    signs: np.ndarray = field(init=False)
    S: np.ndarray = field(init=False)
    Pi: np.ndarray = field(init=False)

    def __post_init__(self):
        assert self.variant in ("mse", "prod")
        assert self.rotation in ("hadamard", "dense")
        if self.dense:
            assert self.d >= 8 and self.d % 8 == 0
        else:
            assert self.d >= 2 and self.d & (self.d - 1) == 0
        self.centroids, self.thresholds, _, _ = _cb.codebook(self.d, self.bm, self.dist)
        self.signs = _prng.signs(self.seed_rot, self.d)
        self.Pi = _rot.haar_matrix(self.seed_rot, self.d).astype(np.float32) if self.dense else None
        self.S = _prng.gaussian_matrix(self.seed_qjl, self.d) if self.prod else None

    @property
    def dense(self) -> bool:
        return self.rotation == "dense"

    @property
    def prod(self) -> bool:
        return self.variant == "prod"

    @property
    def bm(self) -> int:
        """MSE bits per coordinate: b for mse, b - 1 for prod."""
        return self.bits - 1 if self.prod else self.bits

    @property
    def code_bytes(self) -> int:
        return (self.d * self.bm + 7) // 8

    @property
    def qjl_bytes(self) -> int:
        return self.d // 8 if self.prod else 0


def fold_halves_sum_f32(a: np.ndarray) -> np.ndarray:
    """Row sums of [n, d] float32 in the canonical fold-halves order; a d that
    is not a power of two (the dense rotation's) is first padded with zeros
    to the next power of two, which changes no partial sum."""
    assert a.dtype == np.float32
    d = a.shape[1]
    p2 = 1 << max(0, (d - 1).bit_length())
    if p2 != d:
        a = np.concatenate([a, np.zeros((a.shape[0], p2 - d), np.float32)], axis=1)
        d = p2
    h = d // 2
    while h >= 1:
        a = a[:, :h] + a[:, h:2 * h]
        h //= 2
    return a[:, 0]


def pack_bits(idx: np.ndarray, width: int) -> np.ndarray:
    """LSB-first bitstream of the ``width``-bit unsigned fields of each row."""
    n, d = idx.shape
    if width == 0:
        return np.zeros((n, 0), np.uint8)
    bits = ((idx[:, :, None].astype(np.uint32) >> np.arange(width, dtype=np.uint32)) & 1)
    return np.packbits(bits.reshape(n, d * width).astype(np.uint8), axis=1, bitorder="little")


def unpack_bits(packed: np.ndarray, d: int, width: int) -> np.ndarray:
    """Inverse of ``pack_bits``: [n, bytes] uint8 -> [n, d] int64 fields."""
    n = packed.shape[0]
    if width == 0:
        return np.zeros((n, d), np.int64)
    bits = np.unpackbits(packed, axis=1, bitorder="little")[:, : d * width].reshape(n, d, width)
    out = np.zeros((n, d), np.int64)
    for k in range(width):
        out |= bits[:, :, k].astype(np.int64) << k
    return out


def encode(qz: Quantizer, x: np.ndarray, chunk: int = 8192, aux: bool = True) -> dict:
    """Encode rows of ``x`` ([n, d], any float dtype holding the input values).

    Returns dict(codes [n, code_bytes] u8, norms [n] f32, and for prod
    qjl [n, d/8] u8, rnorms [n] f32); with ``aux`` also u [n, d] (f32; f64
    for the dense rotation) and, for prod, z [n, d] f64 (the projections,
    kept so tests can measure the distance to the sign boundary).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    assert d == qz.d
    out = {"codes": [], "norms": [], "u": []}
    if qz.prod:
        out.update(qjl=[], rnorms=[], z=[])
    sqrt_d = np.float32(math.sqrt(d))
    sig = qz.signs.astype(np.float32)
    for s in range(0, n, chunk):
        xb = x[s:s + chunk]
        nrm = np.sqrt(fold_halves_sum_f32(xb * xb))
        if qz.dense:
            y = xb.astype(np.float64) @ qz.Pi.astype(np.float64).T
            n64 = nrm.astype(np.float64)[:, None]
            u = np.zeros_like(y)
            np.divide(y, n64, out=u, where=n64 > 0)
        else:
            y = _rot.fwht_f32(xb * sig[None, :])
            w = nrm * sqrt_d
            inv = np.zeros_like(w)
            np.divide(np.float32(1.0), w, out=inv, where=w > 0)
            u = y * inv[:, None]
        if qz.bm > 0:
            idx = (u[:, :, None] > qz.thresholds[None, None, :]).sum(axis=2)
        else:
            idx = np.zeros(u.shape, np.int64)
        out["codes"].append(pack_bits(idx, qz.bm))
        out["norms"].append(nrm)
        if aux:
            out["u"].append(u)
        if qz.prod:
            r = u - qz.centroids[idx] if qz.bm > 0 else u.copy()
            if qz.dense:
                gam = np.sqrt(np.sum(r * r, axis=1)).astype(np.float32)
            else:
                gam = np.sqrt(fold_halves_sum_f32(r * r))
            z = r.astype(np.float64) @ qz.S.astype(np.float64).T
            out["qjl"].append(pack_bits((z >= 0).astype(np.int64), 1))
            out["rnorms"].append(gam)
            if aux:
                out["z"].append(z)
    return {k: np.concatenate(v, axis=0) for k, v in out.items() if v}


def rotated_estimate(qz: Quantizer, enc: dict) -> np.ndarray:
    """Reconstruction of the rotated unit vector u in float64:
    c[idx] (+ prod: gamma * sqrt(pi/2)/d * S^T (2 bit - 1))."""
    n = enc["norms"].shape[0]
    idx = unpack_bits(enc["codes"], qz.d, qz.bm)
    c = qz.centroids.astype(np.float64)
    uh = c[idx] if qz.bm > 0 else np.zeros((n, qz.d))
    if qz.prod:
        sg = 2.0 * unpack_bits(enc["qjl"], qz.d, 1) - 1.0
        corr = sg @ qz.S.astype(np.float64)          # rows: S^T sign
        uh = uh + (enc["rnorms"].astype(np.float64) * SQRT_HALF_PI / qz.d)[:, None] * corr
    return uh


def dequant(qz: Quantizer, enc: dict) -> np.ndarray:
    """x_hat = ||x|| * Pi^T u_hat, float64 ("内存厂商的噩梦来了", section 4
    pseudocode, dequant)."""
    uh = rotated_estimate(qz, enc)
    if qz.dense:
        back = uh @ qz.Pi.astype(np.float64)          # Pi^T u_hat, row by row
    else:
        back = _rot.unrotate_f64(uh, qz.signs)
    return enc["norms"].astype(np.float64)[:, None] * back
